"""Shared test helpers: device upload of seeded numpy inputs and error norms."""
import numpy as np


def rel_fro(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    den = np.linalg.norm(want)
    num = np.linalg.norm(got - want)
    if den == 0.0:
        return float(num)
    return float(num / den)


def to_dev(a, dtype: str, device="cuda"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.to(device)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def f64(a):
    return None if a is None else np.asarray(a, np.float64)


def oracle_cfg(O, L):
    return O.LayerConfig(L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn, L.rms_eps,
                         L.rope_theta)

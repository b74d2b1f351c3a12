"""ctypes binding of libsbp (the C ABI in include/sbp.h).

Argument marshalling only: tensors are passed as raw device pointers, the workspace is a
torch uint8 tensor, the stream is torch's current CUDA stream.  Every step of the streamed
backward runs inside libsbp's kernels; there is no CPU or PyTorch fallback -- if the library
is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsbp.so")

SBP_F32, SBP_BF16 = 0, 1
STATUS = {0: "SBP_OK", 1: "SBP_ERR_INVALID_ARG", 2: "SBP_ERR_UNSUPPORTED", 3: "SBP_ERR_WORKSPACE",
          4: "SBP_ERR_CUDA", 5: "SBP_ERR_DEVICE_TIMEOUT", 6: "SBP_ERR_BAD_TARGET"}

EXPORTS = [
    "sbp_last_error", "sbp_version", "sbp_chunk_bounds", "sbp_get_device_status",
    "sbp_lmhead_ce_workspace_size", "sbp_lmhead_ce_backward_stream",
    "sbp_decoder_layer_workspace_size", "sbp_decoder_layer_backward_stream",
    "sbp_decoder_layer_forward_stream", "sbp_rmsnorm_forward",
    "sbp_rmsnorm_backward_workspace_size", "sbp_rmsnorm_backward", "sbp_embedding_forward",
    "sbp_embedding_backward_workspace_size", "sbp_embedding_backward", "sbp_debug_gemm_bf16",
    "sbp_launch_count", "sbp_profile_begin", "sbp_profile_end", "sbp_lmhead_ce_backward_noalloc",
    "sbp_debug_attn_fwd_bf16", "sbp_debug_attn_bwd_bf16", "sbp_lmhead_ce_forward_stream",
    "sbp_dpo_workspace_size", "sbp_dpo_token_weights", "sbp_lmhead_ce_workspace_size_host",
    "sbp_lmhead_ce_backward_stream_host", "sbp_decoder_layer_backward_stream_reverse",
    "sbp_debug_gemm_stall_bf16",
]

WEIGHT_FIELDS = ("ln1_g", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "ln2_g", "w_gate", "w_up",
                 "w_down")


class SbpError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Profile(C.Structure):
    _fields_ = [("launches", C.c_longlong * 4), ("ms", C.c_double * 4),
                ("busy_ms", C.c_double * 4)]


class LayerCfg(C.Structure):
    _fields_ = [("batch", C.c_int64), ("seq_len", C.c_int64), ("d_model", C.c_int64),
                ("n_heads", C.c_int64), ("n_kv_heads", C.c_int64), ("head_dim", C.c_int64),
                ("ffn", C.c_int64), ("rms_eps", C.c_float), ("rope_theta", C.c_double),
                ("dtype", C.c_int), ("num_chunks", C.c_int)]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


class LayerGrads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


_lib = None


def load(path: Optional[str] = None):
    """Open libsbp.so (built by build.py).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libsbp.so not found at {p}; run "
                           "`python -m memory_efficient_exact_chunk_b200.build`")
    lib = C.CDLL(p)
    vp, i64, sz = C.c_void_p, C.c_int64, C.c_size_t
    lib.sbp_last_error.restype = C.c_char_p
    lib.sbp_version.restype = C.c_char_p
    lib.sbp_chunk_bounds.argtypes = [i64, C.c_int, C.POINTER(C.c_int64)]
    lib.sbp_get_device_status.argtypes = [vp, vp]
    lib.sbp_lmhead_ce_workspace_size.restype = sz
    lib.sbp_lmhead_ce_workspace_size.argtypes = [i64, i64, i64, C.c_int, C.c_int]
    lib.sbp_lmhead_ce_backward_stream.argtypes = [i64, i64, i64, C.c_int, C.c_int] + [vp] * 7 + \
        [vp, sz, vp]
    lib.sbp_lmhead_ce_workspace_size_host.restype = sz
    lib.sbp_lmhead_ce_workspace_size_host.argtypes = [i64, i64, i64, C.c_int, C.c_int]
    lib.sbp_lmhead_ce_backward_stream_host.argtypes = [i64, i64, i64, C.c_int, C.c_int] + \
        [vp] * 7 + [vp, sz, vp]
    lib.sbp_lmhead_ce_forward_stream.argtypes = [i64, i64, i64, C.c_int, C.c_int] + [vp] * 6 + \
        [vp, sz, vp]
    lib.sbp_dpo_workspace_size.restype = sz
    lib.sbp_dpo_workspace_size.argtypes = [i64]
    lib.sbp_dpo_token_weights.argtypes = [i64, i64, vp, vp, vp, C.c_float, vp, vp, vp, vp, sz, vp]
    lib.sbp_decoder_layer_workspace_size.restype = sz
    lib.sbp_decoder_layer_workspace_size.argtypes = [C.POINTER(LayerCfg)]
    lib.sbp_decoder_layer_backward_stream.argtypes = [C.POINTER(LayerCfg),
                                                      C.POINTER(LayerWeights), vp, vp, vp,
                                                      C.POINTER(LayerGrads), vp, sz, vp]
    lib.sbp_decoder_layer_backward_stream_reverse.argtypes = \
        lib.sbp_decoder_layer_backward_stream.argtypes
    lib.sbp_decoder_layer_forward_stream.argtypes = [C.POINTER(LayerCfg),
                                                     C.POINTER(LayerWeights), vp, vp, vp, sz, vp]
    lib.sbp_rmsnorm_forward.argtypes = [i64, i64, C.c_int, C.c_float, vp, vp, vp, vp, vp]
    lib.sbp_rmsnorm_backward_workspace_size.restype = sz
    lib.sbp_rmsnorm_backward_workspace_size.argtypes = [i64, i64]
    lib.sbp_rmsnorm_backward.argtypes = [i64, i64, C.c_int, vp, vp, vp, vp, vp, C.c_int, vp, vp,
                                         sz, vp]
    lib.sbp_embedding_forward.argtypes = [i64, i64, i64, C.c_int, vp, vp, vp, vp]
    lib.sbp_embedding_backward_workspace_size.restype = sz
    lib.sbp_embedding_backward_workspace_size.argtypes = [i64, i64]
    lib.sbp_embedding_backward.argtypes = [i64, i64, i64, vp, vp, vp, vp, sz, vp]
    lib.sbp_debug_gemm_bf16.argtypes = [i64, i64, i64, vp, C.c_int, i64, vp, C.c_int, i64, vp, i64,
                                         C.c_int, C.c_int, i64, vp, vp]
    lib.sbp_lmhead_ce_backward_noalloc.argtypes = [i64, i64, i64, C.c_int, C.c_int] + [vp] * 7 + \
        [vp]
    lib.sbp_debug_gemm_stall_bf16.argtypes = [i64, i64, i64, vp, vp, vp, i64, vp, vp]
    lib.sbp_debug_attn_fwd_bf16.argtypes = [i64] * 7 + [vp] * 5 + [C.c_int, vp, vp]
    lib.sbp_debug_attn_bwd_bf16.argtypes = [i64] * 7 + [vp] * 9 + [C.c_int, vp, vp]
    lib.sbp_launch_count.restype = C.c_longlong
    lib.sbp_profile_end.argtypes = [C.POINTER(Profile)]
    _lib = lib
    return lib


def _check(code: int):
    if code != 0:
        raise SbpError(code, load().sbp_last_error().decode())


def chunk_bounds(seq_len: int, num_chunks: int):
    arr = (C.c_int64 * (num_chunks + 1))()
    _check(load().sbp_chunk_bounds(seq_len, num_chunks, arr))
    return [(arr[i], arr[i + 1]) for i in range(num_chunks)]


# ----------------------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return SBP_BF16
    if t.dtype == torch.float32:
        return SBP_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device="cuda"):
    """A 256-byte aligned device buffer of at least nbytes (torch allocations are aligned)."""
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def device_status(ws, stream=None):
    _check(load().sbp_get_device_status(_ptr(ws), _stream(stream)))


# ----------------------------------------------------------------------------- LM head
def lmhead_ce_workspace_size(n_tokens, hidden, vocab, num_chunks, dtype_code):
    return load().sbp_lmhead_ce_workspace_size(n_tokens, hidden, vocab, num_chunks, dtype_code)


def lmhead_ce_backward(hidden_states, weight, targets, loss_weights, num_chunks, loss_out,
                       d_hidden, d_weight, ws=None, stream=None):
    """loss_out[0] = sum_t w_t CE_t; d_hidden overwritten; d_weight += (all fp32)."""
    N, d = hidden_states.shape
    V = weight.shape[0]
    dt = _dtype_code(hidden_states)
    need = lmhead_ce_workspace_size(N, d, V, num_chunks, dt)
    if ws is None:
        ws = workspace(need, hidden_states.device)
    _check(load().sbp_lmhead_ce_backward_stream(
        N, d, V, num_chunks, dt, _ptr(hidden_states), _ptr(weight), _ptr(targets),
        _ptr(loss_weights), _ptr(loss_out), _ptr(d_hidden), _ptr(d_weight), _ptr(ws),
        ws.numel(), _stream(stream)))
    return ws


def lmhead_ce_backward_host(hidden_states_host, weight, targets_host, loss_weights_host,
                            num_chunks, loss_out, d_hidden, d_weight, ws=None, stream=None):
    """sbp_lmhead_ce_backward_stream_host: hidden states, targets and loss weights in (pinned)
    host memory, staged chunk by chunk by the library; everything else on the device."""
    N, d = hidden_states_host.shape
    V = weight.shape[0]
    dt = _dtype_code(hidden_states_host)
    if ws is None:
        ws = workspace(int(load().sbp_lmhead_ce_workspace_size_host(N, d, V, num_chunks, dt)),
                       weight.device)
    _check(load().sbp_lmhead_ce_backward_stream_host(
        N, d, V, num_chunks, dt, _ptr(hidden_states_host), _ptr(weight), _ptr(targets_host),
        _ptr(loss_weights_host), _ptr(loss_out), _ptr(d_hidden), _ptr(d_weight), _ptr(ws),
        ws.numel(), _stream(stream)))
    return ws


def lmhead_ce_workspace_size_host(N, d, V, D, dt) -> int:
    return int(load().sbp_lmhead_ce_workspace_size_host(N, d, V, D, dt))


def lmhead_ce_forward(hidden_states, weight, targets, loss_weights, num_chunks, token_ce,
                      loss_out=None, ws=None, stream=None):
    """token_ce[t] = CE_t where loss_weights[t] != 0, else 0 (include/sbp_dpo.h); loss_out[0]
    (optional) = sum_t w_t CE_t."""
    N, d = hidden_states.shape
    V = weight.shape[0]
    dt = _dtype_code(hidden_states)
    need = lmhead_ce_workspace_size(N, d, V, num_chunks, dt)
    if ws is None:
        ws = workspace(need, hidden_states.device)
    _check(load().sbp_lmhead_ce_forward_stream(
        N, d, V, num_chunks, dt, _ptr(hidden_states), _ptr(weight), _ptr(targets),
        _ptr(loss_weights), _ptr(token_ce), _ptr(loss_out) if loss_out is not None else None,
        _ptr(ws), ws.numel(), _stream(stream)))
    return ws


def dpo_workspace_size(n_pairs: int) -> int:
    return int(load().sbp_dpo_workspace_size(n_pairs))


def dpo_token_weights(n_pairs, seq_len, token_ce, response_mask, ref_logp, beta, loss_out,
                      weights, seq_logp=None, ws=None, stream=None):
    """DPO loss into loss_out[0] and per-token loss weights (include/sbp_dpo.h)."""
    if ws is None:
        ws = workspace(dpo_workspace_size(n_pairs), token_ce.device)
    _check(load().sbp_dpo_token_weights(
        n_pairs, seq_len, _ptr(token_ce), _ptr(response_mask), _ptr(ref_logp), float(beta),
        _ptr(loss_out), _ptr(seq_logp) if seq_logp is not None else None, _ptr(weights),
        _ptr(ws), ws.numel(), _stream(stream)))
    return ws


def lmhead_ce_backward_noalloc(hidden_states, weight, targets, loss_weights, num_chunks, loss_out,
                               d_hidden, d_weight, stream=None):
    """As lmhead_ce_backward, with the library's own fixed scratch instead of a workspace
    (include/sbp_noalloc.h): nothing is allocated, sizes above the scratch are rejected."""
    N, d = hidden_states.shape
    V = weight.shape[0]
    _check(load().sbp_lmhead_ce_backward_noalloc(
        N, d, V, num_chunks, _dtype_code(hidden_states), _ptr(hidden_states), _ptr(weight),
        _ptr(targets), _ptr(loss_weights), _ptr(loss_out), _ptr(d_hidden), _ptr(d_weight),
        _stream(stream)))


# ----------------------------------------------------------------------------- decoder layer
def layer_cfg(batch, seq_len, d_model, n_heads, n_kv_heads, head_dim, ffn, rms_eps, rope_theta,
              dtype_code, num_chunks) -> LayerCfg:
    return LayerCfg(batch, seq_len, d_model, n_heads, n_kv_heads, head_dim, ffn, rms_eps,
                    rope_theta, dtype_code, num_chunks)


def _struct(cls, tensors: Dict[str, object]):
    return cls(**{n: (tensors[n].data_ptr() if tensors.get(n) is not None else None)
                  for n in WEIGHT_FIELDS})


def layer_workspace_size(cfg: LayerCfg) -> int:
    return load().sbp_decoder_layer_workspace_size(C.byref(cfg))


def _layer_backward(fn, cfg, weights, x, dy, dx, grads, ws, stream):
    need = layer_workspace_size(cfg)
    if need == 0:
        raise SbpError(1, "invalid layer configuration")
    if ws is None:
        ws = workspace(need, x.device)
    w = _struct(LayerWeights, weights)
    g = _struct(LayerGrads, grads)
    _check(fn(C.byref(cfg), C.byref(w), _ptr(x), _ptr(dy), _ptr(dx), C.byref(g), _ptr(ws),
              ws.numel(), _stream(stream)))
    return ws


def decoder_layer_backward(cfg: LayerCfg, weights, x, dy, dx, grads, ws=None, stream=None):
    return _layer_backward(load().sbp_decoder_layer_backward_stream, cfg, weights, x, dy, dx,
                           grads, ws, stream)


def decoder_layer_backward_reverse(cfg: LayerCfg, weights, x, dy, dx, grads, ws=None,
                                   stream=None):
    """The layer backward with the chunks visited from last to first."""
    return _layer_backward(load().sbp_decoder_layer_backward_stream_reverse, cfg, weights, x, dy,
                           dx, grads, ws, stream)


def decoder_layer_forward(cfg: LayerCfg, weights, x, y, ws=None, stream=None):
    need = layer_workspace_size(cfg)
    if need == 0:
        raise SbpError(1, "invalid layer configuration")
    if ws is None:
        ws = workspace(need, x.device)
    w = _struct(LayerWeights, weights)
    _check(load().sbp_decoder_layer_forward_stream(C.byref(cfg), C.byref(w), _ptr(x), _ptr(y),
                                                   _ptr(ws), ws.numel(), _stream(stream)))
    return ws


# ----------------------------------------------------------------------------- support
def rmsnorm_forward(x2d, g, eps, y2d, rstd=None, stream=None):
    rows, cols = x2d.shape
    _check(load().sbp_rmsnorm_forward(rows, cols, _dtype_code(x2d), eps, _ptr(x2d), _ptr(g),
                                      _ptr(y2d), _ptr(rstd), _stream(stream)))


def rmsnorm_backward(x2d, g, rstd, dy2d, dx2d, dg, accumulate=False, ws=None, stream=None):
    rows, cols = x2d.shape
    need = load().sbp_rmsnorm_backward_workspace_size(rows, cols)
    if ws is None or ws.numel() < need:
        ws = workspace(need, x2d.device)
    _check(load().sbp_rmsnorm_backward(rows, cols, _dtype_code(x2d), _ptr(x2d), _ptr(g),
                                       _ptr(rstd), _ptr(dy2d), _ptr(dx2d), int(accumulate),
                                       _ptr(dg), _ptr(ws), ws.numel(), _stream(stream)))
    return ws


def embedding_forward(ids, table, y, stream=None):
    rows = ids.numel()
    V, cols = table.shape
    _check(load().sbp_embedding_forward(rows, cols, V, _dtype_code(table), _ptr(ids),
                                        _ptr(table), _ptr(y), _stream(stream)))


def embedding_backward(ids, dy2d, d_table, ws=None, stream=None):
    rows = ids.numel()
    V, cols = d_table.shape
    need = load().sbp_embedding_backward_workspace_size(rows, V)
    if ws is None or ws.numel() < need:
        ws = workspace(need, dy2d.device)
    _check(load().sbp_embedding_backward(rows, cols, V, _ptr(ids), _ptr(dy2d), _ptr(d_table),
                                         _ptr(ws), ws.numel(), _stream(stream)))
    return ws


# ----------------------------------------------------------------------------- test hooks
def debug_gemm_bf16(A, a_trans, B, b_trans, C, accumulate=False, path=0, kblk=0, ws=None,
                    stream=None):
    """C (+)= op(A) op(B) with bf16 A/B and fp32 C (see include/sbp_debug.h)."""
    M = A.shape[1] if a_trans else A.shape[0]
    K = A.shape[0] if a_trans else A.shape[1]
    N = B.shape[0] if b_trans else B.shape[1]
    if ws is None:
        ws = workspace(256, C.device)
        ws.zero_()
    _check(load().sbp_debug_gemm_bf16(M, N, K, _ptr(A), int(a_trans), A.stride(0), _ptr(B),
                                      int(b_trans), B.stride(0), _ptr(C), C.stride(0),
                                      int(accumulate), int(path), int(kblk), _ptr(ws),
                                      _stream(stream)))
    return ws


def debug_gemm_stall_bf16(A, B, C, wait_limit_ns, ws=None, stream=None):
    """The single-CTA GEMM of C = A B^T with no operand copies issued, so that its bounded
    waits run out after wait_limit_ns (include/sbp_debug.h); returns the workspace whose
    status word the kernel raises."""
    M, K = A.shape
    N = B.shape[0]
    if ws is None:
        ws = workspace(256, C.device)
        ws.zero_()
    _check(load().sbp_debug_gemm_stall_bf16(M, N, K, _ptr(A), _ptr(B), _ptr(C),
                                            int(wait_limit_ns), _ptr(ws), _stream(stream)))
    return ws


# ----------------------------------------------------------------------------- profiling
def launch_count() -> int:
    return int(load().sbp_launch_count())


def profile_begin():
    _check(load().sbp_profile_begin())


def profile_end() -> dict:
    p = Profile()
    _check(load().sbp_profile_end(C.byref(p)))
    names = ("gemm_tc", "gemm_simt", "attn_fwd", "attn_bwd")
    return {n: {"launches": p.launches[i], "ms": p.ms[i], "busy_ms": p.busy_ms[i]}
            for i, n in enumerate(names)}


def debug_attn_fwd_workspace_bytes(B, Tc, H, hd):
    """Workspace of sbp_debug_attn_fwd_bf16: the status word, then the key-range split's
    partial O (fp32), its maxima and sums, and two flags per query-tile pair."""
    pairs = ((Tc + 127) // 128 + 1) // 2
    return 256 + 4 * B * Tc * H * (hd + 2) + 8 * B * H * pairs


def debug_attn_fwd_bf16(q, Kp, Vp, o, lse, s, path=0, ws=None, stream=None):
    """Attention forward of a chunk (include/sbp_debug.h); q/o [B*Tc, H, hd], Kp/Vp
    [B, T, Hkv, hd] bf16, lse [B*Tc, H] fp32."""
    B, T, Hkv, hd = Kp.shape
    R, H, _ = q.shape
    Tc = R // B
    need = debug_attn_fwd_workspace_bytes(B, Tc, H, hd)
    if ws is None:
        ws = workspace(need, q.device)
        ws.zero_()
    elif ws.numel() * ws.element_size() < need:
        raise ValueError(f"attention forward workspace needs {need} bytes")
    _check(load().sbp_debug_attn_fwd_bf16(B, T, Tc, s, H, Hkv, hd, _ptr(q), _ptr(Kp), _ptr(Vp),
                                          _ptr(o), _ptr(lse), int(path), _ptr(ws),
                                          _stream(stream)))
    return ws


def debug_attn_bwd_bf16(q, Kp, Vp, o, dO, lse, dq, dKp, dVp, s, path=0, stream=None):
    """Attention backward of a chunk (include/sbp_debug.h)."""
    B, T, Hkv, hd = Kp.shape
    R, H, _ = q.shape
    Tc = R // B
    tcp = (Tc + 127) // 128 * 128
    ws = workspace(256 + max(4 * R * H, 8 * H * B * tcp), q.device)
    ws.zero_()
    _check(load().sbp_debug_attn_bwd_bf16(B, T, Tc, s, H, Hkv, hd, _ptr(q), _ptr(Kp), _ptr(Vp),
                                          _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq), _ptr(dKp),
                                          _ptr(dVp), int(path), _ptr(ws), _stream(stream)))
    return ws

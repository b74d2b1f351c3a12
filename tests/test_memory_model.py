"""Host checks of the device-memory model of a streamed stack step (memory_model.py): it adds up
the library's own workspace sizes, its transient part falls as 1/D toward the O(T) K/V prefix,
and max_tokens() returns the longest sequence that fits (the next one does not)."""
from memory_efficient_exact_chunk_b200 import build as sbp_build
from memory_efficient_exact_chunk_b200 import memory_model as MM
from memory_efficient_exact_chunk_b200 import sbp, synth

SHAPE = None


def shape():
    global SHAPE
    if SHAPE is None:
        sbp_build.build()
        SHAPE = MM.StackShape.from_workload(synth.WORKLOADS["llama3_8b_stack4_64k"])
    return SHAPE


def test_parameter_count_of_the_llama_stack():
    s = shape()
    # Llama-3-8B layer: q/o 4096^2, k/v 1024 x 4096, MLP 3 x 14336 x 4096, two gains
    assert s.layer_params() == 2 * 4096 ** 2 + 2 * 1024 * 4096 + 3 * 14336 * 4096 + 2 * 4096
    assert s.params() == 4 * s.layer_params() + 2 * 128256 * 4096 + 4096


def test_parts_match_the_library_and_fall_with_d():
    s = shape()
    T = 65536
    prev = None
    for D in (1, 2, 4, 8, 16):
        p = MM.stack_step_bytes(s, T, D)
        cfg = sbp.layer_cfg(1, T, 4096, 32, 8, 128, 14336, 1e-5, 500000.0, sbp.SBP_BF16, D)
        assert p["layer_workspace"] == sbp.layer_workspace_size(cfg)
        assert p["lmhead_workspace"] == sbp.lmhead_ce_workspace_size(T, 4096, 128256, D,
                                                                     sbp.SBP_BF16)
        assert p["total"] == sum(v for k, v in p.items() if k != "total")
        t = MM.transient_bytes(p)
        if prev is not None:
            assert t < prev
        prev = t
    # the part that does not shrink: K/V prefix (bf16) + its fp32 gradient, 12 KB per token at
    # d_kv = 1024, plus the two fp32 residual-gradient rows
    p16 = MM.stack_step_bytes(s, T, 16)
    assert p16["layer_workspace"] > T * 1024 * 12


def test_max_tokens_is_the_longest_that_fits():
    s = shape()
    budget = 150 * 10 ** 9
    prev = 0
    for D in (1, 4, 16):
        T = MM.max_tokens(s, D, budget)
        assert T % 128 == 0 and T > prev
        assert MM.stack_step_bytes(s, T, D)["total"] <= budget
        assert MM.stack_step_bytes(s, T + 128, D)["total"] > budget
        prev = T
    assert MM.max_tokens(s, 1, 10 ** 9) == 0          # the weights alone do not fit

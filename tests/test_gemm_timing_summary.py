"""The summary of the instrumented pair-GEMM run (memory_efficient_exact_chunk_b200/gemm_timing.py)
on a hand-written log: the warm (second) half is kept, launches without work are dropped, and
the per-shape shares are the sums of cycles over the launches."""
from memory_efficient_exact_chunk_b200 import gemm_timing

WARM = """\
SBPT ISSUE M 4096 N 16384 K 3584 epi 3 kblocks 100 total 80000 w_full 16000 w_tempty 0
SBPT ISSUE M 4096 N 16384 K 3584 epi 3 kblocks 100 total 70000 w_full 14000 w_tempty 7000
SBPT ISSUE M 0 N 16384 K 3584 epi 3 kblocks 0 total 500 w_full 0 w_tempty 0
SBPT PROD cta 0 M 4096 N 16384 K 3584 epi 3 tiles 9 total 1000 w_empty 400
SBPT EPI warp 2 M 4096 N 16384 K 3584 epi 3 total 1000 w_tfull 500 work 450
other output
"""
# the first (cold) call prints the same records with other numbers
COLD = WARM.replace("total 80000", "total 99000").replace("w_empty 400", "w_empty 900") \
           .replace("work 450", "work 50")


def test_summary_numbers(tmp_path):
    p = tmp_path / "t.log"
    # two identical calls: the first half of each kind is dropped
    p.write_text(COLD + WARM + "SBPT DONE T 32768 D 8 loss 1.0\n")
    out = gemm_timing.summarize(str(p))
    # warm ISSUE records with work: 150000 cycles, 200 k-blocks, 30000 + 7000 cycles waiting
    assert "| 4096 | 16384 | 3584 | logit gradient | 2 | 750 | 20 % | 5 % | 565 |" in out
    assert "| 16384 | 3584 | logit gradient | 1 | 40 % |" in out
    assert "| 16384 | 3584 | logit gradient | 1 | 45 % |" in out

"""The summary of the instrumented runs (memory_efficient_exact_chunk_b200/timing.py)
on a hand-written log: the warm (second) half is kept, launches without work are dropped, and
the per-shape shares are the sums of cycles over the launches."""
from memory_efficient_exact_chunk_b200 import timing

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
    out = timing.summarize(str(p))
    # warm ISSUE records with work: 150000 cycles, 200 k-blocks, 30000 + 7000 cycles waiting
    assert "| 4096 | 16384 | 3584 | logit gradient | 2 | 750 | 20 % | 5 % | 565 |" in out
    assert "| 16384 | 3584 | logit gradient | 1 | 40 % |" in out
    assert "| 16384 | 3584 | logit gradient | 1 | 45 % |" in out


KV = """\
SBPT KVPROD s 8192 Tc 8192 pairs 100 total 500000 w_empty 40000
SBPT KVISSUE s 8192 Tc 8192 pairs 100 total 500000 w_ds 90000 w_qd 1000 w_free 200 issue 300000
SBPT KVEW warp 2 s 8192 Tc 8192 pairs 100 total 500000 w_qd 100 w_sdp 200000 work 210000 flush 80000
SBPT KVEW warp 9 s 8192 Tc 8192 pairs 100 total 500000 w_qd 300 w_sdp 220000 work 230000 flush 82000
"""


def test_summary_attention_rows(tmp_path):
    p = tmp_path / "k.log"
    cold = KV.replace("issue 300000", "issue 1").replace("work 210000", "work 1")
    p.write_text(cold + KV + "SBPT DONE T 16384 D 2\n")
    out = timing.summarize(str(p))
    # per pair: total 5000, issuer waits 900 / 10 / 2, issuing 3000; element-wise (mean of the
    # two warps) waits 2100, works 2200, flushes 810; producer waits 400
    assert "| 8192 | 8192 | 100 | 5000 | 900 | 10 | 2 | 3000 | 2100 | 2200 | 810 | 400 |" in out

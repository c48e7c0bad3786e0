"""GPU parity at the long-context stream's full size: one sequence of
32768 + s tokens in a page table sized for the whole stream (32896 tokens),
at the stream's first and last steps (s = 1 and s = 128), every head compared
with the fp64 oracle.  Same launch configuration as the bench's stream leg
(batch 1).  Kept in the last file of the suite: it is the slowest host-side
setup (about 33K oracle-quantised tokens per case).
"""
import numpy as np
import pytest

from harness import gen

from _cases import check_attention
from test_gpu_decode import run_decode

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("s", [1, 128])
def test_stream_length_decode_matches_oracle(s):
    w = gen.workload("longchat7b_stream_b1_t32768_s128")
    L = w.ctx + s
    got, ref, st = run_decode(w, [L], caps=[w.ctx + w.steps])
    assert st == 0
    assert np.isfinite(got).all()
    check_attention(got, ref, f"stream 1 x {L}")

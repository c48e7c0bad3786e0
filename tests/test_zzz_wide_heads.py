"""GPU parity for the widest head count the tensor-core decode admits:
64 query heads over 8 KV heads (two heads per lane in the value kernel's
softmax warps, an N = 64 value accumulator), on both decode paths, ragged
lengths, every head compared with the fp64 oracle.
"""
import pytest

from harness import gen

from _cases import check_attention
from test_gpu_decode import run_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("path", ["tensor-core", "cuda-core"])
def test_sixty_four_query_heads_over_eight_kv_heads(monkeypatch, path):
    if path == "cuda-core":
        monkeypatch.setenv("STARKV_DECODE_PATH", "simt")
    w = gen.shrink(gen.workload("llama3_8b_gqa_decode_b32_t4096to8192"), name="wide_h64", H=64, h_kv=8,
                   hidden=1024, r_k=32, R=512, batch=3, ctx=700, ctx_lo=0)
    got, ref, st = run_decode(w, [1, 333, 700])
    assert st == 0
    check_attention(got, ref, f"64 heads, {path}")

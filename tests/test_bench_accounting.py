"""The bench's roofline denominators against closed forms.

Algorithmic bytes of a decode call and algorithmic flops of a prefill step
are what the reported fractions divide by; these tests recompute them from the
shapes alone (packed bits per channel, metadata per group, factor sizes,
causal pair counts) so a change to either side shows up here.
"""
import pytest

import bench
from harness import gen


def _closed_form_bytes_per_token(w):
    def region(r):
        n_top = int(round(w.top_fraction * r))
        return 2 * (4 * n_top + 3 * (r - n_top))  # one page (16 tokens) of one latent region

    def groups(r):
        import math
        n_top = int(round(w.top_fraction * r))
        g = math.gcd(16, math.gcd(n_top, r - n_top))
        return r // g

    key = w.h_kv * (region(w.r_k) / 16 + 4 * groups(w.r_k))
    val = region(w.R) / 16 + 4 * groups(w.R)
    return key + val


@pytest.mark.parametrize("name,expect", [("longchat7b_decode_b16_t4096", 1600), ("llama3_8b_gqa_decode_b32_t4096to8192", 672)])
def test_bytes_per_token_is_payload_plus_metadata(name, expect):
    w = gen.workload(name)
    assert bench.bytes_per_token(w) == expect
    assert _closed_form_bytes_per_token(w) == expect


def test_decode_algorithmic_bytes_on_the_bench_workload():
    w = gen.workload("longchat7b_decode_b16_t4096")
    tokens, max_pages = w.batch * w.ctx, w.ctx // 16 + 1
    got = bench.decode_algorithmic_bytes(w, tokens, w.batch, max_pages)
    factors = 2 * (32 * 32 * 128 + 1024 * 32 * 128)  # bf16 B_k and B_v
    assert got == tokens * 1600 + factors + 2 * 2 * 16 * 32 * 128 + 4 * 16 * max_pages + 4 * 16
    assert 113e6 < got < 114.5e6  # the scope table quotes 113.5 MB (cache 104.86 MB + B_v 8.39 MB + B_k 0.26 MB)


def test_prefill_flops_match_the_scope_table():
    w = gen.workload("longchat7b_prefill_b4_t30720_c2048")
    fl = bench.prefill_flops(w)
    # per sequence: causal pairs of 2048 queries at positions 30720.. over all earlier keys
    pairs = 2048 * 30720 + 2048 * 2049 // 2
    assert fl["attention"] == 4 * pairs * 32 * 4 * 128
    assert fl["attention"] / 4 == pytest.approx(1.065e12, rel=1e-3)
    assert fl["value_reexpansion"] / 4 == pytest.approx(0.275e12, rel=1e-3)
    assert fl["key_reexpansion"] / 4 == pytest.approx(8.6e9, rel=1e-2)
    assert fl["projection"] / 4 == pytest.approx(34e9, rel=2e-2)
    assert sum(fl.values()) == pytest.approx(5.53e12, rel=1e-3)


def test_packed_staging_buffer_round_trips_every_input():
    """The end-to-end leg stages a step's inputs in one byte buffer: every
    view must start aligned, not overlap the next, and read back its input."""
    import torch
    srcs = [torch.arange(16 * 4096, dtype=torch.float32).to(torch.bfloat16).view(16, 4096),
            torch.randn(16, 32, 128).to(torch.bfloat16),
            torch.arange(16, dtype=torch.int64) * 7 + 3,
            torch.arange(16 * 257, dtype=torch.int32).view(16, 257),
            torch.arange(16, dtype=torch.int32) + 4000]
    offs, total = bench.pack_layout(srcs)
    assert all(o % 256 == 0 for o in offs)
    ends = [o + s.numel() * s.element_size() for o, s in zip(offs, srcs)]
    assert all(e <= n for e, n in zip(ends, offs[1:])) and ends[-1] == total
    buf = torch.zeros(total, dtype=torch.uint8)
    for v, s in zip(bench.packed_views(buf, offs, srcs), srcs):
        v.copy_(s)
    for v, s in zip(bench.packed_views(buf.clone(), offs, srcs), srcs):
        assert v.dtype == s.dtype and v.shape == s.shape and v.is_contiguous()
        assert torch.equal(v, s)


def test_stream_schedule_appends_then_decodes_the_grown_context():
    """Stream step s appends position L0 + s through the block table and then
    decodes L0 + s + 1 tokens, so every decode includes the token just added."""
    import numpy as np
    L0 = np.array([37, 100], np.int32)
    n = 20
    bt, _ = gen.make_block_table(L0 + n, seed=3)
    slots, lens = bench.stream_schedule(L0, n, bt)
    assert slots.shape == (n, 2) and slots.dtype == np.int64
    assert lens.shape == (n, 2) and lens.dtype == np.int32
    for s in range(n):
        for b in range(2):
            pos = int(L0[b]) + s
            assert slots[s, b] == bt[b, pos // 16] * 16 + pos % 16
            assert lens[s, b] == pos + 1
    # distinct physical slots, all inside the sequence's own pages
    for b in range(2):
        assert len(set(slots[:, b].tolist())) == n
        assert set((slots[:, b] // 16).tolist()) <= set(bt[b][bt[b] >= 0].tolist())


def test_stream_workload_dispatches_to_the_stream_leg():
    w = gen.workload("longchat7b_stream_b1_t32768_s128")
    assert w.steps == 128 and w.chunk == 0 and w.batch == 1 and w.ctx == 32768

"""Byte accounting pins: the layout's bytes against the review's closed forms.

[Review] eq. 1 (dense payload), eq. 14 (mean bits, payload compression),
eq. 15 (latent payload), eq. 16 (exempt-layer fraction).  The printed values
live in tests/golden/review_numbers.json.
"""
import json
import os

import pytest

import oracle as O
from harness import gen

NUM = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "review_numbers.json")))


def test_eq14_printed_values():
    assert O.eq14_mean_bits(0.2) == pytest.approx(NUM["eq14_mean_bits_top20"]["value"], abs=1e-12)
    assert O.eq14_payload_compression(0.25, 3.2) == pytest.approx(NUM["eq14_payload_compression_rho0.25"]["value"])
    assert O.eq14_payload_compression(0.4, 3.2) == pytest.approx(NUM["eq14_payload_compression_rho0.4"]["value"])


def test_eq16_printed_values():
    f = O.eq16_retained_fraction()
    assert f == pytest.approx(NUM["eq16_retained_fraction"]["value"], abs=1e-15)
    assert 1 / f == pytest.approx(NUM["eq16_inverse"]["value"], abs=NUM["eq16_inverse"]["tol"])


@pytest.mark.parametrize("i", range(5))
def test_layout_payload_equals_eq15(i):
    w = gen.workload(i)
    cfg = O.config_of(w)
    mean_bits = O.eq14_mean_bits(w.top_fraction)            # 3.25 at top_fraction 0.25
    eq15 = O.eq15_latent_payload_bytes(1, 1, mean_bits, [[w.r_k] * w.h_kv], [w.R])
    assert O.payload_bytes_per_token(cfg) == pytest.approx(eq15, abs=1e-12)
    # metadata: one fp16 (scale, zero) pair per group per token; padding explicit
    meta = 4 * (w.h_kv * w.r_k // cfg.key.g + w.R // cfg.val.g)
    pad = w.h_kv * (cfg.key.region_bytes - cfg.key.payload_bytes) / 16 + (cfg.val.region_bytes - cfg.val.payload_bytes) / 16
    assert O.cache_bytes_per_token(cfg) == pytest.approx(eq15 + meta + pad, abs=1e-12)


def test_longchat_payload_ratio_against_eq1():
    # rank fraction 0.25 of 2 h_kv d_h channels at 3.25 bits vs an fp16 cache: 16/(0.25*3.25)
    w = gen.workload(1)
    cfg = O.config_of(w)
    dense = O.eq1_dense_payload_bytes(1, 1, 1, w.h_kv, w.d_h, 16)
    assert dense / O.payload_bytes_per_token(cfg) == pytest.approx(16 / (0.25 * 3.25), rel=1e-12)
    # the review's 20x at 3.2 bits is reproduced by a 20:80 split
    w2 = gen.shrink(w, top_fraction=0.2)
    r = (w2.h_kv * w2.r_k + w2.R) / (2 * w2.h_kv * w2.d_h)
    assert O.eq14_payload_compression(r, O.eq14_mean_bits(0.2)) == pytest.approx(20.0)


def test_known_per_token_bytes():
    # LongChat-7B shapes: 416 key payload + 512 key meta + 416 value payload + 256 value meta
    assert O.cache_bytes_per_token(O.config_of(gen.workload(1))) == 1600
    assert O.cache_bytes_per_token(O.config_of(gen.workload(3))) == 672

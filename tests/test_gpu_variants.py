"""The review's speed variants ([Review] section 6.1 and the attention-speed
ablation of section 8.1) through the same kernels: the uniform 4-bit latent
(every channel at 4 bits: top_fraction 1.0) and the unquantised latent (rotated
values stored as fp16, STARKV_FLAG_FP16_LATENT).  Quantise/pack (or store)
bit-exact, append, decode and prefill against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, download, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def _u4(i):
    return gen.shrink(gen.workload(i), top_fraction=1.0)


@pytest.mark.parametrize("wi", [0, 1, 3], ids=["tiny", "longchat", "llama3gqa"])
def test_uniform_4bit_quantize_pack_bit_exact(wi):
    S = skv()
    w = _u4(wi)
    kv, f = make_ctx(w, max_position=64)
    try:
        cfg = O.config_of(w)
        for which, lat in ((0, cfg.key), (1, cfg.val)):
            assert lat.n_top == lat.r and lat.g == 16
            rng = np.random.default_rng(which)
            n = 37
            z = (rng.standard_normal((n, lat.r)) * rng.uniform(0.01, 40, (n, 1))).astype(np.float32)
            pages = (n + 15) // 16
            codes = torch.zeros(pages * lat.region_bytes, dtype=torch.uint8, device="cuda")
            meta = torch.zeros(pages * lat.n_groups * 16, dtype=torch.int32, device="cuda")
            S.starkv_quantize_pack(kv.ctx, which, torch.from_numpy(z).cuda(), codes, meta)
            want_c, want_m = O.quantize_pack_region(z, lat)
            np.testing.assert_array_equal(codes.cpu().numpy().reshape(pages, -1), want_c)
            np.testing.assert_array_equal(meta.cpu().numpy().view(np.uint32).reshape(want_m.shape), want_m)
        assert kv.status() == 0
    finally:
        kv.close()


@pytest.mark.parametrize("wi,lens", [(0, [256, 17, 1]), (1, [300, 1000]), (3, [700, 1500, 33])],
                         ids=["tiny", "longchat", "llama3gqa"])
def test_uniform_4bit_decode(wi, lens):
    w = _u4(wi)
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=1)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        qn = gen.make_queries(len(lens), w.H, w.d_h)
        out = kv.decode(lc, bf16_tensor(qn), torch.from_numpy(bt).cuda(), torch.tensor(np.asarray(lens, np.int32)).cuda())
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(), O.decode(oc, qn, f.B_k, f.B_v, bt, lens), "uniform 4-bit decode")
    finally:
        kv.close()


def test_uniform_4bit_append_then_prefill():
    S = skv()
    w = _u4(4)
    existing, chunks = [300, 0], [150, 70]
    totals = [e + c for e, c in zip(existing, chunks)]
    kv, f = make_ctx(w, max_position=max(totals) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, existing, extra_pages=2, caps=totals)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        X = np.concatenate([gen.make_hidden(c, w.hidden, name="X_chunk", sub=b) for b, c in enumerate(chunks)])
        sl = np.concatenate([gen.slots_for(bt, b, np.arange(e, e + c)) for b, (e, c) in enumerate(zip(existing, chunks))])
        lat = torch.zeros((X.shape[0], w.h_kv * w.r_k + w.R), dtype=torch.float32, device="cuda")
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda(), lat)
        assert kv.status() == 0
        # the appended tokens: the oracle quantiser on the exported latents, bit for bit
        zl = lat.cpu().numpy()
        O.write_latents(oc, sl, zl[:, :w.h_kv * w.r_k].reshape(-1, w.h_kv, w.r_k), zl[:, w.h_kv * w.r_k:])
        got = download(lc, oc)
        for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
            np.testing.assert_array_equal(getattr(got, name), getattr(oc, name), err_msg=name)
        q = gen.make_queries(int(cu[-1]), w.H, w.d_h, name="q_chunk")
        sel = {0: list(range(0, 150, 9)), 1: list(range(0, 70, 7))}
        out = kv.prefill(lc, bf16_tensor(q), torch.from_numpy(cu).cuda(), torch.from_numpy(bt).cuda(),
                         torch.tensor(np.asarray(totals, np.int32)).cuda(), max(chunks))
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(), O.prefill(oc, q, cu, f.B_k, f.B_v, bt, totals, select=sel),
                        "uniform 4-bit prefill")
    finally:
        kv.close()


# ---------------------------------------------------------------------------
# the unquantised variant: rotated latents stored as fp16 ([Review] section 8.1)
# ---------------------------------------------------------------------------
def _f16(i):
    return gen.shrink(gen.workload(i), fp16_latent=True)


@pytest.mark.parametrize("wi", [0, 1, 3], ids=["tiny", "longchat", "llama3gqa"])
def test_fp16_latent_store_bit_exact(wi):
    S = skv()
    w = _f16(wi)
    kv, f = make_ctx(w, max_position=64)
    try:
        cfg = O.config_of(w)
        sizes = S.starkv_cache_layout(S.make_config(w.H, w.h_kv, w.d_h, w.hidden, w.r_k, w.R, 64, w.top_fraction,
                                                    w.rope_base, S.FLAG_FP16_LATENT), 1)
        assert sizes["k_meta_bytes"] == 0 and sizes["v_meta_bytes"] == 0
        assert sizes["k_codes_bytes"] == w.h_kv * cfg.key.region_bytes
        for which, lat in ((0, cfg.key), (1, cfg.val)):
            rng = np.random.default_rng(which + 3)
            n = 37
            z = (rng.standard_normal((n, lat.r)) * rng.uniform(0.01, 40, (n, 1))).astype(np.float32)
            pages = (n + 15) // 16
            codes = torch.full((pages * lat.region_bytes,), 0xAB, dtype=torch.uint8, device="cuda")
            meta = torch.zeros(4, dtype=torch.int32, device="cuda")
            S.starkv_quantize_pack(kv.ctx, which, torch.from_numpy(z).cuda(), codes, meta)
            want_c, _ = O.quantize_pack_region(z, lat)
            np.testing.assert_array_equal(codes.cpu().numpy().reshape(pages, -1), want_c)
            zh = torch.empty((n, lat.r), dtype=torch.float32, device="cuda")
            S.starkv_dequantize(kv.ctx, which, torch.from_numpy(want_c.reshape(-1)).cuda(), meta, n, zh)
            np.testing.assert_array_equal(zh.cpu().numpy(), O.dequantize_region(want_c, None, lat, n))
        assert kv.status() == 0
    finally:
        kv.close()


@pytest.mark.parametrize("path", ["tc", "simt"])
@pytest.mark.parametrize("wi,lens", [(0, [256, 17, 1]), (1, [300, 1000]), (3, [700, 1500, 33])],
                         ids=["tiny", "longchat", "llama3gqa"])
def test_fp16_latent_decode(monkeypatch, path, wi, lens):
    if path == "simt":
        monkeypatch.setenv("STARKV_DECODE_PATH", "simt")
    w = _f16(wi)
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, lens, extra_pages=1)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        qn = gen.make_queries(len(lens), w.H, w.d_h)
        out = kv.decode(lc, bf16_tensor(qn), torch.from_numpy(bt).cuda(), torch.tensor(np.asarray(lens, np.int32)).cuda())
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(), O.decode(oc, qn, f.B_k, f.B_v, bt, lens), f"fp16 latent decode ({path})")
    finally:
        kv.close()


@pytest.mark.parametrize("ppath", ["tc", "simt"])
def test_fp16_latent_append_then_prefill(monkeypatch, ppath):
    if ppath == "simt":
        monkeypatch.setenv("STARKV_PREFILL_PATH", "simt")
    S = skv()
    w = _f16(4)
    existing, chunks = [300, 0], [150, 70]
    totals = [e + c for e, c in zip(existing, chunks)]
    kv, f = make_ctx(w, max_position=max(totals) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, existing, extra_pages=2, caps=totals)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        X = np.concatenate([gen.make_hidden(c, w.hidden, name="X_chunk", sub=b) for b, c in enumerate(chunks)])
        sl = np.concatenate([gen.slots_for(bt, b, np.arange(e, e + c)) for b, (e, c) in enumerate(zip(existing, chunks))])
        lat = torch.zeros((X.shape[0], w.h_kv * w.r_k + w.R), dtype=torch.float32, device="cuda")
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda(), lat)
        assert kv.status() == 0
        zl = lat.cpu().numpy()
        O.write_latents(oc, sl, zl[:, :w.h_kv * w.r_k].reshape(-1, w.h_kv, w.r_k), zl[:, w.h_kv * w.r_k:])
        got = download(lc, oc)
        for name in ("k_codes", "v_codes"):
            np.testing.assert_array_equal(getattr(got, name), getattr(oc, name), err_msg=name)
        q = gen.make_queries(int(cu[-1]), w.H, w.d_h, name="q_chunk")
        sel = {0: list(range(0, 150, 9)), 1: list(range(0, 70, 7))}
        out = kv.prefill(lc, bf16_tensor(q), torch.from_numpy(cu).cuda(), torch.from_numpy(bt).cuda(),
                         torch.tensor(np.asarray(totals, np.int32)).cuda(), max(chunks))
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(), O.prefill(oc, q, cu, f.B_k, f.B_v, bt, totals, select=sel),
                        f"fp16 latent prefill ({ppath})")
    finally:
        kv.close()

"""GPU parity of starkv_decode_attn against the fp64 oracle.

Both sides read the same oracle-written packed cache.  Small cases compare every
output; full-size workloads compare sampled sequences (all heads) in the same
launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def run_decode(w, seq_lens, seed=0, extra_pages=3, sample=None, caps=None):
    kv, f = make_ctx(w, seed, max_position=max(int(max(seq_lens)) + 16, 64))
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, seq_lens, seed, extra_pages, caps=caps)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        q = gen.make_queries(len(seq_lens), w.H, w.d_h, seed)
        out = kv.decode(lc, bf16_tensor(q), torch.from_numpy(bt).cuda(),
                        torch.tensor(np.asarray(seq_lens, np.int32)).cuda())
        st = kv.status()
        got = out.float().cpu().numpy()
        ref = O.decode(oc, q, f.B_k, f.B_v, bt, seq_lens, seqs=sample)
        return got, ref, st
    finally:
        kv.close()


def test_tiny_full_workload():
    w = gen.workload(0)
    got, ref, st = run_decode(w, [w.ctx])
    assert st == 0
    check_attention(got, ref, "tiny T=256")


def test_tiny_ragged_lengths():
    w = gen.workload(0)
    lens = [1, 15, 16, 17, 100, 256, 0]
    got, ref, st = run_decode(w, lens)
    assert st == 0
    check_attention(got, ref, "tiny ragged")
    assert np.all(got[-1] == 0)        # empty sequence -> zero row


def test_longchat_shapes_small():
    w = gen.workload(1)
    got, ref, st = run_decode(w, [1, 33, 300, 1000])
    assert st == 0
    check_attention(got, ref, "longchat small")


def test_llama3_gqa_shapes_small():
    w = gen.workload(3)
    got, ref, st = run_decode(w, [7, 64, 129, 700, 1500])
    assert st == 0
    check_attention(got, ref, "llama3 gqa small")


def test_llama3_gqa_empty_sequences_between_others():
    # the score kernel shares out only the tiles that hold tokens: empty
    # sequences first, between others and last must be skipped, not shift them
    w = gen.workload(3)
    lens = [0, 300, 0, 1, 2100, 17, 0]
    got, ref, st = run_decode(w, lens)
    assert st == 0
    check_attention(got, ref, "llama3 gqa with empty sequences")
    for b, L in enumerate(lens):
        if L == 0:
            assert np.all(got[b] == 0)


def test_cuda_core_path_longchat_shapes(monkeypatch):
    # the CUDA-core kernels remain the path for shapes the tensor-core kernels do not cover
    monkeypatch.setenv("STARKV_DECODE_PATH", "simt")
    w = gen.workload(1)
    got, ref, st = run_decode(w, [1, 33, 300])
    assert st == 0
    check_attention(got, ref, "longchat small, cuda-core path")


def test_page_table_with_spare_capacity():
    # block tables longer than the sequences (the decode step's usual state)
    w = gen.workload(1)
    got, ref, st = run_decode(w, [40, 90], caps=[200, 300])
    assert st == 0
    check_attention(got, ref, "spare capacity")


@pytest.mark.slow
def test_longchat_full_size_sampled():
    w = gen.workload(1)
    lens = [w.ctx] * w.batch
    got, ref, st = run_decode(w, lens, sample=[0, 7, 15])
    assert st == 0
    check_attention(got, ref, "longchat b16 t4096 (sampled)")
    assert np.isfinite(got).all()


@pytest.mark.slow
def test_llama3_gqa_full_size_sampled():
    w = gen.workload(3)
    lens = gen.make_seq_lens(w)
    got, ref, st = run_decode(w, lens, sample=[0, int(np.argmax(lens)), int(np.argmin(lens)), 31])
    assert st == 0
    check_attention(got, ref, "llama3 gqa b32 ragged (sampled)")


def test_bad_page_sets_status_and_stays_finite():
    w = gen.workload(0)
    S = skv()
    kv, f = make_ctx(w)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, [64])
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        bt = bt.copy()
        bt[0, 1] = n_pages + 100
        q = bf16_tensor(gen.make_queries(1, w.H, w.d_h))
        out = kv.decode(lc, q, torch.from_numpy(bt).cuda(), torch.tensor([64], dtype=torch.int32).cuda())
        assert kv.status() & S.DEV_BAD_PAGE
        assert torch.isfinite(out.float()).all()
        # a sequence longer than its page row
        out = kv.decode(lc, q, torch.from_numpy(bt[:, :2]).cuda(), torch.tensor([64], dtype=torch.int32).cuda())
        assert kv.status() & S.DEV_BAD_SEQ_LEN
        assert torch.all(out.float() == 0)
    finally:
        kv.close()


def test_workspace_too_small_is_rejected():
    w = gen.workload(0)
    S = skv()
    kv, f = make_ctx(w)
    try:
        lc = kv.new_cache(4)
        q = bf16_tensor(gen.make_queries(1, w.H, w.d_h))
        bt = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
        sl = torch.tensor([10], dtype=torch.int32, device="cuda")
        out = torch.empty_like(q)
        ws = torch.empty(16, dtype=torch.uint8, device="cuda")
        with pytest.raises(S.StarKVError) as e:
            S.starkv_decode_attn(kv.ctx, lc.struct, q, bt, sl, out, ws)
        assert e.value.code == S.ERR_WORKSPACE_TOO_SMALL
    finally:
        kv.close()


def test_streaming_append_then_decode():
    """The long-context loop at reduced length: append one token, decode, repeat.

    Each side appends the same hidden states with its own arithmetic (GPU
    append vs oracle append) and decodes its own cache."""
    w = gen.shrink(gen.workload(2), ctx=500, steps=6)
    S = skv()
    kv, f = make_ctx(w)
    try:
        L0 = w.ctx
        cfg, oc, bt, n_pages = oracle_cache(w, [L0], caps=[L0 + w.steps])
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        btd = torch.from_numpy(bt).cuda()
        for step in range(w.steps):
            pos = L0 + step
            X = gen.make_hidden(1, w.hidden, name="X_step", sub=step)
            q = gen.make_queries(1, w.H, w.d_h, name="q_step", sub=step)
            slot = gen.slots_for(bt, 0, [pos])
            S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(slot).cuda())
            O.append(oc, X, f.A_k, f.A_v, slot)
            out = kv.decode(lc, bf16_tensor(q), btd, torch.tensor([pos + 1], dtype=torch.int32).cuda())
            if step in (0, w.steps - 1):
                ref = O.decode(oc, q, f.B_k, f.B_v, bt, [pos + 1])
                check_attention(out.float().cpu().numpy(), ref, f"stream step {step}")
        assert kv.status() == 0
    finally:
        kv.close()

"""GPU parity of starkv_prefill_attn (causal chunk attention) against the oracle.

The existing context comes from an oracle-written cache; the chunk's own
tokens are appended by each side with its own arithmetic from the same hidden
states, then every chunk query attends causally."""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def run_prefill(w, existing, chunks, seed=0, select=None):
    S = skv()
    totals = [e + c for e, c in zip(existing, chunks)]
    kv, f = make_ctx(w, seed, max_position=max(totals) + 16)
    try:
        cfg, oc, bt, n_pages = oracle_cache(w, existing, seed, extra_pages=2, caps=totals)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        Xs, slots = [], []
        for b, (e, c) in enumerate(zip(existing, chunks)):
            Xs.append(gen.make_hidden(c, w.hidden, seed, name="X_chunk", sub=b))
            slots.append(gen.slots_for(bt, b, np.arange(e, e + c)))
        X = np.concatenate(Xs)
        sl = np.concatenate(slots)
        S.starkv_append(kv.ctx, lc.struct, bf16_tensor(X), torch.from_numpy(sl).cuda())
        O.append(oc, X, f.A_k, f.A_v, sl)
        q = gen.make_queries(int(cu[-1]), w.H, w.d_h, seed, name="q_chunk")
        out = kv.prefill(lc, bf16_tensor(q), torch.from_numpy(cu).cuda(), torch.from_numpy(bt).cuda(),
                         torch.tensor(np.asarray(totals, np.int32)).cuda(), max(chunks))
        st = kv.status()
        ref = O.prefill(oc, q, cu, f.B_k, f.B_v, bt, totals, select=select)
        return out.float().cpu().numpy(), ref, st
    finally:
        kv.close()


def test_tiny_prefill():
    w = gen.workload(0)
    got, ref, st = run_prefill(w, [40, 0, 100], [9, 20, 37])
    assert st == 0
    check_attention(got, ref, "tiny prefill")


def test_longchat_shapes_prefill_small():
    w = gen.workload(4)
    got, ref, st = run_prefill(w, [300, 17], [64, 33])
    assert st == 0
    check_attention(got, ref, "longchat prefill small")


def test_gqa_prefill_small():
    w = gen.workload(3)
    got, ref, st = run_prefill(w, [128, 5], [50, 16])
    assert st == 0
    check_attention(got, ref, "gqa prefill small")


@pytest.mark.slow
def test_longchat_prefill_full_size_sampled():
    w = gen.workload(4)
    sel = {0: [0, 1, 1000, 2047], 3: [5, 2046]}
    got, ref, st = run_prefill(w, [w.ctx] * w.batch, [w.chunk] * w.batch, select=sel)
    assert st == 0
    check_attention(got, ref, "longchat prefill b4 t30720 c2048 (sampled)")

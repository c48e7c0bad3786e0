"""Failure detection without a GPU fault: a bounded device wait that runs out.

Every pipelined kernel waits on shared-memory barriers with a time limit; when
the limit passes it sets STARKV_DEV_WAIT_TIMEOUT in the context's status word
and winds down instead of spinning.  starkv_selftest_wait_timeout runs that
same wait on a barrier nothing completes, with a 1 ms limit, so the test can
check that the status reaches the host and that the context keeps working.
"""
import numpy as np
import pytest
import torch

import oracle as O
from harness import gen

from _cases import bf16_tensor, check_attention, make_ctx, oracle_cache, skv, upload

pytestmark = pytest.mark.gpu


def test_wait_runs_out_sets_status_and_context_survives():
    S = skv()
    w = gen.workload(0)
    lens = [200, 37]
    kv, f = make_ctx(w, max_position=max(lens) + 16)
    try:
        assert kv.status() == 0
        S.starkv_selftest_wait_timeout(kv.ctx, 1_000_000)
        st = kv.status()
        assert st & S.DEV_WAIT_TIMEOUT
        assert kv.status() == 0  # reading clears the word
        # the context still serves a decode that matches the oracle
        cfg, oc, bt, n_pages = oracle_cache(w, lens)
        lc = kv.new_cache(n_pages)
        upload(lc, oc)
        q = gen.make_queries(len(lens), w.H, w.d_h)
        out = kv.decode(lc, bf16_tensor(q), torch.from_numpy(bt).cuda(),
                        torch.tensor(np.asarray(lens, np.int32)).cuda())
        assert kv.status() == 0
        check_attention(out.float().cpu().numpy(), O.decode(oc, q, f.B_k, f.B_v, bt, lens), "after a time-out")
    finally:
        kv.close()

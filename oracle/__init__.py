"""fp64 CPU oracle for STAR-KV latent-cache attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything under ``oracle/``: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` do.  The oracle shares no code with
the CUDA library (no kernels, headers, tables or constants), and the library
never imports it.

Every function states the passage it follows; citations name the page and
the section/equation on it:
  [Review]  "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression"
            (technical review of arXiv 2606.08382).
  [Card]    model card "longchat-7b-starkv-proxima".
  [CaliDrop] machine review of CaliDrop (attention decomposition theorem, eq. 1).

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines (scipy's Hadamard matrix, the
transformers RoPE helper, torch's scaled-dot-product attention), brute force
or exhaustive enumeration.  No function is "parity unpinned".
"""
from .starkv_oracle import *  # noqa: F401,F403

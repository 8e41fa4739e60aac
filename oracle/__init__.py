"""fp64 CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously correct restatement of what the
DeepSeek Sparse Attention hot path computes, written from the pages' equations:

* ``fp8``      -- e4m3 decoding and the per-128 activation quantiser
                  ("详解DSA", indexer code: ``act_quant`` on q and k),
* ``indexer``  -- Lightning-Indexer scores, Eq. (1) of "详解DSA",
* ``topk``     -- token-wise top-k selection S_t, Eq. (2) of "详解DSA",
* ``mla``      -- attention of all query heads over the selected latent entries
                  (MQA mode, "DeepSeek V3.2 稀疏注意力", section on embedding DSA
                  in MLA), plus the dense-masked form the official demo uses,
* ``brute``    -- pure-Python loops of the same formulas for tiny inputs.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import it.  It shares no code with the CUDA library and
never reads anything the CUDA path produced as an input.  All arithmetic is
numpy float64; BLAS matrix products are used as single steps.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against brute force, closed forms, library routines (torch's float8 cast,
``scaled_dot_product_attention``, full sorts) or invariants.
"""

from . import brute, fp8, indexer, mla, topk  # noqa: F401

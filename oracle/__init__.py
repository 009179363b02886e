"""Oracle for the CARVE recurrent core: plain, slow, fp64, CPU only.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import anything here.  The
product path (``chunk_gated_delta_02_b200``) never imports, links or calls it,
and this package imports nothing from the product path.

Modules
-------
``carve_oracle.c``  token-by-token fp64 recurrence and its sequential reverse
                    pass (built into ``_liboracle.so`` by ``build.py``).
``ref``             ctypes wrapper: per (sequence, head) pair and batched.
``chunked``         the WY-form chunk solve written with dense fp64 linear
                    algebra; used only to pin the recurrence (the pages'
                    chunkability theorem says the two must agree).
``decode``          the single-token decode step with its chunk bookkeeping.
``activation``      the decay activation g = -s softplus(a) that the kernels
                    can apply to raw decay logits, and its derivative.

Every function here is pinned by ``tests/test_oracle_pins.py`` to closed
forms, special-case reductions, a hand-computed example and finite
differences.
"""

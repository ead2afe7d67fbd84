"""CPU oracle for the Velox routed block-sparse attention path.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the path computes, used to check the CUDA library.  Only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py`` may import it.  The product path
(``routed_block_sparse_b200``) never imports, calls or falls back to it, and it
shares no code, table or constant generator with the CUDA sources.

Floating point is fp64 throughout, from the exact bf16/fp32 input values.
numpy supplies library primitives only (matmul, exp, sort, sum).

Modules and the passages they follow:

- ``gilbert``    global-aligned Gilbert block order and the 26-neighbour
                 safeguard blocks (Velox project page, "02 · Method",
                 "Keeping neighbours adjacent in the block order" and its
                 figure "Incremental Gilbert order"; arXiv 2610.22311 digest,
                 "Prerequisites", "Gilbert space-filling curve").
- ``importance`` per-head block importance, softmax over history blocks of the
                 mean-query . mean-key product (digest, "Method steps", step
                 four, Eq. 9; onedev.kr summary, "How it differs").
- ``route``      soft geometry fusion and route materialisation (project page,
                 "02 · Method", fusion formula and "Covered and uncovered
                 blocks"; digest, "Core method", Eq. 11, and "Method steps",
                 Eq. 12-14; onedev.kr summary, "How it differs").
- ``attention``  attention over exactly the tokens of the routed 128-token KV
                 tiles (digest, "Core method", Eq. 15; project page, "Why the
                 route is a block, not a token"), and its two-phase form with
                 the current chunk's own keys (digest, "Reproducibility").
- ``geometry``   frustum-slab overlap g_{i,r} and coverage rho_i, the inputs
                 of the route build (project page, "02 · Method", steps 01-02;
                 digest, "Method steps", Eq. 7-8; onedev.kr summary, "How it
                 differs").

- ``audit``      the geometry-model consistency audit: R_geo, R_50, top-80
                 recall with and without fusion, changed blocks (project
                 page, "03 · Results"; digest, results table; onedev.kr
                 summary, "Results").

- ``slabs``      the slab-table build (token rectangle and 10/90 percentile
                 depth interval per history block) and the recency-priority
                 multiwarp query depth (digest, "Method steps", Eq. 4-6;
                 project page, "02 · Method", steps 01-02).

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` against invariants, closed forms, textbook routines
and brute force, not against itself.
"""

from . import gilbert, importance, route, attention, geometry, audit, slabs  # noqa: F401

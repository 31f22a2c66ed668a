"""Oracle for Top-p block routing and block-sparse attention: TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 numpy restatement of what the hot path computes, written
from the FVAttn pages and sharing no code, table or helper with the CUDA
library.  Only tests/, the package smoke check and the bench's CPU-baseline
leg may import it; the product path must never route through it.

Modules:
  hilbert    frame-major 2-D Hilbert token order (enumerated curve)
  route      pooling, block scores, softmax, Top-p CDF, Top-k floor, CSR, L_h
  attention  softmax attention over the retained key blocks; dense attention
  fp8        the same attention with an e4m3 P.V product (per-block V scales)
  masks      window + rotating anchor block masks
  stripes    periodic diagonal stripe block masks (six parameters per head)
  sasa       slack-aware augmentation budget (Eqs. 7-10) and the augmented CSR
  rlb        runtime load balancing: rank loads, rho, the pair-swap plan search

Pin status: every function is pinned by tests/test_oracle_*.py against
closed forms, invariants, brute force or a library routine (see each module's
header).  The pages print no worked numerical example of routing or attention
on realistic inputs, so agreement on the synthetic workloads beyond those pins
rests on the pins themselves.
"""
from .hilbert import frame_hilbert_perm, hilbert_cells, identity_perm  # noqa: F401
from .route import (RouteResult, TIE_REL, block_counts, decode, pool_head, route,  # noqa: F401
                    route_scores, token_perm)
from .attention import attend_block, dense_attention, sparse_attention  # noqa: F401

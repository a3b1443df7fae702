"""fp64 CPU oracle for block-sparse attention over 3D-tiled video tokens.

TEST INFRASTRUCTURE ONLY. Nothing in the library's product path imports,
calls or links this package; only the test suite, the smoke check and the
benchmark's CPU-baseline leg may use it. It shares no code with the CUDA
path: it takes plain arrays (natural token layout [B, L, heads, D]) and
returns plain arrays.

The oracle restates, in the plainest form, what the method computes:

* tiling: tokens grouped into (t, h, w) tiles of the latent grid
  (``tiling``), following the video-aware block organisation of the FVAttn
  summary page (Summary) and the shared 3D tile granularity of the
  FPSAttention page (Approach);
* routing: tile-mean pooled Q/K, coarse block scores, and per query tile a
  kept set of key tiles by top-k, by top-p with a top-k floor (FVAttn page,
  Summary and Abstract) or by a fixed 3D tile window (FPSAttention page,
  ablation table rows on sparsity windows) (``select``);
* per-tile e4m3 quantisation of Q/K at the sparsity tile granularity
  (FPSAttention page, Approach) (``e4m3``);
* attention: dense softmax attention in fp64 under the token mask that the
  kept tile pairs define (``attention``).

Every function is pinned by tests against closed forms, brute force or a
library routine (see tests/test_oracle_*.py). Parity status per function is
listed in each module header.
"""

from . import tiling, select, e4m3, attention  # noqa: F401

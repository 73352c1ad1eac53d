"""The oracle: plain, slow, fp64 CPU definitions of what the coupling computes.

This package is test infrastructure.  Only tests/, the smoke check and the
bench's CPU-baseline leg may import it; the CUDA library never does, and the two
share no code.  Every function cites the passage of "Spatial-Spectral Coupling
as Attention" (project page) or of the ai4snews digest of the same paper that
it restates.

Parity pins (tests/test_oracle_*.py) tie each function to facts the pages and
the mathematics fix: closed forms, invariants, library routines on special cases
(torch scaled_dot_product_attention and autograd in fp64, numpy sorting),
central finite differences and hand-worked golden cases under tests/golden/.
"""
from .coupling import dense_fwd, dense_bwd, geo_fwd, geo_bwd, geo_support
from .patches import fps, csr, pool, scores, topk, patch_pipeline
from .linear import linear_fwd, linear_bwd
from .mesh import fps_mesh, sssp

__all__ = ["dense_fwd", "dense_bwd", "geo_fwd", "geo_bwd", "geo_support",
           "fps", "csr", "pool", "scores", "topk", "patch_pipeline",
           "linear_fwd", "linear_bwd", "fps_mesh", "sssp"]

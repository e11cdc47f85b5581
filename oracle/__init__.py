"""Oracle: plain, slow, fp64 CPU reference for the FG^2-GDN chunkwise forward.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference arm of bench.py may import this package.  It shares
no code with the CUDA library (gated_delta_rule_fg_b200), and the library
never imports it.

Contents and what pins each part (the pins live in tests/test_oracle_*.py):
  gdn_seq            token-by-token eq. (11) in C (gdn_oracle.c).  Pinned by the
                     delta-rule write invariant, the gradient-step identity
                     (autograd), the DeltaNet / GDN / KDA special cases, the
                     beta = 0 and T = 1 closed forms, superposition and scale
                     invariance, the non-expansive bound and the secular
                     spectrum of its one-step transition.
  gdn_chunked        chunkwise WY/UT form in numpy; pinned by agreement with
                     gdn_seq (two independent algorithms) and chunk-size
                     invariance.
  deltaproduct_seq   DeltaProduct n_h with a forget gate in C; pinned by its
                     reductions to gated DeltaNet (beta_2 = 0), to DeltaNet on
                     the interleaved sequence (gamma = 1) and by the Householder
                     reflection at beta = 2.
  spectral.*         closed forms (spectral norm of I - eta j k^T, the GDN2
                     shrink, the secular equation); pinned against numpy SVD /
                     eigenvalues on small matrices.
  backward.gdn_grads gradients of the forward by fp64 autograd through the token
                     loop; pinned by finite differences of the C forward and a
                     one-token closed form (tests/test_oracle_backward_pins.py).
  gdn2.*             GDN2 (non-tied erase / write) with the token-wise stability
                     transforms, token by token and in non-tied WY chunks; pinned
                     by the KDA case through gdn_seq, brute-force SVD of every
                     transformed transition, and the two algorithms' agreement
                     (tests/test_oracle_gdn2_pins.py).
"""
from ._lib import build, deltaproduct_seq, gdn_seq, host_cpu, max_threads  # noqa: F401
from .chunked import gdn_chunked  # noqa: F401
from . import spectral  # noqa: F401
from . import gdn2  # noqa: F401

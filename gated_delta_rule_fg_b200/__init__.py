"""B200-native FG^2-GDN chunkwise forward (gated delta rule, fine-grained gates).

The operator lives in a C-ABI shared library built from csrc/ (CUDA for
sm_100a); `gated_delta_rule_fg_b200.ops` is a thin ctypes binding to it.
"""

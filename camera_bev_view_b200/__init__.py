"""B200-native exact dense Sampling-VT (FlashBEV-style gather-reduction).

The compute lives in ``libbevsample.so`` (hand-written sm_100a CUDA behind a C
ABI, declared in ``include/bevsample.h``).  ``camera_bev_view_b200.ops`` is the
thin ctypes binding; importing this package loads nothing, so the CPU-only
input generator (``camera_bev_view_b200.inputs``) stays usable without a GPU.
"""

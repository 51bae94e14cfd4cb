"""B200-native Video Delta Attention (VDA): bidirectional frame-level delta scan.

The compute path is ``libvda.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/vda.h``); ``frame_level_delta_b200.vda`` is its thin ctypes
binding. ``frame_level_delta_b200.inputs`` draws the seeded synthetic workloads.
"""

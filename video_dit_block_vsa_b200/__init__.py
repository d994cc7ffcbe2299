"""B200-native (sm_100a) video sparse attention (VSA) forward path.

``video_dit_block_vsa_b200.vsa`` is the Python binding of the C ABI in
``include/vsa.h`` (``libvsa.so``, built from ``csrc/``).  Importing it loads the
CUDA library and raises if it has not been built; there is no fallback.
``video_dit_block_vsa_b200.workloads`` draws the seeded synthetic inputs.
"""

"""B200-native forward pass of the VDN-H3 bidirectional linear-attention branch.

The compute path is `libvdn.so` (hand-written sm_100a CUDA behind a C ABI,
declared in include/vdn.h).  `api` is the thin Python binding; `synth` draws the
seeded synthetic inputs.  Importing this package does not load the library.
"""

__all__ = ["api", "synth", "build"]

"""B200-native head-wise segmented paged attention (SegPagedAttention).

Submodules:
  * ``segkv``     -- thin ctypes binding over ``libsegkv.so`` (the C ABI in ``include/segkv.h``);
  * ``workloads`` -- seeded synthetic inputs (no attention arithmetic);
  * ``build``     -- compiles the CUDA library for sm_100a.

Nothing is imported eagerly so that importing ``workloads`` never loads the CUDA library.
"""

__all__ = ["segkv", "workloads", "build"]

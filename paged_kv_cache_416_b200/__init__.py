"""B200-native paged KV-cache decode attention (sm_100a CUDA behind a C ABI).

Modules:
  pagedattn  ctypes binding of ``libpagedattn.so`` (loads the CUDA library;
             raises if it is missing -- there is no CPU fallback)
  alloc      host-side block allocator (free list + reference counts) that
             builds block tables, slot mappings and copy-on-write pairs
  workloads  seeded synthetic inputs
  build      compiles the CUDA library in-tree with nvcc for sm_100a
"""

__version__ = "0.1.0"

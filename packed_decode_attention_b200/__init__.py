"""B200-native Block-GTQ packed KV-cache decode attention.

The work happens in the in-tree CUDA library ``libbgtq.so`` (C ABI in
``include/bgtq.h``); ``bgtq`` is its ctypes binding and ``workloads`` the
seeded synthetic inputs.
"""

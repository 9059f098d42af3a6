"""B200-native top-1 (Switch-style) mixture-of-experts gate.

The compute lives in the CUDA library libmoe_top1.so (C ABI declared in
include/moe_top1.h); bwd_route_b200.ops is its thin ctypes binding. Importing
this package loads nothing: the library is loaded on first use of ops, and a
missing library is an error, never a fallback.
"""

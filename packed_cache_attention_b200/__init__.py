"""libkvq: B200-native packed KV-cache quantization (Block-GTQ / TQ-MSE, NQKV-style NF4).

The compute path lives in the CUDA library libkvq.so (include/kvq.h). This
package holds the ctypes binding (kvq.py) and the seeded input generators
(workloads.py). Importing the package does not load the library; the first
call through kvq.py does, and fails loudly if it is missing.
"""

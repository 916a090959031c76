"""B200-native W4A4 rotated linear layer (sm_100a CUDA kernels behind a C ABI).

Import :mod:`w4a4_bit_gemm_hq_b200.hq` for the calls; :mod:`.synth` draws the
seeded synthetic workloads.  The package imports no CUDA code by itself, so
the input generator stays usable without the built library.
"""

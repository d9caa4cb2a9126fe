"""key_switching_b200 -- CKKS hybrid key switching on NVIDIA B200 (sm_100a).

The hot path (NTT, ModUp, key inner product with in-kernel ChaCha12
regeneration of the key's uniform half, ModDown, fused key switch) lives in
the CUDA library libpc.so behind the C ABI of include/pc.h; the submodule
`pc` is its thin ctypes binding (`from key_switching_b200 import pc`) and
`synth` the seeded synthetic inputs.
"""

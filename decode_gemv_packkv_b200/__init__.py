"""PackKV decode path for NVIDIA B200 (sm_100a).

`decode_gemv_packkv_b200.packkv` binds the C-ABI library `libpackkv.so`
(encoder, token append, fused q·Kᵀ and p·V over the packed cache).
`decode_gemv_packkv_b200.synth` draws the seeded synthetic inputs.
Importing this package loads nothing; importing `.packkv` loads the CUDA
library and raises if it is missing.
"""

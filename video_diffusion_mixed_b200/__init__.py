"""B200-native hot path of 6Bit-Diffusion (NVFP4/INT8 dynamic mixed precision).

The compute lives in ``libsixbit.so`` (hand-written sm_100a CUDA behind a C ABI, declared in
``include/sixbit.h``); ``video_diffusion_mixed_b200.sixbit`` is its thin ctypes binding.
``synth`` draws seeded synthetic inputs.
"""

"""video_dit_b200: RotateAttention's INT4 attention forward for video DiTs with
3D RoPE, as hand-written sm_100a CUDA kernels behind a C ABI.

``rota_attn`` is the thin ctypes binding of ``librota_attn.so``; ``synth``
holds the seeded workload generators.
"""

"""Latent mixture-of-experts FFN block for NVIDIA B200 (sm_100a).

The compute path is liblmoe.so (hand-written CUDA, C ABI in include/lmoe.h);
`binding` mirrors its entry points one to one, `layer` holds a layer's
weights in device memory, `synth` draws seeded synthetic workloads."""
from .binding import *  # noqa: F401,F403
from .binding import LmoeError, lib, make_cfg, make_shared  # noqa: F401

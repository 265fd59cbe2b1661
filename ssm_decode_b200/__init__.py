"""SketchSSM decode path for NVIDIA B200 (sm_100a): a C-ABI CUDA library
(libsketchssm.so, include/sketchssm.h) and its Python binding.

The CUDA library is the only implementation; nothing here falls back to a
CPU or PyTorch path.
"""
from . import binding, synth  # noqa: F401
from .binding import (SS_BF16, SS_F32, SS_GDN, SS_KDA, SS_MAMBA2, Plan, SSError,  # noqa: F401
                      ss_buffer_sizes, ss_create, ss_decode_step, ss_exact_step, ss_flush,
                      ss_get_phase, ss_launch_count, ss_prime, ss_replay_step, ss_set_phase,
                      ss_traffic_bytes)
from .layer import DecodeLayer  # noqa: F401

"""B200-native training step (forward + backward to parameter gradients) of a nanochat-style GPT.

The step runs in hand-written sm_100a CUDA kernels behind the C ABI of ``libgptstep.so``
(declared in ``include/gptstep.h``).  ``gpt_decoder_pretraining_b200.step`` is the thin ctypes
binding; ``config`` holds the presets and FLOP arithmetic; ``inputs`` the seeded synthetic inputs.
The native library is loaded lazily, so the config/inputs modules import without a GPU.
"""
from .config import GptConfig, preset, custom, PRESETS  # noqa: F401

__all__ = ["GptConfig", "preset", "custom", "PRESETS"]

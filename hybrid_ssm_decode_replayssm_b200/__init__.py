"""ReplaySSM decode hot path for NVIDIA B200 (sm_100a).

The compute lives in librssm.so (hand-written CUDA, C ABI in include/rssm.h);
``rssm`` is its ctypes binding.  Build the library with
``python -m hybrid_ssm_decode_replayssm_b200.build``.
"""
from .rssm import (  # noqa: F401
    RSSM_BF16, RSSM_F32, RSSM_GDN, RSSM_MAMBA2, RSSM_READ_FP8_E4M3_ROW, RSSM_READ_FP32,
    RSSM_READ_NVFP4, RSSMError, ReplayLayer, lib, make_desc, workspace_size,
)

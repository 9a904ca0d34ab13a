"""B200 (sm_100a) OneTrans block-stack forward.

The compute lives in ``libonetrans.so`` (hand-written CUDA: tcgen05 / TMEM /
TMA GEMMs and attention, CUDA-core fp32 kernels); this package only binds it.
Build it with ``python -m unified_transformer_recommender_onetrans_b200.build``.
"""

from .binding import (  # noqa: F401
    GRAD_NAMES,
    LIB_PATH,
    SIGNATURES,
    Model,
    OtError,
    backward_launches,
    backward_workspace_bytes,
    embed_gather,
    full_backward,
    lib,
    make_config,
    pyramid_schedule,
)

"""CODA GEMM + epilogue hot path for NVIDIA B200 (sm_100a).

The compute lives in libcoda.so (C ABI, include/coda.h), built in-tree by
``python -m gemm_epilogue_transformer_02_b200.build``.  ``binding`` is the thin
ctypes layer over it; ``synth`` draws the seeded synthetic inputs.
"""
from . import binding  # noqa: F401
from .binding import (  # noqa: F401
    CodaError,
    block_backward,
    gemm_res_partialrms,
    gemm_res_partialrms_bwd,
    gemm_rmsnorm_gemm,
    gemm_rowscale,
    gemm_rowscale_bwd,
    gemm_swiglu,
    lmhead_ce,
    load_library,
    partial_cols,
    poll_status,
    rms_reduce,
    rms_reduce_bwd,
    swiglu_down,
    unfused_block,
)

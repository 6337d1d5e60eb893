"""grouped_nf4_w4a16_b200 -- grouped MoE expert GEMM on NF4-packed weights, B200.

The compute lives in ``libgnf4.so`` (hand-written CUDA for sm_100a, C ABI in
``include/gnf4.h``). This package is a thin ctypes binding with the same entry
point names; it only marshals arguments (tensor -> pointer, current stream).
There is no CPU or PyTorch fallback: without the built library every entry
point raises.
"""
from .binding import (  # noqa: F401
    Gnf4Error,
    GNF4_OK,
    GNF4_EPI_NONE,
    GNF4_EPI_SWIGLU,
    GNF4_EPI_SWIGLU_INTERLEAVED,
    GNF4_FMT_NF4,
    GNF4_FMT_MXFP4,
    GNF4_SCALE_F32,
    GNF4_SCALE_BF16,
    GNF4_SCALE_E8M0,
    GemmDesc,
    GNF4_MODE_AUTO,
    GNF4_MODE_DECODE,
    GNF4_MODE_PREFILL,
    GNF4_OUT_F32,
    GNF4_OUT_BF16,
    GNF4_OP_MOE_ALIGN,
    GNF4_OP_GROUPED_GEMM,
    GNF4_OP_MOE_COMBINE,
    GNF4_OP_GROUPED_DGRAD,
    GNF4_MAX_TOPK,
    DEVERR_BITS,
    EXPORTED_SYMBOLS,
    library_path,
    load_library,
    gnf4_version,
    gnf4_status_string,
    gnf4_workspace_bytes,
    gnf4_moe_align,
    gnf4_grouped_gemm,
    gnf4_grouped_gemm_noalloc,
    gnf4_grouped_gemm_ex,
    gnf4_router_topk,
    gnf4_moe_combine,
    gnf4_grouped_dgrad,
    GNF4_NOALLOC_SCRATCH_BYTES,
    gnf4_dequant_debug,
    gnf4_read_device_status,
    make_workspace,
)

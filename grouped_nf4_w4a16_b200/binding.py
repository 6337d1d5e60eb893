"""ctypes binding of libgnf4 (argument marshalling only; see include/gnf4.h).

Every function here turns tensors into device pointers, picks the current CUDA
stream and calls the C entry point of the same name; every step of the
computation runs in the library's kernels. Tensors must already be on the
GPU: the library refuses host memory (GNF4_ERR_HOST_POINTER) and this module
never copies on the caller's behalf.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgnf4.so")

GNF4_OK = 0
_STATUS_NAMES = {
    0: "GNF4_OK", 1: "GNF4_ERR_INVALID_ARGUMENT", 2: "GNF4_ERR_HOST_POINTER",
    3: "GNF4_ERR_UNSUPPORTED_SHAPE", 4: "GNF4_ERR_WORKSPACE_TOO_SMALL", 5: "GNF4_ERR_CUDA",
    6: "GNF4_ERR_DEVICE_METADATA", 7: "GNF4_ERR_TIMEOUT", 8: "GNF4_ERR_MISALIGNED",
    9: "GNF4_ERR_SCRATCH_LIMIT",
}
GNF4_NOALLOC_SCRATCH_BYTES = 8 << 20
GNF4_EPI_NONE, GNF4_EPI_SWIGLU, GNF4_EPI_SWIGLU_INTERLEAVED = 0, 1, 2
GNF4_FMT_NF4, GNF4_FMT_MXFP4 = 0, 1
GNF4_SCALE_F32, GNF4_SCALE_BF16, GNF4_SCALE_E8M0 = 0, 1, 2
GNF4_MODE_AUTO, GNF4_MODE_DECODE, GNF4_MODE_PREFILL = 0, 1, 2
GNF4_OUT_F32, GNF4_OUT_BF16 = 0, 1
GNF4_OP_MOE_ALIGN, GNF4_OP_GROUPED_GEMM, GNF4_OP_MOE_COMBINE, GNF4_OP_GROUPED_DGRAD = 0, 1, 2, 3
GNF4_MAX_TOPK = 32
DEVERR_BITS = {"sizes": 0x1, "expert": 0x2, "topk": 0x4, "timeout": 0x8, "capacity": 0x10,
               "slot": 0x20}

# Every symbol include/gnf4.h declares.
EXPORTED_SYMBOLS = (
    "gnf4_moe_align", "gnf4_grouped_gemm", "gnf4_dequant_debug", "gnf4_workspace_bytes",
    "gnf4_read_device_status", "gnf4_status_string", "gnf4_version",
    "gnf4_grouped_gemm_noalloc", "gnf4_router_topk", "gnf4_moe_combine", "gnf4_grouped_dgrad",
    "gnf4_grouped_gemm_ex",
)


class GemmDesc(ctypes.Structure):
    """gnf4_gemm_desc of include/gnf4.h, field for field."""
    _fields_ = [
        ("struct_bytes", ctypes.c_uint32), ("format", ctypes.c_int32),
        ("scale_dtype", ctypes.c_int32), ("epilogue", ctypes.c_int32),
        ("swiglu_alpha", ctypes.c_float), ("swiglu_limit", ctypes.c_float),
        ("mode", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("x", ctypes.c_void_p), ("hidden", ctypes.c_void_p), ("sorted_idx", ctypes.c_void_p),
        ("n_tokens", ctypes.c_int64), ("w", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("sizes", ctypes.c_void_p), ("expert_ids", ctypes.c_void_p),
        ("G", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("E", ctypes.c_int32),
        ("M", ctypes.c_int64), ("y", ctypes.c_void_p),
    ]

_lib = None


class Gnf4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libgnf4.so; raise if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m grouped_nf4_w4a16_b200.build` "
            "(this package has no CPU or PyTorch fallback)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.gnf4_moe_align.argtypes = [P, i64, i32, i32, P, P, P, P, P, sz, P]
    lib.gnf4_moe_align.restype = ctypes.c_int
    lib.gnf4_grouped_gemm.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, i32, i32, i32, P,
                                      P, sz, P]
    lib.gnf4_grouped_gemm.restype = ctypes.c_int
    lib.gnf4_grouped_gemm_noalloc.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, i32, i32,
                                              P, P]
    lib.gnf4_grouped_gemm_noalloc.restype = ctypes.c_int
    lib.gnf4_dequant_debug.argtypes = [P, P, i64, i32, i32, i32, P, P]
    lib.gnf4_dequant_debug.restype = ctypes.c_int
    lib.gnf4_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32]
    lib.gnf4_workspace_bytes.restype = sz
    lib.gnf4_read_device_status.argtypes = [P, i32, ctypes.POINTER(ctypes.c_uint32), P]
    lib.gnf4_read_device_status.restype = ctypes.c_int
    lib.gnf4_status_string.argtypes = [ctypes.c_int]
    lib.gnf4_status_string.restype = ctypes.c_char_p
    lib.gnf4_version.argtypes = []
    lib.gnf4_version.restype = ctypes.c_int32
    lib.gnf4_router_topk.argtypes = [P, i64, i32, i32, i32, P, P, P]
    lib.gnf4_router_topk.restype = ctypes.c_int
    lib.gnf4_moe_combine.argtypes = [P, P, P, i64, i32, i32, P, P, sz, P]
    lib.gnf4_moe_combine.restype = ctypes.c_int
    lib.gnf4_grouped_dgrad.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, i32, P, P, sz, P]
    lib.gnf4_grouped_dgrad.restype = ctypes.c_int
    lib.gnf4_grouped_gemm_ex.argtypes = [ctypes.POINTER(GemmDesc), P, sz, P]
    lib.gnf4_grouped_gemm_ex.restype = ctypes.c_int
    _lib = lib
    return lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(st: int, where: str):
    if st != GNF4_OK:
        raise Gnf4Error(st, where)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gnf4_version() -> int:
    return int(load_library().gnf4_version())


def gnf4_status_string(status: int) -> str:
    return load_library().gnf4_status_string(int(status)).decode()


def gnf4_workspace_bytes(op: int, M: int, N: int = 1, K: int = 64, E: int = 1, G: int = 1) -> int:
    return int(load_library().gnf4_workspace_bytes(op, M, N, K, E, G))


def make_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled byte buffer usable as a workspace (zero it once, reuse it)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def gnf4_moe_align(topk_ids: torch.Tensor, E: int, *, sorted_idx=None, sizes=None,
                   expert_ids=None, num_groups=None, workspace=None, stream=None):
    """-> (sorted_idx [T*k], sizes [E], expert_ids [E], num_groups [1]) int32 device tensors."""
    _need(topk_ids, "topk_ids", torch.int32)
    T, k = topk_ids.shape
    dev = topk_ids.device
    sorted_idx = sorted_idx if sorted_idx is not None else torch.empty(T * k, dtype=torch.int32, device=dev)
    sizes = sizes if sizes is not None else torch.empty(E, dtype=torch.int32, device=dev)
    expert_ids = expert_ids if expert_ids is not None else torch.empty(E, dtype=torch.int32, device=dev)
    num_groups = num_groups if num_groups is not None else torch.empty(1, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = make_workspace(gnf4_workspace_bytes(GNF4_OP_MOE_ALIGN, T * k, E=E), dev)
    st = load_library().gnf4_moe_align(
        _ptr(topk_ids), T, k, E, _ptr(sorted_idx), _ptr(sizes), _ptr(expert_ids), _ptr(num_groups),
        _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "gnf4_moe_align")
    return sorted_idx, sizes, expert_ids, num_groups


def gnf4_grouped_gemm(x: torch.Tensor, w: torch.Tensor, absmax: torch.Tensor, sizes: torch.Tensor,
                      expert_ids: torch.Tensor, *, epilogue: int = GNF4_EPI_NONE,
                      mode: int = GNF4_MODE_AUTO, y: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, blocksize: int = 64,
                      stream=None) -> torch.Tensor:
    """y = grouped NF4 GEMM of x [M,K] bf16 with w [E,N,K/2] uint8 / absmax [E,N,K/64] fp32."""
    _need(x, "x", torch.bfloat16)
    _need(w, "w", torch.uint8)
    _need(absmax, "absmax", torch.float32)
    _need(sizes, "sizes", torch.int32)
    _need(expert_ids, "expert_ids", torch.int32)
    M, K = x.shape
    E, N, Kh = w.shape
    if Kh * 2 != K:
        raise ValueError(f"w has K/2={Kh} but x has K={K}")
    G = sizes.numel()
    n_out = N // 2 if epilogue == GNF4_EPI_SWIGLU else N
    if y is None:
        y = torch.empty((M, n_out), dtype=torch.bfloat16, device=x.device)
    else:
        _need(y, "y", torch.bfloat16)
    if workspace is None:
        workspace = make_workspace(gnf4_workspace_bytes(GNF4_OP_GROUPED_GEMM, M, N, K, E, G), x.device)
    st = load_library().gnf4_grouped_gemm(
        _ptr(x), _ptr(w), _ptr(absmax), _ptr(sizes), _ptr(expert_ids), G, M, N, K, E, blocksize,
        epilogue, mode, _ptr(y), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "gnf4_grouped_gemm")
    return y


def gnf4_grouped_gemm_ex(w: torch.Tensor, scales: torch.Tensor, sizes: torch.Tensor,
                         expert_ids: torch.Tensor, *, x: Optional[torch.Tensor] = None,
                         hidden: Optional[torch.Tensor] = None,
                         sorted_idx: Optional[torch.Tensor] = None, top_k: int = 1,
                         M: Optional[int] = None, fmt: int = GNF4_FMT_NF4,
                         epilogue: int = GNF4_EPI_NONE, swiglu_alpha: float = 1.702,
                         swiglu_limit: float = 7.0, mode: int = GNF4_MODE_AUTO,
                         y: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """gnf4_grouped_gemm_ex: the grouped GEMM over NF4 (scales = fp32 or bf16
    absmax [E,N,K/64]) or MXFP4 (fmt=GNF4_FMT_MXFP4, scales = e8m0 uint8
    [E,N,K/32]), rows from x [M,K] or gathered as hidden[sorted_idx[i] //
    top_k] (x=None; M = number of rows, default sorted_idx.numel())."""
    _need(w, "w", torch.uint8)
    _need(sizes, "sizes", torch.int32)
    _need(expert_ids, "expert_ids", torch.int32)
    if fmt == GNF4_FMT_MXFP4:
        _need(scales, "scales", torch.uint8)
        sdt = GNF4_SCALE_E8M0
    elif scales.dtype == torch.bfloat16:
        _need(scales, "scales", torch.bfloat16)
        sdt = GNF4_SCALE_BF16
    else:
        _need(scales, "scales", torch.float32)
        sdt = GNF4_SCALE_F32
    E, N, Kh = w.shape
    K = 2 * Kh
    if x is not None:
        _need(x, "x", torch.bfloat16)
        if hidden is not None:
            raise ValueError("pass x or hidden, not both")
        M = x.shape[0]
        dev = x.device
    else:
        if hidden is None or sorted_idx is None:
            raise ValueError("gathering needs hidden and sorted_idx")
        _need(hidden, "hidden", torch.bfloat16)
        _need(sorted_idx, "sorted_idx", torch.int32)
        M = sorted_idx.numel() if M is None else int(M)
        dev = hidden.device
    G = sizes.numel()
    n_out = N // 2 if epilogue != GNF4_EPI_NONE else N
    if y is None:
        y = torch.empty((M, n_out), dtype=torch.bfloat16, device=dev)
    else:
        _need(y, "y", torch.bfloat16)
    if workspace is None:
        workspace = make_workspace(gnf4_workspace_bytes(GNF4_OP_GROUPED_GEMM, M, N, K, E, G), dev)
    d = GemmDesc()
    d.struct_bytes = ctypes.sizeof(GemmDesc)
    d.format, d.scale_dtype, d.epilogue = fmt, sdt, epilogue
    d.swiglu_alpha, d.swiglu_limit = swiglu_alpha, swiglu_limit
    d.mode, d.top_k = mode, top_k
    d.x = _ptr(x)
    d.hidden = _ptr(hidden) if x is None else None
    d.sorted_idx = _ptr(sorted_idx) if x is None else None
    d.n_tokens = hidden.shape[0] if x is None else 0
    d.w, d.scales, d.sizes, d.expert_ids = _ptr(w), _ptr(scales), _ptr(sizes), _ptr(expert_ids)
    d.G, d.N, d.K, d.E, d.M = G, N, K, E, M
    d.y = _ptr(y)
    st = load_library().gnf4_grouped_gemm_ex(ctypes.byref(d), _ptr(workspace), workspace.numel(),
                                             _stream(stream))
    _check(st, "gnf4_grouped_gemm_ex")
    return y


def gnf4_grouped_gemm_noalloc(x: torch.Tensor, w: torch.Tensor, absmax: torch.Tensor,
                              sizes: torch.Tensor, expert_ids: torch.Tensor, *,
                              epilogue: int = GNF4_EPI_NONE, y: Optional[torch.Tensor] = None,
                              blocksize: int = 64, stream=None) -> torch.Tensor:
    """The decode grouped GEMM without a workspace argument.

    For callers that must not allocate device memory: the library uses its own
    fixed scratch array (GNF4_NOALLOC_SCRATCH_BYTES per GPU). Calls must not
    overlap on the GPU; problems larger than the scratch raise
    GNF4_ERR_SCRATCH_LIMIT. Pass `y` to avoid the output allocation here.
    """
    _need(x, "x", torch.bfloat16)
    _need(w, "w", torch.uint8)
    _need(absmax, "absmax", torch.float32)
    _need(sizes, "sizes", torch.int32)
    _need(expert_ids, "expert_ids", torch.int32)
    M, K = x.shape
    E, N, Kh = w.shape
    if Kh * 2 != K:
        raise ValueError(f"w has K/2={Kh} but x has K={K}")
    n_out = N // 2 if epilogue == GNF4_EPI_SWIGLU else N
    if y is None:
        y = torch.empty((M, n_out), dtype=torch.bfloat16, device=x.device)
    else:
        _need(y, "y", torch.bfloat16)
    st = load_library().gnf4_grouped_gemm_noalloc(
        _ptr(x), _ptr(w), _ptr(absmax), _ptr(sizes), _ptr(expert_ids), sizes.numel(), M, N, K, E,
        blocksize, epilogue, _ptr(y), _stream(stream))
    _check(st, "gnf4_grouped_gemm_noalloc")
    return y


def gnf4_dequant_debug(w: torch.Tensor, absmax: torch.Tensor, out_dtype: int = GNF4_OUT_F32, *,
                       out: Optional[torch.Tensor] = None, blocksize: int = 64,
                       stream=None) -> torch.Tensor:
    """NF4[code] * absmax for every element: fp32 (or bf16) [..., K]."""
    _need(w, "w", torch.uint8)
    _need(absmax, "absmax", torch.float32)
    K = w.shape[-1] * 2
    rows = w.numel() // w.shape[-1] if w.numel() else 0
    dt = torch.bfloat16 if out_dtype == GNF4_OUT_BF16 else torch.float32
    if out is None:
        out = torch.empty(tuple(w.shape[:-1]) + (K,), dtype=dt, device=w.device)
    st = load_library().gnf4_dequant_debug(_ptr(w), _ptr(absmax), rows, K, blocksize, out_dtype,
                                           _ptr(out), _stream(stream))
    _check(st, "gnf4_dequant_debug")
    return out


def gnf4_grouped_dgrad(dy: torch.Tensor, w: torch.Tensor, absmax: torch.Tensor,
                       sizes: torch.Tensor, expert_ids: torch.Tensor, *,
                       dx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       blocksize: int = 64, stream=None) -> torch.Tensor:
    """dx bf16 [M, K] = grouped dy [M, N] bf16 . W (w [E,N,K/2] uint8, absmax [E,N,K/64] fp32)."""
    _need(dy, "dy", torch.bfloat16)
    _need(w, "w", torch.uint8)
    _need(absmax, "absmax", torch.float32)
    _need(sizes, "sizes", torch.int32)
    _need(expert_ids, "expert_ids", torch.int32)
    M, N = dy.shape
    E, Nw, Kh = w.shape
    if Nw != N:
        raise ValueError(f"w has N={Nw} but dy has N={N}")
    K = 2 * Kh
    G = sizes.numel()
    if dx is None:
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dy.device)
    else:
        _need(dx, "dx", torch.bfloat16)
    if workspace is None:
        workspace = make_workspace(gnf4_workspace_bytes(GNF4_OP_GROUPED_DGRAD, M, N, K, E, G),
                                   dy.device)
    st = load_library().gnf4_grouped_dgrad(
        _ptr(dy), _ptr(w), _ptr(absmax), _ptr(sizes), _ptr(expert_ids), G, M, N, K, E, blocksize,
        _ptr(dx), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "gnf4_grouped_dgrad")
    return dx


def gnf4_router_topk(logits: torch.Tensor, top_k: int, *, renormalize: bool = True,
                     topk_ids=None, topk_weights=None, stream=None):
    """-> (topk_ids int32 [T, top_k], topk_weights fp32 [T, top_k]) from fp32 logits [T, E]."""
    _need(logits, "logits", torch.float32)
    T, E = logits.shape
    dev = logits.device
    topk_ids = topk_ids if topk_ids is not None else torch.empty((T, top_k), dtype=torch.int32,
                                                                 device=dev)
    topk_weights = (topk_weights if topk_weights is not None
                    else torch.empty((T, top_k), dtype=torch.float32, device=dev))
    st = load_library().gnf4_router_topk(_ptr(logits), T, E, top_k, 1 if renormalize else 0,
                                         _ptr(topk_ids), _ptr(topk_weights), _stream(stream))
    _check(st, "gnf4_router_topk")
    return topk_ids, topk_weights


def gnf4_moe_combine(y: torch.Tensor, sorted_idx: torch.Tensor, topk_weights: torch.Tensor, *,
                     out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """out bf16 [T, H] = top-k weighted sum of the rows of y bf16 [T*top_k, H] (sorted order)."""
    _need(y, "y", torch.bfloat16)
    _need(sorted_idx, "sorted_idx", torch.int32)
    _need(topk_weights, "topk_weights", torch.float32)
    T, k = topk_weights.shape
    H = y.shape[1]
    if y.shape[0] != T * k or sorted_idx.numel() != T * k:
        raise ValueError(f"y has {y.shape[0]} rows and sorted_idx {sorted_idx.numel()} entries; "
                         f"expected T*top_k = {T * k}")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    else:
        _need(out, "out", torch.bfloat16)
    if workspace is None:
        workspace = make_workspace(gnf4_workspace_bytes(GNF4_OP_MOE_COMBINE, T * k), y.device)
    st = load_library().gnf4_moe_combine(_ptr(y), _ptr(sorted_idx), _ptr(topk_weights), T, k, H,
                                         _ptr(out), _ptr(workspace), workspace.numel(),
                                         _stream(stream))
    _check(st, "gnf4_moe_combine")
    return out


def gnf4_read_device_status(workspace: torch.Tensor, clear: bool = True,
                            stream=None) -> Tuple[int, int]:
    """Synchronise and read the workspace error word -> (status, GNF4_DEVERR bits)."""
    bits = ctypes.c_uint32(0)
    st = load_library().gnf4_read_device_status(_ptr(workspace), 1 if clear else 0,
                                                ctypes.byref(bits), _stream(stream))
    return int(st), int(bits.value)

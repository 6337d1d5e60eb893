"""C ABI of libgnf4 on the CPU: the library loads, exports every symbol that
include/gnf4.h declares, and its host-side argument checks return the
documented status codes before touching the GPU."""
import ctypes
import os
import re

import pytest

import grouped_nf4_w4a16_b200 as gnf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gnf4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gnf4_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(gnf4.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = gnf4.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    raw = ctypes.CDLL(gnf4.library_path())
    for name in declared_functions():
        assert ctypes.cast(getattr(raw, name), ctypes.c_void_p).value


def test_version_and_status_strings():
    assert gnf4.gnf4_version() == 120
    assert gnf4.gnf4_status_string(0) == "GNF4_OK"
    assert "HOST_POINTER" in gnf4.gnf4_status_string(2)
    assert gnf4.gnf4_status_string(99) == "GNF4_ERR_UNKNOWN"


def test_workspace_sizes_are_positive_and_monotone():
    a = gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_ALIGN, 16, E=4)
    assert a >= 256
    s1 = gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, 16, 128, 256, 4, 4)
    s2 = gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, 256, 5760, 2880, 128, 128)
    assert 256 <= s1 <= s2
    assert gnf4.gnf4_workspace_bytes(7, 16, 128, 256, 4, 4) == 0


def _gemm(lib, **kw):
    args = dict(x=1, w=1, absmax=1, sizes=1, expert_ids=1, G=4, M=16, N=128, K=256, E=4,
                blocksize=64, epi=0, mode=0, y=1, ws=1, ws_bytes=1 << 20, stream=None)
    args.update(kw)
    return lib.gnf4_grouped_gemm(args["x"], args["w"], args["absmax"], args["sizes"],
                                 args["expert_ids"], args["G"], args["M"], args["N"], args["K"],
                                 args["E"], args["blocksize"], args["epi"], args["mode"], args["y"],
                                 args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), 1), (dict(y=None), 1), (dict(ws=None), 1),
    (dict(M=-1), 1), (dict(N=0), 1), (dict(E=0), 1), (dict(G=0), 1),
    (dict(epi=5), 1), (dict(mode=9), 1),
    (dict(blocksize=32), 3), (dict(K=96), 3), (dict(E=2000), 3), (dict(G=2000), 3),
    (dict(epi=1, N=127), 3),
    (dict(M=0), 0),
])
def test_grouped_gemm_host_checks(kw, status):
    assert _gemm(gnf4.load_library(), **kw) == status


def test_moe_align_and_dequant_host_checks():
    lib = gnf4.load_library()
    assert lib.gnf4_moe_align(None, 8, 2, 4, 1, 1, 1, 1, 1, 256, None) == 1
    assert lib.gnf4_moe_align(1, 8, 0, 4, 1, 1, 1, 1, 1, 256, None) == 1
    assert lib.gnf4_moe_align(1, 8, 2, 4096, 1, 1, 1, 1, 1, 256, None) == 3
    assert lib.gnf4_moe_align(1, 8, 2, 4, 1, 1, 1, 1, 1, 16, None) == 4
    assert lib.gnf4_dequant_debug(None, 1, 4, 64, 64, 0, 1, None) == 1
    assert lib.gnf4_dequant_debug(1, 1, 4, 96, 64, 0, 1, None) == 3
    assert lib.gnf4_dequant_debug(1, 1, 4, 64, 64, 7, 1, None) == 1
    assert lib.gnf4_dequant_debug(1, 1, 0, 64, 64, 0, 1, None) == 0


def test_router_topk_and_combine_host_checks():
    lib = gnf4.load_library()
    # gnf4_router_topk(logits, T, E, top_k, renormalize, ids, weights, stream)
    assert lib.gnf4_router_topk(1, -1, 8, 2, 1, 1, 1, None) == 1
    assert lib.gnf4_router_topk(1, 4, 8, 0, 1, 1, 1, None) == 1
    assert lib.gnf4_router_topk(1, 4, 8, 2, 2, 1, 1, None) == 1
    assert lib.gnf4_router_topk(1, 4, 8, 9, 1, 1, 1, None) == 3       # top_k > E
    assert lib.gnf4_router_topk(1, 4, 64, 33, 1, 1, 1, None) == 3     # top_k > GNF4_MAX_TOPK
    assert lib.gnf4_router_topk(1, 4, 2048, 2, 1, 1, 1, None) == 3    # E > GNF4_MAX_EXPERTS
    assert lib.gnf4_router_topk(None, 0, 8, 2, 1, None, None, None) == 0
    assert lib.gnf4_router_topk(None, 4, 8, 2, 1, 1, 1, None) == 1
    # gnf4_moe_combine(y, sorted_idx, weights, T, top_k, H, out, ws, ws_bytes, stream)
    ws = gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_COMBINE, 8)
    assert ws >= 256 + 8 * 4
    assert lib.gnf4_moe_combine(1, 1, 1, -1, 2, 64, 1, 1, ws, None) == 1
    assert lib.gnf4_moe_combine(1, 1, 1, 4, 2, 0, 1, 1, ws, None) == 1
    assert lib.gnf4_moe_combine(1, 1, 1, 4, 33, 64, 1, 1, 1 << 20, None) == 3
    assert lib.gnf4_moe_combine(None, None, None, 0, 2, 64, None, None, 0, None) == 0
    assert lib.gnf4_moe_combine(None, 1, 1, 4, 2, 64, 1, 1, ws, None) == 1
    assert lib.gnf4_moe_combine(1, 1, 1, 4, 2, 64, 1, 1, ws - 1, None) == 4


def test_grouped_dgrad_host_checks():
    lib = gnf4.load_library()

    def dg(**kw):
        a = dict(dy=1, w=1, absmax=1, sizes=1, ids=1, G=2, M=8, N=16, K=128, E=2, bs=64, dx=1,
                 ws=1, ws_bytes=256)
        a.update(kw)
        return lib.gnf4_grouped_dgrad(a["dy"], a["w"], a["absmax"], a["sizes"], a["ids"], a["G"],
                                      a["M"], a["N"], a["K"], a["E"], a["bs"], a["dx"], a["ws"],
                                      a["ws_bytes"], None)
    assert dg(dy=None) == 1 and dg(dx=None) == 1 and dg(M=-1) == 1 and dg(G=0) == 1
    assert dg(K=96) == 3 and dg(bs=32) == 3 and dg(E=2000) == 3
    assert dg(ws_bytes=16) == 4
    assert dg(N=12) == 3                                 # the tensor-core dgrad needs N % 8 == 0
    need = gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_DGRAD, 8, 16, 128, 2, 2)
    assert need > 256                                    # header + split counters and partials
    assert dg(ws_bytes=need - 1) == 4
    assert dg(M=0, ws_bytes=need) == 0


def test_host_buffers_are_refused():
    # Host memory is refused with GNF4_ERR_HOST_POINTER (no host path exists).
    buf = (ctypes.c_uint8 * (1 << 16))()
    p = ctypes.addressof(buf)
    assert _gemm(gnf4.load_library(), x=p, w=p, absmax=p, sizes=p, expert_ids=p, y=p, ws=p) == 2
    assert gnf4.load_library().gnf4_dequant_debug(p, p, 4, 64, 64, 0, p, None) == 2
    assert gnf4.load_library().gnf4_router_topk(p, 4, 8, 2, 1, p, p, None) == 2
    assert gnf4.load_library().gnf4_moe_combine(p, p, p, 4, 2, 64, p, p, 1 << 12, None) == 2
    assert gnf4.load_library().gnf4_grouped_dgrad(p, p, p, p, p, 1, 4, 8, 64, 1, 64, p, p,
                                                  1 << 30, None) == 2


def test_grouped_gemm_ex_host_checks():
    # The descriptor entry point refuses bad descriptors before any launch
    # (fake device pointers: every case fails before they are dereferenced).
    import ctypes
    lib = gnf4.load_library()

    def desc(**kw):
        d = gnf4.GemmDesc()
        d.struct_bytes = ctypes.sizeof(gnf4.GemmDesc)
        d.format, d.scale_dtype, d.epilogue = gnf4.GNF4_FMT_NF4, gnf4.GNF4_SCALE_F32, 0
        d.swiglu_alpha, d.swiglu_limit, d.mode, d.top_k = 1.702, 7.0, 0, 1
        d.x, d.w, d.scales, d.sizes, d.expert_ids, d.y = 64, 64, 64, 64, 64, 64
        d.G, d.N, d.K, d.E, d.M = 1, 8, 64, 1, 1
        for k, v in kw.items():
            setattr(d, k, v)
        return d

    def call(d):
        return lib.gnf4_grouped_gemm_ex(ctypes.byref(d), 64, 1 << 20, None)

    assert call(desc(struct_bytes=8)) == 1                       # wrong struct size
    assert call(desc(format=2)) == 1                             # unknown format
    assert call(desc(scale_dtype=gnf4.GNF4_SCALE_E8M0)) == 1     # NF4 with e8m0 scales
    assert call(desc(format=gnf4.GNF4_FMT_MXFP4)) == 1           # MXFP4 with fp32 scales
    assert call(desc(epilogue=3)) == 1
    assert call(desc(epilogue=2, swiglu_limit=0.0)) == 1         # the clamp needs a limit
    assert call(desc(epilogue=2, N=7)) == 3                      # odd N with SwiGLU
    assert call(desc(hidden=64)) == 1                            # x and hidden both given
    assert call(desc(x=None)) == 1                               # neither
    assert call(desc(x=None, hidden=64, sorted_idx=64, top_k=0)) == 1
    assert call(desc(K=96)) == 3                                 # K % 64
    assert call(desc(M=0)) == 0                                  # nothing to do
    assert call(desc()) == 2                                     # fake pointers: not device memory
    assert lib.gnf4_grouped_gemm_ex(None, 64, 1 << 20, None) == 1

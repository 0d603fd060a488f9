"""The C ABI loads on a machine without a GPU, exports every entry point the header
declares, and rejects bad arguments with status codes before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4_moe.h")


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_moe_nvfp4_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^NVFP4_API[^;(]*?\b(\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ("nvfp4_quantize", "nvfp4_dequantize", "moe_nvfp4_forward",
                 "moe_nvfp4_workspace_size", "moe_nvfp4_route", "nvfp4_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.nvfp4_status_string.restype = ctypes.c_char_p
    for code, word in ((0, b"OK"), (-1, b"EINVAL"), (-2, b"ESHAPE"), (-3, b"EWORKSPACE"),
                       (-4, b"ECUDA")):
        assert word in lib.nvfp4_status_string(code)


def test_workspace_queries(lib):
    lib.moe_nvfp4_workspace_size.restype = ctypes.c_size_t
    lib.moe_nvfp4_workspace_size.argtypes = [ctypes.c_int64] * 5
    small = lib.moe_nvfp4_workspace_size(1, 6144, 2048, 256, 8)
    big = lib.moe_nvfp4_workspace_size(4096, 6144, 2048, 256, 8)
    assert 0 < small < big
    # the prefill scratch: gathered x, h and the fp32 per-pair outputs dominate
    TK = 4096 * 8
    assert big >= TK * (2 * 6144 + 2 * 2048 + 4 * 6144)
    assert lib.moe_nvfp4_workspace_size(0, 6144, 2048, 256, 8) == 0


def test_workspace_zero_head(lib):
    """The workspace head that must be zero before first use (error flag and the one-token
    work counters) is the same size in the header and the Python binding, and every
    workspace holds it."""
    m = re.search(r"^#define NVFP4_WORKSPACE_ZERO_BYTES (\d+)", open(HEADER).read(), re.M)
    assert m
    import bit_quantized_moe_nvfp4_b200 as nv
    assert nv.WORKSPACE_ZERO_BYTES == int(m.group(1))
    lib.moe_nvfp4_workspace_size.restype = ctypes.c_size_t
    lib.moe_nvfp4_workspace_size.argtypes = [ctypes.c_int64] * 5
    for shape in ((1, 6144, 2048, 256, 8), (1, 64, 64, 1, 1), (37, 192, 128, 16, 4)):
        assert lib.moe_nvfp4_workspace_size(*shape) >= nv.WORKSPACE_ZERO_BYTES


def test_alloc_moe_workspace_zeroes_its_head(lib):
    """The binding's allocator returns a workspace of the queried size whose head is zero
    (host logic: checked with a CPU tensor)."""
    import bit_quantized_moe_nvfp4_b200 as nv
    ws = nv.alloc_moe_workspace(3, 192, 128, 16, 4, device="cpu")
    assert ws.numel() == nv.moe_nvfp4_workspace_size(3, 192, 128, 16, 4)
    assert int(ws[:nv.WORKSPACE_ZERO_BYTES].abs().sum()) == 0


def _fwd_argtypes(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f = lib.moe_nvfp4_forward_path
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_size_t,
                  ctypes.c_int, P]
    return f


def test_forward_argument_checks_run_before_cuda(lib):
    f = _fwd_argtypes(lib)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails its checks
    good = dict(T=1, H=6144, I=2048, E=256, K=8)

    def call(ptr=fake, ws=fake, ws_bytes=1 << 40, path=0, **over):
        d = dict(good, **over)
        return f(ptr, ptr, ptr, d["T"], d["H"], d["I"], d["E"], d["K"], ptr, ptr, ptr, ptr,
                 ptr, ptr, ptr, ws, ws_bytes, path, None)

    assert call(ptr=None) == -1            # null pointers
    assert call(T=0) == -1
    assert call(path=7) == -1
    assert call(H=6100) == -2              # not a multiple of 64
    assert call(I=2040) == -2
    assert call(K=17) == -2
    assert call(E=2048) == -2
    assert call(ws=None) == -3
    assert call(ws_bytes=16) == -3


def test_codec_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    q = lib.nvfp4_quantize
    q.restype = ctypes.c_int
    q.argtypes = [P, I64, I64, I64, P, P, P, P, ctypes.c_size_t, P]
    fake = ctypes.c_void_p(1 << 20)
    assert q(None, 1, 16, 32, fake, fake, fake, fake, 1 << 20, None) == -1
    assert q(fake, 1, 16, 48, fake, fake, fake, fake, 1 << 20, None) == -2
    assert q(fake, 1, 16, 32, fake, fake, fake, None, 0, None) == -3
    d = lib.nvfp4_dequantize
    d.restype = ctypes.c_int
    d.argtypes = [P, P, P, I64, I64, I64, P, P]
    assert d(fake, fake, fake, 1, 16, 40, fake, None) == -2
    assert d(fake, None, fake, 1, 16, 32, fake, None) == -1


def test_route_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    r = lib.moe_nvfp4_route
    r.restype = ctypes.c_int
    r.argtypes = [P, I64, I64, I64, P, P, P, P, P, P]
    fake = ctypes.c_void_p(1 << 20)
    assert r(None, 4, 2, 8, fake, fake, fake, fake, None, None) == -1
    assert r(fake, 4, 17, 8, fake, fake, fake, fake, None, None) == -2
    assert r(fake, 4, 2, 4096, fake, fake, fake, fake, None, None) == -2


def test_calibration_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    a = lib.nvfp4_amax
    a.restype = ctypes.c_int
    a.argtypes = [P, I64, I64, I64, P, ctypes.c_int, P]
    fake = ctypes.c_void_p(1 << 20)
    assert a(None, 1, 16, 32, fake, 0, None) == -1
    assert a(fake, 1, 16, 48, fake, 0, None) == -2
    assert a(fake, 0, 16, 32, fake, 0, None) == -1
    q = lib.nvfp4_quantize_with_amax
    q.restype = ctypes.c_int
    q.argtypes = [P, I64, I64, I64, P, P, P, P, P]
    assert q(fake, 1, 16, 32, None, fake, fake, fake, None) == -1
    assert q(fake, 1, 16, 40, fake, fake, fake, fake, None) == -2
    assert q(ctypes.c_void_p((1 << 20) + 8), 1, 16, 32, fake, fake, fake, fake, None) == -1


def test_expert_parallel_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f = lib.moe_nvfp4_forward_ep
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, I64, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P,
                  ctypes.c_size_t, ctypes.c_int, P]
    fake = ctypes.c_void_p(1 << 20)
    good = dict(T=1, H=6144, I=2048, E=256, K=8, G=8, r=3)

    def call(ptr=fake, out=fake, ws=fake, ws_bytes=1 << 40, **over):
        d = dict(good, **over)
        return f(ptr, ptr, ptr, d["T"], d["H"], d["I"], d["E"], d["K"], d["G"], d["r"],
                 ptr, ptr, ptr, ptr, ptr, ptr, out, ws, ws_bytes, 0, None)

    assert call(out=None) == -1
    assert call(G=0) == -1
    assert call(r=8) == -1
    assert call(r=-1) == -1
    assert call(G=300) == -1                 # more ranks than experts
    assert call(out=ctypes.c_void_p((1 << 20) + 4)) == -1   # partial not 16-byte aligned
    assert call(H=6100) == -2
    assert call(ws_bytes=16) == -3
    n = lib.moe_nvfp4_ep_local_experts
    n.restype = I64
    n.argtypes = [I64, I64, I64]
    assert [n(10, 4, r) for r in range(4)] == [3, 3, 2, 2]
    assert n(10, 4, 4) == 0 and n(0, 1, 0) == 0
    red = lib.moe_nvfp4_ep_reduce
    red.restype = ctypes.c_int
    red.argtypes = [P, I64, I64, I64, P, P]
    ptrs = (ctypes.c_void_p * 17)(*([1 << 20] * 17))
    assert red(None, 1, 4, 8, fake, None) == -1
    assert red(ptrs, 0, 4, 8, fake, None) == -1
    assert red(ptrs, 17, 4, 8, fake, None) == -2
    assert red(ptrs, 2, 4, 6, fake, None) == -2
    assert red(ptrs, 2, 4, 8, None, None) == -1
    bad = (ctypes.c_void_p * 2)(1 << 20, (1 << 20) + 8)
    assert red(bad, 2, 4, 8, fake, None) == -1          # a partial not 16-byte aligned
    assert red(ptrs, 2, 0, 8, fake, None) == 0          # no rows: nothing to enqueue


def test_router_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    r = lib.moe_nvfp4_router
    r.restype = ctypes.c_int
    r.argtypes = [P, I64, I64, I64, P, P, P]
    fake = ctypes.c_void_p(1 << 20)
    assert r(None, 4, 256, 8, fake, fake, None) == -1
    assert r(fake, 0, 256, 8, fake, fake, None) == -1
    assert r(fake, 4, 256, 0, fake, fake, None) == -1
    assert r(fake, 4, 256, 17, fake, fake, None) == -2
    assert r(fake, 4, 4, 5, fake, fake, None) == -2          # K > E
    assert r(fake, 4, 2048, 8, fake, fake, None) == -2
    assert r(ctypes.c_void_p((1 << 20) + 2), 4, 256, 8, fake, fake, None) == -1
    f = lib.moe_nvfp4_forward_logits
    f.restype = ctypes.c_int
    f.argtypes = [P, P, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P, P, P,
                  ctypes.c_size_t, ctypes.c_int, P]

    def call(logits=fake, ws_bytes=1 << 40, **over):
        d = dict(dict(T=1, H=6144, I=2048, E=256, K=8), **over)
        return f(fake, logits, d["T"], d["H"], d["I"], d["E"], d["K"], fake, fake, fake, fake,
                 fake, fake, fake, None, None, fake, ws_bytes, 0, None)

    assert call(logits=None) == -1
    assert call(E=4, K=8) == -2
    assert call(H=6100) == -2
    assert call(ws_bytes=16) == -3


def test_shared_expert_and_layer_argument_checks_run_before_cuda(lib):
    P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    wss = lib.moe_nvfp4_shared_workspace_size
    wss.restype, wss.argtypes = SZ, [I64, I64]
    assert wss(4, 2048) == 4 * 2048 * 2           # h, bf16 (a multiple of 256 already)
    assert wss(1, 64) == 256                       # rounded up to 256 bytes
    assert wss(0, 2048) == 0 and wss(4, 0) == 0
    sh = lib.moe_nvfp4_shared_expert
    sh.restype = ctypes.c_int
    sh.argtypes = [P, I64, I64, I64, P, P, P, P, P, SZ, P]

    def shared(x=fake, T=4, H=6144, Is=2048, routed=None, out=fake, ws=fake, ws_bytes=1 << 30):
        return sh(x, T, H, Is, fake, fake, routed, out, ws, ws_bytes, None)

    assert shared(x=None) == -1
    assert shared(out=None) == -1
    assert shared(T=0) == -1
    assert shared(H=6100) == -2                    # not a multiple of 64
    assert shared(Is=2000) == -2
    assert shared(H=65536 + 64) == -2
    assert shared(x=odd) == -1                     # 16-byte alignment
    assert shared(routed=ctypes.c_void_p((1 << 20) + 2)) == -1   # fp32 partial: 4 bytes
    assert shared(ws=None) == -3
    assert shared(ws_bytes=wss(4, 2048) - 1) == -3
    lws = lib.moe_nvfp4_layer_workspace_size
    lws.restype, lws.argtypes = SZ, [I64, I64, I64, I64, I64, I64]
    routed = lib.moe_nvfp4_workspace_size
    routed.restype, routed.argtypes = SZ, [I64, I64, I64, I64, I64]
    # routed workspace + the fp32 partial [T, H] + the shared expert's h
    assert lws(4, 6144, 2048, 256, 8, 2048) == \
        routed(4, 6144, 2048, 256, 8) + 4 * 6144 * 4 + wss(4, 2048)
    assert lws(4, 6144, 2048, 256, 8, 0) == 0
    lay = lib.moe_nvfp4_layer
    lay.restype = ctypes.c_int
    lay.argtypes = [P, P, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P, I64, P, P, P, P, SZ,
                    ctypes.c_int, P]

    def layer(logits=fake, ws_bytes=1 << 40, **over):
        d = dict(dict(T=4, H=6144, I=2048, E=256, K=8, Is=2048), **over)
        return lay(fake, logits, d["T"], d["H"], d["I"], d["E"], d["K"], fake, fake, fake, fake,
                   fake, fake, fake, fake, d["Is"], fake, None, None, fake, ws_bytes, 0, None)

    assert layer(logits=None) == -1
    assert layer(Is=100) == -2
    assert layer(E=4, K=8) == -2                   # the router needs K <= E
    assert layer(ws_bytes=16) == -3


def test_w4a4_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fake = ctypes.c_void_p(1 << 20)
    pr = lib.nvfp4_w4a4_prepare_scales
    pr.restype = ctypes.c_int
    pr.argtypes = [P, I64, I64, I64, I64, P, P]
    assert pr(None, 1, 128, 64, 0, fake, None) == -1
    assert pr(fake, 1, 100, 64, 0, fake, None) == -2       # rows % 128
    assert pr(fake, 1, 128, 48, 0, fake, None) == -2       # cols % 64
    assert pr(fake, 1, 256, 64, 64, fake, None) == -2      # gate rows must be half the rows
    assert pr(ctypes.c_void_p((1 << 20) + 2), 1, 128, 64, 0, fake, None) == -1
    f = lib.moe_nvfp4_forward_w4a4
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, I64, I64, I64, I64, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]

    def call(ptr=fake, ws_bytes=1 << 40, **over):
        d = dict(dict(T=4, H=6144, I=2048, E=256, K=8), **over)
        return f(ptr, ptr, ptr, d["T"], d["H"], d["I"], d["E"], d["K"], ptr, ptr, ptr, ptr,
                 ptr, ptr, ptr, fake, ws_bytes, None)

    assert call(ptr=None) == -1
    assert call(H=6208) == -2                               # H % 256
    assert call(I=2112) == -2                               # I % 256
    assert call(K=17) == -2
    assert call(ws_bytes=16) == -3
    ws = lib.moe_nvfp4_w4a4_workspace_size
    ws.restype = ctypes.c_size_t
    ws.argtypes = [I64] * 5
    lib.moe_nvfp4_workspace_size.restype = ctypes.c_size_t
    lib.moe_nvfp4_workspace_size.argtypes = [I64] * 5
    assert ws(4096, 6144, 2048, 256, 8) > lib.moe_nvfp4_workspace_size(4096, 6144, 2048, 256, 8)


def test_selftest_argument_checks_run_before_cuda(lib):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f = lib.nvfp4_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [P, ctypes.c_int, I64, P]
    fake = ctypes.c_void_p(1 << 20)
    assert f(None, 0, 1000000, None) == -1
    assert f(ctypes.c_void_p((1 << 20) + 2), 0, 1000000, None) == -1   # misaligned
    assert f(fake, 3, 1000000, None) == -1
    assert f(fake, -1, 1000000, None) == -1
    assert f(fake, 0, 0, None) == -1
    assert f(fake, 0, 2000000000, None) == -1


def test_oracle_and_product_share_no_code():
    """The product never imports, links or includes the oracle, and the oracle never
    imports or includes the product."""
    pkg = os.path.join(ROOT, "bit_quantized_moe_nvfp4_b200")
    bad_in_product = re.compile(r"^\s*(import|from)\s+oracle\b|liboracle|nvfp4_oracle", re.M)
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".cu", ".cuh", ".py", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not bad_in_product.search(text), fn
    bad_in_oracle = re.compile(
        r"^\s*(import|from)\s+bit_quantized_moe_nvfp4_b200\b|#include\s+\"[^\"]*(csrc|nvfp4_moe)",
        re.M)
    for fn in os.listdir(os.path.join(ROOT, "oracle")):
        if fn.endswith((".c", ".h", ".py")):
            text = open(os.path.join(ROOT, "oracle", fn)).read()
            assert not bad_in_oracle.search(text), fn

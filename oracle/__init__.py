"""CPU oracle for the NVFP4 routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  The oracle is the slow, plain statement of what the CUDA
library computes; it proves the library's results.  Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it.
The product path (``bit_quantized_moe_nvfp4_b200``) never imports, links or runs it,
and the two share no code: they meet only on the seeded inputs made by ``synth``.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp32 codec steps, fp64 MoE
accumulation); this module compiles it with gcc on first use and marshals numpy arrays
through ctypes.  Sources followed: page "GLM-5-NVFP4-MTP", sections "Model
Description" (NVFP4: 4-bit values, one FP8 scale per 16 elements; 256 experts, top-8)
and "What's quantized" (routed-expert gate/up/down projections only).

Pins (tests/test_oracle.py): the exhaustive E2M1 table, every E4M3 code against
torch's float8_e4m3fn, a hand-worked block, quantizer invariants, the routing
permutation against a stable sort, and the MoE against a dense brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# gcc flags: IEEE fp32/fp64 with no contraction into FMA and no fast-math, so every
# operation rounds exactly as the C source states.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall"]


def build(force: bool = False) -> str:
    """Compile liboracle.so next to the C source (gcc).  Returns its path."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            L.oracle_e2m1_value.restype = ctypes.c_double
            L.oracle_e2m1_value.argtypes = [ctypes.c_int]
            L.oracle_e4m3_value.restype = ctypes.c_double
            L.oracle_e4m3_value.argtypes = [ctypes.c_int]
            L.oracle_e2m1_encode.restype = ctypes.c_int
            L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
            L.oracle_e4m3_encode.restype = ctypes.c_int
            L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            L.oracle_bf16_round.restype = ctypes.c_uint16
            L.oracle_bf16_round.argtypes = [ctypes.c_double]
            L.oracle_global_scale.restype = ctypes.c_float
            L.oracle_global_scale.argtypes = [P, I64]
            L.oracle_nvfp4_quantize.restype = None
            L.oracle_nvfp4_quantize.argtypes = [P, I64, I64, I64, P, P, P]
            L.oracle_nvfp4_amax.restype = None
            L.oracle_nvfp4_amax.argtypes = [P, I64, I64, P, ctypes.c_int]
            L.oracle_nvfp4_quantize_with_amax.restype = None
            L.oracle_nvfp4_quantize_with_amax.argtypes = [P, I64, I64, I64, P, P, P, P]
            L.oracle_nvfp4_dequantize.restype = None
            L.oracle_nvfp4_dequantize.argtypes = [P, P, P, I64, I64, I64, P]
            L.oracle_route.restype = I64
            L.oracle_route.argtypes = [P, I64, I64, I64, P, P, P, P]
            L.oracle_moe_forward_w4a4.restype = I64
            L.oracle_moe_forward_w4a4.argtypes = [P, P, P, I64, I64, I64, I64, I64,
                                                  P, P, P, P, P, P, P, I64, P, P]
            L.oracle_shared_expert.restype = None
            L.oracle_shared_expert.argtypes = [P, I64, I64, P, P, P, I64, P]
            L.oracle_bf16_round_array.restype = None
            L.oracle_bf16_round_array.argtypes = [P, I64, P]
            L.oracle_router.restype = None
            L.oracle_router.argtypes = [P, I64, I64, I64, P, P]
            L.oracle_moe_forward.restype = I64
            L.oracle_moe_forward.argtypes = [P, P, P, I64, I64, I64, I64, I64,
                                             P, P, P, P, P, P, P, I64, P, P]
            L.oracle_threads.restype = ctypes.c_int
            L.oracle_threads.argtypes = []
            L.oracle_set_threads.restype = None
            L.oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 numpy array (accepts torch bf16 tensors)."""
    if hasattr(a, "detach"):
        import torch
        a = a.detach().to("cpu").contiguous().view(torch.int16).numpy()
    return np.ascontiguousarray(a).view(np.uint16)


def _np(a, dtype) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").contiguous().numpy()
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(int(code))


def e2m1_encode(v: float) -> int:
    return _load().oracle_e2m1_encode(float(v))


def e4m3_encode(v: float) -> int:
    return _load().oracle_e4m3_encode(float(v))


def bf16_round(v: float) -> int:
    """bf16 bits of the nearest bf16 to v (one rounding from the fp64 value)."""
    return int(_load().oracle_bf16_round(float(v)))


def threads() -> int:
    return int(_load().oracle_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


# ----------------------------------------------------------------------------- codec
def global_scale(x) -> float:
    xs = _u16(x).reshape(-1)
    return float(_load().oracle_global_scale(_p(xs), xs.size))


def quantize(x):
    """x: bf16 [n, rows, cols] (or [rows, cols]) -> (packed u8 [n,rows,cols/2],
    scales u8 [n,rows,cols/16], g fp32 [n])."""
    xs = _u16(x)
    if xs.ndim == 2:
        xs = xs[None]
    n, rows, cols = xs.shape
    assert cols % 16 == 0
    packed = np.zeros((n, rows, cols // 2), np.uint8)
    scales = np.zeros((n, rows, cols // 16), np.uint8)
    g = np.zeros((n,), np.float32)
    _load().oracle_nvfp4_quantize(_p(xs), n, rows, cols, _p(packed), _p(scales), _p(g))
    return packed, scales, g


def amax(x, out=None, merge: bool = False):
    """Per-tensor max |x| of bf16 [n, rows, cols] (or [rows, cols]) -> fp32 [n].  With
    merge=True, `out` holds the amax of earlier calibration passes and becomes the
    element-wise max of it and this pass's (page "GLM-5-NVFP4-MTP", "Calibration dataset")."""
    xs = _u16(x)
    if xs.ndim == 2:
        xs = xs[None]
    n = xs.shape[0]
    per = xs.shape[1] * xs.shape[2]
    if out is None:
        out = np.zeros((n,), np.float32)
    assert out.dtype == np.float32 and out.shape == (n,)
    _load().oracle_nvfp4_amax(_p(xs), n, per, _p(out), int(bool(merge)))
    return out


def quantize_with_amax(x, amax_in):
    """quantize() with the given per-tensor amax (e.g. a calibrated one) in place of each
    tensor's own: g = amax / 2688 (1 for 0).  -> (packed, scales, g)."""
    xs = _u16(x)
    if xs.ndim == 2:
        xs = xs[None]
    n, rows, cols = xs.shape
    assert cols % 16 == 0
    am = _np(amax_in, np.float32).reshape(-1)
    assert am.shape == (n,)
    packed = np.zeros((n, rows, cols // 2), np.uint8)
    scales = np.zeros((n, rows, cols // 16), np.uint8)
    g = np.zeros((n,), np.float32)
    _load().oracle_nvfp4_quantize_with_amax(_p(xs), n, rows, cols, _p(am), _p(packed),
                                            _p(scales), _p(g))
    return packed, scales, g


def dequantize(packed, scales, g):
    """-> bf16 bits as uint16 [n, rows, cols]."""
    pk = _np(packed, np.uint8)
    sc = _np(scales, np.uint8)
    gs = _np(g, np.float32).reshape(-1)
    if pk.ndim == 2:
        pk, sc = pk[None], sc[None]
    n, rows, half = pk.shape
    cols = half * 2
    out = np.zeros((n, rows, cols), np.uint16)
    _load().oracle_nvfp4_dequantize(_p(pk), _p(sc), _p(gs), n, rows, cols, _p(out))
    return out


# ----------------------------------------------------------------------------- routing
def route(ids, E: int):
    """ids int32 [T, K] -> (counts [E], offsets [E+1], perm [n_valid], inv [T*K], n_bad)."""
    a = _np(ids, np.int32)
    T, K = a.shape
    counts = np.zeros((E,), np.int32)
    offsets = np.zeros((E + 1,), np.int32)
    perm = np.zeros((T * K,), np.int32)
    inv = np.zeros((T * K,), np.int32)
    bad = _load().oracle_route(_p(a), T, K, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm[: offsets[E]], inv, int(bad)


def router(logits, K: int):
    """Router decisions from fp32 logits [T, E]: (ids int32 [T, K], w fp64 [T, K])."""
    a = _np(logits, np.float32)
    T, E = a.shape
    if not 1 <= K <= E:
        raise ValueError(f"K={K} outside 1..{E}")
    ids = np.zeros((T, K), np.int32)
    w = np.zeros((T, K), np.float64)
    _load().oracle_router(_p(a), T, E, K, _p(ids), _p(w))
    return ids, w


# ----------------------------------------------------------------------------- MoE
def moe_forward(x, ids, w, w_gu, s_gu, g_gu, w_dn, s_dn, g_dn, tokens=None, w4a4=False):
    """Routed-expert MoE forward for the listed tokens (all when tokens is None).

    x bf16 [T,H]; ids int32 [T,K]; w fp32 [T,K]; w_gu u8 [E,2I,H/2]; s_gu u8 [E,2I,H/16];
    g_gu fp32 [E]; w_dn u8 [E,H,I/2]; s_dn u8 [E,H,I/16]; g_dn fp32 [E].
    Returns (out bf16 bits uint16 [n,H], out fp64 [n,H], number of out-of-range ids).
    w4a4=True: the activations (x rows, then h rows) are NVFP4-quantized per row as well.
    """
    xs = _u16(x)
    T, H = xs.shape
    ia = _np(ids, np.int32)
    wa = _np(w, np.float32)
    K = ia.shape[1]
    pg, sg, gg = _np(w_gu, np.uint8), _np(s_gu, np.uint8), _np(g_gu, np.float32)
    pd, sd, gd = _np(w_dn, np.uint8), _np(s_dn, np.uint8), _np(g_dn, np.float32)
    E = pg.shape[0]
    I = pg.shape[1] // 2
    assert pg.shape == (E, 2 * I, H // 2) and sg.shape == (E, 2 * I, H // 16)
    assert pd.shape == (E, H, I // 2) and sd.shape == (E, H, I // 16)
    tok = np.arange(T, dtype=np.int64) if tokens is None else _np(tokens, np.int64)
    out = np.zeros((tok.size, H), np.uint16)
    out64 = np.zeros((tok.size, H), np.float64)
    fn = _load().oracle_moe_forward_w4a4 if w4a4 else _load().oracle_moe_forward
    bad = fn(_p(xs), _p(ia), _p(wa), T, H, I, E, K,
                                     _p(pg), _p(sg), _p(gg), _p(pd), _p(sd), _p(gd),
                                     _p(tok), tok.size, _p(out), _p(out64))
    return out, out64, int(bad)


def shared_expert(x, w_gu, w_dn, tokens=None):
    """Shared-expert output y fp64 [n_tok, H] for the listed tokens (all when None).
    x bf16 [T, H]; w_gu bf16 [2Is, H]; w_dn bf16 [H, Is] (torch bf16 tensors or uint16)."""
    xs, gu, dn = _u16(x), _u16(w_gu), _u16(w_dn)
    T, H = xs.shape
    Is = gu.shape[0] // 2
    if gu.shape != (2 * Is, H) or dn.shape != (H, Is):
        raise ValueError("w_gu [2Is, H] and w_dn [H, Is]")
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((tok.size, H), np.float64)
    _load().oracle_shared_expert(_p(xs), H, Is, _p(gu), _p(dn), _p(tok), tok.size, _p(y))
    return y


def bf16_round_array(v) -> np.ndarray:
    """bf16 bits (uint16) of the fp64 values v, each rounded once to nearest even."""
    a = np.ascontiguousarray(v, np.float64)
    out = np.zeros(a.shape, np.uint16)
    _load().oracle_bf16_round_array(_p(a), a.size, _p(out))
    return out


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32)

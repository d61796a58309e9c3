"""Plain CPU oracle for the routed 4-bit MoE FFN (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.  The
C source (``moe_oracle.c``) states, function by function, which passage of the
pages it follows and how each function is pinned.

Arrays are numpy; f16/bf16 values travel as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fvisibility=hidden"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C11, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    """The oracle library.  ORACLE_LIB names another build of moe_oracle.c to
    load instead (the mutation tests load deliberately broken copies)."""
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        _declare(_lib)
    return _lib


_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_c_int, _c_f, _c_u16, _c_u8 = ctypes.c_int, ctypes.c_float, ctypes.c_uint16, ctypes.c_uint8
_vp = ctypes.c_void_p


def _declare(L):
    sig = {
        "orc_f16_to_f32": (_c_f, [_c_u16]),
        "orc_f32_to_f16": (_c_u16, [_c_f, _c_int]),
        "orc_bf16_to_f32": (_c_f, [_c_u16]),
        "orc_f32_to_bf16": (_c_u16, [_c_f]),
        "orc_e2m1_to_f32": (_c_f, [_c_u8]),
        "orc_f32_to_e2m1": (_c_u8, [_c_f]),
        "orc_e4m3_to_f32": (_c_f, [_c_u8]),
        "orc_f32_to_e4m3": (_c_u8, [_c_f]),
        "orc_quantize_w4": (None, [_f32p, _c_int, _c_int, _u8p, _u16p, _u16p]),
        "orc_pack_nibbles": (None, [_u8p, _c_int, _c_int, _u32p]),
        "orc_unpack_nibbles": (None, [_u32p, _c_int, _c_int, _u8p]),
        "orc_dequant_one": (_c_f, [_c_u8, _c_u16, _c_u16]),
        "orc_dequant_w4": (None, [_u8p, _u16p, _u16p, _c_int, _c_int, _f32p]),
        "orc_route": (None, [_f32p, _c_int, _c_int, _c_int, _i32p, _f32p]),
        "orc_permute": (None, [_i32p, _c_int, _c_int, _c_int, _i32p, _i32p, _i32p, _i32p]),
        "orc_expert_ffn_w4": (None, [_u16p, _c_int, _c_int, _u8p, _u16p, _u16p, _u8p, _u16p,
                                     _u16p, _f32p, _vp]),
        "orc_combine": (None, [_f32p, _f32p, _c_int, _c_int, _c_int, _u16p]),
        "orc_moe_forward_w4": (None, [_u16p, _f32p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                      _vp, _vp, _vp, _vp, _vp, _vp, _i32p, _f32p, _vp, _u16p]),
        "orc_router_logits": (None, [_u16p, _u16p, _c_int, _c_int, _c_int, _f32p]),
        "orc_moe_forward_w4_shared": (None, [_u16p, _f32p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                             _vp, _vp, _vp, _vp, _vp, _vp, _u8p, _u16p, _u16p, _u8p, _u16p,
                                             _u16p, _i32p, _f32p, _vp, _u16p]),
        "orc_quantize_w4_clip": (None, [_f32p, _c_int, _c_int, _u8p, _u16p, _u16p]),
        "orc_quantize_sym128": (None, [_f32p, _c_int, _c_int, _u8p, _u16p]),
        "orc_dequant_sym128": (_c_f, [_c_u8, _c_u16]),
        "orc_expert_ffn_sym128": (None, [_u16p, _c_int, _c_int, _u8p, _u16p, _u8p, _u16p, _f32p, _vp]),
        "orc_nvfp4_global": (_c_f, [_f32p, ctypes.c_size_t]),
        "orc_nvfp4_quantize": (None, [_f32p, _c_int, _c_int, _c_f, _u8p, _u8p]),
        "orc_nvfp4_gemv": (None, [_u8p, _u8p, _c_f, _u8p, _u8p, _c_f, _c_int, _c_int, _f32p]),
        "orc_expert_ffn_nvfp4": (None, [_u16p, _c_int, _c_int, _u8p, _u8p, _c_f, _u8p, _u8p,
                                        _c_f, _f32p, _vp, _vp, _vp, _vp]),
        "orc_down_nvfp4": (None, [_u8p, _u8p, _c_f, _c_int, _c_int, _u8p, _u8p, _c_f, _f32p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- formats
def f16_to_f32(h):
    L = lib()
    return np.array([L.orc_f16_to_f32(int(v)) for v in np.asarray(h).ravel()],
                    dtype=np.float32).reshape(np.shape(h))


def f32_to_f16(x, mode=0):
    """mode 0 nearest-even, 1 toward -inf, 2 toward +inf (bit patterns)."""
    L = lib()
    return np.array([L.orc_f32_to_f16(float(v), mode) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def bf16_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x):
    L = lib()
    return np.array([L.orc_f32_to_bf16(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def e2m1_to_f32(c):
    L = lib()
    return np.array([L.orc_e2m1_to_f32(int(v)) for v in np.asarray(c).ravel()],
                    dtype=np.float32).reshape(np.shape(c))


def f32_to_e2m1(x):
    L = lib()
    return np.array([L.orc_f32_to_e2m1(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint8).reshape(np.shape(x))


def e4m3_to_f32(c):
    L = lib()
    return np.array([L.orc_e4m3_to_f32(int(v)) for v in np.asarray(c).ravel()],
                    dtype=np.float32).reshape(np.shape(c))


def f32_to_e4m3(x):
    L = lib()
    return np.array([L.orc_f32_to_e4m3(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint8).reshape(np.shape(x))


# ---------------------------------------------------------------- int4 format
def quantize_w4(w):
    """fp32 [N][K] -> (codes u8 [N][K], scale f16-bits [N][K/64], min f16-bits [N][K/64])."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.uint8)
    s = np.empty((N, K // 64), np.uint16)
    m = np.empty((N, K // 64), np.uint16)
    lib().orc_quantize_w4(w, N, K, codes, s, m)
    return codes, s, m


def pack_nibbles(codes):
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    out = np.empty((N, K // 8), np.uint32)
    lib().orc_pack_nibbles(codes, N, K, out)
    return out


def unpack_nibbles(words, K):
    words = _c(words, np.uint32)
    N = words.shape[0]
    out = np.empty((N, K), np.uint8)
    lib().orc_unpack_nibbles(words, N, K, out)
    return out


def dequant_one(q, s_bits, m_bits):
    return lib().orc_dequant_one(int(q), int(s_bits), int(m_bits))


def dequant_w4(codes, scale, minv):
    codes = _c(codes, np.uint8)
    N, K = codes.shape
    out = np.empty((N, K), np.float32)
    lib().orc_dequant_w4(codes, _c(scale, np.uint16), _c(minv, np.uint16), N, K, out)
    return out


# ---------------------------------------------------------------- routing / permute
def route(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    lib().orc_route(logits, T, E, k, idx, w)
    return idx, w


def permute(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    sorted_rows = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().orc_permute(idx, T, k, E, counts, offsets, sorted_rows, inv)
    return counts, offsets, sorted_rows, inv


# ---------------------------------------------------------------- FFN / combine
def expert_ffn_w4(x_bf16, gu, d, return_h=False):
    """x_bf16: uint16 [H]; gu, d: (codes, scale, min) canonical triples."""
    x = _c(x_bf16, np.uint16)
    H = x.shape[0]
    F = gu[0].shape[0] // 2
    Y = np.empty(H, np.float32)
    h = np.empty(F, np.float32) if return_h else None
    lib().orc_expert_ffn_w4(x, H, F, _c(gu[0], np.uint8), _c(gu[1], np.uint16),
                            _c(gu[2], np.uint16), _c(d[0], np.uint8), _c(d[1], np.uint16),
                            _c(d[2], np.uint16), Y, _ptr(h))
    return (Y, h) if return_h else Y


def combine(y_rows, w):
    w = _c(w, np.float32)
    T, k = w.shape
    y_rows = _c(y_rows, np.float32).reshape(T * k, -1)
    H = y_rows.shape[1]
    y = np.empty((T, H), np.uint16)
    lib().orc_combine(y_rows, w, T, k, H, y)
    return y


def moe_forward_w4(x_bf16, logits, k, experts):
    """experts: dict e -> (gu triple, d triple); only routed experts are needed.

    Returns (idx, w, y_rows fp32 [T*k][H], y bf16 bits [T][H])."""
    x = _c(x_bf16, np.uint16)
    logits = _c(logits, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    idx, _ = route(logits, k)
    need = sorted(set(int(e) for e in idx.ravel()))
    missing = [e for e in need if e not in experts]
    if missing:
        raise KeyError(f"oracle needs weights of experts {missing}")
    F = experts[need[0]][0][0].shape[0] // 2
    keep = []

    def table(which, part, dt):
        arr = (ctypes.c_void_p * E)()
        for e in need:
            a = _c(experts[e][which][part], dt)
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    tabs = [table(0, 0, np.uint8), table(0, 1, np.uint16), table(0, 2, np.uint16),
            table(1, 0, np.uint8), table(1, 1, np.uint16), table(1, 2, np.uint16)]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    y_rows = np.empty((T * k, H), np.float32)
    y = np.empty((T, H), np.uint16)
    lib().orc_moe_forward_w4(x, logits, T, E, k, H, F, *[ctypes.cast(t, ctypes.c_void_p) for t in tabs],
                             idx, w, _ptr(y_rows), y)
    return idx, w, y_rows, y


def moe_forward_w4_shared(x_bf16, logits, k, experts, shared):
    """The routed experts plus a shared expert (weight 1, after the routed
    sum).  shared: (gu triple, d triple).  Returns (idx [T][k], w [T][k],
    y_rows fp32 [T][k+1][H], y bf16 bits [T][H])."""
    x = _c(x_bf16, np.uint16)
    logits = _c(logits, np.float32)
    T, H = x.shape
    E = logits.shape[1]
    idx, _ = route(logits, k)
    need = sorted(set(int(e) for e in idx.ravel()))
    missing = [e for e in need if e not in experts]
    if missing:
        raise KeyError(f"oracle needs weights of experts {missing}")
    F = shared[0][0].shape[0] // 2
    keep = []

    def table(which, part, dt):
        arr = (ctypes.c_void_p * E)()
        for e in need:
            a = _c(experts[e][which][part], dt)
            keep.append(a)
            arr[e] = a.ctypes.data
        return arr

    tabs = [table(0, 0, np.uint8), table(0, 1, np.uint16), table(0, 2, np.uint16),
            table(1, 0, np.uint8), table(1, 1, np.uint16), table(1, 2, np.uint16)]
    sh = [_c(shared[0][0], np.uint8), _c(shared[0][1], np.uint16), _c(shared[0][2], np.uint16),
          _c(shared[1][0], np.uint8), _c(shared[1][1], np.uint16), _c(shared[1][2], np.uint16)]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    y_rows = np.empty((T, k + 1, H), np.float32)
    y = np.empty((T, H), np.uint16)
    lib().orc_moe_forward_w4_shared(x, logits, T, E, k, H, F, *[ctypes.cast(t, ctypes.c_void_p) for t in tabs],
                                    *sh, idx, w, _ptr(y_rows), y)
    return idx, w, y_rows, y


# ---------------------------------------------------------------- router linear
def router_logits(x_bf16, wr_bf16):
    """x bf16 bits [T][H], Wr bf16 bits [E][H] -> fp32 logits [T][E]."""
    x = _c(x_bf16, np.uint16)
    wr = _c(wr_bf16, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    lib().orc_router_logits(x, wr, T, E, H, out)
    return out


# ---------------------------------------------------------------- clip search, symmetric group 128
def quantize_w4_clip(w):
    """Asymmetric group-64 int4 with the MSE clip search -> (codes u8 [N][K], scale f16 bits, min f16 bits)."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.uint8)
    scale = np.empty((N, K // 64), np.uint16)
    minv = np.empty((N, K // 64), np.uint16)
    lib().orc_quantize_w4_clip(w, N, K, codes, scale, minv)
    return codes, scale, minv


def quantize_sym128(w):
    """Symmetric group-128 int4 (zero point 8) with the MSE clip search -> (codes u8 [N][K], scale f16 bits)."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.empty((N, K), np.uint8)
    scale = np.empty((N, K // 128), np.uint16)
    lib().orc_quantize_sym128(w, N, K, codes, scale)
    return codes, scale


def dequant_sym128(codes, scale):
    N, K = codes.shape
    out = np.empty((N, K), np.float32)
    L = lib()
    for n in range(N):
        for k in range(K):
            out[n, k] = L.orc_dequant_sym128(int(codes[n, k]), int(scale[n, k // 128]))
    return out


def expert_ffn_sym128(x_bf16, gu, d, return_h=False):
    """x_bf16: uint16 [H]; gu, d: (codes, scale) symmetric group-128 pairs."""
    x = _c(x_bf16, np.uint16)
    H = x.shape[0]
    F = gu[0].shape[0] // 2
    Y = np.empty(H, np.float32)
    h = np.empty(F, np.float32) if return_h else None
    lib().orc_expert_ffn_sym128(x, H, F, _c(gu[0], np.uint8), _c(gu[1], np.uint16), _c(d[0], np.uint8),
                                _c(d[1], np.uint16), Y, _ptr(h))
    return (Y, h) if return_h else Y


# ---------------------------------------------------------------- NVFP4
def nvfp4_global(v):
    v = _c(v, np.float32).ravel()
    return lib().orc_nvfp4_global(v, v.size)


def nvfp4_quantize(v, G):
    v = _c(v, np.float32)
    N, K = v.shape
    codes = np.empty((N, K), np.uint8)
    sf = np.empty((N, K // 16), np.uint8)
    lib().orc_nvfp4_quantize(v, N, K, float(G), codes, sf)
    return codes, sf


def nvfp4_gemv(a_codes, a_sf, Ga, w_codes, w_sf, Gw):
    w_codes = _c(w_codes, np.uint8)
    N, K = w_codes.shape
    y = np.empty(N, np.float32)
    lib().orc_nvfp4_gemv(_c(a_codes, np.uint8), _c(a_sf, np.uint8), float(Ga), w_codes,
                         _c(w_sf, np.uint8), float(Gw), N, K, y)
    return y


def expert_ffn_nvfp4(x_bf16, gu, d, stages=False):
    """gu, d: (codes, sf, G).  With stages=True also returns (h, h_codes, h_sf, h_G)."""
    x = _c(x_bf16, np.uint16)
    H = x.shape[0]
    F = gu[0].shape[0] // 2
    Y = np.empty(H, np.float32)
    h = np.empty(F, np.float32)
    hc = np.empty(F, np.uint8)
    hs = np.empty(F // 16, np.uint8)
    hG = np.empty(1, np.float32)
    lib().orc_expert_ffn_nvfp4(x, H, F, _c(gu[0], np.uint8), _c(gu[1], np.uint8), float(gu[2]),
                               _c(d[0], np.uint8), _c(d[1], np.uint8), float(d[2]), Y,
                               _ptr(h), _ptr(hc), _ptr(hs), _ptr(hG))
    return (Y, (h, hc, hs, float(hG[0]))) if stages else Y


def down_nvfp4(h_codes, h_sf, Gh, d):
    d_codes = _c(d[0], np.uint8)
    H, F = d_codes.shape
    Y = np.empty(H, np.float32)
    lib().orc_down_nvfp4(_c(h_codes, np.uint8), _c(h_sf, np.uint8), float(Gh), H, F, d_codes,
                         _c(d[1], np.uint8), float(d[2]), Y)
    return Y

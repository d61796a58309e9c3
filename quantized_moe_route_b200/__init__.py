"""Python binding of libmoe, the routed 4-bit MoE FFN for B200 (sm_100a).

Argument marshalling only: every function below forwards device pointers and
sizes to the C ABI declared in ``include/moe.h`` under the same name; all work
runs in the library's CUDA kernels.  Tensors are torch CUDA tensors (torch
supplies device memory and streams); bf16/f16 buffers may be torch.bfloat16 /
torch.float16 or int16/uint16 views of the same bits.

The library must be built (``python -m quantized_moe_route_b200.build`` or
``__graft_entry__.build()``); importing the binding without it raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE = 0, 1, 2
MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = 3, 4, 5
MOE_DEVERR_DECODE_H_WAIT, MOE_DEVERR_PREFILL_WAIT = 0x101, 0x201
MOE_DEVERR_DECODE_ROUTER_WAIT = 0x102
MOE_W4_PLAIN, MOE_W4_GATE_UP = 0, 1

_lib = None


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        L = lib()
        msg = L.moe_status_string(status).decode()
        if status == MOE_ERR_CUDA:
            msg += " (" + L.moe_last_error_string().decode() + ")"
        super().__init__(f"{where}: {msg}")


class moe_w4_layer(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("F", ctypes.c_int),
                ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p)]


class moe_nvfp4_layer(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("F", ctypes.c_int),
                ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("g_gu", ctypes.c_void_p), ("g_d", ctypes.c_void_p)]


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_last_error_string": (ctypes.c_char_p, []),
    "moe_version": (ctypes.c_char_p, []),
    "moe_w4_packed_bytes": (_sz, [_i, _i]),
    "moe_quantize_w4": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_pack_w4": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "moe_unpack_w4": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_dequant_w4": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "moe_quantize_w4_clip": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_quantize_w4_sym128": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "moe_pack_w4_sym128_workspace_bytes": (_sz, [_i, _i]),
    "moe_pack_w4_sym128": (_i, [_vp, _vp, _i, _i, _i, _vp, _sz, _vp, _sz, _vp]),
    "moe_nvfp4_packed_bytes": (_sz, [_i, _i]),
    "moe_nvfp4_global": (_i, [_vp, _sz, _vp, _vp]),
    "moe_quantize_nvfp4": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_pack_nvfp4": (_i, [_vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "moe_unpack_nvfp4": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_quantize_nvfp4_rows": (_i, [_vp, _i, _i, _i, _vp, _i, _vp, _vp, _vp, _vp]),
    "moe_route": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_route_shared": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_router_route_workspace_bytes": (_sz, [_i, _i]),
    "moe_router_route": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_workspace_bytes": (_sz, [_i, _i, _i]),
    "moe_permute": (_i, [_vp, _i, _i, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_decode_workspace_bytes": (_sz, [_i, _i, _i]),
    "moe_ffn_w4a16_decode": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _vp, _vp, _sz, _vp]),
    "moe_ffn_w4a16_decode_static": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _vp, _vp]),
    "moe_decode_layer_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "moe_decode_layer_w4a16": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _sz,
                                    _vp]),
    "moe_decode_layer_w4a16_shared": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _vp, _vp, _vp, _vp,
                                           _sz, _vp]),
    "moe_decode_layer_router_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "moe_decode_layer_w4a16_router": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp,
                                           _vp, _sz, _vp]),
    "moe_decode_layer_nvfp4": (_i, [ctypes.POINTER(moe_nvfp4_layer), _vp, _vp, _i, _i, _vp, _vp, _vp, _vp,
                                    _sz, _vp]),
    "moe_prefill_workspace_bytes": (_sz, [_i, _i]),
    "moe_ffn_grouped_prefill": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _vp, _vp, _sz, _vp]),
    "moe_prefill_nvfp4_workspace_bytes": (_sz, [_i, _i]),
    "moe_ffn_grouped_prefill_nvfp4": (_i, [ctypes.POINTER(moe_nvfp4_layer), _vp, _vp, _vp, _vp, _i, _vp, _vp, _sz,
                                           _vp]),
    "moe_unpermute_combine": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_device_error": (_i, [ctypes.POINTER(ctypes.c_int), _vp]),
    "moe_debug_starve_decode": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _i, _vp, _vp, _sz, ctypes.c_uint,
                                     _vp]),
    "moe_debug_starve_prefill": (_i, [ctypes.POINTER(moe_w4_layer), _vp, _vp, _i, _vp, _sz, ctypes.c_uint, _vp]),
}


def lib():
    """The loaded libmoe (raises if the in-tree build is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run quantized_moe_route_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status, where):
    if status != MOE_OK:
        raise MoeError(status, where)


# ---------------------------------------------------------------- int4 weights
def moe_w4_packed_bytes(N: int, K: int) -> int:
    return lib().moe_w4_packed_bytes(N, K)


def moe_quantize_w4(w, codes, scale, minv, stream=None):
    N, K = w.shape
    _check(lib().moe_quantize_w4(_p(w), N, K, _p(codes), _p(scale), _p(minv), _stream(stream)),
           "moe_quantize_w4")


def moe_pack_w4(codes, scale, minv, kind, packed, stream=None):
    N, K = codes.shape
    nbytes = packed.numel() * packed.element_size()
    _check(lib().moe_pack_w4(_p(codes), _p(scale), _p(minv), N, K, kind, _p(packed), nbytes,
                             _stream(stream)), "moe_pack_w4")


def moe_quantize_w4_clip(w, codes, scale, minv, stream=None):
    N, K = w.shape
    _check(lib().moe_quantize_w4_clip(_p(w), N, K, _p(codes), _p(scale), _p(minv), _stream(stream)),
           "moe_quantize_w4_clip")


def moe_quantize_w4_sym128(w, codes, scale, stream=None):
    N, K = w.shape
    _check(lib().moe_quantize_w4_sym128(_p(w), N, K, _p(codes), _p(scale), _stream(stream)),
           "moe_quantize_w4_sym128")


def moe_pack_w4_sym128(codes, scale, kind, packed, ws, stream=None):
    N, K = codes.shape
    _check(lib().moe_pack_w4_sym128(_p(codes), _p(scale), N, K, kind, _p(packed), packed.numel(), _p(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "moe_pack_w4_sym128")


def moe_pack_w4_sym128_workspace_bytes(N, K) -> int:
    return lib().moe_pack_w4_sym128_workspace_bytes(N, K)


def moe_nvfp4_packed_bytes(N: int, K: int) -> int:
    return lib().moe_nvfp4_packed_bytes(N, K)


def moe_nvfp4_global(v, G, stream=None):
    _check(lib().moe_nvfp4_global(_p(v), v.numel(), _p(G), _stream(stream)), "moe_nvfp4_global")


def moe_quantize_nvfp4(v, G, codes, sf, stream=None):
    N, K = v.shape
    _check(lib().moe_quantize_nvfp4(_p(v), N, K, _p(G), _p(codes), _p(sf), _stream(stream)),
           "moe_quantize_nvfp4")


def moe_pack_nvfp4(codes, sf, kind, packed, stream=None):
    N, K = codes.shape
    nbytes = packed.numel() * packed.element_size()
    _check(lib().moe_pack_nvfp4(_p(codes), _p(sf), N, K, kind, _p(packed), nbytes, _stream(stream)),
           "moe_pack_nvfp4")


def moe_unpack_nvfp4(packed, N, K, kind, codes, sf, stream=None):
    _check(lib().moe_unpack_nvfp4(_p(packed), N, K, kind, _p(codes), _p(sf), _stream(stream)),
           "moe_unpack_nvfp4")


def moe_quantize_nvfp4_rows(x, codes, sf, G, src_rows=None, src_div=1, rows=None, stream=None):
    """x: bf16 (or int16 bits) or fp32 [*][K]; rows defaults to x.shape[0]."""
    import torch
    K = x.shape[1]
    rows = x.shape[0] if rows is None else rows
    dt = 1 if x.dtype == torch.float32 else 0
    _check(lib().moe_quantize_nvfp4_rows(_p(x), dt, rows, K, _p(src_rows), src_div, _p(codes), _p(sf),
                                         _p(G), _stream(stream)), "moe_quantize_nvfp4_rows")


def moe_unpack_w4(packed, N, K, kind, codes, scale, minv, stream=None):
    _check(lib().moe_unpack_w4(_p(packed), N, K, kind, _p(codes), _p(scale), _p(minv),
                               _stream(stream)), "moe_unpack_w4")


def moe_dequant_w4(packed, N, K, kind, out, stream=None):
    _check(lib().moe_dequant_w4(_p(packed), N, K, kind, _p(out), _stream(stream)), "moe_dequant_w4")


def make_layer(E, H, F, gate_up, down) -> moe_w4_layer:
    """Host descriptor of one layer's packed experts (device buffers)."""
    return moe_w4_layer(E, H, F, gate_up.data_ptr(), down.data_ptr())


def make_nvfp4_layer(E, H, F, gate_up, down, g_gu, g_d) -> moe_nvfp4_layer:
    """Host descriptor of one layer's packed NVFP4 experts and their globals (device buffers)."""
    return moe_nvfp4_layer(E, H, F, gate_up.data_ptr(), down.data_ptr(), g_gu.data_ptr(), g_d.data_ptr())


# ---------------------------------------------------------------- routing / permutation
def moe_route(logits, k, idx, w, stream=None):
    T, E = logits.shape
    _check(lib().moe_route(_p(logits), T, E, k, _p(idx), _p(w), _stream(stream)), "moe_route")


def moe_route_shared(logits, k, idx, w, stream=None):
    """Routing over E experts plus a shared expert: idx, w [T][k+1], column k = (E, 1.0)."""
    T, E = logits.shape
    _check(lib().moe_route_shared(_p(logits), T, E, k, _p(idx), _p(w), _stream(stream)), "moe_route_shared")


def moe_router_route_workspace_bytes(T, E) -> int:
    return lib().moe_router_route_workspace_bytes(T, E)


def moe_router_route(x, wr, k, idx, w, ws, logits=None, stream=None):
    """Router linear (bf16 Wr [E][H] times x [T][H]) and routing in one launch."""
    T, H = x.shape
    E = wr.shape[0]
    _check(lib().moe_router_route(_p(x), _p(wr), T, E, H, k, _p(logits), _p(idx), _p(w), _p(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "moe_router_route")


def moe_permute_workspace_bytes(T, k, E) -> int:
    return lib().moe_permute_workspace_bytes(T, k, E)


def moe_permute(idx, E, counts, offsets, sorted_rows, inv, ws, x=None, x_perm=None, stream=None):
    T, k = idx.shape
    H = 0 if x is None else x.shape[1]
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().moe_permute(_p(idx), T, k, E, _p(x), H, _p(counts), _p(offsets), _p(sorted_rows),
                             _p(inv), _p(x_perm), _p(ws), nbytes, _stream(stream)), "moe_permute")


# ---------------------------------------------------------------- expert FFN
def moe_decode_workspace_bytes(T, k, F) -> int:
    return lib().moe_decode_workspace_bytes(T, k, F)


def moe_ffn_w4a16_decode(layer: moe_w4_layer, x, idx, y_rows, ws, stream=None):
    T, k = idx.shape
    _check(lib().moe_ffn_w4a16_decode(ctypes.byref(layer), _p(x), _p(idx), T, k, _p(y_rows), _p(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)),
           "moe_ffn_w4a16_decode")


def moe_ffn_w4a16_decode_static(layer: moe_w4_layer, x, idx, y_rows, stream=None):
    """Decode without a workspace (scratch in a fixed library-owned array)."""
    T, k = idx.shape
    _check(lib().moe_ffn_w4a16_decode_static(ctypes.byref(layer), _p(x), _p(idx), T, k, _p(y_rows),
                                             _stream(stream)), "moe_ffn_w4a16_decode_static")


def moe_decode_layer_workspace_bytes(T, k, H, F) -> int:
    return lib().moe_decode_layer_workspace_bytes(T, k, H, F)


def moe_decode_layer_w4a16(layer: moe_w4_layer, x, logits, k, y, ws, idx=None, w=None, stream=None):
    """Route + expert FFN + combine of one layer in one launch."""
    T = x.shape[0]
    _check(lib().moe_decode_layer_w4a16(ctypes.byref(layer), _p(x), _p(logits), T, k, _p(y), _p(idx), _p(w),
                                        _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_decode_layer_w4a16")


def moe_decode_layer_w4a16_shared(layer: moe_w4_layer, x, logits, k, y, ws, idx=None, w=None, stream=None):
    """One layer in one launch with a shared expert: layer holds the routed
    experts then the shared one; logits cover the routed experts only."""
    T = x.shape[0]
    _check(lib().moe_decode_layer_w4a16_shared(ctypes.byref(layer), _p(x), _p(logits), T, k, _p(y), _p(idx),
                                               _p(w), _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_decode_layer_w4a16_shared")


def moe_decode_layer_router_workspace_bytes(T, k, shared, E, H, F) -> int:
    return lib().moe_decode_layer_router_workspace_bytes(T, k, shared, E, H, F)


def moe_decode_layer_w4a16_router(layer: moe_w4_layer, x, wr, k, y, ws, shared=0, idx=None, w=None, logits=None,
                                  stream=None):
    """One layer in one launch from x and the bf16 router weights wr [E - shared][H]:
    router linear, routing, expert FFN (plus the shared expert), combine."""
    T = x.shape[0]
    _check(lib().moe_decode_layer_w4a16_router(ctypes.byref(layer), _p(x), _p(wr), T, k, shared, _p(y), _p(idx),
                                               _p(w), _p(logits), _p(ws), ws.numel() * ws.element_size(),
                                               _stream(stream)), "moe_decode_layer_w4a16_router")


def moe_decode_layer_nvfp4(layer: moe_nvfp4_layer, x, logits, k, y, ws, idx=None, w=None, stream=None):
    """NVFP4 experts: route + in-kernel activation quantisation + FFN + combine, one launch."""
    T = x.shape[0]
    _check(lib().moe_decode_layer_nvfp4(ctypes.byref(layer), _p(x), _p(logits), T, k, _p(y), _p(idx), _p(w),
                                        _p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_decode_layer_nvfp4")


def moe_prefill_nvfp4_workspace_bytes(rows, F) -> int:
    return lib().moe_prefill_nvfp4_workspace_bytes(rows, F)


def moe_ffn_grouped_prefill_nvfp4(layer: moe_nvfp4_layer, x_codes, x_sf, x_G, offsets, y_perm, ws, stream=None):
    rows = x_codes.shape[0]
    _check(lib().moe_ffn_grouped_prefill_nvfp4(ctypes.byref(layer), _p(x_codes), _p(x_sf), _p(x_G), _p(offsets),
                                               rows, _p(y_perm), _p(ws), ws.numel() * ws.element_size(),
                                               _stream(stream)), "moe_ffn_grouped_prefill_nvfp4")


def moe_prefill_workspace_bytes(rows, F) -> int:
    return lib().moe_prefill_workspace_bytes(rows, F)


def moe_ffn_grouped_prefill(layer: moe_w4_layer, x_perm, offsets, y_perm, ws, stream=None):
    rows = x_perm.shape[0]
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().moe_ffn_grouped_prefill(ctypes.byref(layer), _p(x_perm), _p(offsets), rows,
                                         _p(y_perm), _p(ws), nbytes, _stream(stream)),
           "moe_ffn_grouped_prefill")


def moe_unpermute_combine(Y, w, y, inv=None, stream=None):
    T, k = w.shape
    H = y.shape[1]
    y_dtype = 0 if Y.element_size() == 4 else 1
    _check(lib().moe_unpermute_combine(_p(Y), y_dtype, _p(inv), _p(w), T, k, H, _p(y),
                                       _stream(stream)), "moe_unpermute_combine")


def moe_device_error(stream=None) -> int:
    out = ctypes.c_int(0)
    _check(lib().moe_device_error(ctypes.byref(out), _stream(stream)), "moe_device_error")
    return out.value


def moe_debug_starve_decode(layer: moe_w4_layer, x, idx, y_rows, ws, polls, stream=None):
    T, k = idx.shape
    _check(lib().moe_debug_starve_decode(ctypes.byref(layer), _p(x), _p(idx), T, k, _p(y_rows), _p(ws),
                                         ws.numel() * ws.element_size(), polls, _stream(stream)),
           "moe_debug_starve_decode")


def moe_debug_starve_prefill(layer: moe_w4_layer, x_perm, offsets, ws, polls, stream=None):
    rows = x_perm.shape[0]
    _check(lib().moe_debug_starve_prefill(ctypes.byref(layer), _p(x_perm), _p(offsets), rows, _p(ws),
                                          ws.numel() * ws.element_size(), polls, _stream(stream)),
           "moe_debug_starve_prefill")

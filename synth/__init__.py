"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds none of the MoE method's arithmetic: it only draws the
random inputs the workloads call for (expert weights ~N(0, 0.02) before
quantisation, bf16 activations ~N(0, 1), router logits ~N(0, 1), a Zipf-like
per-expert bias for the skewed prefill load).

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
numbers: as easy as 1, 2, 3", SC'11), one call per element.  A call's four
32-bit outputs, each cut to its top 24 bits, are summed (Irwin-Hall of order
4, mean 2^25, variance 2^48/3); the centred integer sum is converted to fp32
(round to nearest even) and multiplied by one fp32 constant, so the value is
bit-identical wherever it is computed.  The CUDA twin of this generator lives
in ``synth/synth_gen.cu`` and is checked against this file bit for bit.

Counter layout for element i of stream (a, b) under seed s:
    counter = (i mod 2^32, i div 2^32, a, b), key = (s, 0x5EEDC0DE).
"""
from __future__ import annotations

import math

import numpy as np

PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = np.uint32(0x9E3779B9)
PHILOX_W1 = np.uint32(0xBB67AE85)
KEY_HI = 0x5EEDC0DE
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32 with 10 rounds; all arguments uint32 arrays/scalars."""
    c0, c1, c2, c3 = (np.asarray(v, np.uint32).astype(np.uint64) for v in (c0, c1, c2, c3))
    k0 = np.uint64(np.uint32(k0))
    k1 = np.uint64(np.uint32(k1))
    for r in range(10):
        if r:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & _MASK32, lo1, (hi0 ^ c3 ^ k1) & _MASK32, lo0
    return tuple(v.astype(np.uint32) for v in (c0, c1, c2, c3))


def irwin_hall_scale(sigma: float) -> np.float32:
    """fp32 constant mapping the centred 4-uniform integer sum to std sigma."""
    return np.float32(sigma * math.sqrt(3.0) / float(1 << 24))


def normal_f32(seed: int, a: int, b: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    """n approximately N(0, sigma^2) fp32 values of stream (a, b) (C twin)."""
    out = np.empty(n, np.float32)
    if n:
        _cpu().synth_normal_f32_cpu(out.ctypes.data, n, 1, a, 0, b, seed,
                                    float(irwin_hall_scale(sigma)), start)
    return out


def normal_f32_numpy(seed: int, a: int, b: int, n: int, sigma: float, start: int = 0) -> np.ndarray:
    """Reference numpy form of normal_f32 (slow; pins the C and CUDA twins)."""
    i = np.arange(start, start + n, dtype=np.uint64)
    r = philox4x32_10((i & _MASK32).astype(np.uint32), (i >> np.uint64(32)).astype(np.uint32),
                      np.uint32(a), np.uint32(b), np.uint32(seed), np.uint32(KEY_HI))
    s = sum((v >> np.uint32(8)).astype(np.int64) for v in r) - (1 << 25)
    return s.astype(np.int32).astype(np.float32) * irwin_hall_scale(sigma)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the bit patterns (inputs only)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# Stream ids: a = 4*expert + proj (proj 0 gate_up, 1 down), b = layer; the
# activation / logit streams use b = 0x10000 + layer with a = 0 (x), 1 (logits).
PROJ_GATE_UP, PROJ_DOWN = 0, 1


def expert_weights(seed: int, layer: int, expert: int, proj: int, N: int, K: int,
                   sigma: float = 0.02) -> np.ndarray:
    """fp32 [N][K] expert matrix (gate_up is [2F][H] with gate rows first)."""
    return normal_f32(seed, 4 * expert + proj, layer, N * K, sigma).reshape(N, K)


def activations_bf16(seed: int, layer: int, T: int, H: int) -> np.ndarray:
    """bf16 bit patterns [T][H] of x ~ N(0, 1)."""
    return f32_to_bf16_bits(normal_f32(seed, 0, 0x10000 + layer, T * H, 1.0)).reshape(T, H)


def router_logits(seed: int, layer: int, T: int, E: int, bf16_rounded: bool = False) -> np.ndarray:
    """fp32 [T][E] logits ~ N(0, 1); optionally rounded to bf16 (so ties occur)."""
    l = normal_f32(seed, 1, 0x10000 + layer, T * E, 1.0).reshape(T, E)
    if bf16_rounded:
        l = bf16_bits_to_f32(f32_to_bf16_bits(l)).reshape(T, E)
    return l


def zipf_bias(seed: int, E: int, s: float = 1.1) -> np.ndarray:
    """Per-expert logit bias -s*ln(rank), rank a seeded permutation of 1..E.

    Adding it to N(0,1) logits skews expert loads like a Zipf(s) popularity."""
    rng = np.random.Generator(np.random.Philox(key=seed))
    rank = rng.permutation(E) + 1
    return (-s * np.log(rank.astype(np.float64))).astype(np.float32)


# ---------------------------------------------------------------- CUDA twin
import ctypes as _ct
import os as _os
import subprocess as _sp

_HERE = _os.path.dirname(_os.path.abspath(__file__))
_CU = _os.path.join(_HERE, "synth_gen.cu")
_SO = _os.path.join(_HERE, "libsynth.so")
_cuda_lib = None
_C = _os.path.join(_HERE, "synth_cpu.c")
_CSO = _os.path.join(_HERE, "libsynth_cpu.so")
_cpu_lib = None


def build_cpu(force: bool = False) -> str:
    if force or not _os.path.exists(_CSO) or _os.path.getmtime(_CSO) < _os.path.getmtime(_C):
        tmp = _CSO + f".tmp{_os.getpid()}"
        _sp.check_call(["gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", tmp, _C])
        _os.replace(tmp, _CSO)
    return _CSO


def _cpu():
    global _cpu_lib
    if _cpu_lib is None:
        L = _ct.CDLL(build_cpu())
        L.synth_normal_f32_cpu.restype = None
        L.synth_normal_f32_cpu.argtypes = [_ct.c_void_p, _ct.c_uint64, _ct.c_int, _ct.c_uint32, _ct.c_uint32,
                                           _ct.c_uint32, _ct.c_uint32, _ct.c_float, _ct.c_uint64]
        _cpu_lib = L
    return _cpu_lib


def build_cuda(force: bool = False) -> str:
    """Compile the CUDA twin of the generator (sm_100a)."""
    if force or not _os.path.exists(_SO) or _os.path.getmtime(_SO) < _os.path.getmtime(_CU):
        tmp = _SO + f".tmp{_os.getpid()}"
        _sp.check_call([_os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O3", "-shared", "-Xcompiler", "-fPIC", "-o", tmp, _CU])
        _os.replace(tmp, _SO)
    return _SO


def _cuda():
    global _cuda_lib
    if _cuda_lib is None:
        L = _ct.CDLL(build_cuda())
        L.synth_normal_f32.restype = _ct.c_int
        L.synth_normal_f32.argtypes = [_ct.c_void_p, _ct.c_uint64, _ct.c_int, _ct.c_uint32, _ct.c_uint32,
                                       _ct.c_uint32, _ct.c_uint32, _ct.c_float, _ct.c_uint64, _ct.c_void_p]
        _cuda_lib = L
    return _cuda_lib


def cuda_expert_weights(out, seed: int, layer: int, expert0: int, proj: int, sigma: float = 0.02,
                        stream=None):
    """Fill torch CUDA fp32 tensor out [count][N][K] with the matrices of experts
    expert0 .. expert0+count-1 (identical bits to expert_weights())."""
    import torch
    count, N, K = out.shape
    s = torch.cuda.current_stream() if stream is None else stream
    rc = _cuda().synth_normal_f32(out.data_ptr(), N * K, count, 4 * expert0 + proj, 4, layer, seed,
                                  float(irwin_hall_scale(sigma)), 0, _ct.c_void_p(s.cuda_stream))
    if rc:
        raise RuntimeError(f"synth_normal_f32 failed with CUDA error {rc}")

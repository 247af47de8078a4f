"""Seeded synthetic inputs for the block-quantised MoE FFN.

Thin ctypes wrapper over ``synth.c`` (SplitMix64, counter-based).  This module
draws raw inputs only -- codes, block scales, activations and router logits --
and holds none of the method's arithmetic.  It is the one module that both the
fp64 oracle side and the CUDA side use.

Stream keys: ``key(seed, layer, tag, expert)``.  Tags used by the workloads:

====  =====================================
tag   stream
====  =====================================
0..5  codes of gate, up, down, shared gate, shared up, shared down
10..15 block scales of the same six matrices
100   expert permutation of the Zipf routing bias
101   router logits (normal draws)
102   router projection weights (normal draws)
200   activations x
====  =====================================
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

KIND_GATE, KIND_UP, KIND_DOWN, KIND_SH_GATE, KIND_SH_UP, KIND_SH_DOWN = range(6)
TAG_SCALE_OFFSET = 10
TAG_PERM = 100
TAG_LOGITS = 101
TAG_WROUTER = 102
TAG_X = 200


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            L.synth_draw.restype = u64
            L.synth_draw.argtypes = [u64, u64]
            L.synth_key.restype = u64
            L.synth_key.argtypes = [u64, u64, u64, u64]
            L.synth_codes.restype = i32
            L.synth_codes.argtypes = [u64, i32, i64, i64, i64, vp]
            L.synth_scales.restype = i32
            L.synth_scales.argtypes = [u64, i32, i64, i64, i64, vp]
            L.synth_normal_f64.restype = None
            L.synth_normal_f64.argtypes = [u64, i64, i64, vp]
            L.synth_normal_bf16.restype = None
            L.synth_normal_bf16.argtypes = [u64, i64, i64, vp]
            L.synth_zipf_bias.restype = None
            L.synth_zipf_bias.argtypes = [u64, i32, ctypes.c_double, vp]
            L.synth_logits.restype = None
            L.synth_logits.argtypes = [u64, vp, i64, i64, i32, vp]
            L.synth_init()
            _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def key(seed: int, a: int, b: int, c: int) -> int:
    return int(lib().synth_key(seed & (2**64 - 1), a, b, c))


def draw(k: int, n: int) -> int:
    return int(lib().synth_draw(k, n))


def codes(k: int, bits: int, rows: int, cols: int, row0: int = 0) -> np.ndarray:
    """uint8 [rows][cols] codes in [0, 2^bits)."""
    out = np.empty((rows, cols), dtype=np.uint8)
    if lib().synth_codes(k, bits, row0, rows, cols, _p(out)) != 0:
        raise ValueError("synth_codes: bad arguments")
    return out


def scales(k: int, bits: int, rows: int, cols: int, row0: int = 0) -> np.ndarray:
    """Block scales [rows][cols/32]: uint16 binary16 bits (bits 2/3) or uint8 E8M0 (bits 4)."""
    out = np.empty((rows, cols // 32), dtype=np.uint8 if bits == 4 else np.uint16)
    if lib().synth_scales(k, bits, row0, rows, cols, _p(out)) != 0:
        raise ValueError("synth_scales: bad arguments")
    return out


def normal_f64(k: int, n: int, n0: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().synth_normal_f64(k, n0, n, _p(out))
    return out


def normal_bf16(k: int, n: int, n0: int = 0) -> np.ndarray:
    """uint16 bf16 bit patterns of N(0,1) draws."""
    out = np.empty(n, dtype=np.uint16)
    lib().synth_normal_bf16(k, n0, n, _p(out))
    return out


def zipf_bias(seed: int, layer: int, E: int, s: float) -> np.ndarray:
    out = np.empty(E, dtype=np.float64)
    lib().synth_zipf_bias(key(seed, layer, TAG_PERM, 0), E, float(s), _p(out))
    return out


def logits(seed: int, layer: int, tok0: int, T: int, E: int, zipf_s: float) -> np.ndarray:
    """fp32 [T][E] router logits N(0,1) + per-expert Zipf log-popularity bias."""
    bias = zipf_bias(seed, layer, E, zipf_s)
    out = np.empty((T, E), dtype=np.float32)
    lib().synth_logits(key(seed, layer, TAG_LOGITS, 0), _p(bias), tok0, T, E, _p(out))
    return out


def router_weight_bf16(seed: int, layer: int, E: int, H: int) -> np.ndarray:
    """uint16 [E][H] bf16 router projection weights: N(0,1) draws in bf16 times
    2^-floor(log2(H)/2) (an exact power of two near 1/sqrt(H), so that W x has
    about unit variance for x ~ N(0,1))."""
    raw = normal_bf16(key(seed, layer, TAG_WROUTER, 0), E * H).reshape(E, H)
    sh = int(np.floor(np.log2(H) / 2))
    f = (raw.astype(np.uint32) << 16).view(np.float32) * np.float32(2.0 ** -sh)   # exact: a power of two
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def router_bias_f32(seed: int, layer: int, E: int, s: float) -> np.ndarray:
    """fp32 [E] per-expert routing bias: the Zipf log-popularity of the logits workload."""
    return zipf_bias(seed, layer, E, s).astype(np.float32)


def x_bf16(seed: int, tok0: int, T: int, H: int, stream: int = 0) -> np.ndarray:
    """uint16 [T][H] bf16 activations, token t uses normal draws t*H .. t*H+H-1."""
    out = np.empty((T, H), dtype=np.uint16)
    lib().synth_normal_bf16(key(seed, stream, TAG_X, 0), tok0 * H, T * H, _p(out))
    return out


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp64."""
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class MatrixSpec:
    """Codes + scales of one synthetic matrix [rows][cols] in format ``bits``."""

    def __init__(self, seed: int, layer: int, kind: int, expert: int, bits: int, rows: int, cols: int):
        self.seed, self.layer, self.kind, self.expert = seed, layer, kind, expert
        self.bits, self.rows, self.cols = bits, rows, cols
        self.code_key = key(seed, layer, kind, expert)
        self.scale_key = key(seed, layer, kind + TAG_SCALE_OFFSET, expert)

    def codes(self, row0: int = 0, nrows: int | None = None) -> np.ndarray:
        n = self.rows - row0 if nrows is None else nrows
        return codes(self.code_key, self.bits, n, self.cols, row0)

    def scales(self, row0: int = 0, nrows: int | None = None) -> np.ndarray:
        n = self.rows - row0 if nrows is None else nrows
        return scales(self.scale_key, self.bits, n, self.cols, row0)


# ------------------------------------------------ device twin (synth_dev.cu) ---

_SRC_DEV = os.path.join(_HERE, "synth_dev.cu")
_SO_DEV = os.path.join(_HERE, "libsynth_dev.so")
_lib_dev = None
_dev_tables = {}


def build_dev(force: bool = False) -> str:
    """Compile ``libsynth_dev.so`` (nvcc, sm_100a)."""
    if force or not os.path.exists(_SO_DEV) or os.path.getmtime(_SO_DEV) < os.path.getmtime(_SRC_DEV):
        tmp = _SO_DEV + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-Xcompiler", "-fPIC",
                               "-shared", "-o", tmp, _SRC_DEV])
        os.replace(tmp, _SO_DEV)
    return _SO_DEV


def lib_dev():
    global _lib_dev
    with _lock:
        if _lib_dev is None:
            build_dev()
            L = ctypes.CDLL(_SO_DEV)
            u64, i64, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
            L.synth_codes_dev.restype = i32
            L.synth_codes_dev.argtypes = [u64, i32, i64, i64, i64, vp, vp]
            L.synth_scales_dev.restype = i32
            L.synth_scales_dev.argtypes = [u64, i32, i64, i64, i64, vp, vp, vp, vp]
            _lib_dev = L
    return _lib_dev


def scale_tables():
    """Host copies of the 65536-entry binary16 and E8M0 scale tables."""
    f16 = np.empty(65536, dtype=np.uint16)
    e8 = np.empty(65536, dtype=np.uint8)
    lib().synth_scale_tables.restype = None
    lib().synth_scale_tables.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib().synth_scale_tables(_p(f16), _p(e8))
    return f16, e8


def _tables_on(device):
    import torch
    key_ = str(device)
    if key_ not in _dev_tables:
        f16, e8 = scale_tables()
        _dev_tables[key_] = (torch.from_numpy(f16.view(np.int16).copy()).to(device),
                             torch.from_numpy(e8.copy()).to(device))
    return _dev_tables[key_]


def _stream_ptr(stream):
    import torch
    return (stream or torch.cuda.current_stream()).cuda_stream


def codes_dev(k: int, bits: int, rows: int, cols: int, out, row0: int = 0, stream=None):
    """Device codes into ``out`` (torch uint8, >= rows*cols bytes, 16-byte aligned)."""
    if lib_dev().synth_codes_dev(k, bits, row0, rows, cols, out.data_ptr(), _stream_ptr(stream)) != 0:
        raise RuntimeError("synth_codes_dev failed")


def scales_dev(k: int, bits: int, rows: int, cols: int, out, row0: int = 0, stream=None):
    tf16, te8 = _tables_on(out.device)
    if lib_dev().synth_scales_dev(k, bits, row0, rows, cols, out.data_ptr(), tf16.data_ptr(), te8.data_ptr(),
                                  _stream_ptr(stream)) != 0:
        raise RuntimeError("synth_scales_dev failed")

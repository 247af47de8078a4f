"""fp64 CPU oracle of the block-quantised MoE FFN step (ctypes over ``oracle.c``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it: it consumes the raw codes and
scales drawn by ``synth`` and computes each step from its definition in fp64.

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
fixed by the pages or by mathematics (closed forms, brute force with library
routines, invariants).  The one part that nothing can pin is the real ROCmFPX
bit layout and level table, which the pages do not print: the oracle follows
the format this library fixes (levels ``c - (2^b-1)/2``, one scale per block).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _Mat(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (plain C, fp64, OpenMP, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
                               "-fopenmp", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load(_SO)
    return _lib


def load(path: str):
    """A compiled oracle library at `path` with the argument types set (lib()
    uses it for the library built here; the mutation test for a planted-bug
    copy)."""
    L = ctypes.CDLL(path)
    i32, i64, vp, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
    L.oracle_block_bytes.restype = i32
    L.oracle_block_bytes.argtypes = [i32]
    L.oracle_bits_per_weight.restype = dbl
    L.oracle_bits_per_weight.argtypes = [i32]
    L.oracle_level.restype = dbl
    L.oracle_level.argtypes = [i32, i32]
    L.oracle_bf16_round.restype = dbl
    L.oracle_bf16_round.argtypes = [dbl]
    L.oracle_silu.restype = dbl
    L.oracle_silu.argtypes = [dbl]
    L.oracle_dequant.restype = i32
    L.oracle_dequant.argtypes = [i32, vp, vp, i64, i64, vp]
    L.oracle_gemv.restype = i32
    L.oracle_gemv.argtypes = [i32, vp, vp, i64, i64, vp, i32, vp, vp]
    L.oracle_gemv_bf16w.restype = i32
    L.oracle_gemv_bf16w.argtypes = [i32, vp, vp, i64, i64, vp, i32, vp, vp]
    L.oracle_router_topk.restype = i32
    L.oracle_router_topk.argtypes = [vp, i64, i32, i32, vp, vp]
    L.oracle_expert_ffn.restype = i32
    L.oracle_expert_ffn.argtypes = [i32, i32, vp, vp, vp, vp, i32, vp, vp, vp]
    L.oracle_moe_token.restype = i32
    L.oracle_moe_token.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp]
    L.oracle_rms_bf16.restype = None
    L.oracle_rms_bf16.argtypes = [vp, i64, vp]
    return L


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed (rc={rc})")


def block_bytes(bits: int) -> int:
    return int(lib().oracle_block_bytes(bits))


def bits_per_weight(bits: int) -> float:
    return float(lib().oracle_bits_per_weight(bits))


def level(bits: int, c: int) -> float:
    return float(lib().oracle_level(bits, c))


def bf16_round(v: float) -> float:
    return float(lib().oracle_bf16_round(float(v)))


def silu(z: float) -> float:
    return float(lib().oracle_silu(float(z)))


class Mat:
    """Raw (unpacked) matrix: codes uint8 [rows][cols], scales [rows][cols/32]."""

    def __init__(self, bits: int, codes: np.ndarray, scales: np.ndarray):
        self.bits = int(bits)
        self.codes = _c(codes, np.uint8)
        self.scales = _c(scales, np.uint8 if bits == 4 else np.uint16)
        assert self.codes.ndim == 2 and self.scales.shape == (self.codes.shape[0], self.codes.shape[1] // 32)

    @property
    def shape(self):
        return self.codes.shape

    def cstruct(self) -> _Mat:
        return _Mat(self.bits, self.codes.ctypes.data, self.scales.ctypes.data)


def dequant(m: Mat) -> np.ndarray:
    rows, cols = m.shape
    W = np.empty((rows, cols), dtype=np.float64)
    _check(lib().oracle_dequant(m.bits, _p(m.codes), _p(m.scales), rows, cols, _p(W)), "dequant")
    return W


def gemv(m: Mat, x: np.ndarray, bf16_weights: bool = False):
    """y[q][N] = W x for x[q][K] (fp64); returns (y, mag) with mag = |W||x|.
    bf16_weights: every weight rounded once to bf16 first (prefill operands)."""
    x = _c(np.atleast_2d(x), np.float64)
    N, K = m.shape
    q = x.shape[0]
    assert x.shape[1] == K
    y = np.empty((q, N), dtype=np.float64)
    mag = np.empty((q, N), dtype=np.float64)
    fn = lib().oracle_gemv_bf16w if bf16_weights else lib().oracle_gemv
    _check(fn(m.bits, _p(m.codes), _p(m.scales), N, K, _p(x), q, _p(y), _p(mag)), "gemv")
    return y, mag


def group_rows(idx: np.ndarray, w: np.ndarray, E: int):
    """Prefill grouping of the routed entries: counts[E] tokens per expert and,
    for the rows grouped by ascending expert with the entries (t, j) of one
    expert in ascending t*k + j order (a stable sort of the flattened ids),
    the token, the combine weight and the entry t*k + j of every row.  Ids
    outside [0, E) get no row."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    ok = (flat >= 0) & (flat < E)
    order = np.argsort(np.where(ok, flat, E), kind="stable")[: int(ok.sum())]
    counts = np.bincount(flat[ok], minlength=E).astype(np.int32)
    return counts, (order // k).astype(np.int32), np.asarray(w, dtype=np.float64).reshape(-1)[order], order


def router_logits(w_router: np.ndarray, bias, x: np.ndarray):
    """Router projection ahead of the top-k: (logits fp64 [T][E], mag fp64 [T][E])
    with logits[t][e] = sum_h W[e][h] x[t][h] + b[e] and mag = sum_h |W[e][h]|
    |x[t][h]| + |b[e]| (for the per-element bound).  W: uint16 bf16 bits [E][H];
    x: uint16 bf16 bits [T][H]; bias: fp32 [E] or None.  Both operands widen
    exactly to fp64; the sum is a plain fp64 matrix product.

    The projection is the MoE gate that decides the routing, kept at high
    precision: FP8 in the bit allocation of ai-manual.ru, "DeepSeek V4 Flash на
    AMD Ryzen AI MAX+ 395…", section "Технические детали ROCmFPX"; sensitive
    projections at FP4 or above in taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI
    MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进 128 GB".  This
    library reads "high precision" as bf16 weights.
    """
    W = _bf16_bits_to_f64(np.asarray(w_router, dtype=np.uint16))
    X = _bf16_bits_to_f64(np.atleast_2d(np.asarray(x, dtype=np.uint16)))
    logits = X @ W.T
    mag = np.abs(X) @ np.abs(W).T
    if bias is not None:
        b = np.asarray(bias, dtype=np.float32).astype(np.float64)
        logits = logits + b[None, :]
        mag = mag + np.abs(b)[None, :]
    return logits, mag


def _bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def router_topk(logits: np.ndarray, k: int):
    """(idx int32 [T][k], w fp64 [T][k]) for fp32 logits [T][E]."""
    logits = _c(np.atleast_2d(logits), np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _check(lib().oracle_router_topk(_p(logits), T, E, k, _p(idx), _p(w)), "router_topk")
    return idx, w


def expert_ffn(gate: Mat, up: Mat, down: Mat, x: np.ndarray, bf16_ops: bool = False):
    """(d[H], mag[H], h[I]) for one token column x[H]."""
    I, H = gate.shape
    x = _c(x, np.float64)
    d = np.empty(H, dtype=np.float64)
    mag = np.empty(H, dtype=np.float64)
    h = np.empty(I, dtype=np.float64)
    g, u, dn = gate.cstruct(), up.cstruct(), down.cstruct()
    _check(lib().oracle_expert_ffn(H, I, ctypes.byref(g), ctypes.byref(u), ctypes.byref(dn), _p(x),
                                   int(bf16_ops), _p(d), _p(mag), _p(h)), "expert_ffn")
    return d, mag, h


def moe_token(experts, w, shared, x: np.ndarray, bf16_ops: bool = False):
    """One token: experts = [(gate, up, down)] * k in routing order, w[k] fp64,
    shared = (gate, up, down) or None.  Returns (y[H], mag[H])."""
    k = len(experts)
    I, H = (experts[0][0] if k else shared[0]).shape
    G = (_Mat * max(k, 1))(*[e[0].cstruct() for e in experts])
    U = (_Mat * max(k, 1))(*[e[1].cstruct() for e in experts])
    D = (_Mat * max(k, 1))(*[e[2].cstruct() for e in experts])
    S = (_Mat * 3)(*[m.cstruct() for m in shared]) if shared is not None else None
    wv = _c(np.asarray(w, dtype=np.float64).reshape(-1), np.float64)
    x = _c(x, np.float64)
    y = np.empty(H, dtype=np.float64)
    mag = np.empty(H, dtype=np.float64)
    _check(lib().oracle_moe_token(H, I, k, G, U, D, _p(wv), S, _p(x), int(bf16_ops), _p(y), _p(mag)),
           "moe_token")
    return y, mag


def rms_bf16(y: np.ndarray) -> np.ndarray:
    """x_next = bf16(y / sqrt(mean(y^2))) as fp64 values."""
    y = _c(y, np.float64)
    out = np.empty_like(y)
    lib().oracle_rms_bf16(_p(y), y.shape[0], _p(out))
    return out

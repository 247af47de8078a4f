"""B200 (sm_100a) block-quantised MoE FFN: thin Python binding of ``librfx.so``.

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels (``csrc/``); PyTorch supplies device memory and streams.  The
binding keeps the C ABI's names (``include/rfx.h``).  There is no CPU fallback:
importing fails if the library is missing and every call raises on a non-OK
status.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librfx.so")

RFX_OK, RFX_EINVAL, RFX_EUNSUPPORTED, RFX_ECUDA, RFX_EDEVICE, RFX_ERANGE = 0, -1, -2, -3, -4, -5
RFX_FP2, RFX_FP3, RFX_FP4 = 2, 3, 4
MAX_T = 8

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python block_quantized_moe_rocmfpx_b200/build.py` "
                      "(nvcc, sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)
_i32, _i64, _sz, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class moe_layer_desc(ctypes.Structure):
    _fields_ = [("H", _i32), ("I", _i32), ("E", _i32), ("k", _i32),
                ("f_gate", _i32), ("f_up", _i32), ("f_down", _i32),
                ("gate", _vp), ("up", _vp), ("down", _vp),
                ("stride_gate", _sz), ("stride_up", _sz), ("stride_down", _sz),
                ("has_shared", _i32),
                ("f_sh_gate", _i32), ("f_sh_up", _i32), ("f_sh_down", _i32),
                ("sh_gate", _vp), ("sh_up", _vp), ("sh_down", _vp)]


class moe_expert_mix(ctypes.Structure):
    _fields_ = [("f_gate_up", _i32), ("f_down", _i32),
                ("off_gate", ctypes.c_uint64), ("off_up", ctypes.c_uint64), ("off_down", ctypes.c_uint64)]


def _proto(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_lib_last_error = _proto("rfx_last_error", ctypes.c_char_p, [])
_packed_bytes = _proto("rfx_packed_bytes", _sz, [_i32, _i64, _i64])
_pack = _proto("rfx_pack", _i32, [_i32, _vp, _vp, _i64, _i64, _vp, _sz])
_unpack = _proto("rfx_unpack", _i32, [_i32, _vp, _i64, _i64, _vp, _vp])
_pack_device = _proto("rfx_pack_device", _i32, [_i32, _vp, _vp, _i64, _i64, _vp, _vp])
_router = _proto("moe_router_topk", _i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp])
_router_logits = _proto("moe_router_logits", _i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp])
_router_proj_topk = _proto("moe_router_project_topk", _i32,
                           [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp])
_gemv = _proto("rfx_gemv_q", _i32, [_i32, _vp, _i64, _i64, _vp, _i32, _i32, _vp, _vp])
_layer_create = _proto("moe_layer_create", _i32, [ctypes.POINTER(moe_layer_desc), ctypes.POINTER(_vp)])
_layer_create_mix = _proto("moe_layer_create_mix", _i32,
                           [ctypes.POINTER(moe_layer_desc), ctypes.POINTER(moe_expert_mix), ctypes.POINTER(_vp)])
_layer_destroy = _proto("moe_layer_destroy", None, [_vp])
_ws_bytes = _proto("moe_ffn_workspace_bytes", _sz, [_vp, _i32])
_ws_init = _proto("rfx_ws_init", _i32, [_vp, _sz, _vp])
_ws_status = _proto("rfx_ws_status", _i32, [_vp, _vp])
_forward = _proto("moe_ffn_forward", _i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp])
_forward_logits = _proto("moe_ffn_forward_logits", _i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_host_scratch = _proto("moe_ffn_host_scratch_bytes", _sz, [_vp, _i32])
_forward_host = _proto("moe_ffn_forward_host", _i32, [_vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp])
_forward_static = _proto("moe_ffn_forward_static", _i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp])
_rms = _proto("moe_rms_norm_bf16", _i32, [_vp, _i32, _i32, _vp, _vp])
_stack_ws = _proto("moe_stack_workspace_bytes", _sz, [_vp, _i32, _i32])
_stack = _proto("moe_stack_forward", _i32, [_vp, _i32, _vp, _vp, _i32, _vp, _vp, _sz, _vp])
_pf_ws_bytes = _proto("moe_prefill_workspace_bytes", _sz, [_vp, _i32])
_debug_fault = _proto("rfx_debug_set_fault", _i32, [_i32, ctypes.c_longlong])
_prefill = _proto("moe_ffn_prefill", _i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp])
_pf_ws_bytes_ex = _proto("moe_prefill_workspace_bytes_ex", _sz, [_vp, _i32, _i32])
_prefill_ex = _proto("moe_ffn_prefill_ex", _i32, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _i32, _vp])
RFX_PREFILL_BF16, RFX_PREFILL_EXACT = 0, 1


class moe_prefill_ws_view(ctypes.Structure):
    _fields_ = [("counts", _vp), ("row_token", _vp), ("row_weight", _vp), ("h", _vp),
                ("routed_rows", _i64), ("h_rows", _i64), ("h_lo", _vp)]


_pf_view = _proto("moe_prefill_view", _i32, [_vp, _i32, _vp, ctypes.POINTER(moe_prefill_ws_view)])

EXPORTED = ["rfx_last_error", "rfx_packed_bytes", "rfx_pack", "rfx_unpack", "rfx_pack_device", "moe_router_topk",
            "rfx_gemv_q", "moe_layer_create", "moe_layer_create_mix", "moe_layer_destroy", "moe_ffn_workspace_bytes", "rfx_ws_init",
            "rfx_ws_status", "moe_ffn_forward", "moe_ffn_forward_logits", "moe_ffn_forward_static", "moe_rms_norm_bf16",
            "moe_stack_workspace_bytes", "moe_stack_forward", "moe_prefill_workspace_bytes", "moe_ffn_prefill",
            "moe_prefill_workspace_bytes_ex", "moe_ffn_prefill_ex",
            "moe_prefill_view", "moe_router_logits", "moe_router_project_topk",
            "moe_ffn_host_scratch_bytes", "moe_ffn_forward_host", "rfx_debug_set_fault"]


class RfxError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"rfx status {code}: {msg}")
        self.code = code


def rfx_last_error() -> str:
    return _lib_last_error().decode()


def _check(rc: int):
    if rc != RFX_OK:
        raise RfxError(rc, rfx_last_error())


def _ptr(t) -> int | None:
    """Device pointer of a torch tensor, host pointer of a numpy array, or an int."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ format ---

def rfx_packed_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(_packed_bytes(fmt, rows, cols))


def rfx_pack(fmt: int, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, cols = codes.shape
    scales = np.ascontiguousarray(scales, dtype=np.uint8 if fmt == RFX_FP4 else np.uint16)
    out = np.empty(rfx_packed_bytes(fmt, rows, cols), dtype=np.uint8)
    _check(_pack(fmt, _ptr(codes), _ptr(scales), rows, cols, _ptr(out), out.nbytes))
    return out


def rfx_unpack(fmt: int, packed: np.ndarray, rows: int, cols: int):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes = np.empty((rows, cols), dtype=np.uint8)
    scales = np.empty((rows, cols // 32), dtype=np.uint8 if fmt == RFX_FP4 else np.uint16)
    _check(_unpack(fmt, _ptr(packed), rows, cols, _ptr(codes), _ptr(scales)))
    return codes, scales


def rfx_pack_device(fmt: int, codes, scales, rows: int, cols: int, dst, stream=None):
    """Pack device arrays (torch uint8 codes [rows][cols], scales) into device dst."""
    _check(_pack_device(fmt, _ptr(codes), _ptr(scales), rows, cols, _ptr(dst), _stream(stream)))


# ---------------------------------------------------------------- kernels ---

def moe_router_topk(logits, k: int, idx, w, stream=None):
    """logits fp32 [T][E] (device) -> idx int32 [T][k], w fp32 [T][k] (device, preallocated)."""
    T, E = logits.shape
    _check(_router(_ptr(logits), T, E, k, _ptr(idx), _ptr(w), _stream(stream)))


def moe_router_logits(w_router, bias, x, logits, stream=None):
    """logits fp32 [T][E] = W x + bias for w_router bf16 [E][H], bias fp32 [E] or
    None, x bf16 [T][H] (device tensors)."""
    E, H = w_router.shape
    T = x.shape[0]
    _check(_router_logits(_ptr(w_router), _ptr(bias), _ptr(x), T, H, E, _ptr(logits), _stream(stream)))


def moe_router_project_topk(w_router, bias, x, k: int, logits, idx, w, stream=None):
    """moe_router_logits, then moe_router_topk: fills logits [T][E], idx [T][k], w [T][k]."""
    E, H = w_router.shape
    T = x.shape[0]
    _check(_router_proj_topk(_ptr(w_router), _ptr(bias), _ptr(x), T, H, E, k, _ptr(logits), _ptr(idx), _ptr(w),
                             _stream(stream)))


def rfx_gemv_q(fmt: int, W, N: int, K: int, x, y, stream=None):
    """y fp32 [q][N] = dequant(W) x for x bf16 [q][K] or fp32 [q][K] (device tensors)."""
    import torch
    q = x.shape[0]
    x_is_fp32 = 1 if x.dtype == torch.float32 else 0
    _check(_gemv(fmt, _ptr(W), N, K, _ptr(x), x_is_fp32, q, _ptr(y), _stream(stream)))


def moe_layer_create(desc: moe_layer_desc) -> int:
    h = _vp()
    _check(_layer_create(ctypes.byref(desc), ctypes.byref(h)))
    return h.value


def moe_layer_create_mix(desc: moe_layer_desc, mix) -> int:
    """mix: E tuples (f_gate_up, f_down, off_gate, off_up, off_down)."""
    arr = (moe_expert_mix * len(mix))(*[moe_expert_mix(*m) for m in mix])
    h = _vp()
    _check(_layer_create_mix(ctypes.byref(desc), arr, ctypes.byref(h)))
    return h.value


def moe_layer_destroy(handle: int):
    _layer_destroy(handle)


def moe_ffn_workspace_bytes(handle: int, T: int) -> int:
    return int(_ws_bytes(handle, T))


def rfx_ws_init(ws, stream=None):
    _check(_ws_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def rfx_ws_status(ws, stream=None) -> int:
    rc = int(_ws_status(_ptr(ws), _stream(stream)))
    return rc


def moe_ffn_forward(handle: int, x, T: int, idx, w, y, ws, stream=None):
    _check(_forward(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                    _stream(stream)))


def moe_ffn_forward_logits(handle: int, x, T: int, logits, idx, w, y, ws, stream=None):
    """Router top-k of logits (fp32 [T][E]) into idx / w, then the MoE FFN
    (moe_router_topk + moe_ffn_forward in one call)."""
    _check(_forward_logits(handle, _ptr(x), T, _ptr(logits), _ptr(idx), _ptr(w), _ptr(y), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)))


def moe_ffn_host_scratch_bytes(handle: int, T: int) -> int:
    return int(_host_scratch(handle, T))


def moe_ffn_forward_host(handle: int, x, logits, T: int, y, scratch, stream=None):
    """Router + MoE FFN from host buffers (x bf16 [T][H], logits fp32 [T][E], y fp32
    [T][H], pinned CPU tensors or arrays); scratch: device, zeroed once."""
    _check(_forward_host(handle, _ptr(x), _ptr(logits), T, _ptr(y), _ptr(scratch),
                         scratch.numel() * scratch.element_size(), _stream(stream)))


def moe_ffn_forward_static(handle: int, x, T: int, idx, w, y, stream=None):
    """moe_ffn_forward with the library's built-in 16 MiB workspace, for callers
    that cannot allocate device memory (see include/rfx.h)."""
    _check(_forward_static(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y), _stream(stream)))


def rfx_debug_set_fault(fault: int, wait_cycles: int = 0):
    """Test hook of the device error path (rfx.h): plant a wait that cannot end
    and shorten every bounded wait; fault=0, wait_cycles=0 restores normal use."""
    _check(_debug_fault(fault, wait_cycles))


def moe_rms_norm_bf16(y, x_next, stream=None):
    """y fp32 [T][H] -> x_next bf16 [T][H] = bf16(y / sqrt(mean(y^2))) per column (device tensors)."""
    T, H = y.shape
    _check(_rms(_ptr(y), T, H, _ptr(x_next), _stream(stream)))


def _handles(layers):
    arr = (_vp * len(layers))(*[(l.handle if hasattr(l, "handle") else l) for l in layers])
    return arr


def moe_stack_workspace_bytes(layers, T: int) -> int:
    return int(_stack_ws(_handles(layers), len(layers), T))


def moe_stack_forward(layers, logits, x, y, ws, stream=None):
    """L layers (MoeLayer or handles); logits fp32 [L][T][E], x bf16 [T][H], y fp32 [T][H] (device)."""
    T = x.shape[0]
    _check(_stack(_handles(layers), len(layers), _ptr(logits), _ptr(x), T, _ptr(y), _ptr(ws),
                  ws.numel() * ws.element_size(), _stream(stream)))


def moe_prefill_workspace_bytes(handle: int, T: int) -> int:
    return int(_pf_ws_bytes(handle, T))


def moe_ffn_prefill(handle: int, x, T: int, idx, w, y, ws, stream=None):
    """Grouped-GEMM prefill (bf16 operands, tcgen05): x bf16 [T][H], idx int32 [T][k],
    w fp32 [T][k], y fp32 [T][H], ws uint8 (moe_prefill_workspace_bytes), all device."""
    _check(_prefill(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                    _stream(stream)))


def moe_prefill_workspace_bytes_ex(handle: int, T: int, precision: int) -> int:
    return int(_pf_ws_bytes_ex(handle, T, precision))


def moe_ffn_prefill_ex(handle: int, x, T: int, idx, w, y, ws, precision: int, stream=None):
    """moe_ffn_prefill at a chosen precision (RFX_PREFILL_BF16 or RFX_PREFILL_EXACT)."""
    _check(_prefill_ex(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                       precision, _stream(stream)))


def moe_prefill_view(handle: int, T: int, ws, I: int, E: int):
    """Tensors viewing a prefill workspace after a call: counts int32 [E], row_token
    int32 [T*k], row_weight fp32 [T*k], h bf16 bits int16 [T*k + T][I]."""
    import torch
    v = moe_prefill_ws_view()
    _check(_pf_view(handle, T, _ptr(ws), ctypes.byref(v)))
    base = ws.data_ptr()

    def sub(ptr, nbytes, dtype):
        off = int(ptr) - base
        return ws[off:off + nbytes].view(dtype)

    rr, hr = int(v.routed_rows), int(v.h_rows)
    return {"counts": sub(v.counts, 4 * E, torch.int32), "row_token": sub(v.row_token, 4 * rr, torch.int32),
            "row_weight": sub(v.row_weight, 4 * rr, torch.float32),
            "h": sub(v.h, 2 * hr * I, torch.int16).view(hr, I),
            "h_lo": sub(v.h_lo, 2 * hr * I, torch.int16).view(hr, I) if int(v.h_lo) + 2 * hr * I <= base + ws.numel()
            else None}


# --------------------------------------------------------- convenience ---

class MoeLayer:
    """One MoE layer over caller-owned packed device buffers.

    ``gate``/``up``/``down`` are uint8 device tensors holding E packed experts
    at a fixed stride (or, with ``mix``, at the table's offsets in the table's
    formats); ``shared`` is (gate, up, down) or None.  Creates the
    host handle and a zeroed workspace for up to ``max_T`` token columns.
    """

    def __init__(self, H, I, E, k, fmts, gate, up, down, strides, shared=None, shared_fmts=(4, 4, 4), max_T=MAX_T,
                 mix=None):
        import torch
        self.H, self.I, self.E, self.k = H, I, E, k
        self._keep = [gate, up, down] + (list(shared) if shared else [])
        d = moe_layer_desc()
        d.H, d.I, d.E, d.k = H, I, E, k
        d.f_gate, d.f_up, d.f_down = fmts
        d.gate, d.up, d.down = _ptr(gate), _ptr(up), _ptr(down)
        d.stride_gate, d.stride_up, d.stride_down = strides
        d.has_shared = 1 if shared else 0
        if shared:
            d.f_sh_gate, d.f_sh_up, d.f_sh_down = shared_fmts
            d.sh_gate, d.sh_up, d.sh_down = (_ptr(s) for s in shared)
        self.desc = d
        # mix: ROCmFPX MIX table, E tuples (f_gate_up, f_down, off_gate, off_up, off_down)
        self.handle = moe_layer_create(d) if mix is None else moe_layer_create_mix(d, mix)
        self.max_T = max_T
        nbytes = moe_ffn_workspace_bytes(self.handle, max_T)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=gate.device)
        rfx_ws_init(self.ws)

    def forward(self, x, idx, w, y, stream=None):
        T = x.shape[0]
        if T > self.max_T:
            raise ValueError(f"T={T} > max_T={self.max_T}")
        moe_ffn_forward(self.handle, x, T, idx, w, y, self.ws, stream)

    def forward_logits(self, x, logits, idx, w, y, stream=None):
        """Routing from the logits, then the FFN (moe_ffn_forward_logits)."""
        T = x.shape[0]
        if T > self.max_T:
            raise ValueError(f"T={T} > max_T={self.max_T}")
        moe_ffn_forward_logits(self.handle, x, T, logits, idx, w, y, self.ws, stream)

    def forward_host(self, x, logits, y, stream=None):
        """Router + FFN from host buffers (see moe_ffn_forward_host); the device
        scratch is kept on the layer (grown on demand, zeroed when made)."""
        import torch
        T = x.shape[0]
        nbytes = moe_ffn_host_scratch_bytes(self.handle, T)
        if nbytes == 0:
            raise RfxError(-2, f"unsupported T={T}")
        if getattr(self, "host_scratch", None) is None or self.host_scratch.numel() < nbytes:
            self.host_scratch = torch.empty(nbytes, dtype=torch.uint8, device=self.ws.device)
            rfx_ws_init(self.host_scratch)
        moe_ffn_forward_host(self.handle, x, logits, T, y, self.host_scratch, stream)

    def host_status(self, stream=None) -> int:
        """Device flag of the host-call scratch (its workspace comes first)."""
        return rfx_ws_status(self.host_scratch, stream)

    def prefill(self, x, idx, w, y, stream=None, exact=False):
        """moe_ffn_prefill (exact: moe_ffn_prefill_ex at RFX_PREFILL_EXACT) with a
        workspace kept on the layer (grown on demand)."""
        import torch
        T = x.shape[0]
        prec = RFX_PREFILL_EXACT if exact else RFX_PREFILL_BF16
        nbytes = moe_prefill_workspace_bytes_ex(self.handle, T, prec)
        if nbytes == 0:
            raise RfxError(-2, f"prefill unsupported for T={T}, H={self.H}, I={self.I}")
        if getattr(self, "pf_ws", None) is None or self.pf_ws.numel() < nbytes:
            self.pf_ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
            rfx_ws_init(self.pf_ws)
        if exact:
            moe_ffn_prefill_ex(self.handle, x, T, idx, w, y, self.pf_ws, prec, stream)
        else:
            moe_ffn_prefill(self.handle, x, T, idx, w, y, self.pf_ws, stream)

    def prefill_view(self, T: int):
        return moe_prefill_view(self.handle, T, self.pf_ws, self.I, self.E)

    def prefill_status(self, stream=None) -> int:
        return rfx_ws_status(self.pf_ws, stream)

    def status(self, stream=None) -> int:
        return rfx_ws_status(self.ws, stream)

    def __del__(self):
        try:
            if getattr(self, "handle", None):
                moe_layer_destroy(self.handle)
                self.handle = None
        except Exception:
            pass

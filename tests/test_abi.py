"""C-ABI library on the host: symbols, packed layout, argument checks.

No kernel is launched here (no GPU needed): the packer is host code and every
argument error is detected before any CUDA call.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import block_quantized_moe_rocmfpx_b200 as rfx
import synth
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "rfx.h")


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", txt)
    skip = {"if", "sizeof", "defined"}
    return sorted({n for n in names if n not in skip and (n.startswith("rfx_") or n.startswith("moe_"))})


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(rfx.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rfx.EXPORTED)


@pytest.mark.parametrize("fmt", [2, 3, 4])
def test_packed_bytes_is_block_bytes(fmt):
    bb = {2: 10, 3: 14, 4: 17}[fmt]
    assert rfx.rfx_packed_bytes(fmt, 2048, 4096) == 2048 * 128 * bb
    assert rfx.rfx_packed_bytes(fmt, 17, 64) == 32 * 2 * bb        # rows padded to 16
    assert rfx.rfx_packed_bytes(fmt, 16, 48) == 0                  # cols % 32 != 0
    assert rfx.rfx_packed_bytes(7, 16, 64) == 0


@pytest.mark.parametrize("fmt", [2, 3, 4])
@pytest.mark.parametrize("rows,cols", [(16, 256), (48, 4096), (33, 352), (16, 160), (5, 32), (64, 96)])
def test_pack_unpack_round_trip(fmt, rows, cols):
    spec = synth.MatrixSpec(1, 0, 0, 0, fmt, rows, cols)
    c, s = spec.codes(), spec.scales()
    packed = rfx.rfx_pack(fmt, c, s)
    assert packed.nbytes == rfx.rfx_packed_bytes(fmt, rows, cols)
    c2, s2 = rfx.rfx_unpack(fmt, packed, rows, cols)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)


@pytest.mark.parametrize("fmt", [2, 3, 4])
def test_pack_extreme_codes(fmt):
    rows, cols = 32, 512
    for c0 in (0, (1 << fmt) - 1):
        c = np.full((rows, cols), c0, np.uint8)
        s = np.full((rows, cols // 32), 0x7BFF if fmt != 4 else 0xFE, np.uint16 if fmt != 4 else np.uint8)
        c2, s2 = rfx.rfx_unpack(fmt, rfx.rfx_pack(fmt, c, s), rows, cols)
        assert np.array_equal(c, c2) and np.array_equal(s, s2)


def _reg_coords(g, t, r):
    m, j = r >> 2, r & 3
    return g + 8 * (j & 1), 16 * m + 2 * t + 8 * (j >> 1)


def _full_field(fmt, b, r):
    """(word, offset, spare) of register r of tile b in a full chunk, as rfx.h states."""
    if fmt == 2:
        return r, 2 * b, False
    if fmt == 4:
        return (r if b < 4 else 8 + r), 4 * (b & 3), False
    if b < 5:
        return r, 3 * b, False
    if b < 7:
        return (8 + r, 3 * (b - 5), False) if r < 4 else (4 + r, 3 * (b - 2), False)
    return (8 + r, 6, False) if r < 4 else (3 * (r - 4), 0, True)


def test_layout_matches_header_description():
    """Rebuild packed chunks from the bit positions rfx.h documents."""
    rows, cols = 16, 256 + 96          # one full chunk and one partial chunk of 3 tiles
    for fmt in (2, 3, 4):
        spec = synth.MatrixSpec(4, 0, 1, 0, fmt, rows, cols)
        c, s = spec.codes(), spec.scales()
        packed = rfx.rfx_pack(fmt, c, s)
        m = (1 << fmt) - 1
        # full chunk 0: plane layout, slab-major words
        for L in (0, 5, 31):
            g, t = L >> 2, L & 3
            words = [int(np.frombuffer(packed[((w // 4) * 32 + L) * 16 + (w % 4) * 4:][:4].tobytes(), np.uint32)[0])
                     for w in range(4 * fmt)]
            for b in range(8):
                for r in range(8):
                    row, k = _reg_coords(g, t, r)
                    lo, hi = int(c[row, 32 * b + k]), int(c[row, 32 * b + k + 1])
                    wi, f, spare = _full_field(fmt, b, r)
                    if not spare:
                        assert (words[wi] >> f) & m == lo and (words[wi] >> (16 + f)) & m == hi
                    else:
                        assert sum(((words[wi + i] >> 15) & 1) << i for i in range(3)) == lo
                        assert sum(((words[wi + i] >> 31) & 1) << i for i in range(3)) == hi
        # partial chunk 1 (3 tiles): tile layout
        chunk1 = packed[8 * 16 * (4 * fmt + (1 if fmt == 4 else 2)):]
        nt = 3
        for L in (0, 9, 31):
            g, t = L >> 2, L & 3
            lane = chunk1[L * nt * 2 * fmt:(L + 1) * nt * 2 * fmt].tobytes()
            for b in range(nt):
                for r in range(8):
                    row, k = _reg_coords(g, t, r)
                    kk = 256 + 32 * b + k
                    lo, hi = int(c[row, kk]), int(c[row, kk + 1])
                    if fmt == 2:
                        w = int(np.frombuffer(lane[4 * b:4 * b + 4], np.uint32)[0])
                        assert (w >> (2 * r)) & 3 == lo and (w >> (16 + 2 * r)) & 3 == hi
                    elif fmt == 4:
                        w = int(np.frombuffer(lane[8 * b + 4 * (r >> 2):8 * b + 4 * (r >> 2) + 4], np.uint32)[0])
                        j = r & 3
                        assert (w >> (4 * j)) & 15 == lo and (w >> (16 + 4 * j)) & 15 == hi
                    else:
                        if b < 2:   # pair (0, 1): 3 words
                            ws = [int(v) for v in np.frombuffer(lane[0:12], np.uint32)]
                            R = 8 * b + r
                            if R < 15:
                                w, p_ = ws[R // 5], R % 5
                                assert (w >> (3 * p_)) & 7 == lo and (w >> (16 + 3 * p_)) & 7 == hi
                            else:
                                assert sum(((ws[i] >> 15) & 1) << i for i in range(3)) == lo
                                assert sum(((ws[i] >> 31) & 1) << i for i in range(3)) == hi
                        else:       # lone tile 2: 48-bit stream
                            st = int.from_bytes(lane[12:18], "little")
                            assert (st >> (3 * (2 * r))) & 7 == lo and (st >> (3 * (2 * r + 1))) & 7 == hi
        # scales of the first (full) chunk: E8M0 [g][tile][row g, row g+8] bytes; binary16 at
        # ((b/4)*8 + g)*16 + (b%4)*4 + 2h
        sb = 1 if fmt == 4 else 2
        sc = packed[8 * 16 * 4 * fmt: 8 * 16 * 4 * fmt + 8 * 8 * 2 * sb].tobytes()
        for g in range(8):
            for b in range(8):
                for h in range(2):
                    if fmt == 4:
                        got = sc[(g * 8 + b) * 2 + h]
                    else:
                        o = ((b // 4) * 8 + g) * 16 + (b % 4) * 4 + 2 * h
                        got = int(np.frombuffer(sc[o:o + 2], np.uint16)[0])
                    assert got == s[g + 8 * h, b]
        # scales of the partial chunk 1: [g][tile][row g, row g+8]
        sc1 = chunk1[nt * 16 * 4 * fmt: nt * 16 * 4 * fmt + 8 * nt * 2 * sb].tobytes()
        sc1 = np.frombuffer(sc1, dtype=np.uint8 if fmt == 4 else np.uint16).reshape(8, nt, 2)
        for g in range(8):
            for b in range(nt):
                assert sc1[g, b, 0] == s[g, 8 + b] and sc1[g, b, 1] == s[g + 8, 8 + b]


def test_pack_rejects_bad_values():
    c = np.zeros((16, 64), np.uint8)
    s16 = np.full((16, 2), 0x3C00, np.uint16)
    with pytest.raises(rfx.RfxError) as e:
        rfx.rfx_pack(2, np.full((16, 64), 4, np.uint8), s16)
    assert e.value.code == rfx.RFX_EINVAL
    with pytest.raises(rfx.RfxError):
        rfx.rfx_pack(3, c, np.full((16, 2), 0x7C00, np.uint16))      # inf scale
    with pytest.raises(rfx.RfxError):
        rfx.rfx_pack(4, c, np.full((16, 2), 0xFF, np.uint8))          # E8M0 NaN
    with pytest.raises(rfx.RfxError):
        rfx.rfx_pack(5, c, s16)
    assert "rfx_pack" in rfx.rfx_last_error()


def test_device_calls_reject_bad_arguments_before_cuda():
    lib = ctypes.CDLL(rfx.LIB_PATH)
    assert lib.moe_router_topk(None, -1, 256, 6, None, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_topk(None, 4, 256, 0, None, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_topk(None, 4, 8, 9, None, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_topk(None, 0, 256, 6, None, None, None) == rfx.RFX_OK       # T = 0: no-op
    assert lib.rfx_gemv_q(2, None, 16, 64, None, 0, 9, None, None) == rfx.RFX_EUNSUPPORTED
    assert lib.rfx_gemv_q(2, None, 16, 48, None, 0, 1, None, None) == rfx.RFX_EINVAL
    assert lib.rfx_gemv_q(6, None, 16, 64, None, 0, 1, None, None) == rfx.RFX_EINVAL
    # router projection: H a positive multiple of 32, E >= 1, T >= 0, aligned operands
    assert lib.moe_router_logits(None, None, None, 4, 48, 256, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_logits(None, None, None, 4, 64, 0, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_logits(None, None, None, -1, 64, 8, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_logits(None, None, None, 0, 64, 8, None, None) == rfx.RFX_OK      # T = 0: no-op
    assert lib.moe_router_logits(None, None, None, 2, 64, 8, None, None) == rfx.RFX_EINVAL  # null pointers
    assert lib.moe_router_logits(ctypes.c_void_p(0x1008), None, ctypes.c_void_p(0x2000), 2, 64, 8,
                                 ctypes.c_void_p(0x3000), None) == rfx.RFX_EINVAL             # W not 16-byte aligned
    assert lib.moe_router_project_topk(None, None, None, 1, 64, 8, 9, None, None, None, None) == rfx.RFX_EINVAL
    assert lib.moe_router_project_topk(None, None, None, 1, 64, 2000, 6, None, None, None, None) == rfx.RFX_EINVAL


def test_layer_create_validation():
    d = rfx.moe_layer_desc()
    d.H, d.I, d.E, d.k = 4096, 2048, 256, 6
    d.f_gate, d.f_up, d.f_down = 2, 2, 3
    d.gate = d.up = d.down = 256
    d.stride_gate = d.stride_up = rfx.rfx_packed_bytes(2, 2048, 4096)
    d.stride_down = rfx.rfx_packed_bytes(3, 4096, 2048)
    h = rfx.moe_layer_create(d)
    assert h
    assert rfx.moe_ffn_workspace_bytes(h, 4) > 0
    # T > 8 takes the prefill path and its workspace
    assert rfx.moe_ffn_workspace_bytes(h, 9) == rfx.moe_prefill_workspace_bytes(h, 9) > 0
    assert rfx.moe_prefill_workspace_bytes(h, 0) == 0 and rfx.moe_ffn_workspace_bytes(h, 0) == 0
    rfx.moe_layer_destroy(h)
    for field, val in (("H", 100), ("k", 9), ("f_up", 3), ("stride_down", 16), ("gate", 8), ("E", 2000)):
        bad = rfx.moe_layer_desc.from_buffer_copy(d)
        setattr(bad, field, val)
        with pytest.raises(rfx.RfxError):
            rfx.moe_layer_create(bad)
    bad = rfx.moe_layer_desc.from_buffer_copy(d)
    bad.has_shared = 1
    with pytest.raises(rfx.RfxError):          # shared pointers missing
        rfx.moe_layer_create(bad)
    lib = ctypes.CDLL(rfx.LIB_PATH)
    assert lib.moe_ffn_forward(None, None, 1, None, None, None, None, 0, None) == rfx.RFX_EINVAL


def test_mix_layer_create_validation():
    """moe_layer_create_mix checks every entry before it touches the device:
    formats 2..4 and 16-byte offsets; the descriptor's own checks still apply."""
    d = rfx.moe_layer_desc()
    d.H, d.I, d.E, d.k = 512, 256, 3, 2
    d.f_gate = d.f_up = d.f_down = 9          # ignored by the MIX entry point
    d.gate = d.up = d.down = 256
    good = [(2, 3, 0, 0, 0), (3, 3, 4096, 4096, 4096), (4, 2, 8192, 8192, 8192)]
    for e, bad_entry in ((1, (5, 3, 4096, 4096, 4096)), (2, (4, 1, 8192, 8192, 8192)),
                         (1, (3, 3, 4100, 4096, 4096)), (2, (4, 2, 8192, 8192, 8200))):
        mix = list(good)
        mix[e] = bad_entry
        with pytest.raises(rfx.RfxError) as ei:
            rfx.moe_layer_create_mix(d, mix)
        assert ei.value.code == rfx.RFX_EINVAL
    bad = rfx.moe_layer_desc.from_buffer_copy(d)
    bad.k = 4                                   # k > E
    with pytest.raises(rfx.RfxError):
        rfx.moe_layer_create_mix(bad, good)


def test_heat_mix_gives_hot_experts_the_widest_codebooks():
    from synth.layers import heat_mix
    mix = heat_mix(0, 0, 256, 1.1)
    order = np.argsort(-synth.zipf_bias(0, 0, 256, 1.1), kind="stable")
    assert [mix[e] for e in order[:32]] == [(4, 4)] * 32
    assert {mix[e] for e in order[32:128]} == {(3, 3)}
    assert {mix[e] for e in order[128:]} == {(2, 3)}


def test_zero_token_calls_are_noops():
    """T = 0 returns OK without touching any buffer (reading: an empty batch is
    a no-op), for every entry point that takes T."""
    lib = ctypes.CDLL(rfx.LIB_PATH)
    d = rfx.moe_layer_desc()
    d.H, d.I, d.E, d.k = 512, 256, 8, 2
    d.f_gate, d.f_up, d.f_down = 2, 2, 3
    d.gate = d.up = d.down = 256
    d.stride_gate = d.stride_up = rfx.rfx_packed_bytes(2, 256, 512)
    d.stride_down = rfx.rfx_packed_bytes(3, 512, 256)
    h = rfx.moe_layer_create(d)
    try:
        assert lib.moe_ffn_forward(ctypes.c_void_p(h), None, 0, None, None, None, None, 0, None) == rfx.RFX_OK
        assert lib.moe_ffn_prefill(ctypes.c_void_p(h), None, 0, None, None, None, None, 0, None) == rfx.RFX_OK
        assert lib.moe_ffn_forward_static(ctypes.c_void_p(h), None, 0, None, None, None, None) == rfx.RFX_OK
        assert lib.moe_ffn_forward_host(ctypes.c_void_p(h), None, None, 0, None, None, 0, None) == rfx.RFX_OK
        assert lib.moe_ffn_forward_logits(ctypes.c_void_p(h), None, 0, None, None, None, None, None, 0,
                                          None) == rfx.RFX_OK
        arr = (ctypes.c_void_p * 1)(h)
        assert lib.moe_stack_forward(arr, 1, None, None, 0, None, None, 0, None) == rfx.RFX_OK
        # a null layer is still an error
        assert lib.moe_ffn_forward(None, None, 0, None, None, None, None, 0, None) == rfx.RFX_EINVAL
        assert lib.moe_ffn_forward_logits(None, None, 1, None, None, None, None, None, 0, None) == rfx.RFX_EINVAL
        # the call from the logits checks its routing buffers before any launch
        assert lib.moe_ffn_forward_logits(ctypes.c_void_p(h), None, 1, None, None, None, None, None, 0,
                                          None) == rfx.RFX_EINVAL
        assert "null pointer" in rfx.rfx_last_error()
    finally:
        rfx.moe_layer_destroy(h)


def test_host_call_scratch_bytes():
    """moe_ffn_host_scratch_bytes = the moe_ffn_forward workspace (decode or
    prefill) + two padded device copies of x and of the logits (used in turn)
    + idx, w and y."""
    d = rfx.moe_layer_desc()
    d.H, d.I, d.E, d.k = 4096, 2048, 256, 6
    d.f_gate, d.f_up, d.f_down = 2, 2, 3
    d.gate = d.up = d.down = 256
    d.stride_gate = d.stride_up = rfx.rfx_packed_bytes(2, 2048, 4096)
    d.stride_down = rfx.rfx_packed_bytes(3, 4096, 2048)
    h = rfx.moe_layer_create(d)
    try:
        up = lambda n: (n + 255) // 256 * 256
        for T in (1, 4, 8, 9, 2048):
            ws = rfx.moe_ffn_workspace_bytes(h, T)
            want = up(ws) + 2 * up(T * 4096 * 2) + 2 * up(T * 256 * 4) + 2 * up(T * 6 * 4) + up(T * 4096 * 4)
            assert rfx.moe_ffn_host_scratch_bytes(h, T) == want, T
        assert rfx.moe_ffn_host_scratch_bytes(h, 0) == 0
    finally:
        rfx.moe_layer_destroy(h)


def test_fault_hook_rejects_bad_arguments():
    with pytest.raises(rfx.RfxError):
        rfx.rfx_debug_set_fault(7, 0)
    with pytest.raises(rfx.RfxError):
        rfx.rfx_debug_set_fault(0, -1)
    rfx.rfx_debug_set_fault(0, 0)

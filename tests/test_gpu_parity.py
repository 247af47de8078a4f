"""GPU (sm_100a) kernels against the fp64 oracle, through the C ABI.

Router indices are compared bit for bit; floating-point outputs must meet
relative L2 <= 1e-5 and |y - y_oracle| <= 1e-4 * sum|w x| per element.
"""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth
from helpers import OracleLayer, check_close, mat
from synth.layers import SynthLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(DEV)


# ------------------------------------------------ generator and packer ---

@pytest.mark.parametrize("fmt,rows,cols", [(2, 64, 4096), (3, 48, 2048), (4, 33, 352)])
def test_device_generator_equals_host(fmt, rows, cols):
    spec = synth.MatrixSpec(9, 2, 1, 17, fmt, rows, cols)
    c = torch.empty(rows * cols, dtype=torch.uint8, device=DEV)
    s = torch.empty(rows * cols // 32 * 2, dtype=torch.uint8, device=DEV)
    synth.codes_dev(spec.code_key, fmt, rows, cols, c)
    synth.scales_dev(spec.scale_key, fmt, rows, cols, s)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy().reshape(rows, cols), spec.codes())
    hs = spec.scales()
    assert np.array_equal(s.cpu().numpy()[:hs.nbytes].view(hs.dtype).reshape(hs.shape), hs)


@pytest.mark.parametrize("fmt", [2, 3, 4])
@pytest.mark.parametrize("rows,cols", [(48, 4096), (33, 352), (16, 160), (7, 32)])
def test_device_pack_equals_host_pack(fmt, rows, cols):
    spec = synth.MatrixSpec(3, 0, 2, 5, fmt, rows, cols)
    c, s = spec.codes(), spec.scales()
    host = rfx.rfx_pack(fmt, c, s)
    dst = torch.full((host.nbytes,), 0xAB, dtype=torch.uint8, device=DEV)
    rfx.rfx_pack_device(fmt, to_dev(c), to_dev(s.view(np.uint8)), rows, cols, dst)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy(), host)


# ------------------------------------------------------------- router ---

@pytest.mark.parametrize("T,E,k", [(64, 256, 6), (5, 8, 2), (3, 16, 16), (7, 1000, 8), (1, 40, 3)])
def test_router_bit_exact(T, E, k):
    L = synth.logits(11, 0, 0, T, E, 1.1 if E == 256 else 0.0)
    L[0, 1] = L[0, E // 2] = L[0, E - 1] = 9.0   # ties go to the lower index
    if T > 1:
        L[1, :] = 0.5                           # all equal
    idx_o, w_o = oracle.router_topk(L, k)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L), k, idx, w)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    np.testing.assert_allclose(w.cpu().numpy(), w_o, rtol=1e-6, atol=0)


# --------------------------------------------------------------- GEMV ---

GEMV_CASES = [
    (2, 2048, 4096), (3, 4096, 2048), (4, 2048, 4096),     # full-size expert matrices
    (2, 40, 352), (3, 33, 160), (4, 24, 96),               # ragged rows, partial chunks, lone FP3 tile
]


@pytest.mark.parametrize("fmt,N,K", GEMV_CASES)
@pytest.mark.parametrize("q", [1, 4, 5, 8])
@pytest.mark.parametrize("xtype", ["bf16", "fp32"])
def test_gemv_matches_oracle(fmt, N, K, q, xtype):
    spec = synth.MatrixSpec(21, 0, 0, fmt, fmt, N, K)
    m = mat(spec)
    W = to_dev(rfx.rfx_pack(fmt, m.codes, m.scales))
    if xtype == "bf16":
        xb = synth.x_bf16(5, 0, q, K)
        x = to_dev(xb, torch.bfloat16)
        xf = synth.bf16_to_f64(xb)
    else:
        xf32 = (synth.normal_f64(synth.key(6, 0, 200, 0), q * K).reshape(q, K) * 3).astype(np.float32)
        x = to_dev(xf32)
        xf = xf32.astype(np.float64)
    y = torch.full((q, N), float("nan"), dtype=torch.float32, device=DEV)
    rfx.rfx_gemv_q(fmt, W, N, K, x, y)
    torch.cuda.synchronize()
    ref, mag = oracle.gemv(m, xf)
    check_close(y.cpu().numpy(), ref, mag, what=f"gemv fmt{fmt} {N}x{K} q{q} {xtype}")


def test_gemv_columns_are_independent_of_q():
    fmt, N, K = 2, 256, 4096
    spec = synth.MatrixSpec(2, 0, 0, 0, fmt, N, K)
    W = to_dev(rfx.rfx_pack(fmt, spec.codes(), spec.scales()))
    xb = synth.x_bf16(1, 0, 5, K)
    y5 = torch.empty((5, N), dtype=torch.float32, device=DEV)
    rfx.rfx_gemv_q(fmt, W, N, K, to_dev(xb, torch.bfloat16), y5)
    for c in range(5):
        y1 = torch.empty((1, N), dtype=torch.float32, device=DEV)
        rfx.rfx_gemv_q(fmt, W, N, K, to_dev(xb[c:c + 1], torch.bfloat16), y1)
        assert torch.equal(y5[c:c + 1], y1)


# ------------------------------------------------------------ MoE FFN ---

def run_layer(lay, L_logits, xb, T, k):
    ml = lay.moe_layer()
    x = to_dev(xb, torch.bfloat16)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L_logits), k, idx, w)
    ml.forward(x, idx, w, y)
    assert ml.status() == rfx.RFX_OK, rfx.rfx_last_error()
    return ml, idx.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_moe_tiny_layer(T):
    H, I, E, k = 512, 256, 8, 2
    lay = SynthLayer(31, 0, H, I, E, k)
    L = synth.logits(31, 0, 0, T, E, 0.0)
    xb = synth.x_bf16(31, 0, T, H)
    _, idx, w, y = run_layer(lay, L, xb, T, k)
    idx_o, w_o = oracle.router_topk(L, k)
    assert np.array_equal(idx, idx_o)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y[t], ref, mag, what=f"tiny T={T} t={t}")


@pytest.mark.parametrize("H,I,E,k,shared", [(352, 160, 6, 3, True), (96, 64, 5, 5, False), (64, 32, 300, 8, True)])
def test_moe_ragged_shapes(H, I, E, k, shared):
    T = 3
    lay = SynthLayer(7, 1, H, I, E, k, has_shared=shared, fmts=(2, 2, 3), shared_fmts=(4, 4, 4))
    L = synth.logits(7, 1, 0, T, E, 0.0)
    xb = synth.x_bf16(7, 0, T, H)
    _, idx, w, y = run_layer(lay, L, xb, T, k)
    idx_o, w_o = oracle.router_topk(L, k)
    assert np.array_equal(idx, idx_o)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y[t], ref, mag, what=f"ragged {H}x{I} t={t}")


@pytest.mark.parametrize("fmts,sfmts", [((3, 3, 2), (2, 2, 3)), ((4, 4, 4), (3, 3, 2))])
def test_moe_other_format_mixes(fmts, sfmts):
    H, I, E, k, T = 512, 256, 8, 2, 4
    lay = SynthLayer(13, 0, H, I, E, k, fmts=fmts, shared_fmts=sfmts)
    L = synth.logits(13, 0, 0, T, E, 0.0)
    xb = synth.x_bf16(13, 0, T, H)
    _, idx, w, y = run_layer(lay, L, xb, T, k)
    idx_o, w_o = oracle.router_topk(L, k)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y[t], ref, mag, what=f"mix {fmts}/{sfmts} t={t}")


@pytest.fixture(scope="module")
def full_layer():
    return SynthLayer(0, 0, 4096, 2048, 256, 6)


@pytest.mark.parametrize("T", [1, 4])
def test_moe_full_size_layer(full_layer, T):
    lay = full_layer
    L = synth.logits(0, 0, 100, T, 256, 1.1)
    xb = synth.x_bf16(0, 100, T, 4096)
    ml, idx, w, y = run_layer(lay, L, xb, T, 6)
    idx_o, w_o = oracle.router_topk(L, 6)
    assert np.array_equal(idx, idx_o)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y[t], ref, mag, what=f"full T={T} t={t}")
    # decode once, apply to every column: each column equals its own 1-column pass, bit for bit
    if T > 1:
        for t in range(T):
            _, _, _, y1 = run_layer(lay, L[t:t + 1], xb[t:t + 1], 1, 6)
            assert np.array_equal(y1[0], y[t])


def test_moe_repeated_calls_reuse_workspace(full_layer):
    lay = full_layer
    ml = lay.moe_layer()
    T = 4
    outs = []
    for rep in range(3):
        L = synth.logits(0, 0, 10 * rep, T, 256, 1.1)
        xb = synth.x_bf16(0, 10 * rep, T, 4096)
        idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
        w = torch.empty((T, 6), dtype=torch.float32, device=DEV)
        y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(to_dev(L), 6, idx, w)
        ml.forward(to_dev(xb, torch.bfloat16), idx, w, y)
        outs.append(y.clone())
        ml.forward(to_dev(xb, torch.bfloat16), idx, w, y)      # same inputs again: same bits
        assert torch.equal(outs[-1], y)
    assert ml.status() == rfx.RFX_OK


def test_moe_bad_expert_ids_set_the_device_flag(full_layer):
    ml = full_layer.moe_layer()
    T = 2
    x = to_dev(synth.x_bf16(1, 0, T, 4096), torch.bfloat16)
    idx = torch.tensor([[1, 2, 3, 4, 5, 300], [7, 7, 1, 2, 3, 4]], dtype=torch.int32, device=DEV)
    w = torch.full((T, 6), 1 / 6, dtype=torch.float32, device=DEV)
    y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
    ml.forward(x, idx, w, y)
    assert ml.status() == rfx.RFX_EDEVICE
    assert ml.status() == rfx.RFX_OK          # the flag is cleared once read


@pytest.mark.parametrize("T", [1, 4])
def test_forward_host_equals_device_path(full_layer, T):
    """moe_ffn_forward_host (host x / logits in, host y out, one call) gives the
    bits of the router call and moe_ffn_forward on device buffers."""
    ml = full_layer.moe_layer()
    L = synth.logits(8, 0, 60 * T, T, 256, 1.1)
    xb = synth.x_bf16(8, 60 * T, T, 4096)
    idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 6), dtype=torch.float32, device=DEV)
    y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L), 6, idx, w)
    ml.forward(to_dev(xb, torch.bfloat16), idx, w, y)
    xh = torch.from_numpy(xb).view(torch.bfloat16).pin_memory()
    lh = torch.from_numpy(L).pin_memory()
    yh = torch.full((T, 4096), float("nan"), dtype=torch.float32).pin_memory()
    for _ in range(2):                          # the scratch is reused
        ml.forward_host(xh, lh, yh)
        torch.cuda.synchronize()
        assert torch.equal(yh, y.cpu())
    assert ml.host_status() == rfx.RFX_OK
    assert ml.status() == rfx.RFX_OK


def test_forward_host_pipelined_calls(full_layer):
    """Back-to-back host-buffer calls with no synchronisation between them:
    each call's uploads overlap the previous call's kernels (two device buffer
    sets in turn); every y equals the device path's bits for its own inputs."""
    ml = full_layer.moe_layer()
    T, n = 2, 6
    Ls = [synth.logits(9, 0, 100 + 7 * i, T, 256, 1.1) for i in range(n)]
    xbs = [synth.x_bf16(9, 100 + 7 * i, T, 4096) for i in range(n)]
    xh = [torch.from_numpy(a).view(torch.bfloat16).pin_memory() for a in xbs]
    lh = [torch.from_numpy(a).pin_memory() for a in Ls]
    yh = [torch.full((T, 4096), float("nan"), dtype=torch.float32).pin_memory() for _ in range(n)]
    for i in range(n):
        ml.forward_host(xh[i], lh[i], yh[i])
    torch.cuda.synchronize()
    assert ml.host_status() == rfx.RFX_OK
    for i in range(n):
        idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
        w = torch.empty((T, 6), dtype=torch.float32, device=DEV)
        y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(to_dev(Ls[i]), 6, idx, w)
        ml.forward(to_dev(xbs[i], torch.bfloat16), idx, w, y)
        assert torch.equal(yh[i], y.cpu()), f"call {i}"


def test_forward_host_pageable_buffers(full_layer):
    """Pageable (not page-locked) host buffers: the copies path, same bits."""
    ml = full_layer.moe_layer()
    T = 3
    L = synth.logits(10, 0, 5, T, 256, 1.1)
    xb = synth.x_bf16(10, 5, T, 4096)
    idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 6), dtype=torch.float32, device=DEV)
    y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L), 6, idx, w)
    ml.forward(to_dev(xb, torch.bfloat16), idx, w, y)
    yh = torch.full((T, 4096), float("nan"), dtype=torch.float32)    # pageable
    ml.forward_host(torch.from_numpy(xb).view(torch.bfloat16), torch.from_numpy(L), yh)
    torch.cuda.synchronize()
    assert torch.equal(yh, y.cpu())


def test_forward_host_mixed_paths(full_layer):
    """Back-to-back host-buffer calls on one layer that alternate the buffer
    kinds: all page-locked (y stored by the kernel straight into host memory),
    page-locked inputs with pageable y (y copied back), all pageable; no
    synchronisation between the calls, every y the device path's bits for its
    own inputs."""
    ml = full_layer.moe_layer()
    T, n = 2, 6
    Ls = [synth.logits(12, 0, 300 + 7 * i, T, 256, 1.1) for i in range(n)]
    xbs = [synth.x_bf16(12, 300 + 7 * i, T, 4096) for i in range(n)]
    ys = []
    for i in range(n):
        pin_in, pin_out = i % 3 != 2, i % 3 == 0
        xh = torch.from_numpy(xbs[i]).view(torch.bfloat16)
        lh = torch.from_numpy(Ls[i])
        yh = torch.full((T, 4096), float("nan"), dtype=torch.float32)
        if pin_in:
            xh, lh = xh.pin_memory(), lh.pin_memory()
        if pin_out:
            yh = yh.pin_memory()
        ml.forward_host(xh, lh, yh)
        ys.append((yh, xh, lh))
    torch.cuda.synchronize()
    assert ml.host_status() == rfx.RFX_OK
    for i in range(n):
        idx = torch.empty((T, 6), dtype=torch.int32, device=DEV)
        w = torch.empty((T, 6), dtype=torch.float32, device=DEV)
        y = torch.empty((T, 4096), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(to_dev(Ls[i]), 6, idx, w)
        ml.forward(to_dev(xbs[i], torch.bfloat16), idx, w, y)
        assert torch.equal(ys[i][0], y.cpu()), f"call {i}"


def test_forward_host_prefill_path():
    H, I, E, k, T = 512, 256, 16, 4, 40
    lay = SynthLayer(29, 0, H, I, E, k)
    ml = lay.moe_layer(max_T=T)
    L = synth.logits(29, 0, 0, T, E, 1.1)
    xb = synth.x_bf16(29, 0, T, H)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L), k, idx, w)
    ml.prefill(to_dev(xb, torch.bfloat16), idx, w, y)
    yh = torch.empty((T, H), dtype=torch.float32).pin_memory()
    ml.forward_host(torch.from_numpy(xb).view(torch.bfloat16).pin_memory(), torch.from_numpy(L).pin_memory(), yh)
    torch.cuda.synchronize()
    # the prefill combine adds with fp32 atomics: equal up to the order of the adds
    assert torch.allclose(yh, y.cpu(), rtol=1e-5, atol=1e-5)
    assert ml.host_status() == rfx.RFX_OK


@pytest.mark.parametrize("T", [1, 3])
def test_moe_wide_hidden_top8(T):
    """H = 7168 (a DeepSeek-V3-like hidden size), top-8 of 256 + shared: the
    widest decode shape tested; at T = 3 the x staging leaves room for a
    2-stage ring only."""
    H, I, E, k = 7168, 2048, 256, 8
    lay = SynthLayer(91, 0, H, I, E, k)
    L = synth.logits(91, 0, 0, T, E, 1.1)
    xb = synth.x_bf16(91, 0, T, H)
    ml, idx, w, y = run_layer(lay, L, xb, T, k)
    idx_o, w_o = oracle.router_topk(L, k)
    assert np.array_equal(idx, idx_o)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y[t], ref, mag, what=f"H={H} top-{k} T={T} t={t}")

"""Exact-precision prefill (moe_ffn_prefill_ex, RFX_PREFILL_EXACT) against the
exact oracle, with no teacher forcing.

The prefill workload dequantises into shared memory for the tensor cores
(BASELINE's prefill configuration: "to bf16 or fp8").  In the exact variant
every weight is the bf16 pair hi + lo (exactly level * scale) and h enters
the down projection as h1 + h2 (16 bits), so y meets the decode path's
bound against the oracle's fp64 result: relative L2 <= 1e-5 and
|y - y_oracle| <= 1e-4 * m per element.  The bf16-operand prefill's own
error against the same exact oracle is measured beside it and reported.
"""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth
from helpers import OracleLayer, check_close
from synth.layers import SynthLayer
from test_gpu_prefill import bf16_bits_to_f64, check_grouping, exact_h

pytestmark = pytest.mark.gpu
DEV = "cuda"
MIX9 = [(2, 2), (2, 3), (2, 4), (3, 2), (3, 3), (3, 4), (4, 2), (4, 3), (4, 4)]


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(DEV)


def run(lay, ml, logits, xb, T, exact):
    idx = torch.empty((T, lay.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, lay.k), dtype=torch.float32, device=DEV)
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(logits), lay.k, idx, w)
    ml.prefill(to_dev(xb, torch.bfloat16), idx, w, y, exact=exact)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    return idx.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()


def exact_check(lay, T, logits, xb, tokens=None, h_rows=True):
    """The exact prefill against the exact oracle; returns the worst relative
    L2 error of y and of the bf16-operand prefill on the same tokens."""
    ml = lay.moe_layer(max_T=T)
    idx, w, y = run(lay, ml, logits, xb, T, True)
    idx_o, w_o = oracle.router_topk(logits, lay.k)
    assert np.array_equal(idx, idx_o)
    v = ml.prefill_view(T)
    counts, ent = check_grouping(idx, w, v, lay.E)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    tokens = range(T) if tokens is None else tokens
    if h_rows:
        # h1 + h2 against the oracle's exact h: 16 bits, relative 2^-18, plus
        # the fp32 accumulation of g and u (1e-6 of their sensitivity)
        h = bf16_bits_to_f64(v["h"]) + bf16_bits_to_f64(v["h_lo"])
        row_of = np.empty(T * lay.k, dtype=np.int64)
        row_of[ent] = np.arange(ent.size)
        for t in list(tokens)[:8]:
            for j in range(lay.k):
                he, sens = exact_h_exact(ol.expert(int(idx[t, j])), xf[t])
                err = np.abs(h[row_of[t * lay.k + j]] - he)
                assert np.all(err <= 2.0 ** -17 * np.abs(he) + 1e-6 * sens + 1e-300), f"h token {t} slot {j}"
    worst = 0.0
    for t in tokens:
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        rel, _ = check_close(y[t], ref, mag, what=f"exact prefill token {t}")
        worst = max(worst, rel)
    # the bf16-operand prefill on the same tokens, against the same exact oracle
    _, _, yb = run(lay, ml, logits, xb, T, False)
    worst_bf16 = 0.0
    for t in tokens:
        ref, _ = ol.token(xf[t], idx_o[t], w_o[t])
        worst_bf16 = max(worst_bf16, np.linalg.norm(yb[t] - ref) / np.linalg.norm(ref))
    print(f"exact prefill T={T}: worst rel-L2 {worst:.2e}; bf16-operand prefill against the exact oracle: "
          f"worst rel-L2 {worst_bf16:.2e}")
    return worst, worst_bf16


def exact_h_exact(mats, x):
    """The oracle's exact h (weights not rounded) and its sensitivity."""
    g, mg = oracle.gemv(mats[0], x)
    u, mu = oracle.gemv(mats[1], x)
    g, mg, u, mu = g[0], mg[0], u[0], mu[0]
    silu = np.vectorize(oracle.silu)(g)
    sig = np.where(g != 0, silu / np.where(g != 0, g, 1.0), 0.5)
    dsilu = sig * (1.0 + g * (1.0 - sig))
    return silu * u, np.abs(dsilu * u) * mg + np.abs(silu) * mu


@pytest.mark.parametrize("T", [9, 100, 700])
def test_exact_prefill_tiny_layer(T):
    lay = SynthLayer(41, 0, 512, 256, 8, 2)
    logits = synth.logits(41, 0, 0, T, 8, 1.1)
    xb = synth.x_bf16(41, 0, T, 512)
    worst, worst_bf16 = exact_check(lay, T, logits, xb)
    assert worst_bf16 > 10 * worst      # the bf16 operands are the error the exact variant removes


@pytest.mark.parametrize("fmts,sfmts", [((3, 3, 2), (2, 2, 3)), ((4, 4, 4), (3, 3, 2))])
def test_exact_prefill_format_mixes(fmts, sfmts):
    T = 40
    lay = SynthLayer(43, 0, 512, 512, 8, 2, fmts=fmts, shared_fmts=sfmts)
    exact_check(lay, T, synth.logits(43, 0, 0, T, 8, 0.0), synth.x_bf16(43, 0, T, 512))


def test_exact_prefill_mix_layer():
    T = 60
    lay = SynthLayer(69, 0, 512, 256, 9, 2, mix=MIX9)
    exact_check(lay, T, synth.logits(69, 0, 0, T, 9, 0.0), synth.x_bf16(69, 0, T, 512))


def test_exact_prefill_full_size_layer():
    T = 512
    lay = SynthLayer(0, 0, 4096, 2048, 256, 6)
    logits = synth.logits(0, 0, 900, T, 256, 1.1)
    xb = synth.x_bf16(0, 900, T, 4096)
    exact_check(lay, T, logits, xb, tokens=range(0, T, 61), h_rows=False)


def test_exact_prefill_workspace_and_precision_arguments():
    lay = SynthLayer(3, 0, 512, 256, 8, 2)
    ml = lay.moe_layer(max_T=16)
    b = rfx.moe_prefill_workspace_bytes_ex(ml.handle, 16, rfx.RFX_PREFILL_BF16)
    e = rfx.moe_prefill_workspace_bytes_ex(ml.handle, 16, rfx.RFX_PREFILL_EXACT)
    assert b == rfx.moe_prefill_workspace_bytes(ml.handle, 16)
    up = lambda n: (n + 255) // 256 * 256
    assert e - b == up(2 * (16 * 2 + 16) * 256 * 2) - up((16 * 2 + 16) * 256 * 2)   # the h2 rows
    assert rfx.moe_prefill_workspace_bytes_ex(ml.handle, 16, 7) == 0
    ws = torch.zeros(e, dtype=torch.uint8, device=DEV)
    x = torch.zeros((16, 512), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((16, 2), dtype=torch.int32, device=DEV)
    w = torch.zeros((16, 2), dtype=torch.float32, device=DEV)
    y = torch.zeros((16, 512), dtype=torch.float32, device=DEV)
    with pytest.raises(rfx.RfxError):
        rfx.moe_ffn_prefill_ex(ml.handle, x, 16, idx, w, y, ws, 7)
    with pytest.raises(rfx.RfxError):   # the bf16 workspace is too small for the exact variant
        rfx.moe_ffn_prefill_ex(ml.handle, x, 16, idx, w, y, ws[:b], rfx.RFX_PREFILL_EXACT)

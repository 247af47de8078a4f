"""The layer stack at full size (m.mzlw.cn, "Lucebox专攻DeepSeek V4…", section
"MoE 专家并行": 43 MoE layers of H=4096, I=2048, 256 experts top-6 + shared).

Three full-size layers, then all 43 resident at once: moe_stack_forward
(one router launch, the unit-RMS bf16 chaining done inside each next
layer's kernel) against the step-by-step calls, bit for bit, and every layer
teacher-forced against the oracle.  The oracle rounds each chained
activation to bf16 from fp64 values and the GPU from fp32 accumulations, so
a value next to a bf16 tie may round the other way at some layer; the
free-running chains are compared and reported (see test_stack_43_layers).
"""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth
from helpers import OracleLayer, check_close
from synth.layers import SynthLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"
H, I, E, K = 4096, 2048, 256, 6


def _bf16_bits_to_f64(t):
    return synth.bf16_to_f64(t.cpu().numpy().view(np.uint16))


def _stack(mls, logits, x0, T):
    ws = torch.empty(rfx.moe_stack_workspace_bytes(mls, T), dtype=torch.uint8, device=DEV)
    rfx.rfx_ws_init(ws)
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.moe_stack_forward(mls, torch.from_numpy(logits).to(DEV), torch.from_numpy(x0).view(torch.bfloat16).to(DEV),
                          y, ws)
    torch.cuda.synchronize()
    assert rfx.rfx_ws_status(ws) == rfx.RFX_OK, rfx.rfx_last_error()
    return y


@pytest.fixture(scope="module")
def three_layers():
    return [SynthLayer(5, l, H, I, E, K) for l in range(3)]


@pytest.mark.parametrize("T", [1, 4])
def test_stack_three_full_size_layers(three_layers, T):
    layers = three_layers
    mls = [lay.moe_layer() for lay in layers]
    logits = np.stack([synth.logits(5, l, 0, T, E, 1.1) for l in range(3)])       # [L][T][E]
    x0 = synth.x_bf16(5, 0, T, H)
    x = torch.from_numpy(x0).view(torch.bfloat16).to(DEV)
    for l, (lay, ml) in enumerate(zip(layers, mls)):
        idx = torch.empty((T, K), dtype=torch.int32, device=DEV)
        w = torch.empty((T, K), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(torch.from_numpy(logits[l]).to(DEV), K, idx, w)
        y = torch.empty((T, H), dtype=torch.float32, device=DEV)
        ml.forward(x, idx, w, y)
        torch.cuda.synchronize()
        assert ml.status() == rfx.RFX_OK
        xf = _bf16_bits_to_f64(x.view(torch.int16))
        idx_o, w_o = oracle.router_topk(logits[l], K)
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        ol = OracleLayer(lay)
        yg = y.cpu().numpy()
        for t in range(T):
            ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
            check_close(yg[t], ref, mag, what=f"layer {l} column {t}")
        if l + 1 < len(layers):
            xn = torch.empty((T, H), dtype=torch.int16, device=DEV)
            rfx.moe_rms_norm_bf16(y, xn)
            x = xn.view(torch.bfloat16)
    y_stack = _stack(mls, logits, x0, T)
    assert torch.equal(y_stack, y)


def test_stack_43_layers():
    """All 43 layers resident at once.  moe_stack_forward equals the
    step-by-step calls bit for bit; every layer, fed the GPU's own bf16 input,
    meets the per-layer bound against the oracle (teacher forcing); and the
    oracle's free-running fp64 chain is compared with the GPU's chain layer by
    layer.  The latter is reported, and bounded only where the two chains
    have the same input: the map of one layer is quadratic in x (h = silu(g)
    u with g, u linear in x), so a bf16 rounding flip of the chained input
    (2^-8 relative on one element) grows from layer to layer, and after tens
    of layers the two free-running chains are unrelated."""
    L, T = 43, 1
    layers = [SynthLayer(0, l, H, I, E, K) for l in range(L)]
    mls = [lay.moe_layer() for lay in layers]
    logits = np.stack([synth.logits(0, l, 0, T, E, 1.1) for l in range(L)])
    x0 = synth.x_bf16(0, 0, T, H)
    y_stack = _stack(mls, logits, x0, T)
    # the GPU chain step by step, each layer teacher-forced against the oracle
    x = torch.from_numpy(x0).view(torch.bfloat16).to(DEV)
    xo = synth.bf16_to_f64(x0)          # the oracle's own chain
    diverged = []
    for l, (lay, ml) in enumerate(zip(layers, mls)):
        idx = torch.empty((T, K), dtype=torch.int32, device=DEV)
        w = torch.empty((T, K), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(torch.from_numpy(logits[l]).to(DEV), K, idx, w)
        y = torch.empty((T, H), dtype=torch.float32, device=DEV)
        ml.forward(x, idx, w, y)
        torch.cuda.synchronize()
        assert ml.status() == rfx.RFX_OK
        idx_o, w_o = oracle.router_topk(logits[l], K)
        ol = OracleLayer(lay)
        xf = _bf16_bits_to_f64(x.view(torch.int16))
        yg = y.cpu().numpy()
        yo = []
        for t in range(T):
            ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
            check_close(yg[t], ref, mag, what=f"layer {l} column {t} (teacher-forced)")
            yo.append(ol.token(xo[t], idx_o[t], w_o[t])[0])
        rel = max(np.linalg.norm(yg[t] - yo[t]) / np.linalg.norm(yo[t]) for t in range(T))
        diverged.append(rel)
        if l == 0:
            assert rel <= 1e-5       # the same input: only fp32 accumulation differs
        if l + 1 < L:
            xn = torch.empty((T, H), dtype=torch.int16, device=DEV)
            rfx.moe_rms_norm_bf16(y, xn)
            x = xn.view(torch.bfloat16)
            xo = np.stack([oracle.rms_bf16(yo[t]) for t in range(T)])
    print("free-running GPU chain vs the oracle's chain, relative L2 per layer:",
          " ".join(f"{r:.1e}" for r in diverged))
    assert torch.equal(y_stack, y)

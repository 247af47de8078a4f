"""Stack chaining on the GPU: the unit-RMS bf16 step against the oracle, and a
stack of layers checked layer by layer, teacher-forced (the oracle takes the
GPU's bf16 input to each layer, since an fp32-vs-fp64 rounding flip of a bf16
input is legitimate), plus moe_stack_forward against the step-by-step path."""
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


def _bf16_bits_to_f64(t):
    return synth.bf16_to_f64(t.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("T,H,scale", [(1, 4096, 1.0), (3, 512, 1e-3), (8, 4096, 37.0), (2, 96, 1e5)])
def test_rms_bf16_matches_oracle(T, H, scale):
    rng = np.random.default_rng(T * 1000 + H)
    y = (rng.standard_normal((T, H)) * scale).astype(np.float32)
    y[0, :7] = 0.0                                   # zeros stay zero
    yd = torch.from_numpy(y).to(DEV)
    xd = torch.empty((T, H), dtype=torch.int16, device=DEV)
    rfx.moe_rms_norm_bf16(yd, xd)
    got = _bf16_bits_to_f64(xd)
    for t in range(T):
        ref = oracle.rms_bf16(y[t].astype(np.float64))
        # the fp64 sums run in a different order: a flip needs a value within
        # ~1e-16 of a bf16 rounding tie, so demand equality almost everywhere
        same = got[t] == ref
        assert same.mean() >= 0.999, f"column {t}: {np.sum(~same)} differences"
        if not same.all():
            ulp = np.abs(ref[~same]) * 2.0 ** -7
            assert np.all(np.abs(got[t][~same] - ref[~same]) <= ulp)


def test_rms_bf16_edge_values():
    # a column whose scaled values round across binades, and a column of equal values
    y = np.stack([np.array([1.0, -1.0, 1.00390625, 3.0, 0.0, 1e-30] * 16, np.float32),
                  np.full(96, -2.5, np.float32)])
    yd = torch.from_numpy(y).to(DEV)
    xd = torch.empty(y.shape, dtype=torch.int16, device=DEV)
    rfx.moe_rms_norm_bf16(yd, xd)
    got = _bf16_bits_to_f64(xd)
    for t in range(2):
        assert np.array_equal(got[t], oracle.rms_bf16(y[t].astype(np.float64)))
    assert np.all(got[1] == -1.0)


def _run_layer(lay, ml, x_dev, logits, k):
    T = x_dev.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(torch.from_numpy(logits).to(DEV), k, idx, w)
    y = torch.empty((T, lay.H), dtype=torch.float32, device=DEV)
    ml.forward(x_dev, idx, w, y)
    return idx, w, y


@pytest.mark.parametrize("T", [1, 3])
def test_stack_teacher_forced_and_stack_entry(T):
    H, I, E, k, L, seed = 512, 256, 8, 2, 4, 41
    layers = [SynthLayer(seed, l, H, I, E, k) for l in range(L)]
    mls = [lay.moe_layer() for lay in layers]
    logits = np.stack([synth.logits(seed, l, 0, T, E, 0.0) for l in range(L)])     # [L][T][E]
    x0 = synth.x_bf16(seed, 0, T, H)
    x = torch.from_numpy(x0).view(torch.bfloat16).to(DEV)
    for l, (lay, ml) in enumerate(zip(layers, mls)):
        idx, w, y = _run_layer(lay, ml, x, logits[l], k)
        torch.cuda.synchronize()
        assert ml.status() == rfx.RFX_OK
        # layer l against the oracle on the GPU's own bf16 input (teacher forcing)
        xf = _bf16_bits_to_f64(x.view(torch.int16))
        idx_o, w_o = oracle.router_topk(logits[l], k)
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        ol = OracleLayer(lay)
        yg = y.cpu().numpy()
        for t in range(T):
            ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
            check_close(yg[t], ref, mag, what=f"layer {l} column {t}")
        if l + 1 < L:
            xn = torch.empty((T, H), dtype=torch.int16, device=DEV)
            rfx.moe_rms_norm_bf16(y, xn)
            got = _bf16_bits_to_f64(xn)
            for t in range(T):
                assert np.mean(got[t] == oracle.rms_bf16(yg[t].astype(np.float64))) >= 0.999
            x = xn.view(torch.bfloat16)
    y_steps = y.clone()
    # the whole stack in one call: the same kernels, so the same bits
    ws = torch.empty(rfx.moe_stack_workspace_bytes(mls, T), dtype=torch.uint8, device=DEV)
    rfx.rfx_ws_init(ws)
    y_stack = torch.full((T, H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.moe_stack_forward(mls, torch.from_numpy(logits).to(DEV), torch.from_numpy(x0).view(torch.bfloat16).to(DEV),
                          y_stack, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_stack, y_steps)


def test_stack_entry_rejects_mismatched_layers():
    a = SynthLayer(3, 0, 512, 256, 8, 2).moe_layer()
    b = SynthLayer(3, 1, 256, 256, 8, 2).moe_layer()
    assert rfx.moe_stack_workspace_bytes([a, b], 1) == 0
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(rfx.RfxError):
        rfx.moe_stack_forward([a, b], torch.zeros((2, 1, 8), device=DEV),
                              torch.zeros((1, 512), dtype=torch.bfloat16, device=DEV),
                              torch.zeros((1, 512), device=DEV), ws)

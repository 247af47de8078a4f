"""The routed step from the logits in one call (moe_ffn_forward_logits).  Its
routing must be moe_router_topk's bit for bit (ties to the lower index
included) and its y that of moe_router_topk followed by moe_ffn_forward (or
the prefill), bit for bit; one case is also checked against the oracle.
"""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth
from helpers import OracleLayer, check_close
from synth.layers import SynthLayer
from test_gpu_mix import MIX9

pytestmark = pytest.mark.gpu
DEV = "cuda"


def two_ways(lay, logits, xb, T):
    """(idx, w, y) of router + forward, and of the call from the logits."""
    ml = lay.moe_layer(max_T=max(T, 8))
    L = torch.from_numpy(np.ascontiguousarray(logits)).to(DEV)
    x = torch.from_numpy(np.ascontiguousarray(xb)).view(torch.bfloat16).to(DEV)
    out = []
    for fused in (False, True):
        idx = torch.full((T, lay.k), -7, dtype=torch.int32, device=DEV)
        w = torch.full((T, lay.k), float("nan"), dtype=torch.float32, device=DEV)
        y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
        if fused:
            ml.forward_logits(x, L, idx, w, y)
        else:
            rfx.moe_router_topk(L, lay.k, idx, w)
            ml.forward(x, idx, w, y) if T <= 8 else ml.prefill(x, idx, w, y)
        torch.cuda.synchronize()
        assert ml.status() == rfx.RFX_OK, rfx.rfx_last_error()
        out.append((idx.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy()))
    return out


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_fused_routing_tiny_layer(T):
    lay = SynthLayer(51, 0, 512, 256, 8, 2)
    logits = synth.logits(51, 0, 0, T, 8, 0.0)
    xb = synth.x_bf16(51, 0, T, 512)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits, xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(y0, y1)
    idx_o, w_o = oracle.router_topk(logits, lay.k)
    assert np.array_equal(i1, idx_o)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(y1[t], ref, mag, what=f"fused routing T={T} t={t}")


@pytest.mark.parametrize("T", [1, 4, 5])   # the widest full-size call that fits shared memory
def test_fused_routing_full_size_layer(T):
    lay = SynthLayer(0, 0, 4096, 2048, 256, 6)
    logits = synth.logits(0, 0, 300, T, 256, 1.1)
    xb = synth.x_bf16(0, 300, T, 4096)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits, xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(y0, y1)


@pytest.mark.parametrize("E,k", [(300, 8), (1000, 8), (33, 3), (256, 1)])
def test_fused_routing_expert_counts(E, k):
    T = 5
    lay = SynthLayer(53, 0, 64, 32, E, k)
    logits = synth.logits(53, 0, 0, T, E, 0.0)
    xb = synth.x_bf16(53, 0, T, 64)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits, xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(y0, y1)


def test_fused_routing_ties_go_to_the_lower_index():
    T, E = 6, 64
    lay = SynthLayer(55, 0, 128, 64, E, 4)
    logits = np.round(synth.logits(55, 0, 0, T, E, 0.0) * 2.0) / 2.0   # few distinct values: many ties
    logits[0, :] = 1.0
    logits[1, 5] = logits[1, 40] = logits[1, 63] = 7.0
    xb = synth.x_bf16(55, 0, T, 128)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits.astype(np.float32), xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(y0, y1)
    assert list(i1[0]) == [0, 1, 2, 3] and list(i1[1][:3]) == [5, 40, 63]


def test_fused_routing_mix_layer():
    T = 4
    lay = SynthLayer(57, 0, 512, 256, 9, 2, mix=MIX9)
    logits = synth.logits(57, 0, 0, T, 9, 0.0)
    xb = synth.x_bf16(57, 0, T, 512)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits, xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1) and np.array_equal(y0, y1)


def test_fused_routing_prefill_path():
    # T > 8: the routing, then the prefill
    T = 40
    lay = SynthLayer(59, 0, 512, 256, 8, 2)
    logits = synth.logits(59, 0, 0, T, 8, 0.0)
    xb = synth.x_bf16(59, 0, T, 512)
    (i0, w0, y0), (i1, w1, y1) = two_ways(lay, logits, xb, T)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1)
    assert np.allclose(y0, y1, rtol=1e-5, atol=1e-6 * np.abs(y0).max())   # fp32 atomics: order may vary


def test_fused_routing_null_pointers_are_rejected():
    lay = SynthLayer(61, 0, 64, 32, 8, 2)
    ml = lay.moe_layer(max_T=2)
    x = torch.zeros((2, 64), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((2, 2), dtype=torch.int32, device=DEV)
    w = torch.zeros((2, 2), dtype=torch.float32, device=DEV)
    y = torch.zeros((2, 64), dtype=torch.float32, device=DEV)
    with pytest.raises(rfx.RfxError):
        rfx._check(rfx._forward_logits(ml.handle, rfx._ptr(x), 2, None, rfx._ptr(idx), rfx._ptr(w), rfx._ptr(y),
                                       rfx._ptr(ml.ws), ml.ws.numel(), None))

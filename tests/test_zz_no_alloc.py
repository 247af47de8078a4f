"""moe_ffn_forward_static: the MoE FFN for callers that cannot allocate device
memory (no-allocation serving loops, plugins that do not own the allocator,
fixed-budget embedded runtimes).  It must give the same result as
moe_ffn_forward with a caller-owned workspace, call after call, although every
call reuses the library's one built-in workspace array.

Collected last on purpose (tests/test_zz_*), and self-contained, so it passes
both alone in a fresh process and after the other GPU tests.
"""
import ctypes

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


def _run_both(lay, seed, tok0, T, k):
    L = synth.logits(seed, 0, tok0, T, lay.E, 1.1 if lay.E == 256 else 0.0)
    xb = synth.x_bf16(seed, tok0, T, lay.H)
    x = torch.from_numpy(xb).view(torch.bfloat16).to(DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(torch.from_numpy(L).to(DEV), k, idx, w)
    ml = lay.moe_layer()
    y_ref = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.forward(x, idx, w, y_ref)                                    # caller-owned workspace
    y_st = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.moe_ffn_forward_static(ml.handle, x, T, idx, w, y_st)      # built-in workspace
    torch.cuda.synchronize()
    assert ml.status() == rfx.RFX_OK
    idx_o, w_o = oracle.router_topk(L, k)
    xf = synth.bf16_to_f64(xb)
    ol = OracleLayer(lay)
    mags = np.stack([ol.token(xf[t], idx_o[t], w_o[t])[1] for t in range(T)])
    return y_st.cpu().numpy(), y_ref.cpu().numpy(), mags


@pytest.mark.parametrize("H,I,E,k,T", [(512, 256, 8, 2, 3), (4096, 2048, 256, 6, 4)])
def test_static_workspace_matches_moe_ffn_forward_twice(H, I, E, k, T):
    lay = SynthLayer(77, 0, H, I, E, k)
    for call, tok0 in enumerate((0, 50)):          # two calls in a row, different inputs
        y_st, y_ref, mags = _run_both(lay, 77, tok0, T, k)
        for t in range(T):
            check_close(y_st[t], y_ref[t], mags[t], what=f"static vs caller workspace, call {call}, column {t}")


def test_static_workspace_rejects_layers_that_do_not_fit():
    d = rfx.moe_layer_desc()
    d.H, d.I, d.E, d.k = 65536, 2048, 256, 6
    d.f_gate, d.f_up, d.f_down = 2, 2, 3
    d.gate = d.up = d.down = 256
    d.stride_gate = d.stride_up = rfx.rfx_packed_bytes(2, 2048, 65536)
    d.stride_down = rfx.rfx_packed_bytes(3, 65536, 2048)
    h = rfx.moe_layer_create(d)
    try:
        lib = ctypes.CDLL(rfx.LIB_PATH)
        rc = lib.moe_ffn_forward_static(ctypes.c_void_p(h), None, 8, None, None, None, None)
        assert rc == rfx.RFX_EUNSUPPORTED
        assert "static" in rfx.rfx_last_error()
    finally:
        rfx.moe_layer_destroy(h)


def test_static_workspace_prefill_path_matches_moe_ffn_prefill_twice():
    """T > 8 takes the prefill path inside the same built-in array."""
    lay = SynthLayer(79, 0, 512, 256, 8, 2)
    T, k = 12, 2
    ml = lay.moe_layer(max_T=T)
    for call, tok0 in enumerate((0, 40)):
        L = synth.logits(79, 0, tok0, T, lay.E, 0.0)
        xb = synth.x_bf16(79, tok0, T, lay.H)
        x = torch.from_numpy(xb).view(torch.bfloat16).to(DEV)
        idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
        w = torch.empty((T, k), dtype=torch.float32, device=DEV)
        rfx.moe_router_topk(torch.from_numpy(L).to(DEV), k, idx, w)
        y_ref = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
        ml.prefill(x, idx, w, y_ref)
        y_st = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
        rfx.moe_ffn_forward_static(ml.handle, x, T, idx, w, y_st)
        torch.cuda.synchronize()
        assert ml.prefill_status() == rfx.RFX_OK
        # the same kernels; only the order of the prefill's fp32 atomic adds may differ
        torch.testing.assert_close(y_st, y_ref, rtol=1e-6, atol=1e-6 * float(y_ref.abs().max()),
                                   msg=f"static prefill path, call {call}")

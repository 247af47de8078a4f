"""The bounded-wait error path on the GPU, driven without a GPU fault.

Every wait of the decode and prefill kernels gives up after a limit, sets
the workspace's timeout flag, drains its own copies and returns.  The test
hook rfx_debug_set_fault plants a wait that cannot end (a barrier that
expects one CTA more than the grid has; an expert whose gate/up rows never
count as done; a down GEMM stage that nothing loads) and shortens the limit
to 1e5-1e6 SM clocks.  Each test then checks that the call returns, that
rfx_ws_status reports RFX_EDEVICE, and that after rfx_ws_init the same
workspace gives the oracle's result again.
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


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(DEV)


@pytest.fixture(autouse=True)
def _clear_fault():
    yield
    rfx.rfx_debug_set_fault(0, 0)


def _inputs(lay, T, seed):
    L = synth.logits(seed, 0, 0, T, lay.E, 0.0)
    xb = synth.x_bf16(seed, 0, T, lay.H)
    idx = torch.empty((T, lay.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, lay.k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(L), lay.k, idx, w)
    return L, xb, idx, w


@pytest.mark.parametrize("fault", [1, 2])
@pytest.mark.parametrize("T", [1, 4])
def test_decode_timeout_sets_flag_and_recovers(fault, T):
    lay = SynthLayer(97, 0, 512, 256, 8, 2)
    ml = lay.moe_layer()
    L, xb, idx, w = _inputs(lay, T, 97)
    x = to_dev(xb, torch.bfloat16)
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.rfx_debug_set_fault(fault, 100000)
    ml.forward(x, idx, w, y)
    assert ml.status() == rfx.RFX_EDEVICE
    rfx.rfx_debug_set_fault(0, 0)
    rfx.rfx_ws_init(ml.ws)
    ml.forward(x, idx, w, y)
    assert ml.status() == rfx.RFX_OK, rfx.rfx_last_error()
    idx_o, w_o = oracle.router_topk(L, lay.k)
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    yh = y.cpu().numpy()
    for t in range(T):
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t])
        check_close(yh[t], ref, mag, what=f"after recovery T={T} t={t}")


def test_prefill_timeout_sets_flag_and_recovers():
    lay = SynthLayer(99, 0, 512, 256, 8, 2)
    T = 20
    ml = lay.moe_layer(max_T=T)
    L, xb, idx, w = _inputs(lay, T, 99)
    x = to_dev(xb, torch.bfloat16)
    y_ref = torch.empty((T, lay.H), dtype=torch.float32, device=DEV)
    ml.prefill(x, idx, w, y_ref)
    assert ml.prefill_status() == rfx.RFX_OK
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    rfx.rfx_debug_set_fault(3, 1000000)
    ml.prefill(x, idx, w, y)
    assert ml.prefill_status() == rfx.RFX_EDEVICE
    rfx.rfx_debug_set_fault(0, 0)
    rfx.rfx_ws_init(ml.pf_ws)
    ml.prefill(x, idx, w, y)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    # the same kernels on the same inputs; only the order of the fp32 atomic adds may differ
    torch.testing.assert_close(y, y_ref, rtol=1e-6, atol=1e-6 * float(y_ref.abs().max()))

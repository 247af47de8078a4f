"""Prefill grouped GEMM (tcgen05, bf16 operands) against the fp64 oracle.

Operand precision of the prefill: every weight is rounded once to bf16 from
its exact value and the SwiGLU output h is rounded to bf16 before the down
projection; the oracle does the same (``bf16_ops`` / ``bf16_weights``).

What is compared:
  * the grouping (tokens per expert, token and weight of every grouped row):
    bit for bit against ``oracle.group_rows``;
  * h: the GPU rounds its fp32 SwiGLU value to bf16, the oracle its fp64
    value; the two agree except where the exact value lies within the fp32
    accumulation error of a rounding boundary.  So: every GPU value is within
    half a bf16 step plus 1e-6 x the sensitivity of h to the accumulated gate
    and up sums (|silu'(g) u| m_g + |silu(g)| m_u, m = sum |w||x|) of the exact
    h, and almost all (>= 99 %) are equal to the oracle's bf16 value;
  * y, teacher-forced: the oracle's down projection and combine of the GPU's
    own bf16 h must match y within relative L2 <= 1e-5 and 1e-4 * m per
    element (m = sum |w| |W~d| |h|);
  * y against the oracle end to end (its own h), within the bound that the
    bf16 rounding flips of h allow.
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


def bf16_bits_to_f64(t):
    return synth.bf16_to_f64(t.cpu().numpy().view(np.uint16))


def run_prefill(lay, ml, logits, xb, T, k):
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(logits), k, idx, w)
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.prefill(to_dev(xb, torch.bfloat16), idx, w, y)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    v = ml.prefill_view(T)
    return idx.cpu().numpy(), w.cpu().numpy(), y.cpu().numpy(), v


def check_grouping(idx, w, v, E):
    counts, tok, wt, ent = oracle.group_rows(idx, w, E)
    R = int(counts.sum())
    assert np.array_equal(v["counts"].cpu().numpy(), counts)
    assert np.array_equal(v["row_token"][:R].cpu().numpy(), tok)
    assert np.array_equal(v["row_weight"][:R].cpu().numpy(), wt.astype(np.float32))
    return counts, ent


def bf16_half_step(v):
    """Half the bf16 spacing at |v|: 2^(e-9) for v = m 2^e (8 significant
    bits), and no less than 2^-134 (bf16 subnormals are spaced 2^-133)."""
    _, e = np.frexp(np.abs(v))
    return np.ldexp(1.0, np.maximum(e - 9, -134))


def exact_h(mats, x):
    """The oracle's unrounded SwiGLU output with bf16 weights, and its sensitivity
    |silu'(g) u| m_g + |silu(g)| m_u to errors in the accumulated sums."""
    g, mg = oracle.gemv(mats[0], x, bf16_weights=True)
    u, mu = oracle.gemv(mats[1], x, bf16_weights=True)
    g, mg, u, mu = g[0], mg[0], u[0], mu[0]
    silu = np.vectorize(oracle.silu)(g)
    sig = np.where(g != 0, silu / np.where(g != 0, g, 1.0), 0.5)
    dsilu = sig * (1.0 + g * (1.0 - sig))
    return silu * u, np.abs(dsilu * u) * mg + np.abs(silu) * mu


class HCheck:
    """Accumulates the h comparison over many rows."""

    def __init__(self):
        self.n = 0
        self.diff = 0

    def add(self, h_gpu, mats, x, what):
        h, sens = exact_h(mats, x)
        h_rne = np.vectorize(oracle.bf16_round)(h)
        err = np.abs(h_gpu - h)
        allow = bf16_half_step(h) * (1 + 1e-9) + 1e-6 * sens + 1e-300
        assert np.all(err <= allow), f"{what}: h off by {float(np.max(err / allow)):.2f} x the allowed error"
        self.n += h.size
        self.diff += int(np.sum(h_gpu != h_rne))

    def done(self):
        assert self.diff <= 0.01 * self.n, f"{self.diff} of {self.n} h values differ from the oracle's rounding"


def teacher_forced_y(ol, lay, idx, w_o, ent, counts, h_gpu, tokens):
    """Oracle down projection + combine of the GPU's bf16 h rows for `tokens`."""
    T, k = idx.shape
    H = lay.H
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[ent] = np.arange(ent.size)
    y = {t: np.zeros(H) for t in tokens}
    mag = {t: np.zeros(H) for t in tokens}
    by_expert = {}
    for t in tokens:
        for j in range(k):
            by_expert.setdefault(int(idx[t, j]), []).append((t, j))
    for e, lst in by_expert.items():
        rows = np.array([row_of[t * k + j] for t, j in lst])
        d, m = oracle.gemv(ol.expert(e)[2], h_gpu[rows], bf16_weights=True)
        for (t, j), dr, mr in zip(lst, d, m):
            y[t] += w_o[t, j] * dr
            mag[t] += abs(w_o[t, j]) * mr
    if lay.has_shared:
        rk = T * k
        rows = np.array([rk + t for t in tokens])
        d, m = oracle.gemv(ol.shared()[2], h_gpu[rows], bf16_weights=True)
        for t, dr, mr in zip(tokens, d, m):
            y[t] += dr
            mag[t] += mr
    return y, mag


def full_check(lay, T, logits, xb, tokens=None, end_to_end_rel=3e-3):
    k, E = lay.k, lay.E
    ml = lay.moe_layer()
    idx, w, y, v = run_prefill(lay, ml, logits, xb, T, k)
    idx_o, w_o = oracle.router_topk(logits, k)
    assert np.array_equal(idx, idx_o)
    counts, ent = check_grouping(idx, w, v, E)
    h_gpu = bf16_bits_to_f64(v["h"])
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    tokens = range(T) if tokens is None else tokens
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[ent] = np.arange(ent.size)
    # h of every row of the checked tokens against the oracle's own h
    hc = HCheck()
    for t in tokens:
        for j in range(k):
            hc.add(h_gpu[row_of[t * k + j]], ol.expert(int(idx[t, j])), xf[t], f"h token {t} slot {j}")
        if lay.has_shared:
            hc.add(h_gpu[T * k + t], ol.shared(), xf[t], f"h token {t} shared")
    hc.done()
    # y from the GPU's own h: the down GEMM and the combine
    ytf, mtf = teacher_forced_y(ol, lay, idx, w_o, ent, counts, h_gpu, list(tokens))
    for t in tokens:
        check_close(y[t], ytf[t], mtf[t], what=f"teacher-forced token {t}")
    # end to end against the oracle's own bf16-operand result
    for t in tokens:
        ref, mag = ol.token(xf[t], idx_o[t], w_o[t], bf16_ops=True)
        rel = np.linalg.norm(y[t] - ref) / np.linalg.norm(ref)
        assert rel <= end_to_end_rel, f"token {t}: end-to-end rel L2 {rel:.2e}"
    return ml, idx, w, y, v


@pytest.mark.parametrize("T", [9, 100, 700])
def test_prefill_tiny_layer(T):
    lay = SynthLayer(41, 0, 512, 256, 8, 2)
    logits = synth.logits(41, 0, 0, T, 8, 1.1)
    xb = synth.x_bf16(41, 0, T, 512)
    full_check(lay, T, logits, xb)


@pytest.mark.parametrize("fmts,sfmts", [((3, 3, 2), (2, 2, 3)), ((4, 4, 4), (3, 3, 2)), ((2, 2, 4), (4, 4, 2))])
def test_prefill_format_mixes(fmts, sfmts):
    T = 40
    lay = SynthLayer(43, 0, 512, 512, 8, 2, fmts=fmts, shared_fmts=sfmts)
    logits = synth.logits(43, 0, 0, T, 8, 0.0)
    xb = synth.x_bf16(43, 0, T, 512)
    full_check(lay, T, logits, xb)


def test_prefill_many_experts_no_shared():
    # E > 256: several grouping CTAs, many tiles, experts left without tokens
    T, E, k = 64, 300, 8
    lay = SynthLayer(47, 0, 256, 256, E, k, has_shared=False)
    logits = synth.logits(47, 0, 0, T, E, 1.1)
    xb = synth.x_bf16(47, 0, T, 256)
    full_check(lay, T, logits, xb, tokens=range(0, T, 5))


@pytest.fixture(scope="module")
def full_layer():
    return SynthLayer(0, 0, 4096, 2048, 256, 6)


def test_prefill_full_size_layer(full_layer):
    # the prefill workload: T = 2048 tokens with Zipf(1.1)-skewed routing;
    # grouping checked whole, h and y on a sample of tokens
    T = 2048
    logits = synth.logits(0, 0, 5000, T, 256, 1.1)
    xb = synth.x_bf16(0, 5000, T, 4096)
    full_check(full_layer, T, logits, xb, tokens=[0, 1, 777, 1500, 2047])


def test_forward_dispatches_large_T_to_prefill():
    lay = SynthLayer(53, 0, 512, 256, 8, 2)
    T = 20
    logits = synth.logits(53, 0, 0, T, 8, 0.0)
    xb = synth.x_bf16(53, 0, T, 512)
    ml = lay.moe_layer(max_T=T)
    idx = torch.empty((T, 2), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 2), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(logits), 2, idx, w)
    y1 = torch.empty((T, 512), dtype=torch.float32, device=DEV)
    y2 = torch.empty((T, 512), dtype=torch.float32, device=DEV)
    x = to_dev(xb, torch.bfloat16)
    ml.forward(x, idx, w, y1)
    ml.prefill(x, idx, w, y2)
    torch.cuda.synchronize()
    # the same kernels; only the order of the fp32 atomic additions may differ
    torch.testing.assert_close(y1, y2, rtol=1e-6, atol=1e-6 * float(y2.abs().max()))


def test_prefill_bad_expert_ids_set_the_device_flag():
    lay = SynthLayer(59, 0, 512, 256, 8, 2)
    ml = lay.moe_layer()
    T = 12
    x = to_dev(synth.x_bf16(59, 0, T, 512), torch.bfloat16)
    idx = torch.tensor([[i % 8, (i + 1) % 8] for i in range(T)], dtype=torch.int32, device=DEV)
    idx[3, 1] = 8
    w = torch.full((T, 2), 0.5, dtype=torch.float32, device=DEV)
    y = torch.empty((T, 512), dtype=torch.float32, device=DEV)
    ml.prefill(x, idx, w, y)
    assert ml.prefill_status() == rfx.RFX_EDEVICE
    assert ml.prefill_status() == rfx.RFX_OK


def test_prefill_rejects_unsupported_shapes():
    lay = SynthLayer(61, 0, 352, 160, 6, 3)
    ml = lay.moe_layer()
    assert rfx.moe_prefill_workspace_bytes(ml.handle, 16) == 0
    with pytest.raises(rfx.RfxError):
        ml.prefill(torch.zeros((16, 352), dtype=torch.bfloat16, device=DEV),
                   torch.zeros((16, 3), dtype=torch.int32, device=DEV),
                   torch.zeros((16, 3), device=DEV), torch.zeros((16, 352), device=DEV))


def _prefill_with_idx(lay, T, idx_np, w_np, xb):
    ml = lay.moe_layer()
    idx = to_dev(idx_np.astype(np.int32))
    w = to_dev(w_np.astype(np.float32))
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.prefill(to_dev(xb, torch.bfloat16), idx, w, y)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    return y.cpu().numpy(), ml.prefill_view(T)


def _check_against_oracle(lay, idx_np, w_np, xb, y, v, tokens):
    """Grouping bit-exact; y teacher-forced on the GPU's h; y end to end."""
    T, k = idx_np.shape
    counts, ent = check_grouping(idx_np, w_np.astype(np.float32), v, lay.E)
    h_gpu = bf16_bits_to_f64(v["h"])
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb)
    w64 = w_np.astype(np.float32).astype(np.float64)
    ytf, mtf = teacher_forced_y(ol, lay, idx_np, w64, ent, counts, h_gpu, list(tokens))
    for t in tokens:
        check_close(y[t], ytf[t], mtf[t], what=f"teacher-forced token {t}")
        ref, _ = ol.token(xf[t], idx_np[t], w64[t], bf16_ops=True)
        assert np.linalg.norm(y[t] - ref) / np.linalg.norm(ref) <= 3e-3


def test_prefill_single_token():
    # T = 1 through the prefill path: every expert tile has one row (N padded to 16)
    lay = SynthLayer(67, 0, 512, 256, 8, 2)
    logits = synth.logits(67, 0, 0, 1, 8, 0.0)
    xb = synth.x_bf16(67, 0, 1, 512)
    full_check(lay, 1, logits, xb)


def test_prefill_every_token_on_the_same_experts():
    # degenerate routing: all T tokens pick experts 5 and 2; the others get no
    # rows; expert 5 and 2 each need ceil(T / 256) token tiles
    lay = SynthLayer(71, 0, 512, 256, 8, 2)
    T = 600
    idx = np.tile(np.array([[5, 2]]), (T, 1))
    w = np.tile(np.array([[0.75, 0.25]]), (T, 1))
    xb = synth.x_bf16(71, 0, T, 512)
    y, v = _prefill_with_idx(lay, T, idx, w, xb)
    assert v["counts"].cpu().numpy().tolist() == [0, 0, T, 0, 0, T, 0, 0]
    _check_against_oracle(lay, idx, w, xb, y, v, tokens=[0, 255, 256, 511, 599])


def test_prefill_repeated_expert_in_a_row_counts_twice():
    # an id repeated within a row makes two rows (two contributions), as the
    # oracle's sum over the k entries does
    lay = SynthLayer(73, 0, 512, 256, 8, 2)
    T = 20
    rng = np.random.default_rng(73)
    idx = rng.integers(0, 8, size=(T, 2))
    idx[3] = [6, 6]
    idx[11] = [0, 0]
    w = rng.random((T, 2)) * 0.5
    xb = synth.x_bf16(73, 0, T, 512)
    y, v = _prefill_with_idx(lay, T, idx, w, xb)
    _check_against_oracle(lay, idx, w, xb, y, v, tokens=[3, 11, 0, 19])


def test_prefill_max_tokens(full_layer):
    """T = 65536, the call's maximum: the whole grouping against the oracle,
    h and y (teacher-forced) on sampled tokens (only their h rows are copied)."""
    lay, T, k = full_layer, 65536, 6
    logits = synth.logits(0, 0, 200000, T, 256, 1.1)
    xb = synth.x_bf16(0, 200000, T, 4096)
    ml = lay.moe_layer()
    idx_d = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w_d = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(to_dev(logits), k, idx_d, w_d)
    y_d = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.prefill(to_dev(xb, torch.bfloat16), idx_d, w_d, y_d)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    idx, w = idx_d.cpu().numpy(), w_d.cpu().numpy()
    idx_o, w_o = oracle.router_topk(logits, k)
    assert np.array_equal(idx, idx_o)
    v = ml.prefill_view(T)
    counts, ent = check_grouping(idx, w, v, lay.E)
    assert int(counts.sum()) == T * k
    tokens = [0, 1, 4097, 32768, 65534, 65535]
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[ent] = np.arange(ent.size)
    rows = [int(row_of[t * k + j]) for t in tokens for j in range(k)] + [T * k + t for t in tokens]
    h_rows = bf16_bits_to_f64(v["h"][torch.tensor(rows, device=DEV)])
    hmap = dict(zip(rows, h_rows))
    ol = OracleLayer(lay)
    xf = synth.bf16_to_f64(xb[tokens])
    y = y_d[torch.tensor(tokens, device=DEV)].cpu().numpy()
    hc = HCheck()
    for i, t in enumerate(tokens):
        yt, mt = np.zeros(lay.H), np.zeros(lay.H)
        for j in range(k):
            mats = ol.expert(int(idx[t, j]))
            hr = hmap[int(row_of[t * k + j])]
            hc.add(hr, mats, xf[i], f"h token {t} slot {j}")
            d, m = oracle.gemv(mats[2], hr[None, :], bf16_weights=True)
            yt += w_o[t, j] * d[0]
            mt += abs(w_o[t, j]) * m[0]
        hs = hmap[T * k + t]
        hc.add(hs, ol.shared(), xf[i], f"h token {t} shared")
        d, m = oracle.gemv(ol.shared()[2], hs[None, :], bf16_weights=True)
        yt += d[0]
        mt += m[0]
        check_close(y[i], yt, mt, what=f"teacher-forced token {t}")
    hc.done()

"""Format edge cases on the GPU against the fp64 oracle.

The block format (taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI MAX+ 上跑到
32 tok/s", section "ROCmFPX：把 284B 权重压进 128 GB": a block holds low-bit
codes and a scale) admits inputs the workload recipe never draws.  This
library's reading accepts any finite binary16 scale for ROCmFP2/FP3 (zero,
negative, subnormal, up to 65504) and any E8M0 exponent for ROCmFP4; codes
run over the whole level range.  Here such blocks go through every kernel:

  * rfx_gemv_q for the three formats (full and partial chunks, q = 1 and 4),
    and unit-vector probes x = v * e_j, whose output is column j of the
    dequantised matrix times v, exactly;
  * moe_ffn_forward at T = 1 and 4 on layers whose experts carry zero,
    negative, subnormal and near-65504 scales, blocks of extreme codes and
    E8M0 exponents 0, 1 and large ones, so that h spans values far below and
    far above the binary16 range, and an expert id repeated within a column;
  * moe_ffn_prefill on the same layer (bf16 operands, teacher-forced y).

Bounds as in the other parity tests: relative L2 <= 1e-5 and |y - y_oracle|
<= 1e-4 * sum |w x| per element (decode, GEMV); probes bit for bit.
"""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth
from helpers import check_close
from test_gpu_prefill import HCheck, bf16_bits_to_f64, check_grouping, teacher_forced_y

pytestmark = pytest.mark.gpu
DEV = "cuda"

# binary16 scale specials: +-0, subnormals, the largest finite values, +-1
F16_SPECIAL = np.array([0x0000, 0x8000, 0x0001, 0x0155, 0x03FF, 0x8200, 0x7BFF, 0xFBFF, 0x3C00, 0xBC00],
                       dtype=np.uint16)
E8M0_SPECIAL = np.array([0, 1, 2, 127, 140, 160, 200], dtype=np.uint8)
# in a whole expert the products reach h = silu(g) u and then the down
# projection: keep the large exponents moderate there (every value in fp32)
E8M0_SPECIAL_FFN = np.array([0, 1, 2, 127, 132], dtype=np.uint8)


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(DEV)


def f16_bits(v):
    return np.asarray(v, dtype=np.float16).view(np.uint16)


def make_codes(rng, fmt, rows, cols, profile):
    c = rng.integers(0, 1 << fmt, size=(rows, cols), dtype=np.uint8)
    if profile in ("extreme", "mixed"):
        nb = cols // 32
        blk = rng.random((rows, nb))
        frac = 1.0 if profile == "extreme" else 0.25
        lo = blk < frac / 2
        hi = (blk >= frac / 2) & (blk < frac)
        lo_m = np.repeat(lo, 32, axis=1)
        hi_m = np.repeat(hi, 32, axis=1)
        c[lo_m] = 0
        c[hi_m] = (1 << fmt) - 1
    return c


def make_scales(rng, fmt, rows, cols, profile):
    nb = cols // 32
    if fmt == 4:
        e = rng.integers(120, 123, size=(rows, nb)).astype(np.uint8)
        if profile in ("mixed", "mixed_ffn"):
            pick = rng.random((rows, nb)) < 0.3
            e[pick] = rng.choice(E8M0_SPECIAL if profile == "mixed" else E8M0_SPECIAL_FFN, size=int(pick.sum()))
        elif profile == "tiny":
            e[:] = rng.integers(0, 3, size=(rows, nb))
        elif profile == "zero":
            e[:] = 0
        return e
    base = 0.02 * np.exp2(rng.uniform(-1, 1, size=(rows, nb)))
    if profile == "zero":
        return np.zeros((rows, nb), dtype=np.uint16)
    if profile == "negative":
        return f16_bits(-base)
    if profile == "subnormal":   # the smallest binary16 subnormals: h far below the binary16 range
        return rng.integers(1, 32, size=(rows, nb)).astype(np.uint16)
    if profile == "huge":
        return f16_bits(rng.choice([65504.0, -65504.0, 32768.0, 20000.0], size=(rows, nb)))
    s = f16_bits(base)
    if profile in ("mixed", "mixed_ffn"):
        pick = rng.random((rows, nb)) < 0.3
        s[pick] = rng.choice(F16_SPECIAL, size=int(pick.sum()))
    return s


def edge_mat(seed, fmt, rows, cols, code_profile="mixed", scale_profile="mixed"):
    rng = np.random.default_rng(seed)
    return oracle.Mat(fmt, make_codes(rng, fmt, rows, cols, code_profile),
                      make_scales(rng, fmt, rows, cols, scale_profile))


# ---------------------------------------------------------------- GEMV ---

@pytest.mark.parametrize("fmt", [2, 3, 4])
@pytest.mark.parametrize("N,K", [(48, 1024), (40, 352)])
@pytest.mark.parametrize("q", [1, 4])
def test_gemv_edge_blocks(fmt, N, K, q):
    m = edge_mat(1000 + 10 * fmt + q, fmt, N, K)
    W = to_dev(rfx.rfx_pack(fmt, m.codes, m.scales))
    xb = synth.x_bf16(81, N, q, K)
    y = torch.full((q, N), float("nan"), dtype=torch.float32, device=DEV)
    rfx.rfx_gemv_q(fmt, W, N, K, to_dev(xb, torch.bfloat16), y)
    torch.cuda.synchronize()
    ref, mag = oracle.gemv(m, synth.bf16_to_f64(xb))
    check_close(y.cpu().numpy(), ref, mag, what=f"gemv edges fmt{fmt} {N}x{K} q{q}")


@pytest.mark.parametrize("fmt", [2, 3, 4])
def test_gemv_unit_vector_probes_return_columns(fmt):
    """x = v e_j: y = v * W[:, j] exactly (one product per row, no rounding),
    for columns in full chunks, the partial chunk and both ends."""
    N, K = 40, 352
    m = edge_mat(2000 + fmt, fmt, N, K)
    Wd = oracle.dequant(m)
    W = to_dev(rfx.rfx_pack(fmt, m.codes, m.scales))
    cols = [0, 31, 32, 255, 256, 300, 351]
    v = [1.0, -0.375, 3.0, 0.0078125, -2.5, 1.5, 1.0]
    q = len(cols)
    x = np.zeros((q, K), dtype=np.float32)
    for i, (j, s) in enumerate(zip(cols, v)):
        x[i, j] = s
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)   # exact: the values are bf16 numbers
    y = torch.full((q, N), float("nan"), dtype=torch.float32, device=DEV)
    rfx.rfx_gemv_q(fmt, W, N, K, to_dev(xb, torch.bfloat16), y)
    torch.cuda.synchronize()
    yh = y.cpu().numpy().astype(np.float64)
    for i, (j, s) in enumerate(zip(cols, v)):
        assert np.array_equal(yh[i], Wd[:, j] * s), f"fmt{fmt} probe column {j}"


# ------------------------------------------------------------- MoE FFN ---

class EdgeLayer:
    """A small MoE layer whose experts carry chosen code / scale profiles,
    packed on the host; also the oracle view (expert, shared, token)."""

    ROUTED = [  # (gate/up scales, down scales, codes) per routed expert
        ("zero", "normal", "uniform"),
        ("negative", "negative", "mixed"),
        ("subnormal", "normal", "uniform"),   # h ~ 1e-12: far below binary16
        ("huge", "normal", "uniform"),        # h ~ 1e10: far above binary16
        ("normal", "normal", "extreme"),
        ("mixed_ffn", "mixed_ffn", "mixed"),
        ("normal", "subnormal", "mixed"),
        ("mixed_ffn", "huge", "extreme"),
    ]

    def __init__(self, seed, H=512, I=256, has_shared=True, fmts=(2, 2, 3), shared_fmts=(4, 4, 4)):
        self.H, self.I, self.E, self.k = H, I, len(self.ROUTED), 2
        self.fmts, self.shared_fmts, self.has_shared = fmts, shared_fmts, has_shared
        shapes = ((I, H), (I, H), (H, I))
        self.routed = []
        for e, (su, sd, cp) in enumerate(self.ROUTED):
            profs = (su, su, sd)
            self.routed.append(tuple(edge_mat(seed + 97 * e + i, f, r, c, cp, pr)
                                     for i, (f, (r, c), pr) in enumerate(zip(fmts, shapes, profs))))
        self.sh = None
        if has_shared:
            self.sh = tuple(edge_mat(seed + 5000 + i, f, r, c, "mixed", "mixed_ffn")
                            for i, (f, (r, c)) in enumerate(zip(shared_fmts, shapes)))
        self.strides = tuple((rfx.rfx_packed_bytes(f, r, c) + 255) // 256 * 256 for f, (r, c) in zip(fmts, shapes))
        self.bufs = []
        for i, (f, s) in enumerate(zip(fmts, self.strides)):
            buf = np.zeros(self.E * s, dtype=np.uint8)
            for e in range(self.E):
                m = self.routed[e][i]
                p = rfx.rfx_pack(f, m.codes, m.scales)
                buf[e * s:e * s + p.size] = p
            self.bufs.append(to_dev(buf))
        self.shared_bufs = [to_dev(rfx.rfx_pack(f, m.codes, m.scales)) for f, m in zip(shared_fmts, self.sh)] \
            if has_shared else None

    def moe_layer(self, max_T=8):
        return rfx.MoeLayer(self.H, self.I, self.E, self.k, self.fmts, *self.bufs, self.strides,
                            shared=self.shared_bufs, shared_fmts=self.shared_fmts, max_T=max_T)

    def expert(self, e):
        return self.routed[int(e)]

    def shared(self):
        return self.sh

    def token(self, x_f64, idx_row, w_row, bf16_ops=False):
        return oracle.moe_token([self.expert(int(e)) for e in idx_row], w_row, self.sh, x_f64, bf16_ops)


# columns routed to chosen experts (an id repeated within a column included)
ROUTES = np.array([[2, 0], [3, 1], [4, 5], [6, 7], [2, 2], [7, 3], [1, 6], [0, 5]], dtype=np.int32)
WEIGHTS = np.array([[0.7, 0.3], [0.55, 0.45], [0.9, 0.1], [0.4, 0.6], [0.8, 0.2], [0.5, 0.5], [0.25, 0.75],
                    [0.6, 0.4]], dtype=np.float32)


def run_decode(lay, ml, xb, idx, w):
    T = xb.shape[0]
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.forward(to_dev(xb, torch.bfloat16), to_dev(idx), to_dev(w), y)
    assert ml.status() == rfx.RFX_OK, rfx.rfx_last_error()
    return y.cpu().numpy()


@pytest.mark.parametrize("has_shared", [True, False])
@pytest.mark.parametrize("T", [1, 4])
def test_moe_decode_edge_experts(has_shared, T):
    lay = EdgeLayer(3000, has_shared=has_shared)
    ml = lay.moe_layer()
    for start in range(0, len(ROUTES), T):
        idx, w = ROUTES[start:start + T], WEIGHTS[start:start + T]
        xb = synth.x_bf16(83, start, T, lay.H)
        y = run_decode(lay, ml, xb, idx, w)
        xf = synth.bf16_to_f64(xb)
        for t in range(T):
            ref, mag = lay.token(xf[t], idx[t], w[t].astype(np.float64))
            check_close(y[t], ref, mag, what=f"edge decode shared={has_shared} T={T} column {start + t} "
                                             f"experts {idx[t].tolist()}")
        if T > 1:   # each column equals its own 1-column pass, bit for bit
            for t in range(T):
                y1 = run_decode(lay, ml, xb[t:t + 1], idx[t:t + 1], w[t:t + 1])
                assert np.array_equal(y1[0], y[t])


def test_moe_decode_extreme_h_values_are_carried():
    """The SwiGLU output of the 'subnormal' expert (about 1e-12) and of the
    'huge' one (about 1e10) lies outside binary16; both reach y at full
    precision (no range error, no flush to zero)."""
    lay = EdgeLayer(3100, has_shared=False)
    xf_b = synth.x_bf16(85, 0, 1, lay.H)
    xf = synth.bf16_to_f64(xf_b)
    for e in (2, 3):
        _, _, h = oracle.expert_ffn(*lay.expert(e), xf[0])
        assert (np.max(np.abs(h)) < 6e-8) if e == 2 else (np.max(np.abs(h)) > 65504), (e, np.max(np.abs(h)))
    ml = lay.moe_layer()
    idx = np.array([[2, 2]], dtype=np.int32)
    w = np.array([[0.5, 0.5]], dtype=np.float32)
    y = run_decode(lay, ml, xf_b, idx, w)
    ref, mag = lay.token(xf[0], idx[0], w[0].astype(np.float64))
    assert np.max(np.abs(ref)) > 0
    check_close(y[0], ref, mag, what="tiny-h column")
    idx = np.array([[3, 3]], dtype=np.int32)
    y = run_decode(lay, ml, xf_b, idx, w)
    ref, mag = lay.token(xf[0], idx[0], w[0].astype(np.float64))
    check_close(y[0], ref, mag, what="huge-h column")


def test_moe_decode_and_prefill_agree_on_a_repeated_id():
    """An id repeated within a token column contributes once per entry in both
    paths (decode T <= 8, prefill T > 8), as the oracle's sum over j does."""
    lay = EdgeLayer(3200)
    ml = lay.moe_layer()
    xb = synth.x_bf16(87, 0, 12, lay.H)
    idx = np.tile(np.array([[5, 5]], dtype=np.int32), (12, 1))
    idx[3] = [1, 4]
    w = np.tile(np.array([[0.7, 0.3]], dtype=np.float32), (12, 1))
    yd = run_decode(lay, ml, xb[:4], idx[:4], w[:4])
    yp = torch.full((12, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.prefill(to_dev(xb, torch.bfloat16), to_dev(idx), to_dev(w), yp)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    yp = yp.cpu().numpy()
    xf = synth.bf16_to_f64(xb)
    for t in range(4):
        ref, mag = lay.token(xf[t], idx[t], w[t].astype(np.float64))
        check_close(yd[t], ref, mag, what=f"decode column {t}")
        refb, _ = lay.token(xf[t], idx[t], w[t].astype(np.float64), bf16_ops=True)
        assert np.linalg.norm(yp[t] - refb) / np.linalg.norm(refb) <= 3e-3


def test_prefill_edge_experts():
    """moe_ffn_prefill on the edge layer: grouping bit for bit, h within its
    rounding bound, y teacher-forced on the GPU's own h."""
    lay = EdgeLayer(3300)
    T, k = 24, 2
    idx = np.concatenate([ROUTES, ROUTES[::-1], ROUTES[[0, 2, 4, 6, 1, 3, 5, 7]]]).astype(np.int32)
    w = np.concatenate([WEIGHTS, WEIGHTS[::-1], WEIGHTS]).astype(np.float32)
    xb = synth.x_bf16(89, 0, T, lay.H)
    ml = lay.moe_layer(max_T=T)
    y = torch.full((T, lay.H), float("nan"), dtype=torch.float32, device=DEV)
    ml.prefill(to_dev(xb, torch.bfloat16), to_dev(idx), to_dev(w), y)
    assert ml.prefill_status() == rfx.RFX_OK, rfx.rfx_last_error()
    y = y.cpu().numpy()
    v = ml.prefill_view(T)
    counts, ent = check_grouping(idx, w, v, lay.E)
    h_gpu = bf16_bits_to_f64(v["h"])
    xf = synth.bf16_to_f64(xb)
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[ent] = np.arange(ent.size)
    hc = HCheck()
    for t in range(T):
        for j in range(k):
            hc.add(h_gpu[row_of[t * k + j]], lay.expert(int(idx[t, j])), xf[t], f"h token {t} slot {j}")
        hc.add(h_gpu[T * k + t], lay.shared(), xf[t], f"h token {t} shared")
    hc.done()
    w64 = w.astype(np.float64)
    ytf, mtf = teacher_forced_y(lay, lay, idx, w64, ent, counts, h_gpu, list(range(T)))
    for t in range(T):
        check_close(y[t], ytf[t], mtf[t], what=f"prefill edge teacher-forced token {t}")

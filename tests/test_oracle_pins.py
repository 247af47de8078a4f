"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (block bytes, bits per weight, model footprint), the fixed level
tables, closed forms, brute force with library routines (numpy matmul, numpy
float16 decoding, torch bfloat16 rounding, scipy softmax/expit, Python's stable
sort) and invariants.  A dropped term, a wrong sign, offset or index, a
transposed operand or swapped gate/up fails at least one of them.
"""
import json
import math
import os
import struct

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from conftest import GOLDEN

GOLD = json.load(open(os.path.join(GOLDEN, "rocmfpx_format.json")))
LEVELS = {int(b): np.array(v, dtype=np.float64) for b, v in GOLD["levels"].items()}


# ---------------------------------------------------------------- helpers ---

def dense_by_table(bits, codes, scales):
    """Dense W from the golden level table and numpy's own binary16 decoding."""
    lv = LEVELS[bits][codes.astype(np.int64)]
    if bits == 4:
        s = np.ldexp(1.0, scales.astype(np.int64) - 127)
    else:
        s = scales.astype(np.uint16).view(np.float16).astype(np.float64)
    return lv * np.repeat(s, 32, axis=1)


def rand_mat(bits, rows, cols, seed, kind=0):
    spec = synth.MatrixSpec(seed, 0, kind, 0, bits, rows, cols)
    return oracle.Mat(bits, spec.codes(), spec.scales())


def silu_ref(z):
    return z * scipy.special.expit(z)


# ------------------------------------------------------- page-printed values

def test_block_bytes_and_bits_match_pages():
    assert GOLD["block_weights"] == 32
    assert oracle.block_bytes(2) == GOLD["bytes_per_block"]["2"]
    for b, bpw in GOLD["bits_per_weight"].items():
        assert oracle.bits_per_weight(int(b)) == pytest.approx(bpw, abs=0.005)
        assert oracle.block_bytes(int(b)) == 32 * int(b) // 8 + GOLD["scale_bytes"][b]


def test_mix_average_near_page_figure():
    # Page figure: 284B parameters in 102.3 GB -> about 2.88 bit per parameter.
    whole = GOLD["model_bytes"] * 8 / GOLD["model_params"]
    assert whole == pytest.approx(GOLD["model_bits_per_param"], abs=0.005)
    # One FFN layer of the benchmark shape with the pages' role assignment:
    # routed gate/up FP2, routed down FP3, shared expert FP4.
    H, I, E = 4096, 2048, 256
    blocks = H * I // 32
    routed = E * blocks * (2 * oracle.block_bytes(2) + oracle.block_bytes(3))
    shared = 3 * blocks * oracle.block_bytes(4)
    assert routed == 256 * 8_912_896
    assert shared == 13_369_344
    ffn_bits = (routed + shared) * 8 / ((E + 1) * 3 * H * I)
    assert ffn_bits == pytest.approx(2.839, abs=0.001)
    assert abs(ffn_bits - whole) < 0.05          # "near 2.88"
    routed_only = (2 * oracle.bits_per_weight(2) + oracle.bits_per_weight(3)) / 3
    assert routed_only == pytest.approx(2.8333, abs=1e-4)


# ------------------------------------------------------------- dequant ---

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_levels_match_fixed_table(bits):
    n = 1 << bits
    for c in range(n):
        assert oracle.level(bits, c) == LEVELS[bits][c]
    codes = np.tile(np.arange(32, dtype=np.uint8) % n, (1, 1))
    scales = np.array([[127]], np.uint8) if bits == 4 else np.array([[0x3C00]], np.uint16)  # 1.0
    W = oracle.dequant(oracle.Mat(bits, codes, scales))
    assert np.array_equal(W[0], LEVELS[bits][np.arange(32) % n])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_matches_table_and_numpy_f16(bits):
    m = rand_mat(bits, 24, 96, seed=11)
    assert np.array_equal(oracle.dequant(m), dense_by_table(bits, m.codes, m.scales))


def test_scale_special_values():
    codes = np.full((1, 32), 3, np.uint8)  # FP2 level +1.5
    for bits_f16, val in [(0x0001, 2.0**-24), (0x3555, float(np.float16(1 / 3))), (0xBC00, -1.0),
                          (0x7BFF, 65504.0), (0x0000, 0.0)]:
        W = oracle.dequant(oracle.Mat(2, codes, np.array([[bits_f16]], np.uint16)))
        assert W[0, 0] == 1.5 * val
    for e, val in [(0, 2.0**-127), (127, 1.0), (130, 8.0), (254, 2.0**127)]:
        W = oracle.dequant(oracle.Mat(4, np.full((1, 32), 15, np.uint8), np.array([[e]], np.uint8)))
        assert W[0, 0] == 7.5 * val
    with pytest.raises(ValueError):   # 0xFF is not a scale
        oracle.dequant(oracle.Mat(4, np.zeros((1, 32), np.uint8), np.array([[0xFF]], np.uint8)))
    with pytest.raises(ValueError):   # binary16 inf is rejected
        oracle.dequant(oracle.Mat(2, np.zeros((1, 32), np.uint8), np.array([[0x7C00]], np.uint16)))


# ---------------------------------------------------------------- GEMV ---

@pytest.mark.parametrize("bits,N,K,q", [(2, 48, 160, 1), (3, 33, 96, 3), (4, 17, 224, 5)])
def test_gemv_matches_numpy_dense(bits, N, K, q):
    m = rand_mat(bits, N, K, seed=5 + bits)
    x = synth.bf16_to_f64(synth.x_bf16(7, 0, q, K))
    y, mag = oracle.gemv(m, x)
    W = dense_by_table(bits, m.codes, m.scales)
    ref = x @ W.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * (np.abs(x) @ np.abs(W).T).max())
    np.testing.assert_allclose(mag, np.abs(x) @ np.abs(W).T, rtol=1e-12)
    assert y.shape == (q, N)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_unit_vector_probe_returns_column(bits):
    m = rand_mat(bits, 20, 64, seed=3)
    W = dense_by_table(bits, m.codes, m.scales)
    for j in (0, 1, 31, 32, 63):
        x = np.zeros((1, 64))
        x[0, j] = 1.0
        y, _ = oracle.gemv(m, x)
        assert np.array_equal(y[0], W[:, j])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gemv_closed_forms(bits):
    K, N = 256, 8
    n = 1 << bits
    for c in (0, n - 1, n // 2):
        codes = np.full((N, K), c, np.uint8)
        if bits == 4:
            scales, s = np.full((N, K // 32), 122, np.uint8), 2.0**-5
        else:
            scales, s = np.full((N, K // 32), 0x2400, np.uint16), 2.0**-6   # binary16 0.015625
        y, _ = oracle.gemv(oracle.Mat(bits, codes, scales), np.ones((1, K)))
        assert np.all(y == K * s * (c - (n - 1) / 2))
    # alternating c and its mirror cancel exactly
    codes = np.tile(np.array([1, n - 2], np.uint8), (N, K // 2))
    scales = np.full((N, K // 32), 127 if bits == 4 else 0x3C00, np.uint8 if bits == 4 else np.uint16)
    y, _ = oracle.gemv(oracle.Mat(bits, codes, scales), np.ones((1, K)))
    assert np.all(y == 0.0)


def test_q_columns_equal_independent_columns():
    m = rand_mat(2, 40, 128, seed=9)
    x = synth.bf16_to_f64(synth.x_bf16(1, 0, 5, 128))
    y, _ = oracle.gemv(m, x)
    for c in range(5):
        yc, _ = oracle.gemv(m, x[c:c + 1])
        assert np.array_equal(y[c], yc[0])


# -------------------------------------------------------------- router ---

def test_router_matches_stable_sort_and_softmax():
    rng = np.random.default_rng(0)
    T, E, k = 64, 256, 6
    L = rng.standard_normal((T, E)).astype(np.float32)
    L[:, 10] = L[:, 200] = L[:, 57] = 5.0            # three-way tie at the top
    L[3, :] = 0.25                                   # a row of all-equal logits
    idx, w = oracle.router_topk(L, k)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k]
        assert list(idx[t]) == order
        np.testing.assert_allclose(w[t], scipy.special.softmax(L[t, order].astype(np.float64)), rtol=1e-13)
        assert math.fsum(w[t]) == pytest.approx(1.0, abs=1e-15)
    assert list(idx[0, :3]) == [10, 57, 200]
    assert list(idx[3]) == list(range(k))


def test_router_k_equals_E_is_full_softmax():
    L = np.random.default_rng(1).standard_normal((3, 8)).astype(np.float32)
    idx, w = oracle.router_topk(L, 8)
    for t in range(3):
        full = scipy.special.softmax(L[t].astype(np.float64))
        np.testing.assert_allclose(w[t], full[idx[t]], rtol=1e-13)
        assert sorted(idx[t]) == list(range(8))


# ------------------------------------------------------- expert / layer ---

def test_silu_matches_scipy():
    for z in (-30.0, -2.5, -1e-3, 0.0, 0.75, 4.0, 40.0):
        assert oracle.silu(z) == pytest.approx(silu_ref(z), rel=1e-15, abs=1e-300)
    assert oracle.silu(0.0) == 0.0


def test_expert_closed_form_distinguishes_gate_up_down():
    H, I = 64, 32
    gate = oracle.Mat(2, np.full((I, H), 3, np.uint8), np.full((I, H // 32), 0x2400, np.uint16))  # +1.5 * 2^-6
    up = oracle.Mat(2, np.full((I, H), 0, np.uint8), np.full((I, H // 32), 0x2800, np.uint16))    # -1.5 * 2^-5
    down = oracle.Mat(3, np.full((H, I), 5, np.uint8), np.full((H, I // 32), 0x2000, np.uint16))  # +1.5 * 2^-7
    d, mag, h = oracle.expert_ffn(gate, up, down, np.ones(H))
    g, u = H * 1.5 * 2**-6, -H * 1.5 * 2**-5
    hv = g / (1 + math.exp(-g)) * u
    assert np.allclose(h, hv, rtol=1e-15)
    np.testing.assert_allclose(d, I * 1.5 * 2**-7 * hv, rtol=1e-14)
    np.testing.assert_allclose(mag, I * 1.5 * 2**-7 * abs(hv), rtol=1e-14)


def _tiny_layer(seed, H=64, I=32, E=4):
    ex = []
    for e in range(E):
        ex.append(tuple(oracle.Mat(b, *(lambda s: (s.codes(), s.scales()))(synth.MatrixSpec(seed, 0, kind, e, b, r, c)))
                        for kind, b, r, c in ((0, 2, I, H), (1, 2, I, H), (2, 3, H, I))))
    sh = tuple(oracle.Mat(4, *(lambda s: (s.codes(), s.scales()))(synth.MatrixSpec(seed, 0, kind, 0, 4, r, c)))
               for kind, r, c in ((3, I, H), (4, I, H), (5, H, I)))
    return ex, sh


def _dense_ffn(mats, x):
    Wg, Wu, Wd = (dense_by_table(m.bits, m.codes, m.scales) for m in mats)
    h = silu_ref(Wg @ x) * (Wu @ x)
    return Wd @ h, np.abs(Wd) @ np.abs(h)


def test_moe_token_matches_dense_numpy():
    ex, sh = _tiny_layer(21)
    x = synth.bf16_to_f64(synth.x_bf16(2, 0, 1, 64))[0]
    sel, w = [2, 0], np.array([0.7, 0.3])
    y, mag = oracle.moe_token([ex[e] for e in sel], w, sh, x)
    ref = sum(wj * _dense_ffn(ex[e], x)[0] for wj, e in zip(w, sel)) + _dense_ffn(sh, x)[0]
    refm = sum(wj * _dense_ffn(ex[e], x)[1] for wj, e in zip(w, sel)) + _dense_ffn(sh, x)[1]
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-13 * refm.max())
    np.testing.assert_allclose(mag, refm, rtol=1e-12)
    assert np.all(mag >= np.abs(y))
    # without the shared expert the result changes by exactly its contribution
    y0, _ = oracle.moe_token([ex[e] for e in sel], w, None, x)
    np.testing.assert_allclose(y - y0, _dense_ffn(sh, x)[0], rtol=0, atol=1e-13 * refm.max())


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(4)
    v = (rng.standard_normal(2000) * np.exp2(rng.integers(-20, 20, 2000))).astype(np.float32).astype(np.float64)
    ref = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_round(t) for t in v])
    assert np.array_equal(got, ref)
    # exact ties go to the even significand
    assert oracle.bf16_round(1.0 + 2.0**-8) == 1.0
    assert oracle.bf16_round(1.0 + 3 * 2.0**-8) == 1.0 + 2.0**-6


def test_prefill_operand_rounding_matches_torch_bf16():
    ex, _ = _tiny_layer(8)
    x = synth.bf16_to_f64(synth.x_bf16(3, 0, 1, 64))[0]
    d, _, h = oracle.expert_ffn(*ex[1], x, bf16_ops=True)
    # weights are products of <= 13 significant bits: exact in fp32, so torch's
    # fp32 -> bf16 conversion rounds them once; h uses the torch-pinned rounder.
    bf = lambda a: torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    Wg, Wu, Wd = (bf(dense_by_table(m.bits, m.codes, m.scales)) for m in ex[1])
    href = np.vectorize(oracle.bf16_round)(silu_ref(Wg @ x) * (Wu @ x))
    assert np.array_equal(h, href)
    np.testing.assert_allclose(d, Wd @ href, rtol=1e-12, atol=1e-14)


def test_gemv_bf16_weights_matches_torch_rounding():
    for bits in (2, 3, 4):
        m = rand_mat(bits, 24, 96, 40 + bits)
        x = synth.bf16_to_f64(synth.x_bf16(11, 0, 3, 96))
        bf = torch.tensor(dense_by_table(bits, m.codes, m.scales), dtype=torch.float32).to(torch.bfloat16)
        W = bf.to(torch.float64).numpy()
        y, mag = oracle.gemv(m, x, bf16_weights=True)
        np.testing.assert_allclose(y, x @ W.T, rtol=1e-13, atol=1e-13 * np.abs(mag).max())
        np.testing.assert_allclose(mag, np.abs(x) @ np.abs(W).T, rtol=1e-13)
        # the rounding is not a no-op for the fp16-scaled formats
        if bits != 4:
            assert not np.array_equal(W, dense_by_table(bits, m.codes, m.scales))


def test_group_rows_brute_force():
    rng = np.random.default_rng(9)
    T, k, E = 37, 3, 11
    idx = rng.integers(0, E, size=(T, k))
    idx[4, 1] = idx[4, 0]            # a repeated id counts twice
    idx[6, 2] = E + 3                # out of range: no row
    w = rng.random((T, k))
    counts, tok, wt, ent = oracle.group_rows(idx, w, E)
    rows = []
    for e in range(E):               # expert by expert, entries in row-major order
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    rows.append((t, w[t, j], t * k + j))
    assert counts.tolist() == [sum(1 for t in range(T) for j in range(k) if idx[t, j] == e) for e in range(E)]
    assert tok.tolist() == [r[0] for r in rows]
    assert np.array_equal(wt, np.array([r[1] for r in rows]))
    assert ent.tolist() == [r[2] for r in rows]
    assert counts.sum() == T * k - 1


def test_rms_bf16_closed_form_and_torch():
    assert np.array_equal(oracle.rms_bf16(np.full(16, -3.0)), -np.ones(16))
    y = np.random.default_rng(2).standard_normal(4096) * 7.0
    ref = np.vectorize(oracle.bf16_round)(y / math.sqrt(math.fsum(y * y) / y.size))
    got = oracle.rms_bf16(y)
    # the mean is summed in a different order here; allow one bf16 ulp where the
    # fp64 sums differ in the last bit, and check the scale closes to unit RMS
    assert np.mean(got == ref) > 0.999
    assert math.sqrt(np.mean(got * got)) == pytest.approx(1.0, abs=4e-3)


def _bf16_bits(vals):
    """bf16 bit patterns (uint16) of values exactly representable in bf16."""
    f = np.asarray(vals, dtype=np.float32)
    u = f.view(np.uint32)
    assert not (u & 0xFFFF).any(), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def _bf16_value(u):
    return struct.unpack("<f", struct.pack("<I", int(u) << 16))[0]


def test_router_logits_unit_vector_probe():
    """Row e of W one-hot at column p(e): logits[t][e] = x[t][p(e)] + b[e]
    exactly (a transposed operand or a wrong index fails)."""
    E, H, T = 12, 64, 3
    perm = np.random.default_rng(3).permutation(H)[:E]
    W = np.zeros((E, H), dtype=np.float32)
    W[np.arange(E), perm] = 1.0
    x = synth.x_bf16(5, 0, T, H)
    b = np.linspace(-2.0, 3.0, E).astype(np.float32)
    lg, mag = oracle.router_logits(_bf16_bits(W), b, x)
    xf = synth.bf16_to_f64(x)
    assert np.array_equal(lg, xf[:, perm] + b.astype(np.float64)[None, :])
    assert np.array_equal(mag, np.abs(xf[:, perm]) + np.abs(b.astype(np.float64))[None, :])


def test_router_logits_closed_form_and_bias_only():
    E, H, T = 5, 96, 2
    W = np.full((E, H), 0.375, dtype=np.float32)            # exact in bf16
    x = _bf16_bits(np.full((T, H), -1.25, dtype=np.float32))
    lg, _ = oracle.router_logits(_bf16_bits(W), None, x)
    assert np.all(lg == H * 0.375 * -1.25)
    b = np.array([0.5, -7.0, 1e-3, 0.0, 42.0], dtype=np.float32)
    lg0, mag0 = oracle.router_logits(np.zeros((E, H), dtype=np.uint16), b, x)
    assert np.array_equal(lg0, np.broadcast_to(b.astype(np.float64), (T, E)))
    assert np.array_equal(mag0, np.broadcast_to(np.abs(b.astype(np.float64)), (T, E)))


def test_router_logits_brute_force():
    """Plain loops over the bf16 values (a second routine) on a tiny case."""
    E, H, T = 4, 32, 2
    W = synth.router_weight_bf16(9, 1, E, H)
    x = synth.x_bf16(9, 3, T, H)
    b = synth.router_bias_f32(9, 1, E, 1.1)
    lg, mag = oracle.router_logits(W, b, x)
    for t in range(T):
        for e in range(E):
            s = 0.0
            m = 0.0
            for h in range(H):
                p = _bf16_value(W[e, h]) * _bf16_value(x[t, h])
                s += p
                m += abs(p)
            s += float(b[e])
            m += abs(float(b[e]))
            assert abs(lg[t, e] - s) <= 1e-14 * m
            assert abs(mag[t, e] - m) <= 1e-14 * m


def test_moe_token_with_a_format_per_expert():
    """ROCmFPX MIX (a format chosen per expert and matrix): each expert's
    matrices decode with their own format; the token equals the dense sum."""
    H, I = 64, 32
    fmts = [(2, 2, 3), (3, 3, 2), (4, 4, 4), (2, 3, 4)]   # (gate, up, down) per expert
    ex = [tuple(oracle.Mat(b, *(lambda s: (s.codes(), s.scales()))(synth.MatrixSpec(33, 0, kind, e, b, r, c)))
                for kind, b, r, c in zip((0, 1, 2), f, (I, I, H), (H, H, I))) for e, f in enumerate(fmts)]
    _, sh = _tiny_layer(33)
    x = synth.bf16_to_f64(synth.x_bf16(3, 0, 1, H))[0]
    sel, w = [3, 1, 2], np.array([0.5, 0.3, 0.2])
    y, mag = oracle.moe_token([ex[e] for e in sel], w, sh, x)
    ref = sum(wj * _dense_ffn(ex[e], x)[0] for wj, e in zip(w, sel)) + _dense_ffn(sh, x)[0]
    refm = sum(wj * _dense_ffn(ex[e], x)[1] for wj, e in zip(w, sel)) + _dense_ffn(sh, x)[1]
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-13 * refm.max())
    np.testing.assert_allclose(mag, refm, rtol=1e-12)

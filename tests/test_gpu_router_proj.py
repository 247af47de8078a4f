"""GPU parity of the router projection (logits = W_router x + bias) and of the
projection + top-k chain, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import block_quantized_moe_rocmfpx_b200 as rfx
import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

# fp32 accumulation depth of one logit, each rounding at most 2^-24 of the
# running magnitude (bounded by mag = sum |W||x| + |b|).  T <= 8 (GEMV): 8-term
# FMA chains per 16-byte chunk, H / (4 * 8 * 32) chunks per lane, a 5-level
# butterfly, a 2-level tree of the quarters and the bias add.  T > 8 (tensor
# core): H / 16 accumulation steps, each counted twice (the tensor core may
# truncate rather than round), and the bias add.
def bound(H, T):
    depth = 8 * max(1, H // 1024) + 5 + 2 + 1 if T <= 8 else 2 * (H // 16) + 1
    return depth * 2.0 ** -24


def run(E, H, T, seed=0, with_bias=True, k=None):
    W = synth.router_weight_bf16(seed, 0, E, H)
    b = synth.router_bias_f32(seed, 0, E, 1.1) if with_bias else None
    x = synth.x_bf16(seed, 11, T, H)
    Wd = torch.from_numpy(W.view(np.int16)).to(DEV)
    xd = torch.from_numpy(x.view(np.int16)).to(DEV)
    bd = torch.from_numpy(b).to(DEV) if b is not None else None
    lg = torch.full((T, E), float("nan"), dtype=torch.float32, device=DEV)
    if k is None:
        rfx.moe_router_logits(Wd, bd, xd, lg)
        torch.cuda.synchronize()
        return W, b, x, lg.cpu().numpy(), None, None
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_project_topk(Wd, bd, xd, k, lg, idx, w)
    torch.cuda.synchronize()
    return W, b, x, lg.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


def check_logits(W, b, x, lg, H, T):
    ref, mag = oracle.router_logits(W, b, x)
    err = np.abs(lg.astype(np.float64) - ref)
    assert np.all(np.isfinite(lg))
    assert np.all(err <= bound(H, T) * mag), float((err / mag).max())
    rel = np.linalg.norm(lg - ref) / np.linalg.norm(ref)
    assert rel <= (1e-6 if T <= 8 else 1e-5), rel


@pytest.mark.parametrize("T", [1, 4, 5, 8, 9, 37, 64, 65, 200])
def test_router_logits_full_size(T):
    E, H = 256, 4096
    W, b, x, lg, _, _ = run(E, H, T, seed=T)
    check_logits(W, b, x, lg, H, T)


@pytest.mark.parametrize("E,H,T,bias", [(8, 512, 1, False), (8, 512, 3, True), (3, 96, 5, True), (1000, 64, 2, True),
                                        (257, 4096, 8, False), (8, 512, 30, True), (3, 96, 70, True),
                                        (1000, 64, 129, False), (257, 4096, 100, True)])
def test_router_logits_shapes(E, H, T, bias):
    W, b, x, lg, _, _ = run(E, H, T, seed=E + H, with_bias=bias)
    check_logits(W, b, x, lg, H, T)


@pytest.mark.parametrize("T,sub", [(8, 1), (300, 9)])
def test_router_logits_columns_independent(T, sub):
    """A column's logits have the same bits whatever the other columns (within
    one path: T <= 8 and T > 8 use different arithmetic)."""
    E, H = 256, 4096
    W, b, x, lg, _, _ = run(E, H, T, seed=2)
    Wd = torch.from_numpy(W.view(np.int16)).to(DEV)
    bd = torch.from_numpy(b).to(DEV)
    for t in (0, 5, T - sub):
        xd = torch.from_numpy(np.ascontiguousarray(x[t:t + sub]).view(np.int16)).to(DEV)
        part = torch.empty((sub, E), dtype=torch.float32, device=DEV)
        rfx.moe_router_logits(Wd, bd, xd, part)
        assert np.array_equal(part.cpu().numpy(), lg[t:t + sub])


@pytest.mark.parametrize("E,H,T,k", [(256, 4096, 1, 6), (256, 4096, 4, 6), (256, 4096, 2048, 6), (8, 512, 3, 2)])
def test_router_project_topk_teacher_forced(E, H, T, k):
    """The chain's idx / w are the oracle router's on the GPU logits (the
    decision is taken in the kernel's precision: fp32 logits)."""
    W, b, x, lg, idx, w = run(E, H, T, seed=7 + T, k=k)
    if T <= 64:
        check_logits(W, b, x, lg, H, T)
    else:   # large T: a seeded sample of columns against the oracle
        rows = np.random.default_rng(T).choice(T, 48, replace=False)
        check_logits(W, b, x[rows], lg[rows], H, T)
    ridx, rw = oracle.router_topk(lg, k)
    assert np.array_equal(idx, ridx)
    assert np.allclose(w, rw, rtol=1e-6, atol=0)


@pytest.mark.parametrize("E,H,T,k", [(256, 4096, 1, 6), (256, 4096, 8, 6), (1000, 512, 5, 16), (24, 256, 3, 4)])
def test_router_project_topk_one_launch_equals_two(E, H, T, k):
    """T <= 8 runs the projection and the top-k in one cooperative launch; its
    logits, idx and w are bitwise those of moe_router_logits followed by
    moe_router_topk."""
    W, b, x, lg, idx, w = run(E, H, T, seed=31 + T, k=k)
    _, _, _, lg2, _, _ = run(E, H, T, seed=31 + T)
    assert np.array_equal(lg, lg2)
    idx2 = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w2 = torch.empty((T, k), dtype=torch.float32, device=DEV)
    rfx.moe_router_topk(torch.from_numpy(lg2).to(DEV), k, idx2, w2)
    assert np.array_equal(idx, idx2.cpu().numpy())
    assert np.array_equal(w, w2.cpu().numpy())


def test_router_logits_empty_is_a_noop():
    Wd = torch.zeros((8, 64), dtype=torch.int16, device=DEV)
    xd = torch.zeros((0, 64), dtype=torch.int16, device=DEV)
    lg = torch.zeros((0, 8), dtype=torch.float32, device=DEV)
    rfx.moe_router_logits(Wd, None, xd, lg)
    torch.cuda.synchronize()

"""Parity of the CUDA CLS-aware losses and router backward (blockffn_cls_losses) with the fp64 oracle.

Inputs follow the decode layer's recipe (router weights N(0, 1/d), bias -beta sigma for a token-level
sparsity near 0.85, chunks of correlated tokens x_t = z_c + 0.3 n_t), so adjacent tokens share most of
their pattern as on the pages.  Tolerances, from the arithmetic: the kernels carry the fp32 operands Wr and
dS as hi + lo bf16 pairs (about 2^-17 relative each) and sum in fp32; dS is a smooth function of s whose
derivative grows with alpha.  Every element must satisfy
  |got - ref| <= 1e-3 |ref| + 1e-4 * scale
where scale is max |dS| for dS, and for the outputs derived from dS the sum of the magnitudes of the
terms of that element with each |dS| raised by that same budget (|x|^T D for dWr, D |Wr|^T for dx,
sum_t D for db, D = |dS| + max |dS|): about ten times the error of the pairs and of fp32 sums over 32768
tokens, with dS's own allowance carried through the products.  The losses must agree to 1e-4
relative.  Runs are bit-identical.
"""
import numpy as np
import pytest

import gen
import oracle

pytestmark = pytest.mark.gpu


def _inputs(C, L, d, E, seed=0, bias=True):
    lay = gen.make_layer(seed, d, E, 8, beta=1.04, var_x=1.09)
    x = gen.make_chunks(seed, lay, C, L, 0.3).reshape(C * L, d)
    return x, lay.Wr, (lay.br if bias else None)


def _run(bffn, x, C, L, Wr, br, alpha, w_al, w_cs):
    import torch
    xg = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    Wg = torch.from_numpy(Wr).cuda()
    bg = None if br is None else torch.from_numpy(br).cuda()
    out = bffn.cls_losses(xg, C, L, Wg, bg, alpha, w_al, w_cs)
    torch.cuda.synchronize()
    return [None if t is None else t.double().cpu().numpy() for t in out]


def _check(name, got, ref, scale):
    err = np.abs(got - ref)
    tol = 1e-3 * np.abs(ref) + 1e-4 * scale
    bad = np.argwhere(err > tol)
    assert bad.size == 0, (f"{name}: {len(bad)} of {ref.size} outside tolerance, first {bad[:3].tolist()}, "
                           f"max err {err.max():.3g}, max ref {np.abs(ref).max():.3g}")


def _compare(x, Wr, got, ref):
    loss_g, dS_g, dWr_g, db_g, dx_g = got
    l_al, l_cs, dS, dWr, db, dx = ref
    xf = np.abs(gen.bf16_bits_to_f32(x).astype(np.float64))
    aW = np.abs(Wr.astype(np.float64))
    assert abs(loss_g[0] - l_al) <= 1e-4 * abs(l_al) + 1e-7, (loss_g[0], l_al)
    assert abs(loss_g[1] - l_cs) <= 1e-4 * abs(l_cs) + 1e-7, (loss_g[1], l_cs)
    D = np.abs(dS) + np.abs(dS).max()
    _check("dS", dS_g, dS, np.abs(dS).max())
    _check("dWr", dWr_g, dWr, xf.T @ D)
    _check("db", db_g, db, D.sum(0))
    _check("dx", dx_g, dx, D @ aW.T)


@pytest.mark.parametrize("C,L,d,E,alpha,bias", [
    (6, 8, 136, 20, 4.0, True),     # fewer tokens than a tile, ragged d and E (E padded to 64)
    (40, 8, 256, 64, 4.0, True),    # 320 tokens: three token tiles, the last ragged
    (9, 3, 64, 200, 8.0, False),    # odd chunk length, four expert groups, no bias
    (17, 1, 72, 64, 4.0, True),     # L = 1: no adjacent pairs
    (2, 128, 128, 64, 2.0, True),   # the longest chunk the kernel takes
    (33, 8, 24, 5, 20.0, True),     # a sharper sigmoid, tiny d and E
])
def test_cls_losses_match_oracle(bffn, C, L, d, E, alpha, bias):
    x, Wr, br = _inputs(C, L, d, E, seed=C + L + d + E, bias=bias)
    w_al, w_cs = 0.7, 1.3
    got = _run(bffn, x, C, L, Wr, br, alpha, w_al, w_cs)
    ref = oracle.cls_losses(x, C, L, Wr, br, alpha, w_al, w_cs)
    _compare(x, Wr, got, ref)


def test_cls_losses_full_training_batch(bffn):
    """The benchmark's batch: 4096 chunks of 8 tokens at d = 2048, E = 64 (x is 128 MiB), against the
    full oracle (about ten seconds of fp64 on one core)."""
    C, L, d, E = 4096, 8, 2048, 64
    x, Wr, br = _inputs(C, L, d, E, seed=5)
    got = _run(bffn, x, C, L, Wr, br, 4.0, 1.0, 1.0)
    ref = oracle.cls_losses(x, C, L, Wr, br, 4.0, 1.0, 1.0)
    _compare(x, Wr, got, ref)


def test_cls_losses_bit_identical_runs_and_optional_outputs(bffn):
    import torch
    C, L, d, E = 64, 8, 512, 64
    x, Wr, br = _inputs(C, L, d, E, seed=3)
    a = _run(bffn, x, C, L, Wr, br, 4.0, 1.0, 1.0)
    b = _run(bffn, x, C, L, Wr, br, 4.0, 1.0, 1.0)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    xg = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    loss, dS, dWr, db, dx = bffn.cls_losses(xg, C, L, torch.from_numpy(Wr).cuda(), torch.from_numpy(br).cuda(), 4.0,
                                            want_dWr=False, want_db=False, want_dx=False)
    torch.cuda.synchronize()
    assert dWr is None and db is None and dx is None
    assert np.array_equal(loss.double().cpu().numpy(), a[0]) and np.array_equal(dS.double().cpu().numpy(), a[1])


def test_cls_losses_weights_scale_the_gradient(bffn):
    """w_al = 0 leaves the chunk term's gradient alone and w_cs = 0 the locality term's; their sum (with
    both weights) equals the full gradient to rounding."""
    C, L, d, E = 24, 8, 128, 64
    x, Wr, br = _inputs(C, L, d, E, seed=8)
    full = _run(bffn, x, C, L, Wr, br, 4.0, 1.0, 1.0)[1]
    al = _run(bffn, x, C, L, Wr, br, 4.0, 1.0, 0.0)[1]
    cs = _run(bffn, x, C, L, Wr, br, 4.0, 0.0, 1.0)[1]
    assert np.allclose(al + cs, full, rtol=1e-5, atol=1e-6 * np.abs(full).max())

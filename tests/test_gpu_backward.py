"""GPU parity of the layer backward (blockffn_layer_backward) with the fp64 oracle (oracle.layer_backward),
on the decode layer's input recipe (router weights N(0, 1/d), a bias for a token-level sparsity near
0.8, correlated chunk tokens) with a random upstream gradient.

Tolerance, from the arithmetic: the kernels carry fp32 operands (dy, r h, du, dS, Wr) as bf16 hi + lo pairs
(about 2^-17 relative) and sum in fp32 over up to E de (or T) terms; each output element must satisfy
|got - ref| <= 1e-3 |ref| + 1e-4 max|ref| over its tensor (ten times the pairs' error on the largest
terms).  Reruns are bit-identical.
"""
import numpy as np
import pytest

import gen
import oracle

pytestmark = pytest.mark.gpu


def _case(seed, T, d, E, de, bias=True, br=None):
    """Tokens drawn against the router they will meet (with or without b), so every pre-activation keeps the
    1e-3 margin from zero and the GPU's and the oracle's ReLU masks agree."""
    lay = gen.make_layer(seed, d, E, de, beta=0.84, var_x=1.09)
    if br is not None:
        lay.br = np.asarray(br, np.float32)
    if not bias:
        lay.br = np.zeros_like(lay.br)
    L = 8 if T % 8 == 0 else 1
    x = gen.make_chunks(seed, lay, T // L, L, 0.3).reshape(T, d)
    dy = np.random.default_rng(seed + 1).standard_normal((T, d)).astype(np.float32)
    return lay, x, dy


def _run(bffn, lay, x, dy, bias=True):
    import torch
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bf = lambda bits: t(bits.view(np.int16)).view(torch.bfloat16)
    out = bffn.layer_backward(bf(x), t(lay.Wr), t(lay.g), bf(lay.W1), bf(lay.W2), t(dy),
                              br=t(lay.br) if bias else None)
    torch.cuda.synchronize()
    return {k: v.double().cpu().numpy() for k, v in out.items()}


def _ref(lay, x, dy, bias=True):
    w = lambda b: gen.bf16_bits_to_f32(b).astype(np.float64)
    return oracle.layer_backward(w(x), lay.Wr, lay.br if bias else None, lay.g, w(lay.W1), w(lay.W2), dy)


def _compare(got, ref):
    for k in ("dx", "dWr", "db", "dg", "dW1", "dW2"):
        err = np.abs(got[k] - ref[k])
        tol = 1e-3 * np.abs(ref[k]) + 1e-4 * np.abs(ref[k]).max()
        bad = err > tol
        assert not bad.any(), f"{k}: {int(bad.sum())} of {bad.size} out of tolerance, max err {err.max():.3g}"


@pytest.mark.parametrize("T,d,E,de,bias", [
    (40, 64, 8, 16, True),      # tiles ragged in every dimension (T, d, E de, E below 64)
    (128, 256, 16, 64, True),   # one token tile
    (200, 136, 24, 40, False),  # no bias; d and de multiples of 8 only
    (256, 512, 16, 128, True),  # several tiles along every dimension
])
def test_layer_backward_matches_oracle(bffn, cuda_device, T, d, E, de, bias):
    lay, x, dy = _case(T + d + E + de, T, d, E, de, bias)
    got = _run(bffn, lay, x, dy, bias)
    _compare(got, _ref(lay, x, dy, bias))


def test_layer_backward_silent_token_and_reruns(bffn, cuda_device):
    """A token with every router output zero passes no router gradient; reruns are bit-identical."""
    base = gen.make_layer(5, 128, 16, 32, beta=0.84, var_x=1.09)
    lay, x, dy = _case(5, 64, 128, 16, 32, br=-np.abs(base.br) - 0.5)  # every b below -0.5
    x = x.copy()
    x[7] = 0  # s = b for this token: no active expert
    a = _run(bffn, lay, x, dy)
    b = _run(bffn, lay, x, dy)
    for k in a:
        assert np.array_equal(a[k], b[k])
    _compare(a, _ref(lay, x, dy))


def test_layer_backward_expert_never_and_always_active(bffn, cuda_device):
    """An expert no token activates (its gradients are exact zeros: no pairs) and one every token activates
    (its pairs span the whole token range)."""
    base = gen.make_layer(9, 128, 16, 32, beta=0.84, var_x=1.09)
    br = base.br.copy()
    br[0], br[1] = -50.0, 50.0
    lay, x, dy = _case(9, 96, 128, 16, 32, br=br)
    got = _run(bffn, lay, x, dy)
    for k in ("dW1", "dW2"):
        assert np.all(got[k][0] == 0.0)
    assert got["db"][0] == 0.0 and got["dg"][0] == 0.0
    _compare(got, _ref(lay, x, dy))


def test_layer_backward_zero_gain(bffn, cuda_device):
    """An expert with gain g = 0: its pairs have r = 0 while a > 0, so they pass no expert gradient but
    their dr still enters dg (the pairs are grouped by s > 0, not by r > 0)."""
    lay, x, dy = _case(13, 64, 128, 16, 32)
    lay.g = lay.g.copy()
    lay.g[3] = 0.0
    s = gen.bf16_bits_to_f32(x).astype(np.float64) @ lay.Wr.astype(np.float64) + lay.br
    assert (s[:, 3] > 0).any()
    got = _run(bffn, lay, x, dy)
    ref = _ref(lay, x, dy)
    assert ref["dg"][3] != 0.0
    for k in ("dW1", "dW2"):
        assert np.all(got[k][3] == 0.0)
    _compare(got, ref)

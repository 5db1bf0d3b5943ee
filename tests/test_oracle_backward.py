"""Pins of the oracle's layer backward (oracle_layer_backward) against facts that do not come from it:
  * PyTorch fp64 autograd of the layer's forward written in torch operations (router, ReLU, RMSNorm,
    Swish experts weighted by r): every gradient, on chunks with a token whose experts are all off;
  * central finite differences of J = sum(dy * y) in entries of x, Wr, br, g, W1 and W2 (fp64, away from
    the ReLU kink);
  * the backward's own forward equal to the pinned layer oracle's on bf16 inputs.
The last test plants each of the backward's built-in mistakes and checks that some pin catches it.
"""
import numpy as np
import pytest
import torch

import gen
import oracle


def _case(seed, T=6, d=12, E=5, de=8, dead_token=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((d, E)) / np.sqrt(d)
    br = 0.1 * rng.standard_normal(E)
    g = rng.uniform(0.5, 2.0, E)
    W1 = rng.standard_normal((E, de, d)) / np.sqrt(d)
    W2 = rng.standard_normal((E, d, de)) / np.sqrt(de)
    dy = rng.standard_normal((T, d))
    if dead_token:  # a token with every pre-activation negative: r = 0, no router gradient
        br = br - 0.2
        x[-1] = 0.0
    # keep every pre-activation away from the ReLU kink (finite differences must not cross it)
    s = x @ Wr + br
    br = br + np.where(np.abs(s).min(axis=0) < 0.05, 0.1, 0.0)
    return x, Wr, br, g, W1, W2, dy


def _torch_grads(x, Wr, br, g, W1, W2, dy):
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in dict(x=x, Wr=Wr, br=br, g=g, W1=W1, W2=W2).items()}
    s = t["x"] @ t["Wr"] + t["br"]
    a = torch.relu(s)
    rho = torch.sqrt((a * a).mean(dim=1, keepdim=True))
    r = torch.where(rho > 0, t["g"] * a / torch.where(rho > 0, rho, torch.ones_like(rho)), torch.zeros_like(a))
    u = torch.einsum("ejk,tk->tej", t["W1"], t["x"])
    h = u * torch.sigmoid(u)
    y = torch.einsum("te,ekj,tej->tk", r, t["W2"], h)
    (y * torch.tensor(dy)).sum().backward()
    return y.detach().numpy(), {k: v.grad.numpy() for k, v in t.items()}


def pin_autograd():
    for seed in (1, 2):
        x, Wr, br, g, W1, W2, dy = _case(seed)
        out = oracle.layer_backward(x, Wr, br, g, W1, W2, dy)
        y_t, gr = _torch_grads(x, Wr, br, g, W1, W2, dy)
        pairs = [("y", y_t), ("dx", gr["x"]), ("dWr", gr["Wr"]), ("db", gr["br"]), ("dg", gr["g"]),
                 ("dW1", gr["W1"]), ("dW2", gr["W2"])]
        for k, ref in pairs:
            if not np.allclose(out[k], ref, rtol=1e-10, atol=1e-12 * max(1.0, np.abs(ref).max())):
                return False
    return True


def pin_finite_differences():
    x, Wr, br, g, W1, W2, dy = _case(3)
    base = dict(x=x, Wr=Wr, br=br, g=g, W1=W1, W2=W2)
    out = oracle.layer_backward(x, Wr, br, g, W1, W2, dy)
    grad = dict(x=out["dx"], Wr=out["dWr"], br=out["db"], g=out["dg"], W1=out["dW1"], W2=out["dW2"])
    rng = np.random.default_rng(7)
    h = 1e-6

    def J(args):
        return float((oracle.layer_backward(args["x"], args["Wr"], args["br"], args["g"], args["W1"], args["W2"],
                                            dy)["y"] * dy).sum())

    for name, arr in base.items():
        for _ in range(4):
            idx = tuple(rng.integers(n) for n in arr.shape)
            plus = {k: v.copy() for k, v in base.items()}
            minus = {k: v.copy() for k, v in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (J(plus) - J(minus)) / (2 * h)
            scale = max(1.0, np.abs(grad[name]).max())
            if abs(fd - grad[name][idx]) > 1e-6 * scale:
                return False
    return True


def pin_forward_equals_layer_oracle():
    lay = gen.make_layer(9, 32, 6, 16, beta=0.6, var_x=1.09)
    xb = gen.make_chunks(9, lay, 1, 5, 0.3)[0]
    widen = lambda b: gen.bf16_bits_to_f32(b).astype(np.float64)
    y_ref, _, _ = oracle.chunk_forward(xb, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=False)
    out = oracle.layer_backward(widen(xb), lay.Wr, lay.br, lay.g, widen(lay.W1), widen(lay.W2), np.zeros((5, 32)))
    return bool(np.allclose(out["y"], y_ref, rtol=1e-12, atol=1e-14))


BACKWARD_PINS = [pin_autograd, pin_finite_differences, pin_forward_equals_layer_oracle]


@pytest.mark.parametrize("pin", BACKWARD_PINS, ids=lambda p: p.__name__)
def test_backward_pin(pin):
    oracle.set_mutation(0)
    assert pin()


@pytest.mark.parametrize("mutation", [14, 15])
def test_planted_backward_mistake_is_caught(mutation):
    """The planted mistakes: Swish' taken as the sigmoid (14), the RMSNorm backward without its
    normaliser term (15)."""
    caught = []
    try:
        oracle.set_mutation(mutation)
        for pin in BACKWARD_PINS:
            try:
                ok = pin()
            except Exception:  # a crash also counts as caught
                ok = False
            if not ok:
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"mutation {mutation} passed every backward pin"


def _pairs_only(x, Wr, br, g, W1, W2, dy, active):
    """The layer's gradients with the expert terms restricted to the (token, expert) pairs in `active`
    (fp64 numpy, written out per pair); the router part as in the chain rule."""
    T, d = x.shape
    E, de, _ = W1.shape
    s = x @ Wr + br
    a = np.maximum(s, 0.0)
    rho = np.sqrt((a * a).mean(axis=1))
    r = np.where(rho[:, None] > 0, g * a / np.where(rho > 0, rho, 1.0)[:, None], 0.0)
    dx = np.zeros((T, d)); dW1 = np.zeros_like(W1); dW2 = np.zeros_like(W2); dr = np.zeros((T, E))
    for t, e in zip(*np.nonzero(active)):
        u = W1[e] @ x[t]
        sg = 1.0 / (1.0 + np.exp(-u))
        h = u * sg
        q = W2[e].T @ dy[t]
        dr[t, e] = h @ q
        du = r[t, e] * q * (sg * (1.0 + u * (1.0 - sg)))
        dW2[e] += np.outer(dy[t], r[t, e] * h)
        dW1[e] += np.outer(du, x[t])
        dx[t] += W1[e].T @ du
    c = (dr * g * a).sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        da = np.where(rho[:, None] > 0, g * dr / rho[:, None] - a * (c / (E * rho ** 3))[:, None], 0.0)
    dS = np.where(s > 0, da, 0.0)
    dg = np.where(rho[:, None] > 0, dr * a / np.where(rho > 0, rho, 1.0)[:, None], 0.0).sum(axis=0)
    return dict(dx=dx + dS @ Wr.T, dWr=x.T @ dS, db=dS.sum(axis=0), dg=dg, dW1=dW1, dW2=dW2)


def test_active_pairs_reading_equals_dense_backward():
    """Evaluating the expert terms only over the pairs with s > 0 gives the dense backward (the other pairs'
    terms are exact zeros through a = 0): pinned against the oracle, including an expert with g = 0, where
    a pair can have r = 0 while a > 0 and its dr still enters dg.  Restricting to r > 0 instead loses dg there."""
    oracle.set_mutation(0)
    x, Wr, br, g, W1, W2, dy = _case(11, T=7, d=10, E=6, de=5)
    g = g.copy()
    g[2] = 0.0
    s = x @ Wr + br
    assert ((s[:, 2] > 0)).any(), "the g = 0 expert must be active somewhere for this pin to bite"
    ref = oracle.layer_backward(x, Wr, br, g, W1, W2, dy)
    got = _pairs_only(x, Wr, br, g, W1, W2, dy, s > 0)
    for k, v in got.items():
        assert np.allclose(v, ref[k], rtol=1e-10, atol=1e-12 * max(1.0, np.abs(ref[k]).max())), k
    a = np.maximum(s, 0.0)
    rho = np.sqrt((a * a).mean(axis=1))
    r = np.where(rho[:, None] > 0, g * a / np.where(rho > 0, rho, 1.0)[:, None], 0.0)
    wrong = _pairs_only(x, Wr, br, g, W1, W2, dy, r > 0)
    assert not np.allclose(wrong["dg"][2], ref["dg"][2])

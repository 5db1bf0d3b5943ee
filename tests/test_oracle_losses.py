"""Pins of the oracle's CLS-aware objectives (lsdiaocha.cn BlockFFN article, section 3) and of their
backward through the router, against facts that do not come from the oracle itself:
  * a hand-worked chunk whose losses and gradient dJ/ds are closed forms (tests/golden);
  * a router with Wr = 0, where every token of a chunk has the same pattern: the activation-locality
    term is then the binary entropy of that pattern and the chunk term 1 - (1 - p)^L;
  * the binary cross-entropy written as entropy + Kullback-Leibler divergence (scipy.stats.entropy);
  * the chunk term brute-forced as the probability, over all 2^L on/off patterns of independent tokens,
    that at least one token is on;
  * a very sharp sigmoid, where the chunk term becomes the chunk-level activation ratio |U| / E;
  * central finite differences of J in Wr and br, and the identity x^T dJ/dx = dJ/dWr Wr^T (both
    derivatives of J along the same change of s = x Wr), which pins dJ/dx once dJ/dWr is pinned.
The last test plants each of the loss oracle's built-in mistakes and checks that some pin catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import entr, expit
from scipy.stats import entropy

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sig(u):
    return 1.0 / (1.0 + math.exp(-u))


def _closed_form(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sig": _sig, "log": math.log, "exp": math.exp}))


def _router_s(x, Wr, br):
    s = gen.bf16_bits_to_f32(x).astype(np.float64) @ Wr.astype(np.float64)
    return s + (0.0 if br is None else br.astype(np.float64))


def _case(seed, C, L, d, E, scale=0.35):
    rng = np.random.default_rng(seed)
    x = gen.f32_to_bf16_bits(rng.standard_normal((C * L, d)).astype(np.float32))
    Wr = (scale * rng.standard_normal((d, E)) / math.sqrt(d)).astype(np.float32)
    br = (0.1 * rng.standard_normal(E)).astype(np.float32)
    return x, Wr, br


# ------------------------------------------------------------------------------------------ pins
def pin_cls_golden():
    with open(os.path.join(GOLDEN, "cls_losses_worked_example.json")) as f:
        spec = json.load(f)
    inp, exp = spec["inputs"], spec["expected"]
    x = gen.f32_to_bf16_bits(np.array(inp["x"], np.float32))
    Wr, br = np.array(inp["Wr"], np.float32), np.array(inp["br"], np.float32)
    l_al, l_cs, dS, dWr, db, dx = oracle.cls_losses(x, inp["C"], inp["L"], Wr, br, inp["alpha"], inp["w_al"],
                                                    inp["w_cs"])
    want_dS = np.vectorize(_closed_form)(np.array(exp["dS"], dtype=object)).astype(float)
    xf = gen.bf16_bits_to_f32(x).astype(np.float64)
    return (abs(l_al - _closed_form(exp["L_AL"])) <= 1e-14 and abs(l_cs - _closed_form(exp["L_CS"])) <= 1e-14
            and np.allclose(dS, want_dS, rtol=0, atol=1e-14)
            and np.allclose(dWr, xf.T @ want_dS, rtol=0, atol=1e-14)
            and np.allclose(db, want_dS.sum(0), rtol=0, atol=1e-14)
            and np.allclose(dx, want_dS @ Wr.astype(np.float64).T, rtol=0, atol=1e-14))


def pin_cls_constant_router():
    """Wr = 0: s_t = b for every token, so each adjacent pair compares a pattern with itself."""
    C, L, d, E, alpha = 3, 5, 8, 7, 2.5
    x, _, _ = _case(2, C, L, d, E)
    Wr = np.zeros((d, E), np.float32)
    br = np.linspace(-1.5, 1.2, E).astype(np.float32)
    l_al, l_cs, *_ = oracle.cls_losses(x, C, L, Wr, br, alpha)
    p = expit(alpha * br.astype(np.float64))
    h = entr(p) + entr(1.0 - p)  # binary entropy in nats
    return (abs(l_al - h.mean()) <= 1e-13 and abs(l_cs - (1.0 - (1.0 - p) ** L).mean()) <= 1e-13)


def pin_cls_bce_is_entropy_plus_kl():
    C, L, d, E, alpha = 4, 6, 16, 5, 3.0
    x, Wr, br = _case(5, C, L, d, E)
    l_al, *_ = oracle.cls_losses(x, C, L, Wr, br, alpha)
    p = expit(alpha * _router_s(x, Wr, br)).reshape(C, L, E)
    terms = []
    for c in range(C):
        for t in range(L - 1):
            for i in range(E):
                q, pt = p[c, t + 1, i], p[c, t, i]
                terms.append(entropy([q, 1 - q]) + entropy([q, 1 - q], [pt, 1 - pt]))
    return abs(l_al - np.mean(terms)) <= 1e-12


def pin_cls_chunk_probability_bruteforce():
    C, L, d, E, alpha = 3, 5, 8, 4, 1.7
    x, Wr, br = _case(7, C, L, d, E, scale=2.0)
    _, l_cs, *_ = oracle.cls_losses(x, C, L, Wr, br, alpha)
    p = expit(alpha * _router_s(x, Wr, br)).reshape(C, L, E)
    total = 0.0
    for c in range(C):
        for i in range(E):
            for a in itertools.product((0, 1), repeat=L):
                if any(a):
                    total += math.prod(p[c, t, i] if a[t] else 1.0 - p[c, t, i] for t in range(L))
    return abs(l_cs - total / (C * E)) <= 1e-13


def pin_cls_sharp_limit_is_chunk_activation_ratio():
    """With |s| >= 1e-3 and alpha = 2e4, sig(alpha s) is within e^-20 of the mask 1[s > 0], so the chunk
    term is the mean over chunks of |U_c| / E, U_c the chunk's union brute-forced from the signs."""
    C, L, d, E = 6, 4, 32, 24
    lay = gen.make_layer(11, d, E, 16, beta=0.6, var_x=1.09)
    x = np.concatenate(gen.make_chunks(11, lay, C, L, 0.3), axis=0)
    _, l_cs, *_ = oracle.cls_losses(x, C, L, lay.Wr, lay.br, 2e4)
    s = _router_s(x, lay.Wr, lay.br).reshape(C, L, E)
    if np.abs(s).min() < 1e-3:
        return False
    ratio = np.mean([(s[c] > 0).any(axis=0).sum() / E for c in range(C)])
    return abs(l_cs - ratio) <= 1e-7


def _fd_case(C, L, d, E, seed, w_al=0.7, w_cs=1.3, alpha=3.0):
    x, Wr, br = _case(seed, C, L, d, E)
    _, _, dS, dWr, db, dx = oracle.cls_losses(x, C, L, Wr, br, alpha, w_al, w_cs)

    def J(Wr_, br_):
        a, b, *_ = oracle.cls_losses(x, C, L, Wr_, br_, alpha, w_al, w_cs)
        return w_al * a + w_cs * b

    return x, Wr, br, dS, dWr, db, dx, J


def pin_cls_finite_differences():
    """Central differences of J in every br_i and in 12 entries of Wr (fp32 inputs perturbed by
    h = 2^-16, exact in fp32 at these magnitudes, with the oracle's fp64 arithmetic: the O(h^2) error is
    about 1e-8 of the gradient's scale here and the rounding error 1e-11), on a case with
    T <= d (x^T has full column rank, so dJ/dWr = x^T dS pins dS) and a case with T >= d (x has full
    column rank, so x^T dx = dWr Wr^T pins dx)."""
    h = 2.0 ** -16
    rng = np.random.default_rng(3)
    for C, L, d, E, seed in ((2, 4, 16, 5, 21), (4, 6, 16, 5, 22)):
        x, Wr, br, dS, dWr, db, dx, J = _fd_case(C, L, d, E, seed)
        scale = max(np.abs(dWr).max(), np.abs(db).max())
        for i in range(E):
            bp, bm = br.copy(), br.copy()
            bp[i] += h
            bm[i] -= h
            if abs((J(Wr, bp) - J(Wr, bm)) / (2 * h) - db[i]) > 1e-7 * scale:
                return False
        for _ in range(12):
            k, i = rng.integers(d), rng.integers(E)
            wp, wm = Wr.copy(), Wr.copy()
            wp[k, i] += h
            wm[k, i] -= h
            if abs((J(wp, br) - J(wm, br)) / (2 * h) - dWr[k, i]) > 1e-7 * scale:
                return False
        xf = gen.bf16_bits_to_f32(x).astype(np.float64)
        if not np.allclose(xf.T @ dS, dWr, rtol=0, atol=1e-12 * max(scale, 1e-30)):
            return False
        lhs, rhs = xf.T @ dx, dWr @ Wr.astype(np.float64).T
        if not np.allclose(lhs, rhs, rtol=0, atol=1e-12 * max(np.abs(rhs).max(), 1e-30)):
            return False
    return True


def pin_cls_single_token_chunks():
    """L = 1: no adjacent pairs (L_AL = 0, no AL gradient) and the chunk term is the mean of p."""
    C, L, d, E, alpha = 5, 1, 8, 3, 2.0
    x, Wr, br = _case(9, C, L, d, E)
    l_al, l_cs, dS, *_ = oracle.cls_losses(x, C, L, Wr, br, alpha, w_al=1.0, w_cs=0.0)
    p = expit(alpha * _router_s(x, Wr, br))
    _, l_cs2, dS2, *_ = oracle.cls_losses(x, C, L, Wr, br, alpha, w_al=0.0, w_cs=1.0)
    return (l_al == 0.0 and np.all(dS == 0.0) and abs(l_cs - p.mean()) <= 1e-14
            and np.allclose(dS2, alpha * p * (1 - p) / (C * E), rtol=1e-13, atol=0))


LOSS_PINS = [pin_cls_golden, pin_cls_constant_router, pin_cls_bce_is_entropy_plus_kl,
             pin_cls_chunk_probability_bruteforce, pin_cls_sharp_limit_is_chunk_activation_ratio,
             pin_cls_finite_differences, pin_cls_single_token_chunks]


@pytest.mark.parametrize("pin", LOSS_PINS, ids=lambda p: p.__name__)
def test_loss_pin(pin):
    oracle.set_mutation(0)
    assert pin()


@pytest.mark.parametrize("mutation", [9, 10, 11])
def test_planted_loss_mistake_is_caught(mutation):
    """The planted mistakes: no gradient through the shifted target (9), the chunk term's product over
    the other tokens taken over all of them (10), the shift taken the other way (11)."""
    caught = []
    try:
        oracle.set_mutation(mutation)
        for pin in LOSS_PINS:
            try:
                ok = pin()
            except Exception:  # a crash also counts as caught
                ok = False
            if not ok:
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"mutation {mutation} passed every loss pin"

"""Pins of the fp64 CPU oracle against facts that do not come from the oracle itself.

Each pin is a function returning True when the oracle agrees with:
  * two hand-worked chunks whose expected values are closed forms (tests/golden/*.json);
  * the RMSNorm invariant rms(r_t / g) = 1 for every token with an active expert;
  * sparse evaluation (only experts in A_t) equal, bit for bit, to dense evaluation (all E experts
    weighted by their router output), as the masking argument of the BlockFFN article's section 4 states;
  * the E=1 special case, which is a plain MLP g * W2 Swish(W1 x), computed here with numpy and
    scipy's logistic function;
  * the union and the sparsity counts brute-forced over every sign pattern of tiny chunks;
  * the scale invariance of RMSNorm and the token independence of the layer.
The last test plants each of the oracle's built-in mistakes and checks that some pin catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sig(u):
    return 1.0 / (1.0 + math.exp(-u))


def _closed_form(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sqrt": math.sqrt, "sig": _sig, "exp": math.exp}))


def _golden_inputs(name):
    with open(os.path.join(GOLDEN, name)) as f:
        spec = json.load(f)
    inp = spec["inputs"]
    x = gen.f32_to_bf16_bits(np.array(inp["x"], np.float32))
    assert np.array_equal(gen.bf16_bits_to_f32(x), np.array(inp["x"], np.float32)), "inputs must be bf16-exact"
    Wr = np.array(inp["Wr"], np.float32)
    br = None if inp["br"] is None else np.array(inp["br"], np.float32)
    g = np.array(inp["g"], np.float32)
    W1 = gen.f32_to_bf16_bits(np.array(inp["W1"], np.float32))
    W2 = gen.f32_to_bf16_bits(np.array(inp["W2"], np.float32))
    return spec, x, Wr, br, g, W1, W2


def _small(seed=3, d=48, E=12, de=16, L=6, gain=None):
    lay = gen.make_layer(seed, d, E, de, beta=0.6, var_x=1.09)
    if gain is not None:
        lay.g = gain.astype(np.float32)
    x = gen.make_chunks(seed, lay, 1, L, 0.3)[0]
    return lay, x


# ------------------------------------------------------------------------------------------ pins
def pin_golden(name):
    spec, x, Wr, br, g, W1, W2 = _golden_inputs(name)
    exp = spec["expected"]
    norm = spec.get("norm", "rms")
    s, r, act = oracle.router(x, Wr, br, g, norm=norm)
    y, r2, act2 = oracle.chunk_forward(x, Wr, br, g, W1, W2, sparse=False, norm=norm)
    idx, tz, cz = oracle.union(act)
    want_s = np.vectorize(_closed_form)(np.array(exp["s"], dtype=object)).astype(float)
    want_r = np.vectorize(_closed_form)(np.array(exp["r"], dtype=object)).astype(float)
    want_y = np.vectorize(_closed_form)(np.array(exp["y"], dtype=object)).astype(float)
    return (np.allclose(s, want_s, rtol=0, atol=1e-15)
            and np.allclose(r, want_r, rtol=0, atol=1e-14)
            and np.allclose(r2, want_r, rtol=0, atol=1e-14)
            and np.allclose(y, want_y, rtol=0, atol=1e-14)
            and list(idx) == exp["active_idx"] and tz == exp["tls_zero"] and cz == exp["cls_zero"])


def pin_golden_e4():
    return pin_golden("worked_example_e4.json")


def pin_golden_bias_gain():
    return pin_golden("worked_example_bias_gain.json")


def pin_golden_e4_sum_norm():
    return pin_golden("worked_example_e4_sum.json")


def pin_sum_norm_invariant():
    """ReMoE router: sum_i r_{t,i} / g_i = 1 for every token with an active expert (r = 0 otherwise), the
    active sets are those of the RMSNorm router, and r is the RMSNorm router's r rescaled per token by
    rms / sum (the two normalisers of the same ReLU outputs)."""
    rng = np.random.default_rng(12)
    gain = rng.uniform(0.5, 2.0, 12)
    lay, x = _small(seed=19, gain=gain)
    s, r, act = oracle.router(x, lay.Wr, lay.br, lay.g, norm="sum")
    _, r_rms, act_rms = oracle.router(x, lay.Wr, lay.br, lay.g, norm="rms")
    ok = np.array_equal(act, act_rms) and bool(act.any()) and not bool(act.all())
    gg = lay.g.astype(np.float64)
    for t in range(x.shape[0]):
        a = np.maximum(s[t], 0.0)
        if act[t].any():
            ok &= abs(np.sum(r[t] / gg) - 1.0) < 1e-14
            ok &= np.allclose(r[t] * a.sum(), r_rms[t] * math.sqrt(np.mean(a ** 2)), rtol=1e-13, atol=1e-15)
        else:
            ok &= bool(np.all(r[t] == 0.0))
    return bool(ok)


def pin_sum_norm_layer_equals_weighted_experts():
    """ReMoE layer: y_t = sum_i r_{t,i} E_i(x_t) with r from the sum-normalised router, every expert
    evaluated on its own (oracle_expert) and weighted here."""
    lay, x = _small(seed=23, L=3)
    y, r, act = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, norm="sum")
    want = np.zeros_like(y)
    for t in range(x.shape[0]):
        for i in range(lay.E):
            want[t] += r[t, i] * oracle.expert(x[t], lay.W1, lay.W2, i)
    return bool(np.allclose(y, want, rtol=1e-12, atol=1e-14))


def pin_rmsnorm_invariant():
    rng = np.random.default_rng(11)
    gain = rng.uniform(0.5, 2.0, 12)
    lay, x = _small(gain=gain)
    _, r, act = oracle.router(x, lay.Wr, lay.br, lay.g)
    ok = True
    for t in range(x.shape[0]):
        if act[t].any():
            ok &= abs(math.sqrt(np.mean((r[t] / lay.g.astype(np.float64)) ** 2)) - 1.0) < 1e-14
        else:
            ok &= bool(np.all(r[t] == 0.0))
        ok &= bool(np.all((r[t] > 0) == act[t]))
    return bool(ok) and bool(act.any()) and not bool(act.all())


def pin_sparse_equals_dense():
    lay, x = _small(seed=5)
    yd, _, _ = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=False)
    ys, _, _ = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=True)
    return bool(np.array_equal(yd, ys))


def pin_single_expert_mlp():
    d, de, L = 40, 24, 3
    lay = gen.make_layer(7, d, 1, de, beta=0.0, var_x=1.0)
    lay.br = np.array([12.0], np.float32)  # every token activates the single expert
    lay.g = np.array([1.75], np.float32)
    x = gen.f32_to_bf16_bits(np.random.default_rng(1).standard_normal((L, d)).astype(np.float32))
    y, r, act = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2)
    xf = gen.bf16_bits_to_f32(x).astype(np.float64)
    W1 = gen.bf16_bits_to_f32(lay.W1[0]).astype(np.float64)  # [de, d]
    W2 = gen.bf16_bits_to_f32(lay.W2[0]).astype(np.float64)  # [d, de]
    u = xf @ W1.T
    want = 1.75 * ((u * expit(u)) @ W2.T)
    return bool(act.all()) and np.allclose(r, 1.75, rtol=0, atol=1e-15) and np.allclose(y, want, rtol=1e-12, atol=1e-13)


def _sign_pattern_chunk(L, E, signs):
    mag = 1.0 + 0.125 * np.arange(L * E).reshape(L, E)
    xf = (mag * np.where(np.array(signs).reshape(L, E), 1.0, -1.0)).astype(np.float32)
    return gen.f32_to_bf16_bits(xf), np.eye(E, dtype=np.float32)


def pin_counts_bruteforce():
    for L, E in ((2, 3), (3, 2), (1, 4)):
        for signs in itertools.product([False, True], repeat=L * E):
            x, Wr = _sign_pattern_chunk(L, E, signs)
            _, _, act = oracle.router(x, Wr, None, np.ones(E, np.float32))
            idx, tz, cz = oracle.union(act)
            pos = np.array(signs).reshape(L, E)
            U = sorted({i for t in range(L) for i in range(E) if pos[t, i]})
            if not (np.array_equal(act, pos) and list(idx) == U and tz == int((~pos).sum())
                    and cz == E - len(U)):
                return False
    # a wider random case, counted with Python sets
    rng = np.random.default_rng(2)
    pos = rng.random((5, 40)) < 0.2
    x, Wr = _sign_pattern_chunk(5, 40, pos.ravel())
    _, _, act = oracle.router(x, Wr, None, np.ones(40, np.float32))
    idx, tz, cz = oracle.union(act)
    U = sorted(set(np.nonzero(pos)[1].tolist()))
    return list(idx) == U and tz == int((~pos).sum()) and cz == 40 - len(U)


def pin_scale_invariance():
    lay, x = _small(seed=9)
    _, r1, a1 = oracle.router(x, lay.Wr, lay.br, lay.g)
    s1, _, _ = oracle.router(x, lay.Wr, lay.br, lay.g)
    s4, r4, a4 = oracle.router(x, lay.Wr * np.float32(4), lay.br * np.float32(4), lay.g)
    _, r3, _ = oracle.router(x, lay.Wr * np.float32(3), lay.br * np.float32(3), lay.g)
    return (np.array_equal(r1, r4) and np.array_equal(a1, a4) and np.array_equal(s4, 4 * s1)
            and np.allclose(r3, r1, rtol=2e-6, atol=1e-12))  # 3*Wr is rounded to fp32 first


def pin_swish():
    u = np.linspace(-30, 30, 241)
    got = np.array([oracle.swish(v) for v in u])
    return bool(np.allclose(got, u * expit(u), rtol=1e-14, atol=1e-300))


def pin_token_permutation():
    lay, x = _small(seed=13, L=5)
    y, r, act = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2)
    perm = np.array([3, 0, 4, 1, 2])
    yp, rp, actp = oracle.chunk_forward(x[perm], lay.Wr, lay.br, lay.g, lay.W1, lay.W2)
    return (np.array_equal(yp, y[perm]) and np.array_equal(rp, r[perm])
            and list(oracle.union(act)[0]) == list(oracle.union(actp)[0]))


def pin_tokens_forward_mt():
    """The threaded call that the parity tests and the CPU baseline use equals the single-threaded
    chunk forward bit for bit (tokens are independent), for thread counts that divide the tokens,
    leave a remainder, equal them and exceed them."""
    lay, x = _small(seed=17, L=8)
    want, _, _ = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=False)
    for threads in (1, 3, 8, 16, x.shape[0] + 5):
        got = oracle.tokens_forward_mt(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, threads, sparse=False)
        if not np.array_equal(got, want):
            return False
    return True


def pin_union_overlap():
    """The overlap of two unions against Python sets on random lists (including duplicates across lists,
    disjoint and identical lists), and |A ∩ A| = |A|."""
    rng = np.random.default_rng(31)
    for E in (1, 7, 40, 1024):
        for _ in range(20):
            a = np.sort(rng.choice(E, rng.integers(0, E + 1), replace=False))
            b = np.sort(rng.choice(E, rng.integers(0, E + 1), replace=False))
            if oracle.union_overlap(a, b, E) != len(set(a.tolist()) & set(b.tolist())):
                return False
            if oracle.union_overlap(a, a, E) != len(a):
                return False
    return oracle.union_overlap([0, 5], [1, 2], 8) == 0 and oracle.union_overlap([3], [3], 4) == 1


ALL_PINS = [pin_golden_e4, pin_golden_bias_gain, pin_rmsnorm_invariant, pin_sparse_equals_dense,
            pin_single_expert_mlp, pin_counts_bruteforce, pin_scale_invariance, pin_swish,
            pin_token_permutation, pin_tokens_forward_mt, pin_golden_e4_sum_norm, pin_sum_norm_invariant,
            pin_sum_norm_layer_equals_weighted_experts, pin_union_overlap]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    oracle.set_mutation(0)
    assert pin()


@pytest.mark.parametrize("mutation", [1, 2, 3, 4, 5, 6, 7, 8])
def test_planted_mistake_is_caught(mutation):
    """Each mistake planted in the oracle (dropped bias, flipped sigmoid sign, RMSNorm mean over the
    active entries only, reversed router index, transposed W2, an expert dropped from the union,
    threaded token ranges that drop tokens, the ReMoE normaliser taken as the mean instead of the sum)
    must make at least one pin fail."""
    caught = []
    try:
        oracle.set_mutation(mutation)
        for pin in ALL_PINS:
            try:
                ok = pin()
            except Exception:  # a crash also counts as caught
                ok = False
            if not ok:
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"mutation {mutation} passed every pin"


def test_threaded_dense_forward_at_the_decode_layer_shape():
    """The parity reference at the 1B-class decode layer's shape (d = 2048, E = 64, de = 256): the
    threaded dense forward equals the single-threaded one bit for bit for thread counts 1, 3, 8, 16 and
    more than the tokens, and the sparse loop over each token's active experts equals the dense sum bit
    for bit (the skipped terms are exactly +0)."""
    w = gen.workload("decode")
    lay = w.layer(0)
    x = w.chunks(lay, 1)[0][:5]
    dense, _, act = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=False)
    sparse, _, _ = oracle.chunk_forward(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, sparse=True)
    assert act.any() and not act.all()
    assert np.array_equal(dense, sparse)
    for threads in (1, 3, 8, 16, x.shape[0] + 5):
        got = oracle.tokens_forward_mt(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, threads, sparse=False)
        assert np.array_equal(got, dense), threads

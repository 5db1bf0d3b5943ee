"""Pins of the oracle's fp8 (e4m3) weight quantiser against facts that do not come from the oracle itself:
  * the value of every e4m3 code against PyTorch's float8_e4m3fn decoding;
  * rounding to the nearest code (ties to the even code, the sign kept) against PyTorch's float32 ->
    float8_e4m3fn conversion on random values, on every midpoint between neighbouring codes, and on the
    subnormal range;
  * the scales: powers of two, the smallest with 448 s >= the row's (column's) largest |w|;
  * the round trip: every dequantised weight is a bf16 value within half a code step of w (2^-4 relative
    in the normal range);
  * the per-layer split of W2's scales: t2 the largest scale of the layer, every ratio s2 <= 1.
The last test plants each of the quantiser's built-in mistakes and checks that some pin catches it.
"""
import numpy as np
import pytest
import torch

import gen
import oracle


def _torch_value(codes):
    return torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_code(values):
    return torch.tensor(np.asarray(values, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_code_values():
    codes = [c for c in range(256) if (c & 0x7F) != 0x7F]  # 0x7F and 0xFF are NaN
    got = np.array([oracle.e4m3_value(c) for c in codes])
    want = _torch_value(codes)
    return np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))


def pin_nearest_code():
    rng = np.random.default_rng(4)
    vals = np.concatenate([
        rng.uniform(-448, 448, 2000), rng.normal(0, 1, 2000), rng.uniform(-2 ** -6, 2 ** -6, 2000),
        [0.0, -0.0, 448.0, -448.0, 2 ** -9, 2 ** -10, 3 * 2 ** -10, -3 * 2 ** -10, 2 ** -11],
    ]).astype(np.float32)
    # every midpoint between neighbouring non-negative codes (ties) and its mirror
    pos = _torch_value(range(127))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    got = np.array([oracle.e4m3_nearest(float(v)) for v in vals], np.uint8)
    return np.array_equal(got, _torch_code(vals))


def _weights(seed, NL=2, E=3, d=40, de=24):
    rng = np.random.default_rng(seed)
    W1 = rng.standard_normal((NL * E, de, d)).astype(np.float32) / np.sqrt(d)
    W2 = rng.standard_normal((NL * E, d, de)).astype(np.float32) / np.sqrt(de)
    W1[0, 1] *= 1e-3          # a small row
    W2[1, :, 2] *= 50.0       # a large column
    W1[2, 3] = 0.0            # an all-zero row: scale 1, codes 0
    return gen.f32_to_bf16_bits(W1), gen.f32_to_bf16_bits(W2), NL


def pin_scales_minimal_powers_of_two():
    W1, W2, NL = _weights(1)
    q1, q2, s1, s2, t2 = oracle.quantize_fp8(W1, W2, NL)
    w1 = np.abs(gen.bf16_bits_to_f32(W1).astype(np.float64))
    w2 = np.abs(gen.bf16_bits_to_f32(W2).astype(np.float64))
    a1 = w1.max(axis=2)                                    # per row of W1
    NE = W1.shape[0]
    lay = np.repeat(np.arange(NL), NE // NL)
    full2 = s2.astype(np.float64) * t2.astype(np.float64)[lay][:, None]
    a2 = w2.max(axis=1)                                    # per column of W2
    ok = True
    for scale, amax in ((s1.astype(np.float64), a1), (full2, a2)):
        m, e = np.frexp(scale)
        ok &= bool(np.all(m == 0.5))                       # powers of two
        nz = amax > 0
        ok &= bool(np.all(448 * scale[nz] >= amax[nz]) and np.all(448 * scale[nz] / 2 < amax[nz]))
        ok &= bool(np.all(scale[~nz] == 1.0))
    # t2 is the largest full scale of its layer and every ratio is at most 1
    for l in range(NL):
        ok &= bool(t2[l] == full2[lay == l].max() and np.all(s2[lay == l] <= 1.0))
    return ok


def pin_round_trip():
    W1, W2, NL = _weights(2)
    q1, q2, s1, s2, t2 = oracle.quantize_fp8(W1, W2, NL)
    D1, D2 = oracle.dequantize_fp8(q1, q2, s1, s2, t2)       # asserts bf16-exactness itself
    NE = W1.shape[0]
    lay = np.repeat(np.arange(NL), NE // NL)
    full2 = (s2.astype(np.float64) * t2.astype(np.float64)[lay][:, None])[:, None, :]
    ok = True
    for W, D, sc in ((W1, D1, s1.astype(np.float64)[:, :, None]), (W2, D2, full2)):
        w = gen.bf16_bits_to_f32(W).astype(np.float64)
        dq = gen.bf16_bits_to_f32(D).astype(np.float64)
        err = np.abs(dq - w)
        # half a code step: 2^-4 |w| for normal codes (|w / s| >= 2^-6), 2^-10 s below
        bound = np.maximum(2.0 ** -4 * np.abs(w), 2.0 ** -10 * sc)
        ok &= bool(np.all(err <= bound))
    return ok


FP8_PINS = [pin_code_values, pin_nearest_code, pin_scales_minimal_powers_of_two, pin_round_trip]


@pytest.mark.parametrize("pin", FP8_PINS, ids=lambda p: p.__name__)
def test_fp8_pin(pin):
    oracle.set_mutation(0)
    assert pin()


@pytest.mark.parametrize("mutation", [12, 13])
def test_planted_fp8_mistake_is_caught(mutation):
    """The planted mistakes: a code rounded one step toward zero (12), a scale twice too large (13)."""
    caught = []
    try:
        oracle.set_mutation(mutation)
        for pin in FP8_PINS:
            try:
                ok = pin()
            except Exception:  # a crash also counts as caught
                ok = False
            if not ok:
                caught.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert caught, f"mutation {mutation} passed every fp8 pin"


def test_single_f16_h_would_eat_the_margin():
    """Why h'' stays an f16 hi + lo pair on the fp8 path: rounding h'' = s2 r Swish(u) once to f16 (everything
    else exact) already puts the decode layer's y errors at a large share of the per-element tolerance
    2e-2 |y| + 1e-3 rms(y).  Four chunks of the decode workload, fp64 elsewhere."""
    import gen
    w = gen.workload("decode")
    lay = w.layer(0)
    q1, q2, s1, s2, t2 = oracle.quantize_fp8(lay.W1, lay.W2, 1)
    D1, D2 = oracle.dequantize_fp8(q1, q2, s1, s2, t2)
    W1 = gen.bf16_bits_to_f32(D1).astype(np.float64)
    W2 = gen.bf16_bits_to_f32(D2).astype(np.float64)
    worst = 0.0
    for c in range(4):
        x = gen.bf16_bits_to_f32(w.chunks(lay, 1, replica=c)[0]).astype(np.float64)
        s = x @ lay.Wr.astype(np.float64) + lay.br
        a = np.maximum(s, 0.0)
        rho = np.sqrt((a * a).mean(axis=1, keepdims=True))
        r = np.where(rho > 0, lay.g * a / np.where(rho > 0, rho, 1.0), 0.0)
        y_ref = np.zeros((x.shape[0], w.d))
        y_f16 = np.zeros_like(y_ref)
        for e in range(w.E):
            if not (r[:, e] > 0).any():
                continue
            u = x @ W1[e].T
            h = r[:, e:e + 1] * u / (1.0 + np.exp(-u))
            s2e = s2[e].astype(np.float64)[None, :]
            codes = W2[e] / (float(t2[0]) * s2e)  # W2 = t2 s2 q2
            y_ref += h @ W2[e].T
            y_f16 += float(t2[0]) * ((s2e * h).astype(np.float16).astype(np.float64) @ codes.T)
        tol = 2e-2 * np.abs(y_ref) + 1e-3 * np.sqrt((y_ref ** 2).mean())
        worst = max(worst, float((np.abs(y_f16 - y_ref) / tol).max()))
    assert 0.3 < worst < 1.0, worst

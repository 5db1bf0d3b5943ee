"""The seeded input generator: determinism, bf16 rounding, the router margin, the sparsity it aims at."""
import numpy as np
import pytest
import torch

import gen
import oracle


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.5e-30], np.float32)])
    ours = gen.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = gen.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_same_seed_same_bytes():
    w = gen.workload("tiny")
    l1, l2 = w.layer(0), w.layer(0)
    for f in ("Wr", "br", "g", "W1", "W2"):
        assert np.array_equal(getattr(l1, f), getattr(l2, f))
    assert np.array_equal(w.chunks(l1, 8), w.chunks(l2, 8))
    l3 = gen.workload("tiny", seed=1).layer(0)
    assert not np.array_equal(l1.W1, l3.W1)
    assert not np.array_equal(l1.W1, w.layer(1).W1)  # replicas differ


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_margin_holds(name):
    w = gen.workload(name)
    lay = w.layer(0)
    x = w.chunks(lay, 4)
    for c in range(x.shape[0]):
        s, _, _ = oracle.router(x[c], lay.Wr, lay.br, lay.g)  # the oracle's own pre-activation
        assert np.abs(s).min() >= gen.MARGIN


def test_iid_chunks_margin():
    w = gen.workload("prefill")
    lay = gen.make_layer(0, 256, 16, 32, w.beta, 1.0)
    x = gen.make_chunks(0, lay, 1, 512, None)[0]
    s, _, _ = oracle.router(x, lay.Wr, lay.br, lay.g)
    assert np.abs(s).min() >= gen.MARGIN


def test_expected_cls_matches_sampling():
    rng = np.random.default_rng(4)
    beta, noise, L, n = gen.beta_for_tls(0.85), 0.4, 8, 200000
    u = rng.standard_normal(n)
    v = rng.standard_normal((n, L))
    inactive = np.all(u[:, None] + noise * v < beta * np.sqrt(1 + noise ** 2), axis=1)
    assert abs(inactive.mean() - gen.expected_cls(noise, L, beta)) < 0.005


def test_decode_noise_hits_cls_target():
    noise = gen.solve_noise_for_cls(0.85, 0.70, 8)
    assert abs(gen.expected_cls(noise, 8, gen.beta_for_tls(0.85)) - 0.70) < 1e-6
    assert 0.35 < noise < 0.45


def test_tiny_workload_sparsity():
    """Realised sparsity of the tiny workload, counted by the oracle: TLS near Phi(0.8) = 0.79 and an
    8-token union near a third of the experts."""
    w = gen.workload("tiny")
    lay = w.layer(0)
    x = w.chunks(lay, w.n_chunks)
    tz = cz = 0
    for c in range(w.n_chunks):
        _, _, act = oracle.router(x[c], lay.Wr, lay.br, lay.g)
        _, a, b = oracle.union(act)
        tz += a
        cz += b
    tls = tz / (w.n_chunks * w.L * w.E)
    cls = cz / (w.n_chunks * w.E)
    assert abs(tls - 0.788) < 0.04
    assert abs(cls - gen.expected_cls(0.3, 8, 0.8)) < 0.06


def test_sequence_chunks_share_more_experts_as_drift_grows():
    # consecutive chunks of a drifting sequence: the mean overlap of consecutive unions (counted with
    # Python sets from the fp64 pre-activations on the bf16 tokens) rises with the drift, and drift 0
    # behaves like independent chunks
    lay = gen.make_layer(3, 256, 32, 16, 1.0, 1.09)
    rates = []
    for drift in (0.0, 0.9, 0.99):
        xs = gen.make_sequence_chunks(5, lay, 24, 8, 0.3, drift)
        assert xs.shape == (24, 8, 256) and xs.dtype == np.uint16
        unions = []
        for x in xs:
            s = gen.bf16_bits_to_f32(x).astype(np.float64) @ lay.Wr.astype(np.float64) + lay.br
            assert np.abs(s).min() >= gen.MARGIN
            unions.append(set(np.nonzero((s > 0).any(axis=0))[0].tolist()))
        rates.append(np.mean([len(unions[k] & unions[k - 1]) / max(1, len(unions[k])) for k in range(1, 24)]))
    assert rates[0] < rates[1] < rates[2]

"""GPU parity of the prefill path (L > 32: token grouping and tcgen05 grouped GEMMs) against the fp64
oracle, through the C ABI.

Bit-exact: per-token active flags, the union list, n_active, the sparsity counts.
Within tolerance: y (|y - y_ref| <= 2e-2 |y_ref| + 1e-3 rms(y_ref)) and r: the prefill router carries Wr
as bf16 hi + lo pairs on the tensor cores, so r gets the fp32 allowance plus the bound that error
propagates to (_parity.pair_router_r_bound).
At the full prefill size (L = 4096, d = 4096, E = 128, de = 256) the flags, union and counts are
compared for every token, y and r on a seeded sample of tokens (the dense fp64 oracle costs about
0.5 GFLOP per token).
"""
import numpy as np
import pytest

import gen

pytestmark = pytest.mark.gpu


def _layer(seed, d, E, de, beta):
    from _parity import DeviceLayer
    return DeviceLayer(gen.make_layer(seed, d, E, de, beta, 1.0))


def _tokens(dl, seed, L):
    return gen.make_chunks(seed, dl.lay, 1, L, None)[0]  # i.i.d. tokens, margin enforced


@pytest.mark.parametrize("shape", [
    dict(L=64, d=256, E=16, de=64, beta=0.8),     # one 128-row tile per expert, N1 = 64
    dict(L=100, d=192, E=40, de=128, beta=0.6),   # ragged L, 40 experts (union words cross 32), N2 = 64
    dict(L=600, d=512, E=24, de=256, beta=0.0),   # TLS 50 %: several 128-row tiles per expert, N1 = 256
    dict(L=257, d=384, E=8, de=192, beta=-0.5),   # most experts on for most tokens, N2 = 128
])
def test_prefill_shapes(bffn, cuda_device, shape):
    from _parity import assert_parity, pair_router_r_bound, reference, run_chunk
    dl = _layer(11, shape["d"], shape["E"], shape["de"], shape["beta"])
    x = _tokens(dl, 12, shape["L"])
    got = run_chunk(bffn, dl, x)
    ref = reference(dl, x)
    assert_parity(got, ref, shape["L"], shape["E"], r_bound=pair_router_r_bound(dl, x))


def test_prefill_twice_same_union_and_close_y(bffn, cuda_device):
    # the down-projection adds pair rows into y in hardware order: y may differ in the last bits
    # between runs, the masks and the union may not
    from _parity import run_chunk, y_violations
    dl = _layer(3, 256, 32, 64, 0.5)
    x = _tokens(dl, 4, 200)
    a = run_chunk(bffn, dl, x)
    b = run_chunk(bffn, dl, x)
    assert np.array_equal(a["active"], b["active"]) and np.array_equal(a["active_idx"], b["active_idx"])
    assert not y_violations(b["y"], a["y"]).any()


def test_prefill_full_size_sampled(bffn, cuda_device):
    import oracle
    from _parity import DeviceLayer, R_ATOL, R_RTOL, pair_router_r_bound, run_chunk

    w = gen.workload("prefill")
    dl = DeviceLayer(w.layer(0))
    x = w.chunks(dl.lay, 1)[0]
    L, E = w.L, w.E
    got = run_chunk(bffn, dl, x)
    lay = dl.lay
    # router, flags, union and counts for every token
    _, r_ref, act_ref = oracle.router(x, lay.Wr, lay.br, lay.g)
    idx_ref, tz, cz = oracle.union(act_ref)
    assert np.array_equal(got["active"], act_ref)
    assert np.array_equal(got["active_idx"], idx_ref) and got["n_active"] == len(idx_ref)
    assert got["counts"] == (tz, cz)
    err = np.abs(got["r"] - r_ref)
    assert np.all(err <= R_ATOL + R_RTOL * np.abs(r_ref) + pair_router_r_bound(dl, x)), err.max()
    # y on a seeded sample of tokens (first, last, and 22 in between), against the dense oracle; the
    # tolerance's rms is that of the call's whole y_ref, taken from the sparse oracle over every token
    # (pinned equal to the dense one bit for bit)
    cores = oracle.available_cores()
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([[0, L - 1], rng.choice(L, 22, replace=False)]))
    y_ref = oracle.tokens_forward_mt(x[toks], lay.Wr, lay.br, lay.g, lay.W1, lay.W2, cores, sparse=False)
    y_all = oracle.tokens_forward_mt(x, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, cores, sparse=True)
    assert np.array_equal(y_all[toks], y_ref)
    rms_all = float(np.sqrt(np.mean(y_all ** 2)))
    bad = np.abs(got["y"][toks] - y_ref) > 2e-2 * np.abs(y_ref) + 1e-3 * rms_all
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} sampled y elements out of tolerance"


def test_prefill_remoe_router_variant(bffn, cuda_device):
    # the sum-normalised (ReMoE) router on the prefill path
    from _parity import assert_parity, pair_router_r_bound, reference, run_chunk
    dl = _layer(17, 256, 24, 128, 0.6)
    x = _tokens(dl, 18, 100)
    got = run_chunk(bffn, dl, x, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM)
    assert_parity(got, reference(dl, x, norm="sum"), 100, 24, r_bound=pair_router_r_bound(dl, x, norm="sum"))

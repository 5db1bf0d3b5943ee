"""GPU parity of the batched decode path (blockffn_chunk_forward_batch: many independent chunks of up
to 8 tokens, stacked layers) against the fp64 oracle, through the C ABI.

Bit-exact per chunk: the per-token active flags, the union list, n_active, the sparsity counts.
Within tolerance per chunk: y (|y - y_ref| <= 2e-2 |y_ref| + 1e-3 rms(y_ref), rms over the chunk's y_ref).
"""
import numpy as np
import pytest

import gen

pytestmark = pytest.mark.gpu


class StackedLayers:
    """Layers of one shape stored one after another, as the batched call takes them."""

    def __init__(self, layers, device="cuda"):
        import torch
        self.layers = layers
        self.d, self.E, self.de = layers[0].d, layers[0].E, layers[0].de
        st = lambda f: np.stack([f(l) for l in layers])
        self.Wr = torch.from_numpy(st(lambda l: l.Wr)).to(device)
        self.br = torch.from_numpy(st(lambda l: l.br)).to(device)
        self.g = torch.from_numpy(st(lambda l: l.g)).to(device)
        self.W1 = torch.from_numpy(st(lambda l: l.W1).view(np.int16)).to(device).view(torch.bfloat16)
        self.W2 = torch.from_numpy(st(lambda l: l.W2).view(np.int16)).to(device).view(torch.bfloat16)


def run_batch(bffn, sl, xs, layer=None, teams=0, workspace=None, bias=True, flags=0):
    import torch
    C, L, d = xs.shape
    E = sl.E
    x = torch.from_numpy(np.ascontiguousarray(xs).view(np.int16)).cuda().view(torch.bfloat16)
    y = torch.full((C, L, d), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((C, E), -7, dtype=torch.int32, device="cuda")
    n = torch.full((C,), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((C, 2), -7, dtype=torch.int32, device="cuda")
    mask = torch.zeros((C, L, (E + 31) // 32), dtype=torch.int32, device="cuda")
    lt = None if layer is None else torch.from_numpy(np.asarray(layer, np.int32)).cuda()
    bffn.chunk_forward_batch(x, sl.Wr, sl.g, sl.W1, sl.W2, y, idx, n, layer=lt, br=sl.br if bias else None,
                             counts=counts, tok_mask=mask, teams=teams, workspace=workspace, flags=flags)
    torch.cuda.synchronize()
    status = bffn.device_status(workspace)
    words = mask.cpu().numpy().view(np.uint32)
    bits = ((words[..., None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(C, L, -1)[:, :, :E]
    return {"y": y.cpu().numpy().astype(np.float64), "idx": idx.cpu().numpy(), "n": n.cpu().numpy(),
            "counts": counts.cpu().numpy(), "active": bits, "status": status}


def check_chunk(got, c, lay, x, bias=True, norm="rms"):
    import oracle
    from _parity import y_violations
    ref = oracle.chunk_reference(x, lay.Wr, lay.br if bias else None, lay.g, lay.W1, lay.W2, norm=norm)
    n = int(got["n"][c])
    assert n == len(ref["active_idx"]), (c, n, len(ref["active_idx"]))
    assert np.array_equal(got["idx"][c][:n], ref["active_idx"]), c
    assert np.array_equal(got["active"][c], ref["active"]), c
    assert tuple(got["counts"][c]) == (ref["tls_zero"], ref["cls_zero"]), c
    bad = y_violations(got["y"][c], ref["y"])
    assert not bad.any(), (f"chunk {c}: {int(bad.sum())} of {bad.size} y elements out of tolerance; max abs err "
                           f"{np.abs(got['y'][c] - ref['y']).max():.3e}")
    silent = ~ref["active"].any(axis=1)
    assert np.all(got["y"][c][silent] == 0.0)


def test_tiny_workload_every_chunk_in_one_call(bffn, cuda_device):
    w = gen.workload("tiny")
    lay = w.layer(0)
    sl = StackedLayers([lay])
    xs = w.chunks(lay, w.n_chunks)
    got = run_batch(bffn, sl, xs)
    assert got["status"] == bffn.BFFN_OK
    for c in range(w.n_chunks):
        check_chunk(got, c, lay, xs[c])


@pytest.mark.parametrize("teams", [0, 1, 3])
def test_decode_layer_two_stacked_layers(bffn, cuda_device, teams):
    # the 1B-class decode layer, two layers stacked, chunk c on layer c % 2, several team counts
    w = gen.workload("decode")
    lays = [w.layer(0), w.layer(1)]
    sl = StackedLayers(lays)
    C = 12
    xs = np.concatenate([w.chunks(lays[0], C // 2, replica=0), w.chunks(lays[1], C // 2, replica=1)])
    order = np.array([c // 2 + (c % 2) * (C // 2) for c in range(C)])  # chunk c from layer c % 2
    xs = xs[order]
    got = run_batch(bffn, sl, xs, teams=teams)
    assert got["status"] == bffn.BFFN_OK
    for c in (0, 1, 6, 11):
        check_chunk(got, c, lays[c % 2], xs[c])


@pytest.mark.parametrize("L", [1, 2, 5, 8])
def test_chunk_lengths_width_4096(bffn, cuda_device, L):
    w = gen.workload("lsweep", L=L)
    lay = w.layer(0)
    sl = StackedLayers([lay])
    xs = w.chunks(lay, 3)
    got = run_batch(bffn, sl, xs, teams=3)
    assert got["status"] == bffn.BFFN_OK
    for c in range(3):
        check_chunk(got, c, lay, xs[c])


@pytest.mark.parametrize("shape", [
    dict(d=256, E=40, de=64, L=5),
    dict(d=256, E=33, de=64, L=7),
    dict(d=128, E=1, de=32, L=3),
    dict(d=64, E=1024, de=16, L=3),
    dict(d=4112, E=24, de=272, L=7),   # ragged tails of d and de
    dict(d=264, E=24, de=72, L=5),     # multiples of 8, not of 16
    dict(d=24, E=8, de=8, L=3),
    dict(d=384, E=40, de=320, L=8),    # groups of 128, 128, 64 rows per expert
])
def test_edge_shapes(bffn, cuda_device, shape):
    lay = gen.make_layer(11, shape["d"], shape["E"], shape["de"], 0.8, 1.09)
    sl = StackedLayers([lay])
    xs = gen.make_chunks(11, lay, 4, shape["L"], 0.3)
    got = run_batch(bffn, sl, xs, teams=2)
    assert got["status"] == bffn.BFFN_OK
    for c in range(4):
        check_chunk(got, c, lay, xs[c])


def test_empty_full_and_silent_chunks(bffn, cuda_device):
    # layer 0: no expert ever active; layer 1: every expert active; layer 2: normal, one silent token
    lays = [gen.make_layer(3 + k, 256, 16, 64, 0.8, 1.09) for k in range(3)]
    lays[0].br[:] = -50.0
    lays[1].br[:] = 50.0
    sl = StackedLayers(lays)
    xs = np.stack([gen.make_chunks(3 + (c % 3), lays[c % 3], 1, 8, 0.3, stream=c)[0] for c in range(6)])
    xs[2][3] = 0  # s = b < 0 for every expert of layer 2: this token's row of y must be exactly zero
    xs[5][0] = 0
    got = run_batch(bffn, sl, xs, teams=2)
    assert got["status"] == bffn.BFFN_OK
    for c in range(6):
        check_chunk(got, c, lays[c % 3], xs[c])
    assert got["n"][0] == 0 and got["n"][3] == 0 and np.all(got["y"][0] == 0.0)
    assert got["n"][1] == 16 and got["n"][4] == 16


def test_layer_index_array_and_repeatability(bffn, cuda_device):
    import torch
    lays = [gen.make_layer(21 + k, 512, 32, 128, 1.0, 1.16) for k in range(3)]
    sl = StackedLayers(lays)
    layer = [2, 0, 0, 1, 2, 1, 0]
    xs = np.stack([gen.make_chunks(21, lays[l], 1, 8, 0.4, stream=c)[0] for c, l in enumerate(layer)])
    ws = bffn.new_batch_workspace(len(layer), 8, 512, 32, 128, teams=2)
    a = run_batch(bffn, sl, xs, layer=layer, teams=2, workspace=ws)
    b = run_batch(bffn, sl, xs, layer=layer, teams=2, workspace=ws)
    assert a["status"] == bffn.BFFN_OK and b["status"] == bffn.BFFN_OK
    assert np.array_equal(a["y"], b["y"])  # bit-reproducible
    for c, l in enumerate(layer):
        check_chunk(a, c, lays[l], xs[c])
    torch.cuda.synchronize()


def test_matches_the_single_chunk_entry_point(bffn, cuda_device):
    # the same chunks through blockffn_chunk_forward_ex: identical unions and counts, y within tolerance
    from _parity import DeviceLayer, run_chunk, y_violations
    w = gen.workload("decode")
    lay = w.layer(0)
    sl = StackedLayers([lay])
    xs = w.chunks(lay, 4)
    got = run_batch(bffn, sl, xs, teams=4)
    dl = DeviceLayer(lay)
    for c in range(4):
        one = run_chunk(bffn, dl, xs[c])
        assert int(got["n"][c]) == one["n_active"]
        assert np.array_equal(got["idx"][c][:one["n_active"]], one["active_idx"])
        assert not y_violations(got["y"][c], one["y"]).any()


def test_bad_layer_index_is_reported(bffn, cuda_device):
    lays = [gen.make_layer(31, 256, 16, 64, 0.8, 1.09)]
    sl = StackedLayers(lays)
    xs = gen.make_chunks(31, lays[0], 3, 8, 0.3)
    got = run_batch(bffn, sl, xs, layer=[0, 5, 0], teams=1)
    assert got["status"] == bffn.BFFN_EINVAL
    assert got["n"][1] == 0 and np.all(got["y"][1] == 0.0)
    assert tuple(got["counts"][1]) == (8 * 16, 16)
    check_chunk(got, 0, lays[0], xs[0])
    check_chunk(got, 2, lays[0], xs[2])


@pytest.mark.parametrize("tls", [0.50, 0.95])
def test_sparsity_sweep_points_width_4096(bffn, cuda_device, tls):
    # the stacked-model sweep's layer (d=4096, E=128, de=256, L=8) at its extreme token-level sparsity
    # points, two layers, 8 teams of SMs, three chunks per team; oracle on the first two chunks
    lays = [gen.make_layer(41 + k, 4096, 128, 256, gen.beta_for_tls(tls), 1.09) for k in range(2)]
    sl = StackedLayers(lays)
    C = 24
    xs = np.stack([gen.make_chunks(41, lays[c % 2], 1, 8, 0.3, stream=c)[0] for c in range(C)])
    got = run_batch(bffn, sl, xs, teams=8)
    assert got["status"] == bffn.BFFN_OK
    for c in (0, 1):
        check_chunk(got, c, lays[c % 2], xs[c])


def test_every_expert_active_long_phases(bffn, cuda_device):
    # every one of 128 experts active at d=4096: up-projection phases of several hundred stages per CTA
    # and several chunks per team (the copy warp and the consumers stay within one pass of the ring)
    lay = gen.make_layer(51, 4096, 128, 256, 0.0, 1.09)
    lay.br[:] = 50.0
    sl = StackedLayers([lay])
    C = 32
    xs = gen.make_chunks(51, lay, C, 8, 0.3)
    got = run_batch(bffn, sl, xs, teams=8)
    assert got["status"] == bffn.BFFN_OK
    assert np.all(got["n"] == 128)
    check_chunk(got, C - 1, lay, xs[C - 1])


def test_remoe_router_variant(bffn, cuda_device):
    # the sum-normalised (ReMoE) router through the batched call: two layers with unequal gains
    lays = [gen.make_layer(61 + k, 512, 32, 128, 1.0, 1.09) for k in range(2)]
    for lay in lays:
        lay.g[:] = np.linspace(0.5, 2.0, 32, dtype=np.float32)
    sl = StackedLayers(lays)
    xs = np.stack([gen.make_chunks(61, lays[c % 2], 1, 8, 0.3, stream=c)[0] for c in range(6)])
    got = run_batch(bffn, sl, xs, teams=2, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM)
    assert got["status"] == bffn.BFFN_OK
    for c in range(6):
        check_chunk(got, c, lays[c % 2], xs[c], norm="sum")

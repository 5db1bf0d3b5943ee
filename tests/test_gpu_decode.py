"""GPU parity of the decode path (L <= 32) against the fp64 oracle, through the C ABI.

Bit-exact: per-token active flags, the union list, n_active, the sparsity counts.
Within tolerance: r (fp32 vs fp64) and y (|y - y_ref| <= 2e-2 |y_ref| + 1e-3 rms(y_ref)).
"""
import numpy as np
import pytest

import gen

pytestmark = pytest.mark.gpu


def _layer(seed, d, E, de, beta=0.8, noise=0.3):
    from _parity import DeviceLayer
    lay = gen.make_layer(seed, d, E, de, beta, 1.0 + noise ** 2)
    return DeviceLayer(lay)


def _check_chunks(bffn, dl, xs, **kw):
    from _parity import assert_parity, reference, run_chunk
    for x in xs:
        got = run_chunk(bffn, dl, x, **kw)
        ref = reference(dl, x, bias=kw.get("bias", True))
        assert_parity(got, ref, x.shape[0], dl.E, check_r=not kw.get("plain", False))


def test_tiny_workload_every_chunk(bffn, cuda_device):
    w = gen.workload("tiny")
    from _parity import DeviceLayer
    dl = DeviceLayer(w.layer(0))
    xs = w.chunks(dl.lay, w.n_chunks)
    _check_chunks(bffn, dl, xs)


def test_decode_1b_layer_sampled_chunks(bffn, cuda_device):
    w = gen.workload("decode")
    from _parity import DeviceLayer
    dl = DeviceLayer(w.layer(0))
    xs = w.chunks(dl.lay, 4)
    _check_chunks(bffn, dl, xs)


@pytest.mark.parametrize("L", [1, 2, 4, 8, 16, 32])
def test_chunk_size_sweep_width_4096(bffn, cuda_device, L):
    w = gen.workload("lsweep", L=L)
    from _parity import DeviceLayer
    dl = DeviceLayer(w.layer(0))
    xs = w.chunks(dl.lay, 1)
    _check_chunks(bffn, dl, xs)


@pytest.mark.parametrize("shape", [
    dict(d=256, E=40, de=64, L=5),     # 40 experts (the expert count the BlockFFN article found best)
    dict(d=256, E=33, de=64, L=13),    # union words cross a 32-expert boundary; L not a multiple of 8
    dict(d=16, E=16, de=16, L=8),      # minimum widths
    dict(d=128, E=1, de=32, L=3),      # a single expert
    dict(d=64, E=1024, de=16, L=3),    # maximum expert count
    dict(d=4112, E=24, de=272, L=7),   # K chunks with a ragged tail in both projections
    # chunks of more than 8 tokens (tcgen05 kernel)
    dict(d=16, E=16, de=16, L=9),      # minimum widths
    dict(d=128, E=1, de=32, L=31),     # a single expert
    dict(d=64, E=1024, de=16, L=12),   # maximum expert count
    dict(d=4112, E=24, de=272, L=17),  # ragged tails in both projections; 3 up-projection blocks per expert
    dict(d=384, E=40, de=320, L=24),   # up-projection blocks of 112, 112 and 96 rows
    # widths that are multiples of 8 but not of 16, on both kernels
    dict(d=264, E=24, de=72, L=5),     # warp MMAs: a 16-byte tail piece of d and a 8-column tail of de
    dict(d=264, E=24, de=72, L=12),    # tcgen05
    dict(d=24, E=8, de=8, L=3),        # minimum widths: one 16-byte piece of de, three of d
    dict(d=24, E=8, de=8, L=9),
])
def test_edge_shapes(bffn, cuda_device, shape):
    dl = _layer(11, shape["d"], shape["E"], shape["de"])
    xs = gen.make_chunks(11, dl.lay, 2, shape["L"], 0.3)
    _check_chunks(bffn, dl, xs)


@pytest.mark.parametrize("L", [8, 24])
def test_no_active_expert(bffn, cuda_device, L):
    from _parity import run_chunk
    dl = _layer(3, 256, 16, 64)
    dl.lay.br[:] = -50.0
    dl.br.fill_(-50.0)
    x = gen.make_chunks(3, dl.lay, 1, L, 0.3)[0]
    got = run_chunk(bffn, dl, x)
    assert got["n_active"] == 0
    assert got["counts"] == (L * 16, 16)
    assert np.all(got["y"] == 0.0) and np.all(got["r"] == 0.0)


@pytest.mark.parametrize("L", [8, 32])
def test_every_expert_active(bffn, cuda_device, L):
    dl = _layer(4, 256, 16, 64)
    dl.lay.br[:] = 50.0
    dl.br.fill_(50.0)
    xs = gen.make_chunks(4, dl.lay, 1, L, 0.3)
    _check_chunks(bffn, dl, xs)


@pytest.mark.parametrize("L", [8, 20])
def test_token_without_active_expert(bffn, cuda_device, L):
    dl = _layer(5, 256, 16, 64)
    x = gen.make_chunks(5, dl.lay, 1, L, 0.3)[0]
    x[3] = 0  # s = b < 0 for every expert: this token's row of y must be exactly zero
    _check_chunks(bffn, dl, [x])


def test_plain_entry_point_without_bias(bffn, cuda_device):
    dl = _layer(6, 512, 32, 128, beta=0.0)
    xs = gen.make_chunks(6, dl.lay, 2, 8, 0.3)
    # with no bias the margin is re-checked against the bias-free pre-activation
    from _parity import reference
    import oracle
    for x in xs:
        s, _, _ = oracle.router(x, dl.lay.Wr, None, dl.lay.g)
        assert np.abs(s).min() >= 1e-3
    _check_chunks(bffn, dl, xs, plain=True, bias=False)


@pytest.mark.parametrize("L", [8, 16])
def test_caller_workspace_and_repeatability(bffn, cuda_device, L):
    from _parity import run_chunk
    dl = _layer(8, 1024, 64, 128, beta=1.0)
    x = gen.make_chunks(8, dl.lay, 1, L, 0.4)[0]
    ws = bffn.new_workspace(L, 1024, 64, 128)
    a = run_chunk(bffn, dl, x, workspace=ws)
    b = run_chunk(bffn, dl, x, workspace=ws)
    c = run_chunk(bffn, dl, x)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["y"], c["y"])  # bitwise reproducible
    assert np.array_equal(a["active_idx"], c["active_idx"])


@pytest.mark.parametrize("share,L", [(2, 8), (4, 8), (4, 16)])
def test_concurrency_hint_keeps_parity(bffn, cuda_device, share, L):
    # flags bits 4-7 = k: the expert kernel takes 1/k of the SMs (a different work split); k calls on
    # k streams with their own workspaces run side by side, each still exact against the oracle
    import torch
    from _parity import assert_parity, bf16_tensor, reference
    w = gen.workload("decode", L=L)
    from _parity import DeviceLayer
    dl = DeviceLayer(w.layer(0))
    xs = w.chunks(dl.lay, share)
    L, d, E, de = w.L, w.d, w.E, w.de
    streams = [torch.cuda.Stream() for _ in range(share)]
    wss = [bffn.new_workspace(L, d, E, de) for _ in range(share)]
    outs = []
    torch.cuda.synchronize()
    for k in range(share):
        x = bf16_tensor(xs[k])
        y = torch.full((L, d), float("nan"), dtype=torch.float32, device="cuda")
        idx = torch.full((E,), -7, dtype=torch.int32, device="cuda")
        n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        mask = torch.zeros((L, (E + 31) // 32), dtype=torch.int32, device="cuda")
        counts = torch.full((2,), -7, dtype=torch.int32, device="cuda")
        r = torch.full((L, E), float("nan"), dtype=torch.float32, device="cuda")
        rc = bffn.blockffn_chunk_forward_ex(x.data_ptr(), L, d, dl.Wr.data_ptr(), dl.g.data_ptr(), dl.W1.data_ptr(),
                                            dl.W2.data_ptr(), E, de, y.data_ptr(), idx.data_ptr(), n.data_ptr(),
                                            dl.br.data_ptr(), mask.data_ptr(), counts.data_ptr(), r.data_ptr(),
                                            bffn.BFFN_FLAGS_SHARE(share), wss[k].data_ptr(), wss[k].numel(),
                                            streams[k].cuda_stream)
        assert rc == 0, bffn.blockffn_status_string(rc)
        outs.append((x, y, idx, n, mask, counts, r))
    torch.cuda.synchronize()
    for k in range(share):
        assert bffn.device_status(workspace=wss[k]) == 0
        x, y, idx, n, mask, counts, r = outs[k]
        nn = int(n.item())
        words = mask.cpu().numpy().view(np.uint32)
        bits = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(L, -1)[:, :E]
        got = {"y": y.cpu().numpy().astype(np.float64), "active_idx": idx.cpu().numpy()[:nn], "n_active": nn,
               "active": bits, "counts": tuple(int(v) for v in counts.cpu().numpy()),
               "r": r.cpu().numpy().astype(np.float64)}
        assert_parity(got, reference(dl, xs[k]), L, E)


@pytest.mark.parametrize("L", [5, 12])
def test_stale_workspace_bytes_do_not_leak(bffn, cuda_device, L):
    # a caller workspace whose every byte past the header is 0xFF (a bf16 NaN pattern): the columns past
    # de of an expert's last h tile must be written (zeroed) before the down-projection reads them
    import torch
    dl = _layer(12, 264, 24, 72)
    xs = gen.make_chunks(12, dl.lay, 2, L, 0.3)
    ws = bffn.new_workspace(L, 264, 24, 72)
    ws[256:] = 255
    torch.cuda.synchronize()
    _check_chunks(bffn, dl, xs, workspace=ws)


@pytest.mark.parametrize("L", [8, 16])
def test_injected_router_timeout_is_reported_and_recovers(bffn, cuda_device, L):
    # the fault-injection flag makes the router barrier wait for one CTA more than the launch has; every
    # CTA gives up after 1 ms, records the timeout and exits; the status query reports BFFN_ETIMEOUT
    # once, and the next call on the same workspace is exact again
    import torch
    from _parity import bf16_tensor, reference, run_chunk, assert_parity
    dl = _layer(13, 512, 32, 128)
    x = gen.make_chunks(13, dl.lay, 1, L, 0.3)[0]
    ws = bffn.new_workspace(L, 512, 32, 128)
    xt = bf16_tensor(x)
    y = torch.zeros((L, 512), dtype=torch.float32, device="cuda")
    idx = torch.zeros(32, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = bffn.blockffn_chunk_forward_ex(xt.data_ptr(), L, 512, dl.Wr.data_ptr(), dl.g.data_ptr(), dl.W1.data_ptr(),
                                        dl.W2.data_ptr(), 32, 128, y.data_ptr(), idx.data_ptr(), n.data_ptr(),
                                        dl.br.data_ptr(), None, None, None, bffn.BFFN_FLAG_INJECT_ROUTER_TIMEOUT,
                                        ws.data_ptr(), ws.numel(), stream)
    assert rc == bffn.BFFN_OK
    assert bffn.device_status(workspace=ws) == bffn.BFFN_ETIMEOUT
    assert bffn.device_status(workspace=ws) == bffn.BFFN_OK  # read and cleared
    got = run_chunk(bffn, dl, x, workspace=ws)
    assert_parity(got, reference(dl, x), L, 32)


def test_allocation_failure_is_reported(bffn, cuda_device, monkeypatch):
    # BFFN_TEST_FAIL_ALLOC=1 makes every call that uses the library's own workspace fail as its
    # allocation would on a device without free memory (a host-side stand-in): BFFN_ENOMEM with nothing
    # enqueued (so the placeholder pointers below are never dereferenced), and a later call runs normally
    import torch
    from _parity import assert_parity, reference, run_chunk
    L, d, E, de = 32, 4096, 1024, 256  # a larger internal workspace than any other test needs
    need = bffn.blockffn_workspace_size(L, d, E, de)
    fake = 1 << 20
    monkeypatch.setenv("BFFN_TEST_FAIL_ALLOC", "1")
    rc = bffn.blockffn_chunk_forward(fake, L, d, fake, fake, fake, fake, E, de, fake, fake, fake,
                                     torch.cuda.current_stream().cuda_stream)
    assert rc == bffn.BFFN_ENOMEM, bffn.blockffn_status_string(rc)
    assert need > 0
    monkeypatch.delenv("BFFN_TEST_FAIL_ALLOC")
    dl = _layer(14, 256, 16, 64)
    x = gen.make_chunks(14, dl.lay, 1, 8, 0.3)[0]
    assert_parity(run_chunk(bffn, dl, x), reference(dl, x), 8, 16)


@pytest.mark.parametrize("L", [5, 8, 16])
def test_remoe_router_variant(bffn, cuda_device, L):
    # BFFN_FLAG_ROUTER_SUM_NORM: r = g relu(s) / sum relu(s) (the ReMoE router) on both per-chunk kernels;
    # masks, union and counts as for RMSNorm, r and y against the oracle's sum-normalised router
    from _parity import assert_parity, reference, run_chunk
    dl = _layer(15, 512, 32, 128)
    dl.lay.g[:] = np.linspace(0.5, 2.0, 32, dtype=np.float32)
    dl.g.copy_(__import__("torch").from_numpy(dl.lay.g))
    for x in gen.make_chunks(15, dl.lay, 2, L, 0.3):
        got = run_chunk(bffn, dl, x, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM)
        assert_parity(got, reference(dl, x, norm="sum"), L, 32)


def test_union_overlap_of_consecutive_chunks(bffn, cuda_device):
    # a drifting sequence's consecutive chunks through the per-chunk path; blockffn_union_overlap of step
    # k's and step k-1's active lists equals the overlap of the oracle's unions (an integer, bit-exact);
    # calls made with BFFN_FLAG_KEEP_EXPERTS_IN_L2 return the same bits as calls without it
    import oracle
    import torch
    from _parity import bf16_tensor, run_chunk, assert_parity, reference
    dl = _layer(16, 512, 32, 128, beta=1.0)
    xs = gen.make_sequence_chunks(16, dl.lay, 6, 8, 0.3, 0.95)
    idx = torch.full((6, 32), -1, dtype=torch.int32, device="cuda")
    n = torch.zeros(6, dtype=torch.int32, device="cuda")
    unions = []
    for k, x in enumerate(xs):
        got = run_chunk(bffn, dl, x, flags=bffn.BFFN_FLAG_KEEP_EXPERTS_IN_L2 if k % 2 else 0)
        ref = reference(dl, x)
        assert_parity(got, ref, 8, 32)
        if k % 2:  # the cache policy changes no arithmetic
            again = run_chunk(bffn, dl, x)
            assert np.array_equal(again["y"], got["y"])
        idx[k, :got["n_active"]] = torch.from_numpy(got["active_idx"].astype(np.int32)).cuda()
        n[k] = got["n_active"]
        unions.append(ref["active_idx"])
    overlap = torch.full((5,), -1, dtype=torch.int32, device="cuda")
    rc = bffn.blockffn_union_overlap(idx[:5].data_ptr(), n[:5].data_ptr(), idx[1:].data_ptr(), n[1:].data_ptr(), 5, 32,
                                     overlap.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == bffn.BFFN_OK
    torch.cuda.synchronize()
    want = [oracle.union_overlap(unions[k], unions[k + 1], 32) for k in range(5)]
    assert overlap.cpu().numpy().tolist() == want
    assert max(want) > 0

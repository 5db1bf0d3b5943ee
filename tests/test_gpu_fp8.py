"""GPU parity of the fp8 expert-weight path (blockffn_quantize_fp8, blockffn_chunk_forward_batch_fp8).

Bit-exact: the codes and the scales against the oracle's quantiser; per chunk the active flags, the union
list, n_active and the counts.  Within tolerance per chunk: y against the fp64 oracle evaluated on the weights
the quantised format stands for (the oracle dequantises its own codes: every dequantised weight is a bf16
value), |y - y_ref| <= 2e-2 |y_ref| + 1e-3 rms(y_ref).  Reruns are bit-identical.
"""
import copy

import numpy as np
import pytest

import gen

pytestmark = pytest.mark.gpu


def _bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _quantised(bffn, layers):
    """Quantise on the GPU, compare with the oracle's quantiser bit for bit, and return the device format
    plus per-layer copies whose W1, W2 are the dequantised weights (for the reference)."""
    import oracle
    W1 = np.concatenate([l.W1 for l in layers])
    W2 = np.concatenate([l.W2 for l in layers])
    q = bffn.quantize_fp8(_bf16(W1), _bf16(W2), len(layers))
    import torch
    torch.cuda.synchronize()
    q1, q2, s1, s2, t2 = oracle.quantize_fp8(W1, W2, len(layers))
    got = [t.cpu().numpy() for t in q]
    assert np.array_equal(got[0], q1) and np.array_equal(got[1], q2), "codes differ from the oracle's"
    for a, b in zip(got[2:], (s1, s2, t2)):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), "scales differ from the oracle's"
    D1, D2 = oracle.dequantize_fp8(q1, q2, s1, s2, t2)
    E = layers[0].E
    deq = []
    for i, l in enumerate(layers):
        c = copy.copy(l)
        c.W1, c.W2 = D1[i * E:(i + 1) * E], D2[i * E:(i + 1) * E]
        deq.append(c)
    return q, deq


def _run(bffn, layers, q, xs, layer=None, flags=0, bias=True):
    import torch
    from test_gpu_batch import StackedLayers
    sl = StackedLayers(layers)
    C, L, d = xs.shape
    E = sl.E
    y = torch.full((C, L, d), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((C, E), -7, dtype=torch.int32, device="cuda")
    n = torch.full((C,), -7, dtype=torch.int32, device="cuda")
    counts = torch.full((C, 2), -7, dtype=torch.int32, device="cuda")
    mask = torch.zeros((C, L, (E + 31) // 32), dtype=torch.int32, device="cuda")
    lt = None if layer is None else torch.from_numpy(np.asarray(layer, np.int32)).cuda()
    bffn.chunk_forward_batch_fp8(_bf16(xs), sl.Wr, sl.g, q, y, idx, n, layer=lt, br=sl.br if bias else None,
                                 counts=counts, tok_mask=mask, flags=flags)
    torch.cuda.synchronize()
    words = mask.cpu().numpy().view(np.uint32)
    bits = ((words[..., None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(C, L, -1)[:, :, :E]
    return {"y": y.cpu().numpy().astype(np.float64), "idx": idx.cpu().numpy(), "n": n.cpu().numpy(),
            "counts": counts.cpu().numpy(), "active": bits}


@pytest.mark.parametrize("shape", [
    dict(d=272, E=24, de=80, L=3, C=37, nl=2),    # ragged d (a 16-byte tail past 256) and de; two layers
    dict(d=512, E=40, de=128, L=8, C=20, nl=1),   # union words cross 32 experts
    dict(d=64, E=1, de=16, L=1, C=9, nl=3),       # minimum widths, one expert, single tokens
])
def test_fp8_shapes(bffn, cuda_device, shape):
    from test_gpu_batch import check_chunk
    layers = [gen.make_layer(70 + k, shape["d"], shape["E"], shape["de"], 0.8, 1.09) for k in range(shape["nl"])]
    q, deq = _quantised(bffn, layers)
    xs = np.stack([gen.make_chunks(71, layers[c % shape["nl"]], 1, shape["L"], 0.3, stream=c)[0]
                   for c in range(shape["C"])])
    got = _run(bffn, layers, q, xs)
    for c in range(shape["C"]):
        check_chunk(got, c, deq[c % shape["nl"]], xs[c])


def test_fp8_decode_layer_sampled(bffn, cuda_device):
    """The 1B-class decode layer (d = 2048, E = 64, de = 256), 64 chunks of 8 tokens over two layers,
    every 8th chunk against the oracle; reruns bit-identical."""
    from test_gpu_batch import check_chunk
    w = gen.workload("decode")
    layers = [w.layer(0), w.layer(1)]
    q, deq = _quantised(bffn, layers)
    xs = np.stack([w.chunks(layers[c % 2], 1, replica=c)[0] for c in range(64)])
    got = _run(bffn, layers, q, xs)
    again = _run(bffn, layers, q, xs)
    assert np.array_equal(got["y"], again["y"])
    for c in range(0, 64, 8):
        check_chunk(got, c, deq[c % 2], xs[c])


def test_fp8_empty_and_full_unions_layer_array_remoe(bffn, cuda_device):
    """A chunk with no active expert (y exactly 0), one with every expert active, chunks routed by a layer
    array, and the ReMoE router."""
    from test_gpu_batch import check_chunk
    layers = [gen.make_layer(80 + k, 256, 32, 64, 0.8, 1.09) for k in range(2)]
    q, deq = _quantised(bffn, layers)
    lay_idx = [1, 0, 0, 1, 1, 0]
    # each chunk drawn against the layer it is routed to, so the 1e-3 margin holds for that layer
    xs = np.stack([gen.make_chunks(81, layers[lay_idx[k]], 1, 8, 0.3, stream=k)[0] for k in range(6)])
    got = _run(bffn, layers, q, xs, layer=lay_idx)
    for c in range(6):
        check_chunk(got, c, deq[lay_idx[c]], xs[c])
    got = _run(bffn, layers, q, xs, layer=lay_idx, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM)
    for c in range(6):
        check_chunk(got, c, deq[lay_idx[c]], xs[c], norm="sum")
    # every expert off (bias far below), then every expert on (bias far above)
    for b in (-50.0, 50.0):
        ls = [copy.copy(l) for l in layers]
        for l in ls:
            l.br = np.full_like(l.br, b)
        dq = [copy.copy(d_) for d_ in deq]
        for l in dq:
            l.br = np.full_like(l.br, b)
        got = _run(bffn, ls, q, xs[:2], layer=lay_idx[:2])
        for c in range(2):
            check_chunk(got, c, dq[lay_idx[c]], xs[c])
        if b < 0:
            assert np.all(got["y"] == 0.0) and np.all(got["n"] == 0)

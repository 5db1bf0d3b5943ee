"""The allocation-free entry point, blockffn_chunk_forward_noalloc.

It exists for callers that cannot call cudaMalloc (a serving engine that has reserved all device
memory up front, code that must not synchronise the device).  It must give the same results as the
regular entry point, blockffn_chunk_forward_ex, on back-to-back calls that share its compiled-in
scratch array.  This file is collected last so that a run stopping at the first failure has already
run every other test.
"""
import numpy as np
import pytest
import torch

import gen


def test_noalloc_rejects_sizes_beyond_its_scratch(bffn):
    # L=32, E=1024, de=256 needs ~32 MiB of scratch, more than the compiled-in 8 MiB: rejected
    # before any pointer is touched or any work is enqueued (no GPU needed).
    assert bffn.blockffn_workspace_size(32, 4096, 1024, 256) > bffn.NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    rc = bffn.blockffn_chunk_forward_noalloc(fake, 32, 4096, fake, fake, fake, fake, 1024, 256, fake, fake, fake,
                                             None, None)
    assert rc == bffn.BFFN_ENOMEM


def test_noalloc_takes_decode_chunks_only(bffn):
    # chunks longer than 32 tokens (the prefill path) are refused before anything is enqueued
    fake = 1 << 20
    rc = bffn.blockffn_chunk_forward_noalloc(fake, 64, 256, fake, fake, fake, fake, 16, 64, fake, fake, fake,
                                             None, None)
    assert rc == bffn.BFFN_EUNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("L", [8, 16])  # 16 tokens: the tcgen05 decode kernel and its stream-K scratch
def test_noalloc_matches_regular_entry_point_on_two_calls(bffn, cuda_device, L):
    from _parity import DeviceLayer, bf16_tensor, y_violations

    w = gen.workload("decode", L=L)
    dl = DeviceLayer(w.layer(0))
    xs = w.chunks(dl.lay, 2)
    L, d, E, de = w.L, w.d, w.E, w.de
    assert bffn.blockffn_workspace_size(L, d, E, de) <= bffn.NOALLOC_SCRATCH_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # two calls in a row share (and reuse) the scratch array
        x = bf16_tensor(xs[call])
        outs = []
        for which in ("regular", "noalloc"):
            y = torch.full((L, d), float("nan"), dtype=torch.float32, device=cuda_device)
            idx = torch.full((E,), -1, dtype=torch.int32, device=cuda_device)
            n = torch.full((1,), -1, dtype=torch.int32, device=cuda_device)
            args = (x.data_ptr(), L, d, dl.Wr.data_ptr(), dl.g.data_ptr(), dl.W1.data_ptr(), dl.W2.data_ptr(),
                    E, de, y.data_ptr(), idx.data_ptr(), n.data_ptr(), dl.br.data_ptr())
            if which == "regular":
                rc = bffn.blockffn_chunk_forward_ex(*args, None, None, None, 0, None, 0, stream)
            else:
                rc = bffn.blockffn_chunk_forward_noalloc(*args, stream)
            assert rc == bffn.BFFN_OK, bffn.blockffn_status_string(rc)
            torch.cuda.synchronize()
            if which == "noalloc":  # no bounded device wait of this entry point ran out
                assert bffn.blockffn_noalloc_device_status(stream) == bffn.BFFN_OK
            nn = int(n.item())
            outs.append((y.cpu().numpy().astype(np.float64), idx.cpu().numpy()[:nn], nn))
        (y_ref, idx_ref, n_ref), (y_new, idx_new, n_new) = outs
        assert n_new == n_ref and np.array_equal(idx_new, idx_ref)
        assert not y_violations(y_new, y_ref).any()

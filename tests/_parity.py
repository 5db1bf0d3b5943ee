"""Shared helpers of the GPU parity tests: run one chunk through the C ABI and compare every output
with the fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import gen
import oracle

# y tolerance: |y - y_ref| <= 2e-2 |y_ref| + 1e-3 rms(y_ref), per element (rms over the call's y_ref)
Y_RTOL = 2e-2
Y_ATOL_RMS = 1e-3
# router output r = g relu(s) / rms: s is an fp32 dot product over d ~ 2-4K terms of size O(1/sqrt(d)),
# so its absolute rounding error is ~1e-6..1e-5 whatever the summation order, and rms(r/g) = 1 puts
# r on the same O(1) scale: |r - r_ref| <= 1e-5 + 1e-5 |r_ref|.
R_RTOL = 1e-5
R_ATOL = 1e-5


class DeviceLayer:
    def __init__(self, lay: gen.Layer, device="cuda"):
        self.lay = lay
        self.d, self.E, self.de = lay.d, lay.E, lay.de
        self.Wr = torch.from_numpy(np.ascontiguousarray(lay.Wr)).to(device)
        self.br = torch.from_numpy(np.ascontiguousarray(lay.br)).to(device)
        self.g = torch.from_numpy(np.ascontiguousarray(lay.g)).to(device)
        self.W1 = torch.from_numpy(lay.W1.view(np.int16)).to(device).view(torch.bfloat16)
        self.W2 = torch.from_numpy(lay.W2.view(np.int16)).to(device).view(torch.bfloat16)


def bf16_tensor(bits: np.ndarray, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def run_chunk(bffn, dl: DeviceLayer, x_bits: np.ndarray, bias=True, path=0, workspace=None, plain=False, flags=0):
    L, d = x_bits.shape
    E = dl.E
    dev = dl.Wr.device
    x = bf16_tensor(x_bits, dev)
    y = torch.full((L, d), float("nan"), dtype=torch.float32, device=dev)
    idx = torch.full((E,), -7, dtype=torch.int32, device=dev)
    n = torch.full((1,), -7, dtype=torch.int32, device=dev)
    out = {"x": x}
    if plain:
        rc = bffn.blockffn_chunk_forward(x.data_ptr(), L, d, dl.Wr.data_ptr(), dl.g.data_ptr(),
                                         dl.W1.data_ptr(), dl.W2.data_ptr(), E, dl.de, y.data_ptr(),
                                         idx.data_ptr(), n.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
        assert rc == 0, bffn.blockffn_status_string(rc)
        mask = counts = r = None
    else:
        mask = torch.zeros((L, (E + 31) // 32), dtype=torch.int32, device=dev)
        counts = torch.full((2,), -7, dtype=torch.int32, device=dev)
        r = torch.full((L, E), float("nan"), dtype=torch.float32, device=dev)
        bffn.chunk_forward(x, dl.Wr, dl.g, dl.W1, dl.W2, y, idx, n, br=dl.br if bias else None,
                           tok_mask=mask, counts=counts, r_out=r, path=path, workspace=workspace, flags=flags)
    torch.cuda.synchronize()
    assert bffn.device_status(workspace) == 0
    n_act = int(n.item())
    out.update(y=y.cpu().numpy().astype(np.float64), active_idx=idx.cpu().numpy()[:max(n_act, 0)],
               n_active=n_act)
    if mask is not None:
        words = mask.cpu().numpy().view(np.uint32)
        bits = ((words[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool).reshape(L, -1)[:, :E]
        out.update(active=bits, counts=tuple(int(v) for v in counts.cpu().numpy()),
                   r=r.cpu().numpy().astype(np.float64))
    return out


def reference(dl: DeviceLayer, x_bits, bias=True, norm="rms"):
    lay = dl.lay
    return oracle.chunk_reference(x_bits, lay.Wr, lay.br if bias else None, lay.g, lay.W1, lay.W2, norm=norm)


def y_violations(y, y_ref):
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    bound = Y_RTOL * np.abs(y_ref) + Y_ATOL_RMS * rms
    return np.abs(y - y_ref) > bound


def pair_router_r_bound(dl: DeviceLayer, x_bits, bias=True, norm="rms"):
    """Extra allowance on r where the router projection carries Wr as bf16 hi + lo pairs (the prefill
    path): hi = bf16(w), lo = bf16(w - hi) leave |w - hi - lo| <= 2^-18 |w|, so the pairs move s_{t,i} by
    at most 2^-18 sum_k |x_tk Wr_ki|; the fp32 accumulation of the products is allowed three times that
    again, |ds| <= 2^-16 sum_k |x_tk Wr_ki|.  With a = relu(s) and r_i = g_i a_i / n(a), n the RMS (or
    the sum for the ReMoE router), n moves by at most max_j |ds_j| (the sum by sum_j |ds_j|), so
    |dr_i| <= (g_i |ds_i| + |r_i| dn) / n(a)."""
    lay = dl.lay
    s, r, _ = oracle.router(x_bits, lay.Wr, lay.br if bias else None, lay.g, norm=norm)
    xa = np.abs(gen.bf16_bits_to_f32(x_bits).astype(np.float64))
    ds = 2.0 ** -16 * (xa @ np.abs(lay.Wr.astype(np.float64)))
    a = np.maximum(s, 0.0)
    if norm == "sum":
        n, dn = a.sum(axis=1, keepdims=True), ds.sum(axis=1, keepdims=True)
    else:
        n, dn = np.sqrt(np.mean(a * a, axis=1, keepdims=True)), ds.max(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        bound = (lay.g.astype(np.float64)[None, :] * ds + np.abs(r) * dn) / n
    return np.where(n > 0, bound, 0.0)


def assert_parity(got, ref, L, E, check_r=True, r_bound=None):
    """Bit-exact: active flags, union list, n_active, counts. Tolerance: r (plus r_bound where given), y."""
    assert got["n_active"] == len(ref["active_idx"]), (got["n_active"], len(ref["active_idx"]))
    assert np.array_equal(got["active_idx"], ref["active_idx"])
    if "active" in got:
        assert np.array_equal(got["active"], ref["active"])
        assert got["counts"] == (ref["tls_zero"], ref["cls_zero"])
        if check_r:
            err = np.abs(got["r"] - ref["r"])
            tol = R_ATOL + R_RTOL * np.abs(ref["r"]) + (0.0 if r_bound is None else r_bound)
            assert np.all(err <= tol), err.max()
    bad = y_violations(got["y"], ref["y"])
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} y elements out of tolerance; "
                           f"max abs err {np.abs(got['y'] - ref['y']).max():.3e}")
    # tokens with no active expert produce exactly zero
    silent = ~ref["active"].any(axis=1)
    assert np.all(got["y"][silent] == 0.0)

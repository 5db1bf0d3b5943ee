"""The C-ABI library: it loads, exports every symbol include/blockffn.h declares, and rejects bad
arguments before touching the GPU (these checks need no device)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "blockffn.h")).read()
    return sorted(set(re.findall(r"BFFN_API\s+[\w\s\*]+?\b(blockffn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = _declared_symbols()
    assert "blockffn_chunk_forward" in syms and "blockffn_chunk_forward_ex" in syms
    assert "blockffn_workspace_size" in syms and "blockffn_status_string" in syms


def test_library_exports_every_declared_symbol(bffn):
    lib = C.CDLL(bffn.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert set(_declared_symbols()) == set(bffn.SIGNATURES), "binding and header disagree"


def test_only_c_symbols_are_exported(bffn):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bffn.LIB_PATH], capture_output=True, text=True).stdout
    ours = [l.split()[-1] for l in out.splitlines() if l.split()[-1].startswith("blockffn_")]
    assert sorted(ours) == _declared_symbols()


def test_status_strings(bffn):
    assert bffn.blockffn_status_string(0) == "ok"
    assert "invalid" in bffn.blockffn_status_string(1)
    assert bffn.blockffn_status_string(99) == "unknown status"
    assert bffn.blockffn_abi_version() >= 100


def test_workspace_size(bffn):
    assert bffn.blockffn_workspace_size(8, 2048, 64, 256) > 256
    big = bffn.blockffn_workspace_size(32, 4096, 128, 256)
    assert big >= 128 * 64 * 256 * 2  # h: E x 2L x de bf16
    for bad in [(0, 256, 16, 64), (8, 250, 16, 64), (8, 256, 0, 64), (8, 256, 2000, 64), (8, 256, 16, 4),
                (8, 260, 16, 64), (8, 256, 16, 68), (8, 0, 16, 64)]:
        assert bffn.blockffn_workspace_size(*bad) == 0
    # widths only need to be multiples of 8
    for ok in [(8, 264, 24, 72), (5, 24, 8, 8), (12, 8, 4, 8)]:
        assert bffn.blockffn_workspace_size(*ok) > 0


FAKE = 1 << 20  # aligned, never dereferenced: every case below must fail validation first


def _call(bffn, **kw):
    a = dict(x=FAKE, L=8, d=256, Wr=FAKE, g=FAKE, W1=FAKE, W2=FAKE, E=16, de=64, y=FAKE,
             active_idx=FAKE, n_active=FAKE, br=None, tok_mask=None, counts=None, r_out=None,
             flags=0, workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return bffn.blockffn_chunk_forward_ex(**a)


@pytest.mark.parametrize("kw", [
    dict(L=0), dict(L=-3), dict(d=250), dict(d=0), dict(d=4), dict(d=260), dict(de=20), dict(de=4), dict(E=0),
    dict(E=1025),
    dict(x=None), dict(Wr=None), dict(g=None), dict(W1=None), dict(W2=None), dict(y=None),
    dict(active_idx=None), dict(n_active=None),
    dict(x=FAKE + 2), dict(W1=FAKE + 8), dict(W2=FAKE + 4), dict(Wr=FAKE + 4), dict(y=FAKE + 2),
    dict(n_active=FAKE + 1), dict(br=FAKE + 2), dict(r_out=FAKE + 1), dict(workspace=FAKE + 16),
    dict(flags=3), dict(flags=1 << 11), dict(flags=1 << 2), dict(flags=1 << 12),
])
def test_invalid_arguments_rejected_before_launch(bffn, kw):
    assert _call(bffn, **kw) == bffn.BFFN_EINVAL


def test_unsupported_path_rejected_before_launch(bffn):
    # a decode-path request for a chunk longer than the decode path takes
    assert _call(bffn, L=33, flags=bffn.BFFN_PATH_DECODE) == bffn.BFFN_EUNSUPPORTED
    # a prefill-path request for a decode-sized chunk
    assert _call(bffn, L=32, flags=bffn.BFFN_PATH_PREFILL) == bffn.BFFN_EUNSUPPORTED
    # prefill widths: d and de multiples of 64, de <= 256
    assert _call(bffn, L=64, de=96) == bffn.BFFN_EUNSUPPORTED
    assert _call(bffn, L=64, de=320) == bffn.BFFN_EUNSUPPORTED
    assert _call(bffn, L=64, d=272) == bffn.BFFN_EUNSUPPORTED


def test_injected_timeout_is_a_decode_path_flag(bffn):
    assert _call(bffn, L=64, flags=bffn.BFFN_FLAG_INJECT_ROUTER_TIMEOUT) == bffn.BFFN_EUNSUPPORTED


def test_prefill_needs_a_16_byte_aligned_y(bffn):
    assert _call(bffn, L=64, y=FAKE + 4) == bffn.BFFN_EINVAL


def test_plain_entry_point_validates(bffn):
    assert bffn.blockffn_chunk_forward(None, 8, 256, FAKE, FAKE, FAKE, FAKE, 16, 64, FAKE, FAKE, FAKE,
                                       None) == bffn.BFFN_EINVAL


def test_workspace_holds_the_selected_decode_kernel_scratch(bffn):
    # decode shapes of the tcgen05 kernel (more than 8 tokens, or d * de >= 2^20) need its stream-K
    # scratch: 160 CTA slots x 2 partial accumulators x 128 rows x LC fp32, LC = 16 or 32
    for L, d, E, de, lc in [(16, 1024, 64, 128, 16), (4, 4096, 128, 256, 16), (32, 2048, 64, 256, 32)]:
        assert bffn.blockffn_workspace_size(L, d, E, de) >= 160 * 2 * 128 * lc * 4, (L, d, E, de)
    # a chunk of 8 tokens of smaller experts takes the mma.sync kernel: header, router parts and h only
    small = bffn.blockffn_workspace_size(8, 2048, 64, 256)
    assert 64 * 4 * 2 * 8 * 128 <= small < 160 * 2 * 128 * 16 * 4


def _batch(bffn, **kw):
    a = dict(x=FAKE, C=4, L=8, d=256, layer=None, n_layers=2, Wr=FAKE, g=FAKE, br=None, W1=FAKE, W2=FAKE, E=16,
             de=64, y=FAKE, active_idx=FAKE, n_active=FAKE, counts=None, tok_mask=None, flags=0, workspace=None,
             workspace_bytes=0, stream=None)
    a.update(kw)
    return bffn.blockffn_chunk_forward_batch(**a)


@pytest.mark.parametrize("kw", [
    dict(C=0), dict(n_layers=0), dict(L=0), dict(d=250), dict(de=20), dict(E=0), dict(E=1025),
    dict(x=None), dict(W1=FAKE + 8), dict(y=None), dict(n_active=FAKE + 2), dict(layer=FAKE + 1),
    dict(flags=1), dict(flags=1 << 8), dict(workspace=FAKE + 16),
])
def test_batch_invalid_arguments_rejected_before_launch(bffn, kw):
    assert _batch(bffn, **kw) == bffn.BFFN_EINVAL


def test_batch_takes_chunks_of_up_to_8_tokens(bffn):
    assert _batch(bffn, L=9) == bffn.BFFN_EUNSUPPORTED


def test_batch_workspace_size(bffn):
    # r [C, L, E] fp32 plus two h images per team of E x ceil(de / 64) tiles of 2 KB
    n = bffn.blockffn_batch_workspace_size(4096, 8, 2048, 64, 256, bffn.BFFN_FLAGS_SHARE(8))
    assert n >= 4096 * 8 * 64 * 4 + 8 * 2 * 64 * 4 * 2048
    assert bffn.blockffn_batch_workspace_size(0, 8, 2048, 64, 256, 0) == 0
    assert bffn.blockffn_batch_workspace_size(4, 8, 2050, 64, 256, 0) == 0


def test_router_variant_flag_is_accepted_by_validation(bffn):
    # the flag passes argument checking (nothing is launched here: the placeholder x is misaligned, so the
    # call still stops at validation) and unknown bits next to it do not
    assert _call(bffn, x=FAKE + 2, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM) == bffn.BFFN_EINVAL
    assert _call(bffn, flags=bffn.BFFN_FLAG_ROUTER_SUM_NORM | (1 << 11)) == bffn.BFFN_EINVAL
    assert bffn.blockffn_batch_workspace_size(4, 8, 256, 16, 64, bffn.BFFN_FLAG_ROUTER_SUM_NORM) > 0
    assert bffn.blockffn_batch_workspace_size(4, 8, 256, 16, 64, 1 << 11) == 0


@pytest.mark.parametrize("kw", [dict(C=0), dict(E=0), dict(E=1025), dict(a=None), dict(overlap=FAKE + 2)])
def test_union_overlap_validates(bffn, kw):
    a = dict(a=FAKE, na=FAKE, b=FAKE, nb=FAKE, C=4, E=16, overlap=FAKE)
    a.update(kw)
    assert bffn.blockffn_union_overlap(a["a"], a["na"], a["b"], a["nb"], a["C"], a["E"], a["overlap"],
                                       None) == bffn.BFFN_EINVAL


def _cls_call(bffn, **kw):
    a = dict(x=FAKE, C=4, L=8, d=256, Wr=FAKE, br=None, E=64, alpha=4.0, w_al=1.0, w_cs=1.0, loss=FAKE, dS=FAKE,
             dWr=FAKE, db=FAKE, dx=FAKE, workspace=FAKE, workspace_bytes=1 << 40)
    a.update(kw)
    return bffn.blockffn_cls_losses(a["x"], a["C"], a["L"], a["d"], a["Wr"], a["br"], a["E"], a["alpha"], a["w_al"],
                                    a["w_cs"], a["loss"], a["dS"], a["dWr"], a["db"], a["dx"], a["workspace"],
                                    a["workspace_bytes"], None)


@pytest.mark.parametrize("kw", [
    dict(C=0), dict(L=0), dict(d=0), dict(d=12), dict(E=0), dict(E=1025), dict(C=1 << 16, L=1 << 15),
    dict(alpha=0.0), dict(alpha=-1.0), dict(alpha=float("inf")), dict(alpha=float("nan")), dict(w_al=float("nan")),
    dict(w_cs=float("inf")), dict(x=None), dict(x=FAKE + 8), dict(Wr=None), dict(Wr=FAKE + 2), dict(br=FAKE + 1),
    dict(loss=None), dict(dS=None), dict(dS=FAKE + 2), dict(dWr=FAKE + 2), dict(db=FAKE + 1), dict(dx=FAKE + 4),
    dict(workspace=None), dict(workspace=FAKE + 16),
])
def test_cls_losses_invalid_arguments_rejected_before_launch(bffn, kw):
    assert _cls_call(bffn, **kw) == bffn.BFFN_EINVAL


def test_cls_losses_unsupported_and_small_workspace(bffn):
    assert _cls_call(bffn, L=129) == bffn.BFFN_EUNSUPPORTED
    need = bffn.blockffn_cls_losses_workspace_size(4, 8, 256, 64)
    assert _cls_call(bffn, workspace_bytes=need - 1) == bffn.BFFN_ENOMEM


def test_cls_losses_workspace_size(bffn):
    T, d, E = 4096 * 8, 2048, 64
    n = bffn.blockffn_cls_losses_workspace_size(4096, 8, d, E)
    assert n >= 2 * d * E * 2 + 2 * T * E * 2  # the hi/lo pairs of Wr and of dS
    for bad in [(0, 8, 256, 64), (4, 0, 256, 64), (4, 8, 250, 64), (4, 8, 0, 64), (4, 8, 256, 0),
                (4, 8, 256, 1025)]:
        assert bffn.blockffn_cls_losses_workspace_size(*bad) == 0
    # experts are padded to 64 in the split copies: E = 1 and E = 64 need the same
    assert (bffn.blockffn_cls_losses_workspace_size(4, 8, 256, 1)
            == bffn.blockffn_cls_losses_workspace_size(4, 8, 256, 64))


@pytest.mark.parametrize("kw", [
    dict(n_layers=0), dict(E=0), dict(E=1025), dict(d=24), dict(de=8), dict(W1=None), dict(W1=FAKE + 8),
    dict(W2q=FAKE + 4), dict(s1=None), dict(t2=FAKE + 2),
])
def test_quantize_fp8_validates(bffn, kw):
    a = dict(W1=FAKE, W2=FAKE, n_layers=2, E=16, d=256, de=64, W1q=FAKE, W2q=FAKE, s1=FAKE, s2=FAKE, t2=FAKE)
    a.update(kw)
    assert bffn.blockffn_quantize_fp8(a["W1"], a["W2"], a["n_layers"], a["E"], a["d"], a["de"], a["W1q"], a["W2q"],
                                      a["s1"], a["s2"], a["t2"], None) == bffn.BFFN_EINVAL


@pytest.mark.parametrize("kw", [
    dict(C=0), dict(L=9), dict(d=24), dict(de=40), dict(x=None), dict(x=FAKE + 8), dict(W1q=FAKE + 4),
    dict(s2=None), dict(y=FAKE + 2), dict(layer=FAKE + 1), dict(flags=1 << 4), dict(flags=1 << 11),
    dict(workspace=FAKE + 16),
])
def test_batch_fp8_validates(bffn, kw):
    a = dict(x=FAKE, C=4, L=8, d=256, layer=None, n_layers=2, Wr=FAKE, g=FAKE, br=None, W1q=FAKE, s1=FAKE, W2q=FAKE,
             s2=FAKE, t2=FAKE, E=16, de=64, y=FAKE, active_idx=FAKE, n_active=FAKE, counts=None, tok_mask=None,
             flags=0, workspace=None, workspace_bytes=0)
    a.update(kw)
    assert bffn.blockffn_chunk_forward_batch_fp8(
        a["x"], a["C"], a["L"], a["d"], a["layer"], a["n_layers"], a["Wr"], a["g"], a["br"], a["W1q"], a["s1"],
        a["W2q"], a["s2"], a["t2"], a["E"], a["de"], a["y"], a["active_idx"], a["n_active"], a["counts"],
        a["tok_mask"], a["flags"], a["workspace"], a["workspace_bytes"], None) == bffn.BFFN_EINVAL


def test_batch_fp8_workspace_size(bffn):
    assert bffn.blockffn_batch_fp8_workspace_size(4096, 8, 2048, 64, 256) > 0
    for bad in [(0, 8, 256, 16, 64), (4, 9, 256, 16, 64), (4, 8, 24, 16, 64), (4, 8, 256, 16, 40)]:
        assert bffn.blockffn_batch_fp8_workspace_size(*bad) == 0
    # the workspace does not grow past the h buffer of one wave of chunks
    a = bffn.blockffn_batch_fp8_workspace_size(4096, 8, 2048, 64, 256)
    b = bffn.blockffn_batch_fp8_workspace_size(8192, 8, 2048, 64, 256)
    assert b - a < 8192 * 8 * 2048 * 2 + 4096 * 8 * 64 * 4 + (1 << 20)


@pytest.mark.parametrize("kw", [
    dict(T=0), dict(T=65535 * 128 + 1, d=8, E=1, de=8), dict(d=12), dict(de=4), dict(E=0), dict(E=1025),
    dict(x=None), dict(x=FAKE + 8), dict(W1=FAKE + 2), dict(dy=FAKE + 4), dict(dx=None), dict(dW2=FAKE + 2),
    dict(br=FAKE + 1), dict(workspace=None), dict(workspace=FAKE + 16),
])
def test_layer_backward_validates(bffn, kw):
    a = dict(x=FAKE, T=64, d=256, Wr=FAKE, br=None, g=FAKE, W1=FAKE, W2=FAKE, E=16, de=64, dy=FAKE, dx=FAKE,
             dWr=FAKE, db=FAKE, dg=FAKE, dW1=FAKE, dW2=FAKE, workspace=FAKE, workspace_bytes=1 << 40)
    a.update(kw)
    assert bffn.blockffn_layer_backward(
        a["x"], a["T"], a["d"], a["Wr"], a["br"], a["g"], a["W1"], a["W2"], a["E"], a["de"], a["dy"], a["dx"],
        a["dWr"], a["db"], a["dg"], a["dW1"], a["dW2"], a["workspace"], a["workspace_bytes"], None) == bffn.BFFN_EINVAL


def test_layer_backward_workspace_size(bffn):
    # sized for every pair active: the pair rows of U, Q, RH, DU and the per-pair dx terms
    assert bffn.blockffn_layer_backward_workspace_size(4096, 2048, 64, 256) > 4096 * 64 * (256 * 12 + 2048 * 4)
    assert bffn.blockffn_layer_backward_workspace_size(65535 * 128, 8, 1, 8) > 0
    assert bffn.blockffn_layer_backward_workspace_size(65535 * 128 + 1, 8, 1, 8) == 0
    for bad in [(0, 256, 16, 64), (64, 250, 16, 64), (64, 256, 0, 64), (64, 256, 16, 60)]:
        assert bffn.blockffn_layer_backward_workspace_size(*bad) == 0

"""Python binding of the BlockFFN chunk-layer C ABI (include/blockffn.h).

The functions named like the C entry points take plain integers (device pointers, sizes, a
cudaStream_t handle) and only marshal arguments; every step of the layer runs in the CUDA kernels of
libblockffn.so.  `chunk_forward` is the same call taking torch CUDA tensors (it checks dtypes,
shapes, devices and contiguity, then passes data pointers).  Importing this package fails loudly when
the extension has not been built: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libblockffn.so")

BFFN_OK, BFFN_EINVAL, BFFN_ECUDA, BFFN_ENOMEM, BFFN_ETIMEOUT, BFFN_EUNSUPPORTED = range(6)
BFFN_PATH_AUTO, BFFN_PATH_DECODE, BFFN_PATH_PREFILL = 0, 1, 2


BFFN_FLAG_INJECT_ROUTER_TIMEOUT = 0x100  # fault injection for tests of the error path (decode path)
BFFN_FLAG_ROUTER_SUM_NORM = 0x200  # the ReMoE router: r = g relu(s) / sum relu(s) instead of the RMS
BFFN_FLAG_KEEP_EXPERTS_IN_L2 = 0x400  # per-chunk decode: expert weights read with the L2 evict-last policy


def BFFN_FLAGS_SHARE(k: int) -> int:
    """Concurrency hint (decode path): the call takes 1/k of the SMs; k calls on k streams with k
    workspaces run side by side."""
    return int(k) << 4

# Every symbol include/blockffn.h declares: name -> (restype, argtypes)
_P, _I, _S, _F = C.c_void_p, C.c_int, C.c_size_t, C.c_float
SIGNATURES = {
    "blockffn_chunk_forward": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P]),
    "blockffn_chunk_forward_ex": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P,
                                       _P, _I, _P, _S, _P]),
    "blockffn_chunk_forward_noalloc": (_I, [_P, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P]),
    "blockffn_noalloc_device_status": (_I, [_P]),
    "blockffn_chunk_forward_batch": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P,
                                         _I, _P, _S, _P]),
    "blockffn_batch_workspace_size": (_S, [_I, _I, _I, _I, _I, _I]),
    "blockffn_union_overlap": (_I, [_P, _P, _P, _P, _I, _I, _P, _P]),
    "blockffn_quantize_fp8": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "blockffn_chunk_forward_batch_fp8": (_I, [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P,
                                             _P, _P, _P, _I, _P, _S, _P]),
    "blockffn_batch_fp8_workspace_size": (_S, [_I, _I, _I, _I, _I]),
    "blockffn_layer_backward": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "blockffn_layer_backward_workspace_size": (_S, [_I, _I, _I, _I]),
    "blockffn_cls_losses": (_I, [_P, _I, _I, _I, _P, _P, _I, _F, _F, _F, _P, _P, _P, _P, _P, _P, _S, _P]),
    "blockffn_cls_losses_workspace_size": (_S, [_I, _I, _I, _I]),
    "blockffn_workspace_size": (_S, [_I, _I, _I, _I]),
    "blockffn_workspace_init": (_I, [_P, _S, _P]),
    "blockffn_device_status": (_I, [_P, _P]),
    "blockffn_status_string": (C.c_char_p, [_I]),
    "blockffn_abi_version": (_I, []),
}


class BlockFFNError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA extension first "
            "(python -c 'import __graft_entry__ as g; g.build()'); there is no fallback path")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


# ------------------------------------------------------------------- C entry points, same names
def blockffn_chunk_forward(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, stream):
    return _lib.blockffn_chunk_forward(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, stream)


def blockffn_chunk_forward_ex(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, tok_mask,
                              counts, r_out, flags, workspace, workspace_bytes, stream):
    return _lib.blockffn_chunk_forward_ex(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br,
                                          tok_mask, counts, r_out, flags, workspace, workspace_bytes,
                                          stream)


def blockffn_chunk_forward_batch(x, C, L, d, layer, n_layers, Wr, g, br, W1, W2, E, de, y, active_idx, n_active,
                                 counts, tok_mask, flags, workspace, workspace_bytes, stream):
    return _lib.blockffn_chunk_forward_batch(x, C, L, d, layer, n_layers, Wr, g, br, W1, W2, E, de, y, active_idx,
                                             n_active, counts, tok_mask, flags, workspace, workspace_bytes, stream)


def blockffn_union_overlap(active_idx_a, n_active_a, active_idx_b, n_active_b, C, E, overlap, stream):
    return _lib.blockffn_union_overlap(active_idx_a, n_active_a, active_idx_b, n_active_b, C, E, overlap, stream)


def blockffn_batch_workspace_size(C, L, d, E, de, flags):
    return _lib.blockffn_batch_workspace_size(C, L, d, E, de, flags)


def blockffn_chunk_forward_noalloc(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br, stream):
    return _lib.blockffn_chunk_forward_noalloc(x, L, d, Wr, g, W1, W2, E, de, y, active_idx, n_active, br,
                                               stream)


def blockffn_noalloc_device_status(stream):
    return _lib.blockffn_noalloc_device_status(stream)


NOALLOC_SCRATCH_BYTES = 8 << 20  # BFFN_NOALLOC_SCRATCH_BYTES in include/blockffn.h


def blockffn_quantize_fp8(W1, W2, n_layers, E, d, de, W1q, W2q, s1, s2, t2, stream):
    return _lib.blockffn_quantize_fp8(W1, W2, n_layers, E, d, de, W1q, W2q, s1, s2, t2, stream)


def blockffn_chunk_forward_batch_fp8(x, C, L, d, layer, n_layers, Wr, g, br, W1q, s1, W2q, s2, t2, E, de, y,
                                     active_idx, n_active, counts, tok_mask, flags, workspace, workspace_bytes,
                                     stream):
    return _lib.blockffn_chunk_forward_batch_fp8(x, C, L, d, layer, n_layers, Wr, g, br, W1q, s1, W2q, s2, t2, E,
                                                 de, y, active_idx, n_active, counts, tok_mask, flags, workspace,
                                                 workspace_bytes, stream)


def blockffn_batch_fp8_workspace_size(C, L, d, E, de):
    return _lib.blockffn_batch_fp8_workspace_size(C, L, d, E, de)


def blockffn_layer_backward(x, T, d, Wr, br, g, W1, W2, E, de, dy, dx, dWr, db, dg, dW1, dW2, workspace,
                            workspace_bytes, stream):
    return _lib.blockffn_layer_backward(x, T, d, Wr, br, g, W1, W2, E, de, dy, dx, dWr, db, dg, dW1, dW2, workspace,
                                        workspace_bytes, stream)


def blockffn_layer_backward_workspace_size(T, d, E, de):
    return _lib.blockffn_layer_backward_workspace_size(T, d, E, de)


def blockffn_cls_losses(x, C, L, d, Wr, br, E, alpha, w_al, w_cs, loss, dS, dWr, db, dx, workspace,
                        workspace_bytes, stream):
    return _lib.blockffn_cls_losses(x, C, L, d, Wr, br, E, alpha, w_al, w_cs, loss, dS, dWr, db, dx, workspace,
                                    workspace_bytes, stream)


def blockffn_cls_losses_workspace_size(C, L, d, E):
    return _lib.blockffn_cls_losses_workspace_size(C, L, d, E)


def blockffn_workspace_size(L, d, E, de):
    return _lib.blockffn_workspace_size(L, d, E, de)


def blockffn_workspace_init(workspace, workspace_bytes, stream):
    return _lib.blockffn_workspace_init(workspace, workspace_bytes, stream)


def blockffn_device_status(workspace, stream):
    return _lib.blockffn_device_status(workspace, stream)


def blockffn_status_string(status):
    return _lib.blockffn_status_string(status).decode()


def blockffn_abi_version():
    return _lib.blockffn_abi_version()


status_string = blockffn_status_string


# ------------------------------------------------------------------- torch-tensor marshalling
def _ptr(t):
    return None if t is None else t.data_ptr()


def _check(t, name, dtype, shape, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name}: want {dtype} {tuple(shape)} contiguous on {device}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def chunk_forward(x, Wr, g, W1, W2, y, active_idx, n_active, br=None, tok_mask=None, counts=None,
                  r_out=None, path=BFFN_PATH_AUTO, workspace=None, stream=None, flags=0):
    """One chunk: x bf16 [L,d], Wr fp32 [d,E], g fp32 [E], W1 bf16 [E,de,d], W2 bf16 [E,d,de];
    outputs y fp32 [L,d], active_idx int32 [E], n_active int32 [1] (+ optional tok_mask int32
    [L,ceil(E/32)] (bit patterns), counts int32 [2], r_out fp32 [L,E]).  `flags` adds BFFN_FLAG_* bits to the
    path.  Raises BlockFFNError."""
    import torch

    L, d = x.shape
    E, de = W1.shape[0], W1.shape[1]
    dev = x.device
    _check(x, "x", torch.bfloat16, (L, d), dev)
    _check(Wr, "Wr", torch.float32, (d, E), dev)
    _check(g, "g", torch.float32, (E,), dev)
    _check(W1, "W1", torch.bfloat16, (E, de, d), dev)
    _check(W2, "W2", torch.bfloat16, (E, d, de), dev)
    _check(y, "y", torch.float32, (L, d), dev)
    _check(active_idx, "active_idx", torch.int32, (E,), dev)
    _check(n_active, "n_active", torch.int32, (1,), dev)
    if br is not None:
        _check(br, "br", torch.float32, (E,), dev)
    if tok_mask is not None:
        _check(tok_mask, "tok_mask", torch.int32, (L, (E + 31) // 32), dev)
    if counts is not None:
        _check(counts, "counts", torch.int32, (2,), dev)
    if r_out is not None:
        _check(r_out, "r_out", torch.float32, (L, E), dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel() * workspace.element_size())
    rc = blockffn_chunk_forward_ex(_ptr(x), L, d, _ptr(Wr), _ptr(g), _ptr(W1), _ptr(W2), E, de, _ptr(y),
                                   _ptr(active_idx), _ptr(n_active), _ptr(br), _ptr(tok_mask),
                                   _ptr(counts), _ptr(r_out), int(path) | int(flags), ws_ptr, ws_bytes, stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_chunk_forward_ex")


def chunk_forward_batch(x, Wr, g, W1, W2, y, active_idx, n_active, layer=None, br=None, counts=None,
                        tok_mask=None, teams=0, workspace=None, stream=None, flags=0):
    """C independent chunks in one call: x bf16 [C,L,d]; stacked weights Wr fp32 [n_layers,d,E],
    g fp32 [n_layers,E], W1 bf16 [n_layers,E,de,d], W2 bf16 [n_layers,E,d,de] (br fp32 [n_layers,E]);
    layer int32 [C] (None: chunk c uses layer c % n_layers); outputs y fp32 [C,L,d], active_idx int32
    [C,E], n_active int32 [C] (+ counts int32 [C,2], tok_mask int32 [C,L,ceil(E/32)]).  teams = k of
    BFFN_FLAGS_SHARE (0: the default).  Raises BlockFFNError."""
    import torch

    C, L, d = x.shape
    nl, E, de = W1.shape[0], W1.shape[1], W1.shape[2]
    dev = x.device
    _check(x, "x", torch.bfloat16, (C, L, d), dev)
    _check(Wr, "Wr", torch.float32, (nl, d, E), dev)
    _check(g, "g", torch.float32, (nl, E), dev)
    _check(W1, "W1", torch.bfloat16, (nl, E, de, d), dev)
    _check(W2, "W2", torch.bfloat16, (nl, E, d, de), dev)
    _check(y, "y", torch.float32, (C, L, d), dev)
    _check(active_idx, "active_idx", torch.int32, (C, E), dev)
    _check(n_active, "n_active", torch.int32, (C,), dev)
    if layer is not None:
        _check(layer, "layer", torch.int32, (C,), dev)
    if br is not None:
        _check(br, "br", torch.float32, (nl, E), dev)
    if counts is not None:
        _check(counts, "counts", torch.int32, (C, 2), dev)
    if tok_mask is not None:
        _check(tok_mask, "tok_mask", torch.int32, (C, L, (E + 31) // 32), dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel() * workspace.element_size())
    rc = blockffn_chunk_forward_batch(_ptr(x), C, L, d, _ptr(layer), nl, _ptr(Wr), _ptr(g), _ptr(br), _ptr(W1),
                                      _ptr(W2), E, de, _ptr(y), _ptr(active_idx), _ptr(n_active), _ptr(counts),
                                      _ptr(tok_mask), BFFN_FLAGS_SHARE(teams) | int(flags), ws_ptr, ws_bytes, stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_chunk_forward_batch")


def new_batch_workspace(C, L, d, E, de, teams=0, device="cuda"):
    """A zero-filled caller-owned workspace for blockffn_chunk_forward_batch."""
    import torch

    n = blockffn_batch_workspace_size(C, L, d, E, de, BFFN_FLAGS_SHARE(teams))
    if n == 0:
        raise BlockFFNError(BFFN_EINVAL, "blockffn_batch_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def cls_losses(x, C, L, Wr, br=None, alpha=1.0, w_al=1.0, w_cs=1.0, loss=None, dS=None, dWr=None, db=None,
               dx=None, want_dWr=True, want_db=True, want_dx=True, workspace=None, stream=None):
    """The CLS-aware objectives over C chunks of L tokens (x bf16 [C*L, d], Wr fp32 [d, E], br fp32 [E])
    and the backward of J = w_al L_AL + w_cs L_CS through the router.  Returns (loss fp32 [2] = {L_AL,
    L_CS}, dS fp32 [C*L, E], dWr fp32 [d, E] or None, db fp32 [E] or None, dx fp32 [C*L, d] or None); the
    outputs are allocated unless given.  Raises BlockFFNError."""
    import torch

    T, d = x.shape
    E = Wr.shape[1]
    dev = x.device
    if T != C * L:
        raise ValueError(f"x has {T} rows, expected C * L = {C * L}")
    _check(x, "x", torch.bfloat16, (T, d), dev)
    _check(Wr, "Wr", torch.float32, (d, E), dev)
    if br is not None:
        _check(br, "br", torch.float32, (E,), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    loss = torch.empty(2, **f32) if loss is None else loss
    dS = torch.empty(T, E, **f32) if dS is None else dS
    dWr = (torch.empty(d, E, **f32) if want_dWr else None) if dWr is None else dWr
    db = (torch.empty(E, **f32) if want_db else None) if db is None else db
    dx = (torch.empty(T, d, **f32) if want_dx else None) if dx is None else dx
    _check(loss, "loss", torch.float32, (2,), dev)
    _check(dS, "dS", torch.float32, (T, E), dev)
    for t, name, shape in ((dWr, "dWr", (d, E)), (db, "db", (E,)), (dx, "dx", (T, d))):
        if t is not None:
            _check(t, name, torch.float32, shape, dev)
    need = blockffn_cls_losses_workspace_size(C, L, d, E)
    if need == 0:
        raise BlockFFNError(BFFN_EINVAL, "blockffn_cls_losses_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = blockffn_cls_losses(_ptr(x), C, L, d, _ptr(Wr), _ptr(br), E, float(alpha), float(w_al), float(w_cs),
                             _ptr(loss), _ptr(dS), _ptr(dWr), _ptr(db), _ptr(dx), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_cls_losses")
    return loss, dS, dWr, db, dx


def layer_backward(x, Wr, g, W1, W2, dy, br=None, workspace=None, stream=None):
    """The layer's backward: x bf16 [T, d], Wr fp32 [d, E], g fp32 [E], W1 bf16 [E, de, d], W2 bf16 [E, d, de],
    dy fp32 [T, d] (br fp32 [E] or None).  Returns a dict of fp32 tensors dx, dWr, db, dg, dW1, dW2.
    Raises BlockFFNError."""
    import torch

    T, d = x.shape
    E, de = W1.shape[0], W1.shape[1]
    dev = x.device
    _check(x, "x", torch.bfloat16, (T, d), dev)
    _check(Wr, "Wr", torch.float32, (d, E), dev)
    _check(g, "g", torch.float32, (E,), dev)
    _check(W1, "W1", torch.bfloat16, (E, de, d), dev)
    _check(W2, "W2", torch.bfloat16, (E, d, de), dev)
    _check(dy, "dy", torch.float32, (T, d), dev)
    if br is not None:
        _check(br, "br", torch.float32, (E,), dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty((T, d), **f32), "dWr": torch.empty((d, E), **f32), "db": torch.empty(E, **f32),
           "dg": torch.empty(E, **f32), "dW1": torch.empty((E, de, d), **f32), "dW2": torch.empty((E, d, de), **f32)}
    need = blockffn_layer_backward_workspace_size(T, d, E, de)
    if need == 0:
        raise BlockFFNError(BFFN_EINVAL, "blockffn_layer_backward_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = blockffn_layer_backward(_ptr(x), T, d, _ptr(Wr), _ptr(br), _ptr(g), _ptr(W1), _ptr(W2), E, de, _ptr(dy),
                                 *[_ptr(out[k]) for k in ("dx", "dWr", "db", "dg", "dW1", "dW2")],
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(), stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_layer_backward")
    return out


def quantize_fp8(W1, W2, n_layers, stream=None):
    """fp8 (e4m3) expert weights with power-of-two scales from bf16 W1 [n_layers*E, de, d] and W2
    [n_layers*E, d, de]: returns (W1q uint8, W2q uint8, s1 fp32 [NE, de], s2 fp32 [NE, de], t2 fp32
    [n_layers]).  Raises BlockFFNError."""
    import torch

    NE, de, d = W1.shape
    dev = W1.device
    _check(W1, "W1", torch.bfloat16, (NE, de, d), dev)
    _check(W2, "W2", torch.bfloat16, (NE, d, de), dev)
    if NE % n_layers != 0:
        raise ValueError("the expert count must be a multiple of n_layers")
    E = NE // n_layers
    W1q = torch.empty((NE, de, d), dtype=torch.uint8, device=dev)
    W2q = torch.empty((NE, d, de), dtype=torch.uint8, device=dev)
    s1 = torch.empty((NE, de), dtype=torch.float32, device=dev)
    s2 = torch.empty((NE, de), dtype=torch.float32, device=dev)
    t2 = torch.empty((n_layers,), dtype=torch.float32, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    rc = blockffn_quantize_fp8(_ptr(W1), _ptr(W2), n_layers, E, d, de, _ptr(W1q), _ptr(W2q), _ptr(s1), _ptr(s2),
                               _ptr(t2), stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_quantize_fp8")
    return W1q, W2q, s1, s2, t2


def chunk_forward_batch_fp8(x, Wr, g, q, y, active_idx, n_active, layer=None, br=None, counts=None, tok_mask=None,
                            workspace=None, stream=None, flags=0):
    """The batched decode forward on fp8 expert weights: q = (W1q, W2q, s1, s2, t2) from quantize_fp8; the
    other arguments as chunk_forward_batch.  Raises BlockFFNError."""
    import torch

    W1q, W2q, s1, s2, t2 = q
    C, L, d = x.shape
    nl = t2.shape[0]
    NE, de = s1.shape
    E = NE // nl
    dev = x.device
    _check(x, "x", torch.bfloat16, (C, L, d), dev)
    _check(Wr, "Wr", torch.float32, (nl, d, E), dev)
    _check(g, "g", torch.float32, (nl, E), dev)
    _check(W1q, "W1q", torch.uint8, (NE, de, d), dev)
    _check(W2q, "W2q", torch.uint8, (NE, d, de), dev)
    _check(s2, "s2", torch.float32, (NE, de), dev)
    _check(y, "y", torch.float32, (C, L, d), dev)
    _check(active_idx, "active_idx", torch.int32, (C, E), dev)
    _check(n_active, "n_active", torch.int32, (C,), dev)
    if layer is not None:
        _check(layer, "layer", torch.int32, (C,), dev)
    if br is not None:
        _check(br, "br", torch.float32, (nl, E), dev)
    if counts is not None:
        _check(counts, "counts", torch.int32, (C, 2), dev)
    if tok_mask is not None:
        _check(tok_mask, "tok_mask", torch.int32, (C, L, (E + 31) // 32), dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel() * workspace.element_size())
    rc = blockffn_chunk_forward_batch_fp8(_ptr(x), C, L, d, _ptr(layer), nl, _ptr(Wr), _ptr(g), _ptr(br), _ptr(W1q),
                                          _ptr(s1), _ptr(W2q), _ptr(s2), _ptr(t2), E, de, _ptr(y), _ptr(active_idx),
                                          _ptr(n_active), _ptr(counts), _ptr(tok_mask), int(flags), ws_ptr, ws_bytes,
                                          stream)
    if rc != BFFN_OK:
        raise BlockFFNError(rc, "blockffn_chunk_forward_batch_fp8")


def device_status(workspace=None, stream=None):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return blockffn_device_status(None if workspace is None else workspace.data_ptr(), stream)


def new_workspace(L, d, E, de, device="cuda"):
    """A zero-filled caller-owned workspace for blockffn_chunk_forward_ex."""
    import torch

    n = blockffn_workspace_size(L, d, E, de)
    if n == 0:
        raise BlockFFNError(BFFN_EINVAL, "blockffn_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)

"""ctypes wrapper of the fp64 CPU oracle of the BlockFFN chunk layer.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  The CUDA path never does.  ``build()`` compiles ``blockffn_oracle.cpp``
with the host C++ compiler into ``liboracle.so`` beside it; importing rebuilds it when the source is
newer than the library.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "blockffn_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O2, no fast-math: fp64 results follow IEEE rounding)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = C.CDLL(_LIB)
            p, i, dptr = C.c_void_p, C.c_int, C.c_void_p
            lib.oracle_set_mutation.argtypes = [i]
            lib.oracle_get_mutation.restype = i
            lib.oracle_swish.argtypes = [C.c_double]
            lib.oracle_swish.restype = C.c_double
            lib.oracle_router.argtypes = [p, i, i, p, p, p, i, i, dptr, dptr, p]
            lib.oracle_union.argtypes = [p, i, i, p, p, p, p]
            lib.oracle_expert.argtypes = [p, i, p, p, i, i, dptr]
            lib.oracle_chunk_forward.argtypes = [p, i, i, p, p, p, p, p, i, i, i, i, dptr, dptr, p]
            lib.oracle_tokens_forward_mt.argtypes = [p, i, i, p, p, p, p, p, i, i, i, i, i, dptr]
            lib.oracle_union_overlap.argtypes = [p, i, p, i, i, p]
            dbl = C.c_double
            lib.oracle_cls_losses.argtypes = [p, i, i, i, p, p, i, dbl, dbl, dbl, dptr, dptr, dptr, dptr, dptr]
            lib.oracle_cls_losses.restype = i
            lib.oracle_e4m3_value.argtypes = [i]
            lib.oracle_e4m3_value.restype = dbl
            lib.oracle_e4m3_nearest.argtypes = [dbl]
            lib.oracle_e4m3_nearest.restype = i
            lib.oracle_quantize_fp8.argtypes = [p, p, i, i, i, i, p, p, p, p, p]
            lib.oracle_quantize_fp8.restype = i
            lib.oracle_layer_backward.argtypes = [dptr, i, i, dptr, dptr, dptr, dptr, dptr, i, i, dptr, dptr, dptr,
                                                  dptr, dptr, dptr, dptr, dptr]
            lib.oracle_layer_backward.restype = i
            for f in ("oracle_router", "oracle_union", "oracle_expert", "oracle_chunk_forward",
                      "oracle_tokens_forward_mt", "oracle_union_overlap"):
                getattr(lib, f).restype = i
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def set_mutation(m: int) -> None:
    """Plant mistake number m in the oracle (0 restores the correct oracle). Tests only."""
    _load().oracle_set_mutation(int(m))


def swish(u: float) -> float:
    return float(_load().oracle_swish(float(u)))


# router normalisation: the RMS of the ReLU outputs (BlockFFN) or their sum (the ReMoE variant)
NORMS = {"rms": 0, "sum": 1}


def router(x, Wr, br, g, norm: str = "rms"):
    """x bf16 bits [L,d]; returns s fp64 [L,E], r fp64 [L,E], active bool [L,E]."""
    lib = _load()
    x = _c(x, np.uint16)
    Wr, g = _c(Wr, np.float32), _c(g, np.float32)
    br = _c(br, np.float32)
    L, d = x.shape
    E = Wr.shape[1]
    s = np.zeros((L, E)); r = np.zeros((L, E)); act = np.zeros((L, E), np.uint8)
    rc = lib.oracle_router(_ptr(x), L, d, _ptr(Wr), _ptr(br), _ptr(g), E, NORMS[norm], _ptr(s), _ptr(r), _ptr(act))
    assert rc == 0
    return s, r, act.astype(bool)


def union(active):
    """active bool [L,E] -> (active_idx int32 [n], tls_zero, cls_zero)."""
    lib = _load()
    act = np.ascontiguousarray(active, dtype=np.uint8)
    L, E = act.shape
    idx = np.zeros(E, np.int32); n = np.zeros(1, np.int32)
    tz = np.zeros(1, np.int64); cz = np.zeros(1, np.int64)
    rc = lib.oracle_union(_ptr(act), L, E, _ptr(idx), _ptr(n), _ptr(tz), _ptr(cz))
    assert rc == 0
    return idx[: n[0]].copy(), int(tz[0]), int(cz[0])


def union_overlap(a, b, E) -> int:
    """|a ∩ b| for two lists of expert indices (the reuse of one union by the next)."""
    lib = _load()
    a = np.ascontiguousarray(a, dtype=np.int32)
    b = np.ascontiguousarray(b, dtype=np.int32)
    out = np.zeros(1, np.int32)
    rc = lib.oracle_union_overlap(_ptr(a), a.size, _ptr(b), b.size, int(E), _ptr(out))
    assert rc == 0
    return int(out[0])


def cls_losses(x, C, L, Wr, br, alpha, w_al=1.0, w_cs=1.0):
    """The CLS-aware objectives over C chunks of L tokens (x bf16 bits [C*L, d]) and their backward through
    the router: returns (L_AL, L_CS, dS [C*L,E], dWr [d,E], db [E], dx [C*L,d]) for J = w_al L_AL + w_cs L_CS."""
    lib = _load()
    x = _c(x, np.uint16)
    Wr, br = _c(Wr, np.float32), _c(br, np.float32)
    T, d = x.shape
    E = Wr.shape[1]
    assert T == C * L
    loss = np.zeros(2); dS = np.zeros((T, E)); dWr = np.zeros((d, E)); db = np.zeros(E); dx = np.zeros((T, d))
    rc = lib.oracle_cls_losses(_ptr(x), int(C), int(L), d, _ptr(Wr), _ptr(br), E, float(alpha), float(w_al),
                               float(w_cs), _ptr(loss), _ptr(dS), _ptr(dWr), _ptr(db), _ptr(dx))
    assert rc == 0
    return loss[0], loss[1], dS, dWr, db, dx


def e4m3_value(code):
    return _load().oracle_e4m3_value(int(code))


def e4m3_nearest(v):
    return _load().oracle_e4m3_nearest(float(v))


def quantize_fp8(W1, W2, n_layers):
    """fp8 (e4m3) expert weights with power-of-two scales: W1 bf16 bits [n_layers*E, de, d] and W2 bf16 bits
    [n_layers*E, d, de] -> (q1 uint8, q2 uint8, s1 fp32 [NE, de], s2 fp32 [NE, de], t2 fp32 [n_layers])."""
    lib = _load()
    W1, W2 = _c(W1, np.uint16), _c(W2, np.uint16)
    NE, de, d = W1.shape
    assert W2.shape == (NE, d, de) and NE % n_layers == 0
    q1 = np.zeros(W1.shape, np.uint8); q2 = np.zeros(W2.shape, np.uint8)
    s1 = np.zeros((NE, de), np.float32); s2 = np.zeros((NE, de), np.float32); t2 = np.zeros(n_layers, np.float32)
    rc = lib.oracle_quantize_fp8(_ptr(W1), _ptr(W2), int(n_layers), NE // n_layers, d, de, _ptr(q1), _ptr(q2),
                                 _ptr(s1), _ptr(s2), _ptr(t2))
    assert rc == 0
    return q1, q2, s1, s2, t2


def dequantize_fp8(q1, q2, s1, s2, t2):
    """The weights the quantised format stands for, as bf16 bits (every one is exactly a bf16 value):
    W1 = s1 q1 (per row), W2 = t2[layer] s2 q2 (per column)."""
    table = np.array([e4m3_value(c) for c in range(256)], np.float64)
    NE = q1.shape[0]
    L = t2.shape[0]
    W1 = table[q1] * s1.astype(np.float64)[:, :, None]
    lay = np.repeat(np.arange(L), NE // L)
    W2 = table[q2] * (s2.astype(np.float64) * t2.astype(np.float64)[lay][:, None])[:, None, :]
    b1 = W1.astype(np.float32).view(np.uint32)
    b2 = W2.astype(np.float32).view(np.uint32)
    assert np.all(b1 & 0xFFFF == 0) and np.all(b2 & 0xFFFF == 0), "dequantised weights must be bf16-exact"
    return (b1 >> 16).astype(np.uint16), (b2 >> 16).astype(np.uint16)


def layer_backward(x, Wr, br, g, W1, W2, dy):
    """The layer's backward for upstream gradient dy, every argument fp64 (widen bf16 inputs first): x [T,d],
    Wr [d,E], br [E] or None, g [E], W1 [E,de,d], W2 [E,d,de], dy [T,d].  Returns a dict with y (the
    forward), dx, dWr, db, dg, dW1, dW2."""
    lib = _load()
    f = lambda a: None if a is None else np.ascontiguousarray(a, dtype=np.float64)
    x, Wr, br, g, W1, W2, dy = map(f, (x, Wr, br, g, W1, W2, dy))
    T, d = x.shape
    E, de = W1.shape[0], W1.shape[1]
    out = {"y": np.zeros((T, d)), "dx": np.zeros((T, d)), "dWr": np.zeros((d, E)), "db": np.zeros(E),
           "dg": np.zeros(E), "dW1": np.zeros((E, de, d)), "dW2": np.zeros((E, d, de))}
    rc = lib.oracle_layer_backward(_ptr(x), T, d, _ptr(Wr), _ptr(br), _ptr(g), _ptr(W1), _ptr(W2), E, de, _ptr(dy),
                                   *[_ptr(out[k]) for k in ("y", "dx", "dWr", "db", "dg", "dW1", "dW2")])
    assert rc == 0
    return out


def expert(xt, W1, W2, i):
    lib = _load()
    xt = _c(xt, np.uint16); W1 = _c(W1, np.uint16); W2 = _c(W2, np.uint16)
    E, de, d = W1.shape
    out = np.zeros(d)
    rc = lib.oracle_expert(_ptr(xt), d, _ptr(W1), _ptr(W2), de, int(i), _ptr(out))
    assert rc == 0
    return out


def chunk_forward(x, Wr, br, g, W1, W2, sparse: bool = False, norm: str = "rms"):
    """Full layer over one chunk -> (y fp64 [L,d], r fp64 [L,E], active bool [L,E])."""
    lib = _load()
    x = _c(x, np.uint16)
    Wr, g, br = _c(Wr, np.float32), _c(g, np.float32), _c(br, np.float32)
    W1, W2 = _c(W1, np.uint16), _c(W2, np.uint16)
    L, d = x.shape
    E, de, _ = W1.shape
    y = np.zeros((L, d)); r = np.zeros((L, E)); act = np.zeros((L, E), np.uint8)
    rc = lib.oracle_chunk_forward(_ptr(x), L, d, _ptr(Wr), _ptr(br), _ptr(g), _ptr(W1), _ptr(W2),
                                  E, de, int(bool(sparse)), NORMS[norm], _ptr(y), _ptr(r), _ptr(act))
    assert rc == 0
    return y, r, act.astype(bool)


def tokens_forward_mt(x, Wr, br, g, W1, W2, threads: int, sparse: bool = False, norm: str = "rms"):
    """Layer over n tokens [n,d] on `threads` host threads -> y fp64 [n,d]."""
    lib = _load()
    x = _c(x, np.uint16)
    Wr, g, br = _c(Wr, np.float32), _c(g, np.float32), _c(br, np.float32)
    W1, W2 = _c(W1, np.uint16), _c(W2, np.uint16)
    n, d = x.shape
    E, de, _ = W1.shape
    y = np.zeros((n, d))
    rc = lib.oracle_tokens_forward_mt(_ptr(x), n, d, _ptr(Wr), _ptr(br), _ptr(g), _ptr(W1),
                                      _ptr(W2), E, de, int(bool(sparse)), NORMS[norm], int(threads), _ptr(y))
    assert rc == 0
    return y


def chunk_reference(x, Wr, br, g, W1, W2, threads: int | None = None, norm: str = "rms"):
    """Everything a parity test compares for one chunk: y, r, active flags, union and counts.

    y is the dense evaluation (every expert computed and multiplied by its router weight, zero for
    the inactive ones), spread over the host's cores by token; the pins check that this threaded call
    equals the single-threaded chunk forward bit for bit."""
    _, r, act = router(x, Wr, br, g, norm=norm)
    y = tokens_forward_mt(x, Wr, br, g, W1, W2, threads or available_cores(), sparse=False, norm=norm)
    idx, tz, cz = union(act)
    return {"y": y, "r": r, "active": act, "active_idx": idx, "tls_zero": tz, "cls_zero": cz}


def available_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1

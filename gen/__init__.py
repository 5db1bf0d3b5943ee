"""Seeded synthetic workloads for the BlockFFN chunk layer.

This module produces INPUTS only: router weights, router bias, RMSNorm gain, expert weights and
token chunks, for both the CPU oracle and the CUDA path.  It holds none of the layer's arithmetic
beyond the one acceptance test the workload definition requires: a router pre-activation that lies
within ``margin`` of zero is resampled, so that the active set (ReLU output > 0) is well defined in
any floating-point precision.  That test is a plain fp64 matrix product on the bf16-rounded tokens.

Shapes and layouts (row-major, matching the layer's definition on the BlockFFN pages):
  x   bf16 bits (uint16) [n_chunks, L, d]
  Wr  fp32 [d, E]        N(0, 1/d)
  br  fp32 [E]           -beta * sigma_i, sigma_i = sqrt(var_x * ||Wr[:, i]||^2)  -> token-level
                         sparsity Phi(beta) per expert
  g   fp32 [E]           RMSNorm gain, 1
  W1  bf16 bits [E, de, d]   N(0, 1/d)
  W2  bf16 bits [E, d, de]   N(0, 1/de)

Chunk tokens are x_t = z_c + noise * n_t (z_c, n_t ~ N(0, I)) for correlated chunks, so
consecutive tokens share experts (the chunk-level sparsity the BlockFFN abstract reports), or
x_t = n_t i.i.d. for the prefill workload.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from statistics import NormalDist

import numpy as np

__all__ = [
    "f32_to_bf16_bits", "bf16_bits_to_f32", "Layer", "make_layer", "make_chunks",
    "expected_cls", "solve_noise_for_cls", "beta_for_tls", "Workload", "workload", "make_sequence_chunks",
    "WORKLOADS",
]

MARGIN = 1e-3


# ----------------------------------------------------------------------------- bf16 storage
def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the 16-bit patterns (no NaN input)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------- calibration
def beta_for_tls(tls: float) -> float:
    """Bias multiplier giving token-level sparsity `tls` (P(s <= 0) = Phi(beta))."""
    return NormalDist().inv_cdf(tls)


def expected_cls(noise: float, L: int, beta: float) -> float:
    """Expected chunk-level sparsity of the correlated generator.

    With u = z.w/||w|| and v_t = n_t.w/||w|| standard normal, expert i is inactive for token t iff
    u + noise*v_t < beta*sqrt(1+noise^2); inactive for the whole chunk with probability
    E_u[Phi((beta*sqrt(1+noise^2) - u)/noise)^L] (Gauss-Hermite quadrature over u).
    """
    nodes, weights = np.polynomial.hermite_e.hermegauss(240)
    weights = weights / weights.sum()
    thr = beta * math.sqrt(1.0 + noise * noise)
    nd = NormalDist()
    vals = np.array([nd.cdf((thr - u) / noise) for u in nodes]) ** L
    return float(np.sum(weights * vals))


def solve_noise_for_cls(tls: float, cls: float, L: int) -> float:
    """Noise coefficient giving chunk-level sparsity `cls` at token-level sparsity `tls` (bisection)."""
    beta = beta_for_tls(tls)
    lo, hi = 0.02, 3.0  # CLS decreases with noise
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        if expected_cls(mid, L, beta) > cls:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ----------------------------------------------------------------------------- generators
def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


@dataclass
class Layer:
    d: int
    E: int
    de: int
    Wr: np.ndarray
    br: np.ndarray
    g: np.ndarray
    W1: np.ndarray
    W2: np.ndarray
    beta: float
    var_x: float

    @property
    def expert_bytes(self) -> int:
        return 2 * self.d * self.de * 2


def make_layer(seed: int, d: int, E: int, de: int, beta: float, var_x: float,
               replica: int = 0, gain: float = 1.0) -> Layer:
    rng = _rng(seed, replica, 0x5EED01)
    Wr = (rng.standard_normal((d, E), dtype=np.float32) * np.float32(1.0 / math.sqrt(d)))
    sigma = np.sqrt(var_x * np.sum(Wr.astype(np.float64) ** 2, axis=0))
    br = (-beta * sigma).astype(np.float32)
    g = np.full(E, gain, dtype=np.float32)
    W1 = f32_to_bf16_bits(rng.standard_normal((E, de, d), dtype=np.float32)
                          * np.float32(1.0 / math.sqrt(d)))
    W2 = f32_to_bf16_bits(rng.standard_normal((E, d, de), dtype=np.float32)
                          * np.float32(1.0 / math.sqrt(de)))
    return Layer(d, E, de, Wr, br, g, W1, W2, beta, var_x)


def _pre_activation(xb: np.ndarray, layer: Layer) -> np.ndarray:
    # acceptance test only: fp64 product of the bf16-rounded tokens with the router weights
    return bf16_bits_to_f32(xb).astype(np.float64) @ layer.Wr.astype(np.float64) + layer.br


def make_chunks(seed: int, layer: Layer, n_chunks: int, L: int, noise: float | None,
                margin: float = MARGIN, stream: int = 0, block: int = 256) -> np.ndarray:
    """Token chunks as bf16 bits [n_chunks, L, d].

    noise=None draws every token i.i.d. N(0, I); otherwise x_t = z_c + noise*n_t.  A token with any
    |pre-activation| < margin gets a fresh noise draw (i.i.d.: a fresh token) until none is left.
    Draw order is fixed, so the result depends only on the arguments.
    """
    d = layer.d
    rng = _rng(seed, stream, 0xC4A9C5)
    out = np.empty((n_chunks, L, d), dtype=np.uint16)
    for c0 in range(0, n_chunks, block):
        nb = min(block, n_chunks - c0)
        if noise is None:
            z = np.zeros((nb, 1, d), dtype=np.float32)
            scale = np.float32(1.0)
        else:
            z = rng.standard_normal((nb, 1, d), dtype=np.float32)
            scale = np.float32(noise)
        n = rng.standard_normal((nb, L, d), dtype=np.float32)
        xb = f32_to_bf16_bits(z + scale * n)
        s = _pre_activation(xb.reshape(nb * L, d), layer)
        bad = np.flatnonzero(np.any(np.abs(s) < margin, axis=1))
        flat = xb.reshape(nb * L, d)
        while bad.size:
            fresh = rng.standard_normal((bad.size, d), dtype=np.float32)
            cand = f32_to_bf16_bits(z.reshape(nb, d)[bad // L] + scale * fresh)
            flat[bad] = cand
            s_b = _pre_activation(cand, layer)
            bad = bad[np.any(np.abs(s_b) < margin, axis=1)]
        out[c0:c0 + nb] = xb
    return out


def make_sequence_chunks(seed: int, layer: Layer, n_steps: int, L: int, noise: float, drift: float,
                         margin: float = MARGIN, stream: int = 0) -> np.ndarray:
    """Consecutive chunks of one sequence as bf16 bits [n_steps, L, d]: the chunk bases follow
    z_k = drift z_{k-1} + sqrt(1 - drift^2) e_k (z_0, e_k ~ N(0, I)), so consecutive chunks share experts
    more as drift -> 1; tokens are x_t = z_k + noise n_t.  The margin rule of make_chunks applies (a
    token within `margin` of a zero pre-activation gets a fresh noise draw)."""
    d = layer.d
    rng = _rng(seed, stream, 0x5E9C4A)
    out = np.empty((n_steps, L, d), dtype=np.uint16)
    z = rng.standard_normal(d, dtype=np.float32)
    keep = np.float32(drift)
    fresh_w = np.float32(math.sqrt(max(0.0, 1.0 - drift * drift)))
    for k in range(n_steps):
        if k > 0:
            z = keep * z + fresh_w * rng.standard_normal(d, dtype=np.float32)
        xb = f32_to_bf16_bits(z[None, :] + np.float32(noise) * rng.standard_normal((L, d), dtype=np.float32))
        bad = np.flatnonzero(np.any(np.abs(_pre_activation(xb, layer)) < margin, axis=1))
        while bad.size:
            cand = f32_to_bf16_bits(z[None, :] + np.float32(noise) * rng.standard_normal((bad.size, d),
                                                                                         dtype=np.float32))
            xb[bad] = cand
            bad = bad[np.any(np.abs(_pre_activation(cand, layer)) < margin, axis=1)]
        out[k] = xb
    return out


# ----------------------------------------------------------------------------- named workloads
@dataclass
class Workload:
    """One named workload: `layers` (one per weight replica) and chunks; chunk c uses layer
    c % len(layers).  Weight replicas stand for distinct layers of a stacked model: they keep the
    working set well above the 126 MB L2, so every chunk streams its experts from HBM."""
    name: str
    d: int
    E: int
    de: int
    L: int
    n_chunks: int
    tls: float
    noise: float | None
    seed: int = 0
    replicas: int = 1
    beta: float = field(init=False)

    def __post_init__(self):
        self.beta = beta_for_tls(self.tls) if self.tls is not None else 0.8

    @property
    def var_x(self) -> float:
        return 1.0 if self.noise is None else 1.0 + self.noise ** 2

    def layer(self, replica: int = 0) -> Layer:
        return make_layer(self.seed, self.d, self.E, self.de, self.beta, self.var_x, replica)

    def chunks(self, layer: Layer, n_chunks: int, replica: int = 0) -> np.ndarray:
        return make_chunks(self.seed, layer, n_chunks, self.L, self.noise, stream=replica)

    def describe(self) -> dict:
        return {"workload": self.name, "d": self.d, "E": self.E, "de": self.de, "L": self.L,
                "chunks": self.n_chunks, "tls_target": self.tls, "noise": self.noise,
                "weight_replicas": self.replicas, "seed": self.seed}


def _tiny(seed=0, **kw):
    w = Workload("tiny_d256_E16_de64_L8", 256, 16, 64, 8, 64, None, 0.3, seed, 1)
    w.beta = 0.8  # bias -0.8 sigma: ~79% of router entries <= 0
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def _decode_1b(seed=0, **kw):
    noise = solve_noise_for_cls(0.85, 0.70, 8)
    w = Workload("decode_d2048_E64_de256_L8", 2048, 64, 256, 8, 4096, 0.85, noise, seed, 16)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def _lsweep(L=8, seed=0, **kw):
    w = Workload(f"lsweep_d4096_E128_de256_L{L}", 4096, 128, 256, L, 1024, 0.85, 0.3, seed, 8)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def _tls_sweep(tls=0.85, seed=0, **kw):
    w = Workload(f"tlssweep_d4096_E128_de256_L8_tls{int(round(tls * 100))}", 4096, 128, 256, 8,
                 256, tls, 0.3, seed, 32)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def _prefill(seed=0, **kw):
    w = Workload("prefill_d4096_E128_de256_L4096", 4096, 128, 256, 4096, 1, 0.85, None, seed, 1)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


WORKLOADS = {"tiny": _tiny, "decode": _decode_1b, "lsweep": _lsweep, "tls_sweep": _tls_sweep,
             "prefill": _prefill}


def workload(name: str, **kw) -> Workload:
    return WORKLOADS[name](**kw)

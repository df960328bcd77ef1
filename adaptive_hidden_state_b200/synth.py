"""Seeded synthetic workloads for the SPA-Cache layer step and decode loop.

This module only *draws* inputs: weights, hidden states, token sequences and
the positions a decode step unmasks.  It holds none of the method's
arithmetic (no projection, similarity, selection, attention or FFN), so the
CUDA path and the CPU oracle can both be fed from it without sharing any
computation.  Everything is numpy on the host; values meant for bf16 configs
are rounded to bf16 here so that both sides start from the same bits.

Workload recipes follow the shapes the SPA-Cache pages report (LLaDA-8B:
d=4096, 32 heads x 128, SwiGLU 12288, vocab 126464, r=128) with random
weights, since trained weights and benchmark datasets are not available.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "LayerShape", "LLADA_LAYER", "TINY_LAYER", "bf16_round", "bf16_bits",
    "haar_orthogonal", "power_law_wv", "layer_weights", "hidden_states",
    "drift_rows", "graded_drift", "DecodeInputs", "decode_inputs",
]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d: int
    n_heads: int
    head_dim: int
    ffn: int
    r: int
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0


# LLaDA-8B-like layer (the pages' model, random weights).
LLADA_LAYER = LayerShape(d=4096, n_heads=32, head_dim=128, ffn=12288, r=128)
# The tiny fp32 model used for full decode-loop parity.
TINY_LAYER = LayerShape(d=256, n_heads=4, head_dim=64, ffn=688, r=16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of bf16-representable float32 values, as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def haar_orthogonal(d: int, rng: np.random.Generator) -> np.ndarray:
    """A Haar-distributed random orthogonal d x d matrix (QR of a Gaussian,
    column signs fixed by the diagonal of R)."""
    g = rng.standard_normal((d, d))
    q, rr = np.linalg.qr(g)
    q *= np.sign(np.diag(rr))[None, :]
    return q


def power_law_wv(d: int, rng: np.random.Generator, exponent: float = 0.8,
                 spectrum: np.ndarray | None = None):
    """W_v = U diag(sigma) V^T with sigma_i = i^-exponent (1-based) unless a
    spectrum is given.  Returns (W_v, U, sigma, V) in float64."""
    u = haar_orthogonal(d, rng)
    v = haar_orthogonal(d, rng)
    if spectrum is None:
        sigma = np.arange(1, d + 1, dtype=np.float64) ** (-exponent)
    else:
        sigma = np.asarray(spectrum, dtype=np.float64)
    return (u * sigma[None, :]) @ v.T, u, sigma, v


def layer_weights(shape: LayerShape, seed: int, bf16: bool, std: float = 0.02,
                  wv_exponent: float = 0.8) -> dict:
    """One transformer layer's weights, stored [out, in] row-major (float32).

    W_q, W_k, W_o, W_gate, W_up, W_down ~ N(0, std^2); W_v has power-law
    singular values.  Norm gains are ones.  With bf16=True every matrix is
    rounded to bf16 values.  The exact SVD factors of W_v (before rounding)
    are returned as ``wv_sigma`` / ``wv_V`` for workloads that want to hand a
    precomputed proxy to the library instead of running its host SVD.
    """
    rng = np.random.default_rng(seed)
    d, f = shape.d, shape.ffn
    w = {}
    w["wq"] = rng.standard_normal((d, d)) * std
    w["wk"] = rng.standard_normal((d, d)) * std
    wv, _, sigma, v = power_law_wv(d, rng, wv_exponent)
    w["wv"] = wv
    w["wo"] = rng.standard_normal((d, d)) * std
    w["w_gate"] = rng.standard_normal((f, d)) * std
    w["w_up"] = rng.standard_normal((f, d)) * std
    w["w_down"] = rng.standard_normal((d, f)) * std
    rnd = bf16_round if bf16 else (lambda a: a)
    out = {k: rnd(np.asarray(a, dtype=np.float32)) for k, a in w.items()}
    out["attn_norm"] = np.ones(d, dtype=np.float32)
    out["ffn_norm"] = np.ones(d, dtype=np.float32)
    out["wv_sigma"] = sigma
    out["wv_V"] = v
    return out


def hidden_states(B: int, N: int, d: int, seed: int, bf16: bool) -> np.ndarray:
    """Layer inputs H ~ N(0, 1), shape [B, N, d], float32."""
    h = np.random.default_rng(seed).standard_normal((B, N, d)).astype(np.float32)
    return bf16_round(h) if bf16 else h


def drift_rows(H: np.ndarray, frac: float, std: float, seed: int, bf16: bool):
    """Perturb round(frac*N) rows of every sequence by N(0, std^2) noise.
    Returns (H', rows) where rows[b] is the sorted array of perturbed rows."""
    rng = np.random.default_rng(seed)
    B, N, d = H.shape
    n_rows = int(round(frac * N))
    out = H.copy()
    rows = []
    for b in range(B):
        rb = np.sort(rng.choice(N, size=n_rows, replace=False))
        out[b, rb] = H[b, rb] + (rng.standard_normal((n_rows, d)) * std).astype(np.float32)
        rows.append(rb)
    return (bf16_round(out) if bf16 else out), rows


def graded_drift(H: np.ndarray, lo: float, hi: float, seed: int, bf16: bool):
    """Every row drifts: H'_i = H_i + eps_i * g_i, eps_i ~ U[lo, hi], g_i ~ N(0, I)."""
    rng = np.random.default_rng(seed)
    B, N, d = H.shape
    eps = rng.uniform(lo, hi, size=(B, N, 1))
    out = (H + eps * rng.standard_normal((B, N, d))).astype(np.float32)
    return bf16_round(out) if bf16 else out


@dataclasses.dataclass
class DecodeInputs:
    tokens: np.ndarray          # [B, N] int64 initial ids (mask id at masked rows)
    mask_id: int
    positions: list             # per step: [B, u] int64 positions unmasked that step
    forced: list                # per step: [B, u] int64 forced token ids


def decode_inputs(B: int, N: int, n_prompt: int, vocab: int, steps: int, u: int,
                  seed: int) -> DecodeInputs:
    """A masked-diffusion decoding job: n_prompt uniform prompt ids then masks
    (mask id = vocab - 1).  For each step, u positions drawn uniformly without
    replacement from the still-masked ones (rng seeded with seed + step), and
    u forced token ids for teacher-forced parity runs."""
    rng0 = np.random.default_rng(seed)
    mask_id = vocab - 1
    tokens = np.full((B, N), mask_id, dtype=np.int64)
    tokens[:, :n_prompt] = rng0.integers(0, vocab - 1, size=(B, n_prompt))
    masked = [set(range(n_prompt, N)) for _ in range(B)]
    positions, forced = [], []
    for t in range(steps):
        rng = np.random.default_rng(seed + 1 + t)
        pos = np.zeros((B, u), dtype=np.int64)
        for b in range(B):
            pool = np.array(sorted(masked[b]), dtype=np.int64)
            pick = np.sort(rng.choice(pool, size=u, replace=False))
            pos[b] = pick
            masked[b].difference_update(pick.tolist())
        positions.append(pos)
        forced.append(rng.integers(0, vocab - 1, size=(B, u)).astype(np.int64))
    return DecodeInputs(tokens=tokens, mask_id=mask_id, positions=positions, forced=forced)

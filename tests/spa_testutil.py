"""Helpers shared by the GPU parity tests: build a layer on both sides from
the same seeded weights, move tensors, and compare with the stated
tolerances (fp32 configs: max|a-b| / max|b| <= 1e-3; bf16 configs:
|a-b|_2 / |b|_2 <= 2e-2; index sets bit-exact given a 1e-4 score margin)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth

TOL_F32 = 1e-3
TOL_BF16 = 2e-2
MARGIN = 1e-4
NAMES = ["wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "attn_norm", "ffn_norm"]


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def max_rel(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    mb = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (mb if mb > 0 else 1.0))


def assert_close(got, ref, bf16: bool, what: str):
    got = np64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite values"
    if bf16:
        e = rel_l2(got, ref)
        assert e <= TOL_BF16, f"{what}: rel-L2 {e:.3e} > {TOL_BF16}"
    else:
        e = max_rel(got, ref)
        assert e <= TOL_F32, f"{what}: max-rel {e:.3e} > {TOL_F32}"
    return e


def assert_index_set(got_I: np.ndarray, s_oracle: np.ndarray, k: int, ref_I: np.ndarray,
                     what: str = "I"):
    """Bit-exact when the k-th/(k+1)-th oracle scores are >= MARGIN apart or
    tie exactly (exact zeros of unchanged rows); otherwise any set that a
    MARGIN-perturbation of the scores could produce is accepted."""
    got_I = np.asarray(got_I, np.int64)
    N = s_oracle.shape[0]
    assert got_I.shape == (k,)
    assert np.all(np.diff(got_I) > 0), what + ": not strictly ascending"
    assert got_I.min() >= 0 and got_I.max() < N
    srt = np.sort(s_oracle)[::-1]
    kth = srt[k - 1]
    nxt = srt[k] if k < N else -np.inf
    if k == N or kth - nxt >= MARGIN or (kth == 0.0 and nxt == 0.0):
        assert np.array_equal(got_I, ref_I), f"{what}: index set differs from the oracle"
    else:
        sel = np.zeros(N, bool)
        sel[got_I] = True
        assert np.all(s_oracle[sel] >= kth - MARGIN), what
        assert np.all(s_oracle[~sel] <= kth + MARGIN), what


def layer_desc(spa, shape: synth.LayerShape, dtype: int):
    return spa.LayerDesc(d=shape.d, n_heads=shape.n_heads, head_dim=shape.head_dim,
                         ffn=shape.ffn, r=shape.r, dtype=dtype, rms_eps=shape.rms_eps,
                         rope_theta=shape.rope_theta)


class LayerPair:
    """One layer on both sides: the library handle (proxy from its own host
    SVD unless given) and the oracle layer (proxy from numpy's SVD, rounded to
    bf16 for bf16 configs)."""

    def __init__(self, spa, shape, seed, dtype, max_B, max_N, w=None, ws=None, std=0.02):
        self.spa, self.shape, self.dtype = spa, shape, dtype
        self.bf16 = dtype == spa.SPA_BF16
        self.w = w if w is not None else synth.layer_weights(shape, seed, bf16=self.bf16, std=std)
        tdt = spa.torch_dtype(dtype)
        self.dev = {k: torch.from_numpy(np.ascontiguousarray(self.w[k])).to("cuda", tdt)
                    for k in NAMES}
        self.desc = layer_desc(spa, shape, dtype)
        self.ws = ws if ws is not None else spa.Workspace(self.desc, max_B, max_N)
        self.layer = spa.Layer(self.desc, self.dev, self.ws, w_r_host=None)
        W_r = O.singular_proxy(self.w["wv"], shape.r)
        if self.bf16:
            W_r = O.round_bf16(W_r)
        self.W_r = W_r
        self.ol = O.OracleLayer.from_weights(self.w, W_r, shape.n_heads, shape.rms_eps,
                                             shape.rope_theta)

    def cache(self, B, N):
        return self.spa.Cache(B, N, self.shape.d, self.shape.r, self.dtype)

    def to_dev(self, H: np.ndarray) -> torch.Tensor:
        return torch.from_numpy(np.ascontiguousarray(H)).to("cuda", self.spa.torch_dtype(self.dtype))


def snapshot_cache(c) -> list:
    """Device copies of one layer cache's K^c, V^c, H^c, P^c."""
    return [t.clone() for t in (c.k, c.v, c.h, c.p)]


def check_layer_step(spa, layer, w: dict, H_in, snap, cache, k, idx, ws, seqs, what):
    """A cached layer step the GPU has just run, checked for the sequences in
    `seqs` against the oracle on the same inputs: H_in (device copy of the
    step's input), snap (snapshot_cache before the step), the layer's weights
    w (device tensors) and its stored proxy.  Index set (exact or valid within
    the score margin), Q, O, H1, A, the rewritten K^c/V^c/H^c/P^c rows, and the
    other rows bit-identical to the snapshot."""
    host = {n: w[n].float().cpu().numpy() for n in NAMES}
    d, F, nh = layer.desc.d, layer.desc.ffn, layer.desc.n_heads
    W_r = layer.proxy_weights().numpy().astype(np.float64)
    ol = O.OracleLayer.from_weights(host, W_r, nh, layer.desc.rms_eps, layer.desc.rope_theta)
    B = H_in.shape[0]
    M = B * k
    views = {name: ws.view(name, (M, width), torch.bfloat16).clone()
             for name, width in (("q", d), ("o", d), ("h1", d), ("a", F))}
    I_all = idx.cpu().numpy()
    after = [np64(t) for t in (cache.k, cache.v, cache.h)]
    p_after = np64(cache.p)
    before = [np64(t) for t in snap[:3]]
    p_before = np64(snap[3])
    for b in seqs:
        Hb = np64(H_in[b])
        cache_b = O.LayerCache(before[0][b].copy(), before[1][b].copy(), before[2][b].copy(),
                               p_before[b].copy())
        a_hat, s = O.proxy_identify(Hb, ol.W_r, cache_b.P_c)
        I_ref = O.select_topk(s, k)
        I = I_all[b].astype(np.int64)
        assert_index_set(I, s, k, I_ref, f"{what} seq {b} I")
        cache_b.P_c[I] = a_hat[I]
        out = O.partial_block(ol, Hb, I, cache_b)
        rows = slice(b * k, (b + 1) * k)
        for name, key in (("q", "Q"), ("o", "O"), ("h1", "H1"), ("a", "A")):
            assert_close(views[name][rows], out[key], True, f"{what} seq {b} {key}")
        for j, (name, ref) in enumerate((("K^c", cache_b.K_c), ("V^c", cache_b.V_c), ("H^c", cache_b.H_c))):
            assert_close(after[j][b][I], ref[I], True, f"{what} seq {b} {name}[I]")
            keep = np.ones(after[j].shape[1], bool)
            keep[I] = False
            assert np.array_equal(after[j][b][keep], before[j][b][keep]), f"{what} seq {b} {name} outside I"
        assert np.max(np.abs(p_after[b][I] - cache_b.P_c[I])) < 2e-3, f"{what} seq {b} P^c[I]"

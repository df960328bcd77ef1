"""Plain CPU oracle of the SPA-Cache cached transformer-block update.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the library.  It shares no
code with the CUDA path.  Everything is float64 numpy, written for a reader to
check against the pages by eye: one function per step, in the pages' order and
notation, no blocking, fusion or reordering.

Sources, cited by tag in every docstring:

[GIST]  gist.science, "SPA-Cache: Singular Proxies for Adaptive Caching in
        Diffusion Language Models", Technical Summary: Problem Statement;
        Methodology: SPA-Cache, items 1 (Update Identification via Singular
        Proxies), 2 (Adaptive Budget Allocation), 3 (Sparse Execution).
[NOTES] papernotes.org (ICML 2026), "SPA-Cache: Singular Proxies for Adaptive
        Caching in Diffusion Language Models": 方法详解 > 整体框架 (the three
        phases of Algorithm 1); 关键设计 2 (singular proxy W_r = Λ_r V_rᵀ,
        f_proxy(h_i) = W_r h_i, Theorem 3.4); 关键设计 3 (piecewise-Gaussian
        budget ρ(l)); 研究背景与动机 (vanilla DLM decoding runs a full forward
        of all N positions at every step).

Readings where the pages are silent are tagged "reading A<n>"; the list with
reasons is kept in the repository's design notes.  Pins: every function here
is checked by ``tests/test_oracle_pins.py`` against closed forms, invariants,
library routines or brute force.  The decode loop beyond those invariants is
"parity unpinned" (the pages print no worked numbers for it).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "rho", "budget_k", "budget_table", "singular_proxy", "round_bf16",
    "truncation_bound", "proxy_identify", "select_topk", "rmsnorm", "rope",
    "attention", "swiglu_ffn", "OracleLayer", "LayerCache", "empty_cache",
    "phase2_attention", "phase3_ffn_scatter", "partial_block", "layer_step",
    "full_block", "vanilla_block", "attn_output_identify", "attn_output_layer_step",
    "attn_output_fill", "OracleModel", "DecodeState",
    "init_decode_state", "decode_step", "lm_head_argmax", "confidence", "confident_positions",
]


# ---------------------------------------------------------------------------
# Budget: piecewise-Gaussian ρ(l) and k = ⌈Nρ⌉
# ---------------------------------------------------------------------------

def rho(l: int, L: int, rho_p: float, l_p: int, rho_1: float, rho_L: float) -> float:
    """Update ratio of layer l (1-based, reading A2) [NOTES 关键设计 3; GIST item 2].

    For l <= l_p:  ρ_p · exp( ln(ρ_1/ρ_p) · ((l − l_p)/(l_p − 1))² )
    For l >  l_p:  ρ_p · exp( ln(ρ_L/ρ_p) · ((l − l_p)/(L − l_p))² )

    The pages write the l > l_p branch only as "the symmetric branch"; the
    form above is the one that meets ρ(L) = ρ_L (reading A1).  With l_p = 1
    the left branch is the single point ρ(1) = ρ_p.
    """
    if not (1 <= l <= L and 1 <= l_p <= L):
        raise ValueError("layer index out of range")
    if not (rho_p > 0 and rho_1 > 0 and rho_L > 0):
        raise ValueError("budgets must be positive")
    if l <= l_p:
        if l_p == 1:
            return rho_p
        t = (l - l_p) / (l_p - 1)
        return rho_p * math.exp(math.log(rho_1 / rho_p) * t * t)
    t = (l - l_p) / (L - l_p)
    return rho_p * math.exp(math.log(rho_L / rho_p) * t * t)


def budget_k(N: int, ratio: float) -> int:
    """Tokens refreshed in a layer: k = ⌈N·ρ⌉, clamped to [1, N]
    [NOTES 整体框架, Phase 1: "k = Nρ"; reading A3]."""
    if N < 1:
        raise ValueError("N must be positive")
    return min(N, max(1, math.ceil(N * ratio)))


def budget_table(N: int, L: int, rho_p: float, l_p: int, rho_1: float, rho_L: float):
    """[k_1, ..., k_L] for a sequence of N tokens."""
    return [budget_k(N, rho(l, L, rho_p, l_p, rho_1, rho_L)) for l in range(1, L + 1)]


# ---------------------------------------------------------------------------
# Phase 1: singular proxy, drift score, top-k
# ---------------------------------------------------------------------------

def singular_proxy(W_v: np.ndarray, r: int) -> np.ndarray:
    """W_r = Λ_r V_rᵀ (r × d) from the SVD W_v ≈ U Λ Vᵀ [NOTES 关键设计 2;
    GIST item 1, "Dimensionality Reduction"].

    W_v is stored [out, in] so that v_i = W_v h_i; its right singular vectors
    live in the input space.  Each row's sign is fixed so that its entry of
    largest magnitude (lowest index on ties) is positive (reading A13; the
    drift score does not depend on row signs).
    """
    W_v = np.asarray(W_v, dtype=np.float64)
    if not (1 <= r <= min(W_v.shape)):
        raise ValueError("rank out of range")
    _, lam, Vt = np.linalg.svd(W_v)
    W_r = lam[:r, None] * Vt[:r, :]
    for i in range(r):
        j = int(np.argmax(np.abs(W_r[i])))
        if W_r[i, j] < 0:
            W_r[i] = -W_r[i]
    return W_r


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even) via torch's CPU conversion; the
    bf16 configs store W_r and every activation in this format (reading A18)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)


def truncation_bound(lam: np.ndarray, r: int) -> float:
    """Theorem 3.4's bound on the cosine error of the rank-r proxy:
    2 (λ_{r+1} / λ_r)² [NOTES 关键设计 2].  lam is sorted descending."""
    return 2.0 * (lam[r] / lam[r - 1]) ** 2


def proxy_identify(H: np.ndarray, W_r: np.ndarray, P_c: np.ndarray):
    """Drift score of every token against its cached proxy [NOTES 整体框架,
    Phase 1; GIST item 1, "Mechanism"].

    a_i = W_r h_i on the raw layer input (reading A4), â_i = a_i / ‖a_i‖
    (â_i = 0 when ‖a_i‖ = 0), and s_i = ½‖â_i − P^c_i‖², which equals
    1 − cos(a_i, cached) when P^c holds unit vectors (reading A6).
    H: [N, d]; W_r: [r, d]; P_c: [N, r].  Returns (â [N, r], s [N]).
    """
    H = np.asarray(H, dtype=np.float64)
    a = H @ np.asarray(W_r, dtype=np.float64).T
    norm = np.sqrt(np.sum(a * a, axis=1))
    a_hat = np.zeros_like(a)
    nz = norm > 0
    a_hat[nz] = a[nz] / norm[nz, None]
    diff = a_hat - np.asarray(P_c, dtype=np.float64)
    s = 0.5 * np.sum(diff * diff, axis=1)
    return a_hat, s


def select_topk(s: np.ndarray, k: int) -> np.ndarray:
    """Index set I of the k least-similar (largest-s) tokens, ties to the
    lowest index, emitted ascending [NOTES 整体框架, Phase 1; reading A7]."""
    s = np.asarray(s)
    N = s.shape[0]
    if not (0 <= k <= N):
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(N), -s))   # primary: -s, secondary: index
    return np.sort(order[:k]).astype(np.int64)


# ---------------------------------------------------------------------------
# Block pieces (pre-norm LLaMA-style block: reading A10)
# ---------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x²) + eps) · γ over the last axis (reading A12)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half pairing (i, i + d_h/2),
    frequency θ^(−2i/d_h) (reading A11).  x: [n, heads, d_h]; pos: [n]."""
    n, heads, dh = x.shape
    half = dh // 2
    inv_freq = theta ** (-(2.0 * np.arange(half)) / dh)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Bidirectional softmax attention of sparse queries against every cached
    key, per head: softmax(Q Kᵀ/√d_h) V, no mask [NOTES 整体框架, Phase 2;
    GIST item 3].  Q: [k, heads, d_h]; K, V: [N, heads, d_h].  Returns
    [k, heads·d_h]."""
    k, heads, dh = Q.shape
    out = np.zeros((k, heads, dh))
    for h in range(heads):
        S = Q[:, h, :] @ K[:, h, :].T / math.sqrt(dh)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ V[:, h, :]
    return out.reshape(k, heads * dh)


def swiglu_ffn(x: np.ndarray, w_gate, w_up, w_down):
    """SwiGLU FFN: W_down (silu(W_gate x) ⊙ W_up x).  Returns (output, A)
    where A is the gated activation [n, F]."""
    g = x @ w_gate.T
    u = x @ w_up.T
    A = g / (1.0 + np.exp(-g)) * u
    return A @ w_down.T, A


# ---------------------------------------------------------------------------
# One layer, one sequence
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class OracleLayer:
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wo: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    attn_norm: np.ndarray
    ffn_norm: np.ndarray
    W_r: np.ndarray
    n_heads: int
    eps: float = 1e-5
    theta: float = 10000.0

    @property
    def d(self):
        return self.wq.shape[1]

    @property
    def head_dim(self):
        return self.d // self.n_heads

    @staticmethod
    def from_weights(w: dict, W_r: np.ndarray, n_heads: int, eps: float = 1e-5,
                     theta: float = 10000.0) -> "OracleLayer":
        f = lambda a: np.asarray(a, dtype=np.float64)
        return OracleLayer(f(w["wq"]), f(w["wk"]), f(w["wv"]), f(w["wo"]),
                           f(w["w_gate"]), f(w["w_up"]), f(w["w_down"]),
                           f(w["attn_norm"]), f(w["ffn_norm"]), f(W_r),
                           n_heads, eps, theta)


@dataclasses.dataclass
class LayerCache:
    """Caches of one layer and one sequence [NOTES 整体框架]: post-RoPE keys
    K^c and values V^c [N, d], layer outputs H^c [N, d], unit proxies P^c [N, r]."""
    K_c: np.ndarray
    V_c: np.ndarray
    H_c: np.ndarray
    P_c: np.ndarray

    def copy(self) -> "LayerCache":
        return LayerCache(self.K_c.copy(), self.V_c.copy(), self.H_c.copy(), self.P_c.copy())


def empty_cache(N: int, d: int, r: int) -> LayerCache:
    return LayerCache(np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, d)), np.zeros((N, r)))


def phase2_attention(layer: OracleLayer, H: np.ndarray, I: np.ndarray, cache: LayerCache):
    """Partial cached attention [NOTES 整体框架, Phase 2; GIST item 3].

    x = RMSNorm(H[I]); Q_I, K_I, V_I = x W_{q,k,v}ᵀ; RoPE on Q_I and K_I at
    positions I; K^c[I] ← K_I, V^c[I] ← V_I (before attending: reading A9);
    O_I = softmax(Q_I K^cᵀ/√d_h) V^c over all N rows.  Updates the cache in
    place; returns (Q_I, O_I) with Q_I shaped [k, d]."""
    hd, nh = layer.head_dim, layer.n_heads
    x = rmsnorm(H[I], layer.attn_norm, layer.eps)
    Q = rope((x @ layer.wq.T).reshape(len(I), nh, hd), I, layer.theta)
    K = rope((x @ layer.wk.T).reshape(len(I), nh, hd), I, layer.theta)
    V = x @ layer.wv.T
    cache.K_c[I] = K.reshape(len(I), -1)
    cache.V_c[I] = V
    N = cache.K_c.shape[0]
    O = attention(Q, cache.K_c.reshape(N, nh, hd), cache.V_c.reshape(N, nh, hd))
    return Q.reshape(len(I), -1), O


def phase3_ffn_scatter(layer: OracleLayer, H: np.ndarray, I: np.ndarray, O: np.ndarray,
                       cache: LayerCache):
    """FFN on the selected rows and scatter into H^c [NOTES 整体框架, Phase 3;
    GIST item 3]: H1 = H[I] + O_I W_oᵀ; H^c[I] = H1 + FFN(RMSNorm(H1)).
    Unselected rows of H^c are left as cached.  Returns (H1, A)."""
    H1 = H[I] + O @ layer.wo.T
    f, A = swiglu_ffn(rmsnorm(H1, layer.ffn_norm, layer.eps), layer.w_gate, layer.w_up,
                      layer.w_down)
    cache.H_c[I] = H1 + f
    return H1, A


def partial_block(layer: OracleLayer, H: np.ndarray, I: np.ndarray, cache: LayerCache) -> dict:
    """Phases 2 and 3 for a given index set (cache updated in place)."""
    H = np.asarray(H, dtype=np.float64)
    I = np.asarray(I, dtype=np.int64)
    Q, O = phase2_attention(layer, H, I, cache)
    H1, A = phase3_ffn_scatter(layer, H, I, O, cache)
    return {"Q": Q, "O": O, "H1": H1, "A": A}


def layer_step(layer: OracleLayer, H: np.ndarray, cache: LayerCache, k: int) -> dict:
    """One cached layer step, Algorithm 1's three phases in order [NOTES
    整体框架]: score against P^c, select I, P^c[I] ← â[I] (reading A5), then
    partial attention and FFN.  Cache updated in place."""
    H = np.asarray(H, dtype=np.float64)
    a_hat, s = proxy_identify(H, layer.W_r, cache.P_c)
    I = select_topk(s, k)
    cache.P_c[I] = a_hat[I]
    out = partial_block(layer, H, I, cache)
    out.update({"I": I, "s": s, "a_hat": a_hat})
    return out


def full_block(layer: OracleLayer, H: np.ndarray, r: int | None = None) -> tuple:
    """ρ = 1 pass that fills every cache (reading A8: the decode loop starts
    with it): every row is selected and P^c holds â of every row."""
    H = np.asarray(H, dtype=np.float64)
    N, d = H.shape
    r = layer.W_r.shape[0] if r is None else r
    cache = empty_cache(N, d, r)
    a_hat, _ = proxy_identify(H, layer.W_r, cache.P_c)
    cache.P_c[:] = a_hat
    out = partial_block(layer, H, np.arange(N), cache)
    return cache, out


def attn_output_identify(layer: OracleLayer, H: np.ndarray, cache: LayerCache):
    """The attention-output identifier, one of the identifiers the pages
    compare with the Value proxy [NOTES 关键设计 1, Table 1: Query, Key,
    Value, attention output; GIST Key Findings, identifier ablation].

    Every token's attention output is computed from fresh projections of
    every row (reading A24): x = RMSNorm(H); Q, K, V = x W_{q,k,v}ᵀ for all N
    rows, RoPE on Q and K; K^c, V^c ← K, V at every row (the identifier needs
    them); O = softmax(Q K^cᵀ/√d_h) V^c; ô_i = O_i/‖O_i‖ (0 for a zero row);
    s_i = ½‖ô_i − P^c_i‖² with P^c holding the cached unit attention outputs
    (r = d).  Updates K^c and V^c in place; returns (O [N, d], ô, s)."""
    H = np.asarray(H, dtype=np.float64)
    N = H.shape[0]
    _, O = phase2_attention(layer, H, np.arange(N), cache)
    norm = np.sqrt(np.sum(O * O, axis=1))
    o_hat = np.zeros_like(O)
    nz = norm > 0
    o_hat[nz] = O[nz] / norm[nz, None]
    diff = o_hat - np.asarray(cache.P_c, dtype=np.float64)
    return O, o_hat, 0.5 * np.sum(diff * diff, axis=1)


def attn_output_layer_step(layer: OracleLayer, H: np.ndarray, cache: LayerCache, k: int,
                           I: np.ndarray | None = None) -> dict:
    """Cached layer step with the attention-output identifier (reading A24):
    phase 1 scores every token by the drift of its attention output (which
    refreshes K^c, V^c at every row), selects the k most drifted (lowest index
    on ties, ascending) and writes P^c[I] ← ô[I]; phase 2 is the attention
    already computed; phase 3 runs the FFN on the selected rows and scatters
    into H^c [NOTES 整体框架, Phase 3].  Cache updated in place.  A given I
    (ascending, k entries) replaces the top-k, for parity runs where several
    index sets are equally valid (reading A22)."""
    H = np.asarray(H, dtype=np.float64)
    O, o_hat, s = attn_output_identify(layer, H, cache)
    I = select_topk(s, k) if I is None else np.asarray(I, dtype=np.int64)
    cache.P_c[I] = o_hat[I]
    H1, A = phase3_ffn_scatter(layer, H, I, O[I], cache)
    return {"I": I, "s": s, "O": O[I], "H1": H1, "A": A}


def attn_output_fill(layer: OracleLayer, H: np.ndarray) -> tuple:
    """ρ = 1 fill for the attention-output identifier: the full block, with
    P^c = ô of every row (r = d)."""
    H = np.asarray(H, dtype=np.float64)
    N, d = H.shape
    cache = empty_cache(N, d, d)
    O, o_hat, _ = attn_output_identify(layer, H, cache)
    cache.P_c[:] = o_hat
    H1, A = phase3_ffn_scatter(layer, H, np.arange(N), O, cache)
    return cache, {"O": O, "H1": H1, "A": A}


def vanilla_block(layer: OracleLayer, H: np.ndarray) -> np.ndarray:
    """The uncached block: full bidirectional forward of all N positions
    [NOTES 研究背景与动机; GIST Problem Statement].  Written independently
    of the cached path so the two can be compared."""
    H = np.asarray(H, dtype=np.float64)
    N = H.shape[0]
    hd, nh = layer.head_dim, layer.n_heads
    pos = np.arange(N)
    x = rmsnorm(H, layer.attn_norm, layer.eps)
    q = rope((x @ layer.wq.T).reshape(N, nh, hd), pos, layer.theta)
    k = rope((x @ layer.wk.T).reshape(N, nh, hd), pos, layer.theta)
    v = (x @ layer.wv.T).reshape(N, nh, hd)
    h1 = H + attention(q, k, v) @ layer.wo.T
    f, _ = swiglu_ffn(rmsnorm(h1, layer.ffn_norm, layer.eps), layer.w_gate, layer.w_up,
                      layer.w_down)
    return h1 + f


# ---------------------------------------------------------------------------
# Decode loop (masked diffusion: full forward per step, unmask u positions)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class OracleModel:
    layers: list
    embed: np.ndarray       # [vocab, d]
    final_norm: np.ndarray  # [d]
    lm_head: np.ndarray     # [vocab, d]
    eps: float = 1e-5


@dataclasses.dataclass
class DecodeState:
    tokens: np.ndarray      # [B, N]
    H0: np.ndarray          # [B, N, d] layer-0 input (token embeddings)
    caches: list            # caches[l][b] -> LayerCache
    step: int = 0


def init_decode_state(model: OracleModel, tokens: np.ndarray) -> DecodeState:
    tokens = np.array(tokens, dtype=np.int64)
    H0 = np.asarray(model.embed, dtype=np.float64)[tokens]
    return DecodeState(tokens=tokens, H0=H0, caches=[None] * len(model.layers), step=0)


def lm_head_argmax(model: OracleModel, h: np.ndarray, bf16_input: bool = False) -> tuple:
    """Final RMSNorm, logits over the vocabulary, argmax with the lowest
    index on ties (reading A14/A15: only the positions being unmasked).
    bf16_input rounds the normalised rows to bf16 before the LM head, the
    rounding point of a bf16 model (reading A18)."""
    x = rmsnorm(h, model.final_norm, model.eps)
    if bf16_input:
        x = round_bf16(x)
    logits = x @ np.asarray(model.lm_head, dtype=np.float64).T
    return np.argmax(logits, axis=-1).astype(np.int64), logits


def confidence(logits: np.ndarray) -> tuple:
    """Per row of logits [n, V]: the argmax id (lowest on ties) and its
    softmax probability 1 / sum_v exp(l_v - max l), the confidence that
    parallel decoding thresholds [GIST Key Findings, "Integration with
    Parallel Decoding"; NOTES 实验关键数据, 叠加并行解码 (Table 3); reading A23]."""
    lg = np.asarray(logits, dtype=np.float64)
    ids = np.argmax(lg, axis=1)
    top = lg[np.arange(lg.shape[0]), ids]
    return ids.astype(np.int64), 1.0 / np.sum(np.exp(lg - top[:, None]), axis=1)


def confident_positions(conf: np.ndarray, tau: float) -> np.ndarray:
    """Reading A23 (the pages name parallel decoding but not its rule): of a
    sequence's still-masked positions with confidences `conf`, unmask every
    one whose confidence is >= tau; if none is, the single most confident one
    (the first on ties).  Returns indices into `conf`, ascending."""
    conf = np.asarray(conf, dtype=np.float64)
    chosen = np.flatnonzero(conf >= tau)
    if chosen.size == 0:
        chosen = np.array([int(np.argmax(conf))])
    return chosen.astype(np.int64)


def decode_step(model: OracleModel, state: DecodeState, positions: np.ndarray,
                k_per_layer, full: bool, forced: np.ndarray | None = None) -> dict:
    """One decoding step.  With full=True (step 0, or vanilla decoding) every
    layer runs the ρ = 1 fill; otherwise layer l runs the cached step with
    k_per_layer[l].  Then the logits at `positions` ([B, u]) give the argmax
    tokens; the tokens written are `forced` when given (teacher forcing),
    else the argmax.  The next step's layer-0 input changes only at those rows
    [NOTES 研究背景与动机; reading A14].  Updates `state`; returns the argmax
    ids, the written ids, per-layer index sets and per-layer drift scores
    (None for a full step)."""
    B = state.tokens.shape[0]
    Ls = len(model.layers)
    index_sets = [[None] * B for _ in range(Ls)]
    scores = [[None] * B for _ in range(Ls)]
    h_final = np.zeros((B, positions.shape[1], state.H0.shape[2]))
    for b in range(B):
        H = state.H0[b]
        for l, layer in enumerate(model.layers):
            if full:
                cache, _ = full_block(layer, H)
                if state.caches[l] is None:
                    state.caches[l] = [None] * B
                state.caches[l][b] = cache
                index_sets[l][b] = np.arange(H.shape[0])
            else:
                cache = state.caches[l][b]
                out = layer_step(layer, H, cache, k_per_layer[l])
                index_sets[l][b] = out["I"]
                scores[l][b] = out["s"]
            H = state.caches[l][b].H_c
        h_final[b] = H[positions[b]]
    argmax, logits = lm_head_argmax(model, h_final)
    written = argmax if forced is None else np.asarray(forced, dtype=np.int64)
    emb = np.asarray(model.embed, dtype=np.float64)
    for b in range(B):
        state.tokens[b, positions[b]] = written[b]
        state.H0[b, positions[b]] = emb[written[b]]
    state.step += 1
    return {"argmax": argmax, "written": written, "logits": logits, "I": index_sets, "s": scores}

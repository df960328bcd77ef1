"""Pins for the CPU oracle: each check ties an oracle function to something
other than itself (closed forms the pages fix, invariants, library routines,
brute force on tiny inputs).  Runs on CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.spatial.distance import cosine as scipy_cosine_distance

import oracle as O
from adaptive_hidden_state_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ budget

def test_rho_endpoints_exact():
    # The pages fix rho(1) = rho_1, rho(l_p) = rho_p (the peak) and rho(L) = rho_L.
    for (L, rp, lp, r1, rL) in [(32, .25, 12, .06, .06), (32, .25, 12, .03, .10),
                                (2, .25, 1, .25, .1), (8, .4, 8, .05, .2), (5, .5, 3, .1, .2)]:
        assert O.rho(1, L, rp, lp, r1, rL) == pytest.approx(r1 if lp > 1 else rp, rel=1e-15)
        assert O.rho(lp, L, rp, lp, r1, rL) == rp
        if lp < L:
            assert O.rho(L, L, rp, lp, r1, rL) == pytest.approx(rL, rel=1e-15)


def test_rho_closed_form_quarter_points():
    # exp(ln(a) t^2) = a^(t^2): at t = +-1/2 the budget is rho_p * a^(1/4).
    L, lp = 9, 5
    rp, r1, rL = 0.3, 0.05, 0.12
    assert O.rho(3, L, rp, lp, r1, rL) == pytest.approx(rp * (r1 / rp) ** 0.25, rel=1e-14)
    assert O.rho(7, L, rp, lp, r1, rL) == pytest.approx(rp * (rL / rp) ** 0.25, rel=1e-14)


def test_rho_unimodal_peak_at_lp():
    L, lp = 32, 12
    vals = [O.rho(l, L, .25, lp, .06, .06) for l in range(1, L + 1)]
    assert all(vals[i] < vals[i + 1] for i in range(lp - 1))
    assert all(vals[i] > vals[i + 1] for i in range(lp - 1, L - 1))
    assert max(vals) == vals[lp - 1] == .25


def test_budget_k_ceil_and_clamp():
    assert O.budget_k(512, 0.25) == 128          # N*rho exact
    assert O.budget_k(1024, 0.06) == 62          # ceil(61.44)
    assert O.budget_k(64, 1.0) == 64
    assert O.budget_k(64, 1e-9) == 1
    assert O.budget_k(64, 3.0) == 64
    for N in (1, 7, 100, 4096):
        for r in (0.1, 0.16, 0.25, 0.5):
            k = O.budget_k(N, r)
            assert k - 1 < N * r <= k or k == 1


def test_budget_table_golden():
    # Regression fixture written by tests/golden/make_golden.py (oracle only).
    with open(os.path.join(GOLDEN, "budget_tables.json")) as fh:
        g = json.load(fh)
    for case in g["cases"]:
        got = O.budget_table(case["N"], case["L"], case["rho_p"], case["l_p"], case["rho_1"],
                             case["rho_L"])
        assert got == case["k"], case["name"]


def test_pages_facts_fixture():
    # Facts the pages state in words (cited in the fixture): the default peak
    # rho_p = 25% is the peak of the curve; r = 128 is the default rank.
    with open(os.path.join(GOLDEN, "pages_facts.json")) as fh:
        facts = json.load(fh)
    rp = facts["rho_p_default"]["value"]
    assert O.rho(12, 32, rp, 12, .06, .06) == rp
    assert facts["r_default"]["value"] == 128
    # the adaptive curve lowers the mean budget below the peak (25% -> ~16%):
    # with the decode workload's curve (rho_1 = rho_L = 6%, peak at layer 12
    # of 32) the mean of k_l / N is 16% to within one percentage point
    ks = O.budget_table(1024, 32, rp, 12, .06, .06)
    mean = sum(ks) / (32 * 1024)
    assert mean < rp
    assert abs(mean - facts["mean_rho_adaptive"]["value"]) < 0.01


# ------------------------------------------------------------------ SVD proxy

def test_singular_proxy_recovers_construction():
    rng = np.random.default_rng(1)
    d, r = 48, 12
    W, U, sigma, V = synth.power_law_wv(d, rng)
    W_r = O.singular_proxy(W, r)
    expect = sigma[:r, None] * V[:, :r].T
    for i in range(r):
        sgn = np.sign(np.dot(W_r[i], expect[i]))
        assert np.max(np.abs(W_r[i] - sgn * expect[i])) < 1e-10
        j = int(np.argmax(np.abs(W_r[i])))
        assert W_r[i, j] > 0


def _cos(a, b):
    return float(np.dot(a, b) / (np.linalg.norm(a) * np.linalg.norm(b)))


def test_proxy_full_rank_equals_value_similarity():
    # r = d: the proxy cosine equals the cosine of the Value states (U orthogonal).
    rng = np.random.default_rng(2)
    d, N = 32, 10
    W, *_ = synth.power_law_wv(d, rng)
    W_r = O.singular_proxy(W, d)
    H0 = rng.standard_normal((N, d))
    H1 = H0 + 0.3 * rng.standard_normal((N, d))
    a0, _ = O.proxy_identify(H0, W_r, np.zeros((N, d)))
    _, s = O.proxy_identify(H1, W_r, a0)
    for i in range(N):
        assert abs((1 - s[i]) - _cos(W @ H0[i], W @ H1[i])) < 1e-12


def test_proxy_exact_rank_truncation_is_lossless():
    rng = np.random.default_rng(3)
    d, r, N = 40, 6, 12
    spec = np.concatenate([np.linspace(2, 1, r), np.zeros(d - r)])
    W, *_ = synth.power_law_wv(d, rng, spectrum=spec)
    W_r = O.singular_proxy(W, r)
    H0 = rng.standard_normal((N, d))
    H1 = H0 + 0.5 * rng.standard_normal((N, d))
    a0, _ = O.proxy_identify(H0, W_r, np.zeros((N, r)))
    _, s = O.proxy_identify(H1, W_r, a0)
    for i in range(N):
        assert abs((1 - s[i]) - _cos(W @ H0[i], W @ H1[i])) < 1e-10


def test_truncation_bound_theorem_3_4_geometric_spectrum():
    # Theorem 3.4: |cos_r - cos_full| <= 2 (lambda_{r+1}/lambda_r)^2; with
    # lambda_i = 2^-i the bound is 0.5 for every r.  The pages do not print the
    # theorem's hypotheses and a state whose proxy is near zero breaks any such
    # bound, so it is checked where the rank-r proxy keeps >= 90% of both
    # states' Value norm; over all states the error must vanish as r grows.
    rng = np.random.default_rng(4)
    d, N = 64, 2000
    spec = 2.0 ** -np.arange(1, d + 1)
    W, *_ = synth.power_law_wv(d, rng, spectrum=spec)
    lam = np.linalg.svd(W, compute_uv=False)
    H0 = rng.standard_normal((N, d))
    H1 = H0 + rng.uniform(0.0, 1.0, (N, 1)) * rng.standard_normal((N, d))
    v0, v1 = H0 @ W.T, H1 @ W.T
    full = np.einsum("ij,ij->i", v0, v1) / (np.linalg.norm(v0, axis=1) *
                                            np.linalg.norm(v1, axis=1))
    worst = []
    assert np.max(np.abs(lam[:16] / spec[:16] - 1)) < 1e-9
    for r in (1, 2, 4, 8, 16, 32):
        bound = O.truncation_bound(spec, r)
        assert bound == 0.5
        W_r = O.singular_proxy(W, r)
        a0, _ = O.proxy_identify(H0, W_r, np.zeros((N, r)))
        _, s = O.proxy_identify(H1, W_r, a0)
        err = np.abs((1 - s) - full)
        keep = np.minimum(np.linalg.norm(H0 @ W_r.T, axis=1) / np.linalg.norm(v0, axis=1),
                          np.linalg.norm(H1 @ W_r.T, axis=1) / np.linalg.norm(v1, axis=1))
        assert np.count_nonzero(keep >= 0.9) > N // 4
        assert np.max(err[keep >= 0.9]) <= bound
        worst.append(np.max(err))
    assert worst[-2] < 1e-6 and worst[-1] < 1e-12


def test_proxy_score_is_scipy_cosine_distance():
    rng = np.random.default_rng(5)
    N, d, r = 20, 24, 8
    W_r = rng.standard_normal((r, d))
    Hp = rng.standard_normal((N, d))
    Hn = Hp + rng.standard_normal((N, d)) * rng.uniform(0, 1, (N, 1))
    Hn[3] = Hp[3]                                  # unchanged row
    ap, _ = O.proxy_identify(Hp, W_r, np.zeros((N, r)))
    a, s = O.proxy_identify(Hn, W_r, ap)
    for i in range(N):
        ref = scipy_cosine_distance(W_r @ Hn[i], W_r @ Hp[i])
        assert abs(s[i] - ref) < 1e-12
    assert s[3] == 0.0                             # exactly zero, not just small
    assert np.allclose(np.linalg.norm(a, axis=1), 1.0, atol=1e-14)


def test_proxy_zero_vector_and_sign_invariance():
    rng = np.random.default_rng(6)
    N, d, r = 6, 10, 4
    W_r = rng.standard_normal((r, d))
    H = rng.standard_normal((N, d))
    H[2] = 0
    Pc = rng.standard_normal((N, r))
    Pc /= np.linalg.norm(Pc, axis=1, keepdims=True)
    a, s = O.proxy_identify(H, W_r, Pc)
    assert np.all(a[2] == 0) and s[2] == pytest.approx(0.5, abs=1e-15)
    flip = np.diag([1, -1, 1, -1])
    a0, _ = O.proxy_identify(H, W_r, np.zeros((N, r)))
    a0f, _ = O.proxy_identify(H, flip @ W_r, np.zeros((N, r)))
    H2 = H + 0.2 * rng.standard_normal((N, d))
    _, s1 = O.proxy_identify(H2, W_r, a0)
    _, s2 = O.proxy_identify(H2, flip @ W_r, a0f)
    assert np.max(np.abs(s1 - s2)) < 1e-14


# ------------------------------------------------------------------ top-k

def _brute_topk(s, k):
    # rank counting: i is chosen iff fewer than k elements beat it
    N = len(s)
    chosen = [i for i in range(N)
              if sum(1 for j in range(N) if s[j] > s[i] or (s[j] == s[i] and j < i)) < k]
    return chosen


def test_topk_matches_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for N in (1, 2, 5, 9, 16, 33, 64):
        for trial in range(6):
            vals = rng.choice([0.0, 0.25, 0.5, 1.0], size=N) if trial % 2 else rng.random(N)
            for k in range(0, N + 1):
                got = O.select_topk(vals, k)
                assert got.tolist() == _brute_topk(vals, k)


def test_topk_exhaustive_tiny():
    # every subset of size k: the selected one has the largest sorted score
    # vector, ties broken by the lexicographically smallest index list
    rng = np.random.default_rng(8)
    for _ in range(20):
        N = int(rng.integers(1, 8))
        s = rng.choice([0.0, 0.1, 0.7], size=N)
        for k in range(N + 1):
            best = max(itertools.combinations(range(N), k),
                       key=lambda c: (sorted((s[i] for i in c), reverse=True),
                                      [-i for i in c]))
            assert O.select_topk(s, k).tolist() == list(best)


# ------------------------------------------------------------------ bf16 rounding

def test_two_bf16_roundings_agree():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000)).astype(np.float32)
    x[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]   # ties to even
    assert np.array_equal(O.round_bf16(x), synth.bf16_round(x).astype(np.float64))


# ------------------------------------------------------------------ block pieces vs torch

def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((7, 32)) * 3
    g = rng.uniform(0.5, 1.5, 32)
    ref = F.rms_norm(_t(x), (32,), weight=_t(g), eps=1e-5).numpy()
    assert np.max(np.abs(O.rmsnorm(x, g, 1e-5) - ref)) < 1e-13


def test_rope_complex_rotation_and_relative_position():
    rng = np.random.default_rng(11)
    n, heads, dh = 9, 3, 16
    x = rng.standard_normal((n, heads, dh))
    pos = rng.integers(0, 5000, n)
    out = O.rope(x, pos, 10000.0)
    half = dh // 2
    z = x[..., :half] + 1j * x[..., half:]
    freq = 10000.0 ** (-np.arange(half) * 2.0 / dh)
    zr = z * np.exp(1j * pos[:, None, None] * freq[None, None, :])
    assert np.max(np.abs(out[..., :half] - zr.real)) < 1e-9
    assert np.max(np.abs(out[..., half:] - zr.imag)) < 1e-9
    assert np.array_equal(O.rope(x, np.zeros(n, dtype=np.int64), 1e4), x)
    q, k = x[:1], x[1:2]
    for shift in (3, 77):
        a = np.sum(O.rope(q, np.array([5]), 1e4) * O.rope(k, np.array([2]), 1e4), axis=-1)
        b = np.sum(O.rope(q, np.array([5 + shift]), 1e4) * O.rope(k, np.array([2 + shift]), 1e4),
                   axis=-1)
        assert np.max(np.abs(a - b)) < 1e-10


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(12)
    k, N, heads, dh = 5, 13, 4, 8
    Q = rng.standard_normal((k, heads, dh)) * 2
    K = rng.standard_normal((N, heads, dh))
    V = rng.standard_normal((N, heads, dh))
    ref = F.scaled_dot_product_attention(_t(Q).transpose(0, 1), _t(K).transpose(0, 1),
                                         _t(V).transpose(0, 1)).transpose(0, 1)
    assert np.max(np.abs(O.attention(Q, K, V) - ref.reshape(k, -1).numpy())) < 1e-13
    # Q = 0: uniform weights, the output is the mean of V per head
    out0 = O.attention(np.zeros_like(Q), K, V).reshape(k, heads, dh)
    assert np.max(np.abs(out0 - V.mean(axis=0)[None])) < 1e-14


def test_swiglu_matches_torch():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((6, 16))
    wg, wu, wd = rng.standard_normal((24, 16)), rng.standard_normal((24, 16)), \
        rng.standard_normal((16, 24))
    y, A = O.swiglu_ffn(x, wg, wu, wd)
    At = F.silu(F.linear(_t(x), _t(wg))) * F.linear(_t(x), _t(wu))
    assert np.max(np.abs(A - At.numpy())) < 1e-12
    assert np.max(np.abs(y - F.linear(At, _t(wd)).numpy())) < 1e-12


# ------------------------------------------------------------------ block level

def _tiny_layer(seed, d=32, heads=4, ffn=48, r=8, std=0.2):
    shape = synth.LayerShape(d=d, n_heads=heads, head_dim=d // heads, ffn=ffn, r=r)
    w = synth.layer_weights(shape, seed, bf16=False, std=std)
    rng = np.random.default_rng(seed + 100)
    w["attn_norm"] = rng.uniform(0.5, 1.5, d).astype(np.float32)
    w["ffn_norm"] = rng.uniform(0.5, 1.5, d).astype(np.float32)
    return O.OracleLayer.from_weights(w, O.singular_proxy(w["wv"], r), heads)


def _torch_block(layer, H):
    """The same pre-norm block assembled from torch library routines."""
    N, d = H.shape
    nh, hd = layer.n_heads, layer.head_dim
    h = _t(H)
    x = F.rms_norm(h, (d,), weight=_t(layer.attn_norm), eps=layer.eps)
    freq = 10000.0 ** (-torch.arange(hd // 2, dtype=torch.float64) * 2.0 / hd)
    rot = torch.polar(torch.ones(N, hd // 2, dtype=torch.float64),
                      torch.arange(N, dtype=torch.float64)[:, None] * freq[None, :])

    def rope_t(t):
        t = t.view(N, nh, hd)
        z = torch.complex(t[..., :hd // 2], t[..., hd // 2:]) * rot[:, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    q = rope_t(F.linear(x, _t(layer.wq)))
    k = rope_t(F.linear(x, _t(layer.wk)))
    v = F.linear(x, _t(layer.wv)).view(N, nh, hd)
    o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1))
    h1 = h + F.linear(o.transpose(0, 1).reshape(N, d), _t(layer.wo))
    x2 = F.rms_norm(h1, (d,), weight=_t(layer.ffn_norm), eps=layer.eps)
    f = F.linear(F.silu(F.linear(x2, _t(layer.w_gate))) * F.linear(x2, _t(layer.w_up)),
                 _t(layer.w_down))
    return (h1 + f).numpy()


def test_vanilla_block_matches_torch_assembly():
    layer = _tiny_layer(20)
    H = np.random.default_rng(21).standard_normal((11, 32))
    assert np.max(np.abs(O.vanilla_block(layer, H) - _torch_block(layer, H))) < 1e-12


def test_rho_one_cached_step_equals_vanilla():
    layer = _tiny_layer(22)
    rng = np.random.default_rng(23)
    N = 12
    H = rng.standard_normal((N, 32))
    cache, _ = O.full_block(layer, H)
    assert np.max(np.abs(cache.H_c - O.vanilla_block(layer, H))) < 1e-12
    H2 = H + 0.5 * rng.standard_normal((N, 32))
    out = O.layer_step(layer, H2, cache, N)                 # k = N
    assert out["I"].tolist() == list(range(N))
    assert np.max(np.abs(cache.H_c - O.vanilla_block(layer, H2))) < 1e-12


def test_zero_drift_step_keeps_cache():
    layer = _tiny_layer(24)
    H = np.random.default_rng(25).standard_normal((10, 32))
    cache, _ = O.full_block(layer, H)
    before = cache.copy()
    out = O.layer_step(layer, H, cache, 4)
    assert np.all(out["s"] == 0.0)
    assert out["I"].tolist() == [0, 1, 2, 3]
    assert np.max(np.abs(cache.H_c - before.H_c)) < 1e-12
    assert np.array_equal(cache.P_c, before.P_c)


def test_changed_rows_inside_selection_give_exact_rows():
    # every K/V is fresh when only selected rows changed, so the selected
    # outputs equal the uncached forward's rows exactly
    layer = _tiny_layer(26)
    rng = np.random.default_rng(27)
    N, k = 14, 5
    H = rng.standard_normal((N, 32))
    cache, _ = O.full_block(layer, H)
    H2 = H.copy()
    changed = [2, 9, 13]
    H2[changed] += 0.7 * rng.standard_normal((3, 32))
    out = O.layer_step(layer, H2, cache, k)
    assert set(changed) <= set(out["I"].tolist())
    ref = O.vanilla_block(layer, H2)
    assert np.max(np.abs(cache.H_c[out["I"]] - ref[out["I"]])) < 1e-12
    untouched = [i for i in range(N) if i not in out["I"]]
    assert np.array_equal(cache.P_c[untouched], O.proxy_identify(H, layer.W_r,
                                                                  np.zeros((N, 8)))[0][untouched])


# ------------------------------------------------------------------ decode loop

def _tiny_model(seed, L=2, vocab=40, d=32):
    rng = np.random.default_rng(seed)
    layers = [_tiny_layer(seed + 10 * i, d=d) for i in range(L)]
    return O.OracleModel(layers=layers, embed=rng.standard_normal((vocab, d)),
                         final_norm=np.ones(d), lm_head=rng.standard_normal((vocab, d)) * 0.2)


def test_decode_full_k_equals_vanilla_decode():
    model = _tiny_model(30)
    job = synth.decode_inputs(B=2, N=12, n_prompt=4, vocab=40, steps=4, u=2, seed=31)
    s_van = O.init_decode_state(model, job.tokens)
    s_spa = O.init_decode_state(model, job.tokens)
    for t in range(4):
        a = O.decode_step(model, s_van, job.positions[t], None, full=True)
        b = O.decode_step(model, s_spa, job.positions[t], [12, 12], full=(t == 0))
        assert np.array_equal(a["argmax"], b["argmax"])
        assert np.max(np.abs(a["logits"] - b["logits"])) < 1e-10
    assert np.array_equal(s_van.tokens, s_spa.tokens)


def test_decode_layer1_selects_unmasked_rows():
    model = _tiny_model(32)
    job = synth.decode_inputs(B=1, N=16, n_prompt=6, vocab=40, steps=3, u=2, seed=33)
    st = O.init_decode_state(model, job.tokens)
    O.decode_step(model, st, job.positions[0], [4, 4], full=True, forced=job.forced[0])
    out = O.decode_step(model, st, job.positions[1], [4, 4], full=False, forced=job.forced[1])
    # layer-1 inputs changed exactly at step-0's unmasked rows: those score > 0,
    # everything else scores 0 and ties resolve to the lowest indices
    chg = set(job.positions[0][0].tolist())
    I1 = out["I"][0][0].tolist()
    assert chg <= set(I1)
    assert I1 == sorted(chg | set(sorted(set(range(16)) - chg)[:2]))
    assert np.array_equal(st.tokens[0, job.positions[1][0]], job.forced[1][0])


def test_layer_inputs_change_only_at_rewritten_rows_and_scores_carry_over():
    """The facts the incremental proxy relies on, in the oracle's own decode
    loop: between two steps, layer l's input changes only at the rows layer
    l-1 rewrote in the later step (layer 0: the rows unmasked at the end of
    the earlier step); a row outside those and outside the rows layer l
    selected in the earlier step keeps its score exactly; a row selected in
    the earlier step and unchanged since scores exactly 0."""
    model = _tiny_model(40, L=3)
    B, N, u, ks = 1, 20, 2, [5, 6, 4]
    job = synth.decode_inputs(B=B, N=N, n_prompt=6, vocab=40, steps=5, u=u, seed=41)
    st = O.init_decode_state(model, job.tokens)
    O.decode_step(model, st, job.positions[0], ks, full=True, forced=job.forced[0])
    prev_in, prev_s, prev_I = None, None, None
    for t in range(1, 5):
        # this step's per-layer inputs, scores and index sets, by the oracle's own layer step
        inputs, scores, sets = [], [], []
        H = st.H0[0].copy()
        for l, layer in enumerate(model.layers):
            inputs.append(H.copy())
            cache = st.caches[l][0]
            _, s = O.proxy_identify(H, layer.W_r, cache.P_c)
            out = O.layer_step(layer, H, cache, ks[l])
            assert np.array_equal(out["s"], s)
            scores.append(s)
            sets.append(out["I"])
            H = cache.H_c
        if prev_in is not None:
            for l in range(3):
                chg = np.flatnonzero(np.any(inputs[l] != prev_in[l], axis=1))
                allowed = set(job.positions[t - 1][0].tolist()) if l == 0 else set(sets[l - 1].tolist())
                assert set(chg.tolist()) <= allowed, (t, l)
                for i in range(N):
                    if i in allowed:
                        continue
                    if i in set(prev_I[l].tolist()):
                        assert scores[l][i] == 0.0, (t, l, i)
                    else:
                        assert scores[l][i] == prev_s[l][i], (t, l, i)
        # finish the step as decode_step does: LM head at this step's positions, write the ids
        emb = np.asarray(model.embed, dtype=np.float64)
        st.tokens[0, job.positions[t][0]] = job.forced[t][0]
        st.H0[0, job.positions[t][0]] = emb[job.forced[t][0]]
        prev_in, prev_s, prev_I = inputs, scores, sets


def test_rope_keeps_the_query_key_drift_cosine():
    """The Query / Key identifiers score the pre-RoPE projections: RoPE turns
    every head of a token's query or key by the same angles (its own
    position), an orthogonal map, so the cosine between a token's old and new
    vectors is the same before and after it."""
    rng = np.random.default_rng(50)
    heads, dh = 4, 16
    for p in (0, 3, 1023, 4095):
        a = rng.standard_normal((1, heads, dh))
        b = a + 0.3 * rng.standard_normal((1, heads, dh))
        pos = np.array([p])
        ra, rb = O.rope(a, pos, 1e4).ravel(), O.rope(b, pos, 1e4).ravel()
        cos_pre = a.ravel() @ b.ravel() / (np.linalg.norm(a) * np.linalg.norm(b))
        cos_post = ra @ rb / (np.linalg.norm(ra) * np.linalg.norm(rb))
        assert abs(cos_pre - cos_post) < 1e-12


def test_confidence_is_softmax_max_probability():
    from scipy.special import softmax
    rng = np.random.default_rng(60)
    lg = rng.standard_normal((7, 50)) * 3
    lg[2, 10] = lg[2, 20] = lg[2].max() + 1.0  # a tie: the lower id wins
    ids, conf = O.confidence(lg)
    p = softmax(lg, axis=1)
    assert np.array_equal(ids, np.argmax(p, axis=1))
    assert ids[2] == 10
    assert np.max(np.abs(conf - p.max(axis=1))) < 1e-12


def test_confident_positions_rule_brute_force():
    rng = np.random.default_rng(61)
    for _ in range(200):
        n = int(rng.integers(1, 8))
        conf = rng.choice([0.1, 0.3, 0.5, 0.7, 0.9], size=n)
        tau = float(rng.choice([0.2, 0.5, 0.8, 0.95]))
        got = O.confident_positions(conf, tau).tolist()
        above = [i for i in range(n) if conf[i] >= tau]
        if above:
            assert got == above
        else:
            best = max(conf)
            assert got == [min(i for i in range(n) if conf[i] == best)]


def test_lm_head_argmax_matches_torch():
    rng = np.random.default_rng(62)
    d, V = 32, 50
    model = O.OracleModel(layers=[], embed=rng.standard_normal((V, d)),
                          final_norm=rng.uniform(0.5, 1.5, d), lm_head=rng.standard_normal((V, d)))
    h = rng.standard_normal((2, 3, d))
    ids, logits = O.lm_head_argmax(model, h)
    ht = torch.from_numpy(h)
    x = ht * torch.rsqrt(ht.pow(2).mean(-1, keepdim=True) + model.eps) * torch.from_numpy(model.final_norm)
    ref = x @ torch.from_numpy(model.lm_head).T
    assert np.max(np.abs(logits - ref.numpy())) < 1e-10
    assert np.array_equal(ids, ref.argmax(-1).numpy())


def test_lm_head_bf16_input_rounds_the_normalised_rows():
    # with the identity as LM head the logits are the normalised rows
    # themselves: with bf16_input they are those rows rounded to bf16 (each
    # representable in bf16 and within half a bf16 ulp, 2^-8 relative, of the
    # unrounded row), and rows already exact in bf16 are left unchanged
    rng = np.random.default_rng(63)
    d = 64
    model = O.OracleModel(layers=[], embed=None, final_norm=np.ones(d), lm_head=np.eye(d), eps=0.0)
    h = rng.standard_normal((3, d))
    _, x = O.lm_head_argmax(model, h)
    _, xr = O.lm_head_argmax(model, h, bf16_input=True)
    assert np.array_equal(xr.astype(np.float32), synth.bf16_round(xr.astype(np.float32)))
    assert np.all(np.abs(xr - x) <= 2.0 ** -8 * np.abs(x))
    assert np.any(xr != x)
    signs = rng.choice([-1.0, 1.0], size=(2, d))      # rms 1: the normalised row is exactly +-1
    _, a = O.lm_head_argmax(model, 3.0 * signs)
    _, b = O.lm_head_argmax(model, 3.0 * signs, bf16_input=True)
    assert np.array_equal(a, b) and np.allclose(np.abs(a), 1.0)


# ------------------------------------------------------- attention-output identifier

def _torch_attention_rows(layer, H):
    """Every row's attention output and post-RoPE keys / values from torch
    routines (the first half of _torch_block)."""
    N, d = H.shape
    nh, hd = layer.n_heads, layer.head_dim
    x = F.rms_norm(_t(H), (d,), weight=_t(layer.attn_norm), eps=layer.eps)
    freq = 10000.0 ** (-torch.arange(hd // 2, dtype=torch.float64) * 2.0 / hd)
    rot = torch.polar(torch.ones(N, hd // 2, dtype=torch.float64),
                      torch.arange(N, dtype=torch.float64)[:, None] * freq[None, :])

    def rope_t(t):
        t = t.view(N, nh, hd)
        z = torch.complex(t[..., :hd // 2], t[..., hd // 2:]) * rot[:, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    q, k = rope_t(F.linear(x, _t(layer.wq))), rope_t(F.linear(x, _t(layer.wk)))
    v = F.linear(x, _t(layer.wv)).view(N, nh, hd)
    o = F.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1))
    return o.transpose(0, 1).reshape(N, d).numpy(), k.reshape(N, d).numpy(), v.reshape(N, d).numpy()


def test_attn_output_fill_is_vanilla_with_unit_outputs_cached():
    layer = _tiny_layer(70)
    H = np.random.default_rng(71).standard_normal((9, 32))
    cache, _ = O.attn_output_fill(layer, H)
    o, k, v = _torch_attention_rows(layer, H)
    assert np.max(np.abs(cache.H_c - _torch_block(layer, H))) < 1e-12
    assert np.max(np.abs(cache.P_c - o / np.linalg.norm(o, axis=1, keepdims=True))) < 1e-12
    assert np.max(np.abs(cache.K_c - k)) < 1e-12 and np.max(np.abs(cache.V_c - v)) < 1e-12


def test_attn_output_step_scores_refreshes_and_selects():
    # the score is the cosine distance of every row's fresh attention output
    # to the one cached at the fill; every K/V row is refreshed; only the k
    # selected rows of H^c change; with k = N the step is the vanilla block
    layer = _tiny_layer(72)
    rng = np.random.default_rng(73)
    N, k = 12, 5
    H = rng.standard_normal((N, 32))
    H2 = H.copy()
    H2[[2, 7, 9]] += 0.7 * rng.standard_normal((3, 32))
    cache, _ = O.attn_output_fill(layer, H)
    o_old = _torch_attention_rows(layer, H)[0]
    before = cache.copy()
    out = O.attn_output_layer_step(layer, H2, cache, k)
    o_new, k_new, v_new = _torch_attention_rows(layer, H2)
    ref = np.array([scipy_cosine_distance(o_new[i], o_old[i]) for i in range(N)])
    assert np.max(np.abs(out["s"] - ref)) < 1e-12
    assert out["I"].tolist() == sorted(np.lexsort((np.arange(N), -out["s"]))[:k].tolist())
    assert np.max(np.abs(cache.K_c - k_new)) < 1e-12 and np.max(np.abs(cache.V_c - v_new)) < 1e-12
    keep = np.setdiff1d(np.arange(N), out["I"])
    assert np.array_equal(cache.H_c[keep], before.H_c[keep])
    assert np.max(np.abs(cache.H_c[out["I"]] - _torch_block(layer, H2)[out["I"]])) < 1e-12
    full = O.attn_output_fill(layer, H)[0]
    O.attn_output_layer_step(layer, H2, full, N)
    assert np.max(np.abs(full.H_c - _torch_block(layer, H2))) < 1e-12


def test_attn_output_zero_drift_selects_lowest_indices():
    layer = _tiny_layer(74)
    H = np.random.default_rng(75).standard_normal((10, 32))
    cache, _ = O.attn_output_fill(layer, H)
    before = cache.copy()
    out = O.attn_output_layer_step(layer, H, cache, 3)
    assert np.all(out["s"] == 0.0) and out["I"].tolist() == [0, 1, 2]
    assert np.max(np.abs(cache.H_c - before.H_c)) < 1e-12

"""GPU parity of the cached layer step (through the C ABI) against the CPU
oracle: the tiny fp32 layer, edge cases of the bf16 path at small widths,
and one LLaDA-8B-shaped bf16 layer (d=4096, 32x128 heads, F=12288, r=128,
N=512, rho=0.25)."""
import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth
from spa_testutil import LayerPair, assert_close, assert_index_set, np64

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")


def _run_fill(lp: LayerPair, H: np.ndarray):
    """rho = 1 fill on both sides; returns (gpu cache, oracle caches per seq)."""
    B, N, _ = H.shape
    cache = lp.cache(B, N)
    spa.spa_full_block(lp.layer, lp.to_dev(H), cache, True)
    lp.ws.check()
    ocs = [O.full_block(lp.ol, H[b])[0] for b in range(B)]
    return cache, ocs


def _compare_cache(lp, cache, ocs, what):
    bf = lp.bf16
    assert_close(cache.k, np.stack([c.K_c for c in ocs]), bf, what + " K^c")
    assert_close(cache.v, np.stack([c.V_c for c in ocs]), bf, what + " V^c")
    assert_close(cache.h, np.stack([c.H_c for c in ocs]), bf, what + " H^c")
    p = np64(cache.p)
    assert np.max(np.abs(p - np.stack([c.P_c for c in ocs]))) < (2e-3 if bf else 1e-5), what + " P^c"


def _compare_rewritten_rows(lp, cache, ocs, I_gpu, before, what):
    """After a cached step: the rewritten rows K^c/V^c/H^c[I] against the
    oracle's, each on its own (so the N - k untouched rows cannot dilute the
    error of the k rewritten ones), and every other row bit-identical to the
    cache before the step."""
    after = [np64(t) for t in (cache.k, cache.v, cache.h)]
    for b in range(I_gpu.shape[0]):
        I = I_gpu[b].astype(np.int64)
        keep = np.ones(after[0].shape[1], bool)
        keep[I] = False
        for j, (name, ref) in enumerate((("K^c", ocs[b].K_c), ("V^c", ocs[b].V_c), ("H^c", ocs[b].H_c))):
            assert_close(after[j][b][I], ref[I], lp.bf16, f"{what} seq {b} {name}[I]")
            assert np.array_equal(after[j][b][keep], before[j][b][keep]), f"{what} seq {b} {name} outside I"


def _step(lp, cache, ocs, H2, k, check_intermediates=True):
    """Cached step on both sides, compared phase by phase."""
    B, N, d = H2.shape
    before = [np64(t) for t in (cache.k, cache.v, cache.h)]
    H2d = lp.to_dev(H2)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    score = torch.empty((B, N), dtype=torch.float32, device="cuda")
    spa.spa_proxy_select(lp.layer, H2d, cache, k, idx, score)
    lp.ws.check()
    outs = [O.layer_step(lp.ol, H2[b], ocs[b], k) for b in range(B)]
    s_gpu = np64(score)
    I_gpu = idx.cpu().numpy()
    for b in range(B):
        s_ref = outs[b]["s"]
        zero = s_ref == 0.0
        assert np.all(s_gpu[b][zero] == 0.0), "unchanged rows must score exactly 0"
        assert np.max(np.abs(s_gpu[b] - s_ref)) < (5e-3 if lp.bf16 else 1e-5)
        assert_index_set(I_gpu[b], s_ref, k, outs[b]["I"], f"I[{b}]")
        # continue the oracle with the GPU's index set when several were valid
        if not np.array_equal(I_gpu[b], outs[b]["I"]):
            raise AssertionError("index sets differ; inputs should carry a margin")
    spa.spa_partial_block(lp.layer, H2d, idx, k, cache)
    lp.ws.check()
    if check_intermediates:
        dt = spa.torch_dtype(lp.dtype)
        M = B * k
        for name, key, width in (("q", "Q", d), ("o", "O", d), ("h1", "H1", d),
                                 ("a", "A", lp.shape.ffn)):
            got = lp.ws.view(name, (M, width), dt)
            ref = np.concatenate([outs[b][key] for b in range(B)])
            assert_close(got, ref, lp.bf16, "step " + key)
    _compare_rewritten_rows(lp, cache, ocs, I_gpu, before, "step")
    _compare_cache(lp, cache, ocs, "step")
    return I_gpu, outs


# ----------------------------------------------------------------- tiny fp32 layer

def test_tiny_fp32_layer_fill_and_cached_step():
    lp = LayerPair(spa, synth.TINY_LAYER, seed=0, dtype=spa.SPA_F32, max_B=1, max_N=64)
    H = synth.hidden_states(1, 64, 256, seed=1, bf16=False)
    cache, ocs = _run_fill(lp, H)
    _compare_cache(lp, cache, ocs, "fill")
    for name, key, width in (("q", "Q", 256), ("o", "O", 256), ("h1", "H1", 256), ("a", "A", 688)):
        got = lp.ws.view(name, (64, width), torch.float32)
        ref = O.full_block(lp.ol, H[0])[1][key]
        assert_close(got, ref, False, "fill " + key)
    H2, rows = synth.drift_rows(H, 0.05, 0.3, seed=2, bf16=False)
    I, _ = _step(lp, cache, ocs, H2, 16)
    assert set(rows[0].tolist()) <= set(I[0].tolist())


def test_tiny_fp32_graded_drift_exact_selection():
    lp = LayerPair(spa, synth.TINY_LAYER, seed=3, dtype=spa.SPA_F32, max_B=2, max_N=64)
    H = synth.hidden_states(2, 64, 256, seed=4, bf16=False)
    cache, ocs = _run_fill(lp, H)
    # re-seed until the oracle's k-th/(k+1)-th scores are >= 1e-4 apart
    for seed in range(100, 200):
        H2 = synth.graded_drift(H, 0.01, 0.1, seed=seed, bf16=False)
        ok = True
        for b in range(2):
            _, s = O.proxy_identify(H2[b], lp.ol.W_r, ocs[b].P_c)
            srt = np.sort(s)[::-1]
            ok &= srt[15] - srt[16] >= 1e-4
        if ok:
            break
    _step(lp, cache, ocs, H2, 16)


# ----------------------------------------------------------------- bf16 edge cases

SMALL_BF16 = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)


@pytest.mark.parametrize("B,N,k", [(1, 1, 1), (1, 7, 3), (2, 130, 1), (1, 130, 130),
                                   (2, 257, 40), (1, 300, 299)])
def test_bf16_small_layer_shapes(B, N, k):
    lp = LayerPair(spa, SMALL_BF16, seed=10 + N, dtype=spa.SPA_BF16, max_B=2, max_N=300, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=N, bf16=True)
    cache, ocs = _run_fill(lp, H)
    _compare_cache(lp, cache, ocs, "fill")
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=N + 1, bf16=True)
    _step(lp, cache, ocs, H2, k)


@pytest.mark.parametrize("bm", ["", "128"])
@pytest.mark.parametrize("B,N,k", [(1, 600, 600), (2, 300, 300), (1, 1030, 520), (2, 520, 40)])
def test_bf16_tiled_gemm_row_tiles(monkeypatch, bm, B, N, k):
    # the tiled GEMMs of the rho = 1 fill and of cached steps with more than 256
    # tokens: 256-row tiles (two TMEM accumulators, the epilogue in two halves)
    # for M >= 512, including ragged last tiles (M = 600, 1030, 1040) and the
    # split-K the planner picks for them, against 128-row tiles (SPA_TC_BM=128)
    if bm:
        monkeypatch.setenv("SPA_TC_BM", bm)
    lp = LayerPair(spa, SMALL_BF16, seed=20 + N + k, dtype=spa.SPA_BF16, max_B=B, max_N=N, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=N + 3, bf16=True)
    cache, ocs = _run_fill(lp, H)
    _compare_cache(lp, cache, ocs, "fill")
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=N + 4, bf16=True)
    _step(lp, cache, ocs, H2, k)


@pytest.mark.parametrize("B,N,k", [(1, 200, 96), (2, 300, 100)])
def test_bf16_separate_ffn_norm(monkeypatch, B, N, k):
    # the FFN RMSNorm as its own kernel (SPA_NORM_FOLD=0) instead of folded into
    # the O-proj and gate/up epilogues of the weight-stationary path
    monkeypatch.setenv("SPA_NORM_FOLD", "0")
    lp = LayerPair(spa, SMALL_BF16, seed=60 + k, dtype=spa.SPA_BF16, max_B=2, max_N=300, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=k + 11, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=k + 12, bf16=True)
    _step(lp, cache, ocs, H2, k)


@pytest.mark.parametrize("nacc", ["2", "4"])
@pytest.mark.parametrize("B,N,k", [(1, 200, 96), (2, 160, 33)])
def test_bf16_wide_weight_tiles(monkeypatch, nacc, B, N, k):
    # more weight rows per CTA than the planner would pick at this width,
    # including tiles that run past the last weight matrix
    monkeypatch.setenv("SPA_WS_NACC", nacc)
    lp = LayerPair(spa, SMALL_BF16, seed=40 + k, dtype=spa.SPA_BF16, max_B=2, max_N=200, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=k, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=k + 1, bf16=True)
    _step(lp, cache, ocs, H2, k)


MID_BF16 = synth.LayerShape(d=1024, n_heads=8, head_dim=128, ffn=1536, r=64)


@pytest.mark.parametrize("glob", ["0", "2", "3", "5", "8", ""])
@pytest.mark.parametrize("B,N,k", [(1, 200, 96), (2, 160, 33), (1, 300, 200)])
def test_bf16_ws_global_split_k(monkeypatch, glob, B, N, k):
    # the weight-stationary GEMMs with their k-blocks split over separate CTAs
    # that reduce through global memory (each split publishes its fp32 partial
    # tile, waits for the tile's other splits, and sums its share of the token
    # rows in split order): 2, 3, 5 and 8 splits of every GEMM whose grid stays
    # resident (QKV 24 tiles of 16 k-blocks, gate/up 12, O-proj and down 8 of 16
    # and 24), the clusters only (0) and the planner's choice.  Two steps: the
    # second finds the counters reset by the first.
    if glob:
        monkeypatch.setenv("SPA_WS_GLOBAL", glob)
    lp = LayerPair(spa, MID_BF16, seed=70 + k, dtype=spa.SPA_BF16, max_B=2, max_N=300, std=0.03)
    H = synth.hidden_states(B, N, MID_BF16.d, seed=k + 7, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=k + 8, bf16=True)
    _step(lp, cache, ocs, H2, k)
    _step(lp, cache, ocs, H, k)


@pytest.mark.parametrize("nacc", ["1", "2"])
@pytest.mark.parametrize("grid", ["1", "5", "12", "24"])
@pytest.mark.parametrize("B,N,k", [(1, 200, 96), (2, 160, 33), (1, 300, 200)])
def test_bf16_stream_k_partitions(monkeypatch, nacc, grid, B, N, k):
    # the opt-in stream-K weight-streaming GEMMs over 1, 5, 12 and 24 CTAs with one
    # or two 128-row tiles per unit: one CTA for everything, ranges that split
    # tiles unevenly, and one k-block per CTA (QKV and gate/up: 24 units of
    # one tile, 12 of two), so every tile is fixed up from 4 partials; k = 200
    # takes one TMEM buffer when two tiles share a unit
    monkeypatch.setenv("SPA_STREAMK", "1")
    monkeypatch.setenv("SPA_SK_GRID", grid)
    monkeypatch.setenv("SPA_SK_NACC", nacc)
    lp = LayerPair(spa, SMALL_BF16, seed=80 + k, dtype=spa.SPA_BF16, max_B=2, max_N=300, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=k + 3, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=k + 4, bf16=True)
    _step(lp, cache, ocs, H2, k)


@pytest.mark.parametrize("grid", ["", "3", "8"])
@pytest.mark.parametrize("B,N,k", [(1, 200, 96), (2, 160, 33), (1, 300, 200)])
def test_bf16_persistent_ffn(monkeypatch, grid, B, N, k):
    # the FFN half as one persistent launch (O-proj, FFN norm, gate/up, down
    # streamed back to back, each phase split over the CTAs), over the
    # planner's grid and over 3 and 8 CTAs (tiles fixed up from up to 4
    # partials); k = 200 takes one 128-row gate/up tile per unit
    monkeypatch.setenv("SPA_FFN", "1")
    if grid:
        monkeypatch.setenv("SPA_FFN_GRID", grid)
    lp = LayerPair(spa, SMALL_BF16, seed=90 + k, dtype=spa.SPA_BF16, max_B=2, max_N=300, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=k + 5, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=k + 6, bf16=True)
    _step(lp, cache, ocs, H2, k)
    _step(lp, cache, ocs, H, k)   # a second launch: the counters were reset by the first


@pytest.mark.parametrize("B,N,k", [(1, 2048, 200), (2, 1000, 62), (1, 1536, 129), (1, 3000, 200)])
def test_bf16_split_key_attention(B, N, k):
    # long caches: the keys of each query tile are split over a cluster of 8
    # CTAs (2, 1, 1-2 and 3 key tiles each; N=1000 and N=3000 end in a partial
    # key tile), with one or two query tiles, the second holding 72 or 1 rows
    # (the LLaDA-shaped layer tests take 4-way and 2-way clusters).  N=3000 also
    # takes the unfused select (more than 2048 scores).
    lp = LayerPair(spa, SMALL_BF16, seed=50 + k, dtype=spa.SPA_BF16, max_B=B, max_N=N, std=0.05)
    H = synth.hidden_states(B, N, 256, seed=k + 7, bf16=True)
    cache, ocs = _run_fill(lp, H)
    H2, _ = synth.drift_rows(H, 0.05, 0.5, seed=k + 8, bf16=True)  # fewer drifted rows than k
    _step(lp, cache, ocs, H2, k)


@pytest.mark.parametrize("bf16,B,N,k", [(False, 2, 64, 16), (True, 2, 1000, 62), (True, 1, 300, 257),
                                        (True, 1, 2048, 200), (True, 2, 512, 128), (True, 1, 64, 64),
                                        (True, 2, 300, 1)])
def test_layer_step_equals_select_then_partial_block(bf16, B, N, k):
    # spa_layer_step selects, gathers and normalises in one launch; its
    # results must be bit-identical to spa_proxy_select + spa_partial_block
    shape = SMALL_BF16 if bf16 else synth.TINY_LAYER
    dtype = spa.SPA_BF16 if bf16 else spa.SPA_F32
    lp = LayerPair(spa, shape, seed=60 + k, dtype=dtype, max_B=B, max_N=N, std=0.05)
    H = synth.hidden_states(B, N, shape.d, seed=k + 9, bf16=bf16)
    H2, _ = synth.drift_rows(H, 0.3, 0.5, seed=k + 10, bf16=bf16)
    Hd, H2d = lp.to_dev(H), lp.to_dev(H2)
    outs = []
    for fused in (True, False):
        cache = lp.cache(B, N)
        spa.spa_full_block(lp.layer, Hd, cache, True)
        idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
        if fused:
            spa.spa_layer_step(lp.layer, H2d, cache, k, idx)
        else:
            spa.spa_proxy_select(lp.layer, H2d, cache, k, idx)
            spa.spa_partial_block(lp.layer, H2d, idx, k, cache)
        lp.ws.check()
        x = lp.ws.view("x", (B * k, shape.d), spa.torch_dtype(dtype)).clone()
        outs.append((idx.clone(), x, cache.k.clone(), cache.v.clone(), cache.h.clone(), cache.p.clone()))
    for name, a, b in zip(("idx", "X", "K^c", "V^c", "H^c", "P^c"), *outs):
        assert torch.equal(a, b), name


def test_bf16_zero_drift_selects_lowest_indices():
    lp = LayerPair(spa, SMALL_BF16, seed=21, dtype=spa.SPA_BF16, max_B=1, max_N=200, std=0.05)
    H = synth.hidden_states(1, 200, 256, seed=22, bf16=True)
    cache, ocs = _run_fill(lp, H)
    h_before = cache.h.clone()
    I, _ = _step(lp, cache, ocs, H, 37)
    assert I[0].tolist() == list(range(37))
    assert_close(cache.h, np64(h_before), True, "zero-drift H^c")


def test_bf16_step_is_deterministic():
    lp = LayerPair(spa, SMALL_BF16, seed=23, dtype=spa.SPA_BF16, max_B=2, max_N=256, std=0.05)
    H = synth.hidden_states(2, 256, 256, seed=24, bf16=True)
    H2, _ = synth.drift_rows(H, 0.1, 0.4, seed=25, bf16=True)
    outs = []
    for _ in range(2):
        cache = lp.cache(2, 256)
        spa.spa_full_block(lp.layer, lp.to_dev(H), cache, True)
        idx = torch.empty((2, 64), dtype=torch.int32, device="cuda")
        spa.spa_layer_step(lp.layer, lp.to_dev(H2), cache, 64, idx)
        lp.ws.check()
        outs.append((idx.clone(), cache.k.clone(), cache.v.clone(), cache.h.clone(), cache.p.clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_device_index_check_reports_without_fault():
    lp = LayerPair(spa, SMALL_BF16, seed=26, dtype=spa.SPA_BF16, max_B=1, max_N=64, std=0.05)
    H = lp.to_dev(synth.hidden_states(1, 64, 256, seed=27, bf16=True))
    cache = lp.cache(1, 64)
    idx = torch.tensor([[0, 5, 64, 70]], dtype=torch.int32, device="cuda")  # 64, 70 out of range
    spa.spa_partial_block(lp.layer, H, idx, 4, cache)
    assert lp.ws.status() == -7
    assert lp.ws.status() == 0       # cleared


# ----------------------------------------------------------------- LLaDA-shaped bf16 layer

@pytest.fixture(scope="module")
def llada():
    lp = LayerPair(spa, synth.LLADA_LAYER, seed=0, dtype=spa.SPA_BF16, max_B=1, max_N=512)
    H = synth.hidden_states(1, 512, 4096, seed=1, bf16=True)
    return lp, H


def test_llada_proxy_weights_match_oracle_svd(llada):
    lp, _ = llada
    got = lp.layer.proxy_weights().numpy().astype(np.float64)
    ref = lp.W_r
    sgn = np.sign(np.sum(got * ref, axis=1))[:, None]
    assert np.all(sgn == 1)
    diff = np.abs(got - ref)
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert np.mean(diff > 0) < 1e-3          # bf16 storage: identical but for rare ties
    assert np.all(diff <= ulp)


def test_llada_fill_then_cached_step(llada):
    lp, H = llada
    cache, ocs = _run_fill(lp, H)
    _compare_cache(lp, cache, ocs, "fill")
    H2, rows = synth.drift_rows(H, 0.05, 0.3, seed=2, bf16=True)   # 26 drifted rows
    I, _ = _step(lp, cache, ocs, H2, 128)
    assert set(rows[0].tolist()) <= set(I[0].tolist())


def test_llada_persistent_ffn_cached_steps(llada, monkeypatch):
    # the persistent FFN launch at the LLaDA layer shape (148 CTAs), over two
    # cached steps (the second one reuses the counters the first reset)
    monkeypatch.setenv("SPA_FFN", "1")
    lp, H = llada
    cache, ocs = _run_fill(lp, H)
    H2, rows = synth.drift_rows(H, 0.05, 0.3, seed=2, bf16=True)
    I, _ = _step(lp, cache, ocs, H2, 128)
    assert set(rows[0].tolist()) <= set(I[0].tolist())
    _step(lp, cache, ocs, H, 200)


def test_llada_graded_drift_exact_selection(llada):
    lp, H = llada
    cache, ocs = _run_fill(lp, H)
    for seed in range(300, 400):
        H2 = synth.graded_drift(H, 0.01, 0.1, seed=seed, bf16=True)
        _, s = O.proxy_identify(H2[0], lp.ol.W_r, ocs[0].P_c)
        srt = np.sort(s)[::-1]
        if srt[127] - srt[128] >= 1e-4:
            break
    else:
        pytest.fail("no seed with a 1e-4 margin")
    _step(lp, cache, ocs, H2, 128)

"""GPU parity of the attention-output identifier (spa_full_block with
fill_proxy = 2, spa_layer_step_attn_identifier), the identifier the pages
compare with the Value proxy (papernotes.org, 关键设计 1, Table 1): every
token's attention output from fresh Q/K/V of every row is scored against the
cached unit output, the k most drifted rows are selected, and the FFN runs on
them.  Checked against the oracle's attn_output_fill / attn_output_layer_step
on the same inputs: the fill (K^c, V^c, H^c, the cached unit outputs P^c),
every row's attention output, the scores and index set in the kernel's own
precision, the selected rows' attention outputs, H1, A, every refreshed
K^c / V^c row, the rewritten H^c and P^c rows, and the other rows bit for
bit.  Small bf16 shape (d = 256, two 128-wide heads, r = d) at B = 1, 2, and
one LLaDA-8B-shaped layer (d = 4096, 32 x 128 heads, F = 12288, N = 512)."""
import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth
from spa_testutil import NAMES, assert_close, np64

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")


def _layer(shape, seed, max_B, max_N, std):
    w = synth.layer_weights(shape, seed, bf16=True, std=std) if shape.d <= 256 else None
    if w is None:  # LLaDA-shaped: seeded on the device, copied to the host for the oracle
        g = torch.Generator(device="cuda").manual_seed(seed)
        rn = lambda s, sd: (torch.randn(s, generator=g, device="cuda") * sd).to(torch.bfloat16)
        d, F = shape.d, shape.ffn
        dev = {"wq": rn((d, d), std), "wk": rn((d, d), std), "wv": rn((d, d), std), "wo": rn((d, d), std),
               "w_gate": rn((F, d), std), "w_up": rn((F, d), std), "w_down": rn((d, F), std),
               "attn_norm": torch.ones(d, device="cuda", dtype=torch.bfloat16),
               "ffn_norm": torch.ones(d, device="cuda", dtype=torch.bfloat16)}
        w = {n: dev[n].float().cpu().numpy() for n in NAMES}
    else:
        dev = {n: torch.from_numpy(np.ascontiguousarray(w[n])).to("cuda", torch.bfloat16) for n in NAMES}
    desc = spa.LayerDesc(d=shape.d, n_heads=shape.n_heads, head_dim=shape.head_dim, ffn=shape.ffn, r=shape.d,
                         dtype=spa.SPA_BF16, rms_eps=shape.rms_eps, rope_theta=shape.rope_theta)
    ws = spa.Workspace(desc, max_B, max_N)
    # the identifier does not use W_r; any r x d proxy makes the handle
    layer = spa.Layer(desc, dev, ws, w_r_host=dev["wv"].float().cpu())
    ol = O.OracleLayer.from_weights(w, np.asarray(w["wv"], np.float64), shape.n_heads, shape.rms_eps,
                                    shape.rope_theta)
    return layer, ws, ol, dev


# The score kernel decides the index set from the GPU's own bf16 attention
# outputs, so the decision is checked in that precision: scores recomputed in
# fp64 from the GPU's outputs and the cached unit outputs before the step must
# match the kernel's to 1e-5, and the index set is the top-k of those scores
# (exactly when the k-th and (k+1)-th are >= 1e-4 apart, otherwise any set
# valid within 1e-4).  The outputs themselves are compared with the oracle's
# within the bf16 tolerance.
MARGIN = 1e-4


def _unit_rows(x):
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def _run(shape, B, N, frac, seed, std):
    layer, ws, ol, dev = _layer(shape, seed, B, N, std)
    d = shape.d
    H = synth.hidden_states(B, N, d, seed=seed + 1, bf16=True)
    H2, rows = synth.drift_rows(H, frac, 0.5, seed=seed + 2, bf16=True)
    k = max(1, N // 4)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)
    cache = spa.Cache(B, N, d, d, spa.SPA_BF16)
    spa.spa_full_block(layer, to(H), cache, 2)
    ws.check()
    ocs = [O.attn_output_fill(ol, H[b])[0] for b in range(B)]
    for name, key in (("k", "K_c"), ("v", "V_c"), ("h", "H_c")):
        assert_close(getattr(cache, name), np.stack([getattr(c, key) for c in ocs]), True, f"fill {name}")
    o_fill = ws.view("o", (B, N, d), torch.bfloat16).clone()
    p_fill = np64(cache.p)
    assert np.max(np.abs(p_fill - _unit_rows(np64(o_fill)))) < 1e-5, "fill P^c = unit rows of the outputs"
    assert_close(cache.p, np.stack([c.P_c for c in ocs]), True, "fill P^c")
    h_before = np64(cache.h)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    spa.spa_layer_step_attn_identifier(layer, to(H2), cache, k, idx)
    ws.check()
    I_gpu = idx.cpu().numpy()
    s_gpu = ws.view("score", (B, N), torch.float32).clone().cpu().numpy().astype(np.float64)
    o_all = np64(ws.view("o", (B, N, d), torch.bfloat16).clone())
    outs = []
    for b in range(B):
        # every row's attention output against the oracle's (fresh Q/K/V of every row)
        o_ref = O.attn_output_identify(ol, H2[b], ocs[b].copy())[0]
        assert_close(o_all[b], o_ref, True, f"seq {b} O (every row)")
        # the kernel's scores and selection, in its own precision
        s_own = 0.5 * np.sum((_unit_rows(o_all[b]) - p_fill[b]) ** 2, axis=1)
        assert np.max(np.abs(s_gpu[b] - s_own)) < 1e-5, f"seq {b} scores"
        srt = np.sort(s_own)[::-1]
        if k == N or srt[k - 1] - srt[k] >= MARGIN:
            assert np.array_equal(I_gpu[b], O.select_topk(s_own, k)), f"seq {b} index set"
        else:
            sel = np.zeros(N, bool)
            sel[I_gpu[b]] = True
            assert np.all(np.diff(I_gpu[b]) > 0)
            assert np.all(s_own[sel] >= srt[k - 1] - MARGIN) and np.all(s_own[~sel] <= srt[k - 1] + MARGIN)
        # the oracle continues with the GPU's index set
        outs.append(O.attn_output_layer_step(ol, H2[b], ocs[b], k, I=I_gpu[b]))
    views = {n: ws.view(n, (B * k, w), torch.bfloat16).clone()
             for n, w in (("x", d), ("h1", d), ("a", shape.ffn))}
    h_after, p_after = np64(cache.h), np64(cache.p)
    for b in range(B):
        r_ = slice(b * k, (b + 1) * k)
        I = I_gpu[b].astype(np.int64)
        keep = np.setdiff1d(np.arange(N), I)
        assert np.array_equal(np64(views["x"][r_]), o_all[b][I]), f"seq {b} gathered O[I]"
        assert_close(views["x"][r_], outs[b]["O"], True, f"seq {b} O[I]")
        assert_close(views["h1"][r_], outs[b]["H1"], True, f"seq {b} H1")
        assert_close(views["a"][r_], outs[b]["A"], True, f"seq {b} A")
        assert_close(h_after[b][I], ocs[b].H_c[I], True, f"seq {b} H^c[I]")
        assert np.array_equal(h_after[b][keep], h_before[b][keep]), f"seq {b} H^c outside I"
        assert np.max(np.abs(p_after[b][I] - _unit_rows(o_all[b][I]))) < 1e-5, f"seq {b} P^c[I]"
        assert np.array_equal(p_after[b][keep], p_fill[b][keep]), f"seq {b} P^c outside I"
    for name, key in (("k", "K_c"), ("v", "V_c")):
        assert_close(getattr(cache, name), np.stack([getattr(c, key) for c in ocs]), True, f"step {name} (every row)")


@pytest.mark.parametrize("B,N,frac", [(1, 200, 0.2), (2, 300, 0.1)])
def test_attn_output_identifier_small(B, N, frac):
    _run(synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=256), B, N, frac, seed=91 + N, std=0.05)


def test_attn_output_identifier_llada_layer():
    _run(synth.LayerShape(d=4096, n_heads=32, head_dim=128, ffn=12288, r=4096), 1, 512, 0.05, seed=95,
         std=0.02)


def test_attn_output_identifier_needs_r_equal_d():
    shape = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)
    w = synth.layer_weights(shape, 7, bf16=True, std=0.05)
    dev = {n: torch.from_numpy(np.ascontiguousarray(w[n])).to("cuda", torch.bfloat16) for n in NAMES}
    desc = spa.LayerDesc(d=256, n_heads=2, head_dim=128, ffn=384, r=16, dtype=spa.SPA_BF16, rms_eps=1e-5,
                         rope_theta=1e4)
    ws = spa.Workspace(desc, 1, 64)
    layer = spa.Layer(desc, dev, ws, w_r_host=np.zeros((16, 256), np.float32))
    cache = spa.Cache(1, 64, 256, 16, spa.SPA_BF16)
    H = torch.zeros((1, 64, 256), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((1, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_layer_step_attn_identifier(layer, H, cache, 8, idx)
    assert ei.value.status == -2
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_full_block(layer, H, cache, 2)
    assert ei.value.status == -2

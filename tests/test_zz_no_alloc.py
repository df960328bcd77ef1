"""GPU test of the allocation-free attention entry point (spa_attention_noalloc).

Callers that may not allocate device memory (custom memory managers and
allocator hooks, hosts with a fixed memory budget, loops where an allocation's
implicit synchronisation is not allowed) use this variant: its split-over-keys
scratch is a fixed array inside the library instead of workspace memory.  The
test runs a cached bf16 layer step through the regular C-ABI call, then feeds
the same compact queries and caches to the allocation-free call twice in a row
and compares both outputs with the regular call's attention output and with
the oracle's attention on the same Q, K^c and V^c, within the bf16 tolerance
the other parity tests use; the device error word stays clear.  A call too
large for the fixed scratch to hold its key splits runs with fewer splits
(here none) and still matches the oracle.

Named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth
from spa_testutil import LayerPair, assert_close, np64

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")

SHAPE = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)


def _oracle_attention(q, kc, vc, B, k, N, nh, hd):
    """O.attention per sequence on the GPU's own compact Q and caches."""
    q, kc, vc = np64(q), np64(kc), np64(vc)
    out = []
    for b in range(B):
        out.append(O.attention(q[b * k:(b + 1) * k].reshape(k, nh, hd), kc[b].reshape(N, nh, hd),
                               vc[b].reshape(N, nh, hd)))
    return np.concatenate(out)


def test_noalloc_attention_matches_layer_step_twice():
    B, N, k = 2, 512, 64
    lp = LayerPair(spa, SHAPE, seed=71, dtype=spa.SPA_BF16, max_B=B, max_N=N, std=0.05)
    H = synth.hidden_states(B, N, SHAPE.d, seed=72, bf16=True)
    H2, _ = synth.drift_rows(H, 0.2, 0.5, seed=73, bf16=True)
    cache = lp.cache(B, N)
    spa.spa_full_block(lp.layer, lp.to_dev(H), cache, True)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    spa.spa_layer_step(lp.layer, lp.to_dev(H2), cache, k, idx)
    lp.ws.check()
    q = lp.ws.view("q", (B * k, SHAPE.d), torch.bfloat16).clone()
    o_ref = lp.ws.view("o", (B * k, SHAPE.d), torch.bfloat16).clone()
    o_oracle = _oracle_attention(q, cache.k, cache.v, B, k, N, SHAPE.n_heads, SHAPE.head_dim)
    for _ in range(2):
        out = torch.full((B * k, SHAPE.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        spa.spa_attention_noalloc(q, cache.k, cache.v, out, B, k, N, SHAPE.n_heads, SHAPE.head_dim)
        assert spa.spa_attention_noalloc_status() == 0
        assert_close(out, np64(o_ref), True, "allocation-free attention vs the workspace path")
        assert_close(out, o_oracle, True, "allocation-free attention vs the oracle")


def test_noalloc_attention_beyond_split_scratch_runs_unsplit():
    # B * n_heads * ceil(k / 128) = 16 * 2 * 8 = 256 query tiles whose split
    # partials would need B * k * (d + 2 h) = 16 * 1024 * 260 fp32 values, more
    # than the fixed array holds: the call runs with the keys unsplit
    B, N, k, h, hd = 16, 1024, 1024, 2, 128
    d = h * hd
    g = torch.Generator(device="cuda").manual_seed(5)
    q = (torch.randn((B * k, d), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    kc = (torch.randn((B, N, d), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    vc = torch.randn((B, N, d), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.full((B * k, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    spa.spa_attention_noalloc(q, kc, vc, out, B, k, N, h, hd)
    assert spa.spa_attention_noalloc_status() == 0
    rows = np.r_[0:64, 7 * k:7 * k + 64, B * k - 64:B * k]   # sampled query rows of three sequences
    ref = []
    for b in (0, 7, B - 1):
        qb = np64(q[b * k:b * k + 64] if b < B - 1 else q[B * k - 64:B * k])
        ref.append(O.attention(qb.reshape(64, h, hd), np64(kc[b]).reshape(N, h, hd),
                               np64(vc[b]).reshape(N, h, hd)))
    assert_close(out[torch.from_numpy(rows).cuda()], np.concatenate(ref), True, "unsplit allocation-free attention")


def test_noalloc_attention_rejects_bad_calls():
    buf = torch.zeros((1, 64, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_attention_noalloc(buf, buf, buf, buf, 1, 8, 64, 2, 64)
    assert ei.value.status == -5                       # head_dim != 128
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_attention_noalloc(buf, buf, buf, buf, 1, 65, 64, 2, 128)
    assert ei.value.status == -2                       # k > N
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_attention_noalloc(buf, buf, buf, buf, 70000, 1, 1, 2, 128)
    assert ei.value.status == -2                       # B beyond the launch grid
    torch.cuda.synchronize()
    assert spa.spa_attention_noalloc_status() == 0

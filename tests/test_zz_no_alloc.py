"""GPU test of the allocation-free attention entry point (spa_attention_noalloc).

Callers that may not allocate device memory (custom memory managers and
allocator hooks, hosts with a fixed memory budget, loops where an allocation's
implicit synchronisation is not allowed) use this variant: its split-over-keys
scratch is a fixed array inside the library instead of workspace memory.  The
test runs a cached bf16 layer step through the regular C-ABI call, then feeds
the same compact queries and caches to the allocation-free call twice in a row
and compares both outputs with the regular call's attention output, within
the bf16 tolerance the other parity tests use.  It also checks that an
oversized call is refused before anything is launched.

Named so that pytest collects it last."""
import numpy as np
import pytest
import torch

from adaptive_hidden_state_b200 import synth
from spa_testutil import LayerPair, assert_close, np64

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")

SHAPE = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)


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
    for _ in range(2):
        out = torch.full((B * k, SHAPE.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        spa.spa_attention_noalloc(q, cache.k, cache.v, out, B, k, N, SHAPE.n_heads, SHAPE.head_dim)
        torch.cuda.synchronize()
        assert_close(out, np64(o_ref), True, "allocation-free attention")


def test_noalloc_attention_rejects_oversized_calls():
    d, h = 256, 2
    buf = torch.zeros((1, 64, d), dtype=torch.bfloat16, device="cuda")
    # B * k * (d + 2h) fp32 partials beyond the fixed 2 Mi-float scratch
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_attention_noalloc(buf, buf, buf, buf, 16, 1024, 1024, h, 128)
    assert ei.value.status == -2
    assert "scratch" in str(ei.value)
    with pytest.raises(spa.SpaError) as ei:
        spa.spa_attention_noalloc(buf, buf, buf, buf, 1, 8, 64, h, 64)
    assert ei.value.status == -5
    torch.cuda.synchronize()

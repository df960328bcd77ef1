"""GPU parity on points of the single-layer sweep at the LLaDA-8B layer shape
(d=4096, 32x128 heads, F=12288, bf16, batch 1): proxy ranks r in {64, 128,
256, 512} and r = d = 4096 (the full-d Value identifier: W_r = Lambda V^T at
full rank scores every token exactly like its value vector W_v h), cache
lengths N in {256, 512, 1024, 4096}, budgets rho in {0.1, 0.16, 0.25, 0.5,
1.0}, inputs N(0, 1) with 5% of the rows drifted by N(0, 0.3) after the
rho = 1 fill.  W_v has the i^-0.8 power-law spectrum and W_r is its exact
rank-r proxy.  r > 256 takes the wide-proxy path (raw proxy tiles, then a
per-row norm and score).  The Query and Key identifiers of the pages'
identifier comparison are the same machinery with W_r = W_q or W_k (r = d;
RoPE rotates a token's query and key by its own position, so their drift
cosines are the pre-RoPE ones).

- Each cached point is compared with the oracle on the same inputs and
  caches (index set, Q, O, H1, A, rewritten cache rows; other rows
  unchanged).  N = 4096 takes the unfused select (more than 2048 scores),
  and k = 410 > 256 tokens the tiled GEMMs.
- At rho = 1 the cached step must equal the rho = 1 full recompute: every
  row is selected, and K^c, V^c, H^c come out bit-identical to
  spa_full_block's on the same input.
"""
import numpy as np
import pytest
import torch

from adaptive_hidden_state_b200 import synth
from spa_testutil import check_layer_step, snapshot_cache

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")

D, NH, HD, F = 4096, 32, 128, 12288


def _layer(r, N, seed, identifier="value"):
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(seed)

    def randn(shape, std):
        return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    def haar(n):
        q, rr = torch.linalg.qr(torch.randn((n, n), generator=g, device=dev, dtype=torch.float32))
        return q * torch.sign(torch.diagonal(rr))[None, :]

    sigma = torch.arange(1, D + 1, device=dev, dtype=torch.float32) ** -0.8
    U, Vm = haar(D), haar(D)
    wv = ((U * sigma[None, :]) @ Vm.T).to(torch.bfloat16)
    w_r = (sigma[:r, None] * Vm[:, :r].T).float().cpu()
    ones = torch.ones(D, device=dev, dtype=torch.bfloat16)
    w = {"wq": randn((D, D), .02), "wk": randn((D, D), .02), "wv": wv, "wo": randn((D, D), .02),
         "w_gate": randn((F, D), .02), "w_up": randn((F, D), .02), "w_down": randn((D, F), .02),
         "attn_norm": ones, "ffn_norm": ones}
    if identifier != "value":  # the Query / Key identifiers: the projection itself as the proxy
        w_r = w["wq" if identifier == "query" else "wk"].float().cpu()
    desc = spa.LayerDesc(d=D, n_heads=NH, head_dim=HD, ffn=F, r=r, dtype=spa.SPA_BF16, rms_eps=1e-5,
                         rope_theta=1e4)
    ws = spa.Workspace(desc, 1, N)
    layer = spa.Layer(desc, w, ws, w_r_host=w_r)
    if identifier != "value":
        assert torch.equal(layer.proxy_weights(), w_r)  # bf16 values, stored exactly
    return layer, w, ws


def _inputs(N, seed):
    H = synth.hidden_states(1, N, D, seed=seed, bf16=True)
    H2, _ = synth.drift_rows(H, 0.05, 0.3, seed=seed + 1, bf16=True)
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)
    return to(H), to(H2)


@pytest.mark.parametrize("r,N,rho,identifier", [(64, 256, 0.5, "value"), (256, 1024, 0.16, "value"),
                                              (128, 4096, 0.1, "value"), (512, 1024, 0.25, "value"),
                                              (4096, 512, 0.25, "value"), (4096, 512, 0.25, "key"),
                                              (4096, 512, 0.25, "query")])
def test_sweep_point_cached_step(r, N, rho, identifier):
    layer, w, ws = _layer(r, N, seed=900 + r + N, identifier=identifier)
    H, H2 = _inputs(N, seed=N + r)
    k = spa.spa_budget_k(N, rho)
    cache = spa.Cache(1, N, D, r, spa.SPA_BF16)
    spa.spa_full_block(layer, H, cache, True)
    ws.check()
    snap = snapshot_cache(cache)
    idx = torch.empty((1, k), dtype=torch.int32, device="cuda")
    spa.spa_layer_step(layer, H2, cache, k, idx)
    ws.check()
    check_layer_step(spa, layer, w, H2.clone(), snap, cache, k, idx, ws, (0,),
                     f"r={r} N={N} rho={rho} {identifier}")


def test_sweep_rho1_cached_step_equals_full_recompute():
    r, N = 128, 2048
    layer, w, ws = _layer(r, N, seed=77)
    H, H2 = _inputs(N, seed=78)
    caches = []
    for cached in (True, False):
        cache = spa.Cache(1, N, D, r, spa.SPA_BF16)
        spa.spa_full_block(layer, H, cache, True)
        if cached:
            idx = torch.empty((1, N), dtype=torch.int32, device="cuda")
            spa.spa_layer_step(layer, H2, cache, N, idx)
            assert torch.equal(idx[0].cpu(), torch.arange(N, dtype=torch.int32))
        else:
            spa.spa_full_block(layer, H2, cache, False)
        ws.check()
        caches.append(cache)
    for name in ("k", "v", "h"):
        assert torch.equal(getattr(caches[0], name), getattr(caches[1], name)), name

"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: the 32-layer LLaDA-8B-shaped bf16 decode loop (d=4096,
32x128 heads, F=12288, vocab 126464, r=128) at B=1, N=1024 (256 prompt ids,
2 unmaskings per step) and at B=8, N=2048 (512 prompt ids, 4 unmaskings per
step), piecewise-Gaussian budget rho_p=0.25, l_p=12, rho_1=rho_L=0.06, with
seeded random weights of that shape (W_v with the i^-0.8 power-law spectrum).

The oracle cannot run whole steps at these sizes, so the checks are sampled
and by property:
- one graph-replayed cached step with the incremental proxy (only rows whose
  layer input changed are projected) equals the same step launched directly
  with the plain proxy, bit for bit (all 32 layers' caches, h0 and the ids);
- at a few layers of a later step (the first, the widest k = 256 / 512, the
  last) and a few sequences, the layer's input and caches are copied before
  the layer runs, and the oracle's proxy scores, top-k and cached block on
  them are compared with the GPU's: the index set (exact, or valid within the
  score margin), Q, O, H1, A and the rewritten K^c, V^c, H^c, P^c rows, with
  the bf16 tolerance; the rows outside I stay bit-identical.
- the full-vocabulary LM head of that step (argmax ids and their softmax
  probabilities through the confidence pass) against the oracle's logits on
  the GPU's final-layer rows.
Layers run through spa_layer_step, the call spa_decode_step makes."""
import gc

import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth
from spa_testutil import check_layer_step, snapshot_cache

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")

D, NH, HD, F, R, VOCAB, L = 4096, 32, 128, 12288, 128, 126464, 32
RHO = dict(rho_p=0.25, l_p=12, rho_1=0.06, rho_L=0.06)


def _build(B, N, seed):
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(seed)

    def randn(shape, std):
        return (torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    def haar(n):
        q, rr = torch.linalg.qr(torch.randn((n, n), generator=g, device=dev, dtype=torch.float32))
        return q * torch.sign(torch.diagonal(rr))[None, :]

    sigma = torch.arange(1, D + 1, device=dev, dtype=torch.float32) ** -0.8
    desc = spa.LayerDesc(d=D, n_heads=NH, head_dim=HD, ffn=F, r=R, dtype=spa.SPA_BF16,
                         rms_eps=1e-5, rope_theta=1e4)
    ws = spa.Workspace(desc, B, N)
    ones = torch.ones(D, device=dev, dtype=torch.bfloat16)
    layers, caches, weights = [], [], []
    for _ in range(L):
        U, Vm = haar(D), haar(D)
        wv = ((U * sigma[None, :]) @ Vm.T).to(torch.bfloat16)
        w_r = (sigma[:R, None] * Vm[:, :R].T).float().cpu()
        del U, Vm
        w = {"wq": randn((D, D), .02), "wk": randn((D, D), .02), "wv": wv, "wo": randn((D, D), .02),
             "w_gate": randn((F, D), .02), "w_up": randn((F, D), .02), "w_down": randn((D, F), .02),
             "attn_norm": ones, "ffn_norm": ones}
        layers.append(spa.Layer(desc, w, ws, w_r_host=w_r))
        weights.append(w)
        caches.append(spa.Cache(B, N, D, R, spa.SPA_BF16))
    embed = randn((VOCAB, D), 1.0)
    lm_head = randn((VOCAB, D), .02)
    h0 = torch.zeros((B, N, D), device=dev, dtype=torch.bfloat16)
    model = spa.Model(layers, caches, h0, embed, ones, lm_head, VOCAB, B, N, RHO["rho_p"], RHO["l_p"],
                      RHO["rho_1"], RHO["rho_L"])
    return model, ws, layers, caches, weights, (embed, lm_head, h0, ones)


def _check_lm_head(model, caches, lm_head, pos, u, B, tok_step):
    """The full-vocabulary LM head (126464 x 4096, the tensor-core argmax
    GEMM with per-tile sums of exp) on the GPU's final-layer rows at pos,
    through the confidence pass, against the oracle's logits on the same rows
    (the normalised rows rounded to bf16, the bf16 model's rounding point):
    every argmax id whose top-2 gap is clear, every softmax probability of the
    argmax within 1e-3 relative, and the step's ids equal to the pass's.  The
    oracle runs over row blocks of the LM head (logits of different vocabulary
    rows are independent), which keeps its fp64 copy small."""
    tok = torch.empty((B, u), dtype=torch.int32, device="cuda")
    conf = torch.empty((B, u), dtype=torch.float32, device="cuda")
    spa.spa_decode_confidence(model, pos, u, tok, conf)
    torch.cuda.synchronize()
    p = pos.cpu().numpy()
    h = np.stack([caches[-1].h[b][pos[b].long()].float().cpu().numpy() for b in range(B)]).astype(np.float64)
    ones = np.ones(D)
    parts = []
    for v0 in range(0, VOCAB, 16384):
        chunk = lm_head[v0:v0 + 16384].float().cpu().numpy()
        om = O.OracleModel(layers=[], embed=None, final_norm=ones, lm_head=chunk, eps=1e-5)
        parts.append(O.lm_head_argmax(om, h, bf16_input=True)[1])
    logits = np.concatenate(parts, axis=-1)
    got_tok, got_conf = tok.cpu().numpy(), conf.cpu().numpy().astype(np.float64)
    assert np.array_equal(got_tok, tok_step.cpu().numpy()), "confidence pass ids differ from the step's"
    for b in range(B):
        ids_ref, conf_ref = O.confidence(logits[b])
        assert np.max(np.abs(got_conf[b] - conf_ref) / conf_ref) < 1e-3, f"seq {b} confidence"
        for j in range(u):
            top2 = np.sort(logits[b, j])[-2:]
            if top2[1] - top2[0] > 1e-4 * max(1.0, abs(top2[1])):
                assert got_tok[b, j] == ids_ref[j], f"seq {b} position {p[b, j]} argmax"


def _run(B, N, n_prompt, u, sample_layers, seqs, check_graph):
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        _run_on_stream(B, N, n_prompt, u, sample_layers, seqs, check_graph)
    stream.synchronize()
    gc.collect()
    torch.cuda.empty_cache()


def _run_on_stream(B, N, n_prompt, u, sample_layers, seqs, check_graph):
    model, ws, layers, caches, weights, keep = _build(B, N, seed=1234 + B)
    steps = 4
    job = synth.decode_inputs(B=B, N=N, n_prompt=n_prompt, vocab=VOCAB, steps=steps, u=u, seed=77 + B)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    pos = [torch.from_numpy(p.astype(np.int32)).cuda() for p in job.positions]
    tok_out = torch.empty((steps, B, u), dtype=torch.int32, device="cuda")
    model.embed_tokens(toks)
    if check_graph:
        model.set_incremental_proxy(True)
    spa.spa_decode_step(model, pos[0], None, u, 1, tok_out[0])
    spa.spa_decode_step(model, pos[1], None, u, 0, tok_out[1])
    ws.check()
    h0 = keep[2]

    if check_graph:
        # the graph-replayed step against the same step launched directly
        state = [h0.clone()] + [t.clone() for c in caches for t in (c.k, c.v, c.h, c.p)]
        pos_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        tok_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        spa.spa_decode_graph_capture(model, pos_buf, None, u, tok_buf)
        pos_buf.copy_(pos[2])
        spa.spa_decode_graph_launch(model)
        torch.cuda.synchronize()
        ws.check()
        graph_out = [tok_buf.clone(), h0.clone()] + [t.clone() for c in caches for t in (c.k, c.v, c.h, c.p)]
        h0.copy_(state[0])
        for i, c in enumerate(caches):
            for j, t in enumerate((c.k, c.v, c.h, c.p)):
                t.copy_(state[1 + 4 * i + j])
        del state
        model.set_incremental_proxy(False)
        spa.spa_decode_step(model, pos[2], None, u, 0, tok_out[2])
        ws.check()
        direct = [tok_out[2], h0] + [t for c in caches for t in (c.k, c.v, c.h, c.p)]
        for i, (a, b) in enumerate(zip(graph_out, direct)):
            assert torch.equal(a, b), f"graph replay differs from direct launch (tensor {i})"
        del graph_out
    else:
        spa.spa_decode_step(model, pos[2], None, u, 0, tok_out[2])
        ws.check()
    torch.cuda.synchronize()
    _check_lm_head(model, caches, keep[1], pos[2], u, B, tok_out[2])

    # step 3, layer by layer, with sampled oracle checks
    for l in range(L):
        H = h0 if l == 0 else caches[l - 1].h
        k = model.k[l]
        Ik = torch.empty((B, k), dtype=torch.int32, device="cuda")
        if l in sample_layers:
            H_in = H.clone()
            snap = snapshot_cache(caches[l])
            spa.spa_layer_step(layers[l], H, caches[l], k, Ik)
            ws.check()
            torch.cuda.synchronize()
            check_layer_step(spa, layers[l], weights[l], H_in, snap, caches[l], k, Ik, ws, seqs, f"layer {l}")
            del H_in, snap
            gc.collect()
        else:
            spa.spa_layer_step(layers[l], H, caches[l], k, Ik)
    ws.check()


def test_llada_decode_full_size_b1_n1024():
    _run(B=1, N=1024, n_prompt=256, u=2, sample_layers=(0, 11, 31), seqs=(0,), check_graph=True)


def test_llada_decode_full_size_b8_n2048():
    # B*k reaches 4096 tokens at the widest layers: the tiled GEMM path
    _run(B=8, N=2048, n_prompt=512, u=4, sample_layers=(0, 11), seqs=(0, 5), check_graph=False)

"""GPU parity of the decode loop (through the C ABI) against the oracle on the
tiny fp32 model: 2 layers, d=256, 4x64 heads, F=688, vocab 1024, N=64 with
half the positions masked, r=16, uniform rho=0.25 (k=16), 8 steps of 2
unmaskings, step 0 the rho=1 fill.  Teacher-forced so that one argmax near a
tie cannot fork the two runs."""
import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth
from spa_testutil import LayerPair, assert_close, assert_index_set, np64

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")


def _tiny_model(dtype, shape, L, vocab, B, N, rho, seed, N_max=None):
    bf = dtype == spa.SPA_BF16
    rng = np.random.default_rng(seed)
    embed = rng.standard_normal((vocab, shape.d)).astype(np.float32)
    lm = (rng.standard_normal((vocab, shape.d)) * 0.02).astype(np.float32)
    if bf:
        embed, lm = synth.bf16_round(embed), synth.bf16_round(lm)
    fnorm = np.ones(shape.d, np.float32)
    lps, ws = [], None
    for l in range(L):
        lp = LayerPair(spa, shape, seed=seed + 1 + l, dtype=dtype, max_B=B, max_N=N, ws=ws)
        ws = lp.ws
        lps.append(lp)
    tdt = spa.torch_dtype(dtype)
    dev = lambda a: torch.from_numpy(a).to("cuda", tdt)
    caches = [lp.cache(B, N) for lp in lps]
    h0 = torch.zeros((B, N, shape.d), dtype=tdt, device="cuda")
    e_d, f_d, l_d = dev(embed), dev(fnorm), dev(lm)
    model = spa.Model([lp.layer for lp in lps], caches, h0, e_d, f_d, l_d, vocab, B, N,
                      rho_p=rho, l_p=1, rho_1=rho, rho_L=rho)
    om = O.OracleModel(layers=[lp.ol for lp in lps], embed=embed, final_norm=fnorm, lm_head=lm,
                       eps=shape.rms_eps)
    keep = (e_d, f_d, l_d)
    return model, om, lps, caches, h0, keep


def _check_index_sets(model, ref, B, what):
    """Every layer's index set of the cached step the GPU has just run against
    the oracle's (exact, or valid within the score margin)."""
    for l in range(len(model.k)):
        I_gpu = model.index_set(l).cpu().numpy()
        for b in range(B):
            assert_index_set(I_gpu[b], ref["s"][l][b], model.k[l], ref["I"][l][b], f"{what} layer {l} seq {b} I")


def _check_lm_head(model, om, caches, pos, u, B, bf16, tok_step, what):
    """The LM head on the GPU's own final-layer rows at pos, through the
    confidence pass (the argmax GEMM epilogue that also keeps per-tile sums
    of exp), against the oracle's logits on the same rows: the argmax ids
    where the oracle's top-2 gap is clear, every softmax probability of the
    argmax within 1e-3 relative, and the step's own ids equal to these."""
    tok = torch.empty((B, u), dtype=torch.int32, device="cuda")
    conf = torch.empty((B, u), dtype=torch.float32, device="cuda")
    spa.spa_decode_confidence(model, pos, u, tok, conf)
    torch.cuda.synchronize()
    p = pos.cpu().numpy()
    hrows = np.stack([np64(caches[-1].h[b])[p[b]] for b in range(B)])
    _, logits = O.lm_head_argmax(om, hrows, bf16_input=bf16)
    got_tok, got_conf = tok.cpu().numpy(), conf.cpu().numpy().astype(np.float64)
    assert np.array_equal(got_tok, tok_step.cpu().numpy()), what + ": confidence pass ids differ from the step's"
    for b in range(B):
        ids_ref, conf_ref = O.confidence(logits[b])
        assert np.max(np.abs(got_conf[b] - conf_ref) / conf_ref) < 1e-3, f"{what} seq {b} confidence"
        for j in range(u):
            top2 = np.sort(logits[b, j])[-2:]
            if top2[1] - top2[0] > 1e-4 * max(1.0, abs(top2[1])):
                assert got_tok[b, j] == ids_ref[j], f"{what} seq {b} position {p[b, j]} argmax"


@pytest.mark.parametrize("inc", [False, True])
def test_tiny_decode_loop_teacher_forced(inc):
    """Teacher-forced decode steps against the oracle, with the plain proxy
    (every row projected at every layer) and the incremental proxy (only rows
    whose layer input changed): ids, index sets of every layer, K^c, H^c, h0."""
    B, N, vocab, steps, u = 1, 64, 1024, 8, 2
    model, om, lps, caches, h0, keep = _tiny_model(spa.SPA_F32, synth.TINY_LAYER, 2, vocab, B, N,
                                                   0.25, seed=0)
    model.set_incremental_proxy(inc)
    assert model.k == [16, 16]
    job = synth.decode_inputs(B=B, N=N, n_prompt=32, vocab=vocab, steps=steps, u=u, seed=5)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    model.embed_tokens(toks)
    state = O.init_decode_state(om, job.tokens)
    tok_out = torch.empty((B, u), dtype=torch.int32, device="cuda")
    for t in range(steps):
        pos = torch.from_numpy(job.positions[t].astype(np.int32)).cuda()
        forced = torch.from_numpy(job.forced[t].astype(np.int32)).cuda()
        spa.spa_decode_step(model, pos, forced, u, 1 if t == 0 else 0, tok_out)
        lps[0].ws.check()
        ref = O.decode_step(om, state, job.positions[t], model.k, full=(t == 0),
                            forced=job.forced[t])
        if t > 0:
            _check_index_sets(model, ref, B, f"step {t}")
        _check_lm_head(model, om, caches, pos, u, B, False, tok_out, f"step {t}")
        # argmax ids: equal wherever the oracle's top-2 logit gap is clear
        got = tok_out.cpu().numpy()
        lg = ref["logits"]
        for b in range(B):
            for j in range(u):
                top2 = np.sort(lg[b, j])[-2:]
                if top2[1] - top2[0] > 1e-3 * max(1.0, abs(top2[1])):
                    assert got[b, j] == ref["argmax"][b, j]
                else:
                    assert lg[b, j, got[b, j]] >= top2[1] - 1e-3
        for l, lp in enumerate(lps):
            c = caches[l]
            assert_close(c.h, np.stack([state.caches[l][b].H_c for b in range(B)]), False,
                         f"step {t} layer {l} H^c")
            assert_close(c.k, np.stack([state.caches[l][b].K_c for b in range(B)]), False,
                         f"step {t} layer {l} K^c")
        assert_close(h0, state.H0, False, f"step {t} h0")


def test_tiny_decode_full_k_matches_vanilla():
    # with k = N at every layer the cached loop is vanilla decoding
    B, N, vocab, u = 2, 32, 256, 2
    model, om, lps, caches, h0, keep = _tiny_model(spa.SPA_F32, synth.TINY_LAYER, 2, vocab, B, N,
                                                   1.0, seed=7)
    job = synth.decode_inputs(B=B, N=N, n_prompt=8, vocab=vocab, steps=3, u=u, seed=8)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    model.embed_tokens(toks)
    out_cached = []
    tok_out = torch.empty((B, u), dtype=torch.int32, device="cuda")
    for t in range(3):
        pos = torch.from_numpy(job.positions[t].astype(np.int32)).cuda()
        forced = torch.from_numpy(job.forced[t].astype(np.int32)).cuda()
        spa.spa_decode_step(model, pos, forced, u, 1 if t == 0 else 0, tok_out)
        out_cached.append(caches[-1].h.clone())
    model.embed_tokens(toks)
    for t in range(3):
        pos = torch.from_numpy(job.positions[t].astype(np.int32)).cuda()
        forced = torch.from_numpy(job.forced[t].astype(np.int32)).cuda()
        spa.spa_decode_step(model, pos, forced, u, 2, tok_out)
        assert_close(caches[-1].h, np64(out_cached[t]), False, f"vanilla step {t}")
    lps[0].ws.check()


SMALL_BF16 = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)


@pytest.mark.parametrize("inc", [False, True])
def test_bf16_decode_loop_and_graph_replay(inc):
    """bf16 model (2 layers of d=256, vocab 8192 so the LM head uses wide
    weight tiles), plain or incremental proxy: teacher-forced steps against
    the oracle (index sets of every layer, H^c, and the tensor-core LM head
    with its argmax and softmax-probability epilogue on the GPU's final rows),
    then the same steps replayed from a captured CUDA graph must reproduce the
    directly launched steps bit for bit."""
    B, N, vocab, steps, u = 2, 96, 8192, 4, 2
    model, om, lps, caches, h0, keep = _tiny_model(spa.SPA_BF16, SMALL_BF16, 2, vocab, B, N,
                                                   0.3, seed=50)
    model.set_incremental_proxy(inc)
    job = synth.decode_inputs(B=B, N=N, n_prompt=32, vocab=vocab, steps=steps, u=u, seed=51)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    model.embed_tokens(toks)
    state = O.init_decode_state(om, job.tokens)
    tok_out = torch.empty((steps, B, u), dtype=torch.int32, device="cuda")
    direct_h = []
    for t in range(steps):
        pos = torch.from_numpy(job.positions[t].astype(np.int32)).cuda()
        forced = torch.from_numpy(job.forced[t].astype(np.int32)).cuda()
        spa.spa_decode_step(model, pos, forced, u, 1 if t == 0 else 0, tok_out[t])
        lps[0].ws.check()
        ref = O.decode_step(om, state, job.positions[t], model.k, full=(t == 0),
                            forced=job.forced[t])
        if t > 0:
            _check_index_sets(model, ref, B, f"bf16 step {t}")
        _check_lm_head(model, om, caches, pos, u, B, True, tok_out[t], f"bf16 step {t}")
        got = tok_out[t].cpu().numpy()
        lg = ref["logits"]
        for b in range(B):
            for j in range(u):
                top2 = np.sort(lg[b, j])[-2:]
                if top2[1] - top2[0] > 2e-2 * max(1.0, abs(top2[1])):
                    assert got[b, j] == ref["argmax"][b, j]
        for l in range(2):
            assert_close(caches[l].h, np.stack([state.caches[l][b].H_c for b in range(B)]), True,
                         f"bf16 step {t} layer {l} H^c")
        direct_h.append(caches[-1].h.clone())
    # replay steps 1.. from a captured graph after redoing step 0 directly
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        pos_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        tin_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        tout_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        model.embed_tokens(toks)
        pos0 = torch.from_numpy(job.positions[0].astype(np.int32)).cuda()
        f0 = torch.from_numpy(job.forced[0].astype(np.int32)).cuda()
        spa.spa_decode_step(model, pos0, f0, u, 1, tout_buf)
        n0 = spa.spa_launch_count()
        spa.spa_decode_graph_capture(model, pos_buf, tin_buf, u, tout_buf)
        # the step's kernels, counted by the library and found in the graph: per layer
        # proxy, select, QKV, attention, O-proj (+ folded FFN norm), gate/up, down; then
        # the written tokens' embeddings, the final norm, the LM head and its argmax
        nodes = spa.spa_decode_graph_kernel_nodes(model)
        assert nodes == spa.spa_launch_count() - n0 == 7 * 2 + 4
        for t in range(1, steps):
            pos_buf.copy_(torch.from_numpy(job.positions[t].astype(np.int32)).cuda())
            tin_buf.copy_(torch.from_numpy(job.forced[t].astype(np.int32)).cuda())
            spa.spa_decode_graph_launch(model)
            assert torch.equal(caches[-1].h, direct_h[t])
            assert torch.equal(tout_buf, tok_out[t])
    stream.synchronize()
    lps[0].ws.check()


def _state(model, caches, h0, tok):
    return [tok.clone(), h0.clone()] + [t.clone() for c in caches for t in (c.k, c.v, c.h, c.p)]


@pytest.mark.parametrize("bf16", [False, True])
def test_incremental_proxy_decode_is_bit_identical(bf16):
    """The incremental proxy (only rows whose layer input changed are
    projected again) against the plain path, from the same start, over cached
    steps with the argmax ids fed back (no teacher forcing), a vanilla step in
    between (the state goes stale and is rebuilt), a re-fill, and graph
    replays of the incremental step: ids, h0 and every cache bit for bit."""
    dtype = spa.SPA_BF16 if bf16 else spa.SPA_F32
    shape = SMALL_BF16 if bf16 else synth.TINY_LAYER
    B, N, vocab, u, L = 2, 96, 1024, 2, 3
    model, om, lps, caches, h0, keep = _tiny_model(dtype, shape, L, vocab, B, N, 0.2, seed=90 + bf16,
                                                   )
    job = synth.decode_inputs(B=B, N=N, n_prompt=24, vocab=vocab, steps=10, u=u, seed=91)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    pos = [torch.from_numpy(p.astype(np.int32)).cuda() for p in job.positions]
    # step t: 0 fill, 1-3 cached, 4 vanilla, 5-6 cached, 7 fill, 8-9 cached (graph in the second run)
    full = [1, 0, 0, 0, 2, 0, 0, 1, 0, 0]
    stream = torch.cuda.Stream()
    runs = []
    with torch.cuda.stream(stream):
        pos_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        tok_buf = torch.empty((B, u), dtype=torch.int32, device="cuda")
        for inc in (False, True):
            model.set_incremental_proxy(inc)
            model.embed_tokens(toks)
            out = []
            for t in range(10):
                if inc and t == 8:
                    spa.spa_decode_graph_capture(model, pos_buf, None, u, tok_buf)
                if inc and t >= 8:
                    pos_buf.copy_(pos[t])
                    spa.spa_decode_graph_launch(model)
                else:
                    spa.spa_decode_step(model, pos[t], None, u, full[t], tok_buf)
                lps[0].ws.check()
                out.append(_state(model, caches, h0, tok_buf))
            runs.append(out)
    stream.synchronize()
    for t in range(10):
        for i, (a, b) in enumerate(zip(runs[0][t], runs[1][t])):
            assert torch.equal(a, b), f"step {t}: tensor {i} differs between the plain and incremental proxy"


def test_confidence_parallel_unmasking_tiny_fp32():
    """Confidence-based parallel unmasking through the split step
    (spa_decode_layers, spa_decode_confidence at every still-masked
    position, spa_model_write_tokens of the chosen ones) against the oracle
    on the tiny fp32 model: argmax ids where the top-2 gap is clear, softmax
    probabilities, and after four steps h0 and every cache.  Both sides
    unmask the positions the threshold rule picks from the GPU's
    confidences, with tau at the 70th percentile of the step's confidences
    (random weights give tiny probabilities, so a fixed tau would pick one)."""
    B, N, vocab = 1, 64, 1024
    model, om, lps, caches, h0, keep = _tiny_model(spa.SPA_F32, synth.TINY_LAYER, 2, vocab, B, N,
                                                   0.25, seed=70)
    job = synth.decode_inputs(B=B, N=N, n_prompt=24, vocab=vocab, steps=1, u=2, seed=71)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    model.embed_tokens(toks)
    state = O.init_decode_state(om, job.tokens)
    emb = np.asarray(om.embed, dtype=np.float64)
    masked = [i for i in range(N) if job.tokens[0, i] == job.mask_id]
    for t in range(4):
        full = t == 0
        spa.spa_decode_layers(model, 1 if full else 0)
        H = state.H0[0]
        for l, layer in enumerate(om.layers):
            if full:
                state.caches[l] = [O.full_block(layer, H)[0]]
            else:
                O.layer_step(layer, H, state.caches[l][0], model.k[l])
            H = state.caches[l][0].H_c
        m = len(masked)
        pos = torch.tensor([masked], dtype=torch.int32, device="cuda")
        tok = torch.empty((1, m), dtype=torch.int32, device="cuda")
        conf = torch.empty((1, m), dtype=torch.float32, device="cuda")
        spa.spa_decode_confidence(model, pos, m, tok, conf)
        lps[0].ws.check()
        logits = O.lm_head_argmax(om, H[masked][None])[1][0]
        ids_ref, conf_ref = O.confidence(logits)
        got_ids, got_conf = tok.cpu().numpy()[0], conf.cpu().numpy()[0].astype(np.float64)
        assert np.max(np.abs(got_conf - conf_ref) / conf_ref) < 1e-3, f"step {t} confidence"
        for j in range(m):
            top2 = np.sort(logits[j])[-2:]
            if top2[1] - top2[0] > 1e-3 * max(1.0, abs(top2[1])):
                assert got_ids[j] == ids_ref[j], f"step {t} position {masked[j]}"
        chosen = O.confident_positions(got_conf, float(np.quantile(got_conf, 0.7)))
        sel_pos = [masked[j] for j in chosen]
        sel_tok = got_ids[chosen]
        spa.spa_model_write_tokens(model, torch.tensor(np.array([sel_pos]), dtype=torch.int32, device="cuda"),
                                   torch.tensor(np.array([sel_tok]), dtype=torch.int32, device="cuda"),
                                   len(sel_pos))
        state.tokens[0, sel_pos] = sel_tok
        state.H0[0, sel_pos] = emb[sel_tok]
        masked = [p for p in masked if p not in set(sel_pos)]
    spa.spa_decode_layers(model, 0)
    H = state.H0[0]
    for l, layer in enumerate(om.layers):
        O.layer_step(layer, H, state.caches[l][0], model.k[l])
        H = state.caches[l][0].H_c
    torch.cuda.synchronize()
    assert_close(h0, state.H0, False, "h0")
    for l in range(2):
        assert_close(caches[l].h, np.stack([state.caches[l][0].H_c]), False, f"layer {l} H^c")
        assert_close(caches[l].k, np.stack([state.caches[l][0].K_c]), False, f"layer {l} K^c")


@pytest.mark.parametrize("inc", [False, True])
def test_split_decode_step_equals_decode_step_bf16(inc):
    """spa_decode_layers + spa_decode_confidence + spa_model_write_tokens at
    the step's positions reproduce spa_decode_step bit for bit (ids, h0,
    caches), with the plain and the incremental proxy; the confidence pass's
    ids are the step's argmax ids."""
    B, N, vocab, u = 2, 96, 8192, 2
    model, om, lps, caches, h0, keep = _tiny_model(spa.SPA_BF16, SMALL_BF16, 2, vocab, B, N, 0.3, seed=80)
    model.set_incremental_proxy(inc)
    job = synth.decode_inputs(B=B, N=N, n_prompt=32, vocab=vocab, steps=4, u=u, seed=81)
    toks = torch.from_numpy(job.tokens.astype(np.int32)).cuda()
    runs = []
    for split in (False, True):
        model.embed_tokens(toks)
        out = []
        for t in range(4):
            pos = torch.from_numpy(job.positions[t].astype(np.int32)).cuda()
            tok = torch.empty((B, u), dtype=torch.int32, device="cuda")
            if split:
                conf = torch.empty((B, u), dtype=torch.float32, device="cuda")
                spa.spa_decode_layers(model, 1 if t == 0 else 0)
                spa.spa_decode_confidence(model, pos, u, tok, conf)
                assert torch.all((conf > 0) & (conf <= 1))
                spa.spa_model_write_tokens(model, pos, tok, u)
            else:
                spa.spa_decode_step(model, pos, None, u, 1 if t == 0 else 0, tok)
            lps[0].ws.check()
            out.append([tok.clone(), h0.clone()] + [x.clone() for c in caches for x in (c.k, c.v, c.h, c.p)])
        runs.append(out)
    for t in range(4):
        for i, (a, b) in enumerate(zip(runs[0][t], runs[1][t])):
            assert torch.equal(a, b), f"step {t}: tensor {i} differs"

"""CPU tests of the C ABI: the library loads, exports every declared symbol,
and its host-side logic (budget, argument checks, host SVD) agrees with the
oracle.  No GPU work is launched here."""
import ctypes
import math
import os
import re

import numpy as np
import pytest
import torch

import oracle as O
from adaptive_hidden_state_b200 import synth

spa = pytest.importorskip("adaptive_hidden_state_b200.spa",
                          reason="libspa.so not built (python -m adaptive_hidden_state_b200.build)")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(spa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(spa.lib, n), n
    assert sorted(spa.EXPORTS) == names


def test_status_strings():
    for code, name in spa.STATUS.items():
        assert spa.spa_status_string(code) == name
    assert spa.spa_status_string(12345) == "SPA_ERR_UNKNOWN"
    assert spa.spa_version() >= 100


@pytest.mark.parametrize("params", [(32, .25, 12, .06, .06), (32, .25, 12, .03, .1),
                                    (28, .3, 9, .02, .1), (2, .25, 1, .25, .25), (7, .5, 7, .1, .2)])
def test_rho_and_budget_match_oracle(params):
    L, rp, lp, r1, rL = params
    for l in range(1, L + 1):
        a = spa.spa_rho(l, L, rp, lp, r1, rL)
        b = O.rho(l, L, rp, lp, r1, rL)
        assert a == pytest.approx(b, rel=1e-14, abs=0)
        for N in (1, 17, 64, 512, 1024, 2048, 4096, 8192):
            assert spa.spa_budget_k(N, a) == O.budget_k(N, b)


def test_budget_invalid_inputs():
    assert math.isnan(spa.spa_rho(0, 32, .25, 12, .06, .06))
    assert math.isnan(spa.spa_rho(33, 32, .25, 12, .06, .06))
    assert math.isnan(spa.spa_rho(3, 32, -.25, 12, .06, .06))
    assert math.isnan(spa.spa_rho(3, 32, .25, 40, .06, .06))
    assert spa.spa_budget_k(0, 0.5) == -1
    assert spa.spa_budget_k(10, 0.0) == -1
    assert spa.spa_budget_k(10, float("nan")) == -1
    assert spa.spa_budget_k(10, 5.0) == 10
    assert spa.spa_budget_k(10, 1e-12) == 1


@pytest.mark.parametrize("d,r,spectrum", [(64, 8, "power"), (256, 16, "power"),
                                           (192, 40, "power"), (96, 12, "geometric")])
def test_host_svd_matches_oracle(d, r, spectrum):
    rng = np.random.default_rng(d + r)
    spec = None if spectrum == "power" else 1.5 ** -np.arange(d)
    W, *_ = synth.power_law_wv(d, rng, spectrum=spec)
    W = W.astype(np.float32)
    got = spa.spa_singular_proxy_host(torch.from_numpy(W), r).numpy().astype(np.float64)
    ref = O.singular_proxy(W.astype(np.float64), r)
    # rows match up to float32 storage, same sign convention
    err = np.max(np.abs(got - ref), axis=1) / np.max(np.abs(ref), axis=1)
    assert np.all(err < 1e-5), err.max()


def test_host_svd_argument_checks():
    w = torch.zeros((8, 8))
    with pytest.raises(spa.SpaError) as e:
        spa.spa_singular_proxy_host(w, 9)
    assert e.value.status == -2
    assert spa.lib.spa_singular_proxy_host(None, 8, 2, None) == -1


def test_layer_calls_reject_bad_arguments_before_any_launch():
    # every check below fails before the library touches the device
    # a wide bf16 proxy (r > 256) must be a multiple of 4; r > d is a shape error
    bad = spa.LayerDesc(d=4096, n_heads=32, head_dim=128, ffn=12288, r=302, dtype=spa.SPA_BF16,
                        rms_eps=1e-5, rope_theta=1e4)
    h = ctypes.c_void_p()
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 1, 512, ctypes.byref(h)) == -5
    bad.r = 4100
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 1, 512, ctypes.byref(h)) == -2
    bad.r, bad.d = 128, 4000
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 1, 512, ctypes.byref(h)) == -2
    bad.d, bad.dtype = 4096, 7
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 1, 512, ctypes.byref(h)) == -1
    bad.dtype = spa.SPA_BF16
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 1, 9000, ctypes.byref(h)) == -5
    assert spa.lib.spa_workspace_create(ctypes.byref(bad), 0, 512, ctypes.byref(h)) == -2
    assert spa.lib.spa_workspace_create(None, 1, 512, ctypes.byref(h)) == -1
    cache = spa.LayerCacheDesc(0, 0, 0, 0, 1, 8)
    assert spa.lib.spa_proxy_select(None, None, ctypes.byref(cache), 1, None, None, None) == -1
    assert spa.lib.spa_partial_block(None, None, None, 1, ctypes.byref(cache), None) == -1
    assert spa.lib.spa_full_block(None, None, ctypes.byref(cache), 1, None) == -1
    assert spa.lib.spa_decode_step(None, None, None, 1, 0, None, None) == -1
    assert spa.lib.spa_model_layer_k(None, 0) == -1
    assert spa.lib.spa_layer_step(None, None, ctypes.byref(cache), 1, None, None) == -1
    assert spa.lib.spa_decode_layers(None, 0, None) == -1
    assert spa.lib.spa_decode_confidence(None, None, 1, None, None, None) == -1
    assert spa.lib.spa_model_write_tokens(None, None, None, 1, None) == -1
    assert spa.lib.spa_model_set_incremental_proxy(None, 1) == -1
    assert spa.lib.spa_model_embed(None, None, None) == -1
    assert spa.lib.spa_decode_graph_launch(None, None) == -1
    assert "null" in spa.lib.spa_last_error().decode()


def test_host_svd_full_rank_gives_the_value_cosine():
    # r = d (the full-d Value identifier): the host proxy scores every pair of
    # inputs exactly like the value projection itself
    rng = np.random.default_rng(70)
    d = 64
    W, *_ = synth.power_law_wv(d, rng)
    W = W.astype(np.float32)
    Wr = spa.spa_singular_proxy_host(torch.from_numpy(W), d).numpy().astype(np.float64)
    h, h2 = rng.standard_normal((2, 10, d))
    cos = lambda A, x, y: np.sum((x @ A.T) * (y @ A.T), 1) / (
        np.linalg.norm(x @ A.T, axis=1) * np.linalg.norm(y @ A.T, axis=1))
    assert np.max(np.abs(cos(Wr, h, h2) - cos(W.astype(np.float64), h, h2))) < 1e-5

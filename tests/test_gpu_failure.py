"""Failure detection through the C ABI, without faulting or hanging the GPU.

- A device allocation made to fail (the library's injection hook) turns into
  SPA_ERR_NOMEM from the call that made it, which frees what it had already
  allocated: the device's free memory is back where it was.
- A bounded device-side wait that nothing completes (a shared-memory barrier
  no thread arrives on; a flag nothing sets) gives up after its limit and
  records a time-out; spa_workspace_status reports SPA_ERR_TIMEOUT once and
  clears it, and the context stays usable: the next wait, whose flag is set,
  and a regular layer step afterwards succeed."""
import ctypes

import numpy as np
import pytest
import torch

from adaptive_hidden_state_b200 import synth
from spa_testutil import LayerPair

pytestmark = pytest.mark.gpu

spa = pytest.importorskip("adaptive_hidden_state_b200.spa")

SMALL_BF16 = synth.LayerShape(d=256, n_heads=2, head_dim=128, ffn=384, r=16)


def _desc():
    return spa.LayerDesc(d=256, n_heads=2, head_dim=128, ffn=384, r=16, dtype=spa.SPA_BF16,
                         rms_eps=1e-5, rope_theta=1e4)


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


def test_injected_allocation_failure_reports_nomem_without_leak():
    desc = _desc()
    h = ctypes.c_void_p()
    # one successful create and free first, so lazily loaded state is in place
    assert spa.lib.spa_workspace_create(ctypes.byref(desc), 2, 128, ctypes.byref(h)) == 0
    spa.lib.spa_workspace_free(h)
    free0 = _free_bytes()
    failures = 0
    try:
        for n in range(64):
            spa.lib.spa_debug_fail_alloc_after(n)
            h = ctypes.c_void_p()
            st = spa.lib.spa_workspace_create(ctypes.byref(desc), 2, 128, ctypes.byref(h))
            if st == 0:            # n exceeds the workspace's allocations: nothing was injected
                spa.lib.spa_workspace_free(h)
                break
            failures += 1
            assert st == -4, spa.lib.spa_status_string(st)
            assert not h.value, "a failed create must not hand out a handle"
            assert b"out of memory" in spa.lib.spa_last_error()
            assert _free_bytes() == free0, f"device memory leaked after a failure at allocation {n}"
    finally:
        spa.lib.spa_debug_fail_alloc_after(-1)
    assert failures >= 10      # every workspace buffer's failure path was taken
    assert _free_bytes() == free0


def test_injected_failure_in_model_and_layer_creation():
    lp = LayerPair(spa, SMALL_BF16, seed=3, dtype=spa.SPA_BF16, max_B=1, max_N=64, std=0.05)
    vocab, N = 512, 64
    embed = torch.zeros((vocab, 256), dtype=torch.bfloat16, device="cuda")
    ones = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    h0 = torch.zeros((1, N, 256), dtype=torch.bfloat16, device="cuda")
    caches = [lp.cache(1, N)]
    free0 = _free_bytes()
    try:
        for n in range(4):      # the model's four buffers
            spa.lib.spa_debug_fail_alloc_after(n)
            with pytest.raises(spa.SpaError) as ei:
                spa.Model([lp.layer], caches, h0, embed, ones, embed, vocab, 1, N, 0.25, 1, 0.25, 0.25)
            assert ei.value.status == -4
            assert _free_bytes() == free0
        spa.lib.spa_debug_fail_alloc_after(0)   # the layer's proxy weights
        with pytest.raises(spa.SpaError) as ei:
            spa.Layer(lp.desc, lp.dev, lp.ws, w_r_host=np.zeros((16, 256), np.float32))
        assert ei.value.status == -4
        assert _free_bytes() == free0
    finally:
        spa.lib.spa_debug_fail_alloc_after(-1)
    model = spa.Model([lp.layer], caches, h0, embed, ones, embed, vocab, 1, N, 0.25, 1, 0.25, 0.25)
    model.close()


@pytest.mark.parametrize("use_flag", [False, True])
def test_bounded_wait_times_out_and_context_stays_usable(use_flag):
    lp = LayerPair(spa, SMALL_BF16, seed=4, dtype=spa.SPA_BF16, max_B=1, max_N=128, std=0.05)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp = flag.data_ptr() if use_flag else None
    assert lp.ws.status() == 0
    # 2 ms limit, nothing completes the wait
    assert spa.lib.spa_debug_bounded_wait(lp.ws.handle, fp, 1, 2000.0, None) == 0
    assert lp.ws.status() == -6
    assert b"timed out" in spa.lib.spa_last_error()
    assert lp.ws.status() == 0                      # read and cleared
    if use_flag:
        flag.fill_(1)                               # now the flag is set: the wait completes
        assert spa.lib.spa_debug_bounded_wait(lp.ws.handle, fp, 1, 2000.0, None) == 0
        assert lp.ws.status() == 0
    # the context still runs the regular path
    H = lp.to_dev(synth.hidden_states(1, 128, 256, seed=5, bf16=True))
    cache = lp.cache(1, 128)
    spa.spa_full_block(lp.layer, H, cache, True)
    idx = torch.empty((1, 16), dtype=torch.int32, device="cuda")
    spa.spa_layer_step(lp.layer, H, cache, 16, idx)
    assert lp.ws.status() == 0
    assert idx.cpu().numpy()[0].tolist() == list(range(16))   # zero drift: the lowest indices

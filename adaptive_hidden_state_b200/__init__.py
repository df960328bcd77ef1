"""SPA-Cache cached-layer decode path for NVIDIA B200 (sm_100a).

The compute path lives in the CUDA library ``libspa.so`` (sources under
``csrc/``); ``adaptive_hidden_state_b200.spa`` is its thin ctypes binding.
``synth`` draws the seeded synthetic workloads.  Importing this package does
not load the library; importing ``.spa`` does, and fails loudly without it.
"""
__all__ = ["synth"]

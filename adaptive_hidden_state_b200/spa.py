"""ctypes binding of libspa (the C ABI in include/spa.h).

Argument marshalling only: tensors are passed as raw device pointers and the
current torch CUDA stream; every step of the computation runs in the CUDA
library.  Importing this module loads ``libspa.so`` from this package's
directory and raises ImportError when it has not been built (there is no
fallback implementation).
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspa.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with "
                      "`python -m adaptive_hidden_state_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

SPA_OK = 0
SPA_F32, SPA_BF16 = 0, 1
STATUS = {0: "SPA_OK", -1: "SPA_ERR_INVALID", -2: "SPA_ERR_SHAPE", -3: "SPA_ERR_CUDA",
          -4: "SPA_ERR_NOMEM", -5: "SPA_ERR_UNSUPPORTED", -6: "SPA_ERR_TIMEOUT",
          -7: "SPA_ERR_DEVICE"}

# every symbol the header declares, in declaration order
EXPORTS = [
    "spa_status_string", "spa_last_error", "spa_version", "spa_rho", "spa_budget_k",
    "spa_singular_proxy_host", "spa_workspace_create", "spa_workspace_free",
    "spa_workspace_status", "spa_workspace_intermediates", "spa_profile_enable",
    "spa_profile_read", "spa_launch_count", "spa_init_layer", "spa_free_layer", "spa_layer_proxy_weights",
    "spa_proxy_select", "spa_partial_block", "spa_layer_step", "spa_full_block",
    "spa_layer_step_attn_identifier",
    "spa_model_create", "spa_model_free", "spa_model_layer_k", "spa_model_index_set", "spa_model_embed",
    "spa_decode_step", "spa_decode_layers", "spa_decode_confidence", "spa_model_write_tokens",
    "spa_decode_graph_capture", "spa_decode_graph_launch", "spa_decode_graph_kernel_nodes",
    "spa_model_set_incremental_proxy", "spa_debug_fail_alloc_after", "spa_debug_bounded_wait",
    "spa_attention_noalloc", "spa_attention_noalloc_status",
]


PROF_CLASSES = ["proxy", "topk", "norm", "qkv", "attn", "oproj", "gateup", "down", "lmhead", "misc", "ffn"]


def spa_launch_count() -> int:
    return lib.spa_launch_count()


class SpaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.spa_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


class LayerDesc(ctypes.Structure):
    _fields_ = [("d", c_int), ("n_heads", c_int), ("head_dim", c_int), ("ffn", c_int),
                ("r", c_int), ("dtype", c_int), ("rms_eps", c_float), ("rope_theta", c_float)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down",
                                        "attn_norm", "ffn_norm")]


class LayerCacheDesc(ctypes.Structure):
    _fields_ = [("k_cache", c_void_p), ("v_cache", c_void_p), ("h_cache", c_void_p),
                ("p_cache", c_void_p), ("B", c_int), ("N", c_int)]


class Intermediates(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("x", "q", "o", "h1", "x2", "a", "a_hat", "score")]


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", c_int), ("vocab", c_int), ("B", c_int), ("N", c_int),
                ("rho_p", c_double), ("rho_1", c_double), ("rho_L", c_double), ("l_p", c_int)]


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("spa_status_string", c_char_p, c_int)
_sig("spa_last_error", c_char_p)
_sig("spa_version", c_int)
_sig("spa_rho", c_double, c_int, c_int, c_double, c_int, c_double, c_double)
_sig("spa_budget_k", c_int, c_int, c_double)
_sig("spa_singular_proxy_host", c_int, c_void_p, c_int, c_int, c_void_p)
_sig("spa_workspace_create", c_int, POINTER(LayerDesc), c_int, c_int, POINTER(c_void_p))
_sig("spa_workspace_free", None, c_void_p)
_sig("spa_workspace_status", c_int, c_void_p, c_void_p)
_sig("spa_workspace_intermediates", c_int, c_void_p, POINTER(Intermediates))
_sig("spa_profile_enable", c_int, c_void_p, c_int)
_sig("spa_profile_read", c_int, c_void_p, POINTER(c_int), POINTER(c_double), POINTER(c_double),
     POINTER(c_double))
_sig("spa_launch_count", ctypes.c_longlong)
_sig("spa_init_layer", c_int, POINTER(LayerDesc), POINTER(LayerWeights), c_void_p, c_void_p,
     POINTER(c_void_p))
_sig("spa_free_layer", None, c_void_p)
_sig("spa_layer_proxy_weights", c_int, c_void_p, c_void_p)
_sig("spa_proxy_select", c_int, c_void_p, c_void_p, POINTER(LayerCacheDesc), c_int, c_void_p,
     c_void_p, c_void_p)
_sig("spa_partial_block", c_int, c_void_p, c_void_p, c_void_p, c_int, POINTER(LayerCacheDesc),
     c_void_p)
_sig("spa_layer_step", c_int, c_void_p, c_void_p, POINTER(LayerCacheDesc), c_int, c_void_p,
     c_void_p)
_sig("spa_full_block", c_int, c_void_p, c_void_p, POINTER(LayerCacheDesc), c_int, c_void_p)
_sig("spa_layer_step_attn_identifier", c_int, c_void_p, c_void_p, POINTER(LayerCacheDesc), c_int, c_void_p,
     c_void_p)
_sig("spa_model_create", c_int, POINTER(ModelDesc), POINTER(c_void_p), POINTER(LayerCacheDesc),
     c_void_p, c_void_p, c_void_p, c_void_p, POINTER(c_void_p))
_sig("spa_model_free", None, c_void_p)
_sig("spa_model_layer_k", c_int, c_void_p, c_int)
_sig("spa_model_index_set", c_int, c_void_p, c_int, c_void_p, c_void_p)
_sig("spa_model_set_incremental_proxy", c_int, c_void_p, c_int)
_sig("spa_model_embed", c_int, c_void_p, c_void_p, c_void_p)
_sig("spa_decode_step", c_int, c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p)
_sig("spa_decode_layers", c_int, c_void_p, c_int, c_void_p)
_sig("spa_decode_confidence", c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p)
_sig("spa_model_write_tokens", c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p)
_sig("spa_decode_graph_capture", c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p)
_sig("spa_decode_graph_launch", c_int, c_void_p, c_void_p)
_sig("spa_decode_graph_kernel_nodes", c_int, c_void_p)
_sig("spa_attention_noalloc", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
     c_int, c_int, c_void_p)
_sig("spa_attention_noalloc_status", c_int, c_void_p)
_sig("spa_debug_fail_alloc_after", c_int, ctypes.c_longlong)
_sig("spa_debug_bounded_wait", c_int, c_void_p, c_void_p, c_int, c_double, c_void_p)


def _check(status: int, where: str):
    if status != SPA_OK:
        raise SpaError(status, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------- thin wrappers

def spa_status_string(status: int) -> str:
    return lib.spa_status_string(status).decode()


def spa_version() -> int:
    return lib.spa_version()


def spa_rho(l: int, L: int, rho_p: float, l_p: int, rho_1: float, rho_L: float) -> float:
    return lib.spa_rho(l, L, rho_p, l_p, rho_1, rho_L)


def spa_budget_k(N: int, rho: float) -> int:
    return lib.spa_budget_k(N, rho)


def spa_singular_proxy_host(w_v: torch.Tensor, r: int) -> torch.Tensor:
    """Host SVD proxy of a [d, d] CPU float32 tensor; returns [r, d] float32."""
    w_v = w_v.detach().to("cpu", torch.float32).contiguous()
    d = w_v.shape[0]
    out = torch.empty((r, d), dtype=torch.float32)
    _check(lib.spa_singular_proxy_host(w_v.data_ptr(), d, r, out.data_ptr()),
           "spa_singular_proxy_host")
    return out


def torch_dtype(dtype: int):
    return torch.bfloat16 if dtype == SPA_BF16 else torch.float32


class Workspace:
    def __init__(self, desc: LayerDesc, max_B: int, max_N: int):
        self.desc = desc
        h = c_void_p()
        _check(lib.spa_workspace_create(ctypes.byref(desc), max_B, max_N, ctypes.byref(h)),
               "spa_workspace_create")
        self.handle = h

    def status(self, stream=None) -> int:
        return lib.spa_workspace_status(self.handle, _stream(stream))

    def check(self, stream=None):
        _check(self.status(stream), "spa_workspace_status")

    def profile_enable(self, on: bool = True):
        _check(lib.spa_profile_enable(self.handle, int(on)), "spa_profile_enable")

    def profile_read(self) -> dict:
        """{class name: (launches, ms, algorithmic bytes, flops)} since the last read."""
        n = len(PROF_CLASSES)
        la, ms, by, fl = (c_int * n)(), (c_double * n)(), (c_double * n)(), (c_double * n)()
        _check(lib.spa_profile_read(self.handle, la, ms, by, fl), "spa_profile_read")
        return {PROF_CLASSES[i]: (la[i], ms[i], by[i], fl[i]) for i in range(n)}

    def intermediates(self) -> dict:
        """Device addresses of the compact intermediates of the last layer call."""
        it = Intermediates()
        _check(lib.spa_workspace_intermediates(self.handle, ctypes.byref(it)),
               "spa_workspace_intermediates")
        return {f[0]: getattr(it, f[0]) for f in Intermediates._fields_}

    def view(self, name: str, shape, dtype) -> torch.Tensor:
        """A torch tensor aliasing an intermediate buffer (no copy)."""
        addr = self.intermediates()[name]
        typestr = {torch.float32: "<f4", torch.bfloat16: "<u2", torch.int32: "<i4"}[dtype]

        class _Iface:
            __cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                        "data": (addr, False), "version": 2, "strides": None}

        t = torch.as_tensor(_Iface(), device="cuda")
        return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t

    def close(self):
        if self.handle:
            lib.spa_workspace_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Layer:
    """A layer handle.  `weights` maps wq, wk, wv, wo, w_gate, w_up, w_down,
    attn_norm, ffn_norm to device tensors (kept referenced here)."""

    def __init__(self, desc: LayerDesc, weights: dict, ws: Workspace, w_r_host=None):
        self.desc, self.ws = desc, ws
        names = [f[0] for f in LayerWeights._fields_]
        self.weights = {k: weights[k].contiguous() for k in names}
        lw = LayerWeights(*[_ptr(self.weights[f[0]]) for f in LayerWeights._fields_])
        wr = None
        if w_r_host is not None:
            wr = torch.as_tensor(w_r_host, dtype=torch.float32).contiguous().cpu()
        h = c_void_p()
        _check(lib.spa_init_layer(ctypes.byref(desc), ctypes.byref(lw),
                                  wr.data_ptr() if wr is not None else None, ws.handle,
                                  ctypes.byref(h)), "spa_init_layer")
        self.handle = h

    def proxy_weights(self) -> torch.Tensor:
        out = torch.empty((self.desc.r, self.desc.d), dtype=torch.float32)
        _check(lib.spa_layer_proxy_weights(self.handle, out.data_ptr()), "spa_layer_proxy_weights")
        return out

    def close(self):
        if self.handle:
            lib.spa_free_layer(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Cache:
    """Device caches of one layer (torch-owned): K^c, V^c, H^c [B, N, d] and P^c [B, N, r]."""

    def __init__(self, B: int, N: int, d: int, r: int, dtype: int, device="cuda"):
        t = torch_dtype(dtype)
        self.k = torch.zeros((B, N, d), dtype=t, device=device)
        self.v = torch.zeros((B, N, d), dtype=t, device=device)
        self.h = torch.zeros((B, N, d), dtype=t, device=device)
        self.p = torch.zeros((B, N, r), dtype=torch.float32, device=device)
        self.B, self.N = B, N
        self.desc = LayerCacheDesc(self.k.data_ptr(), self.v.data_ptr(), self.h.data_ptr(),
                                   self.p.data_ptr(), B, N)


def spa_proxy_select(layer: Layer, H, cache: Cache, k: int, idx, score=None, stream=None):
    _check(lib.spa_proxy_select(layer.handle, _ptr(H), ctypes.byref(cache.desc), k, _ptr(idx),
                                _ptr(score), _stream(stream)), "spa_proxy_select")


def spa_partial_block(layer: Layer, H, idx, k: int, cache: Cache, stream=None):
    _check(lib.spa_partial_block(layer.handle, _ptr(H), _ptr(idx), k, ctypes.byref(cache.desc),
                                 _stream(stream)), "spa_partial_block")


def spa_layer_step(layer: Layer, H, cache: Cache, k: int, idx, stream=None):
    _check(lib.spa_layer_step(layer.handle, _ptr(H), ctypes.byref(cache.desc), k, _ptr(idx),
                              _stream(stream)), "spa_layer_step")


def spa_full_block(layer: Layer, H, cache: Cache, fill_proxy: int = 1, stream=None):
    """fill_proxy: 0 none, 1 (or True) the value proxy, 2 unit attention outputs."""
    _check(lib.spa_full_block(layer.handle, _ptr(H), ctypes.byref(cache.desc), int(fill_proxy),
                              _stream(stream)), "spa_full_block")


def spa_layer_step_attn_identifier(layer: Layer, H, cache: Cache, k: int, idx, stream=None):
    _check(lib.spa_layer_step_attn_identifier(layer.handle, _ptr(H), ctypes.byref(cache.desc), k, _ptr(idx),
                                              _stream(stream)), "spa_layer_step_attn_identifier")


class Model:
    """Decode loop over layer handles that share one workspace."""

    def __init__(self, layers: list, caches: list, h0, embed, final_norm, lm_head, vocab: int,
                 B: int, N: int, rho_p: float, l_p: int, rho_1: float, rho_L: float):
        self.layers, self.caches = layers, caches
        self.h0, self.embed, self.final_norm, self.lm_head = h0, embed, final_norm, lm_head
        self.B, self.N = B, N
        L = len(layers)
        desc = ModelDesc(L, vocab, B, N, rho_p, rho_1, rho_L, l_p)
        handles = (c_void_p * L)(*[ly.handle.value for ly in layers])
        cdesc = (LayerCacheDesc * L)(*[c.desc for c in caches])
        h = c_void_p()
        _check(lib.spa_model_create(ctypes.byref(desc), handles, cdesc, _ptr(h0), _ptr(embed),
                                    _ptr(final_norm), _ptr(lm_head), ctypes.byref(h)),
               "spa_model_create")
        self.handle = h
        self.k = [lib.spa_model_layer_k(h, l) for l in range(L)]

    def embed_tokens(self, tokens, stream=None):
        _check(lib.spa_model_embed(self.handle, _ptr(tokens), _stream(stream)), "spa_model_embed")

    def index_set(self, layer: int, stream=None) -> torch.Tensor:
        """[B, k_l] int32 device copy of layer `layer`'s index set from the last cached step."""
        out = torch.empty((self.B, self.k[layer]), dtype=torch.int32, device="cuda")
        _check(lib.spa_model_index_set(self.handle, layer, _ptr(out), _stream(stream)),
               "spa_model_index_set")
        return out

    def set_incremental_proxy(self, enable: bool = True):
        _check(lib.spa_model_set_incremental_proxy(self.handle, 1 if enable else 0),
               "spa_model_set_incremental_proxy")

    def close(self):
        if self.handle:
            lib.spa_model_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def spa_decode_layers(model: Model, full: int, stream=None):
    _check(lib.spa_decode_layers(model.handle, full, _stream(stream)), "spa_decode_layers")


def spa_decode_confidence(model: Model, pos, u: int, tok_out, conf_out, stream=None):
    _check(lib.spa_decode_confidence(model.handle, _ptr(pos), u, _ptr(tok_out), _ptr(conf_out),
                                     _stream(stream)), "spa_decode_confidence")


def spa_model_write_tokens(model: Model, pos, tok, u: int, stream=None):
    _check(lib.spa_model_write_tokens(model.handle, _ptr(pos), _ptr(tok), u, _stream(stream)),
           "spa_model_write_tokens")


def spa_decode_step(model: Model, pos, tok_in, u: int, full: int, tok_out, stream=None):
    _check(lib.spa_decode_step(model.handle, _ptr(pos), _ptr(tok_in), u, int(full), _ptr(tok_out),
                               _stream(stream)), "spa_decode_step")


def spa_decode_graph_capture(model: Model, pos, tok_in, u: int, tok_out, stream=None):
    _check(lib.spa_decode_graph_capture(model.handle, _ptr(pos), _ptr(tok_in), u, _ptr(tok_out),
                                        _stream(stream)), "spa_decode_graph_capture")


def spa_decode_graph_launch(model: Model, stream=None):
    _check(lib.spa_decode_graph_launch(model.handle, _stream(stream)), "spa_decode_graph_launch")


def spa_decode_graph_kernel_nodes(model: Model) -> int:
    return lib.spa_decode_graph_kernel_nodes(model.handle)


def spa_attention_noalloc(Q, k_cache, v_cache, O, B: int, k: int, N: int, n_heads: int,
                          head_dim: int, stream=None):
    """Attention of the selected queries against the whole cache, with the
    library's fixed scratch instead of allocated memory (see include/spa.h)."""
    _check(lib.spa_attention_noalloc(_ptr(Q), _ptr(k_cache), _ptr(v_cache), _ptr(O), B, k, N,
                                     n_heads, head_dim, _stream(stream)), "spa_attention_noalloc")


def spa_attention_noalloc_status(stream=None) -> int:
    """Reads and clears the allocation-free attention's device error word
    (synchronises the stream): 0, or the negative status of what failed."""
    return lib.spa_attention_noalloc_status(_stream(stream))

"""B200-native block-diffusion MoE denoising step.

The product is libdg.so, a C-ABI library of sm_100a kernels (include/dg.h,
include/dg_ops.h).  This module is its thin Python binding: it marshals torch
device tensors (used only for device memory and streams) into the C calls,
with the same names.  Every step of the pass runs in the library's kernels;
if the library is not built the import of `DG` fails loudly.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _ffi
from ._ffi import DGError, check, dg_config, dg_layer_weights, dg_weights  # noqa: F401

__all__ = ["DG", "DGError", "config_struct", "lm_head_noalloc", "philox_tokens", "route_topk", "weight_shapes"]


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _check(t, name: str, dtype, device: bool, numel: int | None = None, shape=None):
    """Reject, before any C call, a tensor the C ABI cannot take: host memory
    where device memory is expected (or the reverse), another element type, a
    non-contiguous view, or fewer elements than the call reads.  A wrong
    pointer would otherwise reach a kernel as an out-of-range address."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if bool(t.is_cuda) != device:
        raise ValueError(f"{name}: expected {'device (CUDA)' if device else 'host'} memory, got {t.device}")
    dtypes = dtype if isinstance(dtype, tuple) else (dtype,)
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: expected dtype {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: expected at least {numel} elements, got {t.numel()}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _dev(t, name: str, dtype, numel: int | None = None, shape=None, optional: bool = False):
    """Device pointer of a checked CUDA tensor (None for an optional None)."""
    if t is None and optional:
        return None
    return C.c_void_p(_check(t, name, dtype, True, numel, shape).data_ptr())


def _host(t, name: str, dtype, numel: int | None = None):
    """Host pointer of a checked CPU tensor."""
    return C.c_void_p(_check(t, name, dtype, False, numel).data_ptr())


_F32, _I32, _U8, _BF16 = torch.float32, torch.int32, torch.uint8, torch.bfloat16


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def config_struct(cfg) -> dg_config:
    """dg_config from a synth.ModelConfig-like object."""
    return dg_config(cfg.n_layers, cfg.d_model, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.n_experts,
                     cfg.top_k, cfg.ffn_expert, cfg.ffn_shared, cfg.vocab, cfg.canvas, cfg.max_steps,
                     cfg.min_accept, cfg.entropy_thresh, cfg.rope_theta, cfg.norm_eps,
                     getattr(cfg, "sampler", 0), getattr(cfg, "entropy_budget", 0.1),
                     getattr(cfg, "stop_entropy", 0.005), getattr(cfg, "temperature", 0.0),
                     getattr(cfg, "ffn_selfcond", 0), getattr(cfg, "selfcond_topk", 8),
                     getattr(cfg, "expert_fp8", 0))


def philox_tokens(seed: int, block: int, step: int, request: int, pos0: int, n: int, vocab: int,
                  out: torch.Tensor, stream=None) -> None:
    check(_ffi.load().dg_op_philox_tokens(seed, block, step, request, pos0, n, vocab, _dev(out, "out", _I32, n),
                                          _stream(stream)), "dg_op_philox_tokens")


def route_topk(logits: torch.Tensor, k: int, idx: torch.Tensor, w: torch.Tensor, stream=None) -> None:
    T, E = logits.shape
    check(_ffi.load().dg_op_route_topk(_dev(logits, "logits", _F32), T, E, k, _dev(idx, "idx", _I32, T * k),
                                       _dev(w, "w", _F32, T * k), _stream(stream)), "dg_op_route_topk")


def lm_head_noalloc(x: torch.Tensor, final_norm: torch.Tensor, embed: torch.Tensor, norm_eps: float,
                    stats: torch.Tensor, argmax: torch.Tensor, err: torch.Tensor | None = None, stream=None) -> None:
    """dg_op_lm_head_noalloc: LM-head statistics with the library's built-in
    scratch (no workspace, no allocation inside)."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError("x: expected a 2-D [T, d_model] tensor")
    if not isinstance(embed, torch.Tensor) or embed.dim() != 2:
        raise ValueError("embed: expected a 2-D [vocab, d_model] tensor")
    T, d = x.shape
    V = embed.shape[0]
    check(_ffi.load().dg_op_lm_head_noalloc(
        _dev(x, "x", _F32, shape=(T, d)), _dev(final_norm, "final_norm", _F32, shape=(d,)),
        _dev(embed, "embed", _BF16, shape=(V, d)), T, d, V, norm_eps, _dev(stats, "stats", _F32, T * 4), _dev(argmax, "argmax", _I32, T),
        _dev(err, "err", _I32, 1, optional=True), _stream(stream)), "dg_op_lm_head_noalloc")


def weight_shapes(cfg) -> dict:
    """The shape dg_init reads for every weight tensor of a configuration (dg.h,
    dg_layer_weights / dg_weights): a tensor of another shape is rejected before
    the C call, since its TMA descriptors would reach past its end."""
    d, D, E = cfg.d_model, cfg.head_dim, cfg.n_experts
    fe, fs, fsc = cfg.ffn_expert, cfg.ffn_shared, getattr(cfg, "ffn_selfcond", 0)
    return {
        "embed": (cfg.vocab, d), "final_norm": (d,),
        "attn_norm": (d,), "w_qkv": ((cfg.n_q_heads + 2 * cfg.n_kv_heads) * D, d), "w_o": (d, cfg.n_q_heads * D),
        "ffn_norm": (d,), "w_router": (E, d), "w_gate": (E, fe, d), "w_up": (E, fe, d), "w_down": (E, d, fe),
        "ws_gate": (fs, d), "ws_up": (fs, d), "ws_down": (d, fs),
        "w_gate_scale": (E, fe), "w_up_scale": (E, fe), "w_down_scale": (E, d),
        "sc_gate": (fsc, d), "sc_up": (fsc, d), "sc_down": (d, fsc),
    }


class DG:
    """A libdg handle bound to caller-owned torch tensors (weights, workspace)."""

    def __init__(self, cfg, weights: dict, max_requests: int, kv_capacity: int, device="cuda", stream=None):
        lib = _ffi.load()
        self.lib = lib
        self.cfg = cfg
        self.c_cfg = config_struct(cfg)
        self.weights = weights            # keep the tensors alive
        self.stream = stream or torch.cuda.current_stream(device)
        if len(weights["layers"]) != cfg.n_layers:
            raise ValueError(f"weights: {len(weights['layers'])} layers for a {cfg.n_layers}-layer configuration")
        fp8 = bool(getattr(cfg, "expert_fp8", 0))
        shapes = weight_shapes(cfg)
        layers = (dg_layer_weights * cfg.n_layers)()
        for i, lw in enumerate(weights["layers"]):
            ptrs = []
            for n in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "w_gate", "w_up", "w_down", "ws_gate",
                      "ws_up", "ws_down", "w_gate_scale", "w_up_scale", "w_down_scale"):
                if n.endswith("_scale") and not fp8:
                    ptrs.append(None)
                    continue
                dt = _F32 if n.endswith("norm") or n.endswith("_scale") else (
                    _U8 if fp8 and n in ("w_gate", "w_up", "w_down") else _BF16)
                ptrs.append(_check(lw[n], f"layers[{i}].{n}", dt, True, shape=shapes[n]).data_ptr())
            layers[i] = dg_layer_weights(*ptrs)
        self._layers = layers
        sc = [_check(weights[n], n, _BF16, True, shape=shapes[n]).data_ptr()
              if getattr(cfg, "ffn_selfcond", 0) > 0 else None for n in ("sc_gate", "sc_up", "sc_down")]
        self.c_w = dg_weights(_check(weights["embed"], "embed", _BF16, True, shape=shapes["embed"]).data_ptr(),
                              _check(weights["final_norm"], "final_norm", _F32, True,
                                     shape=shapes["final_norm"]).data_ptr(), layers, *sc)
        nbytes = lib.dg_workspace_size(C.byref(self.c_cfg), max_requests, kv_capacity)
        if nbytes == 0:
            raise DGError(-1, "dg_workspace_size")
        self.workspace = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
        base = self.workspace.data_ptr()
        self._ws_off = (-base) % 1024
        h = C.c_void_p()
        check(lib.dg_init(C.byref(self.c_cfg), C.byref(self.c_w), max_requests, kv_capacity,
                          C.c_void_p(base + self._ws_off), nbytes, C.c_void_p(self.stream.cuda_stream),
                          C.byref(h)), "dg_init")
        self.h = h
        self.max_requests = max_requests
        self.kv_capacity = kv_capacity

    def close(self):
        if getattr(self, "h", None):
            self.lib.dg_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- the C ABI, same names ----
    def prefill(self, req: int, tokens: torch.Tensor):
        check(self.lib.dg_prefill(self.h, req, _dev(tokens, "tokens", _I32), tokens.numel()), "dg_prefill")

    def set_kv(self, req: int, layer: int, pos0: int, k: torch.Tensor, v: torch.Tensor):
        shape = (self.cfg.n_kv_heads, k.shape[1] if k.dim() == 3 else -1, self.cfg.head_dim)
        check(self.lib.dg_set_kv(self.h, req, layer, pos0, shape[1], _dev(k, "k", _BF16, shape=shape),
                                 _dev(v, "v", _BF16, shape=shape)), "dg_set_kv")

    def get_kv(self, req: int, layer: int, pos0: int, n: int):
        c = self.cfg
        k = torch.empty((c.n_kv_heads, n, c.head_dim), dtype=torch.bfloat16, device=self.workspace.device)
        v = torch.empty_like(k)
        check(self.lib.dg_get_kv(self.h, req, layer, pos0, n, _ptr(k), _ptr(v)), "dg_get_kv")
        return k, v

    def set_kv_len(self, req: int, n: int):
        check(self.lib.dg_set_kv_len(self.h, req, n), "dg_set_kv_len")

    def kv_len(self, req: int) -> int:
        return self.lib.dg_kv_len(self.h, req)

    def open_canvas(self, req: int, seed: int, block: int):
        check(self.lib.dg_open_canvas(self.h, req, seed, block), "dg_open_canvas")

    def denoise_step(self, reqs, d_remaining: torch.Tensor | None = None):
        arr = (C.c_int * len(reqs))(*reqs)
        check(self.lib.dg_denoise_step(self.h, len(reqs), arr,
                                       _dev(d_remaining, "d_remaining", _I32, len(reqs), optional=True)),
              "dg_denoise_step")

    def read_remaining(self, req: int) -> int:
        r = C.c_int32()
        check(self.lib.dg_read_remaining(self.h, req, C.byref(r)), "dg_read_remaining")
        return r.value

    def commit_block(self, req: int):
        check(self.lib.dg_commit_block(self.h, req), "dg_commit_block")

    def generate(self, req: int, prompt_host: torch.Tensor, n_out: int, seed: int, out_host: torch.Tensor):
        n_blocks = n_out // self.cfg.canvas
        steps = (C.c_int * max(1, n_blocks))()
        check(self.lib.dg_generate(self.h, req, _host(prompt_host, "prompt_host", _I32), prompt_host.numel(), n_out,
                                   seed, _host(out_host, "out_host", _I32, n_out), steps), "dg_generate")
        return list(steps)[:n_blocks]

    def get_canvas(self, req: int):
        dev = self.workspace.device
        C_ = self.cfg.canvas
        tok = torch.empty(C_, dtype=torch.int32, device=dev)
        mask = torch.empty(C_, dtype=torch.uint8, device=dev)
        stats = torch.empty((C_, 4), dtype=torch.float32, device=dev)
        am = torch.empty(C_, dtype=torch.int32, device=dev)
        check(self.lib.dg_get_canvas(self.h, req, _ptr(tok), _ptr(mask), _ptr(stats), _ptr(am)), "dg_get_canvas")
        return tok, mask, stats, am

    def set_canvas(self, req: int, tokens: torch.Tensor, mask: torch.Tensor, step: int):
        C_ = self.cfg.canvas
        check(self.lib.dg_set_canvas(self.h, req, _dev(tokens, "tokens", _I32, C_), _dev(mask, "mask", _U8, C_), step),
              "dg_set_canvas")

    def sync(self):
        check(self.lib.dg_sync(self.h), "dg_sync")

    # ---- operation-level entry points ----
    def op_route_group(self, idx: torch.Tensor, w: torch.Tensor):
        T = idx.shape[0]
        dev = idx.device
        E = self.cfg.n_experts
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(idx.numel(), dtype=torch.int32, device=dev)
        k = self.cfg.top_k
        check(self.lib.dg_op_route_group(self.h, _dev(idx, "idx", _I32, shape=(T, k)), _dev(w, "w", _F32, shape=(T, k)),
                                         T, _ptr(counts), _ptr(offsets), _ptr(perm)), "dg_op_route_group")
        return counts, offsets, perm

    def op_sample(self, req: int, entropy, logconf, argmax, step: int):
        C_ = self.cfg.canvas
        check(self.lib.dg_op_sample(self.h, req, _dev(entropy, "entropy", _F32, C_), _dev(logconf, "logconf", _F32, C_),
                                    _dev(argmax, "argmax", _I32, C_), step), "dg_op_sample")

    def op_lm_head(self, x: torch.Tensor, want_logits: bool = False):
        T = x.shape[0]
        dev = x.device
        stats = torch.empty((T, 4), dtype=torch.float32, device=dev)
        am = torch.empty(T, dtype=torch.int32, device=dev)
        logits = torch.empty((T, self.cfg.vocab), dtype=torch.float32, device=dev) if want_logits else None
        check(self.lib.dg_op_lm_head(self.h, _dev(x, "x", _F32, shape=(T, self.cfg.d_model)), T, _ptr(stats), _ptr(am),
                                     _ptr(logits)), "dg_op_lm_head")
        return stats, am, logits

    def op_lm_sample(self, x: torch.Tensor, temperature: float, seed: int, block: int, step: int, request: int = 0):
        """dg_op_lm_sample: LM-head statistics and drawn candidates of rows = positions 0..T-1."""
        T = x.shape[0]
        dev = x.device
        stats = torch.empty((T, 4), dtype=torch.float32, device=dev)
        am = torch.empty(T, dtype=torch.int32, device=dev)
        cand = torch.empty(T, dtype=torch.int32, device=dev)
        check(self.lib.dg_op_lm_sample(self.h, _dev(x, "x", _F32, shape=(T, self.cfg.d_model)), T, temperature, seed,
                                       block, step, request, _ptr(stats), _ptr(am), _ptr(cand)), "dg_op_lm_sample")
        return stats, am, cand

    def op_selfcond(self, request: int, x: torch.Tensor):
        """dg_op_selfcond: the self-conditioning term [T, d] of hidden rows x and the
        top entries (p [T, 8] f32, ids [T, 8] i32; entries past selfcond_topk undefined)."""
        T, d = x.shape
        sc = torch.empty((T, d), dtype=torch.float32, device=x.device)
        top = torch.empty((T, 8, 2), dtype=torch.float32, device=x.device)
        check(self.lib.dg_op_selfcond(self.h, request, _dev(x, "x", _F32, shape=(T, self.cfg.d_model)), T, _ptr(sc),
                                      _ptr(top)), "dg_op_selfcond")
        return sc, top[..., 0], top.view(torch.int32)[..., 1]

    KERNEL_CLASSES = ("embed", "rmsnorm", "qkv", "attention", "oproj", "group",
                      "experts_gate_up", "experts_down", "shared_gate_up", "shared_down", "lm_head", "lm_combine",
                      "sample", "selfcond", "other", "experts")

    def profile(self, enable: int):
        check(self.lib.dg_profile(self.h, enable), "dg_profile")

    def profile_read(self) -> dict:
        out = {}
        for k in self.KERNEL_CLASSES:
            ms, n = C.c_double(), C.c_int64()
            check(self.lib.dg_profile_read(self.h, k.encode(), C.byref(ms), C.byref(n)), "dg_profile_read")
            out[k] = (ms.value, n.value)
        return out

    def launch_count(self) -> int:
        return self.lib.dg_launch_count(self.h)

    def debug_forward(self, req: int, tokens: torch.Tensor, n_layers: int):
        check(self.lib.dg_debug_forward(self.h, req, _dev(tokens, "tokens", _I32), tokens.numel(), n_layers),
              "dg_debug_forward")

    def debug_forward_hidden(self, req: int, tokens: torch.Tensor, x: torch.Tensor, layer0: int, n_layers: int):
        """dg_debug_forward_hidden: layers layer0.. from the residual stream x [T, d_model] f32."""
        T = tokens.numel()
        check(self.lib.dg_debug_forward_hidden(self.h, req, _dev(tokens, "tokens", _I32),
                                               _dev(x, "x", _F32, shape=(T, self.cfg.d_model)), T, layer0, n_layers),
              "dg_debug_forward_hidden")

    def token_capacity(self) -> int:
        """Rows of the per-pass token buffers (the middle extent of "q")."""
        off, nb = C.c_size_t(), C.c_size_t()
        check(self.lib.dg_debug_buffer(self.h, b"x", C.byref(off), C.byref(nb)), "dg_debug_buffer")
        return nb.value // (self.cfg.d_model * 4)

    def debug_buffer(self, name: str, dtype: torch.dtype, shape=None) -> torch.Tensor:
        off, nb = C.c_size_t(), C.c_size_t()
        check(self.lib.dg_debug_buffer(self.h, name.encode(), C.byref(off), C.byref(nb)), "dg_debug_buffer")
        o = self._ws_off + off.value
        t = self.workspace[o: o + nb.value].view(dtype)
        return t if shape is None else t[: int(torch.tensor(shape).prod())].view(*shape)

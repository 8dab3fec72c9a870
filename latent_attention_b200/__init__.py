"""B200 (sm_100a) Multi-Latent Attention: thin Python binding of ``mla.h``.

Names mirror the C ABI: ``mla_build_rope_tables``, ``mla_prefill_forward``,
``mla_decode_absorbed`` (plus the workspace-size and status helpers).  The
binding only marshals arguments: tensors must already live on a CUDA device
(torch is used for device memory and streams), and every step of the forward
runs in the library's kernels.  A missing library or a CPU tensor raises.
"""
import ctypes as C

from . import _lib
from ._lib import (mla_config, mla_weights, mla_prefill_layout,
                   mla_decode_layout, MLA_F32, MLA_BF16, ROPE_TYPES)

__all__ = ["MlaError", "make_config", "mla_build_rope_tables",
           "mla_prefill_workspace_size", "mla_prefill_forward",
           "mla_decode_workspace_size", "mla_decode_absorbed",
           "mla_check_device_status", "mla_decode_absorbed_noalloc",
           "mla_prefill_chunked_workspace_size", "mla_prefill_chunked",
           "mla_prefill_varlen_workspace_size", "mla_prefill_varlen",
           "abi_version"]


class MlaError(RuntimeError):
    def __init__(self, status, detail):
        self.status = status
        self.name = _lib.STATUS_NAMES.get(status, str(status))
        super().__init__(f"{self.name}: {detail}")


def _check(status):
    if status != _lib.MLA_OK:
        lib = _lib.load()
        raise MlaError(status, lib.mla_last_error_detail().decode())


def make_config(cfg) -> mla_config:
    """ctypes ``mla_config`` from any object with the config field names
    (``mla_inputs.MlaConfig`` for instance).  ``softmax_scale`` None/0 means
    "derive"; ``q_lora_rank`` 0 means None."""
    c = mla_config()
    for f in ("hidden_size", "num_heads", "q_lora_rank", "kv_lora_rank",
              "qk_nope_head_dim", "qk_rope_head_dim", "v_head_dim",
              "original_max_position_embeddings"):
        setattr(c, f, int(getattr(cfg, f)))
    for f in ("rope_theta", "rope_factor", "rope_mscale", "rope_mscale_all_dim",
              "beta_fast", "beta_slow", "rms_eps"):
        setattr(c, f, float(getattr(cfg, f)))
    c.rope_type = ROPE_TYPES[cfg.rope_type]
    c.dtype = {"f32": MLA_F32, "bf16": MLA_BF16}[cfg.dtype]
    c.softmax_scale = float(cfg.softmax_scale or 0.0)
    c.rope_interleave = int(bool(getattr(cfg, "rope_interleave", False)))
    return c


def _ptr(t, name, allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(getattr(stream, "cuda_stream", stream))


def abi_version() -> int:
    return _lib.load().mla_abi_version()


def mla_build_rope_tables(cfg, max_pos, cos_out, sin_out, stream=None):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    _check(_lib.load().mla_build_rope_tables(
        C.byref(c), int(max_pos), _ptr(cos_out, "cos_out"),
        _ptr(sin_out, "sin_out"), _stream(stream)))


def mla_prefill_workspace_size(cfg, B, T):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    lay = mla_prefill_layout()
    n = _lib.load().mla_prefill_workspace_size(C.byref(c), int(B), int(T),
                                               C.byref(lay))
    if n == 0:
        raise MlaError(2, "invalid configuration or sizes")
    return n, {f: getattr(lay, f) for f, _ in lay._fields_}


def mla_prefill_forward(cfg, weights, x, B, T, rope_cos, rope_sin, out,
                        workspace, latent_cache_out=None, stream=None):
    """``weights``: mapping with keys w_q_a, g_q_a, w_q_b, w_q, w_kv_a, g_kv_a,
    w_kv_b, w_o (CUDA tensors or None)."""
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    w = mla_weights()
    for f, _ in w._fields_:
        t = weights.get(f) if hasattr(weights, "get") else getattr(weights, f)
        setattr(w, f, None if t is None else _ptr(t, f).value)
    _check(_lib.load().mla_prefill_forward(
        C.byref(c), C.byref(w), _ptr(x, "x"), int(B), int(T),
        _ptr(rope_cos, "rope_cos", True), _ptr(rope_sin, "rope_sin", True),
        _ptr(out, "out"), _ptr(latent_cache_out, "latent_cache_out", True),
        _ptr(workspace, "workspace"), C.c_size_t(workspace.numel() *
                                                 workspace.element_size()),
        _stream(stream)))


def mla_prefill_chunked_workspace_size(cfg, B, T_new, T_past):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    lay = mla_prefill_layout()
    n = _lib.load().mla_prefill_chunked_workspace_size(
        C.byref(c), int(B), int(T_new), int(T_past), C.byref(lay))
    if n == 0:
        raise MlaError(2, "invalid configuration or sizes")
    return n, {f: getattr(lay, f) for f, _ in lay._fields_}


def _weights(weights):
    w = mla_weights()
    for f, _ in w._fields_:
        t = weights.get(f) if hasattr(weights, "get") else getattr(weights, f)
        setattr(w, f, None if t is None else _ptr(t, f).value)
    return w


def mla_prefill_chunked(cfg, weights, x, B, T_new, past_cache, T_past, rope_cos,
                        rope_sin, out, workspace, latent_cache_out=None,
                        stream=None):
    """Prefill of T_new tokens after T_past tokens held in ``past_cache``
    ([B, T_past, kv_lora_rank + rope], the latent cache rows)."""
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    w = _weights(weights)
    _check(_lib.load().mla_prefill_chunked(
        C.byref(c), C.byref(w), _ptr(x, "x"), int(B), int(T_new),
        _ptr(past_cache, "past_cache", True), int(T_past),
        _ptr(rope_cos, "rope_cos", True), _ptr(rope_sin, "rope_sin", True),
        _ptr(out, "out"), _ptr(latent_cache_out, "latent_cache_out", True),
        _ptr(workspace, "workspace"),
        C.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def mla_prefill_varlen_workspace_size(cfg, n_seq, total, max_seqlen):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    lay = mla_prefill_layout()
    n = _lib.load().mla_prefill_varlen_workspace_size(
        C.byref(c), int(n_seq), int(total), int(max_seqlen), C.byref(lay))
    if n == 0:
        raise MlaError(2, "invalid configuration or sizes")
    return n, {f: getattr(lay, f) for f, _ in lay._fields_}


def mla_prefill_varlen(cfg, weights, x, cu_seqlens, n_seq, total, max_seqlen, rope_cos,
                       rope_sin, out, workspace, latent_cache_out=None, stream=None):
    """Prefill of n_seq packed sequences (rows cu_seqlens[b] .. cu_seqlens[b+1]-1
    of x [total, hidden]); cu_seqlens is a device int32 tensor [n_seq + 1]."""
    import torch
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    w = _weights(weights)
    _check(_lib.load().mla_prefill_varlen(
        C.byref(c), C.byref(w), _ptr(x, "x"), _ptr(cu_seqlens, "cu_seqlens"), int(n_seq),
        int(total), int(max_seqlen), _ptr(rope_cos, "rope_cos", True),
        _ptr(rope_sin, "rope_sin", True), _ptr(out, "out"),
        _ptr(latent_cache_out, "latent_cache_out", True), _ptr(workspace, "workspace"),
        C.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def mla_decode_workspace_size(cfg, B, max_ctx):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    lay = mla_decode_layout()
    n = _lib.load().mla_decode_workspace_size(C.byref(c), int(B), int(max_ctx),
                                              C.byref(lay))
    if n == 0:
        raise MlaError(2, "invalid configuration or sizes")
    return n, {f: getattr(lay, f) for f, _ in lay._fields_}


def mla_decode_absorbed(cfg, q_nope, q_pe, w_kv_b, latent_cache, cu_ctx, B,
                        max_ctx, w_o, out, workspace, stream=None):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    _check(_lib.load().mla_decode_absorbed(
        C.byref(c), _ptr(q_nope, "q_nope"), _ptr(q_pe, "q_pe"),
        _ptr(w_kv_b, "w_kv_b"), _ptr(latent_cache, "latent_cache"),
        _ptr(cu_ctx, "cu_ctx"), int(B), int(max_ctx),
        _ptr(w_o, "w_o", True), _ptr(out, "out"), _ptr(workspace, "workspace"),
        C.c_size_t(workspace.numel() * workspace.element_size()),
        _stream(stream)))


def mla_check_device_status(workspace, stream=None):
    _check(_lib.load().mla_check_device_status(_ptr(workspace, "workspace"),
                                               _stream(stream)))


def mla_decode_absorbed_noalloc(cfg, q_nope, q_pe, w_kv_b, latent_cache, cu_ctx,
                                B, max_ctx, w_o, out, stream=None):
    """``mla_decode_absorbed`` for callers that cannot allocate device memory:
    the library's own static device array replaces the workspace.  Calls on
    one device share that array, so they must not overlap on the GPU."""
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    _check(_lib.load().mla_decode_absorbed_noalloc(
        C.byref(c), _ptr(q_nope, "q_nope"), _ptr(q_pe, "q_pe"),
        _ptr(w_kv_b, "w_kv_b"), _ptr(latent_cache, "latent_cache"),
        _ptr(cu_ctx, "cu_ctx"), int(B), int(max_ctx), _ptr(w_o, "w_o", True),
        _ptr(out, "out"), _stream(stream)))

"""B200 (sm_100a) Multi-Latent Attention: thin Python binding of ``mla.h``.

Names mirror the C ABI: ``mla_build_rope_tables``, ``mla_prefill_forward``,
``mla_decode_absorbed`` (plus the workspace-size and status helpers).  The
binding only marshals arguments: tensors must already live on a CUDA device
(torch is used for device memory and streams), and every step of the forward
runs in the library's kernels.  A missing library or a CPU tensor raises.

The C ABI takes plain pointers and cannot see buffer sizes, so the binding
checks each tensor's dtype and element count against the shapes ``mla.h``
declares for the call before passing its pointer on: a wrong tensor raises
ValueError here instead of reaching the device.
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


def _ptr(t, name, allow_none=False, dtype=None, numel=None, row=None):
    """Device pointer of tensor ``t`` after checking its dtype, that it holds
    at least ``numel`` elements and, with ``row``, whole rows of that many
    elements."""
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call uses {numel}")
    if row is not None and (t.numel() == 0 or t.numel() % row):
        raise ValueError(f"{name} must hold whole rows of {row} elements")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _dt(c):
    """torch dtype of activations, weights and outputs for config ``c``."""
    import torch
    return torch.bfloat16 if c.dtype == MLA_BF16 else torch.float32


def _f32():
    import torch
    return torch.float32


def _i32():
    import torch
    return torch.int32


def _rope_ptrs(c, rope_cos, rope_sin, rows):
    """The two fp32 tables, [>= rows, qk_rope_head_dim] each; unused (and
    unchecked) without rotary."""
    if c.rope_type == ROPE_TYPES["none"]:
        return (_ptr(rope_cos, "rope_cos", True), _ptr(rope_sin, "rope_sin", True))
    n = int(rows) * c.qk_rope_head_dim
    return (_ptr(rope_cos, "rope_cos", True, _f32(), n),
            _ptr(rope_sin, "rope_sin", True, _f32(), n))


def _weights(weights, c):
    """ctypes ``mla_weights`` of a mapping (or object) of weight tensors, each
    checked against its [out, in] shape."""
    H, h, rq, r = c.hidden_size, c.num_heads, c.q_lora_rank, c.kv_lora_rank
    dn, dr, dv = c.qk_nope_head_dim, c.qk_rope_head_dim, c.v_head_dim
    sizes = {"w_q_a": rq * H, "g_q_a": rq, "w_q_b": h * (dn + dr) * rq,
             "w_q": h * (dn + dr) * H, "w_kv_a": (r + dr) * H, "g_kv_a": r,
             "w_kv_b": h * (dn + dv) * r, "w_o": H * h * dv}
    w = mla_weights()
    for f, _ in w._fields_:
        t = weights.get(f) if hasattr(weights, "get") else getattr(weights, f)
        setattr(w, f, None if t is None else _ptr(t, f, False, _dt(c), sizes[f]).value)
    return w


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return C.c_void_p(getattr(stream, "cuda_stream", stream))


def abi_version() -> int:
    return _lib.load().mla_abi_version()


def mla_build_rope_tables(cfg, max_pos, cos_out, sin_out, stream=None):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    n = int(max_pos) * c.qk_rope_head_dim
    _check(_lib.load().mla_build_rope_tables(
        C.byref(c), int(max_pos), _ptr(cos_out, "cos_out", False, _f32(), n),
        _ptr(sin_out, "sin_out", False, _f32(), n), _stream(stream)))


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
    w = _weights(weights, c)
    N, H, dt = int(B) * int(T), c.hidden_size, _dt(c)
    cos, sin = _rope_ptrs(c, rope_cos, rope_sin, T)
    _check(_lib.load().mla_prefill_forward(
        C.byref(c), C.byref(w), _ptr(x, "x", False, dt, N * H), int(B), int(T),
        cos, sin, _ptr(out, "out", False, dt, N * H),
        _ptr(latent_cache_out, "latent_cache_out", True, dt,
             N * (c.kv_lora_rank + c.qk_rope_head_dim)),
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


def mla_prefill_chunked(cfg, weights, x, B, T_new, past_cache, T_past, rope_cos,
                        rope_sin, out, workspace, latent_cache_out=None,
                        stream=None):
    """Prefill of T_new tokens after T_past tokens held in ``past_cache``
    ([B, T_past, kv_lora_rank + rope], the latent cache rows)."""
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    w = _weights(weights, c)
    N, H, dt = int(B) * int(T_new), c.hidden_size, _dt(c)
    row = c.kv_lora_rank + c.qk_rope_head_dim
    cos, sin = _rope_ptrs(c, rope_cos, rope_sin, int(T_past) + int(T_new))
    _check(_lib.load().mla_prefill_chunked(
        C.byref(c), C.byref(w), _ptr(x, "x", False, dt, N * H), int(B), int(T_new),
        _ptr(past_cache, "past_cache", True, dt, int(B) * int(T_past) * row), int(T_past),
        cos, sin, _ptr(out, "out", False, dt, N * H),
        _ptr(latent_cache_out, "latent_cache_out", True, dt, N * row),
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
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    w = _weights(weights, c)
    N, H, dt = int(total), c.hidden_size, _dt(c)
    cos, sin = _rope_ptrs(c, rope_cos, rope_sin, max_seqlen)
    _check(_lib.load().mla_prefill_varlen(
        C.byref(c), C.byref(w), _ptr(x, "x", False, dt, N * H),
        _ptr(cu_seqlens, "cu_seqlens", False, _i32(), int(n_seq) + 1), int(n_seq),
        int(total), int(max_seqlen), cos, sin, _ptr(out, "out", False, dt, N * H),
        _ptr(latent_cache_out, "latent_cache_out", True, dt,
             N * (c.kv_lora_rank + c.qk_rope_head_dim)),
        _ptr(workspace, "workspace"),
        C.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def mla_decode_workspace_size(cfg, B, max_ctx):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    lay = mla_decode_layout()
    n = _lib.load().mla_decode_workspace_size(C.byref(c), int(B), int(max_ctx),
                                              C.byref(lay))
    if n == 0:
        raise MlaError(2, "invalid configuration or sizes")
    return n, {f: getattr(lay, f) for f, _ in lay._fields_}


def _decode_ptrs(c, q_nope, q_pe, w_kv_b, latent_cache, cu_ctx, B, w_o, out):
    """Checked pointers of the decode tensors.  The cache's row count lives in
    cu_ctx on the device, so only its dtype and row width are checked."""
    B, h, r, dt = int(B), c.num_heads, c.kv_lora_rank, _dt(c)
    dn, dr, dv, H = c.qk_nope_head_dim, c.qk_rope_head_dim, c.v_head_dim, c.hidden_size
    return (_ptr(q_nope, "q_nope", False, dt, B * h * dn),
            _ptr(q_pe, "q_pe", False, dt, B * h * dr),
            _ptr(w_kv_b, "w_kv_b", False, dt, h * (dn + dv) * r),
            _ptr(latent_cache, "latent_cache", False, dt, None, r + dr),
            _ptr(cu_ctx, "cu_ctx", False, _i32(), B + 1),
            _ptr(w_o, "w_o", True, dt, H * h * dv),
            _ptr(out, "out", False, dt, B * (H if w_o is not None else h * dv)))


def mla_decode_absorbed(cfg, q_nope, q_pe, w_kv_b, latent_cache, cu_ctx, B,
                        max_ctx, w_o, out, workspace, stream=None):
    c = cfg if isinstance(cfg, mla_config) else make_config(cfg)
    qn, qp, wkvb, cache, cu, wo, o = _decode_ptrs(c, q_nope, q_pe, w_kv_b, latent_cache,
                                                   cu_ctx, B, w_o, out)
    _check(_lib.load().mla_decode_absorbed(
        C.byref(c), qn, qp, wkvb, cache, cu, int(B), int(max_ctx), wo, o,
        _ptr(workspace, "workspace"),
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
    qn, qp, wkvb, cache, cu, wo, o = _decode_ptrs(c, q_nope, q_pe, w_kv_b, latent_cache,
                                                   cu_ctx, B, w_o, out)
    _check(_lib.load().mla_decode_absorbed_noalloc(
        C.byref(c), qn, qp, wkvb, cache, cu, int(B), int(max_ctx), wo, o,
        _stream(stream)))

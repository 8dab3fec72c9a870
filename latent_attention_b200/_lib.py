"""ctypes view of ``include/mla.h`` and the loader of ``libmla_b200.so``.

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  If the shared library is missing this module raises -- there
is no fallback implementation.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# MLA_B200_LIB: another build of the same library (for example a variant to
# compare against); the default is the in-tree build.
LIB_PATH = os.environ.get("MLA_B200_LIB") or os.path.join(HERE, "libmla_b200.so")

MLA_OK = 0
STATUS_NAMES = {0: "MLA_OK", 1: "MLA_ERR_NULL", 2: "MLA_ERR_SHAPE",
                3: "MLA_ERR_ALIGN", 4: "MLA_ERR_DTYPE", 5: "MLA_ERR_WORKSPACE",
                6: "MLA_ERR_UNSUPPORTED", 7: "MLA_ERR_CUDA",
                8: "MLA_ERR_DEVICE_TIMEOUT"}
MLA_F32, MLA_BF16 = 0, 1
# Size of the library's static decode scratch (mla.h MLA_DECODE_NOALLOC_SCRATCH_BYTES).
DECODE_NOALLOC_SCRATCH_BYTES = 16 << 20
ROPE_TYPES = {"none": 0, "plain": 1, "yarn": 2}

# Every symbol the header declares (checked by the CPU tests).
EXPORTED = ["mla_abi_version", "mla_status_string", "mla_last_error_detail",
            "mla_build_rope_tables", "mla_prefill_workspace_size",
            "mla_prefill_forward", "mla_decode_workspace_size",
            "mla_decode_absorbed", "mla_check_device_status",
            "mla_set_stage_events", "mla_kernel_launches",
            "mla_decode_absorbed_noalloc", "mla_selftest_wait_timeout",
            "mla_prefill_chunked_workspace_size", "mla_prefill_chunked",
            "mla_prefill_varlen_workspace_size", "mla_prefill_varlen"]


class mla_config(C.Structure):
    _fields_ = [("hidden_size", C.c_int32), ("num_heads", C.c_int32),
                ("q_lora_rank", C.c_int32), ("kv_lora_rank", C.c_int32),
                ("qk_nope_head_dim", C.c_int32), ("qk_rope_head_dim", C.c_int32),
                ("v_head_dim", C.c_int32), ("rope_type", C.c_int32),
                ("rope_theta", C.c_double), ("rope_factor", C.c_double),
                ("rope_mscale", C.c_double), ("rope_mscale_all_dim", C.c_double),
                ("beta_fast", C.c_double), ("beta_slow", C.c_double),
                ("original_max_position_embeddings", C.c_int32),
                ("dtype", C.c_int32), ("rms_eps", C.c_double),
                ("softmax_scale", C.c_double), ("rope_interleave", C.c_int32)]


class mla_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("w_q_a", "g_q_a", "w_q_b", "w_q", "w_kv_a", "g_kv_a",
                 "w_kv_b", "w_o")]


class mla_prefill_layout(C.Structure):
    _fields_ = [(n, C.c_int64) for n in
                ("status", "ssq_q", "ssq_kv", "q_a", "ckv", "q", "kv", "attn",
                 "total_bytes", "latent", "pos")]


class mla_decode_layout(C.Structure):
    _fields_ = [(n, C.c_int64) for n in
                ("status", "q_lat", "part_o", "part_lse", "o_lat", "o",
                 "total_bytes")] + [("split_tokens", C.c_int32),
                                    ("max_splits", C.c_int32)]


_lib = None


def load():
    """Load the library once.  Raises FileNotFoundError when it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FileNotFoundError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m latent_attention_b200.build` (no fallback exists)")
    lib = C.CDLL(LIB_PATH)
    vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
    cfgp = C.POINTER(mla_config)
    lib.mla_abi_version.restype = i32
    lib.mla_abi_version.argtypes = []
    lib.mla_status_string.restype = C.c_char_p
    lib.mla_status_string.argtypes = [C.c_int]
    lib.mla_last_error_detail.restype = C.c_char_p
    lib.mla_last_error_detail.argtypes = []
    lib.mla_build_rope_tables.restype = C.c_int
    lib.mla_build_rope_tables.argtypes = [cfgp, i32, vp, vp, vp]
    lib.mla_prefill_workspace_size.restype = sz
    lib.mla_prefill_workspace_size.argtypes = [cfgp, i32, i32,
                                               C.POINTER(mla_prefill_layout)]
    lib.mla_prefill_forward.restype = C.c_int
    lib.mla_prefill_forward.argtypes = [cfgp, C.POINTER(mla_weights), vp, i32,
                                        i32, vp, vp, vp, vp, vp, sz, vp]
    lib.mla_decode_workspace_size.restype = sz
    lib.mla_decode_workspace_size.argtypes = [cfgp, i32, i32,
                                              C.POINTER(mla_decode_layout)]
    lib.mla_decode_absorbed.restype = C.c_int
    lib.mla_decode_absorbed.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, i32, vp,
                                        vp, vp, sz, vp]
    lib.mla_check_device_status.restype = C.c_int
    lib.mla_check_device_status.argtypes = [vp, vp]
    lib.mla_set_stage_events.restype = C.c_int
    lib.mla_set_stage_events.argtypes = [C.POINTER(vp), i32]
    lib.mla_kernel_launches.restype = C.c_int64
    lib.mla_kernel_launches.argtypes = []
    lib.mla_prefill_chunked_workspace_size.restype = sz
    lib.mla_prefill_chunked_workspace_size.argtypes = [cfgp, i32, i32, i32,
                                                       C.POINTER(mla_prefill_layout)]
    lib.mla_prefill_chunked.restype = C.c_int
    lib.mla_prefill_chunked.argtypes = [cfgp, C.POINTER(mla_weights), vp, i32, i32, vp,
                                        i32, vp, vp, vp, vp, vp, sz, vp]
    lib.mla_prefill_varlen_workspace_size.restype = sz
    lib.mla_prefill_varlen_workspace_size.argtypes = [cfgp, i32, i32, i32,
                                                      C.POINTER(mla_prefill_layout)]
    lib.mla_prefill_varlen.restype = C.c_int
    lib.mla_prefill_varlen.argtypes = [cfgp, C.POINTER(mla_weights), vp, vp, i32, i32, i32,
                                       vp, vp, vp, vp, vp, sz, vp]
    lib.mla_selftest_wait_timeout.restype = C.c_int
    lib.mla_selftest_wait_timeout.argtypes = [vp, vp]
    lib.mla_decode_absorbed_noalloc.restype = C.c_int
    lib.mla_decode_absorbed_noalloc.argtypes = [cfgp, vp, vp, vp, vp, vp, i32, i32, vp,
                                                vp, vp]
    _lib = lib
    return lib

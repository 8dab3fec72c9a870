"""C ABI checks that need no GPU: the library loads, exports every symbol the
header declares, the ctypes structs match the C layout, and host-side
validation rejects bad arguments before any launch."""
import ctypes as C
import os
import re
import subprocess
import tempfile

import pytest

from conftest import ROOT
from mla_inputs import WORKLOADS

HEADER = os.path.join(ROOT, "include", "mla.h")


@pytest.fixture(scope="module")
def lib():
    from latent_attention_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from latent_attention_b200 import build
        build.build()
    return _lib.load()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", txt)))


def test_header_declares_the_binding_list():
    from latent_attention_b200 import _lib
    assert declared_symbols() == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only",
                          os.path.join(ROOT, "latent_attention_b200",
                                        "libmla_b200.so")],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r" T (mla_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_abi_version_and_status_strings(lib):
    assert lib.mla_abi_version() == 4
    for code, name in {0: b"MLA_OK", 5: b"MLA_ERR_WORKSPACE",
                       8: b"MLA_ERR_DEVICE_TIMEOUT"}.items():
        assert lib.mla_status_string(code) == name


def _c_layout():
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "mla.h"
#define P(T, f) printf(#T "." #f " %zu\n", offsetof(T, f));
int main(void) {
  printf("mla_config %zu\n", sizeof(mla_config));
  printf("mla_weights %zu\n", sizeof(mla_weights));
  printf("mla_prefill_layout %zu\n", sizeof(mla_prefill_layout));
  printf("mla_decode_layout %zu\n", sizeof(mla_decode_layout));
  P(mla_config, rope_theta) P(mla_config, original_max_position_embeddings)
  P(mla_config, dtype) P(mla_config, rms_eps) P(mla_config, softmax_scale)
  P(mla_weights, w_o) P(mla_decode_layout, split_tokens) P(mla_prefill_layout, latent)
  P(mla_prefill_layout, pos) P(mla_config, rope_interleave)
  P(mla_decode_layout, max_splits)
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "l.c"), os.path.join(d, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe],
                       check=True)
        out = subprocess.run([exe], capture_output=True, text=True,
                             check=True).stdout
    return {k: int(v) for k, v in (l.split() for l in out.splitlines())}


def test_ctypes_structs_match_c_layout():
    from latent_attention_b200 import _lib
    L = _c_layout()
    assert C.sizeof(_lib.mla_config) == L["mla_config"]
    assert C.sizeof(_lib.mla_weights) == L["mla_weights"]
    assert C.sizeof(_lib.mla_prefill_layout) == L["mla_prefill_layout"]
    assert C.sizeof(_lib.mla_decode_layout) == L["mla_decode_layout"]
    for k, v in L.items():
        if "." in k:
            t, f = k.split(".")
            assert getattr(getattr(_lib, t), f).offset == v, k


def test_workspace_sizes_are_host_logic(lib):
    from latent_attention_b200 import mla_prefill_workspace_size, \
        mla_decode_workspace_size
    cfg = WORKLOADS["dsv3_prefill"].cfg
    n, lay = mla_prefill_workspace_size(cfg, 1, 4096)
    N = 4096
    assert lay["q"] % 256 == 0 and lay["kv"] % 256 == 0
    assert n >= N * 128 * (192 + 256 + 128) * 2
    assert lay["total_bytes"] == n
    cfg3 = WORKLOADS["directq_prefill"].cfg
    _, lay3 = mla_prefill_workspace_size(cfg3, 4, 8192)
    assert lay3["q_a"] == -1 and lay3["ssq_q"] == -1
    dcfg = WORKLOADS["dsv3_decode"].cfg
    nd, dl = mla_decode_workspace_size(dcfg, 64, 32768)
    # tensor cores: a slice of >= 512 tokens per SM pair, two partial slots per
    # pair, independent of B and max_ctx (148 SMs when no device is visible)
    assert dl["split_tokens"] == 512 and dl["max_splits"] % 2 == 0 and dl["max_splits"] > 0
    assert dl["part_lse"] - dl["part_o"] >= dl["max_splits"] * 128 * 512 * 4
    assert nd == dl["total_bytes"]
    nd2, dl2 = mla_decode_workspace_size(dcfg, 1, 1 << 20)
    assert dl2["max_splits"] == dl["max_splits"] and nd2 < nd
    # other configurations: 1024-token splits of every sequence
    _, dl3 = mla_decode_workspace_size(WORKLOADS["tiny_f32"].cfg, 3, 4000)
    assert dl3["split_tokens"] == 1024 and dl3["max_splits"] == 4


def _fake(addr):
    return C.c_void_p(addr)


def test_validation_rejects_before_launch(lib):
    """Invalid calls return an error without touching a device (there is none
    here, so a launch would fail with MLA_ERR_CUDA instead)."""
    from latent_attention_b200 import make_config, mla_weights
    from latent_attention_b200._lib import mla_config
    cfg = WORKLOADS["dsv3_prefill"].cfg
    c = make_config(cfg)
    w = mla_weights()
    for i, f in enumerate(("w_q_a", "w_q_b", "w_kv_a", "w_kv_b", "w_o")):
        setattr(w, f, 0x100000 + i * 0x1000)
    x, out, cs = _fake(0x200000), _fake(0x300000), _fake(0x400000)
    ws = _fake(0x1000000)
    big = C.c_size_t(1 << 40)
    f = lib.mla_prefill_forward
    assert f(None, C.byref(w), x, 1, 8, cs, cs, out, None, ws, big, None) == 1
    assert f(C.byref(c), C.byref(w), None, 1, 8, cs, cs, out, None, ws, big, None) == 1
    assert f(C.byref(c), C.byref(w), x, 0, 8, cs, cs, out, None, ws, big, None) == 2
    assert f(C.byref(c), C.byref(w), _fake(0x200002), 1, 8, cs, cs, out, None,
             ws, big, None) == 3
    assert f(C.byref(c), C.byref(w), x, 1, 8, cs, cs, out, None, _fake(0x1000010),
             big, None) == 3
    assert f(C.byref(c), C.byref(w), x, 1, 8, cs, cs, out, None, ws,
             C.c_size_t(1024), None) == 5
    assert b"workspace" in lib.mla_last_error_detail()
    assert f(C.byref(c), C.byref(w), x, 1, 8, None, None, out, None, ws, big,
             None) == 1                                   # yarn needs tables
    bad = mla_config.from_buffer_copy(c)
    bad.dtype = 7
    assert f(C.byref(bad), C.byref(w), x, 1, 8, cs, cs, out, None, ws, big, None) == 4
    bad = mla_config.from_buffer_copy(c)
    bad.qk_rope_head_dim = 63
    assert f(C.byref(bad), C.byref(w), x, 1, 8, cs, cs, out, None, ws, big, None) == 2
    w2 = mla_weights.from_buffer_copy(w)
    w2.w_q_b = None
    assert f(C.byref(c), C.byref(w2), x, 1, 8, cs, cs, out, None, ws, big, None) == 1
    d = lib.mla_decode_absorbed
    p = _fake(0x500000)
    assert d(C.byref(c), p, p, p, p, p, 4, 0, None, p, ws, big, None) == 2
    assert d(C.byref(c), p, p, p, None, p, 4, 16, None, p, ws, big, None) == 1
    assert d(C.byref(c), p, p, p, p, p, 4, 16, None, p, ws, C.c_size_t(8), None) == 5
    r = lib.mla_build_rope_tables
    assert r(C.byref(c), 0, p, p, None) == 2
    assert r(C.byref(c), 16, _fake(0x500004), p, None) == 3


def test_binding_refuses_cpu_tensors(lib):
    import torch
    from latent_attention_b200 import mla_build_rope_tables
    cfg = WORKLOADS["tiny_f32"].cfg
    t = torch.empty(4, 16)
    with pytest.raises(ValueError, match="CUDA"):
        mla_build_rope_tables(cfg, 4, t, t)


def test_chunked_prefill_validation_and_sizes(lib):
    from latent_attention_b200 import (make_config, mla_weights,
                                       mla_prefill_workspace_size,
                                       mla_prefill_chunked_workspace_size)
    cfg = WORKLOADS["dsv3_prefill"].cfg
    # no history: the same workspace as a plain prefill
    n0, _ = mla_prefill_workspace_size(cfg, 2, 300)
    n1, l1 = mla_prefill_chunked_workspace_size(cfg, 2, 300, 0)
    assert n0 == n1 and l1["latent"] == -1
    # history: latent rows and kv cover T_past + T_new rows per sequence
    n2, l2 = mla_prefill_chunked_workspace_size(cfg, 2, 300, 1000)
    w = cfg.kv_lora_rank + cfg.qk_rope_head_dim
    assert l2["latent"] >= 0 and n2 >= n1 + 2 * 1300 * w * 2
    c = make_config(cfg)
    wt = mla_weights()
    for i, f in enumerate(("w_q_a", "g_q_a", "w_q_b", "w_kv_a", "g_kv_a",
                           "w_kv_b", "w_o")):
        setattr(wt, f, 0x100000 + i * 0x1000)
    p, ws, big = _fake(0x200000), _fake(0x1000000), C.c_size_t(1 << 40)
    f = lib.mla_prefill_chunked
    assert f(C.byref(c), C.byref(wt), p, 1, 8, None, 4, p, p, p, None, ws, big,
             None) == 1                                 # history without cache
    assert f(C.byref(c), C.byref(wt), p, 1, 8, p, -1, p, p, p, None, ws, big,
             None) == 2
    assert f(C.byref(c), C.byref(wt), p, 1, 8, _fake(0x200008), 4, p, p, p, None,
             ws, big, None) == 3


def test_varlen_prefill_validation_and_sizes(lib):
    from latent_attention_b200 import (make_config, mla_weights,
                                       mla_prefill_workspace_size,
                                       mla_prefill_varlen_workspace_size)
    cfg = WORKLOADS["dsv3_prefill"].cfg
    n0, l0 = mla_prefill_workspace_size(cfg, 1, 1000)
    n1, l1 = mla_prefill_varlen_workspace_size(cfg, 7, 1000, 300)
    assert l0["pos"] == -1 and l1["pos"] >= 0 and n1 >= n0 + 1000 * 4
    for bad in ((0, 10, 5), (2, 0, 1), (2, 10, 11), (2, 10, 0)):
        with pytest.raises(Exception):
            mla_prefill_varlen_workspace_size(cfg, *bad)
    c = make_config(cfg)
    wt = mla_weights()
    for i, f in enumerate(("w_q_a", "g_q_a", "w_q_b", "w_kv_a", "g_kv_a",
                           "w_kv_b", "w_o")):
        setattr(wt, f, 0x100000 + i * 0x1000)
    p, ws, big = _fake(0x200000), _fake(0x1000000), C.c_size_t(1 << 40)
    f = lib.mla_prefill_varlen
    assert f(C.byref(c), C.byref(wt), p, None, 2, 10, 5, p, p, p, None, ws, big, None) == 1
    assert f(C.byref(c), C.byref(wt), p, _fake(0x300002), 2, 10, 5, p, p, p, None, ws, big,
             None) == 3
    assert f(C.byref(c), C.byref(wt), p, p, 2, 10, 11, p, p, p, None, ws, big, None) == 2
    assert f(C.byref(c), C.byref(wt), p, p, 0, 10, 5, p, p, p, None, ws, big, None) == 2
    assert f(C.byref(c), C.byref(wt), p, p, 2, 10, 5, p, p, p, None, ws, C.c_size_t(64),
             None) == 5


@pytest.mark.parametrize("field,value", [("qk_nope_head_dim", 64), ("qk_rope_head_dim", 32),
                                         ("v_head_dim", 64), ("kv_lora_rank", 256),
                                         ("hidden_size", 7164)])
def test_bf16_shapes_off_the_tensor_cores_are_unsupported(lib, field, value):
    """bf16 runs on the tensor-core kernels only: a bf16 shape they do not
    take is refused with MLA_ERR_UNSUPPORTED before any launch (no device is
    present here, so a launch would come back as MLA_ERR_CUDA)."""
    from latent_attention_b200 import make_config, mla_weights
    from latent_attention_b200._lib import mla_config
    c = mla_config.from_buffer_copy(make_config(WORKLOADS["dsv3_prefill"].cfg))
    setattr(c, field, value)
    w = mla_weights()
    for i, f in enumerate(("w_q_a", "w_q_b", "w_kv_a", "w_kv_b", "w_o")):
        setattr(w, f, 0x100000 + i * 0x1000)
    p, ws, big = _fake(0x200000), _fake(0x1000000), C.c_size_t(1 << 40)
    r = lib.mla_prefill_forward(C.byref(c), C.byref(w), p, 1, 8, p, p, p, None, ws, big, None)
    if field == "kv_lora_rank":                   # prefill takes multiples of 64
        assert r != 6
    else:
        assert r == 6 and b"bf16 prefill" in lib.mla_last_error_detail()
    dec_unsupported = field in ("qk_rope_head_dim", "kv_lora_rank")
    # decode: kv_lora_rank 512 and rope 64; hidden_size matters with o_proj only
    r = lib.mla_decode_absorbed(C.byref(c), p, p, p, p, p, 4, 16,
                                p if field == "hidden_size" else None, p, ws, big, None)
    if dec_unsupported or field == "hidden_size":
        assert r == 6 and b"bf16 decode" in lib.mla_last_error_detail()
    # the fp32 configuration of the same shape stays on the CUDA-core path
    c.dtype = 0
    if field not in ("hidden_size", "kv_lora_rank"):
        assert lib.mla_prefill_forward(C.byref(c), C.byref(w), p, 1, 8, p, p, p, None, ws,
                                       big, None) != 6

"""C-ABI boundary checks that need no GPU.

The shared library must load, export every function include/gqa_decode.h
declares, and reject invalid arguments on the host before touching CUDA.
Nothing here launches a kernel.
"""

import ctypes
import json
import os
import re

import pytest

import gqa_mqa_kv_b200 as gq
from gqa_mqa_kv_b200 import build as gq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_decode.h")

GQA_OK, GQA_ERR_INVALID, GQA_ERR_UNSUPPORTED, GQA_ERR_CUDA, GQA_ERR_WORKSPACE = range(5)


@pytest.fixture(scope="module")
def lib():
    gq_build.build()
    return gq.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(gqa_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_expected_entry_points():
    assert set(declared_functions()) == set(gq.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_built_for_sm100a():
    cmd = gq_build.command("x.so")
    assert "arch=compute_100a,code=sm_100a" in cmd


def test_version(lib):
    assert lib.gqa_version() == 1


def test_status_strings(lib):
    for code in range(5):
        assert lib.gqa_status_string(code)
    assert lib.gqa_status_string(99) == b"unknown status"


def test_kv_cache_bytes_matches_printed_table(lib):
    with open(os.path.join(ROOT, "tests", "golden", "kv_cache_table_70b.json")) as f:
        gold = json.load(f)
    m = gold["model"]
    for row in gold["rows"]:
        for col, h_kv in (("MHA_H_KV_64", 64), ("GQA8_H_KV_8", 8), ("MQA_H_KV_1", 1)):
            b = gq.kv_cache_bytes(m["layers"], row["tokens"], h_kv, m["d_k"], m["elem_bytes"])
            assert round(b / 1e9, 2) == pytest.approx(row[col], abs=1e-9)


def params(**kw):
    p = gq.Params()
    base = dict(B=2, H_Q=8, H_KV=2, head_dim=128, max_seq_len=256, page_size=0,
                max_blocks_per_seq=0, num_blocks=0, qkv_dtype=0, out_dtype=1)
    base.update(kw)
    for k, v in base.items():
        setattr(p, k, v)
    return p


def call_decode(lib, p, q=16, k=16, v=16, lens=16, table=None, out=16, ws=256, ws_bytes=1 << 20,
                scale=0.1):
    vp = ctypes.c_void_p
    return lib.gqa_decode(ctypes.byref(p), vp(q), vp(k), vp(v), vp(lens), vp(table),
                          ctypes.c_float(scale), vp(out), vp(ws), ctypes.c_size_t(ws_bytes), vp(None))


@pytest.mark.parametrize(
    "kw,expected",
    [
        (dict(H_Q=6, H_KV=4), GQA_ERR_INVALID),          # R not whole
        (dict(H_KV=0), GQA_ERR_INVALID),
        (dict(B=-1), GQA_ERR_INVALID),
        (dict(max_seq_len=-3), GQA_ERR_INVALID),
        (dict(head_dim=96), GQA_ERR_UNSUPPORTED),
        (dict(page_size=32), GQA_ERR_UNSUPPORTED),
        (dict(qkv_dtype=7), GQA_ERR_INVALID),
        (dict(out_dtype=3), GQA_ERR_INVALID),
        (dict(page_size=64, max_blocks_per_seq=0, num_blocks=4), GQA_ERR_INVALID),
        (dict(page_size=64, max_blocks_per_seq=2, num_blocks=4, max_seq_len=129), GQA_ERR_INVALID),
        (dict(max_blocks_per_seq=3), GQA_ERR_INVALID),   # block fields on a contiguous cache
        (dict(kernel=3), GQA_ERR_INVALID),               # no such gqa_kernel
        (dict(kernel=-1), GQA_ERR_INVALID),
    ],
)
def test_invalid_params_rejected_on_host(lib, kw, expected):
    p = params(**kw)
    assert call_decode(lib, p) == expected
    n = ctypes.c_size_t(0)
    assert lib.gqa_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)) == expected


def test_null_and_misaligned_pointers_rejected(lib):
    p = params()
    assert call_decode(lib, p, q=None) == GQA_ERR_INVALID
    assert call_decode(lib, p, lens=None) == GQA_ERR_INVALID
    assert call_decode(lib, p, out=None) == GQA_ERR_INVALID
    assert call_decode(lib, p, k=24) == GQA_ERR_INVALID       # TMA needs 16-byte alignment
    assert call_decode(lib, p, out=12) == GQA_ERR_INVALID
    assert call_decode(lib, p, table=16) == GQA_ERR_INVALID   # table given for a contiguous cache
    pp = params(page_size=64, max_blocks_per_seq=4, num_blocks=8)
    assert call_decode(lib, pp, table=None) == GQA_ERR_INVALID
    assert call_decode(lib, p, scale=float("nan")) == GQA_ERR_INVALID


@pytest.mark.parametrize(
    "kw",
    [
        dict(kernel=2, head_dim=64),                    # tcgen05 serves head_dim 128 only
        dict(kernel=2, H_Q=64, H_KV=1),                 # R = 64 > 32
        dict(kernel=2, qkv_dtype=1),                    # f32 cache: CUDA cores only
        dict(kernel=1, qkv_dtype=1),
        dict(kernel=1, H_Q=128, H_KV=1),                # R = 128 > 64
    ],
)
def test_unsupported_kernel_choice_refused_on_host(lib, kw):
    assert call_decode(lib, params(**kw)) == GQA_ERR_UNSUPPORTED


def test_fp8_kernel_choice_limits(lib):
    vp = ctypes.c_void_p

    def call(p):
        return lib.gqa_decode_fp8kv(ctypes.byref(p), vp(16), vp(16), vp(16), vp(64), vp(64), vp(16), vp(None),
                                    ctypes.c_float(0.1), vp(16), vp(256), ctypes.c_size_t(1 << 20), vp(None))

    assert call(params(kernel=1, H_Q=32, H_KV=2)) == GQA_ERR_UNSUPPORTED  # mma.sync 8-bit path: R <= 8
    assert call(params(kernel=2, H_Q=128, H_KV=2)) == GQA_ERR_UNSUPPORTED  # tcgen05: R <= 32


def test_empty_batch_is_a_no_op(lib):
    assert call_decode(lib, params(B=0), q=None, k=None, v=None, lens=None, out=None) == GQA_OK


def test_read_status_rejects_nulls(lib):
    flags = ctypes.c_uint32(0)
    assert lib.gqa_read_status(None, None, ctypes.byref(flags), 0) == GQA_ERR_INVALID
    assert lib.gqa_read_status(ctypes.c_void_p(256), None, None, 0) == GQA_ERR_INVALID
    # the built-in workspace's reader checks its output pointer before touching a device
    assert lib.gqa_static_workspace_status(None, None, 0) == GQA_ERR_INVALID


def test_binding_refuses_host_tensors():
    import torch

    q = torch.zeros(1, 8, 64)
    k = torch.zeros(1, 16, 2, 64)
    with pytest.raises(ValueError):
        gq.gqa_decode(q, k, k, torch.ones(1, dtype=torch.int32))


def test_package_does_not_import_the_oracle():
    import sys
    import subprocess

    code = ("import sys, gqa_mqa_kv_b200, gqa_mqa_kv_b200.workloads;"
            "assert 'oracle' not in sys.modules, 'product imported the oracle'")
    subprocess.run([sys.executable, "-c", code], check=True, cwd=ROOT)
    for dirpath, _, files in os.walk(os.path.join(ROOT, "gqa_mqa_kv_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "gqa_oracle" not in text, f


def call_rope(lib, p, q=16, kn=16, vn=16, pos=16, table=None, base=10000.0, pairing=0, qo=16, kc=16,
              vc=16, lens_out=None, ws=None):
    vp = ctypes.c_void_p
    return lib.gqa_rope_append(ctypes.byref(p), vp(q), vp(kn), vp(vn), vp(pos), vp(table),
                               ctypes.c_double(base), pairing, vp(qo), vp(kc), vp(vc), vp(lens_out), vp(ws),
                               vp(None))


def test_rope_append_rejects_bad_arguments_on_host(lib):
    p = params()
    assert call_rope(lib, params(H_Q=6, H_KV=4)) == GQA_ERR_INVALID
    assert call_rope(lib, p, base=0.0) == GQA_ERR_INVALID
    assert call_rope(lib, p, base=float("nan")) == GQA_ERR_INVALID
    assert call_rope(lib, p, pairing=2) == GQA_ERR_INVALID
    assert call_rope(lib, p, kn=None) == GQA_ERR_INVALID
    assert call_rope(lib, p, pos=None) == GQA_ERR_INVALID
    assert call_rope(lib, p, kc=24) == GQA_ERR_INVALID
    assert call_rope(lib, p, table=16) == GQA_ERR_INVALID           # table on a contiguous cache
    assert call_rope(lib, p, pos=4096, lens_out=4100) == GQA_ERR_INVALID  # overlapping int32 [B]
    assert call_rope(lib, p, ws=128) == GQA_ERR_WORKSPACE
    assert call_rope(lib, params(B=0), q=None, kn=None, vn=None, pos=None, qo=None, kc=None,
                     vc=None) == GQA_OK


def test_fp8kv_rejects_bad_arguments_on_host(lib):
    vp = ctypes.c_void_p

    def call(p, ks=64, vs=64, q=16):
        return lib.gqa_decode_fp8kv(ctypes.byref(p), vp(q), vp(16), vp(16), vp(ks), vp(vs), vp(16), vp(None),
                                    ctypes.c_float(0.1), vp(16), vp(256), ctypes.c_size_t(1 << 20), vp(None))

    assert call(params(), ks=None) == GQA_ERR_INVALID
    assert call(params(), vs=None) == GQA_ERR_INVALID
    assert call(params(), ks=66) == GQA_ERR_INVALID          # misaligned float array
    assert call(params(qkv_dtype=1)) == GQA_ERR_UNSUPPORTED  # q must be bf16
    assert call(params(H_Q=6, H_KV=4)) == GQA_ERR_INVALID


def test_wait_selftest_rejects_bad_arguments_on_host(lib):
    vp = ctypes.c_void_p
    assert lib.gqa_wait_selftest(ctypes.c_uint64(0), 0, vp(16), vp(16), vp(None)) == GQA_ERR_INVALID
    assert lib.gqa_wait_selftest(ctypes.c_uint64(10**11), 0, vp(16), vp(16), vp(None)) == GQA_ERR_INVALID
    assert lib.gqa_wait_selftest(ctypes.c_uint64(10**6), 0, vp(None), vp(16), vp(None)) == GQA_ERR_INVALID
    assert lib.gqa_wait_selftest(ctypes.c_uint64(10**6), 0, vp(16), vp(12), vp(None)) == GQA_ERR_INVALID


def call_prefill(lib, p, q=16, cu=16, total_q=10, max_q=10, k=16, v=16, lens=16, table=None, scale=0.1,
                 out=16, ws=256, ws_bytes=256):
    vp = ctypes.c_void_p
    return lib.gqa_prefill(ctypes.byref(p), vp(q), vp(cu), total_q, max_q, vp(k), vp(v), vp(lens), vp(table),
                           ctypes.c_float(scale), vp(out), vp(ws), ctypes.c_size_t(ws_bytes), vp(None))


def test_prefill_refuses_unsupported_problems_on_host(lib):
    assert call_prefill(lib, params(head_dim=64)) == GQA_ERR_UNSUPPORTED
    assert call_prefill(lib, params(qkv_dtype=1)) == GQA_ERR_UNSUPPORTED      # bf16 only
    assert call_prefill(lib, params(kernel=1)) == GQA_ERR_UNSUPPORTED         # tcgen05 only
    assert call_prefill(lib, params(H_Q=256, H_KV=1)) == GQA_ERR_UNSUPPORTED  # R > 128
    assert call_prefill(lib, params(H_Q=6, H_KV=4)) == GQA_ERR_INVALID


def test_prefill_rejects_bad_arguments_on_host(lib):
    p = params()
    assert call_prefill(lib, p, total_q=-1) == GQA_ERR_INVALID
    assert call_prefill(lib, p, max_q=-1) == GQA_ERR_INVALID
    assert call_prefill(lib, p, q=None) == GQA_ERR_INVALID
    assert call_prefill(lib, p, cu=None) == GQA_ERR_INVALID
    assert call_prefill(lib, p, lens=None) == GQA_ERR_INVALID
    assert call_prefill(lib, p, out=None) == GQA_ERR_INVALID
    assert call_prefill(lib, p, q=24) == GQA_ERR_INVALID           # TMA needs 16-byte alignment
    assert call_prefill(lib, p, out=8) == GQA_ERR_INVALID          # 16-byte vector stores
    assert call_prefill(lib, p, cu=18) == GQA_ERR_INVALID
    assert call_prefill(lib, p, table=16) == GQA_ERR_INVALID       # table given for a contiguous cache
    pp = params(page_size=64, max_blocks_per_seq=4, num_blocks=8)
    assert call_prefill(lib, pp, table=None) == GQA_ERR_INVALID
    assert call_prefill(lib, p, scale=float("nan")) == GQA_ERR_INVALID
    assert call_prefill(lib, p, scale=0.0) == GQA_ERR_INVALID       # the scale must be positive
    assert call_prefill(lib, p, scale=-0.1) == GQA_ERR_INVALID
    assert call_prefill(lib, p, scale=float("inf")) == GQA_ERR_INVALID
    assert call_prefill(lib, p, ws=None) == GQA_ERR_WORKSPACE
    assert call_prefill(lib, p, ws=128) == GQA_ERR_WORKSPACE       # not 256-byte aligned
    assert call_prefill(lib, p, ws_bytes=64) == GQA_ERR_WORKSPACE   # no room for the status word


def test_prefill_with_nothing_to_do_is_a_no_op(lib):
    none = dict(q=None, cu=None, k=None, v=None, lens=None, out=None, ws=None)
    assert call_prefill(lib, params(B=0), **none) == GQA_OK
    assert call_prefill(lib, params(), total_q=0, **none) == GQA_OK
    assert call_prefill(lib, params(), max_q=0, **none) == GQA_OK


def test_prefill_workspace_size(lib):
    n = ctypes.c_size_t(0)
    assert lib.gqa_prefill_workspace_size(ctypes.byref(params()), ctypes.byref(n)) == GQA_OK
    assert n.value == 256
    assert lib.gqa_prefill_workspace_size(ctypes.byref(params(H_Q=6, H_KV=4)), ctypes.byref(n)) == GQA_ERR_INVALID

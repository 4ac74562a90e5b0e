"""gqa_decode_static_workspace: decode with the library's own fixed workspace.

Some callers cannot call cudaMalloc -- for example a plugin whose host
application has already handed all device memory to its own pool, or a
latency-critical loop that must not take cudaMalloc's implicit device-wide
synchronisation.  For them the library offers one entry point that allocates
nothing and uses an 8 MiB array built into the library as its workspace.

These tests call that entry point through the C ABI (ctypes, no workspace
argument) and compare it with gqa_decode run on a caller-allocated
workspace, within the same tolerance the parity tests use, on two calls in a
row with different inputs.  The file is named so that pytest collects it last.
"""

import ctypes
import dataclasses
import math

import numpy as np
import pytest
import torch

import gqa_mqa_kv_b200 as gq
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import ATOL, RTOL, errors, to_device

pytestmark = pytest.mark.gpu

GQA_ERR_WORKSPACE = 4


def call_static(d, paged, out, scale):
    k = d["k_paged"] if paged else d["k"]
    v = d["v_paged"] if paged else d["v"]
    table = d["block_table"] if paged else None
    params = gq.make_params(d["q"], k, d["seq_lens"], table, out.dtype)
    lib = gq.library()
    st = lib.gqa_decode_static_workspace(
        ctypes.byref(params), ctypes.c_void_p(d["q"].data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(d["seq_lens"].data_ptr()),
        ctypes.c_void_p(table.data_ptr() if table is not None else None), ctypes.c_float(scale),
        ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream(out.device).cuda_stream))
    return st


def call_reference(d, paged, scale):
    k = d["k_paged"] if paged else d["k"]
    v = d["v_paged"] if paged else d["v"]
    table = d["block_table"] if paged else None
    ws = torch.zeros(gq.workspace_bytes(gq.make_params(d["q"], k, d["seq_lens"], table)),
                     dtype=torch.uint8, device=d["q"].device)
    return gq.gqa_decode(d["q"], k, v, d["seq_lens"], table, scale=scale, workspace=ws)


@pytest.mark.parametrize("paged", [False, True])
def test_fixed_workspace_matches_gqa_decode_twice_in_a_row(cuda_device, paged):
    base = WORKLOADS["paged_long"] if paged else WORKLOADS["llama2_70b_ragged"]
    cases = [
        dataclasses.replace(base, B=4, seq_len=2048, seed=101),
        dataclasses.replace(base, B=3, seq_len=1024, seed=202),
    ]
    for w in cases:  # two calls in a row, different inputs and split layouts
        inp = make_inputs(w)
        if not paged:
            inp["seq_lens"] = torch.tensor([w.seq_len, 1, 700, 65][: w.B], dtype=torch.int32)
        d = to_device(inp, cuda_device)
        out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device=cuda_device)
        assert call_static(d, paged, out, w.softmax_scale) == 0
        ref = call_reference(d, paged, w.softmax_scale)
        torch.cuda.synchronize(cuda_device)
        err, rel = errors(out.cpu().double().numpy(), ref.cpu().double().numpy())
        assert err <= ATOL and rel <= RTOL, (w, err, rel)


def test_fixed_workspace_refuses_problems_that_do_not_fit(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], name="wide", B=2, H_Q=1024, H_KV=1, seq_len=64)
    d = to_device(make_inputs(w), cuda_device)
    out = torch.full(d["q"].shape, 7.0, dtype=torch.float32, device=cuda_device)
    assert call_static(d, False, out, 1.0 / math.sqrt(w.D)) == GQA_ERR_WORKSPACE
    torch.cuda.synchronize(cuda_device)
    assert torch.all(out == 7.0)  # nothing was launched

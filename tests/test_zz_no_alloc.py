"""gqa_decode_static_workspace: decode with the library's own fixed workspace.

Some callers cannot call cudaMalloc -- for example a plugin whose host
application has already handed all device memory to its own pool, or a
latency-critical loop that must not take cudaMalloc's implicit device-wide
synchronisation.  For them the library offers one entry point that allocates
nothing and uses an 8 MiB array built into the library as its workspace, plus
gqa_static_workspace_status to read and clear that array's device status
flags (clamped lengths, out-of-range pages, a pipeline wait that gave up).

These tests call both through the C ABI (ctypes, no workspace argument).
Results are compared with the fp64 oracle and with gqa_decode run on a
caller-allocated workspace, within the same tolerance the parity tests use, on
two calls in a row with different inputs; the status flags are raised by bad
device data and cleared again.  The file is named so that pytest collects it
last.
"""

import ctypes
import dataclasses
import math

import pytest
import torch

import gqa_mqa_kv_b200 as gq
import oracle
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import ATOL, RTOL, assert_parity, errors, to_device

pytestmark = pytest.mark.gpu

GQA_ERR_WORKSPACE = 4


def call_static(d, paged, out, scale, seq_lens=None, table=None):
    k = d["k_paged"] if paged else d["k"]
    v = d["v_paged"] if paged else d["v"]
    if paged and table is None:
        table = d["block_table"]
    lens = d["seq_lens"] if seq_lens is None else seq_lens
    params = gq.make_params(d["q"], k, lens, table, out.dtype)
    lib = gq.library()
    st = lib.gqa_decode_static_workspace(
        ctypes.byref(params), ctypes.c_void_p(d["q"].data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(lens.data_ptr()),
        ctypes.c_void_p(table.data_ptr() if table is not None else None), ctypes.c_float(scale),
        ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream(out.device).cuda_stream))
    return st


def static_flags(device, clear=False):
    """The built-in workspace's status word, read through the C ABI."""
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(device):
        st = gq.library().gqa_static_workspace_status(
            ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream), ctypes.byref(flags), int(clear))
    assert st == 0
    return int(flags.value)


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
    static_flags(cuda_device, clear=True)  # whatever an earlier test left behind
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
        # and directly against the fp64 oracle on the logical contiguous cache
        exact = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale)
        assert_parity(out.cpu(), exact, f"fixed workspace {w.name} seed {w.seed}")
        assert static_flags(cuda_device) == 0


def test_fixed_workspace_reports_and_clears_clamped_lengths(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], B=2, seq_len=256, seed=303)
    inp = make_inputs(w)
    d = to_device(inp, cuda_device)
    static_flags(cuda_device, clear=True)
    bad = torch.tensor([300, -4], dtype=torch.int32, device=cuda_device)  # beyond capacity, negative
    out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device=cuda_device)
    assert call_static(d, False, out, w.softmax_scale, seq_lens=bad) == 0
    flags = static_flags(cuda_device, clear=True)
    assert flags & gq.FLAG_SEQ_LEN_CLAMPED
    assert not flags & gq.FLAG_TIMEOUT
    assert static_flags(cuda_device) == 0  # the clear took effect
    ref = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], torch.tensor([256, 0], dtype=torch.int32), w.softmax_scale)
    assert_parity(out.cpu(), ref, "fixed workspace, clamped lengths")
    # a good call afterwards leaves the word at zero
    out2 = torch.empty_like(out)
    assert call_static(d, False, out2, w.softmax_scale) == 0
    assert static_flags(cuda_device) == 0
    assert_parity(out2.cpu(), oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale),
                  "fixed workspace after the clear")


def test_fixed_workspace_reports_out_of_range_pages(cuda_device):
    w = dataclasses.replace(WORKLOADS["paged_long"], B=2, seq_len=256, seed=404)
    inp = make_inputs(w)
    d = to_device(inp, cuda_device)
    table = d["block_table"].clone()
    table[0, 1] = w.num_blocks + 7  # beyond the cache: read as zeros, flagged
    static_flags(cuda_device, clear=True)
    out = torch.full(d["q"].shape, float("nan"), dtype=torch.float32, device=cuda_device)
    assert call_static(d, True, out, w.softmax_scale, table=table) == 0
    assert static_flags(cuda_device, clear=True) & gq.FLAG_BAD_BLOCK
    assert static_flags(cuda_device) == 0
    k, v = inp["k"].clone(), inp["v"].clone()
    k[0, 64:128] = 0
    v[0, 64:128] = 0
    assert_parity(out.cpu(), oracle.gqa_decode(inp["q"], k, v, inp["seq_lens"], w.softmax_scale),
                  "fixed workspace, bad page")


def test_fixed_workspace_refuses_problems_that_do_not_fit(cuda_device):
    # 1024 query heads per KV head, and enough tiles (2 x 1024) to use every CTA of the
    # grid: the partial slots alone (two per CTA, 1024 x 128 floats each) far exceed 8 MiB
    w = dataclasses.replace(WORKLOADS["llama3_8b"], name="wide", B=2, H_Q=1024, H_KV=1, seq_len=65536)
    d = to_device(make_inputs(w), cuda_device)
    out = torch.full(d["q"].shape, 7.0, dtype=torch.float32, device=cuda_device)
    assert call_static(d, False, out, 1.0 / math.sqrt(w.D)) == GQA_ERR_WORKSPACE
    torch.cuda.synchronize(cuda_device)
    assert torch.all(out == 7.0)  # nothing was launched

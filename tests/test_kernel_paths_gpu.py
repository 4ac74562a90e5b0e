"""Both tensor-core split kernels against the oracle, selected explicitly.

gqa_kernel picks the mma.sync kernel or the tcgen05 kernel for one call.  The
automatic choice sends bf16 caches to mma.sync and 8-bit caches to tcgen05; the
cases here run the other pairings too, so every path a caller can select is
parity-tested: tiles and 128-token steps with ragged tails, one-tile steps,
paged caches, bf16 output, and every group width the tcgen05 kernel serves.
"""

import dataclasses

import numpy as np
import pytest
import torch

import gqa_mqa_kv_b200 as gq
import oracle
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import assert_parity
from tests.test_fp8kv_gpu import ref_fp8, run_fp8
from tests.test_parity_gpu import oracle_full, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("h_q,h_kv", [(32, 8), (64, 8), (32, 2), (48, 2), (32, 1), (12, 3)])
def test_tcgen05_bf16_group_widths(cuda_device, h_q, h_kv):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], name="tc", B=3, H_Q=h_q, H_KV=h_kv, seq_len=1111,
                            ragged=True)
    inp = make_inputs(w, pad_value=float("nan"))
    assert_parity(run_gpu(inp, w, cuda_device, kernel="tcgen05"), oracle_full(inp, w), f"tc {h_q}/{h_kv}")


def test_tcgen05_bf16_edge_lengths(cuda_device):
    # 0, 1, tile and step boundaries (63/64/65, 127/128/129, 191/192/193) and an odd tile count
    w = dataclasses.replace(WORKLOADS["sweep_hkv1"], B=12, seq_len=3000)
    lens = torch.tensor([0, 1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 3000], dtype=torch.int32)
    inp = make_inputs(w, pad_value=float("nan"), seq_lens=lens)
    out = run_gpu(inp, w, cuda_device, kernel="tcgen05")
    assert torch.all(out[0] == 0)
    assert_parity(out, oracle_full(inp, w), "tc edges")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_tcgen05_bf16_paged_equals_contiguous(cuda_device, out_dtype):
    w = dataclasses.replace(WORKLOADS["paged_long"], B=3, H_Q=32, H_KV=2, seq_len=2000)
    inp = make_inputs(w, pad_value=float("nan"))
    paged = run_gpu(inp, w, cuda_device, paged=True, out_dtype=out_dtype, kernel="tcgen05")
    contig = run_gpu(inp, w, cuda_device, out_dtype=out_dtype, kernel="tcgen05")
    iv = torch.int32 if out_dtype == torch.float32 else torch.int16
    assert torch.equal(paged.view(iv), contig.view(iv))
    assert_parity(paged, oracle_full(inp, w), "tc paged")


def test_tcgen05_mqa_full_size_sampled(cuda_device):
    w = WORKLOADS["sweep_hkv1"]
    inp = make_inputs(w)
    out = run_gpu(inp, w, cuda_device, kernel="tcgen05")
    rng = np.random.default_rng(1)
    pairs = [(b, int(h)) for b in range(w.B) for h in {0, w.H_Q - 1, int(rng.integers(0, w.H_Q))}]
    got = torch.stack([out[b, h] for b, h in pairs])
    ref = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale, pairs=pairs)
    assert_parity(got, ref, "tc MQA full size")


def test_both_kernels_agree_closely(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=4, H_Q=32, H_KV=2, seq_len=5000)
    inp = make_inputs(w)
    a = run_gpu(inp, w, cuda_device, kernel="mma_sync")
    b = run_gpu(inp, w, cuda_device, kernel="tcgen05")
    assert (a - b).abs().max().item() < 1e-3


@pytest.mark.parametrize("h_q,h_kv", [(64, 8), (16, 4)])
def test_fp8_on_the_mma_sync_kernel(cuda_device, h_q, h_kv):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], name="mma8", B=4, H_Q=h_q, H_KV=h_kv,
                            seq_len=1500)
    inp = make_inputs(w, pad_value=float("nan"))
    assert_parity(run_fp8(inp, w, cuda_device, kernel="mma_sync"), ref_fp8(inp, w), f"fp8 mma {h_q}/{h_kv}")


def test_unsupported_kernel_choices_are_refused(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], B=1, H_Q=8, H_KV=1, D=64, seq_len=64)
    inp = make_inputs(w)
    q = inp["q"].to(cuda_device)
    k = inp["k"].to(cuda_device)
    lens = inp["seq_lens"].to(cuda_device)
    with pytest.raises(gq.GqaError):
        gq.gqa_decode(q, k, k, lens, kernel="tcgen05")  # head_dim 64
    w = dataclasses.replace(WORKLOADS["llama3_8b"], B=1, H_Q=64, H_KV=1, seq_len=64)
    inp = make_inputs(w)
    with pytest.raises(gq.GqaError):
        gq.gqa_decode(inp["q"].to(cuda_device), inp["k"].to(cuda_device), inp["v"].to(cuda_device),
                      inp["seq_lens"].to(cuda_device), kernel="tcgen05")  # R = 64

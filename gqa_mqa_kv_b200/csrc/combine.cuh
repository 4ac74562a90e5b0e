// combine.cuh -- log-sum-exp merge of split-KV partials.
//
// A unit (sequence b, KV head kv) that the tile schedule cut across CTAs
// c_a..c_b has one partial per CTA: o_j (already divided by its own softmax
// denominator) and lse_j = m_j + log2 l_j in base-2 score units.  The merged
// result is out = sum_j 2^(lse_j - M) o_j / sum_j 2^(lse_j - M) with
// M = max_j lse_j, the split form of the softmax in "Grouped-Query Attention
// (GQA) and Multi-Query Attention (MQA): Mathematical Foundations, ...",
// section 2 (Head_i).  Units whose tiles stayed in one CTA were finished by
// the split kernel; sequences with L_b = 0 get out = 0 here.
//
// One CTA per sequence b; partial slots follow schedule.cuh.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(256) combine_kernel(const KernelArgs a, int grid) {
    __shared__ int64_t red_total[8], red_before[8];
    grid_dependency_wait();
    grid_launch_dependents();

    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t total = 0, before = 0;
    for (int i = threadIdx.x; i < a.B; i += blockDim.x) {
        const int64_t c = static_cast<int64_t>(a.H_KV) * tiles_of(seq_len_at(a, i));
        total += c;
        if (i < b) before += c;
    }
    total = warp_sum_i64(total);
    before = warp_sum_i64(before);
    if (lane == 0) {
        red_total[warp] = total;
        red_before[warp] = before;
    }
    __syncthreads();
    total = before = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
        total += red_total[i];
        before += red_before[i];
    }

    const int n_b = tiles_of(seq_len_at(a, b));
    if (n_b == 0) {
        for (int idx = threadIdx.x; idx < a.H_Q * D; idx += blockDim.x) {
            const int64_t oi = static_cast<int64_t>(b) * a.H_Q * D + idx;
            if constexpr (OUT_BF16)
                static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(0.f);
            else
                static_cast<float*>(a.out)[oi] = 0.f;
        }
        return;
    }
    const int g = effective_grid(total, grid);
    const float NEG_INF = -__int_as_float(0x7f800000);
    for (int kv = 0; kv < a.H_KV; ++kv) {
        const int64_t s_u = before + static_cast<int64_t>(kv) * n_b;
        const int64_t e_u = s_u + n_b;
        const int64_t ca = owner_of_tile(s_u, total, g);
        const int64_t cb = owner_of_tile(e_u - 1, total, g);
        if (ca == cb) continue;  // finished by the split kernel
        const int n_parts = static_cast<int>(cb - ca + 1);
        const int64_t slot0 = cta_first_tile(ca, total, g) < s_u ? 2 * ca + 1 : 2 * ca;
        for (int idx = threadIdx.x; idx < a.R * D; idx += blockDim.x) {
            const int r = idx / D, d = idx % D;
            float M = NEG_INF;
            for (int j = 0; j < n_parts; ++j) {
                const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
                M = fmaxf(M, a.ws_lse[slot * a.R + r]);
            }
            float wsum = 0.f, acc = 0.f;
            for (int j = 0; j < n_parts; ++j) {
                const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
                const float e = exp2f(a.ws_lse[slot * a.R + r] - M);
                wsum += e;
                acc += e * a.ws_o[(slot * a.R + r) * D + d];
            }
            const int64_t oi = (static_cast<int64_t>(b) * a.H_Q + kv * a.R + r) * D + d;
            if constexpr (OUT_BF16)
                static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(acc / wsum);
            else
                static_cast<float*>(a.out)[oi] = acc / wsum;
        }
    }
}

}  // namespace gqa

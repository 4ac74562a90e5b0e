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
// Each CTA owns up to kCombineSpan (head, d) outputs of one unit, every
// thread kCombineEPT of them; the partials' log-sum-exps are staged in shared
// memory kCombineChunk at a time and folded in with a running maximum, so any
// number of partials works and every partial load of a chunk is independent
// of the others.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

constexpr int kCombineThreads = 256;
constexpr int kCombineEPT = 4;                                    // outputs per thread
constexpr int kCombineSpan = kCombineThreads * kCombineEPT;      // outputs per CTA
constexpr int kCombineChunk = 8;                                  // partials staged per pass

template <bool OUT_BF16>
__device__ __forceinline__ void store_out(void* out, int64_t i, float x) {
    if constexpr (OUT_BF16)
        static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(x);
    else
        static_cast<float*>(out)[i] = x;
}

// Grid: (B * H_KV) units x ceil(R * D / kCombineSpan) parts; part z of a unit
// owns its outputs [z * kCombineSpan, (z + 1) * kCombineSpan) in (head, d) order.
template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const KernelArgs a, int grid) {
    constexpr int HPC = kCombineSpan / D;  // heads per part
    __shared__ float s_lse[kCombineChunk][HPC];
    __shared__ int64_t red_total[kCombineThreads / 32], red_before[kCombineThreads / 32];

    grid_launch_dependents();
    const int parts = (a.R * D + kCombineSpan - 1) / kCombineSpan;
    const int unit = blockIdx.x / parts;
    const int part = blockIdx.x % parts;
    const int b = unit / a.H_KV;
    const int kv = unit % a.H_KV;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int R = a.R;
    const int r0 = part * HPC;                       // first head of this part
    const int nr = min(HPC, R - r0);                 // heads in this part

    // seq_lens were final before the split kernel read them, so the tile
    // arithmetic may run while the split grid is still finishing.
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
#pragma unroll
    for (int i = 0; i < kCombineThreads / 32; ++i) {
        total += red_total[i];
        before += red_before[i];
    }
    const int n_b = tiles_of(seq_len_at(a, b));
    const int64_t out_base = (static_cast<int64_t>(b) * a.H_Q + static_cast<int64_t>(kv) * R + r0) * D;

    if (n_b == 0) {
        grid_dependency_wait();
        for (int idx = threadIdx.x; idx < nr * D; idx += blockDim.x) store_out<OUT_BF16>(a.out, out_base + idx, 0.f);
        return;
    }
    const int g = effective_grid(total, grid);
    const int64_t s_u = before + static_cast<int64_t>(kv) * n_b;
    const int64_t ca = owner_of_tile(s_u, total, g);
    const int64_t cb = owner_of_tile(s_u + n_b - 1, total, g);
    if (ca == cb) return;  // finished by the split kernel
    const int n_parts = static_cast<int>(cb - ca + 1);
    const int64_t slot0 = cta_first_tile(ca, total, g) < s_u ? 2 * ca + 1 : 2 * ca;

    grid_dependency_wait();  // partials of the split grid are complete and visible from here

    const float NEG_INF = -__int_as_float(0x7f800000);
    float m[kCombineEPT], sum[kCombineEPT], acc[kCombineEPT];
#pragma unroll
    for (int e = 0; e < kCombineEPT; ++e) {
        m[e] = NEG_INF;
        sum[e] = 0.f;
        acc[e] = 0.f;
    }
    for (int j0 = 0; j0 < n_parts; j0 += kCombineChunk) {
        const int nj = min(kCombineChunk, n_parts - j0);
        __syncthreads();  // previous chunk's s_lse fully consumed
        for (int i = threadIdx.x; i < nj * nr; i += blockDim.x) {
            const int jj = i / nr, rr = i % nr;
            const int j = j0 + jj;
            const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
            s_lse[jj][rr] = a.ws_lse[slot * R + r0 + rr];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < kCombineEPT; ++e) {
            const int idx = e * kCombineThreads + threadIdx.x;
            if (idx >= nr * D) break;
            const int rr = idx / D, d = idx % D;
            float ov[kCombineChunk];
#pragma unroll
            for (int jj = 0; jj < kCombineChunk; ++jj) {
                const int j = j0 + jj;
                const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
                ov[jj] = jj < nj ? a.ws_o[(slot * R + r0 + rr) * D + d] : 0.f;
            }
            float mx = m[e];
#pragma unroll
            for (int jj = 0; jj < kCombineChunk; ++jj)
                if (jj < nj) mx = fmaxf(mx, s_lse[jj][rr]);
            const float rescale = fast_exp2(m[e] - mx);  // m = -inf on the first chunk -> 0
            sum[e] *= rescale;
            acc[e] *= rescale;
#pragma unroll
            for (int jj = 0; jj < kCombineChunk; ++jj) {
                if (jj < nj) {
                    const float wj = fast_exp2(s_lse[jj][rr] - mx);
                    sum[e] += wj;
                    acc[e] = fmaf(wj, ov[jj], acc[e]);
                }
            }
            m[e] = mx;
        }
    }
#pragma unroll
    for (int e = 0; e < kCombineEPT; ++e) {
        const int idx = e * kCombineThreads + threadIdx.x;
        if (idx < nr * D) store_out<OUT_BF16>(a.out, out_base + idx, acc[e] / sum[e]);
    }
}

}  // namespace gqa

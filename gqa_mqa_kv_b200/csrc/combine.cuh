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
// One CTA per unit.  Each thread owns (head, d) output elements; the partials'
// log-sum-exps are staged in shared memory kCombineChunk at a time and folded
// in with a running maximum, so any number of partials works and every
// partial load of a chunk is independent of the others.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

constexpr int kCombineThreads = 256;
constexpr int kCombineChunk = 8;  // partials staged per pass
constexpr int kMaxR = 1024;       // widest group the combine supports (shared memory bound)

template <int D, bool OUT_BF16>
__device__ __forceinline__ void store_out(void* out, int64_t i, float x) {
    if constexpr (OUT_BF16)
        static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(x);
    else
        static_cast<float*>(out)[i] = x;
}

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const KernelArgs a, int grid) {
    extern __shared__ float s_lse[];  // [kCombineChunk][R]
    __shared__ int64_t red_total[kCombineThreads / 32], red_before[kCombineThreads / 32];

    grid_launch_dependents();
    const int b = blockIdx.x / a.H_KV;
    const int kv = blockIdx.x % a.H_KV;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int R = a.R;

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
    const int64_t out_base = (static_cast<int64_t>(b) * a.H_Q + static_cast<int64_t>(kv) * R) * D;

    if (n_b == 0) {
        grid_dependency_wait();  // out may still be in use by the previous call's kernels
        for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) store_out<D, OUT_BF16>(a.out, out_base + idx, 0.f);
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

    constexpr int EPT = 4;  // output elements per thread per pass
    const float NEG_INF = -__int_as_float(0x7f800000);
    for (int base = 0; base < R * D; base += EPT * kCombineThreads) {
        float m[EPT], sum[EPT], acc[EPT];
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            m[e] = NEG_INF;
            sum[e] = 0.f;
            acc[e] = 0.f;
        }
        for (int j0 = 0; j0 < n_parts; j0 += kCombineChunk) {
            const int nj = min(kCombineChunk, n_parts - j0);
            __syncthreads();  // previous chunk's s_lse fully consumed
            for (int i = threadIdx.x; i < nj * R; i += blockDim.x) {
                const int jj = i / R, r = i % R;
                const int j = j0 + jj;
                const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
                s_lse[jj * R + r] = a.ws_lse[slot * R + r];
            }
            __syncthreads();
#pragma unroll
            for (int e = 0; e < EPT; ++e) {
                const int idx = base + e * kCombineThreads + threadIdx.x;
                if (idx >= R * D) break;
                const int r = idx / D, d = idx % D;
                float ov[kCombineChunk];
#pragma unroll
                for (int jj = 0; jj < kCombineChunk; ++jj) {
                    const int j = j0 + jj;
                    const int64_t slot = j == 0 ? slot0 : 2 * (ca + j);
                    ov[jj] = jj < nj ? a.ws_o[(slot * R + r) * D + d] : 0.f;
                }
                float mx = m[e];
#pragma unroll
                for (int jj = 0; jj < kCombineChunk; ++jj)
                    if (jj < nj) mx = fmaxf(mx, s_lse[jj * R + r]);
                const float rescale = exp2f(m[e] - mx);  // m = -inf on the first chunk -> 0
                sum[e] *= rescale;
                acc[e] *= rescale;
#pragma unroll
                for (int jj = 0; jj < kCombineChunk; ++jj) {
                    if (jj < nj) {
                        const float wj = exp2f(s_lse[jj * R + r] - mx);
                        sum[e] += wj;
                        acc[e] = fmaf(wj, ov[jj], acc[e]);
                    }
                }
                m[e] = mx;
            }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int idx = base + e * kCombineThreads + threadIdx.x;
            if (idx < R * D) store_out<D, OUT_BF16>(a.out, out_base + idx, acc[e] / sum[e]);
        }
    }
}

}  // namespace gqa

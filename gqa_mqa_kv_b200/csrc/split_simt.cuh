// split_simt.cuh -- CUDA-core split-KV decode kernel (fp32 or bf16 inputs).
//
// The path for fp32 caches and for groups wider than 64 query heads, where
// the tensor-core kernel does not apply.  Same tile schedule and outputs as
// split_mma.cuh: every segment writes the final output or a partial
// (o / l, m + log2 l).  Four warps take interleaved tokens; each lane holds
// D/32 elements of every row; query heads are handled 8 at a time.  fp32
// arithmetic throughout ("Grouped-Query Attention (GQA) and Multi-Query
// Attention (MQA): Mathematical Foundations, ...", section 2, Head_i).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "combine.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_fp8_e4m3>(__nv_fp8_e4m3 x) { return static_cast<float>(x); }

constexpr int kSimtWarps = 4;
constexpr int kSimtHeads = 8;

// Token tok's key and value rows of KV head w.kv (this lane's D/32 elements);
// an out-of-range page reads as zeros and raises the flag.
template <typename TKV, int D, bool PAGED>
__device__ __forceinline__ void simt_load_row(const KernelArgs& a, const TKV* __restrict__ k,
                                              const TKV* __restrict__ v, const Walk& w, int tok,
                                              float (&kr)[D / 32], float (&vr)[D / 32]) {
    const int lane = threadIdx.x & 31;
    int64_t row;
    bool live = true;
    if constexpr (PAGED) {
        const int page = __ldg(a.block_table + static_cast<int64_t>(w.b) * a.max_blocks + tok / kTile);
        live = page >= 0 && page < a.num_blocks;
        if (!live && lane == 0) atomicOr(a.status, kFlagBadBlock);
        row = (static_cast<int64_t>(live ? page : 0) * kTile + tok % kTile) * a.H_KV + w.kv;
    } else {
        row = (static_cast<int64_t>(w.b) * a.S_max + tok) * a.H_KV + w.kv;
    }
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
        kr[i] = live ? to_f32(k[row * D + lane + 32 * i]) : 0.f;
        vr[i] = live ? to_f32(v[row * D + lane + 32 * i]) : 0.f;
    }
}

// TQ: element type of q; TKV: element type of the cache (fp32, bf16 or E4M3
// bytes, the latter multiplied by per-KV-head k_scale / v_scale).
template <typename TQ, typename TKV, int D, bool PAGED, bool OUT_BF16>
__global__ void __launch_bounds__(32 * kSimtWarps)
    split_simt_kernel(const TQ* __restrict__ q, const TKV* __restrict__ k, const TKV* __restrict__ v,
                      const KernelArgs a) {
    constexpr int DPL = D / 32;
    constexpr int HC = kSimtHeads;
    __shared__ Plan plan;
    __shared__ float sm_m[kSimtWarps][HC];
    __shared__ float sm_l[kSimtWarps][HC];
    __shared__ float sm_o[kSimtWarps][HC][D];
    __shared__ int merge_last;
    __shared__ uint32_t s_epoch;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const float NEG_INF = -__int_as_float(0x7f800000);

    grid_dependency_wait();
    grid_launch_dependents();
    if (warp == 0) make_plan(a, &plan);
    if (threadIdx.x == 32) s_epoch = merge_epoch_take(a);
    __syncthreads();
    uint32_t* const bank = merge_bank(a, s_epoch, 0, blockDim.x);
    zero_empty_sequences<D, OUT_BF16>(a, 0, blockDim.x);
    const int64_t lo = plan.lo, hi = plan.hi;
    if (lo >= hi) return;
    Walk w{plan.b, plan.kv, plan.tile, plan.n_b, plan.L};

    bool first = true;
    int64_t gi = lo;
    while (gi < hi) {
        const int seg_tiles = static_cast<int>(min(static_cast<int64_t>(w.n_b - w.tile), hi - gi));
        const int64_t s_u = gi - w.tile;  // global index of the unit's first tile
        const bool whole = (w.tile == 0) && (seg_tiles == w.n_b);
        const int64_t slot = first ? 2 * static_cast<int64_t>(blockIdx.x) : 2 * static_cast<int64_t>(blockIdx.x) + 1;
        const int t_begin = w.tile * kTile;
        const int t_end = min((w.tile + seg_tiles) * kTile, w.L);
        const float sl2 = a.sl2 * (a.k_scale ? __ldg(a.k_scale + w.kv) : 1.f);
        const float vsc = a.v_scale ? __ldg(a.v_scale + w.kv) : 1.f;

        for (int hc = 0; hc < a.R; hc += HC) {
            const int nh = min(HC, a.R - hc);
            float qr[HC][DPL], o[HC][DPL], m[HC], l[HC];
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                const int64_t qrow = static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R + hc + j;
#pragma unroll
                for (int i = 0; i < DPL; ++i) {
                    qr[j][i] = j < nh ? to_f32(q[qrow * D + lane + 32 * i]) : 0.f;
                    o[j][i] = 0.f;
                }
                m[j] = NEG_INF;
                l[j] = 0.f;
            }
            // The next token's rows are loaded before this token's arithmetic, so a
            // warp waits on memory once per token pair of loads instead of per token.
            float kr[DPL], vr[DPL];
            if (t_begin + warp < t_end) simt_load_row<TKV, D, PAGED>(a, k, v, w, t_begin + warp, kr, vr);
            for (int tok = t_begin + warp; tok < t_end; tok += kSimtWarps) {
                float kn[DPL], vn[DPL];
                const bool more = tok + kSimtWarps < t_end;
                if (more) simt_load_row<TKV, D, PAGED>(a, k, v, w, tok + kSimtWarps, kn, vn);
#pragma unroll
                for (int j = 0; j < HC; ++j) {
                    float s = 0.f;
#pragma unroll
                    for (int i = 0; i < DPL; ++i) s = fmaf(qr[j][i], kr[i], s);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                    s *= sl2;
                    const float mn = fmaxf(m[j], s);
                    const float al = fast_exp2(m[j] - mn);
                    const float p = fast_exp2(s - mn);
                    l[j] = l[j] * al + p;
#pragma unroll
                    for (int i = 0; i < DPL; ++i) o[j][i] = fmaf(p, vr[i], o[j][i] * al);
                    m[j] = mn;
                }
                if (more) {
#pragma unroll
                    for (int i = 0; i < DPL; ++i) {
                        kr[i] = kn[i];
                        vr[i] = vn[i];
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < HC; ++j) {
                if (lane == 0) {
                    sm_m[warp][j] = m[j];
                    sm_l[warp][j] = l[j];
                }
#pragma unroll
                for (int i = 0; i < DPL; ++i) sm_o[warp][j][lane + 32 * i] = o[j][i];
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < nh * D; idx += blockDim.x) {
                const int j = idx / D, d = idx % D;
                float M = NEG_INF;
#pragma unroll
                for (int ww = 0; ww < kSimtWarps; ++ww) M = fmaxf(M, sm_m[ww][j]);
                const float ref = M == NEG_INF ? 0.f : M;
                float L = 0.f, O = 0.f;
#pragma unroll
                for (int ww = 0; ww < kSimtWarps; ++ww) {
                    const float e = fast_exp2(sm_m[ww][j] - ref);
                    L += sm_l[ww][j] * e;
                    O += sm_o[ww][j][d] * e;
                }
                const int r = hc + j;
                O *= vsc;
                if (whole) {
                    const int64_t oi = (static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R + r) * D + d;
                    if constexpr (OUT_BF16)
                        static_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(O / L);
                    else
                        static_cast<float*>(a.out)[oi] = O / L;
                } else {
                    a.ws_o[(slot * a.R + r) * D + d] = O / L;
                    if (d == 0) a.ws_lse[slot * a.R + r] = M + log2f(L);
                }
            }
            __syncthreads();
        }
        if (!whole) {
            // The CTA's partial of this unit is complete: the last of the unit's
            // partials merges them all.
            const SplitUnit su = split_unit_of(s_u, w.n_b, plan.n_tiles, plan.g);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) merge_last = atomicAdd(bank + su.ca, 1u) == static_cast<uint32_t>(su.n_parts - 1);
            __syncthreads();
            if (merge_last && warp == 0) {
                __threadfence();
                merge_unit<D, OUT_BF16>(merge_io(a), su, (static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R) * D, 0, 1);
            }
        }
        first = false;
        gi += seg_tiles;
        w.tile += seg_tiles - 1;
        if (gi < hi) w.advance(a);
    }
}

}  // namespace gqa

// rope_append.cuh -- the step before decode: rotary position embedding of the
// new token's query and key heads, and the append of its key/value rows to
// the cache.
//
// "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA): Mathematical
// Foundations, ...", section 4, "Rotary Position Embeddings (RoPE)
// Interaction": R_{Theta,m} = diag(R_{theta_1,m}, ..., R_{theta_{d/2},m}) is
// applied to each of the H_Q query heads and once to each of the H_KV key
// heads at the token's position m.  theta_i = base^(-2i/d), i = 0..d/2-1
// (the RoFormer frequencies the page cites).  Pairs are adjacent coordinates
// (2i, 2i+1) -- the block-diagonal form as written -- or, on request, the
// half-split pairs (i, i + d/2).
//
// One warp per head row: rows [0, B*H_Q) are query heads, rows
// [B*H_Q, B*(H_Q+H_KV)) are key heads (whose warp also copies the value row).
// The angle m * theta_i and the rotation are evaluated in double, so a
// position of 10^5 loses nothing to fp32 angle rounding; each result is
// rounded once to the storage type.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

struct RopeArgs {
    int B, H_Q, H_KV, D;
    int max_len;                 // positions must lie in [0, max_len)
    int S_max;                   // contiguous cache capacity; 0 when paged
    int max_blocks, num_blocks;  // paged cache
    const int32_t* positions;    // [B]
    const int32_t* block_table;  // [B, max_blocks] or null
    int32_t* seq_lens_out;       // [B] or null: receives position + 1
    uint32_t* status;            // or null
    double log2_base;
    int halves;                  // 0: adjacent pairs, 1: (i, i + D/2)
};

template <typename T>
__device__ __forceinline__ double load_d(const T* p);
template <>
__device__ __forceinline__ double load_d<float>(const float* p) { return static_cast<double>(*p); }
template <>
__device__ __forceinline__ double load_d<__nv_bfloat16>(const __nv_bfloat16* p) {
    return static_cast<double>(__bfloat162float(*p));
}

template <typename T>
__device__ __forceinline__ void store_d(T* p, double x);
template <>
__device__ __forceinline__ void store_d<float>(float* p, double x) { *p = __double2float_rn(x); }
template <>
__device__ __forceinline__ void store_d<__nv_bfloat16>(__nv_bfloat16* p, double x) {
    *p = __double2bfloat16(x);
}

template <typename T>
__global__ void __launch_bounds__(128)
    rope_append_kernel(const T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
                       T* q_out, T* k_cache, T* v_cache, const RopeArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t q_rows = static_cast<int64_t>(a.B) * a.H_Q;
    if (row >= q_rows + static_cast<int64_t>(a.B) * a.H_KV) return;
    const bool is_q = row < q_rows;
    const int b = static_cast<int>(is_q ? row / a.H_Q : (row - q_rows) / a.H_KV);
    const int head = static_cast<int>(is_q ? row % a.H_Q : (row - q_rows) % a.H_KV);
    const int m = __ldg(a.positions + b);
    const int half = a.D / 2;

    // Destination of the key/value rows (null when the position or page is invalid).
    T* kdst = nullptr;
    T* vdst = nullptr;
    if (!is_q) {
        bool ok = m >= 0 && m < a.max_len;
        int64_t cache_row = 0;
        if (ok) {
            if (a.block_table != nullptr) {
                const int page = __ldg(a.block_table + static_cast<int64_t>(b) * a.max_blocks + m / kTile);
                ok = page >= 0 && page < a.num_blocks;
                if (!ok && lane == 0 && a.status) atomicOr(a.status, kFlagBadBlock);
                cache_row = (static_cast<int64_t>(page) * kTile + m % kTile) * a.H_KV + head;
            } else {
                cache_row = (static_cast<int64_t>(b) * a.S_max + m) * a.H_KV + head;
            }
        } else if (lane == 0 && a.status) {
            atomicOr(a.status, kFlagBadPosition);
        }
        if (ok) {
            kdst = k_cache + cache_row * a.D;
            vdst = v_cache + cache_row * a.D;
        }
        if (head == 0 && lane == 0 && a.seq_lens_out != nullptr && ok) a.seq_lens_out[b] = m + 1;
    }

    const T* src = is_q ? q + row * a.D : k_new + (static_cast<int64_t>(b) * a.H_KV + head) * a.D;
    T* dst = is_q ? q_out + row * a.D : kdst;
    for (int i = lane; i < half; i += 32) {
        const int i0 = a.halves ? i : 2 * i;
        const int i1 = a.halves ? i + half : 2 * i + 1;
        const double theta = exp2(-2.0 * i / a.D * a.log2_base);
        double sn, cs;
        sincos(static_cast<double>(m) * theta, &sn, &cs);
        const double x0 = load_d(src + i0), x1 = load_d(src + i1);
        if (dst != nullptr) {
            store_d(dst + i0, x0 * cs - x1 * sn);
            store_d(dst + i1, x0 * sn + x1 * cs);
        }
    }
    if (vdst != nullptr) {
        const T* vs = v_new + (static_cast<int64_t>(b) * a.H_KV + head) * a.D;
        for (int i = lane; i < a.D; i += 32) vdst[i] = vs[i];
    }
}

}  // namespace gqa

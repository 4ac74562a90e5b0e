// combine.cuh -- log-sum-exp merge of split-KV partials, done inside the
// split kernels by the last writer of a split unit.
//
// A unit (sequence b, KV head kv) that the tile schedule cut across CTAs
// ca..cb has one partial per CTA: o_j (already divided by its own softmax
// denominator) and lse_j = m_j + log2 l_j in base-2 score units.  The merged
// result is out = sum_j 2^(lse_j - M) o_j / sum_j 2^(lse_j - M) with
// M = max_j lse_j, the split form of the softmax in "Grouped-Query Attention
// (GQA) and Multi-Query Attention (MQA): Mathematical Foundations, ...",
// section 2 (Head_i).
//
// The warps that write a CTA's partial only arrive on a CTA-local mbarrier
// (release at CTA scope).  A dedicated merge warp of the CTA waits on it,
// publishes the partial at GPU scope (a fence, cumulative over the writes it
// has observed, then a ticket from the unit's counter) and, holding the last
// ticket, merges the unit.  The streaming warps therefore never wait on a
// GPU-scope fence or an atomic round trip.  The sums run over j = 0 ..
// n_parts-1 in that order from the stored values, so the result does not
// depend on which CTA merges.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

template <bool OUT_BF16>
__device__ __forceinline__ void store_out(void* out, int64_t i, float x) {
    if constexpr (OUT_BF16)
        static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(x);
    else
        static_cast<float*>(out)[i] = x;
}

// Warp-collective: publishes the partial this CTA's writers have finished
// (observed through a CTA-scope barrier) and takes a ticket from *cnt; true in
// every lane for the last of `expected` tickets (loads of the other partials
// are ordered after that observation).
__device__ __forceinline__ bool merge_ticket(uint32_t* cnt, int expected) {
    __threadfence();
    uint32_t old = 0;
    if ((threadIdx.x & 31) == 0) old = atomicAdd(cnt, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    const bool last = old == static_cast<uint32_t>(expected - 1);
    if (last) __threadfence();
    return last;
}

// Warp-collective merge of a split unit's R x D outputs (written at
// out[row0 + h D + d]) from its partials, which other SMs wrote during this
// grid and are therefore read at L2 (ld.global.cg).  Element e is head
// e / (D/4), dimensions 4 (e % (D/4)) .. +3.  A block of KG elements
// x JG partials issues all of its loads before using any, so it costs one L2
// round trip; partials are folded in with a running maximum, so any number
// of them works.
// Warp `part` of `parts` cooperating warps takes elements part * 32 + lane +
// 32 parts k.
// The arguments are plain values: a reference to the kernel's argument block
// would make the compiler keep that block in local memory, and every read of
// it in the streaming loops would become a local load.
struct MergeIO {
    const float* ws_o;
    const float* ws_lse;
    void* out;
    int R;
};

__device__ __forceinline__ MergeIO merge_io(const KernelArgs& a) { return MergeIO{a.ws_o, a.ws_lse, a.out, a.R}; }

template <int D, bool OUT_BF16>
__device__ __noinline__ void merge_unit(const MergeIO a, const SplitUnit u, const int64_t row0, const int part,
                                        const int parts) {
    constexpr int KG = 4, JG = 4, Q = D / 4;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const int lane = (threadIdx.x & 31) + 32 * part;
    const int stride = 32 * parts;
    const int E = a.R * Q;
    for (int e0 = 0; e0 < E; e0 += stride * KG) {
        float m[KG], l[KG];
        float4 acc[KG];
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
            m[kk] = NEG_INF;
            l[kk] = 0.f;
            acc[kk] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int j0 = 0; j0 < u.n_parts; j0 += JG) {
            float ls[KG][JG];
            float4 ov[KG][JG];
#pragma unroll
            for (int kk = 0; kk < KG; ++kk) {
                const int e = e0 + stride * kk + lane;
                const int h = e / Q, q4 = e - h * Q;
#pragma unroll
                for (int jj = 0; jj < JG; ++jj) {
                    ls[kk][jj] = NEG_INF;
                    ov[kk][jj] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (e < E && j0 + jj < u.n_parts) {
                        const int64_t sl = part_slot(u, j0 + jj);
                        ls[kk][jj] = __ldcg(a.ws_lse + sl * a.R + h);
                        ov[kk][jj] = __ldcg(reinterpret_cast<const float4*>(a.ws_o + (sl * a.R + h) * D) + q4);
                    }
                }
            }
#pragma unroll
            for (int kk = 0; kk < KG; ++kk) {
                float mx = m[kk];
#pragma unroll
                for (int jj = 0; jj < JG; ++jj) mx = fmaxf(mx, ls[kk][jj]);
                if (mx == NEG_INF) continue;  // an element past the unit's outputs
                const float sc = fast_exp2(m[kk] - mx);  // m = -inf on the first block -> 0
                l[kk] *= sc;
                acc[kk].x *= sc;
                acc[kk].y *= sc;
                acc[kk].z *= sc;
                acc[kk].w *= sc;
#pragma unroll
                for (int jj = 0; jj < JG; ++jj) {
                    const float wj = fast_exp2(ls[kk][jj] - mx);  // 2^-inf = 0 for missing partials
                    l[kk] += wj;
                    acc[kk].x = fmaf(wj, ov[kk][jj].x, acc[kk].x);
                    acc[kk].y = fmaf(wj, ov[kk][jj].y, acc[kk].y);
                    acc[kk].z = fmaf(wj, ov[kk][jj].z, acc[kk].z);
                    acc[kk].w = fmaf(wj, ov[kk][jj].w, acc[kk].w);
                }
                m[kk] = mx;
            }
        }
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
            const int e = e0 + stride * kk + lane;
            if (e >= E) continue;
            const int h = e / Q, q4 = e - h * Q;
            const float inv = 1.f / l[kk];
            const int64_t i = row0 + static_cast<int64_t>(h) * D + 4 * q4;
            // 8-byte stores: out is only required to be 8-byte aligned
            if constexpr (OUT_BF16) {
                const __nv_bfloat162 p0 = __floats2bfloat162_rn(acc[kk].x * inv, acc[kk].y * inv);
                const __nv_bfloat162 p1 = __floats2bfloat162_rn(acc[kk].z * inv, acc[kk].w * inv);
                *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + i) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
            } else {
                float2* dst = reinterpret_cast<float2*>(static_cast<float*>(a.out) + i);
                dst[0] = make_float2(acc[kk].x * inv, acc[kk].y * inv);
                dst[1] = make_float2(acc[kk].z * inv, acc[kk].w * inv);
            }
        }
    }
}

// A CTA's merge jobs: its first and its last segment, each when it is cut
// (holds a partial).  Job k is signalled on mjob[k] by the segment's writers.
struct MergeJobs {
    int n;
    int slot[2];      // which of mjob[0] (first segment) / mjob[1] (last) it waits on
    bool tail[2];     // the job is the CTA's last segment (its writers are then done streaming)
    SplitUnit su[2];
    int b[2], kv[2];
};

// Warp-collective: the jobs of this CTA's tile range [lo, hi) (lo < hi).
__device__ __forceinline__ MergeJobs merge_jobs_of(const KernelArgs& a, const Plan& p) {
    MergeJobs J;
    J.n = 0;
    // the unit holding tile lo
    const int64_t s0 = p.lo - p.tile;
    const bool first_cut = p.tile > 0 || s0 + p.n_b > p.hi;
    if (first_cut) {
        J.slot[J.n] = 0;
        J.tail[J.n] = s0 + p.n_b >= p.hi;
        J.su[J.n] = split_unit_of(s0, p.n_b, p.n_tiles, p.g);
        J.b[J.n] = p.b;
        J.kv[J.n] = p.kv;
        ++J.n;
    }
    if (s0 + p.n_b < p.hi) {
        // another unit holds tile hi - 1: the CTA's last segment
        int b = 0;
        int64_t start = 0;
        warp_find_batch(a, p.hi - 1, &b, &start);
        const int n_b = tiles_of(seq_len_at(a, b));
        const int kv = static_cast<int>((p.hi - 1 - start) / n_b);
        const int64_t su = start + static_cast<int64_t>(kv) * n_b;
        if (su + n_b > p.hi) {
            J.slot[J.n] = 1;
            J.tail[J.n] = true;
            J.su[J.n] = split_unit_of(su, n_b, p.n_tiles, p.g);
            J.b[J.n] = b;
            J.kv[J.n] = kv;
            ++J.n;
        }
    }
    return J;
}

// The merge warp of a split kernel (warp-collective).  Takes the call's merge
// epoch, clears its share of the next call's counters, writes the outputs of
// empty sequences, then serves the CTA's merge jobs in order.  A job of the
// CTA's last segment is merged together with that segment's `helpers` warps,
// which have finished streaming by then: the ticket's outcome goes to *last
// and they are released through *assist (they call merge_assist).  Returns
// false when a wait for the writers gave up (the caller raises the timeout
// flag; helpers time out on *assist in turn).
template <int D, bool OUT_BF16>
__device__ __forceinline__ bool merge_warp(const KernelArgs& a, const Plan& p, uint64_t* mjob, uint64_t* assist,
                                           volatile int* last, int helpers, const volatile int* abort) {
    const int lane = threadIdx.x & 31;
    uint32_t epoch = 0;
    if (lane == 0) epoch = merge_epoch_take(a);
    epoch = __shfl_sync(0xffffffffu, epoch, 0);
    uint32_t* bank = merge_bank(a, epoch, static_cast<int>(threadIdx.x) - lane, 32);
    zero_empty_sequences<D, OUT_BF16>(a, static_cast<int>(threadIdx.x) - lane, 32);
    if (p.lo >= p.hi) return true;
    const MergeJobs J = merge_jobs_of(a, p);
    // k unrolled: J's arrays stay in registers
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (k >= J.n) break;
        if (!mbar_wait_sleepy_warp(smem_addr(&mjob[J.slot[k]]), 0u, abort, 200)) return false;
        const bool mine = merge_ticket(bank + J.su[k].ca, J.su[k].n_parts);
        const int64_t row0 = (static_cast<int64_t>(J.b[k]) * a.H_Q + J.kv[k] * a.R) * D;
        if (J.tail[k]) {
            if (lane == 0) {
                *last = mine ? 1 : 0;
                mbar_arrive(smem_addr(assist));
            }
            if (mine) merge_unit<D, OUT_BF16>(merge_io(a), J.su[k], row0, helpers, helpers + 1);
        } else if (mine) {
            merge_unit<D, OUT_BF16>(merge_io(a), J.su[k], row0, 0, 1);
        }
    }
    return true;
}

// A writer warp of the CTA's last segment, when that segment was cut, after
// streaming: waits for the merge warp's ticket and, if it was the unit's last,
// merges share `part` of `parts` (the merge warp takes the last share).
template <int D, bool OUT_BF16>
__device__ __forceinline__ bool merge_assist(const KernelArgs& a, uint64_t* assist, const volatile int* last,
                                             int b, int kv, int64_t s_u, int n_b, int64_t n_tiles, int g, int part,
                                             int parts, const volatile int* abort) {
    if (!mbar_wait_sleepy_warp(smem_addr(assist), 0u, abort, 100)) return false;
    if (*last) {
        __threadfence();
        merge_unit<D, OUT_BF16>(merge_io(a), split_unit_of(s_u, n_b, n_tiles, g),
                                (static_cast<int64_t>(b) * a.H_Q + kv * a.R) * D, part, parts);
    }
    return true;
}

}  // namespace gqa

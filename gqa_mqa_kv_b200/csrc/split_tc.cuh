// split_tc.cuh -- split-KV decode on the 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory) for head_dim 128.
//
// What it computes is the split kernel's contract (schedule.cuh): for every
// segment, the R query heads of one (sequence, KV head) pair attend over the
// segment's tokens ("Grouped-Query Attention (GQA) and Multi-Query Attention
// (MQA): Mathematical Foundations, ...", section 2, Head_i = softmax(Q_i
// K_{g(i)}^T / sqrt(d_k)) V_{g(i)}), with an fp32 online softmax in base 2;
// a whole-unit segment writes the output, others write (normalised o,
// log2-sum-exp) partials for the combine kernel.
//
// A step covers two consecutive 64-token tiles of one segment (one, zero
// padded, when the segment's tile count is odd):
//   S^T = K Q^T     tcgen05.mma, M = 128 tokens, N = query columns, K = d:
//                   A = the K rows as TMA staged them (K-major, 128-byte
//                   swizzle), B = the query rows; S^T lands in tensor memory
//                   (two buffers, so the next step's product overlaps this
//                   step's softmax).
//   softmax         four warps, thread = token = TMEM lane: p = 2^(s - m)
//                   against a per-head reference m shared by all tokens,
//                   moved only when a score exceeds it by more than 8 (all
//                   threads agree through an mbarrier exchange).  P^T goes
//                   to shared memory as bf16 hi and lo parts -- N = 2 RP
//                   columns -- so the product keeps fp32-level weights.
//   O^T += V^T P^T  tcgen05.mma, M = 128 (d), N = 2 RP, K = 128 tokens:
//                   A = the V rows read MN-major, B = P^T; O^T accumulates in
//                   tensor memory over the segment; hi and lo columns are
//                   summed in the epilogue.
//
// 8-bit caches (KV8, OCP E4M3 with per-KV-head scales): the score product
// runs as kind::f8f6f4 directly on the staged E4M3 key bytes.  Each query
// head is scaled by a power of two 2^a (max |q| * 2^a in [128, 256)) and
// split into two E4M3 terms, q 2^a = t1 + t2 / 16 (exact for every element
// of magnitude >= 2^-6 after scaling; smaller ones err by <= 2^-14), held as
// query columns h and RP + h; s = (S[h] + S[RP + h] / 16) 2^-a.  The value
// product is kind::f8f6f4 as well, on the staged E4M3 value rows read
// MN-major, with each weight split into four E4M3 terms, p = t1 + t2 / 16 +
// t3 / 256 + t4 / 4096 (relative error <= 2^-16 for p >= 2^-6, absolute
// <= 2^-22 below), held as O^T columns [t1 | t2 | t3 | t4] and summed in
// the epilogue.
//
// Warp roles: 0 TMA producer, 1 score products (+ tensor-memory
// allocation), 2 value products, 3..6 softmax and epilogue (sub-partitions
// 3, 0, 1, 2).  Every wait is bounded
// (kWaitTimeoutNs); on a timeout the CTA raises GQA_FLAG_TIMEOUT, lets its
// copies and products drain, frees its tensor memory and returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "combine.cuh"
#include "ptx.cuh"
#include "schedule.cuh"
#include "tcgen05.cuh"

namespace gqa {

constexpr int kStepTiles = 2;                 // 64-token tiles per step
constexpr int kStepTokens = kStepTiles * kTile;

template <int RP, bool KV8>
struct TcCfg {
    static_assert(RP == 8 || RP == 16 || RP == 32, "query columns per KV head: 8, 16 or 32");
    static_assert(KV8 || RP >= 16, "an M = 128 score product needs N >= 16");
    static constexpr int D = 128;
    static constexpr int NS_COLS = KV8 ? 2 * RP : RP;  // S^T columns: heads, or two query terms per head
    // O^T columns: bf16 P hi | lo, or four E4M3 terms of P (KV8), each RP heads wide
    static constexpr int NPT = KV8 ? 4 : 2;            // P terms
    static constexpr int NO_COLS = NPT * RP;
    static constexpr int S_COL = 0;                    // S^T buffer b at S_COL + b * NS_COLS
    static constexpr int O_COL = 2 * NS_COLS;
    static constexpr int TMEM_COLS = 512;              // the whole tensor memory of the SM
    // Softmax warps: one per tensor-memory sub-partition, two (each taking half
    // the query columns) for 32 columns.
    static constexpr int HSPLIT = RP == 32 ? 2 : 1;
    static constexpr int HW = RP / HSPLIT;             // query columns per softmax warp
    static constexpr int NSM = 4 * HSPLIT;
    static constexpr int WARP_QK = 1, WARP_PV = 2, WARP_SM0 = 3;
    static constexpr int WARP_MERGE = WARP_SM0 + NSM;  // merge warp (split partials)
    static constexpr int THREADS = 32 * (4 + NSM);
    static constexpr int HALF_BYTES = kTile * 128;     // one 64-row TMA box of 128-byte rows
    static constexpr int PANEL_BYTES = kStepTokens * 128;  // 128 token rows x 128 bytes
    static constexpr int KV_BYTES = KV8 ? PANEL_BYTES : 2 * PANEL_BYTES;  // one of K, V for a step
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;
    static constexpr int QPANEL_BYTES = RP * 128;      // bf16 query panel: RP rows x 64 d
    static constexpr int QSLOT_BYTES = 2 * QPANEL_BYTES;
    static constexpr int QT_BYTES = KV8 ? NS_COLS * 128 : 0;  // E4M3 query terms: 2 RP rows x 128 d
    // P^T: core matrices of 8 tokens x 16 bytes (8 bf16 or 16 E4M3 columns)
    static constexpr int P_COLS_PER_CORE = KV8 ? 16 : 8;
    static constexpr int P_SBO = (kStepTokens / 8) * 128;     // next 16-byte column group
    static constexpr int P_BYTES = (NO_COLS / P_COLS_PER_CORE) * P_SBO;
    // Buffer counts: the largest bf16 group keeps one query slot and one
    // P^T buffer so three 64 KB stages still fit in shared memory.
    static constexpr int NQ = (!KV8 && RP == 32) ? 1 : 2;
    static constexpr int NP = (!KV8 && RP == 32) ? 1 : 2;
    static constexpr int MAX_STAGES = 8;
    static constexpr int T_LAZY = 8;                   // reference slack, base 2
    // Softmax warps take two steps per pass with 8-bit caches, where halving the
    // per-step exchanges pays (8-bit 70B-shaped batch 200-205 vs 208 us); for bf16
    // the doubled loop costs more in instruction fetch than it saves (R = 16
    // MQA-like sweep 53 vs 61 us).
    static constexpr bool PAIR = KV8 && HW <= 16 && NP == 2;
    // fixed region after the stage ring; every piece 1024-aligned
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_QT = OFF_Q + NQ * QSLOT_BYTES;
    static constexpr int OFF_P = OFF_QT + NQ * QT_BYTES;
    static constexpr int OFF_X = OFF_P + NP * P_BYTES;          // exchange scratch
    static constexpr int X_BYTES = 2 * 4 * 32 * 4 + 2 * 32 * 4 + 2 * 8 * 4;
    static constexpr int OFF_CTRL = OFF_X + ((X_BYTES + 1023) / 1024) * 1024;
    static constexpr int CTRL_BYTES = 1024;
    static constexpr int FIXED_BYTES = OFF_CTRL + CTRL_BYTES;
    static constexpr int smem_bytes(int stages) { return 1024 + stages * STAGE_BYTES + FIXED_BYTES; }
};

struct __align__(16) TcControl {
    uint64_t full[8], empty[8];     // stage ring
    uint64_t qfull[2], qempty[2];   // bf16 query slots (TMA)
    uint64_t qtfull[2], qtempty[2]; // E4M3 query terms (KV8)
    uint64_t sfull[2], sfree[2];    // S^T buffer b written / read by the softmax warps
    uint64_t pfull[2];              // P^T buffer written
    uint64_t pvdone[2];             // value product of the last step using P^T buffer b completed
    uint64_t ofull, ofree;          // O^T of a segment complete / read by the epilogue
    uint64_t xch;                   // softmax-warp exchange (count 4)
    uint64_t drain[2];              // final completion of each issuing warp's products
    uint64_t mjob[2];               // the CTA's first / last segment partial written (merge warp's jobs)
    uint64_t assist;                // the merge warp's ticket for the last segment is known
    int merge_last;                 // ... and it was the unit's last: the softmax warps help merge
    Plan plan;
    uint32_t tmem_base;
    int abort;
};

// Scratch for the softmax warps' exchanges (double-buffered by exchange parity).
struct TcExchange {
    float vals[2][4][32];  // per sub-partition, per head: step maxima or row sums
    float qscale[2][32];   // KV8: 2^-a per head, per query-term slot
    int flags[2][8];       // per softmax warp
};

// One step of a CTA's walk: tiles [tile, tile + n) of the current unit.
struct Step {
    int n;
    bool seg_first, seg_last;
};

__device__ __forceinline__ Step step_at(const Walk& w, int64_t gi, int64_t lo, int64_t hi) {
    Step s;
    s.n = (gi + 1 < hi && w.tile + 1 < w.n_b) ? 2 : 1;
    s.seg_first = (gi == lo) || (w.tile == 0);
    s.seg_last = (gi + s.n == hi) || (w.tile + s.n == w.n_b);
    return s;
}

__device__ __forceinline__ void advance_step(Walk& w, const KernelArgs& a, int64_t& gi, int n, int64_t hi) {
    if (w.tile + n < w.n_b && gi + n < hi) {  // the usual case: the next step is in the same unit
        w.tile += n;
        gi += n;
        return;
    }
    for (int i = 0; i < n; ++i) {
        if (gi + 1 < hi) w.advance(a);
        ++gi;
    }
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_async_smem_writes() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Round-to-nearest-even E4M3 of two floats, packed low byte first (saturating).
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t v) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
    return make_float2(__half2float(__ushort_as_half(h.x)), __half2float(__ushort_as_half(h.y)));
}

// hi + lo split of two weights into the operand type of the value product.
template <bool F16>
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
    if constexpr (F16) {
        const __half2 h = __floats2half2_rn(a, b);
        const float2 hf = __half22float2(h);
        const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
        hi = *reinterpret_cast<const uint32_t*>(&h);
        lo = *reinterpret_cast<const uint32_t*>(&l);
    } else {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
        hi = *reinterpret_cast<const uint32_t*>(&h);
        lo = *reinterpret_cast<const uint32_t*>(&l);
    }
}

template <int RP, bool PAGED, bool OUT_BF16, bool KV8>
__global__ void __launch_bounds__(TcCfg<RP, KV8>::THREADS, 1)
    split_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const KernelArgs a) {
    using C = TcCfg<RP, KV8>;
    static_assert(sizeof(TcControl) <= C::CTRL_BYTES, "control block overflows its slot");
    static_assert(sizeof(TcExchange) <= C::X_BYTES, "exchange scratch overflows its slot");
    constexpr uint32_t IDESC_QK = KV8 ? tc::instr_desc(tc::kFmtE4M3, tc::kFmtE4M3, 0, 0, 128, C::NS_COLS)
                                      : tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 0, 0, 128, C::NS_COLS);
    constexpr uint32_t IDESC_PV = KV8 ? tc::instr_desc(tc::kFmtE4M3, tc::kFmtE4M3, 1, 1, 128, C::NO_COLS)
                                      : tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 1, 1, 128, C::NO_COLS);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const int NS = a.n_stages;
    const uint32_t stages = base;
    const uint32_t fixed = base + NS * C::STAGE_BYTES;
    uint8_t* fixed_ptr = base_ptr + NS * C::STAGE_BYTES;
    const uint32_t q_base = fixed + C::OFF_Q;
    const uint32_t qt_base = fixed + C::OFF_QT;
    const uint32_t p_base = fixed + C::OFF_P;
    TcExchange* X = reinterpret_cast<TcExchange*>(fixed_ptr + C::OFF_X);
    TcControl* ctrl = reinterpret_cast<TcControl*>(fixed_ptr + C::OFF_CTRL);
    volatile int* abort_flag = &ctrl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_addr(&ctrl->full[s]), 1);
            mbar_init(smem_addr(&ctrl->empty[s]), 1);  // freed by the value product
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&ctrl->qfull[s]), 1);
            mbar_init(smem_addr(&ctrl->qempty[s]), KV8 ? C::NSM : 1);
            mbar_init(smem_addr(&ctrl->qtfull[s]), C::NSM);
            mbar_init(smem_addr(&ctrl->qtempty[s]), 1);
            mbar_init(smem_addr(&ctrl->sfull[s]), 1);
            mbar_init(smem_addr(&ctrl->sfree[s]), C::NSM);
            mbar_init(smem_addr(&ctrl->pfull[s]), C::NSM);
            mbar_init(smem_addr(&ctrl->pvdone[s]), 1);
            mbar_init(smem_addr(&ctrl->drain[s]), 1);
        }
        mbar_init(smem_addr(&ctrl->ofull), 1);
        mbar_init(smem_addr(&ctrl->ofree), C::NSM);
        mbar_init(smem_addr(&ctrl->xch), C::NSM);
        for (int k = 0; k < 2; ++k) mbar_init(smem_addr(&ctrl->mjob[k]), C::NSM);
        mbar_init(smem_addr(&ctrl->assist), 1);
        ctrl->abort = 0;
    }
    // Query rows past H_Q come back from TMA as zeros; the P^T buffers start
    // zeroed so their padding columns are finite.
    for (int i = threadIdx.x; i < C::OFF_X / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(fixed_ptr)[i] = make_uint4(0, 0, 0, 0);

    grid_dependency_wait();
    grid_launch_dependents();
    if (warp == 0) make_plan(a, &ctrl->plan);
    if (warp == C::WARP_QK) {
        tc::tmem_alloc(smem_addr(&ctrl->tmem_base), C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    fence_barrier_init();
    fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctrl->tmem_base;

    const int64_t lo = ctrl->plan.lo;
    const int64_t hi = ctrl->plan.hi;
    Walk w{ctrl->plan.b, ctrl->plan.kv, ctrl->plan.tile, ctrl->plan.n_b, ctrl->plan.L};
    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(a.status, kFlagTimeout);
    };

    if (lo < hi && warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        int st = 0, qs = 0;
        uint32_t ph = 0, qph = 0;
        int64_t issued = 0, q_issued = 0;
        bool ok = true;
        for (int64_t gi = lo; gi < hi;) {
            const Step sp = step_at(w, gi, lo, hi);
            if (sp.seg_first) {
                if (!mbar_wait_warp(smem_addr(&ctrl->qempty[qs]), qph ^ 1u, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    const uint32_t bar = smem_addr(&ctrl->qfull[qs]);
                    mbar_arrive_expect_tx(bar, C::QSLOT_BYTES);
                    for (int p = 0; p < 2; ++p)
                        tma_load_3d(q_base + qs * C::QSLOT_BYTES + p * C::QPANEL_BYTES, &tmQ, bar, 64 * p,
                                    w.kv * a.R, w.b, pol_q);
                }
                ++q_issued;
                if (++qs == C::NQ) { qs = 0; qph ^= 1u; }
            }
            // Box coordinates of the step's two tiles; a missing second tile
            // is read from outside the tensor, which fills it with zeros.
            int c2[2], c3[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (PAGED) {
                    int page = a.num_blocks;
                    if (h < sp.n) {
                        page = __ldg(a.block_table + static_cast<int64_t>(w.b) * a.max_blocks + w.tile + h);
                        if ((page < 0 || page >= a.num_blocks) && lane == 0) atomicOr(a.status, kFlagBadBlock);
                    }
                    c2[h] = 0;
                    c3[h] = page;  // out of range: the TMA unit fills the tile with zeros
                } else {
                    c2[h] = h < sp.n ? (w.tile + h) * kTile : a.S_max;
                    c3[h] = w.b;
                }
            }
            if (!mbar_wait_warp(smem_addr(&ctrl->empty[st]), ph ^ 1u, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                const uint32_t bar = smem_addr(&ctrl->full[st]);
                const uint32_t kb = stages + st * C::STAGE_BYTES;
                const uint32_t vb = kb + C::KV_BYTES;
                mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if constexpr (KV8) {
                        tma_load_4d(kb + h * C::HALF_BYTES, &tmK, bar, 0, w.kv, c2[h], c3[h], pol_kv);
                        tma_load_4d(vb + h * C::HALF_BYTES, &tmV, bar, 0, w.kv, c2[h], c3[h], pol_kv);
                    } else {
                        for (int p = 0; p < 2; ++p) {
                            tma_load_4d(kb + p * C::PANEL_BYTES + h * C::HALF_BYTES, &tmK, bar, 64 * p, w.kv,
                                        c2[h], c3[h], pol_kv);
                            tma_load_4d(vb + p * C::PANEL_BYTES + h * C::HALF_BYTES, &tmV, bar, 64 * p, w.kv,
                                        c2[h], c3[h], pol_kv);
                        }
                    }
                }
            }
            ++issued;
            if (++st == NS) { st = 0; ph ^= 1u; }
            advance_step(w, a, gi, sp.n, hi);
        }
        if (!ok) {
            fail();
            // Let copies already in flight land before the CTA's shared memory goes away.
            const int64_t first = issued > NS ? issued - NS : 0;
            for (int64_t i = first; i < issued; ++i)
                mbar_wait(smem_addr(&ctrl->full[i % NS]), static_cast<uint32_t>((i / NS) & 1), nullptr);
            const int64_t qfirst = q_issued > C::NQ ? q_issued - C::NQ : 0;
            for (int64_t i = qfirst; i < q_issued; ++i)
                mbar_wait(smem_addr(&ctrl->qfull[i % C::NQ]), static_cast<uint32_t>((i / C::NQ) & 1), nullptr);
        }
    }

    if (warp == C::WARP_QK) {
        // ------------------------------------------------------------ score products
        // Step j: S^T(j) = K(j) Q^T into buffer j & 1 once the softmax warps
        // have read that buffer's previous contents (step j - 2).
        int st = 0, qs = 0, qcur = 0;
        uint32_t ph = 0, qph = 0;
        bool ok = true;
        if (lo < hi) {
            int j = 0;
            for (int64_t gi = lo; gi < hi; ++j) {
                const Step sp = step_at(w, gi, lo, hi);
                const int sb = j & 1;
                const uint32_t spar = static_cast<uint32_t>(j >> 1) & 1u;
                if (sp.seg_first) {
                    const uint32_t qbar = KV8 ? smem_addr(&ctrl->qtfull[qs]) : smem_addr(&ctrl->qfull[qs]);
                    if (!mbar_wait_warp(qbar, qph, abort_flag)) { ok = false; break; }
                    qcur = qs;
                    if (++qs == C::NQ) { qs = 0; qph ^= 1u; }
                }
                if (!mbar_wait_warp(smem_addr(&ctrl->sfree[sb]), spar ^ 1u, abort_flag)) { ok = false; break; }
                if (!mbar_wait_warp(smem_addr(&ctrl->full[st]), ph, abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    const uint32_t kt = stages + st * C::STAGE_BYTES;
                    const uint32_t sd = tmem + C::S_COL + sb * C::NS_COLS;
                    if constexpr (KV8) {
                        const uint32_t qt = qt_base + qcur * C::QT_BYTES;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t da = tc::smem_desc(kt + 32 * k, 16, 1024, tc::kLayoutSw128);
                            const uint64_t db = tc::smem_desc(qt + 32 * k, 16, 1024, tc::kLayoutSw128);
                            tc::mma_f8(sd, da, db, IDESC_QK, k > 0);
                        }
                    } else {
                        const uint32_t qt = q_base + qcur * C::QSLOT_BYTES;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint64_t da = tc::smem_desc(kt + (k >> 2) * C::PANEL_BYTES + 32 * (k & 3), 16,
                                                              1024, tc::kLayoutSw128);
                            const uint64_t db = tc::smem_desc(qt + (k >> 2) * C::QPANEL_BYTES + 32 * (k & 3), 16,
                                                              1024, tc::kLayoutSw128);
                            tc::mma_f16(sd, da, db, IDESC_QK, k > 0);
                        }
                    }
                    tc::commit(smem_addr(&ctrl->sfull[sb]));
                    if (sp.seg_last)  // the segment's query slot is free once its last score product is done
                        tc::commit(KV8 ? smem_addr(&ctrl->qtempty[qcur]) : smem_addr(&ctrl->qempty[qcur]));
                }
                __syncwarp();
                if (++st == NS) { st = 0; ph ^= 1u; }
                advance_step(w, a, gi, sp.n, hi);
            }
            if (!ok) fail();
        }
        // Every product this warp issued has completed before tensor memory is freed.
        if (tc::elect_one()) tc::commit(smem_addr(&ctrl->drain[0]));
        __syncwarp();
        mbar_wait_warp(smem_addr(&ctrl->drain[0]), 0u, nullptr);
    }

    if (warp == C::WARP_PV) {
        // ------------------------------------------------------------ value products
        // Step j: O^T += V^T(j) P^T(j) once the softmax warps have written P^T(j)
        // (and, KV8, the converters the f16 V rows); a segment's first step
        // overwrites O^T after the epilogue has read the previous segment's.
        int st = 0, seg = -1;
        bool ok = true;
        if (lo < hi) {
            int j = 0;
            for (int64_t gi = lo; gi < hi; ++j) {
                const Step sp = step_at(w, gi, lo, hi);
                const int pb = j % C::NP;
                const uint32_t ppar = static_cast<uint32_t>(j / C::NP) & 1u;
                if (sp.seg_first) ++seg;
                if (!mbar_wait_warp(smem_addr(&ctrl->pfull[pb]), ppar, abort_flag)) { ok = false; break; }
                if (sp.seg_first && seg > 0)
                    if (!mbar_wait_warp(smem_addr(&ctrl->ofree), static_cast<uint32_t>(seg - 1) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    const uint32_t vt = stages + st * C::STAGE_BYTES + C::KV_BYTES;
                    const uint32_t pt = p_base + pb * C::P_BYTES;
                    if constexpr (KV8) {
                        // 32 tokens per product: V^T rows read MN-major (128 d bytes per
                        // token row), P^T as four E4M3 terms per head.
#pragma unroll
                        for (int k = 0; k < kStepTokens / 32; ++k) {
                            const uint64_t da = tc::smem_desc(vt + k * 4096, C::PANEL_BYTES, 1024, tc::kLayoutSw128);
                            const uint64_t db = tc::smem_desc(pt + k * 512, 128, C::P_SBO, tc::kLayoutNone);
                            tc::mma_f8(tmem + C::O_COL, da, db, IDESC_PV, !(sp.seg_first && k == 0));
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < kStepTokens / 16; ++k) {
                            const uint64_t da = tc::smem_desc(vt + k * 2048, C::PANEL_BYTES, 1024, tc::kLayoutSw128);
                            const uint64_t db = tc::smem_desc(pt + k * 256, 128, C::P_SBO, tc::kLayoutNone);
                            tc::mma_f16(tmem + C::O_COL, da, db, IDESC_PV, !(sp.seg_first && k == 0));
                        }
                    }
                    tc::commit(smem_addr(&ctrl->empty[st]));
                    tc::commit(smem_addr(&ctrl->pvdone[pb]));
                    if (sp.seg_last) tc::commit(smem_addr(&ctrl->ofull));
                }
                __syncwarp();
                if (++st == NS) st = 0;
                advance_step(w, a, gi, sp.n, hi);
            }
            if (!ok) fail();
        }
        if (tc::elect_one()) tc::commit(smem_addr(&ctrl->drain[1]));
        __syncwarp();
        mbar_wait_warp(smem_addr(&ctrl->drain[1]), 0u, nullptr);
    }

    if (lo < hi && warp >= C::WARP_SM0 && warp < C::WARP_SM0 + C::NSM) {
        // ------------------------------------------------------------ softmax + epilogue
        const int sp = warp & 3;            // tensor-memory sub-partition of this warp
        const int wi = warp - C::WARP_SM0;  // softmax warp index
        const int h0 = C::HSPLIT == 1 ? 0 : (wi >> 2) * C::HW;  // first query column of this warp
        const int tok = 32 * sp + lane;     // S^T row (token of the step) held by this thread
        constexpr int HW = C::HW;
        const float NEG_INF = -__int_as_float(0x7f800000);
        float m[HW], l[HW];
        uint32_t xpar = 0, qph = 0;
        int qs = 0, qcur = 0, seg = -1, seg_start_tile = 0, st = 0;
        bool tail_cut = false;  // the CTA's last segment so far was cut (its unit is merged)
        int tail_b = 0, tail_kv = 0, tail_nb = 0;
        int64_t tail_su = 0;
        float vfac = 1.f, qf_uniform = a.sl2;
        float qfac[KV8 ? HW : 1];  // KV8: the segment's score factor per head, qf_uniform * 2^-a
        bool ok = true;

        auto exchange = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->xch));
            const bool r = mbar_wait_warp(smem_addr(&ctrl->xch), xpar, abort_flag);
            xpar ^= 1u;
            return r;
        };

        int j = 0;
        for (int64_t gi = lo; gi < hi;) {
            const Step stp = step_at(w, gi, lo, hi);
            if (stp.seg_first) {
                ++seg;
                seg_start_tile = w.tile;
                qcur = qs;
                const uint32_t qpar = qph;  // phase of this use of slot qcur
                (void)qpar;
                if (++qs == C::NQ) { qs = 0; qph ^= 1u; }
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    m[h] = NEG_INF;
                    l[h] = 0.f;
                }
                if constexpr (KV8) {
                    vfac = __ldg(a.v_scale + w.kv);
                    qf_uniform = a.sl2 * __ldg(a.k_scale + w.kv);
                    if (!mbar_wait_warp(smem_addr(&ctrl->qfull[qcur]), qpar, abort_flag)) { ok = false; break; }
                    if (!mbar_wait_warp(smem_addr(&ctrl->qtempty[qcur]), qpar ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // Query head hh -> two E4M3 terms (rows hh and RP + hh of the term slot).
                    const uint32_t qsrc = q_base + qcur * C::QSLOT_BYTES;
                    const uint32_t qdst = qt_base + qcur * C::QT_BYTES;
                    const int d0 = 4 * lane;
                    for (int hh = wi; hh < RP; hh += C::NSM) {
                        const int pnl = d0 >> 6, ch = (d0 & 63) >> 3;
                        const uint2 wq = ld_shared_v2(qsrc + pnl * C::QPANEL_BYTES + hh * 128 +
                                                      ((ch ^ (hh & 7)) << 4) + ((d0 & 7) << 1));
                        float q[4];
                        q[0] = __uint_as_float(wq.x << 16);
                        q[1] = __uint_as_float(wq.x & 0xffff0000u);
                        q[2] = __uint_as_float(wq.y << 16);
                        q[3] = __uint_as_float(wq.y & 0xffff0000u);
                        if (hh >= a.R) q[0] = q[1] = q[2] = q[3] = 0.f;
                        float mx = fmaxf(fmaxf(fabsf(q[0]), fabsf(q[1])), fmaxf(fabsf(q[2]), fabsf(q[3])));
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        // 2^a with max |q| 2^a in [128, 256)
                        const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127;
                        int sa = mx > 0.f ? 7 - e : 0;
                        sa = sa > 120 ? 120 : (sa < -120 ? -120 : sa);
                        const float up = __uint_as_float(static_cast<uint32_t>(sa + 127) << 23);
                        const float down = __uint_as_float(static_cast<uint32_t>(127 - sa) << 23);
                        float x[4], r[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) x[i] = q[i] * up;
                        const uint16_t t1a = f32x2_to_e4m3x2(x[0], x[1]);
                        const uint16_t t1b = f32x2_to_e4m3x2(x[2], x[3]);
                        const float2 b1a = e4m3x2_to_f32x2(t1a), b1b = e4m3x2_to_f32x2(t1b);
                        r[0] = (x[0] - b1a.x) * 16.f;
                        r[1] = (x[1] - b1a.y) * 16.f;
                        r[2] = (x[2] - b1b.x) * 16.f;
                        r[3] = (x[3] - b1b.y) * 16.f;
                        const uint16_t t2a = f32x2_to_e4m3x2(r[0], r[1]);
                        const uint16_t t2b = f32x2_to_e4m3x2(r[2], r[3]);
                        const int row2 = RP + hh;
                        const uint32_t a1 = qdst + hh * 128 + (((d0 >> 4) ^ (hh & 7)) << 4) + (d0 & 15);
                        const uint32_t a2 = qdst + row2 * 128 + (((d0 >> 4) ^ (row2 & 7)) << 4) + (d0 & 15);
                        st_shared_u32(a1, static_cast<uint32_t>(t1a) | (static_cast<uint32_t>(t1b) << 16));
                        st_shared_u32(a2, static_cast<uint32_t>(t2a) | (static_cast<uint32_t>(t2b) << 16));
                        if (lane == 0) X->qscale[qcur][hh] = mx > 0.f ? down : 0.f;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&ctrl->qempty[qcur]));  // bf16 query slot read
                    fence_async_smem_writes();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&ctrl->qtfull[qcur]));
                    if (!exchange()) { ok = false; break; }  // every head's 2^-a is in place
#pragma unroll
                    for (int h = 0; h < HW; ++h) qfac[h] = qf_uniform * X->qscale[qcur][h0 + h];
                }
            }
            // The softmax warps take two steps of a segment per pass (one when the
            // segment ends after the first), so one exchange and one round of
            // barrier hops serve up to 256 tokens.
            int nsub = 1, n_of[2] = {stp.n, 0}, tile_of[2] = {w.tile, 0};
            bool seg_last = stp.seg_last;
            if constexpr (C::PAIR) {
                if (!stp.seg_last) {
                    const int64_t g1 = gi + stp.n;
                    tile_of[1] = w.tile + stp.n;
                    n_of[1] = (g1 + 1 < hi && tile_of[1] + 1 < w.n_b) ? 2 : 1;
                    seg_last = (g1 + n_of[1] == hi) || (tile_of[1] + n_of[1] == w.n_b);
                    nsub = 2;
                }
            }
            const bool last_of_unit = (tile_of[nsub - 1] + n_of[nsub - 1] == w.n_b);
            constexpr int MS = C::PAIR ? 2 : 1;

            // ---- scores of this thread's token in each step
            float s[MS][HW];
#pragma unroll
            for (int u = 0; u < MS; ++u) {
                if (u >= nsub) break;
                const int ju = j + u, sb = ju & 1;
                if (!mbar_wait_warp(smem_addr(&ctrl->sfull[sb]), static_cast<uint32_t>(ju >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t ta = tc::tmem_addr(tmem, 32 * sp, C::S_COL + sb * C::NS_COLS);
                if constexpr (!KV8) {
#pragma unroll
                    for (int c = 0; c < HW / 16; ++c) {
                        uint32_t r[16];
                        tc::tmem_ld16(ta + h0 + 16 * c, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) s[u][16 * c + i] = __uint_as_float(r[i]) * qf_uniform;
                    }
                } else {
                    // columns h (term 1) and RP + h (term 2), 8 heads at a time
#pragma unroll
                    for (int c = 0; c < HW / 8; ++c) {
                        uint32_t r1[8], r2[8];
                        tc::tmem_ld8(ta + h0 + 8 * c, r1);
                        tc::tmem_ld8(ta + RP + h0 + 8 * c, r2);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            s[u][8 * c + i] =
                                (__uint_as_float(r1[i]) + __uint_as_float(r2[i]) * 0.0625f) * qfac[8 * c + i];
                    }
                }
                // S^T buffer sb may take the step after next
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->sfree[sb]));
                const bool valid = tok < kTile * n_of[u] && tile_of[u] * kTile + tok < w.L;
#pragma unroll
                for (int h = 0; h < HW; ++h)
                    if (!valid || h0 + h >= a.R) s[u][h] = NEG_INF;
            }
            if (!ok) break;

            // ---- reference check: does any score exceed its head's reference by more than T?
            // The flags go out first; the weights against the current reference are
            // computed while the other warps' flags arrive, and recomputed only when
            // some warp found an excess (normally the first step of a segment).
            bool exceed = false;
#pragma unroll
            for (int u = 0; u < MS; ++u)
                if (u < nsub) {
#pragma unroll
                    for (int h = 0; h < HW; ++h) exceed |= s[u][h] > m[h] + static_cast<float>(C::T_LAZY);
                }
            float p[MS][HW];
            {
                const uint32_t xb = xpar;
                const bool any = __any_sync(0xffffffffu, exceed);
                if (lane == 0) X->flags[xb][wi] = any ? 1 : 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->xch));
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    const float ref = m[h] == NEG_INF ? 0.f : m[h];
#pragma unroll
                    for (int u = 0; u < MS; ++u) p[u][h] = u < nsub ? fast_exp2(s[u][h] - ref) : 0.f;
                }
                const bool xok = mbar_wait_warp(smem_addr(&ctrl->xch), xpar, abort_flag);
                xpar ^= 1u;
                if (!xok) { ok = false; break; }
                int any_flag = 0;
#pragma unroll
                for (int k = 0; k < C::NSM; ++k) any_flag |= X->flags[xb][k];
                const bool slow = any_flag != 0;
                if (slow) {
                    float mx[HW];
#pragma unroll
                    for (int h = 0; h < HW; ++h) {
                        float v = s[0][h];
                        if (MS > 1 && nsub > 1) v = fmaxf(v, s[MS - 1][h]);
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                        mx[h] = v;
                    }
                    const uint32_t xb2 = xpar;
                    if (lane == 0) {
#pragma unroll
                        for (int h = 0; h < HW; h += 4)
                            *reinterpret_cast<float4*>(&X->vals[xb2][sp][h0 + h]) =
                                make_float4(mx[h], mx[h + 1], mx[h + 2], mx[h + 3]);
                    }
                    if (!exchange()) { ok = false; break; }
                    float alpha[HW];
                    bool moved = false;
#pragma unroll
                    for (int h = 0; h < HW; ++h) {
                        const float M = fmaxf(fmaxf(X->vals[xb2][0][h0 + h], X->vals[xb2][1][h0 + h]),
                                              fmaxf(X->vals[xb2][2][h0 + h], X->vals[xb2][3][h0 + h]));
                        alpha[h] = 1.f;
                        if (M > m[h] + static_cast<float>(C::T_LAZY)) {
                            alpha[h] = m[h] == NEG_INF ? 0.f : fast_exp2(m[h] - M);
                            moved |= m[h] != NEG_INF;
                            m[h] = M;
                        }
                        l[h] *= alpha[h];
                        const float ref = m[h] == NEG_INF ? 0.f : m[h];
#pragma unroll
                        for (int u = 0; u < MS; ++u) p[u][h] = u < nsub ? fast_exp2(s[u][h] - ref) : 0.f;
                    }
                    if (moved && w.tile != seg_start_tile) {
                        // O^T holds this segment's earlier steps: rescale it in place once
                        // the previous step's value product has landed.
                        if (!mbar_wait_warp(smem_addr(&ctrl->pvdone[(j - 1) % C::NP]),
                                            static_cast<uint32_t>((j - 1) / C::NP) & 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
#pragma unroll
                        for (int k = 0; k < C::NPT; ++k)
#pragma unroll
                            for (int c = 0; c < HW / 8; ++c) {
                                const uint32_t oa = tc::tmem_addr(tmem, 32 * sp, C::O_COL + k * RP + h0 + 8 * c);
                                uint32_t r[8];
                                tc::tmem_ld8(oa, r);
                                tc::tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha[8 * c + e]);
                                tc::tmem_st8(oa, r);
                            }
                        tc::tmem_wait_st();
                    }
                }
            }

            // ---- row sums, P^T for each step's value product
#pragma unroll
            for (int h = 0; h < HW; ++h)
#pragma unroll
                for (int u = 0; u < MS; ++u) l[h] += p[u][h];
#pragma unroll
            for (int u = 0; u < MS; ++u) {
                if (u >= nsub) break;
                const int ju = j + u, pb = ju % C::NP;
                if (!mbar_wait_warp(smem_addr(&ctrl->pvdone[pb]), (static_cast<uint32_t>(ju / C::NP) & 1u) ^ 1u,
                                    abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t pt = p_base + pb * C::P_BYTES + (tok >> 3) * 128 + (tok & 7) * 16;
                if constexpr (KV8) {
                    // p = t1 + t2 / 16 + t3 / 256 + t4 / 4096, each term E4M3 (p <= 2^8 < 448);
                    // columns are [t1 | t2 | t3 | t4], RP heads each.
                    uint32_t wd[HW];  // term k, heads 4i..4i+3 -> wd[k * HW / 4 + i]
#pragma unroll
                    for (int i = 0; i < HW / 4; ++i) {
                        float x0 = p[u][4 * i], x1 = p[u][4 * i + 1], x2 = p[u][4 * i + 2], x3 = p[u][4 * i + 3];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint16_t b01 = f32x2_to_e4m3x2(x0, x1);
                            const uint16_t b23 = f32x2_to_e4m3x2(x2, x3);
                            wd[k * (HW / 4) + i] = static_cast<uint32_t>(b01) | (static_cast<uint32_t>(b23) << 16);
                            if (k < 3) {
                                const float2 f01 = e4m3x2_to_f32x2(b01), f23 = e4m3x2_to_f32x2(b23);
                                x0 = (x0 - f01.x) * 16.f;
                                x1 = (x1 - f01.y) * 16.f;
                                x2 = (x2 - f23.x) * 16.f;
                                x3 = (x3 - f23.y) * 16.f;
                            }
                        }
                    }
                    if constexpr (HW >= 16) {
                        // term k: columns k RP + h0 .. + HW, whole 16-column groups
#pragma unroll
                        for (int k = 0; k < 4; ++k)
#pragma unroll
                            for (int gg = 0; gg < HW / 16; ++gg) {
                                const int w0 = k * (HW / 4) + 4 * gg;
                                st_shared_v4(pt + ((k * RP + h0) / 16 + gg) * C::P_SBO, wd[w0], wd[w0 + 1],
                                             wd[w0 + 2], wd[w0 + 3]);
                            }
                    } else {
                        // eight columns per term: two terms per 16-column group
#pragma unroll
                        for (int g = 0; g < HW / 4; ++g)
                            st_shared_v4(pt + g * C::P_SBO, wd[4 * g], wd[4 * g + 1], wd[4 * g + 2], wd[4 * g + 3]);
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < HW / 8; ++g) {
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            split_pair<false>(p[u][8 * g + 2 * e], p[u][8 * g + 2 * e + 1], hw[e], lw[e]);
                        st_shared_v4(pt + (h0 / 8 + g) * C::P_SBO, hw[0], hw[1], hw[2], hw[3]);
                        st_shared_v4(pt + ((RP + h0) / 8 + g) * C::P_SBO, lw[0], lw[1], lw[2], lw[3]);
                    }
                }
                // Loaded value rows past L_b may hold anything; 0 * NaN would poison O^T.
                const bool loaded = tok < kTile * n_of[u];
                if (h0 == 0 && tile_of[u] + n_of[u] == w.n_b && loaded && tile_of[u] * kTile + tok >= w.L) {
                    const int stu = st + u < NS ? st + u : st + u - NS;
                    const uint32_t vrow = stages + stu * C::STAGE_BYTES + C::KV_BYTES + tok * 128;
#pragma unroll
                    for (int pnl = 0; pnl < (KV8 ? 1 : 2); ++pnl)
#pragma unroll
                        for (int c = 0; c < 8; ++c) st_shared_v4(vrow + pnl * C::PANEL_BYTES + 16 * c, 0u, 0u, 0u, 0u);
                }
                fence_async_smem_writes();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->pfull[pb]));
            }
            if (!ok) break;

            if (seg_last) {
                // ---------------------------------------------------- segment end
                float lt[HW];
#pragma unroll
                for (int h = 0; h < HW; ++h) {
                    float v = l[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    lt[h] = v;
                }
                const uint32_t xb3 = xpar;
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < HW; h += 4)
                        *reinterpret_cast<float4*>(&X->vals[xb3][sp][h0 + h]) =
                            make_float4(lt[h], lt[h + 1], lt[h + 2], lt[h + 3]);
                }
                if (!exchange()) { ok = false; break; }
#pragma unroll
                for (int h = 0; h < HW; ++h)
                    lt[h] = (X->vals[xb3][0][h0 + h] + X->vals[xb3][1][h0 + h]) +
                            (X->vals[xb3][2][h0 + h] + X->vals[xb3][3][h0 + h]);
                if (!mbar_wait_warp(smem_addr(&ctrl->ofull), static_cast<uint32_t>(seg) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const int d = 32 * sp + lane;  // O^T row
                const bool whole = (seg_start_tile == 0) && last_of_unit;
                const int64_t slot = 2 * static_cast<int64_t>(blockIdx.x) + (seg == 0 ? 0 : 1);
#pragma unroll
                for (int c = 0; c < HW / 8; ++c) {
                    // the P terms' columns: hi + lo, or t1 + t2 / 16 + t3 / 256 + t4 / 4096
                    float acc[8];
                    {
                        uint32_t tv[8];
                        tc::tmem_ld8(tc::tmem_addr(tmem, 32 * sp, C::O_COL + h0 + 8 * c), tv);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] = __uint_as_float(tv[e]);
                    }
#pragma unroll
                    for (int k = C::NPT - 1; k >= 1; --k) {
                        uint32_t tv[8];
                        tc::tmem_ld8(tc::tmem_addr(tmem, 32 * sp, C::O_COL + k * RP + h0 + 8 * c), tv);
                        tc::tmem_wait_ld();
                        const float wk = KV8 ? 1.f / static_cast<float>(1 << (4 * k)) : 1.f;
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] += __uint_as_float(tv[e]) * wk;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int hl = 8 * c + e, h = h0 + hl;
                        if (h >= a.R) continue;
                        const float o = acc[e] * (vfac / lt[hl]);
                        if (whole) {
                            const int64_t i = (static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R + h) * C::D + d;
                            if constexpr (OUT_BF16)
                                static_cast<__nv_bfloat16*>(a.out)[i] = __float2bfloat16_rn(o);
                            else
                                static_cast<float*>(a.out)[i] = o;
                        } else {
                            a.ws_o[(slot * a.R + h) * C::D + d] = o;
                        }
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->ofree));  // O^T read: the next segment may start
                if (!whole) {
                    if (sp == 0 && lane == 0) {
#pragma unroll
                        for (int h = 0; h < HW; ++h)
                            if (h0 + h < a.R) a.ws_lse[slot * a.R + h0 + h] = m[h] + log2f(lt[h]);
                    }
                    // this warp's share of the partial is written: hand it to the merge warp
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&ctrl->mjob[seg == 0 ? 0 : 1]));
                }
                tail_cut = !whole;
                tail_b = w.b;
                tail_kv = w.kv;
                tail_nb = w.n_b;
                tail_su = gi - w.tile;
            }
            st += nsub;  // nsub <= 2 <= NS: no division on the per-pass path
            if (st >= NS) st -= NS;
            j += nsub;
            advance_step(w, a, gi, stp.n, hi);
            if (nsub > 1) advance_step(w, a, gi, n_of[1], hi);
        }
        if (!ok) fail();
        // The CTA's last segment was cut: help the merge warp merge its unit.
        if (ok && tail_cut &&
            !merge_assist<C::D, OUT_BF16>(a, &ctrl->assist, &ctrl->merge_last, tail_b, tail_kv, tail_su, tail_nb,
                                          ctrl->plan.n_tiles, ctrl->plan.g, wi, C::NSM + 1, abort_flag))
            fail();
    }

    if (warp == C::WARP_MERGE) {
        // ------------------------------------------------------------ merge warp
        if (!merge_warp<C::D, OUT_BF16>(a, ctrl->plan, ctrl->mjob, &ctrl->assist, &ctrl->merge_last, C::NSM,
                                        abort_flag))
            fail();
    }

    // ---------------------------------------------------------------- teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == C::WARP_QK) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace gqa

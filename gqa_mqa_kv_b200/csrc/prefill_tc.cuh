// prefill_tc.cuh -- multi-token (prefill, or a prompt chunk after a cached
// prefix) grouped-query attention on the tcgen05 tensor cores, head_dim 128.
//
// What it computes ("Grouped-Query Attention (GQA) and Multi-Query Attention
// (MQA): Mathematical Foundations, ...", section 2: Head_i = softmax(Q_i
// K_{g(i)}^T / sqrt(d_k) + M) V_{g(i)} with the causal mask M; the opening
// section names prompt processing, prefill, as the compute-bound phase):
// sequence b brings n_b new query tokens -- rows cu_q[b] .. cu_q[b+1]-1 of q
// -- whose keys and values are the last n_b of its L_b cached tokens.  Token
// j sits at position p = L_b - n_b + j and attends to cache positions t <= p.
//
// Work unit: TQ = floor(128 / R) consecutive query tokens of one sequence
// and one KV head kv, as one M = 128 row tile whose row r is token r / R and
// query head kv R + r % R: every K/V row brought on chip serves all R heads
// of the group.  The unit walks its visible keys 128 at a time:
//   S = Q K^T       tcgen05.mma, M = 128 rows, N = 128 keys, K = d: A = the
//                   query rows, B = the key rows, both K-major with the
//                   128-byte swizzle as TMA stages them; S lands in tensor
//                   memory (two buffers: the next step's product overlaps
//                   this step's softmax).
//   softmax         eight warps, two per tensor-memory sub-partition:
//                   thread = row = TMEM lane, each warp of a pair taking 64
//                   of the step's keys in registers.  Base-2 online softmax
//                   against a per-row reference that moves only when a score
//                   exceeds it by more than 8 (O is rescaled in tensor memory
//                   then); the pair agrees on the reference through a
//                   shared-memory exchange of partial maxima each step.  P
//                   replaces S in its own tensor-memory columns as bf16 hi
//                   and lo parts (two per 32-bit column), so the product
//                   keeps ~16 bits of every weight and the two S buffers
//                   double as two P buffers.
//   O += P V        tcgen05.mma, M = 128, N = d = 128, K = 128 keys, once on
//                   the hi part and once on the lo part; A = P read from
//                   tensor memory, B = the value rows read MN-major; O in
//                   tensor memory (two buffers, one per unit in flight),
//                   normalised by the row sum at the end.  The value product
//                   of a step releases its S/P buffer to the score product
//                   two steps later.
//
// Persistent CTAs (one per SM) walk the units in a fixed interleaved order,
// heaviest query tiles first.  Warp roles: 0 TMA producer, 1 score products
// (+ tensor-memory allocation), 2 value products, 3..10 softmax and epilogue
// (warp w on sub-partition w % 4, keys 64 ((w - 3) / 4) ..).  Every wait is
// bounded (kWaitTimeoutNs); on a
// timeout the CTA raises GQA_FLAG_TIMEOUT, lets its copies and products
// drain, frees its tensor memory and returns.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "schedule.cuh"
#include "tcgen05.cuh"

namespace gqa {

struct PrefillArgs {
    const int32_t* seq_lens;     // [B]
    const int32_t* cu_q;         // [B + 1]: query rows of sequence b are cu_q[b] .. cu_q[b+1]-1
    const int32_t* block_table;  // [B, max_blocks] or null
    int B, H_Q, H_KV, R;
    int TQ;          // query tokens per tile: floor(128 / R)
    int QT;          // tiles per sequence: ceil(max_q / TQ)
    int max_q;       // host bound on n_b
    int total_q;     // rows of q and out
    int max_len;     // seq_lens are clamped to [0, max_len]
    int S_max;       // contiguous cache capacity; 0 when paged
    int max_blocks, num_blocks;
    float sl2;       // softmax scale * log2(e)
    void* out;       // [total_q, H_Q, 128]
    uint32_t* status;
};

struct PfCfg {
    static constexpr int D = 128;
    static constexpr int BN = 128;                 // keys per step
    static constexpr int PANEL = 128 * 128;        // 128 rows x 128 bytes (64 bf16 of d, or of keys)
    static constexpr int TILE = 2 * PANEL;         // 128 rows x 128 bf16
    static constexpr int BOX = 64 * 128;           // one 64-row TMA box of 128-byte rows
    static constexpr int NS = 6;                   // K/V ring entries (K and V of a step alternate)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = OFF_Q + TILE;
    static constexpr int OFF_CTRL = OFF_RING + NS * TILE;
    static constexpr int CTRL_BYTES = 2048;
    static constexpr int SMEM_BYTES = 1024 + OFF_CTRL + CTRL_BYTES;  // + 1024-byte alignment slack
    static constexpr int S_COL = 0;                // S buffer b at S_COL + 128 b; P hi | lo replaces S there
    static constexpr int O_COL = 256;              // O buffer b at O_COL + 128 b
    static constexpr int TMEM_COLS = 512;
    static constexpr int WARP_TMA = 0, WARP_QK = 1, WARP_PV = 2, WARP_SM0 = 3;
    static constexpr int NSM = 8;                  // softmax warps: two per sub-partition, 64 keys each
    static constexpr int THREADS = 32 * (3 + NSM);
    static constexpr int T_LAZY = 8;               // reference slack, base 2
};

struct __align__(16) PfControl {
    uint64_t full[PfCfg::NS], empty[PfCfg::NS];  // K/V ring
    uint64_t qfull, qempty;                      // query tile
    uint64_t sfull[2], sfree[2];                 // S buffer written / its P read by the value product
    uint64_t pfull, pvdone;                      // P written / value product of the last step done
    uint64_t ofull[2], ofree[2];                 // O buffer of a unit complete / read by the epilogue
    uint64_t drain[2];                           // last products of each issuing warp complete
    uint64_t xfull[4], xfree[4];                 // per sub-partition: both halves wrote / read xval
    uint32_t tmem_base;
    int abort;
    float xval[2][128];                          // per key half, per row: a partial row max or row sum
};

// One work unit as every warp role derives it from the unit index.
struct PfUnit {
    int b, kv, qt;
    int n_tok;   // query tokens in the tile (rows n_tok * R .. 127 are idle)
    int q_row0;  // row of q / out of the tile's first token
    int pos0;    // cache position of the tile's first token
    int L;       // clamped cache length
    int steps;   // 128-key steps: keys [0, pos0 + n_tok) are visible to some row
};

// Unit u: query tile qt = QT - 1 - u / (B H_KV) (heaviest first), then
// sequence b, then KV head.  Returns false for a unit with no rows; *flags
// gets the status bits the sequence's bounds raise (a clamped length, an
// inconsistent query span -- such a sequence is skipped).
__device__ __forceinline__ bool pf_unit(const PrefillArgs& a, int u, PfUnit& x, uint32_t* flags) {
    const int per = a.B * a.H_KV;
    const int t = u / per;
    const int rem = u - t * per;
    x.qt = a.QT - 1 - t;
    x.b = rem / a.H_KV;
    x.kv = rem - x.b * a.H_KV;
    const int c0 = __ldg(a.cu_q + x.b), c1 = __ldg(a.cu_q + x.b + 1);
    const int raw = __ldg(a.seq_lens + x.b);
    x.L = clamp_len(raw, a.max_len);
    uint32_t f = (raw < 0 || raw > a.max_len) ? kFlagClamped : 0u;
    const int n = c1 - c0;
    const bool span_ok = c0 >= 0 && c1 <= a.total_q && n >= 0 && n <= x.L && n <= a.max_q;
    if (!span_ok) f |= kFlagBadSpan;
    *flags = f;
    if (!span_ok) return false;
    const int tok0 = x.qt * a.TQ;
    if (tok0 >= n) return false;
    x.n_tok = min(a.TQ, n - tok0);
    x.q_row0 = c0 + tok0;
    x.pos0 = x.L - n + tok0;
    x.steps = (x.pos0 + x.n_tok + PfCfg::BN - 1) / PfCfg::BN;
    return true;
}

__device__ __forceinline__ void pf_fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes of work).
__device__ __forceinline__ uint64_t pf_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float2 pf_unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}

__device__ __forceinline__ uint64_t pf_fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t pf_add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float pf_max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// p0, p1 -> bf16 hi parts (truncated: the top 16 bits of each fp32) and bf16
// lo parts (round to nearest of the exact remainder); hi + lo is within
// 2^-15 of each weight.  p0 lands in the low half of each packed word.
__device__ __forceinline__ void pf_split(float p0, float p1, uint64_t neg1, uint32_t& hi, uint32_t& lo) {
    const uint32_t a = __float_as_uint(p0), b = __float_as_uint(p1);
    hi = __byte_perm(a, b, 0x7632);
    const uint64_t rem = pf_fma2(pf_pack(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u)), neg1,
                                 pf_pack(p0, p1));
    const float2 r = pf_unpack(rem);
    const __nv_bfloat162 l2 = __floats2bfloat162_rn(r.x, r.y);
    lo = *reinterpret_cast<const uint32_t*>(&l2);
}

template <bool PAGED, bool OUT_BF16>
__global__ void __launch_bounds__(PfCfg::THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
    using C = PfCfg;
    static_assert(sizeof(PfControl) <= C::CTRL_BYTES, "control block overflows its slot");
    constexpr uint32_t IDESC_QK = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 0, 0, 128, C::BN);
    constexpr uint32_t IDESC_PV = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 0, 1, 128, C::D);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const uint32_t q_smem = base + C::OFF_Q;
    const uint32_t ring = base + C::OFF_RING;
    PfControl* ctrl = reinterpret_cast<PfControl*>(base_ptr + C::OFF_CTRL);
    volatile int* abort_flag = &ctrl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = a.B * a.H_KV * a.QT;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(smem_addr(&ctrl->full[s]), 1);
            mbar_init(smem_addr(&ctrl->empty[s]), 1);
        }
        mbar_init(smem_addr(&ctrl->qfull), 1);
        mbar_init(smem_addr(&ctrl->qempty), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&ctrl->sfull[s]), 1);
            mbar_init(smem_addr(&ctrl->sfree[s]), 1);  // committed by the value product
            mbar_init(smem_addr(&ctrl->ofull[s]), 1);
            mbar_init(smem_addr(&ctrl->ofree[s]), C::NSM);
            mbar_init(smem_addr(&ctrl->drain[s]), 1);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(smem_addr(&ctrl->xfull[s]), 2);
            mbar_init(smem_addr(&ctrl->xfree[s]), 2);
        }
        mbar_init(smem_addr(&ctrl->pfull), C::NSM);
        mbar_init(smem_addr(&ctrl->pvdone), 1);
        ctrl->abort = 0;
    }
    // Query rows the TMA box leaves out (R * TQ < 128) stay zero.
    for (int i = threadIdx.x; i < C::TILE / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base_ptr + C::OFF_Q)[i] = make_uint4(0, 0, 0, 0);
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

    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(a.status, kFlagTimeout);
    };

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------------ producer
        // K/V rows are read again by the sequence's other query tiles: keep them in L2.
        const uint64_t pol_kv = policy_evict_last();
        const uint64_t pol_q = policy_evict_first();
        int64_t ld = 0;  // K/V loads issued: K of step g is load 2g, V is 2g + 1
        int uc = 0;      // units issued
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            PfUnit x;
            uint32_t fl;
            const bool has = pf_unit(a, u, x, &fl);
            if (fl != 0u && lane == 0 && x.kv == 0 && x.qt == a.QT - 1) atomicOr(a.status, fl);
            if (!has) continue;
            if (!mbar_wait_warp(smem_addr(&ctrl->qempty), (static_cast<uint32_t>(uc) & 1u) ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                const uint32_t bar = smem_addr(&ctrl->qfull);
                mbar_arrive_expect_tx(bar, 2u * 128u * static_cast<uint32_t>(a.R * a.TQ));
                for (int p = 0; p < 2; ++p)
                    tma_load_3d(q_smem + p * C::PANEL, &tmQ, bar, 64 * p, x.kv * a.R, x.q_row0, pol_q);
            }
            ++uc;
            const int kv_end = x.pos0 + x.n_tok;
            for (int j = 0; j < x.steps && ok; ++j) {
                // Coordinates of the step's two 64-key tiles; a tile past the visible
                // keys is read from outside the tensor, which fills it with zeros.
                int c2[2], c3[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int t = 2 * j + h;
                    const bool need = t * kTile < kv_end;
                    if constexpr (PAGED) {
                        int page = a.num_blocks;
                        if (need) {
                            page = __ldg(a.block_table + static_cast<int64_t>(x.b) * a.max_blocks + t);
                            if (page < 0 || page >= a.num_blocks) {
                                if (lane == 0) atomicOr(a.status, kFlagBadBlock);
                                page = a.num_blocks;
                            }
                        }
                        c2[h] = 0;
                        c3[h] = page;
                    } else {
                        c2[h] = need ? t * kTile : a.S_max;
                        c3[h] = x.b;
                    }
                }
#pragma unroll
                for (int which = 0; which < 2; ++which) {  // K, then V
                    const int e = static_cast<int>(ld % C::NS);
                    const uint32_t ph = static_cast<uint32_t>(ld / C::NS) & 1u;
                    if (!mbar_wait_warp(smem_addr(&ctrl->empty[e]), ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        const uint32_t bar = smem_addr(&ctrl->full[e]);
                        const uint32_t dst = ring + e * C::TILE;
                        const CUtensorMap* map = which == 0 ? &tmK : &tmV;
                        mbar_arrive_expect_tx(bar, C::TILE);
#pragma unroll
                        for (int p = 0; p < 2; ++p)
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                tma_load_4d(dst + p * C::PANEL + h * C::BOX, map, bar, 64 * p, x.kv, c2[h], c3[h],
                                            pol_kv);
                    }
                    ++ld;
                }
            }
        }
        if (!ok) {
            fail();
            // Let copies already in flight land before the CTA's shared memory goes away.
            const int64_t first = ld > C::NS ? ld - C::NS : 0;
            for (int64_t i = first; i < ld; ++i)
                mbar_wait(smem_addr(&ctrl->full[i % C::NS]), static_cast<uint32_t>((i / C::NS) & 1), nullptr);
            if (uc > 0) mbar_wait(smem_addr(&ctrl->qfull), static_cast<uint32_t>(uc - 1) & 1u, nullptr);
        }
    }

    if (warp == C::WARP_QK) {
        // ------------------------------------------------------------ score products
        // Global step g: S(g) = Q K(g)^T into buffer g & 1 once the value product
        // of step g - 2 has read the P that replaced that buffer's S.
        int64_t g = 0;
        int uc = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            PfUnit x;
            uint32_t fl;
            if (!pf_unit(a, u, x, &fl)) continue;
            if (!mbar_wait_warp(smem_addr(&ctrl->qfull), static_cast<uint32_t>(uc) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            for (int j = 0; j < x.steps; ++j, ++g) {
                const int sb = static_cast<int>(g & 1);
                const uint32_t spar = static_cast<uint32_t>(g >> 1) & 1u;
                const int64_t ki = 2 * g;
                const int e = static_cast<int>(ki % C::NS);
                if (!mbar_wait_warp(smem_addr(&ctrl->sfree[sb]), spar ^ 1u, abort_flag) ||
                    !mbar_wait_warp(smem_addr(&ctrl->full[e]), static_cast<uint32_t>(ki / C::NS) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    const uint32_t kt = ring + e * C::TILE;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t off = (k >> 2) * C::PANEL + 32 * (k & 3);
                        const uint64_t da = tc::smem_desc(q_smem + off, 16, 1024, tc::kLayoutSw128);
                        const uint64_t db = tc::smem_desc(kt + off, 16, 1024, tc::kLayoutSw128);
                        tc::mma_f16(tmem + C::S_COL + sb * C::BN, da, db, IDESC_QK, k > 0);
                    }
                    tc::commit(smem_addr(&ctrl->sfull[sb]));
                    tc::commit(smem_addr(&ctrl->empty[e]));
                    if (j == x.steps - 1) tc::commit(smem_addr(&ctrl->qempty));
                }
                __syncwarp();
            }
            ++uc;
        }
        if (!ok) fail();
        // Every product this warp issued has completed before tensor memory is freed.
        if (tc::elect_one()) tc::commit(smem_addr(&ctrl->drain[0]));
        __syncwarp();
        mbar_wait_warp(smem_addr(&ctrl->drain[0]), 0u, nullptr);
    }

    if (warp == C::WARP_PV) {
        // ------------------------------------------------------------ value products
        // Global step g: O += P_hi V(g) + P_lo V(g), A read from tensor memory
        // (the P that replaced S(g)), once the softmax warps have written P(g);
        // a unit's first step overwrites its O buffer after the epilogue has
        // read that buffer's previous unit.
        int64_t g = 0;
        int uc = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            PfUnit x;
            uint32_t fl;
            if (!pf_unit(a, u, x, &fl)) continue;
            const int ob = uc & 1;
            for (int j = 0; j < x.steps; ++j, ++g) {
                const int64_t vi = 2 * g + 1;
                const int e = static_cast<int>(vi % C::NS);
                if (!mbar_wait_warp(smem_addr(&ctrl->pfull), static_cast<uint32_t>(g) & 1u, abort_flag) ||
                    (j == 0 && !mbar_wait_warp(smem_addr(&ctrl->ofree[ob]),
                                               (static_cast<uint32_t>(uc >> 1) & 1u) ^ 1u, abort_flag)) ||
                    !mbar_wait_warp(smem_addr(&ctrl->full[e]), static_cast<uint32_t>(vi / C::NS) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    const uint32_t vt = ring + e * C::TILE;
                    const int sb = static_cast<int>(g & 1);
#pragma unroll
                    for (int part = 0; part < 2; ++part)
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            // 16 keys = 8 packed columns of P; 16 value rows
                            const uint32_t pa = tmem + C::S_COL + sb * C::BN + part * 64 + 8 * k;
                            const uint64_t db = tc::smem_desc(vt + k * 2048, C::PANEL, 1024, tc::kLayoutSw128);
                            tc::mma_f16_ts(tmem + C::O_COL + ob * C::D, pa, db, IDESC_PV,
                                           !(j == 0 && part == 0 && k == 0));
                        }
                    tc::commit(smem_addr(&ctrl->empty[e]));
                    tc::commit(smem_addr(&ctrl->sfree[sb]));
                    tc::commit(smem_addr(&ctrl->pvdone));
                    if (j == x.steps - 1) tc::commit(smem_addr(&ctrl->ofull[ob]));
                }
                __syncwarp();
            }
            ++uc;
        }
        if (!ok) fail();
        if (tc::elect_one()) tc::commit(smem_addr(&ctrl->drain[1]));
        __syncwarp();
        mbar_wait_warp(smem_addr(&ctrl->drain[1]), 0u, nullptr);
    }

    if (warp >= C::WARP_SM0) {
        // ------------------------------------------------------------ softmax + epilogue
        // Two warps per tensor-memory sub-partition: warp half hf takes keys
        // 64 hf .. 64 hf + 63 of every step (and d columns 64 hf .. of O).  The
        // halves of a row share one reference, agreed each step from their
        // partial maxima.
        const int sp = warp & 3;                    // sub-partition of this warp
        const int hf = (warp - C::WARP_SM0) >> 2;   // key half
        const int r = 32 * sp + lane;               // tile row held by this thread (= TMEM lane)
        const float NEG_INF = -__int_as_float(0x7f800000);
        const uint64_t neg1 = pf_pack(-1.f, -1.f);
        const uint64_t sl2x2 = pf_pack(a.sl2, a.sl2);
        uint32_t xpar = 0;
        // Both halves post a per-row value and read the other's; bounded waits.
        // It also orders each half's tensor-memory reads of S before the other
        // half's writes of P over the same columns.
        auto exchange = [&](float mine, float& other) -> bool {
            if (!mbar_wait_warp(smem_addr(&ctrl->xfree[sp]), xpar ^ 1u, abort_flag)) return false;
            ctrl->xval[hf][r] = mine;
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->xfull[sp]));
            if (!mbar_wait_warp(smem_addr(&ctrl->xfull[sp]), xpar, abort_flag)) return false;
            tc::fence_after_sync();
            other = ctrl->xval[hf ^ 1][r];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->xfree[sp]));
            xpar ^= 1u;
            return true;
        };
        int64_t g = 0;
        int uc = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            PfUnit x;
            uint32_t fl;
            if (!pf_unit(a, u, x, &fl)) continue;
            const int ob = uc & 1;
            const int tq = r / a.R;        // token of the row within the tile
            const int hq = r - tq * a.R;   // query head of the row within the group
            const bool row_ok = tq < x.n_tok;
            const int pos = x.pos0 + tq;   // cache position of the row's token
            float ref = NEG_INF, l = 0.f;  // l: this half's share of the row sum
            for (int j = 0; j < x.steps; ++j, ++g) {
                const int sb = static_cast<int>(g & 1);
                if (!mbar_wait_warp(smem_addr(&ctrl->sfull[sb]), static_cast<uint32_t>(g >> 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                uint32_t sv[64];  // this half's raw scores, then its weights (fp32 bits)
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tc::tmem_ld32(tc::tmem_addr(tmem, 32 * sp, C::S_COL + sb * C::BN + 64 * hf + 32 * c), sv + 32 * c);
                tc::tmem_wait_ld();

                // Key 128 j + 64 hf + c is visible iff it is <= pos.
                const int lim = row_ok ? pos - C::BN * j - 64 * hf : -1;
                if (lim < 63) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c > lim) sv[c] = __float_as_uint(NEG_INF);
                }
                float m4[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
                for (int c = 0; c < 64; c += 2)
                    m4[(c >> 1) & 3] = pf_max3(m4[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
                float mo;
                const float mp = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                if (!exchange(mp, mo)) {
                    ok = false;
                    break;
                }
                // Base-2 row maximum (scale > 0 keeps the order); lazy reference:
                // weights stay <= 2^8 against it.
                const float mx = fmaxf(mp, mo) * a.sl2;
                float alpha = 1.f;
                const bool move = mx > ref + static_cast<float>(C::T_LAZY);
                if (move) {
                    alpha = ref == NEG_INF ? 0.f : fast_exp2(ref - mx);
                    ref = mx;
                    l *= alpha;
                }
                const float rb = ref == NEG_INF ? 0.f : ref;
                const uint64_t nrb = pf_pack(-rb, -rb);
                uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float2 t = pf_unpack(
                        pf_fma2(pf_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2x2, nrb));
                    const float p0 = fast_exp2(t.x), p1 = fast_exp2(t.y);
                    sv[2 * i] = __float_as_uint(p0);
                    sv[2 * i + 1] = __float_as_uint(p1);
                    acc[i & 3] = pf_add2(acc[i & 3], pf_pack(p0, p1));
                }
                {
                    const float2 s2 = pf_unpack(pf_add2(pf_add2(acc[0], acc[1]), pf_add2(acc[2], acc[3])));
                    l += s2.x + s2.y;
                }

                if (j > 0 && __any_sync(0xffffffffu, move)) {
                    // O holds this unit's earlier steps: once the previous step's value
                    // product is done, rescale the moved rows in place (this half's d
                    // columns).
                    if (!mbar_wait_warp(smem_addr(&ctrl->pvdone), static_cast<uint32_t>(g - 1) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t o[32];
                        const uint32_t oa = tc::tmem_addr(tmem, 32 * sp, C::O_COL + ob * C::D + 64 * hf + 32 * c);
                        tc::tmem_ld32(oa, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tc::tmem_st32(oa, o);
                    }
                    tc::tmem_wait_st();
                }
                // Value rows at or past L_b may hold anything, and 0 * NaN would poison O.
                if (C::BN * (j + 1) > x.L) {
                    const int64_t vi = 2 * g + 1;
                    const int e = static_cast<int>(vi % C::NS);
                    if (!mbar_wait_warp(smem_addr(&ctrl->full[e]), static_cast<uint32_t>(vi / C::NS) & 1u,
                                        abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (C::BN * j + r >= x.L) {
                        const uint32_t vrow = ring + e * C::TILE + hf * C::PANEL + r * 128;
#pragma unroll
                        for (int c = 0; c < 8; ++c) st_shared_v4(vrow + ((c ^ (r & 7)) << 4), 0u, 0u, 0u, 0u);
                    }
                    pf_fence_async_smem();
                }
                // P = hi + lo (bf16 pairs) over S's own columns: hi of keys
                // 64 hf .. at columns 32 hf .., lo at 64 + 32 hf .. (both halves have
                // read their scores: the exchange above orders it).
                {
                    uint32_t hi[32], lo[32];
#pragma unroll
                    for (int w = 0; w < 32; ++w)
                        pf_split(__uint_as_float(sv[2 * w]), __uint_as_float(sv[2 * w + 1]), neg1, hi[w], lo[w]);
                    const uint32_t pcol = C::S_COL + sb * C::BN + 32 * hf;
                    tc::tmem_st32(tc::tmem_addr(tmem, 32 * sp, pcol), hi);
                    tc::tmem_st32(tc::tmem_addr(tmem, 32 * sp, pcol + 64), lo);
                    tc::tmem_wait_st();
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->pfull));
            }
            if (!ok) break;

            // ---------------------------------------------------- unit end: O / l -> out
            float lo_half;
            if (!exchange(l, lo_half) ||
                !mbar_wait_warp(smem_addr(&ctrl->ofull[ob]), static_cast<uint32_t>(uc >> 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const float lt = l + lo_half;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const int64_t orow =
                row_ok ? (static_cast<int64_t>(x.q_row0 + tq) * a.H_Q + x.kv * a.R + hq) * C::D + 64 * hf : 0;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tc::tmem_addr(tmem, 32 * sp, C::O_COL + ob * C::D + 64 * hf + 32 * c), o);
                tc::tmem_wait_ld();
                if (row_ok) {
                    if constexpr (OUT_BF16) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow + 32 * c);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint32_t wv[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[8 * q4 + 2 * e]) * inv,
                                                                                __uint_as_float(o[8 * q4 + 2 * e + 1]) * inv);
                                wv[e] = *reinterpret_cast<const uint32_t*>(&h2);
                            }
                            dst[q4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + 32 * c);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            dst[q4] = make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                                  __uint_as_float(o[4 * q4 + 2]) * inv,
                                                  __uint_as_float(o[4 * q4 + 3]) * inv);
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->ofree[ob]));
            ++uc;
        }
        if (!ok) fail();
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

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
// Query tile: TQ = floor(128 / R) consecutive query tokens of one sequence
// and one KV head kv, as one M = 128 row tile whose row r is token r / R and
// query head kv R + r % R, so every K/V row brought on chip serves all R
// heads of the group.  Work unit: two consecutive query tiles (tile 0 and
// tile 1, 2 TQ tokens) that share every K/V step, so each staged K/V row
// serves 256 rows and one tile's softmax runs while the tensor cores work on
// the other tile.  The unit walks its visible keys 128 at a time:
//   S_t = Q_t K^T   tcgen05.mma, M = 128 rows, N = 128 keys, K = d: A = the
//                   query rows, B = the key rows, both K-major with the
//                   128-byte swizzle as TMA stages them; S_t in tensor memory.
//   softmax         four warps per tile, one per tensor-memory sub-partition:
//                   thread = row = TMEM lane, all 128 keys of the step in
//                   registers, so the row maximum needs no exchange.  Base-2
//                   online softmax against a per-row reference that moves
//                   only when a score exceeds it by more than 8 (O_t is
//                   rescaled in tensor memory then).  P replaces S_t in its
//                   own columns as bf16 hi and lo parts: keys 32c .. 32c+31
//                   go to columns 32c .. 32c+15 (hi, two keys per column) and
//                   32c+16 .. 32c+31 (lo), both truncated, so the product
//                   keeps ~15 bits of every weight.
//   O_t += P V      tcgen05.mma, M = 128, N = d = 128, K = 128 keys, once on
//                   the hi part and once on the lo part; A = P read from
//                   tensor memory, B = the value rows read MN-major; O_t in
//                   tensor memory, normalised by the row sum at the unit end.
//
// One thread issues every product, per step i in the order
//   S_0(i), O_1 += P_1(i-1) V(i-1), S_1(i), O_0 += P_0(i) V(i)
// so each tile's softmax is covered by two products of the other tile.  The
// score product that overwrites S_t columns still holding P_t of the step
// before is issued after the value product that reads them: tcgen05.mma
// operations of one thread execute in issue order.
//
// Persistent CTAs (one per SM) walk the units in a fixed interleaved order,
// heaviest first.  Warp roles: 0 TMA producer, 1 tensor-core issue
// (+ tensor-memory allocation), 2..3 idle, 4..7 softmax and epilogue of
// tile 0, 8..11 of tile 1 (warp w on sub-partition w % 4).  Every wait is bounded
// (kWaitTimeoutNs); on a timeout the CTA raises GQA_FLAG_TIMEOUT, lets its
// copies and products drain, frees its tensor memory and returns.
#pragma once

#include <cuda_bf16.h>

#include <utility>

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
    int QT;          // units (tile pairs) per sequence: ceil(max_q / (2 TQ))
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
    static constexpr int NS = 5;                   // K/V ring entries (K and V of a step alternate)
    static constexpr int OFF_Q = 0;                // query tile t at OFF_Q + t TILE
    static constexpr int OFF_RING = OFF_Q + 2 * TILE;
    static constexpr int OFF_CTRL = OFF_RING + NS * TILE;
    static constexpr int CTRL_BYTES = 2048;
    static constexpr int SMEM_BYTES = 1024 + OFF_CTRL + CTRL_BYTES;  // + 1024-byte alignment slack
    static constexpr int S_COL = 0;                // S_t at S_COL + 128 t; P_t hi | lo replaces it
    static constexpr int O_COL = 256;              // O_t at O_COL + 128 t
    static constexpr int TMEM_COLS = 512;
    // Three warpgroups: 0 = TMA producer, tensor-core issue and two idle warps;
    // 1 and 2 = softmax of tile 0 and tile 1.  Registers move from group 0 to
    // the softmax groups (setmaxnreg): 128 x REG_LOW + 256 x REG_HIGH must not
    // exceed the 384 x 168 the block is launched with.
    static constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_SM0 = 4;
    static constexpr int NSM = 8;                  // softmax warps: four per tile
    static constexpr int THREADS = 32 * (WARP_SM0 + NSM);
    static constexpr int REG_LAUNCH = 168, REG_LOW = 88, REG_HIGH = 208;
    static constexpr int T_LAZY = 8;               // reference slack, base 2
};

struct __align__(16) PfControl {
    uint64_t full[PfCfg::NS], empty[PfCfg::NS];  // K/V ring
    uint64_t qfull, qempty;                      // the unit's two query tiles
    uint64_t sfull[2];                           // S_t of a step written
    uint64_t pfull[2];                           // P_t of a step written (four softmax warps)
    uint64_t ofull[2], ofree[2];                 // O_t of a unit complete / read by the epilogue
    uint64_t drain;                              // every issued product complete
    uint32_t tmem_base;
    int abort;
};

// One work unit (a pair of query tiles) as every warp role derives it from
// the unit index.
struct PfUnit {
    int b, kv, qt;
    int n_tok;   // query tokens in the pair (tokens past it in a tile are idle rows)
    int q_row0;  // row of q / out of the pair's first token
    int pos0;    // cache position of the pair's first token
    int L;       // clamped cache length
    int steps;   // 128-key steps: keys [0, pos0 + n_tok) are visible to some row
};

// Unit u: pair qt = QT - 1 - u / (B H_KV) (heaviest first), then sequence b,
// then KV head.  Returns false for a unit with no rows; *flags gets the status
// bits the sequence's bounds raise (a clamped length, an inconsistent query
// span -- such a sequence is skipped).
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
    const int tok0 = x.qt * 2 * a.TQ;
    if (tok0 >= n) return false;
    x.n_tok = min(2 * a.TQ, n - tok0);
    x.q_row0 = c0 + tok0;
    x.pos0 = x.L - n + tok0;
    x.steps = (x.pos0 + x.n_tok + PfCfg::BN - 1) / PfCfg::BN;
    return true;
}

// The unit a CTA takes in its k-th round, or -1 when it has none left.
// Round k covers units [k G, k G + G) of the heaviest-first order
// (G = gridDim.x); even rounds hand them to the CTAs left to right and odd
// rounds right to left, so the per-CTA sums even out over each pair of rounds
// although unit costs fall steadily along the order (a fixed cyclic order
// leaves the first CTAs 6-13% more work than the average).  Only the last
// round can be short, so a CTA with no unit in round k has none after it, and
// the round of a unit u is u / G.
__device__ __forceinline__ int pf_order(int k, int n_units) {
    const int G = static_cast<int>(gridDim.x);
    const int i = (k & 1) ? G - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
    const int64_t u = static_cast<int64_t>(k) * G + i;
    return u < n_units ? static_cast<int>(u) : -1;
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

// p0, p1 -> bf16 hi parts and bf16 lo parts, both by truncation: hi = the
// top 16 bits of each fp32, lo = the top 16 bits of the exact remainder
// p - hi, so hi + lo is within 2^-14 of each weight.  Bit operations only: a
// float-to-bf16 conversion would use the unit that also computes the
// exponentials.  p0 lands in the low half of each packed word.
__device__ __forceinline__ void pf_split(float p0, float p1, uint64_t neg1, uint32_t& hi, uint32_t& lo) {
    const uint32_t a = __float_as_uint(p0), b = __float_as_uint(p1);
    hi = __byte_perm(a, b, 0x7632);
    const uint64_t rem = pf_fma2(pf_pack(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u)), neg1,
                                 pf_pack(p0, p1));
    const float2 r = pf_unpack(rem);
    lo = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
}

// S = Q K^T as 8 products of K = 16 (two 64-column panels of d, four 32-byte
// slices each), offsets fixed at compile time.
template <int... K>
__device__ __forceinline__ void pf_issue_qk(uint32_t d, uint64_t da, uint64_t db, std::integer_sequence<int, K...>) {
    constexpr uint32_t IDESC = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 0, 0, 128, PfCfg::BN);
    (tc::mma_f16_off<static_cast<uint32_t>(((K >> 2) * PfCfg::PANEL + 32 * (K & 3)) >> 4)>(d, da, db, IDESC, K > 0),
     ...);
}

// O += P_hi V + P_lo V as 16 products of K = 16 keys: product i is part i / 8
// (hi, lo) of keys 16 (i % 8) .. +15 -- P columns 32 (k / 2) + 16 part +
// 8 (k % 2) -- against value rows 16 k .. +15 (2048 bytes each).
template <int... I>
__device__ __forceinline__ void pf_issue_pv(uint32_t d, uint32_t pa, uint64_t db, bool fresh,
                                            std::integer_sequence<int, I...>) {
    constexpr uint32_t IDESC = tc::instr_desc(tc::kFmtBF16, tc::kFmtBF16, 0, 1, 128, PfCfg::D);
    (tc::mma_f16_ts_off<static_cast<uint32_t>(32 * ((I & 7) >> 1) + 16 * (I >> 3) + 8 * (I & 1)),
                        static_cast<uint32_t>((I & 7) * 128)>(d, pa, db, IDESC, I > 0 || !fresh),
     ...);
}

// Warpgroup-wide register budget changes (every warp of the warpgroup executes them).
template <int N>
__device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

template <bool PAGED, bool OUT_BF16>
__global__ void __launch_bounds__(PfCfg::THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillArgs a) {
    using C = PfCfg;
    static_assert(sizeof(PfControl) <= C::CTRL_BYTES, "control block overflows its slot");
    static_assert(128 * C::REG_LOW + 256 * C::REG_HIGH <= C::THREADS * C::REG_LAUNCH,
                  "the register split must fit the registers the block is launched with");

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
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_addr(&ctrl->sfull[t]), 1);
            mbar_init(smem_addr(&ctrl->pfull[t]), 4);
            mbar_init(smem_addr(&ctrl->ofull[t]), 1);
            mbar_init(smem_addr(&ctrl->ofree[t]), 4);
        }
        mbar_init(smem_addr(&ctrl->drain), 1);
        ctrl->abort = 0;
    }
    // Query rows the TMA boxes leave out (R * TQ < 128) stay zero.
    for (int i = threadIdx.x; i < 2 * C::TILE / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base_ptr + C::OFF_Q)[i] = make_uint4(0, 0, 0, 0);
    if (warp == C::WARP_MMA) {
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

    if (warp < C::WARP_SM0) {
    reg_dealloc<C::REG_LOW>();
    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------------ producer
        // K/V rows are read again by the sequence's other units: keep them in L2.
        const uint64_t pol_kv = policy_evict_last();
        const uint64_t pol_q = policy_evict_first();
        uint32_t ld = 0;  // K/V loads issued: K of step g is load 2g, V is 2g + 1 (a CTA runs < 2^31 steps)
        int uc = 0;      // units issued
        bool ok = true;
        for (int u = pf_order(0, n_units); u >= 0 && ok; u = pf_order(u / gridDim.x + 1, n_units)) {
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
                // Both tiles: TQ tokens x R heads each; a box reaching past total_q reads zeros.
                const uint32_t bar = smem_addr(&ctrl->qfull);
                mbar_arrive_expect_tx(bar, 2u * 2u * 128u * static_cast<uint32_t>(a.R * a.TQ));
                for (int t = 0; t < 2; ++t)
                    for (int p = 0; p < 2; ++p)
                        tma_load_3d(q_smem + t * C::TILE + p * C::PANEL, &tmQ, bar, 64 * p, x.kv * a.R,
                                    x.q_row0 + t * a.TQ, pol_q);
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
            const uint32_t first = ld > C::NS ? ld - C::NS : 0;
            for (uint32_t i = first; i < ld; ++i)
                mbar_wait(smem_addr(&ctrl->full[i % C::NS]), static_cast<uint32_t>((i / C::NS) & 1), nullptr);
            if (uc > 0) mbar_wait(smem_addr(&ctrl->qfull), static_cast<uint32_t>(uc - 1) & 1u, nullptr);
        }
    }

    if (warp == C::WARP_MMA) {
        // ------------------------------------------------------------ tensor-core issue
        // Global step g of this CTA: K(g) is ring load 2g, V(g) load 2g + 1.
        auto stage = [&](uint32_t li) { return ring + (li % C::NS) * C::TILE; };
        auto loaded = [&](uint32_t li) {
            return mbar_wait_warp(smem_addr(&ctrl->full[li % C::NS]), static_cast<uint32_t>((li / C::NS) & 1),
                                  abort_flag);
        };
        // S_t = Q_t K^T (8 products of K = 16).  Descriptor start addresses are
        // advanced by adding (offset >> 4) to the descriptor: every operand lies
        // below 256 KB, so the 14-bit address field never carries.  The issue
        // sequences are straight-line code with compile-time offsets: one thread
        // issues every product of the CTA, and run-time address arithmetic per
        // product would make the issue itself the bottleneck.
        auto issue_qk = [&](int t, uint32_t kt) {
            pf_issue_qk(tmem + C::S_COL + 128 * t, tc::smem_desc(q_smem + t * C::TILE, 16, 1024, tc::kLayoutSw128),
                        tc::smem_desc(kt, 16, 1024, tc::kLayoutSw128), std::make_integer_sequence<int, 8>{});
        };
        // O_t += P_hi V + P_lo V; keys 32c .. 32c+31 have hi at columns 32c .. +15, lo at 32c+16 .. +31
        auto issue_pv = [&](int t, uint32_t vt, bool fresh) {
            pf_issue_pv(tmem + C::O_COL + 128 * t, tmem + C::S_COL + 128 * t,
                        tc::smem_desc(vt, C::PANEL, 1024, tc::kLayoutSw128), fresh,
                        std::make_integer_sequence<int, 16>{});
        };
        auto wait_p = [&](int t, uint32_t gs) {
            return mbar_wait_warp(smem_addr(&ctrl->pfull[t]), static_cast<uint32_t>(gs) & 1u, abort_flag);
        };
        auto wait_ofree = [&](int t, int uc) {
            return mbar_wait_warp(smem_addr(&ctrl->ofree[t]), (static_cast<uint32_t>(uc) & 1u) ^ 1u, abort_flag);
        };
        uint32_t g = 0;  // steps of this CTA so far (a CTA runs < 2^31 steps)
        int uc = 0;
        bool ok = true;
        for (int u = pf_order(0, n_units); u >= 0 && ok; u = pf_order(u / gridDim.x + 1, n_units)) {
            PfUnit x;
            uint32_t fl;
            if (!pf_unit(a, u, x, &fl)) continue;
            const int n = x.steps;
            if (!mbar_wait_warp(smem_addr(&ctrl->qfull), static_cast<uint32_t>(uc) & 1u, abort_flag) ||
                !loaded(2 * g)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            if (tc::elect_one()) {
                issue_qk(0, stage(2 * g));
                tc::commit(smem_addr(&ctrl->sfull[0]));
                issue_qk(1, stage(2 * g));
                tc::commit(smem_addr(&ctrl->sfull[1]));
                tc::commit(smem_addr(&ctrl->empty[(2 * g) % C::NS]));
                if (n == 1) tc::commit(smem_addr(&ctrl->qempty));
            }
            __syncwarp();
            if (!loaded(2 * g + 1) || !wait_ofree(0, uc) || !wait_p(0, g)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            if (tc::elect_one()) {
                issue_pv(0, stage(2 * g + 1), true);
                if (n == 1) tc::commit(smem_addr(&ctrl->ofull[0]));
            }
            __syncwarp();
            for (int i = 1; i < n; ++i) {
                const uint32_t gi = g + i;
                if (!loaded(2 * gi)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    issue_qk(0, stage(2 * gi));  // after the product that read P_0(gi - 1) from these columns
                    tc::commit(smem_addr(&ctrl->sfull[0]));
                }
                __syncwarp();
                if ((i == 1 && !wait_ofree(1, uc)) || !wait_p(1, gi - 1)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    issue_pv(1, stage(2 * gi - 1), i == 1);
                    tc::commit(smem_addr(&ctrl->empty[(2 * gi - 1) % C::NS]));
                    issue_qk(1, stage(2 * gi));
                    tc::commit(smem_addr(&ctrl->sfull[1]));
                    tc::commit(smem_addr(&ctrl->empty[(2 * gi) % C::NS]));
                    if (i == n - 1) tc::commit(smem_addr(&ctrl->qempty));
                }
                __syncwarp();
                if (!loaded(2 * gi + 1) || !wait_p(0, gi)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (tc::elect_one()) {
                    issue_pv(0, stage(2 * gi + 1), false);
                    if (i == n - 1) tc::commit(smem_addr(&ctrl->ofull[0]));
                }
                __syncwarp();
            }
            if (!ok) break;
            const uint32_t last = g + n - 1;
            if ((n == 1 && !wait_ofree(1, uc)) || !wait_p(1, last)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            if (tc::elect_one()) {
                issue_pv(1, stage(2 * last + 1), n == 1);
                tc::commit(smem_addr(&ctrl->empty[(2 * last + 1) % C::NS]));
                tc::commit(smem_addr(&ctrl->ofull[1]));
            }
            __syncwarp();
            g += n;
            ++uc;
        }
        if (!ok) fail();
        // Every product this warp issued has completed before tensor memory is freed.
        if (tc::elect_one()) tc::commit(smem_addr(&ctrl->drain));
        __syncwarp();
        mbar_wait_warp(smem_addr(&ctrl->drain), 0u, nullptr);
    }
    } else {
        reg_alloc<C::REG_HIGH>();
        // ------------------------------------------------------------ softmax + epilogue
        const int t = (warp - C::WARP_SM0) >> 2;   // query tile of this warp
        const int sp = warp & 3;                   // sub-partition of this warp
        const int r = 32 * sp + lane;              // tile row held by this thread (= TMEM lane)
        const uint32_t trow = tc::tmem_addr(tmem, 32 * sp, 0);
        const uint32_t s_col = C::S_COL + 128 * t, o_col = C::O_COL + 128 * t;
        const float NEG_INF = -__int_as_float(0x7f800000);
        const uint64_t neg1 = pf_pack(-1.f, -1.f);
        const uint64_t sl2x2 = pf_pack(a.sl2, a.sl2);
        uint32_t g = 0;
        int uc = 0;
        bool ok = true;
        for (int u = pf_order(0, n_units); u >= 0 && ok; u = pf_order(u / gridDim.x + 1, n_units)) {
            PfUnit x;
            uint32_t fl;
            if (!pf_unit(a, u, x, &fl)) continue;
            const int n_t = min(max(x.n_tok - t * a.TQ, 0), a.TQ);  // tokens of this tile
            const int tq = r / a.R;        // token of the row within the tile
            const int hq = r - tq * a.R;   // query head of the row within the group
            const bool row_ok = tq < n_t;
            const int pos = x.pos0 + t * a.TQ + tq;  // cache position of the row's token
            float ref = NEG_INF, l = 0.f;
            for (int j = 0; j < x.steps; ++j, ++g) {
                if (!mbar_wait_warp(smem_addr(&ctrl->sfull[t]), static_cast<uint32_t>(g) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                uint32_t sv[128];  // the row's raw scores, then its weights (fp32 bits)
#pragma unroll
                for (int c = 0; c < 4; ++c) tc::tmem_ld32(trow + s_col + 32 * c, sv + 32 * c);
                tc::tmem_wait_ld();

                // Key 128 j + c is visible iff it is <= pos.
                const int lim = row_ok ? pos - C::BN * j : -1;
                if (lim < 127) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > lim) sv[c] = __float_as_uint(NEG_INF);
                }
                float m4[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
                for (int c = 0; c < 128; c += 2)
                    m4[(c >> 1) & 3] = pf_max3(m4[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
                // Base-2 row maximum (scale > 0 keeps the order); lazy reference:
                // weights stay <= 2^8 against it.
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * a.sl2;
                float alpha = 1.f;
                const bool move = mx > ref + static_cast<float>(C::T_LAZY);
                if (move) {
                    alpha = ref == NEG_INF ? 0.f : fast_exp2(ref - mx);
                    ref = mx;
                    l *= alpha;
                }
                const float rb = ref == NEG_INF ? 0.f : ref;
                const uint64_t nrb = pf_pack(-rb, -rb);
                // Weights and P = hi + lo (bf16 pairs) over S_t's own columns, 32 keys
                // at a time, so a chunk's scores die as its P is stored.
                uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int w = 0; w < 16; ++w) {
                        const int k = 32 * c + 2 * w;
                        const float2 e2 =
                            pf_unpack(pf_fma2(pf_pack(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])), sl2x2, nrb));
                        const float p0 = fast_exp2(e2.x), p1 = fast_exp2(e2.y);
                        acc[w & 1] = pf_add2(acc[w & 1], pf_pack(p0, p1));
                        pf_split(p0, p1, neg1, hi[w], lo[w]);
                    }
                    tc::tmem_st16(trow + s_col + 32 * c, hi);
                    tc::tmem_st16(trow + s_col + 32 * c + 16, lo);
                }
                {
                    const float2 s2 = pf_unpack(pf_add2(acc[0], acc[1]));
                    l += s2.x + s2.y;
                }
                tc::tmem_wait_st();

                if (j > 0 && __any_sync(0xffffffffu, move)) {
                    // O_t holds this unit's earlier steps; the previous step's value
                    // product has completed (S_t of this step was committed after it):
                    // rescale the moved rows in place.
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tc::tmem_ld32(trow + o_col + 32 * c, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tc::tmem_st32(trow + o_col + 32 * c, o);
                    }
                    tc::tmem_wait_st();
                }
                // Value rows at or past L_b may hold anything, and 0 * NaN would poison O.
                // Tile 0's warps clear them (before P_0 of the step, which both value
                // products of the step follow).
                if (t == 0 && C::BN * (j + 1) > x.L) {
                    const uint32_t vi = 2 * g + 1;
                    const int e = static_cast<int>(vi % C::NS);
                    if (!mbar_wait_warp(smem_addr(&ctrl->full[e]), static_cast<uint32_t>(vi / C::NS) & 1u,
                                        abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (C::BN * j + r >= x.L) {
                        const uint32_t vrow = ring + e * C::TILE + r * 128;
#pragma unroll
                        for (int pnl = 0; pnl < 2; ++pnl)
#pragma unroll
                            for (int c = 0; c < 8; ++c) st_shared_v4(vrow + pnl * C::PANEL + 16 * c, 0u, 0u, 0u, 0u);
                    }
                    pf_fence_async_smem();
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->pfull[t]));
            }
            if (!ok) break;

            // ---------------------------------------------------- unit end: O_t / l -> out
            if (!mbar_wait_warp(smem_addr(&ctrl->ofull[t]), static_cast<uint32_t>(uc) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int64_t orow =
                row_ok ? (static_cast<int64_t>(x.q_row0 + t * a.TQ + tq) * a.H_Q + x.kv * a.R + hq) * C::D : 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(trow + o_col + 32 * c, o);
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
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->ofree[t]));
            ++uc;
        }
        if (!ok) fail();
    }

    // ---------------------------------------------------------------- teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace gqa

// split_mma.cuh -- bf16 split-KV decode kernel for sm_100a.
//
// Computes, for each segment of the tile schedule (schedule.cuh), the
// attention of the R query heads of one KV group over a run of that group's
// cached tokens ("Grouped-Query Attention (GQA) and Multi-Query Attention
// (MQA): Mathematical Foundations, ...", section 2: Head_i = softmax(Q_i
// K_{g(i)}^T / sqrt(d_k) + M) V_{g(i)}, with g(i) the contiguous group map).
// Each 64-token K/V tile is read from HBM once and serves all R heads.
//
// Persistent CTA, one per SM, warp-specialised:
//   * one producer warp streams 64-token K and V tiles (and each segment's
//     query rows) into a multi-stage shared-memory ring with TMA tensor
//     loads (128-byte swizzle, L2 evict-first for the cache), completing on
//     mbarriers.  Paged caches only change the tile coordinate: the page id
//     from the block table replaces (token, sequence).
//   * consumer warps: head group hg (ROWS = 8*NT query heads) x token group tg
//     (64/NTG tokens of each tile) x tile set (with 8 heads per warp, two
//     sets of four warps take alternate tiles so two dependency chains share
//     each SM sub-partition).  The contraction is laid out
//     token-major: per 16-token chunk a warp computes S^T = K Q^T with
//     mma.sync m16n8k16 (tokens on M, heads on N, so no rows are padding),
//     masks tokens >= L_b, updates an fp32 online softmax per head (column),
//     transposes P^T into B fragments with movmatrix, and accumulates
//     O^T += V^T P^T with P split into bf16 hi + lo parts so the weights keep
//     ~16 significant bits.
//   * at a segment end the token groups are merged in shared memory and the
//     segment writes either the final output or a partial (o / l, m + log2 l).
//
// Every wait is bounded (ptx.cuh); a timeout raises GQA_FLAG_TIMEOUT, lets
// in-flight copies land and returns.  Nothing traps.
#pragma once

#include "combine.cuh"
#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

// Largest base-2 growth of the running maximum absorbed without rescaling.
constexpr float kLazyRescale = 8.f;

template <int D, int NT, int HG, bool KV8 = false>
struct MmaCfg {
    static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
    static_assert(!KV8 || (D == 128 && NT == 1 && HG == 1), "8-bit caches: head_dim 128, <= 8 heads");
    static_assert(NT == 1 || NT == 2 || NT == 4, "8, 16 or 32 query heads per warp");
    static_assert(HG == 1 || HG == 2, "head groups: 1 or 2");
    static constexpr int ROWS = 8 * NT;                 // query heads per warp
    static constexpr int NTG = (NT == 4 && HG == 2) ? 2 : 4;  // token groups
    static constexpr bool Q_IN_REGS = NT <= 2 && NTG * HG == 4;  // else Q is re-read from smem
    static constexpr int TS = NT == 1 ? 2 : 1;          // tile sets taking alternate tiles
    static constexpr int TPW = kTile / NTG;             // tokens per warp per tile
    static constexpr int MGN = NTG * TS;                // partial softmax states per head group
    static constexpr int NC = NTG * HG * TS;            // consumer warps
    static constexpr int TILE_WARPS = NTG * HG;         // consumer warps reading one tile
    static constexpr int PRODUCER = NC;                 // index of the TMA warp
    static constexpr int MERGE = NC + 1;                // index of the merge warp (split partials)
    static constexpr int THREADS = 32 * (NC + 2);
    static constexpr int PANELS = D / 64;               // 128-byte-wide column panels
    static constexpr int PANEL_BYTES = kTile * 128;     // 64 tokens x 64 bf16
    // One stage: K and V tiles of 64 tokens, bf16 in 128-byte panels, or 8-bit
    // rows of D bytes (KV8).
    static constexpr int STAGE_BYTES = KV8 ? 2 * kTile * D : 2 * PANELS * PANEL_BYTES;
    static constexpr int QPANEL_BYTES = ROWS * 128;     // ROWS query rows x 64 bf16
    static constexpr int QSLOT_BYTES = HG * PANELS * QPANEL_BYTES;
    static constexpr int OROW = D + 4;                  // padded merge row (floats)
    static constexpr int MERGE_O_FLOATS = (MGN - 1) * HG * ROWS * OROW;
    static constexpr int MERGE_ML_FLOATS = (MGN - 1) * HG * ROWS * 2;
    static constexpr int MAX_STAGES = KV8 ? 12 : 8;
    static constexpr int CTRL_BYTES = 512;
    static constexpr int FIXED_BYTES =
        2 * QSLOT_BYTES + 4 * (MERGE_O_FLOATS + MERGE_ML_FLOATS) + CTRL_BYTES;
    static constexpr int smem_bytes(int stages) { return 1024 + stages * STAGE_BYTES + FIXED_BYTES; }
};

struct __align__(16) MmaControl {
    uint64_t full[MmaCfg<128, 1, 1, true>::MAX_STAGES];
    uint64_t empty[MmaCfg<128, 1, 1, true>::MAX_STAGES];
    uint64_t qfull[2];
    uint64_t qempty[2];
    uint64_t merge_full;
    uint64_t merge_free;
    uint64_t mjob[2];  // the CTA's first / last segment partial written (merge warp's jobs)
    uint64_t assist;   // the merge warp's ticket for the last segment is known
    int merge_last;    // ... and it was the unit's last: the consumers help merge
    Plan plan;
    int abort;
};
static_assert(sizeof(MmaControl) <= MmaCfg<128, 1, 1, false>::CTRL_BYTES, "control block overflows its slot");

// KV8: the cache holds OCP E4M3 bytes with per-KV-head scales.  TMA stages
// the 8-bit tiles as they are; consumers load them with ldmatrix (viewing
// byte pairs as b16), decode them in registers by bit placement to f16
// holding value * 2^-8 (exact) and run the same contraction on f16
// mma.sync, with 2^8 * k_scale folded into the score scale and 2^8 * v_scale
// into the output.  The byte order ldmatrix delivers permutes the head
// dimension inside each 16-value chunk (K side: Q is loaded with the same
// permutation, so dot products are unchanged; V side: the accumulator rows
// map to d = 16 m + 2 g + h, undone when the output is written).
template <int D, int NT, int HG, bool PAGED, bool OUT_BF16, bool KV8 = false>
__global__ void __launch_bounds__(MmaCfg<D, NT, HG, KV8>::THREADS, 1)
    split_mma_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const KernelArgs a) {
    using C = MmaCfg<D, NT, HG, KV8>;
    constexpr int KS = D / 16;  // k-steps over the head dimension; also 16-row blocks of d
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const int NS = a.n_stages;
    const uint32_t stages = base;
    const int ring_bytes = NS * C::STAGE_BYTES;
    const uint32_t qring = base + ring_bytes;
    float* merge_o = reinterpret_cast<float*>(base_ptr + ring_bytes + 2 * C::QSLOT_BYTES);
    float* merge_ml = merge_o + C::MERGE_O_FLOATS;
    MmaControl* ctrl = reinterpret_cast<MmaControl*>(merge_ml + C::MERGE_ML_FLOATS);
    volatile int* abort_flag = &ctrl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == C::PRODUCER && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_addr(&ctrl->full[s]), 1);
            mbar_init(smem_addr(&ctrl->empty[s]), C::TILE_WARPS);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&ctrl->qfull[s]), 1);
            mbar_init(smem_addr(&ctrl->qempty[s]), C::NC);
        }
        mbar_init(smem_addr(&ctrl->merge_full), (C::MGN - 1) * HG);
        mbar_init(smem_addr(&ctrl->merge_free), HG);
        for (int k = 0; k < 2; ++k) mbar_init(smem_addr(&ctrl->mjob[k]), HG);
        mbar_init(smem_addr(&ctrl->assist), 1);
        ctrl->abort = 0;
    }
    // Query rows a TMA box does not cover (R < ROWS) must read as zeros.
    for (int i = threadIdx.x; i < 2 * C::QSLOT_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base_ptr + ring_bytes)[i] = make_uint4(0, 0, 0, 0);

    grid_dependency_wait();
    grid_launch_dependents();
    if (warp == 0) make_plan(a, &ctrl->plan);
    fence_barrier_init();
    fence_proxy_async_smem();
    __syncthreads();

    if (warp == C::MERGE) {
        // ------------------------------------------------------------ merge warp
        if (!merge_warp<D, OUT_BF16>(a, ctrl->plan, ctrl->mjob, &ctrl->assist, &ctrl->merge_last, C::NC,
                                     abort_flag)) {
            *abort_flag = 1;
            if (lane == 0) atomicOr(a.status, kFlagTimeout);
        }
        return;
    }
    const int64_t lo = ctrl->plan.lo;
    const int64_t hi = ctrl->plan.hi;
    if (lo >= hi) return;
    Walk w{ctrl->plan.b, ctrl->plan.kv, ctrl->plan.tile, ctrl->plan.n_b, ctrl->plan.L};

    if (warp == C::PRODUCER) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        const uint32_t q_bytes = static_cast<uint32_t>(a.q_groups * C::PANELS * a.q_rows * 128);
        int st = 0, qs = 0;
        uint32_t ph = 0, qph = 0;
        int64_t issued = 0, q_issued = 0;
        int page_word = 0, page_base = -1;
        bool ok = true;
        const int RN = NS;
        uint64_t* rfull = ctrl->full;
        uint64_t* rempty = ctrl->empty;
        for (int64_t gi = lo; gi < hi; ++gi) {
            const bool seg_first = (gi == lo) || (w.tile == 0);
            if (seg_first) {
                if (!mbar_wait_warp(smem_addr(&ctrl->qempty[qs]), qph ^ 1u, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    const uint32_t bar = smem_addr(&ctrl->qfull[qs]);
                    mbar_arrive_expect_tx(bar, q_bytes);
                    for (int g = 0; g < a.q_groups; ++g)
                        for (int p = 0; p < C::PANELS; ++p)
                            tma_load_3d(qring + qs * C::QSLOT_BYTES + (g * C::PANELS + p) * C::QPANEL_BYTES,
                                        &tmQ, bar, 64 * p, w.kv * a.R + C::ROWS * g, w.b, pol_q);
                }
                ++q_issued;
                if (++qs == 2) { qs = 0; qph ^= 1u; }
            }
            int c2, c3;
            if constexpr (PAGED) {
                const int tb = w.tile & ~31;
                if (seg_first || tb != page_base) {
                    page_base = tb;
                    const int idx = tb + lane;
                    page_word = idx < w.n_b
                                    ? __ldg(a.block_table + static_cast<int64_t>(w.b) * a.max_blocks + idx)
                                    : 0;
                }
                const int page = __shfl_sync(0xffffffffu, page_word, w.tile & 31);
                if ((page < 0 || page >= a.num_blocks) && lane == 0) atomicOr(a.status, kFlagBadBlock);
                c2 = 0;
                c3 = page;  // out of range: the TMA unit fills the tile with zeros
            } else {
                c2 = w.tile * kTile;
                c3 = w.b;
            }
            if (!mbar_wait_warp(smem_addr(&rempty[st]), ph ^ 1u, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                const uint32_t bar = smem_addr(&rfull[st]);
                if constexpr (KV8) {
                    const uint32_t kb = stages + st * C::STAGE_BYTES;  // K then V: 64 rows x D bytes each
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    tma_load_4d(kb, &tmK, bar, 0, w.kv, c2, c3, pol_kv);
                    tma_load_4d(kb + kTile * D, &tmV, bar, 0, w.kv, c2, c3, pol_kv);
                } else {
                    const uint32_t kb = stages + st * C::STAGE_BYTES;
                    const uint32_t vb = kb + C::PANELS * C::PANEL_BYTES;
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    for (int p = 0; p < C::PANELS; ++p) {
                        tma_load_4d(kb + p * C::PANEL_BYTES, &tmK, bar, 64 * p, w.kv, c2, c3, pol_kv);
                        tma_load_4d(vb + p * C::PANEL_BYTES, &tmV, bar, 64 * p, w.kv, c2, c3, pol_kv);
                    }
                }
            }
            ++issued;
            if (++st == RN) { st = 0; ph ^= 1u; }
            if (gi + 1 < hi) w.advance(a);
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) atomicOr(a.status, kFlagTimeout);
            // Let copies already in flight land before the CTA's shared memory goes away.
            const int64_t first = issued > RN ? issued - RN : 0;
            for (int64_t i = first; i < issued; ++i)
                mbar_wait(smem_addr(&rfull[i % RN]), static_cast<uint32_t>((i / RN) & 1), nullptr);
            const int64_t qfirst = q_issued > 2 ? q_issued - 2 : 0;
            for (int64_t i = qfirst; i < q_issued; ++i)
                mbar_wait(smem_addr(&ctrl->qfull[i % 2]), static_cast<uint32_t>((i / 2) & 1), nullptr);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Fragment ownership (g = lane / 4, t = lane % 4):
    //   S^T, P:  token n0 + g (+8)      x head 8 nt + 2t (+1)
    //   O^T:     d 16 mm + g (+8)       x head 8 nt + 2t (+1)
    const int tset = warp / (C::NTG * HG);          // which alternate tiles this warp takes
    const int hg = (warp / C::NTG) % HG;
    const int tg = warp % C::NTG;
    const int mg = tset * C::NTG + tg;              // partial-state index; 0 merges
    const int g = lane >> 2;
    const int t = lane & 3;
    const float NEG_INF = -__int_as_float(0x7f800000);

    int st = 0, qs = 0;
    uint32_t ph = 0, qph = 0, mfull_ph = 0, mfree_ph = 0;
    bool first_seg = true;
    int seg_start_tile = 0;
    bool tail_cut = false;  // the CTA's last segment so far was cut (its unit is merged)
    int tail_b = 0, tail_kv = 0, tail_nb = 0;
    int64_t tail_su = 0;
    uint32_t qb[C::Q_IN_REGS ? KS : 1][NT][2];  // B fragments of Q^T (k-step, 8-head tile)
    int seg_q = 0;                                  // Q-ring slot of the current segment
    float o[KS][NT][4];      // O^T accumulators, per 16-row block of d and 8-head tile
    float m[NT][2], l[NT][2];
    float seg_sl2 = a.sl2, seg_vs = 1.f;  // score scale (x k_scale) and value scale of the segment's KV head

    auto fail = [&]() {
        *abort_flag = 1;
        if (lane == 0) atomicOr(a.status, kFlagTimeout);
    };

    for (int64_t gi = lo; gi < hi; ++gi) {
        const bool seg_first = (gi == lo) || (w.tile == 0);
        const bool last_tile = (w.tile == w.n_b - 1);
        const bool seg_last = (gi == hi - 1) || last_tile;
        if (seg_first) {
            seg_start_tile = w.tile;
            if (!mbar_wait_warp(smem_addr(&ctrl->qfull[qs]), qph, abort_flag)) { fail(); break; }
            seg_q = qs;
            const uint32_t qbase = qring + qs * C::QSLOT_BYTES + hg * C::PANELS * C::QPANEL_BYTES;
            if constexpr (!C::Q_IN_REGS) {
                // read per chunk from the ring slot; released at the segment end
            } else if constexpr (KV8) {
                // Head g, d = 16 ks + 4t + {0, 2} -> k-slots (2t, 2t+1) and d = 16 ks + 4t + {1, 3}
                // -> k-slots (2t+8, 2t+9), as f16: the order the K decode below produces.
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int p = ks >> 2, ch = ((ks & 3) << 1) + (t >> 1);
                    const uint2 w2 = ld_shared_v2(qbase + p * C::QPANEL_BYTES + g * 128 + ((ch ^ (g & 7)) << 4) +
                                                  ((t & 1) << 3));
                    qb[ks][0][0] = bf16x2_to_f16x2(__byte_perm(w2.x, w2.y, 0x5410));
                    qb[ks][0][1] = bf16x2_to_f16x2(__byte_perm(w2.x, w2.y, 0x7632));
                }
            } else if constexpr (NT == 2) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int p = ks >> 2, c0 = (ks & 3) << 1;
                    const int row = (lane & 7) + ((lane >> 4) << 3);
                    const int ch = c0 + ((lane >> 3) & 1);
                    ldsm_x4(qbase + p * C::QPANEL_BYTES + row * 128 + ((ch ^ (row & 7)) << 4), qb[ks][0][0],
                            qb[ks][0][1], qb[ks][1][0], qb[ks][1][1]);
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < KS; ks += 2) {
                    const int kk = ks + (lane >> 4);
                    const int p = kk >> 2, ch = ((kk & 3) << 1) + ((lane >> 3) & 1);
                    const int row = lane & 7;
                    ldsm_x4(qbase + p * C::QPANEL_BYTES + row * 128 + ((ch ^ row) << 4), qb[ks][0][0],
                            qb[ks][0][1], qb[ks + 1][0][0], qb[ks + 1][0][1]);
                }
            }
            if constexpr (C::Q_IN_REGS) {
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->qempty[qs]));
            }
            if constexpr (KV8) {  // the decode yields e4m3 * 2^-8: fold 2^8 back in
                seg_sl2 = a.sl2 * (256.f * __ldg(a.k_scale + w.kv));
                seg_vs = 256.f * __ldg(a.v_scale + w.kv);
            }
            if (++qs == 2) { qs = 0; qph ^= 1u; }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                m[nt][0] = m[nt][1] = NEG_INF;
                l[nt][0] = l[nt][1] = 0.f;
            }
#pragma unroll
            for (int mm = 0; mm < KS; ++mm)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) o[mm][nt][0] = o[mm][nt][1] = o[mm][nt][2] = o[mm][nt][3] = 0.f;
        }

        const bool mine = C::TS == 1 || ((gi - lo) % C::TS) == tset;  // tiles alternate between tile sets
        if (mine) {
        if (!mbar_wait_warp(smem_addr(&ctrl->full[st]), ph, abort_flag)) { fail(); break; }
        const uint32_t kb = stages + st * C::STAGE_BYTES;
        const uint32_t vb = kb + (KV8 ? kTile * D : C::PANELS * C::PANEL_BYTES);
        const int t0 = w.tile * kTile;

#pragma unroll
        for (int c = 0; c < C::TPW / 16; ++c) {
            const int n0 = tg * C::TPW + c * 16;
            if (last_tile && t0 + n0 >= w.L) break;  // no live token in this chunk
            const bool mask = last_tile && (t0 + n0 + 16 > w.L);

            // S^T = K Q^T: 16 tokens x ROWS heads.  k-steps rotate over NSET
            // accumulator sets so independent mma chains interleave.
            constexpr int NSET = NT == 1 ? 4 : (NT == 2 ? 2 : 1);
            float sa[NSET][NT][4];
#pragma unroll
            for (int q = 0; q < NSET; ++q)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) sa[q][nt][0] = sa[q][nt][1] = sa[q][nt][2] = sa[q][nt][3] = 0.f;
            const int krow = n0 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int ks = 0; ks < KS; ks += 2) {
                uint32_t ka[2][4];
                if constexpr (KV8) {
                    // 8-bit K rows: byte pairs as b16; chunks ks and ks+1 for 16 tokens.  Each
                    // word holds d = 4t .. 4t+3 of one token; the decode pairs (4t, 4t+2) and
                    // (4t+1, 4t+3).
                    uint32_t r0, r1, r2, r3;
                    const int ch = ks + (lane >> 4);
                    ldsm_x4(kb + krow * D + ((ch ^ (lane & 7)) << 4), r0, r1, r2, r3);
                    e4m3x4_to_f16x2_scaled(r0, ka[0][0], ka[0][2]);
                    e4m3x4_to_f16x2_scaled(r1, ka[0][1], ka[0][3]);
                    e4m3x4_to_f16x2_scaled(r2, ka[1][0], ka[1][2]);
                    e4m3x4_to_f16x2_scaled(r3, ka[1][1], ka[1][3]);
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int p = (ks + h) >> 2, ch = (((ks + h) & 3) << 1) + (lane >> 4);
                        ldsm_x4(kb + p * C::PANEL_BYTES + krow * 128 + ((ch ^ (lane & 7)) << 4), ka[h][0],
                                ka[h][1], ka[h][2], ka[h][3]);
                    }
                }
                if constexpr (C::Q_IN_REGS) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_16816<KV8>(sa[(ks + h) % NSET][nt], ka[h], qb[ks + h][nt][0], qb[ks + h][nt][1]);
                } else {
                    const uint32_t qbase = qring + seg_q * C::QSLOT_BYTES + hg * C::PANELS * C::QPANEL_BYTES;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kk = ks + h;
                        const int p = kk >> 2, ch = ((kk & 3) << 1) + ((lane >> 3) & 1);
                        uint32_t qf[NT][2];
#pragma unroll
                        for (int np = 0; np < NT / 2; ++np) {
                            const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                            ldsm_x4(qbase + p * C::QPANEL_BYTES + row * 128 + ((ch ^ (row & 7)) << 4),
                                    qf[2 * np][0], qf[2 * np][1], qf[2 * np + 1][0], qf[2 * np + 1][1]);
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_16816<KV8>(sa[kk % NSET][nt], ka[h], qf[nt][0], qf[nt][1]);
                    }
                }
            }
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float x = sa[0][nt][i];
#pragma unroll
                    for (int q = 1; q < NSET; ++q) x += sa[q][nt][i];
                    s[nt][i] = x * seg_sl2;
                }
            uint32_t vmask_a = 0xffffffffu, vmask_b = 0xffffffffu;
            if (mask) {
                const bool live0 = t0 + n0 + g < w.L, live1 = t0 + n0 + g + 8 < w.L;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (!live0) s[nt][0] = s[nt][1] = NEG_INF;
                    if (!live1) s[nt][2] = s[nt][3] = NEG_INF;
                }
                const int ta = t0 + n0 + 2 * t;
                vmask_a = (ta < w.L ? 0x0000ffffu : 0u) | (ta + 1 < w.L ? 0xffff0000u : 0u);
                vmask_b = (ta + 8 < w.L ? 0x0000ffffu : 0u) | (ta + 9 < w.L ? 0xffff0000u : 0u);
            }

            // Online softmax per head column: reduce over the 8 lanes that share
            // t.  The reference m moves only when the chunk maximum exceeds it
            // by more than kLazyRescale (base 2), so weights stay <= 2^8 and
            // the accumulator is rarely rescaled; o / l is unchanged by the
            // choice of reference.
            float p[NT][4], alpha[NT][2];
            bool rescale = false;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float mx = fmaxf(s[nt][j], s[nt][j + 2]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    alpha[nt][j] = 1.f;
                    if (mx > m[nt][j] + kLazyRescale) {  // also the first live chunk (m = -inf)
                        alpha[nt][j] = fast_exp2(m[nt][j] - mx);
                        m[nt][j] = mx;
                        rescale = true;
                    }
                    const float ref = m[nt][j] == NEG_INF ? 0.f : m[nt][j];
                    p[nt][j] = fast_exp2(s[nt][j] - ref);
                    p[nt][j + 2] = fast_exp2(s[nt][j + 2] - ref);
                    l[nt][j] = l[nt][j] * alpha[nt][j] + (p[nt][j] + p[nt][j + 2]);
                }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int mm = 0; mm < KS; ++mm)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        o[mm][nt][0] *= alpha[nt][0];
                        o[mm][nt][1] *= alpha[nt][1];
                        o[mm][nt][2] *= alpha[nt][0];
                        o[mm][nt][3] *= alpha[nt][1];
                    }
            }
            // P^T as B fragments (tokens x heads), hi and lo bf16 parts.
            uint32_t pbh[NT][2], pbl[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                uint32_t h0, l0, h1, l1;
                split_x2<KV8>(p[nt][0], p[nt][1], h0, l0);  // token g:     heads 2t, 2t+1
                split_x2<KV8>(p[nt][2], p[nt][3], h1, l1);  // token g + 8: heads 2t, 2t+1
                pbh[nt][0] = movmatrix_trans(h0);
                pbh[nt][1] = movmatrix_trans(h1);
                pbl[nt][0] = movmatrix_trans(l0);
                pbl[nt][1] = movmatrix_trans(l1);
            }

            // O^T += V^T P^T.  Hi products of a group of accumulators issue
            // before the lo products that depend on them.
            constexpr int MG = 4 / NT;  // 16-row blocks of d per group
            const int vrow = n0 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int m0 = 0; m0 < KS; m0 += MG) {
                uint32_t va[MG][4];
#pragma unroll
                for (int h = 0; h < MG; ++h) {
                    const int mm = m0 + h;
                    if constexpr (KV8) {
                        // 8-bit V rows: one transposing load gives tokens (2t, 2t+1) of d = 16 mm + 2g
                        // (bytes 0, 2) and of d = 16 mm + 2g + 1 (bytes 1, 3), for token halves 0-7 and
                        // 8-15 of chunks mm and mm + 1; block mm's accumulator rows are d = 16 mm + 2g + {0,1}.
                        if ((h & 1) == 0) {
                            uint32_t r0, r1, r2, r3;
                            ldsm_x4_trans(vb + krow * D + (((mm + (lane >> 4)) ^ (lane & 7)) << 4), r0, r1, r2,
                                          r3);
                            e4m3x4_to_f16x2_scaled(r0, va[h][0], va[h][1]);
                            e4m3x4_to_f16x2_scaled(r1, va[h][2], va[h][3]);
                            e4m3x4_to_f16x2_scaled(r2, va[h + 1][0], va[h + 1][1]);
                            e4m3x4_to_f16x2_scaled(r3, va[h + 1][2], va[h + 1][3]);
                        }
                    } else {
                        const int pnl = mm >> 2, ch = ((mm & 3) << 1) + ((lane >> 3) & 1);
                        ldsm_x4_trans(vb + pnl * C::PANEL_BYTES + vrow * 128 + ((ch ^ (lane & 7)) << 4),
                                      va[h][0], va[h][1], va[h][2], va[h][3]);
                    }
                }
#pragma unroll
                for (int h = 0; h < MG; ++h) {
                    if (mask) {  // rows past L_b may hold anything; 0 * NaN would poison O
                        va[h][0] &= vmask_a;
                        va[h][1] &= vmask_a;
                        va[h][2] &= vmask_b;
                        va[h][3] &= vmask_b;
                    }
                }
#pragma unroll
                for (int h = 0; h < MG; ++h)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_16816<KV8>(o[m0 + h][nt], va[h], pbh[nt][0], pbh[nt][1]);
#pragma unroll
                for (int h = 0; h < MG; ++h)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_16816<KV8>(o[m0 + h][nt], va[h], pbl[nt][0], pbl[nt][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&ctrl->empty[st]));
        }  // mine
        if (++st == NS) { st = 0; ph ^= 1u; }

        if (seg_last) {
            // ---------------------------------------------------- segment end
            if constexpr (!C::Q_IN_REGS) {
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->qempty[seg_q]));
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 4);
                    l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 8);
                    l[nt][j] += __shfl_xor_sync(0xffffffffu, l[nt][j], 16);
                }
            const bool whole = (seg_start_tile == 0) && last_tile;
            tail_cut = !whole;
            tail_b = w.b;
            tail_kv = w.kv;
            tail_nb = w.n_b;
            tail_su = gi - w.tile;
            if (mg > 0) {
                if (!mbar_wait_warp(smem_addr(&ctrl->merge_free), mfree_ph ^ 1u, abort_flag)) { fail(); break; }
                mfree_ph ^= 1u;
                float* mo = merge_o + ((mg - 1) * HG + hg) * C::ROWS * C::OROW;
                float* ml = merge_ml + ((mg - 1) * HG + hg) * C::ROWS * 2;
                if (g == 0) {
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            ml[(8 * nt + 2 * t + j) * 2] = m[nt][j];
                            ml[(8 * nt + 2 * t + j) * 2 + 1] = l[nt][j];
                        }
                }
#pragma unroll
                for (int mm = 0; mm < KS; ++mm)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            mo[(8 * nt + 2 * t + (e & 1)) * C::OROW + 16 * mm + g + 8 * (e >> 1)] = o[mm][nt][e];
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->merge_full));
            } else {
                if (!mbar_wait_warp(smem_addr(&ctrl->merge_full), mfull_ph, abort_flag)) { fail(); break; }
                mfull_ph ^= 1u;
                float M[NT][2], Lsum[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int hl = 8 * nt + 2 * t + j;
                        float mx = m[nt][j];
#pragma unroll
                        for (int k = 1; k < C::MGN; ++k)
                            mx = fmaxf(mx, merge_ml[(((k - 1) * HG + hg) * C::ROWS + hl) * 2]);
                        M[nt][j] = mx;
                        const float ref = mx == NEG_INF ? 0.f : mx;
                        const float f = fast_exp2(m[nt][j] - ref);
                        float L = l[nt][j] * f;
#pragma unroll
                        for (int mm = 0; mm < KS; ++mm) {
                            o[mm][nt][j] *= f;
                            o[mm][nt][j + 2] *= f;
                        }
#pragma unroll
                        for (int k = 1; k < C::MGN; ++k) {
                            const float* ml = merge_ml + (((k - 1) * HG + hg) * C::ROWS + hl) * 2;
                            const float* mo = merge_o + (((k - 1) * HG + hg) * C::ROWS + hl) * C::OROW;
                            const float e = fast_exp2(ml[0] - ref);
                            L += ml[1] * e;
#pragma unroll
                            for (int mm = 0; mm < KS; ++mm) {
                                o[mm][nt][j] += mo[16 * mm + g] * e;
                                o[mm][nt][j + 2] += mo[16 * mm + g + 8] * e;
                            }
                        }
                        Lsum[nt][j] = L;
                    }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->merge_free));
                const int64_t slot = first_seg ? 2 * static_cast<int64_t>(blockIdx.x) : 2 * static_cast<int64_t>(blockIdx.x) + 1;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int r = hg * C::ROWS + 8 * nt + 2 * t + j;
                        if (r >= a.R) continue;
                        const float inv = seg_vs / Lsum[nt][j];
                        if (whole) {
                            const int64_t row = (static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R + r) * D;
#pragma unroll
                            for (int mm = 0; mm < KS; ++mm)
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const float x = o[mm][nt][j + 2 * hh] * inv;
                                    const int64_t i = row + (KV8 ? 16 * mm + 2 * g + hh : 16 * mm + g + 8 * hh);
                                    if constexpr (OUT_BF16)
                                        static_cast<__nv_bfloat16*>(a.out)[i] = __float2bfloat16_rn(x);
                                    else
                                        static_cast<float*>(a.out)[i] = x;
                                }
                        } else {
                            float* dst = a.ws_o + (slot * a.R + r) * D;
#pragma unroll
                            for (int mm = 0; mm < KS; ++mm) {
                                if constexpr (KV8) {
                                    *reinterpret_cast<float2*>(dst + 16 * mm + 2 * g) =
                                        make_float2(o[mm][nt][j] * inv, o[mm][nt][j + 2] * inv);
                                } else {
                                    dst[16 * mm + g] = o[mm][nt][j] * inv;
                                    dst[16 * mm + g + 8] = o[mm][nt][j + 2] * inv;
                                }
                            }
                            if (g == 0) a.ws_lse[slot * a.R + r] = M[nt][j] + log2f(Lsum[nt][j]);
                        }
                    }
                if (!whole) {
                    // This warp wrote its head group's partial (all d, lse): hand it to the merge warp.
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&ctrl->mjob[first_seg ? 0 : 1]));
                }
            }
            first_seg = false;
        }
        if (gi + 1 < hi) w.advance(a);
    }
    // The CTA's last segment was cut: help the merge warp merge its unit.
    if (tail_cut && !*abort_flag &&
        !merge_assist<D, OUT_BF16>(a, &ctrl->assist, &ctrl->merge_last, tail_b, tail_kv, tail_su, tail_nb,
                                   ctrl->plan.n_tiles, ctrl->plan.g, warp, C::NC + 1, abort_flag))
        fail();
}

}  // namespace gqa

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
//   * NTG x HG consumer warps: head group hg (16 query rows) x token group tg
//     (64/NTG tokens of each tile).  Per 16-token chunk a warp computes
//     S = Q K^T with mma.sync m16n8k16 (bf16 in, fp32 out), masks tokens
//     >= L_b, updates an fp32 online softmax (base-2 exponent, warp shuffles
//     for the row max), and accumulates O += P V with P split into bf16
//     hi + lo parts so the weights keep ~16 significant bits.
//   * at a segment end the token groups are merged in shared memory and the
//     segment writes either the final output or a partial (o / l, m + log2 l).
//
// Every wait is bounded (ptx.cuh); a timeout raises GQA_FLAG_TIMEOUT, lets
// in-flight copies land and returns.  Nothing traps.
#pragma once

#include "ptx.cuh"
#include "schedule.cuh"

namespace gqa {

template <int D, int HG>
struct MmaCfg {
    static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
    static_assert(HG == 1 || HG == 2 || HG == 4, "head groups: 1, 2 or 4");
    static constexpr int NTG = HG >= 4 ? 2 : 4;        // token groups
    static constexpr int TPW = kTile / NTG;             // tokens per warp per tile
    static constexpr int NC = NTG * HG;                 // consumer warps
    static constexpr int THREADS = 32 * (NC + 1);
    static constexpr int PANELS = D / 64;               // 128-byte-wide column panels
    static constexpr int PANEL_BYTES = kTile * 128;     // 64 tokens x 64 bf16
    static constexpr int STAGE_BYTES = 2 * PANELS * PANEL_BYTES;
    static constexpr int QPANEL_BYTES = 16 * 128;       // 16 query rows x 64 bf16
    static constexpr int QSLOT_BYTES = HG * PANELS * QPANEL_BYTES;
    static constexpr int OROW = D + 4;                  // padded merge row (floats)
    static constexpr int MERGE_O_FLOATS = (NTG - 1) * HG * 16 * OROW;
    static constexpr int MERGE_ML_FLOATS = (NTG - 1) * HG * 16 * 2;
    static constexpr int MAX_STAGES = 8;
    static constexpr int CTRL_BYTES = 256;
    static constexpr int FIXED_BYTES =
        2 * QSLOT_BYTES + 4 * (MERGE_O_FLOATS + MERGE_ML_FLOATS) + CTRL_BYTES;
    static constexpr int smem_bytes(int stages) { return 1024 + stages * STAGE_BYTES + FIXED_BYTES; }
};

struct __align__(16) MmaControl {
    uint64_t full[MmaCfg<128, 1>::MAX_STAGES];
    uint64_t empty[MmaCfg<128, 1>::MAX_STAGES];
    uint64_t qfull[2];
    uint64_t qempty[2];
    uint64_t merge_full;
    uint64_t merge_free;
    Plan plan;
    int abort;
};
static_assert(sizeof(MmaControl) <= MmaCfg<128, 1>::CTRL_BYTES, "control block overflows its slot");

template <int D, int HG, bool PAGED, bool OUT_BF16>
__global__ void __launch_bounds__(MmaCfg<D, HG>::THREADS, 1)
    split_mma_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const KernelArgs a) {
    using C = MmaCfg<D, HG>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const int NS = a.n_stages;
    const uint32_t stages = base;
    const uint32_t qring = base + NS * C::STAGE_BYTES;
    float* merge_o = reinterpret_cast<float*>(base_ptr + NS * C::STAGE_BYTES + 2 * C::QSLOT_BYTES);
    float* merge_ml = merge_o + C::MERGE_O_FLOATS;
    MmaControl* ctrl = reinterpret_cast<MmaControl*>(merge_ml + C::MERGE_ML_FLOATS);
    volatile int* abort_flag = &ctrl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_addr(&ctrl->full[s]), 1);
            mbar_init(smem_addr(&ctrl->empty[s]), C::NC);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&ctrl->qfull[s]), 1);
            mbar_init(smem_addr(&ctrl->qempty[s]), C::NC);
        }
        mbar_init(smem_addr(&ctrl->merge_full), (C::NTG - 1) * HG);
        mbar_init(smem_addr(&ctrl->merge_free), HG);
        ctrl->abort = 0;
    }
    // Query rows a TMA box does not cover (R < 16) must read as zeros.
    for (int i = threadIdx.x; i < 2 * C::QSLOT_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(base_ptr + NS * C::STAGE_BYTES)[i] = make_uint4(0, 0, 0, 0);

    grid_dependency_wait();
    grid_launch_dependents();
    if (warp == 0) make_plan(a, &ctrl->plan);
    fence_barrier_init();
    fence_proxy_async_smem();
    __syncthreads();

    const int64_t lo = ctrl->plan.lo;
    const int64_t hi = ctrl->plan.hi;
    if (lo >= hi) return;
    Walk w{ctrl->plan.b, ctrl->plan.kv, ctrl->plan.tile, ctrl->plan.n_b, ctrl->plan.L};

    if (warp == C::NC) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const uint64_t pol_kv = policy_evict_first();
        const uint64_t pol_q = policy_evict_last();
        const uint32_t q_bytes = static_cast<uint32_t>(a.q_groups * C::PANELS * a.q_rows * 128);
        int st = 0, qs = 0;
        uint32_t ph = 0, qph = 0;
        int64_t issued = 0, q_issued = 0;
        int page_word = 0, page_base = -1;
        bool ok = true;
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
                                        &tmQ, bar, 64 * p, w.kv * a.R + 16 * g, w.b, pol_q);
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
            if (!mbar_wait_warp(smem_addr(&ctrl->empty[st]), ph ^ 1u, abort_flag)) { ok = false; break; }
            if (lane == 0) {
                const uint32_t bar = smem_addr(&ctrl->full[st]);
                const uint32_t kb = stages + st * C::STAGE_BYTES;
                const uint32_t vb = kb + C::PANELS * C::PANEL_BYTES;
                mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                for (int p = 0; p < C::PANELS; ++p) {
                    tma_load_4d(kb + p * C::PANEL_BYTES, &tmK, bar, 64 * p, w.kv, c2, c3, pol_kv);
                    tma_load_4d(vb + p * C::PANEL_BYTES, &tmV, bar, 64 * p, w.kv, c2, c3, pol_kv);
                }
            }
            ++issued;
            if (++st == NS) { st = 0; ph ^= 1u; }
            if (gi + 1 < hi) w.advance(a);
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) atomicOr(a.status, kFlagTimeout);
            // Let copies already in flight land before the CTA's shared memory goes away.
            const int64_t first = issued > NS ? issued - NS : 0;
            for (int64_t i = first; i < issued; ++i)
                mbar_wait(smem_addr(&ctrl->full[i % NS]), static_cast<uint32_t>((i / NS) & 1), nullptr);
            const int64_t qfirst = q_issued > 2 ? q_issued - 2 : 0;
            for (int64_t i = qfirst; i < q_issued; ++i)
                mbar_wait(smem_addr(&ctrl->qfull[i % 2]), static_cast<uint32_t>((i / 2) & 1), nullptr);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int hg = warp / C::NTG;
    const int tg = warp % C::NTG;
    const int g = lane >> 2;
    const int t = lane & 3;
    const float NEG_INF = -__int_as_float(0x7f800000);

    int st = 0, qs = 0;
    uint32_t ph = 0, qph = 0, mfull_ph = 0, mfree_ph = 0;
    bool first_seg = true;
    int seg_start_tile = 0;
    uint32_t qa[D / 16][4];
    float o[D / 8][4];
    float m0 = NEG_INF, m1 = NEG_INF, l0 = 0.f, l1 = 0.f;

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
            const uint32_t qbase = qring + qs * C::QSLOT_BYTES + hg * C::PANELS * C::QPANEL_BYTES;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int p = ks >> 2, c0 = (ks & 3) << 1;
                const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
                const int ch = c0 + (lane >> 4);
                ldsm_x4(qbase + p * C::QPANEL_BYTES + row * 128 + ((ch ^ (row & 7)) << 4), qa[ks][0],
                        qa[ks][1], qa[ks][2], qa[ks][3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&ctrl->qempty[qs]));
            if (++qs == 2) { qs = 0; qph ^= 1u; }
            m0 = m1 = NEG_INF;
            l0 = l1 = 0.f;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        }

        if (!mbar_wait_warp(smem_addr(&ctrl->full[st]), ph, abort_flag)) { fail(); break; }
        const uint32_t kb = stages + st * C::STAGE_BYTES;
        const uint32_t vb = kb + C::PANELS * C::PANEL_BYTES;
        const int t0 = w.tile * kTile;

#pragma unroll
        for (int c = 0; c < C::TPW / 16; ++c) {
            const int n0 = tg * C::TPW + c * 16;
            if (last_tile && t0 + n0 >= w.L) break;  // no live token in this chunk
            const bool mask = last_tile && (t0 + n0 + 16 > w.L);

            // S = Q K^T for 16 query rows x 16 tokens.  Even and odd k-steps
            // accumulate separately so four independent mma chains interleave.
            float s[2][4], s2[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) s[n][i] = s2[n][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ks += 2) {
                const int row = n0 + (lane & 7) + ((lane >> 4) << 3);
                uint32_t b[2][4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int p = (ks + h) >> 2, c0 = ((ks + h) & 3) << 1;
                    const int ch = c0 + ((lane >> 3) & 1);
                    ldsm_x4(kb + p * C::PANEL_BYTES + row * 128 + ((ch ^ (lane & 7)) << 4), b[h][0], b[h][1],
                            b[h][2], b[h][3]);
                }
                mma_bf16_16816(s[0], qa[ks], b[0][0], b[0][1]);
                mma_bf16_16816(s[1], qa[ks], b[0][2], b[0][3]);
                mma_bf16_16816(s2[0], qa[ks + 1], b[1][0], b[1][1]);
                mma_bf16_16816(s2[1], qa[ks + 1], b[1][2], b[1][3]);
            }
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) s[n][i] = (s[n][i] + s2[n][i]) * a.sl2;
            uint32_t vmask_a = 0xffffffffu, vmask_b = 0xffffffffu;
            if (mask) {
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tok = t0 + n0 + 8 * n + 2 * t + (i & 1);
                        if (tok >= w.L) s[n][i] = NEG_INF;
                    }
                const int ta = t0 + n0 + 2 * t;
                vmask_a = (ta < w.L ? 0x0000ffffu : 0u) | (ta + 1 < w.L ? 0xffff0000u : 0u);
                vmask_b = (ta + 8 < w.L ? 0x0000ffffu : 0u) | (ta + 9 < w.L ? 0xffff0000u : 0u);
            }

            // Online softmax (rows g and g + 8 of the head group).
            float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
            float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float ref0 = mn0 == NEG_INF ? 0.f : mn0;
            const float ref1 = mn1 == NEG_INF ? 0.f : mn1;
            const float al0 = exp2f(m0 - ref0), al1 = exp2f(m1 - ref1);
            m0 = mn0;
            m1 = mn1;
            float p[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                p[n][0] = exp2f(s[n][0] - ref0);
                p[n][1] = exp2f(s[n][1] - ref0);
                p[n][2] = exp2f(s[n][2] - ref1);
                p[n][3] = exp2f(s[n][3] - ref1);
            }
            l0 = l0 * al0 + (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
            l1 = l1 * al1 + (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
            if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= al0;
                    o[n][1] *= al0;
                    o[n][2] *= al1;
                    o[n][3] *= al1;
                }
            }
            uint32_t ph_[4], pl_[4];
            split_bf16x2(p[0][0], p[0][1], ph_[0], pl_[0]);
            split_bf16x2(p[0][2], p[0][3], ph_[1], pl_[1]);
            split_bf16x2(p[1][0], p[1][1], ph_[2], pl_[2]);
            split_bf16x2(p[1][2], p[1][3], ph_[3], pl_[3]);

            // O += P V  (P as hi + lo bf16 parts).  Two 16-column blocks per
            // step: the hi products of four accumulators issue before the lo
            // products that depend on them.
#pragma unroll
            for (int j = 0; j < D / 16; j += 2) {
                const int row = n0 + (lane & 7) + (((lane >> 3) & 1) << 3);
                uint32_t v[2][4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int pnl = (j + h) >> 2, c0 = ((j + h) & 3) << 1;
                    const int ch = c0 + (lane >> 4);
                    ldsm_x4_trans(vb + pnl * C::PANEL_BYTES + row * 128 + ((ch ^ (lane & 7)) << 4), v[h][0],
                                  v[h][1], v[h][2], v[h][3]);
                    v[h][0] &= vmask_a;
                    v[h][1] &= vmask_b;
                    v[h][2] &= vmask_a;
                    v[h][3] &= vmask_b;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mma_bf16_16816(o[2 * (j + h)], ph_, v[h][0], v[h][1]);
                    mma_bf16_16816(o[2 * (j + h) + 1], ph_, v[h][2], v[h][3]);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mma_bf16_16816(o[2 * (j + h)], pl_, v[h][0], v[h][1]);
                    mma_bf16_16816(o[2 * (j + h) + 1], pl_, v[h][2], v[h][3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&ctrl->empty[st]));
        if (++st == NS) { st = 0; ph ^= 1u; }

        if (seg_last) {
            // ---------------------------------------------------- segment end
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            const bool whole = (seg_start_tile == 0) && last_tile;
            if (tg > 0) {
                if (!mbar_wait_warp(smem_addr(&ctrl->merge_free), mfree_ph ^ 1u, abort_flag)) { fail(); break; }
                mfree_ph ^= 1u;
                float* mo = merge_o + ((tg - 1) * HG + hg) * 16 * C::OROW;
                float* ml = merge_ml + ((tg - 1) * HG + hg) * 32;
                if (t == 0) {
                    ml[g * 2] = m0;
                    ml[g * 2 + 1] = l0;
                    ml[(g + 8) * 2] = m1;
                    ml[(g + 8) * 2 + 1] = l1;
                }
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    *reinterpret_cast<float2*>(&mo[g * C::OROW + 8 * n + 2 * t]) = make_float2(o[n][0], o[n][1]);
                    *reinterpret_cast<float2*>(&mo[(g + 8) * C::OROW + 8 * n + 2 * t]) = make_float2(o[n][2], o[n][3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->merge_full));
            } else {
                if (!mbar_wait_warp(smem_addr(&ctrl->merge_full), mfull_ph, abort_flag)) { fail(); break; }
                mfull_ph ^= 1u;
                float M0 = m0, M1 = m1;
#pragma unroll
                for (int k = 1; k < C::NTG; ++k) {
                    const float* ml = merge_ml + ((k - 1) * HG + hg) * 32;
                    M0 = fmaxf(M0, ml[g * 2]);
                    M1 = fmaxf(M1, ml[(g + 8) * 2]);
                }
                const float R0 = M0 == NEG_INF ? 0.f : M0;
                const float R1 = M1 == NEG_INF ? 0.f : M1;
                const float f0 = exp2f(m0 - R0), f1 = exp2f(m1 - R1);
                float L0 = l0 * f0, L1 = l1 * f1;
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= f0;
                    o[n][1] *= f0;
                    o[n][2] *= f1;
                    o[n][3] *= f1;
                }
#pragma unroll
                for (int k = 1; k < C::NTG; ++k) {
                    const float* ml = merge_ml + ((k - 1) * HG + hg) * 32;
                    const float* mo = merge_o + ((k - 1) * HG + hg) * 16 * C::OROW;
                    const float e0 = exp2f(ml[g * 2] - R0), e1 = exp2f(ml[(g + 8) * 2] - R1);
                    L0 += ml[g * 2 + 1] * e0;
                    L1 += ml[(g + 8) * 2 + 1] * e1;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        const float2 x = *reinterpret_cast<const float2*>(&mo[g * C::OROW + 8 * n + 2 * t]);
                        const float2 y = *reinterpret_cast<const float2*>(&mo[(g + 8) * C::OROW + 8 * n + 2 * t]);
                        o[n][0] += x.x * e0;
                        o[n][1] += x.y * e0;
                        o[n][2] += y.x * e1;
                        o[n][3] += y.y * e1;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&ctrl->merge_free));
                const float inv0 = 1.f / L0, inv1 = 1.f / L1;
                const int r0 = hg * 16 + g, r1 = r0 + 8;
                if (whole) {
                    const int64_t row0 = static_cast<int64_t>(w.b) * a.H_Q + w.kv * a.R + r0;
                    const int64_t row1 = row0 + 8;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        const int d = 8 * n + 2 * t;
                        if constexpr (OUT_BF16) {
                            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
                            if (r0 < a.R)
                                *reinterpret_cast<__nv_bfloat162*>(out + row0 * D + d) =
                                    __floats2bfloat162_rn(o[n][0] * inv0, o[n][1] * inv0);
                            if (r1 < a.R)
                                *reinterpret_cast<__nv_bfloat162*>(out + row1 * D + d) =
                                    __floats2bfloat162_rn(o[n][2] * inv1, o[n][3] * inv1);
                        } else {
                            float* out = static_cast<float*>(a.out);
                            if (r0 < a.R)
                                *reinterpret_cast<float2*>(out + row0 * D + d) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
                            if (r1 < a.R)
                                *reinterpret_cast<float2*>(out + row1 * D + d) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
                        }
                    }
                } else {
                    const int64_t slot = first_seg ? 2 * static_cast<int64_t>(blockIdx.x) : 2 * static_cast<int64_t>(blockIdx.x) + 1;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        const int d = 8 * n + 2 * t;
                        if (r0 < a.R)
                            *reinterpret_cast<float2*>(a.ws_o + (slot * a.R + r0) * D + d) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
                        if (r1 < a.R)
                            *reinterpret_cast<float2*>(a.ws_o + (slot * a.R + r1) * D + d) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
                    }
                    if (t == 0) {
                        if (r0 < a.R) a.ws_lse[slot * a.R + r0] = M0 + log2f(L0);
                        if (r1 < a.R) a.ws_lse[slot * a.R + r1] = M1 + log2f(L1);
                    }
                }
            }
            first_seg = false;
        }
        if (gi + 1 < hi) w.advance(a);
    }
}

}  // namespace gqa

// schedule.cuh -- how one decode step's KV work is cut into split-KV pieces.
//
// A "unit" is one (sequence b, KV head kv) pair: the L_b cached tokens of
// key/value head kv that its R query heads attend over ("Grouped-Query
// Attention (GQA) and Multi-Query Attention (MQA): Mathematical Foundations,
// ...", section 2, Head_i = softmax(Q_i K_{g(i)}^T / sqrt(d_k) + M) V_{g(i)}).
// Unit u = b * H_KV + kv holds n_b = ceil(L_b / 64) tiles of 64 tokens.
//
// All units' tiles are laid end to end (b-major, then kv, then tile) into
// N_T global tiles, and CTA c of the G_eff = min(gridDim, N_T) working CTAs
// takes the contiguous range [floor(c N_T / G_eff), floor((c+1) N_T / G_eff)).
// Every CTA therefore streams the same number of tiles (+-1) whatever the
// mix of sequence lengths.  Each run of one unit inside one CTA is a
// "segment" -- a (sequence, KV head, KV split) triple of the split-KV method.
// A segment that covers its whole unit writes the final output; otherwise it
// writes a partial (normalised o, log2-sum-exp) into one of two workspace
// slots of its CTA: 2c for the CTA's first segment, 2c+1 for its last.  A
// unit cut across CTAs c_a..c_b has one partial per CTA; c_a is unique to it
// (only a CTA's last segment can continue past its range), so c_a indexes its
// merge counter.  Each writer arrives on that counter after its partial is
// visible, and the last of the unit's writers merges all partials (found from
// the same arithmetic) into the output -- no separate combine launch.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gqa {

constexpr int kTile = 64;             // tokens per tile; also the page size
constexpr uint32_t kFlagClamped = 1u;  // GQA_FLAG_SEQ_LEN_CLAMPED
constexpr uint32_t kFlagBadBlock = 2u; // GQA_FLAG_BAD_BLOCK
constexpr uint32_t kFlagTimeout = 4u;  // GQA_FLAG_TIMEOUT
constexpr uint32_t kFlagBadPosition = 8u;  // GQA_FLAG_BAD_POSITION
constexpr uint32_t kFlagBadSpan = 16u;     // GQA_FLAG_BAD_QUERY_SPAN

// Merge counters: two banks of kMergeCounters words after the 256-byte
// workspace header.  Header words: [0] status flags, [1] merge epoch, [2] CTAs
// of the running call that have read the epoch.  A call counts arrivals in
// bank (epoch & 1) and zeroes the other bank, which the next call (epoch + 1)
// uses; so a call cut short (a timed-out wait) never leaves stale counts for
// the call after it.
constexpr int kMergeCounters = 2048;
constexpr size_t kMergeCounterBytes = 2 * kMergeCounters * sizeof(uint32_t);

struct KernelArgs {
    const int32_t* seq_lens;     // [B]
    const int32_t* block_table;  // [B, max_blocks] or null
    int B, H_Q, H_KV, R;
    int max_len;     // seq_lens are clamped to [0, max_len]
    int S_max;       // contiguous cache capacity (token stride owner); 0 when paged
    int max_blocks;  // block-table columns (paged)
    int num_blocks;  // pages in the cache (paged)
    float sl2;       // softmax scale * log2(e): scores are kept in base-2 units
    void* out;       // [B, H_Q, D]
    float* ws_o;     // [2G, R, D] partial outputs (normalised)
    float* ws_lse;   // [2G, R] partial log2-sum-exp
    uint32_t* status;  // workspace header: status word, merge epoch, epoch readers
    uint32_t* merge;   // [2][kMergeCounters] merge counters
    int n_stages;    // tensor-core path: pipeline depth
    int q_rows;      // tensor-core path: query rows per TMA box, min(R, 16)
    int q_groups;    // tensor-core path: 16-row head groups holding real rows
    const float* k_scale;  // [H_KV] or null: stored keys are multiplied by k_scale[g]
    const float* v_scale;  // [H_KV] or null: stored values likewise
};

__device__ __forceinline__ int clamp_len(int L, int max_len) {
    return L < 0 ? 0 : (L > max_len ? max_len : L);
}

__device__ __forceinline__ int tiles_of(int L) { return (L + kTile - 1) / kTile; }

__device__ __forceinline__ int seq_len_at(const KernelArgs& a, int b) {
    return clamp_len(__ldg(a.seq_lens + b), a.max_len);
}

__device__ __forceinline__ int64_t warp_sum_i64(int64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Warp-collective: N_T, and whether any seq_lens entry needed clamping.
__device__ __forceinline__ int64_t warp_total_tiles(const KernelArgs& a, bool* clamped) {
    const int lane = threadIdx.x & 31;
    int64_t acc = 0;
    bool bad = false;
    for (int b = lane; b < a.B; b += 32) {
        const int raw = __ldg(a.seq_lens + b);
        bad |= (raw < 0 || raw > a.max_len);
        acc += static_cast<int64_t>(a.H_KV) * tiles_of(clamp_len(raw, a.max_len));
    }
    *clamped = __any_sync(0xffffffffu, bad);
    return warp_sum_i64(acc);
}

// Warp-collective: the sequence b whose tiles [P_b, P_b + H_KV n_b) hold
// global tile `target` (< N_T), and P_b.
__device__ __forceinline__ void warp_find_batch(const KernelArgs& a, int64_t target, int* b_out,
                                                int64_t* start_out) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
        const int b = b0 + lane;
        const int64_t cnt = b < a.B ? static_cast<int64_t>(a.H_KV) * tiles_of(seq_len_at(a, b)) : 0;
        int64_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int64_t excl = incl - cnt;
        const bool hit = (base + excl <= target) && (target < base + incl);
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            *b_out = __shfl_sync(0xffffffffu, b, src);
            *start_out = base + __shfl_sync(0xffffffffu, excl, src);
            return;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    *b_out = a.B;
    *start_out = base;
}

__device__ __forceinline__ int effective_grid(int64_t n_tiles, int grid) {
    return n_tiles < grid ? static_cast<int>(n_tiles) : grid;
}

__device__ __forceinline__ int64_t cta_first_tile(int64_t c, int64_t n_tiles, int64_t g) {
    return c * n_tiles / g;
}

// The CTA whose range holds global tile t.
__device__ __forceinline__ int64_t owner_of_tile(int64_t t, int64_t n_tiles, int64_t g) {
    return ((t + 1) * g - 1) / n_tiles;
}

// Position of a CTA's walk over its tile range.
struct Walk {
    int b, kv, tile, n_b, L;

    __device__ __forceinline__ void advance(const KernelArgs& a) {
        if (++tile < n_b) return;
        tile = 0;
        if (++kv < a.H_KV) return;
        kv = 0;
        do {
            ++b;
            if (b >= a.B) {
                n_b = 0;
                L = 0;
                return;
            }
            L = seq_len_at(a, b);
            n_b = tiles_of(L);
        } while (n_b == 0);
    }
};

// Per-CTA plan, computed once by one warp and shared through shared memory.
struct Plan {
    int64_t lo, hi;  // global tile range of this CTA
    int b, kv, tile, n_b, L;
    int64_t n_tiles; // N_T
    int g;           // working CTAs, min(gridDim, N_T)
};

// One thread per CTA (its merge warp), after the grid dependency wait: this
// call's merge epoch.  The last CTA to take it advances it for the next call; every CTA
// has read it by then (each reads before it counts itself).
__device__ __forceinline__ uint32_t merge_epoch_take(const KernelArgs& a) {
    const uint32_t e = *reinterpret_cast<volatile uint32_t*>(a.status + 1);
    __threadfence();  // the read above is complete before this CTA is counted
    if (atomicAdd(a.status + 2, 1u) == gridDim.x - 1) {
        a.status[2] = 0u;  // plain stores: the next call reads them after this grid has completed
        a.status[1] = e + 1u;
    }
    return e;
}

// Warp-collective; lane 0 writes *plan.  Also raises the clamp flag (CTA 0).
__device__ __forceinline__ void make_plan(const KernelArgs& a, Plan* plan) {
    const int lane = threadIdx.x & 31;
    bool clamped = false;
    const int64_t n_tiles = warp_total_tiles(a, &clamped);
    if (clamped && lane == 0 && blockIdx.x == 0) atomicOr(a.status, kFlagClamped);
    const int g = effective_grid(n_tiles, gridDim.x);
    int64_t lo = 0, hi = 0;
    if (static_cast<int>(blockIdx.x) < g) {
        lo = cta_first_tile(blockIdx.x, n_tiles, g);
        hi = cta_first_tile(blockIdx.x + 1, n_tiles, g);
    }
    int b = 0;
    int64_t start = 0;
    if (lo < hi) warp_find_batch(a, lo, &b, &start);
    if (lane == 0) {
        plan->lo = lo;
        plan->hi = hi;
        plan->n_tiles = n_tiles;
        plan->g = g;
        plan->b = b;
        plan->kv = plan->tile = plan->n_b = plan->L = 0;
        if (lo < hi) {
            const int L = seq_len_at(a, b);
            const int n_b = tiles_of(L);
            const int64_t local = lo - start;
            plan->L = L;
            plan->n_b = n_b;
            plan->kv = static_cast<int>(local / n_b);
            plan->tile = static_cast<int>(local % n_b);
        }
    }
}

// ---------------------------------------------------------------- split units

// The unit whose first global tile is s_u and which has n_b tiles, as the
// schedule cut it: CTAs ca..ca+n_parts-1 each hold one partial of it.
struct SplitUnit {
    int64_t ca;
    int n_parts;
    int64_t slot0;  // workspace slot of part 0 (ca's last segment)
};

__device__ __forceinline__ SplitUnit split_unit_of(int64_t s_u, int n_b, int64_t n_tiles, int64_t g) {
    SplitUnit u;
    u.ca = owner_of_tile(s_u, n_tiles, g);
    u.n_parts = static_cast<int>(owner_of_tile(s_u + n_b - 1, n_tiles, g) - u.ca + 1);
    u.slot0 = cta_first_tile(u.ca, n_tiles, g) < s_u ? 2 * u.ca + 1 : 2 * u.ca;
    return u;
}

// Slot of part j: part 0 is ca's last segment, every later part its CTA's first.
__device__ __forceinline__ int64_t part_slot(const SplitUnit& u, int j) {
    return j == 0 ? u.slot0 : 2 * (u.ca + j);
}

// This call's counter bank; the CTA's share of the other bank is zeroed here
// (by the threads [t0, t0 + nt) of the CTA) for the next call.
__device__ __forceinline__ uint32_t* merge_bank(const KernelArgs& a, uint32_t epoch, int t0, int nt) {
    uint32_t* other = a.merge + ((epoch + 1u) & 1u) * kMergeCounters;
    for (int i = blockIdx.x * nt + (static_cast<int>(threadIdx.x) - t0); i < kMergeCounters; i += gridDim.x * nt)
        other[i] = 0u;
    return a.merge + (epoch & 1u) * kMergeCounters;
}

// Threads [t0, t0 + nt) of the CTA write out = 0 for every sequence with
// L_b = 0 among b = blockIdx.x, blockIdx.x + gridDim.x, ... (an empty sum).
template <int D, bool OUT_BF16>
__device__ __forceinline__ void zero_empty_sequences(const KernelArgs& a, int t0, int nt) {
    const int t = static_cast<int>(threadIdx.x) - t0;
    for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
        if (seq_len_at(a, b) != 0) continue;
        const int64_t base = static_cast<int64_t>(b) * a.H_Q * D;
        const int n = a.H_Q * D;
        // 8-byte stores: out is only required to be 8-byte aligned
        if constexpr (OUT_BF16) {
            for (int i = t; i < n / 4; i += nt)
                reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + base)[i] = make_uint2(0u, 0u);
        } else {
            for (int i = t; i < n / 2; i += nt)
                reinterpret_cast<float2*>(static_cast<float*>(a.out) + base)[i] = make_float2(0.f, 0.f);
        }
    }
}

}  // namespace gqa

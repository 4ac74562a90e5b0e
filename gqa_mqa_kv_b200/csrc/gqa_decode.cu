// gqa_decode.cu -- host side of the C ABI declared in include/gqa_decode.h.
//
// Validates arguments, picks the kernel (tensor-core split kernel for bf16
// with groups of up to 64 query heads, CUDA-core split kernel otherwise),
// encodes the TMA tensor maps, and enqueues the split kernel -- which also
// merges the partials of units it cut across CTAs -- on the caller's stream
// with programmatic dependent launch.  No allocation, no host synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "gqa_decode.h"
#include "combine.cuh"
#include "split_mma.cuh"
#include "split_simt.cuh"
#include "split_tc.cuh"
#include "prefill_tc.cuh"
#include "rope_append.cuh"

namespace {

using namespace gqa;

constexpr size_t kHeaderBytes = 256;  // words 0..2: status flags, merge epoch, epoch readers
constexpr int kSimtCtasPerSm = 4;
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
};

gqa_status device_info(DeviceInfo* info) {
    static std::mutex mu;
    static DeviceInfo cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev].sms == 0) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return GQA_ERR_CUDA;
        cache[dev] = d;
    }
    *info = cache[dev];
    return GQA_OK;
}

bool aligned(const void* p, size_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; }

size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

gqa_status validate_params(const gqa_decode_params* p) {
    if (p == nullptr) return GQA_ERR_INVALID;
    if (p->B < 0 || p->H_Q <= 0 || p->H_KV <= 0 || p->max_seq_len < 0) return GQA_ERR_INVALID;
    if (p->H_Q % p->H_KV != 0) return GQA_ERR_INVALID;
    if (p->qkv_dtype != GQA_BF16 && p->qkv_dtype != GQA_F32) return GQA_ERR_INVALID;
    if (p->out_dtype != GQA_BF16 && p->out_dtype != GQA_F32) return GQA_ERR_INVALID;
    if (p->kernel < GQA_KERNEL_AUTO || p->kernel > GQA_KERNEL_TCGEN05) return GQA_ERR_INVALID;
    if (p->page_size != 0 && p->page_size != kTile) return GQA_ERR_UNSUPPORTED;
    if (p->head_dim != 64 && p->head_dim != 128) return GQA_ERR_UNSUPPORTED;
    if (p->page_size == 0) {
        if (p->max_blocks_per_seq != 0 || p->num_blocks != 0) return GQA_ERR_INVALID;
    } else {
        if (p->max_blocks_per_seq <= 0 || p->num_blocks <= 0) return GQA_ERR_INVALID;
        if (static_cast<int64_t>(p->max_seq_len) > static_cast<int64_t>(p->max_blocks_per_seq) * kTile)
            return GQA_ERR_INVALID;
    }
    // 64-bit element offsets are used throughout; keep 32-bit grid / head math safe.
    if (static_cast<int64_t>(p->B) * p->H_Q > (int64_t(1) << 30)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

enum class SplitKernel { kMmaSync, kTcgen05, kSimt, kNone };

// Which split kernel serves a problem (gqa_kernel in the header).
SplitKernel select_kernel(const gqa_decode_params* p, bool kv8) {
    const int R = p->H_Q / p->H_KV;
    const bool tc_ok = p->head_dim == 128 && R <= 32 && p->qkv_dtype == GQA_BF16;
    const bool mma_ok = p->qkv_dtype == GQA_BF16 && (kv8 ? (p->head_dim == 128 && R <= 8) : R <= 64);
    switch (p->kernel) {
        case GQA_KERNEL_TCGEN05: return tc_ok ? SplitKernel::kTcgen05 : SplitKernel::kNone;
        case GQA_KERNEL_MMA_SYNC: return mma_ok ? SplitKernel::kMmaSync : SplitKernel::kNone;
        default:
            // Measured on one B200: tcgen05 wins for 8-bit caches and for bf16 groups of
            // 9..32 heads (R = 16: 53.3 vs 55.6 us); mma.sync for the HBM-bound groups of
            // up to 8 heads (R = 8: 93.0 vs 94.0 us, R = 4: 51.0 vs 52.6 us).
            if (kv8) return tc_ok ? SplitKernel::kTcgen05 : SplitKernel::kSimt;
            if (tc_ok && R > 8) return SplitKernel::kTcgen05;
            return mma_ok ? SplitKernel::kMmaSync : SplitKernel::kSimt;
    }
}

// CTAs of a split launch: one per SM (tensor-core kernels) or kSimtCtasPerSm per
// SM (CUDA-core kernel), but never more than the step can have tiles,
// B H_KV ceil(max_seq_len / 64): a CTA without tiles would still take the
// merge epoch and clear its share of the counters, which costs a tiny step
// more than its work.
int grid_for(const gqa_decode_params* p, const DeviceInfo& dev, bool kv8 = false) {
    const int full = select_kernel(p, kv8) == SplitKernel::kSimt && !kv8 ? dev.sms * kSimtCtasPerSm : dev.sms;
    const int64_t most = static_cast<int64_t>(p->B) * p->H_KV * ((static_cast<int64_t>(p->max_seq_len) + 63) / 64);
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(full, most)));
}

// Workspace layout: header (status word, merge epoch), two banks of merge
// counters, then the partials ws_o [2G, R, D] and ws_lse [2G, R].
size_t ws_o_bytes(const gqa_decode_params* p, int grid) {
    const size_t R = static_cast<size_t>(p->H_Q / p->H_KV);
    return round_up(2 * static_cast<size_t>(grid) * R * p->head_dim * sizeof(float), 256);
}

size_t workspace_for(const gqa_decode_params* p, int grid) {
    const size_t R = static_cast<size_t>(p->H_Q / p->H_KV);
    const size_t slots = 2 * static_cast<size_t>(grid);
    return kHeaderBytes + kMergeCounterBytes + ws_o_bytes(p, grid) + round_up(slots * R * sizeof(float), 256);
}

// ------------------------------------------------------------------ TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                             &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Tiled tensor map with a 128-byte swizzle; out-of-bounds elements read as zero.
// L2 promotion: 256-byte requests suit rows of 256 bytes or more (a bf16 head
// row at head_dim 128); a 128-byte row (an E4M3 head row) takes 128-byte
// requests, or every fetch would also pull the neighbouring head's row.
bool encode_map(CUtensorMap* map, CUtensorMapDataType type, const void* base, int rank,
                const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                CUtensorMapL2promotion promotion = CU_TENSOR_MAP_L2_PROMOTION_L2_256B) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    return fn(map, type, static_cast<cuuint32_t>(rank),
              const_cast<void*>(base), d, s, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, promotion,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launches

template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                           cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({kernel, dev});
    return e;
}

struct Buffers {
    const void* q;
    const void* k;
    const void* v;
    bool kv8;  // k and v hold E4M3 bytes (scales in KernelArgs)
};

template <int D, int NT, int HG, bool PAGED, bool OUTB, bool KV8 = false>
cudaError_t launch_mma(const gqa_decode_params* p, const Buffers& buf, KernelArgs args,
                       const DeviceInfo& dev, int grid, cudaStream_t stream, bool* encode_ok) {
    using C = MmaCfg<D, NT, HG, KV8>;
    const int R = p->H_Q / p->H_KV;
    int stages = (dev.smem_optin - C::FIXED_BYTES - 1024) / C::STAGE_BYTES;
    if (stages > C::MAX_STAGES) stages = C::MAX_STAGES;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    args.n_stages = stages;
    args.q_rows = R < C::ROWS ? R : C::ROWS;
    args.q_groups = (R + C::ROWS - 1) / C::ROWS;

    CUtensorMap tmQ, tmK, tmV;
    const uint64_t row = static_cast<uint64_t>(D) * 2;
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(p->H_Q),
                                  static_cast<uint64_t>(p->B)};
        const uint64_t strides[2] = {row, row * p->H_Q};
        const uint32_t box[3] = {64, static_cast<uint32_t>(args.q_rows), 1};
        *encode_ok = encode_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, buf.q, 3, dims, strides, box);
    }
    // K/V boxes: 64 tokens x 64 bf16 (128 bytes), or 64 tokens x 128 E4M3 bytes.
    const uint32_t box4[4] = {KV8 ? static_cast<uint32_t>(D) : 64u, 1, static_cast<uint32_t>(kTile), 1};
    const uint64_t kv_row = KV8 ? static_cast<uint64_t>(D) : row;
    if (*encode_ok) {
        uint64_t dims[4], strides[3];
        dims[0] = D;
        dims[1] = p->H_KV;
        strides[0] = kv_row;
        strides[1] = kv_row * p->H_KV;
        if (PAGED) {
            dims[2] = kTile;
            dims[3] = p->num_blocks;
        } else {
            dims[2] = p->max_seq_len > 0 ? p->max_seq_len : 1;
            dims[3] = p->B;
        }
        strides[2] = strides[1] * dims[2];
        const CUtensorMapDataType kv_type = KV8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const CUtensorMapL2promotion promo =
            kv_row * 2 <= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
        *encode_ok = encode_map(&tmK, kv_type, buf.k, 4, dims, strides, box4, promo) &&
                     encode_map(&tmV, kv_type, buf.v, 4, dims, strides, box4, promo);
    }
    if (!*encode_ok) return cudaErrorInvalidValue;
    auto kernel = split_mma_kernel<D, NT, HG, PAGED, OUTB, KV8>;
    const int smem = C::smem_bytes(stages);
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_chained(kernel, grid, C::THREADS, smem, stream, tmQ, tmK, tmV, args);
}

template <int D, bool PAGED, bool OUTB>
cudaError_t launch_mma_groups(const gqa_decode_params* p, const Buffers& buf,
                              const KernelArgs& args, const DeviceInfo& dev, int grid,
                              cudaStream_t stream, bool* encode_ok) {
    const int R = p->H_Q / p->H_KV;
    if (R <= 8) return launch_mma<D, 1, 1, PAGED, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
    if (R <= 16) return launch_mma<D, 2, 1, PAGED, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
    if (R <= 32) return launch_mma<D, 2, 2, PAGED, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
    return launch_mma<D, 4, 2, PAGED, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
}

// tcgen05 split kernel (head_dim 128): RP query columns per KV head.
template <int RP, bool PAGED, bool OUTB, bool KV8>
cudaError_t launch_tc(const gqa_decode_params* p, const Buffers& buf, KernelArgs args, const DeviceInfo& dev,
                      int grid, cudaStream_t stream, bool* encode_ok) {
    using C = TcCfg<RP, KV8>;
    constexpr int D = 128;
    int stages = (dev.smem_optin - C::FIXED_BYTES - 1024) / C::STAGE_BYTES;
    if (stages > C::MAX_STAGES) stages = C::MAX_STAGES;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    args.n_stages = stages;

    CUtensorMap tmQ, tmK, tmV;
    const uint64_t row = static_cast<uint64_t>(D) * 2;
    {
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(p->H_Q),
                                  static_cast<uint64_t>(p->B)};
        const uint64_t strides[2] = {row, row * p->H_Q};
        const uint32_t box[3] = {64, static_cast<uint32_t>(RP), 1};
        *encode_ok = encode_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, buf.q, 3, dims, strides, box);
    }
    // K/V boxes: 64 tokens x 64 bf16 (128 bytes), or 64 tokens x 128 E4M3 bytes.
    const uint32_t box4[4] = {KV8 ? static_cast<uint32_t>(D) : 64u, 1, static_cast<uint32_t>(kTile), 1};
    const uint64_t kv_row = KV8 ? static_cast<uint64_t>(D) : row;
    if (*encode_ok) {
        uint64_t dims[4], strides[3];
        dims[0] = D;
        dims[1] = p->H_KV;
        strides[0] = kv_row;
        strides[1] = kv_row * p->H_KV;
        if (PAGED) {
            dims[2] = kTile;
            dims[3] = p->num_blocks;
        } else {
            dims[2] = p->max_seq_len > 0 ? p->max_seq_len : 1;
            dims[3] = p->B;
        }
        strides[2] = strides[1] * dims[2];
        const CUtensorMapDataType kv_type = KV8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const CUtensorMapL2promotion promo =
            kv_row * 2 <= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
        *encode_ok = encode_map(&tmK, kv_type, buf.k, 4, dims, strides, box4, promo) &&
                     encode_map(&tmV, kv_type, buf.v, 4, dims, strides, box4, promo);
    }
    if (!*encode_ok) return cudaErrorInvalidValue;
    auto kernel = split_tc_kernel<RP, PAGED, OUTB, KV8>;
    const int smem = C::smem_bytes(stages);
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_chained(kernel, grid, C::THREADS, smem, stream, tmQ, tmK, tmV, args);
}

template <bool PAGED, bool OUTB, bool KV8>
cudaError_t launch_tc_groups(const gqa_decode_params* p, const Buffers& buf, const KernelArgs& args,
                             const DeviceInfo& dev, int grid, cudaStream_t stream, bool* encode_ok) {
    const int R = p->H_Q / p->H_KV;
    if constexpr (KV8)
        if (R <= 8) return launch_tc<8, PAGED, OUTB, KV8>(p, buf, args, dev, grid, stream, encode_ok);
    if (R <= 16) return launch_tc<16, PAGED, OUTB, KV8>(p, buf, args, dev, grid, stream, encode_ok);
    return launch_tc<32, PAGED, OUTB, KV8>(p, buf, args, dev, grid, stream, encode_ok);
}

template <typename TQ, typename TKV, int D, bool PAGED, bool OUTB>
cudaError_t launch_simt(const Buffers& buf, const KernelArgs& args, int grid, cudaStream_t stream) {
    return launch_chained(split_simt_kernel<TQ, TKV, D, PAGED, OUTB>, grid, 32 * kSimtWarps, 0, stream,
                          static_cast<const TQ*>(buf.q), static_cast<const TKV*>(buf.k),
                          static_cast<const TKV*>(buf.v), args);
}

template <int D, bool PAGED, bool OUTB>
cudaError_t launch_split(const gqa_decode_params* p, const Buffers& buf, const KernelArgs& args,
                         const DeviceInfo& dev, int grid, cudaStream_t stream, bool* encode_ok) {
    const SplitKernel k = select_kernel(p, buf.kv8);
    if constexpr (D == 128) {
        if (k == SplitKernel::kTcgen05)
            return buf.kv8 ? launch_tc_groups<PAGED, OUTB, true>(p, buf, args, dev, grid, stream, encode_ok)
                           : launch_tc_groups<PAGED, OUTB, false>(p, buf, args, dev, grid, stream, encode_ok);
        if (k == SplitKernel::kMmaSync && buf.kv8)
            return launch_mma<128, 1, 1, PAGED, OUTB, true>(p, buf, args, dev, grid, stream, encode_ok);
    }
    if (k == SplitKernel::kMmaSync) return launch_mma_groups<D, PAGED, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
    if (buf.kv8) return launch_simt<__nv_bfloat16, __nv_fp8_e4m3, D, PAGED, OUTB>(buf, args, grid, stream);
    if (p->qkv_dtype == GQA_F32) return launch_simt<float, float, D, PAGED, OUTB>(buf, args, grid, stream);
    return launch_simt<__nv_bfloat16, __nv_bfloat16, D, PAGED, OUTB>(buf, args, grid, stream);
}

template <int D, bool OUTB>
cudaError_t launch_all(const gqa_decode_params* p, const Buffers& buf, const KernelArgs& args,
                       const DeviceInfo& dev, int grid, cudaStream_t stream, cudaEvent_t ev0,
                       cudaEvent_t ev1, bool* encode_ok) {
    cudaError_t e;
    if (ev0 && (e = cudaEventRecord(ev0, stream)) != cudaSuccess) return e;
    e = p->page_size ? launch_split<D, true, OUTB>(p, buf, args, dev, grid, stream, encode_ok)
                     : launch_split<D, false, OUTB>(p, buf, args, dev, grid, stream, encode_ok);
    if (e != cudaSuccess) return e;
    if (ev1 && (e = cudaEventRecord(ev1, stream)) != cudaSuccess) return e;
    return cudaSuccess;
}

gqa_status run(const gqa_decode_params* p, const void* q, const void* k, const void* v,
               const int32_t* seq_lens, const int32_t* block_table, float scale, void* out,
               void* workspace, size_t workspace_bytes, void* stream_ptr, void* ev0, void* ev1,
               const float* k_scale = nullptr, const float* v_scale = nullptr) {
    const bool kv8 = k_scale != nullptr;
    gqa_status st = validate_params(p);
    if (st != GQA_OK) return st;
    if (select_kernel(p, kv8) == SplitKernel::kNone) return GQA_ERR_UNSUPPORTED;
    if (p->B == 0) return GQA_OK;
    if (!q || !k || !v || !seq_lens || !out) return GQA_ERR_INVALID;
    if ((p->page_size != 0) != (block_table != nullptr)) return GQA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 8) ||
        !aligned(seq_lens, 4) || (block_table && !aligned(block_table, 4)))
        return GQA_ERR_INVALID;
    if (!(scale == scale)) return GQA_ERR_INVALID;  // NaN scale

    DeviceInfo dev;
    if ((st = device_info(&dev)) != GQA_OK) return st;
    // 8-bit caches use at most one CTA per SM, never more than the bf16 choice
    // for the same parameters, so gqa_decode_workspace_size's answer is enough.
    const int grid = kv8 ? std::min(dev.sms, grid_for(p, dev, true)) : grid_for(p, dev);
    if (grid > kMergeCounters) return GQA_ERR_UNSUPPORTED;  // one merge counter per CTA
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < workspace_for(p, grid))
        return GQA_ERR_WORKSPACE;

    const int R = p->H_Q / p->H_KV;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    KernelArgs args;
    std::memset(&args, 0, sizeof args);
    args.seq_lens = seq_lens;
    args.block_table = block_table;
    args.B = p->B;
    args.H_Q = p->H_Q;
    args.H_KV = p->H_KV;
    args.R = R;
    args.max_len = p->max_seq_len;
    args.S_max = p->page_size ? 0 : p->max_seq_len;
    args.max_blocks = p->max_blocks_per_seq;
    args.num_blocks = p->num_blocks;
    args.sl2 = scale * 1.4426950408889634f;  // log2(e): exponentials are taken base 2
    args.out = out;
    args.status = reinterpret_cast<uint32_t*>(ws);
    args.merge = reinterpret_cast<uint32_t*>(ws + kHeaderBytes);
    args.ws_o = reinterpret_cast<float*>(ws + kHeaderBytes + kMergeCounterBytes);
    args.ws_lse = reinterpret_cast<float*>(ws + kHeaderBytes + kMergeCounterBytes + ws_o_bytes(p, grid));
    args.k_scale = k_scale;
    args.v_scale = v_scale;

    const Buffers buf{q, k, v, kv8};
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    cudaEvent_t e0 = static_cast<cudaEvent_t>(ev0), e1 = static_cast<cudaEvent_t>(ev1);
    bool encode_ok = true;
    cudaError_t e;
    const bool outb = p->out_dtype == GQA_BF16;
    if (p->head_dim == 64)
        e = outb ? launch_all<64, true>(p, buf, args, dev, grid, stream, e0, e1, &encode_ok)
                 : launch_all<64, false>(p, buf, args, dev, grid, stream, e0, e1, &encode_ok);
    else
        e = outb ? launch_all<128, true>(p, buf, args, dev, grid, stream, e0, e1, &encode_ok)
                 : launch_all<128, false>(p, buf, args, dev, grid, stream, e0, e1, &encode_ok);
    if (!encode_ok) return GQA_ERR_INVALID;
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// ------------------------------------------------------------------ fixed workspace
//
// Storage for gqa_decode_static_workspace: a workspace that lives in the
// library itself, for callers that cannot call cudaMalloc.  Every GPU that
// loads this library holds these bytes until the process exits.  Host code
// must never hand this name to a kernel: on the host it is only a stand-in,
// and the device address comes from cudaGetSymbolAddress below.
constexpr size_t kStaticWorkspaceBytes = size_t(8) << 20;  // 8 MiB
static_assert(kStaticWorkspaceBytes == GQA_STATIC_WORKSPACE_BYTES,
              "the built-in workspace and the header's stated limit must agree");
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of g_static_workspace on the current device, looked up once
// per device with that device current; its header and merge counters are
// cleared then.
gqa_status static_workspace_on_current_device(void** ptr, cudaStream_t stream) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
            return GQA_ERR_CUDA;
        // status word, merge epoch and merge counters start at zero
        if (cudaMemsetAsync(p, 0, kHeaderBytes + kMergeCounterBytes, stream) != cudaSuccess) return GQA_ERR_CUDA;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    return GQA_OK;
}

// ------------------------------------------------------------------ RoPE + append

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

template <typename T>
cudaError_t launch_rope(const void* q, const void* k_new, const void* v_new, void* q_out, void* k_cache,
                        void* v_cache, const RopeArgs& ra, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(ra.B) * (ra.H_Q + ra.H_KV);
    const int blocks = static_cast<int>((rows + 3) / 4);
    return launch_chained(rope_append_kernel<T>, blocks, 128, 0, stream, static_cast<const T*>(q),
                          static_cast<const T*>(k_new), static_cast<const T*>(v_new), static_cast<T*>(q_out),
                          static_cast<T*>(k_cache), static_cast<T*>(v_cache), ra);
}

// ------------------------------------------------------------------ multi-token (prefill)

template <bool PAGED, bool OUTB>
cudaError_t launch_prefill(const gqa_decode_params* p, const void* q, const void* k, const void* v,
                           const PrefillArgs& args, int grid, cudaStream_t stream, bool* encode_ok) {
    constexpr int D = 128;
    const uint64_t row = static_cast<uint64_t>(D) * 2;
    CUtensorMap tmQ, tmK, tmV;
    {
        // q [total_q, H_Q, D]: box = 64 d x R heads x TQ tokens, rows token-major
        const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(p->H_Q),
                                  static_cast<uint64_t>(args.total_q)};
        const uint64_t strides[2] = {row, row * p->H_Q};
        const uint32_t box[3] = {64, static_cast<uint32_t>(args.R), static_cast<uint32_t>(args.TQ)};
        *encode_ok = encode_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, 3, dims, strides, box);
    }
    if (*encode_ok) {
        uint64_t dims[4], strides[3];
        dims[0] = D;
        dims[1] = p->H_KV;
        strides[0] = row;
        strides[1] = row * p->H_KV;
        if (PAGED) {
            dims[2] = kTile;
            dims[3] = p->num_blocks;
        } else {
            dims[2] = p->max_seq_len > 0 ? p->max_seq_len : 1;
            dims[3] = p->B;
        }
        strides[2] = strides[1] * dims[2];
        const uint32_t box4[4] = {64, 1, static_cast<uint32_t>(kTile), 1};
        *encode_ok = encode_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, 4, dims, strides, box4) &&
                     encode_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, 4, dims, strides, box4);
    }
    if (!*encode_ok) return cudaErrorInvalidValue;
    auto kernel = prefill_tc_kernel<PAGED, OUTB>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel), PfCfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // Plain stream order (no early launch): the kernel reads what earlier work wrote.
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(PfCfg::THREADS);
    cfg.dynamicSmemBytes = PfCfg::SMEM_BYTES;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kernel, tmQ, tmK, tmV, args);
}

}  // namespace

namespace {

// One CTA: warp 0 waits on a barrier nothing arrives on (the kernels' bounded
// wait, with the caller's limit); warp 1 optionally raises the abort flag
// after a quarter of the limit, from a loop bounded by the same clock.
__global__ void wait_selftest_kernel(uint64_t timeout_ns, int abort_early, uint32_t* flags, uint64_t* elapsed) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
    }
    fence_barrier_init();
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int* af = &abort_flag;
    if (warp == 0) {
        const uint64_t t0 = global_timer_ns();
        const bool ok = __all_sync(0xffffffffu, mbar_wait_for(smem_addr(&bar), 0u, af, timeout_ns));
        const uint64_t t1 = global_timer_ns();
        if (lane == 0) {
            if (!ok) atomicOr(flags, kFlagTimeout);
            *elapsed = t1 - t0;
        }
    } else if (abort_early && lane == 0) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < timeout_ns / 4) {
        }
        *af = 1;
    }
}

}  // namespace

extern "C" {

gqa_status gqa_decode_workspace_size(const gqa_decode_params* params, size_t* bytes) {
    if (bytes == nullptr) return GQA_ERR_INVALID;
    gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    DeviceInfo dev;
    if ((st = device_info(&dev)) != GQA_OK) return st;
    *bytes = workspace_for(params, grid_for(params, dev));
    return GQA_OK;
}

gqa_status gqa_decode(const gqa_decode_params* params, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, const int32_t* block_table,
                      float scale, void* out, void* workspace, size_t workspace_bytes,
                      void* stream) {
    return run(params, q, k_cache, v_cache, seq_lens, block_table, scale, out, workspace,
               workspace_bytes, stream, nullptr, nullptr);
}

gqa_status gqa_decode_fp8kv(const gqa_decode_params* params, const void* q, const void* k_cache,
                            const void* v_cache, const float* k_scale, const float* v_scale,
                            const int32_t* seq_lens, const int32_t* block_table, float scale, void* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
    gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    if (params->B == 0) return GQA_OK;
    if (params->qkv_dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;  // q is bf16 on this path
    if (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4)) return GQA_ERR_INVALID;
    return run(params, q, k_cache, v_cache, seq_lens, block_table, scale, out, workspace,
               workspace_bytes, stream, nullptr, nullptr, k_scale, v_scale);
}

gqa_status gqa_decode_timed(const gqa_decode_params* params, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens,
                            const int32_t* block_table, float scale, void* out, void* workspace,
                            size_t workspace_bytes, void* stream, void* split_begin,
                            void* split_end) {
    return run(params, q, k_cache, v_cache, seq_lens, block_table, scale, out, workspace,
               workspace_bytes, stream, split_begin, split_end);
}

gqa_status gqa_decode_static_workspace(const gqa_decode_params* params, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* seq_lens, const int32_t* block_table,
                                       float scale, void* out, void* stream) {
    gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    if (params->B == 0) return GQA_OK;
    DeviceInfo dev;
    if ((st = device_info(&dev)) != GQA_OK) return st;
    if (workspace_for(params, grid_for(params, dev)) > kStaticWorkspaceBytes) return GQA_ERR_WORKSPACE;
    void* ws = nullptr;
    if ((st = static_workspace_on_current_device(&ws, static_cast<cudaStream_t>(stream))) != GQA_OK)
        return st;
    return run(params, q, k_cache, v_cache, seq_lens, block_table, scale, out, ws,
               kStaticWorkspaceBytes, stream, nullptr, nullptr);
}

gqa_status gqa_static_workspace_status(void* stream, uint32_t* flags, int clear) {
    if (flags == nullptr) return GQA_ERR_INVALID;
    void* ws = nullptr;
    const gqa_status st = static_workspace_on_current_device(&ws, static_cast<cudaStream_t>(stream));
    if (st != GQA_OK) return st;
    return gqa_read_status(ws, stream, flags, clear);
}

gqa_status gqa_rope_append(const gqa_decode_params* params, const void* q, const void* k_new,
                           const void* v_new, const int32_t* positions, const int32_t* block_table,
                           double rope_base, int pairing, void* q_out, void* k_cache, void* v_cache,
                           int32_t* seq_lens_out, void* workspace, void* stream) {
    gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    if (params->B == 0) return GQA_OK;
    if (!q || !k_new || !v_new || !positions || !q_out || !k_cache || !v_cache) return GQA_ERR_INVALID;
    if ((params->page_size != 0) != (block_table != nullptr)) return GQA_ERR_INVALID;
    if (!(rope_base > 0.0) || rope_base > 1e300 || (pairing != GQA_ROPE_ADJACENT && pairing != GQA_ROPE_HALVES))
        return GQA_ERR_INVALID;
    const void* bufs[] = {q, k_new, v_new, q_out, k_cache, v_cache};
    for (const void* p : bufs)
        if (!aligned(p, 16)) return GQA_ERR_INVALID;
    if (!aligned(positions, 4) || (seq_lens_out && !aligned(seq_lens_out, 4)) ||
        (block_table && !aligned(block_table, 4)))
        return GQA_ERR_INVALID;
    const size_t lens_bytes = sizeof(int32_t) * static_cast<size_t>(params->B);
    if (seq_lens_out && ranges_overlap(seq_lens_out, lens_bytes, positions, lens_bytes)) return GQA_ERR_INVALID;
    if (workspace && !aligned(workspace, 256)) return GQA_ERR_WORKSPACE;

    RopeArgs ra;
    std::memset(&ra, 0, sizeof ra);
    ra.B = params->B;
    ra.H_Q = params->H_Q;
    ra.H_KV = params->H_KV;
    ra.D = params->head_dim;
    ra.max_len = params->page_size ? params->max_blocks_per_seq * kTile : params->max_seq_len;
    if (params->page_size && params->max_seq_len < ra.max_len) ra.max_len = params->max_seq_len;
    ra.S_max = params->page_size ? 0 : params->max_seq_len;
    ra.max_blocks = params->max_blocks_per_seq;
    ra.num_blocks = params->num_blocks;
    ra.positions = positions;
    ra.block_table = block_table;
    ra.seq_lens_out = seq_lens_out;
    ra.status = static_cast<uint32_t*>(workspace);
    ra.log2_base = std::log2(rope_base);
    ra.halves = pairing == GQA_ROPE_HALVES;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = params->qkv_dtype == GQA_F32
                              ? launch_rope<float>(q, k_new, v_new, q_out, k_cache, v_cache, ra, s)
                              : launch_rope<__nv_bfloat16>(q, k_new, v_new, q_out, k_cache, v_cache, ra, s);
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

gqa_status gqa_prefill_workspace_size(const gqa_decode_params* params, size_t* bytes) {
    if (bytes == nullptr) return GQA_ERR_INVALID;
    const gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    *bytes = kHeaderBytes;
    return GQA_OK;
}

gqa_status gqa_prefill(const gqa_decode_params* params, const void* q, const int32_t* cu_q_lens, int32_t total_q,
                       int32_t max_q_len, const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                       const int32_t* block_table, float scale, void* out, void* workspace,
                       size_t workspace_bytes, void* stream) {
    gqa_status st = validate_params(params);
    if (st != GQA_OK) return st;
    const gqa_decode_params* p = params;
    if (p->head_dim != 128 || p->qkv_dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
    if (p->kernel == GQA_KERNEL_MMA_SYNC) return GQA_ERR_UNSUPPORTED;
    const int R = p->H_Q / p->H_KV;
    if (R > 128) return GQA_ERR_UNSUPPORTED;  // one tile row per head of a token at least
    if (total_q < 0 || max_q_len < 0) return GQA_ERR_INVALID;
    if (p->B == 0 || total_q == 0 || max_q_len == 0) return GQA_OK;
    if (!q || !cu_q_lens || !k_cache || !v_cache || !seq_lens || !out) return GQA_ERR_INVALID;
    if ((p->page_size != 0) != (block_table != nullptr)) return GQA_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(cu_q_lens, 4) || !aligned(seq_lens, 4) || (block_table && !aligned(block_table, 4)))
        return GQA_ERR_INVALID;
    if (!(scale > 0.f) || !std::isfinite(scale)) return GQA_ERR_INVALID;  // a positive scale keeps the score order
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < kHeaderBytes) return GQA_ERR_WORKSPACE;

    const int TQ = 128 / R;  // query tokens per 128-row tile; a unit is two tiles
    const int64_t QT = (static_cast<int64_t>(max_q_len) + 2 * TQ - 1) / (2 * TQ);
    const int64_t units = static_cast<int64_t>(p->B) * p->H_KV * QT;
    if (units >= (int64_t(1) << 31)) return GQA_ERR_UNSUPPORTED;
    DeviceInfo dev;
    if ((st = device_info(&dev)) != GQA_OK) return st;
    if (dev.smem_optin < PfCfg::SMEM_BYTES) return GQA_ERR_UNSUPPORTED;
    const int grid = static_cast<int>(units < dev.sms ? units : dev.sms);

    PrefillArgs args;
    std::memset(&args, 0, sizeof args);
    args.seq_lens = seq_lens;
    args.cu_q = cu_q_lens;
    args.block_table = block_table;
    args.B = p->B;
    args.H_Q = p->H_Q;
    args.H_KV = p->H_KV;
    args.R = R;
    args.TQ = TQ;
    args.QT = static_cast<int>(QT);
    args.max_q = max_q_len;
    args.total_q = total_q;
    args.max_len = p->max_seq_len;
    args.S_max = p->page_size ? 0 : p->max_seq_len;
    args.max_blocks = p->max_blocks_per_seq;
    args.num_blocks = p->num_blocks;
    args.sl2 = scale * 1.4426950408889634f;  // log2(e): exponentials are taken base 2
    args.out = out;
    args.status = static_cast<uint32_t*>(workspace);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bool encode_ok = true;
    const bool outb = p->out_dtype == GQA_BF16;
    cudaError_t e;
    if (p->page_size)
        e = outb ? launch_prefill<true, true>(p, q, k_cache, v_cache, args, grid, s, &encode_ok)
                 : launch_prefill<true, false>(p, q, k_cache, v_cache, args, grid, s, &encode_ok);
    else
        e = outb ? launch_prefill<false, true>(p, q, k_cache, v_cache, args, grid, s, &encode_ok)
                 : launch_prefill<false, false>(p, q, k_cache, v_cache, args, grid, s, &encode_ok);
    if (!encode_ok) return GQA_ERR_INVALID;
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

gqa_status gqa_read_status(const void* workspace, void* stream, uint32_t* flags, int clear) {
    if (workspace == nullptr || flags == nullptr) return GQA_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t host = 0;
    if (cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GQA_ERR_CUDA;
    if (clear) {
        if (cudaMemsetAsync(const_cast<void*>(workspace), 0, sizeof host, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return GQA_ERR_CUDA;
    }
    *flags = host;
    return GQA_OK;
}

uint64_t gqa_kv_cache_bytes(int64_t layers, int64_t tokens, int64_t H_KV, int64_t head_dim,
                            int64_t elem_bytes) {
    if (layers < 0 || tokens < 0 || H_KV < 0 || head_dim < 0 || elem_bytes < 0) return 0;
    return 2ull * static_cast<uint64_t>(layers) * static_cast<uint64_t>(tokens) *
           static_cast<uint64_t>(H_KV) * static_cast<uint64_t>(head_dim) *
           static_cast<uint64_t>(elem_bytes);
}

const char* gqa_status_string(gqa_status status) {
    switch (status) {
        case GQA_OK: return "ok";
        case GQA_ERR_INVALID: return "invalid argument";
        case GQA_ERR_UNSUPPORTED: return "unsupported configuration";
        case GQA_ERR_CUDA: return "CUDA error";
        case GQA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

gqa_status gqa_wait_selftest(uint64_t timeout_ns, int abort_early, uint32_t* flags, uint64_t* elapsed_ns,
                             void* stream) {
    if (timeout_ns < 1000 || timeout_ns > 10000000000ull) return GQA_ERR_INVALID;
    if (flags == nullptr || elapsed_ns == nullptr || !aligned(flags, 4) || !aligned(elapsed_ns, 8))
        return GQA_ERR_INVALID;
    wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns, abort_early, flags,
                                                                         elapsed_ns);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int gqa_version(void) { return GQA_DECODE_VERSION; }

}  // extern "C"

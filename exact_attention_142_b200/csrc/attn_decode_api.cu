// attn_decode_api.cu -- C ABI of the key/value-cache decode (declared in
// attn.h): argument validation, the choice of cache slices and head chunks,
// TMA tensor maps over the caches, and the launches of the slice kernel and of
// the merge kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <numeric>

#include "attn.h"
#include "attn_decode_kernel.cuh"
#include "attn_internal.h"

namespace {

constexpr int kStagesTma128 = 3;  // 32 KB of K + V per stage at d = 128
constexpr int kStagesTma64 = 6;   // 16 KB per stage at d = 64
constexpr int kCtasPerSm = 2;     // both split kernels fit two CTAs per SM
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) ==
                cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// A cache [rows = num_pages * page_size, Hkv * d] bf16 read in boxes of
// box_rows rows x 64 columns (128 bytes) with the 128-byte swizzle; rows
// outside the cache read as zero.
bool make_cache_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estride[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device one-time set-up: compute capability 10.0 and the dynamic
// shared-memory opt-in of every decode kernel instance.
constexpr int kMaxDevices = 64;
int g_ready[kMaxDevices];  // 0 = not yet, 1 = ready, -1 = unsupported device
std::mutex g_mu;

int prepare_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_ready[dev] == 1) return ATTN_OK;
    if (g_ready[dev] == -1) return ATTN_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (major != 10 || minor != 0) {
        g_ready[dev] = -1;
        return ATTN_ERR_UNSUPPORTED;
    }
    using namespace attn::decode;
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    const int g64 = GatherSmem<64>::kBytes, g128 = GatherSmem<128>::kBytes;
    if (cudaFuncSetAttribute(attn_decode_tma<128, kStagesTma128>, a,
                             TmaSmem<128, kStagesTma128>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_tma<64, kStagesTma64>, a,
                             TmaSmem<64, kStagesTma64>::kBytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<64, 4>, a, g64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<64, 8>, a, g64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<64, 16>, a, g64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<128, 4>, a, g128) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<128, 8>, a, g128) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_gather<128, 16>, a, g128) != cudaSuccess)
        return ATTN_ERR_CUDA;
    g_ready[dev] = 1;
    return ATTN_OK;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();  // no device here: clear the error, assume a B200
        return 148;
    }
    return n;
}

struct DecodePlan {
    int heads_per_cta, head_chunks, rows, split_keys, splits;
};

int plan_decode(int Hq, int Hkv, int Nq, int page_size, int pages_per_seq, int num_splits,
                DecodePlan* plan) {
    using attn::decode::kKeyTile;
    using attn::decode::kMaxRows;
    const int group = Hq / Hkv;
    if (Nq > kMaxRows) return ATTN_ERR_UNSUPPORTED;
    const int hpc = std::min(group, kMaxRows / Nq);
    plan->heads_per_cta = hpc;
    plan->head_chunks = (group + hpc - 1) / hpc;
    plan->rows = Nq * hpc;
    const long long max_len = (long long)page_size * pages_per_seq;
    if (max_len > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    const long long per = (max_len + num_splits - 1) / num_splits;
    const long long keys = ((per + kKeyTile - 1) / kKeyTile) * kKeyTile;
    plan->split_keys = (int)std::max<long long>(keys, kKeyTile);
    plan->splits = (int)((max_len + plan->split_keys - 1) / plan->split_keys);
    if (plan->splits < 1) plan->splits = 1;
    return ATTN_OK;
}

size_t decode_workspace(int B, int Hq, int Nq, int d, int splits) {
    if (splits <= 1) return 0;
    const size_t rows = (size_t)B * Nq * Hq;
    return round256((size_t)splits * rows * d * 4) + round256((size_t)splits * rows * 4);
}

template <int D, int STAGES>
int launch_tma(const attn::decode::DecodeParams& p, cudaStream_t s) {
    using namespace attn::decode;
    const uint64_t rows = (uint64_t)p.num_pages * p.page_size;
    const uint64_t cols = (uint64_t)p.Hkv * D;
    CUtensorMap km, vm;
    if (!make_cache_map(&km, p.k_cache, rows, cols, (uint32_t)p.box_rows) ||
        !make_cache_map(&vm, p.v_cache, rows, cols, (uint32_t)p.box_rows))
        return ATTN_ERR_CUDA;
    const dim3 grid(p.num_splits, p.Hkv * p.head_chunks, p.B);
    attn_decode_tma<D, STAGES><<<grid, kTmaThreads, TmaSmem<D, STAGES>::kBytes, s>>>(km, vm, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D>
int launch_gather(const attn::decode::DecodeParams& p, int rows, cudaStream_t s) {
    using namespace attn::decode;
    const dim3 grid(p.num_splits, p.Hkv * p.head_chunks, p.B);
    const int smem = GatherSmem<D>::kBytes;
    if (rows <= 4)
        attn_decode_gather<D, 4><<<grid, kGatherThreads, smem, s>>>(p);
    else if (rows <= 8)
        attn_decode_gather<D, 8><<<grid, kGatherThreads, smem, s>>>(p);
    else
        attn_decode_gather<D, 16><<<grid, kGatherThreads, smem, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D>
int launch_decode(const attn::decode::DecodeParams& p, int rows, bool tma, cudaStream_t s) {
    constexpr int kStages = D == 128 ? kStagesTma128 : kStagesTma64;
    int rc = tma ? launch_tma<D, kStages>(p, s) : launch_gather<D>(p, rows, s);
    if (rc != ATTN_OK) return rc;
    if (p.num_splits > 1) {
        attn::decode::attn_decode_combine<D><<<(unsigned)((size_t)p.B * p.Nq * p.Hq), D, 0, s>>>(p);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

}  // namespace

namespace attn {
int decode_status_take(int* value) {
    if (cudaMemcpyFromSymbol(value, decode::g_decode_status, sizeof(int)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(decode::g_decode_status, &zero, sizeof(int)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}
}  // namespace attn

extern "C" int attn_decode_default_splits(int B, int Hq, int Hkv, int Nq, int max_cache_len) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || max_cache_len <= 0 || Hq % Hkv) return 1;
    DecodePlan plan;
    if (plan_decode(Hq, Hkv, Nq, max_cache_len, 1, 1, &plan) != ATTN_OK) return 1;
    // The kernels are bound by HBM, so a partly filled last wave costs little
    // as long as enough CTAs run at once to keep the copies in flight; a last
    // wave of a few long CTAs does cost (they run at one CTA's bandwidth).
    // Take the smallest slice count that gives at least half the CTA slots
    // and a last wave at least half full (or >= 4 waves, whose tail is
    // amortised).  Slices keep >= 256 keys.
    const long long slots = (long long)kCtasPerSm * sm_count();
    const long long base = (long long)B * Hkv * plan.head_chunks;
    const int cap = std::max(1, std::min(256, max_cache_len / 256));
    for (int s = 1; s <= cap; ++s) {
        const long long ctas = base * s;
        const long long last = ctas % slots;
        if (2 * ctas >= slots && (last == 0 || 2 * last >= slots || ctas >= 4 * slots)) return s;
    }
    return cap;
}

extern "C" size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int page_size,
                                              int pages_per_seq, int num_splits) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || page_size <= 0 ||
        pages_per_seq <= 0 || num_splits <= 0 || Hq % Hkv)
        return 0;
    DecodePlan plan;
    if (plan_decode(Hq, Hkv, Nq, page_size, pages_per_seq, num_splits, &plan) != ATTN_OK) return 0;
    return decode_workspace(B, Hq, Nq, d, plan.splits);
}

namespace {

// Every host-side check of attn_decode's arguments except the workspace; on
// success `plan` holds the launch plan and `need` the workspace it needs.
int validate_decode(const void* q, const void* k_cache, const void* v_cache, const void* o,
                    const float* lse, const int32_t* cache_seqlens, const int32_t* block_table,
                    int B, int Hq, int Hkv, int Nq, int d, int page_size, int pages_per_seq,
                    int num_pages, float scale, int window_left, int window_right, int num_splits,
                    DecodePlan* plan, size_t* need) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || page_size <= 0 || pages_per_seq <= 0 ||
        num_pages <= 0 || num_splits <= 0 || B > 65535)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
    if ((long long)num_pages * page_size > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    if (!block_table && (long long)num_pages < (long long)B * pages_per_seq) return ATTN_ERR_SHAPE;
    if (window_left < -1 || window_right < -1) return ATTN_ERR_WINDOW;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return ATTN_ERR_SCALE;
    if (!q || !k_cache || !v_cache || !o || !lse || !cache_seqlens) return ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    const int rc = plan_decode(Hq, Hkv, Nq, page_size, pages_per_seq, num_splits, plan);
    if (rc != ATTN_OK) return rc;
    if ((long long)Hkv * plan->head_chunks > 65535) return ATTN_ERR_SHAPE;
    *need = decode_workspace(B, Hq, Nq, d, plan->splits);
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                           float* lse, const int32_t* cache_seqlens, const int32_t* block_table,
                           int B, int Hq, int Hkv, int Nq, int d, int page_size, int pages_per_seq,
                           int num_pages, float scale, int causal, int window_left,
                           int window_right, int num_splits, void* workspace,
                           size_t workspace_bytes, struct CUstream_st* stream) {
    DecodePlan plan;
    size_t need = 0;
    int rc = validate_decode(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv,
                             Nq, d, page_size, pages_per_seq, num_pages, scale, window_left,
                             window_right, num_splits, &plan, &need);
    if (rc != ATTN_OK) return rc;
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
        return ATTN_ERR_WORKSPACE;
    rc = prepare_device();
    if (rc != ATTN_OK) return rc;

    attn::decode::DecodeParams p;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.o = o;
    p.lse = lse;
    const size_t rows = (size_t)B * Nq * Hq;
    p.part_o = need ? static_cast<float*>(workspace) : nullptr;
    p.part_lse = need ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                  round256((size_t)plan.splits * rows * d * 4))
                      : nullptr;
    p.cache_seqlens = cache_seqlens;
    p.block_table = block_table;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.group = Hq / Hkv;
    p.heads_per_cta = plan.heads_per_cta;
    p.head_chunks = plan.head_chunks;
    p.page_size = page_size;
    p.pages_per_seq = pages_per_seq;
    p.num_pages = num_pages;
    // TMA copies hold runs of keys that never cross a page: gcd(page_size, 64)
    // rows (any 64 rows for a contiguous cache); the swizzled layout needs runs
    // of a multiple of 8 rows, else the gather kernel runs.
    p.box_rows = block_table ? std::gcd(page_size, attn::decode::kKeyTile) : attn::decode::kKeyTile;
    const bool tma = p.box_rows % 8 == 0;
    p.left = window_left;
    p.right = causal ? 0 : window_right;
    p.num_splits = plan.splits;
    p.split_keys = plan.split_keys;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
    p.wait_limit_ns = kWaitLimitNs;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d == 128 ? launch_decode<128>(p, plan.rows, tma, s)
                    : launch_decode<64>(p, plan.rows, tma, s);
}

// ------------------------------------------------- decode without allocation
// attn_decode_noalloc is attn_decode for callers that must not allocate device
// memory while they run: a serving loop that commits nearly all of HBM to its
// key/value page pool at start-up and keeps a fixed footprint afterwards, or a
// latency-bound step loop, where cudaMalloc / cudaFree (which can block on and
// synchronise with the device, and fail when the pool holds the memory) or a
// framework allocator would stall or fail the step.  The slice partials live in
// the fixed array below instead of a caller-provided workspace.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_DECODE_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices];  // device address of the array, per device
std::mutex g_noalloc_mu;

// The array's address on the current device, looked up once per device (on the
// first call that needs it, with that device current).
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();  // leave no pending error for the caller's next CUDA call
            return ATTN_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                   void* o, float* lse, const int32_t* cache_seqlens,
                                   const int32_t* block_table, int B, int Hq, int Hkv, int Nq,
                                   int d, int page_size, int pages_per_seq, int num_pages,
                                   float scale, int causal, int window_left, int window_right,
                                   int num_splits, struct CUstream_st* stream) {
    // Every argument is checked, and the device is found supported, before
    // the array's address is looked up: a bad call or an unsupported device
    // returns attn_decode's own status and touches nothing.
    DecodePlan plan;
    size_t need = 0;
    int rc = validate_decode(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv,
                             Nq, d, page_size, pages_per_seq, num_pages, scale, window_left,
                             window_right, num_splits, &plan, &need);
    if (rc != ATTN_OK) return rc;
    if (need > (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_WORKSPACE;
    rc = prepare_device();
    if (rc != ATTN_OK) return rc;
    void* scratch = nullptr;
    if (need > 0) {
        rc = noalloc_scratch(&scratch);
        if (rc != ATTN_OK) return rc;
    }
    // Every scratch entry the merge kernel reads is written by the slice kernel
    // of the same call, so nothing left by an earlier call needs clearing.
    return attn_decode(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv, Nq, d,
                       page_size, pages_per_seq, num_pages, scale, causal, window_left,
                       window_right, num_splits, scratch,
                       need > 0 ? (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES : 0, stream);
}

extern "C" size_t attn_decode_noalloc_scratch_bytes(void) {
    return (size_t)ATTN_DECODE_NOALLOC_SCRATCH_BYTES;
}

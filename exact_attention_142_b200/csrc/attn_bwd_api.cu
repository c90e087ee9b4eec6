// attn_bwd_api.cu -- C ABI of the attention backward pass (declared in attn.h):
// argument validation, TMA tensor maps, and the launches of the D kernel, the
// dK/dV kernel and the dQ kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "attn_bwd_kernel.cuh"
#include "attn_internal.h"

namespace {

constexpr int kStages128 = 4;  // 64-row Q + dO (dK/dV kernel) or K + V (dQ kernel): 32 KB per stage
constexpr int kStages64 = 8;
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

// [rows, cols] bf16 in boxes of box_rows rows x 64 columns (128 bytes),
// 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
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

constexpr int kMaxDevices = 64;
int g_ready[kMaxDevices];  // 0 = not yet, 1 = ready, -1 = unsupported device
std::mutex g_mu;

template <int D, int S>
bool set_smem() {
    using namespace attn::bwd;
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    return cudaFuncSetAttribute(attn_bwd_dkv<D, S>, a, (int)DkvLayout<D, S>::kDynamicBytes) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_dq<D, S>, a, (int)DqLayout<D, S>::kDynamicBytes) == cudaSuccess;
}

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
    if (!set_smem<128, kStages128>() || !set_smem<64, kStages64>()) return ATTN_ERR_CUDA;
    g_ready[dev] = 1;
    return ATTN_OK;
}

// Maps with 128-row boxes (the stationary tiles) and 64-row boxes (the streamed steps).
struct Maps {
    CUtensorMap q, k, v, dout, q64, k64, v64, dout64;
};

template <int D, int S>
int launch(const Maps& m, const attn::bwd::BwdParams& p, long long tokens, cudaStream_t s) {
    using namespace attn::bwd;
    const long long rows = tokens * p.Hq;
    long long dblocks = (rows + 7) / 8;
    if (dblocks > 148 * 64) dblocks = 148 * 64;
    if (dblocks < 1) dblocks = 1;
    attn_bwd_dsum<D><<<(unsigned)dblocks, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const unsigned dkv_grid = (unsigned)((long long)p.n_blocks * p.B * p.Hkv);
    attn_bwd_dkv<D, S><<<dkv_grid, kThreads, DkvLayout<D, S>::kDynamicBytes, s>>>(m.q64, m.k, m.v, m.dout64, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    const unsigned dq_grid = (unsigned)((long long)p.n_blocks * p.B * p.Hq);
    attn_bwd_dq<D, S><<<dq_grid, kThreads, DqLayout<D, S>::kDynamicBytes, s>>>(m.q, m.k64, m.v64, m.dout, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

namespace attn {
int bwd_status_take(int* value) {
    if (cudaMemcpyFromSymbol(value, bwd::g_bwd_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(bwd::g_bwd_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    return ATTN_OK;
}
}  // namespace attn

extern "C" size_t attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed) {
    (void)d;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || Hq % Hkv) return 0;
    const size_t tokens = packed ? (size_t)N : (size_t)B * N;
    return round256(tokens * Hq * 4);  // D, laid out like lse
}

extern "C" int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                        int d, float scale, int causal, int window_left, int window_right,
                        const int32_t* cu_seqlens, int max_seqlen, void* workspace,
                        size_t workspace_bytes, struct CUstream_st* stream) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || Hq % Hkv != 0) return ATTN_ERR_SHAPE;
    if (window_left < -1 || window_right < -1) return ATTN_ERR_WINDOW;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return ATTN_ERR_SCALE;
    const long long tokens = cu_seqlens ? (long long)N : (long long)B * N;
    if (tokens > 0x7fffffffLL || (long long)Hq * d > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    if (cu_seqlens && max_seqlen < 0) return ATTN_ERR_SHAPE;
    if (N == 0) return ATTN_OK;
    if (cu_seqlens && max_seqlen == 0) return ATTN_ERR_SHAPE;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    const size_t need = attn_bwd_workspace_bytes(B, Hq, Hkv, N, d, cu_seqlens != nullptr);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;
    int rc = prepare_device();
    if (rc != ATTN_OK) return rc;

    Maps mp;
    const uint64_t T = (uint64_t)tokens, cq = (uint64_t)Hq * d, ck = (uint64_t)Hkv * d;
    if (!make_map(&mp.q, q, T, cq, 128) || !make_map(&mp.k, k, T, ck, 128) ||
        !make_map(&mp.v, v, T, ck, 128) || !make_map(&mp.dout, dout, T, cq, 128) ||
        !make_map(&mp.q64, q, T, cq, 64) || !make_map(&mp.k64, k, T, ck, 64) ||
        !make_map(&mp.v64, v, T, ck, 64) || !make_map(&mp.dout64, dout, T, cq, 64))
        return ATTN_ERR_CUDA;

    attn::bwd::BwdParams p;
    p.o = o;
    p.dout = dout;
    p.lse = lse;
    p.dsum = static_cast<float*>(workspace);
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.cu_seqlens = cu_seqlens;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.group = Hq / Hkv;
    p.left = window_left;
    p.right = causal ? 0 : window_right;
    const int longest = cu_seqlens ? max_seqlen : N;
    p.n_blocks = (longest + attn::bwd::kBM - 1) / attn::bwd::kBM;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
    p.wait_limit_ns = kWaitLimitNs;
    if ((long long)p.n_blocks * B * Hq > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d == 128 ? launch<128, kStages128>(mp, p, tokens, s) : launch<64, kStages64>(mp, p, tokens, s);
}

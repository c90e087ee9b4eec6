// attn_api.cu -- C ABI of the fused attention forward (declared in attn.h):
// argument validation, TMA tensor-map encoding, launch configuration, the
// host-buffer variant, and the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_fwd_fp8_kernel.cuh"
#include "attn_fwd_kernel.cuh"
#include "attn_internal.h"

namespace {

using attn::FwdParams;

constexpr int kStages128 = 4;  // K/V ring depth at d = 128 (32 KB per slot; 5 ran no faster, 4 leave room for the output staging)
constexpr int kStages64 = 8;   // at d = 64 (16 KB per slot)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

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

// [rows, cols] bf16, row stride cols * 2 bytes; boxes of box_rows rows x 64
// columns (128 bytes) with 128-byte swizzling: 128 rows for the Q, K, V loads
// (rows past the end read as zero), 32 for the output stores of one warp.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows = 128) {
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

// [rows, cols] one-byte elements in boxes of 128 rows x 128 bytes, 128-byte
// swizzle (the e4m3 tiles); rows past the end read as zero.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estride[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;
struct DeviceState {
    int checked = 0;  // 1 = supported, -1 = unsupported
    bool smem_set64 = false, smem_set128 = false, smem_set_fp8 = false;
};
DeviceState g_devices[kMaxDevices];
std::mutex g_dev_mu;

// Checks the current device (sm_100) and prepares the kernels' shared-memory
// limit once per device.
int prepare_device(int d) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceState& st = g_devices[dev];
    if (st.checked == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return ATTN_ERR_CUDA;
        st.checked = (major == 10 && minor == 0) ? 1 : -1;
    }
    if (st.checked < 0) return ATTN_ERR_UNSUPPORTED;
    if (d == 128 && !st.smem_set128) {
        const int bytes = (int)attn::SmemLayout<128, kStages128>::kDynamicBytes;
        if (cudaFuncSetAttribute(attn::attn_fwd_sm100<128, kStages128, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess ||
            cudaFuncSetAttribute(attn::attn_fwd_sm100<128, kStages128, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return ATTN_ERR_CUDA;
        st.smem_set128 = true;
    }
    if (d == 8 && !st.smem_set_fp8) {  // d == 8: the e4m3 kernel
        if (cudaFuncSetAttribute(attn::fp8::attn_fwd_fp8_sm100, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)attn::fp8::Layout::kDynamicBytes) != cudaSuccess)
            return ATTN_ERR_CUDA;
        st.smem_set_fp8 = true;
    }
    if (d == 64 && !st.smem_set64) {
        const int bytes = (int)attn::SmemLayout<64, kStages64>::kDynamicBytes;
        if (cudaFuncSetAttribute(attn::attn_fwd_sm100<64, kStages64, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess ||
            cudaFuncSetAttribute(attn::attn_fwd_sm100<64, kStages64, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return ATTN_ERR_CUDA;
        st.smem_set64 = true;
    }
    return ATTN_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host-side checks shared by both entry points.  `tokens` is set to the
// number of packed tokens (B * N in dense mode).
int validate(const void* q, const void* k, const void* v, const void* o, const float* lse, int B,
             int Hq, int Hkv, int N, int d, float scale, int window_left, int window_right,
             bool packed, int max_seqlen, long long* tokens) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0) return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
    if (window_left < -1 || window_right < -1) return ATTN_ERR_WINDOW;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return ATTN_ERR_SCALE;
    const long long t = packed ? (long long)N : (long long)B * N;
    if (t > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    if ((long long)Hq * d > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    if (packed && N > 0 && max_seqlen <= 0) return ATTN_ERR_SHAPE;
    *tokens = t;
    if (t == 0) return ATTN_OK;
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    return ATTN_OK;
}

// One CTA per tile pair; running CTAs take over the pairs of CTAs that have
// not started (the kernel's persistent schedule), so only about one CTA per
// SM ever runs.
template <int D, int STAGES, bool ACC>
int launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
           const FwdParams& p, long long units, cudaStream_t stream) {
    attn::attn_fwd_sm100<D, STAGES, ACC><<<(unsigned)units, attn::kThreads,
                                            attn::SmemLayout<D, STAGES>::kDynamicBytes, stream>>>(mq, mk, mv, mo, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

namespace {

// The forward pass; acc selects the accumulating epilogue (o is then fp32).
int run_fwd(bool acc, const void* q, const void* k, const void* v, void* o, float* lse, int B,
            int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
            int window_right, const int32_t* cu_seqlens, int max_seqlen, cudaStream_t s) {
    const bool packed = cu_seqlens != nullptr;
    long long tokens = 0;
    int rc = validate(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, window_left, window_right, packed,
                      max_seqlen, &tokens);
    if (rc != ATTN_OK) return rc;
    if (tokens == 0) return ATTN_OK;
    rc = prepare_device(d);
    if (rc != ATTN_OK) return rc;

    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, (uint64_t)tokens, (uint64_t)Hq * d) ||
        !make_map(&mk, k, (uint64_t)tokens, (uint64_t)Hkv * d) ||
        !make_map(&mv, v, (uint64_t)tokens, (uint64_t)Hkv * d) ||
        // O, stored per warp; the accumulating epilogue (fp32 o) does not use it
        !make_map(&mo, acc ? q : o, (uint64_t)tokens, (uint64_t)Hq * d, 32))
        return ATTN_ERR_CUDA;

    FwdParams p;
    p.o = o;
    p.lse = lse;
    p.cu_seqlens = cu_seqlens;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.group = Hq / Hkv;
    p.left = window_left;
    p.right = causal ? 0 : window_right;
    p.pair_mode = (p.group % 2 == 0) ? attn::kPairHeads : attn::kPairRows;
    const int max_len = packed ? (max_seqlen < N ? max_seqlen : N) : N;
    p.n_row_blocks = (max_len + attn::kBM - 1) / attn::kBM;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
    p.wait_limit_ns = kWaitLimitNs;

    const long long units = p.pair_mode == attn::kPairHeads
                                ? (long long)p.n_row_blocks * B * (Hq / 2)
                                : (long long)((p.n_row_blocks + 1) / 2) * B * Hq;
    if (units <= 0) return ATTN_OK;
    if (units > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    if (acc)
        return d == 128 ? launch<128, kStages128, true>(mq, mk, mv, mo, p, units, s)
                        : launch<64, kStages64, true>(mq, mk, mv, mo, p, units, s);
    return d == 128 ? launch<128, kStages128, false>(mq, mk, mv, mo, p, units, s)
                    : launch<64, kStages64, false>(mq, mk, mv, mo, p, units, s);
}

}  // namespace

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                        int window_right, const int32_t* cu_seqlens, int max_seqlen,
                        struct CUstream_st* stream) {
    return run_fwd(false, q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window_left,
                   window_right, cu_seqlens, max_seqlen, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc,
                                   float* lse_acc, int B, int Hq, int Hkv, int N, int d,
                                   float scale, int causal, int window_left, int window_right,
                                   const int32_t* cu_seqlens, int max_seqlen,
                                   struct CUstream_st* stream) {
    return run_fwd(true, q, k, v, o_acc, lse_acc, B, Hq, Hkv, N, d, scale, causal, window_left,
                   window_right, cu_seqlens, max_seqlen, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// fp32 accumulator -> bf16 (round to nearest even), 8 values per thread.
__global__ void acc_to_bf16_kernel(const float* in, uint16_t* out, long long n) {
    const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (i + 8 <= n) {
        const float4 a = *reinterpret_cast<const float4*>(in + i);
        const float4 b = *reinterpret_cast<const float4*>(in + i + 4);
        uint4 r;
        r.x = attn::ptx::pack_bf16x2(a.x, a.y);
        r.y = attn::ptx::pack_bf16x2(a.z, a.w);
        r.z = attn::ptx::pack_bf16x2(b.x, b.y);
        r.w = attn::ptx::pack_bf16x2(b.z, b.w);
        *reinterpret_cast<uint4*>(out + i) = r;
    } else {
        for (long long j = i; j < n; ++j)
            out[j] = static_cast<uint16_t>(attn::ptx::pack_bf16x2(in[j], 0.0f) & 0xffffu);
    }
}

}  // namespace

extern "C" int attn_acc_to_bf16(const float* o_acc, void* o, long long n, struct CUstream_st* stream) {
    if (n < 0) return ATTN_ERR_SHAPE;
    if (n == 0) return ATTN_OK;
    if (!o_acc || !o) return ATTN_ERR_NULL;
    if (!aligned(o_acc, 16) || !aligned(o, 16)) return ATTN_ERR_ALIGN;
    const long long threads = (n + 7) / 8;
    const long long blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    acc_to_bf16_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        o_acc, static_cast<uint16_t*>(o), n);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------- e4m3 inputs
namespace {

// Columns of the padded V^T: every sequence rounded up to 128 keys fits in
// tokens + 128 * B; rounded to 16 bytes for the tensor map's row stride.
long long vt_columns(int B, long long tokens) { return (tokens + 128LL * B + 15) / 16 * 16; }

}  // namespace

extern "C" size_t attn_fwd_fp8_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d != 128 || Hq % Hkv) return 0;
    const long long tokens = packed ? (long long)N : (long long)B * N;
    return round256((size_t)Hkv * 128 * (size_t)vt_columns(B, tokens));
}

extern "C" int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                            int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                            int window_right, const int32_t* cu_seqlens, int max_seqlen,
                            void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
    const bool packed = cu_seqlens != nullptr;
    long long tokens = 0;
    int rc = validate(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, window_left, window_right, packed,
                      max_seqlen, &tokens);
    if (rc != ATTN_OK) return rc;
    if (d != 128) return ATTN_ERR_UNSUPPORTED;
    if (tokens == 0) return ATTN_OK;
    if (B > 65535) return ATTN_ERR_SHAPE;
    const size_t need = attn_fwd_fp8_workspace_bytes(B, Hq, Hkv, N, d, packed ? 1 : 0);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;
    rc = prepare_device(8);
    if (rc != ATTN_OK) return rc;
    const long long vt_cols = vt_columns(B, tokens);
    if (vt_cols > 0x7fffffffLL) return ATTN_ERR_SHAPE;

    CUtensorMap mq, mk, mvt;
    if (!make_map_u8(&mq, q, (uint64_t)tokens, (uint64_t)Hq * 128) ||
        !make_map_u8(&mk, k, (uint64_t)tokens, (uint64_t)Hkv * 128) ||
        !make_map_u8(&mvt, workspace, (uint64_t)Hkv * 128, (uint64_t)vt_cols))
        return ATTN_ERR_CUDA;

    FwdParams p;
    p.o = o;
    p.lse = lse;
    p.cu_seqlens = cu_seqlens;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.group = Hq / Hkv;
    p.left = window_left;
    p.right = causal ? 0 : window_right;
    p.pair_mode = (p.group % 2 == 0) ? attn::kPairHeads : attn::kPairRows;
    const int max_len = packed ? (max_seqlen < N ? max_seqlen : N) : N;
    p.n_row_blocks = (max_len + attn::kBM - 1) / attn::kBM;
    p.scale = scale;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
    p.wait_limit_ns = kWaitLimitNs;
    const long long units = p.pair_mode == attn::kPairHeads
                                ? (long long)p.n_row_blocks * B * (Hq / 2)
                                : (long long)((p.n_row_blocks + 1) / 2) * B * Hq;
    if (units <= 0) return ATTN_OK;
    if (units > 0x7fffffffLL || Hkv > 65535) return ATTN_ERR_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // 64-key blocks up to the longest sequence's padded length (pad columns are zeroed)
    const dim3 tgrid((unsigned)((max_len + attn::kBN - 1) / attn::kBN * (attn::kBN / 64)), (unsigned)Hkv,
                     (unsigned)B);
    attn::fp8::attn_vt_transpose_kernel<<<tgrid, 256, 0, s>>>(static_cast<const uint8_t*>(v),
                                                               static_cast<uint8_t*>(workspace), p, vt_cols);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    attn::fp8::attn_fwd_fp8_sm100<<<(unsigned)units, attn::kThreads, attn::fp8::Layout::kDynamicBytes, s>>>(
        mq, mk, mvt, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" size_t attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0) return 0;
    const size_t tokens = packed ? (size_t)N : (size_t)B * (size_t)N;
    size_t total = 0;
    total += round256(tokens * Hq * d * 2);       // q
    total += 2 * round256(tokens * Hkv * d * 2);  // k, v
    total += round256(tokens * Hq * d * 2);       // o
    total += round256(tokens * Hq * 4);           // lse
    if (packed) total += round256((size_t)(B + 1) * 4);
    return total;
}

extern "C" int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                             int window_left, int window_right, const int32_t* cu_seqlens,
                             int max_seqlen, void* workspace, size_t workspace_bytes,
                             struct CUstream_st* stream) {
    const bool packed = cu_seqlens != nullptr;
    if (packed && max_seqlen <= 0) {  // derive it from the host boundaries
        max_seqlen = 0;
        for (int b = 0; b < B; ++b) {
            const int L = cu_seqlens[b + 1] - cu_seqlens[b];
            if (L > max_seqlen) max_seqlen = L;
        }
    }
    long long tokens = 0;
    int rc = validate(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, window_left, window_right, packed,
                      max_seqlen, &tokens);
    if (rc != ATTN_OK) return rc;
    if (tokens == 0) return ATTN_OK;
    const size_t need = attn_fwd_host_workspace_bytes(B, Hq, Hkv, N, d, packed ? 1 : 0);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return ATTN_ERR_WORKSPACE;

    const size_t bq = (size_t)tokens * Hq * d * 2, bkv = (size_t)tokens * Hkv * d * 2;
    const size_t bl = (size_t)tokens * Hq * 4;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* dq = ws;
    uint8_t* dk = dq + round256(bq);
    uint8_t* dv = dk + round256(bkv);
    uint8_t* dout = dv + round256(bkv);
    uint8_t* dlse = dout + round256(bq);
    int32_t* dcu = packed ? reinterpret_cast<int32_t*>(dlse + round256(bl)) : nullptr;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(dq, q, bq, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, bkv, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, bkv, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (packed && cudaMemcpyAsync(dcu, cu_seqlens, (size_t)(B + 1) * 4, cudaMemcpyHostToDevice, s) !=
                      cudaSuccess)
        return ATTN_ERR_CUDA;
    rc = attn_fwd(dq, dk, dv, dout, reinterpret_cast<float*>(dlse), B, Hq, Hkv, N, d, scale, causal,
                  window_left, window_right, dcu, max_seqlen, stream);
    if (rc != ATTN_OK) return rc;
    if (cudaMemcpyAsync(o, dout, bq, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(lse, dlse, bl, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return ATTN_OK;
}

extern "C" const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "a required pointer is NULL";
        case ATTN_ERR_SHAPE: return "invalid sizes (B, Hq, Hkv, N, max_seqlen or Hq % Hkv)";
        case ATTN_ERR_WINDOW: return "window_left / window_right must be -1 or >= 0";
        case ATTN_ERR_UNSUPPORTED: return "unsupported head dimension (64, 128) or device (sm_100)";
        case ATTN_ERR_ALIGN: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
        case ATTN_ERR_CUDA: return "a CUDA runtime or driver call failed";
        case ATTN_ERR_SCALE: return "scale must be finite and > 0";
        case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case ATTN_ERR_DEVICE_TIMEOUT: return "a kernel wait timed out; outputs are undefined";
        case ATTN_ERR_PAGE: return "a page-table entry lies outside the cache; outputs are undefined";
        case ATTN_ERR_SEQLENS:
            return "cu_seqlens do not fit N or max_seqlen; the sequences concerned were skipped";
        default: return "unknown status";
    }
}

extern "C" int attn_device_status(void) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, attn::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    int dv = 0, bv = 0;
    if (attn::decode_status_take(&dv) != ATTN_OK) return ATTN_ERR_CUDA;
    if (attn::bwd_status_take(&bv) != ATTN_OK) return ATTN_ERR_CUDA;
    return v != ATTN_OK ? v : (dv != ATTN_OK ? dv : bv);
}

extern "C" int attn_selftest_bounded_wait(uint64_t limit_ns, struct CUstream_st* stream) {
    if (limit_ns < 1000ull) limit_ns = 1000ull;
    if (limit_ns > 2000000000ull) limit_ns = 2000000000ull;
    attn::selftest_bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_ns);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

namespace {

// y = 2^x through the forward kernels' FMA-pipe exponential, two values per
// thread (the kernels evaluate it on pairs).
__global__ void selftest_exp2_poly_kernel(const float* x, float* y, long long n) {
    const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 2;
    if (i >= n) return;
    const bool two = i + 1 < n;
    float y0, y1;
    attn::exp2_poly_pair(x[i], two ? x[i + 1] : 0.0f, y0, y1);
    y[i] = y0;
    if (two) y[i + 1] = y1;
}

}  // namespace

extern "C" int attn_selftest_exp2_poly(const float* x, float* y, long long n, struct CUstream_st* stream) {
    if (n < 0) return ATTN_ERR_SHAPE;
    if (n == 0) return ATTN_OK;
    if (!x || !y) return ATTN_ERR_NULL;
    if (!aligned(x, 4) || !aligned(y, 4)) return ATTN_ERR_ALIGN;
    const long long blocks = ((n + 1) / 2 + 255) / 256;
    if (blocks > 0x7fffffffLL) return ATTN_ERR_SHAPE;
    const int rc = prepare_device(0);
    if (rc != ATTN_OK) return rc;
    selftest_exp2_poly_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// attn_decode_api.cu -- C ABI of the key/value-cache decode (declared in
// attn.h): argument validation, the choice of cache slices and head chunks,
// and the launches of the split kernel and of the combine kernel.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "attn_decode_kernel.cuh"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

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
    using attn::decode::DecodeSmem;
    using attn::decode::attn_decode_split;
    const int b64 = DecodeSmem<64>::kBytes, b128 = DecodeSmem<128>::kBytes;
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    if (cudaFuncSetAttribute(attn_decode_split<64, 4>, a, b64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_split<64, 8>, a, b64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_split<64, 16>, a, b64) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_split<128, 4>, a, b128) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_split<128, 8>, a, b128) != cudaSuccess ||
        cudaFuncSetAttribute(attn_decode_split<128, 16>, a, b128) != cudaSuccess)
        return ATTN_ERR_CUDA;
    g_ready[dev] = 1;
    return ATTN_OK;
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

template <int D>
int launch_decode(const attn::decode::DecodeParams& p, int rows, cudaStream_t s) {
    using attn::decode::DecodeSmem;
    using attn::decode::kThreads;
    const dim3 grid(p.num_splits, p.Hkv * p.head_chunks, p.B);
    const int smem = DecodeSmem<D>::kBytes;
    if (rows <= 4)
        attn::decode::attn_decode_split<D, 4><<<grid, kThreads, smem, s>>>(p);
    else if (rows <= 8)
        attn::decode::attn_decode_split<D, 8><<<grid, kThreads, smem, s>>>(p);
    else
        attn::decode::attn_decode_split<D, 16><<<grid, kThreads, smem, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    if (p.num_splits > 1) {
        attn::decode::attn_decode_combine<D><<<(unsigned)((size_t)p.B * p.Nq * p.Hq), D, 0, s>>>(p);
        if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_default_splits(int B, int Hq, int Hkv, int Nq, int max_cache_len) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || max_cache_len <= 0 || Hq % Hkv) return 1;
    DecodePlan plan;
    if (plan_decode(Hq, Hkv, Nq, max_cache_len, 1, 1, &plan) != ATTN_OK) return 1;
    const long long base = (long long)B * Hkv * plan.head_chunks;
    const long long want = (4LL * 148 + base - 1) / base;  // about four CTAs per SM
    const long long cap = std::max(1, max_cache_len / 256);  // at least 256 keys per split
    return (int)std::max(1LL, std::min(want, cap));
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

extern "C" int attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                           float* lse, const int32_t* cache_seqlens, const int32_t* block_table,
                           int B, int Hq, int Hkv, int Nq, int d, int page_size, int pages_per_seq,
                           float scale, int causal, int window_left, int window_right,
                           int num_splits, void* workspace, size_t workspace_bytes,
                           struct CUstream_st* stream) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || page_size <= 0 || pages_per_seq <= 0 ||
        num_splits <= 0 || B > 65535)
        return ATTN_ERR_SHAPE;
    if (Hq % Hkv != 0) return ATTN_ERR_SHAPE;
    if (window_left < -1 || window_right < -1) return ATTN_ERR_WINDOW;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return ATTN_ERR_SCALE;
    if (!q || !k_cache || !v_cache || !o || !lse || !cache_seqlens) return ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGN;
    DecodePlan plan;
    int rc = plan_decode(Hq, Hkv, Nq, page_size, pages_per_seq, num_splits, &plan);
    if (rc != ATTN_OK) return rc;
    if ((long long)Hkv * plan.head_chunks > 65535) return ATTN_ERR_SHAPE;
    const size_t need = decode_workspace(B, Hq, Nq, d, plan.splits);
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
    p.left = window_left;
    p.right = causal ? 0 : window_right;
    p.num_splits = plan.splits;
    p.split_keys = plan.split_keys;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return d == 128 ? launch_decode<128>(p, plan.rows, s) : launch_decode<64>(p, plan.rows, s);
}


// attn_decode_kernel.cuh -- attention of the newest tokens against a (paged)
// key/value cache, split along the cache ("FlashAttention", ozercemkelahmet.com/
// tools/flashattention, How it works, Step 9: one new query has little
// parallelism, so the cache is cut into slices along its sequence axis, each
// slice yields a partial result, and the partials are merged; the merge is the
// same rescaling as the online softmax of Step 3 and of "Long context beyond a
// single GPU"; paged cache layouts: "Use the decoding kernels for serving").
//
// Work is HBM-bound (each cached key and value is read once and used by only
// the few query rows that share its head), so it runs on the CUDA cores:
//
//   attn_decode_split   grid (split, kv head x head chunk, sequence), 128 threads.
//       64-key tiles of K and V are gathered through the page table into
//       shared memory with a two-stage cp.async pipeline; scores of the
//       R <= 16 query rows (the Nq newest tokens of the query heads sharing the
//       key/value head; the kernel is instantiated for R <= 4, 8 and 16) are
//       computed with one thread per (key, half of d); an
//       online softmax keeps per-row max and sum; O is accumulated with one
//       thread per output column.  Each CTA writes its partial O (normalised by
//       its own sum, fp32) and partial LSE to the workspace -- or, with a single
//       split, the final bf16 O and fp32 LSE.
//   attn_decode_combine grid (rows), d threads.  O = sum_s 2^(lse_s - M) O_s /
//       sum_s 2^(lse_s - M), LSE = M + log sum_s 2^(lse_s - M).
#pragma once

#include <cstdint>

#include "attn.h"
#include "ptx.cuh"

namespace attn {
namespace decode {

constexpr int kThreads = 128;
constexpr int kKeyTile = 64;   // keys per shared-memory tile
constexpr int kMaxRows = 16;   // query rows (Nq x heads) per CTA
constexpr float kLn2f = 0.693147180559945309f;

struct DecodeParams {
    const void* q;        // [B, Nq, Hq, d] bf16
    const void* k_cache;  // [pages, page_size, Hkv, d] bf16
    const void* v_cache;
    void* o;              // [B, Nq, Hq, d] bf16   (single split)
    float* lse;           // [B, Hq, Nq] fp32      (single split)
    float* part_o;        // [splits, B, Nq, Hq, d] fp32 (several splits)
    float* part_lse;      // [splits, B, Hq, Nq] fp32
    const int32_t* cache_seqlens;  // [B]
    const int32_t* block_table;    // [B, pages_per_seq] or nullptr
    int B, Hq, Hkv, Nq, group;     // group = Hq / Hkv
    int heads_per_cta, head_chunks;
    int page_size, pages_per_seq;
    int left, right;               // -1 = unlimited; causal folded into right = 0
    int num_splits, split_keys;    // keys per split (multiple of kKeyTile)
    float scale_log2;
};

template <int D>
struct DecodeSmem {
    static constexpr int kRowPad = D + 8;  // bf16 elements per padded K/V row (16 B pad)
    static constexpr int kTileElems = kKeyTile * kRowPad;
    // K[2][tile], V[2][tile] bf16; Q[kMaxRows][D] fp32; S halves [2][kMaxRows][kKeyTile]
    // fp32 (the second half is reused for P); row stats.
    static constexpr int kBytesKV = 4 * kTileElems * 2;
    static constexpr int kBytesQ = kMaxRows * D * 4;
    static constexpr int kBytesS = 2 * kMaxRows * kKeyTile * 4;
    static constexpr int kBytesStats = 3 * kMaxRows * 4;
    static constexpr int kBytes = kBytesKV + kBytesQ + kBytesS + kBytesStats;
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
    const uint32_t dst = ptx::smem_addr(smem_dst);
    const int src_bytes = valid ? 16 : 0;  // 0: zero-fill, nothing read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Gather keys [k0, k0 + 64) of one key/value head into a padded shared tile.
template <int D>
__device__ __forceinline__ void load_tile(const DecodeParams& p, const uint16_t* cache, uint16_t* tile,
                                          int b, int g, int k0, int k_end) {
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int idx = threadIdx.x; idx < kKeyTile * kChunks; idx += kThreads) {
        const int r = idx / kChunks, c = idx % kChunks;
        const int key = k0 + r;
        const bool valid = key < k_end;
        const int kk = valid ? key : 0;
        const int lp = kk / p.page_size;
        const int page = p.block_table ? p.block_table[(size_t)b * p.pages_per_seq + lp]
                                       : b * p.pages_per_seq + lp;
        const size_t row = (size_t)page * p.page_size + kk % p.page_size;
        const uint16_t* src = cache + (row * p.Hkv + g) * D + c * 8;
        cp_async16(tile + r * DecodeSmem<D>::kRowPad + c * 8, src, valid);
    }
}

template <int D, int RMAX>
__global__ void __launch_bounds__(kThreads) attn_decode_split(const DecodeParams p) {
    static_assert(RMAX == 4 || RMAX == 8 || RMAX == 16, "row capacity");
    using SM = DecodeSmem<D>;
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* kt = reinterpret_cast<uint16_t*>(smem);            // [2][tile]
    uint16_t* vt = kt + 2 * SM::kTileElems;                      // [2][tile]
    float* qs = reinterpret_cast<float*>(smem + SM::kBytesKV);   // [kMaxRows][D]
    float* ss = qs + kMaxRows * D;                               // [2][kMaxRows][kKeyTile]
    float* ps = ss + kMaxRows * kKeyTile;                        // aliases the second half
    float* st_m = ss + 2 * kMaxRows * kKeyTile;                  // running max (log2 units)
    float* st_l = st_m + kMaxRows;                               // running sum
    float* st_a = st_l + kMaxRows;                               // this tile's correction

    const int split = blockIdx.x;
    const int g = blockIdx.y / p.head_chunks;
    const int hc = blockIdx.y % p.head_chunks;
    const int b = blockIdx.z;
    const int tid = threadIdx.x;
    // Clamped to the cache's capacity so that a bad length cannot index past the
    // page table; valid inputs satisfy Nq <= L <= page_size * pages_per_seq.
    const int L = max(0, min(p.cache_seqlens[b], p.page_size * p.pages_per_seq));
    const int h0 = g * p.group + hc * p.heads_per_cta;
    const int nh = min(p.heads_per_cta, p.group - hc * p.heads_per_cta);
    const int R = p.Nq * nh;  // rows: r = i * nh + hh

    // Keys this split may touch: its slice of the cache, cut to what any of the
    // rows can see (causal / window bounds are aligned to the cache end).
    int k_begin = split * p.split_keys;
    int k_end = min(L, k_begin + p.split_keys);
    {
        const int pos_first = L - p.Nq, pos_last = L - 1;
        if (p.left >= 0) k_begin = max(k_begin, pos_first - p.left);
        if (p.right >= 0) k_end = min(k_end, pos_last + p.right + 1);
        k_begin = max(k_begin, 0);
    }

    // Q rows (fp32) and row state.
    for (int idx = tid; idx < R * D; idx += kThreads) {
        const int r = idx / D, c = idx % D;
        const int i = r / nh, hh = r % nh;
        const uint16_t* qp = static_cast<const uint16_t*>(p.q) + (((size_t)b * p.Nq + i) * p.Hq + h0 + hh) * D;
        qs[r * D + c] = __uint_as_float(static_cast<uint32_t>(qp[c]) << 16);
    }
    if (tid < kMaxRows) {
        st_m[tid] = -INFINITY;
        st_l[tid] = 0.0f;
    }
    __syncthreads();  // row state is read by every thread, even with no tiles

    // output accumulators: D = 128 -> one column per thread, all rows;
    // D = 64 -> one column per thread, every other row.
    constexpr int kRowsPerThread = (D == 128) ? RMAX : RMAX / 2;
    const int col = tid % D;
    const int row_phase = (D == 128) ? 0 : tid / D;
    const int row_step = (D == 128) ? 1 : 2;
    float acc[kRowsPerThread];
#pragma unroll
    for (int e = 0; e < kRowsPerThread; ++e) acc[e] = 0.0f;

    const uint16_t* kc = static_cast<const uint16_t*>(p.k_cache);
    const uint16_t* vc = static_cast<const uint16_t*>(p.v_cache);
    const int ntiles = k_end > k_begin ? (k_end - k_begin + kKeyTile - 1) / kKeyTile : 0;
    if (ntiles > 0) {
        load_tile<D>(p, kc, kt, b, g, k_begin, k_end);
        load_tile<D>(p, vc, vt, b, g, k_begin, k_end);
    }
    cp_async_commit();

    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        const int k0 = k_begin + t * kKeyTile;
        if (t + 1 < ntiles) {
            load_tile<D>(p, kc, kt + (buf ^ 1) * SM::kTileElems, b, g, k0 + kKeyTile, k_end);
            load_tile<D>(p, vc, vt + (buf ^ 1) * SM::kTileElems, b, g, k0 + kKeyTile, k_end);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint16_t* ktile = kt + buf * SM::kTileElems;
        const uint16_t* vtile = vt + buf * SM::kTileElems;

        // scores: thread = (key, half of d)
        {
            const int key = tid % kKeyTile, half = tid / kKeyTile;
            float sacc[RMAX];
#pragma unroll
            for (int r = 0; r < RMAX; ++r) sacc[r] = 0.0f;
            const uint16_t* krow = ktile + key * SM::kRowPad + half * (D / 2);
#pragma unroll
            for (int c8 = 0; c8 < D / 2; c8 += 8) {
                const uint4 kv = *reinterpret_cast<const uint4*>(krow + c8);
                const float kf[8] = {bf16_lo(kv.x), bf16_hi(kv.x), bf16_lo(kv.y), bf16_hi(kv.y),
                                     bf16_lo(kv.z), bf16_hi(kv.z), bf16_lo(kv.w), bf16_hi(kv.w)};
#pragma unroll
                for (int r = 0; r < RMAX; ++r) {
                    if (r < R) {
                        const float* qr = qs + r * D + half * (D / 2) + c8;
#pragma unroll
                        for (int e = 0; e < 8; ++e) sacc[r] = fmaf(qr[e], kf[e], sacc[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RMAX; ++r)
                if (r < R) ss[(half * kMaxRows + r) * kKeyTile + key] = sacc[r];
        }
        __syncthreads();

        // online softmax per row: warp w takes rows w, w + 4, ...; lane takes keys lane, lane + 32
        {
            const int warp = tid / 32, lane = tid % 32;
            for (int r = warp; r < R; r += kThreads / 32) {
                const int i = r / nh;
                const int pos = L - p.Nq + i;
                const int lo = p.left >= 0 ? max(0, pos - p.left) : 0;
                const int hi = p.right >= 0 ? min(L - 1, pos + p.right) : L - 1;
                float x[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int key = lane + 32 * u;
                    const int kidx = k0 + key;
                    const float sv = ss[r * kKeyTile + key] + ss[(kMaxRows + r) * kKeyTile + key];
                    x[u] = (kidx >= lo && kidx <= hi && kidx < k_end) ? sv * p.scale_log2 : -INFINITY;
                }
                float mx = fmaxf(x[0], x[1]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_old = st_m[r];
                const float m_new = fmaxf(m_old, mx);
                const float m_use = m_new == -INFINITY ? 0.0f : m_new;
                const float p0 = ptx::ex2_approx(x[0] - m_use);
                const float p1 = ptx::ex2_approx(x[1] - m_use);
                float sum = p0 + p1;
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                ps[r * kKeyTile + lane] = p0;
                ps[r * kKeyTile + lane + 32] = p1;
                if (lane == 0) {
                    const float alpha = (m_old == -INFINITY) ? 0.0f : ptx::ex2_approx(m_old - m_use);
                    st_a[r] = alpha;
                    st_l[r] = st_l[r] * alpha + sum;
                    st_m[r] = m_new;
                }
            }
        }
        __syncthreads();

        // O += P V (rescaled by this tile's correction)
#pragma unroll
        for (int e = 0; e < kRowsPerThread; ++e) {
            const int r = row_phase + e * row_step;
            if (r < R) acc[e] *= st_a[r];
        }
        for (int key = 0; key < kKeyTile; ++key) {
            const float vv = __uint_as_float(static_cast<uint32_t>(vtile[key * SM::kRowPad + col]) << 16);
#pragma unroll
            for (int e = 0; e < kRowsPerThread; ++e) {
                const int r = row_phase + e * row_step;
                if (r < R) acc[e] = fmaf(ps[r * kKeyTile + key], vv, acc[e]);
            }
        }
        __syncthreads();  // before the next tile overwrites the buffers
    }
    cp_async_wait<0>();

    // write out
#pragma unroll
    for (int e = 0; e < kRowsPerThread; ++e) {
        const int r = row_phase + e * row_step;
        if (r >= R) continue;
        const int i = r / nh, hh = r % nh, h = h0 + hh;
        const float l = st_l[r];
        const float ov = l > 0.0f ? acc[e] / l : 0.0f;
        const float lse2 = l > 0.0f ? st_m[r] + ptx::lg2_approx(l) : -INFINITY;  // log2 units
        const size_t orow = ((size_t)b * p.Nq + i) * p.Hq + h;
        const size_t lrow = ((size_t)b * p.Hq + h) * p.Nq + i;
        if (p.num_splits == 1) {
            uint16_t* op = static_cast<uint16_t*>(p.o) + orow * D;
            op[col] = static_cast<uint16_t>(ptx::pack_bf16x2(ov, 0.0f) & 0xffffu);
            if (col == 0) p.lse[lrow] = lse2 * kLn2f;
        } else {
            const size_t plane = (size_t)p.B * p.Nq * p.Hq;
            p.part_o[((size_t)split * plane + orow) * D + col] = ov;
            if (col == 0) p.part_lse[(size_t)split * plane + lrow] = lse2;
        }
    }
}

// Merge the splits of one output row (d threads).
template <int D>
__global__ void __launch_bounds__(D) attn_decode_combine(const DecodeParams p) {
    const int row = blockIdx.x;  // (b, i, h) in the order of O: ((b * Nq + i) * Hq + h)
    const int h = row % p.Hq;
    const int bi = row / p.Hq;
    const int i = bi % p.Nq, b = bi / p.Nq;
    const size_t plane = (size_t)p.B * p.Nq * p.Hq;
    const size_t lrow = ((size_t)b * p.Hq + h) * p.Nq + i;
    float M = -INFINITY;
    for (int s = 0; s < p.num_splits; ++s) M = fmaxf(M, p.part_lse[s * plane + lrow]);
    float wsum = 0.0f, acc = 0.0f;
    if (M != -INFINITY) {
        for (int s = 0; s < p.num_splits; ++s) {
            const float ls = p.part_lse[s * plane + lrow];
            const float wgt = ls == -INFINITY ? 0.0f : ptx::ex2_approx(ls - M);
            wsum += wgt;
            acc = fmaf(wgt, p.part_o[(s * plane + row) * D + threadIdx.x], acc);
        }
    }
    const float ov = wsum > 0.0f ? acc / wsum : 0.0f;
    uint16_t* op = static_cast<uint16_t*>(p.o) + (size_t)row * D;
    op[threadIdx.x] = static_cast<uint16_t>(ptx::pack_bf16x2(ov, 0.0f) & 0xffffu);
    if (threadIdx.x == 0) p.lse[lrow] = wsum > 0.0f ? (M + ptx::lg2_approx(wsum)) * kLn2f : -INFINITY;
}

}  // namespace decode
}  // namespace attn

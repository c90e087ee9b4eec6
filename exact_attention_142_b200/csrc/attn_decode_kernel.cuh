// attn_decode_kernel.cuh -- attention of the newest tokens against a (paged)
// key/value cache, split along the cache ("FlashAttention", ozercemkelahmet.com/
// tools/flashattention, How it works, Step 9: one new query has little
// parallelism, so the cache is cut into slices along its sequence axis, each
// slice yields a partial result, and the partials are merged; the merge is the
// same rescaling as the online softmax of Step 3 and of "Long context beyond a
// single GPU"; paged cache layouts: "Use the decoding kernels for serving").
//
// The work is bound by HBM: every cached key and value is read once and used
// only by the R <= 16 query rows (Nq newest tokens x the query heads sharing
// one key/value head) of its CTA.  The kernels therefore aim at keeping enough
// bytes in flight, and keep the arithmetic off the critical path:
//
//   attn_decode_tma<D, STAGES>   grid (slice, kv head x head chunk, sequence),
//       5 warps.  Warp 4 gathers 64-key tiles of K and V through the page table
//       with 2-D TMA copies (128-byte swizzle) into a STAGES-deep ring; one
//       copy per run of gcd(page_size, 64) keys, so a run never crosses a page.
//       Warps 0-3 each own 16 keys of every tile and keep their own online
//       softmax: S = Q K^T and O += P V are m16n8k16 bf16 tensor-core
//       fragments (rows = query rows, zero-padded to 16; Q stays in registers
//       for the whole cache), P is rounded to bf16 for the second product.
//       At the end the four warps' (max, sum, O) are merged in shared memory.
//       Needs page_size % 8 == 0 (or a contiguous cache).
//   attn_decode_gather<D, RMAX>  the general path for any page size: cp.async
//       gathers of 16-byte pieces, CUDA-core dot products, fp32 P.
//   attn_decode_combine<D>       one CTA per output row merges the slices:
//       O = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), LSE = M + log2(sum).
//
// With one slice the split kernels write the final bf16 O and fp32 LSE;
// otherwise each writes its slice's normalised fp32 O and log2-domain LSE.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "attn.h"
#include "ptx.cuh"

namespace attn {
namespace decode {

constexpr int kKeyTile = 64;   // keys per tile (both kernels)
constexpr int kMaxRows = 16;   // query rows (Nq x heads) per CTA
constexpr float kLn2f = 0.693147180559945309f;

// Device status of the decode kernels (read and cleared by attn_device_status).
__device__ int g_decode_status;

struct DecodeParams {
    const void* q;        // [B, Nq, Hq, d] bf16
    const void* k_cache;  // [num_pages, page_size, Hkv, d] bf16
    const void* v_cache;
    void* o;              // [B, Nq, Hq, d] bf16   (single slice)
    float* lse;           // [B, Hq, Nq] fp32      (single slice)
    float* part_o;        // [slices, B, Nq, Hq, d] fp32 (several slices)
    float* part_lse;      // [slices, B, Hq, Nq] fp32, log2 units
    const int32_t* cache_seqlens;  // [B]
    const int32_t* block_table;    // [B, pages_per_seq] or nullptr
    int B, Hq, Hkv, Nq, group;     // group = Hq / Hkv
    int heads_per_cta, head_chunks;
    int page_size, pages_per_seq, num_pages;
    int box_rows;                  // keys per TMA copy (divides 64, multiple of 8)
    int left, right;               // -1 = unlimited; causal folded into right = 0
    int num_splits, split_keys;    // keys per slice (multiple of kKeyTile)
    float scale_log2;
    unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_decode_status, 0, code); }

// The rows, heads and key range one CTA works on.
struct Work {
    int b, g, h0, nh, R, L;
    int k_begin, k_end;
};

__device__ __forceinline__ Work work_of(const DecodeParams& p) {
    Work w;
    const int split = blockIdx.x;
    w.g = blockIdx.y / p.head_chunks;
    const int hc = blockIdx.y % p.head_chunks;
    w.b = blockIdx.z;
    // Clamped to the cache's capacity so that a bad length cannot index past the
    // page table; valid inputs satisfy Nq <= L <= page_size * pages_per_seq.
    w.L = max(0, min(p.cache_seqlens[w.b], p.page_size * p.pages_per_seq));
    w.h0 = w.g * p.group + hc * p.heads_per_cta;
    w.nh = min(p.heads_per_cta, p.group - hc * p.heads_per_cta);
    w.R = p.Nq * w.nh;  // rows: r = i * nh + hh
    // Keys this slice may touch, cut to what any of the rows can see (the
    // causal / window bounds are aligned to the end of the cache).
    w.k_begin = split * p.split_keys;
    w.k_end = min(w.L, w.k_begin + p.split_keys);
    const int pos_first = w.L - p.Nq, pos_last = w.L - 1;
    if (p.left >= 0) w.k_begin = max(w.k_begin, pos_first - p.left);
    if (p.right >= 0) w.k_end = min(w.k_end, pos_last + p.right + 1);
    w.k_begin = max(w.k_begin, 0);
    return w;
}

// Visible key range [lo, hi] of query row r (empty for padding rows).
__device__ __forceinline__ void row_range(const DecodeParams& p, const Work& w, int r, int& lo,
                                          int& hi) {
    if (r >= w.R) {
        lo = 1;
        hi = 0;
        return;
    }
    const int pos = w.L - p.Nq + r / w.nh;
    lo = p.left >= 0 ? max(0, pos - p.left) : 0;
    hi = p.right >= 0 ? min(w.L - 1, pos + p.right) : w.L - 1;
}

// Physical page of logical page lp of sequence b, or -1 (recorded) if the page
// table points outside the cache.
__device__ __forceinline__ int page_of(const DecodeParams& p, int b, int lp) {
    const int page = p.block_table ? p.block_table[(size_t)b * p.pages_per_seq + lp]
                                   : b * p.pages_per_seq + lp;
    if (page < 0 || page >= p.num_pages) {
        record_status(ATTN_ERR_PAGE);
        return -1;
    }
    return page;
}

// ------------------------------------------------------------ tensor-core path
constexpr int kConsumerWarps = 4;
constexpr int kTmaThreads = (kConsumerWarps + 1) * 32;

template <int D, int STAGES>
struct TmaSmem {
    static constexpr int kBoxes = D / 64;                  // 64-column (128-byte) boxes
    static constexpr int kBoxBytes = kKeyTile * 128;       // 8 KB
    static constexpr int kTileBytes = kBoxes * kBoxBytes;  // K or V of one tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kRing = STAGES * kStageBytes;
    static constexpr int kMergePitch = D + 8;              // floats; conflict-free float2 stores
    static constexpr int kMergeBytes = kConsumerWarps * kMaxRows * kMergePitch * 4;
    static_assert(kMergeBytes <= kRing, "merge buffer reuses the ring");
    static constexpr int kBars = kRing;                    // full[STAGES], empty[STAGES]
    static constexpr int kStats = kBars + 2 * STAGES * 8;  // [warp][row][m, l_f32, l_bf16]
    static constexpr int kFlag = kStats + kConsumerWarps * kMaxRows * 3 * 4;
    static constexpr int kUsed = kFlag + 16;
    static constexpr int kBytes = kUsed + 1024;            // slack for 1024-byte alignment
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// C(16x8 fp32) += A(16x16 bf16, row-major) * B(16x8 bf16, column-major)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ bool tma_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned long long limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            record_status(ATTN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

// Byte offset of 16-byte chunk `ch` (0 .. D/8-1) of tile row `row` in a K or V
// tile stored as 64-column boxes of 64 rows x 128 bytes with the 128-byte
// swizzle (chunk index XOR row % 8; each box starts on a 1024-byte boundary).
__device__ __forceinline__ uint32_t swz(int row, int ch) {
    return (ch >> 3) * (kKeyTile * 128) + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
}

template <int D, int STAGES>
__global__ void __launch_bounds__(kTmaThreads, 2)
    attn_decode_tma(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const DecodeParams p) {
    using SM = TmaSmem<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const uint32_t bar_full = sbase + SM::kBars;       // + 8 * stage
    const uint32_t bar_empty = bar_full + 8 * STAGES;  // + 8 * stage
    float* stats = reinterpret_cast<float*>(smem + SM::kStats);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SM::kFlag);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const Work w = work_of(p);
    const int t_first = w.k_begin / kKeyTile;
    const int ntiles = w.k_end > w.k_begin ? (w.k_end + kKeyTile - 1) / kKeyTile - t_first : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1);
            ptx::mbar_init(bar_empty + 8 * s, kConsumerWarps);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------ producer (TMA) warp
        if (lane == 0) {
            ptx::prefetch_tensormap(&kmap);
            ptx::prefetch_tensormap(&vmap);
        }
        const uint64_t pol = ptx::policy_evict_first();  // every byte is read once
        const int chunks = kKeyTile / p.box_rows;
        int issued = 0;
        for (int t = 0; t < ntiles; ++t) {
            const int stage = t % STAGES;
            const bool ok = tma_wait(bar_empty + 8 * stage, ((t / STAGES) & 1) ^ 1, abort_flag,
                                     p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int k0 = (t_first + t) * kKeyTile;
            // copies that hold at least one key < L; the rest of the tile is
            // never read unmasked (consumers zero V rows at and past L)
            const int nvalid = min(chunks, (w.L - k0 + p.box_rows - 1) / p.box_rows);
            const uint32_t bytes = (uint32_t)nvalid * p.box_rows * 128 * SM::kBoxes * 2;
            if (lane == 0) ptx::mbar_arrive_expect_tx(bar_full + 8 * stage, bytes);
            __syncwarp();
            const uint32_t kdst = sbase + stage * SM::kStageBytes;
            const uint32_t vdst = kdst + SM::kTileBytes;
            for (int c = lane; c < nvalid; c += 32) {
                const int key = k0 + c * p.box_rows;
                const int lp = key / p.page_size;
                const int page = page_of(p, w.b, lp);
                // an invalid page is read at rows before the tensor: zero fill
                const int y = page >= 0 ? page * p.page_size + (key - lp * p.page_size) : -p.box_rows;
                const uint32_t off = c * p.box_rows * 128;
#pragma unroll
                for (int bx = 0; bx < SM::kBoxes; ++bx) {
                    ptx::tma_load_2d(kdst + bx * SM::kBoxBytes + off, &kmap, bar_full + 8 * stage,
                                     w.g * D + bx * 64, y, pol);
                    ptx::tma_load_2d(vdst + bx * SM::kBoxBytes + off, &vmap, bar_full + 8 * stage,
                                     w.g * D + bx * 64, y, pol);
                }
            }
            ++issued;
        }
        // every copy issued must land before the block may exit
        if (lane == 0) {
            const int first = issued > STAGES ? issued - STAGES : 0;
            for (int i = first; i < issued; ++i) {
                const uint32_t bar = bar_full + 8 * (i % STAGES);
                const uint32_t par = (i / STAGES) & 1;
                const uint64_t t0 = ptx::global_timer_ns();
                while (!ptx::mbar_try_wait(bar, par)) {
                    if (ptx::global_timer_ns() - t0 > p.wait_limit_ns) {
                        record_status(ATTN_ERR_DEVICE_TIMEOUT);
                        break;
                    }
                }
            }
        }
        return;
    }

    // ---------------------------------------------------- consumer warps 0-3
    const int gq = lane >> 2, cq = lane & 3;  // fragment row group / column pair
    int lo[2], hi[2];
    row_range(p, w, gq, lo[0], hi[0]);
    row_range(p, w, gq + 8, lo[1], hi[1]);

    // Q as A fragments: qa[k-step][{row g, row g+8} x {k lo, k hi}]
    uint32_t qa[D / 16][4];
    {
        const uint32_t* q32 = static_cast<const uint32_t*>(p.q);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = gq + 8 * j;
            const bool valid = r < w.R;
            const int i = valid ? r / w.nh : 0, hh = valid ? r % w.nh : 0;
            const size_t base = ((((size_t)w.b * p.Nq + i) * p.Hq + w.h0 + hh) * D) / 2;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qa[ks][j] = valid ? q32[base + ks * 8 + cq] : 0u;
                qa[ks][j + 2] = valid ? q32[base + ks * 8 + 4 + cq] : 0u;
            }
        }
    }

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_f32[2] = {0.0f, 0.0f};   // sum of fp32 weights (for LSE)
    float l_bf16[2] = {0.0f, 0.0f};  // sum of the bf16 weights used in P V (for O)
    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;

    const int lrow = lane & 7, lmat = lane >> 3;  // ldmatrix: row within matrix, matrix
    for (int t = 0; t < ntiles; ++t) {
        const int stage = t % STAGES;
        const bool ok = tma_wait(bar_full + 8 * stage, (t / STAGES) & 1, abort_flag, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int k0 = (t_first + t) * kKeyTile;
        const int kw0 = k0 + warp * 16;  // first key of this warp
        const uint32_t kt = sbase + stage * SM::kStageBytes;
        const uint32_t vt = kt + SM::kTileBytes;

        if (kw0 + 16 > w.L) {
            // keys at and past L: their V rows hold whatever the pages hold (or
            // an earlier tile); make them zero so that 0-weight rows add 0
            for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
                const int n = idx / (D / 8), ch = idx % (D / 8);
                if (kw0 + n >= w.L) {
                    const uint32_t a = vt + swz(warp * 16 + n, ch);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u)
                                 : "memory");
                }
            }
            // order these generic writes before the next TMA write to the stage
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }

        // S = Q K^T over this warp's 16 keys (two n8 tiles)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int row = warp * 16 + (lmat >> 1) * 8 + lrow;
            const int ch = 2 * ks + (lmat & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kt + swz(row, ch), b0, b1, b2, b3);
            mma_16816(s[0], qa[ks], b0, b1);
            mma_16816(s[1], qa[ks], b2, b3);
        }

        // online softmax (log2 units); rows gq (regs 0, 1) and gq + 8 (regs 2, 3)
        float x[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = e >> 1;
                const int key = kw0 + n * 8 + 2 * cq + (e & 1);
                x[n][e] = (key >= lo[j] && key <= hi[j]) ? s[n][e] * p.scale_log2 : -INFINITY;
            }
        float m_use[2], alpha[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float mx = fmaxf(fmaxf(x[0][2 * j], x[0][2 * j + 1]), fmaxf(x[1][2 * j], x[1][2 * j + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[j], mx);
            m_use[j] = m_new == -INFINITY ? 0.0f : m_new;
            alpha[j] = ptx::ex2_approx(m_run[j] - m_use[j]);  // 0 while nothing was seen
            m_run[j] = m_new;
        }
        uint32_t pa[4];  // P as the A fragment of the second product
        float ps[2] = {0.0f, 0.0f}, pbs[2] = {0.0f, 0.0f};
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float p0 = ptx::ex2_approx(x[n][2 * j] - m_use[j]);
                const float p1 = ptx::ex2_approx(x[n][2 * j + 1] - m_use[j]);
                const uint32_t pk = ptx::pack_bf16x2(p0, p1);
                pa[2 * n + j] = pk;
                ps[j] += p0 + p1;
                pbs[j] += __uint_as_float(pk << 16) + __uint_as_float(pk & 0xffff0000u);
            }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            l_f32[j] = l_f32[j] * alpha[j] + ps[j];
            l_bf16[j] = l_bf16[j] * alpha[j] + pbs[j];
        }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            o[n][0] *= alpha[0];
            o[n][1] *= alpha[0];
            o[n][2] *= alpha[1];
            o[n][3] *= alpha[1];
        }

        // O += P V over the same 16 keys
#pragma unroll
        for (int t2 = 0; t2 < D / 16; ++t2) {
            const int row = warp * 16 + (lmat & 1) * 8 + lrow;
            const int ch = 2 * t2 + (lmat >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(vt + swz(row, ch), b0, b1, b2, b3);
            mma_16816(o[2 * t2], pa, b0, b1);
            mma_16816(o[2 * t2 + 1], pa, b2, b3);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * stage);
    }

    // ---- merge the four warps' partial softmax states
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        l_f32[j] += __shfl_xor_sync(0xffffffffu, l_f32[j], 1);
        l_f32[j] += __shfl_xor_sync(0xffffffffu, l_f32[j], 2);
        l_bf16[j] += __shfl_xor_sync(0xffffffffu, l_bf16[j], 1);
        l_bf16[j] += __shfl_xor_sync(0xffffffffu, l_bf16[j], 2);
        if (cq == 0) {
            float* st = stats + (warp * kMaxRows + gq + 8 * j) * 3;
            st[0] = m_run[j];
            st[1] = l_f32[j];
            st[2] = l_bf16[j];
        }
    }
    consumers_sync();  // stats visible; every consumer is done with the ring
    float lse2[2], factor[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int r = gq + 8 * j;
        float M = -INFINITY;
#pragma unroll
        for (int v = 0; v < kConsumerWarps; ++v) M = fmaxf(M, stats[(v * kMaxRows + r) * 3]);
        const float M_use = M == -INFINITY ? 0.0f : M;
        float Lf = 0.0f, Lb = 0.0f;
#pragma unroll
        for (int v = 0; v < kConsumerWarps; ++v) {
            const float* st = stats + (v * kMaxRows + r) * 3;
            const float sc = ptx::ex2_approx(st[0] - M_use);  // 0 for a warp that saw nothing
            Lf += sc * st[1];
            Lb += sc * st[2];
        }
        lse2[j] = Lf > 0.0f ? M + ptx::lg2_approx(Lf) : -INFINITY;
        factor[j] = Lb > 0.0f ? ptx::ex2_approx(m_run[j] - M_use) / Lb : 0.0f;
    }
    float* merge = reinterpret_cast<float*>(smem);  // [warp][row][D + 8]
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        const int col = n * 8 + 2 * cq;
        float* r0 = merge + (warp * kMaxRows + gq) * SM::kMergePitch + col;
        float* r1 = merge + (warp * kMaxRows + gq + 8) * SM::kMergePitch + col;
        *reinterpret_cast<float2*>(r0) = make_float2(o[n][0] * factor[0], o[n][1] * factor[0]);
        *reinterpret_cast<float2*>(r1) = make_float2(o[n][2] * factor[1], o[n][3] * factor[1]);
    }
    consumers_sync();

    const size_t plane = (size_t)p.B * p.Nq * p.Hq;
    const int split = blockIdx.x;
    for (int idx = threadIdx.x; idx < w.R * D; idx += kConsumerWarps * 32) {
        const int r = idx / D, col = idx % D;
        float v = 0.0f;
#pragma unroll
        for (int u = 0; u < kConsumerWarps; ++u) v += merge[(u * kMaxRows + r) * SM::kMergePitch + col];
        const int i = r / w.nh, h = w.h0 + r % w.nh;
        const size_t orow = ((size_t)w.b * p.Nq + i) * p.Hq + h;
        if (p.num_splits == 1)
            static_cast<uint16_t*>(p.o)[orow * D + col] =
                static_cast<uint16_t>(ptx::pack_bf16x2(v, 0.0f) & 0xffffu);
        else
            p.part_o[(split * plane + orow) * D + col] = v;
    }
    if (warp == 0 && cq == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int r = gq + 8 * j;
            if (r >= w.R) continue;
            const int i = r / w.nh, h = w.h0 + r % w.nh;
            const size_t li = ((size_t)w.b * p.Hq + h) * p.Nq + i;
            if (p.num_splits == 1)
                p.lse[li] = lse2[j] * kLn2f;
            else
                p.part_lse[split * plane + li] = lse2[j];
        }
    }
}

// ------------------------------------------------------------- gather path
constexpr int kGatherThreads = 128;

template <int D>
struct GatherSmem {
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

// Gather keys [k0, k0 + 64) of one key/value head into a padded shared tile;
// keys at or past k_end, and keys on an invalid page, read as zero.
template <int D>
__device__ __forceinline__ void load_tile(const DecodeParams& p, const uint16_t* cache, uint16_t* tile,
                                          int b, int g, int k0, int k_end) {
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int idx = threadIdx.x; idx < kKeyTile * kChunks; idx += kGatherThreads) {
        const int r = idx / kChunks, c = idx % kChunks;
        const int key = k0 + r;
        bool valid = key < k_end;
        const int kk = valid ? key : 0;
        const int lp = kk / p.page_size;
        int page = valid ? page_of(p, b, lp) : 0;
        if (page < 0) {
            valid = false;
            page = 0;
        }
        const size_t row = (size_t)page * p.page_size + kk % p.page_size;
        const uint16_t* src = cache + (row * p.Hkv + g) * D + c * 8;
        cp_async16(tile + r * GatherSmem<D>::kRowPad + c * 8, src, valid);
    }
}


template <int D, int RMAX>
__global__ void __launch_bounds__(kGatherThreads) attn_decode_gather(const DecodeParams p) {
    static_assert(RMAX == 4 || RMAX == 8 || RMAX == 16, "row capacity");
    using SM = GatherSmem<D>;
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* kt = reinterpret_cast<uint16_t*>(smem);            // [2][tile]
    uint16_t* vt = kt + 2 * SM::kTileElems;                      // [2][tile]
    float* qs = reinterpret_cast<float*>(smem + SM::kBytesKV);   // [kMaxRows][D]
    float* ss = qs + kMaxRows * D;                               // [2][kMaxRows][kKeyTile]
    float* ps = ss + kMaxRows * kKeyTile;                        // aliases the second half
    float* st_m = ss + 2 * kMaxRows * kKeyTile;                  // running max (log2 units)
    float* st_l = st_m + kMaxRows;                               // running sum
    float* st_a = st_l + kMaxRows;                               // this tile's correction

    const Work w = work_of(p);
    const int split = blockIdx.x;
    const int tid = threadIdx.x;
    const int R = w.R, nh = w.nh, b = w.b, g = w.g, h0 = w.h0;
    const int k_begin = w.k_begin, k_end = w.k_end;

    // Q rows (fp32) and row state.
    for (int idx = tid; idx < R * D; idx += kGatherThreads) {
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
            for (int r = warp; r < R; r += kGatherThreads / 32) {
                int lo, hi;
                row_range(p, w, r, lo, hi);
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

// ------------------------------------------------------------------ combine
// Merge the slices of one output row (d threads).
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

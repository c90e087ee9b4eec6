// attn_bwd_kernel.cuh -- gradients of exact attention for sm_100a.
//
// The backward pass recomputes the score tiles from Q and K and rebuilds the
// weights from each row's saved log-sum-exp ("FlashAttention",
// ozercemkelahmet.com/tools/flashattention, How it works, Step 5, and
// "Backward pass in a bit more detail": key/value gradients accumulate over
// query blocks, query gradients over key blocks).  With P_ij = exp(s_ij - LSE_i),
// D_i = sum_c dO_ic O_ic and dS = P (dP - D):
//
//   attn_bwd_dsum    D_i for every (row, head), fp32, one warp per row.
//   attn_bwd_dkv     one CTA per (sequence, key/value head, 128-key block).  K and
//                    V stay in shared memory; the Q and dO tiles (64 rows) of every
//                    query head of the group and every query step that sees the
//                    keys stream through a 4-stage ring.  Per 64-row step:
//                      S^T = K Q^T, dP^T = V dO^T      (tcgen05, both from smem)
//                      P^T, dS^T                        (16 warps, fp32 -> bf16)
//                      dV += P^T dO, dK += dS^T Q       (A from tensor memory)
//                    S^T / dP^T have two buffers: the products of step t + 1 run
//                    while the elementwise warps work on step t.  dK and dV stay in
//                    tensor memory for the whole loop, so each key row is written
//                    once, already summed over the group.
//   attn_bwd_dq      one CTA per (sequence, query head, 128-row block), over the
//                    64-key steps the rows see: S = Q K^T, dP = dO V^T, dS, then
//                    dQ += dS K, S / dP double-buffered the same way.  dQ stays in
//                    tensor memory; no atomics.
//
// Tensor memory (512 columns): dkv: S^T buffers [0,64) [64,128), dP^T buffers
// [128,192) [192,256), dV [256,256+d), dK [384,384+d); dq: S [0,64) [64,128),
// dP [128,192) [192,256), dQ [256,256+d).  Each column group writes the bf16
// P^T / dS^T (dS) of its 16 columns into the first 8 of those same columns, and
// the next products read them there (one K-step per 16 columns).
//
// Warps: 0-15 elementwise (column group x = warp / 4 takes the tile's columns
// [32x, 32x + 32); warp w % 4 its 32 tensor-memory lanes: four warps per
// sub-partition hide the latency of the exponentials), 16 TMA producer, 17 MMA
// issuer (both converged, one elected lane issues).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "attn.h"
#include "ptx.cuh"

namespace attn {
namespace bwd {

// Device status word of the backward kernels (read by attn_device_status).
__device__ int g_bwd_status;

constexpr int kBM = 128;  // query rows of a dq CTA
constexpr int kBN = 128;  // keys of a dkv CTA
constexpr int kStep = 64; // rows (dkv) or keys (dq) streamed per step
constexpr int kElemWarps = 16;              // 4 column groups x 4 lane quadrants
constexpr int kGroups = kElemWarps / 4;      // column groups
constexpr int kGroupCols = kStep / kGroups;  // columns of a step per group (16)
constexpr int kWarpProducer = kElemWarps;
constexpr int kWarpMma = kElemWarps + 1;
constexpr int kThreads = (kElemWarps + 2) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBox128 = 128 * 128;  // TMA box of a 128-row tile: 128 rows x 128 bytes
constexpr uint32_t kBox64 = 64 * 128;    // TMA box of a 64-row step tile
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    const void* o;
    const void* dout;
    const float* lse;
    float* dsum;  // D, laid out like lse
    void* dq;
    void* dk;
    void* dv;
    const int32_t* cu_seqlens;
    int B, Hq, Hkv;
    int N;         // dense: sequence length; packed: total tokens
    int group;     // Hq / Hkv
    int left, right;
    int n_blocks;  // ceil(longest sequence / 128)
    float scale;
    float scale_log2;
    unsigned long long wait_limit_ns;
};

// ------------------------------------------------------------ small helpers
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicCAS(&g_bwd_status, 0, ATTN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::global_timer_ns() - t0 > limit_ns) {
            atomicCAS(&g_bwd_status, 0, ATTN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns) {
    return __all_sync(0xffffffffu, bounded_wait(bar, parity, abort_flag, limit_ns));
}

// 32 lanes x 32 bits, 16 consecutive columns per thread, then wait.
__device__ __forceinline__ void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// One arrival per elementwise warp, after every lane's tensor-memory stores
// are complete and fenced.
__device__ __forceinline__ void elem_warp_arrive(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

struct Seq {
    int start, len;
};

// Packed boundaries outside [0, N], decreasing, or longer than the blocks the
// launch was sized for (max_seqlen) give an empty sequence: nothing of it is
// read or written, and the block's first thread reports it.
__device__ __forceinline__ Seq seq_of(const BwdParams& p, int b) {
    Seq s;
    if (p.cu_seqlens) {
        const int s0 = p.cu_seqlens[b];
        const int s1 = p.cu_seqlens[b + 1];
        const bool bad = s0 < 0 || s1 < s0 || s1 > p.N || (long long)(s1 - s0) > (long long)p.n_blocks * kBN;
        if (bad && threadIdx.x == 0) atomicCAS(&g_bwd_status, 0, ATTN_ERR_SEQLENS);
        s.start = bad ? 0 : s0;
        s.len = bad ? 0 : s1 - s0;
    } else {
        s.start = b * p.N;
        s.len = p.N;
    }
    return s;
}

// Index of (sequence b, head h, row i) in lse / D: [B, Hq, N] dense, [Hq, T] packed.
__device__ __forceinline__ size_t stat_index(const BwdParams& p, int b, int h, int start, int i) {
    return p.cu_seqlens ? (size_t)h * p.N + start + i : ((size_t)b * p.Hq + h) * p.N + i;
}

__device__ __forceinline__ bool visible(const BwdParams& p, int q, int k) {
    return (p.left < 0 || k >= q - p.left) && (p.right < 0 || k <= q + p.right);
}

// Every (query, key) pair of queries [q0, q0 + nq) x keys [k0, k0 + nk) is
// inside the sequence and visible: no element mask needed.
__device__ __forceinline__ bool block_full(const BwdParams& p, long long q0, int nq, long long k0, int nk,
                                           int len) {
    if (q0 + nq > len || k0 + nk > len) return false;
    if (p.left >= 0 && k0 < q0 + nq - 1 - p.left) return false;
    if (p.right >= 0 && k0 + nk - 1 > q0 + p.right) return false;
    return true;
}

// 64-row query steps [m_lo, m_hi) that see some key of the 128-key block n.
__device__ __forceinline__ void query_steps(const BwdParams& p, int n, int len, int& m_lo, int& m_hi) {
    const long long k0 = (long long)n * kBN;
    long long lo = p.right >= 0 ? k0 - p.right : 0;
    long long hi = p.left >= 0 ? k0 + kBN + p.left : len;  // exclusive
    if (lo < 0) lo = 0;
    if (hi > len) hi = len;
    m_lo = (int)(lo / kStep);
    m_hi = hi > lo ? (int)((hi + kStep - 1) / kStep) : m_lo;
}

// 64-key steps [n_lo, n_hi) that some row of the 128-row query block m sees.
__device__ __forceinline__ void key_steps(const BwdParams& p, int m, int len, int& n_lo, int& n_hi) {
    const long long q0 = (long long)m * kBM;
    long long lo = p.left >= 0 ? q0 - p.left : 0;
    long long hi = p.right >= 0 ? q0 + kBM + p.right : len;  // exclusive
    if (lo < 0) lo = 0;
    if (hi > len) hi = len;
    n_lo = (int)(lo / kStep);
    n_hi = hi > lo ? (int)((hi + kStep - 1) / kStep) : n_lo;
}

// K-major operand (rows x d, 128-byte swizzle, 64-column boxes `box` bytes
// apart): descriptor of the 16-column step kk.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk, uint32_t box) {
    return ptx::smem_desc_sw128(tile + (kk / 4) * box + (kk % 4) * 32, 16, 1024);
}

// MN-major B operand ([K rows, N = d columns], N contiguous, the two 64-column
// halves `box` bytes apart): the 16-row step kk.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk, uint32_t box) {
    return ptx::smem_desc_sw128(tile + kk * 2048, box, 1024);
}

// All K-steps of one product from a single elected lane: the per-step
// descriptors are computed by the converged warp, and one elect.sync block
// issues the steps back to back (the first accumulates into D only if
// `accumulate`, the others always).
__device__ __forceinline__ void mma_ss4_elect(uint32_t d, const uint64_t (&a)[4], const uint64_t (&b)[4],
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %9, 0;\n\t"
        "setp.eq.b32 t, %9, %9;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %10, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %10, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %10, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %10, t;\n\t}" ::"r"(d),
        "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(accumulate), "r"(idesc)
        : "memory");
}

__device__ __forceinline__ void mma_ts4_elect(uint32_t d, const uint32_t (&a)[4], const uint64_t (&b)[4],
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %9, 0;\n\t"
        "setp.eq.b32 t, %9, %9;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %10, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %10, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %10, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %10, t;\n\t}" ::"r"(d),
        "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]),
        "r"(accumulate), "r"(idesc)
        : "memory");
}

// S^T / dP^T (dkv kernel): both operands K-major from shared memory, the
// D / 16 steps of d in groups of four (the second group accumulates).
template <int D>
__device__ __forceinline__ void mma_ss_kmajor_d(uint32_t d, uint32_t a_tile, uint32_t a_box, uint32_t b_tile,
                                                uint32_t b_box, uint32_t idesc) {
#pragma unroll
    for (int g = 0; g < D / 64; ++g) {
        uint64_t a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] = kmajor_desc(a_tile, 4 * g + i, a_box);
            b[i] = kmajor_desc(b_tile, 4 * g + i, b_box);
        }
        mma_ss4_elect(d, a, b, idesc, g > 0 ? 1u : 0u);
    }
}

// S / dP (dq kernel): A from tensor memory (8 columns per step), B K-major.
template <int D>
__device__ __forceinline__ void mma_ts_kmajor_d(uint32_t d, uint32_t a_tmem, uint32_t b_tile, uint32_t b_box,
                                                uint32_t idesc) {
#pragma unroll
    for (int g = 0; g < D / 64; ++g) {
        uint32_t a[4];
        uint64_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] = a_tmem + 8 * (4 * g + i);
            b[i] = kmajor_desc(b_tile, 4 * g + i, b_box);
        }
        mma_ts4_elect(d, a, b, idesc, g > 0 ? 1u : 0u);
    }
}

// Gradient products over one 64-wide step: A from tensor memory (the bf16
// pairs of 16 rows at columns 16 kk), B MN-major.
__device__ __forceinline__ void mma_ts_grad4(uint32_t d, uint32_t a_tmem, uint32_t b_tile, uint32_t b_box,
                                             uint32_t idesc, uint32_t accumulate) {
    uint32_t a[4];
    uint64_t b[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        a[kk] = a_tmem + 16 * kk;
        b[kk] = mnmajor_desc(b_tile, kk, b_box);
    }
    mma_ts4_elect(d, a, b, idesc, accumulate);
}

// ------------------------------------------------------------ D = rowsum(dO * O)
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dsum(const BwdParams p) {
    const int warp = (blockIdx.x * 256 + threadIdx.x) / 32;
    const int lane = threadIdx.x % 32;
    const int nwarps = gridDim.x * 8;
    const long long tokens = p.cu_seqlens ? (long long)p.N : (long long)p.B * p.N;
    const long long rows = tokens * p.Hq;
    constexpr int kPer = D / 32;  // elements per lane (2 or 4)
    for (long long r = warp; r < rows; r += nwarps) {
        const long long t = r / p.Hq;
        const int h = (int)(r % p.Hq);
        const uint16_t* op = static_cast<const uint16_t*>(p.o) + r * D + lane * kPer;
        const uint16_t* dp = static_cast<const uint16_t*>(p.dout) + r * D + lane * kPer;
        float acc = 0.0f;
        if (kPer == 4) {
            const uint2 a = *reinterpret_cast<const uint2*>(op);
            const uint2 c = *reinterpret_cast<const uint2*>(dp);
            acc = __uint_as_float(a.x << 16) * __uint_as_float(c.x << 16) +
                  __uint_as_float(a.x & 0xffff0000u) * __uint_as_float(c.x & 0xffff0000u) +
                  __uint_as_float(a.y << 16) * __uint_as_float(c.y << 16) +
                  __uint_as_float(a.y & 0xffff0000u) * __uint_as_float(c.y & 0xffff0000u);
        } else {
            const uint32_t a = *reinterpret_cast<const uint32_t*>(op);
            const uint32_t c = *reinterpret_cast<const uint32_t*>(dp);
            acc = __uint_as_float(a << 16) * __uint_as_float(c << 16) +
                  __uint_as_float(a & 0xffff0000u) * __uint_as_float(c & 0xffff0000u);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            size_t idx;
            if (p.cu_seqlens) {
                idx = (size_t)h * p.N + t;
            } else {
                const long long b = t / p.N, i = t % p.N;
                idx = ((size_t)b * p.Hq + h) * p.N + i;
            }
            p.dsum[idx] = acc;
        }
    }
}

// ------------------------------------------------------------ dK, dV
// Tensor memory: S^T buffer b at [64b, 64b + 64), dP^T buffer b at
// [128 + 64b, 128 + 64b + 64) (b = step & 1), dV [256, 256 + d), dK [384, 384 + d).
// The bf16 P^T / dS^T of queries [16c, 16c + 16) of a step (8 packed columns) go
// to the first 8 of that buffer's columns 16c.. (the ones their column group just
// read), and the products read K-step c there.  The products of step t + 1 are
// issued before the hand-off of step t, so they run while the elementwise warps
// work on step t.
template <int D, int STAGES>
struct DkvLayout {
    static constexpr uint32_t kTileK = kBN * D * 2;    // K or V: 128 keys
    static constexpr uint32_t kTileQ = kStep * D * 2;  // Q or dO: 64 rows
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kTileK;
    static constexpr uint32_t kRing = 2 * kTileK;
    static constexpr uint32_t kSlot = (2 * kTileQ + 2 * kStep * 4 + 1023) / 1024 * 1024;  // Q, dO, lse2, D
    static constexpr uint32_t kBar = kRing + STAGES * kSlot;
    // kv_loaded, slot_full[S], slot_empty[S], st_full[2], p_ready[2], done
    static constexpr uint32_t kNumBars = 6 + 2 * STAGES;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;
    static constexpr uint32_t kBytes = kMisc + 16;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;

    static __device__ __forceinline__ uint32_t q(uint32_t base, int s) { return base + kRing + s * kSlot; }
    static __device__ __forceinline__ uint32_t dout(uint32_t base, int s) { return q(base, s) + kTileQ; }
    static __device__ __forceinline__ uint32_t stats(uint32_t base, int s) { return q(base, s) + 2 * kTileQ; }
    static __device__ __forceinline__ uint32_t bar_kv(uint32_t base) { return base + kBar; }
    static __device__ __forceinline__ uint32_t bar_full(uint32_t base, int s) { return base + kBar + 8u * (1 + s); }
    static __device__ __forceinline__ uint32_t bar_empty(uint32_t base, int s) {
        return base + kBar + 8u * (1 + STAGES + s);
    }
    static __device__ __forceinline__ uint32_t bar_st(uint32_t base, int b) {
        return base + kBar + 8u * (1 + 2 * STAGES + b);
    }
    static __device__ __forceinline__ uint32_t bar_p(uint32_t base, int b) {
        return base + kBar + 8u * (3 + 2 * STAGES + b);
    }
    static __device__ __forceinline__ uint32_t bar_done(uint32_t base) { return base + kBar + 8u * (5 + 2 * STAGES); }
};

// The (query head, 64-row query step) steps of a key block, in loop order.
struct DkvWork {
    int b, g, n, start, len, m_lo, m_hi, steps;
};

__device__ __forceinline__ DkvWork dkv_work(const BwdParams& p) {
    DkvWork w;
    const int per_n = p.B * p.Hkv;
    w.n = blockIdx.x / per_n;  // key block 0 (the most query steps under a causal mask) first
    const int rem = blockIdx.x % per_n;
    w.b = rem / p.Hkv;
    w.g = rem % p.Hkv;
    const Seq s = seq_of(p, w.b);
    w.start = s.start;
    w.len = s.len;
    if (w.n * kBN >= w.len) {
        w.steps = 0;
        w.m_lo = w.m_hi = 0;
        return w;
    }
    query_steps(p, w.n, w.len, w.m_lo, w.m_hi);
    w.steps = p.group * (w.m_hi - w.m_lo);
    return w;
}

template <int D, int STAGES>
__device__ __forceinline__ void dkv_producer(const DkvWork& w, const BwdParams& p, const CUtensorMap* tm_q64,
                                             const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                             const CUtensorMap* tm_do64, uint32_t sbase,
                                             volatile int* abort_flag, uint8_t* smem) {
    using L = DkvLayout<D, STAGES>;
    constexpr int kBoxes = D / 64;
    const int lane = threadIdx.x % 32;
    const uint64_t pol_kv = ptx::policy_evict_first();
    const uint64_t pol_q = ptx::policy_evict_last();  // reread by the other key blocks
    ptx::mbar_arrive_expect_tx_elect(L::bar_kv(sbase), 2 * L::kTileK);
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx) {
        ptx::tma_load_2d_elect(sbase + L::kK + bx * kBox128, tm_k, L::bar_kv(sbase), w.g * D + bx * 64,
                               w.start + w.n * kBN, pol_kv);
        ptx::tma_load_2d_elect(sbase + L::kV + bx * kBox128, tm_v, L::bar_kv(sbase), w.g * D + bx * 64,
                               w.start + w.n * kBN, pol_kv);
    }
    const int nm = w.m_hi - w.m_lo;
    int issued = 0;
    for (int t = 0; t < w.steps; ++t) {
        const int s = t % STAGES;
        if (!warp_wait(L::bar_empty(sbase, s), ((t / STAGES) & 1) ^ 1, abort_flag, p.wait_limit_ns)) break;
        const int h = w.g * p.group + t / nm;
        const int m = w.m_lo + t % nm;
        ptx::mbar_arrive_expect_tx_elect(L::bar_full(sbase, s), 2 * L::kTileQ);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
            ptx::tma_load_2d_elect(L::q(sbase, s) + bx * kBox64, tm_q64, L::bar_full(sbase, s),
                                   h * D + bx * 64, w.start + m * kStep, pol_q);
            ptx::tma_load_2d_elect(L::dout(sbase, s) + bx * kBox64, tm_do64, L::bar_full(sbase, s),
                                   h * D + bx * 64, w.start + m * kStep, pol_q);
        }
        // lse2 and D of the step's 64 rows (0 past the sequence's end)
        float* st = reinterpret_cast<float*>(smem + (L::stats(sbase, s) - sbase));
#pragma unroll
        for (int e = 0; e < kStep / 32; ++e) {
            const int i = m * kStep + lane * (kStep / 32) + e;
            float l2 = 0.0f, dd = 0.0f;
            if (i < w.len) {
                const size_t idx = stat_index(p, w.b, h, w.start, i);
                l2 = p.lse[idx] * kLog2e;
                dd = p.dsum[idx];
            }
            st[lane * (kStep / 32) + e] = l2;
            st[kStep + lane * (kStep / 32) + e] = dd;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(L::bar_full(sbase, s));
        ++issued;
    }
    drain_wait(L::bar_kv(sbase), 0, p.wait_limit_ns);
    const int first = issued > STAGES ? issued - STAGES : 0;
    for (int i = first; i < issued; ++i)
        drain_wait(L::bar_full(sbase, i % STAGES), (i / STAGES) & 1, p.wait_limit_ns);
}

template <int D, int STAGES>
__device__ __forceinline__ void dkv_mma(const DkvWork& w, const BwdParams& p, uint32_t tmem, uint32_t sbase,
                                        volatile int* abort_flag) {
    using L = DkvLayout<D, STAGES>;
    constexpr uint32_t kIdS = ptx::idesc_bf16_f32(kBN, kStep, false, false);  // M keys, N = 64 queries
    constexpr uint32_t kIdG = ptx::idesc_bf16_f32(kBN, D, false, true);       // M keys, N = d
    const unsigned long long lim = p.wait_limit_ns;
    bool ok = warp_wait(L::bar_kv(sbase), 0, abort_flag, lim);
    ptx::tc_fence_after_sync();
    // S^T(t) and dP^T(t) into buffer t & 1
    auto issue_st = [&](int t) -> bool {
        const int s = t % STAGES;
        if (!warp_wait(L::bar_full(sbase, s), (t / STAGES) & 1, abort_flag, lim)) return false;
        ptx::tc_fence_after_sync();
        const uint32_t buf = (t & 1) * 64;
        mma_ss_kmajor_d<D>(tmem + buf, sbase + L::kK, kBox128, L::q(sbase, s), kBox64, kIdS);  // S^T = K Q^T
        mma_ss_kmajor_d<D>(tmem + 128 + buf, sbase + L::kV, kBox128, L::dout(sbase, s), kBox64,
                           kIdS);  // dP^T = V dO^T
        ptx::tc_commit_elect(L::bar_st(sbase, t & 1));
        return true;
    };
    if (ok && w.steps > 0) ok = issue_st(0);
    for (int t = 0; ok && t < w.steps; ++t) {
        if (t + 1 < w.steps && !(ok = issue_st(t + 1))) break;
        if (!(ok = warp_wait(L::bar_p(sbase, t & 1), (t >> 1) & 1, abort_flag, lim))) break;
        ptx::tc_fence_after_sync();
        const int s = t % STAGES;
        const uint32_t buf = (t & 1) * 64;
        static_assert(kStep == 64, "four 16-row steps per gradient product");
        // dV += P^T dO  (P^T of queries 16kk.. at column 16kk), then dK += dS^T Q
        mma_ts_grad4(tmem + 256, tmem + buf, L::dout(sbase, s), kBox64, kIdG, t > 0 ? 1u : 0u);
        mma_ts_grad4(tmem + 384, tmem + 128 + buf, L::q(sbase, s), kBox64, kIdG, t > 0 ? 1u : 0u);
        ptx::tc_commit_elect(L::bar_empty(sbase, s));
    }
    ptx::tc_commit_elect(L::bar_done(sbase));
    drain_wait(L::bar_done(sbase), 0, lim);
}

// One thread = one key row (tensor-memory lane); column group x = warp / 4
// takes query columns [16x, 16x + 16) of every 64-row step.
template <int D, int STAGES>
__device__ __forceinline__ void dkv_elementwise(const DkvWork& w, const BwdParams& p, uint32_t tmem,
                                                uint32_t sbase, uint8_t* smem, volatile int* abort_flag) {
    using L = DkvLayout<D, STAGES>;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int x = warp / 4, wq = warp % 4;
    const int row = wq * 32 + lane;
    const int key = w.n * kBN + row;  // within the sequence
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tl = tmem + lane_off;
    const float sl2 = p.scale_log2;
    const int nm = w.m_hi - w.m_lo;
    const unsigned long long lim = p.wait_limit_ns;
    bool ok = true;
    for (int t = 0; t < w.steps; ++t) {
        const int s = t % STAGES;
        const uint32_t buf = (t & 1) * 64;
        if (!(ok = warp_wait(L::bar_st(sbase, t & 1), (t >> 1) & 1, abort_flag, lim))) break;
        // the statistics were written by the producer before this slot's arrival
        if (!(ok = warp_wait(L::bar_full(sbase, s), (t / STAGES) & 1, abort_flag, lim))) break;
        ptx::tc_fence_after_sync();
        const int m = w.m_lo + t % nm;
        const float* st = reinterpret_cast<const float*>(smem + (L::stats(sbase, s) - sbase));
        const bool full = block_full(p, (long long)m * kStep, kStep, (long long)w.n * kBN, kBN, w.len);
#pragma unroll
        for (int c = 0; c < kGroupCols / 16; ++c) {
            const int col0 = kGroupCols * x + 16 * c;
            uint32_t sv[16], dv[16], pp[8], pd[8];
            tmem_ld16_sync(tl + buf + col0, sv);
            tmem_ld16_sync(tl + 128 + buf + col0, dv);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const int ql = col0 + i;
                const float2 l2 = *reinterpret_cast<const float2*>(st + ql);
                const float2 dd = *reinterpret_cast<const float2*>(st + kStep + ql);
                float p0 = ptx::ex2_approx(fmaf(__uint_as_float(sv[i]), sl2, -l2.x));
                float p1 = ptx::ex2_approx(fmaf(__uint_as_float(sv[i + 1]), sl2, -l2.y));
                if (!full) {
                    const int q = m * kStep + ql;
                    if (!(q < w.len && key < w.len && visible(p, q, key))) p0 = 0.0f;
                    if (!(q + 1 < w.len && key < w.len && visible(p, q + 1, key))) p1 = 0.0f;
                }
                pp[i / 2] = ptx::pack_bf16x2(p0, p1);
                pd[i / 2] = ptx::pack_bf16x2(p0 * (__uint_as_float(dv[i]) - dd.x),
                                             p1 * (__uint_as_float(dv[i + 1]) - dd.y));
            }
            // P^T / dS^T of these 16 queries go to the first 8 of the 16 columns this
            // thread has just read: no other group reads them, so no barrier is needed
            ptx::tmem_st8(tl + buf + col0, pp);
            ptx::tmem_st8(tl + 128 + buf + col0, pd);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before_sync();
        elem_warp_arrive(L::bar_p(sbase, t & 1));
    }
    if (!ok) return;
    if (!__all_sync(0xffffffffu, bounded_wait(L::bar_done(sbase), 0, abort_flag, lim))) return;
    ptx::tc_fence_after_sync();
    // the 2d output columns (dV then dK) are split evenly over the column groups
    // (dK times the scale)
    constexpr int kOutCols = 2 * D / kGroups;
    const bool store = key < w.len;
    const int c_first = x * kOutCols;  // in [0, 2d)
    const bool is_k = c_first >= D;
    const int c_in = c_first % D;
    const float mul = is_k ? p.scale : 1.0f;
    uint8_t* out = static_cast<uint8_t*>(is_k ? p.dk : p.dv) +
                   ((size_t)(w.start + (store ? key : 0)) * p.Hkv + w.g) * (size_t)D * 2 + c_in * 2;
    const uint32_t src = tl + (is_k ? 384u : 256u) + c_in;
#pragma unroll
    for (int cc = 0; cc < kOutCols / 32; ++cc) {
        uint32_t v[32];
        ptx::tmem_ld32_sync(src + cc * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            pk[i] = ptx::pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
        if (store) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                ptx::st_global_v4(out + cc * 64 + u * 16, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
    }
}

template <int D, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkv(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do64,
                 const BwdParams p) {
    using L = DkvLayout<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const DkvWork w = dkv_work(p);
    if (w.steps == 0) return;  // uniform over the block
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    if (warp == kWarpProducer && lane == 0) {
        ptx::mbar_init(L::bar_kv(sbase), 1);
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(L::bar_full(sbase, s), 2);  // expect_tx arrival + statistics arrival
            ptx::mbar_init(L::bar_empty(sbase, s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(L::bar_st(sbase, b), 1);
            ptx::mbar_init(L::bar_p(sbase, b), kElemWarps);
        }
        ptx::mbar_init(L::bar_done(sbase), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_q64);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_do64);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (warp < kElemWarps) {
        dkv_elementwise<D, STAGES>(w, p, tmem, sbase, smem, abort_flag);
    } else if (warp == kWarpProducer) {
        dkv_producer<D, STAGES>(w, p, &tm_q64, &tm_k, &tm_v, &tm_do64, sbase, abort_flag, smem);
    } else {
        dkv_mma<D, STAGES>(w, p, tmem, sbase, abort_flag);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kWarpMma) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------ dQ
// Tensor memory: S buffer b at [64b, 64b + 64), dP buffer b at
// [128 + 64b, 128 + 64b + 64), dQ [256, 256 + d); dS of keys [16c, 16c + 16)
// (8 packed columns) goes to the first 8 of the S buffer's columns 16c...
template <int D, int STAGES>
struct DqLayout {
    static constexpr uint32_t kTileQ = kBM * D * 2;    // Q or dO: 128 rows
    static constexpr uint32_t kTileK = kStep * D * 2;  // K or V: 64 keys
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kDO = kTileQ;
    static constexpr uint32_t kRing = 2 * kTileQ;
    static constexpr uint32_t kSlot = 2 * kTileK;  // K, V
    static constexpr uint32_t kBar = kRing + STAGES * kSlot;
    // q_loaded, slot_full[S], slot_empty[S], st_full[2], ds_ready[2], done, a_ready
    static constexpr uint32_t kNumBars = 7 + 2 * STAGES;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;
    static constexpr uint32_t kBytes = kMisc + 16;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;
    // Tensor memory: S [0,128) and dP [128,256) as two 64-column buffers each,
    // dQ [256, 256 + D), then Q and dO as bf16 pairs (D / 2 columns each): the
    // A operands of the S and dP products.
    static constexpr uint32_t kTQ = 384;
    static constexpr uint32_t kTDO = kTQ + D / 2;

    static __device__ __forceinline__ uint32_t k(uint32_t base, int s) { return base + kRing + s * kSlot; }
    static __device__ __forceinline__ uint32_t v(uint32_t base, int s) { return k(base, s) + kTileK; }
    static __device__ __forceinline__ uint32_t bar_q(uint32_t base) { return base + kBar; }
    static __device__ __forceinline__ uint32_t bar_full(uint32_t base, int s) { return base + kBar + 8u * (1 + s); }
    static __device__ __forceinline__ uint32_t bar_empty(uint32_t base, int s) {
        return base + kBar + 8u * (1 + STAGES + s);
    }
    static __device__ __forceinline__ uint32_t bar_st(uint32_t base, int b) {
        return base + kBar + 8u * (1 + 2 * STAGES + b);
    }
    static __device__ __forceinline__ uint32_t bar_ds(uint32_t base, int b) {
        return base + kBar + 8u * (3 + 2 * STAGES + b);
    }
    static __device__ __forceinline__ uint32_t bar_done(uint32_t base) { return base + kBar + 8u * (5 + 2 * STAGES); }
    static __device__ __forceinline__ uint32_t bar_a(uint32_t base) { return base + kBar + 8u * (6 + 2 * STAGES); }
};

// Copies this thread's row of Q (groups 0, 1) or dO (groups 2, 3) from the
// TMA tile (128-byte swizzle: 16-byte chunk c of row r sits at chunk
// c ^ (r mod 8) of its 128-byte line) into tensor memory, half a row per
// group, packed two bf16 per column in the order of d.
template <int D, int STAGES>
__device__ __forceinline__ void dq_stage_a(uint32_t tl, uint32_t sbase, int x, int row) {
    using L = DqLayout<D, STAGES>;
    constexpr int kChunks = D / 16;  // 16-byte chunks in half a row
    const uint32_t src = sbase + (x < 2 ? L::kQ : L::kDO);
    const int c0 = (x & 1) * kChunks;
    uint32_t r[4 * kChunks];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int c = c0 + i;
        const uint32_t addr = src + (c >> 3) * kBox128 + row * 128 + (((c & 7) ^ (row & 7)) << 4);
        ptx::ld_shared_v4(addr, r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    }
    const uint32_t dst = tl + (x < 2 ? L::kTQ : L::kTDO) + 4 * c0;
    if constexpr (kChunks == 8)
        ptx::tmem_st32(dst, r);
    else
        ptx::tmem_st16(dst, r);
}

struct DqWork {
    int b, h, g, m, start, len, n_lo, n_hi;
};

__device__ __forceinline__ DqWork dq_work(const BwdParams& p) {
    DqWork w;
    const int per_m = p.B * p.Hq;
    w.m = p.n_blocks - 1 - blockIdx.x / per_m;  // latest rows (most key steps, causal) first
    const int rem = blockIdx.x % per_m;
    w.b = rem / p.Hq;
    w.h = rem % p.Hq;
    w.g = w.h / p.group;
    const Seq s = seq_of(p, w.b);
    w.start = s.start;
    w.len = s.len;
    if (w.m * kBM >= w.len) {
        w.n_lo = w.n_hi = 0;
        return w;
    }
    key_steps(p, w.m, w.len, w.n_lo, w.n_hi);
    return w;
}

template <int D, int STAGES>
__device__ __forceinline__ void dq_producer(const DqWork& w, const BwdParams& p, const CUtensorMap* tm_q,
                                            const CUtensorMap* tm_k64, const CUtensorMap* tm_v64,
                                            const CUtensorMap* tm_do, uint32_t sbase, volatile int* abort_flag) {
    using L = DqLayout<D, STAGES>;
    constexpr int kBoxes = D / 64;
    const uint64_t pol_q = ptx::policy_evict_first();
    const uint64_t pol_kv = ptx::policy_evict_last();
    ptx::mbar_arrive_expect_tx_elect(L::bar_q(sbase), 2 * L::kTileQ);
#pragma unroll
    for (int bx = 0; bx < kBoxes; ++bx) {
        ptx::tma_load_2d_elect(sbase + L::kQ + bx * kBox128, tm_q, L::bar_q(sbase), w.h * D + bx * 64,
                               w.start + w.m * kBM, pol_q);
        ptx::tma_load_2d_elect(sbase + L::kDO + bx * kBox128, tm_do, L::bar_q(sbase), w.h * D + bx * 64,
                               w.start + w.m * kBM, pol_q);
    }
    int issued = 0;
    for (int n = w.n_lo; n < w.n_hi; ++n) {
        const int t = n - w.n_lo, s = t % STAGES;
        if (!warp_wait(L::bar_empty(sbase, s), ((t / STAGES) & 1) ^ 1, abort_flag, p.wait_limit_ns)) break;
        ptx::mbar_arrive_expect_tx_elect(L::bar_full(sbase, s), 2 * L::kTileK);
#pragma unroll
        for (int bx = 0; bx < kBoxes; ++bx) {
            ptx::tma_load_2d_elect(L::k(sbase, s) + bx * kBox64, tm_k64, L::bar_full(sbase, s),
                                   w.g * D + bx * 64, w.start + n * kStep, pol_kv);
            ptx::tma_load_2d_elect(L::v(sbase, s) + bx * kBox64, tm_v64, L::bar_full(sbase, s),
                                   w.g * D + bx * 64, w.start + n * kStep, pol_kv);
        }
        ++issued;
    }
    drain_wait(L::bar_q(sbase), 0, p.wait_limit_ns);
    const int first = issued > STAGES ? issued - STAGES : 0;
    for (int i = first; i < issued; ++i)
        drain_wait(L::bar_full(sbase, i % STAGES), (i / STAGES) & 1, p.wait_limit_ns);
}

template <int D, int STAGES>
__device__ __forceinline__ void dq_mma(const DqWork& w, const BwdParams& p, uint32_t tmem, uint32_t sbase,
                                       volatile int* abort_flag) {
    using L = DqLayout<D, STAGES>;
    constexpr uint32_t kIdS = ptx::idesc_bf16_f32(kBM, kStep, false, false);  // M queries, N = 64 keys
    constexpr uint32_t kIdG = ptx::idesc_bf16_f32(kBM, D, false, true);
    const unsigned long long lim = p.wait_limit_ns;
    const int steps = w.n_hi - w.n_lo;
    // Q and dO reach tensor memory through the elementwise warps (dq_stage_a).
    bool ok = warp_wait(L::bar_a(sbase), 0, abort_flag, lim);
    ptx::tc_fence_after_sync();
    auto issue_st = [&](int t) -> bool {  // S(t) and dP(t) into buffer t & 1
        const int s = t % STAGES;
        if (!warp_wait(L::bar_full(sbase, s), (t / STAGES) & 1, abort_flag, lim)) return false;
        ptx::tc_fence_after_sync();
        const uint32_t buf = (t & 1) * 64;
        // A from tensor memory: shared memory then serves only the 64-key B
        // operand (an SS product of N = 64 would read 1.5x the shared-memory
        // bandwidth that the tensor pipe consumes).
        mma_ts_kmajor_d<D>(tmem + buf, tmem + L::kTQ, L::k(sbase, s), kBox64, kIdS);          // S = Q K^T
        mma_ts_kmajor_d<D>(tmem + 128 + buf, tmem + L::kTDO, L::v(sbase, s), kBox64, kIdS);   // dP = dO V^T
        ptx::tc_commit_elect(L::bar_st(sbase, t & 1));
        return true;
    };
    if (ok && steps > 0) ok = issue_st(0);
    for (int t = 0; ok && t < steps; ++t) {
        if (t + 1 < steps && !(ok = issue_st(t + 1))) break;
        if (!(ok = warp_wait(L::bar_ds(sbase, t & 1), (t >> 1) & 1, abort_flag, lim))) break;
        ptx::tc_fence_after_sync();
        const int s = t % STAGES;
        const uint32_t buf = (t & 1) * 64;
        // dQ += dS K  (dS of keys 16kk.. at column 16kk)
        mma_ts_grad4(tmem + 256, tmem + buf, L::k(sbase, s), kBox64, kIdG, t > 0 ? 1u : 0u);
        ptx::tc_commit_elect(L::bar_empty(sbase, s));
    }
    ptx::tc_commit_elect(L::bar_done(sbase));
    drain_wait(L::bar_done(sbase), 0, lim);
}

// One thread = one query row; column group x = warp / 4 takes key columns
// [16x, 16x + 16) of every 64-key step.
template <int D, int STAGES>
__device__ __forceinline__ void dq_elementwise(const DqWork& w, const BwdParams& p, uint32_t tmem,
                                               uint32_t sbase, volatile int* abort_flag) {
    using L = DqLayout<D, STAGES>;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int x = warp / 4, wq = warp % 4;
    const int row = wq * 32 + lane;
    const int q = w.m * kBM + row;  // within the sequence
    const bool valid = q < w.len;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tl = tmem + lane_off;
    const float sl2 = p.scale_log2;
    float l2 = 0.0f, dd = 0.0f;
    if (valid) {
        const size_t idx = stat_index(p, w.b, w.h, w.start, q);
        l2 = p.lse[idx] * kLog2e;
        dd = p.dsum[idx];
    }
    const unsigned long long lim = p.wait_limit_ns;
    bool ok = warp_wait(L::bar_q(sbase), 0, abort_flag, lim);
    if (ok) {
        dq_stage_a<D, STAGES>(tl, sbase, x, row);
        ptx::tmem_wait_st();
        ptx::tc_fence_before_sync();
        elem_warp_arrive(L::bar_a(sbase));
    }
    for (int n = w.n_lo; ok && n < w.n_hi; ++n) {
        const int t = n - w.n_lo;
        const uint32_t buf = (t & 1) * 64;
        if (!(ok = warp_wait(L::bar_st(sbase, t & 1), (t >> 1) & 1, abort_flag, lim))) break;
        ptx::tc_fence_after_sync();
        const bool full = block_full(p, (long long)w.m * kBM, kBM, (long long)n * kStep, kStep, w.len);
#pragma unroll
        for (int c = 0; c < kGroupCols / 16; ++c) {
            const int col0 = kGroupCols * x + 16 * c;
            uint32_t sv[16], dv[16], pd[8];
            tmem_ld16_sync(tl + buf + col0, sv);
            tmem_ld16_sync(tl + 128 + buf + col0, dv);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                float p0 = ptx::ex2_approx(fmaf(__uint_as_float(sv[i]), sl2, -l2));
                float p1 = ptx::ex2_approx(fmaf(__uint_as_float(sv[i + 1]), sl2, -l2));
                if (!full) {
                    const int k = n * kStep + col0 + i;
                    if (!(valid && k < w.len && visible(p, q, k))) p0 = 0.0f;
                    if (!(valid && k + 1 < w.len && visible(p, q, k + 1))) p1 = 0.0f;
                }
                pd[i / 2] = ptx::pack_bf16x2(p0 * (__uint_as_float(dv[i]) - dd),
                                             p1 * (__uint_as_float(dv[i + 1]) - dd));
            }
            ptx::tmem_st8(tl + buf + col0, pd);  // into the columns this thread has just read
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before_sync();
        elem_warp_arrive(L::bar_ds(sbase, t & 1));
    }
    if (!ok) return;
    if (!__all_sync(0xffffffffu, bounded_wait(L::bar_done(sbase), 0, abort_flag, lim))) return;
    ptx::tc_fence_after_sync();
    // group x stores columns [x * d / groups, (x + 1) * d / groups) of dQ (times the scale)
    constexpr int kCols = D / kGroups;
    uint8_t* out = static_cast<uint8_t*>(p.dq) +
                   ((size_t)(w.start + (valid ? q : 0)) * p.Hq + w.h) * (size_t)D * 2 + x * kCols * 2;
#pragma unroll
    for (int c = 0; c < kCols / 16; ++c) {
        uint32_t v[16];
        tmem_ld16_sync(tl + 256 + x * kCols + 16 * c, v);
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            pk[i] = ptx::pack_bf16x2(__uint_as_float(v[2 * i]) * p.scale, __uint_as_float(v[2 * i + 1]) * p.scale);
        if (valid) {
            ptx::st_global_v4(out + c * 32, pk[0], pk[1], pk[2], pk[3]);
            ptx::st_global_v4(out + c * 32 + 16, pk[4], pk[5], pk[6], pk[7]);
        }
    }
}

template <int D, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k64,
                const __grid_constant__ CUtensorMap tm_v64, const __grid_constant__ CUtensorMap tm_do,
                const BwdParams p) {
    using L = DqLayout<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const DqWork w = dq_work(p);
    if (w.n_hi <= w.n_lo) return;  // uniform over the block
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    if (warp == kWarpProducer && lane == 0) {
        ptx::mbar_init(L::bar_q(sbase), 1);
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(L::bar_full(sbase, s), 1);
            ptx::mbar_init(L::bar_empty(sbase, s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(L::bar_st(sbase, b), 1);
            ptx::mbar_init(L::bar_ds(sbase, b), kElemWarps);
        }
        ptx::mbar_init(L::bar_done(sbase), 1);
        ptx::mbar_init(L::bar_a(sbase), kElemWarps);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k64);
        ptx::prefetch_tensormap(&tm_v64);
        ptx::prefetch_tensormap(&tm_do);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (warp < kElemWarps) {
        dq_elementwise<D, STAGES>(w, p, tmem, sbase, abort_flag);
    } else if (warp == kWarpProducer) {
        dq_producer<D, STAGES>(w, p, &tm_q, &tm_k64, &tm_v64, &tm_do, sbase, abort_flag);
    } else {
        dq_mma<D, STAGES>(w, p, tmem, sbase, abort_flag);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == kWarpMma) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace bwd
}  // namespace attn

// attn_fwd_fp8_kernel.cuh -- the fused attention forward with 8-bit (e4m3)
// query, key and value inputs, d = 128.
//
// "Flash Attention" skill page (skillmd.com), Workflow 3: the inputs are
// converted to float8_e4m3 and the fused kernel runs on them; "FlashAttention"
// explainer page, How it works, Step 8: 8-bit floating point for some of the
// products, with the softmax statistics kept in fp32.  Here both products run
// on e4m3 operands with fp32 accumulation (tcgen05 kind::f8f6f4):
//   S = Q K^T             Q, K e4m3 from shared memory (K-major, 128-byte swizzle)
//   O += P V              P rounded to e4m3 in tensor memory; V^T e4m3 (K-major)
// The softmax is the bf16 kernel's (lazy rescale, fp32 statistics, part of
// the exponentials on the FMA pipe: 1/4 here); O is divided by the sum of the e4m3-rounded
// weights (so it is an exact convex combination of V's rows for those weights),
// the LSE uses the fp32 weights.  O is written as bf16, LSE as fp32.
//
// The products read every operand K-major, so the value tile is the transpose
// V^T [d, keys]; attn_fwd_fp8 writes it first (attn_vt_transpose_kernel) into
// the workspace, each sequence padded to a multiple of 128 keys so that every
// TMA box starts on a 16-byte boundary.
//
// The tile schedule, warp roles, barriers, bounded waits and status word are the
// bf16 kernel's (attn_fwd_kernel.cuh), with 16 KB tiles and an 8-stage ring.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn {
namespace fp8 {

constexpr int kD = 128;
constexpr uint32_t kTileBytes = 128 * 128;  // 128 rows x 128 one-byte elements
constexpr int kStages = 8;
// One in four groups of four weights takes the FMA-pipe exponential: with the
// e4m3 products twice as fast, the exponential unit is relieved a little more
// than in the bf16 kernel (measured: 1/4 beat 1/2, 1/8, 1/16 and none).
constexpr int kPolyPeriodFp8 = 4;
// Register split after launch: 128 x (216 + 216 + 72) = 384 x 168 (this
// kernel's producer and MMA loop need more than the bf16 kernel's 56).
constexpr uint32_t kRegsSoftmaxFp8 = 216;
constexpr uint32_t kRegsOtherFp8 = 72;

// kind::f8f6f4 descriptor: e4m3 A and B (format 0), fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// The four K-steps of a score product (32 one-byte elements, i.e. +32 bytes
// = +2 in the descriptor's start field, per step) from one elected lane.
__device__ __forceinline__ void mma_ss_f8_k4_elect(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc) {
    asm volatile(
        "{\n\t.reg .pred f, t, e;\n\t.reg .b64 a, b;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 f, %3, %3;\n\t"
        "setp.eq.b32 t, %3, %3;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, f;\n\t"
        "add.s64 a, %1, 2;\n\tadd.s64 b, %2, 2;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
        "add.s64 a, %1, 4;\n\tadd.s64 b, %2, 4;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t"
        "add.s64 a, %1, 6;\n\tadd.s64 b, %2, 6;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, t;\n\t}" ::"r"(d_tmem),
        "l"(a0), "l"(b0), "r"(idesc)
        : "memory");
}

// Two K-steps of a P V product: A from tensor memory (+8 columns per step), B
// K-major (+32 bytes per step).
__device__ __forceinline__ void mma_ts_f8_k2_elect(uint32_t d_tmem, uint32_t a_tmem0, uint64_t b0, uint32_t idesc,
                                                   uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 a;\n\t.reg .b64 b;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, %4, %4;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t"
        "add.u32 a, %1, 8;\n\tadd.s64 b, %2, 2;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [a], b, %3, t;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem0), "l"(b0), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four fp32 -> four e4m3 (round to nearest even, saturating) in one word,
// element 0 in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a0, float a1, float a2, float a3) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
    return r;
}

// acc + the four e4m3 values of a packed word, each added in fp32 (e4m3 values
// are exact in f16).
__device__ __forceinline__ float add_e4m3x4_to_f32(float acc, uint32_t packed) {
    asm("{\n\t.reg .b16 lo, hi, h0, h1, h2, h3;\n\t.reg .b32 w01, w23;\n\t"
        "mov.b32 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 w01, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 w23, hi;\n\t"
        "mov.b32 {h0, h1}, w01;\n\t"
        "mov.b32 {h2, h3}, w23;\n\t"
        "add.rn.f32.f16 %0, h0, %0;\n\t"
        "add.rn.f32.f16 %0, h1, %0;\n\t"
        "add.rn.f32.f16 %0, h2, %0;\n\t"
        "add.rn.f32.f16 %0, h3, %0;\n\t}"
        : "+f"(acc)
        : "r"(packed));
    return acc;
}

struct Layout {
    static constexpr uint32_t kQ0 = 0;
    static constexpr uint32_t kQ1 = kTileBytes;
    static constexpr uint32_t kKV = 2 * kTileBytes;
    // Output staging: 4 KB per softmax warp (32 rows x 64 bf16 columns).
    static constexpr uint32_t kStg = kKV + kStages * kTileBytes;
    static constexpr uint32_t kBar = kStg + 8 * 4096;
    // q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2], o_done[2], mma_final,
    // q_empty, o_free[2], clc, unit_full[2], unit_empty[2], p_part[2][kPParts - 1]
    static constexpr uint32_t kNumBars = 16 + 2 * (kPParts - 1) + 2 * kStages;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // tmem address, abort flag
    static constexpr uint32_t kClcResp = kMisc + 16;        // launch-control response (16 B)
    static constexpr uint32_t kUnitQ = kClcResp + 16;       // unit queue: two ints
    static constexpr uint32_t kBytes = kUnitQ + 16;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;
    static_assert(kClcResp % 16 == 0, "the launch-control response needs 16-byte alignment");

    static __device__ __forceinline__ uint32_t bar_q(uint32_t base) { return base + kBar; }
    static __device__ __forceinline__ uint32_t bar_kv_full(uint32_t base, int s) { return base + kBar + 8u * (1 + s); }
    static __device__ __forceinline__ uint32_t bar_kv_empty(uint32_t base, int s) {
        return base + kBar + 8u * (1 + kStages + s);
    }
    static __device__ __forceinline__ uint32_t bar_s_full(uint32_t base, int x) {
        return base + kBar + 8u * (1 + 2 * kStages + x);
    }
    static __device__ __forceinline__ uint32_t bar_p_ready(uint32_t base, int x) {
        return base + kBar + 8u * (3 + 2 * kStages + x);
    }
    static __device__ __forceinline__ uint32_t bar_o_done(uint32_t base, int x) {
        return base + kBar + 8u * (5 + 2 * kStages + x);
    }
    static __device__ __forceinline__ uint32_t bar_mma_final(uint32_t base) {
        return base + kBar + 8u * (7 + 2 * kStages);
    }
    static __device__ __forceinline__ uint32_t bar_q_empty(uint32_t base) {
        return base + kBar + 8u * (8 + 2 * kStages);
    }
    static __device__ __forceinline__ uint32_t bar_o_free(uint32_t base, int x) {
        return base + kBar + 8u * (9 + 2 * kStages + x);
    }
    static __device__ __forceinline__ uint32_t bar_clc(uint32_t base) {
        return base + kBar + 8u * (11 + 2 * kStages);
    }
    static __device__ __forceinline__ uint32_t bar_unit_full(uint32_t base, int slot) {
        return base + kBar + 8u * (12 + 2 * kStages + slot);
    }
    static __device__ __forceinline__ uint32_t bar_unit_empty(uint32_t base, int slot) {
        return base + kBar + 8u * (14 + 2 * kStages + slot);
    }
    static __device__ __forceinline__ uint32_t bar_p_part(uint32_t base, int x, int k) {
        return base + kBar + 8u * (16 + 2 * kStages + (kPParts - 1) * x + k);
    }
};

// First padded column of sequence b in V^T (each sequence rounded up to 128).
__device__ __forceinline__ long long vt_start(const FwdParams& p, int b) {
    if (!p.cu_seqlens) return (long long)b * ((p.N + kBN - 1) / kBN) * kBN;
    long long s = 0;
    for (int i = 0; i < b; ++i) {
        const long long len = (long long)p.cu_seqlens[i + 1] - p.cu_seqlens[i];
        if (len > 0) s += (len + kBN - 1) / kBN * kBN;
    }
    return s;
}

// The bf16 kernel's persistent schedule (UnitSource), with V^T blocks.
__device__ __forceinline__ void producer(const FwdParams& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                         const CUtensorMap* tm_vt, uint32_t sbase, volatile int* abort_flag) {
    using L = Layout;
    const unsigned long long lim = p.wait_limit_ns;
    const uint64_t pol_q = ptx::policy_evict_first();
    const uint64_t pol_kv = ptx::policy_evict_last();
    UnitSource<L> src(sbase);
    int issued = 0;  // K/V ring loads
    int units = 0;   // pairs whose Q was loaded
    bool ok = true;
    int u = src.next(p, abort_flag, ok);
    while (ok) {
        if (!(ok = src.publish(u, abort_flag, lim)) || u < 0) break;
        const TilePair w = decode_pair(u, p);
        const int vs = vt_start(p, w.b);
        if (units > 0 && !(ok = warp_wait(L::bar_q_empty(sbase), (units - 1) & 1, abort_flag, lim))) break;
        ptx::mbar_arrive_expect_tx_elect(L::bar_q(sbase), 2 * kTileBytes);
        for (int x = 0; x < 2; ++x)
            ptx::tma_load_2d_elect(sbase + (x ? L::kQ1 : L::kQ0), tm_q, L::bar_q(sbase), w.h[x] * kD,
                                   w.start + w.r0[x], pol_q);
        ++units;
        for (int j = w.ulo; j < w.uhi && ok; ++j) {
            for (int kv = 0; kv < 2; ++kv) {
                const int s = issued % kStages;
                const uint32_t ph = (issued / kStages) & 1;
                if (!(ok = warp_wait(L::bar_kv_empty(sbase, s), ph ^ 1, abort_flag, lim))) break;
                ptx::mbar_arrive_expect_tx_elect(L::bar_kv_full(sbase, s), kTileBytes);
                if (kv == 0)  // K block: 128 keys x 128 values of head g
                    ptx::tma_load_2d_elect(sbase + L::kKV + s * kTileBytes, tm_k, L::bar_kv_full(sbase, s),
                                           w.g * kD, w.start + j * kBN, pol_kv);
                else  // V^T block: 128 values of head g x 128 keys
                    ptx::tma_load_2d_elect(sbase + L::kKV + s * kTileBytes, tm_vt, L::bar_kv_full(sbase, s),
                                           vs + j * kBN, w.g * kD, pol_kv);
                ++issued;
            }
        }
        if (ok) u = src.next(p, abort_flag, ok);
    }
    src.drain(lim);
    if (units > 0) drain_wait(L::bar_q(sbase), (units - 1) & 1, lim);
    const int first = issued > kStages ? issued - kStages : 0;
    for (int i = first; i < issued; ++i)
        drain_wait(L::bar_kv_full(sbase, i % kStages), (i / kStages) & 1, lim);
}

__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t sbase, int x, int slot) {
    using L = Layout;
    constexpr uint32_t kIdesc = idesc_e4m3_f32(kBM, kBN);
    const uint32_t qa = sbase + (x ? L::kQ1 : L::kQ0);
    const uint32_t ka = sbase + L::kKV + slot * kTileBytes;
    static_assert(kD / 32 == 4, "four 32-byte steps cover one 128-byte row");
    mma_ss_f8_k4_elect(tmem + (x ? 128u : 0u), ptx::smem_desc_sw128(qa, 16, 1024), ptx::smem_desc_sw128(ka, 16, 1024),
                       kIdesc);
}

// Keys [128 part / kPParts, 128 (part + 1) / kPParts) of the block.
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint32_t sbase, int x, int slot, int part, bool accumulate) {
    using L = Layout;
    constexpr uint32_t kIdesc = idesc_e4m3_f32(kBM, kD);
    const uint32_t va = sbase + L::kKV + slot * kTileBytes;  // V^T: d rows x 128 keys
    const uint32_t p_tmem = tmem + (x ? 128u : 0u) + kPOffset;
    constexpr int kSteps = kBN / 32 / kPParts;  // 32 keys per step = 8 packed columns of P
    static_assert(kSteps == 2, "two steps per part");
    const int kk = part * kSteps;
    mma_ts_f8_k2_elect(tmem + kTmemO0 + (x ? 128u : 0u), p_tmem + kk * 8, ptx::smem_desc_sw128(va + kk * 32, 16, 1024),
                       kIdesc, accumulate ? 1u : 0u);
}

// The bf16 kernel's MMA loop (order S0(j), PV1(j-1), S1(j), PV0(j), and its
// barriers) with the e4m3 products.
__device__ __forceinline__ void mma_role(const FwdParams& p, uint32_t tmem, uint32_t sbase,
                                         volatile int* abort_flag) {
    mma_loop<Layout, kStages>(
        p, sbase, abort_flag, [&](int x, int slot) { issue_qk(tmem, sbase, x, slot); },
        [&](int x, int slot, int part, bool acc) { issue_pv(tmem, sbase, x, slot, part, acc); });
}

// One thread per query row, as in the bf16 kernel; P goes to tensor memory as
// e4m3 (4 per column).
__device__ __forceinline__ bool softmax_unit(const TilePair& w, const FwdParams& p, int x, int warp_in_group,
                                             int lane, uint32_t tmem, uint32_t sbase, volatile int* abort_flag,
                                             uint32_t& phases, int u) {
    using L = Layout;
    const int r0 = x ? w.r0[1] : w.r0[0];
    const int blk_lo = x ? w.lo[1] : w.lo[0];
    const int blk_hi = x ? w.hi[1] : w.hi[0];
    const unsigned long long lim = p.wait_limit_ns;
    const int row = r0 + warp_in_group * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
    const uint32_t t_s = tmem + lane_off + (x ? 128u : 0u);
    const uint32_t t_p = t_s + kPOffset;
    const uint32_t t_o = tmem + lane_off + kTmemO0 + (x ? 128u : 0u);
    const float sl2 = p.scale_log2;
    const int key_lo = p.left >= 0 ? (row - p.left > 0 ? row - p.left : 0) : 0;
    long long khi = p.right >= 0 ? (long long)row + p.right : (long long)w.len - 1;
    if (khi > (long long)w.len - 1) khi = (long long)w.len - 1;
    const int key_hi = (int)khi;
    const int tile_last_row = r0 + kBM - 1;

    float m_ref = -INFINITY;
    float l_sum = 0.0f;  // fp32 weights -> LSE
    float l_q = 0.0f;    // e4m3-rounded weights -> O
    bool ok = true;
    for (int j = blk_lo; j < blk_hi; ++j) {
        ok = __all_sync(0xffffffffu, bounded_wait(L::bar_s_full(sbase, x), phases & 1u, abort_flag, lim));
        if (!ok) break;
        phases ^= 1u;
        ptx::tc_fence_after_sync();
        uint32_t s[128];
        ptx::tmem_ld128_sync(t_s, s);
        const int k0 = j * kBN;
        const bool full_block =
            (k0 + kBN <= w.len) && (p.left < 0 || (long long)k0 >= (long long)tile_last_row - p.left) &&
            (p.right < 0 || (long long)k0 + kBN - 1 <= (long long)r0 + p.right);
        if (!full_block) {
            const int c_lo = key_lo - k0, c_hi = key_hi - k0;
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (c < c_lo || c > c_hi) s[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
            mx0 = ptx::fmax3(mx0, __uint_as_float(s[c + 0]), __uint_as_float(s[c + 1]));
            mx1 = ptx::fmax3(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
            mx2 = ptx::fmax3(mx2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
            mx3 = ptx::fmax3(mx3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
        }
        const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
        float alpha = 1.0f;
        bool rescale_o = false;
        if (m_blk > m_ref + kRescaleThreshold) {
            alpha = ptx::ex2_approx(m_ref - m_blk);
            rescale_o = (m_ref != -INFINITY);
            l_sum *= alpha;
            l_q *= alpha;
            m_ref = m_blk;
        }
        if (__any_sync(0xffffffffu, rescale_o)) {
            const float a = rescale_o ? alpha : 1.0f;
#pragma unroll
            for (int cc = 0; cc < kD / 32; ++cc) {
                uint32_t o[32];
                ptx::tmem_ld32_sync(t_o + cc * 32, o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                ptx::tmem_st32(t_o + cc * 32, o);
            }
        }
        const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
        const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
        const uint64_t negm_2 = ptx::f2_pack(neg_m, neg_m);
        uint64_t sum_a = 0, sum_b = 0;
        float rq0 = 0.f, rq1 = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = q * 32 + 4 * i;
                float x0, x1, x2, x3;
                ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(__uint_as_float(s[c + 0]), __uint_as_float(s[c + 1])),
                                          sl2_2, negm_2), x0, x1);
                ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])),
                                          sl2_2, negm_2), x2, x3);
                float p0, p1, p2, p3;
                if (i % kPolyPeriodFp8 == kPolyPeriodFp8 - 1) {
                    exp2_poly_pair(x0, x1, p0, p1);
                    exp2_poly_pair(x2, x3, p2, p3);
                } else {
                    p0 = ptx::ex2_approx(x0);
                    p1 = ptx::ex2_approx(x1);
                    p2 = ptx::ex2_approx(x2);
                    p3 = ptx::ex2_approx(x3);
                }
                sum_a = ptx::fadd2(sum_a, ptx::f2_pack(p0, p1));
                sum_b = ptx::fadd2(sum_b, ptx::f2_pack(p2, p3));
                pk[i] = pack_e4m3x4(p0, p1, p2, p3);
                if (i % 2 == 0)
                    rq0 = add_e4m3x4_to_f32(rq0, pk[i]);
                else
                    rq1 = add_e4m3x4_to_f32(rq1, pk[i]);
            }
            ptx::tmem_st8(t_p + q * 8, pk);
            if ((q + 1) % (4 / kPParts) == 0 && q < 3) {  // a part of P is complete
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(L::bar_p_part(sbase, x, q / (4 / kPParts)));
            }
        }
        {
            float a0, a1, b0, b1;
            ptx::f2_unpack(sum_a, a0, a1);
            ptx::f2_unpack(sum_b, b0, b1);
            l_sum += (a0 + a1) + (b0 + b1);
            l_q += rq0 + rq1;
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before_sync();
        ptx::mbar_arrive(L::bar_p_ready(sbase, x));
    }
    if (!ok) return false;
    ok = __all_sync(0xffffffffu, bounded_wait(L::bar_o_done(sbase, x), (phases >> 1) & 1u, abort_flag, lim));
    if (!ok) return false;
    ptx::tc_fence_after_sync();
    // The pair's indices again (recomputed rather than kept live through the loop).
    int u_again = u;
    asm volatile("" : "+r"(u_again));
    const TilePair we = decode_pair(u_again, p);
    const int h = x ? we.h[1] : we.h[0];
    const bool store = row < we.len;
    const float inv = l_q > 0.0f ? 1.0f / l_q : 0.0f;
    // Row-segment stores from the staging area: TMA box stores measured 4 %
    // slower in this kernel (0.822 -> 0.855 ms on the 8192-token GQA workload).
    store_o_rows<kD>(p, sbase + L::kStg + (uint32_t)(x * 4 + warp_in_group) * 4096u, lane, t_o, inv,
                     r0 + warp_in_group * 32, we.len, we.start, h, nullptr);
    if (store) {
        const float lse = l_sum > 0.0f ? (m_ref + ptx::lg2_approx(l_sum)) * kLn2 : -INFINITY;
        const size_t idx = p.cu_seqlens ? (size_t)h * p.N + we.start + row : ((size_t)we.b * p.Hq + h) * p.N + row;
        p.lse[idx] = lse;
    }
    // O has been read: the next pair's first PV of this tile may overwrite it
    ptx::tc_fence_before_sync();
    ptx::mbar_arrive(L::bar_o_free(sbase, x));
    return true;
}

// The pairs of this CTA for one tile (tiles with no rows skipped).
__device__ __forceinline__ void softmax_role(const FwdParams& p, int x, int warp_in_group, int lane, uint32_t tmem,
                                             uint32_t sbase, volatile int* abort_flag) {
    // bit 0: s_full parity, bit 1: o_done parity, bits 2-3: unit queue index mod 4
    uint32_t phases = 0;
    while (true) {
        const int u = unit_take<Layout>(sbase, phases >> 2, abort_flag, p.wait_limit_ns);
        phases = (phases + 4u) & 15u;
        if (u < 0) break;
        const TilePair w = decode_pair(u, p);
        if (!(x ? w.active[1] : w.active[0])) continue;
        if (!softmax_unit(w, p, x, warp_in_group, lane, tmem, sbase, abort_flag, phases, u)) return;
        phases ^= 2u;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_fp8_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_vt, const FwdParams p) {
    using L = Layout;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    if (warp == kWarpProducer && lane == 0) {
        ptx::mbar_init(L::bar_q(sbase), 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(L::bar_kv_full(sbase, s), 1);
            ptx::mbar_init(L::bar_kv_empty(sbase, s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(L::bar_s_full(sbase, x), 1);
            ptx::mbar_init(L::bar_p_ready(sbase, x), 128);
            ptx::mbar_init(L::bar_o_done(sbase, x), 1);
        }
        ptx::mbar_init(L::bar_mma_final(sbase), 1);
        init_schedule_barriers<L>(sbase);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_vt);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (warp < 8) {
        ptx::setmaxnreg_inc<kRegsSoftmaxFp8>();
        softmax_role(p, warp / 4, warp % 4, lane, tmem, sbase, abort_flag);
    } else {
        ptx::setmaxnreg_dec<kRegsOtherFp8>();
        if (warp == kWarpProducer)
            producer(p, &tm_q, &tm_k, &tm_vt, sbase, abort_flag);
        else if (warp == kWarpMma)
            mma_role(p, tmem, sbase, abort_flag);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// V [tokens, Hkv, 128] e4m3 -> V^T [Hkv * 128 rows, vt_cols] with sequence b's
// keys at columns [vt_start(b), vt_start(b) + L_b) and zeros up to the next
// multiple of 128.  Grid (ceil(longest / 64), Hkv, B); 64 keys x 128 values
// per block through shared memory.
__global__ void __launch_bounds__(256) attn_vt_transpose_kernel(const uint8_t* v, uint8_t* vt, FwdParams p,
                                                                 long long vt_cols) {
    __shared__ uint8_t tile[64][kD + 4];
    const int b = blockIdx.z, g = blockIdx.y;
    const int start = p.cu_seqlens ? p.cu_seqlens[b] : b * p.N;
    const int end = p.cu_seqlens ? p.cu_seqlens[b + 1] : start + p.N;
    // boundaries that do not fit the call: nothing is read or written here (the
    // attention kernel skips the sequence and reports it)
    if (start < 0 || end < start || end > (p.cu_seqlens ? p.N : p.B * p.N) ||
        (long long)(end - start) > (long long)p.n_row_blocks * kBM)
        return;
    const int len = end - start;
    const int padded = (len + kBN - 1) / kBN * kBN;
    const int k0 = blockIdx.x * 64;
    if (k0 >= padded) return;
    const long long vs = vt_start(p, b);
    if (vs + padded > vt_cols) return;
    // load 64 keys x 128 bytes (16 bytes per thread per pass)
    for (int idx = threadIdx.x; idx < 64 * (kD / 16); idx += 256) {
        const int r = idx / (kD / 16), c = idx % (kD / 16);
        const int key = k0 + r;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (key < len) val = *reinterpret_cast<const uint4*>(v + ((size_t)(start + key) * p.Hkv + g) * kD + c * 16);
        const uint8_t* bytes = reinterpret_cast<const uint8_t*>(&val);
#pragma unroll
        for (int e = 0; e < 16; ++e) tile[r][c * 16 + e] = bytes[e];
    }
    __syncthreads();
    // write 128 rows x 64 keys (4 bytes per thread per pass)
    for (int idx = threadIdx.x; idx < kD * 16; idx += 256) {
        const int row = idx / 16, c4 = idx % 16;
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) word |= static_cast<uint32_t>(tile[c4 * 4 + e][row]) << (8 * e);
        *reinterpret_cast<uint32_t*>(vt + ((size_t)g * kD + row) * (size_t)vt_cols + vs + k0 + c4 * 4) = word;
    }
}

}  // namespace fp8
}  // namespace attn

/*
 * attn.h -- C ABI of the B200 (sm_100a) exact fused attention forward pass.
 *
 * Operation ("FlashAttention", ozercemkelahmet.com/tools/flashattention,
 * sections "What it is" and "How it works", Steps 1-5):
 *     O = softmax(scale * Q K^T + mask) V,   LSE = log of each row's softmax
 *     normaliser (natural log, including the scale)
 * computed tile by tile with an online softmax, so the score matrix never
 * reaches device memory.  The result is exact up to rounding order: inputs are
 * bf16, scores, softmax statistics and the O accumulator are fp32, the weights
 * P are rounded to bf16 for the second product ("How it works", Step 8), and O
 * is rounded once to bf16 (round to nearest even).
 *
 * Masks ("Flash Attention" skill page, skillmd.com, "Workflow 2",
 * window_size=(left, right) with -1 for no limit; explainer page, Step 6):
 *     key j is visible to query i of the same sequence iff
 *         (window_left  < 0 || j >= i - window_left) &&
 *         (window_right < 0 || j <= i + window_right)
 *     and causal != 0 forces window_right = 0.  Bounds are inclusive.
 * Grouped / multi-query attention (explainer page, "Variants you may meet"):
 *     query head h reads key/value head h / (Hq / Hkv); Hkv == 1 is MQA.
 * Packed variable-length batches ("Flash Attention 2 in HuggingFace",
 * cloudcodetree.com, "Stack it with sequence packing"): cu_seqlens holds
 * cumulative sequence boundaries and attention never crosses them.
 *
 * Threading and ownership: every buffer belongs to the caller.  The library
 * keeps no per-call state and allocates no device memory; calls are
 * asynchronous on the given stream and may be issued from several host
 * threads.  The only global state is one device-side status word per device
 * (see attn_device_status).
 */
#ifndef EXACT_ATTENTION_B200_ATTN_H
#define EXACT_ATTENTION_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t / CUstream; NULL means the legacy default stream */

enum attn_status {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,          /* a required pointer is NULL                        */
    ATTN_ERR_SHAPE = -2,         /* B, Hq, Hkv <= 0, N < 0, Hq % Hkv != 0, sizes that
                                    overflow 32-bit coordinates, max_seqlen < 0      */
    ATTN_ERR_WINDOW = -3,        /* window_left or window_right < -1                  */
    ATTN_ERR_UNSUPPORTED = -4,   /* d not in {64, 128}, or the device is not sm_100   */
    ATTN_ERR_ALIGN = -5,         /* q, k, v, o not 16-byte aligned or lse not 4-byte  */
    ATTN_ERR_CUDA = -6,          /* a CUDA runtime / driver call failed               */
    ATTN_ERR_SCALE = -7,         /* scale is not a finite number > 0                  */
    ATTN_ERR_WORKSPACE = -8,     /* attn_fwd_host: workspace missing or too small     */
    ATTN_ERR_DEVICE_TIMEOUT = -9, /* reported by attn_device_status(): a kernel wait
                                     ran past its time limit and the kernel gave up  */
    ATTN_ERR_PAGE = -10,         /* reported by attn_device_status(): attn_decode met a
                                    page-table entry outside [0, num_pages)          */
    ATTN_ERR_SEQLENS = -11       /* reported by attn_device_status(): a packed batch's
                                    cu_seqlens do not fit the call (a boundary outside
                                    [0, N] or decreasing, or a sequence longer than
                                    max_seqlen); that sequence was skipped            */
};

/*
 * attn_fwd -- fused exact attention forward on device buffers.
 *
 * Dense mode (cu_seqlens == NULL): B sequences of N tokens each.
 *   q   [B, N, Hq,  d] bf16      k, v [B, N, Hkv, d] bf16
 *   o   [B, N, Hq,  d] bf16      lse  [B, Hq, N] fp32
 *   max_seqlen is ignored.
 * Packed mode (cu_seqlens != NULL): B sequences packed back to back,
 *   N = total number of tokens = cu_seqlens[B].
 *   cu_seqlens: device int32[B + 1], cu_seqlens[0] = 0, non-decreasing.
 *   q   [N, Hq,  d] bf16         k, v [N, Hkv, d] bf16
 *   o   [N, Hq,  d] bf16         lse  [Hq, N] fp32
 *   max_seqlen >= the longest sequence (used only to size the launch).  The
 *   host never reads cu_seqlens.  The kernel checks each sequence's
 *   boundaries before it reads or writes anything of it: a boundary outside
 *   [0, N], a decreasing pair, or a sequence longer than max_seqlen (rounded
 *   up to 128 rows) is skipped -- its rows of o and lse are left as they were
 *   -- and attn_device_status() then reports ATTN_ERR_SEQLENS.
 * All tensors are contiguous (row-major in the order shown).
 *   d: head dimension, 64 or 128.
 *   scale: finite, > 0 (pass 1/sqrt(d) for the usual scaling).
 *   causal: nonzero -> key j visible only if j <= i (overrides window_right).
 *   window_left / window_right: -1 (unlimited) or >= 0.
 *   stream: CUDA stream the work is ordered on.
 * Returns ATTN_OK after enqueueing the kernel (or when N == 0, with nothing
 * enqueued), or a negative attn_status; on error nothing is enqueued.
 * Device-side failures (a bounded wait that timed out) are reported through
 * attn_device_status() once the stream has been synchronised.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int N, int d, float scale, int causal, int window_left, int window_right,
             const int32_t* cu_seqlens, int max_seqlen, struct CUstream_st* stream);

/*
 * attn_fwd_fp8 -- attn_fwd with 8-bit floating-point inputs ("Flash Attention"
 * skill page, Workflow 3: q, k, v converted to float8_e4m3 and passed to the
 * fused kernel; "FlashAttention" explainer page, How it works, Step 8:
 * 8-bit products with fp32 statistics).
 *   q [tokens, Hq, 128], k and v [tokens, Hkv, 128]: e4m3 (OCP "E4M3FN": one
 *   sign, four exponent, three mantissa bits, bias 7, no infinities), one byte
 *   each, 16-byte aligned; the values themselves, with no scale factors.
 *   o bf16 and lse fp32 as in attn_fwd; every other argument as in attn_fwd.
 *   d must be 128 (ATTN_ERR_UNSUPPORTED otherwise).
 * Both products take e4m3 operands with fp32 accumulation: the weights P are
 * rounded to e4m3 (round to nearest even) for O += P V and O is divided by the
 * sum of those rounded weights; the LSE uses the fp32 weights.
 * workspace: device, 256-byte aligned, >= attn_fwd_fp8_workspace_bytes(...):
 * holds V transposed per key/value head, each sequence padded to 128 keys.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                 int Hkv, int N, int d, float scale, int causal, int window_left, int window_right,
                 const int32_t* cu_seqlens, int max_seqlen, void* workspace, size_t workspace_bytes,
                 struct CUstream_st* stream);

/* Device workspace attn_fwd_fp8 needs (packed: nonzero when cu_seqlens is passed;
 * 0 for d != 128 or bad sizes). */
size_t attn_fwd_fp8_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed);

/*
 * attn_fwd_accumulate -- attn_fwd whose result is merged into an fp32
 * accumulator instead of being written: the building block of attention split
 * along the keys ("Long context beyond a single GPU": devices compute partial
 * attention and merge the partial results with the online-softmax rule of
 * "How it works", Step 3).
 *   o_acc   [tokens, Hq, d] fp32 and lse_acc (laid out like lse) hold a
 *           partial result over some other keys; a row whose lse_acc is -inf
 *           holds nothing yet, and its o_acc values are not read (start from
 *           lse_acc = -inf; o_acc may then be uninitialised).
 * With (O', L') this call's attention of q over k, v (natural-log LSE), each
 * row becomes  L = log(e^lse_acc + e^L'),
 *              o_acc = (e^lse_acc o_acc + e^L' O') / e^L,   lse_acc = L,
 * so that after all key blocks o_acc and lse_acc are attn_fwd's O (before
 * rounding) and LSE for all the keys.  Every other argument, rule and status is
 * attn_fwd's; o_acc must be 16-byte aligned.
 */
int attn_fwd_accumulate(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc,
                        int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                        int window_left, int window_right, const int32_t* cu_seqlens,
                        int max_seqlen, struct CUstream_st* stream);

/* Round n fp32 values (an accumulator) to bf16, nearest even; both buffers
 * 16-byte aligned device memory.  Asynchronous on `stream`. */
int attn_acc_to_bf16(const float* o_acc, void* o, long long n, struct CUstream_st* stream);

/*
 * attn_fwd_host_workspace_bytes -- device workspace needed by attn_fwd_host
 * for these sizes (q, k, v, o, lse and cu_seqlens copies, 256-byte aligned).
 * packed: nonzero when cu_seqlens will be passed.  Returns 0 on bad sizes.
 */
size_t attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed);

/*
 * attn_fwd_host -- the same operation on HOST buffers.
 * Copies q, k, v (and cu_seqlens) host -> device into the caller's device
 * workspace, runs attn_fwd on it, and copies o and lse device -> host, all
 * ordered on `stream`.  The call returns after enqueueing; the host outputs
 * are valid once the stream is synchronised.  Pinned (page-locked) host
 * buffers make the copies asynchronous.  The layouts are those of attn_fwd;
 * cu_seqlens is a host int32[B + 1] array here.
 * workspace: device buffer of at least attn_fwd_host_workspace_bytes(...).
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int Hq, int Hkv, int N, int d, float scale, int causal, int window_left,
                  int window_right, const int32_t* cu_seqlens, int max_seqlen, void* workspace,
                  size_t workspace_bytes, struct CUstream_st* stream);

/*
 * attn_bwd -- gradients of attn_fwd's output with respect to q, k and v
 * ("FlashAttention" explainer page, How it works, Step 5, and "Backward pass
 * in a bit more detail": the score tiles are recomputed from q and k and the
 * weights rebuilt from each row's saved log-sum-exp; key/value gradients
 * accumulate over query blocks, query gradients over key blocks).
 *
 * With P = softmax(scale * q k^T + mask) (from lse), dP = dout v^T,
 * D = rowsum(dout * o) and dS = P * (dP - D):
 *     dq = scale * dS k,   dk = scale * dS^T q,   dv = P^T dout,
 * dk and dv summed over the query heads that share a key/value head.
 *   q, o, dout, dq [tokens, Hq, d] bf16;  k, v, dk, dv [tokens, Hkv, d] bf16;
 *   lse: the forward's fp32 log-sum-exp ([B, Hq, N] dense, [Hq, T] packed).
 *   Sizes, masks, cu_seqlens and max_seqlen as in attn_fwd (same values as the
 *   forward call that produced o and lse).
 *   workspace: device, 256-byte aligned, >= attn_bwd_workspace_bytes(...)
 *   (holds D).  P and dS are rounded to bf16 as operands of the products,
 *   accumulation is fp32, outputs are rounded once to bf16.
 * Asynchronous on `stream`; allocates nothing.  Returns ATTN_OK (also for
 * N == 0, with nothing enqueued) or a negative attn_status; device-side
 * timeouts are reported by attn_device_status().
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
             float scale, int causal, int window_left, int window_right, const int32_t* cu_seqlens,
             int max_seqlen, void* workspace, size_t workspace_bytes, struct CUstream_st* stream);

/* Device workspace attn_bwd needs (packed: nonzero when cu_seqlens is passed). */
size_t attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int packed);

/*
 * attn_decode -- attention of the newest tokens against a key/value cache,
 * split along the cache ("FlashAttention" explainer page, How it works, Step 9:
 * decoding with a cache of past keys and values; the slices' partial results
 * are merged by the online-softmax rescaling; paged layouts: "Use the decoding
 * kernels for serving").
 *
 *   q       [B, Nq, Hq, d] bf16: the Nq (1..16) newest tokens of each sequence
 *   k_cache, v_cache [num_pages, page_size, Hkv, d] bf16 (a pool of pages)
 *   block_table  device int32 [B, pages_per_seq]: page of logical page p of
 *           sequence b; NULL means page b * pages_per_seq + p, i.e. a contiguous
 *           cache [B, pages_per_seq * page_size, Hkv, d] (num_pages must then
 *           be >= B * pages_per_seq).  Entries for pages past a sequence's
 *           length are never read.  An entry outside [0, num_pages) is not
 *           followed: attn_device_status() then reports ATTN_ERR_PAGE.
 *   cache_seqlens device int32 [B]: keys held by sequence b, the new tokens
 *           included (Nq <= cache_seqlens[b] <= page_size * pages_per_seq).
 *           Cached keys and values at positions below that length must be
 *           finite; slots past it are never used, whatever they hold.
 *   o       [B, Nq, Hq, d] bf16;  lse [B, Hq, Nq] fp32 (natural log).
 * Query row i of sequence b sits at position pos = cache_seqlens[b] - Nq + i;
 * key j is visible iff (window_left < 0 || j >= pos - window_left) &&
 * (window_right < 0 || j <= pos + window_right), causal forcing window_right = 0.
 *   page_size: any >= 1; a multiple of 8 (or a contiguous cache) takes the
 *           TMA / tensor-core kernel, other sizes a slower gather kernel.
 *   num_splits: number of slices of the cache (>= 1; see
 *           attn_decode_default_splits).  With more than one slice, partial
 *           results go to `workspace` (device, 256-byte aligned, at least
 *           attn_decode_workspace_bytes(...) bytes; may be NULL when that is 0).
 * Asynchronous on `stream`; allocates nothing.  The host never reads
 * cache_seqlens or block_table; their contents are the caller's responsibility.
 * Returns ATTN_OK or a negative attn_status (ATTN_ERR_UNSUPPORTED for Nq > 16,
 * ATTN_ERR_SHAPE when num_pages * page_size exceeds 2^31 - 1).
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                const int32_t* cache_seqlens, const int32_t* block_table, int B, int Hq, int Hkv,
                int Nq, int d, int page_size, int pages_per_seq, int num_pages, float scale,
                int causal, int window_left, int window_right, int num_splits, void* workspace,
                size_t workspace_bytes, struct CUstream_st* stream);

/*
 * attn_decode_noalloc -- attn_decode without a workspace argument and without
 * allocating anything.  The pages have no counterpart to this entry point: it
 * exists for callers that must not allocate device memory while they run, such
 * as a serving loop that gives nearly all of HBM to its key/value page pool at
 * start-up, or a latency-bound decode step, where cudaMalloc / cudaFree (which
 * can block on and synchronise with the device, and fail once the pool holds
 * the memory) or a framework allocator would stall or fail the step.
 *
 * Arguments and result are those of attn_decode.  The slice partials go to one
 * fixed device array of ATTN_DECODE_NOALLOC_SCRATCH_BYTES (8 MiB) inside the
 * library, per device; a call whose attn_decode_workspace_bytes(...) exceeds
 * that returns ATTN_ERR_WORKSPACE before doing anything (use fewer slices, or
 * attn_decode with a workspace).  Every argument is checked as attn_decode
 * checks it before the array is touched.  A single slice uses no scratch.
 *
 * The first call on a device that needs the scratch looks up the array's
 * address (cudaGetSymbolAddress, with that device current) and keeps it; make
 * that first call before any stream capture.  All calls on a device share the
 * one array and it keeps the last call's contents (nothing in it needs to
 * start at zero): calls that may overlap on the GPU -- other streams, other
 * host threads -- race on it, so order them on one stream.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* The size of that array as the library was built (ATTN_DECODE_NOALLOC_SCRATCH_BYTES):
 * bindings read it here instead of copying the constant.  Host arithmetic only. */
size_t attn_decode_noalloc_scratch_bytes(void);

int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                        float* lse, const int32_t* cache_seqlens, const int32_t* block_table,
                        int B, int Hq, int Hkv, int Nq, int d, int page_size, int pages_per_seq,
                        int num_pages, float scale, int causal, int window_left, int window_right,
                        int num_splits, struct CUstream_st* stream);

/* Device workspace attn_decode needs for these sizes (0 when one slice). */
size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int page_size,
                                   int pages_per_seq, int num_splits);

/* A slice count for these sizes: the smallest that occupies at least half of
 * the current device's CTA slots (two per SM) with a last wave at least half
 * full (or at least four waves), keeping >= 256 keys per slice
 * (max_cache_len = page_size * pages_per_seq).  Without a device it assumes
 * 148 SMs. */
int attn_decode_default_splits(int B, int Hq, int Hkv, int Nq, int max_cache_len);

/* Static text for a status code (never NULL). */
const char* attn_status_string(int status);

/*
 * attn_device_status -- read and clear the status words of the current device.
 * Call after synchronising the streams that ran attn_fwd / attn_decode.
 * Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT if any kernel since the last call
 * gave up on a bounded wait, ATTN_ERR_PAGE if attn_decode met a page-table
 * entry outside the cache (the outputs of that call are then undefined),
 * ATTN_ERR_SEQLENS if a packed call's cu_seqlens did not fit its N or
 * max_seqlen (the sequences concerned were skipped), or ATTN_ERR_CUDA if a
 * word could not be read.
 */
int attn_device_status(void);

/*
 * attn_selftest_bounded_wait -- health check of the kernels' failure path.
 * Launches one tiny block that waits on a barrier nothing will ever signal,
 * with a limit of limit_ns nanoseconds (clamped to [1 us, 2 s]); the wait
 * must give up, record ATTN_ERR_DEVICE_TIMEOUT in the status word and return.
 * The GPU is never faulted or hung.  Returns the launch status.
 */
int attn_selftest_bounded_wait(uint64_t limit_ns, struct CUstream_st* stream);

/*
 * attn_selftest_exp2_poly -- evaluates on the GPU the exponential that the
 * forward kernels take from the FMA pipe for part of the softmax weights
 * 2^(s - m) ("FlashAttention" explainer page, How it works, Step 3): with
 * n = rint(x) and f = x - n in [-1/2, 1/2], 2^f from a cubic fitted for
 * minimax relative error (csrc/gen_exp2_poly.py) times 2^n.
 *   x, y: device float[n], 4-byte aligned; y[i] = 2^x[i] for x[i] <= 8 (the
 *   kernels never pass more).  Relative error <= exp2poly::kMaxRelError (plus
 *   fp32 rounding) where 2^x is a normal fp32 number, exact powers of two at
 *   integer x, and exactly 0 for x < -126.5 and for x = -inf (a masked key).
 * Asynchronous on `stream`.  Returns ATTN_OK, ATTN_ERR_SHAPE (n < 0),
 * ATTN_ERR_NULL, ATTN_ERR_ALIGN, ATTN_ERR_UNSUPPORTED or ATTN_ERR_CUDA.
 */
int attn_selftest_exp2_poly(const float* x, float* y, long long n, struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_B200_ATTN_H */

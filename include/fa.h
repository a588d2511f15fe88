/*
 * fa.h -- C ABI of the B200 (sm_100a) exact IO-aware attention library.
 *
 * What the library computes. Exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T) V
 * ("Walk through what FlashAttention does differently from standard attention",
 * zenaique short answer, first paragraph: the textbook formula with scale 1/sqrt(d_k);
 * FlashAttention returns the same output, only floating-point rounding differs).
 * The score matrix is produced tile by tile in on-chip memory and merged with the
 * online softmax (running max m, running denominator l, rescaled output accumulator;
 * "FlashAttention Kernel & Online Softmax" card, first paragraph, and the
 * "FlashAttention" blog's mechanics section). It never reaches device memory.
 * The forward pass also saves each row's log-sum-exp (LSE), which folds the
 * saved statistics m and l into one number. The backward pass recomputes the
 * scores and probabilities from Q, K and that LSE instead of storing them (same
 * short answer, second paragraph).
 *
 * Conventions shared by every entry point.
 *   Layout    Q, O, dO, dQ: [B, Hq, N, d]; K, V, dK, dV: [B, Hkv, N, d]; all
 *             contiguous, row-major, d innermost. LSE and the backward's D: [B, Hq, N].
 *   Types     "bf16" arguments point to IEEE bfloat16 values (2 bytes each);
 *             LSE is float32, natural logarithm.
 *   Heads     Grouped-query attention: query head h reads key/value head
 *             h / (Hq / Hkv). Hq must be a multiple of Hkv.
 *   Causal    causal != 0: query i sees keys j <= i (square N x N). Otherwise all keys.
 *   Scale     scale > 0 and finite, applied to Q K^T (callers normally pass 1/sqrt(d)).
 *   Memory    Every pointer is DEVICE memory owned by the caller. Each pointer
 *             must be 16-byte aligned. Outputs must not alias inputs.
 *   Streams   `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *             asynchronous: they enqueue work and return before it completes.
 *             They neither allocate nor synchronise, so fa_fwd, fa_bwd and
 *             fa_decode can be captured in a CUDA graph once one eager call on
 *             the device has loaded the kernels (fa_get_status synchronises and
 *             stays outside a capture).
 *   Errors    A negative return code means nothing was launched and no output
 *             was touched. FA_OK means the work was enqueued. A failure found on
 *             the device is recorded in a device status word; fa_get_status()
 *             reads it. On the device, every wait is bounded. A wait that runs
 *             out records FA_ERR_DEVICE_TIMEOUT and the kernel returns early; it
 *             never traps or spins forever.
 *   Sizes     B, Hq, Hkv >= 1; N >= 0 (N == 0 is a no-op that returns FA_OK);
 *             B*Hq*N < 2^31.
 *   Contexts  The library caches, per device, the device addresses of its own
 *             __device__ variables (the status word, fa_bwd_noalloc's scratch)
 *             on first use. cudaDeviceReset() destroys the context those
 *             addresses belong to: do not call into the library on a device
 *             after resetting it in the same process.
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1,    /* a size, scale or pointer argument is invalid        */
  FA_ERR_UNSUPPORTED = -2,    /* valid, but not a supported shape (e.g. d not 64/128) */
  FA_ERR_ALIGNMENT = -3,      /* a pointer is not 16-byte aligned                     */
  FA_ERR_LAUNCH = -4,         /* the CUDA runtime refused a launch or a query         */
  FA_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait ran out                   */
  FA_ERR_NO_DEVICE = -6       /* no sm_100 device is current                          */
} fa_status_t;

/*
 * fa_fwd -- bf16 forward pass on the tensor cores.
 *
 * Computes O = softmax(scale * Q K^T) V tile by tile with the online softmax
 * ("FlashAttention Kernel & Online Softmax": m_new = max(m, x),
 * l_new = l e^(m - m_new) + e^(x - m_new), output rescaled by e^(m - m_new) and
 * normalised by 1/l at the end). It also writes lse[i] = m_i + ln(l_i) for
 * every row (the statistics that the short answer's second paragraph says
 * are saved for the backward pass).
 *   q [B,Hq,N,d] bf16, k/v [B,Hkv,N,d] bf16   inputs (read only)
 *   o [B,Hq,N,d] bf16                          output, round-to-nearest-even
 *   lse [B,Hq,N] float32                       output
 *   d must be 64, 128 or 256 (fa_bwd too). Arithmetic: bf16 operands, fp32
 *   accumulation; the probabilities P are rounded to bf16 before the P V product.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * fa_fwd_fp8 -- forward pass with E4M3 inputs (8-bit tensor cores).
 *
 * The third FlashAttention generation adds an FP8 path (E4M3 and E5M2) worth
 * a further 1.5-2x (FlashAttention family short answer, second paragraph, and
 * the version table on the same page). This call computes the forward of
 * fa_fwd on inputs stored as E4M3 bytes with one scale per tensor, whose real
 * values are
 *   Q = descale_q * q,  K = descale_k * k,  V = descale_v * v,
 * and O = softmax(scale * Q K^T) V, lse = m + ln(l) as in fa_fwd.
 *   q [B,Hq,N,d], k/v [B,Hkv,N,d]  E4M3 bytes (OCP FP8, finite max 448), read only
 *   descale_q/k/v                  positive finite float scales
 *   o [B,Hq,N,d] bf16, lse [B,Hq,N] float32  outputs, as in fa_fwd
 *   d must be 128. Arithmetic: E4M3 products with fp32 accumulation for S and
 *   for P V; the probabilities P are rounded to E4M3 (values below 2^-10 of the
 *   tile's reference maximum become 0) before the P V product, while the row
 *   sums l add the unrounded fp32 values.
 * Returns the codes of fa_fwd; FA_ERR_INVALID_ARG also for a descale that is
 * not positive and finite.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k, float descale_v,
               void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * fa_fwd_e5m2 -- fa_fwd_fp8 with the inputs stored as E5M2 bytes (OCP FP8: 2
 * mantissa bits, finite max 57344), the page's other FP8 format. Arguments,
 * layouts and return codes are those of fa_fwd_fp8; P is rounded to E5M2 (values
 * below 2^-17 of the tile's reference maximum become 0), so both operands of
 * every MMA are E5M2.
 */
int fa_fwd_e5m2(const void* q, const void* k, const void* v, float descale_q, float descale_k, float descale_v,
                void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * fa_decode_workspace_bytes -- device scratch that fa_decode needs.
 *
 * A (batch, kv head) group has rows = (Hq / Hkv) * Nq query rows. Up to 32 rows
 * the group is one unit; above that its rows are cut into n_rb = ceil(rows / 128)
 * row blocks, each a unit of its own. The split kernel cuts all units' 128-key
 * chunks, laid end to end, into n_ctas equal slices; each piece of a slice inside
 * one unit has a slot holding a float32 partial output [slot_rows, d] and partial
 * LSE [slot_rows], where slot_rows = rows for n_rb = 1 and 128 otherwise, and 128
 * at d = 64 with rows <= 64 (two partial rows per query row, one per half of
 * every 128-key chunk); there
 * are units + n_ctas - 1 slots, units = B*Hkv*n_rb. The workspace holds all slots'
 * outputs (padded to a multiple of 256 bytes), then all their LSEs. n_ctas is 148
 * for num_splits <= 0 (a fixed rule of the sizes, so no device is needed here),
 * else units*num_splits, and never more than the chunks. Returns 0 for sizes
 * fa_decode rejects.
 */
size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits);

/*
 * fa_decode -- attention of Nq new queries against a cache of Nk keys and values,
 * split along the keys (decode).
 *
 * In serving the kernel runs against a KV cache, and the decode step is bound by
 * reading that cache ("FlashAttention Kernel & Online Softmax" card: KV cache and
 * the decode bandwidth bottleneck). The queries are the last Nq positions of the
 * sequence: query i is at position Nk - Nq + i and, when causal != 0, sees keys
 * j <= Nk - Nq + i (Nq = Nk gives fa_fwd's square causal mask). Each key split
 * computes a partial softmax over its keys; the partials are combined with the
 * online-softmax merge (running max, rescaled denominators: the update of the
 * card's first paragraph), LSE = log sum_s e^(LSE_s), O = sum_s e^(LSE_s - LSE) O_s,
 * by a second kernel (one warp per query row).
 *   q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d] bf16   inputs (read only)
 *   o [B,Hq,Nq,d] bf16, lse [B,Hq,Nq] float32   outputs, as in fa_fwd
 *   workspace   at least fa_decode_workspace_bytes(..., num_splits) bytes of
 *               device memory, 256-byte aligned, contents on entry irrelevant
 *   num_splits  work split: <= 0 gives one CTA per SM of a 148-SM part; > 0 gives
 *               units*num_splits CTAs (about num_splits key splits per group, or
 *               per row block of 128 rows); never more CTAs than 128-key chunks
 *   d must be 64 or 128, else FA_ERR_UNSUPPORTED; causal with Nq > Nk is
 *   FA_ERR_INVALID_ARG. At d = 128 a group of up to 32 query rows is served by
 *   one CTA at a time with the rows as the MMA's N, so its keys are read once;
 *   larger groups, and all groups at d = 64, take 128-row blocks as the MMA's M,
 *   and their keys are read once per block.
 *   Arithmetic: bf16 operands, fp32 accumulation; P is rounded to bf16 before
 *   the P V product; the partials stay fp32.
 */
int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
              int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale, int num_splits,
              void* stream);

/*
 * fa_fwd_f32 -- float32 forward pass (CUDA cores, fp32 throughout).
 *
 * The same computation as fa_fwd, on float32 q, k, v and o. Tiles of queries
 * and keys are staged in shared memory and merged with the same online
 * softmax. d must be a multiple of 4 and at most 128.
 */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse,
               int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * fa_bwd_workspace_bytes -- device scratch that fa_bwd needs.
 *
 * The workspace holds D = rowsum(dO o O) (float32 [B,Hq,N]) and a float32
 * accumulator for dQ ([B,Hq,N,d]). It grows linearly in N: the backward pass
 * never stores an N x N matrix. Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/*
 * fa_bwd -- bf16 backward pass by recomputation.
 *
 * Gradients of L = sum(O o dO) with respect to Q, K and V. The backward pass
 * recomputes S = scale Q K^T and P = exp(S - LSE) tile by tile from the saved
 * LSE instead of storing them (short answer, second paragraph). With
 * D_i = sum_c dO_ic O_ic and dS = P o (dP - D), where dP = dO V^T:
 *   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
 * With grouped-query attention, dK and dV sum over the query heads of a group.
 *   q, k, v, o, dout  bf16 inputs (o and lse as written by fa_fwd)
 *   lse               float32 [B,Hq,N] input
 *   dq [B,Hq,N,d], dk, dv [B,Hkv,N,d]  bf16 outputs
 *   workspace         at least fa_bwd_workspace_bytes(...) bytes of device
 *                     memory, 256-byte aligned; its contents on entry do not matter.
 *                     It must not be used by another call in flight at the same time.
 *   d must be 64, 128 or 256 (d = 256 runs the query loop twice, once per half of
 *   the head dim). dQ is accumulated with float32 atomics, so its last
 *   bits can vary from run to run; dK and dV are deterministic.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, void* workspace,
           int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * The three phases fa_bwd runs, in this order, on one stream. They exist so a
 * caller (or a profiler) can time or interleave them; fa_bwd(...) is exactly
 * fa_bwd_preprocess, then fa_bwd_main, then fa_bwd_convert with the same arguments.
 *   fa_bwd_preprocess  D_i = sum_c dO_ic O_ic into the workspace, and zeroes
 *                      the workspace's fp32 dQ accumulator.
 *   fa_bwd_main        recomputes S and P per tile and accumulates dK, dV
 *                      (written as bf16) and the fp32 dQ accumulator.
 *   fa_bwd_convert     dq = bf16(scale * dQ accumulator).
 * Arguments, layouts and error codes are those of fa_bwd; each phase only reads
 * the pointers it needs (the others may be NULL).
 */
int fa_bwd_preprocess(const void* o, const void* dout, void* workspace, int B, int Hq, int Hkv, int N, int d,
                      void* stream);
int fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dout, void* dk, void* dv,
                void* workspace, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);
int fa_bwd_convert(void* dq, const void* workspace, int B, int Hq, int Hkv, int N, int d, float scale, void* stream);

/*
 * fa_bwd_noalloc -- fa_bwd for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call: it is a property of this
 * library's interface, not of the attention method. Some callers cannot call
 * cudaMalloc: plugins whose host application owns every device allocation,
 * serving loops that must not hit cudaMalloc's implicit synchronisation, and
 * fixed-budget deployments that size all device memory up front. They cannot
 * provide fa_bwd's workspace. This variant computes exactly what fa_bwd
 * computes, with the same arguments except the workspace: its scratch (D and
 * the fp32 dQ accumulator) lives in a static device array of
 * FA_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds until
 * the process exits. The call itself allocates nothing.
 *   Limit     fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) must not exceed
 *             FA_NOALLOC_SCRATCH_BYTES (about B*Hq*N*(d+1)*4 bytes); larger
 *             problems return FA_ERR_UNSUPPORTED and launch nothing.
 *   First use The first call on each device looks up the array's device address
 *             (which loads the library's kernels on that device). Make that
 *             first call before any stream capture.
 *   Sharing   All calls on a device share the one array, which keeps the last
 *             call's contents; each call re-initialises what it reads. Calls
 *             whose work overlaps on the GPU (e.g. on two streams) race on it
 *             and give wrong results: serialise them.
 */
#define FA_NOALLOC_SCRATCH_BYTES (64ull << 20)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                   void* stream);

/*
 * fa_get_status -- synchronise `stream`, then return and clear the device
 * status word of the current device (FA_OK or the first device-side error
 * since the last call). Returns FA_ERR_LAUNCH if the stream reports a CUDA error.
 */
int fa_get_status(void* stream);

/* fa_get_progress -- where each CTA of the last forward or backward main-kernel
 * launch on the current device got to: a diagnostic for a launch that reported
 * FA_ERR_DEVICE_TIMEOUT (the failure-detection side of the bounded waits; the
 * pages describe no such record). Word i belongs to CTA i: for the forward, the
 * number of P V products CTA i had issued (both of its query tiles, every work
 * unit it ran); for the backward main kernel, the number of query tiles whose
 * dV += P^T dO it had issued. Each CTA sets its word to 0 when it starts; words
 * of CTAs that did not run in the last launch keep older values. CTAs with index
 * 65536 or more keep no record.
 *   out     host buffer of n unsigned words; n is clamped to 65536.
 * Synchronises `stream`, then copies. Returns the number of words copied, or a
 * negative fa_status_t (FA_ERR_INVALID_ARG for a null buffer or n < 0). */
int fa_get_progress(unsigned* out, int n, void* stream);

/* fa_set_wait_budget_ns -- budget of each bounded device-side wait (default
 * 2e9 ns). Kernels launched afterwards use the new value. Values outside
 * [1e5, 6e10] ns are clamped to that range. */
void fa_set_wait_budget_ns(uint64_t ns);

/*
 * fa_selftest_wait_timeout -- failure-detection self test. Launches one block
 * that waits on a shared-memory barrier that nothing ever completes, using a
 * budget of `budget_ns`. The bounded wait must run out, record
 * FA_ERR_DEVICE_TIMEOUT and return. The call synchronises `stream` and returns
 * the status it read (FA_ERR_DEVICE_TIMEOUT when the mechanism works). It
 * also clears the status word.
 */
int fa_selftest_wait_timeout(uint64_t budget_ns, void* stream);

/* fa_error_string -- static text for a status code (never NULL). */
const char* fa_error_string(int code);

/* fa_version -- library version as 10000*major + 100*minor + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FA_B200_H_ */

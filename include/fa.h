/*
 * fa.h - exact IO-aware attention for NVIDIA B200 (sm_100a), C ABI.
 *
 * What is computed. For every batch b and query head h,
 *     S = scale * Q K^T            (masked: S_ij = -inf for j > i when causal)
 *     P = softmax(S) row by row,   O = P V,
 *     L_i = log sum_j exp(S_ij)    (natural log, one fp32 per query row)
 * which is the attention of "FlashAttention: IO-aware exact attention"
 * (daily-term page, "NAIVE ATTENTION vs FLASHATTENTION" diagram, NAIVE box
 * for the definition, FLASH box for the tiled online-softmax form and the
 * per-row logsumexp it keeps). The forward never writes the N x N scores to
 * memory; the backward rebuilds P from Q, K and L on chip (same page, "Four
 * ideas" list, item "Recomputation in the backward pass").
 * Grouped-query attention: query head h reads KV head h / (Hq / Hkv).
 *
 * Layout (all row-major, innermost dimension last, no padding):
 *     q, o, dout, dq : bf16 [B][Hq][N][d]
 *     k, v, dk, dv   : bf16 [B][Hkv][N][d]
 *     lse            : fp32 [B][Hq][N]
 * Supported: d in {64, 128}; Hq a multiple of Hkv; N >= 1; scale finite and
 * > 0; every pointer 16-byte aligned; device of compute capability 10.0
 * (B200, sm_100a).
 *
 * Ownership. Every pointer is device memory allocated and owned by the
 * caller; the library never allocates or frees device memory and keeps no
 * pointer after a call returns. Calls are asynchronous on `stream` (a
 * cudaStream_t; NULL means the legacy default stream) and use the current
 * CUDA device. Outputs are overwritten (dk and dv are not accumulated into).
 *
 * Errors. A nonzero status is returned before anything is launched when an
 * argument is invalid (FA_ERR_INVALID_ARGUMENT) or a shape or device is not
 * supported (FA_ERR_UNSUPPORTED); no output is touched in that case.
 * FA_ERR_CUDA means a CUDA call failed while launching (the text of the CUDA
 * error is available through fa_status_string until the next call on this
 * thread). Every wait inside the kernels is bounded by a watchdog; a wait
 * that runs out records a device error word instead of hanging, and
 * fa_check_device_error reports it as FA_ERR_TIMEOUT.
 *
 * Thread safety: calls may be made from several host threads. The only
 * shared state is a per-device cache of the device check and of the
 * address of the error word.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_OK 0
#define FA_ERR_INVALID_ARGUMENT 1
#define FA_ERR_UNSUPPORTED 2
#define FA_ERR_CUDA 3
#define FA_ERR_TIMEOUT 4

/*
 * Forward pass: o = softmax(scale * q k^T [causal]) v and lse = row
 * logsumexp (natural log). Source: "FlashAttention: IO-aware exact
 * attention", FLASH box of the "NAIVE ATTENTION vs FLASHATTENTION" diagram
 * (tiled loop with running max m and sum l; O written once plus one
 * logsumexp per row) and the "PREFILL PATH" diagram (128-row Q blocks,
 * 128-column K/V blocks).
 *   q [B][Hq][N][d], k, v [B][Hkv][N][d]  (bf16, read only)
 *   o [B][Hq][N][d] (bf16, written), lse [B][Hq][N] (fp32, written)
 *   causal: 0 or 1 (query i sees keys j <= i)
 *   stream: cudaStream_t or NULL
 * Rounding: a row's running max is refreshed (and O rescaled) only when it
 * grows by more than 8 in log2 units, so softmax weights reach 2^8 before
 * normalisation and the row's largest weight enters the P v product as a
 * bf16-rounded 2^delta rather than exactly 1 (relative error <= 2^-9, the
 * same as any other weight); lse is formed from unrounded weights.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
           int d, int causal, float scale, void* stream);

/*
 * Forward pass that also writes the bf16 rounding residual of o:
 * o_resid = bf16(O - o), where O is the fp32 result before rounding and o is
 * its bf16 rounding. o + o_resid carries O to ~16 significant bits. This
 * forward refreshes a row's running max whenever it grows, so the largest
 * weight of every row enters P v as exactly 1; its o may differ from
 * fa_fwd's in the last bit.
 * fa_bwd_with_residual uses it to form D_i = sum_c dO_ic O_ic: D multiplies
 * every error of O by dO and sums it over d, so the bf16 rounding of o alone
 * shifts dQ and dK by ~1e-2 on peaky rows. Arguments as fa_fwd, plus
 *   o_resid [B][Hq][N][d] (bf16, written; must not be NULL)
 */
int fa_fwd_with_residual(const void* q, const void* k, const void* v, void* o, void* o_resid, float* lse,
                         int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for this shape: an fp32 row sum
 * D_i = sum_c dout_ic o_ic per query row, and an fp32 dQ accumulator
 * [B][Hq][N][d]. Returns 0 for an invalid or unsupported shape.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d);

/*
 * Backward pass: gradients of sum(dout * O) with respect to q, k and v,
 * rebuilding P from q, k and lse tile by tile. Source: "FlashAttention:
 * IO-aware exact attention", "Four ideas" list, item "Recomputation in the
 * backward pass" (only the per-row logsumexp is kept from the forward pass
 * and P is rebuilt on chip); the gradient formulas are those of the
 * definition above: dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij,
 * dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q, with the query
 * heads of a KV group summed into its dK, dV.
 *   q, k, v, o, dout, lse: as produced for / by fa_fwd (read only). D_i is
 *   formed from the bf16 o; see fa_bwd_with_residual for the variant that
 *   removes o's rounding from D. Measured on B200 against the float64
 *   definition at B = 2, H = 16, N = 8192, d = 128, causal, q and k scaled
 *   by 2 (peaky rows; sampled rows of every head): this pair (fa_fwd then
 *   fa_bwd) reaches max |error| 0.064 in dQ and 0.046 in dK, against 0.030
 *   and 0.030 for the residual pair; the excess is o's rounding carried
 *   through D, and stays inside the bound 2e-2 + 2^-8 |exact| plus that
 *   term (2^-8 sum_c |dout_ic| (sum_j P_ij |v_jc| + |O_ic|) per row, times
 *   scale P |k| for dQ and scale (P D-error)^T |q| for dK).
 *   dq [B][Hq][N][d], dk, dv [B][Hkv][N][d] (bf16, written)
 *   workspace: device memory of at least fa_bwd_workspace_bytes(...) bytes,
 *   16-byte aligned, owned by the caller, contents need not be initialised
 *   and are clobbered. FA_ERR_INVALID_ARGUMENT if it is NULL or too small.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass as fa_bwd, with D_i formed from o + o_resid (o_resid as
 * written by fa_fwd_with_residual, read only, must not be NULL). This is the
 * path whose gradients stay within 2e-2 (plus bf16 output rounding) of the
 * exact gradients on peaky softmax rows.
 */
int fa_bwd_with_residual(const void* q, const void* k, const void* v, const void* o, const void* o_resid,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv,
                         int N, int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * Size of the device array that fa_bwd_noalloc uses as its workspace.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * Backward pass as fa_bwd, without a workspace argument and without
 * allocating anything. The source pages have no counterpart to this entry
 * point; it exists for callers that cannot allocate device memory: hosts
 * that hand a library only its input and output buffers (a fixed plugin
 * signature with no workspace argument), or runtimes that budget all device
 * memory themselves and forbid cudaMalloc, which also synchronises the
 * device.
 *   Arguments: as fa_bwd, minus workspace and workspace_bytes.
 *   Scratch: a file-scope device array of FA_BWD_NOALLOC_SCRATCH_BYTES
 *   (32 MiB) inside libfa, held by every GPU that loads it until the
 *   process exits. The shape must satisfy
 *   fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) <= FA_BWD_NOALLOC_SCRATCH_BYTES
 *   (about 4 bytes * B*Hq*N*(d+1)); larger shapes return FA_ERR_UNSUPPORTED
 *   before anything is launched.
 *   The first call on a device looks up the array's device address (once
 *   per device, with that device current). No call allocates or frees
 *   memory.
 *   Every call shares the array and it keeps the last call's contents; the
 *   kernels rewrite what they read before using it. Calls whose kernels
 *   overlap on the GPU (from several streams or host threads) race on the
 *   array and give wrong results: serialise them.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                   void* stream);

/*
 * Masked forward and backward: causal attention restricted by a sliding
 * window and/or opened by a prefix. Key j is visible to query i iff
 *     (j <= i and i - j <= window) or j < prefix,
 * so every query sees at least its own key. window = -1 means no window
 * (plain causal); window = 0 lets each query see only itself. prefix = 0
 * means no prefix; prefix >= N gives full (bidirectional) attention. This is
 * the sliding-window / prefix-LM family that "FlashAttention: IO-aware exact
 * attention" ("The honest limits") lists as needing its own kernels; here it
 * is one kernel variant that visits only the key tiles a query tile can see
 * (the prefix tiles and the window tiles, skipping any gap between them).
 * Arguments as fa_fwd_with_residual / fa_bwd_with_residual, with the causal
 * flag replaced by (window, prefix); o_resid may be NULL in both (the
 * backward then forms D from o alone). Without o_resid the forward rounds
 * as fa_fwd does (deferred O rescale), with it as fa_fwd_with_residual
 * (exact running max). FA_ERR_INVALID_ARGUMENT when window < -1 or
 * prefix < 0.
 */
int fa_fwd_masked(const void* q, const void* k, const void* v, void* o, void* o_resid, float* lse, int B, int Hq,
                  int Hkv, int N, int d, int window, int prefix, float scale, void* stream);
int fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* o_resid, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, int window,
                  int prefix, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * FP8 mode (e4m3 with block scaling).
 *
 * "FlashAttention: IO-aware exact attention" ("The generations") lists FP8
 * support with block scaling for FlashAttention-3, and ("The honest limits")
 * notes that FP8 changes rounding. Here: e4m3 codes (1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, largest finite 448) with one
 * fp32 scale per block; a value is code * scale.
 *
 * fa_quantize_fp8 quantizes a bf16 tensor x [BH][N][d] (d = 64 or 128) into
 * codes (uint8, same layout) and scales:
 *   per_head = 0: one scale per 128-row block, scales [BH][ceil(N/128)];
 *   per_head = 1: one scale per head,          scales [BH].
 * scale = amax / 448 (amax = largest |x| of the block; 1 for an all-zero
 * block), codes = e4m3(x * (448 / amax)) rounded to nearest even and
 * saturated, both fp32 operations correctly rounded. Q and K use 128-row
 * blocks, V one scale per head. Three small kernels on `stream`.
 *
 * fa_fwd_fp8 is the forward of fa_fwd on the dequantized tensors
 * (q_hat = q8 * sq of its 128-row block, k_hat likewise, v_hat = v8 * sv
 * of its head), for d = 128: q8 [B][Hq][N][128], k8 and v8 [B][Hkv][N][128]
 * e4m3 codes (16-byte aligned); sq [B*Hq][ceil(N/128)], sk [B*Hkv][ceil(N/128)],
 * sv [B*Hkv] fp32 (4-byte aligned); o bf16 [B][Hq][N][128], lse fp32
 * [B][Hq][N]. Both products run on e4m3 operands with fp32 accumulation;
 * the softmax weights enter the second one as e4m3 of 2^(x + 4), x the
 * exponent against a running row max that may lag the true one by up to 4
 * (the rescale of O is skipped for smaller growth), the main rounding
 * beyond the inputs' own.
 *
 * Returns FA_OK; FA_ERR_INVALID_ARGUMENT (null or misaligned pointer,
 * non-positive size, bad causal or per_head flag, non-finite or
 * non-positive scale); FA_ERR_UNSUPPORTED (d other than 128 for the
 * forward, 64/128 for quantization; Hq not a multiple of Hkv; size limits;
 * device not compute capability 10.0); FA_ERR_CUDA on a launch failure.
 */
int fa_quantize_fp8(const void* x, void* codes, float* scales, int BH, int N, int d, int per_head, void* stream);
int fa_fwd_fp8(const void* q8, const float* sq, const void* k8, const float* sk, const void* v8, const float* sv,
               void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * Decode / short-query attention against a KV cache.
 *
 * Nq new queries per head attend to an Nk-key cache, 1 <= Nq <= Nk. The
 * queries are the last Nq positions of the sequence: query i sits at
 * position Nk - Nq + i and, when causal = 1, sees keys j <= Nk - Nq + i
 * (bottom-right alignment; with Nq = 1 every key is visible either way).
 * Computes the same O and L as fa_fwd for those rows ("FlashAttention:
 * IO-aware exact attention", "PREFILL PATH" diagram: the decode loop, one
 * token at a time, reading the KV cache).
 *
 * Layout (bf16 row-major, d contiguous, all device memory owned by the
 * caller):
 *   q, o   [B][Hq][Nq][d]      query head h uses KV head h / (Hq/Hkv)
 *   k, v   [B][Hkv][Nk][d]     the cache
 *   lse    [B][Hq][Nq] fp32    natural-log row logsumexp
 * workspace: device memory of at least fa_decode_workspace_bytes(...) bytes,
 * 16-byte aligned, for the per-split partial results (fp32); its contents
 * on entry do not matter and are overwritten.
 *
 * The cache is split across all SMs (each takes an equal share of the
 * (batch, KV head) key tiles); partial results are merged by logsumexp in a
 * second kernel on the same stream (launched as a programmatic dependent of
 * the first, so it is resident before the first ends). Asynchronous on
 * `stream`. Returns
 * FA_OK; FA_ERR_INVALID_ARGUMENT for a null or misaligned pointer, a
 * non-positive size, Nq > Nk, a bad causal flag, a non-finite or
 * non-positive scale, or a workspace smaller than required;
 * FA_ERR_UNSUPPORTED for d not 64/128, Hq not a multiple of Hkv, a size
 * past the index limits, or a device that is not compute capability 10.0;
 * FA_ERR_CUDA on a launch failure. Nothing is written on an argument error.
 */
size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d);
int fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
              int Nk, int d, int causal, float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Static text for a status code (for FA_ERR_CUDA: the last CUDA error seen by
 * this thread). Never NULL. */
const char* fa_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word. Returns FA_OK, FA_ERR_TIMEOUT when a kernel's bounded wait ran out
 * since the last check, or FA_ERR_CUDA when the synchronisation failed.
 */
int fa_check_device_error(void* stream);

/*
 * Sets the per-wait watchdog budget in nanoseconds for later launches from
 * any thread (default 2e9). Values below 1e6 are raised to 1e6.
 */
void fa_set_watchdog_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

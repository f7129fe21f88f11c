/*
 * forge_attn.h -- C ABI of the B200 (sm_100a) fused causal attention library.
 *
 * The operation is the attention of one decoder-only transformer layer, forward
 * and backward, as the Forge paper ("Building an LLM Training Framework from
 * Scratch in C++ and Metal on Apple Silicon") defines its fused attention:
 *
 *   forward  (section "Attention kernel design"):
 *     S = scale * Q K^T,  S[i][j] = -inf where causal and j > i,
 *     P = softmax(S) row-wise,  O = P V,  LSE[i] = ln sum_j exp(S[i][j])
 *     (the per-row log-sum-exp the backward reuses instead of renormalising);
 *   backward (section "Ecosystem survey", the fused-backward paragraph, and
 *     "Attention kernel design" for the transposed scores S^T = K Q^T,
 *     dP^T = V dO^T):
 *     D = rowsum(dO o O),  P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,
 *     dS = P o (dP - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 * Conventions shared by every entry point
 *   Memory      All tensor pointers are DEVICE pointers owned by the caller; the
 *               library never allocates or frees device memory.
 *   Layout      q, k, v, o, dO, dq, dk, dv are contiguous row-major [B][H][T][d]
 *               (d fastest).  lse and the backward's D are fp32 [B][H][T].
 *               Elements are bf16 bit patterns unless an option bit says fp32
 *               (FORGE_ATTN_OUT_F32, FORGE_ATTN_O_IN_F32) or fp16
 *               (FORGE_ATTN_FP16).
 *   Alignment   Every tensor base must be 16-byte aligned (a TMA requirement);
 *               the workspace must be 256-byte aligned.
 *   Aliasing    Outputs must not overlap inputs or each other.
 *   Streams     `stream` is a cudaStream_t (NULL = the legacy default stream).
 *               Calls are asynchronous and ordered on that stream; nothing
 *               synchronises with the host.
 *   Sizes       B, H, T >= 1; d in {64, 128}; B*H*T*d < 2^31 per tensor;
 *               scale finite; causal in {0, 1} (0 = full attention).
 *               T need not be a multiple of the 128-row tile: rows and keys past
 *               T are masked, never read from the next head, never written.
 *   Errors      Each call returns FORGE_ATTN_OK or a forge_attn_status code and
 *               never throws.  Argument errors are reported before any launch,
 *               in which case nothing is written.  FORGE_ATTN_ERR_CUDA reports a
 *               launch failure (cudaGetLastError).  Device-side waits are
 *               bounded: a wait that runs out is reported by
 *               forge_attn_check_device_error().
 *   Determinism The forward is deterministic.  The backward accumulates dQ with
 *               unordered fp32 reductions, so dQ may differ in the last bits run to
 *               run; dK and dV are deterministic.
 */
#ifndef FORGE_ATTN_H
#define FORGE_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FORGE_ATTN_OK = 0,
    FORGE_ATTN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad flag      */
    FORGE_ATTN_ERR_UNSUPPORTED = 2, /* head dim other than 64/128, sizes too large     */
    FORGE_ATTN_ERR_MISALIGNED = 3,  /* tensor base not 16-byte (workspace 256) aligned */
    FORGE_ATTN_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed               */
    FORGE_ATTN_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out              */
    FORGE_ATTN_ERR_WORKSPACE = 6    /* workspace missing or smaller than required      */
} forge_attn_status;

/*
 * Option bits for the _ex entry points (0 = the plain entry points' behaviour).
 *
 * FORGE_ATTN_OUT_F32   outputs in fp32 instead of bf16: o for the forward; dq, dk
 *                      and dv for the backward.  Needed where output magnitudes
 *                      reach 8 and more, since bf16 rounding alone is then up to
 *                      0.03 per element.
 * FORGE_ATTN_O_IN_F32  backward only: `o` holds fp32 values (as the forward writes
 *                      them with FORGE_ATTN_OUT_F32); D = rowsum(dO o O) then sees
 *                      O unrounded.
 * FORGE_ATTN_PRECISE   every probability or score gradient that enters a
 *                      tensor-core product as bf16 (P in P V and P^T dO, dS in
 *                      dS K and dS^T Q) is split into two bf16 terms hi + lo
 *                      with hi = bf16(x), lo = bf16(x - hi), and both products are
 *                      accumulated.  Costs one extra product per split operand;
 *                      lowers the operand rounding error from ~2^-9 to ~2^-17
 *                      relative.
 * FORGE_ATTN_FP16      fp16 instead of bf16 for every 16-bit tensor: the inputs q,
 *                      k, v, dO and the 16-bit outputs (o, dq, dk, dv, unless
 *                      FORGE_ATTN_OUT_F32 makes them fp32).  P and dS then enter
 *                      the tensor-core products as fp16 (relative rounding 2^-11
 *                      instead of bf16's 2^-8), with fp32 accumulation as before.
 *                      fp16's range ends at 65504: inputs, outputs and scores
 *                      gradients must stay within it.  Not combinable with
 *                      FORGE_ATTN_PRECISE (FORGE_ATTN_ERR_UNSUPPORTED).
 *                      (The paper's operand-type comparison, section "Finding 4",
 *                      measures half and bfloat operands side by side.)
 */
#define FORGE_ATTN_OUT_F32 1
#define FORGE_ATTN_O_IN_F32 2
#define FORGE_ATTN_PRECISE 4
#define FORGE_ATTN_FP16 8

/*
 * Forward.  Reads q, k, v (bf16 [B][H][T][d]); writes o (bf16 [B][H][T][d]) and
 * lse (fp32 [B][H][T], natural log over the scaled, masked scores).
 * One kernel launch.
 */
int forge_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int T, int d, float scale, int causal, void* stream);

/* Forward with option bits (FORGE_ATTN_OUT_F32, FORGE_ATTN_PRECISE, FORGE_ATTN_FP16). */
int forge_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int T, int d, float scale, int causal, int flags, void* stream);

/*
 * Bytes of device workspace forge_attn_bwd needs: the row statistics (fp32
 * [2][B*H][t_pad], t_pad = 128 * ceil(T / 128): -LSE * log2(e), then D) and the fp32
 * dQ accumulator ([B][H][T][d]), each at a 256-byte aligned offset.  Returns 0 for
 * arguments forge_attn_bwd would reject.
 */
size_t forge_attn_bwd_workspace_size(int B, int H, int T, int d);

/*
 * Backward.  Reads q, k, v, o, dO (bf16 [B][H][T][d]) and lse (fp32 [B][H][T],
 * as written by the forward with the same arguments); writes dq, dk, dv (bf16
 * [B][H][T][d]).  workspace: device memory of at least
 * forge_attn_bwd_workspace_size() bytes, 256-byte aligned; its contents on entry
 * do not matter and on return are unspecified.
 * `o` is bf16 here (fp32 with forge_attn_bwd_ex and FORGE_ATTN_O_IN_F32).
 * Launch sequence on `stream`: the pre-pass (row statistics; also zeroes the dQ
 * accumulator), the dK/dV kernel over key tiles (dQ partials added into the fp32
 * accumulator by TMA reduce-add), and the dQ conversion.
 */
int forge_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int H, int T, int d, float scale, int causal,
                   void* stream);

/* Backward with option bits (FORGE_ATTN_OUT_F32, FORGE_ATTN_O_IN_F32,
 * FORGE_ATTN_PRECISE, FORGE_ATTN_FP16).  With FORGE_ATTN_OUT_F32 the dQ accumulator
 * is dq itself and the conversion launch is skipped. */
int forge_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                      const void* dO, const float* lse, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, int B, int H, int T, int d,
                      float scale, int causal, int flags, void* stream);

/*
 * The three backward stages as separate calls, for callers that schedule or time
 * them one by one.  forge_attn_bwd_ex is exactly these three in order.
 *
 * forge_attn_bwd_preprocess: the row statistics rowstats (fp32 [2][B*H][t_pad],
 *   t_pad = 128 * ceil(T / 128), 16-byte aligned): rowstats[0][bh][t] = -lse * log2(e)
 *   and rowstats[1][bh][t] = D = sum_k dO[t][k] * o[t][k], with -inf and 0 in the
 *   padding rows t >= T; and dq_accum (fp32 [B][H][T][d]) set to zero unless it is
 *   NULL.  flags: FORGE_ATTN_O_IN_F32 (o is fp32), FORGE_ATTN_FP16 (dO, and o
 *   unless fp32, are fp16).
 * forge_attn_bwd_dkdv: recomputes P per key tile from the row statistics, writes dk
 *   and dv, and adds scale * dS K into dq_accum (TMA reduce-add).  flags:
 *   FORGE_ATTN_OUT_F32 (dk, dv fp32), FORGE_ATTN_PRECISE, FORGE_ATTN_FP16.
 * forge_attn_bwd_dq_convert: dq = bf16(dq_accum).  Only needed for 16-bit dq;
 *   forge_attn_bwd_dq_convert_ex with FORGE_ATTN_FP16 writes fp16.
 */
int forge_attn_bwd_preprocess(const void* o, const void* dO, const float* lse, float* rowstats,
                              float* dq_accum, int B, int H, int T, int d, int flags,
                              void* stream);
int forge_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO,
                        const float* rowstats, float* dq_accum, void* dk, void* dv, int B, int H,
                        int T, int d, float scale, int causal, int flags, void* stream);
int forge_attn_bwd_dq_convert(const float* dq_accum, void* dq, int B, int H, int T, int d,
                              void* stream);
int forge_attn_bwd_dq_convert_ex(const float* dq_accum, void* dq, int B, int H, int T, int d,
                                 int flags, void* stream);

/*
 * Bytes of the fixed device array that forge_attn_bwd_noalloc uses in place of a
 * workspace: 64 MiB, enough whenever forge_attn_bwd_workspace_size() <= 64 MiB,
 * i.e. B*H*(T*d + 2*t_pad) floats up to about 16.7 million (for example B=4 H=16
 * T=2048 d=64, or B=1 H=16 T=4096 d=64).
 */
#define FORGE_ATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * forge_attn_bwd for callers that cannot allocate device memory (a process whose
 * memory budget is fixed at start-up, a plugin that is handed raw device pointers
 * but no allocator, a latency-critical loop that must not call the allocator).
 * The paper has no counterpart; this is a property of this library, not of the
 * method.  Same arguments, results and launch sequence as forge_attn_bwd, minus the
 * workspace: the row statistics and the fp32 dQ accumulator live in a file-scope
 * __device__ array of
 * FORGE_ATTN_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds
 * until the process exits.  No cudaMalloc, cudaFree or allocating library call is
 * made.
 *   - Sizes whose forge_attn_bwd_workspace_size() exceeds the array are refused
 *     with FORGE_ATTN_ERR_WORKSPACE before any launch.
 *   - The first call in a CUDA context (once per device, and again in the new
 *     primary context after cudaDeviceReset) looks up the array's device address
 *     with that context current; make that first call before any stream capture
 *     begins.
 *   - All calls on a device share the array, which keeps the last call's contents;
 *     each call rewrites the row statistics and clears the accumulator first.  Calls whose kernels
 *     can overlap on the GPU (unordered streams) race on the array and must not be
 *     issued.
 */
int forge_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dO, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int T, int d, float scale, int causal, void* stream);

/*
 * bf16 -> fp16 conversion of n values, for running bf16 tensors through the
 * FORGE_ATTN_FP16 path (whose P and dS then enter the tensor-core products with fp16's
 * 11 significant bits instead of bf16's 8, so fp32 outputs and D from the fp32 O meet
 * the tolerances at T = 8000 without FORGE_ATTN_PRECISE's split products).  src, dst:
 * device pointers, caller-owned, 16-byte aligned, not overlapping.  Each value is
 * rounded to nearest even once: magnitudes in [2^-14, 65504] (and zeros) convert
 * exactly, smaller ones land on fp16's subnormal grid (absolute error at most 2^-25),
 * NaN stays NaN, and larger ones (infinities included) become +-inf; when `overflow`
 * is not NULL the number of those is added atomically to the device counter
 * *overflow (4-byte aligned), for the caller to read after the stream's work.
 * n = 0 does nothing.  One kernel launch on `stream`.
 */
int forge_attn_bf16_to_fp16(const void* src, void* dst, long long n, unsigned int* overflow,
                            void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* forge_attn_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the device error word that
 * bounded waits set.  Returns FORGE_ATTN_OK, FORGE_ATTN_ERR_TIMEOUT (a wait ran
 * out; *detail, if not NULL, receives the raw word: bit 31 set, bits 20..30 the
 * wait site, bits 0..19 the block index), or FORGE_ATTN_ERR_CUDA.
 */
int forge_attn_check_device_error(void* stream, unsigned int* detail);

/* Library version as major*10000 + minor*100 + patch. */
int forge_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FORGE_ATTN_H */

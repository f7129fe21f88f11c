/*
 * forge_attn_testing.h -- test-support entry points of the same library.
 *
 * These exist so the tests can check the tensor-core building blocks the
 * attention kernels are made of, and the bounded-wait error path, through the C
 * ABI.  They are not part of the attention operation; the paper has no
 * counterpart for them.  Conventions (device pointers, stream, status codes) are
 * those of forge_attn.h.
 */
#ifndef FORGE_ATTN_TESTING_H
#define FORGE_ATTN_TESTING_H

#ifdef __cplusplus
extern "C" {
#endif

/* Operand forms of one 128 x N x K tile product on the tensor cores. */
typedef enum {
    FORGE_PROBE_SS_KK = 0, /* D = A B^T; A [128][K], B [N][K]; both staged by TMA, K-major */
    FORGE_PROBE_SS_KMN = 1,/* D = A B;   A [128][K] K-major, B [K][N] MN-major             */
    FORGE_PROBE_TS_KMN = 2,/* as 1, but A is written to tensor memory by threads first     */
    FORGE_PROBE_SS_MNMN = 3/* D = A^T B; A [K][128] MN-major, B [K][N] MN-major            */
} forge_probe_mode;

/*
 * One CTA computes a single 128 x N fp32 tile D from bf16 operands with
 * tcgen05.mma (TMA -> shared memory -> tensor core -> tensor memory -> registers)
 * and writes it row-major to d_out (fp32 [128][N]).  K in {64, 128}; N in
 * {64, 128}.  Operand layouts are given by `mode`.
 */
int forge_probe_mma(const void* a, const void* b, float* d_out, int N, int K, int mode,
                    void* stream);

/*
 * Launches one CTA that waits on an mbarrier nothing will complete, with a wait
 * limit of `limit_ns` nanoseconds.  The kernel must give up, record the timeout
 * in the device error word and exit; forge_attn_check_device_error() then
 * returns FORGE_ATTN_ERR_TIMEOUT.  limit_ns is clamped to [1e3, 1e9].
 */
int forge_probe_wait_timeout(unsigned long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FORGE_ATTN_TESTING_H */

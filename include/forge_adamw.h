/*
 * forge_adamw.h -- C ABI of the fused multi-tensor AdamW step (same library as
 * forge_attn.h, libforge_attn.so).
 *
 * The Forge paper ("Building an LLM Training Framework from Scratch in C++ and
 * Metal on Apple Silicon") trains with AdamW using decoupled weight decay on the
 * parameters of rank two or more only, epsilon outside the square root, and
 * gradient clipping at a global norm whose factor is folded into the optimizer's
 * read of the gradient (sections "Training details" and "Related work"); it issues
 * the per-tensor optimizer dispatches and gradient-norm reductions concurrently
 * (section "Finding 5").  One call here performs that whole step for a list of
 * tensors:
 *
 *   norm = sqrt(sum over every tensor and element of grad^2)
 *   c    = max_norm / norm if max_norm > 0 and norm > max_norm, else 1
 *   per element, with g = c * grad:
 *     m = beta1 * m + (1 - beta1) * g
 *     v = beta2 * v + (1 - beta2) * g^2
 *     p = p - lr * ( (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 *                    + wd * p )          (p on the right: the value before the step)
 *   wd = weight_decay for tensors with decay != 0 (rank >= 2), 0 for the others.
 *
 * Conventions: every pointer in forge_adamw_tensor is a caller-owned DEVICE pointer
 * to n fp32 values, 16-byte aligned; param, exp_avg (m) and exp_avg_sq (v) are
 * updated in place; tensors must not overlap.  The call is asynchronous on `stream`
 * (a cudaStream_t, NULL = legacy default) and returns FORGE_ATTN_OK or a
 * forge_attn_status code (forge_attn.h); argument errors are reported before any
 * launch.  The global norm is reduced in a fixed order, so the step is
 * deterministic.
 */
#ifndef FORGE_ADAMW_H
#define FORGE_ADAMW_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Tensors per kernel launch (the table travels in the kernel parameters); longer
 * lists take several launches per pass. */
#define FORGE_ADAMW_MAX_TENSORS_PER_LAUNCH 256

typedef struct {
    float* param;            /* parameters, updated in place           */
    const float* grad;       /* gradients (read only)                  */
    float* exp_avg;          /* first moment m, updated in place       */
    float* exp_avg_sq;       /* second moment v, updated in place      */
    long long n;             /* elements, >= 1                         */
    int decay;               /* 1: decoupled weight decay (rank >= 2)  */
} forge_adamw_tensor;

/* Bytes of device workspace forge_adamw_step needs for n_tensors tensors (0 if
 * n_tensors < 1).  Its contents on entry do not matter. */
size_t forge_adamw_workspace_size(int n_tensors);

/*
 * One AdamW step.  tensors: a HOST array of n_tensors descriptors (read during the
 * call only).  step >= 1 is the 1-based step number of the bias corrections.
 * beta1, beta2 in [0, 1); eps >= 0; max_norm <= 0 disables clipping.
 * grad_norm_out: optional DEVICE float receiving the global gradient norm (before
 * clipping), or NULL.  workspace: device memory of forge_adamw_workspace_size()
 * bytes, 16-byte aligned.  Launches: a norm pass and an update pass per group of
 * FORGE_ADAMW_MAX_TENSORS_PER_LAUNCH tensors, after a 4-byte memset.
 */
int forge_adamw_step(const forge_adamw_tensor* tensors, int n_tensors, float lr, float beta1,
                     float beta2, float eps, float weight_decay, int step, float max_norm,
                     float* grad_norm_out, void* workspace, size_t workspace_bytes,
                     void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FORGE_ADAMW_H */

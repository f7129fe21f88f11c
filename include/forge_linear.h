/*
 * forge_linear.h -- C ABI of the projection GEMMs around attention (same library as
 * forge_attn.h, libforge_attn.so): the three products of a linear layer without
 * bias in training, on tcgen05 tensor cores.
 *
 * The Forge paper ("Building an LLM Training Framework from Scratch in C++ and
 * Metal on Apple Silicon") measures them in section "Results" (the GEMM table: the
 * forward X W^T, the backward dX = dY W and dW = dY^T X) and section "Finding 4.2"
 * (the transposed variants training needs); it notes that dW lags for want of
 * split-K, which forge_linear_bwd_dw does.  With tokens t, input features i and
 * output features o:
 *
 *   forge_linear_fwd      y[t][o]  = sum_i x[t][i] w[o][i]          (Y = X W^T)
 *   forge_linear_bwd_dx   dx[t][i] = sum_o dy[t][o] w[o][i]         (dX = dY W)
 *   forge_linear_bwd_dw   dw[o][i] (+)= sum_t dy[t][o] x[t][i]      (dW = dY^T X)
 *
 * Conventions: all tensors are caller-owned DEVICE memory, contiguous row-major with
 * the shapes above, 16-byte aligned; 16-bit tensors are bf16 (fp16 with
 * FORGE_ATTN_FP16 in flags; both operands of a product share one type).  tokens,
 * in_features and out_features are multiples of 8 (TMA row strides are multiples of
 * 16 bytes), each product of two of them below 2^31.  Products accumulate in fp32.
 * Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default) and
 * return FORGE_ATTN_OK or a forge_attn_status code (forge_attn.h); argument errors
 * are reported before any launch.  Outputs must not overlap inputs.
 */
#ifndef FORGE_LINEAR_H
#define FORGE_LINEAR_H

#ifdef __cplusplus
extern "C" {
#endif

/* Y = X W^T.  x: [tokens][in_features], w: [out_features][in_features], y:
 * [tokens][out_features], 16-bit, or fp32 with FORGE_ATTN_OUT_F32.  flags:
 * FORGE_ATTN_OUT_F32, FORGE_ATTN_FP16.  One launch; deterministic. */
int forge_linear_fwd(const void* x, const void* w, void* y, int tokens, int in_features,
                     int out_features, int flags, void* stream);

/* dX = dY W.  dy: [tokens][out_features], w: [out_features][in_features], dx:
 * [tokens][in_features], 16-bit, or fp32 with FORGE_ATTN_OUT_F32.  flags as for the
 * forward.  One launch; deterministic. */
int forge_linear_bwd_dx(const void* dy, const void* w, void* dx, int tokens, int in_features,
                        int out_features, int flags, void* stream);

/* dW = dY^T X into fp32 dw [out_features][in_features]; accumulate = 1 adds to dw's
 * contents (gradient accumulation), 0 overwrites it.  The reduction over tokens is
 * split into split_k parts (0 = forge_linear_split_k's choice) whose partial
 * products are added into dw with fp32 reductions; with more than one part, or when
 * accumulating, dw's last bits depend on the order of those additions (not
 * deterministic), and when not accumulating dw is zeroed first (a memset).  flags:
 * FORGE_ATTN_FP16. */
int forge_linear_bwd_dw(const void* dy, const void* x, float* dw, int tokens, int in_features,
                        int out_features, int split_k, int accumulate, int flags, void* stream);

/* The split of forge_linear_bwd_dw's token reduction chosen for split_k = 0: with the
 * tile shape, the plan a cost model rates cheapest (the k-blocks of the most loaded SM,
 * weighted by the tile's shared-memory traffic, plus the fp32 reductions of every
 * part's partial dW), each part at least 512 tokens deep.  0 for arguments
 * forge_linear_bwd_dw would reject. */
int forge_linear_split_k(int tokens, int in_features, int out_features);

#ifdef __cplusplus
}
#endif

#endif /* FORGE_LINEAR_H */

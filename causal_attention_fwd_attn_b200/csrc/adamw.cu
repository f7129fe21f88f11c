// adamw.cu -- one AdamW step over many parameter tensors in a few launches.
//
// The Forge paper ("Building an LLM Training Framework from Scratch in C++ and Metal
// on Apple Silicon") issues its optimizer as one dispatch per parameter tensor plus
// one gradient-norm reduction per tensor, all independent of each other, and puts
// them in a concurrent dispatch region (section "Finding 5").  Its training recipe
// (section "Training details" and "Related work"): AdamW with decoupled weight decay
// applied only to parameters of rank two or more, epsilon added outside the square
// root, and gradient clipping at a global norm whose factor is folded into the
// optimizer's read of the gradient.
//
// On B200 the many small dispatches become a multi-tensor launch: the tensor table
// travels in the kernel parameters, every tensor is cut into fixed chunks, and the
// CTAs of one persistent grid walk all chunks of all tensors.  Two passes:
//   norm      sum of squared gradients, one partial per CTA; the last CTA to finish
//             adds the partials in a fixed order (deterministic), and writes the
//             global norm and the clip factor c = max_norm / norm if norm > max_norm,
//             else 1 (no clipping when max_norm <= 0).
//   update    per element, with g = c * grad:
//               m = beta1 m + (1 - beta1) g,   v = beta2 v + (1 - beta2) g^2
//               p = p - lr * ( (m / bc1) / (sqrt(v / bc2) + eps) + wd * p )
//             bc1 = 1 - beta1^step, bc2 = 1 - beta2^step, wd = weight_decay for tensors
//             flagged for decay, else 0; p on the right is the value before the step.
// Both passes are bound by HBM bandwidth: 4 bytes per element for the norm, 28 for
// the update (read p, g, m, v; write p, m, v), all fp32.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "forge_adamw.h"
#include "forge_attn.h"
#include "forge_internal.h"

namespace forge {
namespace {

constexpr int kAdamThreads = 512;
// elements per chunk: a multiple of 4 * kAdamThreads, so every chunk but a tensor's
// last is whole float4 loads for every thread
constexpr long long kChunk = 1 << 16;
constexpr int kMaxPerLaunch = FORGE_ADAMW_MAX_TENSORS_PER_LAUNCH;

struct TensorTable {
    float* param[kMaxPerLaunch];
    const float* grad[kMaxPerLaunch];
    float* m[kMaxPerLaunch];
    float* v[kMaxPerLaunch];
    long long n[kMaxPerLaunch];
    int chunk0[kMaxPerLaunch + 1];  // first chunk of each tensor; chunk0[count] = total
    unsigned char decay[kMaxPerLaunch];
    int count;
};
static_assert(sizeof(TensorTable) < 30000, "kernel parameter space");

// Workspace layout (floats): [0] clip factor, [1] global norm, [2] completion counter
// (as unsigned), then the per-CTA partial sums.
constexpr int kWsScale = 0, kWsNorm = 1, kWsCounter = 2, kWsPartials = 4;

// The tensor and element range of chunk c.
__device__ __forceinline__ int tensor_of_chunk(const TensorTable& t, int c) {
    int lo = 0, hi = t.count - 1;
    while (lo < hi) {  // last tensor whose first chunk is <= c
        const int mid = (lo + hi + 1) >> 1;
        if (t.chunk0[mid] <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float block_sum(float x, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float s = 0.f;
    if (warp == 0) {
        s = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    }
    __syncthreads();
    return s;  // valid in thread 0
}

// Sum of squares of this launch's gradients into partials[part0 + blockIdx.x]; the
// CTA that completes the last of `total_parts` partials (over every norm launch of
// the step) adds them all in index order and writes the norm and the clip factor.
__global__ void __launch_bounds__(kAdamThreads) adamw_norm_kernel(
    const __grid_constant__ TensorTable t, float* __restrict__ ws, int part0, int total_parts,
    float max_norm, float* __restrict__ norm_out) {
    __shared__ float red[32];
    __shared__ bool last;
    float acc = 0.f;
    const int n_chunks = t.chunk0[t.count];
    for (int c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        const int i = tensor_of_chunk(t, c);
        const long long e0 = (long long)(c - t.chunk0[i]) * kChunk;
        const long long e1 = min(e0 + kChunk, t.n[i]);
        const float* g = t.grad[i];
        const long long n4 = (e1 - e0) >> 2;
        const float4* g4 = reinterpret_cast<const float4*>(g + e0);
        // four independent loads in flight per thread (the pass is bound by memory
        // latency otherwise), then the remainder
        const int bd = (int)blockDim.x;
        long long k = threadIdx.x;
        float a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (; k + 3 * bd < n4; k += 4 * bd) {
            const float4 x0 = g4[k], x1 = g4[k + bd], x2 = g4[k + 2 * bd], x3 = g4[k + 3 * bd];
            acc = fmaf(x0.x, x0.x, fmaf(x0.y, x0.y, fmaf(x0.z, x0.z, fmaf(x0.w, x0.w, acc))));
            a1 = fmaf(x1.x, x1.x, fmaf(x1.y, x1.y, fmaf(x1.z, x1.z, fmaf(x1.w, x1.w, a1))));
            a2 = fmaf(x2.x, x2.x, fmaf(x2.y, x2.y, fmaf(x2.z, x2.z, fmaf(x2.w, x2.w, a2))));
            a3 = fmaf(x3.x, x3.x, fmaf(x3.y, x3.y, fmaf(x3.z, x3.z, fmaf(x3.w, x3.w, a3))));
        }
        for (; k < n4; k += bd) {
            const float4 x = g4[k];
            acc = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, acc))));
        }
        acc += (a1 + a2) + a3;
        for (long long e = e0 + 4 * n4 + threadIdx.x; e < e1; e += blockDim.x)
            acc = fmaf(g[e], g[e], acc);
    }
    const float s = block_sum(acc, red);
    if (threadIdx.x == 0) {
        ws[kWsPartials + part0 + blockIdx.x] = s;
        __threadfence();
        unsigned int* counter = reinterpret_cast<unsigned int*>(ws + kWsCounter);
        last = atomicAdd(counter, 1u) == (unsigned int)total_parts - 1;
    }
    __syncthreads();
    if (!last) return;
    // the last CTA: every partial is written (each writer fenced before counting)
    __threadfence();
    if (threadIdx.x == 0) {
        float tot;
        double sum = 0.0;
        const volatile float* parts = ws + kWsPartials;
        for (int k = 0; k < total_parts; ++k) sum += (double)parts[k];
        tot = (float)sqrt(sum);
        ws[kWsNorm] = tot;
        if (norm_out) *norm_out = tot;
        ws[kWsScale] = (max_norm > 0.f && tot > max_norm) ? max_norm / tot : 1.f;
        *reinterpret_cast<unsigned int*>(ws + kWsCounter) = 0u;  // ready for the next step
    }
}

// The AdamW update of this launch's tensors, with the clip factor from ws.
__global__ void __launch_bounds__(kAdamThreads) adamw_update_kernel(
    const __grid_constant__ TensorTable t, const float* __restrict__ ws, float lr, float beta1,
    float beta2, float eps, float weight_decay, float inv_bc1, float inv_bc2) {
    const float c = ws[kWsScale];
    const float a1 = 1.f - beta1, a2 = 1.f - beta2;
    const int n_chunks = t.chunk0[t.count];
    auto one = [&](float& p, float g, float& m, float& v, float wd) {
        g *= c;
        m = fmaf(beta1, m, a1 * g);
        v = fmaf(beta2, v, a2 * g * g);
        const float mhat = m * inv_bc1;
        const float vhat = v * inv_bc2;
        p = p - lr * (mhat / (sqrtf(vhat) + eps) + wd * p);
    };
    for (int ch = blockIdx.x; ch < n_chunks; ch += gridDim.x) {
        const int i = tensor_of_chunk(t, ch);
        const long long e0 = (long long)(ch - t.chunk0[i]) * kChunk;
        const long long e1 = min(e0 + kChunk, t.n[i]);
        const float wd = t.decay[i] ? weight_decay : 0.f;
        float* P = t.param[i];
        const float* G = t.grad[i];
        float* M = t.m[i];
        float* V = t.v[i];
        const long long n4 = (e1 - e0) >> 2;
        float4* P4 = reinterpret_cast<float4*>(P + e0);
        const float4* G4 = reinterpret_cast<const float4*>(G + e0);
        float4* M4 = reinterpret_cast<float4*>(M + e0);
        float4* V4 = reinterpret_cast<float4*>(V + e0);
        for (long long k = threadIdx.x; k < n4; k += blockDim.x) {
            float4 p = P4[k], m = M4[k], v = V4[k];
            const float4 g = G4[k];
            one(p.x, g.x, m.x, v.x, wd);
            one(p.y, g.y, m.y, v.y, wd);
            one(p.z, g.z, m.z, v.z, wd);
            one(p.w, g.w, m.w, v.w, wd);
            P4[k] = p;
            M4[k] = m;
            V4[k] = v;
        }
        for (long long e = e0 + 4 * n4 + threadIdx.x; e < e1; e += blockDim.x)
            one(P[e], G[e], M[e], V[e], wd);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Fills `t` with tensors [first, first + count) of the caller's table.
int fill_table(TensorTable* t, const forge_adamw_tensor* tensors, int first, int count) {
    std::memset(t, 0, sizeof(*t));
    t->count = count;
    long long chunks = 0;
    for (int k = 0; k < count; ++k) {
        const forge_adamw_tensor& x = tensors[first + k];
        t->param[k] = x.param;
        t->grad[k] = x.grad;
        t->m[k] = x.exp_avg;
        t->v[k] = x.exp_avg_sq;
        t->n[k] = x.n;
        t->decay[k] = x.decay ? 1 : 0;
        t->chunk0[k] = (int)chunks;
        chunks += (x.n + kChunk - 1) / kChunk;
        if (chunks > 0x3fffffff) return FORGE_ATTN_ERR_UNSUPPORTED;
    }
    t->chunk0[count] = (int)chunks;
    return FORGE_ATTN_OK;
}

int grid_for(const TensorTable& t) {
    const int chunks = t.chunk0[t.count];
    const int cap = 2 * sm_count();  // two 512-thread CTAs per SM
    return chunks < cap ? (chunks > 0 ? chunks : 1) : cap;
}

}  // namespace
}  // namespace forge

using namespace forge;

extern "C" {

size_t forge_adamw_workspace_size(int n_tensors) {
    if (n_tensors < 1) return 0;
    const int launches = (n_tensors + kMaxPerLaunch - 1) / kMaxPerLaunch;
    // the grid of a launch is at most two CTAs per SM; 1024 SMs is far beyond any part
    return (size_t)(kWsPartials + launches * 2 * 1024) * sizeof(float);
}

int forge_adamw_step(const forge_adamw_tensor* tensors, int n_tensors, float lr, float beta1,
                     float beta2, float eps, float weight_decay, int step, float max_norm,
                     float* grad_norm_out, void* workspace, size_t workspace_bytes,
                     void* stream) {
    if (!tensors || n_tensors < 1 || step < 1) return FORGE_ATTN_ERR_INVALID_ARG;
    for (float x : {lr, beta1, beta2, eps, weight_decay, max_norm})
        if (!std::isfinite(x)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || eps < 0.f)
        return FORGE_ATTN_ERR_INVALID_ARG;
    for (int k = 0; k < n_tensors; ++k) {
        const forge_adamw_tensor& x = tensors[k];
        if (!x.param || !x.grad || !x.exp_avg || !x.exp_avg_sq || x.n < 1)
            return FORGE_ATTN_ERR_INVALID_ARG;
        if (!aligned16(x.param) || !aligned16(x.grad) || !aligned16(x.exp_avg) ||
            !aligned16(x.exp_avg_sq))
            return FORGE_ATTN_ERR_MISALIGNED;
    }
    if (!workspace || workspace_bytes < forge_adamw_workspace_size(n_tensors))
        return FORGE_ATTN_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return FORGE_ATTN_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(grad_norm_out) & 3u) return FORGE_ATTN_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* ws = static_cast<float*>(workspace);
    const int launches = (n_tensors + kMaxPerLaunch - 1) / kMaxPerLaunch;
    // host-side table per launch (kernel parameters), validated before any launch
    static thread_local TensorTable tables[4];
    TensorTable* tab = launches <= 4 ? tables : new TensorTable[launches];
    int rc = FORGE_ATTN_OK;
    for (int l = 0; l < launches && rc == FORGE_ATTN_OK; ++l) {
        const int first = l * kMaxPerLaunch;
        const int count = n_tensors - first < kMaxPerLaunch ? n_tensors - first : kMaxPerLaunch;
        rc = fill_table(&tab[l], tensors, first, count);
    }
    if (rc == FORGE_ATTN_OK) {
        int parts = 0;
        for (int l = 0; l < launches; ++l) parts += grid_for(tab[l]);
        // the counter starts at zero: cleared here once, then by every norm pass's last CTA
        cudaError_t e = cudaMemsetAsync(ws + kWsCounter, 0, sizeof(float), s);
        int part0 = 0;
        for (int l = 0; l < launches && e == cudaSuccess; ++l) {
            const int grid = grid_for(tab[l]);
            adamw_norm_kernel<<<grid, kAdamThreads, 0, s>>>(tab[l], ws, part0, parts, max_norm,
                                                             grad_norm_out);
            part0 += grid;
            e = cudaGetLastError();
        }
        const double bc1 = 1.0 - std::pow((double)beta1, (double)step);
        const double bc2 = 1.0 - std::pow((double)beta2, (double)step);
        for (int l = 0; l < launches && e == cudaSuccess; ++l) {
            adamw_update_kernel<<<grid_for(tab[l]), kAdamThreads, 0, s>>>(
                tab[l], ws, lr, beta1, beta2, eps, weight_decay, (float)(1.0 / bc1),
                (float)(1.0 / bc2));
            e = cudaGetLastError();
        }
        rc = e == cudaSuccess ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA;
    }
    if (tab != tables) delete[] tab;
    return rc;
}

}  // extern "C"

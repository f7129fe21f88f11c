// convert.cu -- bf16 -> fp16 conversion, for running bf16 data through the fp16-operand
// attention path (FORGE_ATTN_FP16).
//
// fp16 keeps 11 significant bits where bf16 keeps 8, so P and dS enter the tensor-core
// products with a quarter of bf16's relative rounding (2^-11 against 2^-8) at the same
// tensor-core rate; bf16 inputs reach that path through this exact-in-range
// conversion.  Each value goes bf16 -> fp32 (exact) -> fp16 (round to nearest even): one
// rounding of the exact value, which changes nothing for magnitudes in [2^-14, 65504]
// (8 significant bits fit in fp16's 11), puts smaller magnitudes on fp16's subnormal
// grid (absolute error at most 2^-25) and turns larger ones into infinities, which the
// kernel counts.  HBM-bound: 2 bytes read and 2 written per value.
#include "forge_internal.h"
#include "forge_attn.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr int kCvtThreads = 256;
constexpr float kF16Max = 65504.f;

// Eight values per thread and iteration: one 16-byte load, eight conversions, one 16-byte
// store; block 0 also converts the n % 8 values after the last full group.  The number
// of values beyond fp16's finite range is summed per warp and added to *overflow.
__global__ void __launch_bounds__(kCvtThreads)
    bf16_to_fp16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n8,
                        int n_tail, unsigned int* __restrict__ overflow) {
    unsigned int over = 0;
    const long long stride = (long long)gridDim.x * kCvtThreads;
    for (long long i = (long long)blockIdx.x * kCvtThreads + threadIdx.x; i < n8; i += stride) {
        const uint4 a = src[i];
        const uint32_t in[4] = {a.x, a.y, a.z, a.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = unpack16x2<false>(in[j]);
            over += (fabsf(f.x) > kF16Max) + (fabsf(f.y) > kF16Max);
            out[j] = pack16x2<true>(f.x, f.y);
        }
        dst[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < n_tail) {
        const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src + n8);
        uint16_t* d16 = reinterpret_cast<uint16_t*>(dst + n8);
        const float f = __uint_as_float((uint32_t)s16[threadIdx.x] << 16);
        over += fabsf(f) > kF16Max;
        d16[threadIdx.x] = __half_as_ushort(__float2half_rn(f));
    }
    if (overflow) {
        const unsigned int w = __reduce_add_sync(0xffffffffu, over);
        if ((threadIdx.x & 31) == 0 && w) atomicAdd(overflow, w);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace forge

using namespace forge;

extern "C" int forge_attn_bf16_to_fp16(const void* src, void* dst, long long n,
                                       unsigned int* overflow, void* stream) {
    if (n < 0) return FORGE_ATTN_ERR_INVALID_ARG;
    if (n == 0) return FORGE_ATTN_OK;
    if (!src || !dst) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst) ||
        (reinterpret_cast<uintptr_t>(overflow) & 3u))
        return FORGE_ATTN_ERR_MISALIGNED;
    const uintptr_t s = reinterpret_cast<uintptr_t>(src), d = reinterpret_cast<uintptr_t>(dst);
    const uintptr_t bytes = 2u * static_cast<uintptr_t>(n);
    if (s < d + bytes && d < s + bytes) return FORGE_ATTN_ERR_INVALID_ARG;  // overlap
    const long long n8 = n / 8;
    const long long want = (n8 + kCvtThreads - 1) / kCvtThreads;
    const long long cap = 8LL * sm_count();
    const int blocks = (int)(want < 1 ? 1 : (want > cap ? cap : want));
    bf16_to_fp16_kernel<<<blocks, kCvtThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src), static_cast<uint4*>(dst), n8, (int)(n % 8), overflow);
    return cudaGetLastError() == cudaSuccess ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA;
}

// forge_internal.h -- declarations shared by the library's translation units
// (kernel launchers and the C ABI).  Not installed; not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace forge {

// Tile geometry common to all attention kernels: 128 query rows x 128 keys.
constexpr int kTile = 128;

// Raises `kernel`'s dynamic shared memory limit to `bytes` on the current device.
// The attribute is per device, so `done` keeps one bit per device already set
// (devices 64 and up are set on every call).  Concurrent first calls may both set
// it, which is harmless.
template <typename Kernel>
cudaError_t set_max_dynamic_smem(Kernel* kernel, int bytes,
                                 std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit != 0 && (done.load(std::memory_order_relaxed) & bit) != 0) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// Launches `kernel` with programmatic stream serialisation: its CTAs may be scheduled
// while the previous kernel in the stream runs its last CTAs, and they wait in
// grid_dependency_wait() (sm100_ptx.cuh) until that kernel has completed.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Number of SMs of the current device: the persistent kernels launch one CTA per SM.
// Cached per device ordinal (devices 64 and up query on every call); concurrent
// first calls may both query, which is harmless.
inline int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    const bool cached = dev >= 0 && dev < 64;
    if (cached) {
        const int n = cache[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    if (cached) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Launchers.  Tensor maps describe bf16 [B*H][T][d] tensors with a
// {64, 128, 1} box and 128-byte swizzle.
// f16: q, k, v (and dO) are fp16 and the 16-bit outputs are fp16; else bf16.
// The one-query-tile persistent forward; o is 16-bit or fp32 (o_f32).
cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            void* o, float* lse, int BH, int T, int d, float scale, int causal,
                            int o_f32, int precise, int f16, cudaStream_t stream);

// Row statistics of the backward: fp32 [2][B*H][t_pad], t_pad = 128 * ceil(T / 128).
cudaError_t launch_bwd_preprocess(const void* o, const void* dO, const float* lse,
                                  float* rowstats, float* dq_accum, int BH, int T, int d,
                                  int o_f32, int f16, cudaStream_t stream);

// tdq: the fp32 dQ accumulator [B*H][T][d] in {32, 128, 1} boxes, 128-byte swizzle.
cudaError_t launch_bwd_dkdv(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const float* rowstats,
                            float* dq_accum, void* dk, void* dv, int BH, int T, int d,
                            float scale, int causal, int grad_f32, int precise, int f16,
                            cudaStream_t stream);

cudaError_t launch_bwd_dq_convert(const float* dq_accum, void* dq, long long n, int f16,
                                  cudaStream_t stream);

cudaError_t launch_probe_mma(const CUtensorMap& ta, const CUtensorMap& tb, const void* a_raw,
                             float* d_out, int N, int K, int mode, cudaStream_t stream);

cudaError_t launch_probe_wait_timeout(unsigned long long limit_ns, cudaStream_t stream);

// Device error words, one per translation unit with kernels: each reader ORs its
// word into *value and clears it (the stream must have been synchronised).
cudaError_t read_and_clear_device_error_fwd(unsigned int* value);
cudaError_t read_and_clear_device_error_bwd(unsigned int* value);
cudaError_t read_and_clear_device_error_probe(unsigned int* value);
cudaError_t read_and_clear_device_error_gemm(unsigned int* value);

// 2-D 16-bit tensor map: [rows][inner] (inner contiguous), {box_inner, box_rows} boxes,
// 128-byte swizzle, zero fill outside the tensor (defined with the C ABI).
cudaError_t encode_map_2d16(CUtensorMap* map, const void* base, long long inner, long long rows,
                            int box_inner, int box_rows, bool f16);

}  // namespace forge

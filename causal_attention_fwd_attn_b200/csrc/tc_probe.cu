// tc_probe.cu -- test-support kernels: one 128 x N x K tensor-core tile product in
// each operand form the attention kernels use, and a bounded wait that must give
// up.  They exercise exactly the PTX wrappers of sm100_ptx.cuh, so a descriptor
// or layout mistake shows up here on a single tile before it shows up as an
// attention mismatch.
#include "forge_internal.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr int kProbeThreads = 128;
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 128 bytes

struct ProbeBars {
    uint64_t load;
    uint64_t mma;
    uint32_t tmem_base;
    int abort;
};

// Shared memory: A region (2 chunks), B region (2 chunks), barriers.
constexpr int kOffA = 0;
constexpr int kOffB = 2 * kChunkBytes;
constexpr int kOffBar = 4 * kChunkBytes;
constexpr int kProbeSmem = kOffBar + 64 + 1024;

__global__ void __launch_bounds__(kProbeThreads, 1)
    probe_mma_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __nv_bfloat16* __restrict__ a_raw, float* __restrict__ d_out, int N,
                     int K, int mode) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ProbeBars* bars = reinterpret_cast<ProbeBars*>(smem + kOffBar);
    volatile int* abort = &bars->abort;
    const uint32_t warp = warp_id(), lane = lane_id();
    const uint32_t row = (warp << 5) + lane;
    const uint32_t lane_off = (warp << 5) << 16;
    constexpr uint32_t kColD = 0, kColA = 128;

    if (threadIdx.x == 0) {
        mbar_init(&bars->load, 1);
        mbar_init(&bars->mma, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bars->tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (mode == 2) {
        // A [128][K] row-major from global into TMEM: row = lane, 2 bf16 per column
        const uint32_t* src = reinterpret_cast<const uint32_t*>(a_raw + (size_t)row * K);
        for (int c = 0; c < K / 2; c += 32) {
            uint32_t r[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = src[c + e];
            tmem_st32(tmem + lane_off + kColA + c, r);
        }
        tmem_wait_st();
        tc_fence_before();
    }
    __syncthreads();

    if (threadIdx.x == 0) {
        tc_fence_after();
        // loads: chunk c of each operand covers 64 elements of its contiguous dim
        uint32_t bytes = 0;
        const int a_chunks = (mode == 2) ? 0 : (mode == 3 ? 2 : K / 64);
        const int b_chunks = (mode == 0) ? K / 64 : N / 64;
        bytes = (a_chunks + b_chunks) * kChunkBytes;
        mbar_arrive_expect_tx(&bars->load, bytes);
        for (int c = 0; c < a_chunks; ++c)
            tma_load_3d(smem + kOffA + c * kChunkBytes, &tmap_a, &bars->load, 64 * c, 0, 0);
        for (int c = 0; c < b_chunks; ++c)
            tma_load_3d(smem + kOffB + c * kChunkBytes, &tmap_b, &bars->load, 64 * c, 0, 0);
        if (mbar_wait(&bars->load, 0, 1, abort)) {
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + kOffA);
            const uint32_t b_addr = smem_u32(smem + kOffB);
            for (int kk = 0; kk < K / 16; ++kk) {
                const uint32_t kmaj = (kk >> 2) * kChunkBytes + (kk & 3) * 32;  // K-major step
                const uint32_t mnmaj = kk * 2048;                                 // MN-major step
                const uint32_t acc = kk > 0 ? 1u : 0u;
                if (mode == 0) {
                    mma_ss(tmem + kColD, sdesc_sw128(a_addr + kmaj, 16, 1024),
                           sdesc_sw128(b_addr + kmaj, 16, 1024),
                           idesc_bf16_f32(128, N, false, false), acc);
                } else if (mode == 1) {
                    mma_ss(tmem + kColD, sdesc_sw128(a_addr + kmaj, 16, 1024),
                           sdesc_sw128(b_addr + mnmaj, kChunkBytes, 1024),
                           idesc_bf16_f32(128, N, false, true), acc);
                } else if (mode == 2) {
                    mma_ts(tmem + kColD, tmem + kColA + kk * 8,
                           sdesc_sw128(b_addr + mnmaj, kChunkBytes, 1024),
                           idesc_bf16_f32(128, N, false, true), acc);
                } else {
                    mma_ss(tmem + kColD, sdesc_sw128(a_addr + mnmaj, kChunkBytes, 1024),
                           sdesc_sw128(b_addr + mnmaj, kChunkBytes, 1024),
                           idesc_bf16_f32(128, N, true, true), acc);
                }
            }
            mma_commit(&bars->mma);
        } else {
            mbar_wait_drain(&bars->load, 0);
        }
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->mma, 0, 2, abort));
    if (ok) {
        tc_fence_after();
        for (int c = 0; c < N; c += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + kColD + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) d_out[(size_t)row * N + c + e] = __uint_as_float(r[e]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// Waits on a barrier that nothing completes; must give up after limit_ns.
__global__ void probe_wait_timeout_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, 0x7FF, &abort, limit_ns);
    __syncthreads();
}

}  // namespace

cudaError_t launch_probe_mma(const CUtensorMap& ta, const CUtensorMap& tb, const void* a_raw,
                             float* d_out, int N, int K, int mode, cudaStream_t stream) {
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = set_max_dynamic_smem(probe_mma_kernel, kProbeSmem, configured);
    if (e != cudaSuccess) return e;
    probe_mma_kernel<<<1, kProbeThreads, kProbeSmem, stream>>>(
        ta, tb, static_cast<const __nv_bfloat16*>(a_raw), d_out, N, K, mode);
    return cudaGetLastError();
}

cudaError_t launch_probe_wait_timeout(unsigned long long limit_ns, cudaStream_t stream) {
    probe_wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_error_probe(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

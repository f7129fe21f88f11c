// forge_attn_api.cu -- the C ABI declared in include/forge_attn.h and
// include/forge_attn_testing.h: argument checks, TMA tensor-map encoding and
// kernel dispatch.  No computation happens here; every step of the operation
// runs in the kernels of attn_fwd.cu and attn_bwd.cu.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "forge_attn.h"
#include "forge_attn_testing.h"
#include "forge_internal.h"

namespace forge {

cudaError_t read_and_clear_device_error(unsigned int* value, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    unsigned int v = 0;
    if ((e = read_and_clear_device_error_fwd(&v)) != cudaSuccess) return e;
    if ((e = read_and_clear_device_error_bwd(&v)) != cudaSuccess) return e;
    if ((e = read_and_clear_device_error_probe(&v)) != cudaSuccess) return e;
    if ((e = read_and_clear_device_error_gemm(&v)) != cudaSuccess) return e;
    *value = v;
    return cudaSuccess;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 16-bit (bf16, or fp16 when f16) tensor viewed as [planes][rows][inner] (inner
// contiguous), loaded in {64, 128, 1} boxes with 128-byte swizzle.  Rows past `rows`
// read as zero and are clipped on store, so a ragged last tile never touches the next
// plane.
int make_map_16(CUtensorMap* map, const void* base, long long inner, long long rows,
                long long planes, bool f16 = false) {
    auto fn = encode_fn();
    if (!fn) return FORGE_ATTN_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)(inner * 2), (cuuint64_t)(inner * rows * 2)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA;
}

// fp32 tensor [planes][rows][inner] in {32, 128, 1} boxes with 128-byte swizzle (the
// dQ accumulator, written by TMA reduce-add).
int make_map_f32(CUtensorMap* map, const void* base, long long inner, long long rows,
                 long long planes) {
    auto fn = encode_fn();
    if (!fn) return FORGE_ATTN_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)(inner * 4), (cuuint64_t)(inner * rows * 4)};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// 2-D 16-bit tensor [rows][inner] (inner contiguous) in {box_inner, box_rows} boxes,
// 128-byte swizzle, zero fill outside the tensor.
cudaError_t encode_map_2d16(CUtensorMap* map, const void* base, long long inner, long long rows,
                            int box_inner, int box_rows, bool f16) {
    auto fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(inner * 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

int check_shape(int B, int H, int T, int d) {
    if (B < 1 || H < 1 || T < 1 || d < 1) return FORGE_ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FORGE_ATTN_ERR_UNSUPPORTED;
    const long long n = (long long)B * H * T * d;
    if (n >= (1ll << 31)) return FORGE_ATTN_ERR_UNSUPPORTED;
    // with d >= 64 this also keeps B*H and every row index (< 2^25) well inside int
    if ((long long)B * H > 0x7fffffffll) return FORGE_ATTN_ERR_UNSUPPORTED;
    return FORGE_ATTN_OK;
}

int check_common(int B, int H, int T, int d, float scale, int causal) {
    int s = check_shape(B, H, T, d);
    if (s != FORGE_ATTN_OK) return s;
    if (!std::isfinite(scale)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FORGE_ATTN_ERR_INVALID_ARG;
    return FORGE_ATTN_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA; }

size_t round_up_256(size_t x) { return (x + 255) & ~size_t(255); }

// Bytes of the padded row statistics (LSE * log2 e and D, 2 x B*H x t_pad fp32).
size_t rowstats_bytes(int B, int H, int T) {
    const size_t t_pad = (size_t)((T + 127) / 128) * 128;
    return round_up_256(2 * (size_t)B * H * t_pad * sizeof(float));
}

}  // namespace
}  // namespace forge

using namespace forge;

extern "C" {

int forge_attn_version(void) { return 100; }

const char* forge_attn_status_string(int status) {
    switch (status) {
        case FORGE_ATTN_OK: return "ok";
        case FORGE_ATTN_ERR_INVALID_ARG: return "invalid argument";
        case FORGE_ATTN_ERR_UNSUPPORTED: return "unsupported size or head dimension";
        case FORGE_ATTN_ERR_MISALIGNED: return "misaligned pointer";
        case FORGE_ATTN_ERR_CUDA: return "CUDA error";
        case FORGE_ATTN_ERR_TIMEOUT: return "device-side wait timed out";
        case FORGE_ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        default: return "unknown status";
    }
}

int forge_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int T, int d, float scale, int causal, int flags, void* stream) {
    if (!q || !k || !v || !o || !lse) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_common(B, H, T, d, scale, causal);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_OUT_F32 | FORGE_ATTN_PRECISE | FORGE_ATTN_FP16))
        return FORGE_ATTN_ERR_INVALID_ARG;
    const bool f16 = (flags & FORGE_ATTN_FP16) != 0;
    if (f16 && (flags & FORGE_ATTN_PRECISE)) return FORGE_ATTN_ERR_UNSUPPORTED;
    const bool o_f32 = (flags & FORGE_ATTN_OUT_F32) != 0;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return FORGE_ATTN_ERR_MISALIGNED;
    const long long BH = (long long)B * H;
    CUtensorMap tq, tk, tv;
    if ((s = make_map_16(&tq, q, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_16(&tk, k, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_16(&tv, v, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    return cuda_status(launch_attn_fwd(tq, tk, tv, o, lse, (int)BH, T, d, scale, causal,
                                       o_f32, (flags & FORGE_ATTN_PRECISE) != 0, f16,
                                       static_cast<cudaStream_t>(stream)));
}

int forge_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int T, int d, float scale, int causal, void* stream) {
    return forge_attn_fwd_ex(q, k, v, o, lse, B, H, T, d, scale, causal, 0, stream);
}

size_t forge_attn_bwd_workspace_size(int B, int H, int T, int d) {
    if (check_shape(B, H, T, d) != FORGE_ATTN_OK) return 0;
    const size_t rows = (size_t)B * H * T;
    return rowstats_bytes(B, H, T) + round_up_256(rows * d * sizeof(float));
}

int forge_attn_bwd_preprocess(const void* o, const void* dO, const float* lse, float* rowstats,
                              float* dq_accum, int B, int H, int T, int d, int flags,
                              void* stream) {
    if (!o || !dO || !lse || !rowstats) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_shape(B, H, T, d);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_O_IN_F32 | FORGE_ATTN_FP16)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(dO) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
        !aligned16(rowstats) || (dq_accum && !aligned16(dq_accum)))
        return FORGE_ATTN_ERR_MISALIGNED;
    return cuda_status(launch_bwd_preprocess(o, dO, lse, rowstats, dq_accum, B * H, T, d,
                                             (flags & FORGE_ATTN_O_IN_F32) != 0,
                                             (flags & FORGE_ATTN_FP16) != 0,
                                             static_cast<cudaStream_t>(stream)));
}

int forge_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO,
                        const float* rowstats, float* dq_accum, void* dk, void* dv, int B, int H,
                        int T, int d, float scale, int causal, int flags, void* stream) {
    if (!q || !k || !v || !dO || !rowstats || !dq_accum || !dk || !dv)
        return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_common(B, H, T, d, scale, causal);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_OUT_F32 | FORGE_ATTN_PRECISE | FORGE_ATTN_FP16))
        return FORGE_ATTN_ERR_INVALID_ARG;
    const bool f16 = (flags & FORGE_ATTN_FP16) != 0;
    if (f16 && (flags & FORGE_ATTN_PRECISE)) return FORGE_ATTN_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(dq_accum) || !aligned16(rowstats))
        return FORGE_ATTN_ERR_MISALIGNED;
    const long long BH = (long long)B * H;
    CUtensorMap tq, tk, tv, tdo, tdq;
    if ((s = make_map_16(&tq, q, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_16(&tk, k, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_16(&tv, v, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_16(&tdo, dO, d, T, BH, f16)) != FORGE_ATTN_OK) return s;
    if ((s = make_map_f32(&tdq, dq_accum, d, T, BH)) != FORGE_ATTN_OK) return s;
    return cuda_status(launch_bwd_dkdv(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv, (int)BH, T,
                                       d, scale, causal, (flags & FORGE_ATTN_OUT_F32) != 0,
                                       (flags & FORGE_ATTN_PRECISE) != 0, f16,
                                       static_cast<cudaStream_t>(stream)));
}

int forge_attn_bwd_dq_convert_ex(const float* dq_accum, void* dq, int B, int H, int T, int d,
                                 int flags, void* stream) {
    if (!dq_accum || !dq) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_shape(B, H, T, d);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~FORGE_ATTN_FP16) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(dq_accum) || !aligned16(dq)) return FORGE_ATTN_ERR_MISALIGNED;
    return cuda_status(launch_bwd_dq_convert(dq_accum, dq, (long long)B * H * T * d,
                                             (flags & FORGE_ATTN_FP16) != 0,
                                             static_cast<cudaStream_t>(stream)));
}

int forge_attn_bwd_dq_convert(const float* dq_accum, void* dq, int B, int H, int T, int d,
                              void* stream) {
    return forge_attn_bwd_dq_convert_ex(dq_accum, dq, B, H, T, d, 0, stream);
}

int forge_attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                      const void* dO, const float* lse, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, int B, int H, int T, int d,
                      float scale, int causal, int flags, void* stream) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv)
        return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_common(B, H, T, d, scale, causal);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_OUT_F32 | FORGE_ATTN_O_IN_F32 | FORGE_ATTN_PRECISE | FORGE_ATTN_FP16))
        return FORGE_ATTN_ERR_INVALID_ARG;
    if ((flags & FORGE_ATTN_FP16) && (flags & FORGE_ATTN_PRECISE)) return FORGE_ATTN_ERR_UNSUPPORTED;
    const bool grad_f32 = (flags & FORGE_ATTN_OUT_F32) != 0;
    const size_t need = forge_attn_bwd_workspace_size(B, H, T, d);
    if (!workspace || workspace_bytes < need) return FORGE_ATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FORGE_ATTN_ERR_MISALIGNED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return FORGE_ATTN_ERR_MISALIGNED;
    float* rowstats = static_cast<float*>(workspace);
    float* acc = grad_f32 ? static_cast<float*>(dq)
                          : reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                     rowstats_bytes(B, H, T));
    if ((s = forge_attn_bwd_preprocess(o, dO, lse, rowstats, acc, B, H, T, d,
                                       flags & (FORGE_ATTN_O_IN_F32 | FORGE_ATTN_FP16),
                                       stream)) != FORGE_ATTN_OK)
        return s;
    if ((s = forge_attn_bwd_dkdv(q, k, v, dO, rowstats, acc, dk, dv, B, H, T, d, scale, causal,
                                 flags & (FORGE_ATTN_OUT_F32 | FORGE_ATTN_PRECISE | FORGE_ATTN_FP16),
                                 stream)) != FORGE_ATTN_OK)
        return s;
    if (!grad_f32)
        s = forge_attn_bwd_dq_convert_ex(acc, dq, B, H, T, d, flags & FORGE_ATTN_FP16, stream);
    return s;
}

int forge_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int H, int T, int d, float scale, int causal,
                   void* stream) {
    return forge_attn_bwd_ex(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, T,
                             d, scale, causal, 0, stream);
}

int forge_attn_check_device_error(void* stream, unsigned int* detail) {
    unsigned int v = 0;
    cudaError_t e = read_and_clear_device_error(&v, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return FORGE_ATTN_ERR_CUDA;
    if (detail) *detail = v;
    return v ? FORGE_ATTN_ERR_TIMEOUT : FORGE_ATTN_OK;
}

// ------------------------------------------------------------ test support --
int forge_probe_mma(const void* a, const void* b, float* d_out, int N, int K, int mode,
                    void* stream) {
    if (!a || !b || !d_out) return FORGE_ATTN_ERR_INVALID_ARG;
    if ((N != 64 && N != 128) || (K != 64 && K != 128) || mode < 0 || mode > 3)
        return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d_out)) return FORGE_ATTN_ERR_MISALIGNED;
    CUtensorMap ta, tb;
    int s;
    // A: [128][K] (modes 0-2) or [K][128] (mode 3); B: [N][K] (mode 0) or [K][N]
    if (mode == 3)
        s = make_map_16(&ta, a, 128, K, 1);
    else
        s = make_map_16(&ta, a, K, 128, 1);
    if (s != FORGE_ATTN_OK) return s;
    if (mode == 0)
        s = make_map_16(&tb, b, K, N, 1);
    else
        s = make_map_16(&tb, b, N, K, 1);
    if (s != FORGE_ATTN_OK) return s;
    return cuda_status(
        launch_probe_mma(ta, tb, a, d_out, N, K, mode, static_cast<cudaStream_t>(stream)));
}

int forge_probe_wait_timeout(unsigned long long limit_ns, void* stream) {
    if (limit_ns < 1000ull) limit_ns = 1000ull;
    if (limit_ns > 1000000000ull) limit_ns = 1000000000ull;
    return cuda_status(launch_probe_wait_timeout(limit_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// gemm.cu -- the projection GEMMs around attention on tcgen05 tensor cores.
//
// The Forge paper ("Building an LLM Training Framework from Scratch in C++ and Metal
// on Apple Silicon") measures, besides attention, the three products of a linear
// layer in training (section "Results", the GEMM table; section "Finding 4.2" for
// the transposed variants):
//   forward   Y  = X W^T     [tokens][out] = [tokens][in] x [out][in]^T
//   backward  dX = dY W      [tokens][in]  = [tokens][out] x [out][in]
//             dW = dY^T X    [out][in]     = [tokens][out]^T x [tokens][in]
// and notes that dW lags because its reduction runs over all tokens with few output
// tiles, which split-K would fix.  All three are one kernel here,
//   C[m][n] = sum_k A[m][k] B[n][k],
// with each operand either K-major (stored [rows][k]) or MN-major (stored [k][rows]):
//   Y : A = X  (K-major), B = W  (K-major)
//   dX: A = dY (K-major), B = W  (MN-major: W is stored [out = k][in = n])
//   dW: A = dY (MN-major), B = X (MN-major), k = tokens, split over k.
// The transposes are descriptor choices (the operand-role exchange the paper uses for
// its transposed attention products), never data movement.
//
// Design (persistent, one CTA per SM, 6 warps; tiles of BM x BN = 128 x 128, 128 x 256
// or 256 x 256):
//   warp 0      TMA producer: A and B k-blocks (64 deep) into a kStages ring.
//   warp 1      MMA issuer (converged warp, one elected lane): 128 x BN x 16
//               tcgen05 products, BM / 128 of them per 16-deep step sharing the B
//               operand (one per 128-row half of the tile), into tensor memory: two
//               accumulators when the tile fits twice (128-row tiles), so one tile's
//               epilogue overlaps the next tile's products, else one (256 x 256).
//   warps 2..5  epilogue: warp w reads TMEM lanes 32 (w % 4).. (its 32 rows of each
//               128-row half), converts and stores them, or adds them (fp32
//               reductions) into C for split-K and accumulation.
// Work units are (split, tile) pairs walked by all CTAs in the same order; tiles are
// grouped eight M-rows at a time so the CTAs live at once share operand panels in L2.
#include "forge_internal.h"
#include "forge_linear.h"
#include "forge_attn.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr int kGemmThreads = 192;
constexpr int kBM = 128, kBK = 64;
constexpr int kGroupM = 8;

enum : uint32_t { kGSiteFull = 1, kGSiteEmpty, kGSiteAccFull, kGSiteAccEmpty };
enum OutMode : int { kOut16 = 0, kOutF32 = 1, kOutF32Add = 2 };

template <int BM, int BN>
struct GemmCfg {
    static constexpr int kHalves = BM / kBM;          // 128-row halves of a tile
    static constexpr int kHalfBytes = kBM * kBK * 2;  // 16 KB of A per half
    static constexpr int kABytes = kHalves * kHalfBytes;
    static constexpr int kBBytes = BN * kBK * 2;      // 16 or 32 KB
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = kStageBytes >= 65536 ? 3 : (kStageBytes >= 49152 ? 4 : 6);
    static constexpr int kChunkBytes = kBK * 128;  // one 64-element MN chunk of a k-block
    static constexpr int kOffBar = kStages * kStageBytes;
    static constexpr int kSmemBytes = kOffBar + 256 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static constexpr int kAccCols = kHalves * BN;  // one accumulator
    static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
    static constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
    static_assert(kTmemCols <= 512 && kStages <= 6, "tensor memory / barrier budget");
};

struct GemmBarriers {
    uint64_t full[6], empty[6];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mma_final;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(GemmBarriers) <= 256, "barrier block");

struct GemmShape {
    int M, N, K;
    int tiles_m, tiles_n, k_blocks, kb_per_split, splits, units;
};

// Tile (tm, tn) and k-block range of work unit u.
__device__ __forceinline__ void unit_of(const GemmShape& s, int u, int& tm, int& tn, int& kb0,
                                        int& kb1) {
    const int tiles = s.tiles_m * s.tiles_n;
    const int split = u / tiles;
    const int t = u - split * tiles;
    // groups of kGroupM tile rows, column-major inside a group
    const int per_group = kGroupM * s.tiles_n;
    const int grp = t / per_group;
    const int first_m = grp * kGroupM;
    const int rows = min(kGroupM, s.tiles_m - first_m);
    const int r = t - grp * per_group;
    tm = first_m + r % rows;
    tn = r / rows;
    kb0 = split * s.kb_per_split;
    kb1 = min(kb0 + s.kb_per_split, s.k_blocks);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t site,
                                          volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, site, abort));
}

template <int BM, int BN, bool A_MN, bool B_MN, int OUT, bool F16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                const __grid_constant__ CUtensorMap tmap_b, void* __restrict__ c_out,
                const GemmShape shape) {
    using C = GemmCfg<BM, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    GemmBarriers* bars = reinterpret_cast<GemmBarriers*>(smem + C::kOffBar);
    volatile int* abort = &bars->abort;
    const uint32_t warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
        }
        mbar_init(&bars->mma_final, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmap_a);
            tma_prefetch_desc(&tmap_b);
            int it = 0;  // k-blocks loaded so far (all units)
            int last_use[6] = {-1, -1, -1, -1, -1, -1};
            bool run = true;
            for (int u = blockIdx.x; run && u < shape.units; u += gridDim.x) {
                int tm, tn, kb0, kb1;
                unit_of(shape, u, tm, tn, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int st = it % C::kStages, use = it / C::kStages;
                    if (use > 0 &&
                        !mbar_wait(&bars->empty[st], (use - 1) & 1, kGSiteEmpty, abort)) {
                        run = false;
                        break;
                    }
                    uint8_t* sa = smem + st * C::kStageBytes;
                    uint8_t* sb = sa + C::kABytes;
                    mbar_arrive_expect_tx(&bars->full[st], C::kStageBytes);
                    if constexpr (A_MN) {
                        for (int c = 0; c < BM / 64; ++c)
                            tma_load_2d(sa + c * C::kChunkBytes, &tmap_a, &bars->full[st],
                                        tm * BM + 64 * c, kb * kBK);
                    } else {
                        for (int h = 0; h < C::kHalves; ++h)
                            tma_load_2d(sa + h * C::kHalfBytes, &tmap_a, &bars->full[st],
                                        kb * kBK, tm * BM + kBM * h);
                    }
                    if constexpr (B_MN) {
                        for (int c = 0; c < BN / 64; ++c)
                            tma_load_2d(sb + c * C::kChunkBytes, &tmap_b, &bars->full[st],
                                        tn * BN + 64 * c, kb * kBK);
                    } else {
                        tma_load_2d(sb, &tmap_b, &bars->full[st], kb * kBK, tn * BN);
                    }
                    last_use[st] = use;
                }
            }
            if (*abort)  // let copies already issued land before the CTA's memory goes
                for (int s = 0; s < C::kStages; ++s)
                    if (last_use[s] >= 0) mbar_wait_drain(&bars->full[s], last_use[s] & 1);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        constexpr uint32_t kIdesc = idesc_f16kind_f32(kBM, BN, A_MN, B_MN, F16);
        int it = 0, n_unit = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < shape.units; u += gridDim.x, ++n_unit) {
            int tm, tn, kb0, kb1;
            unit_of(shape, u, tm, tn, kb0, kb1);
            const int buf = C::kAccBufs == 2 ? n_unit & 1 : 0;
            const int use = C::kAccBufs == 2 ? n_unit >> 1 : n_unit;
            // the accumulator must have been read out by the epilogue of the unit that
            // used it last (two units ago, or the previous one with a single accumulator)
            if (use > 0 &&
                !warp_wait(&bars->acc_empty[buf], (use - 1) & 1, kGSiteAccEmpty, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem + buf * C::kAccCols;
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int st = it % C::kStages;
                if (!warp_wait(&bars->full[st], (it / C::kStages) & 1, kGSiteFull, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + st * C::kStageBytes);
                const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
                    // K-major: 16 k-values = 32 bytes along the swizzled row;
                    // MN-major: 16 k-rows = two 8-row groups of 1024 bytes
                    const uint64_t bd = B_MN ? sdesc_sw128(b_addr + kk * 2048, C::kChunkBytes, 1024)
                                             : sdesc_sw128(b_addr + kk * 32, 16, 1024);
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h) {
                        const uint32_t ah = a_addr + h * C::kHalfBytes;
                        const uint64_t ad = A_MN ? sdesc_sw128(ah + kk * 2048, C::kChunkBytes, 1024)
                                                 : sdesc_sw128(ah + kk * 32, 16, 1024);
                        mma_ss_warp(tacc + h * BN, ad, bd, kIdesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit_warp(&bars->empty[st]);
            }
            if (ok) mma_commit_warp(&bars->acc_full[buf]);
        }
        mma_commit_warp(&bars->mma_final);
        mbar_wait_drain(&bars->mma_final, 0);
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t quarter = warp & 3;
        const uint32_t lane_off = (quarter * 32u) << 16;
        int n_unit = 0;
        for (int u = blockIdx.x; u < shape.units; u += gridDim.x, ++n_unit) {
            int tm, tn, kb0, kb1;
            unit_of(shape, u, tm, tn, kb0, kb1);
            const int buf = C::kAccBufs == 2 ? n_unit & 1 : 0;
            const int use = C::kAccBufs == 2 ? n_unit >> 1 : n_unit;
            if (!warp_wait(&bars->acc_full[buf], use & 1, kGSiteAccFull, abort)) break;
            tc_fence_after();
            // 32-column chunks of the accumulator, four loads in flight per wait
            constexpr int kChunks = C::kHalves * (BN / 32), kG = 4;
            static_assert(kChunks % kG == 0, "epilogue load groups");
#pragma unroll 1
            for (int g = 0; g < kChunks / kG; ++g) {
                uint32_t r[32 * kG];
#pragma unroll
                for (int j = 0; j < kG; ++j) {
                    const int hc = g * kG + j, h = hc / (BN / 32), c = hc % (BN / 32);
                    tmem_ld32(tmem + lane_off + buf * C::kAccCols + h * BN + c * 32, r + 32 * j);
                }
                tmem_wait_ld();
                if (g == kChunks / kG - 1) {  // the accumulator has been read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
                }
#pragma unroll
                for (int j = 0; j < kG; ++j) {
                    const int hc = g * kG + j, h = hc / (BN / 32), c = hc % (BN / 32);
                    const int row = tm * BM + h * kBM + (int)(quarter * 32 + lane);
                    const int col0 = tn * BN + c * 32;
                    const uint32_t* q = r + 32 * j;
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {  // groups of 8 columns (N % 8 == 0)
                        const int col = col0 + 8 * gq;
                        if (row >= shape.M || col >= shape.N) continue;
                        const size_t off = (size_t)row * shape.N + col;
                        const uint32_t* v = q + 8 * gq;
                        if constexpr (OUT == kOut16) {
                            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(c_out) + off) =
                                make_uint4(
                                    pack16x2<F16>(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                    pack16x2<F16>(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                    pack16x2<F16>(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                    pack16x2<F16>(__uint_as_float(v[6]), __uint_as_float(v[7])));
                        } else if constexpr (OUT == kOutF32) {
                            float4* dst =
                                reinterpret_cast<float4*>(static_cast<float*>(c_out) + off);
                            dst[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]),
                                                 __uint_as_float(v[2]), __uint_as_float(v[3]));
                            dst[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]),
                                                 __uint_as_float(v[6]), __uint_as_float(v[7]));
                        } else {
                            // two 16-byte vector reductions (N % 8 == 0 keeps them aligned)
                            float* dst = static_cast<float*>(c_out) + off;
                            red_add_v4(dst, __uint_as_float(v[0]), __uint_as_float(v[1]),
                                       __uint_as_float(v[2]), __uint_as_float(v[3]));
                            red_add_v4(dst + 4, __uint_as_float(v[4]), __uint_as_float(v[5]),
                                       __uint_as_float(v[6]), __uint_as_float(v[7]));
                        }
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int BM, int BN, bool A_MN, bool B_MN, int OUT, bool F16>
cudaError_t launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, void* c,
                          const GemmShape& s, cudaStream_t stream) {
    using C = GemmCfg<BM, BN>;
    static std::atomic<unsigned long long> configured{0};
    auto* kernel = gemm_kernel<BM, BN, A_MN, B_MN, OUT, F16>;
    cudaError_t e = set_max_dynamic_smem(kernel, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    const int grid = s.units < sm_count() ? s.units : sm_count();
    kernel<<<grid, kGemmThreads, C::kSmemBytes, stream>>>(ta, tb, c, s);
    return cudaGetLastError();
}

// Tile shape of a launch: 128 x 128, 128 x 256 or 256 x 256.
struct Tile {
    int bm, bn;
};

template <bool A_MN, bool B_MN>
cudaError_t launch_gemm_layout(const CUtensorMap& ta, const CUtensorMap& tb, void* c,
                               const GemmShape& s, Tile t, int out, bool f16,
                               cudaStream_t stream) {
#define FORGE_GEMM_OUT(BM_, BN_, F16_)                                                         \
    switch (out) {                                                                             \
        case kOut16:                                                                           \
            return launch_gemm_t<BM_, BN_, A_MN, B_MN, kOut16, F16_>(ta, tb, c, s, stream);    \
        case kOutF32:                                                                          \
            return launch_gemm_t<BM_, BN_, A_MN, B_MN, kOutF32, F16_>(ta, tb, c, s, stream);   \
        default:                                                                               \
            return launch_gemm_t<BM_, BN_, A_MN, B_MN, kOutF32Add, F16_>(ta, tb, c, s, stream);\
    }
#define FORGE_GEMM_TILE(BM_, BN_)                 \
    if (f16) { FORGE_GEMM_OUT(BM_, BN_, true) }   \
    FORGE_GEMM_OUT(BM_, BN_, false)
    if (t.bm == 256) { FORGE_GEMM_TILE(256, 256) }
    if (t.bn == 256) { FORGE_GEMM_TILE(128, 256) }
    FORGE_GEMM_TILE(128, 128)
#undef FORGE_GEMM_TILE
#undef FORGE_GEMM_OUT
}

GemmShape make_shape(int M, int N, int K, Tile t, int splits) {
    GemmShape s;
    s.M = M;
    s.N = N;
    s.K = K;
    s.tiles_m = (M + t.bm - 1) / t.bm;
    s.tiles_n = (N + t.bn - 1) / t.bn;
    s.k_blocks = (K + kBK - 1) / kBK;
    if (splits < 1) splits = 1;
    if (splits > s.k_blocks) splits = s.k_blocks;
    s.kb_per_split = (s.k_blocks + splits - 1) / splits;
    s.splits = (s.k_blocks + s.kb_per_split - 1) / s.kb_per_split;  // no empty split
    s.units = s.splits * s.tiles_m * s.tiles_n;
    return s;
}

// Tile shape and split of the reduction over K for a launch.
struct Plan {
    Tile tile;
    int splits;
};

// Cost model of a plan, fitted on linear-layer shapes.  Shared-memory traffic sets the
// pace of a k-block: the TMA writes of its operands plus the tensor cores' reads of them
// (each 128 x BN x 16 product reads its A and B slices), 64, 96 and 160 KB for 128 x 128,
// 128 x 256 and 256 x 256 tiles (weights 2, 3, 5) for 1, 2 and 4 times the work;
// measured times per unit of work were 1 : 0.76 : 0.67 (square 8192), where these bytes
// give 1 : 0.75 : 0.63 and the tensor-core time alone would give 1 : 1 : 1.  A 256 x 256
// tile's accumulator fills tensor memory alone, so the next tile's products wait for its
// epilogue: weight 32 more per tile.  A plan costs what its most loaded CTA does (units
// are dealt round robin), plus, with more than one split, the fp32 reductions of every
// split's partial output in L2 (after a memset of C): weight 1e-5 per output element and
// split.
double plan_cost(int M, int N, int K, Tile t, int splits, int sms) {
    const GemmShape s = make_shape(M, N, K, t, splits);
    const int w = t.bm == 256 ? 5 : (t.bn == 256 ? 3 : 2);
    double c = (double)((s.units + sms - 1) / sms) *
               ((double)s.kb_per_split * w + (t.bm == 256 ? 32.0 : 0.0));
    if (s.splits > 1) c += 1e-5 * s.splits * (double)M * N;
    return c;
}

// The cheapest plan: over the three tiles (128 x 128 alone when N <= 128) and, when
// splits = 0, every split whose parts are at least eight k-blocks (512) deep, up to two
// per SM (more cannot shorten the most loaded CTA's share); else the split given.  Ties
// go to the larger tile, then to fewer splits.
Plan pick_plan(int M, int N, int K, int splits) {
    const int sms = sm_count();
    const int k_blocks = (K + kBK - 1) / kBK;
    const int lo = splits > 0 ? splits : 1;
    int hi = splits > 0 ? splits : (k_blocks / 8 > 1 ? k_blocks / 8 : 1);
    if (splits == 0 && hi > 2 * sms) hi = 2 * sms;
    Plan best{Tile{128, 128}, lo};
    double best_c = 0.0;
    bool have = false;
    for (const Tile t : {Tile{256, 256}, Tile{128, 256}, Tile{128, 128}}) {
        if (N <= 128 && t.bn != 128) continue;
        for (int sp = lo; sp <= hi; ++sp) {
            const double c = plan_cost(M, N, K, t, sp, sms);
            if (!have || c < best_c) {
                best = Plan{t, sp};
                best_c = c;
                have = true;
            }
        }
    }
    return best;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(int tokens, int in_f, int out_f) {
    if (tokens < 1 || in_f < 1 || out_f < 1) return FORGE_ATTN_ERR_INVALID_ARG;
    if (tokens % 8 || in_f % 8 || out_f % 8) return FORGE_ATTN_ERR_UNSUPPORTED;
    if ((long long)tokens * in_f >= (1ll << 31) || (long long)tokens * out_f >= (1ll << 31) ||
        (long long)out_f * in_f >= (1ll << 31))
        return FORGE_ATTN_ERR_UNSUPPORTED;
    return FORGE_ATTN_OK;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? FORGE_ATTN_OK : FORGE_ATTN_ERR_CUDA; }

}  // namespace

cudaError_t read_and_clear_device_error_gemm(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

using namespace forge;

extern "C" {

int forge_linear_fwd(const void* x, const void* w, void* y, int tokens, int in_features,
                     int out_features, int flags, void* stream) {
    if (!x || !w || !y) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_dims(tokens, in_features, out_features);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_OUT_F32 | FORGE_ATTN_FP16)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return FORGE_ATTN_ERR_MISALIGNED;
    const bool f16 = (flags & FORGE_ATTN_FP16) != 0;
    const Tile t = pick_plan(tokens, out_features, in_features, 1).tile;
    CUtensorMap ta, tb;
    if (encode_map_2d16(&ta, x, in_features, tokens, 64, kBM, f16) != cudaSuccess ||
        encode_map_2d16(&tb, w, in_features, out_features, 64, t.bn, f16) != cudaSuccess)
        return FORGE_ATTN_ERR_CUDA;
    const GemmShape sh = make_shape(tokens, out_features, in_features, t, 1);
    return status_of(launch_gemm_layout<false, false>(
        ta, tb, y, sh, t, (flags & FORGE_ATTN_OUT_F32) ? kOutF32 : kOut16, f16,
        static_cast<cudaStream_t>(stream)));
}

int forge_linear_bwd_dx(const void* dy, const void* w, void* dx, int tokens, int in_features,
                        int out_features, int flags, void* stream) {
    if (!dy || !w || !dx) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_dims(tokens, in_features, out_features);
    if (s != FORGE_ATTN_OK) return s;
    if (flags & ~(FORGE_ATTN_OUT_F32 | FORGE_ATTN_FP16)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(dy) || !aligned16(w) || !aligned16(dx)) return FORGE_ATTN_ERR_MISALIGNED;
    const bool f16 = (flags & FORGE_ATTN_FP16) != 0;
    const Tile t = pick_plan(tokens, in_features, out_features, 1).tile;
    CUtensorMap ta, tb;
    // A = dY [tokens][out] (k = out contiguous); B = W [out = k][in = n], MN-major
    if (encode_map_2d16(&ta, dy, out_features, tokens, 64, kBM, f16) != cudaSuccess ||
        encode_map_2d16(&tb, w, in_features, out_features, 64, 64, f16) != cudaSuccess)
        return FORGE_ATTN_ERR_CUDA;
    const GemmShape sh = make_shape(tokens, in_features, out_features, t, 1);
    return status_of(launch_gemm_layout<false, true>(
        ta, tb, dx, sh, t, (flags & FORGE_ATTN_OUT_F32) ? kOutF32 : kOut16, f16,
        static_cast<cudaStream_t>(stream)));
}

int forge_linear_split_k(int tokens, int in_features, int out_features) {
    if (check_dims(tokens, in_features, out_features) != FORGE_ATTN_OK) return 0;
    return pick_plan(out_features, in_features, tokens, 0).splits;
}

int forge_linear_bwd_dw(const void* dy, const void* x, float* dw, int tokens, int in_features,
                        int out_features, int split_k, int accumulate, int flags, void* stream) {
    if (!dy || !x || !dw) return FORGE_ATTN_ERR_INVALID_ARG;
    int s = check_dims(tokens, in_features, out_features);
    if (s != FORGE_ATTN_OK) return s;
    if (split_k < 0 || (accumulate != 0 && accumulate != 1)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (flags & ~FORGE_ATTN_FP16) return FORGE_ATTN_ERR_INVALID_ARG;
    if (!aligned16(dy) || !aligned16(x) || !aligned16(dw)) return FORGE_ATTN_ERR_MISALIGNED;
    const bool f16 = (flags & FORGE_ATTN_FP16) != 0;
    const Plan plan = pick_plan(out_features, in_features, tokens, split_k);
    const Tile t = plan.tile;
    const GemmShape sh = make_shape(out_features, in_features, tokens, t, plan.splits);
    CUtensorMap ta, tb;
    // A = dY^T: dY [tokens = k][out = m], MN-major; B = X [tokens = k][in = n], MN-major
    if (encode_map_2d16(&ta, dy, out_features, tokens, 64, 64, f16) != cudaSuccess ||
        encode_map_2d16(&tb, x, in_features, tokens, 64, 64, f16) != cudaSuccess)
        return FORGE_ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one split overwriting dw stores; otherwise every split adds into dw, zeroed first
    // unless accumulating
    const bool add = accumulate || sh.splits > 1;
    if (add && !accumulate) {
        cudaError_t e =
            cudaMemsetAsync(dw, 0, (size_t)out_features * in_features * sizeof(float), st);
        if (e != cudaSuccess) return FORGE_ATTN_ERR_CUDA;
    }
    return status_of(launch_gemm_layout<true, true>(ta, tb, dw, sh, t,
                                                    add ? kOutF32Add : kOutF32, f16, st));
}

}  // extern "C"

// attn_bwd.cu -- fused causal attention backward for sm_100a.
//
// The Forge paper ("Building an LLM Training Framework from Scratch in C++ and
// Metal on Apple Silicon") splits its backward into a pre-pass D = rowsum(dO o O)
// in float, a dQ stage over queries and a dK/dV stage over key/value rows
// (section "Ecosystem survey"), recomputes the probabilities from the saved
// log-sum-exp (section "Attention kernel design"), and obtains the transposed
// score matrices S^T = K Q^T and dP^T = V dO^T by exchanging operand roles
// rather than moving data (same section).  Here:
//
//   attn_bwd_preprocess  D[i] = sum_k dO[i][k] O[i][k] (fp32), -LSE[i] * log2(e), both
//                        padded per head to a whole number of 128-row tiles (D = 0,
//                        -LSE = -inf past T, so those queries get P ~ 0), and the fp32
//                        dQ accumulator cleared.  Memory-bound.
//   attn_bwd_dkdv        persistent CTAs (one per SM) walking (head, 128-key tile j)
//                        items heaviest first; per item, a loop over the query tiles i
//                        that see the key tile (i >= j under the causal mask):
//                          S^T  = K_j Q_i^T           (tcgen05, TMEM)
//                          dP^T = V_j dO_i^T          (tcgen05, TMEM)
//                          P^T  = exp2(S^T*scale*log2e - LSE_i*log2e)   (threads)
//                          dS^T = P^T o (dP^T - D_i)                     (threads)
//                          dV  += P^T dO_i ;  dK += dS^T Q_i             (tcgen05, TMEM)
//                          dQ_i = dS K_j  (tcgen05 with dS^T read MN-major), then
//                                 scale * dQ_i staged in shared memory and added to
//                                 the fp32 accumulator by TMA reduce-add.
//                        The dQ stage of the paper is fused here: its partial sums
//                        come out of the same recomputation, and reductions in L2
//                        replace the paper's second pass over the scores.  The steps
//                        of consecutive items form one pipeline: the next item's first
//                        products are issued while this item's dK/dV leave TMEM.
//   attn_bwd_dq_convert  dQ = bf16(accumulator).
//
// dkdv warp roles (512 threads, four warpgroups; setmaxnreg moves registers between
// them):
//   warps 0..3   dQ drain and epilogue: warp w owns TMEM lanes 32w.. (query rows of
//                dQ_i, key rows of dK/dV) and all d columns; it moves dQ_i out of
//                tensor memory into fp32 staging and TMA reduce-adds it into the
//                accumulator, and at the end of an item stores dK and dV, off the
//                compute warps' path.
//   warps 4..11  compute: warp w owns TMEM lanes 32*(w%4).. (key rows of the tile) and
//                half h = (w-4)/4 of the 128 query columns.  Each thread forms its 64
//                P^T values and writes them bf16 into tensor memory (the A operand of
//                dV), then its 64 dS^T values into shared memory (the A operand of
//                dK, and the MN-major A operand of dQ).
//   warp 12      producer (one thread): K_j, V_j per item; Q_i, dO_i by TMA into
//                staged rings; the LSE_i and D_i vectors (128 floats each) by 1-D bulk
//                copies from the padded row statistics, counted on Q_i's barrier.
//   warp 13      MMA issuer (converged warp, one elected lane issues); allocates
//                tensor memory.
//   warps 14,15  idle (they complete the control warpgroup for setmaxnreg).
// Tensor memory: dV [0,d) | dK [d,2d) | S^T [2d,2d+128) | dP^T [2d+128,2d+256) |
//   dQ_i [2d+256, 3d+256) and P^T as bf16 pairs [3d+256, 3d+320) for d = 64; for
//   d = 128 (and precise mode) P^T is written over the S^T columns and dQ_i reuses
//   the dP^T columns once dS^T has been formed (512 columns hold no more).
#include "forge_internal.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

// Which pairs of P^T's exponentials go to the FMA-pipe polynomial (exp2_poly2)
// instead of the MUFU unit: 1 of every 4.  Precise mode keeps all on the MUFU unit.
__device__ __forceinline__ constexpr bool use_poly_pair(int e) { return (e & 3) == 3; }

constexpr int kBwdThreads = 512;
// registers per thread at launch: __launch_bounds__(512, 1) gives each thread 128
constexpr uint32_t kLaunchRegs = 65536 / kBwdThreads;

// Moves this warpgroup's register budget to N: setmaxnreg.inc above the launch
// count, .dec below it (a .dec to a larger count, or an .inc to a smaller one, is
// not a valid instruction).
template <uint32_t N>
__device__ __forceinline__ void set_warpgroup_regs() {
    static_assert(N % 8 == 0 && N >= 24 && N <= 256, "setmaxnreg range");
    if constexpr (N > kLaunchRegs) regs_inc<N>();
    else if constexpr (N < kLaunchRegs) regs_dec<N>();
}
constexpr int kComputeWarps = 8;
constexpr int kDrainWarps = 4;
constexpr uint32_t kWarpCompute0 = 4, kWarpProducer = 12, kWarpMma = 13;
constexpr float kLog2e = 1.4426950408889634f;

enum : uint32_t {
    kSiteKV = 1, kSiteQFull, kSiteDOFull, kSiteQEmpty, kSiteDOEmpty, kSiteSFull,
    kSiteSFree, kSiteDPFull, kSitePFull, kSitePFree, kSiteDSFull, kSiteDSFree, kSiteDQFull,
    kSiteDQFree, kSiteAccDone, kSiteAlign, kSiteStageFree, kSiteStageFull, kSiteStageDone, kSiteKVEmpty,
    kSiteAccFree
};

template <int D, bool PRECISE, bool F16>
struct BwdCfg {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kTile * 128;        // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    // dQ_n leaves tensor memory through 128-byte-swizzled fp32 staging in shared
    // memory, 32-column slices at a time, and a TMA reduce-add.  Default mode: a
    // staging buffer of its own (two slices; two rounds per step at d = 128).
    // Precise mode has no room for it.  At d = 128 it stages dQ_n in the shared
    // memory of Q_n, dead once dK_n (issued before dQ_n) has read it: two rounds of
    // two slices, both loaded from tensor memory before the first round's reduce is
    // waited for, and Q_n's stage goes back to the producer (a second arrival on its
    // empty barrier) once the reduces have read it.  At d = 64 it stages through the
    // dS^T buffer, which dQ_n's products have finished reading once dQ_n is complete
    // (the compute warps then wait for the drain before writing the next dS^T).
    static constexpr bool kStageOwn = !PRECISE;
    static constexpr bool kStageInQ = PRECISE && D == 128;
    // P^T goes back into tensor memory (bf16 pairs) as the A operand of dV: into
    // columns of its own where 64 are left (d = 64 default), otherwise over the S^T
    // columns it was computed from (each 64-query half into the first 32 (hi) and
    // last 32 (lo, precise mode) of its own 64 columns), so the next S^T waits for dV.
    static constexpr bool kPAliasS = !(D == 64 && !PRECISE);
    static constexpr int kStagesQ = (D == 64 && !PRECISE) ? 3 : 2;
    // d = 128 holds one dO stage: dO_{n+1} has from dV_n to dP_{n+1} (issued after
    // dQ_n is drained) to arrive.
    static constexpr int kStagesDO = D == 128 ? 1 : 2;
    // dS^T: [128 keys][128 queries] bf16 = two 64-query chunks; in precise mode a hi
    // buffer followed by a lo buffer.
    static constexpr int kScoreBytes = 2 * kChunkBytes;
    static constexpr int kSplit = PRECISE ? 2 : 1;
    // With d = 64 dQ_i has tensor-memory columns of its own.
    static constexpr bool kSeparateDQ = (D == 64);
    static constexpr int kDQStageBytes = kTile * 32 * 4;  // one slice: [128 rows][32 fp32]
    static constexpr int kStageSlicesDS = kSplit * kScoreBytes / kDQStageBytes;
    static constexpr int kStageSlices =  // per round
        (kStageOwn || kStageInQ) ? 2 : (kStageSlicesDS < D / 32 ? kStageSlicesDS : D / 32);
    static constexpr int kDrainRounds = (D / 32) / kStageSlices;
    static_assert(kDrainRounds * kStageSlices == D / 32, "dQ staging slices");
    // slices moved out of tensor memory per load group: the last group's load frees
    // the columns, before any wait for the staging
    static constexpr int kLoadGroup = (kStageOwn || kStageInQ) ? 2 : 1;
    // K/V buffers.  One: the next item's K_j, V_j load after this item's last dQ,
    // and its first S^T waits for them.  (Two buffers at d = 64 measured slower, both
    // with the next item's first S^T issued at the top of the item's last step, ahead
    // of that step's dV, dQ and dK, and with it kept after them.)
    static constexpr int kKVBufs = 1;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kKVBufs * kTileBytes;
    static constexpr int kOffQ = kOffV + kKVBufs * kTileBytes;
    static constexpr int kOffDO = kOffQ + kStagesQ * kTileBytes;
    static constexpr int kOffDS = kOffDO + kStagesDO * kTileBytes;
    static constexpr int kOffDQS = kOffDS + kSplit * kScoreBytes;
    static constexpr int kOffStage = kStageOwn ? kOffDQS : kOffDS;
    static constexpr int kOffLse = kOffDQS + (kStageOwn ? kStageSlices * kDQStageBytes : 0);
    static constexpr int kOffDelta = kOffLse + kStagesQ * kTile * 4;
    static constexpr int kOffBar = kOffDelta + kStagesQ * kTile * 4;
    static constexpr int kSmemBytes = kOffBar + 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static constexpr uint32_t kColDV = 0, kColDK = D, kColS = 2 * D, kColDP = 2 * D + 128;
    static constexpr uint32_t kColDQ = kSeparateDQ ? 2 * D + 256 : kColDP;
    static constexpr uint32_t kColP = kPAliasS ? kColS : 3 * D + 256;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kColDQ + D <= kTmemCols, "tensor memory budget");
    static_assert(kPAliasS || (kSeparateDQ && kColP + 64 <= kTmemCols), "tensor memory budget");
    // tensor-memory column of P^T's 16-query group kk (0..7), hi part
    static __device__ __forceinline__ constexpr uint32_t p_col(int kk) {
        return kPAliasS ? kColS + (kk >> 2) * 64 + (kk & 3) * 8 : kColP + kk * 8;
    }
    // registers per thread after setmaxnreg (the launch gives 512 x 128): the precise
    // d = 128 MMA issuer needs more, paid for by its compute warps
    static constexpr uint32_t kRegsDrain = 96;
    static constexpr uint32_t kRegsCompute = (D == 128 && PRECISE) ? 160 : 168;
    static constexpr uint32_t kRegsCtl = (D == 128 && PRECISE) ? 96 : 80;
    static_assert(128 * kRegsDrain + 256 * kRegsCompute + 128 * kRegsCtl <=
                      kBwdThreads * kLaunchRegs,
                  "register split exceeds the block's launch allocation");
    // every operand bf16, or every operand fp16 (F16)
    static constexpr uint32_t kIdescScore = idesc_f16kind_f32(128, 128, false, false, F16);
    static constexpr uint32_t kIdescGrad = idesc_f16kind_f32(128, D, false, true, F16);  // dV, dK
    static constexpr uint32_t kIdescDQ = idesc_f16kind_f32(128, D, true, true, F16);     // dQ
};

struct BwdBarriers {
    uint64_t kv_full[2], kv_empty[2];  // K_j, V_j per item (one or two buffers)
    uint64_t q_full[3];
    uint64_t do_full[2];
    uint64_t q_empty[3];
    uint64_t do_empty[2];
    uint64_t s_full, s_free, dp_full, p_full, p_free, ds_full, ds_free, dq_full, dq_free;
    uint64_t stage_free, stage_full;  // dQ staging in shared memory (drain warps)
    uint64_t stage_done;              // staging in the dS^T buffer is over (per step)
    uint64_t acc_done, acc_free;  // an item's dK, dV complete / read out of tensor memory
    uint64_t mma_final;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(BwdBarriers) <= 256, "barrier block");

// Eight fp32 values as bf16 (fp16 with F16) into a 16-byte chunk at base + off; in
// precise mode (bf16 only) the remainders x - bf16(x), rounded to bf16, go to the same
// place in the lo buffer (base + lo_stride + off).
template <bool PRECISE, bool F16>
__device__ __forceinline__ void store_split8(uint8_t* base, int lo_stride, uint32_t off,
                                             const float* x) {
    static_assert(!(PRECISE && F16), "the hi + lo split is a bf16-operand mode");
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = pack16x2<F16>(x[2 * e], x[2 * e + 1]);
    *reinterpret_cast<uint4*>(base + off) = make_uint4(h[0], h[1], h[2], h[3]);
    if (PRECISE) {
        uint32_t l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            l[e] = pack_bf16x2(x[2 * e] - bf16_lo_to_float(h[e]),
                               x[2 * e + 1] - bf16_hi_to_float(h[e]));
        *reinterpret_cast<uint4*>(base + lo_stride + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t site,
                                          volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, site, abort));
}

template <int D, bool PRECISE, bool F16>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_do,
                         const __grid_constant__ CUtensorMap tmap_dq,
                         const float* __restrict__ rowstats, float* __restrict__ dq_accum,
                         void* __restrict__ dk_out, void* __restrict__ dv_out, int T, int BH,
                         int n_kvtiles, int n_items, float scale, float scale_log2, int causal,
                         int grad_f32) {
    using C = BwdCfg<D, PRECISE, F16>;
    extern __shared__ __align__(1024) uint8_t smem[];
    BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::kOffBar);
    volatile int* abort = &bars->abort;
    float* s_lse = reinterpret_cast<float*>(smem + C::kOffLse);
    float* s_delta = reinterpret_cast<float*>(smem + C::kOffDelta);

    const int n_qtiles = n_kvtiles;
    const int t_pad = n_qtiles * kTile;  // row-statistics stride per head
    const int n_ctas = (int)gridDim.x;
    // Persistent CTAs.  The CTA's r-th work item is a (head, key tile) pair; items are
    // numbered heaviest first (key tile 0 sees the most query tiles) and dealt in a
    // zigzag over the CTAs, which keeps every CTA's total close to the mean.  Every
    // role walks the same item sequence; the per-step barriers count steps across
    // items, so one item's last steps overlap the next item's first.
    auto item_of = [&](int r, int& bh_out, int& kt_out) -> bool {
        const int k = r * n_ctas + ((r & 1) ? (n_ctas - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        if (k >= n_items) return false;
        kt_out = k / BH;
        bh_out = k - kt_out * BH;
        return true;
    };
    auto first_qtile = [&](int kt_) { return causal ? kt_ : 0; };
    const uint32_t warp = warp_id();
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->kv_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        mbar_init(&bars->acc_free, kDrainWarps);
        for (int s = 0; s < 3; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], C::kStageInQ ? 2 : 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->do_full[s], 1);
            mbar_init(&bars->do_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, kComputeWarps);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_full, kComputeWarps);
        mbar_init(&bars->p_free, 1);
        mbar_init(&bars->ds_full, kComputeWarps);
        mbar_init(&bars->ds_free, 1);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_free, kDrainWarps);
        mbar_init(&bars->stage_free, 1);
        mbar_init(&bars->stage_full, kDrainWarps);
        mbar_init(&bars->stage_done, 1);
        mbar_init(&bars->acc_done, 1);
        mbar_init(&bars->mma_final, 1);
        bars->abort = (smem_u32(smem) & 1023u) ? 1 : 0;
        if (bars->abort) record_timeout(kSiteAlign);
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&bars->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    // the prologue above overlaps the previous kernel's tail (the pre-pass writes the
    // row statistics and clears the accumulator); global memory is touched only now
    grid_dependency_wait();
    allow_dependents_launch();

    if (warp < kWarpCompute0) {
        // ---------------------------------------------------------- dQ drain
        set_warpgroup_regs<C::kRegsDrain>();
        const uint32_t row = (warp << 5) + lane;  // query row of the tile
        const uint32_t lane_off = (warp << 5) << 16;
        const bool leader = warp == 0 && lane == 0;
        int n_sfree = 0, n_sfull = 0;  // completed phases of the staging barriers
        int g = 0;                     // steps drained so far (all items)
        bool run = true;
        int bh, kt;
        for (int item = 0; run && item_of(item, bh, kt); ++item) {
        for (int i = first_qtile(kt); i < n_qtiles; ++i, ++g) {
            if (!warp_wait(&bars->dq_full, g & 1, kSiteDQFull, abort)) { run = false; break; }
            tc_fence_after();
            bool fine = true;
            // dQ staging: a buffer of its own, Q_i's stage, or the dS^T buffer
            const int stage_off =
                C::kStageInQ ? C::kOffQ + (g % C::kStagesQ) * C::kTileBytes : C::kOffStage;
            constexpr int kG = C::kLoadGroup;
            constexpr int kGroups = D / 32 / kG;
            constexpr int kGroupsPerRound = C::kStageSlices / kG;
#pragma unroll
            for (int pr = 0; pr < kGroups; ++pr) {
                const int rd = pr / kGroupsPerRound, sl0 = kG * (pr % kGroupsPerRound);
                uint32_t r[32 * kG];
#pragma unroll
                for (int h = 0; h < kG; ++h)
                    tmem_ld32(tmem + lane_off + C::kColDQ + 32 * (kG * pr + h), r + 32 * h);
                tmem_wait_ld();
                if (pr == kGroups - 1) {  // every column of dQ_n has been read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->dq_free);
                }
                // a round's staging must have been read by the previous round's reduce
                // (the dS^T buffer is free at the first round of a step by construction);
                // bounded mbarrier waits rather than bar.sync, so an abort strands no warp
                if (sl0 == 0 && (C::kStageOwn || rd > 0)) {
                    if (leader) {
                        tma_store_wait_all_read();
                        mbar_arrive(&bars->stage_free);
                    }
                    if (!warp_wait(&bars->stage_free, n_sfree & 1, kSiteStageFree, abort)) {
                        fine = false;
                        break;
                    }
                    ++n_sfree;
                }
#pragma unroll
                for (int h = 0; h < kG; ++h) {
                    uint8_t* stage = smem + stage_off + (sl0 + h) * C::kDQStageBytes;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        *reinterpret_cast<float4*>(stage + sw128_offset(row, ch)) = make_float4(
                            __uint_as_float(r[32 * h + 4 * ch]) * scale,
                            __uint_as_float(r[32 * h + 4 * ch + 1]) * scale,
                            __uint_as_float(r[32 * h + 4 * ch + 2]) * scale,
                            __uint_as_float(r[32 * h + 4 * ch + 3]) * scale);
                }
                if (sl0 + kG == C::kStageSlices) {  // the round's slices are staged
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->stage_full);
                    if (warp == 0) {
                        if (!warp_wait(&bars->stage_full, n_sfull & 1, kSiteStageFull, abort)) {
                            fine = false;
                            break;
                        }
                        if (leader) {
#pragma unroll
                            for (int sl = 0; sl < C::kStageSlices; ++sl)
                                tma_reduce_add_3d(&tmap_dq,
                                                  smem + stage_off + sl * C::kDQStageBytes,
                                                  (rd * C::kStageSlices + sl) * 32, i * kTile, bh);
                            tma_store_commit();
                        }
                    }
                    ++n_sfull;
                }
            }
            if (!fine) { run = false; break; }
            if constexpr (!C::kStageOwn) {
                // the dS^T buffer goes back to the compute warps, or Q_i's stage to the
                // producer, once the reduces have read it
                if (leader) {
                    tma_store_wait_all_read();
                    mbar_arrive(C::kStageInQ ? &bars->q_empty[g % C::kStagesQ]
                                             : &bars->stage_done);
                }
            }
        }
        if (!run) break;
        // ------------------------------------------------ dK / dV epilogue
        // the item's dV, dK leave tensor memory here, while the compute warps go on
        // with the next item; its first dV, dK products wait for acc_free
        if (!warp_wait(&bars->acc_done, item & 1, kSiteAccDone, abort)) break;
        tc_fence_after();
        {
            const int key = kt * kTile + (int)row;
            const size_t base = ((size_t)bh * T + key) * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = which == 0 ? C::kColDV : C::kColDK;
                const float mul = which == 0 ? 1.f : scale;
                void* out = which == 0 ? dv_out : dk_out;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + col + c * 32, r);
                    tmem_wait_ld();
                    if (which == 1 && c == D / 32 - 1) {
                        // every column of dV and dK has been read
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars->acc_free);
                    }
                    if (key < T) {
                        if (grad_f32) {
                            float4* o =
                                reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + base + c * 32);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                o[e] = make_float4(__uint_as_float(r[4 * e]) * mul,
                                                   __uint_as_float(r[4 * e + 1]) * mul,
                                                   __uint_as_float(r[4 * e + 2]) * mul,
                                                   __uint_as_float(r[4 * e + 3]) * mul);
                        } else {
                            uint4* o = reinterpret_cast<uint4*>(
                                reinterpret_cast<uint16_t*>(out) + base + c * 32);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                o[e] = make_uint4(
                                    pack16x2<F16>(__uint_as_float(r[8 * e]) * mul,
                                                  __uint_as_float(r[8 * e + 1]) * mul),
                                    pack16x2<F16>(__uint_as_float(r[8 * e + 2]) * mul,
                                                  __uint_as_float(r[8 * e + 3]) * mul),
                                    pack16x2<F16>(__uint_as_float(r[8 * e + 4]) * mul,
                                                  __uint_as_float(r[8 * e + 5]) * mul),
                                    pack16x2<F16>(__uint_as_float(r[8 * e + 6]) * mul,
                                                  __uint_as_float(r[8 * e + 7]) * mul));
                        }
                    }
                }
            }
        }
        }  // items
        // the reduces must have read their staging before the CTA's shared memory goes;
        // their global writes complete before the kernel does
        if (leader) tma_store_wait_all_read();
    } else if (warp < kWarpProducer) {
        // ----------------------------------------------------------- compute
        set_warpgroup_regs<C::kRegsCompute>();
        const uint32_t quarter = warp & 3;
        const uint32_t half = (warp - kWarpCompute0) >> 2;  // which 64 query columns
        const uint32_t row = (quarter << 5) + lane;          // key row
        const uint32_t lane_off = (quarter << 5) << 16;
        uint8_t* ds_smem = smem + C::kOffDS + half * C::kChunkBytes;
        const int c0 = half * 64;                            // first query column owned
        bool ok = !*abort;
        int g = 0;  // steps so far (all items)
        int bh, kt;
        for (int item = 0; ok && item_of(item, bh, kt); ++item) {
        for (int i = first_qtile(kt); ok && i < n_qtiles; ++i, ++g) {
            const int sq = g % C::kStagesQ;
            const bool diag = causal && (i == kt);
            // ---- P^T for 64 query columns
            if (!warp_wait(&bars->s_full, g & 1, kSiteSFull, abort)) { ok = false; break; }
            tc_fence_after();
            uint32_t sraw[64];
            tmem_ld32(tmem + lane_off + C::kColS + c0, sraw);
            tmem_ld32(tmem + lane_off + C::kColS + c0 + 32, sraw + 32);
            tmem_wait_ld();
            if constexpr (!C::kPAliasS) {
                // S^T is in registers: its columns may take the next product
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->s_free);
            }
            // LSE_i and D_i arrived with Q_i
            if (!warp_wait(&bars->q_full[sq], (g / C::kStagesQ) & 1, kSiteQFull, abort)) {
                ok = false;
                break;
            }
            // P^T = exp2(S^T * scale * log2(e) - LSE * log2(e)), two queries at a time
            const float4* nlse4 = reinterpret_cast<const float4*>(s_lse + sq * kTile + c0);
            const float2 sl2 = make_float2(scale_log2, scale_log2);
            float p[64];
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                const float4 l = nlse4[c4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = 4 * c4 + 2 * h;
                    const float2 x = ffma2(
                        make_float2(__uint_as_float(sraw[c]), __uint_as_float(sraw[c + 1])), sl2,
                        h == 0 ? make_float2(l.x, l.y) : make_float2(l.z, l.w));
                    float2 e2;
                    if (!PRECISE && use_poly_pair(c >> 1)) {
                        e2 = exp2_poly2(x);
                    } else {
                        e2.x = ex2_approx(x.x);
                        e2.y = ex2_approx(x.y);
                    }
                    p[c] = e2.x;
                    p[c + 1] = e2.y;
                }
            }
            if (diag) {  // a query that precedes the key row
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c0 + c < (int)row) p[c] = 0.f;
            }
            // P^T into tensor memory.  Own columns: they must no longer be read by the
            // previous iteration's dV.  Over S^T: this thread has read its S^T columns,
            // and S_n was issued after dV_{n-1}.
            if (!C::kPAliasS && g > 0 &&
                !warp_wait(&bars->p_free, (g - 1) & 1, kSitePFree, abort)) {
                ok = false;
                break;
            }
            {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack16x2<F16>(p[2 * e], p[2 * e + 1]);
                const uint32_t tp = tmem + lane_off + C::p_col(4 * (int)half);
                tc_fence_after();
                if constexpr (PRECISE) {
                    uint32_t pl[32];  // remainders p - bf16(p), the lo terms
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        pl[e] = pack_bf16x2(p[2 * e] - bf16_lo_to_float(pk[e]),
                                            p[2 * e + 1] - bf16_hi_to_float(pk[e]));
                    tmem_st32(tp, pk);
                    tmem_st32(tp + 32, pl);
                } else {
                    tmem_st32(tp, pk);
                }
                tmem_wait_st();
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full);

            // ---- dS^T = P^T o (dP^T - D), 32 queries at a time
            if (!warp_wait(&bars->dp_full, g & 1, kSiteDPFull, abort)) { ok = false; break; }
            // dS^T buffer: free once dK and dQ of the previous iteration have read it
            // and, where it stages dQ, once the drain is done with it
            constexpr bool kStaged = !C::kStageOwn && !C::kStageInQ;
            if (g > 0 && !warp_wait(kStaged ? &bars->stage_done : &bars->ds_free, (g - 1) & 1,
                                    kStaged ? kSiteStageDone : kSiteDSFree, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float4* d4 = reinterpret_cast<const float4*>(s_delta + sq * kTile + c0);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t dp[32];
                tmem_ld32(tmem + lane_off + C::kColDP + c0 + c * 32, dp);
                tmem_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {  // 4 chunks of 8 queries
                    const float4 da = d4[c * 8 + ch * 2], db = d4[c * 8 + ch * 2 + 1];
                    const float2 dv2[4] = {make_float2(da.x, da.y), make_float2(da.z, da.w),
                                           make_float2(db.x, db.y), make_float2(db.z, db.w)};
                    float ds[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int qc = c * 32 + ch * 8 + 2 * e;
                        const float2 dsv = fmul2(
                            make_float2(p[qc], p[qc + 1]),
                            fsub2(make_float2(__uint_as_float(dp[ch * 8 + 2 * e]),
                                              __uint_as_float(dp[ch * 8 + 2 * e + 1])),
                                  dv2[e]));
                        ds[2 * e] = dsv.x;
                        ds[2 * e + 1] = dsv.y;
                    }
                    store_split8<PRECISE, F16>(ds_smem, C::kScoreBytes,
                                               sw128_offset(row, c * 4 + ch), ds);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ds_full);
        }

        }  // items
    } else {
        set_warpgroup_regs<C::kRegsCtl>();
        if (warp == kWarpProducer && lane == 0) {
            // -------------------------------------------------------- producer
            int last_q[3] = {-1, -1, -1}, last_do[2] = {-1, -1}, last_kv[2] = {-1, -1};
            if (!*abort) {
                tma_prefetch_desc(&tmap_q);
                tma_prefetch_desc(&tmap_k);
                tma_prefetch_desc(&tmap_v);
                tma_prefetch_desc(&tmap_do);
                int g = 0;  // steps so far (all items)
                bool run = true;
                int bh, kt;
                for (int item = 0; run && item_of(item, bh, kt); ++item) {
                    // K_j, V_j into the item's buffer once the item before last is done
                    // with it
                    const int kb = item % C::kKVBufs, ukv = item / C::kKVBufs;
                    if (ukv > 0 &&
                        !mbar_wait(&bars->kv_empty[kb], (ukv - 1) & 1, kSiteKVEmpty, abort))
                        break;
                    mbar_arrive_expect_tx(&bars->kv_full[kb], 2 * C::kTileBytes);
                    for (int c = 0; c < C::kChunks; ++c) {
                        tma_load_3d(smem + C::kOffK + kb * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_k, &bars->kv_full[kb], 64 * c, kt * kTile, bh);
                        tma_load_3d(smem + C::kOffV + kb * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_v, &bars->kv_full[kb], 64 * c, kt * kTile, bh);
                    }
                    last_kv[kb] = ukv;
                    const float* lse2_head = rowstats + (size_t)bh * t_pad;
                    const float* delta_head = rowstats + (size_t)BH * t_pad + (size_t)bh * t_pad;
                    for (int i = first_qtile(kt); i < n_qtiles; ++i, ++g) {
                        // Q_i with the LSE and D vectors of its query tile
                        const int sq = g % C::kStagesQ, uq = g / C::kStagesQ;
                        if (uq > 0 &&
                            !mbar_wait(&bars->q_empty[sq], (uq - 1) & 1, kSiteQEmpty, abort)) {
                            run = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->q_full[sq], C::kTileBytes + 2 * kTile * 4);
                        for (int c = 0; c < C::kChunks; ++c)
                            tma_load_3d(smem + C::kOffQ + sq * C::kTileBytes + c * C::kChunkBytes,
                                        &tmap_q, &bars->q_full[sq], 64 * c, i * kTile, bh);
                        bulk_load(s_lse + sq * kTile, lse2_head + i * kTile, kTile * 4,
                                  &bars->q_full[sq]);
                        bulk_load(s_delta + sq * kTile, delta_head + i * kTile, kTile * 4,
                                  &bars->q_full[sq]);
                        last_q[sq] = uq;
                        // dO_i
                        const int sd = g % C::kStagesDO, ud = g / C::kStagesDO;
                        if (ud > 0 &&
                            !mbar_wait(&bars->do_empty[sd], (ud - 1) & 1, kSiteDOEmpty, abort)) {
                            run = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars->do_full[sd], C::kTileBytes);
                        for (int c = 0; c < C::kChunks; ++c)
                            tma_load_3d(smem + C::kOffDO + sd * C::kTileBytes + c * C::kChunkBytes,
                                        &tmap_do, &bars->do_full[sd], 64 * c, i * kTile, bh);
                        last_do[sd] = ud;
                    }
                }
            }
            if (*abort) {
                // let copies already issued land before the CTA's memory is released
                for (int s = 0; s < 2; ++s)
                    if (last_kv[s] >= 0) mbar_wait_drain(&bars->kv_full[s], last_kv[s] & 1);
                for (int s = 0; s < 3; ++s)
                    if (last_q[s] >= 0) mbar_wait_drain(&bars->q_full[s], last_q[s] & 1);
                for (int s = 0; s < 2; ++s)
                    if (last_do[s] >= 0) mbar_wait_drain(&bars->do_full[s], last_do[s] & 1);
            }
        } else if (warp == kWarpMma) {
            // ------------------------------------------------------ MMA issuer
            // The whole warp runs this loop; one elected lane issues each MMA.
            const uint32_t tS = tmem + C::kColS;
            const uint32_t tDP = tmem + C::kColDP;
            const uint32_t tDQ = tmem + C::kColDQ;
            const uint32_t tDV = tmem + C::kColDV;
            const uint32_t tDK = tmem + C::kColDK;
            auto k_buf = [&](int b) { return smem_u32(smem + C::kOffK + b * C::kTileBytes); };
            auto v_buf = [&](int b) { return smem_u32(smem + C::kOffV + b * C::kTileBytes); };
            const uint32_t ds_addr = smem_u32(smem + C::kOffDS);
            bool ok = __all_sync(0xffffffffu, !*abort);

            // S^T = K Q^T  or  dP^T = V dO^T: M = 128 keys, N = 128 queries, K = d
            auto score_mma = [&](uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    mma_ss_warp(d_tmem, sdesc_sw128(a_addr + off, 16, 1024),
                                sdesc_sw128(b_addr + off, 16, 1024), C::kIdescScore,
                                kk > 0 ? 1u : 0u);
                }
            };
            // dK += dS^T Q: M = 128 keys, N = d, K = 128 queries
            auto grad_mma = [&](uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    mma_ss_warp(d_tmem, sdesc_sw128(a_addr + aoff, 16, 1024),
                                sdesc_sw128(b_addr + kk * 2048, C::kChunkBytes, 1024),
                                C::kIdescGrad, (acc || kk > 0) ? 1u : 0u);
                }
            };
            // dV += P^T dO with P^T in tensor memory (16 queries = 8 columns per step;
            // precise mode adds the lo terms, 32 columns further)
            auto dv_mma = [&](uint32_t b_addr, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t bdesc = sdesc_sw128(b_addr + kk * 2048, C::kChunkBytes, 1024);
                    mma_ts_warp(tDV, tmem + C::p_col(kk), bdesc, C::kIdescGrad,
                                (acc || kk > 0) ? 1u : 0u);
                    if (PRECISE)
                        mma_ts_warp(tDV, tmem + C::p_col(kk) + 32, bdesc, C::kIdescGrad, 1u);
                }
            };
            // dQ_i = dS K: M = 128 queries (dS^T read MN-major), N = d, K = 128 keys
            auto dq_mma = [&](uint32_t a_addr, uint32_t k_addr, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_ss_warp(tDQ, sdesc_sw128(a_addr + kk * 2048, C::kChunkBytes, 1024),
                                sdesc_sw128(k_addr + kk * 2048, C::kChunkBytes, 1024),
                                C::kIdescDQ, (acc || kk > 0) ? 1u : 0u);
            };
            auto q_stage = [&](int g) {
                return smem_u32(smem + C::kOffQ + (g % C::kStagesQ) * C::kTileBytes);
            };
            auto do_stage = [&](int g) {
                return smem_u32(smem + C::kOffDO + (g % C::kStagesDO) * C::kTileBytes);
            };

            int bh, kt;
            bool have = ok && item_of(0, bh, kt);
            // prologue: S and dP^T of the first step
            if (have) {
                ok = warp_wait(&bars->kv_full[0], 0, kSiteKV, abort) &&
                     warp_wait(&bars->q_full[0], 0, kSiteQFull, abort);
                if (ok) {
                    tc_fence_after();
                    score_mma(tS, k_buf(0), q_stage(0));
                    mma_commit_warp(&bars->s_full);
                }
                if (ok) ok = warp_wait(&bars->do_full[0], 0, kSiteDOFull, abort);
                if (ok) {
                    tc_fence_after();
                    score_mma(tDP, v_buf(0), do_stage(0));
                    mma_commit_warp(&bars->dp_full);
                }
            }
            int g = 0;  // steps so far (all items)
            for (int item = 0; ok && have; ++item) {
                const int kb = item % C::kKVBufs, nkb = (item + 1) % C::kKVBufs;
                int nbh, nkt;
                const bool have_next = item_of(item + 1, nbh, nkt);
                const int n_it = n_qtiles - first_qtile(kt);
                for (int n = 0; ok && n < n_it; ++n, ++g) {
                    const bool last = n + 1 == n_it;
                    const bool next_step = !last || have_next;  // a step g + 1 exists
                    const int kb1 = last ? nkb : kb;            // its K/V buffer
                    // with one K/V buffer the next item's K/V arrive only after this
                    // item's last dQ has released them: its first S is issued after that.
                    // With dQ staged in Q's shared memory every S_{g+1} goes after dK_g and
                    // dQ_g: it may wait for Q_{g+1}, whose stage the reduces of dQ_{g-1}
                    // release, and dK_g, dQ_g must not queue behind that wait.
                    const bool s_late = C::kStageInQ || (last && C::kKVBufs == 1);
                    // S_{g+1}; a new item's first also waits for that item's K/V
                    auto issue_s = [&]() -> bool {
                        if (last && !warp_wait(&bars->kv_full[nkb], ((item + 1) / C::kKVBufs) & 1,
                                               kSiteKV, abort))
                            return false;
                        if (!warp_wait(&bars->q_full[(g + 1) % C::kStagesQ],
                                       ((g + 1) / C::kStagesQ) & 1, kSiteQFull, abort))
                            return false;
                        tc_fence_after();
                        score_mma(tS, k_buf(kb1), q_stage(g + 1));
                        mma_commit_warp(&bars->s_full);
                        return true;
                    };
                    // the S^T columns are free for S_{g+1}: own P^T columns, once the
                    // compute warps hold S_g in registers; P^T over S^T, once dV_g (which
                    // reads P^T there) has completed (its commit, not issue order)
                    auto s_cols_free = [&]() -> bool {
                        return C::kPAliasS ? warp_wait(&bars->p_free, g & 1, kSitePFree, abort)
                                           : warp_wait(&bars->s_free, g & 1, kSiteSFree, abort);
                    };
                    if (!C::kPAliasS && next_step && !s_late) {
                        if (!s_cols_free() || !issue_s()) { ok = false; break; }
                    }
                    // dV += P^T dO_g; an item's first step overwrites dV (and dK), so it
                    // waits until the previous item's epilogue has read them
                    if (!warp_wait(&bars->p_full, g & 1, kSitePFull, abort)) { ok = false; break; }
                    if (n == 0 && item > 0 &&
                        !warp_wait(&bars->acc_free, (item - 1) & 1, kSiteAccFree, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    dv_mma(do_stage(g), n > 0);
                    mma_commit_warp(&bars->p_free);
                    mma_commit_warp(&bars->do_empty[g % C::kStagesDO]);  // dP_g, dV_g read it
                    if (C::kPAliasS && next_step && !s_late) {
                        if (!s_cols_free() || !issue_s()) { ok = false; break; }
                    }
                    // dQ_g = dS K and dK += dS^T Q_g.  With a staging buffer of its own, dQ_g
                    // goes first, so that its drain (and, with shared columns, the next
                    // dP^T) starts while dK_g runs.  Staged through the dS^T buffer, the
                    // drain may start only once dK_g has read dS^T too: dK_g goes first.
                    // Separate dQ columns are free once dQ_{g-1} is drained; shared with
                    // dP^T, once dP_g has been read (ds_full).
                    constexpr bool kDQFirst = C::kStageOwn;
                    if (!warp_wait(&bars->ds_full, g & 1, kSiteDSFull, abort)) { ok = false; break; }
                    tc_fence_after();
                    if constexpr (!kDQFirst) {
                        grad_mma(tDK, ds_addr, q_stage(g), n > 0);
                        if (PRECISE) grad_mma(tDK, ds_addr + C::kScoreBytes, q_stage(g), true);
                    }
                    if (C::kSeparateDQ && g > 0 &&
                        !warp_wait(&bars->dq_free, (g - 1) & 1, kSiteDQFree, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    dq_mma(ds_addr, k_buf(kb), false);
                    if (PRECISE) dq_mma(ds_addr + C::kScoreBytes, k_buf(kb), true);
                    mma_commit_warp(&bars->dq_full);
                    if constexpr (kDQFirst) {
                        grad_mma(tDK, ds_addr, q_stage(g), n > 0);
                        if (PRECISE) grad_mma(tDK, ds_addr + C::kScoreBytes, q_stage(g), true);
                    }
                    mma_commit_warp(&bars->ds_free);
                    mma_commit_warp(&bars->q_empty[g % C::kStagesQ]);
                    if (last) {
                        mma_commit_warp(&bars->acc_done);      // the item's dV, dK are complete
                        mma_commit_warp(&bars->kv_empty[kb]);  // and its K, V read for good
                    }
                    if (s_late && next_step) {
                        if (!s_cols_free() || !issue_s()) { ok = false; break; }
                    }
                    // dP_{g+1}: its columns are free once dS_g is formed (separate dQ) or
                    // once dQ_g has left tensor memory (shared columns)
                    if (next_step) {
                        if (!C::kSeparateDQ &&
                            !warp_wait(&bars->dq_free, g & 1, kSiteDQFree, abort)) {
                            ok = false;
                            break;
                        }
                        if (!warp_wait(&bars->do_full[(g + 1) % C::kStagesDO],
                                       ((g + 1) / C::kStagesDO) & 1, kSiteDOFull, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        score_mma(tDP, v_buf(kb1), do_stage(g + 1));
                        mma_commit_warp(&bars->dp_full);
                    }
                }
                kt = nkt;
                bh = nbh;
                have = have_next;
            }
            mma_commit_warp(&bars->mma_final);
            mbar_wait_drain(&bars->mma_final, 0);
        }
    }

    // ------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Row statistics of the backward, padded per head to t_pad = 128 * ceil(T / 128) rows:
// rowstats[0][bh][t] = -LSE * log2(e) (negated: it is the addend of the exponent) and
// rowstats[1][bh][t] = D = rowsum(dO o O) (fp32; -inf and 0 past T), and the dQ
// accumulator cleared.  O is fp32, or 16-bit like dO (F16: fp16, else bf16).  A
// group of D/8 consecutive threads covers one row, 8 elements each, so every load of
// a warp is one contiguous span.
template <int D, bool O_F32, bool F16>
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(
    const void* __restrict__ o_in, const uint16_t* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ rowstats, float* __restrict__ dq_accum,
    int T, int t_pad, long long padded_rows) {
    grid_dependency_wait();
    allow_dependents_launch();
    constexpr int kGroup = D / 8;  // threads per row
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long pr = t / kGroup;  // padded row index
    const int part = (int)(t % kGroup);
    const long long bh = pr / t_pad;
    const int tr = (int)(pr % t_pad);
    const bool valid = pr < padded_rows && tr < T;
    const long long r = bh * T + tr;  // row in the [B*H][T] tensors
    float acc = 0.f;
    if (valid) {
        const uint4 b = reinterpret_cast<const uint4*>(dO + r * D)[part];
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
        float fo[8];
        if constexpr (!O_F32) {
            const uint4 a = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(o_in) +
                                                           r * D)[part];
            const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = unpack16x2<F16>(aw[h]);
                fo[2 * h] = f.x;
                fo[2 * h + 1] = f.y;
            }
        } else {
            const float4* o4 = reinterpret_cast<const float4*>(static_cast<const float*>(o_in) +
                                                               r * D);
            const float4 a0 = o4[2 * part];
            const float4 a1 = o4[2 * part + 1];
            fo[0] = a0.x; fo[1] = a0.y; fo[2] = a0.z; fo[3] = a0.w;
            fo[4] = a1.x; fo[5] = a1.y; fo[6] = a1.z; fo[7] = a1.w;
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float2 fb = unpack16x2<F16>(bw[h]);
            acc = fmaf(fo[2 * h], fb.x, acc);
            acc = fmaf(fo[2 * h + 1], fb.y, acc);
        }
        if (dq_accum) {
            float4* z = reinterpret_cast<float4*>(dq_accum + r * D) + 2 * part;
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
#pragma unroll
    for (int off = kGroup / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (pr < padded_rows && part == 0) {
        rowstats[pr] = valid ? -lse[r] * kLog2e : -INFINITY;
        rowstats[padded_rows + pr] = valid ? acc : 0.f;
    }
}

// dQ = bf16(accumulator) (fp16 with F16), 8 elements per thread.
template <bool F16>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ acc,
                                                                  uint16_t* __restrict__ dq,
                                                                  long long n8) {
    grid_dependency_wait();
    allow_dependents_launch();
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n8) return;
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    reinterpret_cast<uint4*>(dq)[t] =
        make_uint4(pack16x2<F16>(a.x, a.y), pack16x2<F16>(a.z, a.w), pack16x2<F16>(b.x, b.y),
                   pack16x2<F16>(b.z, b.w));
}

template <int D, bool PRECISE, bool F16>
cudaError_t launch_dkdv_dp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tdo, const CUtensorMap& tdq, const float* rowstats,
                           float* dq_accum, void* dk, void* dv, int BH, int T, float scale,
                           int causal, int grad_f32, cudaStream_t stream) {
    using C = BwdCfg<D, PRECISE, F16>;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e =
        set_max_dynamic_smem(attn_bwd_dkdv_kernel<D, PRECISE, F16>, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    const int n_kvtiles = (T + kTile - 1) / kTile;
    const long long items = (long long)BH * n_kvtiles;
    if (items > 0x7fffffff) return cudaErrorInvalidValue;
    const int n_items = (int)items;
    // persistent: one CTA per SM (shared memory and tensor memory allow no more)
    const int grid = n_items < sm_count() ? n_items : sm_count();
    return launch_dependent(attn_bwd_dkdv_kernel<D, PRECISE, F16>, dim3(grid), dim3(kBwdThreads),
                            C::kSmemBytes, stream, tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk,
                            dv, T, BH, n_kvtiles, n_items, scale, scale * kLog2e, causal,
                            grad_f32);
}

template <int D, bool O_F32, bool F16>
cudaError_t launch_pre(const void* o, const void* dO, const float* lse, float* rowstats,
                float* dq_accum, int BH, int T, cudaStream_t stream) {
    const int t_pad = ((T + kTile - 1) / kTile) * kTile;
    const long long padded_rows = (long long)BH * t_pad;
    const int threads = 256;
    const long long total = padded_rows * (D / 8);
    const unsigned blocks = (unsigned)((total + threads - 1) / threads);
    return launch_dependent(attn_bwd_preprocess_kernel<D, O_F32, F16>, dim3(blocks), dim3(threads),
                     0, stream, o, static_cast<const uint16_t*>(dO), lse, rowstats, dq_accum, T,
                     t_pad, padded_rows);
}

template <int D>
cudaError_t launch_pre_d(const void* o, const void* dO, const float* lse, float* rowstats,
                         float* dq_accum, int BH, int T, int o_f32, int f16, cudaStream_t stream) {
    if (o_f32) {
        if (f16) return launch_pre<D, true, true>(o, dO, lse, rowstats, dq_accum, BH, T, stream);
        return launch_pre<D, true, false>(o, dO, lse, rowstats, dq_accum, BH, T, stream);
    }
    if (f16) return launch_pre<D, false, true>(o, dO, lse, rowstats, dq_accum, BH, T, stream);
    return launch_pre<D, false, false>(o, dO, lse, rowstats, dq_accum, BH, T, stream);
}

template <int D>
cudaError_t launch_dkdv_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const float* rowstats,
                          float* dq_accum, void* dk, void* dv, int BH, int T, float scale,
                          int causal, int grad_f32, int precise, int f16, cudaStream_t stream) {
    if (f16)
        return launch_dkdv_dp<D, false, true>(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv,
                                              BH, T, scale, causal, grad_f32, stream);
    if (precise)
        return launch_dkdv_dp<D, true, false>(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv,
                                              BH, T, scale, causal, grad_f32, stream);
    return launch_dkdv_dp<D, false, false>(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv, BH,
                                           T, scale, causal, grad_f32, stream);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const void* o, const void* dO, const float* lse,
                                  float* rowstats, float* dq_accum, int BH, int T, int d,
                                  int o_f32, int f16, cudaStream_t stream) {
    if (d == 64) return launch_pre_d<64>(o, dO, lse, rowstats, dq_accum, BH, T, o_f32, f16, stream);
    return launch_pre_d<128>(o, dO, lse, rowstats, dq_accum, BH, T, o_f32, f16, stream);
}

cudaError_t launch_bwd_dkdv(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdq, const float* rowstats,
                            float* dq_accum, void* dk, void* dv, int BH, int T, int d,
                            float scale, int causal, int grad_f32, int precise, int f16,
                            cudaStream_t stream) {
    if (d == 64)
        return launch_dkdv_d<64>(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv, BH, T, scale,
                                 causal, grad_f32, precise, f16, stream);
    return launch_dkdv_d<128>(tq, tk, tv, tdo, tdq, rowstats, dq_accum, dk, dv, BH, T, scale,
                              causal, grad_f32, precise, f16, stream);
}

cudaError_t launch_bwd_dq_convert(const float* dq_accum, void* dq, long long n, int f16,
                                  cudaStream_t stream) {
    const long long n8 = n / 8;  // d is a multiple of 8, so n is too
    const int threads = 256;
    const unsigned blocks = (unsigned)((n8 + threads - 1) / threads);
    if (f16)
        return launch_dependent(attn_bwd_dq_convert_kernel<true>, dim3(blocks), dim3(threads), 0,
                                stream, dq_accum, static_cast<uint16_t*>(dq), n8);
    return launch_dependent(attn_bwd_dq_convert_kernel<false>, dim3(blocks), dim3(threads), 0,
                            stream, dq_accum, static_cast<uint16_t*>(dq), n8);
}

cudaError_t read_and_clear_device_error_bwd(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

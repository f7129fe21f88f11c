// attn_fwd.cu -- fused causal attention forward for sm_100a.
//
// Computes, per (batch, head) and per 128-row query tile,
//   S = scale * Q K^T (causal mask, keys past T masked), online softmax,
//   O = softmax(S) V, and the per-row natural-log LSE,
// following the Forge paper ("Building an LLM Training Framework from Scratch in
// C++ and Metal on Apple Silicon"), section "Attention kernel design": the tiled
// forward keeps the output accumulator on chip, streams K and V through staged
// tiles, rescales the accumulator by a per-row correction when the running max
// moves, and saves the log-sum-exp for the backward.  The Metal kernel's
// diagonal-matrix trick for the rescale is not needed here: in tensor memory a
// row of the accumulator is one lane, owned by one thread.
//
// Blackwell design (one CTA per query tile, 6 warps):
//   warp 0      TMA producer: Q once, then K/V tiles into an NS-stage ring.
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM, then O += P V with
//               P read from TMEM (tcgen05.mma with A in tensor memory).
//   warps 2..5  softmax: thread r owns query row r (TMEM lane r): loads its S row,
//               masks, updates the running max/sum, writes P (bf16) back to TMEM,
//               and in the epilogue normalises O and stores O (TMA) and LSE.
// Tensor memory (512 columns): S [0,128) | P0 [128,192) | P1 [192,256) | O [256, 256+d)
// | P0 lo [384,448) | P1 lo [448,512) (the lo halves only in precise mode, where P
// enters P V as two bf16 terms, hi = bf16(p) and lo = bf16(p - hi)).
// The MMA warp issues S(n+1) as soon as the softmax has read S(n), so the score
// product of the next tile overlaps the exponentials of the current one; P is
// double-buffered so P V of tile n runs while tile n+1's softmax proceeds.
// The running max is rescaled lazily: O and the row sum are corrected only when
// the max grows by more than 2^8 (all values stay finite and exact to rounding).
#include "forge_internal.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr int kFwdThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Which pairs of a row's exponentials go to the FMA-pipe polynomial (exp2_poly2)
// instead of the MUFU unit.  None: with one softmax warp per SM sub-partition this
// kernel is latency-bound rather than MUFU-bound, and the polynomial's extra
// instructions measured slower at every share tried (3/8 to 6/8).
__device__ __forceinline__ constexpr bool use_poly_pair(int) { return false; }

// wait sites (for the device error word)
enum : uint32_t {
    kSiteQ = 1, kSiteKFull, kSiteVFull, kSiteKVEmpty, kSiteSFull, kSiteSFree, kSitePFull,
    kSitePV, kSiteODone
};

template <int D>
struct FwdCfg {
    static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
    static constexpr int kChunkBytes = kTile * 128;      // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = D == 64 ? 4 : 3;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kBarBytes = 256;
    // 1 KB of slack for aligning the dynamic shared memory base to 1024 bytes.
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
    // tensor memory columns
    static constexpr uint32_t kColS = 0, kColP0 = 128, kColP1 = 192, kColO = 256;
    static constexpr uint32_t kColPlo0 = 384, kColPlo1 = 448;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
};

struct FwdBarriers {
    uint64_t q_full;
    uint64_t k_full[4];
    uint64_t v_full[4];
    uint64_t kv_empty[4];
    uint64_t s_full;
    uint64_t s_free;
    uint64_t p_full;
    uint64_t pv_done;
    uint64_t o_done;
    uint64_t mma_final;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t site,
                                          volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, site, abort));
}

template <int D, bool PRECISE>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_o, void* __restrict__ o_f32_out,
                    float* __restrict__ lse_out, int T, int n_qtiles, float scale_log2,
                    int negate_scores, int causal, int o_f32) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + C::kOffBar);
    volatile int* abort = &bars->abort;

    const int bh = blockIdx.x;
    const int qt = n_qtiles - 1 - blockIdx.y;  // heaviest (most key tiles) first
    const int n_kvtiles_total = (T + kTile - 1) / kTile;
    const int n_tiles = causal ? qt + 1 : n_kvtiles_total;
    const uint32_t warp = warp_id();
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 4);
        mbar_init(&bars->p_full, 4);
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_done, 1);
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
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
            for (int c = 0; c < C::kChunks; ++c)
                tma_load_3d(smem + C::kOffQ + c * C::kChunkBytes, &tmap_q, &bars->q_full, 64 * c,
                            qt * kTile, bh);
            int last_use[4] = {-1, -1, -1, -1};
            for (int n = 0; n < n_tiles; ++n) {
                const int st = n % C::kStages;
                const int use = n / C::kStages;
                if (use > 0 && !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, kSiteKVEmpty, abort))
                    break;
                const int j = causal ? qt - n : n_kvtiles_total - 1 - n;
                mbar_arrive_expect_tx(&bars->k_full[st], C::kTileBytes);
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(smem + C::kOffK + st * C::kTileBytes + c * C::kChunkBytes, &tmap_k,
                                &bars->k_full[st], 64 * c, j * kTile, bh);
                mbar_arrive_expect_tx(&bars->v_full[st], C::kTileBytes);
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(smem + C::kOffV + st * C::kTileBytes + c * C::kChunkBytes, &tmap_v,
                                &bars->v_full[st], 64 * c, j * kTile, bh);
                last_use[st] = use;
            }
            if (*abort) {
                // let copies already issued land before the CTA's memory is released
                mbar_wait_drain(&bars->q_full, 0);
                for (int s = 0; s < C::kStages; ++s)
                    if (last_use[s] >= 0) {
                        mbar_wait_drain(&bars->k_full[s], last_use[s] & 1);
                        mbar_wait_drain(&bars->v_full[s], last_use[s] & 1);
                    }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        // The whole warp runs this loop; one elected lane issues each MMA.
        {
            const uint32_t tS = tmem + C::kColS;
            const uint32_t tO = tmem + C::kColO;
            const uint32_t q_addr = smem_u32(smem + C::kOffQ);
            // bit 13 of the instruction descriptor negates A: S = (-Q) K^T for scale < 0
            const uint32_t idesc_s = C::kIdescS | (negate_scores ? (1u << 13) : 0u);
            bool ok = warp_wait(&bars->q_full, 0, kSiteQ, abort);
            auto issue_pv = [&](int m) -> bool {
                const int st = m % C::kStages;
                if (!warp_wait(&bars->p_full, m & 1, kSitePFull, abort)) return false;
                if (!warp_wait(&bars->v_full[st], (m / C::kStages) & 1, kSiteVFull, abort))
                    return false;
                tc_fence_after();
                const uint32_t tP = tmem + ((m & 1) ? C::kColP1 : C::kColP0);
                const uint32_t tPlo = tmem + ((m & 1) ? C::kColPlo1 : C::kColPlo0);
                const uint32_t v_addr = smem_u32(smem + C::kOffV + st * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    // B = V tile, MN-major: 16 keys = 2 x 8-row groups of 1024 bytes
                    const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, C::kChunkBytes, 1024);
                    mma_ts_warp(tO, tP + kk * 8, bdesc, C::kIdescPV, (m > 0 || kk > 0) ? 1u : 0u);
                    if (PRECISE) mma_ts_warp(tO, tPlo + kk * 8, bdesc, C::kIdescPV, 1u);
                }
                mma_commit_warp(&bars->pv_done);
                mma_commit_warp(&bars->kv_empty[st]);
                return true;
            };
            for (int n = 0; ok && n < n_tiles; ++n) {
                const int st = n % C::kStages;
                if (!warp_wait(&bars->k_full[st], (n / C::kStages) & 1, kSiteKFull, abort)) {
                    ok = false;
                    break;
                }
                if (n > 0 && !warp_wait(&bars->s_free, (n - 1) & 1, kSiteSFree, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_addr = smem_u32(smem + C::kOffK + st * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    const uint64_t adesc = sdesc_sw128(q_addr + koff, 16, 1024);
                    const uint64_t bdesc = sdesc_sw128(k_addr + koff, 16, 1024);
                    mma_ss_warp(tS, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_warp(&bars->s_full);
                if (n > 0 && !issue_pv(n - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = issue_pv(n_tiles - 1);
            if (ok) mma_commit_warp(&bars->o_done);
            // every MMA this thread issued must retire before tensor memory is freed
            mma_commit_warp(&bars->mma_final);
            mbar_wait_drain(&bars->mma_final, 0);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const uint32_t row = ((warp & 3) << 5) + lane;  // TMEM lane owned by this thread
        const uint32_t lane_off = ((warp & 3) << 5) << 16;
        const uint32_t tS = tmem + lane_off + C::kColS;
        const uint32_t tO = tmem + lane_off + C::kColO;
        const int grow = qt * kTile + (int)row;  // query index of this row
        float m_run = -INFINITY;                  // running max, log2 units
        float l_run = 0.f;                        // running sum of exp2(u - m_run)
        bool ok = true;
        for (int n = 0; n < n_tiles; ++n) {
            const int j = causal ? qt - n : n_kvtiles_total - 1 - n;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, kSiteSFull, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sraw[kTile];
#pragma unroll
            for (int c = 0; c < kTile / 32; ++c) tmem_ld32(tS + c * 32, sraw + c * 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->s_free);

            // Row max of the raw scores over the keys this row may see.  scale_log2 is
            // >= 0 (a negative scale is applied by negating Q in the MMA), so the max
            // of the scaled scores is scale_log2 times the raw max.
            const bool diag = causal && j == qt;
            const bool tail = !causal && (j + 1) * kTile > T;
            const bool masked_tile = diag || tail;
            const int key_lim = diag ? (int)row : (tail ? T - 1 - j * kTile : kTile - 1);
            float s[kTile];
#pragma unroll
            for (int c = 0; c < kTile; ++c) s[c] = __uint_as_float(sraw[c]);
            if (masked_tile) {  // the same for every thread of the CTA
#pragma unroll
                for (int c = 0; c < kTile; ++c)
                    if (c > key_lim) s[c] = -INFINITY;
            }
            // eight independent chains of three-input max (16 values each), then 8 -> 1
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                mx[e] = fmaxf(s[16 * e], s[16 * e + 1]);
#pragma unroll
                for (int c = 2; c < 16; c += 2) mx[e] = fmax3(mx[e], s[16 * e + c], s[16 * e + c + 1]);
            }
            const float mt =
                fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                scale_log2;

            float alpha = 1.f;
            bool need = false;
            if (n == 0) {
                m_run = mt;
            } else if (mt > m_run + kRescaleThreshold) {
                need = true;
                alpha = ex2_approx(m_run - mt);
                m_run = mt;
                l_run *= alpha;
            }
            if (n > 0 && __any_sync(0xffffffffu, need)) {
                // O must include P(n-1) V before it is rescaled
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&bars->pv_done, (n - 1) & 1, kSitePV, abort))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tO + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st32(tO + c * 32, r);
                }
                tmem_wait_st();
            }

            // P = exp2(s * scale_log2 - m), row sum, pack to bf16 pairs, store to TMEM
            const uint32_t tP = tmem + lane_off + ((n & 1) ? C::kColP1 : C::kColP0);
            const uint32_t tPlo = tmem + lane_off + ((n & 1) ? C::kColPlo1 : C::kColPlo0);
            const float neg_m = -m_run;
            const float2 sl2 = make_float2(scale_log2, scale_log2);
            const float2 nm2 = make_float2(neg_m, neg_m);
            float2 ls[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) ls[e] = make_float2(0.f, 0.f);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32], pl[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = half * 64 + 2 * e;
                    const float2 x = ffma2(make_float2(s[c], s[c + 1]), sl2, nm2);
                    float2 p;
                    if (!PRECISE && use_poly_pair(e)) {
                        p = exp2_poly2(x);
                    } else {
                        p.x = ex2_approx(x.x);
                        p.y = ex2_approx(x.y);
                    }
                    if (masked_tile) {  // also covers scale 0, where -inf * 0 is NaN
                        p.x = c > key_lim ? 0.f : p.x;
                        p.y = c + 1 > key_lim ? 0.f : p.y;
                    }
                    ls[e & 3] = fadd2(ls[e & 3], p);
                    pk[e] = pack_bf16x2(p.x, p.y);
                    if (PRECISE)
                        pl[e] = pack_bf16x2(p.x - bf16_lo_to_float(pk[e]),
                                            p.y - bf16_hi_to_float(pk[e]));
                }
                tmem_st32(tP + half * 32, pk);
                if (PRECISE) tmem_st32(tPlo + half * 32, pl);
            }
            const float2 ls01 = fadd2(ls[0], ls[1]), ls23 = fadd2(ls[2], ls[3]);
            const float2 lsum = fadd2(ls01, ls23);
            l_run += lsum.x + lsum.y;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full);
        }

        // ----------------------------------------------------------- epilogue
        const bool epi =
            ok && __all_sync(0xffffffffu, mbar_wait(&bars->o_done, 0, kSiteODone, abort));
        uint8_t* stage = smem + C::kOffQ;  // Q is no longer read by any MMA
        if (epi) {
            tc_fence_after();
            const float inv_l = 1.f / l_run;
            if (grow < T) lse_out[(size_t)bh * T + grow] = (m_run + log2f(l_run)) * kLn2;
            float* orow = reinterpret_cast<float*>(o_f32_out) + ((size_t)bh * T + grow) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tO + c * 32, r);  // all lanes: the load is warp-collective
                tmem_wait_ld();
                if (!o_f32) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                            __uint_as_float(r[2 * e + 1]) * inv_l);
                    // 32 columns = 64 bytes = 4 x 16-byte chunks of the row
                    uint8_t* chunk_base = stage + (c >> 1) * C::kChunkBytes;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t ch = (c & 1) * 4 + e;
                        *reinterpret_cast<uint4*>(chunk_base + sw128_offset(row, ch)) =
                            make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                    }
                } else if (grow < T) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        *reinterpret_cast<float4*>(orow + c * 32 + 4 * e) =
                            make_float4(__uint_as_float(r[4 * e]) * inv_l,
                                        __uint_as_float(r[4 * e + 1]) * inv_l,
                                        __uint_as_float(r[4 * e + 2]) * inv_l,
                                        __uint_as_float(r[4 * e + 3]) * inv_l);
                }
            }
            if (!o_f32) fence_proxy_async_smem();
        }
        // every softmax thread reaches this barrier, aborted or not
        named_bar_sync(1, 128);
        if (!o_f32 && warp == 2 && lane == 0 && epi && !*abort) {
            for (int c = 0; c < C::kChunks; ++c)
                tma_store_3d(&tmap_o, stage + c * C::kChunkBytes, 64 * c, qt * kTile, bh);
            tma_store_commit();
            tma_store_wait_all_read();  // the store has read the staged O
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

template <int D, bool PRECISE>
cudaError_t launch_fwd_dp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& to, void* o, float* lse, int BH, int T, float scale,
                          int causal, int o_f32, cudaStream_t stream) {
    using C = FwdCfg<D>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, PRECISE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int n_qtiles = (T + kTile - 1) / kTile;
    dim3 grid(BH, n_qtiles);
    attn_fwd_kernel<D, PRECISE><<<grid, kFwdThreads, C::kSmemBytes, stream>>>(
        tq, tk, tv, to, o, lse, T, n_qtiles, fabsf(scale) * kLog2e, scale < 0.f ? 1 : 0, causal,
        o_f32);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& to, void* o, float* lse, int BH, int T, float scale,
                         int causal, int o_f32, int precise, cudaStream_t stream) {
    if (precise)
        return launch_fwd_dp<D, true>(tq, tk, tv, to, o, lse, BH, T, scale, causal, o_f32,
                                      stream);
    return launch_fwd_dp<D, false>(tq, tk, tv, to, o, lse, BH, T, scale, causal, o_f32, stream);
}

}  // namespace

cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, void* o, float* lse, int BH, int T, int d,
                            float scale, int causal, int o_f32, int precise,
                            cudaStream_t stream) {
    if (d == 64)
        return launch_fwd_d<64>(tq, tk, tv, to, o, lse, BH, T, scale, causal, o_f32, precise,
                                stream);
    return launch_fwd_d<128>(tq, tk, tv, to, o, lse, BH, T, scale, causal, o_f32, precise,
                             stream);
}

cudaError_t read_and_clear_device_error_fwd(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

// attn_fwd_pair.cu -- fused causal attention forward for sm_100a, two query tiles
// per work item, persistent CTAs (the d = 64 forward).
//
// Same operation as attn_fwd.cu (the Forge paper's tiled forward, section
// "Attention kernel design": on-chip output accumulator, K/V streamed through
// staged tiles, per-row rescale when the running max moves, saved log-sum-exp),
// arranged for throughput:
//   * a work item is a pair of adjacent 128-row query tiles (A = 2p, B = 2p + 1) of
//     one head; both read the same K/V tiles, so each K/V tile is loaded once for
//     256 query rows;
//   * two softmax warpgroups, one per tile, so every SM sub-partition runs two
//     softmax warps (one softmax warp per sub-partition leaves the exponentials and
//     tensor-memory loads latency-bound), and two MMA-issuing warps, one per tile,
//     so one tile's products run while the other tile's exponentials do;
//   * CTAs are persistent (one per SM) and walk a list of items ordered by
//     decreasing work, so set-up, the first loads and the epilogue of one item
//     overlap the neighbouring items.
// Warps: 0 TMA producer, 1 and 2 MMA issuers for tiles A and B (each runs converged;
// one elected lane issues), 3 idle (0..3 form the control warpgroup, which hands
// registers to the softmax warpgroups), 4..7 softmax of tile A, 8..11 of tile B.
// Launch: 384 threads x 168 registers; the control warpgroup drops to 72 and each
// softmax warpgroup rises to 216 (4*32*72 + 8*32*216 = 384*168), so a softmax thread
// holds its whole S row in registers.
// Tensor memory: S_A [0,128) | S_B [128,256) | O_A [256, 256+d) | O_B [256+d, 256+2d),
// and for d = 64 also P_A [384,448) | P_B [448,512): the next key tile's S_X is then
// issued as soon as the softmax holds S_X in registers, and overlaps its
// exponentials.  For d = 128 the columns are full, so P_X (bf16) is written over
// the first 64 columns of S_X and the next S_X waits until P_X V has completed;
// that serialisation makes this kernel slower than the one-tile kernel at d = 128,
// so the library uses it for d = 64 only.
#include "forge_internal.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr int kPairThreads = 384;
constexpr uint32_t kControlRegs = 72, kSoftmaxRegs = 216;
static_assert(4 * 32 * kControlRegs + 8 * 32 * kSoftmaxRegs == kPairThreads * 168,
              "register split must equal the launch allocation");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

enum : uint32_t {
    kSiteQFull = 1, kSiteQEmpty, kSiteKFull, kSiteVFull, kSiteKVEmpty, kSiteSFull, kSitePFull,
    kSitePVDone, kSiteOFull, kSiteOFree
};

template <int D>
struct PairCfg {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kTile * 128;
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = D == 64 ? 4 : 2;  // K/V ring
    static constexpr int kOffQ = 0;                   // Q_A, Q_B
    static constexpr int kOffK = kOffQ + 2 * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kSmemBytes = kOffBar + 512 + 1024;  // + alignment slack
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static constexpr uint32_t kColO = 256;
    static constexpr bool kSepP = (D == 64);  // P_X in columns of its own
    static constexpr uint32_t kColP = kSepP ? 384 : 0;  // + 64 X (own) or + 128 X (in S_X)
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
};

struct PairBars {
    uint64_t q_full, q_empty;
    uint64_t k_full[4], v_full[4], kv_empty[4];
    uint64_t s_full[2], s_free[2], p_full[2], pv_done[2], o_full[2], o_free[2];
    uint64_t mma_final;
    uint32_t tmem_base;
    int abort;
};

// One work item: query tiles 2p and 2p + 1 (if it exists) of head bh, and the key
// tiles it visits, from j_top down to j_top - n_steps + 1.
struct Item {
    int bh, p, has_b, j_top, n_steps;
};

__device__ __forceinline__ Item decode_item(int k, int BH, int n_pairs, int n_qtiles,
                                            int causal) {
    Item it;
    it.p = causal ? n_pairs - 1 - k / BH : k / BH;  // heaviest pairs first
    it.bh = k % BH;
    it.has_b = (2 * it.p + 1) < n_qtiles;
    if (causal) {
        it.j_top = it.has_b ? 2 * it.p + 1 : 2 * it.p;
        it.n_steps = it.j_top + 1;
    } else {
        it.j_top = n_qtiles - 1;
        it.n_steps = n_qtiles;
    }
    return it;
}

// Does query tile X (0 = A, 1 = B) of the item take part in step t?
__device__ __forceinline__ bool takes_part(const Item& it, int X, int t, int causal) {
    if (t < 0 || t >= it.n_steps) return false;
    if (X == 1) return it.has_b;
    return !causal || (it.j_top - t) <= 2 * it.p;
}

template <int D>
__global__ void __launch_bounds__(kPairThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, void* __restrict__ o_out,
                         float* __restrict__ lse_out, int T, int BH, int n_qtiles, int n_items,
                         float scale_log2, int negate_scores, int causal, int o_f32) {
    using C = PairCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairBars* bars = reinterpret_cast<PairBars*>(smem + C::kOffBar);
    volatile int* abort = &bars->abort;
    const int n_pairs = (n_qtiles + 1) / 2;
    const uint32_t warp = warp_id();
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        mbar_init(&bars->q_empty, 2);  // both MMA issuers
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 2);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&bars->s_full[x], 1);
            mbar_init(&bars->s_free[x], 4);
            mbar_init(&bars->p_full[x], 4);
            mbar_init(&bars->pv_done[x], 1);
            mbar_init(&bars->o_full[x], 1);
            mbar_init(&bars->o_free[x], 4);
        }
        mbar_init(&bars->mma_final, 2);  // each MMA issuer drains its own products
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

    if (warp < 4) {
      regs_dec<kControlRegs>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            int g = 0, n_item = 0;
            int last_use[4] = {-1, -1, -1, -1};
            int q_loads = 0;
            bool ok = true;
            for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x, ++n_item) {
                const Item it = decode_item(k, BH, n_pairs, n_qtiles, causal);
                if (n_item > 0 && !mbar_wait(&bars->q_empty, (n_item - 1) & 1, kSiteQEmpty, abort)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bars->q_full, (it.has_b ? 2 : 1) * C::kTileBytes);
                for (int x = 0; x < 1 + it.has_b; ++x)
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffQ + x * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_q, &bars->q_full, 64 * c, (2 * it.p + x) * kTile, it.bh);
                ++q_loads;
                for (int t = 0; t < it.n_steps; ++t, ++g) {
                    const int st = g % C::kStages, use = g / C::kStages;
                    if (use > 0 &&
                        !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, kSiteKVEmpty, abort)) {
                        ok = false;
                        break;
                    }
                    const int j = it.j_top - t;
                    mbar_arrive_expect_tx(&bars->k_full[st], C::kTileBytes);
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffK + st * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_k, &bars->k_full[st], 64 * c, j * kTile, it.bh);
                    mbar_arrive_expect_tx(&bars->v_full[st], C::kTileBytes);
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffV + st * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_v, &bars->v_full[st], 64 * c, j * kTile, it.bh);
                    last_use[st] = use;
                }
            }
            if (*abort) {
                // let copies already issued land before the CTA's memory is released
                if (q_loads > 0) mbar_wait_drain(&bars->q_full, (q_loads - 1) & 1);
                for (int s = 0; s < C::kStages; ++s)
                    if (last_use[s] >= 0) {
                        mbar_wait_drain(&bars->k_full[s], last_use[s] & 1);
                        mbar_wait_drain(&bars->v_full[s], last_use[s] & 1);
                    }
            }
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------- MMA issuers, one per tile
        // Warp 1 issues every product of tile A, warp 2 every product of tile B, so
        // neither tile's progress waits on the other's.
        {
            const int X = warp - 1;
            const uint32_t idesc_s = C::kIdescS | (negate_scores ? (1u << 13) : 0u);
            const uint32_t qx_addr = smem_u32(smem + C::kOffQ + X * C::kTileBytes);
            const uint32_t tSX = tmem + 128 * X;
            const uint32_t tO = tmem + C::kColO + X * D;
            const uint32_t tP = tmem + C::kColP + (C::kSepP ? 64 : 128) * X;
            int g = 0, n_item = 0, n_pv = 0, n_o = 0, n_sx = 0;
            bool ok = true;
            auto W = [&](uint64_t* bar, int parity, uint32_t site) {
                if (ok && !__all_sync(0xffffffffu, mbar_wait(bar, parity & 1, site, abort)))
                    ok = false;
                return ok;
            };
            // S_X(t) = Q_X K_t^T into S_X, which must be free: the softmax has read
            // the previous S_X (own P columns) or P_X V has read P_X (P in S_X)
            auto issue_s = [&](int t, int& s_left) {
                if (C::kSepP) {
                    if (n_sx > 0 && !W(&bars->s_free[X], n_sx - 1, kSiteSFull)) return;
                } else if (n_pv > 0 && !W(&bars->pv_done[X], n_pv - 1, kSitePVDone)) {
                    return;
                }
                const int gs = g + t;
                if (!W(&bars->k_full[gs % C::kStages], gs / C::kStages, kSiteKFull)) return;
                tc_fence_after();
                const uint32_t k_addr =
                    smem_u32(smem + C::kOffK + (gs % C::kStages) * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    mma_ss_warp(tSX, sdesc_sw128(qx_addr + koff, 16, 1024),
                           sdesc_sw128(k_addr + koff, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_warp(&bars->s_full[X]);
                ++n_sx;
                if (--s_left == 0) mma_commit_warp(&bars->q_empty);  // Q_X no longer read
            };
            for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x, ++n_item) {
                const Item it = decode_item(k, BH, n_pairs, n_qtiles, causal);
                if (!W(&bars->q_full, n_item, kSiteQFull)) break;
                int s_left = 0, t0 = it.n_steps;
                for (int t = it.n_steps - 1; t >= 0; --t)
                    if (takes_part(it, X, t, causal)) {
                        ++s_left;
                        t0 = t;
                    }
                if (s_left == 0) mma_commit_warp(&bars->q_empty);  // tile B absent: arrive anyway
                else issue_s(t0, s_left);
                bool first_pv = true;
                for (int t = 0; ok && t < it.n_steps; ++t) {
                    const int gs = g + t;
                    const int st = gs % C::kStages;
                    if (takes_part(it, X, t, causal)) {
                        // own P columns: the next score product first, as soon as the
                        // softmax holds this step's scores in registers
                        if (C::kSepP && takes_part(it, X, t + 1, causal)) issue_s(t + 1, s_left);
                        // O_X += P_X V_t, P_X from tensor memory
                        if (!W(&bars->p_full[X], n_pv, kSitePFull)) break;
                        if (!W(&bars->v_full[st], gs / C::kStages, kSiteVFull)) break;
                        if (first_pv && n_o > 0 && !W(&bars->o_free[X], n_o - 1, kSiteOFree)) break;
                        tc_fence_after();
                        const uint32_t v_addr = smem_u32(smem + C::kOffV + st * C::kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_ts_warp(tO, tP + kk * 8,
                                   sdesc_sw128(v_addr + kk * 2048, C::kChunkBytes, 1024),
                                   C::kIdescPV, (!first_pv || kk > 0) ? 1u : 0u);
                        mma_commit_warp(&bars->pv_done[X]);
                        ++n_pv;
                        first_pv = false;
                        // P in S_X: the next S_X right after this P_X V
                        if (!C::kSepP && takes_part(it, X, t + 1, causal)) issue_s(t + 1, s_left);
                    } else {
                        // A step this tile sits out still arrives on kv_empty, but only
                        // once the step's tiles have been loaded: that keeps each
                        // arrival in the phase of its own use of the stage (an issuer
                        // that ran ahead could otherwise arrive twice in one phase).
                        if (!W(&bars->v_full[st], gs / C::kStages, kSiteVFull)) break;
                    }
                    if (!ok) break;
                    mma_commit_warp(&bars->kv_empty[st]);  // both issuers arrive for every step
                }
                if (!ok) break;
                if (!first_pv) {
                    mma_commit_warp(&bars->o_full[X]);
                    ++n_o;
                }
                g += it.n_steps;
            }
            // every MMA this thread issued must retire before tensor memory is freed
            mma_commit_warp(&bars->mma_final);
            mbar_wait_drain(&bars->mma_final, 0);
        }
      }
    } else {
        regs_inc<kSoftmaxRegs>();
        // ------------------------------------------------------------ softmax
        const int X = (warp - 4) >> 2;                    // 0: tile A, 1: tile B
        const uint32_t row = ((warp & 3) << 5) + lane;    // TMEM lane owned
        const uint32_t lane_off = ((warp & 3) << 5) << 16;
        const uint32_t tS = tmem + lane_off + 128 * X;
        const uint32_t tO = tmem + lane_off + C::kColO + X * D;
        const uint32_t tP = tmem + lane_off + C::kColP + (C::kSepP ? 64 : 128) * X;
        int n_s = 0, n_o = 0;
        bool ok = true;
        auto W = [&](uint64_t* bar, int parity, uint32_t site) {
            if (ok && !__all_sync(0xffffffffu, mbar_wait(bar, parity & 1, site, abort)))
                ok = false;
            return ok;
        };
        for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
            const Item it = decode_item(k, BH, n_pairs, n_qtiles, causal);
            if (X == 1 && !it.has_b) continue;
            const int qx = 2 * it.p + X;                  // query tile of this warpgroup
            const int grow = qx * kTile + (int)row;       // query row of this thread
            float m_run = -INFINITY, l_run = 0.f;
            bool first = true;
            for (int t = 0; ok && t < it.n_steps; ++t) {
                if (!takes_part(it, X, t, causal)) continue;
                const int j = it.j_top - t;
                if (!W(&bars->s_full[X], n_s, kSiteSFull)) break;
                tc_fence_after();
                const bool diag = causal && j == qx;
                const bool tail = !causal && (j + 1) * kTile > T;
                const bool masked = diag || tail;
                const int key_lim = diag ? (int)row : (tail ? T - 1 - j * kTile : kTile - 1);

                // the whole S row into registers (one pass over tensor memory)
                uint32_t sv[kTile];
#pragma unroll
                for (int c = 0; c < kTile / 32; ++c) tmem_ld32(tS + 32 * c, sv + 32 * c);
                tmem_wait_ld();
                if (C::kSepP) {  // S_X is free for the next score product
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->s_free[X]);
                }
                // row max of the raw scores the row may see
                float sm[kTile];
#pragma unroll
                for (int c = 0; c < kTile; ++c) sm[c] = __uint_as_float(sv[c]);
                if (masked) {
#pragma unroll
                    for (int c = 0; c < kTile; ++c)
                        if (c > key_lim) sm[c] = -INFINITY;
                }
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    mx[e] = fmaxf(sm[16 * e], sm[16 * e + 1]);
#pragma unroll
                    for (int c = 2; c < 16; c += 2) mx[e] = fmax3(mx[e], sm[16 * e + c], sm[16 * e + c + 1]);
                }
                const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                       fmaxf(mx[6], mx[7])) * scale_log2;

                float alpha = 1.f;
                bool need = false;
                if (first) {
                    m_run = mt;
                } else if (mt > m_run + kRescaleThreshold) {
                    need = true;
                    alpha = ex2_approx(m_run - mt);
                    m_run = mt;
                    l_run *= alpha;
                }
                const bool any_need = !first && __any_sync(0xffffffffu, need);
                if (any_need || (C::kSepP && !first)) {
                    // O_X must hold every earlier P_X V before it is rescaled, and
                    // (own P columns) P_X must have been read before it is rewritten
                    // (the previous product of this warpgroup is number n_s - 1; older
                    // ones, and the last one of an earlier item, have completed)
                    if (C::kSepP && !W(&bars->pv_done[X], n_s - 1, kSitePVDone)) break;
                    tc_fence_after();
                }
                if (any_need) {
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
                first = false;

                // P = exp2(s * scale_log2 - m), packed bf16 pairs, written to P_X
                const float neg_m = -m_run;
                const float2 sl2 = make_float2(scale_log2, scale_log2);
                const float2 nm2 = make_float2(neg_m, neg_m);
                float2 ls[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) ls[e] = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 32 columns -> 16 packed pairs at a time
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int col = 32 * q + 2 * e;
                        const float2 x = ffma2(make_float2(sm[col], sm[col + 1]), sl2, nm2);
                        float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        if (masked) {  // also covers scale 0, where -inf * 0 is NaN
                            p.x = col > key_lim ? 0.f : p.x;
                            p.y = col + 1 > key_lim ? 0.f : p.y;
                        }
                        ls[e & 3] = fadd2(ls[e & 3], p);
                        pk[e] = pack_bf16x2(p.x, p.y);
                    }
                    tmem_st16(tP + 16 * q, pk);
                }
                const float2 lsum = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
                l_run += lsum.x + lsum.y;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[X]);
                ++n_s;
            }
            if (!ok) break;
            // ------------------------------------------------------- epilogue
            if (!W(&bars->o_full[X], n_o, kSiteOFull)) break;
            tc_fence_after();
            const float inv_l = 1.f / l_run;
            if (grow < T)
                lse_out[(size_t)it.bh * T + grow] = (m_run + log2f(l_run)) * kLn2;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tO + c * 32, r);  // all lanes: the load is warp-collective
                tmem_wait_ld();
                if (grow < T) {
                    const size_t base = ((size_t)it.bh * T + grow) * D + c * 32;
                    if (o_f32) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o_out) + base);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l,
                                                 __uint_as_float(r[4 * e + 1]) * inv_l,
                                                 __uint_as_float(r[4 * e + 2]) * inv_l,
                                                 __uint_as_float(r[4 * e + 3]) * inv_l);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(
                            static_cast<__nv_bfloat16*>(o_out) + base);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * e]) * inv_l,
                                            __uint_as_float(r[8 * e + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(r[8 * e + 2]) * inv_l,
                                            __uint_as_float(r[8 * e + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(r[8 * e + 4]) * inv_l,
                                            __uint_as_float(r[8 * e + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(r[8 * e + 6]) * inv_l,
                                            __uint_as_float(r[8 * e + 7]) * inv_l));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->o_free[X]);
            ++n_o;
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

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            n <= 0)
            n = 148;
    }
    return n;
}

template <int D>
cudaError_t launch_pair_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          void* o, float* lse, int BH, int T, float scale, int causal, int o_f32,
                          cudaStream_t stream) {
    using C = PairCfg<D>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(attn_fwd_pair_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const int n_qtiles = (T + kTile - 1) / kTile;
    const int n_items = BH * ((n_qtiles + 1) / 2);
    const int grid = n_items < sm_count() ? n_items : sm_count();
    attn_fwd_pair_kernel<D><<<grid, kPairThreads, C::kSmemBytes, stream>>>(
        tq, tk, tv, o, lse, T, BH, n_qtiles, n_items, fabsf(scale) * kLog2e, scale < 0.f ? 1 : 0,
        causal, o_f32);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, void* o, float* lse, int BH, int T, int d,
                                 float scale, int causal, int o_f32, cudaStream_t stream) {
    if (d != 64) return cudaErrorInvalidValue;  // d = 128 runs the one-tile kernel
    return launch_pair_d<64>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32, stream);
}

cudaError_t read_and_clear_device_error_fwd_pair(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

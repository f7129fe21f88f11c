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
// Blackwell design (persistent CTAs; used for every head dimension and mode).  At
// d = 128 one CTA per SM with 6 warps and two S buffers.  At d = 64 two CTAs share an
// SM, each with 8 warps (a control and a softmax warpgroup, registers moved to the
// softmax by setmaxnreg), one S buffer and half of tensor memory: the two CTAs'
// softmax warps overlap on every sub-partition.  A work item is one (head, query tile); items are dealt
// heaviest first, zigzag over the CTAs, and every role walks the same item sequence,
// so one item's epilogue and the next item's Q load overlap the neighbouring item's
// products.
//   warp 0      TMA producer: Q per item into one of two shared-memory buffers
//               (d = 64; one at d = 128), once the buffer's previous Q has been
//               copied to tensor memory, then K/V tiles into an NS-stage ring.
//   warp 1      MMA issuer (converged warp, one elected lane issues): copies the
//               item's Q into tensor memory (tcgen05.cp), then S = Q K^T with Q read
//               from tensor memory as the A operand and K from shared memory (so a
//               score product reads one operand's bytes from shared memory, not
//               two), and O += P V with P read from tensor memory.  An item's first
//               P V waits until the previous item's O has been read out.
//   warps 2, 3  (d = 64) idle: they complete the control warpgroup.
//   warps 2..5 (d = 128), 4..7 (d = 64)
//               softmax: thread r owns query row r (TMEM lane r): loads its S row,
//               masks, updates the running max/sum, writes P (bf16) back to TMEM,
//               and in the epilogue normalises its O row and writes it and its LSE
//               to global memory.  With bf16 P, from an item's third tile on, the
//               tile's max is taken in the same pass as its exponentials (against the
//               running max), and the tile is redone in the rare case that it moves
//               the max past the lazy-rescale bound.  With fp16 P that bound is 2^15
//               (fp16's range), which logits of a few nats' spread cross on a large
//               share of tiles, so the fp16 kernels take every tile's max first.
// Tensor memory: d = 128, 512 columns: S0 [0,128) | S1 [128,256) | O [256,384) | Q0, Q1
// [384,512); d = 64, 256 columns per CTA: S0 [0,128) | O [128,192) | Q0, Q1 [192,256)
// (Q: d/2 columns each).  Key tile g uses S buffer g % (number of buffers), and its P
// is written over that S (the softmax thread holds
// its whole S row in registers by then): hi = bf16(p) in the buffer's first 64
// columns and, in precise mode, where P enters P V as two bf16 terms, lo =
// bf16(p - hi) in the next 64.  The score products run two key tiles ahead of the
// P V products with two buffers (S0 S1 PV0 S2 PV1 S3 ...): S(g+1) is complete while the
// softmax is still on tile g.  S(g+2) reuses the buffer of P(g), so it is issued once
// P V(g) has completed (its commit).  With one buffer (d = 64) S(g+1) follows P V(g)
// and the SM's other CTA fills the gap.
// The running max is rescaled lazily: O and the row sum are corrected only when
// the max grows by more than 2^64 (2^15 with fp16 P); all values stay finite and
// exact to rounding.
#include <type_traits>

#include "forge_internal.h"
#include "sm100_ptx.cuh"

namespace forge {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// The running max is moved (and O, the row sum rescaled) only when a tile raises it by
// more than this many log2 units, so P <= 2^bound: 2^64 with bf16 P (P, O and the row
// sum stay far inside the bf16 / fp32 range; the relative precision does not depend on
// the magnitude), 2^15 with fp16 P (below the fp16 maximum, 65504).
template <bool F16>
constexpr float kRescaleThreshold = F16 ? 15.0f : 64.0f;

// Which pairs of a row's exponentials go to the FMA-pipe polynomial (exp2_poly2)
// instead of the MUFU unit.  None: every share tried (1/8 to 6/8) measured slower;
// the MUFU unit runs the 128 exponentials of a row in about 1.2K cycles, close to
// its 1K-cycle bound, and the polynomial's extra instructions lengthen the rest.
__device__ __forceinline__ constexpr bool use_poly_pair(int) { return false; }

// wait sites (for the device error word)
enum : uint32_t {
    kSiteQ = 1, kSiteKFull, kSiteVFull, kSiteKVEmpty, kSiteSFull, kSiteSFree, kSitePFull,
    kSitePV, kSiteODone, kSiteQEmpty, kSiteOFree
};

template <int D, bool F16>
struct FwdCfg {
    // d = 64: two CTAs share an SM, each with one S buffer and half of tensor memory,
    // so each sub-partition runs two softmax warps (of different CTAs) whose latencies
    // overlap.  Eight warps per CTA (two whole warpgroups, for the register split).
    // d = 128: one CTA per SM with two S buffers, six warps.
    static constexpr bool kTwoPerSM = D == 64;
    static constexpr int kCtasPerSM = kTwoPerSM ? 2 : 1;
    static constexpr int kThreads = kTwoPerSM ? 256 : 192;
    static constexpr uint32_t kWarpSoftmax0 = kTwoPerSM ? 4 : 2;  // first softmax warp
    static constexpr int kSBufs = kTwoPerSM ? 1 : 2;
    // registers per thread after setmaxnreg (two CTAs of 256 threads leave 128 each at
    // launch): the control warpgroup gives most of them to the softmax warpgroup
    static constexpr uint32_t kRegsCtl = 48, kRegsSoftmax = 208;
    static_assert(!kTwoPerSM || 128 * kRegsCtl + 128 * kRegsSoftmax <= 65536 / kCtasPerSM,
                  "register split exceeds the block's launch allocation");
    static constexpr int kChunks = D / 64;               // 128-byte column chunks per row
    static constexpr int kChunkBytes = kTile * 128;      // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = D == 64 ? 2 : 3;
    // Q buffers: with two (d = 64), the next item's Q is loaded while this item runs,
    // so its first score product never waits for the load; d = 128 has room for one.
    static constexpr int kQBufs = D == 64 ? 2 : 1;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBufs * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kBarBytes = 256;
    // 1 KB of slack for aligning the dynamic shared memory base to 1024 bytes.
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kSmemBytes * kCtasPerSM <= 233472 - 1024 * kCtasPerSM,
                  "shared memory budget of the SM");
    // tensor memory columns
    // kSBufs S buffers; tile g uses buffer g % kSBufs, and its P (bf16, 64 columns;
    // the lo half of precise mode in the next 64) is written over the S it came from
    static constexpr uint32_t kColS0 = 0, kColBuf = 128, kColPlo = 64;
    static constexpr uint32_t kColO = kSBufs * kColBuf;
    // Q of the item in tensor memory (bf16 pairs, d/2 columns), two buffers by item
    // parity: the score product's A operand
    static constexpr uint32_t kColQ = kColO + D;
    static constexpr uint32_t kTmemCols = kTwoPerSM ? 256 : 512;
    static_assert(kColQ + 2 * (D / 2) <= kTmemCols, "tensor memory budget");
    // Q, K, V and P are all bf16, or all fp16 (F16)
    static constexpr uint32_t kIdescS = idesc_f16kind_f32(128, 128, false, false, F16);
    static constexpr uint32_t kIdescPV = idesc_f16kind_f32(128, D, false, true, F16);
};

struct FwdBarriers {
    uint64_t q_full[2], q_empty[2];  // per Q buffer
    uint64_t k_full[4];
    uint64_t v_full[4];
    uint64_t kv_empty[4];
    uint64_t s_full[2];  // per S buffer
    uint64_t p_full[2];  // per S buffer (P is written over S)
    uint64_t pv_done;    // every P V, in order
    uint64_t o_done, o_free;  // an item's O complete / read out of tensor memory
    uint64_t mma_final;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t site,
                                          volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, site, abort));
}

// Register split of the two-CTAs-per-SM configuration (every warp of a warpgroup
// executes it in its own role's branch); a no-op otherwise.
template <int D, bool F16, bool kSoftmax>
__device__ __forceinline__ void fwd_set_regs() {
    using C = FwdCfg<D, F16>;
    if constexpr (C::kTwoPerSM) {
        if constexpr (kSoftmax)
            regs_inc<C::kRegsSoftmax>();
        else
            regs_dec<C::kRegsCtl>();
    }
}

template <int D, bool PRECISE, bool F16>
__global__ void __launch_bounds__(FwdCfg<D, F16>::kThreads, FwdCfg<D, F16>::kCtasPerSM)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    void* __restrict__ o_out, float* __restrict__ lse_out, int T, int BH,
                    int n_qtiles, int n_items, float scale_log2, int negate_scores, int causal,
                    int o_f32) {
    using C = FwdCfg<D, F16>;
    static_assert(sizeof(FwdBarriers) <= C::kBarBytes, "barrier block");
    static_assert(!(PRECISE && F16), "the hi + lo split is a bf16-operand mode");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + C::kOffBar);
    volatile int* abort = &bars->abort;

    const int n_kvtiles_total = (T + kTile - 1) / kTile;
    const int n_ctas = (int)gridDim.x;
    // Persistent CTAs.  The CTA's r-th work item is a (head, query tile) pair; items
    // are numbered heaviest first (the last query tile sees the most key tiles) and
    // dealt in a zigzag over the CTAs.  Every role walks the same item sequence; the
    // per-key-tile barriers count across items.
    auto item_of = [&](int r, int& bh_out, int& qt_out) -> bool {
        const int k = r * n_ctas + ((r & 1) ? (n_ctas - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        if (k >= n_items) return false;
        qt_out = n_qtiles - 1 - k / BH;
        bh_out = k % BH;
        return true;
    };
    auto tiles_of = [&](int qt_) { return causal ? qt_ + 1 : n_kvtiles_total; };
    const uint32_t warp = warp_id();
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->q_full[b], 1);
            mbar_init(&bars->q_empty[b], 1);
        }
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->s_full[b], 1);
            mbar_init(&bars->p_full[b], 4);
        }
        mbar_init(&bars->pv_done, 1);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->o_free, 4);
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
    // the prologue above overlaps the previous kernel's tail; inputs are read only now
    grid_dependency_wait();
    allow_dependents_launch();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        fwd_set_regs<D, F16, false>();
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            int last_use[4] = {-1, -1, -1, -1}, last_q[2] = {-1, -1};
            int g = 0;  // key tiles so far (all items)
            bool run = true;
            int bh, qt;
            for (int item = 0; run && item_of(item, bh, qt); ++item) {
                // Q of the item into its buffer, once the last score product of the item
                // that used that buffer before has read it
                const int qb = item % C::kQBufs, uq = item / C::kQBufs;
                if (uq > 0 &&
                    !mbar_wait(&bars->q_empty[qb], (uq - 1) & 1, kSiteQEmpty, abort))
                    break;
                mbar_arrive_expect_tx(&bars->q_full[qb], C::kTileBytes);
                for (int c = 0; c < C::kChunks; ++c)
                    tma_load_3d(smem + C::kOffQ + qb * C::kTileBytes + c * C::kChunkBytes,
                                &tmap_q, &bars->q_full[qb], 64 * c, qt * kTile, bh);
                last_q[qb] = uq;
                const int n_tiles = tiles_of(qt);
                for (int n = 0; n < n_tiles; ++n, ++g) {
                    const int st = g % C::kStages;
                    const int use = g / C::kStages;
                    if (use > 0 &&
                        !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, kSiteKVEmpty, abort)) {
                        run = false;
                        break;
                    }
                    const int j = causal ? qt - n : n_kvtiles_total - 1 - n;
                    mbar_arrive_expect_tx(&bars->k_full[st], C::kTileBytes);
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffK + st * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_k, &bars->k_full[st], 64 * c, j * kTile, bh);
                    mbar_arrive_expect_tx(&bars->v_full[st], C::kTileBytes);
                    for (int c = 0; c < C::kChunks; ++c)
                        tma_load_3d(smem + C::kOffV + st * C::kTileBytes + c * C::kChunkBytes,
                                    &tmap_v, &bars->v_full[st], 64 * c, j * kTile, bh);
                    last_use[st] = use;
                }
            }
            if (*abort) {
                // let copies already issued land before the CTA's memory is released
                for (int b = 0; b < C::kQBufs; ++b)
                    if (last_q[b] >= 0) mbar_wait_drain(&bars->q_full[b], last_q[b] & 1);
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
        fwd_set_regs<D, F16, false>();
        {
            const uint32_t tO = tmem + C::kColO;
            // bit 13 of the instruction descriptor negates A: S = (-Q) K^T for scale < 0
            const uint32_t idesc_s = C::kIdescS | (negate_scores ? (1u << 13) : 0u);
            // Two cursors walk the CTA's key tiles over all items: the score products
            // run two tiles ahead of the P V products, in the order
            //   S(0) S(1) PV(0) S(2) PV(1) S(3) ...
            // so S(g+1) is in its buffer while the softmax is still on tile g.
            struct Cursor {
                int item, n, n_tiles, g;
                bool valid;
            };
            auto start = [&](Cursor& c) {
                int bh_, qt_;
                c.item = 0;
                c.n = 0;
                c.g = 0;
                c.valid = item_of(0, bh_, qt_);
                c.n_tiles = c.valid ? tiles_of(qt_) : 0;
            };
            auto advance = [&](Cursor& c) {
                ++c.g;
                if (++c.n == c.n_tiles) {
                    int bh_, qt_;
                    ++c.item;
                    c.n = 0;
                    c.valid = item_of(c.item, bh_, qt_);
                    c.n_tiles = c.valid ? tiles_of(qt_) : 0;
                }
            };
            // S(g) = Q K(g)^T into buffer g & 1, once P V(g-2) has read the P there.  An
            // item's first score product is preceded by the copy of its Q from shared
            // into tensor memory (buffer item & 1), after which the shared-memory Q
            // buffer goes back to the producer.  Tensor-memory buffer item & 1 was last
            // read by the score products of item - 2, complete before P V(g-2) (each
            // tile's P V waits for its softmax, which waits for its S).
            auto issue_s = [&](const Cursor& c) -> bool {
                const int g = c.g;
                const int st = g % C::kStages;
                const int qb = c.item % C::kQBufs;
                const uint32_t tQ = tmem + C::kColQ + (c.item & 1) * (D / 2);
                if (c.n == 0) {
                    if (!warp_wait(&bars->q_full[qb], (c.item / C::kQBufs) & 1, kSiteQ, abort))
                        return false;
                    tc_fence_after();
                    const uint32_t q_addr = smem_u32(smem + C::kOffQ + qb * C::kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                        tmem_cp_128x256b_warp(tQ + kk * 8, sdesc_sw128(q_addr + koff, 16, 1024));
                    }
                    mma_commit_warp(&bars->q_empty[qb]);
                }
                if (!warp_wait(&bars->k_full[st], (g / C::kStages) & 1, kSiteKFull, abort))
                    return false;
                if (g >= C::kSBufs &&
                    !warp_wait(&bars->pv_done, (g - C::kSBufs) & 1, kSiteSFree, abort))
                    return false;
                tc_fence_after();
                const uint32_t tS = tmem + C::kColS0 + (g % C::kSBufs) * C::kColBuf;
                const uint32_t k_addr = smem_u32(smem + C::kOffK + st * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * C::kChunkBytes + (kk & 3) * 32;
                    const uint64_t bdesc = sdesc_sw128(k_addr + koff, 16, 1024);
                    mma_ts_warp(tS, tQ + kk * 8, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_warp(&bars->s_full[g % C::kSBufs]);
                return true;
            };
            // O += P(g) V(g).  An item's first P V overwrites O, so it waits until the
            // previous item's epilogue has read O.
            auto issue_pv = [&](const Cursor& c) -> bool {
                const int g = c.g;
                const int st = g % C::kStages;
                if (!warp_wait(&bars->p_full[g % C::kSBufs], (g / C::kSBufs) & 1, kSitePFull,
                               abort))
                    return false;
                if (!warp_wait(&bars->v_full[st], (g / C::kStages) & 1, kSiteVFull, abort))
                    return false;
                if (c.n == 0 && c.item > 0 &&
                    !warp_wait(&bars->o_free, (c.item - 1) & 1, kSiteOFree, abort))
                    return false;
                tc_fence_after();
                const uint32_t tP = tmem + C::kColS0 + (g % C::kSBufs) * C::kColBuf;
                const uint32_t v_addr = smem_u32(smem + C::kOffV + st * C::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    // B = V tile, MN-major: 16 keys = 2 x 8-row groups of 1024 bytes
                    const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, C::kChunkBytes, 1024);
                    mma_ts_warp(tO, tP + kk * 8, bdesc, C::kIdescPV, (c.n > 0 || kk > 0) ? 1u : 0u);
                    if (PRECISE) mma_ts_warp(tO, tP + C::kColPlo + kk * 8, bdesc, C::kIdescPV, 1u);
                }
                mma_commit_warp(&bars->pv_done);
                mma_commit_warp(&bars->kv_empty[st]);
                if (c.n == c.n_tiles - 1) mma_commit_warp(&bars->o_done);
                return true;
            };
            Cursor cs, cp;
            start(cs);
            start(cp);
            bool ok = true;
            for (int i = 0; ok && i < C::kSBufs && cs.valid; ++i) {
                ok = issue_s(cs);
                advance(cs);
            }
            while (ok && cp.valid) {
                ok = issue_pv(cp);
                advance(cp);
                if (ok && cs.valid) {
                    ok = issue_s(cs);
                    advance(cs);
                }
            }
            // every MMA this thread issued must retire before tensor memory is freed
            mma_commit_warp(&bars->mma_final);
            mbar_wait_drain(&bars->mma_final, 0);
        }
    } else if (warp < C::kWarpSoftmax0) {
        fwd_set_regs<D, F16, false>();  // idle: completes the control warpgroup
    } else {
        // ------------------------------------------------------------ softmax
        fwd_set_regs<D, F16, true>();
        const uint32_t row = ((warp & 3) << 5) + lane;  // TMEM lane owned by this thread
        const uint32_t lane_off = ((warp & 3) << 5) << 16;
        const uint32_t tO = tmem + lane_off + C::kColO;
        bool ok = true;
        int g0 = 0;  // key tiles before this item (all items)
        int bh, qt;
        for (int item = 0; ok && item_of(item, bh, qt); ++item) {
        const int n_tiles = tiles_of(qt);
        const int grow = qt * kTile + (int)row;  // query index of this row
        float m_run = -INFINITY;                  // running max, log2 units
        float l_run = 0.f;                        // running sum of exp2(u - m_run)
        for (int n = 0; n < n_tiles; ++n) {
            const int g = g0 + n;
            const int j = causal ? qt - n : n_kvtiles_total - 1 - n;
            const uint32_t tS = tmem + lane_off + C::kColS0 + (g % C::kSBufs) * C::kColBuf;
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[g % C::kSBufs],
                                                   (g / C::kSBufs) & 1, kSiteSFull, abort))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t sraw[kTile];
#pragma unroll
            for (int c = 0; c < kTile / 32; ++c) tmem_ld32(tS + c * 32, sraw + c * 32);
            tmem_wait_ld();

            const bool diag = causal && j == qt;
            const bool tail = !causal && (j + 1) * kTile > T;
            const bool masked_tile = diag || tail;
            const int key_lim = diag ? (int)row : (tail ? T - 1 - j * kTile : kTile - 1);
            float s[kTile];
#pragma unroll
            for (int c = 0; c < kTile; ++c) s[c] = __uint_as_float(sraw[c]);

            // O *= alpha (this thread's row), once O includes P(n-1) V
            auto rescale_o = [&](float alpha) -> bool {
                if (!__all_sync(0xffffffffu,
                                mbar_wait(&bars->pv_done, (g - 1) & 1, kSitePV, abort)))
                    return false;
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
                return true;
            };
            // P = exp2(s * scale_log2 - m_run), its row sum, P packed to bf16 pairs
            // and stored to TMEM over the S it came from (this thread has all of its S
            // row in registers).  With kTrack the same pass also takes the row's raw
            // max (eight independent three-input chains).
            float2 lsum;
            float mraw = -INFINITY;
            auto exp_pass = [&](auto track) {
                constexpr bool kTrack = decltype(track)::value;
                const float2 sl2 = make_float2(scale_log2, scale_log2);
                const float2 nm2 = make_float2(-m_run, -m_run);
                float2 ls[4];
                float mx[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) ls[e] = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
#pragma unroll
                for (int qr = 0; qr < 4; ++qr) {  // 32 keys = 16 columns of P at a time
                    uint32_t pk[16], pl[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c = qr * 32 + 2 * e;
                        if (kTrack) mx[e & 7] = fmax3(mx[e & 7], s[c], s[c + 1]);
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
                        pk[e] = pack16x2<F16>(p.x, p.y);
                        if (PRECISE)
                            pl[e] = pack_bf16x2(p.x - bf16_lo_to_float(pk[e]),
                                                p.y - bf16_hi_to_float(pk[e]));
                    }
                    tmem_st16(tS + qr * 16, pk);
                    if (PRECISE) tmem_st16(tS + C::kColPlo + qr * 16, pl);
                }
                lsum = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
                if (kTrack)
                    mraw = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7]));
            };

            // scale_log2 is >= 0 (a negative scale is applied by negating Q in the MMA),
            // so the max of the scaled scores is scale_log2 times the raw max.
            if (!F16 && n > 1 && !masked_tile) {
                // From an item's third tile on (its first is the only one with masked
                // keys, and after two tiles the running max has seen at least 129 keys
                // of the row) a tile is exponentiated against the running max straight
                // away, taking the tile's max in the same pass: the max is off the
                // critical path.  The result stands unless the tile raises some row's
                // max by more than the lazy-rescale bound; then those rows move to the
                // new max, O is rescaled, and the warp recomputes the tile.  (bf16 P
                // only: under fp16's bound of 2^15 a third of the tiles were recomputed
                // on logits with a 9-nat spread, and the max-first pass below costs
                // less than that.)
                exp_pass(std::true_type{});
                const float mt = mraw * scale_log2;
                const bool need = mt > m_run + kRescaleThreshold<F16>;
                if (__any_sync(0xffffffffu, need)) {
                    float alpha = 1.f;
                    if (need) {
                        alpha = ex2_approx(m_run - mt);
                        m_run = mt;
                        l_run *= alpha;
                    }
                    if (!rescale_o(alpha)) {
                        ok = false;
                        break;
                    }
                    exp_pass(std::false_type{});
                }
            } else {
                // Row max of the raw scores over the keys this row may see, first.
                if (masked_tile) {  // the same for every thread of the CTA
#pragma unroll
                    for (int c = 0; c < kTile; ++c)
                        if (c > key_lim) s[c] = -INFINITY;
                }
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    mx[e] = fmaxf(s[16 * e], s[16 * e + 1]);
#pragma unroll
                    for (int c = 2; c < 16; c += 2)
                        mx[e] = fmax3(mx[e], s[16 * e + c], s[16 * e + c + 1]);
                }
                const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                       fmaxf(mx[6], mx[7])) *
                                 scale_log2;
                float alpha = 1.f;
                bool need = false;
                if (n == 0) {
                    m_run = mt;
                } else if (mt > m_run + kRescaleThreshold<F16>) {
                    need = true;
                    alpha = ex2_approx(m_run - mt);
                    m_run = mt;
                    l_run *= alpha;
                }
                if (n > 0 && __any_sync(0xffffffffu, need) && !rescale_o(alpha)) {
                    ok = false;
                    break;
                }
                exp_pass(std::false_type{});
            }
            l_run += lsum.x + lsum.y;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[g % C::kSBufs]);
        }

        if (!ok) break;
        g0 += n_tiles;

        // ----------------------------------------------------------- epilogue
        // O straight from tensor memory to global memory: each thread writes its
        // own row (d contiguous elements).
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, item & 1, kSiteODone, abort))) {
            ok = false;
            break;
        }
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        if (grow < T) lse_out[(size_t)bh * T + grow] = (m_run + log2f(l_run)) * kLn2;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);  // all lanes: the load is warp-collective
            tmem_wait_ld();
            if (grow < T) {
                const size_t base = ((size_t)bh * T + grow) * D + c * 32;
                if (o_f32) {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o_out) + base);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l,
                                             __uint_as_float(r[4 * e + 1]) * inv_l,
                                             __uint_as_float(r[4 * e + 2]) * inv_l,
                                             __uint_as_float(r[4 * e + 3]) * inv_l);
                } else {
                    uint4* dst =
                        reinterpret_cast<uint4*>(static_cast<uint16_t*>(o_out) + base);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(pack16x2<F16>(__uint_as_float(r[8 * e]) * inv_l,
                                                          __uint_as_float(r[8 * e + 1]) * inv_l),
                                            pack16x2<F16>(__uint_as_float(r[8 * e + 2]) * inv_l,
                                                          __uint_as_float(r[8 * e + 3]) * inv_l),
                                            pack16x2<F16>(__uint_as_float(r[8 * e + 4]) * inv_l,
                                                          __uint_as_float(r[8 * e + 5]) * inv_l),
                                            pack16x2<F16>(__uint_as_float(r[8 * e + 6]) * inv_l,
                                                          __uint_as_float(r[8 * e + 7]) * inv_l));
                }
            }
        }
        // the next item's first P V may now overwrite O
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->o_free);
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

template <int D, bool PRECISE, bool F16>
cudaError_t launch_fwd_dp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          void* o, float* lse, int BH, int T, float scale, int causal, int o_f32,
                          cudaStream_t stream) {
    using C = FwdCfg<D, F16>;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e =
        set_max_dynamic_smem(attn_fwd_kernel<D, PRECISE, F16>, C::kSmemBytes, configured);
    if (e != cudaSuccess) return e;
    const int n_qtiles = (T + kTile - 1) / kTile;
    const int n_items = BH * n_qtiles;
    const int slots = sm_count() * C::kCtasPerSM;
    const int grid = n_items < slots ? n_items : slots;
    return launch_dependent(attn_fwd_kernel<D, PRECISE, F16>, dim3(grid), dim3(C::kThreads),
                            C::kSmemBytes, stream, tq, tk, tv, o, lse, T, BH, n_qtiles, n_items,
                            fabsf(scale) * kLog2e, scale < 0.f ? 1 : 0, causal, o_f32);
}

template <int D>
cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         void* o, float* lse, int BH, int T, float scale, int causal, int o_f32,
                         int precise, int f16, cudaStream_t stream) {
    if (f16)
        return launch_fwd_dp<D, false, true>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32,
                                             stream);
    if (precise)
        return launch_fwd_dp<D, true, false>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32,
                                             stream);
    return launch_fwd_dp<D, false, false>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32, stream);
}

}  // namespace

cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            void* o, float* lse, int BH, int T, int d, float scale, int causal,
                            int o_f32, int precise, int f16, cudaStream_t stream) {
    if (d == 64)
        return launch_fwd_d<64>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32, precise, f16,
                                stream);
    return launch_fwd_d<128>(tq, tk, tv, o, lse, BH, T, scale, causal, o_f32, precise, f16,
                             stream);
}

cudaError_t read_and_clear_device_error_fwd(unsigned int* value) {
    return read_and_clear_unit_error(value);
}

}  // namespace forge

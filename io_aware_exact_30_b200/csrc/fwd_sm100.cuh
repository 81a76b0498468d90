// Forward kernel: exact attention, two 128-row query tiles per CTA sharing
// each 128-key tile of K and V streamed through a TMA pipeline; scores and
// outputs accumulate in tensor memory through tcgen05 MMAs; softmax
// statistics live per row in registers and follow the online (running max /
// running sum) recurrence.
//
// Method: "Is a full day of context better than ten minutes? FlashAttention
// and the sequence-length question" (marketmaker.cc), sections "Flash
// Attention algorithm" (tiles of Q, K, V staged on chip, S_ij and P_ij never
// leave it), "online softmax recurrence" (the accumulator is rescaled by
// exp(m_old - m_new) when the running max grows), "FA2: parallelism"
// (normalise by the running sum once, after the last tile; parallel over
// query tiles; one thread owns one query row so there is no cross-warp
// reduction), "FA3: Hopper" (asynchronous producer and consumer warps; the
// matmul of one block overlaps the softmax of another) and "causal masking"
// (key tiles wholly in the future of a query tile are neither loaded for it
// nor computed; only diagonal tiles are masked element-wise).  The row
// statistic written out is the log-sum-exp — "Performance optimisation with
// Flash-Attention 2" (Medium), section "Flash Attention 2".
//
// B200 form:
//  - Two query tiles (2p, 2p+1) per CTA, each with its own softmax warpgroup;
//    while one group exponentiates its tile, the tensor core computes the
//    other tile's S = Q K^T or P V, so MMA and MUFU work overlap.
//  - P is written back into tensor memory over its S (half precision, two
//    values per 32-bit column) and is the A operand of O += P V, so P never
//    touches shared memory.
//  - The max used for the exponent is only moved (and O rescaled) when the
//    row max grows by more than 2^8; otherwise the stale max is kept.  Every
//    exponent and the final normaliser use the same max, so the result is
//    the same softmax; values stay below 2^8 times their normalised size.
//  - The per-element arithmetic uses the packed fp32x2 instructions; the
//    exponentials stay on the multi-function unit (measured: moving a share
//    of them to a polynomial on the FMA pipe costs more issue slots than it
//    saves here).
//
// Roles (320 threads): warps 0-3 softmax of tile 0, warps 4-7 softmax of tile
// 1 (thread t of a group owns query row t = TMEM lane t), warp 8 TMA
// producer, warp 9 TMEM owner and MMA issuer.
// Tensor memory: S of tile i at column 128 i, O of tile i at 256 + D i; P of
// tile i over its S (d = 128) or, at d = 64, in columns 384 + 64 i of its own.
#pragma once

#include "dropout.cuh"
#include "ptx.cuh"

namespace attn {

struct FwdParams {
    void* o;
    float* lse;
    int BH;
    int N;
    int n_qtiles;
    int n_pairs;         // query-tile pairs per head
    int group;           // heads per scheduling group (their K/V fit in L2)
    int causal;
    float scale_log2;    // scale * log2(e)
    // Block-sparse attention: n_qtiles x n_ktiles bytes, nonzero where query
    // tile i may attend to key tile j (128 x 128 blocks, one mask for every
    // head); nullptr for dense attention.
    const uint8_t* bmask;
    int n_ktiles;
    // FP8 scores (fp8_sm100.cuh): per-(head, 128-row block) dequantisation
    // scales of the e4m3 Q and K; scale_log2 then also holds the 1/d of the
    // rotation.  nullptr for 16-bit Q and K.
    const float* qscale;
    const float* kscale;
    // Dropout on P (kernels instantiated with DROP only).
    DropoutParams drop;
};

// Persistent schedule.  A work item is (head, pair of query tiles); there are
// BH * n_pairs of them, taken through an ItemStream: dynamically under the
// causal mask or a block mask (unequal costs), in static snake order otherwise.  Heads are taken in groups of
// `group` heads whose K/V fit comfortably in L2 together; within a group the
// items are listed heaviest first — under the causal mask pair p costs 4p + 3
// key-tile steps, so the group's list runs from the last pair down, heads in
// order within a pair; without the mask all items cost the same and the list
// is head-major.
__device__ __forceinline__ void fwd_item(const FwdParams& p, int k, int& bh, int& pair) {
    if (p.causal) {
        const int per_group = p.group * p.n_pairs;
        const int g = k / per_group, i = k % per_group;
        const int heads = min(p.group, p.BH - g * p.group);
        pair = p.n_pairs - 1 - i / heads;
        bh = g * p.group + i % heads;
    } else {
        bh = k / p.n_pairs;
        pair = k % p.n_pairs;
    }
}

// Key tiles of a work item.  Query tile t of the pair attends to key tile j
// iff act(t, j): j below its causal bound and, under a block mask, marked.
// K and V are loaded for the union of both tiles' key tiles, walked in order
// by every role (next() gives the union's next tile); without a mask the
// union is 0 .. nkv - 1.
struct FwdItemShape {
    bool has1;
    int nkv0, nkv1;          // key tiles below each query tile's causal bound
    int nkv;                 // max of the two
    const uint8_t* mrow0;    // mask rows of the two query tiles (nullptr: dense)
    const uint8_t* mrow1;
    // (scalars, not arrays: indexed by a run-time tile they would live in
    // local memory, on the MMA issuer's critical path)
    __device__ FwdItemShape(const FwdParams& p, int pair) {
        const int n_kv_all = (p.N + 127) >> 7;
        has1 = 2 * pair + 1 < p.n_qtiles;
        nkv0 = p.causal ? min(n_kv_all, 2 * pair + 1) : n_kv_all;
        nkv1 = has1 ? (p.causal ? min(n_kv_all, 2 * pair + 2) : n_kv_all) : 0;
        nkv = max(nkv0, nkv1);
        mrow0 = p.bmask ? p.bmask + static_cast<size_t>(2 * pair) * p.n_ktiles : nullptr;
        mrow1 = p.bmask && has1 ? mrow0 + p.n_ktiles : nullptr;
    }
    __device__ int nk(int t) const { return t ? nkv1 : nkv0; }
    __device__ const uint8_t* mrow(int t) const { return t ? mrow1 : mrow0; }
    __device__ bool act(int t, int j) const {
        const uint8_t* m = mrow(t);
        return j < nk(t) && (m == nullptr || m[j] != 0);
    }
    __device__ bool any(int j) const { return act(0, j) || act(1, j); }
    // first union tile at or after j (nkv if none)
    __device__ int from(int j) const {
        if (mrow0 == nullptr) return j;
        while (j < nkv && !any(j)) ++j;
        return j;
    }
    __device__ int first() const { return from(0); }
    __device__ int next(int j) const { return from(j + 1); }
};

template <int D, bool FP8 = false>
struct FwdCfg {
    static constexpr int KB = D / 64;                 // 64-column swizzle blocks per row
    static constexpr uint32_t TILE = 128u * D * 2u;   // bytes of a 128 x D half tile (V)
    // Q and K tiles: half, or e4m3 (one 128- or 64-byte swizzled box per row)
    static constexpr uint32_t QKTILE = FP8 ? 128u * D : TILE;
    static constexpr int STAGES = D == 64 ? 4 : (FP8 ? 3 : 2);
    static constexpr uint32_t OFF_Q = 0;              // two query tiles
    static constexpr uint32_t OFF_K = OFF_Q + 2 * QKTILE;
    static constexpr uint32_t OFF_V = OFF_K + STAGES * QKTILE;
    static constexpr uint32_t OFF_BAR = OFF_V + STAGES * TILE;
    static constexpr int B_Q = 0, B_KF = 1, B_VF = B_KF + STAGES, B_KE = B_VF + STAGES,
                         B_SF = B_KE + STAGES, B_PF = B_SF + 2, B_OD = B_PF + 2, B_DR = B_OD + 2,
                         B_QE = B_DR + 1, B_OE = B_QE + 1, B_CLCF = B_OE + 2, B_CLCE = B_CLCF + 2,
                         NBAR = B_CLCE + 2;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t OFF_CLC = (OFF_MISC + 16 + 15) & ~15u;  // 2 x 16-byte responses
    static constexpr uint32_t SMEM_BYTES = OFF_CLC + 32 + 1024;  // + alignment slack
    // arrivals that free a work-item response: producer, MMA and 8 softmax warps
    static constexpr int CLC_CONSUMERS = 10;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
    // At d = 64, S (256 columns) and O (128) leave 128 columns free: P_t gets
    // columns of its own there, so the next S_t need not wait for P_t V.
    static constexpr bool P_OWN = D == 64;
    static constexpr uint32_t COL_P = 384;
    static constexpr int NTHREADS = 320;
    static constexpr int WARP_TMA = 8, WARP_MMA = 9;
    static_assert(SMEM_BYTES <= 232448u, "dynamic shared memory above the sm_100 per-block limit");
};

// Move the running max (and rescale O) only when the row max grows by more
// than this many binary orders of magnitude.
constexpr float kRescaleThreshold = 8.f;

template <int D, bool BF16, bool FP8 = false, bool DROP = false>
__global__ void __launch_bounds__(320, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D, FP8>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bar0 = base + C::OFF_BAR;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::B_Q), 1);
        mbar_init(BAR(C::B_QE), 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(BAR(C::B_KF + s), 1);
            mbar_init(BAR(C::B_VF + s), 1);
            mbar_init(BAR(C::B_KE + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(BAR(C::B_SF + t), 1);
            mbar_init(BAR(C::B_PF + t), 128);
            mbar_init(BAR(C::B_OD + t), 1);
            mbar_init(BAR(C::B_OE + t), 128);
        }
        mbar_init(BAR(C::B_DR), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(C::B_CLCF + i), 1);
            mbar_init(BAR(C::B_CLCE + i), C::CLC_CONSUMERS);
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc(base + C::OFF_MISC, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    ItemStream cs(p.causal != 0 || p.bmask != nullptr, p.BH * p.n_pairs, base + C::OFF_CLC,
                  BAR(C::B_CLCF), BAR(C::B_CLCE));

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued[C::STAGES];
#pragma unroll
            for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
            int kv = 0, items = 0, bh, pair;
            bool ok = true;
            // once an item's loads are issued, ask for the next item
            for (; ok && cs.cur >= 0;
                 ok = ok && cs.request(abort_flag) && cs.advance(abort_flag, false)) {
                fwd_item(p, cs.cur, bh, pair);
                const FwdItemShape sh(p, pair);
                // the previous item's S MMAs are done reading the query tiles
                if (items > 0 && !(ok = wait_bounded(BAR(C::B_QE), (items - 1) & 1, abort_flag)))
                    break;
                mbar_arrive_expect_tx(BAR(C::B_Q), sh.has1 ? 2 * C::QKTILE : C::QKTILE);
                for (int t = 0; t < (sh.has1 ? 2 : 1); ++t) {
                    if constexpr (FP8) {
                        tma_load_3d(base + C::OFF_Q + t * C::QKTILE, &tmQ, BAR(C::B_Q), 0,
                                    (2 * pair + t) * 128, bh);
                    } else {
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb)
                            tma_load_3d(base + C::OFF_Q + t * C::QKTILE + kb * 16384u, &tmQ,
                                        BAR(C::B_Q), kb * 64, (2 * pair + t) * 128, bh);
                    }
                }
                ++items;
                for (int j = sh.first(); j < sh.nkv; j = sh.next(j), ++kv) {
                    const int s = kv % C::STAGES, n = kv / C::STAGES;
                    if (!(ok = wait_bounded(BAR(C::B_KE + s), (n & 1) ^ 1, abort_flag))) break;
                    const uint32_t sk = base + C::OFF_K + s * C::QKTILE;
                    const uint32_t sv = base + C::OFF_V + s * C::TILE;
                    mbar_arrive_expect_tx(BAR(C::B_KF + s), C::QKTILE);
                    if constexpr (FP8) {
                        tma_load_3d(sk, &tmK, BAR(C::B_KF + s), 0, j * 128, bh);
                    } else {
#pragma unroll
                        for (int kb = 0; kb < C::KB; ++kb)
                            tma_load_3d(sk + kb * 16384u, &tmK, BAR(C::B_KF + s), kb * 64, j * 128,
                                        bh);
                    }
                    mbar_arrive_expect_tx(BAR(C::B_VF + s), C::TILE);
#pragma unroll
                    for (int kb = 0; kb < C::KB; ++kb)
                        tma_load_3d(sv + kb * 16384u, &tmV, BAR(C::B_VF + s), kb * 64, j * 128, bh);
                    issued[s] = n + 1;
                }
            }
            if (*abort_flag) {  // let every copy in flight land before the CTA exits
                cs.drain();
                if (items > 0) wait_drain(BAR(C::B_Q), (items - 1) & 1);
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued[s] > 0) {
                        wait_drain(BAR(C::B_KF + s), (issued[s] - 1) & 1);
                        wait_drain(BAR(C::B_VF + s), (issued[s] - 1) & 1);
                    }
            }
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------------- MMA issuer
        // Order per key tile j: O_0 += P_0 V_j, S_0 = Q_0 K_{j+1}^T,
        // O_1 += P_1 V_j, S_1 = Q_1 K_{j+1}^T; each S is issued once the P V
        // that reads the same tensor-memory columns has completed, without
        // waiting for the other tile's softmax.  Phase parities come from
        // running counts across the CTA's work items.
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_f16(BF16, 128, 128, false, false);
            constexpr uint32_t ID_S8 = idesc_f16(false, 128, 128, false, false);  // e4m3 x e4m3
            constexpr uint32_t ID_O = idesc_f16(BF16, 128, D, false, true);
            auto issue_s = [&](int t, int kvi) {
                const uint32_t sq = base + C::OFF_Q + t * C::QKTILE;
                const uint32_t sk = base + C::OFF_K + (kvi % C::STAGES) * C::QKTILE;
                if constexpr (FP8) {
                    // e4m3 rows of D bytes, one swizzled box: K = 32 per step, 32 bytes
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        const uint32_t off = kk * 32u;
                        if constexpr (D == 128)
                            mma_ss_f8(tmem + t * 128u, sdesc_sw128(sq + off, 16, 1024),
                                      sdesc_sw128(sk + off, 16, 1024), ID_S8, kk > 0 ? 1u : 0u);
                        else
                            mma_ss_f8(tmem + t * 128u, sdesc_sw64(sq + off, 16, 512),
                                      sdesc_sw64(sk + off, 16, 512), ID_S8, kk > 0 ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_ss(tmem + t * 128u, sdesc_sw128(sq + off, 16, 1024),
                               sdesc_sw128(sk + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(BAR(C::B_SF + t));
            };
            int kv = 0, items = 0, n_pv[2] = {0, 0}, n_done[2] = {0, 0}, bh, pair;
            bool ok = true;
            for (; ok && cs.cur >= 0; ok = ok && cs.advance(abort_flag, false)) {
                fwd_item(p, cs.cur, bh, pair);
                const FwdItemShape sh(p, pair);
                const int j0 = sh.first();
                // Q of this item, K of its first key tile, and for each tile t
                // that starts there the last P_t V issued (in any earlier item),
                // which read the columns S_t is about to take.  Waits test all
                // their barriers at once: a dependent wait stalls the issue of
                // queued MMAs, so one stall per group.
                const bool a0 = j0 < sh.nkv && sh.act(0, j0), a1 = j0 < sh.nkv && sh.act(1, j0);
                const bool w0 = !C::P_OWN && a0 && n_pv[0] > 0,
                           w1 = !C::P_OWN && a1 && n_pv[1] > 0;
                if (!(ok = wait3(BAR(C::B_Q), items & 1, true, BAR(C::B_KF + kv % C::STAGES),
                                 (kv / C::STAGES) & 1, j0 < sh.nkv, BAR(C::B_OD), (n_pv[0] - 1) & 1,
                                 w0, abort_flag)))
                    break;
                if (w1 && !(ok = wait_bounded(BAR(C::B_OD + 1), (n_pv[1] - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                if (a0) issue_s(0, kv);
                if (a1) issue_s(1, kv);
                int fresh = 3;  // bit t: no P_t V of this item issued yet
                int u = 0;                        // union key tiles of this item so far
                for (int j = j0, jn; ok && j < sh.nkv; j = jn, ++u) {
                    jn = sh.next(j);
                    const int kvj = kv + u;
                    const int s = kvj % C::STAGES, n = kvj / C::STAGES;
                    const uint32_t sv = base + C::OFF_V + s * C::TILE;
                    const int k1 = kvj + 1;
                    bool k_next = false;  // K of the next union tile has landed
                    for (int t = 0; ok && t < 2; ++t) {
                        const bool act = sh.act(t, j);
                        const bool nxt = jn < sh.nkv && sh.act(t, jn);  // S_t of the next union tile
                        if constexpr (C::P_OWN) {
                            // P in columns of its own: the next S_t goes out first,
                            // as soon as P-ready shows the softmax is done with S_t
                            // (and its K has landed), ahead of this P_t V; the
                            // softmax waits for that P V before it writes P_t again
                            if (!(ok = wait3(BAR(C::B_VF + s), n & 1, t == 0, BAR(C::B_PF + t),
                                             n_pv[t] & 1, act, BAR(C::B_KF + k1 % C::STAGES),
                                             (k1 / C::STAGES) & 1, nxt && !k_next, abort_flag)))
                                break;
                            if (nxt) {
                                k_next = true;
                                tc_fence_after();
                                issue_s(t, k1);
                            }
                            // the previous epilogue's read of O_t, which the item's
                            // first P_t V overwrites
                            if (act && ((fresh >> t) & 1) && n_done[t] > 0 &&
                                !(ok = wait_bounded(BAR(C::B_OE + t), (n_done[t] - 1) & 1, abort_flag)))
                                break;
                        } else {
                            // V_j (first tile only), P_t, and at the item's first P_t V
                            // the previous epilogue's read of O_t, which P_t V overwrites
                            if (!(ok = wait3(BAR(C::B_VF + s), n & 1, t == 0, BAR(C::B_PF + t),
                                             n_pv[t] & 1, act, BAR(C::B_OE + t), (n_done[t] - 1) & 1,
                                             act && ((fresh >> t) & 1) && n_done[t] > 0, abort_flag)))
                                break;
                        }
                        if (act) {
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ts(tmem + C::COL_O + t * D,
                                       tmem + (C::P_OWN ? C::COL_P + t * 64u : t * 128u) + kk * 8u,
                                       sdesc_sw128(sv + kk * 2048u, 16384, 1024), ID_O,
                                       (!((fresh >> t) & 1) || kk > 0) ? 1u : 0u);
                            mma_commit(BAR(C::B_OD + t));
                            ++n_pv[t];
                            fresh &= ~(1 << t);
                        }
                        if (!C::P_OWN && nxt) {
                            // S_t of the next union tile, into the columns the last
                            // P_t V read once it has completed
                            if (!(ok = wait3(BAR(C::B_OD + t), (n_pv[t] - 1) & 1, n_pv[t] > 0,
                                             BAR(C::B_KF + k1 % C::STAGES), (k1 / C::STAGES) & 1,
                                             !k_next, 0u, 0u, false, abort_flag)))
                                break;
                            k_next = true;
                            tc_fence_after();
                            issue_s(t, k1);
                        }
                    }
                    if (!ok) break;
                    mma_commit(BAR(C::B_KE + s));
                }
                if (!ok) break;
                mma_commit(BAR(C::B_QE));  // every S of this item is issued
                kv += u;
                ++items;
                for (int t = 0; t < 2; ++t)
                    if (!((fresh >> t) & 1)) ++n_done[t];
            }
            if (*abort_flag) {  // every issued MMA must finish before TMEM is freed
                mma_commit(BAR(C::B_DR));
                wait_drain(BAR(C::B_DR), 0);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax
        const int t = warp >> 2;          // query tile of this warpgroup
        const int r = threadIdx.x & 127;  // row of the tile == TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t colS = t * 128u, colO = C::COL_O + t * D;
        // where P_t is written (at d = 64 its own columns, last read by the
        // previous P_t V, which the softmax waits for first)
        const uint32_t colP = C::P_OWN ? C::COL_P + t * 64u : colS;
        int n_s = 0, bh, pair;  // S tiles of this query-tile slot seen so far
        bool ok = true;
        for (; ok && cs.cur >= 0; ok = ok && cs.advance(abort_flag, true)) {
            fwd_item(p, cs.cur, bh, pair);
            int my_nkv;
            const uint8_t* my_row;  // this tile's block-mask row (nullptr: dense)
            {
                const FwdItemShape sh(p, pair);
                my_nkv = sh.nk(t);
                my_row = sh.mrow(t);
            }
            if (my_nkv == 0) continue;  // the pair has no second tile
            const int qrow = (2 * pair + t) * 128 + r;
            float sl_q = p.scale_log2;  // score multiplier (log2 units), times the Q block scale
            if constexpr (FP8) sl_q *= p.qscale[static_cast<size_t>(bh) * p.n_qtiles + 2 * pair + t];
            float m = -INFINITY, l = 0.f;
            int seen = 0;  // key tiles of this item this tile has processed
            for (int j = 0; j < my_nkv; ++j) {
                if (my_row != nullptr && my_row[j] == 0) continue;
                float sl = sl_q;
                if constexpr (FP8) sl *= p.kscale[static_cast<size_t>(bh) * p.n_ktiles + j];
                ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF + t), n_s & 1, abort_flag));
                if (!ok) break;
                ++n_s;
                // (P in columns of its own) the last P_t V has completed
                bool pv_done = !C::P_OWN || n_s < 2;
                tc_fence_after();
                // keys at or past N, and (causal) keys after this query, are masked
                const int key0 = j * 128;
                int limit = p.N - key0;
                if (p.causal) limit = min(limit, qrow - key0 + 1);
                // tiles without masked columns (all but diagonal and tail tiles)
                // take the unmasked path
                const bool full = __all_sync(0xffffffffu, limit >= 128);
                const uint64_t sl2 = f2(sl, sl);
                // P for the 32 keys of chunk c: 2^(s sl - m), masked keys 0, dropped
                // keys 0 in P but kept in the row sum; xmax gathers the largest
                // exponent s sl - m of the unmasked keys
                auto exp_chunk = [&](const uint32_t(&cur)[32], int c, uint64_t negm2,
                                     uint64_t& sum2, float& xmax, uint32_t(&pk)[16]) {
                    // dropout: keep masks (0xFF bytes) of this chunk's 32 keys
                    uint32_t kw[8];
                    if constexpr (DROP) {
                        if (p.drop.thr < 256u) {
                            const uint32_t g = static_cast<uint32_t>(key0 + 32 * c) / 16u;
                            const uint4 a = dropout_bytes16(p.drop, bh, qrow, g);
                            const uint4 b = dropout_bytes16(p.drop, bh, qrow, g + 1u);
                            const uint32_t thr4 = p.drop.thr * 0x01010101u;
                            kw[0] = keep_bytes(a.x, thr4), kw[1] = keep_bytes(a.y, thr4);
                            kw[2] = keep_bytes(a.z, thr4), kw[3] = keep_bytes(a.w, thr4);
                            kw[4] = keep_bytes(b.x, thr4), kw[5] = keep_bytes(b.y, thr4);
                            kw[6] = keep_bytes(b.z, thr4), kw[7] = keep_bytes(b.w, thr4);
                        } else {
#pragma unroll
                            for (int u = 0; u < 8; ++u) kw[u] = 0xFFFFFFFFu;
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        uint64_t x = fma2(f2(__uint_as_float(cur[2 * q]), __uint_as_float(cur[2 * q + 1])),
                                          sl2, negm2);
                        if (!full) {
                            float2 xv = unf2(x);
                            if (c * 32 + 2 * q >= limit) xv.x = -INFINITY;
                            if (c * 32 + 2 * q + 1 >= limit) xv.y = -INFINITY;
                            x = f2(xv.x, xv.y);
                        }
                        const float2 xv = unf2(x);
                        xmax = max3(xmax, xv.x, xv.y);
                        const uint64_t pp = f2(ex2(xv.x), ex2(xv.y));
                        sum2 = add2(sum2, pp);
                        float2 pv = unf2(pp);
                        if constexpr (DROP) {  // the row sum keeps the dropped values
                            const uint32_t kb = kw[q >> 1] >> (16 * (q & 1));
                            if (!(kb & 0x1u)) pv.x = 0.f;
                            if (!(kb & 0x100u)) pv.y = 0.f;
                        }
                        pk[q] = pack2<BF16>(pv.x, pv.y);
                    }
                };
                // Past a row's first key tile the kept max usually stands, so the
                // exponentials are taken against it in a single pass that also
                // finds the tile's largest exponent.  The pass stands when no row
                // of the warp exceeds the threshold (exactly when the two-pass
                // form would keep the max); otherwise the two-pass form below
                // redoes the tile.  P is written only once the pass stands, so S
                // is still whole for the redo.
                // (Not with dropout: its keep masks leave no registers for the
                // held P.)
                bool done = false;
                uint64_t sum2 = f2(0.f, 0.f);
                if (!DROP && seen > 0) {
                    const uint64_t negm2 = f2(-m, -m);
                    float xmax = -INFINITY;
                    uint32_t pk[4][16];
                    uint32_t cur[32];
                    tmem_ld32(lane_addr + colS, cur);
                    tmem_ld_wait();
                    reg_fence32(cur);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t nxt[32];
                        if (c < 3) tmem_ld32(lane_addr + colS + (c + 1) * 32u, nxt);
                        exp_chunk(cur, c, negm2, sum2, xmax, pk[c]);
                        if (c < 3) {
                            tmem_ld_wait();
                            reg_fence32(nxt);
#pragma unroll
                            for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
                        }
                    }
                    if (__all_sync(0xffffffffu, !(xmax > kRescaleThreshold))) {
                        if (!pv_done) {
                            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OD + t),
                                                                      (n_s - 2) & 1, abort_flag));
                            if (!ok) break;
                            pv_done = true;
                            tc_fence_after();
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) tmem_st16(lane_addr + colP + c * 16u, pk[c]);
                        done = true;
                    } else {
                        sum2 = f2(0.f, 0.f);
                    }
                }
                if (!done) {
                    // pass 1: row max over the 128 scores (two chunks of 64 in flight)
                    float mx = -INFINITY;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t a[32], b[32];
                        tmem_ld32(lane_addr + colS + h * 64u, a);
                        tmem_ld32(lane_addr + colS + h * 64u + 32u, b);
                        tmem_ld_wait();
                        reg_fence32(a);
                        reg_fence32(b);
                        if (full) {
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                mx = max3(mx, __uint_as_float(a[e]), __uint_as_float(a[e + 1]));
                                mx = max3(mx, __uint_as_float(b[e]), __uint_as_float(b[e + 1]));
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int ca = h * 64 + e, cb = ca + 32;
                                if (ca < limit) mx = fmaxf(mx, __uint_as_float(a[e]));
                                if (cb < limit) mx = fmaxf(mx, __uint_as_float(b[e]));
                            }
                        }
                    }
                    const float m_tile = mx * sl;
                    // Move the max only when it grows past the threshold (the first
                    // tile always sets it); rescaling O needs O(j-1) complete.
                    const bool move = m_tile > m + kRescaleThreshold;
                    if (__any_sync(0xffffffffu, move)) {
                        const float m_new = move ? m_tile : m;
                        const float alpha = ex2(m - m_new);  // 0 on the first tile, 1 if not moved
                        if (seen > 0) {
                            ok = __all_sync(0xffffffffu,
                                            wait_bounded(BAR(C::B_OD + t), (n_s - 2) & 1, abort_flag));
                            if (!ok) break;
                            pv_done = true;
                            tc_fence_after();
#pragma unroll
                            for (int c = 0; c < D / 32; ++c) {
                                uint32_t o[32];
                                tmem_ld32(lane_addr + colO + c * 32u, o);
                                tmem_ld_wait();
                                reg_fence32(o);
#pragma unroll
                                for (int i = 0; i < 32; ++i)
                                    o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                                tmem_st32(lane_addr + colO + c * 32u, o);
                            }
                            tmem_st_wait();
                        }
                        l *= alpha;
                        m = m_new;
                    }
                    // pass 2: P = 2^(s scale log2e - m) chunk by chunk, written back as
                    // half over columns pass 2 has already read (P chunk c -> 16c..16c+15)
                    if (!pv_done) {
                        ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OD + t),
                                                                  (n_s - 2) & 1, abort_flag));
                        if (!ok) break;
                        pv_done = true;
                        tc_fence_after();
                    }
                    const uint64_t negm2 = f2(-m, -m);
                    float xmax = -INFINITY;
                    uint32_t cur[32];
                    tmem_ld32(lane_addr + colS, cur);
                    tmem_ld_wait();
                    reg_fence32(cur);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t nxt[32];
                        if (c < 3) tmem_ld32(lane_addr + colS + (c + 1) * 32u, nxt);
                        uint32_t pk[16];
                        exp_chunk(cur, c, negm2, sum2, xmax, pk);
                        tmem_st16(lane_addr + colP + c * 16u, pk);
                        if (c < 3) {
                            tmem_ld_wait();
                            reg_fence32(nxt);
#pragma unroll
                            for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
                        }
                    }
                }
                const float2 sv2 = unf2(sum2);
                const float sum = sv2.x + sv2.y;
                l += sum;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(BAR(C::B_PF + t));
                ++seen;
            }
            if (ok && seen == 0) {
                // block-sparse: no key tile is marked for this query tile, so no
                // row has a visible key; O = 0 and LSE = -inf (the empty sum)
                if (qrow < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.o) +
                                                          (static_cast<size_t>(bh) * p.N + qrow) *
                                                              (D * 2));
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
                    p.lse[static_cast<size_t>(bh) * p.N + qrow] = -INFINITY;
                }
                continue;
            }
            if (ok)
                ok = __all_sync(0xffffffffu,
                                wait_bounded(BAR(C::B_OD + t), (n_s - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float inv_l = 1.f / l;
            if constexpr (DROP) inv_l *= p.drop.inv_keep;  // kept values are scaled by 256 / t
            uint8_t* orow = static_cast<uint8_t*>(p.o) +
                            (static_cast<size_t>(bh) * p.N + qrow) * (D * 2);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_addr + colO + c * 32u, o);
                tmem_ld_wait();
                reg_fence32(o);
                uint32_t h[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    h[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l,
                                       __uint_as_float(o[2 * i + 1]) * inv_l);
                if (qrow < p.N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
                    dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
                    dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
                    dst[2] = make_uint4(h[8], h[9], h[10], h[11]);
                    dst[3] = make_uint4(h[12], h[13], h[14], h[15]);
                }
            }
            tc_fence_before();
            mbar_arrive(BAR(C::B_OE + t));  // O_t has been read: the next item may overwrite it
            if (qrow < p.N)
                p.lse[static_cast<size_t>(bh) * p.N + qrow] = m * 0.69314718055994531f + logf(l);
        }
    }
#undef BAR
    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn

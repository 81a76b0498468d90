// Backward main kernel for head dimension 128: the same recompute backward as
// attn_bwd_main_kernel (see bwd_sm100.cuh for the method and its sources),
// with 64-query inner tiles so that every accumulator of the tile loop has
// tensor memory of its own and no stage waits for another to be drained.
//
// Persistent: CTAs take (head, 128-key tile j) work items through an
// ItemStream (see bwd_item): dynamically under the causal mask, in static
// snake order otherwise.  For each, K_j and V_j are loaded into shared
// memory and 64-query tiles of Q, dO (and their L2, D statistics) stream
// through a 3-stage pipeline that runs on across items.  Per query tile i:
//   S^T  = K_j Q_i^T                     tensor memory, double-buffered
//   P^T  = exp2(S^T scale log2e - L2_i)  written back over S^T as half
//   dP^T = V_j dO_i^T                    tensor memory
//   dV  += P^T dO_i                      A operand read from tensor memory
//   dS^T = P^T (dP^T - D_i)              shared memory, half, double-buffered
//   dK  += dS^T Q_i
//   dQ^T = K_j^T dS^T                    tensor memory, drained by dQ warps
//                                        into a shared fp32 tile that one bulk
//                                        reduction adds into the accumulator
// At the end of an item dK and dV leave tensor memory through 128-byte-swizzled
// shared boxes (the two dS^T buffers and the dQ staging tile) and TMA tensor
// stores.  A separate small kernel converts the fp32 dQ accumulator to the
// output type after the main kernel.
// Tensor memory (512 columns): S^T buffers at 0 and 64, dP^T at 128, dQ^T at
// 192, dV at 256, dK at 384.
//
// Roles (480 threads): warps 0-7 compute P^T and dS^T (warp w reads TMEM
// lanes 32 (w % 4) .. + 31 and query-column half w / 4 of the 64-wide tile),
// warps 8-11 drain dQ^T (lane = feature) through the shared staging tile into
// the fp32 accumulator, warp 12 TMA producer, warp 13 issues S^T and dP^T (and
// owns the tensor memory), warp 14 issues dV, dK and dQ^T.  A thread that
// issues MMAs stalls at each dependent shared-memory access (a barrier test)
// until its queued MMAs have been handed to the tensor core; with two issuers
// on different SM sub-partitions one keeps the tensor core fed while the other
// waits.
#pragma once

#include "bwd_sm100.cuh"
#include "ptx.cuh"

namespace attn {

struct Bwd128Cfg {
    static constexpr int D = 128;
    static constexpr int QT = 64;                     // query rows per inner tile
    static constexpr uint32_t KTILE = 128u * D * 2u;  // 32 KB: K or V tile
    static constexpr uint32_t QTILE = 64u * D * 2u;   // 16 KB: Q or dO tile
    static constexpr int ST = 3;                      // Q / dO / statistics stages
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = OFF_K + KTILE;
    static constexpr uint32_t OFF_Q = OFF_V + KTILE;
    static constexpr uint32_t OFF_DO = OFF_Q + ST * QTILE;
    static constexpr uint32_t DSTILE = 16384u;                // dS^T: 128 keys x 64 queries half
    static constexpr uint32_t OFF_DST = OFF_DO + ST * QTILE;  // two dS^T buffers
    static constexpr uint32_t OFF_STG = OFF_DST + 2 * DSTILE; // dQ tile, 64 x 128 fp32 rows
                                                              // (also the dV boxes at item end)
    static constexpr uint32_t OFF_LD = OFF_STG + 32768u;      // ST x (64 L2 + 64 D) fp32
    static constexpr uint32_t OFF_BAR = OFF_LD + ST * 512u;
    static constexpr int B_KV = 0, B_QF = 1, B_QE = B_QF + ST, B_SF = B_QE + ST, B_DPF = B_SF + 2,
                         B_PTF = B_DPF + 1, B_DVD = B_PTF + 2, B_DSF = B_DVD + 2,
                         B_DSTE = B_DSF + 2, B_DQF = B_DSTE + 2, B_DQE = B_DQF + 1,
                         B_FIN = B_DQE + 1, B_DR = B_FIN + 1, B_KVE = B_DR + 2, B_ACCE = B_KVE + 1,
                         B_SRD = B_ACCE + 1, B_STGF = B_SRD + 2, B_STGE = B_STGF + 2,
                         B_CLCF = B_STGE + 2, B_CLCE = B_CLCF + 2, B_DPE = B_CLCE + 2,
                         B_EPS = B_DPE + 1, B_EPF = B_EPS + 1, B_DQD = B_EPF + 1,
                         NBAR = B_DQD + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t OFF_CLC = (OFF_MISC + 16 + 15) & ~15u;  // 2 x 16-byte responses
    static constexpr uint32_t SMEM_BYTES = OFF_CLC + 32 + 1024;
    static_assert(SMEM_BYTES <= 232448u, "dynamic shared memory above the sm_100 per-block limit");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 192, COL_DV = 256, COL_DK = 384;
    static constexpr int NCOMPUTE = 256, NDQ = 128;
    // arrivals that free a work-item response: producer, 2 MMA issuers, 8 compute
    // and 4 dQ warps
    static constexpr int CLC_CONSUMERS = 3 + NCOMPUTE / 32 + NDQ / 32;
    static constexpr int NTHREADS = NCOMPUTE + NDQ + 96;
    static constexpr int WARP_DQ0 = NCOMPUTE / 32;
    static constexpr int WARP_TMA = WARP_DQ0 + NDQ / 32, WARP_MMA = WARP_TMA + 1,
                         WARP_MMB = WARP_MMA + 1;
};

// Work item k of the list: (head bh, 128-key tile j).  Under the causal mask
// item (bh, j) costs n_q64 - 2j query tiles, otherwise n_q64.  Heads are taken
// in groups whose K, V, Q and dO fit in L2 together; within a group the items
// are listed heaviest first (j ascending, heads in order within a j) when
// causal, head-major otherwise.
__device__ __forceinline__ void bwd_item(const BwdParams& p, int k, int& bh, int& j) {
    if (p.causal) {
        const int per_group = p.group * p.n_ktiles;
        const int g = k / per_group, i = k % per_group;
        const int heads = min(p.group, p.BH - g * p.group);
        j = i / heads;
        bh = g * p.group + i % heads;
    } else {
        bh = k / p.n_ktiles;
        j = k % p.n_ktiles;
    }
}

// The 64-row query tiles an item (head, key tile j) works through: from the
// causal start on, and with a block mask (SPARSE) only those whose 128-row
// query tile is marked for key tile j.  Every role walks the same sequence.
template <bool SPARSE>
struct Bwd128Tiles {
    int begin, end;      // candidate 64-row tiles [begin, end)
    const uint8_t* col;  // mask column of key tile j (stride n_ktiles)
    int stride;
    __device__ Bwd128Tiles(const BwdParams& p, int j, int n_q64)
        : begin(p.causal ? 2 * j : 0), end(n_q64), col(SPARSE ? p.bmask + j : nullptr),
          stride(p.n_ktiles) {}
    __device__ bool act(int i) const { return !SPARSE || col[(i >> 1) * stride] != 0; }
    __device__ int from(int i) const {
        if constexpr (SPARSE)
            while (i < end && !act(i)) ++i;
        return i;
    }
    __device__ int first() const { return from(begin); }
    __device__ int next(int i) const { return from(i + 1); }
    __device__ int count() const {
        if constexpr (!SPARSE) return end - begin;
        int n = 0;
        for (int i = begin; i < end; ++i) n += act(i);
        return n;
    }
};

template <bool BF16, bool DROP = false, bool SPARSE = false>
__global__ void __launch_bounds__(480, 1)
    attn_bwd_main128_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV,
                            const __grid_constant__ CUtensorMap tmDO,
                            const __grid_constant__ CUtensorMap tmDK,
                            const __grid_constant__ CUtensorMap tmDV, const BwdParams p) {
    using C = Bwd128Cfg;
    constexpr int D = C::D;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_q64 = (p.N + 63) / 64;

    const uint32_t bar0 = base + C::OFF_BAR;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC + 4);
    const float* sLD = reinterpret_cast<const float*>(gbase + C::OFF_LD);

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::B_KV), 1);
        mbar_init(BAR(C::B_KVE), 2);  // one commit from each issuer
        mbar_init(BAR(C::B_ACCE), C::NCOMPUTE);
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(BAR(C::B_QF + s), 1);
            mbar_init(BAR(C::B_QE + s), 2);  // one commit from each issuer
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(C::B_SF + i), 1);
            mbar_init(BAR(C::B_PTF + i), C::NCOMPUTE);
            mbar_init(BAR(C::B_DVD + i), 1);
            mbar_init(BAR(C::B_DR + i), 1);
        }
        mbar_init(BAR(C::B_DPF), 1);
        mbar_init(BAR(C::B_DSF), C::NCOMPUTE);
        mbar_init(BAR(C::B_DSF + 1), C::NCOMPUTE);
        mbar_init(BAR(C::B_DSTE), 1);
        mbar_init(BAR(C::B_DSTE + 1), 1);
        mbar_init(BAR(C::B_DPE), C::NCOMPUTE);
        mbar_init(BAR(C::B_EPS), C::NCOMPUTE);
        mbar_init(BAR(C::B_EPF), 1);
        mbar_init(BAR(C::B_DQD), 1);
        mbar_init(BAR(C::B_DQF), 1);
        mbar_init(BAR(C::B_DQE), C::NDQ);
        mbar_init(BAR(C::B_FIN), 1);
        mbar_init(BAR(C::B_SRD), C::NCOMPUTE / 2);
        mbar_init(BAR(C::B_SRD + 1), C::NCOMPUTE / 2);
        for (int h = 0; h < 2; ++h) {
            mbar_init(BAR(C::B_STGF + h), C::NDQ);
            mbar_init(BAR(C::B_STGE + h), 1);
        }
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
    ItemStream cs(p.causal != 0 || p.bmask != nullptr, p.BH * p.n_ktiles, base + C::OFF_CLC,
                  BAR(C::B_CLCF), BAR(C::B_CLCE));

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            int issued[C::ST];
            for (int s = 0; s < C::ST; ++s) issued[s] = 0;
            int g = 0, items = 0, bh = 0, j = 0;
            bool ok = true;
            // query tile i of head bh (Q, dO and their L2, D rows) into ring slot g % ST
            auto load_tile = [&](int i) -> bool {
                const int s = g % C::ST, n = g / C::ST;
                const size_t ld_row0 = static_cast<size_t>(bh) * p.Np;
                if (!wait_bounded(BAR(C::B_QE + s), (n & 1) ^ 1, abort_flag)) return false;
                const uint32_t sq = base + C::OFF_Q + s * C::QTILE;
                const uint32_t sdo = base + C::OFF_DO + s * C::QTILE;
                const uint32_t sld = base + C::OFF_LD + s * 512u;
                mbar_arrive_expect_tx(BAR(C::B_QF + s), 2 * C::QTILE + 512u);
                tma_load_3d(sq, &tmQ, BAR(C::B_QF + s), 0, i * 64, bh);
                tma_load_3d(sq + 8192u, &tmQ, BAR(C::B_QF + s), 64, i * 64, bh);
                tma_load_3d(sdo, &tmDO, BAR(C::B_QF + s), 0, i * 64, bh);
                tma_load_3d(sdo + 8192u, &tmDO, BAR(C::B_QF + s), 64, i * 64, bh);
                bulk_load(sld, p.l2pad + ld_row0 + i * 64, 256u, BAR(C::B_QF + s));
                bulk_load(sld + 256u, p.dpad + ld_row0 + i * 64, 256u, BAR(C::B_QF + s));
                issued[s] = n + 1;
                ++g;
                return true;
            };
            while (ok && cs.cur >= 0) {
                bwd_item(p, cs.cur, bh, j);
                const Bwd128Tiles<SPARSE> tl(p, j, n_q64);
                const int n_it = tl.count();
                const int pre = min(C::ST, n_it);
                int qi = tl.first();
                // The item's first query tiles go ahead of its K/V, which wait
                // until the previous item's MMAs are done with K and V.  (K and V
                // are loaded even for an item without query tiles: its dK, dV
                // are zero, but the per-item handshakes stay in step.)
                for (int it = 0; ok && it < pre; ++it, qi = tl.next(qi)) ok = load_tile(qi);
                if (!ok) break;
                if (items > 0 && !(ok = wait_bounded(BAR(C::B_KVE), (items - 1) & 1, abort_flag)))
                    break;
                mbar_arrive_expect_tx(BAR(C::B_KV), 2 * C::KTILE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_load_3d(base + C::OFF_K + kb * 16384u, &tmK, BAR(C::B_KV), kb * 64, j * 128,
                                bh);
                    tma_load_3d(base + C::OFF_V + kb * 16384u, &tmV, BAR(C::B_KV), kb * 64, j * 128,
                                bh);
                }
                ++items;
                for (int it = pre; ok && it < n_it; ++it, qi = tl.next(qi)) ok = load_tile(qi);
                // once an item's loads are issued, ask for the next item, and start
                // its K and V on their way into L2 (they are loaded into shared
                // memory only when this item's MMAs release K and V)
                if (ok) ok = cs.request(abort_flag) && cs.advance(abort_flag, false);
                if (ok && cs.cur >= 0) {
                    int nbh, nj;
                    bwd_item(p, cs.cur, nbh, nj);
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb) {
                        tma_prefetch_l2_3d(&tmK, kb * 64, nj * 128, nbh);
                        tma_prefetch_l2_3d(&tmV, kb * 64, nj * 128, nbh);
                    }
                }
            }
            if (*abort_flag) {  // let every copy in flight land before the CTA exits
                cs.drain();
                if (items > 0) wait_drain(BAR(C::B_KV), (items - 1) & 1);
                for (int s = 0; s < C::ST; ++s)
                    if (issued[s] > 0) wait_drain(BAR(C::B_QF + s), (issued[s] - 1) & 1);
            }
        }
    } else if (warp == C::WARP_MMA || warp == C::WARP_MMB) {
        // ------------------------------------------------------ MMA issuers
        // Issuer A (warp 13): S^T(g) and dP^T(g).  Issuer B (warp 14): dV(g),
        // dK(g) and dQ^T(g).  Each waits once per group of MMAs, testing all
        // the group's barriers at once.  Every wait is for the newest phase its
        // barrier can have reached before the waiter's own next commit, so no
        // waiter can fall two phases behind; phase parities run on the tile
        // count g across work items.  Q_g / dO_g and K / V are released by one
        // commit from each issuer.
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_f16(BF16, 128, 64, false, false);   // S^T, dP^T
            constexpr uint32_t ID_KV = idesc_f16(BF16, 128, 128, false, true);  // dV, dK
            constexpr uint32_t ID_DQT = idesc_f16(BF16, 128, 64, true, true);   // dQ^T
            const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sDST = base + C::OFF_DST;
            const bool is_a = warp == C::WARP_MMA;
            int g = 0, items = 0, bh = 0, j = 0;
            bool ok = true;
            // S^T(g) = K Q_g^T into S buffer g & 1
            auto issue_s = [&](int g) {
                const uint32_t sQ = base + C::OFF_Q + (g % C::ST) * C::QTILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 8192u + (kk & 3) * 32u;
                    const uint32_t offk = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem + C::COL_S + (g & 1) * 64u, sdesc_sw128(sK + offk, 16, 1024),
                           sdesc_sw128(sQ + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(C::B_SF + (g & 1)));
            };
            while (ok && cs.cur >= 0) {
                bwd_item(p, cs.cur, bh, j);
                const int n_it = Bwd128Tiles<SPARSE>(p, j, n_q64).count();
                if (is_a) {
                    // the item's K, V; Q_g; dV(g-2), the last reader of S buffer g & 1
                    // (an item without query tiles only waits for its K and V to land)
                    if (!(ok = wait3(BAR(C::B_KV), items & 1, true, BAR(C::B_QF + g % C::ST),
                                     (g / C::ST) & 1, n_it > 0, BAR(C::B_DVD + (g & 1)),
                                     ((g - 2) >> 1) & 1, n_it > 0 && g >= 2, abort_flag)))
                        break;
                    tc_fence_after();
                    if (n_it > 0) issue_s(g);
                    for (int it = 0; ok && it < n_it; ++it, ++g) {
                        const int s = g % C::ST, g1 = g + 1;
                        const bool more = it + 1 < n_it;
                        const uint32_t sDO = base + C::OFF_DO + s * C::QTILE;
                        // dP^T(g) overwrites dP^T(g-1), which the compute warps have
                        // loaded (DPE) before they compute dS^T(g-1); S^T(g+1) needs
                        // Q_{g+1} and dV(g-1) done with S buffer (g+1) & 1
                        if (!(ok = wait3(BAR(C::B_DPE), (g - 1) & 1, g >= 1,
                                         BAR(C::B_QF + g1 % C::ST), (g1 / C::ST) & 1, more,
                                         BAR(C::B_DVD + (g1 & 1)), ((g1 - 2) >> 1) & 1,
                                         more && g1 >= 2, abort_flag)))
                            break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * 8192u + (kk & 3) * 32u;
                            const uint32_t offk = (kk >> 2) * 16384u + (kk & 3) * 32u;
                            mma_ss(tmem + C::COL_DP, sdesc_sw128(sV + offk, 16, 1024),
                                   sdesc_sw128(sDO + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(BAR(C::B_DPF));
                        mma_commit(BAR(C::B_QE + s));  // A's reads of Q_g, dO_g
                        if (more) issue_s(g1);
                    }
                    if (!ok) break;
                    mma_commit(BAR(C::B_KVE));  // A's reads of K, V
                } else {
                    for (int it = 0; ok && it < n_it; ++it, ++g) {
                        const uint32_t ph = g & 1;
                        const int s = g % C::ST;
                        const uint32_t sQ = base + C::OFF_Q + s * C::QTILE;
                        const uint32_t sDO = base + C::OFF_DO + s * C::QTILE;
                        const uint32_t sDS = sDST + (g & 1) * C::DSTILE;
                        // dV += P^T dO: P^T(g) in tensor memory, dO_g landed; the item's
                        // first dV (then dK) overwrites accumulators that the previous
                        // item's epilogue must have read
                        if (!(ok = wait3(BAR(C::B_PTF + (g & 1)), (g >> 1) & 1, true,
                                         BAR(C::B_QF + s), (g / C::ST) & 1, true, BAR(C::B_ACCE),
                                         (items - 1) & 1, it == 0 && items > 0, abort_flag)))
                            break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts(tmem + C::COL_DV, tmem + C::COL_S + (g & 1) * 64u + kk * 8u,
                                   sdesc_sw128(sDO + kk * 2048u, 8192, 1024), ID_KV,
                                   (it > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(BAR(C::B_DVD + (g & 1)));
                        // dK += dS^T Q ; dQ^T = K^T dS^T: dS^T(g) stored, dQ^T(g-1)
                        // drained, the item's K landed
                        if (!(ok = wait3(BAR(C::B_DSF + (g & 1)), (g >> 1) & 1, true, BAR(C::B_DQE),
                                         ph ^ 1, g >= 1,
                                         BAR(C::B_KV), items & 1, it == 0, abort_flag)))
                            break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(tmem + C::COL_DK, sdesc_sw128(sDS + kk * 32u, 16, 1024),
                                   sdesc_sw128(sQ + kk * 2048u, 8192, 1024), ID_KV,
                                   (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tmem + C::COL_DQ, sdesc_sw128(sK + kk * 2048u, 16384, 1024),
                                   sdesc_sw128(sDS + kk * 2048u, 8192, 1024), ID_DQT,
                                   kk > 0 ? 1u : 0u);
                        mma_commit(BAR(C::B_QE + s));  // B's reads of Q_g, dO_g
                        mma_commit(BAR(C::B_DQF));
                        mma_commit(BAR(C::B_DSTE + (g & 1)));  // dS^T(g) no longer read
                    }
                    if (!ok) break;
                    if (n_it == 0) {
                        // No query tile, no MMA: the commits below would land at once.
                        // Wait first for the previous item's accumulator release (the
                        // compute warps are past the previous FIN) and for this item's
                        // K and V (the producer saw the previous KVE complete), so that
                        // neither barrier runs two phases ahead of its waiters.
                        if (!(ok = wait3(BAR(C::B_KV), items & 1, true, BAR(C::B_ACCE),
                                         (items - 1) & 1, items > 0, 0u, 0u, false, abort_flag)))
                            break;
                    }
                    mma_commit(BAR(C::B_FIN));  // dK, dV of this item complete
                    mma_commit(BAR(C::B_KVE));  // B's reads of K
                }
                ++items;
                ok = cs.advance(abort_flag, false);
            }
            if (*abort_flag) {  // every issued MMA must finish before TMEM is freed
                const uint32_t dr = BAR(C::B_DR + (is_a ? 0 : 1));
                mma_commit(dr);
                wait_drain(dr, 0);
            }
        }
        __syncwarp();
    } else if (warp >= C::WARP_DQ0) {
        // --------------------------------------------------------- dQ warps
        // Each tile's dQ^T leaves tensor memory at once (freeing its columns),
        // is scaled and written as row-major fp32 rows into a shared staging
        // tile (lane = feature: one 128-byte row segment per warp store), and
        // one thread adds the whole tile into the fp32 accumulator with a
        // single asynchronous bulk reduction.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // TMEM lane = feature of dQ
        const bool issuer = warp == C::WARP_DQ0 && lane == 0;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t stg = base + C::OFF_STG + r * 4u;
        int g = 0, items = 0, bh = 0, j = 0;
        bool dq_ok = true;
        while (dq_ok && cs.cur >= 0) {
            bwd_item(p, cs.cur, bh, j);
            const Bwd128Tiles<SPARSE> tl(p, j, n_q64);
            const int n_it = tl.count();
            float* acc_head = p.dqacc + static_cast<size_t>(bh) * p.N * D;
            int qi = tl.first();
            for (int it = 0; it < n_it; ++it, ++g, qi = tl.next(qi)) {
                const int q0 = qi * 64;
                if (!(dq_ok = __all_sync(0xffffffffu,
                                         wait_bounded(BAR(C::B_DQF), g & 1, abort_flag))))
                    break;
                tc_fence_after();
                uint32_t v[2][32];
                tmem_ld32(lane_addr + C::COL_DQ, v[0]);
                tmem_ld32(lane_addr + C::COL_DQ + 32u, v[1]);
                tmem_ld_wait();
                reg_fence32(v[0]);
                reg_fence32(v[1]);
                tc_fence_before();
                mbar_arrive(BAR(C::B_DQE));  // the values are in registers: columns free
                if constexpr (SPARSE) {
                    // The block-sparse walk keeps the whole 32 KB tile and one
                    // reduction per tile (measured faster there than the two
                    // halves below, which are faster on the dense walk).  The
                    // previous tile's reduction has finished reading the tile.
                    if (g >= 1 && !(dq_ok = __all_sync(0xffffffffu,
                                                       wait_bounded(BAR(C::B_STGE), (g - 1) & 1,
                                                                    abort_flag))))
                        break;
#pragma unroll
                    for (int e = 0; e < 64; ++e)
                        st_shared_f32(stg + e * 512u, __uint_as_float(v[e >> 5][e & 31]) * p.scale);
                    fence_proxy_async_smem();
                    mbar_arrive(BAR(C::B_STGF));
                    if (issuer) {
                        if (!wait_bounded(BAR(C::B_STGF), g & 1, abort_flag)) {
                            dq_ok = false;
                        } else {
                            const int nq = min(64, p.N - q0);
                            bulk_reduce_add_f32(acc_head + static_cast<size_t>(q0) * D,
                                                base + C::OFF_STG, static_cast<uint32_t>(nq) * 512u);
                            bulk_commit();
                            bulk_wait_read_all();
                            mbar_arrive(BAR(C::B_STGE));
                            if (it + 1 == n_it) mbar_arrive(BAR(C::B_DQD));  // item's staging done
                        }
                    }
                } else {
                // The staging tile goes out in two 16 KB halves of 32 queries, each
                // by its own bulk reduction, so that half 1 is written while half
                // 0's reduction reads: a half is rewritten once the previous tile's
                // reduction of it has read it (the issuer waits for all but its
                // newest bulk group, then releases the half).
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (g >= 1) {
                        if (issuer) {
                            bulk_wait_read_but1();
                            mbar_arrive(BAR(C::B_STGE + h));
                        }
                        if (!(dq_ok = __all_sync(0xffffffffu,
                                                 wait_bounded(BAR(C::B_STGE + h), (g - 1) & 1,
                                                              abort_flag))))
                            break;
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        st_shared_f32(stg + (h * 32 + e) * 512u, __uint_as_float(v[h][e]) * p.scale);
                    fence_proxy_async_smem();
                    mbar_arrive(BAR(C::B_STGF + h));
                    if (issuer) {
                        if (!wait_bounded(BAR(C::B_STGF + h), g & 1, abort_flag)) {
                            dq_ok = false;
                        } else {
                            const int nq = min(32, p.N - q0 - 32 * h);
                            if (nq > 0)
                                bulk_reduce_add_f32(acc_head + static_cast<size_t>(q0 + 32 * h) * D,
                                                    base + C::OFF_STG + h * 16384u,
                                                    static_cast<uint32_t>(nq) * 512u);
                            bulk_commit();
                        }
                    }
                    if (!(dq_ok = __all_sync(0xffffffffu, dq_ok))) break;
                }
                if (dq_ok && issuer && it + 1 == n_it) {
                    bulk_wait_read_all();             // the staging tile is free for
                    mbar_arrive(BAR(C::B_DQD));       // the item's epilogue
                }
                }
                dq_ok = __all_sync(0xffffffffu, dq_ok);
                if (!dq_ok) break;
            }
            // An item without query tiles leaves the staging tile as it was.  Its
            // arrival waits for the previous item's epilogue, which follows the
            // compute warps' wait for the previous one: without it, such items in
            // a row would run this barrier two phases ahead of that wait.
            if (dq_ok && n_it == 0 && issuer) {
                if (items > 0 && !wait_bounded(BAR(C::B_EPF), (items - 1) & 1, abort_flag))
                    dq_ok = false;
                else
                    mbar_arrive(BAR(C::B_DQD));
            }
            dq_ok = __all_sync(0xffffffffu, dq_ok);
            ++items;
            if (dq_ok) dq_ok = cs.advance(abort_flag, true);
        }
        if (issuer) bulk_wait_all();  // every reduction complete before the CTA exits
    } else {
        // ---------------------------------------------------------- compute
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;  // TMEM lane = key row of the tile
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const float sl = p.scale_log2;
        const uint32_t sDST = base + C::OFF_DST;
        const int c0 = half * 32;  // first query column of this thread's half
        int g = 0, items = 0, bh = 0, j = 0;
        bool ok = true;
        while (ok && cs.cur >= 0) {
            bwd_item(p, cs.cur, bh, j);
            const Bwd128Tiles<SPARSE> tl(p, j, n_q64);
            const int n_it = tl.count();
            const int key = j * 128 + r;
            const bool key_valid = key < p.N;
            int qi = tl.first();
            for (int it = 0; it < n_it; ++it, ++g, qi = tl.next(qi)) {
                const int q0 = qi * 64;
                const uint32_t ph = g & 1;
                const int s = g % C::ST;
                const float4* L4 = reinterpret_cast<const float4*>(sLD + s * 128 + c0);
                const float4* D4 = reinterpret_cast<const float4*>(sLD + s * 128 + 64 + c0);
                const uint32_t colS = C::COL_S + (g & 1) * 64u;

                // ---- P^T = exp2(S^T scale log2e - L2), written back over S^T
                // (wait on the load barrier too: it makes the bulk-copied L2/D visible)
                ok = __all_sync(0xffffffffu,
                                wait_bounded(BAR(C::B_QF + s), (g / C::ST) & 1, abort_flag));
                if (ok)
                    ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF + (g & 1)), (g >> 1) & 1,
                                                              abort_flag));
                if (!ok) break;
                tc_fence_after();
                float pv[32];
                uint32_t kw[8];  // dropout keep masks of the 32 query columns (bytes)
                {
                    uint32_t sv[32];
                    tmem_ld32(lane_addr + colS + c0, sv);
                    tmem_ld_wait();
                    reg_fence32(sv);
                    // half 1 writes P^T over columns half 0 reads.  One barrier per
                    // S buffer: half 0 cannot arrive for tile g + 2 before S^T(g+2),
                    // which waits for dV(g), which waits for half 1's P^T(g).
                    if (half == 0) {
                        tc_fence_before();
                        mbar_arrive(BAR(C::B_SRD + (g & 1)));
                    }
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 l4 = L4[e4];
                        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            pv[4 * e4 + e] =
                                ex2(fmaf(__uint_as_float(sv[4 * e4 + e]), sl, -lv[e]));
                    }
                    // query q0 + c0 + c sees key j*128 + r iff q0 + c0 + c >= key
                    if (!key_valid || (p.causal && q0 < (j + 1) * 128)) {
                        const int lo = key_valid ? key - q0 - c0 : 32;
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (c < lo) pv[c] = 0.f;
                    }
                    uint32_t pk[16];
                    if constexpr (DROP) {
                        // P^T for dV without the dropped values (256 / t is applied to
                        // dV at the end); dS below uses P and the masked dP
                        if (p.drop.thr < 256u) {
                            dropout_keep_keyrows(p.drop, bh, q0 + c0, j * 128 + quarter * 32, kw);
                        } else {
#pragma unroll
                            for (int t = 0; t < 8; ++t) kw[t] = 0xFFFFFFFFu;
                        }
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const uint32_t kb = kw[c >> 1] >> (16 * (c & 1));
                            pk[c] = pack2<BF16>((kb & 0x1u) ? pv[2 * c] : 0.f,
                                                (kb & 0x100u) ? pv[2 * c + 1] : 0.f);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) pk[c] = pack2<BF16>(pv[2 * c], pv[2 * c + 1]);
                    }
                    if (half == 1) {
                        ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SRD + (g & 1)),
                                                                  (g >> 1) & 1, abort_flag));
                        tc_fence_after();
                    }
                    if (ok) {
                        tmem_st16(lane_addr + colS + half * 16u, pk);
                        tmem_st_wait();
                    }
                }
                if (!ok) break;
                tc_fence_before();
                mbar_arrive(BAR(C::B_PTF + (g & 1)));

                // ---- dS^T = P^T (dP^T - D), half, into shared-memory buffer g & 1
                // once dK(g-2) and dQ^T(g-2) are done reading it
                ok = __all_sync(0xffffffffu,
                                wait3(BAR(C::B_DPF), ph, true, BAR(C::B_DSTE + (g & 1)),
                                      ((g - 2) >> 1) & 1, g >= 2, 0u, 0u, false, abort_flag));
                if (!ok) break;
                tc_fence_after();
                {
                    uint32_t dpv[32];
                    tmem_ld32(lane_addr + C::COL_DP + c0, dpv);
                    tmem_ld_wait();
                    reg_fence32(dpv);
                    tc_fence_before();
                    mbar_arrive(BAR(C::B_DPE));  // dP^T(g) is in registers: dP^T(g+1) may go
                    float dsv[32];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 d4 = D4[e4];
                        const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float dpe = __uint_as_float(dpv[4 * e4 + e]);
                            if constexpr (DROP)
                                dpe = ((kw[e4] >> (8 * e)) & 1u) ? dpe * p.drop.inv_keep : 0.f;
                            dsv[4 * e4 + e] = pv[4 * e4 + e] * (dpe - dd[e]);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c)  // 16-byte chunks 4 half + c of the 128-byte key row
                        st_shared_v4(sDST + (g & 1) * C::DSTILE + sw128_off(r, half * 4 + c),
                                     pack2<BF16>(dsv[8 * c + 0], dsv[8 * c + 1]),
                                     pack2<BF16>(dsv[8 * c + 2], dsv[8 * c + 3]),
                                     pack2<BF16>(dsv[8 * c + 4], dsv[8 * c + 5]),
                                     pack2<BF16>(dsv[8 * c + 6], dsv[8 * c + 7]));
                }
                fence_proxy_async_smem();
                // one barrier per dS^T buffer: the arrival for tile g + 2 needs
                // dK(g) and dQ^T(g), which issuer B starts only after seeing tile g's
                mbar_arrive(BAR(C::B_DSF + (g & 1)));
            }
            if (ok) ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_FIN), items & 1, abort_flag));
            if (!ok) break;
            // dK_j, dV_j: lane r holds key row j*128 + r, this half's 64 features.
            // TMEM -> registers (rounded), then tensor memory is released.  The rows
            // go through 128-byte-swizzled shared boxes, dK into the two dS^T
            // buffers (all MMAs are done with them) and dV into the dQ staging tile
            // once its last reduction has read it, and leave by TMA tensor stores,
            // which skip rows at or past N.
            tc_fence_after();
            uint32_t hk[32], hv[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t v[32];
                tmem_ld32(lane_addr + C::COL_DK + half * 64u + c * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
                // no query tile was marked for this key tile: dK = dV = 0 (the
                // accumulators still hold an earlier item's values)
                if (n_it == 0)
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    hk[16 * c + e] = pack2<BF16>(__uint_as_float(v[2 * e]) * p.scale,
                                                 __uint_as_float(v[2 * e + 1]) * p.scale);
                tmem_ld32(lane_addr + C::COL_DV + half * 64u + c * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
                if (n_it == 0)
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0u;
                const float mv = DROP ? p.drop.inv_keep : 1.f;  // kept P scaled by 256 / t
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    hv[16 * c + e] = pack2<BF16>(__uint_as_float(v[2 * e]) * mv,
                                                 __uint_as_float(v[2 * e + 1]) * mv);
            }
            // dK and dV have been read: the next item may overwrite them
            tc_fence_before();
            mbar_arrive(BAR(C::B_ACCE));
            // The item's last dQ reduction has read the staging tile.  (A parity
            // wait is only valid for a phase whose predecessor has completed; the
            // dQ warps may be two tiles behind here, so the per-tile barrier
            // cannot be used and the per-item one, waited in order, is.)
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_DQD), items & 1, abort_flag));
            if (!ok) break;
            {
                const uint32_t boxk = base + C::OFF_DST + half * C::DSTILE;
                const uint32_t boxv = base + C::OFF_STG + half * 16384u;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    st_shared_v4(boxk + sw128_off(r, c), hk[4 * c], hk[4 * c + 1], hk[4 * c + 2],
                                 hk[4 * c + 3]);
                    st_shared_v4(boxv + sw128_off(r, c), hv[4 * c], hv[4 * c + 1], hv[4 * c + 2],
                                 hv[4 * c + 3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(BAR(C::B_EPS));
            if (threadIdx.x == 0 && wait_bounded(BAR(C::B_EPS), items & 1, abort_flag)) {
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_store_3d(&tmDK, base + C::OFF_DST + kb * C::DSTILE, kb * 64, j * 128, bh);
                    tma_store_3d(&tmDV, base + C::OFF_STG + kb * 16384u, kb * 64, j * 128, bh);
                }
                bulk_commit();
                bulk_wait_read_all();  // the shared boxes may be reused
                mbar_arrive(BAR(C::B_EPF));
            }
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_EPF), items & 1, abort_flag));
            if (!ok) break;
            ++items;
            ok = cs.advance(abort_flag, true);
        }
        if (threadIdx.x == 0) bulk_wait_all();  // every dK/dV store complete before the CTA exits
    }
#undef BAR
    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// dq = dQ accumulator (fp32, scale already applied) rounded to the output type.
template <bool BF16>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float4* __restrict__ acc,
                                                                  uint2* __restrict__ dq,
                                                                  long long n4) {
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n4;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float4 x = acc[e];
        dq[e] = make_uint2(pack2<BF16>(x.x, x.y), pack2<BF16>(x.z, x.w));
    }
}

inline bool bwd128_set_attributes() {
    return cudaFuncSetAttribute(attn_bwd_main128_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_main128_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_main128_kernel<true, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_main128_kernel<false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_main128_kernel<true, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess &&
           cudaFuncSetAttribute(attn_bwd_main128_kernel<false, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Bwd128Cfg::SMEM_BYTES) == cudaSuccess;
}

// mq, mdo must be tensor maps with 64-row boxes; mk, mv, mdk, mdv with 128-row boxes.
// Launches the persistent main kernel, then the dQ conversion.  Causal: one CTA
// per work item, running CTAs take pending CTAs' items; otherwise one CTA per
// multiprocessor.
template <bool BF16>
int bwd_main128_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv,
                       void* dq, void* dk, void* dv, void* ws, int B, int H, int N, int causal,
                       float scale, int sm_count, cudaStream_t st,
                       const uint8_t* bmask = nullptr, const DropoutParams* drop = nullptr) {
    BwdParams p;
    p.bmask = bmask;
    if (drop) p.drop = *drop;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.l2pad = reinterpret_cast<const float*>(w);
    p.dpad = reinterpret_cast<const float*>(w + bwd_ws_off_d(B, H, N));
    p.dqacc = reinterpret_cast<float*>(w + bwd_ws_off_dq(B, H, N));
    p.counters = reinterpret_cast<int*>(w + bwd_ws_off_cnt(B, H, N, 128));
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.BH = B * H;
    p.N = N;
    p.Np = static_cast<int>(bwd_np(N));
    p.n_qtiles = (N + 63) / 64;
    p.n_ktiles = (N + 127) / 128;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    {
        // heads whose K, V, Q and dO together take at most about 96 MB of the
        // 126 MB L2 (measured faster than 48 MB, and than 24 MB or all heads)
        const long long per_head = 4LL * N * 128 * 2;
        const long long g = (96LL << 20) / per_head;
        p.group = static_cast<int>(g < 1 ? 1 : (g > p.BH ? p.BH : g));
    }
    const long long items = 1LL * p.n_ktiles * p.BH;
    if (items >= (1LL << 31)) return -2;
    const bool dynamic = causal || bmask != nullptr;
    const int nblocks = static_cast<int>(dynamic || items < sm_count ? items : sm_count);
    if (drop)
        attn_bwd_main128_kernel<BF16, true><<<static_cast<unsigned>(nblocks), Bwd128Cfg::NTHREADS,
                                              Bwd128Cfg::SMEM_BYTES, st>>>(mq, mk, mv, mdo, mdk,
                                                                           mdv, p);
    else if (bmask)
        attn_bwd_main128_kernel<BF16, false, true><<<static_cast<unsigned>(nblocks),
                                                     Bwd128Cfg::NTHREADS, Bwd128Cfg::SMEM_BYTES,
                                                     st>>>(mq, mk, mv, mdo, mdk, mdv, p);
    else
        attn_bwd_main128_kernel<BF16><<<static_cast<unsigned>(nblocks), Bwd128Cfg::NTHREADS,
                                        Bwd128Cfg::SMEM_BYTES, st>>>(mq, mk, mv, mdo, mdk, mdv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        bwd_record_error(e);
        return -7;
    }
    const long long n4 = 1LL * p.BH * N * 128 / 4;
    const long long want = (n4 + 255) / 256;
    const int cblocks = static_cast<int>(want < 4LL * sm_count ? want : 4LL * sm_count);
    attn_bwd_dq_convert_kernel<BF16><<<cblocks, 256, 0, st>>>(
        reinterpret_cast<const float4*>(p.dqacc), static_cast<uint2*>(dq), n4);
    e = cudaGetLastError();
    if (e != cudaSuccess) bwd_record_error(e);
    return e == cudaSuccess ? 0 : -7;
}

}  // namespace attn

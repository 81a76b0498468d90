// Forward kernel: exact attention, one 128-row query tile per CTA, streaming
// 128-key tiles of K and V through a TMA pipeline, scores and output
// accumulated in tensor memory by tcgen05 MMAs, softmax statistics kept per
// row in registers with the online (running max / running sum) recurrence.
//
// Method: "Is a full day of context better than ten minutes? FlashAttention
// and the sequence-length question" (marketmaker.cc), sections "Flash
// Attention algorithm" (tiles of Q, K, V staged on chip, S_ij and P_ij never
// leave it), "online softmax recurrence" (the accumulator is rescaled by
// exp(m_old - m_new) whenever the running max grows), "FA2: parallelism"
// (normalise by the running sum once, after the last tile; parallel over
// query tiles; one thread owns one query row so no cross-warp reduction),
// "FA3: Hopper" (asynchronous producer/consumer warps, the score MMA of one
// block overlapping the softmax of the previous one) and "causal masking"
// (key tiles wholly in the future of the query tile are neither loaded nor
// computed; only the diagonal tile is masked element-wise).  The statistic
// written out is the log-sum-exp — "Performance optimisation with
// Flash-Attention 2" (Medium), section "Flash Attention 2".
//
// Roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t
//   warp 4     TMA producer (one lane)
//   warp 5     TMEM allocator and tcgen05 MMA issuer (one lane)
// Tensor memory (512 columns): S double buffer at columns 0 and 128 (fp32,
// 128 x 128 each), O accumulator at column 256 (fp32, 128 x D).
// Shared memory: Q tile, STAGES x (K tile, V tile), P tile (bf16/fp16,
// 128 x 128), all in the 128-byte-swizzled K-major layout TMA writes.
#pragma once

#include "ptx.cuh"

namespace attn {

struct FwdParams {
    void* o;
    float* lse;
    int BH;
    int N;
    int n_qtiles;
    int causal;
    float scale_log2;  // scale * log2(e)
};

template <int D>
struct FwdCfg {
    static constexpr int KB = D / 64;                 // 64-column swizzle blocks per row
    static constexpr uint32_t TILE = 128u * D * 2u;   // bytes of a 128 x D half tile
    static constexpr int STAGES = 2;
    static constexpr uint32_t P_BYTES = 128u * 128u * 2u;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + TILE;
    static constexpr uint32_t OFF_V = OFF_K + STAGES * TILE;
    static constexpr uint32_t OFF_P = OFF_V + STAGES * TILE;
    static constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
    // barrier indices
    static constexpr int B_Q = 0;
    static constexpr int B_KF = 1;
    static constexpr int B_VF = B_KF + STAGES;
    static constexpr int B_KE = B_VF + STAGES;
    static constexpr int B_SF = B_KE + STAGES;
    static constexpr int B_SE = B_SF + 2;
    static constexpr int B_PF = B_SE + 2;
    static constexpr int B_OD = B_PF + 1;
    static constexpr int B_DR = B_OD + 1;
    static constexpr int NBAR = B_DR + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
    static constexpr int NTHREADS = 192;
};

template <int D, bool BF16>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: head-major, so the CTAs resident at one time share a few
    // heads' K/V in L2; within a head the heaviest query tile (largest index
    // under the causal mask) goes first.
    const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) % p.n_qtiles;
    const int bh = static_cast<int>(blockIdx.x) / p.n_qtiles;
    const int n_kv_all = (p.N + 127) >> 7;
    const int nkv = p.causal ? min(n_kv_all, qt + 1) : n_kv_all;

    const uint32_t bar0 = base + C::OFF_BAR;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::B_Q), 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(BAR(C::B_KF + s), 1);
            mbar_init(BAR(C::B_VF + s), 1);
            mbar_init(BAR(C::B_KE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(C::B_SF + b), 1);
            mbar_init(BAR(C::B_SE + b), 128);
        }
        mbar_init(BAR(C::B_PF), 128);
        mbar_init(BAR(C::B_OD), 1);
        mbar_init(BAR(C::B_DR), 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(base + C::OFF_MISC, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            mbar_arrive_expect_tx(BAR(C::B_Q), C::TILE);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_3d(base + C::OFF_Q + kb * 16384u, &tmQ, BAR(C::B_Q), kb * 64, qt * 128, bh);
            int issued[C::STAGES];
#pragma unroll
            for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::STAGES, n = j / C::STAGES;
                if (!wait_bounded(BAR(C::B_KE + s), (n & 1) ^ 1, abort_flag)) break;
                const uint32_t sk = base + C::OFF_K + s * C::TILE;
                const uint32_t sv = base + C::OFF_V + s * C::TILE;
                mbar_arrive_expect_tx(BAR(C::B_KF + s), C::TILE);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sk + kb * 16384u, &tmK, BAR(C::B_KF + s), kb * 64, j * 128, bh);
                mbar_arrive_expect_tx(BAR(C::B_VF + s), C::TILE);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sv + kb * 16384u, &tmV, BAR(C::B_VF + s), kb * 64, j * 128, bh);
                issued[s] = n + 1;
            }
            if (*abort_flag) {  // let every copy in flight land before the CTA exits
                wait_drain(BAR(C::B_Q), 0);
                for (int s = 0; s < C::STAGES; ++s)
                    if (issued[s] > 0) {
                        wait_drain(BAR(C::B_KF + s), (issued[s] - 1) & 1);
                        wait_drain(BAR(C::B_VF + s), (issued[s] - 1) & 1);
                    }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_f16(BF16, 128, 128, false, false);
            constexpr uint32_t ID_O = idesc_f16(BF16, 128, D, false, true);
            bool ok = wait_bounded(BAR(C::B_Q), 0, abort_flag);
            tc_fence_after();
            for (int j = 0; ok && j <= nkv; ++j) {
                if (j < nkv) {  // S(j) = Q K_j^T into S buffer j & 1
                    const int s = j % C::STAGES, n = j / C::STAGES, b = j & 1, nb = j >> 1;
                    if (!wait_bounded(BAR(C::B_KF + s), n & 1, abort_flag)) break;
                    if (!wait_bounded(BAR(C::B_SE + b), (nb & 1) ^ 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t sq = base + C::OFF_Q, sk = base + C::OFF_K + s * C::TILE;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_ss(tmem + b * 128u, sdesc_sw128(sq + off, 16, 1024),
                               sdesc_sw128(sk + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(BAR(C::B_SF + b));
                }
                if (j >= 1) {  // O += P(j-1) V_{j-1}
                    const int jp = j - 1, sp = jp % C::STAGES, np = jp / C::STAGES;
                    if (!wait_bounded(BAR(C::B_PF), jp & 1, abort_flag)) break;
                    if (!wait_bounded(BAR(C::B_VF + sp), np & 1, abort_flag)) break;
                    tc_fence_after();
                    const uint32_t sP = base + C::OFF_P, sv = base + C::OFF_V + sp * C::TILE;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        mma_ss(tmem + C::COL_O,
                               sdesc_sw128(sP + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024),
                               sdesc_sw128(sv + kk * 2048u, 16384, 1024), ID_O,
                               (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(BAR(C::B_KE + sp));
                    mma_commit(BAR(C::B_OD));
                }
            }
            if (*abort_flag) {  // every issued MMA must finish before TMEM is freed
                mma_commit(BAR(C::B_DR));
                wait_drain(BAR(C::B_DR), 0);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax
        const int r = threadIdx.x;  // row of the tile == TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const int qrow = qt * 128 + r;
        const float sl = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            const int b = j & 1, nb = j >> 1;
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF + b), nb & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lane_addr + b * 128u + c * 32u, sr[c]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) reg_fence32(sr[c]);
            tc_fence_before();
            mbar_arrive(BAR(C::B_SE + b));

            float s[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
            // keys at or past N, and (causal) keys after this query, are masked
            const int key0 = j * 128;
            int limit = p.N - key0;
            if (p.causal) limit = min(limit, qrow - key0 + 1);
            if (limit < 128) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= limit) s[c] = -INFINITY;
            }
            float mx = s[0];
#pragma unroll
            for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
            const float m_new = fmaxf(m, mx * sl);
            const float alpha = ex2(m - m_new);
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                s[c] = ex2(fmaf(s[c], sl, -m_new));
                sum += s[c];
            }
            l = fmaf(l, alpha, sum);
            m = m_new;

            if (j >= 1) {  // PV(j-1) must be done: O is rescaled and P's buffer reused
                ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OD), (j - 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(lane_addr + C::COL_O + c * 32u, o);
                        tmem_ld_wait();
                        reg_fence32(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(lane_addr + C::COL_O + c * 32u, o);
                    }
                    tmem_st_wait();
                }
            }
            // P (rounded to the input type) into the swizzled K-major tile
            const uint32_t sP = base + C::OFF_P;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const uint32_t addr = sP + (c >> 3) * 16384u + sw128_off(r, c & 7);
                st_shared_v4(addr, pack2<BF16>(s[8 * c + 0], s[8 * c + 1]),
                             pack2<BF16>(s[8 * c + 2], s[8 * c + 3]),
                             pack2<BF16>(s[8 * c + 4], s[8 * c + 5]),
                             pack2<BF16>(s[8 * c + 6], s[8 * c + 7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(BAR(C::B_PF));
        }
        if (ok) {
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_OD), (nkv - 1) & 1, abort_flag));
        }
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            uint8_t* orow = static_cast<uint8_t*>(p.o) +
                            (static_cast<size_t>(bh) * p.N + qrow) * (D * 2);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_addr + C::COL_O + c * 32u, o);
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
            if (qrow < p.N)
                p.lse[static_cast<size_t>(bh) * p.N + qrow] = m * 0.69314718055994531f + logf(l);
        }
    }
#undef BAR
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace attn

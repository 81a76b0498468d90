// Backward kernels: gradients of sum(O * dO) for exact attention, with the
// probabilities recomputed tile by tile from the stored log-sum-exp instead
// of being stored by the forward.
//
// Method: "Is a full day of context better than ten minutes? FlashAttention
// and the sequence-length question" (marketmaker.cc), section "backward:
// recompute instead of store" (only O and the per-row softmax statistic are
// kept, P is rebuilt from Q, K per tile — gradient checkpointing at tile
// granularity) and section "causal masking" (key/query tile pairs wholly in
// the future are skipped); the statistic is the log-sum-exp L —
// "Performance optimisation with Flash-Attention 2" (Medium), section
// "Flash Attention 2".  The chain rule itself is not on the pages; with
// s_ij = scale q_i.k_j, P_ij = exp(s_ij - L_i), D_i = sum_t dO_it O_it:
//   dV_j = sum_i P_ij dO_i,  dP_ij = dO_i.v_j,  dS_ij = P_ij (dP_ij - D_i),
//   dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j.
//
// Kernels
//   attn_bwd_prep_kernel  D_i = rowdot(dO_i, O_i) and L2_i = LSE_i * log2(e),
//                         both fp32 in a per-head array padded to a multiple of
//                         128 rows (padding: D = 0, L2 = +inf so P = 0); zeroes
//                         the fp32 dQ accumulator and the per-head counters.
//   attn_bwd_main_kernel  (head dimension 64; 128 has its own kernel in
//                         bwd128_sm100.cuh)
//                         one CTA per (head, 128-key tile j); K_j, V_j stay in
//                         shared memory while the 128-query tiles i stream
//                         through (Q double-buffered).  Per query tile:
//                           S^T  = K_j Q_i^T          (tensor memory)
//                           dP^T = V_j dO_i^T         (tensor memory)
//                           P^T  = exp2(S^T log2e scale - L2_i), written back
//                                  into tensor memory as bf16/fp16 over S^T
//                           dV  += P^T dO_i           (A read from tensor memory)
//                           dS^T = P^T (dP^T - D_i)   (shared memory, half)
//                           dK  += dS^T Q_i
//                           dQ_i partial = dS K_j, added to the fp32
//                                  accumulator with non-returning reductions
//                         The last CTA of a head to finish converts that head's
//                         dQ to the output type.
//
// Roles (320 threads): warps 0-7 compute (warp w reads TMEM lanes 32 (w % 4)
// .. + 31 and the query-column half w / 4 of each tile), warp 8 TMA producer,
// warp 9 MMA issuer and TMEM owner.
// Tensor memory (512 columns): S^T/P^T at 0, dP^T at 128, dV at 256, dK at
// 256 + D.  For D = 128 the dQ tile is formed transposed, dQ^T = K^T dS^T
// (lane = feature, column = query), in the dP^T columns once dS^T has been
// read out, so each warp's reductions cover 32 consecutive floats of one
// query row.  For D = 64 it is dQ = dS K (lane = query) in columns 384..447.
#pragma once

#include "dropout.cuh"
#include "ptx.cuh"

namespace attn {

// Hook the host side installs to keep the last CUDA error of a launch.
inline void (*&bwd_error_hook())(cudaError_t) {
    static void (*hook)(cudaError_t) = nullptr;
    return hook;
}
inline void bwd_record_error(cudaError_t e) {
    if (bwd_error_hook()) bwd_error_hook()(e);
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: L2 (BH*Np fp32) | D (BH*Np fp32) | dQ accumulator (BH*N*d fp32) |
// counters (BH int32), Np = N rounded up to 128; sections 256-byte aligned.
inline size_t bwd_np(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }
inline size_t bwd_ws_off_d(int B, int H, int N) {
    return align256(static_cast<size_t>(B) * H * bwd_np(N) * 4);
}
inline size_t bwd_ws_off_dq(int B, int H, int N) { return 2 * bwd_ws_off_d(B, H, N); }
inline size_t bwd_ws_off_cnt(int B, int H, int N, int d) {
    return bwd_ws_off_dq(B, H, N) + align256(static_cast<size_t>(B) * H * N * d * 4);
}
inline size_t bwd_workspace_bytes(int B, int H, int N, int d) {
    return bwd_ws_off_cnt(B, H, N, d) + align256(static_cast<size_t>(B) * H * 4);
}

// ------------------------------------------------------------------ prep --
template <int D, bool BF16>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(
    const uint4* __restrict__ o, const uint4* __restrict__ dout, const float* __restrict__ lse,
    float* __restrict__ l2pad, float* __restrict__ dpad, float4* __restrict__ dqacc,
    int* __restrict__ counters, int N, int Np, long long rows_padded, int BH) {
    constexpr int TPR = D / 8;  // threads per row, 8 elements (16 bytes) each
    const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long prow = gid / TPR;  // padded row: bh * Np + i
    const int part = static_cast<int>(gid % TPR);
    const long long bh = prow / Np;
    const int i = static_cast<int>(prow - bh * Np);
    const bool real = prow < rows_padded && i < N;
    const long long row = bh * N + i;
    float acc = 0.f;
    if (real) {
        const uint4 a = o[row * TPR + part];
        const uint4 b = dout[row * TPR + part];
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float2 x = unpack2<BF16>(av[t]), y = unpack2<BF16>(bv[t]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        dqacc[row * (D / 4) + 2 * part] = z;
        dqacc[row * (D / 4) + 2 * part + 1] = z;
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (prow < rows_padded && part == 0) {
        dpad[prow] = real ? acc : 0.f;
        l2pad[prow] = real ? lse[row] * 1.4426950408889634f : INFINITY;
    }
    if (gid < BH) counters[gid] = 0;
}

// ------------------------------------------------------------------ main --
struct BwdParams {
    const float* l2pad;
    const float* dpad;
    float* dqacc;
    int* counters;
    void* dq;
    void* dk;
    void* dv;
    int BH;
    int N;
    int Np;
    int n_qtiles;
    int n_ktiles;
    int group;  // persistent kernels: heads per scheduling group
    int causal;
    float scale;
    float scale_log2;
    // Block-sparse attention: n_qtiles128 x n_ktiles bytes, nonzero where the
    // 128-row query tile i may attend to key tile j (one mask for every head);
    // nullptr for dense attention.
    const uint8_t* bmask = nullptr;
    // Dropout on P (kernels instantiated with DROP only).
    DropoutParams drop{0u, 0u, 256u, 1.f};
};

template <int D>
struct BwdCfg {
    static constexpr int KB = D / 64;
    static constexpr uint32_t TILE = 128u * D * 2u;
    static constexpr int QST = 2;
    static_assert(D == 64, "head dimension 128 has its own kernel (bwd128_sm100.cuh)");
    static constexpr int DOST = 2;
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = OFF_K + TILE;
    static constexpr uint32_t OFF_Q = OFF_V + TILE;
    static constexpr uint32_t OFF_DO = OFF_Q + QST * TILE;
    static constexpr uint32_t OFF_DST = OFF_DO + DOST * TILE;   // 128 x 128 half
    static constexpr uint32_t OFF_LD = OFF_DST + 32768u;       // QST x (128 L2 + 128 D) fp32
    static constexpr uint32_t OFF_BAR = OFF_LD + QST * 1024u;
    static constexpr int B_KV = 0, B_QF = 1, B_QE = B_QF + QST, B_DOF = B_QE + QST,
                         B_DOE = B_DOF + DOST, B_SF = B_DOE + DOST, B_DPF = B_SF + 1,
                         B_PTF = B_DPF + 1, B_DVD = B_PTF + 1, B_DSF = B_DVD + 1,
                         B_DQF = B_DSF + 1, B_DQE = B_DQF + 2, B_FIN = B_DQE + 2,
                         B_DR = B_FIN + 1, B_ENDA = B_DR + 1, B_ENDB = B_ENDA + 1,
                         B_SRD = B_ENDB + 1, NBAR = B_SRD + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
    static constexpr uint32_t COL_DQ = 384;  // two buffers: 384 and 448 (tile parity)
    static constexpr int NCOMPUTE = 256;             // 8 compute warps
    static constexpr int NTHREADS = NCOMPUTE + 64;   // + TMA warp + MMA warp
    static constexpr int WARP_TMA = NCOMPUTE / 32, WARP_MMA = WARP_TMA + 1;
};

template <int D, bool BF16, bool DROP = false>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmDO, const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: under the causal mask key-tile-major, every head's heaviest key
    // tile (j = 0) first, so that the CTAs launched last are the light ones;
    // otherwise head-major.
    const int bh = p.causal ? static_cast<int>(blockIdx.x) % p.BH
                            : static_cast<int>(blockIdx.x) / p.n_ktiles;
    const int j = p.causal ? static_cast<int>(blockIdx.x) / p.BH
                           : static_cast<int>(blockIdx.x) % p.n_ktiles;
    const int i_begin = p.causal ? j : 0;
    // Query tiles i = i_begin .., and under a block mask only those marked for
    // key tile j; every role walks the same sequence (next_tile).
    const uint8_t* mcol = p.bmask ? p.bmask + j : nullptr;
    auto next_tile = [&](int i) {
        if (mcol != nullptr)
            while (i < p.n_qtiles && mcol[static_cast<size_t>(i) * p.n_ktiles] == 0) ++i;
        return i;
    };
    int n_it = p.n_qtiles - i_begin;
    if (mcol != nullptr) {
        n_it = 0;
        for (int i = next_tile(i_begin); i < p.n_qtiles; i = next_tile(i + 1)) ++n_it;
    }

    const uint32_t bar0 = base + C::OFF_BAR;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC + 4);
    volatile uint32_t* last_flag = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC + 8);
    const float* sLD = reinterpret_cast<const float*>(gbase + C::OFF_LD);

    if (threadIdx.x == 0) {
        mbar_init(BAR(C::B_KV), 1);
        for (int s = 0; s < C::QST; ++s) {
            mbar_init(BAR(C::B_QF + s), 1);
            mbar_init(BAR(C::B_QE + s), 1);
        }
        for (int s = 0; s < C::DOST; ++s) {
            mbar_init(BAR(C::B_DOF + s), 1);
            mbar_init(BAR(C::B_DOE + s), 1);
        }
        mbar_init(BAR(C::B_SF), 1);
        mbar_init(BAR(C::B_DPF), 1);
        mbar_init(BAR(C::B_PTF), C::NCOMPUTE);
        mbar_init(BAR(C::B_DVD), 1);
        mbar_init(BAR(C::B_DSF), C::NCOMPUTE);
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(C::B_DQF + b), 1);
            mbar_init(BAR(C::B_DQE + b), C::NCOMPUTE);
        }
        mbar_init(BAR(C::B_FIN), 1);
        mbar_init(BAR(C::B_DR), 1);
        mbar_init(BAR(C::B_ENDA), C::NCOMPUTE);
        mbar_init(BAR(C::B_ENDB), 1);
        mbar_init(BAR(C::B_SRD), C::NCOMPUTE / 2);
        *abort_flag = 0u;
        *last_flag = 0u;
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

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmDO);
            mbar_arrive_expect_tx(BAR(C::B_KV), 2 * C::TILE);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_3d(base + C::OFF_K + kb * 16384u, &tmK, BAR(C::B_KV), kb * 64, j * 128, bh);
                tma_load_3d(base + C::OFF_V + kb * 16384u, &tmV, BAR(C::B_KV), kb * 64, j * 128, bh);
            }
            int q_issued[C::QST], do_issued[C::DOST];
            for (int s = 0; s < C::QST; ++s) q_issued[s] = 0;
            for (int s = 0; s < C::DOST; ++s) do_issued[s] = 0;
            const size_t ld_row0 = static_cast<size_t>(bh) * p.Np;
            for (int it = 0, i = next_tile(i_begin); it < n_it; ++it, i = next_tile(i + 1)) {
                const int qs = it % C::QST, qn = it / C::QST;
                const int ds = it % C::DOST, dn = it / C::DOST;
                if (!wait_bounded(BAR(C::B_QE + qs), (qn & 1) ^ 1, abort_flag)) break;
                const uint32_t sq = base + C::OFF_Q + qs * C::TILE;
                const uint32_t sld = base + C::OFF_LD + qs * 1024u;
                mbar_arrive_expect_tx(BAR(C::B_QF + qs), C::TILE + 1024u);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sq + kb * 16384u, &tmQ, BAR(C::B_QF + qs), kb * 64, i * 128, bh);
                bulk_load(sld, p.l2pad + ld_row0 + i * 128, 512u, BAR(C::B_QF + qs));
                bulk_load(sld + 512u, p.dpad + ld_row0 + i * 128, 512u, BAR(C::B_QF + qs));
                q_issued[qs] = qn + 1;
                if (!wait_bounded(BAR(C::B_DOE + ds), (dn & 1) ^ 1, abort_flag)) break;
                const uint32_t sdo = base + C::OFF_DO + ds * C::TILE;
                mbar_arrive_expect_tx(BAR(C::B_DOF + ds), C::TILE);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_3d(sdo + kb * 16384u, &tmDO, BAR(C::B_DOF + ds), kb * 64, i * 128, bh);
                do_issued[ds] = dn + 1;
            }
            if (*abort_flag) {
                wait_drain(BAR(C::B_KV), 0);
                for (int s = 0; s < C::QST; ++s)
                    if (q_issued[s] > 0) wait_drain(BAR(C::B_QF + s), (q_issued[s] - 1) & 1);
                for (int s = 0; s < C::DOST; ++s)
                    if (do_issued[s] > 0) wait_drain(BAR(C::B_DOF + s), (do_issued[s] - 1) & 1);
            }
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_SS = idesc_f16(BF16, 128, 128, false, false);
            constexpr uint32_t ID_KV = idesc_f16(BF16, 128, D, false, true);
            constexpr uint32_t ID_DQ = idesc_f16(BF16, 128, D, true, true);     // D == 64
            const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sDST = base + C::OFF_DST;
            bool ok = wait_bounded(BAR(C::B_KV), 0, abort_flag);
            for (int it = 0; ok && it < n_it; ++it) {
                const uint32_t ph = it & 1;
                const int qs = it % C::QST, qn = it / C::QST;
                const int ds = it % C::DOST, dn = it / C::DOST;
                const uint32_t sQ = base + C::OFF_Q + qs * C::TILE;
                const uint32_t sDO = base + C::OFF_DO + ds * C::TILE;
                // S^T = K Q^T; the S/P columns must be free: dV(it-1) has read P^T(it-1)
                if (!(ok = wait_bounded(BAR(C::B_QF + qs), qn & 1, abort_flag))) break;
                if (it > 0 && !(ok = wait_bounded(BAR(C::B_DVD), ph ^ 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem + C::COL_S, sdesc_sw128(sK + off, 16, 1024),
                           sdesc_sw128(sQ + off, 16, 1024), ID_SS, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(C::B_SF));
                // dP^T = V dO^T
                if (!(ok = wait_bounded(BAR(C::B_DOF + ds), dn & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem + C::COL_DP, sdesc_sw128(sV + off, 16, 1024),
                           sdesc_sw128(sDO + off, 16, 1024), ID_SS, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(C::B_DPF));
                // dV += P^T dO with P^T read from tensor memory
                if (!(ok = wait_bounded(BAR(C::B_PTF), ph, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(tmem + C::COL_DV, tmem + C::COL_S + kk * 8u,
                           sdesc_sw128(sDO + kk * 2048u, 16384, 1024), ID_KV,
                           (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(BAR(C::B_DVD));
                mma_commit(BAR(C::B_DOE + ds));
                // dK += dS^T Q ; dQ partial into buffer it & 1, once its last
                // contents, dQ(it-2), have been drained
                if (!(ok = wait_bounded(BAR(C::B_DSF), ph, abort_flag))) break;
                if (it >= 2 &&
                    !(ok = wait_bounded(BAR(C::B_DQE + (it & 1)), ((it >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tmem + C::COL_DK,
                           sdesc_sw128(sDST + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024),
                           sdesc_sw128(sQ + kk * 2048u, 16384, 1024), ID_KV,
                           (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // dQ = dS K: A = dS^T read MN-major, B = K MN-major
                    mma_ss(tmem + C::COL_DQ + (it & 1) * 64u, sdesc_sw128(sDST + kk * 2048u, 16384, 1024),
                           sdesc_sw128(sK + kk * 2048u, 16384, 1024), ID_DQ,
                           kk > 0 ? 1u : 0u);
                mma_commit(BAR(C::B_QE + qs));
                mma_commit(BAR(C::B_DQF + (it & 1)));
            }
            if (ok) mma_commit(BAR(C::B_FIN));
            if (*abort_flag) {
                mma_commit(BAR(C::B_DR));
                wait_drain(BAR(C::B_DR), 0);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- compute
        // Warp w owns TMEM lanes 32 (w % 4) .. + 31 (a warp may only touch its
        // lane quarter) and column half h = w / 4 of every 128-wide tile.
        const int quarter = warp & 3, half = warp >> 2;
        const int r = quarter * 32 + lane;  // TMEM lane
        const int tid = threadIdx.x;        // 0 .. NCOMPUTE-1
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const int key = j * 128 + r;
        const bool key_valid = key < p.N;
        const float sl = p.scale_log2;
        const size_t head_row0 = static_cast<size_t>(bh) * p.N;
        const uint32_t sDST = base + C::OFF_DST;
        const int c0 = half * 64;  // first query column of this thread's half
        // dQ of tile t (query rows q0p ..): lane r holds query row q0p + r; this
        // half covers features 32 h .. 32 h + 31
        auto drain_dq = [&](int t, int q0p) {
            tc_fence_after();
            const int qr = q0p + r;
            float* row = p.dqacc + (head_row0 + qr) * D + half * 32;
            uint32_t v[32];
            tmem_ld32(lane_addr + C::COL_DQ + (t & 1) * 64u + half * 32u, v);
            tmem_ld_wait();
            reg_fence32(v);
            tc_fence_before();
            mbar_arrive(BAR(C::B_DQE + (t & 1)));  // in registers: the buffer is free
            if (qr < p.N) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    red_add_v4_f32(row + 4 * e, __uint_as_float(v[4 * e]) * p.scale,
                                   __uint_as_float(v[4 * e + 1]) * p.scale,
                                   __uint_as_float(v[4 * e + 2]) * p.scale,
                                   __uint_as_float(v[4 * e + 3]) * p.scale);
            }
        };
        int prev_q0 = 0;
        bool ok = true;
        for (int it = 0, i = next_tile(i_begin); it < n_it; ++it, i = next_tile(i + 1)) {
            const int q0 = i * 128;
            const uint32_t ph = it & 1;
            const float4* L4 = reinterpret_cast<const float4*>(sLD + (it % C::QST) * 256 + c0);
            const float4* D4 = reinterpret_cast<const float4*>(sLD + (it % C::QST) * 256 + 128 + c0);

            // ---- P^T = exp2(S^T scale log2e - L2), into tensor memory over S^T
            // (wait on the load barrier too: it makes the bulk-copied L2/D visible)
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_QF + it % C::QST),
                                                      (it / C::QST) & 1, abort_flag));
            if (ok) ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SF), ph, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float pv[64];
            uint32_t kw[2][8];  // dropout keep masks of the 64 query columns (bytes)
            {
                uint32_t sv[2][32];
                tmem_ld32(lane_addr + C::COL_S + c0, sv[0]);
                tmem_ld32(lane_addr + C::COL_S + c0 + 32u, sv[1]);
                tmem_ld_wait();
                reg_fence32(sv[0]);
                reg_fence32(sv[1]);
                if (half == 0) {  // half 1 writes P^T over columns half 0 reads
                    tc_fence_before();
                    mbar_arrive(BAR(C::B_SRD));
                }
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                    const float4 l4 = L4[g];
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * g + e;
                        pv[c] = ex2(fmaf(__uint_as_float(sv[c >> 5][c & 31]), sl, -lv[e]));
                    }
                }
                // causal diagonal tile: query q0 + c sees key j*128 + r iff c >= r;
                // key rows past N see nothing
                if (!key_valid || (p.causal && i == j)) {
                    const int lo = key_valid ? r - c0 : 64;
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (c < lo) pv[c] = 0.f;
                }
                uint32_t pk[32];
                if constexpr (DROP) {
                    // P^T for dV without the dropped values (256 / t is applied to dV
                    // at the end); dS below uses P and the masked dP
                    if (p.drop.thr < 256u) {
                        dropout_keep_keyrows(p.drop, bh, q0 + c0, j * 128 + quarter * 32, kw[0]);
                        dropout_keep_keyrows(p.drop, bh, q0 + c0 + 32, j * 128 + quarter * 32, kw[1]);
                    } else {
#pragma unroll
                        for (int t = 0; t < 8; ++t) kw[0][t] = kw[1][t] = 0xFFFFFFFFu;
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const uint32_t kb = kw[c >> 4][(c >> 1) & 7] >> (16 * (c & 1));
                        pk[c] = pack2<BF16>((kb & 0x1u) ? pv[2 * c] : 0.f,
                                            (kb & 0x100u) ? pv[2 * c + 1] : 0.f);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) pk[c] = pack2<BF16>(pv[2 * c], pv[2 * c + 1]);
                }
                if (half == 1) {
                    ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_SRD), ph, abort_flag));
                    tc_fence_after();
                }
                if (ok) {
                    tmem_st32(lane_addr + C::COL_S + half * 32u, pk);
                    tmem_st_wait();
                }
            }
            if (!ok) break;
            tc_fence_before();
            mbar_arrive(BAR(C::B_PTF));

            // ---- dS^T = P^T (dP^T - D), half, into shared memory, once dK and
            // dQ of the previous tile have read it (implied by the dP^T commit,
            // which follows them; kept as a guard)
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_DPF), ph, abort_flag));
            if (ok && it >= 1)
                ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_DQF + ((it - 1) & 1)),
                                                          ((it - 1) >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c4 = 0; c4 < 2; ++c4) {
                uint32_t dpv[32];
                tmem_ld32(lane_addr + C::COL_DP + c0 + c4 * 32u, dpv);
                tmem_ld_wait();
                reg_fence32(dpv);
                float dsv[32];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const float4 d4 = D4[c4 * 8 + g];
                    const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float dpe = __uint_as_float(dpv[4 * g + e]);
                        if constexpr (DROP)
                            dpe = ((kw[c4][g] >> (8 * e)) & 1u) ? dpe * p.drop.inv_keep : 0.f;
                        dsv[4 * g + e] = pv[c4 * 32 + 4 * g + e] * (dpe - dd[e]);
                    }
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int c = half * 8 + c4 * 4 + g;  // 16-byte chunk index (8 columns)
                    st_shared_v4(sDST + (c >> 3) * 16384u + sw128_off(r, c & 7),
                                 pack2<BF16>(dsv[8 * g + 0], dsv[8 * g + 1]),
                                 pack2<BF16>(dsv[8 * g + 2], dsv[8 * g + 3]),
                                 pack2<BF16>(dsv[8 * g + 4], dsv[8 * g + 5]),
                                 pack2<BF16>(dsv[8 * g + 6], dsv[8 * g + 7]));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(BAR(C::B_DSF));

            // ---- dQ of the previous tile into the fp32 accumulator: its product
            // completed before dS^T(it) was written, so the drain no longer waits
            if (it >= 1) drain_dq(it - 1, prev_q0);
            prev_q0 = q0;
        }
        if (ok && n_it > 0) {  // the last tile's dQ
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_DQF + ((n_it - 1) & 1)),
                                                      ((n_it - 1) >> 1) & 1, abort_flag));
            if (ok) drain_dq(n_it - 1, prev_q0);
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_FIN), 0, abort_flag));
        if (ok) {  // dK_j, dV_j rows: lane r holds key row j*128 + r; this half, D/2 features
            tc_fence_after();
            const size_t rowoff = (head_row0 + key) * (D * 2) + half * D;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint8_t* out = static_cast<uint8_t*>(which ? p.dv : p.dk) + rowoff;
                const uint32_t col = (which ? C::COL_DV : C::COL_DK) + half * (D / 2);
                const float mul = which ? (DROP ? p.drop.inv_keep : 1.f) : p.scale;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t v[32];
                    tmem_ld32(lane_addr + col + c * 32u, v);
                    tmem_ld_wait();
                    reg_fence32(v);
                    if (n_it == 0)  // block-sparse: no query tile marked, dK = dV = 0
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0u;
                    uint32_t h[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        h[e] = pack2<BF16>(__uint_as_float(v[2 * e]) * mul,
                                           __uint_as_float(v[2 * e + 1]) * mul);
                    if (key_valid) {
                        uint4* d4 = reinterpret_cast<uint4*>(out + c * 64);
                        d4[0] = make_uint4(h[0], h[1], h[2], h[3]);
                        d4[1] = make_uint4(h[4], h[5], h[6], h[7]);
                        d4[2] = make_uint4(h[8], h[9], h[10], h[11]);
                        d4[3] = make_uint4(h[12], h[13], h[14], h[15]);
                    }
                }
            }
            // The last CTA of this head to finish converts the head's dQ.
            // Bounded mbarrier syncs (not bar.sync): a warp that gave up
            // cannot leave the others waiting for ever.
            __threadfence();
            mbar_arrive(BAR(C::B_ENDA));
            if (tid == 0) {
                if (wait_bounded(BAR(C::B_ENDA), 0, abort_flag)) {
                    const int done = atomicAdd(p.counters + bh, 1);
                    *last_flag = (done == p.n_ktiles - 1) ? 1u : 0u;
                }
                mbar_arrive(BAR(C::B_ENDB));
            }
            ok = __all_sync(0xffffffffu, wait_bounded(BAR(C::B_ENDB), 0, abort_flag));
            if (ok && *last_flag) {
                __threadfence();
                const float4* src = reinterpret_cast<const float4*>(p.dqacc + head_row0 * D);
                uint2* out = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.dq) + head_row0 * D * 2);
                const long long n4 = static_cast<long long>(p.N) * D / 4;
                // eight loads in flight per thread before any is used (one at a
                // time, the head's conversion took ~19 us on one SM)
                constexpr int U = 8;
                for (long long e0 = tid; e0 < n4; e0 += static_cast<long long>(C::NCOMPUTE) * U) {
                    float4 x[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const long long e = e0 + static_cast<long long>(u) * C::NCOMPUTE;
                        if (e < n4) x[u] = __ldcg(src + e);
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const long long e = e0 + static_cast<long long>(u) * C::NCOMPUTE;
                        if (e < n4)
                            out[e] = make_uint2(pack2<BF16>(x[u].x, x[u].y), pack2<BF16>(x[u].z, x[u].w));
                    }
                }
            }
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

inline bool bwd_set_attributes() {
    bool ok = true;
    ok &= cudaFuncSetAttribute(attn_bwd_main_kernel<64, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_bwd_main_kernel<64, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_bwd_main_kernel<64, true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn_bwd_main_kernel<64, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    return ok;
}

template <int D, bool BF16>
int bwd_prep_launch(const void* o, const void* dout, const float* lse, void* ws, int B, int H,
                    int N, cudaStream_t st) {
    const int Np = static_cast<int>(bwd_np(N));
    const long long rows_padded = 1LL * B * H * Np;
    const long long threads = rows_padded * (D / 8);
    const long long blocks = (threads + 255) / 256;
    if (blocks >= (1LL << 31)) return -2;
    uint8_t* w = static_cast<uint8_t*>(ws);
    attn_bwd_prep_kernel<D, BF16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(o), static_cast<const uint4*>(dout), lse,
        reinterpret_cast<float*>(w), reinterpret_cast<float*>(w + bwd_ws_off_d(B, H, N)),
        reinterpret_cast<float4*>(w + bwd_ws_off_dq(B, H, N)),
        reinterpret_cast<int*>(w + bwd_ws_off_cnt(B, H, N, D)), N, Np, rows_padded, B * H);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) bwd_record_error(e);
    return e == cudaSuccess ? 0 : -7;
}

template <int D, bool BF16>
int bwd_main_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mdo, void* dq, void* dk, void* dv, void* ws, int B, int H,
                    int N, int causal, float scale, cudaStream_t st,
                    const uint8_t* bmask = nullptr, const DropoutParams* drop = nullptr) {
    BwdParams p;
    p.bmask = bmask;
    if (drop) p.drop = *drop;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.l2pad = reinterpret_cast<const float*>(w);
    p.dpad = reinterpret_cast<const float*>(w + bwd_ws_off_d(B, H, N));
    p.dqacc = reinterpret_cast<float*>(w + bwd_ws_off_dq(B, H, N));
    p.counters = reinterpret_cast<int*>(w + bwd_ws_off_cnt(B, H, N, D));
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.BH = B * H;
    p.N = N;
    p.Np = static_cast<int>(bwd_np(N));
    p.n_qtiles = (N + 127) / 128;
    p.n_ktiles = (N + 127) / 128;
    p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    const long long nblocks = 1LL * p.n_ktiles * p.BH;
    if (nblocks >= (1LL << 31)) return -2;
    if (drop)
        attn_bwd_main_kernel<D, BF16, true><<<static_cast<unsigned>(nblocks), BwdCfg<D>::NTHREADS,
                                              BwdCfg<D>::SMEM_BYTES, st>>>(mq, mk, mv, mdo, p);
    else
        attn_bwd_main_kernel<D, BF16><<<static_cast<unsigned>(nblocks), BwdCfg<D>::NTHREADS,
                                        BwdCfg<D>::SMEM_BYTES, st>>>(mq, mk, mv, mdo, p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) bwd_record_error(e);
    return e == cudaSuccess ? 0 : -7;
}

}  // namespace attn

// Causal linear attention, chunked: O_i = scale sum_{j <= i} (q_i . k_j) v_j.
//
// Method: "Lightning Attention-2: A Free Lunch for Handling Unlimited
// Sequence Lengths in Large Language Models" (chatpaper.ai summary),
// abstract: the cumulative sum of causal linear attention is tiled into
// intra-block parts, computed like ordinary attention, and inter-block parts,
// computed with the linear-attention kernel trick (a running d x d state);
// "Gated Linear Attention Transformers with Hardware-Efficient Training"
// (nubint.ai review), proposed method: the chunk-wise parallel form.  With
// chunks of C = 128 rows and S_c = sum over earlier chunks of K^T V,
//     O_c = scale [(Q_c K_c^T) o M] V_c + Q_c (scale S_c),   M the causal mask.
// Two forms.  Three kernels, every chunk in parallel (fewer heads):
//   linear_kv_kernel      KV_c = K_c^T V_c (tcgen05, fp32 in tensor memory)
//                         written to a fp32 workspace;
//   linear_prefix_kernel  S_c = scale * sum_{c' < c} KV_c' (exclusive prefix
//                         over chunks, fp32 sums), stored in the input's
//                         16-bit type as the B operand of the next kernel;
//   linear_out_kernel     A = Q_c K_c^T (tensor memory), masked and scaled by
//                         the warps that own its rows and written back as P;
//                         O = Q_c S_c + P V_c (tensor memory), stored.
// and one fused kernel (many heads; below).  Head dimension 128 only (the
// state product K^T V has M = d rows).
#pragma once

#include "ptx.cuh"

namespace attn {

struct LinearParams {
    void* o;
    float* kv;     // (BH, n_chunks, 128, 128) fp32
    void* state;   // (BH, n_chunks, 128, 128) 16-bit, scale * exclusive prefix
    int BH;
    int N;
    int n_chunks;
    float scale;
};

constexpr uint32_t kLinTile = 128u * 128u * 2u;  // one 128 x 128 16-bit tile

// ---------------------------------------------------------------- K^T V --
// One CTA per (head, chunk): warp 0 loads K_c and V_c, warp 1 issues the
// eight MMAs of K^T V (A = K with the feature dimension contiguous, i.e.
// MN-major; B = V likewise) and owns tensor memory, warps 2-5 move the fp32
// result (TMEM lane a = feature of K) to the workspace.
template <bool BF16>
__global__ void __launch_bounds__(192, 1)
    linear_kv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const LinearParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / p.n_chunks, c = blockIdx.x % p.n_chunks;
    const uint32_t sK = base, sV = base + kLinTile, bar = base + 2 * kLinTile;
    const uint32_t B_LD = bar, B_MM = bar + 8, B_DR = bar + 16;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + 2 * kLinTile + 32);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    if (threadIdx.x == 0) {
        mbar_init(B_LD, 1);
        mbar_init(B_MM, 1);
        mbar_init(B_DR, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + 2 * kLinTile + 32, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(B_LD, 2 * kLinTile);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
                tma_load_3d(sK + kb * 16384u, &tmK, B_LD, kb * 64, c * 128, bh);
                tma_load_3d(sV + kb * 16384u, &tmV, B_LD, kb * 64, c * 128, bh);
            }
            if (!wait_bounded(B_LD, 0, abort_flag)) wait_drain(B_LD, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID = idesc_f16(BF16, 128, 128, true, true);
            if (wait_bounded(B_LD, 0, abort_flag)) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // K-dim: 16 tokens (2048 bytes) per step
                    mma_ss(tmem, sdesc_sw128(sK + kk * 2048u, 16384, 1024),
                           sdesc_sw128(sV + kk * 2048u, 16384, 1024), ID, kk > 0 ? 1u : 0u);
                mma_commit(B_MM);
            } else {
                mma_commit(B_DR);
                wait_drain(B_DR, 0);
            }
        }
        __syncwarp();
    } else {
        const int quarter = warp & 3, a = quarter * 32 + lane;  // feature of K = TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        if (__all_sync(0xffffffffu, wait_bounded(B_MM, 0, abort_flag))) {
            tc_fence_after();
            float4* row = reinterpret_cast<float4*>(
                p.kv + ((static_cast<size_t>(bh) * p.n_chunks + c) * 128 + a) * 128);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_addr + cc * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    row[cc * 8 + e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                                  __uint_as_float(v[4 * e + 2]),
                                                  __uint_as_float(v[4 * e + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// ------------------------------------------------------ exclusive prefix --
// Thread t of head bh owns 4 consecutive entries of the 128 x 128 state and
// walks the chunks: S_c = scale * (sum of KV_c' for c' < c), in fp32, stored
// rounded to the 16-bit type.
template <bool BF16>
__global__ void __launch_bounds__(256) linear_prefix_kernel(const LinearParams p) {
    const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long per_head = 128 * 128 / 4;
    if (t >= static_cast<long long>(p.BH) * per_head) return;
    const long long bh = t / per_head, e4 = t % per_head;
    const float4* kv = reinterpret_cast<const float4*>(p.kv) + bh * p.n_chunks * per_head + e4;
    uint2* st = reinterpret_cast<uint2*>(p.state) + bh * p.n_chunks * per_head + e4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < p.n_chunks; ++c) {
        st[c * per_head] = make_uint2(pack2<BF16>(acc.x * p.scale, acc.y * p.scale),
                                      pack2<BF16>(acc.z * p.scale, acc.w * p.scale));
        const float4 x = kv[c * per_head];
        acc.x += x.x, acc.y += x.y, acc.z += x.z, acc.w += x.w;
    }
}

// ------------------------------------------------------------ output --
// One CTA per (head, chunk): warp 0 loads Q_c, K_c, V_c and the state S_c;
// warp 1 owns tensor memory (A at columns 0-127, O at 128-255) and issues
// A = Q K^T, O = Q S_c, then (after the row warps wrote P) O += P V; warps
// 2-5 (thread = row i of the chunk = TMEM lane) mask and scale A into P
// (16-bit, written over A's first 64 columns), then store O.
template <bool BF16>
__global__ void __launch_bounds__(192, 1)
    linear_out_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                      const LinearParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / p.n_chunks, c = blockIdx.x % p.n_chunks;
    const uint32_t sQ = base, sK = base + kLinTile, sV = base + 2 * kLinTile,
                   sS = base + 3 * kLinTile, bar = base + 4 * kLinTile;
    const uint32_t B_LD = bar, B_AF = bar + 8, B_PF = bar + 16, B_OD = bar + 24, B_DR = bar + 32;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + 4 * kLinTile + 64);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    constexpr uint32_t COL_O = 128;
    if (threadIdx.x == 0) {
        mbar_init(B_LD, 1);
        mbar_init(B_AF, 1);
        mbar_init(B_PF, 128);
        mbar_init(B_OD, 1);
        mbar_init(B_DR, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + 4 * kLinTile + 64, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == 0) {
        if (lane == 0) {
            mbar_arrive_expect_tx(B_LD, 4 * kLinTile);
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
                tma_load_3d(sQ + kb * 16384u, &tmQ, B_LD, kb * 64, c * 128, bh);
                tma_load_3d(sK + kb * 16384u, &tmK, B_LD, kb * 64, c * 128, bh);
                tma_load_3d(sV + kb * 16384u, &tmV, B_LD, kb * 64, c * 128, bh);
                tma_load_3d(sS + kb * 16384u, &tmS, B_LD, kb * 64, 0, bh * p.n_chunks + c);
            }
            if (!wait_bounded(B_LD, 0, abort_flag)) wait_drain(B_LD, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t ID_A = idesc_f16(BF16, 128, 128, false, false);  // Q K^T
            constexpr uint32_t ID_O = idesc_f16(BF16, 128, 128, false, true);   // Q S, P V
            bool ok = wait_bounded(B_LD, 0, abort_flag);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // K-dim: 16 features per step
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024),
                           ID_A, kk > 0 ? 1u : 0u);
                }
                mma_commit(B_AF);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // O = Q S: B = S rows (features of K)
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem + COL_O, sdesc_sw128(sQ + off, 16, 1024),
                           sdesc_sw128(sS + kk * 2048u, 16384, 1024), ID_O, kk > 0 ? 1u : 0u);
                }
                ok = wait_bounded(B_PF, 0, abort_flag);
                if (ok) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // O += P V: K-dim 16 tokens per step
                        mma_ts(tmem + COL_O, tmem + kk * 8u, sdesc_sw128(sV + kk * 2048u, 16384, 1024),
                               ID_O, 1u);
                    mma_commit(B_OD);
                }
            }
            if (!ok) {
                mma_commit(B_DR);
                wait_drain(B_DR, 0);
            }
        }
        __syncwarp();
    } else {
        const int quarter = warp & 3, r = quarter * 32 + lane;  // row of the chunk = TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const int row = c * 128 + r;
        bool ok = __all_sync(0xffffffffu, wait_bounded(B_AF, 0, abort_flag));
        if (ok) {
            tc_fence_after();
            // P_ij = scale A_ij for j <= i (rows and keys past N are zero already)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t v[32], pk[16];
                tmem_ld32(lane_addr + cc * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j0 = cc * 32 + 2 * e;
                    pk[e] = pack2<BF16>(j0 <= r ? __uint_as_float(v[2 * e]) * p.scale : 0.f,
                                        j0 + 1 <= r ? __uint_as_float(v[2 * e + 1]) * p.scale : 0.f);
                }
                tmem_st16(lane_addr + cc * 16u, pk);  // over columns already read
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(B_PF);
            ok = __all_sync(0xffffffffu, wait_bounded(B_OD, 0, abort_flag));
        }
        if (ok) {
            tc_fence_after();
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.o) +
                                                  (static_cast<size_t>(bh) * p.N + row) * 256);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_addr + COL_O + cc * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
                uint32_t h[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    h[e] = pack2<BF16>(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                if (row < p.N) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[cc * 4 + e] = make_uint4(h[4 * e], h[4 * e + 1], h[4 * e + 2], h[4 * e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------- fused --
// The same chunked form in one kernel, for many heads: one CTA per (head,
// half h of the value features) walks the chunks in order, so the running
// state never leaves the SM.  Per chunk c (stage c % 2 of Q_c, K_c and the
// half V_c[:, 64h..64h+63] in shared memory):
//   A_c  = Q_c K_c^T                tensor memory, two buffers (c % 2)
//   KV_c = K_c^T V_c,h              tensor memory, two buffers
//   P_c  = scale (A_c o M)          the row warps, written over A_c
//   O_c  = Q_c S_{c-1} + P_c V_c,h  tensor memory, two buffers; S_{c-1} from
//                                   shared memory
// The state S_c = scale * sum_{c' <= c} KV_c' is kept in fp32 registers by the
// state warps (thread = feature of K = tensor-memory lane), which add KV_c
// and store S_c rounded to the 16-bit type into one of two shared buffers,
// the B operand of the next chunk's Q S.  The sums are the ones the
// three-kernel form makes, in the same order.
// Issue order per chunk c: A_c and KV_c (once the chunk has landed), Q_c
// S_{c-1}, then P_c V once P_c is written; the next chunk's loads have the
// whole chunk to land.  O has two buffers and the row warps write P_c before
// they read O_{c-1}, so Q_c S_{c-1} waits only for O_{c-2} to have been read.
// Roles (448 threads): warp 0 TMA producer, warp 1 tensor-memory owner and
// MMA issuer, warps 2-9 mask/scale A into P and store O (thread = row of the
// chunk; warps 2-5 take keys 0-63 of P and features 0-31 of O, warps 6-9
// keys 64-127 and features 32-63), warps 10-13 the state.  Each half of the
// row warps packs its 64 keys of P over the first 32 of its own 64 columns
// of A (columns 0-31 and 64-95), which it has read.  Tensor memory: A at 0
// and 128, O at 256 and 320, KV at 384 and 448.
// The fused form is chosen from this many heads (B H) on: with fewer, its
// grid of 2 B H CTAs, each walking every chunk in turn, leaves most SMs idle
// and the three chunk-parallel kernels are faster.
constexpr int kLinFusedMinHeads = 32;

struct LinFusedCfg {
    static constexpr int ST = 2;                       // Q/K/V stages
    static constexpr uint32_t QK = kLinTile;           // 32 KB: Q or K of a chunk
    static constexpr uint32_t VH = kLinTile / 2;       // 16 KB: half of V
    static constexpr uint32_t STAGE = 2 * QK + VH;     // 80 KB
    static constexpr uint32_t OFF_S = ST * STAGE;      // two 16 KB state buffers
    static constexpr uint32_t OFF_BAR = OFF_S + 2 * VH;
    static constexpr int B_LD = 0, B_KE = B_LD + ST, B_AF = B_KE + ST, B_PF = B_AF + 2,
                         B_PVD = B_PF + 2, B_KVF = B_PVD + 2, B_KVE = B_KVF + 2,
                         B_SSF = B_KVE + 2, B_SE = B_SSF + 2, B_OD = B_SE + 2, B_OE = B_OD + 2,
                         B_DR = B_OE + 2, NBAR = B_DR + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
    static constexpr uint32_t COL_O = 256, COL_KV = 384;
    static constexpr int NROW = 256, NSTATE = 128;    // row and state threads
    static constexpr int NTHREADS = 64 + NROW + NSTATE;
    static constexpr int WARP_STATE = 2 + NROW / 32;
    static_assert(SMEM_BYTES <= 232448u, "dynamic shared memory above the sm_100 per-block limit");
};

template <bool BF16>
__global__ void __launch_bounds__(448, 1)
    linear_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const LinearParams p) {
    using C = LinFusedCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x >> 1, h = blockIdx.x & 1;
    const int nc = p.n_chunks;
    const uint32_t bar0 = base + C::OFF_BAR;
#define LBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::OFF_MISC);
    volatile uint32_t* abort_flag = tmem_slot + 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::ST; ++s) {
            mbar_init(LBAR(C::B_LD + s), 1);
            mbar_init(LBAR(C::B_KE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(LBAR(C::B_AF + b), 1);
            mbar_init(LBAR(C::B_PF + b), C::NROW);
            mbar_init(LBAR(C::B_PVD + b), 1);
            mbar_init(LBAR(C::B_KVF + b), 1);
            mbar_init(LBAR(C::B_KVE + b), C::NSTATE);
            mbar_init(LBAR(C::B_SSF + b), C::NSTATE);
            mbar_init(LBAR(C::B_SE + b), 1);
            mbar_init(LBAR(C::B_OD + b), 1);
            mbar_init(LBAR(C::B_OE + b), C::NROW);
        }
        mbar_init(LBAR(C::B_DR), 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + C::OFF_MISC, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued[C::ST] = {0, 0};
            bool ok = true;
            for (int c = 0; c < nc; ++c) {
                const int s = c % C::ST, n = c / C::ST;
                if (n > 0 && !(ok = wait_bounded(LBAR(C::B_KE + s), (n - 1) & 1, abort_flag))) break;
                const uint32_t sq = base + s * C::STAGE, sk = sq + C::QK, sv = sk + C::QK;
                mbar_arrive_expect_tx(LBAR(C::B_LD + s), C::STAGE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_load_3d(sq + kb * 16384u, &tmQ, LBAR(C::B_LD + s), kb * 64, c * 128, bh);
                    tma_load_3d(sk + kb * 16384u, &tmK, LBAR(C::B_LD + s), kb * 64, c * 128, bh);
                }
                tma_load_3d(sv, &tmV, LBAR(C::B_LD + s), h * 64, c * 128, bh);
                issued[s] = n + 1;
            }
            if (!ok)  // let every copy in flight land before the CTA exits
                for (int s = 0; s < C::ST; ++s)
                    if (issued[s] > 0) wait_drain(LBAR(C::B_LD + s), (issued[s] - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID_A = idesc_f16(BF16, 128, 128, false, false);  // Q K^T
            constexpr uint32_t ID_KV = idesc_f16(BF16, 128, 64, true, true);    // K^T V_h
            constexpr uint32_t ID_O = idesc_f16(BF16, 128, 64, false, true);    // Q S, P V_h
            bool ok = true;
            for (int c = 0; ok && c < nc; ++c) {
                const int s = c % C::ST, n = c / C::ST, b = c & 1, u = c >> 1;
                const uint32_t sq = base + s * C::STAGE, sk = sq + C::QK, sv = sk + C::QK;
                // Q_c, K_c, V_c landed; A buffer b read by P V two chunks back;
                // KV buffer b read by the state warps two chunks back
                if (!(ok = wait3(LBAR(C::B_LD + s), n & 1, true, LBAR(C::B_PVD + b), (u - 1) & 1,
                                 c >= 2, LBAR(C::B_KVE + b), (u - 1) & 1, c >= 2, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // K-dim: 16 features per step
                    const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                    mma_ss(tmem + 128u * b, sdesc_sw128(sq + off, 16, 1024),
                           sdesc_sw128(sk + off, 16, 1024), ID_A, kk > 0 ? 1u : 0u);
                }
                mma_commit(LBAR(C::B_AF + b));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // K-dim: 16 tokens (2048 bytes) per step
                    mma_ss(tmem + C::COL_KV + 64u * b, sdesc_sw128(sk + kk * 2048u, 16384, 1024),
                           sdesc_sw128(sv + kk * 2048u, 16384, 1024), ID_KV, kk > 0 ? 1u : 0u);
                mma_commit(LBAR(C::B_KVF + b));
                // O_c = Q_c S_{c-1} into O buffer b: the row warps have read O_{c-2}
                // from it, and the state warps have stored S_{c-1} (buffer (c - 1) & 1)
                if (c >= 1) {
                    const int bp = (c - 1) & 1, up = (c - 1) >> 1;
                    if (!(ok = wait3(LBAR(C::B_OE + b), (u - 1) & 1, c >= 2, LBAR(C::B_SSF + bp),
                                     up & 1, true, 0u, 0u, false, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint32_t ss = base + C::OFF_S + bp * C::VH;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {  // B = S rows (features of K)
                        const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                        mma_ss(tmem + C::COL_O + 64u * b, sdesc_sw128(sq + off, 16, 1024),
                               sdesc_sw128(ss + kk * 2048u, 16384, 1024), ID_O, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(LBAR(C::B_SE + bp));  // S buffer bp may be rewritten
                }
                // O_c += P_c V_c,h once the row warps have written P_c: keys 0-63
                // packed at columns 0-31 of A buffer b, keys 64-127 at 64-95
                if (!(ok = wait_bounded(LBAR(C::B_PF + b), u & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // K-dim: 16 tokens per step
                    mma_ts(tmem + C::COL_O + 64u * b, tmem + 128u * b + kk * 8u + (kk >> 2) * 32u,
                           sdesc_sw128(sv + kk * 2048u, 16384, 1024), ID_O,
                           (c >= 1 || kk > 0) ? 1u : 0u);
                mma_commit(LBAR(C::B_OD + b));
                mma_commit(LBAR(C::B_PVD + b));
                mma_commit(LBAR(C::B_KE + s));
            }
            if (!ok) {  // every issued MMA must finish before tensor memory is freed
                mma_commit(LBAR(C::B_DR));
                wait_drain(LBAR(C::B_DR), 0);
            }
        }
        __syncwarp();
    } else if (warp < C::WARP_STATE) {
        // ----------------------------------------- P and the output (rows)
        const int hc = (warp - 2) >> 2;        // keys 64 hc.. of P, features 32 hc.. of O
        const int r = (warp & 3) * 32 + lane;  // row of the chunk == TMEM lane
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        // O_c (this half's 32 features) to the output rows; the buffer is
        // released as soon as the values are in registers
        auto store_o = [&](int c) -> bool {
            const int b = c & 1;
            if (!__all_sync(0xffffffffu, wait_bounded(LBAR(C::B_OD + b), (c >> 1) & 1, abort_flag)))
                return false;
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(lane_addr + C::COL_O + 64u * b + 32u * hc, v);
            tmem_ld_wait();
            reg_fence32(v);
            tc_fence_before();
            mbar_arrive(LBAR(C::B_OE + b));
            const int row = c * 128 + r;
            if (row < p.N) {
                uint32_t o16[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    o16[e] = pack2<BF16>(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.o) +
                                                      (static_cast<size_t>(bh) * p.N + row) * 256 +
                                                      h * 128 + hc * 64);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(o16[4 * e], o16[4 * e + 1], o16[4 * e + 2], o16[4 * e + 3]);
            }
            return true;
        };
        bool ok = true;
        for (int c = 0; ok && c < nc; ++c) {
            const int b = c & 1, u = c >> 1;
            ok = __all_sync(0xffffffffu, wait_bounded(LBAR(C::B_AF + b), u & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            // P_ij = scale A_ij for j <= i (rows and keys past N are zero already)
            const uint32_t col = 128u * b + 64u * hc;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t v[32], pk[16];
                tmem_ld32(lane_addr + col + cc * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int j0 = hc * 64 + cc * 32 + 2 * e;
                    pk[e] = pack2<BF16>(j0 <= r ? __uint_as_float(v[2 * e]) * p.scale : 0.f,
                                        j0 + 1 <= r ? __uint_as_float(v[2 * e + 1]) * p.scale : 0.f);
                }
                tmem_st16(lane_addr + col + cc * 16u, pk);  // over columns already read
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(LBAR(C::B_PF + b));
            if (c >= 1) ok = store_o(c - 1);
        }
        if (ok && nc > 0) store_o(nc - 1);
    } else {
        // ------------------------------------------------------ the state
        const int a = (warp & 3) * 32 + lane;  // feature of K == TMEM lane == row of S
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        float st[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) st[i] = 0.f;
        bool ok = true;
        for (int c = 0; ok && c < nc; ++c) {
            const int b = c & 1, u = c >> 1;
            ok = __all_sync(0xffffffffu, wait_bounded(LBAR(C::B_KVF + b), u & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t v[32];
                tmem_ld32(lane_addr + C::COL_KV + 64u * b + cc * 32u, v);
                tmem_ld_wait();
                reg_fence32(v);
#pragma unroll
                for (int e = 0; e < 32; ++e) st[cc * 32 + e] += __uint_as_float(v[e]);
            }
            tc_fence_before();
            mbar_arrive(LBAR(C::B_KVE + b));
            if (c == nc - 1) break;  // no chunk after the last reads its state
            // buffer b was last read by the Q S of chunk c - 1
            if (c >= 2)
                ok = __all_sync(0xffffffffu,
                                wait_bounded(LBAR(C::B_SE + b), (u - 1) & 1, abort_flag));
            if (!ok) break;
            // row a of S_c: 64 values, 128 bytes, eight 16-byte chunks placed by
            // the 128-byte swizzle (chunk j at j ^ (a mod 8))
            uint8_t* srow = gbase + C::OFF_S + b * C::VH + a * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 w = make_uint4(pack2<BF16>(st[8 * j] * p.scale, st[8 * j + 1] * p.scale),
                                           pack2<BF16>(st[8 * j + 2] * p.scale, st[8 * j + 3] * p.scale),
                                           pack2<BF16>(st[8 * j + 4] * p.scale, st[8 * j + 5] * p.scale),
                                           pack2<BF16>(st[8 * j + 6] * p.scale, st[8 * j + 7] * p.scale));
                *reinterpret_cast<uint4*>(srow + ((j ^ (a & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            mbar_arrive(LBAR(C::B_SSF + b));
        }
    }
#undef LBAR
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

constexpr uint32_t kLinKvSmem = 2 * kLinTile + 64 + 1024;
constexpr uint32_t kLinOutSmem = 4 * kLinTile + 128 + 1024;

}  // namespace attn

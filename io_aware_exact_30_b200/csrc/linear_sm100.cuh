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
// Three kernels, every chunk in parallel:
//   linear_kv_kernel      KV_c = K_c^T V_c (tcgen05, fp32 in tensor memory)
//                         written to a fp32 workspace;
//   linear_prefix_kernel  S_c = scale * sum_{c' < c} KV_c' (exclusive prefix
//                         over chunks, fp32 sums), stored in the input's
//                         16-bit type as the B operand of the next kernel;
//   linear_out_kernel     A = Q_c K_c^T (tensor memory), masked and scaled by
//                         the warps that own its rows and written back as P;
//                         O = Q_c S_c + P V_c (tensor memory), stored.
// Head dimension 128 only (the state product K^T V has M = d rows).
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

constexpr uint32_t kLinKvSmem = 2 * kLinTile + 64 + 1024;
constexpr uint32_t kLinOutSmem = 4 * kLinTile + 128 + 1024;

}  // namespace attn

// FP8 scores with incoherent processing: Q and K rows are rotated by a
// randomised Hadamard transform and quantised block-wise to e4m3 before the
// S = Q K^T product runs on the tensor cores at the FP8 rate.
//
// Method: "Is a full day of context better than ten minutes? FlashAttention
// and the sequence-length question" (marketmaker.cc), section "FA3: Hopper",
// third item: naive FP8 attention is hurt by outliers; rotating the vectors
// at random before block-wise quantisation spreads an outlier's magnitude over
// every coordinate (reported 2.6x lower error than naive FP8).  The page gives
// no formulas.  Taken here: y = H (s o x) per row, s a random +-1 vector (an
// input) and H the unnormalised d x d Sylvester-Hadamard matrix, so that
// (H s o q) . (H s o k) = d (q . k) exactly and the forward divides the scores
// by d; blocks of 128 rows of one head share one scale amax / 448; codes are
// e4m3(y * (448 / amax)), rounded to nearest even and saturated.  Every
// operation that decides a code is a single IEEE fp32 operation in a fixed
// order (the butterflies in ascending stride), so the codes are reproducible
// exactly.  Only S uses FP8; P V keeps the 16-bit V.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace attn {

// One CTA per (head, 128-row block) of x: 8 warps, each owning rows w, w + 8,
// ..; lane l holds elements E l .. E l + E - 1 of a row (E = D / 32), so a warp
// reads each row in one coalesced sweep and keeps its 16 rotated rows in
// registers until the block's amax is known.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) attn_fp8_quantize_kernel(
    const uint8_t* __restrict__ x, uint8_t* __restrict__ codes, float* __restrict__ scales,
    const int8_t* __restrict__ signs, int rotate, int N) {
    constexpr int E = D / 32;
    constexpr int RPW = 16;  // rows per warp
    __shared__ float warp_max[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = (N + 127) / 128;
    const int bh = blockIdx.x / nb, blk = blockIdx.x % nb;
    const int row0 = blk * 128;
    float sgn[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sgn[e] = (signs != nullptr && signs[lane * E + e] < 0) ? -1.f : 1.f;

    // every row's load is issued before the first is used, so that a warp has
    // all 16 in flight (the kernel is bound by HBM latency and bandwidth)
    uint32_t raw[RPW][E / 2];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = row0 + warp + 8 * i;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) raw[i][e] = 0u;
        if (r < N) {
            const size_t off = (static_cast<size_t>(bh) * N + r) * D + lane * E;  // elements
            if constexpr (E == 4) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(x + off * 2));
                raw[i][0] = w.x;
                raw[i][1] = w.y;
            } else {
                raw[i][0] = __ldg(reinterpret_cast<const uint32_t*>(x + off * 2));
            }
        }
    }
    float y[RPW][E];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const float2 v = unpack2<BF16>(raw[i][e / 2]);
            y[i][e] = v.x * sgn[e];
            y[i][e + 1] = v.y * sgn[e + 1];
        }
        if (rotate) {
            // butterflies of stride h < E inside the thread, then stride E m
            // (m = 1 .. 16) with the lane that differs in bit m
#pragma unroll
            for (int h = 1; h < E; h *= 2)
#pragma unroll
                for (int b = 0; b < E; b += 2 * h)
#pragma unroll
                    for (int j = b; j < b + h; ++j) {
                        const float a = y[i][j], c = y[i][j + h];
                        y[i][j] = __fadd_rn(a, c);
                        y[i][j + h] = __fsub_rn(a, c);
                    }
#pragma unroll
            for (int m = 1; m < 32; m *= 2) {
                const bool high = (lane & m) != 0;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float other = __shfl_xor_sync(0xffffffffu, y[i][e], m);
                    y[i][e] = high ? __fsub_rn(other, y[i][e]) : __fadd_rn(y[i][e], other);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[i][e]));
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    if (lane == 0) warp_max[warp] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    if (threadIdx.x == 0) scales[static_cast<size_t>(bh) * nb + blk] = __fdiv_rn(amax, 448.f);
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = row0 + warp + 8 * i;
        if (r >= N) continue;
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
                make_float2(__fmul_rn(y[i][e], inv), __fmul_rn(y[i][e + 1], inv)),
                __NV_SATFINITE, __NV_E4M3);
            packed |= static_cast<uint32_t>(c) << (8 * e);
        }
        uint8_t* dst = codes + (static_cast<size_t>(bh) * N + r) * D + lane * E;
        if constexpr (E == 4)
            *reinterpret_cast<uint32_t*>(dst) = packed;
        else
            *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
    }
}

}  // namespace attn

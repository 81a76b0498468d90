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

// One CTA per (head, 128-row block) of x: 16 warps, each owning 8 rows; four
// lanes share a row, lane l holding its elements E q .. E q + E - 1 (q = l mod
// 4, E = D / 4), so that all but the two widest butterfly strides stay inside
// a thread (the cross-lane strides go through shuffles, the unit that bounds
// this kernel).  A warp reads its 8 rows in one coalesced sweep and keeps them
// in registers until the block's amax is known.  The arithmetic per element
// and the ascending order of the strides are those of any other layout, so the
// codes do not depend on it.
template <int D, bool BF16>
__global__ void __launch_bounds__(512) attn_fp8_quantize_kernel(
    const uint8_t* __restrict__ x, uint8_t* __restrict__ codes, float* __restrict__ scales,
    const int8_t* __restrict__ signs, int rotate, int N) {
    constexpr int E = D / 4;  // elements per lane
    __shared__ float warp_max[16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane & 3;  // quarter of the row this lane holds
    const int nb = (N + 127) / 128;
    const int bh = blockIdx.x / nb, blk = blockIdx.x % nb;
    const int r = blk * 128 + warp * 8 + (lane >> 2);
    // bit e: the sign of element E q + e is negative (flipping the sign bit is
    // the exact product with -1)
    uint32_t neg = 0u;
    if (signs != nullptr) {
#pragma unroll
        for (int e = 0; e < E; ++e) neg |= (signs[q * E + e] < 0 ? 1u : 0u) << e;
    }
    uint32_t raw[E / 2];
#pragma unroll
    for (int e = 0; e < E / 2; ++e) raw[e] = 0u;
    if (r < N) {
        const uint4* src = reinterpret_cast<const uint4*>(
            x + ((static_cast<size_t>(bh) * N + r) * D + q * E) * 2);
#pragma unroll
        for (int w = 0; w < E / 8; ++w) {
            const uint4 v = __ldg(src + w);
            raw[4 * w] = v.x, raw[4 * w + 1] = v.y, raw[4 * w + 2] = v.z, raw[4 * w + 3] = v.w;
        }
    }
    float y[E];
#pragma unroll
    for (int e = 0; e < E; e += 2) {
        const float2 v = unpack2<BF16>(raw[e / 2]);
        y[e] = __int_as_float(__float_as_int(v.x) ^ static_cast<int>(((neg >> e) & 1u) << 31));
        y[e + 1] = __int_as_float(__float_as_int(v.y) ^ static_cast<int>(((neg >> (e + 1)) & 1u) << 31));
    }
    if (rotate) {
        // butterflies of stride h < E inside the thread, then strides E and 2 E
        // with the lane of the same row that differs in bit 0, then bit 1
#pragma unroll
        for (int h = 1; h < E; h *= 2)
#pragma unroll
            for (int b = 0; b < E; b += 2 * h)
#pragma unroll
                for (int j = b; j < b + h; ++j) {
                    const float a = y[j], c = y[j + h];
                    y[j] = __fadd_rn(a, c);
                    y[j + h] = __fsub_rn(a, c);
                }
#pragma unroll
        for (int m = 1; m < 4; m *= 2) {
            const bool high = (q & m) != 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float other = __shfl_xor_sync(0xffffffffu, y[e], m);
                y[e] = high ? __fsub_rn(other, y[e]) : __fadd_rn(y[e], other);
            }
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[e]));
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    if (lane == 0) warp_max[warp] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < 16; ++w) amax = fmaxf(amax, warp_max[w]);
    const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    if (threadIdx.x == 0) scales[static_cast<size_t>(bh) * nb + blk] = __fdiv_rn(amax, 448.f);
    if (r >= N) return;
    uint32_t packed[E / 4];
#pragma unroll
    for (int w = 0; w < E / 4; ++w) {
        uint32_t word = 0u;
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
                make_float2(__fmul_rn(y[4 * w + e], inv), __fmul_rn(y[4 * w + e + 1], inv)),
                __NV_SATFINITE, __NV_E4M3);
            word |= static_cast<uint32_t>(c) << (8 * e);
        }
        packed[w] = word;
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + (static_cast<size_t>(bh) * N + r) * D + q * E);
#pragma unroll
    for (int w = 0; w < E / 16; ++w)
        dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1], packed[4 * w + 2], packed[4 * w + 3]);
}

}  // namespace attn

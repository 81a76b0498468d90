// Dropout on the attention probabilities, regenerated identically in the
// forward and the backward from a counter-based generator.
//
// The attention call of "Is a full day of context better than ten minutes?"
// (marketmaker.cc), section "integration is eight lines", takes dropout_p.
// Taken here: P_ij is kept with probability t / 256 and then scaled by
// 256 / t (t = round(256 (1 - p)) in 1 .. 256), else zeroed; the softmax
// statistics (and the stored LSE) are those of P before dropout.  The random
// byte r_ij of (head bh, query i, key j) is byte j % 16 of Philox4x32-10
// (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC 2011) with key (seed low, seed high) and counter (j / 16, i, bh, 0): word
// (j % 16) / 4, little-endian byte j % 4; P_ij is kept iff r_ij < t.
#pragma once

#include <cstdint>

namespace attn {

// Philox4x32 with 10 rounds: words 0 and 2 of the counter are multiplied by
// the generator's two constants, the high and low halves are mixed with the
// other words and the key, and the key advances by the two Weyl increments.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

struct DropoutParams {
    uint32_t seed_lo, seed_hi;
    uint32_t thr;  // keep iff byte < thr; 256 keeps everything
    float inv_keep;  // 256 / thr
};

// Random bytes of keys 16 g .. 16 g + 15 for query row i of head bh: byte e
// (key 16 g + e) is byte e % 4 of word e / 4.
__device__ __forceinline__ uint4 dropout_bytes16(const DropoutParams& dp, uint32_t bh, uint32_t i,
                                                 uint32_t g) {
    return philox4x32_10(make_uint4(g, i, bh, 0u), dp.seed_lo, dp.seed_hi);
}

// 0xFF in each byte of the result where the byte of `bytes` is below thr
// (thr <= 255), 0x00 elsewhere.
__device__ __forceinline__ uint32_t keep_bytes(uint32_t bytes, uint32_t thr4) {
    return __vcmpltu4(bytes, thr4);
}

// Transposes a 32 x 32 byte matrix held by a warp: on entry lane L holds row L
// as 8 words (byte k of the row = byte k % 4 of word k / 4); on exit lane L
// holds column L in the same form.  Five butterfly stages: at stride m the
// lanes L and L ^ m swap the bytes whose index differs from the lane in bit m.
__device__ __forceinline__ void warp_transpose_bytes(uint32_t (&w)[8]) {
    const int lane = threadIdx.x & 31;
    // index bits 4, 3, 2: whole words (word index bits 2, 1, 0)
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        const int m = 16 >> s, tb = 2 - s;
        const bool hi = (lane & m) != 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            if (t & (1 << tb)) continue;
            const int u = t | (1 << tb);
            const uint32_t send = hi ? w[t] : w[u];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
            if (hi)
                w[t] = recv;
            else
                w[u] = recv;
        }
    }
    // index bit 1: byte pairs {0, 1} and {2, 3} of every word
    {
        const bool hi = (lane & 2) != 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t send = hi ? (w[t] & 0xFFFFu) : (w[t] >> 16);
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 2);
            w[t] = hi ? ((w[t] & 0xFFFF0000u) | recv) : ((w[t] & 0xFFFFu) | (recv << 16));
        }
    }
    // index bit 0: bytes {0, 2} and {1, 3} of every word
    {
        const bool hi = (lane & 1) != 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const uint32_t send = hi ? (w[t] & 0x00FF00FFu) : ((w[t] >> 8) & 0x00FF00FFu);
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 1);
            w[t] = hi ? ((w[t] & 0xFF00FF00u) | recv) : ((w[t] & 0x00FF00FFu) | (recv << 8));
        }
    }
}

// Keep masks of a warp whose lane holds key j0 + lane (j0 a multiple of 32)
// against queries i0 .. i0 + 31: byte c of the returned words (word c / 4) is
// 0xFF where P(i0 + c, j0 + lane) is kept.  Each lane generates the bytes of
// its own query i0 + lane for the warp's 32 keys (two generator calls), then
// the warp transposes them.
__device__ __forceinline__ void dropout_keep_keyrows(const DropoutParams& dp, uint32_t bh,
                                                     uint32_t i0, uint32_t j0,
                                                     uint32_t (&keep)[8]) {
    const uint32_t lane = threadIdx.x & 31;
    const uint4 a = dropout_bytes16(dp, bh, i0 + lane, j0 / 16);
    const uint4 b = dropout_bytes16(dp, bh, i0 + lane, j0 / 16 + 1);
    keep[0] = a.x, keep[1] = a.y, keep[2] = a.z, keep[3] = a.w;
    keep[4] = b.x, keep[5] = b.y, keep[6] = b.z, keep[7] = b.w;
    warp_transpose_bytes(keep);
    const uint32_t thr4 = dp.thr * 0x01010101u;
#pragma unroll
    for (int t = 0; t < 8; ++t) keep[t] = keep_bytes(keep[t], thr4);
}

}  // namespace attn

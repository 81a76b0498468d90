/*
 * fp64 CPU oracle for exact scaled-dot-product attention, forward and
 * backward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the CUDA product path never does.
 * It shares no code, header or constant with the GPU library.
 *
 * Sources (titles of the pages, section named):
 *  - "Is a full day of context better than ten minutes? FlashAttention and the
 *    sequence-length question" (marketmaker.cc), section "why attention is
 *    bound by memory": O = softmax(Q K^T / sqrt(d_k)) V.
 *    Same page, "online softmax recurrence": a naive softmax takes two passes
 *    over a row, one for the maximum and one to exponentiate and normalise;
 *    the tiled method is algebraically the same result.
 *    Same page, "causal masking": a query never attends to a later key.
 *    Same page, "Flash Attention algorithm" (the per-block pseudo-code):
 *    restated by oracle_fwd_online below as a self-check only.
 *    Same page, "backward: recompute instead of store": gradients need P,
 *    rebuilt from the stored statistics.
 *  - "Performance optimisation with Flash-Attention 2" (Medium), section
 *    "Flash Attention 2": one statistic L (the log-sum-exp) is kept per row.
 *
 * The forward is the plain definition, row by row, in two passes (maximum,
 * then exponentiate/normalise); the score row is the only O(N) scratch.  The
 * backward is the analytic chain rule of L = sum(O * dO), row by row, with no
 * N x N storage; rows run in parallel (OpenMP) with per-thread dK/dV partials
 * that are summed at the end of each head.
 *
 * Conventions: every tensor is contiguous (BH, N, d) float64, LSE is (BH, N);
 * key j is visible to query i iff !causal || j <= i; LSE is natural-log.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double dot(const double* a, const double* b, int64_t d) {
    double s = 0.0;
    for (int64_t k = 0; k < d; ++k) s += a[k] * b[k];
    return s;
}

/* One query row: fills s[0..nvis) with probabilities, returns LSE, writes O. */
static double row_forward(const double* qi, const double* K, const double* V, int64_t nvis,
                          int64_t d, double scale, double* s, double* oi) {
    double M = -INFINITY;
    for (int64_t j = 0; j < nvis; ++j) {          /* scores and pass 1: max */
        s[j] = scale * dot(qi, K + j * d, d);
        if (s[j] > M) M = s[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < nvis; ++j) {          /* pass 2: exponentiate, sum */
        s[j] = exp(s[j] - M);
        Z += s[j];
    }
    for (int64_t k = 0; k < d; ++k) oi[k] = 0.0;
    for (int64_t j = 0; j < nvis; ++j) {          /* normalise, weight V */
        s[j] /= Z;
        const double* vj = V + j * d;
        for (int64_t k = 0; k < d; ++k) oi[k] += s[j] * vj[k];
    }
    return M + log(Z);
}

static int64_t visible(int64_t i, int64_t N, int causal) { return causal ? i + 1 : N; }

/* Forward on a list of rows; rows[r] = bh * N + i.  o_rows is (nrows, d). */
void oracle_fwd_rows(const double* q, const double* k, const double* v, int64_t BH, int64_t N,
                     int64_t d, int causal, double scale, const int64_t* rows, int64_t nrows,
                     double* o_rows, double* lse_rows) {
    (void)BH;
#pragma omp parallel
    {
        double* s = (double*)malloc((size_t)N * sizeof(double));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t bh = rows[r] / N, i = rows[r] % N;
            const double* base_k = k + bh * N * d;
            const double* base_v = v + bh * N * d;
            lse_rows[r] = row_forward(q + rows[r] * d, base_k, base_v, visible(i, N, causal), d,
                                      scale, s, o_rows + r * d);
        }
        free(s);
    }
}

/* Full forward: O (BH, N, d), LSE (BH, N). */
void oracle_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
                int64_t BH, int64_t N, int64_t d, int causal, double scale) {
#pragma omp parallel
    {
        double* s = (double*)malloc((size_t)N * sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < N; ++i) {
                int64_t row = bh * N + i;
                lse[row] = row_forward(q + row * d, k + bh * N * d, v + bh * N * d,
                                       visible(i, N, causal), d, scale, s, o + row * d);
            }
        free(s);
    }
}

/*
 * The page's per-block pseudo-code, literally: for each query row, walk the
 * key/value blocks of width Bc, keep (m, l) and an O that is normalised after
 * every block (FA1 form).  Blocks lying entirely in the future of the row are
 * skipped, as the causal-masking section describes.  Self-check only.
 */
void oracle_fwd_online(const double* q, const double* k, const double* v, double* o, double* lse,
                       int64_t BH, int64_t N, int64_t d, int causal, double scale, int64_t Bc) {
#pragma omp parallel
    {
        double* p = (double*)malloc((size_t)Bc * sizeof(double));
        double* pv = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < N; ++i) {
                const double* qi = q + (bh * N + i) * d;
                double* oi = o + (bh * N + i) * d;
                double m = -INFINITY, l = 0.0;
                for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
                for (int64_t j0 = 0; j0 < N; j0 += Bc) {
                    if (causal && j0 > i) break;           /* whole block in the future */
                    int64_t j1 = j0 + Bc < N ? j0 + Bc : N;
                    double mij = -INFINITY;
                    for (int64_t j = j0; j < j1; ++j) {    /* S_ij and its row max */
                        int vis = !causal || j <= i;
                        p[j - j0] = vis ? scale * dot(qi, k + (bh * N + j) * d, d) : -INFINITY;
                        if (p[j - j0] > mij) mij = p[j - j0];
                    }
                    double lij = 0.0;
                    for (int64_t j = j0; j < j1; ++j) {    /* P_ij = exp(S_ij - m_ij), l_ij */
                        p[j - j0] = exp(p[j - j0] - mij);
                        lij += p[j - j0];
                    }
                    for (int64_t t = 0; t < d; ++t) pv[t] = 0.0;
                    for (int64_t j = j0; j < j1; ++j) {    /* P_ij V_j */
                        const double* vj = v + (bh * N + j) * d;
                        for (int64_t t = 0; t < d; ++t) pv[t] += p[j - j0] * vj[t];
                    }
                    double mnew = m > mij ? m : mij;
                    double a = exp(m - mnew), b = exp(mij - mnew);
                    double lnew = l * a + lij * b;
                    for (int64_t t = 0; t < d; ++t)
                        oi[t] = oi[t] * (l * a / lnew) + pv[t] * (b / lnew);
                    m = mnew;
                    l = lnew;
                }
                lse[bh * N + i] = m + log(l);
            }
        free(pv);
        free(p);
    }
}

/*
 * Backward of L = sum(O * dO) for the heads listed in heads[0..nheads):
 * dq/dk/dv are (nheads, N, d), in the order of heads[].  The forward
 * quantities (P row, O row, D_i) are recomputed here in fp64 from q, k, v, so
 * the result is the exact gradient of the definition.
 *
 *   P_ij = softmax_j(s_ij),  s_ij = scale q_i.k_j (visible j only)
 *   D_i  = sum_t dO_it O_it            ( = sum_j P_ij dP_ij )
 *   dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i)
 *   dq_i = scale sum_j dS_ij k_j,  dk_j += scale dS_ij q_i,  dv_j += P_ij dO_i
 */
void oracle_bwd_heads(const double* q, const double* k, const double* v, const double* dout,
                      int64_t BH, int64_t N, int64_t d, int causal, double scale,
                      const int64_t* heads, int64_t nheads, double* dq, double* dk, double* dv) {
    (void)BH;
    int nthr = 1;
#ifdef _OPENMP
    nthr = omp_get_max_threads();
#endif
    size_t nd = (size_t)N * (size_t)d;
    double* part = (double*)calloc((size_t)nthr * 2 * nd, sizeof(double));
    for (int64_t hh = 0; hh < nheads; ++hh) {
        int64_t bh = heads[hh];
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        const double* dO = dout + bh * N * d;
        double* dQ = dq + hh * N * d;
        memset(part, 0, (size_t)nthr * 2 * nd * sizeof(double));
#pragma omp parallel
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double* dKp = part + (size_t)tid * 2 * nd;
            double* dVp = dKp + nd;
            double* p = (double*)malloc((size_t)N * sizeof(double));
            double* oi = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < N; ++i) {
                int64_t nv = visible(i, N, causal);
                const double* qi = Q + i * d;
                const double* doi = dO + i * d;
                row_forward(qi, K, V, nv, d, scale, p, oi);
                double Di = dot(doi, oi, d);
                double* dqi = dQ + i * d;
                for (int64_t t = 0; t < d; ++t) dqi[t] = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    const double* vj = V + j * d;
                    const double* kj = K + j * d;
                    double dpij = dot(doi, vj, d);
                    double dsij = p[j] * (dpij - Di);
                    double* dkj = dKp + j * d;
                    double* dvj = dVp + j * d;
                    for (int64_t t = 0; t < d; ++t) {
                        dqi[t] += scale * dsij * kj[t];
                        dkj[t] += scale * dsij * qi[t];
                        dvj[t] += p[j] * doi[t];
                    }
                }
            }
            free(oi);
            free(p);
        }
        double* dK = dk + hh * N * d;
        double* dV = dv + hh * N * d;
        for (size_t e = 0; e < nd; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int t = 0; t < nthr; ++t) {
                sk += part[(size_t)t * 2 * nd + e];
                sv += part[(size_t)t * 2 * nd + nd + e];
            }
            dK[e] = sk;
            dV[e] = sv;
        }
    }
    free(part);
}

/*
 * Block-sparse attention: "FlashAttention の概要" (zenn.dev), the paragraph on
 * Block-Sparse FlashAttention, which approximates attention by computing only
 * the (query block, key block) pairs a block mask marks and is otherwise the
 * same algorithm.  The page describes no more; the readings taken here:
 *  - one mask for every (batch, head): mask[(i / blk) * nb + (j / blk)] != 0
 *    marks the pair of query block i / blk and key block j / blk, with
 *    nb = ceil(N / blk) blocks per side;
 *  - key j is visible to query i iff its block pair is marked and, with the
 *    causal flag, j <= i (the causal rule of "causal masking" on the
 *    marketmaker.cc page still applies inside marked blocks);
 *  - over the visible keys the result is exact softmax attention; a row with
 *    no visible key has O = 0 and LSE = -inf (the empty sum).
 * The forward and backward below are the definitions above written out on an
 * explicit list of each row's visible keys.
 */
static int64_t visible_list(int64_t i, int64_t N, int causal, const uint8_t* mask, int64_t blk,
                            int64_t* idx) {
    int64_t nb = (N + blk - 1) / blk, n = 0;
    for (int64_t j = 0; j < N; ++j)
        if (mask[(i / blk) * nb + j / blk] && (!causal || j <= i)) idx[n++] = j;
    return n;
}

/* One query row over the keys idx[0..nvis): s[0..nvis) gets P, returns LSE. */
static double row_forward_list(const double* qi, const double* K, const double* V,
                               const int64_t* idx, int64_t nvis, int64_t d, double scale,
                               double* s, double* oi) {
    for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
    if (nvis == 0) return -INFINITY;
    double M = -INFINITY;
    for (int64_t r = 0; r < nvis; ++r) {          /* scores and pass 1: max */
        s[r] = scale * dot(qi, K + idx[r] * d, d);
        if (s[r] > M) M = s[r];
    }
    double Z = 0.0;
    for (int64_t r = 0; r < nvis; ++r) {          /* pass 2: exponentiate, sum */
        s[r] = exp(s[r] - M);
        Z += s[r];
    }
    for (int64_t r = 0; r < nvis; ++r) {          /* normalise, weight V */
        s[r] /= Z;
        const double* vj = V + idx[r] * d;
        for (int64_t t = 0; t < d; ++t) oi[t] += s[r] * vj[t];
    }
    return M + log(Z);
}

/* Block-sparse forward: O (BH, N, d), LSE (BH, N). */
void oracle_fwd_blocksparse(const double* q, const double* k, const double* v, double* o,
                            double* lse, int64_t BH, int64_t N, int64_t d, int causal,
                            double scale, const uint8_t* mask, int64_t blk) {
#pragma omp parallel
    {
        double* s = (double*)malloc((size_t)N * sizeof(double));
        int64_t* idx = (int64_t*)malloc((size_t)N * sizeof(int64_t));
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < N; ++i) {
                int64_t row = bh * N + i;
                int64_t nv = visible_list(i, N, causal, mask, blk, idx);
                lse[row] = row_forward_list(q + row * d, k + bh * N * d, v + bh * N * d, idx, nv,
                                            d, scale, s, o + row * d);
            }
        free(idx);
        free(s);
    }
}

/* Block-sparse backward of L = sum(O * dO) for the listed heads; same chain
 * rule as oracle_bwd_heads, over each row's visible keys only. */
void oracle_bwd_blocksparse_heads(const double* q, const double* k, const double* v,
                                  const double* dout, int64_t BH, int64_t N, int64_t d,
                                  int causal, double scale, const uint8_t* mask, int64_t blk,
                                  const int64_t* heads, int64_t nheads, double* dq, double* dk,
                                  double* dv) {
    (void)BH;
    int nthr = 1;
#ifdef _OPENMP
    nthr = omp_get_max_threads();
#endif
    size_t nd = (size_t)N * (size_t)d;
    double* part = (double*)calloc((size_t)nthr * 2 * nd, sizeof(double));
    for (int64_t hh = 0; hh < nheads; ++hh) {
        int64_t bh = heads[hh];
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        const double* dO = dout + bh * N * d;
        double* dQ = dq + hh * N * d;
        memset(part, 0, (size_t)nthr * 2 * nd * sizeof(double));
#pragma omp parallel
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double* dKp = part + (size_t)tid * 2 * nd;
            double* dVp = dKp + nd;
            double* p = (double*)malloc((size_t)N * sizeof(double));
            int64_t* idx = (int64_t*)malloc((size_t)N * sizeof(int64_t));
            double* oi = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < N; ++i) {
                int64_t nv = visible_list(i, N, causal, mask, blk, idx);
                const double* qi = Q + i * d;
                const double* doi = dO + i * d;
                row_forward_list(qi, K, V, idx, nv, d, scale, p, oi);
                double Di = dot(doi, oi, d);
                double* dqi = dQ + i * d;
                for (int64_t t = 0; t < d; ++t) dqi[t] = 0.0;
                for (int64_t r = 0; r < nv; ++r) {
                    int64_t j = idx[r];
                    const double* vj = V + j * d;
                    const double* kj = K + j * d;
                    double dpij = dot(doi, vj, d);
                    double dsij = p[r] * (dpij - Di);
                    double* dkj = dKp + j * d;
                    double* dvj = dVp + j * d;
                    for (int64_t t = 0; t < d; ++t) {
                        dqi[t] += scale * dsij * kj[t];
                        dkj[t] += scale * dsij * qi[t];
                        dvj[t] += p[r] * doi[t];
                    }
                }
            }
            free(oi);
            free(idx);
            free(p);
        }
        double* dK = dk + hh * N * d;
        double* dV = dv + hh * N * d;
        for (size_t e = 0; e < nd; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int t = 0; t < nthr; ++t) {
                sk += part[(size_t)t * 2 * nd + e];
                sv += part[(size_t)t * 2 * nd + nd + e];
            }
            dK[e] = sk;
            dV[e] = sv;
        }
    }
    free(part);
}

/*
 * FP8 with incoherent processing: "Is a full day of context better than ten
 * minutes?" (marketmaker.cc), section "FA3: Hopper", third item: naive FP8
 * attention is hurt by outliers, so the vectors are randomly rotated before
 * block-wise quantisation, which spreads an outlier's magnitude over all
 * coordinates (reported 2.6x lower error than naive FP8).  The page gives no
 * formulas; the readings taken:
 *  - the rotation is a randomised Hadamard transform of each row of Q and K
 *    along the head dimension: y = H (s o x), with s a random +-1 vector (an
 *    input) and H the d x d Sylvester-Hadamard matrix, unnormalised (entries
 *    +-1).  H^T H = d I, so (H s o q) . (H s o k) = d (q . k): the scores are
 *    recovered exactly by dividing by d, and no rounding is added by a
 *    1/sqrt(d) factor.  Without rotation (naive FP8) y = x.
 *  - quantisation is per block of 128 rows of one (batch, head): amax = max
 *    |y| over the block, codes e4m3(y * (448 / amax)) rounded to nearest even
 *    with saturation, dequantisation scale amax / 448 (a block of zeros gets
 *    scale 0 and codes 0);
 *  - only the S = Q K^T product runs in FP8; P V keeps the 16-bit V.
 * The rotation and quantisation decide integer codes, so they are taken in
 * fp32 exactly as stated (the butterflies below in this order, IEEE single
 * operations), the precision the kernel uses; the attention on the
 * dequantised values is then the exact two-pass definition in fp64.
 */

/* fp32 -> nearest e4m3 value (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; normals 2^-6 .. 448, subnormals multiples of 2^-9), ties to even,
 * magnitudes beyond 448 saturate to 448.  Returned as a float (exact). */
float oracle_e4m3_round(float x) {
    if (x != x) return x;
    double a = fabs((double)x), r;
    if (a >= 448.0) {
        r = 448.0;
    } else if (a < 0.015625) {                  /* below 2^-6: subnormal grid 2^-9 */
        r = nearbyint(a * 512.0) / 512.0;
    } else {
        int e;
        frexp(a, &e);                           /* a = f 2^e, f in [0.5, 1) */
        double quantum = ldexp(1.0, e - 4);     /* 3 mantissa bits below 2^(e-1) */
        r = nearbyint(a / quantum) * quantum;
        if (r > 448.0) r = 448.0;
    }
    return (float)(x < 0 ? -r : r);
}

/* In-place Walsh-Hadamard butterflies on d floats (d a power of two), in fp32:
 * for h = 1, 2, 4, ..: (x[j], x[j + h]) <- (x[j] + x[j + h], x[j] - x[j + h]). */
static void fwht32(float* x, int64_t d) {
    for (int64_t h = 1; h < d; h *= 2)
        for (int64_t i = 0; i < d; i += 2 * h)
            for (int64_t j = i; j < i + h; ++j) {
                float a = x[j], b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
}

void oracle_fwht32(float* x, int64_t rows, int64_t d) {
    for (int64_t r = 0; r < rows; ++r) fwht32(x + r * d, d);
}

/*
 * Quantise x (BH, N, d; values exactly representable in fp32) as described
 * above: codes (BH, N, d) as e4m3 values, scales (BH, ceil(N / 128)).
 * signs: d entries +-1 (NULL: no sign flip); rotate: apply H.
 */
void oracle_fp8_quantize(const double* x, int64_t BH, int64_t N, int64_t d,
                         const int8_t* signs, int rotate, float* codes, float* scales) {
    int64_t nb = (N + 127) / 128;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t b = 0; b < nb; ++b) {
            int64_t r0 = b * 128, r1 = r0 + 128 < N ? r0 + 128 : N;
            float* y = codes + (bh * N + r0) * d;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r) {
                float* yr = y + (r - r0) * d;
                for (int64_t t = 0; t < d; ++t) {
                    float v = (float)x[(bh * N + r) * d + t];
                    yr[t] = signs ? (signs[t] < 0 ? -v : v) : v;
                }
                if (rotate) fwht32(yr, d);
                for (int64_t t = 0; t < d; ++t) {
                    float m = fabsf(yr[t]);
                    if (m > amax) amax = m;
                }
            }
            float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
            for (int64_t e = 0; e < (r1 - r0) * d; ++e) {
                float t = y[e] * inv;
                y[e] = oracle_e4m3_round(t);
            }
            scales[bh * nb + b] = amax / 448.0f;
        }
}

/*
 * Dropout on the attention probabilities: the page's integration example
 * ("Is a full day of context better than ten minutes?" (marketmaker.cc),
 * section "integration is eight lines") passes dropout_p to the attention
 * call during training.  The page gives no more; the readings taken:
 *  - each probability P_ij (after the softmax, whose statistics and LSE are
 *    unchanged) is kept with probability 1 - p and scaled by 1 / (1 - p), or
 *    set to 0: O_i = sum_j P_ij Z_ij / (1 - p) V_j, Z_ij in {0, 1};
 *  - Z comes from a counter-based generator, Philox4x32-10 (Salmon, Moraes,
 *    Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
 *    with key (seed low 32 bits, seed high 32 bits) and counter
 *    (j / 16, i, b H + h, 0): byte j % 16 of its four output words (word
 *    (j % 16) / 4, little-endian byte j % 4) is the random byte r_ij, and
 *    Z_ij = [r_ij < t] with the 8-bit threshold t = round(256 (1 - p)) in
 *    1 .. 256, so the keep probability is t / 256 and kept values are scaled
 *    by 256 / t (p is taken to the nearest multiple of 1/256);
 *  - the backward differentiates that: dV_j = sum_i P_ij Z_ij (256/t) dO_i,
 *    dP_ij = Z_ij (256/t) dO_i . v_j, D_i = dO_i . O_i (still sum_j P_ij
 *    dP_ij), dS_ij = P_ij (dP_ij - D_i), dQ and dK as without dropout.
 */
static uint32_t mulhilo32(uint32_t a, uint32_t b, uint32_t* hi) {
    uint64_t p = (uint64_t)a * (uint64_t)b;
    *hi = (uint32_t)(p >> 32);
    return (uint32_t)p;
}

/* Philox4x32 with 10 rounds: the round multiplies counter words 0 and 2 by the
 * paper's constants and mixes the halves with the key; the key is bumped by
 * the two Weyl constants between rounds. */
void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        uint32_t hi0, hi1;
        uint32_t lo0 = mulhilo32(0xD2511F53u, c0, &hi0);
        uint32_t lo1 = mulhilo32(0xCD9E8D57u, c2, &hi1);
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static int dropout_keep(uint64_t seed, int64_t bh, int64_t i, int64_t j, int thr) {
    uint32_t ctr[4] = {(uint32_t)(j >> 4), (uint32_t)i, (uint32_t)bh, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    uint32_t byte = (w[(j & 15) >> 2] >> (8 * (j & 3))) & 0xFFu;
    return (int)byte < thr;
}

/* The dropout mask Z (BH, N, N) as bytes, for tests. */
void oracle_dropout_mask(int64_t BH, int64_t N, uint64_t seed, int thr, uint8_t* z) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < N; ++i)
            for (int64_t j = 0; j < N; ++j)
                z[(bh * N + i) * N + j] = (uint8_t)dropout_keep(seed, bh, i, j, thr);
}

/* Forward with dropout: O (BH, N, d), LSE (BH, N) (LSE of the softmax itself). */
void oracle_fwd_dropout(const double* q, const double* k, const double* v, double* o,
                        double* lse, int64_t BH, int64_t N, int64_t d, int causal, double scale,
                        uint64_t seed, int thr) {
    double inv_keep = 256.0 / (double)thr;
#pragma omp parallel
    {
        double* s = (double*)malloc((size_t)N * sizeof(double));
        double* tmp = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (int64_t bh = 0; bh < BH; ++bh)
            for (int64_t i = 0; i < N; ++i) {
                int64_t row = bh * N + i, nv = visible(i, N, causal);
                lse[row] = row_forward(q + row * d, k + bh * N * d, v + bh * N * d, nv, d, scale,
                                       s, tmp);
                double* oi = o + row * d;
                for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    if (!dropout_keep(seed, bh, i, j, thr)) continue;
                    const double* vj = v + (bh * N + j) * d;
                    for (int64_t t = 0; t < d; ++t) oi[t] += s[j] * inv_keep * vj[t];
                }
            }
        free(tmp);
        free(s);
    }
}

/* Backward with dropout for the listed heads (the chain rule above). */
void oracle_bwd_dropout_heads(const double* q, const double* k, const double* v,
                              const double* dout, int64_t BH, int64_t N, int64_t d, int causal,
                              double scale, uint64_t seed, int thr, const int64_t* heads,
                              int64_t nheads, double* dq, double* dk, double* dv) {
    (void)BH;
    double inv_keep = 256.0 / (double)thr;
    int nthr = 1;
#ifdef _OPENMP
    nthr = omp_get_max_threads();
#endif
    size_t nd = (size_t)N * (size_t)d;
    double* part = (double*)calloc((size_t)nthr * 2 * nd, sizeof(double));
    for (int64_t hh = 0; hh < nheads; ++hh) {
        int64_t bh = heads[hh];
        const double* Q = q + bh * N * d;
        const double* K = k + bh * N * d;
        const double* V = v + bh * N * d;
        const double* dO = dout + bh * N * d;
        double* dQ = dq + hh * N * d;
        memset(part, 0, (size_t)nthr * 2 * nd * sizeof(double));
#pragma omp parallel
        {
            int tid = 0;
#ifdef _OPENMP
            tid = omp_get_thread_num();
#endif
            double* dKp = part + (size_t)tid * 2 * nd;
            double* dVp = dKp + nd;
            double* p = (double*)malloc((size_t)N * sizeof(double));
            double* oi = (double*)malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < N; ++i) {
                int64_t nv = visible(i, N, causal);
                const double* qi = Q + i * d;
                const double* doi = dO + i * d;
                row_forward(qi, K, V, nv, d, scale, p, oi);
                /* O with dropout, then D = dO . O */
                for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
                for (int64_t j = 0; j < nv; ++j)
                    if (dropout_keep(seed, bh, i, j, thr))
                        for (int64_t t = 0; t < d; ++t) oi[t] += p[j] * inv_keep * V[j * d + t];
                double Di = dot(doi, oi, d);
                double* dqi = dQ + i * d;
                for (int64_t t = 0; t < d; ++t) dqi[t] = 0.0;
                for (int64_t j = 0; j < nv; ++j) {
                    const double* vj = V + j * d;
                    const double* kj = K + j * d;
                    double zj = dropout_keep(seed, bh, i, j, thr) ? inv_keep : 0.0;
                    double dpij = zj * dot(doi, vj, d);
                    double dsij = p[j] * (dpij - Di);
                    double* dkj = dKp + j * d;
                    double* dvj = dVp + j * d;
                    for (int64_t t = 0; t < d; ++t) {
                        dqi[t] += scale * dsij * kj[t];
                        dkj[t] += scale * dsij * qi[t];
                        dvj[t] += p[j] * zj * doi[t];
                    }
                }
            }
            free(oi);
            free(p);
        }
        double* dK = dk + hh * N * d;
        double* dV = dv + hh * N * d;
        for (size_t e = 0; e < nd; ++e) {
            double sk = 0.0, sv = 0.0;
            for (int t = 0; t < nthr; ++t) {
                sk += part[(size_t)t * 2 * nd + e];
                sv += part[(size_t)t * 2 * nd + nd + e];
            }
            dK[e] = sk;
            dV[e] = sv;
        }
    }
    free(part);
}

/*
 * Causal linear attention: "Lightning Attention-2: A Free Lunch for Handling
 * Unlimited Sequence Lengths in Large Language Models" (chatpaper.ai
 * summary), abstract: linear attention replaces the softmax so that tokens
 * cost linear time; the causal form needs a cumulative sum, which
 * Lightning Attention-2 tiles into intra-block parts (computed like ordinary
 * attention) and inter-block parts (the linear-attention kernel trick: a
 * running d x d state).  "[論文レビュー] Gated Linear Attention Transformers
 * with Hardware-Efficient Training" (nubint.ai), proposed method: chunk-wise
 * parallel form, recurrence between chunks and parallel computation inside
 * them.  The pages give no formula; the plainest reading, taken here (no
 * feature map, no decay, no normalisation):
 *     O_i = scale * sum_{j <= i} (q_i . k_j) v_j.
 * oracle_linear_attn is that definition, row by row; oracle_linear_attn_chunked
 * restates the chunked form (per chunk of C rows: the masked in-chunk product
 * plus q_i S, S = sum of k_j^T v_j over earlier chunks, updated after the
 * chunk) as a self-check.
 */
void oracle_linear_attn(const double* q, const double* k, const double* v, double* o,
                        int64_t BH, int64_t N, int64_t d, double scale) {
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < N; ++i) {
            const double* qi = q + (bh * N + i) * d;
            double* oi = o + (bh * N + i) * d;
            for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                double a = scale * dot(qi, k + (bh * N + j) * d, d);
                const double* vj = v + (bh * N + j) * d;
                for (int64_t t = 0; t < d; ++t) oi[t] += a * vj[t];
            }
        }
}

void oracle_linear_attn_chunked(const double* q, const double* k, const double* v, double* o,
                                int64_t BH, int64_t N, int64_t d, double scale, int64_t C) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
        double* S = (double*)calloc((size_t)(d * d), sizeof(double));  /* S[a][b] */
        for (int64_t c0 = 0; c0 < N; c0 += C) {
            int64_t c1 = c0 + C < N ? c0 + C : N;
            for (int64_t i = c0; i < c1; ++i) {          /* intra-chunk + inter-chunk */
                const double* qi = q + (bh * N + i) * d;
                double* oi = o + (bh * N + i) * d;
                for (int64_t t = 0; t < d; ++t) {
                    double acc = 0.0;
                    for (int64_t a = 0; a < d; ++a) acc += qi[a] * S[a * d + t];
                    oi[t] = scale * acc;
                }
                for (int64_t j = c0; j <= i; ++j) {
                    double w = scale * dot(qi, k + (bh * N + j) * d, d);
                    const double* vj = v + (bh * N + j) * d;
                    for (int64_t t = 0; t < d; ++t) oi[t] += w * vj[t];
                }
            }
            for (int64_t j = c0; j < c1; ++j) {          /* state update after the chunk */
                const double* kj = k + (bh * N + j) * d;
                const double* vj = v + (bh * N + j) * d;
                for (int64_t a = 0; a < d; ++a)
                    for (int64_t t = 0; t < d; ++t) S[a * d + t] += kj[a] * vj[t];
            }
        }
        free(S);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

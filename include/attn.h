/*
 * attn.h — C ABI of libattn.so: exact scaled-dot-product attention on B200
 * (sm_100a), forward with the online-softmax recurrence and a backward that
 * recomputes the probabilities from the stored output and log-sum-exp.
 *
 * The operation (web pages on IO-aware exact attention):
 *  - O = softmax(Q K^T / sqrt(d) [+ causal mask]) V — "Is a full day of
 *    context better than ten minutes? FlashAttention and the sequence-length
 *    question" (marketmaker.cc), section "why attention is bound by memory";
 *    tensors are (batch, heads, seq, head_dim), half precision, and the causal
 *    mask is built inside the kernel — same page, section "integration is
 *    eight lines".
 *  - The N x N score matrix never reaches device memory: tiles of Q, K, V are
 *    staged on chip and the softmax is renormalised block by block — same
 *    page, sections "Flash Attention algorithm" and "online softmax
 *    recurrence".  Blocks wholly in the future of a query block are skipped —
 *    section "causal masking".
 *  - The backward keeps only O and one softmax statistic per row and
 *    recomputes P tile by tile — same page, section "backward: recompute
 *    instead of store"; the statistic is the log-sum-exp L — "Performance
 *    optimisation with Flash-Attention 2" (Medium), section "Flash Attention 2".
 *
 * Conventions shared by every entry point
 *  - Layout: q, k, v, o, dout, dq, dk, dv are contiguous (B, H, N, d) arrays of
 *    the same element type (bf16 or fp16); lse is a contiguous (B, H, N) fp32
 *    array holding the natural-log log-sum-exp of the scaled scores of each
 *    query row: lse = ln sum_j exp(scale * q_i . k_j) over the visible keys.
 *  - Key j is visible to query i iff causal == 0 or j <= i.
 *  - d must be 64 or 128; 1 <= N; 1 <= B, H; B * H * N * d < 2^31 elements;
 *    every pointer must be device memory aligned to 16 bytes.
 *  - scale is the score multiplier, usually 1/sqrt(d); it must be finite and > 0.
 *  - Ownership: the caller allocates and frees every buffer (torch or
 *    cudaMalloc).  The library never allocates or frees device memory inside
 *    these calls and never materialises an N x N array; it caches tensor-map
 *    descriptors per call only (they are kernel parameters).
 *  - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 *    All launches are asynchronous on it; outputs are valid once the stream
 *    reaches the end of the call.
 *  - Errors: argument errors are returned synchronously and nothing is
 *    launched; launch failures map to ATTN_ERR_LAUNCH.  Every wait inside a
 *    kernel is bounded in time; a wait that runs out sets a device error word
 *    and the kernel frees its tensor memory and returns, after which
 *    attn_last_device_status() reports ATTN_ERR_TIMEOUT.  No exception or
 *    abort crosses the ABI.
 *  - Inputs must be finite; NaN/Inf inputs are outside the contract.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { ATTN_BF16 = 0, ATTN_FP16 = 1 } attn_dtype_t;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,     /* a required pointer is NULL */
    ATTN_ERR_SHAPE = -2,    /* B, H or N < 1, or the tensor is too large */
    ATTN_ERR_HEADDIM = -3,  /* d not in {64, 128} */
    ATTN_ERR_ALIGN = -4,    /* a pointer is not 16-byte aligned */
    ATTN_ERR_DTYPE = -5,    /* dtype not bf16/fp16 */
    ATTN_ERR_DEVICE = -6,   /* no sm_100 device current, or a pointer is not device memory */
    ATTN_ERR_LAUNCH = -7,   /* the CUDA runtime rejected a launch */
    ATTN_ERR_TIMEOUT = -8,  /* a bounded in-kernel wait ran out (device status) */
    ATTN_ERR_ARG = -9,      /* scale not finite and positive, or another bad scalar */
    ATTN_ERR_SCRATCH = -10  /* attn_bwd_noalloc: problem exceeds the built-in scratch;
                               attn_sdpa_host: scratch_bytes too small */
} attn_status_t;

/*
 * Forward.  Reads q, k, v; writes o (same dtype, rounded to nearest even) and
 * lse (fp32).  Computes, for every (b, h) and query row i, the exact softmax
 * weights over the visible keys and their weighted sum of v rows, one query
 * tile of 128 rows at a time, streaming 128-key tiles of k and v through
 * shared memory with the running max / running sum recurrence.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int N, int d, int causal, float scale,
             attn_dtype_t dtype, void* stream);

/*
 * Bytes of device scratch attn_bwd needs: the log2-scaled LSE and D (the row
 * dot products of dO and O), B*H*Np fp32 each with Np = N rounded up to 128,
 * the fp32 dQ accumulator (B*H*N*d) and one int32 completion counter per
 * (b, h), each section 256-byte aligned.  Returns 0 for invalid sizes.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward of the forward above for an upstream gradient dout.  Reads q, k, v,
 * o and lse exactly as attn_fwd wrote them (the probabilities are recomputed
 * from lse, never stored), and dout; writes dq, dk, dv (same dtype as q).
 * `workspace` is caller-owned device memory of attn_bwd_workspace_bytes()
 * bytes, 256-byte aligned; its contents on entry do not matter and are
 * overwritten.  dq accumulates across key tiles in fp32 by atomic addition,
 * so its last bits may differ between runs; dk and dv are deterministic.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, void* workspace,
             int B, int H, int N, int d, int causal, float scale,
             attn_dtype_t dtype, void* stream);

/*
 * The two phases attn_bwd runs, for callers that want to schedule or time them
 * separately; calling attn_bwd_prep then attn_bwd_main on the same stream
 * and workspace is exactly attn_bwd.
 *
 * attn_bwd_prep: reads o, dout and lse; writes into the workspace D_i =
 * sum_t dout_it * o_it and lse_i * log2(e) (fp32, per head padded to a
 * multiple of 128 rows), and clears the fp32 dQ accumulator and the per-head
 * completion counters.
 *
 * attn_bwd_main: for every 128-key tile, recomputes S and P per query tile
 * (128 rows for d = 64, 64 rows for d = 128) from q, k and the statistics
 * attn_bwd_prep staged (never storing P), forms dV, dK in tensor memory and
 * adds the dQ contributions into the workspace accumulator.  dq is the
 * accumulator rounded to the dtype: for d = 64 the last key tile of each head
 * to finish converts that head, found through the completion counters; for
 * d = 128 a second kernel, launched by the same call on the same stream,
 * converts all of it.  Requires the workspace as attn_bwd_prep left it.
 */
int attn_bwd_prep(const void* o, const void* dout, const float* lse, void* workspace, int B,
                  int H, int N, int d, attn_dtype_t dtype, void* stream);

int attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dq,
                  void* dk, void* dv, void* workspace, int B, int H, int N, int d, int causal,
                  float scale, attn_dtype_t dtype, void* stream);

/*
 * Block-sparse attention: the forward and backward above restricted to the
 * (query tile, key tile) pairs a block mask marks, with tiles of 128 rows and
 * 128 keys; blocks not marked are skipped entirely (neither loaded nor
 * computed), as blocks in the future of a query tile are under the causal
 * mask.  Source: "FlashAttention の概要" (zenn.dev), the paragraph on
 * Block-Sparse FlashAttention (an approximation of attention that computes
 * only the blocks of a block mask, otherwise the same algorithm).
 *
 * block_mask: device memory, nb x nb bytes with nb = ceil(N / 128), row-major;
 * block_mask[i * nb + j] != 0 lets the 128 queries of tile i attend to the
 * 128 keys of tile j.  One mask serves every (batch, head).  With causal != 0
 * the causal rule applies as well (key j visible to query i iff its block is
 * marked and j <= i).  Over its visible keys each row is exact softmax
 * attention; a row with no visible key gets O = 0 and lse = -inf (the empty
 * sum), and contributes nothing to the gradients (its dq row is 0).
 * Everything else (layouts, workspace, streams, errors) is as for attn_fwd
 * and attn_bwd; ATTN_ERR_NULL if block_mask is NULL, ATTN_ERR_DEVICE if it is
 * not device memory of the current device.
 */
int attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                         const unsigned char* block_mask, int B, int H, int N, int d,
                         int causal, float scale, attn_dtype_t dtype, void* stream);

int attn_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv,
                         void* workspace, const unsigned char* block_mask, int B, int H, int N,
                         int d, int causal, float scale, attn_dtype_t dtype, void* stream);

/*
 * FP8 scores with incoherent processing: "Is a full day of context better
 * than ten minutes?" (marketmaker.cc), section "FA3: Hopper", third item
 * (random rotation of the vectors before block-wise FP8 quantisation spreads
 * outliers over all coordinates; reported 2.6x lower error than naive FP8).
 *
 * attn_fp8_quantize: x is q or k, (B, H, N, d) bf16/fp16.  Each row is
 * multiplied element-wise by `signs` (d entries of +1/-1, device memory; NULL:
 * all +1) and, if rotate != 0, transformed by the unnormalised d x d
 * Sylvester-Hadamard matrix (entries +-1; the butterflies run in fp32 in
 * ascending stride).  Each block of 128 rows of one (b, h) is quantised with
 * one scale: x8 = e4m3(y * (448 / amax)) (nearest even, saturating; IEEE fp32
 * multiply and divide), scales[(b H + h) ceil(N/128) + block] = amax / 448; a
 * block of zeros gets scale 0.  x8 is (B, H, N, d) bytes (e4m3), scales is
 * (B, H, ceil(N/128)) fp32; both caller-owned device memory.
 *
 * attn_fwd_fp8: the forward of attn_fwd with S = Q K^T computed from the e4m3
 * q8, k8 on the FP8 tensor cores, each tile's scores multiplied by its two
 * block scales, and by scale / d when q8 and k8 were rotated (rotated != 0;
 * the rotation multiplies dot products by d).  P V runs in the dtype of v
 * (bf16/fp16), o has that dtype, lse is fp32, as for attn_fwd.  q8, k8 and
 * their scales must come from attn_fp8_quantize with the same signs and
 * rotate.  Errors as attn_fwd; ATTN_ERR_ALIGN also for scales not 4-byte
 * aligned.
 */
int attn_fp8_quantize(const void* x, unsigned char* x8, float* scales, const signed char* signs,
                      int rotate, int B, int H, int N, int d, attn_dtype_t dtype, void* stream);

int attn_fwd_fp8(const unsigned char* q8, const unsigned char* k8, const float* q_scale,
                 const float* k_scale, const void* v, void* o, float* lse, int B, int H, int N,
                 int d, int causal, float scale, int rotated, attn_dtype_t dtype, void* stream);

/*
 * Dropout on the attention probabilities, as the dropout_p argument of the
 * attention call in "Is a full day of context better than ten minutes?"
 * (marketmaker.cc), section "integration is eight lines".  The forward and
 * backward of attn_fwd / attn_bwd, with each probability P_ij (after the
 * softmax; lse is that of P before dropout) kept with probability t / 256 and
 * then scaled by 256 / t, else set to 0, where t = round(256 (1 - dropout_p))
 * clamped to 1 .. 256 (dropout_p is taken to the nearest multiple of 1/256;
 * 0 keeps everything).  The random byte of (b, h, query i, key j) is byte
 * j % 16 of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011) with key
 * (seed & 0xffffffff, seed >> 32) and counter (j / 16, i, b H + h, 0): word
 * (j % 16) / 4, little-endian byte j % 4; P_ij is kept iff that byte < t.  The
 * backward regenerates the same mask from the same seed: call attn_bwd_dropout
 * with the dropout_p and seed given to attn_fwd_dropout.  Errors as attn_fwd /
 * attn_bwd; ATTN_ERR_ARG unless 0 <= dropout_p < 1.
 */
int attn_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, int causal, float scale, float dropout_p,
                     unsigned long long seed, attn_dtype_t dtype, void* stream);

int attn_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, void* workspace, int B,
                     int H, int N, int d, int causal, float scale, float dropout_p,
                     unsigned long long seed, attn_dtype_t dtype, void* stream);

/*
 * Causal linear attention, chunked: O_i = scale * sum_{j <= i} (q_i . k_j) v_j
 * (no softmax, feature map, decay or normalisation).  Source: "Lightning
 * Attention-2: A Free Lunch for Handling Unlimited Sequence Lengths in Large
 * Language Models" (chatpaper.ai summary), abstract (intra-block parts
 * computed like ordinary attention, inter-block parts by the linear-attention
 * kernel trick), and "Gated Linear Attention Transformers with
 * Hardware-Efficient Training" (nubint.ai review), proposed method (the
 * chunk-wise parallel form).  Chunks of 128 rows: O_c = scale [(Q_c K_c^T) o
 * causal mask] V_c + Q_c (scale S_c), S_c = sum over earlier chunks of K^T V.
 * q, k, v, o: (B, H, N, d) bf16/fp16 device memory, d = 128 only (else
 * ATTN_ERR_HEADDIM).  workspace: caller-owned device memory of
 * attn_linear_workspace_bytes() bytes, 256-byte aligned: the per-chunk K^T V
 * in fp32 and the prefix states S_c in the input's type.  The state reaches
 * the tensor cores rounded to the input's 16-bit type.  With B * H >= 32 one
 * fused kernel runs instead (one CTA per head and half of the value features,
 * walking the chunks in order with the state kept on chip) and the workspace
 * is left untouched; it forms the same fp32 sums in the same order.  Errors
 * as attn_fwd.
 */
size_t attn_linear_workspace_bytes(int B, int H, int N, int d);

int attn_linear_fwd(const void* q, const void* k, const void* v, void* o, void* workspace, int B,
                    int H, int N, int d, float scale, attn_dtype_t dtype, void* stream);

/*
 * Backward that allocates nothing, for callers that cannot get device memory
 * for a workspace: for example a plugin inside a host framework that owns
 * every device allocation through its own pool and hands the plugin only the
 * input and output tensors, or a latency-critical loop that may not call
 * cudaMalloc (which can synchronise the whole device) once it is running.
 * The papers describe no such entry point; it exists only for these callers.
 *
 * Same arguments, semantics and results as attn_bwd, minus `workspace`: the
 * scratch (D, the fp32 dQ accumulator and the per-head counters) lives in a
 * fixed array of ATTN_NOALLOC_SCRATCH_BYTES bytes that every device which
 * loads this library holds until the process exits.  The caller still passes
 * every input and output buffer.  Problems whose attn_bwd_workspace_bytes()
 * exceed that size are rejected with ATTN_ERR_SCRATCH before any launch.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.
 *  - All calls share the one array and it keeps what the last call left;
 *    each call clears what must start at zero.  Calls whose kernels overlap
 *    on the GPU (two streams, or two host threads) race on the array: order
 *    them on one stream or synchronise between them.
 *  - No cudaMalloc, cudaFree or other allocating routine is called.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                     int B, int H, int N, int d, int causal, float scale,
                     attn_dtype_t dtype, void* stream);

/*
 * End-to-end attention from host buffers, for callers whose tensors live in
 * host memory (the pages have no counterpart; it keeps the host link busy in
 * both directions while the kernels run).  q, k, v (and dout for the
 * backward) are read from host memory, and the outputs are written back
 * there: o and lse for the forward alone (dout == NULL; o and lse required);
 * with the backward dq, dk, dv (required), and o, lse too when not NULL.  All
 * tensors have the layouts of attn_fwd / attn_bwd.  Host memory should be
 * page-locked: pageable memory works, but its copies do not overlap.
 *
 * The heads are processed in chunks of `heads_per_chunk` heads (<= 0: about
 * an eighth of B*H, at least 256 query tiles of work per chunk).  The
 * host-to-device copies of chunk c + 1, the kernels of chunk c and the
 * device-to-host copies of chunk c - 1 run on three streams the library
 * creates once per device, in three chunk slots of `scratch`: caller-owned
 * device memory of at least attn_sdpa_host_scratch_bytes() bytes, 16-byte
 * aligned.  The call is asynchronous with respect to the host.  Work queued
 * on `stream` before the call comes first; work queued on `stream` after it
 * waits for the last copy back, also after an error.  Calls are serialised
 * by a per-device lock on the host.
 *
 * Results equal attn_fwd / attn_bwd on the same inputs: o, lse, dk and dv
 * bit for bit, dq up to the order of its fp32 additions.
 * Errors: ATTN_ERR_NULL, _SHAPE, _HEADDIM, _DTYPE and _ARG as attn_fwd;
 * ATTN_ERR_SCRATCH if scratch_bytes is too small; ATTN_ERR_ALIGN if scratch
 * is not 16-byte aligned; ATTN_ERR_DEVICE if scratch is not device memory of
 * the current device; ATTN_ERR_LAUNCH if a copy or launch was refused.
 */
size_t attn_sdpa_host_scratch_bytes(int B, int H, int N, int d, int with_backward,
                                    int heads_per_chunk);

int attn_sdpa_host(const void* q, const void* k, const void* v, const void* dout, void* o,
                   float* lse, void* dq, void* dk, void* dv, void* scratch,
                   size_t scratch_bytes, int B, int H, int N, int d, int causal, float scale,
                   attn_dtype_t dtype, int heads_per_chunk, void* stream);

/*
 * Synchronises `stream`, then returns ATTN_OK, ATTN_ERR_TIMEOUT if a kernel
 * of this library recorded a wait that ran out since the last call, or
 * ATTN_ERR_LAUNCH if the stream reported a CUDA error.  Clears the device
 * error word of the current device.
 */
int attn_last_device_status(void* stream);

/*
 * Diagnostic: launches one block that waits on a shared-memory barrier that
 * nothing ever completes, with the library's bounded wait and the given
 * limit in microseconds (1 .. 10^7).  The wait runs out, the kernel records
 * ATTN_ERR_TIMEOUT in the device error word and returns; the context stays
 * usable.  Lets tests exercise the timeout path without a fault or a hang.
 */
int attn_selftest_wait_timeout(unsigned timeout_us, void* stream);

/* Text of the last CUDA runtime error this library reported (on this host
 * thread) as ATTN_ERR_LAUNCH or ATTN_ERR_DEVICE; "no error" if none. */
const char* attn_last_cuda_error_string(void);

/* Static description of a status code. */
const char* attn_strerror(int status);

/* Library version, e.g. "0.1.0". */
const char* attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */

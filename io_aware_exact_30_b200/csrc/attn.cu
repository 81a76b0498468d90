// C ABI of libattn.so (declared in include/attn.h): argument validation,
// TMA tensor-map encoding and kernel launches on the caller's stream.
// The kernels live in the headers included below; this is the only
// translation unit, so the device error word has a single definition.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "ptx.cuh"
#include "fwd_sm100.cuh"
#include "bwd_sm100.cuh"
#include "bwd128_sm100.cuh"
#include "fp8_sm100.cuh"
#include "linear_sm100.cuh"

namespace {

using attn::FwdCfg;

// Last CUDA runtime error this library turned into ATTN_ERR_LAUNCH/DEVICE.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

bool launch_ok() {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) g_last_cuda_error = e;
    return e == cudaSuccess;
}

constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode;
}

// Per-device state: sm_100 check and the opt-in shared-memory size, done once.
std::mutex g_dev_mu;
int g_dev_state[kMaxDevices];  // 0 unknown, 1 ready, -1 unsupported
int g_sm_count[kMaxDevices];   // multiprocessors: grid size of the static schedules

int check_device(int* dev_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    *dev_out = dev;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev_state[dev] == 1) return ATTN_OK;
    if (g_dev_state[dev] == -1) return ATTN_ERR_DEVICE;
    int maj = 0, mnr = 0;
    cudaDeviceGetAttribute(&maj, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&mnr, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    if (maj != 10 || mnr != 0 || encode_fn() == nullptr || g_sm_count[dev] < 1) {
        cudaGetLastError();
        g_dev_state[dev] = -1;
        return ATTN_ERR_DEVICE;
    }
    bool ok = true;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64, true>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64, true>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128, true>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128, true>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, true, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<64, false, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<64>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, true, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::attn_fwd_kernel<128, false, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FwdCfg<128>::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_kv_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::kLinKvSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_kv_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::kLinKvSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_out_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::kLinOutSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_out_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::kLinOutSmem) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_fused_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::LinFusedCfg::SMEM_BYTES) == cudaSuccess;
    ok &= cudaFuncSetAttribute(attn::linear_fused_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               attn::LinFusedCfg::SMEM_BYTES) == cudaSuccess;
    ok &= attn::bwd_set_attributes();
    ok &= attn::bwd128_set_attributes();
    if (!ok) {
        g_last_cuda_error = cudaGetLastError();
        g_dev_state[dev] = -1;
        return ATTN_ERR_DEVICE;
    }
    attn::bwd_error_hook() = [](cudaError_t e) { g_last_cuda_error = e; };
    g_dev_state[dev] = 1;
    return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The pointer must be device (or managed) memory visible to device `dev`.
bool on_device(const void* p, int dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeManaged) return true;
    return a.type == cudaMemoryTypeDevice && a.device == dev;
}

int check_shape(int B, int H, int N, int d, int dtype, float scale) {
    if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_DTYPE;
    if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
    if (B < 1 || H < 1 || N < 1) return ATTN_ERR_SHAPE;
    const long long elems = 1LL * B * H * N * d;
    if (elems >= (1LL << 31) || 1LL * B * H >= (1LL << 31)) return ATTN_ERR_SHAPE;
    if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_ARG;
    return ATTN_OK;
}

// 3-D view (d, N, B*H) of a contiguous (B, H, N, d) half tensor; box 64 x rows x 1,
// 128-byte swizzle, out-of-range rows read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int dtype, int BH, int N, int d,
              unsigned rows = 128) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[3] = {64, rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_fn()(
        m, dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
        3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D view (d, N, B*H) of a contiguous (B, H, N, d) e4m3 tensor; box d x 128 x 1
// (one swizzled box per row: 128-byte swizzle for d = 128, 64-byte for d = 64).
bool make_map8(CUtensorMap* m, const void* ptr, int BH, int N, int d) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                             static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(d), 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool BF16, bool FP8 = false, bool DROP = false>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const attn::FwdParams& p, int sm_count, cudaStream_t st) {
    // causal: one CTA per work item, running CTAs take pending CTAs' items;
    // otherwise one CTA per multiprocessor
    const long long items = 1LL * p.n_pairs * p.BH;
    if (items >= (1LL << 31)) return ATTN_ERR_SHAPE;
    const bool dynamic = p.causal || p.bmask != nullptr;
    const int nblocks = static_cast<int>(dynamic || items < sm_count ? items : sm_count);
    attn::attn_fwd_kernel<D, BF16, FP8, DROP><<<static_cast<unsigned>(nblocks),
                                                FwdCfg<D, FP8>::NTHREADS, FwdCfg<D, FP8>::SMEM_BYTES,
                                                st>>>(mq, mk, mv, p);
    return launch_ok() ? ATTN_OK : ATTN_ERR_LAUNCH;
}

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t flag;
    if (threadIdx.x == 0) {
        attn::mbar_init(attn::smem_u32(&bar), 1);
        flag = 0;
        attn::fence_mbar_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the wait runs out after limit_ns.
    if (threadIdx.x == 0)
        attn::wait_bounded(attn::smem_u32(&bar), 0, &flag, limit_ns);
    __syncthreads();
}

// Built-in backward scratch for attn_bwd_noalloc: one copy per device that
// loads this library, held until the process exits.  Host code must not pass
// `g_bwd_scratch` itself to a kernel (on the host it names a stand-in, not the
// device copy); the device address is looked up with cudaGetSymbolAddress,
// once per device, with that device current.
__device__ __align__(256) unsigned char g_bwd_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

int scratch_address(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return ATTN_ERR_DEVICE;
        }
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return ATTN_OK;
}

}  // namespace

namespace {
// Forward for attn_fwd (bmask == nullptr) and attn_fwd_blocksparse.
// Dropout parameters from (p, seed): keep threshold t = round(256 (1 - p)) in
// 1 .. 256; ATTN_ERR_ARG unless 0 <= p < 1.
int dropout_params(float dropout_p, unsigned long long seed, attn::DropoutParams* dp) {
    if (!(dropout_p >= 0.f && dropout_p < 1.f)) return ATTN_ERR_ARG;
    long t = std::lround(256.0 * (1.0 - static_cast<double>(dropout_p)));
    if (t < 1) t = 1;
    if (t > 256) t = 256;
    dp->seed_lo = static_cast<uint32_t>(seed);
    dp->seed_hi = static_cast<uint32_t>(seed >> 32);
    dp->thr = static_cast<uint32_t>(t);
    dp->inv_keep = static_cast<float>(256.0 / static_cast<double>(t));
    return ATTN_OK;
}

int fwd_entry(const void* q, const void* k, const void* v, void* o, float* lse,
              const unsigned char* bmask, int B, int H, int N, int d, int causal, float scale,
              attn_dtype_t dtype, void* stream, const attn::DropoutParams* drop = nullptr) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(q, dev) || !on_device(k, dev) || !on_device(v, dev) || !on_device(o, dev) ||
        !on_device(lse, dev) || (bmask && !on_device(bmask, dev)))
        return ATTN_ERR_DEVICE;
    const int BH = B * H;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, dtype, BH, N, d) || !make_map(&mk, k, dtype, BH, N, d) ||
        !make_map(&mv, v, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    attn::FwdParams p;
    p.o = o;
    p.lse = lse;
    p.BH = BH;
    p.N = N;
    p.n_qtiles = (N + 127) / 128;
    p.n_pairs = (p.n_qtiles + 1) / 2;
    {
        // heads whose K and V together take at most about 48 MB of L2
        const long long kv_head = 2LL * N * d * 2;
        const long long g = (48LL << 20) / (kv_head > 0 ? kv_head : 1);
        p.group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
    }
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.bmask = bmask;
    p.n_ktiles = (N + 127) / 128;
    p.qscale = p.kscale = nullptr;
    p.drop = drop ? *drop : attn::DropoutParams{0u, 0u, 256u, 1.f};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf = dtype == ATTN_BF16;
    const int sms = g_sm_count[dev];
    if (drop) {
        if (d == 64)
            return bf ? launch_fwd<64, true, false, true>(mq, mk, mv, p, sms, st)
                      : launch_fwd<64, false, false, true>(mq, mk, mv, p, sms, st);
        return bf ? launch_fwd<128, true, false, true>(mq, mk, mv, p, sms, st)
                  : launch_fwd<128, false, false, true>(mq, mk, mv, p, sms, st);
    }
    if (d == 64)
        return bf ? launch_fwd<64, true>(mq, mk, mv, p, sms, st)
                  : launch_fwd<64, false>(mq, mk, mv, p, sms, st);
    return bf ? launch_fwd<128, true>(mq, mk, mv, p, sms, st)
              : launch_fwd<128, false>(mq, mk, mv, p, sms, st);
}
}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
             int d, int causal, float scale, attn_dtype_t dtype, void* stream) {
    return fwd_entry(q, k, v, o, lse, nullptr, B, H, N, d, causal, scale, dtype, stream);
}

int attn_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, int causal, float scale, float dropout_p,
                     unsigned long long seed, attn_dtype_t dtype, void* stream) {
    attn::DropoutParams dp;
    int rc = dropout_params(dropout_p, seed, &dp);
    if (rc) return rc;
    return fwd_entry(q, k, v, o, lse, nullptr, B, H, N, d, causal, scale, dtype, stream, &dp);
}

int attn_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                         const unsigned char* block_mask, int B, int H, int N, int d, int causal,
                         float scale, attn_dtype_t dtype, void* stream) {
    if (!block_mask) return ATTN_ERR_NULL;
    return fwd_entry(q, k, v, o, lse, block_mask, B, H, N, d, causal, scale, dtype, stream);
}

int attn_fp8_quantize(const void* x, unsigned char* x8, float* scales, const signed char* signs,
                      int rotate, int B, int H, int N, int d, attn_dtype_t dtype, void* stream) {
    if (!x || !x8 || !scales) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, 1.f);
    if (rc) return rc;
    if (!aligned16(x) || !aligned16(x8) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(x, dev) || !on_device(x8, dev) || !on_device(scales, dev) ||
        (signs && !on_device(signs, dev)))
        return ATTN_ERR_DEVICE;
    const long long blocks = 1LL * B * H * ((N + 127) / 128);
    if (blocks >= (1LL << 31)) return ATTN_ERR_SHAPE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const auto* in = static_cast<const uint8_t*>(x);
    const auto* sg = reinterpret_cast<const int8_t*>(signs);
    const bool bf = dtype == ATTN_BF16;
    const unsigned g = static_cast<unsigned>(blocks);
    if (d == 64) {
        if (bf) attn::attn_fp8_quantize_kernel<64, true><<<g, 512, 0, st>>>(in, x8, scales, sg, rotate, N);
        else attn::attn_fp8_quantize_kernel<64, false><<<g, 512, 0, st>>>(in, x8, scales, sg, rotate, N);
    } else {
        if (bf) attn::attn_fp8_quantize_kernel<128, true><<<g, 512, 0, st>>>(in, x8, scales, sg, rotate, N);
        else attn::attn_fp8_quantize_kernel<128, false><<<g, 512, 0, st>>>(in, x8, scales, sg, rotate, N);
    }
    return launch_ok() ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_fwd_fp8(const unsigned char* q8, const unsigned char* k8, const float* q_scale,
                 const float* k_scale, const void* v, void* o, float* lse, int B, int H, int N,
                 int d, int causal, float scale, int rotated, attn_dtype_t dtype, void* stream) {
    if (!q8 || !k8 || !q_scale || !k_scale || !v || !o || !lse) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
        (reinterpret_cast<uintptr_t>(q_scale) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u))
        return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(q8, dev) || !on_device(k8, dev) || !on_device(q_scale, dev) ||
        !on_device(k_scale, dev) || !on_device(v, dev) || !on_device(o, dev) || !on_device(lse, dev))
        return ATTN_ERR_DEVICE;
    const int BH = B * H;
    CUtensorMap mq, mk, mv;
    if (!make_map8(&mq, q8, BH, N, d) || !make_map8(&mk, k8, BH, N, d) ||
        !make_map(&mv, v, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    attn::FwdParams p;
    p.o = o;
    p.lse = lse;
    p.BH = BH;
    p.N = N;
    p.n_qtiles = (N + 127) / 128;
    p.n_pairs = (p.n_qtiles + 1) / 2;
    {
        const long long kv_head = 1LL * N * d * 3;  // e4m3 K and 16-bit V
        const long long g = (48LL << 20) / (kv_head > 0 ? kv_head : 1);
        p.group = static_cast<int>(g < 1 ? 1 : (g > BH ? BH : g));
    }
    p.causal = causal ? 1 : 0;
    // the rotation multiplies every dot product by d
    p.scale_log2 = scale * 1.4426950408889634f / (rotated ? static_cast<float>(d) : 1.f);
    p.bmask = nullptr;
    p.n_ktiles = (N + 127) / 128;
    p.qscale = q_scale;
    p.kscale = k_scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf = dtype == ATTN_BF16;
    if (d == 64)
        return bf ? launch_fwd<64, true, true>(mq, mk, mv, p, g_sm_count[dev], st)
                  : launch_fwd<64, false, true>(mq, mk, mv, p, g_sm_count[dev], st);
    return bf ? launch_fwd<128, true, true>(mq, mk, mv, p, g_sm_count[dev], st)
              : launch_fwd<128, false, true>(mq, mk, mv, p, g_sm_count[dev], st);
}

size_t attn_linear_workspace_bytes(int B, int H, int N, int d) {
    if (check_shape(B, H, N, d, ATTN_BF16, 1.f) || d != 128) return 0;
    const size_t states = static_cast<size_t>(B) * H * ((N + 127) / 128) * 128 * 128;
    return attn::align256(states * 4) + attn::align256(states * 2);
}

int attn_linear_fwd(const void* q, const void* k, const void* v, void* o, void* workspace, int B,
                    int H, int N, int d, float scale, attn_dtype_t dtype, void* stream) {
    if (!q || !k || !v || !o || !workspace) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (d != 128) return ATTN_ERR_HEADDIM;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(q, dev) || !on_device(k, dev) || !on_device(v, dev) || !on_device(o, dev) ||
        !on_device(workspace, dev))
        return ATTN_ERR_DEVICE;
    const int BH = B * H, nc = (N + 127) / 128;
    const long long items = 1LL * BH * nc;
    if (items >= (1LL << 31)) return ATTN_ERR_SHAPE;
    const size_t states = static_cast<size_t>(items) * 128 * 128;
    attn::LinearParams p;
    p.o = o;
    p.kv = static_cast<float*>(workspace);
    p.state = static_cast<uint8_t*>(workspace) + attn::align256(states * 4);
    p.BH = BH;
    p.N = N;
    p.n_chunks = nc;
    p.scale = scale;
    CUtensorMap mq, mk, mv, ms;
    if (!make_map(&mq, q, dtype, BH, N, d) || !make_map(&mk, k, dtype, BH, N, d) ||
        !make_map(&mv, v, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (BH >= attn::kLinFusedMinHeads) {
        // one CTA per (head, half of the value features), the state on chip
        const unsigned gf = static_cast<unsigned>(2 * BH);
        if (dtype == ATTN_BF16)
            attn::linear_fused_kernel<true>
                <<<gf, attn::LinFusedCfg::NTHREADS, attn::LinFusedCfg::SMEM_BYTES, st>>>(mq, mk, mv, p);
        else
            attn::linear_fused_kernel<false>
                <<<gf, attn::LinFusedCfg::NTHREADS, attn::LinFusedCfg::SMEM_BYTES, st>>>(mq, mk, mv, p);
        return launch_ok() ? ATTN_OK : ATTN_ERR_LAUNCH;
    }
    if (!make_map(&ms, p.state, dtype, static_cast<int>(items), 128, 128)) return ATTN_ERR_LAUNCH;
    const unsigned g = static_cast<unsigned>(items);
    const unsigned gp = static_cast<unsigned>((1LL * BH * 4096 + 255) / 256);
    if (dtype == ATTN_BF16) {
        attn::linear_kv_kernel<true><<<g, 192, attn::kLinKvSmem, st>>>(mk, mv, p);
        attn::linear_prefix_kernel<true><<<gp, 256, 0, st>>>(p);
        attn::linear_out_kernel<true><<<g, 192, attn::kLinOutSmem, st>>>(mq, mk, mv, ms, p);
    } else {
        attn::linear_kv_kernel<false><<<g, 192, attn::kLinKvSmem, st>>>(mk, mv, p);
        attn::linear_prefix_kernel<false><<<gp, 256, 0, st>>>(p);
        attn::linear_out_kernel<false><<<g, 192, attn::kLinOutSmem, st>>>(mq, mk, mv, ms, p);
    }
    return launch_ok() ? ATTN_OK : ATTN_ERR_LAUNCH;
}

size_t attn_bwd_workspace_bytes(int B, int H, int N, int d) {
    if (check_shape(B, H, N, d, ATTN_BF16, 1.f)) return 0;
    return attn::bwd_workspace_bytes(B, H, N, d);
}

namespace {
int bwd_common_checks(const void* const* ptrs, int nptr, const void* workspace, int B, int H,
                      int N, int d, attn_dtype_t dtype, float scale, int* dev) {
    for (int i = 0; i < nptr; ++i)
        if (!ptrs[i]) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    for (int i = 0; i < nptr; ++i)
        if (!aligned16(ptrs[i])) return ATTN_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGN;
    if ((rc = check_device(dev))) return rc;
    for (int i = 0; i < nptr; ++i)
        if (!on_device(ptrs[i], *dev)) return ATTN_ERR_DEVICE;
    return ATTN_OK;
}

int bwd_prep_dispatch(const void* o, const void* dout, const float* lse, void* workspace, int B,
                      int H, int N, int d, attn_dtype_t dtype, cudaStream_t st) {
    const bool bf = dtype == ATTN_BF16;
    if (d == 64)
        return bf ? attn::bwd_prep_launch<64, true>(o, dout, lse, workspace, B, H, N, st)
                  : attn::bwd_prep_launch<64, false>(o, dout, lse, workspace, B, H, N, st);
    return bf ? attn::bwd_prep_launch<128, true>(o, dout, lse, workspace, B, H, N, st)
              : attn::bwd_prep_launch<128, false>(o, dout, lse, workspace, B, H, N, st);
}

int bwd_main_dispatch(const void* q, const void* k, const void* v, const void* dout, void* dq,
                      void* dk, void* dv, void* workspace, int B, int H, int N, int d, int causal,
                      float scale, attn_dtype_t dtype, cudaStream_t st,
                      const unsigned char* bmask = nullptr,
                      const attn::DropoutParams* drop = nullptr) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv, mdo;
    if (!make_map(&mq, q, dtype, BH, N, d) || !make_map(&mk, k, dtype, BH, N, d) ||
        !make_map(&mv, v, dtype, BH, N, d) || !make_map(&mdo, dout, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    const bool bf = dtype == ATTN_BF16;
    const int c = causal ? 1 : 0;
    if (d == 64)
        return bf ? attn::bwd_main_launch<64, true>(mq, mk, mv, mdo, dq, dk, dv, workspace, B, H,
                                                    N, c, scale, st, bmask, drop)
                  : attn::bwd_main_launch<64, false>(mq, mk, mv, mdo, dq, dk, dv, workspace, B, H,
                                                     N, c, scale, st, bmask, drop);
    // d = 128: 64-query inner tiles
    // (dK and dV leave through TMA stores)
    CUtensorMap mq64, mdo64, mdk, mdv;
    if (!make_map(&mq64, q, dtype, BH, N, d, 64) || !make_map(&mdo64, dout, dtype, BH, N, d, 64) ||
        !make_map(&mdk, dk, dtype, BH, N, d) || !make_map(&mdv, dv, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    int dev = 0;
    cudaGetDevice(&dev);
    const int sms = g_sm_count[dev];
    return bf ? attn::bwd_main128_launch<true>(mq64, mk, mv, mdo64, mdk, mdv, dq, dk, dv,
                                               workspace, B, H, N, c, scale, sms, st, bmask, drop)
              : attn::bwd_main128_launch<false>(mq64, mk, mv, mdo64, mdk, mdv, dq, dk, dv,
                                                workspace, B, H, N, c, scale, sms, st, bmask, drop);
}
}  // namespace

int attn_bwd_prep(const void* o, const void* dout, const float* lse, void* workspace, int B,
                  int H, int N, int d, attn_dtype_t dtype, void* stream) {
    const void* ptrs[4] = {o, dout, lse, workspace};
    int dev;
    int rc = bwd_common_checks(ptrs, 4, workspace, B, H, N, d, dtype, 1.f, &dev);
    if (rc) return rc;
    return bwd_prep_dispatch(o, dout, lse, workspace, B, H, N, d, dtype,
                             static_cast<cudaStream_t>(stream));
}

int attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dq,
                  void* dk, void* dv, void* workspace, int B, int H, int N, int d, int causal,
                  float scale, attn_dtype_t dtype, void* stream) {
    const void* ptrs[8] = {q, k, v, dout, dq, dk, dv, workspace};
    int dev;
    int rc = bwd_common_checks(ptrs, 8, workspace, B, H, N, d, dtype, scale, &dev);
    if (rc) return rc;
    return bwd_main_dispatch(q, k, v, dout, dq, dk, dv, workspace, B, H, N, d, causal, scale,
                             dtype, static_cast<cudaStream_t>(stream));
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int N,
             int d, int causal, float scale, attn_dtype_t dtype, void* stream) {
    const void* ptrs[10] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
    int dev;
    int rc = bwd_common_checks(ptrs, 10, workspace, B, H, N, d, dtype, scale, &dev);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = bwd_prep_dispatch(o, dout, lse, workspace, B, H, N, d, dtype, st))) return rc;
    return bwd_main_dispatch(q, k, v, dout, dq, dk, dv, workspace, B, H, N, d, causal, scale,
                             dtype, st);
}

int attn_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, void* workspace, int B,
                     int H, int N, int d, int causal, float scale, float dropout_p,
                     unsigned long long seed, attn_dtype_t dtype, void* stream) {
    const void* ptrs[10] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
    attn::DropoutParams dp;  // the scalar first, as in attn_fwd_dropout
    int rc = dropout_params(dropout_p, seed, &dp);
    if (rc) return rc;
    int dev;
    if ((rc = bwd_common_checks(ptrs, 10, workspace, B, H, N, d, dtype, scale, &dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = bwd_prep_dispatch(o, dout, lse, workspace, B, H, N, d, dtype, st))) return rc;
    return bwd_main_dispatch(q, k, v, dout, dq, dk, dv, workspace, B, H, N, d, causal, scale,
                             dtype, st, nullptr, &dp);
}

int attn_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv,
                         void* workspace, const unsigned char* block_mask, int B, int H, int N,
                         int d, int causal, float scale, attn_dtype_t dtype, void* stream) {
    const void* ptrs[11] = {q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask};
    int dev;
    int rc = bwd_common_checks(ptrs, 10, workspace, B, H, N, d, dtype, scale, &dev);
    if (rc) return rc;
    if (!block_mask) return ATTN_ERR_NULL;
    if (!on_device(block_mask, dev)) return ATTN_ERR_DEVICE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = bwd_prep_dispatch(o, dout, lse, workspace, B, H, N, d, dtype, st))) return rc;
    return bwd_main_dispatch(q, k, v, dout, dq, dk, dv, workspace, B, H, N, d, causal, scale,
                             dtype, st, block_mask);
}

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                     int H, int N, int d, int causal, float scale, attn_dtype_t dtype,
                     void* stream) {
    const void* ptrs[9] = {q, k, v, o, lse, dout, dq, dk, dv};
    for (const void* ptr : ptrs)
        if (!ptr) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (attn::bwd_workspace_bytes(B, H, N, d) > ATTN_NOALLOC_SCRATCH_BYTES)
        return ATTN_ERR_SCRATCH;
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    for (const void* ptr : ptrs)
        if (!on_device(ptr, dev)) return ATTN_ERR_DEVICE;
    void* scratch = nullptr;
    if ((rc = scratch_address(dev, &scratch))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The prep kernel rewrites D and clears the dQ accumulator and counters,
    // so whatever the previous call left in the scratch does not matter.
    if ((rc = bwd_prep_dispatch(o, dout, lse, scratch, B, H, N, d, dtype, st))) return rc;
    return bwd_main_dispatch(q, k, v, dout, dq, dk, dv, scratch, B, H, N, d, causal, scale,
                             dtype, st);
}

int attn_last_device_status(void* stream) {
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return ATTN_ERR_LAUNCH;
    int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, attn::g_attn_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(attn::g_attn_error, &zero, sizeof(int)) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
    return word == 0 ? ATTN_OK : ATTN_ERR_TIMEOUT;
}

int attn_selftest_wait_timeout(unsigned timeout_us, void* stream) {
    if (timeout_us < 1 || timeout_us > 10000000u) return ATTN_ERR_ARG;
    int dev;
    int rc = check_device(&dev);
    if (rc) return rc;
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<unsigned long long>(timeout_us) * 1000ull);
    return launch_ok() ? ATTN_OK : ATTN_ERR_LAUNCH;
}

const char* attn_strerror(int status) {
    switch (status) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "a required pointer is NULL";
        case ATTN_ERR_SHAPE: return "B, H and N must be >= 1 and B*H*N*d < 2^31";
        case ATTN_ERR_HEADDIM: return "head dimension d must be 64 or 128";
        case ATTN_ERR_ALIGN: return "pointers must be 16-byte aligned (workspace 256-byte)";
        case ATTN_ERR_DTYPE: return "dtype must be ATTN_BF16 or ATTN_FP16";
        case ATTN_ERR_DEVICE: return "needs an sm_100 device and device-resident buffers";
        case ATTN_ERR_LAUNCH: return "the CUDA runtime rejected a launch or reported an error";
        case ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
        case ATTN_ERR_ARG: return "scale must be finite and > 0 (or a scalar argument is out of range)";
        case ATTN_ERR_SCRATCH: return "not enough scratch: the built-in array (attn_bwd_noalloc) or scratch_bytes (attn_sdpa_host) is too small";
        default: return "unknown status";
    }
}

const char* attn_version(void) { return "0.1.0"; }

const char* attn_last_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda_error); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Attention from host buffers, chunk by chunk over heads: the host-to-device
// copies of chunk c + 1, the kernels of chunk c and the device-to-host copies
// of chunk c - 1 run on three internal streams, so the copies over the host
// link overlap each other and the kernels.
namespace {

constexpr int kSlots = 3;  // chunks in flight: loading, computing, draining

struct HostPipe {
    bool ready = false;
    cudaStream_t in = nullptr, cmp = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t loaded[kSlots] = {}, computed[kSlots] = {}, drained[kSlots] = {};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[kMaxDevices];

bool pipe_init(HostPipe& hp) {
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.cmp, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming) == cudaSuccess;
    for (int s = 0; ok && s < kSlots; ++s)
        ok = cudaEventCreateWithFlags(&hp.loaded[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.computed[s], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&hp.drained[s], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) g_last_cuda_error = cudaGetLastError();
    hp.ready = ok;
    return ok;
}

// Byte offsets of one chunk slot's tensors in the device scratch.
struct SlotLayout {
    size_t q, k, v, o, lse, dout, dq, dk, dv, bytes;
};
SlotLayout slot_layout(int hc, int N, int d, bool bwd) {
    const size_t t = attn::align256(static_cast<size_t>(hc) * N * d * 2);
    const size_t l = attn::align256(static_cast<size_t>(hc) * N * 4);
    SlotLayout s{};
    size_t off = 0;
    s.q = off, off += t;
    s.k = off, off += t;
    s.v = off, off += t;
    s.o = off, off += t;
    s.lse = off, off += l;
    if (bwd) {
        s.dout = off, off += t;
        s.dq = off, off += t;
        s.dk = off, off += t;
        s.dv = off, off += t;
    }
    s.bytes = off;
    return s;
}

// heads per chunk: the caller's choice, else about an eighth of the heads but
// at least 256 query tiles' worth of work per chunk
int chunk_heads(int BH, int N, int want) {
    if (want > 0) return want < BH ? want : BH;
    const int n_qtiles = (N + 127) / 128;
    int hc = (BH + 7) / 8;
    const int fill = (256 + n_qtiles - 1) / n_qtiles;
    if (hc < fill) hc = fill;
    return hc < BH ? hc : BH;
}

}  // namespace

extern "C" size_t attn_sdpa_host_scratch_bytes(int B, int H, int N, int d, int with_backward,
                                               int heads_per_chunk) {
    if (check_shape(B, H, N, d, ATTN_BF16, 1.f) != ATTN_OK) return 0;
    const int hc = chunk_heads(B * H, N, heads_per_chunk);
    size_t total = kSlots * slot_layout(hc, N, d, with_backward != 0).bytes;
    if (with_backward) total += attn::align256(attn_bwd_workspace_bytes(1, hc, N, d));
    return total;
}

extern "C" int attn_sdpa_host(const void* q, const void* k, const void* v, const void* dout,
                              void* o, float* lse, void* dq, void* dk, void* dv, void* scratch,
                              size_t scratch_bytes, int B, int H, int N, int d, int causal,
                              float scale, attn_dtype_t dtype, int heads_per_chunk, void* stream) {
    const bool bwd = dout != nullptr;
    if (!q || !k || !v || !scratch) return ATTN_ERR_NULL;
    if (bwd ? (!dq || !dk || !dv) : (!o || !lse)) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (scratch_bytes < attn_sdpa_host_scratch_bytes(B, H, N, d, bwd ? 1 : 0, heads_per_chunk))
        return ATTN_ERR_SCRATCH;
    if (!aligned16(scratch)) return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(scratch, dev)) return ATTN_ERR_DEVICE;

    std::lock_guard<std::mutex> lk(g_pipe_mu);
    HostPipe& hp = g_pipe[dev];
    if (!hp.ready && !pipe_init(hp)) return ATTN_ERR_DEVICE;
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    const int BH = B * H, hc = chunk_heads(BH, N, heads_per_chunk);
    const SlotLayout L = slot_layout(hc, N, d, bwd);
    uint8_t* base = static_cast<uint8_t*>(scratch);
    uint8_t* ws = base + kSlots * L.bytes;
    const size_t head_t = static_cast<size_t>(N) * d * 2, head_l = static_cast<size_t>(N) * 4;

    // everything the caller queued on its stream before this call comes first
    bool ok = cudaEventRecord(hp.start, user) == cudaSuccess &&
              cudaStreamWaitEvent(hp.in, hp.start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(hp.cmp, hp.start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(hp.out, hp.start, 0) == cudaSuccess;
    auto h2d = [&](uint8_t* dst, const void* src, size_t off, size_t n) {
        ok = ok && cudaMemcpyAsync(dst, static_cast<const uint8_t*>(src) + off, n,
                                   cudaMemcpyDefault, hp.in) == cudaSuccess;
    };
    auto d2h = [&](void* dst, const uint8_t* src, size_t off, size_t n) {
        ok = ok && cudaMemcpyAsync(static_cast<uint8_t*>(dst) + off, src, n, cudaMemcpyDefault,
                                   hp.out) == cudaSuccess;
    };
    for (int c = 0, h0 = 0; ok && rc == ATTN_OK && h0 < BH; ++c, h0 += hc) {
        const int n = hc < BH - h0 ? hc : BH - h0, s = c % kSlots;
        uint8_t* sb = base + s * L.bytes;
        const size_t tb = n * head_t, lb = n * head_l, ot = h0 * head_t, ol = h0 * head_l;
        // the slot's previous chunk has left the device (its kernels ran before)
        ok = cudaStreamWaitEvent(hp.in, hp.drained[s], 0) == cudaSuccess;
        h2d(sb + L.q, q, ot, tb);
        h2d(sb + L.k, k, ot, tb);
        h2d(sb + L.v, v, ot, tb);
        if (bwd) h2d(sb + L.dout, dout, ot, tb);
        ok = ok && cudaEventRecord(hp.loaded[s], hp.in) == cudaSuccess &&
             cudaStreamWaitEvent(hp.cmp, hp.loaded[s], 0) == cudaSuccess;
        if (!ok) break;
        float* slse = reinterpret_cast<float*>(sb + L.lse);
        rc = attn_fwd(sb + L.q, sb + L.k, sb + L.v, sb + L.o, slse, 1, n, N, d, causal, scale,
                      dtype, hp.cmp);
        if (rc == ATTN_OK && bwd)
            rc = attn_bwd(sb + L.q, sb + L.k, sb + L.v, sb + L.o, slse, sb + L.dout, sb + L.dq,
                          sb + L.dk, sb + L.dv, ws, 1, n, N, d, causal, scale, dtype, hp.cmp);
        ok = ok && cudaEventRecord(hp.computed[s], hp.cmp) == cudaSuccess &&
             cudaStreamWaitEvent(hp.out, hp.computed[s], 0) == cudaSuccess;
        if (o) d2h(o, sb + L.o, ot, tb);
        if (lse) d2h(lse, sb + L.lse, ol, lb);
        if (bwd) {
            d2h(dq, sb + L.dq, ot, tb);
            d2h(dk, sb + L.dk, ot, tb);
            d2h(dv, sb + L.dv, ot, tb);
        }
        ok = ok && cudaEventRecord(hp.drained[s], hp.out) == cudaSuccess;
    }
    // the caller's stream continues after the last copy, also after an error,
    // so that nothing it frees is still in use
    const bool fin = cudaEventRecord(hp.done, hp.out) == cudaSuccess &&
                     cudaStreamWaitEvent(user, hp.done, 0) == cudaSuccess;
    if (!ok || !fin) {
        g_last_cuda_error = cudaGetLastError();
        if (rc == ATTN_OK) rc = ATTN_ERR_LAUNCH;
    }
    return rc;
}

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

template <int D, bool BF16>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const attn::FwdParams& p, int sm_count, cudaStream_t st) {
    // causal: one CTA per work item, running CTAs take pending CTAs' items;
    // otherwise one CTA per multiprocessor
    const long long items = 1LL * p.n_pairs * p.BH;
    if (items >= (1LL << 31)) return ATTN_ERR_SHAPE;
    const int nblocks = static_cast<int>(p.causal || items < sm_count ? items : sm_count);
    attn::attn_fwd_kernel<D, BF16><<<static_cast<unsigned>(nblocks), FwdCfg<D>::NTHREADS,
                                     FwdCfg<D>::SMEM_BYTES, st>>>(mq, mk, mv, p);
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

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
             int d, int causal, float scale, attn_dtype_t dtype, void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULL;
    int rc = check_shape(B, H, N, d, dtype, scale);
    if (rc) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return ATTN_ERR_ALIGN;
    int dev;
    if ((rc = check_device(&dev))) return rc;
    if (!on_device(q, dev) || !on_device(k, dev) || !on_device(v, dev) || !on_device(o, dev) ||
        !on_device(lse, dev))
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf = dtype == ATTN_BF16;
    if (d == 64)
        return bf ? launch_fwd<64, true>(mq, mk, mv, p, g_sm_count[dev], st)
                  : launch_fwd<64, false>(mq, mk, mv, p, g_sm_count[dev], st);
    return bf ? launch_fwd<128, true>(mq, mk, mv, p, g_sm_count[dev], st)
              : launch_fwd<128, false>(mq, mk, mv, p, g_sm_count[dev], st);
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
                      float scale, attn_dtype_t dtype, cudaStream_t st) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv, mdo;
    if (!make_map(&mq, q, dtype, BH, N, d) || !make_map(&mk, k, dtype, BH, N, d) ||
        !make_map(&mv, v, dtype, BH, N, d) || !make_map(&mdo, dout, dtype, BH, N, d))
        return ATTN_ERR_LAUNCH;
    const bool bf = dtype == ATTN_BF16;
    const int c = causal ? 1 : 0;
    if (d == 64)
        return bf ? attn::bwd_main_launch<64, true>(mq, mk, mv, mdo, dq, dk, dv, workspace, B, H,
                                                    N, c, scale, st)
                  : attn::bwd_main_launch<64, false>(mq, mk, mv, mdo, dq, dk, dv, workspace, B, H,
                                                     N, c, scale, st);
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
                                               workspace, B, H, N, c, scale, sms, st)
              : attn::bwd_main128_launch<false>(mq64, mk, mv, mdo64, mdk, mdv, dq, dk, dv,
                                                workspace, B, H, N, c, scale, sms, st);
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
        case ATTN_ERR_SCRATCH: return "problem needs more backward scratch than the built-in array holds";
        default: return "unknown status";
    }
}

const char* attn_version(void) { return "0.1.0"; }

const char* attn_last_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda_error); }

}  // extern "C"

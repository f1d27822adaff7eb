// mse.cu -- attention-difference diagnostic: mean over all elements of
// (a - b)^2 between two attention outputs (PAB report, Fig. 1: the
// difference between consecutive diffusion steps' attention outputs,
// quantified by MSE).
//
// HBM-bound: each element is read once from each tensor (2 x size bytes).
// One launch: a grid of (SM count x 8) blocks of 256 threads streams 16-byte
// vectors with a grid-stride loop, accumulates (a - b)^2 in fp64 per thread, reduces each
// warp with shuffles and each block through shared memory, and writes one
// fp64 partial per block.  The block that finishes last (a completion
// ticket counted with an atomic add) sums the partials in a fixed order,
// divides by n and returns the ticket to zero for the next call.  The split
// depends only on n and the SM count, and the final sum's order does not
// depend on which block finishes last, so the result is bitwise reproducible
// on a given device.  A block holds at most 48 registers a thread (12 K a
// block), so when the MSE runs on a side stream its blocks fit on an SM next
// to a flash attention CTA (384 threads of at most 136 registers, under
// 230 KB of shared memory) and stream their bytes while the tensor cores work.
#include "../../include/pab.h"
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

constexpr int kThreads = 256;
constexpr int kMinBlocks = 5;  // 65536 / (256 * 5): at most 48 registers a thread
constexpr int kUnroll = 4;

template <typename T>
struct Vec;  // 16 bytes of T
// Squared differences of one 16-byte vector: the (at most 8) terms are summed
// in fp32 (relative error < 1e-6, far inside the diagnostic's 1e-5) and the
// vector's sum enters the thread's fp64 accumulator, so the fp64 work is one
// conversion and one add per vector instead of per element.
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int kElems = 8;
    PAB_DEV static double sq_sum(const uint4& a, const uint4& b) {
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 fa = __bfloat1622float2(pa[i]);
            const float2 fb = __bfloat1622float2(pb[i]);
            const float d0 = fa.x - fb.x;  // exact unless the exponents differ by more than 16
            const float d1 = fa.y - fb.y;
            acc0 = fmaf(d0, d0, acc0);
            acc1 = fmaf(d1, d1, acc1);
        }
        return (double)(acc0 + acc1);
    }
    PAB_DEV static double sq_one(const __nv_bfloat16* a, const __nv_bfloat16* b, long long i) {
        const double d = (double)(__bfloat162float(a[i]) - __bfloat162float(b[i]));
        return d * d;
    }
};
template <>
struct Vec<float> {
    static constexpr int kElems = 4;
    PAB_DEV static double sq_sum(const uint4& a, const uint4& b) {
        const float* fa = reinterpret_cast<const float*>(&a);
        const float* fb = reinterpret_cast<const float*>(&b);
        double acc = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double d = (double)fa[i] - (double)fb[i];
            acc = fma(d, d, acc);
        }
        return acc;
    }
    PAB_DEV static double sq_one(const float* a, const float* b, long long i) {
        const double d = (double)a[i] - (double)b[i];
        return d * d;
    }
};

PAB_DEV double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Fixed-order block reduction; every thread passes its value, thread 0 gets the sum.
PAB_DEV double block_sum(double x, double* red) {
    x = warp_sum(x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double s = 0.0;
    if (warp == 0) {
        s = (lane < (int)(blockDim.x >> 5)) ? red[lane] : 0.0;
        s = warp_sum(s);
    }
    return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
    mse_kernel(const T* __restrict__ a, const T* __restrict__ b, long long n, unsigned long long* __restrict__ ticket,
               double* __restrict__ partials, double* __restrict__ result) {
    __shared__ double red[kThreads / 32];
    __shared__ bool last;
    constexpr int E = Vec<T>::kElems;
    const long long nvec = n / E;
    const uint4* va = reinterpret_cast<const uint4*>(a);
    const uint4* vb = reinterpret_cast<const uint4*>(b);
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    double acc = 0.0;
    // unrolled body: kUnroll independent 16-byte loads per tensor in flight
    for (; i + (kUnroll - 1) * stride < nvec; i += kUnroll * stride) {
        uint4 ra[kUnroll], rb[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            ra[u] = __ldcs(va + i + u * stride);
            rb[u] = __ldcs(vb + i + u * stride);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc += Vec<T>::sq_sum(ra[u], rb[u]);
    }
    for (; i < nvec; i += stride) acc += Vec<T>::sq_sum(__ldcs(va + i), __ldcs(vb + i));
    // scalar tail (n not a multiple of the vector width): block 0 only
    if (blockIdx.x == 0) {
        const long long t = nvec * E + threadIdx.x;
        if (t < n) acc += Vec<T>::sq_one(a, b, t);
    }
    const double s = block_sum(acc, red);
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = s;
        __threadfence();  // the partial is visible before the ticket is taken
        last = atomicAdd(ticket, 1ull) == (unsigned long long)gridDim.x - 1;
    }
    __syncthreads();
    if (!last) return;
    // the last block: every partial has been published
    __threadfence();
    double acc2 = 0.0;
    for (int k = threadIdx.x; k < (int)gridDim.x; k += blockDim.x) acc2 += __ldcg(partials + k);
    const double tot = block_sum(acc2, red);
    if (threadIdx.x == 0) {
        *result = (n > 0) ? tot / (double)n : 0.0;
        *ticket = 0ull;  // ready for the next call on this scratch
    }
}

}  // namespace

int mse_num_partials(long long n, int elem_size) {
    const long long nvec = n * elem_size / 16;
    const long long per_block = (long long)kThreads * kUnroll;
    long long blocks = (nvec + per_block - 1) / per_block;
    const long long cap = (long long)device_sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

cudaError_t launch_mse(const void* a, const void* b, long long n, int dtype, double* scratch,
                       int num_partials, double* result_dev, cudaStream_t s) {
    unsigned long long* ticket = reinterpret_cast<unsigned long long*>(scratch);
    double* partials = scratch + 1;
    if (dtype == 1)
        mse_kernel<float><<<num_partials, kThreads, 0, s>>>(static_cast<const float*>(a),
                                                          static_cast<const float*>(b), n, ticket, partials,
                                                          result_dev);
    else
        mse_kernel<__nv_bfloat16><<<num_partials, kThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), n, ticket, partials,
            result_dev);
    return cudaGetLastError();
}

}  // namespace pab

// ===========================================================================
// Allocation-free variant of the MSE diagnostic.
//
// Some callers cannot call cudaMalloc: code that runs inside a host framework
// whose memory pool owns all device memory and must account for every byte,
// or latency-critical loops where a device allocation (and the implicit
// synchronisation it may bring) is not acceptable.  For them,
// pab_attn_diff_mse_noalloc keeps its fp64 partial sums in a fixed,
// file-scope device array instead of the lazily allocated per-device buffer
// that pab_attn_diff_mse / pab_attn_diff_mse_async use.
//
// The array holds kNoAllocScratch doubles (32 KiB): slot 0 is the kernel's
// completion ticket, the rest are partial sums (at most kNoAllocMaxPartials).
// Every GPU that loads this library keeps it until the process exits.  Every
// call shares it and it keeps the last call's contents.  Only the ticket must
// start at zero: a file-scope device array is zero when the module is loaded
// on a device, and every call's last block returns the ticket to zero, so no
// call clears it (a clear issued by one call could land under another call's
// kernel still running on another stream).  The partial slots need no
// clearing: each block overwrites its own slot and the final sum reads only
// the slots this call wrote.  Calls whose kernels overlap on the GPU
// (different streams, or different host threads on one device) race on the
// array and must be serialised by the caller.
// ===========================================================================
namespace {

constexpr int kNoAllocScratch = 4096;
constexpr int kNoAllocMaxPartials = kNoAllocScratch - 1;
static __device__ __align__(256) double g_mse_noalloc_scratch[kNoAllocScratch];

// Device address of the array in the current device's context.  Host code
// cannot use the array's name as a device pointer (it names a host-side
// stand-in), so every call looks the address up with cudaGetSymbolAddress
// while the caller's device is current.  Nothing is cached: after a
// cudaDeviceReset the module is loaded again (with a zeroed array) at a
// possibly different address, and the next call sees that address.
int noalloc_scratch(double** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_mse_noalloc_scratch);
    if (e != cudaSuccess || !p)
        return pab::report_error(PAB_ERR_CUDA, "cudaGetSymbolAddress of the MSE scratch array: %s",
                                 cudaGetErrorString(e));
    *out = static_cast<double*>(p);
    return PAB_OK;
}

}  // namespace

extern "C" int pab_attn_diff_mse_noalloc(const void* a, const void* b, long long n, int dtype,
                                         double* result_dev, void* cuda_stream) {
    if (dtype != PAB_BF16 && dtype != PAB_FP32)
        return pab::report_error(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (n < 0) return pab::report_error(PAB_ERR_ARG, "n=%lld must be >= 0", n);
    if (!result_dev || (reinterpret_cast<uintptr_t>(result_dev) & 7u))
        return pab::report_error(PAB_ERR_ARG, "result_dev null or not 8-byte aligned");
    if (n > 0 && (!a || !b)) return pab::report_error(PAB_ERR_ARG, "null input");
    if (n > 0 && ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15u))
        return pab::report_error(PAB_ERR_ARG, "inputs not 16-byte aligned");
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const int parts = pab::mse_num_partials(n, elem);
    if (parts > kNoAllocMaxPartials)
        return pab::report_error(PAB_ERR_UNSUPPORTED,
                                 "this call needs %d partial sums; the static scratch array holds %d",
                                 parts, kNoAllocMaxPartials);
    double* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc != PAB_OK) return rc;
    const cudaError_t e = pab::launch_mse(a, b, n, dtype, scratch, parts, result_dev,
                                          static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess)
        return pab::report_error(PAB_ERR_CUDA, "MSE launch: %s", cudaGetErrorString(e));
    return PAB_OK;
}

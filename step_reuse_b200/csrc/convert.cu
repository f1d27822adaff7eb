// convert.cu -- element-type conversion at the boundary of fp32 plans: the
// inputs are rounded to bf16 (round to nearest even) before the bf16
// attention kernels run, and bf16 outputs are widened to fp32.
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                   long long n4, const float* __restrict__ src_s,
                                   __nv_bfloat16* __restrict__ dst_s, long long n) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 f = src[i];
        dst[i] = make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
    }
    if (blockIdx.x == 0 && threadIdx.x < (n - n4 * 4))
        dst_s[n4 * 4 + threadIdx.x] = __float2bfloat16_rn(src_s[n4 * 4 + threadIdx.x]);
}

__global__ void bf16_to_f32_kernel(const uint2* __restrict__ src, float4* __restrict__ dst,
                                   long long n4, const __nv_bfloat16* __restrict__ src_s,
                                   float* __restrict__ dst_s, long long n) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const uint2 u = src[i];
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        dst[i] = make_float4(a.x, a.y, b.x, b.y);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n - n4 * 4))
        dst_s[n4 * 4 + threadIdx.x] = __bfloat162float(src_s[n4 * 4 + threadIdx.x]);
}

unsigned grid_for(long long n4) {
    long long g = (n4 + 255) / 256;
    const long long cap = (long long)device_sm_count() * 8;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return (unsigned)g;
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float* src, void* dst, long long n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const long long n4 = n / 4;
    f32_to_bf16_kernel<<<grid_for(n4), 256, 0, s>>>(reinterpret_cast<const float4*>(src),
                                                    static_cast<uint2*>(dst), n4, src,
                                                    static_cast<__nv_bfloat16*>(dst), n);
    return cudaGetLastError();
}

cudaError_t launch_bf16_to_f32(const void* src, float* dst, long long n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const long long n4 = n / 4;
    bf16_to_f32_kernel<<<grid_for(n4), 256, 0, s>>>(static_cast<const uint2*>(src),
                                                    reinterpret_cast<float4*>(dst), n4,
                                                    static_cast<const __nv_bfloat16*>(src), dst, n);
    return cudaGetLastError();
}

}  // namespace pab

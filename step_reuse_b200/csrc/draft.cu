// draft.cu -- the low-resolution half of draft attention as PAB's spatial
// kind (crisp3r.com article on "Draft Attention", steps 1-3): the latent
// frame's queries and keys are average-pooled into a sketch of 16 x 16-token
// regions, the sketch's draft scores rank the key regions of every query
// region, and the best `keep` of them form the sparse mask that the
// region-sparse flash kernel (flash_tc.cu, list geometry) runs under.
//
//   draft_pool_kernel    one CTA per (region, frame, tensor, 1024-channel
//                        slice): thread c owns 8 channels and sums the
//                        region's 256 tokens in a fixed order
//                        (deterministic), 16-byte loads, a 16-token row in
//                        flight; writes the fp32 mean.  Small CTAs, many of
//                        them: the grid is several waves, so no SM is left
//                        with a long tail.  HBM-bound: q and k are read once.
//   draft_select_kernel  one warp per (query region, head, frame): for each
//                        key region the lanes split the d channels (the
//                        query's sketch row in registers, the key's read as
//                        one coalesced row) and a fixed butterfly sums the
//                        fp32 products; the score is scaled by 1/sqrt(d).
//                        Then `keep` rounds of a warp arg-max (higher score
//                        wins, equal scores go to the lower index) mark the
//                        kept regions, which are written in ascending order.
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

constexpr int kRegion = 16;
constexpr int kSelectWarps = 4;
constexpr int kPoolThreads = 128;  // 8 channels each: a CTA pools a 1024-channel slice
constexpr int kMaxD = 128;         // head dims the library accepts

// q, k: [T][H][W][C] bf16; sketch: [2][T][R][C] fp32 (q's, then k's)
__global__ void __launch_bounds__(kPoolThreads)
    draft_pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      float* __restrict__ sketch, int T, int H, int W, int C, int slices) {
    const int r = blockIdx.x, t = blockIdx.y, which = blockIdx.z / slices;
    const int rw = W / kRegion, R = (H / kRegion) * rw;
    const int y0 = (r / rw) * kRegion, x0 = (r % rw) * kRegion;
    const __nv_bfloat16* src = (which == 0 ? q : k) + (long long)t * H * W * C;
    float* dst = sketch + ((long long)which * T + t) * R * C + (long long)r * C;
    const int c8 = (blockIdx.z % slices) * kPoolThreads + threadIdx.x;
    if (c8 < C / 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int y = y0; y < y0 + kRegion; ++y) {
            const uint4* row = reinterpret_cast<const uint4*>(src + ((long long)y * W + x0) * C) + c8;
            uint4 u[kRegion];
#pragma unroll
            for (int x = 0; x < kRegion; ++x) u[x] = __ldg(row + (long long)x * (C / 8));
#pragma unroll
            for (int x = 0; x < kRegion; ++x) {
                const uint32_t w[4] = {u[x].x, u[x].y, u[x].z, u[x].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
                    acc[2 * i] += f.x;
                    acc[2 * i + 1] += f.y;
                }
            }
        }
        constexpr float inv = 1.0f / (kRegion * kRegion);  // a power of two: the mean is exact in scale
        float4* out = reinterpret_cast<float4*>(dst + c8 * 8);
        out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    }
}

// sel: [T][heads][R][keep] int32, ascending region index per row
__global__ void draft_select_kernel(const float* __restrict__ sketch, int* __restrict__ sel, int T, int R, int heads,
                                    int d, int keep, float scale) {
    extern __shared__ float sm[];  // [kSelectWarps][R] scores, then [kSelectWarps][R] taken flags
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kSelectWarps + warp, h = blockIdx.y, t = blockIdx.z;
    if (i >= R) return;
    const long long C = (long long)heads * d;
    const float* qb = sketch + ((long long)t * R + i) * C + (long long)h * d;
    const float* kb = sketch + ((long long)(T + t) * R) * C + (long long)h * d;
    float* sc = sm + warp * R;
    unsigned char* taken = reinterpret_cast<unsigned char*>(sm + kSelectWarps * R) + warp * R;
    float qv[kMaxD / 32];
#pragma unroll
    for (int m = 0; m < kMaxD / 32; ++m) qv[m] = lane + 32 * m < d ? qb[lane + 32 * m] : 0.f;
    for (int j = 0; j < R; ++j) {
        const float* kj = kb + (long long)j * C;
        float part = 0.f;
#pragma unroll
        for (int m = 0; m < kMaxD / 32; ++m)
            if (lane + 32 * m < d) part = fmaf(qv[m], kj[lane + 32 * m], part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) {
            const float s = part * scale;
            sc[j] = s == s ? s : -INFINITY;  // a NaN score ranks last, so every round still picks a region
            taken[j] = 0;
        }
    }
    __syncwarp();
    for (int n = 0; n < keep; ++n) {
        float best = -INFINITY;
        int bi = 0x7fffffff;
        for (int j = lane; j < R; j += 32)
            if (!taken[j] && (sc[j] > best || (sc[j] == best && j < bi))) {
                best = sc[j];
                bi = j;
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ob > best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        if (lane == 0 && bi < R) taken[bi] = 1;
        __syncwarp();
    }
    int* row = sel + (((long long)t * heads + h) * R + i) * keep;
    // ascending order: each lane counts the kept regions below its chunk
    int base = 0;
    for (int j0 = 0; j0 < R; j0 += 32) {
        const int j = j0 + lane;
        const bool kept = j < R && taken[j];
        const unsigned m = __ballot_sync(0xffffffffu, kept);
        if (kept) row[base + __popc(m & ((1u << lane) - 1u))] = j;
        base += __popc(m);
    }
}

}  // namespace

size_t draft_sketch_bytes(int T, int H, int W, int heads, int d) {
    const long long R = (long long)(H / kRegion) * (W / kRegion);
    return (size_t)2 * T * R * heads * d * sizeof(float);
}

cudaError_t launch_draft_select(const void* q, const void* k, int T, int H, int W, int heads, int d, int keep,
                                int* sel, void* sketch, cudaStream_t s) {
    if (T == 0 || H == 0 || W == 0) return cudaSuccess;
    const int C = heads * d;
    const int R = (H / kRegion) * (W / kRegion);
    if (H % kRegion || W % kRegion || C % 8 || keep < 1 || keep > R || R > 4096 || T > 65535 || heads > 65535)
        return cudaErrorInvalidValue;
    const int slices = (C / 8 + kPoolThreads - 1) / kPoolThreads;
    if (2LL * slices > 65535) return cudaErrorInvalidValue;
    draft_pool_kernel<<<dim3(R, T, 2 * slices), kPoolThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(q),
                                                                      static_cast<const __nv_bfloat16*>(k),
                                                                      static_cast<float*>(sketch), T, H, W, C,
                                                                      slices);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)kSelectWarps * R * (sizeof(float) + 1);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(draft_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    draft_select_kernel<<<dim3((R + kSelectWarps - 1) / kSelectWarps, heads, T), kSelectWarps * 32, smem, s>>>(
        static_cast<const float*>(sketch), sel, T, R, heads, d, keep, 1.0f / sqrtf((float)d));
    return cudaGetLastError();
}

}  // namespace pab

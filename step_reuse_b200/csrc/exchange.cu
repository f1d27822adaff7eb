// exchange.cu -- the data movement of broadcast sequence parallelism (PAB
// report, "Parallel", Fig. 3): dynamic sequence parallelism gives every rank
// T/G frames; temporal attention needs all frames of a position, so before a
// temporal compute every rank's frames of position chunk g move to rank g,
// and the output moves back after it (none of this happens on a temporal
// broadcast step).
//
// One launch moves up to three tensors.  Each tensor is P * G blocks of
// `block_rows` consecutive token rows; block (p, g) is contiguous in the
// source and lands contiguous in destination buffer g, so the move is a set
// of contiguous copies: the pack of the spatial view [T/G, N, C] into the
// ranks' temporal inputs [T, N/G, C] and the unpack of the output, with the
// packing permutation done by the addressing.  The destinations are device
// pointers: this GPU's buffers, or peer GPUs' buffers mapped into this
// process (CUDA IPC), written with plain 16-byte stores over NVLink -- no
// staging copy, no library collective, no TMA (so no multicast of any kind).
// HBM traffic: each byte read once and written once.
#include <cuda_runtime.h>

#include "../../include/pab.h"
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct ScatterArgs {
    const char* src[kScatterMaxTensors];
    char* dst[kScatterMaxTensors * kScatterMaxRanks];  // [tensor][destination]
    int G, P, src_order;
    long long block_bytes;      // block_rows * row_bytes (a multiple of 16)
    long long dst_offset_bytes;
    long long dst_stride_bytes;
};

// grid: x strides over a block's 16-byte vectors, y = source block, z = tensor
__global__ void __launch_bounds__(kThreads) scatter_blocks_kernel(const __grid_constant__ ScatterArgs a) {
    const int t = blockIdx.z, bi = blockIdx.y;
    int p, g;
    if (a.src_order == 0) {
        p = bi / a.G;
        g = bi - p * a.G;
    } else {
        g = bi / a.P;
        p = bi - g * a.P;
    }
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(a.src[t] + (long long)bi * a.block_bytes);
    uint4* __restrict__ dst =
        reinterpret_cast<uint4*>(a.dst[t * a.G + g] + a.dst_offset_bytes + (long long)p * a.dst_stride_bytes);
    const long long nvec = a.block_bytes >> 4;
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    // kUnroll independent 16-byte loads in flight per thread, then the stores
    for (; i + (kUnroll - 1) * stride < nvec; i += kUnroll * stride) {
        uint4 r[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) r[u] = __ldcs(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) dst[i + u * stride] = r[u];
    }
    for (; i < nvec; i += stride) dst[i] = __ldcs(src + i);
}

}  // namespace

cudaError_t launch_scatter_blocks(const void* const* src, void* const* dst, int ntensors, int G, int P,
                                  long long block_rows, int row_bytes, int src_order, long long dst_offset_rows,
                                  long long dst_stride_rows, cudaStream_t s) {
    ScatterArgs a;
    for (int t = 0; t < kScatterMaxTensors; ++t) a.src[t] = t < ntensors ? static_cast<const char*>(src[t]) : nullptr;
    for (int i = 0; i < kScatterMaxTensors * kScatterMaxRanks; ++i)
        a.dst[i] = i < ntensors * G ? static_cast<char*>(dst[i]) : nullptr;
    a.G = G;
    a.P = P;
    a.src_order = src_order;
    a.block_bytes = block_rows * row_bytes;
    a.dst_offset_bytes = dst_offset_rows * row_bytes;
    a.dst_stride_bytes = dst_stride_rows * row_bytes;
    const long long nvec = a.block_bytes >> 4;
    if (nvec == 0) return cudaSuccess;
    // about eight CTAs of work per SM over the whole launch
    const long long blocks = (long long)P * G * ntensors;
    long long gx = ((long long)device_sm_count() * 8 + blocks - 1) / blocks;
    const long long per_cta = (long long)kThreads * kUnroll;
    const long long need = (nvec + per_cta - 1) / per_cta;
    if (gx > need) gx = need;
    if (gx < 1) gx = 1;
    dim3 grid((unsigned)gx, (unsigned)(P * G), (unsigned)ntensors);
    scatter_blocks_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pab

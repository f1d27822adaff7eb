// layout.cu -- move a video token tensor between the spatial view [T, N, C]
// (frames outer; spatial attention runs within a frame) and the temporal
// view [N, T, C] (positions outer; temporal attention runs across frames) --
// the two views the three PAB attention kinds use (PAB report,
// "Implementation").
//
// Every token row of C channels is contiguous in both views, so the change
// is a permutation of rows of C*elem bytes.  The same engine swaps the two
// outer dimensions of [P][Q][block][C] (blocks of `block` consecutive rows
// move together): with block = 1 that is the view change, with block = N/G
// it packs and unpacks the per-rank chunks of a sequence-parallel
// all-to-all.  A persistent grid works as a
// row-gather DMA engine on the bulk-copy (TMA) unit: each unit of work is R
// consecutive DESTINATION rows; one elected thread issues R untiled
// cp.async.bulk loads (one per source row) into a shared-memory stage,
// waits on the stage's mbarrier, and writes the stage back with ONE bulk
// store of R*row_bytes (destination rows are contiguous).  S stages keep
// S*R rows in flight per CTA.  HBM traffic is the algorithmic 2 x size.
// No multicast.
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

constexpr int kStages = 4;
constexpr int kStageBytes = 16384;  // target bytes per stage
__device__ unsigned int g_layout_err = 0;

struct LayoutArgs {
    const char* src;
    char* dst;
    long long rows;      // T*N
    long long units;     // ceil(rows / R)
    int A;               // destination outer extent (dst block = a*B + b)
    int B;               // destination inner extent; source block = b*A + a
    long long inner;     // rows per block
    int row_bytes;
    int R;               // rows per unit
};

// BLOCKED = false is the view change (one-row blocks): one division per row
// on the issuing thread's path instead of two more for the block split
template <bool BLOCKED>
PAB_DEV long long src_row_of(long long dst_row, int A, int B, long long inner) {
    if constexpr (!BLOCKED) {
        const long long a = dst_row / B;
        return (dst_row - a * B) * A + a;
    } else {
        const long long blk = dst_row / inner;
        const long long w = dst_row - blk * inner;
        const long long a = blk / B;
        const long long b = blk - a * B;
        return (b * A + a) * inner + w;
    }
}

template <bool BLOCKED>
__global__ void __launch_bounds__(32) layout_bulk_kernel(LayoutArgs p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) unsigned long long full_bar[kStages];
    if (threadIdx.x != 0) return;  // one thread drives the copy engine

    const uint32_t stage_bytes = (uint32_t)p.R * p.row_bytes;
    const uint32_t smem_base = smem_u32(smem);
    for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&full_bar[s]), 1);
    fence_mbar_init();

    auto issue_load = [&](long long unit, int s) {
        const long long r0 = unit * p.R;
        long long cnt = p.rows - r0;
        if (cnt > p.R) cnt = p.R;
        const uint32_t bar = smem_u32(&full_bar[s]);
        mbar_arrive_expect_tx(bar, (uint32_t)(cnt * p.row_bytes));
        const uint32_t dst = smem_base + s * stage_bytes;
        for (long long j = 0; j < cnt; ++j) {
            const long long sr = src_row_of<BLOCKED>(r0 + j, p.A, p.B, p.inner);
            bulk_g2s(dst + (uint32_t)(j * p.row_bytes), p.src + sr * p.row_bytes,
                     (uint32_t)p.row_bytes, bar);
        }
    };

    const long long first = blockIdx.x, step = gridDim.x;
    // pending[s]: a load into stage s was issued and not yet waited for
    bool pending[kStages];
    long long waits_done[kStages];
    for (int s = 0; s < kStages; ++s) {
        pending[s] = false;
        waits_done[s] = 0;
        const long long u = first + s * step;
        if (u < p.units) {
            issue_load(u, s);
            pending[s] = true;
        }
    }
    bool ok = true;
    for (long long i = 0;; ++i) {
        const long long u = first + i * step;
        if (u >= p.units) break;
        const int s = (int)(i % kStages);
        const uint32_t parity = (uint32_t)(waits_done[s] & 1);
        if (!mbar_wait_bounded(smem_u32(&full_bar[s]), parity, &g_layout_err)) {
            ok = false;
            break;
        }
        pending[s] = false;
        waits_done[s] += 1;
        const long long r0 = u * p.R;
        long long cnt = p.rows - r0;
        if (cnt > p.R) cnt = p.R;
        bulk_s2g(p.dst + r0 * p.row_bytes, smem_base + s * stage_bytes,
                 (uint32_t)(cnt * p.row_bytes));
        bulk_commit();
        // refill the stage the previous unit used, once its store has read it
        if (i >= 1) {
            const long long nu = first + (i - 1 + kStages) * step;
            if (nu < p.units) {
                const int ps = (int)((i - 1) % kStages);
                bulk_wait_read<1>();
                issue_load(nu, ps);
                pending[ps] = true;
            }
        }
    }
    if (!ok) {
        // A load never completed.  Give every load still in flight one more
        // bounded wait so no copy lands in shared memory after the CTA exits.
        for (int s = 0; s < kStages; ++s)
            if (pending[s])
                mbar_wait_bounded(smem_u32(&full_bar[s]), (uint32_t)(waits_done[s] & 1),
                                  &g_layout_err);
    }
    bulk_wait<0>();
}

}  // namespace

cudaError_t launch_layout(int to_temporal, const void* src, void* dst, int T, int N,
                          int row_bytes, cudaStream_t s) {
    // to_temporal: src [T][N] -> dst [N][T]; else src [N][T] -> dst [T][N]
    return to_temporal ? launch_swap_outer(src, dst, T, N, 1, row_bytes, s)
                       : launch_swap_outer(src, dst, N, T, 1, row_bytes, s);
}

cudaError_t launch_swap_outer(const void* src, void* dst, int P, int Q, long long block, int row_bytes,
                              cudaStream_t s) {
    // src [P][Q][block] rows -> dst [Q][P][block]: dst block q*P + p <- src block p*Q + q
    LayoutArgs p;
    p.src = static_cast<const char*>(src);
    p.dst = static_cast<char*>(dst);
    p.rows = (long long)P * Q * block;
    p.row_bytes = row_bytes;
    p.A = Q;
    p.B = P;
    p.inner = block;
    int R = kStageBytes / row_bytes;
    if (R < 1) R = 1;
    p.R = R;
    p.units = (p.rows + R - 1) / R;
    if (p.rows == 0) return cudaSuccess;
    const size_t smem = (size_t)kStages * R * row_bytes;
    // the kernel's static shared memory (barriers) comes on top of `smem`
    auto kern = block == 1 ? layout_bulk_kernel<false> : layout_bulk_kernel<true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int per_sm = (int)((200 * 1024) / (smem + 1024));
    long long grid = (long long)device_sm_count() * (per_sm < 1 ? 1 : per_sm);
    if (grid > p.units) grid = p.units;
    kern<<<(unsigned)grid, 32, smem, s>>>(p);
    return cudaGetLastError();
}

unsigned int layout_device_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_layout_err, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_layout_err, &z, sizeof(z));
    }
    return v;
}

}  // namespace pab

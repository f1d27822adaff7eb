// temporal.cu -- temporal attention: at every spatial position n and head h
// the T frames attend to each other (PAB report, "Implementation": temporal
// attention, the mid-frequency kind).  q, k, v, out: [N, T, C] (temporal
// view) or, with no separate layout change, [T, N, C] (spatial view: the TMA
// tensor maps gather a position's frames at stride N*C), bf16.  L = T is short (16..64 in the workloads), the batch
// (N * heads) is in the tens of thousands, so the kernel is HBM-bound
// (2 * T * d * 2 flop per loaded byte ~ 8-32 flop/B).
//
// Design:
//  - warp specialisation: a producer warp (one thread) issues each unit's
//    TMA loads into a stage and, once every compute warp has arrived on the
//    stage's done barrier, the TMA store of its output; the 8 compute warps
//    wait only on the stage's full barrier (no block-wide barriers);
//  - persistent grid; a unit of work is (position n, group of G heads), G
//    the smallest head count that gives each of the 8 warps a task when two
//    such stages fit one CTA per SM (d = 128, T = 24: G = 4), else the largest
//    that keeps two CTAs per SM (more warps hide the warp-MMA latency); the
//    unit's q, k, v arrive with TMA tensor loads (one [T rows][P cols] box
//    per tensor and head), double-buffered across units so the next unit's
//    loads overlap this unit's math, and the output leaves with TMA stores;
//  - one warp per (head, 16-query tile): QK^T and PV run on warp-level bf16
//    MMA (m16n8k16, fp32 accumulate) from ldmatrix fragments; the softmax is
//    an online (streaming) softmax over 16-key blocks with quad shuffles;
//  - a head's rows have a pitch of P elements with P/8 odd (P = d or d + 8),
//    so the eight 16-byte rows an ldmatrix phase reads hit distinct banks;
//    the tensor map's innermost extent is d, so columns d..P-1 load as zero;
//    rows T..RT-1 (RT = T rounded up to 16) stay zero from the start.
// Waits on the stage barriers are bounded; on time-out the CTA raises the
// error word and stops after its copies in flight have landed.
#include <cuda.h>

#include "kernels.h"
#include "tc.cuh"

namespace pab {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = (kWarps + 1) * 32;  // 8 compute warps + a TMA producer warp
constexpr int kMaxStageBytes = 56 * 1024;        // two CTAs per SM
constexpr int kMaxStageBytesLarge = 110 * 1024;  // one CTA per SM
constexpr float kLog2e = 1.4426950408889634f;

__device__ unsigned int g_temporal_err = 0;

struct TemporalArgs {
    int N, T, heads, d;
    int spatial_view;  // 1: tensors are [T, N, C] (tensor map dims (d, heads, N, T))
    int G;       // heads per unit
    int P;       // smem row pitch (elements) = TMA box width
    int RT;      // rows per head block in smem (T rounded up to 16)
    long long units;
    float scale_log2;  // log2(e) / sqrt(d)
};

// smem layout of one stage: [3 tensors][G heads][RT rows][P cols] bf16
template <int DN>
__global__ void __launch_bounds__(kThreads) temporal_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_k,
                                                            const __grid_constant__ CUtensorMap tm_v,
                                                            const __grid_constant__ CUtensorMap tm_o,
                                                            TemporalArgs p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) unsigned long long full_bar[2];
    __shared__ __align__(8) unsigned long long done_bar[2];  // every compute warp finished the stage's unit
    __shared__ int abort_flag;
    constexpr int DK = (DN + 1) / 2;  // 16-wide k chunks covering d
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.G, P = p.P, RT = p.RT, T = p.T;
    const int head_elems = RT * P;
    const int tensor_elems = G * head_elems;
    const int stage_elems = 3 * tensor_elems;
    const int hg_count = p.heads / G;
    const uint32_t unit_bytes = 3u * G * T * P * 2;

    // zero both stages once: padding rows are never written afterwards
    {
        uint4* z = reinterpret_cast<uint4*>(smem);
        const int n16 = (2 * stage_elems * 2 + 256) / 16;
        for (int i = tid; i < n16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&done_bar[s]), kWarps);
        }
        abort_flag = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
        tc::prefetch_tmap(&tm_o);
    }
    // generic-proxy zeroing must be visible to the async proxy (TMA writes)
    fence_proxy_async_smem();
    __syncthreads();

    __nv_bfloat16* sbase = reinterpret_cast<__nv_bfloat16*>(smem);
    const uint32_t sbase_u32 = smem_u32(smem);
    auto issue_unit = [&](long long unit, int stage) {
        const int n = (int)(unit / hg_count);
        const int h0 = (int)(unit - (long long)n * hg_count) * G;
        const uint32_t bar = smem_u32(&full_bar[stage]);
        mbar_arrive_expect_tx(bar, unit_bytes);
        // position n is coordinate 3 of the temporal-view map, 2 of the spatial-view one
        const int c2 = p.spatial_view ? n : 0, c3 = p.spatial_view ? 0 : n;
        for (int g = 0; g < G; ++g) {
            const uint32_t dst = sbase_u32 + 2u * (stage * stage_elems + g * head_elems);
            tc::tma_load_4d(dst, &tm_q, 0, h0 + g, c2, c3, bar);
            tc::tma_load_4d(dst + 2u * tensor_elems, &tm_k, 0, h0 + g, c2, c3, bar);
            tc::tma_load_4d(dst + 4u * tensor_elems, &tm_v, 0, h0 + g, c2, c3, bar);
        }
    };

    const long long first = blockIdx.x, step = gridDim.x;
    const int mtiles = RT / 16;
    const int tasks = G * mtiles;
    auto store_unit = [&](long long unit, int stage) {
        const int n = (int)(unit / hg_count);
        const int h0 = (int)(unit - (long long)n * hg_count) * G;
        const int c2 = p.spatial_view ? n : 0, c3 = p.spatial_view ? 0 : n;
        for (int g = 0; g < G; ++g)
            tc::tma_store_4d(&tm_o, sbase_u32 + 2u * (stage * stage_elems + g * head_elems), 0, h0 + g, c2, c3);
        bulk_commit();
    };

    if (warp == kWarps) {
        // ------------------------------------------------ producer warp (one thread)
        if (lane == 0) {
            // unit k of this CTA uses stage k & 1; before stage s takes unit k, the
            // output of unit k-2 (computed in it) is stored and the store has read it
            long long k = 0, n_issued = 0;
            bool ok = true;
            for (long long u = first; u < p.units; u += step, ++k) {
                const int s = (int)(k & 1);
                if (k >= 2) {
                    ok = mbar_wait_bounded(smem_u32(&done_bar[s]), (uint32_t)(((k - 2) >> 1) & 1), &g_temporal_err);
                    if (!ok) break;
                    store_unit(u - 2 * step, s);
                    bulk_wait_read<0>();
                }
                issue_unit(u, s);
                n_issued = k + 1;
            }
            // the last (up to) two units' outputs
            for (long long kk = (k >= 2 ? k - 2 : 0); ok && kk < k; ++kk) {
                const int s = (int)(kk & 1);
                ok = mbar_wait_bounded(smem_u32(&done_bar[s]), (uint32_t)((kk >> 1) & 1), &g_temporal_err);
                if (ok) store_unit(first + kk * step, s);
            }
            if (!ok) {
                abort_flag = 1;
                // let every load this CTA issued land before it exits (bounded)
                for (long long kk = (n_issued > 2 ? n_issued - 2 : 0); kk < n_issued; ++kk)
                    mbar_wait_bounded(smem_u32(&full_bar[kk & 1]), (uint32_t)((kk >> 1) & 1), &g_temporal_err);
            }
            bulk_wait<0>();
        }
    } else {
        // ------------------------------------------------ compute warps
        long long i = 0;
        for (long long u = first; u < p.units; u += step, ++i) {
            const int stage = (int)(i & 1);
            // unit i is the (i >> 1)-th use of its stage
            if (!mbar_wait_bounded(smem_u32(&full_bar[stage]), (uint32_t)((i >> 1) & 1), &g_temporal_err)) {
                abort_flag = 1;
                break;
            }
            if (*(volatile int*)&abort_flag) break;
        __nv_bfloat16* st = sbase + stage * stage_elems;
        for (int task = warp; task < tasks; task += kWarps) {
            const int g = task / mtiles, mt = task - (task / mtiles) * mtiles;
            __nv_bfloat16* qs = st + g * head_elems + mt * 16 * P;
            const __nv_bfloat16* ks = st + tensor_elems + g * head_elems;
            const __nv_bfloat16* vs = st + 2 * tensor_elems + g * head_elems;

            uint32_t qa[DK][4];
#pragma unroll
            for (int kc = 0; kc < DK; ++kc)
                ldsm_x4(smem_u32(qs + (lane & 15) * P + kc * 16 + (lane >> 4) * 8), qa[kc][0], qa[kc][1],
                        qa[kc][2], qa[kc][3]);
            if (DN & 1) {  // d % 16 == 8: the last chunk's upper 8 columns are past d
                qa[DK - 1][2] = 0u;
                qa[DK - 1][3] = 0u;
            }
            float o[DN][4];
#pragma unroll
            for (int j = 0; j < DN; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

            for (int kb = 0; kb < mtiles; ++kb) {
                float s[2][4];
#pragma unroll
                for (int j = 0; j < 2; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
                for (int kc = 0; kc < DK; ++kc) {
                    uint32_t b0, b1, b2, b3;
                    const int krow = kb * 16 + (lane & 7) + ((lane >> 4) << 3);
                    const int kcol = kc * 16 + ((lane >> 3) & 1) * 8;
                    ldsm_x4(smem_u32(ks + krow * P + kcol), b0, b1, b2, b3);
                    mma_bf16_16816(s[0], qa[kc][0], qa[kc][1], qa[kc][2], qa[kc][3], b0, b1);
                    mma_bf16_16816(s[1], qa[kc][0], qa[kc][1], qa[kc][2], qa[kc][3], b2, b3);
                }
                float mx0 = m0, mx1 = m1;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int key = kb * 16 + j * 8 + 2 * (lane & 3);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool valid = (key + e) < T;
                        s[j][e] = valid ? s[j][e] * p.scale_log2 : -INFINITY;
                        s[j][2 + e] = valid ? s[j][2 + e] * p.scale_log2 : -INFINITY;
                        mx0 = fmaxf(mx0, s[j][e]);
                        mx1 = fmaxf(mx1, s[j][2 + e]);
                    }
                }
                mx0 = quad_max(mx0);
                mx1 = quad_max(mx1);
                const float c0 = ex2(m0 - mx0), c1 = ex2(m1 - mx1);
                m0 = mx0;
                m1 = mx1;
                float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        s[j][e] = ex2(s[j][e] - mx0);
                        s[j][2 + e] = ex2(s[j][2 + e] - mx1);
                        ps0 += s[j][e];
                        ps1 += s[j][2 + e];
                    }
                }
                l0 = l0 * c0 + ps0;
                l1 = l1 * c1 + ps1;
#pragma unroll
                for (int j = 0; j < DN; ++j) {
                    o[j][0] *= c0;
                    o[j][1] *= c0;
                    o[j][2] *= c1;
                    o[j][3] *= c1;
                }
                const uint32_t pa0 = pack_bf16x2(s[0][0], s[0][1]);
                const uint32_t pa1 = pack_bf16x2(s[0][2], s[0][3]);
                const uint32_t pa2 = pack_bf16x2(s[1][0], s[1][1]);
                const uint32_t pa3 = pack_bf16x2(s[1][2], s[1][3]);
                const int vrow = kb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
                for (int j = 0; j < DN; j += 2) {
                    if (j + 1 < DN) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(smem_u32(vs + vrow * P + j * 8 + (lane >> 4) * 8), b0, b1, b2, b3);
                        mma_bf16_16816(o[j], pa0, pa1, pa2, pa3, b0, b1);
                        mma_bf16_16816(o[j + 1], pa0, pa1, pa2, pa3, b2, b3);
                    } else {
                        uint32_t b0, b1;
                        ldsm_x2_t(smem_u32(vs + vrow * P + j * 8), b0, b1);
                        mma_bf16_16816(o[j], pa0, pa1, pa2, pa3, b0, b1);
                    }
                }
            }
            l0 = quad_sum(l0);
            l1 = quad_sum(l1);
            const float inv0 = 1.f / l0, inv1 = 1.f / l1;
            // stage O (bf16) over this warp's own q rows
            const int r0 = lane >> 2, cq = 2 * (lane & 3);
#pragma unroll
            for (int j = 0; j < DN; ++j) {
                *reinterpret_cast<uint32_t*>(qs + r0 * P + j * 8 + cq) = pack_bf16x2(o[j][0] * inv0, o[j][1] * inv0);
                *reinterpret_cast<uint32_t*>(qs + (r0 + 8) * P + j * 8 + cq) =
                    pack_bf16x2(o[j][2] * inv1, o[j][3] * inv1);
            }
        }
            // the outputs are written over this warp's own q rows: visible to the
            // TMA store (async proxy) once the producer sees every warp's arrival
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&done_bar[stage]));
        }
    }
}

// 4-D map over the temporal view [N][T][heads][d]: dims (d, heads, T, N),
// box (P, 1, T, 1); or over the spatial view [T][N][heads][d]: dims
// (d, heads, N, T), box (P, 1, 1, T).  Either way one box is a position's T
// frames of one head, landing as [T][P] in shared memory.  No swizzle;
// columns d..P-1 of the box read as zero.
bool make_map(CUtensorMap* m, const void* base, int d, int heads, int T, int N, int P, int spatial_view) {
    typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    const long long C = (long long)heads * d;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)N};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)C * 2, (cuuint64_t)T * C * 2};
    cuuint32_t box[4] = {(cuuint32_t)P, 1, (cuuint32_t)T, 1};
    if (spatial_view) {
        dims[2] = (cuuint64_t)N;
        dims[3] = (cuuint64_t)T;
        strides[2] = (cuuint64_t)N * C * 2;
        box[2] = 1;
        box[3] = (cuuint32_t)T;
    }
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DN>
cudaError_t launch_dn(const CUtensorMap* maps, const TemporalArgs& p, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(temporal_kernel<DN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, temporal_kernel<DN>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    long long grid = (long long)device_sm_count() * per_sm;
    if (grid > p.units) grid = p.units;
    temporal_kernel<DN><<<(unsigned)grid, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_temporal(const void* q, const void* k, const void* v, void* out, int N, int T,
                            int heads, int d, int spatial_view, cudaStream_t s) {
    TemporalArgs p;
    p.spatial_view = spatial_view;
    p.N = N;
    p.T = T;
    p.heads = heads;
    p.d = d;
    p.P = ((d / 8) & 1) ? d : d + 8;
    p.RT = (T + 15) / 16 * 16;
    // heads per unit: the smallest divisor of heads that gives every warp a
    // (head, 16-row tile) task, if its stage fits the large budget (two
    // stages per CTA, one CTA per SM); otherwise the largest divisor whose
    // stage fits the small budget (two CTAs per SM)
    int G = 0;
    const int mt = p.RT / 16;
    for (int g = 1; g <= heads; ++g)
        if (heads % g == 0 && g * mt >= kWarps && 3 * g * p.RT * p.P * 2 <= kMaxStageBytesLarge) {
            G = g;
            break;
        }
    if (G == 0) {
        G = 1;
        for (int g = heads; g >= 1; --g)
            if (heads % g == 0 && 3 * g * p.RT * p.P * 2 <= kMaxStageBytes) {
                G = g;
                break;
            }
    }
    p.G = G;
    p.units = (long long)N * (heads / G);
    p.scale_log2 = kLog2e / sqrtf((float)d);
    if (p.units == 0) return cudaSuccess;
    CUtensorMap maps[4];
    const void* bases[4] = {q, k, v, out};
    for (int i = 0; i < 4; ++i)
        if (!make_map(&maps[i], bases[i], d, heads, T, N, p.P, spatial_view)) return cudaErrorInvalidValue;
    const size_t smem = (size_t)2 * 3 * G * p.RT * p.P * 2 + 256;
    switch (d / 8) {
#define PAB_T_CASE(DNV) \
    case DNV:           \
        return launch_dn<DNV>(maps, p, smem, s);
        PAB_T_CASE(1) PAB_T_CASE(2) PAB_T_CASE(3) PAB_T_CASE(4) PAB_T_CASE(5) PAB_T_CASE(6)
        PAB_T_CASE(7) PAB_T_CASE(8) PAB_T_CASE(9) PAB_T_CASE(10) PAB_T_CASE(11) PAB_T_CASE(12)
        PAB_T_CASE(13) PAB_T_CASE(14) PAB_T_CASE(15) PAB_T_CASE(16)
#undef PAB_T_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

unsigned int temporal_device_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_temporal_err, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_temporal_err, &z, sizeof(z));
    }
    return v;
}

}  // namespace pab

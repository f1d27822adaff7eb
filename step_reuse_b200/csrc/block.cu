// block.cu -- the dense parts of a video DiT block around the PAB attention
// kinds (PAB report, "Implementation": the attention modules whose outputs
// PAB broadcasts sit in DiT blocks between layer norms, projections and an
// MLP).  Two kernels:
//
// gemm_tc_kernel: D = epilogue(A B) on the 5th-generation tensor cores, A
//   [M, K] bf16 row-major (K-major), B [K, N] bf16 row-major (the weights as
//   [in, out], read MN-major), fp32 accumulators in TMEM.  Persistent CTAs
//   walk 128 x BN output tiles (BN = 256 unless N <= 128), the smaller
//   operand's tile index fastest: M
//   fastest within an N column of tiles when B is the larger operand (the
//   CTAs running at one time share B and neighbouring A rows in L2), N
//   fastest within an M row of tiles when A is (an A row block is read from
//   HBM once and reused by the CTAs taking that row's N tiles, instead of A
//   being streamed once per N column when it does not fit in L2):
//     warp 4 (one thread)  TMA producer: a ring of NS stages of one
//                          [128][64] A box and BN/64 [64][64] B boxes;
//     warp 5               MMA issuer (warp-uniform, one elected lane), 4
//                          tcgen05.mma (M 128, N BN, K 16) per stage into one
//                          of two TMEM accumulators, so the epilogue of tile i
//                          runs under the MMAs of tile i+1; also owns TMEM;
//     warps 0-3            epilogue: thread i owns row i of the tile (TMEM
//                          lane i), reads 32 columns at a time and applies
//                            kStore  D = bf16(acc), columns split over up to
//                                    three outputs of `split` columns each
//                                    (q, k, v of one projection),
//                            kGelu   D = bf16(GELU_tanh(acc)),
//                            kResid  X += acc in fp32 (the residual stream)
//                                    and, when Y is given, Y = bf16(acc).
//   Rows past M, columns past N and the K tail past K are zero-filled on
//   load; rows and columns past M and N are not stored.
// ln_rows_kernel: h = bf16(LayerNorm(x)) per row of C fp32 values (no affine,
//   eps 1e-6), optionally after x += y0 + y1 + y2 (broadcast module outputs
//   added to the residual stream, written back): one warp per row, two
//   passes over registers.  HBM-bound.
// Every wait on an mbarrier is bounded; on time-out the CTA raises the error
// word, lets its copies and MMAs drain, frees TMEM and exits.
#include <cuda.h>

#include "kernels.h"
#include "tc.cuh"

namespace pab {
namespace {

__device__ unsigned int g_block_err = 0;

constexpr int kBM = 128, kBK = 64;
constexpr int kABox = 128 * 128;  // [128 rows][64 cols] bf16
constexpr int kBBox = 64 * 128;   // [64 K rows][64 N cols] bf16
constexpr int kThreads = 192;     // 4 epilogue warps + producer + MMA issuer
constexpr int kLnMaxVec = 24;     // layer norm: float4 per lane, C <= 32 * 4 * kLnMaxVec = 3072

enum { kStore = 0, kGelu = 1, kResid = 2 };

struct GemmArgs {
    int M, N, K;
    int m_tiles, n_tiles;
    long long tiles;
    int n_fast;  // tile t is (t / n_tiles, t % n_tiles) when set, else (t % m_tiles, t / m_tiles)
    // kStore: outputs out[0..2], each [M, split] row-major (split = N when one)
    __nv_bfloat16* out[3];
    int split;
    // kResid: X [M, N] fp32 += acc; Y [M, N] bf16 = acc when not null
    float* X;
    __nv_bfloat16* Y;
};

struct GemmBars {
    unsigned long long full[8], empty[8];
    unsigned long long acc_full[2], acc_empty[2];
    unsigned long long mma_done;
    uint32_t tmem_base;
    int abort;
};

PAB_DEV bool gwait(GemmBars* b, unsigned long long* bar, uint32_t parity) {
    if (mbar_test_wait(smem_u32(bar), parity)) return true;
    if (*(volatile int*)&b->abort) return false;
    if (!mbar_wait_bounded(smem_u32(bar), parity, &g_block_err)) {
        *(volatile int*)&b->abort = 1;
        return false;
    }
    return true;
}

PAB_DEV float gelu_tanh(float x) {
    const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
    return 0.5f * x * (1.f + tanhf(k0 * fmaf(0.044715f * x, x * x, x)));
}

template <int BN, int NS, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, GemmArgs g) {
    constexpr int NBB = BN / 64;                     // B boxes per stage
    constexpr uint32_t kStage = kABox + NBB * kBBox;  // bytes per stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ GemmBars bars;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 128) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&bars.full[s]), 1);
            mbar_init(smem_u32(&bars.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bars.acc_full[b]), 1);
            mbar_init(smem_u32(&bars.acc_empty[b]), 128);
        }
        mbar_init(smem_u32(&bars.mma_done), 1);
        bars.abort = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&tm_a);
        tc::prefetch_tmap(&tm_b);
    }
    if (warp == 5) {
        tc::tmem_alloc(smem_u32(&bars.tmem_base), 2 * BN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars.tmem_base;
    const int ksteps = (g.K + kBK - 1) / kBK;  // the K tail reads zeros past K

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            long long it = 0;  // stage uses issued
            bool ok = true;
            for (long long t = blockIdx.x; t < g.tiles && ok; t += gridDim.x) {
                const int mt = g.n_fast ? (int)(t / g.n_tiles) : (int)(t % g.m_tiles);
                const int nt = g.n_fast ? (int)(t % g.n_tiles) : (int)(t / g.m_tiles);
                for (int k = 0; k < ksteps && ok; ++k, ++it) {
                    const int s = (int)(it % NS);
                    if (it >= NS) ok = gwait(&bars, &bars.empty[s], (uint32_t)(((it / NS) - 1) & 1));
                    if (!ok) break;
                    const uint32_t bar = smem_u32(&bars.full[s]);
                    const uint32_t st = sbase + s * kStage;
                    mbar_arrive_expect_tx(bar, kStage);
                    tc::tma_load_4d(st, &tm_a, k * kBK, mt * kBM, 0, 0, bar);
                    for (int j = 0; j < NBB; ++j)
                        tc::tma_load_4d(st + kABox + j * kBBox, &tm_b, nt * BN + j * 64, k * kBK, 0, 0, bar);
                }
            }
            if (!ok || *(volatile int*)&bars.abort) {
                // drain: the loads issued land before the CTA exits (bounded)
                for (long long u = (it > NS ? it - NS : 0); u < it; ++u)
                    mbar_wait_bounded(smem_u32(&bars.full[u % NS]), (uint32_t)((u / NS) & 1), &g_block_err);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer (warp-uniform)
        constexpr uint32_t idesc = tc::idesc_bf16(kBM, BN, 0, 1);
        const uint64_t da = tc::smem_desc(sbase, 16, 1024, 2);
        const uint64_t db = tc::smem_desc(sbase + kABox, kBBox, 1024, 2);
        long long it = 0;
        int i = 0;  // tiles of this CTA
        bool ok = true;
        for (long long t = blockIdx.x; t < g.tiles && ok; t += gridDim.x, ++i) {
            const int ab = i & 1;
            if (i >= 2) ok = __all_sync(0xffffffffu, gwait(&bars, &bars.acc_empty[ab], (uint32_t)(((i - 2) >> 1) & 1)));
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t d = tmem + ab * BN;
            for (int k = 0; k < ksteps && ok; ++k, ++it) {
                const int s = (int)(it % NS);
                ok = __all_sync(0xffffffffu, gwait(&bars, &bars.full[s], (uint32_t)((it / NS) & 1)));
                if (!ok) break;
                tc::fence_after_sync();
                const uint64_t so = (uint64_t)((s * kStage) >> 4);
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    tc::mma_ss_warp(d, da + so + kk * 2, db + so + kk * 128, idesc, (k > 0 || kk > 0) ? 1u : 0u);
                tc::commit_warp(smem_u32(&bars.empty[s]));
            }
            if (ok) tc::commit_warp(smem_u32(&bars.acc_full[ab]));
        }
        tc::commit_warp(smem_u32(&bars.mma_done));
        mbar_wait_bounded(smem_u32(&bars.mma_done), 0, &g_block_err);
    } else if (warp < 4) {
        // ------------------------------------------------ epilogue: thread = row
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const int row = warp * 32 + lane;
        int i = 0;
        bool ok = true;
        for (long long t = blockIdx.x; t < g.tiles && ok; t += gridDim.x, ++i) {
            const int ab = i & 1;
            const int mt = g.n_fast ? (int)(t / g.n_tiles) : (int)(t % g.m_tiles);
            const int nt = g.n_fast ? (int)(t % g.n_tiles) : (int)(t / g.m_tiles);
            ok = gwait(&bars, &bars.acc_full[ab], (uint32_t)((i >> 1) & 1));
            if (!ok) break;
            tc::fence_after_sync();
            const long long m = (long long)mt * kBM + row;
            const bool row_in = m < g.M;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc::ld_32col(lane_addr + ab * BN + c * 32, r);
                tc::wait_ld();
                const int n0 = nt * BN + c * 32;  // the chunk's first column
                if (!row_in || n0 >= g.N) continue;  // N % 32 == 0: a chunk is wholly in or out
                if constexpr (EPI == kResid) {
                    float4* xp = reinterpret_cast<float4*>(g.X + m * g.N + n0);
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        float4 xv = xp[v];
                        xv.x += __uint_as_float(r[4 * v]);
                        xv.y += __uint_as_float(r[4 * v + 1]);
                        xv.z += __uint_as_float(r[4 * v + 2]);
                        xv.w += __uint_as_float(r[4 * v + 3]);
                        xp[v] = xv;
                    }
                    if (g.Y) {
                        uint4* yp = reinterpret_cast<uint4*>(g.Y + m * g.N + n0);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            yp[v] = make_uint4(
                                pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                                pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
                    }
                } else {
                    float f[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        f[e] = __uint_as_float(r[e]);
                        if constexpr (EPI == kGelu) f[e] = gelu_tanh(f[e]);
                    }
                    // column n0 of the concatenated output: output n0 / split, column n0 % split
                    const int o = n0 / g.split, cn = n0 - o * g.split;
                    uint4* dp = reinterpret_cast<uint4*>(g.out[o] + m * g.split + cn);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        dp[v] = make_uint4(pack_bf16x2(f[8 * v], f[8 * v + 1]), pack_bf16x2(f[8 * v + 2], f[8 * v + 3]),
                                           pack_bf16x2(f[8 * v + 4], f[8 * v + 5]),
                                           pack_bf16x2(f[8 * v + 6], f[8 * v + 7]));
                }
            }
            // the accumulator buffer may take the next tile
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.acc_empty[ab]));
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 2 * BN);
    }
}

struct LnArgs {
    float* x;
    const __nv_bfloat16* y[3];  // added to x first (written back) when not null
    __nv_bfloat16* h;           // LN output; null: the adds only
    long long rows;
    int C;
    float eps;
};

PAB_DEV void add_bf16x4(float4& v, const __nv_bfloat16* y, long long r, int C, int c) {
    const uint2 yy = reinterpret_cast<const uint2*>(y + r * C)[c];
    v.x += __uint_as_float(yy.x << 16);
    v.y += __uint_as_float(yy.x & 0xffff0000u);
    v.z += __uint_as_float(yy.y << 16);
    v.w += __uint_as_float(yy.y & 0xffff0000u);
}

// one warp per row: x += y0 + y1 + y2 (in that order, written back), then
// h = bf16(LN(x)) when h is not null
__global__ void __launch_bounds__(256) ln_rows_kernel(const LnArgs p) {
    const int lane = threadIdx.x & 31;
    const int C = p.C;
    const long long r0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long stride = ((long long)gridDim.x * blockDim.x) >> 5;
    const int nv = C / 4;  // float4 per row
    const bool adds = p.y[0] || p.y[1] || p.y[2];
    for (long long r = r0; r < p.rows; r += stride) {
        float4* xr = reinterpret_cast<float4*>(p.x + r * C);
        float4 v[kLnMaxVec];
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kLnMaxVec; ++i) {
            const int c = lane + 32 * i;
            if (c < nv) {
                v[i] = xr[c];
                if (adds) {
                    for (int j = 0; j < 3; ++j)
                        if (p.y[j]) add_bf16x4(v[i], p.y[j], r, C, c);
                    xr[c] = v[i];
                }
                s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
            }
        }
        if (!p.h) continue;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s / (float)C;
        float q = 0.f;
#pragma unroll
        for (int i = 0; i < kLnMaxVec; ++i) {
            const int c = lane + 32 * i;
            if (c < nv) {
                const float a = v[i].x - mean, b = v[i].y - mean, cc = v[i].z - mean, dd = v[i].w - mean;
                q += (a * a + b * b) + (cc * cc + dd * dd);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        const float rstd = rsqrtf(q / (float)C + p.eps);
        uint2* hr = reinterpret_cast<uint2*>(p.h + r * C);
#pragma unroll
        for (int i = 0; i < kLnMaxVec; ++i) {
            const int c = lane + 32 * i;
            if (c < nv)
                hr[c] = make_uint2(pack_bf16x2((v[i].x - mean) * rstd, (v[i].y - mean) * rstd),
                                   pack_bf16x2((v[i].z - mean) * rstd, (v[i].w - mean) * rstd));
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D map (cols, rows) over a row-major [rows][cols] bf16 matrix, box
// (64, box_rows), 128-byte swizzle (as 4-D with unit outer dims)
bool make_map2d(CUtensorMap* m, const void* base, long long rows, long long cols, int box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, 1, 1};
    cuuint64_t strides[3] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2, (cuuint64_t)rows * cols * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int NS, int EPI>
cudaError_t launch_gemm_t(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, cudaStream_t s) {
    constexpr size_t smem = (size_t)NS * (kABox + (BN / 64) * kBBox) + 1024;
    static_assert(smem <= 227 * 1024, "shared memory");
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, NS, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    long long grid = device_sm_count();
    if (grid > g.tiles) grid = g.tiles;
    gemm_tc_kernel<BN, NS, EPI><<<(unsigned)grid, kThreads, smem, s>>>(ma, mb, g);
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_gemm_e(const CUtensorMap& ma, const CUtensorMap& mb, GemmArgs& g, int BN, cudaStream_t s) {
    g.n_tiles = (g.N + BN - 1) / BN;
    g.tiles = (long long)g.m_tiles * g.n_tiles;
    g.n_fast = (long long)g.M * g.K > (long long)g.K * g.N ? 1 : 0;
    return BN == 256 ? launch_gemm_t<256, 4, EPI>(ma, mb, g, s) : launch_gemm_t<128, 6, EPI>(ma, mb, g, s);
}

}  // namespace

cudaError_t launch_gemm(const void* A, const void* B, int M, int N, int K, int epi, void* const* out, int split,
                        float* X, void* Y, cudaStream_t s) {
    if (M == 0 || N == 0) return cudaSuccess;
    if (K <= 0 || K % 8 || N % 32 || M < 0 || (split > 0 && split % 32)) return cudaErrorInvalidValue;
    GemmArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.m_tiles = (M + kBM - 1) / kBM;
    g.split = split > 0 ? split : N;
    for (int i = 0; i < 3; ++i) g.out[i] = (out && i * g.split < N) ? static_cast<__nv_bfloat16*>(out[i]) : nullptr;
    g.X = X;
    g.Y = static_cast<__nv_bfloat16*>(Y);
    CUtensorMap ma, mb;
    if (!make_map2d(&ma, A, M, K, kBM) || !make_map2d(&mb, B, K, N, kBK)) return cudaErrorInvalidValue;
    // 128 x 256 tiles (a last partial N tile computes zero columns past N and
    // stores nothing there); 128 x 128 only for N <= 128
    const int BN = N > 128 ? 256 : 128;
    if (epi == kStore) return launch_gemm_e<kStore>(ma, mb, g, BN, s);
    if (epi == kGelu) return launch_gemm_e<kGelu>(ma, mb, g, BN, s);
    if (epi == kResid) return launch_gemm_e<kResid>(ma, mb, g, BN, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_ln_rows(float* x, const void* const* ys, int ny, void* h, long long rows, int C, float eps,
                           cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    if (C % 4 || C > 32 * 4 * kLnMaxVec || ny < 0 || ny > 3) return cudaErrorInvalidValue;
    LnArgs p;
    p.x = x;
    for (int j = 0; j < 3; ++j) p.y[j] = j < ny ? static_cast<const __nv_bfloat16*>(ys[j]) : nullptr;
    p.h = static_cast<__nv_bfloat16*>(h);
    p.rows = rows;
    p.C = C;
    p.eps = eps;
    const int per_block = 256 / 32;
    long long grid = (rows + per_block - 1) / per_block;
    const long long cap = (long long)device_sm_count() * 16;
    if (grid > cap) grid = cap;
    ln_rows_kernel<<<(unsigned)grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

unsigned int block_device_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_block_err, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_block_err, &z, sizeof(z));
    }
    return v;
}

}  // namespace pab

// cross_tc.cu -- cross attention (video tokens attend to the text tokens;
// PAB report, "Implementation": the most stable kind) for text lengths up
// to 128: softmax(Q Kt^T / sqrt(d)) Vt per head, Q [R, C], Kt / Vt
// [text_len, C].  All text keys fit one 128-key tile, so each query tile is
// one S product, one softmax (no running max) and one PV product; the
// kernel is bound by streaming Q in and O out of HBM.
//
// Persistent CTAs (one per SM) each own a contiguous run of (head, 128-row
// query tile) work items and alternate them between two slots:
//   warp 8 (one thread)      TMA producer: the current head's Kt / Vt
//                            (reloaded when the head changes, once both
//                            issuers' MMAs on the old ones have retired --
//                            a barrier each issuer commits once per change,
//                            so no wait is ever two phases behind) and the query
//                            tiles through a ring of three Q buffers; a
//                            buffer is refilled as soon as its S product has
//                            retired, so loads run two to three tiles ahead;
//   warps 9, 10 (one thread) tcgen05.mma issuers, one per slot: S = Q Kt^T
//                            (SS form, fp32 in TMEM) and O = P Vt (TS form,
//                            P from TMEM);
//   warps 0-3 / 4-7          softmax and epilogue of slot 0 / 1: thread i
//                            owns row i (TMEM lane i), masks keys past
//                            text_len, exponentiates (MUFU ex2 with a share
//                            on the FMA pipes), writes P as bf16 over S, then
//                            normalises O, stages it (128-byte swizzle) in the
//                            slot's output buffer and stores it with TMA.
// TMEM: S_0 [0,128), S_1 [128,256), O_0 [256,256+NO), O_1 [384,384+NO).
// Every wait is bounded; on time-out the CTA raises the error word, drains
// its copies and MMAs, frees TMEM and exits.
#include <cuda.h>

#include "kernels.h"
#include "tc.cuh"

namespace pab {
namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // text keys (one tile; text_len <= 128)
constexpr int kBox = 128 * 128;   // bytes of one [128 rows][64 cols] bf16 box
constexpr int kThreads = 352;     // 2 softmax warpgroups + producer + 2 MMA warps
constexpr uint32_t kTmemCols = 512;
constexpr int kPolyPairsOf8 = 3;  // share of exponentials on the FMA pipes
constexpr float kC0 = 1.0f, kC1 = 0.693282962f, kC2 = 0.242210999f, kC3 = 0.0550089180f;

__device__ unsigned int g_cross_err = 0;

struct CrossArgs {
    int Lk;            // text_len (<= 128)
    int nqt;           // query tiles per head
    long long tiles;   // heads * nqt
    float scale_log2;  // log2(e) / sqrt(d)
};

constexpr int kQBufs = 3;

struct Bars {
    unsigned long long kv_full;
    unsigned long long kv_free;  // both issuers are done with the previous head's Kt / Vt
    unsigned long long q_full[kQBufs];
    unsigned long long q_free[kQBufs];  // the S product reading the buffer retired
    unsigned long long s_done[2];
    unsigned long long p_full[2];
    unsigned long long o_full[2];
    unsigned long long o_free[2];
    unsigned long long mma_done[2];
    uint32_t tmem_base;
    int abort;
};

PAB_DEV float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipes for a pair, x <= 0 here (no running max): range
// reduction x = rint(x) + f, f in [-0.5, 0.5], a degree-3 polynomial for 2^f
// fitted here as a minimax of the relative error with p(0) = 1 fixed (so
// integer x, the row maximum in particular, give exact powers of two; max
// relative error 1.0e-4) and the exponent added directly; x < -120 is
// clamped (result ~1e-36).
PAB_DEV void exp2_poly2(float x0, float x1, float& p0, float& p1) {
    const tc::f32x2 x = tc::pack2(fmaxf(x0, -120.0f), fmaxf(x1, -120.0f));
    const tc::f32x2 magic = tc::pack2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    const tc::f32x2 y = tc::add2(x, magic);
    const tc::f32x2 f = tc::sub2(x, tc::sub2(y, magic));
    tc::f32x2 p = tc::fma2(tc::pack2(kC3, kC3), f, tc::pack2(kC2, kC2));
    p = tc::fma2(p, f, tc::pack2(kC1, kC1));
    p = tc::fma2(p, f, tc::pack2(kC0, kC0));
    float q0, q1, y0, y1;
    tc::unpack2(p, q0, q1);
    tc::unpack2(y, y0, y1);
    p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(y0) << 23));
    p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(y1) << 23));
}

// bounded wait that gives up at once when the CTA has already aborted (a
// phase that has completed is taken without reading the abort flag)
PAB_DEV bool wait_bar(Bars* b, unsigned long long* bar, uint32_t parity) {
    if (mbar_test_wait(smem_u32(bar), parity)) return true;
    if (*(volatile int*)&b->abort) return false;
    if (!mbar_wait_bounded(smem_u32(bar), parity, &g_cross_err)) {
        *(volatile int*)&b->abort = 1;
        return false;
    }
    return true;
}

template <int KSTEPS>
__global__ void __launch_bounds__(kThreads, 1)
    cross_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    CrossArgs a) {
    constexpr int NB = (KSTEPS + 3) / 4;
    constexpr int NO = KSTEPS * 16;
    constexpr uint32_t kTile = NB * kBox;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ Bars bars;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t q_s = sbase;                 // [kQBufs][NB boxes]
    const uint32_t o_s = q_s + kQBufs * kTile;  // [2 slots][NB boxes]: output staging
    const uint32_t k_s = o_s + 2 * kTile;       // [NB boxes]
    const uint32_t v_s = k_s + kTile;           // [NB boxes]
    unsigned char* gen_base = smem_raw + (sbase - smem_u32(smem_raw));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's contiguous run of work items
    // (work-item indices fit 32 bits: heads * query tiles < 2^31, checked on the host)
    const int tiles = (int)a.tiles;
    const int per = (tiles + (int)gridDim.x - 1) / (int)gridDim.x;
    const int t_begin = (int)blockIdx.x * per;
    const int t_end = t_begin + per < tiles ? t_begin + per : tiles;
    const int n = t_begin < t_end ? t_end - t_begin : 0;

    if (threadIdx.x == 256) {
        mbar_init(smem_u32(&bars.kv_full), 1);
        mbar_init(smem_u32(&bars.kv_free), 2);
        for (int b = 0; b < kQBufs; ++b) {
            mbar_init(smem_u32(&bars.q_full[b]), 1);
            mbar_init(smem_u32(&bars.q_free[b]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_done[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 128);
            mbar_init(smem_u32(&bars.o_full[x]), 1);
            mbar_init(smem_u32(&bars.o_free[x]), 128);
            mbar_init(smem_u32(&bars.mma_done[x]), 1);
        }
        bars.abort = 0;
        fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_v);
        tc::prefetch_tmap(&tm_o);
    }
    if (warp == 9) {
        tc::tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int cur_h = -1, heads_loaded = 0, nq = 0;
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                const int t = t_begin + i;
                const int h = t / a.nqt, qt = t - h * a.nqt;
                if (h != cur_h) {
                    // every MMA of the earlier tiles has retired before Kt / Vt change:
                    // each issuer commits kv_free once per head change
                    if (heads_loaded > 0) ok = wait_bar(&bars, &bars.kv_free, (heads_loaded - 1) & 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(smem_u32(&bars.kv_full), 2 * kTile);
                    for (int bx = 0; bx < NB; ++bx) {
                        tc::tma_load_4d(k_s + bx * kBox, &tm_k, bx * 64, h, 0, 0, smem_u32(&bars.kv_full));
                        tc::tma_load_4d(v_s + bx * kBox, &tm_v, bx * 64, h, 0, 0, smem_u32(&bars.kv_full));
                    }
                    cur_h = h;
                    ++heads_loaded;
                }
                const int b = i % kQBufs;
                if (i >= kQBufs) ok = wait_bar(&bars, &bars.q_free[b], ((i / kQBufs) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(smem_u32(&bars.q_full[b]), kTile);
                for (int bx = 0; bx < NB; ++bx)
                    tc::tma_load_4d(q_s + b * kTile + bx * kBox, &tm_q, bx * 64, h, qt * kBM, 0,
                                    smem_u32(&bars.q_full[b]));
                nq = i + 1;
            }
            if (!ok || *(volatile int*)&bars.abort) {
                // drain: every load issued lands before the CTA exits (bounded)
                for (int i = (nq > kQBufs ? nq - kQBufs : 0); i < nq; ++i)
                    mbar_wait_bounded(smem_u32(&bars.q_full[i % kQBufs]), (i / kQBufs) & 1, &g_cross_err);
                if (heads_loaded > 0)
                    mbar_wait_bounded(smem_u32(&bars.kv_full), (heads_loaded - 1) & 1, &g_cross_err);
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------ MMA issuers (slot x: tiles i = x, x+2, ...)
        const int x = warp - 9;
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16(kBM, kBN, 0, 0);
            constexpr uint32_t idesc_o = tc::idesc_bf16(kBM, NO, 0, 1);
            const uint64_t dq = tc::smem_desc(q_s, 16, 1024, 2);
            const uint64_t dk = tc::smem_desc(k_s, 16, 1024, 2);
            const uint64_t dv = tc::smem_desc(v_s, kBox, 1024, 2);
            const uint32_t s_t = tmem + x * 128, o_t = tmem + 256 + x * 128;
            int heads_seen = 0;
            int hcur = -1;
            bool ok = true;
            for (int i = 0; i < n && ok; ++i) {
                // follow every Kt / Vt reload in order (also those at the other
                // slot's tiles), so a wait is never two phases behind
                const int h = (t_begin + i) / a.nqt;
                if (h != hcur) {
                    // release the old head's Kt / Vt once this issuer's MMAs on them
                    // retire, then wait for the new ones
                    if (heads_seen > 0) tc::commit(smem_u32(&bars.kv_free));
                    hcur = h;
                    ++heads_seen;
                    ok = wait_bar(&bars, &bars.kv_full, (heads_seen - 1) & 1);
                    if (!ok) break;
                }
                if ((i & 1) != x) continue;
                const int qb = i % kQBufs;
                if (ok) ok = wait_bar(&bars, &bars.q_full[qb], (i / kQBufs) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                const uint64_t a0 = dq + (uint64_t)((qb * kTile) >> 4);
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint32_t off = (ks >> 2) * (kBox >> 4) + (ks & 3) * 2;
                    tc::mma_ss(s_t, a0 + off, dk + off, idesc_s, ks > 0 ? 1u : 0u);
                }
                tc::commit(smem_u32(&bars.s_done[x]));
                tc::commit(smem_u32(&bars.q_free[qb]));  // the Q buffer may be refilled
                // O_X is free once the previous tile of this slot was read out
                if (i >= 2) ok = wait_bar(&bars, &bars.o_free[x], ((i - 2) >> 1) & 1);
                if (ok) ok = wait_bar(&bars, &bars.p_full[x], (i >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_ts(o_t, s_t + kk * 8, dv + kk * 128, idesc_o, kk > 0 ? 1u : 0u);
                tc::commit(smem_u32(&bars.o_full[x]));
            }
            tc::commit(smem_u32(&bars.mma_done[x]));
            mbar_wait_bounded(smem_u32(&bars.mma_done[x]), 0, &g_cross_err);
        }
    } else {
        // ------------------------------------------------ softmax + epilogue (slot x)
        const int x = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t s_col = x * 128, o_col = 256 + x * 128;
        const tc::f32x2 scale2 = tc::pack2(a.scale_log2, a.scale_log2);
        bool ok = true;
        for (int i = x; i < n && ok; i += 2) {
            ok = wait_bar(&bars, &bars.s_done[x], (i >> 1) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            // pass 1: row max over the text keys (scale > 0 commutes with max)
            float mrow;
            {
                // two halves of 64 scores keep the register footprint low;
                // eight independent 3-input max chains per half
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r0[32], r1[32];
                    tc::ld_32col(lane_addr + s_col + half * 64, r0);
                    tc::ld_32col(lane_addr + s_col + half * 64 + 32, r1);
                    tc::wait_ld();
                    float sv[64];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        sv[c] = __uint_as_float(r0[c]);
                        sv[32 + c] = __uint_as_float(r1[c]);
                    }
                    if ((half + 1) * 64 > a.Lk) {  // uniform: only the half holding the end of the keys
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (half * 64 + c >= a.Lk) sv[c] = -INFINITY;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        float m = tc::max3f(mx[k], sv[k], sv[k + 8]);
                        m = tc::max3f(m, sv[k + 16], sv[k + 24]);
                        m = tc::max3f(m, sv[k + 32], sv[k + 40]);
                        mx[k] = tc::max3f(m, sv[k + 48], sv[k + 56]);
                    }
                }
                mrow = tc::max3f(tc::max3f(mx[0], mx[1], mx[2]), tc::max3f(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7])) * a.scale_log2;
            }
            // pass 2: S again, 32 columns at a time (next chunk's load in
            // flight), exponentiated, summed, written back as bf16 P over the
            // columns already consumed
            const tc::f32x2 negm2 = tc::pack2(-mrow, -mrow);
            tc::f32x2 acc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = tc::pack2(0.f, 0.f);
            uint32_t buf[2][32];
            tc::ld_32col(lane_addr + s_col, buf[0]);
            tc::wait_ld();
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c) {
                if (c + 1 < kBN / 32) tc::ld_32col(lane_addr + s_col + (c + 1) * 32, buf[(c + 1) & 1]);
                uint32_t r[16];
                if (c * 32 >= a.Lk) {
                    // no key of this chunk exists: P = 0 (uniform branch)
#pragma unroll
                    for (int e = 0; e < 16; ++e) r[e] = 0u;
                    tc::st_16col(lane_addr + s_col + c * 16, r);
                    if (c + 1 < kBN / 32) tc::wait_ld();
                    continue;
                }
                const bool tail = (c + 1) * 32 > a.Lk;  // uniform: the chunk holding the end of the keys
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int idx = c * 32 + 2 * e;
                    float s0 = __uint_as_float(buf[c & 1][2 * e]);
                    float s1 = __uint_as_float(buf[c & 1][2 * e + 1]);
                    if (tail) {
                        if (idx >= a.Lk) s0 = -INFINITY;
                        if (idx + 1 >= a.Lk) s1 = -INFINITY;
                    }
                    const tc::f32x2 t = tc::fma2(tc::pack2(s0, s1), scale2, negm2);
                    float t0, t1, p0, p1;
                    tc::unpack2(t, t0, t1);
                    if (((idx >> 1) & 7) < kPolyPairsOf8) {
                        exp2_poly2(t0, t1, p0, p1);
                    } else {
                        p0 = ex2(t0);
                        p1 = ex2(t1);
                    }
                    acc[e & 3] = tc::add2(acc[e & 3], tc::pack2(p0, p1));
                    r[e] = pack_bf16x2(p0, p1);
                }
                tc::st_16col(lane_addr + s_col + c * 16, r);
                if (c + 1 < kBN / 32) tc::wait_ld();
            }
            float l;
            {
                float a0, a1;
                tc::unpack2(tc::add2(tc::add2(acc[0], acc[1]), tc::add2(acc[2], acc[3])), a0, a1);
                l = a0 + a1;
            }
            tc::wait_st();
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.p_full[x]));

            // ---------------- epilogue: O / l -> bf16 -> tile's Q buffer -> TMA store
            ok = wait_bar(&bars, &bars.o_full[x], (i >> 1) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            // the slot's output buffer: tile i-2's store must have read it
            if (row == 0) bulk_wait_read<0>();
            tc::named_bar_sync(1 + x, 128);
            const float inv = 1.f / l;
            unsigned char* stage = gen_base + (o_s - sbase) + x * kTile;
            uint32_t ov[NO / 16][16];
#pragma unroll
            for (int c = 0; c < NO / 16; ++c) tc::ld_16col(lane_addr + o_col + c * 16, ov[c]);
            tc::wait_ld();
#pragma unroll
            for (int c = 0; c < NO / 16; ++c) {
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(ov[c][2 * e]) * inv, __uint_as_float(ov[c][2 * e + 1]) * inv);
                const int col = c * 16;
                const int bx = col >> 6;
                const int ch = (col & 63) >> 3;
                unsigned char* rowp = stage + bx * kBox + row * 128;
                *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4*>(rowp + (((ch + 1) ^ (row & 7)) << 4)) =
                    make_uint4(w[4], w[5], w[6], w[7]);
            }
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.o_free[x]));  // O_X has been read out
            fence_proxy_async_smem();
            tc::named_bar_sync(1 + x, 128);
            if (row == 0) {
                const int t = t_begin + i;
                const int h = t / a.nqt, qt = t - h * a.nqt;
                for (int bx = 0; bx < NB; ++bx)
                    tc::tma_store_4d(&tm_o, o_s + x * kTile + bx * kBox, bx * 64, h, qt * kBM, 0);
                bulk_commit();
            }
        }
        if (row == 0) bulk_wait<0>();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 4-D map (d, heads, rows, 1) over a [rows][heads][d] bf16 tensor, box
// (64, 1, 128, 1), 128-byte swizzle; columns past d and rows past `rows`
// read as zero and are not written.
bool make_map(CUtensorMap* m, const void* base, int d, int heads, long long rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    const long long C = (long long)heads * d;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows, 1};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)C * 2, (cuuint64_t)rows * C * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KSTEPS>
cudaError_t launch_ks(const CUtensorMap* m, const CrossArgs& a, cudaStream_t s) {
    constexpr int NB = (KSTEPS + 3) / 4;
    const size_t smem = (size_t)(kQBufs + 4) * NB * kBox + 1024;
    const size_t smem_req = smem < 120 * 1024 ? 120 * 1024 : smem;  // one CTA per SM (TMEM: 512 columns)
    cudaError_t e = cudaFuncSetAttribute(cross_tc_kernel<KSTEPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_req);
    if (e != cudaSuccess) return e;
    long long grid = device_sm_count();
    if (grid > a.tiles) grid = a.tiles;
    cross_tc_kernel<KSTEPS><<<(unsigned)grid, kThreads, smem_req, s>>>(m[0], m[1], m[2], m[3], a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cross(const void* q, const void* kt, const void* vt, void* out, long long R, int Lk, int heads,
                         int d, cudaStream_t s) {
    if (R == 0) return cudaSuccess;
    if (Lk > kBN) return launch_flash(q, kt, vt, out, 1, R, Lk, heads, d, 0, 0, s);
    CrossArgs a;
    a.Lk = Lk;
    const long long nqt = (R + kBM - 1) / kBM;
    if (nqt * heads >= (1LL << 31)) return cudaErrorInvalidValue;
    a.nqt = (int)nqt;
    a.tiles = (long long)heads * a.nqt;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    CUtensorMap m[4];
    if (!make_map(&m[0], q, d, heads, R) || !make_map(&m[1], kt, d, heads, Lk) ||
        !make_map(&m[2], vt, d, heads, Lk) || !make_map(&m[3], out, d, heads, R))
        return cudaErrorInvalidValue;
    switch ((d + 15) / 16) {
        case 1: return launch_ks<1>(m, a, s);
        case 2: return launch_ks<2>(m, a, s);
        case 3: return launch_ks<3>(m, a, s);
        case 4: return launch_ks<4>(m, a, s);
        case 5: return launch_ks<5>(m, a, s);
        case 6: return launch_ks<6>(m, a, s);
        case 7: return launch_ks<7>(m, a, s);
        case 8: return launch_ks<8>(m, a, s);
        default: return cudaErrorInvalidValue;
    }
}

unsigned int cross_device_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_cross_err, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_cross_err, &z, sizeof(z));
    }
    return v;
}

}  // namespace pab

// cross_tc.cu -- cross attention (video tokens attend to the text tokens;
// PAB report, "Implementation": the most stable kind) for text lengths up
// to 128: softmax(Q Kt^T / sqrt(d)) Vt per head, Q [R, C], Kt / Vt
// [text_len, C].  All text keys fit one 128-key tile, so each query tile is
// one S product, one softmax (no running max) and one PV product; the
// kernel is bound by streaming Q in and O out of HBM.
//
// Persistent CTAs (one per SM) each own a contiguous run of (head, 128-row
// query tile) work items; tile i uses S buffer i & 1 and O buffer i & 1, so
// the next tile's S is computed while the softmax works on this one:
//   warp 12 (one thread)     TMA producer: the current head's Kt / Vt
//                            (reloaded when the head changes, once the MMAs
//                            on the old ones have retired), after which it
//                            writes 1.0 into Vt's column d for every key; and
//                            the query tiles through a ring of three Q
//                            buffers, each refilled as soon as its S product
//                            has retired;
//   warp 13                  tcgen05.mma issuer (one elected lane): S(i) =
//                            Q(i) Kt^T (SS form, fp32 in TMEM) and O(i) =
//                            P(i) Vt (TS form, P from TMEM, N = d plus the
//                            ones column); S(i+2) is queued right behind
//                            P(i) Vt, whose P it overwrites (in-order
//                            execution); a tile that starts a new head also
//                            waits for every earlier P Vt to be queued;
//   warps 0-3 / 4-7          softmax of every tile, warpgroup hf taking keys
//                            [64 hf, 64 hf + 64): thread i owns row i (TMEM
//                            lane i); the two half-row maxima meet through
//                            spare TMEM columns past O_0's N (named barrier
//                            2); each half exponentiates its 64 scores (MUFU
//                            ex2 with a share on the FMA pipes) and writes
//                            its half of P as bf16 over S;
//   warps 8-11               epilogue, tiles in order: O's column d is the
//                            row sum of P (the ones column), so O / O[:, d]
//                            is normalised, staged (128-byte swizzle) in the
//                            tile's output buffer and stored with TMA.
// TMEM: S_0 [0,128), S_1 [128,256), O_0 [256,256+NO), O_1 [384,384+NO),
// exchange columns [368, 372).  Head dims up to 96 (NO <= 112).
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
constexpr int kThreads = 448;     // 2 softmax warpgroups (key halves) + epilogue warpgroup + producer + MMA warp
constexpr uint32_t kTmemCols = 512;
constexpr int kPolyPairsOf8 = 3;  // share of exponentials on the FMA pipes

__device__ unsigned int g_cross_err = 0;

struct CrossArgs {
    int Lk;            // text_len (<= 128)
    int d;             // head dim (<= 96: column d of the PV product carries the row sums)
    int nqt;           // query tiles per head
    long long tiles;   // heads * nqt
    float scale_log2;  // log2(e) / sqrt(d)
};

constexpr int kQBufs = 3;

struct Bars {
    unsigned long long kv_full;   // Kt / Vt landed
    unsigned long long kv_ready;  // ... and Vt's ones column written
    unsigned long long kv_free;   // both issuers are done with the previous head's Kt / Vt
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

PAB_DEV bool wait_bar_warp(Bars* b, unsigned long long* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_bar(b, bar, parity));
}

template <int KSTEPS, int NO>
__global__ void __launch_bounds__(kThreads, 1)
    cross_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    CrossArgs a) {
    constexpr int NB = (KSTEPS + 3) / 4;  // 64-column boxes of Q, Kt and the output (d columns)
    constexpr int NBV = (NO + 63) / 64;   // boxes of Vt: d columns + the ones column
    static_assert(NO <= 112, "O's columns 112..115 carry the softmax halves' maxima");
    constexpr uint32_t kTile = NB * kBox;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ Bars bars;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t q_s = sbase;                 // [kQBufs][NB boxes]
    const uint32_t o_s = q_s + kQBufs * kTile;  // [2 slots][NB boxes]: output staging
    const uint32_t k_s = o_s + 2 * kTile;       // [NB boxes]
    const uint32_t v_s = k_s + kTile;           // [NBV boxes]
    unsigned char* gen_base = smem_raw + (sbase - smem_u32(smem_raw));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's contiguous run of work items
    // (work-item indices fit 32 bits: heads * query tiles < 2^31, checked on the host)
    const int tiles = (int)a.tiles;
    const int per = (tiles + (int)gridDim.x - 1) / (int)gridDim.x;
    const int t_begin = (int)blockIdx.x * per;
    const int t_end = t_begin + per < tiles ? t_begin + per : tiles;
    const int n = t_begin < t_end ? t_end - t_begin : 0;

    if (threadIdx.x == 384) {
        mbar_init(smem_u32(&bars.kv_full), 1);
        mbar_init(smem_u32(&bars.kv_ready), 1);
        mbar_init(smem_u32(&bars.kv_free), 1);
        for (int b = 0; b < kQBufs; ++b) {
            mbar_init(smem_u32(&bars.q_full[b]), 1);
            mbar_init(smem_u32(&bars.q_free[b]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_done[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 256);
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
    if (warp == 13) {
        tc::tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars.tmem_base;

    if (warp == 12) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int cur_h = -1, heads_loaded = 0, nq = 0;
            bool ok = true;
            // Kt / Vt of the latest head are in flight and Vt's ones column is
            // not written yet; finished before the producer blocks on anything
            // the issuers release (they need kv_ready first)
            bool pending = false;
            auto finish_kv = [&]() -> bool {
                if (!pending) return true;
                if (!wait_bar(&bars, &bars.kv_full, (heads_loaded - 1) & 1)) return false;
                // column d of Vt (zero-filled past the head) becomes all ones, so the
                // P Vt product also delivers the row sums of P in O's column d
                const uint32_t col = (uint32_t)a.d;
                unsigned char* vbox = gen_base + (v_s - sbase) + (col >> 6) * kBox;
                const uint32_t ch = (col & 63) >> 3, e = col & 7;
                for (int r = 0; r < kBN; ++r)
                    *reinterpret_cast<uint16_t*>(vbox + r * 128 + ((ch ^ (r & 7)) << 4) + e * 2) = 0x3F80u;
                fence_proxy_async_smem();
                mbar_arrive(smem_u32(&bars.kv_ready));
                pending = false;
                return true;
            };
            for (int i = 0; i < n && ok; ++i) {
                const int t = t_begin + i;
                const int h = t / a.nqt, qt = t - h * a.nqt;
                if (h != cur_h) {
                    // every MMA of the earlier tiles has retired before Kt / Vt change:
                    // each issuer commits kv_free once per head change
                    ok = finish_kv();
                    if (ok && heads_loaded > 0) ok = wait_bar(&bars, &bars.kv_free, (heads_loaded - 1) & 1);
                    if (!ok) break;
                    mbar_arrive_expect_tx(smem_u32(&bars.kv_full), (NB + NBV) * kBox);
                    for (int bx = 0; bx < NB; ++bx)
                        tc::tma_load_4d(k_s + bx * kBox, &tm_k, bx * 64, h, 0, 0, smem_u32(&bars.kv_full));
                    for (int bx = 0; bx < NBV; ++bx)
                        tc::tma_load_4d(v_s + bx * kBox, &tm_v, bx * 64, h, 0, 0, smem_u32(&bars.kv_full));
                    ++heads_loaded;
                    pending = true;
                    cur_h = h;
                }
                const int b = i % kQBufs;
                if (i >= kQBufs) {
                    ok = finish_kv();
                    if (ok) ok = wait_bar(&bars, &bars.q_free[b], ((i / kQBufs) - 1) & 1);
                }
                if (!ok) break;
                mbar_arrive_expect_tx(smem_u32(&bars.q_full[b]), kTile);
                for (int bx = 0; bx < NB; ++bx)
                    tc::tma_load_4d(q_s + b * kTile + bx * kBox, &tm_q, bx * 64, h, qt * kBM, 0,
                                    smem_u32(&bars.q_full[b]));
                nq = i + 1;
            }
            if (ok) ok = finish_kv();
            if (!ok || *(volatile int*)&bars.abort) {
                // drain: every load issued lands before the CTA exits (bounded)
                for (int i = (nq > kQBufs ? nq - kQBufs : 0); i < nq; ++i)
                    mbar_wait_bounded(smem_u32(&bars.q_full[i % kQBufs]), (i / kQBufs) & 1, &g_cross_err);
                if (heads_loaded > 0)
                    mbar_wait_bounded(smem_u32(&bars.kv_full), (heads_loaded - 1) & 1, &g_cross_err);
            }
        }
    } else if (warp == 13) {
        // ------------------------------------------------ MMA issuer (tile i: S and O buffers i & 1)
        {
            constexpr uint32_t idesc_s = tc::idesc_bf16(kBM, kBN, 0, 0);
            constexpr uint32_t idesc_o = tc::idesc_bf16(kBM, NO, 0, 1);
            const uint64_t dq = tc::smem_desc(q_s, 16, 1024, 2);
            const uint64_t dk = tc::smem_desc(k_s, 16, 1024, 2);
            const uint64_t dv = tc::smem_desc(v_s, kBox, 1024, 2);
            int heads_seen = 0, hcur = -1;
            // S(i) = Q(i) Kt^T into buffer i & 1
            auto issue_s = [&](int i) -> bool {
                const int qb = i % kQBufs;
                if (!wait_bar_warp(&bars, &bars.q_full[qb], (i / kQBufs) & 1)) return false;
                tc::fence_after_sync();
                const uint64_t a0 = dq + (uint64_t)((qb * kTile) >> 4);
                const uint32_t s_t = tmem + (i & 1) * 128;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint32_t off = (ks >> 2) * (kBox >> 4) + (ks & 3) * 2;
                    tc::mma_ss_warp(s_t, a0 + off, dk + off, idesc_s, ks > 0 ? 1u : 0u);
                }
                tc::commit_warp(smem_u32(&bars.s_done[i & 1]));
                tc::commit_warp(smem_u32(&bars.q_free[qb]));  // the Q buffer may be refilled
                return true;
            };
            // S(i) goes into the buffer whose P the P Vt product of tile i-2 reads, so
            // it is queued once that product is (in-order execution); a tile that
            // starts a new head also waits for every earlier P Vt product to be
            // queued, then releases the old Kt / Vt and waits for the new ones
            int s_next = 0;
            auto issue_pending = [&](int pv_queued) -> bool {  // P Vt of tiles 0..pv_queued queued
                while (s_next < n && s_next <= pv_queued + 2) {
                    const int h = (t_begin + s_next) / a.nqt;
                    if (h != hcur) {
                        if (s_next > pv_queued + 1) break;
                        if (heads_seen > 0) tc::commit_warp(smem_u32(&bars.kv_free));
                        hcur = h;
                        ++heads_seen;
                        if (!wait_bar_warp(&bars, &bars.kv_ready, (heads_seen - 1) & 1)) return false;
                    }
                    if (!issue_s(s_next)) return false;
                    ++s_next;
                }
                return true;
            };
            bool ok = issue_pending(-1);
            for (int i = 0; i < n && ok; ++i) {
                const int b = i & 1;
                // O buffer b is free once the epilogue has read out tile i-2
                if (i >= 2) ok = wait_bar_warp(&bars, &bars.o_free[b], ((i - 2) >> 1) & 1);
                if (ok) ok = wait_bar_warp(&bars, &bars.p_full[b], (i >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                const uint32_t s_t = tmem + b * 128, o_t = tmem + 256 + b * 128;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_ts_warp(o_t, s_t + kk * 8, dv + kk * 128, idesc_o, kk > 0 ? 1u : 0u);
                tc::commit_warp(smem_u32(&bars.o_full[b]));
                ok = issue_pending(i);
            }
            tc::commit_warp(smem_u32(&bars.mma_done[0]));
            mbar_wait_bounded(smem_u32(&bars.mma_done[0]), 0, &g_cross_err);
        }
    } else if (warp < 8) {
        // ------------------------------------------------ softmax: warpgroup hf takes keys [64 hf, 64 hf + 64)
        // of every tile (S and O buffer i & 1).  The half-row maxima meet through
        // two spare TMEM columns past O_0's N (named barrier of both warpgroups);
        // every thread runs all n tiles and the barrier of each, also after a
        // wait gave up, so the barrier counts always match.
        const int hf = warp >> 2;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t xcol = 256 + 112;  // exchange columns [xcol, xcol + 4): O_0's columns past N (N <= 112)
        const tc::f32x2 scale2 = tc::pack2(a.scale_log2, a.scale_log2);
        const int k0 = hf * 64;  // first key of this half
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int x = i & 1;
            const uint32_t s_col = x * 128;
            if (ok) ok = wait_bar(&bars, &bars.s_done[x], (i >> 1) & 1);
            float sv[64];
            float mp = -INFINITY;
            if (ok) {
                tc::fence_after_sync();
                uint32_t r0[32], r1[32];
                tc::ld_32col(lane_addr + s_col + k0, r0);
                tc::ld_32col(lane_addr + s_col + k0 + 32, r1);
                tc::wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    sv[c] = __uint_as_float(r0[c]);
                    sv[32 + c] = __uint_as_float(r1[c]);
                }
                if (k0 + 64 > a.Lk) {  // uniform: this half holds the end of the keys
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (k0 + c >= a.Lk) sv[c] = -INFINITY;
                }
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float m = tc::max3f(sv[k], sv[k + 8], sv[k + 16]);
                    m = tc::max3f(m, sv[k + 24], sv[k + 32]);
                    m = tc::max3f(m, sv[k + 40], sv[k + 48]);
                    mx[k] = fmaxf(m, sv[k + 56]);
                }
                mp = tc::max3f(tc::max3f(mx[0], mx[1], mx[2]), tc::max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
                tc::st_1col(lane_addr + xcol + x * 2 + hf, __float_as_uint(mp));
                tc::wait_st();
            }
            // both halves' scores are in registers before either writes P over them
            tc::fence_before_sync();
            tc::named_bar_sync(2, 256);  // id 1 is the epilogue warpgroup's
            tc::fence_after_sync();
            if (!ok) continue;
            uint32_t mo_bits;
            tc::ld_1col(lane_addr + xcol + x * 2 + (hf ^ 1), mo_bits);
            tc::wait_ld();
            const float mo = __uint_as_float(mo_bits);
            // the same value in both halves (max is exact and order-free)
            const float mrow = (hf == 0 ? fmaxf(mp, mo) : fmaxf(mo, mp)) * a.scale_log2;
            const tc::f32x2 negm2 = tc::pack2(-mrow, -mrow);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int idx = c * 32 + 2 * e;
                    const tc::f32x2 t = tc::fma2(tc::pack2(sv[idx], sv[idx + 1]), scale2, negm2);
                    float t0, t1, p0, p1;
                    tc::unpack2(t, t0, t1);
                    if ((e & 7) < kPolyPairsOf8) {
                        tc::exp2_poly2(t0, t1, p0, p1);
                    } else {
                        p0 = ex2(t0);
                        p1 = ex2(t1);
                    }
                    r[e] = pack_bf16x2(p0, p1);
                }
                // P of keys [k0 + 32c, k0 + 32c + 32) as bf16 pairs: columns k0/2 + 16c
                tc::st_16col(lane_addr + s_col + hf * 32 + c * 16, r);
            }
            tc::wait_st();
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.p_full[x]));
        }
    } else if (warp < 12) {
        // ------------------------------------------------ epilogue (tiles in order, buffer i & 1)
        // Every thread runs all n iterations and both named barriers of each,
        // also after a wait gave up (then the work is skipped), so the barrier
        // counts always match.
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        constexpr int NC = NO / 16 < NB * 4 ? NO / 16 : NB * 4;  // 16-column chunks staged
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int x = i & 1;
            const uint32_t o_col = 256 + x * 128;
            if (ok) ok = wait_bar(&bars, &bars.o_full[x], (i >> 1) & 1);
            uint32_t ov[NC][16];
            float inv = 0.f;
            if (ok) {
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < NC; ++c) tc::ld_16col(lane_addr + o_col + c * 16, ov[c]);
                uint32_t lbits;  // O's column d: the row sum of P (ones column of Vt)
                tc::ld_1col(lane_addr + o_col + (uint32_t)a.d, lbits);
                tc::wait_ld();
                tc::fence_before_sync();
                mbar_arrive(smem_u32(&bars.o_free[x]));  // O_X has been read out
                inv = 1.f / __uint_as_float(lbits);
            }
            // the slot's staging buffer: the store of tile i-2 must have read it
            if (row == 0) bulk_wait_read<1>();
            tc::named_bar_sync(1, 128);
            if (ok) {
                unsigned char* stage = gen_base + (o_s - sbase) + x * kTile;
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(ov[c][2 * e]) * inv,
                                           __uint_as_float(ov[c][2 * e + 1]) * inv);
                    const int col = c * 16;
                    const int bx = col >> 6;
                    const int ch = (col & 63) >> 3;
                    unsigned char* rowp = stage + bx * kBox + row * 128;
                    *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4*>(rowp + (((ch + 1) ^ (row & 7)) << 4)) =
                        make_uint4(w[4], w[5], w[6], w[7]);
                }
                fence_proxy_async_smem();
            }
            tc::named_bar_sync(1, 128);
            if (ok && row == 0) {
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
    if (warp == 13) {
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

// NO = N of the P Vt product: d rounded up to 16, plus 16 when d is a
// multiple of 16, so that column d (the ones column) exists
template <int KSTEPS, int NO>
cudaError_t launch_ks(const CUtensorMap* m, const CrossArgs& a, cudaStream_t s) {
    constexpr int NB = (KSTEPS + 3) / 4;
    constexpr int NBV = (NO + 63) / 64;
    const size_t smem = (size_t)((kQBufs + 3) * NB + NBV) * kBox + 1024;
    const size_t smem_req = smem < 120 * 1024 ? 120 * 1024 : smem;  // one CTA per SM (TMEM: 512 columns)
    cudaError_t e = cudaFuncSetAttribute(cross_tc_kernel<KSTEPS, NO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_req);
    if (e != cudaSuccess) return e;
    long long grid = device_sm_count();
    if (grid > a.tiles) grid = a.tiles;
    cross_tc_kernel<KSTEPS, NO><<<(unsigned)grid, kThreads, smem_req, s>>>(m[0], m[1], m[2], m[3], a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cross(const void* q, const void* kt, const void* vt, void* out, long long R, int Lk, int heads,
                         int d, cudaStream_t s) {
    if (R == 0) return cudaSuccess;
    // longer texts, and head dims whose P Vt product leaves no columns for the
    // row sums and the maxima exchange, take the general flash kernel
    if (Lk > kBN || d > 96) return launch_flash(q, kt, vt, out, 1, R, Lk, heads, d, 0, 0, s);
    CrossArgs a;
    a.Lk = Lk;
    a.d = d;
    const long long nqt = (R + kBM - 1) / kBM;
    if (nqt * heads >= (1LL << 31)) return cudaErrorInvalidValue;
    a.nqt = (int)nqt;
    a.tiles = (long long)heads * a.nqt;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    CUtensorMap m[4];
    if (!make_map(&m[0], q, d, heads, R) || !make_map(&m[1], kt, d, heads, Lk) ||
        !make_map(&m[2], vt, d, heads, Lk) || !make_map(&m[3], out, d, heads, R))
        return cudaErrorInvalidValue;
    const bool extra = d % 16 == 0;  // no padding column inside ceil16(d): one more 16-column chunk
    switch ((d + 15) / 16) {
        case 1: return extra ? launch_ks<1, 32>(m, a, s) : launch_ks<1, 16>(m, a, s);
        case 2: return extra ? launch_ks<2, 48>(m, a, s) : launch_ks<2, 32>(m, a, s);
        case 3: return extra ? launch_ks<3, 64>(m, a, s) : launch_ks<3, 48>(m, a, s);
        case 4: return extra ? launch_ks<4, 80>(m, a, s) : launch_ks<4, 64>(m, a, s);
        case 5: return extra ? launch_ks<5, 96>(m, a, s) : launch_ks<5, 80>(m, a, s);
        case 6: return extra ? launch_ks<6, 112>(m, a, s) : launch_ks<6, 96>(m, a, s);
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

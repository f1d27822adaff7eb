// flash_tc.cu -- flash (online-softmax) attention on the 5th-generation
// tensor cores (tcgen05 + TMEM) for the long-sequence PAB kinds: spatial
// attention (the tokens of one frame, L = H*W) and cross attention (video
// tokens against one shared set of text keys/values) -- PAB report,
// "Implementation".  softmax(Q K^T / sqrt(d)) V per (batch, head).
//
// A CTA owns 256 query rows of one (batch, head) as two 128-row tiles A and B
// that share every K/V tile, and runs four roles:
//   warp 8 (one thread)   TMA producer: Q_A, Q_B, K_0, K_1 once, then per
//                          step j one ring slot with V_j and K_{j+2} (tiles of
//                          64 keys; K is consumed two steps before V);
//   warps 9, 10 (one thread each)  MMA issuers, one per query tile X:
//                          S_X(j) = Q_X K_j^T (SS form, fp32 in TMEM) and
//                          O_X += P_X(j) V_j (TS form: P from TMEM, V from
//                          shared memory).  S is double-buffered per tile, so
//                          S_X(j+2) is issued right behind PV_X(j) and is
//                          ready before the softmax needs it: the softmax
//                          never waits for a round trip through the tensor
//                          cores.  Warp 9 also owns TMEM;
//   warps 0-3 / 4-7       softmax of tile A / B: thread i owns query row i =
//                          TMEM lane i.  It reads its row of S with tcgen05.ld,
//                          keeps the running max and sum in registers (tree
//                          reductions, no shuffles), writes P as bf16 over S's
//                          columns and rescales O in TMEM only when the running
//                          max grew by more than 2^8 (the final O / l is exact
//                          either way).  Exponentials: 5/8 on the MUFU ex2
//                          unit, 3/8 on the FMA pipes (exp2_poly2).
//                          At the end it normalises O and writes it through
//                          shared memory with a TMA tensor store.
// Rescaling O_X at step j needs PV_X(j-1) retired: the softmax then waits for
// step j-1's slot to be done.
//
// TMEM columns: S_A0 [0,64), S_A1 [64,128), S_B0 [128,192), S_B1 [192,256),
//               O_A [256,256+NO), O_B [384,384+NO).
// Operand layouts (128-byte swizzle, TMA-written):
//   Q, K: [rows][64 cols] boxes (128 rows for Q, 64 for K), K-major (d
//         contiguous); a 16-wide K step advances the descriptor start by 32
//         bytes inside the box.
//   V:    [64 rows][64 cols] boxes read MN-major (B of the PV product has
//         N = d contiguous); a 16-key K step advances by 16 rows = 2048 bytes,
//         the next 64 columns of d are one box (8 KB) further (LBO).
// Head dims that are not a multiple of 64 read zero-filled columns past d
// (the tensor map's innermost extent is d); keys past Lk are masked to -inf;
// query rows past Lq are zero-filled on load and clipped by the TMA store; a
// B tile that lies wholly past Lq is skipped.
// Every wait on an mbarrier is bounded; on time-out the CTA raises the error
// word, lets its own asynchronous copies and MMAs drain, frees TMEM and exits.
#include <cuda.h>

#include "kernels.h"
#include "tc.cuh"

namespace pab {
namespace {

constexpr int kBM = 128;          // query rows per tile (two tiles per CTA)
constexpr int kStaTile = 16;      // sliding tile attention: 16 x 16-token tiles (the CTA's 256 queries)
constexpr int kBN = 64;           // keys per K/V tile
constexpr int kQBox = 128 * 128;  // bytes of one [128 rows][64 cols] bf16 box (Q, O)
constexpr int kKVBox = 64 * 128;  // bytes of one [64 rows][64 cols] bf16 box (K, V)
constexpr int kThreads = 384;     // 2 softmax warpgroups + producer warp + 2 MMA warps + V-ones warp
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
// Exponentials: of every 8 consecutive pairs of a row's scores, this many go
// to exp2_poly2 on the FMA pipes and the rest to the MUFU ex2 unit, which
// alone would bound the softmax (16 results per clock per SM).
#ifndef PAB_POLY_PAIRS_OF_8
#define PAB_POLY_PAIRS_OF_8 3
#endif
constexpr int kPolyPairsOf8 = PAB_POLY_PAIRS_OF_8;
#ifndef PAB_FLASH_ONES
#define PAB_FLASH_ONES 1
#endif

__device__ unsigned int g_flash_err = 0;

struct FlashTcArgs {
    int Lq;            // query rows per batch
    int Lk;            // keys per batch
    int kv_batched;    // 1: K/V have a batch coordinate (spatial); 0: shared (cross)
    int d;             // head dim
    float scale_log2;  // log2(e) / sqrt(d)
    // tile geometries only: the frame in 16 x 16 tiles; the window's reach
    // in tiles on each side of the query tile (window geometry); the key
    // tiles of every query tile, [batches][heads][tiles][kv_count] (list
    // geometry)
    int tiles_h, tiles_w, reach_h, reach_w;
    const int* kv_list;
    int kv_count;
};

// Key geometries of the flash kernel: every key of the (frame, head) row
// range; the window of 16 x 16 tiles around the query tile (sliding tile
// attention); a per-query-tile list of 16 x 16 key tiles (draft attention).
enum { kGeoFull = 0, kGeoWindow = 1, kGeoList = 2 };

constexpr int kMaxStages = 8;

// The pipeline is built around ONE commit per tile and K/V step: slot s of
// the ring holds V_j and K_{j+2} (j = s mod NST); after issuing PV_X(j) and
// S_X(j+2) tile X's issuer commits slot_done[s][X] once.  Its completion
// tells tile X's softmax that S_X(j+2) is in TMEM and proves PV_X(j) retired
// (in-order completion); the producer refills the slot once both tiles'
// barriers of the slot completed.  The tiles never wait on each other's
// MMAs, and tile B's softmax starts only once tile A's first row maximum is
// done: the two tiles' score reads and maxima then fall into each other's
// exponential phases instead of coinciding (measured 5-10% faster at
// d = 64-72; the offset fades over a long key loop).
struct Bars {
    unsigned long long q_full[2];
    unsigned long long k01_full;               // K_0, K_1 (own buffer)
    unsigned long long s01_done[2];            // [tile]: S_X(0), S_X(1) retired
    unsigned long long b_go;                   // tile A's step-0 maximum is done
    unsigned long long slot_full[kMaxStages];  // V_j (+ K_{j+2}) landed
    unsigned long long slot_ready[kMaxStages]; // ... and (ONES) V_j's column d set to 1
    unsigned long long slot_done[kMaxStages][2];  // [slot][tile]: PV_X(j), S_X(j+2) retired
    unsigned long long p_full[2][2];           // [tile][S buffer]
    unsigned long long o_done[2];              // the last PV_X retired
    unsigned long long mma_done[2];
    uint32_t tmem_base;
    int abort;
};

// bounded wait that gives up at once when the CTA has already aborted (a
// phase that has completed is taken without reading the abort flag)
PAB_DEV bool wait_bar(Bars* b, unsigned long long* bar, uint32_t parity) {
    if (mbar_test_wait(smem_u32(bar), parity)) return true;
    if (*(volatile int*)&b->abort) return false;
    if (!mbar_wait_bounded(smem_u32(bar), parity, &g_flash_err)) {
        *(volatile int*)&b->abort = 1;
        return false;
    }
    return true;
}

// ONES (head dims with d % 16 != 0): column d of every V tile -- a padding
// column inside the PV product's N = 16 * KSTEPS -- is set to 1 once the tile
// lands (warp 11), so O's column d accumulates the row sum of P with the same
// bf16 P as the numerator; the softmax then keeps no running sum.
// Tile geometries (GEO != kGeoFull): the CTA's 256 queries are one 16 x 16
// tile of the frame (tile A its upper 8 rows, tile B the lower 8, each read
// as a [8][16]-token TMA box of the [H][W] grid), and the key loop runs over
// 16 x 16 key tiles, each as four [4][16]-token blocks of 64 keys: the tiles
// of the window around the query tile, clipped at the frame edge (window),
// or the tiles listed for it (list; an index outside the frame raises the
// error word and is clamped).  Every block is whole, so nothing is masked.
template <int KSTEPS, int NST, bool ONES, int GEO>
__global__ void __launch_bounds__(kThreads, 1)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    FlashTcArgs a) {
    constexpr int NB = (KSTEPS + 3) / 4;  // 64-column boxes covering d
    constexpr int NO = KSTEPS * 16;       // N of the PV product (d rounded up to 16)
    constexpr uint32_t kQTile = NB * kQBox;
    constexpr uint32_t kKVTile = NB * kKVBox;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ Bars bars;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t q_s = sbase;                  // [2 tiles][NB boxes]
    const uint32_t k01_s = q_s + 2 * kQTile;     // [2][NB boxes]: K_0, K_1
    const uint32_t v_s = k01_s + 2 * kKVTile;    // [NST][NB boxes]: V_j
    const uint32_t k_s = v_s + NST * kKVTile;    // [NST][NB boxes]: K_{j+2}
    unsigned char* gen_base = smem_raw + (sbase - smem_u32(smem_raw));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qblk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    // tile geometries: query tile (ty, tx); window tiles [wy0, wy0 + rows) x
    // [wx0, wx0 + wcols); the list of key tiles
    constexpr bool TILED = GEO != kGeoFull;
    int ty = 0, tx = 0, wy0 = 0, wx0 = 0, wcols = 1, nkv;
    const int* klist = nullptr;
    if constexpr (TILED) {
        ty = qblk / a.tiles_w;
        tx = qblk - ty * a.tiles_w;
    }
    if constexpr (GEO == kGeoWindow) {
        wy0 = max(ty - a.reach_h, 0);
        wx0 = max(tx - a.reach_w, 0);
        const int wy1 = min(ty + a.reach_h + 1, a.tiles_h), wx1 = min(tx + a.reach_w + 1, a.tiles_w);
        wcols = wx1 - wx0;
        nkv = (wy1 - wy0) * wcols * 4;
    } else if constexpr (GEO == kGeoList) {
        klist = a.kv_list + (((long long)b * gridDim.y + h) * gridDim.x + qblk) * a.kv_count;
        nkv = a.kv_count * 4;
    } else {
        nkv = (a.Lk + kBN - 1) / kBN;
    }
    const bool has_b = TILED || qblk * 2 * kBM + kBM < a.Lq;
    const int ntiles = has_b ? 2 : 1;

    if (threadIdx.x == 256) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.q_full[x]), 1);
            for (int u = 0; u < 2; ++u) mbar_init(smem_u32(&bars.p_full[x][u]), 128);
            mbar_init(smem_u32(&bars.o_done[x]), 1);
            mbar_init(smem_u32(&bars.mma_done[x]), 1);
        }
        mbar_init(smem_u32(&bars.k01_full), 1);
        for (int x = 0; x < 2; ++x) mbar_init(smem_u32(&bars.s01_done[x]), 1);
        mbar_init(smem_u32(&bars.b_go), 128);
        for (int st = 0; st < NST; ++st) {
            mbar_init(smem_u32(&bars.slot_full[st]), 1);
            mbar_init(smem_u32(&bars.slot_ready[st]), 1);
            for (int x = 0; x < 2; ++x) mbar_init(smem_u32(&bars.slot_done[st][x]), 1);
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
    const int kvb = a.kv_batched ? b : 0;
    // TMA coordinates of query tile x's box and of key block j's box
    auto load_q = [&](uint32_t dst, int x, int bx, uint32_t bar) {
        if constexpr (TILED)
            tc::tma_load_5d(dst, &tm_q, bx * 64, h, tx * 16, ty * 16 + x * 8, b, bar);
        else
            tc::tma_load_4d(dst, &tm_q, bx * 64, h, (qblk * 2 + x) * kBM, b, bar);
    };
    auto load_kv = [&](uint32_t dst, const CUtensorMap* m, int j, int bx, uint32_t bar) {
        if constexpr (GEO == kGeoWindow) {
            const int t = j >> 2, ky = wy0 + t / wcols, kx = wx0 + t % wcols;
            tc::tma_load_5d(dst, m, bx * 64, h, kx * 16, ky * 16 + (j & 3) * 4, kvb, bar);
        } else if constexpr (GEO == kGeoList) {
            int tile = __ldg(klist + (j >> 2));
            if (tile < 0 || tile >= a.tiles_h * a.tiles_w) {
                atomicOr(&g_flash_err, kDevErrBadIndex);
                tile = tile < 0 ? 0 : a.tiles_h * a.tiles_w - 1;
            }
            const int ky = tile / a.tiles_w, kx = tile - ky * a.tiles_w;
            tc::tma_load_5d(dst, m, bx * 64, h, kx * 16, ky * 16 + (j & 3) * 4, kvb, bar);
        } else {
            tc::tma_load_4d(dst, m, bx * 64, h, j * kBN, kvb, bar);
        }
    };

    if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int x = 0; x < ntiles; ++x) {
                mbar_arrive_expect_tx(smem_u32(&bars.q_full[x]), kQTile);
                for (int bx = 0; bx < NB; ++bx)
                    load_q(q_s + x * kQTile + bx * kQBox, x, bx, smem_u32(&bars.q_full[x]));
            }
            const int n01 = nkv < 2 ? nkv : 2;
            if (n01 > 0) {
                mbar_arrive_expect_tx(smem_u32(&bars.k01_full), n01 * kKVTile);
                for (int j = 0; j < n01; ++j)
                    for (int bx = 0; bx < NB; ++bx)
                        load_kv(k01_s + j * kKVTile + bx * kKVBox, &tm_k, j, bx, smem_u32(&bars.k01_full));
            }
            int nslot = 0;  // slot loads issued
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j % NST;
                for (int x = 0; x < ntiles && ok && j >= NST; ++x)
                    ok = wait_bar(&bars, &bars.slot_done[st][x], ((j / NST) - 1) & 1);
                if (!ok) break;
                const bool with_k = j + 2 < nkv;
                const uint32_t bar = smem_u32(&bars.slot_full[st]);
                mbar_arrive_expect_tx(bar, with_k ? 2 * kKVTile : kKVTile);
                for (int bx = 0; bx < NB; ++bx) load_kv(v_s + st * kKVTile + bx * kKVBox, &tm_v, j, bx, bar);
                if (with_k)
                    for (int bx = 0; bx < NB; ++bx)
                        load_kv(k_s + st * kKVTile + bx * kKVBox, &tm_k, j + 2, bx, bar);
                nslot = j + 1;
            }
            if (!ok || *(volatile int*)&bars.abort) {
                // drain: let this CTA's loads land before it exits (bounded)
                for (int st = 0; st < NST; ++st) {
                    const int uses = (nslot - st + NST - 1) / NST;  // loads issued into slot st
                    if (uses > 0)
                        mbar_wait_bounded(smem_u32(&bars.slot_full[st]), (uses - 1) & 1, &g_flash_err);
                }
                if (n01 > 0) mbar_wait_bounded(smem_u32(&bars.k01_full), 0, &g_flash_err);
                for (int x = 0; x < ntiles; ++x)
                    mbar_wait_bounded(smem_u32(&bars.q_full[x]), 0, &g_flash_err);
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------ MMA issuers
        // One thread per query tile: a wait of one issuer overlaps the other's
        // MMA issue, so the tensor core queue stays fed.
        const int x = warp - 9;
        if (lane == 0 && x < ntiles) {
            constexpr uint32_t idesc_s = tc::idesc_bf16(kBM, kBN, 0, 0);
            constexpr uint32_t idesc_o = tc::idesc_bf16(kBM, NO, 0, 1);
            // Descriptors are built once; a K step, tile or slot only moves the
            // start address (bits 0..13, in 16-byte units), which stays below
            // 2^14 because shared memory is smaller than 256 KB.
            const uint64_t dq = tc::smem_desc(q_s + x * kQTile, 16, 1024, 2);
            const uint64_t dk01 = tc::smem_desc(k01_s, 16, 1024, 2);
            const uint64_t dk = tc::smem_desc(k_s, 16, 1024, 2);
            const uint64_t dv = tc::smem_desc(v_s, kKVBox, 1024, 2);
            auto issue_s = [&](uint64_t kdesc, int j) {  // S_X(j) into buffer j & 1
                const uint32_t d = tmem + x * 128 + (j & 1) * 64;
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint32_t offa = (ks >> 2) * (kQBox >> 4) + (ks & 3) * 2;
                    const uint32_t offb = (ks >> 2) * (kKVBox >> 4) + (ks & 3) * 2;
                    tc::mma_ss(d, dq + offa, kdesc + offb, idesc_s, ks > 0 ? 1u : 0u);
                }
            };
            bool ok = wait_bar(&bars, &bars.q_full[x], 0);
            if (ok && nkv > 0) ok = wait_bar(&bars, &bars.k01_full, 0);
            if (ok && nkv > 0) {
                tc::fence_after_sync();
                issue_s(dk01, 0);
                if (nkv > 1) issue_s(dk01 + (kKVTile >> 4), 1);
                tc::commit(smem_u32(&bars.s01_done[x]));
            }
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j % NST;
                ok = wait_bar(&bars, ONES ? &bars.slot_ready[st] : &bars.slot_full[st], (j / NST) & 1);
                if (ok) ok = wait_bar(&bars, &bars.p_full[x][j & 1], (j >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                // O_X += P_X(j) V_j
                const uint64_t vdesc = dv + (uint64_t)((st * kKVTile) >> 4);
                const uint32_t d = tmem + 256 + x * 128, pa = tmem + x * 128 + (j & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_ts(d, pa + kk * 8, vdesc + kk * 128, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                // S_X(j+2) reuses the buffer PV_X(j) has just been queued on
                if (j + 2 < nkv) issue_s(dk + (uint64_t)((st * kKVTile) >> 4), j + 2);
                tc::commit(smem_u32(&bars.slot_done[st][x]));
                if (j + 1 == nkv) tc::commit(smem_u32(&bars.o_done[x]));
            }
            // all MMAs this thread issued complete before TMEM is released
            tc::commit(smem_u32(&bars.mma_done[x]));
            mbar_wait_bounded(smem_u32(&bars.mma_done[x]), 0, &g_flash_err);
        }
    } else if (warp == 11) {
        // ------------------------------------------------ V-ones warp
        if constexpr (ONES) {
            const uint32_t col = (uint32_t)a.d;
            const uint32_t ch = (col & 63) >> 3, e = col & 7;
            bool ok = true;
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j % NST;
                ok = __all_sync(0xffffffffu, wait_bar(&bars, &bars.slot_full[st], (j / NST) & 1));
                if (!ok) break;
                unsigned char* vbox = gen_base + (v_s - sbase) + st * kKVTile + (col >> 6) * kKVBox;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int r = lane + 32 * h2;
                    *reinterpret_cast<uint16_t*>(vbox + r * 128 + ((ch ^ (r & 7)) << 4) + e * 2) = 0x3F80u;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars.slot_ready[st]));
            }
        }
    } else {
        // ------------------------------------------------ softmax warpgroups
        const int x = warp >> 2;  // tile
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t o_col = 256 + x * 128;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = x < ntiles;
        if (ok && x == 1 && nkv > 0) ok = wait_bar(&bars, &bars.b_go, 0);
        for (int j = 0; j < nkv && ok; ++j) {
            const uint32_t s_col = x * 128 + (j & 1) * 64;
            // S_X(j) was issued with step j-2's slot (or in the prologue)
            if (j < 2)
                ok = wait_bar(&bars, &bars.s01_done[x], 0);
            else
                ok = wait_bar(&bars, &bars.slot_done[(j - 2) % NST][x], ((j - 2) / NST) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            const int valid = TILED ? kBN : a.Lk - j * kBN;  // keys of this tile that exist
            // the row's 64 scores fit in registers: one TMEM read
            float sv[kBN];
            {
                uint32_t r0[32], r1[32];
                tc::ld_32col(lane_addr + s_col + 0, r0);
                tc::ld_32col(lane_addr + s_col + 32, r1);
                tc::wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    sv[i] = __uint_as_float(r0[i]);
                    sv[32 + i] = __uint_as_float(r1[i]);
                }
            }
            if (valid < kBN) {
#pragma unroll
                for (int i = 0; i < kBN; ++i)
                    if (i >= valid) sv[i] = -INFINITY;
            }
            // row max of the raw scores (scale > 0 commutes with max): eight
            // independent 3-input max chains over 8 scores each
            float mt;
            {
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float m = tc::max3f(sv[k], sv[k + 8], sv[k + 16]);
                    m = tc::max3f(m, sv[k + 24], sv[k + 32]);
                    m = tc::max3f(m, sv[k + 40], sv[k + 48]);
                    mx[k] = fmaxf(m, sv[k + 56]);
                }
                mt = tc::max3f(tc::max3f(mx[0], mx[1], mx[2]), tc::max3f(mx[3], mx[4], mx[5]),
                               fmaxf(mx[6], mx[7])) * a.scale_log2;
            }
            if (j == 0) {
                m_ref = mt;
                if (x == 0) mbar_arrive(smem_u32(&bars.b_go));
            } else {
                const bool need = mt > m_ref + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    // O_X must hold exactly PV_X(0..j-1): PV_X(j-1) retired
                    // once step j-1's slot is done
                    ok = wait_bar(&bars, &bars.slot_done[(j - 1) % NST][x], ((j - 1) / NST) & 1);
                    if (!ok) break;
                    tc::fence_after_sync();
                    const float m_new = need ? mt : m_ref;
                    const float f = ex2(m_ref - m_new);
#pragma unroll
                    for (int c = 0; c < NO / 16; ++c) {
                        uint32_t r[16];
                        tc::ld_16col(lane_addr + o_col + c * 16, r);
                        tc::wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                        tc::st_16col(lane_addr + o_col + c * 16, r);
                    }
                    if constexpr (!ONES) l *= f;
                    m_ref = m_new;
                }
            }
            // exponentiate, sum and write P back as bf16 over S's columns
            const tc::f32x2 scale2 = tc::pack2(a.scale_log2, a.scale_log2);
            const tc::f32x2 negm2 = tc::pack2(-m_ref, -m_ref);
            tc::f32x2 acc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = tc::pack2(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t r[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int idx = c * 32 + 2 * i;
                    const tc::f32x2 t = tc::fma2(tc::pack2(sv[idx], sv[idx + 1]), scale2, negm2);
                    float t0, t1, p0, p1;
                    tc::unpack2(t, t0, t1);
                    if (((idx >> 1) & 7) < kPolyPairsOf8) {
                        tc::exp2_poly2(t0, t1, p0, p1);
                    } else {
                        p0 = ex2(t0);
                        p1 = ex2(t1);
                    }
                    if constexpr (!ONES) acc[i & 3] = tc::add2(acc[i & 3], tc::pack2(p0, p1));
                    r[i] = pack_bf16x2(p0, p1);
                }
                tc::st_16col(lane_addr + s_col + c * 16, r);
            }
            if constexpr (!ONES) {
                float a0, a1;
                tc::unpack2(tc::add2(tc::add2(acc[0], acc[1]), tc::add2(acc[2], acc[3])), a0, a1);
                l += a0 + a1;
            }
            tc::wait_st();
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.p_full[x][j & 1]));
        }
        // ---------------- epilogue: O / l -> bf16 -> swizzled smem -> TMA store
        if (ok && nkv > 0) ok = wait_bar(&bars, &bars.o_done[x], 0);
        if (ok) {
            tc::fence_after_sync();
            if constexpr (ONES) {  // O's column d: the row sum of P
                uint32_t lbits;
                tc::ld_1col(lane_addr + o_col + (uint32_t)a.d, lbits);
                tc::wait_ld();
                l = __uint_as_float(lbits);
            }
            const float inv = 1.f / l;
            unsigned char* stage = gen_base + x * kQTile;  // this tile's Q buffer (all S MMAs done)
#pragma unroll
            for (int c = 0; c < NO / 16; ++c) {
                uint32_t r[16];
                tc::ld_16col(lane_addr + o_col + c * 16, r);
                tc::wait_ld();
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                const int col = c * 16;
                const int bx = col >> 6;
                const int ch = (col & 63) >> 3;
                unsigned char* rowp = stage + bx * kQBox + row * 128;
                *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4*>(rowp + (((ch + 1) ^ (row & 7)) << 4)) =
                    make_uint4(w[4], w[5], w[6], w[7]);
            }
            fence_proxy_async_smem();
        }
        tc::named_bar_sync(1 + x, 128);
        if (ok && row == 0) {
            for (int bx = 0; bx < NB; ++bx) {
                if constexpr (TILED)
                    tc::tma_store_5d(&tm_o, q_s + x * kQTile + bx * kQBox, bx * 64, h, tx * 16, ty * 16 + x * 8, b);
                else
                    tc::tma_store_4d(&tm_o, q_s + x * kQTile + bx * kQBox, bx * 64, h, (qblk * 2 + x) * kBM, b);
            }
            bulk_commit();
            bulk_wait<0>();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D map over a [batches][rows][heads][d] bf16 view (row stride C elements):
// dims (d, heads, rows, batches), box (64, 1, box_rows, 1), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int d, int heads, long long rows, long long batches,
              long long row_stride_elems, long long batch_stride_elems, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows, (cuuint64_t)batches};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)row_stride_elems * 2,
                             (cuuint64_t)(batch_stride_elems > 0 ? batch_stride_elems : rows * row_stride_elems) * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 5-D map over the [frames][H][W][heads][d] bf16 spatial view: dims (d,
// heads, W, H, frames), box (64, 1, 16, box_h, 1) -- 16 * box_h tokens of a
// 16-wide tile, row-major, one 128-byte swizzled row each.
bool make_map_grid(CUtensorMap* m, const void* base, int d, int heads, int H, int W, int frames, int box_h) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t C = (cuuint64_t)heads * d;
    cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)frames};
    cuuint64_t strides[4] = {(cuuint64_t)d * 2, C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
    cuuint32_t box[5] = {64, 1, 16, (cuuint32_t)box_h, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int KSTEPS, bool ONES, int GEO>
cudaError_t launch_ks1(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                       const FlashTcArgs& a, dim3 grid, cudaStream_t s) {
    constexpr int NB = (KSTEPS + 3) / 4;
    constexpr int NST = NB == 1 ? 6 : 4;  // ring slots of (V_j, K_{j+2})
    const size_t smem = (size_t)NB * (2 * kQBox + (2 + 2 * NST) * kKVBox) + 1024;
    const size_t smem_req = smem < 120 * 1024 ? 120 * 1024 : smem;  // one CTA per SM (TMEM: 512 columns)
    cudaError_t e = cudaFuncSetAttribute(flash_tc_kernel<KSTEPS, NST, ONES, GEO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_req);
    if (e != cudaSuccess) return e;
    flash_tc_kernel<KSTEPS, NST, ONES, GEO><<<grid, kThreads, smem_req, s>>>(mq, mk, mv, mo, a);
    return cudaGetLastError();
}
template <int KSTEPS, int GEO>
cudaError_t launch_ks(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                      const FlashTcArgs& a, dim3 grid, cudaStream_t s) {
    // a padding column inside the PV product carries the row sums when d % 16 != 0
    if (PAB_FLASH_ONES && a.d % 16 != 0) return launch_ks1<KSTEPS, true, GEO>(mq, mk, mv, mo, a, grid, s);
    return launch_ks1<KSTEPS, false, GEO>(mq, mk, mv, mo, a, grid, s);
}
template <int GEO>
cudaError_t launch_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                     const FlashTcArgs& a, dim3 grid, cudaStream_t s) {
    switch ((a.d + 15) / 16) {
        case 1: return launch_ks<1, GEO>(mq, mk, mv, mo, a, grid, s);
        case 2: return launch_ks<2, GEO>(mq, mk, mv, mo, a, grid, s);
        case 3: return launch_ks<3, GEO>(mq, mk, mv, mo, a, grid, s);
        case 4: return launch_ks<4, GEO>(mq, mk, mv, mo, a, grid, s);
        case 5: return launch_ks<5, GEO>(mq, mk, mv, mo, a, grid, s);
        case 6: return launch_ks<6, GEO>(mq, mk, mv, mo, a, grid, s);
        case 7: return launch_ks<7, GEO>(mq, mk, mv, mo, a, grid, s);
        case 8: return launch_ks<8, GEO>(mq, mk, mv, mo, a, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_flash(const void* q, const void* k, const void* v, void* out, int batches, long long Lq,
                         int Lk, int heads, int d, long long q_bstride, long long kv_bstride, cudaStream_t s) {
    if (Lq == 0 || batches == 0) return cudaSuccess;
    const long long C = (long long)heads * d;
    const long long qblocks = (Lq + 2 * kBM - 1) / (2 * kBM);
    if (qblocks > 0x7fffffffLL || batches > 65535 || heads > 65535 || Lq > 0x7fffffffLL)
        return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    const long long kv_batches = kv_bstride > 0 ? batches : 1;
    if (!make_map(&mq, q, d, heads, Lq, batches, C, q_bstride, kBM) ||
        !make_map(&mk, k, d, heads, Lk, kv_batches, C, kv_bstride, kBN) ||
        !make_map(&mv, v, d, heads, Lk, kv_batches, C, kv_bstride, kBN) ||
        !make_map(&mo, out, d, heads, Lq, batches, C, q_bstride, kBM))
        return cudaErrorInvalidValue;
    FlashTcArgs a;
    a.Lq = (int)Lq;
    a.Lk = Lk;
    a.kv_batched = kv_bstride > 0 ? 1 : 0;
    a.d = d;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    a.tiles_h = a.tiles_w = a.reach_h = a.reach_w = 0;
    a.kv_list = nullptr;
    a.kv_count = 0;
    dim3 grid((unsigned)qblocks, (unsigned)heads, (unsigned)batches);
    return launch_d<kGeoFull>(mq, mk, mv, mo, a, grid, s);
}

cudaError_t launch_flash_sta(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                             int heads, int d, int win_h, int win_w, cudaStream_t s) {
    if (frames == 0 || H == 0 || W == 0) return cudaSuccess;
    if (H % kStaTile || W % kStaTile || win_h % kStaTile || win_w % kStaTile || win_h <= 0 || win_w <= 0 ||
        (win_h / kStaTile) % 2 == 0 || (win_w / kStaTile) % 2 == 0)
        return cudaErrorInvalidValue;
    const long long tiles = (long long)(H / kStaTile) * (W / kStaTile);
    if (tiles > 0x7fffffffLL || frames > 65535 || heads > 65535) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map_grid(&mq, q, d, heads, H, W, frames, 8) || !make_map_grid(&mk, k, d, heads, H, W, frames, 4) ||
        !make_map_grid(&mv, v, d, heads, H, W, frames, 4) || !make_map_grid(&mo, out, d, heads, H, W, frames, 8))
        return cudaErrorInvalidValue;
    FlashTcArgs a;
    a.Lq = H * W;
    a.Lk = H * W;
    a.kv_batched = 1;
    a.d = d;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    a.tiles_h = H / kStaTile;
    a.tiles_w = W / kStaTile;
    a.reach_h = (win_h / kStaTile - 1) / 2;
    a.reach_w = (win_w / kStaTile - 1) / 2;
    a.kv_list = nullptr;
    a.kv_count = 0;
    dim3 grid((unsigned)tiles, (unsigned)heads, (unsigned)frames);
    return launch_d<kGeoWindow>(mq, mk, mv, mo, a, grid, s);
}

cudaError_t launch_flash_tile_list(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                                   int heads, int d, const int* kv_list, int kv_count, cudaStream_t s) {
    if (frames == 0 || H == 0 || W == 0) return cudaSuccess;
    if (H % kStaTile || W % kStaTile || kv_count < 1 || !kv_list) return cudaErrorInvalidValue;
    const long long tiles = (long long)(H / kStaTile) * (W / kStaTile);
    if (kv_count > tiles || tiles > 0x7fffffffLL || frames > 65535 || heads > 65535) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map_grid(&mq, q, d, heads, H, W, frames, 8) || !make_map_grid(&mk, k, d, heads, H, W, frames, 4) ||
        !make_map_grid(&mv, v, d, heads, H, W, frames, 4) || !make_map_grid(&mo, out, d, heads, H, W, frames, 8))
        return cudaErrorInvalidValue;
    FlashTcArgs a;
    a.Lq = H * W;
    a.Lk = H * W;
    a.kv_batched = 1;
    a.d = d;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    a.tiles_h = H / kStaTile;
    a.tiles_w = W / kStaTile;
    a.reach_h = a.reach_w = 0;
    a.kv_list = kv_list;
    a.kv_count = kv_count;
    dim3 grid((unsigned)tiles, (unsigned)heads, (unsigned)frames);
    return launch_d<kGeoList>(mq, mk, mv, mo, a, grid, s);
}

unsigned int flash_device_errors(bool clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_flash_err, sizeof(v)) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_flash_err, &z, sizeof(z));
    }
    return v;
}

}  // namespace pab

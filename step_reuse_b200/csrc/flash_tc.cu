// flash_tc.cu -- flash (online-softmax) attention on the 5th-generation
// tensor cores (tcgen05 + TMEM) for the long-sequence PAB kinds: spatial
// attention (the tokens of one frame, L = H*W) and cross attention (video
// tokens against one shared set of text keys/values) -- PAB report,
// "Implementation".  softmax(Q K^T / sqrt(d)) V per (batch, head).
//
// Persistent CTAs, one per SM, walk a static list of work items: CTA c takes
// items c, c + gridDim.x, ...  An item is 256 query rows of one (batch, head)
// as two 128-row tiles A and B that share every K/V tile (for the tile
// geometries, one 16 x 16 query tile of a frame: A its upper 8 rows, B the
// lower 8).  Consecutive items share (batch, head), so the CTAs running at
// one time read the same K/V from L2.
// The 64-key K/V tiles of all of a CTA's items form ONE sequence of global
// steps g = 0, 1, ...; use s of the ring carries K_s and V_{s-2} in slot
// s mod NST.  Roles:
//   producer warp         TMA producer (one thread): per item the two Q
//                          tiles (Q is double-buffered by item parity), per
//                          ring use one slot;
//   two MMA warps         MMA issuers, one per query tile X, warp-uniform
//                          (one elected lane issues): once P_X(g) is written,
//                          O_X += P_X(g) V_g (TS form: P from TMEM, V from
//                          shared memory) and S_X(g+2) = Q_X K_{g+2}^T (SS
//                          form, fp32 in TMEM) into the S buffer that P_X(g)
//                          is read from (the tensor core executes in order),
//                          then one commit for the slot.  S_X(g+2) may belong
//                          to the next item, so the next item's first two
//                          score tiles are ready when the softmax finishes the
//                          current item's epilogue;
//   V-ones warp           (d % 16 != 0): sets V's padding column
//                          d to 1 as each V tile lands, so O's column d
//                          accumulates the row sums of P with the same bf16 P
//                          as the numerator (the softmax keeps no running sum);
//   softmax warps         per tile X one warp per TMEM lane quarter (for
//                          head dims up to 16 * PAB_FLASH_SPLIT_KSTEPS two,
//                          taking the 64-key steps in turns): the thread of
//                          query row i (TMEM lane i) reads its scores of S
//                          with tcgen05.ld, keeps the running max,
//                          writes P as bf16 over S's columns and rescales O in
//                          TMEM only when the running max grew by more than
//                          2^8 (the final O / l is exact either way);
//                          exponentials 3/4 on the MUFU ex2 unit, 1/4 on the
//                          FMA pipes (tc::exp2_poly2).  Then the item's
//                          epilogue: O / l -> bf16 -> the item's Q buffer (no
//                          score product reads it any more) -> TMA store.  The
//                          store's read of shared memory is waited for during
//                          the next item's first step, which then frees the
//                          buffer for the Q of the item after next.
// Rescaling O_X at step g needs PV_X(g-1) retired: the softmax then waits for
// the commit of ring use g+1 (PV_X(g-1), S_X(g+1)).
//
// TMEM columns: S_A0 [0,64), S_A1 [64,128), S_B0 [128,192), S_B1 [192,256),
//               O_A [256,256+NO), O_B [384,384+NO).
// Operand layouts (TMA-written):
//   Q, K: [rows][64 cols] boxes (128 rows for Q, 64 for K; 128-byte swizzle),
//         K-major (d contiguous), plus for head dims whose 16-column K steps
//         leave one or two over a [rows][16 or 32 cols] tail box (32- or
//         64-byte swizzle); a 16-wide K step advances the descriptor start by
//         32 bytes inside a box.  The output is staged in Q's layout.
//   V:    [64 rows][64 cols] boxes read MN-major (B of the PV product has
//         N = d contiguous); a 16-key K step advances by 16 rows = 2048 bytes,
//         the next 64 columns of d are one box (8 KB) further (LBO).
// Columns past d read as zero (the tensor map's innermost extent is d) and
// are not stored; keys past Lk are masked to -inf;
// query rows past Lq are zero-filled on load and clipped by the TMA store; a
// B tile that lies wholly past Lq issues no MMAs, computes no softmax and
// stores nothing (its barriers still complete, so every role counts the
// same steps).
// Every wait on an mbarrier is bounded; on time-out the CTA raises the error
// word, lets its own asynchronous copies and MMAs drain, frees TMEM and exits.
#include <cuda.h>

#include "kernels.h"
#include "tc.cuh"

namespace pab {
namespace {

constexpr int kBM = 128;          // query rows per tile (two tiles per item)
constexpr int kStaTile = 16;      // sliding tile attention: 16 x 16-token tiles (the item's 256 queries)
constexpr int kBN = 64;           // keys per K/V tile
constexpr int kQBox = 128 * 128;  // bytes of one [128 rows][64 cols] bf16 box (Q, O)
constexpr int kKVBox = 64 * 128;  // bytes of one [64 rows][64 cols] bf16 box (K, V)
constexpr uint32_t kTmemCols = 512;
// SPLIT 2 register split (setmaxnreg): softmax warpgroups / the other warpgroup
constexpr int kSplitRegsSoftmax = 104;
constexpr int kSplitRegsOther = 64;
constexpr float kRescaleLog2 = 8.0f;
// Exponentials: of every 8 consecutive pairs of a row's scores, this many go
// to tc::exp2_poly2 on the FMA pipes and the rest to the MUFU ex2 unit,
// which alone would bound the softmax (16 results per clock per SM); 2 of 8
// measured fastest (0, 2, 3, 4 and 5 of 8 timed at d = 64 and 72).
#ifndef PAB_POLY_PAIRS_OF_8
#define PAB_POLY_PAIRS_OF_8 2
#endif
constexpr int kPolyPairsOf8 = PAB_POLY_PAIRS_OF_8;
#ifndef PAB_FLASH_ONES
#define PAB_FLASH_ONES 1
#endif

__device__ unsigned int g_flash_err = 0;

struct FlashTcArgs {
    int Lq;            // query rows per batch
    int Lk;            // keys per batch (>= 1)
    int kv_batched;    // 1: K/V have a batch coordinate (spatial); 0: shared (cross)
    int d;             // head dim
    float scale_log2;  // log2(e) / sqrt(d)
    int heads;
    int per_bh;        // items per (batch, head): 256-row query blocks, or query tiles
    int items;         // batches * heads * per_bh
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

// One work item, decoded from its index.
struct Item {
    int b, h, qblk;        // batch, head, query block (full) or query tile index (tiled)
    int ty, tx;            // tile geometries: the query tile's position
    int wy0, wx0, wcols;   // window geometry: first window tile and window width in tiles
    int nkv;               // 64-key steps (>= 1)
    bool has_b;            // tile B holds query rows
    const int* klist;      // list geometry: this query tile's key tiles
};

template <int GEO>
PAB_DEV Item decode_item(const FlashTcArgs& a, int it) {
    Item m;
    const int bh = it / a.per_bh;
    m.qblk = it - bh * a.per_bh;
    m.h = bh % a.heads;
    m.b = bh / a.heads;
    m.ty = m.tx = m.wy0 = m.wx0 = 0;
    m.wcols = 1;
    m.klist = nullptr;
    if constexpr (GEO != kGeoFull) {
        m.ty = m.qblk / a.tiles_w;
        m.tx = m.qblk - m.ty * a.tiles_w;
        m.has_b = true;
    } else {
        m.has_b = m.qblk * 2 * kBM + kBM < a.Lq;
    }
    if constexpr (GEO == kGeoWindow) {
        m.wy0 = max(m.ty - a.reach_h, 0);
        m.wx0 = max(m.tx - a.reach_w, 0);
        const int wy1 = min(m.ty + a.reach_h + 1, a.tiles_h), wx1 = min(m.tx + a.reach_w + 1, a.tiles_w);
        m.wcols = wx1 - m.wx0;
        m.nkv = (wy1 - m.wy0) * m.wcols * 4;
    } else if constexpr (GEO == kGeoList) {
        m.klist = a.kv_list + (long long)it * a.kv_count;  // items are ordered (batch, head, tile)
        m.nkv = a.kv_count * 4;
    } else {
        m.nkv = (a.Lk + kBN - 1) / kBN;
    }
    return m;
}

// Position in the CTA's sequence of (item, key step).
template <int GEO>
struct Cursor {
    int it;  // item index (>= a.items once the CTA's items are exhausted)
    int k;   // the item's position among this CTA's items
    int j;   // key step within the item
    Item m;
    PAB_DEV void start(const FlashTcArgs& a) {
        it = blockIdx.x;
        k = j = 0;
        if (it < a.items) m = decode_item<GEO>(a, it);
    }
    PAB_DEV bool valid(const FlashTcArgs& a) const { return it < a.items; }
    PAB_DEV void next_item(const FlashTcArgs& a) {
        j = 0;
        ++k;
        it += gridDim.x;
        if (it < a.items) m = decode_item<GEO>(a, it);
    }
    PAB_DEV void next(const FlashTcArgs& a) {
        if (++j == m.nkv) next_item(a);
    }
};

// Every barrier completes exactly once per use, so each role derives its
// wait parities from counters it keeps anyway:
//   q_full[b][X], q_free[b][X]  once per item with Q buffer b (item k uses k & 1)
//   slot_full/ready/done[s]     once per ring use s (use u of slot s: u / NST)
//   p_full[X][b]                once per global step g with g & 1 == b
//   o_done[X], stage[X]         once per item
//   mref_full[X][q][b]          once per global step g with g & 1 == b (SPLIT 2)
//   xsum_done[X][q]             once per item with work for tile X (SPLIT 2 without the ones column)
struct Bars {
    unsigned long long q_full[2][2];              // [Q buffer][tile]: Q landed
    unsigned long long q_free[2][2];              // [Q buffer][tile]: the output staged there was stored
    unsigned long long b_go;                      // tile A's first row maximum is done
    unsigned long long slot_full[kMaxStages];     // K_s, V_{s-2} landed
    unsigned long long slot_ready[kMaxStages];    // ... and (ONES) V's column d set to 1
    unsigned long long slot_done[kMaxStages][2];  // [slot][tile]: PV_X(s-2), S_X(s) retired
    unsigned long long p_full[2][2];              // [tile][S buffer]: P written
    unsigned long long o_done[2];                 // [tile]: the item's last PV retired
    unsigned long long stage[2];                  // [tile]: the item's output is staged
    unsigned long long mref_full[2][4][2];        // [tile][lane quarter][step parity]: the step's maxima written
    unsigned long long xsum_done[2][4];           // [tile][lane quarter]: both warps' row sums written
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
// Tile geometries (GEO != kGeoFull): an item's 256 queries are one 16 x 16
// tile of the frame (tile A its upper 8 rows, tile B the lower 8, each read
// as a [8][16]-token TMA box of the [H][W] grid), and the key loop runs over
// 16 x 16 key tiles, each as four [4][16]-token blocks of 64 keys: the tiles
// of the window around the query tile, clipped at the frame edge (window),
// or the tiles listed for it (list; an index outside the frame raises the
// error word and is clamped).  Every block is whole, so nothing is masked.
// Operand boxes along d.  Q, K and the staged output of one tile are NB0 full
// 64-column boxes (128-byte swizzle) plus, when the 16-column K steps leave
// one or two over, one narrow tail box of 16 or 32 columns (32- or 64-byte
// swizzle), so a head dim such as 72 (five K steps) holds 80 columns in
// shared memory instead of 128.  V stays in full boxes: the PV product's
// N = 16 * KSTEPS columns (the padding column d included) are read MN-major
// across 64-column atoms.
template <int KSTEPS>
struct DLayout {
    static constexpr int TK0 = KSTEPS % 4;
    static constexpr int NB0 = KSTEPS / 4 + (TK0 == 3 ? 1 : 0);  // full 64-column boxes
    static constexpr int TK = TK0 == 3 ? 0 : TK0;                 // K steps in the tail box
    static constexpr int TB = TK * 32;                            // tail box row bytes (0, 32, 64)
    static constexpr int NBV = (KSTEPS + 3) / 4;                  // V boxes
    static constexpr uint32_t QTile = NB0 * kQBox + 128 * TB;
    static constexpr uint32_t KTile = NB0 * kKVBox + 64 * TB;
    static constexpr uint32_t VTile = NBV * kKVBox;
    static constexpr uint32_t tail_swizzle = TB == 32 ? 6u : 4u;  // descriptor layout: 32- / 64-byte swizzle
    // 16-byte unit u of row r of the tail box, after the TMA swizzle (address
    // bits 7.. XORed into the unit index)
    PAB_DEV static uint32_t tail_unit(int r, int u) {
        return TB == 32 ? (uint32_t)(u ^ ((r >> 2) & 1)) : (uint32_t)(u ^ ((r >> 1) & 3));
    }
};

// Softmax split: SPLIT = 2 gives every query row two warps -- the two warps
// of one TMEM lane quarter on one sub-partition -- that take the row's 64-key
// steps in turns (warp par takes the global steps g with g & 1 == par, i.e.
// the S buffer par), so four softmax warps share each sub-partition and the
// turns keep them out of phase: one warp's TMEM load and row maximum run
// while the other exponentiates.  The row's running maximum passes from step
// to step through shared memory behind an mbarrier per (tile, lane quarter,
// step parity) (a bounded wait, like every wait here), published as soon as
// the step has decided it, before its exponentials; the rescaling of O then
// follows the one sequence of maxima, and without the ones column each warp
// keeps its own row sum in the units of the maximum of its latest step
// (brought to the final one in the epilogue).
#ifndef PAB_FLASH_SPLIT_KSTEPS
#define PAB_FLASH_SPLIT_KSTEPS 0  // head dims up to 16 * this many columns split their rows
#endif
template <int KSTEPS>
constexpr int flash_split() { return KSTEPS <= PAB_FLASH_SPLIT_KSTEPS ? 2 : 1; }
template <int KSTEPS>
constexpr int flash_threads() { return (8 * flash_split<KSTEPS>() + 4) * 32; }

template <int KSTEPS, int NST, bool ONES, int GEO>
__global__ void __launch_bounds__(flash_threads<KSTEPS>(), 1)
    flash_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qt,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kt,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_ot, FlashTcArgs a) {
    static_assert(NST >= 3 && NST <= kMaxStages, "ring depth");
    using DL = DLayout<KSTEPS>;
    constexpr int SPLIT = flash_split<KSTEPS>();
    constexpr int NSW = 8 * SPLIT;           // softmax warps
    constexpr int W_PROD = NSW, W_MMA = NSW + 1, W_ONES = NSW + 3;
    constexpr int NO = KSTEPS * 16;          // N of the PV product (d rounded up to 16)
    constexpr int NC = NO / 16;              // 16-column chunks of O
    constexpr bool TILED = GEO != kGeoFull;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ Bars bars;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const uint32_t q_s = sbase;                      // [2 buffers][2 tiles] Q tiles
    const uint32_t k_s = q_s + 4 * DL::QTile;        // [NST] K_s
    const uint32_t v_s = k_s + NST * DL::KTile;      // [NST] V_{s-2}
    const uint32_t x_s = v_s + NST * DL::VTile;      // SPLIT 2: row maxima and sums
    unsigned char* gen_base = smem_raw + (sbase - smem_u32(smem_raw));
    // [tile][step parity][row] maxima, [item parity][tile][sum of warp 0, 1;
    // maximum of warp 0, 1][row] row sums
    float* mref = reinterpret_cast<float*>(gen_base + (x_s - sbase));
    float* xsum = mref + 2 * 2 * 128;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == W_PROD * 32) {
        for (int x = 0; x < 2; ++x) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(smem_u32(&bars.q_full[u][x]), 1);
                mbar_init(smem_u32(&bars.q_free[u][x]), 1);
                mbar_init(smem_u32(&bars.p_full[x][u]), 128);
            }
            mbar_init(smem_u32(&bars.o_done[x]), 1);
            mbar_init(smem_u32(&bars.mma_done[x]), 1);
        }
        mbar_init(smem_u32(&bars.b_go), 128);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.stage[x]), 128 * SPLIT);
            for (int q = 0; q < 4; ++q) {
                mbar_init(smem_u32(&bars.xsum_done[x][q]), 64);
                for (int u = 0; u < 2; ++u) mbar_init(smem_u32(&bars.mref_full[x][q][u]), 32);
            }
        }
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
        if constexpr (DL::TK > 0) {
            tc::prefetch_tmap(&tm_qt);
            tc::prefetch_tmap(&tm_kt);
            tc::prefetch_tmap(&tm_ot);
        }
    }
    if (warp == W_MMA) {
        tc::tmem_alloc(smem_u32(&bars.tmem_base), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = bars.tmem_base;
    // SPLIT 2: 640 threads launch with 96 registers each; the softmax
    // warpgroups take 104, the producer / MMA / ones warpgroup keeps 64
    // (4 x 128 x 104 + 128 x 64 = 640 x 96), each at the top of its role
    auto regs_other = [&]() {
        if constexpr (SPLIT == 2) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kSplitRegsOther) : "memory");
    };

    // TMA coordinates of query tile x's box at column c0 and of key block j's
    // box at column c0
    auto load_q = [&](uint32_t dst, const CUtensorMap* tm, const Item& m, int x, int c0, uint32_t bar) {
        if constexpr (TILED)
            tc::tma_load_5d(dst, tm, c0, m.h, m.tx * 16, m.ty * 16 + x * 8, m.b, bar);
        else
            tc::tma_load_4d(dst, tm, c0, m.h, (m.qblk * 2 + x) * kBM, m.b, bar);
    };
    auto load_kv = [&](uint32_t dst, const CUtensorMap* tm, const Item& m, int j, int c0, uint32_t bar) {
        const int kvb = a.kv_batched ? m.b : 0;
        if constexpr (GEO == kGeoWindow) {
            const int t = j >> 2, ky = m.wy0 + t / m.wcols, kx = m.wx0 + t % m.wcols;
            tc::tma_load_5d(dst, tm, c0, m.h, kx * 16, ky * 16 + (j & 3) * 4, kvb, bar);
        } else if constexpr (GEO == kGeoList) {
            int tile = __ldg(m.klist + (j >> 2));
            if (tile < 0 || tile >= a.tiles_h * a.tiles_w) {
                atomicOr(&g_flash_err, kDevErrBadIndex);
                tile = tile < 0 ? 0 : a.tiles_h * a.tiles_w - 1;
            }
            const int ky = tile / a.tiles_w, kx = tile - ky * a.tiles_w;
            tc::tma_load_5d(dst, tm, c0, m.h, kx * 16, ky * 16 + (j & 3) * 4, kvb, bar);
        } else {
            tc::tma_load_4d(dst, tm, c0, m.h, j * kBN, kvb, bar);
        }
    };

    if (warp == W_PROD) {
        // ------------------------------------------------ TMA producer
        regs_other();
        if (lane == 0) {
            Cursor<GEO> ck, cv;  // the K part of ring use s (step s) and its V part (step s - 2)
            ck.start(a);
            cv.start(a);
            int qloads[2] = {0, 0};  // Q loads issued per buffer
            int s = 0;               // ring uses issued
            bool ok = true;
            for (;; ++s) {
                const bool has_k = ck.valid(a);
                const bool has_v = s >= 2 && cv.valid(a);
                if (s >= 2 && !has_v) break;  // uses 0, 1 always happen (they carry no V)
                const bool item_start = has_k && ck.j == 0;
                const Item mq = ck.m;
                const int kq = ck.k;
                const int st = s % NST;
                if (s >= NST)
                    for (int x = 0; x < 2 && ok; ++x)
                        ok = wait_bar(&bars, &bars.slot_done[st][x], ((s / NST) - 1) & 1);
                if (!ok) break;
                const uint32_t bar = smem_u32(&bars.slot_full[st]);
                const uint32_t bytes = (has_k ? DL::KTile : 0u) + (has_v ? DL::VTile : 0u);
                if (bytes)
                    mbar_arrive_expect_tx(bar, bytes);
                else
                    mbar_arrive(bar);  // a use with nothing to carry (a one-step run)
                if (has_k) {
                    const uint32_t kt = k_s + st * DL::KTile;
                    for (int bx = 0; bx < DL::NB0; ++bx) load_kv(kt + bx * kKVBox, &tm_k, ck.m, ck.j, bx * 64, bar);
                    if constexpr (DL::TK > 0) load_kv(kt + DL::NB0 * kKVBox, &tm_kt, ck.m, ck.j, DL::NB0 * 64, bar);
                    ck.next(a);
                }
                if (has_v) {
                    for (int bx = 0; bx < DL::NBV; ++bx)
                        load_kv(v_s + st * DL::VTile + bx * kKVBox, &tm_v, cv.m, cv.j, bx * 64, bar);
                    cv.next(a);
                }
                if (item_start) {
                    // Q of item k into buffer k & 1 once item k - 2's output staged there was
                    // stored.  After the ring use: that output's last PV needs this use's V.
                    const int qb = kq & 1;
                    if (kq >= 2)
                        for (int x = 0; x < 2 && ok; ++x)
                            ok = wait_bar(&bars, &bars.q_free[qb][x], ((kq - 2) >> 1) & 1);
                    if (!ok) {
                        ++s;  // this ring use was issued
                        break;
                    }
                    for (int x = 0; x < 2; ++x) {
                        const uint32_t qbar = smem_u32(&bars.q_full[qb][x]);
                        const uint32_t qt = q_s + (qb * 2 + x) * DL::QTile;
                        mbar_arrive_expect_tx(qbar, DL::QTile);
                        for (int bx = 0; bx < DL::NB0; ++bx) load_q(qt + bx * kQBox, &tm_q, mq, x, bx * 64, qbar);
                        if constexpr (DL::TK > 0) load_q(qt + DL::NB0 * kQBox, &tm_qt, mq, x, DL::NB0 * 64, qbar);
                    }
                    ++qloads[qb];
                }
            }
            if (!ok || *(volatile int*)&bars.abort) {
                // drain: let this CTA's loads land before it exits (bounded)
                for (int st = 0; st < NST; ++st) {
                    const int uses = (s - st + NST - 1) / NST;  // uses of slot st issued
                    if (uses > 0)
                        mbar_wait_bounded(smem_u32(&bars.slot_full[st]), (uses - 1) & 1, &g_flash_err);
                }
                for (int qb = 0; qb < 2; ++qb)
                    if (qloads[qb] > 0)
                        for (int x = 0; x < 2; ++x)
                            mbar_wait_bounded(smem_u32(&bars.q_full[qb][x]), (qloads[qb] - 1) & 1, &g_flash_err);
            }
        }
    } else if (warp == W_MMA || warp == W_MMA + 1) {
        // ------------------------------------------------ MMA issuers (warp-uniform)
        regs_other();
        // A wait of one issuer overlaps the other's MMA issue, so the tensor
        // core queue stays fed.
        const int x = warp - W_MMA;
        constexpr uint32_t idesc_s = tc::idesc_bf16(kBM, kBN, 0, 0);
        constexpr uint32_t idesc_o = tc::idesc_bf16(kBM, NO, 0, 1);
        // Descriptors are built once; a K step, buffer or slot only moves the
        // start address (bits 0..13, in 16-byte units), which stays below
        // 2^14 because shared memory is smaller than 256 KB.
        const uint64_t dq = tc::smem_desc(q_s + x * DL::QTile, 16, 1024, 2);
        const uint64_t dk = tc::smem_desc(k_s, 16, 1024, 2);
        const uint64_t dqt = tc::smem_desc(q_s + x * DL::QTile + DL::NB0 * kQBox, 16, 8 * DL::TB, DL::tail_swizzle);
        const uint64_t dkt = tc::smem_desc(k_s + DL::NB0 * kKVBox, 16, 8 * DL::TB, DL::tail_swizzle);
        const uint64_t dv = tc::smem_desc(v_s, kKVBox, 1024, 2);
        // S_X(s) = Q_X(item) K_s^T into S buffer s & 1
        auto issue_s = [&](int qb, int st, int buf) {
            const uint32_t d = tmem + x * 128 + buf * 64;
            const uint64_t qo = (uint64_t)((qb * 2 * DL::QTile) >> 4), ko = (uint64_t)((st * DL::KTile) >> 4);
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                if (ks < DL::NB0 * 4) {
                    const uint32_t offa = (ks >> 2) * (kQBox >> 4) + (ks & 3) * 2;
                    const uint32_t offb = (ks >> 2) * (kKVBox >> 4) + (ks & 3) * 2;
                    tc::mma_ss_warp(d, dq + qo + offa, dk + ko + offb, idesc_s, ks > 0 ? 1u : 0u);
                } else {  // tail box: 32 bytes per K step
                    const uint32_t off = (ks - DL::NB0 * 4) * 2;
                    tc::mma_ss_warp(d, dqt + qo + off, dkt + ko + off, idesc_s, ks > 0 ? 1u : 0u);
                }
            }
        };
        Cursor<GEO> cs;  // the item and step of the next score product S(s)
        cs.start(a);
        bool ok = true;
        // prologue: S(0), S(1) (ring uses 0 and 1 carry K only)
        for (int s = 0; s < 2 && ok; ++s) {
            ok = wait_bar(&bars, &bars.slot_full[s], 0);
            if (ok && cs.valid(a) && cs.j == 0) ok = wait_bar(&bars, &bars.q_full[cs.k & 1][x], (cs.k >> 1) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            if (cs.valid(a)) {
                if (x == 0 || cs.m.has_b) issue_s(cs.k & 1, s, s & 1);
                cs.next(a);
            }
            tc::commit_warp(smem_u32(&bars.slot_done[s][x]));
        }
        Cursor<GEO> cp;  // the item and step of P(g)
        cp.start(a);
        for (int g = 0; ok && cp.valid(a); ++g) {
            const int s = g + 2, st = s % NST;
            ok = wait_bar(&bars, &bars.p_full[x][g & 1], (g >> 1) & 1);
            if (ok) ok = wait_bar(&bars, ONES ? &bars.slot_ready[st] : &bars.slot_full[st], (s / NST) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            if (x == 0 || cp.m.has_b) {
                // O_X += P_X(g) V_g
                const uint64_t vdesc = dv + (uint64_t)((st * DL::VTile) >> 4);
                const uint32_t d = tmem + 256 + x * 128, pa = tmem + x * 128 + (g & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    tc::mma_ts_warp(d, pa + kk * 8, vdesc + kk * 128, idesc_o, (cp.j > 0 || kk > 0) ? 1u : 0u);
            }
            // the item's output is complete once its last PV retires; committed
            // before the next item's Q is waited for (that Q may go where this
            // output is staged)
            if (cp.j + 1 == cp.m.nkv) tc::commit_warp(smem_u32(&bars.o_done[x]));
            // S_X(g+2) reuses the buffer PV_X(g) has just been queued on
            if (cs.valid(a)) {
                if (cs.j == 0) ok = wait_bar(&bars, &bars.q_full[cs.k & 1][x], (cs.k >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                if (x == 0 || cs.m.has_b) issue_s(cs.k & 1, st, s & 1);
                cs.next(a);
            }
            tc::commit_warp(smem_u32(&bars.slot_done[st][x]));
            cp.next(a);
        }
        // all MMAs this warp issued complete before TMEM is released
        tc::commit_warp(smem_u32(&bars.mma_done[x]));
        mbar_wait_bounded(smem_u32(&bars.mma_done[x]), 0, &g_flash_err);
    } else if (warp == W_ONES) {
        // ------------------------------------------------ V-ones warp
        regs_other();
        if constexpr (ONES) {
            const uint32_t col = (uint32_t)a.d;
            const uint32_t ch = (col & 63) >> 3, e = col & 7;
            Cursor<GEO> cv;  // the V part of ring use s (step s - 2)
            cv.start(a);
            bool ok = true;
            for (int s = 0; ok; ++s) {
                const bool has_v = s >= 2 && cv.valid(a);
                if (s >= 2 && !has_v) break;
                const int st = s % NST;
                ok = __all_sync(0xffffffffu, wait_bar(&bars, &bars.slot_full[st], (s / NST) & 1));
                if (!ok) break;
                if (has_v) {
                    unsigned char* vbox = gen_base + (v_s - sbase) + st * DL::VTile + (col >> 6) * kKVBox;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int r = lane + 32 * h2;
                        *reinterpret_cast<uint16_t*>(vbox + r * 128 + ((ch ^ (r & 7)) << 4) + e * 2) = 0x3F80u;
                    }
                    fence_proxy_async_smem();
                    cv.next(a);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bars.slot_ready[st]));
            }
        }
    } else if (warp < NSW) {
        // ------------------------------------------------ softmax warps
        if constexpr (SPLIT == 2)
            asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSplitRegsSoftmax) : "memory");
        const int lq = warp & 3;                      // TMEM lane quarter (= sub-partition)
        const int x = (warp >> 2) & 1;                // tile
        const int par = SPLIT == 2 ? (warp >> 3) : 0; // SPLIT 2: the parity of the global steps taken
        const int row = lq * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(lq * 32) << 16);
        const uint32_t o_col = 256 + x * 128;
        // O's 16-column chunks this warp normalises and stages in the epilogue
        constexpr int NC0 = SPLIT == 2 ? (NC + 1) / 2 : NC;
        const int c_lo = par == 0 ? 0 : NC0, c_hi = par == 0 ? NC0 : NC;
        const bool store_thread = par == 0 && row == 0;
        Cursor<GEO> c;
        c.start(a);
        bool ok = true;
        if (x == 1 && c.valid(a)) ok = wait_bar(&bars, &bars.b_go, 0);
        int g = 0;              // global step
        bool owe_free = false;  // store thread: the previous item's Q buffer is still to be freed
        int ns = 0;             // row-sum exchanges (SPLIT 2 without the ones column)
        for (; ok && c.valid(a); c.next_item(a)) {
            const Item m = c.m;
            const int k = c.k;
            const bool work = x == 0 || m.has_b;
            // m_ref: the maximum P was taken against at this warp's latest step
            // of the item (SPLIT 1: every step); l: the row sum in its units
            float m_ref = -INFINITY, l = 0.f;
            if (SPLIT == 2 && owe_free && m.nkv == 1 && (g & 1) != par) {
                // no step of this item here: free the previous item's Q buffer now
                bulk_wait_read<0>();
                mbar_arrive(smem_u32(&bars.q_free[(k - 1) & 1][x]));
                owe_free = false;
            }
            for (int j = 0; j < m.nkv; ++j, ++g) {
                if (SPLIT == 2 && (g & 1) != par) continue;  // the other warp's step
                // S_X(g) was issued with ring use g
                ok = wait_bar(&bars, &bars.slot_done[g % NST][x], (g / NST) & 1);
                if (!ok) break;
                const uint32_t s_col = x * 128 + (g & 1) * 64;
                // The row's maximum for this step from mt, the row max of its
                // scaled scores: against the maximum so far -- this warp's own
                // (SPLIT 1) or the one the other warp took at step g - 1 (SPLIT
                // 2, read behind the barrier of that step's parity; waited for at
                // every step, so that the slot is not written again before it
                // was read) -- with O rescaled when it grows by more than 2^8.
                // Returns false on an abort.
                auto decide = [&](float mt, float& m_use) -> bool {
                    float m_in = m_ref;
                    if constexpr (SPLIT == 2) {
                        if (g > 0) {
                            const int pg = (g - 1) & 1;
                            if (!wait_bar(&bars, &bars.mref_full[x][lq][pg], ((g - 1) >> 1) & 1)) return false;
                            m_in = mref[(x * 2 + pg) * 128 + row];
                        }
                    }
                    if (j == 0) {
                        m_use = mt;
                        if (g == 0 && x == 0) mbar_arrive(smem_u32(&bars.b_go));
                    } else {
                        m_use = m_in;
                        const bool need = mt > m_in + kRescaleLog2;
                        if (__any_sync(0xffffffffu, need)) {
                            // O_X must hold exactly PV_X(..g-1): PV_X(g-1) was
                            // committed with ring use g + 1
                            if (!wait_bar(&bars, &bars.slot_done[(g + 1) % NST][x], ((g + 1) / NST) & 1))
                                return false;
                            tc::fence_after_sync();
                            if (need) m_use = mt;
                            const float f = ex2(m_in - m_use);
#pragma unroll 1
                            for (int cc = 0; cc < NC; ++cc) {
                                uint32_t r[16];
                                tc::ld_16col(lane_addr + o_col + cc * 16, r);
                                tc::wait_ld();
#pragma unroll
                                for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
                                tc::st_16col(lane_addr + o_col + cc * 16, r);
                            }
                        }
                    }
                    if constexpr (SPLIT == 2) {
                        // publish this step's maximum before the exponentials
                        mref[(x * 2 + (g & 1)) * 128 + row] = m_use;
                        mbar_arrive(smem_u32(&bars.mref_full[x][lq][g & 1]));
                    }
                    // this warp's running sum follows the row's maximum
                    if constexpr (!ONES)
                        if (l != 0.f && m_use != m_ref) l *= ex2(m_ref - m_use);
                    m_ref = m_use;
                    return true;
                };
                if (work) {
                    tc::fence_after_sync();
                    const int valid = TILED ? kBN : a.Lk - j * kBN;  // keys of this tile that exist
                    float sv[kBN];
                    {
                        uint32_t r0[32], r1[32];
                        tc::ld_32col(lane_addr + s_col, r0);
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
                    // row max of the raw scores (scale > 0 commutes with max):
                    // eight independent 3-input max chains
                    float mx[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float mm = tc::max3f(sv[q], sv[q + 8], sv[q + 16]);
                        mm = tc::max3f(mm, sv[q + 24], sv[q + 32]);
                        mm = tc::max3f(mm, sv[q + 40], sv[q + 48]);
                        mx[q] = fmaxf(mm, sv[q + 56]);
                    }
                    const float mt = tc::max3f(tc::max3f(mx[0], mx[1], mx[2]), tc::max3f(mx[3], mx[4], mx[5]),
                                               fmaxf(mx[6], mx[7])) * a.scale_log2;
                    float m_use;
                    ok = decide(mt, m_use);
                    if (!ok) break;
                    // exponentiate, sum and write P back as bf16 over S's columns
                    const tc::f32x2 scale2 = tc::pack2(a.scale_log2, a.scale_log2);
                    const tc::f32x2 negm2 = tc::pack2(-m_use, -m_use);
                    tc::f32x2 acc[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[q] = tc::pack2(0.f, 0.f);
#pragma unroll
                    for (int cc = 0; cc < kBN / 32; ++cc) {
                        uint32_t r[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int idx = cc * 32 + 2 * i;
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
                        tc::st_16col(lane_addr + s_col + cc * 16, r);
                    }
                    if constexpr (!ONES) {
                        float a0, a1;
                        tc::unpack2(tc::add2(tc::add2(acc[0], acc[1]), tc::add2(acc[2], acc[3])), a0, a1);
                        l += a0 + a1;
                    }
                    tc::wait_st();
                } else {
                    float m_use;
                    ok = decide(-INFINITY, m_use);
                    if (!ok) break;
                }
                if (SPLIT == 2 && j == 0 && k > 0) {
                    // the item's first PV overwrites O: both warps of the tile
                    // have read the previous item's O (its stage barrier)
                    ok = wait_bar(&bars, &bars.stage[x], (k - 1) & 1);
                    if (!ok) break;
                }
                tc::fence_before_sync();
                mbar_arrive(smem_u32(&bars.p_full[x][g & 1]));
                if (owe_free) {
                    // the previous item's output store has read its staging: free that Q buffer
                    bulk_wait_read<0>();
                    mbar_arrive(smem_u32(&bars.q_free[(k - 1) & 1][x]));
                    owe_free = false;
                }
            }
            if (!ok) break;
            // ---------------- epilogue: O / l -> bf16 -> swizzled smem -> TMA store
            ok = wait_bar(&bars, &bars.o_done[x], k & 1);
            if (!ok) break;
            // the item's Q buffer: every S of this item has retired
            unsigned char* stage = gen_base + ((k & 1) * 2 + x) * DL::QTile;
            if (work) {
                tc::fence_after_sync();
                if constexpr (ONES) {  // O's column d: the row sum of P
                    uint32_t lbits;
                    tc::ld_1col(lane_addr + o_col + (uint32_t)a.d, lbits);
                    tc::wait_ld();
                    l = __uint_as_float(lbits);
                } else if constexpr (SPLIT == 2) {
                    // the two warps' sums, each in the units of its latest
                    // maximum, brought to the later (larger) one and added in
                    // one order (double-buffered by exchange parity; both warps
                    // of the tile skip the exchange together when the tile is idle)
                    float* xs = xsum + ((ns & 1) * 2 + x) * 4 * 128;
                    xs[par * 128 + row] = l;
                    xs[(2 + par) * 128 + row] = m_ref;
                    mbar_arrive(smem_u32(&bars.xsum_done[x][lq]));
                    ok = wait_bar(&bars, &bars.xsum_done[x][lq], ns & 1);
                    ++ns;
                    if (!ok) break;
                    const float l0 = xs[row], l1 = xs[128 + row];
                    const float m0 = xs[256 + row], m1 = xs[384 + row];
                    const float mf = fmaxf(m0, m1);
                    l = (l0 != 0.f ? l0 * ex2(m0 - mf) : 0.f) + (l1 != 0.f ? l1 * ex2(m1 - mf) : 0.f);
                }
                const float inv = 1.f / l;
                for (int cc = c_lo; cc < c_hi; ++cc) {
                    uint32_t r[16];
                    tc::ld_16col(lane_addr + o_col + cc * 16, r);
                    tc::wait_ld();
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
                    const int col = cc * 16;
                    if (col < DL::NB0 * 64) {
                        const int bx = col >> 6;
                        const int ch = (col & 63) >> 3;
                        unsigned char* rowp = stage + bx * kQBox + row * 128;
                        *reinterpret_cast<uint4*>(rowp + ((ch ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<uint4*>(rowp + (((ch + 1) ^ (row & 7)) << 4)) =
                            make_uint4(w[4], w[5], w[6], w[7]);
                    } else {  // tail box
                        const int u = (col - DL::NB0 * 64) >> 3;
                        unsigned char* rowp = stage + DL::NB0 * kQBox + row * DL::TB;
                        *reinterpret_cast<uint4*>(rowp + (DL::tail_unit(row, u) << 4)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<uint4*>(rowp + (DL::tail_unit(row, u + 1) << 4)) =
                            make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
                fence_proxy_async_smem();
            }
            // Every softmax thread of the tile has staged its part once the stage
            // barrier completes; only the storing thread waits for it here (a
            // bounded wait: no thread can be left behind at a barrier after an
            // abort).  The O columns were read: the next item's first PV, which
            // waits for every thread's P (SPLIT 2: and for this barrier), may
            // overwrite them.
            tc::fence_before_sync();
            mbar_arrive(smem_u32(&bars.stage[x]));
            if (store_thread) ok = wait_bar(&bars, &bars.stage[x], k & 1);
            if (!ok) break;
            if (store_thread) {
                if (work) {
                    const uint32_t src = q_s + ((k & 1) * 2 + x) * DL::QTile;
                    for (int bx = 0; bx < DL::NB0; ++bx) {
                        if constexpr (TILED)
                            tc::tma_store_5d(&tm_o, src + bx * kQBox, bx * 64, m.h, m.tx * 16, m.ty * 16 + x * 8, m.b);
                        else
                            tc::tma_store_4d(&tm_o, src + bx * kQBox, bx * 64, m.h, (m.qblk * 2 + x) * kBM, m.b);
                    }
                    if constexpr (DL::TK > 0) {
                        const uint32_t tsrc = src + DL::NB0 * kQBox;
                        if constexpr (TILED)
                            tc::tma_store_5d(&tm_ot, tsrc, DL::NB0 * 64, m.h, m.tx * 16, m.ty * 16 + x * 8, m.b);
                        else
                            tc::tma_store_4d(&tm_ot, tsrc, DL::NB0 * 64, m.h, (m.qblk * 2 + x) * kBM, m.b);
                    }
                    bulk_commit();
                }
                owe_free = true;
            }
        }
        // shared memory stays valid until every output store has read it
        if (store_thread) bulk_wait_read<0>();
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == W_MMA) {
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

CUtensorMapSwizzle swizzle_for(int box_cols) {
    return box_cols >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// 4-D map over a [batches][rows][heads][d] bf16 view (row stride C elements):
// dims (d, heads, rows, batches), box (box_cols, 1, box_rows, 1), swizzled
// to the box's row bytes (64 columns: 128-byte; 32: 64-byte; 16: 32-byte).
bool make_map(CUtensorMap* m, const void* base, int d, int heads, long long rows, long long batches,
              long long row_stride_elems, long long batch_stride_elems, int box_rows, int box_cols = 64) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows, (cuuint64_t)batches};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)row_stride_elems * 2,
                             (cuuint64_t)(batch_stride_elems > 0 ? batch_stride_elems : rows * row_stride_elems) * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_cols, 1, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(box_cols),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 5-D map over the [frames][H][W][heads][d] bf16 spatial view: dims (d,
// heads, W, H, frames), box (box_cols, 1, 16, box_h, 1) -- 16 * box_h tokens
// of a 16-wide tile, row-major, one swizzled row each.
bool make_map_grid(CUtensorMap* m, const void* base, int d, int heads, int H, int W, int frames, int box_h,
                   int box_cols = 64) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t C = (cuuint64_t)heads * d;
    cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)frames};
    cuuint64_t strides[4] = {(cuuint64_t)d * 2, C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
    cuuint32_t box[5] = {(cuuint32_t)box_cols, 1, 16, (cuuint32_t)box_h, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(box_cols),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The seven tensor maps of one launch: Q, K, V, O with 64-column boxes and,
// for head dims with a tail box, Q, K, O with tail-width boxes.
struct FlashMaps {
    CUtensorMap q, qt, k, kt, v, o, ot;
};

// SPLIT 2 exchange arrays: maxima [2][2][128] and row sums [2][2][4][128] floats
constexpr int kSplitSmem = (2 * 2 * 128 + 2 * 2 * 4 * 128) * 4;

// Ring depth: the deepest ring (at most kMaxStages) that fits the 227 KB of
// shared memory next to the double-buffered Q tiles.
template <int KSTEPS>
constexpr int flash_nst() {
    using DL = DLayout<KSTEPS>;
    constexpr long long budget = 232448 - 2048;  // static shared memory (barriers) and slack
    constexpr long long fixed = 4LL * DL::QTile + (flash_split<KSTEPS>() == 2 ? kSplitSmem : 0) + 1024;
    constexpr long long n = (budget - fixed) / (DL::KTile + DL::VTile);
    return n > kMaxStages ? kMaxStages : (int)n;
}
template <int KSTEPS>
constexpr size_t flash_smem() {
    using DL = DLayout<KSTEPS>;
    return (size_t)4 * DL::QTile + (size_t)flash_nst<KSTEPS>() * (DL::KTile + DL::VTile) +
           (flash_split<KSTEPS>() == 2 ? kSplitSmem : 0) + 1024;
}

template <int KSTEPS, bool ONES, int GEO>
cudaError_t launch_ks1(const FlashMaps& m, const FlashTcArgs& a, cudaStream_t s) {
    constexpr int NST = flash_nst<KSTEPS>();
    static_assert(NST >= 3, "ring of at least three slots");
    constexpr size_t smem = flash_smem<KSTEPS>();
    auto kern = flash_tc_kernel<KSTEPS, NST, ONES, GEO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if constexpr (flash_split<KSTEPS>() == 2) {
        // the softmax warpgroups' setmaxnreg.inc is served by the registers the
        // launch holds: refuse a build whose launch holds fewer than the split takes
        static int regs = -1;
        if (regs < 0) {
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, kern);
            if (e != cudaSuccess) return e;
            regs = fa.numRegs;
        }
        if (regs * flash_threads<KSTEPS>() < kSplitRegsSoftmax * 512 + kSplitRegsOther * 128)
            return cudaErrorInvalidConfiguration;
    }
    // persistent: one CTA per SM (TMEM: 512 columns), each walking its items
    const int grid = a.items < device_sm_count() ? a.items : device_sm_count();
    kern<<<grid, flash_threads<KSTEPS>(), smem, s>>>(m.q, m.qt, m.k, m.kt, m.v, m.o, m.ot, a);
    return cudaGetLastError();
}
template <int KSTEPS, int GEO>
cudaError_t launch_ks(const FlashMaps& m, const FlashTcArgs& a, cudaStream_t s) {
    // a padding column inside the PV product carries the row sums when d % 16 != 0
    if (PAB_FLASH_ONES && a.d % 16 != 0) return launch_ks1<KSTEPS, true, GEO>(m, a, s);
    return launch_ks1<KSTEPS, false, GEO>(m, a, s);
}
template <int GEO>
cudaError_t launch_d(const FlashMaps& m, const FlashTcArgs& a, cudaStream_t s) {
    switch ((a.d + 15) / 16) {
        case 1: return launch_ks<1, GEO>(m, a, s);
        case 2: return launch_ks<2, GEO>(m, a, s);
        case 3: return launch_ks<3, GEO>(m, a, s);
        case 4: return launch_ks<4, GEO>(m, a, s);
        case 5: return launch_ks<5, GEO>(m, a, s);
        case 6: return launch_ks<6, GEO>(m, a, s);
        case 7: return launch_ks<7, GEO>(m, a, s);
        case 8: return launch_ks<8, GEO>(m, a, s);
        default: return cudaErrorInvalidValue;
    }
}

// Width in columns of the tail box for head dim d (0: none)
int tail_cols(int d) {
    const int ks = (d + 15) / 16, tk = ks % 4;
    return tk == 3 ? 0 : tk * 16;
}

// Maps of the tile geometries: Q and O as [8][16]-token boxes, K and V as
// [4][16]-token boxes of the [frames][H][W] grid.
bool make_grid_maps(FlashMaps* m, const void* q, const void* k, const void* v, void* out, int d, int heads, int H,
                    int W, int frames) {
    if (!make_map_grid(&m->q, q, d, heads, H, W, frames, 8) || !make_map_grid(&m->k, k, d, heads, H, W, frames, 4) ||
        !make_map_grid(&m->v, v, d, heads, H, W, frames, 4) || !make_map_grid(&m->o, out, d, heads, H, W, frames, 8))
        return false;
    const int tw = tail_cols(d);
    if (!tw) {
        m->qt = m->q;
        m->kt = m->k;
        m->ot = m->o;
        return true;
    }
    return make_map_grid(&m->qt, q, d, heads, H, W, frames, 8, tw) &&
           make_map_grid(&m->kt, k, d, heads, H, W, frames, 4, tw) &&
           make_map_grid(&m->ot, out, d, heads, H, W, frames, 8, tw);
}

}  // namespace

cudaError_t launch_flash(const void* q, const void* k, const void* v, void* out, int batches, long long Lq,
                         int Lk, int heads, int d, long long q_bstride, long long kv_bstride, cudaStream_t s) {
    if (Lq == 0 || batches == 0) return cudaSuccess;
    if (Lk < 1 || heads < 1 || batches < 0) return cudaErrorInvalidValue;
    const long long C = (long long)heads * d;
    const long long qblocks = (Lq + 2 * kBM - 1) / (2 * kBM);
    if (qblocks * heads * batches > 0x7fffffffLL || Lq > 0x7fffffffLL) return cudaErrorInvalidValue;
    FlashMaps m;
    const long long kv_batches = kv_bstride > 0 ? batches : 1;
    const int tw = tail_cols(d);
    if (!make_map(&m.q, q, d, heads, Lq, batches, C, q_bstride, kBM) ||
        !make_map(&m.k, k, d, heads, Lk, kv_batches, C, kv_bstride, kBN) ||
        !make_map(&m.v, v, d, heads, Lk, kv_batches, C, kv_bstride, kBN) ||
        !make_map(&m.o, out, d, heads, Lq, batches, C, q_bstride, kBM))
        return cudaErrorInvalidValue;
    if (tw) {
        if (!make_map(&m.qt, q, d, heads, Lq, batches, C, q_bstride, kBM, tw) ||
            !make_map(&m.kt, k, d, heads, Lk, kv_batches, C, kv_bstride, kBN, tw) ||
            !make_map(&m.ot, out, d, heads, Lq, batches, C, q_bstride, kBM, tw))
            return cudaErrorInvalidValue;
    } else {
        m.qt = m.q;
        m.kt = m.k;
        m.ot = m.o;
    }
    FlashTcArgs a;
    a.Lq = (int)Lq;
    a.Lk = Lk;
    a.kv_batched = kv_bstride > 0 ? 1 : 0;
    a.d = d;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
    a.heads = heads;
    a.per_bh = (int)qblocks;
    a.items = (int)(qblocks * heads * batches);
    a.tiles_h = a.tiles_w = a.reach_h = a.reach_w = 0;
    a.kv_list = nullptr;
    a.kv_count = 0;
    return launch_d<kGeoFull>(m, a, s);
}

cudaError_t launch_flash_sta(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                             int heads, int d, int win_h, int win_w, cudaStream_t s) {
    if (frames == 0 || H == 0 || W == 0) return cudaSuccess;
    if (H % kStaTile || W % kStaTile || win_h % kStaTile || win_w % kStaTile || win_h <= 0 || win_w <= 0 ||
        (win_h / kStaTile) % 2 == 0 || (win_w / kStaTile) % 2 == 0)
        return cudaErrorInvalidValue;
    const long long tiles = (long long)(H / kStaTile) * (W / kStaTile);
    if (tiles * heads * frames > 0x7fffffffLL || heads < 1) return cudaErrorInvalidValue;
    FlashMaps m;
    if (!make_grid_maps(&m, q, k, v, out, d, heads, H, W, frames)) return cudaErrorInvalidValue;
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
    a.heads = heads;
    a.per_bh = (int)tiles;
    a.items = (int)(tiles * heads * frames);
    return launch_d<kGeoWindow>(m, a, s);
}

cudaError_t launch_flash_tile_list(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                                   int heads, int d, const int* kv_list, int kv_count, cudaStream_t s) {
    if (frames == 0 || H == 0 || W == 0) return cudaSuccess;
    if (H % kStaTile || W % kStaTile || kv_count < 1 || !kv_list) return cudaErrorInvalidValue;
    const long long tiles = (long long)(H / kStaTile) * (W / kStaTile);
    if (kv_count > tiles || tiles * heads * frames > 0x7fffffffLL || heads < 1) return cudaErrorInvalidValue;
    FlashMaps m;
    if (!make_grid_maps(&m, q, k, v, out, d, heads, H, W, frames)) return cudaErrorInvalidValue;
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
    a.heads = heads;
    a.per_bh = (int)tiles;
    a.items = (int)(tiles * heads * frames);
    return launch_d<kGeoList>(m, a, s);
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

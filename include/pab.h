/*
 * pab.h -- C ABI of the B200 (sm_100a) Pyramid Attention Broadcast library.
 *
 * A video diffusion transformer block runs three attention kinds: spatial
 * (tokens of one frame attend to each other), temporal (the frames at one
 * spatial position attend to each other) and cross (video tokens attend to
 * text tokens) -- PAB report (m.sbmmt.com), section "Implementation".
 * Pyramid Attention Broadcast computes every attention in the first and last
 * 15% of diffusion steps and, in the stable middle 70%, computes each kind
 * once per window of r_kind steps and serves ("broadcasts") that output to
 * the rest of the window -- same report, Fig. 2; paper abstract
 * "Real-Time Video Generation with Pyramid Attention Broadcast".
 *
 * Conventions shared by every entry point
 *  - Return value: PAB_OK (0) or a negative PAB_ERR_* code.  Nothing aborts,
 *    throws or traps; pab_last_error_string() describes the last failure of
 *    the calling thread.
 *  - Pointers named q, k, v, out, src, dst, a, b are DEVICE pointers (CUDA
 *    global memory of the current device) unless stated otherwise; the
 *    caller owns them.  cuda_stream is a cudaStream_t (NULL = legacy default
 *    stream); all device work is ordered on it and no call synchronises the
 *    device unless its comment says so.
 *  - Layouts are row-major with the last index contiguous.  C = heads * d and
 *    head h occupies channels [h*d, (h+1)*d) of every token row.  N = H * W.
 *  - Attention is softmax(Q K^T / sqrt(d)) V per head: no mask, no bias, no
 *    output projection.  bf16 storage, fp32 accumulation, bf16 output.  With
 *    dtype PAB_FP32 the inputs are rounded to bf16 (round to nearest even)
 *    before the same bf16 kernels run, and the output is written as fp32.
 *  - Alignment: every device pointer must be 16-byte aligned.
 *  - Limits: 8 <= d <= 128 and d % 8 == 0; temporal length T <= 128;
 *    1 <= text_len <= 512; spatial T <= 65535 frames; sizes must fit the
 *    device; otherwise PAB_ERR_ARG or PAB_ERR_UNSUPPORTED.
 */
#ifndef PAB_H
#define PAB_H

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define PAB_OK 0
#define PAB_ERR_ARG (-1)         /* bad argument (null pointer, bad size, bad kind)   */
#define PAB_ERR_STEP_ORDER (-2)  /* steps of one kind not strictly increasing          */
#define PAB_ERR_NO_CACHE (-3)    /* broadcast step whose source output was never made  */
#define PAB_ERR_CUDA (-4)        /* CUDA runtime error (incl. no device present)       */
#define PAB_ERR_OOM (-5)         /* device allocation failed                           */
#define PAB_ERR_UNSUPPORTED (-6) /* shape outside the kernels' documented limits       */

/* attention kinds */
enum { PAB_SPATIAL = 0, PAB_TEMPORAL = 1, PAB_CROSS = 2 };
/* element types at the boundary */
enum { PAB_BF16 = 0, PAB_FP32 = 1 };

/* Broadcast ranges per kind (each >= 1; 1 = never broadcast) and the edge
 * share in percent: a negative value selects the pages' 15, 0 gives no edge
 * steps (every step follows the range rule), 1..50 as given; other values
 * are rejected with PAB_ERR_ARG.  The pages order the ranges
 * r_cross >= r_temporal >= r_spatial (Fig. 2); that order is not enforced. */
typedef struct {
    int spatial;
    int temporal;
    int cross;
    int edge_pct;
} pab_ranges;

typedef struct pab_plan pab_plan; /* opaque; owns the broadcast cache */

/* Library version, (major << 16) | minor. */
int pab_version(void);

/* Text of the calling thread's last error ("" if none).  Owned by the
 * library; valid until the thread's next failing call. */
const char* pab_last_error_string(void);

/* ---------------------------------------------------------------------- */
/* Stateless attention kernels (each writes into caller memory).           */
/* ---------------------------------------------------------------------- */

/* Spatial attention (PAB report, "Implementation": attention within a frame).
 * q, k, v, out: [T, N, C].  For each frame t and head h:
 *   out[t, n, h] = sum_m softmax_m(q[t, n, h] . k[t, m, h] / sqrt(d)) v[t, m, h].
 * dtype: PAB_BF16 only (the plan handles PAB_FP32 by conversion). */
int pab_spatial_attention(const void* q, const void* k, const void* v, void* out,
                          int T, int N, int heads, int d, void* cuda_stream);

/* Sliding tile attention (STA) as the spatial kind (sgqg.cn summary of
 * "Fast Video Generation with Sliding Tile Attention", section "Sliding Tile
 * Attention (STA)": non-overlapping tiles, each query tile attends to the
 * key tiles inside a window around it, frame and window sizes in whole
 * tiles).  Within each frame of q, k, v, out [T, H*W, C] (token n = y*W + x):
 * tiles of tile x tile tokens; a query in tile (ty, tx) attends to every key
 * whose tile (ky, kx) has |ky - ty| <= (win_h/tile - 1)/2 and
 * |kx - tx| <= (win_w/tile - 1)/2 (the window is centred on the query's tile
 * and cut off at the frame edge), with the softmax of the spatial kind over
 * those keys.  tile must be 16 (the kernel's tile: one CTA's 256 queries);
 * H, W, win_h, win_w must be multiples of it, with odd win_h/tile and
 * win_w/tile (PAB_ERR_ARG else; PAB_ERR_UNSUPPORTED for another tile).
 * A window covering the frame gives pab_spatial_attention's result.
 * PAB_BF16 only. */
int pab_sta_attention(const void* q, const void* k, const void* v, void* out, int T, int H, int W,
                      int heads, int d, int tile, int win_h, int win_w, void* cuda_stream);

/* Draft attention as the spatial kind (crisp3r.com article on "Draft
 * Attention", steps 1-4: a pooled low-resolution sketch of the queries and
 * keys, its draft attention map, the best regions as a structured sparse
 * mask, kept blocks contiguous).  Two calls:
 *
 * pab_draft_select: per frame, average-pool q and k ([T, H*W, C], bf16) over
 * region x region-token regions (R = (H/region)(W/region) per frame); the
 * draft score of query region i and key region j for head h is
 * qbar_i . kbar_j / sqrt(d); every query region keeps the `keep` key regions
 * with the highest scores (equal scores: the lower index), written to sel
 * ([T, heads, R, keep] int32, device memory, ascending index per row).
 * Means and scores are fp32.  workspace: device scratch of at least
 * pab_draft_workspace_bytes(...) bytes, owned by the caller; q, k, sel and
 * workspace must be 16-byte aligned.  region must be 16; H, W multiples of
 * 16; 1 <= keep <= R <= 4096.
 *
 * pab_region_sparse_attention: every query of region i attends to the tokens
 * of the key regions sel[t][h][i][0..keep) (softmax over those only).  sel
 * may come from pab_draft_select or from the caller; an index outside
 * [0, R) sets bit 2 of pab_device_errors and is clamped.
 * Keeping every region (keep = R) gives pab_spatial_attention's result.
 * PAB_BF16 only. */
int pab_draft_workspace_bytes(int T, int H, int W, int heads, int d, int region, long long* bytes);
int pab_draft_select(const void* q, const void* k, int T, int H, int W, int heads, int d, int region,
                     int keep, int* sel, void* workspace, long long workspace_bytes, void* cuda_stream);
int pab_region_sparse_attention(const void* q, const void* k, const void* v, void* out, int T, int H,
                                int W, int heads, int d, int region, int keep, const int* sel,
                                void* cuda_stream);

/* Temporal attention (same section: attention across frames).
 * q, k, v, out: [N, T, C] (the temporal view).  For each position n, head h:
 *   out[n, t, h] = sum_s softmax_s(q[n, t, h] . k[n, s, h] / sqrt(d)) v[n, s, h].
 * T <= 128.  PAB_BF16 only. */
int pab_temporal_attention(const void* q, const void* k, const void* v, void* out,
                           int N, int T, int heads, int d, void* cuda_stream);

/* Temporal attention taking and returning the SPATIAL view: q, k, v, out are
 * [T, N, C]; out[t, n, h] is the same value pab_temporal_attention gives for
 * the permuted tensors.  The kernel gathers each position's T frames at
 * stride N*C itself, so a caller holding the spatial view needs no
 * pab_layout calls around it.  T <= 128.  PAB_BF16 only. */
int pab_temporal_attention_sv(const void* q, const void* k, const void* v, void* out,
                              int T, int N, int heads, int d, void* cuda_stream);

/* Cross attention (same section: video tokens to text tokens).
 * q, out: [R, C] (R video tokens in any order; out keeps it);
 * kt, vt: [text_len, C].  Every text token is attended (no text mask).
 *   out[r, h] = sum_j softmax_j(q[r, h] . kt[j, h] / sqrt(d)) vt[j, h].
 * 1 <= text_len <= 512.  PAB_BF16 only. */
int pab_cross_attention(const void* q, const void* kt, const void* vt, void* out,
                        long long R, int text_len, int heads, int d, void* cuda_stream);

/* ---------------------------------------------------------------------- */
/* Layout change between the two views of a video token tensor.            */
/* ---------------------------------------------------------------------- */

/* The PAB report ("Implementation") attends spatially within each frame and
 * temporally across the frames at each position: the two views of one video
 * token tensor, [T, N, C] (frames outer) and [N, T, C] (positions outer).
 * to_temporal = 1: src [T, N, C] (spatial view) -> dst [N, T, C];
 * to_temporal = 0: src [N, T, C] -> dst [T, N, C].
 * dtype PAB_BF16 or PAB_FP32; bytes are moved unchanged.  src and dst must
 * not overlap.  C * element size must be a multiple of 16 bytes. */
int pab_layout(int to_temporal, const void* src, void* dst, int T, int N, int C,
               int dtype, void* cuda_stream);

/* Swap the two outer dimensions of a block array: src [P, Q, block_rows, C]
 * -> dst [Q, P, block_rows, C], i.e. dst[q][p] = src[p][q] for blocks of
 * block_rows consecutive C-element rows.  pab_layout is the case
 * block_rows = 1; with P = frames per rank, Q = ranks and block_rows =
 * positions per rank it packs a frame-sharded [T/G, N, C] tensor into the
 * per-destination chunks of a sequence-parallel all-to-all (and back).
 * Same element types, alignment, row-size and no-overlap rules as
 * pab_layout; bytes are moved unchanged. */
int pab_permute_blocks(const void* src, void* dst, int P, int Q, long long block_rows, int C, int dtype,
                       void* cuda_stream);

/* Sequence-parallel exchange (PAB report, "Parallel", Fig. 3): dynamic
 * sequence parallelism gives every rank T/G frames, and a temporal compute
 * first moves every rank's frames of position chunk g to rank g (all frames
 * of N/G positions) and afterwards moves the output back; a temporal
 * broadcast step moves nothing.  This call performs one such move for up to
 * three tensors in one launch, writing every block straight into its
 * destination buffer -- on this GPU, or a peer GPU's buffer mapped into this
 * process with pab_ipc_open -- so no packing copy and no collective carries
 * the data.
 *   src[t], t < ntensors (1..3): P * G blocks of block_rows rows of C
 *     elements; src_order 0: block (p, g) is block p * G + g
 *     ([P][G][block_rows][C], e.g. the spatial view [T/G, N, C] with
 *     P = T/G and block_rows = N/G); src_order 1: block g * P + p
 *     ([G][P][block_rows][C], e.g. the temporal output [T, N/G, C]).
 *   dst: HOST array of ntensors * G device pointers, tensor-major
 *     (dst[t * G + g]); block (p, g) of tensor t is written to rows
 *     dst_offset_rows + p * dst_stride_rows ... + block_rows - 1 of
 *     dst[t * G + g].
 * Pack (rank r of G): src_order 0, P = T/G, block_rows = N/G,
 *   dst_offset_rows = r * (T/G) * (N/G), dst_stride_rows = N/G.
 * Unpack (rank r): src_order 1, P = T/G, block_rows = N/G,
 *   dst_offset_rows = r * (N/G), dst_stride_rows = N.
 * 1 <= G <= 32; dtype PAB_BF16 or PAB_FP32; bytes are moved unchanged.
 * C * element size and every pointer 16-byte aligned.  Sources and
 * destinations must not overlap.  The writes are complete when this call's
 * work on cuda_stream is; a caller whose destinations are other GPUs' memory
 * orders them before the readers with a stream-ordered barrier (for example
 * a one-element collective after this call on every rank). */
int pab_scatter_blocks(const void* const* src, void* const* dst, int ntensors, int G, int P,
                       long long block_rows, int C, int src_order, long long dst_offset_rows,
                       long long dst_stride_rows, int dtype, void* cuda_stream);

/* Device memory that the other processes of this node can map (CUDA IPC),
 * for the destinations of pab_scatter_blocks.  pab_ipc_alloc allocates
 * `bytes` on the current device (cudaMalloc, so the handle covers exactly
 * this buffer) and writes its 64-byte IPC handle; pab_ipc_free releases it.
 * pab_ipc_open maps another process's buffer from its handle into this
 * process (peer access enabled on demand); pab_ipc_close unmaps it.  A
 * process cannot open its own handle (CUDA returns an error). */
int pab_ipc_alloc(long long bytes, void** ptr, unsigned char handle[64]);
int pab_ipc_free(void* ptr);
int pab_ipc_open(const unsigned char handle[64], void** ptr);
int pab_ipc_close(void* ptr);

/* ---------------------------------------------------------------------- */
/* Dense parts of a video DiT block around the attention kinds (PAB report, */
/* "Implementation": PAB broadcasts the outputs of attention modules that   */
/* sit in DiT blocks between layer norms, projections and an MLP; a kind    */
/* that broadcasts also skips its norm and projections).                    */
/* ---------------------------------------------------------------------- */

/* D = epilogue(A B) on the tensor cores (bf16 inputs, fp32 accumulation):
 * A [M, K] and B [K, N] bf16 row-major (B holds weights as [in, out]); K a
 * positive multiple of 8, N a multiple of 32.
 *   epilogue 0: bf16(A B) into out[0..N/split-1], output i taking columns
 *               [i*split, (i+1)*split) as an [M, split] row-major matrix
 *               (split 0: one output of N columns; split a multiple of 32
 *               dividing N into at most 3 outputs -- one projection for
 *               q, k and v);
 *   epilogue 1: bf16(GELU(A B)) into out[0], GELU the tanh form
 *               0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)));
 *   epilogue 2: X [M, N] fp32 += A B (the residual stream, read and written),
 *               and Y [M, N] bf16 = bf16(A B) when Y is not NULL.
 * out is a HOST array of device pointers; all device pointers 16-byte
 * aligned.  Outputs must not overlap the inputs. */
int pab_block_gemm(const void* A, const void* B, int M, int N, int K, int epilogue, void* const* out, int split,
                   float* X, void* Y, void* cuda_stream);

/* x += ys[0] + ... + ys[ny-1] (each [rows, C] bf16, added in that order;
 * x [rows, C] fp32 written back) -- the cached outputs of broadcasting
 * modules added to the residual stream -- then, when h is not NULL,
 * h [rows, C] bf16 = LayerNorm(x) over each row (no affine parameters, eps
 * 1e-6; mean and variance in fp32).  ys is a HOST array of ny (0..3) device
 * pointers.  C a multiple of 8, at most 3072. */
int pab_block_layer_norm(float* x, const void* const* ys, int ny, void* h, long long rows, int C,
                         void* cuda_stream);

/* ---------------------------------------------------------------------- */
/* Attention-difference diagnostic (PAB report, Fig. 1: the difference      */
/* between consecutive diffusion steps' attention outputs, as MSE).        */
/* ---------------------------------------------------------------------- */

/* *result (HOST pointer) = mean over n elements of (a - b)^2.  For PAB_FP32
 * every squared difference is formed and accumulated in fp64; for PAB_BF16
 * the squared differences of each 16-byte vector (8 elements) are summed in
 * fp32 (exact differences, relative error < 1e-6 per vector) and that sum
 * is accumulated in fp64.  The order is fixed (bitwise reproducible for a
 * given n and device).  a and b hold n
 * elements of dtype (PAB_BF16 or PAB_FP32).  n == 0 gives 0.  Uses a
 * per-device scratch buffer (fp64 partial sums and a completion ticket) that
 * the library allocates on first use.  SYNCHRONISES cuda_stream before
 * returning. */
int pab_attn_diff_mse(const void* a, const void* b, long long n, int dtype,
                      double* result, void* cuda_stream);

/* As pab_attn_diff_mse, but writes the fp64 result to the DEVICE pointer
 * result_dev (8-byte aligned) and does not synchronise.  Calls that run
 * concurrently on different streams of one device share the scratch buffer
 * and must be serialised by the caller. */
int pab_attn_diff_mse_async(const void* a, const void* b, long long n, int dtype,
                            double* result_dev, void* cuda_stream);

/* Allocation-free variant of pab_attn_diff_mse_async, for callers that
 * cannot call cudaMalloc (code inside a framework whose memory pool owns all
 * device memory, or latency-critical loops that must not allocate).  The
 * paper has no counterpart: this is a property of the library, not of PAB.
 * Same arguments and result as pab_attn_diff_mse_async (result_dev is a
 * DEVICE pointer; no synchronisation), but the fp64 partial sums live in a
 * static device array of 4096 doubles (32 KiB) that every GPU loading the
 * library holds until exit; the call allocates nothing.  A call that would
 * need more than 4095 partial sums (only on devices with more than 1023 SMs)
 * returns PAB_ERR_UNSUPPORTED.  Every call looks up the array's device
 * address in the current device's context (cudaGetSymbolAddress; nothing is
 * cached, so a call after cudaDeviceReset finds the reloaded array).  The
 * array's completion ticket starts at zero when the library's module is
 * loaded on a device and every call returns it to zero; no call clears it.
 * All calls share the array and it keeps the last call's contents: calls
 * whose kernels overlap on the GPU race and must be serialised by the
 * caller. */
int pab_attn_diff_mse_noalloc(const void* a, const void* b, long long n, int dtype,
                              double* result_dev, void* cuda_stream);

/* Device status word of the kernels that wait on asynchronous copies: bit 0
 * is set when a bounded wait gave up (the kernel then returns early and its
 * output is incomplete); bit 2 when a region index read from device memory
 * (pab_region_sparse_attention's selection) lay outside the frame (it was
 * clamped; that output is not meaningful).  Synchronises the device to read
 * it; clear != 0 resets it.  A healthy run reads 0. */
int pab_device_errors(int clear, unsigned int* flags);

/* ---------------------------------------------------------------------- */
/* PAB plan: schedule + broadcast cache.                                   */
/* ---------------------------------------------------------------------- */

/* Create a plan for one video shape.  N = H * W tokens per frame, C = heads*d.
 * steps >= 1 diffusion steps indexed 0..steps-1 in execution order.
 * Schedule (per kind with range r; e = ceil(edge_pct * steps / 100)):
 *   step i computes iff i < e, or i >= steps - e, or (i - e) % r == 0;
 *   otherwise it is a broadcast hit served by the latest compute of the kind.
 * No device memory is allocated here (see pab_plan_prepare).
 * *out_plan receives the handle; destroy it with pab_plan_destroy. */
int pab_plan_create(int T, int H, int W, int heads, int d, int text_len, int steps,
                    pab_ranges ranges, int dtype, pab_plan** out_plan);

/* Free the plan and its cache (device memory freed; no pointer returned by
 * pab_attention stays valid).  NULL is accepted.  The cache is the store of
 * broadcast attention outputs (PAB report, "Implementation" and Fig. 2). */
int pab_plan_destroy(pab_plan* plan);

/* Start a new sampling run: the cache is invalidated and step order restarts.
 * Device memory is kept.  A broadcast reuses an output of the same run only
 * (PAB report, "Implementation" and Fig. 2: one step's attention output is
 * reused by the next few steps of that sampling run). */
int pab_plan_reset(pab_plan* plan);

/* Choose the layout of TEMPORAL q, k, v and of its output for this plan:
 * spatial_view = 0 (default) -> [N, T, C]; 1 -> [T, N, C] (the spatial view,
 * no layout change needed around the call).  Call before the run starts. */
int pab_plan_set_temporal_view(pab_plan* plan, int spatial_view);

/* Make this plan's SPATIAL computes sliding tile attention
 * (pab_sta_attention with the plan's H, W and these tile / window sizes)
 * instead of full attention within the frame; win_h = win_w = 0 restores
 * full attention.  Same argument rules as pab_sta_attention.  Call before
 * the run starts (the broadcast schedule and cache are unchanged). */
int pab_plan_set_spatial_window(pab_plan* plan, int tile, int win_h, int win_w);

/* Make this plan's SPATIAL computes draft attention (pab_draft_select then
 * pab_region_sparse_attention with the plan's H, W, region and keep; the
 * plan owns the scratch and the selection); keep = 0 restores full
 * attention.  A spatial window (pab_plan_set_spatial_window) and a draft
 * setting replace each other.  Same argument rules as pab_draft_select. */
int pab_plan_set_spatial_draft(pab_plan* plan, int region, int keep);

/* Attention-difference diagnostic inside the plan (PAB report, Fig. 1: the
 * difference between consecutive diffusion steps' attention outputs, as MSE).
 * With results_dev set -- a DEVICE array of 3 * steps doubles, kind-major,
 * 8-byte aligned, owned by the caller -- every compute of a kind after the
 * kind's first compute of the run also writes
 *   results_dev[kind * steps + step] = mean over T*N*C of (out - prev)^2,
 * prev being the kind's previous computed output (the plan's other slot).
 * The MSE kernel (the reduction of pab_attn_diff_mse_async) runs on the
 * same stream right after the kind's attention kernel, so the value is
 * ready when the output is, with no host synchronisation.  Nothing is
 * written for broadcast steps (the output is the source step's, bit for
 * bit) or for a kind's first compute.
 * NULL disables.  The first call with a non-NULL array allocates the plan's
 * reduction scratch on the current device (the plan's device). */
int pab_plan_set_diff_mse(pab_plan* plan, double* results_dev);

/* Where the plan's MSE launches run (pab_plan_set_diff_mse).  enable = 1:
 * on cuda_stream (a side stream; NULL is the legacy default stream), so the
 * HBM-bound MSE overlaps the next attention computes: after each compute the
 * compute stream records an event the side stream waits on before the MSE
 * launch, and the kind's next compute -- which overwrites the slot that MSE
 * reads -- waits on the compute stream for an event recorded behind it.  The
 * table entries are then complete once cuda_stream has drained (synchronise
 * it, or the device, before reading them); the values are bit-identical to
 * the in-line ones (the same kernel and reduction).  enable = 0 (the
 * default): in line on the compute stream, after the compute; a pending
 * side-stream MSE is waited for first (the launches share the plan's
 * scratch).  cuda_stream must belong to the plan's device and outlive the
 * plan's use of it; pab_plan_destroy waits for every pending side-stream MSE.
 * The first enable creates the plan's events on the current device.
 * Errors: PAB_ERR_ARG (null plan, enable not 0 or 1), PAB_ERR_CUDA. */
int pab_plan_set_diff_mse_stream(pab_plan* plan, int enable, void* cuda_stream);

/* Allocate the cache (2 output slots per kind, plus bf16 staging for
 * PAB_FP32 plans) on the current device now instead of at each kind's first
 * compute.  Idempotent. */
int pab_plan_prepare(pab_plan* plan);

/* *is_compute = 1 if (kind, step) computes, 0 if it is a broadcast hit, by
 * the rule of pab_plan_create (PAB report, "Implementation" and Fig. 2: every
 * attention computes in the first and last 15% of the steps; in between each
 * kind is computed once per window of its range and broadcast to the rest).
 * Host only, no GPU needed. */
int pab_schedule_query(const pab_plan* plan, int kind, int step, int* is_compute);

/* *source_step = the step whose computed output (kind, step) uses (step
 * itself when it computes).  Host only. */
int pab_schedule_source(const pab_plan* plan, int kind, int step, int* source_step);

/* Number of computing steps of `kind` over the whole run.  Host only. */
int pab_schedule_count(const pab_plan* plan, int kind, int* computes);

/* Run attention `kind` for diffusion step `step` under the schedule.
 *  Compute step: runs the kind's kernel on cuda_stream into one of the
 *    plan's two output slots of that kind and sets *out to it.
 *    Shapes: SPATIAL q,k,v [T, N, C]; TEMPORAL q,k,v [N, T, C] (or
 *    [T, N, C] after pab_plan_set_temporal_view(plan, 1));
 *    CROSS q [T*N, C], k,v [text_len, C].  *out has q's layout.
 *  Broadcast hit: launches nothing, copies nothing, ignores q, k, v (which
 *    may be NULL) and sets *out to the slot that holds the output of the
 *    kind's latest compute (bit-identical to it).
 * Element type: the plan's dtype.  Steps of one kind must be strictly
 * increasing (else PAB_ERR_STEP_ORDER); a hit whose source step was not the
 * kind's latest compute returns PAB_ERR_NO_CACHE.
 * Lifetime: the pointer stays valid and unchanged until the SECOND following
 * compute of the same kind is launched, or reset/destroy -- long enough to
 * compare step i with step i-1. */
int pab_attention(pab_plan* plan, int kind, int step, const void* q, const void* k,
                  const void* v, const void** out, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* PAB_H */

// kernels.h -- host-side launchers of the sm_100a kernels (internal to the
// library; the public ABI is include/pab.h).  Each launcher validates nothing
// beyond what its kernel needs: argument checks live in pab_api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pab {

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Record `code` and a message as the calling thread's last error; returns code.
int report_error(int code, const char* fmt, ...);

// --- attention-difference MSE (one launch, fp64, deterministic) ----------
// Number of per-block partial sums used for n elements on this device.
int mse_num_partials(long long n, int elem_size);
// scratch: num_partials + 1 doubles; scratch[0] is the completion ticket
// (zero before the call, zero again after it), the rest the partials.
cudaError_t launch_mse(const void* a, const void* b, long long n, int dtype, double* scratch,
                       int num_partials, double* result_dev, cudaStream_t s);

// --- layout change [T,N,C] <-> [N,T,C] (bulk-copy engine) ----------------
cudaError_t launch_layout(int to_temporal, const void* src, void* dst, int T, int N,
                          int row_bytes, cudaStream_t s);
// Swap the two outer dimensions of [P][Q][block] rows of row_bytes each:
// dst[q][p][w] = src[p][q][w] (blocks of `block` rows move together).
cudaError_t launch_swap_outer(const void* src, void* dst, int P, int Q, long long block, int row_bytes,
                              cudaStream_t s);
unsigned int layout_device_errors(bool clear);

// --- sequence-parallel exchange: multi-destination block copy --------------
// Up to kScatterMaxTensors tensors of P * G blocks (block_rows rows of
// row_bytes); block (p, g) (source index p*G+g for src_order 0, g*P+p for 1)
// of tensor t goes to dst[t*G + g] + (dst_offset_rows + p*dst_stride_rows)
// rows.  Destinations may be peer-GPU memory mapped into this process.
constexpr int kScatterMaxTensors = 3;
constexpr int kScatterMaxRanks = 32;
cudaError_t launch_scatter_blocks(const void* const* src, void* const* dst, int ntensors, int G, int P,
                                  long long block_rows, int row_bytes, int src_order, long long dst_offset_rows,
                                  long long dst_stride_rows, cudaStream_t s);

// --- temporal short-sequence attention ([N,T,C], L = T) -------------------
// spatial_view = 1: q, k, v, out are [T, N, C] instead of [N, T, C]
cudaError_t launch_temporal(const void* q, const void* k, const void* v, void* out, int N, int T,
                            int heads, int d, int spatial_view, cudaStream_t s);
unsigned int temporal_device_errors(bool clear);

// --- flash attention for spatial (per frame) and cross (shared text K/V) --
// Rows of batch b, head h: q + b*q_bstride + i*C + h*d (elements); likewise
// k/v with kv_bstride (0 = shared K/V).  out has q's layout.
cudaError_t launch_flash(const void* q, const void* k, const void* v, void* out, int batches,
                         long long Lq, int Lk, int heads, int d, long long q_bstride,
                         long long kv_bstride, cudaStream_t s);
// Sliding tile attention within each frame of a [frames][H*W][heads*d] bf16
// spatial view: 16 x 16-token tiles, a window of win_h x win_w tokens (odd
// tile counts) centred on the query's tile and clipped at the frame edge.
// H, W, win_h, win_w must be multiples of 16 (cudaErrorInvalidValue else).
cudaError_t launch_flash_sta(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                             int heads, int d, int win_h, int win_w, cudaStream_t s);

// Attention of every 16 x 16 query tile of each frame over the 16 x 16 key
// tiles kv_list names for it: [frames][heads][tiles][kv_count] tile indices
// (ty * (W/16) + tx) of the same frame.  An index outside the frame raises
// kDevErrBadIndex in the flash status word and is clamped.
cudaError_t launch_flash_tile_list(const void* q, const void* k, const void* v, void* out, int frames, int H, int W,
                                   int heads, int d, const int* kv_list, int kv_count, cudaStream_t s);

unsigned int flash_device_errors(bool clear);

// --- draft attention's low-resolution half: pooled sketch + region selection
// sketch: draft_sketch_bytes(...) of device scratch (fp32 means of q and k
// over 16 x 16-token regions); sel: [T][heads][R][keep] int32, per query
// region the keep key regions with the highest draft scores, ascending.
size_t draft_sketch_bytes(int T, int H, int W, int heads, int d);
cudaError_t launch_draft_select(const void* q, const void* k, int T, int H, int W, int heads, int d, int keep,
                                int* sel, void* sketch, cudaStream_t s);

// --- cross attention (text_len <= 128: persistent cross_tc; longer: flash) --
cudaError_t launch_cross(const void* q, const void* kt, const void* vt, void* out, long long R, int Lk, int heads,
                         int d, cudaStream_t s);
unsigned int cross_device_errors(bool clear);

// --- dense parts of a DiT block around the attention kinds ----------------
// D = epilogue(A B): A [M, K] bf16 row-major, B [K, N] bf16 row-major, K a
// multiple of 8, N of 32.  epi 0: bf16 outputs out[0..2] of `split` columns
// each (split 0: one output of N columns); 1: bf16(GELU_tanh(.)) into out[0];
// 2: X [M, N] fp32 += A B, and Y [M, N] bf16 = A B when Y is not null.
cudaError_t launch_gemm(const void* A, const void* B, int M, int N, int K, int epi, void* const* out, int split,
                        float* X, void* Y, cudaStream_t s);
// x += ys[0] + ... + ys[ny-1] (bf16, in that order; x fp32 written back),
// then h [rows, C] bf16 = LayerNorm(x) (no affine) when h is not null.
// C % 4 == 0, C <= 3072, ny <= 3.
cudaError_t launch_ln_rows(float* x, const void* const* ys, int ny, void* h, long long rows, int C, float eps,
                           cudaStream_t s);
unsigned int block_device_errors(bool clear);

// --- dtype conversion for fp32 plans --------------------------------------
cudaError_t launch_f32_to_bf16(const float* src, void* dst, long long n, cudaStream_t s);
cudaError_t launch_bf16_to_f32(const void* src, float* dst, long long n, cudaStream_t s);

}  // namespace pab

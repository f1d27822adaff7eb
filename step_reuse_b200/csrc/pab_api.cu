// pab_api.cu -- the C ABI of include/pab.h: argument checks, error
// reporting, the Pyramid Attention Broadcast plan (schedule + broadcast
// cache) and dispatch to the sm_100a kernels.
//
// Schedule (PAB report, "Implementation" and Fig. 2; paper abstract): the
// first and last edge_pct% of the diffusion steps compute every attention;
// in the middle segment each kind computes at the first step of every window
// of r_kind steps and the other r_kind - 1 steps are broadcast hits.  With
// e = ceil(edge_pct * steps / 100), lo = e, hi = steps - e:
//     compute(i)  <=>  i < lo  or  i >= hi  or  (i - lo) % r == 0
//     source(i)   =    i if compute(i) else lo + ((i - lo) / r) * r.
// Broadcast cache: two output slots per kind.  A compute writes the slot
// that does not hold the latest output, then becomes the latest; a hit
// returns the latest slot's pointer (no launch, no copy).
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "../../include/pab.h"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    const int code = (e == cudaErrorMemoryAllocation) ? PAB_ERR_OOM : PAB_ERR_CUDA;
    return fail(code, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;

// Per-device scratch of the MSE kernel: a completion ticket, the fp64
// partials and (for the synchronous call) one result slot.  The ticket is
// cleared when the buffer is allocated and returned to zero by every call.
struct MseScratch {
    double* buf = nullptr;
    int capacity = 0;  // doubles
};
std::mutex g_scratch_mu;
MseScratch g_mse_scratch[kMaxDevices];

int current_device(int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (*dev < 0 || *dev >= kMaxDevices) return fail(PAB_ERR_UNSUPPORTED, "device index %d", *dev);
    return PAB_OK;
}

int mse_scratch(int need, double** out, cudaStream_t stream) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    MseScratch& s = g_mse_scratch[dev];
    if (s.capacity < need) {
        if (s.buf) cudaFree(s.buf);
        s.buf = nullptr;
        s.capacity = 0;
        cudaError_t e = cudaMalloc(&s.buf, sizeof(double) * (size_t)need);
        if (e != cudaSuccess) return cuda_fail(e, "MSE scratch allocation");
        e = cudaMemsetAsync(s.buf, 0, sizeof(unsigned long long), stream);  // the completion ticket
        if (e != cudaSuccess) return cuda_fail(e, "MSE scratch clear");
        s.capacity = need;
    }
    *out = s.buf;
    return PAB_OK;
}

int check_dims(int heads, int d) {
    if (heads <= 0 || d <= 0) return fail(PAB_ERR_ARG, "heads (%d) and d (%d) must be positive", heads, d);
    if (d % 8 != 0 || d > 128)
        return fail(PAB_ERR_UNSUPPORTED, "head dim %d unsupported (need d %% 8 == 0, d <= 128)", d);
    return PAB_OK;
}

int check_ptrs(const char* names, const void* a, const void* b, const void* c, const void* o) {
    const void* ps[4] = {a, b, c, o};
    for (int i = 0; i < 4; ++i) {
        if (!ps[i]) return fail(PAB_ERR_ARG, "null device pointer among (%s)", names);
        if (!aligned16(ps[i])) return fail(PAB_ERR_ARG, "device pointer among (%s) not 16-byte aligned", names);
    }
    return PAB_OK;
}

int run_spatial(const void* q, const void* k, const void* v, void* out, int T, int N, int heads,
                int d, cudaStream_t s) {
    const long long C = (long long)heads * d;
    cudaError_t e = pab::launch_flash(q, k, v, out, T, N, N, heads, d, (long long)N * C,
                                      (long long)N * C, s);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "spatial attention launch");
}

int check_sta(int H, int W, int tile, int win_h, int win_w) {
    if (tile != 16) return fail(PAB_ERR_UNSUPPORTED, "sliding tile attention tile %d unsupported (need 16)", tile);
    if (H % tile || W % tile) return fail(PAB_ERR_ARG, "frame %d x %d is not whole %d-token tiles", H, W, tile);
    if (win_h <= 0 || win_w <= 0 || win_h % tile || win_w % tile || (win_h / tile) % 2 == 0 ||
        (win_w / tile) % 2 == 0)
        return fail(PAB_ERR_ARG, "window %d x %d must be an odd number of %d-token tiles each way", win_h, win_w,
                    tile);
    return PAB_OK;
}

int run_sta(const void* q, const void* k, const void* v, void* out, int T, int H, int W, int heads, int d,
            int win_h, int win_w, cudaStream_t s) {
    cudaError_t e = pab::launch_flash_sta(q, k, v, out, T, H, W, heads, d, win_h, win_w, s);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "sliding tile attention launch");
}

int check_draft(int H, int W, int region, int keep) {
    if (region != 16) return fail(PAB_ERR_UNSUPPORTED, "draft attention region %d unsupported (need 16)", region);
    if (H % region || W % region) return fail(PAB_ERR_ARG, "frame %d x %d is not whole %d-token regions", H, W, region);
    const long long R = (long long)(H / region) * (W / region);
    if (R > 4096) return fail(PAB_ERR_UNSUPPORTED, "%lld regions per frame exceed 4096", R);
    if (keep < 1 || keep > R) return fail(PAB_ERR_ARG, "keep=%d outside [1, %lld]", keep, R);
    return PAB_OK;
}

int run_draft(const void* q, const void* k, const void* v, void* out, int T, int H, int W, int heads, int d,
              int keep, int* sel, void* sketch, cudaStream_t s) {
    cudaError_t e = pab::launch_draft_select(q, k, T, H, W, heads, d, keep, sel, sketch, s);
    if (e != cudaSuccess) return cuda_fail(e, "draft selection launch");
    e = pab::launch_flash_tile_list(q, k, v, out, T, H, W, heads, d, sel, keep, s);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "region-sparse attention launch");
}

int run_temporal(const void* q, const void* k, const void* v, void* out, int N, int T, int heads,
                 int d, int spatial_view, cudaStream_t s) {
    cudaError_t e = pab::launch_temporal(q, k, v, out, N, T, heads, d, spatial_view, s);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "temporal attention launch");
}

int run_cross(const void* q, const void* kt, const void* vt, void* out, long long R, int Lt,
              int heads, int d, cudaStream_t s) {
    cudaError_t e = pab::launch_cross(q, kt, vt, out, R, Lt, heads, d, s);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "cross attention launch");
}

}  // namespace

namespace pab {
int report_error(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int device_sm_count() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}
}  // namespace pab

// ============================================================== plan
struct pab_plan {
    int T, H, W, N, heads, d, text_len, steps, dtype;
    long long C;
    int range[3];
    int edge_pct, lo, hi;
    int temporal_sv;  // temporal attention takes / returns the spatial view
    int sta_win_h, sta_win_w;  // > 0: spatial computes are sliding tile attention (16-token tiles)
    int draft_keep;            // > 0: spatial computes are draft attention (16 x 16 regions)
    int* draft_sel;            // [T][heads][R][draft_keep]
    void* draft_sketch;
    size_t draft_sel_bytes, draft_sketch_bytes;
    // cache
    int device;
    void* slot[3][2];
    size_t slot_bytes[3];
    int cur[3];          // slot holding the latest computed output, -1 = none
    int cached_step[3];  // step of that compute
    int last_step[3];    // last step seen (order check)
    // attention-difference MSE of consecutive computes, written to the
    // caller's device array [3][steps]; fp64 scratch: ticket + partials
    double* mse_results;
    double* mse_scratch;
    // optional side stream for those MSE launches: the compute stream records
    // ev_done for the side stream to wait on; ev_mse[kind] marks the kind's
    // latest MSE, which the kind's next compute (it overwrites the slot the
    // MSE reads) waits for while mse_pending[kind] is set
    int mse_on_stream;
    cudaStream_t mse_stream;
    cudaEvent_t ev_done;
    cudaEvent_t ev_mse[3];
    int mse_pending[3];
    // bf16 staging for fp32 plans
    void* stage_in[3];
    void* stage_out;
    size_t stage_in_bytes, stage_out_bytes;
};

namespace {

bool sched_compute(const pab_plan* p, int kind, int i) {
    if (i < p->lo || i >= p->hi) return true;
    return ((i - p->lo) % p->range[kind]) == 0;
}
int sched_source(const pab_plan* p, int kind, int i) {
    if (sched_compute(p, kind, i)) return i;
    return p->lo + ((i - p->lo) / p->range[kind]) * p->range[kind];
}

// Let every side-stream MSE finish (it reads the slots) and release the events.
void plan_free_events(pab_plan* p) {
    for (int k = 0; k < 3; ++k) {
        if (p->mse_pending[k] && p->ev_mse[k]) cudaEventSynchronize(p->ev_mse[k]);
        p->mse_pending[k] = 0;
        if (p->ev_mse[k]) cudaEventDestroy(p->ev_mse[k]);
        p->ev_mse[k] = nullptr;
    }
    if (p->ev_done) cudaEventDestroy(p->ev_done);
    p->ev_done = nullptr;
}

void plan_free_device(pab_plan* p) {
    for (int k = 0; k < 3; ++k)
        for (int j = 0; j < 2; ++j) {
            if (p->slot[k][j]) cudaFree(p->slot[k][j]);
            p->slot[k][j] = nullptr;
        }
    for (int j = 0; j < 3; ++j) {
        if (p->stage_in[j]) cudaFree(p->stage_in[j]);
        p->stage_in[j] = nullptr;
    }
    if (p->stage_out) cudaFree(p->stage_out);
    p->stage_out = nullptr;
    if (p->draft_sel) cudaFree(p->draft_sel);
    if (p->draft_sketch) cudaFree(p->draft_sketch);
    if (p->mse_scratch) cudaFree(p->mse_scratch);
    p->mse_scratch = nullptr;
    p->draft_sel = nullptr;
    p->draft_sketch = nullptr;
    p->device = -1;
}

int plan_alloc_kind(pab_plan* p, int kind) {
    int dev;
    int rc = current_device(&dev);
    if (rc) return rc;
    if (p->device >= 0 && p->device != dev)
        return fail(PAB_ERR_ARG, "plan's cache lives on device %d, current device is %d", p->device, dev);
    p->device = dev;
    for (int j = 0; j < 2; ++j)
        if (!p->slot[kind][j] && p->slot_bytes[kind] > 0) {
            cudaError_t e = cudaMalloc(&p->slot[kind][j], p->slot_bytes[kind]);
            if (e != cudaSuccess) return cuda_fail(e, "broadcast cache allocation");
        }
    if (kind == PAB_SPATIAL && p->draft_keep > 0) {
        if (!p->draft_sel) {
            cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&p->draft_sel), p->draft_sel_bytes);
            if (e != cudaSuccess) return cuda_fail(e, "draft selection allocation");
        }
        if (!p->draft_sketch) {
            cudaError_t e = cudaMalloc(&p->draft_sketch, p->draft_sketch_bytes);
            if (e != cudaSuccess) return cuda_fail(e, "draft sketch allocation");
        }
    }
    if (p->dtype == PAB_FP32) {
        for (int j = 0; j < 3; ++j)
            if (!p->stage_in[j] && p->stage_in_bytes > 0) {
                cudaError_t e = cudaMalloc(&p->stage_in[j], p->stage_in_bytes);
                if (e != cudaSuccess) return cuda_fail(e, "bf16 staging allocation");
            }
        if (!p->stage_out && p->stage_out_bytes > 0) {
            cudaError_t e = cudaMalloc(&p->stage_out, p->stage_out_bytes);
            if (e != cudaSuccess) return cuda_fail(e, "bf16 staging allocation");
        }
    }
    return PAB_OK;
}

int plan_compute(pab_plan* p, int kind, const void* q, const void* k, const void* v, void* out,
                 cudaStream_t s) {
    const long long qn = (long long)p->T * p->N * p->C;
    const long long kvn = (kind == PAB_CROSS) ? (long long)p->text_len * p->C : qn;
    const void *qq = q, *kk = k, *vv = v;
    void* oo = out;
    if (p->dtype == PAB_FP32) {
        const float* src[3] = {static_cast<const float*>(q), static_cast<const float*>(k),
                               static_cast<const float*>(v)};
        const long long cnt[3] = {qn, kvn, kvn};
        for (int j = 0; j < 3; ++j) {
            cudaError_t e = pab::launch_f32_to_bf16(src[j], p->stage_in[j], cnt[j], s);
            if (e != cudaSuccess) return cuda_fail(e, "fp32 -> bf16 conversion");
        }
        qq = p->stage_in[0];
        kk = p->stage_in[1];
        vv = p->stage_in[2];
        oo = p->stage_out;
    }
    int rc;
    if (kind == PAB_SPATIAL && p->draft_keep > 0)
        rc = run_draft(qq, kk, vv, oo, p->T, p->H, p->W, p->heads, p->d, p->draft_keep, p->draft_sel,
                       p->draft_sketch, s);
    else if (kind == PAB_SPATIAL && p->sta_win_h > 0)
        rc = run_sta(qq, kk, vv, oo, p->T, p->H, p->W, p->heads, p->d, p->sta_win_h, p->sta_win_w, s);
    else if (kind == PAB_SPATIAL)
        rc = run_spatial(qq, kk, vv, oo, p->T, p->N, p->heads, p->d, s);
    else if (kind == PAB_TEMPORAL)
        rc = run_temporal(qq, kk, vv, oo, p->N, p->T, p->heads, p->d, p->temporal_sv, s);
    else
        rc = run_cross(qq, kk, vv, oo, (long long)p->T * p->N, p->text_len, p->heads, p->d, s);
    if (rc) return rc;
    if (p->dtype == PAB_FP32) {
        cudaError_t e = pab::launch_bf16_to_f32(p->stage_out, static_cast<float*>(out), qn, s);
        if (e != cudaSuccess) return cuda_fail(e, "bf16 -> fp32 conversion");
    }
    return PAB_OK;
}

}  // namespace

#define PAB_GUARD_BEGIN try {
#define PAB_GUARD_END                                                   \
    }                                                                   \
    catch (const std::bad_alloc&) {                                     \
        return fail(PAB_ERR_OOM, "host allocation failed");             \
    }                                                                   \
    catch (...) {                                                       \
        return fail(PAB_ERR_ARG, "unexpected host exception");          \
    }

extern "C" {

int pab_version(void) { return (0 << 16) | 2; }  // 0.2: sliding tile, draft attention, block permute

const char* pab_last_error_string(void) { return g_last_error.c_str(); }

int pab_spatial_attention(const void* q, const void* k, const void* v, void* out, int T, int N,
                          int heads, int d, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || N < 0) return fail(PAB_ERR_ARG, "T (%d) and N (%d) must be >= 0", T, N);
    if ((long long)T * N == 0) return PAB_OK;
    if (T > 65535) return fail(PAB_ERR_UNSUPPORTED, "T=%d frames exceeds 65535", T);
    rc = check_ptrs("q, k, v, out", q, k, v, out);
    if (rc) return rc;
    return run_spatial(q, k, v, out, T, N, heads, d, static_cast<cudaStream_t>(cuda_stream));
    PAB_GUARD_END
}

int pab_sta_attention(const void* q, const void* k, const void* v, void* out, int T, int H, int W,
                      int heads, int d, int tile, int win_h, int win_w, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || H < 0 || W < 0) return fail(PAB_ERR_ARG, "T, H, W must be >= 0 (got %d, %d, %d)", T, H, W);
    rc = check_sta(H, W, tile, win_h, win_w);
    if (rc) return rc;
    if ((long long)T * H * W == 0) return PAB_OK;
    if (T > 65535) return fail(PAB_ERR_UNSUPPORTED, "T=%d frames exceeds 65535", T);
    if ((long long)H * W > (1LL << 30)) return fail(PAB_ERR_UNSUPPORTED, "H*W too large");
    rc = check_ptrs("q, k, v, out", q, k, v, out);
    if (rc) return rc;
    return run_sta(q, k, v, out, T, H, W, heads, d, win_h, win_w, static_cast<cudaStream_t>(cuda_stream));
    PAB_GUARD_END
}

int pab_draft_workspace_bytes(int T, int H, int W, int heads, int d, int region, long long* bytes) {
    if (!bytes) return fail(PAB_ERR_ARG, "null bytes");
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || H < 0 || W < 0) return fail(PAB_ERR_ARG, "T, H, W must be >= 0 (got %d, %d, %d)", T, H, W);
    rc = check_draft(H, W, region, 1);
    if (rc && H * W > 0) return rc;
    *bytes = (long long)pab::draft_sketch_bytes(T, H, W, heads, d);
    return PAB_OK;
}

int pab_draft_select(const void* q, const void* k, int T, int H, int W, int heads, int d, int region, int keep,
                     int* sel, void* workspace, long long workspace_bytes, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || H < 0 || W < 0) return fail(PAB_ERR_ARG, "T, H, W must be >= 0 (got %d, %d, %d)", T, H, W);
    if ((long long)T * H * W == 0) return PAB_OK;
    rc = check_draft(H, W, region, keep);
    if (rc) return rc;
    if (T > 65535) return fail(PAB_ERR_UNSUPPORTED, "T=%d frames exceeds 65535", T);
    rc = check_ptrs("q, k, sel, workspace", q, k, sel, workspace);
    if (rc) return rc;
    if (workspace_bytes < (long long)pab::draft_sketch_bytes(T, H, W, heads, d))
        return fail(PAB_ERR_ARG, "workspace of %lld bytes is smaller than %lld", workspace_bytes,
                    (long long)pab::draft_sketch_bytes(T, H, W, heads, d));
    cudaError_t e = pab::launch_draft_select(q, k, T, H, W, heads, d, keep, sel, workspace,
                                             static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "draft selection launch");
    PAB_GUARD_END
}

int pab_region_sparse_attention(const void* q, const void* k, const void* v, void* out, int T, int H, int W,
                                int heads, int d, int region, int keep, const int* sel, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || H < 0 || W < 0) return fail(PAB_ERR_ARG, "T, H, W must be >= 0 (got %d, %d, %d)", T, H, W);
    if ((long long)T * H * W == 0) return PAB_OK;
    rc = check_draft(H, W, region, keep);
    if (rc) return rc;
    if (T > 65535) return fail(PAB_ERR_UNSUPPORTED, "T=%d frames exceeds 65535", T);
    rc = check_ptrs("q, k, v, out", q, k, v, out);
    if (rc) return rc;
    if (!sel) return fail(PAB_ERR_ARG, "null selection");
    cudaError_t e = pab::launch_flash_tile_list(q, k, v, out, T, H, W, heads, d, sel, keep,
                                                static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "region-sparse attention launch");
    PAB_GUARD_END
}

int pab_temporal_attention(const void* q, const void* k, const void* v, void* out, int N, int T,
                           int heads, int d, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || N < 0) return fail(PAB_ERR_ARG, "T (%d) and N (%d) must be >= 0", T, N);
    if (T > 128) return fail(PAB_ERR_UNSUPPORTED, "temporal length T=%d exceeds 128", T);
    if ((long long)T * N == 0) return PAB_OK;
    rc = check_ptrs("q, k, v, out", q, k, v, out);
    if (rc) return rc;
    return run_temporal(q, k, v, out, N, T, heads, d, 0, static_cast<cudaStream_t>(cuda_stream));
    PAB_GUARD_END
}

int pab_temporal_attention_sv(const void* q, const void* k, const void* v, void* out, int T, int N,
                              int heads, int d, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (T < 0 || N < 0) return fail(PAB_ERR_ARG, "T (%d) and N (%d) must be >= 0", T, N);
    if (T > 128) return fail(PAB_ERR_UNSUPPORTED, "temporal length T=%d exceeds 128", T);
    if ((long long)T * N == 0) return PAB_OK;
    rc = check_ptrs("q, k, v, out", q, k, v, out);
    if (rc) return rc;
    return run_temporal(q, k, v, out, N, T, heads, d, 1, static_cast<cudaStream_t>(cuda_stream));
    PAB_GUARD_END
}

int pab_cross_attention(const void* q, const void* kt, const void* vt, void* out, long long R,
                        int text_len, int heads, int d, void* cuda_stream) {
    PAB_GUARD_BEGIN
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (R < 0) return fail(PAB_ERR_ARG, "R=%lld must be >= 0", R);
    if (text_len < 1 || text_len > 512)
        return fail(PAB_ERR_UNSUPPORTED, "text_len=%d outside [1, 512]", text_len);
    if (R == 0) return PAB_OK;
    rc = check_ptrs("q, kt, vt, out", q, kt, vt, out);
    if (rc) return rc;
    return run_cross(q, kt, vt, out, R, text_len, heads, d, static_cast<cudaStream_t>(cuda_stream));
    PAB_GUARD_END
}

int pab_layout(int to_temporal, const void* src, void* dst, int T, int N, int C, int dtype,
               void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (T < 0 || N < 0 || C < 0) return fail(PAB_ERR_ARG, "negative size");
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const long long row = (long long)C * elem;
    if ((long long)T * N * C == 0) return PAB_OK;
    if (row % 16 != 0) return fail(PAB_ERR_UNSUPPORTED, "row of %lld bytes is not a multiple of 16", row);
    if (row > 48 * 1024) return fail(PAB_ERR_UNSUPPORTED, "row of %lld bytes exceeds 48 KiB", row);
    if (!src || !dst) return fail(PAB_ERR_ARG, "null src/dst");
    if (!aligned16(src) || !aligned16(dst)) return fail(PAB_ERR_ARG, "src/dst not 16-byte aligned");
    const char* s0 = static_cast<const char*>(src);
    const char* d0 = static_cast<const char*>(dst);
    const long long bytes = (long long)T * N * row;
    if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(PAB_ERR_ARG, "src and dst overlap");
    cudaError_t e = pab::launch_layout(to_temporal ? 1 : 0, src, dst, T, N, (int)row,
                                       static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "layout launch");
    PAB_GUARD_END
}

int pab_permute_blocks(const void* src, void* dst, int P, int Q, long long block_rows, int C, int dtype,
                       void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (P < 0 || Q < 0 || block_rows < 0 || C < 0) return fail(PAB_ERR_ARG, "negative size");
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const long long row = (long long)C * elem;
    if ((long long)P * Q * block_rows * C == 0) return PAB_OK;
    if (row % 16 != 0) return fail(PAB_ERR_UNSUPPORTED, "row of %lld bytes is not a multiple of 16", row);
    if (row > 48 * 1024) return fail(PAB_ERR_UNSUPPORTED, "row of %lld bytes exceeds 48 KiB", row);
    if (!src || !dst) return fail(PAB_ERR_ARG, "null src/dst");
    if (!aligned16(src) || !aligned16(dst)) return fail(PAB_ERR_ARG, "src/dst not 16-byte aligned");
    const char* s0 = static_cast<const char*>(src);
    const char* d0 = static_cast<const char*>(dst);
    const long long bytes = (long long)P * Q * block_rows * row;
    if (s0 < d0 + bytes && d0 < s0 + bytes) return fail(PAB_ERR_ARG, "src and dst overlap");
    cudaError_t e = pab::launch_swap_outer(src, dst, P, Q, block_rows, (int)row,
                                           static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "block permute launch");
    PAB_GUARD_END
}

int pab_scatter_blocks(const void* const* src, void* const* dst, int ntensors, int G, int P,
                       long long block_rows, int C, int src_order, long long dst_offset_rows,
                       long long dst_stride_rows, int dtype, void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (ntensors < 1 || ntensors > pab::kScatterMaxTensors)
        return fail(PAB_ERR_ARG, "ntensors=%d outside [1, %d]", ntensors, pab::kScatterMaxTensors);
    if (G < 1 || G > pab::kScatterMaxRanks) return fail(PAB_ERR_ARG, "G=%d outside [1, %d]", G, pab::kScatterMaxRanks);
    if (P < 0 || block_rows < 0 || C < 0 || dst_offset_rows < 0 || dst_stride_rows < 0)
        return fail(PAB_ERR_ARG, "negative size");
    if (src_order != 0 && src_order != 1) return fail(PAB_ERR_ARG, "src_order=%d must be 0 or 1", src_order);
    if ((long long)P * G > 65535) return fail(PAB_ERR_UNSUPPORTED, "P*G=%lld blocks exceed 65535", (long long)P * G);
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const long long row = (long long)C * elem;
    if ((long long)P * block_rows * C == 0) return PAB_OK;
    if (row % 16 != 0) return fail(PAB_ERR_UNSUPPORTED, "row of %lld bytes is not a multiple of 16", row);
    if (!src || !dst) return fail(PAB_ERR_ARG, "null pointer array");
    if (dst_stride_rows < block_rows && P > 1)
        return fail(PAB_ERR_ARG, "dst_stride_rows=%lld < block_rows=%lld: destination blocks overlap",
                    dst_stride_rows, block_rows);
    for (int t = 0; t < ntensors; ++t)
        if (!src[t] || !aligned16(src[t])) return fail(PAB_ERR_ARG, "src[%d] null or not 16-byte aligned", t);
    for (int i = 0; i < ntensors * G; ++i)
        if (!dst[i] || !aligned16(dst[i])) return fail(PAB_ERR_ARG, "dst[%d] null or not 16-byte aligned", i);
    // a destination buffer that overlaps a source of the same call
    const long long src_bytes = (long long)P * G * block_rows * row;
    const long long dst_bytes = ((dst_offset_rows + (long long)(P - 1) * dst_stride_rows) + block_rows) * row;
    for (int t = 0; t < ntensors; ++t)
        for (int i = 0; i < ntensors * G; ++i) {
            const char* s0 = static_cast<const char*>(src[t]);
            const char* d0 = static_cast<const char*>(dst[i]);
            if (s0 < d0 + dst_bytes && d0 < s0 + src_bytes)
                return fail(PAB_ERR_ARG, "src[%d] and dst[%d] overlap", t, i);
        }
    cudaError_t e = pab::launch_scatter_blocks(src, dst, ntensors, G, P, block_rows, (int)row, src_order,
                                               dst_offset_rows, dst_stride_rows,
                                               static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "block scatter launch");
    PAB_GUARD_END
}

int pab_ipc_alloc(long long bytes, void** ptr, unsigned char handle[64]) {
    PAB_GUARD_BEGIN
    if (!ptr || !handle) return fail(PAB_ERR_ARG, "null output pointer");
    *ptr = nullptr;
    if (bytes <= 0) return fail(PAB_ERR_ARG, "bytes=%lld must be positive", bytes);
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, (size_t)bytes);
    if (e != cudaSuccess) return cuda_fail(e, "IPC buffer allocation");
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, p);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "cudaIpcGetMemHandle");
    }
    static_assert(sizeof(cudaIpcMemHandle_t) == 64, "CUDA IPC handles are 64 bytes");
    memcpy(handle, &h, 64);
    *ptr = p;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_ipc_free(void* ptr) {
    if (!ptr) return PAB_OK;
    cudaError_t e = cudaFree(ptr);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "IPC buffer free");
}

int pab_ipc_open(const unsigned char handle[64], void** ptr) {
    PAB_GUARD_BEGIN
    if (!ptr || !handle) return fail(PAB_ERR_ARG, "null pointer");
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, 64);
    void* p = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
    *ptr = p;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_ipc_close(void* ptr) {
    if (!ptr) return PAB_OK;
    cudaError_t e = cudaIpcCloseMemHandle(ptr);
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "cudaIpcCloseMemHandle");
}

int pab_block_gemm(const void* A, const void* B, int M, int N, int K, int epilogue, void* const* out, int split,
                   float* X, void* Y, void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (M < 0 || N < 0 || K < 0) return fail(PAB_ERR_ARG, "negative size");
    if (epilogue < 0 || epilogue > 2) return fail(PAB_ERR_ARG, "bad epilogue %d", epilogue);
    if ((long long)M * N == 0) return PAB_OK;
    if (K == 0 || K % 8) return fail(PAB_ERR_UNSUPPORTED, "K=%d must be a positive multiple of 8", K);
    if (N % 32) return fail(PAB_ERR_UNSUPPORTED, "N=%d must be a multiple of 32", N);
    if (!A || !B || !aligned16(A) || !aligned16(B)) return fail(PAB_ERR_ARG, "A/B null or not 16-byte aligned");
    if (epilogue == 2) {
        if (!X || !aligned16(X)) return fail(PAB_ERR_ARG, "X null or not 16-byte aligned");
        if (Y && !aligned16(Y)) return fail(PAB_ERR_ARG, "Y not 16-byte aligned");
    } else {
        const int sp = split > 0 ? split : N;
        if (sp % 32 || N % sp || N / sp > 3)
            return fail(PAB_ERR_ARG, "split=%d must divide N=%d into at most 3 outputs of a multiple of 32", split, N);
        if (epilogue == 1 && sp != N) return fail(PAB_ERR_ARG, "the GELU epilogue has one output");
        if (!out) return fail(PAB_ERR_ARG, "null output array");
        for (int i = 0; i < N / sp; ++i)
            if (!out[i] || !aligned16(out[i])) return fail(PAB_ERR_ARG, "out[%d] null or not 16-byte aligned", i);
    }
    cudaError_t e = pab::launch_gemm(A, B, M, N, K, epilogue, out, split, X, Y, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "block GEMM launch");
    PAB_GUARD_END
}

int pab_block_layer_norm(float* x, const void* const* ys, int ny, void* h, long long rows, int C,
                         void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (rows < 0 || C <= 0) return fail(PAB_ERR_ARG, "rows=%lld, C=%d", rows, C);
    if (ny < 0 || ny > 3 || (ny > 0 && !ys)) return fail(PAB_ERR_ARG, "ny=%d outside [0, 3] or null array", ny);
    if (rows == 0) return PAB_OK;
    if (C % 8 || C > 3072) return fail(PAB_ERR_UNSUPPORTED, "C=%d must be a multiple of 8, at most 3072", C);
    if (!x || !aligned16(x) || (h && !aligned16(h))) return fail(PAB_ERR_ARG, "null or misaligned pointer");
    for (int j = 0; j < ny; ++j)
        if (!ys[j] || !aligned16(ys[j])) return fail(PAB_ERR_ARG, "ys[%d] null or not 16-byte aligned", j);
    cudaError_t e = pab::launch_ln_rows(x, ys, ny, h, rows, C, 1e-6f, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "layer norm launch");
    PAB_GUARD_END
}

int pab_attn_diff_mse_async(const void* a, const void* b, long long n, int dtype, double* result_dev,
                            void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (n < 0) return fail(PAB_ERR_ARG, "n=%lld must be >= 0", n);
    if (!result_dev || (reinterpret_cast<uintptr_t>(result_dev) & 7u))
        return fail(PAB_ERR_ARG, "result_dev null or not 8-byte aligned");
    if (n > 0 && (!a || !b)) return fail(PAB_ERR_ARG, "null input");
    if (n > 0 && (!aligned16(a) || !aligned16(b))) return fail(PAB_ERR_ARG, "inputs not 16-byte aligned");
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const int parts = pab::mse_num_partials(n, elem);
    double* scratch = nullptr;
    int rc = mse_scratch(parts + 1, &scratch, static_cast<cudaStream_t>(cuda_stream));
    if (rc) return rc;
    cudaError_t e = pab::launch_mse(a, b, n, dtype, scratch, parts, result_dev,
                                    static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? PAB_OK : cuda_fail(e, "MSE launch");
    PAB_GUARD_END
}

int pab_attn_diff_mse(const void* a, const void* b, long long n, int dtype, double* result,
                      void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (!result) return fail(PAB_ERR_ARG, "null result pointer");
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (n < 0) return fail(PAB_ERR_ARG, "n=%lld must be >= 0", n);
    if (n > 0 && (!a || !b)) return fail(PAB_ERR_ARG, "null input");
    if (n > 0 && (!aligned16(a) || !aligned16(b))) return fail(PAB_ERR_ARG, "inputs not 16-byte aligned");
    const int elem = dtype == PAB_FP32 ? 4 : 2;
    const int parts = pab::mse_num_partials(n, elem);
    double* scratch = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    int rc = mse_scratch(parts + 2, &scratch, s);
    if (rc) return rc;
    double* result_dev = scratch + 1 + parts;
    cudaError_t e = pab::launch_mse(a, b, n, dtype, scratch, parts, result_dev, s);
    if (e != cudaSuccess) return cuda_fail(e, "MSE launch");
    e = cudaMemcpyAsync(result, result_dev, sizeof(double), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "MSE result copy");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "MSE stream synchronise");
    return PAB_OK;
    PAB_GUARD_END
}

int pab_device_errors(int clear, unsigned int* flags) {
    PAB_GUARD_BEGIN
    if (!flags) return fail(PAB_ERR_ARG, "null flags pointer");
    const unsigned int words[5] = {pab::layout_device_errors(clear != 0), pab::flash_device_errors(clear != 0),
                                   pab::temporal_device_errors(clear != 0), pab::cross_device_errors(clear != 0),
                                   pab::block_device_errors(clear != 0)};
    unsigned int v = 0;
    for (unsigned int w : words) {
        if (w == 0xffffffffu) return fail(PAB_ERR_CUDA, "could not read the device status words");
        v |= w;
    }
    *flags = v;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_plan_create(int T, int H, int W, int heads, int d, int text_len, int steps,
                    pab_ranges ranges, int dtype, pab_plan** out_plan) {
    PAB_GUARD_BEGIN
    if (!out_plan) return fail(PAB_ERR_ARG, "null out_plan");
    *out_plan = nullptr;
    if (T < 1 || H < 1 || W < 1) return fail(PAB_ERR_ARG, "T, H, W must be >= 1 (got %d, %d, %d)", T, H, W);
    if (steps < 1) return fail(PAB_ERR_ARG, "steps=%d must be >= 1", steps);
    int rc = check_dims(heads, d);
    if (rc) return rc;
    if (text_len < 1 || text_len > 512) return fail(PAB_ERR_UNSUPPORTED, "text_len=%d outside [1, 512]", text_len);
    if (T > 128) return fail(PAB_ERR_UNSUPPORTED, "T=%d frames exceeds the temporal limit 128", T);
    if (dtype != PAB_BF16 && dtype != PAB_FP32) return fail(PAB_ERR_ARG, "bad dtype %d", dtype);
    if (ranges.spatial < 1 || ranges.temporal < 1 || ranges.cross < 1)
        return fail(PAB_ERR_ARG, "broadcast ranges must be >= 1 (got %d, %d, %d)", ranges.spatial,
                    ranges.temporal, ranges.cross);
    // a negative edge share selects the pages' 15%; 0 means no edge steps
    const int edge = ranges.edge_pct < 0 ? 15 : ranges.edge_pct;
    if (edge > 50) return fail(PAB_ERR_ARG, "edge_pct=%d outside [0, 50] (negative: 15)", ranges.edge_pct);
    const long long N = (long long)H * W;
    if (N > (1LL << 30)) return fail(PAB_ERR_UNSUPPORTED, "H*W too large");
    pab_plan* p = new pab_plan;
    memset(p, 0, sizeof(*p));
    p->T = T;
    p->H = H;
    p->W = W;
    p->N = (int)N;
    p->heads = heads;
    p->d = d;
    p->C = (long long)heads * d;
    p->text_len = text_len;
    p->steps = steps;
    p->dtype = dtype;
    p->range[PAB_SPATIAL] = ranges.spatial;
    p->range[PAB_TEMPORAL] = ranges.temporal;
    p->range[PAB_CROSS] = ranges.cross;
    p->edge_pct = edge;
    const int e = (edge * steps + 99) / 100;
    p->lo = e;
    p->hi = steps - e;
    p->device = -1;
    const size_t elem = dtype == PAB_FP32 ? 4 : 2;
    const size_t video = (size_t)T * N * p->C;
    for (int k = 0; k < 3; ++k) {
        p->slot_bytes[k] = video * elem;
        p->cur[k] = -1;
        p->cached_step[k] = -1;
        p->last_step[k] = -1;
    }
    p->stage_in_bytes = video * 2;
    p->stage_out_bytes = video * 2;
    *out_plan = p;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_plan_destroy(pab_plan* plan) {
    if (!plan) return PAB_OK;
    plan_free_events(plan);
    plan_free_device(plan);
    delete plan;
    return PAB_OK;
}

int pab_plan_reset(pab_plan* plan) {
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    for (int k = 0; k < 3; ++k) {
        plan->cur[k] = -1;
        plan->cached_step[k] = -1;
        plan->last_step[k] = -1;
    }
    return PAB_OK;
}

int pab_plan_set_temporal_view(pab_plan* plan, int spatial_view) {
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    if (spatial_view != 0 && spatial_view != 1) return fail(PAB_ERR_ARG, "spatial_view must be 0 or 1");
    plan->temporal_sv = spatial_view;
    return PAB_OK;
}

int pab_plan_set_spatial_window(pab_plan* plan, int tile, int win_h, int win_w) {
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    if (win_h == 0 && win_w == 0) {
        plan->sta_win_h = plan->sta_win_w = 0;
        return PAB_OK;
    }
    int rc = check_sta(plan->H, plan->W, tile, win_h, win_w);
    if (rc) return rc;
    plan->sta_win_h = win_h;
    plan->sta_win_w = win_w;
    plan->draft_keep = 0;
    return PAB_OK;
}

int pab_plan_set_spatial_draft(pab_plan* plan, int region, int keep) {
    PAB_GUARD_BEGIN
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    if (keep == 0) {
        plan->draft_keep = 0;
        return PAB_OK;
    }
    int rc = check_draft(plan->H, plan->W, region, keep);
    if (rc) return rc;
    const long long R = (long long)(plan->H / region) * (plan->W / region);
    const size_t sel_bytes = (size_t)plan->T * plan->heads * R * keep * sizeof(int);
    if (plan->draft_sel && sel_bytes > plan->draft_sel_bytes) {  // a larger keep: reallocate on next use
        cudaFree(plan->draft_sel);
        plan->draft_sel = nullptr;
    }
    if (!plan->draft_sel) plan->draft_sel_bytes = sel_bytes;
    plan->draft_sketch_bytes = pab::draft_sketch_bytes(plan->T, plan->H, plan->W, plan->heads, plan->d);
    plan->draft_keep = keep;
    plan->sta_win_h = plan->sta_win_w = 0;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_plan_set_diff_mse(pab_plan* plan, double* results_dev) {
    PAB_GUARD_BEGIN
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    if (results_dev && (reinterpret_cast<uintptr_t>(results_dev) & 7u))
        return fail(PAB_ERR_ARG, "results_dev not 8-byte aligned");
    if (results_dev && !plan->mse_scratch) {
        // the completion ticket and the most partial sums one MSE launch takes
        const int need = pab::mse_num_partials(1LL << 40, 2) + 1;
        cudaError_t e = cudaMalloc(&plan->mse_scratch, sizeof(double) * need);
        if (e != cudaSuccess) {
            plan->mse_scratch = nullptr;
            return cuda_fail(e, "MSE scratch allocation");
        }
        e = cudaMemset(plan->mse_scratch, 0, sizeof(unsigned long long));  // the ticket starts at zero
        if (e != cudaSuccess) return cuda_fail(e, "MSE scratch clear");
    }
    plan->mse_results = results_dev;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_plan_set_diff_mse_stream(pab_plan* plan, int enable, void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    if (enable != 0 && enable != 1) return fail(PAB_ERR_ARG, "enable must be 0 or 1");
    if (enable) {
        for (int k = 0; k < 4; ++k) {
            cudaEvent_t* ev = k < 3 ? &plan->ev_mse[k] : &plan->ev_done;
            if (*ev) continue;
            cudaError_t e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
            if (e != cudaSuccess) {
                *ev = nullptr;
                return cuda_fail(e, "MSE stream events");
            }
        }
        plan->mse_stream = static_cast<cudaStream_t>(cuda_stream);
    }
    plan->mse_on_stream = enable;
    return PAB_OK;
    PAB_GUARD_END
}

int pab_plan_prepare(pab_plan* plan) {
    PAB_GUARD_BEGIN
    if (!plan) return fail(PAB_ERR_ARG, "null plan");
    for (int k = 0; k < 3; ++k) {
        int rc = plan_alloc_kind(plan, k);
        if (rc) return rc;
    }
    return PAB_OK;
    PAB_GUARD_END
}

int pab_schedule_query(const pab_plan* plan, int kind, int step, int* is_compute) {
    if (!plan || !is_compute) return fail(PAB_ERR_ARG, "null argument");
    if (kind < 0 || kind > 2) return fail(PAB_ERR_ARG, "bad kind %d", kind);
    if (step < 0 || step >= plan->steps) return fail(PAB_ERR_ARG, "step %d outside [0, %d)", step, plan->steps);
    *is_compute = sched_compute(plan, kind, step) ? 1 : 0;
    return PAB_OK;
}

int pab_schedule_source(const pab_plan* plan, int kind, int step, int* source_step) {
    if (!plan || !source_step) return fail(PAB_ERR_ARG, "null argument");
    if (kind < 0 || kind > 2) return fail(PAB_ERR_ARG, "bad kind %d", kind);
    if (step < 0 || step >= plan->steps) return fail(PAB_ERR_ARG, "step %d outside [0, %d)", step, plan->steps);
    *source_step = sched_source(plan, kind, step);
    return PAB_OK;
}

int pab_schedule_count(const pab_plan* plan, int kind, int* computes) {
    if (!plan || !computes) return fail(PAB_ERR_ARG, "null argument");
    if (kind < 0 || kind > 2) return fail(PAB_ERR_ARG, "bad kind %d", kind);
    int c = 0;
    for (int i = 0; i < plan->steps; ++i) c += sched_compute(plan, kind, i) ? 1 : 0;
    *computes = c;
    return PAB_OK;
}

int pab_attention(pab_plan* plan, int kind, int step, const void* q, const void* k, const void* v,
                  const void** out, void* cuda_stream) {
    PAB_GUARD_BEGIN
    if (!plan || !out) return fail(PAB_ERR_ARG, "null plan or out");
    if (kind < 0 || kind > 2) return fail(PAB_ERR_ARG, "bad kind %d", kind);
    if (step < 0 || step >= plan->steps) return fail(PAB_ERR_ARG, "step %d outside [0, %d)", step, plan->steps);
    if (step <= plan->last_step[kind])
        return fail(PAB_ERR_STEP_ORDER, "kind %d: step %d after step %d", kind, step, plan->last_step[kind]);
    if (!sched_compute(plan, kind, step)) {
        const int src = sched_source(plan, kind, step);
        if (plan->cur[kind] < 0 || plan->cached_step[kind] != src)
            return fail(PAB_ERR_NO_CACHE, "kind %d step %d needs the output of step %d, which was not computed",
                        kind, step, src);
        plan->last_step[kind] = step;
        *out = plan->slot[kind][plan->cur[kind]];
        return PAB_OK;
    }
    int rc = check_ptrs("q, k, v", q, k, v, q);
    if (rc) return rc;
    rc = plan_alloc_kind(plan, kind);
    if (rc) return rc;
    const int slot = plan->cur[kind] < 0 ? 0 : 1 - plan->cur[kind];
    // the attention-difference MSE against the kind's previous compute of this run
    const void* prev = nullptr;
    double* mse_result = nullptr;
    if (plan->mse_results && plan->cur[kind] >= 0) {
        prev = plan->slot[kind][plan->cur[kind]];
        mse_result = plan->mse_results + (long long)kind * plan->steps + step;
    }
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    // the slot about to be written may still be read by this kind's latest
    // side-stream MSE
    if (plan->mse_pending[kind]) {
        cudaError_t e = cudaStreamWaitEvent(s, plan->ev_mse[kind], 0);
        if (e != cudaSuccess) return cuda_fail(e, "wait for the side-stream MSE");
        plan->mse_pending[kind] = 0;
    }
    rc = plan_compute(plan, kind, q, k, v, plan->slot[kind][slot], s);
    if (rc) return rc;
    if (prev) {
        // the difference to the kind's previous output, read back from HBM by
        // the MSE kernel: on the compute stream, or on the side stream once the
        // compute is done there (an inline launch first waits for every
        // side-stream MSE still pending: they share the plan's scratch)
        cudaStream_t ms = s;
        cudaError_t e = cudaSuccess;
        if (plan->mse_on_stream) {
            ms = plan->mse_stream;
            e = cudaEventRecord(plan->ev_done, s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(ms, plan->ev_done, 0);
        } else {
            for (int j = 0; j < 3 && e == cudaSuccess; ++j)
                if (plan->mse_pending[j]) {
                    e = cudaStreamWaitEvent(s, plan->ev_mse[j], 0);
                    plan->mse_pending[j] = 0;
                }
        }
        if (e != cudaSuccess) return cuda_fail(e, "MSE stream ordering");
        const long long qn = (long long)plan->T * plan->N * plan->C;
        const int parts = pab::mse_num_partials(qn, plan->dtype == PAB_FP32 ? 4 : 2);
        e = pab::launch_mse(plan->slot[kind][slot], prev, qn, plan->dtype, plan->mse_scratch, parts, mse_result,
                            ms);
        if (e != cudaSuccess) return cuda_fail(e, "attention-difference MSE launch");
        if (plan->mse_on_stream) {
            e = cudaEventRecord(plan->ev_mse[kind], ms);
            if (e != cudaSuccess) return cuda_fail(e, "side-stream MSE event");
            plan->mse_pending[kind] = 1;
        }
    }
    plan->cur[kind] = slot;
    plan->cached_step[kind] = step;
    plan->last_step[kind] = step;
    *out = plan->slot[kind][slot];
    return PAB_OK;
    PAB_GUARD_END
}

}  // extern "C"

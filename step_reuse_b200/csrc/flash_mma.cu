// flash_mma.cu -- flash (online-softmax) attention for the long-sequence
// PAB kinds: spatial attention (tokens of one frame, L = H*W) and cross
// attention (all video tokens against one shared set of text K/V) -- PAB
// report, "Implementation".  Warp-level bf16 MMA (m16n8k16) version.
//
// A CTA owns 128 query rows of one (batch, head); 8 warps own 16 rows each.
// K/V tiles of 64 keys stream through a cp.async double buffer; S = QK^T and
// O += PV run on warp MMA from ldmatrix fragments, the online softmax keeps
// the running max / sum per row in registers.  Keys past Lk are masked to
// -inf; query rows past Lq are loaded as zeros and never stored.
#include "common.cuh"
#include "kernels.h"

namespace pab {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 64;   // keys per tile
constexpr float kLog2e = 1.4426950408889634f;

struct FlashArgs {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    __nv_bfloat16* out;
    long long Lq;
    int Lk, heads, d, P;
    long long C;
    long long q_bstride, kv_bstride;
    float scale_log2;
};

PAB_DEV float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int DN>
__global__ void __launch_bounds__(kThreads) flash_mma_kernel(FlashArgs p) {
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int DK = (DN + 1) / 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = p.P, d = p.d;
    const int h = blockIdx.y, b = blockIdx.z;
    const long long q0 = (long long)blockIdx.x * kBM;
    const int chunks = d / 8;

    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem);
    __nv_bfloat16* ks = qs + kBM * P;            // [2][kBN][P]
    __nv_bfloat16* vs = ks + 2 * kBN * P;        // [2][kBN][P]
    const int total_elems = kBM * P + 4 * kBN * P;

    // zero everything once (padding columns stay zero)
    {
        uint4* z = reinterpret_cast<uint4*>(smem);
        const int n16 = (total_elems * 2 + 256) / 16;
        for (int i = tid; i < n16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    const __nv_bfloat16* qg = p.q + b * p.q_bstride + (long long)h * d;
    const __nv_bfloat16* kg = p.k + b * p.kv_bstride + (long long)h * d;
    const __nv_bfloat16* vg = p.v + b * p.kv_bstride + (long long)h * d;

    // Q tile (rows past Lq zero-filled)
    for (int c = tid; c < kBM * chunks; c += kThreads) {
        const int r = c / chunks, ch = c - r * chunks;
        const long long row = q0 + r;
        const bool ok = row < p.Lq;
        cp_async16(smem_u32(qs + r * P + ch * 8), qg + (ok ? row : 0) * p.C + ch * 8, ok ? 16 : 0);
    }
    auto load_kv = [&](int kb, int buf) {
        for (int c = tid; c < 2 * kBN * chunks; c += kThreads) {
            const int which = c / (kBN * chunks);
            const int rr = c - which * (kBN * chunks);
            const int r = rr / chunks, ch = rr - r * chunks;
            const int key = kb * kBN + r;
            const bool ok = key < p.Lk;
            const __nv_bfloat16* src = (which ? vg : kg) + (long long)(ok ? key : 0) * p.C + ch * 8;
            __nv_bfloat16* dst = (which ? vs : ks) + (buf * kBN + r) * P + ch * 8;
            cp_async16(smem_u32(dst), src, ok ? 16 : 0);
        }
    };
    load_kv(0, 0);
    cp_async_commit();

    const int nkb = (p.Lk + kBN - 1) / kBN;
    uint32_t qa[DK][4];
    float o[DN][4];
#pragma unroll
    for (int j = 0; j < DN; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const __nv_bfloat16* qw = qs + warp * 16 * P;

    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) load_kv(kb + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (kb == 0) {
#pragma unroll
            for (int kc = 0; kc < DK; ++kc)
                ldsm_x4(smem_u32(qw + (lane & 15) * P + kc * 16 + (lane >> 4) * 8), qa[kc][0],
                        qa[kc][1], qa[kc][2], qa[kc][3]);
            if (DN & 1) {
                qa[DK - 1][2] = 0u;
                qa[DK - 1][3] = 0u;
            }
        }
        const __nv_bfloat16* kt = ks + buf * kBN * P;
        const __nv_bfloat16* vt = vs + buf * kBN * P;
        float s[kBN / 8][4];
#pragma unroll
        for (int j = 0; j < kBN / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int kc = 0; kc < DK; ++kc) {
#pragma unroll
            for (int jj = 0; jj < kBN / 16; ++jj) {
                uint32_t b0, b1, b2, b3;
                const int krow = jj * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int kcol = kc * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4(smem_u32(kt + krow * P + kcol), b0, b1, b2, b3);
                mma_bf16_16816(s[2 * jj], qa[kc][0], qa[kc][1], qa[kc][2], qa[kc][3], b0, b1);
                mma_bf16_16816(s[2 * jj + 1], qa[kc][0], qa[kc][1], qa[kc][2], qa[kc][3], b2, b3);
            }
        }
        float mx0 = m0, mx1 = m1;
        const bool tail = (kb + 1) * kBN > p.Lk;
#pragma unroll
        for (int j = 0; j < kBN / 8; ++j) {
            const int key = kb * kBN + j * 8 + 2 * (lane & 3);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool valid = !tail || (key + e) < p.Lk;
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
        for (int j = 0; j < kBN / 8; ++j) {
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
#pragma unroll
        for (int kc = 0; kc < kBN / 16; ++kc) {
            const uint32_t pa0 = pack_bf16x2(s[2 * kc][0], s[2 * kc][1]);
            const uint32_t pa1 = pack_bf16x2(s[2 * kc][2], s[2 * kc][3]);
            const uint32_t pa2 = pack_bf16x2(s[2 * kc + 1][0], s[2 * kc + 1][1]);
            const uint32_t pa3 = pack_bf16x2(s[2 * kc + 1][2], s[2 * kc + 1][3]);
            const int vrow = kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int j = 0; j < DN; j += 2) {
                if (j + 1 < DN) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(smem_u32(vt + vrow * P + j * 8 + (lane >> 4) * 8), b0, b1, b2, b3);
                    mma_bf16_16816(o[j], pa0, pa1, pa2, pa3, b0, b1);
                    mma_bf16_16816(o[j + 1], pa0, pa1, pa2, pa3, b2, b3);
                } else {
                    uint32_t b0, b1;
                    ldsm_x2_t(smem_u32(vt + vrow * P + j * 8), b0, b1);
                    mma_bf16_16816(o[j], pa0, pa1, pa2, pa3, b0, b1);
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    l0 = quad_sum(l0);
    l1 = quad_sum(l1);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    __nv_bfloat16* ow = qs + warp * 16 * P;
    const int r0 = lane >> 2, cq = 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < DN; ++j) {
        *reinterpret_cast<uint32_t*>(ow + r0 * P + j * 8 + cq) = pack_bf16x2(o[j][0] * inv0, o[j][1] * inv0);
        *reinterpret_cast<uint32_t*>(ow + (r0 + 8) * P + j * 8 + cq) =
            pack_bf16x2(o[j][2] * inv1, o[j][3] * inv1);
    }
    __syncthreads();
    __nv_bfloat16* og = p.out + b * p.q_bstride + (long long)h * d;
    for (int c = tid; c < kBM * chunks; c += kThreads) {
        const int r = c / chunks, ch = c - r * chunks;
        const long long row = q0 + r;
        if (row < p.Lq)
            __stcs(reinterpret_cast<uint4*>(og + row * p.C + ch * 8),
                   *reinterpret_cast<const uint4*>(qs + r * P + ch * 8));
    }
}

template <int DN>
cudaError_t launch_dn(const FlashArgs& p, dim3 grid, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(flash_mma_kernel<DN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    flash_mma_kernel<DN><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_flash_mma(const void* q, const void* k, const void* v, void* out, int batches,
                         long long Lq, int Lk, int heads, int d, long long q_bstride,
                         long long kv_bstride, cudaStream_t s) {
    FlashArgs p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.k = static_cast<const __nv_bfloat16*>(k);
    p.v = static_cast<const __nv_bfloat16*>(v);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.Lq = Lq;
    p.Lk = Lk;
    p.heads = heads;
    p.d = d;
    p.P = ((d / 8) & 1) ? d : d + 8;
    p.C = (long long)heads * d;
    p.q_bstride = q_bstride;
    p.kv_bstride = kv_bstride;
    p.scale_log2 = kLog2e / sqrtf((float)d);
    if (Lq == 0 || batches == 0) return cudaSuccess;
    const long long qtiles = (Lq + kBM - 1) / kBM;
    if (qtiles > 0x7fffffffLL || batches > 65535 || heads > 65535) return cudaErrorInvalidValue;
    dim3 grid((unsigned)qtiles, (unsigned)heads, (unsigned)batches);
    const size_t smem = (size_t)(kBM + 4 * kBN) * p.P * 2 + 256;
    switch (d / 8) {
#define PAB_F_CASE(DNV) \
    case DNV:           \
        return launch_dn<DNV>(p, grid, smem, s);
        PAB_F_CASE(1) PAB_F_CASE(2) PAB_F_CASE(3) PAB_F_CASE(4) PAB_F_CASE(5) PAB_F_CASE(6)
        PAB_F_CASE(7) PAB_F_CASE(8) PAB_F_CASE(9) PAB_F_CASE(10) PAB_F_CASE(11) PAB_F_CASE(12)
        PAB_F_CASE(13) PAB_F_CASE(14) PAB_F_CASE(15) PAB_F_CASE(16)
#undef PAB_F_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace pab

// scm_loss.cu -- the tangent-normalised sCM loss term for B200 (sm_100a).
//
// rCM's sCM term uses tangent normalisation (papernotes.org notes on "Large
// Scale Diffusion Distillation via Score-Regularized Continuous-Time
// Consistency", 损失函数 / 训练策略; ai.info AI summary, Methodology in Plain
// English: c = 0.1).  Per sample b, over its N elements:
//
//   n_b = sum_i g_bi^2,   r_bi = F_bi - F-_bi - g_bi / (n_b + c),
//   loss_b = sum_i r_bi^2,   grad_bi = 2 r_bi = d loss_b / d F_bi.
//
// The work is two streaming passes over HBM with one data-dependent scalar
// between them, so the design is about bandwidth, not arithmetic:
//   * one thread-block cluster per sample, each CTA a contiguous slice of the
//     sample; 8 or 16 CTAs per cluster, whichever finishes B samples in
//     fewer cluster-waves per CTA (the GPU holds fewer 16-CTA clusters);
//   * pass 1 sums g^2 in fp32; the CTAs meet at a cluster barrier and every
//     CTA adds the slice sums from distributed shared memory in the same
//     fixed order, so all hold the same n_b and the result is deterministic;
//   * pass 2 reads F, F- and g again (g mostly from L2) and writes grad and
//     the slice sums of r^2, which CTA 0 adds in a fixed order.
// 16-byte vector loads (8 bf16) when N is a multiple of 8, else bf16 by bf16.
// No scratch memory: the cross-CTA reduction lives in shared memory.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_jvp.h"
#include "scm_loss.h"
#include "sm100.cuh"

namespace scml {

using namespace ajvp;

constexpr int THREADS = 512;
constexpr int MAX_DEVICES = 64;

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void bf2_to_f(uint32_t w, float &lo, float &hi)
{
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

__device__ __forceinline__ uint32_t f_to_bf2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Sum of v over the CTA (every thread gets it).
__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red may still be read by a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) s += red[w];
    return s;
}

// Sum of one shared float over the cluster's CTAs in rank order (same bits in
// every CTA).  The caller has passed a cluster barrier since writing it.
__device__ __forceinline__ float cluster_sum(const float *slot, uint32_t ncta)
{
    const uint32_t a = smem_addr(slot);
    float s = 0.f;
    for (uint32_t k = 0; k < ncta; ++k) s += ld_shared_cluster_f32(mapa_shared(a, k));
    return s;
}

template <bool VEC>
__global__ void __launch_bounds__(THREADS, 1)
    scm_loss_kernel(const __nv_bfloat16 *__restrict__ f, const __nv_bfloat16 *__restrict__ fe,
                    const __nv_bfloat16 *__restrict__ g, float *__restrict__ loss,
                    __nv_bfloat16 *__restrict__ grad, long long N, float c)
{
    __shared__ float red[THREADS / 32];
    __shared__ float part[2];  // this CTA's slice sums: [0] g^2, [1] r^2
    const uint32_t rank = cluster_ctarank();
    const uint32_t ncta = cluster_nctarank();
    const long long b = blockIdx.y;
    const int t = threadIdx.x;
    // this CTA's slice, in units of 8 elements (VEC) or elements
    const long long units = VEC ? N / 8 : N;
    const long long lo = units * rank / ncta, hi = units * (rank + 1) / ncta;
    const size_t base = static_cast<size_t>(b) * static_cast<size_t>(N);

    // ---- pass 1: |g_b|^2
    float acc = 0.f;
    if constexpr (VEC) {
        const uint4 *gv = reinterpret_cast<const uint4 *>(g + base);
#pragma unroll 8
        for (long long u = lo + t; u < hi; u += THREADS) {
            const uint4 w = ld_stream(gv + u);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float a0, a1;
                bf2_to_f(ws[i], a0, a1);
                acc = fmaf(a0, a0, acc);
                acc = fmaf(a1, a1, acc);
            }
        }
    } else {
        for (long long u = lo + t; u < hi; u += THREADS) {
            const float a = __bfloat162float(g[base + u]);
            acc = fmaf(a, a, acc);
        }
    }
    acc = block_sum(acc, red);
    if (t == 0) part[0] = acc;
    cluster_sync();
    const float inv = 1.f / (cluster_sum(&part[0], ncta) + c);

    // ---- pass 2: r = F - F- - g inv, grad = 2 r, |r|^2
    float acc2 = 0.f;
    if constexpr (VEC) {
        const uint4 *fv = reinterpret_cast<const uint4 *>(f + base);
        const uint4 *ev = reinterpret_cast<const uint4 *>(fe + base);
        const uint4 *gv = reinterpret_cast<const uint4 *>(g + base);
        uint4 *dv = grad ? reinterpret_cast<uint4 *>(grad + base) : nullptr;
#pragma unroll 4
        for (long long u = lo + t; u < hi; u += THREADS) {
            const uint4 xf = ld_stream(fv + u), xe = ld_stream(ev + u), xg = ld_stream(gv + u);
            const uint32_t wf[4] = {xf.x, xf.y, xf.z, xf.w}, we[4] = {xe.x, xe.y, xe.z, xe.w},
                           wg[4] = {xg.x, xg.y, xg.z, xg.w};
            uint32_t wo[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float f0, f1, e0, e1, g0, g1;
                bf2_to_f(wf[i], f0, f1);
                bf2_to_f(we[i], e0, e1);
                bf2_to_f(wg[i], g0, g1);
                const float r0 = fmaf(-g0, inv, f0 - e0), r1 = fmaf(-g1, inv, f1 - e1);
                acc2 = fmaf(r0, r0, acc2);
                acc2 = fmaf(r1, r1, acc2);
                wo[i] = f_to_bf2(2.f * r0, 2.f * r1);
            }
            if (dv) dv[u] = make_uint4(wo[0], wo[1], wo[2], wo[3]);
        }
    } else {
        for (long long u = lo + t; u < hi; u += THREADS) {
            const size_t i = base + u;
            const float r = fmaf(-__bfloat162float(g[i]), inv, __bfloat162float(f[i]) - __bfloat162float(fe[i]));
            acc2 = fmaf(r, r, acc2);
            if (grad) grad[i] = __float2bfloat16_rn(2.f * r);
        }
    }
    acc2 = block_sum(acc2, red);
    if (t == 0) part[1] = acc2;
    cluster_sync();
    if (rank == 0 && t == 0) loss[b] = cluster_sum(&part[1], ncta);
    cluster_sync();  // no CTA leaves while CTA 0 may still read its shared memory
}

// How many clusters of `size` CTAs the GPU can hold at once (0 if none).
template <bool VEC>
static int max_active_clusters(int size)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(size), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(size);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, scm_loss_kernel<VEC>, &cfg) != cudaSuccess) n = 0;
    cudaGetLastError();  // a refused query leaves nothing behind
    return n;
}

// Resident clusters of 8 and of 16 CTAs on this device (queried once).
template <bool VEC>
static void cluster_capacity(int dev, int &n8, int &n16)
{
    static std::mutex mu;
    static int cap[MAX_DEVICES][2] = {};
    static bool done[MAX_DEVICES] = {};
    n8 = n16 = 0;
    if (dev < 0 || dev >= MAX_DEVICES) return;
    std::lock_guard<std::mutex> lk(mu);
    if (!done[dev]) {
        cap[dev][0] = max_active_clusters<VEC>(8);
        if (cudaFuncSetAttribute(scm_loss_kernel<VEC>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess)
            cap[dev][1] = max_active_clusters<VEC>(16);
        cudaGetLastError();
        done[dev] = true;
    }
    n8 = cap[dev][0];
    n16 = cap[dev][1];
}

// Cluster size for B samples: each sample's time scales as 1 / size, and
// the samples run in ceil(B / resident clusters) waves; take the smaller of
// waves / size for 8 and 16 CTAs.
template <bool VEC>
static int cluster_size(int dev, int B)
{
    int n8, n16;
    cluster_capacity<VEC>(dev, n8, n16);
    if (n8 <= 0) return n16 > 0 ? 16 : 0;
    if (n16 <= 0) return 8;
    const long long w8 = (B + n8 - 1) / n8, w16 = (B + n16 - 1) / n16;
    return (w16 * 8 < w8 * 16) ? 16 : 8;  // compare w16 / 16 with w8 / 8
}

static bool overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

template <bool VEC>
static int launch(const void *f, const void *fe, const void *g, float *loss, void *grad, int B, long long N,
                  float c, cudaStream_t s)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    const int cl = cluster_size<VEC>(dev, B);
    if (cl == 0) return ATTN_JVP_ERR_LAUNCH;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(cl), static_cast<unsigned>(B), 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, scm_loss_kernel<VEC>, static_cast<const __nv_bfloat16 *>(f),
                           static_cast<const __nv_bfloat16 *>(fe), static_cast<const __nv_bfloat16 *>(g), loss,
                           static_cast<__nv_bfloat16 *>(grad), N, c) != cudaSuccess)
        return ATTN_JVP_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? ATTN_JVP_OK : ATTN_JVP_ERR_LAUNCH;
}

}  // namespace scml

extern "C" int scm_tangent_loss(const void *f, const void *f_ema, const void *g, float *loss, void *grad,
                                int B, long long N, float c, void *stream)
{
    if (!f || !f_ema || !g || !loss) return ATTN_JVP_ERR_NULL;
    if (B < 1 || B > 65535 || N < 1 || N > (1ll << 40)) return ATTN_JVP_ERR_SHAPE;
    const void *v16[4] = {f, f_ema, g, grad};
    for (const void *p : v16)
        if (reinterpret_cast<uintptr_t>(p) & 15) return ATTN_JVP_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(loss) & 3) return ATTN_JVP_ERR_ALIGN;
    if (!std::isfinite(c) || c < 0.f) return ATTN_JVP_ERR_VALUE;
    const size_t nb = static_cast<size_t>(B) * static_cast<size_t>(N) * 2, nl = static_cast<size_t>(B) * 4;
    const void *ins[3] = {f, f_ema, g};
    for (const void *in : ins) {
        if (scml::overlap(loss, nl, in, nb)) return ATTN_JVP_ERR_VALUE;
        if (grad && scml::overlap(grad, nb, in, nb)) return ATTN_JVP_ERR_VALUE;
    }
    if (grad && scml::overlap(grad, nb, loss, nl)) return ATTN_JVP_ERR_VALUE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return (N % 8 == 0) ? scml::launch<true>(f, f_ema, g, loss, grad, B, N, c, s)
                        : scml::launch<false>(f, f_ema, g, loss, grad, B, N, c, s);
}

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
//     sample; the cluster size (1 to 16 CTAs) is the one that finishes B
//     samples soonest, given how many clusters of each size the GPU holds
//     at once;
//   * every thread issues a batch of independent 16-byte loads before it
//     uses any (16 in pass 1, 8 per tensor in pass 2), so each SM keeps tens
//     of KB in flight;
//   * pass 1 sums g^2 in fp32 and reads g with an L2 evict-last hint, so the
//     second pass finds most of it in L2; the CTAs meet at a cluster barrier
//     and every CTA adds the slice sums from distributed shared memory in
//     the same fixed order, so all hold the same n_b and the result is
//     deterministic;
//   * pass 2 reads F, F- (evict-first) and g again and writes grad and the
//     slice sums of r^2, which CTA 0 adds in a fixed order.
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

constexpr int THREADS = 256;
constexpr int MAX_DEVICES = 64;

constexpr int U1 = 16;  // 16-byte loads in flight per thread, pass 1
constexpr int U2 = 8;   // per tensor, pass 2

// 16-byte read-only load that skips L1, with an L2 eviction policy.
__device__ __forceinline__ uint4 ld_stream(const void *p, uint64_t pol)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
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
    const uint4 *fv = reinterpret_cast<const uint4 *>(f + base);
    const uint4 *ev = reinterpret_cast<const uint4 *>(fe + base);
    const uint4 *gv = reinterpret_cast<const uint4 *>(g + base);
    uint4 *dv = grad ? reinterpret_cast<uint4 *>(grad + base) : nullptr;
    const uint64_t keep = l2_policy_evict_last();
    const uint64_t once = l2_policy_evict_first();
    constexpr long long STEP2 = static_cast<long long>(THREADS) * U2;

    // one pass-2 batch: U2 units of F, F- and g per thread
    uint4 xf[U2], xe[U2], xg[U2];
    auto load2 = [&](const long long u0) {
#pragma unroll
        for (int k = 0; k < U2; ++k) {
            const long long u = u0 + static_cast<long long>(k) * THREADS;
            const bool in = u < hi;
            xf[k] = in ? ld_stream(fv + u, once) : make_uint4(0, 0, 0, 0);
            xe[k] = in ? ld_stream(ev + u, once) : make_uint4(0, 0, 0, 0);
            xg[k] = in ? ld_stream(gv + u, once) : make_uint4(0, 0, 0, 0);
        }
    };

    // ---- pass 1: |g_b|^2
    float acc = 0.f;
    if constexpr (VEC) {
        for (long long u0 = lo + t; u0 < hi; u0 += static_cast<long long>(THREADS) * U1) {
            uint4 w[U1];
#pragma unroll
            for (int k = 0; k < U1; ++k) {
                const long long u = u0 + static_cast<long long>(k) * THREADS;
                w[k] = u < hi ? ld_stream(gv + u, keep) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < U1; ++k) {
                const uint32_t ws[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float a0, a1;
                    bf2_to_f(ws[i], a0, a1);
                    acc = fmaf(a0, a0, acc);
                    acc = fmaf(a1, a1, acc);
                }
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
        for (long long u0 = lo + t; u0 < hi; u0 += STEP2) {
            load2(u0);
#pragma unroll
            for (int k = 0; k < U2; ++k) {
                const uint32_t wf[4] = {xf[k].x, xf[k].y, xf[k].z, xf[k].w},
                               we[4] = {xe[k].x, xe[k].y, xe[k].z, xe[k].w},
                               wg[4] = {xg[k].x, xg[k].y, xg[k].z, xg[k].w};
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
                const long long u = u0 + static_cast<long long>(k) * THREADS;
                if (dv && u < hi) dv[u] = make_uint4(wo[0], wo[1], wo[2], wo[3]);
            }
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

constexpr int MAX_CLUSTER = 16;

// Resident clusters of 1 .. 16 CTAs on this device (queried once; 0 where a
// size cannot launch).
template <bool VEC>
static const int *cluster_capacity(int dev)
{
    static std::mutex mu;
    static int cap[MAX_DEVICES][MAX_CLUSTER + 1] = {};
    static bool done[MAX_DEVICES] = {};
    static const int none[MAX_CLUSTER + 1] = {};
    if (dev < 0 || dev >= MAX_DEVICES) return none;
    std::lock_guard<std::mutex> lk(mu);
    if (!done[dev]) {
        const bool big = cudaFuncSetAttribute(scm_loss_kernel<VEC>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                              1) == cudaSuccess;
        cudaGetLastError();
        for (int sz = 1; sz <= MAX_CLUSTER; ++sz) cap[dev][sz] = (sz <= 8 || big) ? max_active_clusters<VEC>(sz) : 0;
        done[dev] = true;
    }
    return cap[dev];
}

// Cluster size for B samples: a sample's time scales as 1 / size, and the
// samples run in ceil(B / resident clusters) waves; take the size with the
// smallest waves / size (the larger size on a tie).
template <bool VEC>
static int cluster_size(int dev, int B)
{
    const int *cap = cluster_capacity<VEC>(dev);
    int best = 0;
    long long bw = 0;  // waves of the best size so far
    for (int sz = 1; sz <= MAX_CLUSTER; ++sz) {
        if (cap[sz] <= 0) continue;
        const long long w = (B + cap[sz] - 1) / cap[sz];
        if (best == 0 || w * best <= bw * sz) {  // w / sz <= bw / best
            best = sz;
            bw = w;
        }
    }
    return best;
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

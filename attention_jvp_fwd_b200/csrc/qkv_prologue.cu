// qkv_prologue.cu -- QKV projection + per-head RMSNorm, with its tangent, for
// B200 (sm_100a): the layer in front of attention as a forward-and-tangent
// function.
//
// rCM refactors each layer to expose forward and tangent functions ("Large
// Scale Diffusion Distillation via Score-Regularized Continuous-Time
// Consistency", ai.info AI summary, Key Contributions 1).  For tokens x and
// their tangent x' (weights fixed):
//
//   y = x W^T, y' = x' W^T          with W = [W_q; W_k; W_v]  [3 H d, D]
//   q = gamma_q y_q r,  q' = gamma_q (y_q' r - y_q r^3 mean(y_q y_q'))
//   (k alike with gamma_k),  v = y_v,  v' = y_v'
//   r = (mean over the head's d channels of y^2 + eps)^(-1/2)
//
// and writes q, k, v, q', k', v' in the attention layout [B, H, L, d], so
// the attention kernel reads them directly.
//
// A tile is 256 tokens x one head, owned by a cluster of two CTAs (a CTA
// pair): two tcgen05 GEMMs that share the weight tile, Y = X W_h^T and
// Y' = X' W_h^T (M = 256, N = d, K = D), issued by the leader CTA as
// cta_group::2 MMAs.  Each CTA stages its own 128 tokens of X and X' and half
// of the rows of W_h, and receives Y, Y' of its own tokens in its TMEM, so
// each CTA reads only half of the weight slice from shared memory per MMA
// (the single-CTA form of this kernel was bound by shared-memory bandwidth).
// The kernel is persistent (one pair per two SMs walks the tiles) with two
// accumulator sets, so the epilogue of one tile overlaps the MMAs of the
// next.  In each CTA a TMA warp streams X, X' and its half of W_h in
// 64-column slices through a 5-stage ring that runs on across tiles; the
// leader's MMA warp issues the MMAs; four epilogue warps (thread = token)
// reduce each row's y^2 and y y' over the head, apply the RMSNorm and its
// tangent, and store bf16.  Waits are bounded like the attention kernel's
// (status word read by qkv_prologue_check).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_jvp.h"
#include "qkv_prologue.h"
#include "sm100.cuh"

namespace qkvp {

using namespace ajvp;

constexpr int BM = 128;   // tokens per CTA per tile (TMEM lanes); a pair covers 2 BM
constexpr int BK = 64;    // D columns per stage (one 128-byte swizzle row)
constexpr int NS = 5;     // ring stages
constexpr int NTHREADS = 192;  // TMA warp, MMA warp, 4 epilogue warps
constexpr uint64_t TIMEOUT_NS = 2000000000ull;

template <int DH>
struct PCfg {
    static constexpr uint32_t A_BYTES = BM * BK * 2;         // one of X, X' per stage
    static constexpr uint32_t B_BYTES = (DH / 2) * BK * 2;   // this CTA's half of the W_h slice
    static constexpr uint32_t ST_BYTES = 2 * A_BYTES + B_BYTES;
    static constexpr uint32_t OFF_BAR = NS * ST_BYTES;
    static constexpr uint32_t OFF_MISC = OFF_BAR + (2 * NS + 5) * 8;  // tmem slot, abort
    static constexpr uint32_t OFF_GAMMA = OFF_MISC + 16;              // float [2][DH]
    static constexpr uint32_t SMEM_BYTES = OFF_GAMMA + 2 * DH * 4;
    static constexpr uint32_t TMEM_COLS = 4 * DH;                      // two sets of Y | Y'
    static constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, DH, false);  // M = 256 over the pair
    static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory budget");
};

struct Params {
    CUtensorMap tm_x, tm_xd, tm_w;
    const float *gamma_q, *gamma_k;
    __nv_bfloat16 *out[6];  // q, k, v, q', k', v'
    int T, L, H, D, tiles_m;  // tiles_m: 256-token blocks
    float eps;
    uint64_t timeout_ns;
};

__device__ int g_status;
__device__ int g_status_taken;  // the word as the last check took it

// Read and clear the status word in one atomic step, ordered on the checking
// stream, so a site recorded by a kernel on another stream between a read
// and a clear cannot be lost.
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status, 0); }

// Host threads that check at the same time take turns on g_status_taken.
static std::mutex g_check_mu;

// Bounded wait (acquire at cluster scope: most of these barriers are
// signalled from the other CTA of the pair); gives up when another role has
// aborted (if honor_abort) or after `limit` ns (then it records `site` and
// aborts the CTA itself).
__device__ __noinline__ bool wait(uint64_t *bar, uint32_t parity, volatile int *abort, uint64_t limit, int site,
                                  bool honor_abort = true)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(a, parity)) return true;
        if (honor_abort && *abort) return false;
        if (globaltimer_ns() - t0 > limit) {
            *abort = 1;
            atomicCAS(&g_status, 0, site);
            return false;
        }
    }
}

template <int DH>
__global__ void __launch_bounds__(NTHREADS, 1) qkv_prologue_kernel(const __grid_constant__ Params p)
{
    using C = PCfg<DH>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 128-byte swizzle atoms want 1024-byte alignment
    uint8_t *smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();  // 0: the leader, which issues the MMAs
    const bool leader = rank == 0;
    const int tiles_n = 3 * p.H;
    const int n_tiles = p.tiles_m * tiles_n;
    const int nk = p.D / BK;
    // this pair's tiles: cl, cl + ncl, ...  (head tile fastest, so pairs
    // running together share the token tile through L2)
    const int cl = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    const int my_tiles = cl < n_tiles ? (n_tiles - 1 - cl) / ncl + 1 : 0;

    // full, acc_empty and drain are used in the leader only; empty and
    // acc_full in both CTAs (the leader's commits reach both)
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);  // [NS] both CTAs' slices landed
    uint64_t *empty = full + NS;         // [NS] the MMAs are done with this CTA's slice
    uint64_t *acc_full = empty + NS;     // [2] accumulator set b holds a finished tile
    uint64_t *acc_empty = acc_full + 2;  // [2] both epilogues have read accumulator set b
    uint64_t *drain = acc_empty + 2;     // MMAs in flight after an abort are done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    float *gamma = reinterpret_cast<float *>(smem + C::OFF_GAMMA);  // [2][DH]: q, k

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // one arrival per epilogue warp of each CTA
        }
        mbar_init(drain, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp >= 2) {
        for (int i = tid - 64; i < 2 * DH; i += 128) gamma[i] = i < DH ? p.gamma_q[i] : p.gamma_k[i - DH];
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t full_lead = mapa_shared(smem_addr(full), 0);
    const uint32_t acc_empty_lead = mapa_shared(smem_addr(acc_empty), 0);

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA: one ring across all tiles
        // Both CTAs' slices complete on the leader's full barrier; the
        // leader announces the bytes of both.
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            long long issued = 0;  // slices loaded so far
            bool ok = true;
            for (int li = 0; li < my_tiles && ok; ++li) {
                const int t = cl + li * ncl;
                const int nt = t % tiles_n, mt = t / tiles_n;
                const int row = mt * 2 * BM + static_cast<int>(rank) * BM;
                const int wrow = nt * DH + static_cast<int>(rank) * (DH / 2);
                for (int k = 0; k < nk; ++k) {
                    const int s = static_cast<int>(issued % NS);
                    if (issued >= NS &&
                        !wait(&empty[s], static_cast<uint32_t>((issued / NS) - 1) & 1, abort, p.timeout_ns, 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * C::ST_BYTES;
                    const uint32_t fb = full_lead + s * 8;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::ST_BYTES);
                    tma_load_3d_pair(st, &p.tm_x, fb, k * BK, row, 0, pol);
                    tma_load_3d_pair(st + C::A_BYTES, &p.tm_xd, fb, k * BK, row, 0, pol);
                    tma_load_3d_pair(st + 2 * C::A_BYTES, &p.tm_w, fb, k * BK, wrow, 0, pol);
                    ++issued;
                }
            }
            // let every load issued land before the CTAs can exit: the
            // leader waits for the last phase of each stage (the peer's
            // loads complete on the same barriers; the final cluster barrier
            // keeps the peer alive until then)
            if (leader)
                for (long long q = (issued > NS ? issued - NS : 0); q < issued; ++q)
                    wait(&full[q % NS], static_cast<uint32_t>(q / NS) & 1, abort, p.timeout_ns, 2, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA (leader; warp-wide, elected lane)
        if (leader) {
            bool ok = true, issued = false;
            long long used = 0;  // slices consumed so far
            for (int li = 0; li < my_tiles && ok; ++li) {
                const int b = li & 1;
                const uint32_t acc = tbase + b * (2 * DH);
                if (li >= 2) {
                    ok = __all_sync(0xffffffffu, wait(&acc_empty[b], ((li >> 1) - 1) & 1, abort, p.timeout_ns, 6));
                    if (!ok) break;
                    tc_fence_after();
                }
                for (int k = 0; k < nk; ++k, ++used) {
                    const int s = static_cast<int>(used % NS);
                    ok = __all_sync(0xffffffffu, wait(&full[s], static_cast<uint32_t>(used / NS) & 1, abort,
                                                      p.timeout_ns, 3));
                    if (!ok) break;
                    tc_fence_after();
                    // the same shared-memory offsets in both CTAs: A rows 0-127
                    // and B rows 0 .. d/2-1 here, the rest in the peer
                    const uint32_t st = smem_addr(smem + s * C::ST_BYTES);
                    const uint64_t dx = sdesc_sw128(st, 16, 1024);
                    const uint64_t dxd = sdesc_sw128(st + C::A_BYTES, 16, 1024);
                    const uint64_t dw = sdesc_sw128(st + 2 * C::A_BYTES, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_ss_pair(acc, desc_add(dx, kk * 32), desc_add(dw, kk * 32), C::IDESC,
                                    (k > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_ss_pair(acc + DH, desc_add(dxd, kk * 32), desc_add(dw, kk * 32), C::IDESC,
                                    (k > 0 || kk > 0) ? 1u : 0u);
                    mma_commit_pair_mc(&empty[s], 0x3);
                    issued = true;
                }
                if (!ok) break;
                mma_commit_pair_mc(&acc_full[b], 0x3);
            }
            if (!ok && issued) {
                // nobody else waits for the MMAs in flight after an abort:
                // drain them here, so TMEM is not freed under them
                mma_commit_pair_mc(drain, 0x1);
                wait(drain, 0, abort, p.timeout_ns, 5, false);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue, thread = token
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        for (int li = 0; li < my_tiles; ++li) {
            const int b = li & 1;
            const int t_idx = cl + li * ncl;
            const int nt = t_idx % tiles_n, mt = t_idx / tiles_n;
            const int part = nt / p.H, head = nt % p.H;
            const uint32_t ty = tbase + lane_off + b * (2 * DH), tyd = ty + DH;
            bool ok = wait(&acc_full[b], (li >> 1) & 1, abort, p.timeout_ns, 4);
            ok = __all_sync(0xffffffffu, ok && !*abort);  // warp-uniform: tcgen05.ld below is collective
            if (!ok) break;
            tc_fence_after();
            const int t = mt * 2 * BM + static_cast<int>(rank) * BM + r;
            const float *g = gamma + (part == 1 ? DH : 0);
            float rs = 1.f, mix = 0.f;
            if (part < 2) {
                // sums over the head's channels: y^2 and y y'
                float s2 = 0.f, sm = 0.f;
#pragma unroll 1
                for (int c = 0; c < DH; c += 32) {
                    uint32_t a[32], e[32];
                    tmem_ld32(ty + c, a);
                    tmem_ld32(tyd + c, e);
                    tmem_ld_wait2(a, e);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float y = __uint_as_float(a[i]);
                        s2 = fmaf(y, y, s2);
                        sm = fmaf(y, __uint_as_float(e[i]), sm);
                    }
                }
                rs = 1.f / sqrtf(s2 / DH + p.eps);
                mix = rs * rs * rs * (sm / DH);  // r^3 mean(y y')
            }
            // every lane loads (tcgen05.ld is warp-collective); only rows of
            // real tokens store
            const bool store = t < p.T;
            const int tt = store ? t : 0;
            const int bb = tt / p.L, l = tt % p.L;
            const size_t o = ((static_cast<size_t>(bb) * p.H + head) * p.L + l) * DH;
            __nv_bfloat16 *dy = p.out[part] + o;
            __nv_bfloat16 *dyd = p.out[3 + part] + o;
#pragma unroll 1
            for (int c = 0; c < DH; c += 32) {
                uint32_t a[32], e[32], py[16], pyd[16];
                tmem_ld32(ty + c, a);
                tmem_ld32(tyd + c, e);
                tmem_ld_wait2(a, e);
                if (c + 32 == DH) {
                    // the last read of this accumulator set: hand it back to
                    // the leader's MMA warp before the stores
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_lead + b * 8);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float y0 = __uint_as_float(a[2 * i]), y1 = __uint_as_float(a[2 * i + 1]);
                    float e0 = __uint_as_float(e[2 * i]), e1 = __uint_as_float(e[2 * i + 1]);
                    if (part < 2) {
                        const float g0 = g[c + 2 * i], g1 = g[c + 2 * i + 1];
                        const float n0 = g0 * (e0 * rs - y0 * mix), n1 = g1 * (e1 * rs - y1 * mix);
                        y0 = g0 * (y0 * rs);
                        y1 = g1 * (y1 * rs);
                        e0 = n0;
                        e1 = n1;
                    }
                    uint32_t u, w;
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(y1), "f"(y0));
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(e1), "f"(e0));
                    py[i] = u;
                    pyd[i] = w;
                }
                if (store) {
                    uint4 *d0 = reinterpret_cast<uint4 *>(dy + c), *d1 = reinterpret_cast<uint4 *>(dyd + c);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        d0[i] = make_uint4(py[4 * i], py[4 * i + 1], py[4 * i + 2], py[4 * i + 3]);
                        d1[i] = make_uint4(pyd[4 * i], pyd[4 * i + 1], pyd[4 * i + 2], pyd[4 * i + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    // neither CTA leaves while the leader's MMAs may still read the peer's
    // shared memory or write its TMEM, or loads may still signal the leader
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tbase, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// [rows, cols] bf16 row-major as a 3-D tensor (cols, rows, 1); box 64 x box_rows,
// 128-byte swizzle, zero fill past the last row.
static bool make_map(CUtensorMap *m, const void *base, long long rows, int cols, int box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1};
    const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(rows) * cols * 2};
    const cuuint32_t box[3] = {BK, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), gdim, gstride, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int MAX_DEVICES = 64;

// Launch configuration of the pair kernel (grid = 2 x pairs, clusters of 2).
template <int DH>
static void pair_config(cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr, unsigned pairs, cudaStream_t s)
{
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = PCfg<DH>::SMEM_BYTES + 1024;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

// Per device, once: the shared-memory opt-in and how many CTA pairs fit on
// the GPU at once (a persistent grid must not spill into a second wave).
template <int DH>
static int resident_pairs(int dev)
{
    static std::mutex mu;
    static int pairs[MAX_DEVICES] = {};
    if (dev < 0 || dev >= MAX_DEVICES) return 0;
    std::lock_guard<std::mutex> g(mu);
    if (pairs[dev] == 0) {
        if (cudaFuncSetAttribute(qkv_prologue_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(PCfg<DH>::SMEM_BYTES + 1024)) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg;
        cudaLaunchAttribute attr[1];
        pair_config<DH>(cfg, attr, 1, nullptr);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, qkv_prologue_kernel<DH>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return 0;
        }
        pairs[dev] = n;
    }
    return pairs[dev];
}

template <int DH>
static int launch_kernel(const Params &prm, long long n_tiles, cudaStream_t s)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    const int fit = resident_pairs<DH>(dev);
    if (fit < 1) return ATTN_JVP_ERR_LAUNCH;
    const unsigned pairs = static_cast<unsigned>(n_tiles < fit ? n_tiles : fit);
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    pair_config<DH>(cfg, attr, pairs, s);
    if (cudaLaunchKernelEx(&cfg, qkv_prologue_kernel<DH>, prm) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    return cudaGetLastError() == cudaSuccess ? ATTN_JVP_OK : ATTN_JVP_ERR_LAUNCH;
}

static bool overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace qkvp

extern "C" {

int qkv_rmsnorm_jvp(const void *x, const void *x_dot, const void *w_qkv, const float *gamma_q,
                    const float *gamma_k, void *q, void *k, void *v, void *q_dot, void *k_dot, void *v_dot,
                    int B, int L, int H, int D, int d, float eps, void *stream)
{
    using namespace qkvp;
    if (!x || !x_dot || !w_qkv || !gamma_q || !gamma_k || !q || !k || !v || !q_dot || !k_dot || !v_dot)
        return ATTN_JVP_ERR_NULL;
    if (B < 1 || L < 1 || H < 1 || D < BK || D % BK) return ATTN_JVP_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_JVP_ERR_HEADDIM;
    const long long T = static_cast<long long>(B) * L;
    if (T >= (1ll << 31) || 3ll * H * d >= (1ll << 31)) return ATTN_JVP_ERR_SHAPE;
    const long long n_tiles = ((T + 2 * BM - 1) / (2 * BM)) * 3ll * H;  // 256-token blocks x heads
    if (n_tiles > INT_MAX) return ATTN_JVP_ERR_SHAPE;
    const void *a16[9] = {x, x_dot, w_qkv, q, k, v, q_dot, k_dot, v_dot};
    for (const void *p : a16)
        if (reinterpret_cast<uintptr_t>(p) & 15) return ATTN_JVP_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(gamma_q) & 3) || (reinterpret_cast<uintptr_t>(gamma_k) & 3))
        return ATTN_JVP_ERR_ALIGN;
    if (!std::isfinite(eps) || eps < 0.f) return ATTN_JVP_ERR_VALUE;
    const size_t nx = static_cast<size_t>(T) * D * 2, nw = static_cast<size_t>(3) * H * d * D * 2;
    const size_t no = static_cast<size_t>(T) * H * d * 2, ng = static_cast<size_t>(d) * 4;
    const void *ins[5] = {x, x_dot, w_qkv, gamma_q, gamma_k};
    const size_t insz[5] = {nx, nx, nw, ng, ng};
    void *outs[6] = {q, k, v, q_dot, k_dot, v_dot};
    for (int i = 0; i < 6; ++i) {
        for (int j = 0; j < 5; ++j)
            if (overlap(outs[i], no, ins[j], insz[j])) return ATTN_JVP_ERR_VALUE;
        for (int j = i + 1; j < 6; ++j)
            if (overlap(outs[i], no, outs[j], no)) return ATTN_JVP_ERR_VALUE;
    }
    Params prm;
    std::memset(&prm, 0, sizeof prm);
    if (!make_map(&prm.tm_x, x, T, D, BM) || !make_map(&prm.tm_xd, x_dot, T, D, BM) ||
        !make_map(&prm.tm_w, w_qkv, 3ll * H * d, D, d / 2))
        return ATTN_JVP_ERR_LAUNCH;
    prm.gamma_q = gamma_q;
    prm.gamma_k = gamma_k;
    for (int i = 0; i < 6; ++i) prm.out[i] = static_cast<__nv_bfloat16 *>(outs[i]);
    prm.T = static_cast<int>(T);
    prm.L = L;
    prm.H = H;
    prm.D = D;
    prm.tiles_m = static_cast<int>((T + 2 * BM - 1) / (2 * BM));
    prm.eps = eps;
    prm.timeout_ns = TIMEOUT_NS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // persistent: as many CTA pairs as fit at once (or one per tile, if there are fewer)
    return d == 128 ? launch_kernel<128>(prm, n_tiles, s) : launch_kernel<64>(prm, n_tiles, s);
}

int qkv_prologue_check(void *stream, int *site)
{
    if (site) *site = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(qkvp::g_check_mu);
    qkvp::take_status_kernel<<<1, 1, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    int st = 0;
    if (cudaMemcpyFromSymbolAsync(&st, qkvp::g_status_taken, sizeof st, 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ATTN_JVP_ERR_LAUNCH;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (st == 0) return ATTN_JVP_OK;
    if (site) *site = st;
    return ATTN_JVP_ERR_TIMEOUT;
}

}  // extern "C"

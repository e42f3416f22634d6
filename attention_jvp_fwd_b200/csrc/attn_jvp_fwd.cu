// attn_jvp_fwd.cu -- attention forward + JVP for B200 (sm_100a), and its C ABI.
//
// The FlashAttention-2 JVP kernel of rCM ("Large Scale Diffusion Distillation
// via Score-Regularized Continuous-Time Consistency", ai.info AI summary, Key
// Contributions 1 and Methodology in Plain English) folds the tangent of
// attention into the block-wise forward pass.  This is a Blackwell-native
// design of that operation:
//
//   * one CTA owns a 128-row query tile of one (b, h); Q and Q' stay in shared
//     memory, K/K' and V/V' tiles of 64 keys stream through two TMA rings;
//   * S = Q K^T and S'_raw = Q K'^T + Q' K^T are tcgen05 MMAs into TMEM.  K and
//     K' sit next to each other in shared memory, so Q [K ; K']^T is a single
//     N = 128 MMA that writes S and Q K'^T side by side; Q' K^T then adds onto
//     the second half.  Together this is the K = 2d product [Q | Q'][K' | K]^T;
//   * one warpgroup (thread = query row) runs the online softmax in registers:
//     running max m (lazily rescaled), denominator l = sum p and
//     a = sum p (s S'_raw - c).  It writes P and P * (s S'_raw - c) back into
//     TMEM as bf16 over the S columns;
//   * O += P V and O'_acc += [P(sS' - c) | P] [V ; V'] are tcgen05 MMAs with A
//     read from TMEM;
//   * the epilogue forms O = O_acc / l and O' = (O'_acc - (a / l) O_acc) / l.
//
// c is a per-row constant (the p-weighted mean of s S'_raw over the first key
// tile).  In exact arithmetic O' does not depend on it; it keeps the bf16
// products P (sS' - c) small when S' has a large row mean.
//
// Every wait on an mbarrier is bounded (default 2 s, wall clock); a wait that
// runs out records a site code in a device status word, tells the other
// roles to stop, lets every copy and MMA already in flight finish, frees
// TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_jvp.h"
#include "sm100.cuh"

namespace ajvp {

constexpr int BM = 128;                   // query rows per CTA (= TMEM lanes)
constexpr int BN = 64;                    // keys per K/V tile
constexpr int NTHREADS = 192;             // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f; // log2 units: rescale when the max grows by 2^8
constexpr uint64_t DEFAULT_TIMEOUT_NS = 2000000000ull;

// Wait sites recorded in the status word when a wait gives up.
enum : int {
    SITE_Q_FULL = 1,
    SITE_K_FULL = 2,
    SITE_K_EMPTY = 3,
    SITE_V_FULL = 4,
    SITE_V_EMPTY = 5,
    SITE_S_FULL = 6,
    SITE_P_FULL = 7,
    SITE_O_DONE = 8,
    SITE_V_TAIL = 9,
    SITE_DRAIN = 10,
};

template <int D>
struct Cfg {
    static constexpr int NKB = D / 64;               // 128-byte column blocks per row
    static constexpr int NK = (D == 128) ? 3 : 4;    // K/K' ring depth
    static constexpr int NV = (D == 128) ? 2 : 4;    // V/V' ring depth
    static constexpr uint32_t Q_BYTES = BM * D * 2;  // one of Q, Q'
    static constexpr uint32_t KST_BYTES = 2 * BN * D * 2;
    static constexpr uint32_t VST_BYTES = 2 * BN * D * 2;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_QD = Q_BYTES;
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NK * KST_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + NV * VST_BYTES;
    static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 + 2 + 1 + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + base alignment slack
    // TMEM columns: O | O'_acc | S buffer 0 (S, S'_raw) | S buffer 1
    static constexpr uint32_t T_O = 0;
    static constexpr uint32_t T_OD = D;
    static constexpr uint32_t T_S = 2 * D;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, 2 * BN, false);
    static constexpr uint32_t IDESC_SD = idesc_bf16_f32(BM, BN, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
    static_assert(T_S + 4 * BN <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Params {
    CUtensorMap tm_q, tm_qd, tm_k, tm_kd, tm_v, tm_vd;
    void *o;
    void *od;
    float *lse;
    const int32_t *kv_len;
    int H, Lq, Lk, nqt;
    float scale;  // s
    float sl2;    // s * log2(e)
    uint64_t timeout_ns;
    int flags;
};

__device__ int g_status;  // first wait site that gave up since the last check

struct WaitCtx {
    volatile int *abort;
    uint64_t limit_ns;
};

// Bounded wait for phase `parity` of `bar`.  Returns false if the limit ran
// out (recording `site`) or, when honor_abort is set, if another role gave up.
__device__ __noinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const WaitCtx &c, int site,
                                      bool honor_abort = true)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(a, parity)) return true;
        if (honor_abort && *c.abort) return false;
        if (globaltimer_ns() - t0 > c.limit_ns) {
            *c.abort = 1;
            atomicCAS(&g_status, 0, site);
            return false;
        }
    }
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_fwd_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int qt = blockIdx.x % p.nqt;
    const int bh = blockIdx.x / p.nqt;
    const int b = bh / p.H;
    const int q0 = qt * BM;
    int nb = p.Lk;
    if (p.kv_len) nb = min(max(p.kv_len[b], 0), p.Lk);
    const int nT = (nb + BN - 1) / BN;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *k_full = q_full + 1;
    uint64_t *k_empty = k_full + C::NK;
    uint64_t *v_full = k_empty + C::NK;
    uint64_t *v_empty = v_full + C::NV;
    uint64_t *s_full = v_empty + C::NV;
    uint64_t *p_full = s_full + 2;
    uint64_t *o_done = p_full + 2;
    uint64_t *drain = o_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 128);
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (tid == 32) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_qd);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_kd);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_vd);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const WaitCtx wc{abort_flag, p.timeout_ns};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nT > 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            const bool load_q = !(p.flags & ATTN_JVP_DEBUG_STARVE_Q);
            if (load_q) {
                mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
                for (int c = 0; c < C::NKB; ++c) {
                    tma_load_3d(smem + C::OFF_Q + c * BM * 128, &p.tm_q, q_full, c * 64, q0, bh, pol_q);
                    tma_load_3d(smem + C::OFF_QD + c * BM * 128, &p.tm_qd, q_full, c * 64, q0, bh,
                                pol_q);
                }
            }
            int nk = 0, nv = 0;
            bool ok = true;
            for (int j = 0; j <= nT && ok; ++j) {
                if (j < nT) {
                    const int s = j % C::NK;
                    if (j >= C::NK) ok = wait_bar(&k_empty[s], ((j / C::NK) - 1) & 1, wc, SITE_K_EMPTY);
                    if (!ok) break;
                    uint8_t *dst = smem + C::OFF_K + s * C::KST_BYTES;
                    mbar_arrive_expect_tx(&k_full[s], C::KST_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NKB; ++c) {
                        tma_load_3d(dst + c * (2 * BN * 128), &p.tm_k, &k_full[s], c * 64, j * BN, bh,
                                    pol_kv);
                        tma_load_3d(dst + c * (2 * BN * 128) + BN * 128, &p.tm_kd, &k_full[s], c * 64,
                                    j * BN, bh, pol_kv);
                    }
                    ++nk;
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s = jj % C::NV;
                    if (jj >= C::NV) ok = wait_bar(&v_empty[s], ((jj / C::NV) - 1) & 1, wc, SITE_V_EMPTY);
                    if (!ok) break;
                    uint8_t *dst = smem + C::OFF_V + s * C::VST_BYTES;
                    mbar_arrive_expect_tx(&v_full[s], C::VST_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NKB; ++c) {
                        tma_load_3d(dst + c * (BN * 128), &p.tm_v, &v_full[s], c * 64, jj * BN, bh, pol_kv);
                        tma_load_3d(dst + (C::NKB + c) * (BN * 128), &p.tm_vd, &v_full[s], c * 64, jj * BN,
                                    bh, pol_kv);
                    }
                    ++nv;
                }
            }
            // Let every load this thread issued land before the CTA can exit.
            if (load_q) wait_bar(q_full, 0, wc, SITE_DRAIN, false);
            for (int s = 0; s < C::NK && s < nk; ++s) {
                const int t = s + ((nk - 1 - s) / C::NK) * C::NK;
                wait_bar(&k_full[s], (t / C::NK) & 1, wc, SITE_DRAIN, false);
            }
            for (int s = 0; s < C::NV && s < nv; ++s) {
                const int t = s + ((nv - 1 - s) / C::NV) * C::NV;
                wait_bar(&v_full[s], (t / C::NV) & 1, wc, SITE_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && nT > 0) {
            bool ok = wait_bar(q_full, 0, wc, SITE_Q_FULL);
            bool issued = false;
            if (ok) tc_fence_after();
            const uint32_t qa = smem_addr(smem + C::OFF_Q);
            const uint32_t qda = smem_addr(smem + C::OFF_QD);
            for (int j = 0; j <= nT && ok; ++j) {
                if (j < nT) {
                    const int s = j % C::NK;
                    ok = wait_bar(&k_full[s], (j / C::NK) & 1, wc, SITE_K_FULL);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t tS = tbase + C::T_S + (j & 1) * (2 * BN);
                    const uint32_t ka = smem_addr(smem + C::OFF_K + s * C::KST_BYTES);
                    // S | Q K'^T  =  Q [K ; K']^T   (N = 2 BN)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                        mma_ss(tS, sdesc_sw128(qa + oa, 16, 1024), sdesc_sw128(ka + ob, 16, 1024),
                               C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    // += Q' K^T into the second half
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                        mma_ss(tS + BN, sdesc_sw128(qda + oa, 16, 1024), sdesc_sw128(ka + ob, 16, 1024),
                               C::IDESC_SD, 1u);
                    }
                    mma_commit(&k_empty[s]);
                    mma_commit(&s_full[j & 1]);
                    issued = true;
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s = jj % C::NV;
                    ok = wait_bar(&p_full[jj & 1], (jj >> 1) & 1, wc, SITE_P_FULL);
                    if (!ok) break;
                    ok = wait_bar(&v_full[s], (jj / C::NV) & 1, wc, SITE_V_FULL);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t tP = tbase + C::T_S + (jj & 1) * (2 * BN);
                    const uint32_t va = smem_addr(smem + C::OFF_V + s * C::VST_BYTES);
                    const uint32_t vda = va + C::NKB * BN * 128;
                    // O += P V
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(tbase + C::T_O, tP + kk * 8, sdesc_sw128(va + kk * 2048, BN * 128, 1024),
                               C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                    // O'_acc += P(sS' - c) V
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(tbase + C::T_OD, tP + BN + kk * 8,
                               sdesc_sw128(va + kk * 2048, BN * 128, 1024), C::IDESC_PV,
                               (jj > 0 || kk > 0) ? 1u : 0u);
                    // O'_acc += P V'
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(tbase + C::T_OD, tP + kk * 8, sdesc_sw128(vda + kk * 2048, BN * 128, 1024),
                               C::IDESC_PV, 1u);
                    mma_commit(&v_empty[s]);
                    mma_commit(o_done);
                }
            }
            if (!ok && issued) {
                mma_commit(drain);
                wait_bar(drain, 0, wc, SITE_DRAIN, false);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may touch
        const int r = quad * 32 + lane;
        const int st = tid - 64;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int grow = q0 + r;
        const size_t orow = (static_cast<size_t>(bh) * p.Lq + grow) * D;
        __nv_bfloat16 *o_ptr = static_cast<__nv_bfloat16 *>(p.o) + orow;
        __nv_bfloat16 *od_ptr = static_cast<__nv_bfloat16 *>(p.od) + orow;

        if (nT == 0) {
            if (grow < p.Lq) {
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    reinterpret_cast<uint4 *>(o_ptr)[c] = z;
                    reinterpret_cast<uint4 *>(od_ptr)[c] = z;
                }
                p.lse[static_cast<size_t>(bh) * p.Lq + grow] = -INFINITY;
            }
        } else {
            const float sl2 = p.sl2;
            const float sc = p.scale;
            const bool neg = sl2 < 0.f;
            float m_used = -INFINITY, l = 0.f, acc_a = 0.f, cctr = 0.f;
            bool ok = true;
            for (int j = 0; j < nT; ++j) {
                const int bsel = j & 1;
                ok = __all_sync(0xffffffffu, wait_bar(&s_full[bsel], (j >> 1) & 1, wc, SITE_S_FULL));
                if (!ok) break;
                tc_fence_after();
                const uint32_t tS = tbase + lane_off + C::T_S + bsel * (2 * BN);
                uint32_t ra[32], rb[32];
                tmem_ld32(tS, ra);
                tmem_ld32(tS + 32, rb);
                tmem_ld_wait2(ra, rb);
                float x[BN];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = u2f(ra[i]);
                    x[32 + i] = u2f(rb[i]);
                }
                const int valid = nb - j * BN;  // >= 1
                const bool tail = valid < BN;
                if (tail) {
                    const float pad = neg ? INFINITY : -INFINITY;
#pragma unroll
                    for (int i = 0; i < BN; ++i) x[i] = (i < valid) ? x[i] : pad;
                }
                float mx = x[0];
                if (neg) {
#pragma unroll
                    for (int i = 1; i < BN; ++i) mx = fminf(mx, x[i]);
                } else {
#pragma unroll
                    for (int i = 1; i < BN; ++i) mx = fmaxf(mx, x[i]);
                }
                const float m_tile = mx * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (j == 0) {
                    m_used = m_tile;
                } else if (m_tile > m_used + RESCALE_THRESHOLD) {
                    alpha = ex2_approx(m_used - m_tile);
                    m_used = m_tile;
                    rescale = true;
                }
                l *= alpha;
                acc_a *= alpha;
                const float nm = -m_used;
                float ps = 0.f;
#pragma unroll
                for (int i = 0; i < BN; ++i) {
                    x[i] = ex2_approx(fmaf(x[i], sl2, nm));
                    ps += x[i];
                }
                l += ps;

                uint32_t da[32], db[32];
                tmem_ld32(tS + BN, da);
                tmem_ld32(tS + BN + 32, db);
                tmem_ld_wait2(da, db);
                if (j == 0) {
                    float num = 0.f;
#pragma unroll
                    for (int i = 0; i < BN; ++i) {
                        const float sd = u2f(i < 32 ? da[i] : db[i - 32]) * sc;
                        num += (tail && i >= valid) ? 0.f : x[i] * sd;
                    }
                    cctr = num / ps;
                }
                uint32_t pk[32], pdk[32];
                float asum = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int c0 = 2 * i, c1 = 2 * i + 1;
                    const float s0 = fmaf(u2f(c0 < 32 ? da[c0] : db[c0 - 32]), sc, -cctr);
                    const float s1 = fmaf(u2f(c1 < 32 ? da[c1] : db[c1 - 32]), sc, -cctr);
                    float d0 = x[c0] * s0;
                    float d1 = x[c1] * s1;
                    if (tail) {
                        d0 = (c0 < valid) ? d0 : 0.f;
                        d1 = (c1 < valid) ? d1 : 0.f;
                    }
                    asum += d0 + d1;
                    pk[i] = pack_bf16x2(x[c0], x[c1]);
                    pdk[i] = pack_bf16x2(d0, d1);
                }
                acc_a += asum;

                if (j >= 1) {
                    // PV of the previous tile must be done before O may be rescaled;
                    // every phase of o_done is observed in order.
                    ok = __all_sync(0xffffffffu, wait_bar(o_done, (j - 1) & 1, wc, SITE_O_DONE));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < 2 * D; c += 32) {
                        uint32_t t[32];
                        tmem_ld32(tbase + lane_off + C::T_O + c, t);
                        tmem_ld_wait(t);
#pragma unroll
                        for (int i = 0; i < 32; ++i) t[i] = f2u(u2f(t[i]) * alpha);
                        tmem_st32(tbase + lane_off + C::T_O + c, t);
                    }
                }
                if (tail) {
                    // Zero the V and V' rows of padded keys so their bits (NaN
                    // included) cannot reach the P V products.
                    const int s = j % C::NV;
                    ok = __all_sync(0xffffffffu, wait_bar(&v_full[s], (j / C::NV) & 1, wc, SITE_V_TAIL));
                    if (!ok) break;
                    uint8_t *vst = smem + C::OFF_V + s * C::VST_BYTES;
                    const int nrow = BN - valid;
                    const int per_blk = nrow * 8;
                    const int chunks = 2 * C::NKB * per_blk;
                    for (int idx = st; idx < chunks; idx += 128) {
                        const int blk = idx / per_blk;
                        const int rem = idx - blk * per_blk;
                        const int row = valid + (rem >> 3);
                        *reinterpret_cast<uint4 *>(vst + blk * (BN * 128) + row * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tmem_st32(tS, pk);
                tmem_st32(tS + BN, pdk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[bsel]);
            }
            if (ok) ok = __all_sync(0xffffffffu, wait_bar(o_done, (nT - 1) & 1, wc, SITE_O_DONE));
            if (ok) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                const float coef = acc_a * inv_l;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ov[32], odv[32];
                    tmem_ld32(tbase + lane_off + C::T_O + c, ov);
                    tmem_ld32(tbase + lane_off + C::T_OD + c, odv);
                    tmem_ld_wait2(ov, odv);
                    uint32_t po[16], pod[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float a0 = u2f(ov[2 * i]), a1 = u2f(ov[2 * i + 1]);
                        const float b0 = u2f(odv[2 * i]), b1 = u2f(odv[2 * i + 1]);
                        po[i] = pack_bf16x2(a0 * inv_l, a1 * inv_l);
                        pod[i] = pack_bf16x2(fmaf(-coef, a0, b0) * inv_l, fmaf(-coef, a1, b1) * inv_l);
                    }
                    if (grow < p.Lq) {
                        uint4 *dst = reinterpret_cast<uint4 *>(o_ptr + c);
                        uint4 *dsd = reinterpret_cast<uint4 *>(od_ptr + c);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            dst[i] = make_uint4(po[4 * i], po[4 * i + 1], po[4 * i + 2], po[4 * i + 3]);
                            dsd[i] = make_uint4(pod[4 * i], pod[4 * i + 1], pod[4 * i + 2], pod[4 * i + 3]);
                        }
                    }
                }
                if (grow < p.Lq)
                    p.lse[static_cast<size_t>(bh) * p.Lq + grow] = (m_used + log2f(l)) * 0.69314718055994531f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
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
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// [BH, L, D] bf16 viewed as a 3-D tensor (D innermost); box 64 x rows x 1,
// 128-byte swizzle, zero fill past the end of each head.
static bool make_map(CUtensorMap *m, const void *base, int D, int L, long long BH, int rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(L) * D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), gdim, gstride, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int MAX_DEVICES = 64;

template <int D>
static int prepare_device(int dev)
{
    static std::mutex mu;
    static bool done[MAX_DEVICES] = {};
    if (dev < 0 || dev >= MAX_DEVICES) return ATTN_JVP_ERR_LAUNCH;
    std::lock_guard<std::mutex> g(mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(attn_jvp_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(Cfg<D>::SMEM_BYTES)) != cudaSuccess)
            return ATTN_JVP_ERR_LAUNCH;
        done[dev] = true;
    }
    return ATTN_JVP_OK;
}

static bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

static int launch(const void *q, const void *k, const void *v, const void *qd, const void *kd,
                  const void *vd, void *o, void *od, float *lse, int B, int H, int Lq, int Lk, int d,
                  float scale, const int32_t *kv_len, void *stream, uint64_t timeout_ns, int flags)
{
    if (!q || !k || !v || !qd || !kd || !vd || !o || !od || !lse) return ATTN_JVP_ERR_NULL;
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return ATTN_JVP_ERR_SHAPE;
    const long long BH = static_cast<long long>(B) * H;
    if (BH * Lq >= (1ll << 31) || BH * Lk >= (1ll << 31)) return ATTN_JVP_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_JVP_ERR_HEADDIM;
    const void *t16[8] = {q, k, v, qd, kd, vd, o, od};
    for (const void *t : t16)
        if (reinterpret_cast<uintptr_t>(t) & 15) return ATTN_JVP_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(kv_len) & 3))
        return ATTN_JVP_ERR_ALIGN;
    if (!std::isfinite(scale)) return ATTN_JVP_ERR_VALUE;
    const size_t nq = static_cast<size_t>(BH) * Lq * d * 2, nk = static_cast<size_t>(BH) * Lk * d * 2;
    const size_t nl = static_cast<size_t>(BH) * Lq * 4;
    const void *ins[6] = {q, k, v, qd, kd, vd};
    const size_t insz[6] = {nq, nk, nk, nq, nk, nk};
    const void *outs[3] = {o, od, lse};
    const size_t outsz[3] = {nq, nq, nl};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 6; ++j)
            if (ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return ATTN_JVP_ERR_VALUE;
        for (int j = i + 1; j < 3; ++j)
            if (ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return ATTN_JVP_ERR_VALUE;
    }

    const int nqt = (Lq + BM - 1) / BM;
    const long long grid = static_cast<long long>(nqt) * BH;
    if (grid > INT_MAX) return ATTN_JVP_ERR_SHAPE;

    Params prm;
    std::memset(&prm, 0, sizeof prm);
    if (!make_map(&prm.tm_q, q, d, Lq, BH, BM) || !make_map(&prm.tm_qd, qd, d, Lq, BH, BM) ||
        !make_map(&prm.tm_k, k, d, Lk, BH, BN) || !make_map(&prm.tm_kd, kd, d, Lk, BH, BN) ||
        !make_map(&prm.tm_v, v, d, Lk, BH, BN) || !make_map(&prm.tm_vd, vd, d, Lk, BH, BN))
        return ATTN_JVP_ERR_LAUNCH;
    prm.o = o;
    prm.od = od;
    prm.lse = lse;
    prm.kv_len = kv_len;
    prm.H = H;
    prm.Lq = Lq;
    prm.Lk = Lk;
    prm.nqt = nqt;
    prm.scale = scale;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.timeout_ns = timeout_ns ? timeout_ns : DEFAULT_TIMEOUT_NS;
    prm.flags = flags;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 64) {
        if (int rc = prepare_device<64>(dev)) return rc;
        attn_jvp_fwd_kernel<64><<<static_cast<unsigned>(grid), NTHREADS, Cfg<64>::SMEM_BYTES, s>>>(prm);
    } else {
        if (int rc = prepare_device<128>(dev)) return rc;
        attn_jvp_fwd_kernel<128><<<static_cast<unsigned>(grid), NTHREADS, Cfg<128>::SMEM_BYTES, s>>>(prm);
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    return ATTN_JVP_OK;
}

}  // namespace ajvp

extern "C" {

int attn_jvp_fwd(const void *q, const void *k, const void *v, const void *q_dot, const void *k_dot,
                 const void *v_dot, void *o, void *o_dot, float *lse, int B, int H, int Lq, int Lk,
                 int d, float scale, const int32_t *kv_len, void *stream)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, B, H, Lq, Lk, d, scale, kv_len,
                        stream, 0, 0);
}

int attn_jvp_fwd_debug(const void *q, const void *k, const void *v, const void *q_dot,
                       const void *k_dot, const void *v_dot, void *o, void *o_dot, float *lse, int B,
                       int H, int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *stream,
                       uint64_t timeout_ns, int flags)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, B, H, Lq, Lk, d, scale, kv_len,
                        stream, timeout_ns, flags);
}

int attn_jvp_check(void *stream, int *site)
{
    if (site) *site = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATTN_JVP_ERR_LAUNCH;
    int st = 0;
    if (cudaMemcpyFromSymbol(&st, ajvp::g_status, sizeof st) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (st == 0) return ATTN_JVP_OK;
    const int zero = 0;
    if (cudaMemcpyToSymbol(ajvp::g_status, &zero, sizeof zero) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (site) *site = st;
    return ATTN_JVP_ERR_TIMEOUT;
}

const char *attn_jvp_status_string(int status)
{
    switch (status) {
    case ATTN_JVP_OK: return "ok";
    case ATTN_JVP_ERR_NULL: return "a required pointer is NULL";
    case ATTN_JVP_ERR_SHAPE: return "B, H, Lq or Lk out of range";
    case ATTN_JVP_ERR_HEADDIM: return "head dimension must be 64 or 128";
    case ATTN_JVP_ERR_ALIGN: return "a tensor pointer is misaligned (bf16 tensors need 16 bytes)";
    case ATTN_JVP_ERR_LAUNCH: return "CUDA launch or runtime query failed";
    case ATTN_JVP_ERR_TIMEOUT: return "a device-side pipeline wait gave up";
    case ATTN_JVP_ERR_VALUE: return "scale not finite, or outputs overlap inputs";
    default: return "unknown status";
    }
}

int attn_jvp_version(void) { return 100; }

}  // extern "C"

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
//   * two warpgroups run the online softmax in registers, thread = query row,
//     each on one half of the tile's 64 key columns; they exchange partial row
//     maxima through shared memory.  Running max m (lazily rescaled),
//     denominator l = sum p and a = sum p (s S'_raw - c).  They write P and
//     P * (s S'_raw - c) back into TMEM as bf16 over the S columns;
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
constexpr int NSOFT = 256;                // softmax threads: two warpgroups (warps 2-9)
constexpr int BAR_SOFT = 1;               // named barrier of the softmax warpgroups
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 4.0f; // log2 units: rescale when the max grows by 2^4
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
    SITE_SMEM_ALIGN = 11,
};

// Two launch shapes share one kernel body:
//  - single CTA (PAIR = false): the CTA computes its own 128 x N MMAs;
//  - CTA pair (PAIR = true, d = 128): a cluster of two CTAs owns two adjacent
//    128-row query tiles of one (b, h); the leader issues M = 256 MMAs that
//    read A and write D in both CTAs while each CTA stages only half of every
//    B operand.  Per tile the leader loads K and the first 32 rows of K, the
//    peer loads K' and the last 32 rows of K, and each loads its 64-column half
//    of V and V'.  That halves the B-operand shared-memory reads, the TMA
//    writes and the L2 reads per SM.
template <int D, bool PAIR>
struct Cfg {
    static_assert(!PAIR || D == 128, "the CTA-pair layout splits V by 64-column halves of d = 128");
    static constexpr int NKB = D / 64;               // 128-byte column blocks per row
    static constexpr int NTHREADS = PAIR ? 352 : 320;  // + relay warp 10 in pair mode
    static constexpr int NCTA = PAIR ? 2 : 1;
    static constexpr int NK = PAIR ? 4 : ((D == 128) ? 3 : 4);  // K ring depth
    static constexpr int NV = PAIR ? 4 : ((D == 128) ? 2 : 4);  // V ring depth
    static constexpr uint32_t Q_BYTES = BM * D * 2;  // one of Q, Q' (per CTA)
    // K stage.  Single CTA: K then K' rows in each column block (one 128-row
    // operand [K; K']).  Pair: X (K in the leader, K' in the peer; 64 rows)
    // then Z (32 rows of K).
    static constexpr uint32_t X_BYTES = BN * D * 2;
    static constexpr uint32_t Z_BYTES = (BN / 2) * D * 2;
    static constexpr uint32_t KST_BYTES = PAIR ? X_BYTES + Z_BYTES : 2 * BN * D * 2;
    // V stage: V then V' (pair: this CTA's 64-column half of each)
    static constexpr uint32_t VHALF_BYTES = PAIR ? BN * 64 * 2 : BN * D * 2;
    static constexpr uint32_t VST_BYTES = 2 * VHALF_BYTES;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_QD = Q_BYTES;
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NK * KST_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + NV * VST_BYTES;
    // q_full, k_full[NK], k_empty[NK], v_full[NV], v_ready[NV], v_empty[NV],
    // s_full[2], p_full[2], pd_full[2], o_done, drain
    static constexpr int NBAR = 1 + 2 * NK + 3 * NV + 2 + 2 + 2 + 1 + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr uint32_t OFF_XCH = OFF_MISC + 16;  // float [2][2][128]
    static constexpr uint32_t SMEM_BYTES = OFF_XCH + 2 * 2 * 128 * 4;
    // TMEM columns: O | O'_acc | S buffer 0 (S, S'_raw) | S buffer 1.  Both
    // softmax warpgroups read all of S (the row max) but only their own half
    // of S'_raw, columns [BN + 32g, BN + 32g + 32).  Warpgroup g writes its
    // bf16 P (keys 32g..32g+31, two per column) over the first 16 of those
    // columns and P (sS' - c) over the last 16, so no one overwrites a
    // column another warp may still read.
    static constexpr uint32_t T_O = 0;
    static constexpr uint32_t T_OD = D;
    static constexpr uint32_t T_S = 2 * D;
    // column of the bf16 P (pd = false) or P (sS' - c) (pd = true) operand of
    // keys 16kk..16kk+15 inside an S buffer
    __host__ __device__ static constexpr uint32_t t_pk(int kk, bool pd) { return BN + (kk >> 1) * 32 + (pd ? 16 : 0) + (kk & 1) * 8; }
    static constexpr int MMA_M = BM * NCTA;
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(MMA_M, 2 * BN, false);
    static constexpr uint32_t IDESC_SD = idesc_bf16_f32(MMA_M, BN, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(MMA_M, D, true);
    static constexpr int P_ARRIVALS = 8 * NCTA;  // one per softmax warp
    static_assert(T_S + 4 * BN <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Params {
    CUtensorMap tm_q, tm_qd, tm_k, tm_kd, tm_v, tm_vd, tm_k32;
    void *o;
    void *od;
    float *lse;
    float *lse_dot;  // NULL: not computed
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
// cluster_scope: acquire at cluster scope (barriers the peer CTA signals).
__device__ __noinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const WaitCtx &c, int site,
                                      bool honor_abort = true, bool cluster_scope = false)
{
    const uint32_t a = smem_addr(bar);
    auto probe = [&]() { return cluster_scope ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity); };
    if (probe()) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (probe()) return true;
        if (honor_abort && *c.abort) return false;
        if (globaltimer_ns() - t0 > c.limit_ns) {
            *c.abort = 1;
            atomicCAS(&g_status, 0, site);
            return false;
        }
    }
}

// One inline probe before falling back to the bounded loop.
__device__ __forceinline__ bool wait_bar_fast(uint64_t *bar, uint32_t parity, const WaitCtx &c, int site,
                                              bool cluster_scope)
{
    const uint32_t a = smem_addr(bar);
    if (cluster_scope ? mbar_test_wait_cluster(a, parity) : mbar_test_wait(a, parity)) return true;
    return wait_bar(bar, parity, c, site, true, cluster_scope);
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// Max (or min) of the 64 floats held as bits in a and b, as a balanced tree
// of 3-input operations (32 of them).  Exact, so the order of the two halves
// does not change the result.
template <bool MIN>
__device__ __forceinline__ float row_ext64(const uint32_t (&a)[32], const uint32_t (&b)[32])
{
    auto op = [](float x, float y, float z) { return MIN ? min3f(x, y, z) : max3f(x, y, z); };
    float t[16], u[8], w[4];
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = op(u2f(a[2 * i]), u2f(a[2 * i + 1]), u2f(b[2 * i]));
#pragma unroll
    for (int k = 0; k < 8; ++k) u[k] = op(t[2 * k], t[2 * k + 1], u2f(b[4 * k + 1]));
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = op(u[2 * k], u[2 * k + 1], u2f(b[8 * k + 3]));
    const float y0 = op(w[0], w[1], u2f(b[7]));
    const float y1 = op(w[2], w[3], u2f(b[23]));
    const float z = op(y0, y1, u2f(b[15]));
    return MIN ? fminf(z, u2f(b[31])) : fmaxf(z, u2f(b[31]));
}
__device__ __forceinline__ float row_max64(const uint32_t (&a)[32], const uint32_t (&b)[32])
{
    return row_ext64<false>(a, b);
}
__device__ __forceinline__ float row_min64(const uint32_t (&a)[32], const uint32_t (&b)[32])
{
    return row_ext64<true>(a, b);
}

// ZKV: K' = V' = 0 (frozen keys and values, e.g. text tokens).  Then S'_raw
// = Q' K^T and O' = P' V: the K' and V' tiles are neither loaded nor
// multiplied, 8 of the 12 FLOP units remain.
template <int D, bool PAIR, bool ZKV>
__global__ void __launch_bounds__(Cfg<D, PAIR>::NTHREADS, 1)
    attn_jvp_fwd_kernel(const __grid_constant__ Params p)
{
    static_assert(!(PAIR && ZKV), "the CTA-pair layout always carries K' and V'");
    using C = Cfg<D, PAIR>;
    extern __shared__ __align__(1024) uint8_t smem[];
    // The 128-byte swizzle atoms must start on 1024-byte boundaries.  The
    // dynamic window is 1024-aligned in practice; if it ever is not, record it
    // and do nothing rather than compute garbage (both CTAs of a pair see the
    // same layout, so both return here).
    if (smem_addr(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(&g_status, 0, SITE_SMEM_ALIGN);
        return;
    }

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    int qt, bh;
    if constexpr (PAIR) {
        const int nqp = (p.nqt + 1) >> 1;  // query-tile pairs per (b, h)
        const int pair = blockIdx.x >> 1;
        qt = 2 * (pair % nqp) + static_cast<int>(rank);
        bh = pair / nqp;
    } else {
        qt = blockIdx.x % p.nqt;
        bh = blockIdx.x / p.nqt;
    }
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
    uint64_t *v_ready = v_full + C::NV;
    uint64_t *v_empty = v_ready + C::NV;
    uint64_t *s_full = v_empty + C::NV;
    uint64_t *p_full = s_full + 2;   // [2] bf16 P written
    uint64_t *pd_full = p_full + 2;  // [2] bf16 P (sS' - c) written
    uint64_t *o_done = pd_full + 2;
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
            mbar_init(&v_ready[s], C::NCTA);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], C::P_ARRIVALS);
            mbar_init(&pd_full[s], C::P_ARRIVALS);
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
        tma_prefetch_desc(&p.tm_v);
        if (!ZKV) {
            tma_prefetch_desc(&p.tm_kd);
            tma_prefetch_desc(&p.tm_vd);
        }
        if (PAIR) tma_prefetch_desc(&p.tm_k32);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(tmem_slot, TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if constexpr (PAIR) {
        cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
    } else {
        __syncthreads();
    }
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const WaitCtx wc{abort_flag, p.timeout_ns};
    // cluster addresses of the leader's barriers that both CTAs signal
    const uint32_t q_full_lead = PAIR ? mapa_shared(smem_addr(q_full), 0) : smem_addr(q_full);
    const uint32_t k_full_lead = PAIR ? mapa_shared(smem_addr(k_full), 0) : smem_addr(k_full);
    const uint32_t v_ready_lead = PAIR ? mapa_shared(smem_addr(v_ready), 0) : smem_addr(v_ready);
    const uint32_t p_full_lead = PAIR ? mapa_shared(smem_addr(p_full), 0) : smem_addr(p_full);
    const uint32_t pd_full_lead = PAIR ? mapa_shared(smem_addr(pd_full), 0) : smem_addr(pd_full);
    (void)v_ready_lead;
    (void)p_full_lead;
    (void)pd_full_lead;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && nT > 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            const bool load_q = !(p.flags & ATTN_JVP_DEBUG_STARVE_Q);
            if (load_q) {
                if constexpr (PAIR) {
                    // the leader's barrier counts both CTAs' Q and Q' bytes
                    if (leader) mbar_arrive_expect_tx(q_full, 2 * 2 * C::Q_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NKB; ++c) {
                        tma_load_3d_pair(smem + C::OFF_Q + c * BM * 128, &p.tm_q, q_full_lead, c * 64, q0, bh,
                                         pol_q);
                        tma_load_3d_pair(smem + C::OFF_QD + c * BM * 128, &p.tm_qd, q_full_lead, c * 64, q0,
                                         bh, pol_q);
                    }
                } else {
                    mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NKB; ++c) {
                        tma_load_3d(smem + C::OFF_Q + c * BM * 128, &p.tm_q, q_full, c * 64, q0, bh, pol_q);
                        tma_load_3d(smem + C::OFF_QD + c * BM * 128, &p.tm_qd, q_full, c * 64, q0, bh,
                                    pol_q);
                    }
                }
            }
            int nk = 0, nv = 0;
            bool ok = true;
            for (int j = 0; j <= nT && ok; ++j) {
                if (j < nT) {
                    const int s = j % C::NK;
                    if (j >= C::NK)
                        ok = wait_bar(&k_empty[s], ((j / C::NK) - 1) & 1, wc, SITE_K_EMPTY, true, PAIR);
                    if (!ok) break;
                    uint8_t *dst = smem + C::OFF_K + s * C::KST_BYTES;
                    if constexpr (PAIR) {
                        if (leader) mbar_arrive_expect_tx(&k_full[s], 2 * C::KST_BYTES);
                        const uint32_t bar = k_full_lead + s * 8;
                        const CUtensorMap *mx = leader ? &p.tm_k : &p.tm_kd;
#pragma unroll
                        for (int c = 0; c < C::NKB; ++c) {
                            tma_load_3d_pair(dst + c * (BN * 128), mx, bar, c * 64, j * BN, bh, pol_kv);
                            tma_load_3d_pair(dst + C::X_BYTES + c * (BN / 2 * 128), &p.tm_k32, bar, c * 64,
                                             j * BN + static_cast<int>(rank) * (BN / 2), bh, pol_kv);
                        }
                    } else {
                        mbar_arrive_expect_tx(&k_full[s], ZKV ? C::KST_BYTES / 2 : C::KST_BYTES);
#pragma unroll
                        for (int c = 0; c < C::NKB; ++c) {
                            tma_load_3d(dst + c * (2 * BN * 128), &p.tm_k, &k_full[s], c * 64, j * BN, bh,
                                        pol_kv);
                            if (!ZKV)
                                tma_load_3d(dst + c * (2 * BN * 128) + BN * 128, &p.tm_kd, &k_full[s], c * 64,
                                            j * BN, bh, pol_kv);
                        }
                    }
                    ++nk;
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s = jj % C::NV;
                    if (jj >= C::NV)
                        ok = wait_bar(&v_empty[s], ((jj / C::NV) - 1) & 1, wc, SITE_V_EMPTY, true, PAIR);
                    if (!ok) break;
                    uint8_t *dst = smem + C::OFF_V + s * C::VST_BYTES;
                    mbar_arrive_expect_tx(&v_full[s], ZKV ? C::VHALF_BYTES : C::VST_BYTES);
                    if constexpr (PAIR) {
                        // this CTA's 64-column half of V and V' (local barrier)
                        const int c0 = static_cast<int>(rank) * 64;
                        tma_load_3d(dst, &p.tm_v, &v_full[s], c0, jj * BN, bh, pol_kv);
                        tma_load_3d(dst + C::VHALF_BYTES, &p.tm_vd, &v_full[s], c0, jj * BN, bh, pol_kv);
                    } else {
#pragma unroll
                        for (int c = 0; c < C::NKB; ++c) {
                            tma_load_3d(dst + c * (BN * 128), &p.tm_v, &v_full[s], c * 64, jj * BN, bh, pol_kv);
                            if (!ZKV)
                                tma_load_3d(dst + (C::NKB + c) * (BN * 128), &p.tm_vd, &v_full[s], c * 64,
                                            jj * BN, bh, pol_kv);
                        }
                    }
                    ++nv;
                }
            }
            // Let every load land before the CTA can exit.  In a pair the K
            // and Q bytes of both CTAs are counted on the leader's barriers,
            // so the leader waits for them; the final cluster barrier keeps
            // the peer alive until then.
            if (load_q && leader) wait_bar(q_full, 0, wc, SITE_DRAIN, false, PAIR);
            if (leader) {
                for (int s = 0; s < C::NK && s < nk; ++s) {
                    const int t = s + ((nk - 1 - s) / C::NK) * C::NK;
                    wait_bar(&k_full[s], (t / C::NK) & 1, wc, SITE_DRAIN, false, PAIR);
                }
            }
            for (int s = 0; s < C::NV && s < nv; ++s) {
                const int t = s + ((nv - 1 - s) / C::NV) * C::NV;
                wait_bar(&v_full[s], (t / C::NV) & 1, wc, SITE_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // The whole warp runs this loop (barrier tests and branches are
        // warp-uniform); one elected lane issues each MMA and commit.
        if (nT > 0 && leader) {
            bool ok = __all_sync(0xffffffffu, wait_bar(q_full, 0, wc, SITE_Q_FULL, true, PAIR));
            bool issued = false;
            if (ok) tc_fence_after();
            // Operand descriptors are built once per buffer; the per-MMA
            // offsets are added to the start-address field (all shared
            // addresses fit its 18 bits), which keeps the issue loop short.
            const uint64_t dq = sdesc_sw128(smem_addr(smem + C::OFF_Q), 16, 1024);
            const uint64_t dqd = sdesc_sw128(smem_addr(smem + C::OFF_QD), 16, 1024);
            // Fixed order S_0, S_1, PV_0, S_2, PV_1, ...: S_{j+1} runs on the
            // tensor core while the softmax works on tile j, and S_{j+1}
            // overwrites the TMEM buffer that held P_{j-1} only after PV_{j-1}
            // was issued (MMAs run in issue order).  Each wait first parks the
            // warp in mbarrier.try_wait, which wakes it when the phase completes.
            auto wait_u = [&](uint64_t *bar, uint32_t parity, int site) {
                const uint32_t a = smem_addr(bar);
                bool r = PAIR ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity);
                if (!__all_sync(0xffffffffu, r)) r = wait_bar(bar, parity, wc, site, true, PAIR);
                return __all_sync(0xffffffffu, r);
            };
            auto issue_s = [&](const int j) {
                const int s = j % C::NK;
                tc_fence_after();
                const uint32_t tS = tbase + C::T_S + (j & 1) * (2 * BN);
                const uint64_t dk = sdesc_sw128(smem_addr(smem + C::OFF_K + s * C::KST_BYTES), 16, 1024);
                if constexpr (PAIR) {
                    // S | Q K'^T = Q [K ; K']^T: B rows 0-63 (K) in the leader, 64-127 (K') in the peer
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                        mma_ss_pair(tS, desc_add(dq, oa), desc_add(dk, ob),
                                    C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    // += Q' K^T: B rows 0-31 of K in the leader, 32-63 in the peer
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = C::X_BYTES + (kk >> 2) * (BN / 2 * 128) + (kk & 3) * 32;
                        mma_ss_pair(tS + BN, desc_add(dqd, oa), desc_add(dk, ob),
                                    C::IDESC_SD, 1u);
                    }
                    mma_commit_pair_mc(&k_empty[s], 0x3);
                    mma_commit_pair_mc(&s_full[j & 1], 0x3);
                } else {
                    // S | Q K'^T  =  Q [K ; K']^T   (N = 2 BN); with K' = 0 only
                    // S = Q K^T (N = BN)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                        mma_ss(tS, desc_add(dq, oa), desc_add(dk, ob),
                               ZKV ? C::IDESC_SD : C::IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    // += Q' K^T into the second half (with K' = 0 it starts it)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                        mma_ss(tS + BN, desc_add(dqd, oa), desc_add(dk, ob),
                               C::IDESC_SD, (!ZKV || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&k_empty[s]);
                    mma_commit(&s_full[j & 1]);
                }
                issued = true;
            };
            // LBO: distance between 64-column blocks of V (single CTA, d = 128);
            // a pair CTA holds one block, so it is unused there
            constexpr uint32_t LBO = BN * 128;
            // PV_j in two groups: A needs only P (O += P V, O'_acc += P V'),
            // B needs P (sS' - c) as well (O'_acc += P (sS' - c) V), which the
            // softmax writes later; A can then start while B's operand is formed.
            auto issue_pa = [&](const int jj) {
                const int s = jj % C::NV;
                tc_fence_after();
                const uint32_t tP = tbase + C::T_S + (jj & 1) * (2 * BN);
                const uint64_t dv = sdesc_sw128(smem_addr(smem + C::OFF_V + s * C::VST_BYTES), LBO, 1024);
                const uint64_t dvd = desc_add(dv, C::VHALF_BYTES);
                (void)dvd;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {  // O += P V
                    const uint32_t a = tP + C::t_pk(kk, false);
                    const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (PAIR) mma_ts_pair(tbase + C::T_O, a, desc_add(dv, kk * 2048), C::IDESC_PV, acc);
                    else mma_ts(tbase + C::T_O, a, desc_add(dv, kk * 2048), C::IDESC_PV, acc);
                }
                if constexpr (!ZKV) {
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {  // O'_acc += P V'
                        const uint32_t a = tP + C::t_pk(kk, false);
                        const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (PAIR) mma_ts_pair(tbase + C::T_OD, a, desc_add(dvd, kk * 2048), C::IDESC_PV, acc);
                        else mma_ts(tbase + C::T_OD, a, desc_add(dvd, kk * 2048), C::IDESC_PV, acc);
                    }
                }
            };
            auto issue_pb = [&](const int jj) {
                const int s = jj % C::NV;
                tc_fence_after();
                const uint32_t tP = tbase + C::T_S + (jj & 1) * (2 * BN);
                const uint64_t dv = sdesc_sw128(smem_addr(smem + C::OFF_V + s * C::VST_BYTES), LBO, 1024);
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {  // O'_acc += P(sS' - c) V
                    const uint32_t a = tP + C::t_pk(kk, true);
                    // with V' = 0 this group starts O'_acc
                    const uint32_t acc = (!ZKV || jj > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (PAIR) mma_ts_pair(tbase + C::T_OD, a, desc_add(dv, kk * 2048), C::IDESC_PV, acc);
                    else mma_ts(tbase + C::T_OD, a, desc_add(dv, kk * 2048), C::IDESC_PV, acc);
                }
                if constexpr (PAIR) {
                    mma_commit_pair_mc(&v_empty[s], 0x3);
                    mma_commit_pair_mc(o_done, 0x3);
                } else {
                    mma_commit(&v_empty[s]);
                    mma_commit(o_done);
                }
            };
            if (ok) ok = wait_u(&k_full[0], 0, SITE_K_FULL);
            if (ok) issue_s(0);
            for (int j = 0; ok && j < nT; ++j) {
                if (j + 1 < nT) {
                    ok = wait_u(&k_full[(j + 1) % C::NK], ((j + 1) / C::NK) & 1, SITE_K_FULL);
                    if (!ok) break;
                    issue_s(j + 1);
                }
                // V_j normally lands before P_j is written: wait for it first
                ok = wait_u(PAIR ? &v_ready[j % C::NV] : &v_full[j % C::NV], (j / C::NV) & 1, SITE_V_FULL);
                if (ok) ok = wait_u(&p_full[j & 1], (j >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                issue_pa(j);
                ok = wait_u(&pd_full[j & 1], (j >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                issue_pb(j);
            }
            if (!ok && issued) {
                if constexpr (PAIR) mma_commit_pair_mc(drain, 0x1);
                else mma_commit(drain);
                wait_bar(drain, 0, wc, SITE_DRAIN, false, PAIR);
            }
        }
        __syncwarp();
    } else if (PAIR && warp == 10) {
        // ------------------------------------------------------------ V relay (pair)
        // Each CTA's V/V' half lands on a local barrier.  This warp zeroes the
        // rows of padded keys in the tail tile (their bits, NaN included, must
        // not reach the PV products) and then tells the leader's MMA warp.
        bool ok = true;
        for (int j = 0; j < nT && ok; ++j) {
            const int s = j % C::NV;
            const bool landed = wait_bar(&v_full[s], (j / C::NV) & 1, wc, SITE_V_TAIL);
            ok = __all_sync(0xffffffffu, landed);
            if (!ok) break;
            const int vt = nb - j * BN;
            if (vt < BN) {
                uint8_t *vst = smem + C::OFF_V + s * C::VST_BYTES;
                const int chunks = 2 * (BN - vt) * 8;  // 16-byte chunks: V and V' rows vt..BN-1
                for (int idx = lane; idx < chunks; idx += 32) {
                    const int half = idx / ((BN - vt) * 8);
                    const int rem = idx - half * ((BN - vt) * 8);
                    *reinterpret_cast<uint4 *>(vst + half * C::VHALF_BYTES + (vt + (rem >> 3)) * 128 +
                                               (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(v_ready_lead + s * 8);
        }
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------------------ softmax + epilogue
        // Two warpgroups, thread = query row.  Warpgroup g owns key columns
        // [32g, 32g + 32) of every tile; at the end it writes output g
        // (0: O and lse, 1: O').
        const int g = (warp - 2) >> 2;
        const int quad = warp & 3;  // TMEM lane quadrant this warp may touch
        const int r = quad * 32 + lane;
        const int gt = tid - 64 - g * 128;  // thread index inside the warpgroup
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int grow = q0 + r;
        const size_t orow = (static_cast<size_t>(bh) * p.Lq + grow) * D;
        __nv_bfloat16 *out_ptr = static_cast<__nv_bfloat16 *>(g == 0 ? p.o : p.od) + orow;
        float *xch = reinterpret_cast<float *>(smem + C::OFF_XCH);  // [slot][warpgroup][row]

        if (nT == 0) {
            if (grow < p.Lq) {
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4 *>(out_ptr)[c] = z;
                if (g == 0) p.lse[static_cast<size_t>(bh) * p.Lq + grow] = -INFINITY;
                if (g == 1 && p.lse_dot) p.lse_dot[static_cast<size_t>(bh) * p.Lq + grow] = 0.f;
            }
        } else {
            const float sl2 = p.sl2;
            const float sc = p.scale;
            const bool neg = sl2 < 0.f;
            const int c0 = 32 * g;
            // l: exact fp32 sum of p (normalises O and O', gives lse);
            // acc_a: sum of the bf16-rounded P (sS' - c) that the MMAs consume,
            // so the rounding of those operands reaches O' only through
            // (v_j - O), which is small for the keys that dominate.
            float m_used = -INFINITY, l = 0.f, acc_a = 0.f, cctr = 0.f;
            // No named barrier inside the loop: every thread reads the whole
            // 64-column row of S and forms the same row max, so the two
            // warpgroups need not meet, and each warp runs through the tiles
            // at its own pace, coupled only by the MMA barriers.  A wait that
            // gives up sets `err` and leaves the loop; the barrier after the
            // loop is reached by all 256 threads either way.
            bool err = false;
            for (int j = 0; j < nT; ++j) {
                const int bsel = j & 1;
                const uint32_t tS = tbase + lane_off + C::T_S + bsel * (2 * BN);
                if (!__all_sync(0xffffffffu, wait_bar_fast(&s_full[bsel], (j >> 1) & 1, wc, SITE_S_FULL, PAIR))) {
                    err = true;
                    if (j == 0) bar_and(BAR_SOFT, NSOFT, false);  // the others wait there at tile 0
                    break;
                }
                tc_fence_after();
                const int vt = nb - j * BN;          // valid keys in the tile
                const int valid = vt - c0;           // valid columns of this half
                const bool tail = vt < BN;
                float mx;
                uint32_t ra[32];
                {
                    uint32_t rb[32];
                    tmem_ld32(tS + c0, ra);         // S, this half
                    tmem_ld32(tS + (c0 ^ 32), rb);  // S, the other half (row max only)
                    tmem_ld_wait2(ra, rb);
                    if (tail) {
                        const float pad = neg ? INFINITY : -INFINITY;
                        const int valid_o = vt - (c0 ^ 32);
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            ra[i] = (i < valid) ? ra[i] : f2u(pad);
                            rb[i] = (i < valid_o) ? rb[i] : f2u(pad);
                        }
                    }
                    mx = neg ? row_min64(ra, rb) : row_max64(ra, rb);
                }
                uint32_t rd[32];
                tmem_ld32(tS + BN + c0, rd);  // S'_raw, this half (waited for below)
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
                float x[32];
                // p = 2^(s * log2(e) * S - m), in pairs
                {
                    const uint64_t sl22 = f2_pack(sl2, sl2);
                    const uint64_t nm2 = f2_pack(-m_used, -m_used);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float t0, t1;
                        f2_unpack(f2_fma(f2_pack(u2f(ra[2 * i]), u2f(ra[2 * i + 1])), sl22, nm2), t0, t1);
                        x[2 * i] = ex2_approx(t0);
                        x[2 * i + 1] = ex2_approx(t1);
                    }
                }
                if (tail) {
                    // padded keys: p = 0 exactly (the pad times a zero scale is NaN)
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = (i < valid) ? x[i] : 0.f;
                }
                {
                    uint64_t s0 = f2_pack(x[0], x[1]), s1 = f2_pack(x[2], x[3]);
#pragma unroll
                    for (int i = 2; i < 16; i += 2) {
                        s0 = f2_add(s0, f2_pack(x[2 * i], x[2 * i + 1]));
                        s1 = f2_add(s1, f2_pack(x[2 * i + 2], x[2 * i + 3]));
                    }
                    float u0, u1, u2, u3;
                    f2_unpack(s0, u0, u1);
                    f2_unpack(s1, u2, u3);
                    l += (u0 + u1) + (u2 + u3);
                }
                tmem_ld_wait(rd);
                if (j == 0) {
                    // centring constant c: the p-weighted mean of s S' over the
                    // first 32 keys (warpgroup 0's half, which always holds a
                    // valid key), handed to warpgroup 1 through shared memory
                    if (g == 0) {
                        float n0 = 0.f, n1 = 0.f, w0 = 0.f, w1 = 0.f;
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            n0 += (tail && i >= valid) ? 0.f : x[i] * (u2f(rd[i]) * sc);
                            n1 += (tail && i + 1 >= valid) ? 0.f : x[i + 1] * (u2f(rd[i + 1]) * sc);
                            w0 += x[i];
                            w1 += x[i + 1];
                        }
                        cctr = (n0 + n1) / (w0 + w1);
                        xch[r] = cctr;
                    }
                    if (!bar_and(BAR_SOFT, NSOFT, true)) {
                        err = true;
                        break;
                    }
                    if (g == 1) cctr = xch[r];
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                if (j >= 1) {
                    // PV of the previous tile must be done before O may be
                    // rescaled; every warp observes every phase of o_done in
                    // order (o_done(j) needs this warp's P of tile j).
                    if (!__all_sync(0xffffffffu, wait_bar_fast(o_done, (j - 1) & 1, wc, SITE_O_DONE, PAIR))) {
                        err = true;
                        break;
                    }
                    tc_fence_after();
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    const uint32_t tacc = tbase + lane_off + (g == 0 ? C::T_O : C::T_OD);
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t t[32];
                        tmem_ld32(tacc + c, t);
                        tmem_ld_wait(t);
#pragma unroll
                        for (int i = 0; i < 32; ++i) t[i] = f2u(u2f(t[i]) * alpha);
                        tmem_st32(tacc + c, t);
                    }
                }
                if (!PAIR && tail && !(ZKV && g == 1)) {  // (no V' tile with V' = 0)
                    // Zero the V (g = 0) / V' (g = 1) rows of padded keys so
                    // their bits (NaN included) cannot reach the PV products.
                    // Each warp zeroes its share and fences before it signals P.
                    const int s = j % C::NV;
                    if (!__all_sync(0xffffffffu, wait_bar(&v_full[s], (j / C::NV) & 1, wc, SITE_V_TAIL))) {
                        err = true;
                        break;
                    }
                    uint8_t *vst = smem + C::OFF_V + s * C::VST_BYTES + g * (C::NKB * BN * 128);
                    const int nrow = BN - vt;
                    const int per_blk = nrow * 8;
                    const int chunks = C::NKB * per_blk;
                    for (int idx = gt; idx < chunks; idx += 128) {
                        const int blk = idx / per_blk;
                        const int rem = idx - blk * per_blk;
                        const int row = vt + (rem >> 3);
                        *reinterpret_cast<uint4 *>(vst + blk * (BN * 128) + row * 128 + (rem & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                // P over the first 16 columns of this half of S'_raw (read above)
                tmem_st16(tS + BN + c0, pk);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) mbar_arrive_cluster(p_full_lead + bsel * 8);
                    else mbar_arrive(&p_full[bsel]);
                }
                // ---- bf16 P (s S' - c) while the tensor core multiplies P
                uint32_t pdk[16];
                {
                    const uint64_t sc2 = f2_pack(sc, sc);
                    const uint64_t nc2 = f2_pack(-cctr, -cctr);
                    uint64_t a0 = 0, a1 = 0;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint64_t p2 = f2_pack(x[2 * i], x[2 * i + 1]);
                        const uint64_t d2 = f2_mul(f2_fma(f2_pack(u2f(rd[2 * i]), u2f(rd[2 * i + 1])), sc2, nc2), p2);
                        float d0, d1;
                        f2_unpack(d2, d0, d1);
                        if (tail) {
                            d0 = (2 * i < valid) ? d0 : 0.f;
                            d1 = (2 * i + 1 < valid) ? d1 : 0.f;
                        }
                        pdk[i] = pack_bf16x2(d0, d1);
                        // the two rounded values as fp32
                        const uint64_t r2 = f2_pack(u2f(pdk[i] << 16), u2f(pdk[i] & 0xFFFF0000u));
                        if (i & 1) a1 = f2_add(a1, r2);
                        else a0 = f2_add(a0, r2);
                    }
                    float u0, u1, u2, u3;
                    f2_unpack(a0, u0, u1);
                    f2_unpack(a1, u2, u3);
                    acc_a += (u0 + u1) + (u2 + u3);
                }
                tmem_st16(tS + BN + c0 + 16, pdk);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR) mbar_arrive_cluster(pd_full_lead + bsel * 8);
                    else mbar_arrive(&pd_full[bsel]);
                }
            }
            bool ok;
            {
                bool done = false;
                if (!err) done = wait_bar(o_done, (nT - 1) & 1, wc, SITE_O_DONE, true, PAIR);
                ok = bar_and(BAR_SOFT, NSOFT, done);  // reached by all 256 threads
            }
            if (ok) {
                tc_fence_after();
                // l and a are split across the two warpgroups; add the halves
                // in a fixed order so both see the same totals.
                xch[g * 128 + r] = l;
                xch[256 + g * 128 + r] = acc_a;
                bar_sync(BAR_SOFT, NSOFT);
                const float lt = xch[r] + xch[128 + r];
                const float inv_l = 1.f / lt;
                const float coef = (xch[256 + r] + xch[384 + r]) * inv_l;
                const uint32_t to = tbase + lane_off + C::T_O;
                const uint32_t tod = tbase + lane_off + C::T_OD;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t ov[32], odv[32];
                    uint32_t pv[16];
                    if (g == 0) {
                        tmem_ld32(to + c, ov);
                        tmem_ld_wait(ov);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pv[i] = pack_bf16x2(u2f(ov[2 * i]) * inv_l, u2f(ov[2 * i + 1]) * inv_l);
                    } else {
                        tmem_ld32(to + c, ov);
                        tmem_ld32(tod + c, odv);
                        tmem_ld_wait2(ov, odv);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pv[i] = pack_bf16x2(fmaf(-coef, u2f(ov[2 * i]), u2f(odv[2 * i])) * inv_l,
                                                fmaf(-coef, u2f(ov[2 * i + 1]), u2f(odv[2 * i + 1])) * inv_l);
                    }
                    if (grow < p.Lq) {
                        uint4 *dst = reinterpret_cast<uint4 *>(out_ptr + c);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pv[4 * i], pv[4 * i + 1], pv[4 * i + 2], pv[4 * i + 3]);
                    }
                }
                if (g == 0 && grow < p.Lq)
                    p.lse[static_cast<size_t>(bh) * p.Lq + grow] = (m_used + log2f(lt)) * 0.69314718055994531f;
                // lse' = sum_j P_j s S'_j = c + a / l
                if (g == 1 && p.lse_dot && grow < p.Lq)
                    p.lse_dot[static_cast<size_t>(bh) * p.Lq + grow] = cctr + coef;
            }
        }
    }

    tc_fence_before();
    if constexpr (PAIR) {
        // Neither CTA may leave while the leader's MMAs can still read the
        // peer's shared memory or TMEM, or loads can still signal the leader.
        cluster_sync();
    } else {
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tbase, TMEM_COLS);
        else tmem_dealloc(tbase, TMEM_COLS);
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

template <int D, bool PAIR, bool ZKV>
static int prepare_device(int dev)
{
    static std::mutex mu;
    static bool done[MAX_DEVICES] = {};
    if (dev < 0 || dev >= MAX_DEVICES) return ATTN_JVP_ERR_LAUNCH;
    std::lock_guard<std::mutex> g(mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(attn_jvp_fwd_kernel<D, PAIR, ZKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(Cfg<D, PAIR>::SMEM_BYTES)) != cudaSuccess)
            return ATTN_JVP_ERR_LAUNCH;
        done[dev] = true;
    }
    return ATTN_JVP_OK;
}

template <int D, bool PAIR, bool ZKV>
static int launch_kernel(const Params &prm, long long grid, cudaStream_t s)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (int rc = prepare_device<D, PAIR, ZKV>(dev)) return rc;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(Cfg<D, PAIR>::NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<D, PAIR>::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (PAIR) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, attn_jvp_fwd_kernel<D, PAIR, ZKV>, prm) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    return ATTN_JVP_OK;
}

static bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// allow_zero_kv: k_dot and v_dot may both be NULL (K' = V' = 0).
static int launch(const void *q, const void *k, const void *v, const void *qd, const void *kd,
                  const void *vd, void *o, void *od, float *lse, float *lse_dot, int B, int H, int Lq,
                  int Lk, int d, float scale, const int32_t *kv_len, void *stream, uint64_t timeout_ns,
                  int flags, bool allow_zero_kv)
{
    const bool zkv = allow_zero_kv && !kd && !vd;
    if (!q || !k || !v || !qd || (!zkv && (!kd || !vd)) || !o || !od || !lse) return ATTN_JVP_ERR_NULL;
    if (flags & ~(ATTN_JVP_DEBUG_STARVE_Q | ATTN_JVP_DEBUG_CTA_PAIR)) return ATTN_JVP_ERR_VALUE;
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return ATTN_JVP_ERR_SHAPE;
    const long long BH = static_cast<long long>(B) * H;
    if (BH * Lq >= (1ll << 31) || BH * Lk >= (1ll << 31)) return ATTN_JVP_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_JVP_ERR_HEADDIM;
    const void *t16[8] = {q, k, v, qd, kd, vd, o, od};
    for (const void *t : t16)
        if (reinterpret_cast<uintptr_t>(t) & 15) return ATTN_JVP_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(lse) & 3) || (reinterpret_cast<uintptr_t>(lse_dot) & 3) ||
        (reinterpret_cast<uintptr_t>(kv_len) & 3))
        return ATTN_JVP_ERR_ALIGN;
    if (!std::isfinite(scale)) return ATTN_JVP_ERR_VALUE;
    const size_t nq = static_cast<size_t>(BH) * Lq * d * 2, nk = static_cast<size_t>(BH) * Lk * d * 2;
    const size_t nl = static_cast<size_t>(BH) * Lq * 4;
    const void *ins[6] = {q, k, v, qd, kd, vd};
    const size_t insz[6] = {nq, nk, nk, nq, nk, nk};
    const void *outs[4] = {o, od, lse, lse_dot};
    const size_t outsz[4] = {nq, nq, nl, nl};
    for (int i = 0; i < 4; ++i) {
        if (!outs[i]) continue;
        for (int j = 0; j < 6; ++j)
            if (ins[j] && ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return ATTN_JVP_ERR_VALUE;
        for (int j = i + 1; j < 4; ++j)
            if (outs[j] && ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return ATTN_JVP_ERR_VALUE;
    }

    const int nqt = (Lq + BM - 1) / BM;
    // One CTA per query tile by default.  The CTA-pair layout (d = 128 only,
    // selected by a test flag) halves the per-SM operand traffic but couples
    // the two CTAs' pipelines; on B200 it measures slightly slower today.
    const bool pair = d == 128 && !zkv && (flags & ATTN_JVP_DEBUG_CTA_PAIR);
    const long long grid = pair ? 2ll * ((nqt + 1) / 2) * BH : static_cast<long long>(nqt) * BH;
    if (grid > INT_MAX) return ATTN_JVP_ERR_SHAPE;

    Params prm;
    std::memset(&prm, 0, sizeof prm);
    if (!make_map(&prm.tm_q, q, d, Lq, BH, BM) || !make_map(&prm.tm_qd, qd, d, Lq, BH, BM) ||
        !make_map(&prm.tm_k, k, d, Lk, BH, BN) || !make_map(&prm.tm_v, v, d, Lk, BH, BN) ||
        (!zkv && (!make_map(&prm.tm_kd, kd, d, Lk, BH, BN) || !make_map(&prm.tm_vd, vd, d, Lk, BH, BN))) ||
        (pair && !make_map(&prm.tm_k32, k, d, Lk, BH, BN / 2)))
        return ATTN_JVP_ERR_LAUNCH;
    prm.o = o;
    prm.od = od;
    prm.lse = lse;
    prm.lse_dot = lse_dot;
    prm.kv_len = kv_len;
    prm.H = H;
    prm.Lq = Lq;
    prm.Lk = Lk;
    prm.nqt = nqt;
    prm.scale = scale;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.timeout_ns = timeout_ns ? timeout_ns : DEFAULT_TIMEOUT_NS;
    prm.flags = flags;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc;
    if (zkv) rc = d == 64 ? launch_kernel<64, false, true>(prm, grid, s) : launch_kernel<128, false, true>(prm, grid, s);
    else if (d == 64) rc = launch_kernel<64, false, false>(prm, grid, s);
    else if (pair) rc = launch_kernel<128, true, false>(prm, grid, s);
    else rc = launch_kernel<128, false, false>(prm, grid, s);
    if (rc) return rc;
    if (cudaGetLastError() != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    return ATTN_JVP_OK;
}

}  // namespace ajvp

extern "C" {

int attn_jvp_fwd(const void *q, const void *k, const void *v, const void *q_dot, const void *k_dot,
                 const void *v_dot, void *o, void *o_dot, float *lse, int B, int H, int Lq, int Lk,
                 int d, float scale, const int32_t *kv_len, void *stream)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, nullptr, B, H, Lq, Lk, d, scale,
                        kv_len, stream, 0, 0, false);
}

int attn_jvp_fwd_ex(const void *q, const void *k, const void *v, const void *q_dot, const void *k_dot,
                    const void *v_dot, void *o, void *o_dot, float *lse, float *lse_dot, int B, int H,
                    int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *stream)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, lse_dot, B, H, Lq, Lk, d, scale,
                        kv_len, stream, 0, 0, true);
}

int attn_jvp_fwd_debug(const void *q, const void *k, const void *v, const void *q_dot,
                       const void *k_dot, const void *v_dot, void *o, void *o_dot, float *lse, int B,
                       int H, int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *stream,
                       uint64_t timeout_ns, int flags)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, nullptr, B, H, Lq, Lk, d, scale,
                        kv_len, stream, timeout_ns, flags, false);
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

int attn_jvp_version(void) { return 200; }

}  // extern "C"

// attn_jvp_fwd.cu -- attention forward + JVP for B200 (sm_100a), and its C ABI.
//
// The FlashAttention-2 JVP kernel of rCM ("Large Scale Diffusion Distillation
// via Score-Regularized Continuous-Time Consistency", ai.info AI summary, Key
// Contributions 1 and Methodology in Plain English) folds the tangent of
// attention into the block-wise forward pass.  This is a Blackwell-native
// design of that operation:
//
//   * a persistent CTA per SM walks 128-row query tiles of one (b, h) each;
//     Q and Q' sit in shared memory, K/K' and V/V' tiles of 64 keys stream
//     through two TMA rings that run on from one query tile to the next;
//   * S = Q K^T and S'_raw = Q K'^T + Q' K^T are tcgen05 MMAs into TMEM.  K and
//     K' sit next to each other in shared memory, so Q [K ; K']^T is a single
//     N = 128 MMA that writes S and Q K'^T side by side; Q' K^T then adds onto
//     the second half.  Together this is the K = 2d product [Q | Q'][K' | K]^T;
//   * two warpgroups run the online softmax in registers, thread = query row:
//     running max m (lazily rescaled), denominator l = sum p and
//     a = sum p (s S'_raw - c).  At d = 128 each takes one half of every
//     tile's 64 keys; at d = 64 each takes every other key tile, with its own
//     m, l, a and accumulators, merged at the end.  They write P and
//     P (s S'_raw - c) as bf16 back into TMEM at d = 128, into shared memory
//     at d = 64;
//   * [O | O'_acc] += P [V | V'] (one N = 2d MMA chain) and O'_acc +=
//     P(sS' - c) V are tcgen05 MMAs with A read from there;
//   * the epilogue forms O = O_acc / l and O' = (O'_acc - (a / l) O_acc) / l,
//     while the first S MMAs and loads of the next query tile already run.
//
// A trace instantiation (TRACE) stamps clock64 at each key tile's pipeline
// events into a caller buffer; it computes the same results.
//
// c is a per-row constant (the p-weighted mean of s S'_raw over the first 32
// keys, or 0 when all their p underflow).  In exact arithmetic O' does not
// depend on it; it keeps the bf16 products P (sS' - c) small when S' has a
// large row mean.
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

constexpr int BM = 128;                   // query rows per tile (= TMEM lanes)
constexpr int BN = 64;                    // keys per K/V tile
constexpr int NSOFT = 256;                // softmax threads: two warpgroups (warps 2-9)
constexpr int NTHREADS = 64 + NSOFT;      // + TMA warp 0 and MMA warp 1
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
    SITE_Q_EMPTY = 12,
    SITE_S_FREE = 13,
};

// Two ways to split the softmax between its two warpgroups:
//  - by columns (d = 128): both work on every key tile, warpgroup g on keys
//    [32g, 32g + 32) of each row, with one running max and one O, O'_acc;
//  - by tiles (ALT, d = 64): warpgroup g takes the key tiles gg with
//    gg % 2 == g, whole 64-key rows, and keeps its own running max, l, a and
//    accumulators O_g, O'_g; the epilogue merges the two.  The two
//    warpgroups then run out of phase (one's exp2 overlaps the other's
//    stores), and a row's per-tile latency is spread over two tiles.  The
//    four accumulators and two S buffers fill TMEM only when d = 64.  Each
//    warpgroup has one S buffer, so its P goes to shared memory: the buffer
//    can then take the warpgroup's next S as soon as S and S'_raw have been
//    read, while the softmax is still busy with the tile.
template <int D>
struct Cfg {
    static constexpr bool ALT = D == 64;
    static constexpr int NKB = D / 64;               // 128-byte column blocks per row
    // K ring depth.  At d = 128 two stages measured as fast as three on T2I
    // and 3 % faster on cross-attention (alternating timing); the 32 KB they
    // leave to the L1 cache is the likely reason.
    static constexpr int NK = (D == 128) ? 2 : 4;
    // V ring depth; at d = 64 the P slots take the room of a fourth stage
    static constexpr int NV = (D == 128) ? 2 : 3;
    static constexpr uint32_t Q_BYTES = BM * D * 2;  // one of Q, Q'
    // K stage: K then K' rows in each column block (one 128-row operand [K; K'])
    static constexpr uint32_t KST_BYTES = 2 * BN * D * 2;
    static constexpr uint32_t VHALF_BYTES = BN * D * 2;  // V stage: V then V'
    static constexpr uint32_t VST_BYTES = 2 * VHALF_BYTES;
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_QD = Q_BYTES;
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NK * KST_BYTES;
    // By tiles the bf16 P and P (sS' - c) operands of the PV MMAs live in
    // shared memory, one slot of each per warpgroup (128 rows x 64 keys,
    // K-major with the 128-byte swizzle): the S buffer is then free as soon
    // as the softmax has read S and S'_raw, and the warpgroup's next S runs
    // while it still works on this key tile.
    static constexpr uint32_t P_BYTES = BM * BN * 2;
    static constexpr uint32_t OFF_P = OFF_V + NV * VST_BYTES;
    __host__ __device__ static constexpr uint32_t off_p(int g, bool pd) { return OFF_P + (2 * g + (pd ? 1 : 0)) * P_BYTES; }
    static constexpr uint32_t OFF_BAR = OFF_P + (ALT ? 4 * P_BYTES : 0);
    // q_full, q_empty, k_full[NK], ks_done[NK], v_full[NV], vo_done[NV],
    // p_full[2], pd_full[2], drain, and by tiles s_free[2]
    static constexpr int NBAR = 2 + 2 * NK + 2 * NV + 2 + 2 + 1 + (ALT ? 2 : 0);
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // tmem slot, abort flag
    // Softmax exchange, floats.  By columns: per-warpgroup partial l, a
    // ([2][2][128]) and the centring constant hand-off ([128]).  By tiles:
    // per-warpgroup m, l, a, c ([2][4][128]).
    static constexpr int XCH_FLOATS = ALT ? 1024 : 640;
    static constexpr uint32_t OFF_XCH = OFF_MISC + 16;
    static constexpr uint32_t SMEM_BYTES = OFF_XCH + XCH_FLOATS * 4;
    // TMEM columns: O | O'_acc | S buffer 0 (S, S'_raw) | S buffer 1.  Both
    // softmax warpgroups read all of S (the row max) but only their own half
    // of S'_raw, columns [BN + 32g, BN + 32g + 32).  Warpgroup g writes its
    // bf16 P (keys 32g..32g+31, two per column) over the first 16 of those
    // columns and P (sS' - c) over the last 16, so no one overwrites a
    // column another warp may still read.
    //   By tiles the columns are O_0 | O'_0 | O_1 | O'_1 | S buffer 0 | S
    // buffer 1 (warpgroup g's), and P goes to shared memory.
    __host__ __device__ static constexpr uint32_t T_O(int g) { return ALT ? g * 2 * D : 0; }
    __host__ __device__ static constexpr uint32_t T_OD(int g) { return T_O(g) + D; }
    static constexpr uint32_t T_S = ALT ? 4 * D : 2 * D;
    // column of the bf16 P (pd = false) or P (sS' - c) (pd = true) operand of
    // keys 16kk..16kk+15 inside an S buffer
    __host__ __device__ static constexpr uint32_t t_pk(int kk, bool pd)
    {
        return BN + (kk >> 1) * 32 + (pd ? 16 : 0) + (kk & 1) * 8;
    }
    static constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, 2 * BN, false);
    static constexpr uint32_t IDESC_SD = idesc_bf16_f32(BM, BN, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
    // P [V | V'] into [O | O'_acc] as one N = 2d MMA: the V stage holds V's
    // and then V''s 64-column blocks at one stride, and O'_acc follows O in TMEM
    static constexpr uint32_t IDESC_PVV = idesc_bf16_f32(BM, 2 * D, true);
    static_assert(2 * D <= 256, "one MMA covers at most 256 columns");
    static constexpr int P_ARRIVALS = ALT ? 4 : 8;  // one per softmax warp that writes the tile
    // quarters of the softmax's exponentials computed on the FMA pipe
    // (ex2_poly2); the rest go to the MUFU unit.  Measured (alternating
    // timing, same inputs): at d = 128 one quarter is 1.9 % faster on T2I
    // than none, two are even, three are 2.5 % slower; at d = 64 every
    // fraction is slower (1.5 % at one quarter), so none is used there.
    static constexpr int POLY_QUARTERS = D == 64 ? 0 : 1;
    static_assert(T_S + 4 * BN <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Params {
    CUtensorMap tm_q, tm_qd, tm_k, tm_kd, tm_v, tm_vd;
    void *o;
    void *od;
    int out_v8;  // o and od are 32-byte aligned: the epilogue stores 32 bytes at a time
    float *lse;
    float *lse_dot;  // NULL: not computed
    const int32_t *kv_len;
    int H, Lq, Lk, nqt, n_tiles;
    float scale;  // s
    float sl2;    // s * log2(e)
    uint64_t timeout_ns;
    int flags;
    // trace build only: clock64 stamps [trace_ctas][trace_tiles][TRACE_EVENTS]
    unsigned long long *trace;
    int trace_tiles, trace_ctas;
    // Last-wave key split.  The first n_full query tiles are walked whole,
    // round robin over the CTAs (n_full is a multiple of the grid when
    // there is a split).  The remaining tiles are each cut into split_S key
    // ranges, and CTA u < n_units takes unit u after its whole tiles: tile
    // n_full + u / split_S, range u % split_S.  A range writes its partial
    // softmax state to part[u]; the last range of a tile to finish (counted
    // in cnt[u / split_S], zeroed before the launch) merges them.
    int n_full, split_S, n_units;
    float *part;
    int *cnt;
};

// Floats of one partial record per query row: m (log2 units), l, a, c, then
// the unnormalised O_acc and O'_acc rows.  A record holds 128 rows with the
// row index fastest, so a warp's loads and stores of one field coalesce.
template <int D>
__host__ __device__ constexpr int part_fields() { return 4 + 2 * D; }
constexpr int SPLIT_MAX = 8;  // ranges per split tile at most

// Events a trace build stamps for each of a CTA's key tiles (gg counts the
// key tiles of all the CTA's query tiles), in SM clock cycles.
enum : int {
    EV_K_LOAD = 0,   // TMA warp: K/K' loads issued
    EV_V_LOAD = 1,   // TMA warp: V/V' loads issued
    EV_S_ISSUE = 2,  // MMA warp: S and S' MMAs issued
    EV_PA_ISSUE = 3, // MMA warp: P V (and P V') MMAs issued
    EV_PB_ISSUE = 4, // MMA warp: P (sS' - c) V MMAs issued
    EV_SM_S = 5,     // softmax, first warp of warpgroup g: S seen   (+ 3g)
    EV_SM_P = 6,     // softmax: bf16 P stored and signalled          (+ 3g)
    EV_SM_PD = 7,    // softmax: bf16 P (sS' - c) stored and signalled (+ 3g)
    TRACE_EVENTS = 11,
};

__device__ __forceinline__ void st_global_v8(void *dst, const uint32_t (&v)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// Columns [c, c + 32) of the output rows of a warp, 32 bf16 (64 bytes) per
// lane in pv; `row` is the lane's own row (row index parity = lane parity),
// `ok_even` / `ok_odd` whether the even / odd row of its lane pair exists.
// Each thread owns a row, so a plain store of the warp touches 32 rows.  When
// the output is 32-byte aligned (v8), lanes 2i and 2i + 1 swap halves: then
// each 32-byte store lands next to its partner's, and one store of the warp
// covers 16 rows x 64 contiguous bytes in whole L2 sectors.  Called by all 32
// lanes (the shuffle); the stores themselves are predicated.
template <int D>
__device__ __forceinline__ void store_cols32(__nv_bfloat16 *row, int c, const uint32_t (&pv)[16], bool v8,
                                             bool odd, bool ok_even, bool ok_odd)
{
    if (v8) {
        uint32_t x[8], a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = __shfl_xor_sync(0xffffffffu, odd ? pv[i] : pv[8 + i], 1);
        // even lane: its first half to its row, the partner's first half to the odd row;
        // odd lane: the partner's second half to the even row, its second half to its row
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] = odd ? x[i] : pv[i];
            b[i] = odd ? pv[8 + i] : x[i];
        }
        __nv_bfloat16 *even_row = odd ? row - D : row;
        const int off = c + (odd ? 16 : 0);
        if (ok_even) st_global_v8(even_row + off, a);
        if (ok_odd) st_global_v8(even_row + D + off, b);
    } else if (odd ? ok_odd : ok_even) {
        uint4 *d4 = reinterpret_cast<uint4 *>(row + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pv[4 * i], pv[4 * i + 1], pv[4 * i + 2], pv[4 * i + 3]);
    }
}

// One work item: rows q0 .. q0 + 127 of head bh, against key tiles
// [jb, jb + nT) of the nb valid keys of its batch (the whole tile has
// ceil(nb / BN) key tiles; a split tile's range has fewer).  part < 0: the
// outputs are written directly; part >= 0: the partial state goes to record
// `part`, and the range is one of nseg of split tile `tsplit`.
struct Tile {
    int q0, bh, nb, jb, nT;
    int part, tsplit, nseg;
};

enum : int { ITEM_END = 0, ITEM_WORK = 1, ITEM_SKIP = 2 };

// The k-th work item of this CTA.  Every role walks the same sequence.
__device__ __forceinline__ int item_of(const Params &p, int k, Tile &t)
{
    const int b = blockIdx.x, G = gridDim.x;
    const int nk_full = b < p.n_full ? (p.n_full - 1 - b) / G + 1 : 0;
    int w, seg = 0, S = 1;
    if (k < nk_full) {
        w = b + k * G;
    } else if (k == nk_full && b < p.n_units) {
        w = p.n_full + b / p.split_S;
        seg = b % p.split_S;
        S = p.split_S;
    } else {
        return ITEM_END;
    }
    const int qt = w % p.nqt;  // query tile fastest: CTAs running together share K/V in L2
    t.bh = w / p.nqt;
    t.q0 = qt * BM;
    int nb = p.Lk;
    if (p.kv_len) nb = min(max(p.kv_len[t.bh / p.H], 0), p.Lk);
    t.nb = nb;
    const int nT = (nb + BN - 1) / BN;
    t.jb = 0;
    t.nT = nT;
    t.part = -1;
    t.tsplit = 0;
    t.nseg = 1;
    if (S > 1) {
        // a tile with fewer key tiles than ranges uses fewer ranges; one
        // without keys is written (as zeros) by its range 0 alone
        const int se = min(S, nT);
        if (seg >= max(se, 1)) return ITEM_SKIP;
        if (se > 1) {
            t.jb = seg * nT / se;
            t.nT = (seg + 1) * nT / se - t.jb;
            t.part = b;
            t.tsplit = b / S;
            t.nseg = se;
        }
    }
    return ITEM_WORK;
}

__device__ int g_status;  // first wait site that gave up since the last check
__device__ int g_status_taken;  // the word as the last check took it

// Read and clear the status word in one atomic step, ordered on the checking
// stream, so a site recorded by a kernel on another stream between a read
// and a clear cannot be lost.
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status, 0); }

// Host threads that check at the same time take turns on g_status_taken.
static std::mutex g_check_mu;

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

// One inline probe before falling back to the bounded loop.
__device__ __forceinline__ bool wait_bar_fast(uint64_t *bar, uint32_t parity, const WaitCtx &c, int site)
{
    if (mbar_test_wait(smem_addr(bar), parity)) return true;
    return wait_bar(bar, parity, c, site, true);
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// 2^a, 2^b (a, b below 2^7) on the FMA pipe, so that the softmax's exponentials
// are shared between the MUFU unit (ex2.approx) and the FMA units instead of
// queueing on the MUFU alone.  Cody-Waite range reduction: t = j + f with j
// the nearest integer (t + 1.5 * 2^23 rounds it into the low mantissa bits)
// and f in [-1/2, 1/2]; 2^f from a degree-3 polynomial whose coefficients
// were fitted here for relative error (at most 7.5e-5 in fp32 Horner form,
// well below the 2^-9 rounding of the bf16 P it feeds); j is then added to
// the exponent field.  Arguments below -125 are raised to -125 (a result
// near 2^-125, where ex2.approx.ftz would give 0; both are negligible
// against the row sum, which holds a term of at least 1/16).
__device__ __forceinline__ void ex2_poly2(float a, float b, float &ya, float &yb)
{
    constexpr float MAGIC = 12582912.0f;  // 1.5 * 2^23
    const uint64_t t = f2_pack(fmaxf(a, -125.0f), fmaxf(b, -125.0f));
    const uint64_t r = f2_add(t, f2_pack(MAGIC, MAGIC));
    const uint64_t j = f2_add(r, f2_pack(-MAGIC, -MAGIC));
    const uint64_t f = f2_fma(j, f2_pack(-1.0f, -1.0f), t);  // t - j, exact
    uint64_t q = f2_fma(f, f2_pack(0.05517115443944931f, 0.05517115443944931f),
                        f2_pack(0.2426101416349411f, 0.2426101416349411f));
    q = f2_fma(q, f, f2_pack(0.6932609677314758f, 0.6932609677314758f));
    q = f2_fma(q, f, f2_pack(0.9999281167984009f, 0.9999281167984009f));
    float qa, qb, ra, rb;
    f2_unpack(q, qa, qb);
    f2_unpack(r, ra, rb);
    // the low bits of r hold 0x4B400000 + j: shifted by 23 they add j to q's exponent
    ya = __uint_as_float(f2u(ra) * 8388608u + f2u(qa));
    yb = __uint_as_float(f2u(rb) * 8388608u + f2u(qb));
}

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

// ---- last-wave key split: partial records and their merge

template <int D>
__device__ __forceinline__ float *part_field(const Params &p, int u, int f)
{
    return p.part + (static_cast<size_t>(u) * part_fields<D>() + f) * BM;
}

template <int D>
__device__ __forceinline__ void part_put_scalars(const Params &p, int u, int r, float m, float l, float a, float c)
{
    part_field<D>(p, u, 0)[r] = m;
    part_field<D>(p, u, 1)[r] = l;
    part_field<D>(p, u, 2)[r] = a;
    part_field<D>(p, u, 3)[r] = c;
}

// Columns [c, c + 32) of O_acc (which = 0) or O'_acc (which = 1).
template <int D>
__device__ __forceinline__ void part_put_cols(const Params &p, int u, int r, int which, int c, const float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i) part_field<D>(p, u, 4 + which * D + c + i)[r] = v[i];
}

// Called by all 256 softmax threads after they wrote this range's partial
// record.  The range that finishes last (a counter per split tile, zeroed
// before the launch) merges the records of all ranges of the tile, with
// M = max m_s, b_s = 2^(m_s - M), L = sum b_s l_s:
//   mu = sum b_s (a_s + c_s l_s) / L,  O = sum b_s O_s / L,
//   O' = sum b_s (O'_s + (c_s - mu) O_s) / L,  lse = (M + log2 L) ln 2,
// and writes the outputs (warpgroup 0: O and lse, warpgroup 1: O' and lse').
// No CTA waits for another: the ranges that finish earlier just leave.
template <int D>
__device__ __noinline__ void split_finish(const Params &p, const Tile &t, int g, int r, __nv_bfloat16 *out_ptr,
                             int grow, size_t lrow, uint8_t *flag_smem)
{
    volatile int *flag = reinterpret_cast<volatile int *>(flag_smem);
    __threadfence();  // this thread's record stores, before the count
    bar_sync(BAR_SOFT, NSOFT);
    if (threadIdx.x == 64) *flag = atomicAdd(&p.cnt[t.tsplit], 1) == t.nseg - 1;
    bar_sync(BAR_SOFT, NSOFT);
    const bool last = *flag != 0;
    bar_sync(BAR_SOFT, NSOFT);  // everyone has read the flag before it can be reused
    if (!last) return;
    __threadfence();
    const int u0 = t.tsplit * p.split_S;
    float M = -INFINITY;
    for (int s = 0; s < t.nseg; ++s) M = fmaxf(M, __ldcg(part_field<D>(p, u0 + s, 0) + r));
    float L = 0.f, num = 0.f;
    for (int s = 0; s < t.nseg; ++s) {
        const float b = ex2_approx(__ldcg(part_field<D>(p, u0 + s, 0) + r) - M);
        const float ls = __ldcg(part_field<D>(p, u0 + s, 1) + r);
        L = fmaf(b, ls, L);
        num = fmaf(b, fmaf(__ldcg(part_field<D>(p, u0 + s, 3) + r), ls, __ldcg(part_field<D>(p, u0 + s, 2) + r)), num);
    }
    const float inv_l = 1.f / L;
    const float mu = num * inv_l;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        for (int s = 0; s < t.nseg; ++s) {
            const float w = ex2_approx(__ldcg(part_field<D>(p, u0 + s, 0) + r) - M) * inv_l;
            const float *o = part_field<D>(p, u0 + s, 4 + c) + r;
            if (g == 0) {
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __ldcg(o + i * BM), acc[i]);
            } else {
                const float kk = w * (__ldcg(part_field<D>(p, u0 + s, 3) + r) - mu);
                const float *od = part_field<D>(p, u0 + s, 4 + D + c) + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __ldcg(od + i * BM), fmaf(kk, __ldcg(o + i * BM), acc[i]));
            }
        }
        // 16-byte stores of the thread's own row (the merge runs for a few
        // tiles only, so the paired 32-byte stores of the main epilogue buy
        // nothing here)
        if (grow < p.Lq) {
            uint4 *d4 = reinterpret_cast<uint4 *>(out_ptr + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d4[i] = make_uint4(pack_bf16x2(acc[8 * i], acc[8 * i + 1]), pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]),
                                   pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]), pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]));
        }
    }
    if (g == 0 && grow < p.Lq) p.lse[lrow] = (M + log2f(L)) * 0.69314718055994531f;
    if (g == 1 && p.lse_dot && grow < p.Lq) p.lse_dot[lrow] = mu;
}

// ZKV: K' = V' = 0 (frozen keys and values, e.g. text tokens).  Then S'_raw
// = Q' K^T and O' = P' V: the K' and V' tiles are neither loaded nor
// multiplied, 8 of the 12 FLOP units remain.
//
// Every role walks the same sequence of query tiles (w = blockIdx.x,
// blockIdx.x + gridDim.x, ...) and skips the tiles without keys the same
// way, so the key tiles of all its query tiles form one sequence gg = 0, 1,
// ...: the K and V ring slots, the S/P TMEM buffer and the phases of the
// per-key-tile barriers all follow gg.
template <int D, bool ZKV, bool TRACE>
__global__ void __launch_bounds__(NTHREADS, 1) attn_jvp_fwd_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<D>;
    // trace build: stamp event `ev` of key tile gk (no code in the normal build)
    auto stamp = [&](const int gk, const int ev) {
        if constexpr (TRACE) {
            if (gk < p.trace_tiles && static_cast<int>(blockIdx.x) < p.trace_ctas)
                p.trace[(static_cast<size_t>(blockIdx.x) * p.trace_tiles + gk) * TRACE_EVENTS + ev] = clock64();
        }
    };
    extern __shared__ __align__(1024) uint8_t smem[];
    // The 128-byte swizzle atoms must start on 1024-byte boundaries.  The
    // dynamic window is 1024-aligned in practice; if it ever is not, record it
    // and do nothing rather than compute garbage.
    if (smem_addr(smem) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(&g_status, 0, SITE_SMEM_ALIGN);
        return;
    }

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *q_empty = q_full + 1;  // the last S MMA of a query tile has read Q, Q'
    uint64_t *k_full = q_empty + 1;
    // ks_done[s]: the S MMAs of the key tile in K slot s are done, so the slot
    // may be refilled (and the softmax may read S).  vo_done[s]:
    // the PV MMAs of the key tile in V slot s are done, so the slot may be
    // refilled (and O may be rescaled or read).  One commit per MMA group
    // thus signals both consumers (each commit costs the tensor pipe about 30
    // clocks).  Neither can fall two phases behind on a slot: the next phase
    // needs the slot's next load, issued by the TMA warp only after its wait,
    // and MMAs that the MMA warp issues, in a fixed order, only after P
    // signals of key tiles that the waiting softmax warp has not yet reached.
    uint64_t *ks_done = k_full + C::NK;
    uint64_t *v_full = ks_done + C::NK;
    uint64_t *vo_done = v_full + C::NV;
    uint64_t *p_full = vo_done + C::NV;  // [2] bf16 P written
    uint64_t *pd_full = p_full + 2;      // [2] bf16 P (sS' - c) written
    uint64_t *drain = pd_full + 2;
    uint64_t *s_free = drain + 1;        // by tiles: [2] warpgroup g has read its S buffer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&ks_done[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&vo_done[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&p_full[s], C::P_ARRIVALS);
            mbar_init(&pd_full[s], C::P_ARRIVALS);
            if (C::ALT) mbar_init(&s_free[s], C::P_ARRIVALS);
        }
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
        // Per query tile: Q and Q' (once the previous tile's S MMAs are done
        // with them), then K_0, K_1, V_0, K_2, V_1, ...; the rings carry on
        // across query tiles, so the next tile's first K and V tiles load
        // while the current one finishes.
        if (lane == 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            const bool load_q = !(p.flags & ATTN_JVP_DEBUG_STARVE_Q);
            int lc = 0;           // query tiles with keys so far
            int nq = 0;           // Q loads issued
            int kc = 0, vc = 0;   // K and V loads issued
            bool ok = true;
            Tile t;
            for (int k = 0; ok; ++k) {
                const int it = item_of(p, k, t);
                if (it == ITEM_END) break;
                if (it == ITEM_SKIP || t.nT == 0) continue;
                if (lc >= 1 && !wait_bar(q_empty, (lc - 1) & 1, wc, SITE_Q_EMPTY)) {
                    ok = false;
                    break;
                }
                ++lc;
                if (load_q) {
                    mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NKB; ++c) {
                        tma_load_3d(smem + C::OFF_Q + c * BM * 128, &p.tm_q, q_full, c * 64, t.q0, t.bh, pol_q);
                        tma_load_3d(smem + C::OFF_QD + c * BM * 128, &p.tm_qd, q_full, c * 64, t.q0, t.bh,
                                    pol_q);
                    }
                    ++nq;
                }
                for (int j = 0; j <= t.nT; ++j) {
                    if (j < t.nT) {
                        const int s = kc % C::NK;
                        if (kc >= C::NK) ok = wait_bar(&ks_done[s], ((kc / C::NK) - 1) & 1, wc, SITE_K_EMPTY);
                        if (!ok) break;
                        uint8_t *dst = smem + C::OFF_K + s * C::KST_BYTES;
                        mbar_arrive_expect_tx(&k_full[s], ZKV ? C::KST_BYTES / 2 : C::KST_BYTES);
#pragma unroll
                        for (int c = 0; c < C::NKB; ++c) {
                            tma_load_3d(dst + c * (2 * BN * 128), &p.tm_k, &k_full[s], c * 64, (t.jb + j) * BN,
                                        t.bh, pol_kv);
                            if (!ZKV)
                                tma_load_3d(dst + c * (2 * BN * 128) + BN * 128, &p.tm_kd, &k_full[s], c * 64,
                                            (t.jb + j) * BN, t.bh, pol_kv);
                        }
                        stamp(kc, EV_K_LOAD);
                        ++kc;
                    }
                    if (j >= 1) {
                        const int s = vc % C::NV;
                        if (vc >= C::NV) ok = wait_bar(&vo_done[s], ((vc / C::NV) - 1) & 1, wc, SITE_V_EMPTY);
                        if (!ok) break;
                        uint8_t *dst = smem + C::OFF_V + s * C::VST_BYTES;
                        mbar_arrive_expect_tx(&v_full[s], ZKV ? C::VHALF_BYTES : C::VST_BYTES);
#pragma unroll
                        for (int c = 0; c < C::NKB; ++c) {
                            tma_load_3d(dst + c * (BN * 128), &p.tm_v, &v_full[s], c * 64, (t.jb + j - 1) * BN,
                                        t.bh, pol_kv);
                            if (!ZKV)
                                tma_load_3d(dst + (C::NKB + c) * (BN * 128), &p.tm_vd, &v_full[s], c * 64,
                                            (t.jb + j - 1) * BN, t.bh, pol_kv);
                        }
                        stamp(vc, EV_V_LOAD);
                        ++vc;
                    }
                }
            }
            // Let every load land before the CTA can exit: wait for the last
            // phase of each barrier a load was issued on (no later load can
            // make that wait ambiguous).
            if (nq > 0) wait_bar(q_full, (nq - 1) & 1, wc, SITE_DRAIN, false);
            for (int s = 0; s < C::NK && s < kc; ++s) {
                const int t = s + ((kc - 1 - s) / C::NK) * C::NK;
                wait_bar(&k_full[s], (t / C::NK) & 1, wc, SITE_DRAIN, false);
            }
            for (int s = 0; s < C::NV && s < vc; ++s) {
                const int t = s + ((vc - 1 - s) / C::NV) * C::NV;
                wait_bar(&v_full[s], (t / C::NV) & 1, wc, SITE_DRAIN, false);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (barrier tests and branches are
        // warp-uniform); one elected lane issues each MMA and commit.
        // Operand descriptors are built once per buffer; the per-MMA offsets
        // are added to the start-address field (all shared addresses fit its
        // 18 bits), which keeps the issue loop short.
        const uint64_t dq = sdesc_sw128(smem_addr(smem + C::OFF_Q), 16, 1024);
        const uint64_t dqd = sdesc_sw128(smem_addr(smem + C::OFF_QD), 16, 1024);
        bool issued = false;
        // Each wait first parks the warp in mbarrier.try_wait, which wakes it
        // when the phase completes.
        auto wait_u = [&](uint64_t *bar, uint32_t parity, int site) {
            bool r = mbar_try_wait(smem_addr(bar), parity);
            if (!__all_sync(0xffffffffu, r)) r = wait_bar(bar, parity, wc, site, true);
            return __all_sync(0xffffffffu, r);
        };
        // S_g | S'_g for key tile g into TMEM buffer g & 1.
        auto issue_s = [&](const int gk) {
            const int s = gk % C::NK;
            tc_fence_after();
            const uint32_t tS = tbase + C::T_S + (gk & 1) * (2 * BN);
            const uint64_t dk = sdesc_sw128(smem_addr(smem + C::OFF_K + s * C::KST_BYTES), 16, 1024);
            // S | Q K'^T  =  Q [K ; K']^T   (N = 2 BN); with K' = 0 only
            // S = Q K^T (N = BN)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                mma_ss(tS, desc_add(dq, oa), desc_add(dk, ob), ZKV ? C::IDESC_SD : C::IDESC_S, kk > 0 ? 1u : 0u);
            }
            // += Q' K^T into the second half (with K' = 0 it starts it)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t oa = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                const uint32_t ob = (kk >> 2) * (2 * BN * 128) + (kk & 3) * 32;
                mma_ss(tS + BN, desc_add(dqd, oa), desc_add(dk, ob), C::IDESC_SD, (!ZKV || kk > 0) ? 1u : 0u);
            }
            mma_commit(&ks_done[s]);
            issued = true;
        };
        // LBO: distance between 64-column blocks of V
        constexpr uint32_t LBO = BN * 128;
        // PV of key tile g in two groups: A needs only P (O += P V,
        // O'_acc += P V'), B needs P (sS' - c) as well (O'_acc += P (sS' - c)
        // V), which the softmax writes later; A can then start while B's
        // operand is formed.  `first`: the first key tile of the query tile
        // for these accumulators, which starts them.  By tiles, key tile gg
        // goes into warpgroup (gg % 2)'s O_g and O'_g.
        // By tiles the A operand (P or P (sS' - c), 64 keys = one 128-byte
        // swizzle row per query row) comes from warpgroup ow's shared slot;
        // by columns from TMEM, over S'_raw.
        auto issue_pa = [&](const int gk, const bool first) {
            const int s = gk % C::NV;
            tc_fence_after();
            const uint32_t tP = tbase + C::T_S + (gk & 1) * (2 * BN);
            const int ow = C::ALT ? (gk & 1) : 0;
            const uint64_t dv = sdesc_sw128(smem_addr(smem + C::OFF_V + s * C::VST_BYTES), LBO, 1024);
            static_assert(C::VHALF_BYTES == C::NKB * LBO, "V' blocks follow V's at the block stride");
            const uint64_t dp = sdesc_sw128(smem_addr(smem + C::off_p(ow, false)), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {  // [O | O'_acc] += P [V | V']  (with V' = 0: O += P V)
                if constexpr (C::ALT)
                    mma_ss(tbase + C::T_O(ow), desc_add(dp, kk * 32), desc_add(dv, kk * 2048),
                           ZKV ? C::IDESC_PV : C::IDESC_PVV, (!first || kk > 0) ? 1u : 0u);
                else
                    mma_ts(tbase + C::T_O(ow), tP + C::t_pk(kk, false), desc_add(dv, kk * 2048),
                           ZKV ? C::IDESC_PV : C::IDESC_PVV, (!first || kk > 0) ? 1u : 0u);
            }
        };
        auto issue_pb = [&](const int gk, const bool first) {
            const int s = gk % C::NV;
            tc_fence_after();
            const uint32_t tP = tbase + C::T_S + (gk & 1) * (2 * BN);
            const int ow = C::ALT ? (gk & 1) : 0;
            const uint64_t dv = sdesc_sw128(smem_addr(smem + C::OFF_V + s * C::VST_BYTES), LBO, 1024);
            const uint64_t dp = sdesc_sw128(smem_addr(smem + C::off_p(ow, true)), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {  // O'_acc += P(sS' - c) V (with V' = 0 it starts O'_acc)
                if constexpr (C::ALT)
                    mma_ss(tbase + C::T_OD(ow), desc_add(dp, kk * 32), desc_add(dv, kk * 2048), C::IDESC_PV,
                           (!ZKV || !first || kk > 0) ? 1u : 0u);
                else
                    mma_ts(tbase + C::T_OD(ow), tP + C::t_pk(kk, true), desc_add(dv, kk * 2048), C::IDESC_PV,
                           (!ZKV || !first || kk > 0) ? 1u : 0u);
            }
            mma_commit(&vo_done[s]);
        };
        // Fixed order per query tile: S_0, S_1, PV_0, S_2, PV_1, ...: S_{j+1}
        // runs on the tensor core while the softmax works on key tile j, and
        // S_{j+1} overwrites the TMEM buffer that held P_{j-1} only after
        // PV_{j-1} was issued (MMAs run in issue order).  The next query
        // tile's S_0 and S_1 follow its last PV at once and overlap the
        // epilogue; its first PV (which restarts O and O'_acc) waits for P,
        // which the softmax warps write only after their epilogue has read O.
        bool ok = true;
        int lc = 0, gg = 0;
        Tile t;
        // By tiles: per query tile S_0 and S_1 first; then for key tile j,
        // P V_j, S_{j+2} as soon as warpgroup (j % 2) has read S_j and S'_j
        // from its buffer, and P (sS' - c) V_j.  S_{j+2} thus runs on the
        // tensor core while that warpgroup's softmax still works on key tile j.
        for (int k = 0; C::ALT && ok; ++k) {
            const int it = item_of(p, k, t);
            if (it == ITEM_END) break;
            if (it == ITEM_SKIP || t.nT == 0) continue;
            ok = wait_u(q_full, lc & 1, SITE_Q_FULL);
            ++lc;
            for (int j = 0; ok && j < 2 && j < t.nT; ++j) {
                ok = wait_u(&k_full[(gg + j) % C::NK], ((gg + j) / C::NK) & 1, SITE_K_FULL);
                if (!ok) break;
                issue_s(gg + j);
                if (lane == 0) stamp(gg + j, EV_S_ISSUE);
            }
            if (!ok) break;
            if (t.nT <= 2) mma_commit(q_empty);  // that was the tile's last S
            for (int j = 0; j < t.nT; ++j) {
                const int gk = gg + j;
                if (j + 2 < t.nT) {
                    ok = wait_u(&s_free[gk & 1], (gk >> 1) & 1, SITE_S_FREE);
                    if (ok) ok = wait_u(&k_full[(gk + 2) % C::NK], ((gk + 2) / C::NK) & 1, SITE_K_FULL);
                    if (!ok) break;
                    issue_s(gk + 2);
                    if (lane == 0) stamp(gk + 2, EV_S_ISSUE);
                    if (j + 3 == t.nT) mma_commit(q_empty);
                }
                ok = wait_u(&v_full[gk % C::NV], (gk / C::NV) & 1, SITE_V_FULL);
                if (ok) ok = wait_u(&p_full[gk & 1], (gk >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                issue_pa(gk, j < 2);
                if (lane == 0) stamp(gk, EV_PA_ISSUE);
                ok = wait_u(&pd_full[gk & 1], (gk >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                issue_pb(gk, j < 2);
                if (lane == 0) stamp(gk, EV_PB_ISSUE);
            }
            gg += t.nT;
        }
        for (int k = 0; !C::ALT && ok; ++k) {
            const int it = item_of(p, k, t);
            if (it == ITEM_END) break;
            if (it == ITEM_SKIP || t.nT == 0) continue;
            ok = wait_u(q_full, lc & 1, SITE_Q_FULL);
            ++lc;
            if (ok) ok = wait_u(&k_full[gg % C::NK], (gg / C::NK) & 1, SITE_K_FULL);
            if (!ok) break;
            issue_s(gg);
            if (lane == 0) stamp(gg, EV_S_ISSUE);
            if (t.nT == 1) mma_commit(q_empty);
            for (int j = 0; j < t.nT; ++j) {
                const int gk = gg + j;
                if (j + 1 < t.nT) {
                    ok = wait_u(&k_full[(gk + 1) % C::NK], ((gk + 1) / C::NK) & 1, SITE_K_FULL);
                    if (!ok) break;
                    issue_s(gk + 1);
                    if (lane == 0) stamp(gk + 1, EV_S_ISSUE);
                    if (j + 2 == t.nT) mma_commit(q_empty);  // that was the tile's last S
                }
                // V_j normally lands before P_j is written: wait for it first
                ok = wait_u(&v_full[gk % C::NV], (gk / C::NV) & 1, SITE_V_FULL);
                if (ok) ok = wait_u(&p_full[gk & 1], (gk >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                const bool first = j == 0;
                issue_pa(gk, first);
                if (lane == 0) stamp(gk, EV_PA_ISSUE);
                ok = wait_u(&pd_full[gk & 1], (gk >> 1) & 1, SITE_P_FULL);
                if (!ok) break;
                issue_pb(gk, first);
                if (lane == 0) stamp(gk, EV_PB_ISSUE);
            }
            gg += t.nT;
        }
        if (!ok && issued) {
            mma_commit(drain);
            wait_bar(drain, 0, wc, SITE_DRAIN, false);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // Two warpgroups, thread = query row.  By columns, warpgroup g owns
        // key columns [32g, 32g + 32) of every key tile; by tiles, the key
        // tiles gg with gg % 2 == g.  At the end of a query tile warpgroup g
        // writes output g (0: O and lse, 1: O' and lse').
        const int g = (warp - 2) >> 2;
        const int quad = warp & 3;  // TMEM lane quadrant this warp may touch
        const int r = quad * 32 + lane;
        const int gt = tid - 64 - g * 128;  // thread index inside the warpgroup
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const bool tracer = TRACE && gt == 0;  // lane 0 of the warpgroup's first warp
        float *xch = reinterpret_cast<float *>(smem + C::OFF_XCH);
        const float sl2 = p.sl2;
        const float sc = p.scale;
        const bool neg = sl2 < 0.f;
        if constexpr (C::ALT) {
            int gg = 0;
            const uint32_t tS = tbase + lane_off + C::T_S + g * (2 * BN);  // this warpgroup's S buffer
            Tile t;
            for (int k = 0;; ++k) {
                const int itk = item_of(p, k, t);
                if (itk == ITEM_END) break;
                if (itk == ITEM_SKIP) continue;
                const int grow = t.q0 + r;
                // output row pointers, formed where they are used so they need
                // no registers across the key loop
                auto out_row = [&]() {
                    return static_cast<__nv_bfloat16 *>(g == 0 ? p.o : p.od) +
                           (static_cast<size_t>(t.bh) * p.Lq + grow) * D;
                };
                auto lse_row = [&]() { return static_cast<size_t>(t.bh) * p.Lq + grow; };
                if (t.nT == 0) {
                    __nv_bfloat16 *out_ptr = out_row();
                    const size_t lrow = lse_row();
                    if (grow < p.Lq) {
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4 *>(out_ptr)[c] = z;
                        if (g == 0) p.lse[lrow] = -INFINITY;
                        if (g == 1 && p.lse_dot) p.lse_dot[lrow] = 0.f;
                    }
                    continue;
                }
                const int nb = t.nb, nT = t.nT;
                // this warpgroup's running max (log2 units), l, a and centring
                // constant over its own key tiles
                float m_used = -INFINITY, l = 0.f, acc_a = 0.f, cctr = 0.f;
                bool err = false;
                int nown = 0, last = 0;
                for (int j = ((gg & 1) == g) ? 0 : 1; j < nT; j += 2) {
                    const int gk = gg + j;
                    if (!__all_sync(0xffffffffu, wait_bar_fast(&ks_done[gk % C::NK], (gk / C::NK) & 1, wc, SITE_S_FULL))) {
                        err = true;
                        break;
                    }
                    if (tracer) stamp(gk, EV_SM_S + 3 * g);
                    tc_fence_after();
                    const int vt = nb - (t.jb + j) * BN;  // valid keys in the tile
                    const bool tail = vt < BN;
                    uint32_t ra[32], rb[32], rd[32];
                    tmem_ld32(tS, ra);       // S, keys 0..31
                    tmem_ld32(tS + 32, rb);  // S, keys 32..63
                    tmem_ld32(tS + BN, rd);  // S'_raw, keys 0..31
                    tmem_ld_wait2(ra, rb);
                    tmem_ld_ready(rd);
                    if (tail) {
                        // padded keys: S to the pad (p = 0 below), S'_raw to 0 so
                        // that P (sS' - c) = 0 (-c) = 0 whatever their bits were
                        const float pad = neg ? INFINITY : -INFINITY;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            ra[i] = (i < vt) ? ra[i] : f2u(pad);
                            rb[i] = (i + 32 < vt) ? rb[i] : f2u(pad);
                            rd[i] = (i < vt) ? rd[i] : 0u;
                        }
                    }
                    const float mx = neg ? row_min64(ra, rb) : row_max64(ra, rb);
                    const float m_tile = mx * sl2;
                    float alpha = 1.f;
                    bool rescale = false;
                    if (nown == 0) {
                        m_used = m_tile;
                    } else if (m_tile > m_used + RESCALE_THRESHOLD) {
                        alpha = ex2_approx(m_used - m_tile);
                        m_used = m_tile;
                        rescale = true;
                    }
                    l *= alpha;
                    acc_a *= alpha;
                    uint32_t pk[32];  // bf16 P, keys 2i and 2i + 1 (low half: key 2i)
                    {
                        float x[64];
                        const uint64_t sl22 = f2_pack(sl2, sl2);
                        const uint64_t nm2 = f2_pack(-m_used, -m_used);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float t0, t1, t2, t3;
                            f2_unpack(f2_fma(f2_pack(u2f(ra[2 * i]), u2f(ra[2 * i + 1])), sl22, nm2), t0, t1);
                            f2_unpack(f2_fma(f2_pack(u2f(rb[2 * i]), u2f(rb[2 * i + 1])), sl22, nm2), t2, t3);
                            x[2 * i] = ex2_approx(t0);
                            x[2 * i + 1] = ex2_approx(t1);
                            x[32 + 2 * i] = ex2_approx(t2);
                            x[33 + 2 * i] = ex2_approx(t3);
                        }
                        if (tail) {
                            // padded keys: p = 0 exactly (the pad times a zero scale is NaN)
#pragma unroll
                            for (int i = 0; i < 64; ++i) x[i] = (i < vt) ? x[i] : 0.f;
                        }
                        uint64_t s0 = f2_pack(x[0], x[1]), s1 = f2_pack(x[2], x[3]);
                        uint64_t s2 = f2_pack(x[32], x[33]), s3 = f2_pack(x[34], x[35]);
#pragma unroll
                        for (int i = 2; i < 16; i += 2) {
                            s0 = f2_add(s0, f2_pack(x[2 * i], x[2 * i + 1]));
                            s1 = f2_add(s1, f2_pack(x[2 * i + 2], x[2 * i + 3]));
                            s2 = f2_add(s2, f2_pack(x[32 + 2 * i], x[33 + 2 * i]));
                            s3 = f2_add(s3, f2_pack(x[34 + 2 * i], x[35 + 2 * i]));
                        }
                        float u0, u1, u2, u3;
                        f2_unpack(f2_add(s0, s2), u0, u1);
                        f2_unpack(f2_add(s1, s3), u2, u3);
                        l += (u0 + u1) + (u2 + u3);
                        if (nown == 0) {
                            // centring constant c: the p-weighted mean of s S' over
                            // keys 0..31 of this warpgroup's first key tile.  Their
                            // p can all be 0 (the tile's max among keys 32..63 and
                            // keys 0..31 more than ~87 logits below it); c cancels
                            // exactly, so any finite value is right, and 0 is taken.
                            float n0 = 0.f, n1 = 0.f, w0 = 0.f, w1 = 0.f;
#pragma unroll
                            for (int i = 0; i < 32; i += 2) {
                                n0 += (tail && i >= vt) ? 0.f : x[i] * (u2f(rd[i]) * sc);
                                n1 += (tail && i + 1 >= vt) ? 0.f : x[i + 1] * (u2f(rd[i + 1]) * sc);
                                w0 += x[i];
                                w1 += x[i + 1];
                            }
                            const float wsum = w0 + w1;
                            cctr = wsum > 0.f ? (n0 + n1) / wsum : 0.f;
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                    }
                    // The rest of S'_raw; then the buffer has been read, and the
                    // MMA warp may put this warpgroup's next S there.
                    uint32_t re[32];
                    tmem_ld32(tS + BN + 32, re);  // S'_raw, keys 32..63
                    tmem_ld_wait(re);
                    if (tail) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) re[i] = (i + 32 < vt) ? re[i] : 0u;
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free[g]);
                    // This warpgroup's previous key tile (gk - 2, possibly of an
                    // earlier query tile): its PV MMAs read the P slots and
                    // write O_g, and must be done before either is touched.
                    // S_gk was issued without waiting for them.
                    if (gk >= 2 && !__all_sync(0xffffffffu, wait_bar_fast(&vo_done[(gk - 2) % C::NV],
                                                                          ((gk - 2) / C::NV) & 1, wc, SITE_O_DONE))) {
                        err = true;
                        break;
                    }
                    if (__any_sync(0xffffffffu, rescale)) {
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 2 * D; c += 16) {  // O_g then O'_g
                            uint32_t tt[16];
                            tmem_ld16_wait(tbase + lane_off + C::T_O(g) + c, tt);
#pragma unroll
                            for (int i = 0; i < 16; ++i) tt[i] = f2u(u2f(tt[i]) * alpha);
                            tmem_st16(tbase + lane_off + C::T_O(g) + c, tt);
                        }
                        tmem_st_wait();
                    }
                    if (tail) {
                        // Zero the V (and V') rows of padded keys so their bits
                        // (NaN included) cannot reach the PV products.
                        const int s = gk % C::NV;
                        if (!__all_sync(0xffffffffu, wait_bar(&v_full[s], (gk / C::NV) & 1, wc, SITE_V_TAIL))) {
                            err = true;
                            break;
                        }
                        uint8_t *vst = smem + C::OFF_V + s * C::VST_BYTES;
                        const int per_blk = (BN - vt) * 8;  // 16-byte chunks per 64-column block
                        const int chunks = (ZKV ? 1 : 2) * C::NKB * per_blk;
                        for (int idx = gt; idx < chunks; idx += 128) {
                            const int blk = idx / per_blk;  // V blocks, then V' blocks
                            const int rem = idx - blk * per_blk;
                            *reinterpret_cast<uint4 *>(vst + blk * (BN * 128) + (vt + (rem >> 3)) * 128 +
                                                       (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
                        }
                    }
                    // Row r of a P slot: 64 keys in 8 chunks of 16 bytes, chunk
                    // c at position c ^ (r % 8) of the row (the 128-byte swizzle
                    // the MMA descriptor names); 8 consecutive rows fill all
                    // 32 banks, so a warp's store takes the minimum 4 wavefronts.
                    const uint32_t prow = smem_addr(smem + C::off_p(g, false)) + (r >> 3) * 1024 + (r & 7) * 128;
                    const uint32_t pdrow = prow + C::P_BYTES;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_shared_v4(prow + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                    // the tensor core reads P (and zeroed V rows) through the async proxy
                    fence_proxy_async_smem();
                    tc_fence_before();  // orders the rescale's TMEM stores before the PV MMAs
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full[g]);
                    if (tracer) stamp(gk, EV_SM_P + 3 * g);
                    // ---- bf16 P (s S' - c) while the tensor core multiplies P.  p
                    // is taken as rounded to bf16, the same p the P V MMAs use
                    // (the fp32 p would need 32 more registers here).
                    const uint64_t sc2 = f2_pack(sc, sc);
                    const uint64_t nc2 = f2_pack(-cctr, -cctr);
                    uint64_t a0 = 0, a1 = 0;
                    // keys [32h, 32h + 32) from v (S'_raw): chunks 4h..4h+3 of the row
                    auto pd_half = [&](const uint32_t (&v)[32], const int h) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            uint32_t w[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int i = 4 * cc + q;
                                const uint32_t pp = pk[16 * h + i];
                                const uint64_t p2 = f2_pack(u2f(pp << 16), u2f(pp & 0xFFFF0000u));
                                const uint64_t d2 =
                                    f2_mul(f2_fma(f2_pack(u2f(v[2 * i]), u2f(v[2 * i + 1])), sc2, nc2), p2);
                                float d0, d1;
                                f2_unpack(d2, d0, d1);
                                w[q] = pack_bf16x2(d0, d1);
                                // the two rounded values as fp32
                                const uint64_t r2 = f2_pack(u2f(w[q] << 16), u2f(w[q] & 0xFFFF0000u));
                                if (i & 1) a1 = f2_add(a1, r2);
                                else a0 = f2_add(a0, r2);
                            }
                            st_shared_v4(pdrow + (((4 * h + cc) ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
                        }
                    };
                    pd_half(rd, 0);
                    pd_half(re, 1);
                    {
                        float u0, u1, u2, u3;
                        f2_unpack(a0, u0, u1);
                        f2_unpack(a1, u2, u3);
                        acc_a += (u0 + u1) + (u2 + u3);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pd_full[g]);
                    if (tracer) stamp(gk, EV_SM_PD + 3 * g);
                    ++nown;
                    last = gk;
                }
                bool ok;
                {
                    bool done = !err;
                    if (!err && nown > 0)
                        done = wait_bar(&vo_done[last % C::NV], (last / C::NV) & 1, wc, SITE_O_DONE, true);
                    ok = bar_and(BAR_SOFT, NSOFT, done);  // reached by all 256 threads
                }
                // whether warpgroup h had key tiles in this query tile (the same
                // for every thread, so the TMEM loads below stay warp-uniform)
                const bool has0 = nT >= 2 || (gg & 1) == 0;
                const bool has1 = nT >= 2 || (gg & 1) == 1;
                gg += nT;
                if (!ok) break;
                tc_fence_after();
                // Merge the two warpgroups' partial softmaxes.  With
                // M = max(m_0, m_1), b_h = 2^(m_h - M), L = sum_h b_h l_h:
                //   O   = sum_h b_h O_h / L,
                //   lse' = mu = sum_h b_h (a_h + c_h l_h) / L,
                //   O'  = sum_h b_h (O'_h + (c_h - mu) O_h) / L.
                xch[(g * 4 + 0) * 128 + r] = m_used;
                xch[(g * 4 + 1) * 128 + r] = l;
                xch[(g * 4 + 2) * 128 + r] = acc_a;
                xch[(g * 4 + 3) * 128 + r] = cctr;
                bar_sync(BAR_SOFT, NSOFT);
                const float m0 = xch[r], l0 = xch[128 + r], a0v = xch[256 + r], c0v = xch[384 + r];
                const float m1 = xch[512 + r], l1 = xch[640 + r], a1v = xch[768 + r], c1v = xch[896 + r];
                const float M = has0 ? (has1 ? fmaxf(m0, m1) : m0) : m1;
                const float b0 = has0 ? ex2_approx(m0 - M) : 0.f;
                const float b1 = has1 ? ex2_approx(m1 - M) : 0.f;
                const float lt = (has0 ? b0 * l0 : 0.f) + (has1 ? b1 * l1 : 0.f);
                const float inv_l = 1.f / lt;
                const float mu = ((has0 ? b0 * fmaf(c0v, l0, a0v) : 0.f) + (has1 ? b1 * fmaf(c1v, l1, a1v) : 0.f)) * inv_l;
                // A key range of a split tile keeps its state unnormalised:
                // m = M, l = L, c = mu, a = 0, O = sum_h b_h O_h and
                // O' = sum_h b_h (O'_h + (c_h - mu) O_h).
                const bool part = t.part >= 0;
                __nv_bfloat16 *out_ptr = out_row();
                const size_t lrow = lse_row();
                const float wn = part ? 1.f : inv_l;
                const float w0 = b0 * wn, w1 = b1 * wn;
                const float k0 = w0 * (c0v - mu), k1 = w1 * (c1v - mu);
                if (part && g == 0) part_put_scalars<D>(p, t.part, r, M, lt, 0.f, mu);
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    float acc[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (!(h == 0 ? has0 : has1)) continue;
                        const float wh = h == 0 ? w0 : w1, kh = h == 0 ? k0 : k1;
                        uint32_t ov[32];
                        tmem_ld32(tbase + lane_off + C::T_O(h) + c, ov);
                        if (g == 0) {
                            tmem_ld_wait(ov);
#pragma unroll
                            for (int i = 0; i < 32; ++i) acc[i] = fmaf(wh, u2f(ov[i]), acc[i]);
                        } else {
                            uint32_t odv[32];
                            tmem_ld32(tbase + lane_off + C::T_OD(h) + c, odv);
                            tmem_ld_wait2(ov, odv);
#pragma unroll
                            for (int i = 0; i < 32; ++i) acc[i] = fmaf(wh, u2f(odv[i]), fmaf(kh, u2f(ov[i]), acc[i]));
                        }
                    }
                    if (part) {
                        part_put_cols<D>(p, t.part, r, g, c, acc);
                        continue;
                    }
                    uint32_t pv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) pv[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
                    store_cols32<D>(out_ptr, c, pv, p.out_v8, lane & 1, (grow & ~1) < p.Lq, (grow | 1) < p.Lq);
                }
                if (part) {
                    split_finish<D>(p, t, g, r, out_ptr, grow, lrow, smem + C::OFF_MISC + 8);
                } else {
                    if (g == 0 && grow < p.Lq) p.lse[lrow] = (M + log2f(lt)) * 0.69314718055994531f;
                    if (g == 1 && p.lse_dot && grow < p.Lq) p.lse_dot[lrow] = mu;
                }
                // Both warpgroups read O_0 and O_1 above; the next query tile's
                // first P (after which the MMAs restart an accumulator) comes
                // from one warpgroup only, so meet here first.  This also
                // keeps the exchange slots from being overwritten early.
                tc_fence_before();
                bar_sync(BAR_SOFT, NSOFT);
            }
        } else {
        // [0, 512): per-warpgroup l and a of the query tile ([slot][g][row]);
        // [512, 640): the centring constant handed from warpgroup 0 to 1.
        // The hand-off has a slot of its own, because warpgroup 0 may start
        // the next query tile while warpgroup 1 still reads the l, a of this one.
        const int c0 = 32 * g;
        int gg = 0;
        Tile t;
        for (int k = 0;; ++k) {
            const int itk = item_of(p, k, t);
            if (itk == ITEM_END) break;
            if (itk == ITEM_SKIP) continue;
            const int grow = t.q0 + r;
            const size_t orow = (static_cast<size_t>(t.bh) * p.Lq + grow) * D;
            __nv_bfloat16 *out_ptr = static_cast<__nv_bfloat16 *>(g == 0 ? p.o : p.od) + orow;
            const size_t lrow = static_cast<size_t>(t.bh) * p.Lq + grow;
            if (t.nT == 0) {
                if (grow < p.Lq) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4 *>(out_ptr)[c] = z;
                    if (g == 0) p.lse[lrow] = -INFINITY;
                    if (g == 1 && p.lse_dot) p.lse_dot[lrow] = 0.f;
                }
                continue;
            }
            const int nb = t.nb, nT = t.nT;
            // l: exact fp32 sum of p (normalises O and O', gives lse);
            // acc_a: sum of the bf16-rounded P (sS' - c) that the MMAs consume,
            // so the rounding of those operands reaches O' only through
            // (v_j - O), which is small for the keys that dominate.
            float m_used = -INFINITY, l = 0.f, acc_a = 0.f, cctr = 0.f;
            // No named barrier inside the key loop: every thread reads the
            // whole 64-column row of S and forms the same row max, so the two
            // warpgroups need not meet, and each warp runs through the key
            // tiles at its own pace, coupled only by the MMA barriers.  A wait
            // that gives up sets `err` and leaves the loop; the barrier after
            // the loop is reached by all 256 threads either way.
            bool err = false;
            for (int j = 0; j < nT; ++j) {
                const int gk = gg + j;
                const int bsel = gk & 1;
                const uint32_t tS = tbase + lane_off + C::T_S + bsel * (2 * BN);
                if (!__all_sync(0xffffffffu, wait_bar_fast(&ks_done[gk % C::NK], (gk / C::NK) & 1, wc, SITE_S_FULL))) {
                    err = true;
                    if (j == 0) bar_and(BAR_SOFT, NSOFT, false);  // the others wait there at key tile 0
                    break;
                }
                if (tracer) stamp(gk, EV_SM_S + 3 * g);
                tc_fence_after();
                const int vt = nb - (t.jb + j) * BN;  // valid keys in the tile
                const int valid = vt - c0;   // valid columns of this half
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
                        // pair i goes to the FMA pipe when (i mod 4) < POLY_QUARTERS
                        if ((i & 3) < C::POLY_QUARTERS) {
                            ex2_poly2(t0, t1, x[2 * i], x[2 * i + 1]);
                        } else {
                            x[2 * i] = ex2_approx(t0);
                            x[2 * i + 1] = ex2_approx(t1);
                        }
                    }
                }
                if (tail) {
                    // padded keys: p = 0 exactly (the pad times a zero scale is NaN)
#pragma unroll
                    for (int i = 0; i < 32; ++i) x[i] = (i < valid) ? x[i] : 0.f;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                // The PV MMAs of the previous key tile must be done before O
                // may be rescaled, so a warp that rescales waits for them.  A
                // warp that does not rescale skips the wait (most tiles): the
                // phase it would wait for can never be confused with another,
                // since S of this tile (seen above) implies that the phases of
                // key tiles <= gk - 2 are complete, and that of gk + 1 needs
                // this warp's P of key tile gk + 1.
                const bool do_rescale = __any_sync(0xffffffffu, rescale);
                if (j >= 1 && do_rescale) {
                    if (!__all_sync(0xffffffffu, wait_bar_fast(&vo_done[(gk - 1) % C::NV], ((gk - 1) / C::NV) & 1,
                                                               wc, SITE_O_DONE))) {
                        err = true;
                        break;
                    }
                    tc_fence_after();
                }
                if (do_rescale) {
                    const uint32_t tacc = tbase + lane_off + (g == 0 ? C::T_O(0) : C::T_OD(0));
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t tt[32];
                        tmem_ld32(tacc + c, tt);
                        tmem_ld_wait(tt);
#pragma unroll
                        for (int i = 0; i < 32; ++i) tt[i] = f2u(u2f(tt[i]) * alpha);
                        tmem_st32(tacc + c, tt);
                    }
                }
                if (tail && !(ZKV && g == 1)) {  // (no V' tile with V' = 0)
                    // Zero the V (g = 0) / V' (g = 1) rows of padded keys so
                    // their bits (NaN included) cannot reach the PV products.
                    // Each warp zeroes its share and fences before it signals P.
                    const int s = gk % C::NV;
                    if (!__all_sync(0xffffffffu, wait_bar(&v_full[s], (gk / C::NV) & 1, wc, SITE_V_TAIL))) {
                        err = true;
                        if (j == 0) bar_and(BAR_SOFT, NSOFT, false);  // the others wait there at key tile 0
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
                if (lane == 0) mbar_arrive(&p_full[bsel]);
                if (tracer) stamp(gk, EV_SM_P + 3 * g);
                // l, S'_raw and (first tile) the centring constant are needed
                // only for P (sS' - c), so they come after P is on its way
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
                        // all p of keys 0..31 can be 0 (the max among keys
                        // 32..63, keys 0..31 far below it): c cancels exactly,
                        // so any finite value is right, and 0 is taken
                        const float wsum = w0 + w1;
                        cctr = wsum > 0.f ? (n0 + n1) / wsum : 0.f;
                        xch[512 + r] = cctr;
                    }
                    if (!bar_and(BAR_SOFT, NSOFT, true)) {
                        err = true;
                        break;
                    }
                    if (g == 1) cctr = xch[512 + r];
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
                if (lane == 0) mbar_arrive(&pd_full[bsel]);
                if (tracer) stamp(gk, EV_SM_PD + 3 * g);
            }
            bool ok;
            {
                bool done = false;
                if (!err) {
                    const int last = gg + nT - 1;
                    done = wait_bar(&vo_done[last % C::NV], (last / C::NV) & 1, wc, SITE_O_DONE, true);
                }
                ok = bar_and(BAR_SOFT, NSOFT, done);  // reached by all 256 threads
            }
            gg += nT;
            if (!ok) break;  // the same for every softmax thread
            tc_fence_after();
            // l and a are split across the two warpgroups; add the halves
            // in a fixed order so both see the same totals.
            xch[g * 128 + r] = l;
            xch[256 + g * 128 + r] = acc_a;
            bar_sync(BAR_SOFT, NSOFT);
            const float lt = xch[r] + xch[128 + r];
            const float inv_l = 1.f / lt;
            const float coef = (xch[256 + r] + xch[384 + r]) * inv_l;
            const uint32_t to = tbase + lane_off + C::T_O(0);
            const uint32_t tod = tbase + lane_off + C::T_OD(0);
            if (t.part >= 0) {
                // a key range of a split tile: its unnormalised state
                if (g == 0) part_put_scalars<D>(p, t.part, r, m_used, lt, xch[256 + r] + xch[384 + r], cctr);
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t v[32];
                    tmem_ld32((g == 0 ? to : tod) + c, v);
                    tmem_ld_wait(v);
                    float acc[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = u2f(v[i]);
                    part_put_cols<D>(p, t.part, r, g, c, acc);
                }
                split_finish<D>(p, t, g, r, out_ptr, grow, lrow, smem + C::OFF_MISC + 8);
                continue;
            }
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
                store_cols32<D>(out_ptr, c, pv, p.out_v8, lane & 1, (grow & ~1) < p.Lq, (grow | 1) < p.Lq);
            }
            if (g == 0 && grow < p.Lq) p.lse[lrow] = (m_used + log2f(lt)) * 0.69314718055994531f;
            // lse' = sum_j P_j s S'_j = c + a / l
            if (g == 1 && p.lse_dot && grow < p.Lq) p.lse_dot[lrow] = cctr + coef;
            // the next query tile's first P (which lets the MMAs restart O and
            // O'_acc) is signalled after a tcgen05 fence that orders these loads
        }
        }  // by columns
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

// Per device, once: the kernel's shared-memory opt-in and the SM count
// (one persistent CTA per SM).
template <int D, bool ZKV, bool TRACE>
static int prepare_device(int dev, int *n_sm)
{
    static std::mutex mu;
    static bool done[MAX_DEVICES] = {};
    static int sms[MAX_DEVICES] = {};
    if (dev < 0 || dev >= MAX_DEVICES) return ATTN_JVP_ERR_LAUNCH;
    std::lock_guard<std::mutex> g(mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(attn_jvp_fwd_kernel<D, ZKV, TRACE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(Cfg<D>::SMEM_BYTES)) != cudaSuccess)
            return ATTN_JVP_ERR_LAUNCH;
        if (cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms[dev] < 1)
            return ATTN_JVP_ERR_LAUNCH;
        done[dev] = true;
    }
    *n_sm = sms[dev];
    return ATTN_JVP_OK;
}

// SM count of the current device (queried once per device).
static int device_sms(int *n_sm)
{
    static std::mutex mu;
    static int sms[MAX_DEVICES] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return ATTN_JVP_ERR_LAUNCH;
    std::lock_guard<std::mutex> g(mu);
    if (sms[dev] == 0 &&
        (cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms[dev] < 1)) {
        sms[dev] = 0;
        return ATTN_JVP_ERR_LAUNCH;
    }
    *n_sm = sms[dev];
    return ATTN_JVP_OK;
}

// How the last wave of query tiles is cut into key ranges.  With T query
// tiles on n_sm persistent CTAs, the first floor(T / n_sm) waves are walked
// whole and the R = T mod n_sm tiles left over are each cut into
// S = min(n_sm / R, key tiles, SPLIT_MAX) ranges, one per CTA, so the last
// wave takes about 1/S of a tile's time instead of a whole one.  No split
// when S < 2 (the last wave is nearly full, or a tile has one key tile).
struct SplitPlan {
    int grid = 0, n_full = 0, S = 0, n_units = 0, n_split_tiles = 0;
    size_t cnt_bytes = 0, bytes = 0;
};

static SplitPlan split_plan(long long T, int n_sm, int Lk, int d)
{
    SplitPlan sp;
    sp.grid = static_cast<int>(T < n_sm ? T : n_sm);
    sp.n_full = static_cast<int>(T);
    const long long nf = T / n_sm * n_sm;
    const int R = static_cast<int>(T - nf);
    const int nT = (Lk + BN - 1) / BN;
    int S = R ? n_sm / R : 0;
    S = S < nT ? S : nT;
    S = S < SPLIT_MAX ? S : SPLIT_MAX;
    if (S >= 2) {
        sp.grid = n_sm;
        sp.n_full = static_cast<int>(nf);
        sp.S = S;
        sp.n_units = R * S;
        sp.n_split_tiles = R;
        sp.cnt_bytes = (static_cast<size_t>(R) * 4 + 255) / 256 * 256;
        sp.bytes = sp.cnt_bytes + static_cast<size_t>(sp.n_units) * (4 + 2 * d) * BM * 4;
    }
    return sp;
}

template <int D, bool ZKV, bool TRACE = false>
static int launch_kernel(const Params &prm, int grid, cudaStream_t s)
{
    int dev = 0, n_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (int rc = prepare_device<D, ZKV, TRACE>(dev, &n_sm)) return rc;
    attn_jvp_fwd_kernel<D, ZKV, TRACE><<<grid, NTHREADS, Cfg<D>::SMEM_BYTES, s>>>(prm);
    return ATTN_JVP_OK;
}

static bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// allow_zero_kv: k_dot and v_dot may both be NULL (K' = V' = 0).
// trace != NULL: the trace build, stamping [trace_ctas][trace_tiles][TRACE_EVENTS].
// workspace != NULL: the last-wave key split, with its records and counters
// in workspace (workspace_bytes at least what split_plan asks for).
static int launch(const void *q, const void *k, const void *v, const void *qd, const void *kd,
                  const void *vd, void *o, void *od, float *lse, float *lse_dot, int B, int H, int Lq,
                  int Lk, int d, float scale, const int32_t *kv_len, void *stream, uint64_t timeout_ns,
                  int flags, bool allow_zero_kv, unsigned long long *trace = nullptr, int trace_tiles = 0,
                  int trace_ctas = 0, void *workspace = nullptr, size_t workspace_bytes = 0,
                  bool use_split = false)
{
    const bool zkv = allow_zero_kv && !kd && !vd;
    if (!q || !k || !v || !qd || (!zkv && (!kd || !vd)) || !o || !od || !lse) return ATTN_JVP_ERR_NULL;
    if (flags & ~ATTN_JVP_DEBUG_STARVE_Q) return ATTN_JVP_ERR_VALUE;
    if (trace && (trace_tiles < 1 || trace_ctas < 1 || (reinterpret_cast<uintptr_t>(trace) & 7)))
        return trace_tiles < 1 || trace_ctas < 1 ? ATTN_JVP_ERR_VALUE : ATTN_JVP_ERR_ALIGN;
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
    const size_t ntr = trace ? static_cast<size_t>(trace_ctas) * trace_tiles * TRACE_EVENTS * 8 : 0;
    const void *outs[5] = {o, od, lse, lse_dot, trace};
    const size_t outsz[5] = {nq, nq, nl, nl, ntr};
    for (int i = 0; i < 5; ++i) {
        if (!outs[i]) continue;
        for (int j = 0; j < 6; ++j)
            if (ins[j] && ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return ATTN_JVP_ERR_VALUE;
        for (int j = i + 1; j < 5; ++j)
            if (outs[j] && ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return ATTN_JVP_ERR_VALUE;
    }

    const int nqt = (Lq + BM - 1) / BM;
    const long long n_tiles = static_cast<long long>(nqt) * BH;  // < 2^31 / BM by the check above
    int n_sm = 0;
    if (int rc = device_sms(&n_sm)) return rc;
    SplitPlan sp;
    if (use_split) {
        sp = split_plan(n_tiles, n_sm, Lk, d);
    } else {  // every tile whole, round robin over min(tiles, SMs) CTAs
        sp.grid = static_cast<int>(n_tiles < n_sm ? n_tiles : n_sm);
        sp.n_full = static_cast<int>(n_tiles);
    }
    const size_t nws = use_split ? sp.bytes : 0;
    if (nws) {
        if (!workspace) return ATTN_JVP_ERR_NULL;
        if (reinterpret_cast<uintptr_t>(workspace) & 255) return ATTN_JVP_ERR_ALIGN;
        if (workspace_bytes < nws) return ATTN_JVP_ERR_VALUE;
        for (int j = 0; j < 6; ++j)
            if (ins[j] && ranges_overlap(workspace, nws, ins[j], insz[j])) return ATTN_JVP_ERR_VALUE;
        for (int j = 0; j < 5; ++j)
            if (outs[j] && ranges_overlap(workspace, nws, outs[j], outsz[j])) return ATTN_JVP_ERR_VALUE;
    }

    Params prm;
    std::memset(&prm, 0, sizeof prm);
    if (!make_map(&prm.tm_q, q, d, Lq, BH, BM) || !make_map(&prm.tm_qd, qd, d, Lq, BH, BM) ||
        !make_map(&prm.tm_k, k, d, Lk, BH, BN) || !make_map(&prm.tm_v, v, d, Lk, BH, BN) ||
        (!zkv && (!make_map(&prm.tm_kd, kd, d, Lk, BH, BN) || !make_map(&prm.tm_vd, vd, d, Lk, BH, BN))))
        return ATTN_JVP_ERR_LAUNCH;
    prm.o = o;
    prm.od = od;
    prm.out_v8 = ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(od)) & 31u) == 0;
    prm.lse = lse;
    prm.lse_dot = lse_dot;
    prm.kv_len = kv_len;
    prm.H = H;
    prm.Lq = Lq;
    prm.Lk = Lk;
    prm.nqt = nqt;
    prm.n_tiles = static_cast<int>(n_tiles);
    prm.scale = scale;
    prm.sl2 = scale * 1.4426950408889634f;
    prm.timeout_ns = timeout_ns ? timeout_ns : DEFAULT_TIMEOUT_NS;
    prm.flags = flags;
    prm.trace = trace;
    prm.trace_tiles = trace_tiles;
    prm.trace_ctas = trace_ctas;
    prm.n_full = sp.n_full;
    prm.split_S = sp.S;
    prm.n_units = sp.n_units;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (nws) {
        prm.cnt = static_cast<int *>(workspace);
        prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + sp.cnt_bytes);
        if (cudaMemsetAsync(workspace, 0, sp.cnt_bytes, s) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    }

    int rc;
    const int grid = sp.grid;
    if (trace) rc = d == 64 ? launch_kernel<64, false, true>(prm, grid, s) : launch_kernel<128, false, true>(prm, grid, s);
    else if (zkv) rc = d == 64 ? launch_kernel<64, true>(prm, grid, s) : launch_kernel<128, true>(prm, grid, s);
    else rc = d == 64 ? launch_kernel<64, false>(prm, grid, s) : launch_kernel<128, false>(prm, grid, s);
    if (rc) return rc;
    if (cudaGetLastError() != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    return ATTN_JVP_OK;
}

// ---- the split path with library-owned scratch (attn_jvp_fwd_noalloc)
//
// For callers that cannot allocate device memory: runtimes that own all of
// the device memory and give a kernel library no allocator (only its inputs
// and outputs), and latency-critical loops that must not call cudaMalloc,
// which can synchronise the device and stall every stream.  The workspace of
// the last-wave split lives in this file-scope array instead: every device
// that loads the library holds its NOALLOC_SCRATCH_BYTES until the process
// exits, and every call on a device shares it.
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(20) << 20;  // 20 MiB: 148 SMs at d = 128 need 19.7 MB
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (host code must not pass the array's name itself: that is a
// host-side stand-in, not a device address).
static int noalloc_scratch(void **ptr)
{
    static std::mutex mu;
    static void *addr[MAX_DEVICES] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return ATTN_JVP_ERR_LAUNCH;
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ATTN_JVP_ERR_LAUNCH;
        addr[dev] = p;
    }
    *ptr = addr[dev];
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

size_t attn_jvp_workspace_bytes(int B, int H, int Lq, int Lk, int d)
{
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1 || (d != 64 && d != 128)) return 0;
    const long long BH = static_cast<long long>(B) * H;
    if (BH * Lq >= (1ll << 31) || BH * Lk >= (1ll << 31)) return 0;
    int n_sm = 0;
    if (ajvp::device_sms(&n_sm)) return 0;
    const long long T = static_cast<long long>((Lq + ajvp::BM - 1) / ajvp::BM) * BH;
    return ajvp::split_plan(T, n_sm, Lk, d).bytes;
}

int attn_jvp_fwd_ws(const void *q, const void *k, const void *v, const void *q_dot, const void *k_dot,
                    const void *v_dot, void *o, void *o_dot, float *lse, float *lse_dot, int B, int H,
                    int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *workspace,
                    size_t workspace_bytes, void *stream)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, lse_dot, B, H, Lq, Lk, d, scale,
                        kv_len, stream, 0, 0, true, nullptr, 0, 0, workspace, workspace_bytes, true);
}

int attn_jvp_fwd_noalloc(const void *q, const void *k, const void *v, const void *q_dot,
                         const void *k_dot, const void *v_dot, void *o, void *o_dot, float *lse,
                         float *lse_dot, int B, int H, int Lq, int Lk, int d, float scale,
                         const int32_t *kv_len, void *stream)
{
    // The same checks as attn_jvp_fwd_ws, with the static scratch as the
    // workspace; a shape whose workspace would not fit is refused before any
    // CUDA call that touches the scratch.
    if (B < 1 || H < 1 || Lq < 1 || Lk < 1) return ATTN_JVP_ERR_SHAPE;
    if (d != 64 && d != 128) return ATTN_JVP_ERR_HEADDIM;
    const long long BH = static_cast<long long>(B) * H;
    if (BH * Lq >= (1ll << 31) || BH * Lk >= (1ll << 31)) return ATTN_JVP_ERR_SHAPE;
    int n_sm = 0;
    if (int rc = ajvp::device_sms(&n_sm)) return rc;
    const long long T = static_cast<long long>((Lq + ajvp::BM - 1) / ajvp::BM) * BH;
    if (ajvp::split_plan(T, n_sm, Lk, d).bytes > ajvp::NOALLOC_SCRATCH_BYTES) return ATTN_JVP_ERR_SCRATCH;
    void *scratch = nullptr;
    if (int rc = ajvp::noalloc_scratch(&scratch)) return rc;
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, lse_dot, B, H, Lq, Lk, d, scale,
                        kv_len, stream, 0, 0, true, nullptr, 0, 0, scratch, ajvp::NOALLOC_SCRATCH_BYTES, true);
}

int attn_jvp_fwd_debug(const void *q, const void *k, const void *v, const void *q_dot,
                       const void *k_dot, const void *v_dot, void *o, void *o_dot, float *lse, int B,
                       int H, int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *stream,
                       uint64_t timeout_ns, int flags)
{
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, nullptr, B, H, Lq, Lk, d, scale,
                        kv_len, stream, timeout_ns, flags, false);
}

int attn_jvp_fwd_trace(const void *q, const void *k, const void *v, const void *q_dot,
                       const void *k_dot, const void *v_dot, void *o, void *o_dot, float *lse, int B,
                       int H, int Lq, int Lk, int d, float scale, const int32_t *kv_len, void *stream,
                       unsigned long long *trace, int trace_tiles, int trace_ctas)
{
    if (!trace) return ATTN_JVP_ERR_NULL;
    return ajvp::launch(q, k, v, q_dot, k_dot, v_dot, o, o_dot, lse, nullptr, B, H, Lq, Lk, d, scale,
                        kv_len, stream, 0, 0, false, trace, trace_tiles, trace_ctas);
}

int attn_jvp_check(void *stream, int *site)
{
    if (site) *site = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(ajvp::g_check_mu);
    ajvp::take_status_kernel<<<1, 1, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    int st = 0;
    if (cudaMemcpyFromSymbolAsync(&st, ajvp::g_status_taken, sizeof st, 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ATTN_JVP_ERR_LAUNCH;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_JVP_ERR_LAUNCH;
    if (st == 0) return ATTN_JVP_OK;
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
    case ATTN_JVP_ERR_SCRATCH: return "the split workspace this shape needs exceeds the library's static scratch";
    default: return "unknown status";
    }
}

int attn_jvp_version(void) { return 200; }

}  // extern "C"

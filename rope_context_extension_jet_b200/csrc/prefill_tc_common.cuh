// prefill_tc_common.cuh -- pieces shared by the two tensor-core prefill kernels
// of dynamic bifocal RoPE attention (one CTA per work unit in prefill_tc.cu, a
// CTA pair sharing every MMA in prefill_pair.cu): tile classification, the
// floor(x / G) division, bounded barrier waits, the in-place RoPE of a swizzled
// shared-memory tile, the softmax role and the host-side TMA descriptors.
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740), Metodologia 1-2: a pair (i, j) with
// i - j < w0 is rotated at (i, j), every other pair at (floor(i/G), floor(j/G));
// both branches feed one softmax.
#pragma once

#include <cuda.h>

#include <mutex>

#include "jl_common.cuh"
#include "jl_ptx.cuh"
#include "tc_ptx.cuh"

namespace jl {
namespace tc {

constexpr int BM = 128, BN = 128;
constexpr int kVarlenMax = 64;  // sequences of one variable-length launch
constexpr int ATOM = 128 * 128;  // bytes of one 128-row x 64-column 16-bit swizzle atom
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
// softmax exponentials of the one-CTA kernel: one pair in every
// kPolyExpPeriod groups of four columns goes to ex2_poly2 (FMA pipe), the rest
// to the MUFU.  (The CTA-pair kernel measured no gain from it: all its
// exponentials use the MUFU.)
constexpr int kPolyExpPeriod = 2;

enum { CLS_REM = 0, CLS_LOC = 1, CLS_BAND = 2 };

// Query rows are positions [P, P + C) (row i of q / out is position P + i),
// keys [0, L), L = P + C; nqb query blocks of BM rows.
struct TcParams {
    int B, Hq, Hkv, L, w0, G, nqb;
    int P, C, Cst;  // Cst: q / out / lse rows per (b, head) in memory
    uint32_t div_m, div_s1, div_s2;  // floor(x / G) by multiply-shift
    float scale_log2;
    RopeTurns turns;
    __nv_bfloat16* out;
    float* out_f32;  // if set, the output rows are written here in fp32 instead of `out`
    float* lse;      // optional
    int window_rot;  // -1 routed; 0 / 1: pairs i - j < w0 only, exact / aliased rotation
    int* dev_error;
    long long wait_cycles;  // limit of every bounded wait
    int inject;             // kInjectNone, or the arrival this launch withholds (test hook)
    // largest |q| and |k| of this call as bf16 magnitude bits, written by the
    // range scan launched just before on the same stream
    const uint32_t* range;
    // variable-length batches (vl_n > 0): sequence b of the launch has length
    // vl_len[b] (rows [0, vl_len[b]) of planes of Cst rows), its own G and
    // floor(x / G) constants; the grid's x runs over (query-block level, b)
    int vl_n, vl_nqb_max;
    int vl_len[kVarlenMax];
    uint32_t vl_div[kVarlenMax][3];
};

// The sequence and query block a CTA (pair) works on, with that sequence's
// length, window and floor(x / G) constants.
struct SeqView {
    int b, qb, L, w0;
    uint32_t div_m, div_s1, div_s2;
};

// Work unit `unit` (the CTA's place along the grid's x, heaviest first) of the
// launch, batch index bz (blockIdx.z).  Returns false for a unit past the end
// of a shorter sequence of a variable-length batch (the CTA then has no work).
__device__ __forceinline__ bool seq_view(const TcParams& p, int unit, int bz, SeqView& v)
{
    if (p.vl_n == 0) {
        v.b = bz;
        v.qb = p.nqb - 1 - unit;
        v.L = p.L;
        v.w0 = p.w0;
        v.div_m = p.div_m;
        v.div_s1 = p.div_s1;
        v.div_s2 = p.div_s2;
        return true;
    }
    // all sequences' blocks of one level (counted from the longest sequence's
    // last block) before the next lighter level
    v.b = unit % p.vl_n;
    v.qb = p.vl_nqb_max - 1 - unit / p.vl_n;
    v.L = p.vl_len[v.b];
    v.w0 = min(p.w0, v.L);
    v.div_m = p.vl_div[v.b][0];
    v.div_s1 = p.vl_div[v.b][1];
    v.div_s2 = p.vl_div[v.b][2];
    return v.qb * BM < v.L;
}

// ------------------------------------------------------------ operand range
// The Q K^T operands are rounded to fp16 (an 11-bit significand: the inputs'
// 8-bit bf16 significand would cost the logits too much precision), whose range
// ends at 65504 while bf16 inputs reach 3.4e38.  So the rotated queries and keys
// are scaled by powers of two 2^e_q and 2^e_k that bring the call's largest
// |q| and |k| into [2^13, 2^14): a rotated value is at most sqrt(2) times the
// largest input of its pair, so every operand stays below 2^14.5, and inputs
// down to 2^27 below the largest keep fp16's full relative precision (smaller
// ones become subnormal or zero; their part of a logit is then below 2^-38 of
// the largest terms).  A power of two is exact both ways, so the softmax, which
// multiplies S by scale * log2(e) * 2^-(e_q + e_k), sees the logits of the
// unscaled operands; for inputs already in range the result is bit-identical.
// Exponents are clamped to [-100, 100].
__device__ __forceinline__ int range_exp(uint32_t mag)
{
    if (mag == 0u || mag >= 0x7f80u) return 0;  // all zero, or non-finite: nothing to rescale
    const int biased = (int)(mag >> 7);
    const int ilogb = (biased == 0 ? 1 : biased) - 127;  // subnormals: at most 2^-126
    return min(100, max(-100, 13 - ilogb));
}

// 2^e as fp32 for e in [-126, 127].
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

__device__ __forceinline__ uint32_t ld_range(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.global.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// 2^y for a pair y (y <= 2^7) on the FMA and integer pipes, sparing the MUFU
// that evaluates the other exponentials of the softmax.  y = n + f with
// n = round(y) (adding 1.5 * 2^23 rounds to an integer held in the low bits)
// and f in [-1/2, 1/2]; 2^f by a cubic fitted to 2^f over that interval for the
// least largest relative error (7.5e-5, against 2^-9 for the bf16 rounding of
// P); 2^n from the exponent field n + 127.  y is first raised to -127 by a
// max that keeps NaN: there the exponent field is 0, so -inf gives exactly 0,
// and a NaN stays NaN.
__device__ __forceinline__ float2 ex2_poly2(float2 y)
{
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    constexpr float C0 = 0.99992806f, C1 = 0.69326097f, C2 = 0.24261114f, C3 = 0.055171669f;
    float a, b;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(a) : "f"(y.x), "f"(-127.f));
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(b) : "f"(y.y), "f"(-127.f));
    const float2 yc = make_float2(a, b);
    const float2 t = add2(yc, make_float2(kRound, kRound));
    const float2 n = add2(t, make_float2(-kRound, -kRound));
    const float2 f = fma2(n, make_float2(-1.f, -1.f), yc);  // exact: y - n
    float2 p = fma2(make_float2(C3, C3), f, make_float2(C2, C2));
    p = fma2(p, f, make_float2(C1, C1));
    p = fma2(p, f, make_float2(C0, C0));
    // low bits of t hold n (two's complement); (n + 127) << 23 is 2^n
    const float2 s = make_float2(__uint_as_float((__float_as_uint(t.x) + 127u) << 23),
                                 __uint_as_float((__float_as_uint(t.y) + 127u) << 23));
    return mul2(p, s);
}

__device__ __forceinline__ uint32_t div_g(uint32_t n, const SeqView& v)
{
    // Granlund & Montgomery, "Division by Invariant Integers using
    // Multiplication" (1994), Fig. 4.1: exact for all 32-bit n.
    const uint32_t t1 = __umulhi(v.div_m, n);
    return (t1 + ((n - t1) >> v.div_s1)) >> v.div_s2;
}

// Class of the tile (query rows from position i_lo, key block kb): every pair
// local, every pair remote, or both (the band i - j = w0 crosses the tile).
__device__ __forceinline__ int tile_class(int i_lo, int kb, int L, int w0)
{
    const int i_hi = min(i_lo + BM - 1, L - 1);
    const int dmax = i_hi - kb * BN;
    const int dmin = max(0, i_lo - (kb * BN + BN - 1));
    if (dmax < w0) return CLS_LOC;
    if (dmin >= w0) return CLS_REM;
    return CLS_BAND;
}

// Key tiles of the query block starting at position i_lo in processing order:
// phase R = [0, nR) (remote and band tiles, rotated at the aliased positions),
// then phase E = [kE0, nkb) (band and local tiles, rotated at the exact
// positions).
struct TilePlan {
    int nR, kE0, nkb;
    __device__ __forceinline__ int count() const { return nR + (nkb - kE0); }
    __device__ __forceinline__ int kb(int e) const { return e < nR ? e : kE0 + (e - nR); }
};

__device__ __forceinline__ TilePlan plan_tiles(int i_lo, int L, int w0)
{
    TilePlan t;
    t.nkb = min(i_lo + BM - 1, L - 1) / BN + 1;
    t.nR = t.nkb;
    t.kE0 = t.nkb;
    for (int kb = 0; kb < t.nkb; ++kb) {
        const int cls = tile_class(i_lo, kb, L, w0);
        if (cls != CLS_REM && t.kE0 == t.nkb) t.kE0 = kb;
        if (cls == CLS_LOC) { t.nR = kb; break; }
    }
    return t;
}

template <bool CLUSTER>
__device__ __forceinline__ bool bar_try_wait(uint64_t* bar, uint32_t parity)
{
    return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
}

// Bounded wait that also gives up once another role of the CTA aborted.  The
// CLUSTER form acquires at cluster scope (the phase was completed by arrivals
// or MMA commits from the other CTA of a pair).
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int* dev_error, long long limit, int code)
{
    if (bar_try_wait<CLUSTER>(bar, parity)) return true;
    const long long t0 = clock64();
    while (!bar_try_wait<CLUSTER>(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            record_error(dev_error, code);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Warp-collective form: every lane polls, and the warp proceeds only if all did.
template <bool CLUSTER = false>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_error, long long limit, int code)
{
    const bool ok = wait_or_abort<CLUSTER>(bar, parity, abort_flag, dev_error, limit, code);
    return __all_sync(0xffffffffu, ok);
}

// Byte offset of 16-byte chunk `ch` (8 16-bit columns, ch < d/8) of row r in a
// ROWS-row tile stored as [d/64 atoms][ROWS rows][128 B] with the 128-byte
// swizzle (chunk index XOR row % 8): the layout TMA writes and UMMA K-major reads.
template <int ROWS>
__device__ __forceinline__ uint32_t sw128_off(int r, int ch)
{
    return (uint32_t)((ch >> 3) * (ROWS * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ float f16_lo(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u & 0xffffu))); }
__device__ __forceinline__ float f16_hi(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u >> 16))); }

// RoPE of a ROWS-row tile in place (pairs (m, m + d/2)), times lam, output fp16.  Thread t
// of the 128 rotation threads owns 8 frequencies (chunk c) of RPT consecutive
// rows.  pos(row) must step by 0 or 1 between consecutive rows (true for j,
// floor(j/G) and i - floor(i/G)); the angles of the first row come from the
// exact fixed-point phase, later rows advance by the per-frequency step
// rotation R(theta_m) (any other step is recomputed exactly).
//
// PACKED: the arithmetic runs on frequency pairs with packed f32x2 FMAs (fewer
// issue slots: the CTA-pair kernel, whose rotation warps compete with the
// softmax warps for issue); otherwise on scalar FMAs (the one-CTA kernel, which
// measured faster that way).  Both compute in fp32, each value as one product
// and one fused multiply-add.
template <int D, int ROWS, bool IN_BF16, bool PACKED, class PosFn>
__device__ __forceinline__ void rotate_tile(unsigned char* tile, int t, const TcParams& p, PosFn pos,
                                            const float2 (&stc)[4], const float2 (&sts)[4], float lam)
{
    constexpr int H = D / 2, CH = H / 8, RPT = ROWS * CH / 128;  // 128 threads = CH chunks x (ROWS / RPT) row groups
    static_assert(RPT >= 1 && ROWS * CH == 128 * RPT, "rotation thread mapping");
    const int c = t % CH, row0 = (t / CH) * RPT;
    // cos / sin of the thread's 8 frequencies as 4 pairs (2w, 2w + 1).  (cs, sn)
    // carry the operand scale lam: the step rotation is linear, so every row it
    // produces keeps it.
    float2 cs[4], sn[4];
    auto exact = [&](uint32_t q) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            float c0, s0, c1, s1;
            rope_cs_fast(q, p.turns.hi[c * 8 + 2 * w], p.turns.lo[c * 8 + 2 * w], c0, s0);
            rope_cs_fast(q, p.turns.hi[c * 8 + 2 * w + 1], p.turns.lo[c * 8 + 2 * w + 1], c1, s1);
            cs[w] = make_float2(c0 * lam, c1 * lam);
            sn[w] = make_float2(s0 * lam, s1 * lam);
        }
    };
    uint32_t prev = pos(row0);
    exact(prev);
#pragma unroll 2
    for (int s = 0; s < RPT; ++s) {
        const int r = row0 + s;
        if (s > 0) {
            const uint32_t cur = pos(r);
            if (cur == prev + 1) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    // (c, s) <- (c cos t - s sin t, s cos t + c sin t)
                    if (PACKED) {
                        const float2 c2 = __ffma2_rn(make_float2(-sn[w].x, -sn[w].y), sts[w], __fmul2_rn(cs[w], stc[w]));
                        sn[w] = __ffma2_rn(cs[w], sts[w], __fmul2_rn(sn[w], stc[w]));
                        cs[w] = c2;
                    } else {
                        const float2 c2 = make_float2(cs[w].x * stc[w].x - sn[w].x * sts[w].x,
                                                      cs[w].y * stc[w].y - sn[w].y * sts[w].y);
                        sn[w] = make_float2(sn[w].x * stc[w].x + cs[w].x * sts[w].x,
                                            sn[w].y * stc[w].y + cs[w].y * sts[w].y);
                        cs[w] = c2;
                    }
                }
            } else if (cur != prev) {
                exact(cur);
            }
            prev = cur;
        }
        uint4* plo = reinterpret_cast<uint4*>(tile + sw128_off<ROWS>(r, c));
        uint4* phi = reinterpret_cast<uint4*>(tile + sw128_off<ROWS>(r, c + CH));
        const uint4 a = *plo, bq = *phi;
        const uint32_t la[4] = {a.x, a.y, a.z, a.w};
        const uint32_t lb[4] = {bq.x, bq.y, bq.z, bq.w};
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            // x = the pair's first members (dims m, m + 1), y = their partners (m + d/2, ...)
            const float2 x = IN_BF16 ? make_float2(bf16_lo(la[w]), bf16_hi(la[w])) : make_float2(f16_lo(la[w]), f16_hi(la[w]));
            const float2 y = IN_BF16 ? make_float2(bf16_lo(lb[w]), bf16_hi(lb[w])) : make_float2(f16_lo(lb[w]), f16_hi(lb[w]));
            if (PACKED) {
                const float2 lo = __ffma2_rn(make_float2(-y.x, -y.y), sn[w], __fmul2_rn(x, cs[w]));  // x c - y s
                const float2 hi = __ffma2_rn(y, cs[w], __fmul2_rn(x, sn[w]));                       // x s + y c
                oa[w] = pack_f16x2(lo.x, lo.y);
                ob[w] = pack_f16x2(hi.x, hi.y);
            } else {
                oa[w] = pack_f16x2(x.x * cs[w].x - y.x * sn[w].x, x.y * cs[w].y - y.y * sn[w].y);
                ob[w] = pack_f16x2(x.x * sn[w].x + y.x * cs[w].x, x.y * sn[w].y + y.y * cs[w].y);
            }
        }
        *plo = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        *phi = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
}

// Per-frequency one-position step rotation R(theta_m) of rotation thread t, as
// the 4 frequency pairs rotate_tile works on.
template <int D>
__device__ __forceinline__ void rope_steps(int t, const TcParams& p, float2 (&stc)[4], float2 (&sts)[4])
{
    const int c = t % (D / 16);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        float c0, s0, c1, s1;
        rope_cs_fast(1u, p.turns.hi[c * 8 + 2 * w], p.turns.lo[c * 8 + 2 * w], c0, s0);
        rope_cs_fast(1u, p.turns.hi[c * 8 + 2 * w + 1], p.turns.lo[c * 8 + 2 * w + 1], c1, s1);
        stc[w] = make_float2(c0, c1);
        sts[w] = make_float2(s0, s1);
    }
}

// Softmax role of one query head: one thread per query row (= TMEM lane), 4
// warps.  For each key tile e: wait for S = Q K^T in TMEM (`sfull`), apply the
// causal / length / band masks, online softmax in base 2 with lazy O rescaling
// (after the previous P.V finished, `pvdone`), write P (bf16) over the first 64
// columns of S in two halves of 64 keys, signalling the MMA issuer after each
// (`arrive_p(half)`); finally O / l -> out.
// s_col / o_col are this warp's TMEM addresses of S and O.
template <int D, bool CLUSTER, class ArriveP>
__device__ __forceinline__ void softmax_role(const TcParams& p, const SeqView& sv, const TilePlan& tp, int head,
                                             int r, uint32_t s_col, uint32_t o_col, uint64_t* sfull,
                                             uint64_t* pvdone, ArriveP arrive_p, volatile int* abort_flag)
{
    const int lane = r & 31;
    const int L = sv.L, b = sv.b;
    const int i_lo = p.P + sv.qb * BM;
    const int i = i_lo + r;
    const int NE = tp.count();
    // scale * log2(e), times 2^-(e_q + e_k) to undo the operand scales; kept in
    // fp32's normal range, so a masked -inf column never meets a zero or
    // infinite factor (logits that small or large are outside fp32 anyway)
    const float sl2 = fminf(fmaxf(p.scale_log2 * pow2i(-range_exp(ld_range(p.range))) *
                                  pow2i(-range_exp(ld_range(p.range + 1))), 1.17549435e-38f), 3.40282347e38f);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int e = 0; e < NE; ++e) {
        const int kb = tp.kb(e);
        const bool phase_r = e < tp.nR;
        const int cls = tile_class(i_lo, kb, L, sv.w0);
        if (!warp_wait<CLUSTER>(sfull, e & 1, abort_flag, p.dev_error, p.wait_cycles, 0x331)) { ok = false; break; }
        tc_fence_after();
        float x[BN];
        {
            uint32_t t0[32], t1[32], t2[32], t3[32];  // four loads in flight, one wait
            tmem_ld32(s_col, t0);
            tmem_ld32(s_col + 32, t1);
            tmem_ld32(s_col + 64, t2);
            tmem_ld32(s_col + 96, t3);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                x[u] = __uint_as_float(t0[u]);
                x[32 + u] = __uint_as_float(t1[u]);
                x[64 + u] = __uint_as_float(t2[u]);
                x[96 + u] = __uint_as_float(t3[u]);
            }
        }
        const int j0 = kb * BN;
        const bool need_mask = (j0 + BN - 1 > i_lo) || (j0 + BN > L) || cls == CLS_BAND;
        if (need_mask) {
            const int dw = i - j0 - sv.w0;  // pair (i, j0 + u) is local iff u > dw
#pragma unroll
            for (int u = 0; u < BN; ++u) {
                const int j = j0 + u;
                bool masked = (j > i) || (j >= L);
                if (cls == CLS_BAND) masked = masked || (phase_r ? (u > dw) : (u <= dw));
                if (masked) x[u] = -INFINITY;
            }
        }
        float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int u = 4; u < BN; u += 8) {
            m4[0] = fmax3(m4[0], x[u], x[u + 1]);
            m4[1] = fmax3(m4[1], x[u + 2], x[u + 3]);
            m4[2] = fmax3(m4[2], x[u + 4], x[u + 5]);
            m4[3] = fmax3(m4[3], x[u + 6], x[u + 7]);
        }
        const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
        const float m_new = fmaxf(m_used, mt);
        const bool resc = m_new > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (resc) {
            alpha = ex2_approx(m_used - m_new);
            m_used = m_new;
            l *= alpha;
        }
        const float ms = m_used == -INFINITY ? 0.f : m_used;
        // p = 2^(x * scale * log2(e) - m), two columns per packed instruction
        // P in two halves of BN / 2 keys, each published (arrive_p(half)) as soon
        // as it is in TMEM, so P.V of the first half overlaps the exponentials of
        // the second
        const float2 sl = make_float2(sl2, sl2), nm = make_float2(-ms, -ms);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t pk[BN / 4];
#pragma unroll
            for (int v = 0; v < BN / 2; v += 4) {
                const int u = half * (BN / 2) + v;
                const float2 y0 = fma2(make_float2(x[u], x[u + 1]), sl, nm);
                const float2 y1 = fma2(make_float2(x[u + 2], x[u + 3]), sl, nm);
                const float2 p0 = make_float2(ex2_approx(y0.x), ex2_approx(y0.y));
                // one-CTA kernel: one pair in every kPolyExpPeriod steps of 4 on the FMA pipe
                const float2 p1 = !CLUSTER && (v / 4) % kPolyExpPeriod == kPolyExpPeriod - 1
                                      ? ex2_poly2(y1)
                                      : make_float2(ex2_approx(y1.x), ex2_approx(y1.y));
                acc0 = add2(acc0, p0);
                acc1 = add2(acc1, p1);
                pk[v >> 1] = pack_bf16x2(p0.x, p0.y);
                pk[(v >> 1) + 1] = pack_bf16x2(p1.x, p1.y);
            }
            // The previous P.V of this head has finished: the MMA issuer issues
            // it before Q K^T of this tile, whose commit (sfull) tracks every
            // earlier MMA of that thread.  So P may overwrite its columns now;
            // the rare O rescale (before any of this tile's P is published, so
            // before this tile's P.V) still checks pvdone explicitly.
            if (half == 0 && e > 0 && __any_sync(0xffffffffu, resc)) {
                if (!warp_wait<CLUSTER>(pvdone, (e - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x332)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t tt[32];
                    tmem_ld32(o_col + cc * 32, tt);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; ++u) tt[u] = __float_as_uint(__uint_as_float(tt[u]) * alpha);
                    tmem_st32(o_col + cc * 32, tt);
                }
            }
            static_assert(BN / 4 == 32, "one 32-column TMEM store per half");
            tmem_st32(s_col + half * 32, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_p(half);
        }
        if (!ok) break;
        l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
    }
    // epilogue: O / l -> bf16 -> out
    if (ok && NE > 0 && warp_wait<CLUSTER>(pvdone, (NE - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x333)) {
        tc_fence_after();
        const float inv = 1.f / l;
        const size_t row = ((size_t)b * p.Hq + head) * (size_t)p.Cst + (size_t)(i - p.P);
        __nv_bfloat16* orow = p.out + row * D;
        // natural log of the softmax denominator: (m + log2 l) * ln 2 (m, l in base 2)
        if (p.lse && i < L) p.lse[row] = (m_used + __log2f(l)) * 0.69314718055994531f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t tt[32];
            tmem_ld32(o_col + cc * 32, tt);
            tmem_wait_ld();
            if (i < L && p.out_f32) {
                // fp32 rows (the passes of the three-pass form, merged afterwards)
                float* frow = p.out_f32 + row * D + cc * 32;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4*>(frow + q * 4) =
                        make_float4(__uint_as_float(tt[q * 4 + 0]) * inv, __uint_as_float(tt[q * 4 + 1]) * inv,
                                    __uint_as_float(tt[q * 4 + 2]) * inv, __uint_as_float(tt[q * 4 + 3]) * inv);
            } else if (i < L) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(tt[q * 8 + 0]) * inv, __uint_as_float(tt[q * 8 + 1]) * inv);
                    v.y = pack_bf16x2(__uint_as_float(tt[q * 8 + 2]) * inv, __uint_as_float(tt[q * 8 + 3]) * inv);
                    v.z = pack_bf16x2(__uint_as_float(tt[q * 8 + 4]) * inv, __uint_as_float(tt[q * 8 + 5]) * inv);
                    v.w = pack_bf16x2(__uint_as_float(tt[q * 8 + 6]) * inv, __uint_as_float(tt[q * 8 + 7]) * inv);
                    *reinterpret_cast<uint4*>(orow + cc * 32 + q * 8) = v;
                }
            }
        }
    }
}

// ------------------------------------------------------------------ host side

// [planes][plane_rows][d] bf16 (fp16 when f16) read as rows [0, rows) of every
// plane (rows >= rows load as zeros), box 64 columns x box_rows rows x 1 plane,
// 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, int d, int rows, int plane_rows, int nplanes,
                     int box_rows, bool f16 = false);

// Parameters shared by both kernels (G magic numbers, RoPE turns, output).
TcParams make_params(const PrefillProblem& pp);

// The CTA-pair kernel (d = 128, query heads per kv head a multiple of 4).
cudaError_t launch_prefill_pair(const PrefillProblem& pp, cudaStream_t st);

}  // namespace tc
}  // namespace jl

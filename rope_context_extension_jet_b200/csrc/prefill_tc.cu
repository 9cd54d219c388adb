// prefill_tc.cu -- bf16 prefill of dynamic bifocal RoPE attention on the
// sm_100a tensor cores (TMA, tcgen05.mma, TMEM accumulators).
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740):
//   Metodologia 1 -- a pair (i, j) with i - j < w0 uses classic RoPE at i and
//   j; every other pair uses RoPE at f(i), f(j), f(x) = floor(x / G).
//   Metodologia 2 -- rotations are applied on the fly to unrotated inputs
//   (they compose additively) and all routed pairs feed one exact softmax.
//   The pages merge three FlashAttention passes by inclusion-exclusion; here
//   one pass computes the routed logits directly.
//
// Work unit: 128 query rows of NH = 2 query heads that share a kv head
// (grouped-query attention), so every raw K tile is loaded and rotated once
// for both heads.  Each CTA makes two passes over its key tiles (128 keys):
//   phase R -- tiles holding remote pairs (remote-only and band tiles), with Q
//              and K rotated to the aliased positions floor(x / G);
//   phase E -- tiles holding local pairs (band and local-only tiles), with Q
//              and K at their exact positions.
// A band tile (it straddles i - j = w0) appears in both phases, each time with
// the other branch's pairs masked out, so both branches feed the same online
// softmax.  Between the phases Q is re-rotated in place by i - floor(i/G)
// (rotations compose additively).
//
// Warp roles (512 threads, 4 warpgroups; registers rebalanced with setmaxnreg):
//   warp 0        TMA producer (raw Q once; raw K and V per tile)
//   warp 1        MMA issuer (one thread): S_h = Q_h K^T (fp16 operands) into
//                 TMEM; O_h += P_h V with P_h read from TMEM (bf16)
//   warp 2        TMEM allocation / release
//   warps 4-7     rotation: RoPE of Q and of every K tile in shared memory,
//                 angles advanced row by row with a per-frequency rotation step
//   warps 8-11    softmax for head 0, warps 12-15 for head 1: one thread per
//                 query row (= TMEM lane); causal / length / band masks, online
//                 softmax in base 2 with lazy O rescaling, P (bf16) back into
//                 TMEM over S, final O / l.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256, 256+d),
// O_1 [384, 384+d); P_h overwrites the first 64 columns of S_h.
//
// Every mbarrier wait is bounded; on expiry the CTA records an error code in
// the library's device error word, stops, drains its own copies and MMAs with
// bounded waits, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "jl_common.cuh"
#include "jl_ptx.cuh"
#include "tc_ptx.cuh"

namespace jl {
namespace {

constexpr int BM = 128, BN = 128, NSK = 2, NSV = 2, NTHREADS = 512;
constexpr int ATOM = 128 * 128;  // bytes of one 128-row x 64-column 16-bit swizzle atom
constexpr long long kTcWaitCycles = 1000000000ll;  // ~0.5 s: every wait here is on work of this CTA
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

enum { CLS_REM = 0, CLS_LOC = 1, CLS_BAND = 2 };
enum {
    B_QFULL = 0, B_QREADY0, B_QREADY1, B_QFREE,
    B_KFULL, B_KREADY = B_KFULL + NSK, B_KEMPTY = B_KREADY + NSK,
    B_VFULL = B_KEMPTY + NSK, B_VEMPTY = B_VFULL + NSV,
    B_SFULL = B_VEMPTY + NSV, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2,
    B_DRAIN = B_PVDONE + 2, NBARS
};

struct TcParams {
    int B, Hq, Hkv, L, w0, G, nqb;
    uint32_t div_m, div_s1, div_s2;  // floor(x / G) by multiply-shift
    float scale_log2;
    RopeTurns turns;
    __nv_bfloat16* out;
    int* dev_error;
};

template <int D, int NH>
struct TcSmem {
    static constexpr int ATOMS = D / 64;
    static constexpr int TILE = BM * D * 2;
    static constexpr int K0 = NH * TILE;
    static constexpr int V0 = K0 + NSK * TILE;
    static constexpr int BAR = V0 + NSV * TILE;
    static constexpr int END = BAR + NBARS * 8 + 16;
    static constexpr int TOTAL = END + 1024;  // slack to align the base to 1024
};

__device__ __forceinline__ uint32_t div_g(uint32_t n, const TcParams& p)
{
    // Granlund & Montgomery, "Division by Invariant Integers using
    // Multiplication" (1994), Fig. 4.1: exact for all 32-bit n.
    const uint32_t t1 = __umulhi(p.div_m, n);
    return (t1 + ((n - t1) >> p.div_s1)) >> p.div_s2;
}

__device__ __forceinline__ int tile_class(int qb, int kb, int L, int w0)
{
    const int i_lo = qb * BM, i_hi = min(qb * BM + BM - 1, L - 1);
    const int dmax = i_hi - kb * BN;
    const int dmin = max(0, i_lo - (kb * BN + BN - 1));
    if (dmax < w0) return CLS_LOC;
    if (dmin >= w0) return CLS_REM;
    return CLS_BAND;
}

// Bounded wait that also gives up once another role of the CTA aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int* dev_error, int code)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kTcWaitCycles) {
            record_error(dev_error, code);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Warp-collective form: every lane polls, and the warp proceeds only if all did.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_error, int code)
{
    const bool ok = wait_or_abort(bar, parity, abort_flag, dev_error, code);
    return __all_sync(0xffffffffu, ok);
}

// Byte offset of 16-byte chunk `ch` (8 16-bit columns, ch < d/8) of row r in a
// 128-row tile stored as [d/64 atoms][128 rows][128 B] with the 128-byte swizzle
// (chunk index XOR row % 8): the layout TMA writes and UMMA K-major reads.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch)
{
    return (uint32_t)((ch >> 3) * ATOM + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ float f16_lo(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u & 0xffffu))); }
__device__ __forceinline__ float f16_hi(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u >> 16))); }

// RoPE of a 128-row tile in place (pairs (m, m + d/2)), output fp16.  Thread t
// of the 128 rotation threads owns 8 frequencies (chunk c) of RPT consecutive
// rows.  pos(row) must step by 0 or 1 between consecutive rows (true for j,
// floor(j/G) and i - floor(i/G)); the angles of the first row come from the
// exact fixed-point phase, later rows advance by the per-frequency step
// rotation R(theta_m) (any other step is recomputed exactly).
template <int D, bool IN_BF16, class PosFn>
__device__ __forceinline__ void rotate_tile(unsigned char* tile, int t, const TcParams& p, PosFn pos,
                                            const float (&stc)[8], const float (&sts)[8])
{
    constexpr int H = D / 2, CH = H / 8, RPT = CH;  // 128 threads = CH chunks x (128 / RPT) row groups
    const int c = t % CH, row0 = (t / CH) * RPT;
    float cs[8], sn[8];
    uint32_t prev = pos(row0);
#pragma unroll
    for (int u = 0; u < 8; ++u) rope_cs_fast(prev, p.turns.hi[c * 8 + u], p.turns.lo[c * 8 + u], cs[u], sn[u]);
#pragma unroll 2
    for (int s = 0; s < RPT; ++s) {
        const int r = row0 + s;
        if (s > 0) {
            const uint32_t cur = pos(r);
            if (cur == prev + 1) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float c2 = cs[u] * stc[u] - sn[u] * sts[u];
                    sn[u] = sn[u] * stc[u] + cs[u] * sts[u];
                    cs[u] = c2;
                }
            } else if (cur != prev) {
#pragma unroll
                for (int u = 0; u < 8; ++u) rope_cs_fast(cur, p.turns.hi[c * 8 + u], p.turns.lo[c * 8 + u], cs[u], sn[u]);
            }
            prev = cur;
        }
        uint4* plo = reinterpret_cast<uint4*>(tile + sw128_off(r, c));
        uint4* phi = reinterpret_cast<uint4*>(tile + sw128_off(r, c + CH));
        const uint4 a = *plo, bq = *phi;
        const uint32_t la[4] = {a.x, a.y, a.z, a.w};
        const uint32_t lb[4] = {bq.x, bq.y, bq.z, bq.w};
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            float x0, x1, y0, y1;
            if (IN_BF16) {
                x0 = bf16_lo(la[w]); x1 = bf16_hi(la[w]); y0 = bf16_lo(lb[w]); y1 = bf16_hi(lb[w]);
            } else {
                x0 = f16_lo(la[w]); x1 = f16_hi(la[w]); y0 = f16_lo(lb[w]); y1 = f16_hi(lb[w]);
            }
            const int u0 = 2 * w, u1 = 2 * w + 1;
            oa[w] = pack_f16x2(x0 * cs[u0] - y0 * sn[u0], x1 * cs[u1] - y1 * sn[u1]);
            ob[w] = pack_f16x2(x0 * sn[u0] + y0 * cs[u0], x1 * sn[u1] + y1 * cs[u1]);
        }
        *plo = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        *phi = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
}

template <int D, int NH>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const TcParams p)
{
    using S = TcSmem<D, NH>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* plan = reinterpret_cast<int*>(tmem_slot + 2);  // nR, kE0

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.x;  // heaviest query blocks first
    const int h0 = blockIdx.y * NH, b = blockIdx.z;
    const int kvh = h0 / (p.Hq / p.Hkv);
    const int L = p.L;
    const int i_hi = min(qb * BM + BM - 1, L - 1);
    const int nkb = i_hi / BN + 1;

    // after a bounded wait expired anywhere in the grid (error word set), later
    // CTAs skip their work so a failed launch ends quickly; the host reads and
    // clears the word with jetlong_device_status
    if (*reinterpret_cast<volatile int*>(p.dev_error) != 0) return;
    if (tid == 0) {
        mbar_init(&bars[B_QFULL], 1);
        mbar_init(&bars[B_QREADY0], 4);
        mbar_init(&bars[B_QREADY1], 4);
        mbar_init(&bars[B_QFREE], 1);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(&bars[B_KFULL + s], 1);
            mbar_init(&bars[B_KREADY + s], 4);
            mbar_init(&bars[B_KEMPTY + s], 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(&bars[B_VFULL + s], 1);
            mbar_init(&bars[B_VEMPTY + s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars[B_SFULL + h], 1);
            mbar_init(&bars[B_PFULL + h], 4);
            mbar_init(&bars[B_PVDONE + h], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        // phase R = tiles [0, nR) (classes REM, BAND); phase E = [kE0, nkb) (BAND, LOC)
        int nR = nkb, kE0 = nkb;
        for (int kb = 0; kb < nkb; ++kb) {
            const int cls = tile_class(qb, kb, L, p.w0);
            if (cls != CLS_REM && kE0 == nkb) kE0 = kb;
            if (cls == CLS_LOC) { nR = kb; break; }
        }
        plan[0] = nR;
        plan[1] = kE0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nR = plan[0], kE0 = plan[1];
    const int NE = nR + (nkb - kE0);
    auto kb_of = [&](int e) { return e < nR ? e : kE0 + (e - nR); };

    if (warp < 4) {
        regs_dec<56>();
        if (warp == 0 && lane == 0) {
            // ---------------------------------------------------------- TMA producer
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const int zkv = b * p.Hkv + kvh;
            mbar_arrive_expect_tx(&bars[B_QFULL], NH * S::TILE);
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a)
                    tma_load_3d(smem + h * S::TILE + a * ATOM, &tmQ, a * 64, qb * BM, b * p.Hq + h0 + h,
                                &bars[B_QFULL]);
            int k_issued = 0, v_issued = 0;
            for (int e = 0; e < NE; ++e) {
                const int kb = kb_of(e);
                const int sk = e % NSK, uk = e / NSK;
                if (e >= NSK && !wait_or_abort(&bars[B_KEMPTY + sk], (uk - 1) & 1, abort_flag, p.dev_error, 0x301)) break;
                mbar_arrive_expect_tx(&bars[B_KFULL + sk], S::TILE);
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a)
                    tma_load_3d(smem + S::K0 + sk * S::TILE + a * ATOM, &tmK, a * 64, kb * BN, zkv, &bars[B_KFULL + sk]);
                k_issued = e + 1;
                const int sv = e % NSV, uv = e / NSV;
                if (e >= NSV && !wait_or_abort(&bars[B_VEMPTY + sv], (uv - 1) & 1, abort_flag, p.dev_error, 0x302)) break;
                mbar_arrive_expect_tx(&bars[B_VFULL + sv], S::TILE);
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a)
                    tma_load_3d(smem + S::V0 + sv * S::TILE + a * ATOM, &tmV, a * 64, kb * BN, zkv, &bars[B_VFULL + sv]);
                v_issued = e + 1;
            }
            // drain: the copies this thread issued have landed before the CTA exits
            mbar_wait(&bars[B_QFULL], 0);
            for (int ee = max(0, k_issued - NSK); ee < k_issued; ++ee) mbar_wait(&bars[B_KFULL + ee % NSK], (ee / NSK) & 1);
            for (int ee = max(0, v_issued - NSV); ee < v_issued; ++ee) mbar_wait(&bars[B_VFULL + ee % NSV], (ee / NSV) & 1);
        } else if (warp == 1 && lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            constexpr uint32_t IDESC_QK = idesc_f16(BM, BN, 0);
            constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 1);
            const uint32_t sbase = smem_u32(smem);
            auto qk = [&](int h, int sk) {
                const uint32_t qaddr = sbase + h * S::TILE, kaddr = sbase + S::K0 + sk * S::TILE;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * ATOM + (k & 3) * 32;
                    umma_bf16_ss(tmem + h * 128, sdesc_sw128(qaddr + off, 16, 1024),
                                 sdesc_sw128(kaddr + off, 16, 1024), IDESC_QK, k > 0 ? 1u : 0u);
                }
                umma_commit(&bars[B_SFULL + h]);
            };
            auto pv = [&](int h, int sv, bool first) {
                const uint32_t vaddr = sbase + S::V0 + sv * S::TILE;
#pragma unroll
                for (int k = 0; k < BN / 16; ++k)
                    umma_bf16_ts(tmem + 256 + h * 128, tmem + h * 128 + k * 8,
                                 sdesc_sw128(vaddr + k * 2048, ATOM, 1024), IDESC_PV, (!first || k > 0) ? 1u : 0u);
                umma_commit(&bars[B_PVDONE + h]);
            };
            bool ok = wait_or_abort(&bars[B_QREADY0], 0, abort_flag, p.dev_error, 0x311);
            tc_fence_after();
            for (int e = 0; e < NE && ok; ++e) {
                const int sk = e % NSK, uk = e / NSK, sv = e % NSV, uv = e / NSV;
                if (e == nR && nR > 0) {
                    // Q of phase R is no longer read once every MMA so far completed
                    umma_commit(&bars[B_QFREE]);
                    if (!wait_or_abort(&bars[B_QREADY1], 0, abort_flag, p.dev_error, 0x312)) { ok = false; break; }
                }
                if (!wait_or_abort(&bars[B_KREADY + sk], uk & 1, abort_flag, p.dev_error, 0x313)) { ok = false; break; }
                if (e > 0 && !wait_or_abort(&bars[B_PVDONE + 0], (e - 1) & 1, abort_flag, p.dev_error, 0x314)) { ok = false; break; }
                tc_fence_after();
                qk(0, sk);
                if (NH == 2) {
                    if (e > 0) {
                        // head 1's P.V of the previous tile runs while head 0's softmax works
                        const int pe = e - 1, psv = pe % NSV, puv = pe / NSV;
                        if (!wait_or_abort(&bars[B_PFULL + 1], pe & 1, abort_flag, p.dev_error, 0x315)) { ok = false; break; }
                        if (!wait_or_abort(&bars[B_VFULL + psv], puv & 1, abort_flag, p.dev_error, 0x316)) { ok = false; break; }
                        tc_fence_after();
                        pv(1, psv, pe == 0);
                        umma_commit(&bars[B_VEMPTY + psv]);
                        if (!wait_or_abort(&bars[B_PVDONE + 1], pe & 1, abort_flag, p.dev_error, 0x317)) { ok = false; break; }
                        tc_fence_after();
                    }
                    qk(1, sk);
                }
                umma_commit(&bars[B_KEMPTY + sk]);
                if (!wait_or_abort(&bars[B_PFULL + 0], e & 1, abort_flag, p.dev_error, 0x318)) { ok = false; break; }
                if (!wait_or_abort(&bars[B_VFULL + sv], uv & 1, abort_flag, p.dev_error, 0x319)) { ok = false; break; }
                tc_fence_after();
                pv(0, sv, e == 0);
                if (NH == 1) umma_commit(&bars[B_VEMPTY + sv]);
            }
            if (ok && NH == 2 && NE > 0) {
                const int pe = NE - 1, psv = pe % NSV, puv = pe / NSV;
                if (wait_or_abort(&bars[B_PFULL + 1], pe & 1, abort_flag, p.dev_error, 0x31a) &&
                    wait_or_abort(&bars[B_VFULL + psv], puv & 1, abort_flag, p.dev_error, 0x31b)) {
                    tc_fence_after();
                    pv(1, psv, pe == 0);
                    umma_commit(&bars[B_VEMPTY + psv]);
                }
            }
            // drain: every MMA issued by this thread completed before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else if (warp < 8) {
        regs_dec<88>();
        // -------------------------------------------------------------- rotation
        const int t = tid - 128;
        constexpr int CH = D / 16;
        const int c = t % CH;
        float stc[8], sts[8];  // per-frequency one-position step R(theta_m)
#pragma unroll
        for (int u = 0; u < 8; ++u) rope_cs_fast(1u, p.turns.hi[c * 8 + u], p.turns.lo[c * 8 + u], stc[u], sts[u]);
        const uint32_t i0 = (uint32_t)(qb * BM);
        bool ok = warp_wait(&bars[B_QFULL], 0, abort_flag, p.dev_error, 0x321);
        if (ok) {
            for (int h = 0; h < NH; ++h) {
                if (nR > 0)
                    rotate_tile<D, true>(smem + h * S::TILE, t, p, [&](int r) { return div_g(i0 + r, p); }, stc, sts);
                else
                    rotate_tile<D, true>(smem + h * S::TILE, t, p, [&](int r) { return i0 + r; }, stc, sts);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QREADY0]);
        }
        for (int e = 0; e < NE && ok; ++e) {
            const int kb = kb_of(e);
            const int sk = e % NSK, uk = e / NSK;
            if (e == nR && nR > 0) {
                // phase switch: Q from floor(i/G) to i, by the extra rotation i - floor(i/G)
                if (!warp_wait(&bars[B_QFREE], 0, abort_flag, p.dev_error, 0x322)) { ok = false; break; }
                for (int h = 0; h < NH; ++h)
                    rotate_tile<D, false>(smem + h * S::TILE, t, p,
                                          [&](int r) { return i0 + r - div_g(i0 + r, p); }, stc, sts);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_QREADY1]);
            }
            if (!warp_wait(&bars[B_KFULL + sk], uk & 1, abort_flag, p.dev_error, 0x323)) { ok = false; break; }
            const uint32_t j0 = (uint32_t)(kb * BN);
            if (e < nR)
                rotate_tile<D, true>(smem + S::K0 + sk * S::TILE, t, p, [&](int r) { return div_g(j0 + r, p); }, stc, sts);
            else
                rotate_tile<D, true>(smem + S::K0 + sk * S::TILE, t, p, [&](int r) { return j0 + r; }, stc, sts);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_KREADY + sk]);
        }
    } else {
        regs_inc<184>();
        // -------------------------------------------------------------- softmax (head hh)
        const int hh = (warp - 8) >> 2;
        if (hh < NH) {
            const int r = tid & 127;
            const int i = qb * BM + r;
            const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
            const uint32_t s_col = lane_base + hh * 128, o_col = lane_base + 256 + hh * 128;
            const float sl2 = p.scale_log2;
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int e = 0; e < NE; ++e) {
                const int kb = kb_of(e);
                const bool phase_r = e < nR;
                const int cls = tile_class(qb, kb, L, p.w0);
                if (!warp_wait(&bars[B_SFULL + hh], e & 1, abort_flag, p.dev_error, 0x331)) { ok = false; break; }
                tc_fence_after();
                float x[BN];
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) {
                    uint32_t tt[32];
                    tmem_ld32(s_col + cc * 32, tt);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; ++u) x[cc * 32 + u] = __uint_as_float(tt[u]);
                }
                const int j0 = kb * BN;
                const bool need_mask = (j0 + BN - 1 > qb * BM) || (j0 + BN > L) || cls == CLS_BAND;
                if (need_mask) {
                    const int dw = i - j0 - p.w0;  // pair (i, j0 + u) is local iff u > dw
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
                for (int u = 4; u < BN; u += 4) {
                    m4[0] = fmaxf(m4[0], x[u]);
                    m4[1] = fmaxf(m4[1], x[u + 1]);
                    m4[2] = fmaxf(m4[2], x[u + 2]);
                    m4[3] = fmaxf(m4[3], x[u + 3]);
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
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[BN / 2];
#pragma unroll
                for (int u = 0; u < BN; u += 2) {
                    const float p0 = ex2_approx(fmaf(x[u], sl2, -ms));
                    const float p1 = ex2_approx(fmaf(x[u + 1], sl2, -ms));
                    l4[(u >> 1) & 3] += p0 + p1;
                    pk[u >> 1] = pack_bf16x2(p0, p1);
                }
                l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
                if (e > 0) {
                    // previous P.V of this head finished: O is stable and P's columns are free
                    if (!warp_wait(&bars[B_PVDONE + hh], (e - 1) & 1, abort_flag, p.dev_error, 0x332)) { ok = false; break; }
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, resc)) {
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
                }
#pragma unroll
                for (int cc = 0; cc < BN / 64; ++cc) {
                    uint32_t tt[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u) tt[u] = pk[cc * 32 + u];
                    tmem_st32(s_col + cc * 32, tt);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_PFULL + hh]);
            }
            // epilogue: O / l -> bf16 -> out
            if (ok && NE > 0 && warp_wait(&bars[B_PVDONE + hh], (NE - 1) & 1, abort_flag, p.dev_error, 0x333)) {
                tc_fence_after();
                const float inv = 1.f / l;
                __nv_bfloat16* orow = p.out + (((size_t)b * p.Hq + h0 + hh) * (size_t)L + (size_t)i) * D;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t tt[32];
                    tmem_ld32(o_col + cc * 32, tt);
                    tmem_wait_ld();
                    if (i < L) {
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
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// --------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err)
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static cudaError_t st = cudaSuccess;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        st = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (st == cudaSuccess && q != cudaDriverEntryPointSuccess) st = cudaErrorSymbolNotFound;
        fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    *err = st;
    return fn;
}

// [planes][L rows][d] bf16, box 64 columns x 128 rows x 1 plane, 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* base, int d, int L, int nplanes)
{
    cudaError_t err;
    EncodeTiledFn fn = encode_fn(&err);
    if (!fn) return err == cudaSuccess ? cudaErrorSymbolNotFound : err;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)nplanes};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)BM, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

void make_div_magic(uint32_t G, uint32_t* m, uint32_t* s1, uint32_t* s2)
{
    uint32_t l = 0;
    while ((1ull << l) < G) ++l;  // ceil(log2 G)
    *m = (uint32_t)(((((uint64_t)1 << 32) * (((uint64_t)1 << l) - G)) / G) + 1);
    *s1 = l < 1 ? l : 1;
    *s2 = l > 1 ? l - 1 : 0;
}

template <int D, int NH>
cudaError_t launch_d(const PrefillProblem& pp, cudaStream_t st)
{
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    if ((e = make_map(&tq, pp.q, D, pp.L, pp.B * pp.Hq)) != cudaSuccess) return e;
    if ((e = make_map(&tk, pp.k, D, pp.L, pp.B * pp.Hkv)) != cudaSuccess) return e;
    if ((e = make_map(&tv, pp.v, D, pp.L, pp.B * pp.Hkv)) != cudaSuccess) return e;
    TcParams p{};
    p.B = pp.B; p.Hq = pp.Hq; p.Hkv = pp.Hkv; p.L = pp.L; p.w0 = pp.w0; p.G = pp.G;
    p.nqb = (pp.L + BM - 1) / BM;
    make_div_magic((uint32_t)pp.G, &p.div_m, &p.div_s1, &p.div_s2);
    p.scale_log2 = pp.scale_log2;
    p.turns = pp.turns;
    p.out = reinterpret_cast<__nv_bfloat16*>(pp.out);
    p.dev_error = pp.dev_error;
    auto kern = prefill_tc_kernel<D, NH>;
    constexpr int smem = TcSmem<D, NH>::TOTAL;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    dim3 grid(p.nqb, pp.Hq / NH, pp.B);
    kern<<<grid, NTHREADS, smem, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillProblem& p, cudaStream_t s, int* nlaunch)
{
    const bool pair = ((p.Hq / p.Hkv) % 2) == 0;  // two query heads of one kv head per CTA
    cudaError_t e;
    if (p.d == 64)
        e = pair ? launch_d<64, 2>(p, s) : launch_d<64, 1>(p, s);
    else
        e = pair ? launch_d<128, 2>(p, s) : launch_d<128, 1>(p, s);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

// prefill_tc.cu -- bf16 prefill of dynamic bifocal RoPE attention on the
// sm_100a tensor cores (TMA, tcgen05.mma, TMEM accumulators).
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740):
//   Metodologia 1 -- a pair (i, j) with i - j < w0 uses classic RoPE at i and
//   j; every other pair uses RoPE at f(i), f(j), f(x) = floor(x / G).
//   Metodologia 2 -- rotations are applied on the fly to unrotated inputs and
//   all routed pairs feed one exact softmax.  The pages merge three
//   FlashAttention passes by inclusion-exclusion; here one pass computes the
//   routed logits directly, tile by tile.
//
// One CTA owns 128 query rows of one head.  Key tiles (128 keys) are visited
// in increasing order: remote-only tiles, then the band of tiles that straddles
// i - j = w0, then local-only tiles.  A band tile is fed through the pipeline
// twice (remote rotation, then exact rotation); its two logit tiles are merged
// per element by the softmax threads, so every tile still makes one P and one
// P.V.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: raw Q once (two copies), raw K and V per entry
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM, O += P V
//   warp 2      TMEM allocation / release
//   warps 4-7   rotation: RoPE of Q (exact and aliased copies) and of each K
//               tile, in place in shared memory (one thread per row)
//   warps 8-11  softmax: one thread per query row (= TMEM lane): S from TMEM,
//               band select, causal mask, online softmax in base 2 with lazy
//               rescaling of O, P (bf16) to shared memory, final O / l.
// TMEM (512 columns): S double buffer at columns [0,128) and [128,256),
// O at [256, 256 + d).
//
// Every mbarrier wait is bounded; on expiry the CTA records an error code in
// the library's device error word, stops its loops, drains its own copies and
// MMAs with bounded waits, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "jl_common.cuh"
#include "jl_ptx.cuh"
#include "tc_ptx.cuh"

namespace jl {
namespace {

constexpr int BM = 128, BN = 128, NS = 2, NTHREADS = 384;
constexpr int ATOM = 128 * 128;  // bytes of one 128-row x 64-column bf16 swizzle atom
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

enum { CLS_REM = 0, CLS_LOC = 1, CLS_BAND = 2 };
enum {
    B_QFULL = 0, B_QREADY, B_KFULL, B_KFULL1, B_VFULL, B_VFULL1, B_KREADY, B_KREADY1,
    B_KEMPTY, B_KEMPTY1, B_VEMPTY, B_VEMPTY1, B_SFULL, B_SFULL1, B_SFREE, B_SFREE1,
    B_PFULL, B_PFREE, B_ODONE, B_DRAIN, NBARS
};

struct TcParams {
    int B, Hq, Hkv, L, w0, G, nqb;
    float scale_log2;
    RopeTurns turns;
    __nv_bfloat16* out;
    int* dev_error;
};

template <int D>
struct TcSmem {
    static constexpr int ATOMS = D / 64;
    static constexpr int TILE = BM * D * 2;
    static constexpr int Q0 = 0;
    static constexpr int Q1 = TILE;
    static constexpr int K0 = 2 * TILE;
    static constexpr int V0 = K0 + NS * TILE;
    static constexpr int P = V0 + NS * TILE;
    static constexpr int BAR = P + BM * BN * 2;
    static constexpr int END = BAR + NBARS * 8 + 16;
    static constexpr int TOTAL = END + 1024;  // slack to align the base to 1024
};

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
        if (clock64() - t0 > kWaitCycles) {
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

// Byte offset of 16-byte chunk `ch` (8 bf16 columns, ch < d/8) of row r in a
// 128-row tile stored as [d/64 atoms][128 rows][128 B] with the 128-byte swizzle
// (chunk index XOR row % 8), the layout TMA writes and UMMA K-major reads.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch)
{
    return (uint32_t)((ch >> 3) * ATOM + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

// Rotate row r of a raw bf16 tile in place to position pos, pairs (m, m + d/2);
// the rotated values are written as fp16 (the Q K^T operands are fp16: three
// more mantissa bits than bf16 keep the logits of large keys accurate).
template <int D>
__device__ __forceinline__ void rotate_row(unsigned char* tile, int r, uint32_t pos, const RopeTurns& tw)
{
    constexpr int H = D / 2;
#pragma unroll 2
    for (int c = 0; c < H / 8; ++c) {
        uint4* plo = reinterpret_cast<uint4*>(tile + sw128_off(r, c));
        uint4* phi = reinterpret_cast<uint4*>(tile + sw128_off(r, c + H / 8));
        uint4 a = *plo, bq = *phi;
        uint32_t la[4] = {a.x, a.y, a.z, a.w};
        uint32_t lb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int m0 = c * 8 + 2 * w;
            float c0, s0, c1, s1;
            rope_cs_fast(pos, tw.hi[m0], tw.lo[m0], c0, s0);
            rope_cs_fast(pos, tw.hi[m0 + 1], tw.lo[m0 + 1], c1, s1);
            const float x0 = bf16_lo(la[w]), x1 = bf16_hi(la[w]);
            const float y0 = bf16_lo(lb[w]), y1 = bf16_hi(lb[w]);
            la[w] = pack_f16x2(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1);
            lb[w] = pack_f16x2(x0 * s0 + y0 * c0, x1 * s1 + y1 * c1);
        }
        *plo = make_uint4(la[0], la[1], la[2], la[3]);
        *phi = make_uint4(lb[0], lb[1], lb[2], lb[3]);
    }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const TcParams p)
{
    using S = TcSmem<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.x;  // heaviest query blocks first
    const int h = blockIdx.y, b = blockIdx.z;
    const int kvh = h / (p.Hq / p.Hkv);
    const int L = p.L;
    const int i_hi = min(qb * BM + BM - 1, L - 1);
    const int nkb = i_hi / BN + 1;

    if (tid == 0) {
        mbar_init(&bars[B_QFULL], 1);
        mbar_init(&bars[B_QREADY], 4);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars[B_KFULL + s], 1);
            mbar_init(&bars[B_VFULL + s], 1);
            mbar_init(&bars[B_KREADY + s], 4);
            mbar_init(&bars[B_KEMPTY + s], 1);
            mbar_init(&bars[B_VEMPTY + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[B_SFULL + s], 1);
            mbar_init(&bars[B_SFREE + s], 4);
        }
        mbar_init(&bars[B_PFULL], 4);
        mbar_init(&bars[B_PFREE], 1);
        mbar_init(&bars[B_ODONE], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const int zq = b * p.Hq + h, zkv = b * p.Hkv + kvh;
            mbar_arrive_expect_tx(&bars[B_QFULL], 2 * S::TILE);
#pragma unroll
            for (int a = 0; a < S::ATOMS; ++a) {
                tma_load_3d(smem + S::Q0 + a * ATOM, &tmQ, a * 64, qb * BM, zq, &bars[B_QFULL]);
                tma_load_3d(smem + S::Q1 + a * ATOM, &tmQ, a * 64, qb * BM, zq, &bars[B_QFULL]);
            }
            int e = 0, k_issued = 0, v_issued = 0;
            bool ok = true;
            for (int kb = 0; kb < nkb && ok; ++kb) {
                const int nent = tile_class(qb, kb, L, p.w0) == CLS_BAND ? 2 : 1;
                for (int x = 0; x < nent; ++x, ++e) {
                    const int s = e % NS, u = e / NS;
                    if (e >= NS && !wait_or_abort(&bars[B_KEMPTY + s], (u - 1) & 1, abort_flag, p.dev_error, 0x201)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[B_KFULL + s], S::TILE);
#pragma unroll
                    for (int a = 0; a < S::ATOMS; ++a)
                        tma_load_3d(smem + S::K0 + s * S::TILE + a * ATOM, &tmK, a * 64, kb * BN, zkv,
                                    &bars[B_KFULL + s]);
                    k_issued = e + 1;
                    if (e >= NS && !wait_or_abort(&bars[B_VEMPTY + s], (u - 1) & 1, abort_flag, p.dev_error, 0x202)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[B_VFULL + s], S::TILE);
#pragma unroll
                    for (int a = 0; a < S::ATOMS; ++a)
                        tma_load_3d(smem + S::V0 + s * S::TILE + a * ATOM, &tmV, a * 64, kb * BN, zkv,
                                    &bars[B_VFULL + s]);
                    v_issued = e + 1;
                }
            }
            // drain: the copies this thread issued have landed before the CTA exits
            mbar_wait(&bars[B_QFULL], 0);
            for (int ee = max(0, k_issued - NS); ee < k_issued; ++ee)
                mbar_wait(&bars[B_KFULL + ee % NS], (ee / NS) & 1);
            for (int ee = max(0, v_issued - NS); ee < v_issued; ++ee)
                mbar_wait(&bars[B_VFULL + ee % NS], (ee / NS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_QK = idesc_f16(BM, BN, 0);
            constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 1);
            const uint32_t sbase = smem_u32(smem);
            bool ok = wait_or_abort(&bars[B_QREADY], 0, abort_flag, p.dev_error, 0x211);
            tc_fence_after();
            int e = 0, pend = -1, npv = 0;
            auto issue_pv = [&](int pe) -> bool {
                const int ps = pe % NS, pu = pe / NS;
                if (!wait_or_abort(&bars[B_PFULL], npv & 1, abort_flag, p.dev_error, 0x212)) return false;
                if (!wait_or_abort(&bars[B_VFULL + ps], pu & 1, abort_flag, p.dev_error, 0x213)) return false;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < BN / 16; ++k) {
                    const uint64_t ad = sdesc_sw128(sbase + S::P + (k >> 2) * ATOM + (k & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sbase + S::V0 + ps * S::TILE + k * 2048, ATOM, 1024);
                    umma_bf16_ss(tmem + 256, ad, bd, IDESC_PV, (npv > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&bars[B_PFREE]);
                umma_commit(&bars[B_VEMPTY + ps]);
                ++npv;
                return true;
            };
            for (int kb = 0; kb < nkb && ok; ++kb) {
                const int cls = tile_class(qb, kb, L, p.w0);
                const int nent = cls == CLS_BAND ? 2 : 1;
                for (int x = 0; x < nent && ok; ++x, ++e) {
                    const int s = e % NS, u = e / NS, sb = e & 1, ub = e >> 1;
                    const bool exact = (cls == CLS_LOC) || (cls == CLS_BAND && x == 1);
                    const bool band_first = (cls == CLS_BAND && x == 0);
                    if (!wait_or_abort(&bars[B_KREADY + s], u & 1, abort_flag, p.dev_error, 0x214)) { ok = false; break; }
                    if (e >= 2 && !wait_or_abort(&bars[B_SFREE + sb], (ub - 1) & 1, abort_flag, p.dev_error, 0x215)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t qaddr = sbase + (exact ? S::Q0 : S::Q1);
                    const uint32_t kaddr = sbase + S::K0 + s * S::TILE;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k >> 2) * ATOM + (k & 3) * 32;
                        umma_bf16_ss(tmem + sb * 128, sdesc_sw128(qaddr + off, 16, 1024),
                                     sdesc_sw128(kaddr + off, 16, 1024), IDESC_QK, k > 0 ? 1u : 0u);
                    }
                    umma_commit(&bars[B_SFULL + sb]);
                    umma_commit(&bars[B_KEMPTY + s]);
                    if (band_first) {
                        // this entry's V copy is unused: release its slot once it has landed
                        if (!wait_or_abort(&bars[B_VFULL + s], u & 1, abort_flag, p.dev_error, 0x216)) { ok = false; break; }
                        umma_commit(&bars[B_VEMPTY + s]);
                    }
                    if (pend >= 0) {
                        if (!issue_pv(pend)) { ok = false; break; }
                        pend = -1;
                    }
                    if (!band_first) pend = e;
                }
            }
            if (ok && pend >= 0) ok = issue_pv(pend);
            umma_commit(&bars[B_ODONE]);
            // drain: every MMA issued by this thread completed before TMEM is released
            umma_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ rotation warps
        const int r = tid - 128;
        bool ok = warp_wait(&bars[B_QFULL], 0, abort_flag, p.dev_error, 0x221);
        if (ok) {
            const uint32_t i = (uint32_t)(qb * BM + r);
            rotate_row<D>(smem + S::Q0, r, i, p.turns);
            rotate_row<D>(smem + S::Q1, r, i / (uint32_t)p.G, p.turns);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QREADY]);
        }
        int e = 0;
        for (int kb = 0; kb < nkb && ok; ++kb) {
            const int cls = tile_class(qb, kb, L, p.w0);
            const int nent = cls == CLS_BAND ? 2 : 1;
            for (int x = 0; x < nent; ++x, ++e) {
                const int s = e % NS, u = e / NS;
                const bool exact = (cls == CLS_LOC) || (cls == CLS_BAND && x == 1);
                if (!warp_wait(&bars[B_KFULL + s], u & 1, abort_flag, p.dev_error, 0x222)) { ok = false; break; }
                const uint32_t j = (uint32_t)(kb * BN + r);
                rotate_row<D>(smem + S::K0 + s * S::TILE, r, exact ? j : j / (uint32_t)p.G, p.turns);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_KREADY + s]);
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ softmax warps
        const int r = tid - 256;
        const int i = qb * BM + r;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        float m_used = -INFINITY, l = 0.f;
        int e = 0, nt = 0;
        bool ok = true;
        for (int kb = 0; kb < nkb && ok; ++kb) {
            const int cls = tile_class(qb, kb, L, p.w0);
            const int eA = e, sbA = eA & 1;
            const int eB = e + 1, sbB = eB & 1;
            if (!warp_wait(&bars[B_SFULL + sbA], (eA >> 1) & 1, abort_flag, p.dev_error, 0x231)) { ok = false; break; }
            if (cls == CLS_BAND &&
                !warp_wait(&bars[B_SFULL + sbB], (eB >> 1) & 1, abort_flag, p.dev_error, 0x232)) { ok = false; break; }
            tc_fence_after();
            float x[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t t[32];
                tmem_ld32(lane_addr + sbA * 128 + c * 32, t);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) x[c * 32 + u] = __uint_as_float(t[u]);
            }
            if (cls == CLS_BAND) {
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t t[32];
                    tmem_ld32(lane_addr + sbB * 128 + c * 32, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int j = kb * BN + c * 32 + u;
                        if (i - j < p.w0) x[c * 32 + u] = __uint_as_float(t[u]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_SFREE + sbA]);
                if (cls == CLS_BAND) mbar_arrive(&bars[B_SFREE + sbB]);
            }
            // scale to base-2 units, causal / length mask, row max
            const bool need_mask = (kb * BN + BN - 1 > qb * BM) || (kb * BN + BN > L);
            float mx = -INFINITY;
#pragma unroll
            for (int u = 0; u < BN; ++u) {
                float v = x[u] * p.scale_log2;
                if (need_mask) {
                    const int j = kb * BN + u;
                    if (j > i || j >= L) v = -INFINITY;
                }
                x[u] = v;
                mx = fmaxf(mx, v);
            }
            const float m_new = fmaxf(m_used, mx);
            const bool resc = m_new > m_used + kRescaleThreshold;
            float alpha = 1.f;
            if (resc) {
                alpha = exp2f(m_used - m_new);
                m_used = m_new;
                l *= alpha;
            }
            float rs = 0.f;
#pragma unroll
            for (int u = 0; u < BN; ++u) {
                const float pe = exp2f(x[u] - m_used);
                x[u] = pe;
                rs += pe;
            }
            l += rs;
            if (nt > 0) {
                // previous P.V finished: O is stable and the P buffer is free
                if (!warp_wait(&bars[B_PFREE], (nt - 1) & 1, abort_flag, p.dev_error, 0x233)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t t[32];
                        tmem_ld32(lane_addr + 256 + c * 32, t);
                        tmem_wait_ld();
#pragma unroll
                        for (int u = 0; u < 32; ++u) t[u] = __float_as_uint(__uint_as_float(t[u]) * alpha);
                        tmem_st32(lane_addr + 256 + c * 32, t);
                    }
                    tmem_wait_st();
                }
            }
            unsigned char* prow = smem + S::P;
#pragma unroll
            for (int ch = 0; ch < BN / 8; ++ch) {
                uint4 v;
                v.x = pack_bf16x2(x[ch * 8 + 0], x[ch * 8 + 1]);
                v.y = pack_bf16x2(x[ch * 8 + 2], x[ch * 8 + 3]);
                v.z = pack_bf16x2(x[ch * 8 + 4], x[ch * 8 + 5]);
                v.w = pack_bf16x2(x[ch * 8 + 6], x[ch * 8 + 7]);
                *reinterpret_cast<uint4*>(prow + sw128_off(r, ch)) = v;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PFULL]);
            ++nt;
            e += (cls == CLS_BAND) ? 2 : 1;
        }
        // epilogue: O / l -> bf16 -> out
        if (ok && warp_wait(&bars[B_ODONE], 0, abort_flag, p.dev_error, 0x234)) {
            tc_fence_after();
            const float inv = 1.f / l;
            __nv_bfloat16* orow = p.out + (((size_t)b * p.Hq + h) * (size_t)L + (size_t)i) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t t[32];
                tmem_ld32(lane_addr + 256 + c * 32, t);
                tmem_wait_ld();
                if (i < L) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(t[q * 8 + 0]) * inv, __uint_as_float(t[q * 8 + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(t[q * 8 + 2]) * inv, __uint_as_float(t[q * 8 + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(t[q * 8 + 4]) * inv, __uint_as_float(t[q * 8 + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(t[q * 8 + 6]) * inv, __uint_as_float(t[q * 8 + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = v;
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

// [rows = L, planes = nplanes] x d bf16, box 64 columns x 128 rows x 1 plane, 128-byte swizzle.
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

template <int D>
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
    p.scale_log2 = pp.scale_log2;
    p.turns = pp.turns;
    p.out = reinterpret_cast<__nv_bfloat16*>(pp.out);
    p.dev_error = pp.dev_error;
    auto kern = prefill_tc_kernel<D>;
    constexpr int smem = TcSmem<D>::TOTAL;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    dim3 grid(p.nqb, pp.Hq, pp.B);
    kern<<<grid, NTHREADS, smem, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillProblem& p, cudaStream_t s, int* nlaunch)
{
    cudaError_t e = p.d == 64 ? launch_d<64>(p, s) : launch_d<128>(p, s);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

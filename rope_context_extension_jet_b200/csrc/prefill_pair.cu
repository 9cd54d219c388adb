// prefill_pair.cu -- bf16 prefill of dynamic bifocal RoPE attention (d = 128)
// on CTA pairs: every tensor-core MMA spans the two SMs of a cluster pair
// (tcgen05 cta_group::2, M = 256).
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740), Metodologia 1-2: local pairs
// (i - j < w0) are rotated at (i, j), remote pairs at (floor(i/G), floor(j/G)),
// one softmax for both.  The keys come rotated both ways, once per call
// (rope_keys.cu: fp16 copies at j and at floor(j/G)); Q is rotated here.
//
// Work unit of a pair: one block of 128 query rows of the four query heads
// that share a kv head.  CTA r (r = 0, 1) holds heads 2r and 2r + 1 of the four:
// their Q tiles, S and O in its own TMEM (lanes = query rows).  A K tile (128
// keys) is split by keys: CTA r loads keys [64r, 64r + 64) of the copy the
// tile's phase uses; a V tile is split by columns: CTA r loads
// V[:, 64r, 64r + 64).  One MMA
//   S_h = Q_h K^T : A = Q_h of both CTAs (M = 256), B = both K halves (N = 128)
//   O_h += P_h V  : A = P_h in both TMEMs, B = both V halves (N = d)
// so each SM stages half of every K/V tile, and reads half of the B operand
// from its shared memory, while the MMA rate per SM is unchanged.
// The phases, masks and softmax are those of the one-CTA kernel
// (prefill_tc.cu): phase R (remote and band tiles, aliased positions), then
// phase E (band and local tiles, exact positions), Q re-rotated in between.
//
// Roles (512 threads per CTA; registers rebalanced with setmaxnreg):
//   warp 0      TMA producer (both CTAs): own Q tiles, own K (rotated copy of
//               the tile's phase) and V halves
//   warp 1      MMA issuer (CTA 0 only; the whole warp runs the loop, one
//               elected lane issues each instruction), cta_group::2
//   warp 2      TMEM allocation / release (cta_group::2, both CTAs)
//   warp 3      CTA 1: tells CTA 0 when its V half landed
//   warps 4-7   rotation of own Q tiles; pass each landed K half on to CTA 0
//   warps 8-15  softmax, heads 2r (8-11) and 2r + 1 (12-15)
// Synchronisation: CTA 0's MMA thread waits on barriers in CTA 0 that both CTAs
// arrive on (Q rotated, K halves landed, P written, V halves landed); its commits arrive
// on the barriers at the same offset in both CTAs (S ready, P.V done, buffers
// free).  Every wait is bounded; on expiry a CTA records an error code, stops,
// and both CTAs meet at the closing cluster barrier before TMEM is released.
#include "prefill_tc_common.cuh"

namespace jl {
namespace tc {
namespace {

constexpr int D = 128;
constexpr int NS = 5;           // ring depth of the K and V halves
constexpr int KROWS = BN / 2;   // keys of a K tile held by one CTA
constexpr int NTHREADS = 512;
// Registers per thread after setmaxnreg: producer / MMA warpgroup, rotation
// warpgroup, each of the two softmax warpgroups.  setmaxnreg.inc takes its
// registers from those the block was launched with (NTHREADS x 128), so the
// split must not ask for more, or the increase would wait for ever.
constexpr int kRegsProducer = 56, kRegsRotation = 72, kRegsSoftmax = 192;
static_assert((kRegsProducer + kRegsRotation + 2 * kRegsSoftmax) * 128 <= NTHREADS * 128,
              "register split exceeds the launch's registers");
static_assert(kRegsProducer % 8 == 0 && kRegsRotation % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");

enum {
    P_QFULL = 0, P_QREADY0, P_QREADY1, P_QFREE,
    P_KFULL, P_KREADY = P_KFULL + NS, P_KEMPTY = P_KREADY + NS,
    P_VFULL = P_KEMPTY + NS, P_VPEER = P_VFULL + NS, P_VEMPTY = P_VPEER + NS,
    P_SFULL = P_VEMPTY + NS, P_PFULL = P_SFULL + 2, P_PVDONE = P_PFULL + 4,
    P_DRAIN = P_PVDONE + 2, P_NBARS
};

struct PairSmem {
    static constexpr int QTILE = BM * D * 2;      // 128 rows x 128 d: 2 atoms of 16 KB
    static constexpr int KATOM = KROWS * 128;     // 64 rows x 64 columns
    static constexpr int KTILE = KROWS * D * 2;   // 64 keys x 128 d: 2 atoms of 8 KB
    static constexpr int VTILE = BN * 64 * 2;     // 128 keys x 64 columns: 1 atom
    static constexpr int K0 = 2 * QTILE;
    static constexpr int V0 = K0 + NS * KTILE;
    static constexpr int BAR = V0 + NS * VTILE;
    static constexpr int END = BAR + P_NBARS * 8 + 32;
    static constexpr int TOTAL = END + 1024;      // slack to align the base to 1024
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKl,
                        const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmV,
                        const TcParams p)
{
    using S = PairSmem;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* skip_word = reinterpret_cast<int*>(tmem_slot + 2);
    TilePlan* plan = reinterpret_cast<TilePlan*>(tmem_slot + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    // the pair's sequence and query block (heaviest query blocks first); a
    // unit past the end of a shorter sequence of a variable-length batch has no
    // work (both CTAs of the pair see the same unit)
    SeqView sv;
    if (!seq_view(p, (int)(blockIdx.x >> 1), (int)blockIdx.z, sv)) return;
    const int qb = sv.qb, b = sv.b;
    const int hq4 = blockIdx.y * 4;                      // first of the pair's four query heads
    const int h0 = hq4 + 2 * (int)rank;                  // this CTA's two heads
    const int kvh = hq4 / (p.Hq / p.Hkv);
    // barriers of CTA 0, as cluster addresses (both CTAs arrive on them)
    const uint32_t lbar = mapa_shared(smem_u32(bars), 0);
    auto lead = [&](int idx) { return lbar + 8u * (uint32_t)idx; };

    if (tid == 0) {
        mbar_init(&bars[P_QFULL], 1);
        mbar_init(&bars[P_QREADY0], 8);
        mbar_init(&bars[P_QREADY1], 8);
        mbar_init(&bars[P_QFREE], 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars[P_KFULL + s], 1);
            mbar_init(&bars[P_KREADY + s], 8);
            mbar_init(&bars[P_KEMPTY + s], 1);
            mbar_init(&bars[P_VFULL + s], 1);
            mbar_init(&bars[P_VPEER + s], 1);
            mbar_init(&bars[P_VEMPTY + s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&bars[P_SFULL + h], 1);
            mbar_init(&bars[P_PFULL + 2 * h], 8);      // first half of P_h
            mbar_init(&bars[P_PFULL + 2 * h + 1], 8);  // second half
            mbar_init(&bars[P_PVDONE + h], 1);
        }
        mbar_init(&bars[P_DRAIN], 1);
        *abort_flag = 0;
        *plan = plan_tiles(p.P + qb * BM, sv.L, sv.w0);
        if (p.window_rot >= 0) plan->nR = 0;  // windowed pass: the local tiles only
        // after a bounded wait expired anywhere in the grid (error word set),
        // later pairs skip their work; CTA 0 decides for both
        if (leader) *skip_word = *reinterpret_cast<volatile int*>(p.dev_error) != 0;
        fence_mbar_init();
    }
    __syncthreads();
    cluster_sync();  // barriers of both CTAs initialised, CTA 0's decision visible
    const bool skip = ld_shared_cluster_u32(mapa_shared(smem_u32(skip_word), 0)) != 0;
    if (!skip && warp == 2) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
        tc_fence_before();
    }
    __syncthreads();
    cluster_sync();  // no CTA reads the other's shared memory before this point is passed
    if (skip) return;
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const TilePlan tp = *plan;
    const int nR = tp.nR, NE = tp.count();

    if (warp < 4) {
        regs_dec<kRegsProducer>();
        if (warp == 0 && lane == 0) {
            // ---------------------------------------------------------- TMA producer
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmKl);
            tma_prefetch_desc(&tmKr);
            tma_prefetch_desc(&tmV);
            const int zkv = b * p.Hkv + kvh;
            mbar_arrive_expect_tx(&bars[P_QFULL], 2 * S::QTILE);
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int a = 0; a < 2; ++a)
                    tma_load_3d(smem + h * S::QTILE + a * ATOM, &tmQ, a * 64, qb * BM, b * p.Hq + h0 + h,
                                &bars[P_QFULL]);
            int k_issued = 0, v_issued = 0;
            for (int e = 0; e < NE; ++e) {
                const int kb = tp.kb(e);
                const int s = e % NS, u = e / NS;
                if (e >= NS && !wait_or_abort<true>(&bars[P_KEMPTY + s], (u - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x401)) break;
                mbar_arrive_expect_tx(&bars[P_KFULL + s], S::KTILE);
                // keys rotated to floor(j / G) in phase R (and in a windowed
                // pass at the aliased positions), to j in phase E
                const CUtensorMap* km = (e < nR || p.window_rot == 1) ? &tmKr : &tmKl;
#pragma unroll
                for (int a = 0; a < 2; ++a)
                    tma_load_3d(smem + S::K0 + s * S::KTILE + a * S::KATOM, km, a * 64, kb * BN + (int)rank * KROWS,
                                zkv, &bars[P_KFULL + s]);
                k_issued = e + 1;
                if (e >= NS && !wait_or_abort<true>(&bars[P_VEMPTY + s], (u - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x402)) break;
                mbar_arrive_expect_tx(&bars[P_VFULL + s], S::VTILE);
                tma_load_3d(smem + S::V0 + s * S::VTILE, &tmV, (int)rank * 64, kb * BN, zkv, &bars[P_VFULL + s]);
                v_issued = e + 1;
            }
            // drain: the copies this thread issued have landed before the CTA exits
            mbar_wait(&bars[P_QFULL], 0);
            for (int ee = max(0, k_issued - NS); ee < k_issued; ++ee) mbar_wait(&bars[P_KFULL + ee % NS], (ee / NS) & 1);
            for (int ee = max(0, v_issued - NS); ee < v_issued; ++ee) mbar_wait(&bars[P_VFULL + ee % NS], (ee / NS) & 1);
        } else if (warp == 1 && leader) {
            // ---------------------------------------------------------- MMA issuer
            // Every value below is warp-uniform (the TMEM base is broadcast from
            // lane 0), every wait is warp-collective, and each MMA / commit is
            // issued by one elected lane.
            constexpr uint32_t IDESC_QK = idesc_f16(2 * BM, BN, 0);
            constexpr uint32_t IDESC_PV = idesc_bf16(2 * BM, D, 1);
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            const uint32_t sbase = smem_u32(smem);
            // (the step offsets inside umma_pair_qk_k128 / _pv_k128 are those of
            // these tiles: Q atoms 16 KB apart, K-half atoms 8 KB apart, V slices 2 KB)
            static_assert(ATOM == 1024 * 16 && S::KATOM == 512 * 16 && BN / 16 == 8 && D / 16 == 8,
                          "tile layout of the grouped MMA issue");
            auto qk = [&](int h, int s) {
                const uint32_t qaddr = sbase + h * S::QTILE, kaddr = sbase + S::K0 + s * S::KTILE;
                umma_pair_qk_k128(tm + h * 128, sdesc_sw128(qaddr, 16, 1024), sdesc_sw128(kaddr, 16, 1024), IDESC_QK, 0u);
                umma_commit_pair_both_elect(&bars[P_SFULL + h]);
            };
            // P_h V of tile pe, issued half by half as the softmax publishes the
            // halves of P_h (V's halves landed in both CTAs: checked for head 0)
            auto pv = [&](int h, int pe) {
                const int s = pe % NS, u = pe / NS;
                if (h == 0 && !(warp_wait(&bars[P_VFULL + s], u & 1, abort_flag, p.dev_error, p.wait_cycles, 0x413) &&
                                warp_wait<true>(&bars[P_VPEER + s], u & 1, abort_flag, p.dev_error, p.wait_cycles, 0x414)))
                    return false;
                const uint64_t vdesc = sdesc_sw128(sbase + S::V0 + s * S::VTILE, S::VTILE, 1024);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!warp_wait<true>(&bars[P_PFULL + 2 * h + half], pe & 1, abort_flag, p.dev_error, p.wait_cycles,
                                         0x411 + h))
                        return false;
                    tc_fence_after();
                    umma_pair_pv_k64(tm + 256 + h * 128, tm + h * 128 + 32 * half, vdesc + 512 * half, IDESC_PV,
                                     (pe == 0 && half == 0) ? 0u : 1u);
                }
                umma_commit_pair_both_elect(&bars[P_PVDONE + h]);
                return true;
            };
            // Issue order per tile e: P_0 V (tile e-1), Q_0 K^T (tile e), P_1 V
            // (tile e-1), Q_1 K^T (tile e).  S_h(e) overwrites P_h(e-1) in TMEM;
            // the P.V reading it was issued earlier by this warp and the tensor
            // pipe runs one issuer's MMAs in issue order.
            bool ok = warp_wait<true>(&bars[P_QREADY0], 0, abort_flag, p.dev_error, p.wait_cycles, 0x415);
            tc_fence_after();
            for (int e = 0; e < NE && ok; ++e) {
                const int s = e % NS, u = e / NS, pe = e - 1, ps = (e + NS - 1) % NS;
                if (e > 0 && !pv(0, pe)) { ok = false; break; }
                if (e == nR && nR > 0) {
                    // Q of phase R is no longer read once every MMA so far completed
                    umma_commit_pair_both_elect(&bars[P_QFREE]);
                    if (!warp_wait<true>(&bars[P_QREADY1], 0, abort_flag, p.dev_error, p.wait_cycles, 0x416)) { ok = false; break; }
                }
                if (!warp_wait<true>(&bars[P_KREADY + s], u & 1, abort_flag, p.dev_error, p.wait_cycles, 0x417)) { ok = false; break; }
                tc_fence_after();
                qk(0, s);
                if (e > 0) {
                    if (!pv(1, pe)) { ok = false; break; }
                    umma_commit_pair_both_elect(&bars[P_VEMPTY + ps]);
                }
                qk(1, s);
                umma_commit_pair_both_elect(&bars[P_KEMPTY + s]);
            }
            if (ok && NE > 0) {
                const int pe = NE - 1, ps = pe % NS;
                if (pv(0, pe) && pv(1, pe)) umma_commit_pair_both_elect(&bars[P_VEMPTY + ps]);
            }
            // drain: every MMA issued by this warp completed before the pair
            // meets at the closing cluster barrier
            umma_commit_pair_local_elect(&bars[P_DRAIN]);
            mbar_wait(&bars[P_DRAIN], 0);
        } else if (warp == 3 && lane == 0 && !leader) {
            // ---------------------------------------------------------- V relay (CTA 1)
            for (int e = 0; e < NE; ++e) {
                const int s = e % NS, u = e / NS;
                if (!wait_or_abort(&bars[P_VFULL + s], u & 1, abort_flag, p.dev_error, p.wait_cycles, 0x421)) break;
                mbar_arrive_cluster(lead(P_VPEER + s));
            }
        }
    } else if (warp < 8) {
        regs_dec<kRegsRotation>();
        // -------------------------------------------------------------- rotation
        const int t = tid - 128;
        float2 stc[4], sts[4];  // per-frequency one-position step R(theta_m)
        rope_steps<D>(t, p, stc, sts);
        // operand scales of this call (powers of two, see range_exp)
        const float lq = pow2i(range_exp(ld_range(p.range)));
        const uint32_t i0 = (uint32_t)(p.P + qb * BM);
        bool ok = warp_wait(&bars[P_QFULL], 0, abort_flag, p.dev_error, p.wait_cycles, 0x431);
        if (ok) {
            for (int h = 0; h < 2; ++h) {
                if (nR > 0 || p.window_rot == 1)
                    rotate_tile<D, BM, true, true>(smem + h * S::QTILE, t, p, [&](int r) { return div_g(i0 + r, sv); }, stc,
                                             sts, lq);
                else
                    rotate_tile<D, BM, true, true>(smem + h * S::QTILE, t, p, [&](int r) { return i0 + r; }, stc, sts, lq);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead(P_QREADY0));
        }
        for (int e = 0; e < NE && ok; ++e) {
            const int s = e % NS, u = e / NS;
            if (e == nR && nR > 0) {
                // phase switch: Q from floor(i/G) to i, by the extra rotation i - floor(i/G)
                if (!warp_wait<true>(&bars[P_QFREE], 0, abort_flag, p.dev_error, p.wait_cycles, 0x432)) { ok = false; break; }
                for (int h = 0; h < 2; ++h)
                    rotate_tile<D, BM, false, true>(smem + h * S::QTILE, t, p,
                                              [&](int r) { return i0 + r - div_g(i0 + r, sv); }, stc, sts, 1.f);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(lead(P_QREADY1));
            }
            // the K half-tile arrives rotated (rope_keys.cu): pass its arrival on
            // to the leader's MMA warp
            if (!warp_wait(&bars[P_KFULL + s], u & 1, abort_flag, p.dev_error, p.wait_cycles, 0x433)) { ok = false; break; }
            __syncwarp();
            // (test hook: the first key tile is never released, so the MMA warp's
            // bounded wait on it expires)
            if (lane == 0 && !(p.inject == kInjectPrefillKeyTile && e == 0)) mbar_arrive_cluster(lead(P_KREADY + s));
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // -------------------------------------------------------------- softmax (head hh)
        const int hh = (warp - 8) >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const uint32_t pfull = lead(P_PFULL + 2 * hh);
        softmax_role<D, true>(p, sv, tp, h0 + hh, tid & 127, lane_base + hh * 128, lane_base + 256 + hh * 128,
                              &bars[P_SFULL + hh], &bars[P_PVDONE + hh],
                              [pfull](int half) { mbar_arrive_cluster(pfull + 8u * (uint32_t)half); }, abort_flag);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the pair's MMAs, copies and remote arrivals are over in both CTAs
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_prefill_pair(const PrefillProblem& pp, cudaStream_t st)
{
    CUtensorMap tq, tkl, tkr, tv;
    cudaError_t e;
    if ((e = make_map(&tq, pp.q, D, pp.C, pp.Cst, pp.B * pp.Hq, BM)) != cudaSuccess) return e;
    if ((e = make_map(&tkl, pp.krot_l, D, pp.L, pp.L, pp.B * pp.Hkv, KROWS, true)) != cudaSuccess) return e;
    if ((e = make_map(&tkr, pp.krot_r, D, pp.L, pp.L, pp.B * pp.Hkv, KROWS, true)) != cudaSuccess) return e;
    if ((e = make_map(&tv, pp.v, D, pp.L, pp.Lcap, pp.B * pp.Hkv, BN)) != cudaSuccess) return e;
    const TcParams p = make_params(pp);
    constexpr int smem = PairSmem::TOTAL;
    if ((e = cudaFuncSetAttribute(prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
        return e;
    // variable-length: x over (query-block level, sequence), one z
    dim3 grid(p.vl_n ? 2 * p.vl_nqb_max * p.vl_n : 2 * p.nqb, pp.Hq / 4, p.vl_n ? 1 : pp.B);
    prefill_pair_kernel<<<grid, NTHREADS, smem, st>>>(tq, tkl, tkr, tv, p);
    return cudaGetLastError();
}

}  // namespace tc
}  // namespace jl

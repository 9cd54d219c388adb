// prefill_tc.cu -- bf16 prefill of dynamic bifocal RoPE attention on the
// sm_100a tensor cores (TMA, tcgen05.mma, TMEM accumulators).
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740):
//   Metodologia 1 -- a pair (i, j) with i - j < w0 uses classic RoPE at i and
//   j; every other pair uses RoPE at f(i), f(j), f(x) = floor(x / G).
//   Metodologia 2 -- rotations compose additively, and all routed pairs feed
//   one exact softmax.
//   The pages merge three FlashAttention passes by inclusion-exclusion; here
//   one pass computes the routed logits directly.
//
// Work unit: 128 query rows of NH = 2 query heads that share a kv head
// (grouped-query attention), so every K tile is loaded once for both heads.
// The keys come rotated once per call (rope_keys.cu: fp16 copies at j and at
// floor(j/G)); each tile is loaded from the copy of its phase.  Each CTA makes
// two passes over its key tiles (128 keys):
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
//   warp 0        TMA producer (raw Q once; rotated K and V per tile)
//   warp 1        MMA issuer (the whole warp; one elected lane issues each
//                 group of MMAs): S_h = Q_h K^T (fp16 operands) into TMEM;
//                 O_h += P_h V with P_h read from TMEM (bf16)
//   warp 2        TMEM allocation / release
//   warps 4-7     rotation: RoPE of Q in shared memory, angles advanced row by
//                 row with a per-frequency rotation step; then the arrival of
//                 each K tile is passed on to the MMA warp
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
#include <algorithm>

#include "prefill_tc_common.cuh"

namespace jl {
namespace tc {
namespace {

constexpr int NSK = 2, NSV = 2, NTHREADS = 512;
// Registers per thread after setmaxnreg: producer / MMA warpgroup, rotation
// warpgroup, each of the two softmax warpgroups.  setmaxnreg.inc takes its
// registers from those the block was launched with (NTHREADS x 128), so the
// split must not ask for more, or the increase would wait for ever.
constexpr int kRegsProducer = 56, kRegsRotation = 88, kRegsSoftmax = 184;
static_assert((kRegsProducer + kRegsRotation + 2 * kRegsSoftmax) * 128 <= NTHREADS * 128,
              "register split exceeds the launch's registers");
static_assert(kRegsProducer % 8 == 0 && kRegsRotation % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");

enum {
    B_QFULL = 0, B_QREADY0, B_QREADY1, B_QFREE,
    B_KFULL, B_KREADY = B_KFULL + NSK, B_KEMPTY = B_KREADY + NSK,
    B_VFULL = B_KEMPTY + NSK, B_VEMPTY = B_VFULL + NSV,
    B_SFULL = B_VEMPTY + NSV, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 4,
    B_DRAIN = B_PVDONE + 2, NBARS
};

template <int D, int NH>
struct TcSmem {
    static constexpr int ATOMS = D / 64;
    static constexpr int TILE = BM * D * 2;
    static constexpr int K0 = NH * TILE;
    static constexpr int V0 = K0 + NSK * TILE;
    static constexpr int BAR = V0 + NSV * TILE;
    static constexpr int END = BAR + NBARS * 8 + 32;  // + TMEM slot, abort flag, tile plan
    static constexpr int TOTAL = END + 1024;  // slack to align the base to 1024
};

template <int D, int NH>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKl,
                      const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmV,
                      const TcParams p)
{
    using S = TcSmem<D, NH>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    TilePlan* plan = reinterpret_cast<TilePlan*>(tmem_slot + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the CTA's sequence and query block (heaviest query blocks first); a unit
    // past the end of a shorter sequence of a variable-length batch has no work
    SeqView sv;
    if (!seq_view(p, (int)blockIdx.x, (int)blockIdx.z, sv)) return;
    const int qb = sv.qb, b = sv.b;
    const int h0 = blockIdx.y * NH;
    const int kvh = h0 / (p.Hq / p.Hkv);

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
            mbar_init(&bars[B_PFULL + 2 * h], 4);      // first half of P_h
            mbar_init(&bars[B_PFULL + 2 * h + 1], 4);  // second half
            mbar_init(&bars[B_PVDONE + h], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        *plan = plan_tiles(p.P + qb * BM, sv.L, sv.w0);
        if (p.window_rot >= 0) plan->nR = 0;  // windowed pass: the local tiles only
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
            mbar_arrive_expect_tx(&bars[B_QFULL], NH * S::TILE);
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a)
                    tma_load_3d(smem + h * S::TILE + a * ATOM, &tmQ, a * 64, qb * BM, b * p.Hq + h0 + h,
                                &bars[B_QFULL]);
            int k_issued = 0, v_issued = 0;
            for (int e = 0; e < NE; ++e) {
                const int kb = tp.kb(e);
                const int sk = e % NSK, uk = e / NSK;
                if (e >= NSK && !wait_or_abort(&bars[B_KEMPTY + sk], (uk - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x301)) break;
                mbar_arrive_expect_tx(&bars[B_KFULL + sk], S::TILE);
                // keys rotated to floor(j / G) in phase R (and in a windowed
                // pass at the aliased positions), to j in phase E
                const CUtensorMap* km = (e < nR || p.window_rot == 1) ? &tmKr : &tmKl;
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a)
                    tma_load_3d(smem + S::K0 + sk * S::TILE + a * ATOM, km, a * 64, kb * BN, zkv, &bars[B_KFULL + sk]);
                k_issued = e + 1;
                const int sv = e % NSV, uv = e / NSV;
                if (e >= NSV && !wait_or_abort(&bars[B_VEMPTY + sv], (uv - 1) & 1, abort_flag, p.dev_error, p.wait_cycles, 0x302)) break;
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
        } else if (warp == 1) {
            // ---------------------------------------------------------- MMA issuer
            // The whole warp runs the loop with warp-uniform values and waits; one
            // elected lane issues each group of MMAs and each commit.
            constexpr uint32_t IDESC_QK = idesc_f16(BM, BN, 0);
            constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, 1);
            static_assert(ATOM == 1024 * 16 && BN / 16 == 8 && (D == 64 || D == 128),
                          "tile layout of the grouped MMA issue");
            const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
            const uint32_t sbase = smem_u32(smem);
            auto qk = [&](int h, int sk) {
                const uint64_t a = sdesc_sw128(sbase + h * S::TILE, 16, 1024);
                const uint64_t bk = sdesc_sw128(sbase + S::K0 + sk * S::TILE, 16, 1024);
                if (D == 128)
                    umma_qk_k128(tm + h * 128, a, bk, IDESC_QK);
                else
                    umma_qk_k64(tm + h * 128, a, bk, IDESC_QK);
                umma_commit_elect(&bars[B_SFULL + h]);
            };
            // P_h V of tile pe (V in stage sv), issued half by half as the
            // softmax publishes the halves of P_h
            auto pv = [&](int h, int pe, int sv, int code) {
                const uint64_t vdesc = sdesc_sw128(sbase + S::V0 + sv * S::TILE, ATOM, 1024);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (!warp_wait(&bars[B_PFULL + 2 * h + half], pe & 1, abort_flag, p.dev_error, p.wait_cycles, code))
                        return false;
                    tc_fence_after();
                    umma_pv_k64(tm + 256 + h * 128, tm + h * 128 + 32 * half, vdesc + 512 * half, IDESC_PV,
                                (pe == 0 && half == 0) ? 0u : 1u);
                }
                umma_commit_elect(&bars[B_PVDONE + h]);
                return true;
            };
            // Issue order per tile e: Q_0 K^T (e), P_1 V (e-1), Q_1 K^T (e), P_0 V (e).
            // S_h(e) overwrites P_h(e-1) in TMEM; the P.V reading it was issued
            // earlier by this warp and the tensor pipe runs one issuer's MMAs in
            // issue order, so no wait separates them.
            bool ok = warp_wait(&bars[B_QREADY0], 0, abort_flag, p.dev_error, p.wait_cycles, 0x311);
            tc_fence_after();
            for (int e = 0; e < NE && ok; ++e) {
                const int sk = e % NSK, uk = e / NSK, sv = e % NSV, uv = e / NSV;
                if (e == nR && nR > 0) {
                    // Q of phase R is no longer read once every MMA so far completed
                    umma_commit_elect(&bars[B_QFREE]);
                    if (!warp_wait(&bars[B_QREADY1], 0, abort_flag, p.dev_error, p.wait_cycles, 0x312)) { ok = false; break; }
                }
                if (!warp_wait(&bars[B_KREADY + sk], uk & 1, abort_flag, p.dev_error, p.wait_cycles, 0x313)) { ok = false; break; }
                tc_fence_after();
                qk(0, sk);
                if (NH == 2) {
                    if (e > 0) {
                        // head 1's P.V of the previous tile runs while head 0's softmax works
                        const int pe = e - 1, psv = pe % NSV, puv = pe / NSV;
                        if (!warp_wait(&bars[B_VFULL + psv], puv & 1, abort_flag, p.dev_error, p.wait_cycles, 0x316)) { ok = false; break; }
                        if (!pv(1, pe, psv, 0x315)) { ok = false; break; }
                        umma_commit_elect(&bars[B_VEMPTY + psv]);
                    }
                    qk(1, sk);
                }
                umma_commit_elect(&bars[B_KEMPTY + sk]);
                if (!warp_wait(&bars[B_VFULL + sv], uv & 1, abort_flag, p.dev_error, p.wait_cycles, 0x319)) { ok = false; break; }
                if (!pv(0, e, sv, 0x318)) { ok = false; break; }
                if (NH == 1) umma_commit_elect(&bars[B_VEMPTY + sv]);
            }
            if (ok && NH == 2 && NE > 0) {
                const int pe = NE - 1, psv = pe % NSV, puv = pe / NSV;
                if (warp_wait(&bars[B_VFULL + psv], puv & 1, abort_flag, p.dev_error, p.wait_cycles, 0x31b) &&
                    pv(1, pe, psv, 0x31a))
                    umma_commit_elect(&bars[B_VEMPTY + psv]);
            }
            // drain: every MMA issued by this warp completed before TMEM is released
            umma_commit_elect(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
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
        bool ok = warp_wait(&bars[B_QFULL], 0, abort_flag, p.dev_error, p.wait_cycles, 0x321);
        if (ok) {
            for (int h = 0; h < NH; ++h) {
                if (nR > 0 || p.window_rot == 1)
                    rotate_tile<D, BM, true, false>(smem + h * S::TILE, t, p, [&](int r) { return div_g(i0 + r, sv); }, stc,
                                             sts, lq);
                else
                    rotate_tile<D, BM, true, false>(smem + h * S::TILE, t, p, [&](int r) { return i0 + r; }, stc, sts, lq);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QREADY0]);
        }
        for (int e = 0; e < NE && ok; ++e) {
            const int sk = e % NSK, uk = e / NSK;
            if (e == nR && nR > 0) {
                // phase switch: Q from floor(i/G) to i, by the extra rotation i - floor(i/G)
                if (!warp_wait(&bars[B_QFREE], 0, abort_flag, p.dev_error, p.wait_cycles, 0x322)) { ok = false; break; }
                for (int h = 0; h < NH; ++h)
                    rotate_tile<D, BM, false, false>(smem + h * S::TILE, t, p,
                                          [&](int r) { return i0 + r - div_g(i0 + r, sv); }, stc, sts, 1.f);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_QREADY1]);
            }
            // the K tile arrives rotated (rope_keys.cu): pass its arrival on
            if (!warp_wait(&bars[B_KFULL + sk], uk & 1, abort_flag, p.dev_error, p.wait_cycles, 0x323)) { ok = false; break; }
            __syncwarp();
            // (test hook: the first key tile is never released, so the MMA
            // thread's bounded wait on it expires)
            if (lane == 0 && !(p.inject == kInjectPrefillKeyTile && e == 0)) mbar_arrive(&bars[B_KREADY + sk]);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // -------------------------------------------------------------- softmax (head hh)
        const int hh = (warp - 8) >> 2;
        if (hh < NH) {
            const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
            uint64_t* pfull = &bars[B_PFULL + 2 * hh];
            softmax_role<D, false>(p, sv, tp, h0 + hh, tid & 127, lane_base + hh * 128,
                                   lane_base + 256 + hh * 128, &bars[B_SFULL + hh], &bars[B_PVDONE + hh],
                                   [pfull](int half) { mbar_arrive(pfull + half); }, abort_flag);
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

template <int D, int NH>
cudaError_t launch_d(const PrefillProblem& pp, cudaStream_t st)
{
    CUtensorMap tq, tkl, tkr, tv;
    cudaError_t e;
    if ((e = make_map(&tq, pp.q, D, pp.C, pp.Cst, pp.B * pp.Hq, BM)) != cudaSuccess) return e;
    if ((e = make_map(&tkl, pp.krot_l, D, pp.L, pp.L, pp.B * pp.Hkv, BN, true)) != cudaSuccess) return e;
    if ((e = make_map(&tkr, pp.krot_r, D, pp.L, pp.L, pp.B * pp.Hkv, BN, true)) != cudaSuccess) return e;
    if ((e = make_map(&tv, pp.v, D, pp.L, pp.Lcap, pp.B * pp.Hkv, BN)) != cudaSuccess) return e;
    const TcParams p = make_params(pp);
    auto kern = prefill_tc_kernel<D, NH>;
    constexpr int smem = TcSmem<D, NH>::TOTAL;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    // variable-length: x over (query-block level, sequence), one z
    dim3 grid(p.vl_n ? p.vl_nqb_max * p.vl_n : p.nqb, pp.Hq / NH, p.vl_n ? 1 : pp.B);
    kern<<<grid, NTHREADS, smem, st>>>(tq, tkl, tkr, tv, p);
    return cudaGetLastError();
}

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

void make_div_magic(uint32_t G, uint32_t* m, uint32_t* s1, uint32_t* s2)
{
    uint32_t l = 0;
    while ((1ull << l) < G) ++l;  // ceil(log2 G)
    *m = (uint32_t)(((((uint64_t)1 << 32) * (((uint64_t)1 << l) - G)) / G) + 1);
    *s1 = l < 1 ? l : 1;
    *s2 = l > 1 ? l - 1 : 0;
}

}  // namespace

cudaError_t make_map(CUtensorMap* m, const void* base, int d, int rows, int plane_rows, int nplanes,
                     int box_rows, bool f16)
{
    cudaError_t err;
    EncodeTiledFn fn = encode_fn(&err);
    if (!fn) return err == cudaSuccess ? cudaErrorSymbolNotFound : err;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)nplanes};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)plane_rows * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

TcParams make_params(const PrefillProblem& pp)
{
    TcParams p{};
    p.B = pp.B; p.Hq = pp.Hq; p.Hkv = pp.Hkv; p.L = pp.L; p.w0 = pp.w0; p.G = pp.G;
    p.P = pp.P; p.C = pp.C; p.Cst = pp.Cst;
    p.nqb = (pp.C + BM - 1) / BM;
    make_div_magic((uint32_t)pp.G, &p.div_m, &p.div_s1, &p.div_s2);
    p.scale_log2 = pp.scale_log2;
    p.turns = pp.turns;
    p.out = pp.out_f32 ? nullptr : reinterpret_cast<__nv_bfloat16*>(pp.out);
    p.out_f32 = pp.out_f32 ? reinterpret_cast<float*>(pp.out) : nullptr;
    p.lse = pp.lse;
    p.window_rot = pp.window_rot;
    p.dev_error = pp.dev_error;
    p.wait_cycles = pp.wait_cycles > 0 ? pp.wait_cycles : kPrefillWaitCycles;
    p.inject = pp.inject;
    p.range = pp.range;
    p.vl_n = pp.vl_n;
    p.vl_nqb_max = 0;
    for (int b = 0; b < pp.vl_n; ++b) {
        p.vl_len[b] = pp.vl_len[b];
        p.vl_nqb_max = std::max(p.vl_nqb_max, (pp.vl_len[b] + BM - 1) / BM);
        make_div_magic((uint32_t)pp.vl_G[b], &p.vl_div[b][0], &p.vl_div[b][1], &p.vl_div[b][2]);
    }
    return p;
}

}  // namespace tc

// d = 128 with a multiple of four query heads per kv head: CTA pairs sharing
// every MMA (prefill_pair.cu); otherwise one CTA per 128 query rows of one or
// two heads of a kv head.
cudaError_t launch_prefill_tc(const PrefillProblem& p, cudaStream_t s, int* nlaunch)
{
    const int group = p.Hq / p.Hkv;
    cudaError_t e;
    if (p.d == 128 && group % 4 == 0)
        e = tc::launch_prefill_pair(p, s);
    else if (p.d == 64)
        e = group % 2 == 0 ? tc::launch_d<64, 2>(p, s) : tc::launch_d<64, 1>(p, s);
    else
        e = group % 2 == 0 ? tc::launch_d<128, 2>(p, s) : tc::launch_d<128, 1>(p, s);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

// prefill_simt.cu -- fp32 CUDA-core prefill of dynamic bifocal RoPE attention
// (whole sequences, or a chunk of query rows at positions [P, P + C) against
// the keys [0, P + C) of a cache).
//
// The fp32 element type (and its 1e-4 accuracy bar) rules out the tensor-core
// path (TF32 keeps 10 mantissa bits), so fp32 inputs run here: a tiled
// online-softmax kernel on fp32 FMA.  One CTA owns BM = 64 query rows of one
// head; it walks key tiles of BN = 64 in order, rotating raw Q and K on the fly
// into shared memory ("Jet-Long: Efficient Long-Context Extension with Dynamic
// Bifocal RoPE", Metodologia 2: rotations applied on the fly, cache untouched).
//
// Tile routing (Metodologia 1, local iff i - j < w0): for tile (qb, kb) the
// causal distances span [dmin, dmax]; dmax < w0 -> local-only (classic RoPE at
// i, j), dmin >= w0 -> remote-only (RoPE at floor(i/G), floor(j/G)), otherwise
// a band tile computes both logits and selects per element.  Every pair lands
// in one softmax (Metodologia 2: one exact distance-routed output).
#include "jl_common.cuh"

namespace jl {
namespace {

constexpr int BM = 64, BN = 64, NT = 256;

template <int D>
struct SimtSmem {
    static constexpr int QS = D + 1;  // padded row stride (floats) for Q/K
    static constexpr int bytes = (4 * 64 * QS + 64 * D + 64 * (BN + 1)) * 4;
};

template <typename T, int D>
__global__ void __launch_bounds__(NT) prefill_simt_kernel(PrefillProblem p)
{
    constexpr int H = D / 2;
    constexpr int QS = D + 1;
    constexpr int CPT = D / 16;  // output columns per thread
    extern __shared__ float sm[];
    float* sQe = sm;                // [BM][QS] exact-rotated q * scale*log2e
    float* sQr = sQe + BM * QS;     // [BM][QS] remote-rotated
    float* sKe = sQr + BM * QS;     // [BN][QS]
    float* sKr = sKe + BN * QS;     // [BN][QS]
    float* sV = sKr + BN * QS;      // [BN][D]
    float* sP = sV + BN * D;        // [BM][BN + 1]

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int nqb = (p.C + BM - 1) / BM;
    const int qb = nqb - 1 - blockIdx.x;  // heaviest query blocks first
    const int h = blockIdx.y, b = blockIdx.z;
    const int kvh = h / (p.Hq / p.Hkv);
    const int G = p.G;
    const bool window = p.window_rot >= 0;  // windowed pass: local pairs only, one rotation
    // positions of the "exact" rotation: i / j, or i / G, j / G in a windowed aliased pass
    auto pe = [&](int x) { return (uint32_t)(p.window_rot == 1 ? x / G : x); };

    // query row i (position P + r of the chunk) is row i - P of q and out
    const T* q = reinterpret_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * (size_t)p.Cst * D;
    const T* k = reinterpret_cast<const T*>(p.k) + ((size_t)b * p.Hkv + kvh) * (size_t)p.Lcap * D;
    const T* v = reinterpret_cast<const T*>(p.v) + ((size_t)b * p.Hkv + kvh) * (size_t)p.Lcap * D;
    T* out = reinterpret_cast<T*>(p.out) + ((size_t)b * p.Hq + h) * (size_t)p.Cst * D;
    float* lse = p.lse ? p.lse + ((size_t)b * p.Hq + h) * (size_t)p.Cst : nullptr;

    // Q tile, rotated at i and at floor(i/G), pre-scaled into base-2 logit units.
    for (int e = tid; e < BM * H; e += NT) {
        int r = e / H, m = e % H;
        int i = p.P + qb * BM + r;
        float a = 0.f, bb = 0.f;
        if (i < p.L) {
            a = load_elem(q + (size_t)(i - p.P) * D + m);
            bb = load_elem(q + (size_t)(i - p.P) * D + m + H);
        }
        float c, s;
        rope_cs_accurate(pe(i), p.turns.hi[m], p.turns.lo[m], c, s);
        sQe[r * QS + m] = (a * c - bb * s) * p.scale_log2;
        sQe[r * QS + m + H] = (a * s + bb * c) * p.scale_log2;
        rope_cs_accurate((uint32_t)(i / G), p.turns.hi[m], p.turns.lo[m], c, s);
        sQr[r * QS + m] = (a * c - bb * s) * p.scale_log2;
        sQr[r * QS + m + H] = (a * s + bb * c) * p.scale_log2;
    }

    float o[4][CPT];
    float mrow[4], lrow[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        mrow[a] = -INFINITY;
        lrow[a] = 0.f;
#pragma unroll
        for (int c = 0; c < CPT; ++c) o[a][c] = 0.f;
    }

    const int i_lo = p.P + qb * BM;
    const int i_hi = min(i_lo + BM - 1, p.L - 1);
    const int nkb = i_hi / BN + 1;
    for (int kb = 0; kb < nkb; ++kb) {
        const int j_lo = kb * BN, j_hi = kb * BN + BN - 1;
        const int dmax = i_hi - j_lo;
        const int dmin = max(0, i_lo - j_hi);
        const bool need_loc = dmax >= 0 && dmin < p.w0;          // some pair is local
        const bool need_rem = !window && dmax >= p.w0;           // some pair is remote
        if (window && !need_loc) continue;  // uniform over the CTA: no local pair here
        __syncthreads();  // previous tile's K/V/P consumers are done
        for (int e = tid; e < BN * H; e += NT) {
            int r = e / H, m = e % H;
            int j = j_lo + r;
            float a = 0.f, bb = 0.f;
            if (j < p.L) {
                a = load_elem(k + (size_t)j * D + m);
                bb = load_elem(k + (size_t)j * D + m + H);
            }
            float c, s;
            if (need_loc) {
                rope_cs_accurate(pe(j), p.turns.hi[m], p.turns.lo[m], c, s);
                sKe[r * QS + m] = a * c - bb * s;
                sKe[r * QS + m + H] = a * s + bb * c;
            }
            if (need_rem) {
                rope_cs_accurate((uint32_t)(j / G), p.turns.hi[m], p.turns.lo[m], c, s);
                sKr[r * QS + m] = a * c - bb * s;
                sKr[r * QS + m + H] = a * s + bb * c;
            }
        }
        for (int e = tid; e < BN * D; e += NT) {
            int r = e / D, c = e % D;
            int j = j_lo + r;
            sV[e] = j < p.L ? load_elem(v + (size_t)j * D + c) : 0.f;
        }
        __syncthreads();

        // S micro-tile: rows ty + 16a, cols tx + 16c
        float s[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[a][c] = 0.f;
        if (need_loc && !need_rem) {
            for (int t = 0; t < D; ++t) {
                float qa[4], kc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) qa[a] = sQe[(ty + 16 * a) * QS + t];
#pragma unroll
                for (int c = 0; c < 4; ++c) kc[c] = sKe[(tx + 16 * c) * QS + t];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) s[a][c] = fmaf(qa[a], kc[c], s[a][c]);
            }
        } else if (need_rem && !need_loc) {
            for (int t = 0; t < D; ++t) {
                float qa[4], kc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) qa[a] = sQr[(ty + 16 * a) * QS + t];
#pragma unroll
                for (int c = 0; c < 4; ++c) kc[c] = sKr[(tx + 16 * c) * QS + t];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) s[a][c] = fmaf(qa[a], kc[c], s[a][c]);
            }
        } else {
            float s2[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) s2[a][c] = 0.f;
            for (int t = 0; t < D; ++t) {
                float qa[4], kc[4], qr[4], kr[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    qa[a] = sQe[(ty + 16 * a) * QS + t];
                    qr[a] = sQr[(ty + 16 * a) * QS + t];
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    kc[c] = sKe[(tx + 16 * c) * QS + t];
                    kr[c] = sKr[(tx + 16 * c) * QS + t];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        s[a][c] = fmaf(qa[a], kc[c], s[a][c]);
                        s2[a][c] = fmaf(qr[a], kr[c], s2[a][c]);
                    }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    int i = i_lo + ty + 16 * a, j = j_lo + tx + 16 * c;
                    if (i - j >= p.w0) s[a][c] = s2[a][c];
                }
        }
        // causal / length mask, online softmax (base 2)
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            int i = i_lo + ty + 16 * a;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int j = j_lo + tx + 16 * c;
                if (j > i || j >= p.L || (window && i - j >= p.w0)) s[a][c] = -INFINITY;
                mx = fmaxf(mx, s[a][c]);
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            float mnew = fmaxf(mrow[a], mx);
            float msafe = mnew == -INFINITY ? 0.f : mnew;
            float alpha = exp2f(mrow[a] - msafe);
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float pe = exp2f(s[a][c] - msafe);
                s[a][c] = pe;
                rs += pe;
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
            lrow[a] = lrow[a] * alpha + rs;
            mrow[a] = mnew;
#pragma unroll
            for (int c = 0; c < CPT; ++c) o[a][c] *= alpha;
#pragma unroll
            for (int c = 0; c < 4; ++c) sP[(ty + 16 * a) * (BN + 1) + tx + 16 * c] = s[a][c];
        }
        __syncthreads();
        for (int j = 0; j < BN; ++j) {
            float vv[CPT];
#pragma unroll
            for (int c = 0; c < CPT; ++c) vv[c] = sV[j * D + tx + 16 * c];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                float pa = sP[(ty + 16 * a) * (BN + 1) + j];
#pragma unroll
                for (int c = 0; c < CPT; ++c) o[a][c] = fmaf(pa, vv[c], o[a][c]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        int i = i_lo + ty + 16 * a;
        if (i >= p.L) continue;
        float inv = 1.f / lrow[a];
#pragma unroll
        for (int c = 0; c < CPT; ++c) store_elem(out + (size_t)(i - p.P) * D + tx + 16 * c, o[a][c] * inv);
        // natural log of the softmax denominator (mrow, lrow are base-2 quantities)
        if (lse && tx == 0) lse[i - p.P] = (mrow[a] + __log2f(lrow[a])) * 0.69314718055994531f;
    }
}

template <typename T, int D>
cudaError_t launch_typed(const PrefillProblem& p, cudaStream_t st)
{
    auto kern = prefill_simt_kernel<T, D>;
    const int smem = SimtSmem<D>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.C + BM - 1) / BM, p.Hq, p.B);
    kern<<<grid, NT, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillProblem& p, jetlong_dtype dt, cudaStream_t s,
                                int* nlaunch)
{
    cudaError_t e;
    if (dt == JETLONG_FP32)
        e = p.d == 64 ? launch_typed<float, 64>(p, s) : launch_typed<float, 128>(p, s);
    else
        e = p.d == 64 ? launch_typed<__nv_bfloat16, 64>(p, s)
                      : launch_typed<__nv_bfloat16, 128>(p, s);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

// decode.cu -- split-K decode of dynamic bifocal RoPE attention over a raw-K cache.
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE",
// Metodologia 2: the KV cache keeps unrotated base keys at their exact
// positions and is never rewritten; the rotation is applied on the fly in
// registers, so generation streams across length boundaries (G changes) with
// no cache rewrite.  Here the cache holds raw K, and each key row is rotated to
// j (local, i - j < w0) or floor(j / G) (remote) as it streams through; the
// query (i = L - 1) is rotated once to i and to floor(i / G).
//
// One CTA = (split of the key range, kv head, batch); it serves all q heads of
// that kv head (grouped-query attention), so every K/V byte is read from HBM
// once.  Warp 4 streams K/V rows into a shared-memory ring with 1-D bulk async
// copies; warps 0-3 consume them: 8 lanes per key row (16-byte loads, pair
// (m, m + d/2) in one lane), warp-shuffle dot products, online softmax per lane
// group in base 2.  The CTA's partial (max, sum, o[d]) goes to the workspace;
// the last CTA of a (b, kv head) -- found with an atomic ticket, no waiting --
// merges all partials with log-sum-exp weights (Metodologia 2: LSE-stabilised
// merge) and writes the output.
#include <cuda.h>

#include <mutex>

#include "jl_common.cuh"
#include "jl_ptx.cuh"

namespace jl {
namespace {

constexpr int KROWS = 32;       // key rows per pipeline stage
constexpr int NCW = 4;          // consumer warps
constexpr int NT = (NCW + 1) * 32;
constexpr int kMaxSplits = 256;
constexpr double kCtaFixedKeys = 256.0;  // per-CTA fixed cost of a decode split, in keys

struct DecodeLaunch {
    int n_splits, chunk, hgroups, hpb;
    uint32_t div_m, div_s1, div_s2;  // floor(j / G) by multiply-shift
    float* partials;                 // [B][Hq][n_splits][D + 2]
    unsigned int* tickets;           // [B][Hkv * hgroups]
    int* dev_error;
    long long wait_cycles;           // limit of every bounded wait
    int inject;                      // kInjectNone, or the arrival this launch withholds (test hook)
};

// Unsigned division by the invariant G (Granlund & Montgomery, "Division by
// Invariant Integers using Multiplication", 1994, Fig. 4.1): exact for all
// 32-bit n.
__device__ __forceinline__ uint32_t div_g(uint32_t n, const DecodeLaunch& dl)
{
    uint32_t t1 = __umulhi(dl.div_m, n);
    return (t1 + ((n - t1) >> dl.div_s1)) >> dl.div_s2;
}

template <typename T, int PPL> struct VecLoad;
template <> struct VecLoad<__nv_bfloat16, 8> {
    __device__ static void run(const __nv_bfloat16* s, float* x)
    {
        uint4 u = *reinterpret_cast<const uint4*>(s);
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
        x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
    }
};
template <> struct VecLoad<__nv_bfloat16, 4> {
    __device__ static void run(const __nv_bfloat16* s, float* x)
    {
        uint2 u = *reinterpret_cast<const uint2*>(s);
        x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    }
};
template <> struct VecLoad<float, 8> {
    __device__ static void run(const float* s, float* x)
    {
        float4 a = *reinterpret_cast<const float4*>(s);
        float4 b = *reinterpret_cast<const float4*>(s + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};
template <> struct VecLoad<float, 4> {
    __device__ static void run(const float* s, float* x)
    {
        float4 a = *reinterpret_cast<const float4*>(s);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    }
};

template <typename T, int D> struct DecodeCfg {
    static constexpr int STAGES = sizeof(T) == 2 ? 4 : 3;
    static constexpr int STAGE_BYTES = 2 * KROWS * D * (int)sizeof(T);  // K then V
    static constexpr int RING = STAGES * STAGE_BYTES;
};

template <int D, int HPB>
__host__ __device__ constexpr int merge_bytes() { return HPB * (NCW * 4) * (D + 2) * 4; }

template <typename T, int D, int HPB>
__host__ __device__ constexpr int decode_smem_bytes()
{
    return (DecodeCfg<T, D>::RING > merge_bytes<D, HPB>() ? DecodeCfg<T, D>::RING
                                                          : merge_bytes<D, HPB>())
           + 2 * HPB * D * 4        // rotated queries: [2][HPB][D]
           + 2 * DecodeCfg<T, D>::STAGES * 8 + 16;  // barriers + flag
}

// Merge the partial softmax states of the GROUPS lane groups (or warps) of this
// CTA -- smem `mo` [HPB][GROUPS][D + 2] holding (o[D], max, sum) in base-2
// units -- into the CTA's split partial in the workspace; the last CTA of this
// (b, kv head, head group) to finish (atomic ticket, no waiting) then merges
// all splits with log-sum-exp weights and writes the output rows.
template <typename T, int D, int HPB, int GROUPS, int NTHR>
__device__ void merge_splits(const float* mo, int* flag, const DecodeProblem& p, const DecodeLaunch& dl,
                             int s, int b, int h0)
{
    const int tid = threadIdx.x;
    float* part_out = dl.partials;
    for (int e = tid; e < HPB * (D + 2); e += NTHR) {
        const int hh = e / (D + 2), col = e % (D + 2);
        float M = -INFINITY;
        for (int grp = 0; grp < GROUPS; ++grp) M = fmaxf(M, mo[((size_t)hh * GROUPS + grp) * (D + 2) + D]);
        float acc = 0.f;
        if (M != -INFINITY) {
            for (int grp = 0; grp < GROUPS; ++grp) {
                const float* row = mo + ((size_t)hh * GROUPS + grp) * (D + 2);
                if (row[D] == -INFINITY) continue;
                const float w = exp2f(row[D] - M);
                acc += w * (col == D ? 0.f : (col == D + 1 ? row[D + 1] : row[col]));
            }
        }
        if (col == D) acc = M;
        const size_t idx = (((size_t)b * p.Hq + h0 + hh) * dl.n_splits + s) * (D + 2) + col;
        part_out[idx] = acc;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        unsigned int* tk = dl.tickets + (size_t)b * p.Hkv * dl.hgroups + blockIdx.y;
        const unsigned int prev = atomicAdd(tk, 1u);
        *flag = (prev == (unsigned int)dl.n_splits - 1) ? 1 : 0;
        if (*flag) *tk = 0u;  // ready for the next call
    }
    __syncthreads();
    if (*flag == 0) return;
    __threadfence();
    T* out = reinterpret_cast<T*>(p.out);
    for (int e = tid; e < HPB * D; e += NTHR) {
        const int hh = e / D, col = e % D;
        const float* base = part_out + ((size_t)b * p.Hq + h0 + hh) * dl.n_splits * (D + 2);
        float M = -INFINITY;
        for (int sp = 0; sp < dl.n_splits; ++sp) M = fmaxf(M, __ldcg(base + (size_t)sp * (D + 2) + D));
        float num = 0.f, den = 0.f;
        for (int sp = 0; sp < dl.n_splits; ++sp) {
            const float* row = base + (size_t)sp * (D + 2);
            const float ms = __ldcg(row + D);
            if (ms == -INFINITY) continue;
            const float w = exp2f(ms - M);
            num += w * __ldcg(row + col);
            den += w * __ldcg(row + D + 1);
        }
        store_elem(out + ((size_t)b * p.Hq + h0 + hh) * D + col, num / den);
    }
}

template <typename T, int D, int HPB>
__global__ void __launch_bounds__(NT, 2) decode_split_kernel(DecodeProblem p, DecodeLaunch dl)
{
    constexpr int H = D / 2;
    constexpr int PPL = D / 16;  // rotation pairs per lane (8 lanes per key row)
    constexpr int STAGES = DecodeCfg<T, D>::STAGES;
    constexpr int ROWB = D * (int)sizeof(T);
    constexpr int GROUPS = NCW * 4;  // lane groups per CTA

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* ring = smem;
    constexpr int RING_SPAN = decode_smem_bytes<T, D, HPB>() - 2 * HPB * D * 4 - 2 * STAGES * 8 - 16;
    float* sq = reinterpret_cast<float*>(smem + RING_SPAN);  // [2][HPB][D]
    uint64_t* full = reinterpret_cast<uint64_t*>(sq + 2 * HPB * D);
    uint64_t* empty = full + STAGES;
    int* flag = reinterpret_cast<int*>(empty + STAGES);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = blockIdx.x;
    const int kvh = blockIdx.y / dl.hgroups, hg = blockIdx.y % dl.hgroups;
    const int b = blockIdx.z;
    const int group = p.Hq / p.Hkv;
    const int h0 = kvh * group + hg * HPB;
    const int L = p.L;
    const int i = L - 1;
    const int j_begin = s * dl.chunk;
    const int j_end = min(L, j_begin + dl.chunk);
    const int nrows = max(0, j_end - j_begin);
    const int nchunks = (nrows + KROWS - 1) / KROWS;
    const int j_exact = i - p.w0 + 1;  // keys j >= j_exact are local

    if (tid == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], NCW);
        }
        fence_mbar_init();
    }
    // rotated queries, pre-scaled to base-2 logit units
    {
        const T* q = reinterpret_cast<const T*>(p.q) + ((size_t)b * p.Hq + h0) * D;
        const uint32_t pe = (uint32_t)i, pr = div_g((uint32_t)i, dl);
        for (int e = tid; e < HPB * H; e += NT) {
            int hh = e / H, m = e % H;
            float a = load_elem(q + (size_t)hh * D + m), c2 = load_elem(q + (size_t)hh * D + m + H);
            float c, sn;
            rope_cs_accurate(pe, p.turns.hi[m], p.turns.lo[m], c, sn);
            sq[(0 * HPB + hh) * D + m] = (a * c - c2 * sn) * p.scale_log2;
            sq[(0 * HPB + hh) * D + m + H] = (a * sn + c2 * c) * p.scale_log2;
            rope_cs_accurate(pr, p.turns.hi[m], p.turns.lo[m], c, sn);
            sq[(1 * HPB + hh) * D + m] = (a * c - c2 * sn) * p.scale_log2;
            sq[(1 * HPB + hh) * D + m + H] = (a * sn + c2 * c) * p.scale_log2;
        }
    }
    __syncthreads();

    const size_t kv_base = ((size_t)b * p.Hkv + kvh) * (size_t)p.Lcap * D;
    const T* kc = reinterpret_cast<const T*>(p.kc) + kv_base;
    const T* vc = reinterpret_cast<const T*>(p.vc) + kv_base;

    // per lane-group softmax state
    float o[HPB][2 * PPL];
    float mrow[HPB], lrow[HPB];
#pragma unroll
    for (int hh = 0; hh < HPB; ++hh) {
        mrow[hh] = -INFINITY;
        lrow[hh] = 0.f;
#pragma unroll
        for (int u = 0; u < 2 * PPL; ++u) o[hh][u] = 0.f;
    }

    bool ok = true;
    if (warp == NCW) {
        // ---------------- producer: one lane streams K/V rows into the ring
        int issued = 0;
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % STAGES;
                if (c >= STAGES && !mbar_wait(&empty[st], ((c / STAGES) - 1) & 1, dl.wait_cycles)) {
                    record_error(dl.dev_error, 0x101);
                    break;
                }
                const int j0 = j_begin + c * KROWS;
                const int rows = min(KROWS, j_end - j0);
                const uint32_t bytes = (uint32_t)(rows * ROWB);
                unsigned char* dst = ring + st * DecodeCfg<T, D>::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[st], 2 * bytes);
                bulk_g2s(dst, kc + (size_t)j0 * D, bytes, &full[st]);
                bulk_g2s(dst + KROWS * ROWB, vc + (size_t)j0 * D, bytes, &full[st]);
                issued = c + 1;
            }
            // drain: every issued copy has landed before the ring is reused / the CTA exits
            for (int c = max(0, issued - STAGES); c < issued; ++c)
                if (!mbar_wait(&full[c % STAGES], (c / STAGES) & 1, dl.wait_cycles)) record_error(dl.dev_error, 0x102);
        }
    } else {
        // ---------------- consumers
        const int g = lane >> 3, t = lane & 7;
        const int m0 = t * PPL;
        uint32_t whi[PPL], wlo[PPL];
#pragma unroll
        for (int u = 0; u < PPL; ++u) {
            whi[u] = p.turns.hi[m0 + u];
            wlo[u] = p.turns.lo[m0 + u];
        }
        int ver = -1;  // which rotated query the registers hold (0 exact, 1 remote)
        float qlo[HPB][PPL], qhi[HPB][PPL];
        for (int c = 0; c < nchunks && ok; ++c) {
            const int st = c % STAGES;
            if (!mbar_wait(&full[st], (c / STAGES) & 1, dl.wait_cycles)) {
                record_error(dl.dev_error, 0x103);
                ok = false;
                break;
            }
            const unsigned char* kst = ring + st * DecodeCfg<T, D>::STAGE_BYTES;
            const unsigned char* vst = kst + KROWS * ROWB;
            const int j0 = j_begin + c * KROWS;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int r = warp * 8 + g + 4 * half;
                const int j = j0 + r;
                const bool valid = j < j_end;
                const bool exact = j >= j_exact;
                const int want = exact ? 0 : 1;
                if (want != ver) {
                    ver = want;
#pragma unroll
                    for (int hh = 0; hh < HPB; ++hh)
#pragma unroll
                        for (int u = 0; u < PPL; ++u) {
                            qlo[hh][u] = sq[(ver * HPB + hh) * D + m0 + u];
                            qhi[hh][u] = sq[(ver * HPB + hh) * D + H + m0 + u];
                        }
                }
                // raw keys go to j or f(j); keys stored at j stay, or move by f(j) - j <= 0
                const uint32_t fj = div_g((uint32_t)j, dl);
                const uint32_t pos = p.rope_cache ? (exact ? 0u : (uint32_t)j - fj) : (exact ? (uint32_t)j : fj);
                const float sgn = (p.rope_cache && !exact) ? -1.f : 1.f;
                float klo[PPL], khi[PPL];
                const T* krow = reinterpret_cast<const T*>(kst + r * ROWB);
                VecLoad<T, PPL>::run(krow + m0, klo);
                VecLoad<T, PPL>::run(krow + H + m0, khi);
                float part[HPB];
#pragma unroll
                for (int hh = 0; hh < HPB; ++hh) part[hh] = 0.f;
#pragma unroll
                for (int u = 0; u < PPL; ++u) {
                    float cs, sn;
                    rope_cs_fast(pos, whi[u], wlo[u], cs, sn);
                    sn *= sgn;
                    const float rl = klo[u] * cs - khi[u] * sn;
                    const float rh = klo[u] * sn + khi[u] * cs;
#pragma unroll
                    for (int hh = 0; hh < HPB; ++hh)
                        part[hh] = fmaf(qlo[hh][u], rl, fmaf(qhi[hh][u], rh, part[hh]));
                }
#pragma unroll
                for (int hh = 0; hh < HPB; ++hh) {
                    part[hh] += __shfl_xor_sync(0xffffffffu, part[hh], 1);
                    part[hh] += __shfl_xor_sync(0xffffffffu, part[hh], 2);
                    part[hh] += __shfl_xor_sync(0xffffffffu, part[hh], 4);
                }
                if (valid) {
                    float vlo[PPL], vhi[PPL];
                    const T* vrow = reinterpret_cast<const T*>(vst + r * ROWB);
                    VecLoad<T, PPL>::run(vrow + m0, vlo);
                    VecLoad<T, PPL>::run(vrow + H + m0, vhi);
#pragma unroll
                    for (int hh = 0; hh < HPB; ++hh) {
                        const float sc = part[hh];
                        if (sc > mrow[hh]) {  // rare after the first keys
                            const float alpha = exp2f(mrow[hh] - sc);
                            lrow[hh] *= alpha;
#pragma unroll
                            for (int u = 0; u < 2 * PPL; ++u) o[hh][u] *= alpha;
                            mrow[hh] = sc;
                        }
                        const float pe = exp2f(sc - mrow[hh]);
                        lrow[hh] += pe;
#pragma unroll
                        for (int u = 0; u < PPL; ++u) {
                            o[hh][u] = fmaf(pe, vlo[u], o[hh][u]);
                            o[hh][PPL + u] = fmaf(pe, vhi[u], o[hh][PPL + u]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
    }
    __syncthreads();  // ring drained; reuse it for the lane-group merge

    float* mo = reinterpret_cast<float*>(ring);  // [HPB][GROUPS][D + 2]
    if (warp < NCW) {
        const int g = lane >> 3, t = lane & 7, grp = warp * 4 + g;
        const int m0 = t * PPL;
#pragma unroll
        for (int hh = 0; hh < HPB; ++hh) {
            float* row = mo + ((size_t)hh * GROUPS + grp) * (D + 2);
#pragma unroll
            for (int u = 0; u < PPL; ++u) {
                row[m0 + u] = o[hh][u];
                row[H + m0 + u] = o[hh][PPL + u];
            }
            if (t == 0) {
                row[D] = mrow[hh];
                row[D + 1] = lrow[hh];
            }
        }
    }
    __syncthreads();
    merge_splits<T, D, HPB, GROUPS, NT>(mo, flag, p, dl, s, b, h0);
}

// ---------------------------------------------------------------------------
// bf16 decode on warp-level tensor-core MMAs (m16n8k16).
//
// The group's query heads are the N = 8 columns of the MMA, 16 keys its M
// rows: S^T (16 keys x 8 heads) = K_rot (16 x d) * Q_rot^T (d x 8), then
// O^T (d x 8) += V^T (d x 16) * P^T (16 x 8).  K and V stream into shared
// memory with 2-D TMA (128-byte swizzle, 64 keys per stage); each warp owns 16
// keys of a stage: ldmatrix brings K fragments to registers, where the pairs
// (m, m + d/2) sit in the same thread (k-steps kb and kb + d/32) and are
// rotated to j or floor(j/G) before the MMA (fp16 operands; Q^T is fp16 too).
// P goes through a 256-byte per-warp buffer to become the B fragment of P V.
// Online softmax per head in base 2 with lazy rescaling (threshold 2^8).

constexpr int TC_KROWS = 64, TC_NCW = 4, TC_NT = (TC_NCW + 1) * 32, TC_STAGES = 3;
constexpr float kDecRescale = 8.0f;

template <int D, int HPB>
struct DecTcCfg {
    static constexpr int ATOMS = D / 64;
    static constexpr int TILE = TC_KROWS * D * 2;  // one K or V stage tile
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING = TC_STAGES * STAGE;
    static constexpr int MERGE = HPB * TC_NCW * (D + 2) * 4;
    static constexpr int BIG = RING > MERGE ? RING : MERGE;
    static constexpr int PBUF = BIG;                       // [TC_NCW][16 keys][8 heads] bf16
    static constexpr int SQ = PBUF + TC_NCW * 256;         // [2][HPB][D] fp32 rotated queries
    static constexpr int TURNS = SQ + 2 * HPB * D * 4;     // [d/2] uint2 phase constants
    static constexpr int DELTA = TURNS + (D / 2) * 8;      // [9][d/4] float4 (cos, cos, sin, sin) of 0..8 steps
    static constexpr int QEXP = DELTA + 9 * (D / 2) * 8;   // [8] int query exponents, [1] large-query flag
    static constexpr int BARS = QEXP + 48;
    static constexpr int END = BARS + 2 * TC_STAGES * 8 + 16;
    static constexpr int TOTAL = END + 1024;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void tma_load_3d_dec(void* dst, const void* tmap, int x, int y, int z, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// shared-memory address of 16-byte chunk `ch` of key row `key` in a stage tile
// stored by TMA as [d/64 atoms][64 keys][128 B], chunk index XOR key % 8
__device__ __forceinline__ uint32_t dec_sw(uint32_t tile, int key, int ch)
{
    return tile + (uint32_t)((ch >> 3) * (TC_KROWS * 128) + key * 128 + (((ch & 7) ^ (key & 7)) << 4));
}

// Operand range of the fp16 Q K^T MMAs.  The rotated keys and queries are
// rounded to fp16 (11-bit significand, largest value 65504; bf16 inputs reach
// 3.4e38), so each key row and each query head is first scaled by a power of
// two that brings its largest |x| into [2^13, 2^14): a rotated value is then
// below 2^14.5, and powers of two are exact both ways, so multiplying a logit by
// 2^-(e_q + e_k) gives the logit of the unscaled vectors.  Exponents are clamped
// to [-100, 100].
__device__ __forceinline__ uint32_t absmax_bf16x2_dec(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Exponent e with m * 2^e in [2^13, 2^14) for a largest magnitude m given by its
// bf16 (15-bit) magnitude bits; 0 for zero or a non-finite m.
__device__ __forceinline__ int range_exp_bf16(uint32_t mag)
{
    if (mag == 0u || mag >= 0x7f80u) return 0;
    const int biased = (int)(mag >> 7);
    return min(100, max(-100, 13 - ((biased == 0 ? 1 : biased) - 127)));
}

__device__ __forceinline__ float pow2i_dec(int e) { return __int_as_float((e + 127) << 23); }

// Rotates two adjacent pairs m, m + 1 of one key row: (x, y) of pair m in the
// low halves of lo / hi, pair m + 1 in the high halves, by the angles with
// cosines c0, c1 and sines s0, s1 (by minus them for NEG), times lam when
// SCALED; packs to fp16.
template <bool SCALED, bool NEG>
__device__ __forceinline__ void rotate_pairs(uint32_t& lo, uint32_t& hi, float c0, float s0, float c1, float s1,
                                             float lam)
{
    if (SCALED) {
        c0 *= lam;
        c1 *= lam;
        s0 *= lam;
        s1 *= lam;
    }
    if (NEG) {
        s0 = -s0;
        s1 = -s1;
    }
    const float x0 = bf16_lo(lo), x1 = bf16_hi(lo);
    const float y0 = bf16_lo(hi), y1 = bf16_hi(hi);
    lo = pack_f16x2(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1);
    hi = pack_f16x2(x0 * s0 + y0 * c0, x1 * s1 + y1 * c1);
}

// S^T for the 16 keys of this warp's block: rotated K fragments times Q^T.
// Keys of rows g and g + 8 are rotated by the angles of positions pa and pb
// (by minus those angles for NEG); pb - pa must lie in [0, 8], as it does for
// rows 8 apart.  Row g's angles come from the phase, row g + 8's from them by
// angle addition with the table of 0..8 steps.  SCALED: each key row is first scaled
// by its own power of two and ka / kc receive the inverse scales of rows
// g / g + 8; otherwise the keys are rounded as they are and ka = kc = 1.
template <int D, bool SCALED, bool NEG>
__device__ __forceinline__ void block_logits(float (&c)[4], uint32_t ktile, int kw, int lane, uint32_t pa, uint32_t pb,
                                             const uint2* sturns, const float4* sdelta,
                                             const uint32_t (&qb)[D / 16][2],
                                             float& ka, float& kc)
{
    const int t = lane & 3;
    // two independent accumulators (first / second halves of the pairs), summed
    // at the end: half the dependent chain of MMAs
    float c2[4] = {0.f, 0.f, 0.f, 0.f};
    c[0] = c[1] = c[2] = c[3] = 0.f;
    // ldmatrix.x4 rows: lanes 0-7 keys 0-7 / chunk lo, 8-15 keys 8-15 / lo, 16-23 keys 0-7 / hi, 24-31 keys 8-15 / hi
    const int lkey = kw + (lane & 7) + ((lane >> 3) & 1) * 8, lhalf = lane >> 4;
    uint32_t lo[D / 32][4], hi[D / 32][4];
#pragma unroll
    for (int kb = 0; kb < D / 32; ++kb) {
        ldsm_x4(dec_sw(ktile, lkey, 2 * kb + lhalf), lo[kb]);
        ldsm_x4(dec_sw(ktile, lkey, 2 * kb + D / 16 + lhalf), hi[kb]);
    }
    float la = 1.f, lc = 1.f;
    ka = kc = 1.f;
    if (SCALED) {
    // largest |k| of rows g (fragments 0, 2) and g + 8 (fragments 1, 3); the four
    // threads t = 0..3 of a row hold its d values between them
    uint32_t aa = 0u, ac = 0u;
#pragma unroll
    for (int kb = 0; kb < D / 32; ++kb) {
        aa = absmax_bf16x2_dec(aa, absmax_bf16x2_dec(absmax_bf16x2_dec(lo[kb][0], lo[kb][2]),
                                                     absmax_bf16x2_dec(hi[kb][0], hi[kb][2])));
        ac = absmax_bf16x2_dec(ac, absmax_bf16x2_dec(absmax_bf16x2_dec(lo[kb][1], lo[kb][3]),
                                                     absmax_bf16x2_dec(hi[kb][1], hi[kb][3])));
    }
    uint32_t ma = max(aa & 0x7fffu, (aa >> 16) & 0x7fffu), mc = max(ac & 0x7fffu, (ac >> 16) & 0x7fffu);
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
    mc = max(mc, __shfl_xor_sync(0xffffffffu, mc, 1));
    ma = max(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
    mc = max(mc, __shfl_xor_sync(0xffffffffu, mc, 2));
    const int ea = range_exp_bf16(ma), ec = range_exp_bf16(mc);
    la = pow2i_dec(ea);
    lc = pow2i_dec(ec);
    ka = pow2i_dec(-ea);
    kc = pow2i_dec(-ec);
    }
    // row g + 8 sits dpos = pb - pa in [0, 8] positions after row g (exact
    // positions: 8; grouped positions: the difference of two floor(j / G))
    const float4* drow = sdelta + min(pb - pa, 8u) * (D / 4);
#pragma unroll
    for (int kb = 0; kb < D / 32; ++kb) {
        // lo[kb][2h] / hi[kb][2h]: row g, pairs m, m + 1 (first / second halves
        // of d); lo[kb][2h + 1] / hi[kb][2h + 1]: row g + 8, same pairs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = 16 * kb + 2 * t + 8 * h;
            const uint4 w = *reinterpret_cast<const uint4*>(sturns + m);  // (hi, lo) of pairs m, m + 1
            float c0, s0, c1, s1;
            rope_cs_fast(pa, w.x, w.y, c0, s0);
            rope_cs_fast(pa, w.z, w.w, c1, s1);
            // angle addition: (c + i s) of row g times that of dpos steps,
            // stored as (cos m, cos m+1, sin m, sin m+1)
            const float4 st = drow[m / 2];
            const float cb0 = c0 * st.x - s0 * st.z, sb0 = s0 * st.x + c0 * st.z;
            const float cb1 = c1 * st.y - s1 * st.w, sb1 = s1 * st.y + c1 * st.w;
            rotate_pairs<SCALED, NEG>(lo[kb][2 * h], hi[kb][2 * h], c0, s0, c1, s1, la);
            rotate_pairs<SCALED, NEG>(lo[kb][2 * h + 1], hi[kb][2 * h + 1], cb0, sb0, cb1, sb1, lc);
        }
        mma_f16(c, lo[kb], qb[kb][0], qb[kb][1]);
        mma_f16(c2, hi[kb], qb[kb + D / 32][0], qb[kb + D / 32][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] += c2[i];
}

// RC: the cache holds keys already rotated to their own positions (rope_cache).
template <int D, int HPB, bool RC>
__global__ void __launch_bounds__(TC_NT, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     DecodeProblem p, DecodeLaunch dl)
{
    using C = DecTcCfg<D, HPB>;
    constexpr int H = D / 2;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    unsigned char* ring = smem;
    float* sq = reinterpret_cast<float*>(smem + C::SQ);           // [2][HPB][D]
    uint2* sturns = reinterpret_cast<uint2*>(smem + C::TURNS);    // (hi, lo) per frequency
    float* sdel = reinterpret_cast<float*>(smem + C::DELTA);       // [9][d/4] (cos m, cos m+1, sin m, sin m+1) of 0..8 steps
    const float4* sdelta = reinterpret_cast<const float4*>(sdel);
    int* qexp = reinterpret_cast<int*>(smem + C::QEXP);            // [HPB] query exponents
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BARS);
    uint64_t* empty = full + TC_STAGES;
    int* flag = reinterpret_cast<int*>(empty + TC_STAGES);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int s = blockIdx.x;
    const int kvh = blockIdx.y / dl.hgroups, hg = blockIdx.y % dl.hgroups;
    const int b = blockIdx.z;
    const int group = p.Hq / p.Hkv;
    const int h0 = kvh * group + hg * HPB;
    const int L = p.L, i = L - 1;
    const int j_begin = s * dl.chunk;
    const int j_end = min(L, j_begin + dl.chunk);
    const int nchunks = max(0, (j_end - j_begin + TC_KROWS - 1) / TC_KROWS);
    const int j_exact = i - p.w0 + 1;  // keys j >= j_exact are local

    if (tid == 0) {
        for (int st = 0; st < TC_STAGES; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], TC_NCW);
        }
        fence_mbar_init();
    }
    for (int m = tid; m < H; m += TC_NT) sturns[m] = make_uint2(p.turns.hi[m], p.turns.lo[m]);
    for (int e = tid; e < 9 * H; e += TC_NT) {
        const int dpos = e / H, m = e % H;
        float c, sn;
        rope_cs_accurate((uint32_t)dpos, p.turns.hi[m], p.turns.lo[m], c, sn);
        float* q4 = sdel + (dpos * (H / 2) + m / 2) * 4 + (m & 1);
        q4[0] = c;
        q4[2] = sn;
    }
    {
        const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + h0) * D;
        const uint32_t pe = (uint32_t)i, pr = div_g((uint32_t)i, dl);
        for (int e = tid; e < HPB * H; e += TC_NT) {
            const int hh = e / H, m = e % H;
            const float a = load_elem(q + (size_t)hh * D + m), c2 = load_elem(q + (size_t)hh * D + m + H);
            float c, sn;
            rope_cs_accurate(pe, p.turns.hi[m], p.turns.lo[m], c, sn);
            sq[(0 * HPB + hh) * D + m] = (a * c - c2 * sn) * p.scale_log2;
            sq[(0 * HPB + hh) * D + m + H] = (a * sn + c2 * c) * p.scale_log2;
            rope_cs_accurate(pr, p.turns.hi[m], p.turns.lo[m], c, sn);
            sq[(1 * HPB + hh) * D + m] = (a * c - c2 * sn) * p.scale_log2;
            sq[(1 * HPB + hh) * D + m + H] = (a * sn + c2 * c) * p.scale_log2;
        }
    }
    __syncthreads();
    // Query scales: a head whose rotated query (both rotations, base-2 logit
    // units) has its largest |x| in [2^-3, 2^14) is used as it is (exponent 0);
    // any other head is scaled to bring it into [2^13, 2^14).  Any scaled head,
    // or an L1 norm above 2^14 (where fp16-subnormal keys could err by more than
    // 2^-11 in a logit), sets qexp[8]: every key block of this CTA then takes the
    // scaled path.  Warp w takes heads w, w + 5, ...
    if (tid == 0) qexp[8] = 0;
    __syncthreads();
    for (int hh = warp; hh < HPB; hh += TC_NT / 32) {
        float mx = 0.f, l1e = 0.f, l1r = 0.f;
        for (int e = lane; e < D; e += 32) {
            const float xe = fabsf(sq[(0 * HPB + hh) * D + e]), xr = fabsf(sq[(1 * HPB + hh) * D + e]);
            mx = fmaxf(mx, fmaxf(xe, xr));
            l1e += xe;
            l1r += xr;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            l1e += __shfl_xor_sync(0xffffffffu, l1e, o);
            l1r += __shfl_xor_sync(0xffffffffu, l1r, o);
        }
        // non-negative floats order like their bit patterns
        const uint32_t bits = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
        if (lane == 0) {
            int e = 0;
            const float mxh = __uint_as_float(bits);
            if (bits != 0u && bits < 0x7f800000u && !(mxh >= 0.125f && mxh < 16384.f)) {
                const int biased = (int)(bits >> 23);
                e = min(100, max(-100, 13 - ((biased == 0 ? 1 : biased) - 127)));
            }
            qexp[hh] = e;
            if (e != 0 || !(fmaxf(l1e, l1r) <= 16384.f)) atomicOr(&qexp[8], 1);
        }
    }
    __syncthreads();

    const int zkv = b * p.Hkv + kvh;
    float* mo = reinterpret_cast<float*>(ring);  // reused after the ring drains: [HPB][TC_NCW][D + 2]
    if (warp == TC_NCW) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c % TC_STAGES;
                if (c >= TC_STAGES && !mbar_wait(&empty[st], ((c / TC_STAGES) - 1) & 1, dl.wait_cycles)) {
                    record_error(dl.dev_error, 0x111);
                    break;
                }
                const int j0 = j_begin + c * TC_KROWS;
                unsigned char* dst = ring + st * C::STAGE;
                // (test hook: the first stage is never loaded, so the consumers'
                // bounded waits on it expire)
                if (c == 0 && dl.inject == kInjectDecodeCopy) continue;
                mbar_arrive_expect_tx(&full[st], C::STAGE);
#pragma unroll
                for (int a = 0; a < C::ATOMS; ++a) {
                    tma_load_3d_dec(dst + a * TC_KROWS * 128, &tmK, a * 64, j0, zkv, &full[st]);
                    tma_load_3d_dec(dst + C::TILE + a * TC_KROWS * 128, &tmV, a * 64, j0, zkv, &full[st]);
                }
                issued = c + 1;
            }
            for (int c = max(0, issued - TC_STAGES); c < issued; ++c)
                if (!mbar_wait(&full[c % TC_STAGES], (c / TC_STAGES) & 1, dl.wait_cycles)) record_error(dl.dev_error, 0x112);
        }
        __syncthreads();
    } else {
        // ---------------------------------------------------------- consumers
        const int g = lane >> 2, t = lane & 3;
        // Q^T fragments (fp16): b0 = (Q[g][16kb+2t], Q[g][16kb+2t+1]), b1 = dims + 8; heads >= HPB are 0
        uint32_t qb_ex[D / 16][2], qb_rm[D / 16][2];
        const float lq = g < HPB ? pow2i_dec(qexp[g]) : 1.f;
        const bool always_scaled = qexp[8] != 0;
        // inverse query scales of this thread's logit columns (heads 2t, 2t + 1)
        const float cq0 = 2 * t < HPB ? pow2i_dec(-qexp[2 * t]) : 1.f;
        const float cq1 = 2 * t + 1 < HPB ? pow2i_dec(-qexp[2 * t + 1]) : 1.f;
#pragma unroll
        for (int kb = 0; kb < D / 16; ++kb) {
            const int m = 16 * kb + 2 * t;
            if (g < HPB) {
                const float* qe = sq + (0 * HPB + g) * D;
                const float* qr = sq + (1 * HPB + g) * D;
                qb_ex[kb][0] = pack_f16x2(qe[m] * lq, qe[m + 1] * lq);
                qb_ex[kb][1] = pack_f16x2(qe[m + 8] * lq, qe[m + 9] * lq);
                qb_rm[kb][0] = pack_f16x2(qr[m] * lq, qr[m + 1] * lq);
                qb_rm[kb][1] = pack_f16x2(qr[m + 8] * lq, qr[m + 9] * lq);
            } else {
                qb_ex[kb][0] = qb_ex[kb][1] = qb_rm[kb][0] = qb_rm[kb][1] = 0u;
            }
        }
        float o[D / 16][4];
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        float mh[2] = {-INFINITY, -INFINITY}, lh[2] = {0.f, 0.f};  // heads 2t, 2t + 1
        const uint32_t pbuf = smem_u32(smem + C::PBUF + warp * 256);
        const int kw = warp * 16;  // this warp's keys within a stage
        for (int c = 0; c < nchunks; ++c) {
            const int st = c % TC_STAGES;
            if (!mbar_wait(&full[st], (c / TC_STAGES) & 1, dl.wait_cycles)) {
                record_error(dl.dev_error, 0x113);
                break;
            }
            const uint32_t ktile = smem_u32(ring + st * C::STAGE), vtile = ktile + C::TILE;
            const int jb = j_begin + c * TC_KROWS + kw;  // first key of this warp's block
            const int ja = jb + g, jc = jb + g + 8;     // the keys of rows g and g + 8
            // raw keys go to j (local) or f(j) (remote); keys stored rotated to
            // j stay (local) or move by f(j) - j <= 0 (remote)
            const uint32_t ea = RC ? 0u : (uint32_t)ja, ec = RC ? 0u : (uint32_t)jc;
            const uint32_t fa = div_g((uint32_t)ja, dl), fc = div_g((uint32_t)jc, dl);
            const uint32_t ra = RC ? (uint32_t)ja - fa : fa, rc = RC ? (uint32_t)jc - fc : fc;
            // Keys are rounded to fp16 as they are unless that could lose the
            // logits: an element beyond fp16's range (seen as a non-finite
            // logit, as it always is) or a query for which the CTA takes the
            // scaled path throughout.  Then each key row is scaled by its own
            // power of two and the logits by the inverse key and query scales.
            float sc[4];
            bool scaled = always_scaled;
            if (!scaled) {
                float ka, kc;
                if (jb >= j_exact) {
                    block_logits<D, false, false>(sc, ktile, kw, lane, ea, ec, sturns, sdelta, qb_ex, ka, kc);
                } else if (jb + 15 < j_exact) {
                    block_logits<D, false, RC>(sc, ktile, kw, lane, ra, rc, sturns, sdelta, qb_rm, ka, kc);
                } else {
                    float se[4];
                    block_logits<D, false, RC>(sc, ktile, kw, lane, ra, rc, sturns, sdelta, qb_rm, ka, kc);
                    block_logits<D, false, false>(se, ktile, kw, lane, ea, ec, sturns, sdelta, qb_ex, ka, kc);
                    if (ja >= j_exact) { sc[0] = se[0]; sc[1] = se[1]; }
                    if (jc >= j_exact) { sc[2] = se[2]; sc[3] = se[3]; }
                }
                scaled = __any_sync(0xffffffffu, !(fabsf(sc[0]) < INFINITY && fabsf(sc[1]) < INFINITY &&
                                                   fabsf(sc[2]) < INFINITY && fabsf(sc[3]) < INFINITY));
            }
            if (scaled) {
                float ka, kc;
                if (jb >= j_exact) {
                    block_logits<D, true, false>(sc, ktile, kw, lane, ea, ec, sturns, sdelta, qb_ex, ka, kc);
                } else if (jb + 15 < j_exact) {
                    block_logits<D, true, RC>(sc, ktile, kw, lane, ra, rc, sturns, sdelta, qb_rm, ka, kc);
                } else {
                    float se[4];
                    block_logits<D, true, RC>(sc, ktile, kw, lane, ra, rc, sturns, sdelta, qb_rm, ka, kc);
                    block_logits<D, true, false>(se, ktile, kw, lane, ea, ec, sturns, sdelta, qb_ex, ka, kc);
                    if (ja >= j_exact) { sc[0] = se[0]; sc[1] = se[1]; }
                    if (jc >= j_exact) { sc[2] = se[2]; sc[3] = se[3]; }
                }
                // undo the operand scales: sc[0], sc[1] are key g with heads 2t,
                // 2t + 1, sc[2], sc[3] key g + 8
                sc[0] = sc[0] * ka * cq0;
                sc[1] = sc[1] * ka * cq1;
                sc[2] = sc[2] * kc * cq0;
                sc[3] = sc[3] * kc * cq1;
            }
            if (ja >= j_end) sc[0] = sc[1] = -INFINITY;
            if (jc >= j_end) sc[2] = sc[3] = -INFINITY;
            // online softmax for heads 2t (sc[0], sc[2]) and 2t + 1 (sc[1], sc[3]) over the 16 keys
            float bm0 = fmaxf(sc[0], sc[2]), bm1 = fmaxf(sc[1], sc[3]);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
                bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
            }
            const float bm[2] = {bm0, bm1};
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float mn = fmaxf(mh[u], bm[u]);
                if (mn > mh[u] + kDecRescale) {
                    const float alpha = exp2f(mh[u] - mn);
                    lh[u] *= alpha;
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        o[mt][u] *= alpha;
                        o[mt][2 + u] *= alpha;
                    }
                    mh[u] = mn;
                }
            }
            const float ms0 = mh[0] == -INFINITY ? 0.f : mh[0], ms1 = mh[1] == -INFINITY ? 0.f : mh[1];
            const float p0 = exp2f(sc[0] - ms0), p1 = exp2f(sc[1] - ms1);
            const float p2 = exp2f(sc[2] - ms0), p3 = exp2f(sc[3] - ms1);
            lh[0] += p0 + p2;
            lh[1] += p1 + p3;
            // P^T fragment through the warp's buffer [16 keys][8 heads] bf16
            __syncwarp();
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(pbuf + g * 16 + t * 4), "r"(pack_bf16x2(p0, p1)) : "memory");
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(pbuf + (g + 8) * 16 + t * 4), "r"(pack_bf16x2(p2, p3)) : "memory");
            __syncwarp();
            uint32_t pb0, pb1;
            ldsm_x2_t(pbuf + (lane & 15) * 16, pb0, pb1);
            // O^T += V^T P^T over the d/16 row tiles of 16 dims
            const int vkey = kw + (lane & 7) + (lane >> 4) * 8, vhalf = (lane >> 3) & 1;
            // keys past the valid range (cache rows >= L may hold anything) contribute
            // exactly zero: their V entries are cleared, not only their P
            const bool tail = jb + 15 >= j_end;
            const uint32_t m_lo = (jb + 2 * t < j_end ? 0x0000ffffu : 0u) | (jb + 2 * t + 1 < j_end ? 0xffff0000u : 0u);
            const uint32_t m_hi = (jb + 2 * t + 8 < j_end ? 0x0000ffffu : 0u) | (jb + 2 * t + 9 < j_end ? 0xffff0000u : 0u);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                uint32_t va[4];
                ldsm_x4_t(dec_sw(vtile, vkey, 2 * mt + vhalf), va);
                if (tail) {
                    va[0] &= m_lo; va[1] &= m_lo; va[2] &= m_hi; va[3] &= m_hi;
                }
                mma_bf16(o[mt], va, pb0, pb1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // per-warp partial states -> smem [HPB][TC_NCW][D + 2]
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float lt = lh[u];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, off);
            lh[u] = lt;
        }
        __syncthreads();  // every warp finished with the ring
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int hh = 2 * t + u;
            if (hh < HPB) {
                float* row = mo + ((size_t)hh * TC_NCW + warp) * (D + 2);
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    row[16 * mt + g] = o[mt][u];
                    row[16 * mt + g + 8] = o[mt][2 + u];
                }
                if (g == 0) {
                    row[D] = mh[u];
                    row[D + 1] = lh[u];
                }
            }
        }
    }
    __syncthreads();
    merge_splits<__nv_bfloat16, D, HPB, TC_NCW, TC_NT>(mo, flag, p, dl, s, b, h0);
}

int pick_hpb(int group)
{
    if (group % 4 == 0) return 4;
    if (group % 2 == 0) return 2;
    return 1;
}

// heads per CTA for the tensor-core kernel: the MMA's N = 8 columns
int pick_hpb_tc(int group)
{
    if (group % 8 == 0) return 8;
    return pick_hpb(group);
}

int max_splits(int Lcap) { return min(kMaxSplits, max(1, (Lcap + 63) / 64)); }

// Split count and chunk length (a multiple of `gran` keys) for `units` CTAs'
// worth of (b, kv head, head group) work: enough splits to fill every SM at the
// kernel's occupancy, never more than the workspace holds.
template <class Kern>
cudaError_t plan_splits(const DecodeProblem& p, int units, Kern kern, int nthreads, int smem, int gran,
                        int* ns_out, int* chunk_out)
{
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nthreads, smem);
    if (occ < 1) occ = 1;
    // Split count with the least modelled time: ceil(CTAs / slots) waves, each
    // as long as one CTA's keys plus a fixed cost per CTA (set-up, pipeline
    // fill, partial write) worth kCtaFixedKeys keys.  A wave that leaves slots
    // empty leaves whole SMs at half occupancy for its full length, so e.g. 64
    // units on 296 slots take 9 splits (576 CTAs, two nearly full waves), not
    // 4 (256 CTAs, 40 SMs with one CTA).  Ties go to fewer splits.
    const long long slots = (long long)nsm * occ;
    const int nsmax = max(1, min(max_splits(p.Lcap), (p.L + 63) / 64));
    int ns = 1;
    double best = 0.0;
    for (int n = 1; n <= nsmax; ++n) {
        const long long waves = ((long long)units * n + slots - 1) / slots;
        const double t = (double)waves * ((double)p.L / n + kCtaFixedKeys);
        if (n == 1 || t < best * 0.999) {
            best = t;
            ns = n;
        }
    }
    int chunk = (p.L + ns - 1) / ns;
    chunk = (chunk + gran - 1) / gran * gran;
    *ns_out = (p.L + chunk - 1) / chunk;
    *chunk_out = chunk;
    return cudaSuccess;
}

template <typename T, int D, int HPB>
cudaError_t plan_scalar(const DecodeProblem& p, DecodeLaunch& dl)
{
    return plan_splits(p, p.B * p.Hkv * dl.hgroups, decode_split_kernel<T, D, HPB>, NT,
                       decode_smem_bytes<T, D, HPB>(), KROWS, &dl.n_splits, &dl.chunk);
}

template <int D, int HPB>
cudaError_t plan_tc(const DecodeProblem& p, DecodeLaunch& dl)
{
    if (p.rope_cache)
        return plan_splits(p, p.B * p.Hkv * dl.hgroups, decode_tc_kernel<D, HPB, true>, TC_NT,
                           DecTcCfg<D, HPB>::TOTAL, TC_KROWS, &dl.n_splits, &dl.chunk);
    return plan_splits(p, p.B * p.Hkv * dl.hgroups, decode_tc_kernel<D, HPB, false>, TC_NT,
                       DecTcCfg<D, HPB>::TOTAL, TC_KROWS, &dl.n_splits, &dl.chunk);
}

template <typename T, int D, int HPB>
cudaError_t launch_scalar(const DecodeProblem& p, DecodeLaunch dl, cudaStream_t st)
{
    cudaError_t e = plan_scalar<T, D, HPB>(p, dl);
    if (e != cudaSuccess) return e;
    const int units = p.B * p.Hkv * dl.hgroups;
    e = cudaMemsetAsync(dl.tickets, 0, sizeof(unsigned int) * (size_t)units, st);
    if (e != cudaSuccess) return e;
    dim3 grid(dl.n_splits, p.Hkv * dl.hgroups, p.B);
    decode_split_kernel<T, D, HPB><<<grid, NT, decode_smem_bytes<T, D, HPB>(), st>>>(p, dl);
    return cudaGetLastError();
}

typedef CUresult (*EncodeTiledFnDec)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                     const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                     const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                     CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// [B*Hkv planes][Lcap rows][d] bf16, box 64 columns x 64 keys x 1 plane, 128-byte swizzle
cudaError_t make_cache_map(CUtensorMap* m, const void* base, int d, int Lcap, int nplanes)
{
    static std::once_flag once;
    static EncodeTiledFnDec fn = nullptr;
    static cudaError_t st = cudaSuccess;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        st = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (st == cudaSuccess && q != cudaDriverEntryPointSuccess) st = cudaErrorSymbolNotFound;
        fn = reinterpret_cast<EncodeTiledFnDec>(f);
    });
    if (!fn) return st == cudaSuccess ? cudaErrorSymbolNotFound : st;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)Lcap, (cuuint64_t)nplanes};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)Lcap * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)TC_KROWS, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, int HPB>
cudaError_t launch_tc(const DecodeProblem& p, DecodeLaunch dl, cudaStream_t st)
{
    CUtensorMap tk, tv;
    cudaError_t e;
    if ((e = make_cache_map(&tk, p.kc, D, p.Lcap, p.B * p.Hkv)) != cudaSuccess) return e;
    if ((e = make_cache_map(&tv, p.vc, D, p.Lcap, p.B * p.Hkv)) != cudaSuccess) return e;
    if ((e = plan_tc<D, HPB>(p, dl)) != cudaSuccess) return e;
    const int units = p.B * p.Hkv * dl.hgroups;
    e = cudaMemsetAsync(dl.tickets, 0, sizeof(unsigned int) * (size_t)units, st);
    if (e != cudaSuccess) return e;
    dim3 grid(dl.n_splits, p.Hkv * dl.hgroups, p.B);
    if (p.rope_cache)
        decode_tc_kernel<D, HPB, true><<<grid, TC_NT, DecTcCfg<D, HPB>::TOTAL, st>>>(tk, tv, p, dl);
    else
        decode_tc_kernel<D, HPB, false><<<grid, TC_NT, DecTcCfg<D, HPB>::TOTAL, st>>>(tk, tv, p, dl);
    return cudaGetLastError();
}

// Head grouping and the split plan/launch for this problem's element type.
void set_groups(const DecodeProblem& p, jetlong_dtype dt, DecodeLaunch& dl)
{
    const int group = p.Hq / p.Hkv;
    dl.hpb = dt == JETLONG_BF16 ? pick_hpb_tc(group) : pick_hpb(group);
    dl.hgroups = group / dl.hpb;
}

template <int D>
cudaError_t dispatch(const DecodeProblem& p, jetlong_dtype dt, DecodeLaunch& dl, cudaStream_t st, bool plan_only)
{
    if (dt == JETLONG_FP32) {
        switch (dl.hpb) {
            case 4: return plan_only ? plan_scalar<float, D, 4>(p, dl) : launch_scalar<float, D, 4>(p, dl, st);
            case 2: return plan_only ? plan_scalar<float, D, 2>(p, dl) : launch_scalar<float, D, 2>(p, dl, st);
            default: return plan_only ? plan_scalar<float, D, 1>(p, dl) : launch_scalar<float, D, 1>(p, dl, st);
        }
    }
    switch (dl.hpb) {
        case 8: return plan_only ? plan_tc<D, 8>(p, dl) : launch_tc<D, 8>(p, dl, st);
        case 4: return plan_only ? plan_tc<D, 4>(p, dl) : launch_tc<D, 4>(p, dl, st);
        case 2: return plan_only ? plan_tc<D, 2>(p, dl) : launch_tc<D, 2>(p, dl, st);
        default: return plan_only ? plan_tc<D, 1>(p, dl) : launch_tc<D, 1>(p, dl, st);
    }
}

void make_div_magic(uint32_t G, uint32_t* m, uint32_t* s1, uint32_t* s2)
{
    uint32_t l = 0;
    while ((1ull << l) < G) ++l;  // ceil(log2 G)
    const uint64_t mm = ((((uint64_t)1 << 32) * (((uint64_t)1 << l) - G)) / G) + 1;
    *m = (uint32_t)mm;
    *s1 = l < 1 ? l : 1;
    *s2 = l > 1 ? l - 1 : 0;
}

}  // namespace

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Lcap, int d)
{
    // tickets are sized for the smaller of the two head groupings (more groups)
    const int hg = (Hq / Hkv) / pick_hpb(Hq / Hkv);
    size_t part = (size_t)B * Hq * max_splits(Lcap) * (d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    return part + (size_t)B * Hkv * hg * sizeof(unsigned int);
}

cudaError_t launch_decode(const DecodeProblem& p, jetlong_dtype dt, cudaStream_t s, int* nlaunch)
{
    DecodeLaunch dl{};
    set_groups(p, dt, dl);
    make_div_magic((uint32_t)p.G, &dl.div_m, &dl.div_s1, &dl.div_s2);
    size_t part = (size_t)p.B * p.Hq * max_splits(p.Lcap) * (p.d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    dl.partials = reinterpret_cast<float*>(p.workspace);
    dl.tickets = reinterpret_cast<unsigned int*>(reinterpret_cast<unsigned char*>(p.workspace) + part);
    dl.dev_error = p.dev_error;
    dl.wait_cycles = p.wait_cycles > 0 ? p.wait_cycles : kDecodeWaitCycles;
    dl.inject = p.inject;
    cudaError_t e = p.d == 64 ? dispatch<64>(p, dt, dl, s, false) : dispatch<128>(p, dt, dl, s, false);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

// ---------------------------------------------------------------------------
// Allocation-free decode.  Some callers cannot allocate device memory at all:
// code running under a caching allocator that must not grow, inside a host
// callback, or in a runtime that hands this library only the tensors of the
// step.  For them, jetlong_decode_noalloc runs the same split-K decode with its
// scratch (the split partials and merge tickets) in the fixed array below
// instead of a caller-provided workspace.  Every GPU that loads this library
// holds the array until the process exits.  All calls on a device share it and
// it keeps the last call's contents: the tickets are cleared at every call and
// the partials are always written before they are read, so stale contents are
// harmless, but two calls that overlap on the GPU (concurrent streams) race on
// it and must be serialised by the caller.
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[JETLONG_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the array, looked up once per device on the first call with
// that device current.  Host code must not use the array's name as a pointer:
// on the host it only names a stand-in for the symbol.
void* noalloc_scratch_address(cudaError_t* err)
{
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* ptr = nullptr;
        *err = cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

}  // namespace

cudaError_t launch_decode_noalloc(const DecodeProblem& p, jetlong_dtype dt, cudaStream_t s,
                                  int* nlaunch, size_t* need_bytes)
{
    *need_bytes = 0;
    cudaError_t e;
    unsigned char* scratch = static_cast<unsigned char*>(noalloc_scratch_address(&e));
    if (!scratch) return e;
    DecodeLaunch dl{};
    set_groups(p, dt, dl);
    // the split count the launch below will use (same planner, same kernel)
    e = p.d == 64 ? dispatch<64>(p, dt, dl, s, true) : dispatch<128>(p, dt, dl, s, true);
    if (e != cudaSuccess) return e;
    size_t part = (size_t)p.B * p.Hq * dl.n_splits * (p.d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    const size_t need = part + (size_t)p.B * p.Hkv * dl.hgroups * sizeof(unsigned int);
    *need_bytes = need;
    if (need > (size_t)JETLONG_DECODE_NOALLOC_SCRATCH_BYTES) return cudaErrorInvalidValue;
    make_div_magic((uint32_t)p.G, &dl.div_m, &dl.div_s1, &dl.div_s2);
    dl.partials = reinterpret_cast<float*>(scratch);
    dl.tickets = reinterpret_cast<unsigned int*>(scratch + part);
    dl.dev_error = p.dev_error;
    dl.wait_cycles = p.wait_cycles > 0 ? p.wait_cycles : kDecodeWaitCycles;
    dl.inject = p.inject;
    e = p.d == 64 ? dispatch<64>(p, dt, dl, s, false) : dispatch<128>(p, dt, dl, s, false);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

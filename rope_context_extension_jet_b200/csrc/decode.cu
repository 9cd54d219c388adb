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
#include <mutex>

#include "jl_common.cuh"
#include "jl_ptx.cuh"

namespace jl {
namespace {

constexpr int KROWS = 32;       // key rows per pipeline stage
constexpr int NCW = 4;          // consumer warps
constexpr int NT = (NCW + 1) * 32;
constexpr int kMaxSplits = 256;

struct DecodeLaunch {
    int n_splits, chunk, hgroups, hpb;
    uint32_t div_m, div_s1, div_s2;  // floor(j / G) by multiply-shift
    float* partials;                 // [B][Hq][n_splits][D + 2]
    unsigned int* tickets;           // [B][Hkv * hgroups]
    int* dev_error;
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
                if (c >= STAGES && !mbar_wait(&empty[st], ((c / STAGES) - 1) & 1)) {
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
                if (!mbar_wait(&full[c % STAGES], (c / STAGES) & 1)) record_error(dl.dev_error, 0x102);
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
            if (!mbar_wait(&full[st], (c / STAGES) & 1)) {
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
                const uint32_t pos = exact ? (uint32_t)j : div_g((uint32_t)j, dl);
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
    float* part_out = dl.partials;
    for (int e = tid; e < HPB * (D + 2); e += NT) {
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
    for (int e = tid; e < HPB * D; e += NT) {
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

int pick_hpb(int group)
{
    if (group % 4 == 0) return 4;
    if (group % 2 == 0) return 2;
    return 1;
}

int max_splits(int Lcap) { return min(kMaxSplits, max(1, (Lcap + 63) / 64)); }

template <typename T, int D, int HPB>
cudaError_t launch_typed(const DecodeProblem& p, DecodeLaunch dl, cudaStream_t st)
{
    auto kern = decode_split_kernel<T, D, HPB>;
    constexpr int smem = decode_smem_bytes<T, D, HPB>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, smem);
    if (occ < 1) occ = 1;
    const int units = p.B * p.Hkv * dl.hgroups;
    int ns = (nsm * occ) / units;
    ns = max(1, min(ns, max_splits(p.Lcap)));
    ns = min(ns, max(1, (p.L + 63) / 64));
    int chunk = (p.L + ns - 1) / ns;
    chunk = (chunk + KROWS - 1) / KROWS * KROWS;
    ns = (p.L + chunk - 1) / chunk;
    dl.n_splits = ns;
    dl.chunk = chunk;
    // tickets live after the partials; zero them for this call
    e = cudaMemsetAsync(dl.tickets, 0, sizeof(unsigned int) * (size_t)units, st);
    if (e != cudaSuccess) return e;
    dim3 grid(ns, p.Hkv * dl.hgroups, p.B);
    kern<<<grid, NT, smem, st>>>(p, dl);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_hpb(const DecodeProblem& p, DecodeLaunch dl, cudaStream_t st)
{
    switch (dl.hpb) {
        case 4: return launch_typed<T, D, 4>(p, dl, st);
        case 2: return launch_typed<T, D, 2>(p, dl, st);
        default: return launch_typed<T, D, 1>(p, dl, st);
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
    const int hg = (Hq / Hkv) / pick_hpb(Hq / Hkv);
    size_t part = (size_t)B * Hq * max_splits(Lcap) * (d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    return part + (size_t)B * Hkv * hg * sizeof(unsigned int);
}

cudaError_t launch_decode(const DecodeProblem& p, jetlong_dtype dt, cudaStream_t s, int* nlaunch)
{
    DecodeLaunch dl{};
    const int group = p.Hq / p.Hkv;
    dl.hpb = pick_hpb(group);
    dl.hgroups = group / dl.hpb;
    make_div_magic((uint32_t)p.G, &dl.div_m, &dl.div_s1, &dl.div_s2);
    size_t part = (size_t)p.B * p.Hq * max_splits(p.Lcap) * (p.d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    dl.partials = reinterpret_cast<float*>(p.workspace);
    dl.tickets = reinterpret_cast<unsigned int*>(reinterpret_cast<unsigned char*>(p.workspace) + part);
    dl.dev_error = p.dev_error;
    cudaError_t e;
    if (dt == JETLONG_FP32)
        e = p.d == 64 ? launch_hpb<float, 64>(p, dl, s) : launch_hpb<float, 128>(p, dl, s);
    else
        e = p.d == 64 ? launch_hpb<__nv_bfloat16, 64>(p, dl, s)
                      : launch_hpb<__nv_bfloat16, 128>(p, dl, s);
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

// Split count that launch_typed<T, D, HPB> will pick for this problem (same
// occupancy query and arithmetic).
template <typename T, int D, int HPB>
int planned_splits(const DecodeProblem& p, int hgroups, cudaError_t* err)
{
    auto kern = decode_split_kernel<T, D, HPB>;
    constexpr int smem = decode_smem_bytes<T, D, HPB>();
    *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (*err != cudaSuccess) return 0;
    int dev = 0, nsm = 148, occ = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, NT, smem);
    if (occ < 1) occ = 1;
    const int units = p.B * p.Hkv * hgroups;
    int ns = (nsm * occ) / units;
    ns = max(1, min(ns, max_splits(p.Lcap)));
    ns = min(ns, max(1, (p.L + 63) / 64));
    int chunk = (p.L + ns - 1) / ns;
    chunk = (chunk + KROWS - 1) / KROWS * KROWS;
    return (p.L + chunk - 1) / chunk;
}

template <typename T, int D>
int planned_splits_hpb(const DecodeProblem& p, int hpb, int hgroups, cudaError_t* err)
{
    switch (hpb) {
        case 4: return planned_splits<T, D, 4>(p, hgroups, err);
        case 2: return planned_splits<T, D, 2>(p, hgroups, err);
        default: return planned_splits<T, D, 1>(p, hgroups, err);
    }
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
    const int group = p.Hq / p.Hkv;
    dl.hpb = pick_hpb(group);
    dl.hgroups = group / dl.hpb;
    int ns;
    if (dt == JETLONG_FP32)
        ns = p.d == 64 ? planned_splits_hpb<float, 64>(p, dl.hpb, dl.hgroups, &e)
                       : planned_splits_hpb<float, 128>(p, dl.hpb, dl.hgroups, &e);
    else
        ns = p.d == 64 ? planned_splits_hpb<__nv_bfloat16, 64>(p, dl.hpb, dl.hgroups, &e)
                       : planned_splits_hpb<__nv_bfloat16, 128>(p, dl.hpb, dl.hgroups, &e);
    if (ns < 1) return e;
    size_t part = (size_t)p.B * p.Hq * ns * (p.d + 2) * sizeof(float);
    part = (part + 255) / 256 * 256;
    const size_t need = part + (size_t)p.B * p.Hkv * dl.hgroups * sizeof(unsigned int);
    *need_bytes = need;
    if (need > (size_t)JETLONG_DECODE_NOALLOC_SCRATCH_BYTES) return cudaErrorInvalidValue;
    make_div_magic((uint32_t)p.G, &dl.div_m, &dl.div_s1, &dl.div_s2);
    dl.partials = reinterpret_cast<float*>(scratch);
    dl.tickets = reinterpret_cast<unsigned int*>(scratch + part);
    dl.dev_error = p.dev_error;
    if (dt == JETLONG_FP32)
        e = p.d == 64 ? launch_hpb<float, 64>(p, dl, s) : launch_hpb<float, 128>(p, dl, s);
    else
        e = p.d == 64 ? launch_hpb<__nv_bfloat16, 64>(p, dl, s)
                      : launch_hpb<__nv_bfloat16, 128>(p, dl, s);
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

// jetlong_api.cu -- the C ABI of libjetlong: argument validation, the dynamic
// group size, RoPE phase constants, error state and dispatch to the kernels.
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740), Metodologia 1: G = max(1,
// ceil(L / w_pretrained)) from the current length; f(x) = floor(x / G).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "jl_common.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
// Per-call largest |q|, |k| of bf16 prefills (written by the range scan, read
// by the prefill kernel that follows it on the same stream).  Each call takes
// the next of kRangeSlots pairs in turn, so calls in flight on different
// streams use different words unless more than kRangeSlots prefill launches
// are queued on the device at once.
constexpr int kRangeSlots = 16384;
__device__ uint32_t g_range_slots[2 * kRangeSlots];
std::atomic<uint64_t> g_range_next{0};
// one-shot failure-detection test hook of this host thread (jetlong_debug_inject_timeout)
thread_local int g_inject_site = 0;
thread_local long long g_inject_cycles = 0;

// Takes the armed test hook, if any, for the attention launch being prepared.
void take_injection(int* site, long long* cycles)
{
    *site = g_inject_site;
    *cycles = g_inject_site ? g_inject_cycles : 0;
    g_inject_site = 0;
    g_inject_cycles = 0;
}
__device__ int g_dev_error;  // set by kernels whose bounded waits expire

int fail(int code, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int ok()
{
    g_last_error.clear();
    return JETLONG_OK;
}

int* dev_error_word(cudaError_t* err)
{
    static std::mutex mu;
    static int* cache[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_dev_error);
        if (*err != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int*>(p);
    }
    return cache[dev];
}

// Device address of the next range slot pair (looked up once per device).
uint32_t* next_range_slot(cudaError_t* err)
{
    static std::mutex mu;
    static uint32_t* base[64] = {nullptr};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    uint32_t* b;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!base[dev]) {
            void* ptr = nullptr;
            *err = cudaGetSymbolAddress(&ptr, g_range_slots);
            if (*err != cudaSuccess) return nullptr;
            base[dev] = static_cast<uint32_t*>(ptr);
        }
        b = base[dev];
    }
    return b + 2 * (g_range_next.fetch_add(1) % kRangeSlots);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Stream-ordered memory pool of this device for the pre-rotated keys of bf16
// prefill calls.  It keeps what it has reserved (release threshold: all), so
// after the first call of a given size the allocation needs no driver call;
// the memory stays reserved by the pool until the process exits.
cudaMemPool_t key_pool(cudaError_t* err)
{
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        *err = cudaMemPoolCreate(&pool, &props);
        if (*err != cudaSuccess) return nullptr;
        uint64_t keep = ~0ull;
        *err = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (*err != cudaSuccess) return nullptr;
        pools[dev] = pool;
    }
    return pools[dev];
}

int check_common(int B, int Hq, int Hkv, int d, int w0, int w_pretrained, double rope_theta,
                 float scale, jetlong_dtype dtype)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 1)
        return fail(JETLONG_ERR_INVALID_ARG, "sizes must be positive (B=%d Hq=%d Hkv=%d d=%d)", B,
                    Hq, Hkv, d);
    if (Hq % Hkv != 0)
        return fail(JETLONG_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
    if (w0 < 0) return fail(JETLONG_ERR_INVALID_ARG, "w0 must be >= 0 (got %d)", w0);
    if (w_pretrained < 1)
        return fail(JETLONG_ERR_INVALID_ARG, "w_pretrained must be >= 1 (got %d)", w_pretrained);
    if (!(rope_theta > 1.0) || !std::isfinite(rope_theta))
        return fail(JETLONG_ERR_INVALID_ARG, "rope_theta must be finite and > 1");
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(JETLONG_ERR_INVALID_ARG, "scale must be finite and > 0");
    if (dtype != JETLONG_BF16 && dtype != JETLONG_FP32)
        return fail(JETLONG_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (d != 64 && d != 128)
        return fail(JETLONG_ERR_UNSUPPORTED, "head dim d=%d not supported (64 or 128)", d);
    if (Hq > 65535 || B > 65535)
        return fail(JETLONG_ERR_UNSUPPORTED, "B and Hq must be <= 65535");
    return JETLONG_OK;
}

}  // namespace

namespace jl {

// omega_m = theta_m / (2 pi) as a 0.64 fixed-point turn fraction (theta_m <= 1,
// so omega_m < 1/(2 pi)); the scaling by 2^64 is done in long double.
void make_rope_turns(RopeTurns* t, int d, double rope_theta)
{
    const long double two_pi = 6.283185307179586476925286766559L;
    memset(t, 0, sizeof *t);
    for (int m = 0; m < d / 2; ++m) {
        const double theta_m = std::pow(rope_theta, -2.0 * (double)m / (double)d);
        const long double w = ((long double)theta_m / two_pi) * 18446744073709551616.0L;
        const uint64_t W = (uint64_t)w;
        t->hi[m] = (uint32_t)(W >> 32);
        t->lo[m] = (uint32_t)W;
    }
}

}  // namespace jl

extern "C" {

int64_t jetlong_group_size(int64_t L, int64_t w_pretrained)
{
    if (L < 0 || w_pretrained < 1) return -1;
    int64_t g = L / w_pretrained + (L % w_pretrained != 0 ? 1 : 0);
    return g < 1 ? 1 : g;
}

const char* jetlong_last_error(void) { return g_last_error.c_str(); }

uint64_t jetlong_launch_count(void) { return g_launches.load(); }

int jetlong_position_map(int32_t* d_out, int64_t L, int64_t w_pretrained, void* stream)
{
    if (!d_out) return fail(JETLONG_ERR_INVALID_ARG, "d_out is null");
    if (L < 1 || L > 2147483647LL) return fail(JETLONG_ERR_INVALID_ARG, "L out of range");
    if (w_pretrained < 1) return fail(JETLONG_ERR_INVALID_ARG, "w_pretrained must be >= 1");
    const int64_t G = jetlong_group_size(L, w_pretrained);
    int n = 0;
    cudaError_t e = jl::launch_position_map(d_out, (int)L, (int)G, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "position map launch: %s", cudaGetErrorString(e));
    return ok();
}

// vl_n > 0 (bf16 only): a variable-length batch of vl_n <= 64 sequences with
// lengths vl_lens[0..vl_n) in planes of Lcap = Cst = C rows, P = 0, in one launch.
static int prefill_entry(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                         int Hq, int Hkv, int P, int C, int Cst, int Lcap, int d, int w0,
                         int w_pretrained, double rope_theta, float scale, jetlong_dtype dtype,
                         void* stream, int window_rot = -1, int g_len = 0, int vl_n = 0,
                         const int32_t* vl_lens = nullptr, bool out_f32 = false)
{
    if (!q || !k || !v || !out) return fail(JETLONG_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(JETLONG_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (P < 0 || C < 1 || Lcap < 1 || (int64_t)P + C > Lcap)
        return fail(JETLONG_ERR_INVALID_ARG, "need P >= 0, C >= 1, P + C <= Lcap (P=%d C=%d Lcap=%d)", P,
                    C, Lcap);
    int st = check_common(B, Hq, Hkv, d, w0, w_pretrained, rope_theta, scale, dtype);
    if (st != JETLONG_OK) return st;
    cudaError_t e;
    int* derr = dev_error_word(&e);
    if (!derr) return fail(JETLONG_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));

    const int L = P + C;
    jl::PrefillProblem p{};
    p.q = q; p.k = k; p.v = v; p.out = out;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.d = d;
    p.P = P; p.C = C; p.Cst = Cst; p.Lcap = Lcap;
    p.lse = lse;
    p.window_rot = window_rot;
    p.out_f32 = out_f32 && dtype == JETLONG_BF16;
    p.w0 = w0 > L ? L : w0;  // any w0 >= L makes every causal pair local
    // G from the current length (a chunk's P + C), or from g_len when the chunk
    // is part of one whole-sequence prefill
    p.G = (int)jetlong_group_size(g_len > 0 ? g_len : L, w_pretrained);
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    jl::make_rope_turns(&p.turns, d, rope_theta);
    p.dev_error = derr;
    jl::ScanRows rows{};
    if (vl_n > 0) {
        p.vl_n = vl_n;
        rows.n = vl_n;
        rows.hq = Hq;
        rows.hkv = Hkv;
        for (int b = 0; b < vl_n; ++b) {
            p.vl_len[b] = rows.len[b] = vl_lens[b];
            p.vl_G[b] = (int)jetlong_group_size(vl_lens[b], w_pretrained);
        }
    }
    int n = 0;
    if (dtype == JETLONG_BF16) {
        // largest |q| and |k| of the rows this call uses, for the power-of-two
        // operand scales of the fp16 Q K^T (see range_scan.cu)
        uint32_t* slot = next_range_slot(&e);
        if (!slot) return fail(JETLONG_ERR_CUDA, "range slots: %s", cudaGetErrorString(e));
        e = jl::launch_range_scan(q, C, Cst, B * Hq, k, L, Lcap, B * Hkv, d, slot, (cudaStream_t)stream, &n,
                                  vl_n > 0 ? &rows : nullptr);
        g_launches += n;
        n = 0;
        if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "range scan launch: %s", cudaGetErrorString(e));
        p.range = slot;
    }
    take_injection(&p.inject, &p.wait_cycles);
    if (dtype != JETLONG_BF16) {
        // fp32: CUDA-core fp32 kernel (TF32 would miss fp32 accuracy)
        e = jl::launch_prefill_simt(p, dtype, (cudaStream_t)stream, &n);
        g_launches += n;
        if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
        return ok();
    }
    // bf16: the keys rotated once to their exact and aliased positions (fp16,
    // in stream-ordered memory of the call), then the tensor-core kernel
    cudaMemPool_t pool = key_pool(&e);
    if (!pool) return fail(JETLONG_ERR_CUDA, "key pool: %s", cudaGetErrorString(e));
    const size_t kbytes = (jl::rope_keys_bytes(p) + 255) & ~(size_t)255;
    const bool remote = jl::rope_keys_need_remote(p);
    void* kbuf = nullptr;
    e = cudaMallocFromPoolAsync(&kbuf, remote ? 2 * kbytes : kbytes, pool, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "rotated-key buffer (%zu bytes): %s",
                                      remote ? 2 * kbytes : kbytes, cudaGetErrorString(e));
    p.krot_l = kbuf;
    p.krot_r = remote ? static_cast<char*>(kbuf) + kbytes : kbuf;
    e = jl::launch_rope_keys(p, kbuf, remote ? static_cast<char*>(kbuf) + kbytes : nullptr, (cudaStream_t)stream, &n);
    if (e == cudaSuccess) e = jl::launch_prefill_tc(p, (cudaStream_t)stream, &n);
    g_launches += n;
    // freed in stream order: the memory is reused only after the kernels above
    const cudaError_t ef = cudaFreeAsync(kbuf, (cudaStream_t)stream);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
    if (ef != cudaSuccess) return fail(JETLONG_ERR_CUDA, "rotated-key buffer release: %s", cudaGetErrorString(ef));
    return ok();
}

int jetlong_prefill(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                    int Hkv, int L, int d, int w0, int w_pretrained, double rope_theta,
                    float scale, jetlong_dtype dtype, void* stream)
{
    if (L < 1) return fail(JETLONG_ERR_INVALID_ARG, "L must be >= 1 (got %d)", L);
    return prefill_entry(q, k, v, out, nullptr, B, Hq, Hkv, 0, L, L, L, d, w0, w_pretrained,
                         rope_theta, scale, dtype, stream);
}

int jetlong_prefill_chunk(const void* q, const void* kcache, const void* vcache, void* out, int B,
                          int Hq, int Hkv, int P, int C, int Lcap, int d, int w0, int w_pretrained,
                          double rope_theta, float scale, jetlong_dtype dtype, void* stream)
{
    return prefill_entry(q, kcache, vcache, out, nullptr, B, Hq, Hkv, P, C, C, Lcap, d, w0,
                         w_pretrained, rope_theta, scale, dtype, stream);
}

int jetlong_prefill_varlen(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                           int Hq, int Hkv, const int32_t* lens, int Lmax, int d, int w0,
                           int w_pretrained, double rope_theta, float scale, jetlong_dtype dtype,
                           void* stream)
{
    if (!lens) return fail(JETLONG_ERR_INVALID_ARG, "null lens");
    if (B < 1 || Lmax < 1) return fail(JETLONG_ERR_INVALID_ARG, "need B >= 1 and Lmax >= 1");
    for (int b = 0; b < B; ++b)
        if (lens[b] < 1 || lens[b] > Lmax)
            return fail(JETLONG_ERR_INVALID_ARG, "lens[%d] = %d outside [1, Lmax = %d]", b, lens[b], Lmax);
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3))
        return fail(JETLONG_ERR_INVALID_ARG, "lse must be 4-byte aligned");
    const size_t el = dtype == JETLONG_FP32 ? 4 : 2;
    // bf16: up to 64 sequences per launch (one grid over their query blocks,
    // heaviest first, each with its own length and G); fp32: one launch per
    // sequence
    const int per = dtype == JETLONG_BF16 ? 64 : 1;
    for (int b0 = 0; b0 < B; b0 += per) {
        const int nb = B - b0 < per ? B - b0 : per;
        const size_t qo = (size_t)b0 * Hq * Lmax * d * el, ko = (size_t)b0 * Hkv * Lmax * d * el;
        int st;
        if (per == 1)
            st = prefill_entry(static_cast<const char*>(q) + qo, static_cast<const char*>(k) + ko,
                               static_cast<const char*>(v) + ko, static_cast<char*>(out) + qo,
                               lse ? lse + (size_t)b0 * Hq * Lmax : nullptr, 1, Hq, Hkv, 0, lens[b0], Lmax,
                               Lmax, d, w0, w_pretrained, rope_theta, scale, dtype, stream);
        else
            st = prefill_entry(static_cast<const char*>(q) + qo, static_cast<const char*>(k) + ko,
                               static_cast<const char*>(v) + ko, static_cast<char*>(out) + qo,
                               lse ? lse + (size_t)b0 * Hq * Lmax : nullptr, nb, Hq, Hkv, 0, Lmax, Lmax, Lmax, d,
                               w0, w_pretrained, rope_theta, scale, dtype, stream, -1, 0, nb, lens + b0);
        if (st != JETLONG_OK) return st;
    }
    return ok();
}

// Workspace of the three-pass form: O_A, O_B, O_C in fp32 (the merge subtracts
// nearly equal terms, so the passes are not rounded to bf16 first), then their
// per-row LSEs (fp32), each segment 256-byte aligned.
static size_t ie_segments(int B, int Hq, int L, int d, jetlong_dtype dtype, size_t* o_bytes, size_t* l_bytes)
{
    (void)dtype;
    *o_bytes = (((size_t)B * Hq * L * d * 4) + 255) & ~(size_t)255;
    *l_bytes = (((size_t)B * Hq * L * 4) + 255) & ~(size_t)255;
    return 3 * (*o_bytes + *l_bytes);
}

size_t jetlong_prefill_ie_workspace_size(int B, int Hq, int L, int d, jetlong_dtype dtype)
{
    if (B < 1 || Hq < 1 || L < 1 || (d != 64 && d != 128)) return 0;
    if (dtype != JETLONG_BF16 && dtype != JETLONG_FP32) return 0;
    size_t ob, lb;
    return ie_segments(B, Hq, L, d, dtype, &ob, &lb);
}

int jetlong_prefill_ie(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                       int L, int d, int w0, int w_pretrained, double rope_theta, float scale,
                       jetlong_dtype dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!workspace) return fail(JETLONG_ERR_INVALID_ARG, "null workspace");
    if (!aligned16(workspace)) return fail(JETLONG_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (L < 1) return fail(JETLONG_ERR_INVALID_ARG, "L must be >= 1 (got %d)", L);
    int st = check_common(B, Hq, Hkv, d, w0, w_pretrained, rope_theta, scale, dtype);
    if (st != JETLONG_OK) return st;
    size_t ob, lb;
    const size_t need = ie_segments(B, Hq, L, d, dtype, &ob, &lb);
    if (workspace_bytes < need)
        return fail(JETLONG_ERR_INVALID_ARG, "workspace too small (%zu < %zu bytes)", workspace_bytes, need);
    char* ws = static_cast<char*>(workspace);
    void* oa = ws;
    void* obuf = ws + ob;
    void* oc = ws + 2 * ob;
    float* la = reinterpret_cast<float*>(ws + 3 * ob);
    float* lbuf = reinterpret_cast<float*>(ws + 3 * ob + lb);
    float* lc = reinterpret_cast<float*>(ws + 3 * ob + 2 * lb);
    if (w0 == 0) {
        // no window: the routed output is pass B alone (A and C hold no pairs),
        // written straight into out
        return prefill_entry(q, k, v, out, nullptr, B, Hq, Hkv, 0, L, L, L, d, 0, w_pretrained, rope_theta, scale,
                             dtype, stream);
    }
    // B: every causal pair at the aliased positions (the routed kernel with
    // w0 = 0); A: window pairs at the exact positions; C: window pairs at the
    // aliased positions; all three as fp32 rows
    st = prefill_entry(q, k, v, obuf, lbuf, B, Hq, Hkv, 0, L, L, L, d, 0, w_pretrained, rope_theta, scale,
                       dtype, stream, -1, 0, 0, nullptr, true);
    if (st != JETLONG_OK) return st;
    st = prefill_entry(q, k, v, oa, la, B, Hq, Hkv, 0, L, L, L, d, w0, w_pretrained, rope_theta, scale, dtype,
                       stream, 0, 0, 0, nullptr, true);
    if (st != JETLONG_OK) return st;
    st = prefill_entry(q, k, v, oc, lc, B, Hq, Hkv, 0, L, L, L, d, w0, w_pretrained, rope_theta, scale, dtype,
                       stream, 1, 0, 0, nullptr, true);
    if (st != JETLONG_OK) return st;
    int n = 0;
    cudaError_t e = jl::launch_ie_merge(oa, obuf, oc, la, lbuf, lc, out, (long long)B * Hq * L, d, dtype,
                                        (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
    return ok();
}

// Two non-blocking copy streams per device (host->device, device->host), made
// once and kept for the process.
static cudaError_t copy_streams(cudaStream_t* h2d, cudaStream_t* d2h)
{
    static std::mutex mu;
    static std::map<int, std::pair<cudaStream_t, cudaStream_t>> per_device;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = per_device.find(dev);
    if (it == per_device.end()) {
        cudaStream_t a = nullptr, b = nullptr;
        if ((e = cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking)) != cudaSuccess) return e;
        it = per_device.emplace(dev, std::make_pair(a, b)).first;
    }
    *h2d = it->second.first;
    *d2h = it->second.second;
    return cudaSuccess;
}

int jetlong_prefill_streamed(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                             void* q_dev, void* k_dev, void* v_dev, void* out_dev, int B, int Hq, int Hkv,
                             int L, int d, int w0, int w_pretrained, double rope_theta, float scale,
                             jetlong_dtype dtype, int nchunks, void* stream)
{
    if (!q_host || !k_host || !v_host || !out_host)
        return fail(JETLONG_ERR_INVALID_ARG, "null host tensor pointer");
    if (!q_dev || !k_dev || !v_dev || !out_dev) return fail(JETLONG_ERR_INVALID_ARG, "null device tensor pointer");
    if (L < 1 || nchunks < 1) return fail(JETLONG_ERR_INVALID_ARG, "need L >= 1 and nchunks >= 1");
    int st = check_common(B, Hq, Hkv, d, w0, w_pretrained, rope_theta, scale, dtype);
    if (st != JETLONG_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream, h2d, d2h;
    cudaError_t e = copy_streams(&h2d, &d2h);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "copy streams: %s", cudaGetErrorString(e));
    const size_t row = (size_t)d * (dtype == JETLONG_FP32 ? 4 : 2), pitch = (size_t)L * row;
    // Chunks of whole 128-row query blocks.  Nothing overlaps the first chunk's
    // copy in or the last chunk's copy out, and a chunk's compute grows with its
    // position while its copies do not, so the first and the last chunk get a
    // quarter of the blocks of each middle chunk.
    const int nblk = (L + 127) / 128;
    const int nch = nchunks < nblk ? nchunks : nblk;
    std::vector<int> first_row(nch + 1, 0);
    {
        const int edge = nch > 2 ? std::max(1, (int)std::lround((double)nblk / (2.0 + 4.0 * (nch - 2)))) : 0;
        const int mid_blocks = nblk - (nch > 2 ? 2 * edge : 0), nmid = nch > 2 ? nch - 2 : nch;
        int blk = 0;
        for (int c = 0; c < nch; ++c) {
            first_row[c] = blk * 128;
            if (nch > 2 && (c == 0 || c == nch - 1)) {
                blk += edge;
            } else {
                const int m = nch > 2 ? c - 1 : c;  // index among the middle chunks
                blk += mid_blocks / nmid + (m < mid_blocks % nmid ? 1 : 0);
            }
        }
        first_row[nch] = L;
    }
    std::vector<cudaEvent_t> ev(2 * nch + 2, nullptr);
    for (auto& x : ev)
        if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) break;
    auto release = [&] {
        for (auto& x : ev)
            if (x) cudaEventDestroy(x);  // destruction waits for pending work on the event
    };
    if (e != cudaSuccess) { release(); return fail(JETLONG_ERR_CUDA, "events: %s", cudaGetErrorString(e)); }
    auto cp = [&](void* dst, const void* src, int P, int C, int planes, cudaMemcpyKind kind, cudaStream_t s2) {
        return cudaMemcpy2DAsync(static_cast<char*>(dst) + (size_t)P * row, pitch,
                                 static_cast<const char*>(src) + (size_t)P * row, pitch, (size_t)C * row,
                                 (size_t)planes, kind, s2);
    };
    // the copies start after the work already queued on the caller's stream
    if ((e = cudaEventRecord(ev[0], cs)) == cudaSuccess && (e = cudaStreamWaitEvent(h2d, ev[0], 0)) == cudaSuccess)
        e = cudaStreamWaitEvent(d2h, ev[0], 0);
    for (int c = 0; c < nch && e == cudaSuccess && st == JETLONG_OK; ++c) {
        const int P = first_row[c], C = first_row[c + 1] - P;
        // rows [P, P + C) of every plane in; the chunk's prefill (keys [0, P + C),
        // later rows of the device buffers are outside its tensor maps); rows out
        if ((e = cp(q_dev, q_host, P, C, B * Hq, cudaMemcpyHostToDevice, h2d)) != cudaSuccess) break;
        if ((e = cp(k_dev, k_host, P, C, B * Hkv, cudaMemcpyHostToDevice, h2d)) != cudaSuccess) break;
        if ((e = cp(v_dev, v_host, P, C, B * Hkv, cudaMemcpyHostToDevice, h2d)) != cudaSuccess) break;
        if ((e = cudaEventRecord(ev[1 + 2 * c], h2d)) != cudaSuccess) break;
        if ((e = cudaStreamWaitEvent(cs, ev[1 + 2 * c], 0)) != cudaSuccess) break;
        st = prefill_entry(static_cast<char*>(q_dev) + (size_t)P * row, k_dev, v_dev,
                           static_cast<char*>(out_dev) + (size_t)P * row, nullptr, B, Hq, Hkv, P, C, L, L, d, w0,
                           w_pretrained, rope_theta, scale, dtype, stream, -1, L);
        if (st != JETLONG_OK) break;
        if ((e = cudaEventRecord(ev[2 + 2 * c], cs)) != cudaSuccess) break;
        if ((e = cudaStreamWaitEvent(d2h, ev[2 + 2 * c], 0)) != cudaSuccess) break;
        e = cp(out_host, out_dev, P, C, B * Hq, cudaMemcpyDeviceToHost, d2h);
    }
    // the caller's stream continues once the last rows are back on the host
    if (e == cudaSuccess && st == JETLONG_OK && (e = cudaEventRecord(ev[2 * nch + 1], d2h)) == cudaSuccess)
        e = cudaStreamWaitEvent(cs, ev[2 * nch + 1], 0);
    if (e != cudaSuccess || st != JETLONG_OK) {
        // a failure part-way: copies may still be queued on the library's copy
        // streams; make the caller's stream (and so anything it later frees or
        // reuses) wait for them, or wait here if even that cannot be arranged
        const std::string msg = g_last_error;
        cudaEvent_t tail[2] = {nullptr, nullptr};
        bool joined = true;
        for (int i = 0; i < 2; ++i) {
            cudaStream_t src = i == 0 ? h2d : d2h;
            joined = joined && cudaEventCreateWithFlags(&tail[i], cudaEventDisableTiming) == cudaSuccess &&
                     cudaEventRecord(tail[i], src) == cudaSuccess && cudaStreamWaitEvent(cs, tail[i], 0) == cudaSuccess;
        }
        if (!joined) {
            cudaStreamSynchronize(h2d);
            cudaStreamSynchronize(d2h);
        }
        for (auto& x : tail)
            if (x) cudaEventDestroy(x);
        g_last_error = msg;
    }
    release();
    if (st != JETLONG_OK) return st;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "streamed prefill: %s", cudaGetErrorString(e));
    return ok();
}

size_t jetlong_decode_workspace_size(int B, int Hq, int Hkv, int Lcap, int d)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Lcap < 1 || d < 1 || Hq % Hkv) return 0;
    if (d != 64 && d != 128) return 0;
    return jl::decode_workspace_bytes(B, Hq, Hkv, Lcap, d);
}

static int decode_entry(const void* q, const void* kcache, const void* vcache, void* out, int B,
                        int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
                        double rope_theta, float scale, jetlong_dtype dtype, void* workspace,
                        size_t workspace_bytes, void* stream, int rope_cache)
{
    if (!q || !kcache || !vcache || !out || !workspace)
        return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out) ||
        !aligned16(workspace))
        return fail(JETLONG_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (L < 1 || Lcap < L)
        return fail(JETLONG_ERR_INVALID_ARG, "need 1 <= L <= Lcap (L=%d Lcap=%d)", L, Lcap);
    int st = check_common(B, Hq, Hkv, d, w0, w_pretrained, rope_theta, scale, dtype);
    if (st != JETLONG_OK) return st;
    if ((int64_t)B * Hkv > 65535 * 64)
        return fail(JETLONG_ERR_UNSUPPORTED, "B * Hkv too large");
    const size_t need = jl::decode_workspace_bytes(B, Hq, Hkv, Lcap, d);
    if (workspace_bytes < need)
        return fail(JETLONG_ERR_INVALID_ARG, "workspace too small (%zu < %zu bytes)",
                    workspace_bytes, need);
    cudaError_t e;
    int* derr = dev_error_word(&e);
    if (!derr) return fail(JETLONG_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));

    jl::DecodeProblem p{};
    p.q = q; p.kc = kcache; p.vc = vcache; p.out = out;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.Lcap = Lcap; p.d = d;
    p.w0 = w0 > L ? L : w0;
    p.G = (int)jetlong_group_size(L, w_pretrained);
    p.rope_cache = rope_cache;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    jl::make_rope_turns(&p.turns, d, rope_theta);
    p.workspace = workspace;
    p.workspace_bytes = workspace_bytes;
    p.dev_error = derr;
    take_injection(&p.inject, &p.wait_cycles);
    int n = 0;
    e = jl::launch_decode(p, dtype, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_decode(const void* q, const void* kcache, const void* vcache, void* out, int B,
                   int Hq, int Hkv, int L, int Lcap, int d, int w0, int w_pretrained,
                   double rope_theta, float scale, jetlong_dtype dtype, void* workspace,
                   size_t workspace_bytes, void* stream)
{
    return decode_entry(q, kcache, vcache, out, B, Hq, Hkv, L, Lcap, d, w0, w_pretrained, rope_theta,
                        scale, dtype, workspace, workspace_bytes, stream, 0);
}

int jetlong_decode_rope_cache(const void* q, const void* kcache, const void* vcache, void* out,
                              int B, int Hq, int Hkv, int L, int Lcap, int d, int w0,
                              int w_pretrained, double rope_theta, float scale, jetlong_dtype dtype,
                              void* workspace, size_t workspace_bytes, void* stream)
{
    return decode_entry(q, kcache, vcache, out, B, Hq, Hkv, L, Lcap, d, w0, w_pretrained, rope_theta,
                        scale, dtype, workspace, workspace_bytes, stream, 1);
}

int jetlong_decode_noalloc(const void* q, const void* kcache, const void* vcache, void* out,
                           int B, int Hq, int Hkv, int L, int Lcap, int d, int w0,
                           int w_pretrained, double rope_theta, float scale, jetlong_dtype dtype,
                           void* stream)
{
    if (!q || !kcache || !vcache || !out) return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out))
        return fail(JETLONG_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if (L < 1 || Lcap < L)
        return fail(JETLONG_ERR_INVALID_ARG, "need 1 <= L <= Lcap (L=%d Lcap=%d)", L, Lcap);
    int st = check_common(B, Hq, Hkv, d, w0, w_pretrained, rope_theta, scale, dtype);
    if (st != JETLONG_OK) return st;
    if ((int64_t)B * Hkv > 65535 * 64)
        return fail(JETLONG_ERR_UNSUPPORTED, "B * Hkv too large");
    cudaError_t e;
    int* derr = dev_error_word(&e);
    if (!derr) return fail(JETLONG_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));

    jl::DecodeProblem p{};
    p.q = q; p.kc = kcache; p.vc = vcache; p.out = out;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.Lcap = Lcap; p.d = d;
    p.w0 = w0 > L ? L : w0;
    p.G = (int)jetlong_group_size(L, w_pretrained);
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    jl::make_rope_turns(&p.turns, d, rope_theta);
    p.dev_error = derr;
    take_injection(&p.inject, &p.wait_cycles);
    int n = 0;
    size_t need = 0;
    e = jl::launch_decode_noalloc(p, dtype, (cudaStream_t)stream, &n, &need);
    g_launches += n;
    if (e == cudaErrorInvalidValue && need > (size_t)JETLONG_DECODE_NOALLOC_SCRATCH_BYTES)
        return fail(JETLONG_ERR_INVALID_ARG,
                    "decode needs %zu bytes of scratch; the fixed no-alloc array holds %u "
                    "(use jetlong_decode with a workspace)",
                    need, (unsigned)JETLONG_DECODE_NOALLOC_SCRATCH_BYTES);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_selftest_wait_timeout(void* stream)
{
    cudaError_t e;
    int* derr = dev_error_word(&e);
    if (!derr) return fail(JETLONG_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
    int n = 0;
    e = jl::launch_wait_selftest(derr, 2000000ll, (cudaStream_t)stream, &n);  // ~1 ms
    g_launches += n;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_debug_inject_timeout(int site, long long wait_cycles)
{
    if (site < JETLONG_INJECT_NONE || site > JETLONG_INJECT_DECODE_COPY)
        return fail(JETLONG_ERR_INVALID_ARG, "unknown injection site %d", site);
    if (site != JETLONG_INJECT_NONE && (wait_cycles < 10000 || wait_cycles > 4000000000ll))
        return fail(JETLONG_ERR_INVALID_ARG, "wait_cycles must be in [1e4, 4e9] (got %lld)", wait_cycles);
    g_inject_site = site;
    g_inject_cycles = wait_cycles;
    return ok();
}

int jetlong_debug_rope_phase(const uint32_t* d_pos, int64_t n, int d, double rope_theta, int accurate,
                             float* d_out, void* stream)
{
    if (!d_pos || !d_out) return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (n < 0 || (d != 64 && d != 128) || !(rope_theta > 1.0) || !std::isfinite(rope_theta))
        return fail(JETLONG_ERR_INVALID_ARG, "need n >= 0, d in {64, 128}, finite rope_theta > 1");
    jl::RopeTurns turns;
    jl::make_rope_turns(&turns, d, rope_theta);
    int nl = 0;
    cudaError_t e = jl::launch_rope_phase(d_pos, n, d, turns, accurate, d_out, (cudaStream_t)stream, &nl);
    g_launches += nl;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "rope phase launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_debug_tile_plan(int P, int C, int w0, int max_kb, int32_t* d_plan, int8_t* d_cls, void* stream)
{
    if (!d_plan || !d_cls) return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (P < 0 || C < 1 || w0 < 0 || max_kb < 1 || (int64_t)P + C > 2147483647LL)
        return fail(JETLONG_ERR_INVALID_ARG, "need P >= 0, C >= 1, w0 >= 0, max_kb >= 1");
    const int L = P + C;
    int nl = 0;
    cudaError_t e = jl::launch_tile_plan(P, C, L, w0 > L ? L : w0, max_kb, d_plan, d_cls, (cudaStream_t)stream, &nl);
    g_launches += nl;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "tile plan launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_debug_ex2(const float* d_y, int64_t n, float* d_out, void* stream)
{
    if (!d_y || !d_out) return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (n < 0 || (n & 1)) return fail(JETLONG_ERR_INVALID_ARG, "need an even n >= 0 (got %lld)", (long long)n);
    int nl = 0;
    cudaError_t e = jl::launch_ex2_poly(d_y, n, d_out, (cudaStream_t)stream, &nl);
    g_launches += nl;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "ex2 launch: %s", cudaGetErrorString(e));
    return ok();
}

int jetlong_debug_rope_keys(const void* d_k, int planes, int L, int d, int G, double rope_theta, void* d_kl,
                            void* d_kr, int* h_exp, void* stream)
{
    if (!d_k || !d_kl || !h_exp) return fail(JETLONG_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(d_k) || !aligned16(d_kl) || (d_kr && !aligned16(d_kr)))
        return fail(JETLONG_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (planes < 1 || L < 1 || (d != 64 && d != 128) || G < 1 || !(rope_theta > 1.0) || !std::isfinite(rope_theta))
        return fail(JETLONG_ERR_INVALID_ARG, "need planes, L, G >= 1, d in {64, 128}, finite rope_theta > 1");
    cudaError_t e;
    uint32_t* slot = next_range_slot(&e);
    if (!slot) return fail(JETLONG_ERR_CUDA, "range slots: %s", cudaGetErrorString(e));
    jl::PrefillProblem p{};
    p.q = d_k; p.k = d_k; p.v = d_k;
    p.B = planes; p.Hq = 1; p.Hkv = 1; p.L = L; p.d = d;
    p.P = 0; p.C = L; p.Cst = L; p.Lcap = L;
    p.G = G;
    jl::make_rope_turns(&p.turns, d, rope_theta);
    p.range = slot;
    int n = 0;
    e = jl::launch_range_scan(d_k, L, L, planes, d_k, L, L, planes, d, slot, (cudaStream_t)stream, &n);
    if (e == cudaSuccess) e = jl::launch_rope_keys(p, d_kl, d_kr, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "key rotation launch: %s", cudaGetErrorString(e));
    uint32_t mag = 0;
    e = cudaMemcpyAsync(&mag, slot + 1, sizeof mag, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "key scale read: %s", cudaGetErrorString(e));
    int ex = 0;
    if (mag != 0u && mag < 0x7f80u) {
        const int biased = (int)(mag >> 7);
        ex = 13 - ((biased == 0 ? 1 : biased) - 127);
        ex = ex < -100 ? -100 : (ex > 100 ? 100 : ex);
    }
    *h_exp = ex;
    return ok();
}

int jetlong_device_status(void* stream)
{
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
    int* derr = dev_error_word(&e);
    if (!derr) return fail(JETLONG_ERR_CUDA, "device error word: %s", cudaGetErrorString(e));
    int h = 0;
    e = cudaMemcpy(&h, derr, sizeof h, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(JETLONG_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
    if (h != 0) {
        int z = 0;
        cudaMemcpy(derr, &z, sizeof z, cudaMemcpyHostToDevice);
        return fail(JETLONG_ERR_TIMEOUT, "a bounded device wait expired (code 0x%x)", h);
    }
    return ok();
}

}  // extern "C"

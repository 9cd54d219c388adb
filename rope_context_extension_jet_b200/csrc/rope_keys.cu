// rope_keys.cu -- the keys of a bf16 prefill call, rotated once per call.
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740), Metodologia 1: a key j enters a logit
// rotated either to its exact position j (local pairs) or to its aliased
// position floor(j / G) (remote pairs), whatever the query.  Each key row is
// therefore rotated here both ways, once, into two fp16 copies the prefill
// kernels load tile by tile with TMA:
//   kl[plane][j] = R(j) k[plane][j] * 2^e_k,
//   kr[plane][j] = R(floor(j / G)) k[plane][j] * 2^e_k,
// with 2^e_k the power-of-two operand scale the range scan chose for the call
// (range_exp of the second range word; the prefill's softmax divides it out).
// When G = 1 for every sequence the two copies are equal and kr is not
// written.  Rows past a sequence's length (variable-length batch) are written
// as zeros: those keys only meet masked logits.
//
// Bandwidth-bound: 2 bytes read and 2 or 4 bytes written per key element.
// One thread takes 8 rotation pairs of one row (16 bytes of each half of d),
// so a warp reads and writes whole 128-byte lines.
#include <algorithm>

#include "prefill_tc_common.cuh"

namespace jl {
namespace {

struct RopeKeysArgs {
    const __nv_bfloat16* k;
    __half* kl;
    __half* kr;          // null: G = 1 throughout, kl serves for both
    int planes, hkv;     // B * Hkv planes; kv heads per sequence
    int rows;            // rows of each output plane (the call's L)
    long long src_rows;  // row stride between input planes (Lcap)
    int G;               // group size (vl_n == 0)
    int vl_n;            // > 0: plane z belongs to sequence z / hkv of vl_len / vl_G
    int vl_len[64], vl_G[64];
    const uint32_t* range;
    RopeTurns turns;
};

template <int D>
__global__ void __launch_bounds__(256) rope_keys_kernel(const RopeKeysArgs a)
{
    constexpr int H = D / 2, CH = H / 8, RPB = 256 / CH;  // threads per row, rows per block pass
    const int c = threadIdx.x % CH;
    const float lk = tc::pow2i(tc::range_exp(tc::ld_range(a.range + 1)));
    uint32_t whi[8], wlo[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        whi[u] = a.turns.hi[c * 8 + u];
        wlo[u] = a.turns.lo[c * 8 + u];
    }
    const long long total = (long long)a.planes * a.rows;
    for (long long r = (long long)blockIdx.x * RPB + threadIdx.x / CH; r < total; r += (long long)gridDim.x * RPB) {
        const int z = (int)(r / a.rows), j = (int)(r % a.rows);
        const int seq = a.vl_n ? z / a.hkv : 0;
        const int len = a.vl_n ? a.vl_len[seq] : a.rows;
        const uint32_t G = (uint32_t)(a.vl_n ? a.vl_G[seq] : a.G);
        uint4* ol = reinterpret_cast<uint4*>(a.kl + ((size_t)z * a.rows + j) * D);
        uint4* orr = a.kr ? reinterpret_cast<uint4*>(a.kr + ((size_t)z * a.rows + j) * D) : nullptr;
        if (j >= len) {
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            ol[c] = zero;
            ol[c + CH] = zero;
            if (orr) {
                orr[c] = zero;
                orr[c + CH] = zero;
            }
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a.k + ((size_t)z * a.src_rows + j) * D);
        const uint4 xa = __ldcs(src + c), ya = __ldcs(src + c + CH);
        const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w}, yw[4] = {ya.x, ya.y, ya.z, ya.w};
        float x[8], y[8];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            x[2 * w] = bf16_lo(xw[w]);
            x[2 * w + 1] = bf16_hi(xw[w]);
            y[2 * w] = bf16_lo(yw[w]);
            y[2 * w + 1] = bf16_hi(yw[w]);
        }
        // one rotated copy: pair u of this thread at position pos
        auto rotate = [&](uint32_t pos, uint4* dst) {
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                float c0, s0, c1, s1;
                rope_cs_fast(pos, whi[2 * w], wlo[2 * w], c0, s0);
                rope_cs_fast(pos, whi[2 * w + 1], wlo[2 * w + 1], c1, s1);
                c0 *= lk; s0 *= lk; c1 *= lk; s1 *= lk;
                const float x0 = x[2 * w], x1 = x[2 * w + 1], y0 = y[2 * w], y1 = y[2 * w + 1];
                lo[w] = pack_f16x2(x0 * c0 - y0 * s0, x1 * c1 - y1 * s1);
                hi[w] = pack_f16x2(x0 * s0 + y0 * c0, x1 * s1 + y1 * c1);
            }
            dst[c] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            dst[c + CH] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        };
        rotate((uint32_t)j, ol);
        if (orr) rotate((uint32_t)j / G, orr);
    }
}

}  // namespace

size_t rope_keys_bytes(const PrefillProblem& p)
{
    return (size_t)(p.vl_n ? p.vl_n : p.B) * p.Hkv * p.L * p.d * 2;
}

bool rope_keys_need_remote(const PrefillProblem& p)
{
    if (!p.vl_n) return p.G > 1;
    for (int s = 0; s < p.vl_n; ++s)
        if (p.vl_G[s] > 1) return true;
    return false;
}

cudaError_t launch_rope_keys(const PrefillProblem& p, void* kl, void* kr, cudaStream_t s, int* nlaunch)
{
    RopeKeysArgs a{};
    a.k = reinterpret_cast<const __nv_bfloat16*>(p.k);
    a.kl = reinterpret_cast<__half*>(kl);
    a.kr = reinterpret_cast<__half*>(kr);
    a.planes = (p.vl_n ? p.vl_n : p.B) * p.Hkv;
    a.hkv = p.Hkv;
    a.rows = p.L;
    a.src_rows = p.Lcap;
    a.G = p.G;
    a.vl_n = p.vl_n;
    for (int i = 0; i < p.vl_n && i < 64; ++i) {
        a.vl_len[i] = p.vl_len[i];
        a.vl_G[i] = p.vl_G[i];
    }
    a.range = p.range;
    a.turns = p.turns;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int rpb = 256 / (p.d / 16);
    const long long total = (long long)a.planes * a.rows;
    const long long need = (total + rpb - 1) / rpb;
    const int grid = (int)std::min<long long>(need, (long long)nsm * 8);
    if (p.d == 128)
        rope_keys_kernel<128><<<grid, 256, 0, s>>>(a);
    else
        rope_keys_kernel<64><<<grid, 256, 0, s>>>(a);
    *nlaunch += 1;
    return cudaGetLastError();
}

}  // namespace jl

// ie_merge.cu -- the pages' inclusion-exclusion merge of three attention passes.
//
// "Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE"
// (gist.science/it/paper/2607.07740), Metodologia 2: the routed attention is
// assembled from three standard passes,
//   A = window pairs (i - j < w0) at the exact positions,
//   B = all causal pairs at the aliased positions,
//   C = window pairs at the aliased positions,
// whose softmax denominators e^lA, e^lB, e^lC combine exactly:
//   out = (e^lA O_A + e^lB O_B - e^lC O_C) / (e^lA + e^lB - e^lC).
// One warp per row (d / 32 elements per lane); HBM-bound.  Passes with no pairs
// (lse = -inf) drop out.
#include "jl_common.cuh"

namespace jl {
namespace {

// The pass outputs arrive in fp32 (the subtraction cancels, so their rounding
// to the output type is left to the merged value); out is T.
template <typename T>
__global__ void __launch_bounds__(256) ie_merge_kernel(const float* __restrict__ oa, const float* __restrict__ ob,
                                                       const float* __restrict__ oc, const float* __restrict__ la,
                                                       const float* __restrict__ lb, const float* __restrict__ lc,
                                                       T* __restrict__ out, long long rows, int d)
{
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float a = la[row], b = lb[row], c = lc[row];
    const float m = fmaxf(fmaxf(a, b), c);
    const float wa = a == -INFINITY ? 0.f : __expf(a - m);
    const float wb = b == -INFINITY ? 0.f : __expf(b - m);
    const float wc = c == -INFINITY ? 0.f : __expf(c - m);
    const float inv = 1.f / (wa + wb - wc);
    const size_t base = (size_t)row * d;
    for (int e = lane; e < d; e += 32) {
        float acc = 0.f;
        if (wa != 0.f) acc += wa * oa[base + e];
        if (wb != 0.f) acc += wb * ob[base + e];
        if (wc != 0.f) acc -= wc * oc[base + e];
        store_elem(out + base + e, acc * inv);
    }
}

}  // namespace

cudaError_t launch_ie_merge(const void* oa, const void* ob, const void* oc, const float* la, const float* lb,
                            const float* lc, void* out, long long rows, int d, jetlong_dtype dt,
                            cudaStream_t s, int* nlaunch)
{
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    const float* a = static_cast<const float*>(oa);
    const float* b = static_cast<const float*>(ob);
    const float* c = static_cast<const float*>(oc);
    if (dt == JETLONG_FP32)
        ie_merge_kernel<float><<<grid, 256, 0, s>>>(a, b, c, la, lb, lc, static_cast<float*>(out), rows, d);
    else
        ie_merge_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(a, b, c, la, lb, lc, static_cast<__nv_bfloat16*>(out),
                                                            rows, d);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

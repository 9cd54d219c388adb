// debug_kernels.cu -- test hooks that run the device helpers of the attention
// kernels on their own, so tests can check them against independent host
// computations: the RoPE phase (fixed-point turns, then sin / cos), the
// prefill's tile classification and per-query-block tile plan, and the
// softmax's exponential on the FMA pipe.
#include "prefill_tc_common.cuh"

namespace jl {
namespace {

// (cos, sin) of position pos[i] times theta_m for every pair m of a d-vector,
// by the accurate (sincospif) or the fast (__sincosf) form the kernels use.
__global__ void rope_phase_kernel(const uint32_t* pos, long long n, int half, const RopeTurns turns,
                                  int accurate, float* out)
{
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n * half) return;
    const long long i = e / half;
    const int m = (int)(e % half);
    float c, s;
    if (accurate)
        rope_cs_accurate(pos[i], turns.hi[m], turns.lo[m], c, s);
    else
        rope_cs_fast(pos[i], turns.hi[m], turns.lo[m], c, s);
    out[2 * e] = c;
    out[2 * e + 1] = s;
}

// One thread per query block qb of rows [P, P + C) against keys [0, L):
// plan[qb] = (nR, kE0, nkb) and cls[qb][kb] = tile_class for kb < nkb
// (cls rows hold max_kb entries; entries past nkb are left alone).
__global__ void tile_plan_kernel(int P, int C, int L, int w0, int max_kb, int32_t* plan, int8_t* cls)
{
    const int qb = blockIdx.x * blockDim.x + threadIdx.x;
    if (qb * tc::BM >= C) return;
    const int i_lo = P + qb * tc::BM;
    const tc::TilePlan tp = tc::plan_tiles(i_lo, L, w0);
    plan[3 * qb] = tp.nR;
    plan[3 * qb + 1] = tp.kE0;
    plan[3 * qb + 2] = tp.nkb;
    for (int kb = 0; kb < tp.nkb && kb < max_kb; ++kb)
        cls[(long long)qb * max_kb + kb] = (int8_t)tc::tile_class(i_lo, kb, L, w0);
}

// out[i] = ex2_poly2(y[i]) (pairs of consecutive elements; n even)
__global__ void ex2_poly_kernel(const float* y, long long n, float* out)
{
    const long long e = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (e + 1 >= n) return;
    const float2 r = tc::ex2_poly2(make_float2(y[e], y[e + 1]));
    out[e] = r.x;
    out[e + 1] = r.y;
}

}  // namespace

cudaError_t launch_ex2_poly(const float* y, long long n, float* out, cudaStream_t s, int* nlaunch)
{
    const long long pairs = n / 2;
    if (pairs <= 0) return cudaSuccess;
    ex2_poly_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(y, n, out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

cudaError_t launch_rope_phase(const uint32_t* pos, long long n, int d, const RopeTurns& turns, int accurate,
                              float* out, cudaStream_t s, int* nlaunch)
{
    const long long total = n * (d / 2);
    if (total <= 0) return cudaSuccess;
    rope_phase_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(pos, n, d / 2, turns, accurate, out);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

cudaError_t launch_tile_plan(int P, int C, int L, int w0, int max_kb, int32_t* plan, int8_t* cls, cudaStream_t s,
                             int* nlaunch)
{
    const int nqb = (C + tc::BM - 1) / tc::BM;
    tile_plan_kernel<<<(nqb + 127) / 128, 128, 0, s>>>(P, C, L, w0, max_kb, plan, cls);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

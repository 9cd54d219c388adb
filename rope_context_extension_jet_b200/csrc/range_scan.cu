// range_scan.cu -- largest |q| and |k| of a bf16 prefill call.
//
// The tensor-core prefill rounds its rotated Q K^T operands to fp16, which
// ends at 65504 (bf16 inputs reach 3.4e38).  Before the prefill kernel this
// bandwidth-bound pass reads the rows the call uses -- q rows [0, C) of every
// (b, head) plane, k rows [0, L) of every (b, kv head) plane, each a contiguous
// run of memory -- and leaves their largest magnitudes, as bf16 magnitude bits,
// in two words the prefill kernel reads to choose its power-of-two operand
// scales.  NaN inputs are ignored here (they reach the output unchanged);
// an infinite input gives the non-finite code 0x7f80 (no rescaling).
#include "jl_common.cuh"

namespace jl {
namespace {

__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// grid: (blocks per plane, planes (strided), 2 tensors); 256 threads.  With
// rows.n > 0, plane pl of q (k) belongs to sequence pl / rows.hq (pl / rows.hkv)
// and only its rows [0, rows.len[that sequence]) are read.
__global__ void __launch_bounds__(256) range_scan_kernel(const uint4* q, long long q_vecs, long long q_stride,
                                                         int q_planes, const uint4* k, long long k_vecs,
                                                         long long k_stride, int k_planes, int vpr,
                                                         const ScanRows rows, uint32_t* range)
{
    const bool is_k = blockIdx.z == 1;
    const uint4* base = is_k ? k : q;
    const long long stride = is_k ? k_stride : q_stride;
    const int planes = is_k ? k_planes : q_planes;
    uint32_t acc = 0u;
    for (int pl = blockIdx.y; pl < planes; pl += gridDim.y) {
        const long long nv = rows.n ? (long long)rows.len[pl / (is_k ? rows.hkv : rows.hq)] * vpr
                                    : (is_k ? k_vecs : q_vecs);
        const uint4* row = base + (long long)pl * stride;
        for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < nv;
             v += (long long)gridDim.x * blockDim.x) {
            const uint4 x = __ldcs(row + v);  // read once: do not keep in L2
            acc = absmax_bf16x2(acc, absmax_bf16x2(absmax_bf16x2(x.x, x.y), absmax_bf16x2(x.z, x.w)));
        }
    }
    uint32_t m = max(acc & 0x7fffu, (acc >> 16) & 0x7fffu);
    m = __reduce_max_sync(0xffffffffu, m);
    __shared__ uint32_t wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = wm[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) b = max(b, wm[w]);
        if (b) atomicMax(range + (is_k ? 1 : 0), b);
    }
}

}  // namespace

cudaError_t launch_range_scan(const void* q, int C, int Cst, int q_planes, const void* k, int L, int Lcap,
                              int k_planes, int d, uint32_t* range, cudaStream_t s, int* nlaunch,
                              const ScanRows* rows)
{
    cudaError_t e = cudaMemsetAsync(range, 0, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    // rows of d bf16 values are d / 8 16-byte vectors (d is 64 or 128)
    const long long vpr = d / 8;
    const long long q_vecs = (long long)C * vpr, k_vecs = (long long)L * vpr;
    const long long most = q_vecs > k_vecs ? q_vecs : k_vecs;
    // enough blocks per plane to cover ~8 vectors per thread, the whole grid a
    // few waves of the 148 SMs
    long long bx = (most + 256 * 8 - 1) / (256 * 8);
    const int planes = q_planes > k_planes ? q_planes : k_planes;
    const int by = planes < 65535 ? planes : 65535;
    const long long cap = (4 * 148 * 8 + by - 1) / by;
    if (bx > cap) bx = cap;
    if (bx < 1) bx = 1;
    dim3 grid((unsigned)bx, (unsigned)by, 2);
    ScanRows r{};
    if (rows) r = *rows;
    range_scan_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(q), q_vecs, (long long)Cst * vpr, q_planes,
                                           static_cast<const uint4*>(k), k_vecs, (long long)Lcap * vpr, k_planes,
                                           (int)vpr, r, range);
    e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

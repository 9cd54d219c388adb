// position_map.cu -- export of the aliased position map f(x) = floor(x / G)
// ("Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE",
// Metodologia 1, the floor-division remote mapping).
#include "jl_common.cuh"
#include "jl_ptx.cuh"

namespace jl {
namespace {

__global__ void position_map_kernel(int32_t* out, int L, int G)
{
    for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < L; x += gridDim.x * blockDim.x)
        out[x] = x / G;
}

// Failure-detection self test: one CTA waits on an mbarrier that nothing
// arrives at, with the kernels' bounded-wait helper and a short limit; the wait
// expires, the kernel records `code` in the error word and returns normally.
__global__ void wait_timeout_selftest_kernel(int* dev_error, long long limit_cycles, int code)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit_cycles)) record_error(dev_error, code);
}

}  // namespace

cudaError_t launch_wait_selftest(int* dev_error, long long limit_cycles, cudaStream_t s, int* nlaunch)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(dev_error, limit_cycles, 0x7e57);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

cudaError_t launch_position_map(int32_t* out, int L, int G, cudaStream_t s, int* nlaunch)
{
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    int blocks = (L + 255) / 256;
    if (blocks > nsm * 8) blocks = nsm * 8;
    position_map_kernel<<<blocks, 256, 0, s>>>(out, L, G);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) *nlaunch += 1;
    return e;
}

}  // namespace jl

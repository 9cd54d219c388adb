// position_map.cu -- export of the aliased position map f(x) = floor(x / G)
// ("Jet-Long: Efficient Long-Context Extension with Dynamic Bifocal RoPE",
// Metodologia 1, the floor-division remote mapping).
#include "jl_common.cuh"

namespace jl {
namespace {

__global__ void position_map_kernel(int32_t* out, int L, int G)
{
    for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < L; x += gridDim.x * blockDim.x)
        out[x] = x / G;
}

}  // namespace

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

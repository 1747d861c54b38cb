// GPU executor of the layer backward: each step of bwd::run_backward runs as
// one grid-stride kernel of 256 threads, one output element per iteration.
#include "backward.cuh"

namespace moe {
namespace {

template <class F>
__global__ void __launch_bounds__(256) for_each_kernel(size_t n, F f) {
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        f(i);
}

struct GpuExec {
    cudaStream_t st;
    cudaError_t err;
    int launches;
    template <class F> void run(size_t n, const F& f) {
        if (err != cudaSuccess || n == 0) return;
        size_t blocks = (n + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;       // 16 blocks per SM, then the loop strides
        for_each_kernel<F><<<static_cast<unsigned>(blocks), 256, 0, st>>>(n, f);
        ++launches;
        err = cudaGetLastError();
    }
};

}  // namespace

size_t backward_ws_bytes(const Dims& dm) { return bwd::bwd_layout(dm).total; }

cudaError_t launch_backward(const Dims& dm, float lam, const moe_backward_io& io, void* bws,
                            cudaStream_t st) {
    GpuExec ex{st, cudaSuccess, 0};
    bwd::run_backward(ex, dm, lam, io, bws);
    count_launches(ex.launches);
    return ex.err;
}

}  // namespace moe

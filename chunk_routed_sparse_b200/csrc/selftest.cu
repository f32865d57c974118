// Diagnostic of the bounded device-side waits (no counterpart in the pages).
//
// The warp-specialised kernels wait on mbarriers with a time limit (2 s);
// when a wait gives up they record ERR_TIMEOUT and a site code in a device
// error word and return instead of hanging. This kernel runs that same wait
// on an mbarrier nothing ever arrives at, so a test can check the reporting
// path and that the context stays usable afterwards - without faulting or
// hanging the GPU.
#include "pipeline.cuh"

namespace moc {
namespace {

constexpr int kSelftestSite = 99;

__global__ void selftest_wait_kernel(int32_t* word) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bar(smem_u32(&bar), 0, &abort_flag, word, kSelftestSite);
}

}  // namespace
}  // namespace moc

extern "C" moc_status moc_selftest_bounded_wait(int32_t* dev_word, moc_stream_t stream) {
    if (!dev_word || (reinterpret_cast<uintptr_t>(dev_word) & 3)) return MOC_ERR_INVALID_ARG;
    moc::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_word);
    return cudaGetLastError() == cudaSuccess ? MOC_OK : MOC_ERR_CUDA;
}

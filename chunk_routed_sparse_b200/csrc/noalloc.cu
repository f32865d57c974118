// moc_attention_fwd_static: the attention stage without a caller workspace.
//
// Some callers cannot hand the library a device workspace: they may not call
// cudaMalloc at all (an inference-server plugin that is given only its input
// and output buffers, a real-time loop that must never take the driver's
// allocation path, which can synchronise the device, or a library embedded in
// a host application that budgets every device byte itself up front).
// This entry point runs the same three stages as moc_attention_fwd (query
// lists, attend, merge) on a fixed scratch area that lives in the library
// itself: a file-scope static __device__ array of kStaticScratchBytes. Every
// GPU that loads the library holds that array until the process exits.
//
// The array's host-side name is only a stand-in; its device address comes from
// cudaGetSymbolAddress, looked up once per device (with that device current)
// on the first call made on it. The scratch is shared by every call and keeps
// the last call's contents; the stages clear what must start at zero (the
// error word and the work counter) themselves. Two calls that overlap on the
// GPU (different streams, or different host threads) race on the scratch.
#include <mutex>

#include "moc_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

void* g_scratch_dev[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

}  // namespace

namespace {

// The static scratch's device address on the current device (looked up once
// per device, with that device current). Returns MOC_OK and sets *dev.
moc_status static_scratch(void** ptr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOC_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOC_ERR_UNSUPPORTED;
    std::call_once(g_scratch_once[dev], [dev] {
        g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_dev[dev], g_static_scratch);
    });
    if (g_scratch_err[dev] != cudaSuccess || !g_scratch_dev[dev]) return MOC_ERR_CUDA;
    *ptr = g_scratch_dev[dev];
    return MOC_OK;
}

}  // namespace

extern "C" moc_status moc_attention_fwd_static(const moc_layout* lay, int B, int H, int d,
                                               const void* Q, const void* K, const void* V,
                                               const int32_t* sel, int k, float softmax_scale,
                                               void* O, float* lse, moc_stream_t stream) {
    if (!lay || B < 0 || H < 0 || (d != 64 && d != 128) || k < 0 || k > moc::kMaxK)
        return MOC_ERR_INVALID_ARG;
    if (lay->device < 0) return MOC_ERR_INVALID_ARG;
    // the problem's scratch must fit the static area
    if (moc::plan_workspace(lay, B, H, d, k).total > kStaticScratchBytes)
        return MOC_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    const moc_status st = static_scratch(&scratch);
    if (st != MOC_OK) return st;
    return moc_attention_fwd(lay, B, H, d, Q, K, V, sel, k, softmax_scale, O, lse, scratch,
                             kStaticScratchBytes, stream);
}

// The device error word of the calls above lives at the head of the static
// scratch, whose address a caller cannot see; this reads and clears it on the
// current device exactly as moc_check_device_error does for a caller workspace
// (a later moc_attention_fwd_static call clears the word when it starts, so
// check it after the call whose errors matter and before the next one).
extern "C" moc_status moc_check_device_error_static(int32_t* detail, moc_stream_t stream) {
    void* scratch = nullptr;
    const moc_status st = static_scratch(&scratch);
    if (st != MOC_OK) return st;
    return moc_check_device_error(scratch, kStaticScratchBytes, detail, stream);
}

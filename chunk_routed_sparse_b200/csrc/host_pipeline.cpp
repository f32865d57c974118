// Whole forward pass on host buffers: pooling, routing, query lists, attention
// and merge for chunks of consecutive (b, h) slices, with the copies of one
// chunk overlapping the compute of its neighbours.
//
// Every stage of the method is independent per (batch, head) ("Mixture of
// Contexts for Long Video Generation | Summary" §3.1: routing and attention are
// per head; the jxzklqfsx.com write-up, "計算效率": all operations are
// head-independent), so a chunk of heads is a complete problem of its own. Three
// streams: an upload stream copies chunk c+1's Q, K, V into one of two input
// stages while the caller's stream computes chunk c from the other, and a
// download stream returns chunk c-1's O, lse and sel from one of two output
// stages. Events order the reuse of each stage. Nothing is allocated on the
// device: the caller passes one buffer of moc_forward_host_device_bytes().
#include <cstring>
#include <vector>

#include "moc_internal.h"

namespace {

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct HostPlan {
    int hc = 0;                  // (b, h) slices per chunk
    size_t qkv = 0;              // bytes of one of Q, K, V for a chunk
    size_t o = 0, lse = 0, sel = 0, kbar = 0, ws = 0;
    size_t in_stage = 0, out_stage = 0;
    size_t off_in[2] = {0, 0}, off_out[2] = {0, 0}, off_kbar = 0, off_ws = 0, total = 0;
};

bool plan_host(const moc_layout* lay, int BH, int d, int k, int heads_per_chunk, HostPlan* p) {
    if (BH <= 0) return false;
    // default: twelve chunks (eight-shot scene, 24 heads: two per chunk measured best -
    // 69.8 ms end to end against 72.5 with three and 80.3 with six; smaller chunks
    // shorten the pipeline's fill and drain, larger ones the per-chunk kernel tails)
    int hc = heads_per_chunk > 0 ? heads_per_chunk : (BH + 11) / 12;
    if (hc > BH) hc = BH;
    p->hc = hc;
    const size_t L = size_t(lay->L), C = size_t(lay->C);
    p->qkv = align256(size_t(hc) * L * size_t(d) * 2);
    p->o = p->qkv;
    p->lse = align256(size_t(hc) * L * sizeof(float));
    p->sel = align256(size_t(hc) * L * size_t(k > 0 ? k : 1) * sizeof(int32_t));
    p->kbar = align256(size_t(hc) * C * size_t(d) * sizeof(float));
    p->ws = align256(moc::plan_workspace(lay, 1, hc, d, k).total);
    p->in_stage = 3 * p->qkv;
    p->out_stage = p->o + p->lse + p->sel;
    size_t off = 0;
    for (int s = 0; s < 2; ++s) { p->off_in[s] = off; off += p->in_stage; }
    for (int s = 0; s < 2; ++s) { p->off_out[s] = off; off += p->out_stage; }
    p->off_kbar = off; off += p->kbar;
    p->off_ws = off; off += p->ws;
    p->total = off;
    return true;
}

// Streams and events of one call, released on every exit path.
struct Pipe {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, in_ready[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr},
                out_free[2] = {nullptr, nullptr}, done = nullptr;
    bool ok = true;
    Pipe() {
        ok = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) == cudaSuccess;
        cudaEvent_t* evs[] = {&start, &in_ready[0], &in_ready[1], &computed[0], &computed[1],
                              &out_free[0], &out_free[1], &done};
        for (cudaEvent_t* e : evs)
            ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    }
    ~Pipe() {
        if (up) cudaStreamSynchronize(up);
        if (down) cudaStreamSynchronize(down);
        cudaEvent_t evs[] = {start, in_ready[0], in_ready[1], computed[0], computed[1],
                             out_free[0], out_free[1], done};
        for (cudaEvent_t e : evs)
            if (e) cudaEventDestroy(e);
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
    }
};

}  // namespace

extern "C" size_t moc_forward_host_device_bytes(const moc_layout* lay, int B, int H, int d, int k,
                                                int heads_per_chunk) {
    if (!lay || B < 0 || H < 0 || (d != 64 && d != 128) || k < 0 || k > moc::kMaxK) return 0;
    HostPlan p;
    if (!plan_host(lay, B * H, d, k, heads_per_chunk, &p)) return 0;
    return p.total;
}

extern "C" moc_status moc_forward_host(const moc_layout* lay, int B, int H, int d, int k, int causal,
                                       float scale, const void* Q, const void* K, const void* V,
                                       void* O, float* lse, int32_t* sel, void* dev,
                                       size_t dev_bytes, int heads_per_chunk, moc_stream_t stream) {
    if (!lay || lay->device < 0 || !lay->dev_block) return MOC_ERR_INVALID_ARG;
    if (B < 0 || H < 0 || int64_t(B) * H > 65535) return MOC_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MOC_ERR_INVALID_ARG;
    if (k < 0 || k > moc::kMaxK) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    const int BH = B * H;
    if (BH == 0) return MOC_OK;
    if (!Q || !K || !V || !O || !dev || (reinterpret_cast<uintptr_t>(dev) & 255))
        return MOC_ERR_INVALID_ARG;
    HostPlan p;
    if (!plan_host(lay, BH, d, k, heads_per_chunk, &p)) return MOC_ERR_INVALID_ARG;
    if (dev_bytes < p.total) return MOC_ERR_WORKSPACE_TOO_SMALL;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOC_ERR_CUDA;
    if (cur != lay->device) return MOC_ERR_INVALID_ARG;

    Pipe pipe;
    if (!pipe.ok) return MOC_ERR_CUDA;
    cudaStream_t cs = (cudaStream_t)stream;
    char* base = static_cast<char*>(dev);
    const size_t L = size_t(lay->L);
    const size_t row_bytes = L * size_t(d) * 2;  // one (b, h) slice of Q, K, V or O
    // chunk boundaries: the first and the last chunk are half size, so that the
    // pipeline fills (first upload) and drains (last download) sooner
    std::vector<int> bounds{0};
    {
        const int half = p.hc > 1 ? p.hc / 2 : 1;
        int h = half < BH ? half : BH;
        bounds.push_back(h);
        const int last = (BH - h) < half ? (BH - h) : half;
        while (h < BH - last) {
            h += (BH - last - h) < p.hc ? (BH - last - h) : p.hc;
            bounds.push_back(h);
        }
        if (last > 0) bounds.push_back(BH);
    }
    const int nch = int(bounds.size()) - 1;
    auto ck = [](cudaError_t e) { return e == cudaSuccess; };

    // the copies start after whatever the caller queued on its stream before this call
    if (!ck(cudaEventRecord(pipe.start, cs)) || !ck(cudaStreamWaitEvent(pipe.up, pipe.start, 0)))
        return MOC_ERR_CUDA;
    void* ws = base + p.off_ws;
    const size_t ws_bytes = p.ws;
    for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        const int h0 = bounds[c], nh = bounds[c + 1] - bounds[c];
        char* in = base + p.off_in[s];
        char* dq = in;
        char* dk = in + p.qkv;
        char* dv = in + 2 * p.qkv;
        char* out = base + p.off_out[s];
        char* dO = out;
        float* dL = reinterpret_cast<float*>(out + p.o);
        int32_t* dS = reinterpret_cast<int32_t*>(out + p.o + p.lse);
        float* kbar = reinterpret_cast<float*>(base + p.off_kbar);
        const size_t nbytes = size_t(nh) * row_bytes;
        // upload: input stage s is free once chunk c-2 has been computed
        if (!ck(cudaStreamWaitEvent(pipe.up, pipe.computed[s], 0)) ||
            !ck(cudaMemcpyAsync(dq, static_cast<const char*>(Q) + size_t(h0) * row_bytes, nbytes,
                                cudaMemcpyHostToDevice, pipe.up)) ||
            !ck(cudaMemcpyAsync(dk, static_cast<const char*>(K) + size_t(h0) * row_bytes, nbytes,
                                cudaMemcpyHostToDevice, pipe.up)) ||
            !ck(cudaMemcpyAsync(dv, static_cast<const char*>(V) + size_t(h0) * row_bytes, nbytes,
                                cudaMemcpyHostToDevice, pipe.up)) ||
            !ck(cudaEventRecord(pipe.in_ready[s], pipe.up)))
            return MOC_ERR_CUDA;
        // compute chunk c on the caller's stream once its inputs are in and output
        // stage s has been copied out (chunk c-2)
        if (!ck(cudaStreamWaitEvent(cs, pipe.in_ready[s], 0)) || !ck(cudaStreamWaitEvent(cs, pipe.out_free[s], 0)))
            return MOC_ERR_CUDA;
        moc_status st = moc_pool_keys(lay, 1, nh, d, dk, kbar, stream);
        if (st == MOC_OK && k > 0) st = moc_route(lay, 1, nh, d, dq, kbar, k, causal, dS, stream);
        if (st == MOC_OK)
            st = moc_attention_fwd(lay, 1, nh, d, dq, dk, dv, k > 0 ? dS : nullptr, k, scale, dO, dL, ws,
                                   ws_bytes, stream);
        if (st != MOC_OK) return st;
        if (!ck(cudaEventRecord(pipe.computed[s], cs))) return MOC_ERR_CUDA;
        // download chunk c
        if (!ck(cudaStreamWaitEvent(pipe.down, pipe.computed[s], 0)) ||
            !ck(cudaMemcpyAsync(static_cast<char*>(O) + size_t(h0) * row_bytes, dO, nbytes,
                                cudaMemcpyDeviceToHost, pipe.down)))
            return MOC_ERR_CUDA;
        if (lse && !ck(cudaMemcpyAsync(lse + size_t(h0) * L, dL, size_t(nh) * L * sizeof(float),
                                       cudaMemcpyDeviceToHost, pipe.down)))
            return MOC_ERR_CUDA;
        if (sel && k > 0 &&
            !ck(cudaMemcpyAsync(sel + size_t(h0) * L * size_t(k), dS, size_t(nh) * L * size_t(k) * sizeof(int32_t),
                                cudaMemcpyDeviceToHost, pipe.down)))
            return MOC_ERR_CUDA;
        if (!ck(cudaEventRecord(pipe.out_free[s], pipe.down))) return MOC_ERR_CUDA;
    }
    // the caller's stream continues after the last download; the host outputs
    // are complete when this call returns
    if (!ck(cudaEventRecord(pipe.done, pipe.down)) || !ck(cudaStreamWaitEvent(cs, pipe.done, 0)) ||
        !ck(cudaStreamSynchronize(pipe.down)) || !ck(cudaStreamSynchronize(cs)))
        return MOC_ERR_CUDA;
    // a bounded wait that gave up or a failed device check in any chunk
    int32_t detail = 0;
    moc_status st = moc_check_device_error(ws, ws_bytes, &detail, stream);
    if (st != MOC_OK) return st;
    return moc_layout_device_error(lay, &detail, stream);
}

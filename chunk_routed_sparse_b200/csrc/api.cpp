// C-ABI entry points: argument validation, workspace carve-up and kernel
// launches. Every compute call is asynchronous on the caller's stream and
// allocates nothing.
#include <atomic>
#include <cmath>
#include <cstring>

#include "moc_internal.h"

namespace {

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

moc_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOC_OK : MOC_ERR_CUDA; }

// Checks shared by the compute calls.
moc_status check_common(const moc_layout* lay, int B, int H, int d, int k) {
    if (!lay) return MOC_ERR_INVALID_ARG;
    if (lay->device < 0 || !lay->dev_block) return MOC_ERR_INVALID_ARG;  // host-only layout
    if (B < 0 || H < 0 || int64_t(B) * H > 65535) return MOC_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return MOC_ERR_INVALID_ARG;
    if (k < 0 || k > moc::kMaxK) return MOC_ERR_INVALID_ARG;
    const int64_t BH = int64_t(B) * H;
    if (BH * lay->L * (k > 0 ? k : 1) >= (int64_t(1) << 31)) return MOC_ERR_UNSUPPORTED;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOC_ERR_CUDA;
    if (cur != lay->device) return MOC_ERR_INVALID_ARG;
    return MOC_OK;
}

}  // namespace

namespace {

std::atomic<int> g_sched_ctas{0}, g_sched_reverse{0}, g_attend_kernel{0};
// the attention stage runs on CTA pairs where that kernel exists (d = 128)
constexpr bool kPairByDefault = false;

}  // namespace

namespace moc {

int attend_kernel_choice() { return g_attend_kernel.load(std::memory_order_relaxed); }

AttendSchedule attend_schedule() {
    AttendSchedule s;
    s.n_ctas = g_sched_ctas.load(std::memory_order_relaxed);
    s.reverse = g_sched_reverse.load(std::memory_order_relaxed);
    return s;
}

WsPlan plan_workspace(const moc_layout* lay, int B, int H, int d, int k) {
    WsPlan p;
    const size_t BH = size_t(B) * H, L = size_t(lay->L), C = size_t(lay->C), S = size_t(k) + 1;
    p.nblk = int((L + kQlistBlock - 1) / kQlistBlock);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    p.hdr = take(64 * sizeof(int32_t));
    p.blk_count = take(BH * size_t(p.nblk) * C * sizeof(int32_t));
    p.qoff = take((BH * C + 1) * sizeof(int32_t));
    p.tile_off = take((BH * C + 1) * sizeof(int32_t));
    p.tile2_off = take((BH * C + 1) * sizeof(int32_t));
    p.qlist = take(BH * L * size_t(k) * sizeof(int32_t));
    p.lse_p = take(BH * L * S * sizeof(float));
    p.o_p = take(BH * L * S * size_t(d) * sizeof(float));
    p.total = off;
    return p;
}

WsPlan plan_workspace_bwd(const moc_layout* lay, int B, int H, int d, int k) {
    WsPlan p = plan_workspace(lay, B, H, d, k);
    const size_t BH = size_t(B) * H, L = size_t(lay->L), S = size_t(k) + 1;
    size_t off = p.lse_p;
    p.lse_p = off;  // D = dO . o per row
    off += align256(BH * L * sizeof(float));
    p.o_p = off;    // dQ partial rows
    off += align256(BH * L * S * size_t(d) * sizeof(float));
    p.total = off;
    return p;
}

}  // namespace moc

extern "C" const char* moc_status_string(moc_status s) {
    switch (s) {
        case MOC_OK: return "ok";
        case MOC_ERR_INVALID_ARG: return "invalid argument";
        case MOC_ERR_LAYOUT: return "invalid layout description";
        case MOC_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOC_ERR_CUDA: return "CUDA error";
        case MOC_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MOC_ERR_UNSUPPORTED: return "unsupported problem size";
        case MOC_ERR_DEVICE_CHECK: return "device-side consistency check failed";
    }
    return "unknown status";
}

extern "C" moc_status moc_pool_keys(const moc_layout* lay, int B, int H, int d, const void* K,
                                    float* Kbar, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, 0);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    if (!K || !Kbar || !aligned16(K) || !aligned16(Kbar)) return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_pool(lay->dv, B * H, d, K, Kbar, (cudaStream_t)stream));
}

extern "C" moc_status moc_route(const moc_layout* lay, int B, int H, int d, const void* Q,
                                const float* Kbar, int k, int causal, int32_t* sel,
                                moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0 || k == 0) return MOC_OK;
    if (!Q || !Kbar || !sel || !aligned16(Q) || !aligned16(Kbar) ||
        (reinterpret_cast<uintptr_t>(sel) & 3))
        return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_route(lay->dv, B * H, lay->total_rtiles, d, Q, Kbar, k,
                                         causal ? 1 : 0, lay->max_cand, nullptr, sel,
                                         (cudaStream_t)stream));
}

extern "C" moc_status moc_outer_route(const moc_layout* lay, int B, int H, int d, const float* Qbar,
                                      const float* Kbar, int M, int causal, uint64_t* seg_mask,
                                      moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, 0);
    if (st != MOC_OK) return st;
    if (M < 0) return MOC_ERR_INVALID_ARG;
    if (lay->n_shots > 64) return MOC_ERR_UNSUPPORTED;  // one 64-bit mask per block
    if (B * H == 0) return MOC_OK;
    if (!Qbar || !Kbar || !seg_mask || (reinterpret_cast<uintptr_t>(Qbar) & 15) ||
        (reinterpret_cast<uintptr_t>(Kbar) & 15) || (reinterpret_cast<uintptr_t>(seg_mask) & 7))
        return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_outer(lay->dv, B * H, d, Qbar, Kbar, M, causal ? 1 : 0, seg_mask,
                                         (cudaStream_t)stream));
}

extern "C" moc_status moc_route_masked(const moc_layout* lay, int B, int H, int d, const void* Q,
                                       const float* Kbar, int k, int causal, const uint64_t* seg_mask,
                                       int32_t* sel, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (lay->n_shots > 64) return MOC_ERR_UNSUPPORTED;
    if (B * H == 0 || k == 0) return MOC_OK;
    if (!Q || !Kbar || !sel || !seg_mask || !aligned16(Q) || !aligned16(Kbar) ||
        (reinterpret_cast<uintptr_t>(sel) & 3) || (reinterpret_cast<uintptr_t>(seg_mask) & 7))
        return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_route(lay->dv, B * H, lay->total_rtiles, d, Q, Kbar, k,
                                         causal ? 1 : 0, lay->max_cand, seg_mask, sel,
                                         (cudaStream_t)stream));
}

extern "C" moc_status moc_route_perturb(const moc_layout* lay, int B, int H, int k, int causal,
                                        const int32_t* sel, const uint32_t* rnd, float p_max,
                                        float lambda, int m_max, int32_t* sel_out, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, 128, k);
    if (st != MOC_OK) return st;
    if (m_max < 0 || k + m_max > moc::kMaxK || k + m_max == 0) return MOC_ERR_INVALID_ARG;
    if (!(p_max >= 0.0f && p_max <= 1.0f) || !(lambda >= 0.0f) || !std::isfinite(lambda))
        return MOC_ERR_INVALID_ARG;
    if (B * H == 0) return MOC_OK;
    if (int64_t(B) * H * lay->L * (2 + k + m_max) >= (int64_t(1) << 31)) return MOC_ERR_UNSUPPORTED;
    if ((k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) || !rnd ||
        (reinterpret_cast<uintptr_t>(rnd) & 3) || !sel_out || (reinterpret_cast<uintptr_t>(sel_out) & 3))
        return MOC_ERR_INVALID_ARG;
    // F(i) accumulated in double from p_0 = exp(-lambda), p_i = p_{i-1} lambda / i
    moc::PoissonThresholds thr{};
    const double lam = double(lambda);
    double p = std::exp(-lam), cdf = p;
    for (int i = 0; i < m_max; ++i) {
        if (i > 0) {
            p = p * lam / double(i);
            cdf = cdf + p;
        }
        const double v = std::floor(cdf * 4294967296.0);
        thr.t[i] = v >= 4294967296.0 ? (uint64_t(1) << 32) : uint64_t(v);
    }
    return cuda_status(moc::launch_perturb(lay->dv, B * H, k, m_max, causal ? 1 : 0, sel, rnd, p_max, thr,
                                           sel_out, (cudaStream_t)stream));
}

extern "C" size_t moc_attention_workspace_bytes(const moc_layout* lay, int B, int H, int d, int k) {
    if (!lay || B < 0 || H < 0 || (d != 64 && d != 128) || k < 0 || k > moc::kMaxK) return 0;
    return moc::plan_workspace(lay, B, H, d, k).total;
}

namespace {

moc_status check_ws(const moc_layout* lay, int B, int H, int d, int k, void* ws, size_t ws_bytes,
                    moc::WsPlan* p) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOC_ERR_INVALID_ARG;
    *p = moc::plan_workspace(lay, B, H, d, k);
    if (ws_bytes < p->total) return MOC_ERR_WORKSPACE_TOO_SMALL;
    return MOC_OK;
}

}  // namespace

extern "C" moc_status moc_build_qlists(const moc_layout* lay, int B, int H, int k,
                                       const int32_t* sel, void* ws, size_t ws_bytes,
                                       moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, 128, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    // the query lists do not depend on d; plan with the smallest d for the check
    if ((st = check_ws(lay, B, H, 64, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_qlists(lay->dv, B * H, k, sel, static_cast<char*>(ws), p,
                                          (cudaStream_t)stream));
}

extern "C" moc_status moc_attend_partials(const moc_layout* lay, int B, int H, int d, const void* Q,
                                          const void* K, const void* V, int k, float scale,
                                          void* ws, size_t ws_bytes, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    if ((st = check_ws(lay, B, H, d, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (!Q || !K || !V || !aligned16(Q) || !aligned16(K) || !aligned16(V)) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    const int variant = moc::attend_kernel_choice();
    if (variant == 2 && !moc::attend_pair_supported(d)) return MOC_ERR_INVALID_ARG;
    if (variant == 2 || (variant == 0 && kPairByDefault && moc::attend_pair_supported(d)))
        return cuda_status(moc::launch_attend_pair(lay->dv, B * H, d, Q, K, V, k, scale,
                                                   int64_t(B) * H * lay->total_atiles2, static_cast<char*>(ws), p,
                                                   (cudaStream_t)stream));
    const int64_t n_anchor = int64_t(B) * H * lay->total_atiles;
    return cuda_status(moc::launch_attend_tc(lay->dv, B * H, d, Q, K, V, k, scale, n_anchor,
                                             static_cast<char*>(ws), p, (cudaStream_t)stream));
}

extern "C" moc_status moc_attend_merged(const moc_layout* lay, int B, int H, int d, const void* Q,
                                        const void* K, const void* V, const int32_t* sel, int k, float scale,
                                        void* O, float* lse, void* ws, size_t ws_bytes, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    if ((st = check_ws(lay, B, H, d, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return MOC_ERR_INVALID_ARG;
    if (k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) return MOC_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    const int64_t n_anchor = int64_t(B) * H * lay->total_atiles;
    return cuda_status(moc::launch_attend_merged(lay->dv, B * H, d, Q, K, V, k, scale, n_anchor,
                                                 static_cast<char*>(ws), p, sel, O, lse, (cudaStream_t)stream));
}

extern "C" moc_status moc_merge(const moc_layout* lay, int B, int H, int d, int k,
                                const int32_t* sel, void* O, float* lse, void* ws, size_t ws_bytes,
                                moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    if ((st = check_ws(lay, B, H, d, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (!O || !aligned16(O) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3))) return MOC_ERR_INVALID_ARG;
    if (k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_merge(B * H, int(lay->L), d, k, sel, O, lse,
                                         static_cast<const char*>(ws), p, (cudaStream_t)stream));
}

extern "C" moc_status moc_attention_fwd(const moc_layout* lay, int B, int H, int d, const void* Q,
                                        const void* K, const void* V, const int32_t* sel, int k,
                                        float scale, void* O, float* lse, void* ws,
                                        size_t ws_bytes, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    if ((st = check_ws(lay, B, H, d, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return MOC_ERR_INVALID_ARG;
    if (k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) return MOC_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3)) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    if ((st = moc_build_qlists(lay, B, H, k, sel, ws, ws_bytes, stream)) != MOC_OK) return st;
    if ((st = moc_attend_partials(lay, B, H, d, Q, K, V, k, scale, ws, ws_bytes, stream)) != MOC_OK)
        return st;
    return moc_merge(lay, B, H, d, k, sel, O, lse, ws, ws_bytes, stream);
}

extern "C" moc_status moc_check_device_error(void* ws, size_t ws_bytes, int32_t* detail,
                                             moc_stream_t stream) {
    if (!ws || ws_bytes < 64 * sizeof(int32_t)) return MOC_ERR_INVALID_ARG;
    int32_t h[2] = {0, 0};
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOC_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOC_ERR_CUDA;
    if (detail) *detail = (h[0] != moc::ERR_NONE) ? h[1] : 0;
    if (h[0] != moc::ERR_NONE) {
        if (cudaMemsetAsync(ws, 0, 2 * sizeof(int32_t), s) != cudaSuccess) return MOC_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return MOC_ERR_CUDA;
    }
    if (h[0] == moc::ERR_TIMEOUT) return MOC_ERR_DEVICE_TIMEOUT;
    if (h[0] == moc::ERR_CHECK) return MOC_ERR_DEVICE_CHECK;
    return MOC_OK;
}

extern "C" moc_status moc_set_attend_kernel(int variant) {
    if (variant < 0 || variant > 2) return MOC_ERR_INVALID_ARG;
    g_attend_kernel.store(variant, std::memory_order_relaxed);
    return MOC_OK;
}

extern "C" moc_status moc_set_attend_schedule(int n_ctas, int item_order) {
    if (n_ctas < 0 || (item_order != 0 && item_order != 1)) return MOC_ERR_INVALID_ARG;
    g_sched_ctas.store(n_ctas, std::memory_order_relaxed);
    g_sched_reverse.store(item_order, std::memory_order_relaxed);
    return MOC_OK;
}

extern "C" size_t moc_attention_bwd_workspace_bytes(const moc_layout* lay, int B, int H, int d, int k) {
    if (!lay || B < 0 || H < 0 || (d != 64 && d != 128) || k < 0 || k > moc::kMaxK) return 0;
    return moc::plan_workspace_bwd(lay, B, H, d, k).total;
}

extern "C" moc_status moc_attention_bwd(const moc_layout* lay, int B, int H, int d, const void* Q,
                                        const void* K, const void* V, const void* O, const float* lse,
                                        const void* dO, const int32_t* sel, int k, float scale, void* dQ,
                                        void* dK, void* dV, void* ws, size_t ws_bytes, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (B * H == 0) return MOC_OK;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return MOC_ERR_INVALID_ARG;
    const moc::WsPlan p = moc::plan_workspace_bwd(lay, B, H, d, k);
    if (ws_bytes < p.total) return MOC_ERR_WORKSPACE_TOO_SMALL;
    for (const void* t : {Q, K, V, O, dO, static_cast<const void*>(dQ), static_cast<const void*>(dK),
                          static_cast<const void*>(dV)})
        if (!t || !aligned16(t)) return MOC_ERR_INVALID_ARG;
    if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3)) return MOC_ERR_INVALID_ARG;
    if (k > 0 && (!sel || (reinterpret_cast<uintptr_t>(sel) & 3))) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    char* w = static_cast<char*>(ws);
    const int BH = B * H;
    cudaError_t e = moc::launch_qlists(lay->dv, BH, k, sel, w, p, s);
    if (e == cudaSuccess) e = moc::launch_bwd_rowdot(BH, int(lay->L), d, O, dO, w, p, s);
    if (e == cudaSuccess)
        e = moc::launch_bwd_dq(lay->dv, BH, d, Q, K, V, dO, lse, k, scale, int64_t(BH) * lay->total_atiles, w, p,
                               s);
    if (e == cudaSuccess) e = moc::launch_bwd_dq_reduce(BH, int(lay->L), lay->C, d, k, sel, dQ, w, p, s);
    if (e == cudaSuccess) e = moc::launch_bwd_dkv(lay->dv, BH, d, Q, K, V, dO, lse, scale, w, p, dK, dV, s);
    return cuda_status(e);
}

extern "C" moc_status moc_quantize_e4m3(int BH, int64_t L, int d, const void* X, void* X8, float* scale,
                                        moc_stream_t stream) {
    if (BH < 0 || L < 0 || (d != 64 && d != 128)) return MOC_ERR_INVALID_ARG;
    if (BH == 0 || L == 0) return MOC_OK;
    if (!X || !X8 || !scale || !aligned16(X) || !aligned16(X8) || (reinterpret_cast<uintptr_t>(scale) & 3))
        return MOC_ERR_INVALID_ARG;
    return cuda_status(moc::launch_quant_e4m3(BH, L, d, X, X8, scale, (cudaStream_t)stream));
}

extern "C" moc_status moc_attend_partials_e4m3(const moc_layout* lay, int B, int H, int d, const void* Q8,
                                               const void* K8, const void* V8, const float* q_scale,
                                               const float* k_scale, const float* v_scale, int k, float scale,
                                               void* ws, size_t ws_bytes, moc_stream_t stream) {
    moc_status st = check_common(lay, B, H, d, k);
    if (st != MOC_OK) return st;
    if (d != 128) return MOC_ERR_UNSUPPORTED;
    if (B * H == 0) return MOC_OK;
    moc::WsPlan p;
    if ((st = check_ws(lay, B, H, d, k, ws, ws_bytes, &p)) != MOC_OK) return st;
    if (!Q8 || !K8 || !V8 || !aligned16(Q8) || !aligned16(K8) || !aligned16(V8)) return MOC_ERR_INVALID_ARG;
    for (const float* t : {q_scale, k_scale, v_scale})
        if (!t || (reinterpret_cast<uintptr_t>(t) & 3)) return MOC_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || scale != scale) return MOC_ERR_INVALID_ARG;
    const int64_t n_anchor = int64_t(B) * H * lay->total_atiles;
    return cuda_status(moc::launch_attend_e4m3(lay->dv, B * H, Q8, K8, V8, q_scale, k_scale, v_scale, k, scale,
                                               n_anchor, static_cast<char*>(ws), p, (cudaStream_t)stream));
}

extern "C" moc_status moc_attention_fwd_e4m3(const moc_layout* lay, int B, int H, int d, const void* Q8,
                                             const void* K8, const void* V8, const float* q_scale,
                                             const float* k_scale, const float* v_scale, const int32_t* sel, int k,
                                             float scale, void* O, float* lse, void* ws, size_t ws_bytes,
                                             moc_stream_t stream) {
    moc_status st;
    if ((st = moc_build_qlists(lay, B, H, k, sel, ws, ws_bytes, stream)) != MOC_OK) return st;
    if ((st = moc_attend_partials_e4m3(lay, B, H, d, Q8, K8, V8, q_scale, k_scale, v_scale, k, scale, ws,
                                       ws_bytes, stream)) != MOC_OK)
        return st;
    return moc_merge(lay, B, H, d, k, sel, O, lse, ws, ws_bytes, stream);
}

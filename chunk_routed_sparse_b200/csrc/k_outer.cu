// (2'') Outer-loop context routing: a coarse router that picks, per query
// block, the top-M context segments whose candidates the inner router (2) may
// then select from.
//
// "Mixture of Contexts for Long Video Generation | Summary", appendix I: a coarse
// router first selects top-M large context segments by the similarity between
// the mean-pooled features of the current query block and of the candidate
// segments, and hands those segments plus the mandatory context to the inner MoC
// routing. Segments are the shots (each shot's video chunks, numbered in stream
// order); a query block is a query group (the queries that share one anchor set);
// both features are token means (the block's queries, the segment's keys), formed
// here from the per-chunk means of (1) weighted by chunk length; the score is the
// unscaled dot product. A block's candidates are the other segments - only the
// earlier ones when causal - and its own segment is always kept (mandatory
// context): mask bit s set = segment s allowed. Top-M by (score descending,
// segment ascending); fewer candidates than M -> all. Caption blocks: mask 0.
// One warp per (b*h, group), lanes split d.
#include "common.cuh"

namespace moc {
namespace {

template <int D>
__device__ __forceinline__ void weighted_mean(const DevLayout& dv, const float* __restrict__ base,
                                              const int32_t* chunks, int n, float (&out)[D / 32], int lane) {
    float acc[D / 32];
    for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
    float tot = 0.f;
    for (int i = 0; i < n; ++i) {
        const int c = chunks[i];
        const float w = float(dv.chunk_off[c + 1] - dv.chunk_off[c]);
        const float* row = base + size_t(c) * D;
        for (int x = 0; x < D / 32; ++x) acc[x] += w * row[lane + 32 * x];
        tot += w;
    }
    for (int x = 0; x < D / 32; ++x) out[x] = acc[x] / tot;
}

template <int D>
__global__ void __launch_bounds__(256) outer_kernel(DevLayout dv, int BH, const float* __restrict__ Qbar,
                                                    const float* __restrict__ Kbar, int M, int causal,
                                                    uint64_t* __restrict__ seg_mask) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (wid >= int64_t(BH) * dv.G) return;
    const int bh = int(wid / dv.G), g = int(wid % dv.G);
    const int own = dv.grp_seg[g];
    if (own < 0) {  // caption block: dense, no routing
        if (lane == 0) seg_mask[wid] = 0;
        return;
    }
    // the block's query feature: its chunks are consecutive, [c0, c1)
    const int c0 = upper_index(dv.chunk_off, dv.C + 1, dv.grp_q0[g]);
    const int c1 = upper_index(dv.chunk_off, dv.C + 1, dv.grp_q1[g] - 1) + 1;
    float q[D / 32];
    {
        float acc[D / 32];
        for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
        float tot = 0.f;
        const float* base = Qbar + size_t(bh) * dv.C * D;
        for (int c = c0; c < c1; ++c) {
            const float w = float(dv.chunk_off[c + 1] - dv.chunk_off[c]);
            for (int x = 0; x < D / 32; ++x) acc[x] += w * base[size_t(c) * D + lane + 32 * x];
            tot += w;
        }
        for (int x = 0; x < D / 32; ++x) q[x] = acc[x] / tot;
    }
    // scores of the candidate segments, segment s held by lane s % 32, slot s / 32
    float sc[2] = {-INFINITY, -INFINITY};
    uint64_t cand = 0;
    const float* kb = Kbar + size_t(bh) * dv.C * D;
    for (int s = 0; s < dv.S; ++s) {
        if (s == own || (causal && s > own)) continue;
        float kf[D / 32];
        weighted_mean<D>(dv, kb, dv.vid + dv.seg_voff[s], dv.seg_voff[s + 1] - dv.seg_voff[s], kf, lane);
        float p = 0.f;
        for (int x = 0; x < D / 32; ++x) p += q[x] * kf[x];
        for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
        if (lane == (s & 31)) sc[s >> 5] = p;
        cand |= 1ull << s;
    }
    // top-M: M rounds of a warp argmax (score desc, segment asc)
    uint64_t mask = 1ull << own;
    for (int r = 0; r < M && cand; ++r) {
        float best = -INFINITY;
        int bs = 64;
        for (int h = 0; h < 2; ++h) {
            const int s = lane + 32 * h;
            if (s < dv.S && ((cand >> s) & 1ull) && (sc[h] > best || (sc[h] == best && s < bs))) {
                best = sc[h];
                bs = s;
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (ob > best || (ob == best && os < bs)) {
                best = ob;
                bs = os;
            }
        }
        if (bs >= 64) break;
        mask |= 1ull << bs;
        cand &= ~(1ull << bs);
    }
    if (lane == 0) seg_mask[wid] = mask;
}

}  // namespace

cudaError_t launch_outer(const DevLayout& dv, int BH, int d, const float* Qbar, const float* Kbar, int M,
                         int causal, uint64_t* seg_mask, cudaStream_t s) {
    const int64_t warps = int64_t(BH) * dv.G;
    if (warps == 0) return cudaSuccess;
    const unsigned grid = unsigned((warps * 32 + 255) / 256);
    if (d == 128)
        outer_kernel<128><<<grid, 256, 0, s>>>(dv, BH, Qbar, Kbar, M, causal, seg_mask);
    else
        outer_kernel<64><<<grid, 256, 0, s>>>(dv, BH, Qbar, Kbar, M, causal, seg_mask);
    return cudaGetLastError();
}

}  // namespace moc

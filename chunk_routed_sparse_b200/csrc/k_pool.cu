// (1) Segmented mean pool of keys per (b, h, chunk).
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: a chunk is
// represented by the mean of its keys; the jxzklqfsx.com MoC write-up,
// "計算效率": the pooled key is computed on the fly (segment_reduce mean), so
// chunks are never materialised.
//
// HBM-bound: every key byte is read once (2*d bytes per token and head).
// One CTA of kThreads per (b*h, chunk); each thread streams 16-byte bf16
// vectors with four loads in flight, accumulates 8 lanes of fp32, and the CTA
// reduces the row groups in a fixed order, so the result is deterministic.
// 1024-thread CTAs (two per SM): the eight-shot scene's 3,072 (chunk, head)
// CTAs then run in ~10 waves of whole chunks instead of ~2.6 with 256-thread
// CTAs, whose partly filled last wave cost 6 % (0.187 -> 0.176 ms, 0.90 -> 0.96
// of the measured copy bandwidth).
#include "common.cuh"

namespace moc {
namespace {

constexpr int kThreads = 1024;

__device__ __forceinline__ void acc8(float* a, uint4 v) {
    a[0] += bf16lo(v.x); a[1] += bf16hi(v.x);
    a[2] += bf16lo(v.y); a[3] += bf16hi(v.y);
    a[4] += bf16lo(v.z); a[5] += bf16hi(v.z);
    a[6] += bf16lo(v.w); a[7] += bf16hi(v.w);
}

template <int D>
__global__ void __launch_bounds__(kThreads) pool_kernel(DevLayout dv, const uint4* __restrict__ K,
                                                   float* __restrict__ Kbar) {
    constexpr int LPR = D / 8;      // threads per key row (16 B each)
    constexpr int RPI = kThreads / LPR;  // rows per pass of the CTA
    __shared__ float red[RPI][D + 4];
    const int c = blockIdx.x, bh = blockIdx.y;
    const int t0 = dv.chunk_off[c], t1 = dv.chunk_off[c + 1];
    const int col = threadIdx.x % LPR, r0 = threadIdx.x / LPR;
    const uint4* base = K + size_t(bh) * size_t(dv.L) * LPR + col;
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int t = t0 + r0;
    for (; t + 3 * RPI < t1; t += 4 * RPI) {
        uint4 v0 = ldg_nc16(base + size_t(t) * LPR);
        uint4 v1 = ldg_nc16(base + size_t(t + RPI) * LPR);
        uint4 v2 = ldg_nc16(base + size_t(t + 2 * RPI) * LPR);
        uint4 v3 = ldg_nc16(base + size_t(t + 3 * RPI) * LPR);
        acc8(a, v0);
        acc8(a, v1);
        acc8(a, v2);
        acc8(a, v3);
    }
    for (; t < t1; t += RPI) acc8(a, ldg_nc16(base + size_t(t) * LPR));
#pragma unroll
    for (int j = 0; j < 8; ++j) red[r0][col * 8 + j] = a[j];
    __syncthreads();
    for (int e = threadIdx.x; e < D; e += kThreads) {
        float s = 0.f;
#pragma unroll 8
        for (int r = 0; r < RPI; ++r) s += red[r][e];
        Kbar[(size_t(bh) * dv.C + c) * D + e] = s / float(t1 - t0);
    }
}

}  // namespace

cudaError_t launch_pool(const DevLayout& dv, int BH, int d, const void* K, float* Kbar,
                        cudaStream_t s) {
    if (BH > 65535) return cudaErrorInvalidValue;
    dim3 grid(dv.C, BH);
    if (d == 128)
        pool_kernel<128><<<grid, kThreads, 0, s>>>(dv, static_cast<const uint4*>(K), Kbar);
    else
        pool_kernel<64><<<grid, kThreads, 0, s>>>(dv, static_cast<const uint4*>(K), Kbar);
    return cudaGetLastError();
}

}  // namespace moc

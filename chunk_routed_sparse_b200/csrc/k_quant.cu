// E4M3 quantisation of Q, K and V for the E4M3 attention variant.
//
// The pages' future-work lists ("Mixture of Contexts for Long Video
// Generation | Summary", limitations; the jxzklqfsx.com write-up,
// "局限性與未來工作") name quantisation as a way to make the sparse attention
// cheaper. Here every (b, h) slice gets one scale, a power of two:
//   scale = 2^ceil(log2(amax / 448))  (1 for an all-zero slice),
//   x8 = E4M3(x / scale), round to nearest even (x / scale is exact and at
//   most 448 in magnitude, so nothing saturates),
// so x8 * scale is exactly representable in bf16 and the quantised tensor can
// be checked against attention evaluated on those exact values.
#include "common.cuh"
#include "sm100.cuh"

namespace moc {
namespace {

// amax over a slice: bits of |x| (non-negative floats order as integers)
__global__ void __launch_bounds__(256) quant_amax_kernel(int64_t n_per, const __nv_bfloat16* __restrict__ X,
                                                         uint32_t* __restrict__ amax) {
    const int bh = blockIdx.y;
    const uint4* x = reinterpret_cast<const uint4*>(X + size_t(bh) * n_per);
    const int64_t n16 = n_per / 8;
    uint32_t m = 0;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += int64_t(gridDim.x) * blockDim.x) {
        const uint4 v = __ldg(x + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            m = max(m, (w[e] << 16) & 0x7fffffffu);
            m = max(m, w[e] & 0x7fff0000u);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax + bh, m);
}

__device__ __forceinline__ int scale_exp(uint32_t amax_bits) {
    const float r = __uint_as_float(amax_bits) / 448.f;
    if (!(r > 0.f)) return 0;
    int e;
    const float m = frexpf(r, &e);  // r = m 2^e, m in [0.5, 1)
    return m == 0.5f ? e - 1 : e;
}

__global__ void __launch_bounds__(256) quant_kernel(int64_t n_per, const __nv_bfloat16* __restrict__ X,
                                                    const uint32_t* __restrict__ amax, uint32_t* __restrict__ X8) {
    const int bh = blockIdx.y;
    const int e = scale_exp(amax[bh]);
    const uint4* x = reinterpret_cast<const uint4*>(X + size_t(bh) * n_per);
    uint2* y = reinterpret_cast<uint2*>(X8) + size_t(bh) * (n_per / 8);
    const int64_t n16 = n_per / 8;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += int64_t(gridDim.x) * blockDim.x) {
        const uint4 v = __ldg(x + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float a = ldexpf(bf16lo(w[2 * h]), -e), b = ldexpf(bf16hi(w[2 * h]), -e);
            const float c = ldexpf(bf16lo(w[2 * h + 1]), -e), d = ldexpf(bf16hi(w[2 * h + 1]), -e);
            o[h] = sm100::pack_e4m3x2(a, b) | (sm100::pack_e4m3x2(c, d) << 16);
        }
        y[i] = make_uint2(o[0], o[1]);
    }
}

__global__ void quant_scale_kernel(int BH, uint32_t* __restrict__ amax_to_scale) {
    for (int bh = threadIdx.x; bh < BH; bh += blockDim.x)
        amax_to_scale[bh] = __float_as_uint(ldexpf(1.f, scale_exp(amax_to_scale[bh])));
}

}  // namespace

cudaError_t launch_quant_e4m3(int BH, int64_t L, int d, const void* X, void* X8, float* scale, cudaStream_t s) {
    const int64_t n_per = L * d;
    uint32_t* amax = reinterpret_cast<uint32_t*>(scale);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t) * size_t(BH), s);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n_per / 8 + 255) / 256;
    const int per = int(want < (4 * sms + BH - 1) / BH ? want : (4 * sms + BH - 1) / BH);
    dim3 grid(per > 0 ? per : 1, BH);
    const auto* x = static_cast<const __nv_bfloat16*>(X);
    quant_amax_kernel<<<grid, 256, 0, s>>>(n_per, x, amax);
    quant_kernel<<<grid, 256, 0, s>>>(n_per, x, amax, static_cast<uint32_t*>(X8));
    quant_scale_kernel<<<1, 256, 0, s>>>(BH, amax);
    return cudaGetLastError();
}

}  // namespace moc

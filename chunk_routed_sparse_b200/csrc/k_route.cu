// (2) Router: per-query top-k over candidate chunks.
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: each query
// scores candidate chunks by the dot product with their mean-pooled keys and
// keeps the k best, independently per head; §3.2: optional edges i->j are
// masked whenever j >= i before top-k. The jxzklqfsx.com MoC write-up,
// "計算效率": mandatory chunks are inserted before top-k so that the router
// spends no budget on them (they are not candidates).
//
// One CTA per (b*h, 128-query tile of one query group). All queries of a
// group share one candidate list. Per block of 64 candidates:
//   * the fp32 pooled keys are split into hi + lo bf16 parts (hi = RN(x),
//     lo = RN(x - hi)); Q is exactly bf16, so q.hi + q.lo on the tensor cores
//     (mma.sync m16n8k16, fp32 accumulate) reproduces q.Kbar to about 2^-17
//     relative per term instead of bf16's 2^-9;
//   * each warp owns 16 queries and keeps their running top-k spread over its
//     lanes (lane x holds entry x); a candidate that ranks before the current
//     k-th entry is inserted with one ballot (its rank) and one shuffle (the
//     shift of the worse entries). Ties rank the lower chunk id first.
#include "common.cuh"

namespace moc {
namespace {

constexpr int kCandBlock = 64;
constexpr int kIdNone = 0x7fffffff;

template <int D>
struct RouteSmem {
    static constexpr int kStride = D + 8;  // bf16 elements per row (+16 B: conflict-free fragments)
    static constexpr int kSStride = kCandBlock + 4;
    __nv_bfloat16 q[kQTile][kStride];
    __nv_bfloat16 khi[kCandBlock][kStride];
    __nv_bfloat16 klo[kCandBlock][kStride];
    float s[8][16][kSStride];
    int cid[kCandBlock];
};

template <int D>
__global__ void __launch_bounds__(256, 2)
    route_kernel(DevLayout dv, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ Kbar,
                 int k, int causal, int32_t* __restrict__ sel) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RouteSmem<D>& sm = *reinterpret_cast<RouteSmem<D>*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y;
    const int tile = blockIdx.x;
    const int g = upper_index(dv.rtile_off, dv.G + 1, tile);
    const int q0 = dv.grp_q0[g] + (tile - dv.rtile_off[g]) * kQTile;
    const int nq = min(kQTile, dv.grp_q1[g] - q0);
    int32_t* out = sel + (size_t(bh) * dv.L + q0) * k;
    const int cbeg = dv.cand_off[g];
    const int ncand = (dv.grp_kind[g] != MOC_VIDEO) ? 0
                      : causal ? dv.cand_ncausal[g] : dv.cand_off[g + 1] - cbeg;
    if (ncand == 0) {
        for (int i = tid; i < nq * k; i += blockDim.x) out[i] = -1;
        return;
    }
    // query tile -> shared memory (rows past the group end are zero)
    constexpr int V8 = D / 8;
    const __nv_bfloat16* qsrc = Q + (size_t(bh) * dv.L + q0) * D;
    for (int i = tid; i < kQTile * V8; i += blockDim.x) {
        const int r = i / V8, c = i % V8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < nq) v = ldg_nc16(qsrc + size_t(r) * D + c * 8);
        *reinterpret_cast<uint4*>(&sm.q[r][c * 8]) = v;
    }
    float top_s[16];
    int top_j[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        top_s[r] = -INFINITY;
        top_j[r] = kIdNone;
    }
    const int g8 = lane >> 2, t4 = lane & 3;
    const float* kb = Kbar + size_t(bh) * dv.C * D;
    for (int cb = 0; cb < ncand; cb += kCandBlock) {
        __syncthreads();  // previous block's candidates fully consumed
        constexpr int V4 = D / 4;
        for (int i = tid; i < kCandBlock * V4; i += blockDim.x) {
            const int r = i / V4, c = i % V4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (cb + r < ncand)
                x = *reinterpret_cast<const float4*>(kb + size_t(dv.cand[cbeg + cb + r]) * D + c * 4);
            __nv_bfloat162 h01 = __floats2bfloat162_rn(x.x, x.y);
            __nv_bfloat162 h23 = __floats2bfloat162_rn(x.z, x.w);
            float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
            __nv_bfloat162 l01 = __floats2bfloat162_rn(x.x - f01.x, x.y - f01.y);
            __nv_bfloat162 l23 = __floats2bfloat162_rn(x.z - f23.x, x.w - f23.y);
            *reinterpret_cast<__nv_bfloat162*>(&sm.khi[r][c * 4]) = h01;
            *reinterpret_cast<__nv_bfloat162*>(&sm.khi[r][c * 4 + 2]) = h23;
            *reinterpret_cast<__nv_bfloat162*>(&sm.klo[r][c * 4]) = l01;
            *reinterpret_cast<__nv_bfloat162*>(&sm.klo[r][c * 4 + 2]) = l23;
        }
        if (tid < kCandBlock) sm.cid[tid] = (cb + tid < ncand) ? dv.cand[cbeg + cb + tid] : kIdNone;
        __syncthreads();

        // scores of this warp's 16 queries x 64 candidates
        float acc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
        const int qr = warp * 16;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const int k0 = ks * 16;
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t*>(&sm.q[qr + g8][k0 + 2 * t4]);
            a[1] = *reinterpret_cast<const uint32_t*>(&sm.q[qr + g8 + 8][k0 + 2 * t4]);
            a[2] = *reinterpret_cast<const uint32_t*>(&sm.q[qr + g8][k0 + 8 + 2 * t4]);
            a[3] = *reinterpret_cast<const uint32_t*>(&sm.q[qr + g8 + 8][k0 + 8 + 2 * t4]);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = j * 8 + g8;
                uint32_t h0 = *reinterpret_cast<const uint32_t*>(&sm.khi[n][k0 + 2 * t4]);
                uint32_t h1 = *reinterpret_cast<const uint32_t*>(&sm.khi[n][k0 + 8 + 2 * t4]);
                uint32_t l0 = *reinterpret_cast<const uint32_t*>(&sm.klo[n][k0 + 2 * t4]);
                uint32_t l1 = *reinterpret_cast<const uint32_t*>(&sm.klo[n][k0 + 8 + 2 * t4]);
                mma_bf16_16816(acc[j], a, h0, h1);
                mma_bf16_16816(acc[j], a, l0, l1);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            *reinterpret_cast<float2*>(&sm.s[warp][g8][j * 8 + 2 * t4]) = make_float2(acc[j][0], acc[j][1]);
            *reinterpret_cast<float2*>(&sm.s[warp][g8 + 8][j * 8 + 2 * t4]) = make_float2(acc[j][2], acc[j][3]);
        }
        __syncwarp();

        // merge the block into each row's running top-k
        const int j1 = sm.cid[lane], j2 = sm.cid[lane + 32];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float s1 = (j1 == kIdNone) ? -INFINITY : sm.s[warp][r][lane];
            float s2 = (j2 == kIdNone) ? -INFINITY : sm.s[warp][r][lane + 32];
            float my_s = top_s[r];
            int my_j = top_j[r];
            float thr_s = __shfl_sync(0xffffffffu, my_s, k - 1);
            int thr_j = __shfl_sync(0xffffffffu, my_j, k - 1);
            unsigned m1 = __ballot_sync(0xffffffffu, ranks_before(s1, j1, thr_s, thr_j));
            unsigned m2 = __ballot_sync(0xffffffffu, ranks_before(s2, j2, thr_s, thr_j));
            while (m1 | m2) {
                float cs;
                int cj;
                if (m1) {
                    const int src = __ffs(m1) - 1;
                    m1 &= m1 - 1;
                    cs = __shfl_sync(0xffffffffu, s1, src);
                    cj = __shfl_sync(0xffffffffu, j1, src);
                } else {
                    const int src = __ffs(m2) - 1;
                    m2 &= m2 - 1;
                    cs = __shfl_sync(0xffffffffu, s2, src);
                    cj = __shfl_sync(0xffffffffu, j2, src);
                }
                if (!ranks_before(cs, cj, thr_s, thr_j)) continue;  // uniform across the warp
                const int pos = __popc(__ballot_sync(0xffffffffu,
                                                     lane < k && ranks_before(my_s, my_j, cs, cj)));
                const float up_s = __shfl_up_sync(0xffffffffu, my_s, 1);
                const int up_j = __shfl_up_sync(0xffffffffu, my_j, 1);
                if (lane > pos) {
                    my_s = up_s;
                    my_j = up_j;
                }
                if (lane == pos) {
                    my_s = cs;
                    my_j = cj;
                }
                thr_s = __shfl_sync(0xffffffffu, my_s, k - 1);
                thr_j = __shfl_sync(0xffffffffu, my_j, k - 1);
            }
            top_s[r] = my_s;
            top_j[r] = my_j;
        }
    }
    const int qr = warp * 16;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        if (qr + r < nq && lane < k) out[size_t(qr + r) * k + lane] = (top_j[r] == kIdNone) ? -1 : top_j[r];
    }
}

template <int D>
cudaError_t launch_route_d(const DevLayout& dv, int BH, int64_t rtiles, const void* Q,
                           const float* Kbar, int k, int causal, int32_t* sel, cudaStream_t s) {
    const int smem = int(sizeof(RouteSmem<D>));
    cudaError_t e = cudaFuncSetAttribute(route_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(rtiles), BH);
    route_kernel<D><<<grid, 256, smem, s>>>(dv, static_cast<const __nv_bfloat16*>(Q), Kbar, k, causal, sel);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const DevLayout& dv, int BH, int64_t rtiles, int d, const void* Q,
                         const float* Kbar, int k, int causal, int32_t* sel, cudaStream_t s) {
    if (BH > 65535 || rtiles <= 0 || rtiles > 0x7fffffff) return cudaErrorInvalidValue;
    if (d == 128) return launch_route_d<128>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
    return launch_route_d<64>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
}

}  // namespace moc

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
//   * the 128 x 64 scores go to shared memory and every query row is scanned
//     by two threads (32 candidates each), each keeping a sorted top-KMAX list
//     in registers (KMAX: compile-time bound >= k). The two lists are merged
//     at the end. Ties rank the lower chunk id first.
#include "common.cuh"

namespace moc {
namespace {

constexpr int kCandBlock = 64;
constexpr int kIdNone = 0x7fffffff;

template <int D>
struct RouteSmem {
    static constexpr int kStride = D + 8;  // bf16 elements per row (+16 B: conflict-free fragments)
    static constexpr int kSStride = kCandBlock + 1;  // odd pitch: row-per-thread scans are conflict-free
    __nv_bfloat16 q[kQTile][kStride];
    __nv_bfloat16 khi[kCandBlock][kStride];
    __nv_bfloat16 klo[kCandBlock][kStride];
    float s[kQTile][kSStride];
    int cid[kCandBlock];
};

// Insert (cs, cj) into a sorted (best first) register list of KMAX entries
// if it ranks before the last entry; the last entry drops out.
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&ts)[KMAX], int (&tj)[KMAX], float cs, int cj) {
    if (!ranks_before(cs, cj, ts[KMAX - 1], tj[KMAX - 1])) return;
    ts[KMAX - 1] = cs;
    tj[KMAX - 1] = cj;
#pragma unroll
    for (int x = KMAX - 1; x > 0; --x) {
        if (ranks_before(ts[x], tj[x], ts[x - 1], tj[x - 1])) {
            const float fs = ts[x]; ts[x] = ts[x - 1]; ts[x - 1] = fs;
            const int fj = tj[x]; tj[x] = tj[x - 1]; tj[x - 1] = fj;
        }
    }
}

template <int D, int KMAX>
__global__ void __launch_bounds__(256, KMAX <= 16 ? 2 : 1)
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
    float ts[KMAX];
    int tj[KMAX];
#pragma unroll
    for (int x = 0; x < KMAX; ++x) {
        ts[x] = -INFINITY;
        tj[x] = kIdNone;
    }
    const int row = tid & (kQTile - 1), half = tid >> 7;
    const int g8 = lane >> 2, t4 = lane & 3;
    const float* kb = Kbar + size_t(bh) * dv.C * D;
    for (int cb = 0; cb < ncand; cb += kCandBlock) {
        __syncthreads();  // previous block's candidates and scores fully consumed
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
            sm.s[qr + g8][j * 8 + 2 * t4] = acc[j][0];
            sm.s[qr + g8][j * 8 + 2 * t4 + 1] = acc[j][1];
            sm.s[qr + g8 + 8][j * 8 + 2 * t4] = acc[j][2];
            sm.s[qr + g8 + 8][j * 8 + 2 * t4 + 1] = acc[j][3];
        }
        __syncthreads();

        // each thread scans 32 candidates of its row
        const int nblk = min(kCandBlock, ncand - cb);
        const int c1 = min(nblk, half * 32 + 32);
        for (int c = half * 32; c < c1; ++c) topk_insert<KMAX>(ts, tj, sm.s[row][c], sm.cid[c]);
    }
    // merge the two halves of every row: half 1 publishes, half 0 merges
    __syncthreads();
    float* pub_s = &sm.s[0][0];
    int* pub_j = reinterpret_cast<int*>(&sm.q[0][0]);  // q is no longer read
    if (half == 1) {
#pragma unroll
        for (int x = 0; x < KMAX; ++x) {
            pub_s[row * KMAX + x] = ts[x];
            pub_j[row * KMAX + x] = tj[x];
        }
    }
    __syncthreads();
    if (half == 0) {
#pragma unroll
        for (int x = 0; x < KMAX; ++x) topk_insert<KMAX>(ts, tj, pub_s[row * KMAX + x], pub_j[row * KMAX + x]);
        if (row < nq) {
            int32_t* o = out + size_t(row) * k;
#pragma unroll
            for (int x = 0; x < KMAX; ++x)
                if (x < k) o[x] = (tj[x] == kIdNone) ? -1 : tj[x];
        }
    }
}

template <int D, int KMAX>
cudaError_t launch_route_dk(const DevLayout& dv, int BH, int64_t rtiles, const void* Q,
                            const float* Kbar, int k, int causal, int32_t* sel, cudaStream_t s) {
    const int smem = int(sizeof(RouteSmem<D>));
    cudaError_t e = cudaFuncSetAttribute(route_kernel<D, KMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(unsigned(rtiles), BH);
    route_kernel<D, KMAX><<<grid, 256, smem, s>>>(dv, static_cast<const __nv_bfloat16*>(Q), Kbar, k,
                                                  causal, sel);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_route_d(const DevLayout& dv, int BH, int64_t rtiles, const void* Q,
                           const float* Kbar, int k, int causal, int32_t* sel, cudaStream_t s) {
    if (k <= 4) return launch_route_dk<D, 4>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
    if (k <= 8) return launch_route_dk<D, 8>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
    if (k <= 16) return launch_route_dk<D, 16>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
    return launch_route_dk<D, 32>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
}

}  // namespace

cudaError_t launch_route(const DevLayout& dv, int BH, int64_t rtiles, int d, const void* Q,
                         const float* Kbar, int k, int causal, int32_t* sel, cudaStream_t s) {
    if (BH > 65535 || rtiles <= 0 || rtiles > 0x7fffffff) return cudaErrorInvalidValue;
    if (d == 128) return launch_route_d<128>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
    return launch_route_d<64>(dv, BH, rtiles, Q, Kbar, k, causal, sel, s);
}

}  // namespace moc

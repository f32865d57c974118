// (5) Log-sum-exp merge of each query's partial attention outputs.
//
// The attention of "Mixture of Contexts for Long Video Generation | Summary"
// §3.1 runs over Omega(q) = anchors + selected chunks. The attend kernel
// computes it in disjoint parts (slot 0: anchors; slot 1+x: the chunk in
// sel[x]), each normalised with its own log-sum-exp l_j. Softmax over a
// disjoint union recombines exactly:
//   M = max_j l_j,  w_j = exp(l_j - M),  O = sum_j w_j O_j / sum_j w_j,
//   lse = M + log sum_j w_j.
// One warp per (b*h, query); slots in fixed order -> deterministic.
// HBM-bound: reads (1+k)*(4d+4) bytes and writes 2d+4 bytes per query.
#include "common.cuh"

namespace moc {
namespace {

// MAXS > 0: at most MAXS slots, every valid slot's partial loaded at once (one
// memory round trip for sel and the log-sum-exps, one for the partials);
// MAXS == 0: any slot count, partials loaded slot by slot.
template <int D, int MAXS>
__global__ void __launch_bounds__(256) merge_kernel(int64_t rows, int L, int k,
                                                    const int32_t* __restrict__ sel,
                                                    const float* __restrict__ lse_p,
                                                    const float* __restrict__ o_p,
                                                    __nv_bfloat16* __restrict__ O,
                                                    float* __restrict__ lse) {
    constexpr int PER = D / 32;  // output columns per lane
    const int lane = threadIdx.x & 31;
    const int S = k + 1;
    const int64_t step = (int64_t(gridDim.x) * blockDim.x) >> 5;
    // sel and the slot log-sum-exps of a row in one round trip (an invalid slot's lse
    // is never used: it may not have been written); with MAXS > 0 the next row's are
    // requested before this row's partials are read, so the two round trips overlap
    // (eight-shot, k = 3: 1.73 -> 1.49 ms; the slot-by-slot path keeps one row at a
    // time, which measured faster there)
    auto head = [&](int64_t r, int32_t& sj, float& l) {
        sj = 0;
        l = -INFINITY;
        if (r < rows && lane < S) {
            if (lane > 0) sj = __ldg(sel + r * k + lane - 1);
            l = __ldg(lse_p + r * S + lane);
        }
    };
    int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    int32_t sj_next = 0;
    float l_next = -INFINITY;
    if (MAXS > 0) head(row, sj_next, l_next);
    for (; row < rows; row += step) {
        int32_t sj;
        float l;
        if (MAXS > 0) {
            sj = sj_next;
            l = l_next;
            head(row + step, sj_next, l_next);
        } else {
            head(row, sj, l);
        }
        const bool valid = lane < S && (lane == 0 || sj >= 0);
        if (!valid) l = -INFINITY;
        float m = l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float w = valid ? expf(l - m) : 0.f;
        float z = w;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const unsigned vmask = __ballot_sync(0xffffffffu, valid);
        float acc[PER];
#pragma unroll
        for (int x = 0; x < PER; ++x) acc[x] = 0.f;
        const float* op = o_p + size_t(row) * S * D + lane * PER;
        if (MAXS > 0) {
            float v[MAXS > 0 ? MAXS : 1][PER];
#pragma unroll
            for (int j = 0; j < MAXS; ++j) {
#pragma unroll
                for (int x = 0; x < PER; ++x) v[j][x] = 0.f;
                if ((vmask >> j) & 1u) {
                    if (PER == 4) {
                        const float4 t = __ldg(reinterpret_cast<const float4*>(op + size_t(j) * D));
                        v[j][0] = t.x; v[j][1] = t.y; v[j][2] = t.z; v[j][3] = t.w;
                    } else {
                        const float2 t = __ldg(reinterpret_cast<const float2*>(op + size_t(j) * D));
                        v[j][0] = t.x; v[j][1] = t.y;
                    }
                }
            }
            // fixed slot order, as in the general path
#pragma unroll
            for (int j = 0; j < MAXS; ++j) {
                const float wj = __shfl_sync(0xffffffffu, w, j) / z;
                if ((vmask >> j) & 1u) {
#pragma unroll
                    for (int x = 0; x < PER; ++x) acc[x] += wj * v[j][x];
                }
            }
        } else {
            for (unsigned mm = vmask; mm; mm &= mm - 1) {
                const int j = __ffs(mm) - 1;
                const float wj = __shfl_sync(0xffffffffu, w, j) / z;
                if (PER == 4) {
                    const float4 t = __ldg(reinterpret_cast<const float4*>(op + size_t(j) * D));
                    acc[0] += wj * t.x; acc[1] += wj * t.y; acc[2] += wj * t.z; acc[3] += wj * t.w;
                } else {
                    const float2 t = __ldg(reinterpret_cast<const float2*>(op + size_t(j) * D));
                    acc[0] += wj * t.x; acc[1] += wj * t.y;
                }
            }
        }
        __nv_bfloat16* orow = O + size_t(row) * D + lane * PER;
        if (PER == 4) {
            uint2 pk = make_uint2(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]));
            *reinterpret_cast<uint2*>(orow) = pk;
        } else {
            *reinterpret_cast<uint32_t*>(orow) = pack_bf16(acc[0], acc[1]);
        }
        if (lse && lane == 0) lse[row] = m + logf(z);
    }
}

}  // namespace

cudaError_t launch_merge(int BH, int L, int d, int k, const int32_t* sel, void* O, float* lse,
                         const char* ws, const WsPlan& p, cudaStream_t s) {
    const int64_t rows = int64_t(BH) * L;
    const float* lse_p = reinterpret_cast<const float*>(ws + p.lse_p);
    const float* o_p = reinterpret_cast<const float*>(ws + p.o_p);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (rows + 7) / 8;
    const int grid = int(want < int64_t(sms) * 16 ? want : int64_t(sms) * 16);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(O);
    if (d == 128) {
        if (k + 1 <= 4) merge_kernel<128, 4><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
        else if (k + 1 <= 8) merge_kernel<128, 8><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
        else merge_kernel<128, 0><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
    } else {
        if (k + 1 <= 4) merge_kernel<64, 4><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
        else if (k + 1 <= 8) merge_kernel<64, 8><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
        else merge_kernel<64, 0><<<grid, 256, 0, s>>>(rows, L, k, sel, lse_p, o_p, o, lse);
    }
    return cudaGetLastError();
}

}  // namespace moc

// (3) Query-list builder: invert the per-query selections into per-chunk
// query lists (count -> exclusive prefix sum -> ordered scatter).
//
// This replaces the "pack every (query, key) group into one variable-length
// attention call" step of the jxzklqfsx.com MoC write-up ("計算效率"): the
// attention kernel walks chunk-major work items, each a chunk's keys against
// up to 256 of the queries that selected it.
//
// Entries are (query << 5 | slot), slot = position in sel. Every list is
// sorted by query: each block owns kQlistBlock consecutive queries and one
// warp walks them in order, ranking equal chunk ids inside a 32-entry step
// with __match_any_sync, so the output is deterministic.
#include "common.cuh"

namespace moc {
namespace {

// blk_count[bh][blk][c] = entries of chunk c among the block's queries
__global__ void __launch_bounds__(32) qlist_count(int L, int C, int k, int nblk,
                                                  const int32_t* __restrict__ sel,
                                                  int32_t* __restrict__ blk_count,
                                                  int32_t* __restrict__ hdr) {
    extern __shared__ int32_t cnt[];
    const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
    for (int c = lane; c < C; c += 32) cnt[c] = 0;
    __syncwarp();
    const int q0 = blk * kQlistBlock, q1 = min(L, q0 + kQlistBlock);
    const int32_t* s = sel + (size_t(bh) * L) * k;
    constexpr int U = 4;  // entries per lane loaded per round trip
    const int64_t e1 = int64_t(q1) * k;
    for (int64_t e0 = int64_t(q0) * k + lane; e0 < e1; e0 += 32 * U) {
        int cs[U];
#pragma unroll
        for (int u = 0; u < U; ++u) cs[u] = (e0 + 32 * u < e1) ? s[e0 + 32 * u] : -1;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (cs[u] >= C) set_error(hdr, ERR_CHECK, 3);  // not a chunk id: entry ignored
            else if (cs[u] >= 0) atomicAdd(&cnt[cs[u]], 1);
        }
    }
    __syncwarp();
    int32_t* out = blk_count + (size_t(bh) * nblk + blk) * C;
    for (int c = lane; c < C; c += 32) out[c] = cnt[c];
}

// Per (bh): blk_count -> exclusive offsets of each block within each chunk's
// list (in place); qoff[bh*C + c] <- list length, tile_off[bh*C + c] <- attention
// work items of kItemRows entries, tile2_off[bh*C + c] <- items of kPairRows entries.
__global__ void __launch_bounds__(256) qlist_scan_blocks(int C, int nblk,
                                                         int32_t* __restrict__ blk_count,
                                                         int32_t* __restrict__ qlen,
                                                         int32_t* __restrict__ ntile,
                                                         int32_t* __restrict__ ntile2) {
    const int bh = blockIdx.x;
    constexpr int U = 8;  // block counts loaded per round trip
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        int32_t run = 0;
        int32_t* p = blk_count + size_t(bh) * nblk * C + c;
        for (int b0 = 0; b0 < nblk; b0 += U) {
            int32_t v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) v[u] = (b0 + u < nblk) ? p[size_t(b0 + u) * C] : 0;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (b0 + u < nblk) p[size_t(b0 + u) * C] = run;
                run += v[u];
            }
        }
        qlen[size_t(bh) * C + c] = run;
        ntile[size_t(bh) * C + c] = (run + kItemRows - 1) / kItemRows;
        ntile2[size_t(bh) * C + c] = (run + kPairRows - 1) / kPairRows;
    }
}

// In-place exclusive scan of three int32 arrays of n values (+ total at [n]),
// one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) qlist_scan_global(int64_t n, int32_t* __restrict__ a0,
                                                          int32_t* __restrict__ a1, int32_t* __restrict__ a2) {
    constexpr int NA = 3;
    int32_t* const arr[NA] = {a0, a1, a2};
    __shared__ int32_t w[NA][32];
    __shared__ int32_t carry[NA];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < NA) carry[tid] = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += 1024) {
        const int64_t i = base + tid;
        int32_t v[NA], x[NA];
#pragma unroll
        for (int j = 0; j < NA; ++j) x[j] = v[j] = (i < n) ? arr[j][i] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
            for (int j = 0; j < NA; ++j) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x[j], o);
                if (lane >= o) x[j] += y;
            }
        }
        if (lane == 31) {
#pragma unroll
            for (int j = 0; j < NA; ++j) w[j][warp] = x[j];
        }
        __syncthreads();
        if (warp == 0) {
#pragma unroll
            for (int j = 0; j < NA; ++j) {
                int32_t sj = w[j][lane];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int32_t y = __shfl_up_sync(0xffffffffu, sj, o);
                    if (lane >= o) sj += y;
                }
                w[j][lane] = sj;
            }
        }
        __syncthreads();
        int32_t pre[NA];
#pragma unroll
        for (int j = 0; j < NA; ++j) {
            pre[j] = carry[j] + (warp ? w[j][warp - 1] : 0) + x[j] - v[j];
            if (i < n) arr[j][i] = pre[j];
        }
        __syncthreads();
        if (tid == 1023) {
#pragma unroll
            for (int j = 0; j < NA; ++j) carry[j] = pre[j] + v[j];
        }
        __syncthreads();
    }
    if (tid == 0) {
#pragma unroll
        for (int j = 0; j < NA; ++j) arr[j][n] = carry[j];
    }
}

__global__ void __launch_bounds__(32) qlist_scatter(int L, int C, int k, int nblk,
                                                    const int32_t* __restrict__ sel,
                                                    const int32_t* __restrict__ blk_count,
                                                    const int32_t* __restrict__ qoff,
                                                    int32_t* __restrict__ qlist) {
    extern __shared__ int32_t cur[];
    const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
    const int32_t* bc = blk_count + (size_t(bh) * nblk + blk) * C;
    const int32_t* qo = qoff + size_t(bh) * C;
    for (int c = lane; c < C; c += 32) cur[c] = qo[c] + bc[c];
    __syncwarp();
    const int q0 = blk * kQlistBlock, q1 = min(L, q0 + kQlistBlock);
    const int32_t* s = sel + (size_t(bh) * L) * k;
    const unsigned lt = (1u << lane) - 1u;
    const int64_t e1 = int64_t(q1) * k;
    // each step's selection entry is loaded one step ahead, so the load latency
    // overlaps the previous step's ranking and stores
    int c_next = (int64_t(q0) * k + lane < e1) ? s[int64_t(q0) * k + lane] : -1;
    for (int64_t e0 = int64_t(q0) * k; e0 < e1; e0 += 32) {
        const int64_t e = e0 + lane;
        int c = c_next;
        c_next = (e + 32 < e1) ? s[e + 32] : -1;
        if (c >= C) c = -1;  // reported by qlist_count
        const unsigned peers = __match_any_sync(0xffffffffu, c);
        const int rank = __popc(peers & lt);
        const int base = (c >= 0) ? cur[c] : 0;
        __syncwarp();
        if (c >= 0) {
            const int q = int(e / k), slot = int(e % k);
            qlist[base + rank] = (q << 5) | slot;
            if (rank == 0) cur[c] = base + __popc(peers);
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_qlists(const DevLayout& dv, int BH, int k, const int32_t* sel, char* ws,
                          const WsPlan& p, cudaStream_t s) {
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    cudaError_t e = cudaMemsetAsync(hdr, 0, 4 * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    int32_t* blk_count = reinterpret_cast<int32_t*>(ws + p.blk_count);
    int32_t* qoff = reinterpret_cast<int32_t*>(ws + p.qoff);
    int32_t* tile_off = reinterpret_cast<int32_t*>(ws + p.tile_off);
    int32_t* tile2_off = reinterpret_cast<int32_t*>(ws + p.tile2_off);
    int32_t* qlist = reinterpret_cast<int32_t*>(ws + p.qlist);
    const int64_t n = int64_t(BH) * dv.C;
    if (k == 0) {  // no routed work: empty lists
        e = cudaMemsetAsync(qoff, 0, size_t(n + 1) * sizeof(int32_t), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(tile_off, 0, size_t(n + 1) * sizeof(int32_t), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(tile2_off, 0, size_t(n + 1) * sizeof(int32_t), s);
        return e;
    }
    if (BH > 65535) return cudaErrorInvalidValue;
    const size_t smem = size_t(dv.C) * sizeof(int32_t);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(qlist_count, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(qlist_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
    }
    dim3 grid(p.nblk, BH);
    qlist_count<<<grid, 32, smem, s>>>(dv.L, dv.C, k, p.nblk, sel, blk_count, hdr);
    qlist_scan_blocks<<<BH, 256, 0, s>>>(dv.C, p.nblk, blk_count, qoff, tile_off, tile2_off);
    qlist_scan_global<<<1, 1024, 0, s>>>(n, qoff, tile_off, tile2_off);
    qlist_scatter<<<grid, 32, smem, s>>>(dv.L, dv.C, k, p.nblk, sel, blk_count, qoff, qlist);
    return cudaGetLastError();
}

}  // namespace moc

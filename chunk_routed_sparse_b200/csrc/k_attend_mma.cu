// (4) Chunk-major attention over work items - warp-MMA (mma.sync) variant.
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: exact
// softmax attention of q over the keys/values of Omega(q), scaled by 1/sqrt(d).
// Omega(q) is split into disjoint parts that are attended separately and
// merged by their log-sum-exp (kernel 5):
//   anchor items  - a tile of <= 128 consecutive queries of one query group
//                   against the group's anchor key ranges (partial slot 0);
//   routed items  - <= 128 gathered queries of one chunk's query list against
//                   that chunk's keys (slot 1 + position in sel).
// Persistent CTAs take items from an atomic counter: anchor items first (most
// keys per item first), then routed items.
//
// This variant uses the legacy warp-level tensor-core path (mma.sync
// m16n8k16, bf16 in, fp32 accumulate) in a flash-attention loop: 8 warps x 16
// query rows, 64-key K/V tiles double-buffered with cp.async into an
// XOR-swizzled shared layout, online softmax in registers.
#include "common.cuh"

namespace moc {
namespace {

constexpr int kKT = 64;  // keys per tile

template <int D>
struct AttnSmem {
    __nv_bfloat16 q[kQTile * D];
    __nv_bfloat16 k[2][kKT * D];
    __nv_bfloat16 v[2][kKT * D];
    int32_t tok[kQTile];
    int32_t slot[kQTile];
    int item;
};

// byte offset of (row, 16-byte chunk) in a swizzled [rows][D] bf16 tile
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return uint32_t(row * D * 2 + ((chunk ^ (row & 7)) << 4));
}

struct ItemInfo {
    int bh, nq, slot_fixed;  // slot_fixed >= 0: anchor item (contiguous rows from q0)
    int q0;
    const int32_t* entries;  // routed: list entries (query << 5 | slot)
    int r_beg, r_end;        // anchor ranges [r_beg, r_end) in dv.ar; routed: r_beg = -1
    int k0, k1;              // routed: key range
};

__device__ __forceinline__ bool decode_item(const DevLayout& dv, int BH, int64_t n_anchor,
                                            int64_t item, const int32_t* tile_off,
                                            const int32_t* qoff, const int32_t* qlist,
                                            ItemInfo& it) {
    if (item < n_anchor) {
        const int pos = upper_index(dv.atile_off, dv.G + 1, item / BH);
        const int64_t local = item - int64_t(BH) * dv.atile_off[pos];
        const int nt = dv.atile_off[pos + 1] - dv.atile_off[pos];
        const int g = dv.a_order[pos];
        it.bh = int(local / nt);
        const int tile = int(local % nt);
        it.q0 = dv.grp_q0[g] + tile * kQTile;
        it.nq = min(kQTile, dv.grp_q1[g] - it.q0);
        it.slot_fixed = 0;
        it.entries = nullptr;
        it.r_beg = dv.ar_off[g];
        it.r_end = dv.ar_off[g + 1];
        return true;
    }
    const int64_t r = item - n_anchor;
    const int64_t nlists = int64_t(BH) * dv.C;
    if (r >= tile_off[nlists]) return false;
    const int x = upper_index(tile_off, int(nlists + 1), r);
    const int tile = int(r - tile_off[x]);
    const int c = x % dv.C;
    it.bh = x / dv.C;
    const int e0 = qoff[x] + tile * kQTile;
    it.nq = min(kQTile, qoff[x + 1] - e0);
    it.entries = qlist + e0;
    it.slot_fixed = -1;
    it.q0 = 0;
    it.r_beg = -1;
    it.r_end = -1;
    it.k0 = dv.chunk_off[c];
    it.k1 = dv.chunk_off[c + 1];
    return true;
}

// Walks the key tiles of an item: ranges [ar[2r], ar[2r+1]) in order, 64 keys a tile.
struct TileCursor {
    const int32_t* ar;
    int r, r_end, pos, end;
    __device__ void init_anchor(const int32_t* a, int rb, int re) {
        ar = a; r = rb; r_end = re;
        pos = ar[2 * r];
        end = ar[2 * r + 1];
    }
    __device__ void init_range(int k0, int k1) {
        ar = nullptr; r = 0; r_end = 1; pos = k0; end = k1;
    }
    __device__ bool valid() const { return r < r_end; }
    // current tile start and valid-key count; then advance
    __device__ void next(int& key0, int& nvalid) {
        key0 = pos;
        nvalid = min(kKT, end - pos);
        pos += kKT;
        if (pos >= end) {
            ++r;
            if (ar && r < r_end) {
                pos = ar[2 * r];
                end = ar[2 * r + 1];
            }
        }
    }
};

template <int D>
__device__ __forceinline__ void load_kv_tile(AttnSmem<D>& sm, int stage, const __nv_bfloat16* Kb,
                                             const __nv_bfloat16* Vb, int key0, int nvalid,
                                             int tid) {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    const uint32_t kbase = smem_u32(sm.k[stage]), vbase = smem_u32(sm.v[stage]);
    for (int i = tid; i < kKT * CH; i += 256) {
        const int row = i / CH, ch = i % CH;
        const bool ok = row < nvalid;
        const size_t g = size_t(key0 + (ok ? row : 0)) * D + ch * 8;
        cp_async16(kbase + swz<D>(row, ch), Kb + g, ok ? 16 : 0);
        cp_async16(vbase + swz<D>(row, ch), Vb + g, ok ? 16 : 0);
    }
}

template <int D>
__global__ void __launch_bounds__(256, 2)
    attend_mma_kernel(DevLayout dv, int BH, int k, float scale_log2, int64_t n_anchor,
                      const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                      const __nv_bfloat16* __restrict__ V, int32_t* __restrict__ hdr,
                      const int32_t* __restrict__ qoff, const int32_t* __restrict__ tile_off,
                      const int32_t* __restrict__ qlist, float* __restrict__ lse_p,
                      float* __restrict__ o_p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(smem_raw);
    constexpr int CH = D / 8;
    constexpr int NT = D / 8;  // 8-wide output column tiles
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int S = k + 1;
    const size_t L = size_t(dv.L);

    for (;;) {
        if (tid == 0) sm.item = atomicAdd(&hdr[HDR_WORK], 1);
        __syncthreads();
        const int64_t item = sm.item;
        ItemInfo it;
        if (!decode_item(dv, BH, n_anchor, item, tile_off, qoff, qlist, it)) break;
        const __nv_bfloat16* Qb = Q + size_t(it.bh) * L * D;
        const __nv_bfloat16* Kb = K + size_t(it.bh) * L * D;
        const __nv_bfloat16* Vb = V + size_t(it.bh) * L * D;

        // query rows of the item
        if (tid < kQTile) {
            int tok = -1, slot = 0;
            if (tid < it.nq) {
                if (it.slot_fixed >= 0) {
                    tok = it.q0 + tid;
                    slot = it.slot_fixed;
                } else {
                    const int e = it.entries[tid];
                    tok = e >> 5;
                    slot = 1 + (e & 31);
                }
            }
            sm.tok[tid] = tok;
            sm.slot[tid] = slot;
        }
        __syncthreads();
        {
            const uint32_t qbase = smem_u32(sm.q);
            for (int i = tid; i < kQTile * CH; i += 256) {
                const int row = i / CH, ch = i % CH;
                const int tok = sm.tok[row];
                cp_async16(qbase + swz<D>(row, ch), Qb + size_t(tok < 0 ? 0 : tok) * D + ch * 8,
                           tok < 0 ? 0 : 16);
            }
        }
        TileCursor cur;
        if (it.r_beg >= 0) cur.init_anchor(dv.ar, it.r_beg, it.r_end);
        else cur.init_range(it.k0, it.k1);
        int key0, nvalid;
        cur.next(key0, nvalid);
        load_kv_tile<D>(sm, 0, Kb, Vb, key0, nvalid, tid);
        cp_async_commit();

        float o[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        const int qr = warp * 16;
        int stage = 0;
        for (;;) {
            const int cur_valid = nvalid;
            const bool more = cur.valid();
            if (more) {
                cur.next(key0, nvalid);
                load_kv_tile<D>(sm, stage ^ 1, Kb, Vb, key0, nvalid, tid);
                cp_async_commit();
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();

            // S = Q K^T for this warp's 16 rows x 64 keys
            float s[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
            const uint32_t qbase = smem_u32(sm.q), kbase = smem_u32(sm.k[stage]);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t a[4];
                {
                    const int mi = lane >> 3;
                    const int row = qr + (lane & 7) + (mi & 1) * 8;
                    ldmatrix_x4(qbase + swz<D>(row, ks * 2 + (mi >> 1)), a[0], a[1], a[2], a[3]);
                }
#pragma unroll
                for (int jp = 0; jp < 4; ++jp) {
                    const int mi = lane >> 3;
                    const int key = jp * 16 + (lane & 7) + (mi >> 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(kbase + swz<D>(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
                    mma_bf16_16816(s[2 * jp], a, b0, b1);
                    mma_bf16_16816(s[2 * jp + 1], a, b2, b3);
                }
            }
            // mask keys past the range end; online softmax (scores in log2 units)
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = j * 8 + 2 * t4 + e;
                    const bool ok = col < cur_valid;
                    s[j][e] = ok ? s[j][e] * scale_log2 : -INFINITY;
                    s[j][2 + e] = ok ? s[j][2 + e] * scale_log2 : -INFINITY;
                    mx0 = fmaxf(mx0, s[j][e]);
                    mx1 = fmaxf(mx1, s[j][2 + e]);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            float rs0 = 0.f, rs1 = 0.f;
            uint32_t p[4][4];  // P as A fragments, one per 16-key step
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float p0 = exp2f(s[j][0] - mn0), p1 = exp2f(s[j][1] - mn0);
                const float p2 = exp2f(s[j][2] - mn1), p3 = exp2f(s[j][3] - mn1);
                rs0 += p0 + p1;
                rs1 += p2 + p3;
                p[j >> 1][(j & 1) * 2 + 0] = pack_bf16(p0, p1);
                p[j >> 1][(j & 1) * 2 + 1] = pack_bf16(p2, p3);
            }
            l0 = l0 * al0 + rs0;
            l1 = l1 * al1 + rs1;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                o[j][0] *= al0; o[j][1] *= al0;
                o[j][2] *= al1; o[j][3] *= al1;
            }
            // O += P V
            const uint32_t vbase = smem_u32(sm.v[stage]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                // A fragment order: a0 (row g, keys 0-7), a1 (row g+8, keys 0-7),
                // a2 (row g, keys 8-15), a3 (row g+8, keys 8-15) of this 16-key step
                uint32_t a[4] = {p[kk][0], p[kk][1], p[kk][2], p[kk][3]};
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    const int mi = lane >> 3;
                    const int key = kk * 16 + (lane & 7) + (mi & 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(vbase + swz<D>(key, np * 2 + (mi >> 1)), b0, b1, b2, b3);
                    mma_bf16_16816(o[2 * np], a, b0, b1);
                    mma_bf16_16816(o[2 * np + 1], a, b2, b3);
                }
            }
            __syncthreads();  // this stage is free for the next prefetch
            stage ^= 1;
            if (!more) break;
        }
        // epilogue: normalise, write the partial rows and their log-sum-exp
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const float inv0 = 1.f / l0, inv1 = 1.f / l1;
        const int ra = qr + g8, rb = qr + g8 + 8;
        const int ta = sm.tok[ra], tb = sm.tok[rb];
        if (ta >= 0) {
            const size_t base = (size_t(it.bh) * L + ta) * S + sm.slot[ra];
            float* dst = o_p + base * D;
#pragma unroll
            for (int j = 0; j < NT; ++j)
                *reinterpret_cast<float2*>(dst + j * 8 + 2 * t4) = make_float2(o[j][0] * inv0, o[j][1] * inv0);
            if (t4 == 0) lse_p[base] = (m0 + log2f(l0)) * 0.69314718055994531f;
        }
        if (tb >= 0) {
            const size_t base = (size_t(it.bh) * L + tb) * S + sm.slot[rb];
            float* dst = o_p + base * D;
#pragma unroll
            for (int j = 0; j < NT; ++j)
                *reinterpret_cast<float2*>(dst + j * 8 + 2 * t4) = make_float2(o[j][2] * inv1, o[j][3] * inv1);
            if (t4 == 0) lse_p[base] = (m1 + log2f(l1)) * 0.69314718055994531f;
        }
        __syncthreads();  // tok/slot and q are rewritten by the next item
    }
}

template <int D>
cudaError_t launch_d(const DevLayout& dv, int BH, const void* Q, const void* K, const void* V,
                     int k, float scale, int64_t n_anchor, char* ws, const WsPlan& p,
                     cudaStream_t s) {
    const int smem = int(sizeof(AttnSmem<D>));
    cudaError_t e = cudaFuncSetAttribute(attend_mma_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attend_mma_kernel<D>, 256, smem);
    if (per_sm < 1) per_sm = 1;
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    e = cudaMemsetAsync(hdr + HDR_WORK, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    attend_mma_kernel<D><<<sms * per_sm, 256, smem, s>>>(
        dv, BH, k, scale * 1.4426950408889634f, n_anchor, static_cast<const __nv_bfloat16*>(Q),
        static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), hdr,
        reinterpret_cast<const int32_t*>(ws + p.qoff), reinterpret_cast<const int32_t*>(ws + p.tile_off),
        reinterpret_cast<const int32_t*>(ws + p.qlist), reinterpret_cast<float*>(ws + p.lse_p),
        reinterpret_cast<float*>(ws + p.o_p));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_mma(const DevLayout& dv, int BH, int d, const void* Q, const void* K,
                              const void* V, int k, float scale, int64_t n_anchor, char* ws,
                              const WsPlan& p, cudaStream_t s) {
    if (d == 128) return launch_d<128>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, s);
    return launch_d<64>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, s);
}

}  // namespace moc

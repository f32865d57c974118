// Backward pass of the attention over Omega(q), query side: dQ.
//
// "Mixture of Contexts for Long Video Generation | Summary", appendix
// (training details): the model is trained through a custom autograd function
// whose gradient is the attention's over the selected keys and values; the
// top-k choice itself is discrete and gets no gradient, so the selection is a
// constant here. For a query row t with output o_t, log-sum-exp lse_t and
// upstream gradient dO_t, and every key u of Omega(t):
//   p_tu = exp(scale * q_t . k_u - lse_t),   D_t = dO_t . o_t,
//   ds_tu = p_tu * (dO_t . v_u - D_t),        dq_t = scale * sum_u ds_tu k_u.
// Omega(t) is cut into the forward pass's work items (items.cuh); every item
// gives dq_t's part over its keys, written to the row's partial slot, and a
// reduce kernel adds a row's parts in fixed slot order (deterministic).
//
// One CTA per SM, 384 threads, one 128-row query tile per work unit (the upper
// or lower half of a forward item). TMEM: two S buffers, dP and the dQ
// accumulator (4 x 128 columns).
//   warp 8 (one lane): scheduler + TMA producer: K tiles into a 3-stage ring
//          (a K tile serves S(j) and, two tiles later, dQ(j)), V tiles into a
//          2-stage ring.
//   warp 9 (one lane): issues S(j) = Q K(j)^T two tiles ahead into buffer j&1,
//          dP(j) = dO V(j)^T, and dQ += dS(j) K(j) with dS read from TMEM and
//          K(j) from shared memory (MN-major).
//   warps 0-7: two warpgroups, each owning half of every tile's 128 key
//          columns for all 128 rows (one thread per row = TMEM lane). They
//          gather the unit's Q and dO rows into the swizzled shared layout
//          (warpgroup 0: Q, warpgroup 1: dO) at its start; per key tile they
//          load their halves of S and dP, form dS in fp32 and write it as bf16
//          pairs over the first 32 columns of their own half of S's buffer
//          (keys 64 w .. 64 w + 63 at columns 64 w .. 64 w + 31), so neither
//          warpgroup writes columns the other still reads; at the end they
//          scale dQ and store the partial row.
// Every wait is bounded, as in the forward kernel.
#include "items.cuh"
#include "pipeline.cuh"
#include "tmap.cuh"

namespace moc {
namespace {

using namespace sm100;
using items::count_tiles;
using items::Cursor;
using items::decode;
using items::Item;
using items::kKT;

constexpr int kThreads = 384;
// launched at 168 registers a thread (384 x 168 = 64512); compute warpgroups
// rise to 216, the producer / MMA warpgroup drops to 72: 2 x 128 x 216 + 128 x 72 = 64512
constexpr int kRegsCompute = 216;
constexpr int kRegsOther = 72;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColDP = 256, kColDQ = 384;

template <int D>
struct DqCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;
    static constexpr int kKStages = 3, kVStages = 2;
    static constexpr int oQ = 0;
    static constexpr int oDO = oQ + kTileBytes;
    static constexpr int oK = oDO + kTileBytes;
    static constexpr int oV = oK + kKStages * kTileBytes;
    static constexpr int oBar = oV + kVStages * kTileBytes;
    static constexpr int kSmem = (oBar + 512 + 1024) > 120 * 1024 ? (oBar + 512 + 1024) : 120 * 1024;
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static constexpr uint32_t kIdescSS = idesc_bf16_f32(128, kKT, 0);  // S = Q K^T, dP = dO V^T
    static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, 1);    // dQ += dS K
};

enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY = 2, B_K_FULL = 4, B_K_EMPTY = 7, B_V_FULL = 10, B_V_EMPTY = 12,
    B_QDO_FULL = 14, B_S_FULL = 15, B_DP_FULL = 17, B_DS_FULL = 18, B_DQ_DONE = 19, B_MMA_DONE = 20,
    B_COUNT = 21
};

struct Shared {  // at oBar + 256
    int item[2];
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t col_s(int b) { return b ? kColS1 : kColS0; }
// TMEM column (from a buffer's first) of the bf16 pairs of keys 16 kk .. 16 kk + 15:
// warpgroup kk / 4 wrote keys 64 (kk / 4) .. + 63 at the start of its own half
__device__ __forceinline__ uint32_t ds_col(int kk) { return 64u * uint32_t(kk >> 2) + 8u * uint32_t(kk & 3); }

// Rows [r0, r0 + nq) of a forward item form one unit; nq <= 0: nothing to do.
__device__ __forceinline__ int unit_rows(const Item& it, int half) { return min(kQTile, it.nq - half * kQTile); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  DevLayout dv, int BH, int k, float scale, int64_t n_anchor,
                  const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ dO,
                  const float* __restrict__ lse, const float* __restrict__ Dsum, int32_t* __restrict__ hdr,
                  const int32_t* __restrict__ qoff, const int32_t* __restrict__ tile_off,
                  const int32_t* __restrict__ qlist, float* __restrict__ dq_p) {
    using C = DqCfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::oQ, sDO = base + C::oDO, sK = base + C::oK, sV = base + C::oV;
    const uint32_t sBar = base + C::oBar;
    Shared& sh = *reinterpret_cast<Shared*>(gbase + C::oBar + 256);
    volatile int* abort = &sh.abort;
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = k + 1;
    const size_t L = size_t(dv.L);
    const float scale_log2 = scale * 1.4426950408889634f;

    if (tid == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(B_ITEM_FULL + x), 1);
            mbar_init(bar(B_ITEM_EMPTY + x), 1 + 256);
            mbar_init(bar(B_V_FULL + x), 1);
            mbar_init(bar(B_V_EMPTY + x), 1);
            mbar_init(bar(B_S_FULL + x), 1);
        }
        for (int x = 0; x < 3; ++x) {
            mbar_init(bar(B_K_FULL + x), 1);
            mbar_init(bar(B_K_EMPTY + x), 1);
        }
        mbar_init(bar(B_QDO_FULL), 256);
        mbar_init(bar(B_DP_FULL), 1);
        mbar_init(bar(B_DS_FULL), 256);
        mbar_init(bar(B_DQ_DONE), 1);
        mbar_init(bar(B_MMA_DONE), 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int64_t n_units = 2 * (n_anchor + int64_t(tile_off[int64_t(BH) * dv.C]));

    if (warp >= 8) {
        regs_dec<kRegsOther>();
        if (warp == 8 && lane == 0) {
            // ------------------------------------------------------------ scheduler + producer
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t gk = 0, gv = 0;
            for (int it = 0;; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_EMPTY + slot), ((it >> 1) & 1) ^ 1, abort, hdr, 31)) break;
                const int64_t u = atomicAdd(&hdr[HDR_WORK], 1);
                const bool ok = u < n_units;
                sh.item[slot] = ok ? int(u) : -1;
                mbar_arrive(bar(B_ITEM_FULL + slot));
                if (!ok) break;
                Item itm;
                decode(dv, BH, n_anchor, u >> 1, tile_off, qoff, qlist, itm);
                if (unit_rows(itm, int(u & 1)) <= 0) continue;
                Cursor cur;
                cur.init(dv, itm);
                const int row0 = itm.bh * dv.L;
                bool stop = false;
                while (cur.more()) {
                    int key0, nvalid;
                    cur.next(key0, nvalid);
                    const uint32_t ks = gk % 3, vs = gv & 1;
                    if (!wait_bar(bar(B_K_EMPTY + ks), ((gk / 3) & 1) ^ 1, abort, hdr, 32)) { stop = true; break; }
                    mbar_expect_tx(bar(B_K_FULL + ks), C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_2d(sK + ks * C::kTileBytes + s * C::kSlabBytes, &tmK, bar(B_K_FULL + ks), 64 * s,
                                    row0 + key0);
                    ++gk;
                    if (!wait_bar(bar(B_V_EMPTY + vs), ((gv >> 1) & 1) ^ 1, abort, hdr, 33)) { stop = true; break; }
                    mbar_expect_tx(bar(B_V_FULL + vs), C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_2d(sV + vs * C::kTileBytes + s * C::kSlabBytes, &tmV, bar(B_V_FULL + vs), 64 * s,
                                    row0 + key0);
                    ++gv;
                }
                if (stop) break;
            }
            // every issued load lands before the CTA exits
            for (uint32_t g = (gk >= 3 ? gk - 3 : 0); g < gk; ++g) drain_bar(bar(B_K_FULL + g % 3), (g / 3) & 1, hdr, 34);
            for (uint32_t g = (gv >= 2 ? gv - 2 : 0); g < gv; ++g) drain_bar(bar(B_V_FULL + (g & 1)), (g >> 1) & 1, hdr, 35);
        } else if (warp == 9 && lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            uint32_t gk = 0, gv = 0, gt = 0, nu = 0, ns[2] = {0, 0};
            bool stop = false;
            auto issue_s = [&](uint32_t kt, int b) -> bool {  // S(b) = Q K(kt)^T
                const uint32_t ks = kt % 3;
                if (!wait_bar(bar(B_K_FULL + ks), (kt / 3) & 1, abort, hdr, 36)) return false;
                tc_fence_after();
                const uint32_t kb = sK + ks * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    umma_ss(tmem + col_s(b), sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                            C::kIdescSS, kk > 0);
                }
                umma_commit(bar(B_S_FULL + b));
                ++ns[b];
                return true;
            };
            auto issue_dp = [&]() -> bool {  // dP = dO V(gv)^T, then V(gv) is free
                const uint32_t vs = gv & 1;
                if (!wait_bar(bar(B_V_FULL + vs), (gv >> 1) & 1, abort, hdr, 37)) return false;
                tc_fence_after();
                const uint32_t vb = sV + vs * C::kTileBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                    umma_ss(tmem + kColDP, sdesc_sw128(sDO + off, 16, 1024), sdesc_sw128(vb + off, 16, 1024),
                            C::kIdescSS, kk > 0);
                }
                umma_commit(bar(B_DP_FULL));
                umma_commit(bar(B_V_EMPTY + vs));
                ++gv;
                return true;
            };
            for (int it = 0; !stop; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 38)) break;
                const int u = sh.item[slot];
                mbar_arrive(bar(B_ITEM_EMPTY + slot));
                if (u < 0) break;
                Item itm;
                decode(dv, BH, n_anchor, u >> 1, tile_off, qoff, qlist, itm);
                if (unit_rows(itm, u & 1) <= 0) continue;
                const int T = count_tiles(dv, itm);
                if (!wait_bar(bar(B_QDO_FULL), nu & 1, abort, hdr, 39)) break;
                ++nu;
                tc_fence_after();
                if (!issue_s(gk, 0) || !issue_dp() || (T > 1 && !issue_s(gk + 1, 1))) break;
                for (int j = 0; j < T; ++j) {
                    if (!wait_bar(bar(B_DS_FULL), gt & 1, abort, hdr, 40)) { stop = true; break; }
                    tc_fence_after();
                    ++gt;
                    if (j + 1 < T && !issue_dp()) { stop = true; break; }
                    // dQ += dS(j) K(j): dS as bf16 pairs over the first 64 columns of S(j)'s buffer
                    const uint32_t ks = (gk + j) % 3;
                    const uint32_t kb = sK + ks * C::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kKT / 16; ++kk)
                        umma_ts(tmem + kColDQ, tmem + col_s(j & 1) + ds_col(kk),
                                sdesc_sw128(kb + kk * 2048, C::kSlabBytes, 1024), C::kIdescDQ, (j > 0 || kk > 0));
                    umma_commit(bar(B_K_EMPTY + ks));
                    if (j + 2 < T && !issue_s(gk + j + 2, j & 1)) { stop = true; break; }
                }
                if (stop) break;
                gk += T;
                umma_commit(bar(B_DQ_DONE));
            }
            umma_commit(bar(B_MMA_DONE));
            drain_bar(bar(B_MMA_DONE), 0, hdr, 41);
        }
        __syncwarp();
    } else {
        regs_inc<kRegsCompute>();
        // ------------------------------------------------------------ compute (warps 0-7)
        const int wg = warp >> 2;           // half of the key columns: [64 wg, 64 wg + 64)
        const int row = tid & 127;          // query row in the tile = TMEM lane
        const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
        uint32_t gt = 0, nu = 0, ns[2] = {0, 0};
        for (int it = 0;; ++it) {
            const int slot = it & 1;
            if (!wait_bar_warp(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 42)) break;
            const int u = sh.item[slot];
            mbar_arrive(bar(B_ITEM_EMPTY + slot));
            if (u < 0) break;
            Item itm;
            decode(dv, BH, n_anchor, u >> 1, tile_off, qoff, qlist, itm);
            const int half = u & 1, nq = unit_rows(itm, half);
            if (nq <= 0) continue;
            int my_tok = -1, my_slot = 0;
            if (row < nq) {
                const int r_item = half * kQTile + row;
                if (itm.slot_fixed >= 0) {
                    my_tok = itm.q0 + r_item;
                } else {
                    const int e = itm.entries[r_item];
                    my_tok = e >> 5;
                    my_slot = 1 + (e & 31);
                }
            }
            const size_t rowg = size_t(itm.bh) * L + (my_tok >= 0 ? my_tok : 0);
            // padding rows: lse = +inf makes every p zero, so their dS is zero too
            const float lse2 = my_tok >= 0 ? __ldg(lse + rowg) * 1.4426950408889634f : INFINITY;
            const float drow = my_tok >= 0 ? __ldg(Dsum + rowg) : 0.f;
            // gather this warp's 32 rows of Q (warpgroup 0) or dO (warpgroup 1)
            {
                constexpr int CH = D / 8;
                const __nv_bfloat16* src = (wg == 0 ? Q : dO) + size_t(itm.bh) * L * D;
                const uint32_t dstb = wg == 0 ? sQ : sDO;
                uint4 v[CH];
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const int tok = __shfl_sync(0xffffffffu, my_tok, (i * 32 + lane) / CH);
                    v[i] = make_uint4(0, 0, 0, 0);
                    if (tok >= 0) v[i] = ldg_nc16(src + size_t(tok) * D + ((i * 32 + lane) % CH) * 8);
                }
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const int idx = i * 32 + lane;
                    const int r = (warp & 3) * 32 + idx / CH, ch = idx % CH;
                    const uint32_t dst = dstb + (ch >> 3) * C::kSlabBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v[i].x), "r"(v[i].y),
                                 "r"(v[i].z), "r"(v[i].w) : "memory");
                }
                fence_proxy_async_smem();
                mbar_arrive(bar(B_QDO_FULL));
            }
            ++nu;
            Cursor cur;
            cur.init(dv, itm);
            bool stop = false;
            for (int j = 0; cur.more(); ++j) {
                int key0, nvalid;
                cur.next(key0, nvalid);
                const int b = j & 1;
                if (!wait_bar_warp(bar(B_S_FULL + b), ns[b] & 1, abort, hdr, 43)) { stop = true; break; }
                ++ns[b];
                if (!wait_bar_warp(bar(B_DP_FULL), gt & 1, abort, hdr, 44)) { stop = true; break; }
                tc_fence_after();
                uint32_t s[64], p[64];
                tmem_ld32(lane_addr + col_s(b) + 64 * wg, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
                tmem_ld32(lane_addr + col_s(b) + 64 * wg + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
                tmem_ld32(lane_addr + kColDP + 64 * wg, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
                tmem_ld32(lane_addr + kColDP + 64 * wg + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
                tmem_wait_ld_regs(s);
                tmem_wait_ld_regs(p);
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int key = 64 * wg + 2 * c;
                    float d0 = 0.f, d1 = 0.f;
                    if (key < nvalid)
                        d0 = ex2(fmaf(__uint_as_float(s[2 * c]), scale_log2, -lse2)) * (__uint_as_float(p[2 * c]) - drow);
                    if (key + 1 < nvalid)
                        d1 = ex2(fmaf(__uint_as_float(s[2 * c + 1]), scale_log2, -lse2)) *
                             (__uint_as_float(p[2 * c + 1]) - drow);
                    pk[c] = pack_bf16(d0, d1);
                }
                tmem_st32(lane_addr + col_s(b) + 64 * wg, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_DS_FULL));
                ++gt;
            }
            if (stop) break;
            // epilogue: dq_t = scale * (sum over the unit's keys of ds_tu k_u) -> partial slot
            if (!wait_bar_warp(bar(B_DQ_DONE), (nu - 1) & 1, abort, hdr, 46)) break;
            tc_fence_after();
            constexpr int HC = D / 2;  // dQ columns of this warpgroup
            float* dst = my_tok >= 0 ? dq_p + (rowg * S + my_slot) * D + wg * HC : nullptr;
#pragma unroll
            for (int c0 = 0; c0 < HC; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(lane_addr + kColDQ + wg * HC + c0, o);
                tmem_wait_ld_regs(o);
                if (dst) {
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        *reinterpret_cast<float4*>(dst + c0 + 4 * x) =
                            make_float4(__uint_as_float(o[4 * x]) * scale, __uint_as_float(o[4 * x + 1]) * scale,
                                        __uint_as_float(o[4 * x + 2]) * scale, __uint_as_float(o[4 * x + 3]) * scale);
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// D_t = dO_t . o_t in fp32 (bf16 inputs), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_rowdot_kernel(int64_t rows, const __nv_bfloat16* __restrict__ O,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         float* __restrict__ Dsum) {
    constexpr int PER = D / 32;  // elements per lane
    const int lane = threadIdx.x & 31;
    for (int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
         row += (int64_t(gridDim.x) * blockDim.x) >> 5) {
        const size_t off = size_t(row) * D + lane * PER;
        float acc = 0.f;
        if (PER == 4) {
            const uint2 a = __ldg(reinterpret_cast<const uint2*>(O + off));
            const uint2 b = __ldg(reinterpret_cast<const uint2*>(dO + off));
            acc = bf16lo(a.x) * bf16lo(b.x) + bf16hi(a.x) * bf16hi(b.x) + bf16lo(a.y) * bf16lo(b.y) +
                  bf16hi(a.y) * bf16hi(b.y);
        } else {
            const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(O + off));
            const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(dO + off));
            acc = bf16lo(a) * bf16lo(b) + bf16hi(a) * bf16hi(b);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) Dsum[row] = acc;
    }
}

// dQ_t = sum of the row's partials (slot 0, then slot 1 + x for every valid
// selection x, in that order), rounded to bf16. One warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_reduce_kernel(int64_t rows, int k, int C,
                                                            const int32_t* __restrict__ sel,
                                                            const float* __restrict__ dq_p,
                                                            __nv_bfloat16* __restrict__ dQ) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int S = k + 1;
    for (int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
         row += (int64_t(gridDim.x) * blockDim.x) >> 5) {
        int32_t sj = -1;
        if (lane < k) sj = __ldg(sel + row * k + lane);
        const unsigned vmask = __ballot_sync(0xffffffffu, lane < k && sj >= 0 && sj < C);
        const float* src = dq_p + size_t(row) * S * D + lane * PER;
        float acc[PER];
#pragma unroll
        for (int x = 0; x < PER; ++x) acc[x] = src[x];
        for (unsigned m = vmask; m; m &= m - 1) {
            const int j = __ffs(m);  // slot 1 + x
#pragma unroll
            for (int x = 0; x < PER; ++x) acc[x] += src[size_t(j) * D + x];
        }
        __nv_bfloat16* out = dQ + size_t(row) * D + lane * PER;
        if (PER == 4) {
            *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]));
        } else {
            *reinterpret_cast<uint32_t*>(out) = pack_bf16(acc[0], acc[1]);
        }
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int D>
cudaError_t launch_dq_d(const DevLayout& dv, int BH, const void* Q, const void* K, const void* V,
                        const void* dO, const float* lse, int k, float scale, int64_t n_anchor, char* ws,
                        const WsPlan& p, cudaStream_t s) {
    CUtensorMap tmK, tmV;
    const int64_t rows = int64_t(BH) * dv.L;
    if (!make_tmap(&tmK, K, D, rows) || !make_tmap(&tmV, V, D, rows)) return cudaErrorInvalidValue;
    const int smem = DqCfg<D>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    e = cudaMemsetAsync(hdr + HDR_WORK, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<D><<<sm_count(), kThreads, smem, s>>>(
        tmK, tmV, dv, BH, k, scale, n_anchor, static_cast<const __nv_bfloat16*>(Q),
        static_cast<const __nv_bfloat16*>(dO), lse, reinterpret_cast<const float*>(ws + p.lse_p), hdr,
        reinterpret_cast<const int32_t*>(ws + p.qoff), reinterpret_cast<const int32_t*>(ws + p.tile_off),
        reinterpret_cast<const int32_t*>(ws + p.qlist), reinterpret_cast<float*>(ws + p.o_p));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_rowdot(int BH, int L, int d, const void* O, const void* dO, char* ws, const WsPlan& p,
                              cudaStream_t s) {
    const int64_t rows = int64_t(BH) * L;
    const int64_t want = (rows + 7) / 8;
    const int grid = int(want < int64_t(sm_count()) * 16 ? want : int64_t(sm_count()) * 16);
    float* Dsum = reinterpret_cast<float*>(ws + p.lse_p);
    const auto* o = static_cast<const __nv_bfloat16*>(O);
    const auto* g = static_cast<const __nv_bfloat16*>(dO);
    if (d == 128) bwd_rowdot_kernel<128><<<grid, 256, 0, s>>>(rows, o, g, Dsum);
    else bwd_rowdot_kernel<64><<<grid, 256, 0, s>>>(rows, o, g, Dsum);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                          const void* dO, const float* lse, int k, float scale, int64_t n_anchor, char* ws,
                          const WsPlan& p, cudaStream_t s) {
    if (d == 128) return launch_dq_d<128>(dv, BH, Q, K, V, dO, lse, k, scale, n_anchor, ws, p, s);
    return launch_dq_d<64>(dv, BH, Q, K, V, dO, lse, k, scale, n_anchor, ws, p, s);
}

cudaError_t launch_bwd_dq_reduce(int BH, int L, int C, int d, int k, const int32_t* sel, void* dQ, const char* ws,
                                 const WsPlan& p, cudaStream_t s) {
    const int64_t rows = int64_t(BH) * L;
    const int64_t want = (rows + 7) / 8;
    const int grid = int(want < int64_t(sm_count()) * 16 ? want : int64_t(sm_count()) * 16);
    const float* dq_p = reinterpret_cast<const float*>(ws + p.o_p);
    auto* out = static_cast<__nv_bfloat16*>(dQ);
    if (d == 128) bwd_dq_reduce_kernel<128><<<grid, 256, 0, s>>>(rows, k, C, sel, dq_p, out);
    else bwd_dq_reduce_kernel<64><<<grid, 256, 0, s>>>(rows, k, C, sel, dq_p, out);
    return cudaGetLastError();
}

}  // namespace moc

// Backward pass of the attention over Omega(q), key side: dK and dV.
//
// "Mixture of Contexts for Long Video Generation | Summary", appendix
// (training details): gradients reach the model through the attention over
// the selected keys and values; the selection is a constant. For a key u,
// summed over every query t whose Omega(t) holds u:
//   p_tu = exp(scale * q_t . k_u - lse_t),  ds_tu = p_tu * (dO_t . v_u - D_t),
//   dv_u = sum_t p_tu dO_t,                 dk_u = scale * sum_t ds_tu q_t.
// The queries that hold u are those of the query groups whose anchor ranges
// contain u's chunk (the layout's key blocks list them) and, for a video
// chunk, the queries that selected it (that chunk's query list from the
// query-list builder). A work unit is one 128-key tile of a key block: it owns
// its keys' dK and dV outright (no partials), so the result is deterministic.
//
// One CTA per SM, 512 threads. TMEM: S^T and dP^T (keys x 128 queries) and
// the dV and dK accumulators (4 x 128 columns).
//   warp 12 (one lane): scheduler + TMA of the unit's K and V tiles.
//   warps 8-11: gather each 128-query tile's Q and dO rows (cp.async, 16-byte
//          pieces straight into the 128-byte-swizzled layout, zero-filled past
//          the end of a list) and its lse and D = dO . o values into a 2-stage
//          ring.
//   warp 13 (one lane): per query tile S^T = K Q^T and dP^T = V dO^T (both
//          operands K-major in shared memory), then dV += P^T dO and
//          dK += dS^T Q with P^T and dS^T read from TMEM and dO, Q from shared
//          memory (MN-major).
//   warps 0-7: two warpgroups, each owning 64 of the tile's query columns for
//          all 128 keys (one thread per key = TMEM lane): P^T and dS^T from
//          S^T, dP^T, lse and D, written as bf16 pairs over the first 32
//          columns of the warpgroup's own halves of S^T and dP^T; at the end
//          they write the unit's dK (scaled) and dV rows in bf16.
// Every wait is bounded, as in the forward kernel.
#include "pipeline.cuh"
#include "tmap.cuh"

namespace moc {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
// launched at 128 registers a thread (512 x 128 = 65536): compute warpgroups 176,
// the gather warpgroup 104, the scheduler / MMA warpgroup 56:
// 2 x 128 x 176 + 128 x 104 + 128 x 56 = 65536; per SM sub-partition (one warp
// of each warpgroup) 32 x (176 + 176 + 104 + 56) = 16384.
constexpr int kRegsCompute = 176;
constexpr int kRegsGather = 104;
constexpr int kRegsOther = 56;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 384;

template <int D>
struct DkvCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kSlabBytes = 128 * 128;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;
    static constexpr int oK = 0;
    static constexpr int oV = oK + kTileBytes;
    static constexpr int oQ = oV + kTileBytes;       // 2 stages
    static constexpr int oDO = oQ + 2 * kTileBytes;  // 2 stages
    static constexpr int oStat = oDO + 2 * kTileBytes;  // [2 stages][lse2 | D][128] fp32
    static constexpr int oBar = oStat + 2 * 2 * 128 * 4;
    static constexpr int kSmem = (oBar + 512 + 1024) > 120 * 1024 ? (oBar + 512 + 1024) : 120 * 1024;
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0);  // S^T = K Q^T, dP^T = V dO^T
    static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 1);   // dV += P^T dO, dK += dS^T Q
};

enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY = 2, B_KV_FULL = 4, B_QT_FULL = 5, B_QT_EMPTY = 7, B_ST_FULL = 9,
    B_P_FULL = 10, B_KV_DONE = 11, B_MMA_DONE = 12, B_COUNT = 13
};

struct Shared {  // at oBar + 256
    int item[2];
    uint32_t tmem_base;
    int abort;
};

// A unit: one 128-key tile of a key block, for one (b, h).
struct KUnit {
    int bh, blk, k0, nk, chunk;
};

// Units in order: the leading blocks (caption runs, attended by every query: the
// longest units) block by block, each for every (b, h); then the video chunks'
// blocks head by head, so that the units running at one time share one head's
// query rows (a head's Q and dO stay in L2 while its chunks' units read them).
__device__ __forceinline__ void decode_k(const DevLayout& dv, int BH, int64_t u, KUnit& x) {
    const int64_t lead = int64_t(BH) * dv.kt_off[dv.kb_lead];
    int pos, tile;
    if (u < lead) {
        pos = upper_index(dv.kt_off, dv.NKB + 1, u / BH);
        const int64_t local = u - int64_t(BH) * dv.kt_off[pos];
        const int nt = dv.kt_off[pos + 1] - dv.kt_off[pos];
        x.bh = int(local / nt);
        tile = int(local % nt);
    } else {
        const int64_t per_head = dv.kt_off[dv.NKB] - dv.kt_off[dv.kb_lead];
        const int64_t r = u - lead;
        x.bh = int(r / per_head);
        const int64_t t = dv.kt_off[dv.kb_lead] + r % per_head;
        pos = upper_index(dv.kt_off, dv.NKB + 1, t);
        tile = int(t - dv.kt_off[pos]);
    }
    x.blk = dv.kb_order[pos];
    x.k0 = dv.kb_range[2 * x.blk] + tile * kQTile;
    x.nk = min(kQTile, dv.kb_range[2 * x.blk + 1] - x.k0);
    x.chunk = dv.kb_chunk[x.blk];
}

// The unit's query tiles in order: each anchoring group's queries in 128-row
// tiles, then the chunk's query list in 128-entry tiles.
struct QWalk {
    int g, g_end, q, q1;              // current group position, its query cursor / end
    const int32_t* ent;               // query list of the chunk (entries query << 5 | slot)
    int e, e_end;
    __device__ void init(const DevLayout& dv, const KUnit& x, const int32_t* qoff, const int32_t* qlist) {
        g = dv.kb_goff[x.blk];
        g_end = dv.kb_goff[x.blk + 1];
        q = q1 = 0;
        if (g < g_end) {
            q = dv.grp_q0[dv.kb_grp[g]];
            q1 = dv.grp_q1[dv.kb_grp[g]];
        }
        ent = nullptr;
        e = e_end = 0;
        if (x.chunk >= 0) {
            const int64_t l = int64_t(x.bh) * dv.C + x.chunk;
            ent = qlist;
            e = qoff[l];
            e_end = qoff[l + 1];
        }
    }
    // number of tiles (walks a copy)
    __device__ int count(const DevLayout& dv) const {
        int n = 0;
        for (int i = g; i < g_end; ++i) {
            const int gg = dv.kb_grp[i];
            n += (dv.grp_q1[gg] - dv.grp_q0[gg] + kQTile - 1) / kQTile;
        }
        return n + (e_end - e + kQTile - 1) / kQTile;
    }
    // next tile: anchor rows [r0, r0 + n) (list == nullptr) or list entries list[0 .. n)
    __device__ void next(const DevLayout& dv, int& r0, int& n, const int32_t*& list) {
        if (g < g_end) {
            r0 = q;
            n = min(kQTile, q1 - q);
            list = nullptr;
            q += kQTile;
            if (q >= q1 && ++g < g_end) {
                q = dv.grp_q0[dv.kb_grp[g]];
                q1 = dv.grp_q1[dv.kb_grp[g]];
            }
        } else {
            r0 = 0;
            n = min(kQTile, e_end - e);
            list = ent + e;
            e += kQTile;
        }
    }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   DevLayout dv, int BH, float scale, const __nv_bfloat16* __restrict__ Q,
                   const __nv_bfloat16* __restrict__ dO, const float* __restrict__ lse,
                   const float* __restrict__ Dsum, int32_t* __restrict__ hdr, const int32_t* __restrict__ qoff,
                   const int32_t* __restrict__ qlist, __nv_bfloat16* __restrict__ dK,
                   __nv_bfloat16* __restrict__ dV) {
    using C = DkvCfg<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sK = base + C::oK, sV = base + C::oV, sQ = base + C::oQ, sDO = base + C::oDO;
    float* stat = reinterpret_cast<float*>(gbase + C::oStat);  // [stage][0: lse2, 1: D][128]
    const uint32_t sBar = base + C::oBar;
    Shared& sh = *reinterpret_cast<Shared*>(gbase + C::oBar + 256);
    volatile int* abort = &sh.abort;
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t L = size_t(dv.L);
    const float scale_log2 = scale * 1.4426950408889634f;
    const int64_t n_units = int64_t(BH) * dv.kt_off[dv.NKB];

    if (tid == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(B_ITEM_FULL + x), 1);
            mbar_init(bar(B_ITEM_EMPTY + x), 1 + 256 + 128);
            mbar_init(bar(B_QT_FULL + x), 128);
            mbar_init(bar(B_QT_EMPTY + x), 1);
        }
        mbar_init(bar(B_KV_FULL), 1);
        mbar_init(bar(B_ST_FULL), 1);
        mbar_init(bar(B_P_FULL), 256);
        mbar_init(bar(B_KV_DONE), 1);
        mbar_init(bar(B_MMA_DONE), 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 13) {
        tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (warp >= 12) {
        regs_dec<kRegsOther>();
        if (warp == 12 && lane == 0) {
            // ------------------------------------------------------------ scheduler + K/V loads
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            uint32_t nkv = 0;
            for (int it = 0;; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_EMPTY + slot), ((it >> 1) & 1) ^ 1, abort, hdr, 51)) break;
                const int64_t u = atomicAdd(&hdr[HDR_WORK], 1);
                const bool ok = u < n_units;
                sh.item[slot] = ok ? int(u) : -1;
                mbar_arrive(bar(B_ITEM_FULL + slot));
                if (!ok) break;
                KUnit x;
                decode_k(dv, BH, u, x);
                // the previous unit's MMAs have read K and V
                if (!wait_bar(bar(B_KV_DONE), (nkv & 1) ^ 1, abort, hdr, 52)) break;
                mbar_expect_tx(bar(B_KV_FULL), 2 * C::kTileBytes);
#pragma unroll
                for (int s = 0; s < C::kSlabs; ++s) {
                    tma_load_2d(sK + s * C::kSlabBytes, &tmK, bar(B_KV_FULL), 64 * s, x.bh * dv.L + x.k0);
                    tma_load_2d(sV + s * C::kSlabBytes, &tmV, bar(B_KV_FULL), 64 * s, x.bh * dv.L + x.k0);
                }
                ++nkv;
            }
            if (nkv > 0) drain_bar(bar(B_KV_FULL), (nkv - 1) & 1, hdr, 53);
        } else if (warp == 13 && lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            uint32_t gq = 0, gt = 0, nu = 0;
            bool stop = false;
            for (int it = 0; !stop; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 54)) break;
                const int u = sh.item[slot];
                mbar_arrive(bar(B_ITEM_EMPTY + slot));
                if (u < 0) break;
                KUnit x;
                decode_k(dv, BH, u, x);
                QWalk w;
                w.init(dv, x, qoff, qlist);
                const int nqt = w.count(dv);
                if (!wait_bar(bar(B_KV_FULL), nu & 1, abort, hdr, 55)) break;
                ++nu;
                tc_fence_after();
                for (int i = 0; i < nqt; ++i) {
                    const uint32_t st = gq & 1;
                    if (!wait_bar(bar(B_QT_FULL + st), (gq >> 1) & 1, abort, hdr, 56)) { stop = true; break; }
                    tc_fence_after();
                    const uint32_t qb = sQ + st * C::kTileBytes, gb = sDO + st * C::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                        umma_ss(tmem + kColST, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(qb + off, 16, 1024),
                                C::kIdescSS, kk > 0);
                    }
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                        umma_ss(tmem + kColDPT, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(gb + off, 16, 1024),
                                C::kIdescSS, kk > 0);
                    }
                    umma_commit(bar(B_ST_FULL));
                    if (!wait_bar(bar(B_P_FULL), gt & 1, abort, hdr, 57)) { stop = true; break; }
                    tc_fence_after();
                    ++gt;
                    // queries 16 kk .. + 15 of P^T / dS^T: warpgroup kk / 4 wrote its 64
                    // queries over the first 32 columns of its own half
#pragma unroll
                    for (int kk = 0; kk < 128 / 16; ++kk) {
                        const uint32_t ac = 64u * uint32_t(kk >> 2) + 8u * uint32_t(kk & 3);
                        umma_ts(tmem + kColDV, tmem + kColST + ac, sdesc_sw128(gb + kk * 2048, C::kSlabBytes, 1024),
                                C::kIdescAcc, (i > 0 || kk > 0));
                    }
#pragma unroll
                    for (int kk = 0; kk < 128 / 16; ++kk) {
                        const uint32_t ac = 64u * uint32_t(kk >> 2) + 8u * uint32_t(kk & 3);
                        umma_ts(tmem + kColDK, tmem + kColDPT + ac, sdesc_sw128(qb + kk * 2048, C::kSlabBytes, 1024),
                                C::kIdescAcc, (i > 0 || kk > 0));
                    }
                    umma_commit(bar(B_QT_EMPTY + st));
                    ++gq;
                }
                if (stop) break;
                umma_commit(bar(B_KV_DONE));
            }
            umma_commit(bar(B_MMA_DONE));
            drain_bar(bar(B_MMA_DONE), 0, hdr, 58);
        }
        __syncwarp();
    } else if (warp >= 8) {
        regs_dec<kRegsGather>();
        // ------------------------------------------------------------ query-tile gather (warps 8-11)
        const int r = tid - 256;             // row of the tile this thread stages lse / D for
        const int wr = (warp - 8) * 32;      // this warp's 32 rows
        uint32_t gq = 0;
        constexpr int CH = D / 8;            // 16-byte pieces per row
        for (int it = 0;; ++it) {
            const int slot = it & 1;
            if (!wait_bar_warp(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 59)) break;
            const int u = sh.item[slot];
            mbar_arrive(bar(B_ITEM_EMPTY + slot));
            if (u < 0) break;
            KUnit x;
            decode_k(dv, BH, u, x);
            QWalk w;
            w.init(dv, x, qoff, qlist);
            const int nqt = w.count(dv);
            const __nv_bfloat16* Qb = Q + size_t(x.bh) * L * D;
            const __nv_bfloat16* Gb = dO + size_t(x.bh) * L * D;
            bool stop = false;
            for (int i = 0; i < nqt; ++i) {
                int r0, n;
                const int32_t* list;
                w.next(dv, r0, n, list);
                const uint32_t st = gq & 1;
                if (!wait_bar_warp(bar(B_QT_EMPTY + st), ((gq >> 1) & 1) ^ 1, abort, hdr, 60)) { stop = true; break; }
                int tok = -1;
                if (r < n) tok = list ? (list[r] >> 5) : r0 + r;
                const size_t rowg = size_t(x.bh) * L + (tok >= 0 ? tok : 0);
                stat[(st * 2 + 0) * 128 + r] = tok >= 0 ? __ldg(lse + rowg) * 1.4426950408889634f : INFINITY;
                stat[(st * 2 + 1) * 128 + r] = tok >= 0 ? __ldg(Dsum + rowg) : 0.f;
                // the warp's 32 rows, CH pieces each, in whole-row runs per instruction
#pragma unroll
                for (int i2 = 0; i2 < CH; ++i2) {
                    const int idx = i2 * 32 + lane;
                    const int rr = wr + idx / CH, ch = idx % CH;
                    const int t = __shfl_sync(0xffffffffu, tok, idx / CH);
                    const uint32_t off = (ch >> 3) * C::kSlabBytes + rr * 128 + (((ch & 7) ^ (rr & 7)) << 4);
                    const size_t src = size_t(t >= 0 ? t : 0) * D + ch * 8;
                    cp_async16(sQ + st * C::kTileBytes + off, Qb + src, t >= 0 ? 16 : 0);
                    cp_async16(sDO + st * C::kTileBytes + off, Gb + src, t >= 0 ? 16 : 0);
                }
                cp_async_commit();
                cp_async_wait<0>();
                fence_proxy_async_smem();
                mbar_arrive(bar(B_QT_FULL + st));
                ++gq;
            }
            if (stop) break;
        }
    } else {
        regs_inc<kRegsCompute>();
        // ------------------------------------------------------------ compute (warps 0-7)
        const int wg = warp >> 2;          // query columns [64 wg, 64 wg + 64)
        const int row = tid & 127;         // key row of the tile = TMEM lane
        const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
        uint32_t gq = 0, gt = 0, nu = 0;
        for (int it = 0;; ++it) {
            const int slot = it & 1;
            if (!wait_bar_warp(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 61)) break;
            const int u = sh.item[slot];
            mbar_arrive(bar(B_ITEM_EMPTY + slot));
            if (u < 0) break;
            KUnit x;
            decode_k(dv, BH, u, x);
            QWalk w;
            w.init(dv, x, qoff, qlist);
            const int nqt = w.count(dv);
            bool stop = false;
            for (int i = 0; i < nqt; ++i) {
                const uint32_t st = gq & 1;
                // the tile's lse / D were staged before QT_FULL; S^T and dP^T are in TMEM
                if (!wait_bar_warp(bar(B_QT_FULL + st), (gq >> 1) & 1, abort, hdr, 62)) { stop = true; break; }
                if (!wait_bar_warp(bar(B_ST_FULL), gt & 1, abort, hdr, 63)) { stop = true; break; }
                tc_fence_after();
                const float* l2 = stat + (st * 2 + 0) * 128 + 64 * wg;
                const float* dd = stat + (st * 2 + 1) * 128 + 64 * wg;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t s[32], g[32];
                    tmem_ld32(lane_addr + kColST + 64 * wg + 32 * c, s);
                    tmem_ld32(lane_addr + kColDPT + 64 * wg + 32 * c, g);
                    tmem_wait_ld_regs(s);
                    tmem_wait_ld_regs(g);
                    uint32_t pp[16], pd[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int q0 = 32 * c + 2 * e;
                        const float p0 = ex2(fmaf(__uint_as_float(s[2 * e]), scale_log2, -l2[q0]));
                        const float p1 = ex2(fmaf(__uint_as_float(s[2 * e + 1]), scale_log2, -l2[q0 + 1]));
                        pp[e] = pack_bf16(p0, p1);
                        pd[e] = pack_bf16(p0 * (__uint_as_float(g[2 * e]) - dd[q0]),
                                          p1 * (__uint_as_float(g[2 * e + 1]) - dd[q0 + 1]));
                    }
                    tmem_st16(lane_addr + kColST + 64 * wg + 16 * c, pp);
                    tmem_st16(lane_addr + kColDPT + 64 * wg + 16 * c, pd);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL));
                ++gt;
                ++gq;
            }
            if (stop) break;
            // epilogue: this warpgroup's half of the d columns of dV and dK for its key rows
            if (!wait_bar_warp(bar(B_KV_DONE), nu & 1, abort, hdr, 64)) break;
            ++nu;
            tc_fence_after();
            constexpr int HC = D / 2;
            const bool valid = row < x.nk;
            const size_t orow = (size_t(x.bh) * L + x.k0 + row) * D + wg * HC;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                __nv_bfloat16* out = t == 0 ? dV : dK;
                const float mul = t == 0 ? 1.f : scale;
#pragma unroll
                for (int c0 = 0; c0 < HC; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + (t == 0 ? kColDV : kColDK) + wg * HC + c0, o);
                    tmem_wait_ld_regs(o);
                    if (valid) {
#pragma unroll
                        for (int x4 = 0; x4 < 4; ++x4)
                            *reinterpret_cast<uint4*>(out + orow + c0 + 8 * x4) = make_uint4(
                                pack_bf16(__uint_as_float(o[8 * x4]) * mul, __uint_as_float(o[8 * x4 + 1]) * mul),
                                pack_bf16(__uint_as_float(o[8 * x4 + 2]) * mul, __uint_as_float(o[8 * x4 + 3]) * mul),
                                pack_bf16(__uint_as_float(o[8 * x4 + 4]) * mul, __uint_as_float(o[8 * x4 + 5]) * mul),
                                pack_bf16(__uint_as_float(o[8 * x4 + 6]) * mul, __uint_as_float(o[8 * x4 + 7]) * mul));
                    }
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_d(const DevLayout& dv, int BH, const void* Q, const void* K, const void* V, const void* dO,
                     const float* lse, float scale, char* ws, const WsPlan& p, void* dK, void* dVout,
                     cudaStream_t s) {
    CUtensorMap tmK, tmV;
    const int64_t rows = int64_t(BH) * dv.L;
    if (!make_tmap(&tmK, K, D, rows) || !make_tmap(&tmV, V, D, rows)) return cudaErrorInvalidValue;
    const int smem = DkvCfg<D>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    e = cudaMemsetAsync(hdr + HDR_WORK, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    bwd_dkv_kernel<D><<<sms, kThreads, smem, s>>>(
        tmK, tmV, dv, BH, scale, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(dO),
        lse, reinterpret_cast<const float*>(ws + p.lse_p), hdr, reinterpret_cast<const int32_t*>(ws + p.qoff),
        reinterpret_cast<const int32_t*>(ws + p.qlist), static_cast<__nv_bfloat16*>(dK),
        static_cast<__nv_bfloat16*>(dVout));
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkv(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                           const void* dO, const float* lse, float scale, char* ws, const WsPlan& p, void* dK,
                           void* dV, cudaStream_t s) {
    if (d == 128) return launch_d<128>(dv, BH, Q, K, V, dO, lse, scale, ws, p, dK, dV, s);
    return launch_d<64>(dv, BH, Q, K, V, dO, lse, scale, ws, p, dK, dV, s);
}

}  // namespace moc

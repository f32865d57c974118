// (2) Router: per-query top-k over candidate chunks, on the tcgen05 tensor
// cores.
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: each query
// scores candidate chunks by the dot product with their mean-pooled keys and
// keeps the k best, independently per head; §3.2: optional edges i->j are
// masked whenever j >= i before top-k. The jxzklqfsx.com MoC write-up,
// "計算效率": mandatory chunks are inserted before top-k so that the router
// spends no budget on them (they are not candidates).
//
// Work unit: a 128-query tile of one query group (all its queries share one
// candidate list) times a block of the group's candidates. One persistent CTA
// per SM walks a contiguous range of tiles - the ranges split the tiles by the
// layout's estimated per-tile cost, so CTAs holding the tiles of late shots
// (many candidates) take fewer of them - with NWG selection warpgroups
// (4 for k <= 8, else 2) and two more warps:
//   warp 4*NWG (one lane): streams each tile's Q rows (two 64-column,
//          128-byte-swizzled slabs) into a ring with TMA (5 stages when every
//          candidate list fits a 128-row operand block, else 2);
//   warp 4*NWG+1: owns 512 TMEM columns (one 512/NWG-column score buffer per
//          selection warpgroup). When the (head, group, 128- or 256-candidate
//          operand block) changes it converts the block's fp32 pooled keys into
//          swizzled bf16 operands hi = RN(Kbar) and lo = RN(Kbar - hi) - Q is
//          exact bf16, so the two bf16 products reproduce q . Kbar to ~2^-17
//          relative per term - and its lane 0 issues S = Q hi^T + Q lo^T for
//          each 512/NWG-candidate slice of the block (M=128, N = slice rounded
//          up to 16, K = d, fp32 accumulation in TMEM);
//   warps 0 .. 4*NWG-1: selection warpgroups taking tiles round robin; one
//          thread per query row (= TMEM lane) reads its scores from TMEM and
//          keeps a sorted top-KMAX list in registers with a branch-free
//          insertion network over packed score / position keys (lists of up
//          to 511 entries; candidates come in ascending id, so equal keys
//          order by lower chunk id), writing the first k entries (-1 padded)
//          after the tile's last slice. The network is a chain of dependent
//          max / min steps per row, so more warpgroups (more rows in flight
//          per scheduler) hide its latency.
// Tiles without candidates (caption groups, the first shot) are written as -1
// rows by their selection warpgroup and skip the other roles. Waits are
// bounded as in the attention kernel; a timeout is recorded in the layout's
// device error word.
#include "pipeline.cuh"
#include "tmap.cuh"

namespace moc {
namespace {

using namespace sm100;

constexpr int kIdNone = 0x7fffffff;

template <int KMAX>
struct RWarps {
    static constexpr int kNwg = KMAX <= 8 ? 4 : 2;   // selection warpgroups
    static constexpr int kSlice = 512 / kNwg;       // TMEM columns per warpgroup = candidates per MMA
    static constexpr int kThreads = kNwg * 128 + 64;
    static constexpr int kProducer = kNwg * 4, kIssuer = kNwg * 4 + 1;
};

// Shared memory of one CTA: a QS-stage ring of 128-row Q tiles and the hi / lo
// operand blocks of KBLK candidates. Groups with at most 128 candidates (every
// group of the eight-shot scene has <= 105) use KBLK = 128 with a 5-stage ring;
// up to 320 candidates (the ragged and stress scenes) KBLK = 320 with a 2-stage
// ring, so that a group's whole list sits in one block; larger lists KBLK = 256.
template <int D, int KBLK, int QS>
struct RCfg {
    static constexpr int kBlk = KBLK;                   // candidates per operand block
    static constexpr int kSlabs = D / 64;
    static constexpr int kQBytes = kSlabs * 128 * 128;  // one 128-row Q tile
    static constexpr int kKbSlab = KBLK * 128;          // KBLK rows x 128 B
    static constexpr int kKbBytes = kSlabs * kKbSlab;   // hi (or lo) block
    static constexpr int kQStages = QS;                 // Q ring depth
    static constexpr int oQ = 0;
    static constexpr int oHi = oQ + kQStages * kQBytes;
    static constexpr int oLo = oHi + kKbBytes;
    static constexpr int oBar = oLo + kKbBytes;
    static constexpr int kSmem = (oBar + 512 + 1024) > 120 * 1024 ? (oBar + 512 + 1024) : 120 * 1024;
    static_assert(QS <= 8, "barrier slots");
    static_assert(kSmem <= 227 * 1024, "shared memory");
};

// R_Q_FULL / R_Q_EMPTY: [ring stage]; R_S_FULL / R_S_FREE: [warpgroup]; R_KB_FREE: the MMAs that read the operand block are done
enum { R_Q_FULL = 0, R_Q_EMPTY = 8, R_S_FULL = 16, R_S_FREE = 20, R_KB_FREE = 24, R_MMA_DONE = 25 };

struct RShared {  // at oBar + 256 (after the barriers)
    uint32_t tmem_base;
    int abort;
    int64_t t_beg, t_end;  // this CTA's tile range
};

// First global tile t (head-major) whose cost prefix reaches `target`; tile costs
// are positive, so the prefix strictly increases.
__device__ int64_t tile_at_cost(const DevLayout& dv, int64_t rtiles, int causal, int64_t total_tiles,
                                int64_t target) {
    const int32_t* pre = dv.rcost[causal ? 1 : 0];
    const int64_t head = pre[rtiles];
    int64_t lo = 0, hi = total_tiles;
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        const int64_t cum = (mid / rtiles) * head + pre[mid % rtiles];
        if (cum >= target) hi = mid; else lo = mid + 1;
    }
    return lo;
}

// Insert (cs, cj) into a register list sorted by descending score (branch
// free: per entry one compare, a max / min pair for the scores and two
// selects for the ids; the carried score passes through a single min per
// entry). Candidates arrive in ascending chunk id (cj is the position in the
// ascending candidate list), so the strict ">" keeps an equal score behind the
// earlier, lower id - the list is ordered by (score desc, id asc) without ever
// comparing ids. The last entry drops out.
template <int KMAX>
__device__ __forceinline__ void topk_push(float (&ts)[KMAX], int (&tj)[KMAX], float cs, int cj) {
#pragma unroll
    for (int x = 0; x < KMAX; ++x) {
        const bool gt = cs > ts[x];
        const float ks = fmaxf(cs, ts[x]);
        const int kj = gt ? cj : tj[x];
        cs = fminf(cs, ts[x]);
        cj = gt ? tj[x] : cj;
        ts[x] = ks;
        tj[x] = kj;
    }
}

// For candidate lists of up to 511 entries (positions fit 9 bits): an
// order-preserving 32-bit key of a score with the candidate's position in its 9
// low bits (larger score first, then lower position), so an insertion step is one
// max and one min instead of a compare, a max / min pair and two selects. The
// score keeps all but the 9 lowest bits of its order-preserving integer image:
// scores closer than 2^-14 of their magnitude compare equal and go by position
// (chunk id), a gap well inside the 1e-4 relative near-tie tolerance that routing
// is checked with. (Eight-shot scene, k = 3: 0.383 -> 0.359 ms.)
__device__ __forceinline__ uint32_t pack_key(float s, int pos) {
    const uint32_t u = __float_as_uint(s);
    const uint32_t o = u ^ (uint32_t(int32_t(u) >> 31) | 0x80000000u);
    return (o & ~0x1FFu) | (0x1FFu - uint32_t(pos));
}
template <int KMAX>
__device__ __forceinline__ void topk_push_key(uint32_t (&t)[KMAX], uint32_t c) {
#pragma unroll
    for (int x = 0; x < KMAX; ++x) {
        const uint32_t hi = max(t[x], c);
        c = min(t[x], c);
        t[x] = hi;
    }
}

struct Tile {
    int bh, g, q0, nq, cbeg, ncand, nb;
};

// Walks a CTA's contiguous range of tiles (head-major, then the tiles of each
// query group in order). A group's table entries are read when the walk
// enters it, not per tile: each read is a dependent global load, and per-tile
// decoding used to cost every role thousands of cycles per tile.
template <int SLICE>
struct TileWalk {
    int bh, rt, g, rt0, rt1;  // head, tile within the head, its group and the group's tile range
    int gq0, gq1, cbeg, ncand;

    __device__ __forceinline__ void load_group(const DevLayout& dv, int causal) {
        rt0 = dv.rtile_off[g];
        rt1 = dv.rtile_off[g + 1];
        gq0 = dv.grp_q0[g];
        gq1 = dv.grp_q1[g];
        cbeg = dv.cand_off[g];
        ncand = (dv.grp_kind[g] != MOC_VIDEO) ? 0 : causal ? dv.cand_ncausal[g] : dv.cand_off[g + 1] - cbeg;
    }
    __device__ __forceinline__ void start(const DevLayout& dv, int64_t rtiles, int causal, int64_t t) {
        bh = int(t / rtiles);
        rt = int(t % rtiles);
        g = upper_index(dv.rtile_off, dv.G + 1, rt);
        load_group(dv, causal);
    }
    // the next tile; groups without tiles are skipped as the binary search does
    __device__ __forceinline__ void advance(const DevLayout& dv, int64_t rtiles, int causal) {
        if (++rt == rtiles) {
            rt = 0;
            ++bh;
            g = 0;
        } else if (rt < rt1) {
            return;
        }
        while (g < dv.G - 1 && dv.rtile_off[g + 1] <= rt) ++g;
        load_group(dv, causal);
    }
    __device__ __forceinline__ Tile tile() const {
        Tile x;
        x.bh = bh;
        x.g = g;
        x.q0 = gq0 + (rt - rt0) * kQTile;
        x.nq = min(kQTile, gq1 - x.q0);
        x.cbeg = cbeg;
        x.ncand = ncand;
        x.nb = (ncand + SLICE - 1) / SLICE;  // MMA slices
        return x;
    }
};

// Fill the hi / lo operand block (K-major, 128-byte swizzle) of candidates
// [cbeg + b * kBlk, + nbc) of head bh; rows up to npad are zero. Run by one warp.
template <int D, int KBSLAB, int KBLK>
__device__ __forceinline__ void build_block(const DevLayout& dv, const float* __restrict__ Kbar, int bh, int cbeg,
                                            int b, int nbc, int npad, uint32_t sHi, uint32_t sLo, int lane) {
    const float* kb = Kbar + size_t(bh) * dv.C * D;
    constexpr int CH = D / 8;  // 16-byte output chunks (8 dims) per row
    constexpr int U = 4;       // chunks per lane in flight: the id and Kbar loads of U chunks before their stores
    const int n = npad * CH;
    for (int i0 = lane; i0 < n; i0 += 32 * U) {
        int cid[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + 32 * u, r = i / CH;
            cid[u] = (i < n && r < nbc) ? dv.cand[cbeg + b * KBLK + r] : -1;
        }
        float4 va[U], vb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            va[u] = vb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (cid[u] >= 0) {
                const int ch = (i0 + 32 * u) % CH;
                va[u] = *reinterpret_cast<const float4*>(kb + size_t(cid[u]) * D + ch * 8);
                vb[u] = *reinterpret_cast<const float4*>(kb + size_t(cid[u]) * D + ch * 8 + 4);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + 32 * u;
            if (i >= n) break;
            const int r = i / CH, ch = i % CH;
            const float v[8] = {va[u].x, va[u].y, va[u].z, va[u].w, vb[u].x, vb[u].y, vb[u].z, vb[u].w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                const float2 hf = __bfloat1622float2(h);
                const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
                hi[e] = *reinterpret_cast<const uint32_t*>(&h);
                lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
            }
            const uint32_t off = (ch >> 3) * KBSLAB + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(sHi + off), "r"(hi[0]), "r"(hi[1]),
                         "r"(hi[2]), "r"(hi[3]) : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(sLo + off), "r"(lo[0]), "r"(lo[1]),
                         "r"(lo[2]), "r"(lo[3]) : "memory");
        }
    }
}

template <int D, int KMAX, int KBLK, int QS, bool PK>
__global__ void __launch_bounds__(RWarps<KMAX>::kThreads, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmQ, DevLayout dv, int64_t total_tiles,
                    int64_t rtiles, const float* __restrict__ Kbar, int k, int causal,
                    const uint64_t* __restrict__ seg_mask, int32_t* __restrict__ sel) {
    using C = RCfg<D, KBLK, QS>;
    constexpr int kBlk = C::kBlk;
    using WP = RWarps<KMAX>;
    constexpr int NWG = WP::kNwg, SLICE = WP::kSlice;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::oQ, sHi = base + C::oHi, sLo = base + C::oLo;
    const uint32_t sBar = base + C::oBar;
    RShared& sh = *reinterpret_cast<RShared*>(gbase + C::oBar + 256);
    volatile int* abort = &sh.abort;
    int32_t* err = dv.err;
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;


    if (tid == 0) {
        for (int x = 0; x < C::kQStages; ++x) {
            mbar_init(bar(R_Q_FULL + x), 1);
            mbar_init(bar(R_Q_EMPTY + x), 1);
        }
        for (int x = 0; x < NWG; ++x) {
            mbar_init(bar(R_S_FULL + x), 1);
            mbar_init(bar(R_S_FREE + x), 128);
        }
        mbar_init(bar(R_KB_FREE), 1);
        mbar_init(bar(R_MMA_DONE), 1);
        sh.abort = 0;
        // this CTA's contiguous range of tiles: equal shares of the estimated work
        const int64_t total_cost = (total_tiles / rtiles) * int64_t(dv.rcost[causal ? 1 : 0][rtiles]);
        sh.t_beg = tile_at_cost(dv, rtiles, causal, total_tiles, total_cost * blockIdx.x / gridDim.x);
        sh.t_end = tile_at_cost(dv, rtiles, causal, total_tiles, total_cost * (blockIdx.x + 1) / gridDim.x);
        fence_mbar_init();
    }
    if (warp == WP::kIssuer) {
        tmem_alloc(smem_u32(&sh.tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int64_t t_beg = sh.t_beg, t_end = sh.t_end;

    if (warp == WP::kProducer) {
        // ------------------------------------------------------------ Q producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            uint32_t qi = 0;
            TileWalk<SLICE> walk;
            if (t_beg < t_end) walk.start(dv, rtiles, causal, t_beg);
            for (int64_t t = t_beg; t < t_end; ++t, walk.advance(dv, rtiles, causal)) {
                const Tile x = walk.tile();
                if (x.ncand == 0) continue;
                const int st = qi % C::kQStages;
                if (!wait_bar(bar(R_Q_EMPTY + st), ((qi / C::kQStages) & 1) ^ 1, abort, err, 21)) break;
                mbar_expect_tx(bar(R_Q_FULL + st), C::kQBytes);
#pragma unroll
                for (int s = 0; s < C::kSlabs; ++s)
                    tma_load_2d(sQ + st * C::kQBytes + s * 128 * 128, &tmQ, bar(R_Q_FULL + st), 64 * s,
                                x.bh * dv.L + x.q0);
                ++qi;
            }
            // outstanding loads land before the CTA exits
            for (uint32_t g = (qi >= C::kQStages ? qi - C::kQStages : 0); g < qi; ++g)
                drain_bar(bar(R_Q_FULL + g % C::kQStages), (g / C::kQStages) & 1, err, 29);
        }
        __syncwarp();
    } else if (warp == WP::kIssuer) {
        // ------------------------------------------------------------ operands + MMA issue
        // The whole warp walks the units; it rebuilds the hi / lo block when the
        // (head, group, block) changes - after the MMAs that read the old block
        // have completed - and lane 0 issues each slice's MMAs into the score
        // buffer of the warpgroup that owns the tile (tiles go round robin).
        uint32_t qi = 0, nkb = 0, uw[NWG];
#pragma unroll
        for (int i = 0; i < NWG; ++i) uw[i] = 0;
        int last_bh = -1, last_g = -1, last_b = -1, ti = 0;
        bool stop = false;
        TileWalk<SLICE> walk;
        if (t_beg < t_end) walk.start(dv, rtiles, causal, t_beg);
        for (int64_t t = t_beg; t < t_end && !stop; ++t, ++ti, walk.advance(dv, rtiles, causal)) {
            const Tile x = walk.tile();
            if (x.ncand == 0) continue;
            const int w = ti % NWG;
            const int st = qi % C::kQStages;
            if (!wait_bar_warp(bar(R_Q_FULL + st), (qi / C::kQStages) & 1, abort, err, 22)) break;
            for (int b = 0; b < x.nb; ++b) {
                const int nbc = min(SLICE, x.ncand - b * SLICE);
                const int npad = (nbc + 15) & ~15;
                const int kb = b * SLICE / kBlk;           // operand block holding this slice
                const int roff = (b * SLICE) % kBlk;       // the slice's first row in it
                if (x.bh != last_bh || x.g != last_g || kb != last_b) {
                    if (last_bh >= 0) {  // the previous block's MMAs are complete
                        if (lane == 0) umma_commit(bar(R_KB_FREE));
                        if (!wait_bar_warp(bar(R_KB_FREE), nkb & 1, abort, err, 23)) { stop = true; break; }
                        ++nkb;
                    }
                    const int nbk = min(kBlk, x.ncand - kb * kBlk);
                    build_block<D, C::kKbSlab, kBlk>(dv, Kbar, x.bh, x.cbeg, kb, nbk, (nbk + 15) & ~15, sHi,
                                                     sLo, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    last_bh = x.bh; last_g = x.g; last_b = kb;
                }
                // one score buffer per warpgroup: its n-th use waits for the (n-1)-th release
                if (!wait_bar_warp(bar(R_S_FREE + w), (uw[w] & 1) ^ 1, abort, err, 24)) { stop = true; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t idesc = idesc_bf16_f32(128, npad, 0);
                    const uint32_t d_s = tmem + w * SLICE;
                    // descriptors of the first K step; later steps add their byte
                    // offset / 16 to the start-address field (no carry: < 2^14)
                    const uint64_t dq = sdesc_sw128(sQ + st * C::kQBytes, 16, 1024);
                    const uint64_t dhi = sdesc_sw128(sHi + roff * 128, 16, 1024);
                    const uint64_t dlo = sdesc_sw128(sLo + roff * 128, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < 2 * (D / 16); ++kk) {  // hi then lo
                        const int kd = kk % (D / 16);
                        const uint32_t qoff = (kd >> 2) * 128 * 128 + (kd & 3) * 32;
                        const uint32_t boff = (kd >> 2) * C::kKbSlab + (kd & 3) * 32;
                        umma_ss(d_s, dq + (qoff >> 4), (kk < D / 16 ? dhi : dlo) + (boff >> 4), idesc, kk > 0);
                    }
                    umma_commit(bar(R_S_FULL + w));
                }
                __syncwarp();
                ++uw[w];
            }
            if (stop) break;
            if (lane == 0) umma_commit(bar(R_Q_EMPTY + st));
            __syncwarp();
            ++qi;
        }
        if (lane == 0) {
            umma_commit(bar(R_MMA_DONE));
            drain_bar(bar(R_MMA_DONE), 0, err, 30);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ selection warpgroups
        const int w = warp >> 2;        // this warpgroup takes tiles ti with ti % NWG == w
        const int row = tid & 127;      // TMEM lane
        const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16) + w * SLICE;
        uint32_t u = 0;
        int ti = 0;
        TileWalk<SLICE> walk;
        if (t_beg < t_end) walk.start(dv, rtiles, causal, t_beg);
        for (int64_t t = t_beg; t < t_end; ++t, ++ti, walk.advance(dv, rtiles, causal)) {
            if (ti % NWG != w) continue;
            const Tile x = walk.tile();
            int32_t* out = sel + (size_t(x.bh) * dv.L + x.q0) * k;
            if (x.ncand == 0) {
                if (row < x.nq)
                    for (int j = 0; j < k; ++j) out[size_t(row) * k + j] = -1;
                continue;
            }
            const uint64_t smask = seg_mask ? seg_mask[size_t(x.bh) * dv.G + x.g] : ~0ull;
            // with 128-row operand blocks every candidate list has <= 128 entries: the
            // warp loads the group's chunk ids now (lane l holds entries l, l+32, ...),
            // so the loads overlap the score wait and the ids are mapped with shuffles
            int cid[4] = {-1, -1, -1, -1};
            if (kBlk == 128) {
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (r * 32 + lane < x.ncand) cid[r] = __ldg(dv.cand + x.cbeg + r * 32 + lane);
            }
            float ts[KMAX];
            int tj[KMAX];
            uint32_t tk[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                ts[j] = -INFINITY;
                tj[j] = kIdNone;
                tk[j] = 0u;
            }
            bool stop = false;
            for (int b = 0; b < x.nb; ++b) {
                const int nbc = min(SLICE, x.ncand - b * SLICE);
                if (!wait_bar_warp(bar(R_S_FULL + w), u & 1, abort, err, 25)) { stop = true; break; }
                tc_fence_after();
                // this row's nbc scores, 32 columns at a time; the list carries the
                // candidate's position in the group's list (ascending like the ids),
                // mapped to chunk ids once the tile is done
                for (int c0 = 0; c0 < nbc; c0 += 32) {
                    uint32_t sc[32];
                    tmem_ld32(lane_addr + c0, sc);
                    tmem_wait_ld_regs(sc);
                    const int pos0 = b * SLICE + c0;
                    // columns of this chunk that take part (warp-uniform): those inside
                    // the slice and, with an outer-loop mask, in a selected segment
                    uint32_t allow = (nbc - c0 >= 32) ? 0xffffffffu : ((1u << (nbc - c0)) - 1u);
                    if (seg_mask) {
                        const bool ok = ((allow >> lane) & 1u) &&
                                        ((smask >> dv.cand_seg[x.cbeg + pos0 + lane]) & 1ull);
                        allow = __ballot_sync(0xffffffffu, ok);
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        if (!((allow >> e) & 1u)) continue;
                        if (PK) topk_push_key<KMAX>(tk, pack_key(__uint_as_float(sc[e]), pos0 + e));
                        else topk_push<KMAX>(ts, tj, __uint_as_float(sc[e]), pos0 + e);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(R_S_FREE + w));
                ++u;
            }
            if (stop) break;
            if (PK) {
#pragma unroll
                for (int j = 0; j < KMAX; ++j) tj[j] = tk[j] == 0u ? kIdNone : int(0x1FFu - (tk[j] & 0x1FFu));
            }
            if (kBlk == 128) {
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    const int pos = tj[j] == kIdNone ? 0 : tj[j];
                    const int src = pos & 31, r = pos >> 5;
                    const int i0 = __shfl_sync(0xffffffffu, cid[0], src), i1 = __shfl_sync(0xffffffffu, cid[1], src);
                    const int i2 = __shfl_sync(0xffffffffu, cid[2], src), i3 = __shfl_sync(0xffffffffu, cid[3], src);
                    const int id = r == 0 ? i0 : r == 1 ? i1 : r == 2 ? i2 : i3;
                    if (row < x.nq && j < k) out[size_t(row) * k + j] = (tj[j] == kIdNone) ? -1 : id;
                }
            } else if (row < x.nq) {
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < k) out[size_t(row) * k + j] = (tj[j] == kIdNone) ? -1 : __ldg(dv.cand + x.cbeg + tj[j]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WP::kIssuer) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, int KMAX, int KBLK, int QS, bool PK>
cudaError_t launch_cfg(const DevLayout& dv, int BH, int64_t rtiles, const void* Q, const float* Kbar, int k,
                       int causal, const uint64_t* seg_mask, int32_t* sel, cudaStream_t s) {
    CUtensorMap tmQ;
    if (!make_tmap(&tmQ, Q, D, int64_t(BH) * dv.L)) return cudaErrorInvalidValue;
    const int smem = RCfg<D, KBLK, QS>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(route_tc_kernel<D, KMAX, KBLK, QS, PK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t total = int64_t(BH) * rtiles;
    const int grid = int(total < sms ? total : sms);
    route_tc_kernel<D, KMAX, KBLK, QS, PK><<<grid, RWarps<KMAX>::kThreads, smem, s>>>(tmQ, dv, total, rtiles, Kbar,
                                                                                      k, causal, seg_mask, sel);
    return cudaGetLastError();
}

// Candidate lists of at most 128 entries fit one 128-row operand block, which
// frees shared memory for a 5-stage Q ring; lists of up to 320 entries take one
// 320-row block and a 2-stage ring; longer lists take 256-row blocks (rebuilt as
// a tile's slices cross them) and a 2-stage ring. (With 2 selection warpgroups a
// slice is 256 candidates, which needs a block of at least 256 rows.)
template <int D, int KMAX>
cudaError_t launch_dk(const DevLayout& dv, int BH, int64_t rtiles, const void* Q, const float* Kbar, int k,
                      int causal, int max_cand, const uint64_t* seg_mask, int32_t* sel, cudaStream_t s) {
    if constexpr (RWarps<KMAX>::kSlice <= 128) {
        if (max_cand <= 128)
            return launch_cfg<D, KMAX, 128, 5, true>(dv, BH, rtiles, Q, Kbar, k, causal, seg_mask, sel, s);
    }
    // lists of up to 320 entries fit one operand block beside a 2-stage ring, so a
    // group's block is built once instead of once per tile and block; the selection
    // uses packed score / position keys (positions below 512): it is the kernel's main
    // cost with lists this long (ragged k = 2: 1.44 -> 0.80 ms)
    if constexpr (KMAX >= 8) {
        if (max_cand <= 320)
            return launch_cfg<D, KMAX, 320, 2, true>(dv, BH, rtiles, Q, Kbar, k, causal, seg_mask, sel, s);
        if (max_cand <= 511)
            return launch_cfg<D, KMAX, 256, 2, true>(dv, BH, rtiles, Q, Kbar, k, causal, seg_mask, sel, s);
    } else {
        if (max_cand <= 320)
            return launch_cfg<D, KMAX, 320, 2, true>(dv, BH, rtiles, Q, Kbar, k, causal, seg_mask, sel, s);
    }
    return launch_cfg<D, KMAX, 256, 2, false>(dv, BH, rtiles, Q, Kbar, k, causal, seg_mask, sel, s);
}

template <int D>
cudaError_t launch_d(const DevLayout& dv, int BH, int64_t rtiles, const void* Q, const float* Kbar, int k,
                     int causal, int max_cand, const uint64_t* seg_mask, int32_t* sel, cudaStream_t s) {
    // exact list length for small k (the insertion network costs one level per entry)
    switch (k) {
        case 1: return launch_dk<D, 1>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
        case 2: return launch_dk<D, 2>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
        case 3: return launch_dk<D, 3>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
        case 4: return launch_dk<D, 4>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
        default: break;
    }
    if (k <= 8) return launch_dk<D, 8>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
    if (k <= 16) return launch_dk<D, 16>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
    return launch_dk<D, 32>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
}

}  // namespace

cudaError_t launch_route(const DevLayout& dv, int BH, int64_t rtiles, int d, const void* Q,
                         const float* Kbar, int k, int causal, int max_cand, const uint64_t* seg_mask,
                         int32_t* sel, cudaStream_t s) {
    if (rtiles <= 0 || BH > 65535) return cudaErrorInvalidValue;
    if (d == 128) return launch_d<128>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
    return launch_d<64>(dv, BH, rtiles, Q, Kbar, k, causal, max_cand, seg_mask, sel, s);
}

}  // namespace moc

// (4) Chunk-major attention over work items on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA).
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: exact
// softmax attention of q over the keys/values of Omega(q), scaled by 1/sqrt(d).
// Omega(q) is split into disjoint parts attended separately and merged by
// their log-sum-exp in kernel (5):
//   anchor items - <= 256 consecutive queries of one query group against the
//                  group's anchor key ranges (partial slot 0);
//   routed items - <= 256 gathered queries of one chunk's query list against
//                  that chunk's keys (slot 1 + position in sel).
// The jxzklqfsx.com MoC write-up ("計算效率", limitations) packs these groups
// into one variable-length FlashAttention call; here a persistent kernel walks
// the items itself, longest first (anchor items, most keys first), then routed
// items.
//
// One CTA per SM, 384 threads, warp-specialised. An item's rows form two
// 128-row tiles A and B that share one K/V stream:
//   warp 8 (one lane): scheduler + TMA producer. Takes items from an atomic
//          counter, publishes them in a 2-slot ring, streams 128-key K and V
//          tiles (64-column, 128-byte-swizzled slabs) into 2-stage K and V rings
//          with cp.async.bulk.tensor, completion counted on mbarriers. K(j) is
//          released as soon as S(j) is computed, so K(j+2) loads while PV(j) and
//          the next S still run.
//          (warps 10-11 only complete the third warpgroup.)
//   warp 9: allocates all 512 TMEM columns (S_A, S_B, O_A, O_B); one lane
//          issues tcgen05.mma in the order
//            S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) ...
//          with S = Q K^T (M=128, N=128, fp32 in TMEM) and O += P V where P is
//          read from TMEM (bf16, written over its own S columns) and V from
//          shared memory (MN-major). While the tensor core works on one tile's
//          PV and next S, the other tile's softmax runs (ping-pong).
//   warps 0-3 / 4-7: softmax of tile A / tile B, one thread per query row
//          (= TMEM lane). Gather the tile's Q rows into the swizzled shared
//          layout; per key tile: load the S row from TMEM, mask keys past the
//          range end, online softmax in exp2 units with a lazily updated
//          running max (O is only rescaled in TMEM when the max grows by more
//          than 2^8, exact because the final normalisation uses the same max),
//          store P as bf16 back into TMEM; finally normalise O and write the
//          partial row and its log-sum-exp.
// Every mbarrier wait is bounded (2 s): on timeout the kernel records
// ERR_TIMEOUT and a site code in the workspace header, every role leaves its
// loop, in-flight copies and MMAs are drained (bounded) and TMEM is freed.
#include "items.cuh"
#include "pipeline.cuh"
#include "tmap.cuh"

namespace moc {
namespace {

using namespace sm100;
using items::Item;
using items::Cursor;
using items::decode;
using items::count_tiles;

using items::kKT;                               // keys per tile
constexpr int kThreads = 384;                   // softmax A, softmax B, producer/MMA warpgroups
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512);
// the producer/MMA warpgroup drops to 72 and the softmax warpgroups rise to
// 216: 2 x 128 x 216 + 128 x 72 = 64512, and per SM sub-partition
// (one warp of each warpgroup) 32 x (216 + 216 + 72) = 16128 <= 16384.
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = 72;
constexpr uint32_t kTmemCols = 512;

// F8: Q, K, V in E4M3 (one byte an element; d = 128 only) and P written to TMEM
// as E4M3, every MMA of kind::f8f6f4 (K = 32 elements an instruction).
template <int D, bool F8>
struct Cfg {
    static_assert(!F8 || D == 128, "the E4M3 path is built for d = 128");
    static constexpr int kEB = F8 ? 1 : 2;                  // bytes per element
    static constexpr int kKStep = F8 ? 32 : 16;             // K elements per MMA
    static constexpr int kSlabs = D * kEB / 128;            // 128-byte slabs per row
    static constexpr int kSlabBytes = 128 * 128;            // 128 rows x 128 B
    static constexpr int kTileBytes = kSlabs * kSlabBytes;  // a 128-row Q, K or V tile
    // K / V ring depths (a third stage of either, the one more tile that fits at
    // d = 128, measured no faster: the copies are not latency-bound)
    static constexpr int kKSt = 2;
    static constexpr int kVSt = 2;
    static constexpr int oQ = 0;                            // Q_A, Q_B
    static constexpr int oK = oQ + 2 * kTileBytes;          // kKSt stages
    static constexpr int oV = oK + kKSt * kTileBytes;       // kVSt stages
    static constexpr int oBar = oV + kVSt * kTileBytes;
    // + 1024 B alignment slack; at least 120 KB so that one CTA owns an SM (and its TMEM)
    static constexpr int kSmem = (oBar + 512 + 1024) > 120 * 1024 ? (oBar + 512 + 1024) : 120 * 1024;
    static_assert(kSmem <= 232448, "shared memory per CTA");
    static constexpr uint32_t kIdescQK = F8 ? idesc_e4m3_f32(128, kKT, 0) : idesc_bf16_f32(128, kKT, 0);
    static constexpr uint32_t kIdescPV = F8 ? idesc_e4m3_f32(128, D, 1) : idesc_bf16_f32(128, D, 1);
    // E4M3 P carries a factor 2^6 (and O is rescaled once the row max grows by more
    // than 2^2), so P * 64 <= 256 stays below E4M3's 448 and small weights stay
    // normal numbers longer
    static constexpr float kPScale = F8 ? 64.f : 1.f;
    // E4M3: the upper two keys of every kFmaExpEvery-th column of P take their
    // exponentials on the FMA pipe (ex2_fma2): the E4M3 MMAs take half the tensor
    // cycles, so the softmax, and with it the MUFU, sets the pace. One in four of
    // the exponentials measured 8 % faster than none (one in eight the same, one in
    // two slower)
    static constexpr int kFmaExpEvery = 2;
    static constexpr float kLazy = F8 ? 2.f : 8.f;
};

// TMEM columns: S_A / S_B (P_A / P_B overwrite their first 64 columns), O_A / O_B
__device__ __forceinline__ uint32_t col_s(int q) { return q ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int q) { return q ? 384u : 256u; }

// mbarrier slots (8 bytes each) from Cfg::oBar; [x] = tile A / B or ring slot
enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY = 2, B_Q_FULL = 4, B_S_FULL = 6, B_P_FULL = 8, B_PV_DONE = 10,
    B_MMA_DONE = 12, B_K_FULL = 13, B_K_EMPTY = 16, B_V_FULL = 19, B_V_EMPTY = 22, B_COUNT = 25
};

struct Shared {  // at oBar + 256
    int item[2];
    uint32_t tmem_base;
    int abort;
};

// FUSED: routed items run first and write their partials; every anchor item
// then merges its own part with the routed partials of its rows in the epilogue
// and writes the bf16 output row and its log-sum-exp (the merge of (5) done in
// place, so slot 0 is never written and read back). Not FUSED: every item writes
// its partial, for the stage call of (4) followed by (5).
template <int D, bool FUSED, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     DevLayout dv, int BH, int k, float scale_log2, int64_t n_anchor,
                     const unsigned char* __restrict__ Q, int32_t* __restrict__ hdr,
                     const int32_t* __restrict__ qoff, const int32_t* __restrict__ tile_off,
                     const int32_t* __restrict__ qlist, float* __restrict__ lse_p,
                     float* __restrict__ o_p, int reverse, const int32_t* __restrict__ sel,
                     __nv_bfloat16* __restrict__ O_out, float* __restrict__ lse_out,
                     const float* __restrict__ q_scale, const float* __restrict__ k_scale,
                     const float* __restrict__ v_scale) {
    using C = Cfg<D, F8>;
    static_assert(!(FUSED && F8), "the fused merge is built for bf16 inputs");
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte aligned base: the 128-byte swizzle atoms of TMA and UMMA repeat every 1024 B
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + C::oQ, sK = base + C::oK, sV = base + C::oV;
    const uint32_t sBar = base + C::oBar;
    Shared& sh = *reinterpret_cast<Shared*>(gbase + C::oBar + 256);
    volatile int* abort = &sh.abort;
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = k + 1;
    const size_t L = size_t(dv.L);

    if (tid == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(B_ITEM_FULL + x), 1);
            mbar_init(bar(B_ITEM_EMPTY + x), 1 + 256);
            mbar_init(bar(B_Q_FULL + x), 128);
            mbar_init(bar(B_S_FULL + x), 1);
            mbar_init(bar(B_P_FULL + x), 128);
            mbar_init(bar(B_PV_DONE + x), 1);
        }
        for (int x = 0; x < C::kKSt; ++x) {
            mbar_init(bar(B_K_FULL + x), 1);
            mbar_init(bar(B_K_EMPTY + x), 1);
        }
        for (int x = 0; x < C::kVSt; ++x) {
            mbar_init(bar(B_V_FULL + x), 1);
            mbar_init(bar(B_V_EMPTY + x), 1);
        }
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

    if (warp >= 8) {
      regs_dec<kRegsOther>();
      if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const int64_t total = n_anchor + tile_off[int64_t(BH) * dv.C];
            uint32_t gt = 0;
            for (int it = 0;; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_EMPTY + slot), ((it >> 1) & 1) ^ 1, abort, hdr, 1)) break;
                const int64_t ticket = atomicAdd(&hdr[HDR_WORK], 1);
                const bool ok = ticket < total;
                int64_t item = reverse ? total - 1 - ticket : ticket;
                if (FUSED) {  // routed items first (each class in natural or reversed order)
                    const int64_t n_routed = total - n_anchor;
                    if (ticket < n_routed) item = n_anchor + (reverse ? n_routed - 1 - ticket : ticket);
                    else item = reverse ? total - 1 - ticket : ticket - n_routed;
                }
                sh.item[slot] = ok ? int(item) : -1;
                mbar_arrive(bar(B_ITEM_FULL + slot));
                if (!ok) break;
                Item itm;
                decode(dv, BH, n_anchor, item, tile_off, qoff, qlist, itm);
                Cursor cur;
                cur.init(dv, itm);
                const int row0 = itm.bh * dv.L;
                bool stop = false;
                while (cur.more()) {
                    int key0, nvalid;
                    cur.next(key0, nvalid);
                    // K and V have rings of their own: K(j) is released once S(j) is computed,
                    // long before V(j) is released by PV(j), so K(j+2) streams in early
                    const int st = gt % C::kKSt, sv = gt % C::kVSt;
                    if (!wait_bar(bar(B_K_EMPTY + st), ((gt / C::kKSt) & 1) ^ 1, abort, hdr, 2)) { stop = true; break; }
                    mbar_expect_tx(bar(B_K_FULL + st), C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_2d(sK + st * C::kTileBytes + s * C::kSlabBytes, &tmK, bar(B_K_FULL + st), 64 * s, row0 + key0);
                    if (!wait_bar(bar(B_V_EMPTY + sv), ((gt / C::kVSt) & 1) ^ 1, abort, hdr, 8)) { stop = true; break; }
                    mbar_expect_tx(bar(B_V_FULL + sv), C::kTileBytes);
#pragma unroll
                    for (int s = 0; s < C::kSlabs; ++s)
                        tma_load_2d(sV + sv * C::kTileBytes + s * C::kSlabBytes, &tmV, bar(B_V_FULL + sv), 64 * s, row0 + key0);
                    ++gt;
                }
                if (stop) break;
            }
            // drain: the last use of each stage has landed before the CTA exits (a load
            // cut short by an abort may have issued K without V; its V wait then times out
            // harmlessly because nothing was issued on it)
            for (int b = 0; b < 2; ++b) {
                const uint32_t n = b ? C::kVSt : C::kKSt;
                for (uint32_t g = (gt >= n ? gt - n : 0); g < gt; ++g) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(bar((b ? B_V_FULL : B_K_FULL) + g % n), (g / n) & 1)) {
                        if (globaltimer() - t0 > kTimeoutNs) { set_error(hdr, ERR_TIMEOUT, 9); break; }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t gt = 0;           // key tiles of all items (K/V ring)
            uint32_t gtt[2] = {0, 0};  // key tiles per query tile (S_FULL / P_FULL / PV_DONE phases)
            uint32_t itq[2] = {0, 0};  // items per query tile (Q_FULL phases)
            bool stop = false;
            for (int it = 0; !stop; ++it) {
                const int slot = it & 1;
                if (!wait_bar(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 3)) break;
                const int item = sh.item[slot];
                mbar_arrive(bar(B_ITEM_EMPTY + slot));
                if (item < 0) break;
                Item itm;
                decode(dv, BH, n_anchor, item, tile_off, qoff, qlist, itm);
                const int T = count_tiles(dv, itm);
                const int nt = itm.nq > kQTile ? 2 : 1;  // query tiles in this item
                for (int q = 0; q < nt && !stop; ++q)
                    if (!wait_bar(bar(B_Q_FULL + q), itq[q] & 1, abort, hdr, 4)) stop = true;
                if (stop) break;
                tc_fence_after();
                for (int j = 0; j <= T && !stop; ++j) {
                    const uint32_t st = gt % C::kKSt;
                    bool k_ready = false, v_ready = false;
                    for (int q = 0; q < nt; ++q) {
                        if (j > 0) {  // O_q += P_q(j-1) V(j-1)
                            const uint32_t g = gtt[q] - 1, pst = (gt - 1) % C::kVSt;
                            if (!v_ready) {
                                if (!wait_bar(bar(B_V_FULL + pst), ((gt - 1) / C::kVSt) & 1, abort, hdr, 15)) { stop = true; break; }
                                v_ready = true;
                            }
                            if (!wait_bar(bar(B_P_FULL + q), g & 1, abort, hdr, 7)) { stop = true; break; }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < kKT / C::kKStep; ++kk) {
                                // P's K step kk: 8 TMEM columns (16 bf16 or 32 E4M3 keys); V's: kKStep rows
                                const uint64_t vd = sdesc_sw128(sV + pst * C::kTileBytes + kk * C::kKStep * 128,
                                                                C::kSlabBytes, 1024);
                                if constexpr (F8)
                                    umma_ts_f8(tmem + col_o(q), tmem + col_s(q) + kk * 8, vd, C::kIdescPV, (j > 1 || kk > 0));
                                else
                                    umma_ts(tmem + col_o(q), tmem + col_s(q) + kk * 8, vd, C::kIdescPV, (j > 1 || kk > 0));
                            }
                            umma_commit(bar(B_PV_DONE + q));
                        }
                        if (j < T) {  // S_q(j) = Q_q K(j)^T, after PV_q(j-1) has read P_q(j-1)
                            if (!k_ready) {
                                if (!wait_bar(bar(B_K_FULL + st), (gt / C::kKSt) & 1, abort, hdr, 5)) { stop = true; break; }
                                k_ready = true;
                                tc_fence_after();
                            }
                            const uint32_t qb = sQ + q * C::kTileBytes, kb = sK + st * C::kTileBytes;
#pragma unroll
                            for (int kk = 0; kk < D / C::kKStep; ++kk) {
                                // 32 bytes of every row per K step in both element types
                                const uint32_t off = (kk >> 2) * C::kSlabBytes + (kk & 3) * 32;
                                if constexpr (F8)
                                    umma_ss_f8(tmem + col_s(q), sdesc_sw128(qb + off, 16, 1024),
                                               sdesc_sw128(kb + off, 16, 1024), C::kIdescQK, kk > 0);
                                else
                                    umma_ss(tmem + col_s(q), sdesc_sw128(qb + off, 16, 1024),
                                            sdesc_sw128(kb + off, 16, 1024), C::kIdescQK, kk > 0);
                            }
                            umma_commit(bar(B_S_FULL + q));
                            ++gtt[q];
                        }
                    }
                    if (stop) break;
                    if (j > 0) umma_commit(bar(B_V_EMPTY + (gt - 1) % C::kVSt));  // V(j-1) read by PV
                    if (j < T) umma_commit(bar(B_K_EMPTY + st));              // K(j) read by S
                    if (j < T) ++gt;
                }
                for (int q = 0; q < nt; ++q) ++itq[q];
            }
            // all issued MMAs complete before TMEM is released
            umma_commit(bar(B_MMA_DONE));
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(bar(B_MMA_DONE), 0)) {
                if (globaltimer() - t0 > kTimeoutNs) { set_error(hdr, ERR_TIMEOUT, 10); break; }
            }
        }
        __syncwarp();
    }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int q = warp >> 2;    // query tile A (0) or B (1)
        const int row = tid & 127;  // row within the tile = TMEM lane
        const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_addr + col_s(q), o_addr = lane_addr + col_o(q);
        const uint32_t sQq = sQ + q * C::kTileBytes;
        uint32_t gtt = 0;
        for (int it = 0;; ++it) {
            const int slot = it & 1;
            if (!wait_bar_warp(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 11)) break;
            const int item = sh.item[slot];
            mbar_arrive(bar(B_ITEM_EMPTY + slot));
            if (item < 0) break;
            Item itm;
            decode(dv, BH, n_anchor, item, tile_off, qoff, qlist, itm);
            if (q == 1 && itm.nq <= kQTile) continue;  // no tile B in this item
            const int r_item = q * kQTile + row;       // row within the item
            const unsigned char* Qb = Q + size_t(itm.bh) * L * D * C::kEB;
            // scores are q . k in the inputs' units; E4M3 inputs carry per-(b, h) scales
            const float sl2 = F8 ? scale_log2 * q_scale[itm.bh] * k_scale[itm.bh] : scale_log2;
            int my_tok = -1, my_slot = 0;
            if (r_item < itm.nq) {
                if (itm.slot_fixed >= 0) {
                    my_tok = itm.q0 + r_item;
                } else {
                    const int e = itm.entries[r_item];
                    my_tok = e >> 5;
                    my_slot = 1 + (e & 31);
                }
            }
            // gather the warp's 32 query rows into the swizzled tile (16-byte chunks):
            // every load is issued before the first store, so the warp waits for
            // one memory round trip instead of one per chunk
            constexpr int CH = D * C::kEB / 16;
            uint4 qv[CH];
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int tok = __shfl_sync(0xffffffffu, my_tok, (i * 32 + lane) / CH);
                qv[i] = make_uint4(0, 0, 0, 0);
                if (tok >= 0) qv[i] = ldg_nc16(Qb + size_t(tok) * D * C::kEB + ((i * 32 + lane) % CH) * 16);
            }
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int idx = i * 32 + lane;
                const int r = (warp & 3) * 32 + idx / CH, ch = idx % CH;
                const uint32_t dst = sQq + (ch >> 3) * C::kSlabBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(qv[i].x), "r"(qv[i].y),
                             "r"(qv[i].z), "r"(qv[i].w) : "memory");
            }
            fence_proxy_async_smem();
            mbar_arrive(bar(B_Q_FULL + q));

            Cursor cur;
            cur.init(dv, itm);
            float m_used = -INFINITY, l = 0.f;
            bool stop = false;
            for (int j = 0; cur.more(); ++j) {
                int key0, nvalid;
                cur.next(key0, nvalid);
                if (!wait_bar_warp(bar(B_S_FULL + q), gtt & 1, abort, hdr, 12)) { stop = true; break; }
                tc_fence_after();
                uint32_t s[kKT];
#pragma unroll
                for (int c = 0; c < kKT / 32; ++c)
                    tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
                tmem_wait_ld_regs(s);
                // keys past the range end (only in a range's last tile) -> -inf, so P = 0
                if (nvalid < kKT) {
#pragma unroll
                    for (int c = 0; c < kKT; ++c)
                        if (c >= nvalid) s[c] = __float_as_uint(-INFINITY);
                }
                // row max of the raw scores (the positive scale commutes with max), as
                // eight independent 3-input max chains
                float a[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) a[i] = fmaxf(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
#pragma unroll
                for (int c = 16; c < kKT; c += 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) a[i] = max3(a[i], __uint_as_float(s[c + 2 * i]), __uint_as_float(s[c + 2 * i + 1]));
                }
                const float mx = max3(max3(a[0], a[1], a[2]), max3(a[3], a[4], a[5]), fmaxf(a[6], a[7])) * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (j == 0) {
                    m_used = mx;
                } else if (mx > m_used + C::kLazy) {  // lazy rescale: only when the max grew by > 2^8 (E4M3: 2^2)
                    alpha = ex2(m_used - mx);
                    m_used = mx;
                    rescale = true;
                }
                if (__any_sync(0xffffffffu, rescale)) {  // warp-collective TMEM access; alpha = 1 elsewhere
                    // O_q must hold PV_q(j-1) before it is scaled
                    if (!wait_bar_warp(bar(B_PV_DONE + q), (gtt - 1) & 1, abort, hdr, 13)) { stop = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + c * 32, o);
                        tmem_wait_ld_regs(o);
#pragma unroll
                        for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
                        tmem_st32(o_addr + c * 32, o);
                    }
                }
                // P = exp2(s * scale - m) as bf16 pairs into the first 64 columns of S_q;
                // scale-and-subtract and the row sum run on packed fp32 pairs
                const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m_used, -m_used);
                uint64_t sum2a = 0, sum2b = 0;
                if constexpr (F8) {
                    // four keys a column: E4M3 of P * 2^6 in the first 32 columns of S_q
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = 4 * c;
                        float x0, x1, x2, x3;
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sc2, nm2), x0, x1);
                        f2_unpack(f2_fma(f2_pack(__uint_as_float(s[e + 2]), __uint_as_float(s[e + 3])), sc2, nm2), x2, x3);
                        const float p0 = ex2(x0), p1 = ex2(x1);
                        float p2, p3;
                        if (c % C::kFmaExpEvery == C::kFmaExpEvery - 1) {  // this share on the FMA pipe
                            f2_unpack(ex2_fma2(x2, x3), p2, p3);
                        } else {
                            p2 = ex2(x2);
                            p3 = ex2(x3);
                        }
                        sum2a = f2_add(sum2a, f2_pack(p0, p1));
                        sum2b = f2_add(sum2b, f2_pack(p2, p3));
                        pk[c] = pack_e4m3x2(p0 * C::kPScale, p1 * C::kPScale) |
                                (pack_e4m3x2(p2 * C::kPScale, p3 * C::kPScale) << 16);
                    }
                    tmem_st32(s_addr, pk);
                } else {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t pk[32];
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int e = h * 64 + 2 * c;
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sc2, nm2), x0, x1);
                            const float p0 = ex2(x0), p1 = ex2(x1);
                            if (c & 1) sum2b = f2_add(sum2b, f2_pack(p0, p1));
                            else sum2a = f2_add(sum2a, f2_pack(p0, p1));
                            pk[c] = pack_bf16(p0, p1);
                        }
                        tmem_st32(s_addr + h * 32, pk);
                    }
                }
                float r0, r1, r2, r3;
                f2_unpack(sum2a, r0, r1);
                f2_unpack(sum2b, r2, r3);
                const float rs = (r0 + r1) + (r2 + r3);
                l = l * alpha + rs;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL + q));
                ++gtt;
            }
            if (stop) break;
            // epilogue: final PV done -> O / l -> partial row, log-sum-exp. Each
            // 32-column chunk of the warp's 32 rows is staged in shared memory - in
            // the warp's own rows of its Q tile, free once every S of the item is
            // done and rewritten only by this warp's next gather - and written back
            // as whole 128-byte row pieces, four rows per store instruction.
            if (!wait_bar_warp(bar(B_PV_DONE + q), (gtt - 1) & 1, abort, hdr, 14)) break;
            tc_fence_after();
            if (FUSED && itm.slot_fixed == 0) {
                // merged epilogue of an anchor item: every routed row of this launch
                // is complete once the counter of written routed rows reaches the
                // number of query-list entries (routed items are handed out before
                // any anchor item, so none of them waits behind this one)
                if (lane == 0) {
                    const int32_t target = qoff[int64_t(BH) * dv.C];
                    const uint64_t t0 = globaltimer();
                    while (ld_acquire_gpu(&hdr[HDR_RDONE]) < target) {
                        if (globaltimer() - t0 > kTimeoutNs) { set_error(hdr, ERR_TIMEOUT, 16); break; }
                    }
                }
                __syncwarp();
                __threadfence();
                const size_t row = size_t(itm.bh) * L + (my_tok >= 0 ? my_tok : 0);
                const float lse0 = (m_used + log2f(l)) * 0.69314718055994531f;
                // slots in fixed order: the own part (slot 0), then sel order
                float M = lse0;
                if (my_tok >= 0) {
                    for (int x = 0; x < k; ++x) {
                        const int32_t sj = sel[row * k + x];
                        if (sj >= 0 && sj < dv.C) M = fmaxf(M, lse_p[row * S + 1 + x]);
                    }
                }
                float Z = expf(lse0 - M);
                if (my_tok >= 0) {
                    for (int x = 0; x < k; ++x) {
                        const int32_t sj = sel[row * k + x];
                        if (sj >= 0 && sj < dv.C) Z += expf(lse_p[row * S + 1 + x] - M);
                    }
                }
                const float a0 = expf(lse0 - M) / (Z * l);  // the own part is O / l
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + c * 32, o);
                    tmem_wait_ld_regs(o);
                    float acc[32];
#pragma unroll
                    for (int x = 0; x < 32; ++x) acc[x] = __uint_as_float(o[x]) * a0;
                    if (my_tok >= 0) {
                        for (int x = 0; x < k; ++x) {
                            const int32_t sj = sel[row * k + x];
                            if (sj < 0 || sj >= dv.C) continue;
                            const float wx = expf(lse_p[row * S + 1 + x] - M) / Z;
                            const float4* src = reinterpret_cast<const float4*>(o_p + (row * S + 1 + x) * D + c * 32);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float4 v = src[i];
                                acc[4 * i] += wx * v.x;
                                acc[4 * i + 1] += wx * v.y;
                                acc[4 * i + 2] += wx * v.z;
                                acc[4 * i + 3] += wx * v.w;
                            }
                        }
                        uint4* dst4 = reinterpret_cast<uint4*>(O_out + row * D + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst4[i] = make_uint4(pack_bf16(acc[8 * i], acc[8 * i + 1]), pack_bf16(acc[8 * i + 2], acc[8 * i + 3]),
                                                 pack_bf16(acc[8 * i + 4], acc[8 * i + 5]),
                                                 pack_bf16(acc[8 * i + 6], acc[8 * i + 7]));
                    }
                }
                tc_fence_before();
                if (my_tok >= 0 && lse_out) lse_out[row] = M + logf(Z);
                continue;
            }
            // E4M3: O accumulates P * 2^6 times the unscaled V
            const float inv = F8 ? v_scale[itm.bh] / (C::kPScale * l) : 1.f / l;
            float* dst = (my_tok >= 0) ? o_p + ((size_t(itm.bh) * L + my_tok) * S + my_slot) * D : nullptr;
            float* rdst[8];  // destination row of this lane in store step i: row 4i + lane / 8
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint64_t p = __shfl_sync(0xffffffffu, reinterpret_cast<uint64_t>(dst), 4 * i + (lane >> 3));
                rdst[i] = reinterpret_cast<float*>(p);
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(o_addr + c * 32, o);
                tmem_wait_ld_regs(o);
                // each slab of the tile holds this warp's rows 32 (warp & 3) .. + 31 at 128 B each
                const uint32_t stg = sQq + (c % C::kSlabs) * C::kSlabBytes + (warp & 3) * 32 * 128;
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const uint32_t a = stg + lane * 128 + ((x ^ (lane & 7)) << 4);
                    asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(a),
                                 "f"(__uint_as_float(o[4 * x]) * inv), "f"(__uint_as_float(o[4 * x + 1]) * inv),
                                 "f"(__uint_as_float(o[4 * x + 2]) * inv), "f"(__uint_as_float(o[4 * x + 3]) * inv)
                                 : "memory");
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 4 * i + (lane >> 3), ch = lane & 7;
                    float4 v;
                    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                 : "r"(stg + r * 128 + ((ch ^ (r & 7)) << 4))
                                 : "memory");
                    if (rdst[i]) *reinterpret_cast<float4*>(rdst[i] + c * 32 + ch * 4) = v;
                }
                __syncwarp();
            }
            tc_fence_before();
            if (dst) lse_p[(size_t(itm.bh) * L + my_tok) * S + my_slot] = (m_used + log2f(l)) * 0.69314718055994531f;
            if (FUSED) {
                // publish this warp's routed rows: every lane's stores, then one count
                __threadfence();
                __syncwarp();
                const unsigned vm = __ballot_sync(0xffffffffu, dst != nullptr);
                if (lane == 0 && vm) atomicAdd(&hdr[HDR_RDONE], __popc(vm));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, bool FUSED, bool F8>
cudaError_t launch_d(const DevLayout& dv, int BH, const void* Q, const void* K, const void* V, int k,
                     float scale, int64_t n_anchor, char* ws, const WsPlan& p, const int32_t* sel, void* O,
                     float* lse, const float* q_scale, const float* k_scale, const float* v_scale,
                     cudaStream_t s) {
    CUtensorMap tmK, tmV;
    const int64_t rows = int64_t(BH) * dv.L;
    if (F8) {
        if (!make_tmap_u8(&tmK, K, D, rows) || !make_tmap_u8(&tmV, V, D, rows)) return cudaErrorInvalidValue;
    } else {
        if (!make_tmap(&tmK, K, D, rows) || !make_tmap(&tmV, V, D, rows)) return cudaErrorInvalidValue;
    }
    const int smem = Cfg<D, F8>::kSmem;
    cudaError_t e =
        cudaFuncSetAttribute(attend_tc_kernel<D, FUSED, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const AttendSchedule sched = attend_schedule();
    if (sched.n_ctas > 0 && sched.n_ctas < sms) sms = sched.n_ctas;
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    e = cudaMemsetAsync(hdr + HDR_WORK, 0, 2 * sizeof(int32_t), s);  // work counter, routed rows done
    if (e != cudaSuccess) return e;
    attend_tc_kernel<D, FUSED, F8><<<sms, kThreads, smem, s>>>(
        tmK, tmV, dv, BH, k, scale * 1.4426950408889634f, n_anchor, static_cast<const unsigned char*>(Q), hdr,
        reinterpret_cast<const int32_t*>(ws + p.qoff), reinterpret_cast<const int32_t*>(ws + p.tile_off),
        reinterpret_cast<const int32_t*>(ws + p.qlist), reinterpret_cast<float*>(ws + p.lse_p),
        reinterpret_cast<float*>(ws + p.o_p), sched.reverse, sel, static_cast<__nv_bfloat16*>(O), lse, q_scale,
        k_scale, v_scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const DevLayout& dv, int BH, int d, const void* Q, const void* K,
                             const void* V, int k, float scale, int64_t n_anchor, char* ws,
                             const WsPlan& p, cudaStream_t s) {
    if (d == 128)
        return launch_d<128, false, false>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, nullptr, nullptr, nullptr,
                                           nullptr, nullptr, nullptr, s);
    return launch_d<64, false, false>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, nullptr, nullptr, nullptr, nullptr,
                                      nullptr, nullptr, s);
}

cudaError_t launch_attend_merged(const DevLayout& dv, int BH, int d, const void* Q, const void* K,
                                 const void* V, int k, float scale, int64_t n_anchor, char* ws,
                                 const WsPlan& p, const int32_t* sel, void* O, float* lse, cudaStream_t s) {
    if (d == 128)
        return launch_d<128, true, false>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, sel, O, lse, nullptr, nullptr,
                                          nullptr, s);
    return launch_d<64, true, false>(dv, BH, Q, K, V, k, scale, n_anchor, ws, p, sel, O, lse, nullptr, nullptr,
                                     nullptr, s);
}

cudaError_t launch_attend_e4m3(const DevLayout& dv, int BH, const void* Q8, const void* K8, const void* V8,
                               const float* q_scale, const float* k_scale, const float* v_scale, int k, float scale,
                               int64_t n_anchor, char* ws, const WsPlan& p, cudaStream_t s) {
    return launch_d<128, false, true>(dv, BH, Q8, K8, V8, k, scale, n_anchor, ws, p, nullptr, nullptr, nullptr,
                                      q_scale, k_scale, v_scale, s);
}

}  // namespace moc

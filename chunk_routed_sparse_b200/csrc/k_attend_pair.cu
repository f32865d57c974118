// (4) on CTA pairs: the chunk-major attention of k_attend_tc.cu with every MMA
// spanning two SMs (tcgen05 cta_group::2, M = 256), bf16 inputs, d = 128.
//
// "Mixture of Contexts for Long Video Generation | Summary" §3.1: exact softmax
// attention of q over the keys/values of Omega(q), scaled by 1/sqrt(d), split
// into the same disjoint parts as k_attend_tc.cu (anchor items: consecutive
// queries of one group against the group's anchor key ranges, partial slot 0;
// routed items: entries of one chunk's query list against that chunk's keys,
// slot 1 + position in sel), merged by their log-sum-exp in kernel (5).
//
// Why pairs: in the single-CTA kernel every S MMA (M=128, N=128, both operands in
// shared memory) reads 8 KB per 64-cycle K step and every 128-key tile lands
// 64 KB of K and V in the same shared memory; taking the TMA copies away alone
// made that kernel 15 % faster. A cluster of two CTAs runs one MMA stream:
// each CTA supplies its own 128 query rows as A and HALF of every B operand
// (64 keys of K for S, 64 of the 128 dimensions of V for P V), and loads only
// that half of every K and V tile. Per SM this halves the B reads and the TMA
// bytes for the same tensor work.
//
// Items are kPairRows = 512 query rows: two pair tiles of 256 (A: rows 0-255,
// B: rows 256-511) that share one K/V stream; CTA r of the pair owns rows
// 128 r .. 128 r + 127 of each pair tile (its TMEM lanes). Per CTA, 384 threads:
//   warp 8 (one lane): producer. In CTA 0 it takes items from an atomic counter
//          and publishes each to both CTAs (a 2-slot ring); in both CTAs it
//          streams this CTA's half of every K tile (64 keys x 128 dims) and V
//          tile (128 keys x 64 dims) into 4-stage rings, completion counted on
//          CTA 0's mbarriers (expected bytes set there for both halves).
//   warp 9: allocates TMEM for the pair (512 columns in each CTA: S_A, S_B, O_A,
//          O_B). In CTA 0 one lane issues every MMA of the pair in the order of
//          the single-CTA kernel (S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) |
//          ...) and commits each to the mbarriers of both CTAs.
//   warps 0-3 / 4-7: softmax of this CTA's rows of pair tile A / B, one thread a
//          row, exactly as in the single-CTA kernel; their arrivals that the MMA
//          warp waits on go to CTA 0 (one per warp).
// Waits on barriers fed by another CTA's plain stores (the item slots, the gathered
// Q rows) acquire at cluster scope; those fed by tcgen05 commits, TMA completion or
// the P hand-off acquire at CTA scope. Every wait is bounded (2 s; ERR_TIMEOUT with
// a site code in the header). The pair leaves together: each producer first waits
// until every stage it filled was released (its copies landed, the commits on its
// barriers arrived), CTA 0 waits for its last MMA, then a cluster barrier, then the
// TMEM is freed.
#include "items.cuh"
#include "pipeline.cuh"
#include "tmap.cuh"

namespace moc {
namespace {

using namespace sm100;
using items::Item;
using items::Cursor;
using items::decode_rows;
using items::count_tiles;
using items::kKT;

constexpr int D = 128;
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 216;  // 2 x 128 x 216 + 128 x 72 = 64512 = 384 x 168
constexpr int kRegsOther = 72;
constexpr uint32_t kTmemCols = 512;
constexpr int kQSlab = 128 * 128;         // 128 rows x 64 dims (128 B a row)
constexpr int kQBytes = 2 * kQSlab;       // this CTA's 128 rows of a pair tile
constexpr int kKSlab = 64 * 128;          // 64 keys x 64 dims
constexpr int kKHalf = 2 * kKSlab;        // this CTA's 64 keys of a K tile
constexpr int kVHalf = 128 * 128;         // 128 keys x this CTA's 64 dims of a V tile
constexpr int kKSt = 4, kVSt = 4;
constexpr int oQ = 0;
constexpr int oK = oQ + 2 * kQBytes;
constexpr int oV = oK + kKSt * kKHalf;
constexpr int oBar = oV + kVSt * kVHalf;
constexpr int kSmem = oBar + 512 + 1024;  // + barriers / shared words + alignment slack
static_assert(kSmem <= 232448, "shared memory per CTA");
constexpr uint32_t kIdescQK = idesc_bf16_f32(256, kKT, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(256, D, 1);

__device__ __forceinline__ uint32_t col_s(int q) { return q ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int q) { return q ? 384u : 256u; }

// mbarrier slots (8 bytes each) from oBar; the same offsets in both CTAs
enum {
    B_ITEM_FULL = 0, B_ITEM_EMPTY = 2, B_Q_FULL = 4, B_S_FULL = 6, B_P_FULL = 8, B_PV_DONE = 10,
    B_MMA_DONE = 12, B_K_FULL = 13, B_K_EMPTY = B_K_FULL + kKSt, B_V_FULL = B_K_EMPTY + kKSt,
    B_V_EMPTY = B_V_FULL + kVSt, B_COUNT = B_V_EMPTY + kVSt
};
static_assert(B_COUNT * 8 <= 256, "barrier slots");
// arrivals on CTA 0's ITEM_EMPTY per use of a slot: its MMA lane, the 8 softmax
// warps of each CTA, CTA 1's producer
constexpr int kItemConsumers = 1 + 8 + 8 + 1;

struct Shared {  // at oBar + 256
    int item[2];
    uint32_t tmem_base;
    int abort;
};

// Bounded waits on this CTA's mbarriers with cluster-scope acquire.
__device__ __forceinline__ bool wait_cl(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* hdr,
                                        int where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                set_error(hdr, ERR_TIMEOUT, where);
                *abort = 1;
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_cl_warp(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* hdr,
                                             int where) {
    const bool ok = wait_cl(bar, parity, abort, hdr, where);
    return __all_sync(0xffffffffu, ok);
}
// bounded by `deadline`, ignoring the abort flag: outstanding copies and commits land first
__device__ __forceinline__ void drain_until(uint32_t bar, uint32_t parity, uint64_t deadline, int32_t* hdr, int where) {
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() > deadline) {
            set_error(hdr, ERR_TIMEOUT, where);
            return;
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attend_pair_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       DevLayout dv, int BH, int k, float scale_log2, int64_t n_anchor,
                       const unsigned char* __restrict__ Q, int32_t* __restrict__ hdr,
                       const int32_t* __restrict__ qoff, const int32_t* __restrict__ tile2_off,
                       const int32_t* __restrict__ qlist, float* __restrict__ lse_p, float* __restrict__ o_p,
                       int reverse) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const uint32_t sQ = base + oQ, sK = base + oK, sV = base + oV;
    const uint32_t sBar = base + oBar;
    Shared& sh = *reinterpret_cast<Shared*>(gbase + oBar + 256);
    volatile int* abort = &sh.abort;
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };
    auto lead_bar = [&](int i) { return mapa(sBar + 8u * uint32_t(i), 0); };  // CTA 0's barrier

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const bool lead = rank == 0;
    const int S = k + 1;
    const size_t L = size_t(dv.L);

    if (tid == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar(B_ITEM_FULL + x), 1);
            mbar_init(bar(B_ITEM_EMPTY + x), kItemConsumers);
            mbar_init(bar(B_Q_FULL + x), 8);
            mbar_init(bar(B_S_FULL + x), 1);
            mbar_init(bar(B_P_FULL + x), 8);
            mbar_init(bar(B_PV_DONE + x), 1);
        }
        for (int x = 0; x < kKSt; ++x) {
            mbar_init(bar(B_K_FULL + x), 1);
            mbar_init(bar(B_K_EMPTY + x), 1);
        }
        for (int x = 0; x < kVSt; ++x) {
            mbar_init(bar(B_V_FULL + x), 1);
            mbar_init(bar(B_V_EMPTY + x), 1);
        }
        mbar_init(bar(B_MMA_DONE), 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc_pair(smem_u32(&sh.tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (warp >= 8) {
        regs_dec<kRegsOther>();
        if (warp == 8 && lane == 0) {
            // ------------------------------------------------------------ producer
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            const int64_t total = n_anchor + tile2_off[int64_t(BH) * dv.C];
            uint32_t gt = 0;
            for (int it = 0;; ++it) {
                const int slot = it & 1;
                int item;
                if (lead) {
                    if (!wait_cl(bar(B_ITEM_EMPTY + slot), ((it >> 1) & 1) ^ 1, abort, hdr, 1)) break;
                    const int64_t ticket = atomicAdd(&hdr[HDR_WORK], 1);
                    item = ticket < total ? int(reverse ? total - 1 - ticket : ticket) : -1;
                    sh.item[slot] = item;
                    st_cluster_u32(mapa(smem_u32(&sh.item[slot]), 1), uint32_t(item));
                    mbar_arrive(bar(B_ITEM_FULL + slot));
                    mbar_arrive_cluster(mapa(bar(B_ITEM_FULL + slot), 1));
                } else {
                    if (!wait_cl(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 17)) break;
                    item = *reinterpret_cast<volatile int*>(&sh.item[slot]);
                    mbar_arrive_cluster(lead_bar(B_ITEM_EMPTY + slot));
                }
                if (item < 0) break;
                Item itm;
                decode_rows<kPairRows>(dv, dv.atile2_off, BH, n_anchor, item, tile2_off, qoff, qlist, itm);
                Cursor cur;
                cur.init(dv, itm);
                const int row0 = itm.bh * dv.L;
                bool stop = false;
                while (cur.more()) {
                    int key0, nvalid;
                    cur.next(key0, nvalid);
                    const int st = gt % kKSt, sv = gt % kVSt;
                    if (!wait_bar(bar(B_K_EMPTY + st), ((gt / kKSt) & 1) ^ 1, abort, hdr, 2)) { stop = true; break; }
                    if (lead) mbar_expect_tx(bar(B_K_FULL + st), 2 * kKHalf);
#pragma unroll
                    for (int s = 0; s < 2; ++s)
                        tma_load_2d_pair(sK + st * kKHalf + s * kKSlab, &tmK, lead_bar(B_K_FULL + st), 64 * s,
                                         row0 + key0 + 64 * int(rank));
                    if (!wait_bar(bar(B_V_EMPTY + sv), ((gt / kVSt) & 1) ^ 1, abort, hdr, 8)) { stop = true; break; }
                    if (lead) mbar_expect_tx(bar(B_V_FULL + sv), 2 * kVHalf);
                    tma_load_2d_pair(sV + sv * kVHalf, &tmV, lead_bar(B_V_FULL + sv), 64 * int(rank), row0 + key0);
                    ++gt;
                }
                if (stop) break;
            }
            // every stage this producer filled has been released by the MMA warp
            // (so its copies have landed and the commits on its barriers arrived)
            const uint64_t deadline = globaltimer() + kTimeoutNs;
            for (uint32_t g = (gt >= uint32_t(kKSt) ? gt - kKSt : 0); g < gt; ++g)
                drain_until(bar(B_K_EMPTY + g % kKSt), (g / kKSt) & 1, deadline, hdr, 9);
            for (uint32_t g = (gt >= uint32_t(kVSt) ? gt - kVSt : 0); g < gt; ++g)
                drain_until(bar(B_V_EMPTY + g % kVSt), (g / kVSt) & 1, deadline, hdr, 18);
        } else if (warp == 9 && lead && lane == 0) {
            // ------------------------------------------------------------ MMA issuer (CTA 0)
            uint32_t gt = 0;
            uint32_t gtt[2] = {0, 0};
            uint32_t itq[2] = {0, 0};
            bool stop = false;
            for (int it = 0; !stop; ++it) {
                const int slot = it & 1;
                if (!wait_cl(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 3)) break;
                const int item = sh.item[slot];
                mbar_arrive(bar(B_ITEM_EMPTY + slot));
                if (item < 0) break;
                Item itm;
                decode_rows<kPairRows>(dv, dv.atile2_off, BH, n_anchor, item, tile2_off, qoff, qlist, itm);
                const int T = count_tiles(dv, itm);
                const int nt = itm.nq > 2 * kQTile ? 2 : 1;  // pair tiles in this item
                for (int q = 0; q < nt && !stop; ++q)
                    if (!wait_cl(bar(B_Q_FULL + q), itq[q] & 1, abort, hdr, 4)) stop = true;
                if (stop) break;
                tc_fence_after();
                for (int j = 0; j <= T && !stop; ++j) {
                    const uint32_t st = gt % kKSt;
                    bool k_ready = false, v_ready = false;
                    for (int q = 0; q < nt; ++q) {
                        if (j > 0) {  // O_q += P_q(j-1) V(j-1)
                            const uint32_t g = gtt[q] - 1, pst = (gt - 1) % kVSt;
                            if (!v_ready) {
                                if (!wait_bar(bar(B_V_FULL + pst), ((gt - 1) / kVSt) & 1, abort, hdr, 15)) { stop = true; break; }
                                v_ready = true;
                            }
                            if (!wait_bar(bar(B_P_FULL + q), g & 1, abort, hdr, 7)) { stop = true; break; }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < kKT / 16; ++kk) {
                                // P's K step kk: 8 TMEM columns (16 keys); V: 16 keys of this CTA's 64 dims
                                const uint64_t vd = sdesc_sw128(sV + pst * kVHalf + kk * 16 * 128, kVHalf, 1024);
                                umma_ts_pair(tmem + col_o(q), tmem + col_s(q) + kk * 8, vd, kIdescPV, (j > 1 || kk > 0));
                            }
                            umma_commit_pair(bar(B_PV_DONE + q), 3);
                        }
                        if (j < T) {  // S_q(j) = Q_q K(j)^T
                            if (!k_ready) {
                                if (!wait_bar(bar(B_K_FULL + st), (gt / kKSt) & 1, abort, hdr, 5)) { stop = true; break; }
                                k_ready = true;
                                tc_fence_after();
                            }
                            const uint32_t qb = sQ + q * kQBytes, kb = sK + st * kKHalf;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t offq = (kk >> 2) * kQSlab + (kk & 3) * 32;
                                const uint32_t offk = (kk >> 2) * kKSlab + (kk & 3) * 32;
                                umma_ss_pair(tmem + col_s(q), sdesc_sw128(qb + offq, 16, 1024),
                                             sdesc_sw128(kb + offk, 16, 1024), kIdescQK, kk > 0);
                            }
                            umma_commit_pair(bar(B_S_FULL + q), 3);
                            ++gtt[q];
                        }
                    }
                    if (stop) break;
                    if (j > 0) umma_commit_pair(bar(B_V_EMPTY + (gt - 1) % kVSt), 3);  // V(j-1) read by PV
                    if (j < T) umma_commit_pair(bar(B_K_EMPTY + st), 3);               // K(j) read by S
                    if (j < T) ++gt;
                }
                for (int q = 0; q < nt; ++q) ++itq[q];
            }
            umma_commit_pair(bar(B_MMA_DONE), 1);
            const uint64_t deadline = globaltimer() + kTimeoutNs;
            drain_until(bar(B_MMA_DONE), 0, deadline, hdr, 10);
        }
        __syncwarp();
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax (warps 0-7)
        const int q = warp >> 2;    // pair tile A (0) or B (1)
        const int row = tid & 127;  // row within this CTA's part of the tile = TMEM lane
        const uint32_t lane_addr = tmem + (uint32_t((warp & 3) * 32) << 16);
        const uint32_t s_addr = lane_addr + col_s(q), o_addr = lane_addr + col_o(q);
        const uint32_t sQq = sQ + q * kQBytes;
        uint32_t gtt = 0;
        for (int it = 0;; ++it) {
            const int slot = it & 1;
            if (!wait_cl_warp(bar(B_ITEM_FULL + slot), (it >> 1) & 1, abort, hdr, 11)) break;
            const int item = *reinterpret_cast<volatile int*>(&sh.item[slot]);
            __syncwarp();
            if (lane == 0) {  // CTA 1's reads of the slot are released at cluster scope
                if (lead) mbar_arrive(bar(B_ITEM_EMPTY + slot));
                else mbar_arrive_cluster(lead_bar(B_ITEM_EMPTY + slot));
            }
            if (item < 0) break;
            Item itm;
            decode_rows<kPairRows>(dv, dv.atile2_off, BH, n_anchor, item, tile2_off, qoff, qlist, itm);
            if (q == 1 && itm.nq <= 2 * kQTile) continue;  // no pair tile B in this item
            const int r_item = q * 2 * kQTile + int(rank) * kQTile + row;  // row within the item
            const unsigned char* Qb = Q + size_t(itm.bh) * L * D * 2;
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
            // gather the warp's 32 query rows into the swizzled tile, every load first
            constexpr int CH = D * 2 / 16;
            uint4 qv[CH];
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int tok = __shfl_sync(0xffffffffu, my_tok, (i * 32 + lane) / CH);
                qv[i] = make_uint4(0, 0, 0, 0);
                if (tok >= 0) qv[i] = ldg_nc16(Qb + size_t(tok) * D * 2 + ((i * 32 + lane) % CH) * 16);
            }
#pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int idx = i * 32 + lane;
                const int r = (warp & 3) * 32 + idx / CH, ch = idx % CH;
                const uint32_t dst = sQq + (ch >> 3) * kQSlab + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(qv[i].x), "r"(qv[i].y),
                             "r"(qv[i].z), "r"(qv[i].w) : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {  // CTA 1's gathered rows are released at cluster scope
                if (lead) mbar_arrive(bar(B_Q_FULL + q));
                else mbar_arrive_cluster(lead_bar(B_Q_FULL + q));
            }

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
                if (nvalid < kKT) {
#pragma unroll
                    for (int c = 0; c < kKT; ++c)
                        if (c >= nvalid) s[c] = __float_as_uint(-INFINITY);
                }
                float a[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) a[i] = fmaxf(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
#pragma unroll
                for (int c = 16; c < kKT; c += 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) a[i] = max3(a[i], __uint_as_float(s[c + 2 * i]), __uint_as_float(s[c + 2 * i + 1]));
                }
                const float mx = max3(max3(a[0], a[1], a[2]), max3(a[3], a[4], a[5]), fmaxf(a[6], a[7])) * scale_log2;
                float alpha = 1.f;
                bool rescale = false;
                if (j == 0) {
                    m_used = mx;
                } else if (mx > m_used + 8.f) {  // lazy rescale: only when the max grew by > 2^8
                    alpha = ex2(m_used - mx);
                    m_used = mx;
                    rescale = true;
                }
                if (__any_sync(0xffffffffu, rescale)) {
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
                const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_used, -m_used);
                uint64_t sum2a = 0, sum2b = 0;
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
                float r0, r1, r2, r3;
                f2_unpack(sum2a, r0, r1);
                f2_unpack(sum2b, r2, r3);
                l = l * alpha + ((r0 + r1) + (r2 + r3));
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                // P lives in TMEM, ordered by the tcgen05 fences: CTA 1's arrival needs no
                // cluster-scope release (that fence on every tile cost ~15 %)
                if (lane == 0) {
                    if (lead) mbar_arrive(bar(B_P_FULL + q));
                    else mbar_arrive_cluster_relaxed(lead_bar(B_P_FULL + q));
                }
                ++gtt;
            }
            if (stop) break;
            // epilogue: O / l -> partial row and its log-sum-exp, staged per 32-column
            // chunk in the warp's own rows of its Q tile (read by this item's S MMAs
            // only, all complete once the last PV_DONE is seen)
            if (!wait_bar_warp(bar(B_PV_DONE + q), (gtt - 1) & 1, abort, hdr, 14)) break;
            tc_fence_after();
            const float inv = 1.f / l;
            float* dst = (my_tok >= 0) ? o_p + ((size_t(itm.bh) * L + my_tok) * S + my_slot) * D : nullptr;
            float* rdst[8];
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
                const uint32_t stg = sQq + (c & 1) * kQSlab + (warp & 3) * 32 * 128;
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
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no MMA, copy or arrival of the pair is outstanding past this point
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

bool attend_pair_supported(int d) { return d == D; }

cudaError_t launch_attend_pair(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                               int k, float scale, int64_t n_anchor2, char* ws, const WsPlan& p, cudaStream_t s) {
    if (d != D) return cudaErrorInvalidValue;
    CUtensorMap tmK, tmV;
    const int64_t rows = int64_t(BH) * dv.L;
    if (!make_tmap_box(&tmK, K, D, rows, 64) || !make_tmap_box(&tmV, V, D, rows, 128)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attend_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // clusters that fit at once (one CTA per SM); a persistent grid of that many
    int clusters = sms / 2;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * clusters);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = s;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, attend_pair_kernel, &cfg) == cudaSuccess && n > 0 && n < clusters)
            clusters = n;
        cudaGetLastError();
    }
    const AttendSchedule sched = attend_schedule();
    if (sched.n_ctas > 0 && sched.n_ctas / 2 < clusters) clusters = sched.n_ctas / 2 > 0 ? sched.n_ctas / 2 : 1;
    int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.hdr);
    e = cudaMemsetAsync(hdr + HDR_WORK, 0, 2 * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    attend_pair_kernel<<<2 * clusters, kThreads, kSmem, s>>>(
        tmK, tmV, dv, BH, k, scale * 1.4426950408889634f, n_anchor2, static_cast<const unsigned char*>(Q), hdr,
        reinterpret_cast<const int32_t*>(ws + p.qoff), reinterpret_cast<const int32_t*>(ws + p.tile2_off),
        reinterpret_cast<const int32_t*>(ws + p.qlist), reinterpret_cast<float*>(ws + p.lse_p),
        reinterpret_cast<float*>(ws + p.o_p), sched.reverse);
    return cudaGetLastError();
}

}  // namespace moc

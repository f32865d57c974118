// Internal declarations shared by the C-ABI glue and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "moc.h"

namespace moc {

constexpr int kQTile = 128;       // query rows per router tile and per attention MMA tile
constexpr int kItemRows = 256;    // query rows per attention work item (two 128-row tiles)
constexpr int kPairRows = 512;    // query rows per work item of the CTA-pair attention kernel
constexpr int kMaxK = 31;         // top-k limit: 1+k partial slots fit one warp
constexpr int kMaxChunks = 16384; // chunk limit (query-list counters live in shared memory)
constexpr int kQlistBlock = 1024; // queries per block of the query-list builder

// Read-only view of a layout's device tables, passed to kernels by value.
struct DevLayout {
    int32_t L, C, G;
    const int32_t* chunk_off;    // [C+1] token offset of every chunk
    const int32_t* grp_q0;       // [G] first token of the group
    const int32_t* grp_q1;       // [G] one past the last token
    const int32_t* grp_kind;     // [G] MOC_CAPTION / MOC_VIDEO
    const int32_t* ar_off;       // [G+1] offsets into ar
    const int32_t* ar;           // anchor key ranges, (start, end) pairs
    const int32_t* cand_off;     // [G+1] offsets into cand
    const int32_t* cand;         // candidate chunk ids, ascending, per group
    const int32_t* cand_ncausal; // [G] length of the causal prefix of the list
    const int32_t* rtile_off;    // [G+1] prefix of router tiles (kQTile queries) per group
    const int32_t* atile_off;    // [G+1] prefix of anchor items (kItemRows queries), groups in a_order
    const int32_t* a_order;      // [G] groups by descending anchor keys per tile
    const int32_t* atile2_off;   // [G+1] prefix of anchor items of kPairRows queries, groups in a_order
    int32_t S;                   // segments (shots) in stream order
    const int32_t* cand_seg;     // segment of every entry of cand
    const int32_t* grp_seg;      // [G] segment of the group's queries (-1: caption group)
    const int32_t* seg_voff;     // [S+1] offsets into vid of every segment's video chunks
    const int32_t* vid;          // video chunk ids in stream order
    const int32_t* rcost[2];     // [rtiles+1] prefix of estimated router tile costs, full / causal lists
    int32_t* err;                // [2] error word + detail of kernels without a workspace (router)
    // backward (key-major dK / dV): key blocks = a video chunk, or a run of caption
    // chunks that the same query groups attend
    int32_t NKB;
    const int32_t* kb_range;     // [NKB][2] token range (k0, k1) of every key block
    const int32_t* kb_chunk;     // [NKB] video chunk whose query list also attends it (-1: caption run)
    const int32_t* kb_goff;      // [NKB+1] offsets into kb_grp
    const int32_t* kb_grp;       // query groups whose anchor ranges hold the block
    const int32_t* kb_order;     // [NKB] blocks by descending anchoring query rows
    const int32_t* kt_off;       // [NKB+1] prefix of 128-key tiles over kb_order
    int32_t kb_lead;             // leading blocks of kb_order handed out block-major (caption runs)
};

}  // namespace moc

struct moc_layout {
    int device = -1;
    int64_t L = 0;
    int32_t C = 0, G = 0, n_shots = 0;
    int32_t max_cand = 0;       // largest candidate list of any group
    int64_t total_rtiles = 0;   // router tiles per (b, h)
    int64_t total_atiles = 0;   // anchor tiles per (b, h)
    int64_t total_atiles2 = 0;  // anchor items of kPairRows queries per (b, h)
    std::vector<int32_t> chunk_off, kind, shot, frame;
    std::vector<int32_t> grp_q0, grp_q1, grp_kind, ar_off, ar, cand_off, cand, cand_ncausal;
    std::vector<int32_t> rtile_off, atile_off, a_order, atile2_off;
    std::vector<int32_t> cand_seg, grp_seg, seg_voff, vid;  // segments (shots) in stream order
    std::vector<int32_t> rcost_full, rcost_causal;          // router tile cost prefixes
    std::vector<int64_t> grp_keys;  // anchor keys of each group
    std::vector<int32_t> kb_range, kb_chunk, kb_goff, kb_grp, kb_order, kt_off;  // backward key blocks
    int64_t total_ktiles = 0;       // 128-key tiles per (b, h)
    int32_t kb_lead = 0;            // caption-run blocks at the head of kb_order
    void* dev_block = nullptr;
    moc::DevLayout dv{};
};

namespace moc {

// Workspace carve-up of moc_attention_fwd (all offsets 256-byte aligned).
struct WsPlan {
    size_t hdr = 0;        // int32[64]: [0] error code, [1] detail, [2] work counter
    size_t blk_count = 0;  // int32 [BH][nblk][C]
    size_t qoff = 0;       // int32 [BH*C + 1] global start of every list
    size_t tile_off = 0;   // int32 [BH*C + 1] prefix of routed items (kItemRows entries each)
    size_t tile2_off = 0;  // int32 [BH*C + 1] prefix of routed items of kPairRows entries
    size_t qlist = 0;      // int32 [BH*L*k] entries (query << 5 | slot)
    size_t lse_p = 0;      // fp32 [BH][L][1+k]
    size_t o_p = 0;        // fp32 [BH][L][1+k][d]
    size_t total = 0;
    int nblk = 0;
};
WsPlan plan_workspace(const moc_layout* lay, int B, int H, int d, int k);

enum { HDR_ERR = 0, HDR_DETAIL = 1, HDR_WORK = 2, HDR_RDONE = 3 };
enum { ERR_NONE = 0, ERR_TIMEOUT = 1, ERR_CHECK = 2 };

// Work schedule of the attention kernel (moc_set_attend_schedule): CTAs
// (0: one per SM) and the order items are handed out in (reverse != 0: last
// first). Results never depend on it.
struct AttendSchedule {
    int n_ctas = 0;
    int reverse = 0;
};
AttendSchedule attend_schedule();

// Kernel launchers (return cudaGetLastError() of the launch).
cudaError_t launch_pool(const DevLayout& dv, int BH, int d, const void* K, float* Kbar,
                        cudaStream_t s);
cudaError_t launch_route(const DevLayout& dv, int BH, int64_t rtiles, int d, const void* Q,
                         const float* Kbar, int k, int causal, int max_cand, const uint64_t* seg_mask,
                         int32_t* sel, cudaStream_t s);
cudaError_t launch_outer(const DevLayout& dv, int BH, int d, const float* Qbar, const float* Kbar, int M,
                         int causal, uint64_t* seg_mask, cudaStream_t s);
cudaError_t launch_qlists(const DevLayout& dv, int BH, int k, const int32_t* sel, char* ws,
                          const WsPlan& p, cudaStream_t s);
cudaError_t launch_attend_tc(const DevLayout& dv, int BH, int d, const void* Q, const void* K,
                             const void* V, int k, float scale, int64_t n_anchor_items, char* ws,
                             const WsPlan& p, cudaStream_t s);
// (4) on CTA pairs (cta_group::2; bf16, d = 128 only): items of kPairRows rows,
// n_anchor2 = B*H x the layout's total_atiles2, routed items from the plan's tile2_off.
bool attend_pair_supported(int d);
cudaError_t launch_attend_pair(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                               int k, float scale, int64_t n_anchor2, char* ws, const WsPlan& p, cudaStream_t s);
// Kernel of the attention stage (moc_set_attend_kernel): 0 default, 1 single CTA, 2 CTA pairs.
int attend_kernel_choice();
cudaError_t launch_attend_merged(const DevLayout& dv, int BH, int d, const void* Q, const void* K,
                                 const void* V, int k, float scale, int64_t n_anchor, char* ws,
                                 const WsPlan& p, const int32_t* sel, void* O, float* lse, cudaStream_t s);
cudaError_t launch_attend_e4m3(const DevLayout& dv, int BH, const void* Q8, const void* K8, const void* V8,
                               const float* q_scale, const float* k_scale, const float* v_scale, int k, float scale,
                               int64_t n_anchor, char* ws, const WsPlan& p, cudaStream_t s);
cudaError_t launch_quant_e4m3(int BH, int64_t L, int d, const void* X, void* X8, float* scale, cudaStream_t s);
cudaError_t launch_merge(int BH, int L, int d, int k, const int32_t* sel, void* O, float* lse,
                         const char* ws, const WsPlan& p, cudaStream_t s);

// Backward pass (dQ, dK, dV). The workspace holds the forward plan's header and
// query lists; lse_p holds D = dO . o per row (fp32 [BH][L]) and o_p the dQ
// partial rows (fp32 [BH][L][1+k][d]).
WsPlan plan_workspace_bwd(const moc_layout* lay, int B, int H, int d, int k);
cudaError_t launch_bwd_rowdot(int BH, int L, int d, const void* O, const void* dO, char* ws, const WsPlan& p,
                              cudaStream_t s);
cudaError_t launch_bwd_dq(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                          const void* dO, const float* lse, int k, float scale, int64_t n_anchor, char* ws,
                          const WsPlan& p, cudaStream_t s);
cudaError_t launch_bwd_dq_reduce(int BH, int L, int C, int d, int k, const int32_t* sel, void* dQ, const char* ws,
                                 const WsPlan& p, cudaStream_t s);
cudaError_t launch_bwd_dkv(const DevLayout& dv, int BH, int d, const void* Q, const void* K, const void* V,
                           const void* dO, const float* lse, float scale, char* ws, const WsPlan& p, void* dK,
                           void* dV, cudaStream_t s);

// Poisson distribution function at 0 .. m_max-1 scaled to 2^32 (drop-in counts)
struct PoissonThresholds {
    uint64_t t[kMaxK];
};
cudaError_t launch_perturb(const DevLayout& dv, int BH, int k, int m_max, int causal, const int32_t* sel,
                           const uint32_t* rnd, float p_max, const PoissonThresholds& thr, int32_t* out,
                           cudaStream_t s);

}  // namespace moc

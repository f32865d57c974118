// Scene layout: chunk tables, query groups, anchor key ranges and candidate
// lists, built once per scene on the host and copied to the device.
//
// Follows the jxzklqfsx.com MoC write-up, "計算效率" (the token stream is
// tagged with frame / shot / text boundaries, prefix-sum tables give
// variable-length chunk starts and ends, and the mandatory links are inserted
// before top-k as a pre-routing mask), "固定的跨模態選擇" (every visual query
// sees all text tokens) and "固定的鏡頭內選擇" (every token sees its own
// shot); and "Mixture of Contexts for Long Video Generation | Summary" §3.2
// (optional edges i->j are masked when j >= i). The local-window anchor of
// single-shot scenes follows the abstract of "Miscela di Contesti per la
// Generazione di Video Lunghi" (mandatory local windows).
//
// Structure used by the kernels: a *query group* is a maximal run of
// consecutive chunks whose queries share one anchor set (a shot, a frame
// window, a chunk, or a run of caption segments). Every group is a contiguous
// token range. Its candidates are the video chunks outside its anchor set in
// ascending id order; under the causal mask exactly the prefix of that list
// with ids below the group's first chunk remains, because every chunk of the
// group is itself mandatory for every query of the group.
#include <algorithm>
#include <cstring>
#include <new>
#include <numeric>
#include <set>

#include "moc_internal.h"

namespace {

moc_status build_host(const moc_layout_desc* d, moc_layout* lay) {
    const int n = d->n_segments;
    if (n < 1 || n > moc::kMaxChunks) return MOC_ERR_LAYOUT;
    if (!d->seg_len || !d->seg_kind || !d->seg_shot || !d->seg_frame) return MOC_ERR_INVALID_ARG;
    if (d->anchor_mode < MOC_ANCHOR_SHOT || d->anchor_mode > MOC_ANCHOR_CHUNK) return MOC_ERR_LAYOUT;
    if (d->local_radius < 0) return MOC_ERR_LAYOUT;
    lay->C = n;
    lay->chunk_off.assign(n + 1, 0);
    lay->kind.assign(d->seg_kind, d->seg_kind + n);
    lay->shot.assign(d->seg_shot, d->seg_shot + n);
    lay->frame.assign(d->seg_frame, d->seg_frame + n);
    int64_t L = 0;
    for (int i = 0; i < n; ++i) {
        if (d->seg_len[i] <= 0) return MOC_ERR_LAYOUT;  // the mean of an empty chunk is undefined
        if (d->seg_kind[i] != MOC_CAPTION && d->seg_kind[i] != MOC_VIDEO) return MOC_ERR_LAYOUT;
        L += d->seg_len[i];
        if (L >= (int64_t(1) << 26)) return MOC_ERR_UNSUPPORTED;  // entries pack (query << 5 | slot)
        lay->chunk_off[i + 1] = int32_t(L);
    }
    lay->L = L;

    // video chunks in stream order and their shot runs
    std::vector<int32_t> vid;
    for (int i = 0; i < n; ++i)
        if (lay->kind[i] == MOC_VIDEO) vid.push_back(i);
    const int NV = int(vid.size());
    std::vector<int32_t> vpos(n, -1);
    for (int v = 0; v < NV; ++v) vpos[vid[v]] = v;
    // each shot's video chunks must be one run of vid, frames non-decreasing
    std::vector<int32_t> run_lo(NV), run_hi(NV);
    std::set<int32_t> seen;
    std::vector<int32_t> vseg(n, -1);  // segment (shot run, stream order) of every video chunk
    lay->seg_voff.assign(1, 0);
    for (int v = 0; v < NV;) {
        int32_t s = lay->shot[vid[v]];
        if (seen.count(s)) return MOC_ERR_LAYOUT;  // shot split by another shot
        seen.insert(s);
        int w = v;
        while (w < NV && lay->shot[vid[w]] == s) {
            if (w > v && lay->frame[vid[w]] < lay->frame[vid[w - 1]]) return MOC_ERR_LAYOUT;
            ++w;
        }
        for (int x = v; x < w; ++x) {
            run_lo[x] = v;
            run_hi[x] = w;
            vseg[vid[x]] = int32_t(lay->seg_voff.size()) - 1;
        }
        lay->seg_voff.push_back(w);
        v = w;
    }
    lay->n_shots = int32_t(seen.size());
    lay->vid = vid;

    // anchor video range [alo, ahi) in vid-space of every video chunk
    std::vector<int32_t> alo(n, -1), ahi(n, -1);
    for (int v = 0; v < NV; ++v) {
        const int i = vid[v];
        if (d->anchor_mode == MOC_ANCHOR_SHOT) {
            alo[i] = run_lo[v];
            ahi[i] = run_hi[v];
        } else if (d->anchor_mode == MOC_ANCHOR_CHUNK) {
            alo[i] = v;
            ahi[i] = v + 1;
        } else {
            const int f = lay->frame[i], r = d->local_radius;
            int lo = v, hi = v + 1;
            while (lo > run_lo[v] && lay->frame[vid[lo - 1]] >= f - r) --lo;
            while (hi < run_hi[v] && lay->frame[vid[hi]] <= f + r) ++hi;
            alo[i] = lo;
            ahi[i] = hi;
        }
    }

    // query groups
    std::vector<std::pair<int, int>> groups;  // chunk range [c0, c1)
    for (int i = 0; i < n;) {
        int j = i + 1;
        if (lay->kind[i] == MOC_CAPTION) {
            while (j < n && lay->kind[j] == MOC_CAPTION) ++j;
        } else {
            while (j < n && lay->kind[j] == MOC_VIDEO && alo[j] == alo[i] && ahi[j] == ahi[i]) ++j;
        }
        groups.push_back({i, j});
        i = j;
    }
    const int G = int(groups.size());
    lay->G = G;
    lay->grp_q0.resize(G);
    lay->grp_q1.resize(G);
    lay->grp_kind.resize(G);
    lay->grp_keys.resize(G);
    lay->ar_off.assign(1, 0);
    lay->cand_off.assign(1, 0);
    lay->cand_ncausal.resize(G);
    lay->grp_seg.assign(G, -1);
    lay->rtile_off.assign(1, 0);
    lay->ar.clear();
    lay->cand.clear();
    lay->cand_seg.clear();
    lay->max_cand = 0;
    for (int g = 0; g < G; ++g) {
        const int c0 = groups[g].first, c1 = groups[g].second;
        lay->grp_q0[g] = lay->chunk_off[c0];
        lay->grp_q1[g] = lay->chunk_off[c1];
        lay->grp_kind[g] = lay->kind[c0];
        std::vector<std::pair<int32_t, int32_t>> rng;
        if (lay->kind[c0] == MOC_CAPTION) {
            rng.push_back({0, int32_t(L)});  // caption queries attend densely
            lay->cand_ncausal[g] = 0;
        } else {
            const int a = alo[c0], b = ahi[c0];
            rng.push_back({lay->chunk_off[vid[a]], lay->chunk_off[vid[b - 1] + 1]});
            for (int c = 0; c < n; ++c)
                if (lay->kind[c] == MOC_CAPTION) rng.push_back({lay->chunk_off[c], lay->chunk_off[c + 1]});
            for (int v = 0; v < a; ++v) lay->cand.push_back(vid[v]);
            lay->cand_ncausal[g] = a;
            for (int v = b; v < NV; ++v) lay->cand.push_back(vid[v]);
            for (int v = 0; v < a; ++v) lay->cand_seg.push_back(vseg[vid[v]]);
            for (int v = b; v < NV; ++v) lay->cand_seg.push_back(vseg[vid[v]]);
            lay->grp_seg[g] = vseg[c0];
        }
        std::sort(rng.begin(), rng.end());
        std::vector<std::pair<int32_t, int32_t>> merged;
        for (auto& r : rng) {
            if (!merged.empty() && r.first <= merged.back().second)
                merged.back().second = std::max(merged.back().second, r.second);
            else
                merged.push_back(r);
        }
        int64_t keys = 0;
        for (auto& r : merged) {
            lay->ar.push_back(r.first);
            lay->ar.push_back(r.second);
            keys += r.second - r.first;
        }
        lay->grp_keys[g] = keys;
        lay->ar_off.push_back(int32_t(lay->ar.size() / 2));
        lay->cand_off.push_back(int32_t(lay->cand.size()));
        lay->max_cand = std::max(lay->max_cand, lay->cand_off[g + 1] - lay->cand_off[g]);
        const int32_t nq = lay->grp_q1[g] - lay->grp_q0[g];
        lay->rtile_off.push_back(lay->rtile_off.back() + (nq + moc::kQTile - 1) / moc::kQTile);
    }
    lay->total_rtiles = lay->rtile_off.back();
    // estimated cost of every router tile, for splitting the tiles into contiguous
    // per-CTA ranges of equal work: a fixed part for a tile that has candidates (Q
    // stream, MMAs, barrier hand-offs) plus a quarter per candidate (the per-row
    // top-k); 1 for a tile without candidates (its rows are only written). The
    // weights were measured: on the eight-shot scene a fixed part of 32 beat 8, 16,
    // 48 and 64 (0.40 ms against 0.47, 0.43, 0.42 and 0.43).
    lay->rcost_full.assign(1, 0);
    lay->rcost_causal.assign(1, 0);
    for (int g = 0; g < G; ++g) {
        const int32_t ntile = lay->rtile_off[g + 1] - lay->rtile_off[g];
        const bool video = lay->grp_kind[g] == MOC_VIDEO;
        const int32_t nfull = video ? lay->cand_off[g + 1] - lay->cand_off[g] : 0;
        const int32_t ncaus = video ? lay->cand_ncausal[g] : 0;
        const int32_t cf = nfull > 0 ? 32 + (nfull + 3) / 4 : 1;
        const int32_t cc = ncaus > 0 ? 32 + (ncaus + 3) / 4 : 1;
        for (int32_t i = 0; i < ntile; ++i) {
            lay->rcost_full.push_back(lay->rcost_full.back() + cf);
            lay->rcost_causal.push_back(lay->rcost_causal.back() + cc);
        }
    }
    // anchor work items of kItemRows queries: groups with the most keys first (longest work first)
    lay->a_order.resize(G);
    std::iota(lay->a_order.begin(), lay->a_order.end(), 0);
    std::stable_sort(lay->a_order.begin(), lay->a_order.end(),
                     [&](int x, int y) { return lay->grp_keys[x] > lay->grp_keys[y]; });
    lay->atile_off.assign(1, 0);
    for (int x = 0; x < G; ++x) {
        const int g = lay->a_order[x];
        const int32_t nq = lay->grp_q1[g] - lay->grp_q0[g];
        lay->atile_off.push_back(lay->atile_off.back() + (nq + moc::kItemRows - 1) / moc::kItemRows);
    }
    lay->total_atiles = lay->atile_off.back();
    lay->atile2_off.assign(1, 0);
    for (int x = 0; x < G; ++x) {
        const int g = lay->a_order[x];
        const int32_t nq = lay->grp_q1[g] - lay->grp_q0[g];
        lay->atile2_off.push_back(lay->atile2_off.back() + (nq + moc::kPairRows - 1) / moc::kPairRows);
    }
    lay->total_atiles2 = lay->atile2_off.back();

    // Key blocks of the backward pass. Every key is attended by the queries of the
    // groups whose anchor ranges hold it and, for a video chunk, by the queries that
    // selected that chunk. A video chunk is its own block (its selecting queries
    // are its own); consecutive caption chunks attended by the same groups (every
    // group: captions are mandatory for all queries) form one block.
    std::vector<std::vector<int32_t>> anch(n);
    for (int g = 0; g < G; ++g) {
        for (int r = lay->ar_off[g]; r < lay->ar_off[g + 1]; ++r) {
            const int32_t a = lay->ar[2 * r], b = lay->ar[2 * r + 1];
            int c = int(std::upper_bound(lay->chunk_off.begin(), lay->chunk_off.end(), a) - lay->chunk_off.begin()) - 1;
            for (; c < n && lay->chunk_off[c] < b; ++c) anch[c].push_back(g);
        }
    }
    lay->kb_range.clear();
    lay->kb_chunk.clear();
    lay->kb_goff.assign(1, 0);
    lay->kb_grp.clear();
    std::vector<int64_t> kb_rows;  // anchoring query rows of every block
    for (int c = 0; c < n;) {
        int e = c + 1;
        if (lay->kind[c] == MOC_CAPTION)
            while (e < n && lay->kind[e] == MOC_CAPTION && anch[e] == anch[c]) ++e;
        lay->kb_range.push_back(lay->chunk_off[c]);
        lay->kb_range.push_back(lay->chunk_off[e]);
        lay->kb_chunk.push_back(lay->kind[c] == MOC_VIDEO ? c : -1);
        int64_t rows = 0;
        for (int32_t g : anch[c]) {
            lay->kb_grp.push_back(g);
            rows += lay->grp_q1[g] - lay->grp_q0[g];
        }
        lay->kb_goff.push_back(int32_t(lay->kb_grp.size()));
        kb_rows.push_back(rows);
        c = e;
    }
    const int NKB = int(kb_rows.size());
    lay->kb_order.resize(NKB);
    std::iota(lay->kb_order.begin(), lay->kb_order.end(), 0);
    std::stable_sort(lay->kb_order.begin(), lay->kb_order.end(),
                     [&](int x, int y) { return kb_rows[x] > kb_rows[y]; });
    lay->kt_off.assign(1, 0);
    for (int x = 0; x < NKB; ++x) {
        const int b = lay->kb_order[x];
        const int32_t nk = lay->kb_range[2 * b + 1] - lay->kb_range[2 * b];
        lay->kt_off.push_back(lay->kt_off.back() + (nk + moc::kQTile - 1) / moc::kQTile);
    }
    lay->total_ktiles = lay->kt_off.back();
    // caption runs are attended by every query (the longest units): they lead
    lay->kb_lead = 0;
    while (lay->kb_lead < NKB && lay->kb_chunk[lay->kb_order[lay->kb_lead]] < 0) ++lay->kb_lead;
    return MOC_OK;
}

moc_status upload(moc_layout* lay) {
    std::vector<const std::vector<int32_t>*> tabs = {
        &lay->chunk_off, &lay->grp_q0, &lay->grp_q1, &lay->grp_kind, &lay->ar_off, &lay->ar,
        &lay->cand_off, &lay->cand, &lay->cand_ncausal, &lay->rtile_off, &lay->atile_off,
        &lay->a_order, &lay->cand_seg, &lay->grp_seg, &lay->seg_voff, &lay->vid,
        &lay->rcost_full, &lay->rcost_causal, &lay->kb_range, &lay->kb_chunk, &lay->kb_goff,
        &lay->kb_grp, &lay->kb_order, &lay->kt_off, &lay->atile2_off};
    std::vector<size_t> offs;
    size_t total = 0;
    for (auto* t : tabs) {
        offs.push_back(total);
        total += ((t->size() * sizeof(int32_t) + 255) / 256) * 256 + 256;
    }
    const size_t err_off = total;  // device error word of the router (zeroed)
    total += 256;
    std::vector<char> host(total, 0);
    for (size_t i = 0; i < tabs.size(); ++i)
        if (!tabs[i]->empty()) memcpy(host.data() + offs[i], tabs[i]->data(), tabs[i]->size() * 4);
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess) return MOC_ERR_CUDA;
    if (cudaSetDevice(lay->device) != cudaSuccess) return MOC_ERR_CUDA;
    moc_status st = MOC_OK;
    if (cudaMalloc(&lay->dev_block, total) != cudaSuccess ||
        cudaMemcpy(lay->dev_block, host.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) {
        st = MOC_ERR_CUDA;
    }
    cudaSetDevice(prev);
    if (st != MOC_OK) return st;
    auto at = [&](int i) { return reinterpret_cast<const int32_t*>(static_cast<char*>(lay->dev_block) + offs[i]); };
    moc::DevLayout& dv = lay->dv;
    dv.L = int32_t(lay->L);
    dv.C = lay->C;
    dv.G = lay->G;
    dv.chunk_off = at(0);
    dv.grp_q0 = at(1);
    dv.grp_q1 = at(2);
    dv.grp_kind = at(3);
    dv.ar_off = at(4);
    dv.ar = at(5);
    dv.cand_off = at(6);
    dv.cand = at(7);
    dv.cand_ncausal = at(8);
    dv.rtile_off = at(9);
    dv.atile_off = at(10);
    dv.a_order = at(11);
    dv.S = lay->n_shots;
    dv.cand_seg = at(12);
    dv.grp_seg = at(13);
    dv.seg_voff = at(14);
    dv.vid = at(15);
    dv.rcost[0] = at(16);
    dv.rcost[1] = at(17);
    dv.NKB = int32_t(lay->kb_chunk.size());
    dv.kb_range = at(18);
    dv.kb_chunk = at(19);
    dv.kb_goff = at(20);
    dv.kb_grp = at(21);
    dv.kb_order = at(22);
    dv.kt_off = at(23);
    dv.kb_lead = lay->kb_lead;
    dv.atile2_off = at(24);
    dv.err = reinterpret_cast<int32_t*>(static_cast<char*>(lay->dev_block) + err_off);
    return MOC_OK;
}

}  // namespace

extern "C" moc_status moc_build_layout(const moc_layout_desc* desc, int device, moc_layout** out) {
    if (!out) return MOC_ERR_INVALID_ARG;
    *out = nullptr;
    if (!desc || device < -1) return MOC_ERR_INVALID_ARG;
    moc_layout* lay = new (std::nothrow) moc_layout();
    if (!lay) return MOC_ERR_INVALID_ARG;
    moc_status st = build_host(desc, lay);
    if (st == MOC_OK && device >= 0) {
        lay->device = device;
        st = upload(lay);
    }
    if (st != MOC_OK) {
        moc_layout_destroy(lay);
        return st;
    }
    *out = lay;
    return MOC_OK;
}

extern "C" void moc_layout_destroy(moc_layout* layout) {
    if (!layout) return;
    if (layout->dev_block) {
        int prev = 0;
        cudaGetDevice(&prev);
        cudaSetDevice(layout->device);
        cudaFree(layout->dev_block);
        cudaSetDevice(prev);
    }
    delete layout;
}

extern "C" moc_status moc_layout_info(const moc_layout* layout, int64_t* L, int32_t* C,
                                      int32_t* n_shots) {
    if (!layout) return MOC_ERR_INVALID_ARG;
    if (L) *L = layout->L;
    if (C) *C = layout->C;
    if (n_shots) *n_shots = layout->n_shots;
    return MOC_OK;
}

extern "C" moc_status moc_layout_device_error(const moc_layout* layout, int32_t* detail,
                                              moc_stream_t stream) {
    if (!layout || !layout->dev_block) return MOC_ERR_INVALID_ARG;
    int32_t h[2] = {0, 0};
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, layout->dv.err, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOC_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOC_ERR_CUDA;
    if (detail) *detail = (h[0] != moc::ERR_NONE) ? h[1] : 0;
    if (h[0] != moc::ERR_NONE) {
        if (cudaMemsetAsync(layout->dv.err, 0, sizeof h, s) != cudaSuccess) return MOC_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return MOC_ERR_CUDA;
    }
    if (h[0] == moc::ERR_TIMEOUT) return MOC_ERR_DEVICE_TIMEOUT;
    if (h[0] == moc::ERR_CHECK) return MOC_ERR_DEVICE_CHECK;
    return MOC_OK;
}

extern "C" moc_status moc_layout_table(const moc_layout* layout, int which, int32_t* out,
                                       int64_t cap, int64_t* count) {
    if (!layout || !count || cap < 0 || (cap > 0 && !out)) return MOC_ERR_INVALID_ARG;
    std::vector<int32_t> tmp;
    const std::vector<int32_t>* src = nullptr;
    switch (which) {
        case 0: src = &layout->chunk_off; break;
        case 1:
            for (int g = 0; g < layout->G; ++g) {
                tmp.push_back(layout->grp_q0[g]);
                tmp.push_back(layout->grp_q1[g]);
            }
            src = &tmp;
            break;
        case 2: src = &layout->ar; break;
        case 3: src = &layout->ar_off; break;
        case 4: src = &layout->cand; break;
        case 5: src = &layout->cand_off; break;
        case 6: src = &layout->cand_ncausal; break;
        case 7: src = &layout->cand_seg; break;
        case 8: src = &layout->grp_seg; break;
        case 9: src = &layout->seg_voff; break;
        case 10: src = &layout->vid; break;
        case 11: src = &layout->rcost_full; break;
        case 12: src = &layout->rcost_causal; break;
        case 13: src = &layout->kb_range; break;
        case 14: src = &layout->kb_chunk; break;
        case 15: src = &layout->kb_goff; break;
        case 16: src = &layout->kb_grp; break;
        case 17: src = &layout->kb_order; break;
        case 18: src = &layout->kt_off; break;
        default: return MOC_ERR_INVALID_ARG;
    }
    *count = int64_t(src->size());
    const int64_t m = std::min<int64_t>(cap, *count);
    if (m > 0) memcpy(out, src->data(), size_t(m) * sizeof(int32_t));
    return MOC_OK;
}

// (2') Context drop-off and drop-in on a routed selection (training-time
// routing perturbations).
//
// "Mixture of Contexts for Long Video Generation | Summary", training details
// of the appendix, and "【DL輪読会】Mixture of Contexts for Long Video
// Generation", slide 14: each query's selection is perturbed - drop-off draws
// p_drop ~ Uniform(0, p_max) and removes floor(p_drop * k) selected chunks at
// random, drop-in draws m ~ Poisson(lambda) and adds m random chunks. Routing is
// per head, so every (b, h, query) is perturbed independently.
//
// The random draws come in as data: per query 2 + k + m_max uint32 words w.
// w[0] gives p_drop = (w[0] / 2^32) p_max and n_drop = floor(p_drop k) (in
// double, left to right, capped at the number of selected chunks); the n_drop
// selected entries with the smallest (w[2 + j], j) are removed (a uniform random
// subset); m = #{i < m_max : thr[i] <= w[1]} with thr the Poisson distribution
// function scaled to 2^32 (inversion, truncated at m_max); the a-th added chunk is
// the floor(w[2 + k + a] * n_left / 2^32)-th of the query's remaining routing
// candidates (causal, not mandatory, not in its original selection, not yet
// added) in ascending chunk order. Output: survivors in their original order,
// then the added chunks, -1 padded to k + m_max. Caption queries get all -1.
// One thread per query row; integer work except the one fp64 product. Selected
// chunks are located in the sorted candidate list by binary search; the
// excluded positions are kept sorted, so each pick walks at most k + m_max of them.
#include "common.cuh"

namespace moc {
namespace {

__global__ void __launch_bounds__(256) perturb_kernel(DevLayout dv, int64_t rows, int k, int m_max,
                                                      int causal, const int32_t* __restrict__ sel,
                                                      const uint32_t* __restrict__ rnd, float p_max,
                                                      PoissonThresholds thr, int32_t* __restrict__ out) {
    const int64_t row = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    const int t = int(row % dv.L);
    const int W = k + m_max;
    int32_t* o = out + row * W;
    const int g = upper_index(dv.grp_q0, dv.G, t);
    if (dv.grp_kind[g] != MOC_VIDEO) {
        for (int j = 0; j < W; ++j) o[j] = -1;
        return;
    }
    const int32_t* cands = dv.cand + dv.cand_off[g];
    const int nc = causal ? dv.cand_ncausal[g] : dv.cand_off[g + 1] - dv.cand_off[g];
    const uint32_t* w = rnd + row * (2 + k + m_max);

    int32_t s[kMaxK];
    int n_sel = 0;
    for (int j = 0; j < k; ++j) {
        const int32_t c = sel[row * k + j];
        if (c < 0) break;  // selections are a prefix, -1 padded
        s[n_sel++] = c;
    }
    // n_drop = floor((w0 / 2^32) * p_max * k), three double products left to right
    double x = __dmul_rn(double(w[0]), 0x1p-32);
    x = __dmul_rn(x, double(p_max));
    x = __dmul_rn(x, double(k));
    int nd = int(floor(x));
    if (nd > n_sel) nd = n_sel;
    int n = 0;
    for (int j = 0; j < n_sel; ++j) {
        int rank = 0;  // entries with a smaller (priority, index)
        for (int i = 0; i < n_sel; ++i)
            rank += (w[2 + i] < w[2 + j]) || (w[2 + i] == w[2 + j] && i < j);
        if (rank >= nd) o[n++] = s[j];
    }
    // drop-in: positions (in the ascending candidate list) that are excluded -
    // the selected chunks, then each added one - kept sorted, so the idx-th free
    // candidate is found by walking them once
    int m = 0;
    for (int i = 0; i < m_max; ++i) m += (thr.t[i] <= uint64_t(w[1])) ? 1 : 0;
    int ex[kMaxK] = {};
    int nex = 0;
    auto exclude = [&](int pos) {  // insert into the sorted list
        int i = nex++;
        while (i > 0 && ex[i - 1] > pos) {
            ex[i] = ex[i - 1];
            --i;
        }
        ex[i] = pos;
    };
    for (int j = 0; j < n_sel; ++j) {
        int lo = 0, hi = nc;  // first candidate >= s[j]
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (cands[mid] < s[j]) lo = mid + 1; else hi = mid;
        }
        if (lo < nc && cands[lo] == s[j]) exclude(lo);
    }
    const int n_rem = nc - nex;
    const int n_add = m < n_rem ? m : n_rem;
    for (int a = 0; a < n_add; ++a) {
        int pos = int((uint64_t(w[2 + k + a]) * uint64_t(n_rem - a)) >> 32);
        for (int i = 0; i < nex && ex[i] <= pos; ++i) ++pos;
        o[n++] = cands[pos];
        exclude(pos);
    }
    for (int j = n; j < W; ++j) o[j] = -1;
}

}  // namespace

cudaError_t launch_perturb(const DevLayout& dv, int BH, int k, int m_max, int causal, const int32_t* sel,
                           const uint32_t* rnd, float p_max, const PoissonThresholds& thr, int32_t* out,
                           cudaStream_t s) {
    const int64_t rows = int64_t(BH) * dv.L;
    if (rows == 0) return cudaSuccess;
    const int64_t grid = (rows + 255) / 256;
    perturb_kernel<<<unsigned(grid), 256, 0, s>>>(dv, rows, k, m_max, causal, sel, rnd, p_max, thr, out);
    return cudaGetLastError();
}

}  // namespace moc

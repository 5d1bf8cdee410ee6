// vs_index.cu -- Vertical-Slash index estimation.
//
// MInference 1.0 (hotpaper.ai summary, "key idea"): a Vertical-Slash head
// estimates its globally important columns and diagonals from the last
// `last_q` queries against every key.  For each of those rows i the causal
// row softmax p_ij = exp(s_ij - m_i) / l_i (s_ij = scale q_i . k_j, j <= i)
// is summed per column j (vertical score) and per diagonal o = i - j (slash
// score); the top vertical_size columns and top slash_size diagonals are
// kept.
//
// Two passes over the keys of each head, both on the tensor cores
// (vs_score_tc.cu: exact bf16 products with fp32 accumulation; the softmax
// argument and the sums carried to fp64 accuracy):
//   pass 1: per key chunk, per row, the partial max and sum;
//   merge (vs_rowmerge, here): once per head, the partials into each row's
//     final max and 1/sum;
//   pass 2: recompute the probabilities and reduce them into column sums and
//     diagonal sums in a fixed order (deterministic).  A chunk owns the
//     diagonals whose first key falls in it and recomputes the keys past its
//     end to finish them.
// Then a block-wide radix top-k per head and list (topk.cuh, here).
#include <cfloat>

#include "internal.h"
#include "topk.cuh"

namespace minfer {

namespace {

// (m, l) <- merge of two partial softmax normalisers
__device__ __forceinline__ void merge_ml(double& m, double& l, double m2, double l2) {
    if (m2 == -DBL_MAX || l2 == 0.0) return;
    if (m == -DBL_MAX || l == 0.0) {
        m = m2;
        l = l2;
        return;
    }
    const double mn = fmax(m, m2);
    l = l * exp(m - mn) + l2 * exp(m2 - mn);
    m = mn;
}

// Final per-row normaliser of every listed head, merged once from the chunk
// partials: mrow = max, linv = 1 / sum (0 for a row with no key).
__global__ void vs_rowmerge_kernel(const double* __restrict__ m_part,
                                                        const double* __restrict__ l_part, int L,
                                                        int nchunks, double* mrow, double* linv) {
    const int pos = blockIdx.x;
    for (int r = threadIdx.x; r < L; r += blockDim.x) {
        double mm = -DBL_MAX, ll = 0.0;
        const size_t base = ((size_t)pos * L + r) * nchunks;
        for (int cc = 0; cc < nchunks; ++cc) merge_ml(mm, ll, m_part[base + cc], l_part[base + cc]);
        mrow[(size_t)pos * L + r] = mm;
        linv[(size_t)pos * L + r] = ll > 0.0 ? 1.0 / ll : 0.0;
    }
}

struct GlobalKeys {
    const float* p;
    __device__ uint32_t operator()(int j) const { return float_order_key(p[j]); }
};

// One batched top-k: rows of scores [rows][n], output row stride out_stride,
// -1 past each row's k.
struct TopkJob {
    const float* scores;
    int32_t* out;
    int k, out_stride;
    RowCounts rk;
};

// Blocks [0, rows) take job a, blocks [rows, 2 rows) job b.
__global__ void __launch_bounds__(1024) topk_rows_kernel(int n, int rows,
                                                         const __grid_constant__ TopkJob a,
                                                         const __grid_constant__ TopkJob b) {
    __shared__ TopkSmem s;
    const bool second = (int)blockIdx.x >= rows;
    const TopkJob* job = second ? &b : &a;
    const int row = (int)blockIdx.x - (second ? rows : 0);
    int32_t* o = job->out + (size_t)row * job->out_stride;
    const int kk = min(row < job->rk.n ? job->rk.k[row] : job->k, n);
    for (int t = kk + threadIdx.x; t < job->out_stride; t += blockDim.x) o[t] = -1;
    if (kk <= 0) return;
    if (kk == n) {
        for (int j = threadIdx.x; j < n; j += blockDim.x) o[j] = j;
        return;
    }
    GlobalKeys get{job->scores + (size_t)row * n};
    uint32_t thr;
    int need_eq;
    block_radix_select(get, n, kk, s, thr, need_eq);
    block_select_compact(get, n, kk, thr, need_eq, s, o);
}

template <int D>
cudaError_t launch_vs_index_d(const bf16* q, const bf16* k, int Hq, int Hkv, int N, double scale,
                              int L, int kv, int ks, const HeadList& heads, int32_t* v_idx,
                              int32_t* s_idx, float* vsc, float* ssc, const VsIndexWs& ws,
                              cudaStream_t st, const int32_t* kv_rows, const int32_t* ks_rows) {
    const int n = heads.n;
    cudaError_t e;
    // the score passes on the tensor cores (vs_score_tc.cu) around the row merge
    if ((e = launch_vs_scores_tc(1, q, k, Hq, Hkv, N, D, scale, L, heads, ws, vsc, ssc, st)) !=
        cudaSuccess)
        return e;
    const int ntc = (N + kVsTcChunk - 1) / kVsTcChunk;
    vs_rowmerge_kernel<<<n, 64, 0, st>>>(ws.m_part, ws.l_part, L, ntc, ws.mrow, ws.linv);
    if ((e = launch_vs_scores_tc(2, q, k, Hq, Hkv, N, D, scale, L, heads, ws, vsc, ssc, st)) !=
        cudaSuccess)
        return e;
    TopkJob jv{vsc, v_idx, kv, kv, {}}, js{ssc, s_idx, ks, ks, {}};
    if (kv_rows) {
        jv.rk.n = n;
        for (int i = 0; i < n; ++i) jv.rk.k[i] = kv_rows[i];
    }
    if (ks_rows) {
        js.rk.n = n;
        for (int i = 0; i < n; ++i) js.rk.k[i] = ks_rows[i];
    }
    topk_rows_kernel<<<2 * n, 1024, 0, st>>>(N, n, jv, js);
    return cudaGetLastError();
}

}  // namespace

VsIndexWs carve_vs_index(WsCarver& c, int n_heads, int N, int L, bool need_vscore,
                         bool need_sscore) {
    const int nchunks = (N + kVsTcChunk - 1) / kVsTcChunk;
    VsIndexWs w{};
    w.m_part = c.take<double>((size_t)n_heads * L * nchunks);
    w.l_part = c.take<double>((size_t)n_heads * L * nchunks);
    w.mrow = c.take<double>((size_t)n_heads * L);
    w.linv = c.take<double>((size_t)n_heads * L);
    w.vscore = need_vscore ? c.take<float>((size_t)n_heads * N) : nullptr;
    w.sscore = need_sscore ? c.take<float>((size_t)n_heads * N) : nullptr;
    // per 64-row group partial scores, merged per head when last_q > 64
    const int G = (L + 63) / 64;
    w.vpart = G > 1 ? c.take<float>((size_t)n_heads * G * N) : nullptr;
    w.spart = G > 1 ? c.take<float>((size_t)n_heads * G * N) : nullptr;
    return w;
}

cudaError_t launch_vs_index(const bf16* q, const bf16* k, int Hq, int Hkv, int N, int d,
                            double scale, int L, int kv, int ks, const HeadList& heads,
                            int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score,
                            const VsIndexWs& ws, cudaStream_t st, const int32_t* kv_rows,
                            const int32_t* ks_rows) {
    if (heads.n == 0) return cudaSuccess;
    float* vsc = v_score ? v_score : ws.vscore;
    float* ssc = s_score ? s_score : ws.sscore;
    if (d == 128)
        return launch_vs_index_d<128>(q, k, Hq, Hkv, N, scale, L, kv, ks, heads, v_idx, s_idx,
                                      vsc, ssc, ws, st, kv_rows, ks_rows);
    return launch_vs_index_d<64>(q, k, Hq, Hkv, N, scale, L, kv, ks, heads, v_idx, s_idx, vsc,
                                 ssc, ws, st, kv_rows, ks_rows);
}

}  // namespace minfer

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
// Two passes over the keys of each head:
//   pass 1: per key chunk, per row, the partial max and sum;
//   merge (vs_rowmerge): once per head, the partials into each row's final
//     max and 1/sum;
//   pass 2: recompute the probabilities and reduce them into column sums and
//     diagonal sums in a fixed order (deterministic).  A chunk owns the
//     diagonals whose first key falls in it and recomputes the L-1 keys past
//     its end to finish them.
// For L <= 64 both passes run on the tensor cores (vs_score_tc.cu: exact bf16
// products with fp32 accumulation, softmax argument and sums in fp64).  For
// larger L they run here on CUDA cores in fp64 (vs_rowstat, vs_colslash),
// where the products of bf16 inputs are exact.
// Then a block-wide radix top-k per head and list (topk.cuh).
#include <cfloat>

#include "internal.h"
#include "topk.cuh"

namespace minfer {

namespace {

constexpr int kThreads = 256;

// 64 rows [row0, row0 + nvalid) of a [rows][D] bf16 matrix into shared
// memory as fp64, transposed: dst[t * 64 + r].  Rows past nvalid read 0.
template <int D>
__device__ void load_rows_T(double* dst, const bf16* base, long long row0, int nvalid) {
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int idx = threadIdx.x; idx < 64 * kChunks; idx += blockDim.x) {
        const int r = idx & 63, c = idx >> 6;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (r < nvalid) raw = *reinterpret_cast<const uint4*>(base + (row0 + r) * D + c * 8);
        const bf16* e = reinterpret_cast<const bf16*>(&raw);
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[(c * 8 + u) * 64 + r] = (double)__bfloat162float(e[u]);
    }
}

// Thread -> 4x4 sub-tile of the 64x64 (rows x keys) tile: warp w covers row
// groups 8*(w/4) .. +7 and key groups 4*(w%4) .. +3, lane l row group
// l/4 and key group l%4 within them.  Per step a warp then reads 8 distinct
// 32-byte Q pieces and 4 distinct K pieces (4 conflict-free wavefronts).
__device__ __forceinline__ void tile_coords(int& ty, int& tx) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    ty = (w >> 2) * 8 + (l >> 2);
    tx = (w & 3) * 4 + (l & 3);
}

// The same 64-row tile in two steps, so that the global loads of the next
// tile can be in flight while the current one is used: fetch into registers
// (kTileChunks 16-byte pieces per thread), then widen and store.
template <int D>
struct TileRegs {
    static constexpr int kChunks = D / 8;
    static constexpr int kPer = 64 * kChunks / kThreads;
    uint4 v[kPer];
    __device__ void fetch(const bf16* base, long long row0, int nvalid) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int idx = threadIdx.x + u * kThreads;
            const int r = idx & 63, c = idx >> 6;
            v[u] = make_uint4(0, 0, 0, 0);
            if (r < nvalid) v[u] = *reinterpret_cast<const uint4*>(base + (row0 + r) * D + c * 8);
        }
    }
    __device__ void store_T(double* dst) const {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int idx = threadIdx.x + u * kThreads;
            const int r = idx & 63, c = idx >> 6;
            const bf16* e = reinterpret_cast<const bf16*>(&v[u]);
#pragma unroll
            for (int w = 0; w < 8; ++w) dst[(c * 8 + w) * 64 + r] = (double)__bfloat162float(e[w]);
        }
    }
};

// acc[a][b] = sum_t Qs[t][4ty+a] * Ks[t][4tx+b]; the operands of step t+1 are
// loaded while step t's FMAs run
template <int D>
__device__ __forceinline__ void dot_4x4(const double* Qs, const double* Ks, int ty, int tx,
                                        double (&acc)[4][4]) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    double2 q01 = *reinterpret_cast<const double2*>(Qs + ty * 4);
    double2 q23 = *reinterpret_cast<const double2*>(Qs + ty * 4 + 2);
    double2 k01 = *reinterpret_cast<const double2*>(Ks + tx * 4);
    double2 k23 = *reinterpret_cast<const double2*>(Ks + tx * 4 + 2);
#pragma unroll 8
    for (int t = 0; t < D; ++t) {
        const int tn = t + 1 < D ? t + 1 : t;
        const double2 nq01 = *reinterpret_cast<const double2*>(Qs + tn * 64 + ty * 4);
        const double2 nq23 = *reinterpret_cast<const double2*>(Qs + tn * 64 + ty * 4 + 2);
        const double2 nk01 = *reinterpret_cast<const double2*>(Ks + tn * 64 + tx * 4);
        const double2 nk23 = *reinterpret_cast<const double2*>(Ks + tn * 64 + tx * 4 + 2);
        const double qa[4] = {q01.x, q01.y, q23.x, q23.y};
        const double kb[4] = {k01.x, k01.y, k23.x, k23.y};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = fma(qa[a], kb[b], acc[a][b]);
        q01 = nq01;
        q23 = nq23;
        k01 = nk01;
        k23 = nk23;
    }
}

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

template <int D>
__global__ void __launch_bounds__(kThreads) vs_rowstat_kernel(const bf16* __restrict__ q,
                                                              const bf16* __restrict__ k, int Hq,
                                                              int Hkv, int N, int L, int nchunks,
                                                              HeadList heads, double scale,
                                                              double* m_part, double* l_part) {
    extern __shared__ __align__(16) double sm[];
    double* Qs = sm;
    double* Ks = sm + D * 64;
    const int c = blockIdx.x, pos = blockIdx.y, rt = blockIdx.z;
    const int qh = head_qh(heads.e[pos]);
    const int g = kv_head_of(qh, Hq, Hkv);
    const int r0 = rt * 64, nr = min(64, L - r0);
    const long long i0 = (long long)N - L + r0;
    int tx, ty;
    tile_coords(ty, tx);

    load_rows_T<D>(Qs, q + (long long)qh * N * D, i0, nr);
    const int jb = c * kVsChunk, je = min(N, jb + kVsChunk);
    double m[4], l[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        m[a] = -DBL_MAX;
        l[a] = 0.0;
    }
    const bf16* kb = k + (long long)g * N * D;
    TileRegs<D> next;
    next.fetch(kb, jb, min(64, je - jb));
    for (int j0 = jb; j0 < je; j0 += 64) {
        if (j0 > i0 + nr - 1) break;  // every key past every row: causal
        __syncthreads();
        next.store_T(Ks);
        __syncthreads();
        if (j0 + 64 < je && j0 + 64 <= i0 + nr - 1) next.fetch(kb, j0 + 64, min(64, je - j0 - 64));
        double acc[4][4];
        dot_4x4<D>(Qs, Ks, ty, tx, acc);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int rr = ty * 4 + a;
            const long long i = i0 + rr;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int j = j0 + tx * 4 + b;
                if (rr < nr && j < je && j <= i) {
                    const double s = acc[a][b] * scale;
                    if (s > m[a]) {
                        l[a] = (m[a] == -DBL_MAX ? 0.0 : l[a] * exp(m[a] - s)) + 1.0;
                        m[a] = s;
                    } else {
                        l[a] += exp(s - m[a]);
                    }
                }
            }
        }
    }
    // merge the 16 key groups of each row: 4 lanes of a warp, then 4 warps
    __syncthreads();  // Ks is reused as the merge buffer [4][64] x (m, l)
    double* red = Ks;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
#pragma unroll
        for (int off = 2; off >= 1; off >>= 1) {
            const double m2 = __shfl_xor_sync(0xffffffffu, m[a], off);
            const double l2 = __shfl_xor_sync(0xffffffffu, l[a], off);
            merge_ml(m[a], l[a], m2, l2);
        }
        if ((threadIdx.x & 3) == 0) {
            const int rr = ty * 4 + a, wq = (threadIdx.x >> 5) & 3;
            red[(wq * 64 + rr) * 2] = m[a];
            red[(wq * 64 + rr) * 2 + 1] = l[a];
        }
    }
    __syncthreads();
    if (threadIdx.x < nr) {
        const int rr = threadIdx.x;
        double mm = red[rr * 2], ll = red[rr * 2 + 1];
        for (int wq = 1; wq < 4; ++wq) merge_ml(mm, ll, red[(wq * 64 + rr) * 2], red[(wq * 64 + rr) * 2 + 1]);
        const size_t o = ((size_t)pos * L + r0 + rr) * nchunks + c;
        m_part[o] = mm;
        l_part[o] = ll;
    }
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

template <int D>
__global__ void __launch_bounds__(kThreads) vs_colslash_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k, int Hq, int Hkv, int N, int L,
    int nchunks, HeadList heads, double scale, const double* __restrict__ mrow_g,
    const double* __restrict__ linv_g, float* vscore, float* sscore) {
    extern __shared__ __align__(16) double sm[];
    double* Qs = sm;
    double* Ks = Qs + D * 64;
    double* Ps = Ks + D * 64;   // [64][65]
    double* mrow = Ps + 64 * 65;  // [L]
    double* linv = mrow + L;      // [L]
    double* vacc = linv + L;      // [kVsChunk]
    double* sacc = vacc + kVsChunk;  // [kVsChunk + L]

    const int c = blockIdx.x, pos = blockIdx.y;
    const int qh = head_qh(heads.e[pos]);
    const int g = kv_head_of(qh, Hq, Hkv);
    const int jb = c * kVsChunk, je = min(N, jb + kVsChunk);
    const int jh = min(N, je + L - 1);  // keys needed to finish owned diagonals
    // diagonal o is owned by the chunk holding its first key max(0, N-L-o)
    const long long o_hi = (c == 0) ? (long long)N - 1 : (long long)N - L - jb;
    const long long o_lo = max(0LL, (long long)N - L - je + 1);
    const int n_own = o_hi >= o_lo ? (int)(o_hi - o_lo + 1) : 0;
    int tx, ty;
    tile_coords(ty, tx);

    for (int r = threadIdx.x; r < L; r += blockDim.x) {
        mrow[r] = mrow_g[(size_t)pos * L + r];
        linv[r] = linv_g[(size_t)pos * L + r];
    }
    for (int t = threadIdx.x; t < kVsChunk; t += blockDim.x) vacc[t] = 0.0;
    for (int t = threadIdx.x; t < n_own; t += blockDim.x) sacc[t] = 0.0;

    for (int r0 = 0; r0 < L; r0 += 64) {
        const int nr = min(64, L - r0);
        const long long i0 = (long long)N - L + r0;
        __syncthreads();
        load_rows_T<D>(Qs, q + (long long)qh * N * D, i0, nr);
        const bf16* kb = k + (long long)g * N * D;
        TileRegs<D> next;
        next.fetch(kb, jb, min(64, jh - jb));
        for (int j0 = jb; j0 < jh; j0 += 64) {
            if (j0 > i0 + nr - 1) break;
            __syncthreads();
            next.store_T(Ks);
            __syncthreads();
            if (j0 + 64 < jh && j0 + 64 <= i0 + nr - 1) next.fetch(kb, j0 + 64, min(64, jh - j0 - 64));
            double acc[4][4];
            dot_4x4<D>(Qs, Ks, ty, tx, acc);
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int rr = ty * 4 + a;
                const long long i = i0 + rr;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int jj = tx * 4 + b;
                    const int j = j0 + jj;
                    double p = 0.0;
                    if (rr < nr && j < jh && j <= i)
                        p = exp(acc[a][b] * scale - mrow[r0 + rr]) * linv[r0 + rr];
                    Ps[rr * 65 + jj] = p;
                }
            }
            __syncthreads();
            const int t = threadIdx.x;
            if (t < 64) {
                const int j = j0 + t;
                if (j < je) {
                    double s = 0.0;
                    for (int rr = 0; rr < 64; ++rr) s += Ps[rr * 65 + t];
                    vacc[j - jb] += s;
                }
            } else if (t >= 128 && t < 255) {
                const int dl = t - 128;  // rr - jj + 63
                const long long o = (i0 - j0) + dl - 63;
                if (o >= o_lo && o <= o_hi) {
                    double s = 0.0;
                    const int rlo = max(0, dl - 63), rhi = min(63, dl);
                    for (int rr = rlo; rr <= rhi; ++rr) s += Ps[rr * 65 + (rr - dl + 63)];
                    sacc[o - o_lo] += s;
                }
            }
        }
    }
    __syncthreads();
    for (int j = jb + threadIdx.x; j < je; j += blockDim.x)
        vscore[(size_t)pos * N + j] = (float)vacc[j - jb];
    for (int t = threadIdx.x; t < n_own; t += blockDim.x)
        sscore[(size_t)pos * N + o_lo + t] = (float)sacc[t];
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
size_t rowstat_smem() {
    return (size_t)2 * D * 64 * sizeof(double);
}
template <int D>
size_t colslash_smem(int L) {
    return ((size_t)2 * D * 64 + 64 * 65 + 2 * (size_t)L + kVsChunk + kVsChunk + L) *
           sizeof(double);
}

template <int D>
cudaError_t launch_vs_index_d(const bf16* q, const bf16* k, int Hq, int Hkv, int N, double scale,
                              int L, int kv, int ks, const HeadList& heads, int32_t* v_idx,
                              int32_t* s_idx, float* vsc, float* ssc, const VsIndexWs& ws,
                              cudaStream_t st, const int32_t* kv_rows, const int32_t* ks_rows) {
    const int n = heads.n;
    const int nchunks = (N + kVsChunk - 1) / kVsChunk;
    const int nrt = (L + 63) / 64;
    const size_t sm1 = rowstat_smem<D>(), sm2 = colslash_smem<D>(L);
    cudaError_t e;
    if (L <= 64) {
        // products on the tensor cores (vs_score_tc.cu), same merge
        if ((e = launch_vs_scores_tc(1, q, k, Hq, Hkv, N, D, scale, L, heads, ws, vsc, ssc, st)) !=
            cudaSuccess)
            return e;
        const int ntc = (N + kVsTcChunk - 1) / kVsTcChunk;
        vs_rowmerge_kernel<<<n, 64, 0, st>>>(ws.m_part, ws.l_part, L, ntc, ws.mrow, ws.linv);
        if ((e = launch_vs_scores_tc(2, q, k, Hq, Hkv, N, D, scale, L, heads, ws, vsc, ssc, st)) !=
            cudaSuccess)
            return e;
    } else {
        if ((e = cudaFuncSetAttribute(vs_rowstat_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1)) !=
            cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(vs_colslash_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2)) !=
            cudaSuccess)
            return e;
        vs_rowstat_kernel<D><<<dim3(nchunks, n, nrt), kThreads, sm1, st>>>(
            q, k, Hq, Hkv, N, L, nchunks, heads, scale, ws.m_part, ws.l_part);
        vs_rowmerge_kernel<<<n, 64, 0, st>>>(ws.m_part, ws.l_part, L, nchunks, ws.mrow, ws.linv);
        vs_colslash_kernel<D><<<dim3(nchunks, n), kThreads, sm2, st>>>(
            q, k, Hq, Hkv, N, L, nchunks, heads, scale, ws.mrow, ws.linv, vsc, ssc);
    }
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
    const int nchunks = (N + kVsChunk - 1) / kVsChunk;
    VsIndexWs w{};
    w.m_part = c.take<double>((size_t)n_heads * L * nchunks);
    w.l_part = c.take<double>((size_t)n_heads * L * nchunks);
    w.mrow = c.take<double>((size_t)n_heads * L);
    w.linv = c.take<double>((size_t)n_heads * L);
    w.vscore = need_vscore ? c.take<float>((size_t)n_heads * N) : nullptr;
    w.sscore = need_sscore ? c.take<float>((size_t)n_heads * N) : nullptr;
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

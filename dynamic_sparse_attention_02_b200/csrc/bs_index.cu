// bs_index.cu -- Block-Sparse index estimation.
//
// MInference 1.0 (hotpaper.ai summary, "key idea"; aifetchly guide,
// "Block-Sparse Kernel Mechanics"): queries and keys are mean-pooled over
// 64-token blocks, each query block scores every causal key block by the
// dot product of the pooled vectors, and the top-k key blocks are kept.
//
//   meanpool:  Qm[h][b] = mean of q rows 64b..64b+63 (fp64, exact),
//              Km[g][b] likewise.  Pure HBM stream with 16-byte loads.
//   bs_topk:   S[bq][bk] = scale * Qm[bq] . Km[bk] for bk <= bq (fp64 dot
//              products on the fp64 tensor path, ranked as fp32), kept on
//              chip, then a warp-wide radix top-k per query block, ascending
//              output.
#include "internal.h"
#include "topk.cuh"

namespace minfer {

namespace {

constexpr int kPoolThreads = 256;

// One 64-row block per warp: lane l reads 16-byte column chunk l % (D/8) of
// the rows of its row group (64 / (32 / (D/8)) rows), eight loads in flight,
// sums them in fp64 (exact), and the row groups meet by shuffles.
template <int D>
__global__ void __launch_bounds__(kPoolThreads) meanpool_kernel(const bf16* __restrict__ x,
                                                                int N, int nB, HeadList items,
                                                                double* __restrict__ out) {
    constexpr int kCPR = D / 8;          // 16-byte chunks per row
    constexpr int kGroups = 32 / kCPR;   // row groups per warp
    constexpr int kRows = 64 / kGroups;  // rows per lane
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.x * (kPoolThreads / 32) + warp, item = blockIdx.y;
    if (b >= nB) return;
    const int hd = head_qh(items.e[item]);
    const int c = lane % kCPR, grp = lane / kCPR;
    const bf16* base = x + ((long long)hd * N + (long long)b * 64 + grp * kRows) * D + c * 8;
    double acc[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[v] = 0.0;
#pragma unroll
    for (int r0 = 0; r0 < kRows; r0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            raw[u] = *reinterpret_cast<const uint4*>(base + (long long)(r0 + u) * D);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bf16* e = reinterpret_cast<const bf16*>(&raw[u]);
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[v] += (double)__bfloat162float(e[v]);
        }
    }
#pragma unroll
    for (int off = kCPR; off < 32; off <<= 1)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], off);
    if (grp == 0) {  // the means, exact in fp64 (a power-of-two division)
        double2* o = reinterpret_cast<double2*>(out + ((size_t)item * nB + b) * D + c * 8);
#pragma unroll
        for (int v = 0; v < 4; ++v) o[v] = make_double2(acc[2 * v] / 64.0, acc[2 * v + 1] / 64.0);
    }
}

constexpr int kMaxR = 16;       // query-block rows per CTA (fewer when the rows are long)
constexpr int kTopkThreads = 512;
constexpr int kKeyTile = 64;     // key blocks per shared-memory tile
constexpr size_t kBsSmemCap = 227 * 1024;

struct SmemKeys {
    const float* p;
    __device__ uint32_t operator()(int j) const { return float_order_key(p[j]); }
};

// fp64 operand rows in shared memory are padded by 4 doubles, so that the
// 8 x 4 fragments of one quarter-warp (4 rows x 4 columns) fall in distinct banks.
template <int D>
constexpr int bs_row() {
    return D + 4;
}

// Shared memory of one CTA: Qm rows [kMaxR][D + 4] and a Km tile
// [kKeyTile][D + 4], both fp64; scores [R][stride] fp32; one 256-bin
// histogram per warp.
template <int D>
constexpr size_t bs_fixed_smem() {
    return (size_t)kMaxR * bs_row<D>() * 8 + (size_t)kKeyTile * bs_row<D>() * 8 +
           (kTopkThreads / 32) * 256 * 4;
}

// D (8 x 8, fp64) += A (8 x 4) B (4 x 8) on the fp64 tensor path; lane l holds
// A[l / 4][l % 4], B[l % 4][l / 4] and D[l / 4][2 (l % 4) + {0, 1}].
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d0), "+d"(d1)
                 : "d"(a), "d"(b));
}

// CTA = R consecutive query blocks of one head.
//  scores: 16 warps; warp w computes rows 8 (w / 8) .. +7 against key blocks
//          8 (w % 8) .. +7 of each 64-block tile, as fp64 sums of exact fp32
//          products over the d coordinates (operands widened once, on their way
//          into shared memory; one 8 x 8 x 4 fp64 MMA per 4 coordinates);
//          S = scale * sum, rounded to fp32 for ranking.
//  top-k:  warp w selects rows w, w + 16, ... by a warp-wide radix select over
//          its row of S, ties toward the lower block, output ascending.
template <int D>
__global__ void __launch_bounds__(kTopkThreads, 1) bs_topk_kernel(
    const double* __restrict__ qm, const double* __restrict__ km, int Hq, int Hkv, int nB,
    int kvmap_n, HeadList heads, HeadList kvpos, int R, double scale, int topk, RowCounts tk,
    int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt) {
    constexpr int RS = bs_row<D>();
    extern __shared__ __align__(16) double dsm[];
    double* Qs = dsm;                          // [kMaxR][D + 4]
    double* Ks = Qs + kMaxR * RS;              // [kKeyTile][D + 4]
    uint32_t* hist = reinterpret_cast<uint32_t*>(Ks + kKeyTile * RS);  // [8][256]
    float* S = reinterpret_cast<float*>(hist + (kTopkThreads / 32) * 256);  // [R][stride]
    const int pos = blockIdx.y;
    const int bq0 = blockIdx.x * R;
    const int nr = min(R, nB - bq0);
    const int ncand = bq0 + nr;
    const int stride = bq0 + R;
    const int qh = head_qh(heads.e[pos]);
    const int g = kv_head_of(qh, Hq, Hkv);
    // Km is stored per KV head in use; kvpos maps KV head -> its row in Km
    int gi = 0;
    for (int t = 0; t < kvmap_n; ++t)
        if (head_qh(kvpos.e[t]) == g) gi = t;
    const double* kmg = km + (size_t)gi * nB * D;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // the rows' means; rows past nr read 0
    for (int t = threadIdx.x; t < kMaxR * (D / 2); t += blockDim.x) {
        const int r = t / (D / 2), c2 = t % (D / 2);
        double2 f = make_double2(0.0, 0.0);
        if (r < nr) f = *reinterpret_cast<const double2*>(qm + ((size_t)pos * nB + bq0 + r) * D + 2 * c2);
        *reinterpret_cast<double2*>(Qs + r * RS + 2 * c2) = f;
    }
    const int fr = lane >> 2, fc = lane & 3;  // fragment row / column of this lane
    // the key tile is fetched one tile ahead into registers, so that its global
    // loads are in flight while the MMAs of the current tile run
    constexpr int kPf = kKeyTile * (D / 2) / kTopkThreads;  // double2 per thread per tile
    double2 pf[kPf];
    auto fetch = [&](int kt) {
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
            const int t = threadIdx.x + u * kTopkThreads;
            const int kb = t / (D / 2), c2 = t % (D / 2);
            pf[u] = make_double2(0.0, 0.0);
            if (kt + kb < ncand)
                pf[u] = *reinterpret_cast<const double2*>(kmg + (size_t)(kt + kb) * D + 2 * c2);
        }
    };
    fetch(0);
    for (int kt0 = 0; kt0 < ncand; kt0 += kKeyTile) {
        __syncthreads();  // the previous tile has been used
#pragma unroll
        for (int u = 0; u < kPf; ++u) {  // consecutive lanes, consecutive 16 bytes
            const int t = threadIdx.x + u * kTopkThreads;
            const int kb = t / (D / 2), c2 = t % (D / 2);
            *reinterpret_cast<double2*>(Ks + kb * RS + 2 * c2) = pf[u];
        }
        __syncthreads();
        if (kt0 + kKeyTile < ncand) fetch(kt0 + kKeyTile);
        // warp w: rows 8 (w / 8) .. +7 against key blocks 8 (w % 8) .. +7 of the tile
        const int mt = warp >> 3, kg = warp & 7;
        if (kt0 + 8 * kg < ncand && 8 * mt < nr) {
            double c0 = 0.0, c1 = 0.0;
            const double* qa = Qs + (8 * mt + fr) * RS + fc;
            const double* kbp = Ks + (8 * kg + fr) * RS + fc;
#pragma unroll 8
            for (int c = 0; c < D; c += 4) dmma_8x8x4(c0, c1, qa[c], kbp[c]);
            const int k0 = kt0 + 8 * kg + 2 * fc;
            const int r = 8 * mt + fr;
            if (r < nr) {
                if (k0 < ncand) S[r * stride + k0] = (float)(c0 * scale);
                if (k0 + 1 < ncand) S[r * stride + k0 + 1] = (float)(c1 * scale);
            }
        }
    }
    __syncthreads();

    const int budget = pos < tk.n ? tk.k[pos] : topk;  // this head's budget (row stride: topk)
    for (int r = warp; r < nr; r += kTopkThreads / 32) {
        const int bq = bq0 + r;
        const int n = bq + 1;
        const int kk = min(budget, n);
        int32_t* o = blk_idx + ((size_t)pos * nB + bq) * topk;
        for (int t = kk + lane; t < topk; t += 32) o[t] = -1;
        if (lane == 0) blk_cnt[(size_t)pos * nB + bq] = kk;
        if (kk == n) {
            for (int t = lane; t < n; t += 32) o[t] = t;
        } else if (kk > 0) {
            SmemKeys get{S + r * stride};
            uint32_t thr;
            int need_eq;
            warp_radix_select(get, n, kk, hist + warp * 256, thr, need_eq);
            warp_select_compact(get, n, kk, thr, need_eq, o);
        }
    }
}

// Rows per CTA: as many (up to kMaxR) as the score rows leave room for.
template <int D>
int rows_per_cta(int nB) {
    const size_t room = kBsSmemCap - bs_fixed_smem<D>() - 1024;
    int R = (int)(room / (4 * (size_t)(nB + kMaxR)));
    if (R > kMaxR) R = kMaxR;
    if (R < 1) R = 1;
    return R;
}

template <int D>
cudaError_t launch_bs_d(const bf16* q, const bf16* k, int Hq, int Hkv, int N, double scale,
                        int topk, const HeadList& heads, int32_t* blk_idx, int32_t* blk_cnt,
                        const BsIndexWs& ws, cudaStream_t st, const int32_t* topk_rows) {
    const int nB = N / 64;
    // KV heads used by the listed query heads, each once
    HeadList kvs{};
    bool used[MI_MAX_HEADS] = {};
    for (int i = 0; i < heads.n; ++i) used[kv_head_of(head_qh(heads.e[i]), Hq, Hkv)] = true;
    for (int g = 0; g < Hkv; ++g)
        if (used[g]) kvs.e[kvs.n++] = pack_head(g, 0, 0);
    const int pool_x = (nB + kPoolThreads / 32 - 1) / (kPoolThreads / 32);
    meanpool_kernel<D><<<dim3(pool_x, heads.n), kPoolThreads, 0, st>>>(q, N, nB, heads, ws.qm);
    meanpool_kernel<D><<<dim3(pool_x, kvs.n), kPoolThreads, 0, st>>>(k, N, nB, kvs, ws.km);
    RowCounts tk{};
    if (topk_rows) {
        tk.n = heads.n;
        for (int i = 0; i < heads.n; ++i) tk.k[i] = topk_rows[i];
    }
    const int R = rows_per_cta<D>(nB);
    const size_t smem = bs_fixed_smem<D>() + (size_t)R * (nB + R) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bs_topk_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bs_topk_kernel<D><<<dim3((nB + R - 1) / R, heads.n), kTopkThreads, smem, st>>>(
        ws.qm, ws.km, Hq, Hkv, nB, kvs.n, heads, kvs, R, scale, topk, tk, blk_idx, blk_cnt);
    return cudaGetLastError();
}

}  // namespace

BsIndexWs carve_bs_index(WsCarver& c, int n_heads, int Hkv, int N, int d) {
    BsIndexWs w{};
    const int nB = N / 64;
    w.qm = c.take<double>((size_t)n_heads * nB * d);
    w.km = c.take<double>((size_t)Hkv * nB * d);
    return w;
}

cudaError_t launch_bs_index(const bf16* q, const bf16* k, int Hq, int Hkv, int N, int d,
                            double scale, int topk, const HeadList& heads, int32_t* blk_idx,
                            int32_t* blk_cnt, const BsIndexWs& ws, cudaStream_t st,
                            const int32_t* topk_rows) {
    if (heads.n == 0) return cudaSuccess;
    if (d == 128)
        return launch_bs_d<128>(q, k, Hq, Hkv, N, scale, topk, heads, blk_idx, blk_cnt, ws, st,
                                topk_rows);
    return launch_bs_d<64>(q, k, Hq, Hkv, N, scale, topk, heads, blk_idx, blk_cnt, ws, st,
                           topk_rows);
}

}  // namespace minfer

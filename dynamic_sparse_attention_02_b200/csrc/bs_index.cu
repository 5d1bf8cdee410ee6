// bs_index.cu -- Block-Sparse index estimation.
//
// MInference 1.0 (hotpaper.ai summary, "key idea"; aifetchly guide,
// "Block-Sparse Kernel Mechanics"): queries and keys are mean-pooled over
// 64-token blocks, each query block scores every causal key block by the
// dot product of the pooled vectors, and the top-k key blocks are kept.
//
//   meanpool:  Qm[h][b] = mean of q rows 64b..64b+63 (fp64 sum, fp32 out),
//              Km[g][b] likewise.  Pure HBM stream with 16-byte loads.
//   bs_topk:   S[bq][bk] = scale * Qm[bq] . Km[bk] for bk <= bq (fp64 sum of
//              exact fp32 products, ranked as fp32), kept on chip, then a
//              block-wide radix top-k per query block, ascending output.
#include "internal.h"
#include "topk.cuh"

namespace minfer {

namespace {

constexpr int kPoolThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) meanpool_kernel(const bf16* __restrict__ x,
                                                                int N, int nB, HeadList items,
                                                                float* __restrict__ out) {
    constexpr int kCPR = D / 8;                 // 16-byte chunks per row
    constexpr int kRG = kPoolThreads / kCPR;    // row groups
    constexpr int kRows = 64 / kRG;             // rows per thread
    __shared__ double red[kRG * D];
    const int b = blockIdx.x, item = blockIdx.y;
    const int hd = head_qh(items.e[item]);
    const bf16* base = x + ((long long)hd * N + (long long)b * 64) * D;
    const int c = threadIdx.x % kCPR, rg = threadIdx.x / kCPR;
    double acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.0;
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
        const int r = rg + u * kRG;
        const uint4 raw = *reinterpret_cast<const uint4*>(base + (long long)r * D + c * 8);
        const bf16* e = reinterpret_cast<const bf16*>(&raw);
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] += (double)__bfloat162float(e[v]);
    }
#pragma unroll
    for (int v = 0; v < 8; ++v) red[rg * D + c * 8 + v] = acc[v];
    __syncthreads();
    for (int col = threadIdx.x; col < D; col += blockDim.x) {
        double s = 0.0;
        for (int g = 0; g < kRG; ++g) s += red[g * D + col];
        out[((size_t)item * nB + b) * D + col] = (float)(s / 64.0);
    }
}

constexpr int kMaxR = 16;
constexpr int kTopkThreads = 256;

struct SmemKeys {
    const float* p;
    __device__ uint32_t operator()(int j) const { return float_order_key(p[j]); }
};

template <int D>
__global__ void __launch_bounds__(kTopkThreads) bs_topk_kernel(
    const float* __restrict__ qm, const float* __restrict__ km, int Hq, int Hkv, int nB,
    int kvmap_n, HeadList heads, HeadList kvpos, int R, double scale, int topk,
    int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt) {
    extern __shared__ __align__(16) float fsm[];
    __shared__ TopkSmem ts;
    const int pos = blockIdx.y;
    const int bq0 = blockIdx.x * R;
    const int nr = min(R, nB - bq0);
    const int ncand = bq0 + nr;
    const int stride = bq0 + R;
    float* Qs = fsm;           // [R][D]
    float* S = fsm + R * D;    // [R][stride]
    const int qh = head_qh(heads.e[pos]);
    const int g = kv_head_of(qh, Hq, Hkv);
    // Km is stored per KV head in use; kvpos maps KV head -> its row in Km
    int gi = 0;
    for (int t = 0; t < kvmap_n; ++t)
        if (head_qh(kvpos.e[t]) == g) gi = t;
    const float* kmg = km + (size_t)gi * nB * D;

    for (int t = threadIdx.x; t < nr * D; t += blockDim.x)
        Qs[t] = qm[((size_t)pos * nB + bq0) * D + t];
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int bk = warp; bk < ncand; bk += kTopkThreads / 32) {
        double acc[kMaxR];
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) acc[r] = 0.0;
#pragma unroll
        for (int u = 0; u < D / 32; ++u) {
            const int t = lane + 32 * u;
            const double kv = (double)kmg[(size_t)bk * D + t];
#pragma unroll
            for (int r = 0; r < kMaxR; ++r)
                if (r < nr) acc[r] = fma((double)Qs[r * D + t], kv, acc[r]);
        }
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) {
            if (r >= nr) break;
            double a = acc[r];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
            if (lane == 0) S[r * stride + bk] = (float)(a * scale);
        }
    }
    __syncthreads();

    for (int r = 0; r < nr; ++r) {
        const int bq = bq0 + r;
        const int n = bq + 1;
        const int kk = min(topk, n);
        int32_t* o = blk_idx + ((size_t)pos * nB + bq) * topk;
        for (int t = kk + threadIdx.x; t < topk; t += blockDim.x) o[t] = -1;
        if (threadIdx.x == 0) blk_cnt[(size_t)pos * nB + bq] = kk;
        if (kk == n) {
            for (int t = threadIdx.x; t < n; t += blockDim.x) o[t] = t;
        } else if (kk > 0) {
            SmemKeys get{S + r * stride};
            uint32_t thr;
            int need_eq;
            block_radix_select(get, n, kk, ts, thr, need_eq);
            block_select_compact(get, n, kk, thr, need_eq, ts, o);
        }
        __syncthreads();
    }
}

int rows_per_cta(int nB) {
    int R = 24576 / (nB > 0 ? nB : 1);
    if (R > kMaxR) R = kMaxR;
    if (R < 1) R = 1;
    return R;
}

template <int D>
cudaError_t launch_bs_d(const bf16* q, const bf16* k, int Hq, int Hkv, int N, double scale,
                        int topk, const HeadList& heads, int32_t* blk_idx, int32_t* blk_cnt,
                        const BsIndexWs& ws, cudaStream_t st) {
    const int nB = N / 64;
    // KV heads used by the listed query heads, each once
    HeadList kvs{};
    bool used[MI_MAX_HEADS] = {};
    for (int i = 0; i < heads.n; ++i) used[kv_head_of(head_qh(heads.e[i]), Hq, Hkv)] = true;
    for (int g = 0; g < Hkv; ++g)
        if (used[g]) kvs.e[kvs.n++] = pack_head(g, 0, 0);
    meanpool_kernel<D><<<dim3(nB, heads.n), kPoolThreads, 0, st>>>(q, N, nB, heads, ws.qm);
    meanpool_kernel<D><<<dim3(nB, kvs.n), kPoolThreads, 0, st>>>(k, N, nB, kvs, ws.km);
    const int R = rows_per_cta(nB);
    const size_t smem = ((size_t)R * D + (size_t)R * (nB + R)) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bs_topk_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bs_topk_kernel<D><<<dim3((nB + R - 1) / R, heads.n), kTopkThreads, smem, st>>>(
        ws.qm, ws.km, Hq, Hkv, nB, kvs.n, heads, kvs, R, scale, topk, blk_idx, blk_cnt);
    return cudaGetLastError();
}

}  // namespace

BsIndexWs carve_bs_index(WsCarver& c, int n_heads, int Hkv, int N, int d) {
    BsIndexWs w{};
    const int nB = N / 64;
    w.qm = c.take<float>((size_t)n_heads * nB * d);
    w.km = c.take<float>((size_t)Hkv * nB * d);
    return w;
}

cudaError_t launch_bs_index(const bf16* q, const bf16* k, int Hq, int Hkv, int N, int d,
                            double scale, int topk, const HeadList& heads, int32_t* blk_idx,
                            int32_t* blk_cnt, const BsIndexWs& ws, cudaStream_t st) {
    if (heads.n == 0) return cudaSuccess;
    if (d == 128)
        return launch_bs_d<128>(q, k, Hq, Hkv, N, scale, topk, heads, blk_idx, blk_cnt, ws, st);
    return launch_bs_d<64>(q, k, Hq, Hkv, N, scale, topk, heads, blk_idx, blk_cnt, ws, st);
}

}  // namespace minfer

// internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/minfer.h"

namespace minfer {

using bf16 = __nv_bfloat16;

// Query heads of one launch, in list order.  Each entry packs
// qh (bits 0-11), pattern (bits 12-13), the Vertical-Slash range flag (bit 14:
// slash diagonals as unaligned 64-key ranges instead of 64x64 tiles) and the
// head's position in the per-pattern index arrays (bits 16-31).
struct HeadList {
    int n;
    uint32_t e[MI_MAX_HEADS];
};

__host__ __device__ inline uint32_t pack_head(int qh, int pattern, int pidx) {
    return (uint32_t)qh | ((uint32_t)pattern << 12) | ((uint32_t)pidx << 16);
}
__host__ __device__ inline int head_qh(uint32_t e) { return (int)(e & 0xFFFu); }
__host__ __device__ inline int head_pattern(uint32_t e) { return (int)((e >> 12) & 0x3u); }
__host__ __device__ inline bool head_ranges(uint32_t e) { return ((e >> 14) & 1u) != 0; }
__host__ __device__ inline uint32_t with_ranges(uint32_t e, bool on) {
    return on ? (e | (1u << 14)) : (e & ~(1u << 14));
}
__host__ __device__ inline int head_pidx(uint32_t e) { return (int)(e >> 16); }
// grouped-query attention, contiguous groups
__host__ __device__ inline int kv_head_of(int qh, int Hq, int Hkv) {
    return (int)(((long long)qh * Hkv) / Hq);
}

// One count per row of a batched top-k (per-head budgets); rows past `n` and
// a null list fall back to the launch's single budget.
struct RowCounts {
    int n;
    int32_t k[MI_MAX_HEADS];
};

// Bump allocator over the caller's workspace.  With base == nullptr it only
// measures, so size queries and launches carve identically.
struct WsCarver {
    char* base;
    size_t off = 0;
    explicit WsCarver(void* b) : base(static_cast<char*>(b)) {}
    template <class T>
    T* take(size_t count) {
        off = (off + 255) & ~size_t(255);
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
    size_t bytes() const { return (off + 255) & ~size_t(255); }
};

// ----------------------------------------------------------- VS index
struct VsIndexWs {
    double* m_part;  // [n_heads][L][ceil(N / kVsTcChunk)]
    double* l_part;
    double* mrow;    // [n_heads][L] merged row max
    double* linv;    // [n_heads][L] 1 / merged row sum
    float* vscore;   // [n_heads][N]
    float* sscore;   // [n_heads][N]
    float* vpart;    // [n_heads][ceil(L / 64)][N] partial scores (L > 64 only, else null)
    float* spart;
};
VsIndexWs carve_vs_index(WsCarver& c, int n_heads, int N, int L, bool need_vscore,
                         bool need_sscore);
// kv / ks: budgets and index row strides; kv_rows / ks_rows (optional, host,
// one per listed head, each <= kv / ks): per-head budgets, -1 past them.
cudaError_t launch_vs_index(const bf16* q, const bf16* k, int Hq, int Hkv, int N, int d,
                            double scale, int L, int kv, int ks, const HeadList& heads,
                            int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score,
                            const VsIndexWs& ws, cudaStream_t st,
                            const int32_t* kv_rows = nullptr, const int32_t* ks_rows = nullptr);

// The two score passes on the tensor cores (vs_score_tc.cu), any L <= 1024.
// Pass 1 writes ws.m_part / ws.l_part for chunks of kVsTcChunk keys (merge
// them with nchunks = ceil(N / kVsTcChunk)); pass 2 reads ws.mrow / ws.linv
// and writes every entry of vscore / sscore [n_heads][N] (through
// ws.vpart / ws.spart when L > 64).
constexpr int kVsTcChunk = 2048;
cudaError_t launch_vs_scores_tc(int pass, const bf16* q, const bf16* k, int Hq, int Hkv, int N,
                                int d, double scale, int L, const HeadList& heads,
                                const VsIndexWs& ws, float* vscore, float* sscore,
                                cudaStream_t st);
cudaError_t read_vs_wait_failure(int* out8);

// ----------------------------------------------------------- BS index
struct BsIndexWs {
    double* qm;  // [n_heads][nB][d] block means
    double* km;  // [Hkv][nB][d]
};
BsIndexWs carve_bs_index(WsCarver& c, int n_heads, int Hkv, int N, int d);
// topk: budget and index row stride; topk_rows (optional, host, one per listed
// head, each <= topk): per-head budgets.
cudaError_t launch_bs_index(const bf16* q, const bf16* k, int Hq, int Hkv, int N, int d,
                            double scale, int topk, const HeadList& heads, int32_t* blk_idx,
                            int32_t* blk_cnt, const BsIndexWs& ws, cudaStream_t st,
                            const int32_t* topk_rows = nullptr);

// ----------------------------------------------------------- attention
struct VsPrepWs {
    uint32_t* dbits;    // [n_heads][nBw]   slash diagonals -> block-diagonal set
    uint32_t* colbits;  // [n_heads][N/32]  vertical columns as a bitmap
    uint32_t* sbits;    // [n_heads][N/32]  slash offsets as a bitmap
    uint64_t* rwords;   // [n_heads][nB]    range words (see vs_prep_kernel)
    int32_t* vlist;     // [n_heads][vcap]  sorted unique columns
    int32_t* vcnt;      // [n_heads]
    int vcap;
};
VsPrepWs carve_vs_prep(WsCarver& c, int n_heads, int N, int kv);
// ranges: also build the range words (needed by heads whose slash diagonals
// select unaligned 64-key ranges)
cudaError_t launch_vs_prep(const int32_t* v_idx, int kv_stride, int kv, const int32_t* s_idx,
                           int ks_stride, int ks, int N, int n_heads, const VsPrepWs& ws,
                           int32_t* err_count, cudaStream_t st, bool ranges = false);

struct AttnLaunch {
    const bf16 *q, *k, *v;
    bf16* out;
    float* lse;
    int Hq, Hkv, N, d;
    double scale;
    HeadList heads;  // pattern + per-pattern position per entry
    // Vertical-Slash (rwords: range words, read by heads with the range flag)
    const uint32_t* dbits;
    const uint64_t* rwords;
    const int32_t* vlist;
    const int32_t* vcnt;
    int vcap;
    // Block-Sparse
    const int32_t* blk_idx;
    const int32_t* blk_cnt;
    int topk;
    // A-shape (sink_h / window_h, optional host arrays indexed by the head's
    // A-shape position, override sink / window per head)
    int sink, window;
    const int32_t* sink_h;
    const int32_t* window_h;
    int n_asw;  // entries in sink_h / window_h
    int32_t* err_count;
};
cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t st);
// Block-Sparse heads on key-major tiles (attn_kt.cu): d = 128 and N up to
// about 8M (its per-item block bitmap lives in shared memory).
bool kt_attn_supported(const AttnLaunch& a);
cudaError_t launch_kt_attn(const AttnLaunch& a, cudaStream_t st);
cudaError_t read_kt_wait_failure(int* out8);
// 2-D TMA map over a [rows][d] bf16 matrix: boxes of 64 columns x box_rows
// rows, 128-byte swizzle, zero fill past the last row.
bool make_tma_map(CUtensorMap* m, const void* base, long long rows, int d, int box_rows);
cudaError_t read_wait_failure(int* out8);

// MI_OK, or MI_ERR_CUDA with the error kept for mi_last_cuda_error().
int cuda_status(cudaError_t e);

// Clock budget of the abortable in-pipeline waits of the kernels launched from
// now on (mi_debug_set_wait_budget; default kWaitBudgetCycles of ptx.cuh);
// teardown waits always keep the full bound.
long long wait_budget_cycles();
void set_wait_budget_cycles(long long cycles);

}  // namespace minfer

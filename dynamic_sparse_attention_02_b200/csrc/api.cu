// api.cu -- the C ABI declared in include/minfer.h: argument validation on
// the host (nothing is launched when a check fails), workspace carving, and
// the per-head pattern dispatcher of mi_prefill_layer (aifetchly guide,
// "Phase 2: The Online Dynamic Kernel Router": each head goes to the kernel
// of its offline-assigned pattern, with no host-device synchronisation).
#include <atomic>
#include <cmath>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

using namespace minfer;

namespace {
thread_local int g_last_cuda_error = 0;
std::atomic<long long> g_wait_budget{0};  // 0: the default bound
std::atomic<int> g_bs_engine{MI_BS_ENGINE_ROW};
}  // namespace

long long minfer::wait_budget_cycles() {
    const long long b = g_wait_budget.load();
    return b > 0 ? b : kWaitBudgetCycles;
}
void minfer::set_wait_budget_cycles(long long cycles) { g_wait_budget.store(cycles > 0 ? cycles : 0); }

// MI_OK, or MI_ERR_CUDA with the error kept for mi_last_cuda_error().
int minfer::cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MI_OK;
    g_last_cuda_error = (int)e;
    return MI_ERR_CUDA;
}

namespace {

// Block-Sparse heads go to the key-major engine only when it is selected and
// serves the launch's shapes.
bool use_key_major(const AttnLaunch& a) {
    return g_bs_engine.load() == MI_BS_ENGINE_KEY && kt_attn_supported(a);
}

// Shapes every entry point shares.  Fills `hl` with the listed heads
// (pattern and per-pattern position filled by the caller).
int check_shapes(const void* q, const void* k, int Hq, int Hkv, int N, int d,
                 const int32_t* heads, int n_heads, HeadList& hl) {
    if (!q || !k) return MI_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || n_heads < 0) return MI_ERR_INVALID_ARG;
    if (Hq % Hkv) return MI_ERR_INVALID_ARG;
    if (Hq > MI_MAX_HEADS) return MI_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return MI_ERR_UNSUPPORTED;
    if (N % MI_BLOCK) return MI_ERR_UNSUPPORTED;
    if ((long long)Hq * N >= (1LL << 31) || N > (1 << 24)) return MI_ERR_UNSUPPORTED;
    hl.n = 0;
    if (!heads) {
        for (int h = 0; h < Hq; ++h) hl.e[hl.n++] = pack_head(h, 0, h);
        return MI_OK;
    }
    if (n_heads > Hq) return MI_ERR_INVALID_ARG;
    bool seen[MI_MAX_HEADS] = {};
    for (int i = 0; i < n_heads; ++i) {
        const int h = heads[i];
        if (h < 0 || h >= Hq || seen[h]) return MI_ERR_INVALID_ARG;
        seen[h] = true;
        hl.e[hl.n++] = pack_head(h, 0, i);
    }
    return MI_OK;
}

void set_pattern(HeadList& hl, int pattern) {
    for (int i = 0; i < hl.n; ++i) hl.e[i] = pack_head(head_qh(hl.e[i]), pattern, i);
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (need == 0) return MI_OK;
    if (!ws || ws_bytes < need) return MI_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return MI_ERR_WORKSPACE;
    return MI_OK;
}

double eff_scale(float scale, int d) {
    return scale > 0.f ? (double)scale : 1.0 / std::sqrt((double)d);
}

int check_vs_params(int N, int last_q, int vertical_size, int slash_size) {
    if (last_q <= 0 || vertical_size < 0 || slash_size < 0) return MI_ERR_INVALID_ARG;
    if (last_q > N || last_q > 1024) return MI_ERR_UNSUPPORTED;
    return MI_OK;
}

size_t vs_index_bytes(int n, int N, int L) {
    WsCarver c(nullptr);
    carve_vs_index(c, n, N, L, true, true);
    return c.bytes();
}
size_t bs_index_bytes(int n, int Hkv, int N, int d) {
    WsCarver c(nullptr);
    carve_bs_index(c, n, Hkv, N, d);
    return c.bytes();
}
size_t vs_prep_bytes(int n, int N, int kv) {
    WsCarver c(nullptr);
    carve_vs_prep(c, n, N, kv);
    return c.bytes();
}

// Layer workspace: the VS and BS index outputs, then the scratch of each stage.
struct LayerWs {
    int32_t *v_idx, *s_idx, *blk_idx, *blk_cnt;
    VsIndexWs vsi;
    BsIndexWs bsi;
    VsPrepWs prep;
};
LayerWs carve_layer(WsCarver& c, int nvs, int nbs, int Hkv, int N, int d, const mi_params& p) {
    LayerWs w{};
    const int nB = N / MI_BLOCK;
    w.v_idx = c.take<int32_t>((size_t)nvs * p.vertical_size);
    w.s_idx = c.take<int32_t>((size_t)nvs * p.slash_size);
    w.blk_idx = c.take<int32_t>((size_t)nbs * nB * p.topk_blocks);
    w.blk_cnt = c.take<int32_t>((size_t)nbs * nB);
    if (nvs) w.vsi = carve_vs_index(c, nvs, N, p.last_q, true, true);
    if (nbs) w.bsi = carve_bs_index(c, nbs, Hkv, N, d);
    if (nvs) w.prep = carve_vs_prep(c, nvs, N, p.vertical_size);
    return w;
}

}  // namespace

extern "C" {

const char* mi_status_str(int status) {
    switch (status) {
        case MI_OK: return "ok";
        case MI_ERR_INVALID_ARG: return "invalid argument";
        case MI_ERR_UNSUPPORTED: return "unsupported shape or parameter";
        case MI_ERR_WORKSPACE: return "workspace too small or misaligned";
        case MI_ERR_CUDA: return "CUDA error (see mi_last_cuda_error)";
        default: return "unknown status";
    }
}

int mi_last_cuda_error(void) { return g_last_cuda_error; }

const char* mi_version(void) { return "minfer 0.1 sm_100a"; }

size_t mi_workspace_bytes(int op, int Hq, int Hkv, int N, int d, int n_heads, int last_q,
                          int vertical_size, int slash_size, int topk_blocks) {
    (void)topk_blocks;
    if (Hq <= 0 || Hkv <= 0 || N <= 0 || N % MI_BLOCK || (d != 64 && d != 128)) return 0;
    const int n = n_heads > 0 ? n_heads : Hq;
    switch (op) {
        case MI_OP_VS_INDEX:
            if (last_q <= 0 || last_q > N) return 0;
            return vs_index_bytes(n, N, last_q);
        case MI_OP_BS_INDEX: return bs_index_bytes(n, Hkv, N, d);
        case MI_OP_VS_ATTN: return vs_prep_bytes(n, N, vertical_size > 0 ? vertical_size : 1);
        case MI_OP_BS_ATTN:
        case MI_OP_ASHAPE_ATTN:
        case MI_OP_DENSE_ATTN: return 256;
        default: return 0;
    }
    (void)slash_size;
}

size_t mi_prefill_workspace_bytes(int Hq, int Hkv, int N, int d, const int8_t* pattern,
                                  const mi_params* p) {
    if (!p || Hq <= 0 || Hkv <= 0 || N <= 0 || N % MI_BLOCK || (d != 64 && d != 128)) return 0;
    int nvs = 0, nbs = 0;
    for (int h = 0; h < Hq; ++h) {
        const int pt = pattern ? pattern[h] : -1;
        if (pt == MI_PATTERN_VS || pt < 0) ++nvs;
        if (pt == MI_PATTERN_BS || pt < 0) ++nbs;
    }
    WsCarver c(nullptr);
    carve_layer(c, nvs, nbs, Hkv, N, d, *p);
    return c.bytes();
}

int mi_vs_index(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N, int d, float scale,
                int last_q, int vertical_size, int slash_size, const int32_t* heads, int n_heads,
                int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score, void* ws,
                size_t ws_bytes, void* stream) {
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if ((rc = check_vs_params(N, last_q, vertical_size, slash_size))) return rc;
    if ((vertical_size > 0 && !v_idx) || (slash_size > 0 && !s_idx)) return MI_ERR_INVALID_ARG;
    const size_t need = vs_index_bytes(hl.n, N, last_q);
    if ((rc = check_ws(ws, ws_bytes, need))) return rc;
    if (hl.n == 0) return MI_OK;
    WsCarver c(ws);
    VsIndexWs w = carve_vs_index(c, hl.n, N, last_q, true, true);
    set_pattern(hl, MI_PATTERN_VS);
    return cuda_status(launch_vs_index(reinterpret_cast<const bf16*>(q),
                                       reinterpret_cast<const bf16*>(k), Hq, Hkv, N, d,
                                       eff_scale(scale, d), last_q, vertical_size, slash_size, hl,
                                       v_idx, s_idx, v_score, s_score, w,
                                       static_cast<cudaStream_t>(stream)));
}

int mi_bs_index(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N, int d, float scale,
                int block, int topk, const int32_t* heads, int n_heads, int32_t* blk_idx,
                int32_t* blk_cnt, void* ws, size_t ws_bytes, void* stream) {
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if (block != MI_BLOCK) return MI_ERR_UNSUPPORTED;
    if (topk < 0) return MI_ERR_INVALID_ARG;
    if (!blk_cnt || (topk > 0 && !blk_idx)) return MI_ERR_INVALID_ARG;
    const size_t need = bs_index_bytes(hl.n, Hkv, N, d);
    if ((rc = check_ws(ws, ws_bytes, need))) return rc;
    if (hl.n == 0) return MI_OK;
    WsCarver c(ws);
    BsIndexWs w = carve_bs_index(c, hl.n, Hkv, N, d);
    set_pattern(hl, MI_PATTERN_BS);
    return cuda_status(launch_bs_index(reinterpret_cast<const bf16*>(q),
                                       reinterpret_cast<const bf16*>(k), Hq, Hkv, N, d,
                                       eff_scale(scale, d), topk, hl, blk_idx, blk_cnt, w,
                                       static_cast<cudaStream_t>(stream)));
}

static void attn_common(AttnLaunch& a, const mi_bf16* q, const mi_bf16* k, const mi_bf16* v,
                        int Hq, int Hkv, int N, int d, float scale, mi_bf16* out, float* lse,
                        int32_t* err_count) {
    memset(&a, 0, sizeof(a));
    a.q = reinterpret_cast<const bf16*>(q);
    a.k = reinterpret_cast<const bf16*>(k);
    a.v = reinterpret_cast<const bf16*>(v);
    a.out = reinterpret_cast<bf16*>(out);
    a.lse = lse;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.N = N;
    a.d = d;
    a.scale = eff_scale(scale, d);
    a.err_count = err_count;
}

}  // extern "C"

namespace {

// Vertical-Slash attention with the diagonals read as 64x64 tiles or, with
// `ranges`, as unaligned 64-key ranges.
int vs_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N, int d,
            float scale, const int32_t* v_idx, int vertical_size, const int32_t* s_idx,
            int slash_size, const int32_t* heads, int n_heads, mi_bf16* out, float* lse,
            int32_t* err_count, void* ws, size_t ws_bytes, void* stream, bool ranges) {
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if (!v || !out || vertical_size < 0 || slash_size < 0) return MI_ERR_INVALID_ARG;
    if ((vertical_size > 0 && !v_idx) || (slash_size > 0 && !s_idx)) return MI_ERR_INVALID_ARG;
    const int kv = vertical_size > 0 ? vertical_size : 1;
    const size_t need = vs_prep_bytes(hl.n, N, kv);
    if ((rc = check_ws(ws, ws_bytes, need))) return rc;
    if (hl.n == 0) return MI_OK;
    WsCarver c(ws);
    VsPrepWs prep = carve_vs_prep(c, hl.n, N, kv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = cuda_status(launch_vs_prep(v_idx, vertical_size, vertical_size, s_idx, slash_size,
                                    slash_size, N, hl.n, prep, err_count, st, ranges));
    if (rc) return rc;
    AttnLaunch a;
    attn_common(a, q, k, v, Hq, Hkv, N, d, scale, out, lse, err_count);
    set_pattern(hl, MI_PATTERN_VS);
    for (int i = 0; i < hl.n; ++i) hl.e[i] = with_ranges(hl.e[i], ranges);
    a.heads = hl;
    a.dbits = prep.dbits;
    a.rwords = prep.rwords;
    a.vlist = prep.vlist;
    a.vcnt = prep.vcnt;
    a.vcap = prep.vcap;
    return cuda_status(launch_sparse_attn(a, st));
}

}  // namespace

extern "C" {

int mi_vs_sparse_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                      int N, int d, float scale, const int32_t* v_idx, int vertical_size,
                      const int32_t* s_idx, int slash_size, const int32_t* heads, int n_heads,
                      mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                      void* stream) {
    return vs_attn(q, k, v, Hq, Hkv, N, d, scale, v_idx, vertical_size, s_idx, slash_size, heads,
                   n_heads, out, lse, err_count, ws, ws_bytes, stream, false);
}

int mi_vs_range_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                     int N, int d, float scale, const int32_t* v_idx, int vertical_size,
                     const int32_t* s_idx, int slash_size, const int32_t* heads, int n_heads,
                     mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                     void* stream) {
    return vs_attn(q, k, v, Hq, Hkv, N, d, scale, v_idx, vertical_size, s_idx, slash_size, heads,
                   n_heads, out, lse, err_count, ws, ws_bytes, stream, true);
}

int mi_block_sparse_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                         int N, int d, float scale, const int32_t* blk_idx,
                         const int32_t* blk_cnt, int topk, int block, const int32_t* heads,
                         int n_heads, mi_bf16* out, float* lse, int32_t* err_count, void* ws,
                         size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if (block != MI_BLOCK) return MI_ERR_UNSUPPORTED;
    if (!v || !out || topk < 0 || !blk_cnt || (topk > 0 && !blk_idx)) return MI_ERR_INVALID_ARG;
    if (hl.n == 0) return MI_OK;
    AttnLaunch a;
    attn_common(a, q, k, v, Hq, Hkv, N, d, scale, out, lse, err_count);
    set_pattern(hl, MI_PATTERN_BS);
    a.heads = hl;
    a.blk_idx = blk_idx;
    a.blk_cnt = blk_cnt;
    a.topk = topk;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return cuda_status(use_key_major(a) ? launch_kt_attn(a, st) : launch_sparse_attn(a, st));
}

int mi_ashape_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N,
                   int d, float scale, int sink, int window, const int32_t* heads, int n_heads,
                   mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                   void* stream) {
    (void)ws;
    (void)ws_bytes;
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if (!v || !out || sink < 0 || window < 1) return MI_ERR_INVALID_ARG;
    if (hl.n == 0) return MI_OK;
    AttnLaunch a;
    attn_common(a, q, k, v, Hq, Hkv, N, d, scale, out, lse, err_count);
    set_pattern(hl, MI_PATTERN_ASHAPE);
    a.heads = hl;
    a.sink = sink;
    a.window = window;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

int mi_dense_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N,
                  int d, float scale, const int32_t* heads, int n_heads, mi_bf16* out,
                  float* lse, int32_t* err_count, void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    HeadList hl;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, heads, n_heads, hl);
    if (rc) return rc;
    if (!v || !out) return MI_ERR_INVALID_ARG;
    if (hl.n == 0) return MI_OK;
    AttnLaunch a;
    attn_common(a, q, k, v, Hq, Hkv, N, d, scale, out, lse, err_count);
    set_pattern(hl, MI_PATTERN_DENSE);
    a.heads = hl;
    return cuda_status(launch_sparse_attn(a, static_cast<cudaStream_t>(stream)));
}

namespace {

// One layer with either one parameter set for every head (per_head = false)
// or one per head.  VS heads must share last_q (the score passes take one row
// count); budgets, block counts, sink and window may differ per head.
struct LayerPlan {
    HeadList all, vs, bs;
    int n_a = 0;
    bool any_ranges = false;  // some VS head reads its diagonals as ranges
    mi_params pp{};  // layer-wide maxima: buffer sizes and index row strides
    int32_t kv_h[MI_MAX_HEADS], ks_h[MI_MAX_HEADS], tk_h[MI_MAX_HEADS];
    int32_t sink_h[MI_MAX_HEADS], win_h[MI_MAX_HEADS];
};

int plan_layer(int Hq, int N, const int8_t* pattern, const mi_params* params, bool per_head,
               LayerPlan& lp) {
    lp.vs.n = lp.bs.n = 0;
    lp.n_a = 0;
    lp.any_ranges = false;
    int L = -1, kv_max = 0, ks_max = 0, tk_max = 0;
    for (int h = 0; h < Hq; ++h) {
        const mi_params& ph = params[per_head ? h : 0];
        switch (pattern[h]) {
            case MI_PATTERN_ASHAPE:
                if (ph.sink < 0 || ph.window < 1) return MI_ERR_INVALID_ARG;
                lp.sink_h[lp.n_a] = ph.sink;
                lp.win_h[lp.n_a] = ph.window;
                lp.all.e[h] = pack_head(h, MI_PATTERN_ASHAPE, lp.n_a++);
                break;
            case MI_PATTERN_DENSE: lp.all.e[h] = pack_head(h, MI_PATTERN_DENSE, 0); break;
            case MI_PATTERN_VS: {
                if (L >= 0 && ph.last_q != L) return MI_ERR_INVALID_ARG;
                L = ph.last_q;
                const int rc = check_vs_params(N, ph.last_q, ph.vertical_size, ph.slash_size);
                if (rc) return rc;
                const int kv = ph.vertical_size < N ? ph.vertical_size : N;
                const int ks = ph.slash_size < N ? ph.slash_size : N;
                lp.kv_h[lp.vs.n] = kv;
                lp.ks_h[lp.vs.n] = ks;
                kv_max = kv > kv_max ? kv : kv_max;
                ks_max = ks > ks_max ? ks : ks_max;
                if (ph.slash_tiles != MI_SLASH_BLOCKS && ph.slash_tiles != MI_SLASH_RANGES)
                    return MI_ERR_INVALID_ARG;
                const bool rg = ph.slash_tiles == MI_SLASH_RANGES;
                lp.any_ranges |= rg;
                lp.all.e[h] = with_ranges(pack_head(h, MI_PATTERN_VS, lp.vs.n), rg);
                lp.vs.e[lp.vs.n] = pack_head(h, MI_PATTERN_VS, lp.vs.n);
                ++lp.vs.n;
                break;
            }
            case MI_PATTERN_BS: {
                if (ph.topk_blocks < 0) return MI_ERR_INVALID_ARG;
                const int nB = N / MI_BLOCK;
                const int tk = ph.topk_blocks < nB ? ph.topk_blocks : nB;
                lp.tk_h[lp.bs.n] = tk;
                tk_max = tk > tk_max ? tk : tk_max;
                lp.all.e[h] = pack_head(h, MI_PATTERN_BS, lp.bs.n);
                lp.bs.e[lp.bs.n] = pack_head(h, MI_PATTERN_BS, lp.bs.n);
                ++lp.bs.n;
                break;
            }
            default: return MI_ERR_INVALID_ARG;
        }
    }
    lp.pp = params[0];
    lp.pp.last_q = L > 0 ? L : params[0].last_q;
    lp.pp.vertical_size = lp.vs.n ? (kv_max > 0 ? kv_max : 1) : 0;  // carved buffers non-empty
    lp.pp.slash_size = lp.vs.n ? ks_max : 0;
    lp.pp.topk_blocks = lp.bs.n ? tk_max : 0;
    return MI_OK;
}

int prefill_layer(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N,
                  int d, float scale, const int8_t* pattern, const mi_params* params,
                  bool per_head, mi_bf16* out, float* lse, int32_t* err_count, void* ws,
                  size_t ws_bytes, void* stream, void* const* stage_events) {
    LayerPlan lp;
    int rc = check_shapes(q, k, Hq, Hkv, N, d, nullptr, 0, lp.all);
    if (rc) return rc;
    if (!v || !out || !pattern || !params) return MI_ERR_INVALID_ARG;
    if ((rc = plan_layer(Hq, N, pattern, params, per_head, lp))) return rc;
    const mi_params& pp = lp.pp;
    WsCarver sizer(nullptr);
    carve_layer(sizer, lp.vs.n, lp.bs.n, Hkv, N, d, pp);
    if ((rc = check_ws(ws, ws_bytes, sizer.bytes()))) return rc;

    WsCarver c(ws);
    LayerWs w = carve_layer(c, lp.vs.n, lp.bs.n, Hkv, N, d, pp);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const double sc = eff_scale(scale, d);
    auto rec = [&](int i) -> int {
        if (!stage_events || !stage_events[i]) return MI_OK;
        return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), st));
    };
    if ((rc = rec(MI_STAGE_START))) return rc;
    const bf16* qb = reinterpret_cast<const bf16*>(q);
    const bf16* kb = reinterpret_cast<const bf16*>(k);
    if (lp.vs.n) {
        rc = cuda_status(launch_vs_index(qb, kb, Hq, Hkv, N, d, sc, pp.last_q, pp.vertical_size,
                                         pp.slash_size, lp.vs, w.v_idx, w.s_idx, nullptr,
                                         nullptr, w.vsi, st, per_head ? lp.kv_h : nullptr,
                                         per_head ? lp.ks_h : nullptr));
        if (rc) return rc;
    }
    if (lp.bs.n) {
        rc = cuda_status(launch_bs_index(qb, kb, Hq, Hkv, N, d, sc, pp.topk_blocks, lp.bs,
                                         w.blk_idx, w.blk_cnt, w.bsi, st,
                                         per_head ? lp.tk_h : nullptr));
        if (rc) return rc;
    }
    if ((rc = rec(MI_STAGE_INDEX_DONE))) return rc;
    if (lp.vs.n) {
        rc = cuda_status(launch_vs_prep(w.v_idx, pp.vertical_size, pp.vertical_size, w.s_idx,
                                        pp.slash_size, pp.slash_size, N, lp.vs.n, w.prep,
                                        err_count, st, lp.any_ranges));
        if (rc) return rc;
    }
    if ((rc = rec(MI_STAGE_PREP_DONE))) return rc;
    AttnLaunch a;
    attn_common(a, q, k, v, Hq, Hkv, N, d, scale, out, lse, err_count);
    a.heads = lp.all;
    a.dbits = w.prep.dbits;
    a.rwords = w.prep.rwords;
    a.vlist = w.prep.vlist;
    a.vcnt = w.prep.vcnt;
    a.vcap = w.prep.vcap;
    a.blk_idx = w.blk_idx;
    a.blk_cnt = w.blk_cnt;
    a.topk = pp.topk_blocks;
    a.sink = pp.sink;
    a.window = pp.window;
    a.sink_h = lp.sink_h;
    a.window_h = lp.win_h;
    a.n_asw = lp.n_a;
    // With the key-major engine selected, Block-Sparse heads run on it where
    // it applies; the rest (all heads otherwise) in one row-major launch
    if (lp.bs.n && use_key_major(a)) {
        AttnLaunch abs = a;
        abs.heads.n = 0;
        a.heads.n = 0;
        for (int i = 0; i < lp.all.n; ++i) {
            HeadList& dst = head_pattern(lp.all.e[i]) == MI_PATTERN_BS ? abs.heads : a.heads;
            dst.e[dst.n++] = lp.all.e[i];
        }
        if ((rc = cuda_status(launch_kt_attn(abs, st)))) return rc;
    }
    if ((rc = cuda_status(launch_sparse_attn(a, st)))) return rc;
    return rec(MI_STAGE_ATTN_DONE);
}

}  // namespace

int mi_prefill_layer(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                     int N, int d, float scale, const int8_t* pattern, const mi_params* p,
                     mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                     void* stream, void* const* stage_events) {
    return prefill_layer(q, k, v, Hq, Hkv, N, d, scale, pattern, p, false, out, lse, err_count,
                         ws, ws_bytes, stream, stage_events);
}

size_t mi_prefill_workspace_bytes_heads(int Hq, int Hkv, int N, int d, const int8_t* pattern,
                                        const mi_params* params) {
    if (!pattern || !params || Hq <= 0 || Hq > MI_MAX_HEADS || Hkv <= 0 || N <= 0 ||
        N % MI_BLOCK || (d != 64 && d != 128))
        return 0;
    LayerPlan lp;
    if (plan_layer(Hq, N, pattern, params, true, lp) != MI_OK) return 0;
    WsCarver c(nullptr);
    carve_layer(c, lp.vs.n, lp.bs.n, Hkv, N, d, lp.pp);
    return c.bytes();
}

int mi_prefill_layer_heads(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq,
                           int Hkv, int N, int d, float scale, const int8_t* pattern,
                           const mi_params* params, mi_bf16* out, float* lse,
                           int32_t* err_count, void* ws, size_t ws_bytes, void* stream,
                           void* const* stage_events) {
    return prefill_layer(q, k, v, Hq, Hkv, N, d, scale, pattern, params, true, out, lse,
                         err_count, ws, ws_bytes, stream, stage_events);
}

int mi_set_bs_engine(int engine) {
    if (engine != MI_BS_ENGINE_ROW && engine != MI_BS_ENGINE_KEY) return MI_ERR_INVALID_ARG;
    g_bs_engine.store(engine);
    return MI_OK;
}

int mi_debug_set_wait_budget(long long cycles) {
    set_wait_budget_cycles(cycles);
    return MI_OK;
}

int mi_debug_wait_failure(int32_t* record8) {
    if (!record8) return MI_ERR_INVALID_ARG;
    // the row-major attention record first, then the key-major attention one
    // (sites 21..27), else the tensor-core VS score passes' (sites 11..15);
    // reading clears all three
    int rec[8], rec_kt[8], rec_vs[8];
    int rc = cuda_status(read_wait_failure(rec));
    if (rc) return rc;
    rc = cuda_status(read_kt_wait_failure(rec_kt));
    if (rc) return rc;
    rc = cuda_status(read_vs_wait_failure(rec_vs));
    if (rc) return rc;
    const int* use = rec[1] != 0 ? rec : (rec_kt[1] != 0 ? rec_kt : rec_vs);
    for (int i = 0; i < 8; ++i) record8[i] = use[i];
    return MI_OK;
}

}  // extern "C"

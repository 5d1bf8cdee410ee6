// vs_score_tc.cu -- the Vertical-Slash score passes on the tensor cores.
//
// MInference 1.0 (hotpaper.ai summary, "key idea"; guide "2. The
// Vertical-Slash Pattern"): the last L queries of a head score every key
// column and every diagonal through their causal row softmax.  The products
// q_i . k_j form a dense contraction, so here they run on tcgen05.  The L rows
// of a head split into 64-row groups counted from the end (the first group
// padded when 64 does not divide L); one M=128 tile stacks two such groups of
// query heads that share a KV head (rows 0-63 the first, 64-127 the second),
// and every 128-key tile of K gives S = Q K^T in TMEM (exact bf16 products,
// fp32 accumulation).
//
//   pass 1: per row, the online max and sum of exp over a 2048-key chunk
//           (exponentials in fp32, the running sum in fp64).  The partials go
//           to the workspace and are merged by vs_rowmerge into each row's
//           max m_i and 1 / l_i.
//   pass 2: p_ij = exp(s_ij - m_i) / l_i with the exponent carried as an
//           unevaluated pair of fp32 values (exp2 of the leading part times a
//           first-order correction for the rest), staged in shared memory as
//           fp32 and summed per column and per diagonal with compensated
//           (Kahan) fp32 sums in a fixed order.  A chunk owns the
//           columns it holds and the diagonals whose first key it holds, and
//           reads one more key tile to finish those diagonals.  With one row
//           group per head (L <= 64) these are the scores; otherwise each
//           group's sums are partials, added per head in group order.
//
// Warp roles: warp 0 loads Q and K tiles by TMA, warp 1 issues the MMAs,
// warps 2.. are the epilogue (8 in pass 1, 16 in pass 2).  TMEM lanes are
// rows: warp w reads lane quadrant w % 4, and the epilogue warps of one
// quadrant split the tile's 128 key columns between them.  Two 128-column
// accumulators let the tensor core fill one while the epilogue drains the
// other.
#include <atomic>
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace minfer {

namespace {

constexpr int kTcKeys = 128;     // keys per tile (MMA N)
constexpr int kTcStages = 2;     // K tiles in flight
constexpr int kEpiWarp0 = 2;     // first epilogue warp
// Staged probabilities are skewed: row r of a slot keeps key column c at
// position c - r + 63, so diagonal u = c - r is position u + 63 of every row.
// 192 words per row (191 used): row stride 192 - 1 = 191 is odd, so the
// 32 rows of a warp store one column to 32 distinct banks.
constexpr int kSkew = 192;
constexpr int kDiag = 191;       // diagonals a 64 x 128 tile touches: u = c - r in [-63, 127]
constexpr uint32_t kTcTmemCols = 256;
constexpr double kLog2e = 1.4426950408889634;
constexpr float kLn2f = 0.69314718055994531f;

// Sequence number of the last launch in which a CTA gave up waiting.
__device__ unsigned int g_vs_abort_seq = 0;
// First wait that gave up: {launch seq, site, block x, thread, tile, parity, block y, 0}.
__device__ int g_vs_wait_fail[8];

enum : int {
    kSiteTcProducer = 11,
    kSiteTcMmaQ = 12,
    kSiteTcMmaK = 13,
    kSiteTcMmaAcc = 14,
    kSiteTcEpilogue = 15
};

__device__ void record_vs_wait_failure(unsigned int seq, int site, int tile, int parity) {
    if (atomicCAS(&g_vs_wait_fail[1], 0, site) == 0) {
        g_vs_wait_fail[0] = (int)seq;
        g_vs_wait_fail[2] = (int)blockIdx.x;
        g_vs_wait_fail[3] = (int)threadIdx.x;
        g_vs_wait_fail[4] = tile;
        g_vs_wait_fail[5] = parity;
        g_vs_wait_fail[6] = (int)blockIdx.y;
        __threadfence();
    }
}

__device__ __forceinline__ void vs_set_abort(volatile int* abort, unsigned int seq) {
    *abort = 1;
    atomicExch(&g_vs_abort_seq, seq);
}

// Work items are 64-row groups of the listed heads' last L rows, counted from
// the end: item = position * G + g (G = ceil(L / 64)) covers the query rows
// N - 64 (g + 1) .. N - 64 g - 1, those before N - L being padding.  The
// items of one KV head are paired into M=128 tiles in order (an odd one out
// runs alone), tile by tile across the KV heads in use.
struct TcParams {
    HeadList heads;
    int16_t hpos[MI_MAX_HEADS];        // listed positions, grouped by KV head
    int16_t hstart[MI_MAX_HEADS + 1];  // per KV head in use: its first entry in hpos
    int tstart[MI_MAX_HEADS + 1];      // per KV head in use: its first tile
    int ngroups, G;
    int Hq, Hkv, N, L, nchunks, chunk;
    double scale;
    unsigned int seq;
    long long wait_budget;  // cycles an abortable wait may take before it gives up
    double* m_part;  // pass 1 out: [n_heads][L][nchunks]
    double* l_part;
    const double* mrow;  // pass 2 in: [n_heads][L]
    const double* linv;
    float* vout;  // pass 2 out: [items][N], the scores themselves when G == 1
    float* sout;  // (items == heads then), else per-item partial sums
};

// An item's head position, its rows' end e (exclusive), the first non-padding
// row rmin of its 64 and the index among the head's L rows of its row 0.
struct TcItem {
    int item, pos, e, rmin, rbase;
};
__device__ __forceinline__ TcItem tc_item(const TcParams& p, int item) {
    TcItem x;
    x.item = item;
    if (item < 0) {
        x.pos = -1;
        x.e = 0;
        x.rmin = 64;
        x.rbase = 0;
        return x;
    }
    const int g = item % p.G;
    x.pos = item / p.G;
    x.e = p.N - 64 * g;
    x.rbase = p.L - 64 * (g + 1);
    x.rmin = x.rbase < 0 ? -x.rbase : 0;
    return x;
}

// Epilogue width per pass: pass 1 runs two CTAs per SM with 8 epilogue warps
// (64 key columns each), pass 2 one CTA per SM with 16 (32 columns each), so
// that each SM sub-partition holds four epilogue warps in both.
template <int PASS>
struct TcShape {
    static constexpr int kEpiWarps = PASS == 1 ? 8 : 16;
    static constexpr int kEpiThreads = kEpiWarps * 32;
    static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
    static constexpr int kGroups = kEpiWarps / 4;   // column groups per lane quadrant
    static constexpr int kCols = kTcKeys / kGroups;  // key columns per epilogue warp
};

template <int D, int PASS>
struct TcLayout {
    static constexpr int kPanels = D / 64;
    static constexpr int kQPanel = 128 * 128;      // 128 rows x 128 bytes
    static constexpr int kKPanel = kTcKeys * 128;  // 128 keys x 128 bytes
    static constexpr int kKStage = kPanels * kKPanel;
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + kPanels * kQPanel;
    static constexpr int p_off = k_off + kTcStages * kKStage;
    static constexpr int p_bytes = PASS == 2 ? 2 * 64 * kSkew * 4 : 0;
    static constexpr int carry_off = p_off + p_bytes;  // [tile parity][slot][64] fp64
    static constexpr int red_off = carry_off + 2 * 2 * 64 * 8;  // [group][128] x (m, l) fp64
    static constexpr int bar_off = red_off + TcShape<PASS>::kGroups * 128 * 2 * 8;
    static constexpr int kBars = 1 + 2 * kTcStages + 4 + 1;
    static constexpr int misc_off = bar_off + kBars * 8;
    static constexpr int bytes = misc_off + 16 + 1024;  // + alignment slack
};

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int PASS>
__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(TcShape<PASS>::kEpiThreads) : "memory");
}

struct TcBars {
    uint64_t* q_full;
    uint64_t* k_full;  // [kTcStages]
    uint64_t* k_empty;
    uint64_t* acc_full;  // [2]
    uint64_t* acc_empty;
    uint64_t* drain;
};

// Warp 0, lane 0: Q of both slots once, then the K tiles [jb, jb + 128 t).
template <int D>
__device__ void tc_producer(const TcParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                            uint8_t* sm, const TcBars& bars, volatile int* abort, int g, int jb,
                            int ntiles, int it_a, int it_b) {
    using Lay = TcLayout<D, 1>;
    prefetch_tmap(tmQ);
    prefetch_tmap(tmK);
    const int nslots = it_b >= 0 ? 2 : 1;
    mbar_arrive_expect_tx(bars.q_full, (uint32_t)(nslots * Lay::kPanels * 64 * 128));
    for (int s = 0; s < nslots; ++s) {
        const TcItem x = tc_item(p, s ? it_b : it_a);
        const int qh = head_qh(p.heads.e[x.pos]);
        const int row = qh * p.N + x.e - 64;
        for (int pn = 0; pn < Lay::kPanels; ++pn)
            tma_load_2d(sm + Lay::q_off + pn * Lay::kQPanel + s * 64 * 128, tmQ, 64 * pn, row,
                        bars.q_full);
    }
    int issued = 0;
    for (int t = 0; t < ntiles; ++t) {
        const int st = t % kTcStages;
        if (t >= kTcStages) {
            const uint32_t par = ((t / kTcStages) - 1) & 1;
            if (!mbar_wait(&bars.k_empty[st], par, abort, p.wait_budget)) {
                if (!*abort) record_vs_wait_failure(p.seq, kSiteTcProducer, t, (int)par);
                vs_set_abort(abort, p.seq);
                break;
            }
        }
        mbar_arrive_expect_tx(&bars.k_full[st], (uint32_t)Lay::kKStage);
        for (int pn = 0; pn < Lay::kPanels; ++pn)
            tma_load_2d(sm + Lay::k_off + st * Lay::kKStage + pn * Lay::kKPanel, tmK, 64 * pn,
                        g * p.N + jb + t * kTcKeys, &bars.k_full[st]);
        issued = t + 1;
    }
    // no copy may still be in flight when the CTA exits
    mbar_wait_budget(bars.q_full, 0);
    for (int t = issued > kTcStages ? issued - kTcStages : 0; t < issued; ++t)
        mbar_wait_budget(&bars.k_full[t % kTcStages], (t / kTcStages) & 1);
}

// Warp 1: per tile, S[buffer t % 2] = Q K_t^T (D / 16 MMAs of 128 x 128 x 16).
template <int D>
__device__ void tc_mma(const TcParams& p, uint8_t* sm, const TcBars& bars, volatile int* abort,
                       uint32_t tmem, int ntiles) {
    using Lay = TcLayout<D, 1>;
    const int lane = threadIdx.x & 31;
    const uint32_t idesc = idesc_bf16_f32(128, kTcKeys, false);
    tmem = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t q_addr = __shfl_sync(0xffffffffu, smem_u32(sm + Lay::q_off), 0);
    const uint32_t k_addr = __shfl_sync(0xffffffffu, smem_u32(sm + Lay::k_off), 0);
    bool ok;
    {
        bool w = true;
        if (lane == 0) {
            w = mbar_wait(bars.q_full, 0, abort, p.wait_budget);
            if (!w && !*abort) record_vs_wait_failure(p.seq, kSiteTcMmaQ, 0, 0);
        }
        ok = __shfl_sync(0xffffffffu, w, 0);
    }
    for (int t = 0; ok && t < ntiles; ++t) {
        const int st = t % kTcStages, b = t & 1;
        bool w = true;
        if (lane == 0) {
            const uint32_t kpar = (t / kTcStages) & 1;
            w = mbar_wait(&bars.k_full[st], kpar, abort, p.wait_budget);
            if (!w && !*abort) record_vs_wait_failure(p.seq, kSiteTcMmaK, t, (int)kpar);
            if (w && t >= 2) {
                const uint32_t apar = ((t >> 1) - 1) & 1;
                w = mbar_wait(&bars.acc_empty[b], apar, abort, p.wait_budget);
                if (!w && !*abort) record_vs_wait_failure(p.seq, kSiteTcMmaAcc, t, (int)apar);
            }
        }
        ok = __shfl_sync(0xffffffffu, w, 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int pn = kk >> 2, off = (kk & 3) * 32;
            const uint64_t adesc = sw128_desc(q_addr + pn * Lay::kQPanel + off, 16, 1024);
            const uint64_t bdesc =
                sw128_desc(k_addr + st * Lay::kKStage + pn * Lay::kKPanel + off, 16, 1024);
            mma_ss_warp(tmem + 128 * b, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(&bars.acc_full[b]);
        mma_commit_warp(&bars.k_empty[st]);
    }
    if (!ok && lane == 0) vs_set_abort(abort, p.seq);
    // every MMA must have finished before TMEM is released
    mma_commit_warp(bars.drain);
    if (lane == 0) mbar_wait_budget(bars.drain, 0);
    __syncwarp();
}

// Epilogue warp: wait for accumulator b of tile t.  A wait that gives up
// marks the warp failed; a failed warp keeps taking the epilogue's named
// barriers (so that no other warp waits on it) but touches no data.
__device__ __forceinline__ bool epi_wait(const TcParams& p, const TcBars& bars,
                                         volatile int* abort, int t) {
    const int lane = threadIdx.x & 31;
    bool w = true;
    if (lane == 0) {
        const uint32_t par = (t >> 1) & 1;
        w = mbar_wait(&bars.acc_full[t & 1], par, abort, p.wait_budget);
        if (!w) {
            if (!*abort) record_vs_wait_failure(p.seq, kSiteTcEpilogue, t, (int)par);
            vs_set_abort(abort, p.seq);
        }
    }
    return __shfl_sync(0xffffffffu, w, 0);
}

__device__ __forceinline__ void epi_release(const TcBars& bars, int t) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.acc_empty[t & 1]);
}

// p = 2^(s c - m') for c = c_hi + c_lo and m' = m_hi + m_lo (prob2 below):
// the product's rounding error (FMA residual) and the subtraction's (TwoSum)
// are kept, and 2^x of the small remainder x is taken as 1 + x ln 2 around the
// MUFU exp2 of the rest.
// ---- packed pairs of fp32 (sm_100 f32x2 arithmetic: two IEEE round-to-
// nearest operations per instruction, the same results as two scalar ones)
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(a), "f"(b));
    return d;
}
__device__ __forceinline__ void upk2(uint64_t d, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(d));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// prob() for two scores at once; the constants come packed (both halves
// equal): nchi = -c_hi, chi = c_hi, mhi = m_hi, clo = c_lo, nmlo = -m_lo.
__device__ __forceinline__ uint64_t prob2(uint64_t s2, uint64_t nchi, uint64_t chi, uint64_t mhi,
                                          uint64_t clo, uint64_t nmlo, uint64_t ln2,
                                          uint64_t one) {
    const uint64_t np1 = mul2(s2, nchi);   // -p1, p1 = fl(s c_hi)
    const uint64_t e1 = fma2(s2, chi, np1);  // exact: s c_hi = p1 + e1
    const uint64_t ny = add2(np1, mhi);      // -y, y = fl(p1 - m_hi)
    const uint64_t bb = sub2(ny, np1);
    const uint64_t e2 = add2(sub2(np1, sub2(ny, bb)), sub2(mhi, bb));  // exact: -p1 + m_hi = -y + e2
    const uint64_t lo = add2(add2(e1, e2), fma2(s2, clo, nmlo));       // s c - m' = y + lo
    float y0, y1;
    upk2(ny, y0, y1);
    const uint64_t ex = pk2(ex2_approx(-y0), ex2_approx(-y1));
    return mul2(ex, fma2(lo, ln2, one));
}

// Two compensated fp32 sums of non-negative terms side by side (error about
// one rounding of each result, whatever the count).
struct KahanSum2 {
    uint64_t s = 0, c = 0;
    __device__ __forceinline__ void add(uint64_t x) {
        const uint64_t y = sub2(x, c);
        const uint64_t t = add2(s, y);
        c = sub2(sub2(t, s), y);
        s = t;
    }
    __device__ __forceinline__ double value() const {
        float s0, s1, c0, c1;
        upk2(s, s0, s1);
        upk2(c, c0, c1);
        return ((double)s0 - (double)c0) + ((double)s1 - (double)c1);
    }
};

// Keys of a 32-column run starting at key jj that row i takes (j <= i).
__device__ __forceinline__ int run_valid(bool valid_row, long long i, long long jj) {
    if (!valid_row) return 0;
    const long long n = i - jj + 1;
    return n <= 0 ? 0 : (n >= 32 ? 32 : (int)n);
}

template <int D, int PASS>
__device__ void tc_epilogue(const TcParams& p, uint8_t* sm, const TcBars& bars,
                            volatile int* abort, uint32_t tmem, int jb, int je, int ntiles,
                            int it_a, int it_b, int chunk) {
    using Lay = TcLayout<D, PASS>;
    using Sh = TcShape<PASS>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int et = threadIdx.x - kEpiWarp0 * 32;  // 0 .. kEpiThreads - 1
    const int quad = warp & 3, grp = (warp - kEpiWarp0) >> 2;
    const int row = 32 * quad + lane;  // tile row = TMEM lane
    const int slot = row >> 6, r = row & 63;
    const TcItem me = tc_item(p, slot ? it_b : it_a);
    const int pos = me.pos;
    const int L = p.L, N = p.N, rmin = me.rmin;
    const bool valid_row = pos >= 0 && r >= rmin;
    const long long i = (long long)me.e - 64 + r;  // this row's query position
    const int rr = me.rbase + r;                     // its index among the L rows
    const uint32_t t_row = tmem + ((uint32_t)(32 * quad) << 16) + Sh::kCols * grp;
    bool failed = false;

    if (PASS == 1) {
        // online max (raw dot-product units) and sum of 2^((s - max) * c)
        const float c = (float)(p.scale * kLog2e);
        float mraw = -FLT_MAX;
        double lsum = 0.0;
        for (int t = 0; t < ntiles; ++t) {
            if (!failed) failed = !epi_wait(p, bars, abort, t);
            if (failed) continue;
            tc_fence_after();
            const long long j0 = (long long)jb + (long long)t * kTcKeys + Sh::kCols * grp;
#pragma unroll
            for (int h = 0; h < Sh::kCols / 32; ++h) {
                uint32_t v[32];
                tmem_ld32(t_row + 128 * (t & 1) + 32 * h, v);
                const int nv = run_valid(valid_row, i, j0 + 32 * h);
                if (nv > 0) {
                    float tmax = -FLT_MAX;
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        if (u < nv) tmax = fmaxf(tmax, __uint_as_float(v[u]));
                    if (tmax > mraw) {
                        if (mraw != -FLT_MAX) lsum *= (double)ex2_approx((mraw - tmax) * c);
                        mraw = tmax;
                    }
                    const float mc = mraw * c;
                    float s = 0.f;
#pragma unroll
                    for (int u = 0; u < 32; ++u)
                        if (u < nv) s += ex2_approx(fmaf(__uint_as_float(v[u]), c, -mc));
                    lsum += (double)s;
                }
            }
            epi_release(bars, t);
        }
        // merge the two column halves of each row, then one partial per (row, chunk)
        double* red = reinterpret_cast<double*>(sm + Lay::red_off);  // [group][128] x (m, l)
        red[(grp * 128 + row) * 2] = mraw == -FLT_MAX ? -DBL_MAX : (double)mraw;
        red[(grp * 128 + row) * 2 + 1] = lsum;
        epi_bar<PASS>();
        if (grp == 0 && valid_row && !failed && !*abort) {
            const double c64 = (double)c;
            double m = red[row * 2], l = red[row * 2 + 1];
            const double m1 = red[(128 + row) * 2], l1 = red[(128 + row) * 2 + 1];
            if (!(m1 == -DBL_MAX || l1 == 0.0)) {
                if (m == -DBL_MAX || l == 0.0) {
                    m = m1;
                    l = l1;
                } else {
                    const double mn = fmax(m, m1);
                    l = l * exp2((m - mn) * c64) + l1 * exp2((m1 - mn) * c64);
                    m = mn;
                }
            }
            const size_t o = ((size_t)pos * L + rr) * p.nchunks + chunk;
            p.m_part[o] = l > 0.0 ? m * p.scale : -DBL_MAX;
            p.l_part[o] = l;
        }
        return;
    }

    // PASS 2
    float* P = reinterpret_cast<float*>(sm + Lay::p_off);           // [slot][64][kSkew]
    double* carry = reinterpret_cast<double*>(sm + Lay::carry_off);  // [tile parity][slot][64]
    // log2 e * (s * scale - m_i) = s * c - m' with c and m' as unevaluated fp32
    // pairs (hi + lo), so the exponent keeps ~48 bits without fp64 arithmetic
    const double c64 = p.scale * kLog2e;
    const float c_hi = (float)c64, c_lo = (float)(c64 - (double)c_hi);
    float m_hi = 0.f, m_lo = 0.f, li = 0.f;
    if (valid_row) {
        const double mq = p.mrow[(size_t)pos * L + rr] * kLog2e;
        m_hi = (float)mq;
        m_lo = (float)(mq - (double)m_hi);
        li = (float)p.linv[(size_t)pos * L + rr];
    }
    const uint64_t k_nchi = pk2(-c_hi, -c_hi), k_chi = pk2(c_hi, c_hi), k_mhi = pk2(m_hi, m_hi);
    const uint64_t k_clo = pk2(c_lo, c_lo), k_nmlo = pk2(-m_lo, -m_lo), k_li = pk2(li, li);
    const uint64_t k_ln2 = pk2(kLn2f, kLn2f), k_one = pk2(1.f, 1.f);
    // positions outside a row's 128 keys are never written: zero them once
    for (int x = et; x < 2 * 64 * kSkew; x += Sh::kEpiThreads) P[x] = 0.f;
    epi_bar<PASS>();
    float* const prow_base = P + slot * 64 * kSkew + r * (kSkew - 1) + 63;  // + column c
    for (int t = 0; t < ntiles; ++t) {
        const long long j0 = (long long)jb + (long long)t * kTcKeys;
        if (!failed) failed = !epi_wait(p, bars, abort, t);
        if (!failed) {
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < Sh::kCols / 32; ++h) {
                uint32_t v[32];
                tmem_ld32(t_row + 128 * (t & 1) + 32 * h, v);
                const int c0 = Sh::kCols * grp + 32 * h;
                const int nv = run_valid(valid_row, i, j0 + c0);
                float* prow = prow_base + c0;
#pragma unroll
                for (int u = 0; u < 32; u += 2) {
                    const uint64_t p2 = mul2(
                        prob2(pk2(__uint_as_float(v[u]), __uint_as_float(v[u + 1])), k_nchi,
                              k_chi, k_mhi, k_clo, k_nmlo, k_ln2, k_one),
                        k_li);
                    float p0, p1;
                    upk2(p2, p0, p1);
                    prow[u] = u < nv ? p0 : 0.f;
                    prow[u + 1] = u + 1 < nv ? p1 : 0.f;
                }
            }
            epi_release(bars, t);
        }
        epi_bar<PASS>();  // the tile's probabilities are staged
        if (!failed && !*abort) {
            // 256 column sums (slot, column) then 2 x 191 diagonal sums (slot,
            // u = c - r), dealt round-robin over the epilogue threads; a diagonal
            // that runs past the tile's last key (u >= 65) is carried into the
            // next tile
            const int tb = t & 1;
            for (int rd = et; rd < 256 + 2 * kDiag; rd += Sh::kEpiThreads) {
                if (rd < 256) {
                    const int cs = rd >> 7, cc = rd & 127;
                    const int citem = cs ? it_b : it_a;
                    const long long j = j0 + cc;
                    if (citem < 0 || j < jb || j >= je) continue;
                    const float* col = P + cs * 64 * kSkew + cc + 63;  // row q at q * (kSkew - 1)
                    KahanSum2 ks[2];  // four independent chains (rows q mod 4) in two pairs
#pragma unroll
                    for (int q = 0; q < 64; q += 4) {
#pragma unroll
                        for (int w = 0; w < 2; ++w)
                            ks[w].add(pk2(col[(q + 2 * w) * (kSkew - 1)],
                                          col[(q + 2 * w + 1) * (kSkew - 1)]));
                    }
                    p.vout[(size_t)citem * N + j] = (float)(ks[0].value() + ks[1].value());
                    continue;
                }
                const int dd = rd - 256;
                const int ds = dd >= kDiag ? 1 : 0;
                const int u = dd - ds * kDiag - 63;
                const TcItem dx = tc_item(p, ds ? it_b : it_a);
                if (dx.item < 0) continue;
                const float* dcol = P + ds * 64 * kSkew + u + 63;  // row q at q * kSkew
                KahanSum2 ks[2];  // four chains in two pairs; positions past a row's keys hold 0
#pragma unroll
                for (int q = 0; q < 64; q += 4) {
#pragma unroll
                    for (int w = 0; w < 2; ++w)
                        ks[w].add(pk2(dcol[(q + 2 * w) * kSkew], dcol[(q + 2 * w + 1) * kSkew]));
                }
                double s = ks[0].value() + ks[1].value();
                if (u < 0 && t > 0) s += carry[((tb ^ 1) * 2 + ds) * 64 + (u + 63)];
                if (u >= 65) {
                    carry[(tb * 2 + ds) * 64 + (u - 65)] = s;
                    continue;
                }
                const long long o = (long long)dx.e - 64 - j0 - u;
                if (o < 0 || o >= N) continue;
                const long long fk = max(0LL, j0 + u + dx.rmin);  // the diagonal's first key
                if (fk >= jb && fk < je) p.sout[(size_t)dx.item * N + o] = (float)s;
            }
        }
        epi_bar<PASS>();  // the staging buffer is free again
    }
}

template <int D, int PASS>
__global__ void __launch_bounds__(TcShape<PASS>::kThreads, PASS == 1 ? 2 : 1)
    vs_score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ TcParams p) {
    using Lay = TcLayout<D, PASS>;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte swizzled operands need a 1024-byte aligned base
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lay::bar_off);
    TcBars bars;
    bars.q_full = bar;
    bars.k_full = bar + 1;
    bars.k_empty = bar + 1 + kTcStages;
    bars.acc_full = bar + 1 + 2 * kTcStages;
    bars.acc_empty = bar + 3 + 2 * kTcStages;
    bars.drain = bar + 5 + 2 * kTcStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::misc_off);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + Lay::misc_off + 4);

    const int tile = blockIdx.x, chunk = blockIdx.y;
    int gi = 0;
    while (gi + 1 < p.ngroups && tile >= p.tstart[gi + 1]) ++gi;
    const int h0 = p.hstart[gi], nit = (p.hstart[gi + 1] - h0) * p.G;
    const int k0 = 2 * (tile - p.tstart[gi]);
    const int it_a = p.hpos[h0 + k0 / p.G] * p.G + k0 % p.G;
    const int it_b = k0 + 1 < nit ? p.hpos[h0 + (k0 + 1) / p.G] * p.G + (k0 + 1) % p.G : -1;
    const int g = kv_head_of(head_qh(p.heads.e[it_a / p.G]), p.Hq, p.Hkv);
    const int jb = chunk * p.chunk;
    const int je = min(p.N, jb + p.chunk);
    const int jend = PASS == 1 ? je : min(p.N, je + kTcKeys);
    const int ntiles = (jend - jb + kTcKeys - 1) / kTcKeys;
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        // one read for the whole CTA: every thread must take the same branch
        *abort = *reinterpret_cast<volatile unsigned int*>(&g_vs_abort_seq) == p.seq ? 1 : 0;
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.acc_full[b], 1);
            mbar_init(&bars.acc_empty[b], TcShape<PASS>::kEpiWarps);
        }
        mbar_init(bars.drain, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (*abort) return;  // an earlier CTA of this launch gave up: skip the work
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if ((threadIdx.x & 31) == 0)
            tc_producer<D>(p, &tmQ, &tmK, sm, bars, abort, g, jb, ntiles, it_a, it_b);
    } else if (warp == 1) {
        tc_mma<D>(p, sm, bars, abort, tmem, ntiles);
        tc_fence_before();
    } else {
        tc_epilogue<D, PASS>(p, sm, bars, abort, tmem, jb, je, ntiles, it_a, it_b, chunk);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
    }
}

// last_q > 64: a head's scores are the sums of its items' partial sums, in row
// group order.  Row group g has no row at or past key (or diagonal) N - 64 g,
// so its partials there are never written and not read.
__global__ void vs_part_merge_kernel(const float* __restrict__ vpart,
                                     const float* __restrict__ spart, int G, int N,
                                     float* __restrict__ vscore, float* __restrict__ sscore) {
    const int pos = blockIdx.y;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < N; j += gridDim.x * blockDim.x) {
        double v = 0.0, sl = 0.0;
        for (int g = 0; g < G && j < N - 64 * g; ++g) {
            v += vpart[((size_t)pos * G + g) * N + j];
            sl += spart[((size_t)pos * G + g) * N + j];
        }
        vscore[(size_t)pos * N + j] = (float)v;
        sscore[(size_t)pos * N + j] = (float)sl;
    }
}

template <int D, int PASS>
cudaError_t launch_pass(const CUtensorMap& tmQ, const CUtensorMap& tmK, const TcParams& p,
                        cudaStream_t st) {
    const int smem = TcLayout<D, PASS>::bytes;
    cudaError_t e = cudaFuncSetAttribute(vs_score_tc_kernel<D, PASS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    vs_score_tc_kernel<D, PASS><<<dim3(p.tstart[p.ngroups], p.nchunks), TcShape<PASS>::kThreads,
                                  smem, st>>>(tmQ, tmK, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vs_scores_tc(int pass, const bf16* q, const bf16* k, int Hq, int Hkv, int N,
                                int d, double scale, int L, const HeadList& heads,
                                const VsIndexWs& ws, float* vscore, float* sscore,
                                cudaStream_t st) {
    if (heads.n == 0) return cudaSuccess;
    if (L < 1 || L > N || L > 1024 || N < 64 || (d != 64 && d != 128)) return cudaErrorInvalidValue;
    CUtensorMap tmQ, tmK;
    if (!make_tma_map(&tmQ, q, (long long)Hq * N, d, 64) ||
        !make_tma_map(&tmK, k, (long long)Hkv * N, d, kTcKeys))
        return cudaErrorInvalidValue;
    // launch sequence number (never 0), unique across host threads
    static std::atomic<unsigned int> next_seq{0};
    unsigned int seq = ++next_seq;
    TcParams p;
    memset(&p, 0, sizeof(p));
    if (seq == 0) seq = ++next_seq;
    p.seq = seq;
    p.wait_budget = wait_budget_cycles();
    p.heads = heads;
    // items of each KV head in list order (each head's row groups together),
    // paired into tiles; an odd one out runs alone
    const int G = (L + 63) / 64;
    int nh = 0, ng = 0, nt = 0;
    for (int g = 0; g < Hkv; ++g) {
        const int start = nh;
        for (int i = 0; i < heads.n; ++i)
            if (kv_head_of(head_qh(heads.e[i]), Hq, Hkv) == g) p.hpos[nh++] = (int16_t)i;
        if (nh > start) {
            p.hstart[ng] = (int16_t)start;
            p.tstart[ng] = nt;
            nt += ((nh - start) * G + 1) / 2;
            ++ng;
        }
    }
    p.hstart[ng] = (int16_t)nh;
    p.tstart[ng] = nt;
    p.ngroups = ng;
    p.G = G;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.N = N;
    p.L = L;
    p.chunk = kVsTcChunk;
    p.nchunks = (N + kVsTcChunk - 1) / kVsTcChunk;
    p.scale = scale;
    p.m_part = ws.m_part;
    p.l_part = ws.l_part;
    p.mrow = ws.mrow;
    p.linv = ws.linv;
    p.vout = G == 1 ? vscore : ws.vpart;
    p.sout = G == 1 ? sscore : ws.spart;
    if (G > 1 && (!ws.vpart || !ws.spart)) return cudaErrorInvalidValue;
    if (pass == 1)
        return d == 128 ? launch_pass<128, 1>(tmQ, tmK, p, st) : launch_pass<64, 1>(tmQ, tmK, p, st);
    cudaError_t e = d == 128 ? launch_pass<128, 2>(tmQ, tmK, p, st)
                             : launch_pass<64, 2>(tmQ, tmK, p, st);
    if (e != cudaSuccess || G == 1) return e;
    vs_part_merge_kernel<<<dim3((N + 255) / 256, heads.n), 256, 0, st>>>(ws.vpart, ws.spart, G, N,
                                                                          vscore, sscore);
    return cudaGetLastError();
}

cudaError_t read_vs_wait_failure(int* out8) {
    int rec[8];
    cudaError_t e = cudaMemcpyFromSymbol(rec, g_vs_wait_fail, sizeof(rec));
    if (e != cudaSuccess) return e;
    for (int i = 0; i < 8; ++i) out8[i] = rec[i];
    const int zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    return cudaMemcpyToSymbol(g_vs_wait_fail, zero, sizeof(zero));
}

}  // namespace minfer

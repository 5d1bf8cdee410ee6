// attn_kt.cu -- Block-Sparse attention on key-major tensor-core tiles.
//
// MInference 1.0 (aifetchly guide, "3. The Block-Sparse Pattern" and
// "Block-Sparse Kernel Mechanics"): each 64-row query block attends only the
// 64-key blocks its index chose, computed as dense tiles.  The chosen sets of
// neighbouring query blocks are close to independent draws, so a 128-row MMA
// tile that stacks two query blocks (the row-major engine of attn.cu) is
// mostly half used here.  This engine turns the tile around: one work item is
// one query block (N = 64 queries) and each MMA tile stacks two of ITS chosen
// key blocks on M (128 keys), so every score the tensor core computes is one
// the item needs:
//   S^T[key, q] = K_chunk . Q^T        M = 128 keys, N = 64, K = d   (SS)
//   O^T[dim, q] += V_chunk^T . P^T     M = d = 128, N = 64, K = 128   (SS)
// with S^T and O^T in TMEM (lane = key, resp. head dimension) and P^T written
// by the softmax warps to shared memory as the second MMA's B operand.
//
// The online softmax runs per query = per TMEM column, across the 128 lanes
// of four warps.  Every thread holds one key and 32 queries; a query's
// reference max is shared by all keys of a chunk (one MMA sums them), so the
// eight softmax warps vote once per chunk whether some score exceeds its
// query's reference by more than 2^8 (lazy rescale, as in attn.cu); only then
// do they reduce the chunk's per-query max across lanes and rescale O^T and
// the running sums.  The first chunk of every item takes that path.
//
// Warps: 0-7 softmax (warp w: TMEM lane quarter w % 4, queries 32 (w / 4) ..
// +31), 8 producer (index -> chunk list, TMA loads), 9 MMA issuer.  The CTA
// is persistent: items (query head, query block) are ordered KV head by KV
// head, latest query block first, and dealt round-robin over the CTAs, so the
// CTAs in flight read one KV head's K/V from L2.  Shared memory: Q (one item),
// three K stages, two V stages and two P^T buffers; TMEM: two S^T buffers and
// two O^T buffers (consecutive items alternate, so an item's epilogue overlaps
// the next item's first chunks).
#include <atomic>
#include <cfloat>
#include <cstring>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "softmax_math.cuh"

namespace minfer {

namespace {

constexpr int kKtD = 128;                 // head dimension this engine serves
constexpr int kKtWarpsSoftmax = 8;
constexpr int kKtProducerWarp = 8;
constexpr int kKtMmaWarp = 9;
constexpr int kKtThreads = 320;
constexpr int kKtKeys = 128;              // keys per chunk (MMA M of S^T)
constexpr int kKtRows = 64;               // queries per item (MMA N)
constexpr int kKtKStages = 3;
constexpr int kKtVStages = 2;
constexpr int kKtDescRing = 8;
constexpr float kKtRescale = 8.0f;        // log2 units: rescale when a score passes its max by 2^8
constexpr uint32_t kKtTmemCols = 256;     // S^T 2 x 64, O^T 2 x 64

enum : int { kKtChunk = 0, kKtEmpty = 1, kKtEnd = 2 };
enum : int {
    kKtFirst = 1,       // first chunk of its item
    kKtLast = 2,        // last chunk of its item
    kKtHalf1 = 4,       // keys 64-127 hold a chosen block (else they repeat block b0, masked)
    kKtDiag0 = 8,       // block b0 is the item's own (diagonal) block: causal mask
    kKtDiag1 = 16       // the same for b1
};

struct KtDesc {
    int type, flags, b0, b1, qh, qb;
};

// Sequence number of the last launch in which a CTA gave up waiting.
__device__ unsigned int g_kt_abort_seq = 0;
// First wait that gave up: {launch seq, site, block, thread, chunk, parity, 0, 0}.
__device__ int g_kt_wait_fail[8];

enum : int {
    kSiteKtProducer = 21,
    kSiteKtMmaQ = 22,
    kSiteKtMmaK = 23,
    kSiteKtMmaP = 24,
    kSiteKtSoftmaxDesc = 25,
    kSiteKtSoftmaxS = 26,
    kSiteKtSoftmaxO = 27
};

__device__ void kt_record_wait_failure(unsigned int seq, int site, int chunk, int parity) {
    if (atomicCAS(&g_kt_wait_fail[1], 0, site) == 0) {
        g_kt_wait_fail[0] = (int)seq;
        g_kt_wait_fail[2] = (int)blockIdx.x;
        g_kt_wait_fail[3] = (int)threadIdx.x;
        g_kt_wait_fail[4] = chunk;
        g_kt_wait_fail[5] = parity;
        __threadfence();
    }
}

struct KtParams {
    unsigned int seq;
    long long wait_budget;
    const bf16* k;
    const bf16* v;
    bf16* out;
    float* lse;
    int Hq, Hkv, N, nB;
    float scale_log2;
    const int32_t* blk_idx;
    const int32_t* blk_cnt;
    int topk;
    int32_t* err;
    int n_items;
    HeadList heads;  // Block-Sparse heads, sorted by KV head
    int ngroups;
    uint16_t grp_start[MI_MAX_HEADS + 1];
};

struct KtLayout {
    static constexpr int kPanelQ = kKtRows * 128;           // 64 rows x 128 bytes
    static constexpr int kPanelKV = kKtKeys * 128;          // 128 rows x 128 bytes
    static constexpr int kQBytes = 2 * kPanelQ;             // d = 128: two panels
    static constexpr int kKVBytes = 2 * kPanelKV;
    static constexpr int kPBytes = kKtKeys * 128;           // 128 keys x 64 queries bf16
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + kQBytes;
    static constexpr int v_off = k_off + kKtKStages * kKVBytes;
    static constexpr int p_off = v_off + kKtVStages * kKVBytes;
    static constexpr int desc_off = p_off + 2 * kPBytes;
    static constexpr int red_off = desc_off + kKtDescRing * (int)sizeof(KtDesc);  // [4][64] f32
    static constexpr int m_off = red_off + 4 * 64 * 4;       // reference max per query (log2 units)
    static constexpr int alpha_off = m_off + 64 * 4;
    static constexpr int linv_off = alpha_off + 64 * 4;
    static constexpr int flag_off = linv_off + 64 * 4;       // [2][8] votes
    static constexpr int misc_off = flag_off + 2 * 8 * 4;    // tmem base, abort
    static constexpr int bar_off = (misc_off + 16 + 15) & ~15;
    static constexpr int kNumBars = 2 + 2 * kKtDescRing + 2 * kKtKStages + 2 * kKtVStages + 3 * 2 +
                                    2 * 2 + 1;
    static constexpr int bitmap_off = bar_off + kNumBars * 8;
    static size_t bytes(int bitmap_words) {
        return (size_t)bitmap_off + (size_t)bitmap_words * 4 + 1024;  // +1024: base alignment
    }
};
static_assert(KtLayout::p_off % 1024 == 0 && KtLayout::k_off % 1024 == 0 &&
                  KtLayout::v_off % 1024 == 0,
              "swizzled operands need 1024-byte alignment");

struct KtBars {
    uint64_t* q_full;
    uint64_t* q_empty;
    uint64_t* desc_full;   // [8]
    uint64_t* desc_empty;  // [8] MMA + 8 softmax warps
    uint64_t* k_full;      // [3]
    uint64_t* k_empty;     // [3] S^T of the chunk has run
    uint64_t* v_full;      // [2]
    uint64_t* v_empty;     // [2] O^T of the chunk has run
    uint64_t* s_full;      // [2] S^T in TMEM buffer
    uint64_t* p_full;      // [2] P^T written (8 softmax warps); the S^T buffer is read
    uint64_t* p_free;      // [2] O^T that reads the P^T buffer has run
    uint64_t* o_full;      // [2] last O^T of an item has run
    uint64_t* o_free;      // [2] the item's epilogue has read O^T (8 softmax warps)
    uint64_t* drain;
};

// kind::f16, bf16 A/B, fp32 D; a_mn / b_mn: operand stored MN-major.
__host__ __device__ constexpr uint32_t kt_idesc(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void kt_set_abort(volatile int* abort, int32_t* err, unsigned int seq) {
    *abort = 1;
    if (err) atomicOr(err, 1 << 30);
    atomicExch(&g_kt_abort_seq, seq);
}

// Named barrier of the eight softmax warps that also ORs a predicate over
// them: every warp gets the same answer to "did any warp want to stop".  (A
// plain barrier followed by each warp reading the CTA's abort flag could split
// the warps, since the producer or MMA warp may set the flag in between, and
// leave some waiting at the next barrier.)
__device__ __forceinline__ bool kt_softmax_bar(bool stop) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 256, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)stop)
        : "memory");
    return r != 0;
}

// Item `it` -> (position in the head list, query block): KV head by KV head,
// latest query block first, the group's heads interleaved.
__device__ __forceinline__ void kt_item(const KtParams& p, int it, int& pos, int& qb) {
    int gi = 0;
    while (gi + 1 < p.ngroups && it >= (int)p.grp_start[gi + 1] * p.nB) ++gi;
    const int gsize = p.grp_start[gi + 1] - p.grp_start[gi];
    const int r = it - (int)p.grp_start[gi] * p.nB;
    qb = p.nB - 1 - r / gsize;
    pos = p.grp_start[gi] + r % gsize;
}

// ------------------------------------------------------------- producer
struct KtProducer {
    const KtParams& p;
    const CUtensorMap* tmQ;
    const CUtensorMap* tmK;
    const CUtensorMap* tmV;
    uint8_t* sm;
    KtBars bars;
    volatile int* abort;
    int lane;
    int nd = 0;  // descriptors published
    int nc = 0;  // chunks (K loads) issued
    int nv = 0;  // V loads issued
    int nq = 0;  // Q loads issued
    int pv0 = -1, pv1 = -1, pg = 0;  // chunk whose V is still to load: blocks, KV head
    bool ok = true;

    __device__ bool wait(uint64_t* bar, int parity, int count) {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar, parity, abort, p.wait_budget);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
            if (lane == 0) {
                if (!*abort) kt_record_wait_failure(p.seq, kSiteKtProducer, count, parity);
                kt_set_abort(abort, p.err, p.seq);
            }
            ok = false;
        }
        return w;
    }

    __device__ bool publish(const KtDesc& d) {
        if (!ok) return false;
        const int slot = nd % kKtDescRing;
        if (nd >= kKtDescRing && !wait(&bars.desc_empty[slot], ((nd / kKtDescRing) - 1) & 1, nd))
            return false;
        if (lane == 0) reinterpret_cast<KtDesc*>(sm + KtLayout::desc_off)[slot] = d;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.desc_full[slot]);
        ++nd;
        return true;
    }

    // the two 64-key halves of a K or V stage: rows g*N + 64 b0 and + 64 b1
    __device__ void load_halves(uint8_t* dst, const CUtensorMap* tm, int g, int b0, int b1,
                                uint64_t* bar, uint64_t pol) {
#pragma unroll
        for (int pn = 0; pn < 2; ++pn) {
            tma_load_2d_hint(dst + pn * KtLayout::kPanelKV, tm, 64 * pn, g * p.N + 64 * b0, bar,
                             pol);
            tma_load_2d_hint(dst + pn * KtLayout::kPanelKV + 64 * 128, tm, 64 * pn,
                             g * p.N + 64 * b1, bar, pol);
        }
    }

    __device__ void load_v_pending() {
        if (!ok || pv0 < 0) return;
        const int st = nv % kKtVStages;
        if (nv >= kKtVStages && !wait(&bars.v_empty[st], ((nv / kKtVStages) - 1) & 1, nv)) return;
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars.v_full[st], KtLayout::kKVBytes);
            load_halves(sm + KtLayout::v_off + st * KtLayout::kKVBytes, tmV, pg, pv0, pv1,
                        &bars.v_full[st], l2_policy_evict_last());
        }
        __syncwarp();
        ++nv;
        pv0 = -1;
    }

    // one chunk: descriptor, K now, the previous chunk's V, and the item's Q
    // on its first chunk (after the previous item's last S^T has read Q)
    __device__ void chunk(int g, int qh, int qb, int b0, int b1, bool first, bool last) {
        KtDesc d;
        d.type = kKtChunk;
        d.flags = (first ? kKtFirst : 0) | (last ? kKtLast : 0) | (b1 >= 0 ? kKtHalf1 : 0) |
                  (b0 == qb ? kKtDiag0 : 0) | (b1 == qb ? kKtDiag1 : 0);
        d.b0 = b0;
        d.b1 = b1 >= 0 ? b1 : b0;  // unused half: a real block (finite data), masked
        d.qh = qh;
        d.qb = qb;
        if (!publish(d)) return;
        const int st = nc % kKtKStages;
        if (nc >= kKtKStages && !wait(&bars.k_empty[st], ((nc / kKtKStages) - 1) & 1, nc)) return;
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars.k_full[st], KtLayout::kKVBytes);
            load_halves(sm + KtLayout::k_off + st * KtLayout::kKVBytes, tmK, g, d.b0, d.b1,
                        &bars.k_full[st], l2_policy_evict_last());
        }
        __syncwarp();
        ++nc;
        load_v_pending();
        pv0 = d.b0;
        pv1 = d.b1;
        pg = g;
        if (first && ok) {
            if (nq > 0 && !wait(bars.q_empty, (nq - 1) & 1, -1 - nq)) return;
            if (lane == 0) {
                mbar_arrive_expect_tx(bars.q_full, KtLayout::kQBytes);
#pragma unroll
                for (int pn = 0; pn < 2; ++pn)
                    tma_load_2d_hint(sm + KtLayout::q_off + pn * KtLayout::kPanelQ, tmQ, 64 * pn,
                                     qh * p.N + 64 * qb, bars.q_full, l2_policy_evict_first());
            }
            __syncwarp();
            ++nq;
        }
    }

    // Wait (bounded) for every copy this warp started, so that no TMA write
    // can reach shared memory after the CTA exits.
    __device__ void drain() {
        if (lane != 0) return;
        for (int u = nc - kKtKStages; u < nc; ++u)
            if (u >= 0) mbar_wait_budget(&bars.k_full[u % kKtKStages], (u / kKtKStages) & 1);
        for (int u = nv - kKtVStages; u < nv; ++u)
            if (u >= 0) mbar_wait_budget(&bars.v_full[u % kKtVStages], (u / kKtVStages) & 1);
        if (nq > 0) mbar_wait_budget(bars.q_full, (nq - 1) & 1);
    }
};

__device__ void kt_run_producer(const KtParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                                const CUtensorMap* tmV, uint8_t* sm, const KtBars& bars,
                                volatile int* abort) {
    const int lane = threadIdx.x & 31;
    uint32_t* bm = reinterpret_cast<uint32_t*>(sm + KtLayout::bitmap_off);
    if (lane == 0) {
        prefetch_tmap(tmQ);
        prefetch_tmap(tmK);
        prefetch_tmap(tmV);
    }
    KtProducer pr{p, tmQ, tmK, tmV, sm, bars, abort, lane};
    for (int it = blockIdx.x; it < p.n_items && pr.ok; it += gridDim.x) {
        int pos, qb;
        kt_item(p, it, pos, qb);
        const uint32_t e = p.heads.e[pos];
        const int qh = head_qh(e), pidx = head_pidx(e);
        const int g = kv_head_of(qh, p.Hq, p.Hkv);
        // the item's key blocks as a bitmap over [0, qb]: duplicates count once,
        // -1 is padding, anything else outside [0, qb] is skipped and counted
        const int nw = qb / 32 + 1;
        for (int w = lane; w < nw; w += 32) bm[w] = 0;
        __syncwarp();
        const int cnt = min(p.blk_cnt[(size_t)pidx * p.nB + qb], p.topk);
        const int32_t* lst = p.blk_idx + ((size_t)pidx * p.nB + qb) * p.topk;
        for (int t = lane; t < cnt; t += 32) {
            const int bk = lst[t];
            if (bk == -1) continue;
            if (bk < 0 || bk > qb) {
                if (p.err) atomicAdd(p.err, 1);
                continue;
            }
            atomicOr(&bm[bk >> 5], 1u << (bk & 31));
        }
        __syncwarp();
        int total = 0;
        for (int w = lane; w < nw; w += 32) total += __popc(bm[w]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        if (total == 0) {
            KtDesc d{kKtEmpty, 0, 0, 0, qh, qb};
            pr.publish(d);
            continue;
        }
        const int nchunks = (total + 1) / 2;
        int emitted = 0, pend = -1;
        for (int base = 0; base < nw && pr.ok; base += 32) {
            const uint32_t word = base + lane < nw ? bm[base + lane] : 0u;
            unsigned nz = __ballot_sync(0xffffffffu, word != 0u);
            while (nz && pr.ok) {
                const int src = __ffs(nz) - 1;
                nz &= nz - 1;
                uint32_t wv = __shfl_sync(0xffffffffu, word, src);
                while (wv && pr.ok) {
                    const int b = (base + src) * 32 + __ffs(wv) - 1;
                    wv &= wv - 1;
                    if (pend < 0) {
                        pend = b;
                    } else {
                        pr.chunk(g, qh, qb, pend, b, emitted == 0, emitted == nchunks - 1);
                        ++emitted;
                        pend = -1;
                    }
                }
            }
        }
        if (pend >= 0 && pr.ok) {
            pr.chunk(g, qh, qb, pend, -1, emitted == 0, true);
            ++emitted;
        }
        __syncwarp();
    }
    pr.load_v_pending();
    KtDesc end{kKtEnd, 0, 0, 0, 0, 0};
    pr.publish(end);
    pr.drain();
}

// ------------------------------------------------------------- MMA issuer
// One converged warp.  An mbarrier probe costs a couple of hundred cycles
// even on a completed phase, so each round tests every barrier the next
// actions need in ONE non-blocking test_wait across lanes, then issues what is
// ready:
//   lane 0  the next descriptor            lane 4  P^T of the oldest pending O
//   lane 1  K of the next S                lane 5  V of that chunk
//   lane 2  its S^T buffer free            lane 6  its O^T buffer free (first
//   lane 3  the item's Q (first chunk)             chunk of an item two back)
// S^T of chunk n goes first (it feeds the softmax), then O^T of the oldest
// chunk whose P^T is ready.  All MMA operands come from lane-0 broadcasts, so
// they stay in uniform registers (operands the compiler cannot prove uniform
// make each MMA issue several times slower than the tensor pipe runs).
__device__ void kt_run_mma(const KtParams& p, uint8_t* sm, const KtBars& bars,
                           volatile int* abort, uint32_t tmem) {
    const int lane = threadIdx.x & 31;
    constexpr uint32_t idS = kt_idesc(128, kKtRows, false, false);
    constexpr uint32_t idO = kt_idesc(128, kKtRows, true, true);
    tmem = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t q_addr = __shfl_sync(0xffffffffu, smem_u32(sm + KtLayout::q_off), 0);
    const uint32_t k_addr = __shfl_sync(0xffffffffu, smem_u32(sm + KtLayout::k_off), 0);
    const uint32_t v_addr = __shfl_sync(0xffffffffu, smem_u32(sm + KtLayout::v_off), 0);
    const uint32_t p_addr = __shfl_sync(0xffffffffu, smem_u32(sm + KtLayout::p_off), 0);
    const KtDesc* desc = reinterpret_cast<const KtDesc*>(sm + KtLayout::desc_off);

    // chunks whose S^T has run but not their O^T yet (at most three), 8 bits
    // each at (chunk % 4) * 8: descriptor flags, O^T buffer parity (bit 5),
    // O^T buffer last used by an item two back (bit 6)
    uint32_t pend = 0;
    int nd = 0;            // next descriptor
    bool have = false;     // descriptor read, its S^T not issued yet
    int dflags = 0;
    int ns = 0, no = 0;    // next S^T / O^T chunk
    int qi = 0, cur_o = 0; // items with chunks so far; the current one's O^T index
    bool done = false, ok = true;
    unsigned idle = 0;
    long long t_last = clock64();
    while (ok && !(done && no == ns)) {
        const uint32_t po = (pend >> ((no & 3) * 8)) & 0xFFu;
        uint64_t* bar = bars.q_full;  // a completed barrier for lanes with nothing to test
        uint32_t par = 0;
        bool live = false;
        if (lane == 0 && !have && !done) {
            bar = &bars.desc_full[nd % kKtDescRing]; par = (nd / kKtDescRing) & 1; live = true;
        } else if (lane == 1 && have) {
            bar = &bars.k_full[ns % kKtKStages]; par = (ns / kKtKStages) & 1; live = true;
        } else if (lane == 2 && have && ns >= 2) {
            bar = &bars.p_full[ns & 1]; par = ((ns - 2) >> 1) & 1; live = true;
        } else if (lane == 3 && have && (dflags & kKtFirst)) {
            bar = bars.q_full; par = qi & 1; live = true;
        } else if (lane == 4 && no < ns) {
            bar = &bars.p_full[no & 1]; par = (no >> 1) & 1; live = true;
        } else if (lane == 5 && no < ns) {
            bar = &bars.v_full[no % kKtVStages]; par = (no / kKtVStages) & 1; live = true;
        } else if (lane == 6 && no < ns && (po & kKtFirst) && (po & 64)) {
            // the O^T buffer was last used by the item two back: its epilogue
            // (completion (item / 2) - 1 of that buffer's o_free) must have read it
            bar = &bars.o_free[(po >> 5) & 1];
            par = ((po >> 7) & 1) ^ 1;
            live = true;
        }
        const bool hit = live ? mbar_test_wait(bar, par) : true;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        const bool desc_ready = !have && !done && (bal & 1u);
        const bool s_ready = have && ((bal >> 1) & 7u) == 7u;
        const bool o_ready = no < ns && ((bal >> 4) & 7u) == 7u;
        if (!(desc_ready || s_ready || o_ready)) {
            if ((++idle & 15) != 0) continue;
            const bool give_up = *abort || clock64() - t_last > p.wait_budget;
            if (__any_sync(0xffffffffu, give_up)) {
                if (lane == 0 && !*abort)
                    kt_record_wait_failure(p.seq, have ? kSiteKtMmaK : kSiteKtMmaP, ns, no);
                ok = false;
            }
            continue;
        }
        t_last = clock64();
        if (desc_ready) {
            const int slot = nd % kKtDescRing;
            const int type = __shfl_sync(0xffffffffu, desc[slot].type, 0);
            dflags = __shfl_sync(0xffffffffu, desc[slot].flags, 0);
            mbar_arrive_warp(&bars.desc_empty[slot]);
            ++nd;
            if (type == kKtChunk) have = true;
            else if (type == kKtEnd) done = true;
        }
        if (s_ready) {  // S^T[key, q] = K . Q^T for chunk ns
            tc_fence_after();
            if (dflags & kKtFirst) cur_o = qi++;
            const int n = ns;
            const uint32_t kst =
                __shfl_sync(0xffffffffu, k_addr + (n % kKtKStages) * KtLayout::kKVBytes, 0);
            const uint32_t tS = __shfl_sync(0xffffffffu, tmem + 64 * (n & 1), 0);
#pragma unroll
            for (int kk = 0; kk < kKtD / 16; ++kk) {
                const int pn = kk >> 2, off = (kk & 3) * 32;
                const uint64_t adesc = sw128_desc(kst + pn * KtLayout::kPanelKV + off, 16, 1024);
                const uint64_t bdesc = sw128_desc(q_addr + pn * KtLayout::kPanelQ + off, 16, 1024);
                mma_ss_warp(tS, adesc, bdesc, idS, kk > 0 ? 1u : 0u);
            }
            mma_commit_warp(&bars.s_full[n & 1]);
            mma_commit_warp(&bars.k_empty[n % kKtKStages]);
            if (dflags & kKtLast) mma_commit_warp(bars.q_empty);
            // bits 0-4 flags, 5 O^T buffer, 6 buffer used before, 7 (item / 2) % 2
            const uint32_t info = (uint32_t)(dflags & 31) | ((uint32_t)(cur_o & 1) << 5) |
                                  ((cur_o >= 2 ? 1u : 0u) << 6) | ((uint32_t)((cur_o >> 1) & 1) << 7);
            pend = (pend & ~(0xFFu << ((n & 3) * 8))) | (info << ((n & 3) * 8));
            ++ns;
            have = false;
        }
        if (o_ready) {  // O^T[dim, q] += V^T . P^T for chunk no
            tc_fence_after();
            const int m = no;
            const uint32_t vst =
                __shfl_sync(0xffffffffu, v_addr + (m % kKtVStages) * KtLayout::kKVBytes, 0);
            const uint32_t pst = __shfl_sync(0xffffffffu, p_addr + (m & 1) * KtLayout::kPBytes, 0);
            const uint32_t tO = __shfl_sync(0xffffffffu, tmem + 128 + 64 * ((po >> 5) & 1), 0);
            const uint32_t acc0 = __shfl_sync(0xffffffffu, (po & kKtFirst) ? 0u : 1u, 0);
#pragma unroll
            for (int kk = 0; kk < kKtKeys / 16; ++kk) {
                // A = V^T (d x keys) stored MN-major: d-panels of 64 at kPanelKV apart,
                // 16 keys = 16 rows of 128 bytes per K-step
                const uint64_t adesc = sw128_desc(vst + kk * 2048, KtLayout::kPanelKV, 1024);
                // B = P^T (64 queries x keys) stored MN-major: one 128-byte row per key
                const uint64_t bdesc = sw128_desc(pst + kk * 2048, KtLayout::kPBytes, 1024);
                mma_ss_warp(tO, adesc, bdesc, idO, kk == 0 ? acc0 : 1u);
            }
            mma_commit_warp(&bars.p_free[m & 1]);
            mma_commit_warp(&bars.v_empty[m % kKtVStages]);
            if (po & kKtLast) mma_commit_warp(&bars.o_full[(po >> 5) & 1]);
            ++no;
        }
    }
    if (!ok && lane == 0) kt_set_abort(abort, p.err, p.seq);
    // every MMA of this warp must have finished before TMEM is released
    mma_commit_warp(bars.drain);
    if (lane == 0) mbar_wait_budget(bars.drain, 0);
    __syncwarp();
}

// ------------------------------------------------------------- softmax
// Warp-wide reduce-scatter of 32 values per lane: afterwards lane j holds the
// reduction over the 32 lanes of value j.
template <bool MAX>
__device__ __forceinline__ float kt_reduce_scatter(float (&v)[32], int lane) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool up = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = up ? v[i] : v[i + s];
            const float keep = up ? v[i + s] : v[i];
            const float r = __shfl_xor_sync(0xffffffffu, send, s);
            v[i] = MAX ? fmaxf(keep, r) : keep + r;
        }
    }
    return v[0];
}

__device__ void kt_run_softmax(const KtParams& p, uint8_t* sm, const KtBars& bars,
                               volatile int* abort, uint32_t tmem) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3, ch = warp >> 2;
    const int kl = 32 * quarter + lane;  // key of the chunk (TMEM lane of S^T)
    const int half = kl >> 6, kk = kl & 63;
    const int tid = threadIdx.x;         // 0..255
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t tbase = __shfl_sync(0xffffffffu, tmem + lane_off + 32 * ch, 0);
    const KtDesc* desc = reinterpret_cast<const KtDesc*>(sm + KtLayout::desc_off);
    float* red = reinterpret_cast<float*>(sm + KtLayout::red_off);      // [4][64]
    float* Mq = reinterpret_cast<float*>(sm + KtLayout::m_off);         // [64]
    float* alpha = reinterpret_cast<float*>(sm + KtLayout::alpha_off);  // [64]
    float* linv = reinterpret_cast<float*>(sm + KtLayout::linv_off);    // [64]
    int* flags_sm = reinterpret_cast<int*>(sm + KtLayout::flag_off);    // [2][8]
    uint8_t* pbuf = sm + KtLayout::p_off;
    const float cs = p.scale_log2;

    float l[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) l[i] = 0.f;
    bool ok = true;  // this warp has seen every wait complete
    int nc = 0, qi = 0;

    // A wait of one warp (lane 0 waits, the warp follows).  A warp whose wait
    // gives up sets the CTA's abort flag and carries on to its next named
    // barrier without touching data; every named barrier ORs the warps' stop
    // requests, so they all leave at the same one and none is left waiting.
    auto wait = [&](uint64_t* bar, int parity, int site, int chunk) -> bool {
        if (!ok) return false;
        bool w = true;
        if (lane == 0) {
            w = mbar_wait(bar, parity, abort, p.wait_budget);
            if (!w) {
                if (!*abort) kt_record_wait_failure(p.seq, site, chunk, parity);
                kt_set_abort(abort, p.err, p.seq);
            }
        }
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) ok = false;
        return w;
    };

    for (int nd = 0;; ++nd) {
        const int slot = nd % kKtDescRing;
        // One probe across lanes for the three barriers a chunk normally waits
        // on (its descriptor, its S^T, its P^T buffer free); those found
        // complete cost no further wait.
        bool pre_desc, pre_s, pre_pf;
        {
            uint64_t* bar = bars.q_full;
            uint32_t par = 0;
            bool live = false;
            if (lane == 0) {
                bar = &bars.desc_full[slot]; par = (nd / kKtDescRing) & 1; live = true;
            } else if (lane == 1) {
                bar = &bars.s_full[nc & 1]; par = (nc >> 1) & 1; live = true;
            } else if (lane == 2 && nc >= 2) {
                bar = &bars.p_free[nc & 1]; par = ((nc - 2) >> 1) & 1; live = true;
            }
            const unsigned bal = __ballot_sync(0xffffffffu, live ? mbar_test_wait(bar, par) : true);
            pre_desc = bal & 1u;
            pre_s = (bal >> 1) & 1u;
            pre_pf = (bal >> 2) & 1u;
        }
        int type = kKtEnd, flags = 0, qh = 0, qb = 0;
        if (pre_desc ||
            wait(&bars.desc_full[slot], (nd / kKtDescRing) & 1, kSiteKtSoftmaxDesc, -1 - nd)) {
            type = desc[slot].type;
            flags = desc[slot].flags;
            qh = desc[slot].qh;
            qb = desc[slot].qb;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.desc_empty[slot]);
        }
        if (!ok || type == kKtEnd) {
            kt_softmax_bar(true);  // matches the other warps' next named barrier
            break;
        }
        const size_t row0 = (size_t)qh * p.N + 64 * (size_t)qb;
        if (type == kKtEmpty) {  // no key at all: zero rows, lse = -inf
            uint4* dst = reinterpret_cast<uint4*>(p.out + row0 * kKtD);
            for (int i = tid; i < kKtRows * kKtD / 8; i += 256) __stcs(dst + i, make_uint4(0, 0, 0, 0));
            if (p.lse && tid < kKtRows) p.lse[row0 + tid] = -INFINITY;
            continue;
        }
        const int n = nc++;
        const int b = n & 1;
        const bool first = (flags & kKtFirst) != 0;
        if (first) ++qi;
        const int ob = (qi - 1) & 1;
        const bool valid = half == 0 || (flags & kKtHalf1);
        const bool diag = (half == 0 ? (flags & kKtDiag0) : (flags & kKtDiag1)) != 0;

        // --- scores of this key for the warp's 32 queries (raw dot products).
        // A warp's 32 keys lie in one half, so `valid` and `diag` are
        // warp-uniform; only an unused half or the diagonal block needs the
        // key's valid queries as a bit mask (applied branch-free: a divergent
        // branch per element costs more than the whole loop).
        float v[32];
        if (pre_s || wait(&bars.s_full[b], (n >> 1) & 1, kSiteKtSoftmaxS, n)) {
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(tbase + 64 * b, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
            if (!valid || diag) {
                const int cut = kk - 32 * ch;  // first valid query of the diagonal block
                const uint32_t vmask =
                    !valid ? 0u : (cut <= 0 ? 0xffffffffu : (cut >= 32 ? 0u : ~0u << cut));
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = (vmask >> i) & 1u ? v[i] : -INFINITY;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = -INFINITY;
        }
        // --- exponent arguments x = s c - M and the vote: does some score pass
        // its query's reference by more than 2^8?  A query without a reference
        // yet (-inf) counts as passing it.  Without a rescale (the usual case)
        // these x are the exponents of P as they stand.
        float x[32];
        float xmax = -INFINITY;
        {
            const float4* m4 = reinterpret_cast<const float4*>(Mq + 32 * ch);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 mm = m4[j];
                const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float mr = mv[u] == -INFINITY ? -3.0e38f : mv[u];
                    x[4 * j + u] = fmaf(v[4 * j + u], cs, -mr);
                }
            }
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                xmax = fmaxf(xmax, fmaxf(fmaxf(x[i], x[i + 1]), fmaxf(x[i + 2], x[i + 3])));
        }
        const bool need = xmax > kKtRescale;
        const bool wneed = __any_sync(0xffffffffu, need);
        if (lane == 0) flags_sm[b * 8 + warp] = wneed ? 1 : 0;
        if (kt_softmax_bar(!ok || *abort)) break;
        bool rescale = false;
        {
            const int4 f0 = reinterpret_cast<const int4*>(flags_sm + b * 8)[0];
            const int4 f1 = reinterpret_cast<const int4*>(flags_sm + b * 8)[1];
            rescale = (f0.x | f0.y | f0.z | f0.w | f1.x | f1.y | f1.z | f1.w) != 0;
        }
        if (rescale) {
            // chunk max per query across the 128 keys, then the new references
            float y[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = v[i] * cs;
            const float ym = kt_reduce_scatter<true>(y, lane);
            red[quarter * 64 + 32 * ch + lane] = ym;
            if (kt_softmax_bar(!ok || *abort)) break;
            if (tid < 64) {
                const float cm = fmaxf(fmaxf(red[tid], red[64 + tid]),
                                       fmaxf(red[128 + tid], red[192 + tid]));
                const float mo = Mq[tid];
                const bool up = cm > -INFINITY && (mo == -INFINITY || cm - mo > kKtRescale);
                const float mn = up ? cm : mo;
                alpha[tid] = up ? ex2(mo - mn) : 1.f;  // 0 while mo is -inf
                Mq[tid] = mn;
            }
            if (kt_softmax_bar(!ok || *abort)) break;
#pragma unroll
            for (int i = 0; i < 32; ++i) l[i] *= alpha[32 * ch + i];
            // O^T holds earlier chunks of this item: rescale once the last O^T has run
            if (!first && wait(&bars.p_free[(n - 1) & 1], ((n - 1) >> 1) & 1, kSiteKtSoftmaxO, n)) {
                tc_fence_after();
                const uint32_t tO = tbase + 128 + 64 * ob;
                uint32_t o[32];
                tmem_ld32(tO, o);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[32 * ch + i]);
                tmem_st32(tO, o);
                tmem_wait_st();
            }
        }
        // --- P^T = 2^(s c - M): the buffer is free once the O^T two chunks back has run
        if (n >= 2 && !pre_pf) wait(&bars.p_free[b], ((n - 2) >> 1) & 1, kSiteKtSoftmaxO, n);
        if (ok) {
            if (rescale) {  // the references moved: exponents against the new ones
                const float4* m4 = reinterpret_cast<const float4*>(Mq + 32 * ch);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 mm = m4[j];
                    const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        x[4 * j + u] =
                            fmaf(v[4 * j + u], cs, -(mv[u] == -INFINITY ? 0.f : mv[u]));
                }
            }
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const uint64_t x2 = f2_pack(x[i], x[i + 1]);
                const uint64_t p2 = ((i >> 1) & 3) == 3 ? exp2_poly2(x2) : f2_pack(ex2(x[i]), ex2(x[i + 1]));
                float p0, p1;
                f2_unpack(p2, p0, p1);
                l[i] += p0;
                l[i + 1] += p1;
                pk[i >> 1] = pack_bf16(p0, p1);
            }
            // row kl of the 128-byte-swizzled P^T tile: 16-byte chunk c at c ^ (kl % 8)
            uint8_t* prow = pbuf + b * KtLayout::kPBytes + kl * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(prow + (((4 * ch + c) ^ (kl & 7)) << 4)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[b]);

        if (!(flags & kKtLast)) continue;
        // --- epilogue of the item: row sums, O / l -> bf16 rows, lse
        const bool have = wait(&bars.o_full[ob], ((qi - 1) >> 1) & 1, kSiteKtSoftmaxO, n);
        const float ls = kt_reduce_scatter<false>(l, lane);
        red[quarter * 64 + 32 * ch + lane] = ls;
        if (kt_softmax_bar(!ok || *abort)) break;
        if (tid < 64) {
            const float L = (red[tid] + red[64 + tid]) + (red[128 + tid] + red[192 + tid]);
            linv[tid] = L > 0.f ? 1.f / L : 0.f;
            if (p.lse)
                p.lse[row0 + tid] = L > 0.f ? (Mq[tid] + __log2f(L)) * 0.6931471805599453f
                                            : -INFINITY;
            Mq[tid] = -INFINITY;  // the next item starts afresh
        }
        if (kt_softmax_bar(!ok || *abort)) break;
        // O^T lanes are head dimensions: transpose through shared memory (P^T
        // buffer 0, free once the item's last O^T has run) into [64][d] rows
        bf16* tile = reinterpret_cast<bf16*>(pbuf);
        if (have) {
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(tbase + 128 + 64 * ob, o);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.o_free[ob]);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                tile[(32 * ch + i) * kKtD + kl] =
                    __float2bfloat16_rn(__uint_as_float(o[i]) * linv[32 * ch + i]);
        }
        if (kt_softmax_bar(!ok || *abort)) break;
        {
            const uint4* src = reinterpret_cast<const uint4*>(tile);
            uint4* dst = reinterpret_cast<uint4*>(p.out + row0 * kKtD);
            for (int i = tid; i < kKtRows * kKtD / 8; i += 256) __stcs(dst + i, src[i]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) l[i] = 0.f;
        // the tile is read before P^T buffer 0 is written again
        if (kt_softmax_bar(!ok || *abort)) break;
    }
}

__global__ void __launch_bounds__(kKtThreads, 1)
    kt_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ KtParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + KtLayout::bar_off);
    KtBars bars;
    {
        uint64_t* q = bar;
        bars.q_full = q++;
        bars.q_empty = q++;
        bars.desc_full = q;
        q += kKtDescRing;
        bars.desc_empty = q;
        q += kKtDescRing;
        bars.k_full = q;
        q += kKtKStages;
        bars.k_empty = q;
        q += kKtKStages;
        bars.v_full = q;
        q += kKtVStages;
        bars.v_empty = q;
        q += kKtVStages;
        bars.s_full = q;
        q += 2;
        bars.p_full = q;
        q += 2;
        bars.p_free = q;
        q += 2;
        bars.o_full = q;
        q += 2;
        bars.o_free = q;
        q += 2;
        bars.drain = q;
    }
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + KtLayout::misc_off);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + KtLayout::misc_off + 4);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        *abort = *reinterpret_cast<volatile unsigned int*>(&g_kt_abort_seq) == p.seq ? 1 : 0;
        mbar_init(bars.q_full, 1);
        mbar_init(bars.q_empty, 1);
        for (int i = 0; i < kKtDescRing; ++i) {
            mbar_init(&bars.desc_full[i], 1);
            mbar_init(&bars.desc_empty[i], 1 + kKtWarpsSoftmax);
        }
        for (int i = 0; i < kKtKStages; ++i) {
            mbar_init(&bars.k_full[i], 1);
            mbar_init(&bars.k_empty[i], 1);
        }
        for (int i = 0; i < kKtVStages; ++i) {
            mbar_init(&bars.v_full[i], 1);
            mbar_init(&bars.v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.p_full[i], kKtWarpsSoftmax);
            mbar_init(&bars.p_free[i], 1);
            mbar_init(&bars.o_full[i], 1);
            mbar_init(&bars.o_free[i], kKtWarpsSoftmax);
        }
        mbar_init(bars.drain, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 64) reinterpret_cast<float*>(sm + KtLayout::m_off)[threadIdx.x] = -INFINITY;
    __syncthreads();
    if (*abort) return;  // an earlier CTA of this launch gave up: skip the work
    if (warp == kKtMmaWarp) {
        tmem_alloc(tmem_slot, kKtTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < kKtWarpsSoftmax) {
        kt_run_softmax(p, sm, bars, abort, tmem);
    } else if (warp == kKtProducerWarp) {
        kt_run_producer(p, &tmQ, &tmK, &tmV, sm, bars, abort);
    } else {
        kt_run_mma(p, sm, bars, abort, tmem);
        tc_fence_before();
    }
    __syncthreads();
    if (warp == kKtMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kKtTmemCols);
    }
}

}  // namespace

bool kt_attn_supported(const AttnLaunch& a) {
    if (a.d != kKtD) return false;
    const int nB = a.N / 64;
    return KtLayout::bytes((nB + 31) / 32) <= 227 * 1024;
}

cudaError_t launch_kt_attn(const AttnLaunch& a, cudaStream_t st) {
    if (a.heads.n == 0) return cudaSuccess;
    if (!kt_attn_supported(a)) return cudaErrorInvalidValue;
    CUtensorMap tmQ, tmK, tmV;
    if (!make_tma_map(&tmQ, a.q, (long long)a.Hq * a.N, kKtD, 64) ||
        !make_tma_map(&tmK, a.k, (long long)a.Hkv * a.N, kKtD, 64) ||
        !make_tma_map(&tmV, a.v, (long long)a.Hkv * a.N, kKtD, 64))
        return cudaErrorInvalidValue;
    static std::atomic<unsigned int> next_seq{0};
    unsigned int seq = ++next_seq;
    KtParams p;
    memset(&p, 0, sizeof(p));
    if (seq == 0) seq = ++next_seq;
    p.seq = seq;
    p.wait_budget = wait_budget_cycles();
    p.k = a.k;
    p.v = a.v;
    p.out = a.out;
    p.lse = a.lse;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.N = a.N;
    p.nB = a.N / 64;
    p.scale_log2 = (float)(a.scale * 1.4426950408889634);
    p.blk_idx = a.blk_idx;
    p.blk_cnt = a.blk_cnt;
    p.topk = a.topk;
    p.err = a.err_count;
    p.heads.n = 0;
    p.ngroups = 0;
    for (int g = 0; g < a.Hkv; ++g) {
        const int start = p.heads.n;
        for (int i = 0; i < a.heads.n; ++i)
            if (kv_head_of(head_qh(a.heads.e[i]), a.Hq, a.Hkv) == g)
                p.heads.e[p.heads.n++] = a.heads.e[i];
        if (p.heads.n > start) p.grp_start[p.ngroups++] = (uint16_t)start;
    }
    p.grp_start[p.ngroups] = (uint16_t)p.heads.n;
    p.n_items = p.heads.n * p.nB;
    const size_t smem = KtLayout::bytes((p.nB + 31) / 32);
    cudaError_t e = cudaFuncSetAttribute(kt_attn_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    const int grid = p.n_items < sms ? p.n_items : sms;
    kt_attn_kernel<<<grid, kKtThreads, smem, st>>>(tmQ, tmK, tmV, p);
    return cudaGetLastError();
}

cudaError_t read_kt_wait_failure(int* out8) {
    int rec[8];
    cudaError_t e = cudaMemcpyFromSymbol(rec, g_kt_wait_fail, sizeof(rec));
    if (e != cudaSuccess) return e;
    for (int i = 0; i < 8; ++i) out8[i] = rec[i];
    const int zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    return cudaMemcpyToSymbol(g_kt_wait_fail, zero, sizeof(zero));
}

}  // namespace minfer

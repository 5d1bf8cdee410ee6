// attn.cu -- dynamic sparse attention on B200 tensor cores (tcgen05 + TMEM,
// operands staged by TMA), one engine for all three MInference patterns.
//
// MInference 1.0 (aifetchly guide, "Technical Deep Dive"): each head runs
// causal flash-style attention with an online softmax over only its selected
// keys: the sink plus local band (A-shape), the chosen 64x64 blocks
// (Block-Sparse), or the gathered vertical columns plus the 64x64 tiles its
// slash diagonals touch (Vertical-Slash), without counting a key twice.  A
// dense head (every causal key) runs on the same engine.
//
// Work item = one query head x one 256-row "super tile" (four 64-row query
// blocks), held as two 128-row slots.  The producer enumerates the item's
// key chunks -- one 64-key block, 64 consecutive keys from any offset (a
// Vertical-Slash head that reads its diagonals as ranges), or up to 64
// gathered vertical columns -- each with a 4-bit mask (one bit per query
// block); a chunk is computed for the slots whose bits it carries.  Each
// softmax row turns the descriptor into a 64-bit mask of the keys it takes
// (causal limit, A-shape sink and window, gathered columns, a range chunk's
// keys per query block); a warp whose query block does not take the chunk
// writes zero P rows and skips the exponentials, and chunks that every row
// takes whole are flagged so that they skip the mask step.
//   warps 0-3  softmax, slot 0 (TMEM lanes 0-127 = rows 0-127)
//   warps 4-7  softmax, slot 1 (rows 128-255)
//   warp 8     producer: chunk list + TMA loads (cp.async gathers), 4 deep
//   warps 9-10 MMA issuers, one per slot: S = Q K^T (SS form), O += P V (TS form)
// Each slot double-buffers S in TMEM, so the tensor core computes S(n+1)
// while the softmax works on S(n); O += P(n) V(n) follows once P(n) is
// ready.  A slot's softmax therefore runs back to back, whether or not the
// other slot needs the same chunk.  The exponentials run on MUFU, a quarter
// of them on the FMA pipe (exp2_poly.h).
//
// TMEM (512 columns): slot x owns [256x, 256x+256): S buffers 0 and 1 at
// +0 and +64 (64 columns each; P, bf16 pairs, reuses the first 32), O at
// +128 (d columns).
#include <atomic>
#include <cfloat>
#include <cstring>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "softmax_math.cuh"

namespace minfer {

namespace {

// 3 warpgroups: two softmax warpgroups (one per 128-row slot) and one for the
// producer warp, the two MMA warps and one idle warp.  Launched at 168 registers
// per thread (65536 / 384, rounded down to 8); the softmax warpgroups then
// take 208 and the third 88: 2*128*208 + 128*88 = 384*168.
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;  // and 10: one MMA warp per slot
constexpr int kSoftmaxRegs = 208;
constexpr int kControlRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168,
              "register split exceeds the launch budget");
constexpr int kSoftmaxThreads = 256;
constexpr int kChunkKeys = 64;            // keys per chunk (one 64-key block)
constexpr int kStages = 4;                // K and V ring depth (chunks)
constexpr int kDescRing = 8;              // chunk descriptors in flight
constexpr int kQPanel = 128 * 128;        // 128 rows x one 64-column (128-byte) panel
constexpr int kKVPanel = kChunkKeys * 128;  // 64 rows x one panel
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by >8

enum : int { kChunkNone = 0, kChunkBlock = 1, kChunkGather = 2, kChunkRange = 3 };
// info flag: every row of the super tile takes every key of the chunk (a block
// below the diagonal that all four query blocks take, outside A-shape)
constexpr int kChunkWhole = 1 << 9;

struct ChunkDesc {
    int info;  // type | need << 4 | last << 8 | whole << 9 (see kChunkWhole)
    int type, last, need, ncols;
    int b, m;  // block chunks: key block and its 4-bit query-block mask; ranges: first key
    int cols[kChunkKeys];      // gathers: the columns, ascending
    uint64_t qmask[4];         // gathers and ranges: per query block, the keys it takes
};

struct GatherHeld {
    int cols[kChunkKeys];
    uint8_t cm[kChunkKeys];
};

// Sequence number of the last launch in which a CTA gave up waiting; later
// CTAs of that launch exit at once instead of timing out one by one.
__device__ unsigned int g_abort_seq = 0;

// First wait that gave up since the record was last read:
// {launch seq, site, block, thread, chunk, parity, 0, 0}; site 0 = none.
__device__ int g_wait_fail[8];

enum : int {
    kSiteProducerEmpty = 1,
    kSiteMmaQ = 2,
    kSiteMmaFull = 3,
    kSiteMmaP = 4,
    kSiteSoftmaxFull = 5,
    kSiteSoftmaxS = 6,
    kSiteSoftmaxO = 7
};

__device__ void record_wait_failure(unsigned int seq, int site, int group, int parity) {
    if (atomicCAS(&g_wait_fail[1], 0, site) == 0) {
        g_wait_fail[0] = (int)seq;
        g_wait_fail[2] = (int)blockIdx.x;
        g_wait_fail[3] = (int)threadIdx.x;
        g_wait_fail[4] = group;
        g_wait_fail[5] = parity;
        __threadfence();
    }
}

struct AttnParams {
    unsigned int seq;  // launch sequence number (never 0)
    long long wait_budget;  // cycles an abortable wait may take before it gives up
    const bf16* k;
    const bf16* v;
    bf16* out;
    float* lse;
    int Hq, Hkv, N, nB, n_super;
    float scale_log2;
    const uint32_t* dbits;
    const uint64_t* rwords;
    int nBw;
    const int32_t* vlist;
    const int32_t* vcnt;
    int vcap;
    const int32_t* blk_idx;
    const int32_t* blk_cnt;
    int topk;
    int2 asw[MI_MAX_HEADS];  // A-shape heads, by A-shape position: (sink, window)
    int32_t* err;
    HeadList heads;  // sorted by KV head
    int ngroups;     // KV heads present in `heads`
    uint16_t grp_start[MI_MAX_HEADS + 1];  // heads of KV group i: [grp_start[i], grp_start[i+1])
};

template <int D>
struct Layout {
    static constexpr int kQBytes = 128 * D * 2;          // one slot of Q
    static constexpr int kKVBytes = kChunkKeys * D * 2;  // one K or V stage
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + 2 * kQBytes;
    static constexpr int v_off = k_off + kStages * kKVBytes;
    static constexpr int desc_off = v_off + kStages * kKVBytes;
    static constexpr int held_off = desc_off + kDescRing * (int)sizeof(ChunkDesc);
    static constexpr int bar_off = (held_off + (int)sizeof(GatherHeld) + 15) & ~15;
    static constexpr int kNumBars = 1 + 2 * kDescRing + 3 * kStages + 12 + 2;
    static constexpr int misc_off = bar_off + kNumBars * 8;
    static constexpr int patmap_off = misc_off + 16;
    static size_t bytes(int patmap_words) {
        size_t b = (size_t)patmap_off + (size_t)patmap_words * 4 + 1024;  // +1024: base alignment
        // d = 64 is small enough for two CTAs per SM, but TMEM holds one: ask for enough
        // shared memory that the SM schedules one at a time.
        return b < 120 * 1024 ? 120 * 1024 : b;
    }
};

// Pipeline barriers.  Chunk g (in publication order) uses descriptor slot
// g % 8 and K/V stage g % 4.  kv_full completes once both tiles have landed
// (the end marker completes it without data); since the producer writes a
// chunk's descriptor before it arms kv_full, the MMA issuer needs only that
// barrier.  K is released once the S of the chunk has run, V once every P V
// that reads it has run.
// Slot x's n-th chunk uses S buffer n % 2: s_full / p_full / pv_done are
// per slot and per buffer, so no waiter can ever be lapped by two phases.
struct Bars {
    uint64_t* q_full;
    uint64_t* desc_full;   // [8] producer -> MMA, softmax
    uint64_t* desc_empty;  // [8] MMA + 256 softmax threads -> producer
    uint64_t* kv_full;     // [4] TMA / gather -> MMA
    uint64_t* k_empty;     // [4] MMA (after S) -> producer
    uint64_t* v_empty;     // [4] MMA (after P V) -> producer
    uint64_t* s_full;      // [2 slots][2 buffers] S ready in TMEM
    uint64_t* p_full;      // [2][2] P written to TMEM (128 softmax threads)
    uint64_t* pv_done;     // [2][2] O += P V of that buffer has run
    uint64_t* drain;       // [2] per MMA warp: all its MMAs have run
};

__device__ __forceinline__ void set_abort(volatile int* abort, int32_t* err, unsigned int seq) {
    *abort = 1;
    if (err) atomicOr(err, 1 << 30);
    atomicExch(&g_abort_seq, seq);
}

// ------------------------------------------------------------- producer
template <int D>
struct Producer {
    using L = Layout<D>;
    const AttnParams& p;
    const CUtensorMap* tmK;
    const CUtensorMap* tmV;
    uint8_t* sm;
    Bars bars;
    volatile int* abort;
    ChunkDesc* desc;
    GatherHeld* held;
    int g;        // KV head
    int pub = 0;  // descriptors published
    int nkv = 0;  // K/V stages armed (one per descriptor)
    int lane;
    bool ok = true;

    // lane 0 waits, the warp follows its verdict
    __device__ bool wait(uint64_t* bar, int parity, int count) {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar, parity, abort, p.wait_budget);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) {
            if (lane == 0) {
                if (!*abort) record_wait_failure(p.seq, kSiteProducerEmpty, count, parity);
                set_abort(abort, p.err, p.seq);
            }
            ok = false;
        }
        return w;
    }
    // A wait costs about 200 cycles even on a long-completed phase, and the
    // next chunk needs three (its descriptor slot, K stage and V stage free).
    // One non-blocking probe across lanes 0-2 checks all three; when they have
    // completed, acquire_desc and acquire_kv skip their waits for this chunk.
    bool free_known = false;
    __device__ void probe_next() {
        uint64_t* b = bars.q_full;
        uint32_t par = 0;
        bool live = false;
        if (lane == 0 && pub >= kDescRing) {
            b = &bars.desc_empty[pub % kDescRing];
            par = ((pub / kDescRing) - 1) & 1;
            live = true;
        } else if ((lane == 1 || lane == 2) && nkv >= kStages) {
            b = lane == 1 ? &bars.k_empty[nkv % kStages] : &bars.v_empty[nkv % kStages];
            par = ((nkv / kStages) - 1) & 1;
            live = true;
        }
        const bool hit = mbar_test_wait(b, par) || !live;
        free_known = __all_sync(0xffffffffu, hit);
    }
    __device__ ChunkDesc* acquire_desc() {
        const int i = pub % kDescRing;
        if (pub >= kDescRing && !free_known &&
            !wait(&bars.desc_empty[i], ((pub / kDescRing) - 1) & 1, pub))
            return nullptr;
        return &desc[i];
    }
    __device__ void publish_desc() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.desc_full[pub % kDescRing]);
        ++pub;
    }
    // the stage of the next descriptor, once its previous K and V are released
    __device__ bool acquire_kv(int& s) {
        s = nkv % kStages;
        const bool known = free_known;  // good for this chunk only
        free_known = false;
        if (nkv < kStages || known) return true;
        const int par = ((nkv / kStages) - 1) & 1;
        return wait(&bars.k_empty[s], par, nkv) && wait(&bars.v_empty[s], par, nkv);
    }

    // one 64-key block with its query-block mask; `whole`: see kChunkWhole
    __device__ void block(int b, int m, bool whole) {
        if (!ok) return;
        probe_next();
        ChunkDesc* d = acquire_desc();
        if (!d) return;
        if (lane == 0) {
            const int need = ((m & 0x3) ? 1 : 0) | ((m & 0xC) ? 2 : 0);
            d->info = kChunkBlock | (need << 4) | (whole ? kChunkWhole : 0);
            d->type = kChunkBlock;
            d->last = 0;
            d->need = need;
            d->ncols = 0;
            d->b = b;
            d->m = m;
        }
        publish_desc();
        int st;
        if (!acquire_kv(st)) return;
        if (lane == 0) {
            const int row = g * p.N + kChunkKeys * b;
            mbar_arrive_expect_tx(&bars.kv_full[st], 2 * L::kKVBytes);
            uint8_t* kd = sm + L::k_off + st * L::kKVBytes;
            uint8_t* vd = sm + L::v_off + st * L::kKVBytes;
            // every query block of the KV head reads these keys again: keep them in L2
            const uint64_t pol = l2_policy_evict_last();
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d_hint(kd + pn * kKVPanel, tmK, 64 * pn, row, &bars.kv_full[st], pol);
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d_hint(vd + pn * kKVPanel, tmV, 64 * pn, row, &bars.kv_full[st], pol);
        }
        __syncwarp();
        ++nkv;
    }

    // 64 consecutive keys from key c0 (any offset; TMA rows past the KV head's
    // end are another head's or zero fill, and no query block takes them) with
    // the keys each query block takes
    __device__ void window(int c0, const uint64_t (&qm)[4]) {
        if (!ok) return;
        probe_next();
        ChunkDesc* d = acquire_desc();
        if (!d) return;
        if (lane == 0) {
            const int need = (qm[0] | qm[1] ? 1 : 0) | (qm[2] | qm[3] ? 2 : 0);
            d->info = kChunkRange | (need << 4);
            d->type = kChunkRange;
            d->last = 0;
            d->need = need;
            d->ncols = 0;
            d->b = c0;
            d->m = 0;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) d->qmask[qq] = qm[qq];
        }
        publish_desc();
        int st;
        if (!acquire_kv(st)) return;
        if (lane == 0) {
            const int row = g * p.N + c0;
            mbar_arrive_expect_tx(&bars.kv_full[st], 2 * L::kKVBytes);
            uint8_t* kd = sm + L::k_off + st * L::kKVBytes;
            uint8_t* vd = sm + L::v_off + st * L::kKVBytes;
            const uint64_t pol = l2_policy_evict_last();
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d_hint(kd + pn * kKVPanel, tmK, 64 * pn, row, &bars.kv_full[st], pol);
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d_hint(vd + pn * kKVPanel, tmV, 64 * pn, row, &bars.kv_full[st], pol);
        }
        __syncwarp();
        ++nkv;
    }

    // up to 64 gathered columns
    __device__ void gather(int n) {
        if (!ok) return;
        probe_next();
        ChunkDesc* d = acquire_desc();
        if (!d) return;
        // lane l holds columns l and l + 32; unused entries repeat a real column
        const int cm0 = lane < n ? held->cm[lane] : 0;
        const int cm1 = lane + 32 < n ? held->cm[lane + 32] : 0;
        d->cols[lane] = lane < n ? held->cols[lane] : held->cols[0];
        d->cols[lane + 32] = lane + 32 < n ? held->cols[lane + 32] : held->cols[0];
        uint64_t qm[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
            qm[qq] = (uint64_t)__ballot_sync(0xffffffffu, (cm0 >> qq) & 1) |
                     ((uint64_t)__ballot_sync(0xffffffffu, (cm1 >> qq) & 1) << 32);
        const int need = (qm[0] | qm[1] ? 1 : 0) | (qm[2] | qm[3] ? 2 : 0);
        if (lane == 0) {
            d->info = kChunkGather | (need << 4);
            d->type = kChunkGather;
            d->last = 0;
            d->need = need;
            d->ncols = n;
            d->b = -1;
            d->m = 0;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) d->qmask[qq] = qm[qq];
        }
        publish_desc();
        int st;
        if (!acquire_kv(st)) return;
        uint8_t* kd = sm + L::k_off + st * L::kKVBytes;
        uint8_t* vd = sm + L::v_off + st * L::kKVBytes;
        constexpr int kChunks = D / 8;  // 16-byte chunks per row
        const bf16* kb = p.k + (size_t)g * p.N * D;
        const bf16* vb = p.v + (size_t)g * p.N * D;
        for (int idx = lane; idx < kChunkKeys * kChunks; idx += 32) {
            const int r = idx / kChunks, c = idx % kChunks;
            const size_t src = (size_t)d->cols[r] * D + c * 8;
            const int dst = (c >> 3) * kKVPanel + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            cp_async_16(kd + dst, kb + src);
            cp_async_16(vd + dst, vb + src);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.kv_full[st]);
        ++nkv;
    }

    // end marker: a descriptor with no keys, signalled through kv_full like the rest
    __device__ void finish() {
        if (!ok) return;
        ChunkDesc* d = acquire_desc();
        if (!d) return;
        if (lane == 0) {
            d->info = kChunkNone | (1 << 8);
            d->type = kChunkNone;
            d->last = 1;
            d->need = 0;
            d->ncols = 0;
        }
        publish_desc();
        int st;
        if (!acquire_kv(st)) return;
        if (lane == 0) mbar_arrive(&bars.kv_full[st]);
        __syncwarp();
        ++nkv;
    }

    // Wait (bounded) until every copy this warp started has landed, so that
    // no TMA write can reach shared memory after the CTA exits.
    __device__ void drain() {
        if (lane != 0) return;
        for (int u = nkv - kStages; u < nkv; ++u)
            if (u >= 0) mbar_wait_budget(&bars.kv_full[u % kStages], (u / kStages) & 1);
    }
};

__device__ __forceinline__ bool bit_of(const uint32_t* bits, int i) {
    return (bits[i >> 5] >> (i & 31)) & 1u;
}

template <int D>
__device__ void run_producer(const AttnParams& p, const CUtensorMap* tmQ, const CUtensorMap* tmK,
                             const CUtensorMap* tmV, uint8_t* sm, const Bars& bars,
                             volatile int* abort, uint32_t* patmap, int pos, int T) {
    using L = Layout<D>;
    const int lane = threadIdx.x & 31;
    const uint32_t e = p.heads.e[pos];
    const int qh = head_qh(e), pattern = head_pattern(e), pidx = head_pidx(e);
    // Vertical-Slash head whose diagonals select unaligned 64-key ranges
    const bool ranges = pattern == MI_PATTERN_VS && head_ranges(e);
    const uint64_t* rw = ranges ? p.rwords + (size_t)pidx * p.nB : nullptr;
    const int g = kv_head_of(qh, p.Hq, p.Hkv);
    const int qb0 = 4 * T;
    const int nqb = min(4, p.nB - qb0);
    const int bmax = min(qb0 + 3, p.nB - 1);

    if (lane == 0) {
        prefetch_tmap(tmQ);
        prefetch_tmap(tmK);
        prefetch_tmap(tmV);
        mbar_arrive_expect_tx(bars.q_full, 2 * L::kQBytes);
        const uint64_t once = l2_policy_evict_first();  // this CTA's rows, read once
        for (int x = 0; x < 2; ++x)
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d_hint(sm + L::q_off + x * L::kQBytes + pn * kQPanel, tmQ, 64 * pn,
                                 qh * p.N + 256 * T + 128 * x, bars.q_full, once);
    }

    // per-pattern block map
    if (pattern == MI_PATTERN_VS && !ranges) {
        const uint32_t* src = p.dbits + (size_t)pidx * p.nBw;
        for (int w = lane; w < p.nBw; w += 32) patmap[w] = src[w];
    } else if (pattern == MI_PATTERN_BS) {
        const int nwords = (bmax + 8) / 8;  // 8 nibbles per word
        for (int w = lane; w < nwords; w += 32) patmap[w] = 0;
        __syncwarp();
        for (int qq = 0; qq < nqb; ++qq) {
            const int qb = qb0 + qq;
            const int cnt = min(p.blk_cnt[(size_t)pidx * p.nB + qb], p.topk);
            const int32_t* lst = p.blk_idx + ((size_t)pidx * p.nB + qb) * p.topk;
            for (int t = lane; t < cnt; t += 32) {
                const int bk = lst[t];
                if (bk == -1) continue;  // padding
                if (bk < 0 || bk > qb) {
                    if (p.err) atomicAdd(p.err, 1);
                    continue;
                }
                atomicOr(&patmap[bk >> 3], (1u << qq) << ((bk & 7) * 4));
            }
        }
    }
    __syncwarp();

    Producer<D> pr{p, tmK, tmV, sm, bars, abort,
                   reinterpret_cast<ChunkDesc*>(sm + L::desc_off),
                   reinterpret_cast<GatherHeld*>(sm + L::held_off), g};
    pr.lane = lane;

    // --- ranges: the keys the super tile's query blocks take, as 64-key windows
    // cut from the first key not yet covered.  Query block qb takes key u of
    // block b iff bit u % 64 of rw[qb - b] is set, so lane `lane` holds, for
    // its block b and each query block, the words of blocks b and b + 1; a
    // window starting at bit s of block b takes bits s.. of the first and
    // bits ..s-1 of the second.  Each 64-key word starts at most one window.
    // (Windows cut per slot instead, from each slot's own keys, double the
    // chunk stream and measured slower.)
    if (ranges) {
        long long cursor = 0;  // keys below it lie in an emitted window
        for (int base = 0; base <= bmax && pr.ok; base += 32) {
            const int b = base + lane;
            uint64_t lo[4], hi[4], nb = 0;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int dl = qb0 + qq - b;
                lo[qq] = (qq < nqb && b <= bmax && dl >= 0) ? rw[dl] : 0ull;
                hi[qq] = (qq < nqb && b + 1 <= bmax && dl >= 1) ? rw[dl - 1] : 0ull;
                nb |= lo[qq];
            }
            unsigned bal = __ballot_sync(0xffffffffu, nb != 0ull);
            while (bal && pr.ok) {
                const int src = __ffs(bal) - 1;
                bal &= bal - 1;
                const long long kb = 64LL * (base + src);
                uint64_t bits = __shfl_sync(0xffffffffu, nb, src);
                const long long c = cursor - kb;
                if (c >= 64) bits = 0ull;
                else if (c > 0) bits &= ~0ull << c;
                if (!bits) continue;  // covered by the window before
                const int sft = __ffsll((long long)bits) - 1;
                uint64_t qm[4];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const uint64_t a = __shfl_sync(0xffffffffu, lo[qq], src);
                    const uint64_t h = __shfl_sync(0xffffffffu, hi[qq], src);
                    qm[qq] = (a >> sft) | (sft ? h << (64 - sft) : 0ull);
                }
                pr.window((int)(kb + sft), qm);
                cursor = kb + sft + 64;
            }
        }
    }

    // --- 64-key blocks, ascending, one chunk each
    for (int base = 0; base <= bmax && pr.ok && !ranges; base += 32) {
        const int b = base + lane;
        int m = 0;
        if (b <= bmax) {
            if (pattern == MI_PATTERN_VS) {
                for (int qq = 0; qq < nqb; ++qq) {
                    const int delta = qb0 + qq - b;
                    if (delta >= 0 && bit_of(patmap, delta)) m |= 1 << qq;
                }
            } else if (pattern == MI_PATTERN_BS) {
                m = (patmap[b >> 3] >> ((b & 7) * 4)) & 0xF;
            } else if (pattern == MI_PATTERN_DENSE) {
                for (int qq = 0; qq < nqb; ++qq)  // every causal block
                    if (b <= qb0 + qq) m |= 1 << qq;
            } else {
                for (int qq = 0; qq < nqb; ++qq) {
                    const int qb = qb0 + qq;
                    if (b <= qb && (64 * b < p.asw[pidx].x || 64 * (qb - b) - 63 < p.asw[pidx].y))
                        m |= 1 << qq;
                }
            }
        }
        unsigned bal = __ballot_sync(0xffffffffu, m != 0);
        while (bal) {
            const int src = __ffs(bal) - 1;
            bal &= bal - 1;
            const int mm = __shfl_sync(0xffffffffu, m, src);
            pr.block(base + src, mm,
                     mm == 0xF && base + src < qb0 && pattern != MI_PATTERN_ASHAPE);
        }
    }

    // --- Vertical-Slash: gathered columns not already inside a computed block
    if (pattern == MI_PATTERN_VS && pr.ok) {
        const int vc = p.vcnt[pidx];
        const int32_t* vl = p.vlist + (size_t)pidx * p.vcap;
        const long long rlast = min(256LL * T + 255, (long long)p.N - 1);
        GatherHeld* held = pr.held;
        int n_held = 0;
        for (int base = 0; base < vc && pr.ok; base += 32) {
            const int t = base + lane;
            const int j = t < vc ? vl[t] : 0x7fffffff;
            int m = 0;
            if (j <= rlast) {
                for (int qq = 0; qq < nqb; ++qq) {
                    const int qb = qb0 + qq;
                    if (j < 64 * (qb + 1)) {
                        const int delta = qb - (j >> 6);
                        const bool covered =
                            ranges ? ((rw[delta] >> (j & 63)) & 1ull) != 0 : bit_of(patmap, delta);
                        if (!covered) m |= 1 << qq;
                    }
                }
            }
            const unsigned bal = __ballot_sync(0xffffffffu, m != 0);
            const int rank = __popc(bal & ((1u << lane) - 1u));
            const int navail = __popc(bal);
            const int take = min(navail, kChunkKeys - n_held);
            if (m && rank < take) {
                held->cols[n_held + rank] = j;
                held->cm[n_held + rank] = (uint8_t)m;
            }
            __syncwarp();
            n_held += take;
            if (n_held == kChunkKeys) {
                pr.gather(n_held);
                n_held = 0;
                if (m && rank >= take) {
                    held->cols[rank - take] = j;
                    held->cm[rank - take] = (uint8_t)m;
                }
                __syncwarp();
                n_held = navail - take;
            }
            if (__any_sync(0xffffffffu, j > rlast)) break;  // the list is sorted
        }
        if (n_held > 0) pr.gather(n_held);
    }
    pr.finish();

    // make sure Q and every started load have landed before the CTA can exit
    if (lane == 0) mbar_wait_budget(bars.q_full, 0);
    pr.drain();
}

// ------------------------------------------------------------- MMA issuers
// One MMA warp per slot (warp 9 for rows 0-127, warp 10 for rows 128-255):
// each issues only its own slot's S and P V, so the two warps' bookkeeping
// overlaps the other's MMAs in the tensor pipe.  They share the K/V stages
// and the descriptors, which are released once both have passed a chunk
// (k_empty, v_empty and the MMA share of desc_empty count two arrivals; a
// warp can see chunk g+4's K/V only after both released chunk g, so no
// arrival can fall into the wrong phase).
//
// The warp runs its loop converged, with every MMA operand derived from
// lane-0 broadcasts and ballots, so the compiler keeps the operands in
// uniform registers (one it cannot prove uniform is moved there on every
// issue, which is slower than the tensor pipe); elect.sync inside the issue
// instructions picks the issuing lane.  An mbarrier probe costs about 200
// cycles even on a completed phase, so each round probes, in one
// non-blocking test_wait, the next chunk's K/V (lane 0; once seen it stays
// landed until used) and the P of the slot's oldest chunk still waiting for
// O += P V (lane 1), and then issues what is ready:
//   O += P V for that chunk, then
//   S = Q K^T of the next chunk (if the slot needs it) into the slot's other
//   S buffer, once at most one chunk waits for P V (the buffer S overwrites
//   holds the P of the chunk before last, which its P V must have read
//   first; one thread's MMAs run in issue order).
// So the tensor core computes S(n+1) while the softmax works on S(n).
template <int D>
__device__ void run_mma(uint8_t* sm, const Bars& bars, volatile int* abort, int32_t* err,
                        unsigned int seq, long long budget, uint32_t tmem, int x) {
    using L = Layout<D>;
    const int lane = threadIdx.x & 31;
    const uint32_t idS = idesc_bf16_f32(128, kChunkKeys, false);
    const uint32_t idO = idesc_bf16_f32(128, D, true);
    tmem = __shfl_sync(0xffffffffu, tmem, 0);
    x = __shfl_sync(0xffffffffu, x, 0);
    const uint32_t tSlot = tmem + 256 * x;
    const uint32_t q_addr = __shfl_sync(0xffffffffu, smem_u32(sm + L::q_off + x * L::kQBytes), 0);
    const uint32_t k_addr = __shfl_sync(0xffffffffu, smem_u32(sm + L::k_off), 0);
    const uint32_t v_addr = __shfl_sync(0xffffffffu, smem_u32(sm + L::v_off), 0);
    const ChunkDesc* desc = reinterpret_cast<const ChunkDesc*>(sm + L::desc_off);
    uint64_t* const p_full = bars.p_full + 2 * x;
    uint64_t* const s_full = bars.s_full + 2 * x;
    uint64_t* const pv_done = bars.pv_done + 2 * x;

    bool ok = true;
    {
        bool w = true;
        if (lane == 0) w = mbar_wait(bars.q_full, 0, abort, budget);
        ok = __shfl_sync(0xffffffffu, w, 0);
        if (!ok && lane == 0 && !*abort) record_wait_failure(seq, kSiteMmaQ, 0, x);
    }

    int g = 0;              // next chunk to read
    bool done = false;      // end marker read
    bool kv_ready = false;  // chunk g's K/V seen landed
    int nS = 0;             // S issued
    int cnt = 0;            // chunks whose P V is still to issue (0..2)
    int pc0 = 0, pc1 = 0;   // the oldest of them, the newer one
    unsigned idle = 0;      // rounds that found nothing to do
    long long t_last = clock64();
    while (ok && !(done && cnt == 0)) {
        const bool want_kv = !done && !kv_ready;
        uint64_t* pb = bars.q_full;  // completed: a harmless target for idle lanes
        uint32_t par = 0;
        bool live = false;
        if (lane == 0 && want_kv) {
            pb = &bars.kv_full[g % kStages];
            par = (g / kStages) & 1;
            live = true;
        } else if (lane == 1 && cnt > 0) {
            const int sidx = nS - cnt;
            pb = &p_full[sidx & 1];
            par = (sidx >> 1) & 1;
            live = true;
        }
        const bool hit = mbar_test_wait(pb, par) && live;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        kv_ready |= (bal & 1u) != 0;
        const bool hp = (bal >> 1) & 1u;
        const bool can_s = kv_ready && cnt - (hp ? 1 : 0) <= 1;
        if (!(hp || can_s)) {
            if ((++idle & 15) != 0) continue;
            const bool give_up = *abort || clock64() - t_last > budget;
            if (__any_sync(0xffffffffu, give_up)) {
                if (lane == 0 && !*abort)
                    record_wait_failure(seq, want_kv ? kSiteMmaFull : kSiteMmaP, g, cnt | x << 4);
                ok = false;
            }
            continue;
        }
        t_last = clock64();
        tc_fence_after();
        if (hp) {  // O += P V for the oldest pending chunk
            const int sidx = nS - cnt, st = pc0 % kStages;
            const uint32_t tP = tSlot + 64 * (sidx & 1);
#pragma unroll
            for (int kk = 0; kk < kChunkKeys / 16; ++kk) {
                const uint64_t bdesc =
                    sw128_desc(v_addr + st * L::kKVBytes + kk * 2048, kKVPanel, 1024);
                mma_ts_warp(tSlot + 128, tP + kk * 8, bdesc, idO, (sidx > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_warp(&pv_done[sidx & 1]);
            mma_commit_warp(&bars.v_empty[st]);  // this slot is done with the V stage
            pc0 = pc1;
            --cnt;
        }
        if (can_s) {  // the next chunk (its descriptor was written before kv_full was armed)
            kv_ready = false;
            const int di = g % kDescRing, s = g % kStages;
            const int info = __shfl_sync(0xffffffffu, desc[di].info, 0);
            const int type = info & 0xF, last = (info >> 8) & 1;
            if ((info >> (4 + x)) & 1) {
                const uint32_t tS = tSlot + 64 * (nS & 1);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int pn = kk >> 2, off = (kk & 3) * 32;
                    const uint64_t adesc = sw128_desc(q_addr + pn * kQPanel + off, 16, 1024);
                    const uint64_t bdesc =
                        sw128_desc(k_addr + s * L::kKVBytes + pn * kKVPanel + off, 16, 1024);
                    mma_ss_warp(tS, adesc, bdesc, idS, kk > 0 ? 1u : 0u);
                }
                mma_commit_warp(&s_full[nS & 1]);
                mma_commit_warp(&bars.k_empty[s]);  // K free once both slots' S have run
                if (cnt == 0) pc0 = g;
                else pc1 = g;
                ++cnt;
                ++nS;
            } else if (type != kChunkNone) {
                // this slot skips the chunk: release its share of the stage now
                mbar_arrive_warp(&bars.k_empty[s]);
                mbar_arrive_warp(&bars.v_empty[s]);
            }
            mbar_arrive_warp(&bars.desc_empty[di]);
            if (last) done = true;
            else ++g;
        }
    }
    if (!ok && lane == 0) set_abort(abort, err, seq);
    // every MMA of this warp must have finished before TMEM is released
    mma_commit_warp(&bars.drain[x]);
    if (lane == 0) mbar_wait_budget(&bars.drain[x], 0);
    __syncwarp();
}

// ------------------------------------------------------------- softmax
template <int D>
__device__ void run_softmax(const AttnParams& p, uint8_t* sm, const Bars& bars,
                            volatile int* abort, uint32_t tmem, int pos, int T) {
    using L = Layout<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int x = warp >> 2, lg = warp & 3;
    const int t = lg * 32 + lane;         // row within the slot = TMEM lane
    const int rloc = 128 * x + t;         // row within the super tile
    const int qi = rloc >> 6;             // query block within the super tile
    const long long i = 256LL * T + rloc; // global row
    const uint32_t e = p.heads.e[pos];
    const int qh = head_qh(e), pattern = head_pattern(e);
    const bool ashape = pattern == MI_PATTERN_ASHAPE;
    const int sink = p.asw[head_pidx(e)].x, window = p.asw[head_pidx(e)].y;  // A-shape only
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    // warp-uniform TMEM address (tcgen05.ld/st take it from a uniform register)
    const uint32_t tSlot = __shfl_sync(0xffffffffu, tmem + 256 * x + lane_off, 0);
    const uint32_t tO = tSlot + 128;
    const ChunkDesc* desc = reinterpret_cast<const ChunkDesc*>(sm + L::desc_off);
    const float cs = p.scale_log2;

    float m = -INFINITY, l = 0.f;
    int n = 0;  // chunks this slot has processed
    bool ok = true;
    for (int g = 0;; ++g) {
        const int di = g % kDescRing;
        const int dpar = (g / kDescRing) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.desc_full[di], dpar, abort, p.wait_budget))) {
            if (!*abort) record_wait_failure(p.seq, kSiteSoftmaxFull, g, dpar);
            ok = false;
            break;
        }
        const ChunkDesc& d = desc[di];
        const int type = d.type, last = d.last;
        if (type != kChunkNone && ((d.need >> x) & 1)) {
            // The chunk's keys this row takes, one bit per column (known from the
            // descriptor, so worked out while S is still being computed).  A
            // warp's 32 rows lie in one 64-row query block, so a chunk that block
            // does not take is dropped by the whole warp at once (P rows of zeros).
            uint64_t keep = ~0ull;
            unsigned kv = 1u;  // bit 0: some row of the warp takes the chunk; bit 1: some row drops a key
            if (d.info & kChunkWhole) {
            } else if (type == kChunkRange) {
                keep = d.qmask[qi] & low_bits(i - (long long)d.b + 1);  // and causal
            } else if (type == kChunkBlock) {
                keep = 0;
                if ((d.m >> qi) & 1) {
                    const long long j0 = 64LL * d.b;
                    keep = low_bits(i - j0 + 1);  // causal: columns <= i
                    if (ashape)  // sink (j < sink) or local window (i - j < window)
                        keep &= low_bits(sink - j0) | ~low_bits(i - j0 - window + 1);
                }
            } else {
                // gathered columns ascend: those <= i form a prefix
                int lo = 0, hi = d.ncols;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if ((long long)d.cols[mid] <= i) lo = mid + 1;
                    else hi = mid;
                }
                keep = d.qmask[qi] & low_bits(lo);
            }
            if (!(d.info & kChunkWhole))
                kv = __reduce_or_sync(0xffffffffu,
                                      (keep != 0 ? 1u : 0u) | (keep != ~0ull ? 2u : 0u));
            const int b = n & 1;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&bars.s_full[2 * x + b], (n >> 1) & 1, abort, p.wait_budget))) {
                if (!*abort) record_wait_failure(p.seq, kSiteSoftmaxS, g, (n >> 1) & 1);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = __shfl_sync(0xffffffffu, tSlot + 64 * b, 0);
            if (!(kv & 1u)) {
                uint32_t z[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) z[u] = 0u;
                tmem_st32(tS, z);
            } else {
                float v[kChunkKeys];
                {
                    uint32_t r[32];
                    tmem_ld32(tS, r);
#pragma unroll
                    for (int u = 0; u < 32; ++u) v[u] = __uint_as_float(r[u]);
                    tmem_ld32(tS + 32, r);
#pragma unroll
                    for (int u = 0; u < 32; ++u) v[32 + u] = __uint_as_float(r[u]);
                }
                if (kv & 2u) {
#pragma unroll
                    for (int c = 0; c < kChunkKeys; ++c)
                        if (!((keep >> c) & 1)) v[c] = -INFINITY;
                }
                // raw scores: the scale (> 0) commutes with the max and is folded into
                // the exponent below (one packed FFMA per pair)
                float mq[2] = {fmaxf(v[0], v[1]), fmaxf(v[2], v[3])};
#pragma unroll
                for (int c = 4; c < kChunkKeys; c += 4) {
                    mq[0] = fmax3(mq[0], v[c], v[c + 1]);
                    mq[1] = fmax3(mq[1], v[c + 2], v[c + 3]);
                }
                const float mx = fmaxf(mq[0], mq[1]) * cs;
                // Lazy rescale: a row moves its reference max only when the max grew by
                // more than 2^8 (p <= 256 otherwise, exact after the final 1/l).  O may be
                // rescaled only once the slot's previous O += P V has run.  The TMEM
                // accesses are .sync.aligned, so the whole warp takes the branch
                // together; rows that do not need it scale by 1.
                const bool want = mx > m + kRescaleThreshold;
                if (__any_sync(0xffffffffu, want)) {
                    const float alpha = want ? ex2(m - mx) : 1.f;  // 0 while m is -inf
                    if (n > 0) {
                        const int pb = (n - 1) & 1;
                        if (!__all_sync(0xffffffffu, mbar_wait(&bars.pv_done[2 * x + pb],
                                                               ((n - 1) >> 1) & 1, abort,
                                                               p.wait_budget))) {
                            if (!*abort) record_wait_failure(p.seq, kSiteSoftmaxO, g, 0);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        uint32_t o[32];
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            tmem_ld32(tO + 32 * c, o);
#pragma unroll
                            for (int u = 0; u < 32; ++u)
                                o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
                            tmem_st32(tO + 32 * c, o);
                        }
                    }
                    l *= alpha;
                    if (want) m = mx;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;
                const uint64_t cs2 = f2_pack(cs, cs), nmu2 = f2_pack(-mu, -mu);
                uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f),
                                    f2_pack(0.f, 0.f)};
                uint32_t pk[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const uint64_t x2 = f2_fma(f2_pack(v[2 * u], v[2 * u + 1]), cs2, nmu2);
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    const uint64_t p2 = (u % 4 == 3) ? exp2_poly2(x2) : f2_pack(ex2(x0), ex2(x1));
                    sum2[u & 3] = f2_add(sum2[u & 3], p2);
                    float p0, p1;
                    f2_unpack(p2, p0, p1);
                    pk[u] = pack_bf16(p0, p1);
                }
                tmem_st32(tS, pk);  // P over the first 32 columns of its S buffer
                float s0, s1;
                f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
                l += s0 + s1;
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[2 * x + b]);
            ++n;
        }
        mbar_arrive(&bars.desc_empty[di]);
        if (last) break;
    }

    // epilogue: O / l -> bf16, lse
    bool have = n > 0 && ok;
    if (have) {
        have = __all_sync(0xffffffffu, mbar_wait(&bars.pv_done[2 * x + ((n - 1) & 1)],
                                                 ((n - 1) >> 1) & 1, abort, p.wait_budget));
        if (!have && !*abort) record_wait_failure(p.seq, kSiteSoftmaxO, -1, 0);
    }
    if (!ok || (n > 0 && !have)) set_abort(abort, p.err, p.seq);
    tc_fence_after();
    const bool row_ok = i < p.N;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    bf16* orow = p.out + ((size_t)qh * p.N + (size_t)(row_ok ? i : 0)) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (have) {
            tmem_ld32(tO + 32 * c, o);
        } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u)
            pk[u] = pack_bf16(__uint_as_float(o[2 * u]) * inv, __uint_as_float(o[2 * u + 1]) * inv);
        if (row_ok) {
            // streaming stores: the output is not read again, so it should not
            // displace the keys and values other CTAs still read from L2
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                __stcs(dst + u, make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]));
        }
    }
    if (row_ok && p.lse)
        p.lse[(size_t)qh * p.N + i] =
            l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    tc_fence_before();
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ AttnParams p) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    // 128-byte swizzled operands need a 1024-byte aligned base
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::bar_off);
    Bars bars;
    {
        uint64_t* q = bar;
        bars.q_full = q;
        q += 1;
        bars.desc_full = q;
        q += kDescRing;
        bars.desc_empty = q;
        q += kDescRing;
        bars.kv_full = q;
        q += kStages;
        bars.k_empty = q;
        q += kStages;
        bars.v_empty = q;
        q += kStages;
        bars.s_full = q;
        q += 4;
        bars.p_full = q;
        q += 4;
        bars.pv_done = q;
        q += 4;
        bars.drain = q;
    }
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::misc_off);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + L::misc_off + 4);
    uint32_t* patmap = reinterpret_cast<uint32_t*>(sm + L::patmap_off);

    // Work order: KV head by KV head (the CTAs in flight then stream one head's K/V,
    // which fits in L2), longest (latest) super tiles first within a head.
    int gi = 0;
    while (gi + 1 < p.ngroups && (int)blockIdx.x >= (int)p.grp_start[gi + 1] * p.n_super) ++gi;
    const int gsize = p.grp_start[gi + 1] - p.grp_start[gi];
    const int rem = (int)blockIdx.x - (int)p.grp_start[gi] * p.n_super;
    const int T = p.n_super - 1 - rem / gsize;
    const int pos = p.grp_start[gi] + rem % gsize;
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        // one read for the whole CTA: every thread must take the same branch
        *abort = *reinterpret_cast<volatile unsigned int*>(&g_abort_seq) == p.seq ? 1 : 0;
        mbar_init(bars.q_full, 1);
        for (int k = 0; k < kDescRing; ++k) {
            mbar_init(&bars.desc_full[k], 1);
            mbar_init(&bars.desc_empty[k], 2 + kSoftmaxThreads);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.k_empty[s], 2);  // one arrival per MMA warp
            mbar_init(&bars.v_empty[s], 2);
        }
        for (int k = 0; k < 4; ++k) {
            mbar_init(&bars.s_full[k], 1);
            mbar_init(&bars.p_full[k], 128);
            mbar_init(&bars.pv_done[k], 1);
        }
        mbar_init(&bars.drain[0], 1);
        mbar_init(&bars.drain[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (*abort) return;  // an earlier CTA of this launch gave up: skip the work
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 8) {
        regs_inc<kSoftmaxRegs>();
        run_softmax<D>(p, sm, bars, abort, tmem, pos, T);
    } else {
        regs_dec<kControlRegs>();
        if (warp == kProducerWarp) {
            run_producer<D>(p, &tmQ, &tmK, &tmV, sm, bars, abort, patmap, pos, T);
        } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
            run_mma<D>(sm, bars, abort, p.err, p.seq, p.wait_budget, tmem, warp - kMmaWarp);
            tc_fence_before();
        }
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------- VS prep
// Per VS head: slash offsets -> block-diagonal bitmap D (offset o touches
// deltas o/64 and, unless o % 64 == 0, o/64 + 1), vertical columns -> sorted
// unique list.  Entries outside [0, N) other than the -1 padding are counted.
//
// With `ranges`, also the range words of the range reading of a diagonal
// (diagonal o gives query block bq the keys 64 bq - o .. 64 bq + 63 - o):
// query block bq takes key u iff some selected o lies in
// [64 bq - u, 64 bq - u + 63], which depends only on delta = bq - u / 64 and
// i = u % 64.  rwords[delta] holds that as bit i:
//   bit i of rwords[delta] = some selected o in [64 delta - i, 64 delta - i + 63].
__global__ void __launch_bounds__(1024) vs_prep_kernel(const int32_t* __restrict__ v_idx,
                                                       int kv_stride, int kv,
                                                       const int32_t* __restrict__ s_idx,
                                                       int ks_stride, int ks, int N,
                                                       VsPrepWs ws, int32_t* err, bool ranges) {
    extern __shared__ uint32_t dsm[];
    __shared__ int warp_tot[33];
    const int pos = blockIdx.x;
    const int nB = N / 64, nBw = (nB + 31) / 32, nW = N / 32;
    uint32_t* col = ws.colbits + (size_t)pos * nW;
    uint32_t* sb = ws.sbits + (size_t)pos * nW;
    for (int w = threadIdx.x; w < nBw; w += blockDim.x) dsm[w] = 0;
    for (int w = threadIdx.x; w < nW; w += blockDim.x) col[w] = 0;
    if (ranges)
        for (int w = threadIdx.x; w < nW; w += blockDim.x) sb[w] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < ks; t += blockDim.x) {
        const int o = s_idx[(size_t)pos * ks_stride + t];
        if (o < 0 || o >= N) {
            if (o != -1 && err) atomicAdd(err, 1);
            continue;
        }
        const int a = o >> 6;
        atomicOr(&dsm[a >> 5], 1u << (a & 31));
        if ((o & 63) && a + 1 < nB) atomicOr(&dsm[(a + 1) >> 5], 1u << ((a + 1) & 31));
        if (ranges) atomicOr(&sb[o >> 5], 1u << (o & 31));
    }
    for (int t = threadIdx.x; t < kv; t += blockDim.x) {
        const int j = v_idx[(size_t)pos * kv_stride + t];
        if (j < 0 || j >= N) {
            if (j != -1 && err) atomicAdd(err, 1);
            continue;
        }
        atomicOr(&col[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    for (int w = threadIdx.x; w < nBw; w += blockDim.x) ws.dbits[(size_t)pos * nBw + w] = dsm[w];
    if (ranges) {
        // 64-bit words of the offset bitmap: word t holds offsets 64 t .. 64 t + 63
        const uint64_t* s64 = reinterpret_cast<const uint64_t*>(sb);
        uint64_t* rw = ws.rwords + (size_t)pos * nB;
        for (int dl = threadIdx.x; dl < nB; dl += blockDim.x) {
            const uint64_t a = dl > 0 ? s64[dl - 1] : 0ull;  // offsets 64 dl - 64 .. 64 dl - 1
            const uint64_t b = s64[dl];                      // offsets 64 dl .. 64 dl + 63
            uint64_t w = b != 0ull ? 1ull : 0ull;
            // i >= 1: offsets 64 dl - i .. 64 dl - 1 are the top i bits of a,
            // offsets 64 dl .. 64 dl + 63 - i the low 64 - i bits of b
            for (int i = 1; i < 64; ++i)
                if ((a >> (64 - i)) != 0ull || (b << i) != 0ull) w |= 1ull << i;
            rw[dl] = w;
        }
    }
    // ordered compaction of the column bitmap
    int32_t* out = ws.vlist + (size_t)pos * ws.vcap;
    int base_out = 0;
    for (int base = 0; base < nW; base += blockDim.x) {
        const int w = base + threadIdx.x;
        const uint32_t bits = w < nW ? col[w] : 0u;
        const int c = __popc(bits);
        const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
        int incl = c;
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_tot[wp] = incl;
        __syncthreads();
        if (wp == 0) {
            const int tv = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
            int ti = tv;
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, ti, off);
                if (lane >= off) ti += y;
            }
            warp_tot[lane] = ti - tv;
            if (lane == 31) warp_tot[32] = ti;
        }
        __syncthreads();
        int o = base_out + warp_tot[wp] + incl - c;
        uint32_t b = bits;
        while (b) {
            const int k = __ffs(b) - 1;
            b &= b - 1;
            if (o < ws.vcap) out[o] = w * 32 + k;
            ++o;
        }
        base_out += warp_tot[32];
        __syncthreads();
    }
    if (threadIdx.x == 0) ws.vcnt[pos] = min(base_out, ws.vcap);
}

template <int D>
cudaError_t launch_attn_d(const AttnLaunch& a, cudaStream_t st) {
    using L = Layout<D>;
    CUtensorMap tmQ, tmK, tmV;
    if (!make_tma_map(&tmQ, a.q, (long long)a.Hq * a.N, D, 128) ||
        !make_tma_map(&tmK, a.k, (long long)a.Hkv * a.N, D, 64) ||
        !make_tma_map(&tmV, a.v, (long long)a.Hkv * a.N, D, 64))
        return cudaErrorInvalidValue;
    // launch sequence number (never 0), unique across host threads
    static std::atomic<unsigned int> next_seq{0};
    unsigned int seq = ++next_seq;
    AttnParams p;
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
    p.n_super = (a.N + 255) / 256;
    p.scale_log2 = (float)(a.scale * 1.4426950408889634);
    p.dbits = a.dbits;
    p.rwords = a.rwords;
    p.nBw = (p.nB + 31) / 32;
    p.vlist = a.vlist;
    p.vcnt = a.vcnt;
    p.vcap = a.vcap;
    p.blk_idx = a.blk_idx;
    p.blk_cnt = a.blk_cnt;
    p.topk = a.topk;
    for (int i = 0; i < MI_MAX_HEADS; ++i)
        p.asw[i] = make_int2(a.sink_h && i < a.n_asw ? a.sink_h[i] : a.sink,
                             a.window_h && i < a.n_asw ? a.window_h[i] : a.window);
    p.err = a.err_count;
    // heads sorted by KV head (stable); each entry keeps its own per-pattern position
    p.heads.n = 0;
    p.ngroups = 0;
    for (int g = 0; g < a.Hkv; ++g) {
        const int start = p.heads.n;
        for (int i = 0; i < a.heads.n; ++i)
            if (kv_head_of(head_qh(a.heads.e[i]), a.Hq, a.Hkv) == g) p.heads.e[p.heads.n++] = a.heads.e[i];
        if (p.heads.n > start) p.grp_start[p.ngroups++] = (uint16_t)start;
    }
    p.grp_start[p.ngroups] = (uint16_t)p.heads.n;
    const int patmap_words = p.nBw > p.nB / 8 + 1 ? p.nBw : p.nB / 8 + 1;
    const size_t smem = L::bytes(patmap_words);
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(a.heads.n * p.n_super);
    sparse_attn_kernel<D><<<grid, kThreads, smem, st>>>(tmQ, tmK, tmV, p);
    return cudaGetLastError();
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D map over [rows][d] bf16, 64-column x box_rows boxes, 128-byte swizzle
bool make_tma_map(CUtensorMap* m, const void* base, long long rows, int d, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t read_wait_failure(int* out8) {
    int rec[8];
    cudaError_t e = cudaMemcpyFromSymbol(rec, g_wait_fail, sizeof(rec));
    if (e != cudaSuccess) return e;
    for (int i = 0; i < 8; ++i) out8[i] = rec[i];
    const int zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    return cudaMemcpyToSymbol(g_wait_fail, zero, sizeof(zero));
}

VsPrepWs carve_vs_prep(WsCarver& c, int n_heads, int N, int kv) {
    VsPrepWs w{};
    const int nB = N / 64, nBw = (nB + 31) / 32;
    w.vcap = kv < N ? kv : N;
    if (w.vcap < 1) w.vcap = 1;
    w.dbits = c.take<uint32_t>((size_t)n_heads * nBw);
    w.colbits = c.take<uint32_t>((size_t)n_heads * (N / 32));
    w.sbits = c.take<uint32_t>((size_t)n_heads * (N / 32));
    w.rwords = c.take<uint64_t>((size_t)n_heads * nB);
    w.vlist = c.take<int32_t>((size_t)n_heads * w.vcap);
    w.vcnt = c.take<int32_t>((size_t)n_heads);
    return w;
}

cudaError_t launch_vs_prep(const int32_t* v_idx, int kv_stride, int kv, const int32_t* s_idx,
                           int ks_stride, int ks, int N, int n_heads, const VsPrepWs& ws,
                           int32_t* err_count, cudaStream_t st, bool ranges) {
    if (n_heads == 0) return cudaSuccess;
    const int nBw = (N / 64 + 31) / 32;
    vs_prep_kernel<<<n_heads, 1024, nBw * sizeof(uint32_t), st>>>(
        v_idx, kv_stride, kv, s_idx, ks_stride, ks, N, ws, err_count, ranges);
    return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t st) {
    if (a.heads.n == 0) return cudaSuccess;
    return a.d == 128 ? launch_attn_d<128>(a, st) : launch_attn_d<64>(a, st);
}

}  // namespace minfer

// attn.cu -- dynamic sparse attention on B200 tensor cores (tcgen05 + TMEM,
// operands staged by TMA), one engine for all three MInference patterns.
//
// MInference 1.0 (aifetchly guide, "Technical Deep Dive"): each head runs
// causal flash-style attention with an online softmax over only its selected
// keys: the sink plus local band (A-shape), the chosen 64x64 blocks
// (Block-Sparse), or the gathered vertical columns plus the 64x64 tiles its
// slash diagonals touch (Vertical-Slash), without counting a key twice.
//
// Work item = one query head x one 256-row "super tile" (four 64-row query
// blocks).  The CTA holds the super tile as two 128-row slots that share
// every key group brought into shared memory:
//   warps 0-3  softmax, slot 0 (TMEM lanes 0-127 = rows 0-127)
//   warps 4-7  softmax, slot 1 (rows 128-255)
//   warp 8     producer: enumerates the key groups of the item and loads
//              them (TMA for pairs of 64-key blocks, cp.async gathers for
//              vertical columns), two stages deep
//   warp 9     MMA issuer: S = Q K^T (SS form) and O += P V (TS form, P read
//              from TMEM), FA-style ping-pong between the two slots.
// A key group is 128 keys: two (not necessarily adjacent) 64-key blocks, or
// up to 128 gathered columns.  Each block / column carries a 4-bit mask, one
// bit per query block, so one group serves rows with different masks; rows
// whose bit is clear see -inf.  Only the diagonal block of a row, the edges
// of an A-shape band and gathered columns need element-level tests.
//
// TMEM (512 columns): slot x uses S at [256x, 256x+128) (P, bf16 pairs,
// aliases its first 64 columns) and O at [256x+128, 256x+128+d).
#include <cfloat>
#include <cstring>
#include <cudaTypedefs.h>

#include "exp2_poly.h"
#include "internal.h"
#include "ptx.cuh"

namespace minfer {

namespace {

// 3 warpgroups: two softmax warpgroups (one per 128-row slot) and one for the
// producer warp, the MMA warp and two idle warps.  Launched at 168 registers
// per thread (65536 / 384, rounded down to 8); the softmax warpgroups then
// take 224 and the third gives back down to 56: 2*128*224 + 128*56 = 384*168.
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168,
              "register split exceeds the launch budget");
constexpr int kSoftmaxThreads = 256;
constexpr int kGroupKeys = 128;
constexpr int kPanelBytes = 128 * 128;  // 128 rows x one 64-column (128-byte) panel
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by >8

enum : int { kGrpNone = 0, kGrpTiles = 1, kGrpGather = 2 };

struct GroupDesc {
    int type, last, need, ncols;
    int b0, b1, m0, m1;
    int cols[kGroupKeys];
    uint8_t cm[kGroupKeys];
};

struct GatherHeld {
    int cols[kGroupKeys];
    uint8_t cm[kGroupKeys];
};

// Sequence number of the last launch in which a CTA gave up waiting; later
// CTAs of that launch exit at once instead of timing out one by one.
__device__ unsigned int g_abort_seq = 0;

// First wait that gave up since the record was last read:
// {launch seq, site, block, thread, group, parity, 0, 0}; site 0 = none.
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
    const bf16* k;
    const bf16* v;
    bf16* out;
    float* lse;
    int Hq, Hkv, N, nB, n_super;
    float scale_log2;
    const uint32_t* dbits;
    int nBw;
    const int32_t* vlist;
    const int32_t* vcnt;
    int vcap;
    const int32_t* blk_idx;
    const int32_t* blk_cnt;
    int topk;
    int sink, window;
    int32_t* err;
    HeadList heads;  // sorted by KV head
    int ngroups;     // KV heads present in `heads`
    uint16_t grp_start[MI_MAX_HEADS + 1];  // heads of KV group i: [grp_start[i], grp_start[i+1])
};

template <int D>
struct Layout {
    static constexpr int kQBytes = 128 * D * 2;   // one slot of Q
    static constexpr int kKVBytes = kGroupKeys * D * 2;
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + 2 * kQBytes;
    static constexpr int v_off = k_off + 2 * kKVBytes;
    static constexpr int kDescRing = 4;  // group descriptors in flight
    static constexpr int desc_off = v_off + 2 * kKVBytes;
    static constexpr int held_off = desc_off + kDescRing * (int)sizeof(GroupDesc);
    static constexpr int bar_off = (held_off + (int)sizeof(GatherHeld) + 15) & ~15;
    static constexpr int kNumBars = 24;
    static constexpr int misc_off = bar_off + kNumBars * 8;
    static constexpr int patmap_off = misc_off + 16;
    static size_t bytes(int patmap_words) {
        size_t b = (size_t)patmap_off + (size_t)patmap_words * 4 + 1024;  // +1024: base alignment
        // d = 64 is small enough for two CTAs per SM, but TMEM holds one: ask for enough
        // shared memory that the SM schedules one at a time.
        return b < 120 * 1024 ? 120 * 1024 : b;
    }
};

// Pipeline barriers.  Group g (in publication order) uses descriptor slot
// g % 4 and, if it carries keys, K stage and V stage g % 2.  K is released as
// soon as the S = Q K^T of its group has run, V only after P V, so the next
// K tile streams in while the current P V is still pending.
struct Bars {
    uint64_t* q_full;
    uint64_t* desc_full;   // [4] producer -> MMA, softmax
    uint64_t* desc_empty;  // [4] MMA + 256 softmax threads -> producer
    uint64_t* k_full;      // [2] TMA / gather -> MMA
    uint64_t* k_empty;     // [2] MMA (after S) -> producer
    uint64_t* v_full;      // [2]
    uint64_t* v_empty;     // [2] MMA (after P V) -> producer
    uint64_t* s_full;      // [2] per slot: S ready in TMEM
    uint64_t* p_full;      // [2] per slot: P written to TMEM
    uint64_t* o_done;      // [2] per slot: last P V done
    uint64_t* drain;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- packed fp32 pairs (one 64-bit register pair, two lanes of work)
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x for a pair on the FMA pipe (method and error bound in exp2_poly.h).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
    float x0, x1;
    f2_unpack(x2, x0, x1);
    const uint64_t xc = f2_pack(fmaxf(x0, kExp2Clamp), fmaxf(x1, kExp2Clamp));
    const uint64_t t = f2_add(xc, f2_pack(kExp2Round, kExp2Round));        // round to nearest
    const uint64_t n = f2_add(t, f2_pack(-kExp2Round, -kExp2Round));       // n as float
    const uint64_t f = f2_fma(n, f2_pack(-1.f, -1.f), xc);                 // x - n, exact
    uint64_t q = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
    q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
    q = f2_fma(q, f, f2_pack(kExp2C0, kExp2C0));
    float q0, q1, t0, t1;
    f2_unpack(q, q0, q1);
    f2_unpack(t, t0, t1);
    // n sits in the low mantissa bits of t; (bits(t) << 23) adds n to the exponent
    const float r0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
    const float r1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
    return f2_pack(r0, r1);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

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
    GroupDesc* desc;
    GatherHeld* held;
    int g;        // KV head
    int pub = 0;  // descriptors published
    int nk = 0;   // K stages filled
    int nv = 0;   // V stages filled
    int lane;
    bool ok = true;

    // lane 0 waits, the warp follows its verdict
    __device__ bool wait(uint64_t* bar, int parity, int count) {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar, parity, abort);
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
    __device__ GroupDesc* acquire_desc() {
        const int i = pub & (L::kDescRing - 1);
        if (pub >= L::kDescRing && !wait(&bars.desc_empty[i], ((pub / L::kDescRing) - 1) & 1, pub))
            return nullptr;
        return &desc[i];
    }
    __device__ void publish_desc() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.desc_full[pub & (L::kDescRing - 1)]);
        ++pub;
    }
    __device__ bool acquire_k(int& s) {
        s = nk & 1;
        return nk < 2 || wait(&bars.k_empty[s], ((nk >> 1) - 1) & 1, nk);
    }
    __device__ bool acquire_v(int& s) {
        s = nv & 1;
        return nv < 2 || wait(&bars.v_empty[s], ((nv >> 1) - 1) & 1, nv);
    }

    __device__ void tiles(int b0, int m0, int b1, int m1) {
        if (!ok) return;
        GroupDesc* d = acquire_desc();
        if (!d) return;
        if (lane == 0) {
            d->type = kGrpTiles;
            d->last = 0;
            d->need = (((m0 | m1) & 0x3) ? 1 : 0) | (((m0 | m1) & 0xC) ? 2 : 0);
            d->ncols = 0;
            d->b0 = b0;
            d->b1 = b1;
            d->m0 = m0;
            d->m1 = m1;
        }
        publish_desc();
        const int row0 = g * p.N + 64 * b0, row1 = g * p.N + 64 * b1;
        int sk;
        if (!acquire_k(sk)) return;
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars.k_full[sk], L::kKVBytes);
            uint8_t* kd = sm + L::k_off + sk * L::kKVBytes;
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn) {
                tma_load_2d(kd + pn * kPanelBytes, tmK, 64 * pn, row0, &bars.k_full[sk]);
                tma_load_2d(kd + pn * kPanelBytes + kPanelBytes / 2, tmK, 64 * pn, row1,
                            &bars.k_full[sk]);
            }
        }
        __syncwarp();
        ++nk;
        int sv;
        if (!acquire_v(sv)) return;
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars.v_full[sv], L::kKVBytes);
            uint8_t* vd = sm + L::v_off + sv * L::kKVBytes;
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn) {
                tma_load_2d(vd + pn * kPanelBytes, tmV, 64 * pn, row0, &bars.v_full[sv]);
                tma_load_2d(vd + pn * kPanelBytes + kPanelBytes / 2, tmV, 64 * pn, row1,
                            &bars.v_full[sv]);
            }
        }
        __syncwarp();
        ++nv;
    }

    __device__ void gather(int n) {
        if (!ok) return;
        GroupDesc* d = acquire_desc();
        if (!d) return;
        int need = 0;
        for (int c = lane; c < kGroupKeys; c += 32) {
            const bool v = c < n;
            const int col = v ? held->cols[c] : held->cols[0];
            const int cm = v ? held->cm[c] : 0;
            d->cols[c] = col;
            d->cm[c] = (uint8_t)cm;
            need |= cm;
        }
        for (int off = 16; off >= 1; off >>= 1) need |= __shfl_xor_sync(0xffffffffu, need, off);
        if (lane == 0) {
            d->type = kGrpGather;
            d->last = 0;
            d->need = ((need & 0x3) ? 1 : 0) | ((need & 0xC) ? 2 : 0);
            d->ncols = n;
            d->b0 = d->b1 = -1;
            d->m0 = d->m1 = 0;
        }
        publish_desc();
        int sk, sv;
        if (!acquire_k(sk) || !acquire_v(sv)) return;
        uint8_t* kd = sm + L::k_off + sk * L::kKVBytes;
        uint8_t* vd = sm + L::v_off + sv * L::kKVBytes;
        constexpr int kChunks = D / 8;  // 16-byte chunks per row
        const bf16* kb = p.k + (size_t)g * p.N * D;
        const bf16* vb = p.v + (size_t)g * p.N * D;
        for (int idx = lane; idx < kGroupKeys * kChunks; idx += 32) {
            const int r = idx / kChunks, c = idx % kChunks;
            const size_t src = (size_t)d->cols[r] * D + c * 8;
            const int dst = (c >> 3) * kPanelBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            cp_async_16(kd + dst, kb + src);
            cp_async_16(vd + dst, vb + src);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bars.k_full[sk]);
            mbar_arrive(&bars.v_full[sv]);
        }
        ++nk;
        ++nv;
    }

    __device__ void finish() {
        if (!ok) return;
        GroupDesc* d = acquire_desc();
        if (!d) return;
        if (lane == 0) {
            d->type = kGrpNone;
            d->last = 1;
            d->need = 0;
            d->ncols = 0;
        }
        publish_desc();
    }

    // Wait (bounded) until every copy this warp started has landed, so that
    // no TMA write can reach shared memory after the CTA exits.
    __device__ void drain() {
        if (lane != 0) return;
        for (int u = nk - 2; u < nk; ++u)
            if (u >= 0) mbar_wait_budget(&bars.k_full[u & 1], (u >> 1) & 1);
        for (int u = nv - 2; u < nv; ++u)
            if (u >= 0) mbar_wait_budget(&bars.v_full[u & 1], (u >> 1) & 1);
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
    const int g = kv_head_of(qh, p.Hq, p.Hkv);
    const int qb0 = 4 * T;
    const int nqb = min(4, p.nB - qb0);
    const int bmax = min(qb0 + 3, p.nB - 1);

    if (lane == 0) {
        prefetch_tmap(tmQ);
        prefetch_tmap(tmK);
        prefetch_tmap(tmV);
        mbar_arrive_expect_tx(bars.q_full, 2 * L::kQBytes);
        for (int x = 0; x < 2; ++x)
            for (int pn = 0; pn < D / 64; ++pn)
                tma_load_2d(sm + L::q_off + x * L::kQBytes + pn * kPanelBytes, tmQ, 64 * pn,
                            qh * p.N + 256 * T + 128 * x, bars.q_full);
    }

    // per-pattern block map
    if (pattern == MI_PATTERN_VS) {
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
                   reinterpret_cast<GroupDesc*>(sm + L::desc_off),
                   reinterpret_cast<GatherHeld*>(sm + L::held_off), g};
    pr.lane = lane;

    // --- 64-key blocks, ascending, paired into 128-key groups
    int pend_b = -1, pend_m = 0;
    for (int base = 0; base <= bmax && pr.ok; base += 32) {
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
            } else {
                for (int qq = 0; qq < nqb; ++qq) {
                    const int qb = qb0 + qq;
                    if (b <= qb && (64 * b < p.sink || 64 * (qb - b) - 63 < p.window))
                        m |= 1 << qq;
                }
            }
        }
        unsigned bal = __ballot_sync(0xffffffffu, m != 0);
        while (bal) {
            const int src = __ffs(bal) - 1;
            bal &= bal - 1;
            const int mm = __shfl_sync(0xffffffffu, m, src);
            if (pend_b < 0) {
                pend_b = base + src;
                pend_m = mm;
            } else {
                pr.tiles(pend_b, pend_m, base + src, mm);
                pend_b = -1;
            }
        }
    }
    if (pend_b >= 0) pr.tiles(pend_b, pend_m, pend_b, 0);

    // --- Vertical-Slash: gathered columns not already inside a computed tile
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
                        if (!bit_of(patmap, delta)) m |= 1 << qq;
                    }
                }
            }
            const unsigned bal = __ballot_sync(0xffffffffu, m != 0);
            const int rank = __popc(bal & ((1u << lane) - 1u));
            const int navail = __popc(bal);
            const int take = min(navail, kGroupKeys - n_held);
            if (m && rank < take) {
                held->cols[n_held + rank] = j;
                held->cm[n_held + rank] = (uint8_t)m;
            }
            __syncwarp();
            n_held += take;
            if (n_held == kGroupKeys) {
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

// ------------------------------------------------------------- MMA issuer
// The whole warp runs this loop converged: bookkeeping and descriptors are
// uniform, lane 0 alone polls the barriers and broadcasts the outcome, and
// elect.sync inside the issue instructions picks the single issuing lane.
template <int D>
__device__ void run_mma(uint8_t* sm, const Bars& bars, volatile int* abort, int32_t* err,
                        unsigned int seq, uint32_t tmem) {
    using L = Layout<D>;
    const int lane = threadIdx.x & 31;
    const uint32_t idS = idesc_bf16_f32(128, kGroupKeys, false);
    const uint32_t idO = idesc_bf16_f32(128, D, true);
    const uint32_t q_addr = smem_u32(sm + L::q_off);
    const uint32_t k_addr = smem_u32(sm + L::k_off);
    const uint32_t v_addr = smem_u32(sm + L::v_off);
    const GroupDesc* desc = reinterpret_cast<const GroupDesc*>(sm + L::desc_off);
    auto wait = [&](uint64_t* bar, int parity) -> bool {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar, parity, abort);
        return __shfl_sync(0xffffffffu, w, 0);
    };

    int pend[2] = {-1, -1}, npv[2] = {0, 0}, np[2] = {0, 0};
    int vuses[2] = {0, 0};
    bool ok = wait(bars.q_full, 0);
    if (!ok && lane == 0 && !*abort) record_wait_failure(seq, kSiteMmaQ, 0, 0);
    int g = 0;
    while (ok) {
        const int di = g & (L::kDescRing - 1);
        if (!wait(&bars.desc_full[di], (g / L::kDescRing) & 1)) {
            if (lane == 0 && !*abort)
                record_wait_failure(seq, kSiteMmaFull, g, (g / L::kDescRing) & 1);
            ok = false;
            break;
        }
        const int type = desc[di].type, need = desc[di].need, last = desc[di].last;
        const int s = g & 1;  // data groups are numbered like descriptors (the end marker is last)
        bool k_ready = false;
        // per slot: first the pending O += P V (needs only P and V), then S of
        // this group (needs K): a late K tile does not hold back the other work
        for (int x = 0; x < 2 && ok; ++x) {
            if (pend[x] >= 0) {
                // P of the slot's previous group, then its V: issue O += P V
                const int pg = pend[x], st = pg & 1;
                if (!wait(&bars.p_full[x], np[x] & 1) || !wait(&bars.v_full[st], (pg >> 1) & 1)) {
                    if (lane == 0 && !*abort) record_wait_failure(seq, kSiteMmaP, g, np[x] & 1);
                    ok = false;
                    break;
                }
                ++np[x];
                tc_fence_after();
                const uint32_t tP = tmem + 256 * x;
                const uint32_t tO = tmem + 256 * x + 128;
#pragma unroll
                for (int kk = 0; kk < kGroupKeys / 16; ++kk) {
                    const uint64_t bdesc =
                        sw128_desc(v_addr + st * L::kKVBytes + kk * 2048, kPanelBytes, 1024);
                    mma_ts_warp(tO, tP + kk * 8, bdesc, idO, (npv[x] > 0 || kk > 0) ? 1u : 0u);
                }
                ++npv[x];
                if (--vuses[st] == 0) mma_commit_warp(&bars.v_empty[st]);
                pend[x] = -1;
            }
            if (type != kGrpNone && ((need >> x) & 1)) {
                if (!k_ready) {
                    if (!wait(&bars.k_full[s], (g >> 1) & 1)) {
                        if (lane == 0 && !*abort)
                            record_wait_failure(seq, kSiteMmaFull, g, (g >> 1) & 1);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    k_ready = true;
                }
                const uint32_t tS = tmem + 256 * x;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int pn = kk >> 2, off = (kk & 3) * 32;
                    const uint64_t adesc =
                        sw128_desc(q_addr + x * L::kQBytes + pn * kPanelBytes + off, 16, 1024);
                    const uint64_t bdesc =
                        sw128_desc(k_addr + s * L::kKVBytes + pn * kPanelBytes + off, 16, 1024);
                    mma_ss_warp(tS, adesc, bdesc, idS, kk > 0 ? 1u : 0u);
                }
                mma_commit_warp(&bars.s_full[x]);
                pend[x] = g;
            }
        }
        if (!ok) break;
        if (type != kGrpNone) {
            mma_commit_warp(&bars.k_empty[s]);  // K free once this group's S has run
            vuses[s] = __popc(need);
        }
        mbar_arrive_warp(&bars.desc_empty[di]);
        if (last) break;
        ++g;
    }
    if (!ok && lane == 0) set_abort(abort, err, seq);
    for (int x = 0; x < 2; ++x)
        if (npv[x] > 0) mma_commit_warp(&bars.o_done[x]);
    // every MMA must have finished before TMEM is released
    mma_commit_warp(bars.drain);
    if (lane == 0) mbar_wait_budget(bars.drain, 0);
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
    const uint32_t lane_off = (uint32_t)(lg * 32) << 16;
    const uint32_t tS = tmem + 256 * x + lane_off;
    const uint32_t tO = tmem + 256 * x + 128 + lane_off;
    const GroupDesc* desc = reinterpret_cast<const GroupDesc*>(sm + L::desc_off);

    float m = -INFINITY, l = 0.f;
    int ns = 0;
    bool ok = true;
    for (int g = 0;; ++g) {
        const int di = g & (L::kDescRing - 1);
        const int dpar = (g / L::kDescRing) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.desc_full[di], dpar, abort))) {
            if (!*abort) record_wait_failure(p.seq, kSiteSoftmaxFull, g, dpar);
            ok = false;
            break;
        }
        const GroupDesc& d = desc[di];
        const int type = d.type, last = d.last;
        if (type != kGrpNone && ((d.need >> x) & 1)) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[x], ns & 1, abort))) {
                if (!*abort) record_wait_failure(p.seq, kSiteSoftmaxS, g, ns & 1);
                ok = false;
                break;
            }
            ++ns;
            tc_fence_after();
            float v[kGroupKeys];
            {
                uint32_t r[kGroupKeys];
                tmem_ld128(tS, r);  // the whole row of S: one TMEM round trip
#pragma unroll
                for (int u = 0; u < kGroupKeys; ++u) v[u] = __uint_as_float(r[u]);
            }
            if (type == kGrpTiles) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = h ? d.b1 : d.b0;
                    const int bit = ((h ? d.m1 : d.m0) >> qi) & 1;
                    const long long j0 = 64LL * b;
                    const bool full = bit && (j0 + 63 <= i) &&
                                      (!ashape || j0 + 63 < p.sink || i - j0 < p.window);
                    if (!full) {
#pragma unroll
                        for (int c = 0; c < 64; ++c) {
                            const long long j = j0 + c;
                            const bool keep = bit && j <= i &&
                                              (!ashape || j < p.sink || i - j < p.window);
                            if (!keep) v[64 * h + c] = -INFINITY;
                        }
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < kGroupKeys; ++c) {
                    const bool keep = ((d.cm[c] >> qi) & 1) && (long long)d.cols[c] <= i;
                    if (!keep) v[c] = -INFINITY;
                }
            }
            // raw scores: the scale (> 0) commutes with the max and is folded into
            // the exponent below (one packed FFMA per pair)
            const float cs = p.scale_log2;
            // four independent max chains (latency), then combined
            float mq[4] = {fmaxf(v[0], v[1]), fmaxf(v[2], v[3]), fmaxf(v[4], v[5]),
                           fmaxf(v[6], v[7])};
#pragma unroll
            for (int c = 8; c < kGroupKeys; c += 8) {
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4)
                    mq[w4] = fmax3(mq[w4], v[c + 2 * w4], v[c + 2 * w4 + 1]);
            }
            float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
            mx *= cs;
            // Lazy rescale: a row moves its reference max only when the max grew by
            // more than 2^8 (p <= 256 otherwise, exact after the final 1/l).  The
            // TMEM accesses are .sync.aligned, so the whole warp takes the branch
            // together; rows that do not need it scale by 1.
            const bool want = mx > m + kRescaleThreshold;
            if (__any_sync(0xffffffffu, want)) {
                const float alpha = want ? ex2(m - mx) : 1.f;  // 0 while m is -inf
                if (ns > 1) {
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
            // four independent packed row-sum accumulators (latency)
            uint64_t sum2[4] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f), f2_pack(0.f, 0.f),
                                f2_pack(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    const uint64_t x2 =
                        f2_fma(f2_pack(v[64 * c + 2 * u], v[64 * c + 2 * u + 1]), cs2, nmu2);
                    // all exponentials on MUFU: measured faster than moving a share to
                    // the FMA pipe, the softmax warp is bound by its own issue rate
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    const uint64_t p2 = f2_pack(ex2(x0), ex2(x1));
                    sum2[u & 3] = f2_add(sum2[u & 3], p2);
                    float p0, p1;
                    f2_unpack(p2, p0, p1);
                    pk[u] = pack_bf16(p0, p1);
                }
                tmem_st32(tS + 32 * c, pk);
            }
            float s0, s1;
            f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), s0, s1);
            const float rs = s0 + s1;
            l += rs;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[x]);
        }
        mbar_arrive(&bars.desc_empty[di]);
        if (last) break;
    }

    // epilogue: O / l -> bf16, lse
    bool have = ns > 0 && ok;
    if (have) {
        have = __all_sync(0xffffffffu, mbar_wait(&bars.o_done[x], 0, abort));
        if (!have && !*abort) record_wait_failure(p.seq, kSiteSoftmaxO, -1, 0);
    }
    if (!ok || (ns > 0 && !have)) set_abort(abort, p.err, p.seq);
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
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
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
    Bars bars{bar + 0,  bar + 1,  bar + 5,  bar + 9,  bar + 11, bar + 13,
              bar + 15, bar + 17, bar + 19, bar + 21, bar + 23};
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
        for (int i = 0; i < L::kDescRing; ++i) {
            mbar_init(&bars.desc_full[i], 1);
            mbar_init(&bars.desc_empty[i], 1 + kSoftmaxThreads);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.v_empty[s], 1);
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.p_full[s], 128);
            mbar_init(&bars.o_done[s], 1);
        }
        mbar_init(bars.drain, 1);
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
        } else if (warp == kMmaWarp) {
            run_mma<D>(sm, bars, abort, p.err, p.seq, tmem);
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
__global__ void __launch_bounds__(1024) vs_prep_kernel(const int32_t* __restrict__ v_idx,
                                                       int kv_stride, int kv,
                                                       const int32_t* __restrict__ s_idx,
                                                       int ks_stride, int ks, int N,
                                                       VsPrepWs ws, int32_t* err) {
    extern __shared__ uint32_t dsm[];
    __shared__ int warp_tot[33];
    const int pos = blockIdx.x;
    const int nB = N / 64, nBw = (nB + 31) / 32, nW = N / 32;
    uint32_t* col = ws.colbits + (size_t)pos * nW;
    for (int w = threadIdx.x; w < nBw; w += blockDim.x) dsm[w] = 0;
    for (int w = threadIdx.x; w < nW; w += blockDim.x) col[w] = 0;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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
bool make_map(CUtensorMap* m, const void* base, long long rows, int d, int box_rows) {
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

template <int D>
cudaError_t launch_attn_d(const AttnLaunch& a, cudaStream_t st) {
    using L = Layout<D>;
    CUtensorMap tmQ, tmK, tmV;
    if (!make_map(&tmQ, a.q, (long long)a.Hq * a.N, D, 128) ||
        !make_map(&tmK, a.k, (long long)a.Hkv * a.N, D, 64) ||
        !make_map(&tmV, a.v, (long long)a.Hkv * a.N, D, 64))
        return cudaErrorInvalidValue;
    static unsigned int seq = 0;
    AttnParams p;
    memset(&p, 0, sizeof(p));
    if (++seq == 0) ++seq;
    p.seq = seq;
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
    p.nBw = (p.nB + 31) / 32;
    p.vlist = a.vlist;
    p.vcnt = a.vcnt;
    p.vcap = a.vcap;
    p.blk_idx = a.blk_idx;
    p.blk_cnt = a.blk_cnt;
    p.topk = a.topk;
    p.sink = a.sink;
    p.window = a.window;
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
    w.vlist = c.take<int32_t>((size_t)n_heads * w.vcap);
    w.vcnt = c.take<int32_t>((size_t)n_heads);
    return w;
}

cudaError_t launch_vs_prep(const int32_t* v_idx, int kv_stride, int kv, const int32_t* s_idx,
                           int ks_stride, int ks, int N, int n_heads, const VsPrepWs& ws,
                           int32_t* err_count, cudaStream_t st) {
    if (n_heads == 0) return cudaSuccess;
    const int nBw = (N / 64 + 31) / 32;
    vs_prep_kernel<<<n_heads, 1024, nBw * sizeof(uint32_t), st>>>(v_idx, kv_stride, kv, s_idx,
                                                                  ks_stride, ks, N, ws, err_count);
    return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t st) {
    if (a.heads.n == 0) return cudaSuccess;
    return a.d == 128 ? launch_attn_d<128>(a, st) : launch_attn_d<64>(a, st);
}

}  // namespace minfer

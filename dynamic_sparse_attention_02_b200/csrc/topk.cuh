// topk.cuh -- block-wide top-k by radix select, ties broken toward the lower
// index, result written in ascending index order.
//
// Keys are fp32 scores mapped to order-preserving uint32 (larger score ->
// larger key).  Four 8-bit histogram passes find the k-th largest key T and
// how many of the keys equal to T are still needed; one ordered compaction
// pass then keeps every key > T and the first `need_eq` keys == T.
#pragma once

#include <cstdint>

namespace minfer {

__device__ __forceinline__ uint32_t float_order_key(float f) {
    uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Block-wide exclusive prefix sum of one int per thread (blockDim.x a
// multiple of 32, <= 1024).  `warp_tot` holds 33 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        if (lane < nwarps) warp_tot[lane] = wi - w;  // exclusive per warp
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    const int res = warp_tot[warp] + incl - v;
    total = warp_tot[32];
    __syncthreads();
    return res;
}

// Shared scratch for one block-wide selection.
struct TopkSmem {
    uint32_t hist[256];
    int warp_tot[33];
    uint32_t prefix;
    int remaining;
    int done;
};

// Find threshold key T and the number of keys equal to T to keep, for the
// top k (1 <= k < n) of keys get(0..n-1).
template <class Get>
__device__ void block_radix_select(const Get& get, int n, int k, TopkSmem& s, uint32_t& thr,
                                   int& need_eq) {
    if (threadIdx.x == 0) {
        s.prefix = 0;
        s.remaining = k;
        s.done = 0;
    }
    uint32_t mask = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += blockDim.x) s.hist[b] = 0;
        __syncthreads();
        const uint32_t prefix = s.prefix;
        // a thread's keys mostly share the leading digits (scores of one list
        // span few binades), so runs of one bin are counted in a register and
        // added once instead of contending on one shared counter
        uint32_t run_bin = 0, run_cnt = 0;
        auto count = [&](uint32_t key) {
            if ((key & mask) == prefix) {
                const uint32_t b = (key >> shift) & 255u;
                if (run_cnt != 0 && b != run_bin) {
                    atomicAdd(&s.hist[run_bin], run_cnt);
                    run_cnt = 0;
                }
                run_bin = b;
                ++run_cnt;
            }
        };
        const int bd = (int)blockDim.x;
        int j = threadIdx.x;
        for (; j + 7 * bd < n; j += 8 * bd) {  // eight loads in flight per thread
            uint32_t kb[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) kb[u] = get(j + u * bd);
#pragma unroll
            for (int u = 0; u < 8; ++u) count(kb[u]);
        }
        for (; j < n; j += bd) count(get(j));
        if (run_cnt != 0) atomicAdd(&s.hist[run_bin], run_cnt);
        __syncthreads();
        if (threadIdx.x == 0) {
            int rem = s.remaining;
            int b = 255;
            for (; b > 0; --b) {
                const int c = (int)s.hist[b];
                if (c >= rem) break;
                rem -= c;
            }
            const uint32_t np = prefix | ((uint32_t)b << shift);
            if ((int)s.hist[b] == rem && np != 0) {
                // the bin is taken whole: every key >= np, none equal to np - 1
                s.prefix = np - 1;
                s.remaining = 0;
                s.done = 1;
            } else {
                s.remaining = rem;
                s.prefix = np;
            }
        }
        __syncthreads();
        if (s.done) break;
        mask |= 255u << shift;
    }
    thr = s.prefix;
    need_eq = s.remaining;
    __syncthreads();
}

// Write the selected indices in ascending order to out[0..k): every key > thr
// and the first need_eq keys == thr.  Each warp owns one contiguous segment of
// the keys and reads it 32 keys at a time (coalesced); one scan over the warps
// (equal keys before the segment, selections before it) places its output,
// and ballots order the lanes within each 32-key step.
struct CompactSmem {
    int eq[32], sel[32];
};
template <class Get>
__device__ void block_select_compact(const Get& get, int n, int k, uint32_t thr, int need_eq,
                                     TopkSmem& s, int32_t* out) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const int per = (((n + nw - 1) / nw) + 31) & ~31;
    const int j0 = min(n, w * per), j1 = min(n, j0 + per);
    int gt = 0, eq = 0;
    for (int base = j0; base < j1; base += 128) {
        uint32_t kb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = base + 32 * u + lane;
            kb[u] = j < j1 ? get(j) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool in = base + 32 * u + lane < j1;
            gt += (in && kb[u] > thr) ? 1 : 0;
            eq += (in && kb[u] == thr) ? 1 : 0;
        }
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    CompactSmem* cs = reinterpret_cast<CompactSmem*>(s.hist);  // the histogram is done
    __syncthreads();
    if (lane == 0) {
        cs->eq[w] = eq;
        cs->sel[w] = gt;
    }
    __syncthreads();
    if (w == 0) {
        const int e = lane < nw ? cs->eq[lane] : 0, g = lane < nw ? cs->sel[lane] : 0;
        int ei = e;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, ei, off);
            if (lane >= off) ei += y;
        }
        const int e_before = ei - e;
        const int take = max(0, min(e, need_eq - e_before));
        const int sv = g + take;
        int si = sv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, si, off);
            if (lane >= off) si += y;
        }
        __syncwarp();
        if (lane < nw) {
            cs->eq[lane] = e_before;
            cs->sel[lane] = si - sv;
        }
    }
    __syncthreads();
    int eq_seen = cs->eq[w], pos = cs->sel[w];
    const int end = pos + gt + max(0, min(eq, need_eq - eq_seen));
    for (int base = j0; base < j1 && pos < end; base += 32) {
        const int j = base + lane;
        const uint32_t key = j < j1 ? get(j) : 0u;
        const bool g1 = j < j1 && key > thr;
        const bool e1 = j < j1 && key == thr;
        const unsigned eqm = __ballot_sync(0xffffffffu, e1);
        const bool sel = g1 || (e1 && eq_seen + __popc(eqm & below) < need_eq);
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        const int p = pos + __popc(selm & below);
        if (sel && p < k) out[p] = j;
        eq_seen += __popc(eqm);
        pos += __popc(selm);
    }
    __syncthreads();
}

// One key into a run-length histogram count: a run of equal bins is held in
// (rb, rc) and added to the shared histogram when the bin changes.
__device__ __forceinline__ void run_count(uint32_t key, uint32_t mask, uint32_t prefix, int shift,
                                          uint32_t* hist, uint32_t& rb, uint32_t& rc) {
    if ((key & mask) == prefix) {
        const uint32_t b = (key >> shift) & 255u;
        if (rc != 0 && b != rb) {
            atomicAdd(&hist[rb], rc);
            rc = 0;
        }
        rb = b;
        ++rc;
    }
}

// ---- one warp per selection (many short rows at once), same contract as above.
// `hist` is this warp's own 256-entry shared histogram.
template <class Get>
__device__ void warp_radix_select(const Get& get, int n, int k, uint32_t* hist, uint32_t& thr,
                                  int& need_eq) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int rem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        // runs of one bin are counted in registers (see block_radix_select); each
        // lane reads four independent streams (keys j = 128 i + 32 t + lane), each
        // with its own run, so that four load/count chains are in flight at once
        uint32_t b0 = 0, b1 = 0, b2 = 0, b3 = 0, c0 = 0, c1 = 0, c2 = 0, c3 = 0;
        int j0 = 0;
        for (; j0 + 128 <= n; j0 += 128) {
            const uint32_t k0 = get(j0 + lane), k1 = get(j0 + 32 + lane);
            const uint32_t k2 = get(j0 + 64 + lane), k3 = get(j0 + 96 + lane);
            run_count(k0, mask, prefix, shift, hist, b0, c0);
            run_count(k1, mask, prefix, shift, hist, b1, c1);
            run_count(k2, mask, prefix, shift, hist, b2, c2);
            run_count(k3, mask, prefix, shift, hist, b3, c3);
        }
        if (j0 + lane < n) run_count(get(j0 + lane), mask, prefix, shift, hist, b0, c0);
        if (j0 + 32 + lane < n) run_count(get(j0 + 32 + lane), mask, prefix, shift, hist, b1, c1);
        if (j0 + 64 + lane < n) run_count(get(j0 + 64 + lane), mask, prefix, shift, hist, b2, c2);
        if (j0 + 96 + lane < n) run_count(get(j0 + 96 + lane), mask, prefix, shift, hist, b3, c3);
        if (c0 != 0) atomicAdd(&hist[b0], c0);
        if (c1 != 0) atomicAdd(&hist[b1], c1);
        if (c2 != 0) atomicAdd(&hist[b2], c2);
        if (c3 != 0) atomicAdd(&hist[b3], c3);
        __syncwarp();
        // lane l owns bins 255-8l down to 248-8l; a scan over the lanes gives the
        // count above each lane's bins, so one lane holds the bin where the
        // running count from the top reaches `rem`
        int c[8], sum = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            c[u] = (int)hist[255 - 8 * lane - u];
            sum += c[u];
        }
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int above = incl - sum;
        const unsigned who = __ballot_sync(0xffffffffu, above < rem && rem <= incl);
        const int src = who ? __ffs(who) - 1 : 31;
        int bsel = 0, left = rem - above;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (left <= c[u]) {
                bsel = 255 - 8 * lane - u;
                break;
            }
            left -= c[u];
        }
        int csel = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (255 - 8 * lane - u == bsel) csel = c[u];
        bsel = __shfl_sync(0xffffffffu, bsel, src);
        rem = __shfl_sync(0xffffffffu, left, src);
        csel = __shfl_sync(0xffffffffu, csel, src);
        prefix |= (uint32_t)bsel << shift;
        mask |= 255u << shift;
        __syncwarp();
        if (csel == rem && prefix != 0) {
            // the bin is taken whole: every key >= prefix, none equal to prefix - 1
            thr = prefix - 1;
            need_eq = 0;
            return;
        }
    }
    thr = prefix;
    need_eq = rem;
}

template <class Get>
__device__ void warp_select_compact(const Get& get, int n, int k, uint32_t thr, int need_eq,
                                    int32_t* out) {
    const int lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    int eq_base = 0, sel_base = 0;
    // four 32-key steps per round: their loads are issued together, then the
    // steps are placed in index order by ballots
    for (int base = 0; base < n && sel_base < k; base += 128) {
        uint32_t kb[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = base + 32 * t + lane;
            kb[t] = j < n ? get(j) : 0u;
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = base + 32 * t + lane;
            const bool gt = j < n && kb[t] > thr;
            const bool eq = j < n && kb[t] == thr;
            const unsigned eqm = __ballot_sync(0xffffffffu, eq);
            const bool sel = gt || (eq && eq_base + __popc(eqm & below) < need_eq);
            const unsigned selm = __ballot_sync(0xffffffffu, sel);
            const int pos = sel_base + __popc(selm & below);
            if (sel && pos < k) out[pos] = j;
            eq_base += __popc(eqm);
            sel_base += __popc(selm);
        }
    }
}

}  // namespace minfer

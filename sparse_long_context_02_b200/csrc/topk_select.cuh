// Exact top-k selection pieces shared by the prefill and decode indexers.
//
// Order (Kwai Keye-VL-2.0 technical-report summary, section 1: each query
// keeps its k best positions; section 8: the selection is deterministic):
// higher score first, then lower key index.  Scores are kept as ord(score),
// a monotone map of IEEE floats to unsigned integers, so the whole order is
// one 64-bit key, larger = better:
//     key = ord(score) << 32 | ~index
// Keys are unique, so "the k largest keys" is one well-defined set.
//
// Collectives run over NT threads that share a named barrier.  The k-th
// largest key is found by searching, first on ord(score) (the largest s with
// at least k entries scoring >= s) with three pivots per pass over scores
// cached in registers, then, among the entries scoring exactly s, on the
// index.  Each pass is compares, warp reductions and one barrier: no
// atomics, no histogram.  Compaction keeps the entries whose key is >= the
// k-th, in their original order.
#pragma once

#include "ptx.cuh"

namespace dsa {
namespace sel {

__device__ __forceinline__ uint32_t ord_f32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t make_key(uint32_t ord, int32_t s) {
    return ((uint64_t)ord << 32) | (uint64_t)(~(uint32_t)s);
}

// Candidates are read through an accessor: ord(e), index(e) for logical
// entry e.  The arrays may live in shared or global memory.
struct FlatAccess {
    const uint32_t* so;
    const int32_t* ix;
    __device__ __forceinline__ uint32_t ord(int e) const { return so[e]; }
    __device__ __forceinline__ int32_t index(int e) const { return ix[e]; }
};

// Up to four lists, logically concatenated (list j holds start[j+1]-start[j]
// entries).
struct SegAccess {
    const uint32_t* so[4];
    const int32_t* ix[4];
    int start[5];
    __device__ __forceinline__ int seg(int e) const {
        return (e >= start[1]) + (e >= start[2]) + (e >= start[3]);
    }
    __device__ __forceinline__ uint32_t ord(int e) const {
        const int j = seg(e);
        return so[j][e - start[j]];
    }
    __device__ __forceinline__ int32_t index(int e) const {
        const int j = seg(e);
        return ix[j][e - start[j]];
    }
};

// Shared-memory scratch of one collective group.
template <int NT>
struct Scratch {
    static_assert(NT % 32 == 0 && NT <= 1024, "one partial per warp, at most one per lane");
    uint32_t red[2][NT / 32];   // per-warp partials, double-buffered by step parity
    uint32_t red2[2][NT / 32];
    uint32_t red3[2][NT / 32];
    int csum[8 * (NT / 32)];    // compaction counts
    int total;
    alignas(16) uint32_t samp[NT];  // one sampled score per thread
};

// Sum of v over the NT threads; `parity` alternates between calls so one
// barrier per call suffices.
template <int NT>
__device__ __forceinline__ uint32_t blk_sum(uint32_t v, Scratch<NT>& S, int& parity, uint32_t bar,
                                            int tid) {
    v = __reduce_add_sync(0xffffffffu, v);
    if ((tid & 31) == 0) S.red[parity][tid >> 5] = v;
    named_bar_sync(bar, NT);
    // every warp reduces the NT / 32 partials itself: one load per lane
    const int lane = tid & 31;
    const uint32_t s = __reduce_add_sync(0xffffffffu, lane < NT / 32 ? S.red[parity][lane] : 0u);
    parity ^= 1;
    return s;
}

// Min of a and max of b over the NT threads (one barrier).
template <int NT>
__device__ __forceinline__ void blk_minmax(uint32_t& a, uint32_t& b, Scratch<NT>& S, int& parity,
                                           uint32_t bar, int tid) {
    a = __reduce_min_sync(0xffffffffu, a);
    b = __reduce_max_sync(0xffffffffu, b);
    if ((tid & 31) == 0) {
        S.red[parity][tid >> 5] = a;
        S.red2[parity][tid >> 5] = b;
    }
    named_bar_sync(bar, NT);
    const int lane = tid & 31;
    a = __reduce_min_sync(0xffffffffu, lane < NT / 32 ? S.red[parity][lane] : 0xffffffffu);
    b = __reduce_max_sync(0xffffffffu, lane < NT / 32 ? S.red2[parity][lane] : 0u);
    parity ^= 1;
}

// Index of the need-th entry (1-based, in position order) whose ord equals s.
// One pass over rounds of NT entries with warp ballots and a scan of the
// per-(round, warp) counts by warp 0.
template <int NT, class A>
__device__ int32_t nth_in_order(const A& a, int n, uint32_t s, uint32_t need, Scratch<NT>& S,
                                uint32_t bar, int tid) {
    constexpr int NW = NT / 32;
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t before = 0;  // ties in earlier chunks
    for (int c0 = 0; c0 < n; c0 += 8 * NT) {
        uint32_t bal[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = c0 + u * NT + tid;
            bal[u] = __ballot_sync(0xffffffffu, e < n && a.ord(e) == s);
        }
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < 8; ++u) S.csum[u * NW + warp] = __popc(bal[u]);
        }
        named_bar_sync(bar, NT);
        if (warp == 0) {  // exclusive scan of the 8 * NW counts, in place
            constexpr int NC = 8 * NW, PER = (NC + 31) / 32;
            int v[PER], t = 0;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = lane * PER + q;
                v[q] = i < NC ? S.csum[i] : 0;
                t += v[q];
            }
            int incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int run = incl - t;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = lane * PER + q;
                if (i < NC) S.csum[i] = run;
                run += v[q];
            }
            if (lane == 31) S.total = incl;
        }
        named_bar_sync(bar, NT);
        const uint32_t chunk = (uint32_t)S.total;
        if (before + chunk >= need) {  // the need-th tie is in this chunk
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if ((bal[u] >> lane) & 1u) {
                    const uint32_t rank = before + (uint32_t)S.csum[u * NW + warp] +
                                          (uint32_t)__popc(bal[u] & ((1u << lane) - 1u));
                    if (rank + 1 == need) S.red[0][0] = (uint32_t)a.index(c0 + u * NT + tid);
                }
            }
            named_bar_sync(bar, NT);
            const int32_t r = (int32_t)S.red[0][0];
            named_bar_sync(bar, NT);
            return r;
        }
        before += chunk;
        named_bar_sync(bar, NT);
    }
    return 0x7fffffff;  // not reached: need <= number of ties
}

// Per-thread register cache of the ordered scores: entry e = tid + r * NT
// for r < R (0 beyond n: below every real ord, so it never counts).
template <int NT, int R, class A>
__device__ __forceinline__ void load_ords(const A& a, int n, int tid, uint32_t (&oc)[R]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = tid + r * NT;
        oc[r] = e < n ? a.ord(e) : 0u;
    }
}

// The k-th largest key among entries [0, n) (n >= k >= 1).  `floor`: an ord
// that at least k entries reach (0 if unknown) — the search starts there.
// Each pass counts three pivots at once (two bits of the answer per pass)
// over scores cached in registers (R per thread; entries beyond R * NT are
// read from memory).
template <int NT, int R, class A>
__device__ uint64_t kth_largest(const A& a, int n, int k, uint32_t floor, Scratch<NT>& S,
                                uint32_t bar, int tid) {
    int parity = 0;
    uint32_t oc[R];
    load_ords<NT, R>(a, n, tid, oc);
    const int tail0 = R * NT;
    // ---- score: the largest s with count(ord >= s) >= k
    uint32_t lo = 0xffffffffu, hi = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (tid + r * NT < n) lo = min(lo, oc[r]);
        hi = max(hi, oc[r]);
    }
    for (int e = tail0 + tid; e < n; e += NT) {
        const uint32_t o = a.ord(e);
        lo = min(lo, o);
        hi = max(hi, o);
    }
    blk_minmax<NT>(lo, hi, S, parity, bar, tid);
    lo = max(lo, min(floor, hi));
    while (lo < hi) {  // count(>= lo) >= k always holds; the answer is in [lo, hi]
        const uint64_t span = (uint64_t)(hi - lo) + 1;
        const uint32_t m1 = lo + (uint32_t)(span / 4), m2 = lo + (uint32_t)(span / 2),
                       m3 = lo + (uint32_t)(3 * span / 4);
        uint32_t c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            c1 += oc[r] >= m1;
            c2 += oc[r] >= m2;
            c3 += oc[r] >= m3;
        }
        for (int e = tail0 + tid; e < n; e += NT) {
            const uint32_t o = a.ord(e);
            c1 += o >= m1;
            c2 += o >= m2;
            c3 += o >= m3;
        }
        c1 = __reduce_add_sync(0xffffffffu, c1);
        c2 = __reduce_add_sync(0xffffffffu, c2);
        c3 = __reduce_add_sync(0xffffffffu, c3);
        if ((tid & 31) == 0) {
            S.red[parity][tid >> 5] = c1;
            S.red2[parity][tid >> 5] = c2;
            S.red3[parity][tid >> 5] = c3;
        }
        named_bar_sync(bar, NT);
        const int ln = tid & 31;
        const bool has = ln < NT / 32;
        const uint32_t t1 = __reduce_add_sync(0xffffffffu, has ? S.red[parity][ln] : 0u);
        const uint32_t t2 = __reduce_add_sync(0xffffffffu, has ? S.red2[parity][ln] : 0u);
        const uint32_t t3 = __reduce_add_sync(0xffffffffu, has ? S.red3[parity][ln] : 0u);
        parity ^= 1;
        const uint32_t K = (uint32_t)k;
        if (t3 >= K) lo = m3;                        // m3 > lo whenever span >= 2
        else if (t2 >= K) { lo = m2; hi = m3 - 1; }
        else if (t1 >= K) { lo = m1; hi = m2 - 1; }
        else hi = m1 - 1;                            // t1 < K implies m1 > lo
    }
    const uint32_t s = lo;
    // ---- index: among entries scoring exactly s, the need-th lowest index
    uint32_t gt = 0, eq = 0;
    int32_t imin = 0x7fffffff, imax = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        gt += oc[r] > s;
        if (oc[r] == s && tid + r * NT < n) {
            eq += 1;
            const int32_t i = a.index(tid + r * NT);
            imin = min(imin, i);
            imax = max(imax, i);
        }
    }
    for (int e = tail0 + tid; e < n; e += NT) {
        const uint32_t o = a.ord(e);
        gt += o > s;
        if (o == s) {
            eq += 1;
            const int32_t i = a.index(e);
            imin = min(imin, i);
            imax = max(imax, i);
        }
    }
    const uint32_t need = (uint32_t)k - blk_sum<NT>(gt, S, parity, bar, tid);
    const uint32_t neq = blk_sum<NT>(eq, S, parity, bar, tid);
    uint32_t ilo = (uint32_t)imin, ihi = (uint32_t)imax;
    blk_minmax<NT>(ilo, ihi, S, parity, bar, tid);
    if (need == neq) return make_key(s, (int32_t)ihi);  // every tie is selected
    // Entries are in ascending index order, so the need-th lowest index among
    // the ties is the index of the need-th tie in position order.
    return make_key(s, nth_in_order<NT>(a, n, s, need, S, bar, tid));
}

// Writes, in order, the entries of [0, n) whose key is >= kth to out_so /
// out_ix (out_so may be null) and returns their count.  A round covers 8 * NT
// consecutive entries, thread tid holding entries tid, tid + NT, ... (so the
// reads are bank-conflict free); every read of a round lands in registers
// before the round writes anything, and a round never writes past the end of
// its own range, so the output may alias a flat input.
template <int NT, class A>
__device__ int compact(const A& a, int n, uint64_t kth, uint32_t* out_so, int32_t* out_ix,
                       Scratch<NT>& S, uint32_t bar, int tid) {
    constexpr int NW = NT / 32;
    constexpr int NC = 8 * NW;            // counts per round, u-major then warp
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t below = (1u << lane) - 1u;
    int out_base = 0;
    for (int r0 = 0; r0 < n; r0 += 8 * NT) {
        uint32_t o8[8];
        int32_t i8[8];
        uint32_t bal[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = r0 + u * NT + tid;
            bool keep = false;
            o8[u] = 0;
            i8[u] = 0;
            if (e < n) {
                o8[u] = a.ord(e);
                i8[u] = a.index(e);
                keep = make_key(o8[u], i8[u]) >= kth;
            }
            bal[u] = __ballot_sync(0xffffffffu, keep);
        }
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < 8; ++u) S.csum[u * NW + warp] = __popc(bal[u]);
        }
        named_bar_sync(bar, NT);
        if (warp == 0) {  // exclusive scan of the NC counts, in place
            constexpr int PER = (NC + 31) / 32;
            int v[PER], s = 0;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = lane * PER + q;
                v[q] = i < NC ? S.csum[i] : 0;
                s += v[q];
            }
            int incl = s;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int run = incl - s;
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = lane * PER + q;
                if (i < NC) S.csum[i] = run;
                run += v[q];
            }
            if (lane == 31) S.total = incl;  // kept entries in the round
        }
        named_bar_sync(bar, NT);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if ((bal[u] >> lane) & 1u) {
                const int pos = out_base + S.csum[u * NW + warp] + __popc(bal[u] & below);
                if (out_so) out_so[pos] = o8[u];
                out_ix[pos] = i8[u];
            }
        }
        out_base += S.total;
        named_bar_sync(bar, NT);
    }
    return out_base;
}

// A threshold ord th with k <= count(ord >= th) <= max_keep, found from a
// sample: each thread contributes one cached score, the sample's rank that
// matches k plus a margin of three standard errors gives th, and one counting
// pass checks both bounds.  Returns 0 when the check fails (the caller then
// selects exactly).
// Keeping every entry with ord >= th is a valid compaction: at least k kept
// entries beat any later key whose ord is <= th.
template <int R>
__device__ uint32_t sampled_threshold(const uint32_t (&oc)[R], int n, int k, int max_keep,
                                      Scratch<128>& S, int& parity, uint32_t bar, int tid) {
    const int rounds = (n + 127) / 128;
    const int pick = tid % rounds;
    uint32_t mine = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) mine = r == pick ? oc[r] : mine;
    if (tid + pick * 128 >= n) mine = 0;
    S.samp[tid] = mine;
    named_bar_sync(bar, 128);
    // rank of this sample (descending; ties by thread id)
    int rank = 0;
    const uint4* s4 = reinterpret_cast<const uint4*>(S.samp);
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
        const uint4 v = s4[i];
        rank += (v.x > mine) || (v.x == mine && 4 * i + 0 < tid);
        rank += (v.y > mine) || (v.y == mine && 4 * i + 1 < tid);
        rank += (v.z > mine) || (v.z == mine && 4 * i + 2 < tid);
        rank += (v.w > mine) || (v.w == mine && 4 * i + 3 < tid);
    }
    // target: k plus 3 sigma of the sample quantile, in entries
    const float pk = (float)k / (float)n;
    const float sig = sqrtf(pk * (1.f - pk) / 128.f);
    int target = (int)(128.f * (pk + 3.f * sig));
    target = target > 127 ? 127 : target;
    named_bar_sync(bar, 128);  // every rank read the samples before they are overwritten
    if (rank == target) S.samp[0] = mine;
    named_bar_sync(bar, 128);
    const uint32_t th = S.samp[0];
    uint32_t c = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) c += oc[r] >= th;
    const uint32_t tot = blk_sum<128>(c, S, parity, bar, tid);
    return (th != 0 && tot >= (uint32_t)k && (int)tot <= max_keep) ? th : 0u;
}

// Intermediate compaction of a flat buffer of n <= 32 * 128 entries: keeps,
// in order, every entry whose ord is at least th, where th is the element of
// descending rank `target` of a 128-entry sample (one cached score per
// thread), provided that leaves between k and max_keep entries; otherwise
// returns false with the buffer untouched.  One warp (sel_warp) finds th by
// a bitwise search over the sample; the counts per (round, warp) go through
// one barrier, and the indices of kept entries are read before it, so the
// writes after it may land on entries that other threads have read already:
// the compaction runs in place with three barriers.
__device__ bool compact_sampled(uint32_t* so, int32_t* ix, int& n_io, int k, int max_keep,
                                Scratch<128>& S, uint32_t bar, int tid, int sel_warp,
                                uint32_t& th_out) {
    constexpr int R = 32;
    const int n = n_io;
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t oc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = tid + r * 128;
        oc[r] = e < n ? so[e] : 0u;
    }
    // ---- sample: entry tid + pick * 128 of every thread
    const int rounds = (n + 127) / 128;
    const int pick = tid % rounds;
    uint32_t mine = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) mine = r == pick ? oc[r] : mine;
    if (tid + pick * 128 >= n) mine = 0;
    S.samp[tid] = mine;
    // target rank: k plus three standard errors of the sample quantile
    const float pk = (float)k / (float)n;
    const float sig = sqrtf(pk * (1.f - pk) / 128.f);
    int target = (int)(128.f * (pk + 3.f * sig));
    target = target > 127 ? 127 : target;
    named_bar_sync(bar, 128);
    if (warp == sel_warp) {
        // the largest x with at least target + 1 samples >= x: that sample
        const uint4 v = reinterpret_cast<const uint4*>(S.samp)[lane];
        uint32_t x = 0;
#pragma unroll 4
        for (int b = 31; b >= 0; --b) {
            const uint32_t c = x | (1u << b);
            const uint32_t m = __reduce_add_sync(
                0xffffffffu, (uint32_t)(v.x >= c) + (uint32_t)(v.y >= c) + (uint32_t)(v.z >= c) +
                                 (uint32_t)(v.w >= c));
            if (m >= (uint32_t)target + 1u) x = c;
        }
        if (lane == 0) S.total = (int)x;
    }
    named_bar_sync(bar, 128);
    const uint32_t th = (uint32_t)S.total;
    // ---- kept entries per (round, warp); indices of kept entries to registers
    int32_t ic[R];
    int* cnt4 = reinterpret_cast<int*>(S.samp);  // the sample is no longer read
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = tid + r * 128;
        const bool keep = e < n && oc[r] >= th;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) cnt4[r * 4 + warp] = __popc(bal);
        ic[r] = keep ? ix[e] : 0;
    }
    named_bar_sync(bar, 128);
    // lane r scans round r: exclusive prefix of the rounds before it, plus
    // the warps before this one within the round
    const int4 c4 = reinterpret_cast<const int4*>(cnt4)[lane];
    const int tot = c4.x + c4.y + c4.z + c4.w;
    int incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    const int basew =
        incl - tot + (warp > 0 ? c4.x : 0) + (warp > 1 ? c4.y : 0) + (warp > 2 ? c4.z : 0);
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (th == 0 || total < k || total > max_keep) return false;  // same answer in every thread
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int b = __shfl_sync(0xffffffffu, basew, r);
        const int e = tid + r * 128;
        const bool keep = e < n && oc[r] >= th;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const int pos = b + __popc(bal & below);
            so[pos] = oc[r];
            ix[pos] = ic[r];
        }
    }
    n_io = total;
    th_out = th;
    return true;
}

// Compaction of G streams at once (all G * 128 threads, stream j being
// warpgroup j) whose keys are disjoint parts of ONE query's key set: a key
// that k keys of the union beat can be dropped from any stream, so all
// streams share one threshold th taken at the union's rank k (plus a margin)
// from a 128-entry sample of each stream, weighted by the streams' sizes
// ng[].  Each stream keeps its entries >= th, in order (its count may fall
// below k).  Returns false, with nothing written, if th would leave fewer
// than k entries in the union or more than max_keep in any one stream.
// Streams hold at most 32 * 128 entries each.
template <int G>
__device__ bool compact_union(uint32_t* so, int32_t* ix, int& n_io, const int (&ng)[G], int k,
                              int max_keep, Scratch<128>& S, Scratch<G * 128>& SA, uint32_t bar,
                              uint32_t gbar, int j, int tid, uint32_t& th_out) {
    constexpr int R = 32, NT = G * 128;
    static_assert(NT / 32 == 4 * G && G <= 4, "one sampling lane group per stream");
    const int n = n_io;
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t oc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = tid + r * 128;
        oc[r] = e < n ? so[e] : 0u;
    }
    const int rounds = n > 0 ? (n + 127) / 128 : 1;
    const int pick = tid % rounds;
    uint32_t mine = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) mine = r == pick ? oc[r] : mine;
    SA.samp[j * 128 + tid] = mine;  // 0 (below everything) where there is no entry
    int ntot = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) ntot += ng[g];
    // union rank to aim at: k plus three standard errors of the sample quantile
    const float pk = (float)k / (float)ntot;
    const float sig = sqrtf(pk * (1.f - pk) / (float)NT);
    const float tgt = (pk + 3.f * sig) * (float)ntot;
    const uint32_t target128 = (uint32_t)(tgt * 128.f);  // sample weights are ng / 128
    named_bar_sync(gbar, NT);
    if (j == 0 && warp == 0) {
        // lane l holds samples PER l .. PER l + PER - 1, all of stream PER l / 128
        constexpr int PER = NT / 32;
        uint32_t v[PER];
#pragma unroll
        for (int i = 0; i < PER / 4; ++i) {
            const uint4 q4 = reinterpret_cast<const uint4*>(SA.samp)[lane * (PER / 4) + i];
            v[4 * i] = q4.x; v[4 * i + 1] = q4.y; v[4 * i + 2] = q4.z; v[4 * i + 3] = q4.w;
        }
        const uint32_t wt = (uint32_t)ng[(lane * PER) / 128];
        uint32_t x = 0;
#pragma unroll 2
        for (int b = 31; b >= 0; --b) {
            const uint32_t c = x | (1u << b);
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < PER; ++i) m += (uint32_t)(v[i] >= c);
            if (__reduce_add_sync(0xffffffffu, m * wt) >= target128) x = c;
        }
        if (lane == 0) SA.total = (int)x;
    }
    named_bar_sync(gbar, NT);
    const uint32_t th = (uint32_t)SA.total;
    int32_t ic[R];
    int* cnt4 = reinterpret_cast<int*>(S.samp);
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = tid + r * 128;
        const bool keep = e < n && oc[r] >= th;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) cnt4[r * 4 + warp] = __popc(bal);
        ic[r] = keep ? ix[e] : 0;
    }
    named_bar_sync(bar, 128);
    const int4 c4 = reinterpret_cast<const int4*>(cnt4)[lane];
    const int tot = c4.x + c4.y + c4.z + c4.w;
    int incl = tot;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    const int basew =
        incl - tot + (warp > 0 ? c4.x : 0) + (warp > 1 ? c4.y : 0) + (warp > 2 ? c4.z : 0);
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (tid == 0) SA.red[0][j] = (uint32_t)total;
    named_bar_sync(gbar, NT);
    int utot = 0, umax = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        utot += (int)SA.red[0][g];
        umax = max(umax, (int)SA.red[0][g]);
    }
    // valid when the union keeps at least k; useful when no stream keeps
    // more than max_keep (each keeps about a G-th of the union)
    if (th == 0 || utot < k || umax > max_keep) return false;  // same answer everywhere
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int b = __shfl_sync(0xffffffffu, basew, r);
        const int e = tid + r * 128;
        const bool keep = e < n && oc[r] >= th;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
            const int pos = b + __popc(bal & below);
            so[pos] = oc[r];
            ix[pos] = ic[r];
        }
    }
    n_io = total;
    th_out = th;
    return true;
}

// Streaming top-k of one query over keys offered in batches of up to T tiles
// of 128 (one key per thread of a warpgroup per tile, warp q holding keys
// 32q..32q+31 of each tile), in ascending key order across batches.
// Candidates that beat the threshold go to a buffer in key order; when it
// fills, the k best are kept in order and the threshold rises to the k-th
// score.  A later key that only ties the threshold can never enter (it would
// lose the tie on its higher index), so `ord > theta` is exact.
//
// Several such streams (one per warpgroup, G of them) run in lockstep: each
// batch ends with one barrier over all G * 128 threads, after which every
// stream sees every stream's counts, and if any buffer is near full they all
// compact at once (each with its own warpgroup barrier), so the compactions
// overlap instead of stalling the shared MMA pipeline one after another.
template <int T, int G, bool UNION = false>
struct WgTopk {
    uint32_t* so;
    int32_t* ix;
    Scratch<128>* S;
    int (*wcnt)[G][T][4];  // [2][G][T][4] per-warp append counts of the batch
    int (*cnts)[G];        // [2][G] buffer counts at the start of the batch
    int j;                 // this stream
    int cap, k;
    uint32_t bar;          // this warpgroup's barrier
    uint32_t gbar;         // barrier over all G warpgroups
    int tid;
    uint32_t theta;        // ord of the threshold score (0: take everything)
    int cnt;
    int parity;            // batch parity: both shared arrays are double-buffered by it
    // UNION: the G streams split one query's keys; compactions then use one
    // threshold for the union (compact_union), with this scratch.
    Scratch<G * 128>* SA = nullptr;

    // Call once, before the first offer, from every thread of the stream.
    __device__ __forceinline__ void start() {
        cnt = 0;
        theta = 0u;
        if (tid == 0) cnts[parity][j] = 0;
    }

    // o[u]: ordered score of this thread's key in tile u of the batch, 0 when
    // the key is not visible (0 is below every threshold); its index is
    // s0 + 128 u.
    __device__ __forceinline__ void offer(const uint32_t (&o)[T], int32_t s0, int ntile) {
        const int lane = tid & 31, q = tid >> 5;
        uint32_t bal[T];
#pragma unroll
        for (int u = 0; u < T; ++u) {
            // One stream: a later key that only ties the threshold loses on its
            // index, so it is not offered.  UNION streams interleave index
            // ranges, so ties are kept and the final selection orders them.
            const bool pass = UNION ? (o[u] != 0u && o[u] >= theta) : o[u] > theta;
            bal[u] = __ballot_sync(0xffffffffu, u < ntile && pass);
            if (lane == 0) wcnt[parity][j][u][q] = __popc(bal[u]);
        }
        // One barrier per batch: the writes of batch b land in slot b % 2 and
        // are read only between this barrier and the next one, which no
        // thread passes before every thread has finished reading.
        named_bar_sync(gbar, G * 128);
        static_assert(G * T <= 32, "one lane per (stream, tile)");
        const uint32_t below = (1u << lane) - 1u;
        // Lane g * T + u reads the four warp counts of stream g, tile u; a
        // segmented scan over u gives every stream's count after the batch
        // and, for this warp's stream, where its offers of each tile go.
        const int gl = lane / T, ul = lane % T;
        int tot = 0, bq = 0, c0 = 0;
        if (lane < G * T) {
            const int4 w4 = *reinterpret_cast<const int4*>(wcnt[parity][gl][ul]);
            tot = w4.x + w4.y + w4.z + w4.w;
            bq = (q > 0 ? w4.x : 0) + (q > 1 ? w4.y : 0) + (q > 2 ? w4.z : 0);
            c0 = cnts[parity][gl];
        }
        int incl = tot;
#pragma unroll
        for (int d = 1; d < T; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (ul >= d) incl += y;
        }
        const int base = c0 + incl - tot + bq;  // first slot of this warp's offers of (g, u)
        const int after = c0 + __shfl_sync(0xffffffffu, incl, (gl * T + T - 1) & 31);
        const bool full =
            __any_sync(0xffffffffu, lane < G * T && ul == T - 1 && after > cap - T * 128);
        cnt = __shfl_sync(0xffffffffu, after, j * T);
#pragma unroll
        for (int u = 0; u < T; ++u) {
            const int bu = __shfl_sync(0xffffffffu, base, j * T + u);
            if ((bal[u] >> lane) & 1u) {
                const int pos = bu + __popc(bal[u] & below);
                so[pos] = o[u];
                ix[pos] = s0 + u * 128;
            }
        }
        parity ^= 1;
        if (full) {  // every stream at once
            if constexpr (UNION) {
                int ng[G];
#pragma unroll
                for (int g = 0; g < G; ++g) ng[g] = __shfl_sync(0xffffffffu, after, (g * T + T - 1) & 31);
                reduce_union(ng);
            } else {
                reduce(false);
            }
        } else if (tid == 0) {
            cnts[parity][j] = cnt;
        }
    }

    // Union compaction (UNION streams); falls back to each stream's own
    // exact k-th when the shared threshold is out of bounds.
    __device__ void reduce_union(const int (&ng)[G]) {
        named_bar_sync(bar, 128);
        bool done = false, small = true;
#pragma unroll
        for (int g = 0; g < G; ++g) small = small && ng[g] <= 32 * 128;
        if (small) {
            const int max_keep = (k + (cap - T * 128)) / 2;
            uint32_t th = 0;
            done = compact_union<G>(so, ix, cnt, ng, k, max_keep, *S, *SA, bar, gbar, j, tid, th);
            if (done) theta = th;
            else named_bar_sync(bar, 128);  // this stream's threads are past the counts
        }
        if (!done && cnt > k) {
            const FlatAccess a{so, ix};
            const uint64_t kth = kth_largest<128, 32>(a, cnt, k, theta, *S, bar, tid);
            cnt = compact<128>(a, cnt, kth, so, ix, *S, bar, tid);
            theta = (uint32_t)(kth >> 32);
        }
        if (tid == 0) cnts[parity][j] = cnt;
    }

    // UNION streams at the end of their keys: one more union compaction when
    // the union holds more than max_keep entries (all G * 128 threads).
    __device__ void shrink_union() {
        named_bar_sync(gbar, G * 128);
        int ng[G], ntot = 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            ng[g] = cnts[parity][g];
            ntot += ng[g];
        }
        const int max_keep = (k + (cap - T * 128)) / 2;
        bool small = true;
#pragma unroll
        for (int g = 0; g < G; ++g) small = small && ng[g] <= 32 * 128;
        if (ntot > max_keep && small) {
            uint32_t th = 0;
            if (compact_union<G>(so, ix, cnt, ng, k, max_keep, *S, *SA, bar, gbar, j, tid, th))
                theta = th;
        }
        named_bar_sync(gbar, G * 128);
    }

    // Shrinks the buffer and publishes the count for the next batch.  The
    // final call (exact = true) keeps exactly the k best, in key order; the
    // intermediate ones keep every entry at or above a sampled threshold
    // (at least k of them), which is cheaper and equally safe.
    __device__ void reduce(bool exact) {
        named_bar_sync(bar, 128);
        if (cnt > k) {
            bool done = false;
            if (!exact && cnt <= 32 * 128) {
                // keep at most half-way between k and the compaction trigger, so
                // the next batch always fits and the compaction frees real room
                const int max_keep = (k + (cap - T * 128)) / 2;
                uint32_t th = 0;
                done = compact_sampled(so, ix, cnt, k, max_keep, *S, bar, tid, j & 3, th);
                if (done) theta = th;
                else named_bar_sync(bar, 128);  // every thread is past the sampler
            }
            if (!done) {
                const FlatAccess a{so, ix};
                const uint64_t kth = kth_largest<128, 32>(a, cnt, k, theta, *S, bar, tid);
                cnt = compact<128>(a, cnt, kth, so, ix, *S, bar, tid);
                if (!exact) theta = (uint32_t)(kth >> 32);
            }
        }
        if (tid == 0) cnts[parity][j] = cnt;
    }
};

}  // namespace sel
}  // namespace dsa

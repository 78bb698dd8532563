// Decode: one new token per sequence over a long cache.
//
// Kwai Keye-VL-2.0 technical-report summary, section 8 (decode-time DSA):
// the same indexer -> top-k -> sparse attention for the single new query of
// each sequence, whose row is the last row of its cache.
//
// The dominant cost is the scan of the indexer-key cache (128 bytes per cached
// key), so the scan is split into equal row ranges, one per CTA, in a single
// wave: CTA c covers packed-cache rows [c R, (c+1) R).  A range may hold the
// tail of one sequence, whole short sequences and the head of another; each
// such piece is a "segment".
// Phase 1 (index): per segment the CTA loads that sequence's query block,
//          its four epilogue warpgroups each scan a contiguous quarter of the
//          segment (the MMA thread interleaves their tiles into eight TMEM
//          accumulators, N = 64 indexer heads of the one query); the quarters
//          share union thresholds, and the segment's candidates (every key at
//          or above a threshold that k of them reach) go to slot c + b.
//          Sequences and chunks are both in row order, so (c, b) pairs of
//          overlapping chunks and sequences have distinct sums c + b, and the
//          slots of sequence b are the contiguous range from
//          cache_off[b] / R + b to (cache_off[b+1] - 1) / R + b.
// Phase 2 (merge): one CTA per sequence selects the top-k of its slots'
//          lists (in key order) into the index row.
// Attention (split over index-row slices) and the split merge live in
// sparse_attn.cuh.
#pragma once

#include "index_topk.cuh"
#include "topk_select.cuh"

namespace dsa {
namespace dec {

using idx::kKeyTile;
using sel::FlatAccess;
using sel::Scratch;
using sel::SegAccess;
using sel::WgTopk;

constexpr int HI = 64;
constexpr int DI = 128;
constexpr int kStages = 5;        // HBM-bound: keep more key tiles in flight
constexpr int kBatch = 4;         // tiles offered to the top-k per barrier
// Candidate buffer entries per query: room for the k kept plus one batch of
// offers, and 2k so that a compaction frees at least k.
__host__ __device__ constexpr int cand_capacity(int k) {
    const int c = 2 * k > k + kBatch * kKeyTile ? 2 * k : k + kBatch * kKeyTile;
    return (c + 127) / 128 * 128;
}
// Entries of one chunk slot in the workspace: a chunk hands its union of
// candidates (at or above a shared threshold, at least k) to the per-sequence
// merge as it is when it fits, and selects exactly k itself only when not.
__host__ __device__ constexpr int slot_capacity(int k) { return (k + k / 2 + 127) / 128 * 128; }
constexpr int kEpiWarps = 16;     // warps 0-15: four warpgroups, one per chunk quarter
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 20 * 32;  // warps 18-19 idle: warpgroup 4 is whole for setmaxnreg
// Register split (setmaxnreg): the launch gives every thread 96 registers (20
// warps: five per scheduler, whose register file holds 5 x 32 x 96 of its
// 16 K), warpgroup 4 (producer, MMA issuer, two idle warps) drops to 56 and
// the four epilogue warpgroups rise to 104, without spills.
constexpr int kEpiRegs = 104;
constexpr int kCtlRegs = 56;
static_assert(4 * 128 * kEpiRegs + 128 * kCtlRegs <= kThreads * 96, "register split");

struct Params {
    const float* w;            // [B][HI]
    const int64_t* cache_off;  // [B + 1]
    int B;
    int64_t total_n;           // rows of the packed caches
    int k;
    int64_t R;                 // cache rows per CTA
    uint32_t* cand_so;         // [slots][slot_capacity(k)] ordered scores (topk_select.cuh)
    int32_t* cand_ix;
    int* cand_cnt;             // [slots]
    uint32_t* cand_th;         // [slots] an ord that at least k of the slot's entries reach
                               // (0 when the slot holds fewer than k or none is known)
    int* err;                  // the call's device error word (null: the per-device word)
    // Cache shards (one part of every sequence's cache per rank): the merge
    // also writes each kept key's ordered score, adds key_base[b] to the
    // keys, and a sequence with no rows here is not an error.
    uint32_t* ord_out;         // [B][k] or null
    const int64_t* key_base;   // [B] or null (0)
    int allow_empty;
};

__device__ __forceinline__ bool seq_ok(const Params& p, int b) {
    const int64_t lo = p.cache_off[b], hi = p.cache_off[b + 1];
    return lo >= 0 && hi > lo && hi <= p.total_n;
}


struct Misc {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t qfull;
    uint64_t qfree;
    uint64_t accfull[4][2];
    uint64_t accempty[4][2];
    uint64_t mma_done;
    alignas(16) int wcnt[2][4][kBatch][4];  // rows read as int4 by WgTopk::offer
    int cnts[2][4];
    int cnt[4];
    uint32_t thr[4];
    uint32_t tmem_base;
    volatile int abort_flag;
};

static_assert(offsetof(Misc, wcnt) % 16 == 0, "wcnt rows are read as int4");

struct Layout {
    int q, stage, w, cs, ci, scratch, scratch_all, misc, total;
    __host__ __device__ explicit Layout(int k) {
        const int cap = cand_capacity(k);
        q = 0;
        stage = HI * DI;                       // 8 KB, 1024-aligned
        w = stage + kStages * kKeyTile * DI;   // one copy of the head weights per warpgroup
        cs = w + 4 * HI * 4;
        ci = cs + 4 * cap * 4;
        scratch = (ci + 4 * cap * 4 + 15) / 16 * 16;
        scratch_all = scratch + 4 * (int)sizeof(Scratch<128>);
        misc = (scratch_all + (int)sizeof(Scratch<512>) + 15) / 16 * 16;
        total = misc + (int)sizeof(Misc);
    }
};

// One piece of a sequence inside this CTA's row range.
struct Segment {
    int b;            // sequence
    int64_t base;     // first cache row of the sequence
    int64_t lo, len;  // sequence-local first key and length of the piece
    int sub;          // keys per quarter (a multiple of the tile)
    // tiles of quarter w
    __device__ __forceinline__ int tiles(int w) const {
        int64_t l = len - (int64_t)w * sub;
        l = l < 0 ? 0 : (l > sub ? sub : l);
        return (int)((l + kKeyTile - 1) / kKeyTile);
    }
};

// Segments of CTA c are the valid sequences overlapping [r0, r1), in order.
// first_seq: the last b with cache_off[b] <= r0.
__device__ __forceinline__ int first_seq(const Params& p, int64_t r0) {
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cache_off[mid] <= r0) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ bool make_segment(const Params& p, int b, int64_t r0, int64_t r1,
                                             Segment& g) {
    if (!seq_ok(p, b)) return false;
    const int64_t off = p.cache_off[b], end = p.cache_off[b + 1];
    const int64_t a = off > r0 ? off : r0, z = end < r1 ? end : r1;
    if (z <= a) return false;
    g.b = b;
    g.base = off;
    g.lo = a - off;
    g.len = z - a;
    g.sub = (int)((g.len + 4 * kKeyTile - 1) / (4 * kKeyTile) * kKeyTile);
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
index_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
             const Params p) {
    constexpr int N = HI;
    constexpr int KT_BYTES = kKeyTile * DI;
    constexpr uint32_t TMEM_COLS = 512;  // 4 warpgroups x 2 accumulators x 64 columns
    constexpr uint32_t IDESC = idesc_e4m3_f32(N);

    pdl_wait();  // the caches and queries may come from the previous kernel
    pdl_launch_dependents();
    const int c = blockIdx.x;
    const int64_t r0 = (int64_t)c * p.R;
    const int64_t r1 = r0 + p.R < p.total_n ? r0 + p.R : p.total_n;
    if (r0 >= r1) return;  // more CTAs than ranges: nothing to do

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Aligned by pointer arithmetic on the shared array itself (not through an
    // integer), so that the compiler keeps every access in the shared window
    // (ld/st.shared with 32-bit addresses instead of generic ones).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Layout lay(p.k);
    const int cap = cand_capacity(p.k);
    Misc* misc = reinterpret_cast<Misc*>(smem + lay.misc);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&misc->full[s]), 1);
            mbar_init(smem_u32(&misc->empty[s]), 1);
        }
        mbar_init(smem_u32(&misc->qfull), 1);
        mbar_init(smem_u32(&misc->qfree), 1);
        for (int w = 0; w < 4; ++w)
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&misc->accfull[w][b]), 1);
                mbar_init(smem_u32(&misc->accempty[w][b]), 4);
            }
        mbar_init(smem_u32(&misc->mma_done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kProducerWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc->tmem_base;
    const int b_first = first_seq(p, r0);
    if (warp >= kEpiWarps) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));

    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            const uint32_t qbar = smem_u32(&misc->qfull);
            int i = 0, nseg = 0;
            bool ok = true;
            Segment g;
            for (int b = b_first; ok && b < p.B && p.cache_off[b] < r1; ++b) {
                if (!make_segment(p, b, r0, r1, g)) continue;
                // the previous segment's MMAs must be done with the query block
                if (nseg > 0 && !mbar_wait_to(p.err, smem_u32(&misc->qfree), (nseg - 1) & 1)) {
                    misc->abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(qbar, HI * DI);
                tma_load_2d(smem_u32(smem + lay.q), &tmap_q, qbar, 0, g.b * HI);
                ++nseg;
                const int nt0 = g.tiles(0);
                for (int u = 0; ok && u < nt0; ++u)
                    for (int w = 0; w < 4; ++w) {
                        if (u >= g.tiles(w)) continue;
                        if (misc->abort_flag) { ok = false; break; }
                        const int s = i % kStages;
                        if (i >= kStages &&
                            !mbar_wait_to(p.err, smem_u32(&misc->empty[s]), ((i / kStages) - 1) & 1)) {
                            misc->abort_flag = 1;
                            ok = false;
                            break;
                        }
                        const uint32_t fb = smem_u32(&misc->full[s]);
                        mbar_arrive_expect_tx(fb, KT_BYTES);
                        const int64_t row = g.base + g.lo + (int64_t)w * g.sub + (int64_t)u * kKeyTile;
                        tma_load_2d(smem_u32(smem + lay.stage + s * KT_BYTES), &tmap_k, fb, 0,
                                    (int32_t)row);
                        ++i;
                    }
            }
            // Never leave with a copy in flight.
            if (nseg > 0) mbar_wait_to(p.err, qbar, (nseg - 1) & 1);
            for (int e = i - kStages < 0 ? 0 : i - kStages; e < i; ++e)
                mbar_wait_to(p.err, smem_u32(&misc->full[e % kStages]), (e / kStages) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t bdesc = smem_desc_kmajor(smem_u32(smem + lay.q), DI);
            int i = 0, nseg = 0;
            int uses[4] = {0, 0, 0, 0};
            bool ok = true;
            Segment g;
            for (int b = b_first; ok && b < p.B && p.cache_off[b] < r1; ++b) {
                if (!make_segment(p, b, r0, r1, g)) continue;
                ok = mbar_wait_to(p.err, smem_u32(&misc->qfull), nseg & 1);
                ++nseg;
                const int nt0 = g.tiles(0);
                for (int u = 0; ok && u < nt0; ++u)
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        if (!ok || u >= g.tiles(w)) continue;
                        if (misc->abort_flag) { ok = false; continue; }
                        const int s = i % kStages;
                        const int use = uses[w]++;
                        const int buf = use & 1;
                        ok = mbar_wait_to(p.err, smem_u32(&misc->full[s]), (i / kStages) & 1);
                        if (ok && use >= 2)
                            ok = mbar_wait_to(p.err, smem_u32(&misc->accempty[w][buf]), ((use >> 1) - 1) & 1);
                        if (!ok) continue;
                        tc_fence_after();
                        const uint64_t adesc =
                            smem_desc_kmajor(smem_u32(smem + lay.stage + s * KT_BYTES), DI);
                        const uint32_t d_tmem = tmem_base + (uint32_t)((w * 2 + buf) * N);
#pragma unroll
                        for (int kk = 0; kk < DI / 32; ++kk)
                            umma_f8f6f4(d_tmem, adesc + (uint64_t)(2 * kk),
                                        bdesc + (uint64_t)(2 * kk), IDESC, kk > 0 ? 1u : 0u);
                        umma_commit(smem_u32(&misc->empty[s]));
                        umma_commit(smem_u32(&misc->accfull[w][buf]));
                        ++i;
                    }
                umma_commit(smem_u32(&misc->qfree));  // query block free once these retire
            }
            if (!ok) misc->abort_flag = 1;
            umma_commit(smem_u32(&misc->mma_done));
            mbar_wait_to(p.err, smem_u32(&misc->mma_done), 0);
        }
    } else if (warp < kEpiWarps) {
        // ------------------------------------------------ epilogue (warps 0-15)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
        const int w = warp >> 2;               // quarter of each segment
        const int q = warp & 3;                // TMEM lane quarter
        const int tid = threadIdx.x - w * 128;
        const int t512 = threadIdx.x;
        const uint32_t bar = 1 + w;
        uint32_t* so = reinterpret_cast<uint32_t*>(smem + lay.cs) + w * cap;
        int32_t* ix = reinterpret_cast<int32_t*>(smem + lay.ci) + w * cap;
        float* w_s = reinterpret_cast<float*>(smem + lay.w) + w * HI;
        Scratch<128>* S = reinterpret_cast<Scratch<128>*>(smem + lay.scratch) + w;
        constexpr int T = kBatch;
        int use = 0;
        Segment g;
        for (int b = b_first; b < p.B && p.cache_off[b] < r1; ++b) {
            if (!make_segment(p, b, r0, r1, g)) continue;
            if (tid < HI) w_s[tid] = p.w[(int64_t)g.b * HI + tid];
            named_bar_sync(bar, 128);
            // the four quarters split one query's keys: one threshold for the union
            WgTopk<T, 4, true> tk{so, ix, S, misc->wcnt, misc->cnts, w, cap, p.k, bar, 5, tid,
                                  0u, 0, 0, reinterpret_cast<Scratch<512>*>(smem + lay.scratch_all)};
            tk.start();
            const int64_t qlo = g.lo + (int64_t)w * g.sub;
            const int64_t qend = g.lo + ((int64_t)(w + 1) * g.sub < g.len ? (int64_t)(w + 1) * g.sub
                                                                          : g.len);
            const int ntw = g.tiles(w);
            const int nt0 = g.tiles(0);  // quarter 0 has the most tiles: every warpgroup
                                         // runs its batch count, offering nothing at the end
            for (int u0 = 0; u0 < nt0; u0 += T) {
                uint32_t o[T];  // ord of this thread's key in each tile; 0 = not offered
#pragma unroll
                for (int v = 0; v < T; ++v) {
                    const int u = u0 + v;
                    o[v] = 0;
                    if (u >= ntw) continue;
                    const int buf = use & 1;
                    if (!misc->abort_flag &&
                        !mbar_wait_to(p.err, smem_u32(&misc->accfull[w][buf]), (use >> 1) & 1))
                        misc->abort_flag = 1;
                    tc_fence_after();
                    const uint32_t taddr =
                        tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((w * 2 + buf) * N);
                    const float score = idx::head_sum<HI>(taddr, w_s);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&misc->accempty[w][buf]));
                    ++use;
                    const int64_t s = qlo + (int64_t)u * kKeyTile + q * 32 + lane;
                    if (s < qend) o[v] = sel::ord_f32(score);
                }
                tk.offer(o, (int32_t)(qlo + (int64_t)u0 * kKeyTile + q * 32 + lane),
                         ntw - u0 < T ? (ntw - u0 > 0 ? ntw - u0 : 0) : T);
            }
            tk.shrink_union();
            if (tid == 0) {
                misc->cnt[w] = tk.cnt;
                misc->thr[w] = tk.theta;
            }
            // ---- merge the four quarter lists into the segment's top-k
            named_bar_sync(5, 512);
            SegAccess a;
            a.start[0] = 0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                a.so[v] = reinterpret_cast<uint32_t*>(smem + lay.cs) + v * cap;
                a.ix[v] = reinterpret_cast<int32_t*>(smem + lay.ci) + v * cap;
                a.start[v + 1] = a.start[v] + misc->cnt[v];
            }
            const int n = a.start[4];
            const int slot = (int)(r0 / p.R) + g.b;  // distinct over (chunk, sequence) pairs
            uint32_t* oso = p.cand_so + (int64_t)slot * slot_capacity(p.k);
            int32_t* oix = p.cand_ix + (int64_t)slot * slot_capacity(p.k);
            int outn;
            if (n <= slot_capacity(p.k)) {  // the merge selects the k
                for (int e = t512; e < n; e += 512) {
                    oso[e] = a.ord(e);
                    oix[e] = a.index(e);
                }
                outn = n;
            } else {
                Scratch<512>* SA = reinterpret_cast<Scratch<512>*>(smem + lay.scratch_all);
                const uint64_t kth = sel::kth_largest<512, 16>(a, n, p.k, 0u, *SA, 5, t512);
                outn = sel::compact<512>(a, n, kth, oso, oix, *SA, 5, t512);
            }
            if (t512 == 0) {
                p.cand_cnt[slot] = misc->abort_flag ? 0 : outn;
                // each quarter's threshold is one that k entries of the union
                // reach (a shared one, or the quarter's own exact k-th), and
                // every entry at or above it is in the slot
                uint32_t th = 0;
                for (int v = 0; v < 4; ++v) th = max(th, misc->thr[v]);
                p.cand_th[slot] = outn >= p.k ? th : 0u;
            }
            named_bar_sync(5, 512);  // the lists are read before the next segment refills them
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kProducerWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// Per-sequence top-k of its slots' lists -> idx[b][0..k) ascending, -1 pad.
// The lists are gathered into one run (shared memory when they fit in
// smem_cap entries, else in place in the candidate arrays), then selected.
__global__ void __launch_bounds__(1024) merge_kernel(const Params p, int32_t* idx_out,
                                                      int smem_cap) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ Scratch<1024> S;
    __shared__ int total_s;
    __shared__ uint32_t floor_s;
    pdl_wait();  // the slots come from index_kernel
    pdl_launch_dependents();
    const int b = blockIdx.x, tid = threadIdx.x;
    int32_t* out = idx_out + (int64_t)b * p.k;
    // A sequence whose rows are empty, out of [0, total_n) or not after the
    // previous sequence's owns no slot: it records DSA_DEVERR_INDEX and its
    // index row is all -1 (its output all zeros).
    const bool ordered = b == 0 || p.cache_off[b] >= p.cache_off[b - 1];
    uint32_t* ord = p.ord_out != nullptr ? p.ord_out + (int64_t)b * p.k : nullptr;
    int s0 = 0, s1 = 0;
    if (seq_ok(p, b) && ordered) {
        s0 = (int)(p.cache_off[b] / p.R) + b;
        s1 = (int)((p.cache_off[b + 1] - 1) / p.R) + b + 1;
    } else if (tid == 0 && !(p.allow_empty && ordered && p.cache_off[b] >= 0 &&
                             p.cache_off[b] == p.cache_off[b + 1] &&
                             p.cache_off[b] <= p.total_n)) {
        record_error_to(p.err, 2);
    }
    if (s1 <= s0) {
        for (int e = tid; e < p.k; e += 1024) {
            out[e] = -1;
            if (ord) ord[e] = 0u;
        }
        return;
    }
    if (tid == 0) {
        int t = 0;
        uint32_t f = 0;
        for (int s = s0; s < s1; ++s) {
            t += p.cand_cnt[s];
            f = max(f, p.cand_th[s]);  // k entries of that slot reach it
        }
        total_s = t;
        floor_s = f;
    }
    __syncthreads();
    const int n = total_s;
    const int sc = slot_capacity(p.k);
    uint32_t* gsc = p.cand_so + (int64_t)s0 * sc;
    int32_t* gix = p.cand_ix + (int64_t)s0 * sc;
    FlatAccess a{gsc, gix};
    if (n <= smem_cap) {
        uint32_t* ssc = reinterpret_cast<uint32_t*>(smem);
        int32_t* six = reinterpret_cast<int32_t*>(smem + (size_t)smem_cap * 4);
        int at = 0;
        for (int s = s0; s < s1; ++s) {
            const int cnt = p.cand_cnt[s];
            const uint32_t* fs = p.cand_so + (int64_t)s * sc;
            const int32_t* fi = p.cand_ix + (int64_t)s * sc;
            for (int e = tid; e < cnt; e += 1024) {
                ssc[at + e] = fs[e];
                six[at + e] = fi[e];
            }
            at += cnt;
        }
        __syncthreads();
        a = FlatAccess{ssc, six};
    } else {
        // Close the gaps between the slots, leftwards, one slot and one chunk
        // of 1024 entries at a time (a chunk's writes end at or before the
        // next chunk's first read, so ascending chunks never overwrite
        // unread entries).
        int at = 0;
        for (int s = s0; s < s1; ++s) {
            const int cnt = p.cand_cnt[s];
            const int from = (s - s0) * sc;
            for (int c0 = 0; c0 < cnt; c0 += 1024) {
                const int e = c0 + tid;
                uint32_t v = 0;
                int32_t x = 0;
                if (e < cnt) {
                    v = gsc[from + e];
                    x = gix[from + e];
                }
                __syncthreads();
                if (e < cnt) {
                    gsc[at + e] = v;
                    gix[at + e] = x;
                }
                __syncthreads();
            }
            at += cnt;
        }
    }
    int cnt = n;
    if (n > p.k) {
        const uint64_t kth = sel::kth_largest<1024, 24>(a, n, p.k, floor_s, S, 0, tid);
        // Only the selected k entries land in the index row.
        cnt = sel::compact<1024>(a, n, kth, ord, out, S, 0, tid);
    } else {
        for (int e = tid; e < n; e += 1024) {
            out[e] = a.index(e);
            if (ord) ord[e] = a.ord(e);
        }
    }
    __syncthreads();
    if (p.key_base != nullptr) {
        const int32_t base = (int32_t)p.key_base[b];
        for (int e = tid; e < cnt; e += 1024) out[e] += base;
    }
    for (int e = cnt + tid; e < p.k; e += 1024) {
        out[e] = -1;
        if (ord) ord[e] = 0u;
    }
}

// Cache shards: the exact top-k of one sequence over the P shards' kept
// (ordered score, global key) lists, ord_in / key_in [P][B][k] (each list in
// ascending key order, -1 padded; shard r's keys all precede shard r+1's).
// The global top-k is contained in the union of the shards' top-k lists
// (any key that k keys of its own shard beat is beaten by k keys overall),
// and the order (score, then lower key) is the same total order, so the row
// equals the one a single decode over the whole cache selects.  One CTA per
// sequence; the lists are gathered into shared memory in shard order, which
// is key order.
constexpr int kMaxShards = 8;

__global__ void __launch_bounds__(1024) merge_shards_kernel(const uint32_t* ord_in,
                                                             const int32_t* key_in, int P, int B,
                                                             int k, int32_t* idx_out, int* err) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ Scratch<1024> S;
    __shared__ int cnt_s[kMaxShards + 1];
    const int b = blockIdx.x, tid = threadIdx.x;
    uint32_t* so = reinterpret_cast<uint32_t*>(smem);
    int32_t* si = reinterpret_cast<int32_t*>(smem + (size_t)P * k * 4);
    if (tid < P) {  // valid entries lead every list
        const int32_t* kl = key_in + ((int64_t)tid * B + b) * k;
        int lo = 0, hi = k;  // the first -1
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (kl[mid] >= 0) lo = mid + 1;
            else hi = mid;
        }
        cnt_s[tid + 1] = lo;
    }
    __syncthreads();
    if (tid == 0) {
        cnt_s[0] = 0;
        for (int r = 0; r < P; ++r) cnt_s[r + 1] += cnt_s[r];
    }
    __syncthreads();
    const int n = cnt_s[P];
    for (int r = 0; r < P; ++r) {
        const int c0 = cnt_s[r], c = cnt_s[r + 1] - c0;
        const uint32_t* os = ord_in + ((int64_t)r * B + b) * k;
        const int32_t* ks = key_in + ((int64_t)r * B + b) * k;
        for (int e = tid; e < c; e += 1024) {
            so[c0 + e] = os[e];
            si[c0 + e] = ks[e];
        }
    }
    __syncthreads();
    // keys must ascend along the gathered run (the output is written in it)
    for (int e = tid; e + 1 < n; e += 1024)
        if (si[e] >= si[e + 1]) record_error_to(err, 2);
    int32_t* out = idx_out + (int64_t)b * k;
    const FlatAccess a{so, si};
    int cnt = n;
    if (n > k) {
        const uint64_t kth = sel::kth_largest<1024, 16>(a, n, k, 0u, S, 0, tid);
        cnt = sel::compact<1024>(a, n, kth, static_cast<uint32_t*>(nullptr), out, S, 0, tid);
    } else {
        for (int e = tid; e < n; e += 1024) out[e] = si[e];
    }
    __syncthreads();
    for (int e = cnt + tid; e < k; e += 1024) out[e] = -1;
}

}  // namespace dec
}  // namespace dsa

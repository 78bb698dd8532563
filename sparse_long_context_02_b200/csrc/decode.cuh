// Decode: one new token per sequence over a long cache.
//
// Kwai Keye-VL-2.0 technical-report summary, section 8 (decode-time DSA):
// the same indexer -> top-k -> sparse attention for the single new query of
// each sequence, whose row is the last row of its cache.
//
// Phase 1 (prep): chunk_start[b] = sum over earlier sequences of
//          ceil(n_b / CK), so every cache chunk of CK keys gets one CTA.
// Phase 2 (index): a CTA scans one chunk.  Its four epilogue warpgroups each
//          own a contiguous quarter; the MMA issuer interleaves their tiles
//          (M = 128 keys, N = 64 indexer heads of the one query) into eight
//          TMEM accumulators, so the dominant HBM stream (128 bytes of k_I per
//          cached key) is read exactly once.  Each warpgroup keeps the top-k
//          of its quarter; the CTA then merges the four lists (which are in
//          ascending key order) into the chunk's top-k.
// Phase 3 (merge): one CTA per sequence selects the top-k of its chunks'
//          lists, again in ascending key order.  Every chunk but the last of a
//          sequence holds exactly k entries (CK >= k), so a sequence's lists
//          are one contiguous run of the candidate arrays.
// Attention (split over index-row slices) and the split merge live in
// sparse_attn.cuh.
#pragma once

#include "index_topk.cuh"

namespace dsa {
namespace dec {

using idx::kKeyTile;
using idx::kStages;
using idx::cand_capacity;
using idx::WgTopk;
using idx::FlatAccess;
using idx::SegAccess;

constexpr int HI = 64;
constexpr int DI = 128;
constexpr int kThreads = 640;
constexpr int kEpiWarps = 16;

struct Params {
    const float* w;            // [B][HI]
    const int64_t* cache_off;  // [B + 1]
    int B;
    int64_t total_n;           // rows of the packed caches
    int k;
    int ck;                    // keys per chunk (multiple of 4 * 128, >= k)
    int* chunk_start;          // [B + 1]
    float* cand_sc;            // [max_chunks][k]
    int32_t* cand_ix;
    int* cand_cnt;             // [max_chunks]
};

// chunk_start[b] for b in [0, B].  A sequence whose rows are empty or do not
// lie inside [0, total_n) owns no chunk and records DSA_DEVERR_INDEX (its
// output is then all zeros), so no later phase reads outside the caches or
// the workspace.
__global__ void __launch_bounds__(1024) prep_kernel(const Params p) {
    __shared__ int wsum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int carry = 0;
    for (int b0 = 0; b0 < p.B; b0 += 1024) {
        const int b = b0 + tid;
        int c = 0;
        if (b < p.B) {
            const int64_t lo = p.cache_off[b], hi = p.cache_off[b + 1];
            const bool good = lo >= 0 && hi > lo && hi <= p.total_n;
            if (!good) record_device_error(2);
            c = good ? (int)((hi - lo + p.ck - 1) / p.ck) : 0;
        }
        int incl = c;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int wv = 0; wv < 32; ++wv) {
            before += wv < warp ? wsum[wv] : 0;
            total += wsum[wv];
        }
        if (b < p.B) p.chunk_start[b] = carry + before + incl - c;
        carry += total;
        __syncthreads();
    }
    if (tid == 0) p.chunk_start[p.B] = carry;
}

struct Misc {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t qfull;
    uint64_t accfull[4][2];
    uint64_t accempty[4][2];
    uint64_t mma_done;
    uint64_t red64[4][4];
    uint64_t red64_all[16];
    int wcnt[4][2][4];
    int scratch[4][4];
    int wsum_all[16];
    int scratch_all[4];
    int cnt[4];
    int seq, chunk_in_seq;
    uint32_t tmem_base;
    volatile int abort_flag;
};

struct Layout {
    int q, stage, w, cs, ci, hist, misc, total;
    __host__ __device__ explicit Layout(int k) {
        const int cap = cand_capacity(k);
        q = 0;
        stage = HI * DI;                       // 8 KB, 1024-aligned
        w = stage + kStages * kKeyTile * DI;
        cs = w + HI * 4;
        ci = cs + 4 * cap * 4;
        hist = ci + 4 * cap * 4;
        misc = hist + 4 * 256 * 4;
        total = misc + 1024;
    }
};

// Tiles of warpgroup w in a chunk of `len` keys split into quarters of `sub`.
__device__ __forceinline__ int quarter_tiles(int len, int sub, int w) {
    int l = len - w * sub;
    l = l < 0 ? 0 : (l > sub ? sub : l);
    return (l + kKeyTile - 1) / kKeyTile;
}

__global__ void __launch_bounds__(kThreads, 1)
index_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
             const Params p) {
    constexpr int N = HI;
    constexpr int KT_BYTES = kKeyTile * DI;
    constexpr uint32_t TMEM_COLS = 512;  // 4 warpgroups x 2 accumulators x 64 columns
    constexpr uint32_t IDESC = idesc_e4m3_f32(N);

    const int c = blockIdx.x;
    if (c >= p.chunk_start[p.B]) return;  // more CTAs than chunks: nothing to do

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Layout lay(p.k);
    const int cap = cand_capacity(p.k);
    Misc* misc = reinterpret_cast<Misc*>(smem + lay.misc);
    float* w_s = reinterpret_cast<float*>(smem + lay.w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        int lo = 0, hi = p.B - 1;  // last b with chunk_start[b] <= c
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.chunk_start[mid] <= c) lo = mid;
            else hi = mid - 1;
        }
        misc->seq = lo;
        misc->chunk_in_seq = c - p.chunk_start[lo];
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&misc->full[s]), 1);
            mbar_init(smem_u32(&misc->empty[s]), 1);
        }
        mbar_init(smem_u32(&misc->qfull), 1);
        for (int w = 0; w < 4; ++w)
            for (int b = 0; b < 2; ++b) {
                mbar_init(smem_u32(&misc->accfull[w][b]), 1);
                mbar_init(smem_u32(&misc->accempty[w][b]), 4);
            }
        mbar_init(smem_u32(&misc->mma_done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(&misc->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc->tmem_base;
    const int b = misc->seq;
    const int64_t base = p.cache_off[b];
    const int64_t n_b = p.cache_off[b + 1] - base;
    const int64_t key0 = (int64_t)misc->chunk_in_seq * p.ck;
    const int len = (int)(n_b - key0 < p.ck ? n_b - key0 : p.ck);
    const int sub = p.ck / 4;
    for (int e = threadIdx.x; e < HI; e += kThreads) w_s[e] = p.w[(int64_t)b * HI + e];
    int nt[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) nt[w] = quarter_tiles(len, sub, w);
    const int umax = nt[0];  // quarter 0 has the most tiles
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            const uint32_t qbar = smem_u32(&misc->qfull);
            mbar_arrive_expect_tx(qbar, HI * DI);
            tma_load_2d(smem_u32(smem + lay.q), &tmap_q, qbar, 0, b * HI);
            int i = 0;
            bool ok = true;
            for (int u = 0; ok && u < umax; ++u)
                for (int w = 0; w < 4; ++w) {
                    if (u >= nt[w]) continue;
                    if (misc->abort_flag) { ok = false; break; }
                    const int s = i % kStages;
                    if (i >= kStages && !mbar_wait(smem_u32(&misc->empty[s]), ((i / kStages) - 1) & 1)) {
                        misc->abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&misc->full[s]);
                    mbar_arrive_expect_tx(fb, KT_BYTES);
                    const int64_t row = base + key0 + (int64_t)w * sub + (int64_t)u * kKeyTile;
                    tma_load_2d(smem_u32(smem + lay.stage + s * KT_BYTES), &tmap_k, fb, 0, (int32_t)row);
                    ++i;
                }
            mbar_wait(qbar, 0);
            for (int e = i - kStages < 0 ? 0 : i - kStages; e < i; ++e)
                mbar_wait(smem_u32(&misc->full[e % kStages]), (e / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(smem_u32(&misc->qfull), 0);
            const uint64_t bdesc = smem_desc_kmajor(smem_u32(smem + lay.q), DI);
            int i = 0;
            for (int u = 0; ok && u < umax; ++u)
                for (int w = 0; w < 4; ++w) {
                    if (u >= nt[w]) continue;
                    if (misc->abort_flag) { ok = false; break; }
                    const int s = i % kStages;
                    const int buf = u & 1;
                    ok = mbar_wait(smem_u32(&misc->full[s]), (i / kStages) & 1);
                    if (ok && u >= 2) ok = mbar_wait(smem_u32(&misc->accempty[w][buf]), ((u >> 1) - 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_kmajor(smem_u32(smem + lay.stage + s * KT_BYTES), DI);
                    const uint32_t d_tmem = tmem_base + (uint32_t)((w * 2 + buf) * N);
#pragma unroll
                    for (int kk = 0; kk < DI / 32; ++kk)
                        umma_f8f6f4(d_tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk),
                                    IDESC, kk > 0 ? 1u : 0u);
                    umma_commit(smem_u32(&misc->empty[s]));
                    umma_commit(smem_u32(&misc->accfull[w][buf]));
                    ++i;
                }
            if (!ok) misc->abort_flag = 1;
            umma_commit(smem_u32(&misc->mma_done));
            mbar_wait(smem_u32(&misc->mma_done), 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        const int w = (warp - 4) >> 2;         // quarter of the chunk
        const int q = warp & 3;                // TMEM lane quarter
        const int tid = threadIdx.x - 128 - w * 128;
        const uint32_t bar = 1 + w;
        float* sc = reinterpret_cast<float*>(smem + lay.cs) + w * cap;
        int32_t* ix = reinterpret_cast<int32_t*>(smem + lay.ci) + w * cap;
        int* hist = reinterpret_cast<int*>(smem + lay.hist) + w * 256;
        WgTopk tk{sc, ix, hist, misc->scratch[w], misc->red64[w], misc->wcnt[w], cap, p.k, bar,
                  tid, -INFINITY, 0};
        const int64_t qend = key0 + (int64_t)((w + 1) * sub < len ? (w + 1) * sub : len);
        bool ok = true;
        for (int u = 0; u < nt[w]; ++u) {
            const int buf = u & 1;
            bool got = mbar_wait(smem_u32(&misc->accfull[w][buf]), (u >> 1) & 1);
            if (!named_bar_and(bar, 128, got && !misc->abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((w * 2 + buf) * N);
            const float score = idx::head_sum<HI>(taddr, w_s);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->accempty[w][buf]));
            const int64_t s = key0 + (int64_t)w * sub + (int64_t)u * kKeyTile + q * 32 + lane;
            tk.offer(s < qend, score, (int32_t)s, u & 1);
        }
        int cnt = 0;
        if (ok) cnt = tk.finish();
        if (tid == 0) misc->cnt[w] = ok ? cnt : -1;
        // ---- merge the four quarter lists into the chunk's top-k
        const int t512 = threadIdx.x - 128;
        named_bar_sync(5, 512);
        const bool all_ok = misc->cnt[0] >= 0 && misc->cnt[1] >= 0 && misc->cnt[2] >= 0 &&
                            misc->cnt[3] >= 0;
        if (all_ok) {
            SegAccess a;
            a.start[0] = 0;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                a.sc[v] = reinterpret_cast<float*>(smem + lay.cs) + v * cap;
                a.ix[v] = reinterpret_cast<int32_t*>(smem + lay.ci) + v * cap;
                a.start[v + 1] = a.start[v] + misc->cnt[v];
            }
            const int n = a.start[4];
            float* osc = p.cand_sc + (int64_t)c * p.k;
            int32_t* oix = p.cand_ix + (int64_t)c * p.k;
            int outn;
            if (n <= p.k) {
                for (int e = t512; e < n; e += 512) {
                    osc[e] = a.score(e);
                    oix[e] = a.index(e);
                }
                outn = n;
            } else {
                int* hist0 = reinterpret_cast<int*>(smem + lay.hist);
                const uint64_t kth = idx::blk_kth_largest<512>(a, n, p.k, hist0, misc->scratch_all,
                                                               misc->red64_all, 5, t512);
                outn = idx::blk_compact<512>(a, n, kth, osc, oix, misc->wsum_all, 5, t512);
            }
            if (t512 == 0) p.cand_cnt[c] = outn;
        } else if (t512 == 0) {
            p.cand_cnt[c] = 0;
            misc->abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// Per-sequence top-k of its chunks' lists -> idx[b][0..k) ascending, -1 pad.
// Stages the lists in shared memory when they fit (smem_cap entries).
__global__ void __launch_bounds__(1024) merge_kernel(const Params p, int32_t* idx_out,
                                                      int smem_cap) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ int hist[256];
    __shared__ int scratch[4];
    __shared__ int wsum[32];
    __shared__ uint64_t red64[32];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int c0 = p.chunk_start[b], c1 = p.chunk_start[b + 1];
    int32_t* out = idx_out + (int64_t)b * p.k;
    if (c1 <= c0) {
        for (int e = tid; e < p.k; e += 1024) out[e] = -1;
        return;
    }
    const int n = (c1 - 1 - c0) * p.k + p.cand_cnt[c1 - 1];
    const float* gsc = p.cand_sc + (int64_t)c0 * p.k;
    const int32_t* gix = p.cand_ix + (int64_t)c0 * p.k;
    FlatAccess a{gsc, gix};
    if (n <= smem_cap) {
        float* ssc = reinterpret_cast<float*>(smem);
        int32_t* six = reinterpret_cast<int32_t*>(smem + (size_t)smem_cap * 4);
        for (int e = tid; e < n; e += 1024) {
            ssc[e] = gsc[e];
            six[e] = gix[e];
        }
        __syncthreads();
        a = FlatAccess{ssc, six};
    }
    int cnt = n;
    if (n > p.k) {
        const uint64_t kth = idx::blk_kth_largest<1024>(a, n, p.k, hist, scratch, red64, 0, tid);
        // Out-of-place into the index row: only the selected k entries land there.
        cnt = idx::blk_compact<1024>(a, n, kth, static_cast<float*>(nullptr), out, wsum, 0,
                                     tid);
    } else {
        for (int e = tid; e < n; e += 1024) out[e] = a.index(e);
    }
    __syncthreads();
    for (int e = cnt + tid; e < p.k; e += 1024) out[e] = -1;
}

}  // namespace dec
}  // namespace dsa

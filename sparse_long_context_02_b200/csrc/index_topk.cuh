// Lightning-Indexer scores + streaming per-query top-k (prefill).
//
// Kwai Keye-VL-2.0 technical-report summary, section 1: an MQA-style indexer
// (one shared key vector per token) scores every visible position and each
// query keeps its k = 2048 best; section 8: the selection must be
// deterministic.  Score form (DeepSeek's indexer, which the pages name):
//     I[t,s] = sum_j w[t,j] * max(0, qI[t,j,:] . kI[s,:]),  s <= t.
//
// One CTA owns a block of 4 query tokens.  It streams the 128-key tiles of
// kI that those tokens can see through a TMA ring, multiplies each tile by
// the resident query block on the tensor cores (tcgen05 kind::f8f6f4,
// M = 128 keys, N = 4 * H_I query-head rows, K = d_I, fp32 accumulator in
// TMEM, two accumulators so the MMA of tile i+1 overlaps the epilogue of
// tile i) and never writes a score to global memory.
//
// Epilogue: warpgroup j (128 threads, one per key of the tile) owns token j.
// Each thread reads its key's H_I head dot products from TMEM, applies the
// ReLU and the weighted head sum in fp32 (exact for integer inputs below
// 2^24), and offers (score, key) to the token's candidate buffer in shared
// memory when the score beats the token's threshold theta.  Keys arrive in
// ascending order, so a later key with a score equal to theta can never
// enter the top-k; the filter is a plain `score > theta`.  When the buffer
// fills, the warpgroup finds the k-th best entry by an MSB-first radix
// select on a 64-bit key (ordered score, then inverted index), keeps the k
// best with an order-preserving compaction and raises theta to the k-th
// score.  The final row is therefore the exact top-k, ascending by index.
#pragma once

#include "ptx.cuh"

namespace dsa {
namespace idx {

constexpr int kTokens = 4;        // query tokens per CTA
constexpr int kKeyTile = 128;     // keys per tile (MMA M)
constexpr int kStages = 3;        // depth of the key-tile ring
constexpr int kThreads = 640;     // warps 0-3 control, warps 4-19 epilogue
constexpr int kEpiWarps = 16;

__host__ __device__ constexpr int cand_capacity(int k) {
    int c = 2 * k > k + kKeyTile ? 2 * k : k + kKeyTile;
    return (c + 127) / 128 * 128;
}

// Shared-memory layout (offsets from a 1024-byte aligned base).
struct Layout {
    int q, stage, w, cs, ci, hist, misc, total;
    __host__ __device__ Layout(int HI, int DI, int k, bool topk) {
        const int n = kTokens * HI;
        const int cap = topk ? cand_capacity(k) : 0;
        q = 0;
        stage = (n * DI + 1023) / 1024 * 1024;
        w = stage + kStages * kKeyTile * DI;
        cs = w + kTokens * HI * 4;
        ci = cs + kTokens * cap * 4;
        hist = ci + kTokens * cap * 4;
        misc = hist + (topk ? kTokens * 256 * 4 : 0);
        total = misc + 1024;
    }
};

// Misc block (inside Layout::misc).
struct Misc {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t qfull;
    uint64_t accfull[2];
    uint64_t accempty[2];
    uint64_t mma_done;
    uint64_t red64[kTokens][4];
    int wcnt[kTokens][2][4];
    int scratch[kTokens][4];
    uint32_t tmem_base;
    volatile int abort_flag;
};

__device__ __forceinline__ uint32_t ord_f32(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float unord_f32(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Larger key = better candidate: higher score, then lower index.
__device__ __forceinline__ uint64_t cand_key(float score, int32_t s) {
    return ((uint64_t)ord_f32(score) << 32) | (uint64_t)(~(uint32_t)s);
}

// ---- collective pieces over NT threads (named barrier `bar`, tid in [0, NT))
// Candidates are read through an accessor (score(e), index(e) for logical
// entry e); the arrays may live in shared or global memory.

struct FlatAccess {
    const float* sc;
    const int32_t* ix;
    __device__ __forceinline__ float score(int e) const { return sc[e]; }
    __device__ __forceinline__ int32_t index(int e) const { return ix[e]; }
};

// Up to four lists, logically concatenated (list j holds start[j+1]-start[j]
// entries).
struct SegAccess {
    const float* sc[4];
    const int32_t* ix[4];
    int start[5];
    __device__ __forceinline__ int seg(int e) const {
        return (e >= start[1]) + (e >= start[2]) + (e >= start[3]);
    }
    __device__ __forceinline__ float score(int e) const {
        const int j = seg(e);
        return sc[j][e - start[j]];
    }
    __device__ __forceinline__ int32_t index(int e) const {
        const int j = seg(e);
        return ix[j][e - start[j]];
    }
};

// k-th largest key among entries [0, n) (n >= k >= 1).  hist: 256 ints,
// scratch: 4 ints, red64: NT / 32 words, all in shared memory.
template <int NT, class A>
__device__ uint64_t blk_kth_largest(const A& a, int n, int k, int* hist, int* scratch,
                                    uint64_t* red64, uint32_t bar, int tid) {
    uint64_t prefix = 0;
    int need = k;
    int shift = 56;
    for (;; shift -= 8) {
        for (int b = tid; b < 256; b += NT) hist[b] = 0;
        named_bar_sync(bar, NT);
        for (int e = tid; e < n; e += NT) {
            const uint64_t key = cand_key(a.score(e), a.index(e));
            const bool match = shift == 56 || (key >> (shift + 8)) == (prefix >> (shift + 8));
            if (match) atomicAdd(&hist[(key >> shift) & 255], 1);
        }
        named_bar_sync(bar, NT);
        if (tid < 32) {
            int c[8], sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                c[u] = hist[255 - 8 * tid - u];
                sum += c[u];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            int above = incl - sum;
            if (above < need && need <= incl) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (above + c[u] >= need) {
                        scratch[0] = 255 - 8 * tid - u;
                        scratch[1] = need - above;
                        scratch[2] = c[u];
                        break;
                    }
                    above += c[u];
                }
            }
        }
        named_bar_sync(bar, NT);
        const int digit = scratch[0];
        need = scratch[1];
        const int bucket = scratch[2];
        prefix |= (uint64_t)digit << shift;
        if (bucket == need || shift == 0) break;
    }
    if (shift == 0) {
        named_bar_sync(bar, NT);  // scratch reads done before it is reused
        return prefix;            // all 64 bits fixed: the key itself
    }
    // Every entry of the bucket is selected: the k-th key is the bucket minimum.
    uint64_t m = ~0ull;
    for (int e = tid; e < n; e += NT) {
        const uint64_t key = cand_key(a.score(e), a.index(e));
        if ((key >> shift) == (prefix >> shift) && key < m) m = key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, m, o);
        m = y < m ? y : m;
    }
    if ((tid & 31) == 0) red64[tid >> 5] = m;
    named_bar_sync(bar, NT);
    uint64_t r = red64[0];
    for (int wv = 1; wv < NT / 32; ++wv) r = red64[wv] < r ? red64[wv] : r;
    named_bar_sync(bar, NT);  // red64 / scratch reads done before reuse
    return r;
}

// Writes, in order, the entries of [0, n) whose key is >= kth to out_sc /
// out_ix (out_sc may be null) and returns their count.  The output may alias a flat input: each
// round reads its entries into registers before anything is written, and a
// round never writes past the end of its own input range.  wsum: NT / 32
// ints of shared memory.
template <int NT, class A>
__device__ int blk_compact(const A& a, int n, uint64_t kth, float* out_sc, int32_t* out_ix,
                           int* wsum, uint32_t bar, int tid) {
    int out_base = 0;
    const int lane = tid & 31, warp = tid >> 5;
    for (int r0 = 0; r0 < n; r0 += NT * 8) {
        float s8[8];
        int32_t i8[8];
        uint32_t flags = 0;
        int m = 0;
        const int e0 = r0 + tid * 8;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            s8[u] = 0.f;
            i8[u] = 0;
            if (e0 + u < n) {
                s8[u] = a.score(e0 + u);
                i8[u] = a.index(e0 + u);
                if (cand_key(s8[u], i8[u]) >= kth) {
                    flags |= 1u << u;
                    ++m;
                }
            }
        }
        int incl = m;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        named_bar_sync(bar, NT);
        int before = 0, total = 0;
        for (int wv = 0; wv < NT / 32; ++wv) {
            const int c = wsum[wv];
            before += wv < warp ? c : 0;
            total += c;
        }
        int pos = out_base + before + incl - m;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (flags & (1u << u)) {
                if (out_sc) out_sc[pos] = s8[u];
                out_ix[pos] = i8[u];
                ++pos;
            }
        }
        out_base += total;
        named_bar_sync(bar, NT);
    }
    return out_base;
}

// Offers one key per thread of a warpgroup (tile of 128 consecutive keys,
// warp q holds keys 32q..32q+31) to a candidate buffer; compacts to the k
// best and raises theta when the buffer runs full.  Keys must arrive in
// ascending order across calls.
struct WgTopk {
    float* sc;
    int32_t* ix;
    int* hist;
    int* scratch;
    uint64_t* red64;
    int (*wcnt)[4];     // [2][4] per-warp append counts, double-buffered by tile
    int cap, k;
    uint32_t bar;
    int tid;
    float theta;
    int cnt;

    __device__ void offer(bool valid, float score, int32_t s, int tile_parity) {
        const int lane = tid & 31, q = tid >> 5;
        const bool take = valid && score > theta;
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        if (lane == 0) wcnt[tile_parity][q] = __popc(bal);
        named_bar_sync(bar, 128);
        int before = 0, total = 0;
#pragma unroll
        for (int wv = 0; wv < 4; ++wv) {
            const int c = wcnt[tile_parity][wv];
            before += wv < q ? c : 0;
            total += c;
        }
        if (take) {
            const int pos = cnt + before + __popc(bal & ((1u << lane) - 1u));
            sc[pos] = score;
            ix[pos] = s;
        }
        cnt += total;
        if (cnt > cap - 128) {
            named_bar_sync(bar, 128);
            const FlatAccess a{sc, ix};
            const uint64_t kth = blk_kth_largest<128>(a, cnt, k, hist, scratch, red64, bar, tid);
            cnt = blk_compact<128>(a, cnt, kth, sc, ix, scratch, bar, tid);
            theta = unord_f32((uint32_t)(kth >> 32));
        }
    }

    // Reduces the buffer to its k best (ascending by index); returns the count.
    __device__ int finish() {
        named_bar_sync(bar, 128);
        if (cnt > k) {
            const FlatAccess a{sc, ix};
            const uint64_t kth = blk_kth_largest<128>(a, cnt, k, hist, scratch, red64, bar, tid);
            cnt = blk_compact<128>(a, cnt, kth, sc, ix, scratch, bar, tid);
        }
        return cnt;
    }
};

// Weighted head sum of one key's ReLU'd head dot products, read from TMEM
// (this thread's lane, HI consecutive columns from taddr).  The "+ 0.0f"
// turns a -0 sum into +0 so that equal scores compare equal bitwise.
template <int HI>
__device__ __forceinline__ float head_sum(uint32_t taddr, const float* wj) {
    float acc = 0.f;
    if constexpr (HI >= 32) {
#pragma unroll
        for (int c = 0; c < HI / 32; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
#pragma unroll
            for (int h = 0; h < 32; ++h) acc = fmaf(wj[c * 32 + h], fmaxf(v[h], 0.f), acc);
        }
    } else {
        float v[4];
        tmem_ld_32x32b_x4(taddr, v);
#pragma unroll
        for (int h = 0; h < 4; ++h) acc = fmaf(wj[h], fmaxf(v[h], 0.f), acc);
    }
    return acc + 0.0f;
}

// ---------------------------------------------------------------- kernel

struct Params {
    const float* w;      // [L][H_I]
    int64_t L;
    int k;
    int32_t* idx;        // [L][k]        (top-k mode)
    float* scores;       // [L][L]        (dense-score mode)
    int nblocks;
};

template <int HI, int DI, bool TOPK>
__global__ void __launch_bounds__(kThreads, 1)
index_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
             const Params p) {
    constexpr int N = kTokens * HI;
    constexpr int KT_BYTES = kKeyTile * DI;
    constexpr int Q_BYTES = N * DI;
    constexpr uint32_t TMEM_COLS = 2 * N < 32 ? 32 : 2 * N;
    constexpr uint32_t IDESC = idesc_e4m3_f32(N);
    static_assert(N % 16 == 0 && N <= 256, "MMA N");
    static_assert(DI == 64 || DI == 128, "d_I");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Layout lay(HI, DI, p.k, TOPK);
    const int cap = TOPK ? cand_capacity(p.k) : 0;
    Misc* misc = reinterpret_cast<Misc*>(smem + lay.misc);
    float* w_s = reinterpret_cast<float*>(smem + lay.w);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t L = p.L;
    const int blk = p.nblocks - 1 - (int)blockIdx.x;  // longest rows first
    const int64_t t0 = (int64_t)blk * kTokens;
    const int64_t tmax = (t0 + kTokens - 1 < L ? t0 + kTokens - 1 : L - 1);
    const int ntiles = TOPK ? (int)(tmax / kKeyTile) + 1 : (int)((L + kKeyTile - 1) / kKeyTile);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&misc->full[s]), 1);
            mbar_init(smem_u32(&misc->empty[s]), 1);
        }
        mbar_init(smem_u32(&misc->qfull), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&misc->accfull[b]), 1);
            mbar_init(smem_u32(&misc->accempty[b]), kEpiWarps);
        }
        mbar_init(smem_u32(&misc->mma_done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(&misc->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    for (int e = threadIdx.x; e < kTokens * HI; e += kThreads) {
        const int64_t t = t0 + e / HI;
        w_s[e] = t < L ? p.w[t * HI + (e % HI)] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            const uint32_t qbar = smem_u32(&misc->qfull);
            mbar_arrive_expect_tx(qbar, Q_BYTES);
            tma_load_2d(smem_u32(smem + lay.q), &tmap_q, qbar, 0, (int32_t)(t0 * HI));
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                if (misc->abort_flag) break;
                const int s = i % kStages;
                if (i >= kStages &&
                    !mbar_wait(smem_u32(&misc->empty[s]), ((i / kStages) - 1) & 1)) {
                    misc->abort_flag = 1;
                    break;
                }
                const uint32_t fb = smem_u32(&misc->full[s]);
                mbar_arrive_expect_tx(fb, KT_BYTES);
                tma_load_2d(smem_u32(smem + lay.stage + s * KT_BYTES), &tmap_k, fb, 0,
                            i * kKeyTile);
                issued = i + 1;
            }
            // Never leave with a copy in flight.
            mbar_wait(qbar, 0);
            for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
                mbar_wait(smem_u32(&misc->full[i % kStages]), (i / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(smem_u32(&misc->qfull), 0);
            const uint64_t bdesc = smem_desc_kmajor(smem_u32(smem + lay.q), DI);
            for (int i = 0; ok && i < ntiles; ++i) {
                if (misc->abort_flag) break;
                const int s = i % kStages;
                const int buf = i & 1;
                ok = mbar_wait(smem_u32(&misc->full[s]), (i / kStages) & 1);
                if (ok && i >= 2) ok = mbar_wait(smem_u32(&misc->accempty[buf]), ((i >> 1) - 1) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint64_t adesc =
                    smem_desc_kmajor(smem_u32(smem + lay.stage + s * KT_BYTES), DI);
                const uint32_t d_tmem = tmem_base + (uint32_t)(buf * N);
#pragma unroll
                for (int kk = 0; kk < DI / 32; ++kk)
                    umma_f8f6f4(d_tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk),
                                IDESC, kk > 0 ? 1u : 0u);
                umma_commit(smem_u32(&misc->empty[s]));
                umma_commit(smem_u32(&misc->accfull[buf]));
            }
            if (!ok) misc->abort_flag = 1;
            // All MMAs of this CTA retired before TMEM is released.
            umma_commit(smem_u32(&misc->mma_done));
            mbar_wait(smem_u32(&misc->mma_done), 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        const int j = (warp - 4) >> 2;        // token of this warpgroup
        const int q = warp & 3;               // TMEM lane quarter
        const int tid = threadIdx.x - 128 - j * 128;
        const uint32_t bar = 1 + j;
        const int64_t t = t0 + j;
        const bool trow = t < L;
        float* sc = reinterpret_cast<float*>(smem + lay.cs) + j * cap;
        int32_t* ix = reinterpret_cast<int32_t*>(smem + lay.ci) + j * cap;
        int* hist = reinterpret_cast<int*>(smem + lay.hist) + j * 256;
        const float* wj = w_s + j * HI;
        WgTopk tk{sc, ix, hist, misc->scratch[j], misc->red64[j], misc->wcnt[j], cap, p.k, bar,
                  tid, -INFINITY, 0};
        bool ok = true;

        for (int i = 0; i < ntiles; ++i) {
            const int buf = i & 1;
            bool got = mbar_wait(smem_u32(&misc->accfull[buf]), (i >> 1) & 1);
            if (!named_bar_and(bar, 128, got && !misc->abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t taddr =
                tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * N + j * HI);
            const float score = head_sum<HI>(taddr, wj);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->accempty[buf]));
            const int64_t s = (int64_t)i * kKeyTile + q * 32 + lane;
            if constexpr (TOPK) {
                tk.offer(trow && s <= t, score, (int32_t)s, i & 1);
            } else {
                if (trow && s < L) p.scores[t * L + s] = s <= t ? score : -INFINITY;
            }
        }

        if constexpr (TOPK) {
            if (ok && trow) {
                const int cnt = tk.finish();
                int32_t* out = p.idx + t * p.k;
                for (int e = tid; e < p.k; e += 128) out[e] = e < cnt ? ix[e] : -1;
            }
        }
        if (!ok) misc->abort_flag = 1;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace idx
}  // namespace dsa

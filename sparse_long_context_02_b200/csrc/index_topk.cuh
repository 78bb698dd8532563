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
// Warps 0-15 are four epilogue warpgroups, one per token (warp w reads TMEM
// lanes 32 * (w % 4) ..); warp 16 is the TMA producer and owns the TMEM
// allocation; warp 17 issues the MMAs from one thread.  Each epilogue thread
// owns one key of the tile: it loads its H_I head dot products from TMEM,
// applies the ReLU and the weighted head sum in fp32 (exact for integer
// inputs below 2^24, in any summation order) and offers (score, key) to the
// token's streaming top-k (topk_select.cuh).  The final row is the exact
// top-k in ascending key order.
#pragma once

#include "ptx.cuh"
#include "topk_select.cuh"

namespace dsa {
namespace idx {

using sel::Scratch;
using sel::WgTopk;  // WgTopk<T, G>

constexpr int kTokens = 4;        // query tokens per CTA
constexpr int kKeyTile = 128;     // keys per tile (MMA M)
constexpr int kStages = 2;        // depth of the key-tile ring (kI is L2-resident)
constexpr int kEpiWarps = 16;     // warps 0-15
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kThreads = 20 * 32;  // warps 18-19 idle: warpgroup 4 is whole for setmaxnreg
// Register split (setmaxnreg): the launch gives every thread 96 registers
// (640 * 96 = 61440); warpgroup 4 drops to 32 and the four epilogue
// warpgroups rise to 112: 4 * 128 * 112 + 128 * 32 = 61440.
constexpr int kEpiRegs = 112;
constexpr int kCtlRegs = 32;
static_assert(4 * 128 * kEpiRegs + 128 * kCtlRegs <= kThreads * 96, "register split");
constexpr int kBatch = 8;         // tiles offered to the top-k per barrier
constexpr uint32_t kAllEpilogueBar = 5;  // named barrier over the 512 epilogue threads

// Candidate buffer entries per query.  A compaction starts once a batch
// leaves more than cap - kBatch * 128 entries (so the next batch always
// fits) and keeps at most half-way between k and that mark, so cap should
// exceed k by well over one batch: 2k + 512 for the usual k (4608 entries
// at k = 2048, which the shared-memory budget allows with a two-stage key
// ring), and at least k + one batch + 512 for small k.
__host__ __device__ constexpr int cand_capacity(int k, int batch) {
    const int a = 2 * k + 512, b = k + batch * kKeyTile + 512;
    return ((a > b ? a : b) + 127) / 128 * 128;
}

// Misc block: barriers and the small shared state.
struct Misc {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t qfull;
    uint64_t accfull[2];
    uint64_t accempty[2];
    uint64_t mma_done;
    alignas(16) int wcnt[2][kTokens][kBatch][4];  // rows read as int4 by WgTopk::offer
    int cnts[2][kTokens];
    uint32_t tmem_base;
    volatile int abort_flag;
};

static_assert(offsetof(Misc, wcnt) % 16 == 0, "wcnt rows are read as int4");

// Shared-memory layout (offsets from a 1024-byte aligned base).
struct Layout {
    int q, stage, w, cs, ci, scratch, misc, total;
    __host__ __device__ Layout(int HI, int DI, int k, bool topk) {
        const int n = kTokens * HI;
        const int cap = topk ? cand_capacity(k, kBatch) : 0;
        q = 0;
        stage = (n * DI + 1023) / 1024 * 1024;
        w = stage + kStages * kKeyTile * DI;
        cs = w + kTokens * HI * 4;
        ci = cs + kTokens * cap * 4;
        scratch = (ci + kTokens * cap * 4 + 15) / 16 * 16;
        misc = scratch + (topk ? kTokens * (int)sizeof(Scratch<128>) : 0);
        misc = (misc + 15) / 16 * 16;
        total = misc + (int)sizeof(Misc);
    }
};

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ float sum2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}

__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// Weighted head sum of one key's ReLU'd head dot products, read from TMEM
// (this thread's lane, HI consecutive columns from taddr).  Four independent
// partial sums (two packed f32x2 accumulators) shorten the FMA chain; for
// integer-valued inputs every partial and the total are exact, so the order
// does not change the result.  "+ 0.0f" turns a -0 sum into +0 so that equal
// scores compare equal bitwise.
template <int HI>
__device__ __forceinline__ float head_sum(uint32_t taddr, const float* wj) {
    if constexpr (HI == 64) {
        const float4* w4 = reinterpret_cast<const float4*>(wj);
        uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(taddr + c * 32, v);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 wq = w4[c * 8 + q];
                fma2(acc[0], pack2(wq.x, wq.y),
                     pack2(fmaxf(v[4 * q], 0.f), fmaxf(v[4 * q + 1], 0.f)));
                fma2(acc[1], pack2(wq.z, wq.w),
                     pack2(fmaxf(v[4 * q + 2], 0.f), fmaxf(v[4 * q + 3], 0.f)));
            }
        }
        return (sum2(acc[0]) + sum2(acc[1])) + 0.0f;
    } else {
        static_assert(HI == 4, "H_I");
        float v[4];
        tmem_ld_32x32b_x4(taddr, v);
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < 4; ++h) acc = fmaf(wj[h], fmaxf(v[h], 0.f), acc);
        return acc + 0.0f;
    }
}


// Weighted head sum with the token's 64 weights held in registers as f32
// pairs: no shared-memory reads beside the tensor core's operand fetches,
// which are what the tile rate depends on.  Same arithmetic and exactness as
// head_sum above.
__device__ __forceinline__ float head_sum_w2(uint32_t taddr, const uint64_t (&w2)[32]) {
    uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float v[16];
        tmem_ld_32x32b_x16(taddr + c * 16, v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            fma2(acc[0], w2[c * 8 + 2 * q], pack2(fmaxf(v[4 * q], 0.f), fmaxf(v[4 * q + 1], 0.f)));
            fma2(acc[1], w2[c * 8 + 2 * q + 1], pack2(fmaxf(v[4 * q + 2], 0.f), fmaxf(v[4 * q + 3], 0.f)));
        }
    }
    return (sum2(acc[0]) + sum2(acc[1])) + 0.0f;
}

// ---------------------------------------------------------------- kernel

struct Params {
    const float* w;      // [L][H_I]
    int64_t L;
    int k;
    int32_t* idx;        // [L][k]        (top-k mode)
    float* scores;       // [L][L]        (dense-score mode)
    int nblocks;         // blocks of kTokens rows launched
    int blk0;            // first block: rows [4 blk0, 4 (blk0 + nblocks)) are computed
    // Packed variable-length batch (top-k mode): query t sees keys
    // [cu_seqlens[b], t] of its own sequence b.  Null: one sequence.
    const int32_t* cu_seqlens;  // [nseq + 1], 0 ... L, non-decreasing
    int nseq;
    int* err;            // the call's device error word (null: the per-device word)
    // Query rows held by the call: q_I, w and idx start at row qrow0 (a
    // multiple of kTokens), so row t is element t - qrow0 of each.  Keys are
    // always rows 0 .. L-1 of k_I.
    int64_t qrow0;
};

// Start of the sequence that holds row t: cu[b] for the last b with
// cu[b] <= t, clamped into [0, t] (so a malformed array never reaches
// outside the rows).
__device__ __forceinline__ int64_t seq_start(const int32_t* cu, int nseq, int64_t t) {
    if (cu == nullptr) return 0;
    int lo = 0, hi = nseq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    int64_t s = cu[lo];
    return s < 0 ? 0 : (s > t ? t : s);
}

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
    // Aligned by pointer arithmetic on the shared array itself (not through an
    // integer), so that the compiler keeps every access in the shared window
    // (ld/st.shared with 32-bit addresses instead of generic ones).
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Layout lay(HI, DI, p.k, TOPK);
    const int cap = TOPK ? cand_capacity(p.k, kBatch) : 0;
    Misc* misc = reinterpret_cast<Misc*>(smem + lay.misc);
    float* w_s = reinterpret_cast<float*>(smem + lay.w);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t L = p.L;
    const int blk = p.blk0 + p.nblocks - 1 - (int)blockIdx.x;  // longest rows first
    const int64_t t0 = (int64_t)blk * kTokens;
    const int64_t tmax = (t0 + kTokens - 1 < L ? t0 + kTokens - 1 : L - 1);
    // token t0 + j sees keys [seq_start(t0 + j), t0 + j]; the CTA's tiles run
    // from the tile of the lowest start (the first token's: starts grow with t)
    const int64_t lo_min = TOPK ? seq_start(p.cu_seqlens, p.nseq, t0) : 0;
    const int tile0 = TOPK ? (int)(lo_min / kKeyTile) : 0;  // first key tile of the CTA
    const int ntiles = TOPK ? (int)(tmax / kKeyTile) + 1 - tile0
                            : (int)((L + kKeyTile - 1) / kKeyTile);  // tiles tile0, tile0 + 1, ...
    if (TOPK && p.cu_seqlens != nullptr && blockIdx.x == 0 && threadIdx.x == 0 &&
        (p.cu_seqlens[0] != 0 || (int64_t)p.cu_seqlens[p.nseq] != L))
        record_error_to(p.err, 2);  // cu_seqlens must run from 0 to L

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
    if (warp == kProducerWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    for (int e = threadIdx.x; e < kTokens * HI; e += kThreads) {
        const int64_t t = t0 + e / HI;
        w_s[e] = t < L ? p.w[(t - p.qrow0) * HI + (e % HI)] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc->tmem_base;

    if (warp >= kEpiWarps) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));
    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tmap_q);
            prefetch_tensormap(&tmap_k);
            const uint32_t qbar = smem_u32(&misc->qfull);
            mbar_arrive_expect_tx(qbar, Q_BYTES);
            tma_load_2d(smem_u32(smem + lay.q), &tmap_q, qbar, 0, (int32_t)((t0 - p.qrow0) * HI));
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                if (misc->abort_flag) break;
                const int s = i % kStages;
                if (i >= kStages &&
                    !mbar_wait_to(p.err, smem_u32(&misc->empty[s]), ((i / kStages) - 1) & 1)) {
                    misc->abort_flag = 1;
                    break;
                }
                const uint32_t fb = smem_u32(&misc->full[s]);
                mbar_arrive_expect_tx(fb, KT_BYTES);
                tma_load_2d(smem_u32(smem + lay.stage + s * KT_BYTES), &tmap_k, fb, 0,
                            (tile0 + i) * kKeyTile);
                issued = i + 1;
            }
            // Never leave with a copy in flight.
            mbar_wait_to(p.err, qbar, 0);
            for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
                mbar_wait_to(p.err, smem_u32(&misc->full[i % kStages]), (i / kStages) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait_to(p.err, smem_u32(&misc->qfull), 0);
            const uint64_t bdesc = smem_desc_kmajor(smem_u32(smem + lay.q), DI);
            for (int i = 0; ok && i < ntiles; ++i) {
                if (misc->abort_flag) break;
                const int s = i % kStages;
                const int buf = i & 1;
                ok = mbar_wait_to(p.err, smem_u32(&misc->full[s]), (i / kStages) & 1);
                if (ok && i >= 2) ok = mbar_wait_to(p.err, smem_u32(&misc->accempty[buf]), ((i >> 1) - 1) & 1);
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
            mbar_wait_to(p.err, smem_u32(&misc->mma_done), 0);
        }
    } else if (warp < kEpiWarps) {
        // ------------------------------------------------ epilogue (warps 0-15)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
        const int j = warp >> 2;              // token of this warpgroup
        const int q = warp & 3;               // TMEM lane quarter
        const int tid = threadIdx.x - j * 128;
        const uint32_t bar = 1 + j;
        const int64_t t = t0 + j;
        const bool trow = t < L;
        // key s of tile i is kb + 128 i; it is visible iff s - lo_t < vis_n
        // (unsigned), i.e. lo_t <= s <= t, with L <= 2^30 in 32 bits
        const int lo_t = TOPK && trow ? (int)seq_start(p.cu_seqlens, p.nseq, t) : 0;
        const uint32_t vis_n = trow ? (uint32_t)(t - lo_t + 1) : 0u;
        const int kb = tile0 * kKeyTile + q * 32 + lane;
        uint32_t* so = reinterpret_cast<uint32_t*>(smem + lay.cs) + j * cap;
        int32_t* ix = reinterpret_cast<int32_t*>(smem + lay.ci) + j * cap;
        Scratch<128>* S = reinterpret_cast<Scratch<128>*>(smem + lay.scratch) + j;
        const float* wj = w_s + j * HI;
        WgTopk<kBatch, kTokens> tk{so, ix, S, misc->wcnt, misc->cnts, j, cap, p.k, bar,
                                   kAllEpilogueBar, tid, 0u, 0, 0};
        tk.start();

        // A wait that times out sets abort_flag; the loop then runs on
        // without waiting (results are discarded), so every warp of the
        // warpgroup still meets every barrier.
        for (int i0 = 0; i0 < ntiles; i0 += kBatch) {
            uint64_t w2[32];  // the token's weights, reloaded per batch: dead across offers,
                              // so the compactions have the registers
            if constexpr (HI == 64) {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 f = reinterpret_cast<const float4*>(wj)[c];
                    w2[2 * c] = pack2(f.x, f.y);
                    w2[2 * c + 1] = pack2(f.z, f.w);
                }
            }
            uint32_t o[kBatch];  // ord of this thread's key in each tile; 0 = not visible
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u;
                o[u] = 0;
                if (i >= ntiles) continue;
                const int buf = i & 1;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->accfull[buf]), (i >> 1) & 1))
                    misc->abort_flag = 1;
                tc_fence_after();
                const uint32_t taddr =
                    tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * N + j * HI);
                float score;
                if constexpr (HI == 64) score = head_sum_w2(taddr, w2);
                else score = head_sum<HI>(taddr, wj);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&misc->accempty[buf]));
                if constexpr (TOPK) {
                    if ((uint32_t)(kb + i * kKeyTile - lo_t) < vis_n) o[u] = sel::ord_f32(score);
                } else {
                    const int64_t s = (int64_t)i * kKeyTile + q * 32 + lane;
                    if (trow && s < L) p.scores[t * L + s] = s <= t ? score : -INFINITY;
                }
            }
            if constexpr (TOPK)
                tk.offer(o, kb + i0 * kKeyTile,
                         ntiles - i0 < kBatch ? ntiles - i0 : kBatch);
        }

        if constexpr (TOPK) {
            tk.reduce(true);
            if (trow && !misc->abort_flag) {
                int32_t* out = p.idx + (t - p.qrow0) * p.k;
                for (int e = tid; e < p.k; e += 128) out[e] = e < tk.cnt ? ix[e] : -1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kProducerWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace idx
}  // namespace dsa

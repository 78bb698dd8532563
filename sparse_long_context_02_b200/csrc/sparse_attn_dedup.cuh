// Sparse GQA attention for blocks of adjacent query tokens that share their
// gathers (adjacent-query dedup).
//
// Kwai Keye-VL-2.0 technical-report summary, section 8: neighbouring queries
// select largely the same positions, so a block of them loads the union of
// their index sets once and keeps each query's own set with a mask inside the
// matrix products.  The result is the attention of dsa_sparse_attn_prefill
// (section 1 of the same page) for every query of the block.
//
// One CTA serves kDedupQB = 6 consecutive query tokens.
// Phase 1 (all threads): the union of the six index rows as a bitmap over the
// key range (it overlays the stage ring, which is idle then), a prefix count
// per 32-key word, the sorted list U of distinct keys, and for every key of U
// one byte whose bit j says whether query j selected it.
// Phase 2: a producer warp gathers the K and V rows of U in chunks of 16
// (16-byte cp.async, as in sparse_attn.cuh); consumer warp (g, p) owns KV
// group g and the query pair (2p, 2p + 1): the pair's 2 x G heads are the 16
// rows of an m16n8k16 tile (query 2p on rows 0..7, query 2p + 1 on rows
// 8..15), keys the columns; a key a query did not select gets a -inf score,
// i.e. probability 0.  Softmax is online per row in the exp2 domain; P is
// rounded to bf16 for the second product, O stays fp32 until the final store.
// The products grow with |U| x 6 rather than 6 k, so the kernel pays where
// the union is small (adjacent queries of clustered video tokens) and not on
// unclustered rows; the caller chooses.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {
namespace attn {

constexpr int kDedupStages = 3;  // gather ring stages of the dedup kernel
constexpr int kDedupQB = 6;               // query tokens per CTA (three pairs)
constexpr int kDedupMaxKeys = 1 << 18;    // keys the bitmap covers (32 KB)
constexpr int kDedupMaxK = 2048;          // index-row length the union buffers allow

template <int D, int HKV>
struct DedupCfg {
    static constexpr int PAIRS = kDedupQB / 2;
    static constexpr int CWARPS = HKV * PAIRS;           // consumer warps
    static constexpr int THREADS = (CWARPS + 1) * 32;    // plus the producer
    static constexpr int ROW = HKV * D * 2;
    static constexpr int STRIDE = ROW + 16;
    static constexpr int STAGE = 2 * kNK * STRIDE;
    static constexpr int UMAX = kDedupQB * kDedupMaxK;   // distinct keys at most
    // the stage ring, at least as large as the phase-1 bitmap that overlays it
    static constexpr int RING = kDedupStages * STAGE > kDedupMaxKeys / 8 ? kDedupStages * STAGE
                                                                     : kDedupMaxKeys / 8;
    static constexpr int OFF_PREFIX = RING;
    static constexpr int OFF_U = OFF_PREFIX + (kDedupMaxKeys / 32) * 4;
    static constexpr int OFF_MASK = OFF_U + UMAX * 4;
    static constexpr int OFF_BAR = OFF_MASK + UMAX;      // one mask byte per key
    static constexpr int SMEM = OFF_BAR + 2 * kDedupStages * 8;
    static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
};

// m16n8k16 bf16 product with all four A registers (rows 0..7 and 8..15).
__device__ __forceinline__ void mma_bf16_full(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The selection bit of query j for key position pos of U (0 past the end).
__device__ __forceinline__ bool selected(const uint32_t* mask32, int pos, int nU, int j) {
    return pos < nU && ((mask32[pos >> 2] >> ((pos & 3) * 8 + j)) & 1u);
}

template <int D, int HKV, int G>
__global__ void __launch_bounds__(DedupCfg<D, HKV>::THREADS, 1)
dedup_kernel(const Params p) {
    using C = DedupCfg<D, HKV>;
    constexpr int HQ = HKV * G;
    constexpr int NT = C::THREADS;
    static_assert(G <= 8, "at most 8 query heads per KV group");
    extern __shared__ __align__(128) uint8_t smem[];
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem);  // phase 1 only
    int* prefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);
    int32_t* U = reinterpret_cast<int32_t*>(smem + C::OFF_U);
    uint32_t* mask32 = reinterpret_cast<uint32_t*>(smem + C::OFF_MASK);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + kDedupStages;
    __shared__ int s_warp[32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t L = p.nkeys;  // rows = keys (one prefill sequence)
    const int64_t q0 = (int64_t)blockIdx.x * kDedupQB;
    const int nq = (int)(L - q0 < kDedupQB ? L - q0 : kDedupQB);
    const int nwords = (int)((L + 31) >> 5);

    // ---------------------------------------------------- phase 1: the union
    for (int i = tid; i < nwords; i += NT) bitmap[i] = 0u;
    if (tid == 0) {
        for (int s = 0; s < kDedupStages; ++s) {
            mbar_init(smem_u32(&full[s]), 33);  // 32 copy-completion arrivals + lane 0
            mbar_init(smem_u32(&empty[s]), C::CWARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int ne = nq * p.k;
    for (int e = tid; e < ne; e += NT) {
        const int32_t u = p.idx[(q0 + e / p.k) * p.k + e % p.k];
        if (u >= 0 && u < L) atomicOr(&bitmap[u >> 5], 1u << (u & 31));
        else if (u >= L) record_error_to(p.err, 2);
    }
    __syncthreads();
    // words [w0, w1) of this thread: count, block scan, prefix, list
    const int per = (nwords + NT - 1) / NT;
    const int w0 = tid * per < nwords ? tid * per : nwords;
    const int w1 = w0 + per < nwords ? w0 + per : nwords;
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bitmap[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int base = 0, nU = 0;
    for (int i = 0; i < NT / 32; ++i) {
        base += i < warp ? s_warp[i] : 0;
        nU += s_warp[i];
    }
    int run = base + incl - cnt;
    for (int w = w0; w < w1; ++w) {
        prefix[w] = run;
        uint32_t b = bitmap[w];
        while (b) {
            U[run++] = w * 32 + (__ffs(b) - 1);
            b &= b - 1u;
        }
    }
    for (int i = tid; i < (nU + 3) / 4; i += NT) mask32[i] = 0u;
    __syncthreads();
    for (int e = tid; e < ne; e += NT) {
        const int j = e / p.k;
        const int32_t u = p.idx[(q0 + j) * p.k + e % p.k];
        if (u >= 0 && u < L) {
            const int pos = prefix[u >> 5] + __popc(bitmap[u >> 5] & ((1u << (u & 31)) - 1u));
            atomicOr(&mask32[pos >> 2], (1u << j) << ((pos & 3) * 8));
        }
    }
    __syncthreads();  // the stage ring (under the bitmap) is free from here
    const int nchunks = (nU + kNK - 1) / kNK;

    if (warp == C::CWARPS) {
        // ------------------------------------------------ gather producer
        constexpr int CPR = C::ROW / 16;
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kDedupStages;
            if (c >= kDedupStages) {
                bool got = false;
                if (lane == 0) got = mbar_wait_to(p.err, smem_u32(&empty[s]), ((c / kDedupStages) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, got, 0)) break;
            }
            const uint32_t sbase = smem_u32(smem + s * C::STAGE);
#pragma unroll 4
            for (int r = 0; r < kNK; ++r) {
                const int e = c * kNK + r;
                const int64_t row = e < nU ? U[e] : 0;  // past the end: a real row, mask 0
                const char* ks = reinterpret_cast<const char*>(p.K + row * HKV * D);
                const char* vs = reinterpret_cast<const char*>(p.V + row * HKV * D);
                const uint32_t dk = sbase + r * C::STRIDE, dv = dk + kNK * C::STRIDE;
#pragma unroll
                for (int q = lane; q < CPR; q += 32) {
                    cp_async16(dk + q * 16, ks + q * 16);
                    cp_async16(dv + q * 16, vs + q * 16);
                }
            }
            const uint32_t fb = smem_u32(&full[s]);
            cp_async_arrive(fb);
            if (lane == 0) mbar_arrive(fb);
            issued = c + 1;
        }
        if (lane == 0) {
            for (int c = issued - kDedupStages < 0 ? 0 : issued - kDedupStages; c < issued; ++c)
                mbar_wait_to(p.err, smem_u32(&full[c % kDedupStages]), (c / kDedupStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------- consumer (g, pair)
    const int g = warp % HKV, pr = warp / HKV;
    const int ja = 2 * pr, jb = 2 * pr + 1;  // queries of rows 0..7 and 8..15
    const int r = lane >> 2;
    const int cq = (lane & 3) * 2;
    const bool hrow = r < G;
    const bool va = ja < nq, vb = jb < nq;

    uint32_t qa[D / 16][4];
    {
        const __nv_bfloat16* qA = p.Q + ((q0 + (va ? ja : 0)) * HQ + g * G + (hrow ? r : 0)) * D;
        const __nv_bfloat16* qB = p.Q + ((q0 + (vb ? jb : 0)) * HQ + g * G + (hrow ? r : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(qA + ks * 16 + cq);
            const uint32_t a2 = *reinterpret_cast<const uint32_t*>(qA + ks * 16 + 8 + cq);
            const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qB + ks * 16 + cq);
            const uint32_t b2 = *reinterpret_cast<const uint32_t*>(qB + ks * 16 + 8 + cq);
            qa[ks][0] = hrow && va ? a0 : 0u;
            qa[ks][1] = hrow && vb ? b0 : 0u;
            qa[ks][2] = hrow && va ? a2 : 0u;
            qa[ks][3] = hrow && vb ? b2 : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    const int mi = lane >> 3, ri = lane & 7;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kDedupStages;
        const bool got = mbar_wait_to(p.err, smem_u32(&full[s]), (c / kDedupStages) & 1);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint32_t kbase = smem_u32(smem + s * C::STAGE) + g * D * 2;
        const uint32_t vbase = kbase + kNK * C::STRIDE;
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
            for (int kp = 0; kp < D / 32; ++kp) {
                uint32_t b[4];
                ldsm_x4(kbase + (nt * 8 + ri) * C::STRIDE + (kp * 32 + mi * 8) * 2, b);
                mma_bf16_full(sacc[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3],
                              b[0], b[1]);
                mma_bf16_full(sacc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2],
                              qa[2 * kp + 1][3], b[2], b[3]);
            }
        }
        // scores of the keys each query selected; -inf elsewhere
        float xa[2][2], xb[2][2];
        float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int pos = c * kNK + nt * 8 + cq + e;
                xa[nt][e] = selected(mask32, pos, nU, ja) ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                xb[nt][e] = selected(mask32, pos, nU, jb) ? sacc[nt][2 + e] * p.scale_log2 : -INFINITY;
                mxa = fmaxf(mxa, xa[nt][e]);
                mxb = fmaxf(mxb, xb[nt][e]);
            }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        const float na = fmaxf(m_a, mxa), nb = fmaxf(m_b, mxb);
        const float ua = na == -INFINITY ? 0.f : na, ub = nb == -INFINITY ? 0.f : nb;
        const float ca = ex2(m_a - ua), cb = ex2(m_b - ub);
        float pa[2][2], pb[2][2];
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                pa[nt][e] = ex2(xa[nt][e] - ua);
                pb[nt][e] = ex2(xb[nt][e] - ub);
                sa += pa[nt][e];
                sb += pb[nt][e];
            }
        l_a = l_a * ca + sa;
        l_b = l_b * cb + sb;
        m_a = na;
        m_b = nb;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            o[n][0] *= ca;
            o[n][1] *= ca;
            o[n][2] *= cb;
            o[n][3] *= cb;
        }
        const uint32_t p0 = pack_bf16(pa[0][0], pa[0][1]);  // row r, keys 0..7
        const uint32_t p1 = pack_bf16(pb[0][0], pb[0][1]);  // row r + 8
        const uint32_t p2 = pack_bf16(pa[1][0], pa[1][1]);  // row r, keys 8..15
        const uint32_t p3 = pack_bf16(pb[1][0], pb[1][1]);
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            uint32_t b[4];
            ldsm_x4_trans(vbase + ((mi & 1) * 8 + ri) * C::STRIDE + (np * 16 + (mi >> 1) * 8) * 2, b);
            mma_bf16_full(o[2 * np], p0, p1, p2, p3, b[0], b[1]);
            mma_bf16_full(o[2 * np + 1], p0, p1, p2, p3, b[2], b[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    if (!ok) return;

    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    if (!hrow) return;
    const int h = g * G + r;
    if (va) {
        const float inv = l_a > 0.f ? 1.f / l_a : 0.f;
        __nv_bfloat16* out = p.O + ((q0 + ja) * HQ + h) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<uint32_t*>(out + n * 8 + cq) = pack_bf16(o[n][0] * inv, o[n][1] * inv);
    }
    if (vb) {
        const float inv = l_b > 0.f ? 1.f / l_b : 0.f;
        __nv_bfloat16* out = p.O + ((q0 + jb) * HQ + h) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<uint32_t*>(out + n * 8 + cq) = pack_bf16(o[n][2] * inv, o[n][3] * inv);
    }
}

}  // namespace attn
}  // namespace dsa

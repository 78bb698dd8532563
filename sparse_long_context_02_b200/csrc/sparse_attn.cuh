// Sparse GQA attention over selected K/V rows (prefill; split form for decode).
//
// Kwai Keye-VL-2.0 technical-report summary, section 1: attention runs only
// over the positions the indexer kept, O(Lk) instead of O(L^2); the base
// model is GQA, and one index set per query token serves every KV group and
// query head.  For query row t and head h in group g = h / G:
//     O[t,h] = sum_{s in idx[t]} softmax_s(scale * Q[t,h] . K[s,g]) V[s,g].
//
// The step is bound by the gather: every selected token contributes its K and
// V rows for all Hkv groups, 2 * Hkv * d * 2 bytes, read once per query token.
// One CTA serves one query token (or one slice of its index row, for decode).
// A producer warp gathers the selected K and V rows (each a contiguous
// Hkv * d * 2 byte run) with 16-byte cp.async copies, all 32 lanes sharing
// each row, into a ring of shared-memory stages; every lane's completion
// arrives on the stage's mbarrier.  (Per-row bulk copies through the copy
// engine reached 5.9 TB/s of gathered rows; the load/store path reaches
// 7.3 TB/s.)  Rows are padded by 16 bytes so that the consumers' ldmatrix
// reads hit distinct banks.  Consumer warp g owns KV group g: its G
// query heads are the rows of an m16n8k16 tile (rows G..15 are zero), keys the
// columns.  S = Q K^T and O += P V run on the tensor cores in bf16 with fp32
// accumulation; the softmax is online in the exp2 domain; P is rounded to
// bf16 for the second product, O stays fp32 until the final store.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dsa {
namespace attn {

constexpr int kNK = 16;      // keys per stage
// Two stages: 67 KB of shared memory per CTA, so three CTAs (15 warps) fit
// on an SM (136 registers x 160 threads x 3 also fits the register file).
constexpr int kStages = 2;

// NP producer warps split each stage's rows (two pay while the gathered rows
// hit L2; one otherwise, see dsa_lib.cu).
template <int D, int HKV, int NP = 1>
struct Cfg {
    static constexpr int ROW = HKV * D * 2;       // bytes of one token's K (or V) row
    static constexpr int STRIDE = ROW + 16;       // padded shared-memory row
    static constexpr int STAGE = 2 * kNK * STRIDE;
    static constexpr int THREADS = (HKV + NP) * 32;
    static constexpr int SMEM = kStages * STAGE + 128;
};

struct Params {
    const __nv_bfloat16* Q;   // [rows][Hq][d]
    const __nv_bfloat16* K;   // [keys][Hkv][d]
    const __nv_bfloat16* V;
    const int32_t* idx;       // [rows][k]
    int64_t nkeys;            // prefill: valid keys are [0, nkeys)
    int k;
    float scale_log2;         // softmax scale * log2(e)
    __nv_bfloat16* O;         // [rows][Hq][d]           (prefill)
    float* lse;               // [rows][Hq] or null      (prefill) natural-log softmax normaliser
    const int64_t* cache_off; // [B + 1]                 (decode)
    int nsplit;               // index-row slices per sequence (decode)
    float* part_o;            // [B][nsplit][Hq][d]      unnormalised partial O
    float* part_ml;           // [B][nsplit][Hq][2]      running max (log2 units), sum
    int* err;                 // the call's device error word (null: the per-device word)
    // Cache shards (decode): index entries are global keys; this shard holds
    // keys [key_base[b], key_base[b] + n_b) of sequence b, and entries
    // outside that range belong to another shard (skipped, not flagged).
    const int64_t* key_base;  // [B] or null (0)
    int skip_foreign;
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
    // A rows 8..15 are zero (a1 = a3 = 0): only d[0], d[1] carry results.
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

template <int D, int HKV, int G, bool SPLIT, int NP = 1>
__global__ void __launch_bounds__(Cfg<D, HKV, NP>::THREADS)
attn_kernel(const Params p) {
    pdl_wait();  // decode: the index rows come from the merge kernel
    pdl_launch_dependents();
    using C = Cfg<D, HKV, NP>;
    constexpr int HQ = HKV * G;
    static_assert(G <= 8, "at most 8 query heads per KV group");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::STAGE);
    uint64_t* empty = full + kStages;
    uint32_t* mask = reinterpret_cast<uint32_t*>(empty + kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- the unit this CTA serves
    const __nv_bfloat16 *Kb = p.K, *Vb = p.V, *qrow;
    const int32_t* irow;
    int nent;
    int64_t nkeys, orow = 0, koff = 0;
    int split = 0;
    if constexpr (SPLIT) {
        const int64_t b = blockIdx.x / p.nsplit;
        split = blockIdx.x % p.nsplit;
        const int per = ((p.k + p.nsplit - 1) / p.nsplit + kNK - 1) / kNK * kNK;
        const int e0 = split * per;
        nent = p.k - e0 < per ? p.k - e0 : per;
        if (nent < 0) nent = 0;
        const int64_t base = p.cache_off[b];
        nkeys = p.cache_off[b + 1] - base;
        if (p.key_base != nullptr) koff = p.key_base[b];
        Kb = p.K + base * HKV * D;
        Vb = p.V + base * HKV * D;
        irow = p.idx + b * p.k + e0;
        qrow = p.Q + b * HQ * D;
        orow = b;
    } else {
        const int64_t t = blockIdx.x;
        nent = p.k;
        nkeys = p.nkeys;
        irow = p.idx + t * p.k;
        qrow = p.Q + t * HQ * D;
        orow = t;
    }
    const int nchunks = (nent + kNK - 1) / kNK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full[s]), 32 * NP + 1);  // copy completions + one lane 0
            mbar_init(smem_u32(&empty[s]), HKV);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp >= HKV) {
        // ------------------------------------------------ gather producers (16-byte cp.async)
        const int pw = warp - HKV;  // rows pw, pw + NP, ... of each stage
        constexpr int CPR = C::ROW / 16;  // 16-byte chunks per row
        int issued = 0;
        // Each chunk's index entries are loaded one chunk ahead, so their
        // latency overlaps the wait and the copies of the chunk before.
        auto load_idx = [&](int c) -> int32_t {
            const int e = c * kNK + lane;
            return lane < kNK && c < nchunks && e < nent ? irow[e] : -1;
        };
        int32_t pre = load_idx(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const int64_t sg = pre;  // the entry: a key of this shard after - koff
            pre = load_idx(c + 1);
            if (c >= kStages) {
                bool got = false;
                if (lane == 0) got = mbar_wait_to(p.err, smem_u32(&empty[s]), ((c / kStages) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, got, 0)) break;
            }
            int32_t si;
            if constexpr (SPLIT) {  // global keys of a cache shard, or sequence-local ones
                const int64_t sl = sg - koff;
                if (sg >= 0 && sl >= nkeys && !p.skip_foreign) record_error_to(p.err, 2);
                si = sg >= 0 && sl >= 0 && sl < nkeys ? (int32_t)sl : -1;
            } else {
                si = (int32_t)sg;
                if (si >= nkeys) record_error_to(p.err, 2);
            }
            const bool valid = si >= 0 && si < nkeys;
            const uint32_t bal = __ballot_sync(0xffffffffu, valid);
            const uint32_t sbase = smem_u32(smem + s * C::STAGE);
            if (bal) {
#pragma unroll 4
                for (int r = pw; r < kNK; r += NP) {
                    // A masked entry still gets a real row (row 0): its P is 0,
                    // and 0 times stale shared memory could be NaN.  (The
                    // shuffle stays outside any branch: a conditional one
                    // costs a third of the kernel's speed.)
                    const int32_t sr = __shfl_sync(0xffffffffu, si, r);
                    const int64_t row = (bal >> r) & 1u ? sr : 0;
                    const char* ks = reinterpret_cast<const char*>(Kb + row * HKV * D);
                    const char* vs = reinterpret_cast<const char*>(Vb + row * HKV * D);
                    const uint32_t dk = sbase + r * C::STRIDE, dv = dk + kNK * C::STRIDE;
#pragma unroll
                    for (int q = lane; q < CPR; q += 32) {
                        cp_async16(dk + q * 16, ks + q * 16);
                        cp_async16(dv + q * 16, vs + q * 16);
                    }
                }
            }
            const uint32_t fb = smem_u32(&full[s]);
            cp_async_arrive(fb);  // this lane's copies of the stage
            if (lane == 0 && pw == 0) {
                mask[s] = bal;
                mbar_arrive(fb);
            }
            issued = c + 1;
        }
        if (lane == 0) {
            for (int c = issued - kStages < 0 ? 0 : issued - kStages; c < issued; ++c)
                mbar_wait_to(p.err, smem_u32(&full[c % kStages]), (c / kStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------- consumer: group g
    const int g = warp;
    const int r = lane >> 2;          // query-head row of this thread (0..7)
    const int cq = (lane & 3) * 2;    // first of the two columns this thread holds
    const bool hrow = r < G;

    uint32_t qa[D / 16][2];
    {
        const __nv_bfloat16* qh = qrow + (g * G + (hrow ? r : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t lo = *reinterpret_cast<const uint32_t*>(qh + ks * 16 + cq);
            uint32_t hi = *reinterpret_cast<const uint32_t*>(qh + ks * 16 + 8 + cq);
            qa[ks][0] = hrow ? lo : 0u;
            qa[ks][1] = hrow ? hi : 0u;
        }
    }

    float o[D / 8][2];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = 0.f;
    float m_run = -INFINITY, l_part = 0.f;

    const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix id, row in matrix
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        bool got = mbar_wait_to(p.err, smem_u32(&full[s]), (c / kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint32_t msk = mask[s];
        if (msk) {
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
                    mma_bf16(sacc[nt], qa[2 * kp][0], qa[2 * kp][1], b[0], b[1]);
                    mma_bf16(sacc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], b[2], b[3]);
                }
            }
            float x[2][2];
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + cq + e;
                    const float v = (msk >> col) & 1u ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                    x[nt][e] = v;
                    mx = fmaxf(mx, v);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float corr = ex2(m_run - m_use);
            float pr[2][2];
            float psum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    pr[nt][e] = ex2(x[nt][e] - m_use);
                    psum += pr[nt][e];
                }
            l_part = l_part * corr + psum;
            m_run = m_new;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= corr;
                o[n][1] *= corr;
            }
            const uint32_t pa0 = pack_bf16(pr[0][0], pr[0][1]);
            const uint32_t pa2 = pack_bf16(pr[1][0], pr[1][1]);
#pragma unroll
            for (int np = 0; np < D / 16; ++np) {
                uint32_t b[4];
                ldsm_x4_trans(vbase + ((mi & 1) * 8 + ri) * C::STRIDE + (np * 16 + (mi >> 1) * 8) * 2,
                              b);
                float d0[4] = {o[2 * np][0], o[2 * np][1], 0.f, 0.f};
                float d1[4] = {o[2 * np + 1][0], o[2 * np + 1][1], 0.f, 0.f};
                mma_bf16(d0, pa0, pa2, b[0], b[1]);
                mma_bf16(d1, pa0, pa2, b[2], b[3]);
                o[2 * np][0] = d0[0];
                o[2 * np][1] = d0[1];
                o[2 * np + 1][0] = d1[0];
                o[2 * np + 1][1] = d1[1];
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    if (!ok) return;

    float l = l_part;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (!hrow) return;
    const int h = g * G + r;
    if constexpr (SPLIT) {
        float* po = p.part_o + (((int64_t)orow * p.nsplit + split) * HQ + h) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<float2*>(po + n * 8 + cq) = make_float2(o[n][0], o[n][1]);
        if ((lane & 3) == 0) {
            float* pm = p.part_ml + (((int64_t)orow * p.nsplit + split) * HQ + h) * 2;
            pm[0] = m_run;
            pm[1] = l;
        }
    } else {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if (p.lse != nullptr && (lane & 3) == 0)
            p.lse[(int64_t)orow * HQ + h] =
                l > 0.f ? (m_run + __log2f(l)) * 0.69314718055994531f : -INFINITY;
        __nv_bfloat16* out = p.O + ((int64_t)orow * HQ + h) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<uint32_t*>(out + n * 8 + cq) = pack_bf16(o[n][0] * inv, o[n][1] * inv);
    }
}

// Merges the nsplit partial results of each (sequence, head):
//   M = max_j m_j,  l = sum_j l_j 2^(m_j - M),  O = sum_j O_j 2^(m_j - M) / l.
// Partial j of sequence b is row (b * bs + j * js) of part_o / part_ml (in
// units of HQ heads): bs = nsplit, js = 1 for the [B][nsplit] layout of one
// decode, bs = 1, js = B for the [P][B] layout of P gathered cache shards.
// FINAL: O is written as bf16; otherwise the merged partial itself (the
// unnormalised sum relative to M, and M, l) goes to out_o / out_ml, rows
// [B][HQ], for a later merge with other shards' partials.
// One CTA per (sequence, head), one thread per output dimension.
template <int D, int HQ, bool FINAL>
__global__ void __launch_bounds__(D) combine_kernel(const float* part_o, const float* part_ml,
                                                    int nsplit, int64_t bs, int64_t js,
                                                    __nv_bfloat16* O, float* out_o,
                                                    float* out_ml) {
    pdl_wait();  // the partials come from the split attention
    const int64_t b = blockIdx.x / HQ;
    const int h = blockIdx.x % HQ, c = threadIdx.x;
    auto row = [&](int j) { return ((b * bs + (int64_t)j * js) * HQ + h); };
    float M = -INFINITY;
    for (int j = 0; j < nsplit; ++j) M = fmaxf(M, part_ml[row(j) * 2]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float l = 0.f, acc = 0.f;
    for (int j = 0; j < nsplit; ++j) {
        const float* ml = part_ml + row(j) * 2;
        const float f = ex2(ml[0] - Mu);
        l += ml[1] * f;
        acc += part_o[row(j) * D + c] * f;
    }
    if constexpr (FINAL) {
        O[(b * HQ + h) * D + c] = __float2bfloat16_rn(l > 0.f ? acc / l : 0.f);
    } else {
        out_o[(b * HQ + h) * D + c] = acc;
        if (c == 0) {
            out_ml[(b * HQ + h) * 2] = M;
            out_ml[(b * HQ + h) * 2 + 1] = l;
        }
    }
}

}  // namespace attn
}  // namespace dsa

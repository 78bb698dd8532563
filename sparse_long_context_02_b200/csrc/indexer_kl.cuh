// Indexer warm-up loss: KL from the full attention's head-mean distribution
// to the Lightning Indexer's softmax, and its gradients with respect to the
// indexer's inputs.
//
// Kwai Keye-VL-2.0 technical-report summary, section 1 (two-stage training):
// in the dense warm-up the full attention stays as it is and only the indexer
// is trained, towards the full attention's distribution, with a KL divergence
// as the measure.  Reading taken (the pages print no formula):
//   I[t,s]  = sum_j w[t,j] relu(q_I[t,j] . k_I[s])             (s <= t)
//   P_I[t]  = softmax_s(scale_I * I[t,s])
//   p[t,s]  = (1/Hq) sum_h softmax_s(scale * Q[t,h] . K[s, h / (Hq/Hkv)])
//   kl[t]   = sum_s p (ln p - ln P_I)
//   G[t,s]  = d(sum_t kl)/dI[t,s] = scale_I * (P_I[t,s] - p[t,s])
//   dw[t,j] = sum_s G relu(S),  dq_I[t,j] = w[t,j] sum_s G [S > 0] k_I[s],
//   dk_I[s] = sum_t sum_j G w[t,j] [S > 0] q_I[t,j],   S = q_I[t,j] . k_I[s].
//
// Kernels here (tiles of 64 query rows x 64 keys; four warps of 16 rows):
//   row_lse_kernel     lse of scale_I * I per row (I from the tcgen05 scorer)
//   head_lse_kernel    lse of every query head's causal attention row
//   target_kernel      p, the row KL partials and G, written over I in place
//   kl_reduce_kernel   kl[t] from the partials in a fixed order
//   dq_kernel          dq_I and dw for one indexer head and 64 query rows
//   dk_kernel          dk_I for 64 keys, over all later query rows and a group
//                      of heads (one partial per group)
//   dk_reduce_kernel   dk_I = sum of the groups' partials, in a fixed order
// Their products use mma.sync (bf16 m16n8k16 for the attention, e4m3
// m16n8k32 for the indexer).  The 5th-generation tensor-core versions of
// head_lse, target, dq and dk (indexer_kl_tc.cuh, 128 x 128 tiles, TMEM
// accumulators) run for d = 128 with Hkv <= 4 (forward) and d_I = 128
// (backward); these serve the other shapes.  dS is rounded to bf16 for the
// dq/dk products, as a flash-attention backward does.  Every result is
// written by exactly one thread, in a fixed order: runs are bit-identical.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {
namespace kl {

constexpr int kTile = 64;     // query rows and keys per tile
constexpr int kThreads = 128; // four warps of 16 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Params {
    const uint8_t* qI;        // [L][HI][DI] e4m3
    const uint8_t* kI;        // [L][DI]     e4m3
    const float* w;           // [L][HI]
    const __nv_bfloat16* Q;   // [L][Hq][D]
    const __nv_bfloat16* K;   // [L][Hkv][D]
    int64_t L;
    int HI, Hq, Hkv;
    int ntiles;               // ceil(L / 64)
    float scale_log2;         // attention scale * log2(e)
    float scale_I;
    float* G;                 // [L][L]: I on entry of target_kernel, G after it
    const float* Gin;         // [L][L]: G for the backward kernels
    float* lse_h;             // [L][Hq] log2-domain lse of each attention row
    float* lse_I;             // [L]     natural-log lse of scale_I * I[t, 0..t]
    float* kl_part;           // [L][ntiles]: row partials of kl, one per key tile
    int kl_tile_log2;         // key tile of the partials: 64 or 128 keys
    int* err;                 // the call's device error word (null: the per-device word)
    float* kl;                // [L]
    float* dq;                // [L][HI][DI]
    float* dk;                // [L][DI]
    float* dw;                // [L][HI]
    int nsplit;               // head groups of dk_kernel (a divisor of HI)
    float* dk_part;           // [nsplit][L][DI] (nsplit > 1)
};

using attn::ex2;
using attn::ldsm_x4;
using attn::ldsm_x4_trans;
using attn::pack_bf16;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Four e4m3 bytes to four bf16 (exact: every e4m3 value is a bf16 value).
__device__ __forceinline__ uint2 e4m3x4_to_bf16x4(uint32_t v) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(v >> 16), __NV_E4M3);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    return make_uint2(pack_bf16(a.x, a.y), pack_bf16(b.x, b.y));
}

// ------------------------------------------------------------------ forward

// lse_I[t] = ln sum_{s <= t} exp(scale_I * I[t,s]); one warp per row.
__global__ void __launch_bounds__(256) row_lse_kernel(const Params p) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= p.L) return;
    const float* row = p.G + t * p.L;
    const float c = p.scale_I * kLog2e;
    float m = -INFINITY, s = 0.f;
    for (int64_t j = lane; j <= t; j += 32) {
        const float z = row[j] * c;
        const float mn = fmaxf(m, z);
        s = s * ex2(m - mn) + ex2(z - mn);
        m = mn;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
        const float so = __shfl_xor_sync(0xffffffffu, s, o);
        const float mn = fmaxf(m, mo);
        s = (m == -INFINITY ? 0.f : s * ex2(m - mn)) + (mo == -INFINITY ? 0.f : so * ex2(mo - mn));
        m = mn;
    }
    if (lane == 0) p.lse_I[t] = (m + lg2(s)) * kLn2;
}

// Shared tile of 64 bf16 rows of D elements, padded for ldmatrix.
template <int D>
struct BfTile {
    static constexpr int STRIDE = D * 2 + 16;  // bytes per row
    static constexpr int BYTES = kTile * STRIDE;
};

// Copies 64 rows (row r at src + r * row_stride elements) into a BfTile with
// cp.async; rows >= nrows are zero-filled with plain stores.
template <int D>
__device__ __forceinline__ void load_bf_tile(uint8_t* dst, const __nv_bfloat16* src,
                                             int64_t row_stride, int nrows) {
    constexpr int CPR = D * 2 / 16;  // 16-byte chunks per row
    for (int i = threadIdx.x; i < kTile * CPR; i += kThreads) {
        const int r = i / CPR, q = i % CPR;
        uint8_t* d = dst + r * BfTile<D>::STRIDE + q * 16;
        if (r < nrows)
            cp_async16(smem_u32(d), reinterpret_cast<const uint8_t*>(src + r * row_stride) + q * 16);
        else
            *reinterpret_cast<uint4*>(d) = make_uint4(0, 0, 0, 0);
    }
}

// A fragments (m16 x k16 per step) of 16 bf16 rows held in a BfTile.
template <int D>
__device__ __forceinline__ void ldsm_a_rows(uint32_t base, int row0, int ks, uint32_t (&a)[4]) {
    const int lane = threadIdx.x & 31;
    const uint32_t addr = base + (row0 + (lane & 7) + ((lane >> 3) & 1) * 8) * BfTile<D>::STRIDE +
                          (ks * 16 + (lane >> 4) * 8) * 2;
    ldsm_x4(addr, a);
}

// S (16 rows x 64 keys) = A . K^T, with A fragments in registers and the 64
// keys' rows in a BfTile.
template <int D>
__device__ __forceinline__ void qk_bf16(float (&S)[8][4], const uint32_t (&qa)[D / 16][4],
                                        uint32_t kbase) {
    const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < D / 32; ++kp)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            uint32_t b[4];
            ldsm_x4(kbase + (nt * 8 + ri) * BfTile<D>::STRIDE + (kp * 32 + mi * 8) * 2, b);
            mma_bf16_16816(S[nt], qa[2 * kp], b[0], b[1]);
            mma_bf16_16816(S[nt], qa[2 * kp + 1], b[2], b[3]);
        }
}

// lse_h[t][h] (log2 domain) of scale * Q[t,h] . K[s,g] over s <= t.
// Grid (ntiles, Hq); the longest query tiles first.
template <int D>
__global__ void __launch_bounds__(kThreads) head_lse_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int qt = p.ntiles - 1 - blockIdx.x, h = blockIdx.y;
    const int g = h / (p.Hq / p.Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int64_t t_a = (int64_t)qt * kTile + warp * 16 + r, t_b = t_a + 8;

    uint32_t qa[D / 16][4];
    {
        const int64_t ra = t_a < p.L ? t_a : p.L - 1, rb = t_b < p.L ? t_b : p.L - 1;
        const __nv_bfloat16* qa_row = p.Q + (ra * p.Hq + h) * D;
        const __nv_bfloat16* qb_row = p.Q + (rb * p.Hq + h) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = *reinterpret_cast<const uint32_t*>(qa_row + ks * 16 + 2 * c);
            qa[ks][1] = *reinterpret_cast<const uint32_t*>(qb_row + ks * 16 + 2 * c);
            qa[ks][2] = *reinterpret_cast<const uint32_t*>(qa_row + ks * 16 + 8 + 2 * c);
            qa[ks][3] = *reinterpret_cast<const uint32_t*>(qb_row + ks * 16 + 8 + 2 * c);
        }
    }
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    const int nkt = qt + 1;
    const int64_t kstride = (int64_t)p.Hkv * D;
    auto load = [&](int kt) {
        const int64_t s0 = (int64_t)kt * kTile;
        const int64_t rem = p.L - s0;
        load_bf_tile<D>(smem + (kt & 1) * BfTile<D>::BYTES, p.K + s0 * kstride + g * D, kstride,
                        rem < kTile ? (int)rem : kTile);
        cp_commit();
    };
    load(0);
    for (int kt = 0; kt < nkt; ++kt) {
        cp_wait_all();
        __syncthreads();
        if (kt + 1 < nkt) load(kt + 1);  // into the other buffer, free since the barrier
        float S[8][4];
        qk_bf16<D>(S, qa, smem_u32(smem + (kt & 1) * BfTile<D>::BYTES));
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t s = (int64_t)kt * kTile + nt * 8 + 2 * c + e;
                S[nt][e] = s <= t_a ? S[nt][e] * p.scale_log2 : -INFINITY;
                S[nt][2 + e] = s <= t_b ? S[nt][2 + e] * p.scale_log2 : -INFINITY;
                mx_a = fmaxf(mx_a, S[nt][e]);
                mx_b = fmaxf(mx_b, S[nt][2 + e]);
            }
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o));
        }
        const float na = fmaxf(m_a, mx_a), nb = fmaxf(m_b, mx_b);
        const float ua = na == -INFINITY ? 0.f : na, ub = nb == -INFINITY ? 0.f : nb;
        float sa = 0.f, sb = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                sa += ex2(S[nt][e] - ua);
                sb += ex2(S[nt][2 + e] - ub);
            }
        l_a = l_a * ex2(m_a - ua) + sa;
        l_b = l_b * ex2(m_b - ub) + sb;
        m_a = na;
        m_b = nb;
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, o);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, o);
    }
    if (c == 0) {
        if (t_a < p.L) p.lse_h[t_a * p.Hq + h] = m_a + lg2(l_a);
        if (t_b < p.L) p.lse_h[t_b * p.Hq + h] = m_b + lg2(l_b);
    }
}

// One (query tile, key tile): p summed over all query heads, then the KL
// partial of each row and G, written over I.  Tiles above the diagonal
// only write G = 0.  Grid (ntiles keys, ntiles queries).
template <int D>
__global__ void __launch_bounds__(kThreads) target_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int kt = blockIdx.x, qt = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int64_t t_a = (int64_t)qt * kTile + warp * 16 + r, t_b = t_a + 8;
    const int64_t s0 = (int64_t)kt * kTile;
    if (kt > qt) {
        for (int i = threadIdx.x; i < kTile * kTile; i += kThreads) {
            const int64_t t = (int64_t)qt * kTile + i / kTile, s = s0 + i % kTile;
            if (t < p.L && s < p.L) p.G[t * p.L + s] = 0.f;
        }
        return;
    }
    // K rows of every group for these 64 keys, then a two-slot ring of Q tiles.
    uint8_t* ktiles = smem;
    uint8_t* qring = smem + p.Hkv * BfTile<D>::BYTES;
    const int64_t krem = p.L - s0;
    const int kn = krem < kTile ? (int)krem : kTile;
    for (int g = 0; g < p.Hkv; ++g)
        load_bf_tile<D>(ktiles + g * BfTile<D>::BYTES, p.K + s0 * p.Hkv * D + g * D,
                        (int64_t)p.Hkv * D, kn);
    const int64_t t0 = (int64_t)qt * kTile;
    const int64_t qrem = p.L - t0;
    const int qn = qrem < kTile ? (int)qrem : kTile;
    const int64_t qstride = (int64_t)p.Hq * D;
    auto load_q = [&](int h) {
        load_bf_tile<D>(qring + (h & 1) * BfTile<D>::BYTES, p.Q + t0 * qstride + h * D, qstride, qn);
        cp_commit();
    };
    load_q(0);

    const int G = p.Hq / p.Hkv;
    float P[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) P[nt][0] = P[nt][1] = P[nt][2] = P[nt][3] = 0.f;
    for (int h = 0; h < p.Hq; ++h) {
        cp_wait_all();
        __syncthreads();
        if (h + 1 < p.Hq) load_q(h + 1);
        const float la = t_a < p.L ? p.lse_h[t_a * p.Hq + h] : 0.f;
        const float lb = t_b < p.L ? p.lse_h[t_b * p.Hq + h] : 0.f;
        const uint32_t qbase = smem_u32(qring + (h & 1) * BfTile<D>::BYTES);
        uint32_t qa[D / 16][4];
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) ldsm_a_rows<D>(qbase, warp * 16, ks, qa[ks]);
        float S[8][4];
        qk_bf16<D>(S, qa, smem_u32(ktiles + (h / G) * BfTile<D>::BYTES));
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t s = s0 + nt * 8 + 2 * c + e;
                if (s <= t_a) P[nt][e] += ex2(S[nt][e] * p.scale_log2 - la);
                if (s <= t_b) P[nt][2 + e] += ex2(S[nt][2 + e] * p.scale_log2 - lb);
            }
    }
    const float inv_h = 1.f / (float)p.Hq;
    const float lse_a = t_a < p.L ? p.lse_I[t_a] : 0.f;
    const float lse_b = t_b < p.L ? p.lse_I[t_b] : 0.f;
    float kla = 0.f, klb = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
            const int64_t t = hv ? t_b : t_a;
            const float lse = hv ? lse_b : lse_a;
            if (t >= p.L) continue;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t s = s0 + nt * 8 + 2 * c + e;
                if (s >= p.L) continue;
                float* gp = p.G + t * p.L + s;
                float gv = 0.f;
                if (s <= t) {
                    const float pv = P[nt][2 * hv + e] * inv_h;
                    const float lq = p.scale_I * *gp - lse;  // ln P_I[t,s]
                    const float term = pv > 0.f ? pv * (lg2(pv) * kLn2 - lq) : 0.f;
                    if (hv) klb += term; else kla += term;
                    gv = p.scale_I * (ex2(lq * kLog2e) - pv);
                }
                *gp = gv;
            }
        }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        kla += __shfl_xor_sync(0xffffffffu, kla, o);
        klb += __shfl_xor_sync(0xffffffffu, klb, o);
    }
    if (c == 0) {
        if (t_a < p.L) p.kl_part[t_a * p.ntiles + kt] = kla;
        if (t_b < p.L) p.kl_part[t_b * p.ntiles + kt] = klb;
    }
}

__global__ void kl_reduce_kernel(const Params p) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= p.L) return;
    float s = 0.f;
    const int n = (int)(t >> p.kl_tile_log2) + 1;
    for (int i = 0; i < n; ++i) s += p.kl_part[t * p.ntiles + i];
    p.kl[t] = s;
}

// ------------------------------------------------------------------ backward

// Shared tile of 64 e4m3 rows of DI bytes plus their bf16 copy.
template <int DI>
struct F8Tile {
    static constexpr int F8_STRIDE = DI + 16;
    static constexpr int BF_STRIDE = DI * 2 + 16;
    static constexpr int F8_BYTES = kTile * F8_STRIDE;
    static constexpr int BYTES = F8_BYTES + kTile * BF_STRIDE;
    static constexpr int PER_THREAD = kTile * DI / 16 / kThreads;  // uint4 per thread
};

// Loads 64 e4m3 rows (row r at src + r * row_stride bytes; rows >= nrows are
// zeros) into registers, then stores them and their bf16 copy.
template <int DI>
struct F8Loader {
    uint4 v[F8Tile<DI>::PER_THREAD];
    __device__ __forceinline__ void load(const uint8_t* src, int64_t row_stride, int nrows) {
        constexpr int CPR = DI / 16;
#pragma unroll
        for (int i = 0; i < F8Tile<DI>::PER_THREAD; ++i) {
            const int idx = threadIdx.x + i * kThreads;
            const int r = idx / CPR, q = idx % CPR;
            v[i] = r < nrows ? *reinterpret_cast<const uint4*>(src + r * row_stride + q * 16)
                             : make_uint4(0, 0, 0, 0);
        }
    }
    __device__ __forceinline__ void store(uint8_t* dst) const {
        constexpr int CPR = DI / 16;
#pragma unroll
        for (int i = 0; i < F8Tile<DI>::PER_THREAD; ++i) {
            const int idx = threadIdx.x + i * kThreads;
            const int r = idx / CPR, q = idx % CPR;
            *reinterpret_cast<uint4*>(dst + r * F8Tile<DI>::F8_STRIDE + q * 16) = v[i];
            uint8_t* b = dst + F8Tile<DI>::F8_BYTES + r * F8Tile<DI>::BF_STRIDE + q * 32;
            const uint2 x0 = e4m3x4_to_bf16x4(v[i].x), x1 = e4m3x4_to_bf16x4(v[i].y);
            const uint2 x2 = e4m3x4_to_bf16x4(v[i].z), x3 = e4m3x4_to_bf16x4(v[i].w);
            *reinterpret_cast<uint4*>(b) = make_uint4(x0.x, x0.y, x1.x, x1.y);
            *reinterpret_cast<uint4*>(b + 16) = make_uint4(x2.x, x2.y, x3.x, x3.y);
        }
    }
};

// A fragments (m16 x k32 per step) of 16 e4m3 rows from global memory.
template <int DI>
__device__ __forceinline__ void load_a_e4m3(uint32_t (&a)[DI / 32][4], const uint8_t* row_a,
                                            const uint8_t* row_b) {
    const int c = threadIdx.x & 3;
#pragma unroll
    for (int ks = 0; ks < DI / 32; ++ks) {
        a[ks][0] = *reinterpret_cast<const uint32_t*>(row_a + ks * 32 + 4 * c);
        a[ks][1] = *reinterpret_cast<const uint32_t*>(row_b + ks * 32 + 4 * c);
        a[ks][2] = *reinterpret_cast<const uint32_t*>(row_a + ks * 32 + 16 + 4 * c);
        a[ks][3] = *reinterpret_cast<const uint32_t*>(row_b + ks * 32 + 16 + 4 * c);
    }
}

// S (16 x 64) = A . B^T with e4m3 A fragments and the 64 B rows in an F8Tile.
template <int DI>
__device__ __forceinline__ void qk_e4m3(float (&S)[8][4], const uint32_t (&a)[DI / 32][4],
                                        uint32_t base) {
    const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < DI / 64; ++kp)
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            uint32_t b[4];
            ldsm_x4(base + (nt * 8 + ri) * F8Tile<DI>::F8_STRIDE + kp * 64 + mi * 16, b);
            mma_e4m3_16832(S[nt], a[2 * kp], b[0], b[1]);
            mma_e4m3_16832(S[nt], a[2 * kp + 1], b[2], b[3]);
        }
}

// acc (16 x DI) += dS (16 x 64, C layout, rounded to bf16) . B (64 x DI) with
// B the bf16 copy in an F8Tile.
template <int DI>
__device__ __forceinline__ void ds_times_rows(float (&acc)[DI / 8][4], const float (&dS)[8][4],
                                              uint32_t base) {
    const int lane = threadIdx.x & 31, mi = lane >> 3, ri = lane & 7;
    const uint32_t bbase = base + F8Tile<DI>::F8_BYTES;
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
        uint32_t a[4];
        a[0] = pack_bf16(dS[2 * kb][0], dS[2 * kb][1]);
        a[1] = pack_bf16(dS[2 * kb][2], dS[2 * kb][3]);
        a[2] = pack_bf16(dS[2 * kb + 1][0], dS[2 * kb + 1][1]);
        a[3] = pack_bf16(dS[2 * kb + 1][2], dS[2 * kb + 1][3]);
#pragma unroll
        for (int np = 0; np < DI / 16; ++np) {
            uint32_t b[4];
            ldsm_x4_trans(bbase + (kb * 16 + (mi & 1) * 8 + ri) * F8Tile<DI>::BF_STRIDE +
                              (np * 16 + (mi >> 1) * 8) * 2,
                          b);
            mma_bf16_16816(acc[2 * np], a, b[0], b[1]);
            mma_bf16_16816(acc[2 * np + 1], a, b[2], b[3]);
        }
    }
}

// dq_I and dw of indexer head j for 64 query rows.  Grid (HI, ntiles): the
// heads of one query tile run side by side and share its G band in L2.
template <int DI>
__global__ void __launch_bounds__(kThreads) dq_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int qt = p.ntiles - 1 - blockIdx.y, j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int64_t t_a = (int64_t)qt * kTile + warp * 16 + r, t_b = t_a + 8;
    const int64_t ra = t_a < p.L ? t_a : p.L - 1, rb = t_b < p.L ? t_b : p.L - 1;

    uint32_t qa[DI / 32][4];
    load_a_e4m3<DI>(qa, p.qI + (ra * p.HI + j) * DI, p.qI + (rb * p.HI + j) * DI);
    const float wa = p.w[ra * p.HI + j], wb = p.w[rb * p.HI + j];

    float acc[DI / 8][4];
#pragma unroll
    for (int n = 0; n < DI / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float dwa = 0.f, dwb = 0.f;

    const int nkt = qt + 1;
    F8Loader<DI> ld;
    auto rows_of = [&](int kt) {
        const int64_t rem = p.L - (int64_t)kt * kTile;
        return rem < kTile ? (int)rem : kTile;
    };
    ld.load(p.kI, DI, rows_of(0));
    ld.store(smem);
    __syncthreads();
    for (int kt = 0; kt < nkt; ++kt) {
        if (kt + 1 < nkt) ld.load(p.kI + (int64_t)(kt + 1) * kTile * DI, DI, rows_of(kt + 1));
        const int64_t s0 = (int64_t)kt * kTile;
        float gv[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t s = s0 + nt * 8 + 2 * c + e;
                gv[nt][e] = s <= t_a && t_a < p.L ? p.Gin[t_a * p.L + s] : 0.f;
                gv[nt][2 + e] = s <= t_b && t_b < p.L ? p.Gin[t_b * p.L + s] : 0.f;
            }
        const uint32_t base = smem_u32(smem + (kt & 1) * F8Tile<DI>::BYTES);
        float S[8][4];
        qk_e4m3<DI>(S, qa, base);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                dwa += gv[nt][e] * fmaxf(S[nt][e], 0.f);
                dwb += gv[nt][2 + e] * fmaxf(S[nt][2 + e], 0.f);
                S[nt][e] = S[nt][e] > 0.f ? gv[nt][e] * wa : 0.f;
                S[nt][2 + e] = S[nt][2 + e] > 0.f ? gv[nt][2 + e] * wb : 0.f;
            }
        ds_times_rows<DI>(acc, S, base);
        if (kt + 1 < nkt) ld.store(smem + ((kt + 1) & 1) * F8Tile<DI>::BYTES);
        __syncthreads();
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        dwa += __shfl_xor_sync(0xffffffffu, dwa, o);
        dwb += __shfl_xor_sync(0xffffffffu, dwb, o);
    }
    if (t_a < p.L) {
        float* out = p.dq + (t_a * p.HI + j) * DI;
#pragma unroll
        for (int n = 0; n < DI / 8; ++n)
            *reinterpret_cast<float2*>(out + n * 8 + 2 * c) = make_float2(acc[n][0], acc[n][1]);
        if (c == 0) p.dw[t_a * p.HI + j] = dwa;
    }
    if (t_b < p.L) {
        float* out = p.dq + (t_b * p.HI + j) * DI;
#pragma unroll
        for (int n = 0; n < DI / 8; ++n)
            *reinterpret_cast<float2*>(out + n * 8 + 2 * c) = make_float2(acc[n][2], acc[n][3]);
        if (c == 0) p.dw[t_b * p.HI + j] = dwb;
    }
}

// dk_I for 64 keys: over every query tile at or after the keys' tile and
// the heads of one group.  Grid (nsplit, ntiles): the groups of one key tile
// run side by side; the longest key tiles (the first) first.  Shared: a two-slot ring of q_I tiles, then w^T of the query tile
// (rows of kWStride floats: the transposing stores avoid bank conflicts).
constexpr int kWStride = kTile + 1;

template <int DI>
__global__ void __launch_bounds__(kThreads) dk_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x, kt = blockIdx.y;
    const int hps = p.HI / p.nsplit, j0 = split * hps;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
    const int64_t s_a = (int64_t)kt * kTile + warp * 16 + r, s_b = s_a + 8;
    const int64_t ra = s_a < p.L ? s_a : p.L - 1, rb = s_b < p.L ? s_b : p.L - 1;
    float* wT = reinterpret_cast<float*>(smem + 2 * F8Tile<DI>::BYTES);  // [hps][kWStride]

    uint32_t ka[DI / 32][4];
    load_a_e4m3<DI>(ka, p.kI + ra * DI, p.kI + rb * DI);

    float acc[DI / 8][4];
#pragma unroll
    for (int n = 0; n < DI / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

    const int64_t qstride = (int64_t)p.HI * DI;
    F8Loader<DI> ld;
    int slot = 0;
    for (int qt = kt; qt < p.ntiles; ++qt) {
        const int64_t t0 = (int64_t)qt * kTile;
        const int64_t rem = p.L - t0;
        const int qn = rem < kTile ? (int)rem : kTile;
        // G^T for these keys and this query tile, and w^T of the tile
        float gv[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t t = t0 + nt * 8 + 2 * c + e;
                const bool tv = t < p.L;
                gv[nt][e] = tv && s_a <= t && s_a < p.L ? p.Gin[t * p.L + s_a] : 0.f;
                gv[nt][2 + e] = tv && s_b <= t && s_b < p.L ? p.Gin[t * p.L + s_b] : 0.f;
            }
        __syncthreads();  // the previous tile's w^T and q slots are no longer read
        for (int i = threadIdx.x; i < kTile * hps; i += kThreads) {
            const int tt = i / hps, jj = i % hps;
            wT[jj * kWStride + tt] = tt < qn ? p.w[(t0 + tt) * p.HI + j0 + jj] : 0.f;
        }
        ld.load(p.qI + t0 * qstride + j0 * DI, qstride, qn);
        ld.store(smem + slot * F8Tile<DI>::BYTES);
        __syncthreads();
        for (int j = 0; j < hps; ++j) {
            if (j + 1 < hps) ld.load(p.qI + t0 * qstride + (j0 + j + 1) * DI, qstride, qn);
            const uint32_t base = smem_u32(smem + slot * F8Tile<DI>::BYTES);
            float S[8][4];
            qk_e4m3<DI>(S, ka, base);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float wv = wT[j * kWStride + nt * 8 + 2 * c + e];
                    S[nt][e] = S[nt][e] > 0.f ? gv[nt][e] * wv : 0.f;
                    S[nt][2 + e] = S[nt][2 + e] > 0.f ? gv[nt][2 + e] * wv : 0.f;
                }
            ds_times_rows<DI>(acc, S, base);
            if (j + 1 < hps) {
                ld.store(smem + (slot ^ 1) * F8Tile<DI>::BYTES);
                __syncthreads();
                slot ^= 1;
            }
        }
    }
    float* dk = p.nsplit > 1 ? p.dk_part + (int64_t)split * p.L * DI : p.dk;
    if (s_a < p.L) {
        float* out = dk + s_a * DI;
#pragma unroll
        for (int n = 0; n < DI / 8; ++n)
            *reinterpret_cast<float2*>(out + n * 8 + 2 * c) = make_float2(acc[n][0], acc[n][1]);
    }
    if (s_b < p.L) {
        float* out = dk + s_b * DI;
#pragma unroll
        for (int n = 0; n < DI / 8; ++n)
            *reinterpret_cast<float2*>(out + n * 8 + 2 * c) = make_float2(acc[n][2], acc[n][3]);
    }
}

// dk_I[i] = sum over the head groups' partials, in group order (float4).
__global__ void dk_reduce_kernel(const Params p, int DI) {
    const int64_t n4 = p.L * DI / 4;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4* part = reinterpret_cast<const float4*>(p.dk_part);
    float4 a = part[i];
    for (int sp = 1; sp < p.nsplit; ++sp) {
        const float4 b = part[sp * n4 + i];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
    }
    reinterpret_cast<float4*>(p.dk)[i] = a;
}

}  // namespace kl
}  // namespace dsa

// Backward pass of the sparse GQA attention (training through the selected
// rows).
//
// Kwai Keye-VL-2.0 technical-report summary, section 1: after the indexer's
// dense warm-up, the sparse-adaptation stage trains every parameter on the
// next-token loss with the attention truly sparse; the gradient therefore
// flows through the attention over each query's selected rows, the index
// rows themselves being fixed.  For query row t, head h, group g = h / G and
// the valid entries i of idx[t] (s_i = idx[t,i]):
//     P[i]  = exp(scale * Q[t,h] . K[s_i,g] - lse[t,h])
//     dP[i] = dO[t,h] . V[s_i,g],   D = dO[t,h] . O[t,h],   dS[i] = P[i] (dP[i] - D)
//     dQ[t,h]   = scale * sum_i dS[i] K[s_i,g]
//     dK[s_i,g] += scale * dS[i] Q[t,h],    dV[s_i,g] += P[i] dO[t,h]
// with lse the forward's log-sum-exp (dsa_sparse_attn_prefill writes it).
//
// One CTA serves one query token, as in the forward: the same producer warp
// gathers each chunk of 16 selected K and V rows into a two-stage ring, and
// consumer warp g owns KV group g (its G query heads are the MMA rows).  Per
// chunk it forms S = Q K^T and dP = dO V^T (mma.sync m16n8k16, bf16 in,
// fp32 out), then P and dS in registers; dQ += dS K accumulates in registers
// for the whole row.  The chunk's dK and dV rows are products over the
// group's heads: dS^T and P^T come from the score fragments by an in-register
// 8x8 transpose (movmatrix), Q_g and dO_g are held as B fragments, and each
// 16 x 8 tile of the products (m16n8k8) goes straight to global memory with
// vector fp32 reductions.  Nothing is staged for the scatter: its cost is the
// L2 reduction traffic, 2 * Hkv * d * 4 bytes per selected row.
#pragma once

#include <cuda_bf16.h>

#include "sparse_attn.cuh"

namespace dsa {
namespace attn {

struct BwdParams {
    const __nv_bfloat16* Q;   // [L][Hq][d]
    const __nv_bfloat16* K;   // [L][Hkv][d]
    const __nv_bfloat16* V;
    const __nv_bfloat16* O;   // [L][Hq][d] forward output
    const __nv_bfloat16* dO;  // [L][Hq][d]
    const float* lse;         // [L][Hq] natural log (-inf: row without a valid entry)
    const int32_t* idx;       // [L][k]
    int64_t nkeys;
    int k;
    float scale;
    float scale_log2;         // scale * log2(e)
    float* dQ;                // [L][Hq][d] fp32, written
    float* dK;                // [L][Hkv][d] fp32, accumulated (zero on entry)
    float* dV;
    int* err;
};

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// d += A (16 x 8, rows a0 / a1) x B (8 x 8, b0), bf16 in, fp32 out.
__device__ __forceinline__ void mma_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ uint32_t bf16_bits(const __nv_bfloat16* p) {
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p));
}

template <int D, int HKV, int G>
__global__ void __launch_bounds__(Cfg<D, HKV>::THREADS)
attn_bwd_kernel(const BwdParams p) {
    using C = Cfg<D, HKV>;
    constexpr int HQ = HKV * G;
    static_assert(G <= 8, "at most 8 query heads per KV group");
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * C::STAGE);
    uint64_t* empty = full + kStages;
    uint32_t* mask = reinterpret_cast<uint32_t*>(empty + kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x;
    const int nent = p.k;
    const int64_t nkeys = p.nkeys;
    const int32_t* irow = p.idx + t * p.k;
    const int nchunks = (nent + kNK - 1) / kNK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full[s]), 33);  // 32 copy-completion arrivals + lane 0
            mbar_init(smem_u32(&empty[s]), HKV);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == HKV) {
        // ------------------------------------------------ gather producer (as the forward's)
        constexpr int CPR = C::ROW / 16;
        int issued = 0;
        auto load_idx = [&](int c) -> int32_t {
            const int e = c * kNK + lane;
            return lane < kNK && c < nchunks && e < nent ? irow[e] : -1;
        };
        int32_t pre = load_idx(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % kStages;
            const int32_t si = pre;
            pre = load_idx(c + 1);
            if (c >= kStages) {
                bool got = false;
                if (lane == 0) got = mbar_wait_to(p.err, smem_u32(&empty[s]), ((c / kStages) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, got, 0)) break;
            }
            if (si >= nkeys) record_error_to(p.err, 2);
            const bool valid = si >= 0 && si < nkeys;
            const uint32_t bal = __ballot_sync(0xffffffffu, valid);
            const uint32_t sbase = smem_u32(smem + s * C::STAGE);
            if (bal) {
#pragma unroll 4
                for (int r = 0; r < kNK; ++r) {
                    // a masked entry still gets a real row (row 0): its P and
                    // dS are 0, and 0 times stale shared memory could be NaN
                    const int32_t sr = __shfl_sync(0xffffffffu, si, r);
                    const int64_t row = (bal >> r) & 1u ? sr : 0;
                    const char* ks = reinterpret_cast<const char*>(p.K + row * HKV * D);
                    const char* vs = reinterpret_cast<const char*>(p.V + row * HKV * D);
                    const uint32_t dk = sbase + r * C::STRIDE, dv = dk + kNK * C::STRIDE;
#pragma unroll
                    for (int q = lane; q < CPR; q += 32) {
                        cp_async16(dk + q * 16, ks + q * 16);
                        cp_async16(dv + q * 16, vs + q * 16);
                    }
                }
            }
            const uint32_t fb = smem_u32(&full[s]);
            cp_async_arrive(fb);
            if (lane == 0) {
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
    const int r = lane >> 2;          // head row of S / dP / dQ; key row of the dK / dV tiles
    const int cq = (lane & 3) * 2;    // first of the two columns this thread holds
    const bool hrow = r < G;
    const int hb = (lane & 3) * 2;    // the two heads of this thread's B fragments

    const __nv_bfloat16* qg = p.Q + (t * HQ + g * G) * D;
    const __nv_bfloat16* dog = p.dO + (t * HQ + g * G) * D;
    const __nv_bfloat16* og = p.O + (t * HQ + g * G) * D;
    uint32_t qa[D / 16][2], da[D / 16][2];  // A fragments of Q_g and dO_g (rows = heads)
    float drow = 0.f;                        // partial dO . O of head row r
    {
        const int hr = hrow ? r : 0;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int c = ks * 16 + half * 8 + cq;
                const uint32_t q2 = *reinterpret_cast<const uint32_t*>(qg + hr * D + c);
                const uint32_t d2 = *reinterpret_cast<const uint32_t*>(dog + hr * D + c);
                const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(og + hr * D + c);
                const __nv_bfloat162 e2 = *reinterpret_cast<const __nv_bfloat162*>(&d2);
                qa[ks][half] = hrow ? q2 : 0u;
                da[ks][half] = hrow ? d2 : 0u;
                drow += __bfloat162float(e2.x) * __bfloat162float(o2.x) +
                        __bfloat162float(e2.y) * __bfloat162float(o2.y);
            }
        }
    }
    drow += __shfl_xor_sync(0xffffffffu, drow, 1);
    drow += __shfl_xor_sync(0xffffffffu, drow, 2);
    if (!hrow) drow = 0.f;
    const float lse2 = hrow ? p.lse[t * HQ + g * G + r] * 1.4426950408889634f : 0.f;

    // B fragments of Q_g and dO_g for the dK / dV products (k = head, n = dim):
    // heads hb, hb + 1 at dim 8 nt + r; heads >= G are zero.
    uint32_t qb[D / 8], db[D / 8];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int c = nt * 8 + r;
        const uint32_t q0 = hb < G ? bf16_bits(qg + hb * D + c) : 0u;
        const uint32_t q1 = hb + 1 < G ? bf16_bits(qg + (hb + 1) * D + c) : 0u;
        const uint32_t d0 = hb < G ? bf16_bits(dog + hb * D + c) : 0u;
        const uint32_t d1 = hb + 1 < G ? bf16_bits(dog + (hb + 1) * D + c) : 0u;
        qb[nt] = q0 | (q1 << 16);
        db[nt] = d0 | (d1 << 16);
    }

    float dq[D / 8][2];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = 0.f;

    const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix id, row in matrix
    float* const dKg = p.dK + g * D + cq;
    float* const dVg = p.dV + g * D + cq;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kStages;
        // keys of this thread's two tile rows (r and r + 8), read while the stage lands
        const int e0 = c * kNK + r, e1 = e0 + 8;
        const int32_t key0 = e0 < nent ? irow[e0] : -1;
        const int32_t key1 = e1 < nent ? irow[e1] : -1;
        bool got = mbar_wait_to(p.err, smem_u32(&full[s]), (c / kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const uint32_t msk = mask[s];
        if (msk) {
            const uint32_t kbase = smem_u32(smem + s * C::STAGE) + g * D * 2;
            const uint32_t vbase = kbase + kNK * C::STRIDE;
            float sacc[2][4], pacc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] = pacc[nt][e] = 0.f;
#pragma unroll
                for (int kp = 0; kp < D / 32; ++kp) {
                    uint32_t b[4];
                    ldsm_x4(kbase + (nt * 8 + ri) * C::STRIDE + (kp * 32 + mi * 8) * 2, b);
                    mma_bf16(sacc[nt], qa[2 * kp][0], qa[2 * kp][1], b[0], b[1]);
                    mma_bf16(sacc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], b[2], b[3]);
                    ldsm_x4(vbase + (nt * 8 + ri) * C::STRIDE + (kp * 32 + mi * 8) * 2, b);
                    mma_bf16(pacc[nt], da[2 * kp][0], da[2 * kp][1], b[0], b[1]);
                    mma_bf16(pacc[nt], da[2 * kp + 1][0], da[2 * kp + 1][1], b[2], b[3]);
                }
            }
            // P and dS of (head r, key 8 nt + cq + e)
            float pr[2][2], ds[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = nt * 8 + cq + e;
                    const bool v = hrow && ((msk >> col) & 1u);
                    const float pv = v ? ex2(sacc[nt][e] * p.scale_log2 - lse2) : 0.f;
                    pr[nt][e] = pv;
                    ds[nt][e] = pv * (pacc[nt][e] - drow);
                }
            // dQ += dS K  (rows = heads, as the forward's P V)
            const uint32_t sa0 = pack_bf16(ds[0][0], ds[0][1]);
            const uint32_t sa2 = pack_bf16(ds[1][0], ds[1][1]);
#pragma unroll
            for (int np = 0; np < D / 16; ++np) {
                uint32_t b[4];
                ldsm_x4_trans(kbase + ((mi & 1) * 8 + ri) * C::STRIDE + (np * 16 + (mi >> 1) * 8) * 2,
                              b);
                float d0[4] = {dq[2 * np][0], dq[2 * np][1], 0.f, 0.f};
                float d1[4] = {dq[2 * np + 1][0], dq[2 * np + 1][1], 0.f, 0.f};
                mma_bf16(d0, sa0, sa2, b[0], b[1]);
                mma_bf16(d1, sa0, sa2, b[2], b[3]);
                dq[2 * np][0] = d0[0];
                dq[2 * np][1] = d0[1];
                dq[2 * np + 1][0] = d1[0];
                dq[2 * np + 1][1] = d1[1];
            }
            // dK and dV tiles (rows = the chunk's 16 keys, k = heads): the
            // transposed score fragments are their A operands
            const uint32_t ka0 = movmatrix_trans(sa0), ka1 = movmatrix_trans(sa2);
            const uint32_t va0 = movmatrix_trans(pack_bf16(pr[0][0], pr[0][1]));
            const uint32_t va1 = movmatrix_trans(pack_bf16(pr[1][0], pr[1][1]));
            const bool v0 = (msk >> r) & 1u, v1 = (msk >> (r + 8)) & 1u;
            float* const k0 = dKg + (int64_t)(v0 ? key0 : 0) * (HKV * D);
            float* const k1 = dKg + (int64_t)(v1 ? key1 : 0) * (HKV * D);
            float* const w0 = dVg + (int64_t)(v0 ? key0 : 0) * (HKV * D);
            float* const w1 = dVg + (int64_t)(v1 ? key1 : 0) * (HKV * D);
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                float dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
                mma_k8(dk, ka0, ka1, qb[nt]);
                mma_k8(dv, va0, va1, db[nt]);
                if (v0) {
                    red_add_v2(k0 + nt * 8, dk[0] * p.scale, dk[1] * p.scale);
                    red_add_v2(w0 + nt * 8, dv[0], dv[1]);
                }
                if (v1) {
                    red_add_v2(k1 + nt * 8, dk[2] * p.scale, dk[3] * p.scale);
                    red_add_v2(w1 + nt * 8, dv[2], dv[3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    if (!ok || !hrow) return;
    float* out = p.dQ + (t * HQ + g * G + r) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
        *reinterpret_cast<float2*>(out + n * 8 + cq) =
            make_float2(dq[n][0] * p.scale, dq[n][1] * p.scale);
}

}  // namespace attn
}  // namespace dsa

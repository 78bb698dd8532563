// Indexer warm-up loss, backward into the query side on the 5th-generation
// tensor cores: dq_I and dw for one indexer head and 128 query rows.
//
// Formulas (Kwai Keye-VL-2.0 technical-report summary, section 1, dense
// warm-up; the reading is stated in indexer_kl.cuh):
//   S[t,s]     = q_I[t,j] . k_I[s]                       (exact in fp32)
//   dS[t,s]    = G[t,s] w[t,j] [S[t,s] > 0]   (s <= t)
//   dq_I[t,j]  = sum_s dS[t,s] k_I[s],  dw[t,j] = sum_s G[t,s] relu(S[t,s])
//
// Per CTA and 128-key tile:
//   1. eight worker warps copy the key rows from global memory into two
//      shared tiles: e4m3 K-major (128-byte swizzle, the operand of S) and
//      bf16 MN-major (128-byte swizzle, the operand of the dq product), two
//      tiles ahead (three stages);
//   2. one thread issues S = q . k^T (tcgen05 kind::f8f6f4, M = N = 128,
//      K = 128) into a double-buffered TMEM accumulator;
//   3. the workers read S rows from TMEM (thread = query row, two warps per
//      32-row lane group, one half of the keys each), build dS in bf16 into
//      a K-major swizzled tile and accumulate dw in fp32;
//   4. the same thread issues dq += dS . k (kind::f16, bf16, B MN-major) into
//      a third TMEM region, which the workers read out at the end.
// The workers build dS of tile i before they wait for the dq product of
// tile i - 1 (to reuse its key stage for tile i + 2), so that wait finds it
// done; the tensor core runs S of tile i + 1 and dq of tile i meanwhile.
// Every wait is bounded (2 s); a wait that gives up sets an abort flag, after which the
// CTA stops issuing, waits (bounded) for its own MMAs, frees TMEM and
// returns with DSA_DEVERR_TIMEOUT recorded.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "ptx.cuh"
#include "indexer_kl.cuh"

namespace dsa {
namespace kltc {

constexpr int kRows = 128;                // query rows per CTA (TMEM lanes)
constexpr int kKeys = 128;                // keys per tile
constexpr int kDI = 128;                  // indexer head dim (one 128-byte e4m3 row)
constexpr int kWorkers = 8;               // worker warps
constexpr int kMmaWarp = kWorkers;        // the warp that allocates TMEM and issues MMAs
constexpr int kThreads = (kWorkers + 1) * 32;
constexpr int kTmemCols = 512;            // S[2] at 0 / 128, dq at 256

// Shared layout, from a 1024-byte aligned base.
constexpr int kQ = 0;                          // e4m3 [128 rows][128 B], K-major SW128
constexpr int kK8 = kQ + kRows * kDI;          // e4m3 k tiles [3]
constexpr int kStages = 3;                     // key tile stages
constexpr int kKB = kK8 + kStages * kKeys * kDI;  // bf16 k tiles [3], MN-major SW128
constexpr int kKB_BYTES = kKeys * kDI * 2;
constexpr int kDS = kKB + kStages * kKB_BYTES;    // bf16 dS tiles [2], K-major SW128 (two 64-key halves)
constexpr int kDS_BYTES = kRows * kKeys * 2;
constexpr int kMisc = kDS + 2 * kDS_BYTES;

struct Misc {
    uint64_t kready[kStages];  // workers: e4m3 + bf16 key tile (and the query tile) written
    uint64_t sfull[2];         // MMA: S of the tile complete
    uint64_t dsready[2];       // workers: S read, dS written
    uint64_t kfree[kStages];   // MMA: dq product of the tile complete (its key stage and dS buffer free)
    uint64_t done;        // MMA: every MMA complete
    uint32_t tmem_base;
    volatile int abort_flag;
    float dw[kRows];      // second half's partial per row (dw, kl, running max)
    float xl[kRows];      // second half's running sum per row (head_lse_tc_kernel)
};
constexpr int kSmemBytes = kMisc + (int)sizeof(Misc) + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory per block");

// Instruction descriptors: M = N = 128, fp32 accumulator.
//   S:  kind::f8f6f4, A and B e4m3, both K-major.
//   dq: kind::f16, A and B bf16, A K-major, B MN-major.
constexpr uint32_t kIdescS = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(kKeys >> 3) << 17) |
                             ((uint32_t)(kRows >> 4) << 24);
constexpr uint32_t kIdescDQ = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              ((uint32_t)(kDI >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory descriptor with 128-byte swizzle, given the leading and the
// stride byte offsets (version 1).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;  // SWIZZLE_128B
    return d;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 bytes from global memory in one request (a whole sector); the address
// is 32-byte aligned.
__device__ __forceinline__ void ld_global_v8(const void* ptr, uint32_t (&v)[8]) {
    asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7])
                 : "l"(ptr));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Byte offset of 16-byte chunk `c` of row `r` in a K-major tile of 128-byte
// rows with the 128-byte swizzle (8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t kmajor_off(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}


// ------------------------------------------------------------ cooperative tile loads
// The 256 worker threads fill a 128-row operand tile in 32-byte pieces
// assigned so that one warp request covers whole rows (8 cache lines rather
// than one line per thread): the tile goes to shared memory for the tensor
// core, so which thread moves which piece does not matter.
constexpr int kWorkerThreads = kWorkers * 32;

struct F8Pieces {  // e4m3 tile of 128 rows x 128 bytes: 2 pieces per thread
    uint32_t x[2][8];
};
struct BfPieces {  // bf16 tile of 128 rows x 128 elements: 4 pieces per thread
    uint32_t x[4][8];
};

__device__ __forceinline__ void ld_piece(const uint8_t* src, bool v8, uint32_t (&x)[8]) {
    if (v8) {
        ld_global_v8(src, x);
    } else {
        const uint4 a = *reinterpret_cast<const uint4*>(src);
        const uint4 b = *reinterpret_cast<const uint4*>(src + 16);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}

// Rows r at row0 + r * stride bytes; rows >= nvalid are zeros.
__device__ __forceinline__ void load_f8_tile(F8Pieces& P, const uint8_t* row0, int64_t nvalid,
                                             int64_t stride, bool v8, int tid) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int pc = i * kWorkerThreads + tid, r = pc >> 2, c4 = pc & 3;
        if (r < nvalid) {
            ld_piece(row0 + r * stride + 32 * c4, v8, P.x[i]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) P.x[i][e] = 0u;
        }
    }
}

// Stores the pieces into a K-major e4m3 tile (with_e4m3) and, if kb != 0,
// their bf16 values into the 2048-byte-group tile described above.
__device__ __forceinline__ void put_f8_tile(const F8Pieces& P, uint32_t k8, bool with_e4m3,
                                            uint32_t kb, int tid) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int pc = i * kWorkerThreads + tid, r = pc >> 2, c4 = pc & 3;
        const uint32_t(&x)[8] = P.x[i];
        if (with_e4m3) {
            st_shared_v4(k8 + kmajor_off(r, 2 * c4), make_uint4(x[0], x[1], x[2], x[3]));
            st_shared_v4(k8 + kmajor_off(r, 2 * c4 + 1), make_uint4(x[4], x[5], x[6], x[7]));
        }
        if (kb) {
            uint32_t o[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint2 b = kl::e4m3x4_to_bf16x4(x[q]);
                o[2 * q] = b.x;
                o[2 * q + 1] = b.y;
            }
            const uint32_t atom = kb + (uint32_t)((r >> 3) * 2048 + (c4 >> 1) * 1024 + (r & 7) * 128);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
                st_shared_v4(atom + ((((c4 & 1) * 4 + qq) ^ (r & 7)) << 4),
                             make_uint4(o[4 * qq], o[4 * qq + 1], o[4 * qq + 2], o[4 * qq + 3]));
        }
    }
}

// bf16 rows r at row0 + r * stride elements; rows >= nvalid are zeros.
__device__ __forceinline__ void load_bf_tile(BfPieces& P, const __nv_bfloat16* row0, int64_t nvalid,
                                             int64_t stride, bool v8, int tid) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pc = i * kWorkerThreads + tid, r = pc >> 3, c8 = pc & 7;
        if (r < nvalid) {
            ld_piece(reinterpret_cast<const uint8_t*>(row0 + r * stride) + 32 * c8, v8, P.x[i]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) P.x[i][e] = 0u;
        }
    }
}

__device__ __forceinline__ void put_bf_tile(const BfPieces& P, uint32_t tile, int tid) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int pc = i * kWorkerThreads + tid, r = pc >> 3, c8 = pc & 7;
        const uint32_t(&x)[8] = P.x[i];
        const uint32_t atom = tile + (uint32_t)((r >> 3) * 2048 + (c8 >> 2) * 1024 + (r & 7) * 128);
        st_shared_v4(atom + ((((c8 & 3) * 2) ^ (r & 7)) << 4), make_uint4(x[0], x[1], x[2], x[3]));
        st_shared_v4(atom + ((((c8 & 3) * 2 + 1) ^ (r & 7)) << 4), make_uint4(x[4], x[5], x[6], x[7]));
    }
}

// Grid (HI, ceil(L / 128)): the heads of one query tile run side by side;
// the longest query tiles first.
__global__ void __launch_bounds__(kThreads, 1) dq_tc_kernel(const kl::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Misc* misc = reinterpret_cast<Misc*>(smem + kMisc);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x;
    const int ntq = (int)((p.L + kRows - 1) / kRows);
    const int qt = ntq - 1 - (int)blockIdx.y;
    const int64_t t0 = (int64_t)qt * kRows;
    const int nkt = qt + 1;  // key tiles 0 .. qt

    if (threadIdx.x == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&misc->kready[b]), kWorkers);
            mbar_init(smem_u32(&misc->kfree[b]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&misc->sfull[b]), 1);
            mbar_init(smem_u32(&misc->dsready[b]), kWorkers);
        }
        mbar_init(smem_u32(&misc->done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint64_t adesc_q = sdesc_sw128(sb + kQ, 16, 1024);
            auto dq_tile = [&](int kt) {
                const int b = kt & 1, st = kt % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->dsready[b]), (kt >> 1) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) return;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kKeys / 16; ++kk) {
                    const uint64_t a = sdesc_sw128(
                        sb + kDS + b * kDS_BYTES + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sb + kKB + st * kKB_BYTES + kk * 4096, 1024, 2048);
                    umma_f16(tmem + 256, a, bd, kIdescDQ, (kt > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&misc->kfree[st]));
            };
            for (int kt = 0; kt < nkt; ++kt) {
                const int b = kt & 1, st = kt % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->kready[st]), (kt / kStages) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) break;
                tc_fence_after();
                const uint64_t bdesc_k = sdesc_sw128(sb + kK8 + st * (kKeys * kDI), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < kDI / 32; ++kk)
                    umma_f8f6f4(tmem + b * 128, adesc_q + (uint64_t)(2 * kk),
                                bdesc_k + (uint64_t)(2 * kk), kIdescS, kk > 0 ? 1u : 0u);
                umma_commit(smem_u32(&misc->sfull[b]));
                if (kt >= 1) dq_tile(kt - 1);
            }
            if (!misc->abort_flag) dq_tile(nkt - 1);
            umma_commit(smem_u32(&misc->done));
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ workers
        const int h = warp >> 2;                       // key half of this warp
        const int m = (warp & 3) * 32 + lane;          // TMEM lane = query row
        const int64_t t = t0 + m;
        const bool trow = t < p.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float wj = trow ? p.w[t * p.HI + j] : 0.f;
        // 32-byte requests where rows are 32-byte aligned
        const bool g_vec = (p.L & 7) == 0 && (reinterpret_cast<uintptr_t>(p.Gin) & 31) == 0;
        const bool q_v8 = (reinterpret_cast<uintptr_t>(p.qI) & 31) == 0;
        const bool k_v8 = (reinterpret_cast<uintptr_t>(p.kI) & 31) == 0;

        const int tid = threadIdx.x;
        // the query tile of head j, written with key tile 0
        {
            F8Pieces P;
            load_f8_tile(P, p.qI + (t0 * p.HI + j) * kDI, p.L - t0, (int64_t)p.HI * kDI, q_v8, tid);
            put_f8_tile(P, sb + kQ, true, 0, tid);
        }
        auto load_k = [&](int kt, F8Pieces& P) {
            const int64_t s0k = (int64_t)kt * kKeys;
            load_f8_tile(P, p.kI + s0k * kDI, p.L - s0k, kDI, k_v8, tid);
        };
        auto put_k = [&](int kt, const F8Pieces& P) {
            const int st = kt % kStages;
            put_f8_tile(P, sb + kK8 + st * (kKeys * kDI), true, sb + kKB + st * kKB_BYTES, tid);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->kready[st]));
        };
        {
            F8Pieces P;
            load_k(0, P);
            put_k(0, P);
            if (nkt > 1) {
                load_k(1, P);
                put_k(1, P);
            }
        }

        float dw_acc = 0.f;
        for (int kt = 0; kt < nkt; ++kt) {
            const int b = kt & 1;
            // the key rows of tile kt + 2 and this tile's G row segment, in flight together
            F8Pieces kv;
            if (kt + 2 < nkt) load_k(kt + 2, kv);
            const int64_t s0 = (int64_t)kt * kKeys + 64 * h;
            float g[64];
            if (trow && g_vec) {  // 32-byte requests, one whole sector each
                const float* gp = p.Gin + t * p.L + s0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint32_t x[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                    if (s0 + 8 * i < p.L) ld_global_v8(gp + 8 * i, x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) g[8 * i + e] = __uint_as_float(x[e]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) g[i] = trow && s0 + i <= t ? p.Gin[t * p.L + s0 + i] : 0.f;
            }
            if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->sfull[b]), (kt >> 1) & 1))
                misc->abort_flag = 1;
            if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // warp-uniform: TMEM loads below
                tc_fence_after();
                float sv[64];
                {
                    float a[32], c[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h, a);
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h + 32, c);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        sv[i] = a[i];
                        sv[32 + i] = c[i];
                    }
                }
                // dS (bf16) into the K-major tile: row m, keys [64 h, 64 h + 64); the
                // buffer's previous tile (kt - 2) was waited for one iteration ago
                const uint32_t ds = sb + kDS + b * kDS_BYTES + h * (kRows * 128);
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    uint32_t o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float d2[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int i = c8 * 8 + 2 * q + e;
                            const bool vis = s0 + i <= t;
                            const float gv = vis ? g[i] : 0.f;
                            dw_acc = fmaf(gv, fmaxf(sv[i], 0.f), dw_acc);
                            d2[e] = sv[i] > 0.f ? gv * wj : 0.f;
                        }
                        o[q] = kl::pack_bf16(d2[0], d2[1]);
                    }
                    st_shared_v4(ds + kmajor_off(m, c8), make_uint4(o[0], o[1], o[2], o[3]));
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&misc->dsready[b]));
            }
            // The dq product of tile kt - 1 must be done before the next
            // iteration writes its dS buffer and before tile kt + 2 takes its
            // key stage.
            if (kt >= 1 && kt + 1 < nkt && !misc->abort_flag &&
                !mbar_wait_to(p.err, smem_u32(&misc->kfree[(kt - 1) % kStages]), ((kt - 1) / kStages) & 1))
                misc->abort_flag = 1;
            if (kt + 2 < nkt && !misc->abort_flag) put_k(kt + 2, kv);
        }
        // dq and dw
        if (!mbar_wait_to(p.err, smem_u32(&misc->done), 0)) misc->abort_flag = 1;
        tc_fence_after();
        if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // the TMEM loads are warp-collective
            float a[32], c[32];
            tmem_ld_32x32b_x32(tmem + lane_base + 256 + 64 * h, a);
            tmem_ld_32x32b_x32(tmem + lane_base + 256 + 64 * h + 32, c);
            if (trow) {
                float* out = p.dq + (t * p.HI + j) * kDI + 64 * h;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    reinterpret_cast<float4*>(out)[i] =
                        make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    reinterpret_cast<float4*>(out + 32)[i] =
                        make_float4(c[4 * i], c[4 * i + 1], c[4 * i + 2], c[4 * i + 3]);
            }
        }
        if (h == 1) misc->dw[m] = dw_acc;
        named_bar_sync(1, kWorkers * 32);
        if (h == 0 && trow && !misc->abort_flag) p.dw[t * p.HI + j] = dw_acc + misc->dw[m];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- dk

// dk_I for 128 keys over the query tiles at or after theirs and a group of
// heads, keys on the TMEM lanes:
//   S^T[s,t]  = k_I[s] . q_I[t,j]            (tcgen05 kind::f16, bf16)
//   dS^T[s,t] = G[t,s] w[t,j] [S > 0]       (t >= s)
//   dk[s]    += sum_t dS^T[s,t] q_I[t,j]     (kind::f16, B MN-major)
// G^T of a query tile is read once (32 consecutive keys per token and
// request) and serves every head of the group; w of the tile is staged in
// shared memory.  Each query tile and head is one unit; the units' q tiles
// go through three stages, as the key tiles of dq_tc_kernel.
constexpr int kMaxHps = 32;                        // heads per group
constexpr int kDkKB = 0;                           // bf16 k tile (A of S^T)
constexpr int kDkQB = kDkKB + kKB_BYTES;           // bf16 q tiles [3]
constexpr int kDkDS = kDkQB + kStages * kKB_BYTES; // bf16 dS^T tiles [2]
constexpr int kDkW = kDkDS + 2 * kDS_BYTES;        // w^T of the query tile [2][hps][128]
constexpr int kDkMisc = kDkW + 2 * kMaxHps * kRows * 4;
constexpr int kDkSmemBytes = kDkMisc + (int)sizeof(Misc) + 1024;
static_assert(kDkSmemBytes <= 232448, "shared memory per block");

constexpr uint32_t kIdescSt = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRows >> 3) << 17) |
                              ((uint32_t)(kRows >> 4) << 24);

// Grid (nsplit, ceil(L / 128)): the groups of one key tile side by side; the
// longest key tiles (the first) first.
__global__ void __launch_bounds__(kThreads, 1) dk_tc_kernel(const kl::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Misc* misc = reinterpret_cast<Misc*>(smem + kDkMisc);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int hps = p.HI / p.nsplit, j0 = split * hps;
    const int ntq = (int)((p.L + kRows - 1) / kRows);
    const int kt = (int)blockIdx.y;
    const int64_t s_base = (int64_t)kt * kRows;
    const int nunits = (ntq - kt) * hps;  // (query tile, head) pairs

    if (threadIdx.x == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&misc->kready[b]), kWorkers);
            mbar_init(smem_u32(&misc->kfree[b]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&misc->sfull[b]), 1);
            mbar_init(smem_u32(&misc->dsready[b]), kWorkers);
        }
        mbar_init(smem_u32(&misc->done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            auto dk_unit = [&](int u) {
                const int b = u & 1, st = u % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->dsready[b]), (u >> 1) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) return;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kRows / 16; ++kk) {
                    const uint64_t a = sdesc_sw128(
                        sb + kDkDS + b * kDS_BYTES + (kk >> 2) * (kRows * 128) + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(sb + kDkQB + st * kKB_BYTES + kk * 4096, 1024, 2048);
                    umma_f16(tmem + 256, a, bd, kIdescDQ, (u > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(smem_u32(&misc->kfree[st]));
            };
            for (int u = 0; u < nunits; ++u) {
                const int b = u & 1, st = u % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->kready[st]), (u / kStages) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kDI / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 32;
                    umma_f16(tmem + b * 128, sdesc_sw128(sb + kDkKB + off, 16, 2048),
                             sdesc_sw128(sb + kDkQB + st * kKB_BYTES + off, 16, 2048), kIdescSt,
                             kk > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&misc->sfull[b]));
                if (u >= 1) dk_unit(u - 1);
            }
            if (!misc->abort_flag && nunits > 0) dk_unit(nunits - 1);
            umma_commit(smem_u32(&misc->done));
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ workers
        const int h = warp >> 2;                  // token half of this warp
        const int m = (warp & 3) * 32 + lane;     // TMEM lane = key row
        const int64_t s = s_base + m;
        const bool srow = s < p.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool q_v8 = (reinterpret_cast<uintptr_t>(p.qI) & 31) == 0;
        const bool k_v8 = (reinterpret_cast<uintptr_t>(p.kI) & 31) == 0;
        const int64_t qstride = (int64_t)p.HI * kDI;
        float* wS = reinterpret_cast<float*>(smem + kDkW);

        const int tid = threadIdx.x;
        // the key tile in bf16, written with unit 0
        {
            F8Pieces P;
            load_f8_tile(P, p.kI + s_base * kDI, p.L - s_base, kDI, k_v8, tid);
            put_f8_tile(P, 0, false, sb + kDkKB, tid);
        }
        auto load_q = [&](int u, F8Pieces& P) {
            const int64_t tq0 = s_base + (int64_t)(u / hps) * kRows;  // first token of the unit
            load_f8_tile(P, p.qI + tq0 * qstride + (j0 + u % hps) * kDI, p.L - tq0, qstride, q_v8, tid);
        };
        auto put_q = [&](int u, const F8Pieces& P) {
            const int st = u % kStages;
            put_f8_tile(P, 0, false, sb + kDkQB + st * kKB_BYTES, tid);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->kready[st]));
        };
        {
            F8Pieces P;
            if (nunits > 0) {
                load_q(0, P);
                put_q(0, P);
            }
            if (nunits > 1) {
                load_q(1, P);
                put_q(1, P);
            }
        }

        float gT[64];
        for (int u = 0; u < nunits; ++u) {
            const int b = u & 1, jj = u % hps, qi = u / hps;
            const int64_t tq = s_base + (int64_t)qi * kRows;  // first token of the query tile
            F8Pieces qv;
            if (u + 2 < nunits) load_q(u + 2, qv);
            if (jj == 0) {
                // G^T of this query tile (token half h), and its w^T
                const int64_t t0h = tq + 64 * h;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const int64_t t = t0h + i;
                    gT[i] = srow && t < p.L && t >= s ? p.Gin[t * p.L + s] : 0.f;
                }
                float* wb = wS + (qi & 1) * (kMaxHps * kRows);
                for (int i = threadIdx.x; i < hps * kRows; i += kWorkers * 32) {
                    const int hh = i / kRows, tt = i % kRows;
                    wb[hh * kRows + tt] = tq + tt < p.L ? p.w[(tq + tt) * p.HI + j0 + hh] : 0.f;
                }
                named_bar_sync(1, kWorkers * 32);
            }
            if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->sfull[b]), (u >> 1) & 1))
                misc->abort_flag = 1;
            if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // warp-uniform: TMEM loads below
                tc_fence_after();
                float sv[64];
                {
                    float a[32], c[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h, a);
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h + 32, c);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        sv[i] = a[i];
                        sv[32 + i] = c[i];
                    }
                }
                const float4* wr =
                    reinterpret_cast<const float4*>(wS + (qi & 1) * (kMaxHps * kRows) + jj * kRows + 64 * h);
                const uint32_t ds = sb + kDkDS + b * kDS_BYTES + h * (kRows * 128);
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const float4 w0 = wr[2 * c8], w1 = wr[2 * c8 + 1];
                    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint32_t o[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float d2[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int i = c8 * 8 + 2 * q + e;
                            d2[e] = sv[i] > 0.f ? gT[i] * wv[2 * q + e] : 0.f;
                        }
                        o[q] = kl::pack_bf16(d2[0], d2[1]);
                    }
                    st_shared_v4(ds + kmajor_off(m, c8), make_uint4(o[0], o[1], o[2], o[3]));
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&misc->dsready[b]));
            }
            if (u >= 1 && u + 1 < nunits && !misc->abort_flag &&
                !mbar_wait_to(p.err, smem_u32(&misc->kfree[(u - 1) % kStages]), ((u - 1) / kStages) & 1))
                misc->abort_flag = 1;
            if (u + 2 < nunits && !misc->abort_flag) put_q(u + 2, qv);
        }
        if (!mbar_wait_to(p.err, smem_u32(&misc->done), 0)) misc->abort_flag = 1;
        tc_fence_after();
        if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // the TMEM loads are warp-collective
            float a[32], c[32];
            tmem_ld_32x32b_x32(tmem + lane_base + 256 + 64 * h, a);
            tmem_ld_32x32b_x32(tmem + lane_base + 256 + 64 * h + 32, c);
            if (srow) {
                float* dk = p.nsplit > 1 ? p.dk_part + (int64_t)split * p.L * kDI : p.dk;
                float* out = dk + s * kDI + 64 * h;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    reinterpret_cast<float4*>(out)[i] =
                        make_float4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    reinterpret_cast<float4*>(out + 32)[i] =
                        make_float4(c[4 * i], c[4 * i + 1], c[4 * i + 2], c[4 * i + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- forward

// S (128 x 128) = A . B^T over D = 128 from two bf16 tiles of that layout.
__device__ __forceinline__ void mma_bf16_tile(uint32_t d_tmem, uint32_t a_tile, uint32_t b_tile) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 32;
        umma_f16(d_tmem, sdesc_sw128(a_tile + off, 16, 2048), sdesc_sw128(b_tile + off, 16, 2048),
                 kIdescSt, kk > 0 ? 1u : 0u);
    }
}

constexpr int kFwdQ = 0;                            // bf16 tile of the fixed operand
constexpr int kFwdS = kFwdQ + kKB_BYTES;            // bf16 streamed tiles [3]
constexpr int kFwdMisc = kFwdS + kStages * kKB_BYTES;
constexpr int kLseSmemBytes = kFwdMisc + (int)sizeof(Misc) + 1024;
constexpr int kD = 128;                             // attention head dim of these kernels

// lse_h[t][h] (log2 domain) of scale * Q[t,h] . K[s,g] over s <= t, for 128
// query rows and one head: S tiles of 128 keys in double-buffered TMEM; each
// worker keeps an online max and sum over its half of the keys.  Grid (Hq,
// ceil(L / 128)): the heads of a query tile side by side, longest first.
__global__ void __launch_bounds__(kThreads, 1) head_lse_tc_kernel(const kl::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Misc* misc = reinterpret_cast<Misc*>(smem + kFwdMisc);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hq = blockIdx.x, g = hq / (p.Hq / p.Hkv);
    const int ntq = (int)((p.L + kRows - 1) / kRows);
    const int qt = ntq - 1 - (int)blockIdx.y;
    const int64_t t0 = (int64_t)qt * kRows;
    const int nkt = qt + 1;

    if (threadIdx.x == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&misc->kready[b]), kWorkers);
            mbar_init(smem_u32(&misc->kfree[b]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&misc->sfull[b]), 1);
            mbar_init(smem_u32(&misc->dsready[b]), kWorkers);  // here: S buffer read
        }
        mbar_init(smem_u32(&misc->done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kMmaWarp) {
        if (lane == 0) {
            for (int kt = 0; kt < nkt; ++kt) {
                const int b = kt & 1, st = kt % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->kready[st]), (kt / kStages) & 1))
                    misc->abort_flag = 1;
                if (!misc->abort_flag && kt >= 2 &&
                    !mbar_wait_to(p.err, smem_u32(&misc->dsready[b]), ((kt - 2) >> 1) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) break;
                tc_fence_after();
                mma_bf16_tile(tmem + b * 128, sb + kFwdQ, sb + kFwdS + st * kKB_BYTES);
                umma_commit(smem_u32(&misc->sfull[b]));
                umma_commit(smem_u32(&misc->kfree[st]));
            }
            umma_commit(smem_u32(&misc->done));
        }
        __syncwarp();
    } else {
        const int h = warp >> 2;
        const int m = (warp & 3) * 32 + lane;
        const int64_t t = t0 + m;
        const bool trow = t < p.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool q_v8 = (reinterpret_cast<uintptr_t>(p.Q) & 31) == 0;
        const bool k_v8 = (reinterpret_cast<uintptr_t>(p.K) & 31) == 0;
        const int64_t kstride = (int64_t)p.Hkv * kD;
        const int tid = threadIdx.x;
        {
            BfPieces P;
            load_bf_tile(P, p.Q + (t0 * p.Hq + hq) * kD, p.L - t0, (int64_t)p.Hq * kD, q_v8, tid);
            put_bf_tile(P, sb + kFwdQ, tid);
        }
        auto load_k = [&](int kt, BfPieces& P) {
            const int64_t s0k = (int64_t)kt * kKeys;
            load_bf_tile(P, p.K + s0k * kstride + g * kD, p.L - s0k, kstride, k_v8, tid);
        };
        auto put_k = [&](int kt, const BfPieces& P) {
            const int st = kt % kStages;
            put_bf_tile(P, sb + kFwdS + st * kKB_BYTES, tid);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->kready[st]));
        };
        {
            BfPieces P;
            load_k(0, P);
            put_k(0, P);
            if (nkt > 1) {
                load_k(1, P);
                put_k(1, P);
            }
        }
        float mrun = -INFINITY, lrun = 0.f;
        for (int kt = 0; kt < nkt; ++kt) {
            const int b = kt & 1;
            BfPieces kv;
            if (kt + 2 < nkt) load_k(kt + 2, kv);
            if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->sfull[b]), (kt >> 1) & 1))
                misc->abort_flag = 1;
            if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // warp-uniform: TMEM loads below
                tc_fence_after();
                const int64_t s0 = (int64_t)kt * kKeys + 64 * h;
                const bool diag = kt == qt;  // only the diagonal tile has keys past a row
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h + 32 * half, x);
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&misc->dsready[b]));
                    }
                    if (diag) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (s0 + 32 * half + i > t) x[i] = -INFINITY;
                    }
                    float mx = -INFINITY;
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, x[i]);
                    // scale > 0: the max of the scaled values is the scaled max
                    const float mn = fmaxf(mrun, mx * p.scale_log2);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    float sum = 0.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) sum += kl::ex2(fmaf(x[i], p.scale_log2, -mu));
                    lrun = lrun * kl::ex2(mrun - mu) + sum;
                    mrun = mn;
                }
            }
            if (kt >= 1 && kt + 1 < nkt && !misc->abort_flag &&
                !mbar_wait_to(p.err, smem_u32(&misc->kfree[(kt - 1) % kStages]), ((kt - 1) / kStages) & 1))
                misc->abort_flag = 1;
            if (kt + 2 < nkt && !misc->abort_flag) put_k(kt + 2, kv);
        }
        // combine the two halves of each row (the second half's max may be
        // -inf: it can hold no visible key)
        if (h == 1) {
            misc->dw[m] = mrun;
            misc->xl[m] = lrun;
        }
        named_bar_sync(1, kWorkers * 32);
        if (h == 0) {
            const float mo = misc->dw[m], lo = misc->xl[m];
            const float mt = fmaxf(mrun, mo);
            const float mu = mt == -INFINITY ? 0.f : mt;
            const float l = lrun * kl::ex2(mrun - mu) + lo * kl::ex2(mo - mu);
            if (trow && !misc->abort_flag) p.lse_h[t * p.Hq + hq] = mt + kl::lg2(l);
        }
        if (!mbar_wait_to(p.err, smem_u32(&misc->done), 0)) misc->abort_flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

constexpr int kTgtK = 0;                                 // bf16 key tiles of every group [Hkv <= 4]
constexpr int kTgtQ = kTgtK + 4 * kKB_BYTES;             // bf16 query tiles [3]
constexpr int kTgtMisc = kTgtQ + kStages * kKB_BYTES;
constexpr int kTgtSmemBytes = kTgtMisc + (int)sizeof(Misc) + 1024;
static_assert(kTgtSmemBytes <= 232448, "shared memory per block");

// One (query tile, key tile) of 128 x 128: p summed over every query head
// (S of each head in double-buffered TMEM, its query tile streamed through
// three stages, the Hkv key tiles resident), then the KL row partials and G
// written over I.  Tiles above the diagonal only write G = 0.  Grid (ntq
// key tiles, ntq query tiles).  Needs Hkv <= 4.
__global__ void __launch_bounds__(kThreads, 1) target_tc_kernel(const kl::Params p) {
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = blockIdx.x, qt = blockIdx.y;
    const int64_t t0 = (int64_t)qt * kRows, s0 = (int64_t)kt * kKeys;
    if (kt > qt) {
        for (int i = threadIdx.x; i < kRows * kKeys; i += kThreads) {
            const int64_t t = t0 + i / kKeys, s = s0 + i % kKeys;
            if (t < p.L && s < p.L) p.G[t * p.L + s] = 0.f;
        }
        return;
    }
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Misc* misc = reinterpret_cast<Misc*>(smem + kTgtMisc);
    const uint32_t sb = smem_u32(smem);
    const int G = p.Hq / p.Hkv;
    const int nunits = p.Hq;

    if (threadIdx.x == 0) {
        for (int b = 0; b < kStages; ++b) {
            mbar_init(smem_u32(&misc->kready[b]), kWorkers);
            mbar_init(smem_u32(&misc->kfree[b]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&misc->sfull[b]), 1);
            mbar_init(smem_u32(&misc->dsready[b]), kWorkers);  // here: S buffer read
        }
        mbar_init(smem_u32(&misc->done), 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&misc->tmem_base), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kMmaWarp) {
        if (lane == 0) {
            for (int u = 0; u < nunits; ++u) {
                const int b = u & 1, st = u % kStages;
                if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->kready[st]), (u / kStages) & 1))
                    misc->abort_flag = 1;
                if (!misc->abort_flag && u >= 2 &&
                    !mbar_wait_to(p.err, smem_u32(&misc->dsready[b]), ((u - 2) >> 1) & 1))
                    misc->abort_flag = 1;
                if (misc->abort_flag) break;
                tc_fence_after();
                mma_bf16_tile(tmem + b * 128, sb + kTgtQ + st * kKB_BYTES,
                              sb + kTgtK + (u / G) * kKB_BYTES);
                umma_commit(smem_u32(&misc->sfull[b]));
                umma_commit(smem_u32(&misc->kfree[st]));
            }
            umma_commit(smem_u32(&misc->done));
        }
        __syncwarp();
    } else {
        const int h = warp >> 2;
        const int m = (warp & 3) * 32 + lane;
        const int64_t t = t0 + m;
        const bool trow = t < p.L;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const bool q_v8 = (reinterpret_cast<uintptr_t>(p.Q) & 31) == 0;
        const bool k_v8 = (reinterpret_cast<uintptr_t>(p.K) & 31) == 0;
        const int64_t kstride = (int64_t)p.Hkv * kD;
        const int tid = threadIdx.x;
        for (int g = 0; g < p.Hkv; ++g) {
            BfPieces P;
            load_bf_tile(P, p.K + s0 * kstride + g * kD, p.L - s0, kstride, k_v8, tid);
            put_bf_tile(P, sb + kTgtK + g * kKB_BYTES, tid);
        }
        auto load_q = [&](int u, BfPieces& P) {
            load_bf_tile(P, p.Q + (t0 * p.Hq + u) * kD, p.L - t0, (int64_t)p.Hq * kD, q_v8, tid);
        };
        auto put_q = [&](int u, const BfPieces& P) {
            const int st = u % kStages;
            put_bf_tile(P, sb + kTgtQ + st * kKB_BYTES, tid);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&misc->kready[st]));
        };
        {
            BfPieces P;
            load_q(0, P);
            put_q(0, P);
            if (nunits > 1) {
                load_q(1, P);
                put_q(1, P);
            }
        }
        const int64_t sh = s0 + 64 * h;  // first key of this thread's half
        float P[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) P[i] = 0.f;
        // Keys past a row (diagonal tile only) accumulate too and are skipped
        // by the epilogue.  Each head's lse is fetched one head ahead.
        float lse_next = trow ? p.lse_h[t * p.Hq] : 0.f;
        for (int u = 0; u < nunits; ++u) {
            const int b = u & 1;
            BfPieces qv;
            if (u + 2 < nunits) load_q(u + 2, qv);
            const float lse = lse_next;
            if (u + 1 < nunits) lse_next = trow ? p.lse_h[t * p.Hq + u + 1] : 0.f;
            if (!misc->abort_flag && !mbar_wait_to(p.err, smem_u32(&misc->sfull[b]), (u >> 1) & 1))
                misc->abort_flag = 1;
            if (!__any_sync(0xffffffffu, misc->abort_flag)) {  // warp-uniform: TMEM loads below
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float x[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + b * 128 + 64 * h + 32 * half, x);
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&misc->dsready[b]));
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        P[32 * half + i] += kl::ex2(fmaf(x[i], p.scale_log2, -lse));
                }
            }
            if (u >= 1 && u + 1 < nunits && !misc->abort_flag &&
                !mbar_wait_to(p.err, smem_u32(&misc->kfree[(u - 1) % kStages]), ((u - 1) / kStages) & 1))
                misc->abort_flag = 1;
            if (u + 2 < nunits && !misc->abort_flag) put_q(u + 2, qv);
        }
        // KL partial and G over this thread's 64 keys of row t
        const float inv_h = 1.f / (float)p.Hq;
        const float lse_I = trow ? p.lse_I[t] : 0.f;
        float klp = 0.f;
        const bool gv8 = (p.L & 7) == 0 && (reinterpret_cast<uintptr_t>(p.G) & 31) == 0;
        if (trow && !misc->abort_flag) {
            float* grow = p.G + t * p.L + sh;
            if (gv8) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (sh + 8 * c >= p.L) continue;
                    uint32_t x[8];
                    ld_global_v8(grow + 8 * c, x);
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 8 * c + e;
                        float gvl = 0.f;
                        if (sh + i <= t) {
                            const float pv = P[i] * inv_h;
                            const float lq = p.scale_I * __uint_as_float(x[e]) - lse_I;
                            klp += pv > 0.f ? pv * (kl::lg2(pv) * kl::kLn2 - lq) : 0.f;
                            gvl = p.scale_I * (kl::ex2(lq * kl::kLog2e) - pv);
                        }
                        o[e] = gvl;
                    }
                    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(grow + 8 * c),
                                 "f"(o[0]), "f"(o[1]), "f"(o[2]), "f"(o[3]), "f"(o[4]), "f"(o[5]),
                                 "f"(o[6]), "f"(o[7])
                                 : "memory");
                }
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if (sh + i >= p.L) continue;
                    float gvl = 0.f;
                    if (sh + i <= t) {
                        const float pv = P[i] * inv_h;
                        const float lq = p.scale_I * grow[i] - lse_I;
                        klp += pv > 0.f ? pv * (kl::lg2(pv) * kl::kLn2 - lq) : 0.f;
                        gvl = p.scale_I * (kl::ex2(lq * kl::kLog2e) - pv);
                    }
                    grow[i] = gvl;
                }
            }
        }
        if (h == 1) misc->dw[m] = klp;
        named_bar_sync(1, kWorkers * 32);
        if (h == 0 && trow && !misc->abort_flag) p.kl_part[t * p.ntiles + kt] = klp + misc->dw[m];
        if (!mbar_wait_to(p.err, smem_u32(&misc->done), 0)) misc->abort_flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace kltc
}  // namespace dsa

// Sparse GQA attention for blocks of adjacent query tokens that share their
// gathers (adjacent-query dedup), on the 5th-generation tensor cores.
//
// Kwai Keye-VL-2.0 technical-report summary, section 8, item 2: neighbouring
// queries select largely the same positions, so a block of them loads the
// union of their index sets once; the block's queries times the heads of one
// KV group fill the M = 128 rows of a tensor-core tile, and each query keeps
// only its own keys through a mask applied where the score tile is read.
// The result is the attention of dsa_sparse_attn_prefill (section 1 of the
// same page) for every query of the block.
//
// Blocks hold QB = 128 / G consecutive query tokens (G = query heads per KV
// group); the row of query j, head h of the group is m = j * G + h.  The
// blocks are processed in waves; per wave, two kernels:
//
// plan_kernel, one CTA per block: the union U of the block's index rows as
// a bitmap over the keys, a prefix count per 32-key word, and from those the
// sorted distinct keys, written to the workspace in chunks of 64 (-1 pads
// the last chunk), and for each chunk and query a 64-bit mask of the keys
// the query selected.  Entries < 0 are holes; entries >= L are skipped and
// flagged (DSA_DEVERR_INDEX); a key repeated in one row counts once.
//
// tc_kernel, one CTA per (KV group g, block), 12 warps, two CTAs per SM:
//   warps 4-5 gather the chunk's K rows of group g (three stages; the
//     block's query rows with chunk 0) and warps 6-7 its V rows (two
//     stages), with 16-byte cp.async into 128-byte-swizzled tiles; each
//     loads the next chunk's key list while the current chunk's copies are
//     issued (the rate of the gather follows the number of warps issuing
//     copies; the register split keeps the softmax at 128 registers);
//   warp 8 allocates TMEM and one thread issues, per chunk c,
//     S_c  = Q K_c^T   (kind::f16 bf16, M = 128, N = 64, K = d; K-major A
//                       and B, both in shared memory) into one of two TMEM
//                       score buffers, and
//     O   += P_c V_c   (M = 128, N = d, K = 64; A = P_c read from TMEM, V the
//                       MN-major B operand, its rows as gathered) into the
//                       TMEM accumulator; S of chunk c + 2 reuses the buffer
//                       of P_c, after P_c V_c in issue order;
//   warps 0-3 (thread = row m, the TMEM lane) read S_c, put -inf on the keys
//     their query did not select (the mask), and keep an online softmax in
//     the exp2 domain.  The offset m_run is raised only when a chunk's
//     maximum exceeds it by more than kRescaleLog2 (then, once the previous
//     product is done, the O row is read out of TMEM, scaled and written
//     back), so probabilities stay below 2^kRescaleLog2 and the accumulator
//     is rarely touched.  P_c goes to TMEM in bf16 over the first half of its
//     score buffer.  At the end each thread divides its O row by the row's
//     sum and stores it in bf16 (zeros for a row without keys).
// Every wait is bounded (2 s); a wait that gives up records
// DSA_DEVERR_TIMEOUT, the CTA stops issuing, waits (bounded) for its own
// MMAs, frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {
namespace dedup {

constexpr int kChunk = 64;              // distinct keys per chunk
constexpr int kMaxKeys = 1 << 18;       // keys the bitmap covers (32 KB)
constexpr int kMaxCap = 32768;          // distinct keys a block may have (QB x k)
constexpr int kWave = 4096;             // blocks per wave (workspace slots)
constexpr int kPlanThreads = 512;
constexpr float kRescaleLog2 = 8.f;     // lazy rescale threshold (factor 256)

// Workspace of one wave: nslot slots of `cap` key positions.
struct Layout {
    int64_t nslot, cap, qb;
    __host__ __device__ int64_t n_off() const { return 0; }
    __host__ __device__ int64_t keys_off() const { return (nslot * 4 + 255) / 256 * 256; }
    __host__ __device__ int64_t masks_off() const { return keys_off() + nslot * cap * 4; }
    __host__ __device__ int64_t bytes() const { return masks_off() + nslot * (cap / kChunk) * qb * 8; }
};

// Positions per block: the union of QB rows of k entries, and never more
// than the L keys there are; a multiple of the chunk.
__host__ __device__ inline int64_t block_cap(int64_t L, int qb, int k) {
    const int64_t c = (int64_t)qb * k < L ? (int64_t)qb * k : L;
    return (c + kChunk - 1) / kChunk * kChunk;
}

struct PlanParams {
    const int32_t* idx;   // [L][k]
    int64_t L;
    int k;
    int64_t blk0;         // first block of the wave
    int64_t cap;
    int32_t* nU;          // [nslot]
    int32_t* keys;        // [nslot][cap]
    uint64_t* masks;      // [nslot][cap / 64][QB]
    int* err;
};

__host__ __device__ inline int plan_smem_bytes(int64_t L, int64_t cap, int qb) {
    const int64_t nwords = (L + 31) / 32;
    return (int)((cap / kChunk) * qb * 8 + nwords * 4 + (nwords * 2 + 15) / 16 * 16);
}

// ORs bit(u) into arr[word(u)] for every valid entry (0 <= u < L) of one
// index row, the warp's lanes reading it in coalesced 16-byte pieces (eight
// pieces in flight per lane); the four entries of a piece are combined per
// word in registers, so rows of ascending keys need about one shared atomic
// per piece.  Entries >= L set *bad.
template <typename W>
__device__ __forceinline__ void or_row(const int32_t* row, int k, int64_t L, int lane, bool* bad,
                                       uint32_t* arr, W&& word_bit) {
    auto put = [&](const int32_t (&u)[4]) {
        int cur = -1;
        uint32_t acc = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (u[i] >= L) *bad = true;
            if (u[i] < 0 || u[i] >= L) continue;
            uint32_t bit;
            const int w = word_bit(u[i], &bit);
            if (w != cur) {
                if (acc) atomicOr(&arr[cur], acc);
                cur = w;
                acc = 0u;
            }
            acc |= bit;
        }
        if (acc) atomicOr(&arr[cur], acc);
    };
    if ((k & 3) == 0) {  // 16-byte aligned rows (the base is 16-byte aligned)
        const int4* r4 = reinterpret_cast<const int4*>(row);
        const int n4 = k >> 2;
        for (int b = 0; b < n4; b += 32 * 8) {
            int4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = b + i * 32 + lane;
                v[i] = e < n4 ? r4[e] : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                put(u);
            }
        }
    } else {
        for (int e = 4 * lane; e < k; e += 128) {
            int32_t u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) u[i] = e + i < k ? row[e + i] : -1;
            put(u);
        }
    }
}

template <int QB>
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const PlanParams p) {
    constexpr int NT = kPlanThreads;
    constexpr int NW = NT / 32;
    extern __shared__ __align__(16) uint8_t plan_smem[];
    const int nwords = (int)((p.L + 31) >> 5);
    const int64_t nmask = (p.cap / kChunk) * QB;
    uint32_t* mk = reinterpret_cast<uint32_t*>(plan_smem);  // [chunk][query] as 32-bit halves
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(plan_smem + nmask * 8);
    uint16_t* prefix = reinterpret_cast<uint16_t*>(plan_smem + nmask * 8 + (int64_t)nwords * 4);
    __shared__ int s_warp[NW];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slot = blockIdx.x;
    const int64_t t0 = (p.blk0 + slot) * QB;
    const int nq = (int)(p.L - t0 < QB ? p.L - t0 : QB);
    int32_t* keys = p.keys + slot * p.cap;
    bool bad = false;

    for (int i = tid; i < nwords; i += NT) bitmap[i] = 0u;
    __syncthreads();
    // the union as a bitmap over the keys (warp w takes rows w, w + NW, ...)
    for (int j = warp; j < nq; j += NW)
        or_row(p.idx + (t0 + j) * p.k, p.k, p.L, lane, &bad, bitmap, [](int32_t u, uint32_t* bit) {
            *bit = 1u << (u & 31);
            return (int)(u >> 5);
        });
    if (bad) record_error_to(p.err, 2);
    __syncthreads();
    // words [w0, w1) of this thread: count, block-wide scan, prefix, list
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
    for (int i = 0; i < NW; ++i) {
        base += i < warp ? s_warp[i] : 0;
        nU += s_warp[i];
    }
    int run = base + incl - cnt;
    for (int w = w0; w < w1; ++w) {
        prefix[w] = (uint16_t)run;
        uint32_t b = bitmap[w];
        while (b) {
            keys[run++] = w * 32 + (__ffs(b) - 1);
            b &= b - 1u;
        }
    }
    const int nch = (nU + kChunk - 1) / kChunk;
    for (int i = tid; i < nch * QB * 2; i += NT) mk[i] = 0u;
    for (int i = nU + tid; i < nch * kChunk; i += NT) keys[i] = -1;
    __syncthreads();
    // per query, the position in U of each selected key: bit (pos & 63) of
    // the 64-bit mask of chunk pos / 64, built in 32-bit halves
    bool unused = false;
    for (int j = warp; j < nq; j += NW)
        or_row(p.idx + (t0 + j) * p.k, p.k, p.L, lane, &unused, mk,
               [&](int32_t u, uint32_t* bit) {
                   const int pos =
                       prefix[u >> 5] + __popc(bitmap[u >> 5] & ((1u << (u & 31)) - 1u));
                   *bit = 1u << (pos & 31);
                   return ((pos >> 6) * QB + j) * 2 + ((pos >> 5) & 1);
               });
    __syncthreads();
    uint64_t* gm = p.masks + slot * nmask;
    for (int i = tid; i < nch * QB; i += NT)
        gm[i] = (uint64_t)mk[2 * i] | ((uint64_t)mk[2 * i + 1] << 32);
    if (tid == 0) p.nU[slot] = nU;
}

// ---------------------------------------------------------------- tc_kernel

struct TcParams {
    const __nv_bfloat16* Q;  // [L][Hq][D]
    const __nv_bfloat16* K;  // [L][Hkv][D]
    const __nv_bfloat16* V;
    __nv_bfloat16* O;        // [L][Hq][D]
    const int32_t* nU;       // plan of the wave
    const int32_t* keys;
    const uint64_t* masks;
    int64_t L;
    int Hq, Hkv;
    int64_t blk0;
    int64_t cap;
    float scale_log2;
    int* err;
};

template <int D, int G>
struct TcCfg {
    static constexpr int QB = 128 / G;             // query tokens per block
    static constexpr int DH = D / 64;              // 128-byte column groups of a row
    static constexpr int GROUP = DH * 1024;        // bytes of 8 rows of a [rows][D] tile
    static constexpr int Q_BYTES = 16 * GROUP;     // 128 rows
    static constexpr int KV_BYTES = 8 * GROUP;     // 64 keys
    static constexpr int KST = 3, VST = 2;         // K and V stages
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr int SMEM = OFF_BAR + 256;
    // two CTAs per SM at most: each allocates half of TMEM
    static constexpr int SMEM_LAUNCH = SMEM > 100 * 1024 ? SMEM : 100 * 1024;
    // warps 0-3 softmax, 4-5 K and 6-7 V gather, 8 MMA issuer, 9-11 idle (whole
    // warpgroups for setmaxnreg): 80 registers at launch, 128 for the
    // softmax warpgroup, 56 for the other two (128 x 128 + 256 x 56 = 384 x 80)
    static constexpr int THREADS = 12 * 32;
    static constexpr int LAUNCH_REGS = 80, SOFTMAX_REGS = 128, OTHER_REGS = 56;
    static constexpr int TMEM_COLS = 256;          // O at 0; S (then P) buffers at 128, 192
    static_assert(G * QB == 128, "block rows");
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
    static_assert(128 * SOFTMAX_REGS + 256 * OTHER_REGS <= THREADS * LAUNCH_REGS, "register split");
};

struct TcBars {
    uint64_t kfull[3], kempty[3], vfull[2], vempty[2], sfull[2], pready[2], pfree[2];
    uint64_t done;
    uint32_t tmem_base;
    volatile int abort_flag;
};

// kind::f16 instruction descriptor: bf16 A and B, fp32 accumulator, M = 128,
// N = n; B K-major, or MN-major with b_mn.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// D[tmem] (+)= A[smem] B[smem]
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] B[smem]: A is 128 lanes (rows) x K, two bf16 per
// 32-bit column, the lower K index in the low half.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory descriptor, 128-byte swizzle, version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// 16 bytes, or 16 zero bytes when nbytes == 0 (nothing is read then).
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t nbytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(nbytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 lanes x 16 columns written from registers, then waited for.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
        "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
        "f"(v[15])
        : "memory");
}

// 32 lanes x 32 columns of 32-bit words written from registers, then waited for.
__device__ __forceinline__ void tmem_st_32x32b_x32_u(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Byte offset of 16-byte piece `pc` of row r in a [rows][D] bf16 tile laid
// out as 8-row groups of DH 1024-byte atoms (128-byte swizzle).
template <int DH>
__device__ __forceinline__ uint32_t tile_off(int r, int pc) {
    return (uint32_t)((r >> 3) * (DH * 1024) + (pc >> 3) * 1024 + (r & 7) * 128 +
                      (((pc & 7) ^ (r & 7)) << 4));
}

// Two fp32 lanes per instruction (sm_100 f32x2 forms) and a 3-input max.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int D, int G>
__global__ void __launch_bounds__(TcCfg<D, G>::THREADS, 2) tc_kernel(const TcParams p) {
    using C = TcCfg<D, G>;
    constexpr int QB = C::QB;
    constexpr int PR = D / 8;          // 16-byte pieces per row
    constexpr int RPI = 32 / PR;       // rows per warp instruction
    extern __shared__ __align__(1024) uint8_t smem[];
    TcBars* bars = reinterpret_cast<TcBars*>(smem + C::OFF_BAR);
    const uint32_t sb = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;
    const int slot = (int)(gridDim.y - 1 - blockIdx.y);  // the longest blocks (last rows) first
    const int64_t t0 = (p.blk0 + slot) * QB;
    const int nU = p.nU[slot];
    const int nch = (nU + kChunk - 1) / kChunk;
    const int32_t* keys = p.keys + slot * p.cap;
    const uint64_t* masks = p.masks + slot * (p.cap / kChunk) * QB;

    if ((sb & 1023u) != 0) {  // the swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) record_error_to(p.err, 1);
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 3; ++s) {
            mbar_init(smem_u32(&bars->kfull[s]), 64);
            mbar_init(smem_u32(&bars->kempty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&bars->vfull[s]), 64);
            mbar_init(smem_u32(&bars->vempty[s]), 1);
            mbar_init(smem_u32(&bars->sfull[s]), 1);
            mbar_init(smem_u32(&bars->pready[s]), 4);
            mbar_init(smem_u32(&bars->pfree[s]), 1);
        }
        mbar_init(smem_u32(&bars->done), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(&bars->tmem_base), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    if (warp >= 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::OTHER_REGS));

    if (warp >= 4 && warp < 8) {
        // ------------------------------------------------ K / V gather
        // Warps 4-5: K rows (3 stages; the query rows with chunk 0), warps
        // 6-7: V rows (2 stages); the two warps of a role take alternate row
        // pairs.  The chunk's key list is loaded one chunk ahead.
        const bool isK = warp < 6;
        const int pw = (warp - 4) & 1;
        const int nst = isK ? C::KST : C::VST;
        const __nv_bfloat16* src = isK ? p.K : p.V;
        const uint32_t tile0 = sb + (isK ? C::OFF_K : C::OFF_V);
        uint64_t* full = isK ? bars->kfull : bars->vfull;
        uint64_t* empty = isK ? bars->kempty : bars->vempty;
        const int rr = lane / PR, pc = lane % PR;
        if (isK && nch > 0) {
            for (int m0 = pw * RPI; m0 < 128; m0 += 2 * RPI) {
                const int m = m0 + rr, j = m / G, h = m % G;
                const bool ok = t0 + j < p.L;
                const __nv_bfloat16* s =
                    p.Q + ((ok ? t0 + j : 0) * p.Hq + (int64_t)g * G + h) * D + pc * 8;
                cp_async16_zfill(sb + C::OFF_Q + tile_off<C::DH>(m, pc), s, ok ? 16u : 0u);
            }
        }
        int32_t k0 = nch > 0 ? keys[lane] : -1, k1 = nch > 0 ? keys[32 + lane] : -1;
        for (int c = 0; c < nch; ++c) {
            const int s = c % nst;
            const int32_t c0 = k0, c1 = k1;
            if (c + 1 < nch) {
                k0 = keys[(c + 1) * kChunk + lane];
                k1 = keys[(c + 1) * kChunk + 32 + lane];
            }
            if (c >= nst) {
                bool got = false;
                if (lane == 0)
                    got = !bars->abort_flag &&
                          mbar_wait_to(p.err, smem_u32(&empty[s]), ((c / nst) - 1) & 1);
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    if (lane == 0) bars->abort_flag = 1;
                    break;
                }
            }
            const uint32_t tile = tile0 + s * C::KV_BYTES;
#pragma unroll 4
            for (int r0 = pw * RPI; r0 < kChunk; r0 += 2 * RPI) {
                const int r = r0 + rr;
                const int32_t a = __shfl_sync(0xffffffffu, c0, r & 31);
                const int32_t b = __shfl_sync(0xffffffffu, c1, r & 31);
                const int32_t u = r0 < 32 ? a : b;
                const __nv_bfloat16* row =
                    src + ((u >= 0 ? (int64_t)u : 0) * p.Hkv + g) * D + pc * 8;
                cp_async16_zfill(tile + tile_off<C::DH>(r, pc), row, u >= 0 ? 16u : 0u);
            }
            cp_async_arrive(smem_u32(&full[s]));
        }
        cp_async_wait_all();
    } else if (warp == 8) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && nch > 0) {
            constexpr uint32_t idS = idesc_bf16(kChunk, false);
            constexpr uint32_t idO = idesc_bf16(D, true);
            auto issue_S = [&](int c) -> bool {
                const int s = c % C::KST;
                if (bars->abort_flag ||
                    !mbar_wait_to(p.err, smem_u32(&bars->kfull[s]), (c / C::KST) & 1)) {
                    bars->abort_flag = 1;
                    return false;
                }
                fence_async_smem();
                tc_fence_after();
                const uint32_t kt = sb + C::OFF_K + s * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 32;
                    umma_bf16_ss(tmem + 128 + (c & 1) * kChunk,
                                 sdesc(sb + C::OFF_Q + off, 16, C::GROUP),
                                 sdesc(kt + off, 16, C::GROUP), idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&bars->sfull[c & 1]));
                umma_commit(smem_u32(&bars->kempty[s]));
                return true;
            };
            bool ok = issue_S(0) && (nch < 2 || issue_S(1));
            for (int c = 0; ok && c < nch; ++c) {
                const int b = c & 1;
                if (bars->abort_flag ||
                    !mbar_wait_to(p.err, smem_u32(&bars->pready[b]), (c >> 1) & 1) ||
                    !mbar_wait_to(p.err, smem_u32(&bars->vfull[b]), (c >> 1) & 1)) {
                    bars->abort_flag = 1;
                    break;
                }
                fence_async_smem();
                tc_fence_after();
                // P of the chunk is the first 32 columns of its score buffer
                const uint32_t vt = sb + C::OFF_V + b * C::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                    umma_bf16_ts(tmem, tmem + 128 + b * kChunk + kk * 8,
                                 sdesc(vt + kk * 2 * C::GROUP, 1024, C::GROUP), idO,
                                 (c > 0 || kk > 0) ? 1u : 0u);
                umma_commit(smem_u32(&bars->vempty[b]));
                umma_commit(smem_u32(&bars->pfree[b]));
                // S of chunk c + 2 overwrites this score buffer, which holds P
                // of chunk c: MMAs of one thread run in issue order, so the
                // product above has read P before the scores are written
                if (c + 2 < nch) ok = issue_S(c + 2);
            }
            umma_commit(smem_u32(&bars->done));
            mbar_wait_to(p.err, smem_u32(&bars->done), 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------ softmax, row m
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
        const int m = warp * 32 + lane;
        const int j = m / G, h = m % G;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        float m_run = -INFINITY, l = 0.f;
        uint64_t mk_next = nch > 0 ? masks[j] : 0ull;
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
            const int b = c & 1;
            const uint64_t mk = mk_next;
            if (c + 1 < nch) mk_next = masks[(c + 1) * QB + j];
            const bool got = !bars->abort_flag &&
                             mbar_wait_to(p.err, smem_u32(&bars->sfull[b]), (c >> 1) & 1);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sbuf = tmem + lane_base + 128 + b * kChunk;
            float x[kChunk];
            {
                float a[32];
                tmem_ld_32x32b_x32(sbuf, a);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = a[i];
                tmem_ld_32x32b_x32(sbuf + 32, a);
#pragma unroll
                for (int i = 0; i < 32; ++i) x[32 + i] = a[i];
            }
            // scores of the keys this query selected; -inf elsewhere
            const uint32_t lo = (uint32_t)mk, hi = (uint32_t)(mk >> 32);
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
                const uint32_t w = i < 32 ? lo : hi;
                x[i] = (w & (1u << (i & 31))) ? x[i] : -INFINITY;
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < kChunk; i += 2) mx4[(i >> 1) & 3] = max3(mx4[(i >> 1) & 3], x[i], x[i + 1]);
            const float mxs = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (mxs > m_run + kRescaleLog2) {  // false while the row has no key (mxs = -inf)
                rescale = m_run != -INFINITY;  // the O row is 0 before the first key
                alpha = rescale ? attn::ex2(m_run - mxs) : 0.f;
                m_run = mxs;
            }
            const float mo = m_run == -INFINITY ? 0.f : m_run;
            const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2), nmo = f2_pack(-mo, -mo);
            uint32_t pk[kChunk / 2];
            uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int i = 0; i < kChunk; i += 2) {
                float y0, y1;
                f2_unpack(f2_fma(f2_pack(x[i], x[i + 1]), sl2, nmo), y0, y1);
                const float p0 = attn::ex2(y0), p1 = attn::ex2(y1);
                sum2[(i >> 1) & 3] = f2_add(sum2[(i >> 1) & 3], f2_pack(p0, p1));
                pk[i / 2] = attn::pack_bf16(p0, p1);
            }
            float sum4[4];
            f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), sum4[0], sum4[1]);
            sum4[2] = sum4[3] = 0.f;
            l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
            // P over the first half of the score buffer (S is in registers)
            tmem_st_32x32b_x32_u(sbuf, pk);
            if (__any_sync(0xffffffffu, rescale)) {
                // O holds exactly the chunks before c once their product is done
                const bool f = !bars->abort_flag &&
                               mbar_wait_to(p.err, smem_u32(&bars->pfree[(c - 1) & 1]),
                                            ((c - 1) >> 1) & 1);
                if (!__all_sync(0xffffffffu, f)) { ok = false; break; }
                tc_fence_after();
                const float f2 = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int cb = 0; cb < D; cb += 16) {
                    float o[16];
                    tmem_ld_32x32b_x16(tmem + lane_base + cb, o);
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] *= f2;
                    tmem_st_32x32b_x16(tmem + lane_base + cb, o);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars->pready[b]));
        }
        if (ok) {
            const int64_t t = t0 + j;
            if (nch > 0) {
                const bool f = !bars->abort_flag &&
                               mbar_wait_to(p.err, smem_u32(&bars->done), 0);
                ok = __all_sync(0xffffffffu, f);
                tc_fence_after();
            }
            if (ok) {  // every lane takes part in the loads; rows past the end store nothing
                const bool valid = t < p.L;
                const float inv = l > 0.f ? 1.f / l : 0.f;
                __nv_bfloat16* out = p.O + ((valid ? t : 0) * p.Hq + (int64_t)g * G + h) * D;
#pragma unroll
                for (int cb = 0; cb < D; cb += 32) {
                    float o[32];
                    if (nch > 0) {
                        tmem_ld_32x32b_x32(tmem + lane_base + cb, o);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = 0.f;
                    }
                    if (valid) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 v;
                            v.x = attn::pack_bf16(o[i] * inv, o[i + 1] * inv);
                            v.y = attn::pack_bf16(o[i + 2] * inv, o[i + 3] * inv);
                            v.z = attn::pack_bf16(o[i + 4] * inv, o[i + 5] * inv);
                            v.w = attn::pack_bf16(o[i + 6] * inv, o[i + 7] * inv);
                            *reinterpret_cast<uint4*>(out + cb + i) = v;
                        }
                    }
                }
            }
        }
        if (!ok && lane == 0) bars->abort_flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace dedup
}  // namespace dsa

// C ABI of the DSA hot path (declarations and contracts in include/dsa.h).
// Host side only: argument validation, TMA descriptor encoding, launches.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <utility>
#include <vector>

#include "dsa.h"
#include "decode.cuh"
#include "sparse_attn_dedup.cuh"
#include "index_topk.cuh"
#include "sparse_attn.cuh"
#include "sparse_attn_bwd.cuh"
#include "indexer_kl.cuh"
#include "indexer_kl_tc.cuh"

namespace {

thread_local char g_last_error[512] = "";

dsa_status_t fail(dsa_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

dsa_status_t ok() {
    g_last_error[0] = '\0';
    return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The caller's device error word: NULL (the per-device word) or 4-byte aligned.
#define CHECK_ERR_WORD(p)                                                              \
    do {                                                                              \
        if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)                                \
            return fail(DSA_ERR_INVALID_ARG, "%s: err is not 4-byte aligned", fn);      \
    } while (0)

#define CHECK_PTR(p)                                                                  \
    do {                                                                              \
        if ((p) == nullptr) return fail(DSA_ERR_INVALID_ARG, "%s: " #p " is NULL", fn); \
        if (!aligned16(p))                                                            \
            return fail(DSA_ERR_INVALID_ARG, "%s: " #p " is not 16-byte aligned", fn); \
    } while (0)

#define CUDA_TRY(call)                                                                     \
    do {                                                                                   \
        cudaError_t e_ = (call);                                                           \
        if (e_ != cudaSuccess)                                                             \
            return fail(DSA_ERR_CUDA, "%s: %s failed: %s", fn, #call, cudaGetErrorString(e_)); \
    } while (0)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D byte tensor [rows][row_bytes] with box [box_rows][row_bytes], swizzled
// to match the UMMA K-major layout for 64- or 128-byte rows.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
              uint32_t box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)row_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw =
        row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int max_optin_smem() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    return v;
}

int num_sms() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return v;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------ indexer

template <int HI, int DI, bool TOPK>
dsa_status_t launch_index(const char* fn, const void* q_I, const void* k_I, const float* w,
                          int64_t L, int k, int32_t* idx, float* scores, const int32_t* cu_seqlens,
                          int nseq, int64_t row0, int64_t row1, int* err, cudaStream_t st,
                          int64_t qrow0) {
    // q_I / w / idx hold rows [qrow0, L) (qrow0 = 0: the whole sequence)
    CUtensorMap mq, mk;
    if (!make_map(&mq, q_I, DI, (uint64_t)(L - qrow0) * HI, dsa::idx::kTokens * HI) ||
        !make_map(&mk, k_I, DI, (uint64_t)L, dsa::idx::kKeyTile))
        return fail(DSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed", fn);
    const dsa::idx::Layout lay(HI, DI, k, TOPK);
    const int smem = lay.total + 1024;
    if (smem > max_optin_smem())
        return fail(DSA_ERR_UNSUPPORTED, "%s: needs %d bytes of shared memory", fn, smem);
    auto kern = dsa::idx::index_kernel<HI, DI, TOPK>;
    // The kernel re-splits its registers between warpgroups (setmaxnreg);
    // the split adds up only if every thread starts with exactly 96.
    cudaFuncAttributes fa;
    CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
    if (fa.numRegs != 96)
        return fail(DSA_ERR_UNSUPPORTED, "%s: kernel built with %d registers per thread, not 96",
                    fn, fa.numRegs);
    CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    dsa::idx::Params p;
    p.w = w;
    p.L = L;
    p.k = k;
    p.idx = idx;
    p.scores = scores;
    // rows [row0, row1), row0 a multiple of kTokens
    p.blk0 = (int)(row0 / dsa::idx::kTokens);
    p.nblocks = (int)((row1 + dsa::idx::kTokens - 1) / dsa::idx::kTokens) - p.blk0;
    p.cu_seqlens = cu_seqlens;
    p.nseq = nseq;
    p.err = err;
    p.qrow0 = qrow0;
    kern<<<p.nblocks, dsa::idx::kThreads, smem, st>>>(mq, mk, p);
    CUDA_TRY(cudaGetLastError());
    return ok();
}

template <bool TOPK>
dsa_status_t dispatch_index(const char* fn, const void* q_I, const void* k_I, const float* w,
                            int64_t L, int H_I, int d_I, int k, int32_t* idx, float* scores,
                            const int32_t* cu, int nseq, int* err, cudaStream_t st,
                            int64_t row0 = 0, int64_t row1 = -1, int64_t qrow0 = 0) {
    if (row1 < 0) row1 = L;
    if (H_I == 64 && d_I == 128)
        return launch_index<64, 128, TOPK>(fn, q_I, k_I, w, L, k, idx, scores, cu, nseq, row0, row1, err, st, qrow0);
    if (H_I == 64 && d_I == 64)
        return launch_index<64, 64, TOPK>(fn, q_I, k_I, w, L, k, idx, scores, cu, nseq, row0, row1, err, st, qrow0);
    if (H_I == 4 && d_I == 128)
        return launch_index<4, 128, TOPK>(fn, q_I, k_I, w, L, k, idx, scores, cu, nseq, row0, row1, err, st, qrow0);
    if (H_I == 4 && d_I == 64)
        return launch_index<4, 64, TOPK>(fn, q_I, k_I, w, L, k, idx, scores, cu, nseq, row0, row1, err, st, qrow0);
    return fail(DSA_ERR_UNSUPPORTED, "%s: (H_I, d_I) = (%d, %d) not in {4, 64} x {64, 128}", fn,
                H_I, d_I);
}

// ------------------------------------------------------------ attention

// Launches `kern` so that it may start while the previous kernel on the
// stream finishes (it calls pdl_wait() before touching that kernel's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int D, int HKV, int G, bool SPLIT, int NP = 1>
dsa_status_t launch_attn(const char* fn, const dsa::attn::Params& p, int64_t grid,
                         cudaStream_t st) {
    using C = dsa::attn::Cfg<D, HKV, NP>;
    auto kern = dsa::attn::attn_kernel<D, HKV, G, SPLIT, NP>;
    CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    if (SPLIT) {  // decode: chained behind the merge kernel
        CUDA_TRY(launch_chained(kern, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, st, p));
    } else {
        kern<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(p);
    }
    CUDA_TRY(cudaGetLastError());
    return DSA_OK;
}

// Workspace layout of the dedup attention (one wave of blocks).
template <int G>
dsa::dedup::Layout dedup_layout(int64_t L, int k) {
    constexpr int QB = 128 / G;
    const int64_t nblk = (L + QB - 1) / QB;
    return dsa::dedup::Layout{nblk < dsa::dedup::kWave ? nblk : dsa::dedup::kWave,
                              dsa::dedup::block_cap(L, QB, k), QB};
}

// The dedup attention's wave loop: per wave of blocks, the plan kernel and
// then the tensor-core kernel (one CTA per KV group and block).
template <int D, int G>
dsa_status_t launch_dedup(const char* fn, dsa::dedup::TcParams tp, const int32_t* idx, int k,
                          void* workspace, cudaStream_t st) {
    namespace dd = dsa::dedup;
    using C = dd::TcCfg<D, G>;
    constexpr int QB = C::QB;
    const int64_t L = tp.L;
    const int64_t nblk = (L + QB - 1) / QB;
    const dd::Layout lay = dedup_layout<G>(L, k);
    const int plan_smem = dd::plan_smem_bytes(L, lay.cap, QB);
    if (plan_smem > max_optin_smem() || C::SMEM_LAUNCH > max_optin_smem())
        return fail(DSA_ERR_UNSUPPORTED, "%s: needs %d bytes of shared memory", fn,
                    plan_smem > C::SMEM_LAUNCH ? plan_smem : C::SMEM_LAUNCH);
    auto plan = dd::plan_kernel<QB>;
    auto tc = dd::tc_kernel<D, G>;
    // the tensor-core kernel re-splits its registers (setmaxnreg); the split
    // adds up only with exactly C::LAUNCH_REGS per thread at launch
    cudaFuncAttributes fa;
    CUDA_TRY(cudaFuncGetAttributes(&fa, tc));
    if (fa.numRegs != C::LAUNCH_REGS)
        return fail(DSA_ERR_UNSUPPORTED, "%s: kernel built with %d registers per thread, not %d", fn,
                    fa.numRegs, C::LAUNCH_REGS);
    CUDA_TRY(cudaFuncSetAttribute(plan, cudaFuncAttributeMaxDynamicSharedMemorySize, plan_smem));
    CUDA_TRY(cudaFuncSetAttribute(tc, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_LAUNCH));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    dd::PlanParams pp{};
    pp.idx = idx;
    pp.L = L;
    pp.k = k;
    pp.cap = lay.cap;
    pp.nU = reinterpret_cast<int32_t*>(ws + lay.n_off());
    pp.keys = reinterpret_cast<int32_t*>(ws + lay.keys_off());
    pp.masks = reinterpret_cast<uint64_t*>(ws + lay.masks_off());
    pp.err = tp.err;
    tp.nU = pp.nU;
    tp.keys = pp.keys;
    tp.masks = pp.masks;
    tp.cap = lay.cap;
    for (int64_t b0 = 0; b0 < nblk; b0 += lay.nslot) {
        const int64_t nb = nblk - b0 < lay.nslot ? nblk - b0 : lay.nslot;
        pp.blk0 = b0;
        tp.blk0 = b0;
        plan<<<(unsigned)nb, dd::kPlanThreads, plan_smem, st>>>(pp);
        CUDA_TRY(cudaGetLastError());
        tc<<<dim3((unsigned)tp.Hkv, (unsigned)nb), C::THREADS, C::SMEM_LAUNCH, st>>>(tp);
        CUDA_TRY(cudaGetLastError());
    }
    return DSA_OK;
}

// Dedup workspace bytes, or 0 for an unsupported shape.
size_t dedup_workspace_bytes(int64_t L, int Hq, int Hkv, int d, int k) {
    if (L < 1 || k < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv) return 0;
    const int G = Hq / Hkv;
    if (d != 64 && d != 128) return 0;
    if (G == 8) return (size_t)dedup_layout<8>(L, k).bytes();
    if (G == 4) return (size_t)dedup_layout<4>(L, k).bytes();
    return 0;
}

// Attention for query rows [row0, row1) over keys [0, L) (arguments
// checked by the caller).
dsa_status_t attn_prefill_rows(const char* fn, const void* Q, const void* K, const void* V,
                               const int32_t* idx, int64_t L, int Hq, int Hkv, int d, int k,
                               float scale, void* O, float* lse, int64_t row0, int64_t row1,
                               int* err, cudaStream_t st) {
    const int G = Hq / Hkv;
    dsa::attn::Params p{};
    p.Q = static_cast<const __nv_bfloat16*>(Q) + row0 * Hq * d;
    p.K = static_cast<const __nv_bfloat16*>(K);
    p.V = static_cast<const __nv_bfloat16*>(V);
    p.idx = idx + row0 * k;
    p.nkeys = L;
    p.k = k;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.O = static_cast<__nv_bfloat16*>(O) + row0 * Hq * d;
    p.lse = lse != nullptr ? lse + row0 * Hq : nullptr;
    p.err = err;
    const int64_t rows = row1 - row0;
    // Two producer warps per CTA (two CTAs per SM instead of three) are faster
    // while the K and V rows stay in L2 (7 % at 32K keys), one when the rows
    // come from HBM (2 % at 128K); the line is 96 MB of K + V.
    const bool l2 = L * Hkv * d * 4 <= (int64_t(96) << 20);
    if (d == 128 && Hkv == 4 && G == 8)
        return l2 ? launch_attn<128, 4, 8, false, 2>(fn, p, rows, st)
                  : launch_attn<128, 4, 8, false>(fn, p, rows, st);
    if (d == 64 && Hkv == 2 && G == 4)
        return l2 ? launch_attn<64, 2, 4, false, 2>(fn, p, rows, st)
                  : launch_attn<64, 2, 4, false>(fn, p, rows, st);
    if (d == 128 && Hkv == 2 && G == 4)
        return l2 ? launch_attn<128, 2, 4, false, 2>(fn, p, rows, st)
                  : launch_attn<128, 2, 4, false>(fn, p, rows, st);
    if (d == 64 && Hkv == 4 && G == 8)
        return l2 ? launch_attn<64, 4, 8, false, 2>(fn, p, rows, st)
                  : launch_attn<64, 4, 8, false>(fn, p, rows, st);
    return fail(DSA_ERR_UNSUPPORTED, "%s: (d, Hkv, Hq/Hkv) = (%d, %d, %d)", fn, d, Hkv, G);
}

}  // namespace

extern "C" {

int dsa_version(void) { return 100; }

const char* dsa_status_string(int status) {
    switch (status) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
        case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
        case DSA_ERR_DEVICE: return "DSA_ERR_DEVICE";
        default: return "DSA_ERR_UNKNOWN";
    }
}

const char* dsa_last_error(void) { return g_last_error; }

dsa_status_t dsa_index_topk(const void* q_I, const void* k_I, const float* w, int64_t L,
                            int H_I, int d_I, int k, int32_t* idx, int32_t* err,
                            dsa_stream_t stream) {
    static const char fn[] = "dsa_index_topk";
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(idx);
    CHECK_ERR_WORD(err);
    if (L < 1 || L > (int64_t(1) << 30)) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (k > 2048) return fail(DSA_ERR_UNSUPPORTED, "%s: k = %d > 2048", fn, k);
    if (L * H_I >= (int64_t(1) << 31))
        return fail(DSA_ERR_UNSUPPORTED, "%s: L * H_I too large", fn);
    return dispatch_index<true>(fn, q_I, k_I, w, L, H_I, d_I, k, idx, nullptr, nullptr, 1, err,
                                static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_index_topk_varlen(const void* q_I, const void* k_I, const float* w,
                                   const int32_t* cu_seqlens, int nseq, int64_t L, int H_I,
                                   int d_I, int k, int32_t* idx, int32_t* err,
                                   dsa_stream_t stream) {
    static const char fn[] = "dsa_index_topk_varlen";
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(idx);
    CHECK_ERR_WORD(err);
    if (cu_seqlens == nullptr) return fail(DSA_ERR_INVALID_ARG, "%s: cu_seqlens is null", fn);
    if (nseq < 1) return fail(DSA_ERR_INVALID_ARG, "%s: nseq = %d", fn, nseq);
    if (L < 1 || L > (int64_t(1) << 30)) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (k > 2048) return fail(DSA_ERR_UNSUPPORTED, "%s: k = %d > 2048", fn, k);
    if (L * H_I >= (int64_t(1) << 31))
        return fail(DSA_ERR_UNSUPPORTED, "%s: L * H_I too large", fn);
    return dispatch_index<true>(fn, q_I, k_I, w, L, H_I, d_I, k, idx, nullptr, cu_seqlens, nseq,
                                err, static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_index_topk_rows(const void* q_I, const void* k_I, const float* w, int64_t row0,
                                 int64_t row1, int H_I, int d_I, int k, int32_t* idx,
                                 int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_index_topk_rows";
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(idx);
    CHECK_ERR_WORD(err);
    if (row0 < 0 || row1 <= row0 || row1 > (int64_t(1) << 30))
        return fail(DSA_ERR_INVALID_ARG, "%s: rows [%lld, %lld)", fn, (long long)row0,
                    (long long)row1);
    if (row0 % dsa::idx::kTokens != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: row0 = %lld is not a multiple of %d", fn,
                    (long long)row0, dsa::idx::kTokens);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (k > 2048) return fail(DSA_ERR_UNSUPPORTED, "%s: k = %d > 2048", fn, k);
    if (row1 * H_I >= (int64_t(1) << 31))
        return fail(DSA_ERR_UNSUPPORTED, "%s: row1 * H_I too large", fn);
    return dispatch_index<true>(fn, q_I, k_I, w, row1, H_I, d_I, k, idx, nullptr, nullptr, 1, err,
                                static_cast<cudaStream_t>(stream), row0, row1, row0);
}

dsa_status_t dsa_sparse_attn_rows(const void* Q, const void* K, const void* V,
                                  const int32_t* idx, int64_t nrows, int64_t nkeys, int Hq,
                                  int Hkv, int d, int k, float scale, void* O, float* lse,
                                  int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_rows";
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(idx);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (nrows < 1 || nrows > (int64_t(1) << 30) || nkeys < 1 || nkeys > (int64_t(1) << 31) - 1)
        return fail(DSA_ERR_INVALID_ARG, "%s: nrows = %lld, nkeys = %lld", fn, (long long)nrows,
                    (long long)nkeys);
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (Hkv < 1 || Hq < 1 || Hq % Hkv) return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d", fn, Hq, Hkv);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: lse is not 4-byte aligned", fn);
    const dsa_status_t r = attn_prefill_rows(fn, Q, K, V, idx, nkeys, Hq, Hkv, d, k, scale, O,
                                             lse, 0, nrows, err,
                                             static_cast<cudaStream_t>(stream));
    return r == DSA_OK ? ok() : r;
}

size_t dsa_sparse_attn_prefill_dedup_workspace_size(int64_t L, int Hq, int Hkv, int d, int k) {
    return dedup_workspace_bytes(L, Hq, Hkv, d, k);
}

dsa_status_t dsa_sparse_attn_prefill_dedup(const void* Q, const void* K, const void* V,
                                           const int32_t* idx, int64_t L, int Hq, int Hkv, int d,
                                           int k, float scale, void* O, void* workspace,
                                           size_t workspace_bytes, int32_t* err,
                                           dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_prefill_dedup";
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(idx);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (L < 1) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (L > dsa::dedup::kMaxKeys)
        return fail(DSA_ERR_UNSUPPORTED, "%s: L = %lld > %d", fn, (long long)L, dsa::dedup::kMaxKeys);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (Hkv < 1 || Hq < 1 || Hq % Hkv) return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d", fn, Hq, Hkv);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    const int G = Hq / Hkv;
    if ((d != 64 && d != 128) || (G != 4 && G != 8))
        return fail(DSA_ERR_UNSUPPORTED, "%s: (d, Hq/Hkv) = (%d, %d)", fn, d, G);
    const int64_t cap = dsa::dedup::block_cap(L, 128 / G, k);
    if (cap > dsa::dedup::kMaxCap)
        return fail(DSA_ERR_UNSUPPORTED, "%s: %d x k = %lld distinct keys per block > %d", fn,
                    128 / G, (long long)cap, dsa::dedup::kMaxCap);
    CHECK_PTR(workspace);
    if (workspace_bytes < dedup_workspace_bytes(L, Hq, Hkv, d, k))
        return fail(DSA_ERR_WORKSPACE, "%s: workspace_bytes = %zu < %zu", fn, workspace_bytes,
                    dedup_workspace_bytes(L, Hq, Hkv, d, k));
    dsa::dedup::TcParams tp{};
    tp.Q = static_cast<const __nv_bfloat16*>(Q);
    tp.K = static_cast<const __nv_bfloat16*>(K);
    tp.V = static_cast<const __nv_bfloat16*>(V);
    tp.O = static_cast<__nv_bfloat16*>(O);
    tp.L = L;
    tp.Hq = Hq;
    tp.Hkv = Hkv;
    tp.scale_log2 = scale * 1.4426950408889634f;
    tp.err = err;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dsa_status_t r;
    if (d == 128 && G == 8) r = launch_dedup<128, 8>(fn, tp, idx, k, workspace, st);
    else if (d == 64 && G == 4) r = launch_dedup<64, 4>(fn, tp, idx, k, workspace, st);
    else if (d == 128 && G == 4) r = launch_dedup<128, 4>(fn, tp, idx, k, workspace, st);
    else r = launch_dedup<64, 8>(fn, tp, idx, k, workspace, st);
    return r == DSA_OK ? ok() : r;
}

dsa_status_t dsa_prefill_from_host(const void* q_I_h, const void* k_I_h, const float* w_h,
                                   const void* Q_h, const void* K_h, const void* V_h, void* O_h,
                                   void* q_I, void* k_I, float* w, void* Q, void* K, void* V,
                                   int32_t* idx, void* O, int64_t L, int H_I, int d_I, int Hq,
                                   int Hkv, int d, int k, float scale, int64_t chunk_rows,
                                   int32_t* err, dsa_stream_t stream, dsa_stream_t h2d_stream,
                                   dsa_stream_t d2h_stream) {
    static const char fn[] = "dsa_prefill_from_host";
    CHECK_PTR(q_I_h);
    CHECK_PTR(k_I_h);
    CHECK_PTR(w_h);
    CHECK_PTR(Q_h);
    CHECK_PTR(K_h);
    CHECK_PTR(V_h);
    CHECK_PTR(O_h);
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(idx);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (L < 1 || L > (int64_t(1) << 30)) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (k > 2048) return fail(DSA_ERR_UNSUPPORTED, "%s: k = %d > 2048", fn, k);
    if (L * H_I >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED, "%s: L * H_I too large", fn);
    if (Hkv < 1 || Hq < 1 || Hq % Hkv) return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d", fn, Hq, Hkv);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    if (chunk_rows < 1) return fail(DSA_ERR_INVALID_ARG, "%s: chunk_rows = %lld", fn, (long long)chunk_rows);
    const int64_t C = (chunk_rows + 127) / 128 * 128;  // whole 4-row blocks and key tiles
    const int nch = (int)((L + C - 1) / C);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t sh = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t sd = static_cast<cudaStream_t>(d2h_stream);
    // per chunk: inputs on the device, outputs ready; then all copies back
    std::vector<cudaEvent_t> ev(2 * nch + 2, nullptr);
    for (auto& e : ev) CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    struct Destroy {
        std::vector<cudaEvent_t>& v;
        ~Destroy() {
            for (auto e : v)
                if (e) cudaEventDestroy(e);  // released once pending work reaches them
        }
    } destroy{ev};
    auto hb = [](const void* p) { return static_cast<const uint8_t*>(p); };
    auto db = [](void* p) { return static_cast<uint8_t*>(p); };
    // the device buffers may still be in use by earlier work on `stream`:
    // neither copy stream starts before it
    CUDA_TRY(cudaEventRecord(ev[2 * nch + 1], st));
    CUDA_TRY(cudaStreamWaitEvent(sh, ev[2 * nch + 1], 0));
    CUDA_TRY(cudaStreamWaitEvent(sd, ev[2 * nch + 1], 0));
    const int64_t rq = (int64_t)H_I * d_I, rk = d_I, rw = (int64_t)H_I * 4,
                  rQ = (int64_t)Hq * d * 2, rK = (int64_t)Hkv * d * 2;
    for (int c = 0; c < nch; ++c) {
        const int64_t r0 = c * C, r1 = r0 + C < L ? r0 + C : L, n = r1 - r0;
        // the chunk's new rows: queries, weights, and the keys/values they add
        CUDA_TRY(cudaMemcpyAsync(db(q_I) + r0 * rq, hb(q_I_h) + r0 * rq, n * rq, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaMemcpyAsync(db(k_I) + r0 * rk, hb(k_I_h) + r0 * rk, n * rk, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaMemcpyAsync(db(w) + r0 * rw, hb(w_h) + r0 * rw, n * rw, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaMemcpyAsync(db(Q) + r0 * rQ, hb(Q_h) + r0 * rQ, n * rQ, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaMemcpyAsync(db(K) + r0 * rK, hb(K_h) + r0 * rK, n * rK, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaMemcpyAsync(db(V) + r0 * rK, hb(V_h) + r0 * rK, n * rK, cudaMemcpyHostToDevice, sh));
        CUDA_TRY(cudaEventRecord(ev[2 * c], sh));
        // rows [r0, r1) need keys [0, r1): all of them are on the device now
        CUDA_TRY(cudaStreamWaitEvent(st, ev[2 * c], 0));
        dsa_status_t r = dispatch_index<true>(fn, q_I, k_I, w, L, H_I, d_I, k, idx, nullptr, nullptr,
                                              1, err, st, r0, r1);
        if (r != DSA_OK) return r;
        r = attn_prefill_rows(fn, Q, K, V, idx, L, Hq, Hkv, d, k, scale, O, nullptr, r0, r1, err,
                              st);
        if (r != DSA_OK) return r;
        CUDA_TRY(cudaEventRecord(ev[2 * c + 1], st));
        CUDA_TRY(cudaStreamWaitEvent(sd, ev[2 * c + 1], 0));
        CUDA_TRY(cudaMemcpyAsync(db(O_h) + r0 * rQ, static_cast<const uint8_t*>(O) + r0 * rQ, n * rQ,
                                 cudaMemcpyDeviceToHost, sd));
    }
    CUDA_TRY(cudaEventRecord(ev[2 * nch], sd));
    CUDA_TRY(cudaStreamWaitEvent(st, ev[2 * nch], 0));  // `stream` ends when O_h is filled
    return ok();
}

dsa_status_t dsa_index_scores(const void* q_I, const void* k_I, const float* w, int64_t L,
                              int H_I, int d_I, float* scores, int32_t* err,
                              dsa_stream_t stream) {
    static const char fn[] = "dsa_index_scores";
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(scores);
    CHECK_ERR_WORD(err);
    if (L < 1 || L * L >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld (L * L must be < 2^31)", fn, (long long)L);
    return dispatch_index<false>(fn, q_I, k_I, w, L, H_I, d_I, 1, nullptr, scores, nullptr, 1, err,
                                 static_cast<cudaStream_t>(stream));
}

dsa_status_t dsa_sparse_attn_prefill(const void* Q, const void* K, const void* V,
                                     const int32_t* idx, int64_t L, int Hq, int Hkv, int d,
                                     int k, float scale, void* O, float* lse, int32_t* err,
                                     dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_prefill";
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(idx);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (L < 1 || L > (int64_t(1) << 30)) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (Hkv < 1 || Hq < 1 || Hq % Hkv) return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d", fn, Hq, Hkv);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: lse is not 4-byte aligned", fn);
    const dsa_status_t r = attn_prefill_rows(fn, Q, K, V, idx, L, Hq, Hkv, d, k, scale, O, lse, 0,
                                             L, err, static_cast<cudaStream_t>(stream));
    return r == DSA_OK ? ok() : r;
}

}  // extern "C"

namespace {

template <int D, int HKV, int G>
dsa_status_t launch_attn_bwd(const char* fn, const dsa::attn::BwdParams& p, int64_t L,
                             cudaStream_t st) {
    using C = dsa::attn::Cfg<D, HKV>;
    auto kern = dsa::attn::attn_bwd_kernel<D, HKV, G>;
    CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    kern<<<(unsigned)L, C::THREADS, C::SMEM, st>>>(p);
    CUDA_TRY(cudaGetLastError());
    return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_sparse_attn_backward(const void* Q, const void* K, const void* V,
                                      const int32_t* idx, const void* O, const float* lse,
                                      const void* dO, int64_t L, int Hq, int Hkv, int d, int k,
                                      float scale, float* dQ, float* dK, float* dV, int32_t* err,
                                      dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_backward";
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(V);
    CHECK_PTR(idx);
    CHECK_PTR(O);
    CHECK_PTR(lse);
    CHECK_PTR(dO);
    CHECK_PTR(dQ);
    CHECK_PTR(dK);
    CHECK_PTR(dV);
    CHECK_ERR_WORD(err);
    if (L < 1 || L > (int64_t(1) << 30)) return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld", fn, (long long)L);
    if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (Hkv < 1 || Hq < 1 || Hq % Hkv) return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d", fn, Hq, Hkv);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    const int G = Hq / Hkv;
    const bool shape_ok = (d == 128 && Hkv == 4 && G == 8) || (d == 64 && Hkv == 2 && G == 4) ||
                          (d == 128 && Hkv == 2 && G == 4) || (d == 64 && Hkv == 4 && G == 8);
    if (!shape_ok)
        return fail(DSA_ERR_UNSUPPORTED, "%s: (d, Hkv, Hq/Hkv) = (%d, %d, %d)", fn, d, Hkv, G);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // dK and dV are sums of reductions from every row that selects the key
    const size_t kv_bytes = (size_t)L * Hkv * d * sizeof(float);
    CUDA_TRY(cudaMemsetAsync(dK, 0, kv_bytes, st));
    CUDA_TRY(cudaMemsetAsync(dV, 0, kv_bytes, st));
    dsa::attn::BwdParams p{};
    p.Q = static_cast<const __nv_bfloat16*>(Q);
    p.K = static_cast<const __nv_bfloat16*>(K);
    p.V = static_cast<const __nv_bfloat16*>(V);
    p.O = static_cast<const __nv_bfloat16*>(O);
    p.dO = static_cast<const __nv_bfloat16*>(dO);
    p.lse = lse;
    p.idx = idx;
    p.nkeys = L;
    p.k = k;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.dQ = dQ;
    p.dK = dK;
    p.dV = dV;
    p.err = err;
    dsa_status_t r;
    if (d == 128 && Hkv == 4 && G == 8) r = launch_attn_bwd<128, 4, 8>(fn, p, L, st);
    else if (d == 64 && Hkv == 2 && G == 4) r = launch_attn_bwd<64, 2, 4>(fn, p, L, st);
    else if (d == 128 && Hkv == 2 && G == 4) r = launch_attn_bwd<128, 2, 4>(fn, p, L, st);
    else r = launch_attn_bwd<64, 4, 8>(fn, p, L, st);
    return r == DSA_OK ? ok() : r;
}

// ------------------------------------------------------------ decode

namespace {
constexpr int64_t kMinRange = 4096;  // cache rows per CTA at least

struct DecodePlan {
    int64_t R;          // cache rows per CTA of the indexer scan
    int ctas, max_slots, nsplit;
    size_t off_sc, off_ix, off_cnt, off_th, off_idx, off_po, off_pml, total;
};

DecodePlan plan_decode(int B, int64_t total_n, int k, int Hq, int d, int sms) {
    DecodePlan pl;
    // one wave: at most one CTA per SM, each scanning an equal row range
    int64_t ctas = (total_n + kMinRange - 1) / kMinRange;
    if (ctas > sms) ctas = sms;
    if (ctas < 1) ctas = 1;
    pl.R = (total_n + ctas - 1) / ctas;
    pl.ctas = (int)((total_n + pl.R - 1) / pl.R);
    pl.max_slots = pl.ctas + B;  // slot = chunk + sequence of an overlapping pair
    // split the index rows so that B * nsplit attention CTAs fill one wave
    // (two resident CTAs per SM)
    int ns = (2 * sms) / B;
    if (ns < 1) ns = 1;
    if (ns > 16) ns = 16;
    pl.nsplit = ns;
    size_t o = 0;
    const size_t sc = (size_t)dsa::dec::slot_capacity(k);
    pl.off_sc = o;  o = align256(o + (size_t)pl.max_slots * sc * 4);
    pl.off_ix = o;  o = align256(o + (size_t)pl.max_slots * sc * 4);
    pl.off_cnt = o; o = align256(o + (size_t)pl.max_slots * 4);
    pl.off_th = o;  o = align256(o + (size_t)pl.max_slots * 4);
    pl.off_idx = o; o = align256(o + (size_t)B * k * 4);
    pl.off_po = o;  o = align256(o + (size_t)B * ns * Hq * d * 4);
    pl.off_pml = o; o = align256(o + (size_t)B * ns * Hq * 2 * 4);
    pl.total = o;
    return pl;
}
}  // namespace

size_t dsa_decode_workspace_size(int B, int64_t total_n, int H_I, int d_I, int k, int Hq,
                                 int Hkv, int d) {
    (void)H_I;
    (void)d_I;
    (void)Hkv;
    if (B < 1 || total_n < 1 || k < 1) return 0;
    return plan_decode(B, total_n, k, Hq, d, num_sms()).total;
}

}  // extern "C"

namespace {

// Argument checks of the decode calls (with and without a caller workspace):
// everything but the workspace itself.
dsa_status_t check_decode_args(const char* fn, const void* q_I, const float* w, const void* Q,
                               const void* kI_cache, const void* K_cache, const void* V_cache,
                               const int64_t* cache_off, int B, int64_t total_n, int H_I,
                               int d_I, int Hq, int Hkv, int d, int k, float scale, void* O,
                               int32_t* idx_out, int32_t* err) {
    CHECK_PTR(q_I);
    CHECK_PTR(w);
    CHECK_PTR(Q);
    CHECK_PTR(kI_cache);
    CHECK_PTR(K_cache);
    CHECK_PTR(V_cache);
    CHECK_PTR(cache_off);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (idx_out && !aligned16(idx_out))
        return fail(DSA_ERR_INVALID_ARG, "%s: idx_out is not 16-byte aligned", fn);
    if (B < 1 || B > 4096) return fail(DSA_ERR_INVALID_ARG, "%s: B = %d", fn, B);
    if (total_n < B || total_n >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: total_n = %lld", fn, (long long)total_n);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    if (H_I != 64 || d_I != 128 || d != 128 || Hkv != 4 || Hq != 32 || k > 2048)
        return fail(DSA_ERR_UNSUPPORTED,
                    "%s: supported H_I=64, d_I=128, d=128, Hkv=4, Hq=32, k<=2048", fn);
    return DSA_OK;
}

// Decode phase 1: the indexer scan over the packed cache and the per-sequence
// merge into index rows (with ordered scores and global keys for a shard).
dsa_status_t launch_decode_select(const char* fn, const DecodePlan& pl, uint8_t* ws,
                                  const void* q_I, const float* w, const void* kI_cache,
                                  const int64_t* cache_off, int B, int64_t total_n, int k,
                                  int32_t* idx, uint32_t* ord_out, const int64_t* key_base,
                                  bool shard, int32_t* err, cudaStream_t st) {
    dsa::dec::Params dp{};
    dp.w = w;
    dp.cache_off = cache_off;
    dp.B = B;
    dp.total_n = total_n;
    dp.k = k;
    dp.R = pl.R;
    dp.cand_so = reinterpret_cast<uint32_t*>(ws + pl.off_sc);
    dp.cand_ix = reinterpret_cast<int32_t*>(ws + pl.off_ix);
    dp.cand_cnt = reinterpret_cast<int*>(ws + pl.off_cnt);
    dp.cand_th = reinterpret_cast<uint32_t*>(ws + pl.off_th);
    dp.err = err;
    dp.ord_out = ord_out;
    dp.key_base = key_base;
    dp.allow_empty = shard ? 1 : 0;

    CUtensorMap mq, mk;
    if (!make_map(&mq, q_I, 128, (uint64_t)B * 64, 64) ||
        !make_map(&mk, kI_cache, 128, (uint64_t)total_n, dsa::idx::kKeyTile))
        return fail(DSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed", fn);
    const int smem_idx = dsa::dec::Layout(k).total + 1024;
    if (smem_idx > max_optin_smem())
        return fail(DSA_ERR_UNSUPPORTED, "%s: needs %d bytes of shared memory", fn, smem_idx);

    // The scan re-splits its registers between warpgroups (setmaxnreg); the
    // split adds up only if every thread starts with exactly 96.
    cudaFuncAttributes fa;
    CUDA_TRY(cudaFuncGetAttributes(&fa, dsa::dec::index_kernel));
    if (fa.numRegs != 96)
        return fail(DSA_ERR_UNSUPPORTED, "%s: scan kernel built with %d registers per thread, not 96",
                    fn, fa.numRegs);
    CUDA_TRY(cudaFuncSetAttribute(dsa::dec::index_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem_idx));
    CUDA_TRY(launch_chained(dsa::dec::index_kernel, dim3(pl.ctas), dim3(dsa::dec::kThreads),
                            smem_idx, st, mq, mk, dp));
    CUDA_TRY(cudaGetLastError());

    const int merge_smem_cap = 24576;  // entries staged in shared memory (192 KB)
    const int smem_merge = merge_smem_cap * 8;
    CUDA_TRY(cudaFuncSetAttribute(dsa::dec::merge_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem_merge));
    CUDA_TRY(launch_chained(dsa::dec::merge_kernel, dim3(B), dim3(1024), smem_merge, st, dp, idx,
                            merge_smem_cap));
    CUDA_TRY(cudaGetLastError());
    return DSA_OK;
}

// Decode phase 2: attention split into nsplit slices of each index row
// (partials in the workspace).
dsa_status_t launch_decode_attn(const char* fn, const DecodePlan& pl, uint8_t* ws, const void* Q,
                                const void* K_cache, const void* V_cache,
                                const int64_t* cache_off, int B, int k, float scale,
                                const int32_t* idx, const int64_t* key_base, int32_t* err,
                                cudaStream_t st) {
    dsa::attn::Params ap{};
    ap.Q = static_cast<const __nv_bfloat16*>(Q);
    ap.K = static_cast<const __nv_bfloat16*>(K_cache);
    ap.V = static_cast<const __nv_bfloat16*>(V_cache);
    ap.idx = idx;
    ap.k = k;
    ap.scale_log2 = scale * 1.4426950408889634f;
    ap.cache_off = cache_off;
    ap.nsplit = pl.nsplit;
    ap.part_o = reinterpret_cast<float*>(ws + pl.off_po);
    ap.part_ml = reinterpret_cast<float*>(ws + pl.off_pml);
    ap.err = err;
    ap.key_base = key_base;
    ap.skip_foreign = key_base != nullptr ? 1 : 0;
    return launch_attn<128, 4, 8, true>(fn, ap, (int64_t)B * pl.nsplit, st);
}

// The decode itself, on checked arguments.
dsa_status_t run_decode(const char* fn, const void* q_I, const float* w, const void* Q,
                        const void* kI_cache, const void* K_cache, const void* V_cache,
                        const int64_t* cache_off, int B, int64_t total_n, int k, int Hq, int d,
                        float scale, void* O, int32_t* idx_out, void* workspace,
                        size_t workspace_bytes, int32_t* err, dsa_stream_t stream) {
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: workspace is not 256-byte aligned", fn);
    const DecodePlan pl = plan_decode(B, total_n, k, Hq, d, num_sms());
    if (workspace_bytes < pl.total)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, workspace_bytes,
                    pl.total);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + pl.off_idx);
    dsa_status_t r = launch_decode_select(fn, pl, ws, q_I, w, kI_cache, cache_off, B, total_n, k,
                                          idx, nullptr, nullptr, false, err, st);
    if (r != DSA_OK) return r;
    r = launch_decode_attn(fn, pl, ws, Q, K_cache, V_cache, cache_off, B, k, scale, idx, nullptr,
                           err, st);
    if (r != DSA_OK) return r;
    const float* po = reinterpret_cast<const float*>(ws + pl.off_po);
    const float* pml = reinterpret_cast<const float*>(ws + pl.off_pml);
    CUDA_TRY(launch_chained(dsa::attn::combine_kernel<128, 32, true>, dim3(B * 32), dim3(128), 0,
                            st, po, pml, pl.nsplit, (int64_t)pl.nsplit, (int64_t)1,
                            static_cast<__nv_bfloat16*>(O), static_cast<float*>(nullptr),
                            static_cast<float*>(nullptr)));
    CUDA_TRY(cudaGetLastError());
    return ok();
}

}  // namespace

extern "C" {

dsa_status_t dsa_sparse_attn_decode(const void* q_I, const float* w, const void* Q,
                                    const void* kI_cache, const void* K_cache,
                                    const void* V_cache, const int64_t* cache_off, int B,
                                    int64_t total_n, int H_I, int d_I, int Hq, int Hkv, int d,
                                    int k, float scale, void* O, int32_t* idx_out,
                                    void* workspace, size_t workspace_bytes, int32_t* err,
                                    dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_decode";
    dsa_status_t r = check_decode_args(fn, q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, B,
                                       total_n, H_I, d_I, Hq, Hkv, d, k, scale, O, idx_out, err);
    if (r != DSA_OK) return r;
    CHECK_PTR(workspace);
    return run_decode(fn, q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, B, total_n, k, Hq, d,
                      scale, O, idx_out, workspace, workspace_bytes, err, stream);
}

dsa_status_t dsa_decode_from_host(const void* q_I_host, const float* w_host, const void* Q_host,
                                  void* O_host, int32_t* idx_host, void* q_I, float* w, void* Q,
                                  const void* kI_cache, const void* K_cache, const void* V_cache,
                                  const int64_t* cache_off, int B, int64_t total_n, int H_I,
                                  int d_I, int Hq, int Hkv, int d, int k, float scale, void* O,
                                  int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                  int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_decode_from_host";
    CHECK_PTR(q_I_host);
    CHECK_PTR(w_host);
    CHECK_PTR(Q_host);
    CHECK_PTR(O_host);
    if (idx_host != nullptr && idx_out == nullptr)
        return fail(DSA_ERR_INVALID_ARG, "%s: idx_host needs idx_out", fn);
    dsa_status_t r = check_decode_args(fn, q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, B,
                                       total_n, H_I, d_I, Hq, Hkv, d, k, scale, O, idx_out, err);
    if (r != DSA_OK) return r;
    CHECK_PTR(workspace);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: workspace is not 256-byte aligned", fn);
    const size_t need = plan_decode(B, total_n, k, Hq, d, num_sms()).total;
    if (workspace_bytes < need)  // checked before any copy is queued
        return fail(DSA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, workspace_bytes, need);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the step's new inputs: one query row per sequence (the caches stay on the device)
    CUDA_TRY(cudaMemcpyAsync(q_I, q_I_host, (size_t)B * H_I * d_I, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(w, w_host, (size_t)B * H_I * 4, cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(Q, Q_host, (size_t)B * Hq * d * 2, cudaMemcpyHostToDevice, st));
    r = run_decode(fn, q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, B, total_n, k, Hq, d,
                   scale, O, idx_out, workspace, workspace_bytes, err, stream);
    if (r != DSA_OK) return r;
    CUDA_TRY(cudaMemcpyAsync(O_host, O, (size_t)B * Hq * d * 2, cudaMemcpyDeviceToHost, st));
    if (idx_host != nullptr)
        CUDA_TRY(cudaMemcpyAsync(idx_host, idx_out, (size_t)B * k * 4, cudaMemcpyDeviceToHost, st));
    return ok();
}

// ------------------------------------------------------------ decode over cache shards

dsa_status_t dsa_decode_select_shard(const void* q_I, const float* w, const void* kI_cache,
                                     const int64_t* cache_off, const int64_t* key_base, int B,
                                     int64_t total_n, int H_I, int d_I, int k, uint32_t* ord_out,
                                     int32_t* key_out, void* workspace, size_t workspace_bytes,
                                     int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_decode_select_shard";
    CHECK_PTR(q_I);
    CHECK_PTR(w);
    CHECK_PTR(kI_cache);
    CHECK_PTR(cache_off);
    CHECK_PTR(ord_out);
    CHECK_PTR(key_out);
    CHECK_PTR(workspace);
    CHECK_ERR_WORD(err);
    if (key_base != nullptr && (reinterpret_cast<uintptr_t>(key_base) & 7u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: key_base is not 8-byte aligned", fn);
    if (B < 1 || B > 4096) return fail(DSA_ERR_INVALID_ARG, "%s: B = %d", fn, B);
    if (total_n < 1 || total_n >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: total_n = %lld", fn, (long long)total_n);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (H_I != 64 || d_I != 128 || k > 2048)
        return fail(DSA_ERR_UNSUPPORTED, "%s: supported H_I=64, d_I=128, k<=2048", fn);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: workspace is not 256-byte aligned", fn);
    const DecodePlan pl = plan_decode(B, total_n, k, 32, 128, num_sms());
    if (workspace_bytes < pl.total)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, workspace_bytes,
                    pl.total);
    const dsa_status_t r = launch_decode_select(
        fn, pl, static_cast<uint8_t*>(workspace), q_I, w, kI_cache, cache_off, B, total_n, k,
        key_out, ord_out, key_base, true, err, static_cast<cudaStream_t>(stream));
    return r == DSA_OK ? ok() : r;
}

dsa_status_t dsa_decode_merge_shards(const uint32_t* ord_in, const int32_t* key_in, int P, int B,
                                     int k, int32_t* idx, int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_decode_merge_shards";
    CHECK_PTR(ord_in);
    CHECK_PTR(key_in);
    CHECK_PTR(idx);
    CHECK_ERR_WORD(err);
    if (P < 1 || P > dsa::dec::kMaxShards)
        return fail(DSA_ERR_UNSUPPORTED, "%s: P = %d (1..%d shards)", fn, P, dsa::dec::kMaxShards);
    if (B < 1 || B > 65535) return fail(DSA_ERR_INVALID_ARG, "%s: B = %d", fn, B);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (k > 2048) return fail(DSA_ERR_UNSUPPORTED, "%s: k = %d > 2048", fn, k);
    const int smem = P * k * 8;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUDA_TRY(cudaFuncSetAttribute(dsa::dec::merge_shards_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    dsa::dec::merge_shards_kernel<<<B, 1024, smem, st>>>(ord_in, key_in, P, B, k, idx, err);
    CUDA_TRY(cudaGetLastError());
    return ok();
}

size_t dsa_decode_attn_shard_workspace_size(int B, int64_t total_n, int k, int Hq, int d) {
    if (B < 1 || total_n < 1 || k < 1) return 0;
    return plan_decode(B, total_n, k, Hq, d, num_sms()).total;
}

dsa_status_t dsa_decode_attn_shard(const void* Q, const void* K_cache, const void* V_cache,
                                   const int64_t* cache_off, const int64_t* key_base,
                                   const int32_t* idx, int B, int64_t total_n, int Hq, int Hkv,
                                   int d, int k, float scale, float* part_o, float* part_ml,
                                   void* workspace, size_t workspace_bytes, int32_t* err,
                                   dsa_stream_t stream) {
    static const char fn[] = "dsa_decode_attn_shard";
    CHECK_PTR(Q);
    CHECK_PTR(K_cache);
    CHECK_PTR(V_cache);
    CHECK_PTR(cache_off);
    CHECK_PTR(idx);
    CHECK_PTR(part_o);
    CHECK_PTR(part_ml);
    CHECK_PTR(workspace);
    CHECK_ERR_WORD(err);
    if (key_base == nullptr || (reinterpret_cast<uintptr_t>(key_base) & 7u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: key_base is NULL or not 8-byte aligned", fn);
    if (B < 1 || B > 4096) return fail(DSA_ERR_INVALID_ARG, "%s: B = %d", fn, B);
    if (total_n < 1 || total_n >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: total_n = %lld", fn, (long long)total_n);
    if (k < 1) return fail(DSA_ERR_INVALID_ARG, "%s: k = %d", fn, k);
    if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "%s: scale", fn);
    if (d != 128 || Hkv != 4 || Hq != 32 || k > 2048)
        return fail(DSA_ERR_UNSUPPORTED, "%s: supported d=128, Hkv=4, Hq=32, k<=2048", fn);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: workspace is not 256-byte aligned", fn);
    const DecodePlan pl = plan_decode(B, total_n, k, Hq, d, num_sms());
    if (workspace_bytes < pl.total)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace %zu < %zu bytes", fn, workspace_bytes,
                    pl.total);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    dsa_status_t r = launch_decode_attn(fn, pl, ws, Q, K_cache, V_cache, cache_off, B, k, scale,
                                        idx, key_base, err, st);
    if (r != DSA_OK) return r;
    const float* po = reinterpret_cast<const float*>(ws + pl.off_po);
    const float* pml = reinterpret_cast<const float*>(ws + pl.off_pml);
    CUDA_TRY(launch_chained(dsa::attn::combine_kernel<128, 32, false>, dim3(B * 32), dim3(128), 0,
                            st, po, pml, pl.nsplit, (int64_t)pl.nsplit, (int64_t)1,
                            static_cast<__nv_bfloat16*>(nullptr), part_o, part_ml));
    CUDA_TRY(cudaGetLastError());
    return ok();
}

dsa_status_t dsa_decode_combine_shards(const float* part_o, const float* part_ml, int P, int B,
                                       int Hq, int d, void* O, int32_t* err,
                                       dsa_stream_t stream) {
    static const char fn[] = "dsa_decode_combine_shards";
    CHECK_PTR(part_o);
    CHECK_PTR(part_ml);
    CHECK_PTR(O);
    CHECK_ERR_WORD(err);
    if (P < 1 || P > 1024) return fail(DSA_ERR_INVALID_ARG, "%s: P = %d", fn, P);
    if (B < 1 || B > 65535) return fail(DSA_ERR_INVALID_ARG, "%s: B = %d", fn, B);
    if (d != 128 || Hq != 32) return fail(DSA_ERR_UNSUPPORTED, "%s: supported d=128, Hq=32", fn);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dsa::attn::combine_kernel<128, 32, true><<<B * 32, 128, 0, st>>>(
        part_o, part_ml, P, (int64_t)1, (int64_t)B, static_cast<__nv_bfloat16*>(O), nullptr,
        nullptr);
    CUDA_TRY(cudaGetLastError());
    return ok();
}

dsa_status_t dsa_check_device_error(int32_t* err, int* code, dsa_stream_t stream) {
    static const char fn[] = "dsa_check_device_error";
    if (!code) return fail(DSA_ERR_INVALID_ARG, "%s: code is NULL", fn);
    CHECK_ERR_WORD(err);
    CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int v = 0, zero = 0;
    if (err != nullptr) {
        CUDA_TRY(cudaMemcpy(&v, err, sizeof(int), cudaMemcpyDeviceToHost));
        CUDA_TRY(cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice));
    } else {
        CUDA_TRY(cudaMemcpyFromSymbol(&v, dsa::g_dsa_device_error, sizeof(int)));
        CUDA_TRY(cudaMemcpyToSymbol(dsa::g_dsa_device_error, &zero, sizeof(int)));
    }
    *code = v;
    return ok();
}

}  // extern "C"

// ------------------------------------------------------------ decode without allocation
//
// Some callers cannot hand the library a workspace: code that runs inside a
// host framework which owns every byte of device memory and forbids
// allocations after start-up, or a latency-critical decode loop where a
// cudaMalloc (which can synchronize the device) is not acceptable.  For them,
// dsa_sparse_attn_decode_noalloc runs the same decode with its scratch in a
// fixed array that is part of this library's device image.
//
// * Every GPU that loads this library holds the array (kNoAllocScratchBytes)
//   until the process exits.
// * Host code cannot use the array's name as a device address; the address
//   is looked up with cudaGetSymbolAddress once per device (and context), on
//   the first call made with that device current.  Make that first call
//   before any stream capture.  If the device's context is replaced (a
//   cudaDeviceReset, for one), the next call sees a different context and
//   looks the address up again.
// * All calls share the one array and it keeps the last call's contents.
//   Nothing in it has to start at zero: every scratch byte a decode reads was
//   written earlier by the same call.  Calls whose work overlaps on the GPU
//   (two streams, or two host threads) race on the array and must be
//   serialized by the caller.
// * Arguments are checked as dsa_sparse_attn_decode checks them; then a
//   request whose scratch need exceeds the array is rejected with
//   DSA_ERR_WORKSPACE before anything is launched.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoAllocSlot {
    CUcontext ctx;  // context the address was looked up in
    void* ptr;
};
NoAllocSlot g_noalloc_slot[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

CUcontext current_ctx() {
    CUcontext c = nullptr;
    const CtxGetCurrentFn f = ctx_get_current_fn();
    if (f == nullptr || f(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

}  // namespace

extern "C" dsa_status_t dsa_sparse_attn_decode_noalloc(
    const void* q_I, const float* w, const void* Q, const void* kI_cache, const void* K_cache,
    const void* V_cache, const int64_t* cache_off, int B, int64_t total_n, int H_I, int d_I,
    int Hq, int Hkv, int d, int k, float scale, void* O, int32_t* idx_out, int32_t* err,
    dsa_stream_t stream) {
    static const char fn[] = "dsa_sparse_attn_decode_noalloc";
    const dsa_status_t r = check_decode_args(fn, q_I, w, Q, kI_cache, K_cache, V_cache,
                                             cache_off, B, total_n, H_I, d_I, Hq, Hkv, d, k,
                                             scale, O, idx_out, err);
    if (r != DSA_OK) return r;
    const size_t need = dsa_decode_workspace_size(B, total_n, H_I, d_I, k, Hq, Hkv, d);
    if (need > kNoAllocScratchBytes)
        return fail(DSA_ERR_WORKSPACE,
                    "%s: these sizes need %zu bytes of scratch but the built-in array holds %zu; "
                    "use dsa_sparse_attn_decode with a caller workspace",
                    fn, need, kNoAllocScratchBytes);
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(DSA_ERR_UNSUPPORTED, "%s: device ordinal %d", fn, dev);
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        NoAllocSlot& sl = g_noalloc_slot[dev];
        const CUcontext ctx = current_ctx();
        if (sl.ptr == nullptr || ctx == nullptr || ctx != sl.ctx) {
            void* p = nullptr;
            CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));  // sets up the context
            sl.ptr = p;
            sl.ctx = current_ctx();
        }
        scratch = sl.ptr;
    }
    return run_decode(fn, q_I, w, Q, kI_cache, K_cache, V_cache, cache_off, B, total_n, k, Hq, d,
                      scale, O, idx_out, scratch, kNoAllocScratchBytes, err, stream);
}

// ---------------------------------------------------------------- indexer warm-up loss

namespace {

struct KlWorkspace {
    size_t lse_h, lse_I, part, total;
    KlWorkspace(int64_t L, int Hq) {
        const int64_t nt = (L + dsa::kl::kTile - 1) / dsa::kl::kTile;
        lse_h = 0;
        lse_I = align256((size_t)L * Hq * 4);
        part = lse_I + align256((size_t)L * 4);
        total = part + align256((size_t)L * nt * 4);
    }
};

template <int D>
dsa_status_t launch_kl_forward(const char* fn, dsa::kl::Params p, cudaStream_t st) {
    using namespace dsa::kl;
    row_lse_kernel<<<(unsigned)((p.L + 7) / 8), 256, 0, st>>>(p);
    if (D == dsa::kltc::kD && p.Hkv <= 4) {  // tcgen05: 128 x 128 tiles of S in TMEM
        namespace tc = dsa::kltc;
        const unsigned ntq = (unsigned)((p.L + tc::kRows - 1) / tc::kRows);
        p.kl_tile_log2 = 7;
        CUDA_TRY(cudaFuncSetAttribute(tc::head_lse_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      tc::kLseSmemBytes));
        CUDA_TRY(cudaFuncSetAttribute(tc::target_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      tc::kTgtSmemBytes));
        tc::head_lse_tc_kernel<<<dim3(p.Hq, ntq), tc::kThreads, tc::kLseSmemBytes, st>>>(p);
        tc::target_tc_kernel<<<dim3(ntq, ntq), tc::kThreads, tc::kTgtSmemBytes, st>>>(p);
    } else {
        p.kl_tile_log2 = 6;
        const int smem_lse = 2 * BfTile<D>::BYTES;
        const int smem_tgt = (p.Hkv + 2) * BfTile<D>::BYTES;
        CUDA_TRY(cudaFuncSetAttribute(head_lse_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem_lse));
        CUDA_TRY(cudaFuncSetAttribute(target_kernel<D>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, smem_tgt));
        head_lse_kernel<D><<<dim3(p.ntiles, p.Hq), kThreads, smem_lse, st>>>(p);
        target_kernel<D><<<dim3(p.ntiles, p.ntiles), kThreads, smem_tgt, st>>>(p);
    }
    kl_reduce_kernel<<<(unsigned)((p.L + 255) / 256), 256, 0, st>>>(p);
    CUDA_TRY(cudaGetLastError());
    return DSA_OK;
}

template <int DI>
dsa_status_t launch_kl_backward(const char* fn, const dsa::kl::Params& p, cudaStream_t st) {
    using namespace dsa::kl;
    const int smem_dq = 2 * F8Tile<DI>::BYTES;
    const int smem_dk = 2 * F8Tile<DI>::BYTES + (p.HI / p.nsplit) * kWStride * 4;
    CUDA_TRY(cudaFuncSetAttribute(dq_kernel<DI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem_dq));
    CUDA_TRY(cudaFuncSetAttribute(dk_kernel<DI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem_dk));
    if (DI == dsa::kltc::kDI) {  // tcgen05: S in e4m3, dq in bf16, both in TMEM
        CUDA_TRY(cudaFuncSetAttribute(dsa::kltc::dq_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      dsa::kltc::kSmemBytes));
        dsa::kltc::dq_tc_kernel<<<dim3(p.HI, (unsigned)((p.L + dsa::kltc::kRows - 1) /
                                                         dsa::kltc::kRows)),
                                  dsa::kltc::kThreads, dsa::kltc::kSmemBytes, st>>>(p);
    } else {
        dq_kernel<DI><<<dim3(p.HI, p.ntiles), kThreads, smem_dq, st>>>(p);
    }
    if (DI == dsa::kltc::kDI && p.HI / p.nsplit <= dsa::kltc::kMaxHps) {
        CUDA_TRY(cudaFuncSetAttribute(dsa::kltc::dk_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      dsa::kltc::kDkSmemBytes));
        dsa::kltc::dk_tc_kernel<<<dim3(p.nsplit, (unsigned)((p.L + dsa::kltc::kRows - 1) /
                                                            dsa::kltc::kRows)),
                                  dsa::kltc::kThreads, dsa::kltc::kDkSmemBytes, st>>>(p);
    } else {
        dk_kernel<DI><<<dim3(p.nsplit, p.ntiles), kThreads, smem_dk, st>>>(p);
    }
    if (p.nsplit > 1)
        dk_reduce_kernel<<<(unsigned)((p.L * DI / 4 + 255) / 256), 256, 0, st>>>(p, DI);
    CUDA_TRY(cudaGetLastError());
    return DSA_OK;
}

// Head groups of dk_kernel: the largest divisor of H_I that is at most 8.
int kl_dk_splits(int H_I) {
    for (int n = 8; n > 1; --n)
        if (H_I % n == 0) return n;
    return 1;
}

}  // namespace

extern "C" {

size_t dsa_indexer_kl_backward_workspace_size(int64_t L, int H_I, int d_I) {
    if (L < 1 || H_I < 1 || d_I < 1) return 0;
    const int n = kl_dk_splits(H_I);
    return n > 1 ? align256((size_t)n * L * d_I * 4) : 256;
}

size_t dsa_indexer_kl_workspace_size(int64_t L, int Hq) {
    if (L < 1 || Hq < 1) return 0;
    return KlWorkspace(L, Hq).total;
}

dsa_status_t dsa_indexer_kl_forward(const void* q_I, const void* k_I, const float* w,
                                    const void* Q, const void* K, int64_t L, int H_I, int d_I,
                                    int Hq, int Hkv, int d, float scale, float scale_I, float* kl,
                                    float* G, void* workspace, size_t workspace_bytes,
                                    int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_indexer_kl_forward";
    CHECK_ERR_WORD(err);
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(Q);
    CHECK_PTR(K);
    CHECK_PTR(kl);
    CHECK_PTR(G);
    CHECK_PTR(workspace);
    if (L < 1 || L * L >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld (L * L must be < 2^31)", fn, (long long)L);
    if (Hkv < 1 || Hkv > 8 || Hq < Hkv || Hq % Hkv != 0)
        return fail(DSA_ERR_INVALID_ARG, "%s: Hq = %d, Hkv = %d (Hkv in 1..8 dividing Hq)", fn, Hq,
                    Hkv);
    if (d != 64 && d != 128) return fail(DSA_ERR_UNSUPPORTED, "%s: d = %d (64 or 128)", fn, d);
    if (!(scale_I > 0.f) || !(scale > 0.f))
        return fail(DSA_ERR_INVALID_ARG, "%s: scale and scale_I must be > 0", fn);
    const KlWorkspace ws(L, Hq);
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", fn);
    if (workspace_bytes < ws.total)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", fn,
                    workspace_bytes, ws.total);
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    dsa_status_t r = dispatch_index<false>(fn, q_I, k_I, w, L, H_I, d_I, 1, nullptr, G, nullptr, 1,
                                           err, st);
    if (r != DSA_OK) return r;
    dsa::kl::Params p{};
    p.Q = static_cast<const __nv_bfloat16*>(Q);
    p.K = static_cast<const __nv_bfloat16*>(K);
    p.L = L;
    p.HI = H_I;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.ntiles = (int)((L + dsa::kl::kTile - 1) / dsa::kl::kTile);
    p.scale_log2 = scale * dsa::kl::kLog2e;
    p.scale_I = scale_I;
    p.G = G;
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    p.lse_h = reinterpret_cast<float*>(wsb + ws.lse_h);
    p.lse_I = reinterpret_cast<float*>(wsb + ws.lse_I);
    p.kl_part = reinterpret_cast<float*>(wsb + ws.part);
    p.kl = kl;
    p.err = err;
    r = d == 128 ? launch_kl_forward<128>(fn, p, st) : launch_kl_forward<64>(fn, p, st);
    return r == DSA_OK ? ok() : r;
}

dsa_status_t dsa_indexer_kl_backward(const void* q_I, const void* k_I, const float* w,
                                     const float* G, int64_t L, int H_I, int d_I, float* dq_I,
                                     float* dk_I, float* dw, void* workspace,
                                     size_t workspace_bytes, int32_t* err, dsa_stream_t stream) {
    static const char fn[] = "dsa_indexer_kl_backward";
    CHECK_ERR_WORD(err);
    CHECK_PTR(q_I);
    CHECK_PTR(k_I);
    CHECK_PTR(w);
    CHECK_PTR(G);
    CHECK_PTR(dq_I);
    CHECK_PTR(dk_I);
    CHECK_PTR(dw);
    if (L < 1 || L * L >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "%s: L = %lld (L * L must be < 2^31)", fn, (long long)L);
    if (H_I < 1 || H_I > 256) return fail(DSA_ERR_INVALID_ARG, "%s: H_I = %d (1..256)", fn, H_I);
    if (d_I != 64 && d_I != 128)
        return fail(DSA_ERR_UNSUPPORTED, "%s: d_I = %d (64 or 128)", fn, d_I);
    CHECK_PTR(workspace);
    const size_t need = dsa_indexer_kl_backward_workspace_size(L, H_I, d_I);
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", fn);
    if (workspace_bytes < need)
        return fail(DSA_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", fn,
                    workspace_bytes, need);
    dsa::kl::Params p{};
    p.nsplit = kl_dk_splits(H_I);
    p.dk_part = static_cast<float*>(workspace);
    p.qI = static_cast<const uint8_t*>(q_I);
    p.kI = static_cast<const uint8_t*>(k_I);
    p.w = w;
    p.L = L;
    p.HI = H_I;
    p.ntiles = (int)((L + dsa::kl::kTile - 1) / dsa::kl::kTile);
    p.Gin = G;
    p.dq = dq_I;
    p.dk = dk_I;
    p.dw = dw;
    p.err = err;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dsa_status_t r =
        d_I == 128 ? launch_kl_backward<128>(fn, p, st) : launch_kl_backward<64>(fn, p, st);
    return r == DSA_OK ? ok() : r;
}

}  // extern "C"

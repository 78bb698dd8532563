/*
 * dsa.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention hot path:
 * Lightning-Indexer scores -> per-query top-k -> sparse GQA attention, for
 * prefill and for single-token decode.
 *
 * Source of the operations: Kwai Keye-VL-2.0 technical-report summary,
 * section 1 (a light MQA-style indexer scans the whole context, each query
 * keeps its 2048 best positions, attention runs over those only, cost falls
 * from O(L^2) to O(Lk); the base model is GQA) and section 8 (decode-time
 * sparse attention; a deterministic top-k so that training and inference
 * select the same keys).  The pages give no formula for the indexer; it is
 * read as DeepSeek's published one:
 *
 *     I[t,s] = sum_j w[t,j] * max(0, sum_c qI[t,j,c] * kI[s,c]),   s <= t.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer is a DEVICE pointer unless stated, 16-byte aligned, to a
 *   dense row-major array with the layout given.  The caller owns all
 *   memory; the library never allocates device memory.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and do not synchronize, except dsa_check_device_error.
 * - Arguments are validated on the host before anything is launched; a
 *   failing call returns a status, launches nothing and leaves a message in
 *   dsa_last_error().  No C++ exception crosses this boundary.
 * - FP8 tensors are OCP e4m3 bytes; bf16 tensors are raw bf16 bits.
 * - Top-k order: higher score first, then lower key index (a total order,
 *   so exactly one set is correct).  Scores are accumulated in fp32; they
 *   are exact (and the selected sets bit-identical to an exact reference)
 *   whenever the inputs are integer-valued with |score| < 2^24, e.g.
 *   indexer values in [-8, 8] with d_I <= 128 and weights in {0..3}.
 * - Index rows list the selected keys in ascending order, then -1 padding.
 *   The result is deterministic: the same inputs give the same bits.
 * - Device error word.  A kernel that detects an error (a bounded wait that
 *   timed out, an index out of range) records a DSA_DEVERR_* code instead
 *   of faulting, and finishes.  Every launching call takes `err`: a device
 *   pointer to a caller-owned int32 (4-byte aligned) that the call's kernels
 *   record into (the first error wins; nothing else is written there), or
 *   NULL, in which case they record into the library's per-device word.
 *   Calls that may run at the same time (two streams, two host threads)
 *   should each pass their own word, so that neither sees nor clears the
 *   other's error.  The word must hold 0 before the call for a later
 *   non-zero value to mean "this call failed"; dsa_check_device_error reads
 *   a word and clears it.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative or inconsistent size */
    DSA_ERR_UNSUPPORTED = 2,   /* a shape outside the compiled variants (see each call) */
    DSA_ERR_WORKSPACE = 3,     /* workspace smaller than the matching *_workspace_size */
    DSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    DSA_ERR_DEVICE = 5         /* a kernel recorded an error in the device error word */
} dsa_status_t;

/* Device error word codes (dsa_check_device_error). */
#define DSA_DEVERR_NONE 0
#define DSA_DEVERR_TIMEOUT 1     /* a bounded wait inside a kernel gave up */
#define DSA_DEVERR_INDEX 2       /* an index row held a key outside the cache */

typedef void* dsa_stream_t;   /* cudaStream_t */

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
DSA_API int dsa_version(void);

/* Human-readable name of a status code; never NULL. */
DSA_API const char* dsa_status_string(int status);

/* Message of the last failing call on this host thread ("" if none). */
DSA_API const char* dsa_last_error(void);

/*
 * dsa_index_topk - prefill indexer + top-k (hot-path steps A1 and A2).
 * Computes I[t,s] for every causal pair with FP8 tcgen05 tensor-core MMAs,
 * applies the per-head ReLU and weighted head sum in the epilogue, and keeps
 * a streaming top-k per query in shared memory; the L x L score matrix is
 * never written.
 *
 *   q_I  [L][H_I][d_I]  e4m3   indexer queries
 *   k_I  [L][d_I]       e4m3   indexer keys (one per token, shared by heads)
 *   w    [L][H_I]       fp32   per-query head weights
 *   idx  [L][k]         int32  OUT: row t = the min(k, t+1) selected keys
 *                              s <= t, ascending, then -1
 * Supported: H_I in {4, 64}, d_I in {64, 128}, 1 <= k <= 2048,
 * 1 <= L <= 2^30.  Others return DSA_ERR_UNSUPPORTED.
 */
DSA_API dsa_status_t dsa_index_topk(const void* q_I, const void* k_I, const float* w, int64_t L,
                            int H_I, int d_I, int k, int32_t* idx, int32_t* err,
                            dsa_stream_t stream);

/*
 * dsa_index_topk_varlen - dsa_index_topk over a packed batch of sequences
 * (the pages' varlen mode and sequence packing, Kwai Keye-VL-2.0 technical
 * report summary, sections 1 and 8).  Row t of sequence b, with
 * cu_seqlens[b] <= t < cu_seqlens[b+1], sees only the keys
 * s in [cu_seqlens[b], t]: the causal mask restarts at every sequence.
 *
 *   cu_seqlens [nseq+1] int32  device; 0 = cu_seqlens[0] <= ... <=
 *                              cu_seqlens[nseq] = L (caller's contract; a
 *                              first or last entry other than 0 and L
 *                              records DSA_DEVERR_INDEX)
 *   q_I, k_I, w, idx           as dsa_index_topk over the packed rows; idx
 *                              holds packed (global) key positions, so
 *                              dsa_sparse_attn_prefill runs on it unchanged
 * Same shape support as dsa_index_topk.
 */
DSA_API dsa_status_t dsa_index_topk_varlen(const void* q_I, const void* k_I, const float* w,
                                   const int32_t* cu_seqlens, int nseq, int64_t L, int H_I,
                                   int d_I, int k, int32_t* idx, int32_t* err,
                                   dsa_stream_t stream);

/*
 * dsa_index_topk_rows - dsa_index_topk for the query rows [row0, row1) only:
 * one rank's share when the query tokens of one long sequence are split
 * across GPUs (each query's selection needs every earlier key, so the keys
 * are gathered to every rank first; the rows themselves are independent).
 * Row t's result equals row t of dsa_index_topk over the whole sequence.
 *
 *   q_I  [row1-row0][H_I][d_I]  e4m3   the rows' indexer queries
 *   k_I  [row1][d_I]            e4m3   keys 0 .. row1-1
 *   w    [row1-row0][H_I]       fp32
 *   idx  [row1-row0][k]         int32  OUT, as dsa_index_topk
 * row0 must be a multiple of 4 (the indexer's query block).  Same shape
 * support as dsa_index_topk.
 */
DSA_API dsa_status_t dsa_index_topk_rows(const void* q_I, const void* k_I, const float* w,
                                 int64_t row0, int64_t row1, int H_I, int d_I, int k,
                                 int32_t* idx, int32_t* err, dsa_stream_t stream);

/*
 * dsa_sparse_attn_rows - dsa_sparse_attn_prefill for nrows query rows whose
 * index rows select among nkeys keys (the query rows of one rank; keys are
 * positions in K and V).
 *
 *   Q    [nrows][Hq][d]  bf16;   K, V [nkeys][Hkv][d] bf16
 *   idx  [nrows][k]      int32;  O [nrows][Hq][d] bf16 OUT;  lse [nrows][Hq] OUT or NULL
 * Same shape support as dsa_sparse_attn_prefill.
 */
DSA_API dsa_status_t dsa_sparse_attn_rows(const void* Q, const void* K, const void* V,
                                  const int32_t* idx, int64_t nrows, int64_t nkeys, int Hq,
                                  int Hkv, int d, int k, float scale, void* O, float* lse,
                                  int32_t* err, dsa_stream_t stream);

/*
 * dsa_sparse_attn_prefill_dedup - the result of dsa_sparse_attn_prefill,
 * computed for blocks of adjacent query tokens that load the union of their
 * index rows once (adjacent-query dedup, Kwai Keye-VL-2.0 technical report
 * summary, section 8, item 2).  A block holds 128 / G tokens (G = Hq / Hkv
 * query heads per KV group), so that its tokens times the G heads of one
 * group are the 128 rows of one tensor-core tile; each key the block selects
 * is gathered once per group, and each token keeps only its own keys through
 * a mask applied to the score tile.  It pays when adjacent rows overlap
 * strongly (clustered video tokens); its products grow with the union, so
 * on unclustered rows it is slower than dsa_sparse_attn_prefill.
 *   Q [L][Hq][d], K, V [L][Hkv][d] bf16; idx [L][k] int32 (entries < 0 are
 *   holes; entries >= L are skipped and record DSA_DEVERR_INDEX; a key that
 *   repeats within one row counts once); O [L][Hq][d] bf16 OUT (a row
 *   without keys is zeros).
 *   workspace / workspace_bytes: device memory of at least
 *   dsa_sparse_attn_prefill_dedup_workspace_size(L, Hq, Hkv, d, k) bytes,
 *   16-byte aligned, owned by the caller and not read before it is written;
 *   the blocks run in waves of at most 4096, which bounds its size.
 * Supported: d in {64, 128}, Hq / Hkv in {4, 8}, L <= 262144, and at most
 * 32768 distinct keys per block ((128 / G) x k, or L when smaller).
 * Errors: null or misaligned pointers, bad sizes (DSA_ERR_INVALID_ARG),
 * other shapes (DSA_ERR_UNSUPPORTED), a short workspace (DSA_ERR_WORKSPACE).
 */
DSA_API size_t dsa_sparse_attn_prefill_dedup_workspace_size(int64_t L, int Hq, int Hkv, int d,
                                                            int k);
DSA_API dsa_status_t dsa_sparse_attn_prefill_dedup(const void* Q, const void* K, const void* V,
                                           const int32_t* idx, int64_t L, int Hq, int Hkv,
                                           int d, int k, float scale, void* O, void* workspace,
                                           size_t workspace_bytes, int32_t* err,
                                           dsa_stream_t stream);

/*
 * dsa_prefill_from_host - the whole prefill (A1 + A2 + A3) for inputs that
 * sit in host memory.  The rows are handled in chunks of chunk_rows (rounded
 * up to a multiple of 128): each chunk's rows of q_I, k_I, w, Q, K and V are
 * copied into the caller's device buffers on h2d_stream; as soon as they are
 * there (with every earlier key), the chunk's index rows and attention run on
 * `stream`; its output rows go back to O_host on d2h_stream.  Copies of
 * later chunks thus overlap the kernels of earlier ones.  Asynchronous: when
 * `stream` reaches the end of this call's work, O_host holds the result and
 * idx the index rows.  The copy streams first wait for the work already
 * queued on `stream` (which may still use the device buffers).  Host buffers
 * must be page-locked for the copies to be asynchronous; the three streams
 * must be distinct.
 *
 *   *_host              host pointers, layouts as the device buffers below
 *   q_I, k_I, w, Q, K, V, idx, O
 *                       caller-owned device buffers, layouts as in
 *                       dsa_index_topk and dsa_sparse_attn_prefill
 * Same shape support as dsa_index_topk and dsa_sparse_attn_prefill.
 */
DSA_API dsa_status_t dsa_prefill_from_host(const void* q_I_host, const void* k_I_host,
                                   const float* w_host, const void* Q_host, const void* K_host,
                                   const void* V_host, void* O_host, void* q_I, void* k_I,
                                   float* w, void* Q, void* K, void* V, int32_t* idx, void* O,
                                   int64_t L, int H_I, int d_I, int Hq, int Hkv, int d, int k,
                                   float scale, int64_t chunk_rows, int32_t* err,
                                   dsa_stream_t stream, dsa_stream_t h2d_stream,
                                   dsa_stream_t d2h_stream);

/*
 * dsa_index_scores - the same indexer, writing the dense causal score
 * matrix instead of selecting (for small L: checks and training losses that
 * need the whole score distribution).
 *
 *   scores [L][L] fp32  OUT: I[t,s] for s <= t, -inf for s > t
 * Same shape support as dsa_index_topk; L * L must fit in 2^31 elements.
 */
DSA_API dsa_status_t dsa_index_scores(const void* q_I, const void* k_I, const float* w, int64_t L,
                              int H_I, int d_I, float* scores, int32_t* err,
                              dsa_stream_t stream);

/*
 * dsa_sparse_attn_prefill - sparse GQA attention over selected rows (A3).
 * For every query token t and query head h, with group g = h / (Hq / Hkv):
 *   O[t,h] = sum_{s in idx[t]} softmax_s(scale * Q[t,h] . K[s,g]) V[s,g]
 * Each selected K/V row is gathered once per token and shared by all query
 * heads of its group; softmax is online in fp32; O is rounded to bf16 (RNE).
 *
 *   Q    [L][Hq][d]   bf16
 *   K, V [L][Hkv][d]  bf16
 *   idx  [L][k]       int32  keys to attend; entries < 0 are skipped, so
 *                            rows may be padded with -1 in any position;
 *                            an entry >= L is skipped and flagged
 *                            DSA_DEVERR_INDEX
 *   O    [L][Hq][d]   bf16   OUT (a row with no valid entry is all zeros)
 *   lse  [L][Hq]      fp32   OUT or NULL: natural log of each row's softmax
 *                            normaliser, log sum_s exp(scale Q[t,h] . K[s,g])
 *                            (-inf for a row with no valid entry); the
 *                            backward's input
 * Supported: d in {64, 128}; (Hkv, Hq/Hkv) in {(2, 4), (4, 8)}; k <= 65536.
 */
DSA_API dsa_status_t dsa_sparse_attn_prefill(const void* Q, const void* K, const void* V,
                                     const int32_t* idx, int64_t L, int Hq, int Hkv, int d,
                                     int k, float scale, void* O, float* lse, int32_t* err,
                                     dsa_stream_t stream);

/*
 * dsa_sparse_attn_backward - gradients of a loss through the sparse GQA
 * attention (the sparse-adaptation training stage: Kwai Keye-VL-2.0
 * technical-report summary, section 1 -- every parameter is trained on the
 * next-token loss through the truly sparse attention; the index rows are
 * fixed).  With P[t,h,i] = exp(scale Q[t,h] . K[s_i,g] - lse[t,h]) over the
 * valid entries s_i of idx[t] and g = h / (Hq / Hkv):
 *   dP = dO[t,h] . V[s_i,g],  D = dO[t,h] . O[t,h],  dS = P (dP - D)
 *   dQ[t,h]   = scale sum_i dS K[s_i,g]
 *   dK[s,g]   = scale sum over (t, h in g, i with s_i = s) of dS Q[t,h]
 *   dV[s,g]   = sum over the same of P dO[t,h]
 * (an index entry that repeats a key counts once per entry, as in the
 * forward).
 *
 *   Q, K, V, idx    as dsa_sparse_attn_prefill
 *   O    [L][Hq][d]   bf16   the forward's output
 *   lse  [L][Hq]      fp32   the forward's lse output
 *   dO   [L][Hq][d]   bf16   gradient of the loss with respect to O
 *   dQ   [L][Hq][d]   fp32   OUT
 *   dK, dV [L][Hkv][d] fp32  OUT (overwritten: the call clears them, then
 *                            accumulates every selecting row's share)
 * dS and P are rounded to bf16 for their products (fp32 accumulation).  dQ
 * is deterministic; dK and dV are sums of fp32 reductions whose order varies
 * from run to run (results agree to rounding).  Supported shapes as
 * dsa_sparse_attn_prefill.
 */
DSA_API dsa_status_t dsa_sparse_attn_backward(const void* Q, const void* K, const void* V,
                                      const int32_t* idx, const void* O, const float* lse,
                                      const void* dO, int64_t L, int Hq, int Hkv, int d, int k,
                                      float scale, float* dQ, float* dK, float* dV,
                                      int32_t* err, dsa_stream_t stream);

/*
 * dsa_decode_workspace_size - bytes of device workspace that
 * dsa_sparse_attn_decode needs for these sizes (256-byte aligned pointer).
 */
DSA_API size_t dsa_decode_workspace_size(int B, int64_t total_n, int H_I, int d_I, int k, int Hq,
                                 int Hkv, int d);

/*
 * dsa_sparse_attn_decode - one new token per sequence over a long cache (A4):
 * indexer over each sequence's whole cache, top-k, sparse GQA attention.
 * The caches are packed: sequence b owns rows [cache_off[b], cache_off[b+1])
 * and its newest row (the token being decoded, appended by the caller
 * before the call) is the last one, so the result equals prefill row
 * t = n_b - 1 of that sequence.
 *
 *   q_I       [B][H_I][d_I]      e4m3
 *   w         [B][H_I]           fp32
 *   Q         [B][Hq][d]         bf16
 *   kI_cache  [total_n][d_I]     e4m3
 *   K_cache, V_cache [total_n][Hkv][d] bf16
 *   cache_off [B+1]              int64, device: prefix sums, cache_off[0] = 0,
 *                                cache_off[B] = total_n, every n_b >= 1
 *   O         [B][Hq][d]         bf16  OUT
 *   idx_out   [B][k]             int32 OUT or NULL: sequence-local keys,
 *                                ascending, -1 padded
 *   workspace / workspace_bytes  >= dsa_decode_workspace_size(...)
 * Supported: H_I = 64, d_I = 128, d = 128, Hkv = 4, Hq = 32, k <= 2048,
 * 1 <= B <= 4096, total_n < 2^31.
 */
DSA_API dsa_status_t dsa_sparse_attn_decode(const void* q_I, const float* w, const void* Q,
                                    const void* kI_cache, const void* K_cache,
                                    const void* V_cache, const int64_t* cache_off, int B,
                                    int64_t total_n, int H_I, int d_I, int Hq, int Hkv, int d,
                                    int k, float scale, void* O, int32_t* idx_out,
                                    void* workspace, size_t workspace_bytes, int32_t* err,
                                    dsa_stream_t stream);

/*
 * dsa_decode_from_host - one decode step whose new inputs and outputs live in
 * host memory while the caches stay resident on the device (a serving loop:
 * the caller appends the new token's cache rows, then calls this).  On
 * `stream`: the B query rows (q_I, w, Q) are copied from the host into the
 * caller's device buffers, dsa_sparse_attn_decode runs, and O (and, with
 * idx_host, the index rows) are copied back.  Host buffers must be
 * page-locked for the copies to be asynchronous; O_host holds the result
 * once `stream` reaches the end of this call's work.
 *
 *   q_I_host, w_host, Q_host, O_host, idx_host (or NULL)   host pointers,
 *       layouts as q_I, w, Q, O, idx_out of dsa_sparse_attn_decode
 *   q_I, w, Q                 device buffers the queries are copied into
 *   everything else           as dsa_sparse_attn_decode (idx_out is
 *                             required with idx_host)
 */
DSA_API dsa_status_t dsa_decode_from_host(const void* q_I_host, const float* w_host,
                                  const void* Q_host, void* O_host, int32_t* idx_host,
                                  void* q_I, float* w, void* Q, const void* kI_cache,
                                  const void* K_cache, const void* V_cache,
                                  const int64_t* cache_off, int B, int64_t total_n, int H_I,
                                  int d_I, int Hq, int Hkv, int d, int k, float scale, void* O,
                                  int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                  int32_t* err, dsa_stream_t stream);

/*
 * dsa_sparse_attn_decode_noalloc - dsa_sparse_attn_decode for callers that
 * cannot pass a workspace (the pages have no counterpart: this is a
 * deployment convenience).  Callers that run inside a host framework owning
 * all device memory, or a decode loop that must not call cudaMalloc, use it:
 * the scratch lives in a fixed 64 MiB array inside the library's device
 * image, held by every GPU that loads the library until the process exits.
 * Arguments, layouts and results are those of dsa_sparse_attn_decode.
 *
 * - Arguments are checked as dsa_sparse_attn_decode checks them (same
 *   statuses); then sizes whose dsa_decode_workspace_size exceeds 64 MiB
 *   are rejected with DSA_ERR_WORKSPACE before any launch.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is cached per device and
 *   context; a call made after the device's context was replaced (e.g. by
 *   cudaDeviceReset) looks it up again.
 * - All calls share the array and it keeps the last call's contents (no
 *   part of it needs to start at zero).  Calls that overlap on the GPU race
 *   on it: serialize them.
 * - It allocates nothing and frees nothing.
 */
DSA_API dsa_status_t dsa_sparse_attn_decode_noalloc(
    const void* q_I, const float* w, const void* Q, const void* kI_cache, const void* K_cache,
    const void* V_cache, const int64_t* cache_off, int B, int64_t total_n, int H_I, int d_I,
    int Hq, int Hkv, int d, int k, float scale, void* O, int32_t* idx_out, int32_t* err,
    dsa_stream_t stream);

/*
 * Decode over cache shards.  When one GPU cannot (or should not) hold the
 * whole cache of a batch, each rank holds one contiguous part of every
 * sequence's cache (rank r: positions [key_base[b], key_base[b] + n_b) of
 * sequence b, the parts of rank r preceding those of rank r + 1).  The
 * selection decomposes exactly: the global top-k of a sequence lies in the
 * union of the ranks' own top-k lists, under the same order (score, then
 * lower position), so after one exchange of k (score, key) pairs per
 * sequence and rank every rank holds the same index rows a single-GPU
 * decode selects.  The attention decomposes by log-sum-exp: each rank
 * attends over the selected keys it holds and the partials are merged.  The
 * two exchanges (all-gathers of [B][k] pairs and of [B][Hq][d + 2] partials)
 * are the caller's (e.g. NCCL over NVLink); these calls are the per-rank
 * steps:
 *
 *   1. dsa_decode_select_shard   this rank's top-k pairs per sequence
 *   2. (all-gather the pairs into [P][B][k])
 *      dsa_decode_merge_shards   the global index rows, on every rank
 *   3. dsa_decode_attn_shard     this rank's attention partial per (b, h)
 *   4. (all-gather the partials into [P][B][Hq][d] and [P][B][Hq][2])
 *      dsa_decode_combine_shards the output rows
 *
 * dsa_decode_select_shard - indexer scan and exact top-k of this rank's
 * rows of each sequence (hot-path step A4, Kwai Keye-VL-2.0 technical
 * report summary, section 8).
 *   q_I, w, kI_cache   as dsa_sparse_attn_decode (the rank's cache rows)
 *   cache_off [B+1]    int64 device: this rank's rows of sequence b are
 *                      [cache_off[b], cache_off[b+1]); a sequence may have none
 *   key_base  [B]      int64 device or NULL (0): global position of the rank's
 *                      first row of each sequence
 *   ord_out   [B][k]   uint32 OUT: ordered score of each kept key (a monotone
 *                      map of the fp32 score, larger = better; 0 = padding)
 *   key_out   [B][k]   int32 OUT: the kept keys (global positions),
 *                      min(k, n_b) of them ascending, then -1
 *   workspace          dsa_decode_workspace_size(B, total_n, 64, 128, k, 32,
 *                      4, 128) bytes, 256-byte aligned
 * Supported: H_I = 64, d_I = 128, k <= 2048, B <= 4096.
 */
DSA_API dsa_status_t dsa_decode_select_shard(const void* q_I, const float* w, const void* kI_cache,
                                     const int64_t* cache_off, const int64_t* key_base, int B,
                                     int64_t total_n, int H_I, int d_I, int k, uint32_t* ord_out,
                                     int32_t* key_out, void* workspace, size_t workspace_bytes,
                                     int32_t* err, dsa_stream_t stream);

/*
 * dsa_decode_merge_shards - the exact top-k of each sequence over the P
 * ranks' lists from dsa_decode_select_shard, gathered rank-major:
 *   ord_in, key_in [P][B][k]   (rank r's keys all below rank r+1's)
 *   idx            [B][k]      int32 OUT: global keys ascending, then -1
 * A gathered run whose keys do not ascend records DSA_DEVERR_INDEX.
 * Supported: 1 <= P <= 8, k <= 2048.
 */
DSA_API dsa_status_t dsa_decode_merge_shards(const uint32_t* ord_in, const int32_t* key_in, int P,
                                     int B, int k, int32_t* idx, int32_t* err,
                                     dsa_stream_t stream);

/*
 * dsa_decode_attn_shard_workspace_size - bytes of workspace for
 * dsa_decode_attn_shard (256-byte aligned pointer).
 */
DSA_API size_t dsa_decode_attn_shard_workspace_size(int B, int64_t total_n, int k, int Hq, int d);

/*
 * dsa_decode_attn_shard - this rank's share of the decode attention: for
 * each sequence and query head, the softmax-weighted sum over the entries of
 * idx[b] that fall in this rank's rows (other entries are skipped), left
 * unnormalised for the merge:
 *   part_o  [B][Hq][d]  fp32 OUT: sum_i 2^(x_i - M) V_i, x in log2 units
 *                       (scale * log2(e) * Q . K)
 *   part_ml [B][Hq][2]  fp32 OUT: (M, sum_i 2^(x_i - M)); M = -inf and 0 for
 *                       a head with no key here
 *   Q, K_cache, V_cache, cache_off, key_base (required)   as above
 *   idx [B][k]          the global index rows from dsa_decode_merge_shards
 * Supported: d = 128, Hkv = 4, Hq = 32, k <= 2048.
 */
DSA_API dsa_status_t dsa_decode_attn_shard(const void* Q, const void* K_cache, const void* V_cache,
                                   const int64_t* cache_off, const int64_t* key_base,
                                   const int32_t* idx, int B, int64_t total_n, int Hq, int Hkv,
                                   int d, int k, float scale, float* part_o, float* part_ml,
                                   void* workspace, size_t workspace_bytes, int32_t* err,
                                   dsa_stream_t stream);

/*
 * dsa_decode_combine_shards - the output rows from the P ranks' partials,
 * gathered rank-major (part_o [P][B][Hq][d], part_ml [P][B][Hq][2]):
 *   O[b,h] = sum_r 2^(M_r - M) part_o[r,b,h] / sum_r 2^(M_r - M) l_r,
 *   M = max_r M_r;  O [B][Hq][d] bf16 OUT.
 * Supported: d = 128, Hq = 32.
 */
DSA_API dsa_status_t dsa_decode_combine_shards(const float* part_o, const float* part_ml, int P,
                                       int B, int Hq, int d, void* O, int32_t* err,
                                       dsa_stream_t stream);

/*
 * Indexer warm-up loss (dense warm-up stage: Kwai Keye-VL-2.0 technical
 * report summary, section 1 -- the full attention is kept and only the
 * Lightning Indexer is trained, towards the full attention's distribution,
 * under a KL divergence).  The pages print no formula; the reading taken:
 *
 *   I[t,s]  = sum_j w[t,j] relu(q_I[t,j] . k_I[s])                (s <= t)
 *   P_I[t]  = softmax_s(scale_I * I[t,s])
 *   p[t,s]  = (1/Hq) sum_h softmax_s(scale * Q[t,h] . K[s, h / (Hq/Hkv)])
 *   kl[t]   = sum_s p[t,s] (ln p[t,s] - ln P_I[t,s])     (0 ln 0 = 0)
 *   G[t,s]  = d(sum_t kl[t]) / dI[t,s] = scale_I (P_I[t,s] - p[t,s])
 *
 * The attention side is the target and gets no gradient.
 *
 * dsa_indexer_kl_workspace_size - bytes of device workspace the forward
 * needs (256-byte aligned pointer).
 */
DSA_API size_t dsa_indexer_kl_workspace_size(int64_t L, int Hq);

/*
 * dsa_indexer_kl_forward - the loss per token and dL/dI.
 *
 *   q_I  [L][H_I][d_I] e4m3,  k_I [L][d_I] e4m3,  w [L][H_I] fp32
 *   Q    [L][Hq][d] bf16,     K   [L][Hkv][d] bf16
 *   kl   [L]    fp32  OUT
 *   G    [L][L] fp32  OUT: G[t,s] for s <= t, 0 above the diagonal
 * Supported: (H_I, d_I) as dsa_index_topk; d in {64, 128}; Hkv <= 8 with
 * Hq a multiple of Hkv; L * L < 2^31.  Work: the indexer scores (tcgen05,
 * FP8), then two tensor-core passes over the attention scores.  Results are
 * bit-identical run to run.  Errors: DSA_ERR_INVALID_ARG for bad sizes or
 * null pointers, DSA_ERR_WORKSPACE if workspace_bytes is short.
 */
DSA_API dsa_status_t dsa_indexer_kl_forward(const void* q_I, const void* k_I, const float* w,
                                    const void* Q, const void* K, int64_t L, int H_I, int d_I,
                                    int Hq, int Hkv, int d, float scale, float scale_I, float* kl,
                                    float* G, void* workspace, size_t workspace_bytes,
                                    int32_t* err, dsa_stream_t stream);

/*
 * dsa_indexer_kl_backward - gradients of sum_t kl[t] with respect to the
 * indexer's inputs, from G:
 *
 *   dw[t,j]   = sum_{s<=t} G[t,s] relu(S)
 *   dq_I[t,j] = w[t,j] sum_{s<=t} G[t,s] [S > 0] k_I[s]
 *   dk_I[s]   = sum_{t>=s} sum_j G[t,s] w[t,j] [S > 0] q_I[t,j]
 *   with S = q_I[t,j] . k_I[s] (exact in fp32 for the e4m3 inputs' range
 *   used here; the ReLU's derivative at 0 is 0).
 *
 *   G     [L][L]         fp32  (only s <= t is read)
 *   dq_I  [L][H_I][d_I]  fp32  OUT,  dk_I [L][d_I] fp32 OUT,  dw [L][H_I] fp32 OUT
 * G [S > 0] w is rounded to bf16 for the two products with k_I and q_I (fp32
 * accumulation); dw is fp32 throughout.  dk_I is summed over groups of heads
 * through the caller's workspace (dsa_indexer_kl_backward_workspace_size
 * bytes, 256-byte aligned), in a fixed order: results are bit-identical run
 * to run.  Supported: d_I in {64, 128}, 1 <= H_I <= 256, L * L < 2^31.
 * Errors: DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE.
 */
DSA_API size_t dsa_indexer_kl_backward_workspace_size(int64_t L, int H_I, int d_I);

DSA_API dsa_status_t dsa_indexer_kl_backward(const void* q_I, const void* k_I, const float* w,
                                     const float* G, int64_t L, int H_I, int d_I, float* dq_I,
                                     float* dk_I, float* dw, void* workspace,
                                     size_t workspace_bytes, int32_t* err, dsa_stream_t stream);

/*
 * dsa_check_device_error - synchronizes `stream`, then reads the device
 * error word `err` (a caller's word as passed to the launching calls, or
 * NULL for the current device's library word) into *code (DSA_DEVERR_*) and
 * sets it back to 0.  Returns DSA_OK if the word could be read (whatever its
 * value), DSA_ERR_INVALID_ARG for a NULL code or a misaligned err,
 * DSA_ERR_CUDA otherwise.
 */
DSA_API dsa_status_t dsa_check_device_error(int32_t* err, int* code, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */

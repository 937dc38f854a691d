/*
 * msa.h -- C ABI of libmsa: the hot path of MiniMax Sparse Attention (MSA)
 * on one NVIDIA B200 (sm_100a).
 *
 * The method (web pages, cited by title and section):
 *   [P2] "MiniMax M3模型算力成本大幅降低原因深度解析", sections "索引分支（Index
 *        Branch）" and "稀疏分支（Sparse Branch）": a lightweight single-head
 *        index key with block max-pooling screens the whole context and keeps
 *        the top-K KV blocks; standard GQA then runs over the kept blocks only,
 *        on raw KV.
 *   [P4] "MiniMax M3 深度实战 ...", section 2.2 "KV Outer Gather Q" (each KV
 *        block gathers the queries that selected it and is read once), section
 *        2.3 "MSA 算法实现" (the own/local block is always kept; softmax of
 *        Q K^T / sqrt(d_head) over the gathered keys), section 3.3 (decode:
 *        one new query, at the newest position).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or retains memory and (apart from the
 *    no-allocation decode entry point below) keeps no global mutable state,
 *    so calls on different workspaces may run concurrently.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on that stream and returns after enqueueing its kernels.
 *  - Layouts are row-major and contiguous, bf16 means IEEE bfloat16 bits:
 *        q_idx [Bt][n_q][d_idx]  bf16     k_idx [Bt][T][d_idx]   bf16
 *        q     [Bt][n_q][Hq][d]  bf16     k, v  [Bt][T][Hkv][d]  bf16
 *        ids   [Bt][n_q][K]      int32    out   [Bt][n_q][Hq][d] fp32
 *        lse   [Bt][n_q][Hq]     fp32
 *    Query i (0 <= i < n_q) of sequence b sits at position t = T - n_q + i of
 *    its length-T context (prefill: n_q = T; decode: n_q = 1).  Block j holds
 *    keys [j*block, min((j+1)*block, T)); N = ceil(T / block); own(t) = t / block.
 *  - Selection: ids[b][i] lists min(K, own(t)+1) distinct blocks in ascending
 *    order, padded with -1: the own block, plus the top min(K, own+1) - 1 of
 *    the blocks j < own(t) ranked by s(t,j) = max_{i in block j} q_idx[t].k_idx[i]
 *    (descending; ties go to the lower block index).  Scores are accumulated in
 *    fp32, which is exact for the integer-valued index keys of the pages'
 *    workloads (|s| < 2^24).
 *  - Attention: for each query head h (kv head h / (Hq/Hkv)), softmax of
 *    q.k_i / sqrt(d) over the keys i <= t of the blocks in ids, output the
 *    weighted sum of v_i (fp32) and lse = ln sum_i exp(q.k_i / sqrt(d)).
 *  - Supported shapes: d, d_idx in {64, 128}; block in {32, 64} or a
 *    multiple of 128; 1 <= K <= 32; 128 % (Hq/Hkv) == 0; N <= 8192;
 *    Bt*T < 2^31, Bt*n_q*K < 2^31 and Bt*n_q*Hq*d < 2^34 (the attention
 *    calls address q in 16-byte units with 32-bit offsets).  Anything else
 *    returns MSA_ERR_UNSUPPORTED before any work is enqueued.
 *  - Alignment (MSA_ERR_INVALID_ARG otherwise, nothing enqueued): q_idx,
 *    k_idx, q, k, v (and their paged stores) and out must be 16-byte aligned
 *    (they are read or written in 16-byte pieces); ids, lse, row_ptr,
 *    entries and page tables 4-byte aligned.
 *  - Errors found on the host return immediately (nothing enqueued).  Errors a
 *    kernel finds (an id outside [-1, N), a bounded wait that expired) are
 *    OR-ed into a sticky status word at the start of the workspace; kernels
 *    skip the offending work and never trap.  Read it with msa_device_status().
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum msa_status {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, n_q > T, Hq % Hkv != 0, K < 1 */
    MSA_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes listed above */
    MSA_ERR_WORKSPACE = 3,   /* workspace pointer null/misaligned or smaller than required */
    MSA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    MSA_ERR_TIMEOUT = 5,     /* device: a bounded wait inside a kernel expired */
    MSA_ERR_BAD_IDS = 6      /* device: an id outside [-1, N) was seen and skipped */
} msa_status;

/*
 * Bytes of device workspace that msa_index_topk, msa_select_invert and
 * msa_sparse_attn need for these sizes (the maximum over the three; a decode
 * shape, n_q == 1, needs far less than a prefill).  The workspace must be
 * 256-byte aligned.  Its first 256 bytes hold the sticky device status word:
 * zero them once before first use (e.g. cudaMemsetAsync(ws, 0, 256)).  The
 * rest is scratch that every call overwrites; two calls that overlap in time
 * must not share a workspace.  Returns 0 for arguments the calls would reject.
 *
 * Prefill attention keeps one bf16 partial (and its lse) per (query row,
 * slot, query head) until the log-sum-exp combine; it attends the kv heads in
 * groups and merges each group before the next, so the workspace holds one
 * group's partials.  msa_workspace_size returns the minimum: the largest
 * group (a divisor of Hkv) whose partials fit in about 4 GiB, at least one kv
 * head.  Given a larger workspace, msa_sparse_attn uses the largest group that
 * fits (fewer, longer launches); msa_workspace_size_kv_group gives the size
 * for kv_group kv heads per pass (kv_group = Hkv: a single pass), or 0 if
 * kv_group does not divide Hkv.
 */
MSA_API size_t msa_workspace_size(int Bt, int n_q, int T, int Hq, int Hkv, int d, int d_idx,
                                  int block, int K);

MSA_API size_t msa_workspace_size_kv_group(int Bt, int n_q, int T, int Hq, int Hkv, int d,
                                           int d_idx, int block, int K, int kv_group);

/*
 * Index branch [P2 "索引分支"]: block max-pooled single-head index scores and
 * top-K block selection with the own block forced.  Writes ids (layout above).
 * Prefill (n_q > 1) runs one fused tcgen05 kernel that never materialises the
 * n_q x T score matrix; decode (n_q == 1) streams k_idx once and selects.
 */
MSA_API msa_status msa_index_topk(const void *q_idx, const void *k_idx, int32_t *ids, int Bt,
                                  int n_q, int T, int d_idx, int block, int K, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * Index branch with signed 8-bit index keys: the same selection as
 * msa_index_topk (same layouts and rules) for q_idx [Bt][n_q][d_idx] and
 * k_idx [Bt][T][d_idx] stored as int8 instead of bf16.  The pages' index key
 * is lightweight ([P2 "索引分支"]) and the workloads' keys are small integers,
 * which int8 holds exactly; the scores are then integer dot products,
 * computed exactly (prefill: tcgen05 kind::i8 with s32 accumulation, twice
 * the bf16 tensor-core rate; decode: dp4a over half the bytes of bf16 keys),
 * so the ids equal those of msa_index_topk on the same integer values.
 * Keys that are not integers must go through msa_index_topk instead.
 */
MSA_API msa_status msa_index_topk_i8(const int8_t *q_idx, const int8_t *k_idx, int32_t *ids,
                                     int Bt, int n_q, int T, int d_idx, int block, int K,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * Selection inversion [P4 section 2.2]: the per-query block lists in ids
 * turned into per-block lists of hit queries, in CSR form over the Bt*N
 * (sequence, block) pairs:
 *   row_ptr [Bt*N + 1] int32: list of pair p = b*N + j is
 *           entries[row_ptr[p] .. row_ptr[p+1]);
 *   entries [Bt*n_q*K] int32 (capacity; row_ptr[Bt*N] are used): each entry
 *           is (b*n_q + i)*K + slot with ids[b][i][slot] == j, listed in
 *           ascending query order.
 * msa_sparse_attn performs the same inversion internally (into its
 * workspace); this entry point exposes it on its own.
 */
MSA_API msa_status msa_select_invert(const int32_t *ids, int32_t *row_ptr, int32_t *entries,
                                     int Bt, int n_q, int T, int block, int K, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Sparse branch [P2 "稀疏分支"; P4 sections 2.2, 2.3]: exact GQA softmax
 * attention over the keys of the selected blocks (causal inside the own block),
 * scale 1/sqrt(d), raw bf16 KV.  Writes out and lse (layouts above).
 * ids must hold, per row, distinct block ids in [0, N) or -1; an id greater
 * than own(t) contributes no key; an id outside [-1, N) is skipped (it
 * contributes no key either) and reported as MSA_ERR_BAD_IDS.  Prefill (n_q > 1): inversion, a
 * KV-block-outer tcgen05 kernel that loads each selected KV block into shared
 * memory and gathers its hit queries, then a log-sum-exp combine of the per
 * slot partials.  With blocks longer than 128 keys, each row's own block is
 * left out of the hit lists and attended by a second, causal launch of the
 * kernel over the consecutive rows of each block, which skips the 128-key
 * sub-tiles past each chunk's last row.  Decode (n_q == 1): a split-K kernel
 * over the selected blocks, then the same combine.
 */
MSA_API msa_status msa_sparse_attn(const void *q, const void *k, const void *v,
                                   const int32_t *ids, float *out, float *lse, int Bt, int n_q,
                                   int T, int Hq, int Hkv, int d, int block, int K,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Paged KV for decode [P4 section 3.2, "MSA 如何降低显存压力": page-managed
 * KV cache; its 4-bit quantisation is not followed, KV stays raw bf16].
 * Same computation as msa_index_topk / msa_sparse_attn for a decode step
 * (n_q = 1, the query at t = T-1), with k_idx, K and V held in pages of
 * `block` rows instead of contiguous [Bt][T] rows:
 *   page_table  [Bt][page_stride] int32 (device): logical block j of
 *               sequence b is physical page page_table[b*page_stride + j],
 *               for j < N = ceil(T / block); page_stride >= N.
 *   k_idx_pages [num_pages][block][d_idx] bf16;
 *   k_pages, v_pages [num_pages][block][Hkv][d] bf16 (16-byte aligned).
 * Rows past T in the last logical block are never read.  The caller owns
 * all buffers; the workspace is msa_workspace_size(Bt, 1, T, ...).  A page id
 * outside [0, num_pages) is skipped and reported as MSA_ERR_BAD_IDS through
 * the status word (msa_device_status).  Host-detected errors as above.
 */
MSA_API msa_status msa_index_topk_paged(const void *q_idx, const void *k_idx_pages,
                                        const int32_t *page_table, int page_stride,
                                        int num_pages, int32_t *ids, int Bt, int T, int d_idx,
                                        int block, int K, void *workspace,
                                        size_t workspace_bytes, void *stream);

MSA_API msa_status msa_sparse_attn_paged(const void *q, const void *k_pages, const void *v_pages,
                                         const int32_t *page_table, int page_stride,
                                         int num_pages, const int32_t *ids, float *out,
                                         float *lse, int Bt, int T, int Hq, int Hkv, int d,
                                         int block, int K, void *workspace,
                                         size_t workspace_bytes, void *stream);

/*
 * Instrumented variants (profiling): the same work as msa_index_topk and
 * msa_sparse_attn, with optional CUDA events recorded on `stream`
 * immediately before (start[i]) and after (stop[i]) the kernels of stage i.
 * Each non-NULL entry must be a cudaEvent_t created on the current device;
 * `events` itself may be NULL.  Stages:
 *   msa_index_topk_ev, msa_index_topk_i8_ev:
 *                       0 = index kernel (prefill) or k_idx scan (decode);
 *                       1 = top-K select (decode only).
 *   msa_sparse_attn_ev: 0 = selection inversion (prefill only);
 *                       1 = attention kernel (KV-block-outer: the hit-list
 *                           launch and, for blocks longer than 128 keys, the
 *                           own-block launch; or split-K);
 *                       2 = log-sum-exp combine.
 *   A prefill that attends its kv heads in several groups (see
 *   msa_workspace_size) records stage 1 from the first group's attention to
 *   the last group's, which spans the combines of all groups but the last,
 *   and stage 2 around the last group's combine.
 */
#define MSA_MAX_STAGES 4
typedef struct msa_stage_events {
    void *start[MSA_MAX_STAGES];
    void *stop[MSA_MAX_STAGES];
} msa_stage_events;

MSA_API msa_status msa_index_topk_ev(const void *q_idx, const void *k_idx, int32_t *ids, int Bt,
                                     int n_q, int T, int d_idx, int block, int K,
                                     void *workspace, size_t workspace_bytes, void *stream,
                                     const msa_stage_events *events);

MSA_API msa_status msa_index_topk_i8_ev(const int8_t *q_idx, const int8_t *k_idx, int32_t *ids,
                                        int Bt, int n_q, int T, int d_idx, int block, int K,
                                        void *workspace, size_t workspace_bytes, void *stream,
                                        const msa_stage_events *events);

MSA_API msa_status msa_sparse_attn_ev(const void *q, const void *k, const void *v,
                                      const int32_t *ids, float *out, float *lse, int Bt,
                                      int n_q, int T, int Hq, int Hkv, int d, int block, int K,
                                      void *workspace, size_t workspace_bytes, void *stream,
                                      const msa_stage_events *events);

/*
 * Decode attention that allocates nothing.  The pages have no counterpart:
 * this entry point is an addition of this library for callers that cannot
 * allocate device memory or hand over a workspace -- for example a serving
 * engine or plugin host that has already given all device memory to its own
 * pool, where a cudaMalloc would fail or stall the whole device, and which
 * has no spare buffer to pass as workspace.
 *
 * It computes exactly what msa_sparse_attn computes for a decode step (n_q = 1,
 * same layouts, same split-K and combine kernels), but its scratch (the
 * per-split partials) is a file-scope static __device__ array of
 * MSA_NOALLOC_SCRATCH_BYTES (16 MiB).  That array is part of the library
 * image: every GPU on which it has been loaded holds it until the process
 * exits.  The caller still owns and passes every input and output.
 *   - Limit: 256 + align256(Bt*K*S*Hq*d*4) + align256(Bt*K*S*Hq*4) bytes must
 *     fit in the array, with S = ceil(block / 64); otherwise the call returns
 *     MSA_ERR_WORKSPACE before enqueueing anything.  (The 4-sequence
 *     1M-context decode, Bt 4, K 8, block 512, Hq 64, d 128, needs 8.5 MB.)
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any
 *     stream capture begins.  The cached address belongs to the device's
 *     primary context: after cudaDeviceReset, or when calling from another
 *     driver context on the same device, it is stale and must not be used.
 *   - Every call uses the same array, which keeps the contents of the last
 *     call.  Calls whose kernels overlap on the GPU (two streams, or two host
 *     threads) race on it and must be serialised by the caller.
 *   - status: optional device int.  Kernels OR 2 into it when they skip an id
 *     outside [-1, N).  With NULL those reports are dropped.
 * No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define MSA_NOALLOC_SCRATCH_BYTES (16u << 20)

MSA_API msa_status msa_sparse_attn_decode_noalloc(const void *q, const void *k, const void *v,
                                                  const int32_t *ids, float *out, float *lse,
                                                  int Bt, int T, int Hq, int Hkv, int d,
                                                  int block, int K, int *status, void *stream);

/*
 * Synchronises `stream`, then reads and clears the sticky device status word
 * of `workspace`: MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_BAD_IDS (the first found,
 * in that order of precedence: timeout first), or MSA_ERR_CUDA if the
 * synchronisation or the copy failed.
 */
MSA_API msa_status msa_device_status(void *workspace, void *stream);

/* Static, NUL-terminated name of a status code ("unknown status" otherwise). */
MSA_API const char *msa_status_string(int status);

/*
 * Tensor-core self-test, not part of the method: C[128][N] = A . B with
 * A [128][Kd] bf16 (K-major) and B either as [N][Kd] (bit 0 of b_mn_major = 0,
 * K-major) or as [Kd][N] (bit 0 = 1), C fp32, through the same TMA,
 * shared-memory descriptor, tcgen05.mma and TMEM read-back code the attention
 * kernels use.  Bit 1 of b_mn_major set: A is first copied into tensor memory
 * and the MMA reads it from there (the layout the attention kernel uses for P).
 * N in {64, 128, 256}, Kd a multiple of 64 up to 256.  Device pointers;
 * `status` is a device int the kernel sets non-zero on a wait timeout.
 */
MSA_API msa_status msa_selftest_umma(const void *A, const void *B, float *C, int N, int Kd,
                                     int b_mn_major, int *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */

/*
 * msa.h - C ABI of the Memory Sparse Attention (MSA) hot path on NVIDIA B200.
 *
 * The method ("MSA: Memory Sparse Attention for Efficient End-to-End Memory
 * Model Scaling to 100M Tokens") serves a memory of N documents in three
 * stages (IRMaD reading, "M. Materials & Methods", three-stage inference item;
 * project overview, "three-stage inference pipeline" figure):
 *   1. offline encoding: K = H W_K with document-wise RoPE, V = H W_V,
 *      K^R = H W^KR, each mean-pooled over 64-token chunks that never cross a
 *      document boundary -> K̄, V̄, K̄^R;
 *   2. online routing: Q^R = H_q W^QR, chunk score = head-mean cosine against
 *      every K̄^R, document score = max over its chunks, top-k documents;
 *   3. sparse generation: GQA decode attention over [selected docs' K̄; local K]
 *      with global RoPE offset by k on the active context.
 *
 * Conventions for every call
 *   - Return an msa_status; no exception or abort crosses the ABI.  The message
 *     of the last failure on the calling thread is msa_last_error().
 *   - Tensor arguments are DEVICE pointers owned by the caller, unless the
 *     comment says host.  bf16 tensors are passed as void* and hold IEEE
 *     bfloat16 bit patterns.  Layouts are dense row-major; the memory tensors
 *     are chunk-major [C, heads, dim].
 *   - The library allocates no device memory.  Scratch comes from the caller's
 *     workspace `ws` of at least msa_*_workspace_size(...) bytes (256-byte
 *     aligned).  `ws` may be NULL only if that size is 0.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Arguments are validated on the host before any
 *     launch; a call that returns an error has launched nothing.  Errors raised
 *     by the device surface at the caller's next synchronisation, or through
 *     msa_check_device_errors().
 *   - Every tensor pointer must be 16-byte aligned (MSA_ERR_INVALID_ARG).
 *   - Device-resident index arrays (doc_off, chunk_off, topk_idx, loc_len) must
 *     hold what their comments say (monotone offsets, ids in range); they are
 *     read on the device and cannot be checked on the host.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1, /* bad size, pointer, alignment or value */
  MSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim not 64/128) */
  MSA_ERR_WORKSPACE = 3,   /* ws_bytes smaller than the matching *_workspace_size */
  MSA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed; see msa_last_error() */
  MSA_ERR_TIMEOUT = 5,     /* a bounded wait gave up (device error word set) */
} msa_status;

/* Model dimensions of one routed layer.  hidden = width of H; n_q / n_kv =
 * query / key-value heads (GQA, n_q a multiple of n_kv, n_kv <= 8, n_q / n_kv <= 16);
 * head_dim in {64, 128}; n_r router heads of dim d_r in {64, 128}, n_r <= 8;
 * chunk = tokens per pooled chunk (P, 64 on the pages); rope_base = RoPE base. */
typedef struct {
  int32_t hidden;
  int32_t n_q;
  int32_t n_kv;
  int32_t head_dim;
  int32_t n_r;
  int32_t d_r;
  int32_t chunk;
  float rope_base;
} msa_dims;

/* Document score from its chunk scores: max over chunks (the pages' s_i =
 * max_j S_ij) or the mean (an alternative reading; see routing notes). */
typedef enum { MSA_AGG_MAX = 0, MSA_AGG_MEAN = 1 } msa_doc_agg;

/* Thread-local message of the last failing call on this thread ("" if none). */
const char* msa_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int32_t msa_version(void);

/* Reads and clears the device error word of the current device (bit 0: a
 * bounded wait gave up; bit 1: a device-side index was out of range).
 * Synchronises the device.  *bits_out may be NULL. */
msa_status msa_check_device_errors(uint32_t* bits_out);

/* Self-test of the library's bounded device waits (failure handling; the paper has
 * no counterpart).  Launches one CTA whose four warps each wait n_waits times, with
 * a limit of limit_us microseconds per wait, on an mbarrier that nothing ever
 * arrives on; no copy or tensor-core operation is outstanding.  The first wait
 * that gives up sets bit 0 of the device error word (msa_check_device_errors then
 * returns MSA_ERR_TIMEOUT) and the CTA's abort flag; every other wait of the CTA
 * then returns at once, as in the library's pipelined kernels, so the kernel ends
 * after about one limit, not n_waits of them.  elapsed_ns: [1] device uint64 out,
 * the kernel's wall time in ns.  Limits: 1 <= limit_us <= 100000, 1 <= n_waits <= 1000. */
msa_status msa_selftest_wait_timeout(int32_t limit_us, int32_t n_waits, uint64_t* elapsed_ns, void* stream);

/* ---------------------------------------------------------------------------
 * Stage 1 - chunk layout (host helper).
 * Pages: digest "Method step details", Stage 1 (chunk mean pooling, P = 64);
 * chunks never cross a document boundary, the last chunk of a document holds
 * the remaining L mod P tokens.
 *   doc_off_host   [n_docs + 1] host, int64 token offsets, doc_off[0] = 0,
 *                  strictly increasing (every document has >= 1 token).
 *   chunk_off_host [n_docs + 1] host, out: chunk_off[i+1] = chunk_off[i] +
 *                  ceil((doc_off[i+1] - doc_off[i]) / chunk).
 *   n_chunks_out   host, out: C = chunk_off[n_docs] (< 2^31).
 * ------------------------------------------------------------------------- */
msa_status msa_chunk_offsets(const int64_t* doc_off_host, int32_t n_docs, int32_t chunk,
                             int32_t* chunk_off_host, int32_t* n_chunks_out);

/* ---------------------------------------------------------------------------
 * Stage 1 - offline memory encoding.
 * Pages: IRMaD "M. Materials & Methods", routing item (K = H W_K, V = H W_V,
 * K^R = H W^KR, K̄ = φ(K), V̄ = φ(V), K̄^R = φ(K^R)) and position item
 * (document-wise RoPE: positions restart at 0 in every document).
 *   H        [T, hidden] bf16, the layer's hidden states of the whole corpus.
 *   doc_off  [n_docs + 1] device int64 token offsets (as msa_chunk_offsets).
 *   chunk_off[n_docs + 1] device int32 chunk offsets from msa_chunk_offsets.
 *   W_K, W_V [hidden, n_kv * head_dim] bf16; W_KR [hidden, n_r * d_r] bf16.
 *   K_bar, V_bar [C, n_kv, head_dim] bf16 out: chunk means of RoPE(H W_K) at
 *            document-relative positions and of H W_V.
 *   KR_bar   bf16 out: chunk means of H W^KR, [C, n_r, d_r] (kr_layout 0) or
 *            head-major [n_r, C, d_r] (kr_layout 1, the layout the scan reads best).
 * Requirements: hidden % 64 == 0; n_kv * head_dim and n_r * d_r multiples of
 * 128; chunk == 64; T < 2^31 - 64.  Rounding: fp32 accumulation, outputs rounded to bf16.
 * ------------------------------------------------------------------------- */
size_t msa_encode_workspace_size(const msa_dims* dims, int64_t T, int32_t n_docs, int32_t n_chunks);
msa_status msa_encode_memory(const msa_dims* dims, const void* H, int64_t T, const int64_t* doc_off,
                             int32_t n_docs, const int32_t* chunk_off, int32_t n_chunks, const void* W_K,
                             const void* W_V, const void* W_KR, void* K_bar, void* V_bar, void* KR_bar,
                             int32_t kr_layout, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Incremental memory append: encode new documents behind an existing memory.
 * Pages: IRMaD "M. Materials & Methods", three-stage inference item (1) (the
 * memory is encoded offline, document by document, and cached); paper digest,
 * "limitations and improvements" section, future directions (streaming memory
 * updates by incremental encoding instead of re-encoding the corpus).  Because
 * positions restart at 0 in every document and chunks never cross documents,
 * the new documents' pooled rows do not depend on the existing ones: appending
 * gives bit for bit the rows a full msa_encode_memory of all documents gives.
 *   H_new [T_new, hidden], doc_off_new [n_docs_new + 1] (device int64, relative
 *            to H_new), chunk_off_new [n_docs_new + 1] (device int32, relative),
 *            n_chunks_new: the new documents alone, as for msa_encode_memory.
 *   K_bar, V_bar [chunk_capacity, n_kv, head_dim], KR_bar [chunk_capacity, n_r, d_r]
 *            chunk-major bf16: rows n_chunks_old .. n_chunks_old + n_chunks_new - 1
 *            are written, earlier rows are left alone.
 *   chunk_off  device int32 [n_docs_old + n_docs_new + 1], the whole memory's
 *            chunk offsets: entries n_docs_old .. n_docs_old + n_docs_new are
 *            written (n_chunks_old + chunk_off_new[i]).
 *   ws, ws_bytes  as msa_encode_workspace_size(dims, T_new, n_docs_new, n_chunks_new).
 * Errors: MSA_ERR_INVALID_ARG when n_chunks_old + n_chunks_new > chunk_capacity;
 * otherwise those of msa_encode_memory.  Stream-ordered; no host synchronisation.
 * ------------------------------------------------------------------------- */
msa_status msa_append_memory(const msa_dims* dims, const void* H_new, int64_t T_new, const int64_t* doc_off_new,
                             int32_t n_docs_new, const int32_t* chunk_off_new, int32_t n_chunks_new,
                             const void* W_K, const void* W_V, const void* W_KR, void* K_bar, void* V_bar,
                             void* KR_bar, int32_t chunk_capacity, int32_t* chunk_off, int32_t n_docs_old,
                             int32_t n_chunks_old, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Stage 2 - online routing and top-k.
 * Pages: IRMaD "M. Materials & Methods", routing item:
 *   Q^R = H_q W^QR;  S_ij = max_t mean_h cos(Q^R_h, K̄^R_ij,h);
 *   s_i = max_j S_ij;  I = Top-k({s_i});  k = 16 on the pages.
 *   q_tokens M >= 1 tokens per query (the t of max_t): row b * M + t of Hq is
 *            token t of query b.  A query's chunk score is the largest over its
 *            tokens of the head-mean cosine.
 *   Hq       [B * M, hidden] bf16 query hidden states, or, when W_QR == NULL,
 *            [B * M, n_r * d_r] bf16 router queries Q^R given directly.
 *   W_QR     [hidden, n_r * d_r] bf16 or NULL.
 *   KR_bar   pooled router keys, bf16: [n_chunks, n_r, d_r] for kr_layout 0, or
 *            head-major [n_r, n_chunks, d_r] for kr_layout 1 (each head's keys contiguous:
 *            the scan then streams whole 32 KB slices instead of 256-byte pieces).
 *            kr_layout | MSA_ROUTE_EARLY_INPUTS: the router query reads H_q and W_QR and
 *            multiplies them, and the scan starts streaming KR_bar, before the preceding work
 *            on the stream has finished (the writes still wait for it).  The caller
 *            guarantees that H_q, W_QR, KR_bar, kr_inv_norm and chunk_off are not written by
 *            the work immediately preceding this call on the stream, and that this work is a
 *            call of this library, a copy, or a kernel that does not start its dependents
 *            early (programmatic dependent launch).  The result is the same as without it.
 *   chunk_off[n_docs + 1] device int32 chunk offsets of the documents.
 *   kr_inv_norm  optional [n_chunks, n_r] fp32 from msa_router_key_norms: the keys'
 *            inverse norms, computed once offline; NULL = computed during the scan
 *            (the same values: both square-sum the stored bf16 keys in fp32).
 *   doc_scores [B, n_docs] fp32 out, optional (NULL = not written).
 *   topk_idx [B, k] int32 out: document ids, descending score, ties to the
 *            lower id.  topk_score [B, k] fp32 out: their scores.
 * Cosines use norms clamped below at 1e-12 (a zero vector scores 0).
 * Limits: 1 <= k <= min(n_docs, 256); 1 <= B; 1 <= M; B * M <= 65535; n_r <= 8;
 * d_r in {64, 128}.
 * Rounding: Q^R in fp32; the cosine dot products run on the tensor cores with
 * the normalised query split into two bf16 terms (hi + lo) and fp32
 * accumulation, so scores carry ~1e-6 relative error.
 * ------------------------------------------------------------------------- */
#define MSA_ROUTE_EARLY_INPUTS 16
size_t msa_route_workspace_size(const msa_dims* dims, int32_t B, int32_t q_tokens, int32_t n_docs,
                                int32_t n_chunks, int32_t k, msa_doc_agg agg);
msa_status msa_route_topk(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B, int32_t q_tokens,
                          const void* KR_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks,
                          int32_t k, msa_doc_agg agg, int32_t kr_layout, const float* kr_inv_norm,
                          float* doc_scores, int32_t* topk_idx,
                          float* topk_score, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Inverse norms of the pooled router keys (offline, once per memory).
 * Pages: IRMaD "M. Materials & Methods", routing item (the cosine divides by the
 * norm of every pooled router key; the keys are fixed once the memory is
 * encoded).  kr_inv_norm[j, h] = 1 / max(||K̄^R_{j,h}||, 1e-12), the norm square-
 * summed in fp32 from the stored bf16 values.  Passing the result to
 * msa_route_topk spares the scan its per-chunk norm work.
 *   KR_bar   [n_chunks, n_r, d_r] (kr_layout 0) or [n_r, n_chunks, d_r] (kr_layout 1) bf16.
 *   kr_inv_norm [n_chunks, n_r] fp32 device out.
 * ------------------------------------------------------------------------- */
msa_status msa_router_key_norms(const msa_dims* dims, const void* KR_bar, int32_t n_chunks, int32_t kr_layout,
                                float* kr_inv_norm, void* stream);

/* ---------------------------------------------------------------------------
 * Merge of top-k candidates (memory-parallel routing).
 * Pages: IRMaD "M. Materials & Methods", Memory Parallel item; EverMind article
 * 2.3: the router keys are sharded over GPUs, the query is broadcast, every GPU
 * scores its shard and a global reduction picks the top-k documents.  After
 * each rank's msa_route_topk on its shard and an exchange of the B x k_local
 * (score, global document id) pairs, this call selects the global top-k.
 *   cand_score [B, n_cand] fp32, cand_idx [B, n_cand] int32 global ids (device).
 *   topk_idx [B, k], topk_score [B, k] out: descending score, ties to the lower id
 *   (the same order as msa_route_topk on the unsharded memory).
 * Limits: 1 <= k <= min(n_cand, 256), n_cand <= 24576.
 * ------------------------------------------------------------------------- */
msa_status msa_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t B, int32_t n_cand, int32_t k,
                          int32_t* topk_idx, float* topk_score, void* stream);

/* ---------------------------------------------------------------------------
 * msa_route_topk_static - msa_route_topk without a caller workspace.
 * The paper has no counterpart: this is a convenience of this library.
 * For callers that cannot allocate device memory where they route: a host
 * program that embeds the library as a plugin without a CUDA allocator, code
 * running while a stream is captured into a CUDA graph (cudaMalloc is not
 * allowed there), or a loop that must not pay cudaMalloc's implicit device
 * synchronisation.  Same arguments and results as msa_route_topk with
 * kr_layout 0 (chunk-major K̄^R [n_chunks, n_r, d_r]) and kr_inv_norm NULL
 * (the scan computes the key norms), minus ws/ws_bytes; the arguments are
 * checked as msa_route_topk checks them and give the same status.  The scratch
 * is a library-owned device array of 8 MiB (8388608 bytes) that every GPU
 * loading the library holds until the process exits; a problem whose
 * msa_route_workspace_size exceeds it is rejected with MSA_ERR_WORKSPACE
 * before any launch.  The first call on a device (with that device current)
 * looks up the array's address once, and again after the device's context has
 * been destroyed and re-created (cudaDeviceReset); make those calls before any
 * stream capture.  All calls on a device share the array, so calls whose work
 * overlaps on the GPU race: order them on one stream.  No cudaMalloc, cudaFree
 * or allocating library routine is called.
 * ------------------------------------------------------------------------- */
msa_status msa_route_topk_static(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B,
                                 int32_t q_tokens, const void* KR_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks,
                                 int32_t k, msa_doc_agg agg, float* doc_scores, int32_t* topk_idx,
                                 float* topk_score, void* stream);

/* ---------------------------------------------------------------------------
 * Router training: the contrastive auxiliary loss and its gradients.
 * Pages: IRMaD "M. Materials & Methods", training item:
 *   L_aux = -(1/|P|) sum_i log( exp(s_i^+/tau) / (exp(s_i^+/tau) + sum_j exp(s_ij^-/tau)) ),
 * applied to every layer's router (the digest's "Core method": it supervises the
 * routing decision that top-k alone cannot pass a gradient through).  Reading: a
 * score s is the routing score of a chunk, the head mean of the cosines between
 * the router query and the chunk's pooled router key (one query token).
 *   QR       [P, n_r, d_r] bf16 router queries, one per positive.
 *   K_pos    [P, n_r, d_r] bf16 pooled router key of each positive chunk.
 *   K_neg    [P, N, n_r, d_r] bf16 pooled router keys of its N negatives (NULL if N = 0).
 *   tau      temperature, > 0.
 *   loss     [1] fp32 device out.
 *   grad_QR, grad_K_pos [P, n_r, d_r], grad_K_neg [P, N, n_r, d_r] fp32 device out;
 *            each optional (NULL = not computed).
 *   ws       >= msa_aux_loss_workspace_size bytes, 256-byte aligned.
 * A norm below 1e-12 is clamped (cosine 0 for a zero vector) and contributes no
 * gradient through the clamp.  fp32 arithmetic throughout; the loss is summed
 * in positive order, independent of scheduling.
 * Limits: 1 <= P <= 2^20; 0 <= N <= 1023; n_r <= 8; d_r in {64, 128}.
 * ------------------------------------------------------------------------- */
size_t msa_aux_loss_workspace_size(const msa_dims* dims, int32_t P, int32_t N);
msa_status msa_aux_loss(const msa_dims* dims, const void* QR, const void* K_pos, const void* K_neg, int32_t P,
                        int32_t N, float tau, float* loss, float* grad_QR, float* grad_K_pos, float* grad_K_neg,
                        void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Stage 3 - sparse generation attention (one decode step).
 * Pages: IRMaD "M. Materials & Methods", routing item (K_ctx = [{K̄_i}_{i in I};
 * K_q], V_ctx likewise, Output = Attention(Q_q, K_ctx, V_ctx)) and position item
 * (global RoPE on the active context, offset by k); project overview "key
 * technical details" 1.
 *   q_tokens M >= 1 query tokens per query: the last M local tokens (M = 1 is
 *            the decode step; M > 1 the query-prefill step of the same call).
 *   q        [B, M, n_q, head_dim] bf16, before RoPE; token t is rotated to
 *            position pos_offset + loc_len[b] - M + t (the query tokens are the
 *            last M local tokens).
 *   K_bar, V_bar [n_chunks, n_kv, head_dim] bf16 pooled memory (device).
 *   chunk_off[n_docs + 1] device int32; topk_idx [B, k] device int32 doc ids.
 *   K_loc, V_loc [B, t_loc_max, n_kv, head_dim] bf16 local KV, K before RoPE;
 *            local token j is rotated to position pos_offset + j.
 *   loc_len  [B] device int32, 0 <= loc_len[b] <= t_loc_max.
 *   rope_cache  optional table from msa_rope_cache_build (NULL = built in ws).
 *   k_loc_rotated  0: K_loc holds keys before RoPE (rotated here, as above);
 *              1: K_loc already holds every local key rotated at pos_offset + j
 *              (see msa_rope_rows); rope_cache is then unused.
 *   softmax_scale  0 -> 1/sqrt(head_dim).
 *   phase    0: the whole call.  1 and 2 split it in two so that the local part can run
 *            while the query is still being routed: phase 1 attends over the local keys
 *            only and leaves its partial results in ws (topk_idx, K_bar, V_bar, chunk_off
 *            and out are not read and may be NULL); phase 2, with the same ws and sizes,
 *            attends over the selected chunks and merges both parts into out (K_loc and
 *            V_loc are not read).  Phase 2 must be ordered after phase 1 (same stream, or
 *            an event).  The result equals phase 0's bit for bit (the same work items and
 *            partial slots).
 *            phase | MSA_ATTEND_EARLY_LOCAL (phases 0 and 1): the work on the local keys may
 *            start before the preceding work on the stream has finished (typically
 *            msa_route_topk producing topk_idx), hiding it behind the routing.  The caller
 *            guarantees that q, K_loc, V_loc, loc_len, chunk_off (and rope_cache) are not
 *            written by the work immediately preceding this call on the stream, that this
 *            work does not use this workspace, and that it is a call of this library, a
 *            copy, or a kernel that does not start its dependents early (programmatic
 *            dependent launch).  The flag has no effect when the call builds its own
 *            rotation table (k_loc_rotated 0 and rope_cache NULL).  The result is the same
 *            as without the flag.
 *   k_new, v_new  optional [B, n_kv, head_dim] bf16 (both or neither; M = 1; not phase 2):
 *            the decode step's new token, the query's own key (before RoPE) and value.
 *            The call first writes them at slot loc_len[b] - 1 of K_loc / V_loc (the key
 *            rotated at pos_offset + slot when k_loc_rotated is 1, as msa_kv_append does;
 *            unrotated otherwise) and attends over the cache as written: the same result
 *            as msa_kv_append followed by this call, one launch fewer.  K_loc and V_loc are
 *            then written (a loc_len of 0 raises the device error bit 1 and writes nothing).
 *   out      [B, M, n_q, head_dim] bf16.
 * Limits: 1 <= M, B * M <= 65535.
 * Query head g attends with KV head g / (n_q / n_kv).  Every query token sees
 * every gathered chunk; token t sees the local tokens j <= loc_len[b] - M + t
 * (causal; for M = 1 that is every local token).  Pooled keys keep their
 * document-wise rotation only.  Rounding: q is rotated and scaled in
 * fp32 then rounded to bf16; local keys are rotated in fp32 and rounded to
 * bf16; products and softmax in fp32.
 * ------------------------------------------------------------------------- */
#define MSA_ATTEND_EARLY_LOCAL 16
size_t msa_attend_workspace_size(const msa_dims* dims, int32_t B, int32_t q_tokens, int32_t k,
                                 int32_t t_loc_max, int32_t pos_offset);
msa_status msa_sparse_attend(const msa_dims* dims, const void* q, int32_t B, int32_t q_tokens, const void* K_bar,
                             const void* V_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks,
                             const int32_t* topk_idx, int32_t k, void* K_loc, void* V_loc,
                             const void* k_new, const void* v_new,
                             const int32_t* loc_len, int32_t t_loc_max, int32_t pos_offset,
                             const void* rope_cache, int32_t k_loc_rotated, float softmax_scale, int32_t phase,
                             void* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Memory-parallel attention: one rank's share, and the merge of the ranks' shares.
 * Pages: IRMaD "M. Materials & Methods", Memory Parallel and tiered storage item;
 * EverMind article 2.3: the memory is sharded over GPUs by documents; after the
 * global top-k (msa_topk_merge) every rank attends over the selected documents it
 * holds and the partial results are reduced into the one softmax over
 * [selected documents' K̄; local K].
 * msa_sparse_attend_share: msa_sparse_attend (phase 0, no fused append) over this
 * rank's shard, with
 *   chunk_off [n_docs + 1], K_bar, V_bar  the shard's documents doc_base ..
 *            doc_base + n_docs - 1 (chunk offsets rebased to the shard's first chunk);
 *   topk_idx [B, k] GLOBAL document ids (the same array on every rank); ids outside
 *            the shard are skipped (no error);
 *   local_keys  1 on the one rank that attends over the local keys (K_loc, V_loc),
 *            0 elsewhere (K_loc, V_loc may be NULL); loc_len and t_loc_max are given on
 *            every rank: they place the query tokens (pos_offset + loc_len - M + t);
 *   o_share  [B, M, n_q, head_dim] fp32 out: the share's softmax-weighted values
 *            (normalised over the share's own keys; 0 for a share with no key);
 *   lse2_share [B, M, n_q] fp32 out: log2 of the share's softmax denominator of the
 *            scaled logits, sum_j 2^(scale log2(e) q.k_j) (-inf for no key).
 * msa_attend_merge: out [rows, head_dim] bf16 = sum_r 2^(lse2_r - L) o_r with
 *   L = log2 sum_r 2^lse2_r, for R shares laid out o_shares [R, rows, head_dim],
 *   lse2_shares [R, rows] fp32 (rows = B * M * n_q); shares are added in rank order,
 *   so every rank computes the same bits.  A row with no key anywhere gives 0.
 * The merged result equals msa_sparse_attend over the unsharded memory up to fp32
 * rounding of the reduction (the split-KV combine already merges partial softmaxes).
 * ------------------------------------------------------------------------- */
msa_status msa_sparse_attend_share(const msa_dims* dims, const void* q, int32_t B, int32_t q_tokens, const void* K_bar,
                                   const void* V_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks,
                                   int32_t doc_base, const int32_t* topk_idx, int32_t k, int32_t local_keys,
                                   const void* K_loc, const void* V_loc, const int32_t* loc_len, int32_t t_loc_max,
                                   int32_t pos_offset, const void* rope_cache, int32_t k_loc_rotated,
                                   float softmax_scale, float* o_share, float* lse2_share, void* ws, size_t ws_bytes,
                                   void* stream);
msa_status msa_attend_merge(const float* o_shares, const float* lse2_shares, int32_t R, int32_t rows,
                            int32_t head_dim, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * Host tier: gather the selected documents' pooled K̄/V̄ from pinned host memory.
 * Pages: IRMaD "M. Materials & Methods", Memory Parallel and tiered storage
 * item; EverMind article 2.3: the content K̄/V̄ live in host DRAM and only the
 * top-k documents are loaded, asynchronously, after routing.
 *   K_bar_host, V_bar_host [n_chunks, n_kv, head_dim] bf16 in pinned (page-locked,
 *            device-mapped) host memory; read by the GPU over the bus.
 *   chunk_off [n_docs + 1], topk_idx [B, k] device int32 (msa_route_topk's output).
 *   K_stage, V_stage  device out, room for capacity_chunks rows each: the chunks of
 *            query b's r-th document land as staged document b * k + r.
 *   stage_chunk_off [B * k + 1] device out: chunk offsets of the staged documents.
 *   stage_topk_idx  [B, k] device out: b * k + r.
 *   ws       device workspace, >= B * k * 4 bytes, 256-byte aligned.
 * msa_sparse_attend(K_stage, V_stage, stage_chunk_off, B * k docs, stage_topk_idx, ...)
 * then attends exactly as over the device-resident memory.  The call needs no
 * host synchronisation (the indices stay on the device); enqueue it on a side
 * stream to overlap the host-to-device traffic with other work.  If the
 * selection needs more than capacity_chunks rows, only what fits is staged and
 * the device error word reports it.
 * ------------------------------------------------------------------------- */
msa_status msa_gather_kv(const msa_dims* dims, const void* K_bar_host, const void* V_bar_host, int32_t n_chunks,
                         const int32_t* chunk_off, int32_t n_docs, const int32_t* topk_idx, int32_t B, int32_t k,
                         void* K_stage, void* V_stage, int32_t capacity_chunks, int32_t* stage_chunk_off,
                         int32_t* stage_topk_idx, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Tiered decode: routing, host-tier gather and sparse attention of several
 * layers in one call, the gather of each layer overlapped with the routing of
 * the next.
 * Pages: IRMaD "M. Materials & Methods", Memory Parallel and tiered storage
 * item (router keys K̄^R resident on the GPU, content K̄/V̄ in host DRAM, loaded
 * asynchronously once the top-k documents are known) and three-stage inference
 * item (stages 2 and 3 per layer); EverMind article 2.3.
 * One msa_layer per layer instance (all pointers as in the single calls):
 *   Hq, W_QR, KR_bar, kr_inv_norm   as msa_route_topk (chunk-major K̄^R);
 *   K_bar_host, V_bar_host          [n_chunks, n_kv, head_dim] bf16, pinned host
 *                                   (as msa_gather_kv);
 *   q, K_loc, V_loc, k_new, v_new   as msa_sparse_attend with k_loc_rotated = 1
 *                                   (the local cache holds rotated keys; k_new /
 *                                   v_new both NULL or both set: the fused append);
 *   topk_idx, topk_score, out       outputs: [B, k] int32, [B, k] fp32 and
 *                                   [B, n_q, head_dim] bf16.
 * `layers` is a host array of n_layers entries.  The layers are independent
 * instances: no layer reads what another layer of the call writes (its inputs
 * must not alias another layer's outputs or local cache).  They share the
 * document layout (chunk_off, n_docs, n_chunks), B, k, loc_len, t_loc_max and
 * pos_offset.  Per layer l the call enqueues msa_route_topk (agg MAX),
 * msa_gather_kv of the routed documents into one of two staging areas in ws,
 * and msa_sparse_attend over the staged documents and the local keys, on two
 * streams joined by events, in one of two orders:
 *   - when the routed documents' rows (B * k average documents over a ~50 GB/s
 *     host link) are expected to cross the bus faster than the next layer's
 *     router keys stream from HBM: `stream` carries the router queries of
 *     all layers, then the scans one after the other, each on all SMs but 8;
 *     `copy_stream`, after an event on a layer's scan, its top-k kernels, the
 *     gather and the attention, which run beside the next layer's scan.  Two
 *     routing workspaces in ws alternate between layers;
 *   - otherwise: `stream` carries each layer's routing and, after the routing
 *     of layer l + 1 and an event on the gather, the attention of layer l;
 *     `copy_stream` the gather of each layer, after an event on its routing.
 * The results equal those calls made one after the other, bit for bit.  The
 * copy-stream work is joined back into `stream` before the call returns, so
 * work enqueued later on `stream` sees every output.
 * copy_stream may be NULL or equal to stream (no overlap; same results).
 *   capacity_chunks  staging rows per layer (>= the chunks of the B * k routed
 *                    documents; a selection needing more stages what fits and
 *                    raises device error bit 1, as msa_gather_kv).
 *   ws        >= msa_tiered_workspace_size(dims, n_layers, ...) bytes, 256-byte
 *             aligned; holds the layout's chunk -> document map (computed by the
 *             call), each layer's router-query rows, two routing workspaces, the
 *             attention workspace and the two staging areas.
 * msa_tiered_workspace_size returns 0 for arguments outside the limits below.
 * The call keeps six CUDA events per host thread and device (created by its
 * first call on that device from that thread: make that call before any stream
 * capture).  Limits: those of msa_route_topk, msa_gather_kv and
 * msa_sparse_attend with q_tokens = 1; 1 <= n_layers <= 4096.
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* Hq;
  const void* W_QR;
  const void* KR_bar;
  const float* kr_inv_norm;
  const void* K_bar_host;
  const void* V_bar_host;
  const void* q;
  void* K_loc;
  void* V_loc;
  const void* k_new;
  const void* v_new;
  int32_t* topk_idx;
  float* topk_score;
  void* out;
} msa_layer;

size_t msa_tiered_workspace_size(const msa_dims* dims, int32_t n_layers, int32_t B, int32_t n_docs, int32_t n_chunks,
                                 int32_t k, int32_t t_loc_max, int32_t pos_offset, int32_t capacity_chunks);
msa_status msa_tiered_decode(const msa_dims* dims, const msa_layer* layers, int32_t n_layers, int32_t B,
                             const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, int32_t k,
                             const int32_t* loc_len, int32_t t_loc_max, int32_t pos_offset, int32_t capacity_chunks,
                             void* ws, size_t ws_bytes, void* stream, void* copy_stream);

/* ---------------------------------------------------------------------------
 * In-place RoPE of key rows (global positions of the active context).
 * Pages: IRMaD "M. Materials & Methods", position item.  A decode loop that
 * keeps its local key cache rotated calls this once per appended token (row
 * at pos_offset + j) and then runs msa_sparse_attend with k_loc_rotated = 1,
 * instead of re-rotating every local key at every step.
 *   x          [rows, heads, head_dim] bf16, rotated in place (rotate-half pairs
 *              (i, i + head_dim/2), theta_i = rope_base^(-2i/head_dim); the angle
 *              p * theta_i is reduced exactly, as a 64-bit fraction of a turn;
 *              result rounded to bf16).
 *   positions  [rows] device int32, absolute positions.
 * ------------------------------------------------------------------------- */
msa_status msa_rope_rows(const msa_dims* dims, void* x, int32_t rows, int32_t heads, const int32_t* positions,
                         void* stream);

/* ---------------------------------------------------------------------------
 * Append one token per query to a rotated local KV cache.
 * Pages: IRMaD "M. Materials & Methods", position item (global RoPE on the
 * active context: local token j at pos_offset + j).  The decode step's new
 * token joins the local context: its key is rotated at its global position and
 * written, with its value, into the cache slot, in one launch.
 *   k_new, v_new  [B, n_kv, head_dim] bf16, the new token's key (before RoPE) and value.
 *   K_loc, V_loc  [B, t_loc_max, n_kv, head_dim] bf16 cache; row slots[b] of query b is
 *            written: K_loc = RoPE(k_new[b], pos_offset + slots[b]), V_loc = v_new[b].
 *   slots    [B] device int32, 0 <= slots[b] < t_loc_max (a slot outside is skipped and
 *            the device error word records it).
 * The result equals msa_rope_rows on a copy of k_new followed by the two row copies.
 * ------------------------------------------------------------------------- */
msa_status msa_kv_append(const msa_dims* dims, const void* k_new, const void* v_new, void* K_loc, void* V_loc,
                         int32_t B, int32_t t_loc_max, const int32_t* slots, int32_t pos_offset, void* stream);

/* ---------------------------------------------------------------------------
 * Global-RoPE cache for the active context (optional input of msa_sparse_attend).
 * Pages: IRMaD "M. Materials & Methods", position item (global RoPE on the
 * active context, positions offset by k).  The rotation angles of the local
 * positions pos_offset + j (j < t_loc_max) depend only on positions, not on
 * data, so a decode session can build them once:
 *   cache  [t_loc_max, head_dim/2] (cos, sin) fp32 pairs, device, caller-owned,
 *          msa_rope_cache_size(...) bytes; entry (j, i) is the rotation of pair
 *          (i, i + head_dim/2) at position pos_offset + j, theta_i =
 *          rope_base^(-2i/head_dim), angle reduced in fp64.
 * msa_sparse_attend uses a cache built for its own (pos_offset, t_loc_max,
 * head_dim, rope_base); passing rope_cache = NULL makes the call build the
 * table in its workspace first.
 * ------------------------------------------------------------------------- */
size_t msa_rope_cache_size(const msa_dims* dims, int32_t t_loc_max);
msa_status msa_rope_cache_build(const msa_dims* dims, int32_t t_loc_max, int32_t pos_offset, void* cache,
                                size_t cache_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Tracing: per-kernel device time.
 * While enabled, every kernel launch is bracketed by CUDA events recorded on
 * the stream it is launched on.  msa_trace_read synchronises on those events
 * and returns, for kernel `kernel_id`, the summed device milliseconds and the
 * launch count since the last reset.  Kernel ids run 0 .. msa_trace_num_kernels()-1.
 * ------------------------------------------------------------------------- */
msa_status msa_trace_enable(int32_t on);
msa_status msa_trace_reset(void);
int32_t msa_trace_num_kernels(void);
const char* msa_trace_kernel_name(int32_t kernel_id);
msa_status msa_trace_read(int32_t kernel_id, double* total_ms, int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */

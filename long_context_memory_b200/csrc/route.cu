// Stage 2 of MSA: online routing and top-k document selection.
//
// Definition (IRMaD reading of the MSA paper, "M. Materials & Methods",
// routing and sparse attention item):
//   Q^R_h = H_q W^QR_h,   S_j = mean_h cos(Q^R_h, K̄^R_{j,h}),   s_i = max_{j in doc i} S_j,
//   I = Top-k({s_i}),  k = 16 on the pages.
// The scan over every pooled router key is the only online term that grows
// with the memory size (complexity item of the same section: O(ML/P)).
//
// Kernels, in launch order:
//   router_query_kernel  Q^R = H_q W^QR (a thread-block cluster per router head,
//                    each CTA a row slab of the head's columns; the split-K
//                    partials meet in distributed shared memory in rank order),
//                    per-head normalisation, bf16 hi + lo rows for the scan's
//                    TMA; clears the doc keys
//   scan_kernel      TMA-staged streaming scan of K̄^R: tensor-core dots,
//                    cosine (precomputed or in-kernel key norms), head mean,
//                    per-document segmented max folded in with atomicMax on
//                    ordered keys; for few queries over one slice of documents
//                    its last CTA also selects the top-k
//   topk_slice_kernel / topk_merge_kernel
//                    exact top-k of the (score, id) keys per slice of
//                    documents (warp thresholds, a bitonic fallback, or a radix
//                    select for k > 32), then a merge of the slice winners
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace msa {

struct RouteWs {
  uint32_t* scan_ticket;  // [1 + B]: scan CTAs finished (fused top-k), then per query its slices
                          // finished (fused merge); zeroed by the router query kernel
  __nv_bfloat16* q_hl; // [passes][n_r][2][NQ][d_r] normalised query, bf16 hi and lo terms
  uint32_t* doc_key;  // [B][n_docs] ordered-uint32 doc max (MAX)
  uint32_t* chunk_k;  // [B][n_chunks] ordered chunk scores (MEAN)
  uint64_t* cand;     // [B][n_slices][k] slice winners
  int nq, passes, n_slices;
};

namespace {

constexpr int kSliceDocs = 4096;   // documents per top-k slice CTA
constexpr int kFuseTopkMaxQueries = 4;  // top-k in the scan's last CTA up to this many queries
constexpr int kTopkThreads = 1024;
constexpr float kEps = 1e-12f;

// --------------------------------------------------------------------------
// Router query: Q^R = H_q W^QR, per-head normalisation, bf16 hi + lo terms in the
// layout the scan's TMA reads (q_hl[pass][head][hi|lo][NQ rows][d_r]; rows of
// padding queries are zero), and the clearing of the scan's max keys.  A row is
// one query token (B queries x M tokens).
//
// Grid (8, n_r), one thread-block cluster of 8 CTAs per router head: CTA r of
// head h multiplies rows [r*RS, (r+1)*RS) of W^QR's head-h column block (staged in
// shared memory with asynchronous 16-byte copies, kRqPiece rows at a time) by the
// matching slice of 16 query rows on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 out).  The 8 partial
// products meet in distributed shared memory: after a cluster barrier CTA r sums,
// in rank order, rows r and r + 8 of the 16-row block over the cluster's CTAs,
// normalises them and writes their hi/lo terms.  No global partials, no counters.
// With W_QR == NULL the rows of Hq already hold Q^R and router_query_direct_kernel
// only normalises them.
// --------------------------------------------------------------------------
constexpr int kRqThreads = 256;
constexpr int kRqCluster = 8;   // CTAs per router head
constexpr int kRqPiece = 384;   // rows of W staged at a time (hidden <= 3072: one piece)

// rows of W per CTA (a multiple of 16)
int rq_split_rows(int hidden) { return ((hidden + kRqCluster - 1) / kRqCluster + 15) / 16 * 16; }

// shared memory: a W piece [kRqPiece][d_r] and 16 query rows [16][kRqPiece], both bf16 with rows
// padded by 16 bytes (ldmatrix's 8 row addresses in distinct bank groups), then the CTA's
// partial product [16][d_r] fp32
__host__ __device__ inline int rq_w_stride(int d_r) { return d_r * 2 + 16; }
__host__ __device__ inline int rq_h_stride() { return kRqPiece * 2 + 16; }
size_t rq_smem_bytes(int d_r) {
  return (size_t)kRqPiece * rq_w_stride(d_r) + 16 * (size_t)rq_h_stride() + 16 * (size_t)d_r * sizeof(float);
}

__device__ __forceinline__ void rq_clear(uint32_t* clear, size_t n_clear, uint32_t* scan_ticket, int n_tickets) {
  if (scan_ticket && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < n_tickets; i += blockDim.x) scan_ticket[i] = 0u;
  if (clear) {
    const size_t cta = (size_t)blockIdx.y * gridDim.x + blockIdx.x, n_cta = (size_t)gridDim.x * gridDim.y;
    for (size_t i = cta * blockDim.x + threadIdx.x; i < n_clear; i += n_cta * blockDim.x) clear[i] = 0u;
  }
}

// one normalised row of head h: hi/lo bf16 terms into the scan's query layout
__device__ __forceinline__ void rq_store_row(__nv_bfloat16* q_hl, int b, int h, int i, float x, int n_r, int d_r,
                                             int nq) {
  const int pass = b / nq, row = b % nq;
  const size_t base = (((size_t)pass * n_r + h) * 2) * nq;
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
  q_hl[(base + row) * d_r + i] = hi;
  q_hl[(base + nq + row) * d_r + i] = lo;
}

__global__ void __launch_bounds__(kRqThreads) router_query_kernel(
    const __nv_bfloat16* __restrict__ Hq, const __nv_bfloat16* __restrict__ W, int B, int b_pad, int hidden,
    int n_r, int d_r, int nq, int split_rows, __nv_bfloat16* __restrict__ q_hl, uint32_t* __restrict__ clear,
    size_t n_clear, uint32_t* __restrict__ scan_ticket, int n_tickets, int early) {
  extern __shared__ __align__(16) uint8_t rq_smem[];
  __shared__ float wsum[kRqThreads / 32];
  // early: H_q, W^QR and the memory the scan reads (K̄^R, its norms, chunk_off) were final
  // before the preceding work was enqueued, so the scan may start at once and every thread
  // reads and multiplies before it waits; the writes (workspace) come after the wait
  bool waited = !early;
  if (waited) {
    pdl_enter();
    rq_clear(clear, n_clear, scan_ticket, n_tickets);
  } else {
    pdl_launch_dependents();
  }
  const int NR = n_r * d_r;
  const int rank = blockIdx.x, h = blockIdx.y;  // the cluster spans blockIdx.x
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint16_t* hq = reinterpret_cast<const uint16_t*>(Hq);

  const int ws = rq_w_stride(d_r), hstr = rq_h_stride();
  uint8_t* wsm = rq_smem;
  uint8_t* hsm = rq_smem + (size_t)kRqPiece * ws;
  float* part = reinterpret_cast<float*>(hsm + 16 * (size_t)hstr);  // [16][d_r]
  const int k0 = rank * split_rows;
  const int nrows = max(0, min(split_rows, hidden - k0));  // a multiple of 16
  const int n_nt = d_r / 8;                 // n-tiles of 8 columns
  const int nt_per_warp = n_nt / 8;         // 2 or 1
  const int n0 = warp * nt_per_warp;        // first n-tile of this warp
  const int per_row = d_r / 8;              // 16-byte pieces of a W row

  for (int b0 = 0; b0 < b_pad; b0 += 16) {
    // two accumulator sets (even and odd k-steps): half the dependent MMA chain
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int p0 = 0; p0 < nrows; p0 += kRqPiece) {
      const int pr = min(kRqPiece, nrows - p0);
      __syncthreads();  // the previous piece is consumed
      // every 16-byte piece of the W piece and of the query rows in flight at once
      const __nv_bfloat16* wsrc = W + (size_t)(k0 + p0) * NR + h * d_r;
      for (int i = tid; i < pr * per_row; i += kRqThreads) {
        const int r = i / per_row, c = i % per_row;
        cp_async16(wsm + (size_t)r * ws + c * 16, reinterpret_cast<const uint4*>(wsrc + (size_t)r * NR) + c);
      }
      const int vec = pr / 8;
      for (int i = tid; i < 16 * vec; i += kRqThreads) {
        const int j = i / vec, v = i % vec;
        if (b0 + j < B)
          cp_async16(hsm + (size_t)j * hstr + v * 16,
                     reinterpret_cast<const uint4*>(hq + (size_t)(b0 + j) * hidden + k0 + p0) + v);
        else
          *reinterpret_cast<uint4*>(hsm + (size_t)j * hstr + v * 16) = make_uint4(0, 0, 0, 0);
      }
      cp_async_wait_all();
      __syncthreads();
      for (int ks = 0; ks < pr / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(a0, a1, a2, a3, smem_u32(hsm + (size_t)(lane & 15) * hstr + (ks * 16 + 8 * (lane >> 4)) * 2));
        const int krow = ks * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        uint32_t b0r, b1r, b2r, b3r;
        float (*dst)[4] = (ks & 1) ? acc2 : acc;
        if (nt_per_warp == 2) {
          ldmatrix_x4_trans(b0r, b1r, b2r, b3r, smem_u32(wsm + (size_t)krow * ws + (8 * n0 + 8 * (lane >> 4)) * 2));
          mma_bf16_16816(dst[0], a0, a1, a2, a3, b0r, b1r);
          mma_bf16_16816(dst[1], a0, a1, a2, a3, b2r, b3r);
        } else {  // two k-halves of one n-tile (the upper lanes' rows repeat)
          ldmatrix_x4_trans(b0r, b1r, b2r, b3r, smem_u32(wsm + (size_t)krow * ws + (8 * n0) * 2));
          mma_bf16_16816(dst[0], a0, a1, a2, a3, b0r, b1r);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] += acc2[t][e];
    // this CTA's partial product of the 16-row block: D fragment rows lane/4 (+8), columns
    // 2 (lane % 4) + {0, 1} of each n-tile
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (t >= nt_per_warp) break;
      const int col = 8 * (n0 + t) + 2 * (lane & 3);
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
        *reinterpret_cast<float2*>(part + ((lane >> 2) + 8 * rr) * d_r + col) =
            make_float2(acc[t][2 * rr], acc[t][2 * rr + 1]);
    }
    cluster_sync();  // every CTA's partial is written

    // rows rank and rank + 8 of the block: the sum over the cluster's CTAs in rank order
    {
      const int q = tid / d_r, i = tid % d_r;  // q: which of the two rows (threads with q > 1 idle)
      const int row = rank + 8 * q;
      float v = 0.f;
      if (q < 2) {
#pragma unroll
        for (int r = 0; r < kRqCluster; ++r) v += ld_dsmem_f32(part + row * d_r + i, r);
      }
      float ss = v * v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) wsum[warp] = ss;
      __syncthreads();
      if (!waited) {  // every thread, before its first write
        pdl_wait();
        rq_clear(clear, n_clear, scan_ticket, n_tickets);
        waited = true;
      }
      if (q < 2) {
        const int w0 = q * d_r / 32, nw = d_r / 32;  // the warps holding this row
        float tot = 0.f;
        for (int w = 0; w < nw; ++w) tot += wsum[w0 + w];
        const float sc = 1.0f / fmaxf(sqrtf(tot), kEps);
        rq_store_row(q_hl, b0 + row, h, i, v * sc, n_r, d_r, nq);
      }
    }
    cluster_sync();  // the partials may be overwritten / the CTAs may exit
  }
  if (!waited) pdl_wait();  // the grid completes only after its predecessor
}

// Q^R given directly (W_QR == NULL): normalise each row of head h, write the hi/lo terms
__global__ void __launch_bounds__(kRqThreads) router_query_direct_kernel(
    const __nv_bfloat16* __restrict__ Hq, int B, int b_pad, int n_r, int d_r, int nq, __nv_bfloat16* __restrict__ q_hl,
    uint32_t* __restrict__ clear, size_t n_clear, uint32_t* __restrict__ scan_ticket, int n_tickets, int early) {
  __shared__ float invn[kRqThreads / 32];
  if (!early) pdl_enter();  // early: H_q is read before the wait, the writes come after it
  else pdl_launch_dependents();
  const int NR = n_r * d_r, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t* hq = reinterpret_cast<const uint16_t*>(Hq);
  for (int b = warp; b < b_pad; b += kRqThreads / 32) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};  // dims lane, lane + 32, ... (d_r <= 128)
    float ss = 0.f;
    if (b < B) {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (lane + 32 * e < d_r) v[e] = bf16_bits_to_float(hq[(size_t)b * NR + h * d_r + lane + 32 * e]);
#pragma unroll
      for (int e = 0; e < 4; ++e) ss = fmaf(v[e], v[e], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) invn[warp] = 1.0f / fmaxf(sqrtf(ss), kEps);
    __syncwarp();
    const float sc = invn[warp];
    __syncwarp();
    if (early && b == warp) pdl_wait();  // this warp's first write
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (lane + 32 * e < d_r) rq_store_row(q_hl, b, h, lane + 32 * e, v[e] * sc, n_r, d_r, nq);
  }
  if (early && warp >= b_pad) pdl_wait();  // warps with no rows
  rq_clear(clear, n_clear, scan_ticket, n_tickets);
}

// --------------------------------------------------------------------------
// the K̄^R scan on tcgen05 tensor cores
//
// Tile = 128 consecutive chunks; the tile is streamed one router head at a
// time.  A pipeline stage holds that head's 128 x d_r slice of K̄^R (the MMA's
// A operand, 128B-swizzled TMA boxes) and the head's normalised query terms
// (B operand: hi and lo bf16 rows, NQ queries).  One thread issues
//   D[128 chunks, h*NQ .. h*NQ+NQ) += K̄^R_h (128 x d_r) . (q_hi + q_lo)^T
// into a double-buffered TMEM accumulator.  Four norm warps read each stage
// from shared memory for the per-chunk squared norms and release it at once;
// four epilogue warps, separate from them, take a finished tile (its TMEM
// buffer and its norms), apply 1/||K̄^R_h||, average the heads and fold each
// document's maximum into doc_key with one atomicMax per document segment,
// while the next tile streams in.
// --------------------------------------------------------------------------
constexpr int kScanM = 128;         // chunks per tile (MMA M)
constexpr int kScanThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..5 norms, warps 6..9 epilogue
constexpr int kScanNormWarps = 4;   // one per TMEM lane quarter (32 rows each)
constexpr int kScanEpiWarps = 4;

__device__ void slice_topk(const uint32_t* doc_key, const uint32_t* chunk_k, const int32_t* chunk_off, int n_docs,
                           int n_chunks, int k, int n_slices, float* doc_scores, uint64_t* cand, int32_t* topk_idx,
                           float* topk_score, int slice, int b, uint64_t* sm64);

struct ScanParams {
  const int32_t* chunk_off;
  uint32_t* doc_key;
  uint32_t* chunk_k;
  // top-k fused into the scan (one slice of documents, few queries): the last CTA to finish
  // (ticket) selects the top-k of every query
  uint32_t* ticket;  // null: top-k runs as its own kernel
  int n_queries, k;
  float* doc_scores;
  int32_t* topk_idx;
  float* topk_score;
  int n_r, n_docs, n_chunks, n_tiles;
  int q_tokens;    // query tokens per query: scan row r belongs to query r / q_tokens
  int q_base, q_count, pass;
  int head_major;  // K̄^R stored [n_r][C][d_r] instead of [C][n_r][d_r]
  const float* inv_norm;  // [C][n_r] 1 / max(||K̄^R_jh||, eps) precomputed, or null (norm warps compute it)
  const int32_t* chunk_doc;  // [C] each chunk's document (-1: none), or null (searched in chunk_off)
  int wait_prior;  // 0: the kernel before this one on the stream writes nothing this scan reads or writes
  uint32_t tmem_cols;
  float inv_nr;
};

template <int DR, int NQ>
struct ScanGeom {
  static constexpr int kHalves = DR / 64;
  static constexpr int kKBox = kScanM * 128;            // one 64-dim x 128-row box
  static constexpr int kQBox = NQ * 128;                // one 64-dim x NQ-row box
  static constexpr int kKBytes = kHalves * kKBox;
  static constexpr int kQBytes = 2 * kHalves * kQBox;   // hi and lo: [half j][hi | lo][NQ rows]
  // one MMA per k-step with N = 2 NQ (the hi and lo rows side by side, summed in the
  // epilogue): half the MMA chain of accumulating hi and lo into one accumulator, so each
  // stage is released sooner.  TMEM (512 columns) holds two tiles' accumulators for NQ = 16,
  // one for NQ = 32; either way a head's columns are released as soon as the epilogue has
  // read them, so the next tile's MMA of that head need not wait for the whole epilogue.
  static constexpr int kCols = 2 * NQ;                  // TMEM columns per head
  static constexpr int kBufs = NQ == 16 ? 2 : 1;        // tiles in flight in TMEM
  static constexpr int kStageBytes = kKBytes + kQBytes;
  static constexpr int kStages = (NQ == 16 || DR == 64) ? 5 : 4;
  static constexpr int kNormBytes = 2 * 8 * kScanM * 4;  // [2 tiles][8 heads][128 rows] fp32
  static constexpr int kBars = 2 * kStages + kBufs * 9 + 5;
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + kNormBytes + kBars * 8 + 16;
};

// The scan's epilogue for one warp: TMEM lane quarter q4 (32 rows of every tile) and the QW
// queries q_off .. q_off + QW - 1.  Per tile: find each row's document (while the tile streams),
// wait for the tile's MMA (and its norms), read each head's accumulator columns (the hi and lo
// halves of this warp's queries) and release them, and fold each document segment's maximum into
// doc_key (or store the chunk scores for the mean).  A warp whose queries are all past q_count still takes part in the
// barrier protocol but does no work.
template <int DR, int NQ, bool MEAN, bool MAPPED, int QW>
__device__ __forceinline__ void scan_epilogue(const ScanParams& p, int q4, int q_off, int lane, int t_begin, int n_lt,
                                              uint32_t tmem_base, uint32_t buf_cols, const float* n2s, uint64_t* tfull,
                                              uint64_t* tempty, uint64_t* nfull, uint64_t* nempty,
                                              volatile int* abort) {
  using Gm = ScanGeom<DR, NQ>;
  const int n_r = p.n_r;
  const int row = 32 * q4 + lane;  // chunk within the tile
  const bool active = q_off < p.q_count;
  int cur = 0;                     // lower bound for this warp's document search
  // With a chunk -> document map the rows' documents and inverse norms of the next tile are
  // loaded while this one is processed (one tile ahead); without it each tile searches chunk_off.
  // (a compile-time choice, so that routing without the map keeps the search's own code; the mean
  // needs no document boundaries)
  constexpr bool mapped = MAPPED && !MEAN;
  int doc_next = -1;
  float invg_next[8];
  auto fetch = [&](int lt_f) {
    const int jr = (t_begin + lt_f) * kScanM + row;
    doc_next = (active && jr < p.n_chunks) ? __ldg(&p.chunk_doc[jr]) : -1;
#pragma unroll
    for (int hh = 0; hh < 8; ++hh)
      invg_next[hh] = (p.inv_norm && active && hh < n_r && jr < p.n_chunks) ? __ldg(&p.inv_norm[(size_t)jr * n_r + hh])
                                                                            : 0.f;
  };
  if (mapped && n_lt > 0) fetch(0);
  for (int lt = 0; lt < n_lt; ++lt) {
    const int tile = t_begin + lt;
    const int nbuf = lt & 1;                                    // norm buffer
    const int buf = lt % Gm::kBufs, use = lt / Gm::kBufs;      // TMEM buffer
    const int jrow = tile * kScanM + row;
    const int j = tile * kScanM + row;
    int doc = -1;
    float invg[8];  // precomputed inverse norms of this row (loads in flight during the waits)
    if (mapped) {
      doc = doc_next;
#pragma unroll
      for (int hh = 0; hh < 8; ++hh) invg[hh] = invg_next[hh];
      if (lt + 1 < n_lt) fetch(lt + 1);
    } else {
      // documents of this warp's 32 rows, found before the accumulators are ready (they depend
      // on the tile alone): a warp-wide 32-ary search for the first row's document, then one
      // lookahead of 32 document boundaries (32 consecutive rows cross at most 31 of them)
      const int j0 = tile * kScanM + 32 * q4;
      if (active && j0 < p.n_chunks) {
        int lo = cur, hi = p.n_docs;  // answer in [lo, hi): largest d with chunk_off[d] <= j0
        while (hi - lo > 1) {
          const int step = (hi - lo + 31) >> 5;
          const int probe = lo + lane * step;
          const bool ok = probe < hi && __ldg(&p.chunk_off[probe]) <= j0;
          const unsigned m = __ballot_sync(0xffffffffu, ok);
          const int L = 31 - __clz(m);  // lane 0 always qualifies (chunk_off[lo] <= j0)
          lo = lo + L * step;
          hi = min(hi, lo + step);
        }
        const int d0 = lo;
        const int bi = d0 + 1 + lane;
        const int bnd = bi <= p.n_docs ? __ldg(&p.chunk_off[bi]) : 0x7fffffff;
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
          const unsigned m = __ballot_sync(0xffffffffu, bnd <= j0 + r);
          if (lane == r) doc = d0 + __popc(m);
        }
        if (j >= p.n_chunks) doc = -1;
        cur = d0;
      }
    }
    const int prev = __shfl_up_sync(0xffffffffu, doc, 1);
    const bool head = (lane == 0) || (prev != doc);
    // the document pattern is the same for every query: which shuffle partners share my document
    uint32_t same = 0;
#pragma unroll
    for (int e = 0; e < 5; ++e) {
      const int od = __shfl_down_sync(0xffffffffu, doc, 1 << e);
      if (lane + (1 << e) < 32 && od == doc) same |= 1u << e;
    }
    if (!mapped && p.inv_norm) {  // (with the map they were loaded a tile ahead)
#pragma unroll
      for (int hh = 0; hh < 8; ++hh)
        invg[hh] = (active && hh < n_r && jrow < p.n_chunks) ? __ldg(&p.inv_norm[(size_t)jrow * n_r + hh]) : 0.f;
    } else if (!p.inv_norm && !warp_wait(&nfull[nbuf], (lt >> 1) & 1, abort)) {
      return;
    }
    if (!warp_wait(&tfull[buf], use & 1, abort)) return;
    tc_fence_after();
    const float* nb2 = n2s + (size_t)nbuf * 8 * kScanM;
    float acc[QW];
#pragma unroll
    for (int b = 0; b < QW; ++b) acc[b] = 0.f;
    const uint32_t t_row = tmem_base + ((uint32_t)(32 * q4) << 16) + buf * buf_cols;
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      if (hh < n_r) {
        if (active) {
          const float inv = p.inv_norm ? invg[hh] : 1.0f / fmaxf(sqrtf(nb2[hh * kScanM + row]), kEps);
          const uint32_t c_hi = t_row + hh * Gm::kCols + q_off, c_lo = c_hi + NQ;
          float v[QW], w[QW];
          if constexpr (QW == 32) {
            tmem_ld32(c_hi, v);
            tmem_ld32(c_lo, w);
          } else if constexpr (QW == 16) {
            tmem_ld16(c_hi, v);
            tmem_ld16(c_lo, w);
          } else {
            tmem_ld8(c_hi, v);
            tmem_ld8(c_lo, w);
          }
          tmem_ld_wait();
#pragma unroll
          for (int b = 0; b < QW; ++b) acc[b] = fmaf(v[b] + w[b], inv, acc[b]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf * 8 + hh]);  // the next tile may reuse these columns
      }
    }
    __syncwarp();
    if (lane == 0 && !p.inv_norm) mbar_arrive(&nempty[nbuf]);
    if (!active) continue;

#pragma unroll
    for (int bb = 0; bb < QW; ++bb) {
      const int b = q_off + bb;
      if (b >= p.q_count) break;  // warp-uniform
      const float sc = acc[bb] * p.inv_nr;
      const size_t qi = (size_t)((p.q_base + b) / p.q_tokens);  // max over a query's tokens: atomicMax
      if (MEAN) {
        if (doc >= 0) {
          uint32_t* dst = &p.chunk_k[qi * p.n_chunks + j];
          if (p.q_tokens == 1) *dst = float_to_ordered(sc);
          else atomicMax(dst, float_to_ordered(sc));
        }
      } else {
        float x = doc >= 0 ? sc : -__int_as_float(0x7f800000);
#pragma unroll
        for (int e = 0; e < 5; ++e) {
          const float ox = __shfl_down_sync(0xffffffffu, x, 1 << e);
          if (same & (1u << e)) x = fmaxf(x, ox);
        }
        if (head && doc >= 0) atomicMax(&p.doc_key[qi * p.n_docs + doc], float_to_ordered(x));
      }
    }
  }
}

template <int DR, int NQ, bool MEAN, bool MAPPED>
__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(const __grid_constant__ CUtensorMap kr_map,
                                                               const __grid_constant__ CUtensorMap q_map,
                                                               const ScanParams p) {
  using Gm = ScanGeom<DR, NQ>;
  constexpr int KS = DR / 16;
  constexpr int S = Gm::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* n2s = reinterpret_cast<float*>(smem + S * Gm::kStageBytes);  // [2 tiles][8 heads][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Gm::kStageBytes + Gm::kNormBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;                 // [kBufs] MMA of a tile committed
  uint64_t* tempty = tfull + Gm::kBufs;        // [kBufs][8] epilogue has read a head's accumulator
  uint64_t* nfull = tempty + Gm::kBufs * 8;    // [2] norms of a tile written
  uint64_t* nempty = nfull + 2;                // [2] epilogue has read a tile's norms
  uint64_t* drained = nempty + 2;              // [1] after an abort: every MMA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  __shared__ int abort_flag;                   // a bounded wait of this CTA gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_r = p.n_r;
  const int t_begin = (int)(((long long)blockIdx.x * p.n_tiles) / gridDim.x);
  const int t_end = (int)(((long long)(blockIdx.x + 1) * p.n_tiles) / gridDim.x);
  const int n_lt = t_end - t_begin;
  const int n_it = n_lt * n_r;  // (tile, head) stages of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + (p.inv_norm ? 0 : kScanNormWarps));  // MMA commit (+ the norm warps)
    }
    for (int b = 0; b < Gm::kBufs; ++b) {
      mbar_init(&tfull[b], 1);
      for (int hh = 0; hh < 8; ++hh) mbar_init(&tempty[b * 8 + hh], p.inv_norm ? 8 : kScanEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&nfull[b], kScanNormWarps);
      mbar_init(&nempty[b], kScanEpiWarps);
    }
    mbar_init(drained, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&kr_map);
    prefetch_tensormap(&q_map);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t buf_cols = (uint32_t)n_r * Gm::kCols;
  // stage it = (tile, head): the head's 128 x DR key rows, then the head's query rows (hi, lo)
  auto load_keys = [&](int it) {
    const int tile = t_begin + it / n_r, h = it % n_r, st = it % S;
    uint8_t* k_s = stages + st * Gm::kStageBytes;
    mbar_arrive_expect_tx(&full[st], Gm::kStageBytes);  // the query rows' bytes included
#pragma unroll
    for (int j = 0; j < Gm::kHalves; ++j) {
      if (p.head_major)
        tma_load_3d(k_s + j * Gm::kKBox, &kr_map, &full[st], j * 64, tile * kScanM, h);
      else
        tma_load_2d(k_s + j * Gm::kKBox, &kr_map, &full[st], h * DR + j * 64, tile * kScanM);
    }
  };
  auto load_query = [&](int it) {
    const int h = it % n_r, st = it % S;
    uint8_t* q_s = stages + st * Gm::kStageBytes + Gm::kKBytes;
#pragma unroll
    for (int j = 0; j < Gm::kHalves; ++j)
#pragma unroll
      for (int hl = 0; hl < 2; ++hl)
        tma_load_2d(q_s + (j * 2 + hl) * Gm::kQBox, &q_map, &full[st], j * 64, ((p.pass * n_r + h) * 2 + hl) * NQ);
  };
  // The previous kernel of this call (the router query, or the previous pass) does not write
  // K̄^R, and it started this grid only after its own wait, so whatever wrote K̄^R has
  // completed: the first ring's key tiles stream in while the router query finishes.
  const int n_pre = min(S, n_it);
  if (warp == 0 && lane == 0)
    for (int it = 0; it < n_pre; ++it) load_keys(it);
  // A scan that follows another routing's scan on the stream (the caller's guarantee: that scan
  // writes another workspace, and everything this one reads was final before it started) does
  // not wait for it: its CTAs stream as soon as they land, beside the other scan's last tiles.
  if (p.wait_prior) pdl_enter();
  else pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------- TMA producer -------------------------
    if (lane == 0) {
      int it = 0;
      for (; it < n_it; ++it) {
        if (it >= n_pre) {
          if (it >= S && !mbar_wait(&empty[it % S], ((it / S) - 1) & 1, &abort_flag)) break;
          load_keys(it);
        }
        load_query(it);
      }
      // after an abort: the stages issued and possibly still in flight land before the CTA exits
      if (abort_flag) mbar_drain_ring(full, S, it - S, it);
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer -------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kScanM, Gm::kCols);
      for (int it = 0; it < n_it; ++it) {
        const int lt = it / n_r, h = it % n_r;
        const int buf = lt % Gm::kBufs, use = lt / Gm::kBufs;
        const int st = it % S;
        if (use >= 1 && !mbar_wait(&tempty[buf * 8 + h], (use - 1) & 1, &abort_flag)) break;  // head's columns read
        if (!mbar_wait(&full[st], (it / S) & 1, &abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * buf_cols + h * Gm::kCols;
        const uint32_t k_addr = smem_u32(stages + st * Gm::kStageBytes);
        const uint32_t q_addr = k_addr + Gm::kKBytes;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int j = ks >> 2, off = (ks & 3) * 32;
          const uint64_t a_desc = umma_desc_k_sw128(k_addr + j * Gm::kKBox + off);
          // B = the 2 NQ rows [hi; lo] of this k-half
          umma_bf16(d_tmem, a_desc, umma_desc_k_sw128(q_addr + j * 2 * Gm::kQBox + off), idesc, ks > 0);
        }
        umma_commit(&empty[st]);
        if (h == n_r - 1) umma_commit(&tfull[buf]);
      }
      if (abort_flag) {  // every MMA issued completes before the TMEM is freed
        umma_commit(drained);
        mbar_drain_ring(drained, 1, 0, 1);
      }
    }
  } else if (warp < 2 + kScanNormWarps && p.inv_norm) {
    // norms given: these four warps take the second half of the queries of each row
    scan_epilogue<DR, NQ, MEAN, MAPPED, NQ / 2>(p, warp & 3, NQ / 2, lane, t_begin, n_lt, tmem_base, buf_cols, n2s, tfull,
                                        tempty, nfull, nempty, &abort_flag);
  } else if (warp < 2 + kScanNormWarps) {
    // ------- norm warps: squared norm of every row's head-h slice, stage released at once -------
    const int row = 32 * (warp & 3) + lane;  // chunk within the tile
    for (int it = 0; it < (p.inv_norm ? 0 : n_it); ++it) {
      const int lt = it / n_r, h = it % n_r;
      const int buf = lt & 1;  // norm buffer
      const int st = it % S;
      if (h == 0 && lt >= 2 && !warp_wait(&nempty[buf], ((lt >> 1) - 1) & 1, &abort_flag)) break;  // n2s[buf] free
      if (!warp_wait(&full[st], (it / S) & 1, &abort_flag)) break;
      const uint8_t* k_s = stages + st * Gm::kStageBytes;
      float n2p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < Gm::kHalves; ++j) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 w = *reinterpret_cast<const uint4*>(k_s + j * Gm::kKBox + row * 128 + ((u ^ (row & 7)) << 4));
          float2 f;
          f = unpack_bf16x2(w.x); n2p[0] = fmaf(f.x, f.x, n2p[0]); n2p[1] = fmaf(f.y, f.y, n2p[1]);
          f = unpack_bf16x2(w.y); n2p[2] = fmaf(f.x, f.x, n2p[2]); n2p[3] = fmaf(f.y, f.y, n2p[3]);
          f = unpack_bf16x2(w.z); n2p[0] = fmaf(f.x, f.x, n2p[0]); n2p[1] = fmaf(f.y, f.y, n2p[1]);
          f = unpack_bf16x2(w.w); n2p[2] = fmaf(f.x, f.x, n2p[2]); n2p[3] = fmaf(f.y, f.y, n2p[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      n2s[(buf * 8 + h) * kScanM + row] = (n2p[0] + n2p[1]) + (n2p[2] + n2p[3]);
      if (h == n_r - 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&nfull[buf]);
      }
    }
  } else {
    // epilogue warps: every query of each row, or the first half when the norms are given
    if (p.inv_norm)
      scan_epilogue<DR, NQ, MEAN, MAPPED, NQ / 2>(p, warp & 3, 0, lane, t_begin, n_lt, tmem_base, buf_cols, n2s, tfull, tempty,
                                          nfull, nempty, &abort_flag);
    else
      scan_epilogue<DR, NQ, MEAN, MAPPED, NQ>(p, warp & 3, 0, lane, t_begin, n_lt, tmem_base, buf_cols, n2s, tfull, tempty,
                                      nfull, nempty, &abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, p.tmem_cols);

  if (p.ticket && !abort_flag) {  // a CTA that gave up leaves the top-k unselected (error word set)
    // every CTA's document maxima are in L2: the last one selects the top-k (the pipeline's
    // shared memory is free again and holds the keys)
    __shared__ bool last_cta;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t prev = atomicAdd(p.ticket, 1u);
      last_cta = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!last_cta) return;
    __threadfence();
    if (threadIdx.x == 0) *p.ticket = 0u;  // ready for the next launch
    for (int b = 0; b < p.n_queries; ++b)
      slice_topk(p.doc_key, p.chunk_k, p.chunk_off, p.n_docs, p.n_chunks, p.k, 1, p.doc_scores, nullptr,
                 p.topk_idx, p.topk_score, 0, b, reinterpret_cast<uint64_t*>(smem));
  }
}

// --------------------------------------------------------------------------
// exact block-wide top-k of distinct 64-bit keys in shared memory
// key = (ordered score << 32) | (0xFFFFFFFF - doc id): larger key = better,
// equal scores prefer the lower id; no key is 0 (the low word is at least 1),
// so 0 serves as an empty slot.  Writes the k best keys, descending, to out[0..k).
// --------------------------------------------------------------------------
__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
}

// 64 keys, element e = lane + 32 r held in x_r, sorted descending over e (bitonic sorting
// network: in a block of `size` elements the lower element of each pair keeps the larger key
// when the block is to end up descending, the smaller when ascending; the last block, all 64,
// is descending).  Pairs 32 apart sit in one lane; the others are one shuffle apart.
__device__ __forceinline__ void warp_sort64_desc(uint64_t& x0, uint64_t& x1, int lane) {
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {
        const uint64_t hi = x0 > x1 ? x0 : x1, lo = x0 > x1 ? x1 : x0;
        x0 = hi;
        x1 = lo;
      } else {
        const uint64_t y0 = shfl_xor_u64(x0, stride), y1 = shfl_xor_u64(x1, stride);
        const bool lower = (lane & stride) == 0;
        const bool desc0 = (lane & size) == 0, desc1 = ((lane + 32) & size) == 0;
        x0 = (lower == desc0) ? (x0 > y0 ? x0 : y0) : (x0 < y0 ? x0 : y0);
        x1 = (lower == desc1) ? (x1 > y1 ? x1 : y1) : (x1 < y1 ? x1 : y1);
      }
    }
  }
}

// the 32 largest keys of two descending lists (one key per lane each), descending: lane i
// takes max(a_i, b_31-i), which holds the 32 largest as a bitonic sequence, and a half-cleaner
// cascade sorts it
__device__ __forceinline__ uint64_t warp_merge_desc(uint64_t a, uint64_t b, int lane) {
  const uint64_t br = shfl_u64(b, 31 - lane);
  uint64_t x = a > br ? a : br;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t y = shfl_xor_u64(x, stride);
    x = ((lane & stride) == 0) ? (x > y ? x : y) : (x < y ? x : y);
  }
  return x;
}

// k <= 32.  (1) Every warp keeps its k best keys sorted across its lanes and folds in 64 keys
// at a time (a round whose keys all fall below the warp's current k-th best is skipped after
// one vote).  (2) The warps' lists, zero-padded to 32, meet in shared memory, and each entry
// counts the larger entries of every list (a 5-step search per sorted list).  An entry with
// fewer than k larger entries is one of the k best overall, and that count is its rank: every
// key above a global winner is itself among its warp's k best, and an entry outside the
// winners sees k larger entries in some list or in total.  lists: [blockDim.x] words, and
// blockDim.x is a multiple of 32.
__device__ void block_topk_small(const uint64_t* keys, int n, int k, uint64_t* out, uint64_t* lists) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  uint64_t best = 0;
  bool first = true;
  for (int base = warp * 64; base < n; base += nw * 64) {
    uint64_t x0 = base + lane < n ? keys[base + lane] : 0ull;
    uint64_t x1 = base + 32 + lane < n ? keys[base + 32 + lane] : 0ull;
    const uint64_t kth = shfl_u64(best, k - 1);
    if (!__any_sync(0xffffffffu, x0 > kth || x1 > kth)) continue;
    warp_sort64_desc(x0, x1, lane);
    best = first ? x0 : warp_merge_desc(best, x0, lane);
    first = false;
  }
  lists[tid] = lane < k ? best : 0ull;
  __syncthreads();
  const uint64_t c = lists[tid];
  if (c != 0ull) {
    int rank = 0;
#pragma unroll 4
    for (int v = 0; v < nw; ++v) {
      const uint64_t* a = lists + v * 32;
      int pos = 0;  // entries of list v above c: a[0 .. pos)
#pragma unroll
      for (int step = 16; step > 0; step >>= 1)
        if (a[pos + step - 1] > c) pos += step;
      if (pos == 31 && a[31] > c) pos = 32;  // all 32 entries (k = 32)
      rank += pos;
    }
    if (rank < k) out[rank] = c;
  }
  __syncthreads();
}

// k <= 32, few candidates: (1) warp w takes keys [w n / nw, (w + 1) n / nw), at most 4 per
// lane, and finds the m-th largest score (the key's upper word) T_w among them (m = ceil(k / nw);
// m rounds of a warp-wide 32-bit max, one owner lane dropping its maximum each time).  (2) T =
// min over warps of T_w: every warp holds m keys scoring >= T_w >= T, so at least k keys score
// >= T and the k best all do.  (3) The keys scoring >= T are compacted (one shared-memory atomic
// per warp) and each counts the larger keys, which is its rank.  Returns false, having written nothing, when the split does not apply (n above 128 keys
// per warp, a warp with fewer than m keys, m above 4) or more than kTopkMaxCand keys pass.
constexpr int kTopkMaxCand = 256;
__device__ bool block_topk_threshold(const uint64_t* keys, int n, int k, uint64_t* out, uint64_t* cand,
                                     uint64_t* warp_t, uint32_t* count) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int m = (k + nw - 1) / nw;
  if (m > 4 || n < m * nw || n > 128 * nw) return false;  // block-uniform
  const int lo = warp * n / nw, hi = (warp + 1) * n / nw;  // n <= 4096: no overflow
  if (tid == 0) *count = 0u;
  uint64_t v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = lo + lane + 32 * j < hi ? keys[lo + lane + 32 * j] : 0ull;
  const uint64_t v0 = v[0], v1 = v[1], v2 = v[2], v3 = v[3];  // kept for the compaction
  // the lane's keys in descending order
#define MSA_CX(a, b) { const uint64_t x_ = v[a] > v[b] ? v[a] : v[b]; v[b] = v[a] > v[b] ? v[b] : v[a]; v[a] = x_; }
  MSA_CX(0, 1) MSA_CX(2, 3) MSA_CX(0, 2) MSA_CX(1, 3) MSA_CX(1, 2)
#undef MSA_CX
  uint32_t t_w = 0;
  for (int r = 0; r < m; ++r) {
    const uint32_t x = __reduce_max_sync(0xffffffffu, (uint32_t)(v[0] >> 32));
    t_w = x;
    // one owner of the maximum score drops it (scores may tie: the lowest such lane)
    const unsigned own = __ballot_sync(0xffffffffu, (uint32_t)(v[0] >> 32) == x);
    if (lane == __ffs(own) - 1) {
      v[0] = v[1];
      v[1] = v[2];
      v[2] = v[3];
      v[3] = 0ull;
    }
  }
  uint32_t* warp_t32 = reinterpret_cast<uint32_t*>(warp_t);
  if (lane == 0) warp_t32[warp] = t_w;
  __syncthreads();
  // T: the smallest warp threshold
  const uint32_t T = __reduce_min_sync(0xffffffffu, lane < nw ? warp_t32[lane] : 0xffffffffu);
  const bool p0 = v0 != 0ull && (uint32_t)(v0 >> 32) >= T, p1 = v1 != 0ull && (uint32_t)(v1 >> 32) >= T;
  const bool p2 = v2 != 0ull && (uint32_t)(v2 >> 32) >= T, p3 = v3 != 0ull && (uint32_t)(v3 >> 32) >= T;
  const unsigned b0 = __ballot_sync(0xffffffffu, p0), b1 = __ballot_sync(0xffffffffu, p1);
  const unsigned b2 = __ballot_sync(0xffffffffu, p2), b3 = __ballot_sync(0xffffffffu, p3);
  const int n0 = __popc(b0), n1 = __popc(b1), n2 = __popc(b2), n3 = __popc(b3);
  uint32_t base = 0;
  if (lane == 0 && n0 + n1 + n2 + n3 > 0) base = atomicAdd(count, (uint32_t)(n0 + n1 + n2 + n3));
  base = __shfl_sync(0xffffffffu, base, 0);
  const unsigned below = (1u << lane) - 1u;
  if (p0 && base + __popc(b0 & below) < (uint32_t)kTopkMaxCand) cand[base + __popc(b0 & below)] = v0;
  base += n0;
  if (p1 && base + __popc(b1 & below) < (uint32_t)kTopkMaxCand) cand[base + __popc(b1 & below)] = v1;
  base += n1;
  if (p2 && base + __popc(b2 & below) < (uint32_t)kTopkMaxCand) cand[base + __popc(b2 & below)] = v2;
  base += n2;
  if (p3 && base + __popc(b3 & below) < (uint32_t)kTopkMaxCand) cand[base + __popc(b3 & below)] = v3;
  __syncthreads();
  const int c = (int)*count;
  if (c > kTopkMaxCand) {
    __syncthreads();  // every thread has read the count before the fallback reuses the scratch
    return false;
  }
  // rank of each candidate among the candidates: 8 independent partial counts per step
  for (int i = tid; i < c; i += blockDim.x) {
    const uint64_t x = cand[i];
    int r8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int j = 0;
    for (; j + 8 <= c; j += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u) r8[u] += cand[j + u] > x;
    }
    for (; j < c; ++j) r8[0] += cand[j] > x;
    const int rank = ((r8[0] + r8[1]) + (r8[2] + r8[3])) + ((r8[4] + r8[5]) + (r8[6] + r8[7]));
    if (rank < k) out[rank] = x;
  }
  __syncthreads();
  return true;
}

// any k (up to 256): radix select from the most significant byte; it stops as soon as the
// k-th key's bucket is taken whole; tmp holds k unsorted winners, then a rank sort
__device__ void block_topk_radix(const uint64_t* keys, int n, int k, uint64_t* out, uint64_t* tmp, uint32_t* hist,
                                 uint64_t* sh_state) {
  const int tid = threadIdx.x, nt = blockDim.x;
  uint64_t prefix = 0, mask = 0;
  int kk = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    // one shared-memory atomic per distinct digit per warp: scores cluster in a few digits
    // (the high bytes of nearby floats agree), and per-lane atomics on one address serialise
    for (int i0 = 0; i0 < n; i0 += nt) {
      const int i = i0 + tid;
      uint64_t key = 0;
      bool in = false;
      if (i < n) {
        key = keys[i];
        in = (key & mask) == prefix;
      }
      const unsigned act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const uint32_t digit = (uint32_t)(key >> shift) & 255u;
        const unsigned grp = __match_any_sync(act, digit);
        if ((threadIdx.x & 31) == __ffs(grp) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(grp));
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane L owns digits 255-8L .. 248-8L (descending)
      uint32_t cnt[8];
      uint32_t tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - 8 * tid - j];
        tot += cnt[j];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += v;
      }
      const uint32_t excl = incl - tot;  // keys in higher digits than this lane's range
      if (excl < (uint32_t)kk && (uint32_t)kk <= incl) {
        uint32_t above = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above < (uint32_t)kk && (uint32_t)kk <= above + cnt[j]) {
            sh_state[0] = above;
            sh_state[1] = (uint64_t)(255 - 8 * tid - j);
            sh_state[3] = (above + cnt[j] == (uint32_t)kk) ? 1ull : 0ull;  // bucket taken whole
            break;
          }
          above += cnt[j];
        }
      }
    }
    __syncthreads();
    kk -= (int)sh_state[0];
    prefix |= (sh_state[1] & 255ull) << shift;
    mask |= 255ull << shift;
    const bool done = sh_state[3] != 0;
    __syncthreads();
    if (done) break;
  }
  // the winners are the keys whose decided high bits are >= prefix (exactly k of them)
  if (tid == 0) sh_state[2] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += nt) {
    const uint64_t key = keys[i];
    if ((key & mask) >= prefix) {
      const int pos = (int)atomicAdd(reinterpret_cast<unsigned long long*>(&sh_state[2]), 1ull);
      if (pos < k) tmp[pos] = key;
    }
  }
  __syncthreads();
  // rank sort: keys are distinct, so each winner's rank is the number of larger winners
  for (int i = tid; i < k; i += nt) {
    const uint64_t key = tmp[i];
    int rank = 0;
    for (int j = 0; j < k; ++j) rank += tmp[j] > key;
    out[rank] = key;
  }
  __syncthreads();
}

// shared memory after the keys: out[256], tmp[256], state[4] (64-bit), hist[256] (32-bit),
// lists[kTopkThreads] (64-bit)
struct TopkScratch {
  uint64_t *out, *tmp, *state, *lists;
  uint32_t* hist;
  __device__ explicit TopkScratch(uint64_t* base) {
    out = base;
    tmp = out + 256;
    state = tmp + 256;
    hist = reinterpret_cast<uint32_t*>(state + 4);
    lists = reinterpret_cast<uint64_t*>(hist + 256);
  }
};
constexpr size_t kTopkScratchBytes = (512 + 4) * sizeof(uint64_t) + 256 * sizeof(uint32_t) + kTopkThreads * 8;

__device__ void block_topk(const uint64_t* keys, int n, int k, const TopkScratch& t) {
  if (k > 32) block_topk_radix(keys, n, k, t.out, t.tmp, t.hist, t.state);
  else if (!block_topk_threshold(keys, n, k, t.out, t.lists, t.tmp, t.hist)) block_topk_small(keys, n, k, t.out, t.lists);
}

__device__ __forceinline__ uint64_t make_key(uint32_t ordered, int id) {
  return ((uint64_t)ordered << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)id);
}

// top-k of one slice of documents for query b (whole block): document scores from the
// scan's max keys (or the mean of its chunk keys), written out when asked, then the block
// top-k; with one slice the result is final, otherwise the slice's winners become
// candidates for the merge.  sm64 holds kSliceDocs 64-bit keys, then the TopkScratch.
__device__ void slice_topk(const uint32_t* doc_key, const uint32_t* chunk_k, const int32_t* chunk_off, int n_docs,
                           int n_chunks, int k, int n_slices, float* doc_scores, uint64_t* cand, int32_t* topk_idx,
                           float* topk_score, int slice, int b, uint64_t* sm64) {
  uint64_t* keys = sm64;  // [kSliceDocs]
  const TopkScratch ts(keys + kSliceDocs);
  uint64_t* out = ts.out;
  const int d0 = slice * kSliceDocs;
  const int n = min(kSliceDocs, n_docs - d0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int doc = d0 + i;
    uint32_t ok;
    if (chunk_k) {
      const int c0 = __ldg(&chunk_off[doc]), c1 = __ldg(&chunk_off[doc + 1]);
      float s = 0.f;
      for (int j = c0; j < c1; ++j) s += ordered_to_float(__ldcg(&chunk_k[(size_t)b * n_chunks + j]));
      const float mean = s / (float)max(1, c1 - c0);
      ok = float_to_ordered(mean);
    } else {
      ok = __ldcg(&doc_key[(size_t)b * n_docs + doc]);
    }
    if (doc_scores) doc_scores[(size_t)b * n_docs + doc] = ordered_to_float(ok);
    keys[i] = make_key(ok, doc);
  }
  __syncthreads();
  const int kk = min(k, n);
  block_topk(keys, n, kk, ts);
  if (n_slices == 1) {
    for (int i = threadIdx.x; i < kk; i += blockDim.x) {
      topk_idx[(size_t)b * k + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(out[i] & 0xFFFFFFFFu));
      topk_score[(size_t)b * k + i] = ordered_to_float((uint32_t)(out[i] >> 32));
    }
  } else {
    for (int i = threadIdx.x; i < k; i += blockDim.x)
      cand[((size_t)b * n_slices + slice) * k + i] = (i < kk) ? out[i] : 0ull;
  }
  __syncthreads();  // shared memory free for the next call
}

__device__ void merge_topk(const uint64_t* cand, int n_slices, int k, int32_t* topk_idx, float* topk_score, int b,
                           uint64_t* sm64);

// top-k of one slice of documents for query blockIdx.y; with several slices and merge_ticket set
// (their candidates fit in one slice's keys), the slice that finishes last for its query also
// merges the query's candidates (a ticket per query), sparing the merge kernel
__global__ void __launch_bounds__(kTopkThreads) topk_slice_kernel(
    const uint32_t* __restrict__ doc_key, const uint32_t* __restrict__ chunk_k, const int32_t* __restrict__ chunk_off,
    int n_docs, int n_chunks, int k, int n_slices, float* __restrict__ doc_scores, uint64_t* __restrict__ cand,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_score, uint32_t* __restrict__ merge_ticket) {
  extern __shared__ uint64_t sm64[];
  __shared__ bool last;
  pdl_enter();
  slice_topk(doc_key, chunk_k, chunk_off, n_docs, n_chunks, k, n_slices, doc_scores, cand, topk_idx, topk_score,
             blockIdx.x, blockIdx.y, sm64);
  if (!merge_ticket || n_slices == 1) return;
  const int b = blockIdx.y;
  __threadfence();  // this slice's candidates are visible before its ticket
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&merge_ticket[b], 1u) == (uint32_t)(n_slices - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x == 0) merge_ticket[b] = 0u;  // ready for the next call (also cleared by the router query)
  merge_topk(cand, n_slices, k, topk_idx, topk_score, b, sm64);
}

// the global top-k of query b from its slices' winners (n_slices * k keys in shared memory first)
__device__ void merge_topk(const uint64_t* cand, int n_slices, int k, int32_t* topk_idx, float* topk_score, int b,
                           uint64_t* sm64) {
  const int n = n_slices * k;
  uint64_t* keys = sm64;
  const TopkScratch ts(keys + n);
  uint64_t* out = ts.out;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = __ldcg(&cand[(size_t)b * n + i]);
  __syncthreads();
  block_topk(keys, n, k, ts);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    topk_idx[(size_t)b * k + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(out[i] & 0xFFFFFFFFu));
    topk_score[(size_t)b * k + i] = ordered_to_float((uint32_t)(out[i] >> 32));
  }
}

__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(const uint64_t* __restrict__ cand,
                                                                  int n_slices, int k,
                                                                  int32_t* __restrict__ topk_idx,
                                                                  float* __restrict__ topk_score) {
  extern __shared__ uint64_t sm64[];
  pdl_enter();
  merge_topk(cand, n_slices, k, topk_idx, topk_score, blockIdx.x, sm64);
}

// exact top-k of (score, global document id) candidate pairs, one block per query
__global__ void __launch_bounds__(kTopkThreads) topk_merge_pairs_kernel(const float* __restrict__ cand_score,
                                                                        const int32_t* __restrict__ cand_idx,
                                                                        int n_cand, int k,
                                                                        int32_t* __restrict__ topk_idx,
                                                                        float* __restrict__ topk_score) {
  extern __shared__ uint64_t sm64[];
  uint64_t* keys = sm64;
  const TopkScratch ts(keys + n_cand);
  uint64_t* out = ts.out;
  pdl_enter();
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < n_cand; i += blockDim.x)
    keys[i] = make_key(float_to_ordered(cand_score[(size_t)b * n_cand + i]), cand_idx[(size_t)b * n_cand + i]);
  __syncthreads();
  block_topk(keys, n_cand, k, ts);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    topk_idx[(size_t)b * k + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(out[i] & 0xFFFFFFFFu));
    topk_score[(size_t)b * k + i] = ordered_to_float((uint32_t)(out[i] >> 32));
  }
}

template <int DR, int NQ, bool MEAN, bool MAPPED = false>
cudaError_t launch_scan_t(const CUtensorMap& kmap, const CUtensorMap& qmap, const ScanParams& p, int grid,
                          cudaStream_t s) {
  auto kern = scan_kernel<DR, NQ, MEAN, MAPPED>;
  static_assert(kSliceDocs * sizeof(uint64_t) + kTopkScratchBytes <=
                    (size_t)ScanGeom<DR, NQ>::kStages * ScanGeom<DR, NQ>::kStageBytes,
                "the fused top-k reuses the pipeline stages");
  const size_t smem = ScanGeom<DR, NQ>::kSmemBytes;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kScanThreads), smem, s, kmap, qmap, p);
}

cudaError_t launch_scan(int d_r, int nq, bool mean, const CUtensorMap& kmap, const CUtensorMap& qmap,
                        const ScanParams& p, int grid, cudaStream_t s) {
  if (!mean && p.chunk_doc) {  // the epilogue reads each row's document from the map
    if (d_r == 128) return nq == 16 ? launch_scan_t<128, 16, false, true>(kmap, qmap, p, grid, s)
                                    : launch_scan_t<128, 32, false, true>(kmap, qmap, p, grid, s);
    return nq == 16 ? launch_scan_t<64, 16, false, true>(kmap, qmap, p, grid, s)
                    : launch_scan_t<64, 32, false, true>(kmap, qmap, p, grid, s);
  }
  if (d_r == 128) {
    if (nq == 16) return mean ? launch_scan_t<128, 16, true>(kmap, qmap, p, grid, s)
                              : launch_scan_t<128, 16, false>(kmap, qmap, p, grid, s);
    return mean ? launch_scan_t<128, 32, true>(kmap, qmap, p, grid, s)
                : launch_scan_t<128, 32, false>(kmap, qmap, p, grid, s);
  }
  if (nq == 16) return mean ? launch_scan_t<64, 16, true>(kmap, qmap, p, grid, s)
                            : launch_scan_t<64, 16, false>(kmap, qmap, p, grid, s);
  return mean ? launch_scan_t<64, 32, true>(kmap, qmap, p, grid, s)
              : launch_scan_t<64, 32, false>(kmap, qmap, p, grid, s);
}

// 1 / max(||K̄^R_jh||, eps) of every pooled router key (one pass over K̄^R): lanes of a row
// each take 16 bytes (coalesced), the row's lanes reduce with shuffles
__global__ void __launch_bounds__(256) kr_norms_kernel(const __nv_bfloat16* __restrict__ KR, int n_chunks, int n_r,
                                                       int d_r, int head_major, float* __restrict__ inv_norm) {
  pdl_enter();
  const int L = d_r / 8;  // lanes per row (16 or 8)
  const int lane = threadIdx.x & 31;
  const int rpw = 32 / L;  // rows per warp step
  const size_t n_rows = (size_t)n_chunks * n_r;
  const size_t warp_id = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const size_t n_warps = (size_t)gridDim.x * blockDim.x / 32;
  for (size_t r0 = warp_id * rpw; r0 < n_rows; r0 += n_warps * rpw) {  // warp-uniform
    const size_t r = r0 + lane / L;
    const bool ok = r < n_rows;
    const uint4 w = ok ? __ldg(reinterpret_cast<const uint4*>(KR + r * d_r) + (lane % L)) : make_uint4(0, 0, 0, 0);
    float ss = 0.f;
    float2 f;
    f = unpack_bf16x2(w.x); ss = fmaf(f.x, f.x, ss); ss = fmaf(f.y, f.y, ss);
    f = unpack_bf16x2(w.y); ss = fmaf(f.x, f.x, ss); ss = fmaf(f.y, f.y, ss);
    f = unpack_bf16x2(w.z); ss = fmaf(f.x, f.x, ss); ss = fmaf(f.y, f.y, ss);
    f = unpack_bf16x2(w.w); ss = fmaf(f.x, f.x, ss); ss = fmaf(f.y, f.y, ss);
    for (int o = 1; o < L; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (ok && lane % L == 0) {
      const size_t out = head_major ? (r % n_chunks) * n_r + r / n_chunks : r;
      inv_norm[out] = 1.0f / fmaxf(sqrtf(ss), kEps);
    }
  }
}

size_t topk_slice_smem() { return kSliceDocs * sizeof(uint64_t) + kTopkScratchBytes; }
size_t topk_merge_smem(int n) { return (size_t)n * sizeof(uint64_t) + kTopkScratchBytes; }

}  // namespace

msa_status topk_merge_launch(const float* cand_score, const int32_t* cand_idx, int B, int n_cand, int k,
                             int32_t* topk_idx, float* topk_score, cudaStream_t s) {
  TraceScope ts(kKTopkMerge, s);
  const size_t sm = topk_merge_smem(n_cand);
  MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(topk_merge_pairs_kernel), (int)sm));
  MSA_CUDA_CHECK(launch_pdl(topk_merge_pairs_kernel, dim3(B), dim3(kTopkThreads), sm, s, cand_score, cand_idx, n_cand,
                            k, topk_idx, topk_score));
  return MSA_OK;
}

msa_status kr_norms_launch(const msa_dims& d, const void* KR_bar, int n_chunks, int kr_layout, float* inv_norm,
                           cudaStream_t s) {
  TraceScope ts(kKKrNorms, s);
  const size_t n_rows = (size_t)n_chunks * d.n_r;
  const int rows_per_cta = 256 / (d.d_r / 8);
  const int blocks = (int)std::max<size_t>(1, std::min<size_t>((n_rows + rows_per_cta - 1) / rows_per_cta,
                                                               (size_t)sm_count() * 8));
  MSA_CUDA_CHECK(launch_pdl(kr_norms_kernel, dim3(blocks), dim3(256), 0, s, static_cast<const __nv_bfloat16*>(KR_bar),
                            n_chunks, d.n_r, d.d_r, kr_layout, inv_norm));
  return MSA_OK;
}

size_t route_workspace(const msa_dims& d, int B, int M, int n_docs, int n_chunks, int k, msa_doc_agg agg, void* ws,
                       RouteWs* out) {
  Carver cv(ws);
  RouteWs w{};
  const int R = B * M;  // query-token rows
  w.nq = R <= 16 ? 16 : 32;
  w.passes = (R + w.nq - 1) / w.nq;
  w.n_slices = (n_docs + kSliceDocs - 1) / kSliceDocs;
  w.q_hl = cv.take<__nv_bfloat16>((size_t)w.passes * d.n_r * 2 * w.nq * d.d_r);
  w.scan_ticket = cv.take<uint32_t>(1 + (size_t)B);  // the tickets, then the document keys: one region
  w.doc_key = agg == MSA_AGG_MAX ? cv.take<uint32_t>((size_t)B * n_docs) : nullptr;
  w.chunk_k = agg == MSA_AGG_MEAN ? cv.take<uint32_t>((size_t)B * n_chunks) : nullptr;
  w.cand = w.n_slices > 1 ? cv.take<uint64_t>((size_t)B * w.n_slices * k) : nullptr;
  if (out) *out = w;
  return cv.size();
}

namespace {
// each chunk's document: one warp per document writes its id over its chunks; chunks outside
// [chunk_off[0], chunk_off[n_docs]) get -1
__global__ void __launch_bounds__(256) chunk_doc_kernel(const int32_t* __restrict__ chunk_off, int n_docs,
                                                        int n_chunks, int32_t* __restrict__ chunk_doc) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  for (int d = gw; d < n_docs; d += warps) {
    const int c0 = max(0, __ldg(&chunk_off[d])), c1 = min(n_chunks, __ldg(&chunk_off[d + 1]));
    for (int c = c0 + lane; c < c1; c += 32) chunk_doc[c] = d;
  }
  const int lo = min(n_chunks, max(0, __ldg(&chunk_off[0]))), hi = max(lo, min(n_chunks, __ldg(&chunk_off[n_docs])));
  const int t = blockIdx.x * blockDim.x + threadIdx.x, nt = gridDim.x * blockDim.x;
  for (int c = t; c < lo; c += nt) chunk_doc[c] = -1;
  for (int c = hi + t; c < n_chunks; c += nt) chunk_doc[c] = -1;
}
}  // namespace

msa_status chunk_doc_launch(const int32_t* chunk_off, int n_docs, int n_chunks, int32_t* chunk_doc, cudaStream_t s) {
  const int blocks = std::max(1, std::min(4 * sm_count(), (n_docs + 7) / 8));
  TraceScope ts(kKChunkDoc, s);
  MSA_CUDA_CHECK(launch_pdl(chunk_doc_kernel, dim3(blocks), dim3(256), 0, s, chunk_off, n_docs, n_chunks, chunk_doc));
  return MSA_OK;
}

size_t route_query_bytes(const msa_dims& d, int B, int M) {
  const int R = B * M, nq = R <= 16 ? 16 : 32;
  return (size_t)((R + nq - 1) / nq) * d.n_r * 2 * nq * d.d_r * sizeof(__nv_bfloat16);
}

void route_clear_region(const msa_dims& d, int B, int M, int n_docs, int n_chunks, int k, void* ws, void** ptr,
                        size_t* bytes) {
  RouteWs w;
  route_workspace(d, B, M, n_docs, n_chunks, k, MSA_AGG_MAX, ws, &w);
  *ptr = w.scan_ticket;
  *bytes = (size_t)(reinterpret_cast<char*>(w.doc_key + (size_t)B * n_docs) - reinterpret_cast<char*>(w.scan_ticket));
}

msa_status route_query_launch(const msa_dims& d, const void* Hq, const void* W_QR, int B, int M, void* q_hl,
                              uint32_t* clear, size_t n_clear, uint32_t* tickets, int n_tickets, cudaStream_t s,
                              bool early_inputs) {
  const int R = B * M, nq = R <= 16 ? 16 : 32, passes = (R + nq - 1) / nq;
  __nv_bfloat16* q = static_cast<__nv_bfloat16*>(q_hl);
  TraceScope ts(kKRouterQuery, s);
  if (W_QR) {
    const size_t sm = rq_smem_bytes(d.d_r);
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(router_query_kernel), (int)sm));
    MSA_CUDA_CHECK(launch_pdl_cluster(router_query_kernel, dim3(kRqCluster, d.n_r), dim3(kRqThreads), sm, s,
                                      kRqCluster, static_cast<const __nv_bfloat16*>(Hq),
                                      static_cast<const __nv_bfloat16*>(W_QR), R, passes * nq, d.hidden, d.n_r, d.d_r,
                                      nq, rq_split_rows(d.hidden), q, clear, n_clear, tickets, n_tickets,
                                      early_inputs ? 1 : 0));
  } else {
    MSA_CUDA_CHECK(launch_pdl(router_query_direct_kernel, dim3(1, d.n_r), dim3(kRqThreads), 0, s,
                              static_cast<const __nv_bfloat16*>(Hq), R, passes * nq, d.n_r, d.d_r, nq, q, clear,
                              n_clear, tickets, n_tickets, early_inputs ? 1 : 0));
  }
  return MSA_OK;
}

msa_status route_launch(const msa_dims& d, const void* Hq, const void* W_QR, int B, int M, const void* KR_bar,
                        const int32_t* chunk_off, int n_docs, int n_chunks, int k, msa_doc_agg agg, int kr_layout,
                        const float* kr_inv_norm, float* doc_scores, int32_t* topk_idx, float* topk_score, void* ws, cudaStream_t s,
                        bool early_inputs, RoutePart part, int scan_sm_reserve, const void* q_ext,
                        const int32_t* chunk_doc, bool after_scan) {
  RouteWs w;
  route_workspace(d, B, M, n_docs, n_chunks, k, agg, ws, &w);
  const int NR = d.n_r * d.d_r;
  const int R = B * M;
  const bool mean = agg == MSA_AGG_MEAN;
  // keys folded in with atomicMax start at 0 (below every ordered score): the document keys,
  // and the chunk keys when several tokens of a query meet in one chunk
  uint32_t* clear = mean ? (M > 1 ? w.chunk_k : nullptr) : w.doc_key;
  // few queries over one slice of documents: the scan's last CTA runs the top-k itself
  const bool fuse_topk = w.n_slices == 1 && w.passes == 1 && B <= kFuseTopkMaxQueries;
  const size_t n_clear = clear ? (size_t)B * (mean ? n_chunks : n_docs) : 0;
  // the scoring parts (kScore, kScan) leave the separate top-k kernels to the selection part
  const bool score = part != RoutePart::kSelect;
  const bool select = part == RoutePart::kAll || part == RoutePart::kSelect;

  // K1: router query (projection, normalisation, hi/lo layout) and document keys cleared
  if (score && part != RoutePart::kScan) {
    msa_status st = route_query_launch(d, Hq, W_QR, B, M, w.q_hl, clear, n_clear, w.scan_ticket, 1 + B, s,
                                       early_inputs);
    if (st != MSA_OK) return st;
  }
  const void* q_src = part == RoutePart::kScan ? q_ext : w.q_hl;
  // K3: scan, NQ (16 or 32) queries per pass
  if (score) {
    CUtensorMap kmap, qmap;
    msa_status st;
    if (kr_layout == 1) {  // head-major [n_r][C][d_r]: one head's rows are contiguous
      const uint64_t dims[3] = {(uint64_t)d.d_r, (uint64_t)n_chunks, (uint64_t)d.n_r};
      const uint64_t strides[2] = {(uint64_t)d.d_r * 2, (uint64_t)n_chunks * d.d_r * 2};
      const uint32_t box[3] = {64, (uint32_t)kScanM, 1};
      st = encode_tensor_map(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(KR_bar), dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
      const uint64_t dims[2] = {(uint64_t)NR, (uint64_t)n_chunks};
      const uint64_t strides[1] = {(uint64_t)NR * 2};
      const uint32_t box[2] = {64, (uint32_t)kScanM};
      st = encode_tensor_map(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(KR_bar), dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (st != MSA_OK) return st;
    const uint64_t qdims[2] = {(uint64_t)d.d_r, (uint64_t)w.passes * d.n_r * 2 * w.nq};
    const uint64_t qstrides[1] = {(uint64_t)d.d_r * 2};
    const uint32_t qbox[2] = {64, (uint32_t)w.nq};
    st = encode_tensor_map(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q_src), qdims, qstrides,
                           qbox, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    const int n_tiles = (n_chunks + kScanM - 1) / kScanM;
    const int grid = std::max(1, std::min(sm_count() - std::max(0, scan_sm_reserve), n_tiles));
    uint32_t cols = 32;
    // columns: 2 NQ per head (hi and lo side by side), two tiles in flight for NQ = 16, one for 32
    while (cols < (w.nq == 16 ? 2u : 1u) * d.n_r * 2u * w.nq) cols <<= 1;
    for (int pass = 0; pass < w.passes; ++pass) {
      ScanParams p;
      p.chunk_off = chunk_off;
      p.doc_key = w.doc_key;
      p.chunk_k = w.chunk_k;
      p.ticket = fuse_topk ? w.scan_ticket : nullptr;
      p.n_queries = B;
      p.k = k;
      p.doc_scores = doc_scores;
      p.topk_idx = topk_idx;
      p.topk_score = topk_score;
      p.q_tokens = M;
      p.n_r = d.n_r;
      p.n_docs = n_docs;
      p.n_chunks = n_chunks;
      p.n_tiles = n_tiles;
      p.q_base = pass * w.nq;
      p.q_count = std::min(R - p.q_base, w.nq);
      p.pass = pass;
      p.head_major = kr_layout == 1;
      p.inv_norm = kr_inv_norm;
      p.chunk_doc = chunk_doc;
      p.wait_prior = (pass == 0 && after_scan) ? 0 : 1;
      p.tmem_cols = cols;
      p.inv_nr = 1.0f / (float)d.n_r;
      TraceScope ts(kKScan, s);
      cudaError_t e = launch_scan(d.d_r, w.nq, mean, kmap, qmap, p, grid, s);
      if (e != cudaSuccess) return cuda_fail(e, "scan_kernel launch");
    }
  }
  // K4: top-k; the slices' winners merged by the last slice of each query when they fit in one
  // slice's keys, otherwise by the merge kernel
  const bool fuse_merge = w.n_slices > 1 && (size_t)w.n_slices * k <= (size_t)kSliceDocs;
  if (!select) return MSA_OK;
  if (!fuse_topk) {
    TraceScope ts(kKTopkSlice, s);
    const size_t sm = topk_slice_smem();
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(topk_slice_kernel), (int)sm));
    MSA_CUDA_CHECK(launch_pdl(topk_slice_kernel, dim3(w.n_slices, B), dim3(kTopkThreads), sm, s,
                              (const uint32_t*)w.doc_key, (const uint32_t*)w.chunk_k, chunk_off, n_docs, n_chunks, k,
                              w.n_slices, doc_scores, w.cand, topk_idx, topk_score,
                              fuse_merge ? w.scan_ticket + 1 : nullptr));
  }
  if (w.n_slices > 1 && !fuse_merge) {
    TraceScope ts(kKTopkMerge, s);
    const size_t sm = topk_merge_smem(w.n_slices * k);
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(topk_merge_kernel), (int)sm));
    MSA_CUDA_CHECK(launch_pdl(topk_merge_kernel, dim3(B), dim3(kTopkThreads), sm, s, (const uint64_t*)w.cand,
                              w.n_slices, k, topk_idx, topk_score));
  }
  return MSA_OK;
}

}  // namespace msa

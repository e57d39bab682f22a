// Stage 3 of MSA: sparse generation attention for one decode step.
//
// Definition (IRMaD reading of the MSA paper, "M. Materials & Methods",
// routing item and position item; project overview, key technical details 1):
//   K_ctx = [{K̄_i}_{i in I}; K_q],  V_ctx = [{V̄_i}_{i in I}; V_q],
//   Output = Attention(Q_q, K_ctx, V_ctx),
// with global RoPE on the active context offset by k: local token j at
// pos_offset + j, the decode query (last local token) at pos_offset + L - 1.
//
// Kernels:
//   rope_table_kernel    cos/sin of (pos_offset + j) * theta_i for every local
//                        position j (angles from 64-bit fixed-point turns)
//   attn_split_kernel    split-KV flash-decode, persistent: each CTA takes work
//                        items (a run of local keys, or a run of the selected
//                        chunks, of one query token group); a producer warp
//                        gathers the rows with per-row bulk async copies into
//                        padded shared memory; one compute warp per KV head runs
//                        QK^T and PV on the tensor cores (mma.sync, the GQA group
//                        x the CTA's query tokens as the M rows), rotates local
//                        keys in registers when needed, online softmax; the local
//                        items can run before the routing result is known
//   attn_combine_kernel, attn_combine_warp_kernel
//                        log-sum-exp merge of the split partials -> bf16
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace msa {

struct AttendWs {
  float2* rope_tab;  // [t_loc_max][D/2] (cos, sin)
  float* part_ml;    // [B][n_q][S][2]  running max (log2 domain) and sum
  float* part_o;     // [B][n_q][S][D]  unnormalised output
  int n_split_local;   // splits of the local keys (partial slots 0 .. n_split_local - 1)
  int n_split_chunk;   // splits of the selected chunks (the slots after the local ones)
  int n_parts;         // partial slots per (query token, q head)
};

namespace {

constexpr int kTK = 16;          // keys per tile (one mma K-step of P V)
constexpr int kMaxStages = 4;
constexpr int kMaxK = 256;
constexpr int kMaxSplits = 1024;
constexpr int kChunksPerDocEst = 40;  // expected pooled chunks per selected document (split planning only)
constexpr int kLatencyGroups = 8;     // (query, token group)s up to which the split plan is one wave
constexpr int kCoSmemMax = 4096;      // chunk_off entries the split kernel may keep in shared memory
constexpr float kLog2e = 1.4426950408889634f;

// cos/sin of (pos_offset + j) * theta_i, theta_i = base^(-2i/D), for local positions j
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ tab, int t_loc_max, int half,
                                                         int pos_offset, const RopeTurns turns) {
  pdl_enter();
  const int64_t n = (int64_t)t_loc_max * half;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(e / half), i = (int)(e % half);
    tab[e] = rope_cos_sin(turns, i, (int64_t)pos_offset + j);
  }
}

struct AttnParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* K_bar;
  const __nv_bfloat16* V_bar;
  const int32_t* chunk_off;
  const int32_t* topk_idx;
  const __nv_bfloat16* K_loc;
  const __nv_bfloat16* V_loc;
  const int32_t* loc_len;
  const __nv_bfloat16* k_new;  // [B][n_kv][D] the new token's key (before RoPE), or null: no append
  const __nv_bfloat16* v_new;  // [B][n_kv][D] its value
  int append_rotate;           // the appended key is rotated at its position (rotated cache)
  const float2* rope_tab;
  float* part_ml;
  float* part_o;
  int n_q, n_kv, k, n_docs, t_loc_max, pos_offset, n_stages;
  int n_queries;     // B
  int q_tokens;      // M: query tokens per query (the last M local tokens)
  int n_loc_splits;    // this launch's splits of the local keys (0: none)
  int n_chunk_splits;  // this launch's splits of the selected chunks (0: none)
  int chunk_part_base;  // partial slot of chunk split 0 (the local splits take slots 0 ..)
  int n_parts;       // partial slots per (query token, q head)
  int early;         // local-key items run before the predecessor kernel has finished
  int doc_base;      // global id of chunk_off's first document (topk_idx holds global ids)
  int foreign_ok;    // a selected document outside [doc_base, doc_base + n_docs) is another rank's: skipped
  int co_cap;        // chunk_off entries copied to shared memory (n_docs + 1), or 0 (read from L2)
  int tok_per_cta;   // MT: tokens per CTA, MT * G <= 16 mma rows
  int n_tgroups;     // ceil(M / MT)
  float scale_log2;  // softmax scale * log2(e)
  RopeTurns turns;   // RoPE frequencies as 64-bit fractions of a turn
};

// Shared memory of one CTA (dynamic size, n_stages stages):
//   stage s: K rows [kTK][krow] | V rows [kTK][krow] | RoPE rows [kTK][D/2] (cos, sin)
//   krow = n_kv * D * 2 + 16 bytes: one key's rows of every KV head, padded so
//   that consecutive rows start one 16-byte unit apart (conflict-free ldmatrix)
//   then barriers, the segment table, the query tokens' cos/sin and raw rows.
struct AttnSmem {
  int krow, kbytes, tbytes, stage_bytes, n_stages;
  __host__ __device__ AttnSmem(int n_kv, int D, int stages, bool table) {
    krow = n_kv * D * 2 + 16;
    kbytes = kTK * krow;
    tbytes = table ? kTK * (D / 2) * 8 : 0;
    stage_bytes = 2 * kbytes + tbytes;
    n_stages = stages;
  }
  // two query buffers, barriers (ring, item header and selection), two item headers and
  // segment tables, the tokens' cos/sin, the document table (co_cap entries, 16-byte multiple)
  __host__ __device__ size_t fixed_bytes(int n_q, int D, int mt, int co_cap) const {
    return 2 * (size_t)mt * n_q * D * 2 + (2 * kMaxStages + 6) * 8 + 2 * 8 * 4 + 2 * (2 * kMaxK + 2) * 4 +
           (size_t)mt * (D / 2) * 8 + (size_t)(co_cap + 3) / 4 * 16;
  }
  __host__ __device__ size_t total(int n_q, int D, int mt, int co_cap) const {
    return (size_t)n_stages * stage_bytes + fixed_bytes(n_q, D, mt, co_cap);
  }
};

// TABLE: the local keys are rotated in registers with the RoPE rows of p.rope_tab (a cache of
// unrotated keys); without it they are used as stored (a cache of rotated keys)
template <int D, bool TABLE>
__global__ void __launch_bounds__(288, 1) attn_split_kernel(const AttnParams p) {
  constexpr int KS = D / 16;
  constexpr int NBLK = D / 8;
  const int n_kv = p.n_kv, G = p.n_q / n_kv;
  constexpr bool table = TABLE;  // local keys still need their global rotation
  const AttnSmem L_(n_kv, D, p.n_stages, table);
  extern __shared__ __align__(128) uint8_t sm[];
  // offsets: every region below starts on a 16-byte boundary (stage rows, query rows and
  // the RoPE rows are bulk-copy or 16-byte vector destinations)
  uint8_t* stage_mem = sm;
  const int MT = p.tok_per_cta;
  const size_t q_elems = (size_t)MT * p.n_q * D;
  uint16_t* qsm = reinterpret_cast<uint16_t*>(sm + (size_t)L_.n_stages * L_.stage_bytes);  // [2][MT][n_q][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(qsm + 2 * q_elems);  // [stage] tile landed
  uint64_t* ebars = bars + kMaxStages;                               // [stage] every warp done with it
  uint64_t* hfull = ebars + kMaxStages;                              // [2] an item's header and query landed
  uint64_t* hempty = hfull + 2;                                      // [2] every warp done with them
  uint64_t* hsel = hempty + 2;                                       // [2] the item's key range is known
  int* hdr = reinterpret_cast<int*>(hsel + 2);                       // [2][8] item headers
  int* segs = hdr + 16;                                              // [2][2 kMaxK + 2] segment tables
  float2* qcs = reinterpret_cast<float2*>(segs + 2 * (2 * kMaxK + 2));  // [MT][D/2] cos/sin at the tokens' positions
  int* co_sm = reinterpret_cast<int*>(qcs + (size_t)MT * (D / 2));   // [co_cap] chunk_off
  __shared__ int abort_flag;                                         // a bounded wait of this CTA gave up

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = warp;               // the KV head this warp serves (warps 0 .. n_kv-1)
  const bool producer = warp == n_kv;  // the last warp builds each item and streams its tiles
  const int k = p.k;
  // items: every (query, token group)'s local-key splits first, then its selected-chunk
  // splits; this CTA takes items blockIdx.x, + gridDim.x, ... in increasing order, so its
  // local-key items come first
  const int n_groups = p.n_queries * p.n_tgroups;
  const int n_loc_items = p.n_loc_splits * n_groups;
  const int n_items = n_loc_items + p.n_chunk_splits * n_groups;

  // ---- no global memory yet: overlaps the previous kernel's tail ----
  for (int i = tid; i < L_.n_stages * L_.stage_bytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(stage_mem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    for (int s = 0; s < L_.n_stages; ++s) {
      mbar_init(&bars[s], 1);
      mbar_init(&ebars[s], n_kv);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&hfull[s], 1);
      mbar_init(&hempty[s], n_kv);
      mbar_init(&hsel[s], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Without `early` every thread waits for the predecessor here.  With it, the caller has
  // guaranteed that q, the local KV, loc_len and chunk_off were final before the
  // predecessor's call was enqueued (and that the predecessor does not touch this workspace):
  // only topk_idx comes from the predecessor, so the producer waits just before it reads
  // topk_idx for its first selected-chunk item, the compute warps once they have built that
  // item's query fragments, and every thread at its end at the latest.
  bool waited = !p.early;
  if (waited) pdl_enter();
  const int row_bytes = n_kv * D * 2;  // one key, every KV head

  if (producer) {
    // ---- the document table in shared memory (one round trip, 16-byte asynchronous copies;
    //      the tail past the last whole 16 bytes with plain loads) ----
    if (p.co_cap && p.n_chunk_splits) {
      const int n = p.n_docs + 1, n16 = n / 4;
      for (int i = lane; i < n16; i += 32) cp_async16(co_sm + 4 * i, reinterpret_cast<const uint4*>(p.chunk_off) + i);
      for (int i = 4 * n16 + lane; i < n; i += 32) co_sm[i] = __ldg(&p.chunk_off[i]);
      cp_async_wait_all();
      __syncwarp();
    }
    // ---- per item: the header and the query rows for the compute warps, then the segment table
    //      (selected docs in top-k order) and the key range, then the item's tiles ----
    int gt = 0;
    int n_hdr = 0;      // items whose query rows were requested
    bool stop = false;  // a wait gave up
    for (int it = blockIdx.x, j = 0; it < n_items && !stop; it += gridDim.x, ++j) {
      const int hb = j & 1;
      const bool is_chunk = it >= n_loc_items;
      const int i2 = is_chunk ? it - n_loc_items : it;
      const int ns = is_chunk ? p.n_chunk_splits : p.n_loc_splits;
      // a query's local splits run last-first: the last one (it holds the newest local row, which
      // a fused append writes first) goes to the lowest CTA, which starts earliest
      const int split = is_chunk ? i2 % ns : ns - 1 - i2 % ns, bq = i2 / ns;
      const int b = bq / p.n_tgroups, t0 = (bq % p.n_tgroups) * MT;
      const int nt = min(MT, p.q_tokens - t0);
      if (j >= 2 && !warp_wait(&hempty[hb], ((j >> 1) - 1) & 1, &abort_flag)) break;  // item j-2's header, query read
      int L = p.loc_len[b];
      L = max(0, min(L, p.t_loc_max));
      int* hd = hdr + hb * 8;
      if (lane == 0) {
        hd[0] = b; hd[1] = t0; hd[2] = nt; hd[3] = L;
        const uint32_t qbytes = (uint32_t)(nt * p.n_q * D * 2);
        mbar_arrive_expect_tx(&hfull[hb], qbytes);  // releases the header writes above
        bulk_load(qsm + hb * q_elems, p.q + ((size_t)b * p.q_tokens + t0) * p.n_q * D, qbytes, &hfull[hb]);
      }
      n_hdr = j + 1;
      if (is_chunk && !waited) {
        pdl_enter();
        waited = true;
      }
      int* seg_v = segs + hb * (2 * kMaxK + 2);  // [k + 1] virtual starts
      int* seg_c = seg_v + kMaxK + 2;            // [k] chunk starts
      for (int r = lane; r < (is_chunk ? k : 0); r += 32) {
        const int doc = p.topk_idx[(size_t)b * k + r] - p.doc_base;
        int c0 = 0, n = 0;
        if (doc >= 0 && doc < p.n_docs) {
          c0 = p.co_cap ? co_sm[doc] : __ldg(&p.chunk_off[doc]);
          n = (p.co_cap ? co_sm[doc + 1] : __ldg(&p.chunk_off[doc + 1])) - c0;
        } else if (!p.foreign_ok) {
          raise_dev_error(kDevErrBadIndex);
        }
        seg_c[r] = c0;
        seg_v[r + 1] = n;
      }
      __syncwarp();
      if (is_chunk) {  // inclusive scan of chunk counts -> virtual starts (lane owns a run of entries)
        const int per = (k + 31) / 32;
        int local = 0;
        for (int q = 0; q < per; ++q) {
          const int r = lane * per + q;
          if (r < k) local += seg_v[r + 1];
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int q = 0; q < per; ++q) {
          const int r = lane * per + q;
          if (r < k) {
            run += seg_v[r + 1];
            seg_v[r + 1] = run;
          }
        }
        if (lane == 0) seg_v[0] = 0;
      }
      __syncwarp();
      // a chunk item covers a run of the selected chunks (virtual keys 0 .. n_sel), a local
      // item a run of the local keys (virtual keys 0 .. L with n_sel = 0)
      const int n_sel = is_chunk ? seg_v[k] : 0;
      const int n_keys = is_chunk ? n_sel : L;
      const int v0 = (int)(((long long)split * n_keys) / ns);  // an even share of the keys
      const int v1 = (int)(((long long)(split + 1) * n_keys) / ns);
      const int n_tiles = (v1 - v0 + kTK - 1) / kTK;
      if (lane == 0) {
        hd[4] = n_sel; hd[5] = v0; hd[6] = v1;
        hd[7] = is_chunk ? p.chunk_part_base + split : split;  // the item's partial slot
        mbar_arrive(&hsel[hb]);  // releases the key-range writes
      }
      // the item holding the query's last local row writes the new token there (no other item
      // reads that row) just before it requests that row's tile, so that its earlier tiles stream
      // meanwhile: key rotated at its position (or as given), value copied; then orders the writes
      // before its bulk copies read the row back.  A lane rotates dims i and i + D/2 of every KV
      // head with one angle.
      const bool appends = p.k_new && !is_chunk && v1 == L && v1 > v0;
      if (p.k_new && !is_chunk && !appends && L == 0 && split == 0 && lane == 0)
        raise_dev_error(kDevErrBadIndex);  // no local position to take the new token
      auto append_token = [&]() {
        const int slot = L - 1;
        const size_t src = (size_t)b * n_kv * D;
        const size_t dst = ((size_t)b * p.t_loc_max + slot) * n_kv * D;
        __nv_bfloat16* kd = const_cast<__nv_bfloat16*>(p.K_loc) + dst;
        __nv_bfloat16* vd = const_cast<__nv_bfloat16*>(p.V_loc) + dst;
        for (int i = lane; i < D / 2; i += 32) {
          const float2 cs = p.append_rotate ? rope_cos_sin(p.turns, i, (int64_t)p.pos_offset + slot)
                                            : make_float2(1.f, 0.f);
          for (int hh = 0; hh < n_kv; ++hh) {
            const __nv_bfloat16* kr = p.k_new + src + (size_t)hh * D;
            if (p.append_rotate) {
              const float x1 = __bfloat162float(kr[i]), x2 = __bfloat162float(kr[i + D / 2]);
              kd[(size_t)hh * D + i] = __float2bfloat16_rn(x1 * cs.x - x2 * cs.y);
              kd[(size_t)hh * D + i + D / 2] = __float2bfloat16_rn(x2 * cs.x + x1 * cs.y);
            } else {
              kd[(size_t)hh * D + i] = kr[i];
              kd[(size_t)hh * D + i + D / 2] = kr[i + D / 2];
            }
          }
        }
        for (int e = lane; e < n_kv * D / 8; e += 32)
          reinterpret_cast<uint4*>(vd)[e] = __ldg(reinterpret_cast<const uint4*>(p.v_new + src) + e);
        fence_proxy_async_global();
        __syncwarp();
      };
      // ---- the item's tiles: kTK keys each, a bulk copy per key and tensor plus the RoPE rows ----
      for (int t = 0; t < n_tiles; ++t, ++gt) {
        const int st = gt % L_.n_stages;
        if (gt >= L_.n_stages && !warp_wait(&ebars[st], ((gt / L_.n_stages) - 1) & 1, &abort_flag)) {
          stop = true;
          break;
        }
        if (appends && t == n_tiles - 1) append_token();  // the last tile holds row L - 1
        const int tv0 = v0 + t * kTK;
        const int rows = min(kTK, v1 - tv0);
        const int n_chunk_rows = max(0, min(rows, n_sel - tv0));
        const int n_loc_rows = rows - n_chunk_rows;
        const uint32_t tb = (table && n_loc_rows > 0) ? (uint32_t)(n_loc_rows * (D / 2) * 8) : 0u;
        if (lane == 0) mbar_arrive_expect_tx(&bars[st], (uint32_t)(2 * rows * row_bytes) + tb);
        __syncwarp();
        uint8_t* kdst = stage_mem + (size_t)st * L_.stage_bytes;
        uint8_t* vdst = kdst + L_.kbytes;
        if (lane < rows) {
          const int v = tv0 + lane;
          const __nv_bfloat16 *ks, *vs;
          if (v < n_sel) {
            int lo = 0, hi = k - 1;  // segment with seg_v[lo] <= v < seg_v[lo + 1]
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (seg_v[mid] <= v) lo = mid; else hi = mid - 1;
            }
            const size_t ch = (size_t)(seg_c[lo] + (v - seg_v[lo]));
            ks = p.K_bar + ch * n_kv * D;
            vs = p.V_bar + ch * n_kv * D;
          } else {
            const size_t off = ((size_t)b * p.t_loc_max + (size_t)(v - n_sel)) * n_kv * D;
            ks = p.K_loc + off;
            vs = p.V_loc + off;
          }
          bulk_load(kdst + lane * L_.krow, ks, row_bytes, &bars[st]);
          bulk_load(vdst + lane * L_.krow, vs, row_bytes, &bars[st]);
        }
        if (tb && lane == 31) {
          const int j0 = tv0 + n_chunk_rows - n_sel;
          bulk_load(vdst + L_.kbytes + n_chunk_rows * (D / 2) * 8, p.rope_tab + (size_t)j0 * (D / 2), tb, &bars[st]);
        }
      }
    }
    if (abort_flag && lane == 0) {  // the copies still in flight land before the CTA exits
      mbar_drain_ring(bars, L_.n_stages, gt - L_.n_stages, gt);
      mbar_drain_ring(hfull, 2, n_hdr - 2, n_hdr);
    }
    __syncwarp();
    if (!waited) pdl_enter();  // the grid completes only after its predecessor
    return;  // the compute warps no longer synchronise with the whole block
  }

  // ---- compute warps, item by item ----
  const int n_compute = 32 * n_kv;
  int gt = 0;
  bool failed = false;  // a wait of this warp gave up: the compute warps leave together at the next item
  // the query fragments stay in registers from one item to the next of the same (query, token
  // group): a CTA that takes several items of one query rotates its query once
  uint32_t qa[KS][4];
  int frag_b = -1, frag_t0 = -1;
  for (int it = blockIdx.x, j = 0; it < n_items; it += gridDim.x, ++j) {
    const int hb = j & 1;
    failed |= !warp_wait(&hfull[hb], (j >> 1) & 1, &abort_flag);
    // every warp has built its previous fragments (qcs is reused), and none has given up a wait
    if (named_bar_any(1, n_compute, failed)) break;
    const int* hd = hdr + hb * 8;
    const int b = hd[0], t0 = hd[1], nt = hd[2], L = hd[3];
    const uint16_t* qsm_b = qsm + hb * q_elems;
    const int g = lane >> 2, c = lane & 3;
    if (b != frag_b || t0 != frag_t0) {  // block-uniform
      // ---- query fragments of this warp's GQA group: mma row = tt * G + gg (token t0 + tt,
      //      q head h * G + gg); token t sits at pos_offset + L - M + t; scale, bf16 ----
      const int64_t pos_q0 = (int64_t)p.pos_offset + L - p.q_tokens + t0;
      for (int i = tid; i < nt * (D / 2); i += n_compute)
        qcs[i] = rope_cos_sin(p.turns, i % (D / 2), pos_q0 + i / (D / 2));
      named_bar_sync(1, n_compute);
  #pragma unroll
      for (int s = 0; s < KS; ++s) {
  #pragma unroll
        for (int rr = 0; rr < 2; ++rr) {        // rows g and g + 8
          const int row = g + 8 * rr;
          const int tt = row / G, gg = row - tt * G;
          const uint16_t* qb = qsm_b + ((size_t)tt * p.n_q + h * G + gg) * D;
  #pragma unroll
          for (int hk = 0; hk < 2; ++hk) {      // k cols 2c.. and 2c+8..: dims d0 and d0 + 1, one half
            const int d0 = 16 * s + 8 * hk + 2 * c;
            float v0 = 0.f, v1 = 0.f;
            if (tt < nt) {
              const bool first = d0 < D / 2;
              const int i0 = first ? d0 : d0 - D / 2;
              const int p0 = first ? d0 + D / 2 : d0 - D / 2;
              const float2 x = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(qb + d0));
              const float2 y = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(qb + p0));
              const float4 cs = *reinterpret_cast<const float4*>(qcs + tt * (D / 2) + i0);  // cos, sin of i0, i0 + 1
              // first half: x cos - y sin; second half: x cos + y sin (y = first-half partner)
              const float r0 = first ? (x.x * cs.x - y.x * cs.y) : (x.x * cs.x + y.x * cs.y);
              const float r1 = first ? (x.y * cs.z - y.y * cs.w) : (x.y * cs.z + y.y * cs.w);
              v0 = r0 * p.scale_log2;
              v1 = r1 * p.scale_log2;
            }
            qa[s][rr + 2 * hk] = pack_bf16x2(v0, v1);
          }
        }
      }
      frag_b = b;
      frag_t0 = t0;
    }

    if (it >= n_loc_items && !waited) {  // the first selected-chunk item: its fragments are ready
      pdl_enter();
      waited = true;
    }
    if (!warp_wait(&hsel[hb], (j >> 1) & 1, &abort_flag)) {
      failed = true;
      continue;
    }
    const int n_sel = hd[4], v0 = hd[5], v1 = hd[6], part = hd[7];
    const int n_tiles = (v1 - v0 + kTK - 1) / kTK;
    __syncwarp();
    if (lane == 0) mbar_arrive(&hempty[hb]);  // header and query rows read: the buffer may refill

    float acc[NBLK][4];
  #pragma unroll
    for (int n = 0; n < NBLK; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    const int hoff = h * D * 2;  // this head's bytes within a key row
    // causal limit of rows g and g + 8: token t sees the chunks and local tokens j <= L - M + t
    int lim[2];
  #pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int tt = (g + 8 * rr) / G;
      lim[rr] = tt < nt ? n_sel + max(0, min(L, L - p.q_tokens + t0 + tt + 1)) : v1;
    }

    for (int t = 0; t < n_tiles; ++t) {
      const int gtt = gt + t;  // tile counter over this CTA's items: the ring position
      const int st = gtt % L_.n_stages;
      if (!warp_wait(&bars[st], (gtt / L_.n_stages) & 1, &abort_flag)) {
        failed = true;
        break;
      }

      const int tv0 = v0 + t * kTK;
      const uint8_t* kst = stage_mem + (size_t)st * L_.stage_bytes;
      const uint32_t kbase = smem_u32(kst) + hoff;
      const uint32_t vbase = kbase + L_.kbytes;
      const float2* tab = reinterpret_cast<const float2*>(kst + 2 * L_.kbytes);

      // ---- S = q K^T (rows = heads, cols = 16 keys), k-steps in pairs (s, s + KS/2): the pair
      //      holds dims i and i + D/2, which the RoPE of a local key mixes; only one pair's K
      //      fragments (B operand, keys = n) are live at a time ----
      float sc[2][4];
  #pragma unroll
      for (int nb = 0; nb < 2; ++nb) sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
      {
        const int key = (lane & 7) + 8 * (lane >> 4);
        const int dsel = 8 * ((lane >> 3) & 1);
  #pragma unroll
        for (int sp = 0; sp < KS / 2; ++sp) {
          uint32_t kx[2][2], ky[2][2];  // [nb][hk] of k-steps sp and sp + KS/2
          ldmatrix_x4(kx[0][0], kx[0][1], kx[1][0], kx[1][1], kbase + key * L_.krow + (16 * sp + dsel) * 2);
          ldmatrix_x4(ky[0][0], ky[0][1], ky[1][0], ky[1][1],
                      kbase + key * L_.krow + (16 * (sp + KS / 2) + dsel) * 2);
          if (table) {  // rotate local keys in registers
  #pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              const int r = 8 * nb + g;
              const int v = tv0 + r;
              if (v >= n_sel && v < v1) {
                const float2* trow = tab + r * (D / 2);
  #pragma unroll
                for (int hk = 0; hk < 2; ++hk) {
                  const int i = 16 * sp + 8 * hk + 2 * c;
                  const float4 cs = *reinterpret_cast<const float4*>(trow + i);  // (cos_i, sin_i, cos_i+1, sin_i+1)
                  const float2 x = unpack_bf16x2(kx[nb][hk]);
                  const float2 y = unpack_bf16x2(ky[nb][hk]);
                  const float x0 = x.x * cs.x - y.x * cs.y, y0 = y.x * cs.x + x.x * cs.y;
                  const float x1 = x.y * cs.z - y.y * cs.w, y1 = y.y * cs.z + x.y * cs.w;
                  kx[nb][hk] = pack_bf16x2(x0, x1);
                  ky[nb][hk] = pack_bf16x2(y0, y1);
                }
              }
            }
          }
  #pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            mma_bf16_16816(sc[nb], qa[sp][0], qa[sp][1], qa[sp][2], qa[sp][3], kx[nb][0], kx[nb][1]);
            mma_bf16_16816(sc[nb], qa[sp + KS / 2][0], qa[sp + KS / 2][1], qa[sp + KS / 2][2], qa[sp + KS / 2][3],
                           ky[nb][0], ky[nb][1]);
          }
        }
      }
  #pragma unroll
      for (int nb = 0; nb < 2; ++nb)
  #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int v = tv0 + 8 * nb + 2 * c + e;
          if (v >= v1 || v >= lim[0]) sc[nb][e] = -INFINITY;
          if (v >= v1 || v >= lim[1]) sc[nb][2 + e] = -INFINITY;
        }
      // ---- online softmax (rows g and g + 8) ----
      float alpha[2];
  #pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        float mx = fmaxf(fmaxf(sc[0][2 * rr], sc[0][2 * rr + 1]), fmaxf(sc[1][2 * rr], sc[1][2 * rr + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run[rr], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[rr] = exp2f(m_run[rr] - m_use);
        m_run[rr] = m_new;
        float ls = 0.f;
  #pragma unroll
        for (int nb = 0; nb < 2; ++nb)
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float pv = exp2f(sc[nb][2 * rr + e] - m_use);
            sc[nb][2 * rr + e] = pv;
            ls += pv;
          }
        l_run[rr] = l_run[rr] * alpha[rr] + ls;
      }
  #pragma unroll
      for (int n = 0; n < NBLK; ++n) {
        acc[n][0] *= alpha[0];
        acc[n][1] *= alpha[0];
        acc[n][2] *= alpha[1];
        acc[n][3] *= alpha[1];
      }
      // ---- O += P V ----
      const uint32_t pa0 = pack_bf16x2(sc[0][0], sc[0][1]);
      const uint32_t pa1 = pack_bf16x2(sc[0][2], sc[0][3]);
      const uint32_t pa2 = pack_bf16x2(sc[1][0], sc[1][1]);
      const uint32_t pa3 = pack_bf16x2(sc[1][2], sc[1][3]);
      {
        const int key = (lane & 7) + 8 * ((lane >> 3) & 1);
        const int dsel = 8 * (lane >> 4);
  #pragma unroll
        for (int n = 0; n < NBLK; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(b0, b1, b2, b3, vbase + key * L_.krow + (8 * n + dsel) * 2);
          mma_bf16_16816(acc[n], pa0, pa1, pa2, pa3, b0, b1);
          mma_bf16_16816(acc[n + 1], pa0, pa1, pa2, pa3, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ebars[st]);  // this warp is done with stage st
    }


    if (failed) continue;  // the item is abandoned; the warps leave at the next item
    gt += n_tiles;

    // ---- this warp's split partial: unnormalised output, running max and sum per q head ----
  #pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
      l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
    }
  #pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = g + 8 * rr;
      const int tt = row / G;
      if (tt < nt) {
        const size_t qh = ((size_t)b * p.q_tokens + t0 + tt) * p.n_q + (size_t)h * G + (row - tt * G);
        const size_t ps = qh * p.n_parts + part;
        float* po = p.part_o + ps * D;
  #pragma unroll
        for (int n = 0; n < NBLK; ++n)
          *reinterpret_cast<float2*>(po + 8 * n + 2 * c) = make_float2(acc[n][2 * rr], acc[n][2 * rr + 1]);
        if (c == 0) {
          p.part_ml[ps * 2 + 0] = m_run[rr];
          p.part_ml[ps * 2 + 1] = l_run[rr];
        }
      }
    }
  }
  if (!waited) pdl_enter();  // the grid completes only after its predecessor
}

// log-sum-exp merge of the split partials of one (query token, q head), or of a 32-dim slice of
// it (SL = D / 32 slices: more CTAs when there are few queries).  Lane l holds W = D / (32 SL)
// consecutive dims of the CTA's part; warp w sums the splits w, w + 8, ...; every CTA reduces
// the (m, l) pairs itself and the warps' sums meet in shared memory.
template <int D, int SL>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_ml,
                                                           const float* __restrict__ part_o, int n_splits,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ out_f32,
                                                           float* __restrict__ out_lse2) {
  constexpr int W = D / (32 * SL);          // dims per lane
  constexpr int kHold = W == 1 ? 24 : 12;   // partial rows per lane loaded before the weights are known
  __shared__ float w_s[kMaxSplits];
  __shared__ float red[2][8];
  __shared__ float osum[8][32 * W];
  pdl_enter();
  const size_t qh = (size_t)blockIdx.y * gridDim.x + blockIdx.x;  // (b * M + t) * n_q + head
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d0 = blockIdx.z * 32 * W;       // this CTA's first dim
  const float* ml = part_ml + qh * n_splits * 2;
  const float* po = part_o + qh * n_splits * D + d0 + lane * W;
  auto load = [&](int sp, float* v) {
    if constexpr (W == 4) {
      const float4 x = *reinterpret_cast<const float4*>(po + (size_t)sp * D);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else if constexpr (W == 2) {
      const float2 x = *reinterpret_cast<const float2*>(po + (size_t)sp * D);
      v[0] = x.x; v[1] = x.y;
    } else {
      v[0] = po[(size_t)sp * D];
    }
  };
  // every load in flight at once: this lane's first kHold partial rows and the (m, l) pairs
  float hold[kHold][W];
#pragma unroll
  for (int i = 0; i < kHold; ++i) {
    const int sp = warp + 8 * i;
    if (sp < n_splits) load(sp, hold[i]);
  }
  float m = -INFINITY;
  for (int sp = tid; sp < n_splits; sp += blockDim.x) m = fmaxf(m, ml[2 * sp]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[0][warp] = m;
  __syncthreads();
  float M = red[0][0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M = fmaxf(M, red[0][w]);
  const float Mu = (M == -INFINITY) ? 0.f : M;
  float l = 0.f;
  for (int sp = tid; sp < n_splits; sp += blockDim.x) {  // (m, l) are L1 hits by now
    const float w = exp2f(ml[2 * sp] - Mu);
    w_s[sp] = w;
    l += w * ml[2 * sp + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[1][warp] = l;
  __syncthreads();
  float Ls = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) Ls += red[1][w];
  float acc[W];
#pragma unroll
  for (int e = 0; e < W; ++e) acc[e] = 0.f;
#pragma unroll
  for (int i = 0; i < kHold; ++i) {
    const int sp = warp + 8 * i;
    if (sp < n_splits) {
      const float w = w_s[sp];
#pragma unroll
      for (int e = 0; e < W; ++e) acc[e] += w * hold[i][e];
    }
  }
#pragma unroll 4
  for (int sp = warp + 8 * kHold; sp < n_splits; sp += 8) {  // splits past the held rows
    float v[W];
    load(sp, v);
    const float w = w_s[sp];
#pragma unroll
    for (int e = 0; e < W; ++e) acc[e] += w * v[e];
  }
#pragma unroll
  for (int e = 0; e < W; ++e) osum[warp][lane * W + e] = acc[e];
  __syncthreads();
  for (int dim = tid; dim < 32 * W; dim += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) o += osum[w][dim];
    const float v = Ls > 0.f ? o / Ls : 0.f;
    if (out_f32) out_f32[qh * D + d0 + dim] = v;  // a rank's share: fp32, merged across ranks later
    else out[qh * D + d0 + dim] = __float2bfloat16_rn(v);
  }
  if (out_lse2 && blockIdx.z == 0 && tid == 0) out_lse2[qh] = Ls > 0.f ? Mu + log2f(Ls) : -INFINITY;
}

int stages_that_fit(int n_kv, int n_q, int D, bool table, int mt, int co_cap) {
  const int budget = 224 * 1024;
  for (int st = kMaxStages; st >= 2; --st) {
    AttnSmem L(n_kv, D, st, table);
    if (L.total(n_q, D, mt, co_cap) <= (size_t)budget) return st;
  }
  return 2;
}

// query tokens per CTA: as many as fill the 16 mma rows of a warp (GQA group G each)
int tokens_per_cta(const msa_dims& d, int M) { return std::max(1, std::min(M, 16 / (d.n_q / d.n_kv))); }

// rotate rows of x [rows, heads, D] in place: pair (i, i + D/2) of row r by pos[r] * theta_i
template <int D>
__global__ void __launch_bounds__(256) rope_rows_kernel(__nv_bfloat16* __restrict__ x, int rows, int heads,
                                                        const int32_t* __restrict__ pos, const RopeTurns turns) {
  pdl_enter();
  const int64_t n = (int64_t)rows * heads * (D / 2);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % (D / 2));
    const int64_t rh = e / (D / 2);
    const int r = (int)(rh / heads);
    const float2 cs = rope_cos_sin(turns, i, (int64_t)pos[r]);
    __nv_bfloat16* v = x + rh * D;
    const float x1 = __bfloat162float(v[i]), x2 = __bfloat162float(v[i + D / 2]);
    v[i] = __float2bfloat16_rn(x1 * cs.x - x2 * cs.y);
    v[i + D / 2] = __float2bfloat16_rn(x2 * cs.x + x1 * cs.y);
  }
}

// log-sum-exp merge with one warp per (query token, q head), 8 per CTA: for many query tokens
// (short CTAs are launched at a limited rate, so a CTA per head or per slice costs more than the
// merge).  Lane l holds dims l*W .. l*W + W - 1; each split's weight is computed by the lane that
// loaded its (m, l) and broadcast with a shuffle; no shared memory, no block barrier.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_warp_kernel(const float* __restrict__ part_ml,
                                                                const float* __restrict__ part_o, int n_splits,
                                                                int n_rows, __nv_bfloat16* __restrict__ out,
                                                                float* __restrict__ out_f32,
                                                                float* __restrict__ out_lse2) {
  constexpr int W = D / 32;
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const size_t qh = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (qh >= (size_t)n_rows) return;
  const float* ml = part_ml + qh * n_splits * 2;
  const float* po = part_o + qh * n_splits * D + lane * W;
  float m = -INFINITY;
  for (int sp = lane; sp < n_splits; sp += 32) m = fmaxf(m, ml[2 * sp]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float Mu = (m == -INFINITY) ? 0.f : m;
  float l = 0.f, acc[W];
#pragma unroll
  for (int e = 0; e < W; ++e) acc[e] = 0.f;
  for (int base = 0; base < n_splits; base += 32) {
    const int sp = base + lane;
    float w = 0.f;
    if (sp < n_splits) {
      w = exp2f(ml[2 * sp] - Mu);
      l = fmaf(w, ml[2 * sp + 1], l);
    }
    const int cnt = min(32, n_splits - base);
#pragma unroll 8
    for (int j = 0; j < cnt; ++j) {
      const float wj = __shfl_sync(0xffffffffu, w, j);
      const float* src = po + (size_t)(base + j) * D;
      if constexpr (W == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(wj, v.x, acc[0]); acc[1] = fmaf(wj, v.y, acc[1]);
        acc[2] = fmaf(wj, v.z, acc[2]); acc[3] = fmaf(wj, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(wj, v.x, acc[0]); acc[1] = fmaf(wj, v.y, acc[1]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  if (out_f32) {  // a rank's share: fp32, merged across ranks later
#pragma unroll
    for (int e = 0; e < W; ++e) out_f32[qh * D + lane * W + e] = acc[e] * inv;
    if (lane == 0) out_lse2[qh] = l > 0.f ? Mu + log2f(l) : -INFINITY;
  } else {
#pragma unroll
    for (int e = 0; e < W; ++e) out[qh * D + lane * W + e] = __float2bfloat16_rn(acc[e] * inv);
  }
}

// merge of R shares of one attention (memory-parallel ranks): out = sum_r w_r o_r / sum_r w_r with
// w_r = 2^(lse2_r - max_r lse2_r); one warp per (query token, q head), lane l holds dims l*W ..
template <int D>
__global__ void __launch_bounds__(256) attend_merge_kernel(const float* __restrict__ o_parts,
                                                           const float* __restrict__ lse2_parts, int R, int n_rows,
                                                           __nv_bfloat16* __restrict__ out) {
  constexpr int W = D / 32;
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= (size_t)n_rows) return;
  float m = -INFINITY;
  for (int r = lane; r < R; r += 32) m = fmaxf(m, lse2_parts[(size_t)r * n_rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float acc[W], wsum = 0.f;
#pragma unroll
  for (int e = 0; e < W; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    for (int r = 0; r < R; ++r) {  // in rank order: the same result on every rank
      const float w = exp2f(lse2_parts[(size_t)r * n_rows + row] - m);
      wsum += w;
      const float* src = o_parts + ((size_t)r * n_rows + row) * D + lane * W;
#pragma unroll
      for (int e = 0; e < W; ++e) acc[e] = fmaf(w, src[e], acc[e]);
    }
  }
  const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
#pragma unroll
  for (int e = 0; e < W; ++e) out[row * D + lane * W + e] = __float2bfloat16_rn(acc[e] * inv);
}

// the decode step's new token into the rotated cache: CTA = one query; key rotated at
// pos_offset + slot, value copied (D/2 pairs x n_kv heads per thread block)
template <int D>
__global__ void __launch_bounds__(256) kv_append_kernel(const __nv_bfloat16* __restrict__ k_new,
                                                        const __nv_bfloat16* __restrict__ v_new,
                                                        __nv_bfloat16* __restrict__ K_loc,
                                                        __nv_bfloat16* __restrict__ V_loc, int n_kv, int t_loc_max,
                                                        const int32_t* __restrict__ slots, int pos_offset,
                                                        const RopeTurns turns) {
  pdl_enter();
  const int b = blockIdx.x;
  const int slot = slots[b];
  if (slot < 0 || slot >= t_loc_max) {
    if (threadIdx.x == 0) raise_dev_error(kDevErrBadIndex);
    return;
  }
  const size_t src = (size_t)b * n_kv * D;
  const size_t dst = ((size_t)b * t_loc_max + slot) * n_kv * D;
  for (int e = threadIdx.x; e < n_kv * (D / 2); e += blockDim.x) {
    const int h = e / (D / 2), i = e % (D / 2);
    const float2 cs = rope_cos_sin(turns, i, (int64_t)pos_offset + slot);
    const __nv_bfloat16* kr = k_new + src + (size_t)h * D;
    const float x1 = __bfloat162float(kr[i]), x2 = __bfloat162float(kr[i + D / 2]);
    __nv_bfloat16* kd = K_loc + dst + (size_t)h * D;
    kd[i] = __float2bfloat16_rn(x1 * cs.x - x2 * cs.y);
    kd[i + D / 2] = __float2bfloat16_rn(x2 * cs.x + x1 * cs.y);
  }
  for (int e = threadIdx.x; e < n_kv * D / 8; e += blockDim.x)
    reinterpret_cast<uint4*>(V_loc + dst)[e] = __ldg(reinterpret_cast<const uint4*>(v_new + src) + e);
}

// splits per query: enough CTAs for about four waves, rounded so that B * splits is a
// whole number of waves on this GPU (one CTA per SM), and at least ~32 keys per split
int choose_splits(int B, int t_loc_max, int k) {
  const int sms = sm_count();
  const int max_useful = std::max(1, std::min((t_loc_max + 16 * k) / 32, kMaxSplits));
  const int want = std::max(1, (4 * sms + B - 1) / B);
  int g = sms, b = B;
  while (b) {
    const int t = g % b;
    g = b;
    b = t;
  }
  const int wave = sms / g;  // B * (multiple of wave) is a multiple of sms
  int s = (want + wave - 1) / wave * wave;
  if (s > max_useful) s = std::min(want, max_useful);
  return std::max(1, s);
}

// ---------------------------------------------------------------------------
// host tier: gather the selected documents' pooled K̄/V̄ rows from pinned host
// memory into a device staging area (zero-copy 16-byte loads over the bus)
// ---------------------------------------------------------------------------
// one block: staged chunk offsets of the B*k selected documents, their new ids
__global__ void __launch_bounds__(1024) gather_plan_kernel(const int32_t* __restrict__ chunk_off, int n_docs,
                                                           const int32_t* __restrict__ topk_idx, int n_sel,
                                                           int capacity, int32_t* __restrict__ stage_off,
                                                           int32_t* __restrict__ stage_src,
                                                           int32_t* __restrict__ stage_idx) {
  __shared__ int cnt[1024];
  __shared__ int carry;
  pdl_enter();
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n_sel; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int n = 0, src = 0;
    if (i < n_sel) {
      const int doc = topk_idx[i];
      if (doc >= 0 && doc < n_docs) {
        src = chunk_off[doc];
        n = chunk_off[doc + 1] - src;
      } else {
        raise_dev_error(kDevErrBadIndex);
      }
      stage_src[i] = src;
      stage_idx[i] = i;  // query b's r-th document is staged document b * k + r
    }
    cnt[threadIdx.x] = n;
    __syncthreads();
    // inclusive scan (Hillis-Steele) over this batch of up to 1024 documents
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
      const int v = threadIdx.x >= (unsigned)o ? cnt[threadIdx.x - o] : 0;
      __syncthreads();
      cnt[threadIdx.x] += v;
      __syncthreads();
    }
    if (i < n_sel) {
      int end = carry + cnt[threadIdx.x];
      if (end > capacity) {  // staging too small: keep what fits, report
        raise_dev_error(kDevErrBadIndex);
        end = capacity;
      }
      stage_off[i + 1] = end;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = carry + cnt[threadIdx.x];
    __syncthreads();
  }
  if (threadIdx.x == 0) stage_off[0] = 0;
}

// copy the planned chunk rows (row = n_kv*D bf16 of K and of V) from host to the staging.
// One warp per row at a time: its lanes hold up to 4 sixteen-byte pieces of the K row and 4 of
// the V row in flight (a 4 KB row pair per warp).  One warp per SM (148 CTAs of 32 threads,
// ~600 KB in flight over the grid: a few times what a ~55 GB/s host link needs at a few
// microseconds of latency).  Spread this thin, the bus reads cost each SM little: measured on
// the 100M-token tiered step, the scan beside the gather took 482 us per launch with one warp per
// SM against 525 us with 16 CTAs of 256 threads (the scan's tiles are split evenly over its CTAs,
// so its slowest SM sets its end), and the gather itself was no slower.
#ifndef MSA_GATHER_THREADS
#define MSA_GATHER_THREADS 32
#endif
#ifndef MSA_GATHER_CTAS
#define MSA_GATHER_CTAS 0
#endif
constexpr int kGatherThreads = MSA_GATHER_THREADS;
constexpr int kGatherCtas = MSA_GATHER_CTAS;  // 0: one CTA per SM
__global__ void __launch_bounds__(kGatherThreads, 1024 / kGatherThreads) gather_copy_kernel(const uint4* __restrict__ K_host,
                                                                        const uint4* __restrict__ V_host,
                                                                        const int32_t* __restrict__ stage_off,
                                                                        const int32_t* __restrict__ stage_src,
                                                                        int n_sel, int row_vec,
                                                                        uint4* __restrict__ K_stage,
                                                                        uint4* __restrict__ V_stage) {
  pdl_enter();
  const int total_rows = stage_off[n_sel];
  const int lane = threadIdx.x & 31;
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int n_warps = (int)((gridDim.x * blockDim.x) >> 5);
  int doc = 0;  // a warp's rows only grow, so its document search starts where the last one ended
  for (int row = warp; row < total_rows; row += n_warps) {
    int lo = doc, hi = n_sel - 1;  // the last staged document starting at or before this row
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (stage_off[mid] <= row) lo = mid; else hi = mid - 1;
    }
    doc = lo;
    const int64_t src = (int64_t)(stage_src[doc] + (row - stage_off[doc])) * row_vec;
    const int64_t dst = (int64_t)row * row_vec;
    for (int v0 = 0; v0 < row_vec; v0 += 128) {
      uint4 kv[4], vv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < row_vec) {
          kv[u] = K_host[src + v];
          vv[u] = V_host[src + v];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + lane + 32 * u;
        if (v < row_vec) {
          K_stage[dst + v] = kv[u];
          V_stage[dst + v] = vv[u];
        }
      }
    }
  }
}

}  // namespace

size_t attend_workspace(const msa_dims& d, int B, int M, int k, int t_loc_max, int pos_offset, void* ws,
                        AttendWs* out) {
  (void)pos_offset;
  Carver cv(ws);
  AttendWs w{};
  const int mt = tokens_per_cta(d, M);
  const int n_tg = (M + mt - 1) / mt;
  // splits per (query, token group), shared between the local keys and the selected chunks in
  // proportion to their expected key counts (the selection's size is known only on the device:
  // about kChunksPerDocEst chunks per selected document), each side at least one split.  Few
  // query groups (latency): one wave, an item per CTA, so that each CTA pays an item's setup
  // (its header, the rotated query fragments, the first tile's round trip) once.  Otherwise a
  // total that makes the item count a whole number of waves.
  const int groups = B * n_tg;
  const bool latency = groups <= kLatencyGroups;
  const int max_useful = std::max(2, std::min((t_loc_max + 16 * k) / 32, kMaxSplits));
  const int n_total = latency ? std::max(2, std::min(sm_count() / groups, max_useful))
                              : std::max(2, choose_splits(groups, t_loc_max, k));
  const double sel_est = (double)kChunksPerDocEst * k;
  int n_chunk = (int)std::lround(n_total * sel_est / (sel_est + std::max(0, t_loc_max)));
  // latency: the selected chunks, which wait for the routing, in splits of about one 16-key tile
  // of the estimate (an underestimate of the selection still leaves them a few tiles each)
  if (latency) n_chunk = std::max(n_chunk, (int)std::ceil(sel_est / 16.0));
  n_chunk = std::max(1, std::min({n_chunk, (latency ? 4 : 2) * k, n_total - 1}));
  w.n_split_chunk = n_chunk;
  w.n_split_local = std::max(1, std::min(n_total - n_chunk, std::max(1, (t_loc_max + kTK - 1) / kTK)));
  w.n_parts = w.n_split_local + w.n_split_chunk;
  w.rope_tab = cv.take<float2>((size_t)std::max(1, t_loc_max) * (d.head_dim / 2));
  w.part_ml = cv.take<float>((size_t)B * M * d.n_q * w.n_parts * 2);
  w.part_o = cv.take<float>((size_t)B * M * d.n_q * w.n_parts * d.head_dim);
  if (out) *out = w;
  return cv.size();
}

msa_status gather_kv_launch(const msa_dims& d, const void* K_host, const void* V_host, const int32_t* chunk_off,
                            int n_docs, const int32_t* topk_idx, int B, int k, void* K_stage, void* V_stage,
                            int capacity_chunks, int32_t* stage_off, int32_t* stage_idx, int32_t* stage_src,
                            cudaStream_t s) {
  const int n_sel = B * k;
  {
    TraceScope ts(kKGatherPlan, s);
    MSA_CUDA_CHECK(launch_pdl(gather_plan_kernel, dim3(1), dim3(1024), 0, s, chunk_off, n_docs, topk_idx, n_sel,
                              capacity_chunks, stage_off, stage_src, stage_idx));
  }
  {
    TraceScope ts(kKGatherCopy, s);
    const int row_vec = d.n_kv * d.head_dim * 2 / 16;
    MSA_CUDA_CHECK(launch_pdl(gather_copy_kernel, dim3(kGatherCtas > 0 ? kGatherCtas : sm_count()),
                              dim3(kGatherThreads), 0, s,
                              static_cast<const uint4*>(K_host), static_cast<const uint4*>(V_host),
                              (const int32_t*)stage_off, (const int32_t*)stage_src, n_sel, row_vec,
                              static_cast<uint4*>(K_stage), static_cast<uint4*>(V_stage)));
  }
  return MSA_OK;
}

msa_status attend_merge_launch(const float* o_parts, const float* lse2_parts, int R, int n_rows, int D, void* out,
                               cudaStream_t s) {
  TraceScope ts(kKAttnMerge, s);
  const dim3 grid((unsigned)((n_rows + 7) / 8));
  auto kern = D == 128 ? attend_merge_kernel<128> : attend_merge_kernel<64>;
  MSA_CUDA_CHECK(launch_pdl(kern, grid, dim3(256), 0, s, o_parts, lse2_parts, R, n_rows,
                            static_cast<__nv_bfloat16*>(out)));
  return MSA_OK;
}

msa_status rope_cache_build(const msa_dims& d, int t_loc_max, int pos_offset, float2* tab, cudaStream_t s) {
  if (t_loc_max <= 0) return MSA_OK;
  const int D = d.head_dim;
  TraceScope ts(kKRopeTable, s);
  RopeTurns turns;
  rope_turns(d, turns.f);
  const int blocks = (int)std::min<int64_t>(((int64_t)t_loc_max * (D / 2) + 255) / 256, 8 * sm_count());
  MSA_CUDA_CHECK(launch_pdl(rope_table_kernel, dim3(blocks), dim3(256), 0, s, tab, t_loc_max, D / 2, pos_offset, turns));
  return MSA_OK;
}

msa_status rope_rows_launch(const msa_dims& d, void* x, int rows, int heads, const int32_t* pos, cudaStream_t s) {
  TraceScope ts(kKRopeRows, s);
  const int64_t n = (int64_t)rows * heads * (d.head_dim / 2);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 8 * sm_count()));
  RopeTurns turns;
  rope_turns(d, turns.f);
  if (d.head_dim == 128)
    MSA_CUDA_CHECK(launch_pdl(rope_rows_kernel<128>, dim3(blocks), dim3(256), 0, s, static_cast<__nv_bfloat16*>(x),
                              rows, heads, pos, turns));
  else
    MSA_CUDA_CHECK(launch_pdl(rope_rows_kernel<64>, dim3(blocks), dim3(256), 0, s, static_cast<__nv_bfloat16*>(x),
                              rows, heads, pos, turns));
  return MSA_OK;
}

msa_status kv_append_launch(const msa_dims& d, const void* k_new, const void* v_new, void* K_loc, void* V_loc, int B,
                            int t_loc_max, const int32_t* slots, int pos_offset, cudaStream_t s) {
  TraceScope ts(kKKvAppend, s);
  RopeTurns turns;
  rope_turns(d, turns.f);
  auto kb = static_cast<const __nv_bfloat16*>(k_new);
  auto vb = static_cast<const __nv_bfloat16*>(v_new);
  auto Kl = static_cast<__nv_bfloat16*>(K_loc);
  auto Vl = static_cast<__nv_bfloat16*>(V_loc);
  if (d.head_dim == 128)
    MSA_CUDA_CHECK(launch_pdl(kv_append_kernel<128>, dim3(B), dim3(256), 0, s, kb, vb, Kl, Vl, d.n_kv, t_loc_max, slots,
                              pos_offset, turns));
  else
    MSA_CUDA_CHECK(launch_pdl(kv_append_kernel<64>, dim3(B), dim3(256), 0, s, kb, vb, Kl, Vl, d.n_kv, t_loc_max, slots,
                              pos_offset, turns));
  return MSA_OK;
}

msa_status attend_launch(const msa_dims& d, const void* q, int B, int M, const void* K_bar, const void* V_bar,
                         const int32_t* chunk_off, int n_docs, const int32_t* topk_idx, int k, const void* K_loc,
                         const void* V_loc, const void* k_new, const void* v_new, const int32_t* loc_len,
                         int t_loc_max, int pos_offset,
                         const void* rope_cache, int k_loc_rotated, float scale, int phase, int early, void* out,
                         void* ws, cudaStream_t s, const AttendShare* share, int max_ctas) {
  AttendWs w;
  attend_workspace(d, B, M, k, t_loc_max, pos_offset, ws, &w);
  const int n_loc = w.n_split_local, n_chk = w.n_split_chunk;
  const int D = d.head_dim;
  const bool side = max_ctas > 0;
  const bool local_keys = phase != 2 && (!share || share->local_keys);
  const float2* tab = (k_loc_rotated || !local_keys) ? nullptr : static_cast<const float2*>(rope_cache);
  if (!tab && !k_loc_rotated && local_keys && t_loc_max > 0) {
    msa_status st = rope_cache_build(d, t_loc_max, pos_offset, w.rope_tab, s);
    if (st != MSA_OK) return st;
    tab = w.rope_tab;
  }
  AttnParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.K_bar = static_cast<const __nv_bfloat16*>(K_bar);
  p.V_bar = static_cast<const __nv_bfloat16*>(V_bar);
  p.chunk_off = chunk_off;
  p.topk_idx = topk_idx;
  p.K_loc = static_cast<const __nv_bfloat16*>(K_loc);
  p.V_loc = static_cast<const __nv_bfloat16*>(V_loc);
  p.loc_len = loc_len;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.append_rotate = k_loc_rotated ? 1 : 0;
  p.rope_tab = tab;
  p.part_ml = w.part_ml;
  p.part_o = w.part_o;
  p.n_q = d.n_q;
  p.n_kv = d.n_kv;
  p.k = k;
  p.n_docs = n_docs;
  p.t_loc_max = t_loc_max;
  p.pos_offset = pos_offset;
  p.n_loc_splits = local_keys ? n_loc : 0;
  p.n_chunk_splits = phase == 1 ? 0 : n_chk;
  // a share without the local keys uses the chunk splits' slots alone
  const bool chunks_only = share && !share->local_keys;
  p.chunk_part_base = chunks_only ? 0 : n_loc;
  p.n_parts = chunks_only ? n_chk : n_loc + n_chk;
  p.doc_base = share ? share->doc_base : 0;
  p.foreign_ok = share ? 1 : 0;
  // the local-key items may start before the predecessor finishes only if this call launches
  // nothing before them (no rotation table built here)
  p.early = early && phase != 2 && (k_loc_rotated || rope_cache || t_loc_max == 0);
  p.n_queries = B;
  p.q_tokens = M;
  p.tok_per_cta = tokens_per_cta(d, M);
  p.n_tgroups = (M + p.tok_per_cta - 1) / p.tok_per_cta;
  p.scale_log2 = (scale > 0.f ? scale : 1.0f / std::sqrt((float)D)) * kLog2e;
  rope_turns(d, p.turns.f);
  // the document table goes to shared memory when it is small and costs no pipeline stage
  p.co_cap = 0;
  if (phase != 1 && n_docs + 1 <= kCoSmemMax) {
    const int st0 = stages_that_fit(d.n_kv, d.n_q, D, tab != nullptr, p.tok_per_cta, 0);
    if (stages_that_fit(d.n_kv, d.n_q, D, tab != nullptr, p.tok_per_cta, n_docs + 1) == st0) p.co_cap = n_docs + 1;
  }
  p.n_stages = stages_that_fit(d.n_kv, d.n_q, D, tab != nullptr, p.tok_per_cta, p.co_cap);
  {
    TraceScope ts(kKAttnSplit, s);
    // persistent: each CTA takes items (split, query, token group) in turn.  The results do not
    // depend on the grid (an item's partial is the same whichever CTA computes it): max_ctas caps
    // it for a launch that runs beside other work on a few SMs, where fewer CTAs that each
    // pipeline many items beat many that each pay an item's setup; such a launch is in plain
    // stream order
    const int n_items = (p.n_loc_splits + p.n_chunk_splits) * B * p.n_tgroups;
    const int cap = side ? std::min(max_ctas, sm_count()) : sm_count();
    dim3 grid(std::max(1, std::min(n_items, cap)));
    const size_t sm = AttnSmem(d.n_kv, D, p.n_stages, tab != nullptr).total(d.n_q, D, p.tok_per_cta, p.co_cap);
    auto kern = D == 128 ? (tab ? attn_split_kernel<128, true> : attn_split_kernel<128, false>)
                         : (tab ? attn_split_kernel<64, true> : attn_split_kernel<64, false>);
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)sm));
    MSA_CUDA_CHECK(launch_ordered(!side, kern, grid, dim3(32 * (d.n_kv + 1)), sm, s, p));
  }
  if (phase != 1) {  // the local-keys phase leaves its partials for the selected-chunks phase's combine
    TraceScope ts(kKAttnCombine, s);
    // few query tokens: a CTA per 32-dim slice of each head (enough CTAs to fill the GPU);
    // many: a warp per head, 8 per CTA
    const long long rows = (long long)B * M * d.n_q;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    // (beside other work: a CTA per head; every output is summed in the same order either way)
    if (rows < 2LL * sm_count()) {
      dim3 grid(d.n_q, B * M, side ? 1 : D / 32);
      auto kern = D == 128 ? (side ? attn_combine_kernel<128, 1> : attn_combine_kernel<128, 4>)
                           : (side ? attn_combine_kernel<64, 1> : attn_combine_kernel<64, 2>);
      MSA_CUDA_CHECK(launch_ordered(!side, kern, grid, dim3(256), 0, s, (const float*)w.part_ml,
                                    (const float*)w.part_o, p.n_parts, o, share ? share->o : nullptr,
                                    share ? share->lse2 : nullptr));
    } else {
      dim3 grid((unsigned)((rows + 7) / 8));
      auto kern = D == 128 ? attn_combine_warp_kernel<128> : attn_combine_warp_kernel<64>;
      MSA_CUDA_CHECK(launch_ordered(!side, kern, grid, dim3(256), 0, s, (const float*)w.part_ml,
                                    (const float*)w.part_o, p.n_parts, (int)rows, o, share ? share->o : nullptr,
                                    share ? share->lse2 : nullptr));
    }
  }
  return MSA_OK;
}

}  // namespace msa

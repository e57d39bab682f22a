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
//   qr_proj_kernel   Q^R partial sums (HBM-bound read of W^QR, split over K)
//   q_prep_kernel    sums the partials, normalises each head, writes the query
//                    as bf16 hi + lo mma B-fragments; clears the doc keys
//   scan_kernel      TMA-staged streaming scan of K̄^R: tensor-core dots and
//                    Gram diagonal (norm), cosine, head mean, per-document
//                    segmented max folded in with atomicMax on ordered keys
//   topk_slice_kernel / topk_merge_kernel
//                    exact radix select of the top-k (score, id) keys per
//                    slice of documents, then a merge of the slice winners
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
  float* qr_part;     // [ksplit][B][NR] fp32 partial sums of Q^R (W_QR given)
  uint4* qfrag;       // [n_r][KS][NBtot][32] bf16 hi/lo query fragments
  uint32_t* doc_key;  // [B][n_docs] ordered-uint32 doc max (MAX)
  float* chunk_s;     // [B][n_chunks] chunk scores (MEAN)
  uint64_t* cand;     // [B][n_slices][k] slice winners
  int ksplit, nb_total, n_slices;
};

namespace {

constexpr int kTileC = 16;         // chunks per pipeline stage (one mma m-tile)
constexpr int kStages = 4;         // TMA ring depth
constexpr int kBoxBytes = kTileC * 128;  // one 64-dim x 16-row box, 128B-swizzled
constexpr int kPartStride = 20;    // padded row stride of the per-head partial tile
constexpr int kSliceDocs = 4096;   // documents per top-k slice CTA
constexpr int kTopkThreads = 1024;
constexpr int kQpCols = 64;
constexpr int kQpQB = 8;
constexpr float kEps = 1e-12f;

// --------------------------------------------------------------------------
// Q^R = H_q W^QR, partial sums over a slice of the hidden dimension
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qr_proj_kernel(const __nv_bfloat16* __restrict__ Hq,
                                                      const __nv_bfloat16* __restrict__ W, int B, int hidden,
                                                      int NR, int rows_per_split, float* __restrict__ part) {
  __shared__ float red[8][kQpQB][kQpCols];
  pdl_launch_dependents();
  pdl_wait();
  const int col0 = blockIdx.x * kQpCols;
  const int split = blockIdx.y;
  const int k_begin = split * rows_per_split;
  const int k_end = min(hidden, k_begin + rows_per_split);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cg = lane & 7, rl = lane >> 3;
  const uint16_t* hq = reinterpret_cast<const uint16_t*>(Hq);
  for (int b0 = 0; b0 < B; b0 += kQpQB) {
    float acc[kQpQB][8];
#pragma unroll
    for (int j = 0; j < kQpQB; ++j)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[j][c] = 0.f;
    for (int k = k_begin + warp * 4 + rl; k < k_end; k += 32) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(W + (size_t)k * NR + col0 + cg * 8));
      float wf[8];
      float2 t;
      t = unpack_bf16x2(w.x); wf[0] = t.x; wf[1] = t.y;
      t = unpack_bf16x2(w.y); wf[2] = t.x; wf[3] = t.y;
      t = unpack_bf16x2(w.z); wf[4] = t.x; wf[5] = t.y;
      t = unpack_bf16x2(w.w); wf[6] = t.x; wf[7] = t.y;
#pragma unroll
      for (int j = 0; j < kQpQB; ++j) {
        if (b0 + j < B) {
          const float h = bf16_bits_to_float(hq[(size_t)(b0 + j) * hidden + k]);
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[j][c] = fmaf(h, wf[c], acc[j][c]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kQpQB; ++j)
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        acc[j][c] += __shfl_xor_sync(0xffffffffu, acc[j][c], 8);
        acc[j][c] += __shfl_xor_sync(0xffffffffu, acc[j][c], 16);
      }
    if (rl == 0) {
#pragma unroll
      for (int j = 0; j < kQpQB; ++j)
#pragma unroll
        for (int c = 0; c < 8; ++c) red[warp][j][cg * 8 + c] = acc[j][c];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < kQpQB * kQpCols; idx += 256) {
      const int j = idx / kQpCols, c = idx % kQpCols;
      if (b0 + j < B) {
        float s = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) s += red[w8][j][c];
        part[((size_t)split * B + b0 + j) * NR + col0 + c] = s;
      }
    }
    __syncthreads();
  }
}

// --------------------------------------------------------------------------
// normalise Q^R per head and lay it out as mma.m16n8k16 B fragments
// (hi and lo bf16 terms); clear the document keys of this query
// --------------------------------------------------------------------------
__global__ void __launch_bounds__(256) q_prep_kernel(const float* __restrict__ part, int ksplit,
                                                     const __nv_bfloat16* __restrict__ qr_direct, int B,
                                                     int n_r, int d_r, int nb_total, uint4* __restrict__ qfrag,
                                                     uint32_t* __restrict__ doc_key, int n_docs) {
  extern __shared__ float qs[];  // [n_r * d_r] then inv norms [n_r]
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;      // padded query index (< 8 * nb_total)
  const int NR = n_r * d_r;
  float* invn = qs + NR;
  const bool real = b < B;
  for (int n = threadIdx.x; n < NR; n += blockDim.x) {
    float v = 0.f;
    if (real) {
      if (qr_direct) {
        v = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(qr_direct)[(size_t)b * NR + n]);
      } else {
        for (int s = 0; s < ksplit; ++s) v += part[((size_t)s * B + b) * NR + n];
      }
    }
    qs[n] = v;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int h = warp; h < n_r; h += blockDim.x / 32) {
    float ss = 0.f;
    for (int i = lane; i < d_r; i += 32) ss = fmaf(qs[h * d_r + i], qs[h * d_r + i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) invn[h] = 1.0f / fmaxf(sqrtf(ss), kEps);
  }
  __syncthreads();
  const int KS = d_r / 16;
  const int nb = b >> 3, g = b & 7;
  for (int idx = threadIdx.x; idx < n_r * KS * 4; idx += blockDim.x) {
    const int h = idx / (KS * 4), s = (idx >> 2) % KS, c = idx & 3;
    const float* qh = qs + h * d_r + 16 * s + 2 * c;
    const float sc = invn[h];
    const float x0 = qh[0] * sc, x1 = qh[1] * sc, x2 = qh[8] * sc, x3 = qh[9] * sc;
    const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
    const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
    const float h2 = __bfloat162float(__float2bfloat16_rn(x2));
    const float h3 = __bfloat162float(__float2bfloat16_rn(x3));
    uint4 f;
    f.x = pack_bf16x2(h0, h1);
    f.y = pack_bf16x2(h2, h3);
    f.z = pack_bf16x2(x0 - h0, x1 - h1);
    f.w = pack_bf16x2(x2 - h2, x3 - h3);
    qfrag[((size_t)(h * KS + s) * nb_total + nb) * 32 + 4 * g + c] = f;
  }
  if (real && doc_key) {
    for (int i = threadIdx.x; i < n_docs; i += blockDim.x) doc_key[(size_t)b * n_docs + i] = 0u;
  }
}

// --------------------------------------------------------------------------
// the K̄^R scan
// --------------------------------------------------------------------------
struct ScanParams {
  const uint4* qfrag;
  const int32_t* chunk_off;
  uint32_t* doc_key;
  float* chunk_s;
  int n_r, n_docs, n_chunks, n_tiles;
  int q_base, q_count, nb_total, nb_base;
  float inv_nr;
};

template <int NB, int DR, bool MEAN>
__global__ void __launch_bounds__(288, 1) scan_kernel(const __grid_constant__ CUtensorMap kr_map,
                                                      const ScanParams p) {
  constexpr int KS = DR / 16;
  constexpr int HALVES = DR / 64;
  constexpr int QP = 8 * NB;  // padded queries in this pass
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int n_r = p.n_r;
  const int stage_bytes = n_r * HALVES * kBoxBytes;
  uint8_t* stages = smem;
  float* partial = reinterpret_cast<float*>(smem + kStages * stage_bytes);  // [2][n_r][QP][kPartStride]
  int* docids = reinterpret_cast<int*>(partial + 2 * n_r * QP * kPartStride);  // [2][16]
  uint64_t* full = reinterpret_cast<uint64_t*>(docids + 32);
  uint64_t* empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_begin = (int)(((long long)blockIdx.x * p.n_tiles) / gridDim.x);
  const int t_end = (int)(((long long)(blockIdx.x + 1) * p.n_tiles) / gridDim.x);
  const int n_it = t_end - t_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], n_r);
    }
    fence_mbar_init();
    prefetch_tensormap(&kr_map);
  }
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();

  if (warp == n_r) {
    // ---------------- producer: one thread streams tiles with TMA ----------------
    if (lane == 0) {
      for (int it = 0; it < n_it; ++it) {
        const int st = it % kStages;
        if (it >= kStages) mbar_wait(&empty[st], ((it / kStages) - 1) & 1);
        mbar_arrive_expect_tx(&full[st], stage_bytes);
        uint8_t* dst = stages + st * stage_bytes;
        const int y = (t_begin + it) * kTileC;
        for (int h = 0; h < n_r; ++h)
          for (int j = 0; j < HALVES; ++j)
            tma_load_2d(dst + (h * HALVES + j) * kBoxBytes, &kr_map, &full[st], h * DR + j * 64, y);
      }
    }
    return;
  }

  // ---------------- consumers: warp h owns router head h ----------------
  const int h = warp;
  uint4 qreg[KS][NB];
#pragma unroll
  for (int s = 0; s < KS; ++s)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
      qreg[s][nb] = p.qfrag[((size_t)(h * KS + s) * p.nb_total + p.nb_base + nb) * 32 + lane];

  const int g = lane >> 2, c = lane & 3;
  const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix source row
  const int khalf = lane >> 4;
  const int diag_src = 4 * g + (g >> 1);
  const int n_consumers = n_r * 32;

  // document cursor (warp 0): index of the document holding this CTA's first chunk
  int cur = 0;
  if (warp == 0 && n_it > 0) {
    const int j0 = t_begin * kTileC;
    int lo = 0, hi = p.n_docs;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(&p.chunk_off[mid]) <= j0) lo = mid; else hi = mid - 1;
    }
    cur = lo;
  }

  for (int it = 0; it < n_it; ++it) {
    const int tile = t_begin + it;
    const int st = it % kStages;
    const int buf = it & 1;
    mbar_wait(&full[st], (it / kStages) & 1);

    float dot[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) dot[nb][0] = dot[nb][1] = dot[nb][2] = dot[nb][3] = 0.f;
    float g0[4] = {0.f, 0.f, 0.f, 0.f}, g1[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t stage_base = smem_u32(stages + st * stage_bytes) + h * HALVES * kBoxBytes;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int unit = ((2 * (s & 3) + khalf) ^ (lrow & 7));
      const uint32_t addr = stage_base + (s >> 2) * kBoxBytes + lrow * 128 + unit * 16;
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a0, a1, a2, a3, addr);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        mma_bf16_16816(dot[nb], a0, a1, a2, a3, qreg[s][nb].x, qreg[s][nb].y);
        mma_bf16_16816(dot[nb], a0, a1, a2, a3, qreg[s][nb].z, qreg[s][nb].w);
      }
      mma_bf16_16816(g0, a0, a1, a2, a3, a0, a2);  // Gram, rows x chunks 0..7
      mma_bf16_16816(g1, a0, a1, a2, a3, a1, a3);  // Gram, rows x chunks 8..15
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);

    // squared norms of rows g and g+8 sit on the Gram diagonals
    const float d0 = (g & 1) ? g0[1] : g0[0];
    const float d1 = (g & 1) ? g1[3] : g1[2];
    const float n2a = __shfl_sync(0xffffffffu, d0, diag_src);
    const float n2b = __shfl_sync(0xffffffffu, d1, diag_src);
    const float inva = 1.0f / fmaxf(sqrtf(n2a), kEps);
    const float invb = 1.0f / fmaxf(sqrtf(n2b), kEps);
    float* P = partial + ((size_t)buf * n_r + h) * QP * kPartStride;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int q0 = 8 * nb + 2 * c;
      P[q0 * kPartStride + g] = dot[nb][0] * inva;
      P[(q0 + 1) * kPartStride + g] = dot[nb][1] * inva;
      P[q0 * kPartStride + g + 8] = dot[nb][2] * invb;
      P[(q0 + 1) * kPartStride + g + 8] = dot[nb][3] * invb;
    }

    if (warp == 0) {
      // document id of every row of this tile (at most 16 boundaries ahead of cur)
      const int j0 = tile * kTileC;
      const int li = lane & 15;
      const int bi = cur + 1 + li;
      const int bnd = (lane < 16 && bi <= p.n_docs) ? __ldg(&p.chunk_off[bi]) : 0x7fffffff;
      int mydoc = cur;
#pragma unroll
      for (int r = 0; r < kTileC; ++r) {
        const unsigned m = __ballot_sync(0xffffffffu, lane < 16 && bnd <= j0 + r);
        if (lane == r) mydoc = cur + __popc(m);
      }
      if (lane < 16) {
        int dv = (j0 + lane < p.n_chunks) ? mydoc : -1;
        if (dv >= p.n_docs) {  // inconsistent chunk_off: drop the row
          raise_dev_error(kDevErrBadIndex);
          dv = -1;
        }
        docids[buf * 16 + lane] = dv;
      }
      cur = __shfl_sync(0xffffffffu, mydoc, 15);
    }
    named_bar_sync(1, n_consumers);

    // head mean + per-document segmented max over the 16 rows
    const float* PB = partial + (size_t)buf * n_r * QP * kPartStride;
    const int r = lane & 15;
    const int doc = docids[buf * 16 + r];
    const int rounds = (p.q_count + 2 * n_r - 1) / (2 * n_r);
    for (int m = 0; m < rounds; ++m) {
      const int qq = m * 2 * n_r + 2 * h + (lane >> 4);
      const bool qok = qq < p.q_count;
      float v = 0.f;
      if (qok) {
        for (int hh = 0; hh < n_r; ++hh) v += PB[(hh * QP + qq) * kPartStride + r];
        v *= p.inv_nr;
      }
      if (MEAN) {
        if (qok && doc >= 0) p.chunk_s[(size_t)(p.q_base + qq) * p.n_chunks + tile * kTileC + r] = v;
      } else {
        float x = (qok && doc >= 0) ? v : -__int_as_float(0x7f800000);
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) {
          const float ox = __shfl_down_sync(0xffffffffu, x, off, 16);
          const int od = __shfl_down_sync(0xffffffffu, doc, off, 16);
          if (r + off < 16 && od == doc) x = fmaxf(x, ox);
        }
        const int prev = __shfl_up_sync(0xffffffffu, doc, 1, 16);
        const bool head = (r == 0) || (prev != doc);
        if (qok && head && doc >= 0)
          atomicMax(&p.doc_key[(size_t)(p.q_base + qq) * p.n_docs + doc], float_to_ordered(x));
      }
    }
  }
}

// --------------------------------------------------------------------------
// exact block-wide top-k of distinct 64-bit keys in shared memory
// key = (ordered score << 32) | (0xFFFFFFFF - doc id): larger key = better,
// equal scores prefer the lower id.  Radix select from the most significant
// byte; it stops as soon as the k-th key's bucket is taken whole.  Writes the
// k best keys, descending, to out[0..k); tmp holds k unsorted winners.
// --------------------------------------------------------------------------
__device__ void block_topk(const uint64_t* keys, int n, int k, uint64_t* out, uint64_t* tmp, uint32_t* hist,
                           uint64_t* sh_state) {
  const int tid = threadIdx.x, nt = blockDim.x;
  uint64_t prefix = 0, mask = 0;
  int kk = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
      const uint64_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1u);
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

__device__ __forceinline__ uint64_t make_key(uint32_t ordered, int id) {
  return ((uint64_t)ordered << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)id);
}

__global__ void __launch_bounds__(kTopkThreads) topk_slice_kernel(
    const uint32_t* __restrict__ doc_key, const float* __restrict__ chunk_s, const int32_t* __restrict__ chunk_off,
    int n_docs, int n_chunks, int k, int n_slices, float* __restrict__ doc_scores, uint64_t* __restrict__ cand,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_score) {
  extern __shared__ uint64_t sm64[];
  uint64_t* keys = sm64;              // [kSliceDocs]
  uint64_t* out = keys + kSliceDocs;  // [256]
  uint64_t* tmp = out + 256;          // [256]
  uint64_t* state = tmp + 256;        // [4]
  uint32_t* hist = reinterpret_cast<uint32_t*>(state + 4);
  pdl_launch_dependents();
  pdl_wait();
  const int slice = blockIdx.x, b = blockIdx.y;
  const int d0 = slice * kSliceDocs;
  const int n = min(kSliceDocs, n_docs - d0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int doc = d0 + i;
    uint32_t ok;
    if (chunk_s) {
      const int c0 = __ldg(&chunk_off[doc]), c1 = __ldg(&chunk_off[doc + 1]);
      float s = 0.f;
      for (int j = c0; j < c1; ++j) s += chunk_s[(size_t)b * n_chunks + j];
      const float mean = s / (float)max(1, c1 - c0);
      ok = float_to_ordered(mean);
    } else {
      ok = doc_key[(size_t)b * n_docs + doc];
    }
    if (doc_scores) doc_scores[(size_t)b * n_docs + doc] = ordered_to_float(ok);
    keys[i] = make_key(ok, doc);
  }
  __syncthreads();
  const int kk = min(k, n);
  block_topk(keys, n, kk, out, tmp, hist, state);
  if (n_slices == 1) {
    for (int i = threadIdx.x; i < kk; i += blockDim.x) {
      topk_idx[(size_t)b * k + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(out[i] & 0xFFFFFFFFu));
      topk_score[(size_t)b * k + i] = ordered_to_float((uint32_t)(out[i] >> 32));
    }
  } else {
    for (int i = threadIdx.x; i < k; i += blockDim.x)
      cand[((size_t)b * n_slices + slice) * k + i] = (i < kk) ? out[i] : 0ull;
  }
}

__global__ void __launch_bounds__(kTopkThreads) topk_merge_kernel(const uint64_t* __restrict__ cand,
                                                                  int n_slices, int k,
                                                                  int32_t* __restrict__ topk_idx,
                                                                  float* __restrict__ topk_score) {
  extern __shared__ uint64_t sm64[];
  const int n = n_slices * k;
  uint64_t* keys = sm64;
  uint64_t* out = keys + n;
  uint64_t* tmp = out + 256;
  uint64_t* state = tmp + 256;
  uint32_t* hist = reinterpret_cast<uint32_t*>(state + 4);
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = cand[(size_t)b * n + i];
  __syncthreads();
  block_topk(keys, n, k, out, tmp, hist, state);
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    topk_idx[(size_t)b * k + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(out[i] & 0xFFFFFFFFu));
    topk_score[(size_t)b * k + i] = ordered_to_float((uint32_t)(out[i] >> 32));
  }
}

template <int NB, int DR, bool MEAN>
cudaError_t launch_scan_t(const CUtensorMap& map, const ScanParams& p, int grid, size_t smem, cudaStream_t s) {
  auto kern = scan_kernel<NB, DR, MEAN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3((p.n_r + 1) * 32), smem, s, map, p);
}

template <int DR, bool MEAN>
cudaError_t launch_scan_nb(int nb, const CUtensorMap& map, const ScanParams& p, int grid, size_t smem,
                           cudaStream_t s) {
  switch (nb) {
    case 1: return launch_scan_t<1, DR, MEAN>(map, p, grid, smem, s);
    case 2: return launch_scan_t<2, DR, MEAN>(map, p, grid, smem, s);
    case 3: return launch_scan_t<3, DR, MEAN>(map, p, grid, smem, s);
    default: return launch_scan_t<4, DR, MEAN>(map, p, grid, smem, s);
  }
}

size_t scan_smem_bytes(int n_r, int d_r, int nb) {
  const size_t stage = (size_t)n_r * (d_r / 64) * kBoxBytes;
  return 1024 + kStages * stage + 2ull * n_r * 8 * nb * kPartStride * sizeof(float) + 32 * sizeof(int) +
         2 * kStages * sizeof(uint64_t);
}

size_t topk_slice_smem() { return (kSliceDocs + 512 + 4) * sizeof(uint64_t) + 256 * sizeof(uint32_t); }
size_t topk_merge_smem(int n) { return ((size_t)n + 512 + 4) * sizeof(uint64_t) + 256 * sizeof(uint32_t); }

}  // namespace

size_t route_workspace(const msa_dims& d, int B, int n_docs, int n_chunks, int k, msa_doc_agg agg, void* ws,
                       RouteWs* out) {
  Carver cv(ws);
  RouteWs w{};
  const int NR = d.n_r * d.d_r;
  w.ksplit = std::max(1, std::min(32, d.hidden / 160));
  w.nb_total = (B + 7) / 8;
  w.n_slices = (n_docs + kSliceDocs - 1) / kSliceDocs;
  w.qr_part = cv.take<float>((size_t)w.ksplit * B * NR);
  w.qfrag = cv.take<uint4>((size_t)d.n_r * (d.d_r / 16) * w.nb_total * 32);
  w.doc_key = agg == MSA_AGG_MAX ? cv.take<uint32_t>((size_t)B * n_docs) : nullptr;
  w.chunk_s = agg == MSA_AGG_MEAN ? cv.take<float>((size_t)B * n_chunks) : nullptr;
  w.cand = w.n_slices > 1 ? cv.take<uint64_t>((size_t)B * w.n_slices * k) : nullptr;
  if (out) *out = w;
  return cv.size();
}

msa_status route_launch(const msa_dims& d, const void* Hq, const void* W_QR, int B, const void* KR_bar,
                        const int32_t* chunk_off, int n_docs, int n_chunks, int k, msa_doc_agg agg,
                        float* doc_scores, int32_t* topk_idx, float* topk_score, void* ws, cudaStream_t s) {
  RouteWs w;
  route_workspace(d, B, n_docs, n_chunks, k, agg, ws, &w);
  const int NR = d.n_r * d.d_r;
  const bool mean = agg == MSA_AGG_MEAN;

  // K1: Q^R partial sums
  if (W_QR) {
    TraceScope ts(kKQrProj, s);
    const int rows = (d.hidden + w.ksplit - 1) / w.ksplit;
    MSA_CUDA_CHECK(launch_pdl(qr_proj_kernel, dim3(NR / kQpCols, w.ksplit), dim3(256), 0, s,
                              static_cast<const __nv_bfloat16*>(Hq), static_cast<const __nv_bfloat16*>(W_QR), B,
                              d.hidden, NR, rows, w.qr_part));
  }
  // K2: normalise + fragments + clear document keys
  {
    TraceScope ts(kKQPrep, s);
    const size_t sm = (size_t)(NR + d.n_r) * sizeof(float);
    MSA_CUDA_CHECK(launch_pdl(q_prep_kernel, dim3(w.nb_total * 8), dim3(256), sm, s, (const float*)w.qr_part,
                              w.ksplit, W_QR ? nullptr : static_cast<const __nv_bfloat16*>(Hq), B, d.n_r, d.d_r,
                              w.nb_total, w.qfrag, w.doc_key, n_docs));
  }
  // K3: scan, 32 queries per pass
  {
    CUtensorMap map;
    const uint64_t dims[2] = {(uint64_t)NR, (uint64_t)n_chunks};
    const uint64_t strides[1] = {(uint64_t)NR * 2};
    const uint32_t box[2] = {64, (uint32_t)kTileC};
    msa_status st = encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(KR_bar), dims,
                                      strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    const int n_tiles = (n_chunks + kTileC - 1) / kTileC;
    const int grid = std::max(1, std::min(sm_count(), n_tiles));
    for (int nb_base = 0; nb_base < w.nb_total; nb_base += 4) {
      const int nb = std::min(4, w.nb_total - nb_base);
      ScanParams p;
      p.qfrag = w.qfrag;
      p.chunk_off = chunk_off;
      p.doc_key = w.doc_key;
      p.chunk_s = w.chunk_s;
      p.n_r = d.n_r;
      p.n_docs = n_docs;
      p.n_chunks = n_chunks;
      p.n_tiles = n_tiles;
      p.q_base = nb_base * 8;
      p.q_count = std::min(B - p.q_base, nb * 8);
      p.nb_total = w.nb_total;
      p.nb_base = nb_base;
      p.inv_nr = 1.0f / (float)d.n_r;
      const size_t smem = scan_smem_bytes(d.n_r, d.d_r, nb);
      TraceScope ts(kKScan, s);
      cudaError_t e;
      if (d.d_r == 128)
        e = mean ? launch_scan_nb<128, true>(nb, map, p, grid, smem, s) : launch_scan_nb<128, false>(nb, map, p, grid, smem, s);
      else
        e = mean ? launch_scan_nb<64, true>(nb, map, p, grid, smem, s) : launch_scan_nb<64, false>(nb, map, p, grid, smem, s);
      if (e != cudaSuccess) return cuda_fail(e, "scan_kernel launch");
    }
  }
  // K4: top-k
  {
    TraceScope ts(kKTopkSlice, s);
    const size_t sm = topk_slice_smem();
    MSA_CUDA_CHECK(cudaFuncSetAttribute(topk_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    MSA_CUDA_CHECK(launch_pdl(topk_slice_kernel, dim3(w.n_slices, B), dim3(kTopkThreads), sm, s,
                              (const uint32_t*)w.doc_key, (const float*)w.chunk_s, chunk_off, n_docs, n_chunks, k,
                              w.n_slices, doc_scores, w.cand, topk_idx, topk_score));
  }
  if (w.n_slices > 1) {
    TraceScope ts(kKTopkMerge, s);
    const size_t sm = topk_merge_smem(w.n_slices * k);
    MSA_CUDA_CHECK(cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    MSA_CUDA_CHECK(launch_pdl(topk_merge_kernel, dim3(B), dim3(kTopkThreads), sm, s, (const uint64_t*)w.cand,
                              w.n_slices, k, topk_idx, topk_score));
  }
  return MSA_OK;
}

}  // namespace msa

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
//                        position j, angle reduced in fp64
//   attn_split_kernel    split-KV flash-decode: CTA = (split, KV head, query);
//                        gathers its key/value rows with per-row bulk async
//                        copies into padded shared memory, QK^T and PV on the
//                        tensor cores (mma.sync, the GQA group as the M rows),
//                        local keys rotated in registers, online softmax
//   attn_combine_kernel  log-sum-exp merge of the split partials -> bf16
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
  int n_splits;
};

namespace {

constexpr int kTK = 64;          // keys per tile
constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 128;
constexpr int kMaxK = 256;
constexpr float kLog2e = 1.4426950408889634f;

// cos/sin of (pos_offset + j) * theta_i, theta_i = base^(-2i/D), for local
// positions j.  One block per 64 positions: the block's base angle
// (pos_offset + 64 jh) theta_i is reduced and evaluated in fp64, the in-block
// offset jl * theta_i (< 64 rad) in fp32, and the two are combined by the
// angle-addition identities.
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ tab, int t_loc_max, int half,
                                                         int pos_offset, double log_base, int head_dim) {
  __shared__ float2 coarse[128];
  __shared__ float theta_f[128];
  pdl_launch_dependents();
  pdl_wait();
  const int jh = blockIdx.x;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double theta = exp(-2.0 * (double)i / (double)head_dim * log_base);
    double a = (double)(pos_offset + 64 * jh) * theta;
    const double two_pi = 6.283185307179586476925286766559;
    a -= two_pi * rint(a / two_pi);
    double sv, cv;
    sincos(a, &sv, &cv);
    coarse[i] = make_float2((float)cv, (float)sv);
    theta_f[i] = (float)theta;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 64 * half; e += blockDim.x) {
    const int jl = e / half, i = e % half;
    const int j = 64 * jh + jl;
    if (j >= t_loc_max) break;
    float sf, cf;
    sincosf((float)jl * theta_f[i], &sf, &cf);
    const float2 cb = coarse[i];
    tab[(size_t)j * half + i] = make_float2(cb.x * cf - cb.y * sf, cb.y * cf + cb.x * sf);
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
  const float2* rope_tab;
  float* part_ml;
  float* part_o;
  int n_q, n_kv, k, n_docs, t_loc_max, pos_offset, n_splits;
  float scale_log2;  // softmax scale * log2(e)
  double log_base;
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads) attn_split_kernel(const AttnParams p) {
  constexpr int KS = D / 16;
  constexpr int ROWB = D * 2 + 16;          // padded smem row (bytes): conflict-free ldmatrix
  constexpr int TILEB = kTK * ROWB;         // one tensor (K or V) of one stage
  constexpr int NBLK = D / 8;               // output column blocks
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t* stage_mem = sm;                                         // [stages][K tile | V tile]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kAttnStages * 2 * TILEB);
  int* seg_v = reinterpret_cast<int*>(bars + kAttnStages);         // [k + 1] virtual starts
  int* seg_c = seg_v + kMaxK + 2;                                  // [k] chunk starts (8-byte aligned end)

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.n_q / p.n_kv;
  const int k = p.k;

  // zero the stage buffers once (rows past a range end are never copied) and set up barriers:
  // nothing here touches global memory, so it overlaps the previous kernel's tail
  for (int i = tid; i < kAttnStages * 2 * TILEB / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(stage_mem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    for (int s = 0; s < kAttnStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  pdl_launch_dependents();
  pdl_wait();

  // ---- segment table of this query: selected docs in top-k order, then local ----
  for (int r = tid; r < k; r += blockDim.x) {
    int doc = p.topk_idx[(size_t)b * k + r];
    int c0 = 0, n = 0;
    if (doc >= 0 && doc < p.n_docs) {
      c0 = __ldg(&p.chunk_off[doc]);
      n = __ldg(&p.chunk_off[doc + 1]) - c0;
    } else {
      raise_dev_error(kDevErrBadIndex);
    }
    seg_c[r] = c0;
    seg_v[r + 1] = n;
  }
  int L = p.loc_len[b];
  L = max(0, min(L, p.t_loc_max));
  __syncthreads();
  if (warp == 0) {
    // inclusive scan of chunk counts -> virtual starts (lane owns a run of entries)
    const int per = (k + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
      const int r = lane * per + j;
      if (r < k) local += seg_v[r + 1];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int j = 0; j < per; ++j) {
      const int r = lane * per + j;
      if (r < k) {
        run += seg_v[r + 1];
        seg_v[r + 1] = run;
      }
    }
    if (lane == 0) seg_v[0] = 0;
  }
  fence_proxy_async_smem();
  __syncthreads();

  const int n_sel = seg_v[k];
  const int n_keys = n_sel + L;
  int per_split = (n_keys + p.n_splits - 1) / p.n_splits;
  per_split = (per_split + 15) & ~15;
  const int v0 = min(n_keys, split * per_split);
  const int v1 = min(n_keys, v0 + per_split);
  const int n_tiles = (v1 - v0 + kTK - 1) / kTK;

  // ---- issue one tile's row copies (warp 0); every other warp just waits ----
  const size_t kv_stride_c = (size_t)p.n_kv * D;  // elements between chunks / local tokens
  auto issue = [&](int t, int st) {
    if (warp != 0) return;
    const int tv0 = v0 + t * kTK;
    const int rows = min(kTK, v1 - tv0);
    if (lane == 0) mbar_arrive_expect_tx(&bars[st], (uint32_t)(2 * rows * D * 2));
    __syncwarp();
    uint8_t* kdst = stage_mem + (size_t)st * 2 * TILEB;
    uint8_t* vdst = kdst + TILEB;
    for (int r = lane; r < rows; r += 32) {
      const int v = tv0 + r;
      const __nv_bfloat16 *ks, *vs;
      if (v < n_sel) {
        int lo = 0, hi = k - 1;  // segment with seg_v[lo] <= v < seg_v[lo + 1]
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (seg_v[mid] <= v) lo = mid; else hi = mid - 1;
        }
        const size_t ch = (size_t)(seg_c[lo] + (v - seg_v[lo]));
        ks = p.K_bar + ch * kv_stride_c + (size_t)h * D;
        vs = p.V_bar + ch * kv_stride_c + (size_t)h * D;
      } else {
        const size_t j = (size_t)(v - n_sel);
        const size_t off = ((size_t)b * p.t_loc_max + j) * kv_stride_c + (size_t)h * D;
        ks = p.K_loc + off;
        vs = p.V_loc + off;
      }
      bulk_load(kdst + r * ROWB, ks, D * 2, &bars[st]);
      bulk_load(vdst + r * ROWB, vs, D * 2, &bars[st]);
    }
  };
  // start streaming before the query fragments are built
  for (int t = 0; t < kAttnStages - 1 && t < n_tiles; ++t) issue(t, t % kAttnStages);

  // ---- query fragments: rotate to pos_offset + L - 1, scale, bf16 (A operand, rows = GQA heads) ----
  float2* qcs = reinterpret_cast<float2*>(seg_c + kMaxK);  // [D/2] cos/sin at the query position
  for (int i = tid; i < D / 2; i += blockDim.x) {
    if (L >= 1) {
      qcs[i] = p.rope_tab[(size_t)(L - 1) * (D / 2) + i];  // the decode token is local token L - 1
    } else {
      double a = (double)(p.pos_offset - 1) * exp(-2.0 * (double)i / (double)D * p.log_base);
      const double two_pi = 6.283185307179586476925286766559;
      a -= two_pi * rint(a / two_pi);
      double sv, cv;
      sincos(a, &sv, &cv);
      qcs[i] = make_float2((float)cv, (float)sv);
    }
  }
  __syncthreads();
  const int g = lane >> 2, c = lane & 3;
  uint32_t qa[KS][4];
  {
    const uint16_t* qb = reinterpret_cast<const uint16_t*>(p.q) + ((size_t)b * p.n_q + (size_t)h * G) * D;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {        // rows g and g + 8
        const int row = g + 8 * rr;
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {      // k cols 2c.. and 2c+8..
          const int dim = 16 * s + 8 * hk + 2 * c;
          float v[2] = {0.f, 0.f};
          if (row < G) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int dd = dim + e;
              const bool first = dd < D / 2;
              const int i = first ? dd : dd - D / 2;
              const int partner = first ? dd + D / 2 : dd - D / 2;
              const float x = bf16_bits_to_float(qb[(size_t)row * D + dd]);
              const float y = bf16_bits_to_float(qb[(size_t)row * D + partner]);
              const float2 cs = qcs[i];
              // first half: x cos - y sin; second half: x cos + y sin (y = first-half partner)
              const float rot = first ? (x * cs.x - y * cs.y) : (x * cs.x + y * cs.y);
              v[e] = rot * p.scale_log2;
            }
          }
          qa[s][rr + 2 * hk] = pack_bf16x2(v[0], v[1]);
        }
      }
    }
  }

  float acc[NBLK][4];
#pragma unroll
  for (int n = 0; n < NBLK; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};

  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % kAttnStages;
    if (t + kAttnStages - 1 < n_tiles) issue(t + kAttnStages - 1, (t + kAttnStages - 1) % kAttnStages);
    mbar_wait(&bars[st], (t / kAttnStages) & 1);

    const int tv0 = v0 + t * kTK;
    const uint32_t kbase = smem_u32(stage_mem + (size_t)st * 2 * TILEB);
    const uint32_t vbase = kbase + TILEB;
    const int wkey0 = 16 * warp;  // this warp's 16 keys within the tile

    if (tv0 + wkey0 < v1) {
      // ---- K fragments (B operand, keys = n) ----
      uint32_t kb[KS][2][2];
      {
        const int key = wkey0 + (lane & 7) + 8 * (lane >> 4);
        const int dsel = 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int s = 0; s < KS; ++s)
          ldmatrix_x4(kb[s][0][0], kb[s][0][1], kb[s][1][0], kb[s][1][1], kbase + key * ROWB + (16 * s + dsel) * 2);
      }
      // ---- rotate local keys in registers (pairs i, i + D/2 sit in ksteps s, s + KS/2) ----
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const int v = tv0 + wkey0 + 8 * nb + g;
        if (v >= n_sel && v < v1) {
          const float2* tab = p.rope_tab + (size_t)(v - n_sel) * (D / 2);
#pragma unroll
          for (int s = 0; s < KS / 2; ++s) {
#pragma unroll
            for (int hk = 0; hk < 2; ++hk) {
              const int i = 16 * s + 8 * hk + 2 * c;
              const float4 cs = *reinterpret_cast<const float4*>(tab + i);  // (cos_i, sin_i, cos_i+1, sin_i+1)
              const float2 x = unpack_bf16x2(kb[s][nb][hk]);
              const float2 y = unpack_bf16x2(kb[s + KS / 2][nb][hk]);
              const float x0 = x.x * cs.x - y.x * cs.y, y0 = y.x * cs.x + x.x * cs.y;
              const float x1 = x.y * cs.z - y.y * cs.w, y1 = y.y * cs.z + x.y * cs.w;
              kb[s][nb][hk] = pack_bf16x2(x0, x1);
              kb[s + KS / 2][nb][hk] = pack_bf16x2(y0, y1);
            }
          }
        }
      }
      // ---- S = q K^T (rows = heads, cols = 16 keys) ----
      float sc[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
#pragma unroll
        for (int s = 0; s < KS; ++s)
          mma_bf16_16816(sc[nb], qa[s][0], qa[s][1], qa[s][2], qa[s][3], kb[s][nb][0], kb[s][nb][1]);
      }
      // mask keys past the range end
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int v = tv0 + wkey0 + 8 * nb + 2 * c + e;
          if (v >= v1) {
            sc[nb][e] = -INFINITY;
            sc[nb][2 + e] = -INFINITY;
          }
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
        const int key = wkey0 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int dsel = 8 * (lane >> 4);
#pragma unroll
        for (int n = 0; n < NBLK; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(b0, b1, b2, b3, vbase + key * ROWB + (8 * n + dsel) * 2);
          mma_bf16_16816(acc[n], pa0, pa1, pa2, pa3, b0, b1);
          mma_bf16_16816(acc[n + 1], pa0, pa1, pa2, pa3, b2, b3);
        }
      }
    }
    __syncthreads();  // every warp is done with stage st before it is refilled
  }

  // ---- merge the 4 warps' partial softmax states and write this split's partial ----
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 1);
    l_run[rr] += __shfl_xor_sync(0xffffffffu, l_run[rr], 2);
  }
  float* wm = reinterpret_cast<float*>(stage_mem);   // [4][16]
  float* wl = wm + 4 * 16;                           // [4][16]
  float* wo = wl + 4 * 16;                           // [4][16][D]
  if (c == 0) {
    wm[warp * 16 + g] = m_run[0];
    wm[warp * 16 + g + 8] = m_run[1];
    wl[warp * 16 + g] = l_run[0];
    wl[warp * 16 + g + 8] = l_run[1];
  }
#pragma unroll
  for (int n = 0; n < NBLK; ++n) {
    wo[(warp * 16 + g) * D + 8 * n + 2 * c] = acc[n][0];
    wo[(warp * 16 + g) * D + 8 * n + 2 * c + 1] = acc[n][1];
    wo[(warp * 16 + g + 8) * D + 8 * n + 2 * c] = acc[n][2];
    wo[(warp * 16 + g + 8) * D + 8 * n + 2 * c + 1] = acc[n][3];
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int row = idx / D, dim = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * 16 + row]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float sw = exp2f(wm[w * 16 + row] - Mu);
      o += sw * wo[(w * 16 + row) * D + dim];
      l += sw * wl[w * 16 + row];
    }
    const size_t qh = (size_t)b * p.n_q + (size_t)h * G + row;
    p.part_o[(qh * p.n_splits + split) * D + dim] = o;
    if (dim == 0) {
      p.part_ml[(qh * p.n_splits + split) * 2 + 0] = M;
      p.part_ml[(qh * p.n_splits + split) * 2 + 1] = l;
    }
  }
}

template <int D>
__global__ void attn_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o,
                                    int n_splits, __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t qh = (size_t)blockIdx.y * gridDim.x + blockIdx.x;  // b * n_q + head
  const float* ml = part_ml + qh * n_splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[2 * s]);
  const float Mu = (M == -INFINITY) ? 0.f : M;
  for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
    float o = 0.f, l = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float w = exp2f(ml[2 * s] - Mu);
      o += w * part_o[(qh * n_splits + s) * D + dim];
      l += w * ml[2 * s + 1];
    }
    out[qh * D + dim] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
  }
}

template <int D>
size_t attn_smem() {
  return (size_t)kAttnStages * 2 * kTK * (D * 2 + 16) + kAttnStages * sizeof(uint64_t) +
         (2 * kMaxK + 2) * sizeof(int) + (D / 2) * sizeof(float2);
}

int choose_splits(int B, int n_kv, int t_loc_max, int k) {
  const int target = 2 * sm_count();
  int s = (target + B * n_kv - 1) / (B * n_kv);
  const int max_useful = std::max(1, (t_loc_max + 64 * k) / 64);
  return std::max(1, std::min({s, max_useful, 128}));
}

}  // namespace

size_t attend_workspace(const msa_dims& d, int B, int k, int t_loc_max, int pos_offset, void* ws, AttendWs* out) {
  (void)pos_offset;
  Carver cv(ws);
  AttendWs w{};
  w.n_splits = choose_splits(B, d.n_kv, t_loc_max, k);
  w.rope_tab = cv.take<float2>((size_t)std::max(1, t_loc_max) * (d.head_dim / 2));
  w.part_ml = cv.take<float>((size_t)B * d.n_q * w.n_splits * 2);
  w.part_o = cv.take<float>((size_t)B * d.n_q * w.n_splits * d.head_dim);
  if (out) *out = w;
  return cv.size();
}

msa_status rope_cache_build(const msa_dims& d, int t_loc_max, int pos_offset, float2* tab, cudaStream_t s) {
  if (t_loc_max <= 0) return MSA_OK;
  const int D = d.head_dim;
  TraceScope ts(kKRopeTable, s);
  MSA_CUDA_CHECK(launch_pdl(rope_table_kernel, dim3((t_loc_max + 63) / 64), dim3(256), 0, s, tab, t_loc_max, D / 2,
                            pos_offset, std::log((double)d.rope_base), D));
  return MSA_OK;
}

msa_status attend_launch(const msa_dims& d, const void* q, int B, const void* K_bar, const void* V_bar,
                         const int32_t* chunk_off, int n_docs, const int32_t* topk_idx, int k, const void* K_loc,
                         const void* V_loc, const int32_t* loc_len, int t_loc_max, int pos_offset,
                         const void* rope_cache, float scale, void* out, void* ws, cudaStream_t s) {
  AttendWs w;
  attend_workspace(d, B, k, t_loc_max, pos_offset, ws, &w);
  const int D = d.head_dim;
  const double log_base = std::log((double)d.rope_base);
  const float2* tab = static_cast<const float2*>(rope_cache);
  if (!tab) {
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
  p.rope_tab = tab;
  p.part_ml = w.part_ml;
  p.part_o = w.part_o;
  p.n_q = d.n_q;
  p.n_kv = d.n_kv;
  p.k = k;
  p.n_docs = n_docs;
  p.t_loc_max = t_loc_max;
  p.pos_offset = pos_offset;
  p.n_splits = w.n_splits;
  p.scale_log2 = (scale > 0.f ? scale : 1.0f / std::sqrt((float)D)) * kLog2e;
  p.log_base = log_base;
  {
    TraceScope ts(kKAttnSplit, s);
    dim3 grid(w.n_splits, d.n_kv, B);
    if (D == 128) {
      const size_t sm = attn_smem<128>();
      MSA_CUDA_CHECK(cudaFuncSetAttribute(attn_split_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
      MSA_CUDA_CHECK(launch_pdl(attn_split_kernel<128>, grid, dim3(kAttnThreads), sm, s, p));
    } else {
      const size_t sm = attn_smem<64>();
      MSA_CUDA_CHECK(cudaFuncSetAttribute(attn_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
      MSA_CUDA_CHECK(launch_pdl(attn_split_kernel<64>, grid, dim3(kAttnThreads), sm, s, p));
    }
  }
  {
    TraceScope ts(kKAttnCombine, s);
    dim3 grid(d.n_q, B);
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
    if (D == 128)
      MSA_CUDA_CHECK(launch_pdl(attn_combine_kernel<128>, grid, dim3(128), 0, s, (const float*)w.part_ml,
                                (const float*)w.part_o, w.n_splits, o));
    else
      MSA_CUDA_CHECK(launch_pdl(attn_combine_kernel<64>, grid, dim3(64), 0, s, (const float*)w.part_ml,
                                (const float*)w.part_o, w.n_splits, o));
  }
  return MSA_OK;
}

}  // namespace msa

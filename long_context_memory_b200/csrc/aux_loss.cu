// Router training signal of MSA: the contrastive auxiliary loss and its gradients.
//
// Definition (IRMaD reading of the MSA paper, "M. Materials & Methods",
// training item; the digest's "Core method" names the same loss):
//   L_aux = -(1/|P|) sum_i log( exp(s_i^+/tau) / (exp(s_i^+/tau) + sum_j exp(s_ij^-/tau)) )
// with s the routing score of a chunk: the head mean of the cosines between
// the router query and the chunk's pooled router key.
//
// Kernel aux_loss_kernel: CTA = one positive i (its query, its positive key
// and its N negative keys).  Pass 1 reads every key once (lane = 8 or 16
// consecutive 16-byte pieces of one head) for the per-head dot products and
// norms, giving the cosines and scores; a block softmax over the 1 + N scores
// gives the loss term and dL/ds.  Pass 2 re-reads the keys (L2-resident: this
// CTA just streamed them) and forms
//   dL/dq_h = (1/n_r) sum_j g_j (k_jh / (|q_h||k_jh|) - cos_jh q_h / |q_h|^2)
//   dL/dk_jh = (g_j/n_r)      (q_h / (|q_h||k_jh|) - cos_jh k_jh / |k_jh|^2)
// (a norm below eps is clamped and its own term dropped).  The per-CTA loss
// terms are summed in positive order by the last CTA (a ticket), so the loss
// does not depend on scheduling.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kAuxThreads = 256;
constexpr int kAuxWarps = kAuxThreads / 32;
constexpr float kAuxEps = 1e-12f;

struct AuxParams {
  const __nv_bfloat16* Q;      // [P][n_r][d_r]
  const __nv_bfloat16* K_pos;  // [P][n_r][d_r]
  const __nv_bfloat16* K_neg;  // [P][N][n_r][d_r]
  float* loss;                 // [1]
  float* dQ;                   // [P][n_r][d_r] or null
  float* dK_pos;               // [P][n_r][d_r] or null
  float* dK_neg;               // [P][N][n_r][d_r] or null
  float* term;                 // [P] per-positive loss terms (workspace)
  uint32_t* ticket;            // [1] CTAs done (workspace, back to 0 after each call)
  int P, N, n_r;
  float inv_tau;
};

// lane -> (head, 16-byte pieces): 4 lanes per head, DR/32 bf16 values per lane
template <int DR>
struct AuxLane {
  static constexpr int kVals = DR / 4;   // values per lane (32 or 16)
  static constexpr int kVecs = kVals / 8;  // uint4 per lane (4 or 2)
};

template <int DR>
__device__ __forceinline__ void load_key(const __nv_bfloat16* row, int h, int part, float* v) {
  using Ln = AuxLane<DR>;
  const uint4* src = reinterpret_cast<const uint4*>(row + (size_t)h * DR + part * Ln::kVals);
  uint4 u[Ln::kVecs];
#pragma unroll
  for (int e = 0; e < Ln::kVecs; ++e) u[e] = __ldg(src + e);
#pragma unroll
  for (int e = 0; e < Ln::kVecs; ++e) {
    float2 f;
    f = unpack_bf16x2(u[e].x); v[8 * e + 0] = f.x; v[8 * e + 1] = f.y;
    f = unpack_bf16x2(u[e].y); v[8 * e + 2] = f.x; v[8 * e + 3] = f.y;
    f = unpack_bf16x2(u[e].z); v[8 * e + 4] = f.x; v[8 * e + 5] = f.y;
    f = unpack_bf16x2(u[e].w); v[8 * e + 6] = f.x; v[8 * e + 7] = f.y;
  }
}

template <int DR>
__global__ void __launch_bounds__(kAuxThreads) aux_loss_kernel(const AuxParams p) {
  using Ln = AuxLane<DR>;
  extern __shared__ __align__(16) float aux_sm[];
  const int n_r = p.n_r, NK = p.N + 1, NR = n_r * DR;
  float* qs = aux_sm;                         // [n_r][DR] query (fp32)
  float* cosv = qs + 8 * DR;                  // [NK][8] cosines
  float* nkv = cosv + (size_t)NK * 8;         // [NK][8] clamped key norms (negative: below eps)
  float* gs = nkv + (size_t)NK * 8;           // [NK] dL/ds_j
  float* red = gs + NK;                       // [kAuxWarps][NR] partial dL/dq
  __shared__ float qn[8];                     // clamped query norms (negative: below eps)
  __shared__ float chead[8];                  // sum_j g_j cos_jh
  __shared__ float wred[kAuxWarps];
  __shared__ bool last;
  pdl_launch_dependents();
  pdl_wait();

  const int i = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = lane >> 2, part = lane & 3;   // this lane's head and quarter of it
  const bool hl = h < n_r;
  const __nv_bfloat16* qrow = p.Q + (size_t)i * NR;
  for (int e = tid; e < NR; e += kAuxThreads) qs[e] = __bfloat162float(qrow[e]);
  __syncthreads();
  if (warp < n_r) {
    float ss = 0.f;
    for (int e = lane; e < DR; e += 32) ss = fmaf(qs[warp * DR + e], qs[warp * DR + e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      const float n = sqrtf(ss);
      qn[warp] = n > kAuxEps ? n : -kAuxEps;  // sign marks a clamped norm
    }
  }
  __syncthreads();

  auto key_row = [&](int j) -> const __nv_bfloat16* {
    return j == 0 ? p.K_pos + (size_t)i * NR : p.K_neg + ((size_t)i * p.N + (j - 1)) * NR;
  };

  // ---- pass 1: cosines and scores ----
  for (int j = warp; j < NK; j += kAuxWarps) {
    float kv[Ln::kVals];
    float dot = 0.f, kk = 0.f;
    if (hl) {
      load_key<DR>(key_row(j), h, part, kv);
      const float* qv = qs + h * DR + part * Ln::kVals;
#pragma unroll
      for (int e = 0; e < Ln::kVals; ++e) {
        dot = fmaf(kv[e], qv[e], dot);
        kk = fmaf(kv[e], kv[e], kk);
      }
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      dot += __shfl_xor_sync(0xffffffffu, dot, o);
      kk += __shfl_xor_sync(0xffffffffu, kk, o);
    }
    if (hl && part == 0) {
      const float nk = sqrtf(kk);
      const float nkc = fmaxf(nk, kAuxEps), nqc = fabsf(qn[h]);
      cosv[(size_t)j * 8 + h] = dot / (nqc * nkc);
      nkv[(size_t)j * 8 + h] = nk > kAuxEps ? nk : -kAuxEps;
    }
  }
  __syncthreads();

  // ---- softmax over the 1 + N scores (z = s / tau) ----
  float zmax = -INFINITY;
  for (int j = tid; j < NK; j += kAuxThreads) {
    float s = 0.f;
    for (int hh = 0; hh < n_r; ++hh) s += cosv[(size_t)j * 8 + hh];
    s /= (float)n_r;
    gs[j] = s * p.inv_tau;  // z_j for now
    zmax = fmaxf(zmax, gs[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
  if (lane == 0) wred[warp] = zmax;
  __syncthreads();
  zmax = wred[0];
#pragma unroll
  for (int w = 1; w < kAuxWarps; ++w) zmax = fmaxf(zmax, wred[w]);
  __syncthreads();
  // the negatives' share, kept apart from the positive's so that neither the loss term
  // log(1 + sum_j e^(z_j - z_0)) nor 1 - p_0 suffers cancellation when p_0 is near 1
  float se = 0.f;
  for (int j = tid; j < NK; j += kAuxThreads)
    if (j > 0) se += expf(gs[j] - zmax);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
  if (lane == 0) wred[warp] = se;
  __syncthreads();
  float se_neg = 0.f;
#pragma unroll
  for (int w = 0; w < kAuxWarps; ++w) se_neg += wred[w];
  const float z0 = gs[0];
  const float e0 = expf(z0 - zmax);
  const float den = e0 + se_neg;  // sum_j e^(z_j - zmax), positive included
  __syncthreads();                // every thread has read gs[0] and wred
  const float inv_p = 1.0f / (float)p.P;
  const float scale = p.inv_tau * inv_p / den;
  // dL/ds_j = p_j / (tau P) for a negative, -(1 - p_0) / (tau P) = -(sum of negatives' p_j) / (tau P)
  for (int j = tid; j < NK; j += kAuxThreads)
    gs[j] = j == 0 ? -se_neg * scale : expf(gs[j] - zmax) * scale;
  if (tid == 0) p.term[i] = (zmax - z0) + log1pf((e0 - 1.0f) + se_neg);  // -log p_0
  __syncthreads();
  if (warp < n_r) {  // c_h = sum_j g_j cos_jh
    float c = 0.f;
    for (int j = lane; j < NK; j += 32) c = fmaf(gs[j], cosv[(size_t)j * 8 + warp], c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) chead[warp] = c;
  }
  __syncthreads();

  // ---- pass 2: gradients ----
  const float inv_nr = 1.0f / (float)n_r;
  float acc[Ln::kVals];
#pragma unroll
  for (int e = 0; e < Ln::kVals; ++e) acc[e] = 0.f;
  const bool want_dk = p.dK_pos != nullptr || p.dK_neg != nullptr;
  if (p.dQ != nullptr || want_dk) {
    for (int j = warp; j < NK; j += kAuxWarps) {
      if (!hl) continue;
      float kv[Ln::kVals];
      load_key<DR>(key_row(j), h, part, kv);
      const float nks = nkv[(size_t)j * 8 + h], nqs = qn[h];
      const float nk = fabsf(nks), nq = fabsf(nqs);
      const float g = gs[j] * inv_nr;
      const float a = g / (nq * nk);  // coefficient of k in dL/dq (summed) and of q in dL/dk
#pragma unroll
      for (int e = 0; e < Ln::kVals; ++e) acc[e] = fmaf(a, kv[e], acc[e]);
      float* dk = j == 0 ? (p.dK_pos ? p.dK_pos + (size_t)i * NR : nullptr)
                         : (p.dK_neg ? p.dK_neg + ((size_t)i * p.N + (j - 1)) * NR : nullptr);
      if (dk) {
        const float b = nks > 0.f ? g * cosv[(size_t)j * 8 + h] / (nk * nk) : 0.f;
        const float* qv = qs + h * DR + part * Ln::kVals;
        float4* d4 = reinterpret_cast<float4*>(dk + h * DR + part * Ln::kVals);
#pragma unroll
        for (int e = 0; e < Ln::kVals / 4; ++e)
          d4[e] = make_float4(a * qv[4 * e + 0] - b * kv[4 * e + 0], a * qv[4 * e + 1] - b * kv[4 * e + 1],
                              a * qv[4 * e + 2] - b * kv[4 * e + 2], a * qv[4 * e + 3] - b * kv[4 * e + 3]);
      }
    }
    if (p.dQ != nullptr) {
      if (hl) {
#pragma unroll
        for (int e = 0; e < Ln::kVals; ++e) red[(size_t)warp * NR + h * DR + part * Ln::kVals + e] = acc[e];
      }
      __syncthreads();
      for (int e = tid; e < NR; e += kAuxThreads) {
        const int hh = e / DR;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kAuxWarps; ++w) v += red[(size_t)w * NR + e];
        const float nqs = qn[hh], nq = fabsf(nqs);
        if (nqs > 0.f) v -= chead[hh] * inv_nr * qs[e] / (nq * nq);
        p.dQ[(size_t)i * NR + e] = v;
      }
    }
  }

  // ---- loss: the last CTA sums the terms in positive order ----
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.ticket, 1u);
    last = prev == (uint32_t)(p.P - 1);
    if (last) *p.ticket = 0u;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (warp == 0) {
    // lane l sums terms l, l + 32, ... in order; the 32 partial sums are added in lane order
    float s = 0.f;
    for (int e = lane; e < p.P; e += 32) s += __ldcg(&p.term[e]);
    float tot = 0.f;
    for (int l = 0; l < 32; ++l) tot += __shfl_sync(0xffffffffu, s, l);
    if (lane == 0) *p.loss = tot / (float)p.P;
  }
}

size_t aux_smem_bytes(int d_r, int n_keys) {
  return ((size_t)8 * d_r + (size_t)n_keys * 8 * 2 + n_keys + (size_t)kAuxWarps * 8 * d_r) * sizeof(float);
}

}  // namespace

size_t aux_workspace(const msa_dims& d, int P, int N, void* ws, AuxWs* out) {
  (void)d;
  (void)N;
  Carver cv(ws);
  AuxWs w{};
  w.term = cv.take<float>((size_t)P);
  w.ticket = cv.take<uint32_t>(1);
  if (out) *out = w;
  return cv.size();
}

msa_status aux_loss_launch(const msa_dims& d, const void* QR, const void* K_pos, const void* K_neg, int P, int N,
                           float tau, float* loss, float* dQ, float* dK_pos, float* dK_neg, void* ws,
                           cudaStream_t s) {
  AuxWs w;
  aux_workspace(d, P, N, ws, &w);
  MSA_CUDA_CHECK(cudaMemsetAsync(w.ticket, 0, sizeof(uint32_t), s));
  AuxParams p;
  p.Q = static_cast<const __nv_bfloat16*>(QR);
  p.K_pos = static_cast<const __nv_bfloat16*>(K_pos);
  p.K_neg = static_cast<const __nv_bfloat16*>(K_neg);
  p.loss = loss;
  p.dQ = dQ;
  p.dK_pos = dK_pos;
  p.dK_neg = dK_neg;
  p.term = w.term;
  p.ticket = w.ticket;
  p.P = P;
  p.N = N;
  p.n_r = d.n_r;
  p.inv_tau = 1.0f / tau;
  const size_t sm = aux_smem_bytes(d.d_r, N + 1);
  TraceScope ts(kKAuxLoss, s);
  if (d.d_r == 128) {
    MSA_CUDA_CHECK(cudaFuncSetAttribute(aux_loss_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    MSA_CUDA_CHECK(launch_pdl(aux_loss_kernel<128>, dim3(P), dim3(kAuxThreads), sm, s, p));
  } else {
    MSA_CUDA_CHECK(cudaFuncSetAttribute(aux_loss_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
    MSA_CUDA_CHECK(launch_pdl(aux_loss_kernel<64>, dim3(P), dim3(kAuxThreads), sm, s, p));
  }
  return MSA_OK;
}

}  // namespace msa

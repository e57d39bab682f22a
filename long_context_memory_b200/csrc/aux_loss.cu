// Router training signal of MSA: the contrastive auxiliary loss and its gradients.
//
// Definition (IRMaD reading of the MSA paper, "M. Materials & Methods",
// training item; the digest's "Core method" names the same loss):
//   L_aux = -(1/|P|) sum_i log( exp(s_i^+/tau) / (exp(s_i^+/tau) + sum_j exp(s_ij^-/tau)) )
// with s the routing score of a chunk: the head mean of the cosines between
// the router query and the chunk's pooled router key.
//
// Kernel aux_loss_kernel: a persistent grid; CTA c takes positives c, c + grid, ...
// One producer warp streams every positive's 1 + N key rows (positive first)
// through a shared-memory ring with bulk async copies, 8 rows per stage, twice:
// pass 1 (from HBM) for the per-head dot products and norms -> cosines ->
// scores -> a block softmax -> the loss term and dL/ds; pass 2 (the same rows,
// now in L2) for
//   dL/dq_h = (1/n_r) sum_j g_j (k_jh / (|q_h||k_jh|) - cos_jh q_h / |q_h|^2)
//   dL/dk_jh = (g_j/n_r)      (q_h / (|q_h||k_jh|) - cos_jh k_jh / |k_jh|^2)
// (a norm below eps is clamped and its own term dropped).  The producer runs
// ahead into the next positive while the compute warps finish the current one,
// so the copy engine never waits on the softmax.  Eight compute warps, one key
// row each per stage; lane = (head, quarter of the head), its query values in
// registers.  The per-positive loss terms are summed in positive order by the
// last CTA (a ticket), so the loss does not depend on scheduling.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace msa {
namespace {

constexpr int kAuxCompute = 8;                      // compute warps
constexpr int kAuxThreads = 32 * (kAuxCompute + 1);  // + the producer warp
constexpr int kAuxRows = 8;                         // key rows per stage (one per compute warp)
constexpr int kAuxStagesMax = 8;  // ring stages when a positive's rows stay resident (<= 64 rows)
constexpr int kAuxStagesRing = 6; // ring stages when they stream twice (more than 63 negatives)

// a positive's rows stay in the ring for both passes when the gradients are wanted and they fit
__host__ __device__ inline bool aux_resident(bool grads, int nk) {
  return grads && (nk + kAuxRows - 1) / kAuxRows <= kAuxStagesMax;
}
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
  uint32_t* ticket;            // [1] CTAs done (workspace)
  int P, N, n_r;
  int stages;                  // ring stages (aux_stages, computed on the host)
  float inv_tau;
};

// shared memory: ring [stages][kAuxRows][n_r * DR] bf16 | cos, |k| [NK][8] fp32 | g [NK] |
// per compute warp two rows of kRow floats (its dK rows, in the gradient's own order, handed to
// bulk stores; then its dQ partial) | barriers
template <int DR>
struct AuxSmem {
  static constexpr int kRowBytes = 8 * DR * 2;  // room for 8 router heads
  static constexpr int kStageBytes = kAuxRows * kRowBytes;
  static constexpr int kRow = 8 * DR;           // one gradient row (room for 8 router heads)
  static constexpr int kStg = 2 * kRow;         // a compute warp's two staging rows
  static constexpr int kQBytes = 8 * DR * 2;    // one query row (room for 8 router heads)
  static __host__ __device__ size_t bytes(int nk, int stages) {
    return (size_t)stages * kStageBytes + 2 * kQBytes + (size_t)nk * 8 * 4 * 2 + (size_t)nk * 4 + 16 +
           (size_t)kAuxCompute * kStg * 4 + (2 * kAuxStagesMax + 4) * 8 + 16;
  }
};

// ring stages: every row of a positive when they stay resident, otherwise kAuxStagesRing, fewer
// when the shared memory would not hold them (many negatives: the per-row cosines and norms grow)
constexpr size_t kAuxSmemBudget = 227 * 1024 - 1024;  // dynamic shared memory, beside the static
template <int DR>
__host__ __device__ inline int aux_stages(bool grads, int nk) {
  if (aux_resident(grads, nk)) return kAuxStagesMax;
  int st = kAuxStagesRing;
  while (st > 2 && AuxSmem<DR>::bytes(nk, st) > kAuxSmemBudget) --st;
  return st;
}

// lane l of a compute warp owns head l / 4, quarter l % 4: U 16-byte units of the row.
// Slot e of a lane holds unit (e + rot) % U of its quarter (rot = l / (8 / U)), so that a
// warp's 16-byte loads from shared memory fall in 8 distinct bank groups (4 wavefronts, no
// conflict).  Every per-lane array (key values, query values, gradient partials) is kept
// in slot order; only addresses are rotated.
template <int DR>
__device__ __forceinline__ int unit_of_slot(int e, int lane) {
  constexpr int U = DR / 32;
  return (e + lane / (8 / U)) % U;
}


__device__ __forceinline__ void aux_bar_sync() { named_bar_sync(1, 32 * kAuxCompute); }
// the same barrier, returning whether any compute thread passed `failed` (then all leave together)
__device__ __forceinline__ bool aux_bar_any(bool failed) { return named_bar_any(1, 32 * kAuxCompute, failed); }

template <int DR>
__global__ void __launch_bounds__(kAuxThreads, 1) aux_loss_kernel(const AuxParams p) {
  using Sm = AuxSmem<DR>;
  constexpr int V = DR / 4;  // values per lane
  extern __shared__ __align__(128) uint8_t aux_sm[];
  const int n_r = p.n_r, NK = p.N + 1, NR = n_r * DR;
  uint8_t* ring = aux_sm;
  const bool grads = p.dQ != nullptr || p.dK_pos != nullptr || p.dK_neg != nullptr;
  const int S = p.stages;  // ring stages
  uint8_t* qbuf = aux_sm + S * Sm::kStageBytes;                                   // [2][n_r * DR] bf16
  float* cosv = reinterpret_cast<float*>(qbuf + 2 * Sm::kQBytes);                 // [NK][8]
  float* nkv = cosv + (size_t)NK * 8;                                            // [NK][8]
  float* gs = nkv + (size_t)NK * 8;                                              // [NK]
  float* red = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(gs + NK) + 15) & ~uintptr_t(15));
  // red: [kAuxCompute][Sm::kStg] (16-byte aligned: bulk-store sources)
  uint64_t* full = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(red + (size_t)kAuxCompute * Sm::kStg) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + kAuxStagesMax;
  uint64_t* qfull = empty + kAuxStagesMax;  // [2] a positive's query row landed
  uint64_t* qempty = qfull + 2;          // [2] every compute warp is done with it
  __shared__ float qn[8];      // clamped query norms (negative: below eps)
  __shared__ float chead[8];   // sum_j g_j cos_jh
  __shared__ float wred[kAuxCompute];
  __shared__ bool last;
  __shared__ int abort_flag;   // a bounded wait of this CTA gave up

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_ch = (NK + kAuxRows - 1) / kAuxRows;  // stages per pass
  const int passes = grads ? 2 : 1;
  // With gradients and at most kAuxStagesMax chunks of rows, a positive's rows stay in the ring for
  // both passes: the producer loads them once and pass 2 reads them again from shared memory.
  const bool resident = aux_resident(grads, NK);
  const int loads = resident ? 1 : passes;  // producer passes over a positive's rows
  const size_t row_bytes = (size_t)NR * 2;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kAuxCompute);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], kAuxCompute);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_enter();

  if (warp == kAuxCompute) {
    // ------------------------- producer -------------------------
    if (lane == 0) {
      int it = 0, pi = 0;
      bool stop = false;
      for (int i = blockIdx.x; i < p.P && !stop; i += gridDim.x, ++pi) {
        {  // the positive's query row (double-buffered)
          const int qb = pi & 1;
          if (pi >= 2 && !mbar_wait(&qempty[qb], ((pi >> 1) - 1) & 1, &abort_flag)) break;
          mbar_arrive_expect_tx(&qfull[qb], (uint32_t)row_bytes);
          bulk_load(qbuf + qb * Sm::kQBytes, p.Q + (size_t)i * NR, (uint32_t)row_bytes, &qfull[qb]);
        }
        for (int pass = 0; pass < loads && !stop; ++pass) {
          for (int c = 0; c < n_ch; ++c, ++it) {
            const int st = it % S;
            if (it >= S && !mbar_wait(&empty[st], ((it / S) - 1) & 1, &abort_flag)) {
              stop = true;
              break;
            }
            const int j0 = c * kAuxRows, j1 = min(NK, j0 + kAuxRows);
            uint8_t* dst = ring + (size_t)st * Sm::kStageBytes;
            mbar_arrive_expect_tx(&full[st], (uint32_t)((j1 - j0) * row_bytes));
            int j = j0;
            if (j == 0) {  // the positive's key, then its negatives (contiguous rows)
              bulk_load(dst, p.K_pos + (size_t)i * NR, (uint32_t)row_bytes, &full[st]);
              ++j;
            }
            if (j < j1)
              bulk_load(dst + (size_t)(j - j0) * row_bytes, p.K_neg + ((size_t)i * p.N + (j - 1)) * NR,
                        (uint32_t)((j1 - j) * row_bytes), &full[st]);
          }
        }
      }
      if (abort_flag) {  // the copies still in flight land before the CTA exits
        const int q_issued = stop ? pi + 1 : pi;
        mbar_drain_ring(full, S, it - S, it);
        mbar_drain_ring(qfull, 2, q_issued - 2, q_issued);
      }
    }
    return;
  }

  // ------------------------- compute warps -------------------------
  const int h = lane >> 2;  // this lane's head (lanes of heads >= n_r idle in the row work)
  const bool hl = h < n_r;
  const float inv_nr = 1.0f / (float)n_r;
  const float inv_p = 1.0f / (float)p.P;
  int it = 0, pi = 0;
  bool failed = false;   // a wait of this warp gave up: the compute warps leave together at their next barrier
  for (int i = blockIdx.x; i < p.P; i += gridDim.x, ++pi) {
    // this lane's query values (in slot order, see unit_of_slot) and the head norms
    const int qb = pi & 1;
    const uint16_t* qrow = reinterpret_cast<const uint16_t*>(qbuf + qb * Sm::kQBytes);
    float q[V];
    {
      failed |= !warp_wait(&qfull[qb], (pi >> 1) & 1, &abort_flag);
#pragma unroll
      for (int e = 0; e < DR / 32; ++e) {
        uint4 w = make_uint4(0, 0, 0, 0);
        if (hl) w = *reinterpret_cast<const uint4*>(qrow + lane * V + unit_of_slot<DR>(e, lane) * 8);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = unpack_bf16x2(wv[t]);
          q[8 * e + 2 * t] = f.x;
          q[8 * e + 2 * t + 1] = f.y;
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < V; ++e) ss = fmaf(q[e], q[e], ss);
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      // the previous positive's readers of qn, cos, g and the dq partials are done; the compute
      // warps leave together here once any of their waits has given up (until then every wait
      // of an aborted CTA returns at once and the warps keep to the same barriers)
      if (aux_bar_any(failed)) break;
      if (warp == 0 && hl && (lane & 3) == 0) {
        const float n = sqrtf(ss);
        qn[h] = n > kAuxEps ? n : -kAuxEps;  // sign marks a clamped norm
      }
    }
    aux_bar_sync();  // qn written

    // ---- pass 1: cosines ----
    const int it_first = it;  // ring position of this positive's first chunk
    for (int c = 0; c < n_ch; ++c, ++it) {
      const int st = it % S;
      failed |= !warp_wait(&full[st], (it / S) & 1, &abort_flag);  // on failure: left at the next barrier
      const int j = c * kAuxRows + warp;
      uint4 kw[DR / 32];
      if (j < NK && hl) {
        const uint8_t* base = ring + (size_t)st * Sm::kStageBytes + (size_t)warp * row_bytes + lane * (DR / 32) * 16;
#pragma unroll
        for (int e = 0; e < DR / 32; ++e) kw[e] = *reinterpret_cast<const uint4*>(base + unit_of_slot<DR>(e, lane) * 16);
      }
      if (!resident) {
        // the row is in registers: the stage may refill.  The proxy fence orders these generic-proxy
        // reads before the bulk copy (async proxy) that will overwrite the stage once every warp
        // has arrived, so the last warp to arrive cannot have its loads overtaken by the refill.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      if (j < NK) {
        float dot = 0.f, kk = 0.f;
        if (hl) {
          float d4[4] = {0.f, 0.f, 0.f, 0.f}, k4[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
          for (int e = 0; e < DR / 32; ++e) {
            const uint32_t wv[4] = {kw[e].x, kw[e].y, kw[e].z, kw[e].w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 f = unpack_bf16x2(wv[t]);
              d4[t] = fmaf(f.x, q[8 * e + 2 * t], d4[t]);
              d4[t] = fmaf(f.y, q[8 * e + 2 * t + 1], d4[t]);
              k4[t] = fmaf(f.x, f.x, k4[t]);
              k4[t] = fmaf(f.y, f.y, k4[t]);
            }
          }
          dot = (d4[0] + d4[1]) + (d4[2] + d4[3]);
          kk = (k4[0] + k4[1]) + (k4[2] + k4[3]);
        }
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        kk += __shfl_xor_sync(0xffffffffu, kk, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        kk += __shfl_xor_sync(0xffffffffu, kk, 2);
        if (hl && (lane & 3) == 0) {
          const float nk = sqrtf(kk);
          cosv[(size_t)j * 8 + h] = dot / (fabsf(qn[h]) * fmaxf(nk, kAuxEps));
          nkv[(size_t)j * 8 + h] = nk > kAuxEps ? nk : -kAuxEps;
        }
      }
    }
    aux_bar_sync();

    // ---- softmax over the 1 + N scores (z = s / tau), the negatives kept apart so that
    //      neither log(1 + sum_j e^(z_j - z_0)) nor 1 - p_0 cancels when p_0 is near 1 ----
    const int ct = tid;  // 0 .. 255
    float zmax = -INFINITY;
    for (int j = ct; j < NK; j += 32 * kAuxCompute) {
      float sc = 0.f;
      for (int hh = 0; hh < n_r; ++hh) sc += cosv[(size_t)j * 8 + hh];
      gs[j] = sc * inv_nr * p.inv_tau;  // z_j for now
      zmax = fmaxf(zmax, gs[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
    if (lane == 0) wred[warp] = zmax;
    aux_bar_sync();
    zmax = wred[0];
#pragma unroll
    for (int w = 1; w < kAuxCompute; ++w) zmax = fmaxf(zmax, wred[w]);
    aux_bar_sync();
    float se = 0.f;
    for (int j = ct; j < NK; j += 32 * kAuxCompute)
      if (j > 0) se += expf(gs[j] - zmax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
    if (lane == 0) wred[warp] = se;
    aux_bar_sync();
    float se_neg = 0.f;
#pragma unroll
    for (int w = 0; w < kAuxCompute; ++w) se_neg += wred[w];
    const float z0 = gs[0];
    const float e0 = expf(z0 - zmax);
    aux_bar_sync();  // every thread has read gs[0] and wred
    const float scale = p.inv_tau * inv_p / (e0 + se_neg);
    for (int j = ct; j < NK; j += 32 * kAuxCompute)
      gs[j] = j == 0 ? -se_neg * scale : expf(gs[j] - zmax) * scale;  // dL/ds_j
    if (ct == 0) p.term[i] = (zmax - z0) + log1pf((e0 - 1.0f) + se_neg);  // -log p_0
    aux_bar_sync();
    if (!grads) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qb]);  // the query buffer may take the positive after next
      continue;
    }
    if (warp < n_r) {  // c_h = sum_j g_j cos_jh
      float cc = 0.f;
      for (int j = lane; j < NK; j += 32) cc = fmaf(gs[j], cosv[(size_t)j * 8 + warp], cc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cc += __shfl_xor_sync(0xffffffffu, cc, o);
      if (lane == 0) chead[warp] = cc;
    }

    // ---- pass 2: gradients (the rows again: still in the ring when resident, otherwise reloaded
    //      from L2), one 16-byte unit of the row at a time ----
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    const float nq = hl ? fabsf(qn[h]) : 1.f;
    float* slice = red + (size_t)warp * Sm::kStg;
    for (int c = 0; c < n_ch; ++c) {
      const int ring_it = resident ? it_first + c : it++;
      const int st = ring_it % S;
      if (!resident)  // on failure: left at the next barrier
        failed |= !warp_wait(&full[st], (ring_it / S) & 1, &abort_flag);
      const int j = c * kAuxRows + warp;
      uint4 kw[DR / 32];
      if (j < NK && hl) {
        const uint8_t* base = ring + (size_t)st * Sm::kStageBytes + (size_t)warp * row_bytes + lane * (DR / 32) * 16;
#pragma unroll
        for (int e = 0; e < DR / 32; ++e) kw[e] = *reinterpret_cast<const uint4*>(base + unit_of_slot<DR>(e, lane) * 16);
      }
      // the row is in registers: the stage may refill.  The proxy fence orders these generic-proxy
      // reads before the bulk copy (async proxy) that will overwrite the stage once every warp has
      // arrived, so the last warp to arrive cannot have its loads overtaken by the refill.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      float* dk = nullptr;
      if (j < NK) dk = j == 0 ? (p.dK_pos ? p.dK_pos + (size_t)i * NR : nullptr)
                              : (p.dK_neg ? p.dK_neg + ((size_t)i * p.N + (j - 1)) * NR : nullptr);
      // the row's dK goes to staging row c & 1 of this warp, in the gradient's order, and from
      // there to global memory by one bulk store; the store issued from that row two rows ago
      // must have read it first (lane 0 issued it: its group count is the warp's)
      float* stg = slice + (c & 1) * Sm::kRow;
      if (dk) {
        if (lane == 0) bulk_store_wait_read<1>();
        __syncwarp();
      }
      if (j < NK && hl) {
        const float nks = nkv[(size_t)j * 8 + h], nk = fabsf(nks);
        const float g = gs[j] * inv_nr;
        const float a = g / (nq * nk);  // coefficient of k in dL/dq and of q in dL/dk
        const float b = nks > 0.f ? g * cosv[(size_t)j * 8 + h] / (nk * nk) : 0.f;
#pragma unroll
        for (int e = 0; e < DR / 32; ++e) {
          float kv[8];
          float2 f;
          f = unpack_bf16x2(kw[e].x); kv[0] = f.x; kv[1] = f.y;
          f = unpack_bf16x2(kw[e].y); kv[2] = f.x; kv[3] = f.y;
          f = unpack_bf16x2(kw[e].z); kv[4] = f.x; kv[5] = f.y;
          f = unpack_bf16x2(kw[e].w); kv[6] = f.x; kv[7] = f.y;
#pragma unroll
          for (int t = 0; t < 8; ++t) acc[8 * e + t] = fmaf(a, kv[t], acc[8 * e + t]);
          if (dk) {  // element lane * V + o of the row: this lane's head and quarter
            float* s8 = stg + lane * V + unit_of_slot<DR>(e, lane) * 8;
            *reinterpret_cast<float4*>(s8) =
                make_float4(a * q[8 * e + 0] - b * kv[0], a * q[8 * e + 1] - b * kv[1], a * q[8 * e + 2] - b * kv[2],
                            a * q[8 * e + 3] - b * kv[3]);
            *reinterpret_cast<float4*>(s8 + 4) =
                make_float4(a * q[8 * e + 4] - b * kv[4], a * q[8 * e + 5] - b * kv[5], a * q[8 * e + 6] - b * kv[6],
                            a * q[8 * e + 7] - b * kv[7]);
          }
        }
      }
      if (dk) {
        fence_proxy_async_smem();  // this lane's staging writes before the bulk store reads them
        __syncwarp();
        if (lane == 0) {
          bulk_store(dk, stg, (uint32_t)NR * 4);
          bulk_store_commit();
        }
      }
    }
    // the staging rows are free again (the dq partial reuses them) once the stores have read them
    if (lane == 0) bulk_store_wait_read<0>();
    __syncwarp();
    if (p.dQ != nullptr) {
      // this warp's dq partial in its slice: element lane * V + o of the row at lane * V +
      // (o + lane) % V, so that the lanes' stores of one o fall in distinct banks (a lane's V
      // values would otherwise start in the same bank for every lane)
      if (hl) {
#pragma unroll
        for (int e = 0; e < V; ++e)
          slice[lane * V + ((unit_of_slot<DR>(e / 8, lane) * 8 + e % 8 + lane) & (V - 1))] = acc[e];
      }
      aux_bar_sync();
      for (int e = ct; e < NR; e += 32 * kAuxCompute) {
        const int hh = e / DR;
        const int se = (e & ~(V - 1)) + ((e + e / V) & (V - 1));  // where element e of a partial sits
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kAuxCompute; ++w) v += red[(size_t)w * Sm::kStg + se];
        const float nqs = qn[hh], nqa = fabsf(nqs);
        if (nqs > 0.f) v -= chead[hh] * inv_nr * bf16_bits_to_float(qrow[e]) / (nqa * nqa);
        p.dQ[(size_t)i * NR + e] = v;
      }
    }
    aux_bar_sync();  // every warp is done with the query row
    if (lane == 0) mbar_arrive(&qempty[qb]);  // the query buffer may take the positive after next
  }

  // every gradient row this warp handed to a bulk store is written before the CTA finishes
  if (lane == 0) bulk_store_wait_all();
  __syncwarp();

  // ---- loss: the last CTA sums the terms in positive order ----
  __threadfence();
  if (aux_bar_any(abort_flag != 0)) return;  // a CTA that gave up leaves the loss unsummed (error word set)
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.ticket, 1u);
    last = prev == gridDim.x - 1;
    if (last) *p.ticket = 0u;
  }
  aux_bar_sync();
  if (!last) return;
  __threadfence();
  if (warp == 0) {
    // lane l sums terms l, l + 32, ... in order; the 32 partial sums are added in lane order
    float sum = 0.f;
    for (int e = lane; e < p.P; e += 32) sum += __ldcg(&p.term[e]);
    float tot = 0.f;
    for (int l = 0; l < 32; ++l) tot += __shfl_sync(0xffffffffu, sum, l);
    if (lane == 0) *p.loss = tot / (float)p.P;
  }
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
  const int grid = std::max(1, std::min(P, sm_count()));
  TraceScope ts(kKAuxLoss, s);
  const bool grads = dQ || dK_pos || dK_neg;
  if (d.d_r == 128) {
    p.stages = aux_stages<128>(grads, N + 1);
    const size_t sm = AuxSmem<128>::bytes(N + 1, p.stages);
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(aux_loss_kernel<128>), (int)sm));
    MSA_CUDA_CHECK(launch_pdl(aux_loss_kernel<128>, dim3(grid), dim3(kAuxThreads), sm, s, p));
  } else {
    p.stages = aux_stages<64>(grads, N + 1);
    const size_t sm = AuxSmem<64>::bytes(N + 1, p.stages);
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(aux_loss_kernel<64>), (int)sm));
    MSA_CUDA_CHECK(launch_pdl(aux_loss_kernel<64>, dim3(grid), dim3(kAuxThreads), sm, s, p));
  }
  return MSA_OK;
}

}  // namespace msa

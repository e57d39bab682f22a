// Tiered decode: stages 2 and 3 of several layers in one call, with the
// content memory in host DRAM.
//
// The memory-parallel deployment of the MSA paper keeps the pooled router keys
// K̄^R on the GPU and the content K̄/V̄ in host memory, and loads the selected
// documents asynchronously once routing has chosen them (IRMaD reading,
// "M. Materials & Methods", Memory Parallel and tiered storage item; EverMind
// article 2.3).  Per layer that is a chain route -> gather -> attend whose
// middle link crosses the host bus.  This file enqueues the chains of many
// layers so that the bus transfer of layer l runs on a copy stream while the
// GPU scans layer l + 1's router keys:
//
//   stream       route(0) | route(1) attend(0) | route(2) attend(1) | ... | attend(L-1)
//   copy_stream        gather(0)         gather(1)           gather(2) ...
//
// with an event from each routing (or, when the transfers are short, from the
// attention of the layer before) to its gather and from each gather to its
// attention.  Two staging areas alternate between layers: the gather of layer
// l + 2 waits (through that event) for the attention of layer l, which reads
// the same area.  Host code only; the kernels are those of the single calls.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "internal.h"

namespace msa {

namespace {

struct TieredWs {
  void* route_ws;
  void* attend_ws;
  void* K_stage[2];
  void* V_stage[2];
  int32_t* stage_off[2];
  int32_t* stage_idx[2];
  int32_t* stage_src[2];
};

size_t tiered_workspace(const msa_dims& d, int B, int n_docs, int n_chunks, int k, int t_loc_max, int pos_offset,
                        int capacity, void* ws, TieredWs* out) {
  Carver cv(ws);
  TieredWs w{};
  const size_t r_bytes = route_workspace(d, B, 1, n_docs, n_chunks, k, MSA_AGG_MAX, nullptr, nullptr);
  const size_t a_bytes = attend_workspace(d, B, 1, k, t_loc_max, pos_offset, nullptr, nullptr);
  w.route_ws = cv.take<uint8_t>(r_bytes);
  w.attend_ws = cv.take<uint8_t>(a_bytes);
  const size_t row = (size_t)d.n_kv * d.head_dim;  // bf16 elements of one staged chunk row
  for (int s = 0; s < 2; ++s) {
    w.K_stage[s] = cv.take<uint16_t>((size_t)capacity * row);
    w.V_stage[s] = cv.take<uint16_t>((size_t)capacity * row);
    w.stage_off[s] = cv.take<int32_t>((size_t)B * k + 1);
    w.stage_idx[s] = cv.take<int32_t>((size_t)B * k);
    w.stage_src[s] = cv.take<int32_t>((size_t)B * k);
  }
  if (out) *out = w;
  return cv.size();
}

// three events per (host thread, device): routing done (reused: each record is waited on at
// once) and one per staging area (gather done)
struct TieredEvents {
  cudaEvent_t routed = nullptr;
  cudaEvent_t staged[2] = {nullptr, nullptr};
};
constexpr int kMaxDevices = 64;

msa_status tiered_events(TieredEvents** out) {
  thread_local TieredEvents ev[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  TieredEvents& t = ev[dev];
  if (!t.routed) {
    cudaEvent_t a, b, c;
    MSA_CUDA_CHECK(cudaEventCreateWithFlags(&a, cudaEventDisableTiming));
    MSA_CUDA_CHECK(cudaEventCreateWithFlags(&b, cudaEventDisableTiming));
    MSA_CUDA_CHECK(cudaEventCreateWithFlags(&c, cudaEventDisableTiming));
    t.routed = a;
    t.staged[0] = b;
    t.staged[1] = c;
  }
  *out = &t;
  return MSA_OK;
}

}  // namespace

size_t tiered_workspace_size(const msa_dims& d, int B, int n_docs, int n_chunks, int k, int t_loc_max, int pos_offset,
                             int capacity) {
  return tiered_workspace(d, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity, nullptr, nullptr);
}

msa_status tiered_launch(const msa_dims& d, const msa_layer* layers, const void* const* K_dev, const void* const* V_dev,
                         int n_layers, int B, const int32_t* chunk_off, int n_docs, int n_chunks, int k,
                         const int32_t* loc_len, int t_loc_max, int pos_offset, int capacity, void* ws,
                         cudaStream_t s, cudaStream_t cs) {
  TieredWs w;
  tiered_workspace(d, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity, ws, &w);
  const bool overlap = cs != nullptr && cs != s;
  TieredEvents* ev = nullptr;
  if (overlap) {
    msa_status st = tiered_events(&ev);
    if (st != MSA_OK) return st;
  }
  const int n_stage_docs = B * k;
  // When the bus transfer of a layer is shorter than the routing of the next one (few queries),
  // the gather of layer l is released only after the attention of layer l - 1, so that it runs
  // beside the next routing alone and the attention has the GPU to itself; when the transfer is
  // the longer (many queries: the step is bound by the host link), it starts as soon as its
  // routing is done.  Expected times: the selected documents' K̄/V̄ rows (the average document)
  // over ~50 GB/s against the router keys over ~6.5 TB/s.
  const double gather_bytes = (double)B * k * ((double)n_chunks / n_docs) * 2.0 * d.n_kv * d.head_dim * 2.0;
  const double scan_bytes = (double)n_chunks * d.n_r * d.d_r * 2.0;
  const bool late = gather_bytes / 50e9 < scan_bytes / 6.5e12;
  auto attend = [&](int l) -> msa_status {
    const msa_layer& L = layers[l];
    const int slot = l & 1;
    if (overlap) MSA_CUDA_CHECK(cudaStreamWaitEvent(s, ev->staged[slot], 0));
    // the local keys may be read while the routing of the next layer finishes: that routing writes
    // neither this layer's query, cache nor attention workspace
    return attend_launch(d, L.q, B, 1, w.K_stage[slot], w.V_stage[slot], w.stage_off[slot], n_stage_docs,
                         w.stage_idx[slot], k, L.K_loc, L.V_loc, L.k_new, L.v_new, loc_len, t_loc_max, pos_offset,
                         nullptr, 1, 0.0f, 0, l + 1 < n_layers ? 1 : 0, L.out, w.attend_ws, s);
  };
  for (int l = 0; l < n_layers; ++l) {
    const msa_layer& L = layers[l];
    const int slot = l & 1;
    // the routing's inputs are never written by the work before it inside this call (the
    // previous layer's attention or routing), so from the second layer on it reads them early
    msa_status st = route_launch(d, L.Hq, L.W_QR, B, 1, L.KR_bar, chunk_off, n_docs, n_chunks, k, MSA_AGG_MAX, 0,
                                 L.kr_inv_norm, nullptr, L.topk_idx, L.topk_score, w.route_ws, s, l > 0);
    if (st != MSA_OK) return st;
    if (overlap && late && l > 0) {  // the previous layer's attention before this layer's gather starts
      st = attend(l - 1);
      if (st != MSA_OK) return st;
    }
    cudaStream_t g = s;
    if (overlap) {
      MSA_CUDA_CHECK(cudaEventRecord(ev->routed, s));
      MSA_CUDA_CHECK(cudaStreamWaitEvent(cs, ev->routed, 0));
      g = cs;
    }
    st = gather_kv_launch(d, K_dev[l], V_dev[l], chunk_off, n_docs, L.topk_idx, B, k, w.K_stage[slot],
                          w.V_stage[slot], capacity, w.stage_off[slot], w.stage_idx[slot], w.stage_src[slot], g);
    if (st != MSA_OK) return st;
    if (overlap) MSA_CUDA_CHECK(cudaEventRecord(ev->staged[slot], cs));
    if (!overlap) {  // one stream: each layer's chain in order
      st = attend(l);
      if (st != MSA_OK) return st;
    } else if (!late && l > 0) {
      st = attend(l - 1);
      if (st != MSA_OK) return st;
    }
  }
  if (overlap) return attend(n_layers - 1);
  return MSA_OK;
}

}  // namespace msa

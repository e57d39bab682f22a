// Tiered decode: stages 2 and 3 of several layers in one call, with the
// content memory in host DRAM.
//
// The memory-parallel deployment of the MSA paper keeps the pooled router keys
// K̄^R on the GPU and the content K̄/V̄ in host memory, and loads the selected
// documents asynchronously once routing has chosen them (IRMaD reading,
// "M. Materials & Methods", Memory Parallel and tiered storage item; EverMind
// article 2.3).  Per layer that is a chain route -> gather -> attend whose
// middle link crosses the host bus.  This file enqueues the chains of many
// layers on two streams so that each layer's bus transfer runs while the GPU
// scans the next layer's router keys.  Which work goes where depends on which
// of the two is the longer:
//
// * Short transfers (few queries): the scan is the step's bound, so it runs
//   alone on `stream`, one layer after the other, on all SMs but a few; the
//   rest of each layer's chain follows on the copy stream, beside the next
//   layer's scan, on the SMs the scan leaves free:
//
//     stream       score(0) | score(1) | score(2) | ...
//     copy_stream           select(0) gather(0) attend(0) | select(1) gather(1) attend(1) | ...
//
//   (score = router query and scan, select = the top-k kernels).  The two
//   routing workspaces alternate between layers; the scoring of layer l + 2
//   waits for the selection of layer l, which reads the same workspace.
//
// * Long transfers (many queries): the bus is the bound, so the copy stream
//   does nothing but gather, each layer's as soon as its routing is done, and
//   the attention of layer l runs on `stream` after the routing of l + 1:
//
//     stream       route(0) | route(1) attend(0) | route(2) attend(1) | ... | attend(L-1)
//     copy_stream        gather(0)         gather(1)           gather(2) ...
//
//   Two staging areas alternate between layers: the gather of layer l + 2
//   waits (through that event) for the attention of layer l.
//
// Host code only; the kernels are those of the single calls, with the same
// arguments, so the results are theirs bit for bit.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "internal.h"

namespace msa {

namespace {

struct TieredWs {
  int32_t* chunk_doc;  // [n_chunks] each chunk's document: the scans' epilogues read it
  uint8_t* q_hl;      // [n_layers][q_bytes] each layer's router-query rows (short transfers)
  size_t q_bytes;
  void* route_ws[2];
  void* attend_ws;
  void* K_stage[2];
  void* V_stage[2];
  int32_t* stage_off[2];
  int32_t* stage_idx[2];
  int32_t* stage_src[2];
};

size_t tiered_workspace(const msa_dims& d, int n_layers, int B, int n_docs, int n_chunks, int k, int t_loc_max,
                        int pos_offset, int capacity, void* ws, TieredWs* out) {
  Carver cv(ws);
  TieredWs w{};
  w.chunk_doc = cv.take<int32_t>((size_t)n_chunks);
  w.q_bytes = (route_query_bytes(d, B, 1) + 255) & ~size_t(255);
  w.q_hl = cv.take<uint8_t>((size_t)n_layers * w.q_bytes);
  const size_t r_bytes = route_workspace(d, B, 1, n_docs, n_chunks, k, MSA_AGG_MAX, nullptr, nullptr);
  const size_t a_bytes = attend_workspace(d, B, 1, k, t_loc_max, pos_offset, nullptr, nullptr);
  w.route_ws[0] = cv.take<uint8_t>(r_bytes);
  w.route_ws[1] = cv.take<uint8_t>(r_bytes);
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

// Events per (host thread, device): routing done (reused: each record is waited on at once), one per
// staging area (gather done), one per routing workspace (its selection done), and the copy stream's
// end of work.
struct TieredEvents {
  cudaEvent_t routed = nullptr;
  cudaEvent_t staged[2] = {nullptr, nullptr};
  cudaEvent_t selected[2] = {nullptr, nullptr};
  cudaEvent_t joined = nullptr;
};
constexpr int kMaxDevices = 64;

msa_status tiered_events(TieredEvents** out) {
  thread_local TieredEvents ev[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  TieredEvents& t = ev[dev];
  if (!t.joined) {
    cudaEvent_t* all[6] = {&t.routed, &t.staged[0], &t.staged[1], &t.selected[0], &t.selected[1], &t.joined};
    for (cudaEvent_t* p : all)
      if (!*p) MSA_CUDA_CHECK(cudaEventCreateWithFlags(p, cudaEventDisableTiming));
  }
  *out = &t;
  return MSA_OK;
}

// SMs the scan leaves free, in the short-transfer order, for the copy stream's selection, gather
// and attention of the previous layer
constexpr int kSideSms = 8;

}  // namespace

size_t tiered_workspace_size(const msa_dims& d, int n_layers, int B, int n_docs, int n_chunks, int k, int t_loc_max,
                             int pos_offset, int capacity) {
  return tiered_workspace(d, n_layers, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity, nullptr, nullptr);
}

msa_status tiered_launch(const msa_dims& d, const msa_layer* layers, const void* const* K_dev, const void* const* V_dev,
                         int n_layers, int B, const int32_t* chunk_off, int n_docs, int n_chunks, int k,
                         const int32_t* loc_len, int t_loc_max, int pos_offset, int capacity, void* ws,
                         cudaStream_t s, cudaStream_t cs) {
  TieredWs w;
  tiered_workspace(d, n_layers, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity, ws, &w);
  const bool overlap = cs != nullptr && cs != s;
  TieredEvents* ev = nullptr;
  if (overlap) {
    msa_status st = tiered_events(&ev);
    if (st != MSA_OK) return st;
  }
  const int n_stage_docs = B * k;
  // Which is the longer per layer: the selected documents' K̄/V̄ rows (the average document) over
  // a ~50 GB/s host link, or the router keys over ~6.5 TB/s of HBM.
  const double gather_bytes = (double)B * k * ((double)n_chunks / n_docs) * 2.0 * d.n_kv * d.head_dim * 2.0;
  const double scan_bytes = (double)n_chunks * d.n_r * d.d_r * 2.0;
  const bool short_transfer = gather_bytes / 50e9 < scan_bytes / 6.5e12;
  // the routing's inputs are never written by the work before it inside this call (an earlier
  // layer's kernels), so from the second layer on it reads them early
  auto route = [&](int l, RoutePart part, int slot, cudaStream_t st, int reserve) -> msa_status {
    const msa_layer& L = layers[l];
    // in the short-transfer order the scans follow one another on `stream`: the scan of layer
    // l > 0 writes the other routing workspace than the scan before it, every input it reads was
    // final before that scan started (the router queries and the chunk map run first), and the
    // reuse of its workspace is ordered by the event on the selection two layers back
    return route_launch(d, L.Hq, L.W_QR, B, 1, L.KR_bar, chunk_off, n_docs, n_chunks, k, MSA_AGG_MAX, 0,
                        L.kr_inv_norm, nullptr, L.topk_idx, L.topk_score, w.route_ws[slot], st, l > 0, part,
                        reserve, w.q_hl + (size_t)l * w.q_bytes, w.chunk_doc, part == RoutePart::kScan && l > 0);
  };
  auto gather = [&](int l, cudaStream_t st) -> msa_status {
    const int slot = l & 1;
    return gather_kv_launch(d, K_dev[l], V_dev[l], chunk_off, n_docs, layers[l].topk_idx, B, k, w.K_stage[slot],
                            w.V_stage[slot], capacity, w.stage_off[slot], w.stage_idx[slot], w.stage_src[slot], st);
  };
  // early: the local keys may be read while the kernel before the attention on its stream finishes
  // (that kernel must write neither this layer's query, cache nor the attention workspace)
  auto attend = [&](int l, cudaStream_t st, int early, int max_ctas) -> msa_status {
    const msa_layer& L = layers[l];
    const int slot = l & 1;
    return attend_launch(d, L.q, B, 1, w.K_stage[slot], w.V_stage[slot], w.stage_off[slot], n_stage_docs,
                         w.stage_idx[slot], k, L.K_loc, L.V_loc, L.k_new, L.v_new, loc_len, t_loc_max, pos_offset,
                         nullptr, 1, 0.0f, 0, early, L.out, w.attend_ws, st, nullptr, max_ctas);
  };
  // the layout's chunk -> document map, once for every scan of the call
  msa_status st = chunk_doc_launch(chunk_off, n_docs, n_chunks, w.chunk_doc, s);
  if (st != MSA_OK) return st;
  if (!overlap) {  // one stream: each layer's chain in order
    for (int l = 0; l < n_layers && st == MSA_OK; ++l) {
      st = route(l, RoutePart::kAll, 0, s, 0);
      if (st == MSA_OK) st = gather(l, s);
      if (st == MSA_OK) st = attend(l, s, 1, 0);  // after the gather
    }
    return st;
  }
  if (short_transfer) {
    // every layer's router query first: its inputs are the call's, so the queries of all layers
    // overlap one another, and the scans then follow one another with nothing between them.  The
    // first two also clear the two routing workspaces; later a workspace is cleared on the copy
    // stream once its selection has read it.
    void* clr[2];
    size_t clr_bytes = 0;
    for (int slot = 0; slot < 2; ++slot)
      route_clear_region(d, B, 1, n_docs, n_chunks, k, w.route_ws[slot], &clr[slot], &clr_bytes);
    for (int l = 0; l < n_layers; ++l) {
      uint32_t* c = l < 2 ? static_cast<uint32_t*>(clr[l]) : nullptr;
      st = route_query_launch(d, layers[l].Hq, layers[l].W_QR, B, 1, w.q_hl + (size_t)l * w.q_bytes, c,
                              c ? clr_bytes / 4 : 0, nullptr, 0, s, l > 0);
      if (st != MSA_OK) return st;
    }
    for (int l = 0; l < n_layers; ++l) {
      const int slot = l & 1;
      if (l >= 2) MSA_CUDA_CHECK(cudaStreamWaitEvent(s, ev->selected[slot], 0));
      st = route(l, RoutePart::kScan, slot, s, kSideSms);
      if (st != MSA_OK) return st;
      MSA_CUDA_CHECK(cudaEventRecord(ev->routed, s));
      MSA_CUDA_CHECK(cudaStreamWaitEvent(cs, ev->routed, 0));
      st = route(l, RoutePart::kSelect, slot, cs, 0);
      if (st != MSA_OK) return st;
      if (l + 2 < n_layers) MSA_CUDA_CHECK(cudaMemsetAsync(clr[slot], 0, clr_bytes, cs));
      MSA_CUDA_CHECK(cudaEventRecord(ev->selected[slot], cs));
      st = gather(l, cs);
      // after the gather, beside the next layer's scan: as many CTAs as the scan leaves SMs
      if (st == MSA_OK) st = attend(l, cs, 1, kSideSms);
      if (st != MSA_OK) return st;
    }
    // the copy stream's work joined back into the caller's stream
    MSA_CUDA_CHECK(cudaEventRecord(ev->joined, cs));
    MSA_CUDA_CHECK(cudaStreamWaitEvent(s, ev->joined, 0));
    return MSA_OK;
  }
  for (int l = 0; l < n_layers; ++l) {
    const int slot = l & 1;
    st = route(l, RoutePart::kAll, 0, s, 0);
    if (st != MSA_OK) return st;
    MSA_CUDA_CHECK(cudaEventRecord(ev->routed, s));
    MSA_CUDA_CHECK(cudaStreamWaitEvent(cs, ev->routed, 0));
    st = gather(l, cs);
    if (st != MSA_OK) return st;
    MSA_CUDA_CHECK(cudaEventRecord(ev->staged[slot], cs));
    if (l > 0) {  // the previous layer's attention, once its gather is done
      MSA_CUDA_CHECK(cudaStreamWaitEvent(s, ev->staged[slot ^ 1], 0));
      st = attend(l - 1, s, 1, 0);  // after the routing of layer l
      if (st != MSA_OK) return st;
    }
  }
  MSA_CUDA_CHECK(cudaStreamWaitEvent(s, ev->staged[(n_layers - 1) & 1], 0));
  return attend(n_layers - 1, s, n_layers == 1 ? 1 : 0, 0);  // after the previous attention: not early
}

}  // namespace msa

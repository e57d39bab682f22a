// msa_route_topk_static: routing without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// a host program that embeds this library as a plugin and owns no CUDA
// allocator, code that runs while a stream is being captured into a CUDA graph
// (cudaMalloc is not allowed there), or a latency-critical loop that must not
// pay cudaMalloc's implicit device synchronisation.  For them this entry point
// runs the same routing kernels on a scratch area that the library itself
// holds: a file-scope device array of kStaticScratchBytes, present on every
// GPU that loads the library until the process exits.
//
// Rules of use:
//   * The first call on a device, with that device current, looks up the
//     array's device address (cudaGetSymbolAddress) and caches it; make that
//     first call before any stream capture.
//   * Every call on a device shares the one array.  Calls whose work overlaps
//     on the GPU (different streams without ordering between them, or several
//     host threads) race on it; order them on one stream.
//   * The array keeps the last call's contents; the routing kernels clear what
//     must start at zero (the per-document maxima) on every call.
//   * Problems whose routing workspace would exceed kStaticScratchBytes are
//     rejected with MSA_ERR_WORKSPACE before anything is launched.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"

namespace msa {

// 8 MiB: for example B = 32 queries over 40K documents (MAX aggregation).
constexpr size_t kStaticScratchBytes = 8u << 20;

static __device__ __align__(256) uint8_t g_route_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (looked up once per device).
msa_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MSA_OK;
}
}  // namespace

}  // namespace msa

using namespace msa;

extern "C" msa_status msa_route_topk_static(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B,
                                            int32_t q_tokens, const void* KR_bar, const int32_t* chunk_off, int32_t n_docs,
                                            int32_t n_chunks, int32_t k, msa_doc_agg agg, float* doc_scores,
                                            int32_t* topk_idx, float* topk_score, void* stream) {
  if (!dims || B < 1 || q_tokens < 1 || (int64_t)B * q_tokens > 65535 || n_docs < 1 || n_chunks < 1 || k < 1)
    return msa_route_topk(dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, 0, nullptr,
                          doc_scores, topk_idx,
                          topk_score, nullptr, 0, stream);  // reports the argument error, launches nothing
  const size_t need = msa_route_workspace_size(dims, B, q_tokens, n_docs, n_chunks, k, agg);
  if (need > kStaticScratchBytes)
    return fail(MSA_ERR_WORKSPACE,
                "problem needs %zu bytes of routing scratch; the static area holds %zu (use msa_route_topk "
                "with a caller workspace)",
                need, kStaticScratchBytes);
  void* scratch = nullptr;
  msa_status st = static_scratch(&scratch);
  if (st != MSA_OK) return st;
  return msa_route_topk(dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, 0, nullptr,
                        doc_scores, topk_idx,
                        topk_score, scratch, kStaticScratchBytes, stream);
}

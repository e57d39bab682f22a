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
//     first call before any stream capture.  The cache is keyed by the CUDA
//     context as well as the device: after the device's context is destroyed
//     and created again (cudaDeviceReset), the next call looks the address up
//     afresh, and that call too must come before any capture.
//   * Every call on a device shares the one array.  Calls whose work overlaps
//     on the GPU (different streams without ordering between them, or several
//     host threads) race on it; order them on one stream.
//   * The array keeps the last call's contents; the routing kernels clear what
//     must start at zero (the per-document maxima and the scan's completion
//     ticket) on every call.
//   * The arguments are checked exactly as msa_route_topk checks them (same
//     status for the same arguments); then problems whose routing workspace
//     would exceed kStaticScratchBytes are rejected with MSA_ERR_WORKSPACE
//     before anything is launched.
#include <cuda.h>
#include <cudaTypedefs.h>
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
struct ScratchAddr {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;  // the context the address belongs to
};
ScratchAddr g_scratch[kMaxDevices];

// The unique id of the calling thread's current context, or 0 when there is none yet or the
// driver does not offer the query.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_route_scratch in the current device's context (looked up once per device and
// context).
msa_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> g(g_scratch_mu);
  ScratchAddr& a = g_scratch[dev];
  const unsigned long long ctx = current_context_id();
  if (!a.ptr || ctx == 0 || ctx != a.ctx_id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);  // creates the device's context if needed
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
    a.ptr = p;
    a.ctx_id = current_context_id();
  }
  *out = a.ptr;
  return MSA_OK;
}
}  // namespace

}  // namespace msa

using namespace msa;

extern "C" msa_status msa_route_topk_static(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B,
                                            int32_t q_tokens, const void* KR_bar, const int32_t* chunk_off, int32_t n_docs,
                                            int32_t n_chunks, int32_t k, msa_doc_agg agg, float* doc_scores,
                                            int32_t* topk_idx, float* topk_score, void* stream) {
  msa_status st = validate_route(dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, 0, nullptr,
                                 doc_scores, topk_idx, topk_score);
  if (st != MSA_OK) return st;  // the same status msa_route_topk gives these arguments; nothing launched
  const size_t need = msa_route_workspace_size(dims, B, q_tokens, n_docs, n_chunks, k, agg);
  if (need > kStaticScratchBytes)
    return fail(MSA_ERR_WORKSPACE,
                "problem needs %zu bytes of routing scratch; the static area holds %zu (use msa_route_topk "
                "with a caller workspace)",
                need, kStaticScratchBytes);
  void* scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != MSA_OK) return st;
  return msa_route_topk(dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, 0, nullptr,
                        doc_scores, topk_idx, topk_score, scratch, kStaticScratchBytes, stream);
}

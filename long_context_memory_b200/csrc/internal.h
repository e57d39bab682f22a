// Host-side internals shared by the MSA C-ABI implementation files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/msa.h"

namespace msa {

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
void set_error(const char* fmt, ...);
msa_status fail(msa_status code, const char* fmt, ...);
msa_status cuda_fail(cudaError_t e, const char* what);

#define MSA_CUDA_CHECK(expr)                             \
  do {                                                   \
    cudaError_t e_ = (expr);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #expr);  \
  } while (0)

// Host-side fault injection for the error-path tests: when the environment
// variable MSA_FAULT is "launch", every entry point fails with MSA_ERR_CUDA
// after validation and before its first launch.
bool fault_injected();

// ---------------------------------------------------------------------------
// kernel ids for tracing
// ---------------------------------------------------------------------------
enum KernelId : int {
  kKRouterQuery = 0,
  kKScan,
  kKTopkSlice,
  kKTopkMerge,
  kKRopeTable,
  kKAttnSplit,
  kKAttnCombine,
  kKEncChunkMap,
  kKEncTransposeW,
  kKEncGemmK,
  kKEncPoolH,
  kKEncGemmPooled,
  kKRopeRows,
  kKGatherPlan,
  kKGatherCopy,
  kKChunkOffExtend,
  kKAuxLoss,
  kKKvAppend,
  kKKrNorms,
  kKAttnMerge,
  kKChunkDoc,
  kKernelCount
};

// Brackets one kernel launch with trace events when tracing is enabled.
struct TraceScope {
  TraceScope(int kernel_id, cudaStream_t s);
  ~TraceScope();
  int id;
  cudaStream_t stream;
  int slot;
  unsigned flags;
};

// ---------------------------------------------------------------------------
// workspace carving: 256-byte aligned bump allocation inside the caller's ws
// ---------------------------------------------------------------------------
struct Carver {
  char* base;  // may be null when only measuring
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t size() const { return (off + 255) & ~size_t(255); }
};

// ---------------------------------------------------------------------------
// device properties and the driver's tensor-map encoder
// ---------------------------------------------------------------------------
int sm_count();
int max_smem_optin();
// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes), skipped when already set
cudaError_t set_max_dynamic_smem(const void* kernel, int bytes);
// cudaFuncSetAttribute(kernel, PreferredSharedMemoryCarveout, max shared), once per device and kernel.
// The large kernels (scan, attention, GEMM) need the largest shared-memory carveout; a small kernel
// that prefers another carveout keeps an SM in that configuration while its CTAs run there, and a
// large kernel's CTA cannot start on that SM until they leave.  With every kernel of the library
// preferring the same carveout, small kernels on a second stream (the host-tier gather) share SMs
// with a running scan or attention instead of holding them.
void prefer_shared_carveout(const void* kernel);
msa_status encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* gaddr,
                             const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                             CUtensorMapSwizzle swizzle);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// theta_i / (2 pi) as 64-bit binary fractions, theta_i = base^(-2i/head_dim) (computed in long double)
constexpr int kRopeMaxHalf = 128;  // head_dim / 2 of the largest supported head
void rope_turns(const msa_dims& d, uint64_t* f /* [head_dim / 2] */);

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel on the stream finishes; every kernel launched this
// way calls pdl_wait() before its first global-memory access.
// Launch with programmatic dependent launch (early: the kernel may start while its predecessor
// on the stream runs, and waits for it inside, pdl_enter) or in plain stream order (the kernel
// starts once its predecessor has completed; its pdl_enter then returns at once).  A kernel that
// runs beside other work on a few SMs is launched in plain order: started early, its CTAs would
// sit on SMs, waiting, that the other work needs.
template <typename... KArgs, typename... Args>
cudaError_t launch_ordered(bool early, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           Args&&... args) {
  prefer_shared_carveout(reinterpret_cast<const void*>(kernel));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = early ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  return launch_ordered(true, kernel, grid, block, smem, s, std::forward<Args>(args)...);
}

// the same with thread-block clusters of cluster_x CTAs along x
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               int cluster_x, Args&&... args) {
  prefer_shared_carveout(reinterpret_cast<const void*>(kernel));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// stage implementations (route.cu, attend.cu, encode.cu)
// ---------------------------------------------------------------------------
size_t route_workspace(const msa_dims& d, int B, int M, int n_docs, int n_chunks, int k, msa_doc_agg agg,
                       void* ws, struct RouteWs* out);
msa_status kr_norms_launch(const msa_dims& d, const void* KR_bar, int n_chunks, int kr_layout, float* inv_norm,
                           cudaStream_t s);
// Which kernels of the routing a call enqueues: all of them; the scoring part (router query and
// scan, and the top-k when the scan's last CTA selects it); the scan alone, on router-query rows
// (q_ext) that route_query_launch wrote earlier; or the remaining top-k kernels.  The parts may go
// to different streams: the selection reads only the workspace, chunk_off and the output
// pointers, after the scoring has completed.
enum class RoutePart { kAll, kScore, kScan, kSelect };

// scan_sm_reserve: SMs the scan leaves free (its grid is the SM count minus this), for work that
// runs beside it on another stream.  after_scan (with kScan): the kernel before this scan on the
// stream is another routing's scan, which writes nothing this routing reads or writes, and every
// input of this routing was final when that scan started: the scan then does not wait for it.
msa_status route_launch(const msa_dims& d, const void* Hq, const void* W_QR, int B, int M, const void* KR_bar,
                        const int32_t* chunk_off, int n_docs, int n_chunks, int k, msa_doc_agg agg, int kr_layout,
                        const float* kr_inv_norm, float* doc_scores, int32_t* topk_idx, float* topk_score, void* ws,
                        cudaStream_t s, bool early_inputs = false, RoutePart part = RoutePart::kAll,
                        int scan_sm_reserve = 0, const void* q_ext = nullptr, const int32_t* chunk_doc = nullptr,
                        bool after_scan = false);

// Each chunk's document id (-1 outside the documents) from chunk_off: the scan's epilogue then
// reads a row's document instead of searching chunk_off for it (chunk_doc argument of
// route_launch).  A property of the layout, computed once for many scans over it.
msa_status chunk_doc_launch(const int32_t* chunk_off, int n_docs, int n_chunks, int32_t* chunk_doc, cudaStream_t s);

// The router query alone: Q^R rows of B x M query tokens into q_hl (route_query_bytes), in the
// layout the scan reads; clears n_clear words at `clear` and n_tickets tickets (either may be
// null) after its wait on the predecessor.
size_t route_query_bytes(const msa_dims& d, int B, int M);
msa_status route_query_launch(const msa_dims& d, const void* Hq, const void* W_QR, int B, int M, void* q_hl,
                              uint32_t* clear, size_t n_clear, uint32_t* tickets, int n_tickets, cudaStream_t s,
                              bool early_inputs);
// The words a routing workspace (MAX aggregation) needs zeroed before its scan: the tickets and
// the document keys, one contiguous region.
void route_clear_region(const msa_dims& d, int B, int M, int n_docs, int n_chunks, int k, void* ws, void** ptr,
                        size_t* bytes);

msa_status validate_route(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B, int32_t q_tokens,
                          const void* KR_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, int32_t k,
                          msa_doc_agg agg, int32_t kr_layout, const float* kr_inv_norm, const float* doc_scores,
                          const int32_t* topk_idx, const float* topk_score);

msa_status topk_merge_launch(const float* cand_score, const int32_t* cand_idx, int B, int n_cand, int k,
                             int32_t* topk_idx, float* topk_score, cudaStream_t s);

size_t attend_workspace(const msa_dims& d, int B, int M, int k, int t_loc_max, int pos_offset, void* ws,
                        struct AttendWs* out);
// One rank's share of a memory-parallel attention: the selected documents it holds (global ids,
// the others skipped), the local keys only where local_keys is set, and the share's normalised
// fp32 output with its base-2 log-sum-exp instead of the bf16 result.
struct AttendShare {
  int doc_base;    // global id of the shard's first document
  int local_keys;  // 1: this share also attends over the local keys
  float* o;        // [B * M * n_q, head_dim] fp32 out
  float* lse2;     // [B * M * n_q] fp32 out
};
msa_status attend_launch(const msa_dims& d, const void* q, int B, int M, const void* K_bar, const void* V_bar,
                         const int32_t* chunk_off, int n_docs, const int32_t* topk_idx, int k,
                         const void* K_loc, const void* V_loc, const void* k_new, const void* v_new,
                         const int32_t* loc_len, int t_loc_max,
                         int pos_offset, const void* rope_cache, int k_loc_rotated, float scale, int phase,
                         int early, void* out, void* ws, cudaStream_t s, const AttendShare* share = nullptr,
                         int max_ctas = 0);
msa_status attend_merge_launch(const float* o_parts, const float* lse2_parts, int R, int n_rows, int D, void* out,
                               cudaStream_t s);
msa_status gather_kv_launch(const msa_dims& d, const void* K_host, const void* V_host, const int32_t* chunk_off,
                            int n_docs, const int32_t* topk_idx, int B, int k, void* K_stage, void* V_stage,
                            int capacity_chunks, int32_t* stage_off, int32_t* stage_idx, int32_t* stage_src,
                            cudaStream_t s);
size_t tiered_workspace_size(const msa_dims& d, int n_layers, int B, int n_docs, int n_chunks, int k, int t_loc_max,
                             int pos_offset, int capacity);
msa_status tiered_launch(const msa_dims& d, const msa_layer* layers, const void* const* K_dev, const void* const* V_dev,
                         int n_layers, int B, const int32_t* chunk_off, int n_docs, int n_chunks, int k,
                         const int32_t* loc_len, int t_loc_max, int pos_offset, int capacity, void* ws,
                         cudaStream_t s, cudaStream_t cs);
msa_status rope_rows_launch(const msa_dims& d, void* x, int rows, int heads, const int32_t* pos, cudaStream_t s);
msa_status rope_cache_build(const msa_dims& d, int t_loc_max, int pos_offset, float2* tab, cudaStream_t s);

msa_status kv_append_launch(const msa_dims& d, const void* k_new, const void* v_new, void* K_loc, void* V_loc, int B,
                            int t_loc_max, const int32_t* slots, int pos_offset, cudaStream_t s);
struct AuxWs {
  float* term;        // [P] per-positive loss terms
  uint32_t* ticket;   // CTAs finished
};
size_t aux_workspace(const msa_dims& d, int P, int N, void* ws, AuxWs* out);
msa_status aux_loss_launch(const msa_dims& d, const void* QR, const void* K_pos, const void* K_neg, int P, int N,
                           float tau, float* loss, float* dQ, float* dK_pos, float* dK_neg, void* ws,
                           cudaStream_t s);
msa_status chunk_off_extend_launch(int32_t* chunk_off, int n_docs_old, int n_chunks_old, const int32_t* chunk_off_new,
                                   int n_docs_new, cudaStream_t s);
size_t encode_workspace(const msa_dims& d, int64_t T, int n_docs, int n_chunks, void* ws,
                        struct EncodeWs* out);
msa_status encode_launch(const msa_dims& d, const void* H, int64_t T, const int64_t* doc_off, int n_docs,
                         const int32_t* chunk_off, int n_chunks, const void* W_K, const void* W_V,
                         const void* W_KR, void* K_bar, void* V_bar, void* KR_bar, int kr_layout, void* ws,
                         cudaStream_t s);

}  // namespace msa

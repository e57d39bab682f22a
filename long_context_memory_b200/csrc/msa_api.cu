// C ABI of the MSA hot path: argument validation, workspace sizing, tracing,
// error reporting.  Every entry point validates on the host before it launches
// anything and never allocates device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace msa {

__device__ uint32_t g_dev_error = 0;

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local char t_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
}

msa_status fail(msa_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return code;
}

msa_status cuda_fail(cudaError_t e, const char* what) {
  set_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
  return MSA_ERR_CUDA;
}

bool fault_injected() {
  const char* f = std::getenv("MSA_FAULT");
  return f && std::strcmp(f, "launch") == 0;
}

void rope_turns(const msa_dims& d, uint64_t* f) {
  // the last (head_dim, base) of this host thread is kept: decode loops ask every step
  thread_local int c_dim = -1;
  thread_local float c_base = 0.f;
  thread_local uint64_t c_f[kRopeMaxHalf];
  const int half = d.head_dim / 2;
  if (c_dim != d.head_dim || c_base != d.rope_base || half > kRopeMaxHalf) {
    const long double two_pi = 6.283185307179586476925286766559005768L;
    const long double lb = logl((long double)d.rope_base);
    for (int i = 0; i < half && i < kRopeMaxHalf; ++i) {
      const long double theta = expl(-2.0L * (long double)i / (long double)d.head_dim * lb);
      const long double turns = theta / two_pi;  // in (0, 1)
      c_f[i] = (uint64_t)ldexpl(turns, 64);
    }
    c_dim = d.head_dim;
    c_base = d.rope_base;
  }
  for (int i = 0; i < half; ++i) f[i] = c_f[i];
}

// ---------------------------------------------------------------------------
// device properties
// ---------------------------------------------------------------------------
namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];  // 0: not queried yet
}  // namespace

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < kMaxDevices) {
    const int c = g_sm_count[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 148;
  if (dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel, size): a decode loop
// calls the same kernels every step
cudaError_t set_max_dynamic_smem(const void* kernel, int bytes) {
  struct Entry {
    int dev;
    const void* fn;
    int bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Entry& e : done)
      if (e.dev == dev && e.fn == kernel && e.bytes >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lk(mu);
    done.push_back({dev, kernel, bytes});
  }
  return e;
}

void prefer_shared_carveout(const void* kernel) {
  struct Entry {
    int dev;
    const void* fn;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    for (const Entry& e : done)
      if (e.dev == dev && e.fn == kernel) return;
  }
  // a hint: a device that cannot honour it keeps its default (the launch still succeeds)
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
      cudaSuccess)
    cudaGetLastError();
  std::lock_guard<std::mutex> lk(mu);
  done.push_back({dev, kernel});
}

int max_smem_optin() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return n;
}

// ---------------------------------------------------------------------------
// tensor maps through the driver entry point (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

msa_status encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, void* gaddr,
                             const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                             CUtensorMapSwizzle swizzle) {
  // the maps of the last calls of this host thread are kept (a decode loop encodes the same
  // few maps every step); the key is every argument
  struct Key {
    int dtype, rank, swizzle;
    void* gaddr;
    uint64_t dims[5], strides[4];
    uint32_t box[5];
    bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
  };
  struct Slot {
    Key key;
    CUtensorMap map;
    bool used;
  };
  constexpr int kSlots = 128;  // a multi-layer call encodes one key map per layer
  thread_local Slot cache[kSlots] = {};
  thread_local int next = 0;
  Key key;
  std::memset(&key, 0, sizeof(key));
  key.dtype = (int)dtype;
  key.rank = rank;
  key.swizzle = (int)swizzle;
  key.gaddr = gaddr;
  for (int i = 0; i < rank && i < 5; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides_bytes[i];
  }
  for (int i = 0; i < kSlots; ++i)
    if (cache[i].used && cache[i].key == key) {
      *map = cache[i].map;
      return MSA_OK;
    }
  auto fn = get_encoder();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  uint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dtype, rank, gaddr, dims, strides_bytes, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  Slot& sl = cache[next];
  next = (next + 1) % kSlots;
  sl.key = key;
  sl.map = *map;
  sl.used = true;
  return MSA_OK;
}

// ---------------------------------------------------------------------------
// tracing
// ---------------------------------------------------------------------------
namespace {
const char* kKernelNames[kKernelCount] = {
    "router_query", "scan", "topk_slice", "topk_merge", "rope_table", "attn_split", "attn_combine",
    "enc_chunk_map", "enc_transpose_w", "enc_gemm_k", "enc_pool_h", "enc_gemm_pooled", "rope_rows", "gather_plan", "gather_copy",
    "chunk_off_extend", "aux_loss", "kv_append", "kr_norms", "attn_merge", "chunk_doc"};

struct TraceState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;  // reusable events
  size_t next = 0;
  struct Rec {
    int id;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  double total_ms[kKernelCount] = {};
  int64_t launches[kKernelCount] = {};
};
TraceState& trace() {
  static TraceState t;
  return t;
}

cudaEvent_t take_event(TraceState& t) {
  if (t.next == t.pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    t.pool.push_back(e);
  }
  return t.pool[t.next++];
}

void flush_trace(TraceState& t) {
  for (auto& r : t.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      t.total_ms[r.id] += ms;
      t.launches[r.id] += 1;
    }
  }
  t.recs.clear();
  t.next = 0;
}
}  // namespace

TraceScope::TraceScope(int kernel_id, cudaStream_t s) : id(kernel_id), stream(s), slot(-1), flags(0) {
  TraceState& t = trace();
  std::lock_guard<std::mutex> g(t.mu);
  if (!t.on) return;
  if (t.pool.size() > 4096 && t.next + 2 > t.pool.size()) flush_trace(t);
  cudaEvent_t a = take_event(t), b = take_event(t);
  if (!a || !b) return;
  // inside stream capture an event becomes a timing node only when recorded as external
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  flags = (cs == cudaStreamCaptureStatusActive) ? cudaEventRecordExternal : cudaEventRecordDefault;
  cudaEventRecordWithFlags(a, s, flags);
  t.recs.push_back({kernel_id, a, b});
  slot = (int)t.recs.size() - 1;
}

TraceScope::~TraceScope() {
  if (slot < 0) return;
  TraceState& t = trace();
  std::lock_guard<std::mutex> g(t.mu);
  if (slot < (int)t.recs.size()) cudaEventRecordWithFlags(t.recs[slot].b, stream, flags);
}

// ---------------------------------------------------------------------------
// self-test of the bounded waits: four warps wait on mbarriers that nothing arrives on
// ---------------------------------------------------------------------------
namespace {
__global__ void __launch_bounds__(128) wait_selftest_kernel(uint64_t limit_ns, int n_waits,
                                                            unsigned long long* elapsed_ns) {
  __shared__ uint64_t bars[4];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);  // no thread ever arrives
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t t0 = globaltimer_ns();
  if (lane == 0)
    for (int i = 0; i < n_waits; ++i) mbar_wait(&bars[warp], 0, &abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0) *elapsed_ns = globaltimer_ns() - t0;
}
}  // namespace

}  // namespace msa

using namespace msa;

// ===========================================================================
// validation helpers
// ===========================================================================
static msa_status check_dims(const msa_dims* d, bool need_kv, bool need_router) {
  if (!d) return fail(MSA_ERR_INVALID_ARG, "dims is NULL");
  if (d->chunk != 64) return fail(MSA_ERR_UNSUPPORTED, "chunk must be 64 (got %d)", d->chunk);
  if (need_router) {
    if (d->n_r < 1 || d->n_r > 8) return fail(MSA_ERR_UNSUPPORTED, "n_r must be in [1, 8] (got %d)", d->n_r);
    if (d->d_r != 64 && d->d_r != 128) return fail(MSA_ERR_UNSUPPORTED, "d_r must be 64 or 128 (got %d)", d->d_r);
  }
  if (need_kv) {
    if (d->head_dim != 64 && d->head_dim != 128)
      return fail(MSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", d->head_dim);
    if (d->n_kv < 1 || d->n_q < 1 || d->n_q % d->n_kv != 0)
      return fail(MSA_ERR_INVALID_ARG, "n_q (%d) must be a positive multiple of n_kv (%d)", d->n_q, d->n_kv);
    if (d->n_q / d->n_kv > 16) return fail(MSA_ERR_UNSUPPORTED, "n_q / n_kv must be <= 16");
    if (d->n_kv > 8) return fail(MSA_ERR_UNSUPPORTED, "n_kv must be <= 8 (got %d)", d->n_kv);
    if (!(d->rope_base > 1.0f) || !std::isfinite(d->rope_base))
      return fail(MSA_ERR_INVALID_ARG, "rope_base must be finite and > 1");
  }
  return MSA_OK;
}

#define CHECK_PTR(p)                                                                           \
  do {                                                                                         \
    if (!(p)) return fail(MSA_ERR_INVALID_ARG, "%s is NULL", #p);                              \
    if (!aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);      \
  } while (0)

#define CHECK_OPT_PTR(p)                                                                       \
  do {                                                                                         \
    if ((p) && !aligned16(p)) return fail(MSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
  } while (0)

// ===========================================================================
// entry points
// ===========================================================================
extern "C" {

const char* msa_last_error(void) { return t_err; }

int32_t msa_version(void) { return 100; }

msa_status msa_check_device_errors(uint32_t* bits_out) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  uint32_t bits = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&bits, g_dev_error, sizeof(bits));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  if (bits_out) *bits_out = bits;
  if (bits & kDevErrWaitTimeout) return fail(MSA_ERR_TIMEOUT, "a bounded device wait gave up (bits 0x%x)", bits);
  if (bits) return fail(MSA_ERR_INVALID_ARG, "device reported an out-of-range index (bits 0x%x)", bits);
  return MSA_OK;
}

msa_status msa_selftest_wait_timeout(int32_t limit_us, int32_t n_waits, uint64_t* elapsed_ns, void* stream) {
  if (limit_us < 1 || limit_us > 100000) return fail(MSA_ERR_INVALID_ARG, "limit_us must be in [1, 100000]");
  if (n_waits < 1 || n_waits > 1000) return fail(MSA_ERR_INVALID_ARG, "n_waits must be in [1, 1000]");
  CHECK_PTR(elapsed_ns);
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  wait_selftest_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull, n_waits,
                                                                         reinterpret_cast<unsigned long long*>(elapsed_ns));
  MSA_CUDA_CHECK(cudaGetLastError());
  return MSA_OK;
}

msa_status msa_chunk_offsets(const int64_t* doc_off_host, int32_t n_docs, int32_t chunk, int32_t* chunk_off_host,
                             int32_t* n_chunks_out) {
  if (!doc_off_host || !chunk_off_host) return fail(MSA_ERR_INVALID_ARG, "NULL offset array");
  if (n_docs < 1) return fail(MSA_ERR_INVALID_ARG, "n_docs must be >= 1 (got %d)", n_docs);
  if (chunk < 1) return fail(MSA_ERR_INVALID_ARG, "chunk must be >= 1 (got %d)", chunk);
  if (doc_off_host[0] != 0) return fail(MSA_ERR_INVALID_ARG, "doc_off[0] must be 0");
  int64_t c = 0;
  chunk_off_host[0] = 0;
  for (int32_t i = 0; i < n_docs; ++i) {
    const int64_t len = doc_off_host[i + 1] - doc_off_host[i];
    if (len < 1) return fail(MSA_ERR_INVALID_ARG, "document %d has %lld tokens (must be >= 1)", i, (long long)len);
    c += (len + chunk - 1) / chunk;
    if (c > INT32_MAX) return fail(MSA_ERR_INVALID_ARG, "more than 2^31-1 chunks");
    chunk_off_host[i + 1] = (int32_t)c;
  }
  if (n_chunks_out) *n_chunks_out = (int32_t)c;
  return MSA_OK;
}

// ------------------------------ routing ------------------------------
size_t msa_route_workspace_size(const msa_dims* dims, int32_t B, int32_t q_tokens, int32_t n_docs, int32_t n_chunks,
                                int32_t k, msa_doc_agg agg) {
  if (!dims || B < 1 || q_tokens < 1 || (int64_t)B * q_tokens > 65535 || n_docs < 1 || n_chunks < 1 || k < 1) return 0;
  return route_workspace(*dims, B, q_tokens, n_docs, n_chunks, k, agg, nullptr, nullptr);
}

}  // extern "C"

namespace msa {
// Every argument check of msa_route_topk except the workspace's (shared with the static-scratch
// entry point, which must report the same errors for the same arguments).
msa_status validate_route(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B, int32_t q_tokens,
                          const void* KR_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, int32_t k,
                          msa_doc_agg agg, int32_t kr_layout, const float* kr_inv_norm, const float* doc_scores,
                          const int32_t* topk_idx, const float* topk_score) {
  msa_status st = check_dims(dims, false, true);
  if (st != MSA_OK) return st;
  if (W_QR && (dims->hidden < 64 || dims->hidden % 64 != 0 || dims->hidden > 8192))
    return fail(MSA_ERR_UNSUPPORTED, "hidden must be a multiple of 64 in [64, 8192] (got %d)", dims->hidden);
  if (B < 1) return fail(MSA_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  if (q_tokens < 1 || (int64_t)B * q_tokens > 65535)
    return fail(MSA_ERR_INVALID_ARG, "q_tokens must be >= 1 with B * q_tokens <= 65535 (got %d, B %d)", q_tokens, B);
  if (n_docs < 1 || n_chunks < n_docs)
    return fail(MSA_ERR_INVALID_ARG, "need 1 <= n_docs <= n_chunks (got %d, %d)", n_docs, n_chunks);
  if (k < 1 || k > n_docs || k > 256)
    return fail(MSA_ERR_INVALID_ARG, "k must be in [1, min(n_docs, 256)] (got %d, n_docs %d)", k, n_docs);
  if (agg != MSA_AGG_MAX && agg != MSA_AGG_MEAN) return fail(MSA_ERR_INVALID_ARG, "unknown aggregation %d", (int)agg);
  kr_layout &= ~MSA_ROUTE_EARLY_INPUTS;
  if (kr_layout != 0 && kr_layout != 1)
    return fail(MSA_ERR_INVALID_ARG, "kr_layout must be 0 or 1, optionally | MSA_ROUTE_EARLY_INPUTS (got %d)", kr_layout);
  const int n_slices = (n_docs + 4095) / 4096;
  if ((size_t)n_slices * k > 24576) return fail(MSA_ERR_UNSUPPORTED, "n_docs * k too large for the top-k merge");
  CHECK_PTR(Hq);
  CHECK_OPT_PTR(W_QR);
  CHECK_PTR(KR_bar);
  CHECK_PTR(chunk_off);
  CHECK_OPT_PTR(doc_scores);
  CHECK_PTR(topk_idx);
  CHECK_PTR(topk_score);
  CHECK_OPT_PTR(kr_inv_norm);
  return MSA_OK;
}
}  // namespace msa

extern "C" {

msa_status msa_route_topk(const msa_dims* dims, const void* Hq, const void* W_QR, int32_t B, int32_t q_tokens,
                          const void* KR_bar,
                          const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, int32_t k, msa_doc_agg agg,
                          int32_t kr_layout, const float* kr_inv_norm, float* doc_scores, int32_t* topk_idx,
                          float* topk_score, void* ws, size_t ws_bytes,
                          void* stream) {
  msa_status st = validate_route(dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, kr_layout,
                                 kr_inv_norm, doc_scores, topk_idx, topk_score);
  if (st != MSA_OK) return st;
  const bool early_inputs = (kr_layout & MSA_ROUTE_EARLY_INPUTS) != 0;
  kr_layout &= ~MSA_ROUTE_EARLY_INPUTS;
  const size_t need = route_workspace(*dims, B, q_tokens, n_docs, n_chunks, k, agg, nullptr, nullptr);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return route_launch(*dims, Hq, W_QR, B, q_tokens, KR_bar, chunk_off, n_docs, n_chunks, k, agg, kr_layout, kr_inv_norm,
                      doc_scores, topk_idx, topk_score, ws, static_cast<cudaStream_t>(stream), early_inputs);
}

msa_status msa_router_key_norms(const msa_dims* dims, const void* KR_bar, int32_t n_chunks, int32_t kr_layout,
                                float* kr_inv_norm, void* stream) {
  msa_status st = check_dims(dims, false, true);
  if (st != MSA_OK) return st;
  if (n_chunks < 1) return fail(MSA_ERR_INVALID_ARG, "n_chunks must be >= 1 (got %d)", n_chunks);
  if (kr_layout != 0 && kr_layout != 1) return fail(MSA_ERR_INVALID_ARG, "kr_layout must be 0 or 1 (got %d)", kr_layout);
  CHECK_PTR(KR_bar);
  CHECK_PTR(kr_inv_norm);
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return kr_norms_launch(*dims, KR_bar, n_chunks, kr_layout, kr_inv_norm, static_cast<cudaStream_t>(stream));
}

msa_status msa_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t B, int32_t n_cand, int32_t k,
                          int32_t* topk_idx, float* topk_score, void* stream) {
  if (B < 1) return fail(MSA_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  if (n_cand < 1 || n_cand > 24576) return fail(MSA_ERR_INVALID_ARG, "n_cand must be in [1, 24576] (got %d)", n_cand);
  if (k < 1 || k > n_cand || k > 256)
    return fail(MSA_ERR_INVALID_ARG, "k must be in [1, min(n_cand, 256)] (got %d)", k);
  CHECK_PTR(cand_score);
  CHECK_PTR(cand_idx);
  CHECK_PTR(topk_idx);
  CHECK_PTR(topk_score);
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return topk_merge_launch(cand_score, cand_idx, B, n_cand, k, topk_idx, topk_score, static_cast<cudaStream_t>(stream));
}

// ------------------------------ attention ------------------------------
size_t msa_attend_workspace_size(const msa_dims* dims, int32_t B, int32_t q_tokens, int32_t k, int32_t t_loc_max,
                                 int32_t pos_offset) {
  if (!dims || B < 1 || q_tokens < 1 || (int64_t)B * q_tokens > 65535 || k < 1 || t_loc_max < 0) return 0;
  if (dims->n_kv < 1 || dims->n_q < dims->n_kv) return 0;
  return attend_workspace(*dims, B, q_tokens, k, t_loc_max, pos_offset, nullptr, nullptr);
}

msa_status msa_sparse_attend(const msa_dims* dims, const void* q, int32_t B, int32_t q_tokens, const void* K_bar,
                             const void* V_bar,
                             const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, const int32_t* topk_idx,
                             int32_t k, void* K_loc, void* V_loc, const void* k_new, const void* v_new,
                             const int32_t* loc_len, int32_t t_loc_max, int32_t pos_offset, const void* rope_cache,
                             int32_t k_loc_rotated, float softmax_scale, int32_t phase, void* out, void* ws,
                             size_t ws_bytes, void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (B < 1) return fail(MSA_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  if (q_tokens < 1 || (int64_t)B * q_tokens > 65535)
    return fail(MSA_ERR_INVALID_ARG, "q_tokens must be >= 1 with B * q_tokens <= 65535 (got %d, B %d)", q_tokens, B);
  if (n_docs < 1 || n_chunks < n_docs)
    return fail(MSA_ERR_INVALID_ARG, "need 1 <= n_docs <= n_chunks (got %d, %d)", n_docs, n_chunks);
  if (k < 1 || k > n_docs || k > 256)
    return fail(MSA_ERR_INVALID_ARG, "k must be in [1, min(n_docs, 256)] (got %d)", k);
  if (t_loc_max < 0) return fail(MSA_ERR_INVALID_ARG, "t_loc_max must be >= 0");
  if (pos_offset < 0 || (int64_t)pos_offset + t_loc_max > (1 << 24))
    return fail(MSA_ERR_INVALID_ARG, "positions must lie in [0, 2^24)");
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(MSA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  const int early = (phase & MSA_ATTEND_EARLY_LOCAL) != 0;
  phase &= ~MSA_ATTEND_EARLY_LOCAL;
  if (phase < 0 || phase > 2)
    return fail(MSA_ERR_INVALID_ARG, "phase must be 0, 1 or 2, optionally | MSA_ATTEND_EARLY_LOCAL (got %d)", phase);
  CHECK_PTR(q);
  if (phase != 1) {  // the selected chunks
    CHECK_PTR(K_bar);
    CHECK_PTR(V_bar);
    CHECK_PTR(chunk_off);
    CHECK_PTR(topk_idx);
    CHECK_PTR(out);
  }
  if (phase != 2 && t_loc_max > 0) {  // the local keys
    CHECK_PTR(K_loc);
    CHECK_PTR(V_loc);
  }
  CHECK_PTR(loc_len);
  CHECK_OPT_PTR(rope_cache);
  CHECK_OPT_PTR(k_new);
  CHECK_OPT_PTR(v_new);
  if ((k_new == nullptr) != (v_new == nullptr)) return fail(MSA_ERR_INVALID_ARG, "k_new and v_new go together");
  if (k_new && (q_tokens != 1 || phase == 2 || t_loc_max < 1))
    return fail(MSA_ERR_INVALID_ARG, "the fused append needs q_tokens 1, a local cache and phase 0 or 1");
  const size_t need = attend_workspace(*dims, B, q_tokens, k, t_loc_max, pos_offset, nullptr, nullptr);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return attend_launch(*dims, q, B, q_tokens, K_bar, V_bar, chunk_off, n_docs, topk_idx, k, K_loc, V_loc, k_new,
                       v_new, loc_len, t_loc_max,
                       pos_offset, rope_cache, k_loc_rotated, softmax_scale, phase, early, out, ws,
                       static_cast<cudaStream_t>(stream));
}

msa_status msa_gather_kv(const msa_dims* dims, const void* K_bar_host, const void* V_bar_host, int32_t n_chunks,
                         const int32_t* chunk_off, int32_t n_docs, const int32_t* topk_idx, int32_t B, int32_t k,
                         void* K_stage, void* V_stage, int32_t capacity_chunks, int32_t* stage_chunk_off,
                         int32_t* stage_topk_idx, void* ws, size_t ws_bytes, void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (B < 1 || k < 1 || k > n_docs || n_docs < 1 || n_chunks < n_docs)
    return fail(MSA_ERR_INVALID_ARG, "bad sizes (B %d, k %d, n_docs %d, n_chunks %d)", B, k, n_docs, n_chunks);
  if (capacity_chunks < 1) return fail(MSA_ERR_INVALID_ARG, "capacity_chunks must be >= 1");
  CHECK_PTR(K_bar_host);
  CHECK_PTR(V_bar_host);
  CHECK_PTR(chunk_off);
  CHECK_PTR(topk_idx);
  CHECK_PTR(K_stage);
  CHECK_PTR(V_stage);
  CHECK_PTR(stage_chunk_off);
  CHECK_PTR(stage_topk_idx);
  const size_t need = (size_t)B * k * sizeof(int32_t);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  // the pooled memory must be pinned host memory that the device can address
  const void* dev_ptr[2] = {nullptr, nullptr};
  const void* host_ptr[2] = {K_bar_host, V_bar_host};
  for (int i = 0; i < 2; ++i) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, host_ptr[i]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
    if (a.type != cudaMemoryTypeHost || !a.devicePointer)
      return fail(MSA_ERR_INVALID_ARG, "%s must be pinned (page-locked, device-mapped) host memory",
                  i ? "V_bar_host" : "K_bar_host");
    dev_ptr[i] = a.devicePointer;
  }
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return gather_kv_launch(*dims, dev_ptr[0], dev_ptr[1], chunk_off, n_docs, topk_idx, B, k, K_stage, V_stage,
                          capacity_chunks, stage_chunk_off, stage_topk_idx, static_cast<int32_t*>(ws),
                          static_cast<cudaStream_t>(stream));
}

msa_status msa_sparse_attend_share(const msa_dims* dims, const void* q, int32_t B, int32_t q_tokens, const void* K_bar,
                                   const void* V_bar, const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks,
                                   int32_t doc_base, const int32_t* topk_idx, int32_t k, int32_t local_keys,
                                   const void* K_loc, const void* V_loc, const int32_t* loc_len, int32_t t_loc_max,
                                   int32_t pos_offset, const void* rope_cache, int32_t k_loc_rotated,
                                   float softmax_scale, float* o_share, float* lse2_share, void* ws, size_t ws_bytes,
                                   void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (B < 1) return fail(MSA_ERR_INVALID_ARG, "B must be >= 1 (got %d)", B);
  if (q_tokens < 1 || (int64_t)B * q_tokens > 65535)
    return fail(MSA_ERR_INVALID_ARG, "q_tokens must be >= 1 with B * q_tokens <= 65535 (got %d, B %d)", q_tokens, B);
  if (n_docs < 1 || n_chunks < n_docs)
    return fail(MSA_ERR_INVALID_ARG, "need 1 <= n_docs <= n_chunks (got %d, %d)", n_docs, n_chunks);
  if (doc_base < 0) return fail(MSA_ERR_INVALID_ARG, "doc_base must be >= 0 (got %d)", doc_base);
  if (k < 1 || k > 256) return fail(MSA_ERR_INVALID_ARG, "k must be in [1, 256] (got %d)", k);
  if (local_keys != 0 && local_keys != 1) return fail(MSA_ERR_INVALID_ARG, "local_keys must be 0 or 1");
  if (t_loc_max < 0) return fail(MSA_ERR_INVALID_ARG, "t_loc_max must be >= 0");
  if (pos_offset < 0 || (int64_t)pos_offset + t_loc_max > (1 << 24))
    return fail(MSA_ERR_INVALID_ARG, "positions must lie in [0, 2^24)");
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(MSA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  CHECK_PTR(q);
  CHECK_PTR(K_bar);
  CHECK_PTR(V_bar);
  CHECK_PTR(chunk_off);
  CHECK_PTR(topk_idx);
  CHECK_PTR(loc_len);
  CHECK_PTR(o_share);
  CHECK_PTR(lse2_share);
  if (local_keys && t_loc_max > 0) {
    CHECK_PTR(K_loc);
    CHECK_PTR(V_loc);
  }
  CHECK_OPT_PTR(rope_cache);
  const size_t need = attend_workspace(*dims, B, q_tokens, k, t_loc_max, pos_offset, nullptr, nullptr);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  AttendShare share{doc_base, local_keys, o_share, lse2_share};
  return attend_launch(*dims, q, B, q_tokens, K_bar, V_bar, chunk_off, n_docs, topk_idx, k, K_loc, V_loc, nullptr,
                       nullptr, loc_len, t_loc_max, pos_offset, rope_cache, k_loc_rotated, softmax_scale, 0, 0, nullptr,
                       ws, static_cast<cudaStream_t>(stream), &share);
}

msa_status msa_attend_merge(const float* o_shares, const float* lse2_shares, int32_t R, int32_t rows,
                            int32_t head_dim, void* out, void* stream) {
  if (R < 1 || R > 4096) return fail(MSA_ERR_INVALID_ARG, "R must be in [1, 4096] (got %d)", R);
  if (rows < 1) return fail(MSA_ERR_INVALID_ARG, "rows must be >= 1 (got %d)", rows);
  if (head_dim != 64 && head_dim != 128)
    return fail(MSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  CHECK_PTR(o_shares);
  CHECK_PTR(lse2_shares);
  CHECK_PTR(out);
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return attend_merge_launch(o_shares, lse2_shares, R, rows, head_dim, out, static_cast<cudaStream_t>(stream));
}

// the device address of pinned host memory, or an error when it is not pinned and device-mapped
static msa_status mapped_host(const void* p, const char* name, const void** dev) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
  if (a.type != cudaMemoryTypeHost || !a.devicePointer)
    return fail(MSA_ERR_INVALID_ARG, "%s must be pinned (page-locked, device-mapped) host memory", name);
  *dev = a.devicePointer;
  return MSA_OK;
}

static bool tiered_sizes_ok(const msa_dims* dims, int32_t B, int32_t n_docs, int32_t n_chunks, int32_t k,
                            int32_t t_loc_max, int32_t pos_offset, int32_t capacity_chunks) {
  return dims && B >= 1 && B <= 65535 && n_docs >= 1 && n_chunks >= n_docs && k >= 1 && k <= n_docs && k <= 256 &&
         t_loc_max >= 1 && pos_offset >= 0 && (int64_t)pos_offset + t_loc_max <= (1 << 24) && capacity_chunks >= 1 &&
         dims->n_kv >= 1 && dims->n_q >= dims->n_kv && dims->n_r >= 1 && dims->d_r >= 1;
}

size_t msa_tiered_workspace_size(const msa_dims* dims, int32_t n_layers, int32_t B, int32_t n_docs, int32_t n_chunks,
                                 int32_t k, int32_t t_loc_max, int32_t pos_offset, int32_t capacity_chunks) {
  if (n_layers < 1 || n_layers > 4096 ||
      !tiered_sizes_ok(dims, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity_chunks))
    return 0;
  return tiered_workspace_size(*dims, n_layers, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity_chunks);
}

msa_status msa_tiered_decode(const msa_dims* dims, const msa_layer* layers, int32_t n_layers, int32_t B,
                             const int32_t* chunk_off, int32_t n_docs, int32_t n_chunks, int32_t k,
                             const int32_t* loc_len, int32_t t_loc_max, int32_t pos_offset, int32_t capacity_chunks,
                             void* ws, size_t ws_bytes, void* stream, void* copy_stream) {
  msa_status st = check_dims(dims, true, true);
  if (st != MSA_OK) return st;
  if (!layers) return fail(MSA_ERR_INVALID_ARG, "layers is NULL");
  if (n_layers < 1 || n_layers > 4096) return fail(MSA_ERR_INVALID_ARG, "n_layers must be in [1, 4096] (got %d)", n_layers);
  if (B < 1 || B > 65535) return fail(MSA_ERR_INVALID_ARG, "B must be in [1, 65535] (got %d)", B);
  if (n_docs < 1 || n_chunks < n_docs)
    return fail(MSA_ERR_INVALID_ARG, "need 1 <= n_docs <= n_chunks (got %d, %d)", n_docs, n_chunks);
  if (k < 1 || k > n_docs || k > 256)
    return fail(MSA_ERR_INVALID_ARG, "k must be in [1, min(n_docs, 256)] (got %d, n_docs %d)", k, n_docs);
  if ((size_t)((n_docs + 4095) / 4096) * k > 24576)
    return fail(MSA_ERR_UNSUPPORTED, "n_docs * k too large for the top-k merge");
  if (t_loc_max < 1) return fail(MSA_ERR_INVALID_ARG, "t_loc_max must be >= 1 (got %d)", t_loc_max);
  if (pos_offset < 0 || (int64_t)pos_offset + t_loc_max > (1 << 24))
    return fail(MSA_ERR_INVALID_ARG, "positions must lie in [0, 2^24)");
  if (capacity_chunks < 1) return fail(MSA_ERR_INVALID_ARG, "capacity_chunks must be >= 1");
  CHECK_PTR(chunk_off);
  CHECK_PTR(loc_len);
  std::vector<const void*> K_dev((size_t)n_layers), V_dev((size_t)n_layers);
  for (int32_t l = 0; l < n_layers; ++l) {
    const msa_layer& L = layers[l];
    if (L.W_QR && (dims->hidden < 64 || dims->hidden % 64 != 0 || dims->hidden > 8192))
      return fail(MSA_ERR_UNSUPPORTED, "hidden must be a multiple of 64 in [64, 8192] (got %d)", dims->hidden);
    if (!L.Hq || !aligned16(L.Hq) || !L.KR_bar || !aligned16(L.KR_bar) || !L.q || !aligned16(L.q) || !L.K_loc ||
        !aligned16(L.K_loc) || !L.V_loc || !aligned16(L.V_loc) || !L.topk_idx || !aligned16(L.topk_idx) ||
        !L.topk_score || !aligned16(L.topk_score) || !L.out || !aligned16(L.out) || !L.K_bar_host ||
        !aligned16(L.K_bar_host) || !L.V_bar_host || !aligned16(L.V_bar_host))
      return fail(MSA_ERR_INVALID_ARG, "layer %d: a required pointer is NULL or not 16-byte aligned", l);
    if ((L.W_QR && !aligned16(L.W_QR)) || (L.kr_inv_norm && !aligned16(L.kr_inv_norm)) ||
        (L.k_new && !aligned16(L.k_new)) || (L.v_new && !aligned16(L.v_new)))
      return fail(MSA_ERR_INVALID_ARG, "layer %d: an optional pointer is not 16-byte aligned", l);
    if ((L.k_new == nullptr) != (L.v_new == nullptr))
      return fail(MSA_ERR_INVALID_ARG, "layer %d: k_new and v_new go together", l);
    st = mapped_host(L.K_bar_host, "K_bar_host", &K_dev[l]);
    if (st != MSA_OK) return st;
    st = mapped_host(L.V_bar_host, "V_bar_host", &V_dev[l]);
    if (st != MSA_OK) return st;
  }
  const size_t need =
      tiered_workspace_size(*dims, n_layers, B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity_chunks);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return tiered_launch(*dims, layers, K_dev.data(), V_dev.data(), n_layers, B, chunk_off, n_docs, n_chunks, k, loc_len,
                       t_loc_max, pos_offset, capacity_chunks, ws, static_cast<cudaStream_t>(stream),
                       static_cast<cudaStream_t>(copy_stream));
}

msa_status msa_rope_rows(const msa_dims* dims, void* x, int32_t rows, int32_t heads, const int32_t* positions,
                         void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (rows < 1 || heads < 1) return fail(MSA_ERR_INVALID_ARG, "rows and heads must be >= 1 (got %d, %d)", rows, heads);
  CHECK_PTR(x);
  if (!positions) return fail(MSA_ERR_INVALID_ARG, "positions is NULL");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return rope_rows_launch(*dims, x, rows, heads, positions, static_cast<cudaStream_t>(stream));
}

msa_status msa_kv_append(const msa_dims* dims, const void* k_new, const void* v_new, void* K_loc, void* V_loc,
                         int32_t B, int32_t t_loc_max, const int32_t* slots, int32_t pos_offset, void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (B < 1 || t_loc_max < 1) return fail(MSA_ERR_INVALID_ARG, "B and t_loc_max must be >= 1 (got %d, %d)", B, t_loc_max);
  if (pos_offset < 0 || (int64_t)pos_offset + t_loc_max > (1 << 24))
    return fail(MSA_ERR_INVALID_ARG, "positions must lie in [0, 2^24)");
  CHECK_PTR(k_new);
  CHECK_PTR(v_new);
  CHECK_PTR(K_loc);
  CHECK_PTR(V_loc);
  if (!slots) return fail(MSA_ERR_INVALID_ARG, "slots is NULL");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return kv_append_launch(*dims, k_new, v_new, K_loc, V_loc, B, t_loc_max, slots, pos_offset,
                          static_cast<cudaStream_t>(stream));
}

size_t msa_rope_cache_size(const msa_dims* dims, int32_t t_loc_max) {
  if (!dims || t_loc_max < 1 || (dims->head_dim != 64 && dims->head_dim != 128)) return 0;
  return (size_t)t_loc_max * (dims->head_dim / 2) * sizeof(float2);
}

msa_status msa_rope_cache_build(const msa_dims* dims, int32_t t_loc_max, int32_t pos_offset, void* cache,
                                size_t cache_bytes, void* stream) {
  msa_status st = check_dims(dims, true, false);
  if (st != MSA_OK) return st;
  if (t_loc_max < 1) return fail(MSA_ERR_INVALID_ARG, "t_loc_max must be >= 1");
  if (pos_offset < 0 || (int64_t)pos_offset + t_loc_max > (1 << 24))
    return fail(MSA_ERR_INVALID_ARG, "positions must lie in [0, 2^24)");
  CHECK_PTR(cache);
  if (cache_bytes < msa_rope_cache_size(dims, t_loc_max))
    return fail(MSA_ERR_WORKSPACE, "rope cache too small: %zu < %zu bytes", cache_bytes,
                msa_rope_cache_size(dims, t_loc_max));
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return rope_cache_build(*dims, t_loc_max, pos_offset, static_cast<float2*>(cache), static_cast<cudaStream_t>(stream));
}

// ------------------------------ router training ------------------------------
size_t msa_aux_loss_workspace_size(const msa_dims* dims, int32_t P, int32_t N) {
  if (!dims || P < 1 || N < 0) return 0;
  return aux_workspace(*dims, P, N, nullptr, nullptr);
}

msa_status msa_aux_loss(const msa_dims* dims, const void* QR, const void* K_pos, const void* K_neg, int32_t P,
                        int32_t N, float tau, float* loss, float* grad_QR, float* grad_K_pos, float* grad_K_neg,
                        void* ws, size_t ws_bytes, void* stream) {
  msa_status st = check_dims(dims, false, true);
  if (st != MSA_OK) return st;
  if (P < 1 || P > (1 << 20)) return fail(MSA_ERR_INVALID_ARG, "P must be in [1, 2^20] (got %d)", P);
  if (N < 0 || N > 1023) return fail(MSA_ERR_INVALID_ARG, "N must be in [0, 1023] (got %d)", N);
  if (!(tau > 0.f) || !std::isfinite(tau)) return fail(MSA_ERR_INVALID_ARG, "tau must be finite and > 0");
  CHECK_PTR(QR);
  CHECK_PTR(K_pos);
  if (N > 0) CHECK_PTR(K_neg);
  CHECK_PTR(loss);
  CHECK_OPT_PTR(grad_QR);
  CHECK_OPT_PTR(grad_K_pos);
  CHECK_OPT_PTR(grad_K_neg);
  const size_t need = aux_workspace(*dims, P, N, nullptr, nullptr);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return aux_loss_launch(*dims, QR, K_pos, K_neg, P, N, tau, loss, grad_QR, grad_K_pos, grad_K_neg, ws,
                         static_cast<cudaStream_t>(stream));
}

// ------------------------------ encode ------------------------------
size_t msa_encode_workspace_size(const msa_dims* dims, int64_t T, int32_t n_docs, int32_t n_chunks) {
  if (!dims || T < 1 || n_docs < 1 || n_chunks < 1) return 0;
  return encode_workspace(*dims, T, n_docs, n_chunks, nullptr, nullptr);
}

msa_status msa_encode_memory(const msa_dims* dims, const void* H, int64_t T, const int64_t* doc_off, int32_t n_docs,
                             const int32_t* chunk_off, int32_t n_chunks, const void* W_K, const void* W_V,
                             const void* W_KR, void* K_bar, void* V_bar, void* KR_bar, int32_t kr_layout, void* ws,
                             size_t ws_bytes, void* stream) {
  msa_status st = check_dims(dims, true, true);
  if (st != MSA_OK) return st;
  if (dims->hidden < 64 || dims->hidden % 64 != 0)
    return fail(MSA_ERR_UNSUPPORTED, "hidden must be a positive multiple of 64 (got %d)", dims->hidden);
  if ((dims->n_kv * dims->head_dim) % 128 != 0 || (dims->n_r * dims->d_r) % 128 != 0)
    return fail(MSA_ERR_UNSUPPORTED, "n_kv*head_dim and n_r*d_r must be multiples of 128");
  if (T < 1 || n_docs < 1 || n_chunks < n_docs || (int64_t)n_chunks > (T + 63) / 64 + n_docs)
    return fail(MSA_ERR_INVALID_ARG, "inconsistent T / n_docs / n_chunks (%lld, %d, %d)", (long long)T, n_docs,
                n_chunks);
  CHECK_PTR(H);
  CHECK_PTR(doc_off);
  CHECK_PTR(chunk_off);
  CHECK_PTR(W_K);
  CHECK_PTR(W_V);
  CHECK_PTR(W_KR);
  CHECK_PTR(K_bar);
  CHECK_PTR(V_bar);
  CHECK_PTR(KR_bar);
  const size_t need = encode_workspace(*dims, T, n_docs, n_chunks, nullptr, nullptr);
  if (ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return fail(MSA_ERR_INVALID_ARG, "workspace must be non-NULL and 256-byte aligned");
  if (kr_layout != 0 && kr_layout != 1) return fail(MSA_ERR_INVALID_ARG, "kr_layout must be 0 or 1 (got %d)", kr_layout);
  if (fault_injected()) return fail(MSA_ERR_CUDA, "injected fault (MSA_FAULT=launch)");
  return encode_launch(*dims, H, T, doc_off, n_docs, chunk_off, n_chunks, W_K, W_V, W_KR, K_bar, V_bar, KR_bar,
                       kr_layout, ws, static_cast<cudaStream_t>(stream));
}

msa_status msa_append_memory(const msa_dims* dims, const void* H_new, int64_t T_new, const int64_t* doc_off_new,
                             int32_t n_docs_new, const int32_t* chunk_off_new, int32_t n_chunks_new,
                             const void* W_K, const void* W_V, const void* W_KR, void* K_bar, void* V_bar,
                             void* KR_bar, int32_t chunk_capacity, int32_t* chunk_off, int32_t n_docs_old,
                             int32_t n_chunks_old, void* ws, size_t ws_bytes, void* stream) {
  if (n_docs_old < 0 || n_chunks_old < n_docs_old || n_chunks_new < 1 ||
      (int64_t)n_chunks_old + n_chunks_new > chunk_capacity)
    return fail(MSA_ERR_INVALID_ARG, "append of %d chunks after %d (%d docs) exceeds the capacity of %d chunks",
                n_chunks_new, n_chunks_old, n_docs_old, chunk_capacity);
  CHECK_PTR(chunk_off);
  CHECK_PTR(K_bar);
  CHECK_PTR(V_bar);
  CHECK_PTR(KR_bar);
  if (!dims) return fail(MSA_ERR_INVALID_ARG, "dims is NULL");
  // the new documents' chunks land after the existing ones (chunk-major rows: a pointer offset)
  const size_t row_kv = (size_t)dims->n_kv * dims->head_dim, row_r = (size_t)dims->n_r * dims->d_r;
  uint16_t* Kb = static_cast<uint16_t*>(K_bar) + (size_t)n_chunks_old * row_kv;
  uint16_t* Vb = static_cast<uint16_t*>(V_bar) + (size_t)n_chunks_old * row_kv;
  uint16_t* KRb = static_cast<uint16_t*>(KR_bar) + (size_t)n_chunks_old * row_r;
  msa_status st = msa_encode_memory(dims, H_new, T_new, doc_off_new, n_docs_new, chunk_off_new, n_chunks_new, W_K,
                                    W_V, W_KR, Kb, Vb, KRb, 0, ws, ws_bytes, stream);
  if (st != MSA_OK) return st;
  return chunk_off_extend_launch(chunk_off, n_docs_old, n_chunks_old, chunk_off_new, n_docs_new,
                                 static_cast<cudaStream_t>(stream));
}

// ------------------------------ tracing ------------------------------
msa_status msa_trace_enable(int32_t on) {
  TraceState& t = trace();
  std::lock_guard<std::mutex> g(t.mu);
  t.on = on != 0;
  return MSA_OK;
}

msa_status msa_trace_reset(void) {
  TraceState& t = trace();
  std::lock_guard<std::mutex> g(t.mu);
  flush_trace(t);
  for (int i = 0; i < kKernelCount; ++i) {
    t.total_ms[i] = 0.0;
    t.launches[i] = 0;
  }
  return MSA_OK;
}

int32_t msa_trace_num_kernels(void) { return kKernelCount; }

const char* msa_trace_kernel_name(int32_t kernel_id) {
  if (kernel_id < 0 || kernel_id >= kKernelCount) return "";
  return kKernelNames[kernel_id];
}

msa_status msa_trace_read(int32_t kernel_id, double* total_ms, int64_t* launches) {
  if (kernel_id < 0 || kernel_id >= kKernelCount) return fail(MSA_ERR_INVALID_ARG, "bad kernel id %d", kernel_id);
  TraceState& t = trace();
  std::lock_guard<std::mutex> g(t.mu);
  flush_trace(t);
  if (total_ms) *total_ms = t.total_ms[kernel_id];
  if (launches) *launches = t.launches[kernel_id];
  return MSA_OK;
}

}  // extern "C"

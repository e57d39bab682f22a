// Stage 1 of MSA: offline memory encoding.
//
// Definition (IRMaD reading of the MSA paper, "M. Materials & Methods",
// routing item and position item; paper digest, "Method step details", Stage 1):
//   K = H W_K with document-wise RoPE (positions restart at 0 in every document),
//   V = H W_V, K^R = H W^KR, each mean-pooled over 64-token chunks that never
//   cross a document boundary (the last chunk of a document is shorter).
//
// Kernels:
//   chunk_map_kernel   first token, length and document-relative position of every chunk
//   transpose_kernel   W [hidden, N] -> W^T [N, hidden] (K-major B operand)
//   gemm_kernel<K>     per-token K projection on tcgen05 tensor cores: M = two
//                      chunks (2 x 64 token rows, each chunk loaded by its own TMA
//                      box), N = 256 (or 128), accumulators in TMEM; the epilogue rotates
//                      each row at its document-relative position and pools the
//                      64 rows of each chunk -> K̄
//   pool_h_kernel      H̄ = chunk mean of H, stored as bf16 hi + lo terms [C, 2*hidden]
//   gemm_kernel<POOL>  (H̄_hi | H̄_lo) [W_V | W^KR] over K = 2*hidden -> V̄, K̄^R.
//                      Pooling before the projection is exact by linearity;
//                      splitting H̄ into two bf16 terms keeps ~16 mantissa bits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace msa {

struct EncodeWs {
  int64_t* tok0;            // [C] first token of each chunk
  int32_t* clen;            // [C] tokens in the chunk (1..64)
  int32_t* pos0;            // [C] document-relative position of the chunk's first token
  __nv_bfloat16* wkT;       // [n_kv*D, hidden]
  __nv_bfloat16* wvrT;      // [n_kv*D + n_r*d_r, hidden]
  __nv_bfloat16* hbar;      // [C, 2*hidden] pooled H, hi | lo
};

namespace {

constexpr int kBM = 128, kBK = 64;
constexpr int kEncStagesMax = 4;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kEncThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue

__global__ void chunk_map_kernel(const int64_t* __restrict__ doc_off, const int32_t* __restrict__ chunk_off,
                                 int n_docs, int n_chunks, int64_t T, int64_t* __restrict__ tok0,
                                 int32_t* __restrict__ clen, int32_t* __restrict__ pos0) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_docs; i += gridDim.x * blockDim.x) {
    const int64_t a = doc_off[i], e = doc_off[i + 1];
    const int c0 = chunk_off[i], c1 = chunk_off[i + 1];
    if (e <= a || e > T || c1 - c0 != (int)((e - a + 63) / 64) || c0 < 0 || c1 > n_chunks) {
      raise_dev_error(kDevErrBadIndex);
      continue;
    }
    for (int j = 0; j < c1 - c0; ++j) {
      tok0[c0 + j] = a + 64ll * j;
      const int64_t rem = e - (a + 64ll * j);
      clen[c0 + j] = rem < 64 ? (int)rem : 64;
      pos0[c0 + j] = 64 * j;
    }
  }
}

// out[n][k] = in[k][n] for an in [K, N] bf16 matrix; out rows start at out_row0
__global__ void transpose_kernel(const uint16_t* __restrict__ in, int K, int N, uint16_t* __restrict__ out,
                                 int out_row0) {
  __shared__ uint16_t tile[64][66];
  const int k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  for (int i = threadIdx.y; i < 64; i += blockDim.y) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    tile[i][threadIdx.x] = (k < K && n < N) ? in[(size_t)k * N + n] : 0;
    const int n2 = n0 + threadIdx.x + 32;
    tile[i][threadIdx.x + 32] = (k < K && n2 < N) ? in[(size_t)k * N + n2] : 0;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 64; i += blockDim.y) {
    const int n = n0 + i;
    if (n >= N) continue;
    const int k = k0 + threadIdx.x, k2 = k0 + threadIdx.x + 32;
    if (k < K) out[(size_t)(out_row0 + n) * K + k] = tile[threadIdx.x][i];
    if (k2 < K) out[(size_t)(out_row0 + n) * K + k2] = tile[threadIdx.x + 32][i];
  }
}

// H̄[c] = mean of the chunk's token rows, as bf16 hi + lo terms.  Work item = (chunk, slice of
// kPoolCols columns); persistent: one CTA per SM takes items blockIdx.x, + gridDim.x, ...  Thread
// 0 streams each item's tile (the chunk's first row and the 63 after it, kPoolCols columns; rows
// past the chunk are not used, past T zero-filled) by TMA into a 2-stage ring; thread t adds
// column t of the chunk's rows in row order.  It lets the K-projection GEMM start at once (the
// GEMM does not read H̄): a pooling CTA (128 threads, 32 KB of shared memory) and a GEMM CTA
// (192 threads, 214 registers, ~187 KB) fit on one SM together, and the pooling's reads of H go
// beside the tensor-bound GEMM.
constexpr int kPoolThreads = 128;
constexpr int kPoolCols = kPoolThreads;  // one column per thread
constexpr int kPoolRows = 64;            // rows per tile: a whole chunk
constexpr int kPoolStageBytes = kPoolRows * kPoolCols * 2;
constexpr size_t kPoolSmem = 2 * (size_t)kPoolStageBytes + 128;
__global__ void __launch_bounds__(kPoolThreads) pool_h_kernel(const __grid_constant__ CUtensorMap h_map, int hidden,
                                                              int n_chunks, const int64_t* __restrict__ tok0,
                                                              const int32_t* __restrict__ clen,
                                                              __nv_bfloat16* __restrict__ hbar) {
  extern __shared__ __align__(128) uint8_t pool_sm_raw[];
  // a TMA tile's shared-memory destination must start on a 128-byte boundary; the dynamic area
  // follows this kernel's static variables, so its start is rounded up by hand (kPoolSmem holds
  // the 128 bytes of slack)
  uint8_t* pool_sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pool_sm_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t full[2], empty[2];
  __shared__ int abort_flag;
  pdl_launch_dependents();  // the GEMM that follows reads nothing this kernel writes
  const int tid = threadIdx.x;
  const int n_slices = (hidden + kPoolCols - 1) / kPoolCols;
  const long long n_items = (long long)n_chunks * n_slices;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kPoolThreads);
    }
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&h_map);
  }
  __syncthreads();
  auto issue = [&](long long item, int k) {  // item's tile into stage k % 2
    const int c = (int)(item / n_slices), sl = (int)(item % n_slices);
    uint64_t* bar = &full[k & 1];
    mbar_arrive_expect_tx(bar, (uint32_t)kPoolStageBytes);
    tma_load_2d(pool_sm + (size_t)(k & 1) * kPoolStageBytes, &h_map, bar, sl * kPoolCols, (int)tok0[c]);
  };
  long long item = blockIdx.x;
  int issued = 0;  // tiles requested (thread 0)
  if (tid == 0 && item < n_items) issue(item, issued++);
  for (int k = 0; item < n_items; ++k, item += gridDim.x) {
    // the next item's tile, once every thread is done with the stage it refills
    const long long nxt = item + gridDim.x;
    if (tid == 0 && nxt < n_items) {
      if (k >= 1 && !mbar_wait(&empty[(k + 1) & 1], ((k - 1) >> 1) & 1, &abort_flag)) break;
      issue(nxt, issued++);
    }
    if (!mbar_wait(&full[k & 1], (k >> 1) & 1, &abort_flag)) break;
    const int c = (int)(item / n_slices), sl = (int)(item % n_slices);
    const int n = clen[c];
    const int col = sl * kPoolCols + tid;
    const uint16_t* t = reinterpret_cast<const uint16_t*>(pool_sm + (size_t)(k & 1) * kPoolStageBytes) + tid;
    float acc = 0.f;
    for (int r = 0; r < n; ++r) acc += bf16_bits_to_float(t[r * kPoolCols]);
    mbar_arrive(&empty[k & 1]);  // this thread has read the stage
    if (col < hidden) {
      const float m = acc * (1.0f / (float)n);
      const __nv_bfloat16 hi = __float2bfloat16_rn(m);
      __nv_bfloat16* dst = hbar + (size_t)c * 2 * hidden + col;
      dst[0] = hi;
      dst[hidden] = __float2bfloat16_rn(m - __bfloat162float(hi));
    }
  }
  // after an abort: the copy this CTA may still have in flight lands before it exits
  if (abort_flag && tid == 0) mbar_drain_ring(full, 2, issued - 2, issued);
}

// Sum of v[0..31] over the 32 lanes of a warp, transposed: on return v[0] of
// lane l holds the warp-wide sum of column l (31 shuffles for 32 columns).
__device__ __forceinline__ void warp_transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
}

enum EncMode { kModeK = 0, kModePooled = 1 };

struct GemmParams {
  int hidden;            // K extent of W (and of H)
  int kblocks;           // K loop length in 64-element blocks (hidden/64, or 2*hidden/64 pooled)
  int n_tiles;           // N / 256
  int m_tiles;
  int n_chunks;
  int head_dim;
  RopeTurns turns;
  const int64_t* tok0;
  const int32_t* clen;
  const int32_t* pos0;
  __nv_bfloat16* out0;   // K̄ (mode K) or V̄ (pooled)
  __nv_bfloat16* out1;   // K̄^R (pooled)
  int n_out0;            // columns of out0 (n_kv*D); pooled: columns >= n_out0 go to out1
  int n_out1;
  int out1_head_major;   // out1 (K̄^R) stored [n_r][C][d_r]
  int d_r;
};

template <int MODE, int kBN>
__global__ void __launch_bounds__(kEncThreads, 1) gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                                              const __grid_constant__ CUtensorMap map_b,
                                                              const GemmParams p) {
  constexpr int kBBytes = kBN * kBK * 2;
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr int kEncStages = MODE == kModeK ? 3 : 4;  // mode K gives one stage to the RoPE tables
  constexpr uint32_t kTmemCols = 2 * kBN;  // two 128 x kBN fp32 accumulators
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* red = reinterpret_cast<float*>(smem + kEncStages * kStageBytes);  // [2][4][kBN]
  // RoPE tables (mode K): fine[i][r] = (cos, sin)(r * theta_i) for the 64 offsets r inside a
  // chunk (pair-major, so the 32 rows of a warp read consecutive words), and per tile
  // coarse[c][i] = (cos, sin)(pos0(c) * theta_i) for its two chunks, reduced in fp64.
  float2* fine = reinterpret_cast<float2*>(red + 2 * 4 * kBN);             // [64 pairs][64 rows]
  float2* coarse = fine + (MODE == kModeK ? 64 * 64 : 0);                  // [2 chunks][64 pairs]
  uint64_t* full = reinterpret_cast<uint64_t*>(coarse + (MODE == kModeK ? 2 * 64 : 0));
  uint64_t* empty = full + kEncStages;
  uint64_t* tfull = empty + kEncStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drained = tempty + 2;  // after an abort: every MMA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drained + 1);
  __shared__ int abort_flag;       // a bounded wait of this CTA gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kEncStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drained, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (MODE == kModeK) {
    const int half = p.head_dim / 2;
    for (int e = threadIdx.x; e < half * 64; e += blockDim.x) fine[e] = rope_cos_sin(p.turns, e / 64, e % 64);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------- TMA producer -------------------------
    if (lane == 0) {
      prefetch_tensormap(&map_a);
      prefetch_tensormap(&map_b);
      int it = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !abort_flag; tile += gridDim.x) {
        const int m = tile / p.n_tiles, n = tile % p.n_tiles;
        int ya0, ya1;
        if (MODE == kModeK) {
          const int c0 = 2 * m;
          const int c1 = min(2 * m + 1, p.n_chunks - 1);
          ya0 = (int)p.tok0[c0];
          ya1 = (int)p.tok0[c1];
        } else {
          ya0 = m * kBM;
          ya1 = m * kBM + 64;
        }
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int st = it % kEncStages;
          if (it >= kEncStages && !mbar_wait(&empty[st], ((it / kEncStages) - 1) & 1, &abort_flag)) break;
          uint8_t* a_s = stages + st * kStageBytes;
          uint8_t* b_s = a_s + kABytes;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          tma_load_2d(a_s, &map_a, &full[st], kb * kBK, ya0);
          tma_load_2d(a_s + kABytes / 2, &map_a, &full[st], kb * kBK, ya1);
          const int kx = (MODE == kModeK) ? kb * kBK : (kb * kBK) % p.hidden;
          tma_load_2d(b_s, &map_b, &full[st], kx, n * kBN);
        }
      }
      // after an abort: the stages issued and possibly still in flight land before the CTA exits
      if (abort_flag) mbar_drain_ring(full, kEncStages, it - kEncStages, it);
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer -------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(kBM, kBN);
      int it = 0, lt = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !abort_flag; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(&tempty[buf], ((lt >> 1) - 1) & 1, &abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kBN;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int st = it % kEncStages;
          if (!mbar_wait(&full[st], (it / kEncStages) & 1, &abort_flag)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + st * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks) {
            umma_bf16(d_tmem, umma_desc_k_sw128(a_addr + ks * 32), umma_desc_k_sw128(b_addr + ks * 32), idesc,
                      (kb | ks) != 0);
          }
          umma_commit(&empty[st]);
        }
        umma_commit(&tfull[buf]);
      }
      if (abort_flag) {  // every MMA issued completes before the TMEM is freed
        umma_commit(drained);
        mbar_drain_ring(drained, 1, 0, 1);
      }
    }
  } else {
    // ------------------------- epilogue (warps 2..5) -------------------------
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = 32 * q + lane;          // accumulator row = TMEM lane
    const int ew = warp - 2;
    int lt = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++lt) {
      const int m = tile / p.n_tiles, n = tile % p.n_tiles;
      const int buf = lt & 1;
      // the four epilogue warps meet at named barriers (mode K): they decide together, at the top of
      // a tile, whether to leave
      const bool ok = warp_wait(&tfull[buf], (lt >> 1) & 1, &abort_flag);
      if (MODE == kModeK ? named_bar_any(3, 128, !ok) : !ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(32 * q) << 16) + buf * kBN;
      if (MODE == kModeK) {
        const int chunk = 2 * m + (row >> 6);
        const int rr = row & 63;
        const bool chunk_ok = chunk < p.n_chunks;
        const int len = chunk_ok ? p.clen[chunk] : 0;
        const bool valid = rr < len;
        const int D = p.head_dim, half = D / 2;
        // this tile's per-chunk base angles: 128 epilogue threads = 2 chunks x 64 pairs
        {
          const int et = threadIdx.x - 64;
          const int c2 = et >> 6, i = et & 63;
          const int ch = 2 * m + c2;
          if (i < half) coarse[c2 * 64 + i] = rope_cos_sin(p.turns, i, ch < p.n_chunks ? p.pos0[ch] : 0);
          named_bar_sync(2, 128);
        }
        const float2* cb = coarse + (row >> 6) * 64;
        float* rbuf = red + (size_t)(buf * 4 + ew) * kBN;
        // kBN columns = kBN/D heads; pairs (i, i + D/2) inside each head, 32 pairs per pass
        for (int c0 = 0; c0 < kBN; c0 += D) {
          for (int i0 = 0; i0 < half; i0 += 32) {
            float x[32], y[32];
            tmem_ld32(t_row + c0 + i0, x);
            tmem_ld32(t_row + c0 + half + i0, y);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float2 f = fine[(i0 + j) * 64 + rr];
              const float2 c = cb[i0 + j];
              const float cs = c.x * f.x - c.y * f.y;   // cos((pos0 + rr) theta)
              const float sn = c.y * f.x + c.x * f.y;   // sin((pos0 + rr) theta)
              const float xr = x[j] * cs - y[j] * sn;
              const float yr = y[j] * cs + x[j] * sn;
              x[j] = valid ? xr : 0.f;
              y[j] = valid ? yr : 0.f;
            }
            warp_transpose_reduce32(x, lane);
            warp_transpose_reduce32(y, lane);
            rbuf[c0 + i0 + lane] = x[0];
            rbuf[c0 + half + i0 + lane] = y[0];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        named_bar_sync(1, 128);
        // chunk A = rows 0..63 = lane quarters 0,1 (warps 4,5 -> ew 2,3); chunk B = quarters 2,3 (ew 0,1)
        const int et = threadIdx.x - 64;
        const float* rb = red + (size_t)buf * 4 * kBN;
        for (int idx = et; idx < 2 * kBN; idx += 128) {
          const int which = idx / kBN, col = idx % kBN;
          const int ch = 2 * m + which;
          if (ch >= p.n_chunks) continue;
          const float s = which == 0 ? (rb[2 * kBN + col] + rb[3 * kBN + col]) : (rb[0 * kBN + col] + rb[1 * kBN + col]);
          const float v = s / (float)p.clen[ch];
          p.out0[(size_t)ch * p.n_out0 + n * kBN + col] = __float2bfloat16_rn(v);
        }
      } else {
        const int chunk = m * kBM + row;
        const int gc0 = n * kBN;
        const bool to0 = gc0 < p.n_out0;
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          float x[32];
          tmem_ld32(t_row + c0, x);
          tmem_ld_wait();
          if (chunk < p.n_chunks) {
            __nv_bfloat16* dst;
            if (to0) {
              dst = p.out0 + (size_t)chunk * p.n_out0 + gc0 + c0;
            } else {
              const int col = gc0 - p.n_out0 + c0;  // 32 columns inside one router head
              dst = p.out1_head_major
                        ? p.out1 + ((size_t)(col / p.d_r) * p.n_chunks + chunk) * p.d_r + col % p.d_r
                        : p.out1 + (size_t)chunk * p.n_out1 + col;
            }
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(x[2 * j], x[2 * j + 1]);
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int j = 0; j < 4; ++j) d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
  // launched early beside the chunk pooling (programmatic dependent launch), the K GEMM completes
  // only after the pooling has: the pooled GEMM after it then reads finished chunk means
  // (a plain launch returns at once here)
  pdl_wait();
}

size_t gemm_smem_bytes(int mode, int bn) {
  const int stages = mode == kModeK ? 3 : 4;
  const size_t tables = mode == kModeK ? (64 * 64 + 2 * 64) * sizeof(float2) : 0;
  return 1024 + (size_t)stages * (kABytes + bn * kBK * 2) + 2 * 4 * bn * sizeof(float) + tables +
         (2 * kEncStagesMax + 5) * sizeof(uint64_t) + 16;
}

template <int MODE>
cudaError_t launch_gemm(int bn, int grid, size_t smem, cudaStream_t s, const CUtensorMap& ma, const CUtensorMap& mb,
                        const GemmParams& p, bool early = false) {
  auto kern = bn == 256 ? gemm_kernel<MODE, 256> : gemm_kernel<MODE, 128>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ordered(early, kern, dim3(grid), dim3(kEncThreads), smem, s, ma, mb, p);
}

}  // namespace

namespace {
// chunk_off[n_docs_old + i] = n_chunks_old + chunk_off_new[i], i = 0 .. n_docs_new
__global__ void __launch_bounds__(256) chunk_off_extend_kernel(int32_t* __restrict__ chunk_off, int n_docs_old,
                                                               int n_chunks_old,
                                                               const int32_t* __restrict__ chunk_off_new,
                                                               int n_docs_new) {
  pdl_enter();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n_docs_new; i += gridDim.x * blockDim.x)
    chunk_off[n_docs_old + i] = n_chunks_old + chunk_off_new[i];
}
}  // namespace

msa_status chunk_off_extend_launch(int32_t* chunk_off, int n_docs_old, int n_chunks_old, const int32_t* chunk_off_new,
                                   int n_docs_new, cudaStream_t s) {
  TraceScope ts(kKChunkOffExtend, s);
  const int blocks = std::max(1, std::min(148, (n_docs_new + 1 + 255) / 256));
  MSA_CUDA_CHECK(launch_pdl(chunk_off_extend_kernel, dim3(blocks), dim3(256), 0, s, chunk_off, n_docs_old,
                            n_chunks_old, chunk_off_new, n_docs_new));
  return MSA_OK;
}

size_t encode_workspace(const msa_dims& d, int64_t T, int n_docs, int n_chunks, void* ws, EncodeWs* out) {
  (void)T;
  (void)n_docs;
  Carver cv(ws);
  EncodeWs w{};
  const int NK = d.n_kv * d.head_dim, NVR = d.n_kv * d.head_dim + d.n_r * d.d_r;
  w.tok0 = cv.take<int64_t>(n_chunks);
  w.clen = cv.take<int32_t>(n_chunks);
  w.pos0 = cv.take<int32_t>(n_chunks);
  w.wkT = cv.take<__nv_bfloat16>((size_t)NK * d.hidden);
  w.wvrT = cv.take<__nv_bfloat16>((size_t)NVR * d.hidden);
  // pooled H rows padded to a whole number of 128-row tiles (rows past C are never stored)
  const size_t rows = ((size_t)n_chunks + kBM - 1) / kBM * kBM;
  w.hbar = cv.take<__nv_bfloat16>(rows * 2 * d.hidden);
  if (out) *out = w;
  return cv.size();
}

msa_status encode_launch(const msa_dims& d, const void* H, int64_t T, const int64_t* doc_off, int n_docs,
                         const int32_t* chunk_off, int n_chunks, const void* W_K, const void* W_V, const void* W_KR,
                         void* K_bar, void* V_bar, void* KR_bar, int kr_layout, void* ws, cudaStream_t s) {
  if (T > INT32_MAX - 64) return fail(MSA_ERR_UNSUPPORTED, "T must be < 2^31 - 64 tokens");
  EncodeWs w;
  encode_workspace(d, T, n_docs, n_chunks, ws, &w);
  const int NK = d.n_kv * d.head_dim, NV = NK, NR = d.n_r * d.d_r;
  const int hidden = d.hidden;
  {
    TraceScope ts(kKEncChunkMap, s);
    chunk_map_kernel<<<std::max(1, std::min((n_docs + 255) / 256, 4 * sm_count())), 256, 0, s>>>(
        doc_off, chunk_off, n_docs, n_chunks, T, w.tok0, w.clen, w.pos0);
    MSA_CUDA_CHECK(cudaGetLastError());
  }
  {
    TraceScope ts(kKEncTransposeW, s);
    dim3 blk(32, 8);
    transpose_kernel<<<dim3((NK + 63) / 64, (hidden + 63) / 64), blk, 0, s>>>(
        static_cast<const uint16_t*>(W_K), hidden, NK, reinterpret_cast<uint16_t*>(w.wkT), 0);
    transpose_kernel<<<dim3((NV + 63) / 64, (hidden + 63) / 64), blk, 0, s>>>(
        static_cast<const uint16_t*>(W_V), hidden, NV, reinterpret_cast<uint16_t*>(w.wvrT), 0);
    transpose_kernel<<<dim3((NR + 63) / 64, (hidden + 63) / 64), blk, 0, s>>>(
        static_cast<const uint16_t*>(W_KR), hidden, NR, reinterpret_cast<uint16_t*>(w.wvrT), NV);
    MSA_CUDA_CHECK(cudaGetLastError());
  }
  // ---- H̄ (hi | lo), the chunk means for the pooled projections; the K GEMM runs beside it ----
  {
    CUtensorMap hm;
    const uint64_t hdims[2] = {(uint64_t)hidden, (uint64_t)T};
    const uint64_t hstr[1] = {(uint64_t)hidden * 2};
    const uint32_t hbox[2] = {(uint32_t)kPoolCols, (uint32_t)kPoolRows};
    msa_status st = encode_tensor_map(&hm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(H), hdims, hstr,
                                      hbox, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != MSA_OK) return st;
    TraceScope ts(kKEncPoolH, s);
    const int grid = std::max(1, std::min(sm_count(), n_chunks));
    MSA_CUDA_CHECK(set_max_dynamic_smem(reinterpret_cast<const void*>(pool_h_kernel), (int)kPoolSmem));
    MSA_CUDA_CHECK(launch_ordered(false, pool_h_kernel, dim3(grid), dim3(kPoolThreads), kPoolSmem, s, hm, hidden,
                                  n_chunks, static_cast<const int64_t*>(w.tok0), static_cast<const int32_t*>(w.clen),
                                  w.hbar));
  }
  // ---- K̄: per-token projection + RoPE + pooling on tcgen05 ----
  {
    CUtensorMap ma, mb;
    const uint64_t adims[2] = {(uint64_t)hidden, (uint64_t)T};
    const uint64_t astr[1] = {(uint64_t)hidden * 2};
    const uint32_t abox[2] = {64, 64};
    msa_status st = encode_tensor_map(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(H), adims, astr,
                                      abox, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    const int bn = (NK % 256 == 0) ? 256 : 128;
    const uint64_t bdims[2] = {(uint64_t)hidden, (uint64_t)NK};
    const uint32_t bbox[2] = {64, (uint32_t)bn};
    st = encode_tensor_map(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.wkT, bdims, astr, bbox,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    GemmParams p{};
    p.hidden = hidden;
    p.kblocks = hidden / kBK;
    p.n_tiles = NK / bn;
    p.m_tiles = (n_chunks + 1) / 2;
    p.n_chunks = n_chunks;
    p.head_dim = d.head_dim;
    rope_turns(d, p.turns.f);
    p.tok0 = w.tok0;
    p.clen = w.clen;
    p.pos0 = w.pos0;
    p.out0 = static_cast<__nv_bfloat16*>(K_bar);
    p.n_out0 = NK;
    const int grid = std::max(1, std::min(sm_count(), p.m_tiles * p.n_tiles));
    TraceScope ts(kKEncGemmK, s);
    MSA_CUDA_CHECK(launch_gemm<kModeK>(bn, grid, gemm_smem_bytes(kModeK, bn), s, ma, mb, p, /*early=*/true));
  }
  // ---- V̄ | K̄^R = H̄ [W_V | W^KR] ----
  {
    CUtensorMap ma, mb;
    const size_t rows = ((size_t)n_chunks + kBM - 1) / kBM * kBM;
    const uint64_t adims[2] = {(uint64_t)2 * hidden, (uint64_t)rows};
    const uint64_t astr[1] = {(uint64_t)4 * hidden};
    const uint32_t abox[2] = {64, 64};
    msa_status st = encode_tensor_map(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.hbar, adims, astr, abox,
                                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    const int bn = (NV % 256 == 0 && NR % 256 == 0) ? 256 : 128;
    const uint64_t bdims[2] = {(uint64_t)hidden, (uint64_t)(NV + NR)};
    const uint64_t bstr[1] = {(uint64_t)hidden * 2};
    const uint32_t bbox[2] = {64, (uint32_t)bn};
    st = encode_tensor_map(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.wvrT, bdims, bstr, bbox,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != MSA_OK) return st;
    GemmParams p{};
    p.hidden = hidden;
    p.kblocks = 2 * hidden / kBK;
    p.n_tiles = (NV + NR) / bn;
    p.m_tiles = (int)(rows / kBM);
    p.n_chunks = n_chunks;
    p.head_dim = d.head_dim;
    p.out0 = static_cast<__nv_bfloat16*>(V_bar);
    p.out1 = static_cast<__nv_bfloat16*>(KR_bar);
    p.n_out0 = NV;
    p.n_out1 = NR;
    p.out1_head_major = kr_layout == 1;
    p.d_r = d.d_r;
    const int grid = std::max(1, std::min(sm_count(), p.m_tiles * p.n_tiles));
    TraceScope ts(kKEncGemmPooled, s);
    MSA_CUDA_CHECK(launch_gemm<kModePooled>(bn, grid, gemm_smem_bytes(kModePooled, bn), s, ma, mb, p));
  }
  return MSA_OK;
}

}  // namespace msa

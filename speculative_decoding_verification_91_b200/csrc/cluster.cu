// Cheap unembedding over token clusters ("Gemma 4 拆解 | 多模态怎么塞进端侧，MTP
// drafter 又是怎么自带投机采样的" §4.3): instead of the logits of the whole
// vocabulary, score the clusters' centroids, keep the best n_select
// clusters and take the argmax over their tokens only.
//
//   cluster logits  h . centroid^T: the streaming GEMM (store mode), [M][C]
//   cluster_select  one CTA per row: packed (logit, cluster id) keys sorted
//                   in shared memory (bitonic), the n_select largest kept
//                   (equal logits: lower cluster id first)
//   cluster_cand    one CTA per (row, selected cluster, 16 of its tokens):
//                   dot products of h with the tokens' LM-head rows (stored
//                   in cluster order, so a cluster is a contiguous block of
//                   rows), each warp two rows with all its 16-byte loads of
//                   a row in flight; the best (logit, token) of the CTA goes
//                   into the row's packed key by atomicMax (equal logits:
//                   lowest token id)
//   cluster_finish  keys -> ids / max logits, keys cleared for the next call
//
// The candidate scoring is a memory-bound matrix-vector product (about
// n_select * S * d * 2 bytes per row); it runs on the CUDA cores.
#include <algorithm>

#include "common.cuh"
#include "gemm_epi.cuh"
#include "internal.h"

namespace sv {

namespace {

constexpr int kSelThreads = 512;
constexpr int kCandWarps = 8;
constexpr int kRowsPerWarp = 2;
constexpr int kRowsPerCta = kCandWarps * kRowsPerWarp;   // 16 tokens of a cluster per CTA

__global__ void __launch_bounds__(kSelThreads) cluster_select_kernel(const float* logits,
                                                                     int C, int P, int n_sel,
                                                                     int32_t* sel) {
  extern __shared__ unsigned long long keys[];   // P = power of two >= C
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i < P; i += kSelThreads)
    keys[i] = i < C ? pack_arg(logits[(size_t)m * C + i], i) : 0ull;   // 0 sorts below every key
  __syncthreads();
  // bitonic sort, ascending
  for (int k = 2; k <= P; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += kSelThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          if (((i & k) == 0) ? (a > b) : (a < b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  for (int t = tid; t < n_sel; t += kSelThreads) {
    float v;
    int c;
    unpack_arg(keys[P - 1 - t], v, c);
    sel[(size_t)m * n_sel + t] = c;
  }
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float dot8(uint4 w, uint4 x, float acc) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w}, xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(__uint_as_float(ws[i] << 16), __uint_as_float(xs[i] << 16), acc);
    acc = fmaf(__uint_as_float(ws[i] & 0xffff0000u), __uint_as_float(xs[i] & 0xffff0000u), acc);
  }
  return acc;
}

// grid (n_sel * ceil(S / 16), M)
__global__ void __launch_bounds__(kCandWarps * 32) cluster_cand_kernel(
    const uint16_t* h, int d, const int32_t* sel, int n_sel,
    const int32_t* tokens, int S, const uint16_t* wc,
    unsigned long long* keys) {
  extern __shared__ uint4 hs[];   // the row's h, d / 8 chunks of 16 bytes
  __shared__ unsigned long long best_w[kCandWarps];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunks_per_cluster = (S + kRowsPerCta - 1) / kRowsPerCta;
  const int j = blockIdx.x / chunks_per_cluster, r0 = (blockIdx.x % chunks_per_cluster) * kRowsPerCta;
  const int m = blockIdx.y;
  const int c = sel[(size_t)m * n_sel + j];
  const int nch = d / 8;
  const uint4* hrow = reinterpret_cast<const uint4*>(h + (size_t)m * d);
  for (int i = threadIdx.x; i < nch; i += kCandWarps * 32) hs[i] = hrow[i];
  __syncthreads();
  unsigned long long best = 0ull;
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int r = r0 + warp * kRowsPerWarp + rr;
    if (r >= S) break;
    const int tok = tokens[(size_t)c * S + r];
    if (tok < 0) continue;   // padding of a short last cluster
    const uint4* wrow = reinterpret_cast<const uint4*>(wc + ((size_t)c * S + r) * d);
    float acc = 0.f;
    constexpr int U = 10;    // loads of this lane in flight together
    for (int i0 = lane; i0 < nch; i0 += 32 * U) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < nch) w[u] = ld_stream16(wrow + i0 + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < nch) acc = dot8(w[u], hs[i0 + 32 * u], acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    best = max(best, pack_arg(acc, tok));
  }
  if (lane == 0) best_w[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long b = best_w[0];
#pragma unroll
    for (int w = 1; w < kCandWarps; ++w) b = max(b, best_w[w]);
    if (b) atomicMax(&keys[m], b);
  }
}

__global__ void cluster_finish_kernel(unsigned long long* keys, int M,
                                      int32_t* ids, float* maxv) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= M) return;
  float v;
  int id;
  unpack_arg(atomicExch(&keys[m], 0ull), v, id);
  ids[m] = id;
  if (maxv) maxv[m] = v;
}

int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

size_t cluster_logit_floats(int M, int C) { return (size_t)M * C; }

cudaError_t launch_cluster_unembed(const ClusterArgs& t, const uint16_t* h, int M, int d,
                                   int32_t* ids, float* maxv, float* cl_logits, int32_t* sel,
                                   unsigned long long* keys, const GemmBuffers& gb, cudaStream_t st) {
  // 1. cluster logits h . centroid^T
  GemmBuffers b = gb;
  b.out = cl_logits;
  cudaError_t e = launch_gemm_any(plan_gemm(M, t.n_clusters, d, kGemmStore), kGemmStore, h,
                                  t.centroids, b, st);
  if (e != cudaSuccess) return e;
  // 2. best clusters of each row
  const int P = pow2_at_least(t.n_clusters);
  const size_t sel_smem = (size_t)P * 8;
  e = cudaFuncSetAttribute(cluster_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sel_smem);
  if (e != cudaSuccess) return e;
  e = launch_k(cluster_select_kernel, dim3(M), dim3(kSelThreads), sel_smem, st,
               static_cast<const float*>(cl_logits), t.n_clusters, P, t.n_select, sel);
  if (e != cudaSuccess) return e;
  // 3. argmax over the selected clusters' tokens
  const int chunks = (t.cluster_size + kRowsPerCta - 1) / kRowsPerCta;
  const size_t h_smem = (size_t)d * 2;
  e = cudaFuncSetAttribute(cluster_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)h_smem);
  if (e != cudaSuccess) return e;
  e = launch_k(cluster_cand_kernel, dim3(t.n_select * chunks, M), dim3(kCandWarps * 32), h_smem, st,
               h, d, static_cast<const int32_t*>(sel), t.n_select, t.cluster_tokens,
               t.cluster_size, static_cast<const uint16_t*>(t.w_clustered), keys);
  if (e != cudaSuccess) return e;
  // 4. keys -> ids
  return launch_k(cluster_finish_kernel, dim3((M + 127) / 128), dim3(128), 0, st, keys, M, ids, maxv);
}

}  // namespace sv

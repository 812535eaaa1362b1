// Distribution-preserving (sampled) verification: speculative sampling
// (Leviathan, Kalman, Matias, ICML 2023, Algorithm 1; Chen et al. 2023) on
// the target's verify rows.  The pages state the property it keeps ("Gemma 4
// 发布时未包含 MTP 数据——为什么这很重要" §MTP 能快多少: the output is what decoding
// the target alone produces).
//
//   softmax_stats   one CTA per logit row: (max, sum of exp) of logits / T
//   sampled_accept  one thread per sequence: accept draft i iff
//                   u_i * q_i(d_i) < p_i(d_i); a = accepted count
//   sampled_draw    grid (sequences, 2048-token chunks): Gumbel-max draw from
//                   max(0, p_a - q_a) (a < k) or p_k: the best
//                   log w_v - log(-log g_v) of the chunk goes into the
//                   sequence's packed key by atomicMax (ties: lowest id)
//   sampled_finish  one thread per sequence: emitted tokens, next token,
//                   seq_lens += a + 1, key cleared
//
// The target logits come from the LM head in store mode (binary32 rows of the
// whole vocabulary, written to the workspace: B*(k+1) rows of V floats).
#include <math.h>

#include "common.cuh"
#include "gemm_epi.cuh"
#include "internal.h"

namespace sv {

namespace {

constexpr int kStatThreads = 1024;
constexpr int kDrawThreads = 256;
constexpr int kDrawChunk = 2048;

__global__ void __launch_bounds__(kStatThreads) softmax_stats_kernel(const float* logits,
                                                                     int V, float T,
                                                                     float2* stats) {
  __shared__ float red[kStatThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* l = logits + (size_t)row * V;
  float mx = -INFINITY;
  for (int v = tid; v < V; v += kStatThreads) mx = fmaxf(mx, __fdiv_rn(l[v], T));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < kStatThreads / 32; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  float s = 0.f;
  for (int v = tid; v < V; v += kStatThreads) s = __fadd_rn(s, expf(__fsub_rn(__fdiv_rn(l[v], T), m)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
  if (lane == 0) red[warp] = s;
  __syncthreads();
  if (tid == 0) {
    float tot = 0.f;
    for (int w = 0; w < kStatThreads / 32; ++w) tot = __fadd_rn(tot, red[w]);
    stats[row] = make_float2(m, tot);
  }
}

__device__ __forceinline__ float prob(const float* row, float2 st, int v, float T) {
  return __fdiv_rn(expf(__fsub_rn(__fdiv_rn(row[v], T), st.x)), st.y);
}

__global__ void sampled_accept_kernel(int B, int k, int V, float T, const float* lt,
                                      const float2* st_t, const float* ld,
                                      const float2* st_d, const int32_t* drafts,
                                      const float* u, int32_t* a_out,
                                      unsigned* status) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int q = k + 1;
  int a = 0;
  while (a < k) {
    const int d = drafts[(size_t)b * k + a];
    if (d < 0 || d >= V) {
      flag_status(status, SPEC_DEV_BAD_TOKEN);
      break;
    }
    const size_t rt = (size_t)b * q + a, rd = (size_t)b * k + a;
    const float p = prob(lt + rt * V, st_t[rt], d, T);
    const float qd = prob(ld + rd * V, st_d[rd], d, T);
    if (__fmul_rn(u[rd], qd) < p) ++a;
    else break;
  }
  a_out[b] = a;
}

__global__ void __launch_bounds__(kDrawThreads) sampled_draw_kernel(
    int k, int V, float T, const float* lt, const float2* st_t,
    const float* ld, const float2* st_d, const int32_t* a_arr,
    const float* g, unsigned long long* keys) {
  __shared__ unsigned long long best_w[kDrawThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = k + 1, a = a_arr[b];
  const size_t rt = (size_t)b * q + a;
  const float* prow = lt + rt * V;
  const float2 sp = st_t[rt];
  const bool resid = a < k;
  const size_t rd = (size_t)b * k + (resid ? a : 0);
  const float* qrow = resid ? ld + rd * V : nullptr;
  const float2 sq = resid ? st_d[rd] : make_float2(0.f, 1.f);
  unsigned long long best = 0ull;
  const int v0 = blockIdx.y * kDrawChunk;
  for (int v = v0 + tid; v < min(V, v0 + kDrawChunk); v += kDrawThreads) {
    float w = prob(prow, sp, v, T);
    if (resid) w = fmaxf(__fsub_rn(w, prob(qrow, sq, v, T)), 0.f);
    if (w > 0.f) {
      const float score = __fsub_rn(logf(w), logf(-logf(g[(size_t)b * V + v])));
      best = max(best, pack_arg(score, v));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, off));
  if (lane == 0) best_w[warp] = best;
  __syncthreads();
  if (tid == 0) {
    unsigned long long bb = best_w[0];
    for (int w = 1; w < kDrawThreads / 32; ++w) bb = max(bb, best_w[w]);
    if (bb) atomicMax(&keys[b], bb);
  }
}

__global__ void sampled_finish_kernel(int B, int k, const int32_t* drafts,
                                      const int32_t* a_arr,
                                      unsigned long long* keys, int32_t* seq_lens,
                                      int32_t* accept_len, int32_t* emitted, int32_t* new_last) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int q = k + 1, a = a_arr[b];
  const unsigned long long key = atomicExch(&keys[b], 0ull);
  float v;
  int tok;
  unpack_arg(key, v, tok);
  // no positive weight at all (p and q equal to the last bit): keep the draft
  if (key == 0ull) tok = a < k ? drafts[(size_t)b * k + a] : 0;
  for (int i = 0; i < q; ++i)
    emitted[(size_t)b * q + i] = i < a ? drafts[(size_t)b * k + i] : (i == a ? tok : -1);
  accept_len[b] = a;
  new_last[b] = tok;
  seq_lens[b] += a + 1;
}

}  // namespace

cudaError_t launch_sampled_tail(int B, int k, int V, float T, const float* lt, const float* ld,
                                float2* st_t, float2* st_d, const int32_t* drafts, const float* u,
                                const float* g, int32_t* a_arr, unsigned long long* keys,
                                int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                                int32_t* new_last, unsigned* status, cudaStream_t st) {
  const int q = k + 1;
  cudaError_t e = launch_k(softmax_stats_kernel, dim3(B * q), dim3(kStatThreads), 0, st, lt, V, T, st_t);
  if (e != cudaSuccess) return e;
  if (k > 0) {
    e = launch_k(softmax_stats_kernel, dim3(B * k), dim3(kStatThreads), 0, st, ld, V, T, st_d);
    if (e != cudaSuccess) return e;
  }
  e = launch_k(sampled_accept_kernel, dim3((B + 127) / 128), dim3(128), 0, st, B, k, V, T, lt,
               static_cast<const float2*>(st_t), ld, static_cast<const float2*>(st_d), drafts, u,
               a_arr, status);
  if (e != cudaSuccess) return e;
  e = launch_k(sampled_draw_kernel, dim3(B, (V + kDrawChunk - 1) / kDrawChunk), dim3(kDrawThreads), 0,
               st, k, V, T, lt, static_cast<const float2*>(st_t), ld, static_cast<const float2*>(st_d),
               static_cast<const int32_t*>(a_arr), g, keys);
  if (e != cudaSuccess) return e;
  return launch_k(sampled_finish_kernel, dim3((B + 127) / 128), dim3(128), 0, st, B, k, drafts,
                  static_cast<const int32_t*>(a_arr), keys, seq_lens, accept_len, emitted, new_last);
}

}  // namespace sv

// Small verify-step kernels: token embedding gather, RMSNorm, and the
// acceptance / bonus-token / commit kernel.
#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace sv {

namespace {

// out[m] = bf16(x[m] / sqrt(mean(x[m]^2) + eps)).  The mean, square root and
// division are float64 (then rounded to binary32 and to bf16), so the
// normalised GEMM input differs from an exact evaluation only when the
// float64 result sits within a few ulps of a binary32 rounding boundary.
constexpr int kNormThreads = 256;
__device__ __forceinline__ void norm_row(const float* row, int d, double eps,
                                         uint16_t* o, double* red) {
  double ss = 0.0;
  for (int e = threadIdx.x; e < d; e += kNormThreads) {
    const double v = row[e];
    ss = fma(v, v, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
  const double rms = sqrt(tot / (double)d + eps);
  for (int e = threadIdx.x; e < d; e += kNormThreads)
    o[e] = f32_to_bf16((float)((double)row[e] / rms));
}

__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const float* x, int d,
                                                               double eps,
                                                               uint16_t* out) {
  __shared__ double red[kNormThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x;
  norm_row(x + (size_t)m * d, d, eps, out + (size_t)m * d, red);
}

// Embedding gather fused with the first layer's RMSNorm and with the
// (cos, sin) table of the row's position for every rotary pair.
__global__ void __launch_bounds__(kNormThreads) embed_norm_kernel(
    const uint16_t* w_emb, int vocab, int d, const int32_t* last_token,
    const int32_t* drafts, const int32_t* tokens_flat, int q, double eps,
    float* x, uint16_t* out, unsigned* status,
    const int32_t* seq_lens, InvFreq inv_freq, int half,
    float2* rope_tab, int n_rows) {
  __shared__ double red[kNormThreads / 32];
  pdl_trigger();
  pdl_wait();
  if ((int)blockIdx.x >= n_rows) {
    // blocks past the rows: the (cos, sin) table, one (row, pair) per thread,
    // in parallel with the gather and normalisation of the other blocks
    const size_t idx = (size_t)(blockIdx.x - n_rows) * kNormThreads + threadIdx.x;
    if (idx < (size_t)n_rows * half) {
      const int m = (int)(idx / half), j = (int)(idx % half);
      rope_tab[idx] = rope_cs(seq_lens[m / q] + m % q, inv_freq.v[j]);
    }
    return;
  }
  const int m = blockIdx.x;
  const int b = m / q, i = m % q;
  const int tok = tokens_flat ? tokens_flat[m]
                              : ((i == 0) ? last_token[b] : drafts[b * (q - 1) + (i - 1)]);
  float* row = x + (size_t)m * d;
  const bool ok = tok >= 0 && tok < vocab;
  if (!ok && threadIdx.x == 0) flag_status(status, SPEC_DEV_BAD_TOKEN);
  const uint16_t* src = w_emb + (size_t)(ok ? tok : 0) * d;
  for (int e = threadIdx.x; e < d; e += kNormThreads) row[e] = ok ? bf16_to_f32(src[e]) : 0.f;
  __syncthreads();
  norm_row(row, d, eps, out + (size_t)m * d, red);
}

// One warp per sequence: a = number of leading drafts equal to the target's
// argmax (ballot of matches, first zero bit), emit them and target[a], commit
// a+1 positions.
__global__ void accept_kernel(const int32_t* drafts, const int32_t* target,
                              int B, int k, int32_t* seq_lens, int32_t* accept_len,
                              int32_t* emitted, int32_t* last_token, int32_t* copy_ids,
                              float* copy_max, const float* maxv) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const int q = k + 1;
  const int32_t* tg = target + (size_t)b * q;
  const bool match = lane < k && drafts[(size_t)b * k + lane] == tg[lane];
  const unsigned mism = ~__ballot_sync(0xffffffffu, match);   // bit i set: draft i not accepted
  const int a = min(__ffs(mism) - 1, k);
  if (lane < q) {
    int v = -1;
    if (lane < a) v = drafts[(size_t)b * k + lane];
    else if (lane == a) v = tg[a];
    emitted[(size_t)b * q + lane] = v;
    if (copy_ids) copy_ids[(size_t)b * q + lane] = tg[lane];
    if (copy_max) copy_max[(size_t)b * q + lane] = maxv[(size_t)b * q + lane];
  }
  __syncwarp();
  if (lane == 0) {
    accept_len[b] = a;
    last_token[b] = tg[a];
    seq_lens[b] += a + 1;
  }
}

// Drafter step input: row b = [target activation (bf16) || drafter embedding
// of the token] (the GEMM input of the down-projection).  Step 0 reads the
// caller's activation (bf16) and token; later steps the previous step's
// up-projection output (binary32, rounded here) and its argmax token.
// Blocks past the B rows fill the (cos, sin) table of position
// seq_lens[b] + pos_off for every rotary pair, as embed_norm_kernel does.
__global__ void __launch_bounds__(kNormThreads) draft_input_kernel(
    const uint16_t* prev_bf16, const float* prev_f32, int d_model,
    const int32_t* token, const uint16_t* w_emb, int vocab, int d_draft,
    uint16_t* u, unsigned* status, const int32_t* seq_lens, int pos_off,
    InvFreq inv_freq, int half, float2* rope_tab, int B) {
  pdl_trigger();
  pdl_wait();
  if ((int)blockIdx.x >= B) {
    const size_t idx = (size_t)(blockIdx.x - B) * kNormThreads + threadIdx.x;
    if (idx < (size_t)B * half) {
      const int b = (int)(idx / half), j = (int)(idx % half);
      rope_tab[idx] = rope_cs(seq_lens[b] + pos_off, inv_freq.v[j]);
    }
    return;
  }
  const int b = blockIdx.x;
  const int width = d_model + d_draft;
  uint16_t* row = u + (size_t)b * width;
  for (int e = threadIdx.x; e < d_model; e += kNormThreads)
    row[e] = prev_bf16 ? prev_bf16[(size_t)b * d_model + e] : f32_to_bf16(prev_f32[(size_t)b * d_model + e]);
  const int tok = token[b];
  const bool ok = tok >= 0 && tok < vocab;
  if (!ok && threadIdx.x == 0) flag_status(status, SPEC_DEV_BAD_TOKEN);
  const uint16_t* src = w_emb + (size_t)(ok ? tok : 0) * d_draft;
  for (int e = threadIdx.x; e < d_draft; e += kNormThreads) row[d_model + e] = ok ? src[e] : 0;
}

// drafts[b][s] = argmax of step s, draft_max[b][s] its logit
__global__ void draft_collect_kernel(const int32_t* ids, const float* maxv,
                                     int B, int k, int s, int32_t* drafts,
                                     float* draft_max) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  drafts[(size_t)b * k + s] = ids[b];
  if (draft_max) draft_max[(size_t)b * k + s] = maxv[b];
}

// out[i] = bf16(x[i]): a binary32 activation entering a projection
__global__ void to_bf16_kernel(const float* x, size_t n, uint16_t* out) {
  pdl_trigger();
  pdl_wait();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    out[i] = f32_to_bf16(x[i]);
}

}  // namespace

cudaError_t launch_embed_norm(const void* w_emb, int vocab, int d, const int32_t* last_token,
                              const int32_t* drafts, const int32_t* tokens_flat, int B, int q,
                              double eps, float* x, uint16_t* out, unsigned* status,
                              const int32_t* seq_lens, const double* inv_freq, int half,
                              float2* rope_tab, cudaStream_t st) {
  InvFreq f{};
  for (int j = 0; j < half && j < 128; ++j) f.v[j] = inv_freq[j];
  // rows, then as many blocks again for the RoPE table (table blocks <= rows
  // since half <= kNormThreads)
  const int rows = B * q;
  const int tab_blocks = rope_tab ? rows : 0;
  return launch_k(embed_norm_kernel, dim3(rows + tab_blocks), dim3(kNormThreads), 0, st,
                  static_cast<const uint16_t*>(w_emb), vocab, d, last_token, drafts, tokens_flat, q,
                  eps, x, out, status, seq_lens, f, half, rope_tab, rows);
}

__global__ void prefill_commit_kernel(const int32_t* ids, const float* maxv,
                                      int B, int n, int32_t* seq_lens, int32_t* next_token,
                                      float* next_max) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  seq_lens[b] += n;
  next_token[b] = ids[b];
  if (next_max) next_max[b] = maxv[b];
}

cudaError_t launch_prefill_commit(const int32_t* ids, const float* maxv, int B, int n,
                                  int32_t* seq_lens, int32_t* next_token, float* next_max,
                                  cudaStream_t st) {
  return launch_k(prefill_commit_kernel, dim3((B + 127) / 128), dim3(128), 0, st, ids, maxv, B, n,
                  seq_lens, next_token, next_max);
}

cudaError_t launch_rmsnorm(const float* x, int M, int d, double eps, uint16_t* out,
                           cudaStream_t st) {
  return launch_k(rmsnorm_kernel, dim3(M), dim3(kNormThreads), 0, st, x, d, eps, out);
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("SPECVERIFY_NO_PDL");
    return !(v && v[0] == '1');
  }();
  return on;
}

void rope_inv_freq(double base, int head_dim, int n_rot, double* out) {
  for (int j = 0; j < n_rot && j < 128; ++j) out[j] = std::pow(base, -2.0 * j / head_dim);
}

cudaError_t launch_accept(const int32_t* drafts, const int32_t* target, int B, int k,
                          int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                          int32_t* last_token, int32_t* copy_ids, float* copy_max,
                          const float* maxv, cudaStream_t st) {
  const int warps = 4;
  return launch_k(accept_kernel, dim3((B + warps - 1) / warps), dim3(warps * 32), 0, st, drafts,
                  target, B, k, seq_lens, accept_len, emitted, last_token, copy_ids, copy_max, maxv);
}

cudaError_t launch_draft_input(const uint16_t* prev_bf16, const float* prev_f32, int d_model,
                               const int32_t* token, const void* w_emb, int vocab, int d_draft,
                               uint16_t* u, unsigned* status, const int32_t* seq_lens, int pos_off,
                               const double* inv_freq, int half, float2* rope_tab, int B,
                               cudaStream_t st) {
  InvFreq f{};
  for (int j = 0; j < half && j < 128; ++j) f.v[j] = inv_freq[j];
  const int tab_blocks = (B * half + kNormThreads - 1) / kNormThreads;
  return launch_k(draft_input_kernel, dim3(B + tab_blocks), dim3(kNormThreads), 0, st, prev_bf16,
                  prev_f32, d_model, token, static_cast<const uint16_t*>(w_emb), vocab, d_draft, u,
                  status, seq_lens, pos_off, f, half, rope_tab, B);
}

cudaError_t launch_draft_collect(const int32_t* ids, const float* maxv, int B, int k, int s,
                                 int32_t* drafts, float* draft_max, cudaStream_t st) {
  return launch_k(draft_collect_kernel, dim3((B + 127) / 128), dim3(128), 0, st, ids, maxv, B, k, s,
                  drafts, draft_max);
}

cudaError_t launch_to_bf16(const float* x, size_t n, uint16_t* out, cudaStream_t st) {
  const int blocks = (int)std::min<size_t>((n + 255) / 256, 1024);
  return launch_k(to_bf16_kernel, dim3(blocks), dim3(256), 0, st, x, n, out);
}

}  // namespace sv

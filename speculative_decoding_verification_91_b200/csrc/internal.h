// Host-side launchers shared by the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sv {

// ----------------------------------------------------------------- TMA maps
// 2D row-major bf16 tensor [rows][cols], box {box_cols, box_rows}, 128-byte
// swizzle, zero fill outside the tensor.  Returns false if the driver call
// fails (the caller reports SPEC_ECUDA) or the layout is not encodable.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows, uint32_t box_cols, uint64_t row_stride = 0);
// 3D row-major bf16 tensor [d2][d1][d0] (strides in elements), box {b0, b1, b2},
// 128-byte swizzle (b0 * 2 must be 128), zero fill outside the tensor.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2);

// --------------------------------------------------------- streaming GEMM
// Y = X . W^T with X [M][K] bf16 (row-major), W [N][K] bf16 (row-major),
// fp32 accumulation, W streamed once per M-block by TMA.
enum GemmMode { kGemmStore = 0, kGemmResidual = 1, kGemmArgmax = 2, kGemmQkvRope = 3 };

struct GemmPlan {
  int M, N, K;
  int n_tiles;   // ceil(N / 128)
  int kchunks;   // ceil(K / 64)
  int splits;    // split-K factor (1 for argmax)
  int mblocks;   // ceil(M / 64)
  int nt;        // n8 tiles per M-block: ceil(min(M, 64) / 8)
  int x_row_stride = 0;   // elements between X rows (0: K)
};
GemmPlan plan_gemm(int M, int N, int K, int mode);
size_t gemm_partial_floats(const GemmPlan& p);   // split-K partial sums
size_t gemm_argmax_entries(const GemmPlan& p);   // argmax keys (one per row)
int gemm_tickets(const GemmPlan& p, int mode);

// Acceptance fused into the LM-head argmax (B = 0: not fused).
struct AcceptFuse {
  int B = 0, k = 0;
  const int32_t* drafts = nullptr;   // [B][k]
  int32_t* seq_lens = nullptr;
  int32_t* accept_len = nullptr;
  int32_t* emitted = nullptr;        // [B][k+1]
  int32_t* last_token = nullptr;
  int32_t* copy_ids = nullptr;       // optional copies of every row's argmax / logit
  float* copy_max = nullptr;
};

// RoPE + cache append fused into the QKV projection's epilogue: the last CTA
// to finish a head (all its splits and column tiles) rotates each pair and
// writes queries (workspace), keys / values / side-band (cache pools).
struct RopeFuse {
  int n_q_heads = 0, n_kv_heads = 0, head_dim = 0, n_rot = 0, q = 0;
  int page_size = 0, num_pages = 0, max_pages = 0;
  const int32_t* seq_lens = nullptr;
  const int32_t* block_table = nullptr;
  const float2* rope_tab = nullptr;  // [M][head_dim/2] (cos, sin) of each row's position
  uint16_t* q_out = nullptr;         // [M][Hq][D]
  uint16_t* k_pool = nullptr;
  uint16_t* v_pool = nullptr;        // null on key-equals-value layers
  uint16_t* ksb_pool = nullptr;      // key-equals-value side-band
};

struct GemmBuffers {
  float* out;          // kGemmStore: [M][N]; kGemmResidual: [M][N] updated in place
  float* partial;      // gemm_partial_floats()
  unsigned long long* arg_keys;   // gemm_argmax_entries() keys, zero on entry and exit
  int32_t* ids;        // kGemmArgmax: [M]
  float* maxv;         // kGemmArgmax: [M] or null
  unsigned* tickets;   // gemm_tickets() counters, zero on entry, zero on exit
  unsigned* status;
  AcceptFuse acc;      // kGemmArgmax with a single M-block only
  RopeFuse rope;       // kGemmQkvRope
  int* accept_fused;   // set by the launcher: 1 if the argmax kernel runs the acceptance
};
cudaError_t launch_gemm(const GemmPlan& p, int mode, const void* x, const void* w,
                        const GemmBuffers& buf, cudaStream_t st);
// The same GEMMs on tcgen05 / TMEM for 32 < M <= 256 rows: every row sits in
// the MMA's N dimension, so the weights stream once.  tc_supported() is false
// outside that range (SPECVERIFY_TC_MIN_ROWS moves the lower bound) or when
// SPECVERIFY_NO_TC=1.
bool tc_supported(int M);
int tc_np(int M);        // rows per tensor-memory block (M rounded up to 16, at most 256)
int tc_mblocks(int M);   // blocks of 256 rows
int tc_ldp(int M);       // row stride of its split-K partials
cudaError_t launch_gemm_tc(const GemmPlan& p, int mode, const void* x, const void* w,
                           const GemmBuffers& buf, cudaStream_t st);
// tcgen05 path when it applies, else the mma.sync path
inline cudaError_t launch_gemm_any(const GemmPlan& p, int mode, const void* x, const void* w,
                                   const GemmBuffers& buf, cudaStream_t st) {
  return tc_supported(p.M) ? launch_gemm_tc(p, mode, x, w, buf, st)
                           : launch_gemm(p, mode, x, w, buf, st);
}

// ------------------------------------------------------------- small kernels
cudaError_t launch_draft_input(const uint16_t* prev_bf16, const float* prev_f32, int d_model,
                               const int32_t* token, const void* w_emb, int vocab, int d_draft,
                               uint16_t* u, unsigned* status, const int32_t* seq_lens, int pos_off,
                               const double* inv_freq, int half, float2* rope_tab, int B,
                               cudaStream_t st);
cudaError_t launch_draft_collect(const int32_t* ids, const float* maxv, int B, int k, int s,
                                 int32_t* drafts, float* draft_max, cudaStream_t st);
// Cheap unembedding over token clusters (cluster.cu).
struct ClusterArgs {
  int n_clusters, cluster_size, n_select;
  const void* centroids;          // bf16 [C][d]
  const int32_t* cluster_tokens;  // [C][S], -1 pads
  const void* w_clustered;        // bf16 [C*S][d]
};
size_t cluster_logit_floats(int M, int C);
cudaError_t launch_cluster_unembed(const ClusterArgs& t, const uint16_t* h, int M, int d,
                                   int32_t* ids, float* maxv, float* cl_logits, int32_t* sel,
                                   unsigned long long* keys, const GemmBuffers& gb, cudaStream_t st);
// Sampled verification tail (sampled.cu): softmax statistics, acceptance,
// Gumbel-max draw, commit.
cudaError_t launch_sampled_tail(int B, int k, int V, float T, const float* lt, const float* ld,
                                float2* st_t, float2* st_d, const int32_t* drafts, const float* u,
                                const float* g, int32_t* a_arr, unsigned long long* keys,
                                int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                                int32_t* new_last, unsigned* status, cudaStream_t st);
cudaError_t launch_to_bf16(const float* x, size_t n, uint16_t* out, cudaStream_t st);
cudaError_t launch_rmsnorm(const float* x, int M, int d, double eps, uint16_t* out,
                           cudaStream_t st);
// embedding gather of [last_token, drafts] into x and its RMSNorm into out;
// also the (cos, sin) table of every row's position for pairs j < half
// (rope_tab [B*q][half], theta_j = inv_freq[j]); rope_tab may be null
// Row m = b*q + i takes tokens_flat[m] when tokens_flat is set (prefill), else
// last_token[b] (i = 0) / drafts[b][i-1] (verify).
cudaError_t launch_embed_norm(const void* w_emb, int vocab, int d, const int32_t* last_token,
                              const int32_t* drafts, const int32_t* tokens_flat, int B, int q,
                              double eps, float* x, uint16_t* out, unsigned* status,
                              const int32_t* seq_lens, const double* inv_freq, int half,
                              float2* rope_tab, cudaStream_t st);
// Prefill commit: seq_lens[b] += n; next_token[b] = ids[b]; next_max[b] = maxv[b] (if set).
cudaError_t launch_prefill_commit(const int32_t* ids, const float* maxv, int B, int n,
                                  int32_t* seq_lens, int32_t* next_token, float* next_max,
                                  cudaStream_t st);
// host: theta_j = base^(-2j/D) for j < n_rot (n_rot <= 128)
void rope_inv_freq(double base, int head_dim, int n_rot, double* out);
cudaError_t launch_accept(const int32_t* drafts, const int32_t* target, int B, int k,
                          int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                          int32_t* last_token, int32_t* copy_ids, float* copy_max,
                          const float* maxv, cudaStream_t st);

// ------------------------------------------------------- RoPE + cache append
struct RopeAppend {
  // geometry
  int n_q_heads, n_kv_heads, head_dim, n_rot;   // n_rot rotated pairs
  double inv_freq[128];                         // theta_j = base^(-2j/D), j < n_rot
  int page_size, num_pages, max_pages;
  // rows: blockIdx.x = i in [0, n_rows), blockIdx.y = sequence b
  int n_rows;
  const int32_t* seq_lens;   // position of row i = seq_lens[b] + i   (if non-null)
  int pos0;                  // ... else pos0 + i
  const int32_t* block_table;
  // sources (pre-RoPE), element strides in elements
  const void* src_q; long q_row_stride, q_seq_stride;   // null: no queries
  const void* src_k; long k_row_stride, k_seq_stride;
  const void* src_v; long v_row_stride, v_seq_stride;   // null on key-equals-value layers
  int src_is_f32;
  // destinations
  uint16_t* q_out;           // [B][n_rows][Hq][D] bf16 rotated queries
  uint16_t* k_pool;
  uint16_t* v_pool;
  uint16_t* ksb_pool;        // key-equals-value side-band
  unsigned* status;
};
cudaError_t launch_rope_append(const RopeAppend& a, int B, cudaStream_t st);

// ---------------------------------------------------------- split-KV attention
constexpr int kMaxSplits = 1024;   // splits one combine can merge
struct AttnGeom {
  int B, q, n_q_heads, n_kv_heads, head_dim, page_size, num_pages, max_pages;
  int window, kv_equal, sb_width, split_tokens;
  int n_splits_grid;   // CTAs per (sequence, kv head, row block)
  int rows;            // G * q
  int qpos_off;        // row i at position L + qpos_off + i (verify: 0)
  int kend_off;        // last visible cached key at L + kend_off (verify: q - 1)
  int row_blocks;      // ceil(rows / 64)
};
AttnGeom plan_attn(int B, int q, int Hq, int Hkv, int D, int page, int num_pages, int max_pages,
                   int window, int kv_equal, int sb_width, int split_tokens);
size_t attn_partial_floats(const AttnGeom& g);
bool attn_tc_supported(const AttnGeom& g);
cudaError_t launch_attn_tc(const AttnGeom& g, const CUtensorMap& tk, const CUtensorMap& tv,
                           const uint16_t* qrot, const int32_t* block_table, const int32_t* seq_lens,
                           float* part_o, float* part_ml, unsigned* status, float scale_log2,
                           cudaStream_t st);
cudaError_t launch_attention(const AttnGeom& g, const uint16_t* qrot, const void* k_pool,
                             const void* v_pool, const void* ksb_pool, const int32_t* block_table,
                             const int32_t* seq_lens, float* part, uint16_t* out, unsigned* status,
                             cudaStream_t st, void (*mark)(cudaStream_t) = nullptr);

}  // namespace sv

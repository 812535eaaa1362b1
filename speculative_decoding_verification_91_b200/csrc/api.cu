// C ABI of the verify step: argument validation, workspace layout, launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cstdlib>
#include <cmath>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/specverify.h"
#include "common.cuh"
#include "internal.h"

namespace sv {

std::atomic<unsigned long long> g_launch_count{0};
void count_launch() { g_launch_count.fetch_add(1, std::memory_order_relaxed); }

// ------------------------------------------------------------------ TMA maps
namespace {
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);
EncodeFn g_encode = nullptr;
std::once_flag g_encode_once;

void resolve_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeFn>(fn);
}
}  // namespace

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows, uint32_t box_cols, uint64_t row_stride) {
  std::call_once(g_encode_once, resolve_encode);
  if (!g_encode || !base) return false;
  if (row_stride == 0) row_stride = cols;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_stride * 2) % 16 || box_cols * 2 > 128 ||
      row_stride < cols)
    return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2) {
  std::call_once(g_encode_once, resolve_encode);
  if (!g_encode || !base) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (stride1 * 2) % 16 || (stride2 * 2) % 16 ||
      b0 * 2 != 128 || b1 < 1 || b1 > 256 || b2 < 1 || b2 > 256)
    return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1 * 2, stride2 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int n_rot_of(const spec_model* m, const spec_layer& L) {
  return (int)lrintf(L.rope_fraction * (float)m->head_dim / 2.0f);
}

int split_of(const spec_model* m, const spec_layer& L) {
  return L.split_tokens > 0 ? L.split_tokens : m->split_tokens;
}

int qkv_out(const spec_model* m, const spec_layer& L) {
  return (m->n_q_heads + m->n_kv_heads + (L.kv_equal ? 0 : m->n_kv_heads)) * m->head_dim;
}

int check_model(const spec_model* m) {
  if (!m || !m->layers || !m->w_lm || !m->w_embed) return SPEC_EINVAL;
  if (m->n_layers < 1 || m->d_model < 8 || m->d_model % 8 || m->n_q_heads < 1 || m->n_kv_heads < 1 ||
      m->n_q_heads % m->n_kv_heads || m->vocab < 1 || m->num_pages < 1)
    return SPEC_EINVAL;
  if (m->page_size != SPEC_PAGE_SIZE) return SPEC_EUNSUPPORTED;
  if (m->head_dim != 128 && m->head_dim != 256) return SPEC_EUNSUPPORTED;
  if (m->split_tokens < m->page_size || m->split_tokens % m->page_size) return SPEC_EINVAL;
  if (!(m->rope_theta > 0.0) || !(m->rms_eps >= 0.0)) return SPEC_EINVAL;
  if ((uint64_t)m->num_pages * m->n_kv_heads * m->page_size > 0x7fffffffull) return SPEC_EUNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(m->w_lm) & 15) return SPEC_EINVAL;
  for (int l = 0; l < m->n_layers; ++l) {
    const spec_layer& L = m->layers[l];
    if (!L.w_qkv || !L.w_o || !L.k_pool) return SPEC_EINVAL;
    if (L.window < 0) return SPEC_EINVAL;
    if (L.split_tokens < 0 || L.split_tokens % m->page_size) return SPEC_EINVAL;
    if (!(L.rope_fraction >= 0.f && L.rope_fraction <= 1.f)) return SPEC_EINVAL;
    const int nr = n_rot_of(m, L);
    if (L.kv_equal) {
      if (!L.ksb_pool || L.v_pool) return SPEC_EINVAL;
      if (2 * nr != 64) return SPEC_EUNSUPPORTED;   // side-band tile is 64 wide
    } else if (!L.v_pool) {
      return SPEC_EINVAL;
    }
    const void* ptrs[5] = {L.w_qkv, L.w_o, L.k_pool, L.v_pool, L.ksb_pool};
    for (const void* p : ptrs)
      if (reinterpret_cast<uintptr_t>(p) & 15) return SPEC_EINVAL;
  }
  return SPEC_OK;
}

// Workspace layout of one forward over q rows per sequence (q = k + 1 for a
// verify step, q = n for a prefill chunk) for (B, q, max_pages).
struct StepLayout {
  size_t x, hn, qrot, attn_out, attn_part, gemm_part, arg_keys, ids, maxv, rope_tab,
      total;
  int tickets;
  bool splits_ok;   // every layer's split count fits the combine kernel
};

StepLayout step_layout(const spec_model* m, int B, int q, int max_pages) {
  StepLayout s{};
  s.splits_ok = true;
  const int M = B * q, d = m->d_model, D = m->head_dim;
  size_t attn_floats = 0, gemm_floats = 0;
  int tickets = 0;
  for (int l = 0; l < m->n_layers; ++l) {
    const spec_layer& L = m->layers[l];
    AttnGeom g = plan_attn(B, q, m->n_q_heads, m->n_kv_heads, D, m->page_size, m->num_pages,
                           max_pages, L.window, L.kv_equal, 2 * n_rot_of(m, L), split_of(m, L));
    attn_floats = std::max(attn_floats, attn_partial_floats(g));
    if (g.n_splits_grid > kMaxSplits) s.splits_ok = false;
    GemmPlan pq = plan_gemm(M, qkv_out(m, L), d, kGemmQkvRope);
    GemmPlan po = plan_gemm(M, d, m->n_q_heads * D, kGemmResidual);
    gemm_floats = std::max({gemm_floats, gemm_partial_floats(pq), gemm_partial_floats(po)});
    tickets = std::max({tickets, gemm_tickets(pq, kGemmQkvRope), gemm_tickets(po, kGemmResidual)});
  }
  GemmPlan pl = plan_gemm(M, m->vocab, d, kGemmArgmax);
  tickets = std::max(tickets, pl.mblocks);
  size_t off = kWsHeaderBytes;
  s.x = off;         off = up(off + (size_t)M * d * 4);
  s.hn = off;        off = up(off + (size_t)M * d * 2);
  s.qrot = off;      off = up(off + (size_t)M * m->n_q_heads * D * 2);
  s.attn_out = off;  off = up(off + (size_t)M * m->n_q_heads * D * 2);
  s.attn_part = off; off = up(off + attn_floats * 4);
  s.gemm_part = off; off = up(off + gemm_floats * 4);
  s.arg_keys = off;  off = up(off + gemm_argmax_entries(pl) * 8);
  s.ids = off;       off = up(off + (size_t)M * 4);
  s.maxv = off;      off = up(off + (size_t)M * 4);
  s.rope_tab = off;  off = up(off + (size_t)M * (D / 2) * 8);
  s.total = off;
  s.tickets = tickets;
  return s;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SPEC_OK : SPEC_ECUDA; }

// Profiling events: per recorded step {step start, LM-head start, LM-head
// stop, step stop}.
struct Prof {
  std::vector<cudaEvent_t> ev;
  int n = 0, used = 0;
  bool on = false;
};
Prof g_prof;
inline void prof_mark(int which, cudaStream_t st) {
  if (g_prof.on && g_prof.used < g_prof.n) cudaEventRecord(g_prof.ev[4 * g_prof.used + which], st);
}
inline void prof_step_done() {
  if (g_prof.on && g_prof.used < g_prof.n) ++g_prof.used;
}
// Per-launch timing of one step (diagnostics): an event after every launch.
struct ProfDetail {
  std::vector<cudaEvent_t> ev;
  int used = 0;
  bool on = false;
};
ProfDetail g_detail;
inline void detail_mark(cudaStream_t st) {
  if (g_detail.on && g_detail.used < (int)g_detail.ev.size())
    cudaEventRecord(g_detail.ev[g_detail.used++], st);
}

void prof_release() {
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.n = g_prof.used = 0;
  g_prof.on = false;
}

// Inputs and outputs of one forward: a verify step (last_token/drafts ->
// acceptance outputs) or a prefill chunk (tokens -> next_token).
struct ForwardIo {
  const int32_t* last_token = nullptr;
  const int32_t* drafts = nullptr;
  int32_t* accept_len = nullptr;
  int32_t* emitted = nullptr;
  int32_t* new_last_token = nullptr;
  int32_t* target_ids = nullptr;
  float* target_maxlogit = nullptr;
  const int32_t* tokens = nullptr;     // prefill: [B][q]
  int32_t* next_token = nullptr;       // prefill: [B]
  float* next_maxlogit = nullptr;
  float* logits = nullptr;             // sampled verify: LM head writes [M][V] logits, no argmax
  float* logits_part = nullptr;        //   and its split-K partials (tensor-memory path)
};

// embed -> per layer (RMSNorm, QKV + RoPE + cache append, split-KV attention,
// O-proj + residual) -> final RMSNorm -> LM head argmax -> acceptance (verify)
// or commit of all q rows (prefill).
int run_forward(const spec_model* m, const int32_t* block_table, int max_pages, int B, int q,
                int32_t* seq_lens, const ForwardIo& io, void* ws, size_t ws_bytes,
                cudaStream_t st) {
  const bool prefill = io.tokens != nullptr;
  StepLayout s = step_layout(m, B, q, max_pages);
  if (s.tickets > kMaxTickets || !s.splits_ok) return SPEC_EUNSUPPORTED;
  if (ws_bytes < s.total) return SPEC_EINVAL;
  WsHeader hdr = ws_header(ws);
  const int k = q - 1, M = B * q, d = m->d_model, D = m->head_dim;
  float* x = at<float>(ws, s.x);
  uint16_t* hn = at<uint16_t>(ws, s.hn);
  uint16_t* qrot = at<uint16_t>(ws, s.qrot);
  uint16_t* attn_out = at<uint16_t>(ws, s.attn_out);
  int rc;

  prof_mark(0, st);
  detail_mark(st);
  double inv_freq[128];
  rope_inv_freq(m->rope_theta, D, D / 2, inv_freq);
  float2* rope_tab = at<float2>(ws, s.rope_tab);
  rc = cuda_status(launch_embed_norm(m->w_embed, m->vocab, d, io.last_token, io.drafts, io.tokens,
                                     B, q, m->rms_eps, x, hn, hdr.status, seq_lens, inv_freq, D / 2,
                                     rope_tab, st));
  if (rc) return rc;
  detail_mark(st);
  for (int l = 0; l < m->n_layers; ++l) {
    const spec_layer& L = m->layers[l];
    const int nqkv = qkv_out(m, L);
    if (l > 0) {
      rc = cuda_status(launch_rmsnorm(x, M, d, m->rms_eps, hn, st));
      if (rc) return rc;
      detail_mark(st);
    }
    // QKV projection with RoPE and the cache append in its epilogue
    GemmPlan pq = plan_gemm(M, nqkv, d, kGemmQkvRope);
    GemmBuffers bq{};
    bq.partial = at<float>(ws, s.gemm_part);
    bq.tickets = hdr.tickets;
    bq.status = hdr.status;
    RopeFuse& f = bq.rope;
    f.n_q_heads = m->n_q_heads;
    f.n_kv_heads = m->n_kv_heads;
    f.head_dim = D;
    f.n_rot = n_rot_of(m, L);
    f.q = q;
    f.page_size = m->page_size;
    f.num_pages = m->num_pages;
    f.max_pages = max_pages;
    f.seq_lens = seq_lens;
    f.block_table = block_table;
    f.rope_tab = rope_tab;
    f.q_out = qrot;
    f.k_pool = static_cast<uint16_t*>(L.k_pool);
    f.v_pool = static_cast<uint16_t*>(L.v_pool);
    f.ksb_pool = static_cast<uint16_t*>(L.ksb_pool);
    rc = cuda_status(launch_gemm_any(pq, kGemmQkvRope, hn, L.w_qkv, bq, st));
    if (rc) return rc;
    detail_mark(st);
    AttnGeom g = plan_attn(B, q, m->n_q_heads, m->n_kv_heads, D, m->page_size, m->num_pages,
                           max_pages, L.window, L.kv_equal, 2 * f.n_rot, split_of(m, L));
    rc = cuda_status(launch_attention(g, qrot, L.k_pool, L.v_pool, L.ksb_pool, block_table, seq_lens,
                                      at<float>(ws, s.attn_part), attn_out, hdr.status, st,
                                      g_detail.on ? detail_mark : nullptr));
    if (rc) return rc;
    detail_mark(st);
    GemmPlan po = plan_gemm(M, d, m->n_q_heads * D, kGemmResidual);
    GemmBuffers bo{};
    bo.out = x;
    bo.partial = at<float>(ws, s.gemm_part);
    bo.tickets = hdr.tickets;
    bo.status = hdr.status;
    rc = cuda_status(launch_gemm_any(po, kGemmResidual, attn_out, L.w_o, bo, st));
    if (rc) return rc;
    detail_mark(st);
  }
  rc = cuda_status(launch_rmsnorm(x, M, d, m->rms_eps, hn, st));
  if (rc) return rc;
  detail_mark(st);
  // LM head: every row (verify) or each sequence's last row (prefill)
  GemmPlan pl = plan_gemm(prefill ? B : M, m->vocab, d, kGemmArgmax);
  GemmBuffers bl{};
  bl.arg_keys = at<unsigned long long>(ws, s.arg_keys);
  bl.ids = at<int32_t>(ws, s.ids);
  bl.maxv = at<float>(ws, s.maxv);
  bl.tickets = hdr.tickets;
  bl.status = hdr.status;
  const uint16_t* lm_x = hn;
  if (prefill) {
    pl.x_row_stride = q * d;
    lm_x = hn + (size_t)(q - 1) * d;
  } else {
    bl.acc.B = B;
    bl.acc.k = k;
    bl.acc.drafts = io.drafts;
    bl.acc.seq_lens = seq_lens;
    bl.acc.accept_len = io.accept_len;
    bl.acc.emitted = io.emitted;
    bl.acc.last_token = io.new_last_token;
    bl.acc.copy_ids = io.target_ids;
    bl.acc.copy_max = io.target_maxlogit;
  }
  prof_mark(1, st);
  if (io.logits) {     // sampled verification: binary32 logits of every row
    GemmBuffers bs{};
    bs.out = io.logits;
    bs.partial = io.logits_part;
    bs.tickets = hdr.tickets;
    bs.status = hdr.status;
    rc = cuda_status(launch_gemm_any(plan_gemm(M, m->vocab, d, kGemmStore), kGemmStore, hn, m->w_lm,
                                     bs, st));
    prof_mark(2, st);
    prof_mark(3, st);
    detail_mark(st);
    g_detail.on = false;
    prof_step_done();
    return rc;
  }
  int fused = 0;
  bl.accept_fused = &fused;
  rc = cuda_status(launch_gemm_any(pl, kGemmArgmax, lm_x, m->w_lm, bl, st));
  prof_mark(2, st);
  detail_mark(st);
  if (rc) return rc;
  if (prefill) {
    rc = cuda_status(launch_prefill_commit(at<int32_t>(ws, s.ids), at<float>(ws, s.maxv), B, q,
                                           seq_lens, io.next_token, io.next_maxlogit, st));
  } else if (!fused) {
    // the LM head runs the acceptance itself when all rows share one block
    rc = cuda_status(launch_accept(io.drafts, at<int32_t>(ws, s.ids), B, k, seq_lens, io.accept_len,
                                   io.emitted, io.new_last_token, io.target_ids,
                                   io.target_maxlogit, at<float>(ws, s.maxv), st));
  }
  prof_mark(3, st);
  detail_mark(st);
  g_detail.on = false;
  prof_step_done();
  return rc;
}

// ---------------------------------------------------------- sampled verify

struct SampledLayout {
  StepLayout s;
  size_t logits, part, st_t, st_d, a, keys, total;
  int tickets;
};
SampledLayout sampled_layout(const spec_model* m, int B, int k, int max_pages) {
  SampledLayout L{};
  L.s = step_layout(m, B, k + 1, max_pages);
  const int M = B * (k + 1), V = m->vocab;
  GemmPlan pl = plan_gemm(M, V, m->d_model, kGemmStore);
  size_t off = L.s.total;
  L.logits = off; off = up(off + (size_t)M * V * 4);
  L.part = off;   off = up(off + ((pl.splits > 1 || tc_supported(M)) ? gemm_partial_floats(pl) : 0) * 4);
  L.st_t = off;   off = up(off + (size_t)M * 8);
  L.st_d = off;   off = up(off + (size_t)B * std::max(k, 1) * 8);
  L.a = off;      off = up(off + (size_t)B * 4);
  L.keys = off;   off = up(off + (size_t)B * 8);
  L.total = off;
  L.tickets = std::max(L.s.tickets, gemm_tickets(pl, kGemmStore));
  return L;
}

// ---------------------------------------------------------------- clusters

constexpr int kMaxClusterCount = 8192;   // keys of one row sorted in shared memory

int check_clusters(const spec_clusters* t, int d) {
  if (!t || !t->centroids || !t->cluster_tokens || !t->w_clustered) return SPEC_EINVAL;
  if (t->n_clusters < 1 || t->cluster_size < 1 || t->n_select < 1 || t->n_select > t->n_clusters)
    return SPEC_EINVAL;
  if (t->n_clusters > kMaxClusterCount || t->cluster_size > 4096) return SPEC_EUNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(t->centroids) & 15) || (reinterpret_cast<uintptr_t>(t->w_clustered) & 15))
    return SPEC_EINVAL;
  if (d < 8 || d % 8) return SPEC_EINVAL;
  return SPEC_OK;
}

ClusterArgs cluster_args(const spec_clusters* t) {
  ClusterArgs c{};
  c.n_clusters = t->n_clusters;
  c.cluster_size = t->cluster_size;
  c.n_select = t->n_select;
  c.centroids = t->centroids;
  c.cluster_tokens = t->cluster_tokens;
  c.w_clustered = t->w_clustered;
  return c;
}

// Scratch of one cheap unembedding of M rows: cluster logits, the centroid
// GEMM's split-K partials, the selected clusters, the per-row argmax keys.
struct ClusterLayout {
  size_t logits, part, sel, keys, bytes;
  int tickets;
};
ClusterLayout cluster_layout(int M, int d, const spec_clusters* t, size_t base) {
  ClusterLayout c{};
  GemmPlan p = plan_gemm(M, t->n_clusters, d, kGemmStore);
  size_t off = base;
  c.logits = off; off = up(off + cluster_logit_floats(M, t->n_clusters) * 4);
  c.part = off;   off = up(off + gemm_partial_floats(p) * 4);
  c.sel = off;    off = up(off + (size_t)M * t->n_select * 4);
  c.keys = off;   off = up(off + (size_t)M * 8);
  c.bytes = off - base;
  c.tickets = gemm_tickets(p, kGemmStore);
  return c;
}

cudaError_t run_clusters(const spec_clusters* t, const uint16_t* h, int M, int d, int32_t* ids,
                         float* maxv, void* ws, const ClusterLayout& c, cudaStream_t st) {
  WsHeader hdr = ws_header(ws);
  GemmBuffers b{};
  b.partial = at<float>(ws, c.part);
  b.tickets = hdr.tickets;
  b.status = hdr.status;
  return launch_cluster_unembed(cluster_args(t), h, M, d, ids, maxv, at<float>(ws, c.logits),
                                at<int32_t>(ws, c.sel), at<unsigned long long>(ws, c.keys), b, st);
}

// ---------------------------------------------------------------- drafter

int check_drafter(const spec_model* m, const spec_drafter* d) {
  if (!d || !d->blocks || !d->w_embed || !d->w_down || !d->w_up) return SPEC_EINVAL;
  if (d->d_draft < 8 || d->d_draft % 8 || d->n_q_heads < 1 || d->n_q_heads % m->n_kv_heads ||
      d->n_blocks < 1 || d->n_blocks > 16)
    return SPEC_EINVAL;
  const void* ptrs[3] = {d->w_embed, d->w_down, d->w_up};
  for (const void* p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 15) return SPEC_EINVAL;
  if (d->clusters) {
    const int rc = check_clusters(d->clusters, m->d_model);
    if (rc) return rc;
  }
  for (int i = 0; i < d->n_blocks; ++i) {
    const spec_draft_block& b = d->blocks[i];
    if (!b.w_q || !b.w_o || b.target_layer < 0 || b.target_layer >= m->n_layers) return SPEC_EINVAL;
    if ((reinterpret_cast<uintptr_t>(b.w_q) & 15) || (reinterpret_cast<uintptr_t>(b.w_o) & 15))
      return SPEC_EINVAL;
  }
  return SPEC_OK;
}

// Workspace of one drafter call for B sequences (q = 1 row each).
struct DraftLayout {
  size_t u, x, hn, qrot, attn_out, attn_part, gemm_part, h, arg_keys, ids, maxv, rope_tab, total;
  ClusterLayout cl;
  int tickets;
  bool splits_ok;
};

DraftLayout draft_layout(const spec_model* m, const spec_drafter* d, int B, int max_pages) {
  DraftLayout s{};
  s.splits_ok = true;
  const int D = m->head_dim, dm = m->d_model, dd = d->d_draft, nq = d->n_q_heads * D;
  size_t attn = 0;
  for (int i = 0; i < d->n_blocks; ++i) {
    const spec_layer& L = m->layers[d->blocks[i].target_layer];
    AttnGeom g = plan_attn(B, 1, d->n_q_heads, m->n_kv_heads, D, m->page_size, m->num_pages,
                           max_pages, L.window, L.kv_equal, 2 * n_rot_of(m, L), split_of(m, L));
    attn = std::max(attn, attn_partial_floats(g));
    if (g.n_splits_grid > kMaxSplits) s.splits_ok = false;
  }
  const int modes[4] = {kGemmStore, kGemmQkvRope, kGemmResidual, kGemmStore};
  const GemmPlan ps[4] = {plan_gemm(B, dd, dm + dd, modes[0]), plan_gemm(B, nq, dd, modes[1]),
                          plan_gemm(B, dd, nq, modes[2]), plan_gemm(B, dm, dd, modes[3])};
  size_t gp = 0;
  int tickets = plan_gemm(B, m->vocab, dm, kGemmArgmax).mblocks;
  for (int i = 0; i < 4; ++i) {
    gp = std::max(gp, gemm_partial_floats(ps[i]));
    tickets = std::max(tickets, gemm_tickets(ps[i], modes[i]));
  }
  size_t off = kWsHeaderBytes;
  s.u = off;         off = up(off + (size_t)B * (dm + dd) * 2);
  s.x = off;         off = up(off + (size_t)B * dd * 4);
  s.hn = off;        off = up(off + (size_t)B * std::max(dd, dm) * 2);
  s.qrot = off;      off = up(off + (size_t)B * nq * 2);
  s.attn_out = off;  off = up(off + (size_t)B * nq * 2);
  s.attn_part = off; off = up(off + attn * 4);
  s.gemm_part = off; off = up(off + gp * 4);
  s.h = off;         off = up(off + (size_t)B * dm * 4);
  s.arg_keys = off;  off = up(off + (size_t)B * 8);
  s.ids = off;       off = up(off + (size_t)B * 4);
  s.maxv = off;      off = up(off + (size_t)B * 4);
  s.rope_tab = off;  off = up(off + (size_t)B * (D / 2) * 8);
  if (d->clusters) {
    s.cl = cluster_layout(B, dm, d->clusters, off);
    off += s.cl.bytes;
    tickets = std::max(tickets, s.cl.tickets);
  }
  s.total = off;
  s.tickets = tickets;
  return s;
}

// k drafter steps: [activation || embedding] -> down -> blocks (RMSNorm, query
// projection + RoPE at position L + s, cross-attention over the target
// layer's cache, output projection + residual) -> bf16 -> up -> final RMSNorm
// -> LM head argmax -> drafts[:, s].
int run_draft(const spec_model* m, const spec_drafter* d, const int32_t* block_table, int max_pages,
              const int32_t* seq_lens, const void* prev_hidden, const int32_t* prev_token, int B, int k,
              int32_t* drafts, float* draft_max, void* ws, size_t ws_bytes, cudaStream_t st) {
  DraftLayout s = draft_layout(m, d, B, max_pages);
  if (s.tickets > kMaxTickets || !s.splits_ok) return SPEC_EUNSUPPORTED;
  if (ws_bytes < s.total) return SPEC_EINVAL;
  WsHeader hdr = ws_header(ws);
  const int D = m->head_dim, dm = m->d_model, dd = d->d_draft, nq = d->n_q_heads * D, half = D / 2;
  uint16_t* u = at<uint16_t>(ws, s.u);
  float* x = at<float>(ws, s.x);
  uint16_t* hn = at<uint16_t>(ws, s.hn);
  uint16_t* qrot = at<uint16_t>(ws, s.qrot);
  uint16_t* attn_out = at<uint16_t>(ws, s.attn_out);
  float* h = at<float>(ws, s.h);
  int32_t* ids = at<int32_t>(ws, s.ids);
  float* maxv = at<float>(ws, s.maxv);
  float2* rope_tab = at<float2>(ws, s.rope_tab);
  double inv_freq[128];
  rope_inv_freq(m->rope_theta, D, half, inv_freq);
  auto bufs = [&]() {
    GemmBuffers b{};
    b.partial = at<float>(ws, s.gemm_part);
    b.tickets = hdr.tickets;
    b.status = hdr.status;
    return b;
  };
  int rc;
  for (int step = 0; step < k; ++step) {
    rc = cuda_status(launch_draft_input(step == 0 ? static_cast<const uint16_t*>(prev_hidden) : nullptr,
                                        step == 0 ? nullptr : h, dm, step == 0 ? prev_token : ids,
                                        d->w_embed, m->vocab, dd, u, hdr.status, seq_lens, step,
                                        inv_freq, half, rope_tab, B, st));
    if (rc) return rc;
    GemmBuffers bd = bufs();
    bd.out = x;
    rc = cuda_status(launch_gemm_any(plan_gemm(B, dd, dm + dd, kGemmStore), kGemmStore, u, d->w_down, bd, st));
    if (rc) return rc;
    for (int i = 0; i < d->n_blocks; ++i) {
      const spec_draft_block& blk = d->blocks[i];
      const spec_layer& L = m->layers[blk.target_layer];
      rc = cuda_status(launch_rmsnorm(x, B, dd, m->rms_eps, hn, st));
      if (rc) return rc;
      GemmBuffers bq = bufs();
      RopeFuse& f = bq.rope;
      f.n_q_heads = d->n_q_heads;     // every projected head is a query head: the cache is not written
      f.n_kv_heads = m->n_kv_heads;
      f.head_dim = D;
      f.n_rot = n_rot_of(m, L);
      f.q = 1;
      f.page_size = m->page_size;
      f.num_pages = m->num_pages;
      f.max_pages = max_pages;
      f.seq_lens = seq_lens;
      f.block_table = block_table;
      f.rope_tab = rope_tab;
      f.q_out = qrot;
      rc = cuda_status(launch_gemm_any(plan_gemm(B, nq, dd, kGemmQkvRope), kGemmQkvRope, hn, blk.w_q, bq, st));
      if (rc) return rc;
      AttnGeom g = plan_attn(B, 1, d->n_q_heads, m->n_kv_heads, D, m->page_size, m->num_pages,
                             max_pages, L.window, L.kv_equal, 2 * f.n_rot, split_of(m, L));
      g.qpos_off = step;   // the query sits at L + step ...
      g.kend_off = -1;     // ... over the cached keys j < L
      rc = cuda_status(launch_attention(g, qrot, L.k_pool, L.v_pool, L.ksb_pool, block_table, seq_lens,
                                        at<float>(ws, s.attn_part), attn_out, hdr.status, st));
      if (rc) return rc;
      GemmBuffers bo = bufs();
      bo.out = x;
      rc = cuda_status(launch_gemm_any(plan_gemm(B, dd, nq, kGemmResidual), kGemmResidual, attn_out, blk.w_o, bo, st));
      if (rc) return rc;
    }
    rc = cuda_status(launch_to_bf16(x, (size_t)B * dd, hn, st));
    if (rc) return rc;
    GemmBuffers bu = bufs();
    bu.out = h;
    rc = cuda_status(launch_gemm_any(plan_gemm(B, dm, dd, kGemmStore), kGemmStore, hn, d->w_up, bu, st));
    if (rc) return rc;
    rc = cuda_status(launch_rmsnorm(h, B, dm, m->rms_eps, hn, st));
    if (rc) return rc;
    if (d->clusters) {         // cheap unembedding over the best token clusters
      rc = cuda_status(run_clusters(d->clusters, hn, B, dm, ids, maxv, ws, s.cl, st));
    } else {                   // the target's full LM head
      GemmBuffers bl = bufs();
      bl.arg_keys = at<unsigned long long>(ws, s.arg_keys);
      bl.ids = ids;
      bl.maxv = maxv;
      rc = cuda_status(launch_gemm_any(plan_gemm(B, m->vocab, dm, kGemmArgmax), kGemmArgmax, hn, m->w_lm, bl, st));
    }
    if (rc) return rc;
    rc = cuda_status(launch_draft_collect(ids, maxv, B, k, step, drafts, draft_max, st));
    if (rc) return rc;
  }
  return SPEC_OK;
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" {

int spec_profile_start(int n_steps) {
  if (n_steps < 1 || n_steps > 65536) return SPEC_EINVAL;
  prof_release();
  g_prof.ev.resize(4 * (size_t)n_steps, nullptr);
  for (auto& e : g_prof.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      prof_release();
      return SPEC_ECUDA;
    }
  g_prof.n = n_steps;
  g_prof.on = true;
  return SPEC_OK;
}

int spec_profile_launches(int max_marks) {
  if (max_marks < 2 || max_marks > 4096) return SPEC_EINVAL;
  for (cudaEvent_t e : g_detail.ev) cudaEventDestroy(e);
  g_detail.ev.assign(max_marks, nullptr);
  for (auto& e : g_detail.ev)
    if (cudaEventCreate(&e) != cudaSuccess) return SPEC_ECUDA;
  g_detail.used = 0;
  g_detail.on = true;
  return SPEC_OK;
}

int spec_profile_launches_collect(float* ms, int max_marks, int* n_intervals) {
  if (!ms || !n_intervals || g_detail.used < 2) return SPEC_EINVAL;
  int n = 0;
  if (cudaEventSynchronize(g_detail.ev[g_detail.used - 1]) != cudaSuccess) return SPEC_ECUDA;
  for (int i = 1; i < g_detail.used && i - 1 < max_marks; ++i, ++n)
    if (cudaEventElapsedTime(&ms[i - 1], g_detail.ev[i - 1], g_detail.ev[i]) != cudaSuccess)
      return SPEC_ECUDA;
  *n_intervals = n;
  for (cudaEvent_t e : g_detail.ev) cudaEventDestroy(e);
  g_detail.ev.clear();
  g_detail.used = 0;
  g_detail.on = false;
  return SPEC_OK;
}

unsigned long long spec_launch_count(void) {
  return g_launch_count.load(std::memory_order_relaxed);
}

int spec_profile_collect(float* step_ms, float* lmhead_ms, int n_steps) {
  if (!g_prof.on || n_steps != g_prof.n || g_prof.used < n_steps || !step_ms) {
    prof_release();
    return SPEC_EINVAL;
  }
  int rc = SPEC_OK;
  for (int i = 0; i < n_steps && rc == SPEC_OK; ++i) {
    cudaEvent_t* e = &g_prof.ev[4 * (size_t)i];
    if (cudaEventSynchronize(e[3]) != cudaSuccess ||
        cudaEventElapsedTime(&step_ms[i], e[0], e[3]) != cudaSuccess ||
        (lmhead_ms && cudaEventElapsedTime(&lmhead_ms[i], e[1], e[2]) != cudaSuccess))
      rc = SPEC_ECUDA;
  }
  prof_release();
  return rc;
}

const char* spec_status_string(int s) {
  switch (s) {
    case SPEC_OK: return "ok";
    case SPEC_EINVAL: return "invalid argument";
    case SPEC_EUNSUPPORTED: return "unsupported configuration";
    case SPEC_ECUDA: return "CUDA error";
    case SPEC_EDEVICE: return "device reported bad data";
    case SPEC_ETIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

size_t spec_layer_pool_bytes(const spec_model* m, int layer, int which) {
  if (!m || !m->layers || layer < 0 || layer >= m->n_layers) return 0;
  const spec_layer& L = m->layers[layer];
  const size_t tok_heads = (size_t)m->num_pages * m->n_kv_heads * m->page_size;
  switch (which) {
    case 0: return tok_heads * m->head_dim * 2;
    case 1: return L.kv_equal ? 0 : tok_heads * m->head_dim * 2;
    case 2: return L.kv_equal ? tok_heads * 2 * n_rot_of(m, L) * 2 : 0;
  }
  return 0;
}

size_t spec_workspace_bytes(const spec_model* m, int max_batch, int max_k, int max_pages) {
  if (!m || !m->layers || max_batch < 1 || max_k < 0 || max_k > SPEC_MAX_K || max_pages < 1) return 0;
  StepLayout s = step_layout(m, max_batch, max_k + 1, max_pages);
  if (s.tickets > kMaxTickets || !s.splits_ok) return 0;
  return s.total;
}

size_t spec_lmhead_workspace_bytes(int M, int V) {
  if (M < 1 || V < 1) return 0;
  GemmPlan p = plan_gemm(M, V, 64, kGemmArgmax);
  return kWsHeaderBytes + up(gemm_argmax_entries(p) * 8);
}

int spec_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeaderBytes) return SPEC_EINVAL;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int spec_read_device_status(void* ws, size_t ws_bytes, void* stream, unsigned* status) {
  if (!ws || ws_bytes < kWsHeaderBytes || !status) return SPEC_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return SPEC_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SPEC_ECUDA;
  if (v && cudaMemsetAsync(ws, 0, 4, st) != cudaSuccess) return SPEC_ECUDA;
  *status = v;
  if (v & SPEC_DEV_TIMEOUT) return SPEC_ETIMEOUT;
  return v ? SPEC_EDEVICE : SPEC_OK;
}

int spec_cache_write(const spec_model* m, int layer, const int32_t* block_table_row, int max_pages,
                     int pos0, int n_tok, const void* k_raw, const void* v_raw, void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  if (layer < 0 || layer >= m->n_layers || !block_table_row || max_pages < 1 || pos0 < 0 ||
      n_tok < 0 || !k_raw)
    return SPEC_EINVAL;
  const spec_layer& L = m->layers[layer];
  if (!L.kv_equal && !v_raw) return SPEC_EINVAL;
  if ((int64_t)pos0 + n_tok > (int64_t)max_pages * m->page_size) return SPEC_EINVAL;
  if (n_tok == 0) return SPEC_OK;
  RopeAppend a{};
  a.n_q_heads = m->n_q_heads;
  a.n_kv_heads = m->n_kv_heads;
  a.head_dim = m->head_dim;
  a.n_rot = n_rot_of(m, L);
  rope_inv_freq(m->rope_theta, m->head_dim, a.n_rot, a.inv_freq);
  a.page_size = m->page_size;
  a.num_pages = m->num_pages;
  a.max_pages = max_pages;
  a.n_rows = n_tok;
  a.pos0 = pos0;
  a.block_table = block_table_row;
  a.src_k = k_raw;
  a.k_row_stride = (long)m->n_kv_heads * m->head_dim;
  a.src_v = L.kv_equal ? nullptr : v_raw;
  a.v_row_stride = a.k_row_stride;
  a.k_pool = static_cast<uint16_t*>(L.k_pool);
  a.v_pool = static_cast<uint16_t*>(L.v_pool);
  a.ksb_pool = static_cast<uint16_t*>(L.ksb_pool);
  return cuda_status(launch_rope_append(a, 1, static_cast<cudaStream_t>(stream)));
}

int spec_verify_attn(const spec_model* m, int layer, const void* q, const void* k_new,
                     const void* v_new, const int32_t* block_table, int max_pages,
                     const int32_t* seq_lens, int B, int k, void* out, void* ws, size_t ws_bytes,
                     void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  if (layer < 0 || layer >= m->n_layers || !q || !k_new || !block_table || !seq_lens || !out || !ws)
    return SPEC_EINVAL;
  if (B < 1 || k < 0 || k > SPEC_MAX_K || max_pages < 1) return SPEC_EINVAL;
  const spec_layer& L = m->layers[layer];
  if (!L.kv_equal && !v_new) return SPEC_EINVAL;
  const int qn = k + 1, D = m->head_dim;
  StepLayout s = step_layout(m, B, k + 1, max_pages);
  if (!s.splits_ok) return SPEC_EUNSUPPORTED;
  if (ws_bytes < s.total) return SPEC_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WsHeader hdr = ws_header(ws);

  RopeAppend a{};
  a.n_q_heads = m->n_q_heads;
  a.n_kv_heads = m->n_kv_heads;
  a.head_dim = D;
  a.n_rot = n_rot_of(m, L);
  rope_inv_freq(m->rope_theta, m->head_dim, a.n_rot, a.inv_freq);
  a.page_size = m->page_size;
  a.num_pages = m->num_pages;
  a.max_pages = max_pages;
  a.n_rows = qn;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.src_q = q;
  a.q_row_stride = (long)m->n_q_heads * D;
  a.q_seq_stride = a.q_row_stride * qn;
  a.src_k = k_new;
  a.k_row_stride = (long)m->n_kv_heads * D;
  a.k_seq_stride = a.k_row_stride * qn;
  a.src_v = L.kv_equal ? nullptr : v_new;
  a.v_row_stride = a.k_row_stride;
  a.v_seq_stride = a.k_seq_stride;
  a.q_out = at<uint16_t>(ws, s.qrot);
  a.k_pool = static_cast<uint16_t*>(L.k_pool);
  a.v_pool = static_cast<uint16_t*>(L.v_pool);
  a.ksb_pool = static_cast<uint16_t*>(L.ksb_pool);
  a.status = hdr.status;
  rc = cuda_status(launch_rope_append(a, B, st));
  if (rc) return rc;
  AttnGeom g = plan_attn(B, qn, m->n_q_heads, m->n_kv_heads, D, m->page_size, m->num_pages,
                         max_pages, L.window, L.kv_equal, 2 * a.n_rot, split_of(m, L));
  return cuda_status(launch_attention(g, at<uint16_t>(ws, s.qrot), L.k_pool, L.v_pool, L.ksb_pool,
                                      block_table, seq_lens, at<float>(ws, s.attn_part),
                                      static_cast<uint16_t*>(out), hdr.status, st));
}

int spec_lmhead_argmax(const void* h, const void* w, int M, int d, int V, int32_t* ids,
                       float* maxlogit, void* ws, size_t ws_bytes, void* stream) {
  if (!h || !w || !ids || !ws || M < 1 || V < 1 || d < 8 || d % 8) return SPEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(h) & 15) || (reinterpret_cast<uintptr_t>(w) & 15)) return SPEC_EINVAL;
  GemmPlan p = plan_gemm(M, V, d, kGemmArgmax);
  if (p.mblocks > kMaxTickets) return SPEC_EUNSUPPORTED;
  const size_t need = spec_lmhead_workspace_bytes(M, V);
  if (ws_bytes < need) return SPEC_EINVAL;
  WsHeader hdr = ws_header(ws);
  GemmBuffers b{};
  b.arg_keys = at<unsigned long long>(ws, kWsHeaderBytes);
  b.ids = ids;
  b.maxv = maxlogit;
  b.tickets = hdr.tickets;
  b.status = hdr.status;
  return cuda_status(launch_gemm_any(p, kGemmArgmax, h, w, b, static_cast<cudaStream_t>(stream)));
}

int spec_accept_commit(const int32_t* drafts, const int32_t* target, int B, int k,
                       int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                       int32_t* last_token, void* stream) {
  if (!target || !seq_lens || !accept_len || !emitted || !last_token) return SPEC_EINVAL;
  if (B < 1 || k < 0 || k > SPEC_MAX_K || (k > 0 && !drafts)) return SPEC_EINVAL;
  return cuda_status(launch_accept(drafts, target, B, k, seq_lens, accept_len, emitted, last_token,
                                   nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream)));
}

int spec_verify_step(const spec_model* m, const int32_t* block_table, int max_pages,
                     const int32_t* last_token, const int32_t* drafts, int B, int k,
                     int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                     int32_t* new_last_token, int32_t* target_ids, float* target_maxlogit,
                     void* ws, size_t ws_bytes, void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  if (!block_table || !last_token || !seq_lens || !accept_len || !emitted || !new_last_token || !ws)
    return SPEC_EINVAL;
  if (B < 1 || k < 0 || k > SPEC_MAX_K || max_pages < 1 || (k > 0 && !drafts)) return SPEC_EINVAL;
  ForwardIo io{};
  io.last_token = last_token;
  io.drafts = drafts;
  io.accept_len = accept_len;
  io.emitted = emitted;
  io.new_last_token = new_last_token;
  io.target_ids = target_ids;
  io.target_maxlogit = target_maxlogit;
  return run_forward(m, block_table, max_pages, B, k + 1, seq_lens, io, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

size_t spec_prefill_workspace_bytes(const spec_model* m, int max_batch, int max_n, int max_pages) {
  if (!m || !m->layers || max_batch < 1 || max_n < 1 || max_n > SPEC_MAX_PREFILL || max_pages < 1)
    return 0;
  StepLayout s = step_layout(m, max_batch, max_n, max_pages);
  if (s.tickets > kMaxTickets || !s.splits_ok) return 0;
  return s.total;
}

int spec_prefill(const spec_model* m, const int32_t* block_table, int max_pages,
                 const int32_t* tokens, int B, int n, int32_t* seq_lens, int32_t* next_token,
                 float* next_maxlogit, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  if (!block_table || !tokens || !seq_lens || !next_token || !ws) return SPEC_EINVAL;
  if (B < 1 || n < 1 || n > SPEC_MAX_PREFILL || max_pages < 1) return SPEC_EINVAL;
  ForwardIo io{};
  io.tokens = tokens;
  io.next_token = next_token;
  io.next_maxlogit = next_maxlogit;
  return run_forward(m, block_table, max_pages, B, n, seq_lens, io, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

size_t spec_draft_workspace_bytes(const spec_model* m, const spec_drafter* d, int B, int max_pages) {
  if (check_model(m) || check_drafter(m, d) || B < 1 || max_pages < 1) return 0;
  DraftLayout s = draft_layout(m, d, B, max_pages);
  if (s.tickets > kMaxTickets || !s.splits_ok) return 0;
  return s.total;
}

int spec_draft(const spec_model* m, const spec_drafter* d, const int32_t* block_table, int max_pages,
               const int32_t* seq_lens, const void* prev_hidden, const int32_t* prev_token, int B,
               int k, int32_t* drafts, float* draft_maxlogit, void* ws, size_t ws_bytes,
               void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  rc = check_drafter(m, d);
  if (rc) return rc;
  if (!block_table || !seq_lens || !prev_hidden || !prev_token || !drafts || !ws) return SPEC_EINVAL;
  if (B < 1 || k < 0 || max_pages < 1) return SPEC_EINVAL;
  if (k == 0) return SPEC_OK;
  return run_draft(m, d, block_table, max_pages, seq_lens, prev_hidden, prev_token, B, k, drafts,
                   draft_maxlogit, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

size_t spec_cluster_unembed_workspace_bytes(int M, int d, const spec_clusters* t) {
  if (M < 1 || check_clusters(t, d)) return 0;
  ClusterLayout c = cluster_layout(M, d, t, kWsHeaderBytes);
  if (c.tickets > kMaxTickets) return 0;
  return kWsHeaderBytes + c.bytes;
}

int spec_cluster_unembed(const void* h, int M, int d, const spec_clusters* t, int32_t* ids,
                         float* maxlogit, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_clusters(t, d);
  if (rc) return rc;
  if (!h || !ids || !ws || M < 1 || (reinterpret_cast<uintptr_t>(h) & 15)) return SPEC_EINVAL;
  ClusterLayout c = cluster_layout(M, d, t, kWsHeaderBytes);
  if (c.tickets > kMaxTickets) return SPEC_EUNSUPPORTED;
  if (ws_bytes < kWsHeaderBytes + c.bytes) return SPEC_EINVAL;
  return cuda_status(run_clusters(t, static_cast<const uint16_t*>(h), M, d, ids, maxlogit, ws, c,
                                  static_cast<cudaStream_t>(stream)));
}

size_t spec_verify_sampled_workspace_bytes(const spec_model* m, int B, int k, int max_pages) {
  if (check_model(m) || B < 1 || k < 0 || k > SPEC_MAX_K || max_pages < 1) return 0;
  SampledLayout L = sampled_layout(m, B, k, max_pages);
  if (L.tickets > kMaxTickets || !L.s.splits_ok) return 0;
  return L.total;
}

int spec_verify_step_sampled(const spec_model* m, const int32_t* block_table, int max_pages,
                             const int32_t* last_token, const int32_t* drafts,
                             const float* draft_logits, int B, int k, float temperature,
                             const float* u_accept, const float* u_draw, int32_t* seq_lens,
                             int32_t* accept_len, int32_t* emitted, int32_t* new_last_token,
                             float* target_logits, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_model(m);
  if (rc) return rc;
  if (!block_table || !last_token || !seq_lens || !accept_len || !emitted || !new_last_token ||
      !u_draw || !ws)
    return SPEC_EINVAL;
  if (B < 1 || k < 0 || k > SPEC_MAX_K || max_pages < 1) return SPEC_EINVAL;
  if (k > 0 && (!drafts || !draft_logits || !u_accept)) return SPEC_EINVAL;
  if (!(temperature > 0.f) || !isfinite(temperature)) return SPEC_EINVAL;
  SampledLayout L = sampled_layout(m, B, k, max_pages);
  if (L.tickets > kMaxTickets || !L.s.splits_ok) return SPEC_EUNSUPPORTED;
  if (ws_bytes < L.total) return SPEC_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ForwardIo io;
  io.last_token = last_token;
  io.drafts = drafts;
  io.logits = at<float>(ws, L.logits);
  io.logits_part = at<float>(ws, L.part);
  rc = run_forward(m, block_table, max_pages, B, k + 1, seq_lens, io, ws, ws_bytes, st);
  if (rc) return rc;
  const int M = B * (k + 1), V = m->vocab;
  if (target_logits &&
      cudaMemcpyAsync(target_logits, io.logits, (size_t)M * V * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SPEC_ECUDA;
  WsHeader hdr = ws_header(ws);
  return cuda_status(launch_sampled_tail(B, k, V, temperature, io.logits, draft_logits,
                                         at<float2>(ws, L.st_t), at<float2>(ws, L.st_d), drafts,
                                         u_accept, u_draw, at<int32_t>(ws, L.a),
                                         at<unsigned long long>(ws, L.keys), seq_lens, accept_len,
                                         emitted, new_last_token, hdr.status, st));
}

}  // extern "C"

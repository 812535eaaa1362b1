/*
 * specverify.h -- C ABI of the speculative-decoding verify step (B200, sm_100a).
 *
 * The operation: a target model checks k drafted tokens in ONE forward.  The
 * last accepted token and the k drafts run as k+1 causal query rows through
 * grouped-query attention against the KV cache the drafter and the target
 * share; the rows' final hidden states go through the LM head and an
 * argmax over the vocabulary; the longest prefix of drafts that agrees with
 * the target is accepted, the target's own token at the first disagreement
 * (or after the last draft) is added, and the cache keeps exactly the
 * accepted positions.
 *
 * Sources (page title, section):
 *   "Gemma 4 拆解 | 多模态怎么塞进端侧，MTP drafter 又是怎么自带投机采样的"
 *       §2   global layers use p-RoPE (p = 0.25) and let the value reuse the
 *            key, cutting the global KV cache by 37.5%;
 *       §4.1 the target checks the k guesses in one forward and cuts at the
 *            first wrong one;
 *       §4.2 `speculative_step`: draft, `main_model.verify`,
 *            `accept_longest_prefix`; the drafter reads the target's cache.
 *   "Accelerating Gemma 4: faster inference with multi-token prediction
 *   drafters" §3  the target verifies in parallel, accepts the agreeing run
 *            and adds one token of its own.
 *   "Gemma 4 发布时未包含 MTP 数据——为什么这很重要" §什么是 Gemma 4
 *            alternating local sliding-window / global layers, p-RoPE,
 *            shared KV cache, key-equals-value.
 *
 * Conventions fixed by this library where the pages are silent:
 *   - rows i = 0..k hold [last_token, draft_0 .. draft_{k-1}] at positions
 *     L..L+k (L = committed length); row i's argmax predicts position L+i+1;
 *   - acceptance is greedy: draft i is accepted iff it equals row i's argmax;
 *   - attention scale 1/sqrt(head_dim); key j is visible to the query at
 *     position t iff j <= t and, on a window-W layer, j > t - W;
 *   - RoPE pairs dimension i with i + D/2, theta_i = rope_theta^(-2i/D),
 *     angle = position * theta_i; p-RoPE rotates only pairs i < p*D/2;
 *   - key-equals-value layers: V is the pre-RoPE key; the cache keeps the
 *     post-RoPE key plus a side-band with the pre-RoPE values of the 2*n_rot
 *     rotated dimensions (n_rot = p*D/2), so per token and KV head it holds
 *     (1+p)*D values instead of 2*D;
 *   - the target layer is x <- x + W_o Attn(RMSNorm(x)) (no MLP), then a
 *     final RMSNorm and the LM head; RMSNorm eps from the model, unit
 *     gain; fp32 residual stream, bf16 for normalised GEMM inputs, q/k/v after
 *     RoPE, cache entries, attention outputs and the final hidden state;
 *   - argmax ties go to the lowest token id.
 *
 * Memory and ownership: every tensor argument is a DEVICE pointer owned by
 * the caller, unless marked "host".  The library never allocates device
 * memory; kernels that need scratch use the caller's workspace.  All calls
 * are asynchronous on the given stream (cudaStream_t passed as void*; NULL =
 * legacy default stream).  bf16 tensors are raw 16-bit bfloat16 patterns.
 *
 * Empty work: a batch of zero sequences (B < 1) or zero rows (M < 1) is an
 * invalid argument (SPEC_EINVAL, nothing launched), not a no-op; k = 0 (no
 * drafts) is valid and is one plain greedy decode step.
 *
 * Errors: arguments are validated on the host before any launch; on error
 * the call returns a negative spec_status and launches nothing (the cache is
 * untouched).  A launch failure returns SPEC_ECUDA.  Conditions only the
 * device can see (a page id outside the pool, a sequence longer than its
 * block-table row, a bounded wait that ran out) set bits in a status word in
 * the workspace; the affected work is skipped (never trapped), and
 * spec_read_device_status() returns them.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPEC_OK = 0,
  SPEC_EINVAL = -1,        /* bad argument (null pointer, size, alignment, range) */
  SPEC_EUNSUPPORTED = -2,  /* valid but outside what the kernels implement */
  SPEC_ECUDA = -3,         /* a CUDA runtime call or launch failed */
  SPEC_EDEVICE = -4,       /* the device flagged bad data (see device status bits) */
  SPEC_ETIMEOUT = -5       /* a bounded device wait ran out */
} spec_status;

/* Device status bits (spec_read_device_status). */
#define SPEC_DEV_BAD_PAGE 0x1u    /* block table entry outside [0, num_pages) */
#define SPEC_DEV_BAD_LENGTH 0x2u  /* L + k + 1 exceeds the sequence's block-table row */
#define SPEC_DEV_TIMEOUT 0x4u     /* a bounded mbarrier wait gave up */
#define SPEC_DEV_BAD_TOKEN 0x8u   /* a token id outside [0, vocab) */

/* Limits of this implementation. */
#define SPEC_MAX_K 16             /* drafts per step, k in [0, 16] */
#define SPEC_PAGE_SIZE 64         /* tokens per cache page */

/* One attention layer: its weights and its cache pools.
 * Pools are indexed by the same page ids for every layer (one block table
 * per sequence).  Layouts (bf16):
 *   k_pool   [num_pages][n_kv_heads][page_size][head_dim]  post-RoPE keys
 *   v_pool   [num_pages][n_kv_heads][page_size][head_dim]  values (NULL when kv_equal)
 *   ksb_pool [num_pages][n_kv_heads][page_size][2*n_rot]   kv_equal only: the pre-RoPE
 *            values of dims 0..n_rot-1 followed by dims D/2..D/2+n_rot-1
 * All three must be 16-byte aligned. */
typedef struct spec_layer {
  const void* w_qkv;    /* [(Hq + Hkv + (kv_equal ? 0 : Hkv)) * D][d_model]: q heads | k heads | v heads */
  const void* w_o;      /* [d_model][Hq * D] */
  void* k_pool;
  void* v_pool;
  void* ksb_pool;
  int window;           /* 0 = global; else keys t-W < j <= t are visible */
  int kv_equal;         /* 1: value = pre-RoPE key (no v projection, no v_pool) */
  float rope_fraction;  /* fraction of rotary pairs rotated (1.0 or 0.25 here) */
  int split_tokens;     /* this layer's split-KV chunk, 0 = the model's */
} spec_layer;

typedef struct spec_model {
  int n_layers;
  int d_model;
  int n_q_heads;
  int n_kv_heads;
  int head_dim;          /* 128 or 256 */
  int vocab;
  int page_size;         /* must be SPEC_PAGE_SIZE */
  int num_pages;         /* pages in each layer's pools */
  int split_tokens;      /* split-KV chunk: a multiple of page_size; fixed per model (and
                            optionally per layer) so that results do not depend on batch
                            size, k or the GPU */
  double rope_theta;     /* RoPE base (10000) */
  double rms_eps;        /* RMSNorm epsilon (1e-6) */
  const void* w_lm;      /* [vocab][d_model] bf16: LM head */
  const void* w_embed;   /* [vocab][d_model] bf16: token embedding (may equal w_lm: tied) */
  const spec_layer* layers;  /* host array of n_layers */
} spec_model;

/* Human-readable name of a spec_status value. */
const char* spec_status_string(int status);

/* Bytes of one layer pool for num_pages pages.  which: 0 = k_pool,
 * 1 = v_pool, 2 = ksb_pool.  Returns 0 for a pool the layer does not have. */
size_t spec_layer_pool_bytes(const spec_model* m, int layer, int which);

/* Workspace bytes needed by spec_verify_step / spec_verify_attn /
 * spec_lmhead_argmax for batches up to max_batch, k up to max_k and block
 * tables up to max_pages pages per sequence.  0 on invalid arguments. */
size_t spec_workspace_bytes(const spec_model* m, int max_batch, int max_k, int max_pages);

/* Workspace bytes spec_lmhead_argmax needs on its own for M rows and vocab V. */
size_t spec_lmhead_workspace_bytes(int M, int V);

/* Clears the whole workspace (async memset): counters, status word and the
 * argmax keys must start at zero.  Call once after allocating a workspace;
 * every kernel leaves them at zero again. */
int spec_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Reads and clears the device status word (synchronises the stream).
 * *status receives SPEC_DEV_* bits.  Returns SPEC_EDEVICE if any bit was set. */
int spec_read_device_status(void* ws, size_t ws_bytes, void* stream, unsigned* status);

/* Writes cache entries for n_tok consecutive positions pos0..pos0+n_tok-1 of
 * one sequence into layer `layer` (the RoPE + cache-append step, applied to
 * given pre-RoPE projections; used to fill a context and by the verify step
 * for its own rows).
 *   k_raw [n_tok][Hkv][D] bf16 pre-RoPE keys; v_raw [n_tok][Hkv][D] bf16
 *   values, NULL on kv_equal layers; block_table_row [max_pages] int32.
 * Page ids come from block_table_row[pos / page_size]. */
int spec_cache_write(const spec_model* m, int layer, const int32_t* block_table_row, int max_pages,
                     int pos0, int n_tok, const void* k_raw, const void* v_raw, void* stream);

/* Verify attention of one layer ("Gemma 4 拆解" §4.2 `main_model.verify`;
 * "Accelerating Gemma 4" §3).  For each sequence b with committed length
 * L = seq_lens[b]: rotates q and the new keys at positions L..L+k, writes the
 * k+1 new keys/values (or keys + side-band) into the layer's pools, and
 * computes grouped-query attention of the k+1 rows over keys 0..L+k (causal,
 * plus the layer's window).  seq_lens is not changed.
 *   q     [B][k+1][Hq][D]  bf16, pre-RoPE
 *   k_new [B][k+1][Hkv][D] bf16, pre-RoPE
 *   v_new [B][k+1][Hkv][D] bf16, NULL on kv_equal layers
 *   block_table [B][max_pages] int32, seq_lens [B] int32
 *   out   [B][k+1][Hq][D]  bf16
 * Requires (L + k + 1) <= max_pages * page_size (else SPEC_DEV_BAD_LENGTH and
 * the sequence is skipped). */
int spec_verify_attn(const spec_model* m, int layer, const void* q, const void* k_new,
                     const void* v_new, const int32_t* block_table, int max_pages,
                     const int32_t* seq_lens, int B, int k, void* out, void* ws, size_t ws_bytes,
                     void* stream);

/* Fused LM head + argmax ("Gemma 4 拆解" §4.2 `unembed_argmax`; the
 * vocabulary projection of §4.3): ids[m] = argmax_v h[m] . w[v], ties to the
 * lowest v; maxlogit[m] = that logit (binary32), may be NULL.  Logits are
 * never written to memory.
 *   h [M][d] bf16, w [V][d] bf16 (16-byte aligned, d a multiple of 8),
 *   ids [M] int32.  M >= 1, V >= 1. */
int spec_lmhead_argmax(const void* h, const void* w, int M, int d, int V, int32_t* ids,
                       float* maxlogit, void* ws, size_t ws_bytes, void* stream);

/* Acceptance, bonus token and commit ("Gemma 4 拆解" §4.1/§4.2
 * `accept_longest_prefix`; "Accelerating Gemma 4" §3).  For each b:
 *   a = number of leading i with drafts[b][i] == target[b][i]   (0 <= a <= k)
 *   emitted[b] = drafts[b][0..a-1], target[b][a], then -1 padding ([B][k+1])
 *   accept_len[b] = a;  last_token[b] = target[b][a];  seq_lens[b] += a + 1
 * Positions beyond the new length are rolled back: they stay in the pages but
 * are never read again before being overwritten.
 *   drafts [B][k], target [B][k+1] int32; seq_lens in/out. */
int spec_accept_commit(const int32_t* drafts, const int32_t* target, int B, int k,
                       int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                       int32_t* last_token, void* stream);

/* The whole verify step ("Gemma 4 拆解" §4.2 `speculative_step` steps 2-3):
 * embed [last_token, drafts] -> per layer (RMSNorm, QKV projection, RoPE,
 * cache append, split-KV attention, output projection + residual) -> final
 * RMSNorm -> LM head argmax -> acceptance and commit.
 *   last_token [B] int32 (read), drafts [B][k] int32 (may be NULL when k = 0),
 *   seq_lens [B] int32 in/out, accept_len [B], emitted [B][k+1],
 *   new_last_token [B] int32 (may alias last_token);
 *   target_ids [B][k+1] int32 and target_maxlogit [B][k+1] float: optional
 *   copies of every row's argmax and its logit (NULL to skip).
 * The workspace must come from spec_workspace_bytes(m, >= B, >= k, >= max_pages)
 * and have been cleared once with spec_workspace_init. */
int spec_verify_step(const spec_model* m, const int32_t* block_table, int max_pages,
                     const int32_t* last_token, const int32_t* drafts, int B, int k,
                     int32_t* seq_lens, int32_t* accept_len, int32_t* emitted,
                     int32_t* new_last_token, int32_t* target_ids, float* target_maxlogit,
                     void* ws, size_t ws_bytes, void* stream);

/* Prefill: the target forward over n new tokens per sequence at positions
 * L..L+n-1 (L = seq_lens[b]) through the same kernels as the verify step, so
 * the cache holds exactly what a token-by-token decode would have written
 * ("Gemma 4 拆解" §4.2: the target's prefilled cache that the drafter and the
 * verify step share).  All n rows are committed: seq_lens[b] += n.  The
 * argmax of each sequence's last row (the first token after the chunk) goes
 * to next_token[b], its logit to next_maxlogit[b] (may be NULL).
 *   tokens [B][n] int32, n in [1, SPEC_MAX_PREFILL]; the workspace comes
 *   from spec_prefill_workspace_bytes(m, >= B, >= n, >= max_pages). */
#define SPEC_MAX_PREFILL 256
size_t spec_prefill_workspace_bytes(const spec_model* m, int max_batch, int max_n, int max_pages);
int spec_prefill(const spec_model* m, const int32_t* block_table, int max_pages,
                 const int32_t* tokens, int B, int n, int32_t* seq_lens, int32_t* next_token,
                 float* next_maxlogit, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Sampled (distribution-preserving) verification.  The pages state the
 * property ("Gemma 4 发布时未包含 MTP 数据——为什么这很重要" §MTP 能快多少: the output is
 * what decoding the target alone would produce); for sampling this is
 * speculative sampling (Leviathan, Kalman, Matias, ICML 2023, Algorithm 1):
 * with p_i = softmax(target logits of verify row i / T) and q_i =
 * softmax(draft_logits[b][i] / T), draft i is accepted iff
 * u_accept[b][i] * q_i(d_i) < p_i(d_i); at the first rejection a token is
 * drawn from max(0, p_i - q_i), and after k acceptances from p_k.  A draw
 * from weights w is argmax_v log w_v - log(-log u_draw[b][v]) (w_v = 0
 * never drawn; equal scores: lowest id).  Emits the accepted drafts and the
 * drawn token, commits a+1 positions like spec_verify_step.
 *   draft_logits [B][k][V] binary32, u_accept [B][k] in [0, 1), u_draw
 *   [B][V] in (0, 1): device inputs; temperature > 0;
 *   target_logits [B][k+1][V] (out, device) or NULL.
 * ws: spec_verify_sampled_workspace_bytes (it holds the B*(k+1) x V target
 * logits), set up once with spec_workspace_init.
 * ------------------------------------------------------------------------- */
size_t spec_verify_sampled_workspace_bytes(const spec_model* m, int B, int k, int max_pages);
int spec_verify_step_sampled(const spec_model* m, const int32_t* block_table, int max_pages,
                             const int32_t* last_token, const int32_t* drafts,
                             const float* draft_logits, int B, int k, float temperature,
                             const float* u_accept, const float* u_draw, int32_t* seq_lens,
                             int32_t* accept_len, int32_t* emitted, int32_t* new_last_token,
                             float* target_logits, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * MTP drafter on the target's shared KV cache ("Gemma 4 拆解 | 多模态怎么塞进端侧，
 * MTP drafter 又是怎么自带投机采样的" §4.2: the drafter's input is the target's
 * last-layer activation plus the embedding of the previous token, projected
 * down to the drafter width; its blocks (three sliding-window, one global)
 * attend to the target's cache instead of keeping one of their own, so it
 * needs no prefill; its output is projected back up and the target's
 * unembedding picks the next draft token; k tokens are drafted one after the
 * other).
 *
 * Each block is x <- x + W_o CrossAttn(RMSNorm(x)) with n_q_heads heads of
 * the target's head_dim over the cache of target layer `target_layer`, read
 * as stored (post-RoPE keys; values or the key-equals-value side-band) with
 * that layer's window and RoPE fraction.  Draft step s of sequence b sits at
 * position seq_lens[b] + s and sees the cached keys j < seq_lens[b] (window
 * layers: also j > seq_lens[b] + s - window); a query that sees no key gets
 * a zero attention output.  The up-projection's output (binary32) is the
 * next step's activation; the target's final RMSNorm and LM head turn it
 * into the draft token (argmax, ties to the lowest id).  Every projection
 * input is bf16.  The drafter writes nothing to the cache and does not
 * change seq_lens.
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* w_q;     /* bf16 [n_q_heads * head_dim][d_draft] */
  const void* w_o;     /* bf16 [d_draft][n_q_heads * head_dim] */
  int target_layer;    /* target layer whose cache this block reads */
} spec_draft_block;

/* Token clusters for the cheap unembedding ("Gemma 4 拆解 ..." §4.3: score the
 * clusters' centroids, keep the best few, and take the argmax over their
 * tokens only, ~4096 candidates instead of the whole vocabulary).  A
 * cluster's logit is h . centroid; the n_select largest are kept (equal
 * logits: lower cluster id); every token of those clusters is scored with
 * its LM-head row and the largest logit wins (equal logits: lowest token
 * id).  All pointers are device memory owned by the caller. */
typedef struct {
  int n_clusters;                 /* C, 1..8192 */
  int cluster_size;               /* S, tokens per cluster, 1..4096 */
  int n_select;                   /* clusters kept per row, 1..C */
  const void* centroids;          /* bf16 [C][d_model] */
  const int32_t* cluster_tokens;  /* [C][S] token ids; -1 pads a short cluster */
  const void* w_clustered;        /* bf16 [C*S][d_model]: row c*S+i = LM-head row of
                                     cluster_tokens[c][i] (rows of pads are never read) */
} spec_clusters;

/* Workspace bytes of spec_cluster_unembed for M rows of width d (0 if unsupported). */
size_t spec_cluster_unembed_workspace_bytes(int M, int d, const spec_clusters* t);

/* ids[M] (and maxlogit[M], or NULL) = the cheap clustered argmax of h
 * (bf16 [M][d], device).  ws: spec_cluster_unembed_workspace_bytes, set up
 * once with spec_workspace_init. */
int spec_cluster_unembed(const void* h, int M, int d, const spec_clusters* t, int32_t* ids,
                         float* maxlogit, void* ws, size_t ws_bytes, void* stream);

typedef struct {
  int d_draft;         /* drafter width, multiple of 8 */
  int n_q_heads;       /* query heads per block, multiple of the target's n_kv_heads */
  int n_blocks;        /* 1..16 */
  const void* w_embed; /* bf16 [vocab][d_draft]: the drafter's own token embedding */
  const void* w_down;  /* bf16 [d_draft][d_model + d_draft]: input [activation || embedding] */
  const void* w_up;    /* bf16 [d_model][d_draft] */
  const spec_draft_block* blocks;
  const spec_clusters* clusters; /* NULL: the target's full LM head picks each draft token;
                                    else the cheap clustered unembedding does */
} spec_drafter;

/* Workspace bytes of spec_draft for up to B sequences (0 if unsupported). */
size_t spec_draft_workspace_bytes(const spec_model* m, const spec_drafter* d, int B, int max_pages);

/* k drafter steps for B sequences.
 *   block_table [B][max_pages], seq_lens [B]: the target's committed cache
 *     (device, read only);
 *   prev_hidden: bf16 [B][d_model], the target's last-layer activation for
 *     the last accepted token (device);
 *   prev_token [B]: that token (device);
 *   drafts [B][k] (out, device), draft_maxlogit [B][k] (out, device, or NULL).
 * ws: caller-owned device workspace of spec_draft_workspace_bytes, set up
 * once with spec_workspace_init.  Host-detectable errors return before any
 * launch; a bad token id sets SPEC_DEV_BAD_TOKEN (read with
 * spec_read_device_status).  k = 0 launches nothing. */
int spec_draft(const spec_model* m, const spec_drafter* d, const int32_t* block_table, int max_pages,
               const int32_t* seq_lens, const void* prev_hidden, const int32_t* prev_token, int B,
               int k, int32_t* drafts, float* draft_maxlogit, void* ws, size_t ws_bytes,
               void* stream);

/* LM head + argmax without a workspace, for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a deployment aid.
 *
 * Who needs it: callers that have no way to hand the library a workspace --
 * a runtime whose device memory plan is fixed before decoding starts and
 * forbids allocation on the decode path, a plugin that a host framework
 * gives only its input and output tensors, a latency-critical loop that
 * cannot take cudaMalloc's implicit device synchronisation.
 *
 * Same operation and arguments as spec_lmhead_argmax, minus the workspace,
 * and the same kernels (the tensor-memory GEMM above 32 rows, the streaming
 * one below).  Its scratch (a status word, the completion counters and one
 * argmax key per row) is a file-scope __device__ array inside the library,
 * of 4 KiB + 8 bytes per row, that every GPU which loads the library holds
 * until the process exits.
 * Limit: M <= SPEC_NOALLOC_MAX_ROWS (the keys the array holds); larger M
 * returns SPEC_EUNSUPPORTED and launches nothing.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Each call clears the counters and the keys (an
 * async memset on `stream`) and allocates nothing.  Device-detected errors
 * (a bounded wait that ran out) set bits in the array's status word, which
 * calls do not clear: they accumulate until spec_noalloc_read_status reads
 * and clears them.  All calls share the one array, which keeps the last
 * call's contents: calls that overlap on the GPU (different streams, or
 * concurrent host threads on one device) race and must be serialised by the
 * caller. */
#define SPEC_NOALLOC_MAX_ROWS 64
int spec_lmhead_argmax_noalloc(const void* h, const void* w, int M, int d, int V, int32_t* ids,
                               float* maxlogit, void* stream);
/* Reads and clears the status word of spec_lmhead_argmax_noalloc's scratch on
 * the current device (synchronises the stream).  *status receives SPEC_DEV_*
 * bits; returns SPEC_ETIMEOUT if SPEC_DEV_TIMEOUT was set, SPEC_EDEVICE for
 * any other bit, else SPEC_OK. */
int spec_noalloc_read_status(void* stream, unsigned* status);
/* Fault injection on the host side: ORs `bits` into that status word (one
 * one-thread kernel on `stream`), so that callers can test their handling of
 * device-detected errors without making the device fail. */
int spec_noalloc_inject_status(unsigned bits, void* stream);

/* Timing hook (no counterpart in the pages; measurement only).
 * spec_profile_start(n): the next n spec_verify_step calls record CUDA events
 * (created and owned by the library) on their stream around the whole step
 * and around the LM-head launch.  spec_profile_collect(step_ms, lmhead_ms, n)
 * waits for those events, writes the n per-step durations in milliseconds
 * (host arrays) and releases the events.  Process-wide; not thread-safe.
 * n must be in [1, 65536]; collect returns SPEC_EINVAL if fewer than n steps
 * were recorded. */
int spec_profile_start(int n_steps);
int spec_profile_collect(float* step_ms, float* lmhead_ms, int n_steps);
/* Per-launch timing of the next spec_verify_step / spec_prefill call: an event
 * after every kernel launch of that call (at most max_marks).  The events
 * serialise the launches (no programmatic overlap), so the sum exceeds a
 * normal step; the intervals show each kernel's own time.  collect writes
 * the intervals in launch order, in milliseconds. */
int spec_profile_launches(int max_marks);
int spec_profile_launches_collect(float* ms, int max_marks, int* n_intervals);

/* Number of kernels the library has launched successfully since it was
 * loaded (all devices and threads; a relaxed atomic counter).  The
 * difference across a region counts that region's launches. */
unsigned long long spec_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPECVERIFY_H */

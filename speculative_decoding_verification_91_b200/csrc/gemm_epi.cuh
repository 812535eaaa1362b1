// Epilogues shared by the streaming GEMM kernels (mma.sync and tcgen05):
// argmax reduction + fused acceptance, split-K sum + store / residual, and
// the QKV projection's RoPE + cache append.  All run on kEpiThreads threads
// (four warps) that synchronise with named barrier 1.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace sv {

constexpr int kTileN = 128;     // weight rows (output features / vocab entries) per tile
constexpr int kTileK = 64;      // bf16 elements per 128-byte K chunk
constexpr int kEpiThreads = 128;

struct Args {
  int M, N, K, kchunks, splits, n_tiles;
  int np;           // tcgen05 kernel: padded token count (MMA N)
  int ldp;          // partials: element (split s, feature f, row m) at (s*n_tiles*128 + f)*ldp + m
  int grid_reduce;  // 1: the split partials are reduced by splitk_reduce_kernel, not the last CTA
  float* out;
  float* partial;
  unsigned long long* arg_keys;   // [M] packed (value, id) keys, zero between launches
  int32_t* ids;
  float* maxv;
  unsigned* tickets;
  unsigned* status;
  AcceptFuse acc;   // acc.B > 0: the argmax's last CTA also runs the acceptance
  RopeFuse rope;    // kGemmQkvRope
};

// Acceptance of sequence b from the argmax ids of its k+1 rows (one warp).
__device__ __forceinline__ void accept_one(const AcceptFuse& f, int b, const int32_t* tg, int lane) {
  const int k = f.k, q = k + 1;
  const bool match = lane < k && f.drafts[(size_t)b * k + lane] == tg[lane];
  const unsigned mism = ~__ballot_sync(0xffffffffu, match);   // bit i: draft i not accepted
  const int a = min(__ffs(mism) - 1, k);
  if (lane < q) {
    int v = -1;
    if (lane < a) v = f.drafts[(size_t)b * k + lane];
    else if (lane == a) v = tg[a];
    f.emitted[(size_t)b * q + lane] = v;
  }
  __syncwarp();
  if (lane == 0) {
    f.accept_len[b] = a;
    f.last_token[b] = tg[a];
    f.seq_lens[b] += a + 1;
  }
}

// Argmax candidates are published as one 64-bit key per row and merged with
// atomicMax: the key orders by value (order-preserving binary32 bits) and, for
// equal values, by the lower token id (id stored as 0xFFFFFFFF - id).  The
// maximum of a set of keys does not depend on the order of the atomics, so
// the result is deterministic.  A zero key is below every real candidate.
__device__ __forceinline__ unsigned long long pack_arg(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)idx);
}
__device__ __forceinline__ void unpack_arg(unsigned long long key, float& v, int& idx) {
  const uint32_t hi = (uint32_t)(key >> 32);
  v = __uint_as_float((hi & 0x80000000u) ? (hi & 0x7FFFFFFFu) : ~hi);
  idx = (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

// After this CTA merged its per-tile candidates into the row keys: the last
// CTA of the M-block turns the keys of its rows into ids / max logits, clears
// them for the next launch and, when fused, runs the acceptance of every
// sequence.  ids_s: shared scratch of >= mrows ints.
__device__ __forceinline__ void argmax_finish(const Args& a, int n_parts, int mblk, int m0,
                                              int mrows, int ctid, int* flag, int* ids_s) {
  const int warp = ctid >> 5, lane = ctid & 31;
  __threadfence();
  named_bar(1, kEpiThreads);
  if (ctid == 0) {
    const unsigned prev = atomicAdd(&a.tickets[mblk], 1u);
    *flag = (prev == (unsigned)(n_parts - 1));
  }
  named_bar(1, kEpiThreads);
  if (!*flag) return;
  __threadfence();
  const int mcount = min(mrows, a.M - m0);
  for (int mm = ctid; mm < mcount; mm += kEpiThreads) {
    const int m = m0 + mm;
    float bv;
    int bi;
    unpack_arg(atomicExch(&a.arg_keys[m], 0ull), bv, bi);
    a.ids[m] = bi;
    if (a.maxv) a.maxv[m] = bv;
    ids_s[mm] = bi;
    if (a.acc.copy_ids) a.acc.copy_ids[m] = bi;
    if (a.acc.copy_max) a.acc.copy_max[m] = bv;
  }
  if (ctid == 0) a.tickets[mblk] = 0u;
  if (a.acc.B > 0) {                 // all rows are in this block
    named_bar(1, kEpiThreads);
    for (int b = warp; b < a.acc.B; b += kEpiThreads / 32)
      accept_one(a.acc, b, ids_s + b * (a.acc.k + 1), lane);
  }
}

// QKV projection epilogue: after this CTA published its split partial, the
// last CTA to finish a head (all splits of its D/128 column tiles) sums the
// partials in split order, rotates each (j, j + D/2) pair of query and key
// heads at its row's position and writes queries to the workspace and keys,
// values and the key-equals-value side-band to the cache pools.
__device__ __forceinline__ void rope_epilogue(const Args& a, int MP, int n_tile, int mblk, int m0,
                                              int ctid, int* flag) {
  const RopeFuse& f = a.rope;
  const int D = f.head_dim, half = D / 2, tph = D / kTileN;
  const int head = n_tile / tph, n_heads = a.N / D;
  if (ctid == 0) {
    const unsigned prev = atomicAdd(&a.tickets[mblk * n_heads + head], 1u);
    *flag = (prev == (unsigned)(a.splits * tph - 1));
  }
  named_bar(1, kEpiThreads);
  if (!*flag) return;
  __threadfence();
  const int mcount = min(MP, a.M - m0);
  const size_t split_stride = (size_t)a.n_tiles * kTileN * a.ldp;
  const int n_items = half * mcount;
  for (int it0 = ctid; it0 < n_items; it0 += 2 * kEpiThreads) {
   float xs0[2] = {0.f, 0.f}, xs1[2] = {0.f, 0.f};
   for (int sp0 = 0; sp0 < a.splits; sp0 += 8) {
    float u0[2][8], u1[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int item = it0 + u * kEpiThreads;
      const int mm = item / half, j = item % half;
      const int f0 = head * D + j, f1 = f0 + half;
      const float* p0 = a.partial + (size_t)f0 * a.ldp + m0 + mm;
      const float* p1 = a.partial + (size_t)f1 * a.ldp + m0 + mm;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const bool ok = item < n_items && sp0 + w < a.splits;
        u0[u][w] = ok ? __ldcg(p0 + (size_t)(sp0 + w) * split_stride) : 0.f;
        u1[u][w] = ok ? __ldcg(p1 + (size_t)(sp0 + w) * split_stride) : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 8; ++w)
        if (sp0 + w < a.splits) {
          xs0[u] = __fadd_rn(xs0[u], u0[u][w]);
          xs1[u] = __fadd_rn(xs1[u], u1[u][w]);
        }
   }
   for (int u = 0; u < 2; ++u) {
    const int item = it0 + u * kEpiThreads;
    if (item >= n_items) break;
    const int mm = item / half, j = item % half;
    const float x0 = xs0[u], x1 = xs1[u];
    const int m = m0 + mm, b = m / f.q, i = m % f.q;
    const bool rot = j < f.n_rot && head < f.n_q_heads + f.n_kv_heads;
    float y0 = x0, y1 = x1;
    if (rot) {
      const float2 cs = f.rope_tab[(size_t)m * half + j];
      rope_pair(x0, x1, cs.x, cs.y, y0, y1);
    }
    if (head < f.n_q_heads) {
      uint16_t* qo = f.q_out + ((size_t)m * f.n_q_heads + head) * D;
      qo[j] = f32_to_bf16(y0);
      qo[j + half] = f32_to_bf16(y1);
      continue;
    }
    const int pos = f.seq_lens[b] + i;
    if (pos < 0 || pos / f.page_size >= f.max_pages) {
      flag_status(a.status, SPEC_DEV_BAD_LENGTH);
      continue;
    }
    const int page = f.block_table[(size_t)b * f.max_pages + pos / f.page_size];
    if (page < 0 || page >= f.num_pages) {
      flag_status(a.status, SPEC_DEV_BAD_PAGE);
      continue;
    }
    const int kvh = head < f.n_q_heads + f.n_kv_heads ? head - f.n_q_heads
                                                      : head - f.n_q_heads - f.n_kv_heads;
    const size_t row = ((size_t)page * f.n_kv_heads + kvh) * f.page_size + pos % f.page_size;
    if (head < f.n_q_heads + f.n_kv_heads) {
      f.k_pool[row * D + j] = f32_to_bf16(y0);
      f.k_pool[row * D + j + half] = f32_to_bf16(y1);
      if (f.ksb_pool && j < f.n_rot) {
        f.ksb_pool[row * 2 * f.n_rot + j] = f32_to_bf16(x0);
        f.ksb_pool[row * 2 * f.n_rot + f.n_rot + j] = f32_to_bf16(x1);
      }
    } else {
      f.v_pool[row * D + j] = f32_to_bf16(x0);
      f.v_pool[row * D + j + half] = f32_to_bf16(x1);
    }
   }
  }
  if (ctid == 0) a.tickets[mblk * n_heads + head] = 0u;
}

// After this CTA published its split partial: the last split of the tile
// sums all partials in split order and applies the store / residual epilogue.
template <int MODE>
__device__ __forceinline__ void splitk_finish(const Args& a, int MP, int n_tile, int mblk, int m0,
                                              int ctid, int* flag) {
  if (ctid == 0) {
    unsigned* tk = &a.tickets[mblk * a.n_tiles + n_tile];
    const unsigned prev = atomicAdd(tk, 1u);
    *flag = (prev == (unsigned)(a.splits - 1));
  }
  named_bar(1, kEpiThreads);
  if (!*flag) return;
  __threadfence();
  // last split of this tile: sum partials in split order, then the epilogue.
  // Work item = (output feature r, row mm); the split loads of an item are
  // issued together (independent) and then added in split order.
  const int mcount = min(MP, a.M - m0);
  const size_t split_stride = (size_t)a.n_tiles * kTileN * a.ldp;
  const float* base = a.partial + (size_t)n_tile * kTileN * a.ldp + m0;
  const int n_items = kTileN * mcount;
  // four items per thread at a time, their split loads issued together
  for (int it0 = ctid; it0 < n_items; it0 += 4 * kEpiThreads) {
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sp0 = 0; sp0 < a.splits; sp0 += 8) {
      float v[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int item = it0 + u * kEpiThreads;
        const int mm = item / kTileN, r = item % kTileN;
        const float* p = base + (size_t)r * a.ldp + mm;
#pragma unroll
        for (int w = 0; w < 8; ++w)
          v[u][w] = (item < n_items && sp0 + w < a.splits) ? __ldcg(p + (size_t)(sp0 + w) * split_stride)
                                                           : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 8; ++w)
          if (sp0 + w < a.splits) s[u] = __fadd_rn(s[u], v[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int item = it0 + u * kEpiThreads;
      if (item >= n_items) continue;
      const int mm = item / kTileN, r = item % kTileN;
      const int n = n_tile * kTileN + r;
      if (n >= a.N) continue;
      float* dst = a.out + (size_t)(m0 + mm) * a.N + n;
      if (MODE == kGemmResidual)
        *dst = __fadd_rn(*dst, s[u]);
      else
        *dst = s[u];
    }
  }
  if (ctid == 0) a.tickets[mblk * a.n_tiles + n_tile] = 0u;
}

// Grid-wide split-K sum + epilogue (store / residual / QKV + RoPE) for
// problems whose rows are too many for one CTA per tile to finish quickly.
cudaError_t launch_splitk_reduce(const Args& a, int mode, cudaStream_t st);

}  // namespace sv

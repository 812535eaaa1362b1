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
constexpr int kEpiMaxRows = 16;   // rows the last-CTA epilogues handle (more: the grid-wide reduce)

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

// The split partials of one 128-feature tile are, per split, one contiguous
// block of 128 x ldp floats (feature-major, rows contiguous, ldp a multiple of
// 8).  The last-CTA epilogues below read them as float4 runs of four rows of
// one feature, so that a warp's loads cover 512 contiguous bytes, and keep the
// loads of several splits in flight before adding them in split order
// (starting from 0, exactly as splitk_reduce_kernel does).
__device__ __forceinline__ float4 add4_rn(float4 s, float4 v) {
  return make_float4(__fadd_rn(s.x, v.x), __fadd_rn(s.y, v.y), __fadd_rn(s.z, v.z), __fadd_rn(s.w, v.w));
}
__device__ __forceinline__ float lane4(const float4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}

// QKV projection epilogue: after this CTA published its split partial, the
// last CTA to finish a head (all splits of its D/128 column tiles) sums the
// partials in split order, rotates each (j, j + D/2) pair of query and key
// heads at its row's position and writes queries to the workspace and keys,
// values and the key-equals-value side-band to the cache pools.  Work item =
// (pair j, four consecutive rows).
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
  const int ld = a.ldp, q4 = ld / 4;
  const size_t split_stride = (size_t)a.n_tiles * kTileN * ld;
  const int n_items = half * q4;
  // cache row of every verify row of a key or value head, once per row
  // (-1: invalid length or page, flagged)
  __shared__ long long row_s[kEpiMaxRows];
  if (head >= f.n_q_heads && ctid < mcount) {
    const int m = m0 + ctid, b = m / f.q, i = m % f.q;
    const int kvh = head < f.n_q_heads + f.n_kv_heads ? head - f.n_q_heads
                                                      : head - f.n_q_heads - f.n_kv_heads;
    const int pos = f.seq_lens[b] + i;
    long long r = -1;
    if (pos < 0 || pos / f.page_size >= f.max_pages) {
      flag_status(a.status, SPEC_DEV_BAD_LENGTH);
    } else {
      const int page = f.block_table[(size_t)b * f.max_pages + pos / f.page_size];
      if (page < 0 || page >= f.num_pages)
        flag_status(a.status, SPEC_DEV_BAD_PAGE);
      else
        r = ((long long)page * f.n_kv_heads + kvh) * f.page_size + pos % f.page_size;
    }
    row_s[ctid] = r;
  }
  named_bar(1, kEpiThreads);
  constexpr int kU = 4;                  // items per thread per pass
  for (int it0 = ctid; it0 < n_items; it0 += kU * kEpiThreads) {
    float4 s0[kU], s1[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) s0[u] = s1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp0 = 0; sp0 < a.splits; sp0 += 2) {
      float4 v0[kU][2], v1[kU][2];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int item = it0 + u * kEpiThreads;
        const int j = item / q4, mq = (item % q4) * 4;
        const float* p0 = a.partial + (size_t)(head * D + j) * ld + m0 + mq;
        const float* p1 = p0 + (size_t)half * ld;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const bool ok = item < n_items && sp0 + w < a.splits;
          const size_t o = (size_t)(sp0 + w) * split_stride;
          v0[u][w] = ok ? __ldcg(reinterpret_cast<const float4*>(p0 + o)) : make_float4(0.f, 0.f, 0.f, 0.f);
          v1[u][w] = ok ? __ldcg(reinterpret_cast<const float4*>(p1 + o)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if (sp0 + w < a.splits) {
            s0[u] = add4_rn(s0[u], v0[u][w]);
            s1[u] = add4_rn(s1[u], v1[u][w]);
          }
    }
    // every load before the first store (a store may alias a later load as
    // far as the compiler knows): the (cos, sin) entries of rotated pairs
    const bool rot_head = head < f.n_q_heads + f.n_kv_heads;
    float2 cs[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int item = it0 + u * kEpiThreads;
      const int j = item / q4, mq = (item % q4) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        cs[u][e] = (item < n_items && mq + e < mcount && rot_head && j < f.n_rot)
                       ? f.rope_tab[(size_t)(m0 + mq + e) * half + j]
                       : make_float2(1.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int item = it0 + u * kEpiThreads;
      if (item >= n_items) break;
      const int j = item / q4, mq = (item % q4) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int mm = mq + e;
        if (mm >= mcount) break;
        const float x0 = lane4(s0[u], e), x1 = lane4(s1[u], e);
        const int m = m0 + mm;
        float y0 = x0, y1 = x1;
        if (rot_head && j < f.n_rot) rope_pair(x0, x1, cs[u][e].x, cs[u][e].y, y0, y1);
        if (head < f.n_q_heads) {
          uint16_t* qo = f.q_out + ((size_t)m * f.n_q_heads + head) * D;
          qo[j] = f32_to_bf16(y0);
          qo[j + half] = f32_to_bf16(y1);
          continue;
        }
        const long long rowi = row_s[mm];
        if (rowi < 0) continue;
        const size_t row = (size_t)rowi;
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
  }
  if (ctid == 0) a.tickets[mblk * n_heads + head] = 0u;
}

// After this CTA published its split partial: the last split of the tile
// sums all partials in split order and applies the store / residual epilogue.
// Work item = (output feature r, four consecutive rows).
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
  const int mcount = min(MP, a.M - m0);
  const int ld = a.ldp, q4 = ld / 4;
  const size_t split_stride = (size_t)a.n_tiles * kTileN * ld;
  const float* base = a.partial + (size_t)n_tile * kTileN * ld + m0;
  const int n_items = kTileN * q4;
  constexpr int kU = 4;
  for (int it0 = ctid; it0 < n_items; it0 += kU * kEpiThreads) {
    float4 s[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) s[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp0 = 0; sp0 < a.splits; sp0 += 4) {
      float4 v[kU][4];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int item = it0 + u * kEpiThreads;
        const float* p = base + (size_t)(item / q4) * ld + (item % q4) * 4;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          v[u][w] = (item < n_items && sp0 + w < a.splits)
                        ? __ldcg(reinterpret_cast<const float4*>(p + (size_t)(sp0 + w) * split_stride))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (sp0 + w < a.splits) s[u] = add4_rn(s[u], v[u][w]);
    }
    // the residuals are read before the first store (a store may alias a
    // later load as far as the compiler knows)
    float res[kU][4];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int item = it0 + u * kEpiThreads;
      const int n = n_tile * kTileN + item / q4, mq = (item % q4) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        res[u][e] = (MODE == kGemmResidual && item < n_items && n < a.N && mq + e < mcount)
                        ? a.out[(size_t)(m0 + mq + e) * a.N + n]
                        : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int item = it0 + u * kEpiThreads;
      if (item >= n_items) break;
      const int r = item / q4, mq = (item % q4) * 4;
      const int n = n_tile * kTileN + r;
      if (n >= a.N) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int mm = mq + e;
        if (mm >= mcount) break;
        float* dst = a.out + (size_t)(m0 + mm) * a.N + n;
        *dst = (MODE == kGemmResidual) ? __fadd_rn(res[u][e], lane4(s[u], e)) : lane4(s[u], e);
      }
    }
  }
  if (ctid == 0) a.tickets[mblk * a.n_tiles + n_tile] = 0u;
}

// Grid-wide split-K sum + epilogue (store / residual / QKV + RoPE) for
// problems whose rows are too many for one CTA per tile to finish quickly.
cudaError_t launch_splitk_reduce(const Args& a, int mode, cudaStream_t st);

}  // namespace sv

// Split-KV verify attention on the 5th-generation tensor cores (sm_100a).
//
// One CTA per (sequence, KV head, absolute split of `split_tokens` keys, row
// block of up to NP query rows); 6 warps:
//   warp 0    TMA producer.  Keys arrive in blocks of 128 (two 64-token pages)
//             as four 128 x 64 swizzled atoms; on key-equals-value layers the
//             side-band atom (pre-RoPE rotated dims) rides with the keys, on
//             separate-K/V layers the values have their own buffer.
//   warp 1    allocates TMEM and issues the MMAs (one thread):
//               S^T[128 keys][NP rows] = K . Q^T          (A = K, K-major)
//               O^T[dims][NP rows]   += V^T . P_hi^T + V^T . P_lo^T
//                                                          (A = V^T, MN-major)
//             with the accumulators in TMEM (lane = key or value dim,
//             column = query row).
//   warps 2-5 softmax: thread t owns key t of the block (TMEM lane t): it
//             reads its NP scores, the row maxima and sums are reduced over
//             the 128 keys (warp transpose-reduce, then 4 warps in order),
//             it writes its probabilities as bf16 head + bf16 tail into the
//             P tiles, and it rescales its lanes of O when a row maximum
//             moved.  At the end it writes the partial (o, m, l) of its
//             rows, the same layout the mma.sync kernel writes.
//
// Value rows of keys outside the split's valid range (or on pages that were
// not loaded) are zeroed in shared memory before the PV product, so stale or
// poisoned slots never reach it.  Keys are visited in blocks at absolute
// 128-key boundaries and every reduction tree depends only on absolute key
// positions, so a row's partial does not depend on k, the batch or its row
// slot.  Every wait is bounded; the CTA always frees its TMEM.
#include <math.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sv {

namespace {

constexpr int kTaThreads = 192;
constexpr int kBlk = 128;                    // keys per MMA block
constexpr int kPg = 64;                      // tokens per page
constexpr int kDim = 256;                    // head_dim of this kernel
constexpr uint32_t kAtom = kBlk * 128;       // 128 keys x 64 dims of bf16: 16 KB
constexpr uint32_t kHalfAtom = kPg * 128;    // one page's rows of an atom: 8 KB

template <bool KVEQ, int NP>
struct TaCfg {
  static constexpr uint32_t kKsBytes = 4 * kAtom + (KVEQ ? kAtom : 0);   // K atoms (+ side-band)
  static constexpr uint32_t kVBytes = KVEQ ? 0 : 4 * kAtom;
  static constexpr uint32_t kQBytes = 4u * NP * 128u;
  static constexpr uint32_t kPBytes = 2u * NP * 128u;                   // one of P_hi / P_lo
  static constexpr uint32_t kTailBytes = 4096;
  // P_hi/P_lo are double-buffered when shared memory allows (the softmax of
  // block j+1 then writes its P while the PV product of block j reads its own)
  static constexpr int kPBufs =
      (1024 + 2 * kKsBytes + kVBytes + kQBytes + 4 * kPBytes + kTailBytes <= 227 * 1024) ? 2 : 1;
  static constexpr uint32_t kOffV = 2 * kKsBytes;
  static constexpr uint32_t kOffQ = kOffV + kVBytes;
  static constexpr uint32_t kOffP = kOffQ + kQBytes;                    // [buf][hi, lo]
  static constexpr uint32_t kOffTail = kOffP + 2 * kPBufs * kPBytes;
  static constexpr uint32_t kSmem = 1024 + kOffTail + kTailBytes;
  static constexpr int kOTiles = KVEQ ? 3 : 2;
  // TMEM columns: O tiles, then two score buffers
  static constexpr uint32_t kColS = kOTiles * NP;
  static constexpr uint32_t kColsUsed = (kOTiles + 2) * NP;
  static constexpr uint32_t kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64
                                      : kColsUsed <= 128 ? 128 : 256;
  static_assert(NP % 16 == 0 && NP >= 16 && NP <= 64, "rows per block");
  static_assert(kColsUsed <= 256, "TMEM columns");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// A row's exponentials are taken against a reference maximum that moves only
// when the block maximum exceeds it by more than 2^kLazy (in the log2 domain),
// so the running output is rescaled in TMEM only then; p <= 2^kLazy.
constexpr float kLazy = 8.f;
constexpr int kMaxSplitPages = 256;          // page ids of one split kept in shared memory

struct TaArgs {
  int q, Hq, Hkv, G, max_pages, num_pages, window, split, n_splits_grid, rows;
  const uint16_t* qrot;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* part_o;
  float* part_ml;
  unsigned* status;
  float scale_log2;
};

// v[0..31] per lane in, lane l out: the max (or sum) over the warp's 32 lanes
// of column l.  Each round halves the columns a lane keeps; the pairing is
// by lane bit 4, 3, 2, 1, 0 for every column, so every column gets the same
// reduction tree.
template <bool MAX>
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int off = 16 >> r;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = up ? v[j] : v[j + off];
      const float keep = up ? v[j + off] : v[j];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[j] = MAX ? fmaxf(keep, got) : __fadd_rn(keep, got);
    }
  }
  return v[0];
}

// Value dims held by TMEM lane quadrant `quad` of O tile `t`: first dim, or -1.
// Key-equals-value tiles: [K0;K1] dims 0..127, [K2;K3] dims 128..255 (the
// rotated dims 0..31 and 128..159 there hold post-RoPE keys and are not
// values), [SB;-] lanes 0..31 = dims 0..31, lanes 32..63 = dims 128..159.
template <bool KVEQ>
__device__ __forceinline__ int o_dim0(int t, int quad) {
  if (!KVEQ) return t * 128 + quad * 32;
  if (t < 2) return quad == 0 ? -1 : t * 128 + quad * 32;
  return quad == 0 ? 0 : (quad == 1 ? 128 : -1);
}

template <bool KVEQ, int NP>
__global__ void __launch_bounds__(kTaThreads, 1) attn_tc_kernel(
    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, TaArgs a) {
  using C = TaCfg<KVEQ, NP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ks = smem;                      // [2][K atoms (+ side-band)]
  uint8_t* vb = smem + C::kOffV;           // separate-K/V values
  uint8_t* qs = smem + C::kOffQ;
  uint8_t* pbase = smem + C::kOffP;        // P_hi of buffer u at u * 2 * kPBytes, P_lo after it
  uint8_t* tail = smem + C::kOffTail;
  uint64_t* ks_full = reinterpret_cast<uint64_t*>(tail);   // [2]
  uint64_t* ks_empty = ks_full + 2;                         // [2]
  uint64_t* v_full = ks_empty + 2;
  uint64_t* v_empty = v_full + 1;
  uint64_t* s_full = v_empty + 1;                           // [2] per score buffer
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* o_full = pv_done + 1;
  uint64_t* q_full = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
  volatile int* fail = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tail + 256);       // [4][64]
  float* m_sh = red + 4 * 64;                               // [64] reference max of each row
  float* al_sh = m_sh + 64;                                 // [64] rescale factor of the block
  int* rpos = reinterpret_cast<int*>(al_sh + 64);           // [64] position of each row
  int* pid_sh = rpos + 64;                                  // [kMaxSplitPages] page ids

  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, kvh = blockIdx.y % a.Hkv, rb = blockIdx.y / a.Hkv;
  const int L = a.seq_lens[b];
  if (L < 0 || L + a.q > a.max_pages * kPg) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0 && rb == 0)
      flag_status(a.status, SPEC_DEV_BAD_LENGTH);
    return;
  }
  const int klo = a.window > 0 ? max(0, L - a.window + 1) : 0;
  const int khi = L + a.q - 1;
  const int s_abs = klo / a.split + blockIdx.x;
  if (s_abs * a.split > khi) return;   // beyond this sequence's last split
  const int lo = max(s_abs * a.split, klo);
  const int hi = min(s_abs * a.split + a.split - 1, khi);
  const int blk0 = lo / kBlk, nb = hi / kBlk - blk0 + 1;
  const int r0 = rb * NP;
  const int nrows = min(NP, a.rows - r0);
  const int32_t* bt = a.block_table + (long)b * a.max_pages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ks_full[i], 1);
      mbar_init(&ks_empty[i], 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 1);
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(q_full, 1);
    *fail = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // cache page of absolute page index pg if it holds keys of [lo, hi]: its id,
  // -1 when it is not needed, -2 when the block table entry is invalid
  auto page_of = [&](int pg) -> int {
    if (pg * kPg > hi || pg * kPg + kPg - 1 < lo) return -1;
    const int id = bt[pg];
    return (id >= 0 && id < a.num_pages) ? id : -2;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      const uint64_t pol = policy_evict_first();
      auto load_ks = [&](int j) {
        const int slot = j & 1;
        uint8_t* dst = ks + slot * C::kKsBytes;
        int id[2];
        uint32_t bytes = 0;
        for (int h = 0; h < 2; ++h) {
          id[h] = page_of((blk0 + j) * 2 + h);
          if (id[h] == -2) flag_status(a.status, SPEC_DEV_BAD_PAGE);
          if (id[h] >= 0) bytes += (KVEQ ? 5u : 4u) * kHalfAtom;
        }
        mbar_arrive_expect_tx(&ks_full[slot], bytes);
        for (int h = 0; h < 2; ++h) {
          if (id[h] < 0) continue;
          const int y = (id[h] * a.Hkv + kvh) * kPg;
          for (int at = 0; at < 4; ++at)
            tma_load_2d(dst + at * kAtom + h * kHalfAtom, &tk, &ks_full[slot], at * 64, y, pol);
          if (KVEQ) tma_load_2d(dst + 4 * kAtom + h * kHalfAtom, &tv, &ks_full[slot], 0, y, pol);
        }
      };
      auto load_v = [&](int j) {
        int id[2];
        uint32_t bytes = 0;
        for (int h = 0; h < 2; ++h) {
          id[h] = page_of((blk0 + j) * 2 + h);
          if (id[h] >= 0) bytes += 4u * kHalfAtom;
        }
        mbar_arrive_expect_tx(v_full, bytes);
        for (int h = 0; h < 2; ++h) {
          if (id[h] < 0) continue;
          const int y = (id[h] * a.Hkv + kvh) * kPg;
          for (int at = 0; at < 4; ++at)
            tma_load_2d(vb + at * kAtom + h * kHalfAtom, &tv, v_full, at * 64, y, pol);
        }
      };
      int ks_issued = 0, v_issued = 0;
      if (KVEQ) {
        for (int j = 0; j < nb; ++j) {
          if (j >= 2 && (*fail || !mbar_wait(&ks_empty[j & 1], ((j >> 1) - 1) & 1, a.status))) {
            *fail = 1;
            break;
          }
          load_ks(j);
          ks_issued = j + 1;
        }
      } else {
        // keys run two blocks ahead of values: K slot j+2 frees when QK_j is
        // done, the value buffer when PV_j is done
        load_ks(0);
        ks_issued = 1;
        if (nb > 1) {
          load_ks(1);
          ks_issued = 2;
        }
        for (int j = 0; j < nb; ++j) {
          if (j >= 1 && (*fail || !mbar_wait(v_empty, (j - 1) & 1, a.status))) {
            *fail = 1;
            break;
          }
          load_v(j);
          v_issued = j + 1;
          if (j + 2 < nb) {
            if (*fail || !mbar_wait(&ks_empty[j & 1], (j >> 1) & 1, a.status)) {
              *fail = 1;
              break;
            }
            load_ks(j + 2);
            ks_issued = j + 3;
          }
        }
      }
      // every issued copy has landed before the CTA may exit
      for (int j = (ks_issued > 2 ? ks_issued - 2 : 0); j < ks_issued; ++j)
        mbar_wait(&ks_full[j & 1], (j >> 1) & 1, a.status);
      if (v_issued > 0) mbar_wait(v_full, (v_issued - 1) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // order: QK_0, then per block j: QK_{j+1} (other score buffer, as soon as
    // its keys landed), wait for P_j, PV_j.  The tensor core thus computes the
    // next scores while the softmax works on the current ones.
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(NP);
      const uint32_t id_pv = idesc_bf16(NP, true);
      const uint32_t q_addr = smem_u32(qs);
      const uint32_t p_addr = smem_u32(pbase);
      auto issue_qk = [&](int j) -> bool {
        if (*fail || !mbar_wait(&ks_full[j & 1], (j >> 1) & 1, a.status)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(ks + (j & 1) * C::kKsBytes);
        const uint32_t t_s = tmem + C::kColS + (j & 1) * NP;
#pragma unroll
        for (int kk = 0; kk < kDim / 16; ++kk)   // K = 16 dims per MMA
          umma_bf16(t_s, sw128_desc(k_addr + (kk >> 2) * kAtom + (kk & 3) * 32),
                    sw128_desc(q_addr + (kk >> 2) * (NP * 128) + (kk & 3) * 32), id_qk, kk > 0);
        umma_commit(&s_full[j & 1]);
        if (!KVEQ) umma_commit(&ks_empty[j & 1]);   // keys no longer needed
        return true;
      };
      bool ok = mbar_wait(q_full, 0, a.status) && (nb < 1 || issue_qk(0));
      for (int j = 0; ok && j < nb; ++j) {
        if (j + 1 < nb && !issue_qk(j + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(p_full, j & 1, a.status) ||
            (!KVEQ && !mbar_wait(v_full, j & 1, a.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t v_addr = KVEQ ? smem_u32(ks + (j & 1) * C::kKsBytes) : smem_u32(vb);
        const uint32_t ph_addr = p_addr + (j % C::kPBufs) * 2 * C::kPBytes;
        const uint32_t pl_addr = ph_addr + C::kPBytes;
#pragma unroll
        for (int t = 0; t < C::kOTiles; ++t) {
          // [atom 2t ; atom 2t+1] (the side-band tile pairs its atom with the
          // next 16 KB of shared memory, whose lanes are never read)
          const uint32_t a0 = v_addr + 2 * t * kAtom;
#pragma unroll
          for (int kk = 0; kk < kBlk / 16; ++kk) {   // K = 16 keys per MMA
            const uint64_t ad = sw128_desc_mn(a0 + kk * 2048, kAtom);
            const uint32_t po = (kk >> 2) * (NP * 128) + (kk & 3) * 32;
            umma_bf16(tmem + t * NP, ad, sw128_desc(ph_addr + po), id_pv, (j > 0 || kk > 0));
            umma_bf16(tmem + t * NP, ad, sw128_desc(pl_addr + po), id_pv, 1u);
          }
        }
        umma_commit(pv_done);
        umma_commit(KVEQ ? &ks_empty[j & 1] : v_empty);
      }
      if (!ok) *fail = 1;
      umma_commit(o_full);
      // nothing may be in flight when TMEM is freed
      mbar_wait(o_full, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int ctid = threadIdx.x - 64;       // 0..127
    const int quad = warp & 3;               // TMEM lanes 32*quad ..
    const int t = quad * 32 + lane;          // key of the block / O lane
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);

    // Q rows of this block -> K-major swizzled tile (zero padding rows)
    for (int idx = ctid; idx < NP * (kDim / 8); idx += 128) {
      const int r = idx / (kDim / 8), c = idx % (kDim / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nrows) {
        const int rg = r0 + r, gh = rg / a.q, i = rg % a.q;
        const int h = kvh * a.G + gh;
        v = *reinterpret_cast<const uint4*>(a.qrot + (((long)b * a.q + i) * a.Hq + h) * kDim + c * 8);
      }
      *reinterpret_cast<uint4*>(qs + (c >> 3) * (NP * 128) + swz128(r, c & 7)) = v;
    }
    if (ctid < NP) rpos[ctid] = ctid < nrows ? L + (r0 + ctid) % a.q : -1;
    // cache page ids of the split's pages (-1 / -2: not loaded)
    for (int i = ctid; i < 2 * nb; i += 128) pid_sh[i] = page_of(2 * blk0 + i);
    float m_ref = -INFINITY, l_run = 0.f;    // row ctid (ctid < NP)
    fence_proxy_async_smem();
    named_bar(1, 128);
    if (ctid == 0) mbar_arrive(q_full);

    for (int j = 0; j < nb; ++j) {
      bool ok = !*fail && mbar_wait(&s_full[j & 1], (j >> 1) & 1, a.status);
      ok = __all_sync(0xffffffffu, ok);   // TMEM loads are warp-collective
      if (!ok) *fail = 1;
      tc_fence_after();
      const int key = (blk0 + j) * kBlk + t;
      const bool in_range = key >= lo && key <= hi && pid_sh[2 * j + (t >> 6)] >= 0;
      float s[NP];
      if (ok) {
#pragma unroll
        for (int c0 = 0; c0 < NP; c0 += 16) {
          uint32_t r[16];
          tmem_ld16_nowait(tq + C::kColS + (j & 1) * NP + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c0 + i] = __uint_as_float(r[i]);
        }
      }
#pragma unroll
      for (int r = 0; r < NP; ++r) {
        const int p = rpos[r];
        const bool vis = ok && in_range && key <= p && (a.window == 0 || key > p - a.window);
        s[r] = vis ? __fmul_rn(s[r], a.scale_log2) : -INFINITY;
      }
      // ---- row maxima of the block -> reference maxima
#pragma unroll
      for (int c0 = 0; c0 < NP; c0 += 32) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = (c0 + i < NP) ? s[c0 + i] : -INFINITY;
        const float mx = transpose_reduce32<true>(v, lane);
        if (c0 + lane < NP) red[quad * 64 + c0 + lane] = mx;
      }
      named_bar(1, 128);
      if (ctid < NP) {
        const float mb = fmaxf(fmaxf(red[ctid], red[64 + ctid]), fmaxf(red[128 + ctid], red[192 + ctid]));
        float al = 1.f;
        if (m_ref == -INFINITY) {
          m_ref = mb;                          // nothing accumulated yet: no rescale
        } else if (mb > __fadd_rn(m_ref, kLazy)) {
          al = exp2f(__fsub_rn(m_ref, mb));
          m_ref = mb;
        }
        m_sh[ctid] = m_ref;
        al_sh[ctid] = al;
      }
      named_bar(1, 128);
      // ---- probabilities and the block's row sums
      float p[NP];
#pragma unroll
      for (int r = 0; r < NP; ++r)
        p[r] = (s[r] == -INFINITY) ? 0.f : exp2f(__fsub_rn(s[r], m_sh[r]));
#pragma unroll
      for (int c0 = 0; c0 < NP; c0 += 32) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = (c0 + i < NP) ? p[c0 + i] : 0.f;
        const float sm = transpose_reduce32<false>(v, lane);
        if (c0 + lane < NP) red[quad * 64 + c0 + lane] = sm;
      }
      bool moved = false;
#pragma unroll
      for (int r = 0; r < NP; ++r) moved |= al_sh[r] != 1.f;
      // PV of the previous block must be done before its P buffer is
      // rewritten (single buffer) or its output is rescaled
      if (ok && j > 0 && (C::kPBufs == 1 || moved)) ok = mbar_wait(pv_done, (j - 1) & 1, a.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) *fail = 1;
      // ---- P = P_hi + P_lo as bf16 (K-major tiles: row r, key t)
      {
        uint8_t* ph = pbase + (j % C::kPBufs) * 2 * C::kPBytes;
        uint8_t* pl = ph + C::kPBytes;
        const uint32_t off = (t >> 6) * (NP * 128) + ((t & 7) << 1);
        const uint32_t ch = (t & 63) >> 3;
#pragma unroll
        for (int r = 0; r < NP; ++r) {
          const uint16_t hb = f32_to_bf16(p[r]);
          const uint16_t lb = f32_to_bf16(__fsub_rn(p[r], bf16_to_f32(hb)));
          const uint32_t o = off + swz128(r, ch);
          *reinterpret_cast<uint16_t*>(ph + o) = hb;
          *reinterpret_cast<uint16_t*>(pl + o) = lb;
        }
      }
      // ---- value rows of keys outside the valid range: zero them
      if (ok && !in_range && (KVEQ || mbar_wait(v_full, j & 1, a.status))) {
        // (separate values: their copy must have landed first)
        uint8_t* base = KVEQ ? ks + (j & 1) * C::kKsBytes : vb;
        const int n_at = KVEQ ? 5 : 4;
        for (int at = 0; at < n_at; ++at)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(base + at * kAtom + t * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      // ---- rescale the running output of rows whose reference max moved
      if (ok && j > 0 && moved) {
#pragma unroll
        for (int tt = 0; tt < C::kOTiles; ++tt) {
          if (o_dim0<KVEQ>(tt, quad) < 0) continue;
#pragma unroll
          for (int c0 = 0; c0 < NP; c0 += 16) {
            uint32_t r[16];
            tmem_ld16_nowait(tq + tt * NP + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[i]), al_sh[c0 + i]));
            tmem_st16(tq + tt * NP + c0, r);
          }
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar(1, 128);
      if (ctid < NP) {
        const float rs = __fadd_rn(__fadd_rn(red[ctid], red[64 + ctid]), __fadd_rn(red[128 + ctid], red[192 + ctid]));
        l_run = __fadd_rn(__fmul_rn(l_run, al_sh[ctid]), rs);
      }
      if (ctid == 0) mbar_arrive(p_full);
      named_bar(1, 128);   // red / m_sh / al_sh are rewritten by the next block
    }

    // ---- partial (o unnormalised, m and l in the log2 domain) of each row
    const bool ok = __all_sync(0xffffffffu, !*fail && mbar_wait(o_full, 0, a.status));
    tc_fence_after();
    if (ok) {
      const long slot = ((long)(b * a.Hkv + kvh) * a.n_splits_grid + blockIdx.x) * a.rows + r0;
#pragma unroll
      for (int tt = 0; tt < C::kOTiles; ++tt) {
        const int d0 = o_dim0<KVEQ>(tt, quad);
        if (d0 < 0) continue;
        const int dim = d0 + lane;
#pragma unroll
        for (int c0 = 0; c0 < NP; c0 += 16) {
          uint32_t r[16];
          tmem_ld16_nowait(tq + tt * NP + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < nrows) __stcg(a.part_o + (slot + c0 + i) * kDim + dim, __uint_as_float(r[i]));
        }
      }
      if (ctid < nrows)
        __stcg(reinterpret_cast<float2*>(a.part_ml + (slot + ctid) * 2), make_float2(m_ref, l_run));
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

template <bool KVEQ, int NP>
cudaError_t launch_ta(const AttnGeom& g, int row_blocks, const CUtensorMap& tk, const CUtensorMap& tv,
                      const TaArgs& a, cudaStream_t st) {
  using C = TaCfg<KVEQ, NP>;
  auto kern = attn_tc_kernel<KVEQ, NP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(g.n_splits_grid, g.n_kv_heads * row_blocks, g.B), dim3(kTaThreads),
                  C::kSmem, st, tk, tv, a);
}

int ta_np(const AttnGeom& g) {
  if (!g.kv_equal) return 16;
  const int r = std::min(g.rows, 48);
  return (r + 15) / 16 * 16;
}

}  // namespace

// Opt-in (SPECVERIFY_TC_ATTN=1): at the verify shapes measured so far (8 to
// 40 query rows per KV head) the mma.sync kernel is faster, because the
// skinny tcgen05 MMAs and the per-block softmax chain leave the tensor core
// and the load pipe idle most of the time.
bool attn_tc_supported(const AttnGeom& g) {
  static const bool on = [] {
    const char* v = getenv("SPECVERIFY_TC_ATTN");
    const char* off = getenv("SPECVERIFY_NO_TC");
    return v && v[0] == '1' && !(off && off[0] == '1');
  }();
  return on && g.qpos_off == 0 && g.kend_off == g.q - 1 &&   // verify rows only
         g.head_dim == kDim && g.page_size == kPg && g.split_tokens % kBlk == 0 &&
         g.split_tokens <= kPg * kMaxSplitPages && (!g.kv_equal || g.sb_width == 64);
}

cudaError_t launch_attn_tc(const AttnGeom& g, const CUtensorMap& tk, const CUtensorMap& tv,
                           const uint16_t* qrot, const int32_t* block_table, const int32_t* seq_lens,
                           float* part_o, float* part_ml, unsigned* status, float scale_log2,
                           cudaStream_t st) {
  if (!attn_tc_supported(g)) return cudaErrorInvalidValue;
  TaArgs a{};
  a.q = g.q;
  a.Hq = g.n_q_heads;
  a.Hkv = g.n_kv_heads;
  a.G = g.n_q_heads / g.n_kv_heads;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.window = g.window;
  a.split = g.split_tokens;
  a.n_splits_grid = g.n_splits_grid;
  a.rows = g.rows;
  a.qrot = qrot;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.status = status;
  a.scale_log2 = scale_log2;
  const int np = ta_np(g);
  const int row_blocks = (g.rows + np - 1) / np;
  if (!g.kv_equal) return launch_ta<false, 16>(g, row_blocks, tk, tv, a, st);
  switch (np) {
    case 16: return launch_ta<true, 16>(g, row_blocks, tk, tv, a, st);
    case 32: return launch_ta<true, 32>(g, row_blocks, tk, tv, a, st);
    case 48: return launch_ta<true, 48>(g, row_blocks, tk, tv, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sv

// Split-KV verify attention on the 5th-generation tensor cores (sm_100a),
// head_dim 256, persistent.
//
// Work item = (sequence b, KV head, row block, absolute split of split_tokens
// keys).  Items are ordered (b, kv head, row block, split) and every CTA (one
// per SM) takes a contiguous range of them, so consecutive items mostly share
// their queries; its producer streams their keys without a break between
// items.  10 warps:
//   warp 0    TMA producer.  Keys arrive in blocks of 128 (two 64-token pages)
//             as four 128 x 64 swizzled atoms; on key-equals-value layers the
//             side-band atom (pre-RoPE rotated dims) rides with the keys (two
//             stages), on separate-K/V layers keys have two stages and values
//             one buffer.  Queries come by a 3D TMA box {64 dims, G heads, PB
//             positions} straight from the rotated-query buffer, once per
//             (b, kv head, row block).
//   warp 1    allocates TMEM and issues the MMAs (one thread):
//               S^T[128 keys][NP rows] = K . Q^T          (A = K, K-major)
//               O^T[dims][NP rows]    += V^T . P^T        (A = V^T, MN-major)
//             accumulators in TMEM (lane = key or value dim, column = query
//             row); the scores of the next block are computed while the
//             softmax works on the current one (two score buffers), and the
//             output has two buffers by item parity, so P . V of an item's
//             first block never waits for the previous item's read-out.
//   warps 2-9 softmax: thread t of a lane quadrant owns key t of the block;
//             the warps of one half of the columns (query rows) form a group
//             of 128 threads.  Per block: the scores of the thread's key for
//             its NP/2 rows; p = 2^(s - m) against a per-row reference maximum
//             m that moves only when a block maximum exceeds it by more than
//             2^8 (one OR-vote per block decides; the exact block maxima are
//             reduced only then, and the running output is rescaled in TMEM
//             only for rows that moved); p is written once as bf16 for P . V
//             and summed unrounded into per-thread row sums, reduced over the
//             keys at the end of the item, when (m, l) go out; the item's o is
//             read out of TMEM one block later, after the next item's first
//             block.  The partials go out in the layout the split combine reads.
//
// Value rows of keys outside the item's range (or on pages that were not
// loaded) are zeroed in shared memory before P . V, so stale or poisoned
// slots never reach it.  Keys are visited in blocks at absolute 128-key
// boundaries; a row's reference maximum, its probabilities and the reduction
// trees depend only on its own scores and absolute key positions, so a row's
// partial does not depend on k, the batch, its row slot or the CTA that
// computed it.  Every wait is bounded; after a timeout the CTA stops issuing
// work, drains what it issued, writes nothing and frees its TMEM.
#include <math.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sv {

namespace {

constexpr int kBlk = 128;                    // keys per MMA block
constexpr int kPg = 64;                      // tokens per page
constexpr int kDim = 256;                    // head_dim of this kernel
constexpr uint32_t kAtom = kBlk * 128;       // 128 keys x 64 dims of bf16: 16 KB
constexpr uint32_t kHalfAtom = kPg * 128;    // one page's rows of an atom: 8 KB
constexpr int kSoftWarps = 8;
constexpr int kFaThreads = (2 + kSoftWarps) * 32;
constexpr uint32_t kSmemMax = 227u * 1024u;
constexpr uint32_t kTailBytes = 4096;
// p <= 2^kLazy: a row's reference maximum moves only when a block maximum
// exceeds it by more than this (log2 domain)
constexpr float kLazy = 8.f;
constexpr int kMaxItemPages = 128;           // pages one item (split) may span
// Reference maximum of a row that has seen no key yet: finite, so that
// 2^(s - m) is exactly 0 for a masked score (s = -inf) and any visible score
// exceeds it by more than the lazy margin.  A partial whose rows saw no key
// carries m = kNoKey, l = 0, o = 0, which the split combine weighs by
// 2^(kNoKey - M) = 0.
constexpr float kNoKey = -1e30f;

// 2^x (the hardware approximation, relative error ~2^-22; 2^-inf = +0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool KVEQ, int NP>
struct FaCfg {
  static constexpr uint32_t kStage = 4 * kAtom + (KVEQ ? kAtom : 0);   // keys (+ side-band)
  static constexpr uint32_t kVBytes = KVEQ ? 0 : 4 * kAtom;           // separate values
  static constexpr uint32_t kQBytes = 4u * NP * 128u;
  static constexpr uint32_t kPBytes = 2u * NP * 128u;                 // [NP rows][128 keys]
  static constexpr uint32_t bytes(int pb, int qb) {
    return 1024u + 2u * kStage + kVBytes + pb * kPBytes + qb * kQBytes + kTailBytes;
  }
  static constexpr int kPBufs = bytes(2, 1) <= kSmemMax ? 2 : 1;
  static constexpr int kQBufs = bytes(kPBufs, 2) <= kSmemMax ? 2 : 1;
  static constexpr uint32_t kOffV = 2 * kStage;
  static constexpr uint32_t kOffP = kOffV + kVBytes;
  static constexpr uint32_t kOffQ = kOffP + kPBufs * kPBytes;
  static constexpr uint32_t kOffTail = kOffQ + kQBufs * kQBytes;
  static constexpr uint32_t kSmem = 1024 + kOffTail + kTailBytes;
  static constexpr int kOTiles = KVEQ ? 3 : 2;
  static constexpr int kOBufs = 2;                       // output accumulators (by item parity)
  static constexpr uint32_t kColS = kOBufs * kOTiles * NP;   // two score buffers after the outputs
  static constexpr uint32_t kCols = kColS + 2 * NP;
  static constexpr uint32_t kTmemCols =
      kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(NP % 16 == 0 && NP >= 16 && NP <= 64, "rows per block");
  static_assert(kCols <= 512, "tensor memory");
  static_assert(kSmem <= kSmemMax, "shared memory");
  // the side-band MMA pairs each side-band atom with the next 16 KB of shared
  // memory (lanes never read); for the second stage that is what follows it
  static_assert(!KVEQ || kOffTail + kTailBytes >= 2 * kStage + kAtom, "side-band pairing");
};

struct FaArgs {
  int B, q, Hq, Hkv, G, max_pages, num_pages, window, split, n_splits_grid, rows;
  int qpos_off, kend_off;
  int PB, RB;                 // query positions per row block, row blocks per KV head
  int lgG;                    // log2 G (G is a power of two)
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* part_o;
  float* part_ml;
  unsigned* status;
  float scale_log2;
};

// Keys any row of sequence b may see and the number of absolute splits they
// touch (0 for an invalid length: the combine then writes zeros).
__device__ __forceinline__ int seq_splits(const FaArgs& a, int L, int& klo, int& khi) {
  klo = a.window > 0 ? max(0, L + a.qpos_off - a.window + 1) : 0;
  khi = L + a.kend_off;
  if (L < 0 || L + a.q > a.max_pages * kPg || khi < klo) return 0;
  return khi / a.split - klo / a.split + 1;
}

// Walks this CTA's items in order.  Every role keeps its own walker; all
// walkers see the same sequence.
struct Walker {
  const FaArgs* a;
  int b, kvh, rb, sidx, ns, L, lo, hi, blk0, nb;
  bool new_q;           // this item's queries differ from the previous item's
  __device__ void load_seq() {
    L = a->seq_lens[b];
    int klo, khi;
    ns = seq_splits(*a, L, klo, khi);
  }
  __device__ void derive() {
    int klo, khi;
    seq_splits(*a, L, klo, khi);
    const int s_abs = klo / a->split + sidx;
    lo = max(s_abs * a->split, klo);
    hi = min(s_abs * a->split + a->split - 1, khi);
    blk0 = lo / kBlk;
    nb = hi / kBlk - blk0 + 1;
  }
  __device__ void start(const FaArgs* args, int b0, int kvh0, int rb0, int s0) {
    a = args;
    b = b0;
    kvh = kvh0;
    rb = rb0;
    sidx = s0;
    load_seq();
    derive();
    new_q = true;
  }
  __device__ void next() {
    new_q = false;
    if (++sidx < ns) {
      derive();
      return;
    }
    sidx = 0;
    new_q = true;
    if (++rb < a->RB) {
      derive();
      return;
    }
    rb = 0;
    if (++kvh < a->Hkv) {
      derive();
      return;
    }
    kvh = 0;
    do {
      ++b;
      if (b >= a->B) return;   // past the last item; callers stop by count
      load_seq();
    } while (ns == 0);
    derive();
  }
};

// v[0..31] per lane in, lane l out: the max (or sum) over the warp's 32 lanes
// of column l.  Each round halves the columns a lane keeps; the pairing is by
// lane bit 4, 3, 2, 1, 0 for every column, so every column gets the same
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

// Bounded wait that gives up at once after an earlier timeout in the CTA.
__device__ __forceinline__ bool fwait(uint64_t* bar, uint32_t parity, unsigned* status,
                                      volatile int* fail) {
  if (*fail) return false;
  if (mbar_wait(bar, parity, status)) return true;
  *fail = 1;
  return false;
}

template <bool KVEQ, int NP>
__global__ void __launch_bounds__(kFaThreads, 1) attn_fa_kernel(
    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ FaArgs a) {
  using C = FaCfg<KVEQ, NP>;
  constexpr int NH = NP / 2;                 // columns (query rows) per softmax half
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage = smem;                     // [2][K atoms (+ side-band)]
  uint8_t* vbuf = smem + C::kOffV;           // separate-K/V values
  uint8_t* pbuf = smem + C::kOffP;           // [kPBufs][P]
  uint8_t* qbuf = smem + C::kOffQ;           // [kQBufs][Q]
  uint8_t* tail = smem + C::kOffTail;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(tail);    // [2]
  uint64_t* k_empty = k_full + 2;                           // [2]
  uint64_t* v_full = k_empty + 2;
  uint64_t* v_empty = v_full + 1;
  uint64_t* q_full = v_empty + 1;                           // [2]
  uint64_t* q_empty = q_full + 2;                           // [2]
  uint64_t* s_full = q_empty + 2;                           // [2]
  uint64_t* p_full = s_full + 2;                            // [2] by block parity
  uint64_t* pv_done = p_full + 2;                           // [2] by block parity
  uint64_t* o_free = pv_done + 2;                           // [2] by item parity
  uint64_t* mma_done = o_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* fail = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* start = reinterpret_cast<int*>(tmem_slot + 4);      // b, kvh, rb, sidx, count
  float* red = reinterpret_cast<float*>(tail + 256);       // [2 halves][2 bufs][4 quads][32]
  int* pvalid_all = reinterpret_cast<int*>(red + 512);      // [2][kMaxItemPages] page validity of an item

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&pv_done[i], 1);
      mbar_init(&p_full[i], kSoftWarps);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(&o_free[0], kSoftWarps);
    mbar_init(&o_free[1], kSoftWarps);
    mbar_init(mma_done, 1);
    *fail = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&tq);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  pdl_trigger();
  pdl_wait();

  // ---- this CTA's items: [i0, i1) of the (b, kvh, rb, split) list
  if (warp == 2) {
    const int per_b = a.Hkv * a.RB;
    long total = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      int klo, khi, n = 0;
      if (b0 + lane < a.B) n = seq_splits(a, a.seq_lens[b0 + lane], klo, khi);
      if (n == 0 && b0 + lane < a.B && blockIdx.x == 0) {
        const int L = a.seq_lens[b0 + lane];
        if (L < 0 || L + a.q > a.max_pages * kPg) flag_status(a.status, SPEC_DEV_BAD_LENGTH);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
      total += (long)n * per_b;
    }
    const long i0 = (long)blockIdx.x * total / gridDim.x;
    const long i1 = (long)(blockIdx.x + 1) * total / gridDim.x;
    // locate item i0
    long pre = 0;
    int found_b = -1;
    long found_pre = 0;
    for (int b0 = 0; b0 < a.B && found_b < 0 && i1 > i0; b0 += 32) {
      int klo, khi, n = 0;
      if (b0 + lane < a.B) n = seq_splits(a, a.seq_lens[b0 + lane], klo, khi);
      long c = (long)n * per_b, incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const long excl = pre + incl - c;
      const bool mine = c > 0 && i0 >= excl && i0 < excl + c;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (bal) {
        const int src = __ffs(bal) - 1;
        found_b = b0 + src;
        found_pre = __shfl_sync(0xffffffffu, excl, src);
      }
      pre += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      if (found_b >= 0) {
        int klo, khi;
        const int ns = seq_splits(a, a.seq_lens[found_b], klo, khi);
        const long rem = i0 - found_pre;
        start[0] = found_b;
        start[1] = (int)(rem / ((long)a.RB * ns));
        start[2] = (int)((rem / ns) % a.RB);
        start[3] = (int)(rem % ns);
        start[4] = (int)(i1 - i0);
      } else {
        start[4] = 0;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int count = start[4];
  const int32_t* bt_all = a.block_table;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && count > 0) {
      const uint64_t pol = policy_evict_first();
      const uint64_t pol_q = policy_evict_normal();
      Walker w;
      w.start(&a, start[0], start[1], start[2], start[3]);
      int gk = 0, gv = 0, nq = 0;
      auto page_id = [&](const Walker& it, int pg) -> int {   // -1 not needed, -2 invalid
        if (pg * kPg > it.hi || pg * kPg + kPg - 1 < it.lo) return -1;
        const int id = bt_all[(long)it.b * a.max_pages + pg];
        return (id >= 0 && id < a.num_pages) ? id : -2;
      };
      auto load_k = [&](const Walker& it, int j) -> bool {
        const int s = gk & 1;
        if (gk >= 2 && !fwait(&k_empty[s], ((gk >> 1) - 1) & 1, a.status, fail)) return false;
        uint8_t* dst = stage + s * C::kStage;
        int id[2];
        uint32_t bytes = 0;
        for (int h = 0; h < 2; ++h) {
          id[h] = page_id(it, (it.blk0 + j) * 2 + h);
          if (id[h] == -2) flag_status(a.status, SPEC_DEV_BAD_PAGE);
          if (id[h] >= 0) bytes += (KVEQ ? 5u : 4u) * kHalfAtom;
        }
        mbar_arrive_expect_tx(&k_full[s], bytes);
        for (int h = 0; h < 2; ++h) {
          if (id[h] < 0) continue;
          const int y = (id[h] * a.Hkv + it.kvh) * kPg;
#pragma unroll
          for (int at = 0; at < 4; ++at)
            tma_load_2d(dst + at * kAtom + h * kHalfAtom, &tk, &k_full[s], at * 64, y, pol);
          if (KVEQ) tma_load_2d(dst + 4 * kAtom + h * kHalfAtom, &tv, &k_full[s], 0, y, pol);
        }
        ++gk;
        return true;
      };
      auto load_v = [&](const Walker& it, int j) -> bool {
        if (gv >= 1 && !fwait(v_empty, (gv - 1) & 1, a.status, fail)) return false;
        int id[2];
        uint32_t bytes = 0;
        for (int h = 0; h < 2; ++h) {
          id[h] = page_id(it, (it.blk0 + j) * 2 + h);
          if (id[h] >= 0) bytes += 4u * kHalfAtom;
        }
        mbar_arrive_expect_tx(v_full, bytes);
        for (int h = 0; h < 2; ++h) {
          if (id[h] < 0) continue;
          const int y = (id[h] * a.Hkv + it.kvh) * kPg;
#pragma unroll
          for (int at = 0; at < 4; ++at)
            tma_load_2d(vbuf + at * kAtom + h * kHalfAtom, &tv, v_full, at * 64, y, pol);
        }
        ++gv;
        return true;
      };
      auto load_q = [&](const Walker& it) -> bool {
        const int qb = nq % C::kQBufs;
        if (nq >= C::kQBufs && !fwait(&q_empty[qb], ((nq / C::kQBufs) - 1) & 1, a.status, fail))
          return false;
        uint8_t* dst = qbuf + qb * C::kQBytes;
        mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
        const int z = it.b * a.q + it.rb * a.PB;
#pragma unroll
        for (int sub = 0; sub < 4; ++sub)
          tma_load_3d(dst + sub * (NP * 128), &tq, &q_full[qb], sub * 64, it.kvh * a.G, z, pol_q);
        ++nq;
        return true;
      };
      bool ok = true;
      if (KVEQ) {
        for (int i = 0; ok && i < count; ++i, w.next()) {
          if (w.new_q) ok = load_q(w);
          for (int j = 0; ok && j < w.nb; ++j) ok = load_k(w, j);
        }
      } else {
        // keys run up to two blocks ahead of the values (a key stage frees
        // when its scores are done, the value buffer when P . V is done)
        Walker wk = w;
        int ik = 0, jk = 0;          // next key block to load: item ik, block jk of wk
        auto key_ahead = [&](int limit) -> bool {   // load keys while gk < limit
          while (ik < count && gk < limit) {
            if (jk == 0 && wk.new_q && !load_q(wk)) return false;
            if (!load_k(wk, jk)) return false;
            if (++jk >= wk.nb) {
              jk = 0;
              ++ik;
              if (ik < count) wk.next();
            }
          }
          return true;
        };
        int gblk = 0;
        for (int i = 0; ok && i < count; ++i, w.next()) {
          for (int j = 0; ok && j < w.nb; ++j, ++gblk) {
            ok = key_ahead(gblk + 2) && load_v(w, j);
          }
        }
      }
      // every issued copy must land before the CTA may exit
      for (int i = (gk > 2 ? gk - 2 : 0); i < gk; ++i) mbar_wait(&k_full[i & 1], (i >> 1) & 1, a.status);
      if (gv > 0) mbar_wait(v_full, (gv - 1) & 1, a.status);
      for (int i = (nq > C::kQBufs ? nq - C::kQBufs : 0); i < nq; ++i)
        mbar_wait(&q_full[i % C::kQBufs], (i / C::kQBufs) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && count > 0) {
      const uint32_t id_qk = idesc_bf16(NP);
      const uint32_t id_pv = idesc_bf16(NP, true);
      // The scores of block g (QK) and the product P . V of block g - 1 are
      // independent: each is issued as soon as its inputs are ready (polled
      // with the non-blocking test, P . V first), so P . V never waits for
      // the next block's keys (which, on key-equals-value layers, could not be
      // requested before that P . V frees its stage).
      //   QK(g):  keys of g landed; score buffer g % 2 read by the softmax
      //           (g <= npv + 1); new queries landed at a query-group start.
      //   PV(g):  P(g) written; values landed (separate-K/V); at an item's
      //           first block, the output buffer of two items back read out.
      Walker ws, wp;
      ws.start(&a, start[0], start[1], start[2], start[3]);
      wp = ws;
      int is = 0, js = 0, ip = 0, jp = 0;   // QK / PV positions: item, block in item
      int nqk = 0, npv = 0, nq_used = -1;
      uint64_t t_last = globaltimer_ns();
      uint32_t polls = 0;
      while (ip < count) {
        bool progressed = false;
        // P . V first: it frees a stage for the next copy
        if (npv < nqk) {
          bool ready = mbar_test_wait(&p_full[npv & 1], (npv >> 1) & 1);
          if (!KVEQ) ready = ready && mbar_test_wait(v_full, npv & 1);
          if (jp == 0 && ip >= 2) ready = ready && mbar_test_wait(&o_free[ip & 1], ((ip >> 1) - 1) & 1);
          if (ready) {
            tc_fence_after();
            const uint32_t v_addr = KVEQ ? smem_u32(stage + (npv & 1) * C::kStage) : smem_u32(vbuf);
            const uint32_t p_addr = smem_u32(pbuf + (npv % C::kPBufs) * C::kPBytes);
            const uint32_t t_o = tmem + (ip & 1) * (C::kOTiles * NP);
#pragma unroll
            for (int t = 0; t < C::kOTiles; ++t) {
              // [atom 2t ; atom 2t+1] (the side-band tile pairs its atom with the
              // next 16 KB of shared memory, whose lanes are never read)
              const uint32_t a0 = v_addr + 2 * t * kAtom;
#pragma unroll
              for (int kk = 0; kk < kBlk / 16; ++kk) {   // K = 16 keys per MMA
                const uint64_t ad = sw128_desc_mn(a0 + kk * 2048, kAtom);
                const uint32_t po = (kk >> 2) * (NP * 128) + (kk & 3) * 32;
                umma_bf16(t_o + t * NP, ad, sw128_desc(p_addr + po), id_pv, (jp > 0 || kk > 0) ? 1u : 0u);
              }
            }
            umma_commit(&pv_done[npv & 1]);
            umma_commit(KVEQ ? &k_empty[npv & 1] : v_empty);
            ++npv;
            if (++jp >= wp.nb) {
              jp = 0;
              ++ip;
              if (ip < count) wp.next();
            }
            progressed = true;
          }
        }
        if (is < count && nqk <= npv + 1) {
          const bool newq = js == 0 && ws.new_q;
          const int qb = (nq_used + 1) % C::kQBufs;
          bool ready = !newq || mbar_test_wait(&q_full[qb], ((nq_used + 1) / C::kQBufs) & 1);
          ready = ready && mbar_test_wait(&k_full[nqk & 1], (nqk >> 1) & 1);
          if (ready) {
            if (newq) ++nq_used;
            tc_fence_after();
            const int s = nqk & 1;
            const uint32_t k_addr = smem_u32(stage + s * C::kStage);
            const uint32_t q_addr = smem_u32(qbuf + (nq_used % C::kQBufs) * C::kQBytes);
            const uint32_t t_s = tmem + C::kColS + s * NP;
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk)   // K = 16 dims per MMA
              umma_bf16(t_s, sw128_desc(k_addr + (kk >> 2) * kAtom + (kk & 3) * 32),
                        sw128_desc(q_addr + (kk >> 2) * (NP * 128) + (kk & 3) * 32), id_qk, kk > 0);
            umma_commit(&s_full[s]);
            if (!KVEQ) umma_commit(&k_empty[s]);     // keys no longer needed
            // last block of the last item of this query group: release the queries
            bool last_of_group = false;
            if (js + 1 >= ws.nb) {
              if (is + 1 >= count) {
                last_of_group = true;
              } else {
                Walker peek = ws;
                peek.next();
                last_of_group = peek.new_q;
              }
            }
            if (last_of_group) umma_commit(&q_empty[nq_used % C::kQBufs]);
            ++nqk;
            if (++js >= ws.nb) {
              js = 0;
              ++is;
              if (is < count) ws.next();
            }
            progressed = true;
          }
        }
        if (progressed) {
          polls = 0;
        } else if ((++polls & 255u) != 0) {
          __nanosleep(20);                      // leave the issue slots to the softmax warps
        } else {
          const uint64_t now = globaltimer_ns();
          if (polls == 256) t_last = now;       // first idle check of this stretch
          else if (now - t_last > kWaitNs || *fail) {
            flag_status(a.status, SPEC_DEV_TIMEOUT);
            *fail = 1;
            break;
          }
        }
      }
    }
    // nothing may be in flight when TMEM is freed
    if (lane == 0) {
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;                 // 0..7
    const int quad = warp & 3;               // TMEM lanes 32*quad .. (fixed by the warp id)
    const int half = sw >> 2;                // columns [half*NH, half*NH + NH)
    const int c0 = half * NH;
    const int t = quad * 32 + lane;          // key of the block / O lane
    const uint32_t tq_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const int bar_id = 1 + half;
    float* red_h = red + half * (2 * 128);
    // P tile address of (row c0 + r, key t): a per-thread base plus the
    // 128-byte swizzle term (chunk ^ (row & 7)) << 4, where row & 7 = r & 7
    // because c0 is a multiple of 8
    const uint32_t chs = (uint32_t)((t & 63) >> 3) << 4;
    const uint32_t p_off = (t >> 6) * (NP * 128) + c0 * 128 + ((t & 7) << 1);
    Walker w;
    if (count > 0) w.start(&a, start[0], start[1], start[2], start[3]);
    int g = 0;                                // global block counter
    int nslow = 0;                            // slow-path rounds (double-buffered reductions)
    // the item whose output still waits in TMEM to be read out
    bool pend = false;
    int pend_item = 0, pend_g = 0, pend_rb = 0, pend_npos = 0;
    long pend_slot = 0;
    auto read_out = [&]() {
      // o of item pend_item: all its P . V done (the last one committed on
      // pv_done of block pend_g - 1)
      const int gl = pend_g - 1;
      fwait(&pv_done[gl & 1], (gl >> 1) & 1, a.status, fail);
      tc_fence_after();
      const uint32_t ob = (uint32_t)((pend_item & 1) * (C::kOTiles * NP));
      const bool out_ok = !*fail && (c0 >> a.lgG) < pend_npos;
      // eight columns at a time (few registers: this runs inside the block loop)
#pragma unroll 1
      for (int tt = 0; tt < C::kOTiles; ++tt) {
        const int d0 = o_dim0<KVEQ>(tt, quad);
        if (d0 < 0 || !out_ok) continue;
#pragma unroll 1
        for (int cc = 0; cc < NH; cc += 8) {
          uint32_t r8[8];
          tmem_ld8_nowait(tq_lane + ob + tt * NP + c0 + cc, r8);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = c0 + cc + e;
            if ((c >> a.lgG) >= pend_npos) continue;
            const int prow = (c & (a.G - 1)) * a.q + pend_rb * a.PB + (c >> a.lgG);
            __stcg(a.part_o + (pend_slot + prow) * kDim + d0 + lane, __uint_as_float(r8[e]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[pend_item & 1]);
      pend = false;
    };
    for (int i = 0; i < count; ++i, w.next()) {
      // rows of this half: column c = i_pos * G + gh holds query position
      // i_pos of the row block (position L + qpos_off + rb*PB + i_pos), or
      // nothing past the sequence's q positions
      const int npos = min(a.PB, a.q - w.rb * a.PB);            // positions in this row block
      const int pos0 = w.L + a.qpos_off + w.rb * a.PB;
      auto row_pos = [&](int r) -> int {                         // -1: padding column
        const int ip = (c0 + r) >> a.lgG;
        return ip < npos ? pos0 + ip : -1;
      };
      // a half whose columns are all padding only keeps the barriers going
      const bool active = row_pos(0) >= 0;
      const int pmin = pos0, pmax = pos0 + npos - 1;
      const uint32_t t_ob = (uint32_t)((i & 1) * (C::kOTiles * NP));   // this item's output buffer
      // page ids of the item's blocks -> validity bits in shared memory (one
      // load per page, before the first block; two buffers by item parity, so
      // that the next item's writes never meet this item's reads)
      int* pvalid = pvalid_all + (i & 1) * kMaxItemPages;
      {
        const int np_item = 2 * w.nb;
        const int st_ = sw * 32 + lane;
        if (st_ < np_item) {
          const int pg = 2 * w.blk0 + st_;
          int ok = 0;
          if (pg < a.max_pages) {
            const int id = bt_all[(long)w.b * a.max_pages + pg];
            ok = id >= 0 && id < a.num_pages;
          }
          pvalid[st_] = ok;
        }
        named_bar(3, kSoftWarps * 32);
      }
      // running state per row: the reference maximum (log2 domain; kNoKey
      // until the row has seen a key, so that 2^(s - m) of a masked score is
      // exactly 0 and every visible score moves it) and the row sum
      float mref[NH], lt[NH];
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        mref[r] = kNoKey;
        lt[r] = 0.f;
      }
      for (int j = 0; j < w.nb; ++j, ++g) {
        const int s = g & 1;
        const int kb = (w.blk0 + j) * kBlk;
        const bool pv0 = pvalid[2 * j] != 0, pv1 = pvalid[2 * j + 1] != 0;
        const bool interior = kb >= w.lo && kb + kBlk - 1 <= w.hi && pv0 && pv1 &&
                              kb + kBlk - 1 <= pmin && (a.window == 0 || kb > pmax - a.window);
        const int key = kb + t;
        const bool in_range = key >= w.lo && key <= w.hi && ((t < kPg) ? pv0 : pv1);
        fwait(&s_full[s], (g >> 1) & 1, a.status, fail);
        tc_fence_after();
        float sc[NH];
        bool need = false;
        if (active) {
          uint32_t r8[NH / 8][8];
#pragma unroll
          for (int c = 0; c < NH / 8; ++c) tmem_ld8_nowait(tq_lane + C::kColS + s * NP + c0 + 8 * c, r8[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < NH / 8; ++c)
#pragma unroll
            for (int e = 0; e < 8; ++e) sc[8 * c + e] = __fmul_rn(__uint_as_float(r8[c][e]), a.scale_log2);
          if (!interior) {
#pragma unroll
            for (int r = 0; r < NH; ++r) {
              const int p = row_pos(r);
              const bool vis = in_range && key <= p && (a.window == 0 || key > p - a.window);
              if (!vis) sc[r] = -INFINITY;
            }
          }
#pragma unroll
          for (int r = 0; r < NH; ++r) need |= sc[r] > __fadd_rn(mref[r], kLazy);
        }
        // ---- the reference maxima move only when some row needs it
        if (bar_red_or(bar_id, 128, need)) {
          float* rb_ = red_h + (nslow & 1) * 128;
          ++nslow;
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = e < NH ? sc[e] : -INFINITY;
          const float mx = transpose_reduce32<true>(v, lane);
          rb_[quad * 32 + lane] = mx;
          named_bar(bar_id, 128);
          float alpha[NH];
          bool moved = false;
#pragma unroll
          for (int r = 0; r < NH; ++r) {
            const float bm = fmaxf(fmaxf(rb_[r], rb_[32 + r]), fmaxf(rb_[64 + r], rb_[96 + r]));
            alpha[r] = 1.f;
            if (bm > __fadd_rn(mref[r], kLazy)) {
              alpha[r] = ex2_approx(__fsub_rn(mref[r], bm));   // 0 while the row had no key
              mref[r] = bm;
              lt[r] = __fmul_rn(lt[r], alpha[r]);
              moved = true;
            }
          }
          if (moved && j > 0) {
            // rescale this half's columns of the running output (all P . V of
            // the earlier blocks must have completed)
            fwait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, a.status, fail);
            tc_fence_after();
#pragma unroll
            for (int tt = 0; tt < C::kOTiles; ++tt) {
#pragma unroll
              for (int c = 0; c < NH; c += 8) {
                uint32_t r8[8];
                tmem_ld8_nowait(tq_lane + t_ob + tt * NP + c0 + c, r8);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  r8[e] = __float_as_uint(__fmul_rn(__uint_as_float(r8[e]), alpha[c + e]));
                tmem_st8(tq_lane + t_ob + tt * NP + c0 + c, r8);
              }
            }
            tmem_st_wait();
          }
        }
        // the P buffer of this block was last read by P . V of block g - kPBufs
        if (g >= C::kPBufs)
          fwait(&pv_done[(g - C::kPBufs) & 1], ((g - C::kPBufs) >> 1) & 1, a.status, fail);
        if (active) {
          // ---- probabilities: unrounded into the row sums, bf16 into P
          // (2^-inf = 0: masked keys and rows without a key so far give 0)
          uint8_t* pp = pbuf + (g % C::kPBufs) * C::kPBytes + p_off;
#pragma unroll
          for (int r = 0; r < NH; ++r) {
            const float p = ex2_approx(__fsub_rn(sc[r], mref[r]));
            lt[r] = __fadd_rn(lt[r], p);
            *reinterpret_cast<uint16_t*>(pp + r * 128 + (chs ^ ((uint32_t)(r & 7) << 4))) = f32_to_bf16(p);
          }
        }
        // ---- value rows of keys no row of the item may use: zero them
        if (!interior && !in_range && half == 0) {
          if (KVEQ) {
            uint8_t* base = stage + s * C::kStage;
#pragma unroll
            for (int at = 0; at < 5; ++at)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(base + at * kAtom + t * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          } else if ((g == 0 || fwait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, a.status, fail)) &&
                     fwait(v_full, g & 1, a.status, fail)) {
            // the single value buffer takes block g's values only after P . V
            // of block g - 1; from then on its current phase is block g's
#pragma unroll
            for (int at = 0; at < 4; ++at)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(vbuf + at * kAtom + t * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g & 1]);
        // the previous item's output, one block after its last P . V
        if (pend) read_out();
      }

      // ---- the item's (m, l) now (log2 domain); its o, unnormalised, after
      //      the next item's first block
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = e < NH ? lt[e] : 0.f;
      const float lq = transpose_reduce32<false>(v, lane);
      float* rl = red_h + (nslow & 1) * 128;
      ++nslow;
      rl[quad * 32 + lane] = lq;
      named_bar(bar_id, 128);
      const long slot = ((long)(w.b * a.Hkv + w.kvh) * a.n_splits_grid + w.sidx) * a.rows;
      if (quad == 0 && lane < NH && !*fail && active) {
        const int c = c0 + lane;
        const int ip = w.rb * a.PB + (c >> a.lgG);
        if ((c >> a.lgG) < npos && ip < a.q) {
          float mv = kNoKey;
#pragma unroll
          for (int r = 0; r < NH; ++r)
            if (r == lane) mv = mref[r];
          const float l = __fadd_rn(__fadd_rn(rl[lane], rl[32 + lane]), __fadd_rn(rl[64 + lane], rl[96 + lane]));
          const int prow = (c & (a.G - 1)) * a.q + ip;
          __stcg(reinterpret_cast<float2*>(a.part_ml + (slot + prow) * 2), make_float2(mv, l));
        }
      }
      pend = true;
      pend_item = i;
      pend_g = g;
      pend_rb = w.rb;
      pend_npos = npos;
      pend_slot = slot;
    }
    if (pend) read_out();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

int g_num_sms = 0;

template <bool KVEQ, int NP>
cudaError_t launch_fa(int grid, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                      const FaArgs& a, cudaStream_t st) {
  using C = FaCfg<KVEQ, NP>;
  auto kern = attn_fa_kernel<KVEQ, NP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(grid), dim3(kFaThreads), C::kSmem, st, tk, tv, tq, a);
}

// Rows per CTA tile: the KV head's G*q rows rounded up to 16 when they fit
// (64 on key-equals-value layers, 32 with separate values, whose larger
// stages leave less shared memory), else row blocks of whole query positions.
int fa_np(const AttnGeom& g, int G) {
  const int cap = g.kv_equal ? 64 : 32;
  const int rows = G * g.q;
  if (rows <= cap) return (rows + 15) / 16 * 16;
  return cap;
}

}  // namespace

// Which layers take the tensor-memory attention: head_dim 256 with 64-token
// pages, no sliding window, and at least SPECVERIFY_TC_ATTN_MIN_G query heads
// per KV head (default 4).  The choice depends on the model only, never on k
// or the batch, so a row is computed by the same kernel whatever k is.  With
// G = 2 (8 to 10 rows per KV head at the benchmark's k) the mma.sync kernel's
// lighter per-block work is faster (batch 64 global layer 475-500 vs about
// 800 us, batch 1 layers 11 / 18 vs 15 / 27 us); from G = 4 on the tensor
// cores win (batch 8, G = 8: 143 vs 255 us).  Sliding-window layers stay on
// the mma.sync kernel: a window of about a thousand keys leaves one or two
// 128-key blocks per split, too little work to cover this kernel's set-up
// (one sequence, 2 KV heads, G = 4, 9 query positions, window 1024: 15-16 vs
// 11-12 us); SPECVERIFY_TC_ATTN_LOCAL=1 admits them.  SPECVERIFY_NO_TC_ATTN=1
// or SPECVERIFY_NO_TC=1 turns the path off.
bool attn_tc_supported(const AttnGeom& g) {
  static const bool local_ok = [] {
    const char* v = getenv("SPECVERIFY_TC_ATTN_LOCAL");
    return v != nullptr && v[0] == '1';
  }();
  static const int min_g = [] {
    const char* v = getenv("SPECVERIFY_NO_TC_ATTN");
    const char* off = getenv("SPECVERIFY_NO_TC");
    if ((v && v[0] == '1') || (off && off[0] == '1')) return 1 << 30;
    const char* m = getenv("SPECVERIFY_TC_ATTN_MIN_G");
    const int r = m ? atoi(m) : 4;
    return r < 1 ? 1 : r;
  }();
  const int G = g.n_q_heads / g.n_kv_heads;
  return G >= min_g && (g.window == 0 || local_ok) && g.head_dim == kDim && g.page_size == kPg && (!g.kv_equal || g.sb_width == 64) &&
         G <= 16 && 16 % G == 0 && g.split_tokens % kPg == 0 &&
         g.split_tokens / kPg + 2 <= kMaxItemPages;
}

cudaError_t launch_attn_tc(const AttnGeom& g, const CUtensorMap& tk, const CUtensorMap& tv,
                           const uint16_t* qrot, const int32_t* block_table, const int32_t* seq_lens,
                           float* part_o, float* part_ml, unsigned* status, float scale_log2,
                           cudaStream_t st) {
  if (!attn_tc_supported(g)) return cudaErrorInvalidValue;
  const int G = g.n_q_heads / g.n_kv_heads;
  const int np = fa_np(g, G);
  FaArgs a{};
  a.B = g.B;
  a.q = g.q;
  a.Hq = g.n_q_heads;
  a.Hkv = g.n_kv_heads;
  a.G = G;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.window = g.window;
  a.split = g.split_tokens;
  a.n_splits_grid = g.n_splits_grid;
  a.rows = g.rows;
  a.qpos_off = g.qpos_off;
  a.kend_off = g.kend_off;
  a.PB = np / G;
  a.lgG = __builtin_ctz((unsigned)G);
  a.RB = (g.q + a.PB - 1) / a.PB;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.status = status;
  a.scale_log2 = scale_log2;
  // queries: [B*q positions][Hq heads][D], box {64 dims, G heads, PB positions}
  CUtensorMap tq;
  if (!make_tmap_bf16_3d(&tq, qrot, kDim, g.n_q_heads, (uint64_t)g.B * g.q, kDim,
                         (uint64_t)g.n_q_heads * kDim, 64, G, a.PB))
    return cudaErrorInvalidValue;
  if (g_num_sms == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      return cudaErrorInvalidValue;
    g_num_sms = n;
  }
  const long items = (long)g.B * g.n_kv_heads * a.RB * g.n_splits_grid;   // upper bound
  const int grid = (int)std::max(1L, std::min<long>(items, g_num_sms));
  if (!g.kv_equal) {
    switch (np) {
      case 16: return launch_fa<false, 16>(grid, tk, tv, tq, a, st);
      case 32: return launch_fa<false, 32>(grid, tk, tv, tq, a, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (np) {
    case 16: return launch_fa<true, 16>(grid, tk, tv, tq, a, st);
    case 32: return launch_fa<true, 32>(grid, tk, tv, tq, a, st);
    case 48: return launch_fa<true, 48>(grid, tk, tv, tq, a, st);
    case 64: return launch_fa<true, 64>(grid, tk, tv, tq, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sv

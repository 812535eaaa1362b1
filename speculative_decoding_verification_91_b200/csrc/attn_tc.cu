// Split-KV verify attention on the 5th-generation tensor cores (sm_100a),
// head_dim 256, persistent.
//
// Work item = (sequence b, KV head, row block, absolute split of split_tokens
// keys).  Items are ordered (b, kv head, row block, split) and every CTA (one
// per SM) takes a contiguous range of them, so consecutive items mostly share
// their queries; its producer streams their keys without a break between
// items.  Keys are visited one 64-token page at a time, so that several pages
// are in flight per SM (a page is held from its copy until P . V of it has
// completed).  10 warps:
//   warp 0    TMA producer.  A page arrives as four 64 x 64 swizzled key atoms
//             plus, on key-equals-value layers, the side-band atom (pre-RoPE
//             rotated dims; 40 KB, four stages), or plus four value atoms on
//             separate-K/V layers (64 KB, three stages).  Queries come by a 3D
//             TMA box {64 dims, G heads, PB positions} straight from the
//             rotated-query buffer, once per (b, kv head, row block).
//   warp 1    allocates TMEM and issues the MMAs (one thread):
//               S^T[64 keys][NP rows]  = K . Q^T          (M = 64, A = K)
//               O^T[dims][NP rows]    += V^T . P^T        (M = 128, A = V^T,
//                                                          MN-major)
//             accumulators in TMEM (lane = key or value dim, column = query
//             row).  Scores run up to kSBufs pages ahead of the softmax; the
//             output has two buffers, so P . V of an item's first page does
//             not wait for the previous item's output to be read out.
//   warps 2-9 softmax: in the M = 64 score layout key 16q + l of the page sits
//             on TMEM lane 32q + l, so lanes 0-15 of the warp of lane
//             quadrant q own one key each; the warps of one half of the
//             columns (query rows) form a group of 128 threads.  Per page:
//             the scores of the thread's key for its NP/2 rows; p = 2^(s - m)
//             against a per-row reference maximum m that moves only when a
//             page maximum exceeds it by more than 2^8 (one OR-vote per page
//             decides; the exact page maxima are reduced only then, and the
//             running output is rescaled in TMEM only for rows that moved);
//             p is written once as bf16 for P . V and summed unrounded into
//             per-thread row sums, reduced over the keys at the end of the
//             item, when (m, l) go out.  The output o of an item is read out
//             of TMEM one page later, after the next item's first page, when
//             its last P . V has long completed.  Partials go out in the
//             layout the split combine reads.
//
// Value rows of keys outside the item's range (or on pages that were not
// loaded) are zeroed in shared memory before P . V, so stale or poisoned
// slots never reach it.  A row's reference maximum, its probabilities and the
// reduction trees depend only on its own scores and absolute key positions,
// so a row's partial does not depend on k, the batch, its row slot or the
// CTA that computed it.  Every wait is bounded; after a timeout the CTA stops
// issuing work, drains what it issued, writes nothing and frees its TMEM.
#include <math.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sv {

namespace {

constexpr int kPg = 64;                      // tokens per page = keys per block
constexpr int kDim = 256;                    // head_dim of this kernel
constexpr uint32_t kAtom = kPg * 128;        // 64 keys x 64 dims of bf16: 8 KB
constexpr int kSoftWarps = 8;
constexpr int kFaThreads = (2 + kSoftWarps) * 32;
constexpr uint32_t kSmemMax = 227u * 1024u;
constexpr uint32_t kTailBytes = 4096;
// p <= 2^kLazy: a row's reference maximum moves only when a page maximum
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

// Instruction descriptor, kind::f16 with M = 64: D fp32, A and B bf16, both
// K-major, N = n.
__device__ __forceinline__ uint32_t idesc_bf16_m64(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);
}

template <bool KVEQ, int NP>
struct FaCfg {
  static constexpr int kStages = KVEQ ? 4 : 3;
  static constexpr uint32_t kStage = (KVEQ ? 5u : 8u) * kAtom;   // keys + side-band, or keys + values
  static constexpr uint32_t kQBytes = 4u * NP * 128u;
  static constexpr uint32_t kPBytes = NP * 128u;                 // [NP rows][64 keys]
  static constexpr uint32_t bytes(int pb, int qb) {
    return 1024u + kStages * kStage + pb * kPBytes + qb * kQBytes + kTailBytes;
  }
  static constexpr int kPBufs = bytes(4, 1) <= kSmemMax ? 4 : bytes(3, 1) <= kSmemMax ? 3 : 2;
  static constexpr int kQBufs = bytes(kPBufs, 2) <= kSmemMax ? 2 : 1;
  static constexpr uint32_t kOffP = kStages * kStage;
  static constexpr uint32_t kOffQ = kOffP + kPBufs * kPBytes;
  static constexpr uint32_t kOffTail = kOffQ + kQBufs * kQBytes;
  static constexpr uint32_t kSmem = 1024 + kOffTail + kTailBytes;
  static constexpr int kOTiles = KVEQ ? 3 : 2;
  static constexpr int kOBufs = 2;
  static constexpr uint32_t kColS = kOBufs * kOTiles * NP;        // score buffers after the outputs
  static constexpr int kSBufs = (512 - (int)kColS) / NP >= 4 ? 4 : (512 - (int)kColS) / NP;
  static constexpr uint32_t kCols = kColS + kSBufs * NP;
  static constexpr uint32_t kTmemCols =
      kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
  static_assert(NP % 16 == 0 && NP >= 16 && NP <= 64, "rows per block");
  static_assert(kSBufs >= 2 && kCols <= 512, "tensor memory");
  static_assert(bytes(2, 1) <= kSmemMax && kSmem <= kSmemMax, "shared memory");
  // the side-band MMA pairs each side-band atom with the next 8 KB of shared
  // memory (lanes never read); for the last stage that is what follows it
  static_assert(!KVEQ || kOffTail + kTailBytes >= kStages * kStage + kAtom, "side-band pairing");
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
  int b, kvh, rb, sidx, ns, L, lo, hi, pg0, np;
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
    pg0 = lo / kPg;
    np = hi / kPg - pg0 + 1;
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

// v[0..15] per lane in, lane l out: the max (or sum) over the 16 lanes of
// l's half-warp of column l & 15.  Pairing by lane bit 3, 2, 1, 0 for every
// column, so every column gets the same reduction tree.
template <bool MAX>
__device__ __forceinline__ float transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int off = 8 >> r;
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
  constexpr int NS = C::kStages;
  constexpr int NPB = C::kPBufs;
  constexpr int NSB = C::kSBufs;
  constexpr int NOB = C::kOBufs;
  constexpr int NH = NP / 2;                 // columns (query rows) per softmax half
  constexpr int NQ = NH / 2;                 // columns per thread (a half-warp's share)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage = smem;                     // [NS][key atoms + side-band or value atoms]
  uint8_t* pbuf = smem + C::kOffP;           // [NPB][P]
  uint8_t* qbuf = smem + C::kOffQ;           // [kQBufs][Q]
  uint8_t* tail = smem + C::kOffTail;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(tail);    // [NS]
  uint64_t* k_empty = k_full + NS;                          // [NS]
  uint64_t* q_full = k_empty + NS;                          // [2]
  uint64_t* q_empty = q_full + 2;                           // [2]
  uint64_t* s_full = q_empty + 2;                           // [NSB]
  uint64_t* p_full = s_full + NSB;                          // [NPB]
  uint64_t* pv_done = p_full + NPB;                         // [NPB]
  uint64_t* o_free = pv_done + NPB;                         // [NOB]
  uint64_t* mma_done = o_free + NOB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* fail = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* start = reinterpret_cast<int*>(tmem_slot + 4);      // b, kvh, rb, sidx, count
  float* red = reinterpret_cast<float*>(tail + 512);       // [2 halves][2 bufs][4 quads][32]
  int* pvalid_all = reinterpret_cast<int*>(red + 512);      // [2][kMaxItemPages] page validity of an item
  static_assert(512 + 512 * 4 + 2 * kMaxItemPages * 4 <= (int)kTailBytes, "tail layout");
  static_assert((2 * NS + 4 + NSB + 2 * NPB + NOB + 1) * 8 + 32 <= 512, "barriers");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < NSB; ++i) mbar_init(&s_full[i], 1);
    for (int i = 0; i < NPB; ++i) {
      mbar_init(&p_full[i], kSoftWarps);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < NOB; ++i) mbar_init(&o_free[i], kSoftWarps);
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
      int gk = 0, nq = 0;
      auto load_page = [&](const Walker& it, int j) -> bool {
        const int s = gk % NS;
        if (gk >= NS && !fwait(&k_empty[s], ((gk / NS) - 1) & 1, a.status, fail)) return false;
        uint8_t* dst = stage + s * C::kStage;
        const int pg = it.pg0 + j;
        int id = bt_all[(long)it.b * a.max_pages + pg];
        if (id < 0 || id >= a.num_pages) {
          flag_status(a.status, SPEC_DEV_BAD_PAGE);
          id = -1;
        }
        mbar_arrive_expect_tx(&k_full[s], id >= 0 ? C::kStage : 0u);
        if (id >= 0) {
          const int y = (id * a.Hkv + it.kvh) * kPg;
#pragma unroll
          for (int at = 0; at < 4; ++at) tma_load_2d(dst + at * kAtom, &tk, &k_full[s], at * 64, y, pol);
          if (KVEQ) {
            tma_load_2d(dst + 4 * kAtom, &tv, &k_full[s], 0, y, pol);
          } else {
#pragma unroll
            for (int at = 0; at < 4; ++at)
              tma_load_2d(dst + (4 + at) * kAtom, &tv, &k_full[s], at * 64, y, pol);
          }
        }
        ++gk;
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
      for (int i = 0; ok && i < count; ++i, w.next()) {
        if (w.new_q) ok = load_q(w);
        for (int j = 0; ok && j < w.np; ++j) ok = load_page(w, j);
      }
      // every issued copy must land before the CTA may exit
      for (int i = (gk > NS ? gk - NS : 0); i < gk; ++i) mbar_wait(&k_full[i % NS], (i / NS) & 1, a.status);
      for (int i = (nq > C::kQBufs ? nq - C::kQBufs : 0); i < nq; ++i)
        mbar_wait(&q_full[i % C::kQBufs], (i / C::kQBufs) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0 && count > 0) {
      const uint32_t id_qk = idesc_bf16_m64(NP);
      const uint32_t id_pv = idesc_bf16(NP, true);
      // The scores of page g (QK) and the product P . V of an earlier page are
      // independent: each is issued as soon as its inputs are ready (polled
      // with the non-blocking test, so that waiting for one never delays the
      // other).
      //   QK(g):  keys of g landed; score buffer g % NSB read by the softmax
      //           (P . V of page g - NSB issued); new queries landed at a
      //           query-group start.
      //   PV(g):  P(g) written; at an item's first page, the output buffer
      //           of two items back read out.
      Walker ws, wp;
      ws.start(&a, start[0], start[1], start[2], start[3]);
      wp = ws;
      int is = 0, js = 0, ip = 0, jp = 0;   // QK / PV positions: item, page in item
      int nqk = 0, npv = 0, nq_used = -1;
      uint64_t t_last = globaltimer_ns();
      uint32_t polls = 0;
      while (ip < count) {
        bool progressed = false;
        // P . V first: it frees a stage for the next copy
        if (npv < nqk) {
          bool ready = mbar_test_wait(&p_full[npv % NPB], (npv / NPB) & 1);
          if (jp == 0 && ip >= NOB) ready = ready && mbar_test_wait(&o_free[ip % NOB], ((ip / NOB) - 1) & 1);
          if (ready) {
            tc_fence_after();
            const uint32_t v_addr = smem_u32(stage + (npv % NS) * C::kStage) + (KVEQ ? 0u : 4u * kAtom);
            const uint32_t p_addr = smem_u32(pbuf + (npv % NPB) * C::kPBytes);
            const uint32_t t_o = tmem + (ip % NOB) * (C::kOTiles * NP);
#pragma unroll
            for (int t = 0; t < C::kOTiles; ++t) {
              // [atom 2t ; atom 2t+1] (the side-band tile pairs its atom with the
              // next 8 KB of shared memory, whose lanes are never read)
              const uint32_t a0 = v_addr + 2 * t * kAtom;
#pragma unroll
              for (int kk = 0; kk < kPg / 16; ++kk) {    // K = 16 keys per MMA
                const uint64_t ad = sw128_desc_mn(a0 + kk * 2048, kAtom);
                umma_bf16(t_o + t * NP, ad, sw128_desc(p_addr + kk * 32), id_pv, (jp > 0 || kk > 0) ? 1u : 0u);
              }
            }
            umma_commit(&pv_done[npv % NPB]);
            umma_commit(&k_empty[npv % NS]);
            ++npv;
            if (++jp >= wp.np) {
              jp = 0;
              ++ip;
              if (ip < count) wp.next();
            }
            progressed = true;
          }
        }
        if (is < count && nqk - npv < NSB) {
          const bool newq = js == 0 && ws.new_q;
          const int qb = (nq_used + 1) % C::kQBufs;
          bool ready = !newq || mbar_test_wait(&q_full[qb], ((nq_used + 1) / C::kQBufs) & 1);
          ready = ready && mbar_test_wait(&k_full[nqk % NS], (nqk / NS) & 1);
          if (ready) {
            if (newq) ++nq_used;
            tc_fence_after();
            const uint32_t k_addr = smem_u32(stage + (nqk % NS) * C::kStage);
            const uint32_t q_addr = smem_u32(qbuf + (nq_used % C::kQBufs) * C::kQBytes);
            const uint32_t t_s = tmem + C::kColS + (nqk % NSB) * NP;
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk)   // K = 16 dims per MMA
              umma_bf16(t_s, sw128_desc(k_addr + (kk >> 2) * kAtom + (kk & 3) * 32),
                        sw128_desc(q_addr + (kk >> 2) * (NP * 128) + (kk & 3) * 32), id_qk, kk > 0);
            umma_commit(&s_full[nqk % NSB]);
            // last page of the last item of this query group: release the queries
            bool last_of_group = false;
            if (js + 1 >= ws.np) {
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
            if (++js >= ws.np) {
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
    const int hs = lane >> 4;                // column group of this half-warp
    const int t = quad * 16 + (lane & 15);   // key of the page
    // The M = 64 scores of key t sit on TMEM lane 32*quad + (t & 15); a
    // split-half load gives both half-warps those 16 lanes, each its own
    // columns: half-warp hs owns columns c0 + 8i + 4hs + e (i < NH/8, e < 4),
    // listed as j = 4i + e < NQ.
    const uint32_t tq_lane = tmem + ((uint32_t)(quad * 32) << 16);
    const int bar_id = 1 + half;
    float* red_h = red + half * (2 * 128);
    auto colj = [&](int j) -> int { return 8 * (j >> 2) + 4 * hs + (j & 3); };   // column in the half
    // P tile address of (row c0 + colj(j), key t): a per-thread base plus the
    // 128-byte swizzle term (chunk ^ (row & 7)) << 4, where row & 7 = 4hs + e
    // because c0 is a multiple of 8
    const uint32_t chs = (uint32_t)(t >> 3) << 4;
    const uint32_t p_off = c0 * 128 + ((t & 7) << 1);
    Walker w;
    if (count > 0) w.start(&a, start[0], start[1], start[2], start[3]);
    int g = 0;                                // global page counter
    int nslow = 0;                            // slow-path rounds (double-buffered reductions)
    // the item whose output still waits in TMEM to be read out
    bool pend = false;
    int pend_item = 0, pend_g = 0, pend_rb = 0, pend_npos = 0;
    long pend_slot = 0;
    auto read_out = [&]() {
      // o of item pend_item: all its P . V done (the last one committed on
      // pv_done of page pend_g - 1)
      const int gl = pend_g - 1;
      fwait(&pv_done[gl % NPB], (gl / NPB) & 1, a.status, fail);
      tc_fence_after();
      const uint32_t ob = (uint32_t)((pend_item % NOB) * (C::kOTiles * NP));
      const bool out_ok = !*fail && (c0 >> a.lgG) < pend_npos;
      // eight columns at a time (few registers: this runs inside the page loop)
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
      if (lane == 0) mbar_arrive(&o_free[pend_item % NOB]);
      pend = false;
    };
    for (int i = 0; i < count; ++i, w.next()) {
      // rows of this half: column c = i_pos * G + gh holds query position
      // i_pos of the row block (position L + qpos_off + rb*PB + i_pos), or
      // nothing past the sequence's q positions
      const int npos = min(a.PB, a.q - w.rb * a.PB);            // positions in this row block
      const int pos0 = w.L + a.qpos_off + w.rb * a.PB;
      auto row_pos = [&](int r) -> int {                         // r: column in the half; -1: padding
        const int ip = (c0 + r) >> a.lgG;
        return ip < npos ? pos0 + ip : -1;
      };
      // a half whose columns are all padding only keeps the barriers going
      const bool active = row_pos(0) >= 0;
      const int pmin = pos0, pmax = pos0 + npos - 1;
      const uint32_t t_ob = (uint32_t)((i % NOB) * (C::kOTiles * NP));
      // page ids of the item -> validity bits in shared memory (one load per
      // page, before the first page; two buffers by item parity, so that the
      // next item's writes never meet this item's reads)
      int* pvalid = pvalid_all + (i & 1) * kMaxItemPages;
      {
        const int st_ = sw * 32 + lane;
        if (st_ < w.np) {
          const int id = bt_all[(long)w.b * a.max_pages + w.pg0 + st_];
          pvalid[st_] = id >= 0 && id < a.num_pages;
        }
        named_bar(3, kSoftWarps * 32);
      }
      // running state per row: the reference maximum (log2 domain; kNoKey
      // until the row has seen a key, so that 2^(s - m) of a masked score is
      // exactly 0 and every visible score moves it), kept for every column of
      // the half (the output rescale needs all of them), and the row sum over
      // this thread's key, for its own NQ columns
      // (mq: mref of the thread's own columns; every array index below is a
      // compile-time constant, the half-warp picks by predicate)
      float mref[NH], mq[NQ], lt[NQ];
#pragma unroll
      for (int r = 0; r < NH; ++r) mref[r] = kNoKey;
#pragma unroll
      for (int j = 0; j < NQ; ++j) {
        mq[j] = kNoKey;
        lt[j] = 0.f;
      }
      for (int jp = 0; jp < w.np; ++jp, ++g) {
        const int kb = (w.pg0 + jp) * kPg;
        const bool pv = pvalid[jp] != 0;
        const bool interior = kb >= w.lo && kb + kPg - 1 <= w.hi && pv && kb + kPg - 1 <= pmin &&
                              (a.window == 0 || kb > pmax - a.window);
        const int key = kb + t;
        const bool in_range = pv && key >= w.lo && key <= w.hi;
        fwait(&s_full[g % NSB], (g / NSB) & 1, a.status, fail);
        tc_fence_after();
        float sc[NQ];
        bool need = false;
        if (active) {
          uint32_t r4[NH / 8][4];
#pragma unroll
          for (int c = 0; c < NH / 8; ++c)
            tmem_ld16x2_4_nowait(tq_lane + C::kColS + (g % NSB) * NP + c0 + 8 * c, r4[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < NH / 8; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[4 * c + e] = __fmul_rn(__uint_as_float(r4[c][e]), a.scale_log2);
          if (!interior) {
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
              const int p = row_pos(colj(j));
              const bool vis = in_range && key <= p && (a.window == 0 || key > p - a.window);
              if (!vis) sc[j] = -INFINITY;
            }
          }
#pragma unroll
          for (int j = 0; j < NQ; ++j) need |= sc[j] > __fadd_rn(mq[j], kLazy);
        }
        // ---- the reference maxima move only when some row needs it
        if (bar_red_or(bar_id, 128, need)) {
          float* rb_ = red_h + (nslow & 1) * 128;
          ++nslow;
          float v[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = e < NQ ? sc[e] : -INFINITY;
          const float mx = transpose_reduce16<true>(v, lane);
          rb_[quad * 32 + lane] = mx;     // column j = lane & 15 of half-warp hs
          named_bar(bar_id, 128);
          float alpha[NH];
          bool moved = false;
#pragma unroll
          for (int r = 0; r < NH; ++r) {
            const int ix = ((r >> 2) & 1) * 16 + 4 * (r >> 3) + (r & 3);   // (hs, j) of column r
            const float bm = fmaxf(fmaxf(rb_[ix], rb_[32 + ix]), fmaxf(rb_[64 + ix], rb_[96 + ix]));
            alpha[r] = 1.f;
            if (bm > __fadd_rn(mref[r], kLazy)) {
              alpha[r] = ex2_approx(__fsub_rn(mref[r], bm));   // 0 while the row had no key
              mref[r] = bm;
              moved = true;
            }
          }
#pragma unroll
          for (int j = 0; j < NQ; ++j) {
            const int lo_ = 8 * (j >> 2) + (j & 3);
            mq[j] = hs ? mref[lo_ + 4] : mref[lo_];
            lt[j] = __fmul_rn(lt[j], hs ? alpha[lo_ + 4] : alpha[lo_]);
          }
          if (moved && jp > 0) {
            // rescale this half's columns of the running output (all P . V of
            // the item's earlier pages must have completed)
            fwait(&pv_done[(g - 1) % NPB], ((g - 1) / NPB) & 1, a.status, fail);
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
        // the P buffer of this page was last read by P . V of page g - NPB
        if (g >= NPB) fwait(&pv_done[g % NPB], ((g / NPB) - 1) & 1, a.status, fail);
        if (active) {
          // ---- probabilities: unrounded into the row sums, bf16 into P
          // (2^-inf = 0: masked keys and rows without a key so far give 0)
          uint8_t* pp = pbuf + (g % NPB) * C::kPBytes + p_off;
#pragma unroll
          for (int j = 0; j < NQ; ++j) {
            const int r = colj(j);
            const float p = ex2_approx(__fsub_rn(sc[j], mq[j]));
            lt[j] = __fadd_rn(lt[j], p);
            *reinterpret_cast<uint16_t*>(pp + r * 128 + (chs ^ ((uint32_t)(4 * hs + (j & 3)) << 4))) =
                f32_to_bf16(p);
          }
        }
        // ---- value rows of keys no row of the item may use: zero them
        if (!interior && !in_range && half == 0) {
          uint8_t* base = stage + (g % NS) * C::kStage + (KVEQ ? 0u : 4u * kAtom);
          constexpr int kVAtoms = KVEQ ? 5 : 4;
          for (int at = hs; at < kVAtoms; at += 2)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(base + at * kAtom + t * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g % NPB]);
        // the previous item's output, one page after its last P . V
        if (pend) read_out();
      }

      // ---- the item's (m, l) now; its o after the next item's first page
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = e < NQ ? lt[e] : 0.f;
      const float lq = transpose_reduce16<false>(v, lane);
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
          const int ix = ((lane >> 2) & 1) * 16 + 4 * (lane >> 3) + (lane & 3);
          const float l = __fadd_rn(__fadd_rn(rl[ix], rl[32 + ix]), __fadd_rn(rl[64 + ix], rl[96 + ix]));
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
// pages, and at least SPECVERIFY_TC_ATTN_MIN_G query heads per KV head
// (default 4).  The choice depends on the model only, never on k or the
// batch, so a row is computed by the same kernel whatever k is.  With G = 2
// (8 to 10 rows per KV head at the benchmark's k) the mma.sync kernel's lighter
// per-block work is faster (batch 64 global layer 479 vs 660 us, batch 1
// sliding-window layer 12 vs 19 us); from G = 4 on the tensor cores win
// (batch 8, G = 8: 168 vs 255 us).  Sliding-window layers stay on the mma.sync
// kernel: a window of about a thousand keys leaves one or two 128-key blocks
// per split, too little work to cover this kernel's set-up (one sequence,
// 2 KV heads, G = 4, 9 query positions, window 1024: 16-21 vs 12 us);
// SPECVERIFY_TC_ATTN_LOCAL=1 admits them.  SPECVERIFY_NO_TC_ATTN=1 or
// SPECVERIFY_NO_TC=1 turns the path off.
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

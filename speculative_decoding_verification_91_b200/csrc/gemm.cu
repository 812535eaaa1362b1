// Streaming skinny GEMM for the verify step: Y = X . W^T where X holds the
// few verify rows (M = B*(k+1), tens of rows) and W is a large bf16 weight
// matrix read once from HBM.  Used for the QKV projection, the output
// projection (+ residual) and the LM head with a fused argmax (and, when all
// rows fit one M-block, the acceptance of every sequence).
//
// Design (sm_100a):
//   * one producer warp issues TMA tile loads (W box 128 rows x 64 k, X box
//     (8*NT) rows x 64 k, both 128-byte swizzled) into a ring of stages
//     guarded by mbarriers; W uses an evict-first L2 policy (read once), X
//     evict-last (re-read by every CTA).  W does not depend on earlier
//     kernels, so the first ring of W tiles is requested before the
//     programmatic-launch wait and overlaps the previous kernel's tail;
//   * four consumer warps each own 32 W rows of the 128-row tile and all
//     M-block rows: swap-AB mma.sync m16n8k16 (W rows are the MMA's M side,
//     the verify rows its N side), fp32 accumulators in registers;
//   * split-K over a fixed number of K chunks per CTA (a function of N and K
//     only, never of M, so a row's sum order does not depend on the batch);
//     partial sums are added in split order by the last CTA to finish a tile
//     (atomic ticket, no spin waits);
//   * argmax epilogue: per-tile (max, index) per row, ties to the lowest
//     index, reduced across tiles by the last CTA; logits never reach HBM.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace sv {

namespace {

constexpr int kTileN = 128;
constexpr int kTileK = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMBlock = 64;

template <int NT>
struct Cfg {
  static constexpr int kStages = NT <= 2 ? 6 : 5;
  static constexpr int kWBytes = kTileN * 128;
  static constexpr int kXBytes = NT * 8 * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kRedBytes = 2 * kConsumerWarps * NT * 8 * 4;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 2 * kStages * 8 + kRedBytes + 64;
};

struct Args {
  int M, N, K, kchunks, splits, n_tiles;
  float* out;
  float* partial;
  float* arg_val;
  int* arg_idx;
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

// QKV projection epilogue: after this CTA published its split partial, the
// last CTA to finish a head (all splits of its D/128 column tiles) sums the
// partials in split order, rotates each (j, j + D/2) pair of query and key
// heads at its row's position and writes queries to the workspace and keys,
// values and the key-equals-value side-band to the cache pools.
template <int MP>
__device__ __forceinline__ void rope_epilogue(const Args& a, int n_tile, int mblk, int m0, int ctid,
                                              int* flag) {
  const RopeFuse& f = a.rope;
  const int D = f.head_dim, half = D / 2, tph = D / kTileN;
  const int head = n_tile / tph, n_heads = a.N / D;
  if (ctid == 0) {
    const unsigned prev = atomicAdd(&a.tickets[mblk * n_heads + head], 1u);
    *flag = (prev == (unsigned)(a.splits * tph - 1));
  }
  named_bar(1, kConsumerWarps * 32);
  if (!*flag) return;
  __threadfence();
  const int mcount = min(MP, a.M - m0);
  const size_t split_stride = (size_t)a.n_tiles * kTileN * MP;
  const float* base = a.partial + (size_t)mblk * a.splits * a.n_tiles * kTileN * MP;
  for (int item = ctid; item < half * mcount; item += kConsumerWarps * 32) {
    const int mm = item / half, j = item % half;
    const int f0 = head * D + j, f1 = f0 + half;
    const float* p0 = base + ((size_t)(f0 / kTileN) * kTileN + f0 % kTileN) * MP + mm;
    const float* p1 = base + ((size_t)(f1 / kTileN) * kTileN + f1 % kTileN) * MP + mm;
    float x0 = 0.f, x1 = 0.f;
    int sp = 0;
    for (; sp + 4 <= a.splits; sp += 4) {
      float u[4], v[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        u[w] = __ldcg(p0 + (size_t)(sp + w) * split_stride);
        v[w] = __ldcg(p1 + (size_t)(sp + w) * split_stride);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        x0 = __fadd_rn(x0, u[w]);
        x1 = __fadd_rn(x1, v[w]);
      }
    }
    for (; sp < a.splits; ++sp) {
      x0 = __fadd_rn(x0, __ldcg(p0 + (size_t)sp * split_stride));
      x1 = __fadd_rn(x1, __ldcg(p1 + (size_t)sp * split_stride));
    }
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
  if (ctid == 0) a.tickets[mblk * n_heads + head] = 0u;
}

template <int NT, int MODE>
__global__ void __launch_bounds__(kThreads) stream_gemm_kernel(
    const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, Args a) {
  using C = Cfg<NT>;
  constexpr int MP = NT * 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  float* red_v = reinterpret_cast<float*>(empty + C::kStages);
  int* red_i = reinterpret_cast<int*>(red_v + kConsumerWarps * MP);
  int* flag = red_i + kConsumerWarps * MP;
  volatile int* fail = flag + 1;  // set by any consumer warp whose wait ran out

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, split = blockIdx.y, mblk = blockIdx.z;
  const int m0 = mblk * kMBlock;
  const int kc0 = (int)((long)split * a.kchunks / a.splits);
  const int kc1 = (int)((long)(split + 1) * a.kchunks / a.splits);
  const int nk = kc1 - kc0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *fail = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tw);
      prefetch_tmap(&tx);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int pre = min(nk, C::kStages);
      for (int it = 0; it < pre; ++it) {   // weights only: independent of earlier kernels
        mbar_arrive_expect_tx(&full[it], C::kStageBytes);
        tma_load_2d(smem + it * C::kStageBytes, &tw, &full[it], (kc0 + it) * kTileK,
                    n_tile * kTileN, pol_w);
      }
      pdl_wait();
      for (int it = 0; it < pre; ++it)
        tma_load_2d(smem + it * C::kStageBytes + C::kWBytes, &tx, &full[it], (kc0 + it) * kTileK, m0,
                    pol_x);
      int issued = pre;
      for (int it = pre; it < nk; ++it) {
        const int s = it % C::kStages;
        if (!mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1, a.status)) break;
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        const int kx = (kc0 + it) * kTileK;
        tma_load_2d(st, &tw, &full[s], kx, n_tile * kTileN, pol_w);
        tma_load_2d(st + C::kWBytes, &tx, &full[s], kx, m0, pol_x);
        issued = it + 1;
      }
      // Drain: every issued stage must have landed before the CTA may exit.
      for (int it = (issued > C::kStages ? issued - C::kStages : 0); it < issued; ++it)
        mbar_wait(&full[it % C::kStages], (it / C::kStages) & 1, a.status);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

  // On a timed-out wait a warp stops consuming but still reaches every named
  // barrier below, so the other warps never block on it; the CTA then skips
  // its outputs as a whole.
  for (int it = 0; it < nk; ++it) {
    const int s = it % C::kStages;
    if (*fail) break;
    if (!mbar_wait(&full[s], (it / C::kStages) & 1, a.status)) {
      *fail = 1;
      break;
    }
    const uint32_t wb = smem_u32(smem + s * C::kStageBytes);
    const uint32_t xb = wb + C::kWBytes;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t row = warp * 32 + mt * 16 + (lane & 15);
        ldsm_x4(wb + swz128(row, ks * 2 + (lane >> 4)), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint32_t b0, b1;
        const uint32_t row = nt * 8 + (lane & 7);
        ldsm_x2(xb + swz128(row, ks * 2 + ((lane >> 3) & 1)), b0, b1);
        mma_bf16(acc[0][nt], af[0], b0, b1);
        mma_bf16(acc[1][nt], af[1], b0, b1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  named_bar(1, kConsumerWarps * 32);
  if (*fail) return;

  const int g = lane >> 2, t = lane & 3;
  const int ctid = threadIdx.x;  // 0..127 among consumers

  if (MODE == kGemmArgmax) {
    // ---- per-tile argmax of every verify row (column of the MMA tile)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = n_tile * kTileN + warp * 32 + mt * 16 + g + h * 8;
            const float v = acc[mt][nt][h * 2 + j];
            if (n < a.N && better(v, n, bv, bi)) {
              bv = v;
              bi = n;
            }
          }
        }
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (better(ov, oi, bv, bi)) {
            bv = ov;
            bi = oi;
          }
        }
        if (g == 0) {
          const int col = nt * 8 + 2 * t + j;
          red_v[warp * MP + col] = bv;
          red_i[warp * MP + col] = bi;
        }
      }
    }
    named_bar(1, kConsumerWarps * 32);
    if (ctid < MP && m0 + ctid < a.M) {
      float bv = red_v[ctid];
      int bi = red_i[ctid];
      for (int w = 1; w < kConsumerWarps; ++w) {
        const float v = red_v[w * MP + ctid];
        const int i = red_i[w * MP + ctid];
        if (better(v, i, bv, bi)) {
          bv = v;
          bi = i;
        }
      }
      const size_t o = (size_t)n_tile * a.M + m0 + ctid;
      a.arg_val[o] = bv;
      a.arg_idx[o] = bi;
    }
    __threadfence();
    named_bar(1, kConsumerWarps * 32);
    if (ctid == 0) {
      const unsigned prev = atomicAdd(&a.tickets[mblk], 1u);
      *flag = (prev == (unsigned)(a.n_tiles - 1));
    }
    named_bar(1, kConsumerWarps * 32);
    if (!*flag) return;
    __threadfence();
    // ---- last CTA of this M-block: each warp reduces whole rows over all
    //      tiles (lanes stride the tiles), lowest index wins ties
    const int mcount = min(kMBlock, a.M - m0);
    int* ids_s = red_i;   // reused: final ids of this block's rows (mcount <= MP)
    for (int mm = warp; mm < mcount; mm += kConsumerWarps) {
      const int m = m0 + mm;
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll 8
      for (int tile = lane; tile < a.n_tiles; tile += 32) {
        const float v = __ldcg(&a.arg_val[(size_t)tile * a.M + m]);
        const int i = __ldcg(&a.arg_idx[(size_t)tile * a.M + m]);
        if (better(v, i, bv, bi)) {
          bv = v;
          bi = i;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) {
        a.ids[m] = bi;
        if (a.maxv) a.maxv[m] = bv;
        ids_s[mm] = bi;
        if (a.acc.copy_ids) a.acc.copy_ids[m] = bi;
        if (a.acc.copy_max) a.acc.copy_max[m] = bv;
      }
    }
    if (ctid == 0) a.tickets[mblk] = 0u;
    if (a.acc.B > 0) {                 // all rows are in this block (M <= 64)
      named_bar(1, kConsumerWarps * 32);
      for (int b = warp; b < a.acc.B; b += kConsumerWarps)
        accept_one(a.acc, b, ids_s + b * (a.acc.k + 1), lane);
    }
    return;
  }

  // ---- store / residual epilogues
  if (a.splits == 1 && MODE != kGemmQkvRope) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int n = n_tile * kTileN + warp * 32 + mt * 16 + g + (e >> 1) * 8;
          const int m = m0 + nt * 8 + 2 * t + (e & 1);
          if (n < a.N && m < a.M) {
            float* dst = a.out + (size_t)m * a.N + n;
            if (MODE == kGemmResidual)
              *dst = __fadd_rn(*dst, acc[mt][nt][e]);
            else
              *dst = acc[mt][nt][e];
          }
        }
    return;
  }
  // split-K: publish this split's partial tile [128][MP]
  float* mine = a.partial + (((size_t)mblk * a.splits + split) * a.n_tiles + n_tile) * kTileN * MP;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = warp * 32 + mt * 16 + g + h * 8;
        const int c = nt * 8 + 2 * t;
        __stcg(reinterpret_cast<float2*>(mine + (size_t)r * MP + c),
               make_float2(acc[mt][nt][h * 2], acc[mt][nt][h * 2 + 1]));
      }
  __threadfence();
  named_bar(1, kConsumerWarps * 32);
  if (MODE == kGemmQkvRope) {
    rope_epilogue<MP>(a, n_tile, mblk, m0, ctid, flag);
    return;
  }
  if (ctid == 0) {
    unsigned* tk = &a.tickets[mblk * a.n_tiles + n_tile];
    const unsigned prev = atomicAdd(tk, 1u);
    *flag = (prev == (unsigned)(a.splits - 1));
  }
  named_bar(1, kConsumerWarps * 32);
  if (!*flag) return;
  __threadfence();
  // last split of this tile: sum partials in split order, then the epilogue.
  // Work item = (output feature r, row mm); the split loads of an item are
  // issued together (independent) and then added in split order.
  const int mcount = min(MP, a.M - m0);
  const size_t split_stride = (size_t)a.n_tiles * kTileN * MP;
  const float* base = a.partial + ((size_t)mblk * a.splits * a.n_tiles + n_tile) * kTileN * MP;
  for (int item = ctid; item < kTileN * mcount; item += kConsumerWarps * 32) {
    const int mm = item / kTileN, r = item % kTileN;
    const int n = n_tile * kTileN + r;
    if (n >= a.N) continue;
    const float* p = base + (size_t)r * MP + mm;
    float s = 0.f;
    int sp = 0;
    for (; sp + 8 <= a.splits; sp += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(p + (size_t)(sp + u) * split_stride);
#pragma unroll
      for (int u = 0; u < 8; ++u) s = __fadd_rn(s, v[u]);
    }
    for (; sp < a.splits; ++sp) s = __fadd_rn(s, __ldcg(p + (size_t)sp * split_stride));
    float* dst = a.out + (size_t)(m0 + mm) * a.N + n;
    if (MODE == kGemmResidual)
      *dst = __fadd_rn(*dst, s);
    else
      *dst = s;
  }
  if (ctid == 0) a.tickets[mblk * a.n_tiles + n_tile] = 0u;
}

template <int NT, int MODE>
cudaError_t launch_nt(const GemmPlan& p, const CUtensorMap& tw, const CUtensorMap& tx,
                      const Args& a, cudaStream_t st) {
  auto kern = stream_gemm_kernel<NT, MODE>;
  const int smem = Cfg<NT>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(p.n_tiles, p.splits, p.mblocks), dim3(kThreads), smem, st, tw, tx, a);
}

template <int MODE>
cudaError_t launch_mode(const GemmPlan& p, const CUtensorMap& tw, const CUtensorMap& tx,
                        const Args& a, cudaStream_t st) {
  switch (p.nt) {
    case 1: return launch_nt<1, MODE>(p, tw, tx, a, st);
    case 2: return launch_nt<2, MODE>(p, tw, tx, a, st);
    case 3: return launch_nt<3, MODE>(p, tw, tx, a, st);
    case 4: return launch_nt<4, MODE>(p, tw, tx, a, st);
    case 5: return launch_nt<5, MODE>(p, tw, tx, a, st);
    case 6: return launch_nt<6, MODE>(p, tw, tx, a, st);
    case 7: return launch_nt<7, MODE>(p, tw, tx, a, st);
    case 8: return launch_nt<8, MODE>(p, tw, tx, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

GemmPlan plan_gemm(int M, int N, int K, int mode) {
  GemmPlan p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_tiles = (N + kTileN - 1) / kTileN;
  p.kchunks = (K + kTileK - 1) / kTileK;
  p.mblocks = (M + kMBlock - 1) / kMBlock;
  p.nt = (std::min(M, kMBlock) + 7) / 8;
  if (mode == kGemmArgmax) {
    p.splits = 1;
  } else {
    // about 256 CTAs per M-block, at least 4 K chunks each; depends on N, K only
    int s = (256 + p.n_tiles - 1) / p.n_tiles;
    s = std::min(s, std::max(1, p.kchunks / 4));
    p.splits = std::max(1, s);
  }
  return p;
}

size_t gemm_partial_floats(const GemmPlan& p) {
  return (size_t)p.mblocks * p.splits * p.n_tiles * kTileN * (p.nt * 8);
}
size_t gemm_argmax_entries(const GemmPlan& p) { return (size_t)p.n_tiles * p.M; }
int gemm_tickets(const GemmPlan& p) { return p.mblocks * p.n_tiles; }

cudaError_t launch_gemm(const GemmPlan& p, int mode, const void* x, const void* w,
                        const GemmBuffers& b, cudaStream_t st) {
  CUtensorMap tw, tx;
  if (!make_tmap_bf16_2d(&tw, w, p.N, p.K, kTileN, kTileK)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tx, x, p.M, p.K, p.nt * 8, kTileK, p.x_row_stride))
    return cudaErrorInvalidValue;
  Args a{};
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.kchunks = p.kchunks;
  a.splits = p.splits;
  a.n_tiles = p.n_tiles;
  a.out = b.out;
  a.partial = b.partial;
  a.arg_val = b.arg_val;
  a.arg_idx = b.arg_idx;
  a.ids = b.ids;
  a.maxv = b.maxv;
  a.tickets = b.tickets;
  a.status = b.status;
  a.acc = b.acc;
  a.rope = b.rope;
  if (mode != kGemmArgmax || p.mblocks != 1) a.acc.B = 0;
  switch (mode) {
    case kGemmStore: return launch_mode<kGemmStore>(p, tw, tx, a, st);
    case kGemmResidual: return launch_mode<kGemmResidual>(p, tw, tx, a, st);
    case kGemmArgmax: return launch_mode<kGemmArgmax>(p, tw, tx, a, st);
    case kGemmQkvRope: return launch_mode<kGemmQkvRope>(p, tw, tx, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sv

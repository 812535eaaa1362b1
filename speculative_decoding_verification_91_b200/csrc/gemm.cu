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
#include <cstdlib>

#include "common.cuh"
#include "gemm_epi.cuh"
#include "internal.h"

namespace sv {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMBlock = 64;
constexpr int kFusedTailMaxRows = kEpiMaxRows;   // up to this many rows the last CTA runs the epilogue

template <int NT>
struct Cfg {
  static constexpr int kStages = NT <= 2 ? 6 : 5;
  static constexpr int kWBytes = kTileN * 128;
  static constexpr int kXBytes = NT * 8 * 128;
  static constexpr int kStageBytes = kWBytes + kXBytes;
  static constexpr int kRedBytes = 2 * kConsumerWarps * NT * 8 * 4;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 2 * kStages * 8 + kRedBytes + 64;
};

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
      atomicMax(&a.arg_keys[m0 + ctid], pack_arg(bv, bi));
    }
    argmax_finish(a, a.n_tiles, mblk, m0, kMBlock, ctid, flag, red_i);
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
  // split-K: publish this split's partial tile (128 features x this block's rows)
  float* mine = a.partial + ((size_t)split * a.n_tiles + n_tile) * kTileN * a.ldp + m0;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = warp * 32 + mt * 16 + g + h * 8;
        const int c = nt * 8 + 2 * t;
        __stcg(reinterpret_cast<float2*>(mine + (size_t)r * a.ldp + c),
               make_float2(acc[mt][nt][h * 2], acc[mt][nt][h * 2 + 1]));
      }
  if (a.grid_reduce) return;   // splitk_reduce_kernel finishes
  __threadfence();
  named_bar(1, kConsumerWarps * 32);
  if (MODE == kGemmQkvRope) {
    rope_epilogue(a, MP, n_tile, mblk, m0, ctid, flag);
    return;
  }
  splitk_finish<MODE>(a, MP, n_tile, mblk, m0, ctid, flag);
}

// Split-K sum (in split order) + epilogue over the whole grid, one output
// per thread, 32x32 tiles transposed through shared memory so that both the
// partial reads (along rows) and the output writes (along features) coalesce.
//   store / residual: tile = 32 features x 32 rows, out[m][n] (+)= sum
//   QKV + RoPE: tile = 32 pairs (j, j + D/2) of one head x 32 rows
template <int MODE>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(Args a) {
  __shared__ float t0[32][33], t1[32][33];
  pdl_trigger();
  pdl_wait();
  const int ld = a.ldp, tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  const int m_base = blockIdx.y * 32;
  const size_t split_stride = (size_t)a.n_tiles * kTileN * ld;
  // Each thread sums four (feature or pair, row) elements; the loads of four
  // splits of all four are in flight together, then added in split order.
  if (MODE != kGemmQkvRope) {
    const int n_base = blockIdx.x * 32;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    const int m = m_base + tx;
    for (int sp0 = 0; sp0 < a.splits; sp0 += 4) {
      float v[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {                // u: feature ty + 8u of the tile
        const int n = n_base + ty + 8 * u;
        const float* p = a.partial + (size_t)n * ld + m;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          v[u][w] = (n < a.N && m < a.M && sp0 + w < a.splits) ? __ldcg(p + (size_t)(sp0 + w) * split_stride)
                                                               : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (sp0 + w < a.splits) s[u] = __fadd_rn(s[u], v[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) t0[ty + 8 * u][tx] = s[u];
    __syncthreads();
    // the residuals are read before the first store (a store may alias a
    // later load as far as the compiler knows)
    const int n = n_base + tx;
    float res[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {                  // u: row ty + 8u of the tile
      const int m = m_base + ty + 8 * u;
      res[u] = (MODE == kGemmResidual && n < a.N && m < a.M) ? a.out[(size_t)m * a.N + n] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = ty + 8 * u, m = m_base + r;
      if (n < a.N && m < a.M)
        a.out[(size_t)m * a.N + n] = (MODE == kGemmResidual) ? __fadd_rn(res[u], t0[tx][r]) : t0[tx][r];
    }
    return;
  }
  const RopeFuse& f = a.rope;
  const int D = f.head_dim, half = D / 2;
  const int pairs_per_head = half / 32;
  const int head = blockIdx.x / pairs_per_head, j0 = (blockIdx.x % pairs_per_head) * 32;
  {
    const int m = m_base + tx;
    float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sp0 = 0; sp0 < a.splits; sp0 += 2) {
      float v0[4][2], v1[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {                // u: pair ty + 8u of the tile
        const int j = j0 + ty + 8 * u;
        const float* p0 = a.partial + (size_t)(head * D + j) * ld + m;
        const float* p1 = a.partial + (size_t)(head * D + j + half) * ld + m;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const bool ok = m < a.M && sp0 + w < a.splits;
          v0[u][w] = ok ? __ldcg(p0 + (size_t)(sp0 + w) * split_stride) : 0.f;
          v1[u][w] = ok ? __ldcg(p1 + (size_t)(sp0 + w) * split_stride) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if (sp0 + w < a.splits) {
            x0[u] = __fadd_rn(x0[u], v0[u][w]);
            x1[u] = __fadd_rn(x1[u], v1[u][w]);
          }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      t0[ty + 8 * u][tx] = x0[u];
      t1[ty + 8 * u][tx] = x1[u];
    }
  }
  __syncthreads();
  // every load (table entries, lengths, pages) before the first store
  const int j = j0 + tx;
  const bool rot = j < f.n_rot && head < f.n_q_heads + f.n_kv_heads;
  const bool kv_head = head >= f.n_q_heads;
  const int kvh = head < f.n_q_heads + f.n_kv_heads ? head - f.n_q_heads
                                                    : head - f.n_q_heads - f.n_kv_heads;
  float2 cs[4];
  long long rowi[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {                    // u: row ty + 8u of the tile
    const int m = m_base + ty + 8 * u;
    cs[u] = (m < a.M && rot) ? f.rope_tab[(size_t)m * half + j] : make_float2(1.f, 0.f);
    rowi[u] = -1;
    if (m < a.M && kv_head) {
      const int b = m / f.q, i = m % f.q;
      const int pos = f.seq_lens[b] + i;
      if (pos < 0 || pos / f.page_size >= f.max_pages) {
        flag_status(a.status, SPEC_DEV_BAD_LENGTH);
      } else {
        const int page = f.block_table[(size_t)b * f.max_pages + pos / f.page_size];
        if (page < 0 || page >= f.num_pages)
          flag_status(a.status, SPEC_DEV_BAD_PAGE);
        else
          rowi[u] = ((long long)page * f.n_kv_heads + kvh) * f.page_size + pos % f.page_size;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = ty + 8 * u, m = m_base + r;
    if (m >= a.M) continue;
    const float x0 = t0[tx][r], x1 = t1[tx][r];
    float y0 = x0, y1 = x1;
    if (rot) rope_pair(x0, x1, cs[u].x, cs[u].y, y0, y1);
    if (head < f.n_q_heads) {
      uint16_t* qo = f.q_out + ((size_t)m * f.n_q_heads + head) * D;
      qo[j] = f32_to_bf16(y0);
      qo[j + half] = f32_to_bf16(y1);
      continue;
    }
    if (rowi[u] < 0) continue;
    const size_t row = (size_t)rowi[u];
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

// partial row stride of the mma.sync path (the tcgen05 path uses its padded N <= this)
static int mma_ldp(const GemmPlan& p) { return p.mblocks > 1 ? p.mblocks * kMBlock : p.nt * 8; }

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
    // about one CTA per SM per M-block, at least 4 K chunks each; depends
    // on N, K only (SPECVERIFY_SPLIT_TARGET overrides the target, for tuning)
    static const int target = [] {
      const char* v = getenv("SPECVERIFY_SPLIT_TARGET");
      const int t = v ? atoi(v) : 0;
      return t > 0 ? t : 148;   // one CTA per SM of a B200
    }();
    // One target for both GEMM paths: the K partition must not depend on M,
    // so a row's sums (and the bits of its cache entries and logits) are the
    // same whatever k is (a separate target for the many-row path was 2%
    // faster at 256 rows but broke that).
    int s = (target + p.n_tiles - 1) / p.n_tiles;
    s = std::min(s, std::max(1, p.kchunks / 4));
    p.splits = std::max(1, s);
  }
  return p;
}

// Split-K partial floats of either path: the tensor-memory kernel writes
// rows padded to 16 (tc_np), the mma.sync kernel to its M-block width.
size_t gemm_partial_floats(const GemmPlan& p) {
  const size_t ldp = tc_supported(p.M) ? std::max<size_t>(mma_ldp(p), (size_t)tc_ldp(p.M)) : mma_ldp(p);
  return (size_t)p.splits * p.n_tiles * kTileN * ldp;
}
size_t gemm_argmax_entries(const GemmPlan& p) { return (size_t)p.M; }
// Completion counters the fused last-CTA epilogue needs: one per (M-block,
// tile) when it runs (few rows, more than one K split or the RoPE
// epilogue), none when the tile is stored directly or the grid-wide reduce
// does the epilogue (more rows).
int gemm_tickets(const GemmPlan& p, int mode) {
  if (p.M > kFusedTailMaxRows) return 0;
  if (p.splits == 1 && mode != kGemmQkvRope) return 0;   // stored directly, no last-CTA tail
  return p.mblocks * p.n_tiles;
}

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
  a.arg_keys = b.arg_keys;
  a.ids = b.ids;
  a.maxv = b.maxv;
  a.tickets = b.tickets;
  a.status = b.status;
  a.acc = b.acc;
  a.rope = b.rope;
  a.ldp = mma_ldp(p);
  // more than a few rows: reduce the split partials with the whole grid
  a.grid_reduce = (mode != kGemmArgmax && p.M > kFusedTailMaxRows) ? 1 : 0;
  if (mode != kGemmArgmax || p.mblocks != 1) a.acc.B = 0;   // acceptance needs every row
  if (b.accept_fused) *b.accept_fused = a.acc.B > 0 ? 1 : 0;
  switch (mode) {
    case kGemmArgmax: return launch_mode<kGemmArgmax>(p, tw, tx, a, st);
  }
  cudaError_t e = cudaErrorInvalidValue;
  switch (mode) {
    case kGemmStore: e = launch_mode<kGemmStore>(p, tw, tx, a, st); break;
    case kGemmResidual: e = launch_mode<kGemmResidual>(p, tw, tx, a, st); break;
    case kGemmQkvRope: e = launch_mode<kGemmQkvRope>(p, tw, tx, a, st); break;
  }
  // a single K split stores / adds its tile directly (no partials to reduce)
  if (e != cudaSuccess || !a.grid_reduce || (p.splits == 1 && mode != kGemmQkvRope)) return e;
  return launch_splitk_reduce(a, mode, st);
}

cudaError_t launch_splitk_reduce(const Args& a, int mode, cudaStream_t st) {
  const int mt = (a.M + 31) / 32;
  switch (mode) {
    case kGemmStore:
      return launch_k(splitk_reduce_kernel<kGemmStore>, dim3((a.N + 31) / 32, mt), dim3(32, 8), 0, st, a);
    case kGemmResidual:
      return launch_k(splitk_reduce_kernel<kGemmResidual>, dim3((a.N + 31) / 32, mt), dim3(32, 8), 0, st,
                      a);
    case kGemmQkvRope: {
      const int D = a.rope.head_dim;
      return launch_k(splitk_reduce_kernel<kGemmQkvRope>, dim3((a.N / D) * (D / 2 / 32), mt),
                      dim3(32, 8), 0, st, a);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace sv

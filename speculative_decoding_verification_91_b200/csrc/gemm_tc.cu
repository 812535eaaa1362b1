// Streaming GEMM on the 5th-generation tensor cores (tcgen05 + TMEM) for
// verify steps with many rows (M = B*(k+1) above 32, e.g. batch 64 x 4
// rows): Y = X . W^T with W [N][K] streamed once from HBM and up to 256
// verify rows in the MMA's N dimension, so the weights are read once per
// 256 rows whatever M is (more rows: blocks of 256 on grid z).
//
// One CTA per (NW 128-row weight tiles, K split, row block); 6 warps:
//   warp 0   TMA producer: NW W boxes 128 x 64 and an X box NP x 64 (128-byte
//            swizzle) per stage into a ring (mbarrier full/empty); the first
//            ring of W tiles is requested before the programmatic-launch wait;
//   warp 1   allocates NW TMEM accumulators (128 lanes x NP fp32 columns) and
//            one elected thread issues tcgen05.mma kind::f16 (A = W tile,
//            B = X tile, both K-major SW128 shared-memory descriptors), 4 MMAs
//            of K = 16 per stage and accumulator; tcgen05.commit releases each
//            stage and, after the last, signals the accumulators;
//   warps 2-5 read the accumulators with tcgen05.ld (warp w owns TMEM lanes
//            32*(w%4)..: one weight row per thread and tile) and run the
//            epilogue: the argmax over the CTA's weight rows of every verify
//            row, or the split-K partial tile for the store / residual / RoPE
//            epilogues (NW = 1).  NW = 2 serves LM heads above 128 padded
//            rows, where the tensor cores bound the kernel: the row tile is
//            then read from L2 once per 256 weight rows.
//
// Every wait is bounded; the CTA always reaches its final barrier and frees
// its TMEM, also after a timeout.
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "gemm_epi.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace sv {

namespace {

constexpr int kTcThreads = 192;
constexpr int kTcMaxRows = 256;              // verify rows per TMEM accumulator (MMA N)
constexpr int kTcEpiWarp0 = 2;
constexpr uint32_t kABytes = kTileN * 128;   // 16 KB weight tile per stage
// LM heads with more (padded) rows than this take two weight tiles per CTA
constexpr int kPairMinRows = 128;

// barriers, TMEM slot, flags, then red_v / red_i [4][256] for the argmax
constexpr uint32_t kTailBytes = 256u + 2u * 4u * 256u * 4u;

struct TcLayout {
  int stages;
  uint32_t stage_bytes;   // kABytes + np * 128
  uint32_t smem;          // dynamic shared memory bytes
};

// nw weight tiles per CTA: 1 (two CTAs per SM when the ring fits 2 stages in
// ~110 KB), or 2 (one CTA per SM, the whole shared memory)
__host__ __device__ inline TcLayout tc_layout(int np, int nw) {
  TcLayout t{};
  t.stage_bytes = (uint32_t)nw * kABytes + (uint32_t)np * 128u;
  const uint32_t budget = nw == 1 ? 110u * 1024u : 227u * 1024u;
  int s = (int)((budget - 1024u - kTailBytes) / t.stage_bytes);
  s = s < 2 ? 2 : (s > 6 ? 6 : s);
  t.stages = s;
  t.smem = 1024u + (uint32_t)s * t.stage_bytes + kTailBytes;
  return t;
}

template <int MODE, int NW>
__global__ void __launch_bounds__(kTcThreads, NW == 1 ? 2 : 1) tc_gemm_kernel(
    const __grid_constant__ CUtensorMap tw, const __grid_constant__ CUtensorMap tx, Args a) {
  static_assert(NW == 1 || (NW == 2 && MODE == kGemmArgmax), "weight tiles per CTA");
  const int np = a.np;
  const TcLayout L = tc_layout(np, NW);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* tail = smem + L.stages * L.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + L.stages;
  uint64_t* acc_full = empty + L.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  int* flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* fail = flag + 1;
  float* red_v = reinterpret_cast<float*>(smem + L.stages * L.stage_bytes + 256);   // [4][256]
  int* red_i = reinterpret_cast<int*>(red_v + 4 * 256);                              // [4][256]

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x * NW, split = blockIdx.y, mblk = blockIdx.z;   // first weight tile
  const int m0 = mblk * kTcMaxRows;          // first verify row of this block
  const int kc0 = (int)((long)split * a.kchunks / a.splits);
  const int kc1 = (int)((long)(split + 1) * a.kchunks / a.splits);
  const int nk = kc1 - kc0;
  const uint32_t ncols = np <= 32 ? 32u : (np <= 64 ? 64u : (np <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < L.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *fail = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, ncols * NW);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tw);
      prefetch_tmap(&tx);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int pre = min(nk, L.stages);
      // (a weight tile past N reads zeros; its rows are masked in the epilogue)
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&full[it], L.stage_bytes);
#pragma unroll
        for (int w = 0; w < NW; ++w)
          tma_load_2d(smem + it * L.stage_bytes + w * kABytes, &tw, &full[it], (kc0 + it) * kTileK,
                      (n_tile + w) * kTileN, pol_w);
      }
      pdl_wait();
      for (int it = 0; it < pre; ++it)
        tma_load_2d(smem + it * L.stage_bytes + NW * kABytes, &tx, &full[it], (kc0 + it) * kTileK, m0,
                    pol_x);
      int issued = pre;
      for (int it = pre; it < nk; ++it) {
        const int s = it % L.stages;
        if (*fail || !mbar_wait(&empty[s], ((it / L.stages) - 1) & 1, a.status)) {
          *fail = 1;
          break;
        }
        uint8_t* st = smem + s * L.stage_bytes;
        mbar_arrive_expect_tx(&full[s], L.stage_bytes);
        const int kx = (kc0 + it) * kTileK;
#pragma unroll
        for (int w = 0; w < NW; ++w) tma_load_2d(st + w * kABytes, &tw, &full[s], kx, (n_tile + w) * kTileN, pol_w);
        tma_load_2d(st + NW * kABytes, &tx, &full[s], kx, m0, pol_x);
        issued = it + 1;
      }
      for (int it = (issued > L.stages ? issued - L.stages : 0); it < issued; ++it)
        mbar_wait(&full[it % L.stages], (it / L.stages) & 1, a.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(np);
      int done = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % L.stages;
        if (*fail || !mbar_wait(&full[s], (it / L.stages) & 1, a.status)) {
          *fail = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * L.stage_bytes);
        const uint32_t b_addr = a_addr + NW * kABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // K = 16 per MMA: +32 bytes inside the swizzled rows
#pragma unroll
          for (int w = 0; w < NW; ++w)   // accumulator w: weight tile n_tile + w
            umma_bf16(tmem + w * ncols, sw128_desc(a_addr + w * kABytes + kk * 32), sw128_desc(b_addr + kk * 32),
                      idesc, (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
        done = it + 1;
      }
      umma_commit(acc_full);             // fires once every MMA issued above has completed
      // the accumulator must be complete before the CTA may free its TMEM
      mbar_wait(acc_full, 0, a.status);
      (void)done;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ctid = threadIdx.x - kTcEpiWarp0 * 32;      // 0..127
    const int quad = warp & 3;                             // TMEM lanes 32*quad ..
    const int row = quad * 32 + lane;                      // weight row within the tile
    const bool ok = mbar_wait(acc_full, 0, a.status);
    tc_fence_after();
    if (!ok) *fail = 1;
    named_bar(1, kEpiThreads);
    if (!*fail) {
      const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
      if (MODE == kGemmArgmax) {
        // per verify row (column): max over this CTA's NW x 128 weight rows
        const int n = n_tile * kTileN + row;
        for (int c0 = 0; c0 < np; c0 += 32) {
          float v[32];
          int id[32];
          tmem_ld32(tq + c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            id[j] = n;
            if (n >= a.N) v[j] = -INFINITY;
          }
          if (NW == 2) {
            // the second tile's row of this thread (ids n + 128 > n: on equal
            // values the first tile's row wins, as the lower id must)
            float v2[32];
            tmem_ld32(tq + ncols + c0, v2);
            const int n2 = n + kTileN;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float x = n2 < a.N ? v2[j] : -INFINITY;
              if (better(x, n2, v[j], id[j])) {
                v[j] = x;
                id[j] = n2;
              }
            }
          }
          // transpose-reduce: after the 5 rounds lane l holds column c0 + l
#pragma unroll
          for (int r = 0; r < 5; ++r) {
            const int off = 16 >> r, half = 16 >> r;
            const bool up = (lane & off) != 0;
#pragma unroll
            for (int j = 0; j < half; ++j) {
              const float sv = up ? v[j] : v[j + half];
              const int si = up ? id[j] : id[j + half];
              const float kv = up ? v[j + half] : v[j];
              const int ki = up ? id[j + half] : id[j];
              const float ov = __shfl_xor_sync(0xffffffffu, sv, off);
              const int oi = __shfl_xor_sync(0xffffffffu, si, off);
              const bool take = better(ov, oi, kv, ki);
              v[j] = take ? ov : kv;
              id[j] = take ? oi : ki;
            }
          }
          if (c0 + lane < np) {
            red_v[quad * 256 + c0 + lane] = v[0];
            red_i[quad * 256 + c0 + lane] = id[0];
          }
        }
        named_bar(1, kEpiThreads);
        for (int c = ctid; c < np && m0 + c < a.M; c += kEpiThreads) {
          float bv = red_v[c];
          int bi = red_i[c];
          for (int q2 = 1; q2 < 4; ++q2)
            if (better(red_v[q2 * 256 + c], red_i[q2 * 256 + c], bv, bi)) {
              bv = red_v[q2 * 256 + c];
              bi = red_i[q2 * 256 + c];
            }
          atomicMax(&a.arg_keys[m0 + c], pack_arg(bv, bi));
        }
      } else {
        // split-K partial tile [128 rows][np], then the shared epilogues
        float* mine = a.partial + ((size_t)split * a.n_tiles + n_tile) * kTileN * a.ldp + m0;
        for (int c0 = 0; c0 < np; c0 += 32) {
          float v[32];
          tmem_ld32(tq + c0, v);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (c0 + j < np)   // np is a multiple of 16: a float4 is wholly inside or outside
              __stcg(reinterpret_cast<float4*>(mine + (size_t)row * a.ldp + c0 + j),
                     make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols * NW);
  if (warp < kTcEpiWarp0 || *fail) return;

  // ---- cross-CTA completion of the argmax (epilogue warps only); the other
  //      modes finish in splitk_reduce_kernel, which sums the split partials with
  //      the whole grid instead of one CTA per tile
  if (MODE == kGemmArgmax) {
    const int ctid = threadIdx.x - kTcEpiWarp0 * 32;
    argmax_finish(a, gridDim.x, mblk, m0, np, ctid, flag, red_i);
  }
}

template <int MODE, int NW>
cudaError_t launch_tc_mode(const GemmPlan& p, const CUtensorMap& tw, const CUtensorMap& tx,
                           const Args& a, cudaStream_t st) {
  auto kern = tc_gemm_kernel<MODE, NW>;
  const TcLayout L = tc_layout(a.np, NW);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.smem);
  if (e != cudaSuccess) return e;
  e = launch_k(kern, dim3((p.n_tiles + NW - 1) / NW, p.splits, tc_mblocks(p.M)), dim3(kTcThreads), L.smem,
               st, tw, tx, a);
  if (e != cudaSuccess || MODE == kGemmArgmax) return e;
  return launch_splitk_reduce(a, MODE, st);
}

}  // namespace

// Row counts for the tensor-memory GEMM: above 32 (up to there the mma.sync
// kernel streams the weights at the same HBM speed; at 40 and 64 rows it
// becomes compute-bound: LM head at d 2560, 64 rows 442 us vs 230 us here).
// Up to 256 rows sit in one TMEM accumulator (N = 256 columns); more rows run
// as blocks of 256 (grid z), each streaming the weights once -- against the
// mma.sync kernel's blocks of 64 rows, a quarter of the weight traffic.
// SPECVERIFY_TC_MIN_ROWS overrides the lower bound (>= 16),
// SPECVERIFY_NO_TC=1 turns the path off.
bool tc_supported(int M) {
  static const int min_rows = [] {
    const char* v = getenv("SPECVERIFY_NO_TC");
    if (v && v[0] == '1') return 1 << 30;
    const char* m = getenv("SPECVERIFY_TC_MIN_ROWS");
    const int r = m ? atoi(m) : 32;
    return r < 16 ? 16 : r;
  }();
  return M > min_rows && M <= kTcMaxRows * kMaxTickets;
}

int tc_np(int M) { return M <= kTcMaxRows ? (M + 15) / 16 * 16 : kTcMaxRows; }
int tc_mblocks(int M) { return (M + kTcMaxRows - 1) / kTcMaxRows; }
int tc_ldp(int M) { return M <= kTcMaxRows ? tc_np(M) : tc_mblocks(M) * kTcMaxRows; }

cudaError_t launch_gemm_tc(const GemmPlan& p, int mode, const void* x, const void* w,
                           const GemmBuffers& b, cudaStream_t st) {
  const int np = tc_np(p.M);
  if (!tc_supported(p.M)) return cudaErrorInvalidValue;
  CUtensorMap tw, tx;
  if (!make_tmap_bf16_2d(&tw, w, p.N, p.K, kTileN, kTileK)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tx, x, p.M, p.K, np, kTileK, p.x_row_stride)) return cudaErrorInvalidValue;
  Args a{};
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.kchunks = p.kchunks;
  a.splits = p.splits;
  a.n_tiles = p.n_tiles;
  a.np = np;
  a.ldp = tc_ldp(p.M);
  a.grid_reduce = 1;
  a.out = b.out;
  a.partial = b.partial;
  a.arg_keys = b.arg_keys;
  a.ids = b.ids;
  a.maxv = b.maxv;
  a.tickets = b.tickets;
  a.status = b.status;
  a.acc = b.acc;
  a.rope = b.rope;
  if (mode != kGemmArgmax || tc_mblocks(p.M) > 1) a.acc.B = 0;   // acceptance needs every row
  if (b.accept_fused) *b.accept_fused = a.acc.B > 0 ? 1 : 0;
  switch (mode) {
    case kGemmStore: return launch_tc_mode<kGemmStore, 1>(p, tw, tx, a, st);
    case kGemmResidual: return launch_tc_mode<kGemmResidual, 1>(p, tw, tx, a, st);
    case kGemmArgmax:
      // many rows: the MMAs bound the LM head, and two weight tiles per CTA
      // halve the re-reads of the row tile from L2
      return np > kPairMinRows ? launch_tc_mode<kGemmArgmax, 2>(p, tw, tx, a, st)
                               : launch_tc_mode<kGemmArgmax, 1>(p, tw, tx, a, st);
    case kGemmQkvRope: return launch_tc_mode<kGemmQkvRope, 1>(p, tw, tx, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace sv

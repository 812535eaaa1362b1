// Verify-step attention over a paged KV cache (sm_100a).
//
// rope_append_kernel  RoPE / p-RoPE of the new rows' queries and keys at their
//                     absolute positions and the cache append (keys, values,
//                     or keys + side-band on key-equals-value layers).
// attn_split_kernel   one CTA per (sequence, KV head, absolute split of
//                     `split_tokens` keys, row block): the G*(k+1) query rows
//                     of a KV head are packed into the MMA row dimension,
//                     64-token pages stream in through TMA (128-byte
//                     swizzle) into a stage ring, QK^T and PV run on
//                     mma.sync m16n8k16 (bf16 in, fp32 accumulate), the
//                     softmax is online with warp-shuffle row reductions.
//                     Writes the unnormalised partial (o, m, l).
// attn_combine_kernel merges the splits of a row in ascending split order.
//
// Split boundaries are absolute multiples of split_tokens, keys inside a
// split are visited in a fixed order and masked keys contribute exactly 0,
// so a row's result depends only on its own query and the keys it can see,
// not on k, the batch or which MMA row it occupies.
#include <math.h>

#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"

namespace sv {

namespace {

// ======================================================================
// RoPE + cache append
// ======================================================================
__device__ __forceinline__ float load_src(const void* base, long off, int is_f32) {
  return is_f32 ? static_cast<const float*>(base)[off]
                : bf16_to_f32(static_cast<const uint16_t*>(base)[off]);
}

// One thread per rotated pair (queries, keys) or value pair; grid (rows,
// sequences, chunks of 256 work items).
constexpr int kRopeThreads = 256;
__global__ void __launch_bounds__(kRopeThreads) rope_append_kernel(RopeAppend a) {
  __shared__ float cs[128], sn[128];
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x, b = blockIdx.y;
  const int D = a.head_dim, half = D / 2, n_rot = a.n_rot;
  const int pos = (a.seq_lens ? a.seq_lens[b] : a.pos0) + i;
  for (int j = threadIdx.x; j < n_rot; j += blockDim.x) {
    // angle = position * theta_j in double (theta_j from the host), reduced to
    // [-pi, pi] and rounded to binary32 after the trigonometry
    const float2 c = rope_cs(pos, a.inv_freq[j]);
    cs[j] = c.x;
    sn[j] = c.y;
  }
  __syncthreads();

  const int nq = a.src_q ? a.n_q_heads * half : 0;
  const int nk = a.n_kv_heads * half;
  const int nv = a.src_v ? a.n_kv_heads * half : 0;
  const int idx = blockIdx.z * kRopeThreads + threadIdx.x;
  if (idx >= nq + nk + nv) return;

  if (idx < nq) {  // query pair (h, j)
    const int h = idx / half, j = idx % half;
    const long base = (long)b * a.q_seq_stride + (long)i * a.q_row_stride + (long)h * D;
    const float x0 = load_src(a.src_q, base + j, a.src_is_f32);
    const float x1 = load_src(a.src_q, base + j + half, a.src_is_f32);
    float y0 = x0, y1 = x1;
    if (j < n_rot) {
      y0 = __fsub_rn(__fmul_rn(x0, cs[j]), __fmul_rn(x1, sn[j]));
      y1 = __fadd_rn(__fmul_rn(x0, sn[j]), __fmul_rn(x1, cs[j]));
    }
    uint16_t* qo = a.q_out + (((long)b * a.n_rows + i) * a.n_q_heads + h) * D;
    qo[j] = f32_to_bf16(y0);
    qo[j + half] = f32_to_bf16(y1);
    return;
  }

  // cache slot of this position
  if (pos < 0 || pos / a.page_size >= a.max_pages) {
    if (idx == nq) flag_status(a.status, SPEC_DEV_BAD_LENGTH);
    return;
  }
  const int page = a.block_table[(long)b * a.max_pages + pos / a.page_size];
  if (page < 0 || page >= a.num_pages) {
    if (idx == nq) flag_status(a.status, SPEC_DEV_BAD_PAGE);
    return;
  }
  const int slot = pos % a.page_size;
  if (idx < nq + nk) {  // key pair (h, j), plus the side-band of rotated dims
    const int h = (idx - nq) / half, j = (idx - nq) % half;
    const long base = (long)b * a.k_seq_stride + (long)i * a.k_row_stride + (long)h * D;
    const float x0 = load_src(a.src_k, base + j, a.src_is_f32);
    const float x1 = load_src(a.src_k, base + j + half, a.src_is_f32);
    float y0 = x0, y1 = x1;
    if (j < n_rot) {
      y0 = __fsub_rn(__fmul_rn(x0, cs[j]), __fmul_rn(x1, sn[j]));
      y1 = __fadd_rn(__fmul_rn(x0, sn[j]), __fmul_rn(x1, cs[j]));
    }
    const long row = ((long)page * a.n_kv_heads + h) * a.page_size + slot;
    a.k_pool[row * D + j] = f32_to_bf16(y0);
    a.k_pool[row * D + j + half] = f32_to_bf16(y1);
    if (a.ksb_pool && j < n_rot) {
      const int sbw = 2 * n_rot;
      a.ksb_pool[row * sbw + j] = f32_to_bf16(x0);
      a.ksb_pool[row * sbw + n_rot + j] = f32_to_bf16(x1);
    }
    return;
  }
  {  // value pair: elements e, e+1 of head h
    const int w = idx - nq - nk;
    const int h = w / half, e = (w % half) * 2;
    const long base = (long)b * a.v_seq_stride + (long)i * a.v_row_stride + (long)h * D + e;
    const long row = ((long)page * a.n_kv_heads + h) * a.page_size + slot;
    a.v_pool[row * D + e] = f32_to_bf16(load_src(a.src_v, base, a.src_is_f32));
    a.v_pool[row * D + e + 1] = f32_to_bf16(load_src(a.src_v, base + 1, a.src_is_f32));
  }
}

// ======================================================================
// Split-KV attention
// ======================================================================
constexpr int kPage = 64;
constexpr int kCW = 4;                  // consumer warps
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kSbw = 64;                // side-band width supported (2 * n_rot)
constexpr int kSmemBudget = 227 * 1024;

template <int D, int MT, bool KVEQ>
struct ACfg {
  static constexpr int kRowsPad = MT * 16;
  static constexpr int kKBytes = kPage * D * 2;
  static constexpr int kVBytes = KVEQ ? kPage * kSbw * 2 : kPage * D * 2;
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr int kQBytes = kRowsPad * D * 2;
  static constexpr int kPBytes = kRowsPad * 128;       // P as bf16
  static constexpr int kRedBytes = 2 * kCW * kRowsPad * 4;
  static constexpr int kFixed = 1024 + kQBytes + kPBytes + kRedBytes + 256;
  // Prefer a footprint that lets two CTAs share an SM (two pages in flight
  // per SM hide the per-page latency chain); else use the whole budget.
  static constexpr int kStagesHalf = (kSmemBudget / 2 - 1024 - kFixed) / kStageBytes;
  static constexpr int kStagesRaw =
      kStagesHalf >= 2 ? kStagesHalf : (kSmemBudget - kFixed) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 4 ? 4 : kStagesRaw;
  static constexpr int kSmem = kFixed + kStages * kStageBytes;
  static_assert(kStages >= 2, "attention tile does not fit in shared memory");
};

struct AttnArgs {
  int q, Hq, Hkv, G, max_pages, num_pages, window, split, n_splits_grid, rows, n_rot;
  int qpos_off;   // row i of a sequence sits at position L + qpos_off + i
  int kend_off;   // its last cached key is at position L + kend_off
  int row_blocks; // row blocks of a KV head (blockIdx.x = split * row_blocks + block)
  const uint16_t* qrot;
  const int32_t* block_table;
  const int32_t* seq_lens;
  float* part_o;
  float* part_ml;
  unsigned* status;
  float scale_log2;
};

// Keys any row of a sequence may see: from the first row's window start
// (global layers: 0) to the last cached key.  Verify rows: positions L..L+q-1
// after appending their own keys (qpos_off 0, kend_off q-1); drafter rows:
// position L + s over the cache [0, L) (qpos_off s, kend_off -1).
__device__ __forceinline__ void seq_key_range(int L, const AttnArgs& a, int& klo, int& khi) {
  klo = a.window > 0 ? max(0, L + a.qpos_off - a.window + 1) : 0;
  khi = L + a.kend_off;
}

template <int D, int MT, bool KVEQ>
__global__ void __launch_bounds__(kThreads) attn_split_kernel(
    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, AttnArgs a) {
  using C = ACfg<D, MT, KVEQ>;
  constexpr int RP = C::kRowsPad;
  constexpr int NSUB = D / 64;       // 128-byte column sub-tiles of a K / V / Q row
  constexpr int NTO = D / kCW / 8;   // n8 output tiles per warp in PV

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* q_s = stages + C::kStages * C::kStageBytes;
  uint8_t* p_s = q_s + C::kQBytes;
  float* red_max = reinterpret_cast<float*>(p_s + C::kPBytes);
  float* red_sum = red_max + kCW * RP;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_sum + kCW * RP);
  uint64_t* empty = full + C::kStages;
  volatile int* fail = reinterpret_cast<volatile int*>(empty + C::kStages);

  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the row blocks of one split are neighbours in the grid, so the CTAs that
  // read the same keys run together and share them through L2
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int sidx = blockIdx.x / a.row_blocks, rb = blockIdx.x % a.row_blocks;
  const int L = a.seq_lens[b];
  if (L < 0 || L + a.q > a.max_pages * kPage) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0 && rb == 0)
      flag_status(a.status, SPEC_DEV_BAD_LENGTH);
    return;
  }
  int klo, khi;
  seq_key_range(L, a, klo, khi);
  const int s_abs = klo / a.split + sidx;
  if (s_abs * a.split > khi) return;  // beyond this sequence's last split
  const int lo = max(s_abs * a.split, klo);
  const int hi = min(s_abs * a.split + a.split - 1, khi);
  const int p_first = lo / kPage, np = hi / kPage - p_first + 1;
  const int r0 = rb * RP;                                 // first query row of this block
  const int nrows = min(RP, a.rows - r0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    *fail = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const int32_t* bt = a.block_table + (long)b * a.max_pages;

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      // streamed once: evict first; shared by the split's row blocks: normal
      const uint64_t pol = a.row_blocks > 1 ? policy_evict_normal() : policy_evict_first();
      int issued = 0;
      for (int it = 0; it < np; ++it) {
        const int s = it % C::kStages;
        if (it >= C::kStages && !mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1, a.status)) break;
        const int page = bt[p_first + it];
        if (page < 0 || page >= a.num_pages) {
          flag_status(a.status, SPEC_DEV_BAD_PAGE);
          mbar_arrive(&full[s]);
        } else {
          uint8_t* st = stages + s * C::kStageBytes;
          const int y = (page * a.Hkv + kvh) * kPage;
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
#pragma unroll
          for (int j = 0; j < NSUB; ++j) tma_load_2d(st + j * kPage * 128, &tk, &full[s], j * 64, y, pol);
          if (KVEQ) {
            tma_load_2d(st + C::kKBytes, &tv, &full[s], 0, y, pol);
          } else {
#pragma unroll
            for (int j = 0; j < NSUB; ++j)
              tma_load_2d(st + C::kKBytes + j * kPage * 128, &tv, &full[s], j * 64, y, pol);
          }
        }
        issued = it + 1;
      }
      for (int it = (issued > C::kStages ? issued - C::kStages : 0); it < issued; ++it)
        mbar_wait(&full[it % C::kStages], (it / C::kStages) & 1, a.status);
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int ctid = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;

  // Q rows of this block -> swizzled shared tile (zero padding rows)
  for (int idx = ctid; idx < RP * (D / 8); idx += kCW * 32) {
    const int r = idx / (D / 8), c = idx % (D / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    const int rg = r0 + r;
    if (r < nrows) {
      const int gh = rg / a.q, i = rg % a.q;
      const int h = kvh * a.G + gh;
      v = *reinterpret_cast<const uint4*>(a.qrot + (((long)b * a.q + i) * a.Hq + h) * D + c * 8);
    }
    *reinterpret_cast<uint4*>(q_s + (c >> 3) * (RP * 128) + swz128(r, c & 7)) = v;
  }

  // positions of the rows this thread holds in MMA fragments: (mt, half)
  int rpos[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      rpos[mt][h] = (r < nrows) ? L + a.qpos_off + (r0 + r) % a.q : -1;
    }

  float m_run[MT][2], l_run[MT][2];
  float o[MT][NTO][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      m_run[mt][h] = -INFINITY;
      l_run[mt][h] = 0.f;
    }
#pragma unroll
    for (int nt = 0; nt < NTO; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
  }
  named_bar(1, kCW * 32);  // Q tile ready

  const uint32_t q_base = smem_u32(q_s);
  const uint32_t p_base = smem_u32(p_s);
  const int half = D / 2;
  const int n_rot = a.n_rot;

  for (int it = 0; it < np; ++it) {
    const int s = it % C::kStages;
    if (*fail) break;
    if (!mbar_wait(&full[s], (it / C::kStages) & 1, a.status)) *fail = 1;
    // (a warp whose wait ran out still takes every barrier of this page)
    uint8_t* st = stages + s * C::kStageBytes;
    const uint32_t k_base = smem_u32(st);
    const uint32_t v_base = k_base + C::kKBytes;
    const int key0 = (p_first + it) * kPage;
    const int page = bt[p_first + it];
    const bool valid = page >= 0 && page < a.num_pages && !*fail;

    // ---- S = Q K^T for this warp's 16 keys
    float sc[MT][2][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[mt][nt][e] = 0.f;
    if (valid) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int sub = kk >> 2, ch = (kk & 3) * 2;
        uint32_t b0, b1, b2, b3;
        const uint32_t krow = warp * 16 + ((lane >> 4) & 1) * 8 + (lane & 7);
        ldsm_x4(k_base + sub * (kPage * 128) + swz128(krow, ch + ((lane >> 3) & 1)), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          uint32_t af[4];
          ldsm_x4(q_base + sub * (RP * 128) + swz128(mt * 16 + (lane & 15), ch + (lane >> 4)),
                  af[0], af[1], af[2], af[3]);
          mma_bf16(sc[mt][0], af, b0, b1);
          mma_bf16(sc[mt][1], af, b2, b3);
        }
      }
    }
    // ---- scale (log2 domain) and mask
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = key0 + warp * 16 + nt * 8 + 2 * t + (e & 1);
          const int p = rpos[mt][e >> 1];
          const bool vis = valid && p >= 0 && j >= klo && j <= p && j <= khi &&
                           (a.window == 0 || j > p - a.window);
          sc[mt][nt][e] = vis ? __fmul_rn(sc[mt][nt][e], a.scale_log2) : -INFINITY;
        }
    // ---- row maxima over this warp's keys
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mx = fmaxf(fmaxf(sc[mt][0][2 * h], sc[mt][0][2 * h + 1]),
                         fmaxf(sc[mt][1][2 * h], sc[mt][1][2 * h + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (t == 0) red_max[warp * RP + mt * 16 + g + 8 * h] = mx;
      }
    // ---- keys no row may use (outside [klo, khi] or on a bad page): zero
    //      their value rows so that 0 * garbage cannot reach the PV product
    if (!valid || key0 < klo || key0 + kPage - 1 > khi) {
      for (int idx = ctid; idx < kPage * (C::kVBytes / kPage / 16); idx += kCW * 32) {
        const int kr = idx / (C::kVBytes / kPage / 16), c = idx % (C::kVBytes / kPage / 16);
        const int j = key0 + kr;
        if (!valid || j < klo || j > khi) {
          // V (or side-band) row kr: its chunks live in 128-byte sub-tiles
          *reinterpret_cast<uint4*>(st + C::kKBytes + (c >> 3) * (kPage * 128) + kr * 128 +
                                    (c & 7) * 16) = make_uint4(0, 0, 0, 0);
          if (KVEQ) {  // values of unrotated dims come from the key rows
#pragma unroll
            for (int j2 = 0; j2 < NSUB; ++j2)
              if (c < 8) *reinterpret_cast<uint4*>(st + j2 * (kPage * 128) + kr * 128 + c * 16) =
                             make_uint4(0, 0, 0, 0);
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar(1, kCW * 32);

    // ---- new running max, probabilities, partial row sums, P tile
    float alpha[MT][2], mnew[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = mt * 16 + g + 8 * h;
        float pm = red_max[r];
#pragma unroll
        for (int w = 1; w < kCW; ++w) pm = fmaxf(pm, red_max[w * RP + r]);
        const float mn = fmaxf(m_run[mt][h], pm);
        mnew[mt][h] = mn;
        alpha[mt][h] = (mn == -INFINITY) ? 1.f : exp2f(__fsub_rn(m_run[mt][h], mn));
      }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = sc[mt][nt][e];
          pv[e] = (x == -INFINITY) ? 0.f : exp2f(__fsub_rn(x, mnew[mt][e >> 1]));
          rs[e >> 1] = __fadd_rn(rs[e >> 1], pv[e]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // p rounded once to bf16 for P V (the row sums keep the unrounded
          // values), as in the tensor-memory kernel
          const int r = mt * 16 + g + 8 * h;
          const uint32_t addr = p_base + swz128(r, 2 * warp + nt) + 4 * t;
          const uint32_t pb = pack_bf16x2(pv[2 * h], pv[2 * h + 1]);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(pb));
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v = rs[h];
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));
        if (t == 0) red_sum[warp * RP + mt * 16 + g + 8 * h] = v;
      }
    }
    named_bar(1, kCW * 32);

    // ---- running sums, rescale, O += P V over this warp's D/4 dims
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int r = mt * 16 + g + 8 * h;
        float ps = red_sum[r];
#pragma unroll
        for (int w = 1; w < kCW; ++w) ps = __fadd_rn(ps, red_sum[w * RP + r]);
        l_run[mt][h] = __fadd_rn(__fmul_rn(l_run[mt][h], alpha[mt][h]), ps);
        m_run[mt][h] = mnew[mt][h];
      }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NTO; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][nt][e] = __fmul_rn(o[mt][nt][e], alpha[mt][e >> 1]);
    if (valid) {
#pragma unroll
      for (int kk = 0; kk < kPage / 16; ++kk) {
        uint32_t af[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const uint32_t pa = p_base + swz128(mt * 16 + (lane & 15), kk * 2 + (lane >> 4));
          ldsm_x4(pa, af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
        }
        const uint32_t vrow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int np2 = 0; np2 < NTO / 2; ++np2) {
          const int d0 = warp * (D / kCW) + np2 * 16;
          uint32_t addr;
          if (KVEQ && (d0 < n_rot || (d0 >= half && d0 < half + n_rot))) {
            const int col = d0 < half ? d0 : n_rot + d0 - half;   // side-band column
            addr = v_base + swz128(vrow, (col >> 3) + (lane >> 4));
          } else if (KVEQ) {
            addr = k_base + (d0 >> 6) * (kPage * 128) + swz128(vrow, ((d0 & 63) >> 3) + (lane >> 4));
          } else {
            addr = v_base + (d0 >> 6) * (kPage * 128) + swz128(vrow, ((d0 & 63) >> 3) + (lane >> 4));
          }
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mma_bf16(o[mt][2 * np2], af[mt], b0, b1);
            mma_bf16(o[mt][2 * np2 + 1], af[mt], b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  named_bar(1, kCW * 32);
  if (*fail) return;

  // ---- publish the partial (o unnormalised, m and l in the log2 domain)
  const long slot = ((long)(b * a.Hkv + kvh) * a.n_splits_grid + sidx) * a.rows;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = mt * 16 + g + 8 * h;
      if (r >= nrows) continue;
      float* po = a.part_o + (slot + r0 + r) * D;
#pragma unroll
      for (int nt = 0; nt < NTO; ++nt) {
        const int d = warp * (D / kCW) + nt * 8 + 2 * t;
        __stcg(reinterpret_cast<float2*>(po + d), make_float2(o[mt][nt][2 * h], o[mt][nt][2 * h + 1]));
      }
      if (warp == 0 && t == 0)
        __stcg(reinterpret_cast<float2*>(a.part_ml + (slot + r0 + r) * 2),
               make_float2(m_run[mt][h], l_run[mt][h]));
    }
}

// out[b][i][h] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// Every reduction tree here is keyed by the ABSOLUTE split index a (split a
// covers keys [a*split, a*split + split)), never by a split's position in the
// sequence's list, whose first entry depends on where the layer's window
// starts for the first query row (on sliding-window layers it moves with k):
//   - the denominator: lane a % 32 sums its splits in ascending order, then a
//     butterfly over the lanes;
//   - the numerator: four parts, part v taking the chunks of four splits
//     c = a / 4 with c % 4 == v in ascending order (lane: 8 output dims), the
//     parts added in order.
// Splits that hold none of a row's keys (m at or below the no-key reference,
// l = 0, o = 0) only add exact zeros at their fixed places, so a row's result
// is the same whichever other rows, and so whichever k, the step had.  Both
// thread mappings compute exactly this:
//   warp_per_row = 1: one warp per query row (4 rows per CTA) walks the four
//                     parts itself (few splits, many rows);
//   warp_per_row = 0: one CTA of four warps per query row, warp v sums part
//                     v (many splits, few rows).
constexpr int kCombineWarps = 4;
constexpr int kMaxCombineSplits = kMaxSplits;
__global__ void __launch_bounds__(kCombineWarps * 32) attn_combine_kernel(AttnArgs a, int D, int n_items,
                                                                          int warp_per_row,
                                                                          uint16_t* out) {
  __shared__ float msh[kCombineWarps][kMaxCombineSplits];
  __shared__ float lsh[kCombineWarps][kMaxCombineSplits];
  __shared__ float part[kCombineWarps][256];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int item = warp_per_row ? blockIdx.x * kCombineWarps + warp : blockIdx.x;
  if (item >= n_items) return;   // (warp_per_row only: whole warps leave, no CTA barrier follows)
  const int r = item % a.rows, kvh = (item / a.rows) % a.Hkv, b = item / (a.rows * a.Hkv);
  const int L = a.seq_lens[b];
  const int gh = r / a.q, i = r % a.q;
  const int h = kvh * a.G + gh;
  uint16_t* dst = out + (((long)b * a.q + i) * a.Hq + h) * D;
  if (L < 0 || L + a.q > a.max_pages * kPage) {
    if (warp_per_row || warp == 0)
      for (int e = lane; e < D; e += 32) dst[e] = 0;
    return;
  }
  int klo, khi;
  seq_key_range(L, a, klo, khi);
  const int sf = klo / a.split;   // absolute index of the sequence's first split (partial slot 0)
  const int ns = khi < klo ? 0 : min(khi / a.split - sf + 1, kMaxCombineSplits);
  const long slot0 = ((long)(b * a.Hkv + kvh) * a.n_splits_grid) * a.rows + r;
  float* m_s = msh[warp_per_row ? warp : 0];
  float* l_s = lsh[warp_per_row ? warp : 0];
  const int t0 = warp_per_row ? lane : tid, nt = warp_per_row ? 32 : kCombineWarps * 32;
  for (int s = t0; s < ns; s += nt) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml + (slot0 + (long)s * a.rows) * 2));
    m_s[s] = ml.x;
    l_s[s] = ml.y;
  }
  if (warp_per_row) __syncwarp(); else __syncthreads();
  // every warp of the row forms the same maximum and denominator
  float mloc = -INFINITY;
  for (int s = lane; s < ns; s += 32) mloc = fmaxf(mloc, m_s[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
  const float M = mloc;
  // lane (sf + s) % 32 owns split s: the first split of this lane is s0
  const int s0_lane = ((lane - sf) % 32 + 32) % 32;
  float den = 0.f;
  for (int s = s0_lane; s < ns; s += 32) {
    const float m = m_s[s];
    den = __fadd_rn(den, __fmul_rn((m == -INFINITY) ? 0.f : exp2f(__fsub_rn(m, M)), l_s[s]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den = __fadd_rn(den, __shfl_xor_sync(0xffffffffu, den, off));
  if (!(den > 0.f)) {   // the row sees no key (drafter rows past a short window): zero output
    if (warp_per_row || warp == 0)
      for (int e = lane; e < D; e += 32) dst[e] = 0;
    return;
  }

  const int per_lane = D / 32;   // 8 (D = 256) or 4 (D = 128)
  const float* po = a.part_o + slot0 * D + lane * per_lane;
  const long sstride = (long)a.rows * D;
  // part v: chunks c = a / 4 of absolute splits with c % 4 == v, ascending,
  // each chunk's (up to) four loads in flight together
  const int c_first = sf >> 2, c_last = (sf + ns - 1) >> 2;
  auto part_sum = [&](int v, float (&acc)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    constexpr int U = 4;
    for (int c = c_first + ((v - c_first) % 4 + 4) % 4; c <= c_last; c += 4) {
      float4 x[U][2];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = 4 * c + u - sf;          // position of absolute split 4c + u in the list
        const bool in = s >= 0 && s < ns;
        const float* pp = po + (long)s * sstride;
        x[u][0] = in ? __ldcg(reinterpret_cast<const float4*>(pp)) : make_float4(0, 0, 0, 0);
        x[u][1] = (in && per_lane == 8) ? __ldcg(reinterpret_cast<const float4*>(pp + 4))
                                        : make_float4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int s = 4 * c + u - sf;
        if (s < 0 || s >= ns) continue;
        const float m = m_s[s];
        const float ws = (m == -INFINITY) ? 0.f : exp2f(__fsub_rn(m, M));
        const float xs[8] = {x[u][0].x, x[u][0].y, x[u][0].z, x[u][0].w,
                             x[u][1].x, x[u][1].y, x[u][1].z, x[u][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], __fmul_rn(ws, xs[e]));
      }
    }
  };
  float num[8];
  if (warp_per_row) {
    part_sum(0, num);
#pragma unroll 1
    for (int q = 1; q < 4; ++q) {
      float acc[8];
      part_sum(q, acc);
#pragma unroll
      for (int e = 0; e < 8; ++e) num[e] = __fadd_rn(num[e], acc[e]);
    }
  } else {
    float acc[8];
    part_sum(warp, acc);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < per_lane) part[warp][lane * per_lane + e] = acc[e];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (e >= per_lane) break;
      const int d = lane * per_lane + e;
      num[e] = __fadd_rn(__fadd_rn(__fadd_rn(part[0][d], part[1][d]), part[2][d]), part[3][d]);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e)
    if (e < per_lane) dst[lane * per_lane + e] = f32_to_bf16(__fdiv_rn(num[e], den));
}

template <int D, int MT, bool KVEQ>
cudaError_t launch_split(const AttnGeom& g, const CUtensorMap& tk, const CUtensorMap& tv,
                         const AttnArgs& a, cudaStream_t st) {
  auto kern = attn_split_kernel<D, MT, KVEQ>;
  const int smem = ACfg<D, MT, KVEQ>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_k(kern, dim3(g.n_splits_grid * g.row_blocks, g.n_kv_heads, g.B), dim3(kThreads),
                  smem, st, tk, tv, a);
}

template <int D, bool KVEQ>
cudaError_t launch_mt(int mt, const AttnGeom& g, const CUtensorMap& tk, const CUtensorMap& tv,
                      const AttnArgs& a, cudaStream_t st) {
  switch (mt) {
    case 1: return launch_split<D, 1, KVEQ>(g, tk, tv, a, st);
    case 2: return launch_split<D, 2, KVEQ>(g, tk, tv, a, st);
    case 3: return launch_split<D, 3, KVEQ>(g, tk, tv, a, st);
    case 4: return launch_split<D, 4, KVEQ>(g, tk, tv, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rope_append(const RopeAppend& a, int B, cudaStream_t st) {
  if (a.n_rows <= 0 || B <= 0) return cudaSuccess;
  const int half = a.head_dim / 2;
  const int items = (a.src_q ? a.n_q_heads * half : 0) + a.n_kv_heads * half +
                    (a.src_v ? a.n_kv_heads * half : 0);
  return launch_k(rope_append_kernel, dim3(a.n_rows, B, (items + kRopeThreads - 1) / kRopeThreads),
                  dim3(kRopeThreads), 0, st, a);
}

// 16-row MMA tiles per CTA of the mma.sync kernel.  One tile (16 query rows)
// per CTA by default: the row blocks of a KV head re-read its keys, mostly
// from L2, but the lighter CTAs (fewer registers and accumulators) let
// several share an SM and hide the mma.sync latency chains.  With 40 rows per
// KV head (batch 8, 32/4 heads, k 4) the split kernel takes 264 us with one
// tile, 289 with two and 305 with three (everything in one CTA).
// SPECVERIFY_ATTN_MT_MAX (1..4) sets the cap.
int attn_mt(int rows) {
  static const int cap = [] {
    const char* v = getenv("SPECVERIFY_ATTN_MT_MAX");
    const int c = v ? atoi(v) : 1;
    return c < 1 ? 1 : (c > 4 ? 4 : c);
  }();
  return std::min(cap, (rows + 15) / 16);
}

AttnGeom plan_attn(int B, int q, int Hq, int Hkv, int D, int page, int num_pages, int max_pages,
                   int window, int kv_equal, int sb_width, int split_tokens) {
  AttnGeom g{};
  g.B = B;
  g.q = q;
  g.n_q_heads = Hq;
  g.n_kv_heads = Hkv;
  g.head_dim = D;
  g.page_size = page;
  g.num_pages = num_pages;
  g.max_pages = max_pages;
  g.window = window;
  g.kv_equal = kv_equal;
  g.sb_width = sb_width;
  g.split_tokens = split_tokens;
  g.rows = (Hq / Hkv) * q;
  g.qpos_off = 0;
  g.kend_off = q - 1;
  const int mt = attn_mt(g.rows);
  g.row_blocks = (g.rows + mt * 16 - 1) / (mt * 16);
  if (window > 0) {
    // keys of the rows span at most window + q - 1 positions: that many
    // tokens can touch this many absolute splits
    g.n_splits_grid = (window + q - 2) / split_tokens + 2;
  } else {
    g.n_splits_grid = (max_pages * page + split_tokens - 1) / split_tokens;
  }
  return g;
}

size_t attn_partial_floats(const AttnGeom& g) {
  const size_t slots = (size_t)g.B * g.n_kv_heads * g.n_splits_grid * g.rows;
  return slots * (g.head_dim + 2);
}

cudaError_t launch_attention(const AttnGeom& g, const uint16_t* qrot, const void* k_pool,
                             const void* v_pool, const void* ksb_pool, const int32_t* block_table,
                             const int32_t* seq_lens, float* part, uint16_t* out, unsigned* status,
                             cudaStream_t st, void (*mark)(cudaStream_t)) {
  const uint64_t rows = (uint64_t)g.num_pages * g.n_kv_heads * g.page_size;
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_2d(&tk, k_pool, rows, g.head_dim, 64, 64)) return cudaErrorInvalidValue;
  if (g.kv_equal) {
    if (!make_tmap_bf16_2d(&tv, ksb_pool, rows, g.sb_width, 64, 64)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_bf16_2d(&tv, v_pool, rows, g.head_dim, 64, 64)) return cudaErrorInvalidValue;
  }
  AttnArgs a{};
  a.q = g.q;
  a.Hq = g.n_q_heads;
  a.Hkv = g.n_kv_heads;
  a.G = g.n_q_heads / g.n_kv_heads;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.window = g.window;
  a.split = g.split_tokens;
  a.qpos_off = g.qpos_off;
  a.kend_off = g.kend_off;
  a.row_blocks = g.row_blocks;
  a.n_splits_grid = g.n_splits_grid;
  a.rows = g.rows;
  a.n_rot = g.sb_width / 2;
  a.qrot = qrot;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  const size_t slots = (size_t)g.B * g.n_kv_heads * g.n_splits_grid * g.rows;
  a.part_o = part;
  a.part_ml = part + slots * g.head_dim;
  a.status = status;
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)g.head_dim));
  const int mt = attn_mt(g.rows);
  cudaError_t e;
  if (attn_tc_supported(g)) {
    e = launch_attn_tc(g, tk, tv, qrot, block_table, seq_lens, a.part_o, a.part_ml, status,
                       a.scale_log2, st);
  } else if (g.head_dim == 256) {
    e = g.kv_equal ? launch_mt<256, true>(mt, g, tk, tv, a, st) : launch_mt<256, false>(mt, g, tk, tv, a, st);
  } else if (g.head_dim == 128) {
    e = g.kv_equal ? launch_mt<128, true>(mt, g, tk, tv, a, st) : launch_mt<128, false>(mt, g, tk, tv, a, st);
  } else {
    return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if (mark) mark(st);
  // few splits: a warp per row; many: four warps per row (same arithmetic)
  const int items = g.B * g.n_kv_heads * g.rows;
  const int wpr = g.n_splits_grid <= 16 ? 1 : 0;
  return launch_k(attn_combine_kernel,
                  dim3(wpr ? (items + kCombineWarps - 1) / kCombineWarps : items),
                  dim3(kCombineWarps * 32), 0, st, a, g.head_dim, items, wpr, out);
}

}  // namespace sv

// Segment-local causal attention on 5th-generation tensor cores (sm_100a), 16-bit in, fp32
// accumulate and softmax; head_dim 64 or 128.
//
// Each (layer, segment) cell attends only within its own M = seg + n_mem rows (causal,
// diagonal included); query head h reads key/value head h / (H / Hkv). No key or value
// crosses a segment: across segments the model carries state only through its
// associative memory (arXiv 2506.05229 abstract: recurrent memory transformers process
// the input segment by segment).
//
// A work item is 128 query rows of one head of one cell; key/value tiles have 128 rows. In
// the last query tile of a cell, which holds rem = M mod 128 rows, the heads of a key/value
// group share one item when they fit (their rows stacked, see attn_pack_tail): at M = 1040
// and 4 query heads per group that turns 4 items of 16 useful rows into one of 64, and the
// softmax warps whose 32 rows hold none of them skip their arithmetic. The CTAs are
// persistent (two per SM for head_dim 64) and take items round-robin, longest first, so the
// loads of an item overlap the tail of the previous one.
//   warp 0      one thread: TMA loads of Q tiles (2 stages, one per item), K and V tiles
//               (2 stages each, a ring that runs on across items);
//   warp 1      TMEM allocation; one thread issues S = Q K^T (M=128, N=128) into TMEM and
//               O += P V (M=128, N=head_dim; P read from TMEM, V read MN-major from shared
//               memory) into a second TMEM range;
//   warps 2-5   softmax, one query row per thread: read S from TMEM, scale and mask, keep
//               the running max and sum in registers, write P as 16-bit pairs into a third
//               TMEM range; at the end of an item read O, divide by the row sum and store.
// S of tile j+1 is computed while the softmax of tile j runs. The running max is only
// raised (and O rescaled in TMEM) when it grows by more than 2^8, so P stays <= 256.
// All waits are bounded; a timeout drains in-flight copies and MMAs, frees TMEM and sets
// the error word.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

template <int HD>
struct TaCfg {
  static constexpr int SUB = 128 * 64 * 2;  // one 128-row x 64-column 16-bit swizzled block
  static constexpr int NSUB = HD / 64;      // blocks per Q / K / V tile
  static constexpr int TILE = NSUB * SUB;
  static constexpr int Q_OFF = 0;                 // two stages: the next item's Q lands early
  static constexpr int K_OFF = Q_OFF + 2 * TILE;  // two stages: K_{j+1} lands while S_j and softmax j run
  static constexpr int V_OFF = K_OFF + 2 * TILE;  // two stages: V_{j+1} lands while P.V_j runs
  static constexpr int BAR_OFF = V_OFF + 2 * TILE;
  static constexpr int NBAR = 18;
  static constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8 + 16;
  static constexpr int CTAS_PER_SM = HD == 64 ? 2 : 1;
  // TMEM: S in columns 0..127, O in 128 .. 128+HD-1, P (128 x 128, 16-bit pairs) in the next 64
  static constexpr int O_COL = 128, P_COL = 128 + HD;
  static constexpr int TMEM_COLS = P_COL + 64 <= 256 ? 256 : 512;
};

enum : int { kQFull = 0, kQEmpty = 2, kKFull = 4, kKEmpty = 6, kVFull = 8, kVEmpty = 10, kSFull = 12, kSFree = 13,
             kPReady = 14, kOReady = 15, kOFree = 16, kDrain = 17 };

// max(a, b, c) in one instruction (three-input form of PTX max.f32, sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the special-function unit (relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

template <int HD, typename OpT>
__global__ void __launch_bounds__(192, TaCfg<HD>::CTAS_PER_SM)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tm_tail,
                   const AttnArgs a) {
  using C = TaCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + C::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // the stacking parameters come from the launch (kernel parameters: no registers held)
  const int nqt = (a.M + 127) / 128;
  const int rem = a.tail_rows, gq = a.group;
  const bool pack = rem > 0;
  const int per_rank = a.H * a.G;  // items per query-tile rank
  const int n_tail = a.n_tail;     // items of the last query tile
  const int nitems = n_tail + (nqt - 1) * per_rank;
  // item i: the last query tile first (longest first): one item per key/value group when its
  // heads are stacked (h = the group's first head), else one per head; then query tiles
  // nqt-2 .. 0. Within a tile the head runs fastest, so the heads of a key/value group run
  // close together, then the cell.
  auto decode = [&](int i, int& qt, int& h, int& g) {
    if (i < n_tail) {
      qt = nqt - 1;
      const int nh = pack ? a.Hkv : a.H;
      h = (i % nh) * (pack ? gq : 1);
      g = i / nh;
      return;
    }
    i -= n_tail;
    qt = nqt - 2 - i / per_rank;
    const int r = i % per_rank;
    h = r % a.H;
    g = r / a.H;
  };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      sm100::mbar_init(bar(kQFull + s), 1);
      sm100::mbar_init(bar(kQEmpty + s), 1);
      sm100::mbar_init(bar(kKFull + s), 1);
      sm100::mbar_init(bar(kKEmpty + s), 1);
      sm100::mbar_init(bar(kVFull + s), 1);
      sm100::mbar_init(bar(kVEmpty + s), 1);
    }
    sm100::mbar_init(bar(kSFull), 1);
    sm100::mbar_init(bar(kSFree), 128);
    sm100::mbar_init(bar(kPReady), 128);
    sm100::mbar_init(bar(kOReady), 1);
    sm100::mbar_init(bar(kOFree), 128);
    sm100::mbar_init(bar(kDrain), 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
    sm100::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tm);
    if (pack) sm100::tma_prefetch_desc(&tm_tail);
  }
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), C::TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();  // this CTA holds its TMEM: the next kernel may be scheduled
  pdl_wait();     // q, k, v come from the previous kernel of the stream

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      long tq = -1, tkv = -1;  // last item whose Q load, and last ring tile whose K and V loads, were issued
      long kv = 0;             // ring tiles loaded so far
      int ik = 0;              // items taken so far
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++ik) {
        int qt, h, g;
        decode(it, qt, h, g);
        const Cell c = load_cell(a.cells, g);
        const int kvh = h / (a.H / a.Hkv);
        const int slice = cell_index(a.mode, a.L, c);
        const int xq = h * HD, xk = (a.H + kvh) * HD, xv = (a.H + a.Hkv + kvh) * HD;
        const int qs = ik & 1;
        if (!sm100::mbar_wait(bar(kQEmpty + qs), ((ik >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (pack && qt == nqt - 1) {
          // the group's gq heads, rem rows each, stacked at rows hh * rem (1024-byte aligned:
          // rem is a multiple of 8 rows of 128 bytes); rows gq * rem .. 127 are not loaded
          sm100::mbar_arrive_expect_tx(bar(kQFull + qs), C::NSUB * gq * rem * 128);
          for (int hh = 0; hh < gq; ++hh)
            for (int sb = 0; sb < C::NSUB; ++sb)
              sm100::tma_load_3d(base + C::Q_OFF + qs * C::TILE + sb * C::SUB + hh * rem * 128, &tm_tail,
                                 xq + hh * HD + 64 * sb, qt * 128, slice, bar(kQFull + qs));
        } else {
          sm100::mbar_arrive_expect_tx(bar(kQFull + qs), C::TILE);
          for (int sb = 0; sb < C::NSUB; ++sb)
            sm100::tma_load_3d(base + C::Q_OFF + qs * C::TILE + sb * C::SUB, &tm, xq + 64 * sb, qt * 128, slice,
                               bar(kQFull + qs));
        }
        tq = ik;
        for (int j = 0; j <= qt; ++j, ++kv) {  // key/value tiles 0..qt hold every key the rows may see
          const int st = static_cast<int>(kv & 1);
          const uint32_t ph = static_cast<uint32_t>((kv >> 1) & 1);
          if (!sm100::mbar_wait(bar(kKEmpty + st), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          sm100::mbar_arrive_expect_tx(bar(kKFull + st), C::TILE);
          for (int sb = 0; sb < C::NSUB; ++sb)
            sm100::tma_load_3d(base + C::K_OFF + st * C::TILE + sb * C::SUB, &tm, xk + 64 * sb, j * 128, slice,
                               bar(kKFull + st));
          if (!sm100::mbar_wait(bar(kVEmpty + st), ph ^ 1u, abort_flag)) {
            ok = false;
            sm100::mbar_wait_drain(bar(kKFull + st), ph);  // this tile's K is in flight
            break;
          }
          sm100::mbar_arrive_expect_tx(bar(kVFull + st), C::TILE);
          for (int sb = 0; sb < C::NSUB; ++sb)
            sm100::tma_load_3d(base + C::V_OFF + st * C::TILE + sb * C::SUB, &tm, xv + 64 * sb, j * 128, slice,
                               bar(kVFull + st));
          tkv = kv;
        }
      }
      if (!ok) {
        if (a.err) atomicOr(a.err, kErrTimeoutProducer);
        // let the copies already in flight land before the CTA's shared memory goes away
        for (long q = tq; q >= 0 && q >= tq - 1; --q)
          sm100::mbar_wait_drain(bar(kQFull + static_cast<int>(q & 1)), static_cast<uint32_t>((q >> 1) & 1));
        for (long q = tkv; q >= 0 && q >= tkv - 1; --q) {
          sm100::mbar_wait_drain(bar(kKFull + static_cast<int>(q & 1)), static_cast<uint32_t>((q >> 1) & 1));
          sm100::mbar_wait_drain(bar(kVFull + static_cast<int>(q & 1)), static_cast<uint32_t>((q >> 1) & 1));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tS = tmem_base, tO = tmem_base + C::O_COL, tP = tmem_base + C::P_COL;
      constexpr uint32_t idS = sm100::idesc_f32acc(128, 128, OpFormat<OpT>::value);
      constexpr uint32_t idO = sm100::idesc_f32acc_bmn(128, HD, OpFormat<OpT>::value);
      bool ok = true;
      // S of ring tile t, against the Q tile in stage qs
      auto issue_s = [&](long t, int qs) -> bool {
        const int st = static_cast<int>(t & 1);
        if (!sm100::mbar_wait(bar(kKFull + st), static_cast<uint32_t>((t >> 1) & 1), abort_flag)) return false;
        sm100::tc_fence_after();
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const int sb = k >> 2, kk = k & 3;
          const uint64_t ad = sm100::smem_desc_k128(base + C::Q_OFF + qs * C::TILE + sb * C::SUB) + 2ull * kk;
          const uint64_t bd = sm100::smem_desc_k128(base + C::K_OFF + st * C::TILE + sb * C::SUB) + 2ull * kk;
          sm100::mma_bf16(tS, ad, bd, idS, k > 0);
        }
        sm100::mma_commit(bar(kSFull));
        sm100::mma_commit(bar(kKEmpty + st));
        return true;
      };
      // this CTA's tiles in sequence: its items in order, key/value tiles 0..qt of each
      long t = 0;
      int ik = 0, it = blockIdx.x, qt = 0, h, g;
      if (it < nitems) {
        decode(it, qt, h, g);
        ok = sm100::mbar_wait(bar(kQFull), 0, abort_flag) && issue_s(0, 0);
      }
      while (it < nitems && ok) {
        const int qs = ik & 1;
        for (int j = 0; j <= qt && ok; ++j, ++t) {
          const bool last = j == qt;
          if (last) sm100::mma_commit(bar(kQEmpty + qs));  // the item's last S has read its Q
          // S of the next tile: the next tile of this item, or tile 0 of the next item
          if (!last || it + static_cast<int>(gridDim.x) < nitems) {
            if (!sm100::mbar_wait(bar(kSFree), static_cast<uint32_t>(t & 1), abort_flag)) {
              ok = false;
              break;
            }
            int nqs = qs;
            if (last) {
              nqs = (ik + 1) & 1;
              if (!sm100::mbar_wait(bar(kQFull + nqs), static_cast<uint32_t>(((ik + 1) >> 1) & 1), abort_flag)) {
                ok = false;
                break;
              }
            }
            if (!issue_s(t + 1, nqs)) {
              ok = false;
              break;
            }
          }
          const int vs = static_cast<int>(t & 1);
          if (!sm100::mbar_wait(bar(kPReady), static_cast<uint32_t>(t & 1), abort_flag) ||
              !sm100::mbar_wait(bar(kVFull + vs), static_cast<uint32_t>((t >> 1) & 1), abort_flag)) {
            ok = false;
            break;
          }
          // the first P.V of an item overwrites O: the previous item's O must have been read
          if (j == 0 && ik > 0 &&
              !sm100::mbar_wait(bar(kOFree), static_cast<uint32_t>((ik - 1) & 1), abort_flag)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k) {  // P from TMEM: 16 keys per step = 8 columns of pairs
            const uint64_t bd = sm100::smem_desc_mn128(base + C::V_OFF + vs * C::TILE + k * 2048, C::SUB);
            sm100::mma_f16_tmem_a(tO, tP + 8 * k, bd, idO, (j > 0 || k > 0));
          }
          sm100::mma_commit(bar(kOReady));
          sm100::mma_commit(bar(kVEmpty + vs));
        }
        it += gridDim.x;
        ++ik;
        if (it < nitems) decode(it, qt, h, g);
      }
      if (!ok) {
        if (a.err) atomicOr(a.err, kErrTimeoutMma);
        sm100::mma_commit(bar(kDrain));
        sm100::mbar_wait_drain(bar(kDrain), 0);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row of the tile (= TMEM lane)
    const uint32_t loff = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem_base + loff, tO = tmem_base + loff + C::O_COL, tP = tmem_base + loff + C::P_COL;
    const float sl2 = rsqrtf(static_cast<float>(HD)) * 1.4426950408889634f;  // 1/sqrt(dh) * log2(e)
    bool ok = true;
    long t = 0;  // tiles processed so far (barrier phases)
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      // a stacked tail tile holds head h + r / rem at row r < gq * rem; a warp whose rows are
      // all past that (warp-uniform) keeps the barrier protocol but skips the arithmetic
      int qt, vlim, mlim;
      bool idle;
      {
        int h, g;
        decode(it, qt, h, g);
        const int kvlim = cell_rows(load_cell(a.cells, g), a.M);  // keys past the cell's tokens are masked
        const bool packed = pack && qt == nqt - 1;
        idle = packed && quarter * 32 >= gq * rem;
        vlim = min(qt * 128 + (packed ? r % rem : r), kvlim - 1);  // the last key this row sees
        mlim = min(kvlim, qt * 128 + 1);  // a key tile reaching past this needs the mask
      }
      float m_use = 0.f, l = 0.f;
      for (int j = 0; j <= qt; ++j, ++t) {
        ok = __all_sync(0xffffffffu, sm100::mbar_wait(bar(kSFull), static_cast<uint32_t>(t & 1), abort_flag));
        if (!ok) break;
        if (idle) {
          // the same waits and arrivals as the busy warps, in the same order
          sm100::mbar_arrive(bar(kSFree));
          if (j > 0) {
            ok = __all_sync(0xffffffffu,
                            sm100::mbar_wait(bar(kOReady), static_cast<uint32_t>((t - 1) & 1), abort_flag));
            if (!ok) break;
          }
          sm100::mbar_arrive(bar(kPReady));
          continue;
        }
        sm100::tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) sm100::tmem_ld32(tS + 32 * q4, s[q4]);
        sm100::tmem_wait_ld();
        sm100::tc_fence_before();
        sm100::mbar_arrive(bar(kSFree));
        const int k0 = j * 128;
        const bool need_mask = k0 + 128 > mlim;  // the diagonal tile, or keys past the cell's end
        // causal mask (and the cell's ragged end) only on the tiles that need it: key k0 + e is
        // visible iff e <= vis, so each element costs one compare with a constant and a select
        if (need_mask) {
          const int vis = vlim - k0;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * q4 + i > vis) s[q4][i] = __float_as_uint(-INFINITY);
          }
        }
        // row max over 4 independent partials (short dependency chains)
        float mxp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mxp[(i >> 1) & 3] = max3(mxp[(i >> 1) & 3], u2f(s[q4][i]), u2f(s[q4][i + 1]));
        }
        float mx = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
        mx *= sl2;  // max of the scaled scores (the scale is positive)
        float corr = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_use = mx;  // finite: key 0 is visible to every row
        } else if (mx > m_use + 8.f) {
          corr = ex2(m_use - mx);
          m_use = mx;
          rescale = true;
        }
        if (j > 0) {
          // P of tile j-1 must be consumed (and O final for it) before P and O change; for
          // j = 0 the end of the previous item already waited for its last P.V
          ok = __all_sync(0xffffffffu,
                          sm100::mbar_wait(bar(kOReady), static_cast<uint32_t>((t - 1) & 1), abort_flag));
          if (!ok) break;
          sm100::tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
            for (int oc = 0; oc < HD / 16; ++oc) {
              uint32_t o[16];
              sm100::tmem_ld16(tO + 16 * oc, o);
              sm100::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(u2f(o[i]) * corr);
              sm100::tmem_st16(tO + 16 * oc, o);
            }
          }
        }
        // P row r -> TMEM lane r: keys 2c and 2c + 1 packed into column c (even key low). Each
        // 32-key block goes out as soon as its exponentials are done, packed in place into its
        // first 16 words.
        float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p = ex2(fmaf(u2f(s[q4][i]), sl2, -m_use));
            sp[i & 3] += p;
            s[q4][i] = __float_as_uint(p);
          }
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) s[q4][c2] = pack2<OpT>(u2f(s[q4][2 * c2]), u2f(s[q4][2 * c2 + 1]));
          sm100::tmem_st16(tP + 16 * q4, s[q4]);
        }
        const float sum = (sp[0] + sp[1]) + (sp[2] + sp[3]);
        l = l * corr + sum;
        sm100::tmem_wait_st();
        sm100::tc_fence_before();
        sm100::mbar_arrive(bar(kPReady));
      }
      if (!ok) break;
      // end of the item: O after its last P.V, normalised and stored; then O is free again
      ok = __all_sync(0xffffffffu, sm100::mbar_wait(bar(kOReady), static_cast<uint32_t>((t - 1) & 1), abort_flag));
      if (!ok) break;
      sm100::tc_fence_after();
      const float inv = 1.f / l;
      // the item's row and head again, from an opaque copy of the item index: recomputing
      // them here keeps them out of the registers of the tile loop above
      int it2;
      asm volatile("mov.b32 %0, %1;" : "=r"(it2) : "r"(it));
      int qt2, h, g;
      decode(it2, qt2, h, g);
      const Cell c = load_cell(a.cells, g);
      const bool packed = pack && qt2 == nqt - 1;
      const int qrow = qt2 * 128 + (packed ? r % rem : r);
      const bool row_out = packed ? r < gq * rem : qrow < a.M;
      const int ldo = a.ldo ? a.ldo : a.H * HD;
      OpT* const dst = static_cast<OpT*>(a.out) +
                       (static_cast<size_t>(cell_index(a.mode, a.L, c)) * a.M + qrow) * ldo +
                       (packed ? h + min(r / rem, gq - 1) : h) * HD;
#pragma unroll 1
      for (int oc = 0; oc < (idle ? 0 : HD / 32); ++oc) {
        uint32_t o[32];
        sm100::tmem_ld32(tO + 32 * oc, o);
        sm100::tmem_wait_ld();
        if (row_out) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = u2f(o[i]) * inv;
          store32_16(dst + 32 * oc, v);
        }
      }
      // O read (the MMA warp reads none of the output stores: no release needed)
      sm100::tc_fence_before();
      sm100::mbar_arrive_relaxed(bar(kOFree));
    }
    if (!ok && lane == 0 && a.err) atomicOr(a.err, kErrTimeoutEpilogue);
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int HD, typename OpT>
cudaError_t launch_hd(const CUtensorMap& tm, const CUtensorMap& tm_tail, const AttnArgs& a0, cudaStream_t st) {
  AttnArgs a = a0;
  const bool pack = attn_pack_tail(a.M, a.H, a.Hkv);
  a.tail_rows = pack ? attn_tail_rows(a.M) : 0;
  a.group = a.H / a.Hkv;
  a.n_tail = (pack ? a.Hkv : a.H) * a.G;
  using C = TaCfg<HD>;
  static bool attr[64] = {false};
  static int sms[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, OpT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    attr[dev] = true;
  }
  const long items = a.n_tail + static_cast<long>((a.M + 127) / 128 - 1) * a.H * a.G;
  const long cap = static_cast<long>(sms[dev] > 0 ? sms[dev] : 148) * C::CTAS_PER_SM;
  const int grid = static_cast<int>(items < cap ? items : cap);
  const cudaError_t e = launch_pdl(attn_tc_kernel<HD, OpT>, dim3(grid), dim3(192), C::SMEM, st, tm, tm_tail, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(int dh) { return dh == 64 || dh == 128; }

cudaError_t launch_attention_tc(const CUtensorMap& tm_qkv, const CUtensorMap& tm_tail, const AttnArgs& a, bool f16,
                                cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.Hkv <= 0 || a.H % a.Hkv != 0) return cudaErrorInvalidValue;
  const CUtensorMap& tt = tm_tail;
  if (a.dh == 64)
    return f16 ? launch_hd<64, __half>(tm_qkv, tt, a, st) : launch_hd<64, __nv_bfloat16>(tm_qkv, tt, a, st);
  if (a.dh == 128)
    return f16 ? launch_hd<128, __half>(tm_qkv, tt, a, st) : launch_hd<128, __nv_bfloat16>(tm_qkv, tt, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace rmt

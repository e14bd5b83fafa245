// Grouped GEMM on CTA pairs (tcgen05.mma.cta_group::2, sm_100a), transposed orientation.
//
// "Architecture Overview" of the diagonal-batching skill page: the products of all layers on
// one diagonal run as one GroupedGEMM launch, each group (one (layer, segment) cell) with its
// own layer's weights. This kernel computes each group's Y^T = W_l . X^T: output features run
// along the MMA's M (256 per CTA pair, 128 per CTA) and the cell's tokens along N, in tiles of
// pair_token_tile(M) tokens. Two things follow from that orientation:
//   * a cell of M = 1040 rows needs no padding tile (N is any multiple of 16 up to 256);
//   * one TMEM lane holds one output feature over consecutive tokens, so each epilogue
//     instruction of a warp reads or writes 32 consecutive features of one token row.
// The pair halves the bytes each SM fetches per MMA: each CTA loads 128 weight rows and half
// of the token rows, and the MMA reads the other token half from the peer's shared memory.
//
// Roles per CTA (320 threads, one CTA per SM, persistent over pair tiles):
//   warp 0      one thread issues the TMA loads of this CTA's weight half (128 rows) and token
//               half (NT/2 rows), 128 K-columns per ring stage (two 64-column swizzle blocks);
//               both CTAs' byte counts complete on the even CTA's barrier, which the even CTA
//               arms for the pair;
//   warp 1      TMEM (512 columns: two accumulators 256 apart); in the even CTA one thread
//               issues the pair MMAs (M = 256, N = tile tokens, K = 16), 8 per stage, and
//               releases each stage to both CTAs with one commit;
//   warps 2-9   epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (32 features) over one
//               half of the tile's tokens, 16 or 32 tokens per step, with the global loads
//               a step needs issued before its TMEM wait.
// Every wait is bounded (see sm100.cuh); on a timeout the CTA records it in the error word,
// stops issuing work and meets its peer at the final cluster barrier before freeing TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

// Shared memory: [barriers 1 KB][sums of squares 8 KB][row scales 2 KB][ring], 1024-aligned.
// A ring stage holds two 64-column blocks, each this CTA's weight half (16 KB) and token half
// (NT/2 rows of 128 B, rounded to 1 KB); the ring takes as many stages as fit (3 at NT = 208).
// Fewer, wider stages beat more, narrower ones: each commit stalls the MMA pipe for a while.
// Each stage is released by one commit that arrives on the empty barriers of both CTAs.
struct PairCfg {
  static constexpr int FM = 128;               // weight rows (output features) per CTA
  static constexpr int BK = 64;                // K-columns per swizzle block
  static constexpr int W_BYTES = FM * BK * 2;  // 16 KB
  static constexpr int MAX_STAGES = 8;
  static constexpr int ACC_COLS = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int NBAR = 2 * MAX_STAGES + 2 + 2 + 2 + 1;  // ring, tfull, tempty, warpgroup sync, drain
  static constexpr int BAR_BYTES = 1024;
  static constexpr int RED_OFF = BAR_BYTES;  // [2 acc][2 wg][4 quarters][128] fp32
  static constexpr int RED_BYTES = 2 * 2 * 4 * 128 * 4;
  static constexpr int RS_OFF = RED_OFF + RED_BYTES;  // [2 acc][2 wg][128] fp32 row scales
  static constexpr int RS_BYTES = 2 * 2 * 128 * 4;
  static constexpr int RING_OFF = RS_OFF + RS_BYTES;
  static constexpr int SMEM_BYTES = 232448;  // the per-block maximum; the ring fills the rest
  static constexpr int RING_BYTES = SMEM_BYTES - 1024 - RING_OFF;
  static_assert(8 * NBAR + 16 <= BAR_BYTES, "barrier area");
  static_assert(RING_OFF % 1024 == 0, "ring alignment");
  __host__ __device__ static int x_bytes(int NT) { return ((NT / 2) * BK * 2 + 1023) / 1024 * 1024; }
  __host__ __device__ static int block_bytes(int NT) { return W_BYTES + x_bytes(NT); }
  __host__ __device__ static int stages(int NT) {
    const int s = RING_BYTES / (2 * block_bytes(NT));
    return s < MAX_STAGES ? s : MAX_STAGES;
  }
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// silu(x) = x / (1 + e^-x) with the fast exponential and division intrinsics (relative error
// of a few 1e-7; for x below about -87 the quotient is 0, the limit of silu): the epilogue
// shares issue slots with the MMA issuer, so its instruction count shows in the GEMM's time.
__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.f + __expf(-x)); }

// Per-token sums of s[0..15] over the warp's 32 lanes (15 + 1 shuffles, fixed order): token t
// ends up in lanes 2t and 2t + 1.
__device__ __forceinline__ float warp_sum16_transposed(float (&s)[16], int lane) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    const bool hi = lane & (2 * o);
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float keep = hi ? s[o + k] : s[k];
      const float give = hi ? s[k] : s[o + k];
      s[k] = keep + __shfl_xor_sync(0xffffffffu, give, 2 * o);
    }
  }
  return s[0] + __shfl_xor_sync(0xffffffffu, s[0], 1);
}

// RMSNorm row scale from one row of per-block sums of squares, with every load of the row in
// flight at once when the row is a whole number of 16-byte vectors (at most 32 blocks).
__device__ __forceinline__ float row_scale(const float* ss_row, int parts, float inv_d, float eps) {
  if ((parts & 3) == 0 && parts <= 32) {
    const float4* p = reinterpret_cast<const float4*>(ss_row);
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 4 * i < parts ? p[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = (((s + v[i].x) + v[i].y) + v[i].z) + v[i].w;
    return rsqrtf(s * inv_d + eps);
  }
  return rms_row_scale(ss_row, parts, inv_d, eps);
}

// Epilogue of one warp: its 32 features (f = this lane's output column) over tokens
// tok0 .. tok0 + cnt - 1 of the cell (cnt a multiple of 8, at most 128), accumulator columns
// from tacc. A step covers 32 columns; columns past cnt (at most 24) are read, not stored.
// SPLIT: the split-operand mode's stores (low terms, fp32 q/k/v) are compiled in; without it
// the epilogue carries no trace of them.
template <int EPI, typename OpT, bool SPLIT>
__device__ __forceinline__ void pair_epilogue(const TcGemmArgs& a, Cell c, uint32_t tacc, int tok0, int cnt, int f,
                                              int lane, const float* rs, float* red, float& amax) {
  const EpiParams& ep = a.ep;
  const int M = a.M;
  const int lim = min(cnt, M - tok0);  // valid tokens of this warp's range
  if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
    // 16 tokens per step; the next step's residual loads go out before this step's TMEM wait
    const size_t si = cell_index(ep.src_mode, a.L, c), di = cell_index(ep.dst_mode, a.L, c);
    const float* src = ep.x + (si * M + tok0) * ep.ldx + f;
    float* dst = ep.x + (di * M + tok0) * ep.ldx + f;
    OpT* xb = nullptr;
    const int ldxb = ep.ldxb ? ep.ldxb : ep.ldx;
    if constexpr (EPI == kEpiResidCast) xb = static_cast<OpT*>(ep.xb) + (di * M + tok0) * ldxb + f;
    const bool want_ss = ep.ss_out != nullptr;
    float xs[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) xs[j] = j < lim ? src[static_cast<size_t>(j) * ep.ldx] : 0.f;
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 16) {
      uint32_t r[16];
      sm100::tmem_ld16(tacc + j0, r);
      float xn[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) xn[j] = j0 + 16 + j < lim ? src[static_cast<size_t>(j0 + 16 + j) * ep.ldx] : 0.f;
      sm100::tmem_wait_ld();
      float sq[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float y = xs[j] + u2f(r[j]);
        if (j0 + j < lim) {
          dst[static_cast<size_t>(j0 + j) * ep.ldx] = y;
          if constexpr (EPI == kEpiResidCast) {
            OpT* xr = xb + static_cast<size_t>(j0 + j) * ldxb;
            *xr = from_f32<OpT>(y);
            if constexpr (SPLIT) xr[ep.lo_off] = from_f32<OpT>(lo_term<OpT>(y));
            track_amax<OpT>(amax, y);
          }
        }
        sq[j] = j0 + j < lim ? y * y : 0.f;
        xs[j] = xn[j];
      }
      if (want_ss) {
        const float s = warp_sum16_transposed(sq, lane);
        if ((lane & 1) == 0 && j0 + (lane >> 1) < cnt) red[j0 + (lane >> 1)] = s;
      }
    }
  } else if constexpr (EPI == kEpiStoreF32 || EPI == kEpiStoreAct) {
    const size_t o0 = (cell_index(ep.out_mode, a.L, c) * static_cast<size_t>(M) + tok0) * ep.ldo + f;
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      uint32_t r[32];
      sm100::tmem_ld32(tacc + j0, r);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j0 + j < lim) {
          const size_t o = o0 + static_cast<size_t>(j0 + j) * ep.ldo;
          if constexpr (EPI == kEpiStoreF32)
            static_cast<float*>(ep.out)[o] = u2f(r[j]);
          else {
            static_cast<OpT*>(ep.out)[o] = from_f32<OpT>(u2f(r[j]));
            track_amax<OpT>(amax, u2f(r[j]));
          }
        }
      }
    }
  } else if constexpr (EPI == kEpiRope) {
    // lanes 2p and 2p + 1 of a rotated head hold the pair (x_p, x_{p + dh/2}). The angle of
    // token t is t * theta_p: each step reads (cos, sin) at its first token from the table and
    // advances one token at a time by the rotation of position 1 (complex multiplication in
    // fp32; 31 steps add a few units of 1e-6 of error), so a step needs two table reads.
    const int dh = ep.head_dim, hh = dh >> 1;
    const int i = f % dh, p = i >> 1;
    const bool odd = i & 1, rot = f < ep.rope_cols;
    const size_t o0 = (static_cast<size_t>(cell_index(ep.out_mode, a.L, c)) * M + tok0) * ep.ldo + f;
    OpT* out = static_cast<OpT*>(ep.out) + o0;
    float* out32 = static_cast<float*>(ep.out) + o0;  // out_f32
    const float2 step = (rot && M > 1) ? ep.rope[hh + p] : make_float2(1.f, 0.f);
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      float2 cs = (rot && j0 < lim) ? ep.rope[static_cast<size_t>(tok0 + j0) * hh + p] : make_float2(1.f, 0.f);
      uint32_t r[32];
      sm100::tmem_ld32(tacc + j0, r);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float x = u2f(r[j]) * rs[j0 + j];
        const float other = __shfl_xor_sync(0xffffffffu, x, 1);
        const float y = odd ? fmaf(x, cs.x, other * cs.y) : fmaf(x, cs.x, -other * cs.y);
        if (j0 + j < lim) {
          if constexpr (SPLIT) {
            out32[static_cast<size_t>(j0 + j) * ep.ldo] = y;
          } else {
            out[static_cast<size_t>(j0 + j) * ep.ldo] = from_f32<OpT>(y);
            track_amax<OpT>(amax, y);
          }
        }
        cs = make_float2(fmaf(cs.x, step.x, -cs.y * step.y), fmaf(cs.y, step.x, cs.x * step.y));
      }
    }
  } else if constexpr (EPI == kEpiSwiGLU) {
    // even lanes hold gate_j, odd lanes up_j (j = f / 2); after one exchange the even lane
    // finishes tokens 0..15 of the step and the odd lane tokens 16..31
    const bool odd = lane & 1;
    OpT* out = static_cast<OpT*>(ep.out) + (static_cast<size_t>(cell_index(ep.out_mode, a.L, c)) * M + tok0) * ep.ldo +
               (f >> 1);
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      uint32_t r[32];
      sm100::tmem_ld32(tacc + j0, r);
      sm100::tmem_wait_ld();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = u2f(r[j]) * rs[j0 + j];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float got = __shfl_xor_sync(0xffffffffu, odd ? v[j] : v[16 + j], 1);
        const float g = odd ? got : v[j], u = odd ? v[16 + j] : got;
        const int t = j0 + (odd ? 16 : 0) + j;
        if (t < lim) {
          const float y = silu_fast(g) * u;
          OpT* o = out + static_cast<size_t>(t) * ep.ldo;
          *o = from_f32<OpT>(y);
          if constexpr (SPLIT) o[ep.lo_off] = from_f32<OpT>(lo_term<OpT>(y));
          track_amax<OpT>(amax, y);
        }
      }
    }
  }
}

// Chained projections. One launch runs one to three projections ("phases") of the same cells
// in order -- in the forward: the O projection, gate/up, then down. Tiles are numbered phase by
// phase (cell, feature pair, token tile within a phase) and each CTA pair takes its tiles in
// increasing order, so a pair reaches its tiles of phase p only after all of its tiles of
// phase p-1. A tile of phase p >= 1 for (cell g, token tile tt) reads what phase p-1 wrote for
// the same tokens over all of its feature pairs (residual rows and RMSNorm statistics, or the
// SwiGLU output): its loads and its epilogue wait (bounded) until a counter in global memory
// shows that every one of those tiles has been stored. Each epilogue warp adds 1 to the
// counter of (phase, g, tt) with a release once it has stored its share of a tile and made the
// stores visible to the tensor-memory-access proxy; waiters read it with acquire loads. No wait closes a cycle: a tile waits only on tiles of the previous phase, which every
// pair reaches before any of its own tiles of a later phase, and the grid never holds more
// pairs than can be resident together. The launch ends as soon as the last tile is stored, so
// the drain and refill between the projections of a diagonal disappear with their launches.
constexpr int kNoEpi = -1;  // an unused phase slot
constexpr unsigned kSignalsPerTile = 2 * PairCfg::EPI_WARPS;  // one per epilogue warp of each CTA of the pair

template <int E0, int E1, int E2, typename OpT, bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::THREADS, 1)
    tc_pair_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmX0,
                        const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX1,
                        const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmX2,
                        const PairChainArgs args) {
  using C = PairCfg;
  constexpr int NP = E1 == kNoEpi ? 1 : (E2 == kNoEpi ? 2 : 3);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bar0 = base;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::MAX_STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::MAX_STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::MAX_STAGES + 2 + a); };
  auto wg_bar = [&](int w) { return bar0 + 8u * (2 * C::MAX_STAGES + 4 + w); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::MAX_STAGES + 6);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const TcGemmArgs& a0 = args.ph[0];
  const int M = a0.M, G = a0.G;
  const int NT = a0.nt > 0 ? a0.nt : pair_token_tile(M);
  const int STAGES = C::stages(NT);
  const uint32_t BLK = static_cast<uint32_t>(C::block_bytes(NT));
  const uint32_t ring = base + C::RING_OFF;

  const uint32_t rank = sm100::cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(tfull_bar(a), 1);
      sm100::mbar_init(tempty_bar(a), 2 * C::EPI_WARPS);  // the epilogue warps of both CTAs
      sm100::mbar_init(wg_bar(a), 4);
    }
    sm100::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
    sm100::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmW0);
    sm100::tma_prefetch_desc(&tmX0);
    if (NP > 1) {
      sm100::tma_prefetch_desc(&tmW1);
      sm100::tma_prefetch_desc(&tmX1);
    }
    if (NP > 2) {
      sm100::tma_prefetch_desc(&tmW2);
      sm100::tma_prefetch_desc(&tmX2);
    }
  }
  if (warp == 1) sm100::tmem_alloc_pair(sm100::smem_u32(tmem_slot), C::TMEM_COLS);
  sm100::tc_fence_before();
  sm100::cluster_sync();  // both CTAs' barriers initialised and TMEM allocated before any remote use
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();  // this CTA holds its TMEM: the next kernel may be scheduled
  pdl_wait();     // operands and residuals come from the previous kernels of the stream
  if (NP > 1 && blockIdx.x == 0) {
    // the next chained launch uses the other parity's counters: this launch started after the
    // one that used them ended, and the next one starts after this one ends
    unsigned* next = args.ctr + static_cast<size_t>(args.parity ^ 1) * (kMaxPhases - 1) * args.ctr_len;
    for (int i = threadIdx.x; i < (kMaxPhases - 1) * args.ctr_len; i += blockDim.x) next[i] = 0u;
  }

  const int ntt = (M + NT - 1) / NT;
  // tiles of the phases: [0, t1) phase 0, [t1, t2) phase 1, [t2, tiles) phase 2
  const int np0 = a0.N / 256, np1 = NP > 1 ? args.ph[1].N / 256 : 0, np2 = NP > 2 ? args.ph[2].N / 256 : 0;
  const int t1 = G * np0 * ntt, t2 = t1 + G * np1 * ntt, tiles = t2 + G * np2 * ntt;
  auto npair_of = [&](int p) { return p == 0 ? np0 : (p == 1 ? np1 : np2); };
  auto k_of = [&](int p) { return p == 0 ? a0.K : (p == 1 ? args.ph[1].K : args.ph[2].K); };
  auto kx_lo_of = [&](int p) { return p == 0 ? a0.kx_lo : (p == 1 ? args.ph[1].kx_lo : args.ph[2].kx_lo); };
  auto decode = [&](int t, int& p, int& g, int& fp, int& tt) {
    p = (NP > 1 && t >= t1) ? ((NP > 2 && t >= t2) ? 2 : 1) : 0;
    const int r0 = t - (p == 0 ? 0 : (p == 1 ? t1 : t2)), per = npair_of(p) * ntt;
    g = r0 / per;
    const int r = r0 % per;
    fp = r / ntt;
    tt = r % ntt;
  };
  // completed CTA halves of phase p's tiles of (cell g, token tile tt)
  auto counter = [&](int p, int g, int tt) {
    return args.ctr + (static_cast<size_t>(args.parity) * (kMaxPhases - 1) + p) * args.ctr_len + g * ntt + tt;
  };
  const int cl = static_cast<int>(sm100::cluster_id_x()), ncl = static_cast<int>(sm100::cluster_count_x());
  // tokens of token tile tt (the last one rounded up to 16; rows past M read as zeros)
  auto tile_tokens = [&](int tt) {
    const int rem = M - tt * NT;
    return rem >= NT ? NT : ((rem + 15) & ~15);
  };

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t blk_tx = 2u * (C::W_BYTES + static_cast<uint32_t>(NT / 2) * C::BK * 2);  // one block, both CTAs
      int stage = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto acquire = [&]() { return sm100::mbar_wait(empty_bar(stage), ph ^ 1u, abort_flag); };
      for (int t = cl; t < tiles && ok; t += ncl) {
        int p, g, fp, tt;
        decode(t, p, g, fp, tt);
        const CUtensorMap* tw = p == 0 ? &tmW0 : (p == 1 ? &tmW1 : &tmW2);
        const CUtensorMap* tx = p == 0 ? &tmX0 : (p == 1 ? &tmX1 : &tmX2);
        const IndexMode amode = p == 0 ? a0.a_mode : (p == 1 ? args.ph[1].a_mode : args.ph[2].a_mode);
        const int kbw = k_of(p) / C::BK;            // 64-column blocks of the weight
        const int kxl = kx_lo_of(p);                 // split-operand mode: column of the low terms
        const int kblk = kxl ? 2 * kbw : kbw;        // 64-column blocks of the product
        const int kst = (kblk + 1) / 2;    // ring stages per tile (the last may hold one block)
        const Cell c = load_cell(a0.cells, g);
        const int a3 = cell_index(amode, a0.L, c);
        if (NP > 1 && p > 0) {
          // every tile of the previous phase for these tokens is stored
          if (!sm100::counter_wait(counter(p - 1, g, tt), kSignalsPerTile * static_cast<unsigned>(npair_of(p - 1)),
                                   abort_flag)) {
            ok = false;
            break;
          }
          sm100::fence_proxy_async_global();
        }
        const int wrow = fp * 256 + static_cast<int>(rank) * C::FM;
        const int xrow = tt * NT + static_cast<int>(rank) * (tile_tokens(tt) / 2);
        for (int ks = 0; ks < kst; ++ks) {
          if (!acquire()) {
            ok = false;
            break;
          }
          const int nb = (2 * ks + 1 < kblk) ? 2 : 1;
          if (rank == 0) sm100::mbar_arrive_expect_tx(full_bar(stage), static_cast<uint32_t>(nb) * blk_tx);
          const uint32_t sa = ring + static_cast<uint32_t>(stage) * 2u * BLK;
          const uint32_t fb = sm100::mapa_shared(full_bar(stage), 0);
          for (int b = 0; b < nb; ++b) {
            const int blk = 2 * ks + b, kw = (blk % kbw) * C::BK, kx = kw + (blk / kbw) * kxl;
            sm100::tma_load_3d_pair(sa + b * BLK, tw, kw, wrow, c.l, fb);
            sm100::tma_load_3d_pair(sa + b * BLK + C::W_BYTES, tx, kx, xrow, a3, fb);
          }
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      // every stage's last fill consumed: no MMA can still read this CTA's ring and no commit
      // can still arrive on it
      for (int i = 0; i < STAGES && ok; ++i) {
        ok = acquire();
        if (++stage == STAGES) {
          stage = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        if (a0.err) atomicOr(a0.err, kErrTimeoutProducer);
        // copies already issued complete on the even CTA's barriers, which this CTA cannot
        // wait on: give them a millisecond to land before shared memory can be released
        const uint64_t t0 = sm100::global_timer_ns();
        while (sm100::global_timer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      const uint32_t idesc0 = sm100::idesc_f32acc(256, 0, OpFormat<OpT>::value);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int t = cl; t < tiles && ok; t += ncl) {
        int p, g, fp, tt;
        decode(t, p, g, fp, tt);
        const int kblk = (k_of(p) / C::BK) * (kx_lo_of(p) ? 2 : 1), kst = (kblk + 1) / 2;
        const uint32_t idesc = idesc0 | (static_cast<uint32_t>(tile_tokens(tt) >> 3) << 17);
        if (!sm100::mbar_wait(tempty_bar(acc), aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::ACC_COLS);
        for (int ks = 0; ks < kst; ++ks) {
          if (!sm100::mbar_wait(full_bar(stage), ph, abort_flag)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const int nb = (2 * ks + 1 < kblk) ? 2 : 1;
          const uint32_t sa = ring + static_cast<uint32_t>(stage) * 2u * BLK;
          for (int b = 0; b < nb; ++b) {
            const uint64_t adesc = sm100::smem_desc_k128(sa + b * BLK);
            const uint64_t bdesc = sm100::smem_desc_k128(sa + b * BLK + C::W_BYTES);
#pragma unroll
            for (int k = 0; k < C::BK / 16; ++k)
              sm100::mma_pair(d_tmem, adesc + 2ull * k, bdesc + 2ull * k, idesc, (ks | b | k) != 0);
          }
          sm100::mma_commit_pair_cta_mask(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        sm100::mma_commit_pair_cta_mask(tfull_bar(acc), 0x3);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        if (a0.err) atomicOr(a0.err, kErrTimeoutMma);
        sm100::mma_commit_pair(sm100::mapa_shared(drain_bar, 0));
        sm100::mbar_wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;    // TMEM lanes 32 * quarter .. +31 belong to this warp
    const int wg = (warp - 2) >> 2;  // token half of the tile handled by this warpgroup
    const int wq = (warp - 2) & 3;   // this warp's rank inside its warpgroup
    const int ew = warp - 2;
    float* red_all = reinterpret_cast<float*>(smem + C::RED_OFF);
    float* rs_all = reinterpret_cast<float*>(smem + C::RS_OFF);
    const uint32_t tempty_lead0 = sm100::mapa_shared(tempty_bar(0), 0);
    const uint32_t tempty_lead1 = sm100::mapa_shared(tempty_bar(1), 0);
    int acc = 0;
    uint32_t aph = 0, wph = 0;
    float amax = 0.f;  // largest magnitude stored as an f16 operand
    bool ok = true;
    // the four warps of this warpgroup meet (bounded); false on a timeout
    auto wg_sync = [&]() {
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(wg_bar(wg));
      const bool r = __all_sync(0xffffffffu, sm100::mbar_wait(wg_bar(wg), wph, abort_flag));
      wph ^= 1u;
      if (!r && lane == 0 && a0.err) atomicOr(a0.err, kErrTimeoutEpilogue);
      return r;
    };
    // one tile of phase epilogue kind EPI with that phase's arguments; the next tile's cell and
    // position (gn < 0: none in this phase) for the residual epilogue's L2 warm-up
    auto epi_tile = [&](auto epi_kind, const TcGemmArgs& a, const Cell& c, int fp, int tt, int gn, int fpn,
                        int ttn) -> bool {
      constexpr int EPI = decltype(epi_kind)::value;
      const EpiParams& ep = a.ep;
      const int nt = tile_tokens(tt), cnt = nt / 2;
      const int tok0 = tt * NT + wg * cnt;
      const int fcta = fp * 256 + static_cast<int>(rank) * C::FM;  // first feature of this CTA
      const int f = fcta + quarter * 32 + lane;
      float* rs = rs_all + (acc * 2 + wg) * 128;
      if constexpr (EPI == kEpiRope || EPI == kEpiSwiGLU) {
        // folded RMSNorm: each warp computes the row scales of 32 of the warpgroup's tokens,
        // ahead of the accumulator wait, and the warpgroup shares them
        const int k = wq * 32 + lane, tok = tok0 + k;
        if (k < cnt)
          rs[k] = (ep.ss_in && tok < M)
                      ? row_scale(ep.ss_in + (static_cast<size_t>(c.k) * M + tok) * ep.ss_parts, ep.ss_parts, ep.inv_d,
                                  ep.rms_eps)
                      : 1.f;
        if (!wg_sync()) return false;
      }
      if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
        // warm L2 with the residual rows of this CTA's next tile (its rows of 128 features)
        if (gn >= 0) {
          const Cell cn = load_cell(a.cells, gn);
          const int k = ew * 32 + lane, ntn = tile_tokens(ttn);
          if (k < ntn && ttn * NT + k < M) {
            const size_t si = cell_index(ep.src_mode, a.L, cn);
            sm100::prefetch_l2_bulk(ep.x + (si * M + ttn * NT + k) * ep.ldx + fpn * 256 + rank * C::FM, C::FM * 4);
          }
        }
      }
      if (!__all_sync(0xffffffffu, sm100::mbar_wait(tfull_bar(acc), aph, abort_flag))) {
        if (lane == 0 && a0.err) atomicOr(a0.err, kErrTimeoutEpilogue);
        return false;
      }
      sm100::tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(acc * C::ACC_COLS + wg * cnt);
      float* red = red_all + ((acc * 2 + wg) * 4 + quarter) * 128;
      pair_epilogue<EPI, OpT, SPLIT>(a, c, tacc, tok0, cnt, f, lane, rs, red, amax);
      // accumulator drained (every lane's tcgen05.ld waited for): release it to the even CTA's
      // MMA issuer. The issuer reads none of this warp's global stores, so the arrive is
      // relaxed and does not wait for them to drain.
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive_cluster_relaxed(acc ? tempty_lead1 : tempty_lead0);
      if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
        if (ep.ss_out) {
          // the four warps of this warpgroup hold 32-feature sums of the same tokens: combine
          // them in quarter order into one partial per (token, 128-feature block)
          if (!wg_sync()) return false;
          const float* rb = red_all + (acc * 2 + wg) * 4 * 128;
          const int k = wq * 32 + lane;
          const int tok = tok0 + k;
          if (k < cnt && tok < M)
            ep.ss_out[(static_cast<size_t>(c.k) * M + tok) * ep.ss_parts + fcta / C::FM] =
                ((rb[k] + rb[128 + k]) + rb[256 + k]) + rb[384 + k];
        }
      }
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
      return true;
    };
    for (int t = cl; t < tiles && ok; t += ncl) {
      int p, g, fp, tt;
      decode(t, p, g, fp, tt);
      const Cell c = load_cell(a0.cells, g);
      int gn = -1, fpn = 0, ttn = 0;
      if (t + ncl < tiles) {
        int pn;
        decode(t + ncl, pn, gn, fpn, ttn);
        if (pn != p) gn = -1;
      }
      if (NP > 1 && p > 0) {
        // the stores of the previous phase this tile's epilogue reads (residual rows, RMSNorm
        // statistics) are complete: the producer saw the same counter, and this acquire makes
        // them visible to this warp as well
        bool r = true;
        if (lane == 0)
          r = sm100::counter_wait(counter(p - 1, g, tt), kSignalsPerTile * static_cast<unsigned>(npair_of(p - 1)),
                                  abort_flag);
        __syncwarp();
        if (!__shfl_sync(0xffffffffu, r ? 1 : 0, 0)) {
          if (lane == 0 && a0.err) atomicOr(a0.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
      }
      if (p == 0) {
        ok = epi_tile(std::integral_constant<int, E0>{}, args.ph[0], c, fp, tt, gn, fpn, ttn);
      } else if (p == 1) {
        if constexpr (NP > 1) ok = epi_tile(std::integral_constant<int, E1>{}, args.ph[1], c, fp, tt, gn, fpn, ttn);
      } else {
        if constexpr (NP > 2) ok = epi_tile(std::integral_constant<int, E2>{}, args.ph[2], c, fp, tt, gn, fpn, ttn);
      }
      if (!ok) break;
      if (NP > 1 && p < NP - 1) {
        // this warp's share of the tile is stored: publish it to the next phase's tiles of the
        // same tokens (one release add per warp, after the warp's stores are ordered before it
        // and made visible to the tensor-memory-access proxy)
        sm100::fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) sm100::counter_release_add(counter(p, g, tt), 1u);
      }
    }
    report_f16_range<OpT>(amax, a0.err);
  }

  sm100::tc_fence_before();
  sm100::cluster_sync();  // no remote arrival or MMA can still target either CTA after this
  sm100::tc_fence_after();
  if (warp == 1) sm100::tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

int max_pair_clusters(const void* fn) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cached[dev]) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(PairCfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sms / 2;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// Split-operand launches (any phase with low terms, or fp32 q/k/v) take the SPLIT kernel.
inline bool pair_split(const PairChainArgs& args) {
  for (int p = 0; p < args.nphase; ++p)
    if (args.ph[p].kx_lo || args.ph[p].ep.lo_off || args.ph[p].ep.out_f32) return true;
  return false;
}

template <int E0, int E1, int E2, typename OpT, bool SPLIT>
cudaError_t launch_pair_chain_t(const CUtensorMap* tw, const CUtensorMap* tx, const PairChainArgs& args,
                                cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  const void* fn = reinterpret_cast<const void*>(tc_pair_gemm_kernel<E0, E1, E2, OpT, SPLIT>);
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const TcGemmArgs& a0 = args.ph[0];
  const int NT = a0.nt > 0 ? a0.nt : pair_token_tile(a0.M), ntt = (a0.M + NT - 1) / NT;
  if (NT % 16 != 0 || NT > 256) return cudaErrorInvalidValue;
  long tiles = 0;
  for (int p = 0; p < args.nphase; ++p) tiles += static_cast<long>(a0.G) * (args.ph[p].N / 256) * ntt;
  if (tiles <= 0) return cudaSuccess;
  const int maxc = max_pair_clusters(fn);  // every pair resident at once (the chained waits rely on it)
  const int clusters = static_cast<int>(tiles < maxc ? tiles : maxc);
  const int np = args.nphase;
  const cudaError_t e = launch_pdl(tc_pair_gemm_kernel<E0, E1, E2, OpT, SPLIT>, dim3(2 * clusters), dim3(PairCfg::THREADS),
                                   PairCfg::SMEM_BYTES, st, tw[0], tx[0], tw[np > 1 ? 1 : 0], tx[np > 1 ? 1 : 0],
                                   tw[np > 2 ? 2 : 0], tx[np > 2 ? 2 : 0], args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename OpT>
cudaError_t launch_pair_op(const CUtensorMap& tw, const CUtensorMap& tx, const TcGemmArgs& args, cudaStream_t st) {
  PairChainArgs c{};
  c.ph[0] = args;
  c.nphase = 1;
  if (pair_split(c)) {  // split-operand mode: the f16 operands only
    if constexpr (std::is_same<OpT, __half>::value) {
      switch (args.epi) {
        case kEpiResidCast: return launch_pair_chain_t<kEpiResidCast, kNoEpi, kNoEpi, OpT, true>(&tw, &tx, c, st);
        case kEpiRope: return launch_pair_chain_t<kEpiRope, kNoEpi, kNoEpi, OpT, true>(&tw, &tx, c, st);
        case kEpiSwiGLU: return launch_pair_chain_t<kEpiSwiGLU, kNoEpi, kNoEpi, OpT, true>(&tw, &tx, c, st);
      }
    }
    return cudaErrorInvalidValue;
  }
  switch (args.epi) {
    case kEpiStoreF32: return launch_pair_chain_t<kEpiStoreF32, kNoEpi, kNoEpi, OpT, false>(&tw, &tx, c, st);
    case kEpiStoreAct: return launch_pair_chain_t<kEpiStoreAct, kNoEpi, kNoEpi, OpT, false>(&tw, &tx, c, st);
    case kEpiResidCast: return launch_pair_chain_t<kEpiResidCast, kNoEpi, kNoEpi, OpT, false>(&tw, &tx, c, st);
    case kEpiRope: return launch_pair_chain_t<kEpiRope, kNoEpi, kNoEpi, OpT, false>(&tw, &tx, c, st);
    case kEpiSwiGLU: return launch_pair_chain_t<kEpiSwiGLU, kNoEpi, kNoEpi, OpT, false>(&tw, &tx, c, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool tc_pair_supported(int M, int N, int K, int epi, int head_dim) {
  if (M <= 0 || N <= 0 || N % 256 != 0 || K <= 0 || K % 64 != 0) return false;
  if (epi == kEpiResid) return false;  // 16-bit operands always refresh the operand copy (kEpiResidCast)
  if (epi == kEpiRope && (head_dim <= 0 || head_dim % 2 != 0)) return false;
  return pair_token_tile(M) <= 256;
}

int pair_pick_nt(int M, long G, long pairs) {
  const int coarse = pair_token_tile(M);
  if (coarse <= kPairFineTile) return coarse;
  static int clusters[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!clusters[dev]) {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    clusters[dev] = sms > 1 ? sms / 2 : 1;
  }
  // makespan in token-equivalents: rounds of the resident pairs x (tile tokens + a fixed
  // pipeline fill and drain of about 48 tokens' worth of MMA)
  auto cost = [&](int nt) {
    const long tiles = G * pairs * ((M + nt - 1) / nt);
    return ((tiles + clusters[dev] - 1) / clusters[dev]) * (nt + 48);
  };
  return cost(kPairFineTile) < cost(coarse) ? kPairFineTile : coarse;
}

// A split-operand X keeps its low terms at a 16-byte aligned column at or past its high terms.
static bool kx_lo_ok(const TcGemmArgs& a) { return a.kx_lo == 0 || (a.kx_lo >= a.K && a.kx_lo % 8 == 0); }

cudaError_t launch_tc_pair_gemm(const CUtensorMap& tw, const CUtensorMap& tx, const TcGemmArgs& args, bool f16,
                                cudaStream_t st) {
  if (!tc_pair_supported(args.M, args.N, args.K, args.epi, args.ep.head_dim) || !kx_lo_ok(args))
    return cudaErrorInvalidValue;
  return f16 ? launch_pair_op<__half>(tw, tx, args, st) : launch_pair_op<__nv_bfloat16>(tw, tx, args, st);
}

cudaError_t launch_tc_pair_chain_o_mlp(const CUtensorMap* tw, const CUtensorMap* tx, const PairChainArgs& args,
                                       cudaStream_t st) {
  const TcGemmArgs* a = args.ph;
  if (args.nphase != 3 || !args.ctr || args.ctr_len <= 0 || a[0].epi != kEpiResidCast || a[1].epi != kEpiSwiGLU ||
      a[2].epi != kEpiResidCast)
    return cudaErrorInvalidValue;
  for (int p = 0; p < 3; ++p) {
    if (!tc_pair_supported(a[p].M, a[p].N, a[p].K, a[p].epi, a[p].ep.head_dim) || !kx_lo_ok(a[p]) || a[p].M != a[0].M ||
        a[p].G != a[0].G || a[p].cells != a[0].cells)
      return cudaErrorInvalidValue;
  }
  const int NT = a[0].nt > 0 ? a[0].nt : pair_token_tile(a[0].M);
  if (static_cast<long>(a[0].G) * ((a[0].M + NT - 1) / NT) > args.ctr_len) return cudaErrorInvalidValue;
  if (pair_split(args)) return launch_pair_chain_t<kEpiResidCast, kEpiSwiGLU, kEpiResidCast, __half, true>(tw, tx, args, st);
  return launch_pair_chain_t<kEpiResidCast, kEpiSwiGLU, kEpiResidCast, __half, false>(tw, tx, args, st);
}

}  // namespace rmt

// Grouped GEMM on 5th-generation tensor cores (sm_100a): Y_g = epi(X_g . W_l(g)^T).
//
// "Architecture Overview" of the diagonal-batching skill page: GroupedGEMM operations
// batch the matrix products of all layers on one diagonal into a single launch, each
// group with its own layer's weights. Here a group is one (layer, segment) cell; its
// weight is slice l of a [L, N, K] stack, addressed through the third coordinate of one
// TMA tensor map (no per-group pointer copies).
//
// Design (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      one thread issues TMA loads of A (128 x 64) and B (BN x 64) bf16 tiles,
//               128-byte swizzled, into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, K=16) into
//               one of two TMEM accumulators and commits to mbarriers;
//   warps 2-9   epilogue, two warpgroups each taking half of the tile's columns:
//               tcgen05.ld of the finished accumulator (one row per thread), fused RoPE /
//               SwiGLU / residual add / cast, stores to global memory.
// The two accumulators let the epilogue of tile i overlap the MMAs of tile i+1.
// Every wait is bounded (see sm100.cuh); on a timeout the CTA drains its in-flight copies
// and MMAs, frees TMEM, records the failure in the error word and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {

// NBUF: 32 x 32 residual blocks per epilogue warp (two keep the next block's load in flight).
// Each epilogue warp also has a 32 x 32 staging block for the 16-bit copy of the residual.
template <int BN, int NBUF = 2>
struct TcCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BUF = NBUF * 32 * 32 * 4;  // per epilogue warp: NBUF 32 x 32 fp32 residual blocks
  static constexpr int XS_ROW = 80;             // staging row: 64 B of 16-bit values + 16 B of padding
  static constexpr int XS_BUF = 32 * XS_ROW;     // per epilogue warp
  static constexpr int RING_BUDGET = 232448 - 1024 - 2048 - 8 * EPI_BUF - 8 * XS_BUF;
  static constexpr int STAGES = (RING_BUDGET / STAGE_BYTES) > 8 ? 8 : (RING_BUDGET / STAGE_BYTES);
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static constexpr int NBAR = 2 * STAGES + 5 + 8 * NBUF;  // ring, accumulators, drain, NBUF per epilogue warp
  static constexpr int BAR_BYTES = 1024 * ((8 * NBAR + 16 + 1023) / 1024);
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int XS_OFF = EPI_OFF + 8 * EPI_BUF;
  static constexpr int SMEM_BYTES = 1024 + XS_OFF + 8 * XS_BUF;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

namespace {

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ void store32_f32(float* dst, const float* v) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// The epilogue runs on two warpgroups; each owns every TMEM lane (one row per thread, four
// warps covering the 128 rows) and half of the tile's columns, so twice the rows' bytes
// are in flight for the memory-bound residual and RoPE epilogues.
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;

// Epilogue of one 32-column chunk of one row (row per thread). `src` holds the residual
// values of the chunk for the residual kinds (loaded by the caller before the TMEM wait).
template <int EPI, typename OpT>
__device__ __forceinline__ float epi_chunk(const TcGemmArgs& a, Cell c, int row, int col, const uint32_t (&r)[32],
                                           const float4 (&src)[8], float& amax) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = u2f(r[j]);
  const EpiParams& ep = a.ep;
  if constexpr (EPI == kEpiStoreF32) {
    const size_t idx = cell_index(ep.out_mode, a.L, c);
    store32_f32(static_cast<float*>(ep.out) + (idx * a.M + row) * ep.ldo + col, v);
  } else if constexpr (EPI == kEpiStoreAct) {
    const size_t idx = cell_index(ep.out_mode, a.L, c);
    store32_16_split(static_cast<OpT*>(ep.out) + (idx * a.M + row) * ep.ldo + col, v, ep.lo_off);
    track_amax<OpT>(amax, v);
  } else if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
    const size_t di = cell_index(ep.dst_mode, a.L, c);
    float* dst = ep.x + (di * a.M + row) * ep.ldx + col;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[4 * q] += src[q].x;
      v[4 * q + 1] += src[q].y;
      v[4 * q + 2] += src[q].z;
      v[4 * q + 3] += src[q].w;
    }
    store32_f32(dst, v);
    if constexpr (EPI == kEpiResidCast) {
      const int ldxb = ep.ldxb ? ep.ldxb : ep.ldx;
      store32_16_split(static_cast<OpT*>(ep.xb) + (di * a.M + row) * ldxb + col, v, ep.lo_off);
      track_amax<OpT>(amax, v);
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
    return ss;
  }
  return 0.f;
}

// Epilogue of one tile row for column half `part` (0 or 1) of the tile.
template <int BN, int EPI, typename OpT>
__device__ __forceinline__ void epilogue_tile(const TcGemmArgs& a, uint32_t tacc, Cell c, int row, int n0, int part,
                                              float& amax) {
  const bool valid = row < a.M;
  const EpiParams& ep = a.ep;
  float rs = 1.f;  // folded RMSNorm scale of this row (RoPE and SwiGLU epilogues)
  if constexpr (EPI == kEpiRope || EPI == kEpiSwiGLU) {
    if (ep.ss_in && valid)
      rs = rms_row_scale(ep.ss_in + (static_cast<size_t>(c.k) * a.M + row) * ep.ss_parts, ep.ss_parts, ep.inv_d,
                         ep.rms_eps);
  }
  if constexpr (EPI == kEpiRope) {
    const int dh = ep.head_dim, half = dh >> 1;
    const size_t idx = cell_index(ep.out_mode, a.L, c);
    OpT* orow = static_cast<OpT*>(ep.out) + (idx * a.M + row) * ep.ldo;
    float* orow32 = static_cast<float*>(ep.out) + (idx * a.M + row) * ep.ldo;  // out_f32
    auto put = [&](int col, const float* v) {
      if (ep.out_f32)
        store32_f32(orow32 + col, v);
      else
        store32_16(orow + col, v);
    };
    const int heads = BN / dh;
    // rotation pairs (i, i + dh/2) of each head, in 32-wide units: heads * max(1, half/32)
    const int per_head = half >= 32 ? half / 32 : 1;
    const int units = heads * per_head;
    const int u0 = part * units / 2, u1 = (part + 1) * units / 2;
#pragma unroll 1
    for (int u = u0; u < u1; ++u) {
      const int h0 = (u / per_head) * dh;
      const bool rot = (n0 + h0) < ep.rope_cols;
      if (half >= 32) {
        const int p = (u % per_head) * 32;
        uint32_t lo[32], hi[32];
        sm100::tmem_ld32(tacc + h0 + p, lo);
        sm100::tmem_ld32(tacc + h0 + half + p, hi);
        sm100::tmem_wait_ld();
        if (valid) {
          float x1[32], x2[32];
          // (cos, sin) of two frequencies per 16-byte load
          const float4* cs = reinterpret_cast<const float4*>(ep.rope + (size_t)row * half + p);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float a1 = u2f(lo[j]) * rs, a2 = u2f(hi[j]) * rs;
            if (rot) {
              const float4 t4 = cs[j >> 1];
              const float2 t = (j & 1) ? make_float2(t4.z, t4.w) : make_float2(t4.x, t4.y);
              x1[j] = a1 * t.x - a2 * t.y;
              x2[j] = a2 * t.x + a1 * t.y;
            } else {
              x1[j] = a1;
              x2[j] = a2;
            }
          }
          put(n0 + h0 + p, x1);
          put(n0 + h0 + half + p, x2);
          track_amax<OpT>(amax, x1);
          track_amax<OpT>(amax, x2);
        }
      } else {  // head_dim 32: both halves of the head in one 32-column chunk
        uint32_t r[32];
        sm100::tmem_ld32(tacc + h0, r);
        sm100::tmem_wait_ld();
        if (valid) {
          float x[32];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float a1 = u2f(r[j]) * rs, a2 = u2f(r[j + 16]) * rs;
            if (rot) {
              const float2 t = ep.rope[(size_t)row * 16 + j];
              x[j] = a1 * t.x - a2 * t.y;
              x[j + 16] = a2 * t.x + a1 * t.y;
            } else {
              x[j] = a1;
              x[j + 16] = a2;
            }
          }
          put(n0 + h0, x);
          track_amax<OpT>(amax, x);
        }
      }
    }
  } else if constexpr (EPI == kEpiSwiGLU) {
    const size_t idx = cell_index(ep.out_mode, a.L, c);
    OpT* orow = static_cast<OpT*>(ep.out) + (idx * a.M + row) * ep.ldo;
    constexpr int per_blk = kSwiGLUBlock / 32;  // 32-wide output units per gate/up block pair
    constexpr int units = (BN / (2 * kSwiGLUBlock)) * per_blk;
    const int u0 = part * units / 2, u1 = (part + 1) * units / 2;
#pragma unroll 1
    for (int u = u0; u < u1; ++u) {
      const int b0 = (u / per_blk) * 2 * kSwiGLUBlock, p = (u % per_blk) * 32;
      uint32_t g[32], up[32];
      sm100::tmem_ld32(tacc + b0 + p, g);
      sm100::tmem_ld32(tacc + b0 + kSwiGLUBlock + p, up);
      sm100::tmem_wait_ld();
      if (valid) {
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = silu_f(u2f(g[j]) * rs) * (u2f(up[j]) * rs);
        store32_16_split(orow + (n0 + b0) / 2 + p, y, ep.lo_off);
        track_amax<OpT>(amax, y);
      }
    }
  } else {
    constexpr int chunks = BN / 32;
    const int c0 = part * chunks / 2, c1 = (part + 1) * chunks / 2;
    const float* src_row = nullptr;
    if constexpr (EPI == kEpiResid || EPI == kEpiResidCast)
      src_row = ep.x + (static_cast<size_t>(cell_index(ep.src_mode, a.L, c)) * a.M + (valid ? row : 0)) * ep.ldx + n0;
    float ss = 0.f;
#pragma unroll 1
    for (int cc = c0; cc < c1; ++cc) {
      uint32_t r[32];
      float4 src[8];
      sm100::tmem_ld32(tacc + cc * 32, r);
      if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
        // residual loads go out before the TMEM wait so both latencies overlap
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q) src[q] = reinterpret_cast<const float4*>(src_row + cc * 32)[q];
        }
      }
      sm100::tmem_wait_ld();
      if (valid) ss += epi_chunk<EPI, OpT>(a, c, row, n0 + cc * 32, r, src, amax);
    }
    if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
      if (ep.ss_out && valid)
        ep.ss_out[(static_cast<size_t>(c.k) * a.M + row) * ep.ss_parts + (n0 / BN) * 2 + part] = ss;
    }
  }
}

// Residual epilogue of one warp (tile rows rowbase .. rowbase+31, one per lane) over its
// column half, through TMA: each 32 x 32 block of the residual stream is loaded into one of
// the warp's NBUF swizzled shared blocks, the accumulator rows are added in place, and the
// block is stored back with one bulk copy; the operand-type copy goes out with plain stores.
// Up to NBUF block loads are in flight: a block is refilled with chunk k + NBUF as soon as the
// store of chunk k has read it. rbar is block 0's barrier (block b's is 8 b bytes further);
// bit b of rph is block b's phase.
template <int BN, int EPI, typename OpT, int NBUF>
__device__ __forceinline__ bool epilogue_resid_tma(const TcGemmArgs& a, const CUtensorMap* tmX, uint32_t tacc, Cell c,
                                                   int rowbase, int n0, int part, int lane, uint8_t* buf,
                                                   uint32_t buf_s, uint32_t rbar, uint32_t& rph,
                                                   volatile int* abort_flag, uint8_t* xstage, float& amax) {
  const EpiParams& ep = a.ep;
  if (rowbase >= a.M) return true;  // the whole block lies past the cell
  const int row = rowbase + lane;
  const bool valid = row < a.M;
  const int src = cell_index(ep.src_mode, a.L, c), dst = cell_index(ep.dst_mode, a.L, c);
  constexpr int chunks = BN / 32, BLK = 32 * 32 * 4;
  const int c0 = part * chunks / 2, c1 = (part + 1) * chunks / 2;
  uint32_t pend = 0;  // blocks whose load is in flight (lane 0's view)
  auto issue = [&](int cc, int b) {
    sm100::bulk_wait_read_all();  // the last store from block b has read it
    sm100::mbar_arrive_expect_tx(rbar + 8u * b, BLK);
    sm100::tma_load_3d(buf_s + b * BLK, tmX, n0 + cc * 32, rowbase, src, rbar + 8u * b);
    pend |= 1u << b;
  };
  if (lane == 0)
    for (int j = 0; j < NBUF && c0 + j < c1; ++j) issue(c0 + j, j);
  float ss = 0.f;
#pragma unroll 1
  for (int cc = c0; cc < c1; ++cc) {
    const int b = (cc - c0) % NBUF;
    const int col = n0 + cc * 32;
    uint32_t r[32];
    sm100::tmem_ld32(tacc + cc * 32, r);
    sm100::tmem_wait_ld();
    if (!__all_sync(0xffffffffu, sm100::mbar_wait(rbar + 8u * b, (rph >> b) & 1u, abort_flag))) {
      if (lane == 0) {  // let every load in flight land before the blocks are reused
        for (int x = 0; x < NBUF; ++x)
          if (pend & (1u << x)) sm100::mbar_wait_drain(rbar + 8u * x, (rph >> x) & 1u);
      }
      return false;
    }
    rph ^= 1u << b;
    pend &= ~(1u << b);
    float4* rowp = reinterpret_cast<float4*>(buf + b * BLK + lane * 128);
    float y[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 xv = rowp[q ^ (lane & 7)];  // 128-byte swizzle: chunk q of row r sits at q ^ (r % 8)
      xv.x += u2f(r[4 * q]);
      xv.y += u2f(r[4 * q + 1]);
      xv.z += u2f(r[4 * q + 2]);
      xv.w += u2f(r[4 * q + 3]);
      rowp[q ^ (lane & 7)] = xv;
      y[4 * q] = xv.x;
      y[4 * q + 1] = xv.y;
      y[4 * q + 2] = xv.z;
      y[4 * q + 3] = xv.w;
    }
    if (valid) {
#pragma unroll
      for (int j = 0; j < 32; ++j) ss = fmaf(y[j], y[j], ss);
    }
    if constexpr (EPI == kEpiResidCast) {
      if (valid) track_amax<OpT>(amax, y);
      // the 16-bit copy: stage the warp's 32 x 32 block, then store it row by row, each
      // instruction covering 8 rows x 64 contiguous bytes
      // (split-operand mode: a second pass stores the low terms lo_off columns further)
      const int ldxb = ep.ldxb ? ep.ldxb : ep.ldx;
      uint4* mine = reinterpret_cast<uint4*>(xstage + lane * 80);
      OpT* xb = static_cast<OpT*>(ep.xb) + ((size_t)dst * a.M + rowbase) * ldxb + col + (lane & 3) * 8;
#pragma unroll 1
      for (int pass = 0; pass < (ep.lo_off ? 2 : 1); ++pass) {
        if (pass == 1) {
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = lo_term<OpT>(y[j]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          mine[q] = make_uint4(pack2<OpT>(y[8 * q], y[8 * q + 1]), pack2<OpT>(y[8 * q + 2], y[8 * q + 3]),
                               pack2<OpT>(y[8 * q + 4], y[8 * q + 5]), pack2<OpT>(y[8 * q + 6], y[8 * q + 7]));
        __syncwarp();
        OpT* xp = xb + pass * ep.lo_off;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r2 = (lane >> 2) + 8 * k;
          if (rowbase + r2 < a.M)
            *reinterpret_cast<uint4*>(xp + static_cast<size_t>(r2) * ldxb) =
                *reinterpret_cast<const uint4*>(xstage + r2 * 80 + (lane & 3) * 16);
        }
        __syncwarp();
      }
    }
    sm100::fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (!ep.resid_no_store) {
        sm100::tma_store_3d(tmX, buf_s + b * BLK, col, rowbase, dst);
        sm100::bulk_commit();
      }
      if (cc + NBUF < c1) issue(cc + NBUF, b);
    }
  }
  if (ep.ss_out && valid) ep.ss_out[(static_cast<size_t>(c.k) * a.M + row) * ep.ss_parts + (n0 / BN) * 2 + part] = ss;
  return true;
}

// RoPE epilogue of one warp (tile rows rowbase .. rowbase+31, one per lane) over its share
// of the tile's heads. The (cos, sin) pairs of the warp's 32 rows and 32 frequencies come
// into the warp's shared block with one TMA load (f16 pairs, 128-byte rows, swizzled) and
// are reused for every head of the tile; units are ordered frequency block first, so a
// warp loads each block once per tile. Only for head_dim >= 64.
template <int BN, typename OpT>
__device__ __forceinline__ bool epilogue_rope_tma(const TcGemmArgs& a, const CUtensorMap* tmR, uint32_t tacc, Cell c,
                                                  int rowbase, int n0, int part, int lane, const uint8_t* buf,
                                                  uint32_t buf_s, uint32_t rbar, uint32_t& rph,
                                                  volatile int* abort_flag, float& amax) {
  const EpiParams& ep = a.ep;
  if (rowbase >= a.M) return true;
  const int row = rowbase + lane;
  const bool valid = row < a.M;
  const int dh = ep.head_dim, half = dh >> 1;
  const int heads = BN / dh, per_head = half / 32, units = heads * per_head;
  const int u0 = part * units / 2, u1 = (part + 1) * units / 2;
  float rs = 1.f;
  if (ep.ss_in && valid)
    rs = rms_row_scale(ep.ss_in + (static_cast<size_t>(c.k) * a.M + row) * ep.ss_parts, ep.ss_parts, ep.inv_d,
                       ep.rms_eps);
  const size_t idx = cell_index(ep.out_mode, a.L, c);
  OpT* orow = static_cast<OpT*>(ep.out) + (idx * a.M + row) * ep.ldo;
  const uint4* rowp = reinterpret_cast<const uint4*>(buf + lane * 128);
  int loaded = -1;
#pragma unroll 1
  for (int u = u0; u < u1; ++u) {
    const int pb = u / heads, h0 = (u % heads) * dh, p = pb * 32;
    const bool rot = (n0 + h0) < ep.rope_cols;
    if (rot && pb != loaded) {
      if (lane == 0) {
        sm100::mbar_arrive_expect_tx(rbar, 32 * 32 * 4);
        sm100::tma_load_3d(buf_s, tmR, 2 * p, rowbase, 0, rbar);
      }
      if (!__all_sync(0xffffffffu, sm100::mbar_wait(rbar, rph & 1u, abort_flag))) {
        if (lane == 0) sm100::mbar_wait_drain(rbar, rph & 1u);
        return false;
      }
      rph ^= 1u;
      loaded = pb;
    }
    uint32_t lo[32], hi[32];
    sm100::tmem_ld32(tacc + h0 + p, lo);
    sm100::tmem_ld32(tacc + h0 + half + p, hi);
    sm100::tmem_wait_ld();
    if (valid) {
      float x1[32], x2[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // 16-byte chunk q of the row holds frequencies 4q .. 4q+3
        const uint4 w = rowp[q ^ (lane & 7)];
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * q + e;
          const float a1 = u2f(lo[j]) * rs, a2 = u2f(hi[j]) * rs;
          if (rot) {
            const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
            x1[j] = a1 * t.x - a2 * t.y;
            x2[j] = a2 * t.x + a1 * t.y;
          } else {
            x1[j] = a1;
            x2[j] = a2;
          }
        }
      }
      store32_16(orow + n0 + h0 + p, x1);
      store32_16(orow + n0 + h0 + half + p, x2);
      track_amax<OpT>(amax, x1);
      track_amax<OpT>(amax, x2);
    }
  }
  return true;
}

// Memory-read epilogue: stage this warp's half of the cell's A (columns part*dv/2 .. +dv/2,
// row-major [dk][dv/2]) and z into the warp's own shared block, before the accumulator wait.
// Each warp holds a private copy, so only the warp itself must be done with the previous one.
template <int BN>
__device__ __forceinline__ void stage_mem_state(const TcGemmArgs& a, Cell c, int part, int lane, float* As, float* zs) {
  const EpiParams& ep = a.ep;
  const int dv = ep.mem_dv, hv = dv / 2;
  const size_t si = cell_index(kByLayer, a.L, c);
  const float* A = ep.mem_A + si * BN * dv + part * hv;
  __syncwarp();  // the warp's previous tile has read its copy
  for (int e = lane; e < BN * hv / 4; e += 32) {
    const int i = e / (hv / 4), j4 = e % (hv / 4);
    reinterpret_cast<float4*>(As)[e] = *reinterpret_cast<const float4*>(A + static_cast<size_t>(i) * dv + 4 * j4);
  }
  for (int i = lane; i < BN; i += 32) zs[i] = ep.mem_z[si * BN + i];
  __syncwarp();
}

// Memory-read epilogue of one row (row per thread), output columns part*dv/2 .. +dv/2: the
// query row is the accumulator (BN = d_k columns); o = phi(q) A / (phi(q) . z + eps) with
// both sums over i ascending in fp32.
template <int BN, typename OpT>
__device__ __forceinline__ void epilogue_mem_read(const TcGemmArgs& a, uint32_t tacc, Cell c, int row, int part,
                                                  const float* As, const float* zs, float& amax) {
  const EpiParams& ep = a.ep;
  constexpr int HV = 32;  // output columns per thread (d_v = 64)
  float fq[BN];
#pragma unroll
  for (int c32 = 0; c32 < BN / 32; ++c32) {
    uint32_t r[32];
    sm100::tmem_ld32(tacc + 32 * c32, r);
    sm100::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) fq[32 * c32 + j] = phi_f(u2f(r[j]));
  }
  if (row >= a.M) return;
  float den = 0.f;
#pragma unroll
  for (int i = 0; i < BN; ++i) den = fmaf(fq[i], zs[i], den);
  den += ep.mem_eps;
  float acc[HV];
#pragma unroll
  for (int j = 0; j < HV; ++j) acc[j] = 0.f;
#pragma unroll
  for (int i = 0; i < BN; ++i) {  // fully unrolled: fq stays in registers
    const float4* Ai = reinterpret_cast<const float4*>(As + i * HV);
#pragma unroll
    for (int j4 = 0; j4 < HV / 4; ++j4) {
      const float4 av = Ai[j4];
      acc[4 * j4] = fmaf(fq[i], av.x, acc[4 * j4]);
      acc[4 * j4 + 1] = fmaf(fq[i], av.y, acc[4 * j4 + 1]);
      acc[4 * j4 + 2] = fmaf(fq[i], av.z, acc[4 * j4 + 2]);
      acc[4 * j4 + 3] = fmaf(fq[i], av.w, acc[4 * j4 + 3]);
    }
  }
  const float inv = 1.f / den;
#pragma unroll
  for (int j = 0; j < HV; ++j) acc[j] *= inv;
  const size_t idx = cell_index(ep.out_mode, a.L, c);
  store32_16_split(static_cast<OpT*>(ep.out) + (idx * a.M + row) * ep.ldo + part * HV, acc, ep.lo_off);
  track_amax<OpT>(amax, acc);
}

template <int BN, int EPI, typename OpT, int NBUF>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmX, const TcGemmArgs args) {
  using C = TcCfg<BN, NBUF>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t bar0 = base + C::STAGES * C::STAGE_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 4);
  auto resid_bar = [&](int w) { return bar0 + 8u * (2 * C::STAGES + 5 + NBUF * w); };  // and the NBUF-1 after it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::STAGES * C::STAGE_BYTES + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(tfull_bar(a), 1);
      sm100::mbar_init(tempty_bar(a), kEpiWarps);
    }
    sm100::mbar_init(drain_bar, 1);
    for (int w = 0; w < NBUF * kEpiWarps; ++w) sm100::mbar_init(resid_bar(0) + 8u * w, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
    sm100::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmA);
    sm100::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), C::TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();  // this CTA holds its TMEM: the next kernel may be scheduled
  pdl_wait();     // operands and residuals come from the previous kernels of the stream

  const int mt = (args.M + C::BM - 1) / C::BM;
  const int nt = args.N / BN;
  const int kbw = args.K / C::BK;                    // 64-column blocks of the weight
  const int kbn = args.kx_lo ? 2 * kbw : kbw;        // of the product (split-operand mode: twice)
  const int tiles = args.G * mt * nt;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int g = t / (mt * nt), r = t % (mt * nt);
        const int n_tile = r / mt, m_tile = r % mt;
        const Cell c = load_cell(args.cells, g);
        const int a3 = cell_index(args.a_mode, args.L, c);
        for (int kb = 0; kb < kbn; ++kb) {
          if (!sm100::mbar_wait(empty_bar(stage), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t sa = base + stage * C::STAGE_BYTES;
          sm100::mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
          const int kw = (kb % kbw) * C::BK, kx = kw + (kb / kbw) * args.kx_lo;
          sm100::tma_load_3d(sa, &tmA, kx, m_tile * C::BM, a3, full_bar(stage));
          sm100::tma_load_3d(sa + C::A_BYTES, &tmB, kw, n_tile * BN, c.l, full_bar(stage));
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        if (args.err) atomicOr(args.err, kErrTimeoutProducer);
        // let the copies already in flight land before the CTA's shared memory goes away
        for (long j = issued - 1; j >= 0 && j >= issued - C::STAGES; --j)
          sm100::mbar_wait_drain(full_bar(static_cast<int>(j % C::STAGES)), static_cast<uint32_t>((j / C::STAGES) & 1));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_f32acc(C::BM, BN, OpFormat<OpT>::value);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        if (!sm100::mbar_wait(tempty_bar(acc), aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < kbn; ++kb) {
          if (!sm100::mbar_wait(full_bar(stage), ph, abort_flag)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t sa = base + stage * C::STAGE_BYTES;
          const uint64_t adesc = sm100::smem_desc_k128(sa);
          const uint64_t bdesc = sm100::smem_desc_k128(sa + C::A_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / 16; ++k) {
            // advance 16 bf16 (32 bytes) along K inside the swizzled 128-byte rows
            sm100::mma_bf16(d_tmem, adesc + 2ull * k, bdesc + 2ull * k, idesc, (kb | k) != 0);
          }
          sm100::mma_commit(empty_bar(stage));
          if (++stage == C::STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        sm100::mma_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        if (args.err) atomicOr(args.err, kErrTimeoutMma);
        sm100::mma_commit(drain_bar);
        sm100::mbar_wait_drain(drain_bar, 0);
      }
    }
    __syncwarp();
  } else {
    const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31 belong to this warp
    const int part = (warp - 2) / 4;     // column half of the tile handled by this warpgroup
    const int ew = warp - 2;
    uint8_t* rbuf = smem + C::EPI_OFF + ew * C::EPI_BUF;
    const uint32_t rbuf_s = base + C::EPI_OFF + ew * C::EPI_BUF;
    uint32_t rph = 0;
    int acc = 0;
    uint32_t aph = 0;
    float amax = 0.f;  // largest magnitude stored as an f16 operand
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int g = t / (mt * nt), r = t % (mt * nt);
      const int n_tile = r / mt, m_tile = r % mt;
      const Cell c = load_cell(args.cells, g);
      if constexpr (EPI == kEpiMemRead)
        stage_mem_state<BN>(args, c, part, lane, reinterpret_cast<float*>(rbuf),
                            reinterpret_cast<float*>(smem + C::XS_OFF + ew * C::XS_BUF));
      bool ok = __all_sync(0xffffffffu, sm100::mbar_wait(tfull_bar(acc), aph, abort_flag));
      if (!ok) {
        if (lane == 0 && args.err) atomicOr(args.err, kErrTimeoutEpilogue);
        break;
      }
      sm100::tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if constexpr (EPI == kEpiResid || EPI == kEpiResidCast) {
        ok = epilogue_resid_tma<BN, EPI, OpT, NBUF>(args, &tmX, tacc, c, m_tile * C::BM + quarter * 32, n_tile * BN, part,
                                                    lane, rbuf, rbuf_s, resid_bar(ew), rph, abort_flag,
                                                    smem + C::XS_OFF + ew * C::XS_BUF, amax);
        if (!ok) {
          if (lane == 0 && args.err) atomicOr(args.err, kErrTimeoutEpilogue);
          break;
        }
      } else if (EPI == kEpiRope && args.ep.rope_tma) {
        ok = epilogue_rope_tma<BN, OpT>(args, &tmX, tacc, c, m_tile * C::BM + quarter * 32, n_tile * BN, part, lane,
                                        rbuf, rbuf_s, resid_bar(ew), rph, abort_flag, amax);
        if (!ok) {
          if (lane == 0 && args.err) atomicOr(args.err, kErrTimeoutEpilogue);
          break;
        }
      } else if constexpr (EPI == kEpiMemRead) {
        epilogue_mem_read<BN, OpT>(args, tacc, c, m_tile * C::BM + quarter * 32 + lane, part,
                                   reinterpret_cast<const float*>(rbuf),
                                   reinterpret_cast<const float*>(smem + C::XS_OFF + ew * C::XS_BUF), amax);
      } else {
        epilogue_tile<BN, EPI, OpT>(args, tacc, c, m_tile * C::BM + quarter * 32 + lane, n_tile * BN, part, amax);
      }
      // accumulator read: the MMA issuer reads none of the epilogue's stores, so the arrive is
      // relaxed and does not wait for them
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive_relaxed(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    report_f16_range<OpT>(amax, args.err);
    if (lane == 0) sm100::bulk_wait_all();  // residual stores complete before the CTA leaves
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

int sm_count_cached() {
  static int count[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
  return count[dev];
}

template <int BN, int EPI, typename OpT, int NBUF = 2>
cudaError_t launch_bn_epi(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tx, const TcGemmArgs& args,
                          cudaStream_t st) {
  using C = TcCfg<BN, NBUF>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<BN, EPI, OpT, NBUF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int mt = (args.M + C::BM - 1) / C::BM;
  const long tiles = static_cast<long>(args.G) * mt * (args.N / BN);
  if (tiles <= 0) return cudaSuccess;
  const int grid = static_cast<int>(tiles < sm_count_cached() ? tiles : sm_count_cached());
  const cudaError_t e =
      launch_pdl(tc_gemm_kernel<BN, EPI, OpT, NBUF>, dim3(grid), dim3(kGemmThreads), C::SMEM_BYTES, st, ta, tb, tx, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int BN, typename OpT>
cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tx, const TcGemmArgs& args,
                      cudaStream_t st) {
  switch (args.epi) {
    case kEpiStoreF32: return launch_bn_epi<BN, kEpiStoreF32, OpT>(ta, tb, tx, args, st);
    case kEpiStoreAct: return launch_bn_epi<BN, kEpiStoreAct, OpT>(ta, tb, tx, args, st);
    case kEpiResid: return launch_bn_epi<BN, kEpiResid, OpT>(ta, tb, tx, args, st);
    case kEpiResidCast: return launch_bn_epi<BN, kEpiResidCast, OpT>(ta, tb, tx, args, st);
    case kEpiRope:
      if constexpr (BN >= 64) return launch_bn_epi<BN, kEpiRope, OpT>(ta, tb, tx, args, st);
      break;
    case kEpiSwiGLU:
      if constexpr (BN >= 128) return launch_bn_epi<BN, kEpiSwiGLU, OpT>(ta, tb, tx, args, st);
      break;
    case kEpiMemRead:  // d_k = d_v = 64: each epilogue warp's copy of half of A fills its residual buffer
      if constexpr (BN == 64) {
        if (args.N == 64 && args.ep.mem_dv == 64) return launch_bn_epi<BN, kEpiMemRead, OpT>(ta, tb, tx, args, st);
      }
      break;
  }
  return cudaErrorInvalidValue;
}

template <typename OpT>
cudaError_t launch_op(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tx, const TcGemmArgs& args,
                      int bn, cudaStream_t st) {
  switch (bn) {
    case 256: return launch_bn<256, OpT>(ta, tb, tx, args, st);
    case 128: return launch_bn<128, OpT>(ta, tb, tx, args, st);
    case 64: return launch_bn<64, OpT>(ta, tb, tx, args, st);
    case 32: return launch_bn<32, OpT>(ta, tb, tx, args, st);
  }
  return cudaErrorInvalidValue;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

bool make_tmap_16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                     uint32_t box_rows, bool f16) {
  auto encode = get_encode_fn();
  if (!encode || !base || inner % 8 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_16_3d_strided(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                             uint64_t row_stride, uint32_t box_rows, bool f16) {
  auto encode = get_encode_fn();
  if (!encode || !base || inner % 8 != 0 || row_stride % 8 != 0 || row_stride < inner ||
      (reinterpret_cast<uintptr_t>(base) & 15) != 0)
    return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {row_stride * 2, row_stride * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                       uint32_t box_rows) {
  return make_tmap_16_3d(map, base, inner, rows, depth, box_rows, false);
}

int tc_pick_bn(int N, int epi, int head_dim) {
  const int cands[4] = {256, 128, 64, 32};
  for (int bn : cands) {
    if (N % bn) continue;
    if (epi == kEpiSwiGLU && bn < 128) continue;
    if (epi == kEpiRope && (bn < 64 || bn % head_dim)) continue;
    return bn;
  }
  return 0;
}

bool make_tmap_f32_resid(CUtensorMap* map, const float* base, uint64_t inner, uint64_t rows, uint64_t depth) {
  auto encode = get_encode_fn();
  if (!encode || !base || inner % 32 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {inner * 4, inner * rows * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_tc_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tx, const TcGemmArgs& args,
                           int bn, bool f16, cudaStream_t st) {
  if (args.K % 64 != 0 || args.M <= 0) return cudaErrorInvalidValue;
  if (args.kx_lo && (args.kx_lo < args.K || args.kx_lo % 8 != 0)) return cudaErrorInvalidValue;
  if (args.ep.out_f32 && (args.epi != kEpiRope || args.ep.rope_tma)) return cudaErrorInvalidValue;
  return f16 ? launch_op<__half>(ta, tb, tx, args, bn, st) : launch_op<__nv_bfloat16>(ta, tb, tx, args, bn, st);
}

}  // namespace rmt

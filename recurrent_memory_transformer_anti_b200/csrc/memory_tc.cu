// Associative-memory read on 5th-generation tensor cores (sm_100a), for 16-bit outputs and
// d_k a multiple of 64: o = phi(q) A / (phi(q) . z + eps), row by row.
//
// The read of a cell is a product of its query rows with [A | z] (d_k x (d_v + 1)): the
// numerators are columns 0..d_v-1 and the denominator is column d_v of the same product. q, A
// and z are fp32, so each operand is split into two bf16 terms (x = x1 + x2 with x1 = bf16(x),
// x2 = bf16(x - x1)) and the product is accumulated in fp32 as x1 y1 + x1 y2 + x2 y1: the
// dropped term x2 y2 is about 2^-16 of the result, well under the 16-bit output's rounding.
// In tcgen05 terms, per 128-row tile: D (128 x N, N = d_v + 16 with the z column and padding,
// in TMEM) = X1 Y1^T + X1 Y2^T + X2 Y1^T, three passes over d_k in K = 16 steps.
//
// Two kernels share this arithmetic. At d_k = 64, mem_read_ws_kernel (further down) gives each
// step of a tile (bulk loads, conversion, MMA, epilogue) warps of its own. At d_k = 128,
// mem_read_tc_kernel runs them in lockstep:
// a CTA (8 warps) is persistent over a contiguous range of the launch's 128-row tiles, so it
// meets few cell boundaries; at each one it writes the cell's [A | z], split and transposed
// (rows = output columns, as the K-major operand wants them), into shared memory. Per tile
// every thread converts its share of the query rows -- loaded into registers one tile ahead --
// to phi(q), splits it and writes both terms in the 128-byte-swizzled K-major layout that
// the MMA reads; one thread then issues the tile's MMAs into one of two TMEM accumulators,
// and the warps finish the previous tile: read its accumulator rows (one row per TMEM lane),
// divide, round and store. Loads of tile i+1, the MMAs of tile i and the epilogue of tile i-1
// overlap. Every wait is bounded; on a timeout the CTA records it in the error word and stops.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

constexpr int kRtThreads = 256;
constexpr int kRtRows = 128;  // rows per tile (the MMA's M)

template <int DK>
struct RtCfg {
  static constexpr int KB = DK / 64;                 // 64-column (128-byte) blocks of d_k
  static constexpr int XBLK = kRtRows * 128;         // one block of a query-term tile: 16 KB
  static constexpr int XTILE = 2 * KB * XBLK;        // both terms of one tile
  static constexpr int CHUNKS = kRtRows * DK / 8;    // 16-byte chunks (8 values) of one term of a tile
  static constexpr int PER_THREAD = CHUNKS / kRtThreads;
  static_assert(CHUNKS % kRtThreads == 0, "tile chunks per thread");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk c of row r in a K-major tile of 128-byte rows with the
// 128-byte swizzle (8-row groups 1024 bytes apart; the tile starts 1024-byte aligned).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// phi(x) = elu(x) + 1 without a branch, the exponential from the fast intrinsic (relative error
// about 2^-21, far below the 16-bit output's rounding): x + 1 for x > 0, exp(x) otherwise.
__device__ __forceinline__ float phi_fast(float x) { return x > 0.f ? x + 1.f : __expf(fminf(x, 0.f)); }

// phi as phi_fast without the clamp (the same values): for x > 0 the exponential (inf above
// about 88) is computed and not taken
__device__ __forceinline__ float phi_pos(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// Bounded CTA-wide barrier on an mbarrier that counts every thread's arrival.
__device__ __forceinline__ bool cta_sync_bounded(uint32_t bar, uint32_t& phase, volatile int* abort) {
  sm100::mbar_arrive(bar);
  const bool ok = sm100::mbar_wait(bar, phase, abort);
  phase ^= 1u;
  return ok;
}

template <typename T, int DK>
__global__ void __launch_bounds__(kRtThreads, DK == 64 ? 2 : 1) mem_read_tc_kernel(const MemReadArgs a, int* err) {
  using C = RtCfg<DK>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int dv = a.dv, M = a.M;
  const int N = dv + 16;  // MMA N: d_v numerators, the denominator column, zero padding
  // [query terms: 2 buffers x XTILE][Y1, Y2: KB blocks of N rows x 128 B each][barriers]
  const uint32_t xbuf = base;
  const uint32_t ybuf = base + 2 * C::XTILE;
  const uint32_t yblk = static_cast<uint32_t>(N) * 128;  // one 64-column block of a Y term
  const uint32_t bar0 = (ybuf + 2 * C::KB * yblk + 1023u) & ~1023u;
  const uint32_t mma_done0 = bar0, cta_bar = bar0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bar0 + 32 - base));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int acc_stride = N <= 128 ? 128 : 256;  // TMEM columns between the two accumulators
  const uint32_t tmem_cols = 2 * acc_stride;
  if (tid == 0) {
    sm100::mbar_init(mma_done0, 1);
    sm100::mbar_init(mma_done0 + 8, 1);
    sm100::mbar_init(cta_bar, kRtThreads);
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 0) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), tmem_cols);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream

  const int mt = (M + kRtRows - 1) / kRtRows;
  const long total = static_cast<long>(a.G) * mt;
  const long per_cta = (total + gridDim.x - 1) / gridDim.x;
  const long t_beg = blockIdx.x * per_cta, t_end = t_beg + per_cta < total ? t_beg + per_cta : total;
  const uint32_t idesc = sm100::idesc_f32acc(kRtRows, N, 1u);
  uint32_t cph = 0;  // cta_bar phase
  bool ok = true;

  // this thread's chunks of a tile: chunk e = tid + 256 u -> row e / (DK / 8), chunk e % (DK / 8)
  float4 q_reg[C::PER_THREAD][2];
  auto load_tile = [&](long t) {
    const int g = static_cast<int>(t / mt), r0 = static_cast<int>(t % mt) * kRtRows;
    const Cell c = load_cell(a.cells, g);
    const float* q = a.q + static_cast<size_t>(cell_index(a.mode, a.L, c)) * M * DK;
#pragma unroll
    for (int u = 0; u < C::PER_THREAD; ++u) {
      const int e = tid + kRtThreads * u, r = e / (DK / 8), ch = e % (DK / 8);
      if (r0 + r < M) {
        const float4* src = reinterpret_cast<const float4*>(q + static_cast<size_t>(r0 + r) * DK + 8 * ch);
        q_reg[u][0] = src[0];
        q_reg[u][1] = src[1];
      } else {
        q_reg[u][0] = q_reg[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  // [A | z] of cell g, split and transposed: row n < d_v is column n of A, row d_v is z, the
  // rest zero; 8 consecutive k of one row per 16-byte chunk
  auto load_state = [&](int g) {
    const Cell c = load_cell(a.cells, g);
    const size_t si = cell_index(a.state_mode, a.L, c);
    const float* A = a.A + si * DK * dv;
    const float* z = a.z + si * DK;
    for (int e = tid; e < N * (DK / 8); e += kRtThreads) {
      const int n = e % N, kc = e / N;  // consecutive threads: consecutive columns of A
      float x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int kk = 8 * kc + k;
        x[k] = n < dv ? A[static_cast<size_t>(kk) * dv + n] : (n == dv ? z[kk] : 0.f);
      }
      uint32_t h1[4], h2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a0 = x[2 * k], a1 = x[2 * k + 1];
        const float b0 = __bfloat162float(__float2bfloat16_rn(a0)), b1 = __bfloat162float(__float2bfloat16_rn(a1));
        h1[k] = pack_bf16x2(b0, b1);
        h2[k] = pack_bf16x2(a0 - b0, a1 - b1);
      }
      const uint32_t off = static_cast<uint32_t>(kc / 8) * yblk + swz128(n, kc % 8);
      uint8_t* y1 = smem + (ybuf - base) + off;
      *reinterpret_cast<uint4*>(y1) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
      *reinterpret_cast<uint4*>(y1 + C::KB * yblk) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
  };
  // the registers of one tile -> phi, split, swizzled into query-term buffer b
  auto store_tile = [&](int b) {
    uint8_t* x1 = smem + b * C::XTILE;
#pragma unroll
    for (int u = 0; u < C::PER_THREAD; ++u) {
      const int e = tid + kRtThreads * u, r = e / (DK / 8), ch = e % (DK / 8);
      const float v[8] = {q_reg[u][0].x, q_reg[u][0].y, q_reg[u][0].z, q_reg[u][0].w,
                          q_reg[u][1].x, q_reg[u][1].y, q_reg[u][1].z, q_reg[u][1].w};
      uint32_t h1[4], h2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p0 = phi_fast(v[2 * k]), p1 = phi_fast(v[2 * k + 1]);
        const float b0 = __bfloat162float(__float2bfloat16_rn(p0)), b1 = __bfloat162float(__float2bfloat16_rn(p1));
        h1[k] = pack_bf16x2(b0, b1);
        h2[k] = pack_bf16x2(p0 - b0, p1 - b1);
      }
      const uint32_t off = static_cast<uint32_t>(ch / 8) * C::XBLK + swz128(r, ch % 8);
      *reinterpret_cast<uint4*>(x1 + off) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
      *reinterpret_cast<uint4*>(x1 + C::KB * C::XBLK + off) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
    }
  };
  // one thread: D[acc] = X1 Y1^T + X1 Y2^T + X2 Y1^T for the tile in buffer b
  auto issue_mma = [&](int b) {
    const uint32_t d = tmem_base + static_cast<uint32_t>(b * acc_stride);
    const uint32_t xb = xbuf + b * C::XTILE;
    int s = 0;
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
      const uint32_t xa = xb + (pass == 2 ? C::KB * C::XBLK : 0);  // X1, X1, X2
      const uint32_t ya = ybuf + (pass == 1 ? C::KB * yblk : 0);   // Y1, Y2, Y1
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        const uint64_t ad = sm100::smem_desc_k128(xa + kb * C::XBLK);
        const uint64_t bd = sm100::smem_desc_k128(ya + kb * yblk);
#pragma unroll
        for (int k = 0; k < 4; ++k, ++s) sm100::mma_bf16(d, ad + 2ull * k, bd + 2ull * k, idesc, s > 0);
      }
    }
    sm100::mma_commit(mma_done0 + 8u * b);
  };
  // the finished tile t in accumulator b: rows of TMEM lanes 32 (warp % 4) .., columns of half
  // warp / 4 of the numerators, and the denominator column
  auto epilogue = [&](long t, int b) {
    const int g = static_cast<int>(t / mt), r0 = static_cast<int>(t % mt) * kRtRows;
    const Cell c = load_cell(a.cells, g);
    const int row = r0 + (warp & 3) * 32 + lane;
    const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t acc = tmem_base + lanes + static_cast<uint32_t>(b * acc_stride);
    uint32_t dn[16];
    sm100::tmem_ld16(acc + dv, dn);
    sm100::tmem_wait_ld();
    const float inv = 1.f / (__uint_as_float(dn[0]) + a.eps);
    const int ldo = a.ldo ? a.ldo : dv;
    T* o = static_cast<T*>(a.o) + (static_cast<size_t>(cell_index(a.mode, a.L, c)) * M + row) * ldo;
    const int half = dv / 2, c0 = (warp >> 2) * half;
    for (int cc = c0; cc < c0 + half; cc += 16) {
      uint32_t v[16];
      sm100::tmem_ld16(acc + cc, v);
      sm100::tmem_wait_ld();
      if (row < M) {
        float y[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) y[k] = __uint_as_float(v[k]) * inv;
#pragma unroll 1
        for (int pass = 0; pass < (a.lo_off ? 2 : 1); ++pass) {  // split-operand mode: then the low terms
          if (pass == 1) {
#pragma unroll
            for (int k = 0; k < 16; ++k) y[k] = lo_term<T>(y[k]);
          }
          uint32_t p[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) p[k] = pack2<T>(y[2 * k], y[2 * k + 1]);
          uint4* dst = reinterpret_cast<uint4*>(o + cc + pass * a.lo_off);
          dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
          dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
        }
      }
    }
  };

  int cell = -1;
  uint32_t mph[2] = {0u, 0u};  // phase of each accumulator's completion barrier
  if (t_beg < t_end) load_tile(t_beg);
  for (long t = t_beg; t < t_end && ok; ++t) {
    const int i = static_cast<int>(t - t_beg), b = i & 1;
    const int g = static_cast<int>(t / mt);
    if (g != cell) {
      // a new cell: the previous tile's MMAs must be done with [A | z] before it is rewritten
      if (i > 0 && !sm100::mbar_wait(mma_done0 + 8u * (b ^ 1), mph[b ^ 1], abort_flag)) {
        ok = false;
        break;
      }
      load_state(g);
      cell = g;
    }
    store_tile(b);  // buffer b was last read by the MMAs of tile i-2, finished before epilogue i-2
    if (t + 1 < t_end) load_tile(t + 1);
    sm100::fence_async_smem();
    if (!cta_sync_bounded(cta_bar, cph, abort_flag)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      sm100::tc_fence_after();
      issue_mma(b);
    }
    if (i > 0) {
      if (!sm100::mbar_wait(mma_done0 + 8u * (b ^ 1), mph[b ^ 1], abort_flag)) {
        ok = false;
        break;
      }
      mph[b ^ 1] ^= 1u;
      sm100::tc_fence_after();
      epilogue(t - 1, b ^ 1);
      sm100::tc_fence_before();
    }
  }
  if (ok && t_end > t_beg) {
    const int b = static_cast<int>(t_end - 1 - t_beg) & 1;
    if (sm100::mbar_wait(mma_done0 + 8u * b, mph[b], abort_flag)) {
      sm100::tc_fence_after();
      epilogue(t_end - 1, b);
    } else {
      ok = false;
    }
  }
  if (!ok) {
    if (tid == 0 && err) atomicOr(err, kErrTimeoutEpilogue);
    // let the MMAs already issued finish before the shared memory and TMEM go away
    if (tid == 0) {
      sm100::mma_commit(mma_done0);
      sm100::mbar_wait_drain(mma_done0, mph[0]);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ----------------------------------------------------------------- d_k = 64: warp-specialised
//
// At d_k = 64 a 128-row tile of query rows is 32 KB of contiguous fp32, so the read is a
// stream, and its pace is set by how far ahead of each other the per-tile steps can run. Each
// step has warps of its own, linked by mbarriers:
//   - the stream warp bulk-copies each tile's query rows into a ring of shared-memory stages,
//     and each cell's A and z into a staging buffer, running ahead of the rest;
//   - 8 converter warps turn a stage, in place, into the two bf16 terms of phi(q): the
//     MMA operands are K-major with the 128-byte swizzle and their 8-row groups 2048 bytes
//     apart, X1 in the first 1024 bytes of a group and X2 in the second, which are exactly the
//     bytes of the group's 8 fp32 rows, so a warp that owns whole groups reads them, syncs and
//     overwrites them (and, at the first tile of a cell, writes the staged [A | z] into Y);
//   - one MMA warp issues the tile's 12 MMAs into one of four TMEM accumulators (two when
//     d_v + 16 > 128) and hands the stage back to the stream when they finish;
//   - 4 epilogue warps (one per TMEM lane quarter) read a finished accumulator, release it,
//     and divide, round and store their rows.
// A stage is thus held from its load to its MMAs, and the ring (4-6 stages) keeps that many
// tiles in flight. The arithmetic is the same as in mem_read_tc_kernel, term for term.
constexpr int kWsConvWarps = 8;
constexpr int kWsEpiWarps = 4;  // 8 (two per lane quarter, half the columns each) measured the same
constexpr int kWsStreamWarp = kWsConvWarps + kWsEpiWarps;  // warp 12
constexpr int kWsMmaWarp = kWsStreamWarp + 1;               // warp 13
constexpr int kWsThreads = (kWsMmaWarp + 1) * 32;
static_assert(kWsEpiWarps % 4 == 0, "whole TMEM lane quarters");
constexpr uint32_t kWsStage = kRtRows * 64 * 4;  // one tile of fp32 query rows, then of its operands
constexpr uint32_t kWsGroup = 2048;              // one 8-row group: 8 fp32 rows, or X1 | X2
constexpr int kWsMaxStages = 6;

__host__ __device__ constexpr uint32_t ws_round1k(uint32_t b) { return (b + 1023u) & ~1023u; }

struct WsLayout {  // byte offsets from the 1024-byte-aligned base
  uint32_t y, st, bar, total;
  __host__ __device__ constexpr WsLayout(int dv, int nst)
      : y(static_cast<uint32_t>(nst) * kWsStage),
        st(y + ws_round1k(2u * static_cast<uint32_t>(dv + 16) * 128u)),
        bar(st + ws_round1k((64u * static_cast<uint32_t>(dv) + 64u) * 4u)),
        total(bar + 256) {}
};
// barriers (8 bytes each) from lay.bar: per stage, per accumulator, then single ones
constexpr uint32_t kWsFull = 0, kWsXFull = 48, kWsEmpty = 96, kWsMmaDone = 144, kWsAccFree = 176, kWsStFull = 208,
                   kWsStEmpty = 216, kWsFin = 224, kWsSlot = 232;

template <typename T>
__global__ void __launch_bounds__(kWsThreads, 1) mem_read_ws_kernel(const MemReadArgs a, int* err, int nst) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const int dv = a.dv, M = a.M;
  const int N = dv + 16;  // MMA N: d_v numerators, the denominator column, zero padding
  const WsLayout lay(dv, nst);
  const uint32_t ring = base, ybuf = base + lay.y, stbuf = base + lay.st;
  const uint32_t bar = base + lay.bar;
  const uint32_t full0 = bar + kWsFull, xfull0 = bar + kWsXFull, empty0 = bar + kWsEmpty;
  const uint32_t mma_done0 = bar + kWsMmaDone, acc_free0 = bar + kWsAccFree;
  const uint32_t st_full = bar + kWsStFull, st_empty = bar + kWsStEmpty, fin = bar + kWsFin;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + lay.bar + kWsSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t yblk = static_cast<uint32_t>(N) * 128;  // one term of Y
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // TMEM accumulators of N columns each: four 128 apart, or two 256 apart when N > 128
  const int nacc = N <= 128 ? 4 : 2;
  const uint32_t acc_stride = N <= 128 ? 128u : 256u;
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      sm100::mbar_init(full0 + 8 * s, 1);
      sm100::mbar_init(xfull0 + 8 * s, kWsConvWarps);
      sm100::mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 4; ++b) {
      sm100::mbar_init(mma_done0 + 8 * b, 1);
      sm100::mbar_init(acc_free0 + 8 * b, kWsEpiWarps);
    }
    sm100::mbar_init(st_full, 1);
    sm100::mbar_init(st_empty, kWsConvWarps);
    sm100::mbar_init(fin, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == kWsMmaWarp) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), 512);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream

  const int mt = (M + kRtRows - 1) / kRtRows;
  const long total = static_cast<long>(a.G) * mt;
  const long per_cta = (total + gridDim.x - 1) / gridDim.x;
  const long t_beg = blockIdx.x * per_cta, t_end = t_beg + per_cta < total ? t_beg + per_cta : total;
  long issued = 0;        // stream warp: tiles whose rows were requested
  uint32_t st_loads = 0;  // stream warp: cell states requested

  if (warp == kWsStreamWarp) {
    if (lane == 0) {
      int cell = -1;
      for (long t = t_beg; t < t_end; ++t) {
        const int g = static_cast<int>(t / mt), r0 = static_cast<int>(t % mt) * kRtRows;
        const Cell c = load_cell(a.cells, g);
        if (g != cell) {  // the cell's [A | z], once the converters are done with the previous one
          if (st_loads > 0 && !sm100::mbar_wait(st_empty, (st_loads - 1u) & 1u, abort_flag)) break;
          const size_t si = cell_index(a.state_mode, a.L, c);
          const uint32_t abytes = 64u * static_cast<uint32_t>(dv) * 4u;
          sm100::mbar_arrive_expect_tx(st_full, abytes + 256u);
          sm100::bulk_load(stbuf, a.A + si * 64 * dv, abytes, st_full);
          sm100::bulk_load(stbuf + abytes, a.z + si * 64, 256u, st_full);
          ++st_loads;
          cell = g;
        }
        const int s = static_cast<int>(issued % nst);
        const uint32_t use = static_cast<uint32_t>(issued / nst);
        // the stage is free once the MMAs of the tile nst before have read its operands
        if (use > 0 && !sm100::mbar_wait(empty0 + 8u * s, (use - 1u) & 1u, abort_flag)) break;
        const int rows = M - r0 < kRtRows ? M - r0 : kRtRows;
        const uint32_t bytes = static_cast<uint32_t>(rows) * 256u;
        sm100::mbar_arrive_expect_tx(full0 + 8u * s, bytes);
        sm100::bulk_load(ring + static_cast<uint32_t>(s) * kWsStage,
                         a.q + (static_cast<size_t>(cell_index(a.mode, a.L, c)) * M + r0) * 64, bytes, full0 + 8u * s);
        ++issued;
      }
    }
  } else if (warp == kWsMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = sm100::idesc_f32acc(kRtRows, N, 1u);
      long i = 0;
      for (long t = t_beg; t < t_end; ++t, ++i) {
        const int s = static_cast<int>(i % nst), b = static_cast<int>(i % nacc);
        const uint32_t u = static_cast<uint32_t>(i / nacc);
        if (!sm100::mbar_wait(xfull0 + 8u * s, static_cast<uint32_t>(i / nst) & 1u, abort_flag)) break;
        if (u > 0 && !sm100::mbar_wait(acc_free0 + 8u * b, (u - 1u) & 1u, abort_flag)) break;
        sm100::tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b) * acc_stride;
        const uint32_t xb = ring + static_cast<uint32_t>(s) * kWsStage;
        int k = 0;
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {  // X1 Y1, X1 Y2, X2 Y1
          const uint64_t ad = sm100::smem_desc_k128_sbo(xb + (pass == 2 ? 1024u : 0u), kWsGroup);
          const uint64_t bd = sm100::smem_desc_k128(ybuf + (pass == 1 ? yblk : 0u));
#pragma unroll
          for (int j = 0; j < 4; ++j, ++k) sm100::mma_bf16(d, ad + 2ull * j, bd + 2ull * j, idesc, k > 0);
        }
        sm100::mma_commit(empty0 + 8u * s);     // the stage's operands are read: back to the stream
        sm100::mma_commit(mma_done0 + 8u * b);  // the accumulator is complete
      }
    }
  } else if (warp >= kWsConvWarps) {
    // epilogue: warp 8 + e reads TMEM lane quarter e % 4 (one row per lane) and stores column
    // block e / 4 of those rows (all of them with four warps)
    const int e = warp - kWsConvWarps;
    const uint32_t lanes = static_cast<uint32_t>(32 * (e & 3)) << 16;
    const int ldo = a.ldo ? a.ldo : dv;
    const int width = dv / (kWsEpiWarps / 4), cb = (e >> 2) * width, ce = cb + width;
    long i = 0;
    for (long t = t_beg; t < t_end; ++t, ++i) {
      const int b = static_cast<int>(i % nacc);
      const uint32_t u = static_cast<uint32_t>(i / nacc);
      if (!sm100::mbar_wait(mma_done0 + 8u * b, u & 1u, abort_flag)) break;
      sm100::tc_fence_after();
      const int g = static_cast<int>(t / mt), r0 = static_cast<int>(t % mt) * kRtRows;
      const uint32_t acc = tmem_base + lanes + static_cast<uint32_t>(b) * acc_stride;
      const int row = r0 + 32 * (e & 3) + lane;
      const Cell c = load_cell(a.cells, g);
      T* o = static_cast<T*>(a.o) + (static_cast<size_t>(cell_index(a.mode, a.L, c)) * M + row) * ldo;
      uint32_t dn[8];
      sm100::tmem_ld8(acc + dv, dn);
      for (int c0 = cb; c0 < ce; c0 += 32) {  // 32 columns at a time
        const int nc = ce - c0 < 32 ? ce - c0 : 32;
        uint32_t v[2][16];
#pragma unroll
        for (int q = 0; q < 2; ++q)
          if (16 * q < nc) sm100::tmem_ld16(acc + c0 + 16 * q, v[q]);
        sm100::tmem_wait_ld();
        if (c0 + 32 >= ce) {  // this warp's last TMEM read of the accumulator
          sm100::tc_fence_before();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive_relaxed(acc_free0 + 8u * b);
        }
        const float inv = 1.f / (__uint_as_float(dn[0]) + a.eps);
        if (row < M) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (16 * q >= nc) break;
            float y[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) y[k] = __uint_as_float(v[q][k]) * inv;
#pragma unroll 1
            for (int pass = 0; pass < (a.lo_off ? 2 : 1); ++pass) {  // split-operand mode: then the low terms
              if (pass == 1) {
#pragma unroll
                for (int k = 0; k < 16; ++k) y[k] = lo_term<T>(y[k]);
              }
              uint32_t p[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) p[k] = pack2<T>(y[2 * k], y[2 * k + 1]);
              uint4* dst = reinterpret_cast<uint4*>(o + c0 + 16 * q + pass * a.lo_off);
              dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
              dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
            }
          }
        }
      }
    }
  } else {
    // converters (warps 0-7): warp w owns 8-row groups w and w + 8 of every tile
    int cell = -1;
    uint32_t st_used = 0;
    long i = 0;
    for (long t = t_beg; t < t_end; ++t, ++i) {
      const int s = static_cast<int>(i % nst);
      const int g = static_cast<int>(t / mt), r0 = static_cast<int>(t % mt) * kRtRows;
      if (!sm100::mbar_wait(full0 + 8u * s, static_cast<uint32_t>(i / nst) & 1u, abort_flag)) break;
      if (g != cell) {
        // a new cell: Y is read by the MMAs of tile i - 1 (and so of all before it); then the
        // staged [A | z] -> Y, split and transposed (row n < d_v: column n of A; row d_v: z;
        // the rest zero)
        if (i > 0 && !sm100::mbar_wait(empty0 + 8u * static_cast<uint32_t>((i - 1) % nst),
                                       static_cast<uint32_t>((i - 1) / nst) & 1u, abort_flag))
          break;
        if (!sm100::mbar_wait(st_full, st_used & 1u, abort_flag)) break;
        const float* As = reinterpret_cast<const float*>(smem + lay.st);
        const float* zs = As + 64 * dv;
        for (int e = tid; e < N * 8; e += kWsConvWarps * 32) {
          const int n = e % N, kc = e / N;
          float x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int kk = 8 * kc + k;
            x[k] = n < dv ? As[kk * dv + n] : (n == dv ? zs[kk] : 0.f);
          }
          uint32_t h1[4], h2[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            h1[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
            const float b0 = __uint_as_float(h1[k] << 16), b1 = __uint_as_float(h1[k] & 0xffff0000u);
            h2[k] = pack_bf16x2(x[2 * k] - b0, x[2 * k + 1] - b1);
          }
          uint8_t* y1 = smem + lay.y + swz128(n, kc);
          *reinterpret_cast<uint4*>(y1) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
          *reinterpret_cast<uint4*>(y1 + yblk) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
        }
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(st_empty);
        ++st_used;
        cell = g;
      }
      // this warp's two 8-row groups: all four 32-byte row chunks into registers, then the
      // operand terms over the same bytes; rows past the cell's end become zeros
      uint8_t* st = smem + static_cast<uint32_t>(s) * kWsStage;
      float4 q[4][2];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int grp = warp + 8 * (w >> 1), e = lane + 32 * (w & 1);  // chunk e of the group's 64
        const float4* src = reinterpret_cast<const float4*>(st + grp * kWsGroup + (e >> 3) * 256 + (e & 7) * 32);
        q[w][0] = src[0];
        q[w][1] = src[1];
      }
      __syncwarp();  // every lane has read its chunks before any lane overwrites them
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int grp = warp + 8 * (w >> 1), e = lane + 32 * (w & 1);
        const int rg = e >> 3, ch = e & 7;  // row within the group, 16-byte chunk of the operand row
        const bool on = r0 + 8 * grp + rg < M;
        const float v[8] = {q[w][0].x, q[w][0].y, q[w][0].z, q[w][0].w, q[w][1].x, q[w][1].y, q[w][1].z, q[w][1].w};
        uint32_t h1[4], h2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p0 = on ? phi_pos(v[2 * k]) : 0.f, p1 = on ? phi_pos(v[2 * k + 1]) : 0.f;
          h1[k] = pack_bf16x2(p0, p1);  // both high terms in one rounding, then unpacked exactly
          const float b0 = __uint_as_float(h1[k] << 16), b1 = __uint_as_float(h1[k] & 0xffff0000u);
          h2[k] = pack_bf16x2(p0 - b0, p1 - b1);
        }
        uint8_t* x1 = st + grp * kWsGroup + rg * 128 + ((ch ^ rg) << 4);
        *reinterpret_cast<uint4*>(x1) = make_uint4(h1[0], h1[1], h1[2], h1[3]);
        *reinterpret_cast<uint4*>(x1 + 1024) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
      }
      sm100::fence_async_smem();  // this thread's operand writes, before the MMA (async proxy) reads them
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(xfull0 + 8u * s);
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == kWsStreamWarp && lane == 0) {
    // copies still in flight (the others stopped early) land before the CTA exits
    for (long j = issued > nst ? issued - nst : 0; j < issued; ++j)
      sm100::mbar_wait_drain(full0 + 8u * static_cast<uint32_t>(j % nst), static_cast<uint32_t>(j / nst) & 1u);
    if (st_loads > 0) sm100::mbar_wait_drain(st_full, (st_loads - 1u) & 1u);
  }
  if (warp == kWsMmaWarp) {
    if (lane == 0) {
      sm100::mma_commit(fin);  // every MMA this thread issued has finished
      sm100::mbar_wait_drain(fin, 0u);
      if (*abort_flag && err) atomicOr(err, kErrTimeoutEpilogue);
    }
    __syncwarp();
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, 512);
  }
}

// ring stages that fit next to Y and the state staging, at most kWsMaxStages (5 at d_v = 64,
// 4 at d_v = 128)
constexpr size_t ws_smem(int dv, int nst) { return 1024 + WsLayout(dv, nst).total; }
constexpr int ws_stages(int dv) {
  int n = kWsMaxStages;
  while (n > 1 && ws_smem(dv, n) > 232448) --n;
  return n;
}
constexpr size_t ws_smem_max() {
  size_t m = 0;
  for (int dv = 32; dv <= 128; dv += 32) m = ws_smem(dv, ws_stages(dv)) > m ? ws_smem(dv, ws_stages(dv)) : m;
  return m;
}
static_assert(ws_smem_max() <= 232448, "shared memory budget");
static_assert(ws_stages(128) >= 4 && ws_stages(64) >= 5, "ring depth");

template <typename T>
cudaError_t launch_ws(const MemReadArgs& a, int* err, cudaStream_t st) {
  const int nst = ws_stages(a.dv);
  const size_t smem = ws_smem(a.dv, nst);
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    const void* fn = reinterpret_cast<const void*>(mem_read_ws_kernel<T>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ws_smem_max()));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long tiles = static_cast<long>(a.G) * ((a.M + kRtRows - 1) / kRtRows);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  const cudaError_t e = launch_pdl(mem_read_ws_kernel<T>, dim3(grid), dim3(kWsThreads), smem, st, a, err, nst);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int DK>
constexpr size_t rt_smem(int dv) {
  return 1024 + 2 * RtCfg<DK>::XTILE + ((2 * RtCfg<DK>::KB * static_cast<size_t>(dv + 16) * 128 + 1023) / 1024) * 1024 + 64;
}

template <typename T, int DK>
cudaError_t launch_dk(const MemReadArgs& a, int* err, cudaStream_t st) {
  const size_t smem = rt_smem<DK>(a.dv);
  constexpr size_t smem_max = rt_smem<DK>(128);  // the attribute covers every d_v
  static_assert(smem_max <= 232448, "shared memory budget");
  static bool attr[64] = {false};
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    const void* fn = reinterpret_cast<const void*>(mem_read_tc_kernel<T, DK>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_max));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // as many CTAs per SM as the registers and shared memory allow (two at d_k = 64: two tiles'
    // loads in flight per SM)
    cudaFuncAttributes fa{};
    int smem_sm = 0, regs_sm = 0;
    cudaFuncGetAttributes(&fa, fn);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    const int by_smem = static_cast<int>(smem_sm / (smem_max + 1024));
    const int by_regs = fa.numRegs > 0 ? regs_sm / (fa.numRegs * kRtThreads) : 1;
    per_sm[dev] = std::max(1, std::min(by_smem, by_regs));
    attr[dev] = true;
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long tiles = static_cast<long>(a.G) * ((a.M + kRtRows - 1) / kRtRows);
  const long cap = static_cast<long>(sms) * per_sm[dev];
  const int grid = static_cast<int>(tiles < cap ? tiles : cap);
  const cudaError_t e = launch_pdl(mem_read_tc_kernel<T, DK>, dim3(grid), dim3(kRtThreads), smem, st, a, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool mem_read_tc_supported(int dk, int dv) { return (dk == 64 || dk == 128) && dv % 32 == 0 && dv <= 128; }

cudaError_t launch_mem_read_tc(const MemReadArgs& a, bool f16, int* err, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (!mem_read_tc_supported(a.dk, a.dv)) return cudaErrorInvalidValue;
  if (a.dk == 64) return f16 ? launch_ws<__half>(a, err, st) : launch_ws<__nv_bfloat16>(a, err, st);
  return f16 ? launch_dk<__half, 128>(a, err, st) : launch_dk<__nv_bfloat16, 128>(a, err, st);
}

}  // namespace rmt

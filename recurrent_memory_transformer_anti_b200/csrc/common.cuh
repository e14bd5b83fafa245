// Shared device-side definitions: cell tables, activation-slot addressing, epilogue kinds.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace rmt {

// Device error word values (OR-ed together; read and cleared by rmt_sync).
enum : int {
  kErrTimeoutProducer = 1,
  kErrTimeoutMma = 2,
  kErrTimeoutEpilogue = 4,
  kErrBadArgs = 8,
  kErrTimeoutSelftest = 16,  // the bounded-wait check (rmt_wait_selftest) gave up, as it should
  kErrF16Range = 32,         // a value stored as an f16 tensor-core operand overflowed (see below)
  kErrBounds = 64,           // debug build: a cell's index fell outside the buffers it addresses
};

// f16 operand range. In bf16 mode the tensor-core operands the forward writes (the residual
// stream's operand copy, q/k/v, the SwiGLU output, the memory read-out) are f16, whose largest
// finite value is 65504: a magnitude of 65520 or more rounds to infinity. Each kernel that
// stores such an operand keeps, per thread, the largest magnitude it stored and reports an
// overflow in the error word (kErrF16Range), which rmt_sync turns into RMT_ERANGE.
constexpr float kF16Overflow = 65520.f;

template <typename T>
__device__ __forceinline__ void track_amax(float& m, float v) {
  if constexpr (std::is_same_v<T, __half>) m = fmaxf(m, fabsf(v));
}
template <typename T, int N>
__device__ __forceinline__ void track_amax(float& m, const float (&v)[N]) {
  if constexpr (std::is_same_v<T, __half>) {
#pragma unroll
    for (int j = 0; j < N; ++j) m = fmaxf(m, fabsf(v[j]));
  }
}
// Called by all 32 lanes of a warp: one atomic per warp that stored an overflowing value.
template <typename T>
__device__ __forceinline__ void report_f16_range(float m, int* err) {
  if constexpr (std::is_same_v<T, __half>) {
    if (__any_sync(0xffffffffu, m >= kF16Overflow) && (threadIdx.x & 31) == 0 && err) atomicOr(err, kErrF16Range);
  }
}

// Programmatic dependent launch. The forward launches its kernels with programmatic stream
// serialization, so a kernel may be scheduled while the previous one in the stream is still
// finishing. pdl_wait() blocks until every earlier kernel of the stream has completed and its
// writes are visible: each kernel calls it before its first global-memory access to data
// another kernel writes or reads. pdl_trigger() lets the next kernel be scheduled once every
// CTA of this grid has issued it (or exited); kernels that allocate TMEM issue it only after
// the allocation, so that an early dependent CTA can never hold TMEM this grid still needs.
// Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// One (layer, segment) cell of the grid of one sequence of the batch, with the indices the
// kernels need precomputed on the host:
//   l      layer: selects the weights
//   s      segment of the sequence (recorded by the trace)
//   b      sequence of the batch
//   m      valid rows of the cell: the segment's tokens, then its n_mem memory tokens
//          (M for every segment but a short last one). Rows m..M-1 are padding: they start
//          as zeros, no valid row reads them (attention masks keys >= m; the memory write
//          reads rows m-n_mem..m-1) and they are never emitted.
//   k      per-(sequence, layer) index: memory state A, z and the layer scratch buffers
//   xin    residual slot the cell reads, xout the slot it writes
//   t0     row of the segment's first token in the packed embeddings / outputs
struct Cell {
  int l, s, b, m, k, xin, xout, t0;
#ifdef RMT_DEBUG
  // Debug build (-DRMT_DEBUG, librmt_debug.so): the sizes of the buffers this cell's indices
  // address, and the error word a violation is reported to (null: the identity cells of the
  // kernel-level entry points, whose indices the grid itself bounds). See load_cell.
  int lim_L, lim_state, lim_slot, lim_M, lim_nmem;
  long long lim_tokens;
  int* lim_err;
#endif
};

// Every kernel reads its cells through load_cell. In the debug build it checks each index
// against the limits the host stored in the cell -- layer < L, state and scratch slice <
// sequences x L, residual slots < sequences x (2L + 2), n_mem <= rows <= M, and the segment's
// token rows inside the embeddings -- and on a violation records kErrBounds in the error word
// (rmt_sync then returns RMT_EDEBUG) and hands the kernel a cell whose indices are all in range
// (slot 0, state 0, no token rows), so that no access leaves its buffer. The release build
// compiles to the plain load.
__device__ __forceinline__ Cell load_cell(const Cell* cells, int g) {
  Cell c = cells[g];
#ifdef RMT_DEBUG
  if (c.lim_err) {
    const bool ok = c.l >= 0 && c.l < c.lim_L && c.k >= 0 && c.k < c.lim_state && c.xin >= 0 &&
                    c.xin < c.lim_slot && c.xout >= 0 && c.xout < c.lim_slot && c.m >= c.lim_nmem &&
                    c.m <= c.lim_M && c.t0 >= 0 && static_cast<long long>(c.t0) + (c.m - c.lim_nmem) <= c.lim_tokens;
    if (!ok) {
      atomicOr(c.lim_err, kErrBounds);
      c.l = c.k = c.xin = c.xout = c.t0 = 0;
      c.m = c.lim_nmem;
    }
  }
#endif
  return c;
}

// Activation slots of one sequence, each an [M, d] fp32 residual block; sequence b owns
// slots b*n_slots(L) .. (b+1)*n_slots(L)-1.
//   output slot  : ((l + s) % 2) * L + l            (written by cell (l, s))
//   input slot   : output slot of (l-1, s), or 2L + s % 2 for layer 0 (embeddings + memory)
// Cell (l, s) runs on diagonal l + s; its input was written on diagonal l + s - 1 and is
// next overwritten on diagonal l + s + 1, so two parities suffice for both schedules.
__host__ __device__ inline int out_slot(int L, int l, int s) { return ((l + s) & 1) * L + l; }
__host__ __device__ inline int in_slot(int L, int l, int s) {
  return l == 0 ? 2 * L + (s & 1) : ((l + s - 1) & 1) * L + (l - 1);
}
constexpr int n_slots(int L) { return 2 * L + 2; }

// How a kernel turns a cell into an index of a stacked [*, M, cols] buffer.
enum IndexMode : int { kByLayer = 0, kInSlot = 1, kOutSlot = 2 };

__host__ __device__ inline int cell_index(IndexMode mode, int /*L*/, Cell c) {
  return mode == kByLayer ? c.k : (mode == kInSlot ? c.xin : c.xout);
}

// Rows of the cell that hold tokens (keys past them are masked), given the buffer's M.
__host__ __device__ inline int cell_rows(const Cell& c, int M) { return c.m < M ? c.m : M; }

// Cell g of the kernel-level entry points: group g uses slice g of every stacked operand.
__host__ __device__ inline Cell identity_cell(int g) {
  Cell c{};
  c.l = c.k = c.xin = c.xout = g;
  c.m = 0x7fffffff;
  return c;
}

// GEMM epilogues shared by the tensor-core and the fp32 kernels.
enum EpiKind : int {
  kEpiStoreF32 = 0,   // out(f32) = acc
  kEpiStoreAct = 1,   // out(T) = acc
  kEpiResid = 2,      // x(f32)[dst] = x(f32)[src] + acc
  kEpiResidCast = 3,  // as kEpiResid, and also xb(bf16)[dst] = bf16(result)
  kEpiRope = 4,       // out(T) = RoPE(acc) for columns < rope_cols, acc elsewhere
  kEpiSwiGLU = 5,     // out(T)[:, j] = silu(gate_j) * up_j, gate/up interleaved in blocks of 64
  kEpiMemRead = 6,    // out(T) = phi(acc) A / (phi(acc) . z + eps): the memory read of the query rows
};

constexpr int kSwiGLUBlock = 64;

// Token tile of the CTA-pair GEMM (tokens along the MMA's N): the cell's M rows split into
// ceil(M / 256) near-equal tiles, each rounded up to a multiple of 16 (M = 1040 gives 5 x 208,
// no padding). The pair kernel packs its projections differently from the other GEMMs:
// RoPE partners (i, i + head_dim/2) of each rotated head sit on adjacent weight rows
// (2p, 2p + 1), and gate/up rows alternate (gate_j at 2j, up_j at 2j + 1).
__host__ __device__ inline int pair_token_tile(int M) {
  const int n = (M + 255) / 256;
  const int t = (M + n - 1) / n;
  return (t + 15) / 16 * 16;
}

struct EpiParams {
  void* out;             // kEpiStore*, kEpiRope, kEpiSwiGLU output (stacked [*, M, ldo])
  int ldo;               // output row stride (elements)
  IndexMode out_mode;
  float* x;              // residual stream base ([n_slots, M, ldx] fp32)
  int ldx;
  IndexMode src_mode, dst_mode;
  void* xb;              // operand-type copy of the residual stream ([n_slots, M, ldx]) or null
  const float2* rope;    // [M, head_dim/2] (cos, sin)
  int rope_cols;         // columns (q and k heads) that get RoPE
  int head_dim;
  int rope_tma;          // tensor-core kernel: (cos, sin) come as f16 pairs through the tx map
  // RMSNorm folded into the GEMMs around it. A residual epilogue with ss_out writes, per row,
  // the sum of squares of the new residual over each of its column blocks:
  // ss_out[(layer * M + row) * ss_parts + block]. A RoPE or SwiGLU epilogue with ss_in scales
  // each accumulator row by rsqrt(sum of that row's ss_parts blocks, in block order,
  // * inv_d + rms_eps); the RMSNorm gain is folded into the weight columns at pack time.
  float* ss_out;
  const float* ss_in;
  int ss_parts;
  float inv_d, rms_eps;
  // kEpiMemRead: the accumulator row is the raw memory query q (d_k = the tile width); the
  // epilogue writes o = phi(q) A / (phi(q) . z + mem_eps) (d_v = mem_dv columns) to out,
  // with A [d_k][d_v] and z [d_k] fp32 of state slice cell_index(kByLayer).
  const float* mem_A;
  const float* mem_z;
  int mem_dv;
  float mem_eps;
  // kEpiResidCast on the single-CTA kernel: keep the sum x[src] + acc in registers for the
  // operand copy and the row sums of squares, but do not store it to x[dst] (its consumer
  // adds the same product itself)
  int resid_no_store;
  // Split-operand mode (RMT_BF16_SPLIT): every 16-bit operand this epilogue writes (the
  // residual copy xb, the SwiGLU output, the memory read-out o) also gets its low term, lo_off
  // elements after the high term in the same row (0: high terms only). xb rows are ldxb
  // elements apart (0: ldx). kEpiRope with out_f32 writes q, k and v as fp32 instead.
  int lo_off;
  int ldxb;
  int out_f32;
};

// RMSNorm row scale from the per-block sums of squares of one row (fixed summation order).
__device__ __forceinline__ float rms_row_scale(const float* ss_row, int parts, float inv_d, float eps) {
  float s = 0.f;
  for (int t = 0; t < parts; ++t) s += ss_row[t];
  return rsqrtf(s * inv_d + eps);
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// Two fp32 values rounded to a 16-bit type and packed into one 32-bit word (low half first).
template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) { return pack2<__nv_bfloat16>(a, b); }

// Split-operand mode: v reaches the tensor cores as hi = T(v) and lo = T(v - hi); the pair
// carries about twice the significand bits of T (22 for f16), and one MMA per term with the
// same weight operand accumulates W.hi + W.lo in fp32.
template <typename T> __device__ __forceinline__ float lo_term(float v) { return v - to_f32<T>(from_f32<T>(v)); }

// Store 32 consecutive fp32 values as a 16-bit type (64 bytes, four 16-byte stores).
template <typename T>
__device__ __forceinline__ void store32_16(T* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    d[q] = make_uint4(pack2<T>(v[8 * q + 0], v[8 * q + 1]), pack2<T>(v[8 * q + 2], v[8 * q + 3]),
                      pack2<T>(v[8 * q + 4], v[8 * q + 5]), pack2<T>(v[8 * q + 6], v[8 * q + 7]));
  }
}
__device__ __forceinline__ void store32_bf16(__nv_bfloat16* dst, const float* v) { store32_16(dst, v); }

// store32_16, plus (lo_off != 0) the 32 low terms at dst + lo_off.
template <typename T>
__device__ __forceinline__ void store32_16_split(T* dst, const float* v, int lo_off) {
  store32_16(dst, v);
  if (lo_off) {
    float l[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) l[j] = lo_term<T>(v[j]);
    store32_16(dst + lo_off, l);
  }
}

// Tensor-core operand format code of the instruction descriptor (kind::f16): f16 0, bf16 1.
template <typename T> struct OpFormat;
template <> struct OpFormat<__half> { static constexpr uint32_t value = 0; };
template <> struct OpFormat<__nv_bfloat16> { static constexpr uint32_t value = 1; };

// phi(x) = elu(x) + 1
__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : expf(x); }

// silu(x) = x * sigmoid(x)
__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

}  // namespace rmt

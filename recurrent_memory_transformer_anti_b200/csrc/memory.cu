// Associative memory of an ARMT layer (the model the diagonal-batching paper accelerates;
// arXiv 2506.05229 applies it to a LLaMA-1B ARMT). The pages cite ARMT by name only; the
// kernels implement phi(x) = elu(x) + 1 and
//   read   : o = phi(q) A / (phi(q) . z + eps)                     per row
//   update : v_bar = phi(K) A / (phi(K) . z + eps)
//            A += phi(K)^T (V - v_bar),  z += sum over rows of phi(K)   (pre-update A, z)
// with A (d_k x d_v) and z (d_k) in fp32. Every reduction runs in a fixed order, so a cell
// gives the same bits whichever other cells share its launch.
#include "common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace rmt {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------- mma.sync helpers
__device__ __forceinline__ uint32_t pack_bf16_bits(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// Three-term bf16 split of two fp32 values (columns k, k + 1), packed as A-fragment registers.
__device__ __forceinline__ void split3(float2 v, uint32_t& t1, uint32_t& t2, uint32_t& t3) {
  const __nv_bfloat16 a1 = __float2bfloat16_rn(v.x), b1 = __float2bfloat16_rn(v.y);
  const float ra = v.x - __bfloat162float(a1), rb = v.y - __bfloat162float(b1);
  const __nv_bfloat16 a2 = __float2bfloat16_rn(ra), b2 = __float2bfloat16_rn(rb);
  const __nv_bfloat16 a3 = __float2bfloat16_rn(ra - __bfloat162float(a2));
  const __nv_bfloat16 b3 = __float2bfloat16_rn(rb - __bfloat162float(b2));
  t1 = pack_bf16_bits(a1, b1);
  t2 = pack_bf16_bits(a2, b2);
  t3 = pack_bf16_bits(a3, b3);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// ----------------------------------------------------------------------------- read
// CTA = 32 rows of one cell, 8 warps x 4 rows, all 4 rows of a warp in flight together.
// A and z sit in shared memory; lane j owns output columns j, j+32, ...; q_i reaches all
// lanes by shuffle. Small CTAs keep many warps resident: the work per row is a chain of
// shuffles and FMAs, so latency, not bandwidth, sets the pace.
constexpr int kReadRows = 32, kReadWarps = 8, kReadBatch = 4;

template <typename T>
__global__ void __launch_bounds__(kReadWarps * 32) mem_read_kernel(const MemReadArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ float sm[];
  const int dk = a.dk, dv = a.dv, nk = dk >> 5, nv = dv >> 5;
  float* As = sm;            // [dk][dv]
  float* zs = sm + dk * dv;  // [dk]
  const Cell c = load_cell(a.cells, blockIdx.y);
  const size_t si = cell_index(a.state_mode, a.L, c), qi = cell_index(a.mode, a.L, c);
  const float4* A4 = reinterpret_cast<const float4*>(a.A + si * dk * dv);
  for (int i = threadIdx.x; i < (dk * dv) >> 2; i += blockDim.x) reinterpret_cast<float4*>(As)[i] = A4[i];
  for (int i = threadIdx.x; i < dk; i += blockDim.x) zs[i] = a.z[si * dk + i];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* q = a.q + qi * a.M * dk;
  T* o = static_cast<T*>(a.o) + qi * a.M * dv;
  const int r_begin = blockIdx.x * kReadRows + warp * (kReadRows / kReadWarps);
  const int r_end = min(r_begin + kReadRows / kReadWarps, a.M);
  for (int r0 = r_begin; r0 < r_end; r0 += kReadBatch) {
    float fq[kReadBatch][4], acc[kReadBatch][4], den[kReadBatch];
#pragma unroll
    for (int b = 0; b < kReadBatch; ++b) {
      const int row = r0 + b;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        fq[b][u] = (u < nk && row < r_end) ? phi_f(q[static_cast<size_t>(row) * dk + 32 * u + lane]) : 0.f;
        acc[b][u] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < kReadBatch; ++b) {
      float d = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (u < nk) d = fmaf(fq[b][u], zs[32 * u + lane], d);
      den[b] = warp_sum(d) + a.eps;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u >= nk) break;
      for (int j = 0; j < 32; ++j) {
        const float* Ai = As + (32 * u + j) * dv;
        float qb[kReadBatch];
#pragma unroll
        for (int b = 0; b < kReadBatch; ++b) qb[b] = __shfl_sync(0xffffffffu, fq[b][u], j);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          if (v < nv) {
            const float av = Ai[32 * v + lane];
#pragma unroll
            for (int b = 0; b < kReadBatch; ++b) acc[b][v] = fmaf(qb[b], av, acc[b][v]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kReadBatch; ++b) {
      const int row = r0 + b;
      if (row >= r_end) break;
      const float inv = 1.f / den[b];
#pragma unroll
      for (int v = 0; v < 4; ++v)
        if (v < nv) o[static_cast<size_t>(row) * dv + 32 * v + lane] = from_f32<T>(acc[b][v] * inv);
    }
  }
}

// Tensor-core read for 16-bit outputs (mma.sync m16n8k16, fp32 accumulation). The read is
// a product of the query rows with [A | z] (d_k x (d_v + 1)): per 16-row tile, the numerators
// are columns 0..d_v-1 and the denominator phi(q) . z is column d_v of the same accumulation,
// so no reduction across lanes is needed. phi(q) and [A | z] are fp32; each is split into two
// bf16 terms (x = x1 + x2, x1 = bf16(x), x2 = bf16(x - x1)) and the products x1 y1, x1 y2,
// x2 y1 go into the fp32 accumulator in that order, k-steps ascending: the dropped terms are
// about 2^-16 of the result, well under the 16-bit output's rounding. [A | z] is split and
// transposed into shared memory once per CTA (columns as rows, as ldmatrix wants them). Each
// warp then streams 16-row tiles of its rows through a kReadStages-deep ring of shared-memory
// stages filled with cp.async (16-byte chunks into padded rows, so that the fragment loads hit
// every bank once), keeping two tiles' loads in flight while it multiplies the third, and
// stages its output tile in shared memory for 16-byte row stores. A CTA takes a block of rows
// of one cell, sized so that a launch has at least two CTAs per SM.
constexpr int kReadMmaWarps = 4;
constexpr int kReadStages = 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename T, int DK>
__global__ void __launch_bounds__(kReadMmaWarps * 32) mem_read_mma_kernel(const MemReadArgs a, int rows_per_cta) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ __align__(16) unsigned char rd_sm[];
  constexpr int QS = DK + 8;          // fp32 row stride of a staged query tile (32 B of padding)
  constexpr int NKS = DK / 16;        // 16-column k-steps
  constexpr int BS = DK + 8;          // bf16 row stride of the transposed [A | z]
  const int dv = a.dv, M = a.M;
  const int nb = dv + 8;              // rows of the transposed [A | z]: d_v columns of A, z, 7 zero rows
  const int ostride = dv + 8;         // 16-bit row stride of a warp's output staging tile
  float* Qs = reinterpret_cast<float*>(rd_sm);                                   // [warps][stages][16][QS]
  __nv_bfloat16* B1 = reinterpret_cast<__nv_bfloat16*>(Qs + kReadMmaWarps * kReadStages * 16 * QS);
  __nv_bfloat16* B2 = B1 + nb * BS;
  T* Os = reinterpret_cast<T*>(B2 + nb * BS);
  const Cell c = load_cell(a.cells, blockIdx.y);
  const size_t si = cell_index(a.state_mode, a.L, c), qi = cell_index(a.mode, a.L, c);
  const float* A = a.A + si * DK * dv;
  const float* z = a.z + si * DK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const float* q = a.q + qi * static_cast<size_t>(M) * DK;
  T* o = static_cast<T*>(a.o) + qi * static_cast<size_t>(M) * dv;
  const int r_beg = blockIdx.x * rows_per_cta, r_end = min(M, r_beg + rows_per_cta);
  // this warp's tiles: rows r_beg + 16 (warp + kReadMmaWarps i)
  const int ntile = (r_end - r_beg + 15) / 16;
  const int mine = ntile > warp ? (ntile - warp + kReadMmaWarps - 1) / kReadMmaWarps : 0;
  float* qs_w = Qs + warp * kReadStages * 16 * QS;
  auto issue = [&](int i) {  // cp.async of this warp's i-th tile into stage i % kReadStages
    const int r0 = r_beg + 16 * (warp + kReadMmaWarps * i);
    float* dst = qs_w + (i % kReadStages) * 16 * QS;
#pragma unroll
    for (int u = 0; u < (16 * DK / 4) / 32; ++u) {
      const int e = lane + 32 * u, rr = e / (DK / 4), ch = e % (DK / 4);
      const int row = r0 + rr;
      const bool in = row < r_end;
      cp_async16(sm100::smem_u32(dst + rr * QS + 4 * ch), q + static_cast<size_t>(in ? row : r_beg) * DK + 4 * ch,
                 in ? 16u : 0u);
    }
  };
#pragma unroll
  for (int i = 0; i < kReadStages - 1; ++i) {
    if (i < mine) issue(i);
    cp_async_commit();
  }
  // [A | z], split and transposed, with its loads batched
  for (int e0 = tid; e0 < nb * DK; e0 += 8 * kReadMmaWarps * 32) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * kReadMmaWarps * 32;
      const int j = e % nb, i = e / nb;
      x[u] = (e >= nb * DK) ? 0.f : (j < dv ? A[static_cast<size_t>(i) * dv + j] : (j == dv ? z[i] : 0.f));
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * kReadMmaWarps * 32;
      if (e >= nb * DK) break;
      const int j = e % nb, i = e / nb;
      const __nv_bfloat16 x1 = __float2bfloat16_rn(x[u]);
      B1[j * BS + i] = x1;
      B2[j * BS + i] = __float2bfloat16_rn(x[u] - __bfloat162float(x1));
    }
  }
  __syncthreads();

  const int ntn = dv / 8 + 1;  // 8-column tiles (the last holds z)
  T* os = Os + warp * 16 * ostride;
  const int lr = lane & 7, lm = lane >> 3;  // ldmatrix: lane's row, and its matrix (hi k0-7, hi k8-15, lo k0-7, lo k8-15)
  const uint32_t bsel = sm100::smem_u32((lm < 2 ? B1 : B2) + lr * BS + (lm & 1) * 8);
  for (int i = 0; i < mine; ++i) {
    if (i + kReadStages - 1 < mine) issue(i + kReadStages - 1);
    cp_async_commit();
    cp_async_wait<kReadStages - 1>();  // tile i has landed (this lane's chunks)
    __syncwarp();                      // ... and every lane's
    const float* qt = qs_w + (i % kReadStages) * 16 * QS + 2 * tq;
    float acc[17][4];
#pragma unroll
    for (int t = 0; t < 17; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < NKS; ++ks) {
      float2 v[4];
      v[0] = *reinterpret_cast<const float2*>(qt + gq * QS + 16 * ks);
      v[1] = *reinterpret_cast<const float2*>(qt + (gq + 8) * QS + 16 * ks);
      v[2] = *reinterpret_cast<const float2*>(qt + gq * QS + 16 * ks + 8);
      v[3] = *reinterpret_cast<const float2*>(qt + (gq + 8) * QS + 16 * ks + 8);
      uint32_t f1[4], f2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x = phi_f(v[u].x), y = phi_f(v[u].y);
        const __nv_bfloat16 x1 = __float2bfloat16_rn(x), y1 = __float2bfloat16_rn(y);
        f1[u] = pack_bf16_bits(x1, y1);
        f2[u] = pack_bf16_bits(__float2bfloat16_rn(x - __bfloat162float(x1)), __float2bfloat16_rn(y - __bfloat162float(y1)));
      }
#pragma unroll
      for (int t = 0; t < 17; ++t) {
        if (t < ntn) {
          uint32_t b[4];
          ldmatrix_x4(bsel + 2u * (t * 8 * BS + 16 * ks), b);
          mma_bf16_16816(acc[t], f1, b[0], b[1]);
          mma_bf16_16816(acc[t], f1, b[2], b[3]);
          mma_bf16_16816(acc[t], f2, b[0], b[1]);
        }
      }
    }
    __syncwarp();  // every lane has read its fragments of the stage before it is refilled
    // denominators: column d_v (z) sits in tile ntn-1, column 0, i.e. with lane 4 gq (tq = 0)
    float den_a = 0.f, den_b = 0.f;
#pragma unroll
    for (int t = 0; t < 17; ++t) {
      if (t == ntn - 1) {
        den_a = acc[t][0];
        den_b = acc[t][2];
      }
    }
    den_a = __shfl_sync(0xffffffffu, den_a, lane & ~3) + a.eps;
    den_b = __shfl_sync(0xffffffffu, den_b, lane & ~3) + a.eps;
    const float ia = 1.f / den_a, ib = 1.f / den_b;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if (t < ntn - 1) {
        *reinterpret_cast<uint32_t*>(os + gq * ostride + 8 * t + 2 * tq) = pack2<T>(acc[t][0] * ia, acc[t][1] * ia);
        *reinterpret_cast<uint32_t*>(os + (gq + 8) * ostride + 8 * t + 2 * tq) = pack2<T>(acc[t][2] * ib, acc[t][3] * ib);
      }
    }
    __syncwarp();
    const int r0 = r_beg + 16 * (warp + kReadMmaWarps * i);
    const int chunks = dv / 8;  // 16-byte chunks per output row
    for (int e = lane; e < 16 * chunks; e += 32) {
      const int rr = e / chunks, ch = e % chunks;
      if (r0 + rr < r_end)
        *reinterpret_cast<uint4*>(o + static_cast<size_t>(r0 + rr) * dv + 8 * ch) =
            *reinterpret_cast<const uint4*>(os + rr * ostride + 8 * ch);
    }
    __syncwarp();  // the staging tile has been read before the next tile overwrites it
  }
  cp_async_wait<0>();
}

// ------------------------------------------------------------------ key/value projection
// CTA = one split of kMemKvSplit columns of d_model for one cell and one block of up to
// kKvCols output columns: the n memory rows and those weight rows of the split are staged in
// shared memory, k-major; each thread then forms a 4-row x 2-column block of the partial dot
// products over the split, k ascending.
// Staging reads 16-byte vectors: one lane takes 8 consecutive columns of one weight row (4 of
// one memory row) and writes them down a column of the k-major block, so the lanes of a warp
// write consecutive words.
constexpr int kKvThreads = 256;
constexpr int kKvCols = 128;  // output columns per CTA (blockIdx.z selects the block of dkv)

template <typename T>
__global__ void __launch_bounds__(kKvThreads) mem_kv_kernel(const MemKvArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ float sm[];
  constexpr int KS = kMemKvSplit;
  const int n4 = (a.n + 3) & ~3;  // rows padded to a multiple of 4 (padding rows are zero)
  const int j_base = blockIdx.z * kKvCols, cols = min(kKvCols, a.dkv - j_base);
  float* Ys = sm;                 // [KS][n4]
  float* Ws = sm + KS * n4;       // [KS][cols]: weight rows j_base .. j_base + cols - 1
  const Cell c = load_cell(a.cells, blockIdx.y);
  const int split = blockIdx.x, k0 = split * KS;
  const int kw = min(KS, a.d - k0);
  // the cell's memory rows are its last n valid rows
  const int row0 = cell_rows(c, a.M) - a.n;
  const float* Y = a.x + (static_cast<size_t>(cell_index(a.x_mode, a.L, c)) * a.M + row0) * a.d + k0;
  const T* W = static_cast<const T*>(a.w) + (static_cast<size_t>(c.l) * a.dkv + j_base) * a.d + k0;
  // 16-byte vectors only where every row start is 16-byte aligned
  const bool y_vec = (a.d % 4 == 0) && (reinterpret_cast<uintptr_t>(a.x) % 16 == 0);
  const bool w_vec = sizeof(T) == 2 && (a.d % 8 == 0) && (reinterpret_cast<uintptr_t>(a.w) % 16 == 0);
  // memory rows: one lane per (row, 4 columns), rows fastest
  for (int e = threadIdx.x; e < n4 * (KS / 4); e += kKvThreads) {
    const int r = e % n4, k = 4 * (e / n4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < a.n) {
      const float* yr = Y + static_cast<size_t>(r) * a.d + k;
      if (y_vec && k + 3 < kw) {
        v = *reinterpret_cast<const float4*>(yr);
      } else {
        if (k < kw) v.x = yr[0];
        if (k + 1 < kw) v.y = yr[1];
        if (k + 2 < kw) v.z = yr[2];
        if (k + 3 < kw) v.w = yr[3];
      }
    }
    Ys[(k + 0) * n4 + r] = v.x;
    Ys[(k + 1) * n4 + r] = v.y;
    Ys[(k + 2) * n4 + r] = v.z;
    Ys[(k + 3) * n4 + r] = v.w;
  }
  // weight rows: one lane per (row, 8 columns), rows fastest
  for (int e = threadIdx.x; e < cols * (KS / 8); e += kKvThreads) {
    const int j = e % cols, k = 8 * (e / cols);
    float w8[8];
    if (w_vec && k + 7 < kw) {
      const uint4 u = *reinterpret_cast<const uint4*>(W + static_cast<size_t>(j) * a.d + k);
      const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int t = 0; t < 8; ++t) w8[t] = to_f32<T>(h[t]);
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) w8[t] = k + t < kw ? to_f32<T>(W[static_cast<size_t>(j) * a.d + k + t]) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) Ws[(k + t) * cols + j] = w8[t];
  }
  __syncthreads();
  const int nsplit = (a.d + KS - 1) / KS;
  const int nout = a.n * a.dkv;
  float* part = a.part + (static_cast<size_t>(c.k) * nsplit + split) * nout;
  const int jt = cols / 2, tiles = (n4 / 4) * jt;
  for (int t = threadIdx.x; t < tiles; t += kKvThreads) {
    const int r0 = (t / jt) * 4, j0 = (t % jt) * 2;
    float acc[4][2] = {};
#pragma unroll 8
    for (int k = 0; k < KS; ++k) {
      const float4 y = *reinterpret_cast<const float4*>(Ys + k * n4 + r0);
      const float2 w = *reinterpret_cast<const float2*>(Ws + k * cols + j0);
      const float yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[i][0] = fmaf(yv[i], w.x, acc[i][0]);
        acc[i][1] = fmaf(yv[i], w.y, acc[i][1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (r0 + i < a.n)
        *reinterpret_cast<float2*>(part + (r0 + i) * a.dkv + j_base + j0) = make_float2(acc[i][0], acc[i][1]);
  }
}

// Tensor-core variant for bf16 weights (mma.sync m16n8k16 with fp32 accumulation): the same
// partials, from one CTA per (split, cell, block of output columns). The memory rows are fp32,
// so each value is split into three bf16 terms y = y1 + y2 + y3 (y1 = bf16(y), y2 = bf16(y - y1),
// y3 = bf16(y - y1 - y2)), which carry all of its 24 significand bits; the weights are exact in
// bf16, so the three products per 16-column step go into one fp32 accumulator, terms in that
// order, steps ascending. The rows and the weight rows of the split are staged with cp.async
// (all of a CTA's 16-byte chunks in flight at once); the CTA then splits the rows once into
// three bf16 planes, and every warp reads its A fragments from them and its B fragments from
// the weights with ldmatrix (the warps share the rows: splitting while forming the fragments
// would repeat the conversion in every warp). Warp w computes the 8-column output tiles w and
// w + 8 of every 16-row tile.
// WHOLE: one CTA per (cell, block of output columns) runs the splits one after another, forms
// each split's partial exactly as above and adds it to a running sum in split order -- the sum
// the update forms from the partials, bit for bit -- and writes that sum alone (one "split").
// Three such CTAs per SM interleave their loads and products (a ring of four stages in one CTA
// per SM measured slower). For launches of many cells, where the partials' round trip through
// memory would cost more than the splits' parallelism gains.
constexpr int kKvMmaThreads = 256;
constexpr int kKvWholeStages = 1;  // 57 KB at n <= 16: three CTAs per SM
constexpr int kKvYStride = kMemKvSplit + 8;  // fp32 row stride of the staged rows
constexpr int kKvWStride = kMemKvSplit + 8;  // bf16 row stride of the staged weights (272 B: ldmatrix rows on distinct banks)
constexpr int kKvPStride = kMemKvSplit + 8;  // bf16 row stride of the split planes (same reason)

// Shared memory of the tensor-core k/v kernel: `stages` x (fp32 rows, weight rows), then three
// split planes.
inline size_t kv_mma_smem(int n, int cols, int stages = 1) {
  const size_t n16 = (n + 15) & ~15, wrows = (cols + 7) / 8 * 8;
  return stages * (sizeof(float) * n16 * kKvYStride + 2 * wrows * kKvWStride) + 3 * 2 * n16 * kKvPStride;
}

template <bool WHOLE>
__global__ void __launch_bounds__(kKvMmaThreads, WHOLE ? 3 : 1) mem_kv_mma_kernel(const MemKvArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ __align__(16) unsigned char kv_sm[];
  constexpr int KS = kMemKvSplit;
  constexpr int NB = WHOLE ? kKvWholeStages : 1;  // stages of rows and weights
  const int n16 = (a.n + 15) & ~15;
  const int j_base = blockIdx.z * kKvCols, cols = min(kKvCols, a.dkv - j_base);
  const int ntiles = (cols + 7) / 8;
  const size_t ybytes = sizeof(float) * n16 * kKvYStride, wbytes = 2 * 8 * ntiles * kKvWStride;
  auto Ys_of = [&](int b) { return reinterpret_cast<float*>(kv_sm + b * (ybytes + wbytes)); };  // [n16][kKvYStride]
  auto Ws_of = [&](int b) {  // [8*ntiles][kKvWStride]
    return reinterpret_cast<__nv_bfloat16*>(kv_sm + b * (ybytes + wbytes) + ybytes);
  };
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(kv_sm + NB * (ybytes + wbytes));  // [3][n16][kKvPStride]
  const Cell c = load_cell(a.cells, blockIdx.y);
  const int nsplit = (a.d + KS - 1) / KS;
  const int row0 = cell_rows(c, a.M) - a.n;  // the cell's memory rows are its last n valid rows
  const float* Yc = a.x + (static_cast<size_t>(cell_index(a.x_mode, a.L, c)) * a.M + row0) * a.d;
  const __nv_bfloat16* Wc = static_cast<const __nv_bfloat16*>(a.w) + (static_cast<size_t>(c.l) * a.dkv + j_base) * a.d;
  const bool y_vec = (a.d % 4 == 0) && (reinterpret_cast<uintptr_t>(a.x) % 16 == 0);
  const bool w_vec = (a.d % 8 == 0) && (reinterpret_cast<uintptr_t>(a.w) % 16 == 0);
  const int tid = threadIdx.x;
  // rows (zero past n and past the split's columns) and the weight rows of this column block
  // (zero past cols and past the split's columns) of one split into stage b: whole 16-byte chunks
  // by cp.async; chunks at a ragged edge, or of unaligned rows, element by element
  auto issue = [&](int split, int b) {
    const int k0 = split * KS, kw = min(KS, a.d - k0);
    const float* Y = Yc + k0;
    const __nv_bfloat16* W = Wc + k0;
    float* Ys = Ys_of(b);
    __nv_bfloat16* Ws = Ws_of(b);
    for (int e = tid; e < n16 * (KS / 4); e += kKvMmaThreads) {
      const int r = e / (KS / 4), k = 4 * (e % (KS / 4));
      float* dst = Ys + r * kKvYStride + k;
      const float* yr = Y + static_cast<size_t>(r < a.n ? r : 0) * a.d + k;
      if (y_vec && (r >= a.n || k + 3 < kw)) {
        cp_async16(sm100::smem_u32(dst), r < a.n ? yr : Y, r < a.n ? 16u : 0u);
      } else {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < a.n) {
          if (k < kw) v.x = yr[0];
          if (k + 1 < kw) v.y = yr[1];
          if (k + 2 < kw) v.z = yr[2];
          if (k + 3 < kw) v.w = yr[3];
        }
        *reinterpret_cast<float4*>(dst) = v;
      }
    }
    for (int e = tid; e < 8 * ntiles * (KS / 8); e += kKvMmaThreads) {
      const int j = e / (KS / 8), k = 8 * (e % (KS / 8));
      __nv_bfloat16* dst = Ws + j * kKvWStride + k;
      const __nv_bfloat16* wr = W + static_cast<size_t>(j < cols ? j : 0) * a.d + k;
      if (w_vec && (j >= cols || k + 7 < kw)) {
        cp_async16(sm100::smem_u32(dst), j < cols ? wr : W, j < cols ? 16u : 0u);
      } else {
        uint32_t h[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) h[t] = (j < cols && k + t < kw) ? __bfloat16_as_ushort(wr[t]) : 0u;
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      }
    }
  };
  // the rows of stage b -> their three bf16 terms, two columns per step
  auto split_rows = [&](int b) {
    const float* Ys = Ys_of(b);
    for (int e = tid; e < n16 * (KS / 2); e += kKvMmaThreads) {
      const int r = e / (KS / 2), k = 2 * (e % (KS / 2));
      uint32_t t1, t2, t3;
      split3(*reinterpret_cast<const float2*>(Ys + r * kKvYStride + k), t1, t2, t3);
      uint32_t* p = reinterpret_cast<uint32_t*>(Ps + r * kKvPStride + k);
      p[0] = t1;
      p[n16 * kKvPStride / 2] = t2;
      p[n16 * kKvPStride] = t3;
    }
  };
  const int warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int nt0 = warp, nt1 = warp + 8;  // this warp's output tiles (kKvCols = 128: at most 16)
  const bool has0 = nt0 < ntiles, has1 = nt1 < ntiles;
  // ldmatrix row addresses: lanes 0-7 give the rows of the k 0..7 matrix, lanes 8-15 of k 8..15
  const int lr = lane & 7, lk = ((lane >> 3) & 1) * 8;
  // ldmatrix x4 row addresses of a 16 x 16 A tile: lanes 0-15 rows 0-15 at k 0, lanes 16-31 at k 8
  const uint32_t plane = 2u * n16 * kKvPStride;  // bytes
  const uint32_t pa0 =
      sm100::smem_u32(Ps + ((lane & 7) + ((lane >> 3) & 1) * 8) * kKvPStride + (lane >> 4) * 8);
  // the partial of 16-row tile mt over the split in stage b: acc0 (tile nt0), acc1 (tile nt1)
  auto partial = [&](int b, int mt, float (&acc0)[4], float (&acc1)[4]) {
    const __nv_bfloat16* Ws = Ws_of(b);
    const uint32_t wb0 = sm100::smem_u32(Ws + (nt0 * 8 + lr) * kKvWStride + lk);
    const uint32_t wb1 = has1 ? sm100::smem_u32(Ws + (nt1 * 8 + lr) * kKvWStride + lk) : wb0;
#pragma unroll
    for (int q = 0; q < 4; ++q) acc0[q] = acc1[q] = 0.f;
    const uint32_t pa = pa0 + 2u * 16 * kKvPStride * mt;
#pragma unroll 2
    for (int ks = 0; ks < KS / 16; ++ks) {
      uint32_t t1[4], t2[4], t3[4];
      ldmatrix_x4(pa + 32u * ks, t1);
      ldmatrix_x4(pa + plane + 32u * ks, t2);
      ldmatrix_x4(pa + 2 * plane + 32u * ks, t3);
      uint32_t b0, b1;
      ldmatrix_x2(wb0 + 32u * ks, b0, b1);
      mma_bf16_16816(acc0, t1, b0, b1);
      mma_bf16_16816(acc0, t2, b0, b1);
      mma_bf16_16816(acc0, t3, b0, b1);
      if (has1) {
        ldmatrix_x2(wb1 + 32u * ks, b0, b1);
        mma_bf16_16816(acc1, t1, b0, b1);
        mma_bf16_16816(acc1, t2, b0, b1);
        mma_bf16_16816(acc1, t3, b0, b1);
      }
    }
  };
  auto store = [&](float* part, const float (&acc)[4], int mt, int nt) {
    const int r = mt * 16 + gq, col = nt * 8 + 2 * tq;
    if (col >= cols) return;
    if (r < a.n) *reinterpret_cast<float2*>(part + r * a.dkv + j_base + col) = make_float2(acc[0], acc[1]);
    if (r + 8 < a.n) *reinterpret_cast<float2*>(part + (r + 8) * a.dkv + j_base + col) = make_float2(acc[2], acc[3]);
  };

  if constexpr (!WHOLE) {
    const int split = blockIdx.x;
    issue(split, 0);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    split_rows(0);
    __syncthreads();
    float* part = a.part + (static_cast<size_t>(c.k) * nsplit + split) * a.n * a.dkv;
    if (!has0) return;
    for (int mt = 0; mt < n16 / 16; ++mt) {
      float acc0[4], acc1[4];
      partial(0, mt, acc0, acc1);
      store(part, acc0, mt, nt0);
      if (has1) store(part, acc1, mt, nt1);
    }
  } else {
    float s0[4][4], s1[4][4];  // running sums of row tiles mt < 4 (n <= 64; this route takes n <= 16)
#pragma unroll
    for (int j = 0; j < NB - 1; ++j) {
      if (j < nsplit) issue(j, j);
      cp_async_commit();
    }
    for (int sp = 0; sp < nsplit; ++sp) {
      const int b = sp % NB;
      // the stage of split sp - 1, freed by the barrier that closed it, takes split sp + NB - 1
      if (sp + NB - 1 < nsplit) issue(sp + NB - 1, (sp + NB - 1) % NB);
      cp_async_commit();
      cp_async_wait<NB - 1>();  // this split's stage has landed
      __syncthreads();
      split_rows(b);
      __syncthreads();
      if (has0) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          if (mt < n16 / 16) {
            float acc0[4], acc1[4];
            partial(b, mt, acc0, acc1);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              s0[mt][q] = sp == 0 ? acc0[q] : s0[mt][q] + acc0[q];
              s1[mt][q] = sp == 0 ? acc1[q] : s1[mt][q] + acc1[q];
            }
          }
        }
      }
      __syncthreads();  // the planes and stage b are free
    }
    cp_async_wait<0>();
    float* part = a.part + static_cast<size_t>(c.k) * a.n * a.dkv;
    if (has0) {
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        if (mt < n16 / 16) {
          store(part, s0[mt], mt, nt0);
          if (has1) store(part, s1[mt], mt, nt1);
        }
      }
    }
  }
}

// --------------------------------------------------------------------------- update
// The delta rule separates by value column: column j of A' needs column j of A and of V, and,
// through the row denominators, all of phi(K) and z. A cell's update therefore runs on a
// cluster of S CTAs, CTA `slice` owning columns slice*CS .. slice*CS+CS-1 (CS = d_v / S):
//   1. each CTA reduces its own share of the key rows (sum of the split partials in split
//      order, then phi) and its own value columns into shared memory; the cluster meets, and
//      each CTA copies the other key rows from its peers' shared memory;
//   2. den[r] = phi(k_r) . z + eps, one warp per row (lanes over i, then a butterfly);
//   3. v_bar and D = V - v_bar for the slice's columns over i ascending (one row x 4 columns
//      per thread);
//   4. A' = A + phi(K)^T D for the slice's columns, 4 x 4 blocks over rows ascending; the CTA of
//      slice 0 also writes z' = z + sum of the phi(k) rows.
// Every sum runs in a fixed order whatever S is, so the bits do not depend on the slicing or on
// the cells sharing the launch. S is picked per launch: more slices when the launch holds few
// cells (a diagonal), whole cells when it holds many.
constexpr int kUpdThreads = 256;

struct UpdLayout {  // shared-memory layout in floats (every region starts 16-byte aligned)
  int n4, fk, As, Vs, D, zs, den, gram, total;
  __host__ __device__ UpdLayout(int n, int dk, int cs) {
    n4 = (n + 3) & ~3;
    fk = 0;                 // [n][dk]    phi(keys)
    As = fk + n * dk;       // [dk][cs]   this slice's columns of A
    Vs = As + dk * cs;      // [n][cs]    this slice's columns of V
    D = Vs + n * cs;        // [n4][cs]   V - v_bar
    zs = D + n4 * cs;       // [dk]
    den = zs + dk;          // [n4]
    gram = den + n4;        // [n][n4]    per-token rule: phi(k_r) . phi(k_j), j < r
    total = gram + n * n4;
  }
};

// Per-token delta rule (rows written one after another) from the batched quantities. Row r
// meets the state A_r = A + sum_{j<r} phi(k_j)^T d_j, z_r = z + sum_{j<r} phi(k_j), so with
// G_rj = phi(k_r) . phi(k_j):
//   den_r = phi(k_r) . z + eps + sum_{j<r} G_rj
//   d_r   = V_r - phi(k_r) A / den_r - sum_{j<r} G_rj d_j / den_r
// and after the last row A' = A + phi(K)^T D, z' = z + sum_r phi(k_r), as in the batched rule.
// seq_gram_den: G (lower triangle; one warp per row, lanes over i, then a butterfly) and the
// denominators (den holds phi(k_r) . z + eps on entry; j ascending). seq_substitute: D holds
// V_r - phi(k_r) A / den_r on entry and d_r on exit, rows ascending, one thread per column.
// Both run the same order in every kernel.
__device__ __forceinline__ void seq_gram_den(const float* fk, int n, int dk, int ldg, float* gram, float* den,
                                             int tid, int nthreads) {
  // one warp per row r: lanes over i (ascending within a lane), then the butterfly, per j < r
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = 1 + warp; r < n; r += nthreads >> 5) {
    for (int j = 0; j < r; ++j) {
      float s = 0.f;
      for (int i = lane; i < dk; i += 32) s = fmaf(fk[r * dk + i], fk[j * dk + i], s);
      s = warp_sum(s);
      if (lane == 0) gram[r * ldg + j] = s;
    }
  }
  __syncthreads();
  for (int r = tid; r < n; r += nthreads) {
    float d = den[r];
    for (int j = 0; j < r; ++j) d += gram[r * ldg + j];
    den[r] = d;
  }
  __syncthreads();
}

__device__ __forceinline__ void seq_substitute(float* D, int ldd, int cols, int n, const float* gram, int ldg,
                                               const float* den, int tid, int nthreads) {
  for (int c = tid; c < cols; c += nthreads) {
    for (int r = 1; r < n; ++r) {
      float acc = 0.f;
      for (int j = 0; j < r; ++j) acc = fmaf(gram[r * ldg + j], D[j * ldd + c], acc);
      D[r * ldd + c] -= acc / den[r];
    }
  }
}

// Raw key|value elements (r, col) of the cell, as the sum of the split partials in split order,
// starting from the first (or the plain inputs without partials). EPT elements per call; their partial loads go out
// in batches of kUpdBatch splits x EPT elements before any of them is added.
constexpr int kUpdBatch = 8;
template <int EPT>
__device__ __forceinline__ void kv_values(const MemUpdateArgs& a, size_t ki, const int (&r)[EPT],
                                          const int (&col)[EPT], const bool (&on)[EPT], float (&val)[EPT]) {
  const int dk = a.dk, dkv = a.dk + a.dv;
  if (a.part) {
    const float* p = a.part + ki * a.nsplit * a.n * dkv;
    const size_t stride = static_cast<size_t>(a.n) * dkv;
    for (int sp0 = 0; sp0 < a.nsplit; sp0 += kUpdBatch) {
      float x[kUpdBatch][EPT];
#pragma unroll
      for (int b = 0; b < kUpdBatch; ++b)
#pragma unroll
        for (int u = 0; u < EPT; ++u)
          x[b][u] = (on[u] && sp0 + b < a.nsplit) ? p[(sp0 + b) * stride + r[u] * dkv + col[u]] : 0.f;
#pragma unroll
      for (int b = 0; b < kUpdBatch; ++b)
#pragma unroll
        for (int u = 0; u < EPT; ++u)
          if (sp0 + b < a.nsplit) val[u] = (sp0 + b == 0) ? x[b][u] : val[u] + x[b][u];
    }
  } else {
#pragma unroll
    for (int u = 0; u < EPT; ++u)
      val[u] = !on[u] ? 0.f
                      : (col[u] < dk ? a.k[(ki * a.n + r[u]) * dk + col[u]]
                                     : a.v[(ki * a.n + r[u]) * a.dv + (col[u] - dk)]);
  }
}

__global__ void __launch_bounds__(kUpdThreads, 2) mem_update_kernel(const MemUpdateArgs a, int S) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ __align__(16) float sm[];
  const int n = a.n, dk = a.dk, dv = a.dv, cs = dv / S;
  const int slice = static_cast<int>(blockIdx.x) % S, g = static_cast<int>(blockIdx.x) / S;
  const int j0 = slice * cs;
  const UpdLayout lay(n, dk, cs);
  float* fk = sm + lay.fk;
  float* As = sm + lay.As;
  float* Vs = sm + lay.Vs;
  float* D = sm + lay.D;
  float* zs = sm + lay.zs;
  float* den = sm + lay.den;
  float* gram = sm + lay.gram;
  const Cell c = load_cell(a.cells, g);
  const size_t ki = cell_index(a.kv_mode, a.L, c), si = cell_index(a.state_mode, a.L, c);
  float* A = a.A + si * dk * dv;
  float* z = a.z + si * dk;
  const int tid = threadIdx.x;

  // 1. this CTA's key rows [kr0, kr1) and its value columns (one loop, so that their loads
  //    are in flight together), its columns of A, and z
  constexpr int EPT = 4;
  const int kr0 = slice * n / S, kr1 = (slice + 1) * n / S;
  const int nkey = (kr1 - kr0) * dk, nval = n * cs;
  for (int e0 = tid; e0 < nkey + nval; e0 += EPT * kUpdThreads) {
    int r[EPT], col[EPT];
    bool on[EPT];
    float val[EPT];
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
      const int e = e0 + u * kUpdThreads;
      on[u] = e < nkey + nval;
      if (e < nkey) {
        r[u] = kr0 + e / dk;
        col[u] = e % dk;
      } else {
        const int ev = on[u] ? e - nkey : 0;
        r[u] = ev / cs;
        col[u] = dk + j0 + ev % cs;
      }
    }
    kv_values<EPT>(a, ki, r, col, on, val);
#pragma unroll
    for (int u = 0; u < EPT; ++u) {
      if (!on[u]) continue;
      if (col[u] < dk)
        fk[r[u] * dk + col[u]] = phi_f(val[u]);
      else
        Vs[r[u] * cs + (col[u] - dk - j0)] = val[u];
    }
  }
  for (int e = tid; e < dk * (cs / 4); e += kUpdThreads) {
    const int i = e / (cs / 4), q = e % (cs / 4);
    reinterpret_cast<float4*>(As + i * cs)[q] = *reinterpret_cast<const float4*>(A + static_cast<size_t>(i) * dv + j0 + 4 * q);
  }
  for (int i = tid; i < dk; i += kUpdThreads) zs[i] = z[i];
  if (S > 1) {
    // the key rows of the other slices, from their owners' shared memory (same layout)
    sm100::cluster_sync();
    for (int q = 0; q < S; ++q) {
      if (q == slice) continue;
      const int r0 = q * n / S, r1 = (q + 1) * n / S;
      for (int e = r0 * (dk / 4) + tid; e < r1 * (dk / 4); e += kUpdThreads) {
        const uint32_t src = sm100::mapa_shared(sm100::smem_u32(fk + 4 * e), static_cast<uint32_t>(q));
        reinterpret_cast<float4*>(fk)[e] = sm100::ld_dsmem_f4(src);
      }
    }
    sm100::cluster_arrive_release();  // this CTA has read its peers' rows (waited for at exit)
  }
  __syncthreads();

  // 2. row denominators
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < n; r += kUpdThreads / 32) {
    float d = 0.f;
    for (int i = lane; i < dk; i += 32) d = fmaf(fk[r * dk + i], zs[i], d);
    d = warp_sum(d);
    if (lane == 0) den[r] = d + a.eps;
  }
  __syncthreads();
  if (a.seq) seq_gram_den(fk, n, dk, lay.n4, gram, den, tid, kUpdThreads);

  // 3. D = V - phi(K) A / den for this slice's columns, i ascending per element: one row x 4
  //    columns per thread, so every thread has work; a warp's reads of a key row and of an A
  //    row are broadcasts
  for (int b = tid; b < n * (cs / 4); b += kUpdThreads) {
    const int r = b / (cs / 4), c0 = 4 * (b % (cs / 4));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i0 = 0; i0 < dk; i0 += 4) {
      const float4 f = *reinterpret_cast<const float4*>(fk + r * dk + i0);
      const float fr[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 av = *reinterpret_cast<const float4*>(As + (i0 + x) * cs + c0);
        acc[0] = fmaf(fr[x], av.x, acc[0]);
        acc[1] = fmaf(fr[x], av.y, acc[1]);
        acc[2] = fmaf(fr[x], av.z, acc[2]);
        acc[3] = fmaf(fr[x], av.w, acc[3]);
      }
    }
#pragma unroll
    for (int y = 0; y < 4; ++y) D[r * cs + c0 + y] = Vs[r * cs + c0 + y] - acc[y] / den[r];
  }
  __syncthreads();
  if (a.seq) {  // per-token rule: the innovations row after row
    seq_substitute(D, cs, cs, n, gram, lay.n4, den, tid, kUpdThreads);
    __syncthreads();
  }

  // 4. A' = A + phi(K)^T D for this slice's columns: 4 rows of A x 4 columns per thread
  for (int b = tid; b < (dk / 4) * (cs / 4); b += kUpdThreads) {
    const int i0 = 4 * (b / (cs / 4)), c0 = 4 * (b % (cs / 4));
    float s[4][4] = {};
    for (int r = 0; r < n; ++r) {
      const float4 f = *reinterpret_cast<const float4*>(fk + r * dk + i0);
      const float4 dd = *reinterpret_cast<const float4*>(D + r * cs + c0);
      const float fr[4] = {f.x, f.y, f.z, f.w}, dr[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) s[x][y] = fmaf(fr[x], dr[y], s[x][y]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float4 old = *reinterpret_cast<const float4*>(As + (i0 + x) * cs + c0);
      *reinterpret_cast<float4*>(A + static_cast<size_t>(i0 + x) * dv + j0 + c0) =
          make_float4(old.x + s[x][0], old.y + s[x][1], old.z + s[x][2], old.w + s[x][3]);
    }
  }
  if (slice == 0) {
    for (int i = tid; i < dk; i += kUpdThreads) {
      float t = 0.f;
      for (int r = 0; r < n; ++r) t += fk[r * dk + i];
      z[i] = zs[i] + t;
    }
    if (a.trace && tid == 0) {
      int* t = a.trace + 3 * (a.trace_base + g);
      t[0] = a.step;
      t[1] = c.l;
      t[2] = c.s;
    }
  }
  if (S > 1) sm100::cluster_wait_acquire();  // peers are done reading this CTA's key rows
}

// The update for launches of many cells (a throughput regime): persistent CTAs over contiguous
// ranges of cells, each cell's keys, values, A and z brought into shared memory by cp.async one
// cell ahead (two stages), so that the loads of the next cell overlap the arithmetic of this
// one. The arithmetic is mem_update_kernel's, element for element in the same order (the
// same bits): den by one warp per row, then v_bar and D over i ascending, then A' over rows
// ascending. Every thread works in every phase (1 x 4 and 4 x 4 register blocks), laid out so
// that a warp's shared-memory reads of a key row or an A row are broadcasts. Keys and values
// come as plain arrays or as whole sums (one split, [n][d_k + d_v] per cell).
constexpr int kUpdStreamThreads = 256;

struct UpdStreamLayout {  // in floats; every region starts 16-byte aligned
  int n8, stage, fk, D, den, gram, total;
  bool d_in_stage;  // D [n8][dv] over the cell's raw keys in its stage, dead once phi(K) is formed
  __host__ __device__ UpdStreamLayout(int n, int dk, int dv, int nst) {
    n8 = (n + 7) & ~7;
    stage = n * dk + n * dv + dk * dv + dk;  // K [n][dk], V [n][dv], A [dk][dv], z [dk]
    fk = nst * stage;                        // phi(K) [n][dk]
    d_in_stage = n8 * dv <= n * dk;
    D = d_in_stage ? -1 : fk + n * dk;       // [n8][dv] when it has a region of its own
    den = d_in_stage ? fk + n * dk : D + n8 * dv;  // [n8]
    gram = den + n8;                         // [n][n8] (per-token rule)
    total = gram + n * n8;
  }
};

// A ring of NST cell stages: the loads of cells g+1 .. g+NST-1 are in flight while cell g is
// computed (the stage of cell g+NST-1 is the one cell g-1 just released).
template <int NST>
__global__ void __launch_bounds__(kUpdStreamThreads, 4) mem_update_stream_kernel(const MemUpdateArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ __align__(16) float us[];
  const int n = a.n, dk = a.dk, dv = a.dv, dkv = dk + dv;
  const UpdStreamLayout lay(n, dk, dv, NST);
  float* fk = us + lay.fk;
  float* den = us + lay.den;
  float* gram = us + lay.gram;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per = (a.G + gridDim.x - 1) / gridDim.x;
  const int c_beg = blockIdx.x * per, c_end = min(a.G, c_beg + per);
  auto stage = [&](int i) { return us + (i % NST) * lay.stage; };
  auto issue = [&](int g, float* dst) {
    const Cell c = load_cell(a.cells, g);
    const size_t ki = cell_index(a.kv_mode, a.L, c), si = cell_index(a.state_mode, a.L, c);
    const float* kb = a.part ? a.part + ki * n * dkv : a.k + ki * n * dk;
    const float* vb = a.part ? kb + dk : a.v + ki * n * dv;
    const int ks = a.part ? dkv : dk, vs = a.part ? dkv : dv;
    for (int e = tid; e < n * (dk / 4); e += kUpdStreamThreads) {
      const int r = e / (dk / 4), q = e % (dk / 4);
      cp_async16(sm100::smem_u32(dst + r * dk + 4 * q), kb + static_cast<size_t>(r) * ks + 4 * q, 16u);
    }
    for (int e = tid; e < n * (dv / 4); e += kUpdStreamThreads) {
      const int r = e / (dv / 4), q = e % (dv / 4);
      cp_async16(sm100::smem_u32(dst + n * dk + r * dv + 4 * q), vb + static_cast<size_t>(r) * vs + 4 * q, 16u);
    }
    const float* A = a.A + si * dk * dv;
    for (int e = tid; e < (dk * dv + dk) / 4; e += kUpdStreamThreads) {
      const float* src = e < dk * dv / 4 ? A + 4 * e : a.z + si * dk + 4 * (e - dk * dv / 4);
      cp_async16(sm100::smem_u32(dst + n * dk + n * dv + 4 * e), src, 16u);
    }
  };
#pragma unroll
  for (int j = 0; j < NST - 1; ++j) {
    if (c_beg + j < c_end) issue(c_beg + j, stage(j));
    cp_async_commit();
  }
  for (int g = c_beg; g < c_end; ++g) {
    const int i = g - c_beg;
    float* st = stage(i);
    const float* Kr = st;
    float* D = lay.d_in_stage ? st : us + lay.D;  // over Kr: written only after phi(K) is formed
    const float* Vr = st + n * dk;
    const float* Ar = Vr + n * dv;
    const float* zr = Ar + dk * dv;
    // the stage of cell g-1 is free (the barrier that closed its iteration): refill it with
    // cell g+NST-1
    if (g + NST - 1 < c_end) issue(g + NST - 1, stage(i + NST - 1));
    cp_async_commit();
    cp_async_wait<NST - 1>();  // this cell's stage has landed (the later ones may still be in flight)
    __syncthreads();
    for (int e = tid; e < n * dk; e += kUpdStreamThreads) fk[e] = phi_f(Kr[e]);
    __syncthreads();
    for (int r = warp; r < n; r += kUpdStreamThreads / 32) {
      float d = 0.f;
      for (int i = lane; i < dk; i += 32) d = fmaf(fk[r * dk + i], zr[i], d);
      d = warp_sum(d);
      if (lane == 0) den[r] = d + a.eps;
    }
    __syncthreads();
    if (a.seq) seq_gram_den(fk, n, dk, lay.n8, gram, den, tid, kUpdStreamThreads);
    // D = V - phi(K) A / den: one row x 4 columns per thread, i ascending; a warp holds two rows
    // x 16 column blocks, so its reads of a row of phi(K) and of a row of A are broadcasts
    for (int b = tid; b < n * (dv / 4); b += kUpdStreamThreads) {
      const int r = b / (dv / 4), c0 = 4 * (b % (dv / 4));
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int i0 = 0; i0 < dk; i0 += 4) {
        const float4 f = *reinterpret_cast<const float4*>(fk + r * dk + i0);
        const float fr[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 av = *reinterpret_cast<const float4*>(Ar + (i0 + x) * dv + c0);
          acc[0] = fmaf(fr[x], av.x, acc[0]);
          acc[1] = fmaf(fr[x], av.y, acc[1]);
          acc[2] = fmaf(fr[x], av.z, acc[2]);
          acc[3] = fmaf(fr[x], av.w, acc[3]);
        }
      }
#pragma unroll
      for (int y = 0; y < 4; ++y) D[r * dv + c0 + y] = Vr[r * dv + c0 + y] - acc[y] / den[r];
    }
    __syncthreads();
    if (a.seq) {  // per-token rule: the innovations row after row
      seq_substitute(D, dv, dv, n, gram, lay.n8, den, tid, kUpdStreamThreads);
      __syncthreads();
    }
    // A' = A + phi(K)^T D: 4 rows of A x 4 columns per thread, rows of K ascending
    const Cell c = load_cell(a.cells, g);
    const size_t si = cell_index(a.state_mode, a.L, c);
    float* A = a.A + si * dk * dv;
    for (int b = tid; b < (dk / 4) * (dv / 4); b += kUpdStreamThreads) {
      const int i0 = 4 * (b / (dv / 4)), c0 = 4 * (b % (dv / 4));
      float s4[4][4] = {};
#pragma unroll 4
      for (int r = 0; r < n; ++r) {
        const float4 f = *reinterpret_cast<const float4*>(fk + r * dk + i0);
        const float4 dd = *reinterpret_cast<const float4*>(D + r * dv + c0);
        const float fr[4] = {f.x, f.y, f.z, f.w}, dr[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 4; ++y) s4[x][y] = fmaf(fr[x], dr[y], s4[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 old = *reinterpret_cast<const float4*>(Ar + (i0 + x) * dv + c0);
        *reinterpret_cast<float4*>(A + static_cast<size_t>(i0 + x) * dv + c0) =
            make_float4(old.x + s4[x][0], old.y + s4[x][1], old.z + s4[x][2], old.w + s4[x][3]);
      }
    }
    for (int i = tid; i < dk; i += kUpdStreamThreads) {
      float t = 0.f;
      for (int r = 0; r < n; ++r) t += fk[r * dk + i];
      a.z[si * dk + i] = zr[i] + t;
    }
    if (a.trace && tid == 0) {
      int* t = a.trace + 3 * (a.trace_base + g);
      t[0] = a.step;
      t[1] = c.l;
      t[2] = c.s;
    }
    __syncthreads();  // the stage, phi(K) and D are free again
  }
  cp_async_wait<0>();
}

}  // namespace

template <typename T>
cudaError_t launch_mem_read_t(const MemReadArgs& a, size_t smem, cudaStream_t st) {
  if (smem > 48 * 1024) cudaFuncSetAttribute(mem_read_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((a.M + kReadRows - 1) / kReadRows, a.G);
  const cudaError_t e = launch_pdl(mem_read_kernel<T>, grid, dim3(kReadWarps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int DK>
cudaError_t launch_mem_read_mma_dk(const MemReadArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * kReadMmaWarps * kReadStages * 16 * (DK + 8) +
                      2 * sizeof(__nv_bfloat16) * (a.dv + 8) * (DK + 8) + sizeof(T) * kReadMmaWarps * 16 * (a.dv + 8);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(mem_read_mma_kernel<T, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // rows per CTA: a whole cell when the launch has cells enough for two CTAs per SM, else
  // blocks of 64-row multiples that give it about that many CTAs
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long want = 2L * (sms > 0 ? sms : 148);
  const long per_cell = (want + a.G - 1) / a.G;
  int rows = static_cast<int>((a.M + per_cell - 1) / per_cell);
  rows = (rows + 63) / 64 * 64;
  if (rows > a.M) rows = a.M;
  dim3 grid((a.M + rows - 1) / rows, a.G);
  const cudaError_t e = launch_pdl(mem_read_mma_kernel<T, DK>, grid, dim3(kReadMmaWarps * 32), smem, st, a, rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_mem_read_mma_t(const MemReadArgs& a, cudaStream_t st) {
  switch (a.dk) {
    case 32: return launch_mem_read_mma_dk<T, 32>(a, st);
    case 64: return launch_mem_read_mma_dk<T, 64>(a, st);
    case 96: return launch_mem_read_mma_dk<T, 96>(a, st);
    case 128: return launch_mem_read_mma_dk<T, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_mem_read(const MemReadArgs& a, ElemType out_type, cudaStream_t st, int* err) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.dk % 32 || a.dv % 32 || a.dk > 128 || a.dv > 128) return cudaErrorInvalidValue;
  const size_t smem = (static_cast<size_t>(a.dk) * a.dv + a.dk) * sizeof(float);
  const bool tc = mem_read_tc_supported(a.dk, a.dv);
  // an output row stride and low terms only on the tensor-core read
  if ((a.ldo && a.ldo != a.dv) || a.lo_off) {
    if (!tc || out_type == kElemF32 || a.ldo < a.dv + a.lo_off || a.ldo % 8 || a.lo_off % 8)
      return cudaErrorInvalidValue;
  }
  switch (out_type) {
    case kElemF32: return launch_mem_read_t<float>(a, smem, st);
    case kElemBF16: return tc ? launch_mem_read_tc(a, false, err, st) : launch_mem_read_mma_t<__nv_bfloat16>(a, st);
    case kElemF16: return tc ? launch_mem_read_tc(a, true, err, st) : launch_mem_read_mma_t<__half>(a, st);
  }
  return cudaErrorInvalidValue;
}


bool mem_kv_whole(int G, int n, bool bf16) {
  if (!bf16 || n > 16) return false;  // the running sums of one 16-row tile in registers
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return static_cast<long>(G) >= 4L * (sms > 0 ? sms : 148);
}

cudaError_t launch_mem_kv(const MemKvArgs& a, bool bf16, cudaStream_t st) {
  if (a.G <= 0) return cudaSuccess;
  if (a.n > 64 || a.dkv % 4) return cudaErrorInvalidValue;
  dim3 grid((a.d + kMemKvSplit - 1) / kMemKvSplit, a.G, (a.dkv + kKvCols - 1) / kKvCols);
  if (bf16) {  // tensor cores: three-term split of the fp32 rows against the bf16 weights
    const int cols = a.dkv < kKvCols ? a.dkv : kKvCols;
    const bool whole = mem_kv_whole(a.G, a.n, true);
    size_t smem = kv_mma_smem(a.n, cols, whole ? kKvWholeStages : 1);
    if (whole && smem > 227 * 1024) return cudaErrorInvalidValue;  // n > 16 is kept off this route
    void (*kern)(MemKvArgs) = whole ? mem_kv_mma_kernel<true> : mem_kv_mma_kernel<false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (whole) grid.x = 1;
    const cudaError_t e = launch_pdl(kern, grid, dim3(kKvMmaThreads), smem, st, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const size_t n4 = (a.n + 3) & ~3;
  const size_t cols = a.dkv < kKvCols ? a.dkv : kKvCols;
  const size_t smem = (n4 * kMemKvSplit + static_cast<size_t>(kMemKvSplit) * cols) * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(mem_kv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const cudaError_t e = launch_pdl(mem_kv_kernel<float>, grid, dim3(kKvThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}




cudaError_t launch_mem_update(const MemUpdateArgs& a, cudaStream_t st) {
  if (a.G <= 0) return cudaSuccess;
  if (a.n <= 0 || a.dk % 32 || a.dv % 32 || a.dk > 128 || a.dv > 128) return cudaErrorInvalidValue;
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // many cells, whole keys and values: the streaming kernel (the same bits as the one below),
  // two cell stages per CTA (a 4-stage ring measured no faster: the arithmetic, not the loads,
  // sets its pace)
  const size_t smem_stream = static_cast<size_t>(UpdStreamLayout(a.n, a.dk, a.dv, 2).total) * sizeof(float);
  if (static_cast<long>(a.G) >= 4L * sms && (!a.part || a.nsplit == 1) && smem_stream <= 200 * 1024) {
    void (*kern)(MemUpdateArgs) = mem_update_stream_kernel<2>;
    if (smem_stream > 48 * 1024)
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_stream);
    int fit = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fit, kern, kUpdStreamThreads, smem_stream) != cudaSuccess ||
        fit <= 0) {
      cudaGetLastError();
      fit = 1;
    }
    const long cap = static_cast<long>(sms) * fit;
    const int grid = static_cast<int>(a.G < cap ? a.G : cap);
    const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(kUpdStreamThreads), smem_stream, st, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  // column slices: the widest of 64, 32, 16 columns that still gives two CTAs per SM; else 16
  int cs = 16;
  for (int w = 64; w >= 16; w /= 2) {
    if (a.dv % w == 0 && static_cast<long>(a.G) * (a.dv / w) >= 2L * sms) {
      cs = w;
      break;
    }
  }
  const int S = a.dv / cs;  // at most 8: a portable cluster
  const size_t smem = static_cast<size_t>(UpdLayout(a.n, a.dk, cs).total) * sizeof(float);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(mem_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.G * S);
  cfg.blockDim = dim3(kUpdThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mem_update_kernel, a, S);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}


}  // namespace rmt

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

namespace rmt {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
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
  const Cell c = a.cells[blockIdx.y];
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
  const Cell c = a.cells[blockIdx.y];
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

// --------------------------------------------------------------------------- update
// CTA = one cell. Shared memory: raw k|v rows, phi(k), A, z, row denominators, V - v_bar.
constexpr int kUpdThreads = 512;

__global__ void __launch_bounds__(kUpdThreads) mem_update_kernel(const MemUpdateArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  extern __shared__ float sm[];
  const int n = a.n, dk = a.dk, dv = a.dv, dkv = dk + dv;
  float* KV = sm;              // [n][dkv]: phi(k) in columns < dk, v after
  float* As = KV + n * dkv;    // [dk][dv]
  float* zs = As + dk * dv;    // [dk]
  float* den = zs + dk;        // [n]
  float* D = den + n;          // [n][dv]
  const Cell c = a.cells[blockIdx.x];
  const size_t ki = cell_index(a.kv_mode, a.L, c), si = cell_index(a.state_mode, a.L, c);
  float* A = a.A + si * dk * dv;
  float* z = a.z + si * dk;

  if (a.part) {
    // each thread sums 4 elements at once over the splits (ascending, as one element at a
    // time would), so 4 x 8 partial loads are in flight instead of 8
    constexpr int EPT = 4;
    const float* p = a.part + ki * a.nsplit * n * dkv;
    const size_t stride = static_cast<size_t>(n) * dkv;
    for (int e0 = threadIdx.x; e0 < n * dkv; e0 += EPT * kUpdThreads) {
      float val[EPT] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int sp = 0; sp < a.nsplit; ++sp) {
#pragma unroll
        for (int u = 0; u < EPT; ++u) {
          const int e = e0 + u * kUpdThreads;
          if (e < n * dkv) val[u] += p[sp * stride + e];
        }
      }
#pragma unroll
      for (int u = 0; u < EPT; ++u) {
        const int e = e0 + u * kUpdThreads;
        if (e < n * dkv) KV[e] = e % dkv < dk ? phi_f(val[u]) : val[u];
      }
    }
  } else {
    for (int e = threadIdx.x; e < n * dkv; e += kUpdThreads) {
      const int r = e / dkv, j = e % dkv;
      const float val = j < dk ? a.k[(ki * n + r) * dk + j] : a.v[(ki * n + r) * dv + (j - dk)];
      KV[e] = j < dk ? phi_f(val) : val;
    }
  }
  for (int e = threadIdx.x; e < dk * dv; e += kUpdThreads) As[e] = A[e];
  for (int e = threadIdx.x; e < dk; e += kUpdThreads) zs[e] = z[e];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < n; r += kUpdThreads / 32) {
    float d = 0.f;
    for (int i = lane; i < dk; i += 32) d = fmaf(KV[r * dkv + i], zs[i], d);
    d = warp_sum(d);
    if (lane == 0) den[r] = d + a.eps;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * dv; e += kUpdThreads) {
    const int r = e / dv, j = e % dv;
    float num = 0.f;
    for (int i = 0; i < dk; ++i) num = fmaf(KV[r * dkv + i], As[i * dv + j], num);
    D[e] = KV[r * dkv + dk + j] - num / den[r];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < dk * dv; e += kUpdThreads) {
    const int i = e / dv, j = e % dv;
    float s = 0.f;
    for (int r = 0; r < n; ++r) s = fmaf(KV[r * dkv + i], D[r * dv + j], s);
    A[e] = As[e] + s;
  }
  for (int i = threadIdx.x; i < dk; i += kUpdThreads) {
    float s = 0.f;
    for (int r = 0; r < n; ++r) s += KV[r * dkv + i];
    z[i] = zs[i] + s;
  }
  if (a.trace && threadIdx.x == 0) {
    int* t = a.trace + 3 * (a.trace_base + blockIdx.x);
    t[0] = a.step;
    t[1] = c.l;
    t[2] = c.s;
  }
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

cudaError_t launch_mem_read(const MemReadArgs& a, ElemType out_type, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.dk % 32 || a.dv % 32 || a.dk > 128 || a.dv > 128) return cudaErrorInvalidValue;
  const size_t smem = (static_cast<size_t>(a.dk) * a.dv + a.dk) * sizeof(float);
  switch (out_type) {
    case kElemF32: return launch_mem_read_t<float>(a, smem, st);
    case kElemBF16: return launch_mem_read_t<__nv_bfloat16>(a, smem, st);
    case kElemF16: return launch_mem_read_t<__half>(a, smem, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_mem_kv(const MemKvArgs& a, bool bf16, cudaStream_t st) {
  if (a.G <= 0) return cudaSuccess;
  if (a.n > 64 || a.dkv % 4) return cudaErrorInvalidValue;
  const size_t n4 = (a.n + 3) & ~3;
  const size_t cols = a.dkv < kKvCols ? a.dkv : kKvCols;
  const size_t smem = (n4 * kMemKvSplit + static_cast<size_t>(kMemKvSplit) * cols) * sizeof(float);
  dim3 grid((a.d + kMemKvSplit - 1) / kMemKvSplit, a.G, (a.dkv + kKvCols - 1) / kKvCols);
  if (bf16) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(mem_kv_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_pdl(mem_kv_kernel<__nv_bfloat16>, grid, dim3(kKvThreads), smem, st, a);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(mem_kv_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return launch_pdl(mem_kv_kernel<float>, grid, dim3(kKvThreads), smem, st, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_mem_update(const MemUpdateArgs& a, cudaStream_t st) {
  if (a.G <= 0) return cudaSuccess;
  const size_t smem = (static_cast<size_t>(a.n) * (a.dk + a.dv) + static_cast<size_t>(a.dk) * a.dv + a.dk + a.n +
                       static_cast<size_t>(a.n) * a.dv) *
                      sizeof(float);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(mem_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const cudaError_t e = launch_pdl(mem_update_kernel, dim3(a.G), dim3(kUpdThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rmt

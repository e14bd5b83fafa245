// Row-streaming kernels (HBM-bound): RMSNorm, layer-0 input assembly, segment output.
#include "common.cuh"
#include "launch.h"

namespace rmt {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T> struct Vec4;
template <> struct Vec4<float> {
  static __device__ __forceinline__ void store(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
  static __device__ __forceinline__ float4 load(const float* p) { return *reinterpret_cast<const float4*>(p); }
};
template <> struct Vec4<__half> {
  static __device__ __forceinline__ void store(__half* p, float4 v) {
    __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
};
template <> struct Vec4<__nv_bfloat16> {
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
  }
  static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
  }
};

// RMSNorm: one warp per row, y = x * rsqrt(mean(x^2) + eps) * g, statistics in fp32.
constexpr int kRmsWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kRmsWarps * 32) rmsnorm_kernel(const RmsArgs a) {
  const Cell c = load_cell(a.cells, blockIdx.y);
  const int row = blockIdx.x * kRmsWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= a.M) return;
  const float* x = a.x + (static_cast<size_t>(cell_index(a.x_mode, a.L, c)) * a.M + row) * a.d;
  T* y = static_cast<T*>(a.y) + (static_cast<size_t>(cell_index(a.y_mode, a.L, c)) * a.M + row) * a.d;
  const T* g = static_cast<const T*>(a.g) + static_cast<size_t>(c.l) * a.d;
  float ss = 0.f;
  for (int k = lane * 4; k < a.d; k += 128) {
    const float4 v = Vec4<float>::load(x + k);
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / static_cast<float>(a.d) + a.eps);
  for (int k = lane * 4; k < a.d; k += 128) {
    const float4 v = Vec4<float>::load(x + k);
    const float4 gv = Vec4<T>::load(g + k);
    Vec4<T>::store(y + k, make_float4(v.x * r * gv.x, v.y * r * gv.y, v.z * r * gv.z, v.w * r * gv.w));
  }
}

// Layer-0 input of cell blockIdx.y (row blockIdx.x of M): the segment's tokens from the packed
// embeddings, then the memory tokens, then zero padding up to M. An f16 operand copy that
// overflows is reported in the error word.
template <typename T>
__global__ void assemble_kernel(const Cell* cells, const T* emb, const T* mem, float* x, __half* xb, int M, int n_mem,
                                int d, int split, int* err) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  const Cell c = load_cell(cells, blockIdx.y);
  const int r = blockIdx.x, m = cell_rows(c, M), seg = m - n_mem;
  const T* src = r < seg ? emb + (static_cast<size_t>(c.t0) + r) * d
                         : (r < m ? mem + static_cast<size_t>(r - seg) * d : nullptr);
  const size_t row = (static_cast<size_t>(c.xin) * M + r) * d;
  const size_t rowb = split ? 2 * row : row;  // split-operand mode: [high terms | low terms] rows of 2d
  float amax = 0.f;
  for (int k = threadIdx.x * 4; k < d; k += blockDim.x * 4) {
    const float4 v = src ? Vec4<T>::load(src + k) : make_float4(0.f, 0.f, 0.f, 0.f);
    Vec4<float>::store(x + row + k, v);
    if (xb) {
      Vec4<__half>::store(xb + rowb + k, v);
      if (split)
        Vec4<__half>::store(xb + rowb + d + k, make_float4(lo_term<__half>(v.x), lo_term<__half>(v.y),
                                                           lo_term<__half>(v.z), lo_term<__half>(v.w)));
      amax = fmaxf(fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y))), fmaxf(fabsf(v.z), fabsf(v.w)));
    }
  }
  report_f16_range<__half>(amax, err);
}

// Output rows of cell blockIdx.y: its segment's tokens (row blockIdx.x), cast to T, to the
// packed output at the segment's first token.
template <typename T>
__global__ void emit_kernel(const Cell* cells, const float* x, T* out, int M, int n_mem, int d) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  const Cell c = load_cell(cells, blockIdx.y);
  const int r = blockIdx.x;
  if (r >= cell_rows(c, M) - n_mem) return;
  const float* src = x + (static_cast<size_t>(c.xout) * M + r) * d;
  T* dst = out + (static_cast<size_t>(c.t0) + r) * d;
  for (int k = threadIdx.x * 4; k < d; k += blockDim.x * 4) Vec4<T>::store(dst + k, Vec4<float>::load(src + k));
}

// Row sums of squares of an fp32 [M, d] block, per column block b of width w = d / parts
// (ss[row * parts + b]): the RMSNorm statistics a folded projection reads. One warp per
// block: each lane squares 4 consecutive columns per 128-column step, then a fixed butterfly
// adds the lanes.
__global__ void row_ssq_kernel(const float* x, float* ss, int d, int parts) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  const int row = blockIdx.x, b = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (b >= parts) return;
  const int w = d / parts;
  const float* xb = x + static_cast<size_t>(row) * d + static_cast<size_t>(b) * w;
  float s = 0.f;
  for (int k = lane * 4; k < w; k += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xb + k);
    s += ((v.x * v.x + v.y * v.y) + v.z * v.z) + v.w * v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) ss[static_cast<size_t>(row) * parts + b] = s;
}

// W[l][n][k] *= g[l][k]: folds an RMSNorm gain into the weight that consumes its output.
template <typename WT, typename GT>
__global__ void scale_cols_kernel(WT* w, const GT* g, int N, int K) {
  WT* wl = w + static_cast<size_t>(blockIdx.y) * N * K;
  const GT* gl = g + static_cast<size_t>(blockIdx.y) * K;
  const size_t n = static_cast<size_t>(N) * K;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    wl[e] = from_f32<WT>(to_f32<WT>(wl[e]) * to_f32<GT>(gl[e % K]));
}

__global__ void bf16_to_f16_kernel(uint16_t* p, size_t n) {
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = __uint_as_float(static_cast<uint32_t>(p[e]) << 16);
    const __half hv = __float2half_rn(v);
    p[e] = *reinterpret_cast<const uint16_t*>(&hv);
  }
}

}  // namespace

cudaError_t launch_scale_cols(void* w, const void* g, int L, int N, int K, bool bf16, bool w_f16, cudaStream_t st) {
  dim3 grid(1024, L);
  if (bf16 && w_f16)
    scale_cols_kernel<__half, __nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<__half*>(w),
                                                                    static_cast<const __nv_bfloat16*>(g), N, K);
  else if (bf16)
    scale_cols_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<__nv_bfloat16*>(w),
                                                                           static_cast<const __nv_bfloat16*>(g), N, K);
  else
    scale_cols_kernel<float, float><<<grid, 256, 0, st>>>(static_cast<float*>(w), static_cast<const float*>(g), N, K);
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f16(void* p, size_t n, cudaStream_t st) {
  bf16_to_f16_kernel<<<2048, 256, 0, st>>>(static_cast<uint16_t*>(p), n);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const RmsArgs& a, bool bf16, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.d % 4) return cudaErrorInvalidValue;
  dim3 grid((a.M + kRmsWarps - 1) / kRmsWarps, a.G);
  if (bf16)
    rmsnorm_kernel<__nv_bfloat16><<<grid, kRmsWarps * 32, 0, st>>>(a);
  else
    rmsnorm_kernel<float><<<grid, kRmsWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_assemble(const Cell* cells, int G, const void* emb, const void* mem, float* x, __half* xb, int M,
                            int n_mem, int d, bool bf16, int* err, cudaStream_t st, bool split) {
  if (d % 4) return cudaErrorInvalidValue;
  if (G <= 0) return cudaSuccess;
  const int threads = d >= 1024 ? 256 : 128;
  const int sp = split ? 1 : 0;
  if (bf16)
    return launch_pdl(assemble_kernel<__nv_bfloat16>, dim3(M, G), dim3(threads), 0, st, cells,
                      static_cast<const __nv_bfloat16*>(emb), static_cast<const __nv_bfloat16*>(mem), x, xb, M, n_mem, d,
                      sp, err);
  return launch_pdl(assemble_kernel<float>, dim3(M, G), dim3(threads), 0, st, cells, static_cast<const float*>(emb),
                    static_cast<const float*>(mem), x, xb, M, n_mem, d, sp, err);
}

cudaError_t launch_row_ssq(const float* x, float* ss, int M, int d, int parts, cudaStream_t st) {
  if (parts <= 0 || parts > 32 || d % parts || (d / parts) % 4) return cudaErrorInvalidValue;
  if (M <= 0) return cudaSuccess;
  return launch_pdl(row_ssq_kernel, dim3(M), dim3(32 * parts), 0, st, x, ss, d, parts);
}

cudaError_t launch_emit(const Cell* cells, int G, const float* x, void* out, int M, int n_mem, int d, bool bf16,
                        cudaStream_t st) {
  if (d % 4) return cudaErrorInvalidValue;
  if (G <= 0) return cudaSuccess;
  const int threads = d >= 1024 ? 256 : 128;
  if (bf16)
    return launch_pdl(emit_kernel<__nv_bfloat16>, dim3(M - n_mem, G), dim3(threads), 0, st, cells, x,
                      static_cast<__nv_bfloat16*>(out), M, n_mem, d);
  return launch_pdl(emit_kernel<float>, dim3(M - n_mem, G), dim3(threads), 0, st, cells, x, static_cast<float*>(out), M,
                    n_mem, d);
}

}  // namespace rmt

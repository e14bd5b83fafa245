// Grouped GEMM in fp32 FMA (no tensor cores), for the fp32 storage mode: tf32 tensor-core
// products would not meet a 1e-4 relative tolerance. Same contract and epilogues as the
// tensor-core kernel: group g = one (layer, segment) cell, weight slice = its layer.
// Tiles of 64 x 128 with K steps of 16; the finished tile is staged in shared memory so
// that epilogues which pair columns (RoPE halves, SwiGLU gate/up) see the whole tile.
#include "common.cuh"
#include "launch.h"

namespace rmt {
namespace {

constexpr int BM = 64, BN = 128, BK = 16, NT = 256;

__global__ void __launch_bounds__(NT) simt_gemm_kernel(const SimtGemmArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  __shared__ float As[BK][BM];
  __shared__ float Bs[BK][BN];
  __shared__ float Cs[BM][BN + 1];
  const Cell c = load_cell(a.cells, blockIdx.z);
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const float* A = a.a + static_cast<size_t>(cell_index(a.a_mode, a.L, c)) * a.M * a.lda;
  const float* W = a.w + static_cast<size_t>(c.l) * a.N * a.K;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  float acc[4][8] = {};
  for (int k0 = 0; k0 < a.K; k0 += BK) {
    {  // A tile: 64 rows x 16 k, 4 per thread
      const int r = t >> 2, kk = (t & 3) * 4;
      for (int q = 0; q < 4; ++q) {
        const int gr = m0 + r, gk = k0 + kk + q;
        As[kk + q][r] = (gr < a.M && gk < a.K) ? A[static_cast<size_t>(gr) * a.lda + gk] : 0.f;
      }
    }
    {  // B tile: 128 rows (n) x 16 k, 8 per thread
      const int n = t >> 1, kk = (t & 1) * 8;
      for (int q = 0; q < 8; ++q) {
        const int gn = n0 + n, gk = k0 + kk + q;
        Bs[kk + q][n] = (gn < a.N && gk < a.K) ? W[static_cast<size_t>(gn) * a.K + gk] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float av[4], bv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) bv[j] = Bs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) Cs[ty * 4 + i][tx + 16 * j] = acc[i][j];
  __syncthreads();

  const EpiParams& ep = a.ep;
  __shared__ float rs[BM];  // folded RMSNorm row scales (RoPE and SwiGLU epilogues)
  if ((a.epi == kEpiRope || a.epi == kEpiSwiGLU) && t < BM) {
    const int row = m0 + t;
    rs[t] = (ep.ss_in && row < a.M)
                ? rms_row_scale(ep.ss_in + (static_cast<size_t>(c.k) * a.M + row) * ep.ss_parts, ep.ss_parts, ep.inv_d,
                                ep.rms_eps)
                : 1.f;
  }
  __syncthreads();
  if (a.epi == kEpiSwiGLU) {
    // output column j of this tile pair: gate at block-start + p, up at block-start + 64 + p
    float* out = static_cast<float*>(ep.out) + static_cast<size_t>(cell_index(ep.out_mode, a.L, c)) * a.M * ep.ldo;
    for (int e = t; e < BM * (BN / 2); e += NT) {
      const int r = e / (BN / 2), j = e % (BN / 2);
      const int blk = j / kSwiGLUBlock, p = j % kSwiGLUBlock;
      const int cg = blk * 2 * kSwiGLUBlock + p;
      if (m0 + r >= a.M || n0 + cg >= a.N) continue;
      out[static_cast<size_t>(m0 + r) * ep.ldo + n0 / 2 + j] = silu_f(Cs[r][cg] * rs[r]) * (Cs[r][cg + kSwiGLUBlock] * rs[r]);
    }
    return;
  }
  for (int e = t; e < BM * BN; e += NT) {
    const int r = e / BN, cc = e % BN;
    const int row = m0 + r, col = n0 + cc;
    if (row >= a.M || col >= a.N) continue;
    float v = Cs[r][cc];
    switch (a.epi) {
      case kEpiStoreF32:
      case kEpiStoreAct: {
        float* out = static_cast<float*>(ep.out) + static_cast<size_t>(cell_index(ep.out_mode, a.L, c)) * a.M * ep.ldo;
        out[static_cast<size_t>(row) * ep.ldo + col] = v;
        break;
      }
      case kEpiRope: {
        v *= rs[r];
        if (col < ep.rope_cols) {
          const int half = ep.head_dim >> 1, i = col % ep.head_dim;
          const float2 cs = ep.rope[static_cast<size_t>(row) * half + (i % half)];
          v = i < half ? v * cs.x - Cs[r][cc + half] * rs[r] * cs.y : v * cs.x + Cs[r][cc - half] * rs[r] * cs.y;
        }
        float* out = static_cast<float*>(ep.out) + static_cast<size_t>(cell_index(ep.out_mode, a.L, c)) * a.M * ep.ldo;
        out[static_cast<size_t>(row) * ep.ldo + col] = v;
        break;
      }
      case kEpiResid:
      case kEpiResidCast: {
        const float* src = ep.x + static_cast<size_t>(cell_index(ep.src_mode, a.L, c)) * a.M * ep.ldx;
        float* dst = ep.x + static_cast<size_t>(cell_index(ep.dst_mode, a.L, c)) * a.M * ep.ldx;
        const float y = src[static_cast<size_t>(row) * ep.ldx + col] + v;
        dst[static_cast<size_t>(row) * ep.ldx + col] = y;
        Cs[r][cc] = y;  // kept for the row sums of squares below
        break;
      }
      default:
        break;
    }
  }
  if ((a.epi == kEpiResid || a.epi == kEpiResidCast) && ep.ss_out) {
    __syncthreads();
    if (t < BM && m0 + t < a.M) {
      float ss = 0.f;
      for (int cc = 0; cc < BN && n0 + cc < a.N; ++cc) ss = fmaf(Cs[t][cc], Cs[t][cc], ss);
      ep.ss_out[(static_cast<size_t>(c.k) * a.M + m0 + t) * ep.ss_parts + blockIdx.x] = ss;
    }
  }
}

}  // namespace

cudaError_t launch_simt_gemm(const SimtGemmArgs& a, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0 || a.N <= 0) return cudaSuccess;
  if (a.epi == kEpiRope && (BN % a.ep.head_dim != 0)) return cudaErrorInvalidValue;
  dim3 grid((a.N + BN - 1) / BN, (a.M + BM - 1) / BM, a.G);
  const cudaError_t e = launch_pdl(simt_gemm_kernel, grid, dim3(NT), 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rmt

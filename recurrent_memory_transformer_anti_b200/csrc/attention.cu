// Segment-local causal attention with grouped key/value heads, one (layer, segment) cell
// per group: every query row i of the cell attends to rows 0..i of the same cell (its
// segment tokens, then its memory tokens); query head h reads key/value head
// h / (H / Hkv). No key/value crosses a segment boundary: the recurrence carries state
// only through the associative memory (arXiv 2506.05229 abstract: recurrent memory
// transformers process a long input segment by segment).
//
// 16-bit (bf16 or f16): flash-attention style, 64 query rows per CTA (16 per warp),
// key/value tiles of 64 rows double-buffered with cp.async, QK^T and PV on mma.sync
// m16n8k16 (16-bit in, fp32 accumulate), online softmax in fp32 registers. Used for
// head_dim 32 (the tensor-core kernel covers 64 and 128).
// fp32: one thread per query row, key/value chunks staged in shared memory.
#include "common.cuh"
#include "launch.h"

namespace rmt {
namespace {

// ----------------------------------------------------------------------------- helpers

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

template <typename OpT>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (OpFormat<OpT>::value == 1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// ---------------------------------------------------------------------- 16-bit kernel

template <int HD>
struct AttnSmem {
  static constexpr int BQ = 64, BKV = 64, LDS = HD + 8;  // +16 B per row: conflict-free ldmatrix
  static constexpr int TILE = BKV * LDS;                 // elements
  static constexpr int BYTES = (BQ * LDS + 4 * TILE) * 2;
};

template <int HD, typename OpT>
__global__ void __launch_bounds__(128) attn_mma_kernel(const AttnArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  using S = AttnSmem<HD>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  OpT* Qs = reinterpret_cast<OpT*>(smem_raw);
  OpT* Ks = Qs + S::BQ * S::LDS;  // [2][BKV][LDS]
  OpT* Vs = Ks + 2 * S::TILE;     // [2][BKV][LDS]

  const int nqt = (a.M + S::BQ - 1) / S::BQ;
  const int qt = nqt - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y;
  const Cell c = load_cell(a.cells, blockIdx.z);
  const int kvlim = cell_rows(c, a.M);  // keys past the cell's tokens are masked
  const int rep = a.H / a.Hkv, kvh = h / rep;
  const int ldq = (a.H + 2 * a.Hkv) * HD, ldo = a.ldo ? a.ldo : a.H * HD;
  const size_t slice = cell_index(a.mode, a.L, c);
  const OpT* base = static_cast<const OpT*>(a.qkv) + slice * a.M * ldq;
  const OpT* qsrc = base + h * HD;
  const OpT* ksrc = base + (a.H + kvh) * HD;
  const OpT* vsrc = base + (a.H + a.Hkv + kvh) * HD;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = qt * S::BQ;
  constexpr int CH = HD / 8;  // 16-byte chunks per row

  for (int i = tid; i < S::BQ * CH; i += 128) {
    const int r = i / CH, ch = i % CH, row = q0 + r;
    const int rr = row < a.M ? row : a.M - 1;
    cp_async16(Qs + r * S::LDS + ch * 8, qsrc + static_cast<size_t>(rr) * ldq + ch * 8, row < a.M ? 16 : 0);
  }
  auto load_kv = [&](int kt, int buf) {
    const int k0 = kt * S::BKV;
    for (int i = tid; i < S::BKV * CH; i += 128) {
      const int r = i / CH, ch = i % CH, row = k0 + r;
      const int rr = row < a.M ? row : a.M - 1;
      const int nb = row < a.M ? 16 : 0;  // rows past the cell read as zeros
      cp_async16(Ks + buf * S::TILE + r * S::LDS + ch * 8, ksrc + static_cast<size_t>(rr) * ldq + ch * 8, nb);
      cp_async16(Vs + buf * S::TILE + r * S::LDS + ch * 8, vsrc + static_cast<size_t>(rr) * ldq + ch * 8, nb);
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  const float sl2 = rsqrtf(static_cast<float>(HD)) * 1.4426950408889634f;  // 1/sqrt(dh) * log2(e)
  uint32_t qf[HD / 16][4];
  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const int g = lane >> 2, tq = lane & 3;
  const int qrow0 = q0 + warp * 16 + g;  // this thread's rows: qrow0 and qrow0 + 8

  const int nkt = qt + 1;
  for (int kt = 0; kt < nkt; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nkt) {
      load_kv(kt + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk)
        ldsm_x4(qf[kk], Qs + (warp * 16 + (lane & 15)) * S::LDS + kk * 16 + (lane >> 4) * 8);
    }
    const OpT* Kb = Ks + buf * S::TILE;
    const OpT* Vb = Vs + buf * S::TILE;

    float s[8][4];
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int nb = 0; nb < 8; nb += 2) {
        uint32_t b[4];
        ldsm_x4(b, Kb + (nb * 8 + (lane >> 4) * 8 + (lane & 7)) * S::LDS + kk * 16 + ((lane >> 3) & 1) * 8);
        mma16816<OpT>(s[nb], qf[kk], b[0], b[1]);
        mma16816<OpT>(s[nb + 1], qf[kk], b[2], b[3]);
      }
    }
    // scale, causal mask (and rows of the cell's ragged end), running max
    const int k0 = kt * S::BKV;
    const bool need_mask = (kt == qt) || (k0 + S::BKV > kvlim);
    float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[nb][e] * sl2;
        if (need_mask) {
          const int kv = k0 + nb * 8 + 2 * tq + (e & 1);
          const int qr = qrow0 + (e >> 1) * 8;
          if (kv > qr || kv >= kvlim) v = -INFINITY;
        }
        s[nb][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2], msafe[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      msafe[r] = mx[r] == -INFINITY ? 0.f : mx[r];
      corr[r] = exp2f(mrow[r] - msafe[r]);
      mrow[r] = mx[r];
      lrow[r] *= corr[r];
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nb][e] - msafe[e >> 1]);
        s[nb][e] = p;
        lrow[e >> 1] += p;
      }
    }
#pragma unroll
    for (int nd = 0; nd < HD / 8; ++nd) {
      o[nd][0] *= corr[0];
      o[nd][1] *= corr[0];
      o[nd][2] *= corr[1];
      o[nd][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < S::BKV / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack2<OpT>(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack2<OpT>(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack2<OpT>(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack2<OpT>(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nd = 0; nd < HD / 8; nd += 2) {
        uint32_t b[4];
        ldsm_x4_t(b, Vb + (kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * S::LDS + nd * 8 + (lane >> 4) * 8);
        mma16816<OpT>(o[nd], pa, b[0], b[1]);
        mma16816<OpT>(o[nd + 1], pa, b[2], b[3]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  OpT* obase = static_cast<OpT*>(a.out) + slice * a.M * ldo + h * HD;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = qrow0 + r * 8;
    if (row >= a.M) continue;
    const float inv = 1.f / lrow[r];
    uint32_t* dst = reinterpret_cast<uint32_t*>(obase + static_cast<size_t>(row) * ldo);
#pragma unroll
    for (int nd = 0; nd < HD / 8; ++nd) dst[(nd * 8 + 2 * tq) >> 1] = pack2<OpT>(o[nd][2 * r] * inv, o[nd][2 * r + 1] * inv);
  }
}

// ------------------------------------------------------------------------ fp32 kernel

template <int HD>
__global__ void __launch_bounds__(64) attn_f32_kernel(const AttnArgs a) {
  pdl_trigger();
  pdl_wait();  // inputs come from the previous kernels of the stream
  constexpr int BQ = 64, CK = 32;
  __shared__ float Kc[CK][HD];
  __shared__ float Vc[CK][HD];
  const int qc = blockIdx.x, h = blockIdx.y;
  const Cell c = load_cell(a.cells, blockIdx.z);
  const int kvlim = cell_rows(c, a.M);  // keys past the cell's tokens are masked
  const int rep = a.H / a.Hkv, kvh = h / rep;
  const int ldq = (a.H + 2 * a.Hkv) * HD, ldo = a.ldo ? a.ldo : a.H * HD;
  const size_t slice = cell_index(a.mode, a.L, c);
  const float* base = static_cast<const float*>(a.qkv) + slice * a.M * ldq;
  const int row = qc * BQ + threadIdx.x;
  const bool valid = row < a.M;
  float q[HD], o[HD];
  const float scale = rsqrtf(static_cast<float>(HD));
#pragma unroll
  for (int i = 0; i < HD; ++i) {
    q[i] = valid ? base[static_cast<size_t>(row) * ldq + h * HD + i] * scale : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int last = min(kvlim, (qc + 1) * BQ);  // keys 0..last-1 can be seen by this block
  for (int k0 = 0; k0 < last; k0 += CK) {
    __syncthreads();
    for (int e = threadIdx.x; e < CK * HD; e += BQ) {
      const int r = e / HD, i = e % HD, kr = k0 + r;
      Kc[r][i] = kr < a.M ? base[static_cast<size_t>(kr) * ldq + (a.H + kvh) * HD + i] : 0.f;
      Vc[r][i] = kr < a.M ? base[static_cast<size_t>(kr) * ldq + (a.H + a.Hkv + kvh) * HD + i] : 0.f;
    }
    __syncthreads();
    if (!valid) continue;
    for (int r = 0; r < CK; ++r) {
      const int kr = k0 + r;
      if (kr > row || kr >= kvlim) break;
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < HD; ++i) sc = fmaf(q[i], Kc[r][i], sc);
      const float mn = fmaxf(m, sc);
      const float corr = expf(m - mn), p = expf(sc - mn);
      l = l * corr + p;
#pragma unroll
      for (int i = 0; i < HD; ++i) o[i] = o[i] * corr + p * Vc[r][i];
      m = mn;
    }
  }
  if (!valid) return;
  const size_t off = slice * a.M * ldo + static_cast<size_t>(row) * ldo + h * HD;
  const float inv = 1.f / l;
  if (a.out_lo) {  // split-operand mode: f16 high and low terms for the O projection
    __half* dst = static_cast<__half*>(a.out) + off;
#pragma unroll
    for (int i = 0; i < HD; ++i) {
      const float v = o[i] * inv;
      dst[i] = __float2half_rn(v);
      dst[i + a.out_lo] = __float2half_rn(lo_term<__half>(v));
    }
    return;
  }
  float* dst = static_cast<float*>(a.out) + off;
#pragma unroll
  for (int i = 0; i < HD; ++i) dst[i] = o[i] * inv;
}

template <int HD, typename OpT>
cudaError_t launch_mma(const AttnArgs& a, cudaStream_t st) {
  using S = AttnSmem<HD>;
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<HD, OpT>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::BYTES);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  dim3 grid((a.M + S::BQ - 1) / S::BQ, a.H, a.G);
  const cudaError_t e = launch_pdl(attn_mma_kernel<HD, OpT>, grid, dim3(128), S::BYTES, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int HD>
cudaError_t launch_f32(const AttnArgs& a, cudaStream_t st) {
  dim3 grid((a.M + 63) / 64, a.H, a.G);
  const cudaError_t e = launch_pdl(attn_f32_kernel<HD>, grid, dim3(64), 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int HD>
cudaError_t launch_typed(const AttnArgs& a, ElemType t, cudaStream_t st) {
  switch (t) {
    case kElemF32: return launch_f32<HD>(a, st);
    case kElemBF16: return launch_mma<HD, __nv_bfloat16>(a, st);
    case kElemF16: return launch_mma<HD, __half>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, ElemType t, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.Hkv <= 0 || a.H % a.Hkv != 0 || (a.out_lo && t != kElemF32)) return cudaErrorInvalidValue;
  switch (a.dh) {
    case 32: return launch_typed<32>(a, t, st);
    case 64: return launch_typed<64>(a, t, st);
    case 128: return launch_typed<128>(a, t, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rmt

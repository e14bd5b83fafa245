// Segment-local causal attention on 5th-generation tensor cores (sm_100a), bf16 in, fp32
// accumulate and softmax; head_dim 64 or 128.
//
// Each (layer, segment) cell attends only within its own M = seg + n_mem rows (causal,
// diagonal included); query head h reads key/value head h / (H / Hkv). No key or value
// crosses a segment: across segments the model carries state only through its
// associative memory (arXiv 2506.05229 abstract: recurrent memory transformers process
// the input segment by segment).
//
// CTA = 128 query rows of one head of one cell; key/value tiles of 128 rows.
//   warp 0      one thread: TMA loads of the Q tile (once), K tiles (1 stage), V tiles (2 stages);
//   warp 1      TMEM allocation; one thread issues S = Q K^T (M=128, N=128) into TMEM and
//               O += P V (M=128, N=head_dim, V read MN-major) into a second TMEM range;
//   warps 2-5   softmax, one query row per thread: read S from TMEM, scale and mask, keep
//               the running max and sum in registers, write P (bf16) to shared memory in
//               the 128-byte-swizzled K-major layout of an MMA operand; finally read O,
//               divide by the row sum and store.
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
  static constexpr int SUB = 128 * 64 * 2;  // one 128-row x 64-column bf16 swizzled block
  static constexpr int NSUB = HD / 64;      // blocks per Q / K / V tile
  static constexpr int TILE = NSUB * SUB;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;      // one stage: K_{j+1} is needed only after softmax j starts
  static constexpr int V_OFF = K_OFF + TILE;      // two stages: V_{j+1} lands while P.V_j runs
  static constexpr int P_OFF = V_OFF + 2 * TILE;  // 128 x 128 bf16: two blocks
  static constexpr int BAR_OFF = P_OFF + 2 * SUB;
  static constexpr int NBAR = 12;
  static constexpr int SMEM = 1024 + BAR_OFF + NBAR * 8 + 16;
  static constexpr int TMEM_COLS = 256;  // S: columns 0..127, O: 128 .. 128+HD-1
};

enum : int { kQFull = 0, kKFull = 1, kKEmpty = 2, kVFull = 3, kVEmpty = 5, kSFull = 7, kSFree = 8, kPReady = 9,
             kOReady = 10, kDrain = 11 };

// 2^x on the special-function unit (relative error ~2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

template <int HD, typename OpT>
__global__ void __launch_bounds__(192, HD == 64 ? 2 : 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  using C = TaCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = sm100::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + C::BAR_OFF + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int nqt = (a.M + 127) / 128;
  const int qt = nqt - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int h = blockIdx.y;
  const Cell c = a.cells[blockIdx.z];
  const int kvh = h / (a.H / a.Hkv);
  const int slice = cell_index(a.mode, a.L, c);
  const int xq = h * HD, xk = (a.H + kvh) * HD, xv = (a.H + a.Hkv + kvh) * HD;
  const int n = qt + 1;  // key/value tiles 0..qt hold every key a row of this tile may see
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    sm100::mbar_init(bar(kQFull), 1);
    sm100::mbar_init(bar(kKFull), 1);
    sm100::mbar_init(bar(kKEmpty), 1);
    sm100::mbar_init(bar(kVFull), 1);
    sm100::mbar_init(bar(kVFull + 1), 1);
    sm100::mbar_init(bar(kVEmpty), 1);
    sm100::mbar_init(bar(kVEmpty + 1), 1);
    sm100::mbar_init(bar(kSFull), 1);
    sm100::mbar_init(bar(kSFree), 128);
    sm100::mbar_init(bar(kPReady), 128);
    sm100::mbar_init(bar(kOReady), 1);
    sm100::mbar_init(bar(kDrain), 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
    sm100::fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) sm100::tma_prefetch_desc(&tm);
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), C::TMEM_COLS);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int jk = -1, jv = -1;  // last K and V tiles whose loads were issued
      sm100::mbar_arrive_expect_tx(bar(kQFull), C::TILE);
      for (int sb = 0; sb < C::NSUB; ++sb)
        sm100::tma_load_3d(base + C::Q_OFF + sb * C::SUB, &tm, xq + 64 * sb, qt * 128, slice, bar(kQFull));
      for (int j = 0; j < n; ++j) {
        if (!sm100::mbar_wait(bar(kKEmpty), (j & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        sm100::mbar_arrive_expect_tx(bar(kKFull), C::TILE);
        for (int sb = 0; sb < C::NSUB; ++sb)
          sm100::tma_load_3d(base + C::K_OFF + sb * C::SUB, &tm, xk + 64 * sb, j * 128, slice, bar(kKFull));
        jk = j;
        const int st = j & 1;
        if (!sm100::mbar_wait(bar(kVEmpty + st), ((j >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        sm100::mbar_arrive_expect_tx(bar(kVFull + st), C::TILE);
        for (int sb = 0; sb < C::NSUB; ++sb)
          sm100::tma_load_3d(base + C::V_OFF + st * C::TILE + sb * C::SUB, &tm, xv + 64 * sb, j * 128, slice,
                             bar(kVFull + st));
        jv = j;
      }
      if (!ok) {
        if (a.err) atomicOr(a.err, kErrTimeoutProducer);
        sm100::mbar_wait_drain(bar(kQFull), 0);
        if (jk >= 0) sm100::mbar_wait_drain(bar(kKFull), jk & 1);
        for (int j = jv; j >= 0 && j >= jv - 1; --j) sm100::mbar_wait_drain(bar(kVFull + (j & 1)), (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t tS = tmem_base, tO = tmem_base + 128;
      constexpr uint32_t idS = sm100::idesc_f32acc(128, 128, OpFormat<OpT>::value);
      constexpr uint32_t idO = sm100::idesc_f32acc_bmn(128, HD, OpFormat<OpT>::value);
      bool ok = sm100::mbar_wait(bar(kQFull), 0, abort_flag);
      auto issue_s = [&](int j) -> bool {
        if (!sm100::mbar_wait(bar(kKFull), j & 1, abort_flag)) return false;
        sm100::tc_fence_after();
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const int sb = k >> 2, kk = k & 3;
          const uint64_t ad = sm100::smem_desc_k128(base + C::Q_OFF + sb * C::SUB) + 2ull * kk;
          const uint64_t bd = sm100::smem_desc_k128(base + C::K_OFF + sb * C::SUB) + 2ull * kk;
          sm100::mma_bf16(tS, ad, bd, idS, k > 0);
        }
        sm100::mma_commit(bar(kSFull));
        sm100::mma_commit(bar(kKEmpty));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) {
          if (!sm100::mbar_wait(bar(kSFree), j & 1, abort_flag) || !issue_s(j + 1)) {
            ok = false;
            break;
          }
        }
        const int vs = j & 1;
        if (!sm100::mbar_wait(bar(kPReady), j & 1, abort_flag) ||
            !sm100::mbar_wait(bar(kVFull + vs), (j >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
#pragma unroll
        for (int k = 0; k < 128 / 16; ++k) {
          const uint64_t ad = sm100::smem_desc_k128(base + C::P_OFF + (k >> 2) * C::SUB) + 2ull * (k & 3);
          const uint64_t bd = sm100::smem_desc_mn128(base + C::V_OFF + vs * C::TILE + k * 2048, C::SUB);
          sm100::mma_bf16(tO, ad, bd, idO, (j > 0 || k > 0));
        }
        sm100::mma_commit(bar(kOReady));
        sm100::mma_commit(bar(kVEmpty + vs));
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
    const int qrow = qt * 128 + r;
    const uint32_t loff = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem_base + loff, tO = tmem_base + loff + 128;
    const float sl2 = rsqrtf(static_cast<float>(HD)) * 1.4426950408889634f;  // 1/sqrt(dh) * log2(e)
    uint8_t* P = smem + C::P_OFF;
    float m_use = 0.f, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, sm100::mbar_wait(bar(kSFull), j & 1, abort_flag));
      if (!ok) break;
      sm100::tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) sm100::tmem_ld32(tS + 32 * q4, s[q4]);
      sm100::tmem_wait_ld();
      sm100::tc_fence_before();
      sm100::mbar_arrive(bar(kSFree));
      const int k0 = j * 128;
      const bool need_mask = (j == qt) || (k0 + 128 > a.M);
      // causal mask (and the cell's ragged end) only on the tiles that need it
      if (need_mask) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kv = k0 + 32 * q4 + i;
            if (kv > qrow || kv >= a.M) s[q4][i] = __float_as_uint(-INFINITY);
          }
        }
      }
      // row max and row sum over 4 independent partials (short dependency chains)
      float mxp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
        for (int i = 0; i < 32; ++i) mxp[i & 3] = fmaxf(mxp[i & 3], u2f(s[q4][i]));
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
      float sp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = ex2(fmaf(u2f(s[q4][i]), sl2, -m_use));
          sp[i & 3] += p;
          s[q4][i] = __float_as_uint(p);
        }
      }
      const float sum = (sp[0] + sp[1]) + (sp[2] + sp[3]);
      l = l * corr + sum;
      if (j > 0) {
        // P of tile j-1 must be consumed (and O final for it) before P and O change
        ok = __all_sync(0xffffffffu, sm100::mbar_wait(bar(kOReady), (j - 1) & 1, abort_flag));
        if (!ok) break;
        sm100::tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int oc = 0; oc < HD / 32; ++oc) {
            uint32_t o[32];
            sm100::tmem_ld32(tO + 32 * oc, o);
            sm100::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(u2f(o[i]) * corr);
            sm100::tmem_st32(tO + 32 * oc, o);
          }
          sm100::tmem_wait_st();
        }
      }
      // P row r -> two 128 x 64 swizzled blocks: 16-byte chunk cc of a row lands at cc ^ (r % 8)
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int q4 = ch >> 2, i0 = (ch & 3) * 8;
        const uint4 w = make_uint4(pack2<OpT>(u2f(s[q4][i0]), u2f(s[q4][i0 + 1])),
                                   pack2<OpT>(u2f(s[q4][i0 + 2]), u2f(s[q4][i0 + 3])),
                                   pack2<OpT>(u2f(s[q4][i0 + 4]), u2f(s[q4][i0 + 5])),
                                   pack2<OpT>(u2f(s[q4][i0 + 6]), u2f(s[q4][i0 + 7])));
        *reinterpret_cast<uint4*>(P + (ch >> 3) * C::SUB + r * 128 + (((ch & 7) ^ (r & 7)) << 4)) = w;
      }
      sm100::fence_async_smem();
      sm100::tc_fence_before();
      sm100::mbar_arrive(bar(kPReady));
    }
    if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(bar(kOReady), (n - 1) & 1, abort_flag));
    if (ok) {
      sm100::tc_fence_after();
      const float inv = 1.f / l;
      const int ldo = a.H * HD;
      OpT* dst = static_cast<OpT*>(a.out) + (static_cast<size_t>(slice) * a.M + qrow) * ldo + h * HD;
#pragma unroll 1
      for (int oc = 0; oc < HD / 32; ++oc) {
        uint32_t o[32];
        sm100::tmem_ld32(tO + 32 * oc, o);
        sm100::tmem_wait_ld();
        if (qrow < a.M) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = u2f(o[i]) * inv;
          store32_16(dst + 32 * oc, v);
        }
      }
    } else if (lane == 0 && a.err) {
      atomicOr(a.err, kErrTimeoutEpilogue);
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int HD, typename OpT>
cudaError_t launch_hd(const CUtensorMap& tm, const AttnArgs& a, cudaStream_t st) {
  using C = TaCfg<HD>;
  static bool attr[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<HD, OpT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  dim3 grid((a.M + 127) / 128, a.H, a.G);
  attn_tc_kernel<HD, OpT><<<grid, 192, C::SMEM, st>>>(tm, a);
  return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(int dh) { return dh == 64 || dh == 128; }

cudaError_t launch_attention_tc(const CUtensorMap& tm_qkv, const AttnArgs& a, bool f16, cudaStream_t st) {
  if (a.G <= 0 || a.M <= 0) return cudaSuccess;
  if (a.Hkv <= 0 || a.H % a.Hkv != 0) return cudaErrorInvalidValue;
  if (a.dh == 64) return f16 ? launch_hd<64, __half>(tm_qkv, a, st) : launch_hd<64, __nv_bfloat16>(tm_qkv, a, st);
  if (a.dh == 128) return f16 ? launch_hd<128, __half>(tm_qkv, a, st) : launch_hd<128, __nv_bfloat16>(tm_qkv, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace rmt

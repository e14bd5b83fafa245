// Internal launcher interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

#include "common.cuh"

namespace rmt {

// Launch `kernel` on `st` with programmatic stream serialization (see pdl_wait in
// common.cuh): the kernel may be scheduled while the previous one finishes, and it must call
// pdl_wait() before touching data other kernels produce.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Element type of a buffer handed to a kernel.
enum ElemType : int { kElemF32 = 0, kElemBF16 = 1, kElemF16 = 2 };

// ------------------------------------------------------------------ grouped GEMMs
// Group g computes rows 0..M-1 of cell cells[g]: Y = X . W^T with
//   X = slice cell_index(a_mode, cells[g]) of a [*, M, K] stack,
//   W = slice cells[g].l of a [L, N, K] stack.
struct TcGemmArgs {
  int M, N, K;
  int G;
  const Cell* cells;  // device array of G cells
  int L;
  IndexMode a_mode;
  EpiKind epi;
  EpiParams ep;
  int* err;  // device error word (may be null)
  // split-operand mode: the X operand holds each row's high terms in columns 0..K-1 and its
  // low terms from column kx_lo on; the GEMM runs 2K/64 blocks, block b reading X at column
  // (b mod K/64) * 64 + (b div K/64) * kx_lo and W at (b mod K/64) * 64 (0: K blocks)
  int kx_lo;
  // CTA-pair kernel: tokens per tile (a multiple of 16, at most 256; the activation maps' box
  // is nt / 2 rows); 0: pair_token_tile(M). In a chained launch phase 0's value holds for all.
  int nt;
};

// tensor-core path: 16-bit operands (f16 or bf16, one type per launch) in TMA tensor maps
// As make_tmap_16_3d over a [depth][rows][inner] view whose rows are row_stride elements apart
// (row_stride >= inner, a multiple of 8; base 16-byte aligned).
bool make_tmap_16_3d_strided(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                             uint64_t row_stride, uint32_t box_rows, bool f16);
bool make_tmap_16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                     uint32_t box_rows, bool f16);
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                       uint32_t box_rows);
int tc_pick_bn(int N, int epi, int head_dim);  // 0 if no tile width fits
// Residual-stream map for the residual epilogues: fp32 [depth, rows, inner], 32 x 32 boxes.
bool make_tmap_f32_resid(CUtensorMap* map, const float* base, uint64_t inner, uint64_t rows, uint64_t depth);
// f16: operands (and 16-bit epilogue outputs) are f16, else bf16. tx: the residual-stream map
// (read and written by the residual epilogues; any valid map otherwise).
cudaError_t launch_tc_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tx, const TcGemmArgs& args,
                           int bn, bool f16, cudaStream_t st);

// CTA-pair path (features along M, tokens along N): tw maps the [L, N, K] weights with
// 128-row boxes, tx the [*, M, K] activations with pair_token_tile(M)/2-row boxes. RoPE and
// SwiGLU expect the pair packing described with pair_token_tile.
bool tc_pair_supported(int M, int N, int K, int epi, int head_dim);
// Token tile of a CTA-pair launch over G cells of M rows whose phases have `pairs` 256-row
// feature pairs in all: pair_token_tile(M), or kPairFineTile when a launch of few tiles
// finishes sooner in more, smaller ones (fewer rounds of the resident CTA pairs; each tile
// also costs a fixed pipeline fill and drain).
constexpr int kPairFineTile = 128;
int pair_pick_nt(int M, long G, long pairs);
cudaError_t launch_tc_pair_gemm(const CUtensorMap& tw, const CUtensorMap& tx, const TcGemmArgs& args, bool f16,
                                cudaStream_t st);

// Several projections of the same cells in one CTA-pair launch ("phases", run in order; see
// tc_gemm_pair.cu): phase p >= 1 of (cell g, token tile tt) starts once every tile of phase p-1
// for those tokens is stored, which a counter per (phase, cell, token tile) in global memory
// records (one increment per epilogue warp and tile). The counters of one launch sit in block `parity` of ctr, laid out
// [2 parities][kMaxPhases - 1][ctr_len] with ctr_len >= G * token tiles; the launch zeroes the
// other parity's block for the next launch, so consecutive launches alternate the parity and
// the buffer starts zeroed.
constexpr int kMaxPhases = 3;
struct PairChainArgs {
  TcGemmArgs ph[kMaxPhases];  // per phase; M, G, cells, L and err are phase 0's for all
  int nphase;
  unsigned* ctr;
  int ctr_len;
  int parity;
};
// The O projection, gate/up and down of one diagonal in one launch (f16 operands): tw / tx hold
// each phase's weight and activation maps, as launch_tc_pair_gemm takes them.
cudaError_t launch_tc_pair_chain_o_mlp(const CUtensorMap* tw, const CUtensorMap* tx, const PairChainArgs& args,
                                       cudaStream_t st);

// fp32 FMA path (fp32 operands by pointer)
struct SimtGemmArgs {
  int M, N, K;
  int G;
  const Cell* cells;
  int L;
  const float* a;  // [*, M, lda]
  int lda;
  IndexMode a_mode;
  const float* w;  // [L, N, K]
  EpiKind epi;
  EpiParams ep;
};
cudaError_t launch_simt_gemm(const SimtGemmArgs& args, cudaStream_t st);

// ------------------------------------------------------------------ attention
// qkv: [*, M, (H + 2 Hkv) dh] slice by layer; out: [*, M, H dh] slice by layer.
struct AttnArgs {
  const void* qkv;
  void* out;
  int M, H, Hkv, dh;
  int G;
  const Cell* cells;
  IndexMode mode;  // slice index of both buffers
  int L;
  int* err;        // device error word for bounded waits (tensor-core kernel), may be null
  int ldo;         // row stride of out in elements (0: H * dh, rows packed)
  // fp32 kernel only: write out as f16 high terms and, out_lo elements further, low terms
  // (split-operand mode; 0: fp32 out)
  int out_lo;
  // filled in by launch_attention_tc: rows of the stacked last query tile (0: not stacked,
  // see attn_pack_tail), H / Hkv, and the work items of the last query tile
  int tail_rows, group, n_tail;
};
// mma.sync (bf16) or fp32 FMA kernels, any head_dim in {32, 64, 128}
cudaError_t launch_attention(const AttnArgs& a, ElemType t, cudaStream_t st);
// The last 128-row query tile of a cell holds rem = M - 128 (ceil(M / 128) - 1) rows. When the
// H / Hkv query heads of one key/value group fit in a single 128-row tile there, and rem is a
// multiple of 8 (so that each head's rows start on a 1024-byte swizzle atom), the tcgen05 kernel
// stacks them: query head kvh * H / Hkv + i at tile rows i * rem .. i * rem + rem - 1, one work
// item per group instead of one per head.
__host__ __device__ inline int attn_tail_rows(int M) { return M - ((M + 127) / 128 - 1) * 128; }
__host__ __device__ inline bool attn_pack_tail(int M, int H, int Hkv) {
  const int rem = attn_tail_rows(M), gq = Hkv > 0 ? H / Hkv : 0;
  return gq >= 2 && rem % 8 == 0 && rem * gq <= 128;
}
// Box height of the tail map: rem when the tail is stacked, else the 128-row tile
inline uint32_t attn_tail_box(int M, int H, int Hkv) {
  return attn_pack_tail(M, H, Hkv) ? static_cast<uint32_t>(attn_tail_rows(M)) : 128u;
}
// tcgen05 kernel (16-bit, head_dim 64 or 128): tm_qkv maps qkv as [*, M, (H+2Hkv)dh] with box
// 64 x 128; tm_tail maps the same tensor with box 64 x attn_tail_box(M, H, Hkv)
bool attention_tc_supported(int dh);
cudaError_t launch_attention_tc(const CUtensorMap& tm_qkv, const CUtensorMap& tm_tail, const AttnArgs& a, bool f16,
                                cudaStream_t st);

// ------------------------------------------------------------------ associative memory
struct MemReadArgs {
  const float* q;  // [*, M, dk] raw (before phi)
  const float* A;  // [*, dk, dv]
  const float* z;  // [*, dk]
  void* o;         // [*, M, dv]
  int M, dk, dv;
  float eps;
  int G;
  const Cell* cells;
  IndexMode mode;        // slice of q and o
  IndexMode state_mode;  // slice of A and z
  int L;
  int ldo;     // row stride of o in elements (0: dv)
  int lo_off;  // tcgen05 read, split-operand mode: low terms of o lo_off elements after the high terms (0: none)
};
// 16-bit outputs take the tcgen05 read when it supports d_k (err: its bounded waits' error word,
// may be null), else the mma.sync read; fp32 outputs the fp32 FMA read
cudaError_t launch_mem_read(const MemReadArgs& a, ElemType out_type, cudaStream_t st, int* err = nullptr);
// tcgen05 read for 16-bit outputs with d_k of 64 or 128 (memory_tc.cu); err: error word of the
// bounded waits (may be null)
bool mem_read_tc_supported(int dk, int dv);
cudaError_t launch_mem_read_tc(const MemReadArgs& a, bool f16, int* err, cudaStream_t st);

// Partial products of the memory-token rows with [W_mk; W_mv], split along d_model so the
// reduction order is fixed: part[l][split][r][j] = sum_{k in split} Y[r][k] W_mkv[l][j][k],
// Y = rows row0 .. row0+n-1 of the cell's output slot; the update adds the splits in order.
constexpr int kMemKvSplit = 128;  // d_model columns per split
inline int mem_kv_splits(int d, bool /*bf16*/) { return (d + kMemKvSplit - 1) / kMemKvSplit; }
struct MemKvArgs {
  const float* x;  // [*, M, d] fp32: the residual stream slots (forward) or caller rows
  int M, d, n;     // the n rows read are the cell's last n valid rows (cell_rows(c, M) - n ..)
  IndexMode x_mode;  // slice of x holding the cell's rows (kOutSlot in the forward)
  const void* w;   // [L, dkv, d] in T
  float* part;     // [L, nsplit, n, dkv] fp32
  int dkv;
  int G;
  const Cell* cells;
  int L;
};
// Launches of many cells (at least four per SM, bf16 weights, n <= 16) write whole sums instead: one
// split, [L, 1, n, dkv], each element the sum of the partials above in split order (the same
// bits the update forms from them). The update then takes nsplit = 1.
bool mem_kv_whole(int G, int n, bool bf16);
inline int mem_kv_written_splits(int G, int n, int d, bool bf16) {
  return mem_kv_whole(G, n, bf16) ? 1 : mem_kv_splits(d, bf16);
}
cudaError_t launch_mem_kv(const MemKvArgs& a, bool bf16, cudaStream_t st);

// Delta-rule update of A, z from raw keys/values of n rows. Keys/values come either from
// the split partials above (part != null: k = columns 0..dk-1, v = columns dk..dk+dv-1 of
// the reduced rows) or from plain arrays k [*, n, dk], v [*, n, dv].
struct MemUpdateArgs {
  const float* part;  // [*, nsplit, n, dk + dv] or null
  int nsplit;
  const float* k;     // [*, n, dk] (when part == null)
  const float* v;     // [*, n, dv]
  float* A;           // [*, dk, dv]
  float* z;           // [*, dk]
  int n, dk, dv;
  float eps;
  int G;
  const Cell* cells;
  IndexMode kv_mode, state_mode;
  int L;
  int* trace;         // optional: trace[3*(trace_base+g) + {0,1,2}] = (step, l, s)
  int trace_base, step;
  // 0: every row is written against the pre-update A, z (batched). 1: the rows are written one
  // after another, each against the state the earlier rows left (per-token delta rule).
  int seq;
};
cudaError_t launch_mem_update(const MemUpdateArgs& a, cudaStream_t st);

// ------------------------------------------------------------------ row kernels
struct RmsArgs {
  const float* x;  // [*, M, d] fp32
  const void* g;   // [L, d] in T
  void* y;         // [*, M, d] in T
  int M, d;
  float eps;
  int G;
  const Cell* cells;
  IndexMode x_mode, y_mode;
  int L;
};
cudaError_t launch_rmsnorm(const RmsArgs& a, bool bf16, cudaStream_t st);

// W[l][n][k] *= g[l][k] for l < L (an RMSNorm gain folded into the next projection).
// W and g share the model's storage type (f32 or bf16), or W is f16 and g bf16 (w_f16).
cudaError_t launch_scale_cols(void* w, const void* g, int L, int N, int K, bool bf16, bool w_f16, cudaStream_t st);
// In-place bf16 -> f16 conversion of n elements (the values of a bf16 weight as f16 operands).
cudaError_t launch_bf16_to_f16(void* p, size_t n, cudaStream_t st);
// Layer-0 inputs of the G cells (all of layer 0): in slot c.xin of x (and of xb, if given),
// rows 0..m-n_mem-1 from emb rows c.t0.., rows m-n_mem..m-1 from the memory tokens, rows
// m..M-1 zero (m = cell_rows(c, M)). An f16 copy that overflows sets kErrF16Range in *err.
// split: xb rows are 2d wide, the high terms then the low terms (split-operand mode).
cudaError_t launch_assemble(const Cell* cells, int G, const void* emb, const void* mem, float* x, __half* xb, int M,
                            int n_mem, int d, bool bf16, int* err, cudaStream_t st, bool split = false);
// RMSNorm statistics of rows 0..M-1 of an fp32 [M, d] block: ss[row * parts + b] = sum of
// squares of columns b*w .. b*w+w-1, w = d / parts (a multiple of 4; at most 32 parts).
// One CTA waits on an mbarrier nothing signals, with the kernels' bounded wait limited to
// limit_ns, and ORs kErrTimeoutSelftest into *err when the wait gives up (see selftest.cu).
cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t st);
#ifdef RMT_DEBUG
// Debug build: one thread passes load_cell a cell with an out-of-range slot; kErrBounds must
// reach *err (and kErrBadArgs too if the returned cell is not the in-range substitute).
cudaError_t launch_bounds_selftest(int* err, cudaStream_t st);
#endif
cudaError_t launch_row_ssq(const float* x, float* ss, int M, int d, int parts, cudaStream_t st);
// Segment outputs of the G cells: rows 0..m-n_mem-1 of slot c.xout, cast to T, to out rows c.t0...
cudaError_t launch_emit(const Cell* cells, int G, const float* x, void* out, int M, int n_mem, int d, bool bf16,
                        cudaStream_t st);

}  // namespace rmt

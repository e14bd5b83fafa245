// C ABI of the diagonal-batched ARMT prefill library: handle, weight packing, the host
// scheduler and the launch sequence of one schedule step.
//
// Scheduler ("Implementation" of the diagonal-batching skill page): the (layer, segment)
// grid is swept in anti-diagonals d = l + s, cells of a diagonal in ascending layer order,
// d = 0 .. L+S-2; the layers on diagonal d are max(0, d-S+1) .. min(d, L-1). The
// sequential schedule runs one cell per step, segments outermost. Either way one step is
// the same fixed launch sequence over the step's cells (a cell table on the device):
//   [layer-0 input] -> mem-q GEMM -> memory read -> mem-o GEMM (+residual) -> RMSNorm
//   -> QKV GEMM (+RoPE) -> attention -> O GEMM (+residual) -> RMSNorm
//   -> gate/up GEMM (+SwiGLU) -> down GEMM (+residual) -> memory k/v -> memory update
//   -> [segment output]
// The RMSNorms launch nothing (statistics from the residual epilogues, gains folded into the
// next weights). In bf16 mode with d_k = d_v = 64 the read runs in the mem-q GEMM's
// epilogue, and with the O GEMM on CTA pairs the mem-o residual add moves into the O GEMM
// (fold_mo), so a step is nine launches.
// Each kernel does the same arithmetic for a cell whatever else shares its launch, so the
// two schedules give identical bits ("Dependency Preservation" in "Architecture
// Overview"; arXiv 2506.05229 abstract: a pure run-time reordering with exact recurrence).
#include <algorithm>
#include <climits>
#include <cstdio>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <deque>
#include <map>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "launch.h"
#include "rmt.h"

using namespace rmt;

namespace {

thread_local std::string g_last_error;

rmt_status fail(rmt_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

#define RMT_CUDA(call)                                                                             \
  do {                                                                                             \
    cudaError_t e_ = (call);                                                                       \
    if (e_ != cudaSuccess) return fail(RMT_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_host_ptr(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return true;
  }
  return attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged;
}

// Page-locked (or registered) host memory: asynchronous copies from and to it overlap kernels.
bool is_pinned_host_ptr(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeHost;
}

struct Table {
  std::vector<Cell> cells;  // host copy, execution order
  std::vector<int> off, cnt;
  // per step: its first n_first cells are of layer 0 (assembled from the embeddings) and its
  // last n_last cells of layer L-1 (emitted)
  std::vector<int> n_first, n_last;
  std::vector<int> seg_base;  // per sequence: ordinal of its first segment among all segments
  Cell* dev = nullptr;
};

// Execution order of the cells (b, l, s) of a batch, sequence b having S[b] segments.
// Diagonal: step d holds every cell with l + s = d, in ascending layer and, within a layer,
// ascending sequence; steps with no cell are skipped. Sequential: one cell per step,
// sequences outermost, then segments, then layers. Only l, s and b are set.
void order_cells(int L, const std::vector<int>& S, rmt_schedule sch, Table& t) {
  t.cells.clear();
  t.off.clear();
  t.cnt.clear();
  t.n_first.clear();
  t.n_last.clear();
  const int B = static_cast<int>(S.size());
  int smax = 0;
  for (int sb : S) smax = sb > smax ? sb : smax;
  auto push_step = [&](size_t begin) {
    const int n = static_cast<int>(t.cells.size() - begin);
    int nf = 0, nl = 0;
    while (nf < n && t.cells[begin + nf].l == 0) ++nf;
    while (nl < n && t.cells[t.cells.size() - 1 - nl].l == L - 1) ++nl;
    t.off.push_back(static_cast<int>(begin));
    t.cnt.push_back(n);
    t.n_first.push_back(nf);
    t.n_last.push_back(nl);
  };
  if (sch == RMT_DIAGONAL) {
    for (int d = 0; d <= L + smax - 2; ++d) {
      const size_t begin = t.cells.size();
      for (int l = 0; l < L && l <= d; ++l)
        for (int b = 0; b < B; ++b)
          if (d - l < S[b]) t.cells.push_back(Cell{l, d - l, b, 0, 0, 0, 0, 0});
      if (t.cells.size() > begin) push_step(begin);
    }
  } else {
    for (int b = 0; b < B; ++b)
      for (int s = 0; s < S[b]; ++s)
        for (int l = 0; l < L; ++l) {
          const size_t begin = t.cells.size();
          t.cells.push_back(Cell{l, s, b, 0, 0, 0, 0, 0});
          push_step(begin);
        }
  }
}

// The full cell table of a batch whose sequence b holds T[b] tokens (packed one after
// another): ceil(T[b] / seg) segments, the last one possibly short.
void build_table(int L, int seg, int n_mem, const std::vector<int>& T, rmt_schedule sch, Table& t) {
  std::vector<int> S(T.size()), base(T.size());
  t.seg_base.assign(T.size(), 0);
  int rows = 0, segs = 0;
  for (size_t b = 0; b < T.size(); ++b) {
    S[b] = (T[b] + seg - 1) / seg;
    base[b] = rows;
    t.seg_base[b] = segs;
    rows += T[b];
    segs += S[b];
  }
  order_cells(L, S, sch, t);
  for (Cell& c : t.cells) {
    const int tokens = T[c.b] - c.s * seg;
    c.m = (tokens < seg ? tokens : seg) + n_mem;
    c.k = c.b * L + c.l;
    c.xin = c.b * n_slots(L) + in_slot(L, c.l, c.s);
    c.xout = c.b * n_slots(L) + out_slot(L, c.l, c.s);
    c.t0 = base[c.b] + c.s * seg;
  }
}

// Identity cell table (g, 0), g = 0..n-1, for the kernel-level entry points.
struct DeviceScratch {
  Cell* cells = nullptr;
  int cap = 0;
  int* err = nullptr;
};
DeviceScratch g_dev_scratch[64];

rmt_status device_scratch(int G, const Cell** cells, int** err) {
  int dev = 0;
  RMT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RMT_EINVAL, "device index out of range");
  DeviceScratch& s = g_dev_scratch[dev];
  if (!s.err) {
    RMT_CUDA(cudaMalloc(&s.err, sizeof(int)));
    RMT_CUDA(cudaMemset(s.err, 0, sizeof(int)));
  }
  if (G > s.cap) {
    const int cap = G > 4096 ? G : 4096;
    std::vector<Cell> h(cap);
    for (int g = 0; g < cap; ++g) h[g] = identity_cell(g);
    Cell* p = nullptr;
    if (cudaMalloc(&p, sizeof(Cell) * cap) != cudaSuccess) return fail(RMT_ENOMEM, "cell table allocation failed");
    RMT_CUDA(cudaMemcpy(p, h.data(), sizeof(Cell) * cap, cudaMemcpyHostToDevice));
    if (s.cells) cudaFree(s.cells);
    s.cells = p;
    s.cap = cap;
  }
  *cells = s.cells;
  if (err) *err = s.err;
  return RMT_OK;
}

// Split-K partial sums of rmt_memory_write, grown on demand (one buffer per device).
struct PartialScratch {
  float* p = nullptr;
  size_t cap = 0;
};
PartialScratch g_part_scratch[64];

rmt_status partial_scratch(size_t floats, float** out) {
  int dev = 0;
  RMT_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(RMT_EINVAL, "device index out of range");
  PartialScratch& s = g_part_scratch[dev];
  if (floats > s.cap) {
    float* p = nullptr;
    if (cudaMalloc(&p, floats * sizeof(float)) != cudaSuccess) return fail(RMT_ENOMEM, "scratch allocation failed");
    if (s.p) cudaFree(s.p);
    s.p = p;
    s.cap = floats;
  }
  *out = s.p;
  return RMT_OK;
}

}  // namespace

namespace rmt {
// Lets other translation units of the library report through rmt_last_error().
void set_last_error(const std::string& msg) { g_last_error = msg; }
}  // namespace rmt

struct rmt_handle {
  rmt_cfg cfg{};
  int dev = 0;
  bool bf16 = false;
  // RMT_BF16_SPLIT: every f16 activation operand is stored as high and low terms side by side
  // in one row ([hi | lo], twice the width), each tensor-core GEMM reads 2K columns against
  // its K weight columns, q/k/v stay fp32 and attention runs on the fp32 kernel
  bool split = false;
  int M = 0, es = 4, Nqkv = 0, nsplit = 0;
  // packed weights (cfg dtype)
  void *w_qkv = nullptr, *w_o = nullptr, *w_gu = nullptr, *w_d = nullptr, *w_mq = nullptr, *w_mo = nullptr,
       *w_mkv = nullptr, *g1 = nullptr, *g2 = nullptr, *memtok = nullptr;
  // activations and state
  float* x = nullptr;
  __half* xb = nullptr;  // bf16 mode: f16 operand copy of the residual stream
  void *qkv = nullptr, *att = nullptr, *u = nullptr, *om = nullptr;
  float *qm = nullptr, *part = nullptr, *A = nullptr, *z = nullptr;
  float *ss1 = nullptr, *ss2 = nullptr;  // per-row sums of squares for the folded RMSNorms
  int ss_parts = 0;
  float2* rope = nullptr;
  __half2* rope_h = nullptr;  // (cos, sin) as f16 pairs for the tensor-core RoPE epilogue
  int* err = nullptr;
  int* trace = nullptr;
  size_t trace_cap = 0;
  int traced_cells = -1;
  void* emb_stage = nullptr;
  size_t emb_stage_bytes = 0;
  void* out_stage = nullptr;
  size_t out_stage_bytes = 0;
  // per-segment host<->device copies for page-locked host buffers, overlapped with the steps
  cudaStream_t h2d = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> copy_events;  // [0]: forward start, [1]: copies done, then 2 per segment
  bool copy_resources(size_t n_segments) {
    if (!h2d && cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (!d2h && cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) != cudaSuccess) return false;
    while (copy_events.size() < 2 + 2 * n_segments) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
      copy_events.push_back(e);
    }
    return true;
  }
  std::map<std::pair<std::vector<int>, int>, Table> tables;  // keyed by (token counts, schedule)
  std::deque<std::pair<std::vector<int>, int>> table_order;  // insertion order, for eviction
  static constexpr size_t kMaxTables = 64;
  CUtensorMap tm_xb, tm_om, tm_att, tm_u, tm_wqkv, tm_wo, tm_wgu, tm_wd, tm_wmq, tm_wmo, tm_qkv, tm_qkv_tail, tm_x,
      tm_rope;
  // activation maps of the CTA-pair GEMM (pair_token_tile(M)/2-row boxes), and the same with
  // kPairFineTile/2-row boxes for launches of few cells (pair_pick_nt)
  CUtensorMap tp_xb, tp_om, tp_att, tp_u, tq_xb, tq_om, tq_att, tq_u;
  int bn_mq = 0, bn_mo = 0, bn_qkv = 0, bn_o = 0, bn_gu = 0, bn_d = 0;
  // bf16 mode: projections that run on the CTA-pair GEMM (decided before packing, which
  // depends on it for the RoPE and SwiGLU row orders)
  bool pair_mo = false, pair_qkv = false, pair_o = false, pair_gu = false, pair_d = false;
  // bf16 mode with d_k = d_v = 64: the memory read runs in the mem-q GEMM's epilogue (the
  // query never goes to memory) and has no launch of its own
  bool fuse_read = false;
  // with fuse_read and the O projection on CTA pairs: the read-out o sits in d_v extra columns
  // of the attention output and W_mo in d_v extra columns of W_o, so the O projection adds
  // W_o att + W_mo o to the layer input in one accumulator; the read-out projection then only
  // forms the f16 operand copy and RMSNorm statistics of x + W_mo o (no fp32 store)
  bool fold_mo = false;
  int ld_att = 0;  // row stride of the attention output (n_heads * head_dim, + d_v with fold_mo)
  // bf16 mode with O, gate/up and down all on CTA pairs: the three run as one chained launch
  // per step (launch_tc_pair_chain_o_mlp), ordered per (cell, token tile) by counters in
  // global memory; the parity alternates from launch to launch
  bool chain_mlp = false;
  unsigned* chain_ctr = nullptr;
  int chain_ctr_len = 0, chain_parity = 0;
  std::vector<void*> allocs;
  // activations and memory state, sized for cap_b sequences (rmt_reserve)
  int cap_b = 0;
  std::vector<void*> act_allocs;
  // full-attention forward (rmt_full_attention_forward): one causal segment of up to full_cap
  // tokens, no memory; its own activations and tensor maps, allocated on first use
  int full_cap = 0, full_T = 0;
  std::vector<void*> full_allocs;
  float* fx = nullptr;     // [2][T][d] residual slots (layer l reads slot l % 2, writes the other)
  __half* fxb = nullptr;   // [2][T][d] f16 operand copies
  void *fqkv = nullptr, *fatt = nullptr, *fu = nullptr;
  float *fss1 = nullptr, *fss2 = nullptr;
  float2* frope = nullptr;
  __half2* frope_h = nullptr;
  Cell* fcells = nullptr;  // [L]: cell l = layer l of the one segment
  CUtensorMap fm_xb, fm_att, fm_u, fm_qkv, fm_qkv_tail, fm_x, fm_rope, fp_xb, fp_att, fp_u;
  // launch probe (rmt_probe): CUDA event pairs around the launches of the kinds in mask
  struct ProbeRec {
    int kind;
    double flops, bytes;
    cudaEvent_t a, b;
  };
  uint32_t probe_mask = 0;
  std::vector<cudaEvent_t> probe_pool;
  size_t probe_used = 0;
  std::vector<ProbeRec> probe_recs;
  int64_t launches = 0;

  cudaEvent_t probe_event() {
    if (probe_used == probe_pool.size()) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
      probe_pool.push_back(e);
    }
    return probe_pool[probe_used++];
  }

  void* alloc(size_t bytes) {
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    allocs.push_back(p);
    return p;
  }
  void* act_alloc(size_t bytes) {
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    act_allocs.push_back(p);
    return p;
  }
  void free_acts() {
    for (void* p : act_allocs) cudaFree(p);
    act_allocs.clear();
    cap_b = 0;
    x = nullptr;
    xb = nullptr;
    qkv = att = u = om = nullptr;
    qm = part = A = z = ss1 = ss2 = nullptr;
    chain_ctr = nullptr;
  }
  void free_full() {
    for (void* p : full_allocs) cudaFree(p);
    full_allocs.clear();
    full_cap = full_T = 0;
    fx = nullptr;
    fxb = nullptr;
    fqkv = fatt = fu = nullptr;
    fss1 = fss2 = nullptr;
    frope = nullptr;
    frope_h = nullptr;
    fcells = nullptr;
  }
  void release() {
    for (void* p : allocs) cudaFree(p);
    allocs.clear();
    free_acts();
    free_full();
    for (auto& kv : tables)
      if (kv.second.dev) cudaFree(kv.second.dev);
    tables.clear();
    table_order.clear();
    if (trace) cudaFree(trace);
    if (emb_stage) cudaFree(emb_stage);
    if (out_stage) cudaFree(out_stage);
    trace = nullptr;
    emb_stage = out_stage = nullptr;
    for (cudaEvent_t e : probe_pool) cudaEventDestroy(e);
    probe_pool.clear();
    for (cudaEvent_t e : copy_events) cudaEventDestroy(e);
    copy_events.clear();
    if (h2d) cudaStreamDestroy(h2d);
    if (d2h) cudaStreamDestroy(d2h);
    h2d = d2h = nullptr;
    probe_recs.clear();
    probe_used = 0;
  }
};

namespace {

bool validate_cfg(const rmt_cfg* c, std::string& why) {
  if (c->n_layers <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
      c->d_ff <= 0 || c->seg_len <= 0 || c->n_mem <= 0 || c->d_k <= 0 || c->d_v <= 0) {
    why = "all sizes must be positive";
    return false;
  }
  if (c->dtype != RMT_F32 && c->dtype != RMT_BF16 && c->dtype != RMT_BF16_SPLIT)
    return why = "dtype must be RMT_F32, RMT_BF16 or RMT_BF16_SPLIT", false;
  if (c->mem_update != RMT_MEM_BATCHED && c->mem_update != RMT_MEM_SEQUENTIAL)
    return why = "mem_update must be RMT_MEM_BATCHED or RMT_MEM_SEQUENTIAL", false;
  if (c->n_heads % c->n_kv_heads) return why = "n_heads must be a multiple of n_kv_heads", false;
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return why = "head_dim must be 32, 64 or 128", false;
  if (c->d_k % 32 || c->d_v % 32 || c->d_k > 128 || c->d_v > 128)
    return why = "d_k and d_v must be multiples of 32, at most 128", false;
  if (c->n_mem > 64 || c->n_mem * (c->d_k + c->d_v) > 4096) return why = "n_mem <= 64 and n_mem*(d_k+d_v) <= 4096", false;
  if (c->d_ff % 64) return why = "d_ff must be a multiple of 64", false;
  if (c->d_model % 4) return why = "d_model must be a multiple of 4", false;
  if (!(c->rope_theta > 0.f) || !(c->rms_eps >= 0.f) || !(c->mem_eps >= 0.f))
    return why = "rope_theta > 0, rms_eps >= 0, mem_eps >= 0", false;
  if (c->dtype == RMT_BF16_SPLIT && c->d_k != 64 && c->d_k != 128)
    return why = "bf16 split operands: d_k must be 64 or 128", false;
  if (c->dtype != RMT_F32) {
    const int hd = c->n_heads * c->head_dim, nqkv = (c->n_heads + 2 * c->n_kv_heads) * c->head_dim;
    if (c->d_model % 64 || hd % 64 || c->d_v % 64)
      return why = "bf16: d_model, n_heads*head_dim and d_v must be multiples of 64", false;
    if (!tc_pick_bn(nqkv, kEpiRope, c->head_dim) || !tc_pick_bn(2 * c->d_ff, kEpiSwiGLU, 0) ||
        !tc_pick_bn(c->d_model, kEpiResid, 0) || !tc_pick_bn(c->d_k, kEpiStoreF32, 0))
      return why = "bf16: projection widths do not fit the tensor-core tiles", false;
  }
  const double slot_bytes = double(2 * c->n_layers + 2) * (c->seg_len + c->n_mem) * c->d_model * 4.0;
  if (slot_bytes > 64e9) return why = "model too large for one device", false;
  return true;
}

rmt_status copy_in(void* dst, const void* src, size_t bytes, const char* what) {
  if (!src) return fail(RMT_EINVAL, std::string("null weight pointer: ") + what);
  RMT_CUDA(cudaMemcpy(dst, src, bytes, cudaMemcpyDefault));
  return RMT_OK;
}

#define RMT_TRY(expr)            \
  do {                           \
    rmt_status s_ = (expr);      \
    if (s_ != RMT_OK) return s_; \
  } while (0)

rmt_status pack_weights(rmt_handle* h, const rmt_weights* w) {
  const rmt_cfg& c = h->cfg;
  const size_t es = h->es, L = c.n_layers, d = c.d_model, hd = size_t(c.n_heads) * c.head_dim,
               kvd = size_t(c.n_kv_heads) * c.head_dim, F = c.d_ff, dk = c.d_k, dv = c.d_v;
  const void* const* arrays[] = {w->wq, w->wk, w->wv, w->wo, w->w_gate, w->w_up, w->w_down,
                                 w->w_mq, w->w_mk, w->w_mv, w->w_mo, w->g_attn, w->g_mlp};
  for (auto a : arrays)
    if (!a) return fail(RMT_EINVAL, "null per-layer weight array");
  auto at = [&](void* base, size_t elems_per_layer, size_t l, size_t off = 0) {
    return static_cast<char*>(base) + (l * elems_per_layer + off) * es;
  };
  const size_t nqkv = size_t(h->Nqkv);
  // pair packing of a rotated projection: rows p and p + dh/2 of each head go to 2p, 2p + 1
  auto copy_rope_pairs = [&](char* dst, const void* src, size_t heads, const char* what) -> rmt_status {
    if (!src) return fail(RMT_EINVAL, std::string("null weight pointer: ") + what);
    const size_t row = d * es, dh = c.head_dim, half = dh / 2;
    for (size_t hh = 0; hh < heads; ++hh) {
      const char* s0 = static_cast<const char*>(src) + hh * dh * row;
      char* d0 = dst + hh * dh * row;
      RMT_CUDA(cudaMemcpy2D(d0, 2 * row, s0, row, row, half, cudaMemcpyDefault));
      RMT_CUDA(cudaMemcpy2D(d0 + row, 2 * row, s0 + half * row, row, row, half, cudaMemcpyDefault));
    }
    return RMT_OK;
  };
  for (size_t l = 0; l < L; ++l) {
    if (h->pair_qkv) {
      RMT_TRY(copy_rope_pairs(at(h->w_qkv, nqkv * d, l), w->wq[l], c.n_heads, "wq"));
      RMT_TRY(copy_rope_pairs(at(h->w_qkv, nqkv * d, l, hd * d), w->wk[l], c.n_kv_heads, "wk"));
    } else {
      RMT_TRY(copy_in(at(h->w_qkv, nqkv * d, l), w->wq[l], hd * d * es, "wq"));
      RMT_TRY(copy_in(at(h->w_qkv, nqkv * d, l, hd * d), w->wk[l], kvd * d * es, "wk"));
    }
    RMT_TRY(copy_in(at(h->w_qkv, nqkv * d, l, (hd + kvd) * d), w->wv[l], kvd * d * es, "wv"));
    if (h->fold_mo) {  // row n of layer l: W_o[n][0..hd) then W_mo[n][0..dv)
      const size_t ldw = hd + dv;
      if (!w->wo[l] || !w->w_mo[l]) return fail(RMT_EINVAL, "null wo/w_mo");
      RMT_CUDA(cudaMemcpy2D(at(h->w_o, d * ldw, l), ldw * es, w->wo[l], hd * es, hd * es, d, cudaMemcpyDefault));
      RMT_CUDA(cudaMemcpy2D(at(h->w_o, d * ldw, l, hd), ldw * es, w->w_mo[l], dv * es, dv * es, d, cudaMemcpyDefault));
    } else {
      RMT_TRY(copy_in(at(h->w_o, d * hd, l), w->wo[l], d * hd * es, "wo"));
    }
    // gate/up interleaved: row by row for the pair GEMM, else in blocks of kSwiGLUBlock rows
    if (!w->w_gate[l] || !w->w_up[l]) return fail(RMT_EINVAL, "null w_gate/w_up");
    const size_t rows = h->pair_gu ? 1 : kSwiGLUBlock, blk = rows * d * es;
    RMT_CUDA(cudaMemcpy2D(at(h->w_gu, 2 * F * d, l), 2 * blk, w->w_gate[l], blk, blk, F / rows, cudaMemcpyDefault));
    RMT_CUDA(cudaMemcpy2D(at(h->w_gu, 2 * F * d, l) + blk, 2 * blk, w->w_up[l], blk, blk, F / rows,
                          cudaMemcpyDefault));
    RMT_TRY(copy_in(at(h->w_d, d * F, l), w->w_down[l], d * F * es, "w_down"));
    RMT_TRY(copy_in(at(h->w_mq, dk * d, l), w->w_mq[l], dk * d * es, "w_mq"));
    RMT_TRY(copy_in(at(h->w_mo, d * dv, l), w->w_mo[l], d * dv * es, "w_mo"));
    RMT_TRY(copy_in(at(h->w_mkv, (dk + dv) * d, l), w->w_mk[l], dk * d * es, "w_mk"));
    RMT_TRY(copy_in(at(h->w_mkv, (dk + dv) * d, l, dk * d), w->w_mv[l], dv * d * es, "w_mv"));
    RMT_TRY(copy_in(at(h->g1, d, l), w->g_attn[l], d * es, "g_attn"));
    RMT_TRY(copy_in(at(h->g2, d, l), w->g_mlp[l], d * es, "g_mlp"));
  }
  RMT_TRY(copy_in(h->memtok, w->mem_tokens, size_t(c.n_mem) * d * es, "mem_tokens"));
  return RMT_OK;
}

rmt_status build_maps(rmt_handle* h) {
  const rmt_cfg& c = h->cfg;
  // stacks of the cap_b sequences: residual slots [cap_b * n_slots], layer scratch [cap_b * L]
  const uint64_t L = uint64_t(h->cap_b) * c.n_layers, d = c.d_model, hd = uint64_t(c.n_heads) * c.head_dim,
                 F = c.d_ff, M = h->M, NS = uint64_t(h->cap_b) * n_slots(c.n_layers);
  const uint64_t LW = c.n_layers;  // weight stacks
  h->bn_mq = tc_pick_bn(c.d_k, kEpiStoreF32, 0);
  h->bn_mo = tc_pick_bn(c.d_model, kEpiResid, 0);
  h->bn_qkv = tc_pick_bn(h->Nqkv, kEpiRope, c.head_dim);
  h->bn_o = tc_pick_bn(c.d_model, kEpiResid, 0);
  h->bn_gu = tc_pick_bn(2 * c.d_ff, kEpiSwiGLU, 0);
  h->bn_d = tc_pick_bn(c.d_model, kEpiResidCast, 0);
  auto map = [](CUtensorMap* m, const void* p, uint64_t inner, uint64_t rows, uint64_t depth, uint32_t box) {
    return make_tmap_16_3d(m, p, inner, rows, depth, box, true);
  };
  // weight boxes: 128 rows per CTA on the pair GEMM, else the tile width
  const uint32_t pb = static_cast<uint32_t>(pair_token_tile(static_cast<int>(M)) / 2),
                 qb = static_cast<uint32_t>(std::min(pair_token_tile(static_cast<int>(M)), kPairFineTile) / 2);
  const bool any_pair = h->pair_mo || h->pair_qkv || h->pair_o || h->pair_gu || h->pair_d;
  // the read-out o: its own buffer, or (fold_mo) the last d_v columns of the attention output
  const uint64_t lda = uint64_t(h->ld_att);
  // split-operand mode: the activation rows hold [high terms | low terms], twice as wide
  const uint64_t sw = h->split ? 2 : 1, xw = sw * d, aw = sw * lda, uw = sw * F, ow = sw * c.d_v;
  auto map_om = [&](CUtensorMap* m, uint32_t box) {
    // folded: from column hd of the attention rows, the high terms of o, then (split) the rest
    // of the row up to its low terms ld_att columns further
    return h->fold_mo ? make_tmap_16_3d_strided(m, static_cast<__half*>(h->att) + hd, aw - hd, M, L, aw, box, true)
                      : map(m, h->om, ow, M, L, box);
  };
  bool ok = map(&h->tm_xb, h->xb, xw, M, NS, 128) && map_om(&h->tm_om, 128) &&
            map(&h->tm_att, h->att, aw, M, L, 128) && map(&h->tm_u, h->u, uw, M, L, 128) &&
            map(&h->tm_wmq, h->w_mq, d, c.d_k, LW, h->bn_mq) &&
            map(&h->tm_wmo, h->w_mo, c.d_v, d, LW, h->pair_mo ? 128 : h->bn_mo) &&
            map(&h->tm_wqkv, h->w_qkv, d, h->Nqkv, LW, h->pair_qkv ? 128 : h->bn_qkv) &&
            map(&h->tm_wo, h->w_o, lda, d, LW, h->pair_o ? 128 : h->bn_o) &&
            map(&h->tm_wgu, h->w_gu, d, 2 * F, LW, h->pair_gu ? 128 : h->bn_gu) &&
            map(&h->tm_wd, h->w_d, F, d, LW, h->pair_d ? 128 : h->bn_d) &&
            (!any_pair || (map(&h->tp_xb, h->xb, xw, M, NS, pb) && map_om(&h->tp_om, pb) &&
                           map(&h->tp_att, h->att, aw, M, L, pb) && map(&h->tp_u, h->u, uw, M, L, pb) &&
                           map(&h->tq_xb, h->xb, xw, M, NS, qb) && map_om(&h->tq_om, qb) &&
                           map(&h->tq_att, h->att, aw, M, L, qb) && map(&h->tq_u, h->u, uw, M, L, qb))) &&
            map(&h->tm_qkv, h->qkv, h->Nqkv, M, L, 128) &&
            map(&h->tm_qkv_tail, h->qkv, h->Nqkv, M, L, attn_tail_box(int(M), c.n_heads, c.n_kv_heads)) &&
            make_tmap_f32_resid(&h->tm_x, h->x, d, M, NS) &&
            (c.head_dim < 64 || map(&h->tm_rope, h->rope_h, c.head_dim, M, 1, 32));
  return ok ? RMT_OK : fail(RMT_ECUDA, "cuTensorMapEncodeTiled failed");
}

// (Re)allocate the activations, the layer scratch and the memory state for B sequences and
// rebuild the tensor maps over them. Waits for the device first: earlier forwards may still
// use the old buffers.
rmt_status reserve_acts(rmt_handle* h, int B) {
  if (B <= h->cap_b) return RMT_OK;
  RMT_CUDA(cudaDeviceSynchronize());
  h->free_acts();
  const rmt_cfg& c = h->cfg;
  const size_t nb = B, L = c.n_layers, d = c.d_model, M = h->M, es = h->es, F = c.d_ff, dk = c.d_k, dv = c.d_v,
               BL = nb * L, sw = h->split ? 2 : 1;  // sw: operand row width factor (split: hi | lo)
  struct {
    void** p;
    size_t bytes;
  } plan[] = {
      {reinterpret_cast<void**>(&h->x), nb * n_slots(c.n_layers) * M * d * 4},
      {&h->qkv, BL * M * h->Nqkv * (h->split ? 4 : es)}, {&h->att, BL * M * size_t(h->ld_att) * es * sw},
      {reinterpret_cast<void**>(&h->ss1), BL * M * (d / 16 + 1) * 4},
      {reinterpret_cast<void**>(&h->ss2), BL * M * (d / 16 + 1) * 4},
      {&h->u, BL * M * F * es * sw},      {&h->om, BL * M * dv * es * sw},
      {reinterpret_cast<void**>(&h->qm), BL * M * dk * 4},
      {reinterpret_cast<void**>(&h->part), BL * h->nsplit * size_t(c.n_mem) * (dk + dv) * 4},
      {reinterpret_cast<void**>(&h->A), BL * dk * dv * 4},
      {reinterpret_cast<void**>(&h->z), BL * dk * 4},
  };
  for (auto& e : plan) {
    *e.p = h->act_alloc(e.bytes);
    if (!*e.p) {
      h->free_acts();
      return fail(RMT_ENOMEM, "activation allocation failed");
    }
  }
  if (h->bf16) {
    h->xb = static_cast<__half*>(h->act_alloc(nb * n_slots(c.n_layers) * M * d * 2 * sw));
    if (!h->xb) {
      h->free_acts();
      return fail(RMT_ENOMEM, "activation allocation failed");
    }
  }
  if (cudaMemset(h->x, 0, nb * n_slots(c.n_layers) * M * d * 4) != cudaSuccess) {
    h->free_acts();
    return fail(RMT_ECUDA, "cudaMemset failed");
  }
  if (h->chain_mlp) {  // one counter per (cell, token tile) of a step, both parities, both boundaries
    const int nt = std::min(pair_token_tile(M), kPairFineTile);  // the finer of the two token tiles
    h->chain_ctr_len = static_cast<int>(BL) * ((M + nt - 1) / nt);
    const size_t bytes = size_t(2) * (kMaxPhases - 1) * h->chain_ctr_len * sizeof(unsigned);
    h->chain_ctr = static_cast<unsigned*>(h->act_alloc(bytes));
    if (!h->chain_ctr || cudaMemset(h->chain_ctr, 0, bytes) != cudaSuccess) {
      h->free_acts();
      return fail(RMT_ENOMEM, "activation allocation failed");
    }
    h->chain_parity = 0;
  }
  h->cap_b = B;
  if (h->bf16) {
    rmt_status st = build_maps(h);
    if (st != RMT_OK) {
      h->free_acts();
      return st;
    }
    h->ss_parts = (c.d_model / h->bn_o) * 2;  // memo and O projections: N = d_model, two halves per tile
    if (h->bn_mo != h->bn_o) {
      h->free_acts();
      return fail(RMT_EINVAL, "inconsistent projection tiles");
    }
  } else {
    h->ss_parts = (c.d_model + 127) / 128;  // fp32 kernel: one block per 128-column tile
  }
  return RMT_OK;
}

enum Proj { kProjMemQ, kProjMemO, kProjQkv, kProjO, kProjGateUp, kProjDown };

// A CTA-pair projection's launch arguments, collected instead of launched (for the chain):
// tx maps the activations in pair_token_tile(M) token tiles, tq in kPairFineTile ones.
struct PairLaunch {
  TcGemmArgs a;
  const CUtensorMap* tw;
  const CUtensorMap* tx;
  const CUtensorMap* tq;
};

cudaError_t run_proj(rmt_handle* h, Proj p, const Cell* cells, int G, cudaStream_t st, PairLaunch* collect = nullptr) {
  const rmt_cfg& c = h->cfg;
  const int d = c.d_model, hd = c.n_heads * c.head_dim;
  EpiParams ep{};
  ep.x = h->x;
  ep.ldx = d;
  ep.rope = h->rope;
  ep.head_dim = c.head_dim;
  ep.rope_cols = (c.n_heads + c.n_kv_heads) * c.head_dim;
  ep.out_mode = ep.src_mode = ep.dst_mode = kByLayer;
  ep.ss_parts = h->ss_parts;
  ep.inv_d = 1.f / float(d);
  ep.rms_eps = c.rms_eps;
  const EpiKind resid = h->bf16 ? kEpiResidCast : kEpiResid;  // bf16: also refresh the bf16 copy
  // split-operand mode: X rows are [high terms | low terms]; kx_lo = column of the low terms
  const int sw = h->split ? 2 : 1;
  int kx_lo = 0;
  if (h->split) ep.ldxb = 2 * d;
  int N = 0, K = 0;
  EpiKind epi = kEpiStoreF32;
  IndexMode amode = kByLayer;
  const float* a32 = nullptr;
  const void* w = nullptr;
  const CUtensorMap *ta = nullptr, *tb = nullptr, *tp = nullptr, *tq = nullptr;
  int bn = 0;
  bool pair = false;
  switch (p) {
    case kProjMemQ:
      N = c.d_k, K = d, epi = kEpiStoreF32, amode = kInSlot;
      ep.out = h->qm, ep.ldo = c.d_k;
      a32 = h->x, w = h->w_mq, ta = &h->tm_xb, tb = &h->tm_wmq, bn = h->bn_mq;
      if (h->fuse_read) {  // o = phi(q) A / (phi(q) . z + eps) straight from the accumulator
        epi = kEpiMemRead;
        if (h->fold_mo)  // o goes to the last d_v columns of the attention output rows
          ep.out = static_cast<__half*>(h->att) + hd, ep.ldo = sw * h->ld_att, ep.lo_off = h->split ? h->ld_att : 0;
        else
          ep.out = h->om, ep.ldo = sw * c.d_v, ep.lo_off = h->split ? c.d_v : 0;
        ep.mem_A = h->A, ep.mem_z = h->z, ep.mem_dv = c.d_v, ep.mem_eps = c.mem_eps;
      }
      kx_lo = h->split ? d : 0;
      break;
    case kProjMemO:  // x_out = x_in + read-out; emits the row sums of squares of RMSNorm 1
      N = d, K = c.d_v, epi = resid;
      ep.src_mode = kInSlot, ep.dst_mode = kOutSlot, ep.xb = h->xb, ep.ss_out = h->ss1;
      ep.resid_no_store = h->fold_mo;  // the O projection adds W_mo o itself
      a32 = static_cast<const float*>(h->om), w = h->w_mo, ta = &h->tm_om, tb = &h->tm_wmo, bn = h->bn_mo;
      tp = &h->tp_om, tq = &h->tq_om, pair = h->pair_mo;
      ep.lo_off = h->split ? d : 0;
      kx_lo = h->split ? (h->fold_mo ? h->ld_att : c.d_v) : 0;
      break;
    case kProjQkv:  // rows of x_out scaled by RMSNorm 1 (gain folded into the weight), then RoPE
      N = h->Nqkv, K = d, epi = kEpiRope, amode = kOutSlot;
      ep.out = h->qkv, ep.ldo = h->Nqkv, ep.ss_in = h->ss1;
      a32 = h->x, w = h->w_qkv, ta = &h->tm_xb, tb = &h->tm_wqkv, bn = h->bn_qkv;
      tp = &h->tp_xb, tq = &h->tq_xb, pair = h->pair_qkv;
      ep.out_f32 = h->split;  // split-operand mode: attention reads fp32 q, k, v
      kx_lo = h->split ? d : 0;
      break;
    case kProjO:  // x_out += attention output; emits the row sums of squares of RMSNorm 2
      N = d, K = hd, epi = resid;
      ep.src_mode = ep.dst_mode = kOutSlot, ep.xb = h->xb, ep.ss_out = h->ss2;
      if (h->fold_mo) {  // x_out = x_in + [W_o | W_mo] [att ; o]
        K = h->ld_att;
        ep.src_mode = kInSlot;
      }
      a32 = static_cast<const float*>(h->att), w = h->w_o, ta = &h->tm_att, tb = &h->tm_wo, bn = h->bn_o;
      tp = &h->tp_att, tq = &h->tq_att, pair = h->pair_o;
      ep.lo_off = h->split ? d : 0;
      kx_lo = h->split ? h->ld_att : 0;
      break;
    case kProjGateUp:  // rows of x_out scaled by RMSNorm 2 (gain folded into the weight), SwiGLU
      N = 2 * c.d_ff, K = d, epi = kEpiSwiGLU, amode = kOutSlot;
      ep.out = h->u, ep.ldo = sw * c.d_ff, ep.ss_in = h->ss2;
      a32 = h->x, w = h->w_gu, ta = &h->tm_xb, tb = &h->tm_wgu, bn = h->bn_gu;
      tp = &h->tp_xb, tq = &h->tq_xb, pair = h->pair_gu;
      ep.lo_off = h->split ? c.d_ff : 0;
      kx_lo = h->split ? d : 0;
      break;
    case kProjDown:  // x_out += MLP output; the bf16 copy feeds the next layer's memory query
      N = d, K = c.d_ff, epi = resid;
      ep.src_mode = ep.dst_mode = kOutSlot, ep.xb = h->xb;
      a32 = static_cast<const float*>(h->u), w = h->w_d, ta = &h->tm_u, tb = &h->tm_wd, bn = h->bn_d;
      tp = &h->tp_u, tq = &h->tq_u, pair = h->pair_d;
      ep.lo_off = h->split ? d : 0;
      kx_lo = h->split ? c.d_ff : 0;
      break;
  }
  if (h->bf16 && pair) {
    TcGemmArgs a{h->M, N, K, G, cells, c.n_layers, amode, epi, ep, h->err, kx_lo};
    if (collect) {
      *collect = PairLaunch{a, tb, tp, tq};
      return cudaSuccess;
    }
    a.nt = pair_pick_nt(h->M, G, N / 256);
    return launch_tc_pair_gemm(*tb, a.nt == pair_token_tile(h->M) ? *tp : *tq, a, /*f16=*/true, st);
  }
  if (collect) return cudaErrorInvalidValue;
  if (h->bf16) {
    const bool rope_tma = p == kProjQkv && c.head_dim >= 64 && !h->split;
    ep.rope_tma = rope_tma;
    TcGemmArgs a{h->M, N, K, G, cells, c.n_layers, amode, epi, ep, h->err, kx_lo};
    return launch_tc_gemm(*ta, *tb, rope_tma ? h->tm_rope : h->tm_x, a, bn, /*f16=*/true, st);
  }
  const int lda = (p == kProjMemQ || p == kProjQkv || p == kProjGateUp) ? d : K;
  SimtGemmArgs a{h->M, N, K, G, cells, c.n_layers, a32, lda, amode, static_cast<const float*>(w), epi, ep};
  return launch_simt_gemm(a, st);
}

// The O projection, gate/up and down of a step in one chained CTA-pair launch.
cudaError_t run_chain_o_mlp(rmt_handle* h, const Cell* cells, int G, cudaStream_t st) {
  PairLaunch o{}, gu{}, dn{};
  cudaError_t e = run_proj(h, kProjO, cells, G, st, &o);
  if (e == cudaSuccess) e = run_proj(h, kProjGateUp, cells, G, st, &gu);
  if (e == cudaSuccess) e = run_proj(h, kProjDown, cells, G, st, &dn);
  if (e != cudaSuccess) return e;
  PairChainArgs a{};
  a.ph[0] = o.a;
  a.ph[1] = gu.a;
  a.ph[2] = dn.a;
  a.nphase = 3;
  a.ctr = h->chain_ctr;
  a.ctr_len = h->chain_ctr_len;
  a.parity = h->chain_parity;
  const int nt = pair_pick_nt(h->M, G, (o.a.N + gu.a.N + dn.a.N) / 256);
  const bool fine = nt != pair_token_tile(h->M);
  for (int p = 0; p < 3; ++p) a.ph[p].nt = nt;
  const CUtensorMap tw[3] = {*o.tw, *gu.tw, *dn.tw};
  const CUtensorMap tx[3] = {fine ? *o.tq : *o.tx, fine ? *gu.tq : *gu.tx, fine ? *dn.tq : *dn.tx};
  e = launch_tc_pair_chain_o_mlp(tw, tx, a, st);
  if (e == cudaSuccess) h->chain_parity ^= 1;
  return e;
}

// NVTX range names of the kernel kinds (rmt_kernel order). The ranges cost nothing
// measurable without a tool attached and give a profiler's timeline the step structure.
const char* const kKindNames[RMT_K_COUNT] = {"assemble", "memq",      "memread",   "memo", "rmsnorm1",
                                             "qkv",      "attention", "o",         "rmsnorm2", "gateup",
                                             "down",     "memkv",     "memupdate", "emit"};

struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// Launch one kernel of a step: count it and, if its kind is probed, bracket it with events.
template <typename F>
cudaError_t launch_kind(rmt_handle* h, int kind, double flops, double bytes, cudaStream_t st, F&& fn) {
  NvtxRange range(kKindNames[kind]);
  const bool on = (h->probe_mask >> kind) & 1u;
  cudaEvent_t a = nullptr, b = nullptr;
  if (on && (a = h->probe_event()) != nullptr) cudaEventRecord(a, st);
  const cudaError_t e = fn();
  ++h->launches;
  if (on && a && (b = h->probe_event()) != nullptr) {
    cudaEventRecord(b, st);
    h->probe_recs.push_back(rmt_handle::ProbeRec{kind, flops, bytes, a, b});
  }
  return e;
}

cudaError_t enqueue_step(rmt_handle* h, const Table& t, int step, const void* emb, void* out, cudaStream_t st) {
  const rmt_cfg& c = h->cfg;
  const int L = c.n_layers, d = c.d_model, M = h->M, G = t.cnt[step], off = t.off[step];
  const Cell* cells = t.dev + off;
  const int n_first = t.n_first[step], n_last = t.n_last[step];
  // algorithmic work per launch (flops; bytes that must cross HBM at least once), over the
  // valid rows of the step's cells: g * m = their rows, pairs = their causal (query, key) pairs
  double rows = 0, pairs = 0, rows_first = 0, rows_last = 0;
  for (int i = 0; i < G; ++i) {
    const double mc = cell_rows(t.cells[off + i], M);
    rows += mc;
    pairs += mc * (mc + 1) / 2;
    if (i < n_first) rows_first += mc;
    if (i >= G - n_last) rows_last += mc - c.n_mem;
  }
  const double g = G, m = rows / G, dd = d, es = h->es, dk = c.d_k, dv = c.d_v, hd = double(c.n_heads) * c.head_dim,
               nq = h->Nqkv, F = c.d_ff, n = c.n_mem, ea = h->bf16 ? 2.0 : 4.0;
  cudaError_t e;
  if (n_first > 0) {
    e = launch_kind(h, RMT_K_ASSEMBLE, 0, rows_first * dd * (es + 4 + (h->bf16 ? 2 : 0)), st, [&] {
      return launch_assemble(cells, n_first, emb, h->memtok, h->x, h->bf16 ? h->xb : nullptr, M, c.n_mem, d, h->bf16,
                             h->err, st, h->split);
    });
    if (e != cudaSuccess) return e;
  }
  if (h->fuse_read) {  // mem-q GEMM with the memory read in its epilogue
    e = launch_kind(h, RMT_K_MEMQ, g * m * (2 * dk * dd + 2 * dk * dv + 2 * dk),
                    g * (m * dd * ea + dk * dd * es + dk * dv * 4 + dk * 4 + m * dv * es), st,
                    [&] { return run_proj(h, kProjMemQ, cells, G, st); });
    if (e != cudaSuccess) return e;
  } else {
    e = launch_kind(h, RMT_K_MEMQ, 2 * g * m * dk * dd, g * (m * dd * ea + dk * dd * es + m * dk * 4), st,
                    [&] { return run_proj(h, kProjMemQ, cells, G, st); });
    if (e != cudaSuccess) return e;
    e = launch_kind(h, RMT_K_MEMREAD, g * m * (2 * dk * dv + 2 * dk),
                    g * (m * dk * 4 + dk * dv * 4 + dk * 4 + m * dv * es), st, [&] {
                      MemReadArgs a{h->qm, h->A, h->z, h->om, M, c.d_k, c.d_v, c.mem_eps, G, cells, kByLayer, kByLayer, L};
                      if (h->split) a.ldo = 2 * c.d_v, a.lo_off = c.d_v;  // [high terms | low terms] rows
                      return launch_mem_read(a, h->bf16 ? kElemF16 : kElemF32, st, h->err);
                    });
    if (e != cudaSuccess) return e;
  }
  // with fold_mo the read-out projection stores only the f16 copy, and the O projection
  // carries the d_v extra columns of K
  const double fold = h->fold_mo ? 1.0 : 0.0;
  e = launch_kind(h, RMT_K_MEMO, 2 * g * m * dd * dv,
                  g * (m * dv * es + dd * dv * es + m * dd * 4 + (fold ? m * dd * 2 : m * dd * 4)), st,
                  [&] { return run_proj(h, kProjMemO, cells, G, st); });
  if (e != cudaSuccess) return e;
  e = launch_kind(h, RMT_K_QKV, 2 * g * m * nq * dd, g * (m * dd * es + nq * dd * es + m * nq * es), st,
                  [&] { return run_proj(h, kProjQkv, cells, G, st); });
  if (e != cudaSuccess) return e;
  e = launch_kind(h, RMT_K_ATTENTION, c.n_heads * 4.0 * c.head_dim * pairs,
                  g * (m * nq * es + m * hd * es), st, [&] {
                    AttnArgs a{h->qkv, h->att, M, c.n_heads, c.n_kv_heads, c.head_dim, G, cells, kByLayer, L, h->err,
                               h->ld_att};
                    if (h->split) {  // fp32 q, k, v in; f16 high and low terms out
                      a.ldo = 2 * h->ld_att, a.out_lo = h->ld_att;
                      return launch_attention(a, kElemF32, st);
                    }
                    if (h->bf16 && attention_tc_supported(c.head_dim))
                      return launch_attention_tc(h->tm_qkv, h->tm_qkv_tail, a, /*f16=*/true, st);
                    return launch_attention(a, h->bf16 ? kElemF16 : kElemF32, st);
                  });
  if (e != cudaSuccess) return e;
  // (the folded W_mo o is counted once, with the read-out projection, as the model defines it)
  const double o_flops = 2 * g * m * dd * hd, gu_flops = 2 * g * m * 2 * F * dd, d_flops = 2 * g * m * dd * F;
  const double o_bytes = g * (m * (hd + fold * dv) * es + dd * (hd + fold * dv) * es + 2 * m * dd * 4),
               gu_bytes = g * (m * dd * es + 2 * F * dd * es + m * F * es),
               d_bytes = g * (m * F * es + dd * F * es + 2 * m * dd * 4 + (h->bf16 ? m * dd * 2 : 0));
  if (h->chain_mlp) {  // one launch: reported under GATEUP with the work of all three projections
    e = launch_kind(h, RMT_K_GATEUP, o_flops + gu_flops + d_flops, o_bytes + gu_bytes + d_bytes, st,
                    [&] { return run_chain_o_mlp(h, cells, G, st); });
    if (e != cudaSuccess) return e;
  } else {
    e = launch_kind(h, RMT_K_O, o_flops, o_bytes, st, [&] { return run_proj(h, kProjO, cells, G, st); });
    if (e != cudaSuccess) return e;
    e = launch_kind(h, RMT_K_GATEUP, gu_flops, gu_bytes, st, [&] { return run_proj(h, kProjGateUp, cells, G, st); });
    if (e != cudaSuccess) return e;
    e = launch_kind(h, RMT_K_DOWN, d_flops, d_bytes, st, [&] { return run_proj(h, kProjDown, cells, G, st); });
    if (e != cudaSuccess) return e;
  }
  // many cells: whole sums in one "split" (the same bits as the partials' sum)
  const int kv_splits = mem_kv_written_splits(G, c.n_mem, d, h->bf16);
  e = launch_kind(h, RMT_K_MEMKV, 2 * g * n * (dk + dv) * dd,
                  g * (n * dd * 4 + (dk + dv) * dd * es + kv_splits * n * (dk + dv) * 4), st, [&] {
                    MemKvArgs a{h->x, M, d, c.n_mem, kOutSlot, h->w_mkv, h->part, c.d_k + c.d_v, G, cells, L};
                    return launch_mem_kv(a, h->bf16, st);
                  });
  if (e != cudaSuccess) return e;
  e = launch_kind(h, RMT_K_MEMUPDATE, g * 4 * n * dk * dv,
                  g * (kv_splits * n * (dk + dv) * 4 + 2 * (dk * dv + dk) * 4), st, [&] {
                    MemUpdateArgs a{h->part, kv_splits, nullptr, nullptr, h->A, h->z, c.n_mem, c.d_k, c.d_v, c.mem_eps,
                                    G, cells, kByLayer, kByLayer, L, h->trace, off, step,
                                    c.mem_update == RMT_MEM_SEQUENTIAL ? 1 : 0};
                    return launch_mem_update(a, st);
                  });
  if (e != cudaSuccess) return e;
  if (n_last > 0) {
    e = launch_kind(h, RMT_K_EMIT, 0, rows_last * dd * (4 + es), st, [&] {
      return launch_emit(cells + G - n_last, n_last, h->x, out, M, c.n_mem, d, h->bf16, st);
    });
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------ full-attention forward (comparison model)

// Buffers, RoPE tables, cell table and tensor maps of the full-attention forward for T tokens
// (reallocated when T exceeds the current capacity; the maps are rebuilt for every new T).
rmt_status full_buffers(rmt_handle* h, int T) {
  const rmt_cfg& c = h->cfg;
  const size_t d = c.d_model, hd = size_t(c.n_heads) * c.head_dim, F = c.d_ff, half = c.head_dim / 2;
  if (T > h->full_cap) {
    RMT_CUDA(cudaDeviceSynchronize());  // an earlier full forward may still use the old buffers
    h->free_full();
    const size_t Tn = size_t(T);
    struct {
      void** p;
      size_t bytes;
    } plan[] = {
        {reinterpret_cast<void**>(&h->fx), 2 * Tn * d * 4},      {reinterpret_cast<void**>(&h->fxb), 2 * Tn * d * 2},
        {&h->fqkv, Tn * h->Nqkv * 2},                            {&h->fatt, Tn * hd * 2},
        {&h->fu, Tn * F * 2},                                    {reinterpret_cast<void**>(&h->fss1), Tn * (d / 16 + 1) * 4},
        {reinterpret_cast<void**>(&h->fss2), Tn * (d / 16 + 1) * 4},
        {reinterpret_cast<void**>(&h->frope), Tn * half * sizeof(float2)},
        {reinterpret_cast<void**>(&h->frope_h), Tn * half * sizeof(__half2)},
        {reinterpret_cast<void**>(&h->fcells), size_t(c.n_layers) * sizeof(Cell)},
    };
    for (auto& e : plan) {
      void* q = nullptr;
      if (cudaMalloc(&q, e.bytes) != cudaSuccess) {
        cudaGetLastError();
        h->free_full();
        return fail(RMT_ENOMEM, "full-attention buffer allocation failed");
      }
      h->full_allocs.push_back(q);
      *e.p = q;
    }
    // RoPE angles p * theta^(-2i/dh) at positions 0..T-1, in double precision
    std::vector<float2> tab(Tn * half);
    std::vector<__half2> tab_h(Tn * half);
    for (size_t q = 0; q < Tn; ++q)
      for (size_t i = 0; i < half; ++i) {
        const double ang = double(q) * std::pow(double(c.rope_theta), -2.0 * double(i) / c.head_dim);
        tab[q * half + i] = make_float2(float(std::cos(ang)), float(std::sin(ang)));
        tab_h[q * half + i] = __floats2half2_rn(tab[q * half + i].x, tab[q * half + i].y);
      }
    RMT_CUDA(cudaMemcpy(h->frope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice));
    RMT_CUDA(cudaMemcpy(h->frope_h, tab_h.data(), tab_h.size() * sizeof(__half2), cudaMemcpyHostToDevice));
    h->full_cap = T;
  }
  if (T != h->full_T) {
    std::vector<Cell> cells(c.n_layers);
    for (int l = 0; l < c.n_layers; ++l) {
      cells[l] = Cell{l, 0, 0, T, 0, l & 1, (l + 1) & 1, 0};
#ifdef RMT_DEBUG
      cells[l].lim_L = c.n_layers;
      cells[l].lim_state = 1;
      cells[l].lim_slot = 2;
      cells[l].lim_M = T;
      cells[l].lim_nmem = 0;
      cells[l].lim_tokens = T;
      cells[l].lim_err = h->err;
#endif
    }
    RMT_CUDA(cudaMemcpy(h->fcells, cells.data(), cells.size() * sizeof(Cell), cudaMemcpyHostToDevice));
    auto map = [](CUtensorMap* m, const void* q, uint64_t inner, uint64_t rows, uint64_t depth, uint32_t box) {
      return make_tmap_16_3d(m, q, inner, rows, depth, box, true);
    };
    const uint64_t Tu = uint64_t(T), pb = uint64_t(pair_token_tile(T) / 2);
    const bool ok = map(&h->fm_xb, h->fxb, d, Tu, 2, 128) && map(&h->fm_att, h->fatt, hd, Tu, 1, 128) &&
                    map(&h->fm_u, h->fu, F, Tu, 1, 128) && map(&h->fm_qkv, h->fqkv, h->Nqkv, Tu, 1, 128) &&
                    map(&h->fm_qkv_tail, h->fqkv, h->Nqkv, Tu, 1, attn_tail_box(T, c.n_heads, c.n_kv_heads)) &&
                    map(&h->fp_xb, h->fxb, d, Tu, 2, uint32_t(pb)) && map(&h->fp_att, h->fatt, hd, Tu, 1, uint32_t(pb)) &&
                    map(&h->fp_u, h->fu, F, Tu, 1, uint32_t(pb)) && make_tmap_f32_resid(&h->fm_x, h->fx, d, Tu, 2) &&
                    (c.head_dim < 64 || map(&h->fm_rope, h->frope_h, c.head_dim, Tu, 1, 32));
    if (!ok) return fail(RMT_ECUDA, "cuTensorMapEncodeTiled failed");
    h->full_T = T;
  }
  return RMT_OK;
}

// One projection of layer `cell` of the full-attention forward: the layer reads its input
// slot for QKV; O adds the attention output to it into the output slot (and emits the RMSNorm
// 2 statistics); gate/up reads the output slot; down adds the MLP output in place and emits
// the RMSNorm 1 statistics of the next layer's input.
cudaError_t run_proj_full(rmt_handle* h, Proj p, const Cell* cell, cudaStream_t st) {
  const rmt_cfg& c = h->cfg;
  const int d = c.d_model, hd = c.n_heads * c.head_dim, T = h->full_T;
  EpiParams ep{};
  ep.x = h->fx;
  ep.ldx = d;
  ep.rope = h->frope;
  ep.head_dim = c.head_dim;
  ep.rope_cols = (c.n_heads + c.n_kv_heads) * c.head_dim;
  ep.out_mode = ep.src_mode = ep.dst_mode = kByLayer;
  ep.ss_parts = h->ss_parts;
  ep.inv_d = 1.f / float(d);
  ep.rms_eps = c.rms_eps;
  int N = 0, K = 0, bn = 0;
  EpiKind epi = kEpiStoreAct;
  IndexMode amode = kByLayer;
  const CUtensorMap *ta = nullptr, *tb = nullptr, *tp = nullptr;
  bool pair = false;
  switch (p) {
    case kProjQkv:
      N = h->Nqkv, K = d, epi = kEpiRope, amode = kInSlot;
      ep.out = h->fqkv, ep.ldo = h->Nqkv, ep.ss_in = h->fss1;
      ta = &h->fm_xb, tb = &h->tm_wqkv, tp = &h->fp_xb, bn = h->bn_qkv, pair = h->pair_qkv;
      break;
    case kProjO:
      N = d, K = hd, epi = kEpiResidCast;
      ep.src_mode = kInSlot, ep.dst_mode = kOutSlot, ep.xb = h->fxb, ep.ss_out = h->fss2;
      ta = &h->fm_att, tb = &h->tm_wo, tp = &h->fp_att, bn = h->bn_o, pair = h->pair_o;
      break;
    case kProjGateUp:
      N = 2 * c.d_ff, K = d, epi = kEpiSwiGLU, amode = kOutSlot;
      ep.out = h->fu, ep.ldo = c.d_ff, ep.ss_in = h->fss2;
      ta = &h->fm_xb, tb = &h->tm_wgu, tp = &h->fp_xb, bn = h->bn_gu, pair = h->pair_gu;
      break;
    case kProjDown:
      N = d, K = c.d_ff, epi = kEpiResidCast;
      ep.src_mode = ep.dst_mode = kOutSlot, ep.xb = h->fxb, ep.ss_out = h->fss1;
      ta = &h->fm_u, tb = &h->tm_wd, tp = &h->fp_u, bn = h->bn_d, pair = h->pair_d;
      break;
    default:
      return cudaErrorInvalidValue;
  }
  TcGemmArgs a{T, N, K, 1, cell, c.n_layers, amode, epi, ep, h->err};
  if (pair && tc_pair_supported(T, N, K, epi, c.head_dim)) return launch_tc_pair_gemm(*tb, *tp, a, /*f16=*/true, st);
  if (pair) return cudaErrorInvalidValue;  // the weights are packed for the CTA-pair kernel
  const bool rope_tma = p == kProjQkv && c.head_dim >= 64;
  a.ep.rope_tma = rope_tma;
  return launch_tc_gemm(*ta, *tb, rope_tma ? h->fm_rope : h->fm_x, a, bn, /*f16=*/true, st);
}

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (dev >= 0 && cudaGetDevice(&prev) == cudaSuccess && prev != dev)
      cudaSetDevice(dev);
    else
      prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" {

const char* rmt_last_error(void) { return g_last_error.c_str(); }

rmt_status rmt_schedule_table(int32_t n_layers, int32_t n_segments, rmt_schedule schedule, int32_t* out_dls,
                              size_t cap) {
  if (n_layers <= 0 || n_segments <= 0) return fail(RMT_EINVAL, "n_layers and n_segments must be positive");
  if (schedule != RMT_DIAGONAL && schedule != RMT_SEQUENTIAL) return fail(RMT_EINVAL, "unknown schedule");
  if (!out_dls) return fail(RMT_EINVAL, "out_dls is null");
  const size_t need = 3 * size_t(n_layers) * size_t(n_segments);
  if (cap < need) return fail(RMT_EINVAL, "out_dls capacity below 3*n_layers*n_segments");
  Table t;
  order_cells(n_layers, std::vector<int>{n_segments}, schedule, t);
  size_t k = 0;
  for (size_t step = 0; step < t.off.size(); ++step)
    for (int i = 0; i < t.cnt[step]; ++i) {
      const Cell c = t.cells[t.off[step] + i];
      out_dls[k++] = int32_t(step);
      out_dls[k++] = c.l;
      out_dls[k++] = c.s;
    }
  return RMT_OK;
}

rmt_status rmt_schedule_table_batch(int32_t n_layers, int32_t batch, const int32_t* n_segments, rmt_schedule schedule,
                                    int32_t* out_dbls, size_t cap) {
  if (n_layers <= 0 || batch <= 0 || !n_segments) return fail(RMT_EINVAL, "n_layers and batch must be positive");
  if (schedule != RMT_DIAGONAL && schedule != RMT_SEQUENTIAL) return fail(RMT_EINVAL, "unknown schedule");
  if (!out_dbls) return fail(RMT_EINVAL, "out_dbls is null");
  std::vector<int> S(n_segments, n_segments + batch);
  size_t cells = 0;
  for (int v : S) {
    if (v <= 0) return fail(RMT_EINVAL, "every sequence needs at least one segment");
    cells += size_t(v) * size_t(n_layers);
  }
  if (cap < 4 * cells) return fail(RMT_EINVAL, "out_dbls capacity below 4 * cells");
  Table t;
  order_cells(n_layers, S, schedule, t);
  size_t k = 0;
  for (size_t step = 0; step < t.off.size(); ++step)
    for (int i = 0; i < t.cnt[step]; ++i) {
      const Cell c = t.cells[t.off[step] + i];
      out_dbls[k++] = int32_t(step);
      out_dbls[k++] = c.b;
      out_dbls[k++] = c.l;
      out_dbls[k++] = c.s;
    }
  return RMT_OK;
}

rmt_status rmt_get_schedule(const rmt_handle* h, int32_t n_segments, rmt_schedule schedule, int32_t* out_dls,
                            size_t cap) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  return rmt_schedule_table(h->cfg.n_layers, n_segments, schedule, out_dls, cap);
}

rmt_status rmt_create(const rmt_weights* weights, const rmt_cfg* cfg, rmt_handle** out) {
  if (!weights || !cfg || !out) return fail(RMT_EINVAL, "null argument to rmt_create");
  std::string why;
  if (!validate_cfg(cfg, why)) return fail(RMT_EINVAL, "invalid cfg: " + why);
  rmt_handle* h = new rmt_handle();
  h->cfg = *cfg;
  auto bail = [&](rmt_status st) {
    h->release();
    delete h;
    return st;
  };
  if (cudaGetDevice(&h->dev) != cudaSuccess) return bail(fail(RMT_ECUDA, "no CUDA device"));
  const rmt_cfg& c = h->cfg;
  h->bf16 = c.dtype != RMT_F32;
  h->split = c.dtype == RMT_BF16_SPLIT;
  h->es = h->bf16 ? 2 : 4;
  h->M = c.seg_len + c.n_mem;
  h->Nqkv = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  h->nsplit = mem_kv_splits(c.d_model, h->bf16);
  const size_t L = c.n_layers, d = c.d_model, M = h->M, es = h->es, F = c.d_ff, dk = c.d_k, dv = c.d_v;
  if (h->bf16) {
    const int Mi = h->M, di = c.d_model, hdi = c.n_heads * c.head_dim, Fi = c.d_ff;
    // the memory read-out projection (K = d_v) is a pure stream over the residual; it stays on
    // the single-CTA kernel, whose residual epilogue moves whole blocks through TMA
    h->pair_mo = false;
    h->fuse_read = c.d_k == 64 && c.d_v == 64 && tc_pick_bn(c.d_k, kEpiStoreF32, 0) == 64;
    h->pair_qkv = tc_pair_supported(Mi, h->Nqkv, di, kEpiRope, c.head_dim);
    h->pair_gu = tc_pair_supported(Mi, 2 * Fi, di, kEpiSwiGLU, 0);
    h->pair_d = tc_pair_supported(Mi, di, Fi, kEpiResidCast, 0);
    h->pair_o = tc_pair_supported(Mi, di, hdi, kEpiResidCast, 0);
    h->fold_mo = h->fuse_read && h->pair_o && tc_pair_supported(Mi, di, hdi + c.d_v, kEpiResidCast, 0);
    h->chain_mlp = h->pair_o && h->pair_gu && h->pair_d;
  }
  h->ld_att = c.n_heads * c.head_dim + (h->fold_mo ? c.d_v : 0);
  const size_t ldw_o = size_t(h->ld_att);  // W_o rows: [W_o | W_mo] with fold_mo
  struct {
    void** p;
    size_t bytes;
  } plan[] = {
      {&h->w_qkv, L * h->Nqkv * d * es}, {&h->w_o, L * d * ldw_o * es},     {&h->w_gu, L * 2 * F * d * es},
      {&h->w_d, L * d * F * es},         {&h->w_mq, L * dk * d * es},       {&h->w_mo, L * d * dv * es},
      {&h->w_mkv, L * (dk + dv) * d * es}, {&h->g1, L * d * es},            {&h->g2, L * d * es},
      {&h->memtok, size_t(c.n_mem) * d * es},
      {reinterpret_cast<void**>(&h->rope), M * (c.head_dim / 2) * sizeof(float2)},
      {reinterpret_cast<void**>(&h->rope_h), M * (c.head_dim / 2) * sizeof(__half2)},
      {reinterpret_cast<void**>(&h->err), sizeof(int)},
  };
  for (auto& e : plan) {
    *e.p = h->alloc(e.bytes);
    if (!*e.p) return bail(fail(RMT_ENOMEM, "device allocation failed"));
  }
  rmt_status st = pack_weights(h, weights);
  if (st != RMT_OK) return bail(st);
  // bf16 mode: the tensor-core operands are f16 (3 more mantissa bits than bf16, same MMA
  // rate); the bf16 weight values convert exactly (bar magnitudes below 2^-17).
  if (h->bf16) {
    const size_t L_ = c.n_layers, d_ = c.d_model, F_ = c.d_ff;
    const struct {
      void* p;
      size_t n;
    } ops[] = {{h->w_qkv, L_ * h->Nqkv * d_}, {h->w_o, L_ * d_ * size_t(h->ld_att)}, {h->w_gu, L_ * 2 * F_ * d_},
               {h->w_d, L_ * d_ * F_},        {h->w_mq, L_ * c.d_k * d_},    {h->w_mo, L_ * d_ * c.d_v}};
    for (const auto& o : ops)
      if (launch_bf16_to_f16(o.p, o.n, 0) != cudaSuccess) return bail(fail(RMT_ECUDA, "weight conversion failed"));
  }
  // RMSNorm gains folded into the projections that consume the normalized rows
  if (launch_scale_cols(h->w_qkv, h->g1, c.n_layers, h->Nqkv, c.d_model, h->bf16, h->bf16, 0) != cudaSuccess ||
      launch_scale_cols(h->w_gu, h->g2, c.n_layers, 2 * c.d_ff, c.d_model, h->bf16, h->bf16, 0) != cudaSuccess)
    return bail(fail(RMT_ECUDA, "gain folding failed"));
  // RoPE table: angle p * theta^(-2i/dh) at segment-local position p, in double precision
  {
    const int half = c.head_dim / 2;
    std::vector<float2> tab(M * half);
    for (size_t p = 0; p < M; ++p)
      for (int i = 0; i < half; ++i) {
        const double ang = double(p) * std::pow(double(c.rope_theta), -2.0 * i / c.head_dim);
        tab[p * half + i] = make_float2(float(std::cos(ang)), float(std::sin(ang)));
      }
    std::vector<__half2> tab_h(tab.size());
    for (size_t i = 0; i < tab.size(); ++i) tab_h[i] = __floats2half2_rn(tab[i].x, tab[i].y);
    if (cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(h->rope_h, tab_h.data(), tab_h.size() * sizeof(__half2), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(RMT_ECUDA, "rope table upload failed"));
  }
  if (cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess) return bail(fail(RMT_ECUDA, "cudaMemset failed"));
  if ((st = reserve_acts(h, 1)) != RMT_OK) return bail(st);
  if (cudaDeviceSynchronize() != cudaSuccess) return bail(fail(RMT_ECUDA, "weight packing failed"));
  *out = h;
  return RMT_OK;
}

namespace {

// Sequences of a forward: token counts, checked. A sequence needs at least one token; t0 of
// every cell (an int) must stay in range.
rmt_status check_lengths(int32_t batch, const int32_t* n_tokens, std::vector<int>& T, size_t& total) {
  if (batch <= 0) return fail(RMT_EINVAL, "batch must be positive");
  if (!n_tokens) return fail(RMT_EINVAL, "n_tokens is null");
  T.assign(n_tokens, n_tokens + batch);
  total = 0;
  for (int v : T) {
    if (v <= 0) return fail(RMT_EINVAL, "every sequence needs at least one token");
    total += size_t(v);
  }
  if (total > size_t(INT32_MAX) / 2) return fail(RMT_EINVAL, "too many tokens");
  return RMT_OK;
}

rmt_status forward_impl(rmt_handle* h, const void* emb, const std::vector<int>& T, size_t total_tokens,
                        rmt_schedule schedule, const float* in_A, const float* in_z, void* out_hidden, float* out_A,
                        float* out_z, void* stream) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  if ((in_A == nullptr) != (in_z == nullptr)) return fail(RMT_EINVAL, "in_A and in_z must both be given or both be NULL");
  if (!emb || !out_hidden) return fail(RMT_EINVAL, "emb and out_hidden must not be null");
  if (schedule != RMT_DIAGONAL && schedule != RMT_SEQUENTIAL) return fail(RMT_EINVAL, "unknown schedule");
  DeviceGuard guard(h->dev);
  const rmt_cfg& c = h->cfg;
  const int B = static_cast<int>(T.size());
  RMT_TRY(reserve_acts(h, B));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = size_t(c.d_model) * h->es;
  const size_t io_bytes = total_tokens * row_bytes;
  const auto key = std::make_pair(T, int(schedule));
  auto it = h->tables.find(key);
  if (it == h->tables.end()) {
    // keep at most kMaxTables cell tables on the device: drop the oldest (cudaFree waits for
    // the device, so no forward still reads it)
    while (h->tables.size() >= rmt_handle::kMaxTables && !h->table_order.empty()) {
      auto old = h->tables.find(h->table_order.front());
      if (old != h->tables.end()) {
        if (old->second.dev) cudaFree(old->second.dev);
        h->tables.erase(old);
      }
      h->table_order.pop_front();
    }
    Table t;
    build_table(c.n_layers, c.seg_len, c.n_mem, T, schedule, t);
#ifdef RMT_DEBUG
    for (Cell& x : t.cells) {  // the buffers this forward's cells address, for the in-kernel checks
      x.lim_L = c.n_layers;
      x.lim_state = B * c.n_layers;
      x.lim_slot = B * n_slots(c.n_layers);
      x.lim_M = h->M;
      x.lim_nmem = c.n_mem;
      x.lim_tokens = static_cast<long long>(total_tokens);
      x.lim_err = h->err;
    }
#endif
    if (cudaMalloc(&t.dev, sizeof(Cell) * t.cells.size()) != cudaSuccess)
      return fail(RMT_ENOMEM, "cell table allocation failed");
    if (cudaMemcpy(t.dev, t.cells.data(), sizeof(Cell) * t.cells.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(t.dev);
      return fail(RMT_ECUDA, "cell table upload failed");
    }
    it = h->tables.emplace(key, std::move(t)).first;
    h->table_order.push_back(key);
  }
  const Table& t = it->second;
  const size_t ncell = t.cells.size();
  size_t n_segments = 0;
  for (int v : T) n_segments += size_t((v + c.seg_len - 1) / c.seg_len);
  // page-locked host buffers: one copy per segment on side streams, each segment's input just
  // ahead of the step that assembles it and its output right after the step that emits it
  const bool in_pinned = is_pinned_host_ptr(emb), out_pinned = is_pinned_host_ptr(out_hidden);
  if ((in_pinned || out_pinned) && !h->copy_resources(n_segments))
    return fail(RMT_ECUDA, "copy stream or event creation failed");
  auto seg_ord = [&](const Cell& x) { return size_t(t.seg_base[x.b]) + size_t(x.s); };
  auto seg_rows = [&](const Cell& x) { return size_t(x.m - c.n_mem); };
  const void* emb_dev = emb;
  if (is_host_ptr(emb)) {
    if (h->emb_stage_bytes < io_bytes) {
      if (h->emb_stage) cudaFree(h->emb_stage);
      h->emb_stage = nullptr;
      h->emb_stage_bytes = 0;
      if (cudaMalloc(&h->emb_stage, io_bytes) != cudaSuccess) return fail(RMT_ENOMEM, "staging allocation failed");
      h->emb_stage_bytes = io_bytes;
    }
    if (in_pinned) {
      // the staging buffer may still be read by an earlier forward on `st`
      RMT_CUDA(cudaEventRecord(h->copy_events[0], st));
      RMT_CUDA(cudaStreamWaitEvent(h->h2d, h->copy_events[0], 0));
      // segments in the order their layer-0 cells run
      for (size_t i = 0; i < ncell; ++i) {
        const Cell& x = t.cells[i];
        if (x.l != 0) continue;
        const size_t o = size_t(x.t0) * row_bytes;
        RMT_CUDA(cudaMemcpyAsync(static_cast<char*>(h->emb_stage) + o, static_cast<const char*>(emb) + o,
                                 seg_rows(x) * row_bytes, cudaMemcpyHostToDevice, h->h2d));
        RMT_CUDA(cudaEventRecord(h->copy_events[2 + 2 * seg_ord(x)], h->h2d));
      }
    } else {
      RMT_CUDA(cudaMemcpyAsync(h->emb_stage, emb, io_bytes, cudaMemcpyHostToDevice, st));
    }
    emb_dev = h->emb_stage;
  }
  void* out_dev = out_hidden;
  const bool out_host = is_host_ptr(out_hidden);
  if (out_host) {
    if (h->out_stage_bytes < io_bytes) {
      if (h->out_stage) cudaFree(h->out_stage);
      h->out_stage = nullptr;
      h->out_stage_bytes = 0;
      if (cudaMalloc(&h->out_stage, io_bytes) != cudaSuccess) return fail(RMT_ENOMEM, "staging allocation failed");
      h->out_stage_bytes = io_bytes;
    }
    out_dev = h->out_stage;
  }
  if (h->trace_cap < ncell) {
    if (h->trace) cudaFree(h->trace);
    h->trace = nullptr;
    h->trace_cap = 0;
    if (cudaMalloc(&h->trace, 3 * sizeof(int) * ncell) != cudaSuccess) return fail(RMT_ENOMEM, "trace allocation failed");
    h->trace_cap = ncell;
  }
  const size_t BL = size_t(B) * c.n_layers;
  if (in_A) {  // continue from the caller's state (the state after an earlier run's last segment)
    RMT_CUDA(cudaMemcpyAsync(h->A, in_A, BL * c.d_k * c.d_v * sizeof(float), cudaMemcpyDefault, st));
    RMT_CUDA(cudaMemcpyAsync(h->z, in_z, BL * c.d_k * sizeof(float), cudaMemcpyDefault, st));
  } else {
    RMT_CUDA(cudaMemsetAsync(h->A, 0, BL * c.d_k * c.d_v * sizeof(float), st));
    RMT_CUDA(cudaMemsetAsync(h->z, 0, BL * c.d_k * sizeof(float), st));
  }
  const bool split_in = in_pinned && emb_dev != emb, split_out = out_host && out_pinned;
  NvtxRange fwd_range(schedule == RMT_DIAGONAL ? "rmt_forward diagonal" : "rmt_forward sequential");
  char step_name[48];
  for (int step = 0; step < int(t.off.size()); ++step) {
    const int off = t.off[step], G = t.cnt[step];
    snprintf(step_name, sizeof(step_name), "step %d (%d cells)", step, G);
    NvtxRange step_range(step_name);
    if (split_in)
      for (int i = 0; i < t.n_first[step]; ++i)
        RMT_CUDA(cudaStreamWaitEvent(st, h->copy_events[2 + 2 * seg_ord(t.cells[off + i])], 0));
    cudaError_t e = enqueue_step(h, t, step, emb_dev, out_dev, st);
    if (e != cudaSuccess) return fail(RMT_ECUDA, std::string("launch failed: ") + cudaGetErrorString(e));
    if (split_out && t.n_last[step] > 0) {
      cudaEvent_t done = h->copy_events[3 + 2 * seg_ord(t.cells[off + G - 1])];
      RMT_CUDA(cudaEventRecord(done, st));
      RMT_CUDA(cudaStreamWaitEvent(h->d2h, done, 0));
      for (int i = G - t.n_last[step]; i < G; ++i) {
        const Cell& x = t.cells[off + i];
        const size_t o = size_t(x.t0) * row_bytes;
        RMT_CUDA(cudaMemcpyAsync(static_cast<char*>(out_hidden) + o, static_cast<const char*>(out_dev) + o,
                                 seg_rows(x) * row_bytes, cudaMemcpyDeviceToHost, h->d2h));
      }
    }
  }
  if (split_out) {
    RMT_CUDA(cudaEventRecord(h->copy_events[1], h->d2h));
    RMT_CUDA(cudaStreamWaitEvent(st, h->copy_events[1], 0));
  } else if (out_host) {
    RMT_CUDA(cudaMemcpyAsync(out_hidden, out_dev, io_bytes, cudaMemcpyDeviceToHost, st));
  }
  if (out_A) RMT_CUDA(cudaMemcpyAsync(out_A, h->A, BL * c.d_k * c.d_v * sizeof(float), cudaMemcpyDefault, st));
  if (out_z) RMT_CUDA(cudaMemcpyAsync(out_z, h->z, BL * c.d_k * sizeof(float), cudaMemcpyDefault, st));
  h->traced_cells = int(ncell);
  RMT_CUDA(cudaGetLastError());
  return RMT_OK;
}

}  // namespace

rmt_status rmt_forward(rmt_handle* h, const void* emb, int32_t n_segments, rmt_schedule schedule, void* out_hidden,
                       float* out_A, float* out_z, void* stream) {
  return rmt_forward_resume(h, emb, n_segments, schedule, nullptr, nullptr, out_hidden, out_A, out_z, stream);
}

rmt_status rmt_forward_resume(rmt_handle* h, const void* emb, int32_t n_segments, rmt_schedule schedule,
                              const float* in_A, const float* in_z, void* out_hidden, float* out_A, float* out_z,
                              void* stream) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  if (n_segments <= 0) return fail(RMT_EINVAL, "n_segments must be positive");
  if (int64_t(n_segments) * h->cfg.seg_len > INT32_MAX / 2) return fail(RMT_EINVAL, "too many tokens");
  const int32_t tokens = n_segments * h->cfg.seg_len;
  return rmt_forward_batch(h, emb, 1, &tokens, schedule, in_A, in_z, out_hidden, out_A, out_z, stream);
}

rmt_status rmt_forward_batch(rmt_handle* h, const void* emb, int32_t batch, const int32_t* n_tokens,
                             rmt_schedule schedule, const float* in_A, const float* in_z, void* out_hidden,
                             float* out_A, float* out_z, void* stream) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  std::vector<int> T;
  size_t total = 0;
  RMT_TRY(check_lengths(batch, n_tokens, T, total));
  return forward_impl(h, emb, T, total, schedule, in_A, in_z, out_hidden, out_A, out_z, stream);
}

rmt_status rmt_full_attention_forward(rmt_handle* h, const void* emb, int32_t n_tokens, void* out_hidden,
                                      void* stream) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  if (!emb || !out_hidden) return fail(RMT_EINVAL, "emb and out_hidden must not be null");
  if (!h->bf16 || h->split) return fail(RMT_EINVAL, "the full-attention forward needs an RMT_BF16 handle");
  if (n_tokens <= 0) return fail(RMT_EINVAL, "n_tokens must be positive");
  const rmt_cfg& c = h->cfg;
  if (h->ss_parts > 32 || c.d_model % h->ss_parts || (c.d_model / h->ss_parts) % 4)
    return fail(RMT_EINVAL, "d_model does not fit the RMSNorm statistics blocks");
  DeviceGuard guard(h->dev);
  RMT_TRY(full_buffers(h, n_tokens));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int L = c.n_layers, d = c.d_model, T = n_tokens;
  const size_t io_bytes = size_t(T) * d * h->es;
  const void* emb_dev = emb;
  if (is_host_ptr(emb)) {
    if (h->emb_stage_bytes < io_bytes) {
      if (h->emb_stage) cudaFree(h->emb_stage);
      h->emb_stage = nullptr;
      h->emb_stage_bytes = 0;
      if (cudaMalloc(&h->emb_stage, io_bytes) != cudaSuccess) return fail(RMT_ENOMEM, "staging allocation failed");
      h->emb_stage_bytes = io_bytes;
    }
    RMT_CUDA(cudaMemcpyAsync(h->emb_stage, emb, io_bytes, cudaMemcpyHostToDevice, st));
    emb_dev = h->emb_stage;
  }
  void* out_dev = out_hidden;
  const bool out_host = is_host_ptr(out_hidden);
  if (out_host) {
    if (h->out_stage_bytes < io_bytes) {
      if (h->out_stage) cudaFree(h->out_stage);
      h->out_stage = nullptr;
      h->out_stage_bytes = 0;
      if (cudaMalloc(&h->out_stage, io_bytes) != cudaSuccess) return fail(RMT_ENOMEM, "staging allocation failed");
      h->out_stage_bytes = io_bytes;
    }
    out_dev = h->out_stage;
  }
  auto launch_fail = [&](cudaError_t e) {
    return fail(RMT_ECUDA, std::string("launch failed: ") + cudaGetErrorString(e));
  };
  // the input: the embeddings into slot 0 (fp32 and the f16 copy), and their RMSNorm statistics
  cudaError_t e = launch_assemble(h->fcells, 1, emb_dev, h->memtok, h->fx, h->fxb, T, 0, d, true, h->err, st);
  if (e == cudaSuccess) e = launch_row_ssq(h->fx, h->fss1, T, d, h->ss_parts, st);
  if (e != cudaSuccess) return launch_fail(e);
  for (int l = 0; l < L; ++l) {
    const Cell* cell = h->fcells + l;
    if ((e = run_proj_full(h, kProjQkv, cell, st)) != cudaSuccess) return launch_fail(e);
    AttnArgs a{h->fqkv, h->fatt, T, c.n_heads, c.n_kv_heads, c.head_dim, 1, cell, kByLayer, L, h->err};
    e = attention_tc_supported(c.head_dim) ? launch_attention_tc(h->fm_qkv, h->fm_qkv_tail, a, /*f16=*/true, st)
                                           : launch_attention(a, kElemF16, st);
    if (e != cudaSuccess) return launch_fail(e);
    if ((e = run_proj_full(h, kProjO, cell, st)) != cudaSuccess) return launch_fail(e);
    if ((e = run_proj_full(h, kProjGateUp, cell, st)) != cudaSuccess) return launch_fail(e);
    if ((e = run_proj_full(h, kProjDown, cell, st)) != cudaSuccess) return launch_fail(e);
  }
  if ((e = launch_emit(h->fcells + L - 1, 1, h->fx, out_dev, T, 0, d, true, st)) != cudaSuccess) return launch_fail(e);
  if (out_host) RMT_CUDA(cudaMemcpyAsync(out_hidden, out_dev, io_bytes, cudaMemcpyDeviceToHost, st));
  RMT_CUDA(cudaGetLastError());
  return RMT_OK;
}

rmt_status rmt_reserve(rmt_handle* h, int32_t max_batch) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  if (max_batch <= 0) return fail(RMT_EINVAL, "max_batch must be positive");
  DeviceGuard guard(h->dev);
  return reserve_acts(h, max_batch);
}

rmt_status rmt_get_trace(rmt_handle* h, int32_t* out_dls, size_t cap) {
  if (!h || !out_dls) return fail(RMT_EINVAL, "null argument");
  if (h->traced_cells < 0) return fail(RMT_ESTATE, "no forward has run on this handle");
  if (cap < 3 * size_t(h->traced_cells)) return fail(RMT_EINVAL, "out_dls capacity too small");
  DeviceGuard guard(h->dev);
  RMT_CUDA(cudaDeviceSynchronize());
  RMT_CUDA(cudaMemcpy(out_dls, h->trace, 3 * sizeof(int) * h->traced_cells, cudaMemcpyDeviceToHost));
  return RMT_OK;
}

rmt_status rmt_sync(rmt_handle* h, void* stream) {
  int* err = nullptr;
  if (h) {
    err = h->err;
  } else {
    const Cell* cells = nullptr;
    rmt_status s = device_scratch(1, &cells, &err);
    if (s != RMT_OK) return s;
  }
  DeviceGuard guard(h ? h->dev : -1);
  RMT_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  RMT_CUDA(cudaGetLastError());
  int word = 0;
  RMT_CUDA(cudaMemcpy(&word, err, sizeof(int), cudaMemcpyDeviceToHost));
  if (word) {
    RMT_CUDA(cudaMemset(err, 0, sizeof(int)));
    if (word & kErrBounds)
      return fail(RMT_EDEBUG, "a kernel's bounds check failed: a cell index fell outside its buffers (error word " +
                                  std::to_string(word) + ")");
    if (word == kErrF16Range)
      return fail(RMT_ERANGE,
                  "a value of magnitude 65520 or more was stored as an f16 tensor-core operand (bf16 mode): the "
                  "outputs of this forward are not valid");
    return fail(RMT_ETIMEOUT, "a bounded device wait gave up (error word " + std::to_string(word) + ")");
  }
  return RMT_OK;
}

rmt_status rmt_probe(rmt_handle* h, uint32_t mask) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  DeviceGuard guard(h->dev);
  RMT_CUDA(cudaDeviceSynchronize());
  h->probe_mask = mask;
  h->probe_recs.clear();
  h->probe_used = 0;
  h->launches = 0;
  return RMT_OK;
}

rmt_status rmt_probe_read(rmt_handle* h, rmt_kernel kind, double* ms, int64_t* launches, double* flops, double* bytes,
                          int64_t* all_launches) {
  if (!h) return fail(RMT_EINVAL, "null handle");
  if (int(kind) < 0 || int(kind) >= RMT_K_COUNT) return fail(RMT_EINVAL, "unknown kernel kind");
  DeviceGuard guard(h->dev);
  RMT_CUDA(cudaDeviceSynchronize());
  double t = 0, f = 0, b = 0;
  int64_t nl = 0;
  for (const auto& r : h->probe_recs) {
    if (r.kind != int(kind)) continue;
    float e = 0.f;
    RMT_CUDA(cudaEventElapsedTime(&e, r.a, r.b));
    t += e;
    f += r.flops;
    b += r.bytes;
    ++nl;
  }
  if (ms) *ms = t;
  if (launches) *launches = nl;
  if (flops) *flops = f;
  if (bytes) *bytes = b;
  if (all_launches) *all_launches = h->launches;
  return RMT_OK;
}

rmt_status rmt_destroy(rmt_handle* h) {
  if (!h) return RMT_OK;
  {
    DeviceGuard guard(h->dev);
    cudaDeviceSynchronize();
    h->release();
  }
  delete h;
  return RMT_OK;
}

// ----------------------------------------------------------------- kernel-level entry points

rmt_status rmt_wait_selftest(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 10000000) return fail(RMT_EINVAL, "limit_us must be in 1 .. 10^7");
  int* err = nullptr;
  const Cell* cells = nullptr;
  RMT_TRY(device_scratch(1, &cells, &err));
  RMT_CUDA(launch_wait_selftest(err, 1000ull * limit_us, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
}

rmt_status rmt_bounds_selftest(void* stream) {
#ifdef RMT_DEBUG
  int* err = nullptr;
  const Cell* cells = nullptr;
  RMT_TRY(device_scratch(1, &cells, &err));
  RMT_CUDA(launch_bounds_selftest(err, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
#else
  (void)stream;
  return fail(RMT_ESTATE, "rmt_bounds_selftest needs the debug build (librmt_debug.so)");
#endif
}

rmt_status rmt_grouped_gemm_bf16(const void* A, const void* B, void* C, int32_t G, int32_t M, int32_t N, int32_t K,
                                 rmt_dtype out_dtype, void* stream) {
  if (!A || !B || !C) return fail(RMT_EINVAL, "null pointer");
  if (G <= 0 || M <= 0 || N <= 0 || K <= 0) return fail(RMT_EINVAL, "sizes must be positive");
  if (K % 64 || N % 64) return fail(RMT_EINVAL, "K and N must be multiples of 64");
  if (out_dtype != RMT_F32 && out_dtype != RMT_BF16) return fail(RMT_EINVAL, "bad out_dtype");
  const Cell* cells = nullptr;
  int* err = nullptr;
  RMT_TRY(device_scratch(G, &cells, &err));
  CUtensorMap ta, tb;
  const int epi = out_dtype == RMT_F32 ? kEpiStoreF32 : kEpiStoreAct;
  EpiParams ep{};
  ep.out = C;
  ep.ldo = N;
  ep.out_mode = kByLayer;
  TcGemmArgs a{M, N, K, G, cells, G, kByLayer, static_cast<EpiKind>(epi), ep, err};
  if (tc_pair_supported(M, N, K, epi, 0)) {  // widths in multiples of 256: CTA-pair kernel
    a.nt = pair_pick_nt(M, G, N / 256);
    if (!make_tmap_bf16_3d(&ta, A, K, M, G, static_cast<uint32_t>(a.nt / 2)) ||
        !make_tmap_bf16_3d(&tb, B, K, N, G, 128))
      return fail(RMT_EINVAL, "tensor map encoding failed (pointers must be 16-byte aligned)");
    RMT_CUDA(launch_tc_pair_gemm(tb, ta, a, /*f16=*/false, static_cast<cudaStream_t>(stream)));
    return RMT_OK;
  }
  const int bn = tc_pick_bn(N, epi, 0);
  if (!make_tmap_bf16_3d(&ta, A, K, M, G, 128) || !make_tmap_bf16_3d(&tb, B, K, N, G, bn))
    return fail(RMT_EINVAL, "tensor map encoding failed (pointers must be 16-byte aligned)");
  RMT_CUDA(launch_tc_gemm(ta, tb, ta, a, bn, /*f16=*/false, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
}

rmt_status rmt_attention(const void* qkv, void* out, int32_t G, int32_t M, int32_t H, int32_t Hkv, int32_t dh,
                         rmt_dtype dtype, void* stream) {
  if (!qkv || !out) return fail(RMT_EINVAL, "null pointer");
  if (G <= 0 || M <= 0 || H <= 0 || Hkv <= 0 || H % Hkv) return fail(RMT_EINVAL, "bad sizes");
  if (dh != 32 && dh != 64 && dh != 128) return fail(RMT_EINVAL, "dh must be 32, 64 or 128");
  if (dtype != RMT_F32 && dtype != RMT_BF16) return fail(RMT_EINVAL, "bad dtype");
  const Cell* cells = nullptr;
  int* err = nullptr;
  RMT_TRY(device_scratch(G, &cells, &err));
  AttnArgs a{qkv, out, M, H, Hkv, dh, G, cells, kByLayer, G, err};
  if (dtype == RMT_BF16 && attention_tc_supported(dh)) {
    CUtensorMap tm, tt;
    const uint64_t inner = uint64_t(H + 2 * Hkv) * dh;
    if (!make_tmap_bf16_3d(&tm, qkv, inner, M, G, 128) ||
        !make_tmap_bf16_3d(&tt, qkv, inner, M, G, attn_tail_box(M, H, Hkv)))
      return fail(RMT_EINVAL, "tensor map encoding failed (qkv must be 16-byte aligned)");
    RMT_CUDA(launch_attention_tc(tm, tt, a, /*f16=*/false, static_cast<cudaStream_t>(stream)));
    return RMT_OK;
  }
  RMT_CUDA(launch_attention(a, dtype == RMT_BF16 ? kElemBF16 : kElemF32, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
}

rmt_status rmt_memory_read(const float* q, const float* A, const float* z, void* o, int32_t G, int32_t M, int32_t dk,
                           int32_t dv, float eps, rmt_dtype dtype, void* stream) {
  if (!q || !A || !z || !o) return fail(RMT_EINVAL, "null pointer");
  if (!aligned16(q) || !aligned16(A) || !aligned16(z) || !aligned16(o))
    return fail(RMT_EINVAL, "q, A, z and o must be 16-byte aligned");
  if (G <= 0 || M <= 0 || dk <= 0 || dv <= 0 || dk % 32 || dv % 32 || dk > 128 || dv > 128)
    return fail(RMT_EINVAL, "bad sizes");
  if (dtype != RMT_F32 && dtype != RMT_BF16) return fail(RMT_EINVAL, "bad dtype");
  const Cell* cells = nullptr;
  int* err = nullptr;
  RMT_TRY(device_scratch(G, &cells, &err));
  MemReadArgs a{q, A, z, o, M, dk, dv, eps, G, cells, kByLayer, kByLayer, G};
  RMT_CUDA(launch_mem_read(a, dtype == RMT_BF16 ? kElemBF16 : kElemF32, static_cast<cudaStream_t>(stream), err));
  return RMT_OK;
}

namespace {
rmt_status memory_update_impl(const float* k, const float* v, float* A, float* z, int32_t G, int32_t n, int32_t dk,
                              int32_t dv, float eps, int seq, void* stream) {
  if (!k || !v || !A || !z) return fail(RMT_EINVAL, "null pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(A) || !aligned16(z))
    return fail(RMT_EINVAL, "k, v, A and z must be 16-byte aligned");
  if (G <= 0 || n <= 0 || n > 64 || dk % 32 || dv % 32 || dk <= 0 || dv <= 0 || dk > 128 || dv > 128)
    return fail(RMT_EINVAL, "bad sizes");
  const Cell* cells = nullptr;
  RMT_TRY(device_scratch(G, &cells, nullptr));
  MemUpdateArgs a{nullptr, 0, k, v, A, z, n, dk, dv, eps, G, cells, kByLayer, kByLayer, G, nullptr, 0, 0, seq};
  RMT_CUDA(launch_mem_update(a, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
}
}  // namespace

rmt_status rmt_memory_update(const float* k, const float* v, float* A, float* z, int32_t G, int32_t n, int32_t dk,
                             int32_t dv, float eps, void* stream) {
  return memory_update_impl(k, v, A, z, G, n, dk, dv, eps, 0, stream);
}

rmt_status rmt_memory_update_sequential(const float* k, const float* v, float* A, float* z, int32_t G, int32_t n,
                                        int32_t dk, int32_t dv, float eps, void* stream) {
  return memory_update_impl(k, v, A, z, G, n, dk, dv, eps, 1, stream);
}

rmt_status rmt_rmsnorm(const float* x, const void* g, void* y, int32_t rows, int32_t d, float eps, rmt_dtype dtype,
                       void* stream) {
  if (!x || !g || !y) return fail(RMT_EINVAL, "null pointer");
  if (rows <= 0 || d <= 0 || d % 4) return fail(RMT_EINVAL, "bad sizes");
  if (dtype != RMT_F32 && dtype != RMT_BF16) return fail(RMT_EINVAL, "bad dtype");
  const Cell* cells = nullptr;
  RMT_TRY(device_scratch(1, &cells, nullptr));
  RmsArgs a{x, g, y, rows, d, eps, 1, cells, kByLayer, kByLayer, 1};
  RMT_CUDA(launch_rmsnorm(a, dtype == RMT_BF16, static_cast<cudaStream_t>(stream)));
  return RMT_OK;
}

rmt_status rmt_memory_write(const float* y, const void* w_mkv, float* A, float* z, int32_t G, int32_t n, int32_t d,
                            int32_t dk, int32_t dv, float eps, rmt_dtype dtype, void* stream) {
  if (!y || !w_mkv || !A || !z) return fail(RMT_EINVAL, "null pointer");
  if (!aligned16(A) || !aligned16(z)) return fail(RMT_EINVAL, "A and z must be 16-byte aligned");
  if (G <= 0 || n <= 0 || n > 64 || d <= 0 || dk <= 0 || dv <= 0 || dk % 32 || dv % 32 || dk > 128 || dv > 128 ||
      n * (dk + dv) > 4096)
    return fail(RMT_EINVAL, "bad sizes");
  if (dtype != RMT_F32 && dtype != RMT_BF16) return fail(RMT_EINVAL, "bad dtype");
  const Cell* cells = nullptr;
  RMT_TRY(device_scratch(G, &cells, nullptr));
  const int nsplit = mem_kv_splits(d, dtype == RMT_BF16);
  float* part = nullptr;
  RMT_TRY(partial_scratch(size_t(G) * nsplit * n * (dk + dv), &part));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MemKvArgs ka{y, n, d, n, kByLayer, w_mkv, part, dk + dv, G, cells, G};
  RMT_CUDA(launch_mem_kv(ka, dtype == RMT_BF16, st));
  MemUpdateArgs ua{part, mem_kv_written_splits(G, n, d, dtype == RMT_BF16), nullptr, nullptr, A, z, n, dk, dv, eps, G,
                   cells, kByLayer, kByLayer, G, nullptr, 0, 0};
  RMT_CUDA(launch_mem_update(ua, st));
  return RMT_OK;
}

}  // extern "C"

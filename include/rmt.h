/*
 * rmt.h -- C ABI of the diagonal-batched ARMT prefill library (librmt.so, sm_100a).
 *
 * The method: "Diagonal Batching Unlocks Parallelism in Recurrent Memory Transformers
 * for Long Contexts" (arXiv 2506.05229; abstract, and the skill page of the same title:
 * "Core Concept", "Architecture Overview", "Implementation"). An ARMT runs a grid of
 * (layer l, segment s) cells; cell (l, s) needs the output of (l-1, s) and layer l's
 * associative memory after (l, s-1). The grid is swept in anti-diagonals d = l + s and
 * every cell of a diagonal runs in the same grouped launches, each cell with its own
 * layer's weights. The result is the sequential model's result, reordered only.
 *
 * Conventions for every entry point:
 *  - Status codes only: no exceptions or aborts cross the ABI. A non-OK status leaves
 *    a message for rmt_last_error() (thread-local) and leaves any handle usable.
 *  - "device or host" pointers may point to device memory or to host memory (pinned or
 *    pageable); host buffers are copied inside the call, on the given stream.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *    stream) and the call returns without waiting, unless stated otherwise. Device-side
 *    faults of a bounded wait show up at rmt_sync() as RMT_ETIMEOUT.
 *  - Matrices are row-major; projection weights are [out_features, in_features] like
 *    nn.Linear. bf16 values are passed as their 16-bit patterns.
 */
#ifndef RMT_H
#define RMT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RMT_OK = 0,
  RMT_EINVAL = 1,    /* bad argument: null pointer, unsupported shape, size out of range */
  RMT_ENOMEM = 2,    /* device or pinned allocation failed */
  RMT_ECUDA = 3,     /* a CUDA runtime call or launch failed */
  RMT_ETIMEOUT = 4,  /* a bounded device-side wait gave up (reported by rmt_sync) */
  RMT_ESTATE = 5,    /* call not valid in this state (e.g. trace before any forward) */
  RMT_ERANGE = 6,    /* bf16 mode: a value overflowed an f16 tensor-core operand (reported by rmt_sync) */
  RMT_EDEBUG = 7     /* debug build (librmt_debug.so) only: an in-kernel bounds check failed (rmt_sync) */
} rmt_status;

typedef enum { RMT_DIAGONAL = 0, RMT_SEQUENTIAL = 1 } rmt_schedule;

/* Storage type of weights, embeddings, outputs and inter-kernel activations.
 * RMT_F32: every GEMM is an fp32 FMA kernel (no tensor cores).
 * RMT_BF16: weights, embeddings and outputs are bf16. GEMMs and attention run on tensor cores
 * with f16 operands and fp32 accumulation; the residual stream, softmax, RMSNorm statistics
 * and the memory state stay fp32. f16 has 3 more mantissa bits than bf16, which the
 * delta-rule memory update needs, and a smaller range: the values stored as f16 operands --
 * the residual stream (embeddings included) before each projection, q/k/v, the SwiGLU output
 * silu(gate)*up and the memory read-out -- must stay below 65504 in magnitude. Weights are
 * converted to f16 at rmt_create, with the RMSNorm gains folded into the projections that
 * follow them (exact for bf16 magnitudes from 2^-17 up; smaller ones lose bits).
 * A forward that stores an operand of magnitude 65520 or more (which rounds to infinity) is
 * reported by rmt_sync as RMT_ERANGE; its outputs are then not valid. */
/* RMT_BF16_SPLIT: bf16 storage and f16 range as RMT_BF16, with every activation operand of a
 * tensor-core GEMM carried as two f16 terms (hi = f16(v), lo = f16(v - hi): about 22
 * significant bits), so each projection runs twice the MMAs of RMT_BF16 against the same
 * weights; q, k and v stay fp32 and attention runs on the fp32 FMA kernel. The memory
 * recurrence carries rounding differences from segment to segment and amplifies them, so
 * over hundreds of segments RMT_BF16's f16 rounding can drift past the bf16 tolerance of the
 * outputs and memory state where this mode does not; it costs about twice the GEMM time.
 * Needs d_k of 64 or 128. rmt_full_attention_forward does not take it. */
typedef enum { RMT_F32 = 0, RMT_BF16 = 1, RMT_BF16_SPLIT = 2 } rmt_dtype;

/* How a cell writes its n_mem memory rows (the delta rule of rmt_memory_update):
 * RMT_MEM_BATCHED: every row against the pre-update A, z (the rows' writes are summed).
 * RMT_MEM_SEQUENTIAL: the rows one after another, each against the state the earlier rows of
 * the cell left -- the per-token delta rule (rmt_memory_update_sequential). */
typedef enum { RMT_MEM_BATCHED = 0, RMT_MEM_SEQUENTIAL = 1 } rmt_mem_update;

/* Model shape. A cell has M = seg_len + n_mem rows: the segment's tokens followed by the
 * n_mem memory tokens. Limits (else RMT_EINVAL): all sizes > 0; n_heads % n_kv_heads == 0;
 * head_dim in {32, 64, 128}; d_k, d_v multiples of 32, at most 128; n_mem <= 64 and
 * n_mem*(d_k+d_v) <= 4096; d_ff % 64 == 0; d_model % 4 == 0.
 * RMT_BF16 also needs d_model, n_heads*head_dim and d_v multiples of 64, and projection
 * widths that tile by 256/128/64/32 columns: (n_heads+2*n_kv_heads)*head_dim in whole
 * heads, 2*d_ff by at least 128, d_model and d_k. */
typedef struct {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, d_ff, seg_len, n_mem, d_k, d_v;
  float rope_theta; /* RoPE base (500000 for the LLaMA-shaped models) */
  float rms_eps;    /* RMSNorm epsilon (1e-5) */
  float mem_eps;    /* associative-memory epsilon in both denominators (1e-6) */
  rmt_dtype dtype;
  rmt_mem_update mem_update; /* RMT_MEM_BATCHED or RMT_MEM_SEQUENTIAL */
} rmt_cfg;

/* Model weights, in cfg.dtype. Each `const void* const*` member is a host array of
 * n_layers pointers (one per layer); each pointer may be device or host memory.
 *   wq [H*dh, d]  wk [Hkv*dh, d]  wv [Hkv*dh, d]  wo [d, H*dh]
 *   w_gate [F, d]  w_up [F, d]  w_down [d, F]                 (SwiGLU MLP)
 *   w_mq [d_k, d]  w_mk [d_k, d]  w_mv [d_v, d]  w_mo [d, d_v] (associative memory)
 *   g_attn [d]  g_mlp [d]                                      (RMSNorm gains)
 *   mem_tokens [n_mem, d]: one matrix, appended after every segment at layer 0. */
typedef struct {
  const void* const* wq;
  const void* const* wk;
  const void* const* wv;
  const void* const* wo;
  const void* const* w_gate;
  const void* const* w_up;
  const void* const* w_down;
  const void* const* w_mq;
  const void* const* w_mk;
  const void* const* w_mv;
  const void* const* w_mo;
  const void* const* g_attn;
  const void* const* g_mlp;
  const void* mem_tokens;
} rmt_weights;

typedef struct rmt_handle rmt_handle;

/* Validate cfg, copy and pack the weights into library-owned device memory (on the
 * current CUDA device), allocate activations and state for one sequence. Synchronous. The
 * caller may free its weight buffers when this returns. *out is set only on RMT_OK. */
rmt_status rmt_create(const rmt_weights* weights, const rmt_cfg* cfg, rmt_handle** out);

/* Size the handle's activations and memory state for up to max_batch sequences per forward
 * (rmt_create sizes them for one). Synchronizes the device and reallocates when max_batch is
 * above the current size; a smaller max_batch is a no-op. A forward with a larger batch does
 * this itself, so calling it first keeps later forwards free of device allocations.
 * RMT_ENOMEM leaves the handle without activations until a later reservation succeeds. */
rmt_status rmt_reserve(rmt_handle* h, int32_t max_batch);

/* ARMT prefill of n_segments segments (batch 1).
 *   emb        [n_segments*seg_len, d_model] in cfg.dtype, device or host.
 *   out_hidden [n_segments*seg_len, d_model] in cfg.dtype, device or host: the last
 *              layer's hidden states at the segment-token rows (memory rows dropped).
 *   out_A      [n_layers, d_k, d_v] fp32 or NULL; out_z [n_layers, d_k] fp32 or NULL:
 *              the memory state after the last segment. The state starts at zero.
 * schedule RMT_DIAGONAL runs one grouped launch per step over all cells of an
 * anti-diagonal; RMT_SEQUENTIAL runs the same kernels one cell per step, segments
 * outermost. Both give the same bits. Asynchronous on `stream`; a handle runs one forward
 * at a time (calls on one handle must be ordered on one stream). */
rmt_status rmt_forward(rmt_handle* h, const void* emb, int32_t n_segments, rmt_schedule schedule,
                       void* out_hidden, float* out_A, float* out_z, void* stream);

/* rmt_forward starting from a given memory state instead of zeros: in_A [n_layers, d_k, d_v]
 * and in_z [n_layers, d_k] fp32, device or host, both given or both NULL (NULL: zeros, as
 * rmt_forward). The state after segment s depends only on the segments up to s, so a
 * sequence may be prefilled in chunks: running segments 0..S1-1, then resuming with the
 * state it returned over segments S1..S-1, gives the same bits as one run over 0..S-1.
 * in_A / in_z may alias out_A / out_z. Other arguments, errors and ordering as rmt_forward.
 * Streaming continuation of the recurrent memory (the pages' recurrence carries only A and z
 * from one segment to the next). */
rmt_status rmt_forward_resume(rmt_handle* h, const void* emb, int32_t n_segments, rmt_schedule schedule,
                              const float* in_A, const float* in_z, void* out_hidden, float* out_A, float* out_z,
                              void* stream);

/* Batched, variable-length ARMT prefill ("Implementation" of the diagonal-batching skill
 * page: a [B, T, D] input cut into ceil(T / seg_len) segments, the last one ending at T).
 *   batch      number of sequences, >= 1.
 *   n_tokens   host array [batch]: tokens of each sequence, each >= 1. Sequence b has
 *              ceil(n_tokens[b] / seg_len) segments; its last segment holds the remaining
 *              r = n_tokens[b] - (segments - 1) * seg_len tokens, followed as every segment by
 *              the n_mem memory tokens (positions r .. r + n_mem - 1 of that segment).
 *   emb        [sum(n_tokens), d_model] in cfg.dtype, device or host: the sequences packed one
 *              after another (equal lengths T: the row-major [batch, T, d_model] tensor).
 *   out_hidden same shape and packing: the last layer's hidden states at the token rows.
 *   in_A/in_z  [batch, n_layers, d_k, d_v] / [batch, n_layers, d_k] fp32 initial states,
 *              device or host, both given or both NULL (zeros); may alias out_A / out_z.
 *   out_A/out_z the same shapes, or NULL: each sequence's state after its last segment.
 * Sequences do not interact: each result is that of the sequence run alone. RMT_DIAGONAL
 * puts every cell (b, l, s) with l + s = d of all sequences into step d (layers ascending,
 * then sequences); RMT_SEQUENTIAL runs one cell per step, sequences outermost, then segments,
 * then layers. Both give the same bits. Grows the activations (rmt_reserve) when batch is
 * above the reserved size. The handle keeps the cell table of each (n_tokens, schedule) on
 * the device, at most 64 of them; a new one beyond that frees the oldest (which waits for
 * the device). RMT_EINVAL on a non-positive batch or length, or more than 2^30
 * tokens. Other behaviour as rmt_forward. */
rmt_status rmt_forward_batch(rmt_handle* h, const void* emb, int32_t batch, const int32_t* n_tokens,
                             rmt_schedule schedule, const float* in_A, const float* in_z, void* out_hidden,
                             float* out_A, float* out_z, void* stream);

/* The comparison model of the ARMT paper (arXiv 2506.05229 abstract: ARMT with diagonal
 * batching against full-attention LLaMA-1B at 131,072 tokens): the handle's decoder stack
 * without its associative memory -- no memory tokens, no memory read or write -- over one
 * sequence of n_tokens, causal over all of them, RoPE at positions 0 .. n_tokens-1, on the
 * handle's weights.
 *   emb        [n_tokens, d_model] bf16, device or host.
 *   out_hidden [n_tokens, d_model] bf16, device or host: the last layer's hidden states.
 * bf16 handles only (RMT_EINVAL otherwise, or for n_tokens <= 0). The first call with a
 * longer sequence allocates the activations for it (about 50 KB per token at the 1B shape)
 * and synchronizes the device; RMT_ENOMEM if they do not fit. Asynchronous on `stream`
 * otherwise; same ordering rules as rmt_forward. */
rmt_status rmt_full_attention_forward(rmt_handle* h, const void* emb, int32_t n_tokens, void* out_hidden,
                                      void* stream);

/* The execution order as int32 triples (step, layer, segment), one per cell, n_layers*
 * n_segments of them: steps ascend; within a diagonal step layers ascend. Host memory,
 * cap = capacity of out_dls in int32 elements (>= 3*L*S). Needs no GPU. */
rmt_status rmt_schedule_table(int32_t n_layers, int32_t n_segments, rmt_schedule schedule,
                              int32_t* out_dls, size_t cap);
rmt_status rmt_get_schedule(const rmt_handle* h, int32_t n_segments, rmt_schedule schedule,
                            int32_t* out_dls, size_t cap);

/* The execution order of rmt_forward_batch as int32 quadruples (step, sequence, layer,
 * segment), one per cell; n_segments is a host array [batch] (>= 1 each) and cap the capacity
 * of out_dbls in int32 elements (>= 4 * n_layers * sum(n_segments)). Needs no GPU. */
rmt_status rmt_schedule_table_batch(int32_t n_layers, int32_t batch, const int32_t* n_segments,
                                    rmt_schedule schedule, int32_t* out_dbls, size_t cap);

/* The (step, layer, segment) triples the device recorded for each cell during the last
 * forward, in schedule-table order (written by the memory-update kernel of each cell); after
 * rmt_forward_batch, the order of rmt_schedule_table_batch without its sequence column.
 * Synchronizes the device. RMT_ESTATE before the first forward. */
rmt_status rmt_get_trace(rmt_handle* h, int32_t* out_dls, size_t cap);

/* Wait for `stream`, then report (and clear) the handle's device error word: RMT_ETIMEOUT
 * if a bounded device wait gave up, RMT_ERANGE if the only fault since the last check is an
 * f16 operand overflow (see rmt_dtype), RMT_EDEBUG if a bounds check of the debug build
 * failed (see rmt_bounds_selftest), RMT_ECUDA on a CUDA error. With h == NULL the error
 * word of the kernel-level entry points on the current device is checked. */
rmt_status rmt_sync(rmt_handle* h, void* stream);

/* Check of the failure path: one CTA waits on an mbarrier that nothing signals, with the
 * bounded wait every kernel of this library uses, then on a global counter that nothing
 * increments, with the bounded wait of the chained projections, each limited here to limit_us
 * microseconds (1 .. 10^7; the kernels use 2 s). The waits give up, the CTA sets the device error word of
 * the kernel-level entry points and returns normally; rmt_sync(NULL, stream) then reports
 * RMT_ETIMEOUT (and clears the word), and the context stays usable. Asynchronous on stream. */
rmt_status rmt_wait_selftest(uint32_t limit_us, void* stream);

/* The debug build. librmt_debug.so is this library compiled with -DRMT_DEBUG, a stand-in for
 * a memory checker: every kernel reads its (layer, segment) cells through a check of each
 * index against the buffers the host sized for that forward (layer, state slice, residual
 * slot, rows, token rows); a violation is recorded in the error word, which rmt_sync reports
 * as RMT_EDEBUG, and the kernel continues with in-range indices, so no access leaves its
 * buffer. rmt_bounds_selftest checks that mechanism: one thread presents an out-of-range cell
 * to the check, and rmt_sync(NULL, stream) must then return RMT_EDEBUG with error word 64.
 * The release library returns RMT_ESTATE here. Asynchronous on stream. */
rmt_status rmt_bounds_selftest(void* stream);

/* Kernel kinds of one schedule step, in launch order (see rmt_forward). Kinds that are fused
 * into another kind's kernel launch nothing of their own and read zero in rmt_probe_read:
 * RMSNORM1 and RMSNORM2 always (their statistics come from the residual epilogues and their
 * gains are folded into the next projection's weights); MEMREAD in bf16 mode with
 * d_k = d_v = 64, where the read runs in the MEMQ kernel's epilogue (and then MEMO forms only
 * the operand copy and statistics, the O projection adding the read-out to the residual); and
 * O and DOWN in bf16 mode when O, gate/up and down all run on CTA pairs: the three projections
 * then run as one chained launch per step (the tiles of each projection start as soon as the
 * previous projection has stored the rows they read), reported under GATEUP with the flops
 * and bytes of all three. */
typedef enum {
  RMT_K_ASSEMBLE = 0,  /* layer-0 input: segment embeddings + memory tokens */
  RMT_K_MEMQ = 1,      /* memory-query projection (grouped GEMM), with the read when fused */
  RMT_K_MEMREAD = 2,   /* associative read */
  RMT_K_MEMO = 3,      /* read-out projection + residual (grouped GEMM) */
  RMT_K_RMSNORM1 = 4,
  RMT_K_QKV = 5,       /* QKV projection + RoPE (grouped GEMM) */
  RMT_K_ATTENTION = 6,
  RMT_K_O = 7,         /* output projection + residual (grouped GEMM) */
  RMT_K_RMSNORM2 = 8,
  RMT_K_GATEUP = 9,    /* gate/up projection + SwiGLU (grouped GEMM); or O + gate/up + down chained */
  RMT_K_DOWN = 10,     /* down projection + residual (grouped GEMM) */
  RMT_K_MEMKV = 11,    /* memory key/value projection of the memory-token rows */
  RMT_K_MEMUPDATE = 12,/* delta-rule update */
  RMT_K_EMIT = 13,     /* segment output */
  RMT_K_COUNT = 14
} rmt_kernel;

/* Start (or restart) timing every launch of the kernel kinds in `mask` (bit k = kind k)
 * in later forwards on this handle, with a CUDA event pair around each launch on the
 * forward's stream; mask 0 stops timing. Resets all probe counters. */
rmt_status rmt_probe(rmt_handle* h, uint32_t mask);

/* Probe totals since rmt_probe for one kind: summed event time in ms, launches, and the
 * algorithmic flops and bytes of those launches (the minimum a launch must compute and
 * move); plus the number of kernels of all kinds the handle launched. Any output may be
 * NULL. Synchronizes the device. */
rmt_status rmt_probe_read(rmt_handle* h, rmt_kernel kind, double* ms, int64_t* launches, double* flops,
                          double* bytes, int64_t* all_launches);

/* Free everything the handle owns. Synchronizes the device. NULL is accepted. */
rmt_status rmt_destroy(rmt_handle* h);

/* Message of the last non-OK status on this thread ("" if none). */
const char* rmt_last_error(void);

/* ------------------------------------------------------------------------------------
 * Kernel-level entry points: the same kernels the forward launches, on caller buffers
 * (device pointers only), for testing and measurement. All asynchronous on `stream`.
 * ------------------------------------------------------------------------------------ */

/* Grouped GEMM on tensor cores (tcgen05, TMEM accumulators, TMA-fed):
 *   C[g] = A[g] . B[g]^T for g in 0..G-1, bf16 inputs, fp32 accumulation.
 * A [G, M, K] bf16, B [G, N, K] bf16 (a distinct weight per group, [out, in]),
 * C [G, M, N] in out_dtype (RMT_F32 or RMT_BF16). Needs K % 64 == 0 and N % 64 == 0;
 * M is arbitrary (ragged last tile). Pointers 16-byte aligned. When N % 256 == 0 the
 * product runs on CTA pairs (2-SM MMAs, tokens along the MMA's N), else on single CTAs.
 * "Architecture Overview": GroupedGEMM operations batched across layers within a diagonal. */
rmt_status rmt_grouped_gemm_bf16(const void* A, const void* B, void* C, int32_t G, int32_t M,
                                 int32_t N, int32_t K, rmt_dtype out_dtype, void* stream);

/* Segment-local causal attention with grouped KV heads, per cell:
 *   out[g, i, h] = softmax_j<=i(q[g,i,h] . k[g,j,h/(H/Hkv)] / sqrt(dh)) v[g,j,h/(H/Hkv)]
 * qkv [G, M, (H + 2*Hkv)*dh] (q heads, then k heads, then v heads, RoPE already applied),
 * out [G, M, H*dh]; dtype RMT_F32 or RMT_BF16 (softmax in fp32). dh in {32, 64, 128}. */
rmt_status rmt_attention(const void* qkv, void* out, int32_t G, int32_t M, int32_t H, int32_t Hkv,
                         int32_t dh, rmt_dtype dtype, void* stream);

/* Associative read, per row r of each group g (phi(x) = elu(x) + 1):
 *   o[g,r] = phi(q[g,r]) A[g] / (phi(q[g,r]) . z[g] + eps)
 * q [G, M, dk] fp32 (before phi), A [G, dk, dv] fp32, z [G, dk] fp32, o [G, M, dv] in
 * dtype. dk, dv multiples of 32, <= 128; every pointer 16-byte aligned (RMT_EINVAL otherwise). */
rmt_status rmt_memory_read(const float* q, const float* A, const float* z, void* o, int32_t G,
                           int32_t M, int32_t dk, int32_t dv, float eps, rmt_dtype dtype, void* stream);

/* Delta-rule write of n rows per group, all rows against the pre-update state:
 *   v_bar = phi(k) A / (phi(k) . z + eps);  A += phi(k)^T (v - v_bar);  z += sum_r phi(k_r)
 * k [G, n, dk] fp32 (before phi), v [G, n, dv] fp32, A [G, dk, dv] and z [G, dk] fp32,
 * updated in place. n <= 64; dk, dv multiples of 32, <= 128; every pointer 16-byte aligned
 * (RMT_EINVAL otherwise). */
rmt_status rmt_memory_update(const float* k, const float* v, float* A, float* z, int32_t G,
                             int32_t n, int32_t dk, int32_t dv, float eps, void* stream);

/* The per-token delta rule: rows r = 0 .. n-1 of each group written one after another, row r
 * against the state rows 0 .. r-1 left:
 *   v_bar_r = phi(k_r) A_r / (phi(k_r) . z_r + eps);  A_{r+1} = A_r + phi(k_r)^T (v_r - v_bar_r);
 *   z_{r+1} = z_r + phi(k_r).
 * Same arguments, layouts and errors as rmt_memory_update. The kernels form it from the
 * batched quantities and the rows' Gram matrix G_rj = phi(k_r) . phi(k_j) (forward
 * substitution over the rows), so it agrees with the row-by-row loop up to rounding. */
rmt_status rmt_memory_update_sequential(const float* k, const float* v, float* A, float* z, int32_t G,
                                        int32_t n, int32_t dk, int32_t dv, float eps, void* stream);

/* Memory write from n rows per group (a layer's memory-token outputs):
 *   k = y W_mk^T, v = y W_mv^T, then the delta-rule update above (phi applied to k).
 * y [G, n, d] fp32; w_mkv [G, dk + dv, d] in dtype (the dk rows of W_mk, then the dv rows
 * of W_mv); A [G, dk, dv] and z [G, dk] fp32, updated in place. The projection is split
 * along d in blocks of 128 columns (tensor cores for bf16 weights, the fp32 rows split into
 * three bf16 terms) whose partial sums go to a library-owned device scratch buffer (grown
 * with cudaMalloc on demand) and are added in a fixed order. With bf16 weights, n <= 16 and at
 * least four groups per SM, one CTA adds a group's partials in that same order itself and only
 * the sums go through the buffer (the same bits).
 * n <= 64, n*(dk+dv) <= 4096; dk, dv multiples of 32, <= 128; A and z 16-byte aligned. */
rmt_status rmt_memory_write(const float* y, const void* w_mkv, float* A, float* z, int32_t G, int32_t n,
                            int32_t d, int32_t dk, int32_t dv, float eps, rmt_dtype dtype, void* stream);

/* rmt_memory_write without any device allocation. The paper has no counterpart: this is
 * for callers that cannot let a library call cudaMalloc, such as a serving engine or a
 * caching allocator that has already claimed the device memory for its own pool (there a
 * cudaMalloc can fail, and it synchronizes the whole device, stalling the caller's other
 * streams). Same arguments and results as rmt_memory_write; the cell table and the split-K
 * partial sums live in a fixed 8 MiB array in the library's device memory. Sizes whose
 * partial sums need more than 8 MiB - 256 KiB (G*s*n*(dk+dv)*4 bytes, s = ceil(d/128), or s = 1
 * with bf16 weights, n <= 16 and at least four groups per SM), or
 * G > 8192, return RMT_EINVAL. It calls no cudaMalloc or cudaFree. The first call on each
 * device loads the module that holds the array (CUDA loads modules lazily by default), which
 * reserves the 8 MiB on that device until the process exits, and looks up the array's
 * device address (cudaGetSymbolAddress). Make that first call at start-up: before the
 * caller's allocator claims the device memory, and before any stream capture. The address is
 * kept per device and does not survive a cudaDeviceReset of that device.
 * All calls share the array, which keeps the last call's contents (every
 * value a call reads is written earlier in the same call): calls that overlap on the GPU,
 * e.g. on two streams, race and give wrong results. */
rmt_status rmt_memory_write_noalloc(const float* y, const void* w_mkv, float* A, float* z, int32_t G,
                                    int32_t n, int32_t d, int32_t dk, int32_t dv, float eps, rmt_dtype dtype,
                                    void* stream);

/* RMSNorm of fp32 rows into dtype: y[r] = x[r] / sqrt(mean(x[r]^2) + eps) * g.
 * x [rows, d] fp32, g [d] and y [rows, d] in dtype. d % 4 == 0. */
rmt_status rmt_rmsnorm(const float* x, const void* g, void* y, int32_t rows, int32_t d, float eps,
                       rmt_dtype dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RMT_H */

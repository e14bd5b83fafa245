"""Oracle for ARMT prefill under diagonal batching -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs may import this
module. The CUDA path never calls it and shares no code with it.

A plain, slow numpy implementation of what the hot path computes, run strictly
sequentially: for segment s = 0..S-1, for layer l = 0..L-1, one (layer, segment) cell.
Source pages:

* [P1] skill page "Diagonal Batching for Recurrent Memory Transformers"
  (skillsmp.com, title "Diagonal Batching Unlocks Parallelism in Recurrent Memory
  Transformers for Long Contexts"): "Core Concept", "Architecture Overview" and the
  scheduler in "Implementation".
* [P2] arXiv 2506.05229 record, abstract: diagonal batching is a pure run-time
  reordering that keeps the exact recurrence; LLaMA-1B ARMT at 131,072 tokens.

Because diagonal batching only reorders the (layer, segment) grid [P2 abstract; P1
"Architecture Overview": dependency preservation, zero model modification], the
sequential model below *is* the definition of the result; a diagonal execution must
reach the same numbers.

Readings where the pages are silent (the pages cite ARMT by name only and print no
layer equations):
* memory: phi(x) = elu(x) + 1; read o = phi(q) A / (phi(q) . z + eps); delta-rule update
  A += phi(K)^T (V - phi(K) A / (phi(K) . z + eps)), z += sum of phi(K) rows, batched over
  the memory-token rows of the cell with the pre-update A, z; eps = 1e-6. The rule is
  written for one key; cfg.mem_update = "sequential" applies it to the cell's rows one
  after another instead (each row against the state the earlier rows left).
* the read sits at the layer input (all rows of the cell) and is added back through W_mo;
  the update keys/values are projected from the layer's memory-token output rows.
* the layer is a LLaMA decoder layer: RMSNorm (eps 1e-5), RoPE rotate-half with
  theta = 500000 at segment-local positions, causal GQA attention over the segment and
  memory tokens, SwiGLU MLP; no biases.
* memory tokens are appended after each segment's tokens at layer 0; state starts at 0.
* a sequence whose length is not a multiple of the segment length ends in a shorter
  segment (the sketch in P1 "Implementation" cuts with ceil division); its memory tokens
  follow its last token, and its memory write reads the cell's last n_mem rows.
* a batch is a set of independent sequences, each with its own memory state.
* the output is the last layer's rows of the segment tokens.

Arithmetic runs in the dtype given (float32 or float64); RoPE angles and their cos/sin
are computed in float64 and then rounded to that dtype.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["phi", "silu", "rms_norm", "rope", "causal_gqa_attention", "memory_read",
           "memory_update", "memory_update_sequential", "decoder_layer", "armt_cell", "forward",
           "forward_tokens", "forward_batch", "full_attention_forward", "diagonals",
           "sequential_steps", "schedule_triples", "schedule_quads"]


# ----------------------------------------------------------------------------- schedule

def diagonals(n_layers: int, n_segments: int) -> list:
    """The (layer, segment) grid swept in anti-diagonals d = l + s.

    [P1 "Implementation": the diagonal scheduler] for every diagonal index d in
    0 .. L+S-2 and every layer l in ascending order, the cell (l, d - l) belongs to
    diagonal d when 0 <= d - l < S; empty diagonals are dropped.
    """
    out = []
    for d in range(n_layers + n_segments - 1):
        cells = []
        for l in range(n_layers):
            s = d - l
            if 0 <= s < n_segments:
                cells.append((l, s))
        if cells:
            out.append(cells)
    return out


def sequential_steps(n_layers: int, n_segments: int) -> list:
    """The sequential execution [P1 "Core Concept"]: one cell per step, segments outermost."""
    return [[(l, s)] for s in range(n_segments) for l in range(n_layers)]


def schedule_triples(n_layers: int, n_segments: int, schedule: str) -> np.ndarray:
    """Flattened schedule as int32 rows (step, layer, segment), in execution order."""
    steps = diagonals(n_layers, n_segments) if schedule == "diagonal" else sequential_steps(n_layers, n_segments)
    rows = [(t, l, s) for t, cells in enumerate(steps) for (l, s) in cells]
    return np.asarray(rows, dtype=np.int32).reshape(-1, 3)


def schedule_quads(n_layers: int, n_segments: list, schedule: str) -> np.ndarray:
    """Schedule of a batch whose sequence b has n_segments[b] segments, as int32 rows
    (step, sequence, layer, segment) in execution order.

    [P1 "Implementation": the input is a [B, T, D] batch; one diagonal step runs the cell
    (l, s) for the whole batch.] Diagonal: step d holds every (b, l, s) with l + s = d, layers
    ascending and, within a layer, sequences ascending; steps without a cell are dropped.
    Sequential: one cell per step, sequence by sequence, each in the single-sequence order.
    """
    rows = []
    if schedule == "diagonal":
        step = 0
        for d in range(n_layers + max(n_segments) - 1):
            cells = [(b, l, d - l) for l in range(n_layers) for b in range(len(n_segments))
                     if 0 <= d - l < n_segments[b]]
            if cells:
                rows += [(step, b, l, s) for (b, l, s) in cells]
                step += 1
    else:
        step = 0
        for b, nb in enumerate(n_segments):
            for (cell,) in sequential_steps(n_layers, nb):
                rows.append((step, b) + cell)
                step += 1
    return np.asarray(rows, dtype=np.int32).reshape(-1, 4)


# ------------------------------------------------------------------ elementwise pieces

def phi(x: np.ndarray) -> np.ndarray:
    """elu(x) + 1 (alpha = 1): x + 1 where x > 0, exp(x) elsewhere."""
    with np.errstate(over="ignore"):
        return np.where(x > 0, x + 1, np.exp(np.minimum(x, 0)))


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x)."""
    with np.errstate(over="ignore"):
        return x / (1 + np.exp(-x))


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + x.dtype.type(eps)) * g


def rope(x: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half pairing (i, i + dh/2), positions 0..M-1.

    x: [M, H, dh]. Pair i is rotated by the angle p * theta^(-2i/dh) at position p.
    """
    m, _, dh = x.shape
    half = dh // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / dh)
    ang = np.arange(m, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang).astype(x.dtype)[:, None, :]
    sin = np.sin(ang).astype(x.dtype)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def causal_gqa_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(dh) + causal mask) v per head, within one cell.

    q: [M, Hq, dh]; k, v: [M, Hkv, dh]. Query head h reads key/value head h // (Hq/Hkv).
    Row i attends to rows 0..i (its own row included).
    """
    m, hq, dh = q.shape
    hkv = k.shape[1]
    rep = hq // hkv
    future = np.triu(np.ones((m, m), dtype=bool), k=1)
    scale = q.dtype.type(1.0 / math.sqrt(dh))
    out = np.empty_like(q)
    for h in range(hq):
        kv = h // rep
        s = (q[:, h, :] @ k[:, kv, :].T) * scale
        s[future] = -np.inf
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, kv, :]
    return out


# ------------------------------------------------------------------- associative memory

def memory_read(q_raw: np.ndarray, A: np.ndarray, z: np.ndarray, eps: float) -> np.ndarray:
    """Associative read, row by row: o = phi(q) A / (phi(q) . z + eps).

    q_raw: [M, dk] (before phi); A: [dk, dv]; z: [dk] -> o: [M, dv].
    """
    fq = phi(q_raw)
    return (fq @ A) / (fq @ z + q_raw.dtype.type(eps))[:, None]


def memory_update(k_raw: np.ndarray, v: np.ndarray, A: np.ndarray, z: np.ndarray, eps: float):
    """Delta-rule write of n key/value rows, all against the pre-update state.

    v_bar = phi(K) A / (phi(K) . z + eps)   (what the memory returns for each key now)
    A'    = A + phi(K)^T (V - v_bar)
    z'    = z + sum over rows of phi(K)
    k_raw: [n, dk] (before phi); v: [n, dv]. Returns (A', z').
    """
    fk = phi(k_raw)
    v_bar = (fk @ A) / (fk @ z + k_raw.dtype.type(eps))[:, None]
    return A + fk.T @ (v - v_bar), z + fk.sum(axis=0)


def memory_update_sequential(k_raw: np.ndarray, v: np.ndarray, A: np.ndarray, z: np.ndarray, eps: float):
    """Delta-rule write of n key/value rows, one after another: row r is written into the
    state that rows 0 .. r-1 left (for each row, the single-key rule of memory_update).
    k_raw: [n, dk] (before phi); v: [n, dv]. Returns (A', z')."""
    fk = phi(k_raw)
    e = k_raw.dtype.type(eps)
    A = A.copy()
    z = z.copy()
    for r in range(fk.shape[0]):
        k = fk[r]
        v_bar = (k @ A) / (k @ z + e)
        A = A + np.outer(k, v[r] - v_bar)
        z = z + k
    return A, z


# ------------------------------------------------------------------------------- model

def decoder_layer(x: np.ndarray, lw: dict, cfg) -> np.ndarray:
    """The LLaMA decoder layer of a cell (no memory): x [m, d] at positions 0..m-1, causal
    attention over its own rows. Returns the layer output [m, d]."""
    m = x.shape[0]
    hq, hkv, dh = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    # attention block
    h = rms_norm(x, lw["g_attn"], cfg.rms_eps)
    q = rope((h @ lw["wq"].T).reshape(m, hq, dh), cfg.rope_theta)
    k = rope((h @ lw["wk"].T).reshape(m, hkv, dh), cfg.rope_theta)
    v = (h @ lw["wv"].T).reshape(m, hkv, dh)
    a = causal_gqa_attention(q, k, v).reshape(m, hq * dh)
    x = x + a @ lw["wo"].T
    # SwiGLU MLP block
    h = rms_norm(x, lw["g_mlp"], cfg.rms_eps)
    u = silu(h @ lw["w_gate"].T) * (h @ lw["w_up"].T)
    return x + u @ lw["w_down"].T


def armt_cell(x: np.ndarray, lw: dict, A: np.ndarray, z: np.ndarray, cfg) -> tuple:
    """One (layer, segment) cell: x [M, d] is the layer input (segment rows, then memory rows).

    lw holds this layer's matrices ([out, in]) and gains. Returns (layer output, A', z').
    """
    m = x.shape[0]
    # associative read at the layer input, projected back to d_model and added
    o = memory_read(x @ lw["w_mq"].T, A, z, cfg.mem_eps)
    x = x + o @ lw["w_mo"].T
    x = decoder_layer(x, lw, cfg)
    # memory write from this layer's memory-token output rows (the cell's last n_mem rows)
    y = x[m - cfg.n_mem:]
    write = memory_update_sequential if getattr(cfg, "mem_update", "batched") == "sequential" else memory_update
    A, z = write(y @ lw["w_mk"].T, y @ lw["w_mv"].T, A, z, cfg.mem_eps)
    return x, A, z


def layer_weights(weights: dict, l: int, dtype) -> dict:
    return {k: np.asarray(v[l], dtype=dtype) for k, v in weights.items() if k != "mem_tokens"}


def forward_tokens(cfg, weights: dict, emb: np.ndarray, dtype=np.float32, A0=None, z0=None):
    """Sequential ARMT prefill of one sequence of T = emb.shape[0] tokens.

    [P1 "Implementation": the sequence is cut into ceil(T / segment_length) segments, each
    ending at min(start + segment_length, T).] So every segment holds seg_len tokens except
    possibly the last, which holds the rest; each segment is followed by the memory tokens.
    Cell (l, s) takes layer l-1's output for segment s (for l = 0: the segment's embeddings
    followed by the memory tokens) and layer l's memory state after segment s-1 (A0, z0, or
    zeros, before segment 0). Returns (out [T, d], A [L, dk, dv], z [L, dk]) in `dtype`.
    """
    L, seg = cfg.n_layers, cfg.seg_len
    emb = np.asarray(emb, dtype=dtype)
    T = emb.shape[0]
    mem = np.asarray(weights["mem_tokens"], dtype=dtype)
    lws = [layer_weights(weights, l, dtype) for l in range(L)]
    A = [np.zeros((cfg.d_k, cfg.d_v), dtype) if A0 is None else np.array(A0[l], dtype) for l in range(L)]
    z = [np.zeros(cfg.d_k, dtype) if z0 is None else np.array(z0[l], dtype) for l in range(L)]
    out = np.empty((T, cfg.d_model), dtype)
    for s in range(-(-T // seg)):
        lo, hi = s * seg, min((s + 1) * seg, T)
        x = np.concatenate([emb[lo:hi], mem], axis=0)
        for l in range(L):
            x, A[l], z[l] = armt_cell(x, lws[l], A[l], z[l], cfg)
        out[lo:hi] = x[:hi - lo]
    return out, np.stack(A), np.stack(z)


def forward(cfg, weights: dict, emb: np.ndarray, n_segments: int, dtype=np.float32,
            A0=None, z0=None):
    """Sequential ARMT prefill over n_segments full segments of emb [n_segments*seg_len, d].

    Returns (out [n_segments*seg_len, d], A [L, dk, dv], z [L, dk]) in `dtype`.
    """
    return forward_tokens(cfg, weights, np.asarray(emb)[:n_segments * cfg.seg_len], dtype, A0, z0)


def forward_batch(cfg, weights: dict, embs: list, dtype=np.float32, A0=None, z0=None):
    """A batch of independent sequences (embs[b]: [T_b, d]), each run by forward_tokens with
    its own memory state (A0[b], z0[b] or zeros). Returns ([out_b], A [B, L, dk, dv],
    z [B, L, dk])."""
    outs, As, zs = [], [], []
    for b, e in enumerate(embs):
        o, A, z = forward_tokens(cfg, weights, e, dtype, None if A0 is None else A0[b], None if z0 is None else z0[b])
        outs.append(o)
        As.append(A)
        zs.append(z)
    return outs, np.stack(As), np.stack(zs)


def full_attention_forward(cfg, weights: dict, emb: np.ndarray, dtype=np.float32) -> np.ndarray:
    """The comparison model of the ARMT paper [P2 abstract: ARMT with diagonal batching against
    full-attention LLaMA-1B at 131,072 tokens]: the same decoder layers without the memory (no
    memory tokens, no read or write), run over the whole sequence emb [T, d] as one causal
    segment at positions 0..T-1. Returns the last layer's hidden states [T, d] in `dtype`."""
    x = np.asarray(emb, dtype=dtype)
    for l in range(cfg.n_layers):
        x = decoder_layer(x, layer_weights(weights, l, dtype), cfg)
    return x

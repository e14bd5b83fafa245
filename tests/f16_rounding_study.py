"""How far f16 operand rounding carries through the memory recurrence (CPU study, not a test).

The bf16 mode of the library stores every tensor-core activation operand as f16: the residual
stream copy before each projection (x), the memory read-out (o), q, k and v (qkv), the softmax
numerators (p), the attention output (att) and the SwiGLU output (u). This script runs the
fp32 oracle's layer with rounding to f16 inserted at chosen points and reports how far the
final memory state A and the outputs move from the plain fp32 oracle run:

  python tests/f16_rounding_study.py points 3b-512 2     each point alone, then all of them
  python tests/f16_rounding_study.py rows 3b-512 16      every row rounded, then the segment
                                                         rows only (memory-token rows exact)

The layer below restates the oracle's cell (oracle/armt.py, built from its helpers) with the
rounding hooks; it calls only the oracle and the seeded input generators. Errors are the
normwise max relative error of the parity tests. On 8 host cores a 3b-512 segment takes
about 11 s per run.
"""
from __future__ import annotations

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from armt_synthetic import CONFIGS, make_embeddings, make_weights  # noqa: E402
from oracle import armt  # noqa: E402

POINTS = ("x", "o", "q", "k", "v", "p", "att", "u")


def to_f16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.float16).float().numpy()


def rounder(active: set, seg_rows: int | None):
    """Per point: f16 rounding if the point is active (only rows < seg_rows if given)."""
    def make(pt):
        if pt not in active:
            return lambda a: a
        if seg_rows is None:
            return to_f16

        def part(a):
            b = a.copy()
            b[:seg_rows] = to_f16(a[:seg_rows])
            return b
        return part
    return {pt: make(pt) for pt in POINTS}


def cell(cfg, x, lw, A, z, R):
    m, hq, hkv, dh = x.shape[0], cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    o = armt.memory_read(R["x"](x) @ lw["w_mq"].T, A, z, cfg.mem_eps)
    x = x + R["o"](o) @ lw["w_mo"].T
    r = 1.0 / np.sqrt(np.mean(x * x, -1, keepdims=True) + cfg.rms_eps)
    hx = R["x"](x)
    q = R["q"](armt.rope(((hx @ (lw["wq"] * lw["g_attn"]).T) * r).reshape(m, hq, dh), cfg.rope_theta))
    k = R["k"](armt.rope(((hx @ (lw["wk"] * lw["g_attn"]).T) * r).reshape(m, hkv, dh), cfg.rope_theta))
    v = R["v"](((hx @ (lw["wv"] * lw["g_attn"]).T) * r).reshape(m, hkv, dh))
    rep, out = hq // hkv, np.empty_like(q)
    future = np.triu(np.ones((m, m), bool), 1)
    for h in range(hq):
        s = (q[:, h] @ k[:, h // rep].T) / np.sqrt(dh)
        s[future] = -np.inf
        p = np.exp(s - s.max(1, keepdims=True))
        out[:, h] = (R["p"](p) @ v[:, h // rep]) / p.sum(1, keepdims=True)
    x = x + R["att"](out.reshape(m, hq * dh)) @ lw["wo"].T
    r = 1.0 / np.sqrt(np.mean(x * x, -1, keepdims=True) + cfg.rms_eps)
    hx = R["x"](x)
    g = (hx @ (lw["w_gate"] * lw["g_mlp"]).T) * r
    u = (hx @ (lw["w_up"] * lw["g_mlp"]).T) * r
    x = x + R["u"](armt.silu(g) * u) @ lw["w_down"].T
    y = x[cfg.seg_len:]
    A, z = armt.memory_update(y @ lw["w_mk"].T, y @ lw["w_mv"].T, A, z, cfg.mem_eps)
    return x, A, z


def run(cfg, w, emb, S, R):
    """Per segment: the last layer's segment rows and every layer's A after the segment."""
    lws = [armt.layer_weights(w, l, np.float32) for l in range(cfg.n_layers)]
    A = [np.zeros((cfg.d_k, cfg.d_v), np.float32) for _ in range(cfg.n_layers)]
    z = [np.zeros(cfg.d_k, np.float32) for _ in range(cfg.n_layers)]
    outs, states = [], []
    seg = cfg.seg_len
    for s in range(S):
        x = np.concatenate([emb[s * seg:(s + 1) * seg], w["mem_tokens"]])
        for l in range(cfg.n_layers):
            x, A[l], z[l] = cell(cfg, x, lws[l], A[l], z[l], R)
        outs.append(x[:seg])
        states.append(np.stack(A))
    return outs, states


def normwise(a, b) -> float:
    return float(np.abs(np.asarray(a, np.float64) - b).max() / np.abs(b).max())


def main() -> None:
    mode, name, S = sys.argv[1], sys.argv[2], int(sys.argv[3])
    cfg = CONFIGS[name]
    w, emb = make_weights(cfg), make_embeddings(cfg, S)
    ref = run(cfg, w, emb, S, rounder(set(), None))
    marks = sorted({0, S // 4, S // 2, S - 1})

    def report(label, got):
        print(f"{name} S={S} {label}: out", {s: round(normwise(got[0][s], ref[0][s]), 6) for s in marks},
              "A", {s: round(normwise(got[1][s], ref[1][s]), 6) for s in marks}, flush=True)

    if mode == "points":
        for pt in POINTS:
            report(f"f16 at {pt}", run(cfg, w, emb, S, rounder({pt}, None)))
        report("f16 at all points", run(cfg, w, emb, S, rounder(set(POINTS), None)))
    else:
        report("all rows", run(cfg, w, emb, S, rounder(set(POINTS), None)))
        report("segment rows only", run(cfg, w, emb, S, rounder(set(POINTS), cfg.seg_len)))


if __name__ == "__main__":
    main()

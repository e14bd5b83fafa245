"""Helpers shared by the GPU tests: model construction and forward runs through the C ABI."""
import numpy as np
import torch

from armt_synthetic import make_embeddings, make_weights
from recurrent_memory_transformer_anti_b200 import rmt


def normwise(a, b) -> float:
    """max |a - b| / max |b| (the tolerance metric of the parity tests)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def build(cfg, weights=None, seed=0):
    w = make_weights(cfg, seed=seed) if weights is None else weights
    wt = rmt.weights_storage(w, cfg.dtype, device="cuda")
    h = rmt.rmt_create(wt, cfg)
    del wt
    torch.cuda.synchronize()
    return w, h


def forward(h, cfg, emb, n_segments, schedule="diagonal"):
    """Run rmt_forward on device buffers; returns (out, A, z) as float32 numpy arrays."""
    e = rmt.storage(emb, cfg.dtype, device="cuda")
    out = torch.empty_like(e)
    A = torch.empty(cfg.n_layers, cfg.d_k, cfg.d_v, device="cuda")
    z = torch.empty(cfg.n_layers, cfg.d_k, device="cuda")
    rmt.rmt_forward(h, e, n_segments, schedule, out, A, z)
    rmt.rmt_sync(h)
    return to_np(out), to_np(A), to_np(z)


def embeddings(cfg, n_segments, seed=1):
    return make_embeddings(cfg, n_segments, seed=seed)


def forward_batch(h, cfg, embs, schedule="diagonal", in_A=None, in_z=None, host=False):
    """rmt_forward_batch over the sequences embs[b] ([T_b, d] each), packed one after another.

    host=True passes page-locked host buffers for the embeddings and the outputs. Returns
    ([out_b] as float32 numpy, A [B, L, dk, dv], z [B, L, dk])."""
    lens = [int(e.shape[0]) for e in embs]
    e = rmt.storage(np.concatenate(embs), cfg.dtype, device="cuda")
    if host:
        e = e.cpu().pin_memory()
    out = torch.empty_like(e)
    if host:
        out = out.pin_memory()
    B = len(embs)
    A = torch.empty(B, cfg.n_layers, cfg.d_k, cfg.d_v, device="cuda")
    z = torch.empty(B, cfg.n_layers, cfg.d_k, device="cuda")
    rmt.rmt_forward_batch(h, e, lens, schedule, out, in_A, in_z, A, z)
    rmt.rmt_sync(h)
    o = to_np(out)
    starts = np.cumsum([0] + lens)
    return [o[starts[b]:starts[b + 1]] for b in range(B)], to_np(A), to_np(z)

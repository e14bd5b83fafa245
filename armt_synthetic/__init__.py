"""Seeded synthetic inputs for ARMT prefill: model shapes, random-init weights, embeddings.

This module is shared by the oracle and by the CUDA path's tests and bench. It holds
no arithmetic of the method: only shapes, seeded random draws, and rounding of the drawn
values to the storage type of a bf16 model.

Shapes follow the workloads of "Diagonal Batching Unlocks Parallelism in Recurrent
Memory Transformers for Long Contexts" (arXiv 2506.05229, abstract): a LLaMA-1B-shaped
ARMT on sequences of up to 131,072 tokens. The pages give no checkpoint, so weights are
random: every projection ~ N(0, 0.02), RMSNorm gains = 1, memory tokens ~ N(0, 0.02),
embeddings ~ N(0, 1).

Streams (numpy PCG64 seeded with an integer tuple; float32 standard normals, row-major):
  weight matrix k of layer l:  PCG64([seed, l, i_k]), i_k = position of k in LAYER_KEYS
  memory tokens:               PCG64([seed, L, 0])
  embeddings of segment s:     PCG64([emb_seed, s])   (so a prefix of segments is the same
                                                       whatever the total segment count)
Independent streams let the draws run in parallel threads.
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import os
from dataclasses import dataclass

import numpy as np

__all__ = ["ArmtConfig", "CONFIGS", "make_weights", "make_embeddings", "round_to_bf16",
           "bf16_bits", "bf16_bits_to_f32", "WEIGHT_SEED", "EMB_SEED", "LAYER_KEYS"]

WEIGHT_SEED = 0
EMB_SEED = 1

# Per-layer projection matrices, row-major [out, in] like nn.Linear.
LAYER_KEYS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "w_mq", "w_mk", "w_mv", "w_mo")


@dataclass(frozen=True)
class ArmtConfig:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ff: int
    seg_len: int
    n_mem: int
    d_k: int
    d_v: int
    rope_theta: float = 500000.0
    rms_eps: float = 1e-5
    mem_eps: float = 1e-6
    dtype: str = "f32"          # "f32" or "bf16": storage type of weights and activations
    mem_update: str = "batched"  # "batched" or "sequential": how a cell writes its memory rows

    @property
    def m_tokens(self) -> int:
        """Rows of one (layer, segment) cell: segment tokens followed by memory tokens."""
        return self.seg_len + self.n_mem

    def with_(self, **kw) -> "ArmtConfig":
        return dataclasses.replace(self, **kw)

    def weight_shapes(self) -> dict:
        d, hq, hkv, dh, f = self.d_model, self.n_heads, self.n_kv_heads, self.head_dim, self.d_ff
        return {
            "wq": (hq * dh, d), "wk": (hkv * dh, d), "wv": (hkv * dh, d), "wo": (d, hq * dh),
            "w_gate": (f, d), "w_up": (f, d), "w_down": (d, f),
            "w_mq": (self.d_k, d), "w_mk": (self.d_k, d), "w_mv": (self.d_v, d), "w_mo": (d, self.d_v),
        }


CONFIGS = {
    # 4 layers x 4 segments of 64 + 8 memory tokens, d_model 128, 4 heads of 32, fp32.
    "tiny": ArmtConfig(n_layers=4, d_model=128, n_heads=4, n_kv_heads=4, head_dim=32, d_ff=512,
                       seg_len=64, n_mem=8, d_k=32, d_v=32, dtype="f32"),
    # A small bf16 model for parity tests: GQA 4/2, a ragged 208-row cell (one 128-row tile + 80).
    "small-bf16": ArmtConfig(n_layers=4, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ff=512,
                             seg_len=200, n_mem=8, d_k=64, d_v=64, dtype="bf16"),
    # LLaMA-1B-shaped ARMT: 16 layers, d 2048, 32/8 heads of 64, SwiGLU 8192, 1024 + 16 tokens per segment.
    "1b": ArmtConfig(n_layers=16, d_model=2048, n_heads=32, n_kv_heads=8, head_dim=64, d_ff=8192,
                     seg_len=1024, n_mem=16, d_k=64, d_v=64, dtype="bf16"),
    # LLaMA-3B-shaped ARMT: 28 layers, d 3072, 24/8 heads of 128, SwiGLU 8192.
    "3b-512": ArmtConfig(n_layers=28, d_model=3072, n_heads=24, n_kv_heads=8, head_dim=128, d_ff=8192,
                         seg_len=512, n_mem=16, d_k=128, d_v=128, dtype="bf16"),
    "3b-2048": ArmtConfig(n_layers=28, d_model=3072, n_heads=24, n_kv_heads=8, head_dim=128, d_ff=8192,
                          seg_len=2048, n_mem=16, d_k=128, d_v=128, dtype="bf16"),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32 holding them."""
    out = np.array(a, dtype=np.float32, copy=True)
    _round_bf16_inplace(out)
    return out


def _round_bf16_inplace(a: np.ndarray) -> None:
    u = a.reshape(-1).view(np.uint32)
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values, round to nearest even. Inputs are finite."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(key: tuple, shape: tuple, std: float, bf16: bool) -> np.ndarray:
    a = np.random.Generator(np.random.PCG64(list(key))).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if bf16:
        _round_bf16_inplace(a)
    return a


def _pool():
    return cf.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def make_weights(cfg: ArmtConfig, seed: int = WEIGHT_SEED, std: float = 0.02) -> dict:
    """Random-init weights of an ARMT with cfg's shapes.

    Returns {key: [L arrays]} for the per-layer matrices and gains, plus "mem_tokens"
    [n_mem, d_model]. Values are float32; for a bf16 model they are already rounded to
    bf16 (so float32 and bf16 storage hold the same numbers).
    """
    shapes = cfg.weight_shapes()
    bf16 = cfg.dtype == "bf16"
    jobs = [(l, i, k) for l in range(cfg.n_layers) for i, k in enumerate(LAYER_KEYS)]
    with _pool() as ex:
        mats = list(ex.map(lambda j: _normal((seed, j[0], j[1]), shapes[j[2]], std, bf16), jobs))
    w = {k: [None] * cfg.n_layers for k in LAYER_KEYS}
    for (l, _, k), m in zip(jobs, mats):
        w[k][l] = m
    w["mem_tokens"] = _normal((seed, cfg.n_layers, 0), (cfg.n_mem, cfg.d_model), std, bf16)
    w["g_attn"] = [np.ones(cfg.d_model, np.float32) for _ in range(cfg.n_layers)]
    w["g_mlp"] = [np.ones(cfg.d_model, np.float32) for _ in range(cfg.n_layers)]
    return w


def make_embeddings(cfg: ArmtConfig, n_segments: int, seed: int = EMB_SEED) -> np.ndarray:
    """Input embeddings [n_segments * seg_len, d_model] ~ N(0, 1) (bf16-rounded for a bf16 model)."""
    out = np.empty((n_segments * cfg.seg_len, cfg.d_model), np.float32)
    seg = cfg.seg_len

    def fill(s):
        out[s * seg:(s + 1) * seg] = _normal((seed, s), (seg, cfg.d_model), 1.0, cfg.dtype == "bf16")

    with _pool() as ex:
        list(ex.map(fill, range(n_segments)))
    return out

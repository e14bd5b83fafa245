"""Write the oracle's results for the full-length bf16 workloads to tests/golden/long_*.npz.

This script calls only the oracle (oracle/armt.py) and the seeded input generators
(armt_synthetic). Nothing here comes from the CUDA path. Each file holds, for one workload
run through the fp32 oracle from a zero memory state:

  A        [L, d_k, d_v] float32   every layer's memory state after the last segment
  z        [L, d_k]      float32   every layer's normaliser after the last segment
  rows     [R]           int32     token rows of the sequence whose hidden states are kept
  hidden   [R, d_model]  float32   the last layer's output at those rows
  config, n_segments, weight_seed, emb_seed   what was run

The kept rows are the first 8, the last 8 and 24 evenly spaced rows of the first, the middle
and the last segment. Workloads (the LLaMA-1B- and LLaMA-3B-shaped ARMTs of the arXiv
2506.05229 abstract, at its 131,072-token length):

  long_1b_s32.npz        1b, 32 segments of 1024 + 16 tokens (32,768 tokens)
  long_1b_s128.npz       1b, 128 segments (131,072 tokens); continues the 32-segment run
  long_3b-512_s64.npz    3b-512, 64 segments of 512 + 16 tokens (32,768 tokens)
  long_3b-512_s256.npz   3b-512, 256 segments of 512 + 16 tokens (131,072 tokens); continues
                         the 64-segment run
  long_3b-2048_s64.npz   3b-2048, 64 segments of 2048 + 16 tokens (131,072 tokens)

The longer run of a workload resumes the oracle from the shorter run's state (the state after
a segment depends only on the segments before it, which the oracle tests pin). On an 8-core
host the oracle takes about 16 min for the 1B runs, 35 min for 3b-512 and 45 min for
3b-2048.

Usage: python tests/golden/make_long_goldens.py [1b] [3b-512] [3b-2048] [NAME:STOP,...]
(NAME:STOP,... runs that workload to the given stops only, e.g. 3b-512:64.)
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from armt_synthetic import CONFIGS, EMB_SEED, WEIGHT_SEED, make_embeddings, make_weights  # noqa: E402
from oracle import armt  # noqa: E402


def sample_rows(seg_len: int) -> np.ndarray:
    """Rows kept within one segment: the first 8, the last 8 and 24 evenly spaced ones."""
    spread = np.linspace(0, seg_len - 1, 24).round().astype(int)
    rows = np.unique(np.concatenate([np.arange(min(8, seg_len)), spread, np.arange(max(0, seg_len - 8), seg_len)]))
    return rows.astype(np.int32)


def kept_rows(seg_len: int, n_segments: int) -> np.ndarray:
    segs = sorted({0, n_segments // 2, n_segments - 1})
    r = sample_rows(seg_len)
    return np.concatenate([s * seg_len + r for s in segs]).astype(np.int32)


def save(name: str, cfg_name: str, n_segments: int, out: np.ndarray, A, z) -> None:
    cfg = CONFIGS[cfg_name]
    rows = kept_rows(cfg.seg_len, n_segments)
    path = os.path.join(HERE, f"long_{name}.npz")
    np.savez_compressed(path, A=np.asarray(A, np.float32), z=np.asarray(z, np.float32), rows=rows,
                        hidden=np.asarray(out[rows], np.float32), config=np.array(cfg_name),
                        n_segments=np.int32(n_segments), weight_seed=np.int32(WEIGHT_SEED),
                        emb_seed=np.int32(EMB_SEED))
    print(f"wrote {path}", flush=True)


def run(cfg_name: str, stops: list) -> None:
    """Run the oracle over max(stops) segments in chunks, saving a golden at each stop."""
    cfg = CONFIGS[cfg_name]
    w = make_weights(cfg)
    seg = cfg.seg_len
    S = max(stops)
    emb = make_embeddings(cfg, S)
    out = np.empty((S * seg, cfg.d_model), np.float32)
    A = z = None
    done = 0
    t0 = time.time()
    for stop in sorted(stops):
        o, A, z = armt.forward(cfg, w, emb[done * seg:stop * seg], stop - done, dtype=np.float32, A0=A, z0=z)
        out[done * seg:stop * seg] = o
        done = stop
        print(f"{cfg_name}: {stop} segments in {time.time() - t0:.0f} s", flush=True)
        save(f"{cfg_name}_s{stop}", cfg_name, stop, out[:stop * seg], A, z)


JOBS = {"1b": [32, 128], "3b-512": [64, 256], "3b-2048": [64]}

if __name__ == "__main__":
    for job in sys.argv[1:] or list(JOBS):
        name, _, stops = job.partition(":")
        run(name, [int(x) for x in stops.split(",")] if stops else JOBS[name])

"""Whole-forward parity on the GPU, through the C ABI.

* fp32 storage mode vs the fp32 oracle: normwise max relative error <= 1e-4.
* bf16 storage mode vs the fp32 oracle on the same bf16-rounded weights and embeddings:
  <= 2e-2.
* bf16 storage with split (high + low f16 term) operands: the memory state within the fp32
  tolerance on short runs; the 256-segment LLaMA-3B-shaped run within 2e-2, where the plain
  f16 operands drift past it.
* DIAGONAL vs SEQUENTIAL on the GPU: identical bits (each kernel's arithmetic for a cell
  does not depend on which cells share its launch).
* The device trace of executed cells equals the schedule, which equals the oracle's
  enumeration.
"""
import dataclasses
import os

import numpy as np
import pytest
import torch

from armt_synthetic import CONFIGS, make_weights
from oracle import armt
from recurrent_memory_transformer_anti_b200 import rmt
from tests.gpu_util import build, embeddings, forward, forward_batch, normwise

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_TOL = 2e-2
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def tiny(cuda_ok):
    cfg = CONFIGS["tiny"]
    w, h = build(cfg)
    yield cfg, w, h
    rmt.rmt_destroy(h)


@pytest.fixture(scope="module")
def small_bf16(cuda_ok):
    cfg = CONFIGS["small-bf16"]
    w, h = build(cfg)
    yield cfg, w, h
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("S", [4, 1, 9])
def test_tiny_fp32_matches_oracle(tiny, S):
    cfg, w, h = tiny
    emb = embeddings(cfg, S)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g, r, name in zip(got, ref, ("out", "A", "z")):
        assert normwise(g, r) < F32_TOL, name


@pytest.mark.parametrize("S", [4, 9])
def test_tiny_diagonal_equals_sequential_bitwise(tiny, S):
    cfg, w, h = tiny
    emb = embeddings(cfg, S)
    d = forward(h, cfg, emb, S, "diagonal")
    s = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(d, s):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("L,S", [(1, 3), (4, 1), (3, 7)])
def test_fp32_grid_shapes(cuda_ok, L, S):
    cfg = CONFIGS["tiny"].with_(n_layers=L)
    w, h = build(cfg, seed=5)
    emb = embeddings(cfg, S, seed=6)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g, r in zip(got, ref):
        assert normwise(g, r) < F32_TOL
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_device_trace_equals_schedule(tiny, schedule):
    cfg, w, h = tiny
    S = 6
    forward(h, cfg, embeddings(cfg, S), S, schedule)
    table = rmt.rmt_get_schedule(h, S, schedule)
    np.testing.assert_array_equal(table, armt.schedule_triples(cfg.n_layers, S, schedule))
    np.testing.assert_array_equal(rmt.rmt_get_trace(h, cfg.n_layers * S), table)


def test_host_buffers_give_the_same_bits(tiny):
    cfg, w, h = tiny
    S = 3
    emb = embeddings(cfg, S)
    dev = forward(h, cfg, emb, S, "diagonal")
    out = np.empty_like(emb)
    A = np.empty((cfg.n_layers, cfg.d_k, cfg.d_v), np.float32)
    z = np.empty((cfg.n_layers, cfg.d_k), np.float32)
    rmt.rmt_forward(h, np.ascontiguousarray(emb), S, "diagonal", out, A, z)
    rmt.rmt_sync(h)
    for a, b in zip(dev, (out, A, z)):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("name", ["tiny", "small-bf16"])
def test_pinned_host_buffers_give_the_same_bits(cuda_ok, name):
    """Page-locked host buffers take the overlapped path: one copy per segment on side
    streams, ordered against the steps by events. Two back-to-back forwards on the same
    staging buffers check that a forward's copies wait for the previous one."""
    cfg = CONFIGS[name]
    w, h = build(cfg)
    S = 4
    emb = embeddings(cfg, S, seed=16)
    emb2 = embeddings(cfg, S, seed=17)
    for schedule in ("diagonal", "sequential"):
        refs = [forward(h, cfg, x, S, schedule) for x in (emb, emb2)]
        e_host = [rmt.storage(x, cfg.dtype).pin_memory() for x in (emb, emb2)]
        outs = [torch.empty_like(e).pin_memory() for e in e_host]
        As = [torch.empty(cfg.n_layers, cfg.d_k, cfg.d_v).pin_memory() for _ in e_host]
        zs = [torch.empty(cfg.n_layers, cfg.d_k).pin_memory() for _ in e_host]
        for i in range(2):  # enqueued back to back, synchronized once
            rmt.rmt_forward(h, e_host[i], S, schedule, outs[i], As[i], zs[i])
        rmt.rmt_sync(h)
        for i in range(2):
            np.testing.assert_array_equal(refs[i][0], outs[i].float().numpy())
            np.testing.assert_array_equal(refs[i][1], As[i].numpy())
            np.testing.assert_array_equal(refs[i][2], zs[i].numpy())
    rmt.rmt_destroy(h)


def test_forward_argument_errors(tiny):
    cfg, w, h = tiny
    e = torch.zeros(cfg.seg_len, cfg.d_model, device="cuda")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_forward(h, e, 0, "diagonal", e)
    assert ex.value.status == rmt.RMT_EINVAL
    with pytest.raises(rmt.RmtError):
        rmt.rmt_forward(h, e, 1, 5, e)
    # the handle stays usable after a rejected call
    forward(h, cfg, embeddings(cfg, 1), 1)


@pytest.mark.parametrize("S", [4, 2])
def test_small_bf16_matches_oracle(small_bf16, S):
    cfg, w, h = small_bf16
    emb = embeddings(cfg, S)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g, r, name in zip(got, ref, ("out", "A", "z")):
        assert normwise(g, r) < BF16_TOL, name


def test_small_bf16_diagonal_equals_sequential_bitwise(small_bf16):
    cfg, w, h = small_bf16
    S = 5
    emb = embeddings(cfg, S)
    d = forward(h, cfg, emb, S, "diagonal")
    s = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(d, s):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------- the full-length workloads against oracle goldens
#
# tests/golden/long_*.npz hold the fp32 oracle's results for the bench's workloads, written by
# tests/golden/make_long_goldens.py (which calls only the oracle and the input generators):
# every layer's A and z after the last segment, and the last layer's hidden states at 40
# sampled rows of the first, middle and last segments.


def _golden(name):
    return np.load(os.path.join(GOLDEN, f"long_{name}.npz"))


def _check_golden(got, g, cfg):
    """cfg: the workload's configuration (its bf16 storage; a split-operand handle runs the same
    workload)."""
    out, A, z = got
    n = int(g["n_segments"])
    assert str(g["config"]) in CONFIGS and CONFIGS[str(g["config"])] == cfg
    assert out.shape == (n * cfg.seg_len, cfg.d_model)
    errs = {"hidden": normwise(out[g["rows"]], g["hidden"]), "A": normwise(A, g["A"]), "z": normwise(z, g["z"])}
    per_layer_A = [normwise(A[l], g["A"][l]) for l in range(cfg.n_layers)]
    assert max(errs.values()) < BF16_TOL, (errs, per_layer_A)
    assert np.isfinite(out).all()
    return errs


@pytest.fixture(scope="module")
def model_1b(cuda_ok):
    cfg = CONFIGS["1b"]
    w, h = build(cfg)
    yield cfg, w, h
    rmt.rmt_destroy(h)


def test_1b_131k_matches_oracle_golden(model_1b):
    """The bench's workload: the LLaMA-1B-shaped ARMT over 128 segments of 1024 + 16 tokens
    (131,072 tokens, bf16). The hidden states at the sampled rows of segments 0, 64 and 127
    and every layer's final A and z match the oracle within the bf16 tolerance; SEQUENTIAL
    gives the bits of DIAGONAL; and the first 32 segments, run alone, give the same bits and
    match the oracle's 32-segment results (the 32,768-token workload)."""
    cfg, w, h = model_1b
    S, P = 128, 32
    emb = embeddings(cfg, S)
    full_d = forward(h, cfg, emb, S, "diagonal")
    print("1b x 128 segments: normwise errors", _check_golden(full_d, _golden("1b_s128"), cfg))
    full_s = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(full_d, full_s):
        np.testing.assert_array_equal(a, b)
    del full_s
    part = forward(h, cfg, emb[:P * cfg.seg_len], P, "diagonal")
    np.testing.assert_array_equal(full_d[0][:P * cfg.seg_len], part[0])
    print("1b x 32 segments: normwise errors", _check_golden(part, _golden("1b_s32"), cfg))


@pytest.mark.parametrize("name,S,dtype", [("3b-2048", 64, "bf16"), ("3b-512", 64, "bf16"),
                                          ("3b-512", 256, "bf16-split")])
def test_3b_131k_matches_oracle_golden(cuda_ok, name, S, dtype):
    """The LLaMA-3B-shaped workloads (28 layers, d 3072, 24/8 heads of 128, d_k = d_v = 128,
    segments of 512 or 2048 + 16 tokens; the 2064-row cells end in a ragged token tile): the
    sampled hidden rows and all 28 layers' final A and z match the oracle within the bf16
    tolerance, and SEQUENTIAL gives the bits of DIAGONAL. With plain f16 operands: 3b-2048 at
    131,072 tokens and 3b-512 at 32,768; the 256 segments of 3b-512 (131,072 tokens) carry
    the f16 rounding through the memory recurrence past 2e-2 (A about 4.5%), so that run
    uses split operands."""
    cfg = CONFIGS[name]
    hcfg = dataclasses.replace(cfg, dtype=dtype)
    w, h = build(hcfg, weights=make_weights(cfg))
    del w
    emb = embeddings(cfg, S)
    full_d = forward(h, hcfg, emb, S, "diagonal")
    print(f"{name} x {S} segments, {dtype}: normwise errors", _check_golden(full_d, _golden(f"{name}_s{S}"), cfg))
    full_s = forward(h, hcfg, emb, S, "sequential")
    rmt.rmt_destroy(h)
    for a, b in zip(full_d, full_s):
        np.testing.assert_array_equal(a, b)


@pytest.fixture(scope="module")
def small_split(cuda_ok):
    base = CONFIGS["small-bf16"]
    cfg = dataclasses.replace(base, dtype="bf16-split")
    w = make_weights(base)
    _, h = build(cfg, weights=w)
    yield base, cfg, w, h
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("S", [4, 2])
def test_split_operands_match_oracle(small_split, S):
    """Split operands carry about 22 significant bits into every product and attention runs
    in fp32: the memory state A, z matches the fp32 oracle within the fp32 tolerance; the
    hidden output is stored as bf16, so it is held to the bf16 rounding bound (2^-8)."""
    base, cfg, w, h = small_split
    emb = embeddings(base, S)
    out, A, z = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(base, w, emb, S, dtype=np.float32)
    assert normwise(out, ref[0]) < 2.0 ** -8
    assert normwise(A, ref[1]) < F32_TOL and normwise(z, ref[2]) < F32_TOL, (normwise(A, ref[1]), normwise(z, ref[2]))


@pytest.mark.parametrize("name,S,tol", [("tiny", 4, F32_TOL), ("small-bf16", 3, BF16_TOL)])
def test_per_token_memory_update_matches_oracle(cuda_ok, name, S, tol):
    """cfg.mem_update = "sequential": each cell writes its memory rows one after another (the
    oracle's row loop; the kernels' Gram forward substitution). DIAGONAL gives the bits of
    SEQUENTIAL, and the result differs from the batched write."""
    base = CONFIGS[name]
    cfg = dataclasses.replace(base, mem_update="sequential")
    w = make_weights(base)
    _, h = build(cfg, weights=w)
    emb = embeddings(base, S)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g, r, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g, r) < tol, what
    for a, b in zip(got, forward(h, cfg, emb, S, "sequential")):
        np.testing.assert_array_equal(a, b)
    rmt.rmt_destroy(h)
    batched = armt.forward(base, w, emb, S, dtype=np.float32)
    assert normwise(ref[1], batched[1]) > 5 * tol  # A differs by 12-18% between the two rules


def test_split_operands_diagonal_equals_sequential_bitwise(small_split):
    base, cfg, w, h = small_split
    S = 5
    emb = embeddings(base, S)
    d = forward(h, cfg, emb, S, "diagonal")
    s_ = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(d, s_):
        np.testing.assert_array_equal(a, b)


def test_split_operands_reject_the_full_attention_forward(small_split):
    base, cfg, w, h = small_split
    e = rmt.storage(embeddings(base, 1), cfg.dtype, device="cuda")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_full_attention_forward(h, e[:10], 10, torch.empty_like(e[:10]))
    assert ex.value.status == rmt.RMT_EINVAL


@pytest.mark.parametrize("name,S,tol", [("tiny", 3, F32_TOL), ("small-bf16", 3, BF16_TOL)])
def test_random_rmsnorm_gains_match_oracle(cuda_ok, name, S, tol):
    """Gains far from 1 exercise the folding of each RMSNorm gain into the next projection."""
    from armt_synthetic import make_weights, round_to_bf16
    cfg = CONFIGS[name]
    w = make_weights(cfg, seed=9)
    rng = np.random.default_rng(10)
    for key in ("g_attn", "g_mlp"):
        g = [np.abs(1 + 0.5 * rng.standard_normal(cfg.d_model)).astype(np.float32) for _ in range(cfg.n_layers)]
        w[key] = [round_to_bf16(x) for x in g] if cfg.dtype == "bf16" else g
    w, h = build(cfg, weights=w)
    emb = embeddings(cfg, S, seed=11)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g_, r, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g_, r) < tol, what
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("name", ["small-bf16", "mixed-tiles"])
def test_large_magnitudes_within_f16_range_match_oracle(cuda_ok, name):
    """bf16 mode keeps its tensor-core operands in f16 (largest finite value 65504): the
    residual stream's operand copy, q/k/v, the SwiGLU output and the memory read-out.
    Embeddings scaled to magnitudes of about 10^4 and RMSNorm gains between 0 and 8 keep
    every such operand in range; the result still matches the oracle and no overflow is
    reported. Both the CTA-pair and the single-CTA GEMM epilogues store operands here."""
    import dataclasses

    from armt_synthetic import make_weights, round_to_bf16
    cfg = CONFIGS["small-bf16"]
    if name != "small-bf16":
        cfg = dataclasses.replace(cfg, **MIXED_CONFIGS[name])
    w = make_weights(cfg, seed=21)
    rng = np.random.default_rng(22)
    for key in ("g_attn", "g_mlp"):
        w[key] = [round_to_bf16(np.abs(1 + 2 * rng.standard_normal(cfg.d_model)).astype(np.float32))
                  for _ in range(cfg.n_layers)]
    w, h = build(cfg, weights=w)
    S = 3
    emb = round_to_bf16(embeddings(cfg, S, seed=23) * np.float32(3000))
    assert 9e3 < np.abs(emb).max() < 3e4
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g_, r, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g_, r) < BF16_TOL, what
    rmt.rmt_destroy(h)


def test_f16_operand_overflow_is_reported(small_bf16):
    """Embeddings of magnitude 10^5 overflow the f16 operand copy of the residual stream:
    rmt_sync reports RMT_ERANGE (no fault; the infinities only spoil the outputs), and the
    handle's next forward gives the bits it gave before."""
    cfg, w, h = small_bf16
    S = 2
    emb = embeddings(cfg, S, seed=24)
    before = forward(h, cfg, emb, S, "diagonal")
    big = rmt.storage(emb * np.float32(1e5), cfg.dtype, device="cuda")
    rmt.rmt_forward(h, big, S, "diagonal", torch.empty_like(big))
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_sync(h)
    assert ex.value.status == rmt.RMT_ERANGE
    after = forward(h, cfg, emb, S, "diagonal")
    for a, b in zip(before, after):
        np.testing.assert_array_equal(a, b)


MIXED_CONFIGS = {
    # d_model 192: memo, QKV, O and down stay on single-CTA tiles, gate/up runs on CTA pairs
    "mixed-tiles": dict(n_layers=3, d_model=192, n_heads=3, n_kv_heads=1, head_dim=64, d_ff=384, seg_len=100,
                        n_mem=8, d_k=64, d_v=64),
    # head_dim 128 on CTA pairs; 158 rows per cell end in a ragged token tile
    "pairs-dh128": dict(n_layers=3, d_model=256, n_heads=2, n_kv_heads=1, head_dim=128, d_ff=512, seg_len=150,
                        n_mem=8, d_k=64, d_v=64),
    # 152 rows per cell: the last query tile (24 rows) stacks the 4 heads of the key/value group
    "tail-stacked": dict(n_layers=3, d_model=256, n_heads=4, n_kv_heads=1, head_dim=64, d_ff=512, seg_len=144,
                         n_mem=8, d_k=64, d_v=64),
    # d_k = d_v = 128: the mem-q GEMM stores q, the tcgen05 read runs as a launch of its own and
    # the read-out projection keeps its residual store (no fold)
    "memory-128": dict(n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64, d_ff=512, seg_len=200,
                       n_mem=8, d_k=128, d_v=128),
}


@pytest.mark.parametrize("name", sorted(MIXED_CONFIGS))
def test_bf16_tile_paths_match_oracle(cuda_ok, name):
    import dataclasses
    cfg = dataclasses.replace(CONFIGS["small-bf16"], **MIXED_CONFIGS[name])
    w, h = build(cfg)
    S = 3
    emb = embeddings(cfg, S, seed=12)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g_, r, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g_, r) < BF16_TOL, what
    seq = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(got, seq):
        np.testing.assert_array_equal(a, b)
    if name == "tail-stacked":
        # short last segments: the stacked tail rows past a cell's tokens are masked keys
        embs = [emb[:2 * cfg.seg_len + 37], emb[:cfg.seg_len - 5]]
        outs, A, z = forward_batch(h, cfg, embs, "diagonal")
        outs_ref, A_ref, z_ref = armt.forward_batch(cfg, w, embs, dtype=np.float32)
        for b_ in range(2):
            assert normwise(outs[b_], outs_ref[b_]) < BF16_TOL, b_
        assert normwise(A, A_ref) < BF16_TOL and normwise(z, z_ref) < BF16_TOL
    rmt.rmt_destroy(h)


def _resume(h, cfg, emb, n_segments, A0, z0, schedule="diagonal"):
    """rmt_forward_resume on device buffers from a state (A0, z0); returns (out, A, z) as numpy."""
    e = rmt.storage(emb, cfg.dtype, device="cuda")
    out = torch.empty_like(e)
    A = torch.empty(cfg.n_layers, cfg.d_k, cfg.d_v, device="cuda")
    z = torch.empty(cfg.n_layers, cfg.d_k, device="cuda")
    rmt.rmt_forward_resume(h, e, n_segments, schedule, A0, z0, out, A, z)
    rmt.rmt_sync(h)
    return out.float().cpu().numpy(), A.cpu().numpy(), z.cpu().numpy()


@pytest.mark.parametrize("name,S1,S2", [("tiny", 3, 2), ("small-bf16", 2, 3)])
def test_resume_in_chunks_equals_one_run_bitwise(cuda_ok, name, S1, S2):
    """Prefilling in two chunks (the second resumed from the state the first returned) gives
    the bits of one run: the state after a segment depends only on the segments before it."""
    cfg = CONFIGS[name]
    w, h = build(cfg)
    S, n1 = S1 + S2, S1 * cfg.seg_len
    emb = embeddings(cfg, S, seed=13)
    full = forward(h, cfg, emb, S, "diagonal")
    first = forward(h, cfg, emb[:n1], S1, "diagonal")
    np.testing.assert_array_equal(first[0], full[0][:n1])
    A1 = torch.from_numpy(first[1]).cuda()
    z1 = torch.from_numpy(first[2]).cuda()
    for schedule in ("diagonal", "sequential"):
        second = _resume(h, cfg, emb[n1:], S2, A1, z1, schedule)
        np.testing.assert_array_equal(second[0], full[0][n1:])
        np.testing.assert_array_equal(second[1], full[1])
        np.testing.assert_array_equal(second[2], full[2])
    # host state buffers give the same bits
    host = _resume(h, cfg, emb[n1:], S2, torch.from_numpy(first[1]), torch.from_numpy(first[2]))
    np.testing.assert_array_equal(host[0], full[0][n1:])
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_forward_resume(h, rmt.storage(emb[:cfg.seg_len], cfg.dtype, device="cuda"), 1, "diagonal", A1, None,
                               torch.empty(cfg.seg_len, cfg.d_model, device="cuda"))
    assert ex.value.status == rmt.RMT_EINVAL
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("name,tol", [("tiny", F32_TOL), ("small-bf16", BF16_TOL)])
def test_resume_from_a_given_state_matches_oracle(cuda_ok, name, tol):
    """Both sides start from the same seeded synthetic state (z > 0, as a sum of phi values)."""
    cfg = CONFIGS[name]
    w, h = build(cfg)
    rng = np.random.default_rng(14)
    A0 = (0.1 * rng.standard_normal((cfg.n_layers, cfg.d_k, cfg.d_v))).astype(np.float32)
    z0 = (1.0 + np.abs(rng.standard_normal((cfg.n_layers, cfg.d_k)))).astype(np.float32)
    S = 3
    emb = embeddings(cfg, S, seed=15)
    got = _resume(h, cfg, emb, S, torch.from_numpy(A0).cuda(), torch.from_numpy(z0).cuda())
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32, A0=A0, z0=z0)
    for g_, r, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g_, r) < tol, what
    rmt.rmt_destroy(h)


# ------------------------------------------------ short last segments and batches

@pytest.mark.parametrize("name,tol", [("tiny", F32_TOL), ("small-bf16", BF16_TOL)])
@pytest.mark.parametrize("extra", [1, 37])
def test_short_last_segment_matches_oracle(cuda_ok, name, tol, extra):
    """2 full segments and a third of `extra` tokens: its memory tokens follow its last
    token, keys past them are masked and its memory write reads its last n_mem rows."""
    cfg = CONFIGS[name]
    w, h = build(cfg)
    extra = min(extra, cfg.seg_len - 1)
    emb = embeddings(cfg, 3, seed=16)[:2 * cfg.seg_len + extra]
    got = forward_batch(h, cfg, [emb], "diagonal")
    ref = armt.forward_tokens(cfg, w, emb, dtype=np.float32)
    assert normwise(got[0][0], ref[0]) < tol
    assert normwise(got[1][0], ref[1]) < tol
    assert normwise(got[2][0], ref[2]) < tol
    seq = forward_batch(h, cfg, [emb], "sequential")
    np.testing.assert_array_equal(got[0][0], seq[0][0])
    np.testing.assert_array_equal(got[1], seq[1])
    # the full segments are those of a run without the short one
    full = forward(h, cfg, emb[:2 * cfg.seg_len], 2, "diagonal")
    np.testing.assert_array_equal(got[0][0][:2 * cfg.seg_len], full[0])
    rmt.rmt_destroy(h)


@pytest.mark.parametrize("name,tol", [("tiny", F32_TOL), ("small-bf16", BF16_TOL)])
def test_batch_matches_oracle_and_each_sequence_alone(cuda_ok, name, tol):
    """Sequences of different lengths (short last segments, one shorter than a segment) in
    one batch: each result equals the oracle's and, bit for bit, the sequence run alone."""
    cfg = CONFIGS[name]
    w, h = build(cfg)
    seg = cfg.seg_len
    lens = [3 * seg + 5, seg, 2 * seg - 1, 3]
    embs = [embeddings(cfg, 4, seed=20 + b)[:n] for b, n in enumerate(lens)]
    got = forward_batch(h, cfg, embs, "diagonal")
    outs, A_ref, z_ref = armt.forward_batch(cfg, w, embs, dtype=np.float32)
    for b in range(len(lens)):
        assert got[0][b].shape == (lens[b], cfg.d_model)
        assert normwise(got[0][b], outs[b]) < tol, b
        assert normwise(got[1][b], A_ref[b]) < tol, b
        assert normwise(got[2][b], z_ref[b]) < tol, b
        alone = forward_batch(h, cfg, [embs[b]], "diagonal")
        np.testing.assert_array_equal(got[0][b], alone[0][0])
        np.testing.assert_array_equal(got[1][b], alone[1][0])
        np.testing.assert_array_equal(got[2][b], alone[2][0])
    seq = forward_batch(h, cfg, embs, "sequential")
    for b in range(len(lens)):
        np.testing.assert_array_equal(got[0][b], seq[0][b])
    np.testing.assert_array_equal(got[1], seq[1])
    np.testing.assert_array_equal(got[2], seq[2])
    # the device trace is the batch schedule without its sequence column
    segs = [-(-n // seg) for n in lens]
    trace = rmt.rmt_get_trace(h, cfg.n_layers * sum(segs))
    np.testing.assert_array_equal(trace, armt.schedule_quads(cfg.n_layers, segs, "sequential")[:, [0, 2, 3]])
    rmt.rmt_destroy(h)


def test_batch_with_initial_states_and_pinned_host_buffers(cuda_ok):
    cfg = CONFIGS["small-bf16"]
    w, h = build(cfg)
    rmt.rmt_reserve(h, 3)
    seg = cfg.seg_len
    lens = [2 * seg + 9, seg + 1, 2 * seg]
    embs = [embeddings(cfg, 3, seed=30 + b)[:n] for b, n in enumerate(lens)]
    rng = np.random.default_rng(31)
    A0 = (0.1 * rng.standard_normal((3, cfg.n_layers, cfg.d_k, cfg.d_v))).astype(np.float32)
    z0 = (1.0 + np.abs(rng.standard_normal((3, cfg.n_layers, cfg.d_k)))).astype(np.float32)
    dev = forward_batch(h, cfg, embs, "diagonal", torch.from_numpy(A0).cuda(), torch.from_numpy(z0).cuda())
    pinned = forward_batch(h, cfg, embs, "diagonal", torch.from_numpy(A0), torch.from_numpy(z0), host=True)
    outs, A_ref, z_ref = armt.forward_batch(cfg, w, embs, dtype=np.float32, A0=A0, z0=z0)
    for b in range(3):
        np.testing.assert_array_equal(dev[0][b], pinned[0][b])
        assert normwise(dev[0][b], outs[b]) < BF16_TOL, b
        assert normwise(dev[1][b], A_ref[b]) < BF16_TOL, b
    np.testing.assert_array_equal(dev[1], pinned[1])
    np.testing.assert_array_equal(dev[2], pinned[2])
    rmt.rmt_destroy(h)


def test_batch_argument_errors(tiny):
    cfg, w, h = tiny
    e = rmt.storage(embeddings(cfg, 1), cfg.dtype, device="cuda")
    out = torch.empty_like(e)
    for lens in ([], [0], [cfg.seg_len, -3]):
        with pytest.raises(rmt.RmtError) as ex:
            rmt.rmt_forward_batch(h, e, lens, "diagonal", out)
        assert ex.value.status == rmt.RMT_EINVAL
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_reserve(h, 0)
    assert ex.value.status == rmt.RMT_EINVAL
    # the handle is still usable
    rmt.rmt_forward_batch(h, e, [cfg.seg_len], "diagonal", out)
    rmt.rmt_sync(h)


# ------------------------------------------------ full-attention comparison model

def _full(h, cfg, emb):
    e = rmt.storage(emb, cfg.dtype, device="cuda")
    out = torch.empty_like(e)
    rmt.rmt_full_attention_forward(h, e, emb.shape[0], out)
    rmt.rmt_sync(h)
    return out.float().cpu().numpy()


@pytest.mark.parametrize("T", [1, 130, 176, 455])
def test_full_attention_matches_oracle(cuda_ok, T):
    """The decoder stack without the memory, causal over T tokens (one or several query tiles
    with a ragged tail), against the oracle's comparison model."""
    cfg = CONFIGS["small-bf16"]
    w, h = build(cfg)
    emb = embeddings(cfg, 3, seed=40)[:T]
    got = _full(h, cfg, emb)
    ref = armt.full_attention_forward(cfg, w, emb, dtype=np.float32)
    assert normwise(got, ref) < BF16_TOL
    # a longer call reallocates; a shorter one after it reuses the buffers with the same bits
    if T > 1:
        _full(h, cfg, embeddings(cfg, 3, seed=41))
        np.testing.assert_array_equal(_full(h, cfg, emb), got)
    # host buffers (staged through device copies) give the same bits
    e_host = rmt.storage(emb, cfg.dtype, device="cuda").cpu()
    o_host = torch.empty_like(e_host)
    rmt.rmt_full_attention_forward(h, e_host, T, o_host)
    rmt.rmt_sync(h)
    np.testing.assert_array_equal(o_host.float().numpy(), got)
    rmt.rmt_destroy(h)


def test_full_attention_argument_errors(tiny, cuda_ok):
    cfg, w, h = tiny  # an fp32 handle
    e = rmt.storage(embeddings(cfg, 1), cfg.dtype, device="cuda")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_full_attention_forward(h, e, cfg.seg_len, torch.empty_like(e))
    assert ex.value.status == rmt.RMT_EINVAL
    cfg2 = CONFIGS["small-bf16"]
    w2, h2 = build(cfg2)
    e2 = rmt.storage(embeddings(cfg2, 1), cfg2.dtype, device="cuda")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_full_attention_forward(h2, e2, 0, torch.empty_like(e2))
    assert ex.value.status == rmt.RMT_EINVAL
    rmt.rmt_destroy(h2)


def test_full_attention_1b_at_131k(model_1b):
    """The comparison model at the bench's size: LLaMA-1B shape, 131,072 tokens, one causal
    segment. The oracle cannot run it in seconds, so: the first 1024 rows equal a 1024-token
    run bit for bit (a row never depends on later tokens, and both runs tile tokens by 256),
    and that run matches the oracle within the bf16 tolerance."""
    cfg, w, h = model_1b
    T, P = 131072, 1024
    emb = embeddings(cfg, T // cfg.seg_len)
    full = _full(h, cfg, emb)
    assert np.isfinite(full).all()
    part = _full(h, cfg, emb[:P])
    np.testing.assert_array_equal(full[:P], part)
    ref = armt.full_attention_forward(cfg, w, emb[:P], dtype=np.float32)
    assert normwise(part, ref) < BF16_TOL


def test_failed_reservation_leaves_the_handle_usable(cuda_ok):
    """A reservation that cannot fit on the device fails with RMT_ENOMEM (a real cudaMalloc
    failure, no fault), and the next forward reserves again and gives the same bits."""
    cfg = CONFIGS["small-bf16"]
    w, h = build(cfg)
    emb = embeddings(cfg, 2, seed=50)
    before = forward(h, cfg, emb, 2, "diagonal")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_reserve(h, 10_000_000)  # several TB of activations
    assert ex.value.status == rmt.RMT_ENOMEM
    after = forward(h, cfg, emb, 2, "diagonal")
    for a, b in zip(before, after):
        np.testing.assert_array_equal(a, b)
    rmt.rmt_destroy(h)


def _random_bf16_config(seed):
    """A small valid bf16 shape drawn from a seeded generator: d_model, heads x head_dim, d_v
    multiples of 64; d_ff a multiple of 64; any segment length; n_mem * (d_k + d_v) <= 4096."""
    import dataclasses
    r = np.random.default_rng(seed)
    dh = int(r.choice([64, 128]))
    hkv = int(r.integers(1, 3))
    hq = hkv * int(r.integers(1, 4))
    d = int(r.choice([128, 192, 256, 320, 512]))  # multiples of 256 put O and down on CTA pairs
    # d_k = d_v = 64 takes the fused read (and, with O on CTA pairs, the read-out fold)
    dk, dv = [(32, 64), (64, 64), (64, 64), (64, 128), (128, 128)][int(r.integers(0, 5))]
    n_mem = int(r.integers(1, 4096 // (dk + dv) + 1)) if r.random() < 0.3 else int(r.integers(1, 17))
    return dataclasses.replace(CONFIGS["small-bf16"], n_layers=int(r.integers(1, 4)), d_model=d, n_heads=hq,
                               n_kv_heads=hkv, head_dim=dh, d_ff=64 * int(r.integers(2, 9)),
                               seg_len=int(r.integers(1, 300)), n_mem=min(n_mem, 64), d_k=dk, d_v=dv)


@pytest.mark.parametrize("seed", range(10))
def test_random_bf16_shapes_match_oracle(cuda_ok, seed):
    """Seeded random shapes (head_dim 64 or 128, GQA ratios, widths that put the projections
    on CTA pairs or single CTAs, d_k / d_v that do or do not take the fused read, ragged
    token tiles): every one matches the oracle, DIAGONAL equals SEQUENTIAL bit for bit, and a
    two-sequence batch with a short last segment equals its sequences run alone."""
    cfg = _random_bf16_config(seed)
    w, h = build(cfg)
    S = 3
    emb = embeddings(cfg, S, seed=60 + seed)
    got = forward(h, cfg, emb, S, "diagonal")
    ref = armt.forward(cfg, w, emb, S, dtype=np.float32)
    for g_, r_, what in zip(got, ref, ("out", "A", "z")):
        assert normwise(g_, r_) < BF16_TOL, (what, cfg)
    seq = forward(h, cfg, emb, S, "sequential")
    for a, b in zip(got, seq):
        np.testing.assert_array_equal(a, b)
    lens = [2 * cfg.seg_len + max(1, cfg.seg_len // 3), cfg.seg_len]
    embs = [emb[:lens[0]], embeddings(cfg, 1, seed=70 + seed)]
    batch = forward_batch(h, cfg, embs, "diagonal")
    for b_ in range(2):
        alone = forward_batch(h, cfg, [embs[b_]], "diagonal")
        np.testing.assert_array_equal(batch[0][b_], alone[0][0])
    rmt.rmt_destroy(h)


def test_many_distinct_lengths_evict_old_tables(tiny):
    """Each distinct (token counts, schedule) keeps a cell table on the device, at most 64 of
    them: 70 different lengths evict the oldest, and a length whose table was evicted runs
    again with the same bits."""
    cfg, w, h = tiny
    emb = embeddings(cfg, 2)
    first = forward_batch(h, cfg, [emb[:1]], "diagonal")
    for n in range(2, 72):
        forward_batch(h, cfg, [emb[:n]], "diagonal")
    again = forward_batch(h, cfg, [emb[:1]], "diagonal")  # its table was evicted and is rebuilt
    np.testing.assert_array_equal(first[0][0], again[0][0])
    np.testing.assert_array_equal(first[1], again[1])
    last = forward_batch(h, cfg, [emb[:71]], "diagonal")
    ref = armt.forward_tokens(cfg, w, emb[:71], dtype=np.float32)
    assert normwise(last[0][0], ref[0]) < F32_TOL

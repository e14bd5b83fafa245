"""Pins for the oracle (CPU only): library routines, closed forms, invariants, fp64.

Each test checks the oracle against something other than itself: torch's functional
ops (elu, silu, rms_norm, scaled_dot_product_attention, complex rotation for RoPE),
hand-derived memory cases (tests/golden/memory_worked.json), closed forms, and
structural invariants of the segment recurrence.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from armt_synthetic import CONFIGS, make_embeddings, make_weights
from oracle import armt

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def normwise(a, b):
    return float(np.max(np.abs(np.asarray(a, np.float64) - b)) / max(np.max(np.abs(b)), 1e-300))


# ------------------------------------------------------------------ elementwise pieces

def test_phi_special_values_and_elu():
    assert armt.phi(np.array([0.0]))[0] == 1.0
    assert armt.phi(np.array([2.0]))[0] == 3.0
    assert armt.phi(np.array([-1.0]))[0] == pytest.approx(math.exp(-1.0), rel=1e-15)
    assert armt.phi(np.array([-1000.0]))[0] == 0.0
    x = np.random.default_rng(3).standard_normal(10000) * 4
    ref = (F.elu(torch.from_numpy(x)) + 1).numpy()
    # torch forms elu as expm1(x) and then adds 1: one ulp of 1.0 apart for tiny exp(x)
    np.testing.assert_allclose(armt.phi(x), ref, rtol=1e-14, atol=3e-16)


def test_silu_matches_torch():
    x = np.random.default_rng(4).standard_normal(10000) * 6
    np.testing.assert_allclose(armt.silu(x), F.silu(torch.from_numpy(x)).numpy(), rtol=1e-13, atol=1e-300)


def test_rms_norm_matches_torch():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 96))
    g = rng.standard_normal(96)
    ref = F.rms_norm(torch.from_numpy(x), (96,), weight=torch.from_numpy(g), eps=1e-5).numpy()
    np.testing.assert_allclose(armt.rms_norm(x, g, 1e-5), ref, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    x = np.random.default_rng(6).standard_normal((5, 3, 16))
    y = armt.rope(x, 500000.0)
    np.testing.assert_array_equal(y[0], x[0])


def test_rope_two_dims_is_rotation_by_position_radians():
    # dh = 2: one pair with inverse frequency theta^0 = 1, so position p rotates by p rad.
    m = 9
    x = np.tile(np.array([[[1.0, 0.0]]]), (m, 1, 1))
    y = armt.rope(x, 10000.0)
    p = np.arange(m)
    np.testing.assert_allclose(y[:, 0, 0], np.cos(p), rtol=0, atol=1e-15)
    np.testing.assert_allclose(y[:, 0, 1], np.sin(p), rtol=0, atol=1e-15)


def test_rope_as_complex_multiplication():
    rng = np.random.default_rng(7)
    m, h, dh, theta = 40, 3, 64, 500000.0
    x = rng.standard_normal((m, h, dh))
    half = dh // 2
    z = x[..., :half] + 1j * x[..., half:]
    w = np.exp(1j * np.outer(np.arange(m), theta ** (-np.arange(half) / half)))
    zr = z * w[:, None, :]
    np.testing.assert_allclose(armt.rope(x, theta), np.concatenate([zr.real, zr.imag], -1), atol=1e-12)


def test_rope_scores_depend_on_position_difference_only():
    rng = np.random.default_rng(8)
    dh = 32
    q, k = rng.standard_normal(dh), rng.standard_normal(dh)
    m = 50
    rq = armt.rope(np.tile(q, (m, 1, 1)), 500000.0)[:, 0]
    rk = armt.rope(np.tile(k, (m, 1, 1)), 500000.0)[:, 0]
    for delta in (0, 3, 17):
        vals = [rq[i + delta] @ rk[i] for i in range(0, m - delta, 5)]
        np.testing.assert_allclose(vals, vals[0], rtol=1e-11)


# ---------------------------------------------------------------------------- attention

@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 1)])
def test_attention_matches_sdpa(hq, hkv):
    rng = np.random.default_rng(9)
    m, dh = 37, 16
    q = rng.standard_normal((m, hq, dh))
    k = rng.standard_normal((m, hkv, dh))
    v = rng.standard_normal((m, hkv, dh))
    tq, tk, tv = (torch.from_numpy(a).transpose(0, 1)[None] for a in (q, k, v))
    ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=True)[0].transpose(0, 1).numpy()
    np.testing.assert_allclose(armt.causal_gqa_attention(q, k, v), ref, rtol=1e-12, atol=1e-13)


def test_attention_first_row_returns_first_value():
    rng = np.random.default_rng(10)
    q, k, v = (rng.standard_normal((6, 2, 8)) for _ in range(3))
    out = armt.causal_gqa_attention(q, k, v)
    np.testing.assert_array_equal(out[0], v[0])


# ------------------------------------------------------------------- associative memory

def _memory_cases():
    with open(os.path.join(GOLDEN, "memory_worked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _memory_cases(), ids=lambda c: c["name"])
@pytest.mark.parametrize("dtype,tol", [(np.float64, 1e-12), (np.float32, 2e-6)])
def test_memory_worked_cases(case, dtype, tol):
    A0 = np.array(case["A0"], dtype)
    z0 = np.array(case["z0"], dtype)
    A, z = armt.memory_update(np.array(case["k"], dtype), np.array(case["v"], dtype), A0, z0, case["eps_update"])
    np.testing.assert_allclose(A, case["A"], rtol=tol, atol=tol)
    np.testing.assert_allclose(z, case["z"], rtol=tol, atol=tol)
    for r in case["reads"]:
        o = armt.memory_read(np.array([r["q"]], dtype), A, z, r["eps"])[0]
        np.testing.assert_allclose(o, r["o"], rtol=tol, atol=tol)


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (16, 48)])
def test_memory_orthonormal_keys_return_their_values(dk, dv):
    """Keys with phi(k_i) = e_i: after one write from empty, reading k_j returns v_j/(1+eps);
    a second write of the same keys with values v' makes reads return (v' + v eps/(1+eps))/(2+eps)."""
    eps = 1e-6
    rng = np.random.default_rng(11)
    k = np.full((dk, dk), -1000.0)
    np.fill_diagonal(k, 0.0)
    v = rng.standard_normal((dk, dv))
    A, z = armt.memory_update(k, v, np.zeros((dk, dv)), np.zeros(dk), eps)
    np.testing.assert_array_equal(z, np.ones(dk))
    np.testing.assert_allclose(armt.memory_read(k, A, z, eps), v / (1 + eps), rtol=1e-14, atol=1e-15)
    v2 = rng.standard_normal((dk, dv))
    A2, z2 = armt.memory_update(k, v2, A, z, eps)
    np.testing.assert_array_equal(z2, 2 * np.ones(dk))
    expect = (v2 + v * eps / (1 + eps)) / (2 + eps)
    np.testing.assert_allclose(armt.memory_read(k, A2, z2, eps), expect, rtol=1e-13, atol=1e-15)


def test_memory_rewrite_of_stored_pair_is_nearly_noop():
    eps = 1e-6
    k = np.array([[0.0, -1000.0, -1000.0]])
    v = np.array([[1.5, -2.0]])
    A, z = armt.memory_update(k, v, np.zeros((3, 2)), np.zeros(3), eps)
    A2, _ = armt.memory_update(k, v, A, z, eps)
    np.testing.assert_allclose((A2 - A)[0], v[0] * eps / (1 + eps), rtol=1e-9, atol=0)
    np.testing.assert_array_equal((A2 - A)[1:], 0.0)


# per-token delta rule (cfg.mem_update = "sequential")

def test_sequential_update_of_one_row_is_the_batched_update():
    rng = np.random.default_rng(21)
    k, v = rng.standard_normal((1, 24)), rng.standard_normal((1, 40))
    A, z = rng.standard_normal((24, 40)), rng.uniform(1, 10, 24)
    for got, want in zip(armt.memory_update_sequential(k, v, A, z, 1e-6), armt.memory_update(k, v, A, z, 1e-6)):
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)


def test_sequential_update_writes_the_same_key_twice_as_two_writes():
    """Keys with phi(k) = e_0 twice in one cell, values v then v': the per-token rule stores v,
    reads it back as v/(1+eps) and corrects toward v', so a read of e_0 returns
    (v' + v eps/(1+eps)) / (2+eps); the batched rule sees the empty memory for both rows and
    returns the average (v + v')/(2+eps)."""
    eps = 1e-6
    rng = np.random.default_rng(23)
    k = np.full((2, 5), -1000.0)
    k[:, 0] = 0.0
    v = rng.standard_normal((2, 3))
    A0, z0 = np.zeros((5, 3)), np.zeros(5)
    q = k[:1]
    A, z = armt.memory_update_sequential(k, v, A0, z0, eps)
    np.testing.assert_array_equal(z, [2.0, 0, 0, 0, 0])
    np.testing.assert_allclose(armt.memory_read(q, A, z, eps)[0], (v[1] + v[0] * eps / (1 + eps)) / (2 + eps),
                               rtol=1e-13, atol=1e-15)
    Ab, zb = armt.memory_update(k, v, A0, z0, eps)
    np.testing.assert_allclose(armt.memory_read(q, Ab, zb, eps)[0], (v[0] + v[1]) / (2 + eps), rtol=1e-13, atol=1e-15)


def test_sequential_update_equals_one_row_writes_in_order():
    rng = np.random.default_rng(25)
    k, v = rng.standard_normal((9, 16)), rng.standard_normal((9, 12))
    A, z = rng.standard_normal((16, 12)), rng.uniform(1, 10, 16)
    As, zs = armt.memory_update_sequential(k, v, A, z, 1e-6)
    for r in range(9):
        A, z = armt.memory_update(k[r:r + 1], v[r:r + 1], A, z, 1e-6)
    np.testing.assert_allclose(As, A, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(zs, z, rtol=1e-13, atol=1e-13)


def test_sequential_update_matches_the_gram_forward_substitution():
    """The same write from the batched quantities: with G = phi(K) phi(K)^T,
    den_r = phi(k_r) . z + eps + sum_{j<r} G_rj and d_r = V_r - (phi(k_r) A + sum_{j<r} G_rj d_j) / den_r,
    A' = A + phi(K)^T D, z' = z + sum_r phi(k_r) (the form the kernels use)."""
    rng = np.random.default_rng(27)
    n, dk, dv, eps = 16, 32, 24, 1e-6
    k, v = rng.standard_normal((n, dk)), rng.standard_normal((n, dv))
    A, z = 0.1 * rng.standard_normal((dk, dv)), rng.uniform(1, 10, dk)
    fk = np.where(k > 0, k + 1.0, np.exp(np.minimum(k, 0.0)))
    G = fk @ fk.T
    den = fk @ z + eps + np.array([G[r, :r].sum() for r in range(n)])
    D = np.zeros((n, dv))
    for r in range(n):
        D[r] = v[r] - (fk[r] @ A + G[r, :r] @ D[:r]) / den[r]
    As, zs = armt.memory_update_sequential(k, v, A, z, eps)
    np.testing.assert_allclose(As, A + fk.T @ D, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(zs, z + fk.sum(axis=0), rtol=1e-13, atol=1e-13)


# ------------------------------------------------------ independent torch reference model

def _torch_cell(x, lw, A, z, cfg):
    """A LLaMA decoder layer from torch functional ops, with the associative read at the
    input and the delta-rule write from the memory-token rows (elu from torch)."""
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))  # noqa: E731
    X, A, z = t(x), t(A), t(z)
    W = {k: t(v) for k, v in lw.items()}
    m, hq, hkv, dh = X.shape[0], cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    fq = F.elu(X @ W["w_mq"].T) + 1
    X = X + ((fq @ A) / (fq @ z + cfg.mem_eps)[:, None]) @ W["w_mo"].T
    H = F.rms_norm(X, (cfg.d_model,), weight=W["g_attn"], eps=cfg.rms_eps)
    half = dh // 2
    ang = torch.outer(torch.arange(m, dtype=torch.float64),
                      cfg.rope_theta ** (-torch.arange(half, dtype=torch.float64) / half))
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]

    def rotary(y):
        c = torch.complex(y[..., :half], y[..., half:]) * rot
        return torch.cat([c.real, c.imag], -1)

    q = rotary((H @ W["wq"].T).view(m, hq, dh)).transpose(0, 1)[None]
    k = rotary((H @ W["wk"].T).view(m, hkv, dh)).transpose(0, 1)[None]
    v = (H @ W["wv"].T).view(m, hkv, dh).transpose(0, 1)[None]
    a = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)[0].transpose(0, 1).reshape(m, hq * dh)
    X = X + a @ W["wo"].T
    H = F.rms_norm(X, (cfg.d_model,), weight=W["g_mlp"], eps=cfg.rms_eps)
    X = X + (F.silu(H @ W["w_gate"].T) * (H @ W["w_up"].T)) @ W["w_down"].T
    Y = X[cfg.seg_len:]
    fk = F.elu(Y @ W["w_mk"].T) + 1
    vv = Y @ W["w_mv"].T
    vbar = (fk @ A) / (fk @ z + cfg.mem_eps)[:, None]
    return X.numpy(), (A + fk.T @ (vv - vbar)).numpy(), (z + fk.sum(0)).numpy()


def _torch_forward(cfg, w, emb, S):
    L, seg = cfg.n_layers, cfg.seg_len
    A = [np.zeros((cfg.d_k, cfg.d_v)) for _ in range(L)]
    z = [np.zeros(cfg.d_k) for _ in range(L)]
    outs = []
    for s in range(S):
        x = np.concatenate([emb[s * seg:(s + 1) * seg], w["mem_tokens"]]).astype(np.float64)
        for l in range(L):
            lw = {k: v[l] for k, v in w.items() if k != "mem_tokens"}
            x, A[l], z[l] = _torch_cell(x, lw, A[l], z[l], cfg)
        outs.append(x[:seg])
    return np.concatenate(outs), np.stack(A), np.stack(z)


SMALL = CONFIGS["tiny"].with_(n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, d_ff=96,
                               seg_len=12, n_mem=4, d_k=8, d_v=12)


def _random_gains(w, seed):
    rng = np.random.default_rng(seed)
    for key in ("g_attn", "g_mlp"):
        w[key] = [1 + 0.3 * rng.standard_normal(a.shape).astype(np.float32) for a in w[key]]
    return w


def test_cell_with_nonzero_memory_matches_torch_layer():
    cfg = SMALL
    w = _random_gains(make_weights(cfg, seed=21, std=0.2), 22)
    rng = np.random.default_rng(23)
    x = rng.standard_normal((cfg.m_tokens, cfg.d_model))
    A = rng.standard_normal((cfg.d_k, cfg.d_v))
    z = rng.uniform(0.5, 2.0, cfg.d_k)
    lw = armt.layer_weights(w, 1, np.float64)
    got = armt.armt_cell(x, lw, A, z, cfg)
    ref = _torch_cell(x, lw, A, z, cfg)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-11)


def test_forward_matches_torch_reference_model():
    cfg = SMALL
    w = _random_gains(make_weights(cfg, seed=31, std=0.2), 32)
    S = 3
    emb = make_embeddings(cfg, S, seed=33)
    got = armt.forward(cfg, w, emb, S, dtype=np.float64)
    ref = _torch_forward(cfg, w, emb, S)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-11)
    # the memory carries information: the reads of later segments are not trivial
    assert np.abs(got[1]).max() > 0.1


def _torch_forward_tokens(cfg, w, emb):
    """The torch reference model over one sequence of any length: its last segment, if
    short, runs as a segment of a model whose segment length is that segment's length."""
    L, seg, T = cfg.n_layers, cfg.seg_len, emb.shape[0]
    A = [np.zeros((cfg.d_k, cfg.d_v)) for _ in range(L)]
    z = [np.zeros(cfg.d_k) for _ in range(L)]
    outs = []
    for lo in range(0, T, seg):
        part = emb[lo:lo + seg]
        c = cfg.with_(seg_len=part.shape[0])
        x = np.concatenate([part, w["mem_tokens"]]).astype(np.float64)
        for l in range(L):
            lw = {k: v[l] for k, v in w.items() if k != "mem_tokens"}
            x, A[l], z[l] = _torch_cell(x, lw, A[l], z[l], c)
        outs.append(x[:part.shape[0]])
    return np.concatenate(outs), np.stack(A), np.stack(z)


@pytest.mark.parametrize("extra", [1, 5, 11])
def test_short_last_segment_matches_torch_reference_model(extra):
    cfg = SMALL
    w = _random_gains(make_weights(cfg, seed=34, std=0.2), 35)
    emb = make_embeddings(cfg, 3, seed=36)[:2 * cfg.seg_len + extra]
    got = armt.forward_tokens(cfg, w, emb, dtype=np.float64)
    ref = _torch_forward_tokens(cfg, w, emb)
    assert got[0].shape == (2 * cfg.seg_len + extra, cfg.d_model)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-11)


def test_short_sequence_is_one_segment_of_its_own_length():
    """A sequence shorter than a segment gives the result of a model whose segments are
    exactly that long (memory tokens at positions T .. T + n_mem - 1)."""
    cfg = SMALL
    w = make_weights(cfg, seed=37, std=0.2)
    emb = make_embeddings(cfg, 1, seed=38)[:7]
    got = armt.forward_tokens(cfg, w, emb, dtype=np.float64)
    ref = armt.forward(cfg.with_(seg_len=7), w, emb, 1, dtype=np.float64)
    for g, r in zip(got, ref):
        np.testing.assert_array_equal(g, r)
    # and the memory rows are the cell's last rows, not rows seg_len.. of a full segment
    full = armt.forward(cfg, w, make_embeddings(cfg, 1, seed=38), 1, dtype=np.float64)
    assert np.abs(full[1] - got[1]).max() > 1e-6


def test_batch_entries_are_the_sequences_alone():
    cfg = SMALL
    w = make_weights(cfg, seed=39, std=0.2)
    embs = [make_embeddings(cfg, 3, seed=40 + b)[:n] for b, n in enumerate([2 * cfg.seg_len + 3, cfg.seg_len, 4])]
    outs, A, z = armt.forward_batch(cfg, w, embs, dtype=np.float64)
    assert A.shape == (3, cfg.n_layers, cfg.d_k, cfg.d_v) and z.shape == (3, cfg.n_layers, cfg.d_k)
    for b, e in enumerate(embs):
        ref = _torch_forward_tokens(cfg, w, e)
        np.testing.assert_allclose(outs[b], ref[0], rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(A[b], ref[1], rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(z[b], ref[2], rtol=1e-10, atol=1e-11)


def test_full_attention_model_matches_torch_layers():
    """The comparison model: torch decoder layers over the whole sequence. With a zero memory
    state the torch cell's read is exactly zero, and with n_mem = 0 it writes nothing."""
    cfg = SMALL
    w = _random_gains(make_weights(cfg, seed=24, std=0.2), 25)
    T = 2 * cfg.seg_len + 7
    emb = make_embeddings(cfg, 3, seed=26)[:T]
    got = armt.full_attention_forward(cfg, w, emb, dtype=np.float64)
    c = cfg.with_(seg_len=T, n_mem=0)
    x = emb.astype(np.float64)
    for l in range(cfg.n_layers):
        lw = {k: v[l] for k, v in w.items() if k != "mem_tokens"}
        x, _, _ = _torch_cell(x, lw, np.zeros((cfg.d_k, cfg.d_v)), np.zeros(cfg.d_k), c)
    np.testing.assert_allclose(got, x, rtol=1e-10, atol=1e-11)


def test_full_attention_equals_the_first_segment_of_the_armt():
    """Before any memory is written the ARMT's read is exactly zero, and its memory tokens come
    after the segment's tokens, which the causal mask hides from them: a sequence that fits in
    one segment gets the same hidden states from both models."""
    cfg = SMALL
    w = make_weights(cfg, seed=27, std=0.2)
    emb = make_embeddings(cfg, 1, seed=28)[:9]
    full = armt.full_attention_forward(cfg, w, emb, dtype=np.float64)
    armt_out, _, _ = armt.forward_tokens(cfg, w, emb, dtype=np.float64)
    np.testing.assert_allclose(full, armt_out, rtol=1e-12, atol=1e-12)
    # and a second segment does see the memory: the models part there
    emb2 = make_embeddings(cfg, 2, seed=28)
    full2 = armt.full_attention_forward(cfg, w, emb2[cfg.seg_len:], dtype=np.float64)
    armt2, _, _ = armt.forward(cfg, w, emb2, 2, dtype=np.float64)
    assert np.abs(full2 - armt2[cfg.seg_len:]).max() > 1e-6


# -------------------------------------------------------------- recurrence invariants

def test_later_segments_do_not_change_earlier_outputs():
    cfg = SMALL
    w = make_weights(cfg, seed=41, std=0.2)
    S = 3
    emb = make_embeddings(cfg, S, seed=42)
    out, _, _ = armt.forward(cfg, w, emb, S, dtype=np.float64)
    emb2 = emb.copy()
    emb2[2 * cfg.seg_len:] += 1.0
    out2, _, _ = armt.forward(cfg, w, emb2, S, dtype=np.float64)
    np.testing.assert_array_equal(out[:2 * cfg.seg_len], out2[:2 * cfg.seg_len])
    assert np.abs(out[2 * cfg.seg_len:] - out2[2 * cfg.seg_len:]).max() > 1e-3
    # and an earlier segment does change a later one, only through the memory
    emb3 = emb.copy()
    emb3[:cfg.seg_len] += 1.0
    out3, _, _ = armt.forward(cfg, w, emb3, S, dtype=np.float64)
    assert np.abs(out[cfg.seg_len:] - out3[cfg.seg_len:]).max() > 1e-6


def test_segments_are_independent_without_memory_readout():
    cfg = SMALL
    w = make_weights(cfg, seed=51, std=0.2)
    w["w_mo"] = [np.zeros_like(a) for a in w["w_mo"]]
    S = 3
    emb = make_embeddings(cfg, S, seed=52)
    out, A, _ = armt.forward(cfg, w, emb, S, dtype=np.float64)
    seg = cfg.seg_len
    for s in range(S):
        alone, _, _ = armt.forward(cfg, w, emb[s * seg:(s + 1) * seg], 1, dtype=np.float64)
        np.testing.assert_array_equal(out[s * seg:(s + 1) * seg], alone)
    assert np.abs(A).max() > 0  # the memory is still written


def test_state_continuation():
    cfg = SMALL
    w = make_weights(cfg, seed=61, std=0.2)
    emb = make_embeddings(cfg, 3, seed=62)
    seg = cfg.seg_len
    out, A, z = armt.forward(cfg, w, emb, 3, dtype=np.float64)
    o2, A2, z2 = armt.forward(cfg, w, emb[:2 * seg], 2, dtype=np.float64)
    o3, A3, z3 = armt.forward(cfg, w, emb[2 * seg:], 1, dtype=np.float64, A0=A2, z0=z2)
    np.testing.assert_array_equal(out, np.concatenate([o2, o3]))
    np.testing.assert_array_equal(A, A3)
    np.testing.assert_array_equal(z, z3)


def test_first_segment_memory_is_outer_product_of_keys_and_values():
    """From the empty state, v_bar = 0, so A = phi(K)^T V and z = column sums of phi(K)."""
    cfg = SMALL.with_(n_layers=1)
    w = make_weights(cfg, seed=71, std=0.2)
    emb = make_embeddings(cfg, 1, seed=72)
    x = np.concatenate([emb, w["mem_tokens"]]).astype(np.float64)
    lw = armt.layer_weights(w, 0, np.float64)
    y, A, z = armt.armt_cell(x, lw, np.zeros((cfg.d_k, cfg.d_v)), np.zeros(cfg.d_k), cfg)
    K = (F.elu(torch.from_numpy(y[cfg.seg_len:] @ lw["w_mk"].T)) + 1).numpy()
    V = y[cfg.seg_len:] @ lw["w_mv"].T
    np.testing.assert_allclose(A, K.T @ V, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(z, K.sum(0), rtol=1e-13)


def test_fp32_oracle_agrees_with_fp64_on_tiny():
    cfg = CONFIGS["tiny"]
    w = make_weights(cfg)
    emb = make_embeddings(cfg, 4)
    o32, A32, z32 = armt.forward(cfg, w, emb, 4, dtype=np.float32)
    o64, A64, z64 = armt.forward(cfg, w, emb, 4, dtype=np.float64)
    assert normwise(o32, o64) < 1e-5
    assert normwise(A32, A64) < 1e-5
    assert normwise(z32, z64) < 1e-5

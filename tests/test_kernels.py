"""Kernel-level parity on the GPU, through the C ABI, against the oracle's functions (numpy,
float64) and, for the grouped GEMM, against a float64 matmul of the same bf16 operands."""
import numpy as np
import pytest
import torch

from armt_synthetic import round_to_bf16
from oracle import armt
from recurrent_memory_transformer_anti_b200 import rmt
from tests.gpu_util import normwise, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_ok):
    torch.backends.cuda.matmul.allow_tf32 = False
    yield


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ----------------------------------------------------------------------- grouped GEMM

# N % 256 == 0 runs on CTA pairs (tokens along the MMA's N, ragged last token tile), other
# widths on single CTAs (ragged last row tile)
GEMM_CASES = [(g, 1040, n, 2048) for n in (2048, 8192) for g in (1, 2, 4, 8, 16)] + [
    (3, 528, 256, 512), (2, 2064, 128, 128), (1, 100, 64, 64), (5, 16, 320, 192), (2, 1040, 64, 2048),
    (2, 1040, 2048, 64), (1, 129, 192, 8192), (2, 2064, 256, 128), (1, 1, 256, 64), (3, 100, 512, 192),
    (1, 257, 256, 64), (4, 17, 768, 128), (2, 1040, 16384, 128)]


@pytest.mark.parametrize("G,M,N,K", GEMM_CASES)
def test_grouped_gemm_matches_matmul(G, M, N, K):
    r = rng(100 + G * 7 + N)
    a = torch.from_numpy(r.standard_normal((G, M, K), dtype=np.float32)).to(torch.bfloat16).cuda()
    b = torch.from_numpy(r.standard_normal((G, N, K), dtype=np.float32) * np.float32(0.02)).to(torch.bfloat16).cuda()
    c = torch.full((G, M, N), float("nan"), device="cuda")
    rmt.rmt_grouped_gemm_bf16(a, b, c, G, M, N, K, "f32")
    rmt.rmt_sync(None)
    ref = torch.bmm(a.double(), b.double().transpose(1, 2))
    err = ((c.double() - ref).abs().max() / ref.abs().max()).item()
    assert err < 1e-5, err
    cb = torch.empty((G, M, N), device="cuda", dtype=torch.bfloat16)
    rmt.rmt_grouped_gemm_bf16(a, b, cb, G, M, N, K, "bf16")
    rmt.rmt_sync(None)
    err_b = ((cb.double() - ref).abs().max() / ref.abs().max()).item()
    assert err_b < 8e-3, err_b


@pytest.mark.parametrize("N", [128, 256])
def test_grouped_gemm_each_group_uses_its_own_weight(N):
    G, M, K = 4, 200, 128
    a = torch.ones((G, M, K), device="cuda", dtype=torch.bfloat16)
    b = torch.stack([torch.full((N, K), float(g + 1) / 64, device="cuda") for g in range(G)]).to(torch.bfloat16)
    c = torch.empty((G, M, N), device="cuda")
    rmt.rmt_grouped_gemm_bf16(a, b, c, G, M, N, K, "f32")
    rmt.rmt_sync(None)
    for g in range(G):
        assert torch.all(c[g] == 2.0 * (g + 1)), g


# -------------------------------------------------------------------------- attention

ATTN_CASES = [("bf16", 2, 1040, 32, 8, 64), ("bf16", 3, 208, 4, 2, 64), ("bf16", 2, 300, 4, 1, 128),
              ("bf16", 2, 72, 4, 4, 32), ("bf16", 1, 1, 2, 1, 64), ("bf16", 1, 65, 2, 2, 64),
              ("f32", 2, 72, 4, 4, 32), ("f32", 2, 208, 4, 2, 64), ("f32", 1, 130, 2, 1, 128),
              # last query tile stacked across the heads of a key/value group: 3 x 16 rows
              # (two warps idle, one half used), 4 x 8, 3 x 40 in the only tile, 4 x 32 (full)
              ("bf16", 2, 528, 24, 8, 128), ("bf16", 2, 136, 8, 2, 64), ("bf16", 1, 40, 6, 2, 64),
              ("bf16", 2, 160, 8, 2, 64)]


@pytest.mark.parametrize("dtype,G,M,H,Hkv,dh", ATTN_CASES)
def test_attention_matches_oracle(dtype, G, M, H, Hkv, dh):
    r = rng(200 + M + H)
    qkv = r.standard_normal((G, M, (H + 2 * Hkv) * dh), dtype=np.float32)
    if dtype == "bf16":
        qkv = round_to_bf16(qkv)
    t = rmt.storage(qkv, dtype, "cuda")
    out = torch.empty((G, M, H * dh), device="cuda", dtype=t.dtype)
    rmt.rmt_attention(t, out, G, M, H, Hkv, dh, dtype)
    rmt.rmt_sync(None)
    got = to_np(out)
    for g in range(G):
        x = qkv[g].astype(np.float64)
        q = x[:, :H * dh].reshape(M, H, dh)
        k = x[:, H * dh:(H + Hkv) * dh].reshape(M, Hkv, dh)
        v = x[:, (H + Hkv) * dh:].reshape(M, Hkv, dh)
        ref = armt.causal_gqa_attention(q, k, v).reshape(M, H * dh)
        tol = 1.2e-2 if dtype == "bf16" else 2e-5
        assert normwise(got[g], ref) < tol


# ------------------------------------------------------------------------------ memory

# 16-bit outputs with d_k of 64 or 128 take the tcgen05 read (persistent CTAs over 128-row
# tiles, crossing cells: G = 300 puts several cells and a ragged tile in every CTA's range),
# other d_k the mma.sync read; fp32 outputs the fp32 read
@pytest.mark.parametrize("dtype,G,M,dk,dv", [("f32", 3, 1040, 64, 64), ("bf16", 3, 1040, 64, 64),
                                             ("f32", 2, 72, 32, 32), ("f32", 2, 77, 128, 128),
                                             ("f32", 2, 50, 32, 96), ("bf16", 4, 130, 128, 64),
                                             ("bf16", 2, 2064, 128, 128), ("bf16", 300, 130, 64, 32),
                                             ("bf16", 300, 130, 64, 64), ("bf16", 40, 1040, 64, 128),
                                             ("bf16", 1, 1, 64, 64), ("bf16", 2, 300, 32, 64), ("bf16", 3, 77, 96, 96)])
def test_memory_read_matches_oracle(dtype, G, M, dk, dv):
    r = rng(300 + M + dk)
    q = r.standard_normal((G, M, dk), dtype=np.float32)
    A = r.standard_normal((G, dk, dv), dtype=np.float32)
    z = r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)
    out = torch.empty((G, M, dv), device="cuda", dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    tq, tA, tz = (torch.from_numpy(x).cuda() for x in (q, A, z))
    rmt.rmt_memory_read(tq, tA, tz, out, G, M, dk, dv, 1e-6, dtype)
    rmt.rmt_sync(None)
    got = to_np(out)
    for g in range(G):
        ref = armt.memory_read(q[g].astype(np.float64), A[g].astype(np.float64), z[g].astype(np.float64), 1e-6)
        assert normwise(got[g], ref) < (8e-3 if dtype == "bf16" else 1e-5)


# a launch picks its kernel from G: column slices of 16 (a cluster of d_v / 16 CTAs per cell)
# for few cells, 32 or 64 for more, and the streaming kernel (persistent CTAs, one cell ahead
# in shared memory) for at least four cells per SM; the sums run in the same order in all
@pytest.mark.parametrize("G,n,dk,dv", [(5, 16, 64, 64), (3, 8, 32, 32), (2, 16, 128, 128), (2, 64, 64, 32),
                                       (1, 1, 32, 64), (200, 16, 64, 64), (300, 16, 64, 64), (150, 13, 128, 128),
                                       (700, 16, 64, 64), (650, 7, 32, 96)])
def test_memory_update_matches_oracle(G, n, dk, dv):
    r = rng(400 + n + dk)
    k = r.standard_normal((G, n, dk), dtype=np.float32)
    v = r.standard_normal((G, n, dv), dtype=np.float32)
    A = r.standard_normal((G, dk, dv), dtype=np.float32)
    z = r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)
    tk, tv, tA, tz = (torch.from_numpy(x).cuda() for x in (k, v, A, z))
    rmt.rmt_memory_update(tk, tv, tA, tz, G, n, dk, dv, 1e-6)
    rmt.rmt_sync(None)
    for g in range(G):
        rA, rz = armt.memory_update(k[g].astype(np.float64), v[g].astype(np.float64), A[g].astype(np.float64),
                                    z[g].astype(np.float64), 1e-6)
        assert normwise(to_np(tA[g]), rA) < 1e-5
        assert normwise(to_np(tz[g]), rz) < 1e-6


def test_memory_update_bits_do_not_depend_on_the_column_slicing():
    """The same cells updated in a launch of 4 cells (16-column slices), of 400 cells (64-column
    slices) and of 700 cells (the streaming kernel) give the same bits."""
    r = rng(450)
    G, n, dk, dv = 700, 16, 64, 64
    k = torch.from_numpy(r.standard_normal((G, n, dk), dtype=np.float32)).cuda()
    v = torch.from_numpy(r.standard_normal((G, n, dv), dtype=np.float32)).cuda()
    A0 = torch.from_numpy(r.standard_normal((G, dk, dv), dtype=np.float32)).cuda()
    z0 = torch.from_numpy(r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)).cuda()
    A_all, z_all = A0.clone(), z0.clone()
    rmt.rmt_memory_update(k, v, A_all, z_all, G, n, dk, dv, 1e-6)
    for m in (4, 400):
        A_few, z_few = A0[:m].clone(), z0[:m].clone()
        rmt.rmt_memory_update(k[:m].contiguous(), v[:m].contiguous(), A_few, z_few, m, n, dk, dv, 1e-6)
        rmt.rmt_sync(None)
        assert torch.equal(A_all[:m], A_few) and torch.equal(z_all[:m], z_few), m


@pytest.mark.parametrize("G,n,dk,dv", [(5, 16, 64, 64), (3, 8, 32, 32), (2, 16, 128, 128), (2, 64, 64, 32),
                                       (1, 1, 32, 64), (300, 16, 64, 64), (150, 13, 128, 128), (700, 16, 64, 64)])
def test_memory_update_sequential_matches_oracle(G, n, dk, dv):
    """The per-token delta rule (rows written one after another) against the oracle's row loop;
    G = 700 runs the streaming kernel, the others the cluster kernel."""
    r = rng(600 + n + dk)
    k = r.standard_normal((G, n, dk), dtype=np.float32)
    v = r.standard_normal((G, n, dv), dtype=np.float32)
    A = r.standard_normal((G, dk, dv), dtype=np.float32)
    z = r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)
    tk, tv, tA, tz = (torch.from_numpy(x).cuda() for x in (k, v, A, z))
    rmt.rmt_memory_update_sequential(tk, tv, tA, tz, G, n, dk, dv, 1e-6)
    rmt.rmt_sync(None)
    for g in range(G):
        rA, rz = armt.memory_update_sequential(k[g].astype(np.float64), v[g].astype(np.float64),
                                               A[g].astype(np.float64), z[g].astype(np.float64), 1e-6)
        assert normwise(to_np(tA[g]), rA) < 1e-5
        assert normwise(to_np(tz[g]), rz) < 1e-6


def test_memory_update_sequential_bits_do_not_depend_on_the_launch():
    r = rng(650)
    G, n, dk, dv = 700, 16, 64, 64
    k = torch.from_numpy(r.standard_normal((G, n, dk), dtype=np.float32)).cuda()
    v = torch.from_numpy(r.standard_normal((G, n, dv), dtype=np.float32)).cuda()
    A0 = torch.from_numpy(r.standard_normal((G, dk, dv), dtype=np.float32)).cuda()
    z0 = torch.from_numpy(r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)).cuda()
    A_all, z_all = A0.clone(), z0.clone()
    rmt.rmt_memory_update_sequential(k, v, A_all, z_all, G, n, dk, dv, 1e-6)
    for m in (4, 400):
        A_few, z_few = A0[:m].clone(), z0[:m].clone()
        rmt.rmt_memory_update_sequential(k[:m].contiguous(), v[:m].contiguous(), A_few, z_few, m, n, dk, dv, 1e-6)
        rmt.rmt_sync(None)
        assert torch.equal(A_all[:m], A_few) and torch.equal(z_all[:m], z_few), m


def test_memory_update_sequential_overwrites_a_key_written_twice():
    """phi(k) = e_0 for both rows of one cell, values v then v': the per-token rule leaves
    e_0 reading (v' + v eps/(1+eps)) / (2+eps) (the batched rule would give the average)."""
    dk, dv, eps = 32, 32, 1e-6
    k = np.full((1, 2, dk), -1000.0, np.float32)
    k[0, :, 0] = 0.0
    v = rng(8).standard_normal((1, 2, dv), dtype=np.float32)
    A = torch.zeros((1, dk, dv), device="cuda")
    z = torch.zeros((1, dk), device="cuda")
    tk = torch.from_numpy(k).cuda()
    rmt.rmt_memory_update_sequential(tk, torch.from_numpy(v).cuda(), A, z, 1, 2, dk, dv, eps)
    o = torch.empty((1, 1, dv), device="cuda")
    rmt.rmt_memory_read(tk[:, :1].contiguous(), A, z, o, 1, 1, dk, dv, eps, "f32")
    rmt.rmt_sync(None)
    expect = (v[0, 1].astype(np.float64) + v[0, 0] * eps / (1 + eps)) / (2 + eps)
    np.testing.assert_allclose(to_np(o)[0, 0], expect, rtol=1e-6, atol=1e-7)


def test_memory_write_then_read_orthonormal_keys_on_gpu():
    """phi(k_i) = e_i (k = 0 on the diagonal, -1000 elsewhere): after one write from an empty
    memory, the read of k_j returns v_j / (1 + eps)."""
    dk = dv = 64
    eps = 1e-6
    k = np.full((1, dk, dk), -1000.0, np.float32)
    for i in range(dk):
        k[0, i, i] = 0.0
    v = rng(7).standard_normal((1, dk, dv), dtype=np.float32)
    tk, tv = torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()
    A = torch.zeros((1, dk, dv), device="cuda")
    z = torch.zeros((1, dk), device="cuda")
    rmt.rmt_memory_update(tk, tv, A, z, 1, dk, dk, dv, eps)
    o = torch.empty((1, dk, dv), device="cuda")
    rmt.rmt_memory_read(tk, A, z, o, 1, dk, dk, dv, eps, "f32")
    rmt.rmt_sync(None)
    assert torch.all(z == 1.0)
    np.testing.assert_allclose(to_np(o)[0], v[0] / (1 + eps), rtol=2e-7, atol=1e-7)


# ----------------------------------------------------------------------------- RMSNorm

@pytest.mark.parametrize("dtype,rows,d", [("f32", 1040, 2048), ("bf16", 1040, 2048), ("f32", 7, 128),
                                          ("bf16", 33, 3072)])
def test_rmsnorm_matches_oracle(dtype, rows, d):
    r = rng(500 + rows)
    x = r.standard_normal((rows, d), dtype=np.float32) * 3
    g = 1 + 0.1 * r.standard_normal(d, dtype=np.float32)
    if dtype == "bf16":
        g = round_to_bf16(g)
    y = torch.empty((rows, d), device="cuda", dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    rmt.rmt_rmsnorm(torch.from_numpy(x).cuda(), rmt.storage(g, dtype, "cuda"), y, rows, d, 1e-5, dtype)
    rmt.rmt_sync(None)
    ref = armt.rms_norm(x.astype(np.float64), g.astype(np.float64), 1e-5)
    assert normwise(to_np(y), ref) < (5e-3 if dtype == "bf16" else 2e-6)


# bf16 widths that are not a multiple of 8 take the scalar staging path (no 16-byte vectors)
@pytest.mark.parametrize("dtype,G,n,d,dk,dv", [("bf16", 4, 16, 2048, 64, 64), ("f32", 3, 8, 128, 32, 32),
                                               ("bf16", 2, 16, 3072, 128, 128), ("f32", 2, 5, 200, 32, 64),
                                               ("bf16", 2, 16, 100, 32, 32), ("bf16", 2, 7, 260, 32, 64)])
def test_memory_write_matches_oracle(dtype, G, n, d, dk, dv):
    """Key/value projection of n rows (split-K partials reduced in fixed order) + update."""
    r = rng(600 + d + n)
    y = r.standard_normal((G, n, d), dtype=np.float32)
    w = r.standard_normal((G, dk + dv, d), dtype=np.float32) * np.float32(0.02)
    if dtype == "bf16":
        w = round_to_bf16(w)
    A = r.standard_normal((G, dk, dv), dtype=np.float32)
    z = r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)
    tA, tz = torch.from_numpy(A).cuda(), torch.from_numpy(z).cuda()
    rmt.rmt_memory_write(torch.from_numpy(y).cuda(), rmt.storage(w, dtype, "cuda"), tA, tz, G, n, d, dk, dv, 1e-6,
                         dtype)
    rmt.rmt_sync(None)
    for g in range(G):
        y64, w64 = y[g].astype(np.float64), w[g].astype(np.float64)
        rA, rz = armt.memory_update(y64 @ w64[:dk].T, y64 @ w64[dk:].T, A[g].astype(np.float64),
                                    z[g].astype(np.float64), 1e-6)
        assert normwise(to_np(tA[g]), rA) < 2e-5
        assert normwise(to_np(tz[g]), rz) < 2e-6


def test_memory_write_whole_sums_equal_split_partials_bitwise():
    """A write of many groups (at least four per SM, bf16 weights) adds each group's split-K
    partials inside one CTA and hands the update whole sums (the streaming update kernel); a
    write of few groups goes through the partials and the cluster update. The same groups give
    the same bits either way, so one launch of 600 groups equals six launches of 100."""
    G, chunk, n, d, dk, dv = 600, 100, 16, 2048, 64, 64
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert G >= 4 * sms > chunk  # the two routes
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    y = torch.randn(G, n, d, device="cuda", generator=gen)
    w = (torch.randn(G, dk + dv, d, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    A0 = torch.randn(G, dk, dv, device="cuda", generator=gen)
    z0 = torch.rand(G, dk, device="cuda", generator=gen) * 99 + 1
    A1, z1 = A0.clone(), z0.clone()
    rmt.rmt_memory_write(y, w, A1, z1, G, n, d, dk, dv, 1e-6, "bf16")
    A2, z2 = A0.clone(), z0.clone()
    for g0 in range(0, G, chunk):
        sl = slice(g0, g0 + chunk)
        a_, z_ = A2[sl].contiguous(), z2[sl].contiguous()
        rmt.rmt_memory_write(y[sl].contiguous(), w[sl].contiguous(), a_, z_, chunk, n, d, dk, dv, 1e-6, "bf16")
        A2[sl], z2[sl] = a_, z_
    rmt.rmt_sync(None)
    assert torch.equal(A1, A2) and torch.equal(z1, z2)
    assert not torch.equal(A1, A0)
    # and the whole route against the oracle on a few groups
    for g in (0, 299, 599):
        y64 = y[g].double().cpu().numpy()
        w64 = w[g].float().double().cpu().numpy()
        rA, rz = armt.memory_update(y64 @ w64[:dk].T, y64 @ w64[dk:].T, A0[g].double().cpu().numpy(),
                                    z0[g].double().cpu().numpy(), 1e-6)
        assert normwise(to_np(A1[g]), rA) < 2e-5
        assert normwise(to_np(z1[g]), rz) < 2e-6


def test_bounded_wait_gives_up_and_reports_without_a_fault(cuda_ok):
    """The failure path of every kernel: a wait on a barrier that nothing signals, and a wait on a
    global counter that nothing increments (the chained projections' dependency wait), each
    give up after their limit, the error word reaches the host as RMT_ETIMEOUT, and the context
    stays usable."""
    import time

    rmt.rmt_sync(None)  # clean error word
    t0 = time.perf_counter()
    rmt.rmt_wait_selftest(20000)  # 20 ms
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_sync(None)
    assert ex.value.status == rmt.RMT_ETIMEOUT
    assert time.perf_counter() - t0 >= 0.035
    rmt.rmt_sync(None)  # the word was cleared
    # the device still runs kernels: a small grouped GEMM after the timeout is correct
    G, M, N, K = 2, 130, 256, 128
    a = torch.randn(G, M, K, device="cuda").to(torch.bfloat16)
    b = (torch.randn(G, N, K, device="cuda") * 0.05).to(torch.bfloat16)
    c = torch.empty(G, M, N, device="cuda")
    rmt.rmt_grouped_gemm_bf16(a, b, c, G, M, N, K, "f32")
    rmt.rmt_sync(None)
    ref = torch.einsum("gmk,gnk->gmn", a.float(), b.float())
    assert (c - ref).abs().max().item() / ref.abs().max().item() < 1e-2
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_wait_selftest(0)
    assert ex.value.status == rmt.RMT_EINVAL

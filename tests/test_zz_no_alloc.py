"""rmt_memory_write_noalloc against rmt_memory_write, on the GPU through the C ABI.

The allocation-free variant is for callers that cannot let a library call cudaMalloc,
such as a serving engine or caching allocator that already owns the device's memory
(there cudaMalloc can fail, and it synchronizes the device). It must give the results of
the allocating entry point, call after call, although its scratch (cell table and split-K
partial sums) lives in one fixed device array that every call reuses.
"""
import numpy as np
import pytest
import torch

from armt_synthetic import round_to_bf16
from recurrent_memory_transformer_anti_b200 import rmt

pytestmark = pytest.mark.gpu


def normwise(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("dtype,G,n,d,dk,dv", [("bf16", 16, 16, 2048, 64, 64), ("f32", 3, 8, 200, 32, 32)])
def test_noalloc_memory_write_matches_allocating_entry_point(cuda_ok, dtype, G, n, d, dk, dv):
    r = np.random.Generator(np.random.PCG64(700 + d))
    A0 = torch.from_numpy(r.standard_normal((G, dk, dv), dtype=np.float32)).cuda()
    z0 = torch.from_numpy(r.uniform(1.0, 100.0, (G, dk)).astype(np.float32)).cuda()
    A_ref, z_ref = A0.clone(), z0.clone()
    A_new, z_new = A0.clone(), z0.clone()
    for _ in range(2):  # two calls in a row: the second reuses the scratch the first left behind
        y = torch.from_numpy(r.standard_normal((G, n, d), dtype=np.float32)).cuda()
        w = r.standard_normal((G, dk + dv, d), dtype=np.float32) * np.float32(0.02)
        w = rmt.storage(round_to_bf16(w) if dtype == "bf16" else w, dtype, "cuda")
        rmt.rmt_memory_write(y, w, A_ref, z_ref, G, n, d, dk, dv, 1e-6, dtype)
        rmt.rmt_memory_write_noalloc(y, w, A_new, z_new, G, n, d, dk, dv, 1e-6, dtype)
        rmt.rmt_sync(None)
        assert normwise(A_new, A_ref) < 2e-5
        assert normwise(z_new, z_ref) < 2e-6
        assert normwise(A_new, A0) > 1e-6  # the state really moved


def test_noalloc_allocates_no_device_memory(cuda_ok):
    """After one call on the device (which loads the module that holds the fixed array), a
    call larger than any before it leaves the device's free memory exactly as it was: no
    allocation, no growth of a scratch buffer."""
    G0, G, n, d, dk, dv = 2, 48, 16, 2048, 64, 64  # 48*16*16*128*4 B = 6 MiB of partial sums
    r = np.random.Generator(np.random.PCG64(710))
    y = torch.from_numpy(r.standard_normal((G, n, d), dtype=np.float32)).cuda()
    w = rmt.storage(round_to_bf16(r.standard_normal((G, dk + dv, d), dtype=np.float32) * np.float32(0.02)), "bf16",
                    "cuda")
    A = torch.zeros((G, dk, dv), device="cuda")
    z = torch.zeros((G, dk), device="cuda")
    rmt.rmt_memory_write_noalloc(y, w, A, z, G0, n, d, dk, dv, 1e-6, "bf16")
    rmt.rmt_sync(None)
    free_before = torch.cuda.mem_get_info()[0]
    rmt.rmt_memory_write_noalloc(y, w, A, z, G, n, d, dk, dv, 1e-6, "bf16")
    rmt.rmt_sync(None)
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.isfinite(A).all() and A.abs().max() > 0


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_ok):
    G, n, d, dk, dv = 64, 16, 2048, 128, 128  # 64*16*16*256*4 B = 16 MiB of partial sums > 8 MiB
    y = torch.zeros((G, n, d), device="cuda")
    w = torch.zeros((G, dk + dv, d), device="cuda")
    A = torch.zeros((G, dk, dv), device="cuda")
    z = torch.zeros((G, dk), device="cuda")
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_memory_write_noalloc(y, w, A, z, G, n, d, dk, dv, 1e-6, "f32")
    assert ex.value.status == rmt.RMT_EINVAL
    assert "scratch" in str(ex.value)


def test_noalloc_many_groups_take_whole_sums_and_match_bitwise(cuda_ok):
    """A launch of at least four groups per SM (bf16 weights, n <= 16) adds each group's split-K
    partials inside one CTA, so only the sums (G*n*(dk+dv)*4 bytes, 4.9 MB at 600 groups) use the
    fixed scratch: a size whose partials (78 MB) it could not hold. The results are the
    allocating entry point's, bit for bit."""
    G, n, d, dk, dv = 600, 16, 2048, 64, 64
    assert G >= 4 * torch.cuda.get_device_properties(0).multi_processor_count
    gen = torch.Generator(device="cuda")
    gen.manual_seed(12)
    y = torch.randn(G, n, d, device="cuda", generator=gen)
    w = (torch.randn(G, dk + dv, d, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    A0 = torch.randn(G, dk, dv, device="cuda", generator=gen)
    z0 = torch.rand(G, dk, device="cuda", generator=gen) * 99 + 1
    A_ref, z_ref = A0.clone(), z0.clone()
    A_new, z_new = A0.clone(), z0.clone()
    rmt.rmt_memory_write(y, w, A_ref, z_ref, G, n, d, dk, dv, 1e-6, "bf16")
    rmt.rmt_memory_write_noalloc(y, w, A_new, z_new, G, n, d, dk, dv, 1e-6, "bf16")
    rmt.rmt_sync(None)
    assert torch.equal(A_new, A_ref) and torch.equal(z_new, z_ref)
    assert not torch.equal(A_new, A0)

"""C-ABI checks that need no GPU: exported symbols, the host scheduler, argument errors."""
import ctypes
import os
import re

import numpy as np
import pytest

from armt_synthetic import CONFIGS
from oracle import armt
from recurrent_memory_transformer_anti_b200 import rmt

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rmt.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rmt_[a-z0-9_]+)\s*\(", text)))


@pytest.mark.parametrize("which", ["release", "debug"])
def test_every_declared_symbol_is_exported(which):
    names = declared_functions()
    assert len(names) >= 13
    path = rmt.LIB_PATH if which == "release" else rmt.DEBUG_LIB_PATH
    assert os.path.exists(path), path
    lib = ctypes.CDLL(path)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rmt.EXPORTED)


def test_release_library_has_no_bounds_selftest():
    with pytest.raises(rmt.RmtError) as ex:
        rmt.rmt_bounds_selftest()
    assert ex.value.status == rmt.RMT_ESTATE


@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_library_schedule_equals_oracle_enumeration(schedule):
    for L in range(1, 13):
        for S in range(1, 13):
            np.testing.assert_array_equal(rmt.rmt_schedule_table(L, S, schedule),
                                          armt.schedule_triples(L, S, schedule))


@pytest.mark.parametrize("schedule", ["diagonal", "sequential"])
def test_library_batch_schedule_equals_oracle_enumeration(schedule):
    rng = np.random.default_rng(5)
    for L in (1, 2, 3, 16):
        for _ in range(12):
            S = [int(v) for v in rng.integers(1, 9, size=int(rng.integers(1, 5)))]
            np.testing.assert_array_equal(rmt.rmt_schedule_table_batch(L, S, schedule),
                                          armt.schedule_quads(L, S, schedule))


def test_batch_schedule_argument_errors():
    lib = rmt.lib()
    buf = (ctypes.c_int32 * 64)()
    ns = (ctypes.c_int32 * 2)(2, 1)
    assert lib.rmt_schedule_table_batch(2, 2, ns, 0, buf, 64) == rmt.RMT_OK
    assert lib.rmt_schedule_table_batch(2, 2, ns, 0, buf, 4 * 6 - 1) == rmt.RMT_EINVAL
    assert lib.rmt_schedule_table_batch(2, 0, ns, 0, buf, 64) == rmt.RMT_EINVAL
    assert lib.rmt_schedule_table_batch(2, 2, None, 0, buf, 64) == rmt.RMT_EINVAL
    bad = (ctypes.c_int32 * 2)(2, 0)
    assert lib.rmt_schedule_table_batch(2, 2, bad, 0, buf, 64) == rmt.RMT_EINVAL
    assert lib.rmt_schedule_table_batch(2, 2, ns, 5, buf, 64) == rmt.RMT_EINVAL


def test_schedule_of_the_131k_workload():
    t = rmt.rmt_schedule_table(16, 128, "diagonal")
    np.testing.assert_array_equal(t, armt.schedule_triples(16, 128, "diagonal"))
    assert t[-1, 0] == 16 + 128 - 2  # 143 diagonals
    sizes = np.bincount(t[:, 0])
    assert sizes.max() == 16 and (sizes == 16).sum() == 128 - 16 + 1


def test_schedule_argument_errors():
    lib = rmt.lib()
    buf = (ctypes.c_int32 * 12)()
    assert lib.rmt_schedule_table(0, 4, 0, buf, 12) == rmt.RMT_EINVAL
    assert lib.rmt_schedule_table(3, 4, 7, buf, 12) == rmt.RMT_EINVAL
    assert lib.rmt_schedule_table(3, 4, 0, buf, 11 * 3) == rmt.RMT_EINVAL  # capacity below 3*L*S
    assert lib.rmt_schedule_table(3, 4, 0, None, 36) == rmt.RMT_EINVAL
    assert "capacity" in rmt.rmt_last_error() or "null" in rmt.rmt_last_error()


def _cfg(**kw):
    return rmt.make_cfg(CONFIGS["tiny"].with_(**kw))


@pytest.mark.parametrize("bad", [dict(n_layers=0), dict(n_heads=3, n_kv_heads=2), dict(head_dim=48),
                                 dict(d_k=40), dict(n_mem=65), dict(d_ff=100), dict(rope_theta=-1.0),
                                 dict(dtype="bf16", d_model=96)])
def test_create_rejects_bad_cfg_without_touching_the_gpu(bad):
    lib = rmt.lib()
    c = _cfg(**bad)
    w = rmt.rmt_weights()
    out = ctypes.c_void_p()
    assert lib.rmt_create(ctypes.byref(w), ctypes.byref(c), ctypes.byref(out)) == rmt.RMT_EINVAL
    assert out.value is None
    assert "invalid cfg" in rmt.rmt_last_error()


def test_null_arguments_return_einval():
    lib = rmt.lib()
    c = _cfg()
    out = ctypes.c_void_p()
    assert lib.rmt_create(None, ctypes.byref(c), ctypes.byref(out)) == rmt.RMT_EINVAL
    assert lib.rmt_forward(None, None, 1, 0, None, None, None, None) == rmt.RMT_EINVAL
    assert lib.rmt_get_trace(None, None, 0) == rmt.RMT_EINVAL
    assert lib.rmt_get_schedule(None, 1, 0, None, 0) == rmt.RMT_EINVAL
    assert lib.rmt_destroy(None) == rmt.RMT_OK
    assert lib.rmt_grouped_gemm_bf16(None, None, None, 1, 1, 64, 64, 0, None) == rmt.RMT_EINVAL
    assert lib.rmt_attention(None, None, 1, 1, 1, 1, 64, 1, None) == rmt.RMT_EINVAL
    assert lib.rmt_memory_read(None, None, None, None, 1, 1, 32, 32, 1e-6, 0, None) == rmt.RMT_EINVAL
    assert lib.rmt_memory_update(None, None, None, None, 1, 1, 32, 32, 1e-6, None) == rmt.RMT_EINVAL
    assert lib.rmt_rmsnorm(None, None, None, 1, 4, 1e-5, 0, None) == rmt.RMT_EINVAL


def test_kernel_entry_points_reject_bad_sizes_before_any_launch():
    lib = rmt.lib()
    p = ctypes.c_void_p(16)  # never dereferenced: the size checks come first
    assert lib.rmt_grouped_gemm_bf16(p, p, p, 1, 16, 64, 100, 0, None) == rmt.RMT_EINVAL  # K % 64
    assert lib.rmt_grouped_gemm_bf16(p, p, p, 1, 16, 96, 64, 0, None) == rmt.RMT_EINVAL   # N % 64
    assert lib.rmt_attention(p, p, 1, 8, 3, 2, 64, 1, None) == rmt.RMT_EINVAL             # H % Hkv
    assert lib.rmt_attention(p, p, 1, 8, 4, 2, 48, 1, None) == rmt.RMT_EINVAL             # dh
    assert lib.rmt_memory_read(p, p, p, p, 1, 8, 40, 32, 1e-6, 0, None) == rmt.RMT_EINVAL
    assert lib.rmt_memory_update(p, p, p, p, 1, 65, 32, 32, 1e-6, None) == rmt.RMT_EINVAL
    assert lib.rmt_rmsnorm(p, p, p, 4, 6, 1e-5, 0, None) == rmt.RMT_EINVAL

"""ctypes binding of librmt.so (include/rmt.h): the same entry points, argument marshalling only.

Every step of the ARMT prefill runs in the library's CUDA kernels. Arrays may be torch
tensors (device or host) or numpy arrays (host); pointers are passed through unchanged.
If librmt.so is missing this module raises at import: there is no fallback path. The
environment variable RMT_LIBRARY selects another build of the same ABI (librmt_debug.so,
the in-kernel bounds-checking build).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("RMT_LIBRARY") or os.path.join(_HERE, "librmt.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "librmt_debug.so")

RMT_OK, RMT_EINVAL, RMT_ENOMEM, RMT_ECUDA, RMT_ETIMEOUT, RMT_ESTATE, RMT_ERANGE, RMT_EDEBUG = range(8)
RMT_DIAGONAL, RMT_SEQUENTIAL = 0, 1
RMT_F32, RMT_BF16, RMT_BF16_SPLIT = 0, 1, 2
SCHEDULES = {"diagonal": RMT_DIAGONAL, "sequential": RMT_SEQUENTIAL}
# "bf16-split": bf16 storage, split (high + low f16 term) tensor-core operands (include/rmt.h)
DTYPES = {"f32": RMT_F32, "bf16": RMT_BF16, "bf16-split": RMT_BF16_SPLIT}
# how a cell writes its memory rows (include/rmt.h rmt_mem_update)
MEM_UPDATES = {"batched": 0, "sequential": 1}
STORAGE_BF16 = ("bf16", "bf16-split")
STATUS_NAMES = {0: "RMT_OK", 1: "RMT_EINVAL", 2: "RMT_ENOMEM", 3: "RMT_ECUDA", 4: "RMT_ETIMEOUT", 5: "RMT_ESTATE",
                6: "RMT_ERANGE", 7: "RMT_EDEBUG"}

EXPORTED = ("rmt_create", "rmt_reserve", "rmt_forward", "rmt_forward_resume", "rmt_forward_batch",
            "rmt_full_attention_forward", "rmt_schedule_table",
            "rmt_schedule_table_batch", "rmt_get_schedule", "rmt_get_trace", "rmt_sync", "rmt_wait_selftest",
            "rmt_bounds_selftest",
            "rmt_destroy", "rmt_last_error", "rmt_grouped_gemm_bf16", "rmt_attention", "rmt_memory_read",
            "rmt_memory_update", "rmt_memory_update_sequential", "rmt_memory_write", "rmt_memory_write_noalloc", "rmt_rmsnorm", "rmt_probe",
            "rmt_probe_read")

KERNELS = ("assemble", "memq", "memread", "memo", "rmsnorm1", "qkv", "attention", "o", "rmsnorm2", "gateup", "down",
           "memkv", "memupdate", "emit")


class RmtError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class rmt_cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "d_ff",
                                               "seg_len", "n_mem", "d_k", "d_v")] + \
               [("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("mem_eps", ctypes.c_float),
                ("dtype", ctypes.c_int), ("mem_update", ctypes.c_int)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class rmt_weights(ctypes.Structure):
    _fields_ = [(n, _PP) for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down", "w_mq", "w_mk", "w_mv", "w_mo",
                                   "g_attn", "g_mlp")] + [("mem_tokens", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m recurrent_memory_transformer_anti_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    p32 = ctypes.POINTER(ctypes.c_int32)
    sigs = {
        "rmt_create": [ctypes.POINTER(rmt_weights), ctypes.POINTER(rmt_cfg), ctypes.POINTER(vp)],
        "rmt_forward": [vp, vp, i32, ctypes.c_int, vp, vp, vp, vp],
        "rmt_forward_resume": [vp, vp, i32, ctypes.c_int, vp, vp, vp, vp, vp, vp],
        "rmt_forward_batch": [vp, vp, i32, p32, ctypes.c_int, vp, vp, vp, vp, vp, vp],
        "rmt_reserve": [vp, i32],
        "rmt_full_attention_forward": [vp, vp, i32, vp, vp],
        "rmt_schedule_table": [i32, i32, ctypes.c_int, p32, sz],
        "rmt_schedule_table_batch": [i32, i32, p32, ctypes.c_int, p32, sz],
        "rmt_get_schedule": [vp, i32, ctypes.c_int, p32, sz],
        "rmt_get_trace": [vp, p32, sz],
        "rmt_sync": [vp, vp],
        "rmt_wait_selftest": [ctypes.c_uint32, vp],
        "rmt_bounds_selftest": [vp],
        "rmt_destroy": [vp],
        "rmt_grouped_gemm_bf16": [vp, vp, vp, i32, i32, i32, i32, ctypes.c_int, vp],
        "rmt_attention": [vp, vp, i32, i32, i32, i32, i32, ctypes.c_int, vp],
        "rmt_memory_read": [vp, vp, vp, vp, i32, i32, i32, i32, f32, ctypes.c_int, vp],
        "rmt_memory_update": [vp, vp, vp, vp, i32, i32, i32, i32, f32, vp],
        "rmt_memory_update_sequential": [vp, vp, vp, vp, i32, i32, i32, i32, f32, vp],
        "rmt_memory_write": [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, ctypes.c_int, vp],
        "rmt_memory_write_noalloc": [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, ctypes.c_int, vp],
        "rmt_rmsnorm": [vp, vp, vp, i32, i32, f32, ctypes.c_int, vp],
        "rmt_probe": [vp, ctypes.c_uint32],
        "rmt_probe_read": [vp, ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                           ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double),
                           ctypes.POINTER(ctypes.c_int64)],
    }
    for name, args in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.rmt_last_error.argtypes = []
    lib.rmt_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def rmt_last_error() -> str:
    return _lib.rmt_last_error().decode()


def _check(status: int, fn: str) -> None:
    if status != RMT_OK:
        raise RmtError(status, fn, rmt_last_error())


def _ptr(x):
    """Raw address of a torch tensor / numpy array (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("numpy arrays must be C-contiguous")
        return x.ctypes.data
    if hasattr(x, "data_ptr"):
        if not x.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return x.data_ptr()
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream if isinstance(stream, int) else stream.cuda_stream


def make_cfg(cfg) -> rmt_cfg:
    """rmt_cfg from an object with the ArmtConfig field names."""
    c = rmt_cfg()
    for n, _ in rmt_cfg._fields_[:10]:
        setattr(c, n, int(getattr(cfg, n)))
    c.rope_theta, c.rms_eps, c.mem_eps = float(cfg.rope_theta), float(cfg.rms_eps), float(cfg.mem_eps)
    c.dtype = DTYPES[cfg.dtype] if isinstance(cfg.dtype, str) else int(cfg.dtype)
    mu = getattr(cfg, "mem_update", "batched")
    c.mem_update = MEM_UPDATES[mu] if isinstance(mu, str) else int(mu)
    return c


class Handle:
    """An rmt_handle* together with the Python objects its creation referenced."""

    def __init__(self, ptr: int, cfg):
        self.ptr = ptr
        self.cfg = cfg

    def __del__(self):
        if getattr(self, "ptr", None) and _lib is not None:  # the module may be torn down at exit
            _lib.rmt_destroy(self.ptr)
            self.ptr = None


def rmt_create(weights: dict, cfg) -> Handle:
    """weights: {key: [per-layer arrays]} + "mem_tokens", stored in cfg.dtype (see include/rmt.h)."""
    keep = []

    def arr(key):
        ptrs = (ctypes.c_void_p * cfg.n_layers)(*[_ptr(a) for a in weights[key]])
        keep.append(ptrs)
        return ctypes.cast(ptrs, _PP)

    w = rmt_weights()
    for n, _ in rmt_weights._fields_[:-1]:
        setattr(w, n, arr(n))
    w.mem_tokens = _ptr(weights["mem_tokens"])
    c = make_cfg(cfg)
    out = ctypes.c_void_p()
    _check(_lib.rmt_create(ctypes.byref(w), ctypes.byref(c), ctypes.byref(out)), "rmt_create")
    return Handle(out.value, cfg)


def rmt_forward(h: Handle, emb, n_segments: int, schedule, out_hidden, out_A=None, out_z=None, stream=None) -> None:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    _check(_lib.rmt_forward(h.ptr, _ptr(emb), int(n_segments), sch, _ptr(out_hidden), _ptr(out_A), _ptr(out_z),
                            _stream(stream)), "rmt_forward")


def rmt_forward_resume(h: Handle, emb, n_segments: int, schedule, in_A, in_z, out_hidden, out_A=None, out_z=None,
                       stream=None) -> None:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    _check(_lib.rmt_forward_resume(h.ptr, _ptr(emb), int(n_segments), sch, _ptr(in_A), _ptr(in_z), _ptr(out_hidden),
                                   _ptr(out_A), _ptr(out_z), _stream(stream)), "rmt_forward_resume")


def rmt_forward_batch(h: Handle, emb, n_tokens, schedule, out_hidden, in_A=None, in_z=None, out_A=None, out_z=None,
                      stream=None) -> None:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    nt = np.ascontiguousarray(np.asarray(n_tokens, dtype=np.int32).reshape(-1))
    _check(_lib.rmt_forward_batch(h.ptr, _ptr(emb), int(nt.size), nt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                  sch, _ptr(in_A), _ptr(in_z), _ptr(out_hidden), _ptr(out_A), _ptr(out_z),
                                  _stream(stream)), "rmt_forward_batch")


def rmt_full_attention_forward(h: Handle, emb, n_tokens: int, out_hidden, stream=None) -> None:
    _check(_lib.rmt_full_attention_forward(h.ptr, _ptr(emb), int(n_tokens), _ptr(out_hidden), _stream(stream)),
           "rmt_full_attention_forward")


def rmt_reserve(h: Handle, max_batch: int) -> None:
    _check(_lib.rmt_reserve(h.ptr, int(max_batch)), "rmt_reserve")


def rmt_schedule_table_batch(n_layers: int, n_segments, schedule) -> np.ndarray:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    ns = np.ascontiguousarray(np.asarray(n_segments, dtype=np.int32).reshape(-1))
    out = np.zeros(4 * n_layers * int(ns.sum()), np.int32)
    _check(_lib.rmt_schedule_table_batch(n_layers, int(ns.size), ns.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), sch,
                                         out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), out.size),
           "rmt_schedule_table_batch")
    return out.reshape(-1, 4)


def rmt_schedule_table(n_layers: int, n_segments: int, schedule) -> np.ndarray:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    out = np.zeros(3 * n_layers * n_segments, np.int32)
    _check(_lib.rmt_schedule_table(n_layers, n_segments, sch, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                   out.size), "rmt_schedule_table")
    return out.reshape(-1, 3)


def rmt_get_schedule(h: Handle, n_segments: int, schedule) -> np.ndarray:
    sch = SCHEDULES[schedule] if isinstance(schedule, str) else int(schedule)
    out = np.zeros(3 * h.cfg.n_layers * n_segments, np.int32)
    _check(_lib.rmt_get_schedule(h.ptr, n_segments, sch, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                 out.size), "rmt_get_schedule")
    return out.reshape(-1, 3)


def rmt_get_trace(h: Handle, n_cells: int) -> np.ndarray:
    out = np.zeros(3 * n_cells, np.int32)
    _check(_lib.rmt_get_trace(h.ptr, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), out.size), "rmt_get_trace")
    return out.reshape(-1, 3)


def rmt_sync(h: Handle | None, stream=None) -> None:
    _check(_lib.rmt_sync(h.ptr if h is not None else None, _stream(stream)), "rmt_sync")


def rmt_wait_selftest(limit_us: int, stream=None) -> None:
    _check(_lib.rmt_wait_selftest(int(limit_us), _stream(stream)), "rmt_wait_selftest")


def rmt_bounds_selftest(stream=None) -> None:
    _check(_lib.rmt_bounds_selftest(_stream(stream)), "rmt_bounds_selftest")


def rmt_destroy(h: Handle) -> None:
    if h.ptr:
        _check(_lib.rmt_destroy(h.ptr), "rmt_destroy")
        h.ptr = None


def rmt_probe(h: Handle, kernels=()) -> None:
    """Time every launch of the named kernel kinds (see KERNELS) in later forwards."""
    mask = 0
    for k in kernels:
        mask |= 1 << KERNELS.index(k)
    _check(_lib.rmt_probe(h.ptr, mask), "rmt_probe")


def rmt_probe_read(h: Handle, kernel: str) -> dict:
    ms, fl, by = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    nl, al = ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.rmt_probe_read(h.ptr, KERNELS.index(kernel), ctypes.byref(ms), ctypes.byref(nl), ctypes.byref(fl),
                               ctypes.byref(by), ctypes.byref(al)), "rmt_probe_read")
    return {"ms": ms.value, "launches": nl.value, "flops": fl.value, "bytes": by.value, "all_launches": al.value}


def rmt_grouped_gemm_bf16(A, B, C, G, M, N, K, out_dtype="f32", stream=None) -> None:
    _check(_lib.rmt_grouped_gemm_bf16(_ptr(A), _ptr(B), _ptr(C), G, M, N, K, DTYPES[out_dtype], _stream(stream)),
           "rmt_grouped_gemm_bf16")


def rmt_attention(qkv, out, G, M, H, Hkv, dh, dtype="bf16", stream=None) -> None:
    _check(_lib.rmt_attention(_ptr(qkv), _ptr(out), G, M, H, Hkv, dh, DTYPES[dtype], _stream(stream)), "rmt_attention")


def rmt_memory_read(q, A, z, o, G, M, dk, dv, eps, dtype="f32", stream=None) -> None:
    _check(_lib.rmt_memory_read(_ptr(q), _ptr(A), _ptr(z), _ptr(o), G, M, dk, dv, eps, DTYPES[dtype],
                                _stream(stream)), "rmt_memory_read")


def rmt_memory_update(k, v, A, z, G, n, dk, dv, eps, stream=None) -> None:
    _check(_lib.rmt_memory_update(_ptr(k), _ptr(v), _ptr(A), _ptr(z), G, n, dk, dv, eps, _stream(stream)),
           "rmt_memory_update")


def rmt_memory_update_sequential(k, v, A, z, G, n, dk, dv, eps, stream=None) -> None:
    _check(_lib.rmt_memory_update_sequential(_ptr(k), _ptr(v), _ptr(A), _ptr(z), G, n, dk, dv, eps,
                                             _stream(stream)), "rmt_memory_update_sequential")


def rmt_memory_write(y, w_mkv, A, z, G, n, d, dk, dv, eps, dtype="f32", stream=None) -> None:
    _check(_lib.rmt_memory_write(_ptr(y), _ptr(w_mkv), _ptr(A), _ptr(z), G, n, d, dk, dv, eps, DTYPES[dtype],
                                 _stream(stream)), "rmt_memory_write")


def rmt_memory_write_noalloc(y, w_mkv, A, z, G, n, d, dk, dv, eps, dtype="f32", stream=None) -> None:
    """rmt_memory_write with its scratch in the library's fixed device array (no cudaMalloc)."""
    _check(_lib.rmt_memory_write_noalloc(_ptr(y), _ptr(w_mkv), _ptr(A), _ptr(z), G, n, d, dk, dv, eps,
                                         DTYPES[dtype], _stream(stream)), "rmt_memory_write_noalloc")


def rmt_rmsnorm(x, g, y, rows, d, eps, dtype="f32", stream=None) -> None:
    _check(_lib.rmt_rmsnorm(_ptr(x), _ptr(g), _ptr(y), rows, d, eps, DTYPES[dtype], _stream(stream)), "rmt_rmsnorm")


def storage(a, dtype: str, device=None):
    """A float32 array as a torch tensor in the model's storage dtype (marshalling helper)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype in STORAGE_BF16 else t
    return t.to(device) if device is not None else t


def weights_storage(weights: dict, dtype: str, device=None) -> dict:
    return {k: ([storage(a, dtype, device) for a in v] if isinstance(v, list) else storage(v, dtype, device))
            for k, v in weights.items()}

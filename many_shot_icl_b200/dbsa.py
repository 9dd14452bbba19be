"""ctypes binding of libdbsa.so (see include/dbsa.h for the contract).

Argument marshalling only: torch tensors are passed as raw device pointers,
host arrays as numpy int32 buffers, and the current torch CUDA stream as the
call's stream.  Every step of the computation runs in the library's CUDA
kernels; there is no fallback.  If the library is missing, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdbsa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
BF16, F32 = 0, 1
PATTERN_SINK_PREV_SELF, PATTERN_FULL, PATTERN_SINK_SELF, PATTERN_SELF = range(4)

SYMBOLS = (
    "dbsa_group_blocks", "dbsa_encode_workspace_size", "dbsa_encode_blocks",
    "dbsa_append_workspace_size", "dbsa_append_block", "dbsa_gather_workspace_size",
    "dbsa_gather_rope_attend", "dbsa_last_error", "dbsa_read_status", "dbsa_stage1_plan",
    "dbsa_stage1_tile_count", "dbsa_version", "dbsa_kernel_launches", "dbsa_set_profile_events",
    "dbsa_gather_rope_attend_noalloc", "dbsa_block_keys_size", "dbsa_block_keys",
    "dbsa_gather_rope_attend_prepared", "dbsa_noalloc_read_status", "dbsa_test_wait_expiry",
    "dbsa_host_allocation_calls",
)


class DbsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("dbsa status %d: %s" % (status, msg))
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("window_j", ctypes.c_int32),
                ("pattern", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("reserved", ctypes.c_int32)]


class TileItem(ctypes.Structure):
    _fields_ = [("head", ctypes.c_int32), ("q_row0", ctypes.c_int32), ("q_pos0", ctypes.c_int32),
                ("n_rows", ctypes.c_int32), ("n_ranges", ctypes.c_int32), ("block", ctypes.c_int32),
                ("k_row0", ctypes.c_int32 * 2), ("v_row0", ctypes.c_int32 * 2),
                ("pos0", ctypes.c_int32 * 2), ("len", ctypes.c_int32 * 2)]


@dataclass(frozen=True)
class DbsaConfig:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str = "bf16"          # "bf16" or "f32"
    rope_theta: float = 1e4
    window_j: int = 2
    pattern: int = PATTERN_SINK_PREV_SELF
    softmax_scale: float = 0.0

    def c(self) -> Config:
        return Config(self.n_q_heads, self.n_kv_heads, self.head_dim,
                      F32 if self.dtype == "f32" else BF16, float(self.rope_theta),
                      self.window_j, self.pattern, float(self.softmax_scale), 0)


_lib = None


def load(path: str = LIB_PATH):
    """Load libdbsa.so (once) and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libdbsa.so not found at %s: build it with "
                           "`python -m many_shot_icl_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(Config)
    lib.dbsa_group_blocks.argtypes = [vp, i32, i32, vp]
    lib.dbsa_group_blocks.restype = i32
    lib.dbsa_encode_workspace_size.argtypes = [cfgp, i64, i32]
    lib.dbsa_encode_workspace_size.restype = sz
    lib.dbsa_encode_blocks.argtypes = [cfgp, vp, vp, vp, vp, i32, vp, vp, i64, vp, vp, sz, vp]
    lib.dbsa_encode_blocks.restype = ctypes.c_int
    lib.dbsa_append_workspace_size.argtypes = [cfgp, vp, i32, i32]
    lib.dbsa_append_workspace_size.restype = sz
    lib.dbsa_append_block.argtypes = [cfgp, vp, vp, vp, i32, vp, i32, vp, vp, i64, vp, vp, sz, vp]
    lib.dbsa_append_block.restype = ctypes.c_int
    lib.dbsa_gather_workspace_size.argtypes = [cfgp, vp, i32, i32, vp, vp, i32, i32]
    lib.dbsa_gather_workspace_size.restype = sz
    lib.dbsa_gather_rope_attend.argtypes = [cfgp, vp, vp, i64, vp, i32, i32, vp, vp, vp, i32, vp,
                                            vp, i32, i32, vp, vp, i64, vp, sz, vp]
    lib.dbsa_gather_rope_attend.restype = ctypes.c_int
    lib.dbsa_gather_rope_attend_noalloc.argtypes = [cfgp, vp, vp, i64, vp, i32, i32, vp, vp, vp,
                                                    i32, vp, vp, i32, i32, vp, vp, i64, vp]
    lib.dbsa_gather_rope_attend_noalloc.restype = ctypes.c_int
    lib.dbsa_block_keys_size.argtypes = [cfgp, vp, i32]
    lib.dbsa_block_keys_size.restype = sz
    lib.dbsa_block_keys.argtypes = [cfgp, vp, vp, i64, vp, i32, vp, sz, vp]
    lib.dbsa_block_keys.restype = ctypes.c_int
    lib.dbsa_gather_rope_attend_prepared.argtypes = [cfgp, vp, vp, i64, vp, i32, i32, vp, vp, vp,
                                                     i32, vp, vp, i32, i32, vp, vp, i64, vp, sz,
                                                     vp, sz, vp]
    lib.dbsa_gather_rope_attend_prepared.restype = ctypes.c_int
    lib.dbsa_last_error.argtypes = []
    lib.dbsa_last_error.restype = ctypes.c_char_p
    lib.dbsa_read_status.argtypes = [vp, vp]
    lib.dbsa_read_status.restype = ctypes.c_int
    lib.dbsa_stage1_plan.argtypes = [cfgp, vp, i32, vp, i64]
    lib.dbsa_stage1_plan.restype = i64
    lib.dbsa_stage1_tile_count.argtypes = [cfgp, vp, i32]
    lib.dbsa_stage1_tile_count.restype = i64
    lib.dbsa_version.argtypes = []
    lib.dbsa_version.restype = ctypes.c_char_p
    lib.dbsa_kernel_launches.argtypes = []
    lib.dbsa_kernel_launches.restype = i64
    lib.dbsa_set_profile_events.argtypes = [vp, vp]
    lib.dbsa_set_profile_events.restype = None
    lib.dbsa_noalloc_read_status.argtypes = [vp]
    lib.dbsa_noalloc_read_status.restype = ctypes.c_int
    lib.dbsa_test_wait_expiry.argtypes = [ctypes.c_uint64]
    lib.dbsa_test_wait_expiry.restype = None
    lib.dbsa_host_allocation_calls.argtypes = []
    lib.dbsa_host_allocation_calls.restype = i64
    _lib = lib
    return lib


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _hp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dp(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status: int):
    if status != OK:
        raise DbsaError(status, load().dbsa_last_error().decode())


def last_error() -> str:
    return load().dbsa_last_error().decode()


def version() -> str:
    return load().dbsa_version().decode()


def group_blocks(demo_len, k: int) -> np.ndarray:
    dl = _i32(demo_len)
    offs = np.zeros((len(dl) + k - 1) // k + 1, dtype=np.int32)
    nb = load().dbsa_group_blocks(_hp(dl), len(dl), k, _hp(offs))
    if nb < 0:
        raise DbsaError(ERR_INVALID_ARG, last_error())
    return offs


def stage1_plan(cfg: DbsaConfig, offs) -> list:
    o = _i32(offs)
    c = cfg.c()
    lib = load()
    n = lib.dbsa_stage1_plan(ctypes.byref(c), _hp(o), len(o) - 1, None, 0)
    if n < 0:
        raise DbsaError(ERR_INVALID_ARG, last_error())
    arr = (TileItem * max(n, 1))()
    lib.dbsa_stage1_plan(ctypes.byref(c), _hp(o), len(o) - 1, ctypes.cast(arr, ctypes.c_void_p), n)
    return list(arr[:n])


def stage1_tile_count(cfg: DbsaConfig, offs) -> int:
    o = _i32(offs)
    c = cfg.c()
    return int(load().dbsa_stage1_tile_count(ctypes.byref(c), _hp(o), len(o) - 1))


def encode_workspace_size(cfg: DbsaConfig, n_tokens: int, nb: int) -> int:
    c = cfg.c()
    return int(load().dbsa_encode_workspace_size(ctypes.byref(c), n_tokens, nb))


def append_workspace_size(cfg: DbsaConfig, offs, L: int) -> int:
    o = _i32(offs)
    c = cfg.c()
    return int(load().dbsa_append_workspace_size(ctypes.byref(c), _hp(o), len(o) - 1, L))


def gather_workspace_size(cfg: DbsaConfig, offs, sel_ptr, sel_blocks, n_new: int,
                          tail_len: int) -> int:
    o, sp, sb = _i32(offs), _i32(sel_ptr), _i32(sel_blocks)
    c = cfg.c()
    return int(load().dbsa_gather_workspace_size(ctypes.byref(c), _hp(o), len(o) - 1,
                                                 len(sp) - 1, _hp(sp), _hp(sb), n_new, tail_len))


def encode_blocks(cfg: DbsaConfig, q, k, v, offs, k_cache, v_cache, out, workspace, stream=None):
    """Stage 1 over all blocks: fills k_cache/v_cache rows [0, T) and out."""
    o = _i32(offs)
    c = cfg.c()
    _check(load().dbsa_encode_blocks(
        ctypes.byref(c), _dp(q), _dp(k), _dp(v), _hp(o), len(o) - 1, _dp(k_cache), _dp(v_cache),
        k_cache.shape[1], _dp(out), _dp(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def append_block(cfg: DbsaConfig, q, k, v, offs, k_cache, v_cache, out, workspace, stream=None):
    """Encode one new block after the blocks of `offs` (its length = q.shape[0])."""
    o = _i32(offs)
    c = cfg.c()
    _check(load().dbsa_append_block(
        ctypes.byref(c), _dp(q), _dp(k), _dp(v), q.shape[0], _hp(o), len(o) - 1, _dp(k_cache),
        _dp(v_cache), k_cache.shape[1], _dp(out), _dp(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def gather_rope_attend(cfg: DbsaConfig, k_cache, v_cache, offs, sel_ptr, sel_blocks, q_new,
                       k_tail, v_tail, tail_len: int, out, workspace, dbg_map=None, stream=None,
                       block_keys=None):
    """Stage 2 for a batch of queries (see dbsa_gather_rope_attend); with
    block_keys (from block_keys()), dbsa_gather_rope_attend_prepared."""
    o, sp, sb = _i32(offs), _i32(sel_ptr), _i32(sel_blocks)
    c = cfg.c()
    args = [ctypes.byref(c), _dp(k_cache), _dp(v_cache), k_cache.shape[1], _hp(o), len(o) - 1,
            len(sp) - 1, _hp(sp), _hp(sb), _dp(q_new), q_new.shape[1], _dp(k_tail), _dp(v_tail),
            tail_len, k_tail.shape[1], _dp(out), _dp(dbg_map),
            0 if dbg_map is None else dbg_map.shape[1]]
    ws = [_dp(workspace), workspace.numel() * workspace.element_size(), _stream(stream)]
    if block_keys is None:
        _check(load().dbsa_gather_rope_attend(*args, *ws))
    else:
        _check(load().dbsa_gather_rope_attend_prepared(
            *args, _dp(block_keys), block_keys.numel() * block_keys.element_size(), *ws))


def block_keys_size(cfg: DbsaConfig, offs) -> int:
    o = _i32(offs)
    c = cfg.c()
    return int(load().dbsa_block_keys_size(ctypes.byref(c), _hp(o), len(o) - 1))


def block_keys(cfg: DbsaConfig, k_cache, v_cache, offs, buf, stream=None):
    """Keys of every cache row rotated at their position inside their block,
    into buf (uint8 device tensor of block_keys_size() bytes)."""
    o = _i32(offs)
    c = cfg.c()
    _check(load().dbsa_block_keys(
        ctypes.byref(c), _dp(k_cache), _dp(v_cache), k_cache.shape[1], _hp(o), len(o) - 1,
        _dp(buf), buf.numel() * buf.element_size(), _stream(stream)))


def kernel_launches() -> int:
    return int(load().dbsa_kernel_launches())


def set_profile_events(start, stop):
    """Record torch.cuda.Event objects around the next call's main kernel."""
    def handle(ev):
        if ev is None:
            return None
        if not ev.cuda_event:   # torch creates the CUDA event on its first record()
            ev.record()
        return ev.cuda_event
    load().dbsa_set_profile_events(handle(start), handle(stop))


def gather_rope_attend_noalloc(cfg: DbsaConfig, k_cache, v_cache, offs, sel_ptr, sel_blocks,
                               q_new, k_tail, v_tail, tail_len: int, out, dbg_map=None,
                               stream=None):
    """Stage 2 without a workspace: for callers that cannot allocate device
    memory.  Scratch is the library's fixed 16 MiB per-device array, shared
    by every call (serialise calls that would overlap on the GPU)."""
    o, sp, sb = _i32(offs), _i32(sel_ptr), _i32(sel_blocks)
    c = cfg.c()
    _check(load().dbsa_gather_rope_attend_noalloc(
        ctypes.byref(c), _dp(k_cache), _dp(v_cache), k_cache.shape[1], _hp(o), len(o) - 1,
        len(sp) - 1, _hp(sp), _hp(sb), _dp(q_new), q_new.shape[1], _dp(k_tail), _dp(v_tail),
        tail_len, k_tail.shape[1], _dp(out), _dp(dbg_map),
        0 if dbg_map is None else dbg_map.shape[1], _stream(stream)))


def read_status(workspace, stream=None) -> int:
    return int(load().dbsa_read_status(_dp(workspace), _stream(stream)))


def noalloc_read_status(stream=None) -> int:
    return int(load().dbsa_noalloc_read_status(_stream(stream)))


def test_wait_expiry(limit_ns: int):
    """Test hook: the next call on this thread loads no tile, so its device
    waits run out after limit_ns nanoseconds (see dbsa_test_wait_expiry)."""
    load().dbsa_test_wait_expiry(int(limit_ns))


def host_allocation_calls() -> int:
    return int(load().dbsa_host_allocation_calls())


def selection_csr(selections) -> tuple[np.ndarray, np.ndarray]:
    """CSR (sel_ptr, sel_blocks) from a list of per-query block-id arrays."""
    ptr = np.zeros(len(selections) + 1, dtype=np.int32)
    ptr[1:] = np.cumsum([len(s) for s in selections])
    return ptr, (np.concatenate(selections).astype(np.int32) if selections else
                 np.zeros(0, np.int32))

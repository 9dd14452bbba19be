"""The no-allocation Stage-2 entry point against the workspace one (GPU).

dbsa_gather_rope_attend_noalloc serves callers that cannot allocate device
memory when they call in (a framework's fixed memory budget, a thread that
must not call cudaMalloc): it runs Stage 2 out of the library's own fixed
scratch array instead of a caller workspace.  Here it is called through the
C ABI twice in a row, on different batches, and each result must be
bit-identical to dbsa_gather_rope_attend's on the same inputs (the same plan
runs the same kernels); neither call may make an allocating call (the
library counts its page-locked allocations and event creations), and the
status word it leaves in its scratch must read DBSA_OK.
The file is named to be collected last, so that a run stopping at the first
failure has run every other test already; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from many_shot_icl_b200 import dbsa
from tests.gpu_helpers import offsets, rand

pytestmark = pytest.mark.gpu


def _inputs(seed):
    rng = np.random.default_rng(seed)
    offs = offsets(rng.integers(300, 900, size=10))
    sels = [np.array([0, 3, 7, 9]), np.array([0, 1, 2]), np.array([0, 8, 4, 6, 5])]
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    T, nq, tail_len, n_new = int(offs[-1]), len(sels), 12, 1
    ins = dict(
        kc=rand((2, T, 128), seed * 10 + 1, "bf16"), vc=rand((2, T, 128), seed * 10 + 2, "bf16"),
        qn=rand((nq, n_new, 8, 128), seed * 10 + 3, "bf16"),
        kt=rand((nq, tail_len, 2, 128), seed * 10 + 4, "bf16"),
        vt=rand((nq, tail_len, 2, 128), seed * 10 + 5, "bf16"))
    return cfg, offs, sels, tail_len, n_new, ins


def _reference(cfg, offs, sels, tail_len, n_new, ins):
    sp, sb = dbsa.selection_csr(sels)
    out = torch.empty((len(sels), n_new, 8, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dbsa.gather_workspace_size(cfg, offs, sp, sb, n_new, tail_len),
                     dtype=torch.uint8, device="cuda")
    dbsa.gather_rope_attend(cfg, ins["kc"], ins["vc"], offs, sp, sb, ins["qn"], ins["kt"],
                            ins["vt"], tail_len, out, ws)
    assert dbsa.read_status(ws) == dbsa.OK
    return out


def _noalloc_via_cabi(cfg, offs, sels, tail_len, n_new, ins):
    lib = dbsa.load()
    sp, sb = dbsa.selection_csr(sels)
    o = np.ascontiguousarray(offs, np.int32)
    out = torch.full((len(sels), n_new, 8, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    c = cfg.c()
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    st = lib.dbsa_gather_rope_attend_noalloc(
        ctypes.byref(c), ins["kc"].data_ptr(), ins["vc"].data_ptr(), ins["kc"].shape[1], vp(o),
        len(o) - 1, len(sels), vp(sp), vp(sb), ins["qn"].data_ptr(), n_new, ins["kt"].data_ptr(),
        ins["vt"].data_ptr(), tail_len, ins["kt"].shape[1], out.data_ptr(), None, 0,
        torch.cuda.current_stream().cuda_stream)
    assert st == dbsa.OK, dbsa.last_error()
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_workspace_entry_point_twice():
    case1 = _inputs(1)
    case2 = _inputs(2)          # a different batch: the second call reuses the scratch
    want1, want2 = _reference(*case1), _reference(*case2)
    torch.cuda.synchronize()
    allocs = dbsa.host_allocation_calls()
    got1 = _noalloc_via_cabi(*case1)
    assert dbsa.noalloc_read_status() == dbsa.OK
    got2 = _noalloc_via_cabi(*case2)
    assert dbsa.noalloc_read_status() == dbsa.OK
    assert dbsa.host_allocation_calls() == allocs, "the no-allocation call allocated"
    assert torch.isfinite(got1.float()).all() and torch.isfinite(got2.float()).all()
    assert torch.equal(got1, want1)
    assert torch.equal(got2, want2)


def test_noalloc_rejects_batches_beyond_its_scratch():
    cfg, offs, sels, tail_len, n_new, ins = _inputs(3)
    many = [np.arange(10)] * 64          # 64 queries x 40-token prompt: > 16 MiB of partials
    n_big = 40
    qn = rand((64, n_big, 8, 128), 7, "bf16")
    kt = rand((64, n_big, 2, 128), 8, "bf16")
    sp, sb = dbsa.selection_csr(many)
    assert dbsa.gather_workspace_size(cfg, offs, sp, sb, n_big, n_big) > (16 << 20)
    out = torch.empty((64, n_big, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dbsa.DbsaError) as ei:
        dbsa.gather_rope_attend_noalloc(cfg, ins["kc"], ins["vc"], offs, sp, sb, qn, kt, kt, n_big, out)
    assert ei.value.status == dbsa.ERR_WORKSPACE and "16777216" in str(ei.value)

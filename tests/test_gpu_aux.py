"""Failure detection and checkpoint/resume on a B200.

Bounded waits: every device wait of the tensor-core kernel gives up after a
limit (4 s by default) and reports DBSA_ERR_TIMEOUT through the status word,
after finishing its copies and tensor-core work in flight and releasing its
tensor memory.  dbsa_test_wait_expiry() makes the next call's kernel load no
tile, so its waits are for barriers that nothing completes, with a limit of
one millisecond; the test reads the status, then runs the same call normally
on the same stream and checks it against the oracle: the context is still
usable and the tensor memory was given back (a kernel that kept it would
leave the next one without columns).

Checkpoint/resume ([DBSA notes] §Stage 1, item 4: new blocks can be encoded
at any time): the cache is the caller's tensors, so saving them with
torch.save, reloading, and appending a block gives bits identical to the
append on the uninterrupted cache.
"""
import io

import numpy as np
import pytest
import torch

import oracle
from many_shot_icl_b200 import dbsa
from tests.gpu_helpers import Stage1Run, compare, host_f32, offsets, rand

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from many_shot_icl_b200 import build
    build.build()
    dbsa.load()
    assert torch.cuda.is_available()


def test_stage1_wait_expiry_then_next_call_is_correct():
    cfg = dbsa.DbsaConfig(4, 2, 128, "bf16", 5e5, 2)
    run = Stage1Run(cfg, offsets([300, 129, 128, 257, 400]), seed=21)
    dbsa.test_wait_expiry(1_000_000)
    dbsa.encode_blocks(cfg, run.q, run.k, run.v, run.offs, run.kc, run.vc, run.out, run.ws)
    assert dbsa.read_status(run.ws) == dbsa.ERR_TIMEOUT
    assert "expired" in dbsa.last_error()
    run.out.fill_(float("nan"))
    run.run()                                   # default limit again: status OK
    T, Hq = run.T, cfg.n_q_heads
    hh, tt = np.meshgrid(np.arange(Hq), np.arange(T))
    want = run.oracle_rows(hh.ravel(), tt.ravel()).reshape(T, Hq, -1)
    compare(host_f32(run.out), want, head_axis=1, what="after a timed-out call")


def test_stage2_wait_expiry_then_next_call_is_correct():
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    offs = offsets([400, 300, 350, 280, 500])
    sels = [np.array([0, 2, 4]), np.array([0, 1, 3])]
    Hkv, D, n_new, tail = 2, 128, 4, 6
    T = int(offs[-1])
    kc, vc = rand((Hkv, T, D), 31, "bf16"), rand((Hkv, T, D), 32, "bf16")
    qn = rand((2, n_new, 8, D), 33, "bf16")
    kt, vt = rand((2, tail, Hkv, D), 34, "bf16"), rand((2, tail, Hkv, D), 35, "bf16")
    sp, sb = dbsa.selection_csr(sels)
    ws = torch.empty(dbsa.gather_workspace_size(cfg, offs, sp, sb, n_new, tail),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((2, n_new, 8, D), dtype=torch.bfloat16, device="cuda")
    dbsa.test_wait_expiry(1_000_000)
    dbsa.gather_rope_attend(cfg, kc, vc, offs, sp, sb, qn, kt, vt, tail, out, ws)
    assert dbsa.read_status(ws) == dbsa.ERR_TIMEOUT
    out.fill_(float("nan"))
    dbsa.gather_rope_attend(cfg, kc, vc, offs, sp, sb, qn, kt, vt, tail, out, ws)
    assert dbsa.read_status(ws) == dbsa.OK
    for q in range(2):
        want = oracle.stage2_all(host_f32(kc), host_f32(vc), offs, sels[q], host_f32(qn[q]),
                                 host_f32(kt[q]), host_f32(vt[q]), cfg.rope_theta)
        compare(host_f32(out[q]), want, head_axis=1, what="stage 2 after a timed-out call q%d" % q)


def test_checkpoint_reload_append_bit_identical():
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    lens = [260, 300, 190, 410, 233]
    offs_all = offsets(lens)
    offs = offs_all[:-1]
    T0, L = int(offs[-1]), lens[-1]
    Hq, Hkv, D = 8, 2, 128
    q, k, v = (rand((T0 + L, Hq, D), 41, "bf16"), rand((T0 + L, Hkv, D), 42, "bf16"),
               rand((T0 + L, Hkv, D), 43, "bf16"))
    cap = T0 + L
    kc = torch.empty((Hkv, cap, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    out0 = torch.empty((T0, Hq, D), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(dbsa.encode_workspace_size(cfg, T0, len(offs) - 1), dtype=torch.uint8,
                     device="cuda")
    dbsa.encode_blocks(cfg, q[:T0], k[:T0], v[:T0], offs, kc, vc, out0, ws)
    assert dbsa.read_status(ws) == dbsa.OK
    # checkpoint: the cache and the offsets, through torch.save / torch.load
    buf = io.BytesIO()
    torch.save({"k_cache": kc[:, :T0].cpu(), "v_cache": vc[:, :T0].cpu(),
                "offs": torch.from_numpy(offs.copy())}, buf)
    buf.seek(0)
    ck = torch.load(buf)
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[:, :T0].copy_(ck["k_cache"])
    vc2[:, :T0].copy_(ck["v_cache"])
    offs2 = ck["offs"].numpy().astype(np.int32)
    wsa = torch.empty(dbsa.append_workspace_size(cfg, offs, L), dtype=torch.uint8, device="cuda")
    out_a = torch.empty((L, Hq, D), dtype=torch.bfloat16, device="cuda")
    out_b = torch.empty_like(out_a)
    dbsa.append_block(cfg, q[T0:], k[T0:], v[T0:], offs, kc, vc, out_a, wsa)       # uninterrupted
    dbsa.append_block(cfg, q[T0:], k[T0:], v[T0:], offs2, kc2, vc2, out_b, wsa)    # resumed
    assert dbsa.read_status(wsa) == dbsa.OK
    assert torch.equal(out_a, out_b)
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    # and the resumed block against the oracle on all blocks
    rows = np.arange(T0, T0 + L)
    heads = rows % Hq
    want = oracle.stage1_rows(host_f32(q), host_f32(k), host_f32(v), offs_all, 2, 5e5, heads, rows)
    got = out_b[torch.from_numpy(rows - T0).cuda(), torch.from_numpy(heads).cuda()]
    compare(host_f32(got)[:, None, :], want[:, None, :], head_axis=1, what="resumed append")

"""Stage-1 parity on a B200: dbsa_encode_blocks / dbsa_append_block against
the CPU oracle on the same seeded inputs (every output row at sizes that
span several 128-row and 128-key tiles with ragged tails)."""
import numpy as np
import pytest
import torch

import oracle
from many_shot_icl_b200 import dbsa, inputs
from tests.gpu_helpers import ATOL, ATOL_PEAKY, Stage1Run, compare, host_f32, offsets, rand

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from many_shot_icl_b200 import build
    build.build()
    dbsa.load()
    assert torch.cuda.is_available()


def full_check(run: Stage1Run, what: str, atol: float = ATOL):
    T, Hq = run.T, run.cfg.n_q_heads
    hh, tt = np.meshgrid(np.arange(Hq), np.arange(T))
    want = run.oracle_rows(hh.ravel(), tt.ravel()).reshape(T, Hq, -1)
    return compare(host_f32(run.out), want, head_axis=1, what=what, atol=atol)


def test_tiny_workload_fp32():
    w = inputs.TINY
    offs = oracle.group_blocks(inputs.demo_lengths(w), w.demos_per_block)
    cfg = dbsa.DbsaConfig(w.n_q_heads, w.n_kv_heads, w.head_dim, "f32", w.rope_theta, w.window_j)
    run = Stage1Run(cfg, offs, seed=1, cap_extra=5).run()
    full_check(run, "tiny fp32")
    # the cache holds the pre-RoPE inputs bit for bit
    assert torch.equal(run.kc[:, :run.T], run.k.permute(1, 0, 2))
    assert torch.equal(run.vc[:, :run.T], run.v.permute(1, 0, 2))


@pytest.mark.parametrize("Hq,Hkv,D,theta", [(4, 2, 128, 5e5), (8, 2, 128, 1e4), (2, 2, 64, 1e4),
                                            (64, 1, 64, 1e4)])
def test_multi_tile_bf16(Hq, Hkv, D, theta):
    lens = [300, 129, 128, 1, 257, 400, 77]
    cfg = dbsa.DbsaConfig(Hq, Hkv, D, "bf16", theta, 2)
    run = Stage1Run(cfg, offsets(lens), seed=2).run()
    full_check(run, "bf16 Hq=%d Hkv=%d D=%d" % (Hq, Hkv, D))
    assert torch.equal(run.kc, run.k.permute(1, 0, 2))


@pytest.mark.parametrize("pattern,j", [(dbsa.PATTERN_FULL, 0), (dbsa.PATTERN_SINK_SELF, 0),
                                       (dbsa.PATTERN_SELF, 0), (dbsa.PATTERN_SINK_PREV_SELF, 0),
                                       (dbsa.PATTERN_SINK_PREV_SELF, 1),
                                       (dbsa.PATTERN_SINK_PREV_SELF, 4)])
def test_patterns(pattern, j):
    lens = [200, 180, 260, 90, 310, 150]
    cfg = dbsa.DbsaConfig(4, 1, 128, "bf16", 1e4, j, pattern)
    run = Stage1Run(cfg, offsets(lens), seed=3).run()
    full_check(run, "pattern %d j %d" % (pattern, j))


def test_peaky_queries():
    # Q x 4: sharp softmax, so a wrong mask or position cannot hide in an average
    lens = [250, 300, 140, 333]
    cfg = dbsa.DbsaConfig(4, 2, 128, "bf16", 5e5, 2)
    run = Stage1Run(cfg, offsets(lens), seed=4, q_scale=4.0).run()
    full_check(run, "peaky", atol=ATOL_PEAKY)


def test_single_block_and_tiny_blocks():
    for lens in ([1], [5], [128], [1, 1, 1, 1], [3, 130, 2]):
        cfg = dbsa.DbsaConfig(2, 1, 64, "bf16", 1e4, 2)
        run = Stage1Run(cfg, offsets(lens), seed=5).run()
        full_check(run, "lens %s" % lens)


def test_deterministic_and_local():
    # identical inputs -> bit-identical outputs; perturbing K/V outside block
    # b's window (not the sink, index < b - j) leaves block b bit-identical
    lens = [150, 140, 170, 160, 155, 145]
    offs = offsets(lens)
    cfg = dbsa.DbsaConfig(4, 2, 128, "bf16", 1e4, 2)
    a = Stage1Run(cfg, offs, seed=6).run()
    out1 = a.out.clone()
    a.run()
    assert torch.equal(out1, a.out)
    b = 5
    k2, v2 = a.k.clone(), a.v.clone()
    k2[offs[1]:offs[b - 2]] += 3.0
    v2[offs[1]:offs[b - 2]] -= 2.0
    a.k, a.v = k2, v2
    a.run()
    assert torch.equal(out1[offs[b]:offs[b + 1]], a.out[offs[b]:offs[b + 1]])
    assert torch.equal(out1[:offs[1]], a.out[:offs[1]])


def test_append_matches_encode_and_oracle():
    lens = [220, 180, 260, 140, 199]
    offs_all = offsets(lens)
    L = lens[-1]
    for dtype, Hq, Hkv, D in (("bf16", 4, 2, 128), ("f32", 2, 1, 64)):
        cfg = dbsa.DbsaConfig(Hq, Hkv, D, dtype, 5e5, 2)
        full = Stage1Run(cfg, offs_all, seed=7, cap_extra=0).run()
        # encode the first nb blocks into a cache with room for one more
        head = Stage1Run(cfg, offs_all[:-1], seed=99, cap_extra=L)
        T0 = int(offs_all[-2])
        head.q, head.k, head.v = full.q[:T0].clone(), full.k[:T0].clone(), full.v[:T0].clone()
        head.run()
        qn, kn, vn = full.q[T0:].clone(), full.k[T0:].clone(), full.v[T0:].clone()
        out = torch.full((L, Hq, D), float("nan"), dtype=full.out.dtype, device="cuda")
        ws = torch.empty(dbsa.append_workspace_size(cfg, offs_all[:-1], L), dtype=torch.uint8,
                         device="cuda")
        dbsa.append_block(cfg, qn, kn, vn, offs_all[:-1], head.kc, head.vc, out, ws)
        assert dbsa.read_status(ws) == dbsa.OK
        # the cache after the append equals the cache of the full encode, bit for bit
        assert torch.equal(head.kc, full.kc) and torch.equal(head.vc, full.vc)
        # same tile schedule for the new block -> same bits as the full encode
        assert torch.equal(out, full.out[T0:]), dtype
        hh, tt = np.meshgrid(np.arange(Hq), np.arange(T0, T0 + L))
        want = full.oracle_rows(hh.ravel(), tt.ravel()).reshape(L, Hq, -1)
        compare(host_f32(out), want, head_axis=1, what="append " + dtype)

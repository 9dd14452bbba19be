"""Stage-2 parity on a B200: dbsa_gather_rope_attend against the CPU oracle
on the same seeded inputs.  Gathered cache rows and fresh positions are
compared exactly: dbg_map is written by the attention kernels themselves
(the block-by-block tensor-core kernel's epilogue from the tile it loaded and
the rotation the query rows got; the per-query kernel from its own segment
walk and rotation table indices).  Attention outputs within the stated
tolerance."""
import numpy as np
import pytest
import torch

import oracle
from many_shot_icl_b200 import dbsa, inputs
from tests.gpu_helpers import (ATOL, ATOL_PEAKY, check_gather_map, compare, host_f32, offsets,
                               rand, tdtype)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from many_shot_icl_b200 import build
    build.build()
    dbsa.load()
    assert torch.cuda.is_available()


class Stage2Run:
    def __init__(self, cfg, offs, sels, n_new, tail_len, seed=0, tail_cap=None, q_scale=1.0,
                 cap_extra=3):
        self.cfg, self.offs, self.sels = cfg, np.asarray(offs, np.int32), sels
        Hq, Hkv, D = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
        T = int(self.offs[-1])
        self.cap = T + cap_extra
        self.nq = len(sels)
        self.n_new, self.tail_len = n_new, tail_len
        self.tail_cap = tail_cap or tail_len + 2
        self.kc = rand((Hkv, self.cap, D), seed * 10 + 1, cfg.dtype)
        self.vc = rand((Hkv, self.cap, D), seed * 10 + 2, cfg.dtype)
        self.q_new = rand((self.nq, n_new, Hq, D), seed * 10 + 3, cfg.dtype, q_scale)
        self.kt = rand((self.nq, self.tail_cap, Hkv, D), seed * 10 + 4, cfg.dtype)
        self.vt = rand((self.nq, self.tail_cap, Hkv, D), seed * 10 + 5, cfg.dtype)
        self.sel_ptr, self.sel = dbsa.selection_csr(sels)
        self.out = torch.full((self.nq, n_new, Hq, D), float("nan"), dtype=tdtype(cfg.dtype),
                              device="cuda")
        Tmax = max(int(sum(self.offs[b + 1] - self.offs[b] for b in s)) for s in sels)
        self.dbg = torch.full((self.nq, Tmax, 2), -1, dtype=torch.int32, device="cuda")
        nbytes = dbsa.gather_workspace_size(cfg, self.offs, self.sel_ptr, self.sel, n_new, tail_len)
        assert nbytes > 0, dbsa.last_error()
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")

    def run(self):
        dbsa.gather_rope_attend(self.cfg, self.kc, self.vc, self.offs, self.sel_ptr, self.sel,
                                self.q_new, self.kt, self.vt, self.tail_len, self.out, self.ws,
                                dbg_map=self.dbg)
        assert dbsa.read_status(self.ws) == dbsa.OK
        return self

    def check(self, what, queries=None, atol=ATOL):
        kc, vc = host_f32(self.kc), host_f32(self.vc)
        qn, kt, vt = host_f32(self.q_new), host_f32(self.kt), host_f32(self.vt)
        out = host_f32(self.out)
        dbg = self.dbg.cpu().numpy()
        for q in (range(self.nq) if queries is None else queries):
            m = oracle.stage2_gather_map(self.offs, self.sels[q])
            check_gather_map(dbg[q], m, "%s q%d" % (what, q))
            want = oracle.stage2_all(kc, vc, self.offs, self.sels[q], qn[q],
                                     kt[q, :self.tail_len], vt[q, :self.tail_len],
                                     self.cfg.rope_theta, scale=self.cfg.softmax_scale)
            compare(out[q], want, head_axis=1, what="%s q%d" % (what, q), atol=atol)


def test_tiny_workload_fp32():
    w = inputs.TINY
    offs = oracle.group_blocks(inputs.demo_lengths(w), w.demos_per_block)
    sels = inputs.selections(w)
    cfg = dbsa.DbsaConfig(w.n_q_heads, w.n_kv_heads, w.head_dim, "f32", w.rope_theta, w.window_j)
    Stage2Run(cfg, offs, sels, n_new=w.query_tokens, tail_len=w.query_tokens, seed=1).run().check("tiny")


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (4, 4, 128), (4, 1, 64)])
@pytest.mark.parametrize("n_new,tail_len", [(1, 1), (1, 9), (3, 7), (40, 40), (17, 20)])
def test_bf16_prefill_and_decode(Hq, Hkv, D, n_new, tail_len):
    rng = np.random.default_rng(Hq * 100 + n_new)
    lens = rng.integers(40, 400, size=9)
    offs = offsets(lens)
    sels = [np.array([0, 2, 5, 7]), np.array([0, 8, 1]), np.array([0]), np.array([0, 3, 4, 6, 8, 1])]
    cfg = dbsa.DbsaConfig(Hq, Hkv, D, "bf16", 5e5, 2)
    Stage2Run(cfg, offs, sels, n_new, tail_len, seed=2).run().check(
        "Hq%d Hkv%d D%d n%d t%d" % (Hq, Hkv, D, n_new, tail_len))


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 128), (2, 1, 64)])
@pytest.mark.parametrize("n_new,tail_len", [(16, 16), (1, 9)])
def test_fp32_cache_block_major(Hq, Hkv, D, n_new, tail_len):
    """fp32 caches whose selected blocks average well over one 128-key tile:
    the block-by-block tensor-core path, which reads a bf16 copy of V made
    next to the block-relative keys."""
    rng = np.random.default_rng(Hq * 7 + n_new)
    offs = offsets(rng.integers(150, 420, size=8))
    sels = [np.array([0, 2, 5, 7]), np.array([0, 6, 1]), np.array([0]), np.array([0, 3, 4, 1, 7])]
    cfg = dbsa.DbsaConfig(Hq, Hkv, D, "f32", 5e5, 2)
    gath = [int(sum(offs[b + 1] - offs[b] for b in s_)) for s_ in sels]
    assert sum(gath) >= 128 * sum(len(s_) for s_ in sels)   # the block-major mode
    Stage2Run(cfg, offs, sels, n_new, tail_len, seed=11).run().check(
        "fp32 block-major Hq%d D%d n%d" % (Hq, D, n_new))


@pytest.mark.parametrize("n_new,tail_len", [(3, 5), (1, 4)])
def test_largest_head_ratio(n_new, tail_len):
    """64 query heads on one KV head, the largest ratio the ABI accepts: the
    packed rows of one (query, block) pair span two 128-row tiles."""
    offs = offsets([180, 260, 140, 300])
    sels = [np.array([0, 3, 1]), np.array([0, 2])]
    cfg = dbsa.DbsaConfig(64, 1, 64, "bf16", 1e4, 2)
    Stage2Run(cfg, offs, sels, n_new, tail_len, seed=12).run().check("Hq/Hkv=64 n%d" % n_new)


def test_long_gather_many_splits_peaky():
    # long selections force several splits per query; Q x 4 sharpens the softmax
    rng = np.random.default_rng(5)
    lens = rng.integers(900, 1600, size=12)
    offs = offsets(lens)
    sels = [np.concatenate([[0], np.sort(rng.choice(np.arange(1, 12), 8, replace=False))])
            for _ in range(3)]
    sels.append(np.concatenate([[0], rng.permutation(np.arange(1, 12))]))   # non-encoding order
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    for n_new, tail_len in ((1, 41), (40, 40)):
        Stage2Run(cfg, offs, sels, n_new, tail_len, seed=3, q_scale=4.0).run().check(
            "long n%d" % n_new, atol=ATOL_PEAKY)
        Stage2Run(cfg, offs, sels, n_new, tail_len, seed=13).run().check("long n%d" % n_new)


def test_staged_and_direct_items_share_q_slots():
    """A prompt pass whose blocks alternate between short ones (at most two
    128-key tiles: the kernel stores those items' rows directly and frees
    their Q slot at the last QK) and long ones (three or more tiles: rows
    staged in the Q tile, slot freed after the copies), with several items
    per CTA, so that each Q slot is reused by both kinds in turn; then a
    decode step on the same cache (a launch without staging)."""
    rng = np.random.default_rng(21)
    lens = [int(rng.integers(60, 250)) if b % 2 else int(rng.integers(390, 600))
            for b in range(16)]
    offs = offsets(lens)
    sels = [np.concatenate([[0], np.sort(rng.choice(np.arange(1, 16), 8, replace=False))])
            for _ in range(24)]
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    run = Stage2Run(cfg, offs, sels, 40, 40, seed=21).run()
    rows = 4 * 40 * np.bincount(np.concatenate(sels), minlength=16)
    items = 2 * int(np.sum((rows + 127) // 128))
    assert items > 3 * 148   # several items per CTA of the persistent kernel
    run.check("staged/direct prompt", queries=[0, 5, 11, 23])
    Stage2Run(cfg, offs, sels, 1, 41, seed=22).run().check("decode", queries=[0, 23])


def test_all_blocks_in_order_equals_stage1_positions():
    # selecting every block in encoding order reproduces the original positions
    lens = [100, 130, 90]
    offs = offsets(lens)
    cfg = dbsa.DbsaConfig(2, 1, 64, "bf16", 1e4, 2)
    r = Stage2Run(cfg, offs, [np.array([0, 1, 2])], 4, 4, seed=4).run()
    dbg = r.dbg.cpu().numpy()[0]
    np.testing.assert_array_equal(dbg[:, 0], np.arange(320))
    np.testing.assert_array_equal(dbg[:, 1], np.arange(320))
    r.check("all blocks")


def test_deterministic():
    lens = [300, 200, 250, 270]
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    r = Stage2Run(cfg, offsets(lens), [np.array([0, 2, 3])], 1, 5, seed=6).run()
    o1 = r.out.clone()
    r.run()
    assert torch.equal(o1, r.out)


def _run_both(cfg, offs, sels, n_new, tail_len, seed):
    """dbsa_gather_rope_attend and the prepared-keys path on the same inputs."""
    plain = Stage2Run(cfg, offs, sels, n_new, tail_len, seed=seed).run()
    bk = torch.empty(dbsa.block_keys_size(cfg, plain.offs), dtype=torch.uint8, device="cuda")
    dbsa.block_keys(cfg, plain.kc, plain.vc, plain.offs, bk)
    out = torch.full_like(plain.out, float("nan"))
    dbg = torch.full_like(plain.dbg, -1)
    dbsa.gather_rope_attend(cfg, plain.kc, plain.vc, plain.offs, plain.sel_ptr, plain.sel,
                            plain.q_new, plain.kt, plain.vt, tail_len, out, plain.ws,
                            dbg_map=dbg, block_keys=bk)
    assert dbsa.read_status(plain.ws) == dbsa.OK
    return plain, out, dbg, bk


@pytest.mark.parametrize("dtype,Hq,Hkv,D,n_new,tail_len", [("bf16", 8, 2, 128, 40, 40),
                                                          ("bf16", 8, 2, 128, 1, 41),
                                                          ("f32", 2, 1, 64, 16, 16)])
def test_prepared_block_keys_bit_identical(dtype, Hq, Hkv, D, n_new, tail_len):
    """One dbsa_block_keys() call, then the prepared path gives the plain path's
    bits (same kernels, same rotated keys) for prompt and decode passes, and
    the prepared buffer serves a second pass with other queries."""
    cfg = dbsa.DbsaConfig(Hq, Hkv, D, dtype, 5e5, 2)
    offs = offsets(np.random.default_rng(7).integers(20, 150, size=9))
    rng = np.random.default_rng(8)
    sels = [np.concatenate([[0], rng.permutation(np.arange(1, 9))[:k]]) for k in (3, 5, 1, 8)]
    plain, out, dbg, bk = _run_both(cfg, offs, sels, n_new, tail_len, seed=3)
    assert torch.equal(out, plain.out)
    assert torch.equal(dbg, plain.dbg)
    plain.check("prepared", queries=[0, 3])
    # the same block keys, another batch over the same cache
    other = [np.array([0, 8, 2]), np.array([0, 1])]
    run2 = Stage2Run(cfg, offs, other, n_new, tail_len, seed=3)
    run2.kc, run2.vc = plain.kc, plain.vc
    run2.run()
    out2 = torch.full_like(run2.out, float("nan"))
    dbsa.gather_rope_attend(cfg, run2.kc, run2.vc, run2.offs, run2.sel_ptr, run2.sel, run2.q_new,
                            run2.kt, run2.vt, tail_len, out2, run2.ws, block_keys=bk)
    assert torch.equal(out2, run2.out)


@pytest.mark.parametrize("n_new,tail_len", [(16, 16), (1, 9)])
def test_demonstration_granular_gather(n_new, tail_len):
    """Example-level selection ([DBSA notes] §Ablations, selection granularity):
    the offsets table makes every demonstration after the sink block its own
    block, and each query selects the sink and single demonstrations.  These
    few queries share little, so the keys are not shared across queries:
    with 64 query rows per (query, KV head) (16 tokens x 4 heads) each query's
    gathered keys are rotated into a compact buffer and attended on the
    tensor core; a single-token pass takes the per-query split kernel (its
    workspace holds no rotated keys).  Checked against the oracle, gather
    maps exact."""
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    rng = np.random.default_rng(21)
    lens = np.concatenate([[200], rng.integers(8, 31, size=60)])
    offs = offsets(lens)
    nb = len(lens)
    sels = [np.concatenate([[0], rng.permutation(np.arange(1, nb))[:k]]) for k in (18, 3, 40, 1)]
    run = Stage2Run(cfg, offs, sels, n_new, tail_len, seed=5)
    T = int(offs[-1])
    gathered = sum(int(sum(offs[b + 1] - offs[b] for b in s_)) for s_ in sels)
    if n_new == 1:
        assert run.ws.numel() < cfg.n_kv_heads * T * cfg.head_dim * 2
    else:       # the compact buffers: rotated keys and values of every gathered token
        assert run.ws.numel() >= 2 * cfg.n_kv_heads * gathered * cfg.head_dim * 2
    run.run().check("demo-granular")
    peaky = Stage2Run(cfg, offs, sels[:2], n_new, tail_len, seed=6, q_scale=4.0).run()
    peaky.check("demo-granular peaky", atol=ATOL_PEAKY)


def test_demonstration_granular_decode_shares_blocks():
    """Decode steps over a demonstration-granular selection (one block per
    demonstration, many queries selecting overlapping sets): the planner
    prices the per-(query, demonstration) partials and packed query rows
    below streaming every query's own keys, so the pass runs block-major on
    the tensor core, each demonstration's keys read once for all queries.
    Every query is checked against the oracle, gather maps exact."""
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 5e5, 2)
    rng = np.random.default_rng(33)
    lens = np.concatenate([[200], rng.integers(12, 31, size=200)])
    offs = offsets(lens)
    nb, T = len(lens), int(offs[-1])
    sels = [np.concatenate([[0], np.sort(rng.permutation(np.arange(1, nb))[:60])])
            for _ in range(32)]
    run = Stage2Run(cfg, offs, sels, 1, 9, seed=34)
    assert run.ws.numel() >= cfg.n_kv_heads * T * cfg.head_dim * 2   # the block-major layout
    run.run().check("demo-granular decode")
    peaky = Stage2Run(cfg, offs, sels[:8], 1, 9, seed=35, q_scale=4.0).run()
    peaky.check("demo-granular decode peaky", atol=ATOL_PEAKY)


def test_plan_staging_reuse_and_threads():
    """A call's host-built plan reaches the device through a per-thread ring of
    eight page-locked staging slots; a slot is refilled only after the read
    behind its previous use has completed, and a thread keeps its last plan
    for calls with the same inputs.  Calls that wrap the ring several times
    with plans of different sizes, repeated calls that reuse the kept plan,
    and two threads calling at once on their own streams give the same bits
    as the first run of each call."""
    import threading
    cfg = dbsa.DbsaConfig(8, 2, 128, "bf16", 1e4, 2)
    rng = np.random.default_rng(77)
    lens = rng.integers(40, 400, size=9)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    shapes = [([0, 3, 5], 1, 9), ([0, 1, 2, 7, 8], 40, 40), ([0, 6], 3, 7), ([0, 2, 4, 8], 1, 1)]

    def make(seed0):
        return [Stage2Run(cfg, offs, [np.array(s), np.array(s[:2])], n_new, tail, seed=seed0 + i)
                for i, (s, n_new, tail) in enumerate(shapes)]

    runs = make(30)
    first = [r.run().out.clone() for r in runs]
    for _ in range(3):                      # 24 more calls: the ring wraps
        for r, want in zip(runs, first):
            # a new plan, then the same plan again (the thread's plan cache)
            assert torch.equal(r.run().out, want)
            assert torch.equal(r.run().out, want)
    per_thread = [make(30), make(30)]
    torch.cuda.synchronize()                # inputs are made on the default stream
    errors = []

    def worker(rs):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(3):
                    for r in rs:
                        r.run()
            s.synchronize()
        except Exception as e:              # reported below, in the test's thread
            errors.append(e)

    th = [threading.Thread(target=worker, args=(rs,)) for rs in per_thread]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    for rs in per_thread:
        for r, want in zip(rs, first):
            assert torch.equal(r.out, want)

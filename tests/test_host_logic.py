"""Host-side logic of libdbsa.so, CPU only (no kernel runs here).

- the library loads and exports every function include/dbsa.h declares;
- the block table equals the oracle's;
- the Stage-1 tile list covers exactly the oracle's allowed (row, key) pairs,
  once each, for every pattern of the sparse-pattern ablation;
- invalid arguments are rejected with the documented status before any
  device work.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from many_shot_icl_b200 import dbsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from many_shot_icl_b200 import build
    build.build()
    return dbsa.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "dbsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dbsa_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(dbsa.SYMBOLS)
    assert "sm_100a" in dbsa.version()


def test_group_blocks_matches_oracle(lib):
    rng = np.random.default_rng(0)
    for n, k in ((1, 1), (7, 3), (1000, 50), (173, 50), (50, 50)):
        lens = rng.integers(15, 46, size=n).astype(np.int32)
        np.testing.assert_array_equal(dbsa.group_blocks(lens, k), oracle.group_blocks(lens, k))
    with pytest.raises(dbsa.DbsaError):
        dbsa.group_blocks(np.array([3, 0, 4], np.int32), 2)


def covered_pairs(items, head):
    pairs = set()
    for it in items:
        if it.head != head:
            continue
        assert 1 <= it.n_rows <= 128 and it.n_ranges in (1, 2)
        for t in range(it.q_pos0, it.q_pos0 + it.n_rows):
            for r in range(it.n_ranges):
                for s in range(it.pos0[r], it.pos0[r] + it.len[r]):
                    if s <= t:
                        assert (t, s) not in pairs, "pair covered twice"
                        pairs.add((t, s))
    return pairs


@pytest.mark.parametrize("pattern", range(4))
@pytest.mark.parametrize("j", [0, 1, 2, 5])
def test_stage1_plan_covers_exactly_the_mask(lib, pattern, j):
    rng = np.random.default_rng(10 + j)
    lens = rng.integers(1, 300, size=7)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(offs[-1])
    cfg = dbsa.DbsaConfig(4, 2, 64, window_j=j, pattern=pattern)
    items = dbsa.stage1_plan(cfg, offs)
    # rows: every token of every head exactly once, tiles never straddle a block
    for h in range(4):
        rows = sorted(t for it in items if it.head == h
                      for t in range(it.q_pos0, it.q_pos0 + it.n_rows))
        assert rows == list(range(T))
    for it in items:
        b = int(np.searchsorted(offs, it.q_pos0, side="right") - 1)
        assert it.block == b and it.q_pos0 + it.n_rows <= offs[b + 1]
        assert it.q_row0 == it.q_pos0 and list(it.k_row0)[:it.n_ranges] == list(it.pos0)[:it.n_ranges]
    # pairs: exactly the oracle's explicit mask (sampled rows, all keys)
    got = covered_pairs(items, head=1)
    sample = sorted(set(rng.integers(0, T, size=40).tolist()) | {0, T - 1} |
                    set(int(o) for o in offs[:-1]))
    for t in sample:
        want = {s for s in range(t + 1) if oracle.stage1_allowed(offs, j, t, s, pattern)}
        have = {s for (tt, s) in got if tt == t}
        assert have == want, (t, sorted(want ^ have)[:10])
    # the tile count is the sum of the items' key tiles
    assert dbsa.stage1_tile_count(cfg, offs) == sum(
        sum((it.len[r] + 127) // 128 for r in range(it.n_ranges)) for it in items)


def test_stage1_plan_allowed_count_matches_oracle(lib):
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 200, size=9)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cfg = dbsa.DbsaConfig(2, 1, 64, window_j=2)
    pairs = covered_pairs(dbsa.stage1_plan(cfg, offs), head=0)
    cnt = np.zeros(int(offs[-1]), np.int64)
    for t, _ in pairs:
        cnt[t] += 1
    np.testing.assert_array_equal(cnt, oracle.stage1_allowed_counts(offs, 2))


def _cfgp(cfg):
    c = cfg.c()
    return c, ctypes.byref(c)


def test_invalid_arguments_are_rejected_before_device_work(lib):
    fake = ctypes.c_void_p(4096)  # aligned, never dereferenced: validation fails first
    offs = np.array([0, 5, 9, 20], np.int32)
    ok_cfg = dbsa.DbsaConfig(4, 2, 128)
    ws = ctypes.c_void_p(1 << 20)

    def gather(cfg, sel_ptr, sel, n_new=1, tail_len=1, tail_cap=4, offs=offs, cap=64):
        c, cp = _cfgp(cfg)
        sp, sb = np.asarray(sel_ptr, np.int32), np.asarray(sel, np.int32)
        return lib.dbsa_gather_rope_attend(
            cp, fake, fake, cap, offs.ctypes.data_as(ctypes.c_void_p), len(offs) - 1, len(sp) - 1,
            sp.ctypes.data_as(ctypes.c_void_p), sb.ctypes.data_as(ctypes.c_void_p), fake, n_new,
            fake, fake, tail_len, tail_cap, fake, None, 0, ws, 1 << 30, None)

    assert gather(ok_cfg, [0, 2], [1, 0]) == dbsa.ERR_INVALID_ARG       # sink not first
    assert "sink" in dbsa.last_error()
    assert gather(ok_cfg, [0, 3], [0, 2, 2]) == dbsa.ERR_INVALID_ARG    # duplicate
    assert gather(ok_cfg, [0, 2], [0, 3]) == dbsa.ERR_INVALID_ARG       # out of range
    assert gather(ok_cfg, [0, 0], []) == dbsa.ERR_INVALID_ARG           # empty selection
    assert gather(ok_cfg, [0, 2, 1], [0, 1]) == dbsa.ERR_INVALID_ARG    # sel_ptr decreases
    # more blocks than exist: rejected before sel (one entry here) is read past its end
    assert gather(ok_cfg, [0, 1 << 30], [0]) == dbsa.ERR_INVALID_ARG
    assert "blocks of 3" in dbsa.last_error()
    assert gather(ok_cfg, [0, 1], [0], n_new=3, tail_len=2) == dbsa.ERR_INVALID_ARG
    assert gather(ok_cfg, [0, 1], [0], tail_len=5, tail_cap=4) == dbsa.ERR_INVALID_ARG
    assert gather(ok_cfg, [0, 1], [0], cap=10) == dbsa.ERR_CAPACITY
    assert gather(dbsa.DbsaConfig(4, 3, 128), [0, 1], [0]) == dbsa.ERR_UNSUPPORTED
    assert gather(dbsa.DbsaConfig(4, 2, 96), [0, 1], [0]) == dbsa.ERR_UNSUPPORTED
    bad_offs = np.array([0, 5, 5, 20], np.int32)
    assert gather(ok_cfg, [0, 1], [0], offs=bad_offs) == dbsa.ERR_INVALID_ARG

    def encode(cfg, offs=offs, cap=64, ws_bytes=1 << 30, q=fake, ws=ws):
        c, cp = _cfgp(cfg)
        return lib.dbsa_encode_blocks(cp, q, fake, fake, offs.ctypes.data_as(ctypes.c_void_p),
                                      len(offs) - 1, fake, fake, cap, fake, ws, ws_bytes, None)

    assert encode(ok_cfg, cap=19) == dbsa.ERR_CAPACITY
    assert encode(ok_cfg, offs=np.array([1, 5], np.int32)) == dbsa.ERR_INVALID_ARG
    assert encode(ok_cfg, q=ctypes.c_void_p(4097)) == dbsa.ERR_INVALID_ARG   # misaligned
    assert encode(ok_cfg, q=None) == dbsa.ERR_INVALID_ARG
    assert encode(ok_cfg, ws_bytes=100) == dbsa.ERR_WORKSPACE
    assert encode(ok_cfg, ws=ctypes.c_void_p(4096 + 16)) == dbsa.ERR_WORKSPACE
    assert encode(dbsa.DbsaConfig(4, 2, 128, rope_theta=0.5)) == dbsa.ERR_INVALID_ARG
    assert encode(dbsa.DbsaConfig(4, 2, 128, window_j=-1)) == dbsa.ERR_INVALID_ARG
    assert encode(dbsa.DbsaConfig(4, 2, 128, pattern=7)) == dbsa.ERR_INVALID_ARG

    def prepared(bk, bk_bytes, cfg=ok_cfg):
        c, cp = _cfgp(cfg)
        sp, sb = np.array([0, 1], np.int32), np.array([0], np.int32)
        return lib.dbsa_gather_rope_attend_prepared(
            cp, fake, fake, 64, offs.ctypes.data_as(ctypes.c_void_p), len(offs) - 1, 1,
            sp.ctypes.data_as(ctypes.c_void_p), sb.ctypes.data_as(ctypes.c_void_p), fake, 1,
            fake, fake, 1, 4, fake, None, 0, bk, bk_bytes, ws, 1 << 30, None)

    need = dbsa.block_keys_size(ok_cfg, offs)
    assert prepared(None, need) == dbsa.ERR_INVALID_ARG                  # no block keys
    assert prepared(ctypes.c_void_p(4096 + 16), need) == dbsa.ERR_WORKSPACE   # misaligned
    assert prepared(ctypes.c_void_p(4096), need - 1) == dbsa.ERR_WORKSPACE    # too small
    assert "block_keys" in dbsa.last_error()

    def block_keys(cap=64, bk=ctypes.c_void_p(1 << 20), bk_bytes=1 << 30, k=fake):
        c, cp = _cfgp(ok_cfg)
        return lib.dbsa_block_keys(cp, k, fake, cap, offs.ctypes.data_as(ctypes.c_void_p),
                                   len(offs) - 1, bk, bk_bytes, None)

    assert block_keys(cap=19) == dbsa.ERR_CAPACITY
    assert block_keys(k=None) == dbsa.ERR_INVALID_ARG
    assert block_keys(bk_bytes=need - 1) == dbsa.ERR_WORKSPACE

    c, cp = _cfgp(ok_cfg)
    assert lib.dbsa_append_block(cp, fake, fake, fake, 0, offs.ctypes.data_as(ctypes.c_void_p),
                                 3, fake, fake, 64, fake, ws, 1 << 30, None) == dbsa.ERR_INVALID_ARG
    assert lib.dbsa_append_block(cp, fake, fake, fake, 50, offs.ctypes.data_as(ctypes.c_void_p),
                                 3, fake, fake, 64, fake, ws, 1 << 30, None) == dbsa.ERR_CAPACITY


def test_workspace_sizes(lib):
    cfg = dbsa.DbsaConfig(32, 8, 128, rope_theta=5e5)
    offs = np.arange(0, 61 * 1500, 1500, dtype=np.int32)
    T = int(offs[-1])
    ws = dbsa.encode_workspace_size(cfg, T, 60)
    # k_rot dominates: 8 KV heads x T x 128 x 2 bytes (the queries are rotated
    # by the tensor-core kernel as it reads them: no rotated copy)
    assert 8 * T * 256 <= ws < 8 * T * 256 * 1.05
    wa = dbsa.append_workspace_size(cfg, offs, 1500)
    assert 0 < wa < ws / 10
    sel_ptr, sel = dbsa.selection_csr([np.array([0, 3, 9]), np.array([0, 1])])
    wg = dbsa.gather_workspace_size(cfg, offs, sel_ptr, sel, 40, 40)
    assert wg > 0
    # a block-major pass over 1 500-token blocks (~12 key tiles per item): the
    # tensor-core kernel rotates the packed query rows itself, so the workspace
    # holds K at block-relative positions [Hkv][T][D] and the partials of the
    # 5 (query, block) items + 2 tail items, plus small tables, and no packed
    # query rows (they would add 8 x 5 x 160 rows x 256 B = 1.6 MB)
    k_hat = 8 * T * 256
    partials = 7 * 32 * 40 * (128 * 2 + 8)
    assert k_hat + partials <= wg < k_hat + partials + (1 << 20)
    assert dbsa.gather_workspace_size(cfg, offs, sel_ptr, np.array([2, 3, 9, 0, 1]), 40, 40) == 0
    # a demonstration-granular selection (blocks of ~30 tokens) of one query
    # shares nothing across queries, so it goes per query.  A single-token
    # pass runs on the per-query kernel: its workspace holds no rotated keys.
    # A 40-token pass (160 query rows per KV head) runs in compact mode: the
    # query's gathered keys, rotated, and its values, bf16 [Hkv][T'][D] each
    lens = np.concatenate([[1500], np.full(100, 30)])
    doffs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    dsp, dsel = dbsa.selection_csr([np.arange(0, 101, 3)])
    gathered = 1500 + 30 * (len(dsel) - 1)
    wd1 = dbsa.gather_workspace_size(cfg, doffs, dsp, dsel, 1, 41)
    assert 0 < wd1 < 8 * int(doffs[-1]) * 256
    wd = dbsa.gather_workspace_size(cfg, doffs, dsp, dsel, 40, 40)
    compact = 2 * 8 * gathered * 128 * 2
    assert compact <= wd < compact + (8 << 20)
    # a decode step over 30-token demonstrations, shared by 64 queries, runs
    # block-major with items of one key tile: its packed query rows are written
    # before the tensor-core pass (bf16 [Hkv][pairs x g][D]), on top of the keys
    # and the partials
    rng = np.random.default_rng(5)
    dl = np.concatenate([[1500], np.full(2950, 30)])
    do = np.concatenate([[0], np.cumsum(dl)]).astype(np.int32)
    sels = [np.concatenate([[0], np.sort(rng.permutation(np.arange(1, len(dl)))[:885])])
            for _ in range(64)]
    dp, db = dbsa.selection_csr(sels)
    pairs = sum(len(x) for x in sels)
    need = 8 * int(do[-1]) * 256 + (pairs + 64) * 32 * (128 * 2 + 8) + 8 * pairs * 4 * 256
    assert need <= dbsa.gather_workspace_size(cfg, do, dp, db, 1, 41) < need + (16 << 20)
    # prepared block keys: K at block-relative positions, bf16 [Hkv][T][D], plus
    # RoPE tables (cos and sin, D/2 floats a row) for positions below T + 8192:
    # (T + 8192) / 16 coarse rows and 16 fine rows
    bk = dbsa.block_keys_size(cfg, offs)
    tables = ((T + 8192) // 16 + 1 + 16) * 64 * 2 * 4
    assert 8 * T * 256 + tables <= bk < 8 * T * 256 + tables + (1 << 20)
    assert dbsa.block_keys_size(dbsa.DbsaConfig(2, 1, 64, "f32"), offs) >= 2 * T * 128


def test_softmax_polynomial_exp2_error_bound():
    """The Stage-1 softmax evaluates part of P = 2^x with a cubic on the FMA
    pipe.  Emulate its float32 steps (clamp at -125, round by adding and
    subtracting 1.5 * 2^23, cubic in f = x - n, n added to the exponent field)
    with the coefficients parsed from the kernel source, and check the result
    against 2^x in fp64: relative error far below the bf16 half-ulp (2^-9) of
    the P it feeds, positive and finite everywhere, masked scores tiny."""
    src = open(os.path.join(ROOT, "many_shot_icl_b200", "csrc", "stage1_attn.cu")).read()
    c = [np.float32(float(re.search(r"kExp2C%d = ([0-9.e+-]+)f" % i, src).group(1)))
         for i in range(4)]
    x = np.concatenate([np.linspace(-140, 9, 1_000_001, dtype=np.float32),
                        np.float32([-np.inf, 0.0, -0.5, 0.5, 8.0, -125.0, -124.5])])
    magic = np.float32(12582912.0)
    xc = np.maximum(x, np.float32(-125.0))
    j = (xc + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (xc - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    q = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    r = (q.view(np.uint32) + (j.view(np.uint32) << np.uint32(23))).view(np.float32)
    assert np.all(np.isfinite(r)) and np.all(r > 0)
    live = x >= -125
    rel = np.abs(r[live].astype(np.float64) / np.exp2(x[live].astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4 < 2.0 ** -9
    assert np.all(r[~live] < 1e-37)

"""Parity at the workloads' full sizes, in the configuration the bench times.

One full layer of each workload runs through the C ABI exactly as bench.py
calls it; the oracle recomputes a sample of output rows one by one: the
first and last row of every block, the rows on each side of every 128-row
tile edge, and seeded random rows (Stage 1); every row of the batch's first
and last query and the exact gather maps of every query (Stage 2).  Inputs are the seeded
N(0, 1) tensors of many_shot_icl_b200.inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from many_shot_icl_b200 import dbsa, inputs
from tests.gpu_helpers import ATOL, ATOL_PEAKY, check_gather_map, compare, host_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from many_shot_icl_b200 import build
    build.build()
    dbsa.load()
    assert torch.cuda.is_available()


def workload_offsets(w):
    return oracle.group_blocks(inputs.demo_lengths(w), w.demos_per_block)


def cfg_of(w, j=None):
    return dbsa.DbsaConfig(w.n_q_heads, w.n_kv_heads, w.head_dim, w.dtype, w.rope_theta,
                           w.window_j if j is None else j)


def sample_rows(offs, Hq, n_random, seed):
    rng = np.random.default_rng(seed)
    toks = set()
    for b in range(len(offs) - 1):
        a, e = int(offs[b]), int(offs[b + 1])
        toks.update((a, e - 1))
        for m in range(a + 128, e, 128):          # q-tile edges inside the block
            toks.update((m - 1, m))
    toks.update(rng.integers(0, int(offs[-1]), n_random).tolist())
    toks = np.array(sorted(toks))
    heads = rng.integers(0, Hq, len(toks))
    return heads, toks


def run_stage1(w, j=None, layer=0):
    cfg = cfg_of(w, j)
    offs = workload_offsets(w)
    T, Hq, Hkv, D = int(offs[-1]), w.n_q_heads, w.n_kv_heads, w.head_dim
    q = inputs.randn((T, Hq, D), inputs.tensor_seed(w, layer, 0), w.dtype, "cuda")
    k = inputs.randn((T, Hkv, D), inputs.tensor_seed(w, layer, 1), w.dtype, "cuda")
    v = inputs.randn((T, Hkv, D), inputs.tensor_seed(w, layer, 2), w.dtype, "cuda")
    kc = torch.empty((Hkv, T, D), dtype=q.dtype, device="cuda")
    vc = torch.empty_like(kc)
    out = torch.full((T, Hq, D), float("nan"), dtype=q.dtype, device="cuda")
    ws = torch.empty(dbsa.encode_workspace_size(cfg, T, len(offs) - 1), dtype=torch.uint8,
                     device="cuda")
    dbsa.encode_blocks(cfg, q, k, v, offs, kc, vc, out, ws)
    assert dbsa.read_status(ws) == dbsa.OK
    return cfg, offs, q, k, v, kc, vc, out


@pytest.mark.parametrize("name,j", [("llama2-7b-30k", None), ("llama3.1-8b-90k", None),
                                    ("llama3.1-8b-128k", 2), ("llama3.1-8b-128k", 4)])
def test_stage1_full_layer_sampled(name, j):
    w = inputs.WORKLOADS[name]
    cfg, offs, q, k, v, kc, vc, out = run_stage1(w, j)
    assert torch.equal(kc, k.permute(1, 0, 2)) and torch.equal(vc, v.permute(1, 0, 2))
    heads, toks = sample_rows(offs, w.n_q_heads, 64, seed=len(offs))
    want = oracle.stage1_rows(host_f32(q), host_f32(k), host_f32(v), offs, cfg.window_j,
                              w.rope_theta, heads, toks)
    got = out[torch.from_numpy(toks).cuda(), torch.from_numpy(heads).cuda()]
    compare(host_f32(got)[:, None, :], want[:, None, :], head_axis=1, what=name)


def test_append_at_full_size():
    # C4: a 90k pool of 60 blocks, then one more 50-demo block; the new
    # block's rows are compared with the oracle on 61 blocks.
    w = inputs.L31_8B_APPEND
    lens = inputs.demo_lengths(w, n_blocks=w.n_blocks + 1)
    offs_all = oracle.group_blocks(lens, w.demos_per_block)
    T0, T = int(offs_all[-2]), int(offs_all[-1])
    L = T - T0
    cfg = cfg_of(w)
    Hq, Hkv, D = w.n_q_heads, w.n_kv_heads, w.head_dim
    q = inputs.randn((T, Hq, D), inputs.tensor_seed(w, 0, 0), w.dtype, "cuda")
    k = inputs.randn((T, Hkv, D), inputs.tensor_seed(w, 0, 1), w.dtype, "cuda")
    v = inputs.randn((T, Hkv, D), inputs.tensor_seed(w, 0, 2), w.dtype, "cuda")
    kc = torch.empty((Hkv, T, D), dtype=q.dtype, device="cuda")
    vc = torch.empty_like(kc)
    out0 = torch.empty((T0, Hq, D), dtype=q.dtype, device="cuda")
    ws = torch.empty(dbsa.encode_workspace_size(cfg, T0, w.n_blocks), dtype=torch.uint8,
                     device="cuda")
    dbsa.encode_blocks(cfg, q[:T0], k[:T0], v[:T0], offs_all[:-1], kc, vc, out0, ws)
    out = torch.full((L, Hq, D), float("nan"), dtype=q.dtype, device="cuda")
    wsa = torch.empty(dbsa.append_workspace_size(cfg, offs_all[:-1], L), dtype=torch.uint8,
                      device="cuda")
    dbsa.append_block(cfg, q[T0:], k[T0:], v[T0:], offs_all[:-1], kc, vc, out, wsa)
    assert dbsa.read_status(wsa) == dbsa.OK
    assert torch.equal(kc, k.permute(1, 0, 2)) and torch.equal(vc, v.permute(1, 0, 2))
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([[T0, T0 + 127, T0 + 128, T - 1], rng.integers(T0, T, 40)]))
    heads = rng.integers(0, Hq, len(toks))
    want = oracle.stage1_rows(host_f32(q), host_f32(k), host_f32(v), offs_all, w.window_j,
                              w.rope_theta, heads, toks)
    got = out[torch.from_numpy(toks - T0).cuda(), torch.from_numpy(heads).cuda()]
    compare(host_f32(got)[:, None, :], want[:, None, :], head_axis=1, what="append")


def run_stage2(w, cfg, kc, vc, offs, sels, n_new, tail_len, seed, q_scale=1.0):
    nq = len(sels)
    Hq, Hkv, D = w.n_q_heads, w.n_kv_heads, w.head_dim
    tail_cap = tail_len
    qn = inputs.randn((nq, n_new, Hq, D), seed, w.dtype, "cuda", scale=q_scale)
    kt = inputs.randn((nq, tail_cap, Hkv, D), seed + 1, w.dtype, "cuda")
    vt = inputs.randn((nq, tail_cap, Hkv, D), seed + 2, w.dtype, "cuda")
    sp, sb = dbsa.selection_csr(sels)
    out = torch.full((nq, n_new, Hq, D), float("nan"), dtype=kc.dtype, device="cuda")
    Tmax = max(int(sum(offs[b + 1] - offs[b] for b in s)) for s in sels)
    dbg = torch.full((nq, Tmax, 2), -1, dtype=torch.int32, device="cuda")
    ws = torch.empty(dbsa.gather_workspace_size(cfg, offs, sp, sb, n_new, tail_len),
                     dtype=torch.uint8, device="cuda")
    dbsa.gather_rope_attend(cfg, kc, vc, offs, sp, sb, qn, kt, vt, tail_len, out, ws, dbg_map=dbg)
    assert dbsa.read_status(ws) == dbsa.OK
    return qn, kt, vt, out, dbg


@pytest.mark.parametrize("name,order,n_new,tail_len,q_scale", [
    ("llama2-7b-30k", "encoding", 32, 32, 1.0),
    ("llama3.1-8b-90k", "encoding", 40, 40, 1.0),     # prompt pass
    ("llama3.1-8b-90k", "encoding", 1, 45, 1.0),      # a decode step
    ("llama3.1-8b-90k", "encoding", 40, 40, 4.0),     # peaky: Q x 4, sharp softmax
    ("llama3.1-8b-90k", "encoding", 1, 45, 4.0),
    ("llama3.1-8b-128k", "encoding", 32, 32, 1.0),
    ("llama3.1-8b-128k", "ascending", 32, 32, 1.0),
])
def test_stage2_full_batch_sampled(name, order, n_new, tail_len, q_scale):
    w = inputs.WORKLOADS[name]
    cfg, offs, q, k, v, kc, vc, _ = run_stage1(w)
    del q, k, v
    sels = inputs.selections(w, order=order)
    qn, kt, vt, out, dbg = run_stage2(w, cfg, kc, vc, offs, sels, n_new, tail_len,
                                      seed=inputs.tensor_seed(w, 0, 3, n_new), q_scale=q_scale)
    dbg = dbg.cpu().numpy()
    tag = "%s %s n%d%s" % (name, order, n_new, " peaky" if q_scale != 1.0 else "")
    for qi, s in enumerate(sels):                     # exact gather maps, every query
        check_gather_map(dbg[qi], oracle.stage2_gather_map(offs, s), "%s q%d" % (tag, qi))
    kch, vch = host_f32(kc), host_f32(vc)
    for qi in sorted({0, len(sels) - 1}):
        want = oracle.stage2_all(kch, vch, offs, sels[qi], host_f32(qn[qi]),
                                 host_f32(kt[qi, :tail_len]), host_f32(vt[qi, :tail_len]),
                                 w.rope_theta)
        compare(host_f32(out[qi]), want, head_axis=1, what="%s q%d" % (tag, qi),
                atol=ATOL if q_scale == 1.0 else ATOL_PEAKY)


def demo_granular(w, offs, seed):
    """The same context as one block per demonstration after the sink block,
    and per query the sink plus a seeded 30 % of the demonstrations."""
    lens = inputs.demo_lengths(w)
    k = w.demos_per_block
    d_offs = np.concatenate([[0, offs[1]], offs[1] + np.cumsum(lens[k:])]).astype(np.int32)
    assert d_offs[-1] == offs[-1]
    n = len(d_offs) - 1
    rng = np.random.default_rng(seed)
    pick = int(round(w.retrieval_ratio * (n - 1)))
    sels = [np.concatenate([[0], np.sort(rng.permutation(np.arange(1, n))[:pick])]).astype(np.int32)
            for _ in range(w.n_queries)]
    return d_offs, sels


@pytest.mark.parametrize("n_new,tail_len", [(40, 40), (1, 41)])
def test_stage2_demo_granular_full_size(n_new, tail_len):
    """90k cache, 64 queries selecting single demonstrations (~885 segments
    each), checked like the block-granular batches.  The 40-token prompt pass
    takes the per-query split path; a decode step takes the block-major path
    at demonstration granularity (each demonstration's keys shared by the
    ~19 queries that selected it)."""
    w = inputs.L31_8B_90K
    cfg, offs, q, k, v, kc, vc, _ = run_stage1(w)
    del q, k, v
    d_offs, sels = demo_granular(w, offs, seed=9)
    qn, kt, vt, out, dbg = run_stage2(w, cfg, kc, vc, d_offs, sels, n_new, tail_len,
                                      seed=inputs.tensor_seed(w, 0, 3, 77 + n_new))
    dbg = dbg.cpu().numpy()
    for qi, s in enumerate(sels):
        check_gather_map(dbg[qi], oracle.stage2_gather_map(d_offs, s), "demo-granular q%d" % qi)
    kch, vch = host_f32(kc), host_f32(vc)
    for qi in (0, len(sels) - 1):
        want = oracle.stage2_all(kch, vch, d_offs, sels[qi], host_f32(qn[qi]),
                                 host_f32(kt[qi, :tail_len]), host_f32(vt[qi, :tail_len]),
                                 w.rope_theta)
        compare(host_f32(out[qi]), want, head_axis=1, what="demo-granular n%d q%d" % (n_new, qi))


def test_prepared_block_keys_full_size():
    """90k cache, the bench's batch: dbsa_block_keys once, then the prompt pass
    and a decode step through the prepared call, bit-identical to the plain
    call."""
    w = inputs.L31_8B_90K
    cfg, offs, q, k, v, kc, vc, _ = run_stage1(w)
    del q, k, v
    sels = inputs.selections(w)
    bk = torch.empty(dbsa.block_keys_size(cfg, offs), dtype=torch.uint8, device="cuda")
    dbsa.block_keys(cfg, kc, vc, offs, bk)
    sp, sb = dbsa.selection_csr(sels)
    for n_new, tail_len in ((w.query_tokens, w.query_tokens), (1, w.query_tokens + 3)):
        qn, kt, vt, out, _ = run_stage2(w, cfg, kc, vc, offs, sels, n_new, tail_len,
                                        seed=inputs.tensor_seed(w, 0, 3, n_new))
        ws = torch.empty(dbsa.gather_workspace_size(cfg, offs, sp, sb, n_new, tail_len),
                         dtype=torch.uint8, device="cuda")
        out2 = torch.full_like(out, float("nan"))
        dbsa.gather_rope_attend(cfg, kc, vc, offs, sp, sb, qn, kt, vt, tail_len, out2, ws,
                                block_keys=bk)
        assert dbsa.read_status(ws) == dbsa.OK
        assert torch.equal(out2, out), "prepared path differs at n_new=%d" % n_new

"""Pins for the CPU oracle (oracle/dbsa_oracle.c), CPU only.

Each test ties the oracle to something other than itself: a dense brute
force written as matrix algebra with complex-number RoPE (a different
formulation), torch's fp64 scaled_dot_product_attention, closed forms,
invariants and the page's storage figure.  Citations are to the paper-notes
page "Efficient Many-Shot In-Context Learning with Dynamic Block-Sparse
Attention": §Stage 1 (block-sparse streaming encoding), §Stage 2 (dynamic
selection and generation), §Ablations (sparse patterns), §Storage cost.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def rope_complex(x, pos, theta):
    """RoPE as complex multiplication: (x_i + i x_{i+h}) * exp(i pos w_i)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    w = np.power(float(theta), -np.arange(h) * 2.0 / d)
    z = x[..., :h] + 1j * x[..., h:]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * w)
    return np.concatenate([z.real, z.imag], axis=-1)


def block_ids(offs, T):
    return np.searchsorted(np.asarray(offs), np.arange(T), side="right") - 1


def dense_mask(offs, j, pattern=0):
    T = int(offs[-1])
    b = block_ids(offs, T)
    t = np.arange(T)[:, None]
    s = np.arange(T)[None, :]
    bt, bs = b[:, None], b[None, :]
    causal = s <= t
    if pattern == oracle.PATTERN_FULL:
        return causal
    if pattern == oracle.PATTERN_SELF:
        return causal & (bs == bt)
    if pattern == oracle.PATTERN_SINK_SELF:
        return causal & ((bs == 0) | (bs == bt))
    return causal & ((bs == 0) | ((bs >= bt - j) & (bs <= bt)))


def brute_stage1(q, k, v, offs, j, theta, pattern=0):
    T, Hq, d = q.shape
    g = Hq // k.shape[1]
    pos = np.arange(T)
    M = dense_mask(offs, j, pattern)
    out = np.zeros((T, Hq, d))
    for h in range(Hq):
        qr = rope_complex(q[:, h].astype(np.float64), pos, theta)
        kr = rope_complex(k[:, h // g].astype(np.float64), pos, theta)
        S = qr @ kr.T / math.sqrt(d)
        S = np.where(M, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P /= P.sum(axis=1, keepdims=True)
        out[:, h] = P @ v[:, h // g].astype(np.float64)
    return out


def rand_offs(rng, nb, lo, hi):
    lens = rng.integers(lo, hi + 1, size=nb)
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def randf(rng, *shape):
    return rng.standard_normal(shape).astype(np.float32)


# ---------------------------------------------------------------- a1: grouping
def test_group_blocks_closed_form():
    lens = np.full(20, 3, dtype=np.int32)
    offs = oracle.group_blocks(lens, 4)
    assert offs.tolist() == [0, 12, 24, 36, 48, 60]
    # partial last block keeps the remainder
    offs = oracle.group_blocks(np.arange(1, 11, dtype=np.int32), 4)
    assert offs.tolist() == [0, 1 + 2 + 3 + 4, 55 - 9 - 10, 55]


def test_group_blocks_brute_force():
    rng = np.random.default_rng(1)
    for k in (1, 3, 50):
        lens = rng.integers(15, 46, size=173).astype(np.int32)
        offs = oracle.group_blocks(lens, k)
        nb = -(-173 // k)
        assert len(offs) == nb + 1
        for b in range(nb):
            assert offs[b + 1] - offs[b] == lens[b * k:(b + 1) * k].sum()


# ---------------------------------------------------------------- RoPE
def test_rope_textbook_rotation_d2():
    # d = 2: w_0 = 1, so R(p) is the plane rotation by p radians.
    x = np.array([0.3, -1.7])
    for p in (0.0, 1.0, 2.5, 100.0):
        Rm = np.array([[math.cos(p), -math.sin(p)], [math.sin(p), math.cos(p)]])
        np.testing.assert_allclose(oracle.rope(x, p, 1e4), Rm @ x, rtol=0, atol=1e-13)


@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 5e5)])
def test_rope_group_identities(d, theta):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(d)
    np.testing.assert_array_equal(oracle.rope(x, 0.0, theta), x)               # R(0) = I
    for p in (1.0, 1234.0, 131071.0):
        y = oracle.rope(x, p, theta)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)
        np.testing.assert_allclose(oracle.rope(oracle.rope(x, p, theta), 77.0, theta),
                                   oracle.rope(x, p + 77.0, theta), atol=1e-9)  # R(a)R(b)=R(a+b)
        np.testing.assert_allclose(y, rope_complex(x, p, theta), atol=1e-9)


@pytest.mark.parametrize("c", [1.0, 1e3, 1e5, 1e6])
def test_rope_score_shift_invariance(c):
    # R(a)^T R(b) = R(b - a): q'.k' depends only on the position difference.
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for a, b in ((0.0, 5.0), (300.0, 17.0), (90000.0, 1500.0)):
        s0 = oracle.rope(q, a, 5e5) @ oracle.rope(k, b, 5e5)
        s1 = oracle.rope(q, a + c, 5e5) @ oracle.rope(k, b + c, 5e5)
        assert abs(s0 - s1) < 1e-8 * np.linalg.norm(q) * np.linalg.norm(k)


def test_rope_frequencies():
    # frequency of pair i is theta^(-2i/d): the angle turned per position.
    d, theta = 128, 5e5
    for i in (0, 1, 17, 63):
        e = np.zeros(d)
        e[i] = 1.0
        y = oracle.rope(e, 1.0, theta)
        ang = math.atan2(y[i + d // 2], y[i])
        assert abs(ang - theta ** (-2 * i / d)) < 1e-14


# ---------------------------------------------------------------- Stage-1 mask
def test_stage1_mask_matches_dense_mask():
    rng = np.random.default_rng(4)
    offs = rand_offs(rng, 7, 1, 9)
    T = int(offs[-1])
    for j in (0, 1, 2, 5):
        for pattern in range(4):
            M = dense_mask(offs, j, pattern)
            got = np.array([[oracle.stage1_allowed(offs, j, t, s, pattern) for s in range(T)]
                            for t in range(T)])
            np.testing.assert_array_equal(got, M)


def test_stage1_allowed_count_closed_form():
    # row t in block b: (t - offs[b] + 1) self keys + the lengths of the
    # distinct blocks in {0} U {max(0, b-j) .. b-1}.
    rng = np.random.default_rng(5)
    offs = rand_offs(rng, 9, 1, 12)
    for j in (0, 1, 2, 3, 20):
        cnt = oracle.stage1_allowed_counts(offs, j)
        for t in range(int(offs[-1])):
            b = int(np.searchsorted(offs, t, side="right") - 1)
            others = set(range(max(0, b - j), b)) | ({0} if b > 0 else set())
            want = (t - offs[b] + 1) + sum(int(offs[x + 1] - offs[x]) for x in others)
            assert cnt[t] == want


# ---------------------------------------------------------------- Stage 1
@pytest.mark.parametrize("seed", range(4))
def test_stage1_brute_force(seed):
    rng = np.random.default_rng(10 + seed)
    Hkv, g = [(1, 2), (2, 1), (2, 3), (1, 1)][seed]
    d = [8, 16, 32, 64][seed]
    offs = rand_offs(rng, 2 + seed * 2, 1, 9)
    T = int(offs[-1])
    q, k, v = randf(rng, T, Hkv * g, d), randf(rng, T, Hkv, d), randf(rng, T, Hkv, d)
    for j in (0, 1, 2):
        for pattern in range(4):
            got = oracle.stage1_all(q, k, v, offs, j, 1e4, pattern=pattern)
            want = brute_stage1(q, k, v, offs, j, 1e4, pattern)
            np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def sdpa_causal(qr, kr, v):
    """torch fp64 SDPA, causal; inputs [T, H, d] already rotated (kv repeated)."""
    Q = torch.from_numpy(qr).permute(1, 0, 2)[None]
    K = torch.from_numpy(kr).permute(1, 0, 2)[None]
    V = torch.from_numpy(v).permute(1, 0, 2)[None]
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("j_extra", [0, 3])
def test_stage1_large_window_is_causal_sdpa(j_extra):
    # j >= nb - 1: every earlier block is in the window, so the DBSA pattern
    # is plain causal attention (pin against a library routine).
    rng = np.random.default_rng(20)
    offs = rand_offs(rng, 6, 3, 20)
    T = int(offs[-1])
    Hq, Hkv, d, theta = 4, 2, 32, 1e4
    q, k, v = randf(rng, T, Hq, d), randf(rng, T, Hkv, d), randf(rng, T, Hkv, d)
    got = oracle.stage1_all(q, k, v, offs, len(offs) - 2 + j_extra, theta)
    pos = np.arange(T)
    qr = rope_complex(q, pos[:, None], theta)
    kr = np.repeat(rope_complex(k, pos[:, None], theta), Hq // Hkv, axis=1)
    want = sdpa_causal(qr, kr, np.repeat(v.astype(np.float64), Hq // Hkv, axis=1))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # the FULL pattern of the ablation table is the same thing
    got_full = oracle.stage1_all(q, k, v, offs, 0, theta, pattern=oracle.PATTERN_FULL)
    np.testing.assert_allclose(got_full, want, rtol=0, atol=1e-12)


def test_stage1_self_only_is_block_diagonal_causal():
    # §Ablations "Self only": each block is an independent causal sequence
    # (positions still global, which RoPE's shift invariance makes irrelevant).
    rng = np.random.default_rng(21)
    offs = rand_offs(rng, 5, 2, 15)
    T = int(offs[-1])
    q, k, v = randf(rng, T, 2, 16), randf(rng, T, 2, 16), randf(rng, T, 2, 16)
    got = oracle.stage1_all(q, k, v, offs, 2, 1e4, pattern=oracle.PATTERN_SELF)
    for b in range(len(offs) - 1):
        a, e = offs[b], offs[b + 1]
        local = np.arange(e - a)
        want = sdpa_causal(rope_complex(q[a:e], local[:, None], 1e4),
                           rope_complex(k[a:e], local[:, None], 1e4), v[a:e].astype(np.float64))
        np.testing.assert_allclose(got[a:e], want, rtol=0, atol=1e-12)


def test_stage1_closed_forms():
    rng = np.random.default_rng(22)
    offs = rand_offs(rng, 7, 3, 11)
    T = int(offs[-1])
    Hq, Hkv, d, j = 2, 1, 16, 2
    q, k, v = randf(rng, T, Hq, d), randf(rng, T, Hkv, d), randf(rng, T, Hkv, d)
    out = oracle.stage1_all(q, k, v, offs, j, 1e4)
    # the first token of the sink block sees only itself
    np.testing.assert_array_equal(out[0, 0], v[0, 0].astype(np.float64))
    # constant values give a constant output (rows normalised to 1)
    vc = np.full_like(v, 0.75)
    np.testing.assert_allclose(oracle.stage1_all(q, k, vc, offs, j, 1e4), 0.75, rtol=0, atol=1e-13)
    # zero queries give the plain mean of the allowed values, allowed set in
    # closed form: [0, offs[1]) U [offs[max(0, b-j)], t]
    out0 = oracle.stage1_all(np.zeros_like(q), k, v, offs, j, 1e4)
    for t in range(T):
        b = int(np.searchsorted(offs, t, side="right") - 1)
        idx = set(range(0, offs[1])) | set(range(offs[max(0, b - j)], t + 1))
        idx = sorted(i for i in idx if i <= t)
        np.testing.assert_allclose(out0[t, 1], v[idx, 0].astype(np.float64).mean(axis=0),
                                   rtol=0, atol=1e-13)


def test_stage1_masked_keys_have_zero_mass():
    # perturbing K/V of keys outside every window leaves a row bit-identical
    rng = np.random.default_rng(23)
    offs = rand_offs(rng, 8, 4, 9)
    T = int(offs[-1])
    q, k, v = randf(rng, T, 2, 16), randf(rng, T, 1, 16), randf(rng, T, 1, 16)
    j, b = 2, 6
    rows = np.arange(offs[b], offs[b + 1])
    base = oracle.stage1_rows(q, k, v, offs, j, 1e4, np.zeros(len(rows)), rows)
    k2, v2 = k.copy(), v.copy()
    k2[offs[1]:offs[b - j]] += 5.0
    v2[offs[1]:offs[b - j]] -= 3.0
    k2[offs[b + 1]:] = 9.0   # later blocks (not causal-visible)
    pert = oracle.stage1_rows(q, k2, v2, offs, j, 1e4, np.zeros(len(rows)), rows)
    np.testing.assert_array_equal(base, pert)


def test_hand_worked_two_tokens():
    # One block of two tokens, d = 2, so R(p) rotates by p radians.
    # q_1 = (1, 0) at position 1 -> (cos 1, sin 1); k_0 = (1, 0) at 0;
    # k_1 = (0, 1) at 1 -> (-sin 1, cos 1).  Scores / sqrt(2): cos(1)/sqrt(2), 0.
    q = np.array([[[0.0, 0.0]], [[1.0, 0.0]]], dtype=np.float32)
    k = np.array([[[1.0, 0.0]], [[0.0, 1.0]]], dtype=np.float32)
    v = np.array([[[2.0, -1.0]], [[0.5, 4.0]]], dtype=np.float32)
    out = oracle.stage1_all(q, k, v, np.array([0, 2]), 2, 1e4)
    a = math.exp(math.cos(1.0) / math.sqrt(2.0))
    want = (a * np.array([2.0, -1.0]) + np.array([0.5, 4.0])) / (a + 1.0)
    np.testing.assert_allclose(out[1, 0], want, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(out[0, 0], [2.0, -1.0])


# ---------------------------------------------------------------- Stage 2
def test_gather_map_exact_and_validation():
    offs = np.array([0, 5, 9, 16, 20], dtype=np.int32)
    m = oracle.stage2_gather_map(offs, [0, 3, 1])
    want_rows = list(range(0, 5)) + list(range(16, 20)) + list(range(5, 9))
    assert m[:, 0].tolist() == want_rows
    assert m[:, 1].tolist() == list(range(len(want_rows)))
    for bad in ([1, 0], [0, 2, 2], [0, 4], [0, -1], []):
        with pytest.raises(ValueError):
            oracle.stage2_gather_map(offs, bad)


def brute_stage2(kc, vc, offs, sel, qn, kt, vt, theta):
    Hkv, cap, d = kc.shape
    n_new, Hq, _ = qn.shape
    g = Hq // Hkv
    rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in sel])
    Tg = len(rows)
    tail_len = kt.shape[0]
    out = np.zeros((n_new, Hq, d))
    for h in range(Hq):
        c = h // g
        keys = np.concatenate([kc[c, rows], kt[:, c]]).astype(np.float64)
        vals = np.concatenate([vc[c, rows], vt[:, c]]).astype(np.float64)
        kpos = np.arange(Tg + tail_len)
        kr = rope_complex(keys, kpos, theta)
        qpos = Tg + tail_len - n_new + np.arange(n_new)
        qr = rope_complex(qn[:, h].astype(np.float64), qpos, theta)
        S = qr @ kr.T / math.sqrt(d)
        S = np.where(kpos[None, :] <= qpos[:, None], S, -np.inf)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        out[:, h] = (P / P.sum(axis=1, keepdims=True)) @ vals
    return out


@pytest.mark.parametrize("seed", range(3))
def test_stage2_brute_force(seed):
    rng = np.random.default_rng(30 + seed)
    nb, Hkv, g, d = 9, [1, 2, 2][seed], [2, 1, 4][seed], [16, 32, 64][seed]
    offs = rand_offs(rng, nb, 2, 12)
    cap = int(offs[-1]) + 7
    kc, vc = randf(rng, Hkv, cap, d), randf(rng, Hkv, cap, d)
    sel = np.concatenate([[0], rng.choice(np.arange(1, nb), size=4, replace=False)])
    tail_len, n_new = [5, 8, 3][seed], [5, 1, 2][seed]
    qn = randf(rng, n_new, Hkv * g, d)
    kt, vt = randf(rng, tail_len, Hkv, d), randf(rng, tail_len, Hkv, d)
    got = oracle.stage2_all(kc, vc, offs, sel, qn, kt, vt, 1e4)
    want = brute_stage2(kc, vc, offs, sel, qn, kt, vt, 1e4)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_stage2_all_blocks_in_encoding_order_is_standard_attention():
    # Selecting every block in encoding order gives fresh positions equal to
    # the original ones, so the query attends exactly as in full causal
    # attention over [context ; query tokens] (library routine).
    rng = np.random.default_rng(40)
    nb, Hq, Hkv, d, theta = 6, 4, 2, 32, 5e5
    offs = rand_offs(rng, nb, 3, 14)
    T = int(offs[-1])
    kc, vc = randf(rng, Hkv, T, d), randf(rng, Hkv, T, d)
    tail_len, n_new = 6, 4
    qn = randf(rng, n_new, Hq, d)
    kt, vt = randf(rng, tail_len, Hkv, d), randf(rng, tail_len, Hkv, d)
    sel = np.arange(nb)
    m = oracle.stage2_gather_map(offs, sel)
    np.testing.assert_array_equal(m[:, 0], m[:, 1])
    got = oracle.stage2_all(kc, vc, offs, sel, qn, kt, vt, theta)
    # full sequence: context then tail; queries are the last n_new tail tokens
    K = np.concatenate([kc.transpose(1, 0, 2), kt]).astype(np.float64)
    V = np.concatenate([vc.transpose(1, 0, 2), vt]).astype(np.float64)
    pos = np.arange(T + tail_len)
    Qfull = np.zeros((T + tail_len, Hq, d))
    Qfull[T + tail_len - n_new:] = qn
    want = sdpa_causal(rope_complex(Qfull, pos[:, None], theta),
                       np.repeat(rope_complex(K, pos[:, None], theta), Hq // Hkv, axis=1),
                       np.repeat(V, Hq // Hkv, axis=1))
    np.testing.assert_allclose(got, want[T + tail_len - n_new:], rtol=0, atol=1e-12)


def test_stage2_closed_forms():
    rng = np.random.default_rng(41)
    nb, Hkv, g, d = 7, 2, 2, 16
    offs = rand_offs(rng, nb, 2, 9)
    cap = int(offs[-1])
    kc, vc = randf(rng, Hkv, cap, d), randf(rng, Hkv, cap, d)
    sel = np.array([0, 5, 2])
    tail_len, n_new = 4, 2
    qn = randf(rng, n_new, Hkv * g, d)
    kt, vt = randf(rng, tail_len, Hkv, d), randf(rng, tail_len, Hkv, d)
    # constant values -> constant output
    got = oracle.stage2_all(kc, np.full_like(vc, -2.5), offs, sel, qn, kt, np.full_like(vt, -2.5), 1e4)
    np.testing.assert_allclose(got, -2.5, rtol=0, atol=1e-13)
    # zero query -> mean of gathered values and the visible tail values
    got = oracle.stage2_all(kc, vc, offs, sel, np.zeros_like(qn), kt, vt, 1e4)
    rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in sel])
    for u in range(n_new):
        tu = tail_len - n_new + u
        for h in range(Hkv * g):
            c = h // g
            vals = np.concatenate([vc[c, rows], vt[:tu + 1, c]]).astype(np.float64)
            np.testing.assert_allclose(got[u, h], vals.mean(axis=0), rtol=0, atol=1e-13)


def test_stage2_order_changes_positions_not_keys():
    # With zero queries the output ignores positions, so any order of the
    # same blocks gives the same mean; with real queries positions matter.
    rng = np.random.default_rng(42)
    offs = rand_offs(rng, 6, 3, 9)
    kc, vc = randf(rng, 1, int(offs[-1]), 16), randf(rng, 1, int(offs[-1]), 16)
    qn = randf(rng, 1, 1, 16) * 4
    kt, vt = randf(rng, 1, 1, 16), randf(rng, 1, 1, 16)
    a = oracle.stage2_all(kc, vc, offs, [0, 2, 4], np.zeros_like(qn), kt, vt, 1e4)
    b = oracle.stage2_all(kc, vc, offs, [0, 4, 2], np.zeros_like(qn), kt, vt, 1e4)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    a = oracle.stage2_all(kc, vc, offs, [0, 2, 4], qn, kt, vt, 1e4)
    b = oracle.stage2_all(kc, vc, offs, [0, 4, 2], qn, kt, vt, 1e4)
    assert np.abs(a - b).max() > 1e-6


# ---------------------------------------------------------------- storage figure
def test_storage_per_token_matches_page():
    # §Storage cost: Llama-3.1-8B KV cache is 0.125 MiB per token.
    with open(os.path.join(GOLDEN, "storage_llama31_8b.json")) as f:
        gold = json.load(f)
    layers, kv_heads, head_dim, kv, bytes_per = 32, 8, 128, 2, 2
    per_token = layers * kv_heads * head_dim * kv * bytes_per
    assert per_token / 2**20 == gold["mib_per_token"]
    for ctx, gb in gold["total_gb_at_context"].items():
        assert abs(int(ctx) * per_token / 2**30 - gb) / gb < 0.02

"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

The pages print no worked example with numbers, so the oracle is pinned by
closed forms, special cases that reduce to a library routine, invariants of
the definition and an independent dense-mask restatement on tiny inputs.
The degenerate case "top-k at least the sequence length is dense attention"
is stated on the DSA page ("DeepSeek V3.2-Exp sparse attention", section on
the indexer); the branch structure and gate follow the NSA config page,
sections 1 and 3.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import workloads as wl
from tests.nsa_brute import bf16_to_f64, nsa_dense


def _rand_inputs(seed, T, Hq, Hkv, D, l):
    rng = np.random.default_rng(seed)
    q = wl.bf16_bits(rng.standard_normal((T, Hq, D), dtype=np.float32))
    k = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    v = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    gates = rng.random((T, Hq, 3), dtype=np.float32)
    wk = (rng.standard_normal((Hkv, D, l * D), dtype=np.float32) / np.float32(math.sqrt(l * D)))
    wv = (rng.standard_normal((Hkv, D, l * D), dtype=np.float32) / np.float32(math.sqrt(l * D)))
    return q, k, v, gates, wk, wv


def _run(p, q, k, v, gates, wk, wv, rows=None, kc=None, vc=None):
    T = q.shape[0]
    _, kc16 = oracle.compress(p, k, wk)
    _, vc16 = oracle.compress(p, v, wv)
    kc = kc16 if kc is None else kc
    vc = vc16 if vc is None else vc
    if kc.shape[0] == 0:
        kc = np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16)
        vc = np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16)
    rows = np.arange(T) if rows is None else rows
    # score columns: every selection block a query of this sequence may rank
    cmax = max(1, T // p.sel_block + 1)
    return oracle.nsa_rows(p, q, k, v, kc, vc, gates, rows, cmax=cmax), kc, vc


def _dense_causal(q, k, v, D, G):
    """torch fp64 SDPA, causal, GQA by head repetition: [T,Hq,D]."""
    qt = torch.from_numpy(bf16_to_f64(q)).permute(1, 0, 2)
    kt = torch.from_numpy(bf16_to_f64(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(bf16_to_f64(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                         scale=1.0 / math.sqrt(D))
    return o.permute(1, 0, 2).numpy()


# ------------------------------------------------------------------ bf16 rounding
def test_bf16_single_rounding_ties_to_even():
    # exact bf16 values stay
    assert oracle.bf16_round_f64(1.0) == 0x3F80
    assert oracle.bf16_round_f64(-2.0) == 0xC000
    # halfway between 1 and 1+2^-7 -> even (1.0); halfway between 1+2^-7 and 1+2^-6 -> 1+2^-6
    assert oracle.bf16_round_f64(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.bf16_round_f64(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above a tie: one rounding goes up; rounding through fp32 first would tie to even
    assert oracle.bf16_round_f64(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    # underflow to the subnormal grid and overflow to infinity
    assert oracle.bf16_round_f64(2.0 ** -133) == 0x0001
    assert oracle.bf16_round_f64(3.5e38) == 0x7F80


# ------------------------------------------------------------------ step 1
def test_mean_pool_compressor_by_hand():
    # T = 4 tokens, D = 2, one KV head, l = d = 2; W = [I/2, I/2] gives block means.
    p = OracleParams(2, 1, 1, 2, 2, 2, 1, 1)
    k = wl.bf16_bits(np.array([[[1, 2]], [[3, 4]], [[5, 6]], [[7, 9]]], dtype=np.float32))
    w = np.zeros((1, 2, 4), dtype=np.float32)
    w[0, 0, 0] = w[0, 0, 2] = 0.5
    w[0, 1, 1] = w[0, 1, 3] = 0.5
    f, b = oracle.compress(p, k, w)
    # blocks: mean([1,2],[3,4]) = [2,3]; mean([5,6],[7,9]) = [6,7.5]
    assert np.array_equal(f[:, 0, :], np.array([[2.0, 3.0], [6.0, 7.5]]))
    assert np.array_equal(b[:, 0, :], wl.bf16_bits(np.array([[2, 3], [6, 7.5]], np.float32)))


def test_compress_matches_einsum_and_block_count():
    p = OracleParams(16, 4, 2, 8, 8, 8, 2, 8)
    q, k, v, gates, wk, wv = _rand_inputs(3, 45, 4, 2, 16, 8)
    f, b = oracle.compress(p, k, wk)
    assert f.shape[0] == (45 - 8) // 8 + 1 == 5
    kf = bf16_to_f64(k)[:40].reshape(5, 8, 2, 16).transpose(0, 2, 1, 3).reshape(5, 2, 128)
    ref = np.einsum("ihk,hck->ihc", kf, wk.astype(np.float64))
    assert np.allclose(f, ref, rtol=0, atol=1e-12)
    assert np.array_equal(b, np.vectorize(oracle.bf16_round_f64)(f).astype(np.uint16))


# ------------------------------------------------------------------ dense reductions
def test_selected_and_window_reduce_to_dense_causal():
    T, Hq, Hkv, D, l = 96, 4, 2, 16, 8
    p = OracleParams(D, Hq, Hkv, l, l, l, T // l, T)
    q, k, v, gates, wk, wv = _rand_inputs(5, T, Hq, Hkv, D, l)
    r, _, _ = _run(p, q, k, v, gates, wk, wv)
    dense = _dense_causal(q, k, v, D, Hq // Hkv)
    assert np.max(np.abs(r["o_slc"] - dense)) < 1e-12
    assert np.max(np.abs(r["o_win"] - dense)) < 1e-12


def test_compressed_branch_reduces_to_dense_with_identity_compressor():
    T, Hq, Hkv, D = 40, 2, 1, 8
    p = OracleParams(D, Hq, Hkv, 1, 1, 1, 1, 1)
    q, k, v, gates, _, _ = _rand_inputs(6, T, Hq, Hkv, D, 1)
    eye = np.eye(D, dtype=np.float32)[None]
    r, kc, vc = _run(p, q, k, v, gates, eye, eye)
    assert np.array_equal(kc, k) and np.array_equal(vc, v)
    dense = _dense_causal(q, k, v, D, Hq // Hkv)
    assert np.max(np.abs(r["o_cmp"] - dense)) < 1e-12


def test_window_of_one_returns_v_t():
    T, Hq, Hkv, D, l = 33, 4, 2, 8, 4
    p = OracleParams(D, Hq, Hkv, l, l, l, 2, 1)
    q, k, v, gates, wk, wv = _rand_inputs(7, T, Hq, Hkv, D, l)
    r, _, _ = _run(p, q, k, v, gates, wk, wv)
    vt = np.repeat(bf16_to_f64(v), Hq // Hkv, axis=1)
    assert np.array_equal(r["o_win"], vt)


# ------------------------------------------------------------------ gates
@pytest.mark.parametrize("branch", [0, 1, 2])
def test_one_hot_gates_isolate_each_branch(branch):
    T, Hq, Hkv, D, l = 70, 4, 1, 8, 8
    p = OracleParams(D, Hq, Hkv, l, l, l, 3, 16)
    q, k, v, _, wk, wv = _rand_inputs(8, T, Hq, Hkv, D, l)
    gates = np.zeros((T, Hq, 3), np.float32)
    gates[..., branch] = 1.0
    r, _, _ = _run(p, q, k, v, gates, wk, wv)
    name = ("o_cmp", "o_slc", "o_win")[branch]
    assert np.array_equal(r["out"], r[name])


# ------------------------------------------------------------------ invariants
def test_score_mass_softmax_and_convex_hull():
    T, Hq, Hkv, D, l = 130, 8, 2, 8, 8
    G = Hq // Hkv
    p = OracleParams(D, Hq, Hkv, l, l, l, 4, 20)
    q, k, v, gates, wk, wv = _rand_inputs(9, T, Hq, Hkv, D, l)
    r, kc, vc = _run(p, q, k, v, gates, wk, wv)
    vcf, vf = bf16_to_f64(vc), bf16_to_f64(v)
    for t in range(T):
        ncmp = (t + 1 - l) // l + 1 if t + 1 >= l else 0
        mass = r["scores"][t].sum(axis=-1)
        if ncmp:
            assert np.allclose(mass, G, atol=1e-12)
        else:
            assert np.all(mass == 0) and np.all(r["o_cmp"][t] == 0)
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            if ncmp:
                lo, hi = vcf[:ncmp, g].min(0), vcf[:ncmp, g].max(0)
                assert np.all(r["o_cmp"][t, hs] >= lo - 1e-12) and np.all(r["o_cmp"][t, hs] <= hi + 1e-12)
            win = vf[max(0, t - 19):t + 1, g]
            assert np.all(r["o_win"][t, hs] >= win.min(0) - 1e-12)
            assert np.all(r["o_win"][t, hs] <= win.max(0) + 1e-12)
            sel = r["sel"][t, g]
            keys = np.concatenate([np.arange(j * l, min((j + 1) * l, t + 1)) for j in sel if j >= 0])
            assert np.all(r["o_slc"][t, hs] >= vf[keys, g].min(0) - 1e-12)
            assert np.all(r["o_slc"][t, hs] <= vf[keys, g].max(0) + 1e-12)
    # log-sum-exp equals the normaliser of the compressed softmax
    t = T - 1
    z = bf16_to_f64(q[t, 0]) @ bf16_to_f64(kc[: (t + 1) // l, 0]).T / math.sqrt(D)
    assert abs(r["lse"][t, 0] - (z.max() + np.log(np.exp(z - z.max()).sum()))) < 1e-12


def test_causality_future_tokens_do_not_matter():
    T, Hq, Hkv, D, l = 64, 4, 2, 8, 8
    p = OracleParams(D, Hq, Hkv, l, l, l, 2, 10)
    q, k, v, gates, wk, wv = _rand_inputs(10, T, Hq, Hkv, D, l)
    rows = np.arange(40)
    r1, _, _ = _run(p, q, k, v, gates, wk, wv, rows=rows)
    k2, v2, q2 = k.copy(), v.copy(), q.copy()
    rng = np.random.default_rng(11)
    k2[40:] = wl.bf16_bits(rng.standard_normal(k2[40:].shape, dtype=np.float32))
    v2[40:] = wl.bf16_bits(rng.standard_normal(v2[40:].shape, dtype=np.float32))
    q2[40:] = wl.bf16_bits(rng.standard_normal(q2[40:].shape, dtype=np.float32))
    r2, _, _ = _run(p, q2, k2, v2, gates, wk, wv, rows=rows)
    for key in ("out", "scores", "sel"):
        assert np.array_equal(r1[key], r2[key])


def test_permuting_heads_within_a_group_keeps_scores():
    T, Hq, Hkv, D, l = 80, 8, 2, 8, 8
    p = OracleParams(D, Hq, Hkv, l, l, l, 3, 8)
    q, k, v, gates, wk, wv = _rand_inputs(12, T, Hq, Hkv, D, l)
    r1, _, _ = _run(p, q, k, v, gates, wk, wv)
    perm = np.array([2, 0, 3, 1, 7, 5, 4, 6])
    r2, _, _ = _run(p, q[:, perm], k, v, gates[:, perm], wk, wv)
    assert np.allclose(r1["scores"], r2["scores"], rtol=0, atol=1e-14)
    assert np.array_equal(r1["sel"], r2["sel"])
    assert np.array_equal(r1["out"][:, perm], r2["out"])


def test_tie_goes_to_lower_block_index():
    # Blocks a=1 and b=4 hold identical keys, so their compressed keys and
    # scores tie exactly; a planted direction makes them the top two.
    T, Hq, Hkv, D, l = 64, 4, 1, 8, 8
    p = OracleParams(D, Hq, Hkv, l, l, l, 1, 4)
    q, k, v, gates, wk, wv = _rand_inputs(13, T, Hq, Hkv, D, l)
    u = np.zeros(D, np.float32)
    u[0] = 1.0
    kf = wl.bf16_to_f32(k)
    kf[8:16, 0, :] = 3.0 * u + 0.1 * kf[8:16, 0, :]
    kf[32:40, 0, :] = kf[8:16, 0, :]
    k = wl.bf16_bits(kf)
    wk = np.tile(np.eye(D, dtype=np.float32)[:, None, :] / l, (1, l, 1)).reshape(D, l * D)[None]
    qf = wl.bf16_to_f32(q)
    qf[:] = 4.0 * u
    q = wl.bf16_bits(qf)
    r, kc, _ = _run(p, q, k, v, gates, wk, wv)
    assert np.array_equal(kc[1], kc[4])
    t = T - 1
    assert r["scores"][t, 0, 1] == r["scores"][t, 0, 4]
    assert r["scores"][t, 0, 1] == r["scores"][t, 0].max()
    assert list(r["sel"][t, 0]) == [1]
    assert r["gap"][t, 0] == 0.0


def test_select_brute_force_over_all_subsets():
    rng = np.random.default_rng(14)
    for trial in range(60):
        ncand = int(rng.integers(1, 9))
        n = int(rng.integers(1, 6))
        S = rng.integers(0, 4, size=ncand).astype(np.float32) / 4.0  # many ties
        cmp_n = ncand - int(rng.integers(0, 2))                      # maybe an incomplete last block
        sel, gap = oracle.select_f32(S[None, :], np.array([ncand]), np.array([cmp_n]), n)
        Sx = np.array([S[j] if j < cmp_n else 0.0 for j in range(ncand)])
        if ncand <= n:
            want = list(range(ncand)) + [-1] * (n - ncand)
        else:
            # the unique n-subset whose every member precedes every non-member
            # under (score desc, index asc)
            def before(a, b):
                return Sx[a] > Sx[b] or (Sx[a] == Sx[b] and a < b)
            good = [c for c in itertools.combinations(range(ncand), n)
                    if all(before(a, b) for a in c for b in range(ncand) if b not in c)]
            assert len(good) == 1
            want = list(good[0])
        assert list(sel[0]) == want, (S, cmp_n, n)


# ------------------------------------------------------------------ independent restatement
@pytest.mark.parametrize("T,Hq,Hkv,D,l,n,w", [
    (1, 2, 1, 8, 4, 2, 3),        # single token, no complete block
    (7, 2, 1, 8, 8, 1, 3),        # shorter than a block
    (100, 4, 2, 16, 8, 3, 13),    # ragged tail
    (96, 8, 2, 8, 4, 5, 1),       # window of one
    (64, 4, 4, 8, 16, 2, 100),    # window longer than the sequence, G = 1
    (129, 16, 1, 8, 8, 4, 32),    # G = 16
])
def test_oracle_matches_dense_mask_statement(T, Hq, Hkv, D, l, n, w):
    p = OracleParams(D, Hq, Hkv, l, l, l, n, w)
    q, k, v, gates, wk, wv = _rand_inputs(100 + T, T, Hq, Hkv, D, l)
    r, kc, vc = _run(p, q, k, v, gates, wk, wv)
    C = T // l
    ref = nsa_dense(bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v), bf16_to_f64(kc[:C]),
                    bf16_to_f64(vc[:C]), gates.astype(np.float64), D, Hq, Hkv, l, n, w)
    for key in ("o_cmp", "o_slc", "o_win", "out"):
        assert np.max(np.abs(r[key] - ref[key])) < 1e-12, key
    if C:
        assert np.max(np.abs(r["scores"][:, :, :C] - ref["scores"][:, :, :C])) < 1e-12
    for t in range(T):
        for g in range(Hkv):
            got = [j for j in r["sel"][t, g] if j >= 0]
            assert got == list(ref["sel"][(t, g)]), (t, g)


@pytest.mark.parametrize("T,Hq,Hkv,D,l,d,lsel,n,w", [
    (100, 4, 2, 8, 8, 4, 8, 3, 13),   # overlapping compression (d < l)
    (100, 4, 1, 8, 8, 4, 16, 2, 9),   # overlapping, selection block 2 l
    (97, 2, 1, 8, 4, 4, 8, 3, 5),     # l = d, selection block 2 l
    (64, 4, 2, 8, 8, 8, 4, 4, 7),     # selection block shorter than a compressed block
    (50, 2, 1, 8, 6, 3, 5, 2, 4),     # sizes that share no factor
    (5, 2, 1, 8, 4, 2, 2, 1, 2),      # barely one compressed block
])
def test_oracle_matches_dense_mask_statement_general_geometry(T, Hq, Hkv, D, l, d, lsel, n, w):
    """Compression stride d and selection block l' independent of l: each
    compressed block adds its probability to every selection block it
    overlaps.  The oracle's row walk must agree with the dense-mask statement,
    whose overlap is a [C, J] boolean matrix."""
    p = OracleParams(D, Hq, Hkv, l, d, lsel, n, w)
    q, k, v, gates, wk, wv = _rand_inputs(300 + T + d + lsel, T, Hq, Hkv, D, l)
    r, kc, vc = _run(p, q, k, v, gates, wk, wv)
    C = oracle.num_cmp_blocks(p, T)
    assert C == (0 if T < l else (T - l) // d + 1)
    ref = nsa_dense(bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v), bf16_to_f64(kc[:max(C, 0)]),
                    bf16_to_f64(vc[:max(C, 0)]), gates.astype(np.float64), D, Hq, Hkv, l, n, w,
                    d=d, lsel=lsel)
    for key in ("o_cmp", "o_slc", "o_win", "out"):
        assert np.max(np.abs(r[key] - ref[key])) < 1e-12, key
    J = T // lsel + 1
    assert np.max(np.abs(r["scores"][:, :, :J] - ref["scores"][:, :, :J])) < 1e-12
    for t in range(T):
        for g in range(Hkv):
            got = [j for j in r["sel"][t, g] if j >= 0]
            assert got == list(ref["sel"][(t, g)]), (t, g)


def test_selection_block_score_sums_its_compressed_blocks():
    """With d = l and l' = 2 l every compressed block lies in exactly one
    selection block: the score of selection block J is the sum of the scores
    of compressed blocks 2J and 2J + 1 under l' = l."""
    T, Hq, Hkv, D, l = 120, 4, 2, 8, 4
    q, k, v, gates, wk, wv = _rand_inputs(77, T, Hq, Hkv, D, l)
    r1, _, _ = _run(OracleParams(D, Hq, Hkv, l, l, l, 3, 5), q, k, v, gates, wk, wv)
    r2, _, _ = _run(OracleParams(D, Hq, Hkv, l, l, 2 * l, 3, 5), q, k, v, gates, wk, wv)
    s1 = r1["scores"]
    J = T // (2 * l) + 1
    for j in range(J):
        want = s1[:, :, 2 * j] + (s1[:, :, 2 * j + 1] if 2 * j + 1 < s1.shape[2] else 0.0)
        assert np.max(np.abs(r2["scores"][:, :, j] - want)) < 1e-13, j
    # the compressed branch does not depend on the selection block
    assert np.array_equal(r1["o_cmp"], r2["o_cmp"]) and np.array_equal(r1["lse"], r2["lse"])


def test_overlapping_compression_worked_example():
    """Eight tokens, one head, D = 2, l = 4, d = 2, l' = 4, n = 1, w = 1, zero
    queries (uniform softmaxes) and mean pooling, worked out by hand:
      compressed block i covers tokens 2i .. 2i + 3 and is visible once
      2i + 3 <= t;  v = (1,0) (0,1) (2,2) (4,0) (0,0) (2,0) (0,4) (8,8), so
      Vc0 = (7/4, 3/4), Vc1 = (2, 1/2), Vc2 = (5/2, 3);
      t = 5: blocks 0, 1 visible, p = 1/2 each; block 0 meets selection block
        0, block 1 (tokens 2..5) meets selection blocks 0 and 1: S = (1, 1/2);
        O_cmp = (15/8, 5/8);
      t = 7: blocks 0, 1, 2, p = 1/3: S = (2/3, 2/3), an exact tie the lower
        block wins; O_cmp = (25/12, 17/12); O_slc = mean of v0..v3 = (7/4, 3/4);
        O_win = v7."""
    D, l, d, lsel = 2, 4, 2, 4
    p = OracleParams(D, 1, 1, l, d, lsel, 1, 1)
    q = wl.bf16_bits(np.zeros((8, 1, D), dtype=np.float32))
    k = wl.bf16_bits(np.arange(16, dtype=np.float32).reshape(8, 1, D))
    v = wl.bf16_bits(np.array([[[1, 0]], [[0, 1]], [[2, 2]], [[4, 0]], [[0, 0]], [[2, 0]],
                               [[0, 4]], [[8, 8]]], dtype=np.float32))
    gates = np.tile(np.array([1.0, 0.0, 0.0], dtype=np.float32), (8, 1, 1))
    w = np.zeros((1, D, l * D), dtype=np.float32)
    for c in range(D):
        for pos in range(l):
            w[0, c, pos * D + c] = 1.0 / l
    _, kc = oracle.compress(p, k, w)
    _, vc = oracle.compress(p, v, w)
    assert np.array_equal(bf16_to_f64(vc)[:, 0], [[1.75, 0.75], [2.0, 0.5], [2.5, 3.0]])
    r = oracle.nsa_rows(p, q, k, v, kc, vc, gates, np.array([5, 7], dtype=np.int32), cmax=2)
    assert np.allclose(r["scores"][:, 0, :], [[1.0, 0.5], [2 / 3, 2 / 3]], rtol=0, atol=1e-15)
    assert np.array_equal(r["sel"][:, 0, 0], [0, 0])
    assert np.allclose(r["o_cmp"][:, 0], [[15 / 8, 5 / 8], [25 / 12, 17 / 12]], rtol=0, atol=1e-15)
    assert np.allclose(r["o_slc"][1, 0], [1.75, 0.75], rtol=0, atol=1e-15)
    assert np.array_equal(r["o_win"][1, 0], [8.0, 8.0])
    assert r["gap"][1, 0] == 0.0


@pytest.mark.parametrize("l,d,lsel", [(8, 8, 8), (8, 4, 16)])
def test_decode_query_equals_last_prefill_row(l, d, lsel):
    T, Hq, Hkv, D = 128, 4, 2, 8
    p = OracleParams(D, Hq, Hkv, l, d, lsel, 3, 16)
    q, k, v, gates, wk, wv = _rand_inputs(15, T, Hq, Hkv, D, l)
    r, kc, vc = _run(p, q, k, v, gates, wk, wv)
    for L in (T, T - 3):  # L = T completes the last compressed block with the new token
        inputs = {"q": q[L - 1][None], "k": k[None, :L], "v": v[None, :L],
                  "kc": kc[None], "vc": vc[None], "gates": gates[L - 1][None],
                  "seqlens": np.array([L]), "w_k": wk, "w_v": wv}
        C = oracle.num_cmp_blocks(p, L)
        if (C - 1) * d + l == L:
            inputs["kc"] = inputs["kc"].copy()
            inputs["kc"][0, C - 1] = 0  # must be recomputed from the cache
            inputs["vc"] = inputs["vc"].copy()
            inputs["vc"][0, C - 1] = 0
        dr = oracle.decode_reference(p, inputs, 0)
        assert np.array_equal(dr["out"], r["out"][L - 1])
        assert np.array_equal(dr["sel"], r["sel"][L - 1])


def test_workload_generator_is_seeded_and_bf16():
    cfg = wl.CONFIGS["tiny"]
    a = wl.prefill_inputs(cfg)
    b = wl.prefill_inputs(cfg)
    for key in ("q", "k", "v", "gates", "w_k", "w_v"):
        assert np.array_equal(a[key], b[key])
    assert a["q"].dtype == np.uint16 and a["q"].shape == (1024, 4, 64)
    assert a["w_k"].shape == (1, 64, 32 * 64)
    assert abs(float(np.std(a["w_k"])) - 1 / math.sqrt(32 * 64)) < 1e-3
    lens = wl.varlen_lengths(5)
    assert len(lens) == 8 and sum(lens) <= 131072 and all(4096 <= x <= 32768 for x in lens)
    # bf16 rounding of the generator is round-to-nearest-even
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -3.0], np.float32)
    assert list(wl.bf16_bits(x)) == [0x3F80, 0x3F82, 0xC040]


def test_worked_example_by_hand():
    """Four tokens, worked out by hand from the definition (zero queries make
    every softmax uniform; mean-pooling weights make the compressed values
    block means; all numbers are exact dyadic fractions).

    D = 2, one head, l = d = l' = 2, n = 1, w = 1; v = (1,0), (0,1), (2,2), (4,0);
    gates (g_cmp, g_slc, g_win) = (1/2, 1/4, 1/4) for every token.
      compressed: Vc0 = (1/2, 1/2), Vc1 = (3, 1); token t sees blocks i with
        2i + 1 <= t, so O_cmp = 0, Vc0, Vc0, (Vc0 + Vc1)/2 = (7/4, 3/4);
      scores: t = 1, 2: S0 = 1 (block 1 is incomplete at t = 2, score 0);
        t = 3: S0 = S1 = 1/2, an exact tie that the lower index wins;
      selected: block 0 for every t, keys u <= t in it: O_slc = v0, then
        (v0 + v1)/2 = (1/2, 1/2) for t = 1, 2, 3;
      window of one: O_win = v_t;
      out = O_cmp/2 + O_slc/4 + O_win/4 =
        (1/2, 0), (3/8, 5/8), (7/8, 7/8), (2, 1/2)."""
    D, l = 2, 2
    p = OracleParams(D, 1, 1, l, l, l, 1, 1)
    q = wl.bf16_bits(np.zeros((4, 1, D), dtype=np.float32))
    k = wl.bf16_bits(np.array([[[1, 2]], [[3, -1]], [[0, 5]], [[-2, 2]]], dtype=np.float32))
    v = wl.bf16_bits(np.array([[[1, 0]], [[0, 1]], [[2, 2]], [[4, 0]]], dtype=np.float32))
    gates = np.tile(np.array([0.5, 0.25, 0.25], dtype=np.float32), (4, 1, 1))
    w = np.zeros((1, D, l * D), dtype=np.float32)
    for c in range(D):
        for pos in range(l):
            w[0, c, pos * D + c] = 1.0 / l
    _, kc = oracle.compress(p, k, w)
    _, vc = oracle.compress(p, v, w)
    assert np.array_equal(bf16_to_f64(vc)[:, 0], [[0.5, 0.5], [3.0, 1.0]])
    r = oracle.nsa_rows(p, q, k, v, kc, vc, gates, np.arange(4, dtype=np.int32), cmax=2)
    assert np.array_equal(r["o_cmp"][:, 0], [[0, 0], [0.5, 0.5], [0.5, 0.5], [1.75, 0.75]])
    assert np.array_equal(r["scores"][1:, 0, :], [[1, 0], [1, 0], [0.5, 0.5]])
    assert np.array_equal(r["sel"][:, 0, 0], [0, 0, 0, 0])
    assert np.array_equal(r["o_slc"][:, 0], [[1, 0], [0.5, 0.5], [0.5, 0.5], [0.5, 0.5]])
    assert np.array_equal(r["o_win"][:, 0], [[1, 0], [0, 1], [2, 2], [4, 0]])
    assert np.array_equal(r["out"][:, 0], [[0.5, 0], [0.375, 0.625], [0.875, 0.875], [2.0, 0.5]])

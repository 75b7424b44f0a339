"""Pins of the oracle's select-only block attention (MoBA style).

"NSA vs MoBA" (gtnt.cn/news/122266), section 1, describes MoBA as a gate that
routes each query to a few key blocks, like a mixture of experts.  The
oracle's reading (mean-pooled routing keys, the query's own block always
attended, n - 1 more blocks by routing score) is pinned here by facts that do
not come from the oracle: numpy's mean with an integer bf16 rounding, torch
fp64 attention when every block is attended or only the own block is, an
independent dense-mask statement with numpy's lexsort, and a planted exact tie.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import workloads as wl
from tests.nsa_brute import bf16_to_f64, masked_softmax


def f64_to_bf16_bits(x):
    """Round fp64 values (normal range, or 0) to bf16 bits, nearest even, on
    the integer fields of the fp64 encoding."""
    b = np.asarray(x, dtype=np.float64).view(np.uint64)
    sign = (b >> np.uint64(63)).astype(np.int64)
    exp = ((b >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    man = (b & np.uint64((1 << 52) - 1)).astype(np.int64)
    keep = man >> 45
    rem = man & ((1 << 45) - 1)
    half = 1 << 44
    up = (rem > half) | ((rem == half) & ((keep & 1) == 1))
    keep = keep + up
    exp = exp + (keep >> 7)
    keep = keep & 0x7F
    bexp = np.where(exp == 0, 0, exp - 1023 + 127)
    bits = (sign << 15) | (bexp << 7) | np.where(exp == 0, 0, keep)
    return bits.astype(np.uint16)


def _params(D, Hq, Hkv, lsel, n):
    return OracleParams(head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, cmp_block=lsel,
                        cmp_stride=lsel, sel_block=lsel, top_n=n, window=1)


def _inputs(seed, T, Hq, Hkv, D):
    rng = np.random.default_rng(seed)
    q = wl.bf16_bits(rng.standard_normal((T, Hq, D), dtype=np.float32))
    k = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    v = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    return q, k, v


def _run(p, q, k, v):
    _, kb = oracle.block_means(p, k)
    kb_use = kb if kb.shape[0] else np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16)
    T = q.shape[0]
    return oracle.block_select_rows(p, q, k, v, kb_use, np.arange(T), cmax=max(1, T // p.sel_block)), kb


def test_integer_bf16_rounding_by_hand():
    one = 1.0
    assert f64_to_bf16_bits(one) == 0x3F80
    assert f64_to_bf16_bits(1.0 + 2.0 ** -8) == 0x3F80          # halfway, to even
    assert f64_to_bf16_bits(1.0 + 3 * 2.0 ** -8) == 0x3F82      # halfway, to even (up)
    assert f64_to_bf16_bits(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert f64_to_bf16_bits(-2.0) == 0xC000
    assert f64_to_bf16_bits(0.0) == 0


@pytest.mark.parametrize("lsel", [32, 64])
def test_block_means_are_numpy_means(lsel):
    p = _params(64, 4, 2, lsel, 4)
    _, k, _ = _inputs(1, 5 * lsel + 7, 4, 2, 64)
    f, b = oracle.block_means(p, k)
    nb = k.shape[0] // lsel
    assert f.shape[0] == nb
    ref = bf16_to_f64(k[:nb * lsel]).reshape(nb, lsel, 2, 64).mean(axis=1)
    np.testing.assert_array_equal(f, ref)
    np.testing.assert_array_equal(b, f64_to_bf16_bits(ref))


def _sdpa(q, k, v, D, G, mask):
    qt = torch.from_numpy(bf16_to_f64(q)).permute(1, 0, 2)
    kt = torch.from_numpy(bf16_to_f64(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(bf16_to_f64(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=1.0 / math.sqrt(D))
    return o.permute(1, 0, 2).numpy()


def test_every_block_attended_is_dense_causal_attention():
    T, Hq, Hkv, D, lsel = 230, 4, 2, 64, 32
    p = _params(D, Hq, Hkv, lsel, T // lsel + 1)
    q, k, v = _inputs(2, T, Hq, Hkv, D)
    r, _ = _run(p, q, k, v)
    mask = np.tril(np.ones((T, T), dtype=bool))
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v, D, Hq // Hkv, mask), atol=1e-12, rtol=0)


def test_top1_is_attention_inside_the_own_block():
    T, Hq, Hkv, D, lsel = 200, 2, 1, 64, 32
    p = _params(D, Hq, Hkv, lsel, 1)
    q, k, v = _inputs(3, T, Hq, Hkv, D)
    r, _ = _run(p, q, k, v)
    t = np.arange(T)[:, None]
    u = np.arange(T)[None, :]
    mask = (u <= t) & (u // lsel == t // lsel)
    np.testing.assert_allclose(r["out"], _sdpa(q, k, v, D, Hq // Hkv, mask), atol=1e-12, rtol=0)
    assert (r["sel"][:, :, 0] == (np.arange(T) // lsel)[:, None]).all()


def _dense_statement(q, k, v, kbar, D, Hq, Hkv, lsel, n):
    """Whole-matrix restatement: routing logits [T, J], lexsort ranking, a
    boolean token mask per (t, g), one masked softmax per head."""
    T = q.shape[0]
    G = Hq // Hkv
    J = kbar.shape[0]
    qf, kf, vf, kbf = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v), bf16_to_f64(kbar)
    out = np.zeros((T, Hq, D))
    sel = np.full((T, Hkv, n), -1, dtype=np.int32)
    scores = np.zeros((T, Hkv, max(1, J)))
    u = np.arange(T)
    for g in range(Hkv):
        route = qf[:, g * G:(g + 1) * G, :].sum(axis=1) @ kbf[:, g, :].T if J else np.zeros((T, 0))
        for t in range(T):
            cur = t // lsel
            cand = np.arange(cur)
            s = route[t, :cur]
            scores[t, g, :cur] = s
            order = np.lexsort((cand, -s))            # score descending, index ascending
            chosen = np.sort(cand[order[:n - 1]]) if n > 1 else np.array([], dtype=int)
            blocks = list(chosen) + [cur]
            sel[t, g, :len(blocks)] = blocks
            keep = np.isin(u // lsel, blocks) & (u <= t)
            for hh in range(G):
                h = g * G + hh
                z = (qf[t, h] @ kf[:, g, :].T) / math.sqrt(D)
                pr = masked_softmax(z[None, :], keep[None, :])[0]
                out[t, h] = pr @ vf[:, g, :]
    return out, sel, scores


@pytest.mark.parametrize("T,Hq,Hkv,D,lsel,n", [(300, 4, 2, 64, 32, 4), (260, 2, 2, 64, 64, 2),
                                               (129, 8, 1, 64, 32, 3)])
def test_oracle_matches_dense_mask_statement(T, Hq, Hkv, D, lsel, n):
    p = _params(D, Hq, Hkv, lsel, n)
    q, k, v = _inputs(4 + T, T, Hq, Hkv, D)
    r, kb = _run(p, q, k, v)
    out, sel, scores = _dense_statement(q, k, v, kb, D, Hq, Hkv, lsel, n)
    np.testing.assert_array_equal(r["sel"], sel)
    np.testing.assert_allclose(r["scores"], scores, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["out"], out, atol=1e-12, rtol=0)


def test_exact_routing_tie_goes_to_the_lower_block():
    T, Hq, Hkv, D, lsel = 6 * 32, 2, 1, 64, 32
    p = _params(D, Hq, Hkv, lsel, 2)  # the own block and one more
    q, k, v = _inputs(5, T, Hq, Hkv, D)
    t = T - 1
    # blocks 1 and 3 hold the same keys, all along the group's summed query:
    # equal routing scores, larger than the other blocks' (whose keys are 0)
    direction = bf16_to_f64(q[t]).sum(axis=0)
    row = wl.bf16_bits((direction / np.abs(direction).max()).astype(np.float32))
    kk = np.zeros_like(k)
    kk[1 * lsel:2 * lsel, 0] = row
    kk[3 * lsel:4 * lsel, 0] = row
    kk[5 * lsel:, 0] = k[5 * lsel:, 0]
    r, _ = _run(p, q, kk, v)
    s = r["scores"][t, 0]
    assert s[1] == s[3] and s[1] > 0 and s[0] == s[2] == s[4] == 0
    assert list(r["sel"][t, 0]) == [1, 5]
    assert r["gap"][t, 0] == 0.0


def test_future_tokens_do_not_change_a_row():
    T, Hq, Hkv, D, lsel = 200, 4, 2, 64, 32
    p = _params(D, Hq, Hkv, lsel, 3)
    q, k, v = _inputs(6, T, Hq, Hkv, D)
    r, _ = _run(p, q, k, v)
    t = 150
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[t + 1:] ^= 0x0101
    k2[t + 1:] ^= 0x0101
    v2[t + 1:] ^= 0x0101
    r2, _ = _run(p, q2, k2, v2)
    np.testing.assert_array_equal(r["out"][:t + 1], r2["out"][:t + 1])
    np.testing.assert_array_equal(r["sel"][:t + 1], r2["sel"][:t + 1])


@pytest.mark.parametrize("L", [1, 31, 32, 33, 96, 130])
def test_decode_step_equals_the_last_prefill_row(L):
    D, Hq, Hkv, lsel, n = 64, 4, 2, 32, 3
    p = _params(D, Hq, Hkv, lsel, n)
    q, k, v = _inputs(40 + L, L, Hq, Hkv, D)
    r, kb = _run(p, q, k, v)
    # the routing keys of the blocks complete before the newest token
    before = (L - 1) // lsel
    _, kb_before = oracle.block_means(p, k[:before * lsel])
    d = oracle.block_select_decode_reference(p, q[L - 1], k, v, kb_before, L)
    np.testing.assert_array_equal(d["sel"], r["sel"][L - 1])
    np.testing.assert_array_equal(d["out"], r["out"][L - 1])
    if L % lsel == 0:
        np.testing.assert_array_equal(d["written"], kb[L // lsel - 1])
    else:
        assert d["written"] is None

"""Pins of the oracle's token-level top-k attention (DSA style: "DeepSeek
V3.2-Exp sparse attention" page, sections 1 and 3: a ReLU indexer with 8 or
16 heads scores the earlier tokens, the top_k of them enter the attention).

Pinned by facts outside the oracle: torch fp64 causal attention when top_k
covers every token (the degenerate case the page's complexity argument
implies), an independent dense restatement with numpy's lexsort, the ReLU
floor (indexer products that are all negative tie at 0, so the lowest tokens
win), invariance of the selection under a positive scaling of the head
weights, and causality."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import workloads as wl
from tests.nsa_brute import bf16_to_f64, masked_softmax


def _params(D, Hq, Hkv):
    return OracleParams(head_dim=D, num_q_heads=Hq, num_kv_heads=Hkv, cmp_block=32, cmp_stride=32,
                        sel_block=32, top_n=1, window=1)


def _inputs(seed, T, Hq, Hkv, D, Hi, Di):
    rng = np.random.default_rng(seed)
    q = wl.bf16_bits(rng.standard_normal((T, Hq, D), dtype=np.float32))
    k = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    v = wl.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32))
    qi = wl.bf16_bits(rng.standard_normal((T, Hi, Di), dtype=np.float32))
    ki = wl.bf16_bits(rng.standard_normal((T, Di), dtype=np.float32))
    w = rng.random((T, Hi), dtype=np.float32)
    return q, k, v, qi, w, ki


def _dense(q, k, v, qi, w, ki, D, Hq, Hkv, top_k):
    T = q.shape[0]
    G = Hq // Hkv
    qf, kf, vf = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v)
    I = np.einsum("tjc,sc->tjs", bf16_to_f64(qi), bf16_to_f64(ki))
    I = np.einsum("tj,tjs->ts", w.astype(np.float64), np.maximum(I, 0.0))
    I = np.where(np.arange(T)[None, :] <= np.arange(T)[:, None], I, 0.0)
    out = np.zeros((T, Hq, D))
    sel = np.full((T, top_k), -1, dtype=np.int32)
    for t in range(T):
        cand = np.arange(t + 1)
        order = np.lexsort((cand, -I[t, :t + 1]))
        chosen = np.sort(cand[order[:top_k]])
        sel[t, :len(chosen)] = chosen
        keep = np.zeros(T, dtype=bool)
        keep[chosen] = True
        for h in range(Hq):
            z = (qf[t, h] @ kf[:, h // G, :].T) / math.sqrt(D)
            p = masked_softmax(z[None, :], keep[None, :])[0]
            out[t, h] = p @ vf[:, h // G, :]
    return out, sel, I


@pytest.mark.parametrize("T,Hq,Hkv,D,Hi,Di,top_k", [(70, 4, 2, 64, 4, 32, 16), (40, 8, 1, 64, 8, 64, 7),
                                                   (33, 2, 2, 64, 16, 32, 1)])
def test_oracle_matches_dense_statement(T, Hq, Hkv, D, Hi, Di, top_k):
    p = _params(D, Hq, Hkv)
    q, k, v, qi, w, ki = _inputs(T, T, Hq, Hkv, D, Hi, Di)
    r = oracle.dsa_rows(p, top_k, q, k, v, qi, w, ki, np.arange(T), with_index=True)
    out, sel, I = _dense(q, k, v, qi, w, ki, D, Hq, Hkv, top_k)
    np.testing.assert_array_equal(r["sel"], sel)
    np.testing.assert_allclose(r["index"], I, atol=1e-9, rtol=0)
    np.testing.assert_allclose(r["out"], out, atol=1e-12, rtol=0)


def test_top_k_covering_every_token_is_dense_causal_attention():
    T, Hq, Hkv, D = 50, 4, 2, 64
    p = _params(D, Hq, Hkv)
    q, k, v, qi, w, ki = _inputs(3, T, Hq, Hkv, D, 4, 32)
    r = oracle.dsa_rows(p, T, q, k, v, qi, w, ki, np.arange(T))
    G = Hq // Hkv
    qt = torch.from_numpy(bf16_to_f64(q)).permute(1, 0, 2)
    kt = torch.from_numpy(bf16_to_f64(k)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    vt = torch.from_numpy(bf16_to_f64(v)).permute(1, 0, 2).repeat_interleave(G, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                         scale=1.0 / math.sqrt(D))
    np.testing.assert_allclose(r["out"], ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)
    assert np.all(r["gap"] == np.inf)


def test_relu_floor_ties_at_zero_pick_the_lowest_tokens():
    T, Hq, Hkv, D, Hi, Di, top_k = 40, 2, 1, 64, 4, 32, 5
    p = _params(D, Hq, Hkv)
    q, k, v, qi, w, ki = _inputs(4, T, Hq, Hkv, D, Hi, Di)
    qi = wl.bf16_bits(np.abs(wl.bf16_to_f32(qi)))
    ki = wl.bf16_bits(-np.abs(wl.bf16_to_f32(ki)) - 0.01)  # every product negative
    r = oracle.dsa_rows(p, top_k, q, k, v, qi, w, ki, np.arange(T), with_index=True)
    assert np.all(r["index"] == 0.0)
    for t in range(top_k, T):
        assert list(r["sel"][t]) == list(range(top_k))
        assert r["gap"][t] == 0.0


def test_selection_ignores_a_positive_scaling_of_the_head_weights():
    T, Hq, Hkv, D, Hi, Di, top_k = 60, 4, 2, 64, 8, 32, 9
    p = _params(D, Hq, Hkv)
    q, k, v, qi, w, ki = _inputs(5, T, Hq, Hkv, D, Hi, Di)
    r1 = oracle.dsa_rows(p, top_k, q, k, v, qi, w, ki, np.arange(T))
    r2 = oracle.dsa_rows(p, top_k, q, k, v, qi, (w * np.float32(4.0)).astype(np.float32), ki,
                         np.arange(T))
    np.testing.assert_array_equal(r1["sel"], r2["sel"])
    np.testing.assert_array_equal(r1["out"], r2["out"])


def test_future_tokens_do_not_change_a_row():
    T, Hq, Hkv, D, Hi, Di, top_k = 60, 4, 2, 64, 4, 32, 8
    p = _params(D, Hq, Hkv)
    ins = list(_inputs(6, T, Hq, Hkv, D, Hi, Di))
    t = 40
    r1 = oracle.dsa_rows(p, top_k, *ins, np.arange(t + 1))
    for a in (0, 1, 2, 3, 5):
        ins[a] = ins[a].copy()
        ins[a][t + 1:] ^= 0x0101
    ins[4] = ins[4].copy()
    ins[4][t + 1:] *= 3
    r2 = oracle.dsa_rows(p, top_k, *ins, np.arange(t + 1))
    np.testing.assert_array_equal(r1["sel"], r2["sel"])
    np.testing.assert_array_equal(r1["out"], r2["out"])

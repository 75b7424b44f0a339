"""Pins of the fp64 backward oracle (``oracle/backward.py``), CPU only.

  - its forward with the selection held fixed equals the C oracle's forward
    (same selection, the C oracle's bf16 compressed keys and values), and its
    fp64 step 1 equals the C oracle's fp64 step 1;
  - every gradient (q, k, v, gates, both compressor weights) equals central
    finite differences of that forward, on the plain geometry (l = d = l')
    and on overlapping compression (d < l);
  - with every candidate block chosen and the window covering the sequence,
    the selected and the window branch are dense causal attention: their
    gradients equal torch's fp64 autograd of scaled_dot_product_attention;
  - with l = d = 1 and identity compressors the compressed branch is dense
    causal attention too: same check;
  - restricted to the query rows that read a key range (the form sampled
    parity at full sizes uses), dk and dv on that range and dq on those rows
    equal the full backward's;
  - the C/OpenMP backward (``oracle.backward_c``) equals this numpy one, with
    and without given compressed tensors and row restriction.
"""
import numpy as np
import pytest

import oracle
from oracle import OracleParams
from oracle import backward as bw
from sparse_attention_long_06_b200 import workloads as wl


def _random_case(p, T, seed):
    rng = np.random.default_rng(seed)
    D, Hq, Hkv, l = p.head_dim, p.num_q_heads, p.num_kv_heads, p.cmp_block
    case = {"q": rng.standard_normal((T, Hq, D)), "k": rng.standard_normal((T, Hkv, D)),
            "v": rng.standard_normal((T, Hkv, D)), "gates": rng.random((T, Hq, 3)),
            "w_k": rng.standard_normal((Hkv, D, l * D)) / np.sqrt(l * D),
            "w_v": rng.standard_normal((Hkv, D, l * D)) / np.sqrt(l * D),
            "dout": rng.standard_normal((T, Hq, D))}
    # any valid fixed selection: up to n distinct candidate blocks j l' <= t
    sel = np.full((T, Hkv, p.top_n), -1, dtype=np.int32)
    for t in range(T):
        cand = np.arange(t // p.sel_block + 1)
        for g in range(Hkv):
            m = min(p.top_n, len(cand))
            sel[t, g, :m] = np.sort(rng.choice(cand, size=m, replace=False))
    case["sel"] = sel
    return case


def _loss(p, c, **over):
    a = {**c, **over}
    f = bw.forward_fixed(p, a["q"], a["k"], a["v"], a["gates"], a["w_k"], a["w_v"], a["sel"])
    return float(np.sum(a["dout"] * f["out"]))


def test_forward_fixed_matches_the_c_oracle():
    cfg = wl.NsaConfig("bwd_fwd", 41, 64, 4, 2, 8, 8, 8, 2, 12, seqlens=(50,))
    p = OracleParams.of(cfg)
    inp = wl.prefill_inputs(cfg)
    f64 = lambda bits: wl.bf16_to_f32(bits).astype(np.float64)  # noqa: E731
    kc64, kcb = oracle.compress(p, inp["k"], inp["w_k"])
    vc64, vcb = oracle.compress(p, inp["v"], inp["w_v"])
    r = oracle.nsa_rows(p, inp["q"], inp["k"], inp["v"], kcb, vcb, inp["gates"],
                        np.arange(50, dtype=np.int32))
    q, k, v = f64(inp["q"]), f64(inp["k"]), f64(inp["v"])
    w_k, w_v = inp["w_k"].astype(np.float64), inp["w_v"].astype(np.float64)
    np.testing.assert_allclose(bw.compress_f64(p, k, w_k), kc64, rtol=0, atol=1e-12)
    np.testing.assert_allclose(bw.compress_f64(p, v, w_v), vc64, rtol=0, atol=1e-12)
    f = bw.forward_fixed(p, q, k, v, inp["gates"].astype(np.float64), w_k, w_v, r["sel"],
                         kc=f64(kcb), vc=f64(vcb))
    for name in ("o_cmp", "o_slc", "o_win", "out"):
        np.testing.assert_allclose(f[name], r[name], rtol=0, atol=1e-12, err_msg=name)


@pytest.mark.parametrize("geom", [
    # D, Hq, Hkv, l, d, l', n, w, T
    (4, 4, 2, 3, 3, 3, 2, 4, 13),
    (4, 4, 1, 4, 2, 4, 2, 5, 14),  # overlapping compression (d < l)
])
def test_gradients_match_central_differences(geom):
    D, Hq, Hkv, l, d, ls, n, w, T = geom
    p = OracleParams(D, Hq, Hkv, l, d, ls, n, w)
    c = _random_case(p, T, seed=sum(geom))
    g = bw.backward(p, c["q"], c["k"], c["v"], c["gates"], c["w_k"], c["w_v"], c["sel"], c["dout"])
    rng = np.random.default_rng(7)
    eps = 1e-6
    for name, grad in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("gates", "dgates"),
                       ("w_k", "dw_k"), ("w_v", "dw_v")):
        x = c[name]
        flat = rng.choice(x.size, size=min(x.size, 48), replace=False)
        for idx in flat:
            pos = np.unravel_index(idx, x.shape)
            xp, xm = x.copy(), x.copy()
            xp[pos] += eps
            xm[pos] -= eps
            fd = (_loss(p, c, **{name: xp}) - _loss(p, c, **{name: xm})) / (2 * eps)
            an = g[grad][pos]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, pos, fd, an)


def _torch_dense_grads(q, k, v, dout, G):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    qt = torch.tensor(q.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(v.transpose(1, 0, 2), dtype=torch.float64, requires_grad=True)
    o = F.scaled_dot_product_attention(qt, kt.repeat_interleave(G, dim=0),
                                       vt.repeat_interleave(G, dim=0), is_causal=True,
                                       scale=1.0 / np.sqrt(q.shape[2]))
    (o * torch.tensor(dout.transpose(1, 0, 2), dtype=torch.float64)).sum().backward()
    return (qt.grad.numpy().transpose(1, 0, 2), kt.grad.numpy().transpose(1, 0, 2),
            vt.grad.numpy().transpose(1, 0, 2))


@pytest.mark.parametrize("branch", [1, 2])  # selected, window
def test_dense_reduction_gradients_equal_causal_attention_autograd(branch):
    D, Hq, Hkv, ls, T = 8, 4, 2, 4, 20
    n = -(-T // ls)  # every block, the incomplete one included
    p = OracleParams(D, Hq, Hkv, 4, 4, ls, n, T)
    c = _random_case(p, T, seed=30 + branch)
    for t in range(T):
        c["sel"][t, :, :] = -1
        c["sel"][t, :, :t // ls + 1] = np.arange(t // ls + 1)
    c["gates"][:] = 0.0
    c["gates"][:, :, branch] = 1.0
    g = bw.backward(p, c["q"], c["k"], c["v"], c["gates"], c["w_k"], c["w_v"], c["sel"], c["dout"])
    dq, dk, dv = _torch_dense_grads(c["q"], c["k"], c["v"], c["dout"], Hq // Hkv)
    np.testing.assert_allclose(g["dq"], dq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dk"], dk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dv"], dv, rtol=0, atol=1e-12)
    assert not g["dw_k"].any() and not g["dw_v"].any()


def test_identity_compressor_gradients_equal_causal_attention_autograd():
    D, Hq, Hkv, T = 8, 4, 2, 18
    p = OracleParams(D, Hq, Hkv, 1, 1, 1, 2, 3)
    c = _random_case(p, T, seed=44)
    c["w_k"] = np.broadcast_to(np.eye(D), (Hkv, D, D)).copy()
    c["w_v"] = c["w_k"].copy()
    c["gates"][:] = 0.0
    c["gates"][:, :, 0] = 1.0
    g = bw.backward(p, c["q"], c["k"], c["v"], c["gates"], c["w_k"], c["w_v"], c["sel"], c["dout"])
    dq, dk, dv = _torch_dense_grads(c["q"], c["k"], c["v"], c["dout"], Hq // Hkv)
    np.testing.assert_allclose(g["dq"], dq, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dk"], dk, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dv"], dv, rtol=0, atol=1e-12)


def test_rows_touching_a_key_range_give_its_exact_gradients():
    D, Hq, Hkv, l, d, ls, n, w, T = 4, 4, 2, 4, 2, 4, 2, 5, 30
    p = OracleParams(D, Hq, Hkv, l, d, ls, n, w)
    c = _random_case(p, T, seed=91)
    args = (p, c["q"], c["k"], c["v"], c["gates"], c["w_k"], c["w_v"], c["sel"], c["dout"])
    full = bw.backward(*args)
    for lo, hi in ((8, 12), (0, 4), (26, 30)):
        rows = bw.rows_touching_keys(p, c["sel"], T, lo, hi)
        assert len(rows) > 0 and rows.min() >= lo  # causal: no earlier row reads the range
        part = bw.backward(*args, rows=rows)
        np.testing.assert_allclose(part["dk"][lo:hi], full["dk"][lo:hi], rtol=0, atol=1e-13)
        np.testing.assert_allclose(part["dv"][lo:hi], full["dv"][lo:hi], rtol=0, atol=1e-13)
        np.testing.assert_allclose(part["dq"][rows], full["dq"][rows], rtol=0, atol=1e-13)
        # leaving out one row of the set changes the range's gradients (dv:
        # a row attending one key alone has p = 1 and adds nothing to dk)
        fewer = bw.backward(*args, rows=rows[1:])
        assert not np.allclose(fewer["dv"][lo:hi], full["dv"][lo:hi], rtol=0, atol=1e-13)


@pytest.mark.parametrize("geom", [
    # D, Hq, Hkv, l, d, l', n, w, T
    (8, 8, 2, 4, 4, 4, 3, 7, 40),
    (8, 4, 1, 4, 2, 8, 2, 9, 37),  # d < l and l' = 2 l
])
def test_c_backward_equals_the_numpy_backward(geom):
    D, Hq, Hkv, l, d, ls, n, w, T = geom
    p = OracleParams(D, Hq, Hkv, l, d, ls, n, w)
    c = _random_case(p, T, seed=200 + T)
    args = (p, c["q"], c["k"], c["v"], c["gates"], c["w_k"], c["w_v"], c["sel"], c["dout"])
    C = bw.num_blocks(p, T)
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((C, Hkv, D))
    vc = rng.standard_normal((C, Hkv, D))
    rows = bw.rows_touching_keys(p, c["sel"], T, 12, 20)
    for extra in ({}, {"kc": kc, "vc": vc}, {"rows": rows}):
        a = bw.backward(*args, **extra)
        b = oracle.backward_c(*args, **extra)
        for name in ("dq", "dk", "dv", "dgates", "dw_k", "dw_v", "dkc", "dvc"):
            np.testing.assert_allclose(b[name], a[name], rtol=0, atol=1e-12,
                                       err_msg=f"{name} {sorted(extra)}")

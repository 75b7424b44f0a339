"""fp64 backward pass of the NSA forward, with the block selection held fixed.

Test infrastructure only: see the package docstring.

The pages name training as a use of the method ("DeepSeek NSA ... config.toml"
page, section 1, on end-to-end trainable sparsity and faster backward
passes; "DeepSeek NSA in manufacturing" page, on training with the method)
but give no gradient formulas.  The readings taken here:

  - the forward is the oracle's definition (three branches, gate combine;
    ``nsa_oracle.c`` states it step by step), evaluated in fp64 on the given
    values;
  - the top-n selection is a discrete choice: the gradient is that of the
    forward with the chosen blocks held fixed (no gradient through the block
    scores or their ranking);
  - the bf16 rounding of the compressed keys and values is taken as the
    identity (the gradient reaches the compressor weights and the raw keys
    and values through the linear map as if the stored tensor were exact);
  - an empty branch has output 0 and passes no gradient.

Everything is written as plain loops over (token, query head) with numpy
vector operations over one row's keys, slow and direct: step 1 is
K~[i, g] = W[g] vec(K[i d : i d + l, g]) (vec index = token p * D + channel c);
each branch is softmax(s q . k_u) over its key set and the weighted sum of
the values; out = g_cmp O_cmp + g_slc O_slc + g_win O_win.  The backward of
one branch with upstream gradient dO_b = g_b dO is the chain rule of those
three operations: dp_u = v_u . dO_b, dz_u = p_u (dp_u - sum_u' p_u' dp_u'),
dq += s sum_u dz_u k_u, dk_u += s dz_u q, dv_u += p_u dO_b; the gate
gradient is dO . O_b; the compressor's gradients are dW[g] += dK~[i, g]
vec(block)^T and d vec(block) += W[g]^T dK~[i, g].
"""
from __future__ import annotations

import math

import numpy as np


def _geometry(p):
    scale = p.scale if p.scale > 0 else 1.0 / math.sqrt(p.head_dim)
    return (p.head_dim, p.num_q_heads, p.num_kv_heads, p.cmp_block, p.cmp_stride, p.sel_block,
            p.window, scale)


def num_blocks(p, T: int) -> int:
    """Complete compressed blocks of a sequence of T tokens: floor((T - l) / d) + 1."""
    return (T - p.cmp_block) // p.cmp_stride + 1 if T >= p.cmp_block else 0


def compress_f64(p, x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Step 1 in fp64 without rounding: x [T,Hkv,D], w [Hkv,D,l*D] -> [C,Hkv,D]."""
    D, _, Hkv, l, d, _, _, _ = _geometry(p)
    C = num_blocks(p, x.shape[0])
    out = np.zeros((C, Hkv, D))
    for i in range(C):
        for g in range(Hkv):
            out[i, g] = w[g] @ x[i * d:i * d + l, g, :].reshape(l * D)
    return out


def _key_sets(p, t: int, sel_tg, C: int):
    """Key positions of the three branches for query t and one KV group:
    compressed blocks i with i d + l - 1 <= t; tokens u <= t of the chosen
    selection blocks (l' tokens each); the w tokens ending at t."""
    _, _, _, l, d, ls, w, _ = _geometry(p)
    cmp = [i for i in range(C) if i * d + l - 1 <= t]
    slc = sorted(u for j in sel_tg if j >= 0 for u in range(j * ls, j * ls + ls) if u <= t)
    win = list(range(max(0, t - w + 1), t + 1))
    return cmp, slc, win


def _attend(qv, keys, vals, scale):
    """softmax(scale q . k) over the rows of `keys`, then the weighted sum of
    `vals`; (probabilities, output); an empty key set gives output 0."""
    if keys.shape[0] == 0:
        return np.zeros(0), np.zeros(vals.shape[1] if vals.ndim == 2 else qv.shape[0])
    z = scale * (keys @ qv)
    e = np.exp(z - z.max())
    pr = e / e.sum()
    return pr, pr @ vals


def forward_fixed(p, q, k, v, gates, w_k, w_v, sel, kc=None, vc=None) -> dict:
    """fp64 forward of one sequence with the selection `sel` [T,Hkv,n]
    (-1 padded) held fixed.  q [T,Hq,D], k/v [T,Hkv,D], gates [T,Hq,3],
    w_k/w_v [Hkv,D,l*D], all taken as fp64 values.  kc/vc [C,Hkv,D]: the
    compressed keys and values to attend to (default: step 1 in fp64).
    Returns out, o_cmp, o_slc, o_win [T,Hq,D] and the kc, vc used."""
    D, Hq, Hkv, _, _, _, _, scale = _geometry(p)
    T = q.shape[0]
    G = Hq // Hkv
    kc = compress_f64(p, k, w_k) if kc is None else np.asarray(kc, dtype=np.float64)
    vc = compress_f64(p, v, w_v) if vc is None else np.asarray(vc, dtype=np.float64)
    C = kc.shape[0]
    res = {name: np.zeros((T, Hq, D)) for name in ("o_cmp", "o_slc", "o_win", "out")}
    for t in range(T):
        for h in range(Hq):
            g = h // G
            cmp, slc, win = _key_sets(p, t, sel[t, g], C)
            _, oc = _attend(q[t, h], kc[cmp, g], vc[cmp, g], scale)
            _, os_ = _attend(q[t, h], k[slc, g], v[slc, g], scale)
            _, ow = _attend(q[t, h], k[win, g], v[win, g], scale)
            res["o_cmp"][t, h], res["o_slc"][t, h], res["o_win"][t, h] = oc, os_, ow
            res["out"][t, h] = gates[t, h, 0] * oc + gates[t, h, 1] * os_ + gates[t, h, 2] * ow
    res["kc"], res["vc"] = kc, vc
    return res


def _branch_backward(qv, keys, vals, dob, scale):
    """Gradients (dq, dkeys, dvals) of one branch's output O = softmax(scale
    K q) V for the upstream gradient `dob`."""
    pr, _ = _attend(qv, keys, vals, scale)
    if pr.size == 0:
        return np.zeros_like(qv), np.zeros_like(keys), np.zeros_like(vals)
    dp = vals @ dob
    dz = pr * (dp - pr @ dp)
    return scale * (dz @ keys), scale * np.outer(dz, qv), np.outer(pr, dob)


def rows_touching_keys(p, sel, T: int, key_lo: int, key_hi: int) -> np.ndarray:
    """Query rows t (ascending) of a sequence of T tokens whose forward reads
    any key or value token in [key_lo, key_hi) through any branch and any KV
    group: the window, a chosen block, or a visible compressed block whose
    tokens overlap the range.  The gradients reaching those tokens come from
    these rows only."""
    _, _, Hkv, _, _, _, _, _ = _geometry(p)
    C = num_blocks(p, T)
    l, d = p.cmp_block, p.cmp_stride
    out = []
    for t in range(T):
        hit = False
        for g in range(Hkv):
            cmp, slc, win = _key_sets(p, t, sel[t, g], C)
            if (any(key_lo <= u < key_hi for u in slc) or any(key_lo <= u < key_hi for u in win)
                    or any(i * d < key_hi and key_lo < i * d + l for i in cmp)):
                hit = True
                break
        if hit:
            out.append(t)
    return np.asarray(out, dtype=np.int64)


def backward(p, q, k, v, gates, w_k, w_v, sel, dout, kc=None, vc=None, rows=None) -> dict:
    """Gradients of sum(dout * out) for the forward of ``forward_fixed`` (same
    arguments).  Returns dq [T,Hq,D], dk, dv [T,Hkv,D], dgates [T,Hq,3],
    dw_k, dw_v [Hkv,D,l*D] and dkc, dvc [C,Hkv,D] (the gradients reaching the
    compressed keys and values).  rows: the query rows whose terms are
    summed (default all): dq and dgates are exact on those rows, and dk, dv
    are exact on every token that only those rows read (see
    ``rows_touching_keys``); everything else holds partial sums."""
    D, Hq, Hkv, l, d, _, _, scale = _geometry(p)
    T = q.shape[0]
    G = Hq // Hkv
    fwd = forward_fixed(p, q, k, v, gates, w_k, w_v, sel, kc, vc)
    kc, vc = fwd["kc"], fwd["vc"]
    C = kc.shape[0]
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    dkc = np.zeros(kc.shape)
    dvc = np.zeros(vc.shape)
    dgates = np.zeros(gates.shape)
    for t in (range(T) if rows is None else rows):
        for h in range(Hq):
            g = h // G
            cmp, slc, win = _key_sets(p, t, sel[t, g], C)
            do = dout[t, h]
            dgates[t, h, 0] = do @ fwd["o_cmp"][t, h]
            dgates[t, h, 1] = do @ fwd["o_slc"][t, h]
            dgates[t, h, 2] = do @ fwd["o_win"][t, h]
            gq, gk, gv = _branch_backward(q[t, h], kc[cmp, g], vc[cmp, g], gates[t, h, 0] * do, scale)
            dq[t, h] += gq
            for a, i in enumerate(cmp):
                dkc[i, g] += gk[a]
                dvc[i, g] += gv[a]
            for keys_of, gate in ((slc, gates[t, h, 1]), (win, gates[t, h, 2])):
                gq, gk, gv = _branch_backward(q[t, h], k[keys_of, g], v[keys_of, g], gate * do, scale)
                dq[t, h] += gq
                for a, u in enumerate(keys_of):
                    dk[u, g] += gk[a]
                    dv[u, g] += gv[a]
    # step 1: K~[i, g] = W[g] vec(x[i d : i d + l, g])
    dw_k = np.zeros(np.shape(w_k))
    dw_v = np.zeros(np.shape(w_v))
    for i in range(C):
        for g in range(Hkv):
            for x, dx, w, dw, dc in ((k, dk, w_k, dw_k, dkc), (v, dv, w_v, dw_v, dvc)):
                blk = x[i * d:i * d + l, g, :].reshape(l * D)
                dw[g] += np.outer(dc[i, g], blk)
                dx[i * d:i * d + l, g, :] += (np.asarray(w[g]).T @ dc[i, g]).reshape(l, D)
    return {"dq": dq, "dk": dk, "dv": dv, "dgates": dgates, "dw_k": dw_k, "dw_v": dw_v,
            "dkc": dkc, "dvc": dvc}

"""Independent dense-mask statement of the NSA forward pass (tests only).

The oracle (oracle/nsa_oracle.c) walks each query row and gathers the key
rows of each branch.  This module states the same definition the other way
round: full [T, T] (or [T, C]) logit matrices, boolean masks for the three
branches, a masked row softmax and numpy's lexsort for the block ranking.  A
wrong block range, window bound, causality test, score sum or tie order in
either statement makes the two disagree.  Used only on tiny inputs.
"""
import numpy as np


def bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def masked_softmax(z, mask):
    """Row softmax of z over mask; rows without any True give all-zero rows."""
    if z.shape[-1] == 0:
        return np.zeros_like(z)
    z = np.where(mask, z, -np.inf)
    m = np.max(z, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(z - m), 0.0)
    s = e.sum(axis=-1, keepdims=True)
    return np.divide(e, s, out=np.zeros_like(e), where=s > 0)


def nsa_dense(q, k, v, kc, vc, gates, D, Hq, Hkv, l, n, w, scale=None, d=None, lsel=None):
    """q [T,Hq,D], k/v [T,Hkv,D], kc/vc [C,Hkv,D] (float64), gates [T,Hq,3].
    Block geometry: compression block l, stride d (default l), selection
    block lsel (default l).  Returns dict of [T,Hq,D] arrays plus scores
    [T,Hkv,J] (selection-block scores, J = T // lsel + 1) and sel (per-(t,g)
    index arrays)."""
    d = l if d is None else d
    lsel = l if lsel is None else lsel
    T = q.shape[0]
    C = kc.shape[0]
    G = Hq // Hkv
    J = T // lsel + 1
    s = 1.0 / np.sqrt(D) if scale is None else scale
    tt = np.arange(T)[:, None]
    uu = np.arange(T)[None, :]
    ii = np.arange(C)[None, :]
    cmp_mask = (ii * d + l - 1) <= tt                       # [T, C]
    win_mask = (uu <= tt) & (uu > tt - w)                   # [T, T]
    # overlap[i, j]: compressed block i (tokens [i d, i d + l)) meets
    # selection block j (tokens [j lsel, (j + 1) lsel))
    ci = np.arange(C)[:, None]
    jj = np.arange(J)[None, :]
    overlap = ((ci * d) < (jj + 1) * lsel) & ((ci * d + l) > jj * lsel)
    out = {key: np.zeros((T, Hq, D)) for key in ("o_cmp", "o_slc", "o_win", "out")}
    scores = np.zeros((T, Hkv, J))
    sel = {}
    for g in range(Hkv):
        P = []
        for hh in range(G):
            h = g * G + hh
            z = s * q[:, h, :] @ kc[:, g, :].T
            p = masked_softmax(z, cmp_mask)
            P.append(p)
            out["o_cmp"][:, h, :] = p @ vc[:, g, :]
        S = np.sum(P, axis=0) @ overlap.astype(np.float64)   # [T, J]
        scores[:, g, :] = S
        slc_mask = np.zeros((T, T), dtype=bool)
        for t in range(T):
            ncand = t // lsel + 1
            cand = S[t, :ncand]
            order = np.lexsort((np.arange(ncand), -cand))     # score desc, index asc
            chosen = np.sort(order[:n])
            sel[(t, g)] = chosen
            for j in chosen:
                slc_mask[t, j * lsel:(j + 1) * lsel] = True
        slc_mask &= (uu <= tt)
        for hh in range(G):
            h = g * G + hh
            z = s * q[:, h, :] @ k[:, g, :].T
            out["o_slc"][:, h, :] = masked_softmax(z, slc_mask) @ v[:, g, :]
            out["o_win"][:, h, :] = masked_softmax(z, win_mask) @ v[:, g, :]
    out["out"] = (gates[..., 0:1] * out["o_cmp"] + gates[..., 1:2] * out["o_slc"]
                  + gates[..., 2:3] * out["o_win"])
    out["scores"] = scores
    out["sel"] = sel
    return out

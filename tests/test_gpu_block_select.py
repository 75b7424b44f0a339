"""GPU parity of select-only block attention (nsa_block_select_prefill, MoBA
style: "NSA vs MoBA" page, section 1) against the fp64 oracle.

Stages, as for the NSA branch:
  - routing keys: the mean keys are bit-exact (both sides sum in fp64 and
    round once to bf16);
  - stage A: the oracle's selection replayed on the GPU's own fp32 routing
    scores must give the GPU's attended blocks bit for bit;
  - stage B: the oracle over the GPU's routing keys: scores within the fp32
    accumulation bound, equal block sets except where the oracle's gap
    between the (n-1)-th and n-th score is below twice that bound, and the
    outputs of the rows with equal sets within the output tolerance.
"""
import numpy as np
import pytest

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import nsa
from sparse_attention_long_06_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# |GPU fp32 routing score - fp64 score|: sums of G * D exact bf16 products
# accumulated in fp32 by the tensor cores.  Observed at most 6.9e-6 over the
# configurations below (scores of magnitude up to about 30); the bound keeps
# a margin of about 15x.
SCORE_TOL = 1e-4


def run_block_select(cfg, inputs, out_dtype=nsa.OUT_F32, max_seqlen=None):
    import torch
    lens = inputs["seqlens"]
    total = int(inputs["cu_seqlens"][-1])
    max_seqlen = max_seqlen or max(max(lens), cfg.sel_block)
    D, Hq, Hkv, n = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.top_n
    dev = {k: gu.to_dev(inputs[k]) for k in ("q", "k", "v", "cu_seqlens")}
    plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max_seqlen,
                               max_total_tokens=total, out_dtype=out_dtype)
    rows = max(plan.block_rows(total), 1)
    out = torch.empty((max(total, 1), Hq, D),
                      dtype=torch.float32 if out_dtype == nsa.OUT_F32 else torch.int16, device="cuda")
    km = torch.full((rows, Hkv, D), 0x7F7F, dtype=torch.int16, device="cuda")
    sel = torch.full((max(total, 1), Hkv, n), -7, dtype=torch.int32, device="cuda")
    ws = plan.alloc_workspace(nsa.MODE_BLOCK_SELECT)
    plan.block_select_prefill(dev["q"], dev["k"], dev["v"], dev["cu_seqlens"], out, km, ws,
                              sel_idx=sel)
    status = nsa.read_device_status(ws)
    res = {"status": status, "launches": nsa.last_launch_count(), "km": gu.bits(km),
           "sel": sel.cpu().numpy(), "total": total}
    if out_dtype == nsa.OUT_F32:
        res["out"] = out.cpu().numpy().astype(np.float64)
    else:
        res["out_bits"] = gu.bits(out)
        res["out"] = wl.bf16_to_f32(res["out_bits"]).astype(np.float64)
    off, _ = plan.workspace_region(nsa.WS_SCORES, nsa.MODE_BLOCK_SELECT)
    cap = max(1, max_seqlen // cfg.sel_block)
    wsn = ws.cpu().numpy()
    cnt = total * Hkv * cap
    res["scores"] = wsn[off:off + cnt * 4].view(np.float32).reshape(total, Hkv, cap).copy()
    res["cap"] = cap
    return res


def check_block_select(cfg, inputs, res, rows_per_seq):
    """Returns a report dict; asserts every stage."""
    p = OracleParams.of(cfg)
    ls, n, Hkv = cfg.sel_block, cfg.top_n, cfg.num_kv_heads
    cu = inputs["cu_seqlens"]
    assert res["status"] == nsa.NSA_OK
    boff = 0
    rep = {"rows": 0, "stage_a_rows": 0, "score_max_err": 0.0, "idx_mismatch": 0,
           "idx_near_tie": 0, "max_abs": 0.0}
    num = den = 0.0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        T = e - s
        nb = T // ls
        _, kb16 = oracle.block_means(p, inputs["k"][s:e])
        np.testing.assert_array_equal(res["km"][boff:boff + nb], kb16)
        gpu_kb = res["km"][boff:boff + nb]
        boff += nb
        rows = np.asarray(rows_per_seq[b], dtype=np.int32)
        if len(rows) == 0:
            continue
        gsel = res["sel"][s + rows]                         # [R, Hkv, n]
        cur = rows // ls
        # stage A: replay on the GPU's scores
        if n > 1:
            for g in range(Hkv):
                sc = res["scores"][s + rows, g, :]
                chosen, _ = oracle.select_f32(sc, cur, cur, n - 1)
                taken = np.minimum(cur, n - 1)
                exp = np.full((len(rows), n), -1, dtype=np.int32)
                exp[:, :n - 1] = chosen
                exp[np.arange(len(rows)), taken] = cur
                np.testing.assert_array_equal(gsel[:, g, :], exp)
        else:
            assert (gsel[:, :, 0] == cur[:, None]).all()
        rep["stage_a_rows"] += len(rows)
        # stage B: the oracle on the GPU's routing keys
        r = oracle.block_select_rows(p, inputs["q"][s:e], inputs["k"][s:e], inputs["v"][s:e],
                                     gpu_kb if nb else np.zeros((1, Hkv, cfg.head_dim), np.uint16),
                                     rows, cmax=res["cap"])
        for i, t in enumerate(rows):
            c = int(t) // ls
            if c:
                err = np.abs(res["scores"][s + t, :, :c].astype(np.float64) - r["scores"][i, :, :c])
                rep["score_max_err"] = max(rep["score_max_err"], float(err.max()))
        same = np.all(r["sel"] == gsel, axis=2)              # [R, Hkv]
        near = r["gap"] < 2 * SCORE_TOL
        rep["idx_mismatch"] += int(np.count_nonzero(~same & ~near))
        rep["idx_near_tie"] += int(np.count_nonzero(~same & near))
        ok_rows = np.all(same, axis=1)
        got = res["out"][s + rows][ok_rows]
        ref = r["out"][ok_rows]
        if got.size:
            diff = np.abs(got - ref)
            rep["max_abs"] = max(rep["max_abs"], float(diff.max()))
            num += float(np.sum(diff ** 2))
            den += float(np.sum(ref ** 2))
        rep["rows"] += len(rows)
    rep["rel_l2"] = (num / den) ** 0.5 if den > 0 else 0.0
    gu.log_report(f"block_select:{cfg.name}", rep)
    assert rep["score_max_err"] <= SCORE_TOL, rep
    assert rep["idx_mismatch"] == 0, rep
    assert rep["max_abs"] <= 1e-2 and rep["rel_l2"] <= 5e-3, rep
    return rep


def _cfg(name, seed, D, Hq, Hkv, ls, n):
    return wl.NsaConfig(name, seed, D, Hq, Hkv, ls, ls, ls, n, 1)


@pytest.mark.parametrize("case", [
    # name, D, Hq, Hkv, l', n, lengths
    ("bs_small", 64, 4, 2, 32, 4, [1, 31, 32, 33, 100, 300, 700]),
    ("bs_g16", 128, 64, 4, 64, 16, [5000, 64, 1500]),
    ("bs_g1", 64, 8, 8, 64, 8, [3000, 65]),
    ("bs_own_block_only", 64, 16, 2, 32, 1, [400, 129]),
    ("bs_g8_l32", 128, 32, 4, 32, 12, [2100]),
])
def test_block_select_geometries(case):
    name, D, Hq, Hkv, ls, n, lens = case
    cfg = _cfg(name, 41, D, Hq, Hkv, ls, n)
    inp = wl.prefill_inputs(cfg, seqlens=lens)
    res = run_block_select(cfg, inp)
    assert res["launches"] == 5
    rows = [np.arange(T) if T <= 800 else gu.sample_rows(T, 160, 7 + b, 128 // cfg.group, ls)
            for b, T in enumerate(lens)]
    check_block_select(cfg, inp, res, rows)


def test_block_select_8k_and_bf16_output():
    base = wl.CONFIGS["prefill_8k"]
    inp = wl.prefill_inputs(base)
    res = run_block_select(base, inp)
    rows = [gu.sample_rows(8192, 384, 11, 8, 64)]
    check_block_select(base, inp, res, rows)
    rb = run_block_select(base, inp, out_dtype=nsa.OUT_BF16)
    assert rb["status"] == nsa.NSA_OK
    np.testing.assert_array_equal(rb["out_bits"], wl.bf16_bits(res["out"].astype(np.float32)))
    np.testing.assert_array_equal(rb["sel"], res["sel"])


def test_block_select_64k_sampled_rows():
    base = wl.CONFIGS["prefill_64k"]
    inp = wl.prefill_inputs(base)
    res = run_block_select(base, inp)
    T = 65536
    rows = np.unique(np.concatenate([np.arange(0, T, 64)[::4], gu.sample_rows(T, 256, 12, 8, 64)]))
    check_block_select(base, inp, res, [rows.astype(np.int32)])


def test_block_select_many_candidates_and_exact_ties():
    # l' = 32 over 40000 tokens: rows near the end rank more than 1024 blocks
    # (the radix path of the top-n kernel); keys repeating every 3 blocks give
    # bit-identical routing keys, hence exact score ties, which go to the
    # lower block
    cfg = _cfg("bs_ties", 43, 128, 64, 4, 32, 16)
    inp = wl.make_keys_periodic(cfg, wl.prefill_inputs(cfg, seqlens=[40000]), 3)
    res = run_block_select(cfg, inp)
    rows = np.unique(np.concatenate([np.arange(39000, 40000, 7), [32799, 32800, 32831, 32832]]))
    rep = check_block_select(cfg, inp, res, [rows.astype(np.int32)])
    assert rep["idx_mismatch"] == 0
    # the blocks of one residue class (mod 3) share their score: the 15
    # attended besides the own block are the lowest 15 of the best class
    s = res["sel"][int(rows[-1])]
    own = int(rows[-1]) // 32
    for g in range(4):
        picked = [int(j) for j in s[g] if j >= 0 and j != own]
        assert len(picked) == 15
        assert picked[0] < 3 and picked == list(range(picked[0], picked[0] + 45, 3))


def test_block_select_empty_call_is_a_no_op():
    import torch
    cfg = _cfg("bs_empty", 1, 64, 4, 2, 32, 4)
    plan = nsa.Plan.for_config(cfg, max_batch=2, max_seqlen=256, max_total_tokens=0)
    ws = plan.alloc_workspace(nsa.MODE_BLOCK_SELECT)
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    e = torch.empty((0, 4, 64), dtype=torch.int16, device="cuda")
    plan.block_select_prefill(e, e, e, cu, e, None, ws)
    assert nsa.last_launch_count() == 0
    assert nsa.read_device_status(ws) == nsa.NSA_OK


def test_block_select_rejects_inconsistent_seqlens_on_device():
    cfg = _cfg("bs_bad", 2, 64, 4, 2, 32, 4)
    inp = wl.prefill_inputs(cfg, seqlens=[100, 50])
    bad = dict(inp)
    bad["cu_seqlens"] = np.array([0, 120, 150], dtype=np.int32)  # 120 > max_seqlen 100
    res = run_block_select(cfg, bad, max_seqlen=100)
    assert res["status"] == nsa.NSA_ERR_DEVICE_BAD_INPUT


# ---------------------------------------------------------------- decode
def _mean_cache(p, inp, cap):
    """Routing keys of the blocks complete before each sequence's newest
    token (the state earlier steps leave), from the oracle; other rows hold a
    sentinel."""
    B = len(inp["seqlens"])
    ls = p.sel_block
    km = np.full((B, cap // ls, p.num_kv_heads, p.head_dim), 0x7F7F, dtype=np.uint16)
    for b, L in enumerate(inp["seqlens"]):
        nb = (int(L) - 1) // ls
        if nb:
            _, kb = oracle.block_means(p, inp["k"][b][:nb * ls])
            km[b, :nb] = kb
    return km


def run_block_select_decode(cfg, inp, km, out_dtype=nsa.OUT_F32):
    import torch
    B = len(inp["seqlens"])
    cap = int(inp["capacity"])
    plan = nsa.Plan.for_config(cfg, max_batch=B, max_seqlen=cap, out_dtype=out_dtype)
    d = {k: gu.to_dev(inp[k]) for k in ("q", "k", "v", "seqlens")}
    kmd = gu.to_dev(km)
    out = torch.empty((B, cfg.num_q_heads, cfg.head_dim),
                      dtype=torch.float32 if out_dtype == nsa.OUT_F32 else torch.int16, device="cuda")
    sel = torch.full((B, cfg.num_kv_heads, cfg.top_n), -7, dtype=torch.int32, device="cuda")
    ws = plan.alloc_workspace(nsa.MODE_BLOCK_SELECT_DECODE)
    plan.block_select_decode(d["q"], d["k"], d["v"], kmd, d["seqlens"], out, ws, sel_idx=sel)
    res = {"status": nsa.read_device_status(ws), "launches": nsa.last_launch_count(),
           "sel": sel.cpu().numpy(), "km": gu.bits(kmd)}
    res["out"] = (out.cpu().numpy().astype(np.float64) if out_dtype == nsa.OUT_F32
                  else wl.bf16_to_f32(gu.bits(out)).astype(np.float64))
    return res


def check_block_select_decode(cfg, inp, km_in, res, seqs):
    p = OracleParams.of(cfg)
    ls = cfg.sel_block
    rep = {"seqs": 0, "idx_mismatch": 0, "idx_near_tie": 0, "max_abs": 0.0}
    num = den = 0.0
    assert res["status"] == nsa.NSA_OK
    for b in seqs:
        L = int(inp["seqlens"][b])
        nb = (L - 1) // ls
        r = oracle.block_select_decode_reference(p, inp["q"][b], inp["k"][b], inp["v"][b],
                                                 km_in[b, :nb], L)
        # the routing key of a block the newest token completes, bit for bit;
        # every other row of the cache untouched
        exp = km_in[b].copy()
        if r["written"] is not None:
            exp[L // ls - 1] = r["written"]
        np.testing.assert_array_equal(res["km"][b], exp)
        same = np.all(r["sel"] == res["sel"][b], axis=1)
        near = r["gap"] < 2 * SCORE_TOL
        rep["idx_mismatch"] += int(np.count_nonzero(~same & ~near))
        rep["idx_near_tie"] += int(np.count_nonzero(~same & near))
        if np.all(same):
            diff = np.abs(res["out"][b] - r["out"])
            rep["max_abs"] = max(rep["max_abs"], float(diff.max()))
            num += float(np.sum(diff ** 2))
            den += float(np.sum(r["out"] ** 2))
        rep["seqs"] += 1
    rep["rel_l2"] = (num / den) ** 0.5 if den > 0 else 0.0
    gu.log_report(f"block_select_decode:{cfg.name}", rep)
    assert rep["idx_mismatch"] == 0, rep
    assert rep["max_abs"] <= 1e-2 and rep["rel_l2"] <= 5e-3, rep
    return rep


@pytest.mark.parametrize("geom", [
    # D, Hq, Hkv, l', n, lengths, capacity
    (64, 4, 1, 32, 4, [1, 31, 32, 33, 100, 640, 1000], 1024),
    (128, 64, 4, 64, 16, [700, 4096, 5000, 63, 64, 9000], 9024),
    (64, 16, 2, 32, 1, [200, 32, 1], 256),
    (128, 32, 4, 32, 12, [2048, 2047, 40000], 40000),
])
def test_block_select_decode_geometries(geom):
    D, Hq, Hkv, ls, n, lens, cap = geom
    cfg = wl.NsaConfig("bsd", 51, D, Hq, Hkv, ls, ls, ls, n, 1, decode_batch=len(lens))
    inp = wl.decode_inputs(cfg, lengths=lens, capacity=cap)
    km = _mean_cache(OracleParams.of(cfg), inp, int(inp["capacity"]))
    res = run_block_select_decode(cfg, inp, km)
    assert res["launches"] == 3
    check_block_select_decode(cfg, inp, km, res, range(len(lens)))


def test_block_select_decode_64k_batch_and_bf16_output():
    cfg = wl.CONFIGS["decode_64k"]
    inp = wl.decode_inputs(cfg)
    km = _mean_cache(OracleParams.of(cfg), inp, int(inp["capacity"]))
    res = run_block_select_decode(cfg, inp, km)
    check_block_select_decode(cfg, inp, km, res, [0, 13, 31])
    rb = run_block_select_decode(cfg, inp, km, out_dtype=nsa.OUT_BF16)
    assert rb["status"] == nsa.NSA_OK
    np.testing.assert_array_equal(rb["sel"], res["sel"])
    np.testing.assert_array_equal(wl.bf16_bits(res["out"].astype(np.float32)),
                                  wl.bf16_bits(rb["out"].astype(np.float32)))


def test_block_select_decode_exact_ties_go_to_the_lower_block():
    # keys repeating every three blocks: equal routing keys, equal scores
    cfg = wl.NsaConfig("bsd_ties", 52, 128, 64, 4, 32, 32, 32, 8, 1, decode_batch=2)
    inp = wl.decode_inputs(cfg, lengths=[3000, 1500], capacity=3008)
    for b, L in enumerate(inp["seqlens"]):
        idx = np.arange(int(L)) % 96
        inp["k"][b][:L] = inp["k"][b][idx]
    km = _mean_cache(OracleParams.of(cfg), inp, int(inp["capacity"]))
    res = run_block_select_decode(cfg, inp, km)
    rep = check_block_select_decode(cfg, inp, km, res, [0, 1])
    assert rep["idx_near_tie"] == 0
    for b, L in enumerate(inp["seqlens"]):
        own = (int(L) - 1) // 32
        for g in range(4):
            picked = [int(j) for j in res["sel"][b, g] if j >= 0 and j != own]
            assert len(picked) == 7 and picked[0] < 3
            assert picked == list(range(picked[0], picked[0] + 21, 3))

"""GPU parity of token-level top-k attention (nsa_token_select_prefill, DSA
style: "DeepSeek V3.2-Exp sparse attention" page, sections 1 and 3) against
the fp64 oracle.

  - stage A: the oracle's selection replayed on the GPU's own fp32 index
    scores reproduces the GPU's chosen tokens bit for bit;
  - stage B: the GPU's index scores within the fp32 accumulation bound of the
    oracle's, the chosen tokens equal the oracle's except where its gap
    between the top_k-th and (top_k+1)-th score is below twice that bound,
    and the outputs of rows with equal sets within max-abs 1e-2 and
    relative L2 5e-3.
"""
import numpy as np
import pytest

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import nsa
from sparse_attention_long_06_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# |GPU fp32 index score - fp64|: sums of the head weights times ReLU of
# Di-term bf16 products accumulated in fp32; scores reach about 100 at
# Di = 128, 16 heads, so the bound is relative.
INDEX_RTOL = 2e-6
INDEX_ATOL = 1e-4


def run_token_select(cfg, inputs, idx, top_k, out_dtype=nsa.OUT_F32):
    import torch
    lens = inputs["seqlens"]
    total = int(inputs["cu_seqlens"][-1])
    max_seqlen = max(max(lens), top_k)
    D, Hq = cfg.head_dim, cfg.num_q_heads
    dev = {k: gu.to_dev(inputs[k]) for k in ("q", "k", "v", "cu_seqlens")}
    dev.update({k: gu.to_dev(idx[k]) for k in ("q_index", "w_index", "k_index")})
    plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max_seqlen,
                               max_total_tokens=total, out_dtype=out_dtype)
    out = torch.empty((total, Hq, D), dtype=torch.float32 if out_dtype == nsa.OUT_F32 else torch.int16,
                      device="cuda")
    sel = torch.full((total, top_k), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(plan.token_select_workspace_size(top_k), dtype=torch.uint8, device="cuda")
    plan.token_select_prefill(dev["q"], dev["k"], dev["v"], dev["q_index"], dev["w_index"],
                              dev["k_index"], top_k, dev["cu_seqlens"], out, ws, sel_idx=sel)
    res = {"status": nsa.read_device_status(ws), "launches": nsa.last_launch_count(),
           "sel": sel.cpu().numpy()}
    res["out"] = (out.cpu().numpy().astype(np.float64) if out_dtype == nsa.OUT_F32
                  else wl.bf16_to_f32(gu.bits(out)).astype(np.float64))
    # index scores: the workspace region after the header and the metadata
    wsn = ws.cpu().numpy()
    meta = 256 + ((16 + 8 * (len(lens) + 1) + 255) // 256) * 256
    stride = (max_seqlen + 3) // 4 * 4  # row stride of the index-score table
    res["index"] = wsn[meta:meta + total * stride * 4].view(np.float32).reshape(total, stride).copy()
    return res


def check_token_select(cfg, inputs, idx, res, top_k, rows_per_seq):
    p = OracleParams.of(cfg)
    cu = inputs["cu_seqlens"]
    assert res["status"] == nsa.NSA_OK
    rep = {"rows": 0, "index_max_err": 0.0, "idx_mismatch": 0, "idx_near_tie": 0, "max_abs": 0.0}
    num = den = 0.0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        rows = np.asarray(rows_per_seq[b], dtype=np.int32)
        if len(rows) == 0:
            continue
        gsel = res["sel"][s + rows]
        # stage A
        sc = res["index"][s + rows, :]
        ncand = (rows + 1).astype(np.int32)
        selA, _ = oracle.select_f32(sc, ncand, ncand, top_k)
        np.testing.assert_array_equal(gsel, selA)
        # stage B
        r = oracle.dsa_rows(p, top_k, inputs["q"][s:e], inputs["k"][s:e], inputs["v"][s:e],
                            idx["q_index"][s:e], idx["w_index"][s:e], idx["k_index"][s:e], rows,
                            with_index=True)
        bound = 0.0
        for i, t in enumerate(rows):
            ref = r["index"][i, :t + 1]
            err = np.abs(res["index"][s + t, :t + 1].astype(np.float64) - ref)
            assert np.all(err <= INDEX_ATOL + INDEX_RTOL * np.abs(ref)), (t, float(err.max()))
            rep["index_max_err"] = max(rep["index_max_err"], float(err.max()))
            bound = max(bound, float(INDEX_ATOL + INDEX_RTOL * np.abs(ref).max()))
        same = np.all(r["sel"] == gsel, axis=1)
        near = r["gap"] < 2 * bound
        rep["idx_mismatch"] += int(np.count_nonzero(~same & ~near))
        rep["idx_near_tie"] += int(np.count_nonzero(~same & near))
        if np.any(same):
            got, ref = res["out"][s + rows][same], r["out"][same]
            diff = np.abs(got - ref)
            rep["max_abs"] = max(rep["max_abs"], float(diff.max()))
            num += float(np.sum(diff ** 2))
            den += float(np.sum(ref ** 2))
        rep["rows"] += len(rows)
    rep["rel_l2"] = (num / den) ** 0.5 if den > 0 else 0.0
    gu.log_report(f"token_select:{cfg.name}:k{top_k}", rep)
    assert rep["idx_mismatch"] == 0, rep
    assert rep["max_abs"] <= 1e-2 and rep["rel_l2"] <= 5e-3, rep
    return rep


def _cfg(name, D, Hq, Hkv):
    return wl.NsaConfig(name, 61, D, Hq, Hkv, 32, 32, 32, 1, 1)


@pytest.mark.parametrize("case", [
    # name, D, Hq, Hkv, indexer heads, indexer dim, top_k, lengths
    ("ts_small", 64, 4, 2, 4, 64, 16, [1, 15, 16, 17, 300, 129]),
    ("ts_g16", 128, 64, 4, 16, 128, 256, [2000, 257]),
    ("ts_g1", 64, 8, 8, 8, 64, 40, [700]),
    ("ts_k1", 128, 16, 2, 1, 128, 1, [333]),
])
def test_token_select_geometries(case):
    name, D, Hq, Hkv, Hi, Di, top_k, lens = case
    cfg = _cfg(name, D, Hq, Hkv)
    inp = wl.prefill_inputs(cfg, seqlens=lens)
    idx = wl.indexer_inputs(lens, Hi, Di, seed=7)
    res = run_token_select(cfg, inp, idx, top_k)
    assert res["launches"] == 4
    rows = [np.arange(T) if T <= 700 else gu.sample_rows(T, 200, 3 + b, 128 // Hi, 32)
            for b, T in enumerate(lens)]
    check_token_select(cfg, inp, idx, res, top_k, rows)


def test_token_select_8k_top2048_and_bf16_output():
    cfg = wl.CONFIGS["prefill_8k"]
    inp = wl.prefill_inputs(cfg)
    idx = wl.indexer_inputs([8192], 16, 128, seed=8)
    res = run_token_select(cfg, inp, idx, 2048)
    rows = [np.unique(np.concatenate([np.arange(0, 8192, 97), [2046, 2047, 2048, 2049, 8191]]))]
    check_token_select(cfg, inp, idx, res, 2048, rows)
    rb = run_token_select(cfg, inp, idx, 2048, out_dtype=nsa.OUT_BF16)
    assert rb["status"] == nsa.NSA_OK
    np.testing.assert_array_equal(rb["sel"], res["sel"])
    np.testing.assert_array_equal(wl.bf16_bits(res["out"].astype(np.float32)),
                                  wl.bf16_bits(rb["out"].astype(np.float32)))


@pytest.mark.parametrize("top_k", [24, 40])  # warp path (top_k <= 32), CTA path
def test_token_select_relu_floor_ties_go_to_the_lowest_tokens(top_k):
    # every indexer product negative: all scores are exactly 0 and the
    # lowest top_k tokens are chosen
    cfg = _cfg("ts_floor", 64, 4, 1)
    lens = [500]
    inp = wl.prefill_inputs(cfg, seqlens=lens)
    idx = wl.indexer_inputs(lens, 4, 64, seed=9)
    idx["q_index"] = wl.bf16_bits(np.abs(wl.bf16_to_f32(idx["q_index"])))
    idx["k_index"] = wl.bf16_bits(-np.abs(wl.bf16_to_f32(idx["k_index"])) - 0.01)
    res = run_token_select(cfg, inp, idx, top_k)
    rep = check_token_select(cfg, inp, idx, res, top_k, [np.arange(500)])
    assert rep["idx_near_tie"] == 0
    assert np.all(res["index"][np.arange(500)[:, None] >= np.arange(500)[None, :]] == 0.0)
    assert (res["sel"][top_k:] == np.arange(top_k)[None, :]).all()


def test_token_select_partial_ties_at_the_threshold():
    # index scores on a coarse grid (many equal values around every row's
    # threshold): the top-k takes the lowest tokens among the equal ones
    cfg = _cfg("ts_grid", 64, 4, 1)
    lens = [1500, 301]
    inp = wl.prefill_inputs(cfg, seqlens=lens)
    idx = wl.indexer_inputs(lens, 1, 64, seed=11)
    rng = np.random.default_rng(12)
    T = sum(lens)
    # one indexer head of weight 1, a query with one unit coordinate and keys
    # of 0..7 on that coordinate: the score of token s is exactly k_s[0]
    qi = np.zeros((T, 1, 64), dtype=np.float32)
    qi[:, 0, 0] = 1.0
    ki = np.zeros((T, 64), dtype=np.float32)
    ki[:, 0] = rng.integers(0, 8, size=T).astype(np.float32)
    idx["q_index"] = wl.bf16_bits(qi)
    idx["k_index"] = wl.bf16_bits(ki)
    idx["w_index"] = np.ones((T, 1), dtype=np.float32)
    for top_k in (33, 200):
        res = run_token_select(cfg, inp, idx, top_k)
        rows = [np.arange(T_b) for T_b in lens]
        rep = check_token_select(cfg, inp, idx, res, top_k, rows)
        assert rep["idx_near_tie"] == 0 and rep["idx_mismatch"] == 0


def test_token_select_rejects_inconsistent_seqlens_on_device():
    cfg = _cfg("ts_bad", 64, 4, 2)
    inp = wl.prefill_inputs(cfg, seqlens=[100, 50])
    idx = wl.indexer_inputs([100, 50], 4, 64, seed=10)
    bad = dict(inp)
    bad["cu_seqlens"] = np.array([0, 120, 150], dtype=np.int32)
    bad["seqlens"] = [100, 16]  # plan max_seqlen 100 < 120
    res = run_token_select(cfg, bad, idx, 16)
    assert res["status"] == nsa.NSA_ERR_DEVICE_BAD_INPUT

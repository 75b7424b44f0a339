"""The work counts behind the bench's roofline fractions (CPU): the
algorithmic FLOPs of NSA, select-only and token-level attention are checked
against per-(token, head) counts of the keys each branch attends to, taken
from the oracle's own selections, and the decode byte count against a closed
form when the selection covers every block."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from oracle import OracleParams  # noqa: E402
from sparse_attention_long_06_b200 import workloads as wl  # noqa: E402


def test_algorithmic_flops_match_a_key_count():
    cfg = wl.NsaConfig("count", 31, 64, 4, 2, 32, 32, 32, 3, 40, seqlens=(200,))
    inp = wl.prefill_inputs(cfg)
    T, D, l, Hkv, G = 200, cfg.head_dim, cfg.cmp_block, cfg.num_kv_heads, cfg.group
    p = OracleParams.of(cfg)
    _, kc = oracle.compress(p, inp["k"], inp["w_k"])
    _, vc = oracle.compress(p, inp["v"], inp["w_v"])
    rows = np.arange(T, dtype=np.int32)
    r = oracle.nsa_rows(p, inp["q"], inp["k"], inp["v"], kc, vc, inp["gates"], rows, cmax=T // l)
    sel = r["sel"]  # [T, Hkv, n], -1 padded
    keys = 0
    for t in range(T):
        cmp_keys = sum(1 for i in range(T // l) if i * l + l - 1 <= t)
        win_keys = sum(1 for u in range(T) if t - cfg.window + 1 <= u <= t)
        for g in range(Hkv):
            slc_keys = sum(1 for b in sel[t, g] if b >= 0 for u in range(b * l, b * l + l) if u <= t)
            keys += G * (cmp_keys + win_keys + slc_keys)
    f = bench.algorithmic_flops(cfg, T, sel)
    assert f["cmp"] + f["slc"] + f["win"] == 4 * D * keys
    assert f["compress"] == 4 * (T // l) * Hkv * l * D * D
    assert f["total"] == f["cmp"] + f["slc"] + f["win"] + f["compress"]


def test_decode_bytes_closed_form_when_every_block_is_selected():
    cfg = wl.NsaConfig("dec", 32, 64, 4, 2, 32, 32, 32, 16, 64, decode_batch=2, decode_len=300)
    lens = [300, 97]
    D, Hq, Hkv, l = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.cmp_block
    n = cfg.top_n
    sel = np.full((2, Hkv, n), -1, dtype=np.int32)
    for b, L in enumerate(lens):
        nb = (L - 1) // l + 1  # every candidate block, the incomplete one included
        sel[b, :, :nb] = np.arange(nb)
    got = bench.decode_bytes(cfg, lens, sel)
    want = 0
    for L in lens:
        # every cached token is read once (window and blocks overlap), plus the
        # complete compressed blocks, per group; q, gates and out per sequence
        want += Hkv * ((L // l) * D * 2 * 2 + L * D * 2 * 2) + Hq * D * 2 + Hq * 3 * 4 + Hq * D * 2
    assert got == want


def test_block_select_flops_match_a_key_count():
    cfg = wl.NsaConfig("bscount", 33, 64, 4, 2, 32, 32, 32, 3, 40, seqlens=(150, 77))
    inp = wl.prefill_inputs(cfg)
    D, G, ls, Hkv = cfg.head_dim, cfg.group, cfg.sel_block, cfg.num_kv_heads
    p = OracleParams.of(cfg)
    res = oracle.block_select_reference(p, inp)
    route = keys = 0
    for r, T in zip(res, cfg.seqlens):
        for t in range(T):
            route += G * Hkv * (t // ls)  # complete blocks before t's own block
            for g in range(Hkv):
                for blk in r["sel"][t, g]:
                    if blk >= 0:
                        keys += G * sum(1 for u in range(blk * ls, blk * ls + ls) if u <= t)
    sel = np.concatenate([r["sel"] for r in res])
    f = bench.block_select_flops(cfg, list(cfg.seqlens), sel)
    assert f["route"] == 2 * D * route
    assert f["attn"] == 4 * D * keys
    assert f["total"] == f["route"] + f["attn"]


def test_token_select_work_matches_a_key_count():
    cfg = wl.NsaConfig("tscount", 34, 64, 4, 2, 32, 32, 32, 3, 40, seqlens=(90, 41))
    lens = list(cfg.seqlens)
    inp = wl.prefill_inputs(cfg)
    Hi, Di, top_k = 2, 64, 20
    idx = wl.indexer_inputs(lens, Hi, Di, seed=5)
    p = OracleParams.of(cfg)
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    cu = inp["cu_seqlens"]
    index = chosen = 0
    for b, T in enumerate(lens):
        s, e = int(cu[b]), int(cu[b + 1])
        r = oracle.dsa_rows(p, top_k, inp["q"][s:e], inp["k"][s:e], inp["v"][s:e],
                            idx["q_index"][s:e], idx["w_index"][s:e], idx["k_index"][s:e],
                            np.arange(T, dtype=np.int32))
        for t in range(T):
            index += Hi * (t + 1)  # every token up to and including t is scored
            chosen += int(np.count_nonzero(r["sel"][t] >= 0))
    w = bench.token_select_work(lens, D, Hq, Hkv, Hi, Di, top_k)
    assert w["index"] == 2 * Di * index
    assert w["attn"] == 4 * D * Hq * chosen
    assert w["gather_bytes"] == chosen * Hkv * D * 2 * 2

"""Parity of the sm_100a decode path (nsa_decode through the C ABI) with the
fp64 oracle: the newest token of each sequence attends to its KV cache and
its compressed cache; a block completed by the newest token is compressed
first.  Stage-wise as for prefill: the oracle runs on the GPU's compressed
cache (which holds the newly compressed block), index sets must match except
where the oracle's n-th/(n+1)-th score gap is below 1e-6, fp32 outputs within
max-abs 1e-2 and relative L2 5e-3; the newly compressed block within half a
bf16 ulp plus 1e-5 of the exact value."""
import numpy as np
import pytest

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import nsa
from sparse_attention_long_06_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from sparse_attention_long_06_b200 import build
    build.build()
    nsa.lib()


def run_decode(cfg, inp, out_dtype=nsa.OUT_F32):
    import torch
    B = len(inp["seqlens"])
    cap = int(inp["capacity"])
    plan = nsa.Plan.for_config(cfg, max_batch=B, max_seqlen=cap, out_dtype=out_dtype)
    d = {k: gu.to_dev(inp[k]) for k in ("q", "k", "v", "kc", "vc", "gates", "w_k", "w_v", "seqlens")}
    out = torch.empty((B, cfg.num_q_heads, cfg.head_dim),
                      dtype=torch.float32 if out_dtype == nsa.OUT_F32 else torch.int16, device="cuda")
    sel = torch.full((B, cfg.num_kv_heads, cfg.top_n), -7, dtype=torch.int32, device="cuda")
    ws = plan.alloc_workspace(nsa.MODE_DECODE)
    plan.decode(d["q"], d["k"], d["v"], d["kc"], d["vc"], d["seqlens"], d["gates"], d["w_k"],
                d["w_v"], out, ws, sel_idx=sel)
    status = nsa.read_device_status(ws)
    res = {"status": status, "launches": nsa.last_launch_count(), "sel": sel.cpu().numpy(),
           "kc": gu.bits(d["kc"]), "vc": gu.bits(d["vc"])}
    res["out"] = (out.cpu().numpy().astype(np.float64) if out_dtype == nsa.OUT_F32
                  else wl.bf16_to_f32(gu.bits(out)).astype(np.float64))
    return res


def check(cfg, inp, res, seqs):
    p = OracleParams.of(cfg)
    worst, num, den, bad_idx = 0.0, 0.0, 0.0, 0
    for b in seqs:
        L = int(inp["seqlens"][b])
        C = gu.num_cmp(cfg, L)
        if C > 0 and (C - 1) * cfg.cmp_stride + cfg.cmp_block == L:  # completed by the new token
            blk = C - 1
            seg = slice(blk * cfg.cmp_stride, blk * cfg.cmp_stride + cfg.cmp_block)
            for name, wname, gname in (("k", "w_k", "kc"), ("v", "w_v", "vc")):
                exact, _ = oracle.compress(p, inp[name][b][seg], inp[wname])
                got = wl.bf16_to_f32(res[gname][b, blk]).astype(np.float64)
                assert np.all(np.abs(got - exact[0]) <= gu.kc_bound(exact[0]))
        r = oracle.decode_reference(p, inp, b, kc=res["kc"][b], vc=res["vc"][b])
        same = np.all(r["sel"] == res["sel"][b], axis=1)
        bad_idx += int(np.count_nonzero(~same & (r["gap"] >= 1e-6)))
        diff = np.abs(res["out"][b] - r["out"])
        worst = max(worst, float(diff.max()))
        num += float(np.sum(diff ** 2))
        den += float(np.sum(r["out"] ** 2))
    rel = (num / den) ** 0.5
    print({"max_abs": worst, "rel_l2": rel, "bad_idx": bad_idx})
    assert bad_idx == 0
    assert worst <= 1e-2 and rel <= 5e-3


@pytest.mark.parametrize("geom", [
    # D, Hq, Hkv, l, n, w, lengths, capacity
    (64, 4, 1, 32, 4, 128, [1, 31, 32, 100, 640, 1000], 1024),
    (128, 64, 4, 64, 16, 512, [700, 4096, 5000, 63, 64, 9000], 9024),
    (128, 16, 2, 64, 8, 200, [1500, 1536, 333], 1536),
    (64, 8, 8, 32, 32, 1000, [2000, 2048], 2048),
])
def test_decode_geometries(geom):
    D, Hq, Hkv, l, n, w, lens, cap = geom
    cfg = wl.NsaConfig("dec", 31, D, Hq, Hkv, l, l, l, n, w, decode_batch=len(lens))
    inp = wl.decode_inputs(cfg, lengths=lens, capacity=cap)
    res = run_decode(cfg, inp)
    assert res["status"] == nsa.NSA_OK
    assert res["launches"] == 3
    check(cfg, inp, res, range(len(lens)))


def test_decode_64k_config_sampled_sequences():
    cfg = wl.CONFIGS["decode_64k"]
    inp = wl.decode_inputs(cfg)
    res = run_decode(cfg, inp)
    assert res["status"] == nsa.NSA_OK
    check(cfg, inp, res, [0, 13, 31])
    # bf16 output is the rounding of the fp32 output
    res16 = run_decode(cfg, inp, out_dtype=nsa.OUT_BF16)
    assert np.array_equal(wl.bf16_bits(res["out"].astype(np.float32)),
                          wl.bf16_bits(res16["out"].astype(np.float32)))


@pytest.mark.parametrize("geom", [
    # D, Hq, Hkv, l, d, l', n, w, lengths, capacity
    (128, 64, 4, 32, 16, 64, 16, 512, [700, 4000, 5000, 9008], 9024),  # overlapping, l' = 2 l
    (64, 8, 2, 64, 32, 32, 8, 200, [63, 64, 96, 2000, 2016], 2048),    # overlapping, l' < l
    (128, 16, 1, 32, 32, 64, 4, 128, [31, 32, 1000, 4064], 4096),      # l = d, l' = 2 l
])
def test_decode_general_geometry(geom):
    """Compression stride and selection block independent of the compression
    block: the newest token completes a compressed block when (len - l) % d
    == 0, and selection scores sum the compressed blocks overlapping each
    selection block."""
    D, Hq, Hkv, l, d, ls, n, w, lens, cap = geom
    cfg = wl.NsaConfig("dec_geo", 37, D, Hq, Hkv, l, d, ls, n, w, decode_batch=len(lens))
    inp = wl.decode_inputs(cfg, lengths=lens, capacity=cap)
    res = run_decode(cfg, inp)
    assert res["status"] == nsa.NSA_OK
    check(cfg, inp, res, range(len(lens)))


@pytest.mark.parametrize("period", [1, 3])
def test_decode_exact_score_ties_go_to_the_lower_block(period):
    """Compressed caches that repeat every `period` blocks give exactly equal
    block scores: the decode selection must equal the oracle's on every
    sequence, with no gap exemption (ties broken toward the lower index)."""
    cfg = wl.NsaConfig("dec_ties", 33, 128, 64, 4, 64, 64, 64, 16, 512, decode_batch=4)
    lens = [700, 4000, 5000, 9000]  # none completes a block: the cache is used as given
    inp = wl.decode_inputs(cfg, lengths=lens, capacity=9024)
    for name in ("kc", "vc"):
        c = inp[name]
        c[:] = c[:, np.arange(c.shape[1]) % period]
    res = run_decode(cfg, inp)
    assert res["status"] == nsa.NSA_OK
    p = OracleParams.of(cfg)
    for b, L in enumerate(lens):
        r = oracle.decode_reference(p, inp, b, kc=res["kc"][b], vc=res["vc"][b])
        assert np.array_equal(r["sel"], res["sel"][b]), b
        if period == 1 and (L - 1) // 64 + 1 > 16:
            # more candidates than n, every complete block ties: the lowest n win
            assert np.array_equal(res["sel"][b], np.tile(np.arange(16), (4, 1)))
    check(cfg, inp, res, range(len(lens)))


def test_decode_rejects_lengths_beyond_capacity():
    cfg = wl.NsaConfig("dec", 32, 64, 4, 1, 32, 32, 32, 4, 128, decode_batch=2)
    inp = wl.decode_inputs(cfg, lengths=[100, 200], capacity=256)
    inp["seqlens"] = np.array([100, 300], dtype=np.int32)
    res = run_decode(cfg, inp)
    assert res["status"] == nsa.NSA_ERR_DEVICE_BAD_INPUT

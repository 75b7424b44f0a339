"""Helpers for the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and compare it with the fp64 oracle."""
from __future__ import annotations

import json
import os

import numpy as np

import oracle
from oracle import OracleParams
from sparse_attention_long_06_b200 import nsa
from sparse_attention_long_06_b200 import workloads as wl


def to_dev(a: np.ndarray):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def run_prefill(cfg, inputs, out_dtype=nsa.OUT_F32, max_seqlen=None, both_dtypes=False):
    """Runs nsa_prefill and returns host copies of every output and of the
    workspace regions (O_cmp, LSE, scores).  With both_dtypes the call is made
    once with fp32 output ("out") and once with bf16 output ("out_bf16")."""
    import torch
    lens = inputs["seqlens"]
    total = int(inputs["cu_seqlens"][-1])
    max_seqlen = max_seqlen or max(max(lens), cfg.cmp_block, cfg.sel_block)
    D, Hq, Hkv, n = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.top_n
    dev = {k: to_dev(inputs[k]) for k in ("q", "k", "v", "gates", "w_k", "w_v", "cu_seqlens")}
    res = {}
    dtypes = [nsa.OUT_F32, nsa.OUT_BF16] if both_dtypes else [out_dtype]
    for dt in dtypes:
        plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max_seqlen,
                                   max_total_tokens=total, out_dtype=dt)
        crow = max(plan.cmp_rows(total), 1)
        out = torch.empty((total, Hq, D), dtype=torch.float32 if dt == nsa.OUT_F32 else torch.int16,
                          device="cuda")
        kc = torch.empty((crow, Hkv, D), dtype=torch.int16, device="cuda")
        vc = torch.empty((crow, Hkv, D), dtype=torch.int16, device="cuda")
        sel = torch.full((max(total, 1), Hkv, n), -7, dtype=torch.int32, device="cuda")
        ws = plan.alloc_workspace()
        plan.prefill(dev["q"], dev["k"], dev["v"], dev["gates"], dev["w_k"], dev["w_v"],
                     dev["cu_seqlens"], out, kc, vc, ws, sel_idx=sel)
        status = nsa.read_device_status(ws)
        if dt == nsa.OUT_BF16 and both_dtypes:
            res["out_bf16"] = bits(out)
            res["status_bf16"] = status
            continue
        res.update(status=status, plan=plan, launches=nsa.last_launch_count())
        if dt == nsa.OUT_F32:
            res["out"] = out.cpu().numpy().astype(np.float64)
        else:
            res["out"] = wl.bf16_to_f32(bits(out)).astype(np.float64)
        res["kc"], res["vc"] = bits(kc), bits(vc)
        res["sel"] = sel.cpu().numpy()
        wsn = ws.cpu().numpy()

        def region(r, dtype, shape):
            off, nb = plan.workspace_region(r)
            count = int(np.prod(shape))
            return wsn[off:off + count * 4].view(dtype).reshape(shape).copy()

        cap = num_cmp(cfg, max_seqlen)
        res["o_cmp"] = region(nsa.WS_O_CMP, np.float32, (total, Hq, D)).astype(np.float64)
        res["lse"] = region(nsa.WS_LSE, np.float32, (total, Hq)).astype(np.float64)
        res["scores"] = region(nsa.WS_SCORES, np.float32, (total, Hkv, cap))
        if remaps(cfg):
            res["sel_scores"] = region(nsa.WS_SEL_SCORES, np.float32,
                                       (total, Hkv, max_seqlen // cfg.sel_block + 1))
        res["o_win_g"] = region(nsa.WS_WIN, np.float32, (total, Hq, D)).astype(np.float64)
        res["cap"] = cap
        del ws
    return res


def num_cmp(cfg, T):
    """Complete compressed blocks of a sequence of T tokens (block l, stride d)."""
    return 0 if T < cfg.cmp_block else (T - cfg.cmp_block) // cfg.cmp_stride + 1


def remaps(cfg) -> bool:
    """Whether selection scores are sums over overlapping compressed blocks
    (any geometry other than l == d == l')."""
    return not (cfg.cmp_stride == cfg.cmp_block == cfg.sel_block)


def cmp_offsets(cfg, lens):
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    off[1:] = np.cumsum([num_cmp(cfg, T) for T in lens])
    return off


def tol_bf16(ref: np.ndarray) -> np.ndarray:
    """max(1e-2, half a bf16 ulp of the reference) elementwise."""
    mag = np.maximum(np.abs(ref), 1e-30)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    return np.maximum(1e-2, 0.5 * ulp)


def kc_bound(exact: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp of the exact value plus 1e-5: the fp32 accumulation
    error of an (l * D)-term dot product of O(1) inputs with O(1/sqrt(l*D))
    weights stays below about 1e-6, so 1e-5 bounds it with a wide margin."""
    mag = np.maximum(np.abs(exact), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(mag)) - 7) + 1e-5


def rel_l2(a, b) -> float:
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def sample_rows(T: int, k: int, seed: int, tile: int, block: int) -> np.ndarray:
    """Rows that cover the start, block and tile edges, the tail, and random ones."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, block - 2, block - 1, block, 2 * block - 1, tile - 1, tile, T - 1, T - 2,
             T - tile, T - 1 - (T % tile)}
    fixed = {r for r in fixed if 0 <= r < T}
    extra = rng.choice(T, size=min(T, max(0, k - len(fixed))), replace=False)
    return np.array(sorted(fixed | set(int(x) for x in extra)), dtype=np.int32)


def check_prefill(cfg, inputs, res, rows_per_seq, check_e2e=True):
    """Stage-wise parity of one prefill run against the oracle (see
    tests/test_gpu_prefill.py for the acceptance rules).  Returns a report."""
    p = OracleParams.of(cfg)
    lens = inputs["seqlens"]
    cu = inputs["cu_seqlens"]
    coff = cmp_offsets(cfg, lens)
    rep = {"kc_diff": 0, "kc_total": 0, "kc_bound_fail": 0, "kc_max_err": 0.0, "idx_rows": 0, "idx_exempt": 0,
           "idx_bad_stageB": 0, "max_abs": 0.0, "rel_l2_num": 0.0, "rel_l2_den": 0.0,
           "e2e_idx_mismatch": 0, "e2e_rows": 0, "e2e_max_abs": 0.0, "out_tol_fail": 0}
    for b, T in enumerate(lens):
        s = int(cu[b])
        rows = rows_per_seq[b]
        if len(rows) == 0:
            continue
        C = num_cmp(cfg, T)
        kc_gpu = res["kc"][coff[b]:coff[b] + C]
        vc_gpu = res["vc"][coff[b]:coff[b] + C]
        # step 1: compressed KV = bf16 rounding of an fp32 accumulation: within
        # half a bf16 ulp of the exact value plus the fp32 accumulation error
        if C:
            blocks = np.unique(np.concatenate([np.arange(min(C, 4)), np.arange(max(0, C - 4), C),
                                               np.linspace(0, C - 1, num=min(C, 24)).astype(int)]))
            for blk in blocks:
                seg = slice(s + blk * cfg.cmp_stride, s + blk * cfg.cmp_stride + cfg.cmp_block)
                kf, kb = oracle.compress(p, inputs["k"][seg], inputs["w_k"])
                vf, vb = oracle.compress(p, inputs["v"][seg], inputs["w_v"])
                for exact, ref, got in ((kf[0], kb[0], kc_gpu[blk]), (vf[0], vb[0], vc_gpu[blk])):
                    rep["kc_diff"] += int(np.count_nonzero(ref != got))
                    rep["kc_total"] += ref.size
                    err = np.abs(wl.bf16_to_f32(got).astype(np.float64) - exact)
                    rep["kc_bound_fail"] += int(np.count_nonzero(err > kc_bound(exact)))
                    rep["kc_max_err"] = max(rep["kc_max_err"], float(err.max()))
        # stage A: the oracle's selection replayed on the GPU's fp32 scores
        tg = s + rows
        ncand = rows // cfg.sel_block + 1
        ncmp = np.array([num_cmp(cfg, t + 1) for t in rows], dtype=np.int32)
        for g in range(cfg.num_kv_heads):
            if remaps(cfg):  # the GPU's selection-block scores, every candidate defined
                selA, _ = oracle.select_f32(res["sel_scores"][tg, g, :], ncand, ncand, cfg.top_n)
            else:
                selA, _ = oracle.select_f32(res["scores"][tg, g, :], ncand, ncmp, cfg.top_n)
            assert np.array_equal(selA, res["sel"][tg, g, :]), f"stage A selection, seq {b} group {g}"
        # stage B: oracle steps 2-7 on the GPU's compressed KV
        kcb = kc_gpu if C else np.zeros((1, cfg.num_kv_heads, cfg.head_dim), np.uint16)
        vcb = vc_gpu if C else np.zeros((1, cfg.num_kv_heads, cfg.head_dim), np.uint16)
        jmax = T // cfg.sel_block + 1
        r = oracle.nsa_rows(p, inputs["q"][s:s + T], inputs["k"][s:s + T], inputs["v"][s:s + T],
                            kcb, vcb, inputs["gates"][s:s + T], rows, cmax=max(C, jmax, 1))
        # compressed branch and scores (fp32 vs fp64)
        assert np.max(np.abs(res["o_cmp"][tg] - r["o_cmp"])) < 1e-2
        # window branch times its gate (the window kernel's own output)
        win_ref = r["o_win"] * inputs["gates"][tg][:, :, 2:3].astype(np.float64)
        rep["win_max_abs"] = max(rep.get("win_max_abs", 0.0),
                                 float(np.max(np.abs(res["o_win_g"][tg] - win_ref))))
        assert rep["win_max_abs"] < 1e-2
        vis = ncmp > 0
        if np.any(vis):
            assert np.max(np.abs(res["lse"][tg][vis] - r["lse"][vis])) < 1e-4
        for ri, t in enumerate(rows):
            if remaps(cfg):  # selection-block scores
                nj = t // cfg.sel_block + 1
                assert np.max(np.abs(res["sel_scores"][s + t, :, :nj] - r["scores"][ri, :, :nj])) < 1e-5
                continue
            nc = num_cmp(cfg, t + 1)
            if nc:
                assert np.max(np.abs(res["scores"][s + t, :, :nc] - r["scores"][ri, :, :nc])) < 1e-5
        for g in range(cfg.num_kv_heads):
            same = np.all(r["sel"][:, g, :] == res["sel"][tg, g, :], axis=1)
            exempt = r["gap"][:, g] < 1e-6
            rep["idx_rows"] += len(rows)
            rep["idx_exempt"] += int(np.count_nonzero(~same & exempt))
            rep["idx_bad_stageB"] += int(np.count_nonzero(~same & ~exempt))
        # outputs of the rows whose index sets agree (a row exempted above as a
        # near tie attends to other blocks, so its output legitimately differs)
        agree_b = np.all(r["sel"] == res["sel"][tg], axis=(1, 2))
        rep["out_rows_skipped"] = rep.get("out_rows_skipped", 0) + int(np.count_nonzero(~agree_b))
        if np.any(agree_b):
            got, ref = res["out"][tg][agree_b], r["out"][agree_b]
            diff = np.abs(got - ref)
            rep["max_abs"] = max(rep["max_abs"], float(diff.max()))
            rep["out_tol_fail"] += int(np.count_nonzero(diff > tol_bf16(ref)))
            rep["rel_l2_num"] += float(np.sum((got - ref) ** 2))
            rep["rel_l2_den"] += float(np.sum(ref ** 2))
        # end to end: the oracle's own compressed KV
        if check_e2e and C:
            _, kco = oracle.compress(p, inputs["k"][s:s + T], inputs["w_k"])
            _, vco = oracle.compress(p, inputs["v"][s:s + T], inputs["w_v"])
            r2 = oracle.nsa_rows(p, inputs["q"][s:s + T], inputs["k"][s:s + T],
                                 inputs["v"][s:s + T], kco, vco, inputs["gates"][s:s + T], rows,
                                 cmax=max(C, jmax))
            for g in range(cfg.num_kv_heads):
                same = np.all(r2["sel"][:, g, :] == res["sel"][tg, g, :], axis=1)
                rep["e2e_idx_mismatch"] += int(np.count_nonzero(~same & (r2["gap"][:, g] >= 1e-6)))
                rep["e2e_rows"] += len(rows)
            agree = np.all(r2["sel"] == res["sel"][tg], axis=(1, 2))
            if np.any(agree):
                rep["e2e_max_abs"] = max(rep["e2e_max_abs"],
                                         float(np.abs(res["out"][tg][agree] - r2["out"][agree]).max()))
    rep["rel_l2"] = (rep["rel_l2_num"] / rep["rel_l2_den"]) ** 0.5 if rep["rel_l2_den"] else 0.0
    return rep


def log_report(name: str, rep: dict) -> None:
    """Prints a parity report and, when NSA_PARITY_LOG names a file, appends
    it there as one JSON line (so that the observed counts of a GPU run are
    kept beside its pass/fail status)."""
    rec = {"test": name}
    rec.update({k: (float(v) if isinstance(v, (float, np.floating)) else v)
                for k, v in rep.items() if isinstance(v, (int, float, np.integer, np.floating))})
    print(json.dumps(rec))
    path = os.environ.get("NSA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def topn_path(score_row: np.ndarray, ncmp: int, ncand: int, n: int, cand_cap: int = 64) -> str:
    """Which branch of the prefill top-n kernel a row takes, from its fp32
    scores: "all" (at most n candidates), "regs" (the register selection) or
    "radix" (the radix-select fallback: more than 1024 candidates, or more
    than `cand_cap` keys at or above the n-th largest per-lane maximum of the
    64-bit (score bits, inverted index) keys dealt to lanes by j % 32)."""
    if ncand <= n:
        return "all"
    if ncand > 1024 or n > 32:
        return "radix"
    j = np.arange(1024, dtype=np.uint64)
    b = np.zeros(1024, dtype=np.uint64)
    b[:ncmp] = np.ascontiguousarray(score_row[:ncmp], dtype=np.float32).view(np.uint32)
    key = (b << np.uint64(32)) | (np.uint64(0xFFFFFFFF) - j)
    key[ncand:] = 0
    lmax = key.reshape(32, 32).max(axis=0)      # lane = j % 32
    t0 = np.sort(lmax)[::-1][n - 1]
    count = int(np.count_nonzero((key >= t0) & (key != 0)))
    return "radix" if count > cand_cap else "regs"

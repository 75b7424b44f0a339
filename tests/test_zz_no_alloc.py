"""nsa_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (it runs on a static device array inside the library
instead of a caller workspace).  Its results must match nsa_prefill's on the
same inputs, call after call, within the parity tolerance of the other GPU
tests (max-abs 1e-2, relative L2 5e-3, equal index sets)."""
import numpy as np
import pytest

from sparse_attention_long_06_b200 import nsa
from sparse_attention_long_06_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from sparse_attention_long_06_b200 import build
    build.build()
    cfg = wl.CONFIGS["tiny"]
    inp = wl.prefill_inputs(cfg)
    T = int(inp["cu_seqlens"][-1])

    def dev(a):
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    d = {k: dev(inp[k]) for k in ("q", "k", "v", "gates", "w_k", "w_v", "cu_seqlens")}
    plan = nsa.Plan.for_config(cfg, max_batch=1, max_seqlen=T, max_total_tokens=T,
                               out_dtype=nsa.OUT_F32)
    assert plan.workspace_size() <= 32 << 20

    def buffers():
        out = torch.full((T, cfg.num_q_heads, cfg.head_dim), float("nan"), device="cuda")
        kc = torch.zeros((plan.cmp_rows(T), cfg.num_kv_heads, cfg.head_dim), dtype=torch.int16,
                         device="cuda")
        sel = torch.full((T, cfg.num_kv_heads, cfg.top_n), -9, dtype=torch.int32, device="cuda")
        return out, kc, torch.zeros_like(kc), sel

    ref_out, ref_kc, ref_vc, ref_sel = buffers()
    ws = plan.alloc_workspace()
    plan.prefill(d["q"], d["k"], d["v"], d["gates"], d["w_k"], d["w_v"], d["cu_seqlens"],
                 ref_out, ref_kc, ref_vc, ws, sel_idx=ref_sel)
    assert nsa.read_device_status(ws) == nsa.NSA_OK
    ref = ref_out.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out, kc, vc, sel = buffers()
        plan.prefill_noalloc(d["q"], d["k"], d["v"], d["gates"], d["w_k"], d["w_v"],
                             d["cu_seqlens"], out, kc, vc, sel_idx=sel)
        assert nsa.noalloc_read_device_status() == nsa.NSA_OK
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.max(np.abs(got - ref)) <= 1e-2
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3
        assert np.array_equal(sel.cpu().numpy(), ref_sel.cpu().numpy())
        assert np.array_equal(kc.cpu().numpy(), ref_kc.cpu().numpy())
        assert np.array_equal(vc.cpu().numpy(), ref_vc.cpu().numpy())


def test_noalloc_reports_device_side_input_errors():
    """A sequence longer than the plan's max_seqlen is caught on the device;
    the caller reads the fault from the static array's status word."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from sparse_attention_long_06_b200 import build
    build.build()
    cfg = wl.NsaConfig("bad", 21, 64, 4, 1, 32, 32, 32, 4, 128, seqlens=(100, 100))
    inp = wl.prefill_inputs(cfg)
    plan = nsa.Plan.for_config(cfg, max_batch=2, max_seqlen=128, max_total_tokens=200,
                               out_dtype=nsa.OUT_F32)

    def dev(a):
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    d = {k: dev(inp[k]) for k in ("q", "k", "v", "gates", "w_k", "w_v")}
    cu = torch.tensor([0, 150, 200], dtype=torch.int32, device="cuda")  # first length > 128
    out = torch.zeros((200, 4, 64), device="cuda")
    kc = torch.zeros((plan.cmp_rows(200), 1, 64), dtype=torch.int16, device="cuda")
    vc = torch.zeros_like(kc)
    plan.prefill_noalloc(d["q"], d["k"], d["v"], d["gates"], d["w_k"], d["w_v"], cu, out, kc, vc)
    assert nsa.noalloc_read_device_status() == nsa.NSA_ERR_DEVICE_BAD_INPUT
    assert nsa.noalloc_read_device_status() == nsa.NSA_OK  # cleared by the read


def test_noalloc_rejects_plans_beyond_the_static_array():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = wl.CONFIGS["prefill_8k"]
    plan = nsa.Plan.for_config(cfg, max_batch=1, max_seqlen=8192, max_total_tokens=8192)
    assert plan.workspace_size() > 32 << 20
    t = torch.zeros(16, dtype=torch.int16, device="cuda")
    cu = torch.tensor([0, 8192], dtype=torch.int32, device="cuda")
    with pytest.raises(nsa.NsaError) as e:
        plan.prefill_noalloc(t, t, t, t, t, t, cu, t, t, t)
    assert e.value.code == nsa.NSA_ERR_WORKSPACE

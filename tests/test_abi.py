"""The C-ABI library loads on a machine without a GPU, exports every entry
point declared in include/nsa.h, and validates arguments on the host (every
error below is returned before anything touches the device)."""
import ctypes
import os
import re

import pytest

from sparse_attention_long_06_b200 import build as nsa_build
from sparse_attention_long_06_b200 import nsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nsa_build.build()
    return nsa.lib()


def _declared():
    text = open(os.path.join(ROOT, "include", "nsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "nsa_prefill" in names and "nsa_decode" in names and "nsa_plan_create" in names
    for name in names:
        assert hasattr(L, name), name
    assert sorted(names) == sorted(nsa.EXPORTED)


def test_no_link_dependency_on_libtorch_or_libcuda(L):
    # the library carries its own CUDA runtime and reaches the driver at run time
    out = os.popen(f"ldd {nsa.LIB_PATH}").read()
    assert "libtorch" not in out and "libc10" not in out
    assert "libcuda.so" not in out


def _params(**kw):
    base = dict(head_dim=128, num_q_heads=64, num_kv_heads=4, cmp_block=64, cmp_stride=64,
                sel_block=64, top_n=16, window=512, max_batch=8, max_seqlen=65536,
                max_total_tokens=65536)
    base.update(kw)
    return base


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(num_q_heads=63), nsa.NSA_ERR_INVALID_ARG),
    (dict(top_n=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(window=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(cmp_stride=128), nsa.NSA_ERR_INVALID_ARG),       # stride longer than the block
    (dict(head_dim=96), nsa.NSA_ERR_UNSUPPORTED),
    (dict(num_q_heads=96, num_kv_heads=4), nsa.NSA_ERR_UNSUPPORTED),  # G = 24
    (dict(cmp_stride=48), nsa.NSA_ERR_INVALID_ARG),        # stride that does not divide the block
    (dict(cmp_stride=8), nsa.NSA_ERR_UNSUPPORTED),         # overlap of 7/8 of a block
    (dict(sel_block=128), nsa.NSA_ERR_UNSUPPORTED),
    (dict(sel_block=32, top_n=33), nsa.NSA_ERR_UNSUPPORTED),  # more than one warp of blocks
    (dict(top_n=17), nsa.NSA_ERR_UNSUPPORTED),             # > 8 chunks of 128 keys
    (dict(max_seqlen=16), nsa.NSA_ERR_INVALID_ARG),
])
def test_plan_validation(L, kw, code):
    with pytest.raises(nsa.NsaError) as e:
        nsa.Plan(**_params(**kw))
    assert e.value.code == code


def test_general_geometry_plans(L):
    # overlapping compression and selection blocks other than l are planned
    p = nsa.Plan(**_params(cmp_block=32, cmp_stride=16, sel_block=64))
    assert p.cmp_rows(65536) == 65536 // 16
    off, nb = p.workspace_region(nsa.WS_SEL_SCORES)
    assert nb == 65536 * 4 * (65536 // 64 + 1) * 4
    off, nb = p.workspace_region(nsa.WS_SCORES)
    assert nb == 65536 * 4 * ((65536 - 32) // 16 + 1) * 4
    # with l == d == l' the selection scores are the compressed-block scores
    q = nsa.Plan(**_params())
    assert q.workspace_region(nsa.WS_SEL_SCORES)[1] == 0


def test_plan_sizes(L):
    p = nsa.Plan(**_params())
    ws = p.workspace_size(nsa.MODE_PREFILL)
    T, Hq, Hkv, D = 65536, 64, 4, 128
    assert ws >= T * Hq * D * 4 + T * Hkv * 1024 * 4
    off, nb = p.workspace_region(nsa.WS_O_CMP)
    assert off % 256 == 0 and nb == T * Hq * D * 4
    off2, nb2 = p.workspace_region(nsa.WS_SCORES)
    assert off2 >= off + nb and nb2 == T * Hkv * 1024 * 4 and off2 + nb2 <= ws
    # every region is 256-byte aligned, inside the workspace, and disjoint
    regions = sorted(p.workspace_region(r) for r in (nsa.WS_O_CMP, nsa.WS_LSE, nsa.WS_SCORES,
                                                     nsa.WS_SEL, nsa.WS_WIN))
    for (o1, n1), (o2, _) in zip(regions, regions[1:]):
        assert o1 % 256 == 0 and o1 + n1 <= o2
    assert regions[-1][0] + regions[-1][1] <= ws
    assert p.workspace_region(nsa.WS_WIN)[1] == T * Hq * D * 4
    assert p.cmp_rows(65536) == 1024 and p.cmp_rows(100) == 1
    assert nsa.Plan(**_params(head_dim=64, num_q_heads=4, num_kv_heads=1, cmp_block=32,
                              cmp_stride=32, sel_block=32, top_n=4, window=128)).workspace_size() > 0


def test_prefill_rejects_bad_arguments_before_launch(L):
    p = nsa.Plan(**_params(max_total_tokens=4096))
    fake = 1 << 20  # an aligned address that is never dereferenced
    ws = p.workspace_size()
    args = dict(q=fake, k=fake, v=fake, gates=fake, w_k=fake, w_v=fake, cu=fake, batch=1,
                total=4096, out=fake, kc=fake, vc=fake, sel=None, ws=fake, wsb=ws)

    def call(**over):
        a = dict(args)
        a.update(over)
        return L.nsa_prefill(p.handle, a["q"], a["k"], a["v"], a["gates"], a["w_k"], a["w_v"],
                             a["cu"], a["batch"], a["total"], a["out"], a["kc"], a["vc"], a["sel"],
                             a["ws"], a["wsb"], None)

    assert call(q=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=9) == nsa.NSA_ERR_INVALID_ARG
    assert call(total=4097) == nsa.NSA_ERR_INVALID_ARG
    assert call(ws=None) == nsa.NSA_ERR_WORKSPACE
    assert call(wsb=ws - 1) == nsa.NSA_ERR_WORKSPACE
    assert call(ws=fake + 16) == nsa.NSA_ERR_WORKSPACE        # workspace not 256-byte aligned
    assert call(q=fake + 2) == nsa.NSA_ERR_MISALIGNED
    assert call(kc=fake + 8) == nsa.NSA_ERR_MISALIGNED
    assert call(kc=None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_last_launch_count() == 0
    assert L.nsa_plan_create(None, ctypes.byref(ctypes.c_void_p())) == nsa.NSA_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments_before_launch(L):
    p = nsa.Plan(**_params(max_batch=4, max_seqlen=65536 + 64))
    fake = 1 << 20  # an aligned address that is never dereferenced
    wsb = p.workspace_size(nsa.MODE_DECODE)
    assert wsb > 256  # status, counters, selection and the partial results
    args = dict(q=fake, k=fake, v=fake, kc=fake, vc=fake, lens=fake, batch=2, cap=4096,
                gates=fake, w_k=fake, w_v=fake, out=fake, sel=None, ws=fake, wsb=wsb)

    def call(**over):
        a = dict(args)
        a.update(over)
        return L.nsa_decode(p.handle, a["q"], a["k"], a["v"], a["kc"], a["vc"], a["lens"],
                            a["batch"], a["cap"], a["gates"], a["w_k"], a["w_v"], a["out"],
                            a["sel"], a["ws"], a["wsb"], None)

    assert call(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=5) == nsa.NSA_ERR_INVALID_ARG
    assert call(cap=4000) == nsa.NSA_ERR_INVALID_ARG            # not a multiple of l
    assert call(cap=65536 + 128) == nsa.NSA_ERR_INVALID_ARG     # above the plan's max_seqlen
    assert call(ws=None) == nsa.NSA_ERR_WORKSPACE
    assert call(wsb=255) == nsa.NSA_ERR_WORKSPACE
    assert call(cap=65536 + 64, batch=4, wsb=wsb - 1) == nsa.NSA_ERR_WORKSPACE
    assert call(q=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(k=fake + 2) == nsa.NSA_ERR_MISALIGNED
    assert call(lens=fake + 2) == nsa.NSA_ERR_MISALIGNED
    wide = nsa.Plan(**_params(max_seqlen=70 * 1024 + 64, window=2048))
    assert L.nsa_decode(wide.handle, fake, fake, fake, fake, fake, fake, 1, 4096, fake, fake,
                        fake, fake, None, fake, 256, None) == nsa.NSA_ERR_UNSUPPORTED  # w > 1024
    assert L.nsa_last_launch_count() == 0


def test_block_select_sizes_and_bad_arguments(L):
    p = nsa.Plan(**_params(max_total_tokens=4096, max_seqlen=4096))
    T, Hkv, n = 4096, 4, 16
    wsb = p.workspace_size(nsa.MODE_BLOCK_SELECT)
    # status + metadata, routing scores [T, Hkv, max_seqlen / l'], selection
    assert wsb >= T * Hkv * (4096 // 64) * 4 + T * Hkv * n * 4
    assert wsb < p.workspace_size(nsa.MODE_PREFILL)
    assert p.workspace_region(nsa.WS_SCORES, nsa.MODE_BLOCK_SELECT)[1] == T * Hkv * 64 * 4
    assert p.workspace_region(nsa.WS_SEL, nsa.MODE_BLOCK_SELECT)[1] == T * Hkv * n * 4
    with pytest.raises(nsa.NsaError):
        p.workspace_region(nsa.WS_O_CMP, nsa.MODE_BLOCK_SELECT)
    assert p.block_rows(4096) == 64 and p.block_rows(100) == 1 and p.block_rows(63) == 0
    fake = 1 << 20  # an aligned address that is never dereferenced
    args = dict(q=fake, k=fake, v=fake, cu=fake, batch=1, total=4096, out=fake, km=fake,
                sel=None, ws=fake, wsb=wsb)

    def call(**over):
        a = dict(args)
        a.update(over)
        return L.nsa_block_select_prefill(p.handle, a["q"], a["k"], a["v"], a["cu"], a["batch"],
                                          a["total"], a["out"], a["km"], a["sel"], a["ws"],
                                          a["wsb"], None)

    assert call(q=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(km=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(total=4097) == nsa.NSA_ERR_INVALID_ARG
    assert call(ws=None) == nsa.NSA_ERR_WORKSPACE
    assert call(wsb=wsb - 1) == nsa.NSA_ERR_WORKSPACE
    assert call(ws=fake + 16) == nsa.NSA_ERR_WORKSPACE
    assert call(v=fake + 2) == nsa.NSA_ERR_MISALIGNED
    assert call(km=fake + 8) == nsa.NSA_ERR_MISALIGNED
    assert call(sel=fake + 2) == nsa.NSA_ERR_MISALIGNED
    assert L.nsa_block_select_prefill(None, fake, fake, fake, fake, 1, 1, fake, fake, None, fake,
                                      wsb, None) == nsa.NSA_ERR_INVALID_ARG
    assert L.nsa_last_launch_count() == 0


def test_block_select_decode_rejects_bad_arguments_before_launch(L):
    p = nsa.Plan(**_params(max_batch=4, max_seqlen=65536))
    fake = 1 << 20  # an aligned address that is never dereferenced
    wsb = p.workspace_size(nsa.MODE_BLOCK_SELECT_DECODE)
    assert 256 < wsb < p.workspace_size(nsa.MODE_DECODE)  # selected units only
    args = dict(q=fake, k=fake, v=fake, km=fake, lens=fake, batch=2, cap=4096, out=fake, sel=None,
                ws=fake, wsb=wsb)

    def call(**over):
        a = dict(args)
        a.update(over)
        return L.nsa_block_select_decode(p.handle, a["q"], a["k"], a["v"], a["km"], a["lens"],
                                         a["batch"], a["cap"], a["out"], a["sel"], a["ws"],
                                         a["wsb"], None)

    assert call(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=5) == nsa.NSA_ERR_INVALID_ARG
    assert call(cap=4000) == nsa.NSA_ERR_INVALID_ARG            # not a multiple of l'
    assert call(cap=65536 + 64) == nsa.NSA_ERR_INVALID_ARG      # above the plan's max_seqlen
    assert call(ws=None) == nsa.NSA_ERR_WORKSPACE
    assert call(wsb=255) == nsa.NSA_ERR_WORKSPACE
    assert call(km=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(km=fake + 8) == nsa.NSA_ERR_MISALIGNED
    assert call(lens=fake + 2) == nsa.NSA_ERR_MISALIGNED
    big = nsa.Plan(**_params(max_batch=1, max_seqlen=4097 * 64))
    assert L.nsa_block_select_decode(big.handle, fake, fake, fake, fake, fake, 1, 4097 * 64, fake,
                                     None, fake, 1 << 30, None) == nsa.NSA_ERR_UNSUPPORTED
    assert L.nsa_last_launch_count() == 0


def test_token_select_sizes_and_bad_arguments(L):
    p = nsa.Plan(**_params(max_total_tokens=4096, max_seqlen=4096))
    wsb = p.token_select_workspace_size(2048)
    assert wsb >= 4096 * 4096 * 4 + 4096 * 2048 * 4  # index scores + selection
    assert p.token_select_workspace_size(0) == 0
    fake = 1 << 20  # an aligned address that is never dereferenced
    args = dict(q=fake, k=fake, v=fake, qi=fake, wi=fake, ki=fake, hi=16, di=128, top_k=2048,
                cu=fake, batch=1, total=4096, out=fake, sel=None, ws=fake, wsb=wsb)

    def call(**over):
        a = dict(args)
        a.update(over)
        return L.nsa_token_select_prefill(p.handle, a["q"], a["k"], a["v"], a["qi"], a["wi"],
                                          a["ki"], a["hi"], a["di"], a["top_k"], a["cu"],
                                          a["batch"], a["total"], a["out"], a["sel"], a["ws"],
                                          a["wsb"], None)

    assert call(top_k=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(top_k=4097) == nsa.NSA_ERR_INVALID_ARG       # above max_seqlen
    assert call(hi=3) == nsa.NSA_ERR_UNSUPPORTED
    assert call(di=96) == nsa.NSA_ERR_UNSUPPORTED
    assert call(qi=None) == nsa.NSA_ERR_INVALID_ARG
    assert call(batch=0) == nsa.NSA_ERR_INVALID_ARG
    assert call(ws=None) == nsa.NSA_ERR_WORKSPACE
    assert call(wsb=wsb - 1) == nsa.NSA_ERR_WORKSPACE
    assert call(ki=fake + 8) == nsa.NSA_ERR_MISALIGNED
    assert call(wi=fake + 2) == nsa.NSA_ERR_MISALIGNED
    wide = nsa.Plan(**_params(num_q_heads=128, num_kv_heads=8))
    assert L.nsa_token_select_prefill(wide.handle, fake, fake, fake, fake, fake, fake, 16, 128, 16,
                                      fake, 1, 16, fake, None, fake, 1 << 40,
                                      None) == nsa.NSA_ERR_UNSUPPORTED  # Hq > 64
    assert L.nsa_last_launch_count() == 0


def test_noalloc_rejects_plans_beyond_its_static_array(L):
    big = nsa.Plan(**_params())  # 64k tokens: several GB of workspace
    assert big.workspace_size() > 32 << 20
    fake = 1 << 20
    rc = L.nsa_prefill_noalloc(big.handle, fake, fake, fake, fake, fake, fake, fake, 1, 65536,
                               fake, fake, fake, None, None)
    assert rc == nsa.NSA_ERR_WORKSPACE
    assert L.nsa_prefill_noalloc(None, fake, fake, fake, fake, fake, fake, fake, 1, 1, fake,
                                 fake, fake, None, None) == nsa.NSA_ERR_INVALID_ARG


def test_strerror_covers_every_code(L):
    for code in range(8):
        assert nsa.strerror(code) not in ("unknown status", "")
    assert nsa.strerror(99) == "unknown status"

"""C ABI checks that need no GPU: the library loads, exports every declared entry point,
and rejects bad arguments on the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

import patch_attention_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "patchattn.h")

FAKE = 0x7F0000000000  # 16-byte aligned fake device address, never dereferenced on these paths


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pf_[a-z0-9_]+)\s*\(", src)))


def _cfg(**kw):
    base = dict(batch=1, heads=2, head_dim=64, n_img=256, n_patches=4, n_txt=0, n_layers=2)
    base.update(kw)
    return pa.make_config(**base)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(pa.library_path())
    declared = _declared()
    assert set(declared) == set(pa.EXPORTED), declared
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    for s in range(0, 9):
        assert pa.pf_status_string(s)
    assert pa.pf_status_string(99) == "unknown status"
    assert pa.pf_version() >= 100


def test_kvbuf_bytes():
    c = _cfg()
    assert pa.pf_kvbuf_bytes(c) == 2 * 1 * 256 * 2 * 64 * 2
    c = _cfg(schedule=pa.PF_SCHED_DISTRIFUSION)
    assert pa.pf_kvbuf_bytes(c) == 2 * 2 * 1 * 256 * 2 * 64 * 2
    assert pa.pf_kvbuf_bytes(_cfg(n_img=255)) == 0
    assert pa.pf_kvbuf_bytes(_cfg(head_dim=96)) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(n_img=250), pa.PF_ERR_SHAPE),
    (dict(head_dim=96), pa.PF_ERR_UNSUPPORTED),
    (dict(heads=0), pa.PF_ERR_SHAPE),
    (dict(n_txt=-1), pa.PF_ERR_SHAPE),
    (dict(schedule=7), pa.PF_ERR_UNSUPPORTED),
    (dict(softmax_scale=-1.0), pa.PF_ERR_INVALID_ARG),
])
def test_create_rejects_bad_config(kw, status):
    with pytest.raises(pa.PatchAttnError) as e:
        pa.pf_create(_cfg(**kw), [FAKE, FAKE])
    assert e.value.status == status


def test_create_rejects_bad_buffers():
    with pytest.raises(pa.PatchAttnError) as e:
        pa.pf_create(_cfg(), [FAKE, 0])
    assert e.value.status == pa.PF_ERR_INVALID_ARG
    with pytest.raises(pa.PatchAttnError) as e:
        pa.pf_create(_cfg(), [FAKE, FAKE + 8])
    assert e.value.status == pa.PF_ERR_ALIGN


def _raw_step(ctx, layer, patch, ptrs, txt=(None, None)):
    L = pa._lib()
    q, k, v, o = ptrs
    return L.pf_patch_attn_step(ctx, layer, patch, q, k, v, txt[0], txt[1], o, None)


def test_step_state_and_order_checks():
    ctx = pa.pf_create(_cfg(), [FAKE, FAKE])
    try:
        good = (FAKE, FAKE + 4096, FAKE + 8192, FAKE + 16384)
        # before the start-up pass
        assert _raw_step(ctx, 0, 0, good) == pa.PF_ERR_STATE
        # bad layer / patch / pointers are argument errors
        assert _raw_step(ctx, 2, 0, good) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, -1, 0, good) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, 0, 4, good) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, 0, 0, (None, FAKE, FAKE, FAKE)) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, 0, 0, (FAKE + 2, FAKE, FAKE, FAKE)) == pa.PF_ERR_ALIGN
        # text pointers must be NULL when there is no text
        assert _raw_step(ctx, 0, 0, good, (FAKE, FAKE)) == pa.PF_ERR_INVALID_ARG
        # restore a checkpointed counter, then the order is enforced
        pa.pf_set_state(ctx, 0, 2)
        assert pa.pf_get_state(ctx, 0) == 2
        assert _raw_step(ctx, 0, 0, good) == pa.PF_ERR_ORDER
        assert _raw_step(ctx, 0, 3, good) == pa.PF_ERR_ORDER
        with pytest.raises(pa.PatchAttnError):
            pa.pf_get_state(ctx, 1)  # layer 1 never initialised
        with pytest.raises(pa.PatchAttnError):
            pa.pf_set_state(ctx, 0, 4)
    finally:
        pa.pf_destroy(ctx)


def test_step_requires_text_when_configured():
    ctx = pa.pf_create(_cfg(n_txt=8), [FAKE, FAKE])
    try:
        pa.pf_set_state(ctx, 0, 0)
        good = (FAKE, FAKE, FAKE, FAKE)
        assert _raw_step(ctx, 0, 0, good) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, 0, 0, good, (FAKE, None)) == pa.PF_ERR_INVALID_ARG
        assert _raw_step(ctx, 0, 0, good, (FAKE, FAKE + 4)) == pa.PF_ERR_ALIGN
    finally:
        pa.pf_destroy(ctx)


def test_failed_launch_does_not_advance_order():
    # Without a usable device the call fails after validation; the counter must not move.
    import torch
    if torch.cuda.is_available():
        pytest.skip("needs a host without a GPU")
    ctx = pa.pf_create(_cfg(), [FAKE, FAKE])
    try:
        pa.pf_set_state(ctx, 0, 1)
        st = _raw_step(ctx, 0, 1, (FAKE, FAKE, FAKE, FAKE))
        assert st == pa.PF_ERR_CUDA
        assert pa.pf_get_state(ctx, 0) == 1
    finally:
        pa.pf_destroy(ctx)


def test_destroy_null_is_ok():
    assert pa._lib().pf_destroy(None) == pa.PF_OK


def test_null_context_everywhere():
    L = pa._lib()
    assert L.pf_kvbuf_init(None, 0, FAKE, FAKE, None) == pa.PF_ERR_INVALID_ARG
    assert L.pf_patch_attn_step(None, 0, 0, FAKE, FAKE, FAKE, None, None, FAKE, None) == pa.PF_ERR_INVALID_ARG
    assert L.pf_check_device_status(None, None) == pa.PF_ERR_INVALID_ARG
    out = ctypes.c_void_p()
    assert L.pf_create(None, None, ctypes.byref(out)) == pa.PF_ERR_INVALID_ARG
    assert out.value is None


def test_cfg_argument_checks():
    L = pa._lib()
    ws = pa.pf_cfg_workspace_bytes(2, 1024)
    assert ws >= 2 * 16
    assert pa.pf_cfg_workspace_bytes(2, 1022) == 0
    call = lambda **kw: L.pf_cfg_combine_relmae(
        kw.get("c", FAKE), kw.get("u", FAKE), kw.get("b", 2), kw.get("n", 1024), kw.get("w", 7.0),
        kw.get("of", FAKE), kw.get("ob", None), kw.get("r", FAKE), kw.get("ws", FAKE),
        kw.get("wsb", ws), None)
    assert call(c=None) == pa.PF_ERR_INVALID_ARG
    assert call(r=None) == pa.PF_ERR_INVALID_ARG
    assert call(n=1022) == pa.PF_ERR_SHAPE
    assert call(b=0) == pa.PF_ERR_SHAPE
    assert call(w=float("nan")) == pa.PF_ERR_INVALID_ARG
    assert call(u=FAKE + 4) == pa.PF_ERR_ALIGN
    assert call(ob=FAKE + 2) == pa.PF_ERR_ALIGN
    assert call(wsb=ws - 1) == pa.PF_ERR_INVALID_ARG


def test_workspace_sizes_and_checks():
    # SD3-like call: 192 query-tile pairs; the workspace holds at least their counters
    c = _cfg(heads=24, n_img=16384, n_patches=8, n_txt=154, head_dim=64, n_layers=1)
    ws = pa.pf_workspace_bytes(c)
    assert ws >= 192 * 2 * 2 * 4 + 16
    assert pa.pf_workspace_bytes(_cfg(head_dim=96)) == 0
    ctx = pa.pf_create(c, [FAKE])
    try:
        L = pa._lib()
        assert L.pf_set_workspace(ctx, FAKE + 8, ws, None) == pa.PF_ERR_ALIGN
        assert L.pf_set_workspace(ctx, FAKE, 16, None) == pa.PF_ERR_INVALID_ARG
        assert L.pf_set_workspace(ctx, None, 0, None) == pa.PF_OK
        assert L.pf_set_workspace(None, FAKE, ws, None) == pa.PF_ERR_INVALID_ARG
    finally:
        pa.pf_destroy(ctx)


def test_workspace_covers_the_text_query_call():
    # 64-row patches but 512 text tokens: the text-query call has more query-tile groups (2 per
    # head, 16 in all) than a patch call (1 per head), so the counters at the front of the
    # workspace (two per query tile of every pair, then two 64-bit ordering counters per
    # layer) are sized by it.  (Partial slots come after them only for calls that split; a
    # call whose preferred split does not fit the workspace takes a smaller one.)
    few = _cfg(heads=8, n_img=1024, n_patches=16, n_txt=8, head_dim=128, n_layers=1)
    many = _cfg(heads=8, n_img=1024, n_patches=16, n_txt=512, head_dim=128, n_layers=1)
    assert pa.pf_workspace_bytes(few) >= 8 * 2 * 2 * 4 + 16
    assert pa.pf_workspace_bytes(many) >= 16 * 2 * 2 * 4 + 16


def test_two_half_pipefusion_schedule_on_the_host():
    # the same rows as PIPEFUSION in twice the buffer memory; order enforced the same way;
    # only a step start can be restored; the half read starts at 0
    one = _cfg(n_layers=2)
    two = _cfg(n_layers=2, schedule=pa.PF_SCHED_PIPEFUSION_2H)
    assert pa.pf_kvbuf_bytes(two) == 2 * pa.pf_kvbuf_bytes(one)
    assert pa.pf_kvbuf_bytes(_cfg(schedule=3)) == 0
    ctx = pa.pf_create(two, [FAKE, FAKE])
    try:
        assert pa.pf_get_read_half(ctx, 0) == 0 and pa.pf_get_read_half(ctx, 1) == 0
        with pytest.raises(pa.PatchAttnError) as e:
            pa.pf_get_read_half(ctx, 2)
        assert e.value.status == pa.PF_ERR_INVALID_ARG
        with pytest.raises(pa.PatchAttnError) as e:
            pa.pf_set_state(ctx, 0, 1)
        assert e.value.status == pa.PF_ERR_UNSUPPORTED
        pa.pf_set_state(ctx, 0, 0)
        assert pa.pf_get_state(ctx, 0) == 0
        L = pa._lib()
        # patch 1 before patch 0 is out of order (checked before anything is enqueued)
        assert L.pf_patch_attn_step(ctx, 0, 1, FAKE, FAKE, FAKE, None, None, FAKE, None) == pa.PF_ERR_ORDER
    finally:
        pa.pf_destroy(ctx)


def test_selftest_rejects_limits_out_of_range():
    L = pa._lib()
    assert L.pf_selftest_bounded_wait(0, None) == pa.PF_ERR_INVALID_ARG
    assert L.pf_selftest_bounded_wait(10_000_000_001, None) == pa.PF_ERR_INVALID_ARG


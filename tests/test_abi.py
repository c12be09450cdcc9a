"""The C ABI library: it loads without a GPU, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call."""
import ctypes as ct
import os
import re

import pytest

from hybrid_model_ssm_replay_b200 import rssm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from hybrid_model_ssm_replay_b200 import build
    build.build()
    return rssm.lib()


def declared_functions():
    """Every function declared in include/*.h."""
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(rssm_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 18 and "rssm_stage_conv" in names and "rssm_stage_gate_norm" in names
    for n in names:
        assert hasattr(L, n), n
    assert L.rssm_abi_version() == 2


def cfg(**kw):
    base = dict(batch=256, nheads=64, head_dim=64, d_state=128, ngroups=8)
    base.update(kw)
    return rssm.make_desc(**base)


def test_check_desc():
    ok = cfg()
    assert rssm.rssm_check_desc(ok) == 0
    bad = [
        (dict(d_state=96), 2), (dict(nheads=63), 2), (dict(head_dim=0), 2), (dict(head_dim=257), 2),
        (dict(batch=0), 2), (dict(interval=0), 2), (dict(interval=30, max_draft=4), 2),
        (dict(max_draft=8), 2), (dict(in_dtype=2), 1), (dict(update_dtype=7), 1), (dict(out_copy=2), 1),
        (dict(update_dtype=rssm.RSSM_FP4, out_copy=rssm.RSSM_OUTCOPY_FP4), 3),
        (dict(flags=2), 1), (dict(flags=1, update_dtype=rssm.RSSM_BF16), 3),
        (dict(head_dim=3, d_state=16, update_dtype=rssm.RSSM_FP4), 2),
    ]
    for kw, status in bad:
        assert rssm.rssm_check_desc(cfg(**kw)) == status, kw
    d = cfg()
    d.reserved = 1
    assert rssm.rssm_check_desc(d) == 1
    assert rssm.lib().rssm_check_desc(None) == 1


def test_field_bytes():
    d = cfg()
    fb = lambda f: rssm.rssm_state_field_bytes(d, f)
    # fp32 checkpoint 64 x 128, dt 16 floats, x 16 rows of 64 bf16: 34880 -> 128-byte multiple
    lay = rssm.rssm_record_layout(d)
    assert (lay.tile_bytes, lay.scales_offset, lay.dt_offset, lay.x_offset) == (32768, 0, 32768, 32832)
    assert lay.bytes == 34944
    assert fb(rssm.FIELD_RECORD) == 256 * 64 * 34944
    assert fb(rssm.FIELD_CKPT) == 0
    assert fb(rssm.FIELD_BBUF) == 256 * 8 * 16 * 128 * 2
    assert fb(rssm.FIELD_POS) == fb(rssm.FIELD_ARRIVE) == 1024 and fb(rssm.FIELD_ERR) == 4
    # dt rows round the capacity up to a multiple of 4
    l1 = rssm.rssm_record_layout(cfg(max_draft=1))
    assert l1.x_offset - l1.dt_offset == 20 * 4
    # split precision: the record holds the FP4 output copy, the bf16 update copy is separate
    s = cfg(update_dtype=rssm.RSSM_BF16, out_copy=rssm.RSSM_OUTCOPY_FP4, max_draft=4)
    fs = lambda f: rssm.rssm_state_field_bytes(s, f)
    ls = rssm.rssm_record_layout(s)
    assert (ls.tile_bytes, ls.scales_offset, ls.dt_offset, ls.x_offset) == (4096, 4096, 4608, 4688)
    assert ls.bytes == 7296  # 4688 + 20 rows x 64 x 2 = 7248 -> 7296
    assert fs(rssm.FIELD_CKPT) == 256 << 20
    assert fs(rssm.FIELD_RECORD) == 256 * 64 * 7296
    # shared FP4: codes and scales in the record, nothing separate
    f4 = cfg(update_dtype=rssm.RSSM_FP4, in_dtype=rssm.RSSM_F32)
    l4 = rssm.rssm_record_layout(f4)
    assert (l4.scales_offset, l4.dt_offset, l4.x_offset, l4.bytes) == (4096, 4608, 4672, 8832)
    assert rssm.rssm_state_field_bytes(f4, rssm.FIELD_CKPT) == 0
    assert rssm.rssm_state_field_bytes(cfg(d_state=7), rssm.FIELD_RECORD) == 0
    assert rssm.rssm_state_field_bytes(d, 99) == 0
    assert rssm.lib().rssm_record_layout(ct.byref(cfg(d_state=7)), ct.byref(rssm.RecordLayout())) == 2
    assert rssm.lib().rssm_record_layout(ct.byref(d), None) == 1


def fake_state():
    # non-null placeholders: the calls below must fail validation before any device access
    return rssm.StateStruct(*([0x1000] * 7))


def test_host_validation_needs_no_device(L):
    d = cfg(max_draft=2)
    st = fake_state()
    p = ct.c_void_p(0x1000)
    null = None
    # null state / null inputs
    assert L.rssm_decode_step(ct.byref(d), None, p, p, p, p, p, p, p, None) == 1
    assert L.rssm_decode_step(ct.byref(d), ct.byref(st), null, p, p, p, p, p, p, None) == 1
    # verify with too many drafts
    assert L.rssm_verify(ct.byref(d), ct.byref(st), 3, p, p, p, p, p, p, p, None) == 4
    assert L.rssm_verify(ct.byref(d), ct.byref(st), -1, p, p, p, p, p, p, p, None) == 4
    # fp32 flush on a split-precision state is refused
    dl = cfg(update_dtype=rssm.RSSM_BF16, out_copy=rssm.RSSM_OUTCOPY_FP4)
    assert L.rssm_flush(ct.byref(dl), ct.byref(st), p, 0, None) == 3
    # invalid descriptions propagate from every entry point
    bad = cfg(d_state=100)
    assert L.rssm_flush(ct.byref(bad), ct.byref(st), p, 0, None) == 2
    assert L.rssm_lowprec_refresh(ct.byref(bad), ct.byref(st), p, 0, None) == 2
    assert L.rssm_accept(ct.byref(bad), ct.byref(st), p, None) == 2
    assert L.rssm_conv_step(ct.byref(bad), p, p, p, p, p, p, p, p, None) == 2
    assert L.rssm_conv_verify(ct.byref(d), p, p, 8, p, p, p, p, p, p, p, None) == 4
    assert L.rssm_conv_accept(ct.byref(d), None, p, 1, None, None) == 1
    # a split-precision state needs its separate update copy; every state needs records
    st2 = fake_state()
    st2.ckpt = None
    assert L.rssm_lowprec_refresh(ct.byref(dl), ct.byref(st2), p, 0, None) == 1
    st3 = fake_state()
    st3.record = None
    assert L.rssm_decode_step(ct.byref(d), ct.byref(st3), p, p, p, p, p, p, p, None) == 1
    assert L.rssm_get_error(ct.byref(d), None, None, None) == 1
    assert L.rssm_round_test(9, 16, p, 0, 0, 0, 0, p, None) == 1
    assert L.rssm_round_test(3, 15, p, 0, 0, 0, 0, p, None) == 2
    # prefill: fp32 state only, T0 >= 0, inputs needed when T0 > 0
    assert L.rssm_prefill(ct.byref(dl), ct.byref(st), 4, p, p, p, p, None) == 3
    assert L.rssm_prefill(ct.byref(d), ct.byref(st), -1, p, p, p, p, None) == 1
    assert L.rssm_prefill(ct.byref(d), ct.byref(st), 4, null, p, p, p, None) == 1
    assert L.rssm_prefill(ct.byref(bad), ct.byref(st), 4, p, p, p, p, None) == 2
    assert rssm.status_string(4) == "more tokens than the buffer capacity"


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        rssm._ptr(torch.zeros(4), torch.float32, "x")


def test_stage_calls_reject_bad_arguments_on_the_host(L):
    """The stage's element-wise calls check their arguments before any CUDA
    call: null pointers, an fp32 input description, a bad eps."""
    from hybrid_model_ssm_replay_b200 import stage  # noqa: F401  (sets the signatures)
    stage._lib()
    d = cfg()
    p = ct.c_void_p(0x1000)
    assert L.rssm_stage_conv(ct.byref(d), None, p, p, p, p, p, p, p, p, None) == 1
    assert L.rssm_stage_gate_norm(ct.byref(d), p, p, p, ct.c_float(0.0), p, None) == 1
    f = cfg(in_dtype=rssm.RSSM_F32)
    assert L.rssm_stage_conv(ct.byref(f), p, p, p, p, p, p, p, p, p, None) == 3
    assert L.rssm_stage_gate_norm(ct.byref(f), p, p, p, ct.c_float(1e-5), p, None) == 3
    assert L.rssm_stage_conv(None, p, p, p, p, p, p, p, p, p, None) == 1

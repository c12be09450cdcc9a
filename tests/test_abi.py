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
    text = open(os.path.join(ROOT, "include", "rssm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rssm_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert L.rssm_abi_version() == 1


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
    assert fb(rssm.FIELD_CKPT) == 256 * 64 * 64 * 128 * 4 == 512 << 20
    assert fb(rssm.FIELD_CKPT_SCALES) == 0 and fb(rssm.FIELD_OUT_CODES) == 0
    assert fb(rssm.FIELD_XBUF) == 256 * 64 * 16 * 64 * 2
    assert fb(rssm.FIELD_BBUF) == 256 * 8 * 16 * 128 * 2
    assert fb(rssm.FIELD_DTBUF) == 256 * 64 * 16 * 4
    assert rssm.rssm_state_field_bytes(cfg(max_draft=1), rssm.FIELD_DTBUF) == 256 * 64 * 20 * 4
    assert fb(rssm.FIELD_POS) == fb(rssm.FIELD_ARRIVE) == 1024 and fb(rssm.FIELD_ERR) == 4
    s = cfg(update_dtype=rssm.RSSM_BF16, out_copy=rssm.RSSM_OUTCOPY_FP4, max_draft=4)
    fs = lambda f: rssm.rssm_state_field_bytes(s, f)
    assert fs(rssm.FIELD_CKPT) == 256 << 20
    assert fs(rssm.FIELD_OUT_CODES) == 64 << 20 and fs(rssm.FIELD_OUT_SCALES) == 8 << 20
    assert fs(rssm.FIELD_XBUF) == 256 * 64 * 20 * 64 * 2
    assert rssm.rssm_state_field_bytes(cfg(d_state=7), rssm.FIELD_CKPT) == 0
    assert rssm.rssm_state_field_bytes(d, 99) == 0


def fake_state():
    # non-null placeholders: the calls below must fail validation before any device access
    return rssm.StateStruct(*([0x1000] * 11))


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
    # missing FP4 copy pointers
    st2 = fake_state()
    st2.out_codes = None
    assert L.rssm_lowprec_refresh(ct.byref(dl), ct.byref(st2), p, 0, None) == 1
    assert L.rssm_get_error(ct.byref(d), None, None, None) == 1
    assert L.rssm_round_test(9, 16, p, 0, 0, 0, 0, p, None) == 1
    assert L.rssm_round_test(3, 15, p, 0, 0, 0, 0, p, None) == 2
    assert rssm.status_string(4) == "more tokens than the buffer capacity"


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        rssm._ptr(torch.zeros(4), torch.float32, "x")

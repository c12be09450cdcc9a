"""RssmState's named views map onto the record geometry the library reports
(rssm_record_layout): every view aliases the bytes rssm.h assigns to it.
Host-only (the state is allocated on the CPU here; no kernel runs)."""
import pytest
import torch

from hybrid_model_ssm_replay_b200 import rssm


def byte_offset(view, base):
    return view.data_ptr() - base.data_ptr()


@pytest.mark.parametrize("kw", [dict(), dict(update_dtype=rssm.RSSM_BF16, out_copy=rssm.RSSM_OUTCOPY_FP4),
                                dict(update_dtype=rssm.RSSM_FP4), dict(update_dtype=rssm.RSSM_E4M3),
                                dict(in_dtype=rssm.RSSM_F32, max_draft=4)],
                         ids=["f32", "bf16+fp4", "shared-fp4", "shared-e4m3", "f32-inputs-k4"])
def test_views_follow_the_record_layout(kw):
    d = rssm.make_desc(3, 4, 32, 128, 2, **kw)
    st = rssm.RssmState(d, device="cpu")
    lay = rssm.rssm_record_layout(d)
    B, H, P, N = 3, 4, 32, 128
    cap = d.interval + d.max_draft
    es = 2 if d.in_dtype == rssm.RSSM_BF16 else 4
    rec = st.record
    assert tuple(rec.shape) == (B, H, lay.bytes) and rec.is_contiguous()
    # (b, h) record at (b H + h) * bytes; x rows and dt inside it
    b, h = 2, 3
    base = (b * H + h) * lay.bytes
    assert byte_offset(st.xbuf[b, h, 0], rec) == base + lay.x_offset
    assert byte_offset(st.xbuf[b, h, 1], rec) == base + lay.x_offset + P * es
    assert byte_offset(st.dtbuf[b, h], rec) == base + lay.dt_offset
    assert tuple(st.xbuf.shape) == (B, H, cap, P) and tuple(st.dtbuf.shape) == (B, H, (cap + 3) // 4 * 4)
    if d.out_copy == rssm.RSSM_OUTCOPY_FP4:
        assert byte_offset(st.out_codes[b, h], rec) == base
        assert byte_offset(st.out_scales[b, h], rec) == base + lay.scales_offset
        assert st.ckpt.is_contiguous() and st.struct.ckpt == st.ckpt.data_ptr()
    else:
        assert byte_offset(st.ckpt[b, h], rec) == base and st.struct.ckpt is None
        if d.update_dtype == rssm.RSSM_FP4:
            assert byte_offset(st.ckpt_scales[b, h], rec) == base + lay.scales_offset
    assert st.struct.record == rec.data_ptr() and st.struct.bbuf == st.bbuf.data_ptr()
    assert tuple(st.bbuf.shape) == (B, 2, cap, N)
    # a write through a view lands in the record bytes
    st.dtbuf[1, 2, 5] = 3.5
    off = (1 * H + 2) * lay.bytes + lay.dt_offset + 5 * 4
    assert rec.view(-1)[off:off + 4].view(torch.float32).item() == 3.5

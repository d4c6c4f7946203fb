"""Host-side facts of the step pipeline that need no GPU.

The end-to-end measurement copies a step's per-request inputs in and its
scores out every step.  These checks pin which tensors count as per-request
(the fields the two-slot host pipeline double-buffers) and the byte counts
the bench reports for the standard workload.
"""
import dataclasses

from recsys_decoupled_link_b200 import pipeline, synth


def test_request_fields_are_device_inputs():
    names = {f.name for f in dataclasses.fields(pipeline.DeviceInputs)}
    assert set(pipeline.REQUEST_FIELDS) <= names
    # the model state stays resident: weights, global links, item table
    for resident in ("L", "layers", "ctx_w", "T", "Wq_c", "Wk_c"):
        assert resident not in pipeline.REQUEST_FIELDS


def test_standard_step_copy_bytes():
    # 64 users x 1,024 history rows of d = 128 bf16, a 64-wide bf16 context per
    # user, 1,024 int32 candidate IDs per user, two int64 offset arrays of
    # B + 1 entries; the scores are [65,536 x 128] bf16
    w = synth.workload("standard")
    us, cs = synth.user_side(w), synth.candidate_side(w)
    req = {"E": us.E, "ctx": us.ctx, "hist_offsets": us.hist_offsets,
           "cand_ids": cs.cand_ids, "cand_offsets": cs.cand_offsets}
    assert set(req) == set(pipeline.REQUEST_FIELDS)
    h2d = sum(t.numel() * t.element_size() for t in req.values())
    assert h2d == 65536 * 128 * 2 + 64 * 64 * 2 + 65 * 8 + 65536 * 4 + 65 * 8 == 17_048_592
    d2h = int(cs.cand_offsets[-1]) * w.d * 2
    assert d2h == 16_777_216

"""The two-stage QK-cache build (lime_fold_qk on its own stream, then
lime_build_qk_cache_folded) against the one-call build and the fp64 oracle.

Both forms run the same kernels on the same folded image, so their caches
must agree bit for bit; the oracle check uses the bf16 tolerance (max-abs
<= 2e-2, rel-L2 <= 5e-3).  The full step with the fold forked onto a side
stream must also give the same scores, bit for bit, as the step run in one
stream with the one-call build.
"""
import pytest
import torch

from oracle import lime_oracle as O
from recsys_decoupled_link_b200 import lime, pipeline, synth
from parity_util import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,l,n_items", [(4, 32, 1000), (4, 16, 300), (4, 64, 257),
                                         (2, 32, 129), (8, 32, 1)])
def test_two_stage_cache_matches_one_call_and_oracle(H, l, n_items):
    w = synth.workload("standard", H=H, l=l, n_items=n_items, B=2, layers=1)
    us = synth.user_side(w, [1, 1])
    cs = synth.candidate_side(w, [1, 1])
    T = synth.item_table(w)
    dims = lime.make_dims(w.d, H, l, w.f, w.c, "bf16")
    Td, Ld, Wq, Wk = (t.cuda() for t in (T, us.L, cs.Wq_c, cs.Wk_c))
    ws = lime.Workspace(dims, 0, 0)
    one = torch.empty(n_items, H, l, dtype=torch.bfloat16, device="cuda")
    two = torch.full_like(one, float("nan"))
    lime.lime_build_qk_cache(dims, Td, Ld, Wq, Wk, one, ws)
    image = torch.empty(lime.lime_qk_image_bytes(dims), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    lime.lime_fold_qk(dims, Ld, Wq, Wk, image, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    lime.lime_build_qk_cache_folded(dims, Td, image, two, ws)
    torch.cuda.synchronize()
    assert lime.lime_get_status(ws) == 0
    assert torch.equal(one.view(torch.int16), two.view(torch.int16))
    ref = O.qk_cache(f64(T), f64(us.L), f64(cs.Wq_c), f64(cs.Wk_c), H)
    assert_close(two, ref, "bf16", "two-stage QK cache")


def test_forked_step_matches_single_stream_step():
    w = synth.workload("standard", B=8, n_items=5000)
    us = synth.user_side(w)
    cs = synth.candidate_side(w)
    T = synth.item_table(w)
    x = pipeline.to_device(w, us, cs, T)
    buf = pipeline.alloc(x)
    assert buf.image is not None
    for _ in range(2):                 # the second step overwrites the image again
        O_fork = pipeline.step(x, buf).clone()
    LP = pipeline.user_encode(x, buf)
    pipeline.build_cache(x, buf)       # one-call build on the main stream
    pipeline.score(x, buf, LP)
    torch.cuda.synchronize()
    assert lime.lime_get_status(buf.ws) == 0
    assert torch.equal(O_fork.view(torch.int16), buf.O.view(torch.int16))


def test_graph_replay_matches_eager():
    # the step captured in CUDA graphs (whole step; and user side, cache,
    # scoring as three graphs) replays to the eager step's scores bit for bit
    w = synth.workload("standard", B=8, n_items=5000)
    x = pipeline.to_device(w, synth.user_side(w), synth.candidate_side(w), synth.item_table(w))
    buf = pipeline.alloc(x)
    O_eager = pipeline.step(x, buf).clone()
    graphs = pipeline.step_graphs(x, buf)
    for replay in ([graphs[0]], graphs[1:]):
        buf.O.zero_()
        buf.cache.zero_()
        for g in replay:
            g.replay()
        torch.cuda.synchronize()
        assert lime.lime_get_status(buf.ws) == 0
        assert torch.equal(O_eager.view(torch.int16), buf.O.view(torch.int16))


def test_host_pipeline_alternating_batches_match_single_steps():
    # two request batches of the same shapes (different histories, contexts
    # and candidate IDs; shared weights and catalogue) submitted as A, B, A, B
    # through the two-slot host pipeline give each batch's single-step scores
    # bit for bit: neither slot's inputs nor scores leak into the other's
    import dataclasses
    w = synth.workload("standard", B=4, n_items=5000)
    n_hist, n_cand = [300, 0, 129, 1024], [64, 3, 100, 200]
    xa = pipeline.to_device(w, synth.user_side(w, n_hist), synth.candidate_side(w, n_cand),
                            synth.item_table(w))
    w2 = dataclasses.replace(w, seed=w.seed + 77)
    src = pipeline.to_device(w2, synth.user_side(w2, n_hist), synth.candidate_side(w2, n_cand),
                             None)
    xb = dataclasses.replace(xa, **{k: getattr(src, k) for k in pipeline.REQUEST_FIELDS})
    buf = pipeline.alloc(xa)
    ref = [pipeline.step(xa, buf).clone(), pipeline.step(xb, buf).clone()]
    assert not torch.equal(ref[0], ref[1])
    host = [{k: getattr(xs, k).cpu().pin_memory() for k in pipeline.REQUEST_FIELDS}
            for xs in (xa, xb)]
    outs = [torch.empty(buf.O.shape, dtype=buf.O.dtype).pin_memory() for _ in range(4)]
    hp = pipeline.HostPipeline(xa, buf)
    hp.start()
    for k in range(4):
        hp.submit(host[k % 2], outs[k])
    hp.drain()
    torch.cuda.synchronize()
    assert lime.lime_get_status(buf.ws) == 0
    for k in range(4):
        assert torch.equal(outs[k].view(torch.int16), ref[k % 2].cpu().view(torch.int16)), k

"""The layer stack captured into a CUDA graph before any eager call.

On the tensor-core path a non-final LIME-XOR layer runs its link tail on a
library-owned side stream beside the history GatedMLP.  The library creates
that stream on the first call on a device that is not being captured; a
capture that comes first must run the layer in order on the capturing stream
instead, and give the same link rows, bit for bit, as the forked eager call
that follows it.  The check runs in a fresh process, so that no earlier test
has created the side stream already.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SCRIPT = r"""
import torch
from recsys_decoupled_link_b200 import lime, pipeline, synth

torch.cuda.set_device(0)
w = synth.workload("standard", B=4, n_items=1000, layers=3)
x = pipeline.to_device(w, synth.user_side(w, [300, 0, 129, 1024]),
                       synth.candidate_side(w, [5, 5, 5, 5]), synth.item_table(w))
buf = pipeline.alloc(x)
pipeline.build_cache(x, buf)   # library set-up (tensor-map encoder) outside the capture
torch.cuda.synchronize()
g = torch.cuda.CUDAGraph()
with torch.cuda.graph(g):
    LP = pipeline.user_encode(x, buf)
g.replay()
torch.cuda.synchronize()
LP_graph = LP.clone()
LP_eager = pipeline.user_encode(x, buf).clone()
torch.cuda.synchronize()
assert lime.lime_get_status(buf.ws) == 0, "device status flags set"
assert torch.equal(LP_graph.view(torch.int16), LP_eager.view(torch.int16)), "graph != eager"
print("capture-first ok")
"""


def test_layers_captured_before_any_eager_call_match_the_forked_eager_calls():
    # every kernel is loaded with the library, so none is first loaded inside the capture
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""),
               CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _SCRIPT], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "capture-first ok" in r.stdout, r.stdout + r.stderr

"""The bench's pipelined end-to-end leg moves the same bytes and computes the same results as
one step run on its own: host -> device and device -> host copies on their own streams, two
alternating sets of device buffers, events ordering every copy (a missing edge would show as
results taken from the wrong step's buffers or before a GEMM finished)."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402
from nvfp4_testlib import need_gpu  # noqa: E402

pytestmark = pytest.mark.gpu


def test_pipelined_end_to_end_matches_a_plain_step():
    need_gpu()
    dev = torch.device("cuda", 0)
    wl = synth.Workload("e2e_check", 7, [synth.Linear("a", 1024, 1024, 2048),
                                         synth.Linear("b", 1024, 2048, 1024)])
    step = bench.Step(wl, dev)
    # reference: one plain step on the step's own buffers, results copied synchronously
    step.run()
    torch.cuda.synchronize()
    ref = [L["out"][op].cpu().clone() for L in step.layers for op in bench.OPS]
    assert int(step.dev_status.item()) == 0
    # poison the device outputs of both buffer sets, then run the pipelined leg for 5 steps
    for L in step.layers:
        for op in bench.OPS:
            L["out"][op].fill_(float("nan"))
    outs = step.output_host_buffers()
    for o in outs:
        o.fill_(float("nan"))
    step.run_end_to_end(5, outs)
    torch.cuda.synchronize()
    assert int(step.dev_status.item()) == 0
    for k, (o, r) in enumerate(zip(outs, ref)):
        assert torch.equal(o.view(torch.int16 if o.dtype == torch.bfloat16 else torch.int32),
                           r.view(torch.int16 if r.dtype == torch.bfloat16 else torch.int32)), k

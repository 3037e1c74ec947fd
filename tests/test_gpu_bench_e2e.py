"""The bench's end-to-end steps on the GPU: with the copies of neighbouring
steps overlapped (two device buffer sets, two copy streams), every result read
back must equal the serial step's result bit for bit (every step has the same
inputs), for each kind of step the bench times."""
import os
import sys

import pytest
import torch

from gpu_util import require_gpu

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("llama", {}),
                                     ("mix", {}), ("long", {}),
                                     ("prefill", {}),
                                     ("llama", {"unfused": True})],
                         ids=["tiny-fused", "llama-fused", "mix-balanced",
                              "long-split", "prefill", "llama-unfused"])
def test_pipelined_steps_read_back_the_serial_result(name, kw):
    device = torch.device("cuda", 0)
    wl = bench._workload(name)
    r = bench.TVRunner(wl, name, device, **kw)
    r.setup_e2e()
    r.e2e_step()
    torch.cuda.synchronize()
    ref = r.h_out.clone()
    r.setup_e2e_pipelined()
    for _ in range(5):          # both buffer sets, each reused
        r.e2e_step_pipelined()
    r.e2e_join()
    torch.cuda.synchronize()
    for _, _, _, h_out in r.e2e_sets:
        assert torch.equal(h_out.view(torch.int16), ref.view(torch.int16))
    assert int(r.db.err.item()) == 0
    assert r.h_stage.numel() >= sum(t.numel() * t.element_size()
                                    for t in r.h_in.values())

"""The end-to-end path with host buffers: steps pipelined over two sets of
device buffers hand back exactly what the device computed, and the same
results as one step at a time."""
import pytest
import torch

from swiglu_ar_tts_b200.step import Step, run_e2e_pipelined

pytestmark = pytest.mark.gpu


def test_pipelined_end_to_end_steps_match_serial_steps():
    dev = torch.device("cuda", torch.cuda.current_device())
    a = Step(dev)
    a.setup_e2e()
    b = Step(dev, like=a)
    b.setup_e2e(share=a)
    run_e2e_pipelined([a, b], 4)  # steps 0..3 on sets a, b, a, b
    torch.cuda.synchronize()
    assert (a.decode_step_index, b.decode_step_index) == (2, 2)
    host = {}
    for g, _ in b.E2E_GROUPS:
        host[g] = []
        for dst, src in b._e2e_out(g):  # the last step ran on set b
            assert torch.equal(dst, src.cpu()), f"{g}: host copy differs from the device"
            host[g].append(dst.clone())
    # one serial step on fresh buffers at the same decode position
    c = Step(dev, like=a)
    c.setup_e2e()
    c.decode_step_index = 1
    c.run_e2e()
    torch.cuda.synchronize()
    for g, _ in c.E2E_GROUPS:
        for (dst, _), h in zip(c._e2e_out(g), host[g]):
            assert torch.equal(dst, h), f"{g}: pipelined and serial steps differ"

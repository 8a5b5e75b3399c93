"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The grid barrier of the layer kernel waits for a count that a test hook has
made unreachable (one CTA is told not to arrive).  Every CTA gives up after the 2 s limit, records the
"grid barrier wait gave up" bit in the device error word and runs to its end.
The host then reads the error through ts_moe_device_status.  That call re-zeroes
the handle's counters, and the next call is the same, bit for bit, as one made
before the hook ran."""
import time

import pytest
import torch

from quantized_moe_routed_router_b200 import synth

pytestmark = pytest.mark.gpu

EDEVICE = 5
ERR_TIMEOUT_GRID = 0x40


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_moe_routed_router_b200 import build
    build.build()


def test_grid_barrier_wait_gives_up_and_the_handle_recovers():
    from quantized_moe_routed_router_b200 import binding
    shape = synth.MoEShape("wait", 256, 256, 8, 2, cfg_id=131)
    moe = binding.MoE(shape, [synth.make_layer(shape, 0, device="cuda")])
    x = synth.make_x(shape, 0, 16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream

    y_ref = torch.empty(16, shape.hidden, device="cuda")
    moe.forward(0, x, None, y_ref)
    moe.device_status()

    assert binding.lib.ts_moe_debug_skew_barrier(moe.h, stream) == 0
    y = torch.empty_like(y_ref)
    t0 = time.monotonic()
    moe.forward(0, x, None, y)
    with pytest.raises(binding.TsMoeError) as err:
        moe.device_status()
    waited = time.monotonic() - t0
    assert err.value.status == EDEVICE
    word = int(str(err.value).split("device error word 0x")[1].split()[0], 16)
    assert word == ERR_TIMEOUT_GRID, hex(word)
    assert waited >= 1.5, waited                     # the wait ran to its limit

    for _ in range(2):                               # the counters were re-zeroed
        y2 = torch.empty_like(y_ref)
        moe.forward(0, x, None, y2)
        moe.device_status()
        assert torch.equal(y2, y_ref)
    moe.close()

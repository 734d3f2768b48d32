"""The end-to-end entry points from host memory: one batch (``forward_host``) and a
pipelined sequence of batches whose copies overlap the neighbouring layer calls
(``forward_host_stream``) give, in pinned host memory, exactly what the layer gives on the
device (fixed-order mode, so every call is bit-for-bit repeatable)."""
import pytest
import torch

from workloads import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["decode", "tiny"])
def test_host_entry_points_match_the_device_call(moe, name):
    inp = make_inputs(CONFIGS[name]).to("cuda")
    layer = moe.MoELayer.from_inputs(inp, deterministic=True)
    g = torch.Generator(device="cuda").manual_seed(3)
    xs = [inp.x] + [torch.randn(inp.x.shape, generator=g, device="cuda").to(torch.bfloat16)
                    for _ in range(4)]
    want = [layer(x).cpu() for x in xs]
    torch.cuda.synchronize()

    x_hosts = [x.cpu().pin_memory() for x in xs]
    y_hosts = [torch.empty_like(w).pin_memory() for w in want]
    x_devs = [torch.empty_like(inp.x) for _ in range(2)]
    y_devs = [torch.empty_like(inp.x) for _ in range(2)]
    # five batches through two device buffers each: buffer reuse waits on both copy streams
    layer.forward_host_stream(x_hosts, y_hosts, x_devs, y_devs)
    torch.cuda.synchronize()
    for i, (got, ref) in enumerate(zip(y_hosts, want)):
        assert torch.equal(got, ref), f"batch {i}"

    y_host = torch.empty_like(want[2]).pin_memory()
    layer.forward_host(x_hosts[2], y_host, x_devs[0], y_devs[0])
    torch.cuda.synchronize()
    assert torch.equal(y_host, want[2])
    assert layer.device_status() == 0

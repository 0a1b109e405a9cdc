"""strata_moe_forward_noalloc against strata_moe_forward, through the C interface.

The no-allocation forward runs the ordinary small-batch kernels with their
workspace in the library's fixed device array, so its output must equal the
ordinary forward's bit for bit -- on two calls in a row, the second of which
finds what the first left in the array.  This file is collected last on
purpose: it must pass both alone in a fresh process and after every other
test has used the library."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(torch, t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


# (config, tokens of the first call, tokens of the second call)
CASES = [("dsv2lite", 8, 3), ("tiny", 64, 5), ("mixtral", 4, 1)]


@pytest.mark.parametrize("name,t1,t2", CASES)
def test_noalloc_matches_forward_twice(name, t1, t2):
    import torch

    from quantized_routed_expert_04_b200.binding import Status
    from tests.harness import GpuLayer
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg)  # a fresh handle whose own workspace was never grown
    xs = [lay.x_dev(synth.make_x(cfg, t, step=20 + i)) for i, t in enumerate((t1, t2))]
    outs = [torch.full_like(x, 7) for x in xs]
    refs = [torch.full_like(x, 7) for x in xs]
    torch.cuda.synchronize()

    lay.layer.forward_noalloc(xs[0], outs[0])
    assert lay.layer.status()[0] == Status.OK
    free_before = torch.cuda.mem_get_info()[0]
    lay.layer.forward_noalloc(xs[1], outs[1])
    assert lay.layer.status()[0] == Status.OK
    assert torch.cuda.mem_get_info()[0] == free_before

    for x, ref in zip(xs, refs):
        lay.layer.forward(x, ref)
        assert lay.layer.status()[0] == Status.OK
    for out, ref in zip(outs, refs):
        assert _bits(torch, out).tolist() == _bits(torch, ref).tolist()
    lay.close()


def test_noalloc_rejects_requests_beyond_the_scratch():
    import torch

    from quantized_routed_expert_04_b200 import binding
    from quantized_routed_expert_04_b200.binding import Status, StrataError
    # y alone needs 64 * 8 * 8192 * 4 bytes = 16 MiB at 64 tokens
    H, I, E, k = 8192, 1024, 64, 8
    lay = binding.StrataMoE(H, I, E, k, 0, E)
    W = torch.zeros(E, H, dtype=torch.float32, device="cuda")
    lay.set_router(W)
    for T in (binding.NOALLOC_MAX_TOKENS + 1, binding.NOALLOC_MAX_TOKENS):
        x = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
        out = torch.zeros_like(x)
        with pytest.raises(StrataError) as err:
            lay.forward_noalloc(x, out)
        assert err.value.status == Status.SCRATCH_LIMIT
        assert lay.status()[0] == Status.OK  # nothing was enqueued
        assert not out.any()
    lay.close()

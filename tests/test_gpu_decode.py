"""The small-batch (decode) layer kernel, one cooperative launch per forward,
through the C interface: both top-k paths (every CTA selecting all tokens, or
one token per CTA published through a grid barrier), the largest small batch,
and the time-out path of its bounded waits (a wait limit short enough that
waits run out: the status is reported, nothing faults, and the next call is
clean and bit-identical to one before)."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth
from tests.harness import GpuLayer, assert_within_tolerance, oracle_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_routed_expert_04_b200 import build
    build.build()


@pytest.mark.parametrize("name,T", [("dsv2lite", 12), ("dsv2lite", 13), ("dsv2lite", 9),
                                    ("mixtral", 2), ("wide", 64), ("sigmoid", 20)])
def test_decode_token_counts(name, T):
    """12 tokens: every CTA selects; 13: one token per CTA; 9: 16-pair items;
    64: the largest small batch."""
    import oracle
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg, bind="all" if cfg.n_slots == cfg.n_experts else "none")
    if cfg.routing == "sigmoid":
        from quantized_routed_expert_04_b200 import binding
        corr = synth.make_correction_bias(cfg, 0)
        lay.corr_dev = lay.torch.from_numpy(corr).cuda()
        lay.layer.set_routing(binding.ROUTE_SIGMOID, lay.corr_dev, cfg.routed_scale)
        x = synth.make_x(cfg, T, step=31)
        _, idx, w = oracle.route_sigmoid(x, lay.W, lay.b, corr, cfg.routed_scale, cfg.top_k)
        ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x, idx, w)
    else:
        x = synth.make_x(cfg, T, step=31)
        ref, idx, w = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    if cfg.n_slots < cfg.n_experts:
        distinct = sorted(set(idx.reshape(-1).tolist()))
        if len(distinct) > cfg.n_slots:
            pytest.skip("more distinct experts than slots")
        lay.bind_only(distinct)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    assert_within_tolerance(out, ref, "%s T=%d" % (name, T))
    lay.close()


@pytest.mark.parametrize("T", [8, 20])
def test_wait_timeout_reports_and_recovers(T):
    from quantized_routed_expert_04_b200.binding import DEFAULT_WAIT_NS, Status
    cfg = synth.CONFIGS["dsv2lite"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=32)
    st, ref = lay.forward(x)
    assert int(st[0]) == 0
    lay.layer.set_wait_limit(0)          # every wait not already satisfied gives up
    (st, bits), _ = lay.forward(x)
    assert st == Status.DEVICE_STATUS and bits & 4, (st, bits)
    lay.layer.set_wait_limit(DEFAULT_WAIT_NS)
    for _ in range(2):
        (st, bits), out = lay.forward(x)
        assert st == Status.OK and bits == 0, (st, bits)
        assert np.array_equal(out, ref)
    lay.close()


def test_forward_routed_matches_forward_bitwise():
    """The kernel with the routing given (skipping its router) and with the
    routing computed give the same output bit for bit."""
    import oracle
    cfg = synth.CONFIGS["dsv2lite"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 8, step=33)
    st, a = lay.forward(x)
    assert int(st[0]) == 0
    _, idx, w = lay.route(x)
    _, oidx, _ = oracle.route(x, lay.W, lay.b, cfg.top_k)
    np.testing.assert_array_equal(idx, oidx)
    st, b = lay.forward_routed(x, idx, w)
    assert int(st[0]) == 0
    assert np.array_equal(a, b)
    lay.close()

"""Sigmoid routing with a correction bias and a routed scale, on the GPU
against the CPU oracle: routing (small-batch and large-batch paths) and the
whole layer."""
import dataclasses

import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth
from tests.harness import GpuLayer, assert_within_tolerance, oracle_reference

pytestmark = pytest.mark.gpu


def ulp_diff(a, b):
    return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))


def _sigmoid_layer(cfg, blobs=None):
    import torch

    from quantized_routed_expert_04_b200 import binding
    lay = GpuLayer(cfg, blobs=blobs)
    corr = synth.make_correction_bias(cfg)
    corr_dev = torch.from_numpy(corr).cuda()
    lay.layer.set_routing(binding.ROUTE_SIGMOID, corr_dev, cfg.routed_scale)
    lay.corr, lay.corr_dev = corr, corr_dev
    return lay


@pytest.mark.parametrize("T", [4, 64, 200])   # route_small (<= 64), router GEMM + top-k
def test_sigmoid_route_matches_oracle(T):
    import oracle
    cfg = synth.CONFIGS["sigmoid"]
    lay = _sigmoid_layer(cfg, blobs=np.zeros((cfg.n_experts, 256), np.uint8))
    x = synth.make_x(cfg, T, step=7)
    logits, idx, w = lay.route(x)
    rl, ridx, rw = oracle.route_sigmoid(x, lay.W, lay.b, lay.corr, cfg.routed_scale, cfg.top_k)
    assert ulp_diff(logits, rl).max() <= 1
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=1e-7)
    np.testing.assert_allclose(w.sum(axis=1), cfg.routed_scale, rtol=1e-5)
    lay.close()


@pytest.mark.parametrize("T", [8, 100])
def test_sigmoid_forward_matches_oracle(T):
    import oracle
    base = synth.custom_config("sigfwd", 512, 256, 32, 4, n_shared=1, tokens=(T,))
    cfg = dataclasses.replace(base, routing="sigmoid", routed_scale=2.5)
    lay = _sigmoid_layer(cfg)
    x = synth.make_x(cfg, T, step=2)
    st, out = lay.forward(x)
    assert int(st[0]) == 0
    _, idx, w = oracle.route_sigmoid(x, lay.W, lay.b, lay.corr, cfg.routed_scale, cfg.top_k)
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x, idx, w)
    assert_within_tolerance(out, ref, "sigmoid T=%d" % T)
    lay.close()


def test_set_routing_rejects_bad_arguments():
    import torch

    from quantized_routed_expert_04_b200 import binding
    cfg = synth.CONFIGS["tiny"]
    lay = binding.StrataMoE(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k, 0, cfg.n_slots)
    corr = torch.zeros(cfg.n_experts, dtype=torch.float32, device="cuda")
    for args in [(2, None, 1.0), (binding.ROUTE_SIGMOID, None, 0.0),
                 (binding.ROUTE_SIGMOID, None, float("inf")), (binding.ROUTE_SOFTMAX, corr, 1.0),
                 (binding.ROUTE_SOFTMAX, None, 2.0)]:
        with pytest.raises(binding.StrataError) as err:
            lay.set_routing(*args)
        assert err.value.status == binding.Status.INVALID_ARG
    lay.set_routing(binding.ROUTE_SIGMOID, corr, 2.5)
    lay.set_routing(binding.ROUTE_SOFTMAX)
    lay.close()

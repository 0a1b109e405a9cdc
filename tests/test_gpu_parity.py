"""GPU parity: the CUDA library (through its C interface) against the CPU
oracle on seeded synthetic inputs, plus the paged-vs-resident invariants."""
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


def ulp_diff(a, b):
    return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("name,T", [("tiny", 4), ("dsv2lite", 1), ("dsv2lite", 8),
                                    ("mixtral", 16), ("wide", 4), ("wide", 200)])
def test_route_matches_oracle(name, T):
    import oracle
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg, bind="all" if cfg.n_slots == cfg.n_experts else "none",
                   blobs=np.zeros((cfg.n_experts + cfg.n_shared, 256), np.uint8))
    x = synth.make_x(cfg, T, step=3)
    logits, idx, w = lay.route(x)
    rl, ridx, rw = oracle.route(x, lay.W, lay.b, cfg.top_k)
    assert ulp_diff(logits, rl).max() <= 1
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-5, atol=1e-7)
    lay.close()


def test_route_prefill_all_tokens():
    """8192 prefill tokens x 256 experts: every index equals the oracle's."""
    import oracle
    cfg = synth.CONFIGS["prefill"]
    lay = GpuLayer(cfg, blobs=np.zeros((cfg.n_experts + cfg.n_shared, 256), np.uint8))
    x = synth.make_x(cfg, 8192)
    logits, idx, w = lay.route(x)
    rl, ridx, rw = oracle.route(x, lay.W, lay.b, cfg.top_k)
    assert ulp_diff(logits, rl).max() <= 1
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-5, atol=1e-7)
    lay.close()


def test_route_ties_lowest_index():
    cfg = synth.custom_config("ties", 128, 128, 8, 3, tokens=(2,))
    lay = GpuLayer(cfg)
    W = lay.W.copy()
    W[6] = W[2] = W[5] = 0.5
    lay.W_dev.copy_(lay.torch.from_numpy(W))
    x = synth.f32_to_bf16_bits(np.abs(np.random.default_rng(0).standard_normal((2, 128))))
    _, idx, w = lay.route(x)
    assert idx.tolist() == [[2, 5, 6], [2, 5, 6]]
    np.testing.assert_allclose(w, 1 / 3, rtol=1e-6)
    lay.close()


# ------------------------------------------------------------------ layer output

CASES = [("tiny", 4), ("dsv2lite", 1), ("dsv2lite", 8), ("mixtral", 1), ("mixtral", 4),
         ("wide", 1), ("wide", 4)]


@pytest.mark.parametrize("name,T", CASES)
def test_forward_matches_oracle(name, T):
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg, bind="all" if cfg.n_slots == cfg.n_experts else "none")
    x = synth.make_x(cfg, T, step=1)
    ref, idx, w = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    if cfg.n_slots < cfg.n_experts:
        lay.bind_only(idx.reshape(-1))
    st, out = lay.forward(x)
    assert st[0] == 0, st
    assert_within_tolerance(out, ref, "%s T=%d" % (name, T))
    lay.close()


def test_forward_mixtral_16_tokens():
    cfg = synth.CONFIGS["mixtral"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 16, step=2)
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    st, out = lay.forward(x)
    assert st[0] == 0
    assert_within_tolerance(out, ref, "mixtral T=16")
    lay.close()


@pytest.mark.parametrize("T", [1, 7, 37, 100])
def test_forward_ragged_token_groups(T):
    """Experts with more than 16 pairs (several token groups), ragged tails,
    shared experts, hidden/inter not multiples of 1024."""
    cfg = synth.custom_config("ragged", 384, 256, 6, 2, n_shared=1, tokens=(T,), bias="normal",
                              bias_var=0.5)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=5)
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    st, out = lay.forward(x)
    assert st[0] == 0
    assert_within_tolerance(out, ref, "ragged T=%d" % T)
    lay.close()


@pytest.mark.parametrize("E,k,S,T", [
    (8, 8, 0, 4),     # top_k = n_experts: every expert takes every token
    (1, 1, 1, 5),     # one routed expert (weight 1) plus a shared one
    (8, 2, 0, 65),    # one token past the small-batch path: tensor-core path
    (8, 2, 1, 64),    # the largest small batch
])
def test_forward_degenerate_shapes(E, k, S, T):
    cfg = synth.custom_config("deg", 256, 256, E, k, n_shared=S, tokens=(T,))
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=4)
    st, out = lay.forward(x)
    assert int(st[0]) == 0
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    assert_within_tolerance(out, ref, "E=%d k=%d S=%d T=%d" % (E, k, S, T))
    lay.close()


# ------------------------------------------------------------------ invariants
# "How these numbers are measured", Fidelity: paged output is bit-identical to
# resident output.

@pytest.mark.parametrize("name,T", [("tiny", 4), ("dsv2lite", 8)])
def test_slot_permutation_bitwise(name, T):
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=7)
    _, ref = lay.forward(x)
    for p in range(1, 5):
        lay.bind_permutation(synth.make_slot_permutation(cfg, 0, p))
        st, out = lay.forward(x)
        assert st[0] == 0
        assert out.tolist() == ref.tolist()
    lay.close()


@pytest.mark.parametrize("name,T", [("tiny", 4), ("dsv2lite", 8), ("wide", 4)])
def test_routed_only_binding_bitwise(name, T):
    import oracle
    cfg = synth.CONFIGS[name]
    lay = GpuLayer(cfg, bind="none")
    x = synth.make_x(cfg, T, step=8)
    _, idx, _ = oracle.route(x, lay.W, lay.b, cfg.top_k)
    routed = sorted(set(idx.reshape(-1).tolist()))
    lay.bind_only(routed, rng_seed=1)
    st, a = lay.forward(x)
    assert st[0] == 0
    if cfg.n_slots == cfg.n_experts:
        lay.bind_permutation(synth.make_slot_permutation(cfg, 0, 3))
    else:
        extra = [e for e in range(cfg.n_experts) if e not in routed][:cfg.n_slots - len(routed)]
        lay.bind_only(routed + extra, rng_seed=2)
    st, b = lay.forward(x)
    assert st[0] == 0
    assert a.tolist() == b.tolist()
    lay.close()


def test_two_runs_bitwise_equal():
    cfg = synth.CONFIGS["dsv2lite"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 8, step=9)
    _, a = lay.forward(x)
    _, b = lay.forward(x)
    assert a.tolist() == b.tolist()
    lay.close()


# ------------------------------------------------------------------ device-side errors

def test_unbound_routed_expert_reports_status():
    import oracle
    cfg = synth.CONFIGS["tiny"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 4, step=1)
    _, full = lay.forward(x)
    _, idx, _ = oracle.route(x, lay.W, lay.b, cfg.top_k)
    victim = int(idx[0, 0])
    slot = int(np.nonzero(lay.slot_expert == victim)[0][0])
    lay.layer.bind_slot(slot, -1, None)
    (st, bits), out = lay.forward(x)
    assert int(st) == 3 and bits & 1
    for t in range(4):
        if victim in idx[t]:
            assert np.all(out[t] == 0)
        else:
            assert out[t].tolist() == full[t].tolist()
    # the status word was cleared by the read
    lay.layer.bind_slot(slot, victim, lay.blob_ptr(victim))
    st, _ = lay.forward(x)
    assert int(st[0]) == 0
    lay.close()


def test_forward_routed_bad_id():
    cfg = synth.CONFIGS["tiny"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 4, step=1)
    _, full = lay.forward(x)
    import oracle
    _, idx, w = oracle.route(x, lay.W, lay.b, cfg.top_k)
    st, same = lay.forward_routed(x, idx, w)
    assert int(st[0]) == 0 and same.tolist() == full.tolist()
    bad = idx.copy()
    bad[2, 1] = 99
    (st, bits), out = lay.forward_routed(x, bad, w)
    assert int(st) == 8 and bits & 2
    assert np.all(out[2] == 0)
    assert out[0].tolist() == full[0].tolist()
    lay.close()


def test_zero_tokens():
    import torch
    cfg = synth.CONFIGS["tiny"]
    lay = GpuLayer(cfg)
    x = torch.empty(0, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    lay.layer.forward(x, out)
    assert int(lay.layer.status()[0]) == 0
    lay.close()

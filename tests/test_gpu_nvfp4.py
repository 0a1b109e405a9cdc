"""NVFP4 experts (ro99/strata README, model table: E2M1 weights, E4M3 scales
per 16, an fp32 global scale, 16-bit activations) on the GPU through the C
interface, against the oracle's NVFP4 path: the small-batch kernel and the
tensor-core path element by element, and the paged-vs-resident invariant bit
for bit on both."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth
from tests.harness import (GpuLayer, assert_within_tolerance, oracle_reference,
                           oracle_reference_parallel)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_routed_expert_04_b200 import build
    build.build()


def test_blob_size_matches_format():
    from quantized_routed_expert_04_b200 import binding
    for H, I in [(256, 512), (2048, 1408), (4096, 2048)]:
        assert binding.strata_moe_expert_bytes_fmt(H, I, binding.FORMAT_NVFP4) == \
            synth.expert_bytes(H, I, "nvfp4")


def mid_config(T):
    return synth.custom_config("nvfp4_mid", 512, 256, 64, 8, n_shared=1, tokens=(T,),
                               bias="zipf", zipf_s=0.8, zipf_beta=1.0)


CASES = [("tiny", 4, None), ("dsv2lite", 8, None), ("dsv2lite", 13, None),
         ("mid", 300, None), ("mid", 2048, None)]


@pytest.mark.parametrize("name,T,_", CASES)
def test_nvfp4_forward_matches_oracle(name, T, _):
    cfg = mid_config(T) if name == "mid" else synth.CONFIGS[name]
    lay = GpuLayer(cfg, fmt="nvfp4")
    x = synth.make_x(cfg, T, step=51)
    ref, _, _ = oracle_reference_parallel(cfg, lay.blobs, lay.W, lay.b, x, fmt="nvfp4")
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    assert_within_tolerance(out, ref, "nvfp4 %s T=%d" % (name, T))
    lay.close()


@pytest.mark.parametrize("T", [8, 300])
def test_nvfp4_slot_permutation_bitwise(T):
    cfg = mid_config(T)
    lay = GpuLayer(cfg, fmt="nvfp4")
    x = synth.make_x(cfg, T, step=52)
    st, ref = lay.forward(x)
    assert int(st[0]) == 0
    for p in (1, 2):
        lay.bind_permutation(synth.make_slot_permutation(cfg, 0, p))
        st, out = lay.forward(x)
        assert int(st[0]) == 0 and np.array_equal(out, ref)
    lay.close()


def test_set_format_only_before_binding():
    from quantized_routed_expert_04_b200.binding import FORMAT_INT4, StrataError
    cfg = synth.CONFIGS["tiny"]
    lay = GpuLayer(cfg)
    with pytest.raises(StrataError):
        lay.layer.set_format(FORMAT_INT4)
    lay.close()

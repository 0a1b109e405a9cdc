"""GPU parity of the tensor-core (prefill) path, T > 64 tokens, through the C
interface: element-by-element against the CPU oracle on a prefill-shaped layer
whose tiles take every branch of the kernel, a strided quarter-thousand tokens
of the full 8192-token prefill, the paged-vs-resident invariants bit for bit
("How these numbers are measured", "Fidelity (paged vs resident output)"),
fp16 scales at the edges of their range on both the decode and the
tensor-core path, and the f16 range status."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth
from tests.harness import (GpuLayer, assert_within_tolerance, layer_errors,
                           oracle_reference, oracle_reference_parallel)

pytestmark = pytest.mark.gpu

TILE_PAIRS = 256      # pairs per tensor-core tile (one MMA N)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_routed_expert_04_b200 import build
    build.build()


def mid_config(T=2048):
    # the prefill layer's routing structure (256-pair tiles, Zipf(0.8) skew,
    # one shared expert) at a size the oracle finishes in seconds
    return synth.custom_config("prefill_mid", 512, 256, 64, 8, n_shared=1, tokens=(T,),
                               bias="zipf", zipf_s=0.8, zipf_beta=1.0)


def tile_sizes(counts):
    """Pair counts of the tensor-core tiles: each expert's pairs cut into
    chunks of TILE_PAIRS."""
    sizes = []
    for c in counts:
        c = int(c)
        while c > 0:
            sizes.append(min(c, TILE_PAIRS))
            c -= TILE_PAIRS
    return sizes


# ------------------------------------------------------------------ element-wise parity

def test_mid_prefill_every_element_and_every_tile_branch():
    import oracle
    cfg = mid_config()
    T = cfg.tokens[0]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=11)
    _, idx, w = oracle.route(x, lay.W, lay.b, cfg.top_k)
    counts = np.bincount(idx.reshape(-1), minlength=cfg.n_experts)
    sizes = tile_sizes(list(counts) + [T] * cfg.n_shared)
    # the hottest expert spans three or more tiles, and the kernel's three
    # activation-box cases (one 64-row box, up to three, one 256-row box) occur
    assert counts.max() > 2 * TILE_PAIRS, counts.max()
    assert any(s <= 64 for s in sizes) and any(64 < s <= 192 for s in sizes)
    assert any(s > 192 for s in sizes)
    ref, _, _ = oracle_reference_parallel(cfg, lay.blobs, lay.W, lay.b, x, idx, w)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    assert_within_tolerance(out, ref, "prefill_mid T=%d" % T)
    lay.close()


@pytest.mark.parametrize("T", [65, 129, 300])
def test_mid_prefill_ragged_token_counts(T):
    cfg = mid_config(T)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=12)
    ref, _, _ = oracle_reference_parallel(cfg, lay.blobs, lay.W, lay.b, x)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    assert_within_tolerance(out, ref, "prefill_mid T=%d" % T)
    lay.close()


def test_full_prefill_strided_tokens():
    """The 8192-token, 256-expert prefill in the configuration the benchmark
    times; every 32nd token (256 of them, spread over the whole batch and so
    over every expert's tiles) against the oracle."""
    cfg = synth.CONFIGS["prefill"]
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 8192)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    rows = np.arange(0, 8192, 32)
    ref, _, _ = oracle_reference_parallel(cfg, lay.blobs, lay.W, lay.b, x[rows])
    assert_within_tolerance(out[rows], ref, "prefill strided")
    lay.close()


# ------------------------------------------------------------------ bitwise invariants

@pytest.mark.parametrize("T", [65, 2048])
def test_tc_slot_permutation_bitwise(T):
    cfg = mid_config(T)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=13)
    st, ref = lay.forward(x)
    assert int(st[0]) == 0
    for p in range(1, 5):
        lay.bind_permutation(synth.make_slot_permutation(cfg, 0, p))
        st, out = lay.forward(x)
        assert int(st[0]) == 0
        assert np.array_equal(out, ref), "permutation %d" % p
    lay.close()


@pytest.mark.parametrize("T", [65, 2048])
def test_tc_routed_only_binding_bitwise(T):
    import oracle
    cfg = mid_config(T)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=14)
    st, full = lay.forward(x)
    assert int(st[0]) == 0
    _, idx, _ = oracle.route(x, lay.W, lay.b, cfg.top_k)
    routed = sorted(set(idx.reshape(-1).tolist()))
    lay.bind_only(routed, rng_seed=5)
    st, part = lay.forward(x)
    assert int(st[0]) == 0
    assert np.array_equal(part, full)
    lay.close()


def test_tc_swapped_and_plain_units_bitwise():
    """An expert's last block of <= 128 pairs goes to swapped units (the
    pairs' activations as the MMA's A, with M = 64 for <= 64 pairs, 256 weight
    rows as its B), other blocks to plain ones (128 weight rows as A, the pairs
    as B); a token's output must not depend on which.  Tokens are routed to
    four experts (and the shared one): an 80-token batch whose halves use
    different experts runs swapped units of M = 64 (40 pairs each) and of
    M = 128 (the shared expert), a 100-token batch swapped units of M = 128, a
    300-token batch plain ones only, and a 600-token batch a plain block of
    512 pairs and a swapped block of 88: the same tokens give the same bits
    in each.  (Batches of <= 64 tokens take the other kernel.)"""
    cfg = synth.custom_config("forms", 512, 256, 16, 4, n_shared=1, tokens=(600,))
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 600, step=21)
    idx = np.tile(np.array([[3, 0, 9, 5]], np.int32), (600, 1))
    w = np.random.default_rng(7).dirichlet(np.ones(4), size=600).astype(np.float32)
    idx80 = idx[:80].copy()
    idx80[40:] = [1, 2, 4, 6]
    st, e80 = lay.forward_routed(x[:80], idx80, w[:80])
    assert int(st[0]) == 0, st
    st, a100 = lay.forward_routed(x[:100], idx[:100], w[:100])
    assert int(st[0]) == 0, st
    st, b300 = lay.forward_routed(x[:300], idx[:300], w[:300])
    assert int(st[0]) == 0, st
    st, c600 = lay.forward_routed(x, idx, w)
    assert int(st[0]) == 0, st
    assert np.array_equal(e80[:40], b300[:40])
    assert np.array_equal(a100, b300[:100])
    assert np.array_equal(b300, c600[:300])
    # tokens 512..599: swapped in the 600-token batch, plain in this one
    mix = np.concatenate([np.arange(512, 600), np.arange(0, 212)])
    st, d300 = lay.forward_routed(x[mix], idx[mix], w[mix])
    assert int(st[0]) == 0, st
    assert np.array_equal(d300[:88], c600[512:600])
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x, idx, w)
    assert_within_tolerance(c600, ref, "swapped and plain units")
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x[:80], idx80, w[:80])
    assert_within_tolerance(e80, ref, "swapped units of M = 64")
    lay.close()


def test_tc_two_runs_bitwise_equal():
    cfg = mid_config(2048)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, 2048, step=15)
    _, a = lay.forward(x)
    _, b = lay.forward(x)
    assert np.array_equal(a, b)
    lay.close()


# ------------------------------------------------------------------ edge scales and range

F16_2M24, F16_SUBNORMAL, F16_2M14, F16_8188 = 0x0001, 0x0155, 0x0400, 0x6FFF
F16_16384, F16_65504 = 0x7400, 0x7BFF


def set_down_row_scales(blob, H, I, row, bits):
    """Every fp16 scale of row `row` of Wd (all blocks of the row)."""
    lay = synth.blob_layout(H, I)
    tile, tr = row // 16, row % 16
    G = I // 128
    v = np.full(4, bits, np.uint16).view(np.uint8)
    for g in range(G):
        off = lay["ds"] + ((tile * G + g) * 16 + tr) * 8
        blob[off:off + 8] = v


def set_gate_up_scales(blob, H, I, bits):
    lay = synth.blob_layout(H, I)
    n = I * H // 16   # fp16 scales of Wg and Wu
    blob[lay["gus"]:lay["gus"] + 2 * n] = np.full(n, bits, np.uint16).view(np.uint8)


EDGE_GROUPS = [(F16_2M24, "2^-24"), (F16_SUBNORMAL, "subnormal"), (F16_2M14, "2^-14"),
               (F16_8188, "8188")]


def edge_config(T):
    return synth.custom_config("edge", 256, 256, 8, 2, n_shared=1, tokens=(T,))


def edge_blobs(cfg, groups):
    blobs = synth.make_all_blobs(cfg, 0)
    for e in range(cfg.n_experts + cfg.n_shared):
        for gi, (bits, _) in enumerate(groups):
            for r in range(16 * gi, 16 * gi + 16):
                set_down_row_scales(blobs[e], cfg.hidden, cfg.inter, r, bits)
    return blobs


def check_row_groups(out, ref, groups, what):
    """Tolerance over the whole output and, separately, over each group of 16
    output rows whose down-projection rows carry one edge scale (so that the
    tiny-scale rows are not hidden by the large ones)."""
    assert_within_tolerance(out, ref, what)
    for gi, (_, name) in enumerate(groups):
        cols = slice(16 * gi, 16 * gi + 16)
        mx, mean = layer_errors(np.ascontiguousarray(out[:, cols]), ref[:, cols])
        assert mx <= 2e-2 and mean <= 2e-3, "%s rows with scale %s: %.3e %.3e" % (
            what, name, mx, mean)


@pytest.mark.parametrize("T", [4, 100])
def test_edge_scales_both_paths(T):
    """Scales 2^-24, a subnormal, 2^-14 and 8188 (the largest whose int4
    multiples stay finite in f16) in whole down-projection rows: decode (T = 4)
    and tensor-core (T = 100) outputs within tolerance row group by row group,
    and no status."""
    cfg = edge_config(T)
    blobs = edge_blobs(cfg, EDGE_GROUPS)
    lay = GpuLayer(cfg, blobs=blobs)
    x = synth.make_x(cfg, T, step=16)
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    check_row_groups(out, ref, EDGE_GROUPS, "edge scales T=%d" % T)
    lay.close()


def test_large_scales_exact_on_decode_path():
    """Scales 16384 and 65504 in down-projection rows: the decode path applies
    them in fp32 and stays within tolerance."""
    groups = [(F16_16384, "16384"), (F16_65504, "65504")]
    cfg = edge_config(4)
    lay = GpuLayer(cfg, blobs=edge_blobs(cfg, groups))
    x = synth.make_x(cfg, 4, step=17)
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    st, out = lay.forward(x)
    assert int(st[0]) == 0, st
    check_row_groups(out, ref, groups, "large scales T=4")
    lay.close()


def test_large_scale_reports_range_on_tensor_core_path():
    """A scale of 16384 cannot be dequantised to f16 for every int4 value:
    the tensor-core path reports STRATA_ERR_RANGE instead of a silent inf, and
    the next call on clean blobs is clean."""
    from quantized_routed_expert_04_b200.binding import Status
    cfg = edge_config(100)
    lay = GpuLayer(cfg, blobs=edge_blobs(cfg, [(F16_16384, "16384")]))
    x = synth.make_x(cfg, 100, step=18)
    (st, bits), _ = lay.forward(x)
    assert st == Status.RANGE and bits & 16, (st, bits)
    lay.close()
    lay = GpuLayer(cfg)
    (st, bits), _ = lay.forward(x)
    assert st == Status.OK and bits == 0
    lay.close()


@pytest.mark.parametrize("T", [4, 100])
def test_activation_beyond_f16_reports_range(T):
    from quantized_routed_expert_04_b200.binding import Status
    cfg = edge_config(T)
    lay = GpuLayer(cfg)
    x = synth.make_x(cfg, T, step=19)
    big = x.copy()
    big[T // 2, 7] = synth.f32_to_bf16_bits(np.array([1.0e5], np.float32))[0]
    (st, bits), _ = lay.forward(big)
    assert st == Status.RANGE and bits & 16, (st, bits)
    # the status was cleared by the read; an ordinary batch is clean
    (st, bits), out = lay.forward(x)
    assert st == Status.OK and bits == 0
    ref, _, _ = oracle_reference(cfg, lay.blobs, lay.W, lay.b, x)
    assert_within_tolerance(out, ref, "after range T=%d" % T)
    lay.close()


@pytest.mark.parametrize("T", [4, 100])
def test_swiglu_output_beyond_f16_reports_range(T):
    """Gate and up scales of 16384 on every expert make |h| overflow f16
    (on the tensor-core path the scale check fires as well)."""
    from quantized_routed_expert_04_b200.binding import Status
    cfg = edge_config(T)
    blobs = synth.make_all_blobs(cfg, 0)
    for e in range(cfg.n_experts + cfg.n_shared):
        set_gate_up_scales(blobs[e], cfg.hidden, cfg.inter, F16_16384)
    lay = GpuLayer(cfg, blobs=blobs)
    x = synth.make_x(cfg, T, step=20)
    (st, bits), _ = lay.forward(x)
    assert st == Status.RANGE and bits & 16, (st, bits)
    lay.close()

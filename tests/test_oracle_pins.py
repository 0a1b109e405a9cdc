"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test names the passage or mathematical fact it rests on.  A plausible
mistake in the oracle (nibble order, sign handling, scale indexing, a dropped
term, a transposed operand, the tie-break, the combine order) fails at least
one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_routed_expert_04_b200 import synth
from tests import naive

RNG = np.random.default_rng(1234)


def rand_q(rows, K, rng=RNG):
    return rng.integers(-8, 8, size=(rows, K))


def rand_s(rows, K, rng=RNG):
    return rng.uniform(0.005, 0.02, size=(rows, K // 32)).astype(np.float16)


def rand_blob(H, I, rng=RNG):
    parts = dict(gq=rand_q(I, H, rng), uq=rand_q(I, H, rng), dq=rand_q(H, I, rng),
                 gs=rand_s(I, H, rng), us=rand_s(I, H, rng), ds=rand_s(H, I, rng))
    return synth.build_blob(H, I, **parts), parts


def bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


# --------------------------------------------------------------------- format

def binding_free_layout_ok(H, I):
    lay = synth.blob_layout(H, I)
    return all(lay[k] % 256 == 0 for k in lay)


def test_pack_int4_hand_bytes():
    # element 2j -> low nibble, 2j+1 -> high nibble, two's complement
    q = np.array([[-8, 7, 1, -1, 0, -2]])
    assert synth.pack_int4(q).tolist() == [[0x78, 0xF1, 0xE0]]


def test_group_layout_hand_bytes():
    """One gate row, one group: element 32b + 8w + m sits at byte 16w + 4b + m/2."""
    H, I = 128, 128
    q = np.zeros((I, H), int)
    q[0, 0] = 1        # b0 w0 m0 -> byte 0 low
    q[0, 9] = 2        # b0 w1 m1 -> byte 16 high
    q[0, 32 + 7] = -1  # b1 w0 m7 -> byte 4 + 3 high
    q[0, 96 + 24] = 3  # b3 w3 m0 -> byte 48 + 12 low
    z = np.zeros((I, H // 32), np.float16)
    blob = synth.build_blob(H, I, q, np.zeros_like(q), np.zeros((H, I), int), z, z,
                            np.zeros((H, I // 32), np.float16))
    row0 = blob[:64]
    assert row0[0] == 0x01 and row0[16] == 0x20 and row0[7] == 0xF0 and row0[60] == 0x03
    assert np.count_nonzero(row0) == 4
    # up row 0 is tile row 8 of tile 0: bytes 8*64 .. 9*64
    assert not blob[8 * 64:9 * 64].any()


def test_blob_size_formula():
    # B_e = 3*H*I*(1/2 + 2/32) when every section is a multiple of 256 bytes
    for H, I in [(256, 512), (2048, 1408), (4096, 14336), (4096, 1024), (4096, 2048)]:
        assert oracle.expert_bytes(H, I) == synth.expert_bytes(H, I) == int(3 * H * I * 0.5625)
        assert binding_free_layout_ok(H, I)


def test_dequant_matches_drawn_values_one_hot():
    """x = identity makes g[t] the t-th column of Wg: oracle g must equal
    float(scale) * q for the drawn ints, exactly (one nonzero product)."""
    H, I = 128, 256
    blob, p = rand_blob(H, I)
    # edge fp16 scales: min subnormal, a subnormal, min normal, max
    p["gs"][0, 0] = np.float16(2.0 ** -24)
    p["gs"][1, 1] = np.float16(3 * 2.0 ** -20)
    p["us"][2, 0] = np.float16(2.0 ** -14)
    p["us"][3, 1] = np.float16(65504.0)
    blob = synth.build_blob(H, I, **p)
    x = np.eye(H, dtype=np.float32)
    g, u, h, y = oracle.expert_ffn(blob, H, I, x)
    want_g = (p["gs"].astype(np.float32).repeat(32, axis=1) * p["gq"].astype(np.float32)).T
    want_u = (p["us"].astype(np.float32).repeat(32, axis=1) * p["uq"].astype(np.float32)).T
    np.testing.assert_array_equal(g, want_g)
    np.testing.assert_array_equal(u, want_u)


def test_down_projection_columns():
    """y = Wd h with Wd dequantised from the drawn ints (fp64 reference)."""
    H, I = 128, 128
    blob, p = rand_blob(H, I)
    x = np.eye(H, dtype=np.float32)
    g, u, h, y = oracle.expert_ffn(blob, H, I, x)
    Wd = p["ds"].astype(np.float64).repeat(32, axis=1) * p["dq"]
    ref = h.astype(np.float64) @ Wd.T
    np.testing.assert_allclose(y, ref, rtol=2e-5, atol=2e-5 * np.abs(ref).max())


def test_swiglu_formula():
    """h = silu(g) * u with silu(z) = z / (1 + e^-z): the SwiGLU expert FFN
    of the W4A16 layer (ro99/strata README, model table)."""
    H, I = 128, 128
    blob, _ = rand_blob(H, I)
    x = synth.bf16_bits_to_f32(bf16(RNG.standard_normal((5, H)) * 4))
    g, u, h, _ = oracle.expert_ffn(blob, H, I, x)
    g64 = g.astype(np.float64)
    ref = g64 / (1 + np.exp(-g64)) * u
    np.testing.assert_allclose(h, ref, rtol=1e-5, atol=1e-6)


def test_gate_all_equal_weights_closed_form():
    """All q = 1 with scale s: g_i = s * sum(x) for every row."""
    H, I = 128, 128
    s = np.float16(0.0125)
    parts = dict(gq=np.ones((I, H), int), uq=np.ones((I, H), int), dq=np.ones((H, I), int),
                 gs=np.full((I, H // 32), s), us=np.full((I, H // 32), s),
                 ds=np.full((H, I // 32), s))
    blob = synth.build_blob(H, I, **parts)
    x = synth.bf16_bits_to_f32(bf16(RNG.standard_normal((3, H))))
    g, u, h, y = oracle.expert_ffn(blob, H, I, x)
    want = float(s) * x.astype(np.float64).sum(axis=1)
    np.testing.assert_allclose(g, np.repeat(want[:, None], I, axis=1), rtol=1e-5, atol=1e-6)
    # then every h_i is equal and y_r = s * I * h
    np.testing.assert_allclose(y, float(s) * I * h[:, :1].astype(np.float64).repeat(H, 1),
                               rtol=1e-5, atol=1e-6)


def test_negative_extreme_nibble():
    """q = -8 everywhere (nibble 0x8) must read as -8, not +8."""
    H, I = 128, 128
    s = np.float16(1.0)
    parts = dict(gq=np.full((I, H), -8), uq=np.full((I, H), 7), dq=np.zeros((H, I), int),
                 gs=np.full((I, 4), s), us=np.full((I, 4), s), ds=np.full((H, 4), s))
    blob = synth.build_blob(H, I, **parts)
    x = np.ones((1, H), np.float32)
    g, u, _, _ = oracle.expert_ffn(blob, H, I, x)
    assert np.all(g == -8.0 * H) and np.all(u == 7.0 * H)


# --------------------------------------------------------------------- router

def test_route_exact_logits_and_subset_topk():
    """Logits equal the exact sum rounded once to fp32 (within 1 ulp, since the
    oracle sums in double); idx equals the brute-force subset top-k; w equals
    fp64 softmax renormalised over the selection."""
    for (E, k, H, T) in [(4, 1, 64, 3), (6, 2, 96, 3), (8, 3, 64, 2), (5, 5, 32, 2)]:
        x = bf16(RNG.standard_normal((T, H)))
        W = (RNG.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
        b = (RNG.standard_normal(E) * 0.7).astype(np.float32)
        logits, idx, w = oracle.route(x, W, b, k)
        ex = naive.exact_logits(x, W, b)
        ulps = np.abs(logits.view(np.int32).astype(np.int64) - ex.view(np.int32).astype(np.int64))
        assert ulps.max() <= 1
        for t in range(T):
            sel = naive.topk_by_subsets(logits[t], k)
            assert idx[t].tolist() == sel
            l64 = logits[t].astype(np.float64)
            p = np.exp(l64 - l64.max())
            p /= p.sum()
            np.testing.assert_allclose(w[t], p[sel] / p[sel].sum(), rtol=2e-6)


def test_route_tie_break_lowest_index():
    """Duplicate router rows give equal logits; the lower expert index wins."""
    H, E = 64, 8
    W = (RNG.standard_normal((E, H)) / 64).astype(np.float32)
    x = bf16(RNG.standard_normal((1, H)))
    xf = synth.bf16_bits_to_f32(x)[0]
    big = (np.sign(xf) * 0.5).astype(np.float32)   # a row far above the others
    for e in (6, 2, 5):
        W[e] = big
    _, idx, w = oracle.route(x, W, None, 3)
    assert idx[0].tolist() == [2, 5, 6]
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-6)
    # k = 2 of three tied experts: the two lowest indices
    _, idx, _ = oracle.route(x, W, None, 2)
    assert idx[0].tolist() == [2, 5]
    # all rows equal: the first k experts, equal weights
    W2 = np.repeat(W[:1], E, axis=0)
    _, idx2, w2 = oracle.route(x, W2, None, 4)
    assert idx2[0].tolist() == [0, 1, 2, 3]
    np.testing.assert_allclose(w2[0], 0.25, rtol=0, atol=0)


def test_route_bias_shifts_logits():
    """Bias is added to the logit before softmax: a large bias forces selection."""
    H, E = 32, 6
    W = np.zeros((E, H), np.float32)
    b = np.array([0, 0, 0, 5, 0, 4], np.float32)
    x = bf16(RNG.standard_normal((2, H)))
    logits, idx, w = oracle.route(x, W, b, 2)
    assert np.all(logits == b)
    assert idx.tolist() == [[3, 5], [3, 5]]
    e = np.exp(np.array([5.0, 4.0]) - 5.0)
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=1e-6)


# --------------------------------------------------------------------- layer

def _bind_all(blobs, perm=None):
    E = len(blobs)
    perm = np.arange(E) if perm is None else np.asarray(perm)
    return perm.astype(np.int32), [blobs[e] for e in perm]


@pytest.mark.parametrize("E,k,S,T,H,I", [(4, 1, 0, 2, 128, 128), (6, 2, 1, 3, 128, 256),
                                          (8, 3, 2, 2, 256, 128), (5, 2, 0, 1, 128, 128)])
def test_layer_matches_naive_bruteforce(E, k, S, T, H, I):
    rng = np.random.default_rng(E * 100 + k * 10 + S)
    blobs = [rand_blob(H, I, rng)[0] for _ in range(E)]
    shared = [rand_blob(H, I, rng)[0] for _ in range(S)]
    W = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    b = (rng.standard_normal(E) * 0.5).astype(np.float32)
    x = bf16(rng.standard_normal((T, H)))
    se, sb = _bind_all(blobs, rng.permutation(E))
    st, out, logits, idx, w = oracle.forward(x, H, I, W, b, k, se, sb, shared)
    assert st == oracle.OK
    ref, ridx, rw = naive.layer64(x, blobs, shared, W, b, k, H, I)
    assert idx.tolist() == ridx.tolist()
    np.testing.assert_allclose(w, rw, rtol=2e-6)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(out, ref, rtol=0, atol=2e-5 * scale)


def test_topk_all_experts_is_dense_softmax_mixture():
    """top_k = n_experts: out = sum_e softmax(l)_e FFN_e(x) (torch fp64)."""
    E, H, I, T = 5, 128, 128, 3
    rng = np.random.default_rng(7)
    blobs = [rand_blob(H, I, rng)[0] for _ in range(E)]
    W = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    x = bf16(rng.standard_normal((T, H)))
    se, sb = _bind_all(blobs)
    st, out, logits, idx, w = oracle.forward(x, H, I, W, None, E, se, sb, [])
    assert st == oracle.OK
    xt = torch.tensor(synth.bf16_bits_to_f32(x), dtype=torch.float64)
    Wt = torch.tensor(W, dtype=torch.float64)
    p = torch.softmax(xt @ Wt.T, dim=-1)
    ref = torch.zeros(T, H, dtype=torch.float64)
    for e in range(E):
        Wg, Wu, Wd = (torch.tensor(m) for m in naive.dense_expert(blobs[e], H, I))
        ye = (torch.nn.functional.silu(xt @ Wg.T) * (xt @ Wu.T)) @ Wd.T
        ref += p[:, e:e + 1] * ye
    ref = ref.numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=2e-5 * np.abs(ref).max())


def test_single_expert_weight_one_is_swiglu_ffn():
    """E = 1, k = 1: w = 1 and out = Wd (silu(Wg x) * (Wu x)) (torch fp64)."""
    H, I, T = 256, 128, 4
    rng = np.random.default_rng(11)
    blob = rand_blob(H, I, rng)[0]
    W = rng.standard_normal((1, H)).astype(np.float32)
    x = bf16(rng.standard_normal((T, H)))
    st, out, _, idx, w = oracle.forward(x, H, I, W, None, 1, np.array([0]), [blob], [])
    assert st == oracle.OK and np.all(idx == 0) and np.all(w == 1.0)
    xt = torch.tensor(synth.bf16_bits_to_f32(x), dtype=torch.float64)
    Wg, Wu, Wd = (torch.tensor(m) for m in naive.dense_expert(blob, H, I))
    ref = ((torch.nn.functional.silu(xt @ Wg.T) * (xt @ Wu.T)) @ Wd.T).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=2e-5 * np.abs(ref).max())


def test_paged_vs_resident_bitwise():
    """strata.amperor.ai "/methods/", Fidelity: paged output is bit-identical to
    resident.  Any slot permutation, and binding only the routed experts, give
    the same fp32 bits."""
    cfg = synth.custom_config("t", 128, 128, 8, 2, n_shared=1, n_slots=8, tokens=(3,))
    blobs = [synth.make_expert_blob(cfg, e) for e in range(8)]
    shared = [synth.make_expert_blob(cfg, 8)]
    W, b = synth.make_router(cfg)
    x = synth.make_x(cfg, 3)
    st, ref, _, idx, w = oracle.forward(x, 128, 128, W, b, 2, *_bind_all(blobs), shared)
    assert st == oracle.OK
    for p in range(4):
        perm = synth.make_slot_permutation(cfg, index=p)
        st, out, *_ = oracle.forward(x, 128, 128, W, b, 2, *_bind_all(blobs, perm), shared)
        assert st == oracle.OK and out.view(np.uint32).tolist() == ref.view(np.uint32).tolist()
    routed = sorted(set(idx.reshape(-1).tolist()))
    se = np.full(8, -1, np.int32)
    sb = [None] * 8
    for s, e in zip(np.random.default_rng(3).permutation(8)[:len(routed)], routed):
        se[s] = e
        sb[s] = blobs[e]
    st, out = oracle.forward_routed(x, 128, 128, 8, 2, se, sb, shared, idx, w)
    assert st == oracle.OK and out.view(np.uint32).tolist() == ref.view(np.uint32).tolist()


def test_unbound_expert_reports_and_zeroes_token():
    cfg = synth.custom_config("t", 128, 128, 6, 2, tokens=(4,))
    blobs = [synth.make_expert_blob(cfg, e) for e in range(6)]
    W, b = synth.make_router(cfg)
    x = synth.make_x(cfg, 4)
    st, ref, _, idx, w = oracle.forward(x, 128, 128, W, b, 2, *_bind_all(blobs), [])
    victim = int(idx[1, 0])
    se = np.arange(6, dtype=np.int32)
    se[victim] = -1
    sb = [None if e == victim else blobs[e] for e in range(6)]
    st, out = oracle.forward_routed(x, 128, 128, 6, 2, se, sb, [], idx, w)
    assert st == oracle.NOT_BOUND
    for t in range(4):
        if victim in idx[t]:
            assert np.all(out[t] == 0)
        else:
            np.testing.assert_array_equal(out[t], ref[t])


def test_slot_conflict():
    cfg = synth.custom_config("t", 128, 128, 4, 1, tokens=(1,))
    blobs = [synth.make_expert_blob(cfg, e) for e in range(4)]
    x = synth.make_x(cfg, 1)
    se = np.array([0, 1, 1, 3], np.int32)
    st, _ = oracle.forward_routed(x, 128, 128, 4, 1, se, blobs, [], np.array([[0]]), np.array([[1.0]]))
    assert st == oracle.SLOT_CONFLICT


def test_combine_order_is_weighted_then_shared():
    """out = sum_j w_j y_j + sum_s y_s: with a zero routed weight the output is
    exactly the shared expert's y, and with w = (1, 0) it is y_0 + y_shared."""
    H, I = 128, 128
    rng = np.random.default_rng(5)
    blobs = [rand_blob(H, I, rng)[0] for _ in range(3)]
    sh = rand_blob(H, I, rng)[0]
    x = bf16(rng.standard_normal((1, H)))
    xf = synth.bf16_bits_to_f32(x)
    ys = [oracle.expert_ffn(b, H, I, xf)[3][0] for b in blobs + [sh]]
    idx = np.array([[2, 0]])
    st, out = oracle.forward_routed(x, H, I, 3, 2, np.arange(3), blobs, [sh], idx,
                                    np.array([[1.0, 0.0]], np.float32))
    assert st == oracle.OK
    np.testing.assert_array_equal(out[0], (np.float32(0) + ys[2]) + np.float32(0) * ys[0] + ys[3])


def test_wide_zipf_share():
    """Wide layer: Zipf(1.1) bias such that ~80% of routed hits land in the 64
    highest-ranked experts (the layer's stated intent); checked on 256 seed-0
    tokens with the oracle router."""
    cfg = synth.CONFIGS["wide"]
    W, b = synth.make_router(cfg)
    ranks = synth.zipf_ranks(cfg)
    x = synth.make_x(cfg, 256, step=0)
    _, idx, _ = oracle.route(x, W, b, cfg.top_k)
    share = np.mean(ranks[idx.reshape(-1)] <= 64)
    assert 0.78 <= share <= 0.82, share


# ------------------------------------------------------------ sigmoid routing
# (sigmoid top-k with a correction bias and a routed scale)

def test_route_sigmoid_hand_case():
    # x = 0, so every logit is its bias: 0 -> score exactly 0.5.  The
    # correction bias alone decides the selection; the weights are
    # 0.5 / (0.5 + 0.5) * 2.5 = 1.25 exactly.
    E, H, k = 4, 64, 2
    x = np.zeros((1, H), np.uint16)
    W = np.ones((E, H), np.float32)
    corr = np.array([0.0, 0.25, -0.25, 0.125], np.float32)
    logits, idx, w = oracle.route_sigmoid(x, W, np.zeros(E, np.float32), corr, 2.5, k)
    assert logits.tolist() == [[0.0] * E]
    assert idx.tolist() == [[1, 3]]
    assert w.tolist() == [[1.25, 1.25]]
    # a large negative logit has a tiny score: a big correction still selects
    # it (keys 0.5, 0.75, 0.25, 0.625), but its share of the weight is tiny
    bias = np.array([0.0, -30.0, 0.0, 0.0], np.float32)
    corr2 = np.array([0.0, 0.75, -0.25, 0.125], np.float32)
    _, idx, w = oracle.route_sigmoid(x, W, bias, corr2, 1.0, k)
    assert idx.tolist() == [[1, 3]]
    tiny = 1.0 / (1.0 + np.exp(30.0))
    assert w[0, 0] == pytest.approx(tiny / (tiny + 0.5), rel=1e-5)
    assert w[0, 1] == pytest.approx(0.5 / (tiny + 0.5), rel=1e-6)


def test_route_sigmoid_without_correction_selects_like_softmax():
    # the sigmoid is increasing, so without a correction bias the selection is
    # the top-k of the logits, as in the softmax router
    cfg = synth.custom_config("sg", 256, 128, 16, 4)
    x = synth.make_x(cfg, 12, seed=5)
    W, _ = synth.make_router(cfg, seed=5)
    _, idx_s, _ = oracle.route(x, W, None, 4)
    logits, idx_g, w_g = oracle.route_sigmoid(x, W, None, None, 1.0, 4)
    assert idx_g.tolist() == idx_s.tolist()
    sc = 1.0 / (1.0 + np.exp(-logits.astype(np.float64)))
    sel = np.take_along_axis(sc, idx_g.astype(np.int64), axis=1)
    np.testing.assert_allclose(w_g, sel / sel.sum(axis=1, keepdims=True), rtol=2e-6)
    np.testing.assert_allclose(w_g.sum(axis=1), 1.0, rtol=2e-6)


def test_route_sigmoid_subset_topk_of_keys():
    # selection = the subset with the largest sum of keys (score + correction)
    E, k, H = 7, 3, 128
    rng = np.random.default_rng(11)
    x = synth.f32_to_bf16_bits(rng.standard_normal((6, H)).astype(np.float32))
    W = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    corr = (rng.standard_normal(E) * 0.2).astype(np.float32)
    logits, idx, w = oracle.route_sigmoid(x, W, None, corr, 2.5, k)
    for t in range(x.shape[0]):
        sc = (1.0 / (1.0 + np.exp(-logits[t].astype(np.float64)))).astype(np.float32)
        key = (sc + corr).astype(np.float32)
        assert idx[t].tolist() == naive.topk_by_subsets(key, k)
        assert float(w[t].sum()) == pytest.approx(2.5, rel=1e-6)


# ------------------------------------------------------------ NVFP4 experts
# (E2M1 codes in the int4 nibble places, one E4M3 scale per 16 along K, one
# fp32 global scale per matrix)

def _nvfp4_blob(H, I, gc=None, gs=None, glob=(1.0, 1.0, 1.0)):
    gc = np.zeros((I, H), np.int64) if gc is None else gc
    gs = np.full((I, H // 16), 0x38, np.uint8) if gs is None else gs   # 0x38 = 1.0
    zc = np.zeros((I, H), np.int64)
    return synth.build_blob_nvfp4(H, I, gc, zc, np.zeros((H, I), np.int64), gs,
                                  np.full((I, H // 16), 0x38, np.uint8),
                                  np.full((H, I // 16), 0x38, np.uint8), glob)


def test_nvfp4_blob_size():
    for H, I in [(128, 128), (4096, 1024)]:
        assert oracle.expert_bytes(H, I, "nvfp4") == oracle.expert_bytes(H, I) + 256
        assert oracle.expert_bytes(H, I, "nvfp4") == synth.expert_bytes(H, I, "nvfp4")


def test_nvfp4_e2m1_codes_hand_table():
    H, I = 128, 128
    gc = np.zeros((I, H), np.int64)
    gc[0, :16] = np.arange(16)
    blob = _nvfp4_blob(H, I, gc=gc)
    x = np.eye(H, dtype=np.float32)[:16]                 # one-hot activations
    g, _, _, _ = oracle.expert_ffn(blob, H, I, x, fmt="nvfp4")
    want = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert g[:, 0].tolist() == want


def test_nvfp4_e4m3_scales_match_library_decoder():
    H, I = 2048, 128
    gc = np.full((I, H), 2, np.int64)                    # E2M1 code 2 = 1.0
    gs = np.full((I, H // 16), 0x38, np.uint8)
    codes = np.arange(256, dtype=np.int64)
    codes[(codes & 0x7F) == 0x7F] = 0x38                 # the two NaN encodings
    gs[0, :128] = codes[:128]
    gs[1, :128] = codes[128:]
    blob = _nvfp4_blob(H, I, gc=gc, gs=gs)
    x = np.eye(H, dtype=np.float32)[::16]                # first element of each group
    g, _, _, _ = oracle.expert_ffn(blob, H, I, x, fmt="nvfp4")
    got = np.concatenate([g[:, 0], g[:, 1]])
    np.testing.assert_array_equal(got, naive.e4m3_values(codes.astype(np.uint8)).astype(np.float32))


def test_nvfp4_weights_are_code_times_scale_times_global():
    H, I = 256, 128
    rng = np.random.default_rng(21)
    gc = rng.integers(0, 16, size=(I, H))
    gs = rng.choice(np.array([(e << 3) | m for e in range(1, 15) for m in range(8)], np.uint8),
                    size=(I, H // 16))
    glob = (0.0371, 1.0, 1.0)
    blob = _nvfp4_blob(H, I, gc=gc, gs=gs, glob=glob)
    x = np.eye(H, dtype=np.float32)
    g, _, _, _ = oracle.expert_ffn(blob, H, I, x, fmt="nvfp4")
    Wg, _, _ = naive.dense_expert_nvfp4(blob, H, I)
    np.testing.assert_array_equal(g.T, Wg.astype(np.float32))   # one rounding, exact otherwise


@pytest.mark.parametrize("E,k,S,T", [(4, 2, 1, 3), (3, 3, 0, 2)])
def test_nvfp4_layer_matches_naive_fp64(E, k, S, T):
    H, I = 128, 128
    cfg = synth.custom_config("fp4", H, I, E, k, n_shared=S, tokens=(T,))
    blobs = [synth.make_expert_blob_nvfp4(cfg, e, seed=4) for e in range(E + S)]
    W, b = synth.make_router(cfg, seed=4)
    x = synth.make_x(cfg, T, seed=4)
    _, idx, w = oracle.route(x, W, b, k)
    st, out = oracle.forward_routed(x, H, I, E, k, np.arange(E), blobs[:E], blobs[E:], idx, w,
                                    fmt="nvfp4")
    assert st == oracle.OK
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    dense = [naive.dense_expert_nvfp4(bl, H, I) for bl in blobs]
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            ref[t] += float(w[t, j]) * naive.ffn64(dense[idx[t, j]], xf[t])
        for s in range(S):
            ref[t] += naive.ffn64(dense[E + s], xf[t])
    err = np.abs(out - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err

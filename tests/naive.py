"""A deliberately naive fp64 restatement of the layer, used only to pin the oracle.

It shares no code with the oracle: its own int4 unpacking (vectorised numpy),
dense dequantisation of every expert, every expert evaluated for every token,
exact router sums (fractions), top-k found by enumerating all expert subsets,
and fp64 softmax / combine.  It is far too slow for anything but tiny shapes.
"""
from __future__ import annotations

import itertools
from fractions import Fraction

import numpy as np

from quantized_routed_expert_04_b200 import synth


def unpack_tiles(raw: np.ndarray, tiles: int, K: int) -> np.ndarray:
    """u8 bytes of a tiled section -> int [tiles][16][K].

    Byte 16w + 4b + c of a row's 64-byte group holds elements 32b + 8w + 2c
    (low nibble) and 32b + 8w + 2c + 1 (high nibble)."""
    b = np.asarray(raw, np.uint8).reshape(tiles, K // 128, 16, 4, 4, 4)  # t, g, row, w, blk, c
    out = np.empty((tiles, K // 128, 16, 4, 4, 8), np.int16)               # t, g, row, w, blk, m
    lo = (b & 0xF).astype(np.int16)
    hi = (b >> 4).astype(np.int16)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    # element index within the group = 32*blk + 8*w + m
    return out.transpose(0, 2, 1, 4, 3, 5).reshape(tiles, 16, K)


def tile_scales(raw: np.ndarray, tiles: int, K: int) -> np.ndarray:
    """f16 bytes of a tiled scale section -> float64 [tiles][16][K/32]."""
    s = np.asarray(raw, np.uint8).view(np.float16).reshape(tiles, K // 128, 16, 4)
    return s.transpose(0, 2, 1, 3).reshape(tiles, 16, K // 32).astype(np.float64)


def dense_expert(blob: np.ndarray, H: int, I: int):
    """(Wg [I][H], Wu [I][H], Wd [H][I]) dequantised to float64."""
    lay = synth.blob_layout(H, I)
    gu = unpack_tiles(blob[lay["guq"]:lay["guq"] + I * H], I // 8, H)
    gus = tile_scales(blob[lay["gus"]:lay["gus"] + I * H // 8], I // 8, H)
    d = unpack_tiles(blob[lay["dq"]:lay["dq"] + H * I // 2], H // 16, I)
    ds = tile_scales(blob[lay["ds"]:lay["ds"] + H * I // 16], H // 16, I)
    w_gu = gu * np.repeat(gus, 32, axis=2)
    Wg = w_gu[:, :8, :].reshape(I, H)
    Wu = w_gu[:, 8:, :].reshape(I, H)
    Wd = (d * np.repeat(ds, 32, axis=2)).reshape(H, I)
    return Wg, Wu, Wd


# E2M1 magnitudes by (exponent, mantissa) code: the eight values of the
# format, written out by hand.
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def unpack_codes(raw: np.ndarray, tiles: int, K: int) -> np.ndarray:
    """u8 bytes of a tiled section -> 4-bit codes [tiles][16][K] (0..15)."""
    signed = unpack_tiles(raw, tiles, K)
    return np.where(signed < 0, signed + 16, signed)


def e2m1_values(codes: np.ndarray) -> np.ndarray:
    mag = np.asarray(E2M1_MAGNITUDES)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_values(raw: np.ndarray) -> np.ndarray:
    """E4M3 bytes -> float64, decoded by torch's float8_e4m3fn type."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(raw, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def tile_scales_e4m3(raw: np.ndarray, tiles: int, K: int) -> np.ndarray:
    """E4M3 bytes of a tiled scale section -> float64 [tiles][16][K/16]."""
    s = e4m3_values(np.asarray(raw, np.uint8)).reshape(tiles, K // 128, 16, 8)
    return s.transpose(0, 2, 1, 3).reshape(tiles, 16, K // 16)


def dense_expert_nvfp4(blob: np.ndarray, H: int, I: int):
    """(Wg, Wu, Wd) of an NVFP4 blob in float64 (before the fp32 rounding)."""
    lay = synth.blob_layout(H, I, "nvfp4")
    glob = np.asarray(blob[lay["glob"]:lay["glob"] + 12]).view(np.float32).astype(np.float64)
    gu = e2m1_values(unpack_codes(blob[lay["guq"]:lay["guq"] + I * H], I // 8, H))
    gus = tile_scales_e4m3(blob[lay["gus"]:lay["gus"] + I * H // 8], I // 8, H)
    d = e2m1_values(unpack_codes(blob[lay["dq"]:lay["dq"] + H * I // 2], H // 16, I))
    ds = tile_scales_e4m3(blob[lay["ds"]:lay["ds"] + H * I // 16], H // 16, I)
    w_gu = gu * np.repeat(gus, 16, axis=2)
    Wg = w_gu[:, :8, :].reshape(I, H) * glob[0]
    Wu = w_gu[:, 8:, :].reshape(I, H) * glob[1]
    Wd = (d * np.repeat(ds, 16, axis=2)).reshape(H, I) * glob[2]
    return Wg, Wu, Wd


def ffn64(dense, x: np.ndarray) -> np.ndarray:
    Wg, Wu, Wd = dense
    g = Wg @ x
    u = Wu @ x
    h = g / (1.0 + np.exp(-g)) * u
    return Wd @ h


def exact_logits(x_bf16: np.ndarray, W: np.ndarray, bias) -> np.ndarray:
    """fp32 logits from the exact real-number sum (fractions), rounded once.

    Rounding Fraction -> float64 -> float32 can double-round; the chance is
    about 2^-29 per logit, negligible for the tiny sizes used here.
    """
    x = synth.bf16_bits_to_f32(x_bf16).astype(np.float64)
    T, H = x.shape
    E = W.shape[0]
    out = np.zeros((T, E), np.float32)
    for t in range(T):
        for e in range(E):
            acc = Fraction(0)
            for h in range(H):
                acc += Fraction(float(x[t, h])) * Fraction(float(W[e, h]))
            if bias is not None:
                acc += Fraction(float(bias[e]))
            out[t, e] = np.float32(float(acc))
    return out


def topk_by_subsets(l: np.ndarray, k: int):
    """Top-k set = the subset with the largest exact logit sum; among equal sums
    the lexicographically smallest sorted index tuple (lower indices first).
    Returned in descending logit order, ties by ascending index."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(l)), k):
        s = sum(Fraction(float(l[e])) for e in sub)
        if best is None or s > best_sum:
            best, best_sum = sub, s
    return sorted(best, key=lambda e: (-float(l[e]), e))


def layer64(x_bf16, blobs, shared, W, bias, k, H, I):
    """Naive layer: returns (out fp64 [T][H], idx [T][k], w fp64 [T][k])."""
    E = W.shape[0]
    logits = exact_logits(x_bf16, W, bias)
    x = synth.bf16_bits_to_f32(x_bf16).astype(np.float64)
    dense = [dense_expert(b, H, I) for b in blobs]
    dense_sh = [dense_expert(b, H, I) for b in shared]
    T = x.shape[0]
    out = np.zeros((T, H))
    idx = np.zeros((T, k), np.int64)
    wts = np.zeros((T, k))
    for t in range(T):
        ys = [ffn64(d, x[t]) for d in dense]          # every expert, every token
        l64 = logits[t].astype(np.float64)
        p = np.exp(l64 - l64.max())
        p /= p.sum()
        sel = topk_by_subsets(logits[t], k)
        w = p[sel] / p[sel].sum()
        idx[t] = sel
        wts[t] = w
        out[t] = sum(w[j] * ys[sel[j]] for j in range(k))
        for d in dense_sh:
            out[t] += ffn64(d, x[t])
    return out, idx, wts

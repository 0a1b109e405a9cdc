"""Seeded synthetic inputs for the routed int4 expert layer.

This module draws inputs and packs them into the expert-blob format; it holds
none of the layer's arithmetic (no routing, no dequantisation, no matmul).  It
is the one module that both the CPU oracle's tests and the CUDA path's tests
and benchmarks use, so that both sides see byte-identical inputs.

Workloads (shapes, distributions) follow the five layer configurations of the
problem statement: a tiny layer, a DeepSeek-V2-Lite-shaped decode layer, a
Mixtral-shaped decode layer, a 256-expert "wide" decode layer with a 64-slot
arena, and a 256-expert prefill layer.  The pages (Strata "docs/MAC.md",
"Strata on a Mac"; ro99/strata README, "Residency" and "Kernels") describe the
same problem on real checkpoints; nothing here reads a checkpoint.

Expert blob format (one contiguous blob per expert, after Strata "docs/MAC.md",
"What you need", which keeps each expert's matrices together so one request
reads an expert).  H = hidden, I = inter, both multiples of 128.

    section  content                                   bytes
    GU_q     gate + up int4 weights, I/8 row tiles      I*H
    D_q      down int4 weights, H/16 row tiles          H*I/2
    GU_s     gate + up fp16 scales, same tiling         I*H/8
    D_s      down fp16 scales, same tiling              H*I/16

Each section starts at a multiple of 256 bytes; the blob size is rounded up
to 256 bytes.  A row tile has 16 rows: gate/up tile t holds rows 8t..8t+7 of
Wg as tile rows 0..7 and the same rows of Wu as tile rows 8..15; down tile t
holds rows 16t..16t+15 of Wd.  A tile is stored K-group by K-group (128
consecutive K elements), each group as its 16 rows of 64 bytes (q) or of four
fp16 scales (one per block of 32 K elements, block b = elements 32b..32b+31
of the group).  Inside the 64 bytes of one row and group, byte 16w + 4b + m/2
(w, b in 0..3, m in 0..7) holds element 32b + 8w + m, in the low nibble for
even m; a nibble is a two's-complement int4 in [-8, 7].  The weight is
float(scale) * q.  (So the 16 bytes at 16w are word w of each of the four
blocks: one 16-byte load gives the word of every block that an mma.m16n8k16
A fragment needs.)
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

QBLOCK = 32  # K elements per fp16 scale


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    n_shared: int
    n_slots: int
    tokens: tuple
    bias: str = "none"          # "none" | "normal" | "zipf"
    bias_var: float = 0.0       # variance of the normal bias
    zipf_s: float = 0.0         # Zipf exponent of the bias
    zipf_beta: float = 1.0      # multiplier on the Zipf log-pmf
    description: str = ""
    routing: str = "softmax"    # "softmax" | "sigmoid" (with correction bias)
    routed_scale: float = 1.0


# beta for the wide layer: the value at which ~80% of the routed hits of the
# seed-0 tokens land in the 64 highest-ranked experts (checked by
# tests/test_oracle_pins.py::test_wide_zipf_share; derived by
# tests/golden/calibrate_zipf_beta.py, which calls only the oracle).
WIDE_ZIPF_BETA = 0.5390625

CONFIGS = {
    "tiny": LayerConfig(
        "tiny", 256, 512, 8, 2, 0, 8, (4,),
        description="hidden 256, inter 512, 8 experts top-2, 8 slots bound in "
                    "shuffled order, 4 tokens"),
    "dsv2lite": LayerConfig(
        "dsv2lite", 2048, 1408, 64, 6, 2, 64, (1, 8), bias="normal", bias_var=0.5,
        description="DeepSeek-V2-Lite-shaped decode: hidden 2048, inter 1408, 64 "
                    "experts top-6 + 2 shared, per-expert router bias ~N(0,0.5)"),
    "mixtral": LayerConfig(
        "mixtral", 4096, 14336, 8, 2, 0, 8, (1, 4, 16),
        description="Mixtral-shaped decode: hidden 4096, inter 14336, 8 experts "
                    "top-2"),
    "wide": LayerConfig(
        "wide", 4096, 1024, 256, 10, 0, 64, (1, 4), bias="zipf", zipf_s=1.1,
        zipf_beta=WIDE_ZIPF_BETA,
        description="wide-expert decode: hidden 4096, inter 1024, 256 experts "
                    "top-10, 64-slot arena, Zipf(1.1) router bias"),
    "prefill": LayerConfig(
        "prefill", 4096, 2048, 256, 8, 1, 256, (8192,), bias="zipf", zipf_s=0.8,
        zipf_beta=1.0,
        description="prefill: hidden 4096, inter 2048, 256 experts top-8 + 1 "
                    "shared, 8192 tokens, Zipf(0.8) router bias"),
    # the wide-expert layer's shapes, all experts resident, routed like the
    # pages' sigmoid models: sigmoid scores, a per-expert correction bias on
    # the selection, a 2.5x routed scale
    "sigmoid": LayerConfig(
        "sigmoid", 4096, 1024, 256, 10, 0, 256, (1, 4), routing="sigmoid", routed_scale=2.5,
        description="sigmoid-routed decode: hidden 4096, inter 1024, 256 experts top-10, "
                    "correction bias ~N(0, 0.05^2), routed scale 2.5"),
    # the prefill layer over an arena of half its experts, filled chunk by
    # chunk (chunked prefill with a partial arena)
    "prefill_paged": LayerConfig(
        "prefill_paged", 4096, 2048, 256, 8, 1, 128, (8192,), bias="zipf", zipf_s=0.8,
        zipf_beta=1.0,
        description="prefill through a 128-slot arena: hidden 4096, inter 2048, 256 experts "
                    "top-8 + 1 shared, 8192 tokens, Zipf(0.8) router bias"),
    # the prefill layer's shapes with 32 experts and 2048 tokens: small enough
    # (about 0.5 GB of blobs) for profiler captures and quick parity runs
    "prefill_small": LayerConfig(
        "prefill_small", 4096, 2048, 32, 8, 1, 32, (2048,), bias="zipf", zipf_s=0.8,
        zipf_beta=1.0,
        description="prefill-shaped, small: hidden 4096, inter 2048, 32 experts "
                    "top-8 + 1 shared, 2048 tokens, Zipf(0.8) router bias"),
}


def custom_config(name, hidden, inter, n_experts, top_k, n_shared=0, n_slots=None,
                  tokens=(4,), bias="none", bias_var=0.0, zipf_s=0.0, zipf_beta=1.0):
    """A config with the same distributions at other sizes (tests, edge cases)."""
    return LayerConfig(name, hidden, inter, n_experts, top_k, n_shared,
                       n_experts if n_slots is None else n_slots, tuple(tokens),
                       bias, bias_var, zipf_s, zipf_beta)


# ----------------------------------------------------------------------------
# format helpers (layout only; no arithmetic of the layer)

def _align256(v: int) -> int:
    return (v + 255) // 256 * 256


def blob_layout(hidden: int, inter: int, fmt: str = "int4") -> dict:
    """Byte offsets of the sections and the blob size.  NVFP4 adds a 256-byte
    section of three fp32 global scales (gate, up, down)."""
    H, I = hidden, inter
    sizes = [("guq", I * H), ("dq", H * I // 2), ("gus", I * H // 8), ("ds", H * I // 16)]
    if fmt == "nvfp4":
        sizes.append(("glob", 12))
    off, out = 0, {}
    for name, size in sizes:
        out[name] = off
        off = _align256(off + size)
    out["total"] = off
    return out


def expert_bytes(hidden: int, inter: int, fmt: str = "int4") -> int:
    return blob_layout(hidden, inter, fmt)["total"]


def _check_int4(q):
    q = np.asarray(q)
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("int4 values must lie in [-8, 7]")
    return q


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Plain row-major packing: int [rows][K] -> u8 [rows][K/2] (element 2j in
    the low nibble of byte j).  Used to state the nibble convention."""
    n = (_check_int4(q).astype(np.int16) & 0xF).astype(np.uint8)
    return (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)


def pack_tiles(q_tiles: np.ndarray) -> np.ndarray:
    """int [tiles][16][K] -> u8 [tiles][K/128][16][64] in the group layout."""
    q = _check_int4(q_tiles)
    t, r, K = q.shape
    assert r == 16 and K % 128 == 0
    # element 32b + 8w + m of a group -> (b, w, m); stored in order (w, b, m)
    g = q.reshape(t, 16, K // 128, 4, 4, 8).transpose(0, 2, 1, 4, 3, 5)
    n = (g.astype(np.int16) & 0xF).astype(np.uint8)
    packed = n[..., 0::2] | (n[..., 1::2] << 4)          # [t][G][16][w][b][4]
    return packed.reshape(t, K // 128, 16, 64)


def pack_tile_scales(s_tiles: np.ndarray) -> np.ndarray:
    """f16 [tiles][16][K/32] -> f16 [tiles][K/128][16][4]."""
    s = np.asarray(s_tiles, np.float16)
    t, r, nb = s.shape
    return s.reshape(t, 16, nb // 4, 4).transpose(0, 2, 1, 3).copy()


def pack_tile_codes(c_tiles: np.ndarray) -> np.ndarray:
    """4-bit codes (0..15) [tiles][16][K] -> u8 [tiles][K/128][16][64], placed
    like the int4 values (NVFP4 stores E2M1 codes in the same nibbles)."""
    c = np.asarray(c_tiles)
    if c.min(initial=0) < 0 or c.max(initial=0) > 15:
        raise ValueError("codes must lie in [0, 15]")
    return pack_tiles(np.where(c >= 8, c - 16, c))


def pack_tile_scales_e4m3(s_tiles: np.ndarray) -> np.ndarray:
    """E4M3 scale bytes [tiles][16][K/16] -> u8 [tiles][K/128][16][8]."""
    s = np.asarray(s_tiles, np.uint8)
    t, r, ng = s.shape
    return s.reshape(t, 16, ng // 8, 8).transpose(0, 2, 1, 3).copy()


def gate_up_tiles(wg: np.ndarray, wu: np.ndarray) -> np.ndarray:
    """[I][K] gate and up arrays -> [I/8][16][K] tiles (8 gate rows, 8 up rows)."""
    wg, wu = np.asarray(wg), np.asarray(wu)
    I = wg.shape[0]
    return np.concatenate([wg.reshape(I // 8, 8, -1), wu.reshape(I // 8, 8, -1)], axis=1)


def down_tiles(wd: np.ndarray) -> np.ndarray:
    wd = np.asarray(wd)
    return wd.reshape(wd.shape[0] // 16, 16, -1)


def build_blob(hidden, inter, gq, uq, dq, gs, us, ds) -> np.ndarray:
    """Assemble one expert blob from explicit int4 values and fp16 scales.

    gq, uq: int [I][H]; dq: int [H][I]; gs, us: float16 [I][H/32];
    ds: float16 [H][I/32].
    """
    H, I = hidden, inter
    lay = blob_layout(H, I)
    blob = np.zeros(lay["total"], np.uint8)

    def put(name, arr):
        raw = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
        blob[lay[name]:lay[name] + raw.size] = raw

    put("guq", pack_tiles(gate_up_tiles(np.asarray(gq).reshape(I, H), np.asarray(uq).reshape(I, H))))
    put("dq", pack_tiles(down_tiles(np.asarray(dq).reshape(H, I))))
    put("gus", pack_tile_scales(gate_up_tiles(np.asarray(gs, np.float16).reshape(I, H // QBLOCK),
                                              np.asarray(us, np.float16).reshape(I, H // QBLOCK))))
    put("ds", pack_tile_scales(down_tiles(np.asarray(ds, np.float16).reshape(H, I // QBLOCK))))
    return blob


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even); returns u16 bits."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# seeded draws; every stream is keyed by (seed, purpose, index)

_STREAM_X, _STREAM_ROUTER, _STREAM_BIAS, _STREAM_EXPERT, _STREAM_SLOTS, _STREAM_RANK = range(6)
_STREAM_CORR = 6
_STREAM_EXPERT_FP4 = 7


def _rng(seed: int, stream: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), stream, int(index)]))


def make_x(cfg: LayerConfig, n_tokens: int, seed: int = 0, step: int = 0) -> np.ndarray:
    """Token activations: bf16 (round to nearest even) of N(0,1); u16 bits [T][H]."""
    r = _rng(seed, _STREAM_X, step)
    return f32_to_bf16_bits(r.standard_normal((n_tokens, cfg.hidden), dtype=np.float32))


def zipf_ranks(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """Rank (1 = most popular) of every expert under the Zipf bias."""
    r = _rng(seed, _STREAM_RANK)
    return r.permutation(cfg.n_experts).astype(np.int64) + 1


def make_router(cfg: LayerConfig, seed: int = 0):
    """Router weights fp32 [E][H] ~ N(0, 1/H) and bias fp32 [E] (or None)."""
    r = _rng(seed, _STREAM_ROUTER)
    W = (r.standard_normal((cfg.n_experts, cfg.hidden), dtype=np.float64)
         / math.sqrt(cfg.hidden)).astype(np.float32)
    if cfg.bias == "none":
        b = None
    elif cfg.bias == "normal":
        rb = _rng(seed, _STREAM_BIAS)
        b = (rb.standard_normal(cfg.n_experts) * math.sqrt(cfg.bias_var)).astype(np.float32)
    elif cfg.bias == "zipf":
        ranks = zipf_ranks(cfg, seed)
        b = (-cfg.zipf_beta * cfg.zipf_s * np.log(ranks.astype(np.float64))).astype(np.float32)
    else:
        raise ValueError(cfg.bias)
    return W, b


def build_blob_nvfp4(hidden, inter, gc, uc, dc, gs, us, ds, glob) -> np.ndarray:
    """Assemble one NVFP4 expert blob.  gc, uc: E2M1 codes [I][H]; dc: [H][I];
    gs, us: E4M3 scale bytes [I][H/16]; ds: [H][I/16]; glob: three fp32 global
    scales (gate, up, down)."""
    H, I = hidden, inter
    lay = blob_layout(H, I, "nvfp4")
    blob = np.zeros(lay["total"], np.uint8)

    def put(name, arr):
        raw = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
        blob[lay[name]:lay[name] + raw.size] = raw

    put("guq", pack_tile_codes(gate_up_tiles(np.asarray(gc).reshape(I, H),
                                             np.asarray(uc).reshape(I, H))))
    put("dq", pack_tile_codes(down_tiles(np.asarray(dc).reshape(H, I))))
    put("gus", pack_tile_scales_e4m3(gate_up_tiles(np.asarray(gs).reshape(I, H // 16),
                                                   np.asarray(us).reshape(I, H // 16))))
    put("ds", pack_tile_scales_e4m3(down_tiles(np.asarray(ds).reshape(H, I // 16))))
    put("glob", np.asarray(glob, np.float32))
    return blob


# E4M3 scale bytes drawn for synthetic NVFP4 experts: exponent field 3..6 with
# any mantissa, i.e. values in [2^-4, 1.875 * 2^-1].
_E4M3_SCALE_CODES = np.array([(e << 3) | m for e in range(3, 7) for m in range(8)], np.uint8)


def make_expert_blob_nvfp4(cfg: LayerConfig, expert: int, seed: int = 0) -> np.ndarray:
    """One NVFP4 expert blob: uniform random E2M1 codes (random bytes), scale
    bytes uniform over _E4M3_SCALE_CODES, global scales U[0.02, 0.08]."""
    H, I = cfg.hidden, cfg.inter
    lay = blob_layout(H, I, "nvfp4")
    r = _rng(seed, _STREAM_EXPERT_FP4, expert)
    blob = np.zeros(lay["total"], np.uint8)
    for name, nbytes in (("guq", I * H), ("dq", H * I // 2)):
        blob[lay[name]:lay[name] + nbytes] = np.frombuffer(r.bytes(nbytes), np.uint8)
    for name, count in (("gus", I * H // 8), ("ds", H * I // 16)):
        blob[lay[name]:lay[name] + count] = r.choice(_E4M3_SCALE_CODES, size=count)
    glob = r.uniform(0.02, 0.08, size=3).astype(np.float32)
    blob[lay["glob"]:lay["glob"] + 12] = glob.view(np.uint8)
    return blob


def make_correction_bias(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """Per-expert correction bias of the sigmoid router, fp32 [E] ~ N(0, 0.05^2)
    (same order as the scores' spread near 0.5, so it reorders experts)."""
    r = _rng(seed, _STREAM_CORR)
    return (r.standard_normal(cfg.n_experts) * 0.05).astype(np.float32)


def make_expert_blob(cfg: LayerConfig, expert: int, seed: int = 0) -> np.ndarray:
    """One expert blob; expert in [0, E) routed, [E, E+S) shared.

    int4 values are uniform in [-8, 7] (a uniform random byte is two independent
    uniform nibbles, whatever the byte's place in the layout); scales are fp16
    (round to nearest even) of U[0.005, 0.02].
    """
    H, I = cfg.hidden, cfg.inter
    lay = blob_layout(H, I)
    r = _rng(seed, _STREAM_EXPERT, expert)
    blob = np.zeros(lay["total"], np.uint8)
    for name, nbytes in (("guq", I * H), ("dq", H * I // 2)):
        blob[lay[name]:lay[name] + nbytes] = np.frombuffer(r.bytes(nbytes), np.uint8)
    for name, count in (("gus", I * H // 16), ("ds", H * I // 32)):
        s = r.uniform(0.005, 0.02, size=count).astype(np.float32).astype(np.float16)
        raw = s.view(np.uint8)
        blob[lay[name]:lay[name] + raw.size] = raw
    return blob


def make_all_blobs(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """All E + S blobs as one u8 array [E+S][expert_bytes]."""
    nb = expert_bytes(cfg.hidden, cfg.inter)
    out = np.empty((cfg.n_experts + cfg.n_shared, nb), np.uint8)
    for e in range(cfg.n_experts + cfg.n_shared):
        out[e] = make_expert_blob(cfg, e, seed)
    return out


def make_all_blobs_nvfp4(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """All E + S NVFP4 blobs as one u8 array [E+S][expert_bytes(..., "nvfp4")]."""
    nb = expert_bytes(cfg.hidden, cfg.inter, "nvfp4")
    out = np.empty((cfg.n_experts + cfg.n_shared, nb), np.uint8)
    for e in range(cfg.n_experts + cfg.n_shared):
        out[e] = make_expert_blob_nvfp4(cfg, e, seed)
    return out


def make_slot_permutation(cfg: LayerConfig, seed: int = 0, index: int = 0) -> np.ndarray:
    """Seeded permutation: slot s holds expert perm[s] (all experts bound)."""
    return _rng(seed, _STREAM_SLOTS, index).permutation(cfg.n_experts).astype(np.int32)

// CPU oracle for the routed int4 expert layer -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, single-threaded restatement of what the layer computes, used
// to check the CUDA library.  Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load it; the library itself never does.
// It shares no code with the CUDA path (its own format reader, its own fp16
// decoder, its own routing), and nothing here is blocked, fused or reordered
// beyond what the definition states.
//
// What it computes, and the passages it follows:
//  * Routing: each token goes to its k best experts by an fp32 router
//    GEMV, softmax, top-k with lowest-index tie-break and renormalisation
//    (the layer statement this library implements; the fused router dispatch
//    of Strata "docs/MAC.md", section "Switches", two opt-ins paragraph).
//    Reading taken where the pages are silent: products x*W are exact in
//    double and are summed in double in ascending h order, the bias is added
//    in double, the sum is rounded once to an fp32 logit; top-k compares the
//    fp32 logits; softmax is fp32 with max subtraction over all experts; the
//    selected probabilities are divided by their sum.
//  * Expert lookup through a slot table (the engine keeps the routed experts
//    of each decode step in GPU memory under LRU replacement: ro99/strata
//    README, "Residency").
//  * Expert FFN on 4-bit weights with 16-bit activations (the int4 weight
//    format of ro99/strata README, model table), read from the tiled blob
//    format described at
//    place_of(): w = float(fp16 scale) * q, exact in fp32; gate and
//    up dot products in fp32 in ascending K; h = silu(g) * u with
//    silu(z) = z / (1 + exp(-z)) in fp32; down projection in fp32 ascending K.
//  * Combine: out[t] = sum_j w[t][j] * y[t][j] (j = 0..k-1, descending logit)
//    followed by + y_shared[t][s] (s = 0..S-1), fp32, in that fixed order
//    (a fixed order is what the bit-exact fidelity tier of
//    strata.amperor.ai "/methods/", "Fidelity (paged vs resident output)",
//    requires).
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

namespace {

enum {
  ORC_OK = 0,
  ORC_BAD_ARG = 1,
  ORC_NOT_BOUND = 2,
  ORC_SLOT_CONFLICT = 3,
};

size_t round_up_256(size_t v) { return (v + 255) / 256 * 256; }

// Weight formats of an expert blob.
//  FMT_INT4:  4-bit two's-complement integers, one fp16 scale per 32 along K.
//  FMT_NVFP4: 4-bit E2M1 floats, one E4M3 scale per 16 along K, one fp32
//             global scale per matrix (the NVFP4 routed-expert format of
//             ro99/strata README, model table); weights are used with 16-bit
//             activations as for int4.
enum Format { FMT_INT4 = 0, FMT_NVFP4 = 1 };

// Section offsets of one expert blob, in bytes from its start:
// gate+up weights, down weights, gate+up scales, down scales, and for NVFP4
// a 256-byte section of three fp32 global scales (gate, up, down).
struct Layout {
  size_t guq, dq, gus, ds, glob, total;
};

Layout layout_of(int H, int I, int fmt = FMT_INT4) {
  Layout L;
  size_t off = 0;
  L.guq = off; off = round_up_256(off + (size_t)I * H);
  L.dq = off;  off = round_up_256(off + (size_t)H * I / 2);
  L.gus = off; off = round_up_256(off + (size_t)I * H / 8);
  L.ds = off;  off = round_up_256(off + (size_t)H * I / 16);
  L.glob = off;
  if (fmt == FMT_NVFP4) off = round_up_256(off + 3 * sizeof(float));
  L.total = off;
  return L;
}

// bfloat16 bits -> float: the top 16 bits of an IEEE binary32.
float bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// IEEE binary16 bits -> float, from the definition of the format:
// sign, 5-bit exponent (bias 15), 10-bit fraction; subnormals have exponent
// field 0 and value 2^-14 * fraction / 1024.
float f16_value(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 10) & 0x1F;
  int frac = bits & 0x3FF;
  double v;
  if (expo == 0) {
    v = std::ldexp((double)frac, -24);
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = std::ldexp(1.0 + frac / 1024.0, expo - 15);
  }
  return (float)(sign ? -v : v);
}

// E2M1 (sign, 2-bit exponent with bias 1, 1-bit mantissa), from the format's
// definition: exponent 0 is subnormal (0 or 0.5), else 2^(e-1) * (1 + m/2).
float e2m1_value(int code) {
  const int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double v = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return (float)(sign ? -v : v);
}

// E4M3 (sign, 4-bit exponent with bias 7, 3-bit mantissa; no infinities,
// exponent 15 with mantissa 7 is NaN), from the format's definition.
float e4m3_value(uint8_t byte) {
  const int sign = (byte >> 7) & 1, e = (byte >> 3) & 0xF, m = byte & 7;
  double v;
  if (e == 0)
    v = std::ldexp((double)m / 8.0, -6);
  else if (e == 15 && m == 7)
    v = NAN;
  else
    v = std::ldexp(1.0 + m / 8.0, e - 7);
  return (float)(sign ? -v : v);
}

// The three matrices of an expert and where their rows live.  A section is
// split into tiles of 16 rows; gate row i is row i % 8 of tile i / 8 and up
// row i is row 8 + i % 8 of the same tile; down row r is row r % 16 of tile
// r / 16.  A tile is stored group by group (128 K elements), each group as
// 16 rows of 64 bytes; element k of a row sits in group k / 128, block
// b = (k % 128) / 32, word w = (k % 32) / 8, nibble m = k % 8, at byte
// 16 w + 4 b + m / 2 of the row's 64 bytes (low nibble for even m).  Scales:
// per tile, group, row: four fp16 values, one per block (INT4), or eight
// E4M3 bytes, scale i for elements 16 i .. 16 i + 15 of the group (NVFP4;
// the same 8 bytes per row and group).
enum Matrix { GATE, UP, DOWN };

struct RowPlace {
  const uint8_t *q;      // section start
  const uint16_t *s;     // scale section start
  int K, tile, trow;
  float glob;            // NVFP4 global scale of the matrix
};

RowPlace place_of(const uint8_t *blob, int H, int I, Matrix mat, int row,
                  int fmt = FMT_INT4) {
  Layout L = layout_of(H, I, fmt);
  RowPlace p;
  p.glob = 1.0f;
  if (fmt == FMT_NVFP4) std::memcpy(&p.glob, blob + L.glob + sizeof(float) * (int)mat, sizeof(float));
  if (mat == DOWN) {
    p.q = blob + L.dq;
    p.s = (const uint16_t *)(blob + L.ds);
    p.K = I;
    p.tile = row / 16;
    p.trow = row % 16;
  } else {
    p.q = blob + L.guq;
    p.s = (const uint16_t *)(blob + L.gus);
    p.K = H;
    p.tile = row / 8;
    p.trow = (mat == GATE ? 0 : 8) + row % 8;
  }
  return p;
}

// The 4-bit code of element k (both formats place codes alike).
int nibble_at(const RowPlace &p, int k) {
  const int j = k / 128, b = (k % 128) / 32, w = (k % 32) / 8, m = k % 8;
  const size_t row_base = (((size_t)p.tile * (p.K / 128) + j) * 16 + p.trow) * 64;
  const uint8_t byte = p.q[row_base + 16 * w + 4 * b + m / 2];
  return (m % 2 == 0) ? (byte & 0xF) : (byte >> 4);
}

int int4_at(const RowPlace &p, int k) {
  const int n = nibble_at(p, k);
  return n >= 8 ? n - 16 : n;
}

// NVFP4 group scale of element k: E4M3 byte (k % 128) / 16 of the row's 8.
float e4m3_scale_at(const RowPlace &p, int k) {
  const int j = k / 128, i = (k % 128) / 16;
  const uint8_t *s8 = reinterpret_cast<const uint8_t *>(p.s);
  return e4m3_value(s8[(((size_t)p.tile * (p.K / 128) + j) * 16 + p.trow) * 8 + i]);
}

float scale_at(const RowPlace &p, int k) {
  const int j = k / 128, b = (k % 128) / 32;
  return f16_value(p.s[(((size_t)p.tile * (p.K / 128) + j) * 16 + p.trow) * 4 + b]);
}

// One dequantised row of an expert matrix (K = H for gate/up, I for down).
// INT4: w = float(fp16 scale) * q, exact in fp32.  NVFP4: w = (e2m1 value *
// E4M3 scale, exact in fp32) * fp32 global scale, rounded once.
void dequant_row(const uint8_t *blob, int H, int I, Matrix mat, int row, float *out,
                 int fmt = FMT_INT4) {
  const RowPlace p = place_of(blob, H, I, mat, row, fmt);
  if (fmt == FMT_NVFP4) {
    for (int k = 0; k < p.K; ++k) {
      const float v = e2m1_value(nibble_at(p, k)) * e4m3_scale_at(p, k);
      out[k] = v * p.glob;
    }
    return;
  }
  for (int b0 = 0; b0 < p.K; b0 += 32) {
    const float scale = scale_at(p, b0);
    for (int k = b0; k < b0 + 32; ++k) out[k] = scale * (float)int4_at(p, k);
  }
}

float silu(float z) { return z / (1.0f + std::exp(-z)); }

// y[n][H] = FFN(x[n][H]) for n tokens through one expert blob.
// Optional g, u, h outputs are [n][I].
void expert_ffn(const uint8_t *blob, int H, int I, const float *x, int n,
                float *g_out, float *u_out, float *h_out, float *y, int fmt = FMT_INT4) {
  std::vector<float> wg(H), wu(H), wd(I), h((size_t)n * I);
  for (int i = 0; i < I; ++i) {
    dequant_row(blob, H, I, GATE, i, wg.data(), fmt);
    dequant_row(blob, H, I, UP, i, wu.data(), fmt);
    for (int t = 0; t < n; ++t) {
      const float *xt = x + (size_t)t * H;
      float g = 0.0f, u = 0.0f;
      for (int c = 0; c < H; ++c) {
        g = g + wg[c] * xt[c];
        u = u + wu[c] * xt[c];
      }
      float hv = silu(g) * u;
      h[(size_t)t * I + i] = hv;
      if (g_out) g_out[(size_t)t * I + i] = g;
      if (u_out) u_out[(size_t)t * I + i] = u;
      if (h_out) h_out[(size_t)t * I + i] = hv;
    }
  }
  for (int r = 0; r < H; ++r) {
    dequant_row(blob, H, I, DOWN, r, wd.data(), fmt);
    for (int t = 0; t < n; ++t) {
      const float *ht = h.data() + (size_t)t * I;
      float acc = 0.0f;
      for (int c = 0; c < I; ++c) acc = acc + wd[c] * ht[c];
      y[(size_t)t * H + r] = acc;
    }
  }
}

// Blob bound to expert e in the slot table, or nullptr.
const uint8_t *lookup(const int32_t *slot_expert, const uint8_t *const *slot_blob,
                      int n_slots, int e) {
  for (int s = 0; s < n_slots; ++s)
    if (slot_expert[s] == e && slot_blob[s]) return slot_blob[s];
  return nullptr;
}

}  // namespace

extern "C" {

size_t oracle_expert_bytes(int H, int I) { return layout_of(H, I).total; }
size_t oracle_expert_bytes_fmt(int H, int I, int fmt) { return layout_of(H, I, fmt).total; }

// Router for T tokens.  x: bf16 bits [T][H]; Wr: fp32 [E][H]; bias: fp32 [E]
// or null.  Outputs: logits fp32 [T][E] (may be null), idx [T][k], w [T][k].
int oracle_route(const uint16_t *x, int T, int H, const float *Wr, const float *bias,
                 int E, int k, float *logits, int32_t *idx, float *w) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return ORC_BAD_ARG;
  std::vector<float> l(E), p(E);
  std::vector<char> taken(E);
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)bf16_value(x[(size_t)t * H + h]) * (double)Wr[(size_t)e * H + h];
      if (bias) acc += (double)bias[e];
      l[e] = (float)acc;
      if (logits) logits[(size_t)t * E + e] = l[e];
    }
    // top-k: repeatedly take the largest remaining logit; a strict comparison
    // keeps the lowest index among equal logits.
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    // softmax over all experts (fp32, max subtracted), then renormalise the
    // selected probabilities.
    float m = l[0];
    for (int e = 1; e < E; ++e) m = l[e] > m ? l[e] : m;
    float Z = 0.0f;
    for (int e = 0; e < E; ++e) {
      p[e] = std::exp(l[e] - m);
      Z = Z + p[e];
    }
    for (int e = 0; e < E; ++e) p[e] = p[e] / Z;
    float sel = 0.0f;
    for (int j = 0; j < k; ++j) sel = sel + p[idx[(size_t)t * k + j]];
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]] / sel;
  }
  return ORC_OK;
}

// Sigmoid router with a correction bias and a routed scale (the "sigmoid
// top-10 routing with a correction bias and a 2.5x routed scale" of
// ro99/strata README, model notes under the model table).  Logits as in
// oracle_route; score s_e = 1 / (1 + exp(-l_e)) evaluated in double and
// rounded to fp32; selection key = s_e + corr[e] (fp32; corr may be null =
// zeros); the k largest keys, lower index first among equal keys; weights =
// s_e / (sum of the selected scores, added in selection order) * scale, fp32.
int oracle_route_sigmoid(const uint16_t *x, int T, int H, const float *Wr, const float *bias,
                         const float *corr, float scale, int E, int k, float *logits,
                         int32_t *idx, float *w) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return ORC_BAD_ARG;
  std::vector<float> l(E), sc(E), key(E);
  std::vector<char> taken(E);
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)bf16_value(x[(size_t)t * H + h]) * (double)Wr[(size_t)e * H + h];
      if (bias) acc += (double)bias[e];
      l[e] = (float)acc;
      if (logits) logits[(size_t)t * E + e] = l[e];
      sc[e] = (float)(1.0 / (1.0 + std::exp(-(double)l[e])));
      key[e] = corr ? sc[e] + corr[e] : sc[e];
    }
    std::fill(taken.begin(), taken.end(), 0);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
      taken[best] = 1;
      idx[(size_t)t * k + j] = best;
    }
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum = sum + sc[idx[(size_t)t * k + j]];
    for (int j = 0; j < k; ++j)
      w[(size_t)t * k + j] = sc[idx[(size_t)t * k + j]] / sum * scale;
  }
  return ORC_OK;
}

// One expert on n tokens given as fp32 activations.  Any of g, u, h may be
// null; y is [n][H].
int oracle_expert_ffn_fmt(const uint8_t *blob, int H, int I, int fmt, const float *x, int n,
                          float *g, float *u, float *h, float *y) {
  if (!blob || H <= 0 || I <= 0 || H % 128 || I % 128 || n < 0) return ORC_BAD_ARG;
  if (fmt != FMT_INT4 && fmt != FMT_NVFP4) return ORC_BAD_ARG;
  expert_ffn(blob, H, I, x, n, g, u, h, y, fmt);
  return ORC_OK;
}

int oracle_expert_ffn(const uint8_t *blob, int H, int I, const float *x, int n,
                      float *g, float *u, float *h, float *y) {
  return oracle_expert_ffn_fmt(blob, H, I, FMT_INT4, x, n, g, u, h, y);
}

// Layer output for T tokens with routing given.  Experts are found through
// the slot table (slot s holds expert slot_expert[s] at slot_blob[s]; -1 or a
// null blob = empty).  out: fp32 [T][H].  A token whose routed expert is not
// bound gets a zero output row and the call returns ORC_NOT_BOUND.
int oracle_forward_routed_fmt(const uint16_t *x, int T, int H, int I, int E, int k, int S,
                              const int32_t *slot_expert, const uint8_t *const *slot_blob,
                              int n_slots, const uint8_t *const *shared_blob,
                              const int32_t *idx, const float *w, float *out, int fmt) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || S < 0 || n_slots < 0)
    return ORC_BAD_ARG;
  if (fmt != FMT_INT4 && fmt != FMT_NVFP4) return ORC_BAD_ARG;
  if (H % 128 || I % 128) return ORC_BAD_ARG;
  // the same expert in two slots is a conflict
  for (int a = 0; a < n_slots; ++a)
    for (int b = a + 1; b < n_slots; ++b)
      if (slot_expert[a] >= 0 && slot_expert[a] == slot_expert[b]) return ORC_SLOT_CONFLICT;
  int status = ORC_OK;
  std::vector<float> xf((size_t)T * H);
  for (size_t i = 0; i < xf.size(); ++i) xf[i] = bf16_value(x[i]);
  // y[t][j] for j < k + S, computed expert by expert (each expert's weights
  // are decoded once and applied to every token routed to it).
  std::vector<float> y((size_t)T * (k + S) * H, 0.0f);
  std::vector<char> token_ok(T, 1);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) return ORC_BAD_ARG;
      if (!lookup(slot_expert, slot_blob, n_slots, e)) token_ok[t] = 0;
    }
  std::vector<float> xin, yout;
  for (int e = 0; e < E + S; ++e) {
    std::vector<std::pair<int, int>> uses;  // (t, j)
    for (int t = 0; t < T; ++t) {
      if (!token_ok[t]) continue;
      if (e < E) {
        for (int j = 0; j < k; ++j)
          if (idx[(size_t)t * k + j] == e) uses.push_back({t, j});
      } else {
        uses.push_back({t, k + (e - E)});
      }
    }
    if (uses.empty()) continue;
    const uint8_t *blob = e < E ? lookup(slot_expert, slot_blob, n_slots, e) : shared_blob[e - E];
    if (!blob) return ORC_BAD_ARG;  // a shared expert must be given
    int n = (int)uses.size();
    xin.assign((size_t)n * H, 0.0f);
    yout.assign((size_t)n * H, 0.0f);
    for (int a = 0; a < n; ++a)
      std::memcpy(&xin[(size_t)a * H], &xf[(size_t)uses[a].first * H], sizeof(float) * H);
    expert_ffn(blob, H, I, xin.data(), n, nullptr, nullptr, nullptr, yout.data(), fmt);
    for (int a = 0; a < n; ++a)
      std::memcpy(&y[((size_t)uses[a].first * (k + S) + uses[a].second) * H],
                  &yout[(size_t)a * H], sizeof(float) * H);
  }
  for (int t = 0; t < T; ++t) {
    float *o = out + (size_t)t * H;
    for (int r = 0; r < H; ++r) o[r] = 0.0f;
    if (!token_ok[t]) {
      status = ORC_NOT_BOUND;
      continue;
    }
    for (int j = 0; j < k; ++j) {
      float wj = w[(size_t)t * k + j];
      const float *yj = &y[((size_t)t * (k + S) + j) * H];
      for (int r = 0; r < H; ++r) o[r] = o[r] + wj * yj[r];
    }
    for (int s = 0; s < S; ++s) {
      const float *ys = &y[((size_t)t * (k + S) + k + s) * H];
      for (int r = 0; r < H; ++r) o[r] = o[r] + ys[r];
    }
  }
  return status;
}

int oracle_forward_routed(const uint16_t *x, int T, int H, int I, int E, int k, int S,
                          const int32_t *slot_expert, const uint8_t *const *slot_blob,
                          int n_slots, const uint8_t *const *shared_blob,
                          const int32_t *idx, const float *w, float *out) {
  return oracle_forward_routed_fmt(x, T, H, I, E, k, S, slot_expert, slot_blob, n_slots,
                                   shared_blob, idx, w, out, FMT_INT4);
}

// Router followed by the routed layer.  idx/w/logits outputs may be null.
int oracle_forward(const uint16_t *x, int T, int H, int I, int E, int k, int S,
                   const float *Wr, const float *bias, const int32_t *slot_expert,
                   const uint8_t *const *slot_blob, int n_slots,
                   const uint8_t *const *shared_blob, float *logits, int32_t *idx_out,
                   float *w_out, float *out) {
  if (T < 0 || k <= 0 || k > E) return ORC_BAD_ARG;
  std::vector<int32_t> idx((size_t)T * k);
  std::vector<float> w((size_t)T * k);
  int st = oracle_route(x, T, H, Wr, bias, E, k, logits, idx.data(), w.data());
  if (st != ORC_OK) return st;
  if (idx_out) std::memcpy(idx_out, idx.data(), sizeof(int32_t) * idx.size());
  if (w_out) std::memcpy(w_out, w.data(), sizeof(float) * w.size());
  return oracle_forward_routed(x, T, H, I, E, k, S, slot_expert, slot_blob, n_slots,
                               shared_blob, idx.data(), w.data(), out);
}

}  // extern "C"

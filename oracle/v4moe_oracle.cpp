// CPU oracle of the routed MoE FFN layer of DeepSeek-V4-Flash.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, single-threaded fp64
// definition that the CUDA library is checked against. Only the tests, the
// package's smoke check and the benchmark's CPU-baseline leg may load it. It
// shares no source, header, table or helper with the CUDA library.
//
// Sources (web pages on the subject; each function names the passage it
// follows):
//  [P1] "DeepSeek-V4-Flash export design" (onnxruntime mobius design note),
//       section "Source configuration".
//  [P3] "Tidalluna/DeepSeek-V4-Flash-0731-Tina-CQ4KM" model card, section
//       "llama.cpp / GGUF incompatibility", item 2 (routing semantics).
//  [P4] "DeepSeek-V4-Flash-0731" catalog page (models.inteligile.com), table
//       "Checked in its code", rows "Mixture of experts", "Shared expert",
//       "Auxiliary-loss-free load balancing (selection bias)", "SwiGLU
//       feed-forward".
//  [P5] "appmana/deepseek-v4-mxfp4-int8 config.json": keys
//       quantization_config.config_groups.experts_w4a16 / linears_w8a16,
//       scoring_func, norm_topk_prob, routed_scaling_factor, swiglu_limit,
//       topk_method, num_hash_layers.
//  [OCP] OCP Microscaling Formats (MX) v1.0 specification: E2M1 element
//       encoding and the E8M0 scale (the pages name the format "mxfp4" with
//       scale dtype "e8m0" and group size 32 but do not print the tables).
//
// Readings where the pages are silent (each is listed in the design notes):
//  * E2M1/E8M0 decode per OCP MX v1.0; E8M0 0xFF (NaN) never occurs in inputs.
//  * Packing: two codes per byte along K, even K index in the low nibble.
//  * w13 rows [0, I) are the gate projection (w1), rows [I, 2I) the up
//    projection (w3).
//  * Learned routing emits the k selected ids in ascending expert id; ties in
//    the biased score go to the lower expert index. Hash routing emits the
//    table's columns in order.
//  * Routing weights: unbiased scores of the selected experts, normalised to
//    sum 1, then multiplied by routed_scaling_factor; no epsilon. Hash layers
//    use the same weights at the table's experts.
//  * The shared expert sees the same x, is added with weight 1, and uses the
//    same clamped SwiGLU.
//
// Parity status: every function here is pinned by the not-gpu test suite
// (closed forms, hand-built blocks, invariants, brute force on tiny shapes).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

extern "C" {

struct OrcLayer {
  int32_t T, H, E, k, I, Is, vocab, pad_;
  double routed_scale, swiglu_limit;
  const uint16_t* x;         // [T, H] bf16 bits
  const uint16_t* gate;      // [E, H] bf16 bits
  const float* bias;         // [E] (learned routing) or null
  const int32_t* token_ids;  // [T] (hash routing) or null
  const int32_t* tid2eid;    // [vocab, k] (hash routing) or null
  const uint8_t* w13_codes;  // [E, 2I, H/2]
  const uint8_t* w13_scales; // [E, 2I, H/32]
  const uint8_t* w2_codes;   // [E, H, I/2]
  const uint8_t* w2_scales;  // [E, H, I/32]
  const int8_t* sh13;        // [2Is, H] or null
  const float* sh13_scale;   // [2Is]
  const int8_t* sh2;         // [H, Is]
  const float* sh2_scale;    // [H]
};

// bf16 -> double: a bf16 value is the upper half of an fp32 pattern; the
// conversion to double is exact.
double orc_bf16_to_double(uint16_t b) {
  const uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// [OCP] E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
// Exponent 0 is subnormal: value = mantissa * 2^(1-1) * 0.5.
double orc_e2m1(int code) {
  const int s = (code >> 3) & 1;
  const int e = (code >> 1) & 3;
  const int m = code & 1;
  double mag;
  if (e == 0)
    mag = 0.5 * m;
  else
    mag = std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// [OCP] E8M0 scale: 2^(e - 127); e = 255 encodes NaN.
double orc_e8m0(int e) {
  if (e == 255) return std::numeric_limits<double>::quiet_NaN();
  return std::ldexp(1.0, e - 127);
}

// [P5] experts_w4a16: 4-bit float weights, one e8m0 scale per group of 32
// along K. Element k of a row: nibble of byte k/2 (low nibble for even k).
double orc_mxfp4_at(const uint8_t* codes_row, const uint8_t* scales_row, int64_t k) {
  const uint8_t byte = codes_row[k >> 1];
  const int code = (k & 1) ? (byte >> 4) : (byte & 0xF);
  return orc_e2m1(code) * orc_e8m0(scales_row[k >> 5]);
}

// [P1] "normalized sqrt(softplus(logit)) routing"; [P5] scoring_func
// "sqrtsoftplus". softplus(z) = log(1 + e^z), evaluated in its stable form.
double orc_sqrt_softplus(double z) {
  const double sp = std::max(z, 0.0) + std::log1p(std::exp(-std::fabs(z)));
  return std::sqrt(sp);
}

// [P5] hidden_act "silu": silu(v) = v / (1 + e^-v).
double orc_silu(double v) { return v / (1.0 + std::exp(-v)); }

// [P4] "SwiGLU feed-forward": gate clamped from above only, up clamped on both
// sides at swiglu_limit ([P5] 10.0), then silu(gate) * up.
double orc_clamped_swiglu(double g, double u, double limit) {
  const double gc = std::min(g, limit);
  const double uc = std::min(std::max(u, -limit), limit);
  return orc_silu(gc) * uc;
}

// Router logits and scores for one token: z_e = sum_h x[h] * gate[e][h] (fp64),
// s_e = sqrt(softplus(z_e)).  [P4] "Mixture of experts" (scores over the
// gate), [P5] gate weights are not quantised ("*.gate.*" in ignore).
static void token_scores(const OrcLayer* L, int64_t t, std::vector<double>& s) {
  s.assign(size_t(L->E), 0.0);
  const uint16_t* xr = L->x + t * L->H;
  for (int e = 0; e < L->E; ++e) {
    const uint16_t* gr = L->gate + int64_t(e) * L->H;
    double z = 0.0;
    for (int h = 0; h < L->H; ++h) z += orc_bf16_to_double(xr[h]) * orc_bf16_to_double(gr[h]);
    s[size_t(e)] = orc_sqrt_softplus(z);
  }
}

// Routing of all T tokens.
//  Learned ([P4] "Auxiliary-loss-free load balancing": the bias enters only
//  the top-k selection, the weights come from the unbiased scores; [P5]
//  topk_method noaux_tc, num_experts_per_tok 6): ids = top-k of s + bias,
//  ties to the lower index, emitted in ascending id; margin = b_(k) - b_(k+1).
//  Hash ([P1] first three layers select experts from a token-id hash table;
//  [P3] item 2, ffn.gate.tid2eid): ids = tid2eid[token_id] in column order.
//  Weights ([P5] norm_topk_prob true, routed_scaling_factor 1.5):
//  w_j = scale * s_{ids_j} / sum_j s_{ids_j}.
// Returns 0, or 1 for an out-of-range token id / table entry.
int orc_route(const OrcLayer* L, int32_t* ids, double* w, double* margin, double* scores) {
  const int E = L->E, k = L->k;
  std::vector<double> s;
  std::vector<int> order(static_cast<size_t>(E));
  for (int64_t t = 0; t < L->T; ++t) {
    token_scores(L, t, s);
    if (scores)
      for (int e = 0; e < E; ++e) scores[t * E + e] = s[size_t(e)];
    int32_t* id = ids + t * k;
    if (L->bias) {
      std::vector<double> b(static_cast<size_t>(E));
      for (int e = 0; e < E; ++e) b[size_t(e)] = s[size_t(e)] + double(L->bias[e]);
      for (int e = 0; e < E; ++e) order[size_t(e)] = e;
      std::sort(order.begin(), order.end(), [&](int a, int c) {
        if (b[size_t(a)] != b[size_t(c)]) return b[size_t(a)] > b[size_t(c)];
        return a < c;
      });
      if (margin)
        margin[t] = (k < E) ? b[size_t(order[size_t(k - 1)])] - b[size_t(order[size_t(k)])]
                            : std::numeric_limits<double>::infinity();
      std::vector<int> sel(order.begin(), order.begin() + k);
      std::sort(sel.begin(), sel.end());
      for (int j = 0; j < k; ++j) id[j] = sel[size_t(j)];
    } else {
      const int32_t tok = L->token_ids[t];
      if (tok < 0 || tok >= L->vocab) return 1;
      for (int j = 0; j < k; ++j) {
        const int32_t e = L->tid2eid[int64_t(tok) * k + j];
        if (e < 0 || e >= E) return 1;
        id[j] = e;
      }
      if (margin) margin[t] = std::numeric_limits<double>::infinity();
    }
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += s[size_t(id[j])];
    for (int j = 0; j < k; ++j) w[t * k + j] = L->routed_scale * s[size_t(id[j])] / sum;
  }
  return 0;
}

// Token permutation by expert (the grouping behind "experts(flat, indices,
// weights)", [P4] "Shared expert" row): counts via a histogram, offsets as the
// exclusive prefix sum, sorted_slot lists slots s = t*k + j grouped by
// ascending expert and by ascending s within an expert, slot_pos its inverse.
// Returns 0, or 1 for an out-of-range expert id.
int orc_permute(int32_t T, int32_t k, int32_t E, const int32_t* ids, int32_t* counts, int32_t* offsets,
                int32_t* sorted_slot, int32_t* slot_pos) {
  const int64_t S = int64_t(T) * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < S; ++s) {
    if (ids[s] < 0 || ids[s] >= E) return 1;
    counts[ids[s]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> cursor(offsets, offsets + E);
  for (int64_t s = 0; s < S; ++s) {
    const int32_t pos = cursor[size_t(ids[s])]++;
    sorted_slot[pos] = int32_t(s);
    slot_pos[s] = pos;
  }
  return 0;
}

// One routed expert e applied to one token row x (fp64), following [P4]
// "SwiGLU feed-forward" and [P5] experts_w4a16: [g; u] = W13_e x with exact
// MXFP4 dequantisation, h = swiglu(g, u), y = W2_e h. h_out may be null.
static void routed_expert(const OrcLayer* L, int e, const double* x, double* y, double* h_out) {
  const int H = L->H, I = L->I;
  const int64_t rows13 = 2 * int64_t(I);
  std::vector<double> h(static_cast<size_t>(I));
  for (int n = 0; n < I; ++n) {
    const int64_t rg = int64_t(e) * rows13 + n, ru = int64_t(e) * rows13 + I + n;
    const uint8_t* cg = L->w13_codes + rg * (H / 2);
    const uint8_t* sg = L->w13_scales + rg * (H / 32);
    const uint8_t* cu = L->w13_codes + ru * (H / 2);
    const uint8_t* su = L->w13_scales + ru * (H / 32);
    double g = 0.0, u = 0.0;
    for (int64_t kk = 0; kk < H; ++kk) {
      g += x[kk] * orc_mxfp4_at(cg, sg, kk);
      u += x[kk] * orc_mxfp4_at(cu, su, kk);
    }
    h[size_t(n)] = orc_clamped_swiglu(g, u, L->swiglu_limit);
  }
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * size_t(I));
  for (int m = 0; m < H; ++m) {
    const int64_t r = int64_t(e) * H + m;
    const uint8_t* c = L->w2_codes + r * (I / 2);
    const uint8_t* sc = L->w2_scales + r * (I / 32);
    double acc = 0.0;
    for (int64_t n = 0; n < I; ++n) acc += h[size_t(n)] * orc_mxfp4_at(c, sc, n);
    y[m] = acc;
  }
}

// The shared expert on one token ([P4] "Shared expert": added unconditionally;
// [P5] linears_w8a16: int8 symmetric per output channel), dequantised as
// q * scale[row].
static void shared_expert(const OrcLayer* L, const double* x, double* y, double* h_out) {
  const int H = L->H, Is = L->Is;
  std::vector<double> h(static_cast<size_t>(Is));
  for (int n = 0; n < Is; ++n) {
    const int8_t* qg = L->sh13 + int64_t(n) * H;
    const int8_t* qu = L->sh13 + int64_t(Is + n) * H;
    const double sg = L->sh13_scale[n], su = L->sh13_scale[Is + n];
    double g = 0.0, u = 0.0;
    for (int kk = 0; kk < H; ++kk) {
      g += x[kk] * (double(qg[kk]) * sg);
      u += x[kk] * (double(qu[kk]) * su);
    }
    h[size_t(n)] = orc_clamped_swiglu(g, u, L->swiglu_limit);
  }
  if (h_out) std::memcpy(h_out, h.data(), sizeof(double) * size_t(Is));
  for (int m = 0; m < H; ++m) {
    const int8_t* q = L->sh2 + int64_t(m) * Is;
    const double sc = L->sh2_scale[m];
    double acc = 0.0;
    for (int n = 0; n < Is; ++n) acc += h[size_t(n)] * (double(q[n]) * sc);
    y[m] = acc;
  }
}

// Layer output for a list of tokens ([P4] "Shared expert" row: the block
// returns routed + shared_experts(residual)):
//   out[t] = sum_j w[t, j] * expert_{ids[t, j]}(x[t]) + shared(x[t]).
// ids/w are [T, k] for all T tokens (any routing); tok lists which tokens to
// evaluate; out is [n, H]. h_dbg (optional) receives [n, k, I] routed
// intermediates, hs_dbg (optional) [n, Is] shared intermediates.
int orc_moe_tokens(const OrcLayer* L, int32_t n, const int32_t* tok, const int32_t* ids, const double* w,
                   double* out, double* h_dbg, double* hs_dbg) {
  const int H = L->H, k = L->k;
  std::vector<double> x(static_cast<size_t>(H)), y(static_cast<size_t>(H));
  for (int32_t i = 0; i < n; ++i) {
    const int64_t t = tok[i];
    if (t < 0 || t >= L->T) return 1;
    for (int h = 0; h < H; ++h) x[size_t(h)] = orc_bf16_to_double(L->x[t * H + h]);
    double* o = out + int64_t(i) * H;
    for (int m = 0; m < H; ++m) o[m] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e < 0 || e >= L->E) return 1;
      routed_expert(L, e, x.data(), y.data(), h_dbg ? h_dbg + (int64_t(i) * k + j) * L->I : nullptr);
      const double wj = w[t * k + j];
      for (int m = 0; m < H; ++m) o[m] += wj * y[size_t(m)];
    }
    if (L->Is > 0 && L->sh13) {
      shared_expert(L, x.data(), y.data(), hs_dbg ? hs_dbg + int64_t(i) * L->Is : nullptr);
      for (int m = 0; m < H; ++m) o[m] += y[size_t(m)];
    }
  }
  return 0;
}

// Brute-force dense evaluation for tiny shapes: dequantise every weight tensor
// up front, run every expert on every token, and combine with the dense [T, E]
// weight matrix that scatters w onto ids (zeros elsewhere). Written as a
// separate code path so it can pin orc_moe_tokens.
int orc_moe_dense(const OrcLayer* L, const int32_t* ids, const double* w, double* out) {
  const int T = L->T, H = L->H, E = L->E, I = L->I, k = L->k, Is = L->Is;
  std::vector<double> W13(size_t(E) * 2 * I * H), W2(size_t(E) * H * I);
  for (int64_t r = 0; r < int64_t(E) * 2 * I; ++r)
    for (int kk = 0; kk < H; ++kk) {
      const uint8_t byte = L->w13_codes[r * (H / 2) + kk / 2];
      const int code = (kk % 2 == 0) ? (byte & 15) : (byte >> 4);
      W13[size_t(r * H + kk)] = orc_e2m1(code) * orc_e8m0(L->w13_scales[r * (H / 32) + kk / 32]);
    }
  for (int64_t r = 0; r < int64_t(E) * H; ++r)
    for (int n = 0; n < I; ++n) {
      const uint8_t byte = L->w2_codes[r * (I / 2) + n / 2];
      const int code = (n % 2 == 0) ? (byte & 15) : (byte >> 4);
      W2[size_t(r * I + n)] = orc_e2m1(code) * orc_e8m0(L->w2_scales[r * (I / 32) + n / 32]);
    }
  std::vector<double> dense(size_t(T) * E, 0.0);
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      if (e < 0 || e >= E) return 1;
      dense[size_t(t) * E + e] += w[t * k + j];
    }
  std::vector<double> x(static_cast<size_t>(H)), gu(size_t(2) * I), hh(static_cast<size_t>(I));
  for (int t = 0; t < T; ++t) {
    for (int h = 0; h < H; ++h) x[size_t(h)] = orc_bf16_to_double(L->x[int64_t(t) * H + h]);
    double* o = out + int64_t(t) * H;
    for (int m = 0; m < H; ++m) o[m] = 0.0;
    for (int e = 0; e < E; ++e) {
      for (int r = 0; r < 2 * I; ++r) {
        double acc = 0.0;
        const double* wr = &W13[(size_t(e) * 2 * I + r) * H];
        for (int h = 0; h < H; ++h) acc += wr[h] * x[size_t(h)];
        gu[size_t(r)] = acc;
      }
      for (int n = 0; n < I; ++n) hh[size_t(n)] = orc_clamped_swiglu(gu[size_t(n)], gu[size_t(I + n)], L->swiglu_limit);
      const double de = dense[size_t(t) * E + e];
      for (int m = 0; m < H; ++m) {
        double acc = 0.0;
        const double* wr = &W2[(size_t(e) * H + m) * I];
        for (int n = 0; n < I; ++n) acc += wr[n] * hh[size_t(n)];
        o[m] += de * acc;
      }
    }
    if (Is > 0 && L->sh13) {
      std::vector<double> hs(static_cast<size_t>(Is));
      for (int n = 0; n < Is; ++n) {
        double g = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
          g += double(L->sh13[int64_t(n) * H + h]) * double(L->sh13_scale[n]) * x[size_t(h)];
          u += double(L->sh13[int64_t(Is + n) * H + h]) * double(L->sh13_scale[Is + n]) * x[size_t(h)];
        }
        hs[size_t(n)] = orc_clamped_swiglu(g, u, L->swiglu_limit);
      }
      for (int m = 0; m < H; ++m) {
        double acc = 0.0;
        for (int n = 0; n < Is; ++n) acc += double(L->sh2[int64_t(m) * Is + n]) * double(L->sh2_scale[m]) * hs[size_t(n)];
        o[m] += acc;
      }
    }
  }
  return 0;
}

// [P5] quantization_config, group linears_w8a16 (weights: 8-bit int,
// symmetric, strategy channel; input activations: 16-bit float; targets the
// attention projections and the shared expert's two projections): the
// dequantised weight is q[n, k] * scale[n], and the linear is
//   out[t, n] = sum_k x[t, k] * q[n, k] * scale[n]     (fp64, bf16 x exact).
void orc_linear_w8a16(int32_t T, int32_t N, int32_t K, const uint16_t* x, const int8_t* q, const float* scale,
                      double* out) {
  for (int t = 0; t < T; ++t)
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k)
        acc += orc_bf16_to_double(x[int64_t(t) * K + k]) * (double(q[int64_t(n) * K + k]) * double(scale[n]));
      out[int64_t(t) * N + n] = acc;
    }
}

}  // extern "C"

// Reference oracle for the routed Mixture-of-Experts FFN at decode time.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product library links, includes or
// calls this file; only the tests, the smoke check and the benchmark's CPU
// baseline leg load it. It shares no code, header or table with the CUDA path.
//
// It is a plain, slow, obviously-correct restatement of what the layer
// computes, written from these pages:
//   * "Pacotes de Swiftlet 80B Qwen no Mac ..." (xix.ai), paragraph 4: every
//     layer routes each token to 8 of 256 experts (35B) or 10 of 512 (80B);
//     routers and shared experts stay resident.
//   * same article, paragraph 8: MLX-style int4/int8 group quantization and a
//     sparse MoE with shared experts.
//   * Runnel README, introduction and "Streaming CLI": the routed experts'
//     gate and up projections are stored and run as one packed matrix;
//     "Target": 256 routed experts, top-8, plus one shared expert.
// The pages print no formula, layout or worked example for the layer. Where
// they are silent this file takes the plain reading and says so beside the
// step:
//   dequantisation   w = float(scale) * float(q) + float(bias), per group of
//                    `group` consecutive elements along K (the input
//                    dimension), computed in fp32 as two roundings (no FMA);
//   4-bit packing    two codes per byte along K, the low nibble holding the
//                    even element;
//   packed gate/up   rows [0, I) are the gate projection, rows [I, 2I) up;
//   routing          softmax over all E logits, the k largest, weights
//                    renormalised over the k (optional per-expert logit bias
//                    added before the softmax); ties go to the lower index;
//   expert           o = W_down (silu(W_gate x) * (W_up x)), silu(z) = z/(1+e^-z);
//   shared expert    same form, weighted by sigmoid(x . w_sg), not renormalised;
//   combine          y = sum_j w_j o_j + sigmoid(x . w_sg) o_shared, summed in
//                    rank order, shared last, in double, then fp32, then bf16
//                    (round to nearest even);
//   stacking         r <- r + y; x <- bf16(r / sqrt(mean(r^2) + eps)) (a
//                    parameter-free pre-norm residual stream; harness glue,
//                    not described by the pages).
// Accumulation is in double throughout; the intermediate h is stored as fp32.
// Build with -ffp-contract=off so no multiply-add is fused.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

float bf16_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round-to-nearest-even from fp32 to bf16, NaN kept quiet.
uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0) {
    return static_cast<uint16_t>((u >> 16) | 0x0040u);
  }
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

// Code of element k of one row: 8-bit is one byte per element; 4-bit holds
// two elements per byte, the even element in the low nibble.
int code_at(const uint8_t* row, int64_t k, int bits) {
  if (bits == 8) return row[k];
  uint8_t byte = row[k / 2];
  return (k % 2 == 0) ? (byte & 0x0f) : (byte >> 4);
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

double sigmoid(double z) { return 1.0 / (1.0 + std::exp(-z)); }

}  // namespace

extern "C" {

// One quantised matrix [rows][K] on the host: codes row-major with
// K*bits/8 bytes per row, bf16 scales and biases [rows][K/group].
struct orc_qmat {
  const uint8_t* q;
  const uint16_t* scales;
  const uint16_t* biases;
  int64_t rows;
  int64_t K;
};

float orc_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16(f); }

// Dequantise a whole matrix into fp32 [rows][K].
int orc_dequant(const orc_qmat* m, int bits, int group, float* out) {
  if (!m || !out || (bits != 4 && bits != 8) || group <= 0 || m->K % group != 0) return 1;
  const int64_t row_bytes = m->K * bits / 8;
  const int64_t ngroups = m->K / group;
  for (int64_t r = 0; r < m->rows; ++r) {
    const uint8_t* row = m->q + r * row_bytes;
    for (int64_t k = 0; k < m->K; ++k) {
      const int64_t g = k / group;
      const float s = bf16_to_f32(m->scales[r * ngroups + g]);
      const float b = bf16_to_f32(m->biases[r * ngroups + g]);
      const float q = static_cast<float>(code_at(row, k, bits));
      const float sq = s * q;      // first fp32 rounding
      out[r * m->K + k] = sq + b;  // second fp32 rounding
    }
  }
  return 0;
}

// Router logits for T tokens: logits[t][e] = sum_h x[t][h] * Wr[e][h] (+ bias[e]).
int orc_router_logits(const uint16_t* x, int64_t T, int64_t H, const uint16_t* wr, int64_t E,
                      const float* rbias, double* logits) {
  if (!x || !wr || !logits) return 1;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int64_t h = 0; h < H; ++h) {
        acc += static_cast<double>(bf16_to_f32(x[t * H + h])) *
               static_cast<double>(bf16_to_f32(wr[e * H + h]));
      }
      if (rbias) acc += static_cast<double>(rbias[e]);
      logits[t * E + e] = acc;
    }
  }
  return 0;
}

// Softmax over all E logits of one token, then the k most probable experts
// by a full stable sort (probability descending, index ascending), then the
// weights renormalised over those k (or left as softmax probabilities when
// renorm == 0). idx and w come out in descending-weight order.
int orc_softmax_topk(const double* logits, int64_t E, int64_t k, int renorm, int32_t* idx,
                     double* w) {
  if (!logits || !idx || !w || k < 1 || k > E) return 1;
  double mx = logits[0];
  for (int64_t e = 1; e < E; ++e) mx = std::max(mx, logits[e]);
  std::vector<double> p(E);
  double z = 0.0;
  for (int64_t e = 0; e < E; ++e) {
    p[e] = std::exp(logits[e] - mx);
    z += p[e];
  }
  for (int64_t e = 0; e < E; ++e) p[e] /= z;
  std::vector<int32_t> order(E);
  for (int64_t e = 0; e < E; ++e) order[e] = static_cast<int32_t>(e);
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
    if (p[a] != p[b]) return p[a] > p[b];
    return a < b;
  });
  double sel = 0.0;
  for (int64_t j = 0; j < k; ++j) sel += p[order[j]];
  for (int64_t j = 0; j < k; ++j) {
    idx[j] = order[j];
    w[j] = renorm ? p[order[j]] / sel : p[order[j]];
  }
  return 0;
}

// Sigmoid gate of the shared expert for one token: 1 / (1 + exp(-x . w_sg)).
double orc_shared_gate(const uint16_t* x, const uint16_t* wsg, int64_t H) {
  double acc = 0.0;
  for (int64_t h = 0; h < H; ++h) {
    acc += static_cast<double>(bf16_to_f32(x[h])) * static_cast<double>(bf16_to_f32(wsg[h]));
  }
  return sigmoid(acc);
}

// One expert on one token from dequantised matrices:
//   gu = Wgu x (Wgu is [2I][H], gate rows first), h_i = fp32(silu(gu_i) * gu_{I+i}),
//   o = Wd h (Wd is [H][I]).
int orc_expert_ffn(const float* wgu, const float* wd, int64_t H, int64_t I, const double* x,
                   double* o, float* h_out) {
  if (!wgu || !wd || !x || !o) return 1;
  std::vector<double> gu(2 * I);
  for (int64_t r = 0; r < 2 * I; ++r) {
    double acc = 0.0;
    for (int64_t c = 0; c < H; ++c) acc += static_cast<double>(wgu[r * H + c]) * x[c];
    gu[r] = acc;
  }
  std::vector<float> h(I);
  for (int64_t i = 0; i < I; ++i) h[i] = static_cast<float>(silu(gu[i]) * gu[I + i]);
  if (h_out) std::memcpy(h_out, h.data(), sizeof(float) * I);
  for (int64_t r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i) acc += static_cast<double>(wd[r * I + i]) * h[i];
    o[r] = acc;
  }
  return 0;
}

// The routed experts plus the shared expert for one token, from the packed
// bytes of the nsel selected experts:
//   y = sum_j w[j] * E_j(x) + gate * S(x)        (in double, rank order, shared last)
// sh_gate_up / sh_down may be null (no shared expert). y_f64 gets the sum;
// y_f32 and y_bf16 (optional) its fp32 and bf16 roundings. `threads` splits
// the selected experts over std::threads (each expert's arithmetic unchanged).
int orc_moe_token(int64_t H, int64_t I, int64_t Is, int bits, int group, const uint16_t* x,
                  int64_t nsel, const orc_qmat* gate_up, const orc_qmat* down, const double* w,
                  const orc_qmat* sh_gate_up, const orc_qmat* sh_down, double gate, double* y_f64,
                  float* y_f32, uint16_t* y_bf16, int threads) {
  if (!x || !y_f64 || (nsel > 0 && (!gate_up || !down || !w))) return 1;
  std::vector<double> xd(H);
  for (int64_t h = 0; h < H; ++h) xd[h] = bf16_to_f32(x[h]);
  const bool has_shared = sh_gate_up && sh_down && Is > 0;
  const int64_t nexp = nsel + (has_shared ? 1 : 0);
  std::vector<std::vector<double>> outs(nexp, std::vector<double>(H));
  std::vector<int> rc(nexp, 0);
  auto run = [&](int64_t j) {
    const orc_qmat* gu = (j < nsel) ? &gate_up[j] : sh_gate_up;
    const orc_qmat* dn = (j < nsel) ? &down[j] : sh_down;
    const int64_t ii = (j < nsel) ? I : Is;
    if (gu->rows != 2 * ii || gu->K != H || dn->rows != H || dn->K != ii) {
      rc[j] = 1;
      return;
    }
    std::vector<float> wgu(2 * ii * H), wd(H * ii);
    rc[j] |= orc_dequant(gu, bits, group, wgu.data());
    rc[j] |= orc_dequant(dn, bits, group, wd.data());
    if (rc[j] == 0) rc[j] = orc_expert_ffn(wgu.data(), wd.data(), H, ii, xd.data(), outs[j].data(), nullptr);
  };
  if (threads <= 1) {
    for (int64_t j = 0; j < nexp; ++j) run(j);
  } else {
    std::vector<std::thread> pool;
    for (int tid = 0; tid < threads; ++tid) {
      pool.emplace_back([&, tid]() {
        for (int64_t j = tid; j < nexp; j += threads) run(j);
      });
    }
    for (auto& th : pool) th.join();
  }
  for (int64_t j = 0; j < nexp; ++j)
    if (rc[j]) return rc[j];
  for (int64_t r = 0; r < H; ++r) {
    double acc = 0.0;
    for (int64_t j = 0; j < nsel; ++j) acc += w[j] * outs[j][r];
    if (has_shared) acc += gate * outs[nsel][r];
    y_f64[r] = acc;
    const float f = static_cast<float>(acc);
    if (y_f32) y_f32[r] = f;
    if (y_bf16) y_bf16[r] = f32_to_bf16(f);
  }
  return 0;
}

// Groups the T*k (token, slot) pairs by expert, in a stable order: within an
// expert, pairs keep ascending (token, slot) order. With with_shared != 0 the
// shared expert is a pseudo-expert E taken by every token (slot k). perm
// receives the flat pair ids (t*k + slot, or T*k + t for the shared pairs),
// offsets[e] the first position of expert e (offsets[E(+1)] = pair count).
int orc_sort_by_expert(const int32_t* idx, int64_t T, int64_t k, int64_t E, int with_shared,
                       int32_t* perm, int32_t* offsets) {
  if (!idx || !perm || !offsets) return 1;
  struct pair_t {
    int64_t expert, token, slot, id;
  };
  std::vector<pair_t> pairs;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      const int64_t e = idx[t * k + j];
      if (e < 0 || e >= E) return 2;
      pairs.push_back({e, t, j, t * k + j});
    }
  }
  if (with_shared) {
    for (int64_t t = 0; t < T; ++t) pairs.push_back({E, t, k, T * k + t});
  }
  std::stable_sort(pairs.begin(), pairs.end(), [](const pair_t& a, const pair_t& b) {
    if (a.expert != b.expert) return a.expert < b.expert;
    if (a.token != b.token) return a.token < b.token;
    return a.slot < b.slot;
  });
  const int64_t nbins = E + (with_shared ? 1 : 0);
  for (size_t p = 0; p < pairs.size(); ++p) perm[p] = static_cast<int32_t>(pairs[p].id);
  for (int64_t e = 0; e <= nbins; ++e) {
    int64_t first = 0;
    while (first < static_cast<int64_t>(pairs.size()) && pairs[first].expert < e) ++first;
    offsets[e] = static_cast<int32_t>(first);
  }
  return 0;
}

// Residual plus parameter-free RMSNorm between stacked layers, per token:
//   r' = r + y ; x' = bf16(r' / sqrt(mean(r'^2) + eps)).
// r is carried in double here.
int orc_residual_rmsnorm(const double* r, const uint16_t* y, int64_t T, int64_t H, double eps,
                         double* r_out, uint16_t* x_out) {
  if (!r || !y || !r_out || !x_out) return 1;
  for (int64_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int64_t h = 0; h < H; ++h) {
      const double v = r[t * H + h] + static_cast<double>(bf16_to_f32(y[t * H + h]));
      r_out[t * H + h] = v;
      ss += v * v;
    }
    const double inv = 1.0 / std::sqrt(ss / static_cast<double>(H) + eps);
    for (int64_t h = 0; h < H; ++h) {
      x_out[t * H + h] = f32_to_bf16(static_cast<float>(r_out[t * H + h] * inv));
    }
  }
  return 0;
}

}  // extern "C"

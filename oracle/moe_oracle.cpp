// FP64 CPU oracle of the forward pass of one fine-grained-FP8 MoE layer,
// written as plain loops.
//
// TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
// CPU-baseline legs may load this library. It shares no code with the CUDA
// library (no kernels, headers, helpers, tables or constant generators); the
// two meet only in the seeded inputs of gen/.
//
// The layer (transformers docs page "Dots 3 Note Preview",
// Dots3NoteTextConfig; model card dots-studio/dots3-note-prev, "Model
// Overview"): hidden H, E routed SwiGLU experts plus S (0 or 1) shared
// experts, top-K routing, expert FFN width F, no biases. Weights are a
// fine-grained FP8 checkpoint (transformers PR #47844, "What does this PR
// do?"): E4M3 codes with one fp32 scale per 128 x 128 block; activations are
// quantised at run time per token per 128 channels.
//
// Readings where the pages are silent (the same as the numpy oracle's):
//   route    logits in FP64; p = softmax over the E experts; selection score
//            s = p + bias (bias 0 unless given); with n_group > 1 the experts
//            form n_group contiguous groups scored by their best member and
//            only the topk_group best groups (ties to the lower group) are
//            eligible; the K best eligible experts by s, ties to the lower
//            id, listed in ascending id; weights = the selected p,
//            renormalised to sum 1 when norm_topk, times routed_scaling. The
//            near-tie gap is s_(K) - s_(K+1) (and the group-score gap).
//   permute  counting sort of the (token, slot) pairs by expert in token
//            order; group E (shared) holds one row per token, in token order.
//   quantise per row, per 128 channels: s = fp32(amax) / 448 in fp32,
//            q = E4M3(fp32(v) / s) in fp32, round to nearest even,
//            saturating; an all-zero group has s = 0 and q = 0.
//   expert   G = A Wg^T, U = A Wu^T on the dequantised operands (FP64),
//            h = silu(G) U, h rounded to fp32 and quantised like the
//            activations, y = dequant(h) Wd^T (FP64).
//   combine  out[t] = sum_k w[t,k] y[row(t,k)] + y[shared row of t] (FP64).
// E4M3 is the OCP "FN" flavour: 1 sign, 4 exponent (bias 7), 3 mantissa
// bits, no infinities, S.1111.111 = NaN, largest finite 448.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr int kGroup = 128;

// ------------------------------------------------------------------ E4M3

// Value of one E4M3 code from the format's definition.
double e4m3_value(int code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  const int e = (code >> 3) & 0xF;
  const int m = code & 0x7;
  if (e == 0xF && m == 0x7) return std::numeric_limits<double>::quiet_NaN();
  if (e == 0) return sign * (m / 8.0) * std::ldexp(1.0, -6);         // subnormal
  return sign * (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
}

struct Table {
  double v[256];
  Table() {
    for (int c = 0; c < 256; ++c) v[c] = e4m3_value(c);
  }
};
const Table& table() {
  static const Table t;
  return t;
}

// Nearest finite E4M3 value to v (codes 0..126 are the non-negative finite
// values in increasing order), ties to the even code, |v| >= 448 -> 448.
// The sign of v (zero included) goes to the sign bit.
uint8_t e4m3_encode(float v) {
  const double* tab = table().v;
  const double a = std::fabs(double(v));
  int code;
  if (a >= 448.0) {
    code = 126;
  } else {
    int hi = 0;
    while (tab[hi] < a) ++hi;                  // first code whose value is >= a
    if (tab[hi] == a || hi == 0) {
      code = hi;
    } else {
      const int lo = hi - 1;
      const double dlo = a - tab[lo], dhi = tab[hi] - a;
      if (dhi < dlo) code = hi;
      else if (dlo < dhi) code = lo;
      else code = (hi % 2 == 0) ? hi : lo;   // tie: the even code
    }
  }
  return uint8_t(code | (std::signbit(v) ? 0x80 : 0));
}

// ------------------------------------------------------------------ numbers

double bf16_bits_to_double(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

// v -> fp32 (round to nearest even, the C++ conversion) -> bf16 (round to
// nearest even on the fp32 bit pattern) -> double.
double round_bf16(double v) {
  const float f = float(v);
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  u = ((u + 0x7FFFu + lsb) >> 16) << 16;
  float r;
  std::memcpy(&r, &u, 4);
  return double(r);
}

double silu(double g) { return g / (1.0 + std::exp(-g)); }

// One row of C channels, quantised per 128-channel group.
void quantize_row(const float* v, int C, uint8_t* codes, float* scales) {
  for (int g = 0; g * kGroup < C; ++g) {
    const int c0 = g * kGroup, c1 = std::min(C, c0 + kGroup);
    float amax = 0.0f;
    for (int c = c0; c < c1; ++c) amax = std::max(amax, std::fabs(v[c]));
    const float s = amax / 448.0f;
    scales[g] = s;
    for (int c = c0; c < c1; ++c) codes[c] = amax > 0.0f ? e4m3_encode(v[c] / s) : uint8_t(0);
  }
}

// ------------------------------------------------------------------ threads

int worker_count() {
  const unsigned n = std::thread::hardware_concurrency();
  return n == 0 ? 1 : int(n);
}

// Runs body(i) for i in [0, n) on all cores; items are taken in order from a
// shared counter.
template <typename F>
void parallel_for(int n, F body) {
  const int nw = std::min(n, worker_count());
  if (nw <= 1) {
    for (int i = 0; i < n; ++i) body(i);
    return;
  }
  std::atomic<int> next(0);
  std::vector<std::thread> pool;
  for (int w = 0; w < nw; ++w)
    pool.emplace_back([&]() {
      for (int i = next++; i < n; i = next++) body(i);
    });
  for (auto& t : pool) t.join();
}

}  // namespace

// ------------------------------------------------------------------ C API

extern "C" {

// The layer's weights, laid out like the checkpoint (expert index E is the
// shared expert when S = 1):
//   w_gate, w_up [E+S][F][H] codes, s_gate, s_up [E+S][FB][HB]
//   w_down [E+S][H][ld_f] codes, s_down [E+S][HB][FB]
// with FB = ceil(F/128), HB = ceil(H/128).
struct oracle_layer {
  int H, E, S, K, F, ld_f;
  const uint8_t* w_gate;
  const float* s_gate;
  const uint8_t* w_up;
  const float* s_up;
  const uint8_t* w_down;
  const float* s_down;
};

int oracle_threads() { return worker_count(); }

void oracle_e4m3_table(double* out) {
  for (int c = 0; c < 256; ++c) out[c] = table().v[c];
}

void oracle_e4m3_encode(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(v[i]);
}

void oracle_round_bf16(const double* v, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(v[i]);
}

void oracle_silu(const double* g, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(g[i]);
}

// codes [rows][C], scales [rows][ceil(C/128)]
void oracle_quantize_rows(const float* v, int64_t rows, int C, uint8_t* codes, float* scales) {
  const int ng = (C + kGroup - 1) / kGroup;
  for (int64_t r = 0; r < rows; ++r) quantize_row(v + r * C, C, codes + r * C, scales + r * ng);
}

// out[r][c] = decode(codes[r][c]) * scales[r][c / 128]; codes have row stride ldc
void oracle_dequant_rows(const uint8_t* codes, int64_t ldc, const float* scales, int64_t rows, int C, double* out) {
  const int ng = (C + kGroup - 1) / kGroup;
  for (int64_t r = 0; r < rows; ++r)
    for (int c = 0; c < C; ++c) out[r * C + c] = table().v[codes[r * ldc + c]] * double(scales[r * ng + c / kGroup]);
}

// out[n][k] = decode(codes[n][k]) * scales[n / 128][k / 128]; codes row stride ldc
void oracle_dequant_block(const uint8_t* codes, int64_t ldc, const float* scales, int rows, int cols, double* out) {
  const int cb = (cols + kGroup - 1) / kGroup;
  for (int n = 0; n < rows; ++n)
    for (int k = 0; k < cols; ++k)
      out[int64_t(n) * cols + k] =
          table().v[codes[int64_t(n) * ldc + k]] * double(scales[(n / kGroup) * cb + k / kGroup]);
}

// logits[t][e] = sum_h x[t][h] * router_w[e][h] (x as bf16 bit patterns)
void oracle_router_logits(const uint16_t* x, int T, int H, const float* router_w, int E, double* logits) {
  parallel_for(T, [&](int t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h) acc += bf16_bits_to_double(x[int64_t(t) * H + h]) * double(router_w[int64_t(e) * H + h]);
      logits[int64_t(t) * E + e] = acc;
    }
  });
}

// p[t][e] = exp(l[t][e] - max_e l[t]) / sum_e exp(l[t][e] - max_e l[t])
void oracle_softmax(const double* logits, int T, int E, double* probs) {
  for (int t = 0; t < T; ++t) {
    const double* l = logits + int64_t(t) * E;
    double m = l[0];
    for (int e = 1; e < E; ++e) m = std::max(m, l[e]);
    double sum = 0.0;
    for (int e = 0; e < E; ++e) sum += std::exp(l[e] - m);
    for (int e = 0; e < E; ++e) probs[int64_t(t) * E + e] = std::exp(l[e] - m) / sum;
  }
}

// Selection (see the header comment): idx [T][K], w [T][K], gap [T].
void oracle_select_topk(const double* probs, int T, int E, int K, double routed_scaling, int n_group, int topk_group,
                        const double* bias, int norm_topk, int32_t* idx, double* w, double* gap) {
  const int gsize = E / n_group;
  for (int t = 0; t < T; ++t) {
    const double* p = probs + int64_t(t) * E;
    std::vector<double> s(E);
    for (int e = 0; e < E; ++e) s[e] = p[e] + (bias ? bias[e] : 0.0);
    double group_gap = std::numeric_limits<double>::infinity();
    std::vector<int> cand;
    if (n_group > 1) {
      std::vector<double> gscore(n_group, -std::numeric_limits<double>::infinity());
      for (int e = 0; e < E; ++e) gscore[e / gsize] = std::max(gscore[e / gsize], s[e]);
      std::vector<int> gorder(n_group);
      for (int g = 0; g < n_group; ++g) gorder[g] = g;
      std::stable_sort(gorder.begin(), gorder.end(), [&](int a, int b) { return gscore[a] > gscore[b]; });
      if (topk_group < n_group) group_gap = gscore[gorder[topk_group - 1]] - gscore[gorder[topk_group]];
      std::vector<char> keep(n_group, 0);
      for (int i = 0; i < topk_group; ++i) keep[gorder[i]] = 1;
      for (int e = 0; e < E; ++e)
        if (keep[e / gsize]) cand.push_back(e);
    } else {
      for (int e = 0; e < E; ++e) cand.push_back(e);
    }
    // cand is in ascending id, so a stable sort by score keeps ties in id order
    std::vector<int> order(cand);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return s[a] > s[b]; });
    std::vector<int> sel(order.begin(), order.begin() + K);
    std::sort(sel.begin(), sel.end());
    double psum = 0.0;
    for (int k = 0; k < K; ++k) psum += p[sel[k]];
    for (int k = 0; k < K; ++k) {
      idx[int64_t(t) * K + k] = sel[k];
      w[int64_t(t) * K + k] = (norm_topk ? p[sel[k]] / psum : p[sel[k]]) * routed_scaling;
    }
    const double expert_gap =
        K < int(order.size()) ? s[order[K - 1]] - s[order[K]] : std::numeric_limits<double>::infinity();
    gap[t] = std::min(expert_gap, group_gap);
  }
}

// offsets [E+2], perm [T*K + T*S], inv [T][K]
void oracle_permute(const int32_t* idx, int T, int K, int E, int S, int32_t* offsets, int32_t* perm, int32_t* inv) {
  std::vector<int64_t> count(E, 0);
  for (int64_t i = 0; i < int64_t(T) * K; ++i) count[idx[i]] += 1;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = int32_t(offsets[e] + count[e]);
  offsets[E + 1] = offsets[E] + T * S;
  std::vector<int64_t> cursor(offsets, offsets + E);
  for (int t = 0; t < T; ++t)
    for (int k = 0; k < K; ++k) {
      const int e = idx[int64_t(t) * K + k];
      const int64_t row = cursor[e]++;
      perm[row] = t;
      inv[int64_t(t) * K + k] = int32_t(row);
    }
  for (int t = 0; t < T * S; ++t) perm[int64_t(T) * K + t] = t;
}

// h = silu(a Wg^T) * (a Wu^T) for one dequantised row a [H] of group g -> h [F]
static void gate_up_row(const oracle_layer* L, int g, const double* a, double* h) {
  const int H = L->H, F = L->F, HB = (H + kGroup - 1) / kGroup, FB = (F + kGroup - 1) / kGroup;
  const double* tab = table().v;
  const uint8_t* wg = L->w_gate + int64_t(g) * F * H;
  const uint8_t* wu = L->w_up + int64_t(g) * F * H;
  const float* sg = L->s_gate + int64_t(g) * FB * HB;
  const float* su = L->s_up + int64_t(g) * FB * HB;
  for (int n = 0; n < F; ++n) {
    double gs = 0.0, us = 0.0;
    for (int k = 0; k < H; ++k) {
      const int blk = (n / kGroup) * HB + k / kGroup;
      gs += a[k] * (tab[wg[int64_t(n) * H + k]] * double(sg[blk]));
      us += a[k] * (tab[wu[int64_t(n) * H + k]] * double(su[blk]));
    }
    h[n] = silu(gs) * us;
  }
}

// y = b Wd^T for one dequantised row b [F] of group g -> y [H]
static void down_row(const oracle_layer* L, int g, const double* b, double* y) {
  const int H = L->H, F = L->F, HB = (H + kGroup - 1) / kGroup, FB = (F + kGroup - 1) / kGroup;
  const double* tab = table().v;
  const uint8_t* wd = L->w_down + int64_t(g) * H * L->ld_f;
  const float* sd = L->s_down + int64_t(g) * HB * FB;
  for (int m = 0; m < H; ++m) {
    double acc = 0.0;
    for (int n = 0; n < F; ++n) acc += b[n] * (tab[wd[int64_t(m) * L->ld_f + n]] * double(sd[(m / kGroup) * FB + n / kGroup]));
    y[m] = acc;
  }
}

// Work items: rows of the selected groups in chunks, so that one busy group
// spreads over all cores.
struct RowChunk {
  int g;
  int64_t r0, r1;
};
static std::vector<RowChunk> chunks(const int32_t* offsets, const int32_t* groups, int ngroups) {
  std::vector<RowChunk> out;
  for (int i = 0; i < ngroups; ++i) {
    const int g = groups[i];
    for (int64_t r = offsets[g]; r < offsets[g + 1]; r += 8) out.push_back({g, r, std::min<int64_t>(offsets[g + 1], r + 8)});
  }
  return out;
}

// Grouped expert FFN over permuted rows (only the listed groups' rows are
// written): xq [rows][H] codes, xs [rows][HB]; h [rows][F] (FP64 SwiGLU
// output), hq [rows][F] and hs [rows][FB] (its quantisation), y [rows][H].
void oracle_expert_ffn_rows(const oracle_layer* L, const uint8_t* xq, const float* xs, const int32_t* offsets,
                            const int32_t* groups, int ngroups, double* h, uint8_t* hq, float* hs, double* y) {
  const int H = L->H, F = L->F, HB = (H + kGroup - 1) / kGroup, FB = (F + kGroup - 1) / kGroup;
  const std::vector<RowChunk> work = chunks(offsets, groups, ngroups);
  parallel_for(int(work.size()), [&](int i) {
    const RowChunk c = work[i];
    std::vector<double> a(H), b(F);
    std::vector<float> h32(F);
    for (int64_t r = c.r0; r < c.r1; ++r) {
      oracle_dequant_rows(xq + r * H, H, xs + r * HB, 1, H, a.data());
      gate_up_row(L, c.g, a.data(), h + r * F);
      for (int n = 0; n < F; ++n) h32[n] = float(h[r * F + n]);
      quantize_row(h32.data(), F, hq + r * F, hs + r * FB);
      oracle_dequant_rows(hq + r * F, F, hs + r * FB, 1, F, b.data());
      down_row(L, c.g, b.data(), y + r * H);
    }
  });
}

// The down projection alone: hq [rows][F], hs [rows][FB] -> y [rows][H].
void oracle_expert_down_rows(const oracle_layer* L, const uint8_t* hq, const float* hs, const int32_t* offsets,
                             const int32_t* groups, int ngroups, double* y) {
  const int H = L->H, F = L->F, FB = (F + kGroup - 1) / kGroup;
  const std::vector<RowChunk> work = chunks(offsets, groups, ngroups);
  parallel_for(int(work.size()), [&](int i) {
    const RowChunk c = work[i];
    std::vector<double> b(F);
    for (int64_t r = c.r0; r < c.r1; ++r) {
      oracle_dequant_rows(hq + r * F, F, hs + r * FB, 1, F, b.data());
      down_row(L, c.g, b.data(), y + r * H);
    }
  });
}

// out [T][H] = sum_k w[t][k] y[inv[t][k]] (+ y[T*K + t] when S = 1)
void oracle_combine(const double* y, int H, const int32_t* inv, const double* w, int T, int K, int S, double* out) {
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += w[int64_t(t) * K + k] * y[int64_t(inv[int64_t(t) * K + k]) * H + c];
      out[int64_t(t) * H + c] = S ? acc + y[(int64_t(T) * K + t) * H + c] : acc;
    }
}

// Direct per-token evaluation, no permutation: for each token t,
// out[t] = sum_k w[t][k] FFN_{idx[t][k]}(x_t) + FFN_shared(x_t) (S = 1), with
// x_t and h quantised exactly as on the grouped path.
//   x [T][H] bf16 bits, idx/w [T][K] the routing to use -> out [T][H]
void oracle_token_outputs(const oracle_layer* L, const uint16_t* x, int T, const int32_t* idx, const double* w,
                          double* out) {
  const int H = L->H, F = L->F, K = L->K, HB = (H + kGroup - 1) / kGroup, FB = (F + kGroup - 1) / kGroup;
  parallel_for(T, [&](int t) {
    std::vector<float> x32(H), h32(F);
    std::vector<uint8_t> q(H), hq(F);
    std::vector<float> qs(HB), hs(FB);
    std::vector<double> a(H), h(F), b(F), y(H);
    for (int k = 0; k < H; ++k) x32[k] = float(bf16_bits_to_double(x[int64_t(t) * H + k]));
    quantize_row(x32.data(), H, q.data(), qs.data());
    oracle_dequant_rows(q.data(), H, qs.data(), 1, H, a.data());
    double* o = out + int64_t(t) * H;
    std::fill(o, o + H, 0.0);
    for (int j = 0; j < K + L->S; ++j) {
      const int g = j < K ? idx[int64_t(t) * K + j] : L->E;
      const double wt = j < K ? w[int64_t(t) * K + j] : 1.0;
      gate_up_row(L, g, a.data(), h.data());
      for (int n = 0; n < F; ++n) h32[n] = float(h[n]);
      quantize_row(h32.data(), F, hq.data(), hs.data());
      oracle_dequant_rows(hq.data(), F, hs.data(), 1, F, b.data());
      down_row(L, g, b.data(), y.data());
      for (int m = 0; m < H; ++m) o[m] += wt * y[m];
    }
  });
}

// BF16-checkpoint path (transformers PR #47844, "What does this PR do?":
// BF16 and FP8 checkpoints): weights W = bf16(fp32(decode(q) s)), the input
// x as given (bf16), no activation or h quantisation, FP64 sums.
//   x [T][H] bf16 bits, idx/w [T][K] the routing to use -> out [T][H]
void oracle_layer_forward_bf16(const oracle_layer* L, const uint16_t* x, int T, const int32_t* idx, const double* w,
                               double* out) {
  const int H = L->H, F = L->F, K = L->K, HB = (H + kGroup - 1) / kGroup, FB = (F + kGroup - 1) / kGroup;
  const double* tab = table().v;
  std::fill(out, out + int64_t(T) * H, 0.0);
  parallel_for(T, [&](int t) {
    std::vector<double> a(H), h(F);
    for (int k = 0; k < H; ++k) a[k] = bf16_bits_to_double(x[int64_t(t) * H + k]);
    for (int j = 0; j < K + L->S; ++j) {
      const int g = j < K ? idx[int64_t(t) * K + j] : L->E;
      const double wt = j < K ? w[int64_t(t) * K + j] : 1.0;
      const uint8_t* wg = L->w_gate + int64_t(g) * F * H;
      const uint8_t* wu = L->w_up + int64_t(g) * F * H;
      const uint8_t* wd = L->w_down + int64_t(g) * H * L->ld_f;
      const float* sg = L->s_gate + int64_t(g) * FB * HB;
      const float* su = L->s_up + int64_t(g) * FB * HB;
      const float* sd = L->s_down + int64_t(g) * HB * FB;
      for (int n = 0; n < F; ++n) {
        double gs = 0.0, us = 0.0;
        for (int k = 0; k < H; ++k) {
          const int blk = (n / kGroup) * HB + k / kGroup;
          gs += a[k] * round_bf16(tab[wg[int64_t(n) * H + k]] * double(sg[blk]));
          us += a[k] * round_bf16(tab[wu[int64_t(n) * H + k]] * double(su[blk]));
        }
        h[n] = silu(gs) * us;
      }
      for (int m = 0; m < H; ++m) {
        double acc = 0.0;
        for (int n = 0; n < F; ++n)
          acc += h[n] * round_bf16(tab[wd[int64_t(m) * L->ld_f + n]] * double(sd[(m / kGroup) * FB + n / kGroup]));
        out[int64_t(t) * H + m] += wt * acc;
      }
    }
  });
}

}  // extern "C"

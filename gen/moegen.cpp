// Seeded synthetic inputs for the FP8 MoE-layer forward.
//
// This module only draws random numbers and writes them out as a synthetic
// checkpoint and synthetic activations. It serves both the CUDA path and the
// CPU oracle and holds none of the layer's forward arithmetic.
//
// Random numbers: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC'11), a counter-based generator, so every
// element is a pure function of (seed, stream, element index) and the result
// does not depend on the thread count. Normals come from the Box-Muller
// transform of two 32-bit uniforms.
//
// Synthetic checkpoint: the model card of dots-studio/dots3-note-prev
// ("Model Overview") and transformers PR #47844 ("What does this PR do?")
// describe fine-grained FP8 checkpoints with E4M3 weights and one scale per
// 128 x 128 weight block. The generator builds such a checkpoint offline from
// Gaussian weights: per block, scale = amax / 448 in fp32 and each weight is
// stored as the E4M3 (OCP "FN") code nearest to w / scale, ties to the even
// code, saturating at +-448. This encoder is written here from the format
// definition and is independent of the oracle's and the GPU's.

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr uint32_t kMul0 = 0xD2511F53u;
constexpr uint32_t kMul1 = 0xCD9E8D57u;
constexpr uint32_t kWeyl0 = 0x9E3779B9u;
constexpr uint32_t kWeyl1 = 0xBB67AE85u;

inline void philox_round(uint32_t c[4], const uint32_t k[2]) {
  uint64_t p0 = uint64_t(kMul0) * c[0];
  uint64_t p1 = uint64_t(kMul1) * c[2];
  uint32_t hi0 = uint32_t(p0 >> 32), lo0 = uint32_t(p0);
  uint32_t hi1 = uint32_t(p1 >> 32), lo1 = uint32_t(p1);
  uint32_t n0 = hi1 ^ c[1] ^ k[0];
  uint32_t n1 = lo1;
  uint32_t n2 = hi0 ^ c[3] ^ k[1];
  uint32_t n3 = lo0;
  c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
}

inline void philox10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    if (r) { k[0] += kWeyl0; k[1] += kWeyl1; }
    philox_round(c, k);
  }
  out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

// Four normals for block index `blk` of (seed, stream): Box-Muller on the
// uniform pairs (o0, o1) and (o2, o3), each mapped to the open interval (0, 1).
inline void normals4(uint64_t seed, uint32_t stream, uint64_t blk, double z[4]) {
  uint32_t ctr[4] = {uint32_t(blk), uint32_t(blk >> 32), stream, 0u};
  uint32_t key[2] = {uint32_t(seed), uint32_t(seed >> 32)};
  uint32_t o[4];
  philox10(ctr, key, o);
  const double inv = 1.0 / 4294967296.0;
  const double two_pi = 6.283185307179586476925286766559;
  for (int p = 0; p < 2; ++p) {
    double u1 = (double(o[2 * p]) + 0.5) * inv;
    double u2 = (double(o[2 * p + 1]) + 0.5) * inv;
    double r = std::sqrt(-2.0 * std::log(u1));
    z[2 * p] = r * std::cos(two_pi * u2);
    z[2 * p + 1] = r * std::sin(two_pi * u2);
  }
}

// out[j] = sigma * normal sample (base + j) of (seed, stream), j in [0, n).
inline void fill_normals(uint64_t seed, uint32_t stream, uint64_t base, uint64_t n, float sigma,
                         float* out) {
  uint64_t i = base, end = base + n;
  double z[4];
  while (i < end) {
    normals4(seed, stream, i >> 2, z);
    for (uint64_t j = i & 3; j < 4 && i < end; ++j, ++i) out[i - base] = sigma * float(z[j]);
  }
}

// E4M3 "FN" code of v, nearest value with ties to the even code, saturating.
inline uint8_t e4m3_code(float v) {
  uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  float a = std::fabs(v);
  if (!(a < 448.0f)) return sign | 0x7E;  // saturate (NaN never reaches here)
  if (a < 0.015625f) {                    // below 2^-6: step 2^-9
    float q = std::nearbyint(a * 512.0f); // exact scaling, RNE
    return sign | uint8_t(q);             // q == 8 is code 0x08 = 2^-6
  }
  int e;
  float m = std::frexp(a, &e);            // a = m * 2^e, m in [0.5, 1)
  float f = m * 2.0f - 1.0f;              // a = (1 + f) * 2^(e-1), exact
  float q = std::nearbyint(f * 8.0f);
  int ee = e - 1;
  if (q == 8.0f) { q = 0.0f; ee += 1; }
  int code = ((ee + 7) << 3) | int(q);
  if (code > 0x7E) code = 0x7E;
  return sign | uint8_t(code);
}

template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
  if (nthreads <= 0) nthreads = int(std::thread::hardware_concurrency());
  if (nthreads <= 0) nthreads = 1;
  if (n < nthreads) nthreads = int(n > 0 ? n : 1);
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      int64_t i = next.fetch_add(1);
      if (i >= n) break;
      fn(i);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nthreads; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// Raw Philox4x32-10 block (for known-answer tests).
void moegen_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  philox10(ctr, key, out);
}

// out[i] = sigma * N(0,1) sample i of (seed, stream), i in [0, n).
void moegen_normal_f32(uint64_t seed, uint32_t stream, uint64_t n, float sigma, float* out,
                       int nthreads) {
  const int64_t chunk = 1 << 16;
  int64_t nchunks = int64_t((n + chunk - 1) / chunk);
  parallel_for(nchunks, nthreads, [&](int64_t c) {
    uint64_t lo = uint64_t(c) * chunk, hi = lo + chunk < n ? lo + chunk : n;
    fill_normals(seed, stream, lo, hi - lo, sigma, out + lo);
  });
}

// out[i] = 32-bit word i of (seed, stream).
void moegen_u32(uint64_t seed, uint32_t stream, uint64_t n, uint32_t* out) {
  uint32_t key[2] = {uint32_t(seed), uint32_t(seed >> 32)};
  for (uint64_t b = 0; b * 4 < n; ++b) {
    uint32_t ctr[4] = {uint32_t(b), uint32_t(b >> 32), stream, 0u};
    uint32_t o[4];
    philox10(ctr, key, o);
    for (int j = 0; j < 4 && b * 4 + j < n; ++j) out[b * 4 + j] = o[j];
  }
}

// Encode n fp32 values to E4M3 codes (exposed so tests can pin this encoder).
void moegen_e4m3_encode(const float* v, uint64_t n, uint8_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = e4m3_code(v[i]);
}

// Synthetic fine-grained FP8 checkpoint: nmat matrices of rows x cols Gaussian
// weights (std sigma), element (m, r, c) drawn as sample (m*rows + r)*cols + c
// of (seed, stream). Output codes[m][r][ld] (columns >= cols are zero) and
// scales[m][ceil(rows/128)][ceil(cols/128)] (dequant multipliers, w ~ q*s).
// Partial edge blocks take their amax over the real rows/columns only.
// Returns 0, or -1 on bad arguments.
int moegen_fp8_blocks(uint64_t seed, uint32_t stream, int nmat, int rows, int cols, int ld,
                      float sigma, uint8_t* codes, float* scales, int nthreads) {
  if (nmat < 0 || rows <= 0 || cols <= 0 || ld < cols || !codes || !scales) return -1;
  const int rb_n = (rows + 127) / 128, cb_n = (cols + 127) / 128;
  parallel_for(int64_t(nmat) * rb_n, nthreads, [&](int64_t task) {
    const int m = int(task / rb_n), rb = int(task % rb_n);
    const int r0 = rb * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
    std::vector<float> w(size_t(r1 - r0) * cols);
    fill_normals(seed, stream, (uint64_t(m) * rows + r0) * uint64_t(cols),
                 uint64_t(r1 - r0) * cols, sigma, w.data());
    for (int cb = 0; cb < cb_n; ++cb) {
      const int c0 = cb * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
      float amax = 0.0f;
      for (int r = r0; r < r1; ++r)
        for (int c = c0; c < c1; ++c) amax = std::fmax(amax, std::fabs(w[size_t(r - r0) * cols + c]));
      float s = amax / 448.0f;
      scales[(size_t(m) * rb_n + rb) * cb_n + cb] = s;
      for (int r = r0; r < r1; ++r) {
        uint8_t* dst = codes + (size_t(m) * rows + r) * size_t(ld);
        for (int c = c0; c < c1; ++c)
          dst[c] = (s == 0.0f) ? uint8_t(0) : e4m3_code(w[size_t(r - r0) * cols + c] / s);
      }
    }
    for (int r = r0; r < r1; ++r) {
      uint8_t* dst = codes + (size_t(m) * rows + r) * size_t(ld);
      if (ld > cols) std::memset(dst + cols, 0, size_t(ld - cols));
    }
  });
  return 0;
}

}  // extern "C"

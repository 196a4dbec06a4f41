// Weighted combine of the K routed expert rows of each token plus its shared
// expert row (weight 1), in FP32, rounded once to bf16.
//
// The layer output is the renormalised-weight sum of the selected experts'
// outputs plus the shared expert's (transformers docs page "Dots 3 Note
// Preview", Dots3NoteTextConfig: n_shared_experts 1, norm_topk_prob True,
// routed_scaling_factor 1.0). This is the "combine" of the pages' DeepEP
// transport (SGLang cookbook "Dots3-Note", "2. Configuration Tips"), here a
// deterministic gather: fixed slot order, shared row last, no atomics.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int CB_THREADS = 128;

// CTA (token, chunk of CB_THREADS*8 channels); each thread owns one
// 8-channel (16-byte) piece and loads its K+1 rows at once.
__global__ void __launch_bounds__(CB_THREADS) combine_kernel(const uint16_t* __restrict__ y,
                                                             const int32_t* __restrict__ inv,
                                                             const float* __restrict__ w, int T, int K, int S, int H,
                                                             uint16_t* __restrict__ out, int ldo) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  __shared__ int s_row[9];
  __shared__ float s_w[9];
  if (threadIdx.x < K) {
    s_row[threadIdx.x] = inv[size_t(t) * K + threadIdx.x];
    s_w[threadIdx.x] = w[size_t(t) * K + threadIdx.x];
  }
  __syncthreads();
  const size_t shared_row = size_t(T) * K + t;
  const int c = (blockIdx.y * CB_THREADS + threadIdx.x) * 8;
  if (c < H) {
    uint4 raws[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = k < K ? s_row[k] : -1;
      raws[k] = r >= 0 ? *reinterpret_cast<const uint4*>(y + size_t(r) * H + c) : make_uint4(0, 0, 0, 0);
    }
    const uint4 raw_shared = S ? *reinterpret_cast<const uint4*>(y + shared_row * H + c) : make_uint4(0, 0, 0, 0);
    float acc[8] = {};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= K || s_row[k] < 0) continue;
      const float wk = s_w[k];
      const uint4 raw = raws[k];
      const uint32_t p[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[2 * j] = fmaf(wk, bf16_bits_to_f32(uint16_t(p[j] & 0xFFFFu)), acc[2 * j]);
        acc[2 * j + 1] = fmaf(wk, bf16_bits_to_f32(uint16_t(p[j] >> 16)), acc[2 * j + 1]);
      }
    }
    const uint32_t p[4] = {raw_shared.x, raw_shared.y, raw_shared.z, raw_shared.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = acc[2 * j] + bf16_bits_to_f32(uint16_t(p[j] & 0xFFFFu));
      const float b = acc[2 * j + 1] + bf16_bits_to_f32(uint16_t(p[j] >> 16));
      o[j] = uint32_t(f32_to_bf16_bits(a)) | (uint32_t(f32_to_bf16_bits(b)) << 16);
    }
    *reinterpret_cast<uint4*>(out + size_t(t) * ldo + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const moe_layer_s* L, const uint16_t* y, const int32_t* inv, const float* w, int T,
                           uint16_t* out, int ldo, cudaStream_t st) {
  dim3 grid(T, (L->H + CB_THREADS * 8 - 1) / (CB_THREADS * 8));
  return launch_pdl(combine_kernel, grid, dim3(CB_THREADS), 0, st, y, inv, w, T, L->K, L->S, L->H, out, ldo);
}

}  // namespace moe

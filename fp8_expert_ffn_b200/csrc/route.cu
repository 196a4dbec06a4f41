// Router: FP32 logits = x . Wr^T, then top-K per token with renormalised
// softmax weights.
//
// transformers docs page "Dots 3 Note Preview", Dots3NoteTextConfig:
// n_routed_experts 256, num_experts_per_tok 8, n_group 1 / topk_group 1
// (ungrouped), norm_topk_prob True, routed_scaling_factor 1.0. The logits are
// FP32 (transformers PR #47844 states FP32 routing for the vision MoE router;
// the same precision is taken for the text router).
//
// Kernel 1 (route_logits): CTA tile of 64 tokens x 64 experts over a range of
// 128-channel K blocks (split-K when there are too few tiles to fill the
// GPU); per-thread 4 x 4 register tile; each K block is summed on its own and
// then added to the running sum (blocked summation keeps the FP32 error well
// under the near-tie threshold). Partial sums go to partial[s][t][e].
// Kernel 2 (route_topk): one warp per token sums the S partials in order,
// selects the top K by logit with ties to the lower id (an order-preserving
// 64-bit key), and writes the slots in ascending expert id with weights
// softmax(selected logits) * routed_scaling, which equals the softmax over
// all experts renormalised over the selection.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int RT_T = 64;    // tokens per CTA tile
constexpr int RT_E = 64;    // experts per CTA tile
constexpr int RT_KC = 32;   // channels per shared-memory chunk
constexpr int RT_THREADS = 256;

__global__ void __launch_bounds__(RT_THREADS) route_logits_kernel(const uint16_t* __restrict__ x, int T, int ldx,
                                                                  const float* __restrict__ wr, int E, int H,
                                                                  int kb_per_split, float* __restrict__ partial) {
  __shared__ __align__(16) float xs[RT_KC][RT_T];
  __shared__ __align__(16) float ws[RT_KC][RT_E];
  const int tid = threadIdx.x;
  const int e0 = blockIdx.x * RT_E, t0 = blockIdx.y * RT_T, split = blockIdx.z;
  const int HB = H / 128;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(HB, kb0 + kb_per_split);
  const int ty = tid / 16, tx = tid % 16;   // thread tile: tokens ty*4.., experts tx*4..

  float acc[4][4] = {};
  // loader mapping: 8 consecutive channels of one row per thread
  const int lrow = tid / 4, lk = (tid % 4) * 8;

  for (int kb = kb0; kb < kb1; ++kb) {
    float part[4][4] = {};
    for (int kc = 0; kc < 128; kc += RT_KC) {
      const int k = kb * 128 + kc + lk;
      {  // x chunk: token t0+lrow, channels k..k+7 (bf16)
        const int t = t0 + lrow;
        float v[8] = {};
        if (t < T) {
          uint4 raw = *reinterpret_cast<const uint4*>(x + size_t(t) * ldx + k);
          const uint16_t* p = reinterpret_cast<const uint16_t*>(&raw);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = bf16_bits_to_f32(p[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) xs[lk + j][lrow] = v[j];
      }
      {  // W chunk: expert e0+lrow, channels k..k+7
        const int e = e0 + lrow;
        float v[8] = {};
        if (e < E) {
          const float4* p = reinterpret_cast<const float4*>(wr + size_t(e) * H + k);
          float4 a = p[0], b = p[1];
          v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) ws[lk + j][lrow] = v[j];
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < RT_KC; ++kk) {
        float4 xv = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
        float4 wv = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
        const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
        const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) part[i][j] = fmaf(xa[i], wa[j], part[i][j]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) partial[(size_t(split) * T + t) * E + e] = acc[i][j];
    }
  }
}

__device__ __forceinline__ uint32_t ordered_bits(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ordered_bits(uint32_t o) {
  uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(u);
}

__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ partial, int S, int T, int E,
                                                         int K, float scaling, int32_t* __restrict__ idx,
                                                         float* __restrict__ w, float* __restrict__ logits_out) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  // expert e = lane + 32*j
  unsigned long long key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    key[j] = 0ull;
    if (e < E) {
      float l = 0.0f;
      for (int s = 0; s < S; ++s) l += partial[(size_t(s) * T + t) * E + e];
      l += 0.0f;  // -0 -> +0 so that equal logits compare equal
      if (logits_out) logits_out[size_t(t) * E + e] = l;
      key[j] = (static_cast<unsigned long long>(ordered_bits(l)) << 32) | (0xFFFFFFFFu - uint32_t(e));
    }
  }
  int my_e = -1;
  float my_l = 0.0f;
  for (int r = 0; r < K; ++r) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int j = 0; j < 8; ++j) best = key[j] > best ? key[j] : best;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      unsigned long long o = __shfl_xor_sync(0xFFFFFFFFu, best, off);
      best = o > best ? o : best;
    }
    const int e = int(0xFFFFFFFFu - uint32_t(best & 0xFFFFFFFFull));
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j == e) key[j] = 0ull;      // remove the winner
    if (lane == r) {
      my_e = e;
      my_l = from_ordered_bits(uint32_t(best >> 32));
    }
  }
  // weights: softmax over the selected logits; the first pick is the max.
  const float lmax = __shfl_sync(0xFFFFFFFFu, my_l, 0);
  const float ex = (lane < K) ? expf(my_l - lmax) : 0.0f;
  float sum = 0.0f;
  for (int r = 0; r < K; ++r) sum += __shfl_sync(0xFFFFFFFFu, ex, r);
  // slot position = rank of the expert id among the selected ids
  int pos = 0;
  for (int r = 0; r < K; ++r) {
    const int er = __shfl_sync(0xFFFFFFFFu, my_e, r);
    pos += (er < my_e) ? 1 : 0;
  }
  if (lane < K) {
    idx[size_t(t) * K + pos] = my_e;
    w[size_t(t) * K + pos] = (ex / sum) * scaling;
  }
}

}  // namespace

int route_splits(const moe_layer_s* L, int T) {
  const int tiles = ((T + RT_T - 1) / RT_T) * ((L->E + RT_E - 1) / RT_E);
  int s = (2 * L->num_sms + tiles - 1) / tiles;
  if (s < 1) s = 1;
  if (s > L->HB) s = L->HB;
  return s;
}

cudaError_t launch_route(const moe_layer_s* L, const uint16_t* x, int T, int ldx, int32_t* idx, float* w,
                         float* logits, float* partial, cudaStream_t st) {
  const int S = route_splits(L, T);
  const int kb_per = (L->HB + S - 1) / S;
  const int S_eff = (L->HB + kb_per - 1) / kb_per;
  dim3 grid((L->E + RT_E - 1) / RT_E, (T + RT_T - 1) / RT_T, S_eff);
  route_logits_kernel<<<grid, RT_THREADS, 0, st>>>(x, T, ldx, L->w.router_w, L->E, L->H, kb_per, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_topk_kernel<<<(T + 7) / 8, 256, 0, st>>>(partial, S_eff, T, L->E, L->K, L->d.routed_scaling, idx, w,
                                                  logits);
  return cudaGetLastError();
}

}  // namespace moe

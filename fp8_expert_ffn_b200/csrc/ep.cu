// Expert parallelism: the row movement around the two all-to-all exchanges
// of the DeepEP transport that the SGLang cookbook "Dots3-Note" names for the
// MoE layer ("2. Configuration Tips": expert parallelism across 8 GPUs with
// DeepEP dispatch and combine).
//
// The routed experts are split into P contiguous blocks of El experts, one
// per rank; the shared expert is replicated. A source rank's permuted rows
// are already grouped by expert, so the rows it sends to rank p (experts
// [p*El, (p+1)*El)) are one contiguous range, in expert order. After the
// dispatch exchange an owner holds them sender-major: for each sender s, its
// rows for local expert 0, 1, ..., El-1. The grouped GEMMs want them
// expert-major (each expert's rows contiguous), with the owner's own shared
// rows last, and the activation scales group-major. The kernels here:
//   ep_pack_scales  source side: the routed rows' scales, group-major
//                   [HB][rows] -> row-major [R][HB], so that a destination's
//                   rows and their scales are contiguous for the exchange
//   ep_regroup      owner side: sender-major received rows + own shared rows
//                   -> the expert-major GEMM input, group-major scales and
//                   the group offsets
//   ep_unregroup    owner side: the GEMM output back to sender-major order
//                   for the return exchange; the shared rows to the owner's
//                   own output rows
// Segment (s, e) = the rows from sender s for local expert e. Every CTA
// derives both segment tables from the P x El counts with two block-wide
// prefix scans, then copies one row per warp with 16-byte accesses.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int EP_THREADS = 256;
constexpr int EP_SCAN = EP_THREADS * (kEpMaxSegments / EP_THREADS);

// Exclusive prefix of v[0..n) in the order given by at(i) (n <= kEpMaxSegments);
// out[i] is the sum of the values before position i; returns the total.
template <typename At>
__device__ int block_exclusive_scan(int n, At at, int* out, int* warp_sums) {
  const int per = kEpMaxSegments / EP_THREADS;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  int local[per];
  int sum = 0;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    const int i = t * per + j;
    local[j] = i < n ? at(i) : 0;
    sum += local[j];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < wid; ++w) base += warp_sums[w];
  int run = base + incl - sum;
#pragma unroll
  for (int j = 0; j < per; ++j) {
    const int i = t * per + j;
    if (i < n) out[i] = run;
    run += local[j];
  }
  int total = 0;
  for (int w = 0; w < EP_THREADS / 32; ++w) total += warp_sums[w];
  __syncthreads();
  return total;
}

struct EpPlan {
  int* seg_in;    // [P*El] sender-major: row of segment (s, e) in the received buffer, index s*El + e
  int* seg_out;   // [P*El + 1] expert-major: row of segment (s, e) in the GEMM input, index e*P + s
};

// Both segment tables of the counts cnt[s*El + e], in shared memory.
__device__ void ep_plan(const int32_t* __restrict__ cnt, int P, int El, EpPlan& pl, int* warp_sums) {
  const int n = P * El;
  block_exclusive_scan(n, [&](int i) { return int(cnt[i]); }, pl.seg_in, warp_sums);
  const int total = block_exclusive_scan(n, [&](int i) { return int(cnt[(i % P) * El + i / P]); }, pl.seg_out,
                                         warp_sums);
  if (threadIdx.x == 0) pl.seg_out[n] = total;
  __syncthreads();
}

// Segment (in expert-major order) holding GEMM-input row o < N.
__device__ __forceinline__ int seg_of(const int* seg_out, int n, int o) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {   // last k with seg_out[k] <= o
    const int mid = (lo + hi + 1) >> 1;
    if (seg_out[mid] <= o) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) ep_pack_scales_kernel(const float* __restrict__ xs, int rows, int R, int HB,
                                                              float* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= size_t(R) * HB) return;
  const int r = int(i / HB), g = int(i - size_t(r) * HB);
  out[i] = xs[size_t(g) * rows + r];
}

__global__ void __launch_bounds__(EP_THREADS) ep_regroup_kernel(
    const int32_t* __restrict__ cnt, int P, int El, int N, const uint8_t* __restrict__ recv_q,
    const float* __restrict__ recv_s, const uint8_t* __restrict__ own_q, const float* __restrict__ own_s,
    int own_rows, int R, int T_shared, int H, int HB, uint8_t* __restrict__ out_q, float* __restrict__ out_s,
    int32_t* __restrict__ out_offsets, uint32_t* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int s_in[EP_SCAN], s_out[EP_SCAN + 1], s_w[EP_THREADS / 32];
  EpPlan pl{s_in, s_out};
  ep_plan(cnt, P, El, pl, s_w);
  const int n = P * El;
  const int rows_out = N + T_shared;
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= El; e += blockDim.x) out_offsets[e] = e < El ? s_out[e * P] : N;
    if (threadIdx.x == 0) out_offsets[El + 1] = rows_out;
  }
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (EP_THREADS / 32);
  for (int o = blockIdx.x * (EP_THREADS / 32) + (threadIdx.x >> 5); o < rows_out; o += nwarps) {
    const uint8_t* src_q;
    const float* src_s;
    size_t src_stride_s;   // distance between a row's consecutive scales in the source
    if (o < N) {
      const int k = seg_of(s_out, n, o);
      const int e = k / P, s = k - e * P;
      const int in = s_in[s * El + e] + (o - s_out[k]);
#ifdef MOE_CHECKS
      if (in < 0 || in >= N) {   // counts that do not describe the received rows
        if (lane == 0) set_status(status, STATUS_BOUNDS);
        continue;
      }
#endif
      src_q = recv_q + size_t(in) * H;
      src_s = recv_s + size_t(in) * HB;
      src_stride_s = 1;
    } else {
      const int r = R + (o - N);
      src_q = own_q + size_t(r) * H;
      src_s = own_s + r;
      src_stride_s = size_t(own_rows);
    }
    uint8_t* dst = out_q + size_t(o) * H;
    for (int c = lane; c < H / 16; c += 32)
      reinterpret_cast<uint4*>(dst)[c] = reinterpret_cast<const uint4*>(src_q)[c];
    for (int g = lane; g < HB; g += 32) out_s[size_t(g) * rows_out + o] = src_s[size_t(g) * src_stride_s];
  }
}

__global__ void __launch_bounds__(EP_THREADS) ep_unregroup_kernel(const int32_t* __restrict__ cnt, int P, int El,
                                                                  int N, const uint16_t* __restrict__ y_g, int R,
                                                                  int T_shared, int H, uint16_t* __restrict__ y_send,
                                                                  uint16_t* __restrict__ y_own, uint32_t* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int s_in[EP_SCAN], s_out[EP_SCAN + 1], s_w[EP_THREADS / 32];
  EpPlan pl{s_in, s_out};
  ep_plan(cnt, P, El, pl, s_w);
  const int n = P * El;
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (EP_THREADS / 32);
  for (int o = blockIdx.x * (EP_THREADS / 32) + (threadIdx.x >> 5); o < N + T_shared; o += nwarps) {
    uint16_t* dst;
    if (o < N) {
      const int k = seg_of(s_out, n, o);
      const int e = k / P, s = k - e * P;
      const int in = s_in[s * El + e] + (o - s_out[k]);
#ifdef MOE_CHECKS
      if (in < 0 || in >= N) {
        if (lane == 0) set_status(status, STATUS_BOUNDS);
        continue;
      }
#endif
      dst = y_send + size_t(in) * H;
    } else {
      dst = y_own + size_t(R + (o - N)) * H;
    }
    const uint4* src = reinterpret_cast<const uint4*>(y_g + size_t(o) * H);
    for (int c = lane; c < H / 8; c += 32) reinterpret_cast<uint4*>(dst)[c] = src[c];
  }
}

int ep_grid(int rows) {
  const int warps = EP_THREADS / 32;
  int g = (rows + warps - 1) / warps;
  return g < 1 ? 1 : (g > 1184 ? 1184 : g);   // up to 8 CTAs per SM, then grid-stride
}

}  // namespace

cudaError_t launch_ep_pack_scales(const moe_layer_s* L, const float* xs, int T, float* out, cudaStream_t st) {
  const int rows = T * (L->K + L->S), R = T * L->K;
  const size_t n = size_t(R) * L->HB;
  if (n == 0) return cudaSuccess;
  return launch_pdl(ep_pack_scales_kernel, dim3(unsigned((n + 255) / 256)), dim3(256), 0, st, xs, rows, R, L->HB, out);
}

cudaError_t launch_ep_regroup(const moe_layer_s* L, int P, const int32_t* cnt, int N, const uint8_t* recv_q,
                              const float* recv_s, const uint8_t* own_q, const float* own_s, int T, uint8_t* out_q,
                              float* out_s, int32_t* out_offsets, cudaStream_t st) {
  const int Ts = T * L->S;
  return launch_pdl(ep_regroup_kernel, dim3(ep_grid(N + Ts)), dim3(EP_THREADS), 0, st, cnt, P, L->E, N, recv_q,
                    recv_s, own_q, own_s, T * (L->K + L->S), T * L->K, Ts, L->H, L->HB, out_q, out_s, out_offsets,
                    L->status);
}

cudaError_t launch_ep_unregroup(const moe_layer_s* L, int P, const int32_t* cnt, int N, const uint16_t* y_g, int T,
                                uint16_t* y_send, uint16_t* y_own, cudaStream_t st) {
  const int Ts = T * L->S;
  return launch_pdl(ep_unregroup_kernel, dim3(ep_grid(N + Ts)), dim3(EP_THREADS), 0, st, cnt, P, L->E, N, y_g,
                    T * L->K, Ts, L->H, y_send, y_own, L->status);
}

}  // namespace moe

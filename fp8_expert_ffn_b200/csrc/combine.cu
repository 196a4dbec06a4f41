// Weighted combine of the K routed expert rows of each token plus its shared
// expert row (weight 1), in FP32, rounded once to bf16.
//
// The layer output is the renormalised-weight sum of the selected experts'
// outputs plus the shared expert's (transformers docs page "Dots 3 Note
// Preview", Dots3NoteTextConfig: n_shared_experts 1, norm_topk_prob True,
// routed_scaling_factor 1.0). This is the "combine" of the pages' DeepEP
// transport (SGLang cookbook "Dots3-Note", "2. Configuration Tips"), here a
// deterministic gather: fixed slot order, shared row last, no atomics. With
// expert parallelism over peer memory (combine_kernel<true>) each slot's row
// is read from the output rows of its expert's owner rank.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int CB_THREADS = 128;

struct CombineArgs {
  const uint16_t* y;       // local: [rows][H], routed rows then the shared rows
  const int32_t* inv;      // [T][K] row of (token, slot), -1 if none
  const float* w;          // [T][K]
  int T, K, S, H;
  uint16_t* out;
  int ldo;
  // expert parallel: slot k's row is in the y buffer of its expert's owner
  const int32_t* idx;      // [T][K]
  const uint64_t* peer_y;  // [ranks] rows [cap][H] bf16
  const int32_t* goff;     // [El+2] this rank's group offsets: its shared rows start at goff[El]
  int rank, El;
  int rows_limit;          // rows of each y buffer (bounds-checked build)
  uint32_t* status;
};

// CTA (token, chunk of CB_THREADS*8 channels); each thread owns one
// 8-channel (16-byte) piece and loads its K+1 rows at once. With EP the rows
// are read from their owners' buffers (a peer's memory over NVLink, plain
// 16-byte loads).
template <bool EP>
__global__ void __launch_bounds__(CB_THREADS) combine_kernel(const CombineArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x, K = a.K, H = a.H;
  __shared__ const uint16_t* s_src[9];
  __shared__ float s_w[9];
  if (threadIdx.x < K) {
    int r = a.inv[size_t(t) * K + threadIdx.x];
#ifdef MOE_CHECKS
    if (r >= a.rows_limit) {
      set_status(a.status, STATUS_BOUNDS);
      r = -1;
    }
#endif
    const uint16_t* src = nullptr;
    if (r >= 0) {
      const uint16_t* ybase = EP ? reinterpret_cast<const uint16_t*>(a.peer_y[a.idx[size_t(t) * K + threadIdx.x] / a.El])
                                 : a.y;
      src = ybase + size_t(r) * H;
    }
    s_src[threadIdx.x] = src;
    s_w[threadIdx.x] = a.w[size_t(t) * K + threadIdx.x];
  } else if (threadIdx.x == K) {
    const uint16_t* src = nullptr;
    if (a.S && !EP) {
      src = a.y + (size_t(a.T) * K + t) * H;
    } else if (a.S) {
      // this rank's shared rows are [goff[El], goff[El+1]) of its own buffer
      // (both 0 after an overflow: then nothing is read)
      const int row = a.goff[a.El] + t;
      bool ok = row < a.goff[a.El + 1];
#ifdef MOE_CHECKS
      if (ok && (row < 0 || row >= a.rows_limit)) {
        set_status(a.status, STATUS_BOUNDS);
        ok = false;
      }
#endif
      if (ok) src = reinterpret_cast<const uint16_t*>(a.peer_y[a.rank]) + size_t(row) * H;
    }
    s_src[K] = src;
  }
  __syncthreads();
  const int c = (blockIdx.y * CB_THREADS + threadIdx.x) * 8;
  if (c < H) {
    uint4 raws[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint16_t* src = k < K ? s_src[k] : nullptr;
      raws[k] = src ? *reinterpret_cast<const uint4*>(src + c) : make_uint4(0, 0, 0, 0);
    }
    const uint4 raw_shared = s_src[K] ? *reinterpret_cast<const uint4*>(s_src[K] + c) : make_uint4(0, 0, 0, 0);
    float acc[8] = {};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= K || !s_src[k]) continue;
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
      const float a0 = acc[2 * j] + bf16_bits_to_f32(uint16_t(p[j] & 0xFFFFu));
      const float a1 = acc[2 * j + 1] + bf16_bits_to_f32(uint16_t(p[j] >> 16));
      o[j] = uint32_t(f32_to_bf16_bits(a0)) | (uint32_t(f32_to_bf16_bits(a1)) << 16);
    }
    *reinterpret_cast<uint4*>(a.out + size_t(t) * a.ldo + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const moe_layer_s* L, const uint16_t* y, const int32_t* inv, const float* w, int T,
                           uint16_t* out, int ldo, cudaStream_t st) {
  CombineArgs a = {};
  a.y = y;
  a.inv = inv;
  a.w = w;
  a.T = T;
  a.K = L->K;
  a.S = L->S;
  a.H = L->H;
  a.out = out;
  a.ldo = ldo;
  a.rows_limit = T * (L->K + L->S);
  a.status = L->status;
  dim3 grid(T, (L->H + CB_THREADS * 8 - 1) / (CB_THREADS * 8));
  return launch_pdl(combine_kernel<false>, grid, dim3(CB_THREADS), 0, st, a);
}

cudaError_t launch_ep_combine(const moe_layer_s* L, const moe_ep_comm_s* c, const int32_t* idx, const int32_t* inv_ep,
                              const float* w, const int32_t* goff, int T, uint16_t* out, int ldo, cudaStream_t st) {
  CombineArgs a = {};
  a.inv = inv_ep;
  a.w = w;
  a.T = T;
  a.K = L->K;
  a.S = L->S;
  a.H = L->H;
  a.out = out;
  a.ldo = ldo;
  a.idx = idx;
  a.peer_y = c->d_peer_y;
  a.goff = goff;
  a.rank = c->rank;
  a.El = L->E / c->ranks;
  a.rows_limit = c->cap;
  a.status = L->status;
  dim3 grid(T, (L->H + CB_THREADS * 8 - 1) / (CB_THREADS * 8));
  return launch_pdl(combine_kernel<true>, grid, dim3(CB_THREADS), 0, st, a);
}

}  // namespace moe

// Router: FP32-accurate logits = x . Wr^T on the tensor cores, then top-K per
// token with renormalised softmax weights.
//
// transformers docs page "Dots 3 Note Preview", Dots3NoteTextConfig:
// n_routed_experts 256, num_experts_per_tok 8, n_group 1 / topk_group 1
// (ungrouped), norm_topk_prob True, routed_scaling_factor 1.0. The logits are
// FP32 (transformers PR #47844 states FP32 routing for the vision MoE router;
// the same precision is taken for the text router).
//
// FP32 accuracy from bf16 tensor cores: x is bf16 already, and every fp32
// router weight splits exactly into three bf16 terms, w = hi + mid + lo
// (8 significant bits each; the split is written once at layer creation). A
// product of two bf16 values is exact in fp32, so x . Wr^T = sum over the
// three terms of bf16 GEMMs, each with exact products. The tensor cores sum
// the 3 x 64 products of one 64-channel K block into an fp32 TMEM partial;
// epilogue warps add each partial into an fp32 register accumulator (blocked
// summation, error far below the near-tie threshold of the routing).
//
// Kernel 1 (route_tc_kernel): CTA tile 128 tokens x 128 experts over a range of
// 64-channel K blocks (split-K when there are fewer tiles than SMs); warp 0
// TMA (x box 128 x 64 bf16 plus three 128 x 64 weight boxes per stage, 3
// stages of 64 KB), warp 1 tcgen05.mma kind::f16 (M 128, N 128, K 16; 12 per
// stage) into two 128-column TMEM buffers, warps 4-11 promote (two per TMEM
// lane quarter, one per 64-column half). Partial sums go to partial[s][t][e].
// Kernel 2 (route_topk): one warp per token sums the S partials in order,
// selects the top K by logit with ties to the lower id (an order-preserving
// 64-bit key), and writes the slots in ascending expert id with weights
// softmax(selected logits) * routed_scaling, which equals the softmax over
// all experts renormalised over the selection.
// Router variants of the config schema: with a selection-only bias the key
// is p + bias (p the softmax over all experts); with n_group > 1 only the
// topk_group groups whose best member scores highest (ties to the lower
// group) are eligible; with norm_topk_prob off the weights are p itself.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int RM = 128;                  // tokens per tile
constexpr int RN = int(kRouterExperts);  // experts per tile
constexpr int RK = 64;                   // channels per K block (128 bytes of bf16)
constexpr int R_STAGES = 3;
constexpr int R_A_BYTES = RM * RK * 2;   // 16 KB
constexpr int R_B_BYTES = RN * RK * 2;   // 16 KB per split term
constexpr int R_STAGE_BYTES = R_A_BYTES + 3 * R_B_BYTES;   // 64 KB
constexpr int R_EPI_WARPS = 8;
constexpr int R_FIRST_EPI_WARP = 4;
constexpr int R_THREADS = 32 * (R_FIRST_EPI_WARP + R_EPI_WARPS);   // 384
constexpr int R_SMEM_DYN = R_STAGES * R_STAGE_BYTES + 1024;
constexpr uint32_t R_TMEM_COLS = 2 * RN;   // two partial buffers
// register split as in the grouped GEMM: the first warpgroup (TMA, MMA)
// drops to R_PRODUCER_REGS, the two epilogue warpgroups rise to R_EPILOGUE_REGS
constexpr int R_LAUNCH_REGS = 168;
constexpr int R_PRODUCER_REGS = 40;
constexpr int R_EPILOGUE_REGS = 232;
static_assert(128 * R_PRODUCER_REGS + 256 * R_EPILOGUE_REGS <= R_THREADS * R_LAUNCH_REGS, "register split");

// kind::f16 instruction descriptor: A = B = BF16, D = F32, both K-major.
constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
constexpr uint32_t R_IDESC = idesc_bf16_f32(RM, RN);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(R_THREADS, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int E,
                    int kb_per_split, int nkb, float* __restrict__ partial, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[R_STAGES];
  __shared__ __align__(8) uint64_t empty_bar[R_STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int s_abort_store;
  __shared__ uint32_t s_consumed;
  volatile int* s_abort = &s_abort_store;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * RN, t0 = blockIdx.y * RM, split = blockIdx.z;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(nkb, kb0 + kb_per_split);
  const int n = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], R_EPI_WARPS);
    }
    mbar_init(&done_bar, 1);
    s_abort_store = 0;
    s_consumed = 0;
    fence_mbar_init();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) tmem_alloc(&tmem_base_s, R_TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();   // set-up above overlaps the previous kernel; x and the partials are touched below
  pdl_launch_dependents();
  const uint32_t tmem_base = tmem_base_s;
  uint32_t issued = 0;

  // The two warpgroup kinds run to the end on separate paths (each with its
  // own copy of the teardown) so the setmaxnreg limits hold throughout.
  if (warp < R_FIRST_EPI_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R_PRODUCER_REGS));
    if (warp == 0) {
      if (lane == 0) {
        uint32_t it = 0;
        for (int kb = 0; kb < n; ++kb) {
          const int s = it % R_STAGES;
          const uint32_t ph = (it / R_STAGES) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u, s_abort, status)) break;
          uint8_t* a = smem + s * R_STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], R_STAGE_BYTES);
          const int k = (kb0 + kb) * RK;
          tma_load_2d(a, &tmX, &full_bar[s], k, t0);
#pragma unroll
          for (int j = 0; j < 3; ++j) tma_load_3d(a + R_A_BYTES + j * R_B_BYTES, &tmW, &full_bar[s], k, e0, j);
          ++it;
        }
        issued = it;
      }
    } else if (warp == 1) {
      if (lane == 0) {
        uint32_t it = 0;
        for (int kb = 0; kb < n; ++kb) {
          const int s = it % R_STAGES;
          const uint32_t ph = (it / R_STAGES) & 1u;
          const uint32_t buf = it & 1u, tph = (it >> 1) & 1u;
          if (!mbar_wait(&tempty_bar[buf], tph ^ 1u, s_abort, status)) break;
          if (!mbar_wait(&full_bar[s], ph, s_abort, status)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * R_STAGE_BYTES);
          const uint64_t ad = smem_desc_sw128(a_addr);
          const uint32_t d = tmem_base + buf * RN;
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            const uint64_t bd = smem_desc_sw128(a_addr + R_A_BYTES + j * R_B_BYTES);
#pragma unroll
            for (int k = 0; k < RK / 16; ++k)   // 16 bf16 = 32 bytes = 2 in the 16-byte address field
              mma_bf16(d, ad + uint64_t(2 * k), bd + uint64_t(2 * k), R_IDESC, (j | k) ? 1u : 0u);
          }
          tc_commit(&empty_bar[s]);
          tc_commit(&tfull_bar[buf]);
          ++it;
        }
        s_consumed = it;
        tc_commit(&done_bar);
        int never = 0;
        mbar_wait(&done_bar, 0, &never, status);
      }
    }
    asm volatile("bar.sync 0;" ::: "memory");
    if (warp == 0 && lane == 0) {
      int never = 0;
      for (uint32_t j = s_consumed; j < issued; ++j)
        mbar_wait(&full_bar[j % R_STAGES], (j / R_STAGES) & 1u, &never, status);
    }
    tc_fence_before();
    asm volatile("bar.sync 0;" ::: "memory");
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem_base, R_TMEM_COLS);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R_EPILOGUE_REGS));
    // warp w reads TMEM lanes 32*(w%4).. (its 32 tokens) and one half of the
    // 256 expert columns
    const int q = warp & 3;
    const int half = (warp - R_FIRST_EPI_WARP) >> 2;
    const int t = t0 + q * 32 + lane;
    float acc[RN / 2];
#pragma unroll
    for (int j = 0; j < RN / 2; ++j) acc[j] = 0.0f;
    bool ok = true;
    for (int kb = 0; kb < n; ++kb) {
      const uint32_t buf = kb & 1u, tph = (kb >> 1) & 1u;
      if (!mbar_wait(&tfull_bar[buf], tph, s_abort, status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + buf * RN + half * (RN / 2);
#pragma unroll
      for (int c = 0; c < RN / 2 / 32; c += 2) {
        float va[32], vb[32];
        tmem_ld32(tbase + c * 32, va);
        tmem_ld32(tbase + c * 32 + 32, vb);
        tmem_ld_wait();
        if (c + 2 >= RN / 2 / 32) {   // the buffer is in registers: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[buf]);
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          acc[c * 32 + j] += va[j];
          acc[c * 32 + 32 + j] += vb[j];
        }
      }
    }
    const int eh = e0 + half * (RN / 2);
    if (ok && t < T) {
      float* dst = partial + (size_t(split) * T + t) * E + eh;
      if (eh + RN / 2 <= E && (E % 4) == 0) {
#pragma unroll
        for (int j = 0; j < RN / 2; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < RN / 2; ++j)
          if (eh + j < E) dst[j] = acc[j];
      }
    }
    asm volatile("bar.sync 0;" ::: "memory");
    tc_fence_before();
    asm volatile("bar.sync 0;" ::: "memory");
  }
}

// hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid); both
// differences are exact in fp32.
__global__ void router_split_kernel(const float* __restrict__ w, size_t n, uint16_t* __restrict__ out) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = w[i];
  const uint16_t hi = f32_to_bf16_bits(v);
  const float r1 = v - bf16_bits_to_f32(hi);
  const uint16_t mid = f32_to_bf16_bits(r1);
  const float r2 = r1 - bf16_bits_to_f32(mid);
  out[i] = hi;
  out[n + i] = mid;
  out[2 * n + i] = f32_to_bf16_bits(r2);
}

__device__ __forceinline__ uint32_t ordered_bits(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkArgs {
  const float* partial;  // [S][T][E] split-K partial logits
  int S, T, E, K;
  float scaling;         // routed_scaling_factor
  int norm;              // norm_topk_prob
  int n_group, topk_group;
  const float* bias;     // [E] selection-only bias or null
  int32_t* idx;
  float* w;
  float* logits_out;     // [T][E] or null
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const unsigned long long o = __shfl_xor_sync(0xFFFFFFFFu, v, off);
    v = o > v ? o : v;
  }
  return v;
}

__global__ void __launch_bounds__(256) route_topk_kernel(const TopkArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ unsigned long long s_key[8][256];   // per warp: the selection keys, for group scores
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + wid;
  if (t >= a.T) return;
  const int E = a.E, K = a.K;
  // expert e = lane + 32*j; the S split-K partials are added in order s = 0..S-1
  float l[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) l[j] = 0.0f;
  const float* pt = a.partial + size_t(t) * E + lane;
  const size_t ps = size_t(a.T) * E;
  // eight split slices in flight at a time; the sum stays in split order
  int s = 0;
  for (; s + 8 <= a.S; s += 8) {
    float v[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) v[u][j] = (lane + 32 * j < E) ? __ldg(pt + (s + u) * ps + 32 * j) : 0.0f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) l[j] += v[u][j];
  }
  if (s + 4 <= a.S) {
    float v[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) v[u][j] = (lane + 32 * j < E) ? __ldg(pt + (s + u) * ps + 32 * j) : 0.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) l[j] += v[u][j];
    s += 4;
  }
  for (; s < a.S; ++s) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (lane + 32 * j < E) ? __ldg(pt + s * ps + 32 * j) : 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) l[j] += v[j];
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    l[j] += 0.0f;  // -0 -> +0 so that equal logits compare equal
    if (a.logits_out && lane + 32 * j < E) a.logits_out[size_t(t) * E + lane + 32 * j] = l[j];
  }
  // softmax over all E experts, needed for a selection bias (s = p + b) and
  // for weights that are not renormalised
  const bool full_p = a.bias != nullptr || !a.norm;
  float lmax_all = 0.0f, sum_all = 1.0f;
  float ex[8];
  if (full_p) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < E) m = fmaxf(m, l[j]);
    lmax_all = warp_max(m);
    float sl = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ex[j] = (lane + 32 * j < E) ? expf(l[j] - lmax_all) : 0.0f;
      sl += ex[j];
    }
    sum_all = warp_sum(sl);
  }
  // selection keys: order-preserving bits of the score, inverted id as tie-break
  unsigned long long key[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    key[j] = 0ull;
    if (e < E) {
      const float sc = a.bias ? ex[j] / sum_all + __ldg(a.bias + e) : l[j];
      key[j] = (static_cast<unsigned long long>(ordered_bits(sc)) << 32) | (0xFFFFFFFFu - uint32_t(e));
    }
  }
  if (a.n_group > 1) {
    // group g = experts [g*gs, (g+1)*gs), scored by its best member; the
    // topk_group best groups (ties to the lower group) stay eligible
    const int gs = E / a.n_group;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j < E) s_key[wid][lane + 32 * j] = key[j];
    __syncwarp();
    unsigned long long gk = 0ull;
    if (lane < a.n_group) {
      uint32_t best = 0u;
      for (int e = lane * gs; e < (lane + 1) * gs; ++e) {
        const uint32_t sb = uint32_t(s_key[wid][e] >> 32);
        best = sb > best ? sb : best;
      }
      gk = (static_cast<unsigned long long>(best) << 32) | (0xFFFFFFFFu - uint32_t(lane));
    }
    uint32_t keep = 0u;
    for (int r = 0; r < a.topk_group; ++r) {
      const unsigned long long b = warp_max_u64(gk);
      const int g = int(0xFFFFFFFFu - uint32_t(b & 0xFFFFFFFFull));
      keep |= 1u << g;
      if (lane == g) gk = 0ull;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((keep >> (e / gs)) & 1u)) key[j] = 0ull;
    }
  }
  int my_e = -1;
  float my_l = 0.0f;
  for (int r = 0; r < K; ++r) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int j = 0; j < 8; ++j) best = key[j] > best ? key[j] : best;
    best = warp_max_u64(best);
    const int e = int(0xFFFFFFFFu - uint32_t(best & 0xFFFFFFFFull));
    float le = 0.0f;   // the winner's logit, from the lane that holds it
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (lane + 32 * j == e) {
        key[j] = 0ull;  // remove the winner
        le = l[j];
      }
    le = __shfl_sync(0xFFFFFFFFu, le, e & 31);
    if (lane == r) {
      my_e = e;
      my_l = le;
    }
  }
  // weights from the unbiased probabilities: renormalised, the softmax over
  // the selected logits; otherwise the softmax over all experts
  float wv;
  if (a.norm) {
    const float lmax = warp_max(lane < K ? my_l : -INFINITY);
    const float es = (lane < K) ? expf(my_l - lmax) : 0.0f;
    float sum = 0.0f;
    for (int r = 0; r < K; ++r) sum += __shfl_sync(0xFFFFFFFFu, es, r);
    wv = es / sum;
  } else {
    wv = expf(my_l - lmax_all) / sum_all;
  }
  // slot position = rank of the expert id among the selected ids
  int pos = 0;
  for (int r = 0; r < K; ++r) {
    const int er = __shfl_sync(0xFFFFFFFFu, my_e, r);
    pos += (er < my_e) ? 1 : 0;
  }
  if (lane < K) {
    a.idx[size_t(t) * K + pos] = my_e;
    a.w[size_t(t) * K + pos] = wv * a.scaling;
  }
}

}  // namespace

int route_splits(const moe_layer_s* L, int T) {
  const int nkb = L->H / RK;
  const int tiles = ((T + RM - 1) / RM) * ((L->E + RN - 1) / RN);
  int s = L->num_sms / tiles;               // one wave: tiles * s <= SMs
  s = s > nkb / 4 ? nkb / 4 : s;          // at least 4 K blocks per split
  return s < 1 ? 1 : s;
}

cudaError_t launch_router_split(const float* w, int E, int H, uint16_t* out, cudaStream_t st) {
  const size_t n = size_t(E) * H;
  router_split_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(w, n, out);
  return cudaGetLastError();
}

cudaError_t launch_route(const moe_layer_s* L, const uint16_t* x, int T, int ldx, int32_t* idx, float* w,
                         float* logits, float* partial, cudaStream_t st) {
  static std::atomic<bool> configured[kMaxDevices];   // the attribute is per device
  cudaError_t ce = once_per_device(configured, []() {
    // setmaxnreg.inc draws on the CTA's launch registers: refuse a build
    // whose register count cannot fund the split
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, route_tc_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * R_THREADS < 128 * R_PRODUCER_REGS + 256 * R_EPILOGUE_REGS) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, R_SMEM_DYN);
  });
  if (ce != cudaSuccess) return ce;
  const int nkb = L->H / RK;
  const int S = route_splits(L, T);
  const int kb_per = (nkb + S - 1) / S;
  const int S_eff = (nkb + kb_per - 1) / kb_per;
  CUtensorMap tmX;
  if (!encode_tmap(&tmX, true, x, L->H, T, 1, uint64_t(ldx) * 2, 0)) return cudaErrorInvalidValue;
  dim3 grid((L->E + RN - 1) / RN, (T + RM - 1) / RM, S_eff);
  cudaError_t e = launch_pdl(route_tc_kernel, grid, dim3(R_THREADS), R_SMEM_DYN, st, tmX, L->tm_router, T, L->E,
                             kb_per, nkb, partial, L->status);
  if (e != cudaSuccess) return e;
  TopkArgs ta;
  ta.partial = partial;
  ta.S = S_eff;
  ta.T = T;
  ta.E = L->E;
  ta.K = L->K;
  ta.scaling = L->d.routed_scaling;
  ta.norm = L->d.norm_topk;
  ta.n_group = L->d.n_group;
  ta.topk_group = L->d.topk_group;
  ta.bias = L->router_bias;
  ta.idx = idx;
  ta.w = w;
  ta.logits_out = logits;
  return launch_pdl(route_topk_kernel, dim3((T + 7) / 8), dim3(256), 0, st, ta);
}

}  // namespace moe

// Token permutation by expert with the dynamic activation quantiser fused
// into the gather.
//
// Grouping tokens by expert is the "dispatch" of the pages' DeepEP transport
// (SGLang cookbook "Dots3-Note", "2. Configuration Tips", MoE runner); on one
// GPU it is a counting sort. Activation quantisation follows transformers
// PR #47844 ("What does this PR do?": dynamic activations, E4M3): per token
// per 128 channels, s = fp32(amax) / 448, q = E4M3_RNE_satfinite(x / s), both
// divisions IEEE fp32; an all-zero group gives s = 0 and q = 0.
//
// Determinism without ordering atomics: every (token, expert) pair sets one
// bit of a per-expert token bitmap (atomicOr, order-independent). The row of
// (t, k) inside expert e's group is the number of earlier tokens that chose
// e: a prefix popcount over e's bitmap words. Kernels:
//   1. permute_clear    zero the bitmap and the completion counter
//   2. permute_bitmap   one thread per (t, k): validate, set the bit
//   3. permute_count    one CTA per expert: per-word prefix popcounts, count;
//                       the last CTA to finish scans the counts -> offsets[E+2]
//   (small batches: 1-3 in one CTA, permute_plan_small, when the bitmap fits
//   in shared memory)
//   4. gather_rows      one warp per token and 16 groups of 128 channels (4
//                       for small batches):
//                       rows of its K slots and its shared-expert row,
//                       inv/perm, then the groups of x quantised once and
//                       stored to all rows with 16-byte stores.
// With expert parallelism over peer memory the same gather is the dispatch
// (gather_rows<GATHER_EP>): each routed row goes to the receive buffer of
// its expert's owner rank, at the row the owner's grouped GEMMs read.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// Zeroes the token bitmap (n words) that the bitmap kernel ORs into, and the
// count kernel's completion counter.
__global__ void __launch_bounds__(256) permute_clear_kernel(uint32_t* __restrict__ bitmap, size_t n,
                                                            uint32_t* __restrict__ done) {
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0 && threadIdx.x == 0) *done = 0u;
  const size_t i = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 4 <= n) *reinterpret_cast<uint4*>(bitmap + i) = make_uint4(0u, 0u, 0u, 0u);
  else for (size_t k = i; k < n; ++k) bitmap[k] = 0u;
}

__global__ void permute_bitmap_kernel(const int32_t* __restrict__ idx, int T, int K, int E, int W,
                                      uint32_t* __restrict__ bitmap, uint32_t* status) {
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * K) return;
  const int t = i / K;
  const int e = idx[i];
  if (e < 0 || e >= E) {
    set_status(status, STATUS_BAD_EXPERT);
    return;
  }
  const uint32_t bit = 1u << (t & 31);
  const uint32_t old = atomicOr(&bitmap[size_t(e) * W + (t >> 5)], bit);
  if (old & bit) set_status(status, STATUS_DUP_EXPERT);
}

// One CTA (256 threads) per expert: wprefix[e][w] = set bits of e's words
// before word w; counts[e] = all set bits. The last CTA to finish (a device
// counter, zeroed by the clear kernel) turns the counts into the offsets:
// offsets[g] = sum of counts[0..g), offsets[E+1] = offsets[E] + T*S. The
// offsets depend only on the counts, so the result is the same whichever CTA
// is last.
__global__ void __launch_bounds__(256) permute_count_kernel(const uint32_t* __restrict__ bitmap, int W,
                                                            uint32_t* __restrict__ wprefix, int32_t* counts, int E,
                                                            int T, int S, int32_t* __restrict__ offsets,
                                                            uint32_t* done) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ uint32_t warp_sums[8];
  __shared__ bool s_last;
  const int e = blockIdx.x, tid = threadIdx.x;
  const uint32_t* row = bitmap + size_t(e) * W;
  uint32_t* out = wprefix + size_t(e) * W;
  const int per = (W + 255) / 256;
  const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
  uint32_t local = 0;
  for (int w = w0; w < w1; ++w) local += __popc(row[w]);
  // exclusive scan of `local` over the CTA
  const int lane = tid & 31, wid = tid >> 5;
  uint32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  uint32_t base = 0;
  for (int j = 0; j < wid; ++j) base += warp_sums[j];
  uint32_t run = base + incl - local;
  for (int w = w0; w < w1; ++w) {
    out[w] = run;
    run += __popc(row[w]);
  }
  if (tid == 255) counts[e] = int32_t(base + incl);
  __threadfence();   // this CTA's count is visible device-wide before it signals
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(done, 1u) == uint32_t(E - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // the last CTA: exclusive scan of the E <= 256 counts (read past L1)
  const int v = tid < E ? __ldcg(counts + tid) : 0;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
    if (lane >= off) inc += o;
  }
  __syncthreads();   // warp_sums is reused below
  if (lane == 31) warp_sums[wid] = uint32_t(inc);
  __syncthreads();
  int b = 0;
  for (int j = 0; j < wid; ++j) b += int(warp_sums[j]);
  if (tid < E) offsets[tid] = b + inc - v;
  if (tid == E - 1) {
    offsets[E] = b + inc;
    offsets[E + 1] = b + inc + T * S;
  }
}

// Small batches: the whole plan in one CTA. When the token bitmap (E x W
// words) fits in shared memory, one CTA zeroes it, sets the bits, counts and
// scans: the bitmap, the per-word prefixes and the offsets it writes are the
// same as those of the three-kernel path (clear, bitmap, count).
constexpr int kPlanSmallWords = 8192;     // 32 KB of shared memory
constexpr int kPlanSmallThreads = 1024;

__global__ void __launch_bounds__(kPlanSmallThreads) permute_plan_small_kernel(
    const int32_t* __restrict__ idx, int T, int K, int E, int W, int S, uint32_t* __restrict__ bitmap,
    uint32_t* __restrict__ wprefix, int32_t* __restrict__ counts, int32_t* __restrict__ offsets, uint32_t* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ uint32_t s_bits[kPlanSmallWords];
  __shared__ int s_cnt[256];
  __shared__ int s_wsum[kPlanSmallThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int nw = E * W;
  for (int i = tid; i < nw; i += kPlanSmallThreads) s_bits[i] = 0u;
  __syncthreads();
  for (int i = tid; i < T * K; i += kPlanSmallThreads) {
    const int t = i / K, e = idx[i];
    if (e < 0 || e >= E) {
      set_status(status, STATUS_BAD_EXPERT);
      continue;
    }
    const uint32_t bit = 1u << (t & 31);
    if (atomicOr(&s_bits[e * W + (t >> 5)], bit) & bit) set_status(status, STATUS_DUP_EXPERT);
  }
  __syncthreads();
  // expert e: prefix popcounts over its W words (one thread per expert)
  for (int e = tid; e < E; e += kPlanSmallThreads) {
    uint32_t run = 0;
    for (int w = 0; w < W; ++w) {
      const uint32_t b = s_bits[e * W + w];
      bitmap[size_t(e) * W + w] = b;
      wprefix[size_t(e) * W + w] = run;
      run += __popc(b);
    }
    s_cnt[e] = int(run);
    counts[e] = int(run);
  }
  __syncthreads();
  // exclusive scan of the E <= 256 counts
  const int v = tid < E ? s_cnt[tid] : 0;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) s_wsum[wid] = inc;
  __syncthreads();
  int base = 0;
  for (int j = 0; j < wid; ++j) base += s_wsum[j];
  if (tid < E) offsets[tid] = base + inc - v;
  if (tid == E - 1) {
    offsets[E] = base + inc;
    offsets[E + 1] = base + inc + T * S;
  }
}

// 128-channel groups per warp (steps of 4 groups): 16 for large batches;
// 4 while the batch is small (a decode batch of 64 tokens then spreads over
// 640 warps instead of 192, and each warp's chain of loads is shorter)
constexpr int GATHER_GROUPS_LARGE = 16;
constexpr int GATHER_GROUPS_SMALL = 4;
constexpr int kGatherSmallT = 512;
constexpr int GATHER_THREADS = 256;

enum GatherMode { GATHER_LOCAL = 0, GATHER_EP = 1 };

struct GatherArgs {
  const uint16_t* x;
  int T, ldx, H;
  const int32_t* idx;
  int K, E, W, S;
  const uint32_t* bitmap;
  const uint32_t* wprefix;
  // GATHER_LOCAL: this GPU's grouped layout
  const int32_t* offsets;
  int rows;
  int32_t* perm;
  int32_t* inv;
  uint8_t* xq;
  float* xs;
  // GATHER_EP: the rows' owners' receive buffers
  const int32_t* all_off;   // [ranks][E+2] every rank's local offsets
  int rank, ranks, El, cap;
  const uint64_t* peer_q;   // [ranks] code buffers [cap][H]
  const uint64_t* peer_s;   // [ranks] scale buffers [HB][cap]
  int32_t* inv_ep;          // [T][K] row in the owner's buffer, -1 if none
  int32_t* goff;            // [El+2] this rank's group offsets as an owner
  uint32_t* status;
};

// Expert-parallel layout, computed by every CTA from the ranks' offsets.
// Owner p holds local expert e's rows from sender 0, 1, ..., ranks-1 in turn,
// experts in order, then its own shared rows. For a global expert g the rows
// this rank sends start at base[g] in g's owner's buffer.
__device__ void ep_layout(const GatherArgs& a, int* s_base, int* s_excl, int* s_wsum, int* s_nr, int* s_over) {
  const int i = threadIdx.x, lane = i & 31, wid = i >> 5;
  const int E = a.E, stride = E + 2;
  int tot = 0, pre = 0;
  bool bad = false;
  if (i < E) {
    for (int s = 0; s < a.ranks; ++s) {
      const int c = a.all_off[s * stride + i + 1] - a.all_off[s * stride + i];
      bad |= c < 0;
      tot += c;
      if (s < a.rank) pre += c;
    }
  }
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) s_wsum[wid] = incl;
  if (i == 0) *s_over = 0;
  __syncthreads();
  if (bad) {   // offsets not ascending: nothing is dispatched
    atomicOr(s_over, 2);
    set_status(a.status, STATUS_BAD_PLAN);
  }
  int before = 0;
  for (int j = 0; j < wid; ++j) before += s_wsum[j];
  if (i < E) s_excl[i] = before + incl - tot;
  if (i == E - 1) s_excl[E] = before + incl;
  __syncthreads();
  if (i < E) s_base[i] = s_excl[i] - s_excl[(i / a.El) * a.El] + pre;
  if (i < a.ranks) {   // owner i's routed rows plus its own shared rows must fit its buffer
    const int n = s_excl[(i + 1) * a.El] - s_excl[i * a.El];
    const int sh = a.all_off[i * stride + E + 1] - a.all_off[i * stride + E];
    if (sh < 0) {
      atomicOr(s_over, 2);
      set_status(a.status, STATUS_BAD_PLAN);
    } else if (n + sh > a.cap) {
      atomicOr(s_over, 1);
    }
  }
  if (i == 0) *s_nr = s_excl[(a.rank + 1) * a.El] - s_excl[a.rank * a.El];
  __syncthreads();
  if (blockIdx.x == 0) {
    const bool over = *s_over != 0;
    const int e0 = a.rank * a.El;
    for (int e = i; e < a.El; e += blockDim.x) a.goff[e] = over ? 0 : s_excl[e0 + e] - s_excl[e0];
    if (i == 0) {
      const int sh = a.all_off[a.rank * stride + E + 1] - a.all_off[a.rank * stride + E];
      a.goff[a.El] = over ? 0 : *s_nr;
      a.goff[a.El + 1] = over ? 0 : *s_nr + sh;
      if (*s_over & 1) set_status(a.status, STATUS_EP_OVERFLOW);
    }
  }
}

// One warp per (token, chunk of GATHER_GROUPS groups). In each step the warp
// covers 4 consecutive groups: lanes 8j..8j+7 hold group j of the step, 16
// channels per lane (one 32-byte load of x, one 16-byte store of codes per
// row), so a row's store instruction writes 512 contiguous bytes. Lane k < K
// owns slot k's row, lane K the shared row; the chunk-0 warp writes the row
// maps. GATHER_LOCAL writes the rows of this GPU's grouped layout (and inv,
// perm); GATHER_EP writes each routed row into its expert's owner's receive
// buffer (a peer's memory over NVLink; every store is a plain 16- or 4-byte
// store, no bulk or tensor copy) and the shared row into this rank's own.
template <int MODE, int GATHER_GROUPS>
__global__ void __launch_bounds__(GATHER_THREADS, 4) gather_rows_kernel(const GatherArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int s_base[MODE == GATHER_EP ? 256 : 1];
  __shared__ int s_excl[MODE == GATHER_EP ? 257 : 1];
  __shared__ int s_wsum[GATHER_THREADS / 32];
  __shared__ int s_nr, s_over;
  __shared__ uint64_t s_peer[MODE == GATHER_EP ? 2 * kEpMaxRanks : 1];   // codes, then scales
  const int T = a.T, K = a.K, E = a.E, H = a.H;
  const int lane = threadIdx.x & 31;
  const int gl = lane & 7, gs = lane >> 3;   // lane within its group, group slot of the step
  const int HB = H / 128;
  const int nchunk = (HB + GATHER_GROUPS - 1) / GATHER_GROUPS;
  const int wid = blockIdx.x * (GATHER_THREADS / 32) + (threadIdx.x >> 5);
  const int t = wid / nchunk, chunk = wid - t * nchunk;
  const bool has_token = t < T;
  const int g0 = chunk * GATHER_GROUPS;
  // issue the x loads of the whole chunk before anything waits on memory
  // (with EP, before the layout is computed)
  uint4 raw[GATHER_GROUPS / 4][2];
#pragma unroll
  for (int i = 0; i < GATHER_GROUPS / 4; ++i) {
    const int g = g0 + 4 * i + gs;
    if (has_token && g < HB) {
      const uint4* src = reinterpret_cast<const uint4*>(a.x + size_t(t) * a.ldx + g * 128 + gl * 16);
      raw[i][0] = src[0];
      raw[i][1] = src[1];
    } else {
      raw[i][0] = raw[i][1] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (MODE == GATHER_EP) {
    for (int i = threadIdx.x; i < a.ranks; i += GATHER_THREADS) {
      s_peer[i] = a.peer_q[i];
      s_peer[kEpMaxRanks + i] = a.peer_s[i];
    }
    ep_layout(a, s_base, s_excl, s_wsum, &s_nr, &s_over);   // ends with a CTA barrier
  }
  if (!has_token) return;
  const int W = a.W;

  // this lane's row; with EP the row in its owner's buffer, packed with the
  // owner's index (rows < 2^24, owners < 64)
  int my_row = -1;
  const bool over = MODE == GATHER_EP && s_over != 0;
  if (lane < K) {
    const int e = a.idx[size_t(t) * K + lane];
    bool ok = (e >= 0 && e < E) && !over;
    for (int j = 0; j < lane && ok; ++j) ok = (a.idx[size_t(t) * K + j] != e);  // first slot of a repeat wins
    int row = -1;
    if (ok) {
      const uint32_t word = a.bitmap[size_t(e) * W + (t >> 5)];
      const int within = int(a.wprefix[size_t(e) * W + (t >> 5)]) + __popc(word & ((1u << (t & 31)) - 1u));
      if (MODE == GATHER_LOCAL) {
        row = a.offsets[e] + within;
#ifdef MOE_CHECKS
        if (row < 0 || row >= a.rows) {
          set_status(a.status, STATUS_BOUNDS);
          row = -1;
        }
#endif
        my_row = row;
      } else if (within < a.all_off[a.rank * (E + 2) + e + 1] - a.all_off[a.rank * (E + 2) + e]) {
        // (a row beyond this rank's own count in all_offsets is not this
        // rank's plan: skipped and flagged, so no store leaves its range)
        row = s_base[e] + within;
        my_row = row | ((e / a.El) << 24);
      } else {
        set_status(a.status, STATUS_BAD_PLAN);
      }
    }
    if (chunk == 0) {
      if (MODE == GATHER_LOCAL) {
        a.inv[size_t(t) * K + lane] = row;
        if (row >= 0) a.perm[row] = t;
      } else {
        a.inv_ep[size_t(t) * K + lane] = row;
      }
    }
  } else if (lane == K && a.S) {
    if (MODE == GATHER_LOCAL) {
      my_row = a.offsets[E] + t;
#ifdef MOE_CHECKS
      if (my_row < 0 || my_row >= a.rows) {
        set_status(a.status, STATUS_BOUNDS);
        my_row = -1;
      }
#endif
      if (chunk == 0 && my_row >= 0) a.perm[my_row] = t;
    } else if (!over) {
      if (t < a.all_off[a.rank * (E + 2) + E + 1] - a.all_off[a.rank * (E + 2) + E])
        my_row = (s_nr + t) | (a.rank << 24);
      else
        set_status(a.status, STATUS_BAD_PLAN);
    }
  }
  // the token's rows, known to every lane
  int rowv[9];
#pragma unroll
  for (int j = 0; j < 9; ++j) rowv[j] = __shfl_sync(0xFFFFFFFFu, my_row, j);
  const size_t sstride = MODE == GATHER_LOCAL ? size_t(a.rows) : size_t(a.cap);

#pragma unroll
  for (int i = 0; i < GATHER_GROUPS / 4; ++i) {
    const int g = g0 + 4 * i + gs;
    const bool valid = g < HB;   // uniform over the 8 lanes of a group
    const uint32_t w32[8] = {raw[i][0].x, raw[i][0].y, raw[i][0].z, raw[i][0].w,
                             raw[i][1].x, raw[i][1].y, raw[i][1].z, raw[i][1].w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[2 * j] = bf16_bits_to_f32(uint16_t(w32[j] & 0xFFFFu));
      v[2 * j + 1] = bf16_bits_to_f32(uint16_t(w32[j] >> 16));
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
    float s = 0.0f;
    if (amax > 0.0f) {
      s = __fdiv_rn(amax, 448.0f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = e4m3x2(__fdiv_rn(v[4 * j], s), __fdiv_rn(v[4 * j + 1], s));
        const uint32_t hi = e4m3x2(__fdiv_rn(v[4 * j + 2], s), __fdiv_rn(v[4 * j + 3], s));
        packed[j] = lo | (hi << 16);
      }
    }
    if (!valid) continue;
    const uint4 q = make_uint4(packed[0], packed[1], packed[2], packed[3]);
#pragma unroll
    for (int j = 0; j < 9; ++j) {
      if (j > K) break;
      const int r = rowv[j];
      if (r < 0) continue;
      uint8_t* qb;
      float* sb;
      if (MODE == GATHER_LOCAL) {
        qb = a.xq + size_t(r) * H;
        sb = a.xs + r;
      } else {
        const int p = r >> 24, rr = r & 0xFFFFFF;
        qb = reinterpret_cast<uint8_t*>(s_peer[p]) + size_t(rr) * H;
        sb = reinterpret_cast<float*>(s_peer[kEpMaxRanks + p]) + rr;
      }
      *reinterpret_cast<uint4*>(qb + g * 128 + gl * 16) = q;
      if (gl == (j & 7)) sb[size_t(g) * sstride] = s;
    }
  }
  // the rows written into peers' memory are complete, system-wide, before
  // the warp finishes (the owners read them after a barrier that follows
  // this kernel): one system-scope fence per warp, after the warp's lanes
  // have synchronised, orders all of the warp's stores (fences are
  // cumulative)
  if (MODE == GATHER_EP) {
    __syncwarp();
    if (lane == 0) __threadfence_system();
  }
}

}  // namespace

int permute_kernels(const moe_layer_s* L, int T) {
  return size_t(L->E) * ((T + 31) / 32) <= size_t(kPlanSmallWords) ? 2 : 4;
}

// One warp per (token, chunk of groups); at least one CTA (with EP it writes
// the owner offsets even when this rank sends nothing).
template <int MODE>
static cudaError_t launch_gather(const GatherArgs& a, int HB, int T, cudaStream_t st) {
  const bool small = T <= kGatherSmallT;
  const int groups = small ? GATHER_GROUPS_SMALL : GATHER_GROUPS_LARGE;
  const long long warps = static_cast<long long>(T) * ((HB + groups - 1) / groups);
  const int wpc = GATHER_THREADS / 32;
  const long long ctas = (warps + wpc - 1) / wpc;
  const dim3 grid(unsigned(ctas > 0 ? ctas : 1));
  if (small) return launch_pdl(gather_rows_kernel<MODE, GATHER_GROUPS_SMALL>, grid, dim3(GATHER_THREADS), 0, st, a);
  return launch_pdl(gather_rows_kernel<MODE, GATHER_GROUPS_LARGE>, grid, dim3(GATHER_THREADS), 0, st, a);
}

// The plan of the permutation: the token bitmap and its per-word prefixes in
// the scratch, the counts, and offsets[E+2].
static cudaError_t launch_plan(const moe_layer_s* L, const int32_t* idx, int T, int32_t* offsets, const Scratch& s,
                        cudaStream_t st) {
  const int K = L->K, E = L->E, W = (T + 31) / 32;
  const int S = L->S;
  const size_t nwords = size_t(E) * W;
  cudaError_t e;
  if (permute_kernels(L, T) == 2)
    return launch_pdl(permute_plan_small_kernel, dim3(1), dim3(kPlanSmallThreads), 0, st, idx, T, K, E, W, S,
                      s.bitmap, s.wprefix, s.counts, offsets, L->status);
  uint32_t* done = reinterpret_cast<uint32_t*>(s.counts + E);
  e = launch_pdl(permute_clear_kernel, dim3(unsigned((nwords + 1023) / 1024)), dim3(256), 0, st, s.bitmap, nwords,
                 done);
  if (e != cudaSuccess) return e;
  e = launch_pdl(permute_bitmap_kernel, dim3((T * K + 255) / 256), dim3(256), 0, st, idx, T, K, E, W, s.bitmap,
                 L->status);
  if (e != cudaSuccess) return e;
  return launch_pdl(permute_count_kernel, dim3(E), dim3(256), 0, st, static_cast<const uint32_t*>(s.bitmap), W,
                    s.wprefix, s.counts, E, T, S, offsets, done);
}

cudaError_t launch_permute(const moe_layer_s* L, const uint16_t* x, int T, int ldx, const int32_t* idx,
                           int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs,
                           const Scratch& s, cudaStream_t st) {
  const int K = L->K, E = L->E, W = (T + 31) / 32;
  const int S = L->S;
  const int rows = T * (K + S);
  cudaError_t e = launch_plan(L, idx, T, offsets, s, st);
  if (e != cudaSuccess) return e;
  GatherArgs a = {};
  a.x = x;
  a.T = T;
  a.ldx = ldx;
  a.H = L->H;
  a.idx = idx;
  a.K = K;
  a.E = E;
  a.W = W;
  a.S = S;
  a.bitmap = s.bitmap;
  a.wprefix = s.wprefix;
  a.offsets = offsets;
  a.rows = rows;
  a.perm = perm;
  a.inv = inv;
  a.xq = xq;
  a.xs = xs;
  a.status = L->status;
  return launch_gather<GATHER_LOCAL>(a, L->HB, T, st);
}

cudaError_t launch_ep_plan(const moe_layer_s* L, const int32_t* idx, int T, int32_t* offsets, const Scratch& s,
                           cudaStream_t st) {
  return launch_plan(L, idx, T, offsets, s, st);
}

cudaError_t launch_ep_dispatch(const moe_layer_s* L, const moe_ep_comm_s* c, const uint16_t* x, int T, int ldx,
                               const int32_t* idx, const int32_t* all_off, int32_t* inv_ep, int32_t* goff,
                               const Scratch& s, cudaStream_t st) {
  GatherArgs a = {};
  a.x = x;
  a.T = T;
  a.ldx = ldx;
  a.H = L->H;
  a.idx = idx;
  a.K = L->K;
  a.E = L->E;
  a.W = (T + 31) / 32;
  a.S = L->S;
  a.bitmap = s.bitmap;
  a.wprefix = s.wprefix;
  a.all_off = all_off;
  a.rank = c->rank;
  a.ranks = c->ranks;
  a.El = L->E / c->ranks;
  a.cap = c->cap;
  a.peer_q = c->d_peer_q;
  a.peer_s = c->d_peer_s;
  a.inv_ep = inv_ep;
  a.goff = goff;
  a.status = L->status;
  return launch_gather<GATHER_EP>(a, L->HB, T, st);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the permutation: its scratch (the per-expert
// token bitmap, the per-word prefix counts and the expert counts) lives in
// one file-scope device array instead of a caller workspace, sized for
// kNoAllocMaxTokens tokens and kNoAllocMaxExperts experts. Every GPU that
// loads the library holds the array (about 257 KB) until the process exits.
// All calls on a device share it and it keeps the last call's contents: the
// bitmap is cleared at the start of every call (the prefixes and counts are
// fully rewritten), and calls whose kernels overlap on the GPU race on it.
namespace {

constexpr int kNoAllocWords = kNoAllocMaxExperts * ((kNoAllocMaxTokens + 31) / 32);
static __device__ __align__(256) uint32_t g_permute_scratch[2 * kNoAllocWords + kNoAllocMaxExperts + 1];

uint32_t* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_permute_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is asked of
// the runtime once per device (with that device current) and cached.
cudaError_t noalloc_scratch(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_permute_noalloc(const moe_layer_s* L, const uint16_t* x, int T, int ldx, const int32_t* idx,
                                   int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs,
                                   cudaStream_t st) {
  uint32_t* base = nullptr;
  cudaError_t e = noalloc_scratch(&base);
  if (e != cudaSuccess) return e;
  const int W = (T + 31) / 32;
  Scratch s = {};
  s.bitmap = base;
  s.wprefix = base + size_t(L->E) * W;
  s.counts = reinterpret_cast<int32_t*>(base + 2 * kNoAllocWords);
  return launch_permute(L, x, T, ldx, idx, offsets, perm, inv, xq, xs, s, st);
}

}  // namespace moe

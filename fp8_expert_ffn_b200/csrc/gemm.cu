// Grouped FP8 GEMMs of the expert FFN with per-128-K-block scale promotion.
//
// Fine-grained FP8 (transformers PR #47844, "What does this PR do?"): E4M3
// weights with one fp32 scale per 128 x 128 block and dynamically quantised
// activations with one fp32 scale per token per 128 channels. Both scales are
// constant over one 128-wide K block, so a GEMM over K = sum of K blocks is
//   C[r, n] = sum_kb  P_kb[r, n] * sw[n/128, kb] * sa[r, kb],
//   P_kb[r, n] = sum_{k in kb} qa[r, k] * qw[n, k]   (E4M3 x E4M3, fp32).
// The tensor cores compute each P_kb (tcgen05.mma kind::f8f6f4, 4 MMAs of
// K = 32 into a TMEM buffer); epilogue warps read it back and promote it into
// an FP32 register accumulator with the scalar sw * sa of their row. The
// scales are arbitrary fp32 values, which the hardware's power-of-two block
// scaling cannot represent, hence the software promotion.
//
// Expert FFN (Dots3NoteTextConfig: hidden_act silu, mlp_bias False,
// moe_intermediate_size 1536; SwiGLU experts with gate_proj, up_proj,
// down_proj):
//   gate/up GEMM: tile = 128 rows x (128 gate + 128 up channels of one
//     128-channel block); the epilogue forms h = silu(G) * U in fp32 and
//     quantises it per row per 128 channels (s = amax/448, E4M3 RNE), so the
//     quantisation group is exactly one tile's channel block;
//   down GEMM: tile = 128 rows x 256 output columns (two 128-column weight
//     blocks); the epilogue rounds y to bf16 (or, with the K blocks split
//     over CTAs for batches with few tiles, writes its FP32 partial).
//
// Kernel layout (one CTA per SM, persistent over a device-side tile list):
//   warp 0      TMA producer: A tile 128 x 128 B, two B tiles 128 x 128 B per
//               stage, 4-stage mbarrier ring (48 KB per stage, 128-byte swizzle)
//   warp 1      TMEM allocator (512 columns) and single-thread MMA issuer;
//               two 256-column TMEM buffers hold consecutive K-block partials
//   warp 2      decodes the tile list one tile ahead into a two-slot ring and
//               pulls each tile's first scales into L1; warp 3 idles
//   warps 4-11  epilogue: warp w reads TMEM lanes 32*(w%4).. (its rows) and
//               one half of the 256 columns; promotion, then the fused
//               SwiGLU+quant or bf16 tail, written through swizzled shared
//               memory boxes by bulk tensor stores.
// Tile order: per group (expert), chunks of up to 8 row tiles, then the
// n tiles, then the row tiles of the chunk -- the row tiles that share one
// weight tile run side by side, so that weight tile comes from HBM once.
//
// Every wait is bounded (1 s); a timeout sets the layer's status word and
// all roles leave their loops; the producer then waits for its own copies in
// flight, the MMA thread for its own MMAs, and the TMEM is released.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int BM = 128;                    // rows per tile
constexpr int BK = 128;                    // K bytes per stage = one scale block
constexpr int BN = 256;                    // columns per tile (two 128-column halves)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;           // 16 KB
constexpr int BH_BYTES = 128 * BK;         // 16 KB per B half
constexpr int STAGE_BYTES = A_BYTES + 2 * BH_BYTES;
constexpr int EPI_WARPS = 8;
// Three warpgroups: warpgroup 0 = TMA warp, MMA warp and two idle warps;
// warpgroups 1 and 2 = the epilogue. setmaxnreg moves registers from the
// first to the other two: the launch gets LAUNCH_REGS per thread (the
// 384-thread, one-CTA-per-SM cap), the producer warpgroup keeps PRODUCER_REGS
// and each epilogue thread gets EPILOGUE_REGS (128 FP32 accumulators plus
// two 32-column TMEM loads in flight). The split adds up to the launch total.
constexpr int THREADS = 384;
constexpr int FIRST_EPI_WARP = 4;
constexpr int LAUNCH_REGS = 168;
constexpr int PRODUCER_REGS = 40;
constexpr int EPILOGUE_REGS = 232;
static_assert(128 * PRODUCER_REGS + 256 * EPILOGUE_REGS <= THREADS * LAUNCH_REGS, "register split exceeds launch");
static_assert(THREADS == 32 * (FIRST_EPI_WARP + EPI_WARPS), "warp layout");
constexpr int MCHUNK = 8;                  // row tiles per chunk of the tile order
constexpr int MAX_GROUPS = 257;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_e4m3_f32(BM, BN);
// Output staging, one box of a bulk tensor store per epilogue warp: down,
// 32 rows x 64 bf16 columns (4 KB, 128-byte swizzle); gate/up, 32 rows x the
// warp's 64 h channels (2 KB, 64-byte swizzle).
constexpr int stg_warp_bytes(int mode) { return mode == 1 ? 32 * 128 : 32 * 64; }
constexpr int smem_dyn(int mode) { return STAGES * STAGE_BYTES + 1024 + EPI_WARPS * stg_warp_bytes(mode); }

enum { MODE_GATEUP = 0, MODE_DOWN = 1 };
// EPI_SPLIT (down GEMM only): the tile's K blocks are split over ksplit
// CTAs, each writes its promoted FP32 partial, and a second kernel sums the
// partials in split order and rounds to bf16 (batches with fewer output
// tiles than SMs, e.g. the dense FFN at decode sizes).
enum { EPI_FUSED = 0, EPI_F32 = 1, EPI_SPLIT = 2 };

struct GemmArgs {
  const int32_t* offsets;  // [ngroups + 1] row offsets of the groups
  int ngroups;
  int ntn;                 // n tiles per group
  int nkb;                 // K blocks
  int rows;                // rows in the permuted buffers
  const float* as;         // activation scales [nkb][rows]
  const float* ws0;        // weight scales [group][ws_nb][ws_kb]
  const float* ws1;
  int ws_nb, ws_kb;
  int nb_count;            // valid 128-column output blocks (down GEMM)
  uint8_t* h;              // gate/up: quantised h [rows][ld_h]
  float* hs;               // gate/up: h scales [ntn][rows]
  int ld_h;
  uint16_t* y;             // down: y [rows][ld_y] bf16
  int ld_y;
  float* out;              // test: promoted accumulators [rows][ld_out]
  int ld_out;
  int ksplit;              // K splits per output tile (1 unless EPI_SPLIT)
  float* part;             // EPI_SPLIT: partials [ksplit][rows][ld_y] fp32
  uint32_t* status;
  unsigned long long wait_ns;  // limit of every pipeline wait (kWaitLimitNs; a test may shorten it)
  int withhold;            // test only: CTA 0's producer skips its first stage, so a wait must time out
};

struct TileInfo {
  int g, nt, row0, nvalid;
  int kb0, kb1, sp;        // K blocks [kb0, kb1) of split sp
};

// K blocks of split sp of ksplit (contiguous, sizes differ by at most one).
__device__ __forceinline__ void split_range(int sp, int ksplit, int nkb, int& kb0, int& kb1) {
  kb0 = sp * nkb / ksplit;
  kb1 = (sp + 1) * nkb / ksplit;
}

// Tile i of the list: output tile i / ksplit, split i % ksplit.
__device__ __forceinline__ TileInfo decode_tile(int i, const int* s_prefix, const int* __restrict__ off, int ngroups,
                                                int ntn, int ksplit, int nkb) {
  const int sp = i % ksplit;
  i /= ksplit;
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {  // last group whose prefix is <= i
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= i) lo = mid; else hi = mid - 1;
  }
  TileInfo t;
  t.g = lo;
  const int local = i - s_prefix[lo];
  const int g0 = __ldg(off + lo);
  const int n_g = __ldg(off + lo + 1) - g0;
  const int mt = (n_g + BM - 1) / BM;
  const int per_chunk = MCHUNK * ntn;
  const int chunk = local / per_chunk;
  const int within = local - chunk * per_chunk;
  const int mc = min(MCHUNK, mt - chunk * MCHUNK);
  t.nt = within / mc;
  const int m = chunk * MCHUNK + (within - t.nt * mc);
  t.row0 = g0 + m * BM;
  t.nvalid = min(BM, n_g - m * BM);
  t.sp = sp;
  split_range(sp, ksplit, nkb, t.kb0, t.kb1);
  return t;
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status,
                                                unsigned long long limit_ns) {
  int never = 0;
  mbar_wait(bar, parity, &never, status, limit_ns);
}

template <int MODE, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmY,
                        const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t amax_bar[2][4];   // [tile parity][TMEM lane quarter]
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ __align__(8) uint64_t tinfo_full[2];    // tile list handed from warp 2 to the epilogue
  __shared__ __align__(8) uint64_t tinfo_empty[2];
  __shared__ int4 s_tinfo[2][2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int s_prefix[MAX_GROUPS + 1];
  __shared__ float s_amax[2][2][BM];
  __shared__ int s_abort_store;
  __shared__ uint32_t s_consumed;
  volatile int* s_abort = &s_abort_store;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], EPI_WARPS);
      for (int qq = 0; qq < 4; ++qq) mbar_init(&amax_bar[b][qq], 2);   // the two warps sharing those rows
    }
    mbar_init(&done_bar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tinfo_full[b], 1);
      mbar_init(&tinfo_empty[b], EPI_WARPS);
    }
    s_abort_store = 0;
    s_consumed = 0;
    fence_mbar_init();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) tmem_alloc(&tmem_base_s, TMEM_COLS);
  // the set-up above overlaps the previous kernel; its outputs (offsets, the
  // A operand) and this kernel's outputs are touched only below
  pdl_wait();
  pdl_launch_dependents();

  // Group offsets and the exclusive prefix of the tile counts (every CTA
  // derives the same tile list from the device-side offsets).
  // Offsets that decrease, start below 0 or end beyond the row count would
  // send tiles outside the buffers: the launch then does no work and sets
  // STATUS_BAD_PLAN.
  int bad_plan;
  {
    __shared__ int s_wsum[THREADS / 32];
    const int g = threadIdx.x;
    int v = 0;
    bool bad = false;
    if (g < p.ngroups) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      bad = o0 < 0 || o1 < o0 || (g == p.ngroups - 1 && o1 > p.rows);
      if (!bad) v = ((o1 - o0 + BM - 1) / BM) * p.ntn;
    }
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if ((threadIdx.x & 31) >= off) incl += o;
    }
    if ((threadIdx.x & 31) == 31) s_wsum[threadIdx.x >> 5] = incl;
    bad_plan = __syncthreads_or(bad ? 1 : 0);
    int base = 0;
    for (int j = 0; j < (threadIdx.x >> 5); ++j) base += s_wsum[j];
    if (g < p.ngroups) s_prefix[g] = base + incl - v;
    if (g == p.ngroups - 1) s_prefix[p.ngroups] = base + incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  if (bad_plan && threadIdx.x == 0) set_status(p.status, STATUS_BAD_PLAN);
  const int total = bad_plan ? 0 : s_prefix[p.ngroups] * p.ksplit;
  uint32_t issued = 0;
  uint32_t withheld = 0xFFFFFFFFu;   // the stage a test made the producer skip

  // The two warpgroup kinds run to the end of the kernel on separate paths
  // (each with its own copy of the teardown), so that the register limits
  // set by setmaxnreg hold on every instruction they execute.
  if (warp < FIRST_EPI_WARP) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PRODUCER_REGS));
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
        const TileInfo t = decode_tile(i, s_prefix, p.offsets, p.ngroups, p.ntn, p.ksplit, p.nkb);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u, s_abort, p.status, p.wait_ns)) { ok = false; break; }
          if (p.withhold && blockIdx.x == 0 && it == 0) {   // test only: this stage never arrives
            withheld = it++;
            continue;
          }
          uint8_t* a = smem + s * STAGE_BYTES;
          uint8_t* b = a + A_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], STAGE_BYTES);
          tma_load_2d(a, &tmA, &full_bar[s], kb * BK, t.row0);
          if (MODE == MODE_GATEUP) {
            tma_load_3d(b, &tmB0, &full_bar[s], kb * BK, t.nt * 128, t.g);
            tma_load_3d(b + BH_BYTES, &tmB1, &full_bar[s], kb * BK, t.nt * 128, t.g);
          } else {
            tma_load_3d(b, &tmB0, &full_bar[s], kb * BK, (2 * t.nt) * 128, t.g);
            tma_load_3d(b + BH_BYTES, &tmB0, &full_bar[s], kb * BK, (2 * t.nt + 1) * 128, t.g);
          }
          ++it;
        }
      }
      issued = it;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tb = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < total; i += gridDim.x) {
        int kb0, kb1;
        split_range(i % p.ksplit, p.ksplit, p.nkb, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const uint32_t buf = tb & 1u, tph = (tb >> 1) & 1u;
          if (!mbar_wait(&tempty_bar[buf], tph ^ 1u, s_abort, p.status, p.wait_ns)) { ok = false; break; }
          if (!mbar_wait(&full_bar[s], ph, s_abort, p.status, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint64_t ad = smem_desc_sw128(a_addr);
          const uint64_t bd = smem_desc_sw128(a_addr + A_BYTES);
          const uint32_t d = tmem_base + buf * BN;
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)   // advance 32 bytes of K = 2 in the 16-byte address field
            mma_e4m3(d, ad + uint64_t(2 * k), bd + uint64_t(2 * k), IDESC, k > 0 ? 1u : 0u);
          tc_commit(&empty_bar[s]);
          tc_commit(&tfull_bar[buf]);
          ++it;
          ++tb;
        }
      }
      s_consumed = it;
      tc_commit(&done_bar);                 // all MMAs issued above have completed
      mbar_wait_drain(&done_bar, 0, p.status, p.wait_ns);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile list
    // Decodes this CTA's tiles one ahead of the epilogue into a two-slot
    // ring and pulls each tile's first activation scales and its weight
    // scales into L1, so a tile starts without global-memory latency.
    uint32_t k = 0;
    for (int i = blockIdx.x; i < total; i += gridDim.x, ++k) {
      const uint32_t b = k & 1u, ph = (k >> 1) & 1u;
      bool go = true;
      if (lane == 0) go = mbar_wait(&tinfo_empty[b], ph ^ 1u, s_abort, p.status, p.wait_ns);
      if (!__shfl_sync(0xFFFFFFFFu, go ? 1 : 0, 0)) break;
      const TileInfo t = decode_tile(i, s_prefix, p.offsets, p.ngroups, p.ntn, p.ksplit, p.nkb);
      if (lane == 0) {
        s_tinfo[b][0] = make_int4(t.g, t.nt, t.row0, t.nvalid);
        s_tinfo[b][1] = make_int4(t.kb0, t.kb1, t.sp, 0);
        mbar_arrive(&tinfo_full[b]);   // release: the slot's contents precede the arrival
      }
      for (int r = lane; r < t.nvalid; r += 32)
        for (int kk = t.kb0; kk < t.kb0 + 4 && kk < t.kb1; ++kk) prefetch_l1(p.as + size_t(kk) * p.rows + t.row0 + r);
      for (int kk = t.kb0 + lane; kk < t.kb1; kk += 32) {
        if (MODE == MODE_GATEUP) {
          prefetch_l1(p.ws0 + (size_t(t.g) * p.ws_nb + t.nt) * p.ws_kb + kk);
          prefetch_l1(p.ws1 + (size_t(t.g) * p.ws_nb + t.nt) * p.ws_kb + kk);
        } else {
          for (int hh = 0; hh < 2; ++hh)
            prefetch_l1(p.ws0 + (size_t(t.g) * p.ws_nb + min(2 * t.nt + hh, p.ws_nb - 1)) * p.ws_kb + kk);
        }
      }
    }
  }
  // ---------------------------------------------------- teardown (warpgroup 0)
  asm volatile("bar.sync 0;" ::: "memory");
  if (warp == 0 && lane == 0) {
    // copies issued but never consumed (only after an abort) must land first
    for (uint32_t j = s_consumed; j < issued; ++j)
      if (j != withheld) mbar_wait_drain(&full_bar[j % STAGES], (j / STAGES) & 1u, p.status, p.wait_ns);
  }
  tc_fence_before();
  asm volatile("bar.sync 0;" ::: "memory");
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(EPILOGUE_REGS));
    // ------------------------------------------------------------ epilogue
    const int ew = warp - FIRST_EPI_WARP;
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int half = ew >> 2;        // column half of the tile (one per warpgroup)
    const int r_in = q * 32 + lane;  // row within the tile
    uint32_t tb = 0;
    uint32_t tile_iter = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok && i < total; i += gridDim.x, ++tile_iter) {
      TileInfo t;
      {  // the tile, decoded ahead by warp 2
        const uint32_t b = tile_iter & 1u;
        if (!mbar_wait(&tinfo_full[b], (tile_iter >> 1) & 1u, s_abort, p.status, p.wait_ns)) break;
        const int4 v = s_tinfo[b][0], u = s_tinfo[b][1];
        t.g = v.x;
        t.nt = v.y;
        t.row0 = v.z;
        t.nvalid = v.w;
        t.kb0 = u.x;
        t.kb1 = u.y;
        t.sp = u.z;
        __syncwarp();
        if (lane == 0) mbar_arrive(&tinfo_empty[b]);
      }
      const bool warp_active = q * 32 < t.nvalid;
      const bool valid = r_in < t.nvalid;
      const int row = t.row0 + r_in;
      const float* w0;
      const float* w1;
      int nb = 0;
      if (MODE == MODE_GATEUP) {
        w0 = p.ws0 + (size_t(t.g) * p.ws_nb + t.nt) * p.ws_kb;
        w1 = p.ws1 + (size_t(t.g) * p.ws_nb + t.nt) * p.ws_kb;
      } else {
        nb = 2 * t.nt + half;
        w0 = p.ws0 + (size_t(t.g) * p.ws_nb + min(nb, p.ws_nb - 1)) * p.ws_kb;
        w1 = w0;
      }
      float acc[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.0f;

      // Scales stay off the critical path: lane l holds the weight scales
      // of K block (window + l), broadcast by a shuffle; the row's
      // activation scales are prefetched four K blocks ahead.
      // (kr counts the tile's K blocks from its split's first, t.kb0)
      float wr0 = 0.0f, wr1 = 0.0f;
      const size_t ast = size_t(p.rows);
      const float* asp = p.as + size_t(t.kb0) * ast + row;
      const int nk = t.kb1 - t.kb0;
      float pf0 = 0.0f, pf1 = 0.0f, pf2 = 0.0f, pf3 = 0.0f;
      if (valid) {
        pf0 = __ldg(asp);
        if (nk > 1) pf1 = __ldg(asp + ast);
        if (nk > 2) pf2 = __ldg(asp + 2 * ast);
        if (nk > 3) pf3 = __ldg(asp + 3 * ast);
      }

      for (int kr = 0; kr < nk; ++kr) {
        const uint32_t buf = tb & 1u, tph = (tb >> 1) & 1u;
        if ((kr & 31) == 0) {
          const int k = t.kb0 + kr + lane;
          wr0 = k < t.kb1 ? __ldg(w0 + k) : 0.0f;
          wr1 = k < t.kb1 ? __ldg(w1 + k) : 0.0f;
        }
        const float sa = pf0;
        pf0 = pf1;
        pf1 = pf2;
        pf2 = pf3;
        pf3 = (valid && kr + 4 < nk) ? __ldg(asp + size_t(kr + 4) * ast) : 0.0f;
        const float f0 = __shfl_sync(0xFFFFFFFFu, wr0, kr & 31) * sa;
        const float f1 = __shfl_sync(0xFFFFFFFFu, wr1, kr & 31) * sa;
        if (!mbar_wait(&tfull_bar[buf], tph, s_abort, p.status, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (warp_active) {
          const uint32_t tbase = tmem_base + (uint32_t(q * 32) << 16) + buf * BN;
#pragma unroll
          for (int c = 0; c < 4; c += 2) {   // two 32-column chunks per TMEM round trip
            const uint32_t col = (MODE == MODE_GATEUP) ? uint32_t((c >> 1) * 128 + half * 64)
                                                       : uint32_t(half * 128 + c * 32);
            float va[32], vb[32];
            tmem_ld32(tbase + col, va);
            tmem_ld32(tbase + col + 32, vb);
            tmem_ld_wait();
            if (c == 2) {   // the buffer is in registers: hand it back before the last FMAs
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty_bar[buf]);
            }
            const float f = (MODE == MODE_GATEUP && c >= 2) ? f1 : f0;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              ffma2(acc[c * 32 + j], acc[c * 32 + j + 1], va[j], va[j + 1], f);
              ffma2(acc[c * 32 + 32 + j], acc[c * 32 + 33 + j], vb[j], vb[j + 1], f);
            }
          }
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty_bar[buf]);
        }
        ++tb;
      }
      if (!ok) break;

      if (EPI == EPI_SPLIT) {
        // this split's promoted FP32 partial; the reduce kernel adds the splits
        if (valid && nb < p.nb_count) {
          float* dst = p.part + (size_t(t.sp) * p.rows + row) * p.ld_y + nb * 128;
#pragma unroll
          for (int v = 0; v < 32; ++v)
            *reinterpret_cast<float4*>(dst + 4 * v) = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
        }
      } else if (EPI == EPI_F32) {
        if (valid) {
          float* dst = p.out + size_t(row) * p.ld_out;
          if (MODE == MODE_GATEUP) {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              dst[t.nt * 256 + half * 64 + j] = acc[j];
              dst[t.nt * 256 + 128 + half * 64 + j] = acc[64 + j];
            }
          } else if (nb < p.nb_count) {
#pragma unroll
            for (int j = 0; j < 128; ++j) dst[nb * 128 + j] = acc[j];
          }
        }
      } else if (MODE == MODE_GATEUP) {
        // h = silu(G) * U for this thread's 64 channels, then the row's
        // 128-channel amax across the two column halves.
        float amax = 0.0f;
        if (warp_active) {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            // silu(g) * u = g * u / (1 + 2^(-g log2 e)): the exponential on
            // the special-function unit, the reciprocal on the FMA pipe
            // (rcp2_newton), so the unit does one operation per channel; the
            // exponent is capped at 126 so that the denominator stays finite
            // (gates below -87 give |h| < 2^-120 either way)
            const float g0 = acc[j], g1 = acc[j + 1];
            const float d0 = 1.0f + ex2_approx(fminf(-1.4426950408889634f * g0, 126.0f));
            const float d1 = 1.0f + ex2_approx(fminf(-1.4426950408889634f * g1, 126.0f));
            float r0, r1;
            rcp2_newton(d0, d1, r0, r1);
            const float h0 = g0 * acc[64 + j] * r0, h1 = g1 * acc[65 + j] * r1;
            acc[j] = h0;
            acc[j + 1] = h1;
            amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
          }
        }
        const uint32_t xb = tile_iter & 1u;
        s_amax[xb][half][r_in] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&amax_bar[xb][q]);
        if (!mbar_wait(&amax_bar[xb][q], (tile_iter >> 1) & 1u, s_abort, p.status, p.wait_ns)) { ok = false; break; }
        amax = fmaxf(amax, s_amax[xb][half ^ 1][r_in]);
        if (valid) {
          uint32_t pk[16];
          float s = 0.0f;
          if (amax > 0.0f) {
            // same scale rule as the activations (s = amax/448, an IEEE
            // divide); h/s is taken as h times the correctly rounded 1/s,
            // within one fp32 ulp of the quotient
            s = __fdiv_rn(amax, 448.0f);
            const float inv = __frcp_rn(s);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t lo = e4m3x2(acc[4 * j] * inv, acc[4 * j + 1] * inv);
              const uint32_t hi = e4m3x2(acc[4 * j + 2] * inv, acc[4 * j + 3] * inv);
              pk[j] = lo | (hi << 16);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) pk[j] = 0u;
          }
          if (q * 32 + 32 <= t.nvalid) {
            // 32 full rows: this warp's 64 channels into its 64-byte-swizzled
            // box (16-byte chunk c of row r at chunk c ^ ((r / 2) % 4)), then
            // one asynchronous bulk tensor store
            uint8_t* stg = smem + STAGES * STAGE_BYTES + ew * stg_warp_bytes(MODE);
            if (lane == 0) bulk_wait_read0();   // the previous store has read the box
            __syncwarp();
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(stg + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) =
                  make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, stg, t.nt * 128 + half * 64, t.row0 + q * 32);
              bulk_commit();
            }
          } else {
            // the group's last rows (a partial warp): direct stores, so that
            // no row of the next group is written
            uint8_t* dst = p.h + size_t(row) * p.ld_h + t.nt * 128 + half * 64;
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(dst + 16 * v) = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
          if (half == 0) p.hs[size_t(t.nt) * p.rows + row] = s;
        }
      } else if (warp_active && nb < p.nb_count) {
        if (q * 32 + 32 <= t.nvalid) {
          // 32 full rows: bf16 into this warp's 128-byte-swizzled staging box
          // (16-byte chunk c of row r at chunk c ^ (r % 8)), then one bulk
          // tensor store per 64 columns; the copy runs while the warp moves on
          uint8_t* stg = smem + STAGES * STAGE_BYTES + ew * stg_warp_bytes(MODE);
          uint8_t* rowp = stg + lane * 128;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (lane == 0) bulk_wait_read0();   // the previous store has read the box
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float* v = acc + 64 * j + 8 * c;
              *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(bf16x2_rn(v[0], v[1]), bf16x2_rn(v[2], v[3]), bf16x2_rn(v[4], v[5]), bf16x2_rn(v[6], v[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, stg, nb * 128 + 64 * j, t.row0 + q * 32);
              bulk_commit();
            }
          }
        } else if (valid) {
          // the group's last rows (a partial warp): direct stores, so that no
          // row of the next group is written
          uint16_t* dst = p.y + size_t(row) * p.ld_y + nb * 128;
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const float* a8 = acc + 8 * v;
            *reinterpret_cast<uint4*>(dst + 8 * v) =
                make_uint4(bf16x2_rn(a8[0], a8[1]), bf16x2_rn(a8[2], a8[3]), bf16x2_rn(a8[4], a8[5]), bf16x2_rn(a8[6], a8[7]));
          }
        }
      }
    }

    // ------------------------------------------------ teardown (epilogue side)
    if (lane == 0) bulk_wait0();   // bulk stores complete before the CTA exits
    asm volatile("bar.sync 0;" ::: "memory");
    tc_fence_before();
    asm volatile("bar.sync 0;" ::: "memory");
  }
}

template <int MODE, int EPI>
cudaError_t launch_gemm(const moe_layer_s* L, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                        const CUtensorMap& tmB1, const CUtensorMap& tmY, const GemmArgs& args, cudaStream_t st) {
  constexpr int SMEM_DYN = smem_dyn(MODE);
  static std::atomic<bool> configured[kMaxDevices];   // the attribute is per device
  cudaError_t ce = once_per_device(configured, []() {
    // setmaxnreg.inc waits until the registers it asks for are free; they
    // come only from this CTA's launch allocation, so refuse to launch a
    // build whose register count cannot fund the split.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, grouped_gemm_kernel<MODE, EPI>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * THREADS < 128 * PRODUCER_REGS + 256 * EPILOGUE_REGS) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(grouped_gemm_kernel<MODE, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_DYN);
  });
  if (ce != cudaSuccess) return ce;
  GemmArgs a = args;
  a.wait_ns = kWaitLimitNs;
  a.withhold = 0;
  if (L->test_stall_ns) {   // a test armed a stall for this one launch
    a.wait_ns = L->test_stall_ns;
    a.withhold = 1;
    L->test_stall_ns = 0;
  }
  // upper bound on the number of tiles: every group may add one partial row tile
  const long long bound = (static_cast<long long>(a.rows) / BM + a.ngroups) * a.ntn * a.ksplit;
  const int grid = int(bound < L->num_sms ? bound : L->num_sms);
  if (grid <= 0) return cudaSuccess;
  return launch_pdl(grouped_gemm_kernel<MODE, EPI>, dim3(grid), dim3(THREADS), SMEM_DYN, st, tmA, tmB0, tmB1, tmY, a);
}

// y = bf16(sum over the splits s = 0..ks-1 of part[s]), 8 columns per thread.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, int ks, size_t n,
                                                            uint16_t* __restrict__ y) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t i = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = 0.0f;
  for (int s = 0; s < ks; ++s) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(part + s * n + i));
    const float4 b = __ldg(reinterpret_cast<const float4*>(part + s * n + i + 4));
    v[0] += a.x;
    v[1] += a.y;
    v[2] += a.z;
    v[3] += a.w;
    v[4] += b.x;
    v[5] += b.y;
    v[6] += b.z;
    v[7] += b.w;
  }
  *reinterpret_cast<uint4*>(y + i) =
      make_uint4(bf16x2_rn(v[0], v[1]), bf16x2_rn(v[2], v[3]), bf16x2_rn(v[4], v[5]), bf16x2_rn(v[6], v[7]));
}

}  // namespace

// K splits of the down GEMM for `rows` rows: more than one only when the
// batch has fewer output tiles than half the SMs (a layer with one or two
// groups at small batches), at least 4 K blocks per split.
int down_ksplit(const moe_layer_s* L, int rows) {
  const int ntn = (L->HB + 1) / 2;
  const long long tiles = (static_cast<long long>(rows) / BM + L->E + L->S) * ntn;   // groups with rows
  if (!L->splitk || rows > kSplitRows || tiles * 2 > L->num_sms) return 1;
  int ks = int(L->num_sms / tiles);
  ks = ks < kSplitMax ? ks : kSplitMax;
  return ks < L->FB / 4 ? ks : L->FB / 4;
}

static GemmArgs gateup_args(const moe_layer_s* L, const int32_t* offsets, int rows, const float* xs) {
  GemmArgs a = {};
  a.offsets = offsets;
  a.ngroups = L->E + 1;
  a.ntn = L->FB;
  a.nkb = L->HB;
  a.rows = rows;
  a.as = xs;
  a.ws0 = L->w.s_gate;
  a.ws1 = L->w.s_up;
  a.ws_nb = L->FB;
  a.ws_kb = L->HB;
  a.nb_count = L->FB;
  a.ksplit = 1;
  a.status = L->status;
  return a;
}

static GemmArgs down_args(const moe_layer_s* L, const int32_t* offsets, int rows, const float* hs) {
  GemmArgs a = {};
  a.offsets = offsets;
  a.ngroups = L->E + 1;
  a.ntn = (L->HB + 1) / 2;
  a.nkb = L->FB;
  a.rows = rows;
  a.as = hs;
  a.ws0 = L->w.s_down;
  a.ws1 = L->w.s_down;
  a.ws_nb = L->HB;
  a.ws_kb = L->FB;
  a.nb_count = L->HB;
  a.ksplit = 1;
  a.status = L->status;
  return a;
}

cudaError_t launch_gate_up(const moe_layer_s* L, const uint8_t* xq, const float* xs, const int32_t* offsets, int rows,
                           uint8_t* h, float* hs, cudaStream_t st) {
  CUtensorMap tmX, tmHst;
  if (!encode_tmap_u8(&tmX, xq, L->H, rows, 1, L->H, 0)) return cudaErrorInvalidValue;
  if (!encode_tmap_store(&tmHst, false, h, L->ld_hh, rows, L->ld_hh)) return cudaErrorInvalidValue;
  GemmArgs a = gateup_args(L, offsets, rows, xs);
  a.h = h;
  a.hs = hs;
  a.ld_h = L->ld_hh;
  return launch_gemm<MODE_GATEUP, EPI_FUSED>(L, tmX, L->tm_gate, L->tm_up, tmHst, a, st);
}

cudaError_t launch_down(const moe_layer_s* L, const uint8_t* h, const float* hs, const int32_t* offsets, int rows,
                        uint16_t* y, cudaStream_t st) {
  CUtensorMap tmH;
  if (!encode_tmap_u8(&tmH, h, L->F, rows, 1, L->ld_hh, 0)) return cudaErrorInvalidValue;
  CUtensorMap tmY;
  if (!encode_tmap_store(&tmY, true, y, L->H, rows, size_t(L->H) * 2)) return cudaErrorInvalidValue;
  GemmArgs a = down_args(L, offsets, rows, hs);
  a.y = y;
  a.ld_y = L->H;
  const int ks = down_ksplit(L, rows);
  if (ks < 2) return launch_gemm<MODE_DOWN, EPI_FUSED>(L, tmH, L->tm_down, L->tm_down, tmY, a, st);
  a.ksplit = ks;
  a.part = L->splitk;
  cudaError_t e = launch_gemm<MODE_DOWN, EPI_SPLIT>(L, tmH, L->tm_down, L->tm_down, tmY, a, st);
  if (e != cudaSuccess) return e;
  const size_t n = size_t(rows) * L->H;
  return launch_pdl(splitk_reduce_kernel, dim3(unsigned((n / 8 + 255) / 256)), dim3(256), 0, st,
                    static_cast<const float*>(L->splitk), ks, n, y);
}

cudaError_t launch_test_gemm_f32(const moe_layer_s* L, int which, const uint8_t* a_ptr, const float* as,
                                 const int32_t* offsets, int T, float* out, cudaStream_t st) {
  const int rows = T * (L->K + L->S);
  CUtensorMap tmA;
  if (which == 0) {
    if (!encode_tmap_u8(&tmA, a_ptr, L->H, rows, 1, L->H, 0)) return cudaErrorInvalidValue;
    GemmArgs a = gateup_args(L, offsets, rows, as);
    a.out = out;
    a.ld_out = 2 * L->FB * 128;
    return launch_gemm<MODE_GATEUP, EPI_F32>(L, tmA, L->tm_gate, L->tm_up, tmA, a, st);
  }
  if (!encode_tmap_u8(&tmA, a_ptr, L->F, rows, 1, L->ld_hh, 0)) return cudaErrorInvalidValue;
  GemmArgs a = down_args(L, offsets, rows, as);
  a.out = out;
  a.ld_out = L->H;
  return launch_gemm<MODE_DOWN, EPI_F32>(L, tmA, L->tm_down, L->tm_down, tmA, a, st);
}

}  // namespace moe

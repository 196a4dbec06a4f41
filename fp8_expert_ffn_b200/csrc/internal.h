// Host-side layer handle and the launchers each .cu file provides.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "../../include/moe.h"

struct moe_layer_s {
  moe_layer_desc d;
  moe_weights w;
  int H, E, K, F;
  int S;         // shared experts (0 or 1); a token fills K + S rows
  int HB;        // H / 128
  int FB;        // ceil(F / 128)
  int ld_hh;     // row stride of the quantised SwiGLU output h: FB * 128
  int device;
  int num_sms;
  bool has_experts;  // false: a routing-only handle (route, permute, combine)
  uint32_t* status;  // device status word
  uint16_t* router_split;  // [3][E][H] bf16 terms of router_w (library-owned)
  float* router_bias;      // [E] selection-only bias (library-owned copy) or null
  float* splitk;           // [kSplitMax][kSplitRows][H] fp32 partials of the split down GEMM
  CUtensorMap tm_router;   // over router_split, box 64 x 256 x 1
  CUtensorMap tm_gate;  // [E+1][F][ld_h] E4M3, box 128 x 128 x 1
  CUtensorMap tm_up;
  CUtensorMap tm_down;  // [E+1][H][ld_f] E4M3, box 128 x 128 x 1
  // test only (moe_test_inject_stall): when nonzero, the next grouped-GEMM
  // launch withholds one pipeline stage and uses this wait limit
  mutable unsigned long long test_stall_ns;
};

// Exchange buffers of one rank for the expert-parallel dispatch and combine
// over peer memory (ep.cu): one device allocation holding this rank's
// receive buffers and output rows, and device tables of every rank's
// buffers (a peer's through a CUDA IPC mapping, or a buffer of this process
// when the ranks are emulated on one GPU).
struct moe_ep_comm_s {
  int device;
  int rank, ranks;
  int cap;             // rows of each buffer
  int H, HB;
  void* base;          // this rank's allocation
  size_t bytes;
  size_t off_s, off_y; // byte offsets of the scales and of y in an allocation
  uint64_t* d_peer_q;  // [ranks] device table: codes [cap][H] u8
  uint64_t* d_peer_s;  // [ranks] scales [HB][cap] f32
  uint64_t* d_peer_y;  // [ranks] rows [cap][H] bf16
  void* opened[64];    // IPC mappings to close (by rank), null if none
  bool connected;
};

namespace moe {

// Workspace carving shared by every entry point.
struct Scratch {
  // route
  float* route_partial;   // [S][T][E]
  // permute
  uint32_t* bitmap;       // [E][W]
  uint32_t* wprefix;      // [E][W]
  int32_t* counts;        // [E] + 1 word: the count kernel's completion counter
  // expert ffn
  uint8_t* h;             // [rows][ld_hh]
  float* hs;              // [FB][rows]
  // forward intermediates
  int32_t* idx;           // [T][K]
  float* topw;            // [T][K]
  int32_t* offsets;       // [E+2]
  int32_t* perm;          // [rows]
  int32_t* inv;           // [T][K]
  uint8_t* xq;            // [rows][H]
  float* xs;              // [HB][rows]
  uint16_t* y;            // [rows][H]
  size_t total;
};

int route_splits(const moe_layer_s* L, int T);
Scratch carve(const moe_layer_s* L, int T, void* base);

cudaError_t launch_route(const moe_layer_s* L, const uint16_t* x, int T, int ldx, int32_t* idx, float* w,
                         float* logits, float* partial, cudaStream_t st);
cudaError_t launch_permute(const moe_layer_s* L, const uint16_t* x, int T, int ldx, const int32_t* idx,
                           int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs,
                           const Scratch& s, cudaStream_t st);
// Kernels launch_permute issues for T tokens: 2 when the token bitmap fits
// one CTA's shared memory (one plan kernel + the gather), else 4.
int permute_kernels(const moe_layer_s* L, int T);
// Limits of the allocation-free permutation (moe_permute_noalloc).
constexpr int kNoAllocMaxTokens = MOE_NOALLOC_MAX_TOKENS;
constexpr int kNoAllocMaxExperts = 256;
// Split-K of the down GEMM (batches with fewer output tiles than half the
// SMs): at most kSplitMax splits over at most kSplitRows rows.
constexpr int kSplitMax = 8;
constexpr int kSplitRows = 256;
int down_ksplit(const moe_layer_s* L, int rows);
cudaError_t launch_permute_noalloc(const moe_layer_s* L, const uint16_t* x, int T, int ldx, const int32_t* idx,
                                   int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs,
                                   cudaStream_t st);
// rows: the permuted row count (the group stride of the scale arrays)
cudaError_t launch_gate_up(const moe_layer_s* L, const uint8_t* xq, const float* xs, const int32_t* offsets, int rows,
                           uint8_t* h, float* hs, cudaStream_t st);
cudaError_t launch_down(const moe_layer_s* L, const uint8_t* h, const float* hs, const int32_t* offsets, int rows,
                        uint16_t* y, cudaStream_t st);
// Expert parallelism over peer memory: the permutation plan alone (bitmap,
// prefixes, offsets), the dispatch (quantise and write each routed row into
// its owner's receive buffer, the shared rows into this rank's; the owner's
// group offsets) and the combine (read the rows back from the owners' y).
constexpr int kEpMaxRanks = 64;
cudaError_t launch_ep_plan(const moe_layer_s* L, const int32_t* idx, int T, int32_t* offsets, const Scratch& s,
                           cudaStream_t st);
cudaError_t launch_ep_dispatch(const moe_layer_s* L, const moe_ep_comm_s* c, const uint16_t* x, int T, int ldx,
                               const int32_t* idx, const int32_t* all_off, int32_t* inv_ep, int32_t* goff,
                               const Scratch& s, cudaStream_t st);
cudaError_t launch_ep_combine(const moe_layer_s* L, const moe_ep_comm_s* c, const int32_t* idx, const int32_t* inv_ep,
                              const float* w, const int32_t* goff, int T, uint16_t* out, int ldo, cudaStream_t st);
// Expert parallelism (ep.cu): at most kEpMaxSegments = ranks x local experts.
constexpr int kEpMaxSegments = 2048;
cudaError_t launch_ep_pack_scales(const moe_layer_s* L, const float* xs, int T, float* out, cudaStream_t st);
cudaError_t launch_ep_regroup(const moe_layer_s* L, int P, const int32_t* cnt, int N, const uint8_t* recv_q,
                              const float* recv_s, const uint8_t* own_q, const float* own_s, int T, uint8_t* out_q,
                              float* out_s, int32_t* out_offsets, cudaStream_t st);
cudaError_t launch_ep_unregroup(const moe_layer_s* L, int P, const int32_t* cnt, int N, const uint16_t* y_g, int T,
                                uint16_t* y_send, uint16_t* y_own, cudaStream_t st);
cudaError_t launch_test_gemm_f32(const moe_layer_s* L, int which, const uint8_t* a, const float* as,
                                 const int32_t* offsets, int T, float* out, cudaStream_t st);
cudaError_t launch_combine(const moe_layer_s* L, const uint16_t* y, const int32_t* inv, const float* w, int T,
                           uint16_t* out, int ldo, cudaStream_t st);

// TMA descriptor for a row-major byte matrix [rows][inner] with row stride
// `ld` bytes, 128 x 128 boxes, 128-byte swizzle (3-D when depth > 1).
// Store map of a [rows][inner] matrix for the GEMM epilogues: bf16, boxes of
// 64 columns x 32 rows with 128-byte swizzle (the down GEMM's y); u8, boxes
// of 64 columns x 32 rows with 64-byte swizzle (the gate/up GEMM's h).
// Launch with programmatic dependent launch allowed: the kernel's CTAs may
// start while the previous kernel on the stream is finishing. Every kernel of
// the library calls pdl_wait() before it touches memory that an earlier
// kernel writes or reads, and pdl_launch_dependents() right after, so each
// kernel's set-up overlaps the tail of the one before.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Kernel attributes (the dynamic shared-memory limit) are set per device:
// once_per_device runs `setup` the first time it is called with each device
// current and records success in done[device]; a failed setup is retried on
// the next call. Safe to call from several host threads.
constexpr int kMaxDevices = 64;
std::mutex& device_setup_mutex();
template <typename F>
cudaError_t once_per_device(std::atomic<bool>* done, F setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(device_setup_mutex());
  if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
  return e;
}

bool encode_tmap_store(CUtensorMap* tm, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t ld_bytes);
bool encode_tmap_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                    uint64_t ld, uint64_t depth_stride);
// Same for bf16 (box 64 x 128 elements = 128 bytes of K per row) or u8.
bool encode_tmap(CUtensorMap* tm, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                 uint64_t ld_bytes, uint64_t depth_stride_bytes, bool force3d = false, uint32_t box_rows = 128);
// Experts per router tile (the router weight map's box height).
constexpr uint32_t kRouterExperts = 128;

// Router weight split into three bf16 terms (hi + mid + lo == w exactly for
// normal-range fp32 w), [3][E][H]; written once at layer creation.
cudaError_t launch_router_split(const float* w, int E, int H, uint16_t* out, cudaStream_t st);

}  // namespace moe

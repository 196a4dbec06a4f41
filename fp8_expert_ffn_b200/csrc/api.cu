// C ABI of the FP8 MoE-layer library: argument validation, the layer handle,
// workspace carving and the composition of the stages. No entry point
// allocates device memory except moe_layer_create (a 4-byte status word and
// the router weight's bf16 split).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <new>

#include "internal.h"

namespace moe {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_device_setup_mutex;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

std::mutex& device_setup_mutex() { return g_device_setup_mutex; }

bool encode_tmap(CUtensorMap* tm, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                 uint64_t ld_bytes, uint64_t depth_stride_bytes, bool force3d, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, depth};
  cuuint64_t strides[2] = {ld_bytes, depth_stride_bytes};
  cuuint32_t box[3] = {bf16 ? 64u : 128u, box_rows, 1};   // 128 bytes of K per box row
  cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = (depth > 1 || force3d) ? 3 : 2;
  CUresult r = fn(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, rank,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_store(CUtensorMap* tm, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t ld_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {ld_bytes};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows, uint64_t depth, uint64_t ld,
                    uint64_t depth_stride) {
  return encode_tmap(tm, false, base, inner, rows, depth, ld, depth_stride);
}

Scratch carve(const moe_layer_s* L, int T, void* base) {
  Scratch s = {};
  const int K = L->K, E = L->E;
  const size_t rows = size_t(T) * (K + L->S);
  const size_t W = (size_t(T) + 31) / 32;
  char* b = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    off = align_up(off, 256);
    void* p = b ? b + off : nullptr;
    off += bytes;
    return p;
  };
  s.route_partial = static_cast<float*>(take(sizeof(float) * size_t(route_splits(L, T)) * T * E));
  s.bitmap = static_cast<uint32_t*>(take(sizeof(uint32_t) * E * W));
  s.wprefix = static_cast<uint32_t*>(take(sizeof(uint32_t) * E * W));
  s.counts = static_cast<int32_t*>(take(sizeof(int32_t) * (E + 1)));   // + the count kernel's completion counter
  if (!L->has_experts) {   // a routing-only handle: route and permutation scratch only
    s.total = align_up(off, 256);
    return s;
  }
  s.h = static_cast<uint8_t*>(take(rows * L->ld_hh));
  s.hs = static_cast<float*>(take(sizeof(float) * L->FB * rows));
  s.idx = static_cast<int32_t*>(take(sizeof(int32_t) * size_t(T) * K));
  s.topw = static_cast<float*>(take(sizeof(float) * size_t(T) * K));
  s.offsets = static_cast<int32_t*>(take(sizeof(int32_t) * (E + 2)));
  s.perm = static_cast<int32_t*>(take(sizeof(int32_t) * rows));
  s.inv = static_cast<int32_t*>(take(sizeof(int32_t) * size_t(T) * K));
  s.xq = static_cast<uint8_t*>(take(rows * L->H));
  s.xs = static_cast<float*>(take(sizeof(float) * L->HB * rows));
  s.y = static_cast<uint16_t*>(take(sizeof(uint16_t) * rows * L->H));
  s.total = align_up(off, 256);
  return s;
}

}  // namespace moe

using namespace moe;

namespace {

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status check_x(const moe_layer_s* L, const uint16_t* x, int ldx) {
  if (!x) return MOE_ERR_INVALID_ARG;
  if (ldx < L->H) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || (size_t(ldx) * 2) % 16 != 0) return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status check_ws(const moe_layer_s* L, int T, void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MOE_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_MISALIGNED;
  if (ws_bytes < carve(L, T, nullptr).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

constexpr int kMaxT = 1 << 20;

}  // namespace

#pragma GCC visibility push(default)
extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case MOE_ERR_UNSUPPORTED: return "unsupported layer shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_DEVICE: return "a kernel reported bad data or a timed-out wait";
  }
  return "unknown status";
}

moe_status moe_layer_create(const moe_layer_desc* d, const moe_weights* w, moe_layer_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d || !w) return MOE_ERR_INVALID_ARG;
  if (d->hidden <= 0 || d->n_routed <= 0 || d->top_k <= 0 || d->ffn <= 0) return MOE_ERR_INVALID_ARG;
  if (d->hidden % 128 != 0 || d->hidden > 16384 || d->n_routed > 256 || d->n_shared < 0 || d->n_shared > 1 ||
      d->top_k > 8 || d->top_k > d->n_routed || d->ffn > 16384 || (d->n_shared == 1 && d->shared_ffn != d->ffn) ||
      d->block != 128 || (d->norm_topk != 0 && d->norm_topk != 1))
    return MOE_ERR_UNSUPPORTED;
  if (d->n_group < 1 || d->n_group > 32 || d->n_routed % d->n_group != 0 || d->topk_group < 1 ||
      d->topk_group > d->n_group || d->top_k > d->topk_group * (d->n_routed / d->n_group))
    return MOE_ERR_UNSUPPORTED;
  if (!(d->routed_scaling == d->routed_scaling)) return MOE_ERR_INVALID_ARG;
  if (!w->router_w) return MOE_ERR_INVALID_ARG;
  // all six expert arrays, or none (a routing-only handle: route, permute, combine)
  const void* experts[] = {w->w_gate, w->w_up, w->w_down, w->s_gate, w->s_up, w->s_down};
  int given = 0;
  for (const void* p : experts) given += p != nullptr;
  if (given != 0 && given != 6) return MOE_ERR_INVALID_ARG;
  const bool has_experts = given == 6;
  if (has_experts) {
    if (w->ld_h < d->hidden || w->ld_f < d->ffn) return MOE_ERR_INVALID_ARG;
    if (w->ld_h % 16 != 0 || w->ld_f % 16 != 0) return MOE_ERR_MISALIGNED;
    for (const void* p : experts)
      if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  if (!aligned16(w->router_w)) return MOE_ERR_MISALIGNED;
  if (w->router_bias && !aligned16(w->router_bias)) return MOE_ERR_MISALIGNED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10) return MOE_ERR_UNSUPPORTED;

  moe_layer_s* L = new (std::nothrow) moe_layer_s();
  if (!L) return MOE_ERR_CUDA;
  L->d = *d;
  L->w = *w;
  L->H = d->hidden;
  L->E = d->n_routed;
  L->K = d->top_k;
  L->S = d->n_shared;
  L->F = d->ffn;
  L->HB = d->hidden / 128;
  L->FB = (d->ffn + 127) / 128;
  L->ld_hh = L->FB * 128;
  L->device = dev;
  L->num_sms = prop.multiProcessorCount;
  L->has_experts = has_experts;
  // weight maps are always 3-D (expert index = z), even with a single expert
  const uint64_t E1 = uint64_t(L->E) + L->S;
  if (has_experts &&
      (!encode_tmap(&L->tm_gate, false, w->w_gate, L->H, L->F, E1, w->ld_h, uint64_t(L->F) * w->ld_h, true) ||
       !encode_tmap(&L->tm_up, false, w->w_up, L->H, L->F, E1, w->ld_h, uint64_t(L->F) * w->ld_h, true) ||
       !encode_tmap(&L->tm_down, false, w->w_down, L->F, L->H, E1, w->ld_f, uint64_t(L->H) * w->ld_f, true))) {
    delete L;
    return MOE_ERR_CUDA;
  }
  const size_t split_bytes = 3 * size_t(L->E) * L->H * sizeof(uint16_t);
  bool ok = cudaMalloc(&L->status, sizeof(uint32_t)) == cudaSuccess;
  ok = ok && cudaMalloc(&L->router_split, split_bytes) == cudaSuccess;
  if (has_experts)
    ok = ok && cudaMalloc(&L->splitk, sizeof(float) * size_t(kSplitMax) * kSplitRows * L->H) == cudaSuccess;
  ok = ok && cudaMemset(L->status, 0, sizeof(uint32_t)) == cudaSuccess;
  if (w->router_bias) {
    ok = ok && cudaMalloc(&L->router_bias, sizeof(float) * L->E) == cudaSuccess;
    ok = ok && cudaMemcpy(L->router_bias, w->router_bias, sizeof(float) * L->E, cudaMemcpyDeviceToDevice) ==
                   cudaSuccess;
  }
  ok = ok && launch_router_split(w->router_w, L->E, L->H, L->router_split, nullptr) == cudaSuccess;
  ok = ok && cudaDeviceSynchronize() == cudaSuccess;
  ok = ok && encode_tmap(&L->tm_router, true, L->router_split, L->H, L->E, 3, uint64_t(L->H) * 2,
                         uint64_t(L->E) * L->H * 2, false, kRouterExperts);
  if (!ok) {
    cudaFree(L->status);
    cudaFree(L->router_split);
    cudaFree(L->router_bias);
    cudaFree(L->splitk);
    delete L;
    return MOE_ERR_CUDA;
  }
  *out = L;
  return MOE_OK;
}

moe_status moe_layer_destroy(moe_layer_t L) {
  if (!L) return MOE_OK;
  cudaError_t e = cudaFree(L->status);
  cudaError_t e2 = cudaFree(L->router_split);
  const cudaError_t e4 = cudaFree(L->splitk);
  if (e2 == cudaSuccess) e2 = e4;
  if (L->router_bias) {
    const cudaError_t e3 = cudaFree(L->router_bias);
    if (e2 == cudaSuccess) e2 = e3;
  }
  delete L;
  return from_cuda(e != cudaSuccess ? e : e2);
}

size_t moe_workspace_size(moe_layer_t L, int T) {
  if (!L || T < 0 || T > kMaxT) return 0;
  return carve(L, T, nullptr).total;
}

moe_status moe_route(moe_layer_t L, const uint16_t* x, int T, int ldx, int32_t* idx, float* w, float* logits,
                     void* ws, size_t ws_bytes, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_status s;
  if ((s = check_x(L, x, ldx)) != MOE_OK) return s;
  if (!idx || !w) return MOE_ERR_INVALID_ARG;
  if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
  Scratch sc = carve(L, T, ws);
  return from_cuda(launch_route(L, x, T, ldx, idx, w, logits, sc.route_partial, static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(moe_layer_t L, const uint16_t* x, int T, int ldx, const int32_t* idx, int32_t* offsets,
                       int32_t* perm, int32_t* inv, uint8_t* xq, float* xs, void* ws, size_t ws_bytes,
                       void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_status s;
  if ((s = check_x(L, x, ldx)) != MOE_OK) return s;
  if (!idx || !offsets || !perm || !inv || !xq || !xs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq)) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
  Scratch sc = carve(L, T, ws);
  return from_cuda(
      launch_permute(L, x, T, ldx, idx, offsets, perm, inv, xq, xs, sc, static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute_noalloc(moe_layer_t L, const uint16_t* x, int T, int ldx, const int32_t* idx,
                               int32_t* offsets, int32_t* perm, int32_t* inv, uint8_t* xq, float* xs, void* stream) {
  if (!L || T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (T > kNoAllocMaxTokens || L->E > kNoAllocMaxExperts) return MOE_ERR_UNSUPPORTED;
  moe_status s;
  if ((s = check_x(L, x, ldx)) != MOE_OK) return s;
  if (!idx || !offsets || !perm || !inv || !xq || !xs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq)) return MOE_ERR_MISALIGNED;
  return from_cuda(
      launch_permute_noalloc(L, x, T, ldx, idx, offsets, perm, inv, xq, xs, static_cast<cudaStream_t>(stream)));
}

moe_status moe_gate_up(moe_layer_t L, const uint8_t* xq, const float* xs, const int32_t* offsets, int T,
                       uint8_t* h, float* hs, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;   // a routing-only handle
  if (T == 0) return MOE_OK;
  if (!xq || !xs || !offsets || !h || !hs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(h)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_gate_up(L, xq, xs, offsets, T * (L->K + L->S), h, hs, static_cast<cudaStream_t>(stream)));
}

moe_status moe_down(moe_layer_t L, const uint8_t* h, const float* hs, const int32_t* offsets, int T, uint16_t* y,
                    void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;   // a routing-only handle
  if (T == 0) return MOE_OK;
  if (!h || !hs || !offsets || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(y)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_down(L, h, hs, offsets, T * (L->K + L->S), y, static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_gate_up(moe_layer_t L, const uint8_t* xq, const float* xs, const int32_t* offsets, int rows,
                               uint8_t* h, float* hs, void* stream) {
  if (!L || rows < 0 || rows > kMaxT * 9) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!xq || !xs || !offsets || !h || !hs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(h)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_gate_up(L, xq, xs, offsets, rows, h, hs, static_cast<cudaStream_t>(stream)));
}

moe_status moe_grouped_down(moe_layer_t L, const uint8_t* h, const float* hs, const int32_t* offsets, int rows,
                            uint16_t* y, void* stream) {
  if (!L || rows < 0 || rows > kMaxT * 9) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!h || !hs || !offsets || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(y)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_down(L, h, hs, offsets, rows, y, static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_pack_scales(moe_layer_t L, const float* xs, int T, float* xs_rows, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!xs || !xs_rows) return MOE_ERR_INVALID_ARG;
  return from_cuda(launch_ep_pack_scales(L, xs, T, xs_rows, static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_regroup(moe_layer_t L, int ranks, const int32_t* seg_counts, int n_recv, const uint8_t* recv_q,
                          const float* recv_s, const uint8_t* own_q, const float* own_s, int T, uint8_t* out_q,
                          float* out_s, int32_t* out_offsets, void* stream) {
  if (!L || ranks < 1 || ranks * L->E > kEpMaxSegments || n_recv < 0 || T < 0 || T > kMaxT)
    return MOE_ERR_INVALID_ARG;
  if (!seg_counts || !out_q || !out_s || !out_offsets) return MOE_ERR_INVALID_ARG;
  if (n_recv > 0 && (!recv_q || !recv_s)) return MOE_ERR_INVALID_ARG;
  if (T * L->S > 0 && (!own_q || !own_s)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(recv_q) || !aligned16(own_q) || !aligned16(out_q)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_ep_regroup(L, ranks, seg_counts, n_recv, recv_q, recv_s, own_q, own_s, T, out_q, out_s,
                                     out_offsets, static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_unregroup(moe_layer_t L, int ranks, const int32_t* seg_counts, int n_recv, const uint16_t* y_g,
                            int T, uint16_t* y_send, uint16_t* y_own, void* stream) {
  if (!L || ranks < 1 || ranks * L->E > kEpMaxSegments || n_recv < 0 || T < 0 || T > kMaxT)
    return MOE_ERR_INVALID_ARG;
  if (!seg_counts || !y_g) return MOE_ERR_INVALID_ARG;
  if ((n_recv > 0 && !y_send) || (T * L->S > 0 && !y_own)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_g) || !aligned16(y_send) || !aligned16(y_own)) return MOE_ERR_MISALIGNED;
  if (n_recv + T * L->S == 0) return MOE_OK;
  return from_cuda(launch_ep_unregroup(L, ranks, seg_counts, n_recv, y_g, T, y_send, y_own,
                                       static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(moe_layer_t L, const uint8_t* xq, const float* xs, const int32_t* offsets, int T,
                          uint16_t* y, void* ws, size_t ws_bytes, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;   // a routing-only handle
  if (T == 0) return MOE_OK;
  if (!xq || !xs || !offsets || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(y)) return MOE_ERR_MISALIGNED;
  moe_status s;
  if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
  Scratch sc = carve(L, T, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = T * (L->K + L->S);
  cudaError_t e = launch_gate_up(L, xq, xs, offsets, rows, sc.h, sc.hs, st);
  if (e == cudaSuccess) e = launch_down(L, sc.h, sc.hs, offsets, rows, y, st);
  return from_cuda(e);
}

moe_status moe_combine(moe_layer_t L, const uint16_t* y, const int32_t* inv, const float* w, int T, uint16_t* out,
                       int ldo, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !inv || !w || !out || ldo < L->H) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(out) || (size_t(ldo) * 2) % 16 != 0) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_combine(L, y, inv, w, T, out, ldo, static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(moe_layer_t L, const uint16_t* x, int T, int ldx, uint16_t* out, int ldo, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!L || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;   // a routing-only handle
  if (T == 0) return MOE_OK;
  moe_status s;
  if ((s = check_x(L, x, ldx)) != MOE_OK) return s;
  if (!out || ldo < L->H) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out) || (size_t(ldo) * 2) % 16 != 0) return MOE_ERR_MISALIGNED;
  if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
  Scratch sc = carve(L, T, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_route(L, x, T, ldx, sc.idx, sc.topw, nullptr, sc.route_partial, st);
  if (e == cudaSuccess) e = launch_permute(L, x, T, ldx, sc.idx, sc.offsets, sc.perm, sc.inv, sc.xq, sc.xs, sc, st);
  const int rows = T * (L->K + L->S);
  if (e == cudaSuccess) e = launch_gate_up(L, sc.xq, sc.xs, sc.offsets, rows, sc.h, sc.hs, st);
  if (e == cudaSuccess) e = launch_down(L, sc.h, sc.hs, sc.offsets, rows, sc.y, st);
  if (e == cudaSuccess) e = launch_combine(L, sc.y, sc.inv, sc.topw, T, out, ldo, st);
  return from_cuda(e);
}

int moe_kernels_per_forward(moe_layer_t L, int T) {
  if (!L || T <= 0 || T > kMaxT) return 0;
  const int rows = T * (L->K + L->S);
  return 2 + permute_kernels(L, T) + 1 + 1 + (down_ksplit(L, rows) > 1 ? 1 : 0) + 1;
}

moe_status moe_get_device_status(moe_layer_t L, void* stream, uint32_t* detail) {
  if (!L) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, L->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v && cudaMemset(L->status, 0, sizeof(v)) != cudaSuccess) return MOE_ERR_CUDA;
  if (detail) *detail = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

moe_status moe_test_inject_stall(moe_layer_t L, unsigned long long wait_limit_ns) {
  if (!L || wait_limit_ns == 0) return MOE_ERR_INVALID_ARG;
  L->test_stall_ns = wait_limit_ns;
  return MOE_OK;
}

moe_status moe_test_grouped_gemm_f32(moe_layer_t L, int which, const uint8_t* a, const float* as,
                                     const int32_t* offsets, int T, float* out, void* stream) {
  if (!L || T < 0 || T > kMaxT || (which != 0 && which != 1)) return MOE_ERR_INVALID_ARG;
  if (!L->has_experts) return MOE_ERR_INVALID_ARG;   // a routing-only handle
  if (T == 0) return MOE_OK;
  if (!a || !as || !offsets || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a)) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_test_gemm_f32(L, which, a, as, offsets, T, out, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// Expert parallelism over peer memory

static_assert(sizeof(cudaIpcMemHandle_t) == MOE_EP_HANDLE_BYTES, "IPC handle size");

// Makes the comm's device current for the scope of a call (IPC mappings and
// the tables belong to it) and restores the caller's device.
struct DeviceScope {
  int prev = -1;
  bool ok = false;
  explicit DeviceScope(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceScope() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

static moe_status ep_upload_tables(moe_ep_comm_s* c, const uint64_t* q, const uint64_t* s, const uint64_t* y) {
  uint64_t tab[3 * kEpMaxRanks];
  for (int i = 0; i < c->ranks; ++i) {
    tab[i] = q[i];
    tab[c->ranks + i] = s[i];
    tab[2 * c->ranks + i] = y[i];
  }
  return from_cuda(cudaMemcpy(c->d_peer_q, tab, sizeof(uint64_t) * 3 * c->ranks, cudaMemcpyHostToDevice));
}

static void ep_own(const moe_ep_comm_s* c, const char* base, uint64_t* q, uint64_t* s, uint64_t* y) {
  *q = reinterpret_cast<uint64_t>(base);
  *s = reinterpret_cast<uint64_t>(base + c->off_s);
  *y = reinterpret_cast<uint64_t>(base + c->off_y);
}

moe_status moe_ep_comm_create(moe_layer_t L, int rank, int ranks, int capacity, moe_ep_comm_t* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (!L || ranks < 1 || ranks > kEpMaxRanks || rank < 0 || rank >= ranks || capacity < 1 || capacity > kMaxT)
    return MOE_ERR_INVALID_ARG;
  moe_ep_comm_s* c = new (std::nothrow) moe_ep_comm_s();
  if (!c) return MOE_ERR_CUDA;
  if (cudaGetDevice(&c->device) != cudaSuccess) {
    delete c;
    return MOE_ERR_CUDA;
  }
  c->rank = rank;
  c->ranks = ranks;
  c->cap = capacity;
  c->H = L->H;
  c->HB = L->HB;
  c->off_s = align_up(size_t(capacity) * L->H, 256);
  c->off_y = c->off_s + align_up(sizeof(float) * L->HB * size_t(capacity), 256);
  c->bytes = c->off_y + sizeof(uint16_t) * size_t(capacity) * L->H;
  void* tab = nullptr;
  if (cudaMalloc(&c->base, c->bytes) != cudaSuccess || cudaMalloc(&tab, sizeof(uint64_t) * 3 * ranks) != cudaSuccess) {
    if (c->base) cudaFree(c->base);
    delete c;
    return MOE_ERR_CUDA;
  }
  c->d_peer_q = static_cast<uint64_t*>(tab);
  c->d_peer_s = c->d_peer_q + ranks;
  c->d_peer_y = c->d_peer_s + ranks;
  uint64_t q[kEpMaxRanks] = {}, sc[kEpMaxRanks] = {}, y[kEpMaxRanks] = {};
  ep_own(c, static_cast<const char*>(c->base), &q[rank], &sc[rank], &y[rank]);
  moe_status st = ep_upload_tables(c, q, sc, y);
  if (st != MOE_OK) {
    cudaFree(tab);
    cudaFree(c->base);
    delete c;
    return st;
  }
  c->connected = ranks == 1;
  *out = c;
  return MOE_OK;
}

moe_status moe_ep_comm_export(moe_ep_comm_t c, unsigned char handle[MOE_EP_HANDLE_BYTES]) {
  if (!c || !handle) return MOE_ERR_INVALID_ARG;
  DeviceScope scope(c->device);
  if (!scope.ok) return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, c->base) != cudaSuccess) return MOE_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  return MOE_OK;
}

static void ep_close_opened(moe_ep_comm_s* c) {
  for (int i = 0; i < kEpMaxRanks; ++i)
    if (c->opened[i]) {
      cudaIpcCloseMemHandle(c->opened[i]);
      c->opened[i] = nullptr;
    }
}

moe_status moe_ep_comm_connect(moe_ep_comm_t c, const unsigned char* handles) {
  if (!c || !handles || c->connected) return MOE_ERR_INVALID_ARG;
  DeviceScope scope(c->device);
  if (!scope.ok) return MOE_ERR_CUDA;
  uint64_t q[kEpMaxRanks] = {}, sc[kEpMaxRanks] = {}, y[kEpMaxRanks] = {};
  for (int i = 0; i < c->ranks; ++i) {
    if (i == c->rank) {
      ep_own(c, static_cast<const char*>(c->base), &q[i], &sc[i], &y[i]);
      continue;
    }
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handles + size_t(i) * MOE_EP_HANDLE_BYTES, sizeof(h));
    void* p = nullptr;
    if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
      ep_close_opened(c);
      return MOE_ERR_CUDA;
    }
    c->opened[i] = p;
    ep_own(c, static_cast<const char*>(p), &q[i], &sc[i], &y[i]);
  }
  moe_status st = ep_upload_tables(c, q, sc, y);
  if (st != MOE_OK) {
    ep_close_opened(c);
    return st;
  }
  c->connected = true;
  return MOE_OK;
}

moe_status moe_ep_comm_connect_local(moe_ep_comm_t* comms, int ranks) {
  if (!comms || ranks < 1 || ranks > kEpMaxRanks) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < ranks; ++i) {
    const moe_ep_comm_s* c = comms[i];
    if (!c || c->rank != i || c->ranks != ranks || c->cap != comms[0]->cap || c->H != comms[0]->H ||
        c->device != comms[0]->device || c->connected != (ranks == 1))
      return MOE_ERR_INVALID_ARG;
  }
  uint64_t q[kEpMaxRanks] = {}, sc[kEpMaxRanks] = {}, y[kEpMaxRanks] = {};
  for (int i = 0; i < ranks; ++i) ep_own(comms[i], static_cast<const char*>(comms[i]->base), &q[i], &sc[i], &y[i]);
  for (int i = 0; i < ranks; ++i) {
    moe_status st = ep_upload_tables(comms[i], q, sc, y);
    if (st != MOE_OK) return st;
    comms[i]->connected = true;
  }
  return MOE_OK;
}

moe_status moe_ep_comm_buffers(moe_ep_comm_t c, uint8_t** recv_q, float** recv_s, uint16_t** y) {
  if (!c) return MOE_ERR_INVALID_ARG;
  char* b = static_cast<char*>(c->base);
  if (recv_q) *recv_q = reinterpret_cast<uint8_t*>(b);
  if (recv_s) *recv_s = reinterpret_cast<float*>(b + c->off_s);
  if (y) *y = reinterpret_cast<uint16_t*>(b + c->off_y);
  return MOE_OK;
}

moe_status moe_ep_comm_destroy(moe_ep_comm_t c) {
  if (!c) return MOE_OK;
  DeviceScope scope(c->device);
  moe_status st = scope.ok ? from_cuda(cudaDeviceSynchronize()) : MOE_ERR_CUDA;
  ep_close_opened(c);
  if (cudaFree(c->d_peer_q) != cudaSuccess) st = MOE_ERR_CUDA;
  if (cudaFree(c->base) != cudaSuccess) st = MOE_ERR_CUDA;
  delete c;
  return st;
}

moe_status moe_ep_plan(moe_layer_t L, const int32_t* idx, int T, int32_t* offsets, void* ws, size_t ws_bytes,
                       void* stream) {
  if (!L || T < 0 || T > kMaxT || !offsets) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) return from_cuda(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (L->E + 2), st));
  if (!idx) return MOE_ERR_INVALID_ARG;
  moe_status s;
  if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
  return from_cuda(launch_ep_plan(L, idx, T, offsets, carve(L, T, ws), st));
}

static moe_status ep_check(const moe_layer_s* L, const moe_ep_comm_s* c, int T) {
  if (!L || !c || T < 0 || T > kMaxT) return MOE_ERR_INVALID_ARG;
  if (!c->connected || L->E % c->ranks != 0 || c->H != L->H) return MOE_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev != c->device) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status moe_ep_dispatch(moe_layer_t L, moe_ep_comm_t c, const uint16_t* x, int T, int ldx, const int32_t* idx,
                           const int32_t* all_offsets, int32_t* inv_ep, int32_t* group_offsets, void* ws,
                           size_t ws_bytes, void* stream) {
  moe_status s;
  if ((s = ep_check(L, c, T)) != MOE_OK) return s;
  if (!all_offsets || !group_offsets) return MOE_ERR_INVALID_ARG;
  Scratch sc = {};
  if (T > 0) {
    if (!idx || !inv_ep) return MOE_ERR_INVALID_ARG;
    if ((s = check_x(L, x, ldx)) != MOE_OK) return s;
    if ((s = check_ws(L, T, ws, ws_bytes)) != MOE_OK) return s;
    sc = carve(L, T, ws);
  }
  return from_cuda(launch_ep_dispatch(L, c, x, T, ldx, idx, all_offsets, inv_ep, group_offsets, sc,
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_combine(moe_layer_t L, moe_ep_comm_t c, const int32_t* idx, const int32_t* inv_ep, const float* w,
                          const int32_t* group_offsets, int T, uint16_t* out, int ldo, void* stream) {
  moe_status s;
  if ((s = ep_check(L, c, T)) != MOE_OK) return s;
  if (T == 0) return MOE_OK;
  if (!idx || !inv_ep || !w || !group_offsets || !out || ldo < L->H) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out) || (size_t(ldo) * 2) % 16 != 0) return MOE_ERR_MISALIGNED;
  return from_cuda(launch_ep_combine(L, c, idx, inv_ep, w, group_offsets, T, out, ldo,
                                     static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
#pragma GCC visibility pop

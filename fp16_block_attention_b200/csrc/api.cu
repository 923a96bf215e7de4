// C ABI of the library (declared in include/thrift.h): argument checks,
// workspace carving and kernel launches.  Nothing here allocates device
// memory.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdint>

#include "common.h"
#include "ptx.cuh"

namespace thrift {

namespace {

// Device error word: one per device, in the library's static device memory.
__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
// Device address of the error word per device (atomic: first calls from
// several host threads may overlap).
std::atomic<uint32_t*> g_err_ptr[kMaxDevices];

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A failed launch or call also leaves its error as the runtime's last error,
// which the next launch's check would report again: read it here, so that one
// failed call does not fail the next (an error that poisons the context
// stays, as it must).
thrift_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return THRIFT_OK;
  cudaGetLastError();
  return THRIFT_ERR_CUDA;
}

struct QuantSizes {
  size_t codes, scales;
};

QuantSizes quant_sizes(const thrift_shape& s, thrift_operand op) {
  const size_t NT = static_cast<size_t>(num_tiles(s.N));
  const size_t H = (op == THRIFT_Q) ? s.Hq : s.Hkv;
  const size_t BH = static_cast<size_t>(s.B) * H;
  QuantSizes q;
  q.codes = BH * s.N * (s.D / 2);
  if (op == THRIFT_V)
    q.scales = BH * 2 * NT * 512;
  else
    q.scales = BH * NT * (s.D / 64) * 512;
  return q;
}

struct FusedWs {
  uint8_t *q4, *qs, *k4, *ks, *v4, *vs, *mask;
  void* sel;
  uint8_t *q8, *qs8, *k8, *ks8, *v8, *vs8;  // MXFP8 copies (eight only)
  size_t total;
};

FusedWs carve_fused(void* base, const thrift_shape& s, bool eight = false) {
  FusedWs w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* r = p ? p + off : nullptr;
    off += align_up(bytes);
    return reinterpret_cast<uint8_t*>(r);
  };
  const QuantSizes q = quant_sizes(s, THRIFT_Q), k = quant_sizes(s, THRIFT_K), v = quant_sizes(s, THRIFT_V);
  w.q4 = take(q.codes);
  w.qs = take(q.scales);
  w.k4 = take(k.codes);
  w.ks = take(k.scales);
  w.v4 = take(v.codes);
  w.vs = take(v.scales);
  const size_t nb = s.N / s.blk;
  w.mask = take(static_cast<size_t>(s.B) * s.Hq * nb * nb);
  w.sel = take(select_workspace_bytes(s));
  w.q8 = w.qs8 = w.k8 = w.ks8 = w.v8 = w.vs8 = nullptr;
  if (eight) {
    w.q8 = take(mx8_codes_bytes(s, THRIFT_Q));
    w.qs8 = take(mx8_scales_bytes(s, THRIFT_Q));
    w.k8 = take(mx8_codes_bytes(s, THRIFT_K));
    w.ks8 = take(mx8_scales_bytes(s, THRIFT_K));
    w.v8 = take(mx8_codes_bytes(s, THRIFT_V));
    w.vs8 = take(mx8_scales_bytes(s, THRIFT_V));
  }
  w.total = off;
  return w;
}

}  // namespace

uint32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  uint32_t* w = g_err_ptr[dev].load(std::memory_order_relaxed);
  if (!w) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    w = static_cast<uint32_t*>(p);
    g_err_ptr[dev].store(w, std::memory_order_relaxed);
  }
  return w;
}

namespace {
std::atomic<uint64_t> g_wait_ns{kWaitNs};
}  // namespace

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

int test_withhold_tile() {
  const char* v = std::getenv("THRIFT_TEST_WITHHOLD_TILE");
  if (!v || !*v) return -1;
  char* end = nullptr;
  const long t = std::strtol(v, &end, 10);
  return (end && *end == 0 && t >= 0 && t < (1L << 20)) ? static_cast<int>(t) : -1;
}

thrift_status check_shape(const thrift_shape* s) {
  if (!s) return THRIFT_ERR_INVALID_ARG;
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->N <= 0 || s->D <= 0 || s->blk <= 0) return THRIFT_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return THRIFT_ERR_INVALID_ARG;
  if (!std::isfinite(s->sm_scale) || !(s->sm_scale > 0.0f)) return THRIFT_ERR_INVALID_ARG;  // softmax scale > 0
  if (s->causal != 0 && s->causal != 1) return THRIFT_ERR_INVALID_ARG;
  if (s->D != 64 && s->D != 128) return THRIFT_ERR_UNSUPPORTED;
  if (s->blk != 64 && s->blk != 128) return THRIFT_ERR_UNSUPPORTED;
  if (s->N % s->blk != 0) return THRIFT_ERR_UNSUPPORTED;
  if (s->N > 131072) return THRIFT_ERR_UNSUPPORTED;                       // key tiles per query tile <= 1024
  if (static_cast<long long>(s->B) * s->Hq > 65535) return THRIFT_ERR_UNSUPPORTED;  // grid y/z extents
  return THRIFT_OK;
}

}  // namespace thrift

using namespace thrift;

extern "C" {

thrift_status thrift_quant_bytes(const thrift_shape* shape, thrift_operand op, size_t* codes_bytes,
                                 size_t* scales_bytes) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (op != THRIFT_Q && op != THRIFT_K && op != THRIFT_V) return THRIFT_ERR_INVALID_ARG;
  if (!codes_bytes || !scales_bytes) return THRIFT_ERR_INVALID_ARG;
  const QuantSizes q = quant_sizes(*shape, op);
  *codes_bytes = q.codes;
  *scales_bytes = q.scales;
  return THRIFT_OK;
}

thrift_status thrift_quantize_nvfp4(const void* x, thrift_operand op, const thrift_shape* shape, void* codes,
                                    void* scales, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (op != THRIFT_Q && op != THRIFT_K && op != THRIFT_V) return THRIFT_ERR_INVALID_ARG;
  if (!x || !codes || !scales) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return THRIFT_ERR_INVALID_ARG;
  const thrift_shape& s = *shape;
  const size_t H = (op == THRIFT_Q) ? s.Hq : s.Hkv;
  const size_t BH = static_cast<size_t>(s.B) * H;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (op == THRIFT_V) return from_cuda(launch_quantize_v(x, BH, s.N, s.D, codes, scales, cs));
  return from_cuda(launch_quantize_qk(x, BH * s.N, s.N, s.D, codes, scales, cs));
}

thrift_status thrift_quantize_pool_nvfp4(const void* x, thrift_operand op, const thrift_shape* shape, void* codes,
                                         void* scales, float* means, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (op != THRIFT_Q && op != THRIFT_K) return THRIFT_ERR_INVALID_ARG;
  if (!x || !codes || !scales || !means) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || (reinterpret_cast<uintptr_t>(means) & 3u))
    return THRIFT_ERR_INVALID_ARG;
  const thrift_shape& s = *shape;
  const size_t BH = static_cast<size_t>(s.B) * ((op == THRIFT_Q) ? s.Hq : s.Hkv);
  return from_cuda(
      launch_quantize_pool_qk(x, BH, s.N, s.D, s.blk, codes, scales, means, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_quant8_bytes(const thrift_shape* shape, thrift_operand op, size_t* codes_bytes,
                                  size_t* scales_bytes) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (op != THRIFT_Q && op != THRIFT_K && op != THRIFT_V) return THRIFT_ERR_INVALID_ARG;
  if (!codes_bytes || !scales_bytes) return THRIFT_ERR_INVALID_ARG;
  *codes_bytes = mx8_codes_bytes(*shape, op);
  *scales_bytes = mx8_scales_bytes(*shape, op);
  return THRIFT_OK;
}

thrift_status thrift_quantize_mxfp8(const void* x, thrift_operand op, const thrift_shape* shape, void* codes,
                                    void* scales, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (op != THRIFT_Q && op != THRIFT_K && op != THRIFT_V) return THRIFT_ERR_INVALID_ARG;
  if (!x || !codes || !scales) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return THRIFT_ERR_INVALID_ARG;
  return from_cuda(launch_quantize_mx8(x, op, *shape, codes, scales, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_select_workspace_bytes(const thrift_shape* shape, size_t* bytes) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!bytes) return THRIFT_ERR_INVALID_ARG;
  *bytes = select_workspace_bytes(*shape);
  return THRIFT_OK;
}

thrift_status thrift_select_blocks(const void* Q, const void* K, const thrift_shape* shape, double rho,
                                   uint8_t* mask, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !mask || !(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return THRIFT_ERR_INVALID_ARG;
  if (!ws || ws_bytes < select_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  return from_cuda(launch_select(Q, K, *shape, rho, mask, ws, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_select_blocks_pooled(const float* qm, const float* km, const thrift_shape* shape, double rho,
                                          uint8_t* mask, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!qm || !km || !mask || !(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(qm) & 3u) || (reinterpret_cast<uintptr_t>(km) & 3u)) return THRIFT_ERR_INVALID_ARG;
  if (!ws || ws_bytes < select_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  return from_cuda(launch_select_pooled(qm, km, *shape, rho, mask, ws, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_select_blocks_tiered(const void* Q, const void* K, const thrift_shape* shape, double rho,
                                          double rho8, double sigma, uint8_t* mask, void* ws, size_t ws_bytes,
                                          void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !mask || !(rho >= 0.0 && rho <= 1.0) || !(rho8 >= 0.0 && rho8 <= 1.0) ||
      !(sigma >= 0.0 && sigma <= 1.0))
    return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return THRIFT_ERR_INVALID_ARG;
  if (!ws || ws_bytes < select_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  return from_cuda(
      launch_select_tiered(Q, K, *shape, rho, rho8, sigma, mask, ws, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_select_blocks_vertical_window(const void* Q, const void* K, const thrift_shape* shape, double rho,
                                                   int window, uint8_t* mask, void* ws, size_t ws_bytes,
                                                   void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !mask || !(rho >= 0.0 && rho <= 1.0) || window < 0) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return THRIFT_ERR_INVALID_ARG;
  if (shape->N / shape->blk > kMaxVWBlocks) return THRIFT_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < select_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  return from_cuda(
      launch_select_vertical_window(Q, K, *shape, rho, window, mask, ws, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_select_blocks_static(const void* Q, const void* K, const thrift_shape* shape, double rho,
                                          uint8_t* mask, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !mask || !(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return THRIFT_ERR_INVALID_ARG;
  if (select_workspace_bytes(*shape) > kSelectStaticBytes) return THRIFT_ERR_WORKSPACE;
  return from_cuda(launch_select_static(Q, K, *shape, rho, mask, static_cast<cudaStream_t>(stream)));
}

namespace {
thrift_status attention_entry(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4,
                              const void* qs, const void* k4, const void* ks, const void* v4, const void* vs,
                              const thrift_shape* shape, void* O, bool skip, const Mx8Copies* eight, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  const void* ptrs[] = {Q, K, V, q4, qs, k4, ks, v4, vs, O};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return THRIFT_ERR_INVALID_ARG;
  if (!mask) return THRIFT_ERR_INVALID_ARG;
  if (eight) {
    const void* p8[] = {eight->q8, eight->qs8, eight->k8, eight->ks8, eight->v8, eight->vs8};
    for (const void* ptr : p8)
      if (!ptr || !aligned16(ptr)) return THRIFT_ERR_INVALID_ARG;
    if (shape->blk != 128) return THRIFT_ERR_UNSUPPORTED;
  }
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  return from_cuda(launch_attention(Q, K, V, mask, q4, qs, k4, ks, v4, vs, *shape, O, skip, eight, err,
                                    static_cast<cudaStream_t>(stream)));
}
}  // namespace

thrift_status thrift_attention(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4,
                               const void* qs, const void* k4, const void* ks, const void* v4, const void* vs,
                               const thrift_shape* shape, void* O, void* stream) {
  return attention_entry(Q, K, V, mask, q4, qs, k4, ks, v4, vs, shape, O, false, nullptr, stream);
}

thrift_status thrift_attention_tiered(const void* Q, const void* K, const void* V, const uint8_t* mask,
                                      const void* q4, const void* qs, const void* k4, const void* ks, const void* v4,
                                      const void* vs, const void* q8, const void* qs8, const void* k8,
                                      const void* ks8, const void* v8, const void* vs8, const thrift_shape* shape,
                                      void* O, void* stream) {
  const bool none = !q8 && !qs8 && !k8 && !ks8 && !v8 && !vs8;
  const Mx8Copies eight = {q8, qs8, k8, ks8, v8, vs8};
  return attention_entry(Q, K, V, mask, q4, qs, k4, ks, v4, vs, shape, O, true, none ? nullptr : &eight, stream);
}

thrift_status thrift_fused_workspace_bytes(const thrift_shape* shape, size_t* bytes) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!bytes) return THRIFT_ERR_INVALID_ARG;
  *bytes = carve_fused(nullptr, *shape).total;
  return THRIFT_OK;
}

thrift_status thrift_attention_fused(const void* Q, const void* K, const void* V, const thrift_shape* shape,
                                     double rho, void* O, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !V || !O || !(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return THRIFT_ERR_INVALID_ARG;
  const FusedWs need = carve_fused(nullptr, *shape);
  if (!ws || ws_bytes < need.total || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  const FusedWs w = carve_fused(ws, *shape);
  const thrift_shape& s = *shape;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  // Q and K are read once: quantised and pooled in one pass (the block means
  // go straight into the selection workspace)
  float *qm = nullptr, *km = nullptr;
  select_means(w.sel, s, &qm, &km);
  if (launch_quantize_pool_qk(Q, static_cast<size_t>(s.B) * s.Hq, s.N, s.D, s.blk, w.q4, w.qs, qm, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (launch_quantize_pool_qk(K, static_cast<size_t>(s.B) * s.Hkv, s.N, s.D, s.blk, w.k4, w.ks, km, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (launch_quantize_v(V, static_cast<size_t>(s.B) * s.Hkv, s.N, s.D, w.v4, w.vs, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (launch_select_pooled(nullptr, nullptr, s, rho, w.mask, w.sel, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
  return from_cuda(launch_attention(Q, K, V, w.mask, w.q4, w.qs, w.k4, w.ks, w.v4, w.vs, s, O, false, nullptr, err, cs));
}

thrift_status thrift_fused_tiered_workspace_bytes(const thrift_shape* shape, double rho8, size_t* bytes) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!bytes || !(rho8 >= 0.0 && rho8 <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  *bytes = carve_fused(nullptr, *shape, rho8 > 0.0).total;
  return THRIFT_OK;
}

thrift_status thrift_attention_fused_tiered(const void* Q, const void* K, const void* V, const thrift_shape* shape,
                                            double rho, double rho8, double sigma, void* O, void* ws,
                                            size_t ws_bytes, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!Q || !K || !V || !O || !(rho >= 0.0 && rho <= 1.0) || !(rho8 >= 0.0 && rho8 <= 1.0) ||
      !(sigma >= 0.0 && sigma <= 1.0))
    return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return THRIFT_ERR_INVALID_ARG;
  const bool eight = rho8 > 0.0;
  if (eight && shape->blk != 128) return THRIFT_ERR_UNSUPPORTED;
  const FusedWs need = carve_fused(nullptr, *shape, eight);
  if (!ws || ws_bytes < need.total || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  const FusedWs w = carve_fused(ws, *shape, eight);
  const thrift_shape& s = *shape;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  float *qm = nullptr, *km = nullptr;  // Q and K quantised and pooled in one pass
  select_means(w.sel, s, &qm, &km);
  if (launch_quantize_pool_qk(Q, static_cast<size_t>(s.B) * s.Hq, s.N, s.D, s.blk, w.q4, w.qs, qm, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (launch_quantize_pool_qk(K, static_cast<size_t>(s.B) * s.Hkv, s.N, s.D, s.blk, w.k4, w.ks, km, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  if (launch_quantize_v(V, static_cast<size_t>(s.B) * s.Hkv, s.N, s.D, w.v4, w.vs, cs) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  Mx8Copies copies = {w.q8, w.qs8, w.k8, w.ks8, w.v8, w.vs8};
  if (eight) {
    if (launch_quantize_mx8(Q, THRIFT_Q, s, w.q8, w.qs8, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
    if (launch_quantize_mx8(K, THRIFT_K, s, w.k8, w.ks8, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
    if (launch_quantize_mx8(V, THRIFT_V, s, w.v8, w.vs8, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
  }
  if (launch_select_tiered_pooled(s, rho, rho8, sigma, w.mask, w.sel, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
  return from_cuda(launch_attention(Q, K, V, w.mask, w.q4, w.qs, w.k4, w.ks, w.v4, w.vs, s, O, true,
                                    eight ? &copies : nullptr, err, cs));
}

namespace {
// Decode supports D = 128, blk = 128 and up to 16 query heads per kv head.
thrift_status check_decode_shape(const thrift_shape* shape) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (shape->D != 128 || shape->blk != 128 || shape->Hq / shape->Hkv > 16) return THRIFT_ERR_UNSUPPORTED;
  return THRIFT_OK;
}
}  // namespace

thrift_status thrift_pool_keys(const void* K, const thrift_shape* shape, float* km, void* stream) {
  thrift_status st = check_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!K || !km || !aligned16(K) || !aligned16(km)) return THRIFT_ERR_INVALID_ARG;
  return from_cuda(launch_pool_keys(K, *shape, km, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_decode_select(const void* q, const float* km, const thrift_shape* shape, double rho,
                                   uint8_t* mask, void* stream) {
  thrift_status st = check_decode_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!q || !km || !mask || !(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(km)) return THRIFT_ERR_INVALID_ARG;
  return from_cuda(launch_decode_select(q, km, *shape, rho, mask, static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_decode_workspace_bytes(const thrift_shape* shape, size_t* bytes) {
  thrift_status st = check_decode_shape(shape);
  if (st != THRIFT_OK) return st;
  if (!bytes) return THRIFT_ERR_INVALID_ARG;
  *bytes = decode_workspace_bytes(*shape);
  return THRIFT_OK;
}

thrift_status thrift_decode_attention(const void* q, const void* K, const void* V, const void* k4, const void* ks,
                                      const void* v4, const void* vs, const uint8_t* mask, const thrift_shape* shape,
                                      void* O, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = check_decode_shape(shape);
  if (st != THRIFT_OK) return st;
  const void* ptrs[] = {q, K, V, k4, ks, v4, vs, O};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return THRIFT_ERR_INVALID_ARG;
  if (!mask) return THRIFT_ERR_INVALID_ARG;
  if (!ws || ws_bytes < decode_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  return from_cuda(launch_decode_attention(q, K, V, k4, ks, v4, vs, mask, *shape, O, decode_carve(ws, *shape), err,
                                           static_cast<cudaStream_t>(stream)));
}

thrift_status thrift_decode_step(const void* q, const void* K, const void* V, const void* k4, const void* ks,
                                 const void* v4, const void* vs, const float* km, const thrift_shape* shape,
                                 double rho, void* O, void* ws, size_t ws_bytes, void* stream) {
  thrift_status st = check_decode_shape(shape);
  if (st != THRIFT_OK) return st;
  const void* ptrs[] = {q, K, V, k4, ks, v4, vs, km, O};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return THRIFT_ERR_INVALID_ARG;
  if (!(rho >= 0.0 && rho <= 1.0)) return THRIFT_ERR_INVALID_ARG;
  if (!ws || ws_bytes < decode_workspace_bytes(*shape) || !aligned16(ws)) return THRIFT_ERR_WORKSPACE;
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const DecodeWs w = decode_carve(ws, *shape);
  if (launch_decode_select(q, km, *shape, rho, w.mask, cs) != cudaSuccess) return THRIFT_ERR_CUDA;
  return from_cuda(launch_decode_attention(q, K, V, k4, ks, v4, vs, w.mask, *shape, O, w, err, cs));
}

thrift_status thrift_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return THRIFT_ERR_CUDA;
  uint32_t* err = device_error_word();
  if (!err) return THRIFT_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return THRIFT_ERR_CUDA;
    return v == DEV_BAD_ARG ? THRIFT_ERR_INVALID_ARG : THRIFT_ERR_TIMEOUT;
  }
  return THRIFT_OK;
}

thrift_status thrift_set_wait_limit(uint64_t ns) {
  if (ns < 1000 || ns > 60000000000ull) return THRIFT_ERR_INVALID_ARG;
  g_wait_ns.store(ns, std::memory_order_relaxed);
  return THRIFT_OK;
}

const char* thrift_strerror(thrift_status status) {
  switch (status) {
    case THRIFT_OK: return "ok";
    case THRIFT_ERR_INVALID_ARG: return "invalid argument";
    case THRIFT_ERR_UNSUPPORTED: return "unsupported shape";
    case THRIFT_ERR_CUDA: return "CUDA runtime error";
    case THRIFT_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case THRIFT_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

}  // extern "C"

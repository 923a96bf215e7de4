// Shared host/device definitions of the library: shape checks, buffer sizes,
// the scale-factor layout and the kernel launch entry points.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/thrift.h"

namespace thrift {

constexpr int kTile = 128;        // rows of a query tile and keys of a key tile
constexpr int kPLog2 = 11;        // pre-scale 2^11 of P before its FP16 / NVFP4 encoding
constexpr uint64_t kWaitNs = 2000000000ull;  // bound of every in-kernel wait (2 s)

__host__ __device__ inline int num_tiles(int N) { return (N + kTile - 1) / kTile; }

// Validate a shape; returns THRIFT_OK, INVALID_ARG or UNSUPPORTED.
thrift_status check_shape(const thrift_shape* s);

// Byte offset of the scale of (row n, 16-group g) of a Q/K operand.
__host__ __device__ inline size_t qk_scale_index(size_t bh, int n, int g, int NT, int D) {
  return ((bh * NT + static_cast<size_t>(n / kTile)) * (D / 64) + g / 4) * 512 + (n % 32) * 16 +
         ((n % kTile) / 32) * 4 + (g % 4);
}
// Byte offset of the scale of (channel d, key group n/16) of V.
__host__ __device__ inline size_t v_scale_index(size_t bh, int d, int n, int NT) {
  return (bh * 2 * NT + static_cast<size_t>(n / 64)) * 512 + (d % 32) * 16 + (d / 32) * 4 + (n % 64) / 16;
}

// Device error word of the current device (allocated statically in the library).
uint32_t* device_error_word();

// Bound of every wait inside the attention kernels launched from now on, in
// nanoseconds (thrift_set_wait_limit; kWaitNs by default).
uint64_t wait_limit_ns();

// Failure-detection tests only: the processed key tile whose copies the
// attention kernels' producer does not issue, from the environment variable
// THRIFT_TEST_WITHHOLD_TILE read at each launch; -1 (the default) withholds
// nothing.
int test_withhold_tile();

// ---- launchers (return cudaError_t of the launch) --------------------------
cudaError_t launch_quantize_qk(const void* x, size_t rows, int N, int D, void* codes, void* scales,
                               cudaStream_t st);
cudaError_t launch_quantize_v(const void* v, size_t bh, int N, int D, void* codes, void* scales, cudaStream_t st);
// Q or K quantised along D and pooled in one pass: the NVFP4 copy as
// launch_quantize_qk writes it, and the FP32 block means [bh][N/blk][D] of
// the selection (quantize.cu).
cudaError_t launch_quantize_pool_qk(const void* x, size_t bh_count, int N, int D, int blk, void* codes, void* scales,
                                    float* means, cudaStream_t st);

// MXFP8 copies (quantize8.cu).
size_t mx8_codes_bytes(const thrift_shape& s, thrift_operand op);
size_t mx8_scales_bytes(const thrift_shape& s, thrift_operand op);
cudaError_t launch_quantize_mx8(const void* x, thrift_operand op, const thrift_shape& s, void* codes, void* scales,
                                cudaStream_t st);

size_t select_workspace_bytes(const thrift_shape& s);
// Size of the library's static selection scratch (thrift_select_blocks_static).
constexpr size_t kSelectStaticBytes = size_t(16) << 20;
cudaError_t launch_select_static(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask,
                                 cudaStream_t st);
cudaError_t launch_select(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask, void* ws,
                          cudaStream_t st);
// The block means in a selection workspace (launch_quantize_pool_qk writes
// them), and the selection from those means (no pooling pass).
void select_means(void* ws, const thrift_shape& s, float** qm, float** km);
// qm / km: the block means, or null for those already in the workspace.
cudaError_t launch_select_pooled(const float* qm, const float* km, const thrift_shape& s, double rho, uint8_t* mask,
                                 void* ws, cudaStream_t st);
cudaError_t launch_select_tiered_pooled(const thrift_shape& s, double rho, double rho8, double sigma, uint8_t* mask,
                                        void* ws, cudaStream_t st);
// Tiered selection (select.cu): mask 1 FP16, 3 MXFP8, 0 NVFP4, 2 skipped.
cudaError_t launch_select_tiered(const void* Q, const void* K, const thrift_shape& s, double rho, double rho8,
                                 double sigma, uint8_t* mask, void* ws, cudaStream_t st);
// Vertical-line / local-window selector (select.cu); nb = N / blk <= kMaxVWBlocks.
constexpr int kMaxVWBlocks = 2048;
cudaError_t launch_select_vertical_window(const void* Q, const void* K, const thrift_shape& s, double rho, int window,
                                          uint8_t* mask, void* ws, cudaStream_t st);

// ---- decode (decode.cu) -----------------------------------------------------
// Block means of K for the decode selection: km [B][Hkv][nb][D] FP32 (select.cu).
cudaError_t launch_pool_keys(const void* K, const thrift_shape& s, float* km, cudaStream_t st);
struct DecodePlan {
  int grid16;  // persistent CTAs of the FP16 pass (one per SM unless its chunk tables need more)
  int ch16;    // FP16 chunk slots per (batch, kv head)
  int C;       // key tiles per NVFP4 chunk
  int cpu;     // NVFP4 chunks per (batch, kv head)
  int grid4;   // persistent CTAs of the NVFP4 pass
};
DecodePlan decode_plan(const thrift_shape& s);
struct DecodeWs {
  uint8_t* mask;     // [B][Hq][nb] (thrift_decode_step)
  float* part_o;     // [B][Hq][slots][D]
  float* part_l;     // [B][Hq][slots]
  float* part_m;     // [B][Hq][slots]
  uint16_t* hbits;   // [B][Hkv][nb]: FP16 bits of the group's query heads per key tile
  uint32_t* list16;  // [B][Hkv][nb]: the tiles some head keeps in FP16
  int* n16;          // [B][Hkv]
};
size_t decode_workspace_bytes(const thrift_shape& s);
DecodeWs decode_carve(void* ws, const thrift_shape& s);
cudaError_t launch_decode_select(const void* q, const float* km, const thrift_shape& s, double rho, uint8_t* mask,
                                 cudaStream_t st);
cudaError_t launch_decode_attention(const void* q, const void* K, const void* V, const void* k4, const void* ks,
                                    const void* v4, const void* vs, const uint8_t* mask, const thrift_shape& s,
                                    void* O, const DecodeWs& w, uint32_t* err, cudaStream_t st);

// MXFP8 copies of Q, K, V (codes and scales, as launch_quantize_mx8 writes them).
struct Mx8Copies {
  const void *q8, *qs8, *k8, *ks8, *v8, *vs8;
};

// skip: the mask may hold 2 (skipped pairs); selects the kernels' skip-aware
// instantiations.  eight: null, or the MXFP8 copies for masks that may hold 3
// (8-bit pairs; blk = 128 only).
cudaError_t launch_attention(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4,
                             const void* qs, const void* k4, const void* ks, const void* v4, const void* vs,
                             const thrift_shape& s, void* O, bool skip, const Mx8Copies* eight, uint32_t* err,
                             cudaStream_t st);

}  // namespace thrift

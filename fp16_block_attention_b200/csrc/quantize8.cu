// MXFP8 copies of the attention operands for 8-bit block pairs (HBM-bound).
//
// 8-bit pairs follow TriAttention's 8-bit precision (abstract on the paper
// page of arXiv 2611.07256), in MXFP8: the OCP microscaling format with E4M3
// elements and one E8M0 scale per 32 consecutive elements, X =
// 2^(floor(log2 amax) - 8) (8 = the exponent of E4M3's largest normal); an
// element is E4M3(v / X), nearest even, saturating at 448.  X is a power of
// two, so v / X is exact and the hardware conversion (round to nearest even,
// saturate to finite) gives the code directly; an all-zero group takes the
// E8M0 byte 0 and zero codes.
//
// Layouts (bytes):
//   Q, K codes [B][H][N][D] (E4M3); V codes [B][Hkv][D][N] (keys contiguous).
//   Scales in the tensor-core scale-factor layout of 128-row tiles, one
//   512-byte chunk per tile (128 rows x 4 scales = 128 contracted elements):
//     Q/K: chunk (bh * NT + n/128), byte (n%32)*16 + ((n%128)/32)*4 + d/32;
//     V:   chunk (bh * NT + n/128), byte (d%32)*16 + (d/32)*4 + (n%128)/32.
//   Bytes no element maps to (rows past N, channels past D, D = 64's upper
//   half of each row) are 0.
#include <cuda_fp16.h>

#include "common.h"
#include "ptx.cuh"

namespace thrift {
namespace {

// E8M0 byte of a group's amax (floor(log2 amax) - 8 + 127, clamped to 0..254;
// 0 for amax = 0) and the factor 1 / X as an FP32 power of two.
__device__ __forceinline__ uint32_t mx8_scale(float amax, float& inv_x) {
  if (!(amax > 0.f)) {
    inv_x = 0.f;
    return 0u;
  }
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 8;  // biased exponent - 8
  const int eb = e < 0 ? 0 : (e > 254 ? 254 : e);
  inv_x = __uint_as_float(static_cast<uint32_t>(254 - eb) << 23);            // 2^(127 - eb)
  return static_cast<uint32_t>(eb);
}

// 32 values -> 32 E4M3 codes in 8 words (element i in byte i % 4 of word i / 4).
__device__ __forceinline__ void mx8_encode32(const float (&x)[32], float inv_x, uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = cvt_e4m3x2(x[4 * i] * inv_x, x[4 * i + 1] * inv_x);
    const uint32_t hi = cvt_e4m3x2(x[4 * i + 2] * inv_x, x[4 * i + 3] * inv_x);
    w[i] = (lo & 0xFFFFu) | (hi << 16);
  }
}

// One thread per 32-element group of a Q / K row.  rows = B*H*N.
__global__ void __launch_bounds__(256) quantize_qk_mx8_kernel(const __half* __restrict__ x, size_t rows, int N,
                                                              int D, uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ scales) {
  const int gpr = D / 32;
  const size_t total = rows * gpr;
  const int NT = num_tiles(N);
  for (size_t gi = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; gi < total;
       gi += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = gi / gpr;
    const int g = static_cast<int>(gi % gpr);
    const uint4* src = reinterpret_cast<const uint4*>(x + row * D + g * 32);
    float v[32];
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(src + q);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[8 * q + 2 * i] = f.x;
        v[8 * q + 2 * i + 1] = f.y;
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    float inv_x;
    const uint32_t sb = mx8_scale(amax, inv_x);
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // an all-zero group: zero codes
    if (amax > 0.f) mx8_encode32(v, inv_x, w);
    uint4* dst = reinterpret_cast<uint4*>(codes + row * D + g * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const size_t bh = row / N;
    const int n = static_cast<int>(row % N);
    scales[(bh * NT + n / kTile) * 512 + (n % 32) * 16 + ((n % kTile) / 32) * 4 + g] = static_cast<uint8_t>(sb);
  }
}

// V along keys: one CTA per (bh, 128-key tile).  The tile [128][D] is staged
// through shared memory with 16-byte loads, all of a thread's loads in flight
// at once; thread (d, g) encodes keys 32 g .. 32 g + 31 of channel d.  Groups
// past N (N a multiple of 64) keep scale 0 and write no codes.
__global__ void __launch_bounds__(256) quantize_v_mx8_kernel(const __half* __restrict__ v, int N, int D,
                                                             uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales) {
  __shared__ __half tile[128][128 + 2];
  const int NT = num_tiles(N);
  const size_t bh = blockIdx.y;
  const int n0 = blockIdx.x * kTile;
  const int nk = min(kTile, N - n0);  // 64 or 128 keys
  const int tid = threadIdx.x;
  const int vpr = D / 8;  // 16-byte pieces per key row
  const uint4* src = reinterpret_cast<const uint4*>(v + (bh * N + n0) * D);
  constexpr int kMaxLoads = 128 * 128 / 8 / 256;  // 8
  uint4 buf[kMaxLoads];
#pragma unroll
  for (int q = 0; q < kMaxLoads; ++q) {
    const int i = tid + q * 256;
    if (i < nk * vpr) buf[q] = __ldg(src + i);
  }
#pragma unroll
  for (int q = 0; q < kMaxLoads; ++q) {
    const int i = tid + q * 256;
    if (i < nk * vpr) {
      const int k = i / vpr, d = (i % vpr) * 8;
      const __half2* h = reinterpret_cast<const __half2*>(&buf[q]);
#pragma unroll
      for (int e = 0; e < 4; ++e) *reinterpret_cast<__half2*>(&tile[k][d + 2 * e]) = h[e];
    }
  }
  __syncthreads();
  uint8_t* sc_block = scales + (bh * NT + blockIdx.x) * 512;
  for (int t = tid; t < D * 4; t += blockDim.x) {
    const int d = t % D, g = t / D;  // consecutive lanes, consecutive channels: conflict-free column reads
    if (32 * g >= nk) continue;
    float x[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      x[i] = __half2float(tile[32 * g + i][d]);
      amax = fmaxf(amax, fabsf(x[i]));
    }
    float inv_x;
    const uint32_t sb = mx8_scale(amax, inv_x);
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // an all-zero group: zero codes
    if (amax > 0.f) mx8_encode32(x, inv_x, w);
    uint4* dst = reinterpret_cast<uint4*>(codes + (bh * D + d) * static_cast<size_t>(N) + n0 + 32 * g);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    sc_block[(d % 32) * 16 + (d / 32) * 4 + g] = static_cast<uint8_t>(sb);
  }
}

}  // namespace

size_t mx8_codes_bytes(const thrift_shape& s, thrift_operand op) {
  const size_t H = op == THRIFT_Q ? s.Hq : s.Hkv;
  return static_cast<size_t>(s.B) * H * s.N * s.D;
}

size_t mx8_scales_bytes(const thrift_shape& s, thrift_operand op) {
  const size_t H = op == THRIFT_Q ? s.Hq : s.Hkv;
  return static_cast<size_t>(s.B) * H * num_tiles(s.N) * 512;
}

cudaError_t launch_quantize_mx8(const void* x, thrift_operand op, const thrift_shape& s, void* codes, void* scales,
                                cudaStream_t st) {
  const size_t H = op == THRIFT_Q ? s.Hq : s.Hkv;
  const size_t bh = static_cast<size_t>(s.B) * H;
  cudaError_t e = cudaMemsetAsync(scales, 0, mx8_scales_bytes(s, op), st);
  if (e != cudaSuccess) return e;
  if (op == THRIFT_V) {
    quantize_v_mx8_kernel<<<dim3(num_tiles(s.N), static_cast<unsigned>(bh)), 256, 0, st>>>(
        static_cast<const __half*>(x), s.N, s.D, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
    return cudaGetLastError();
  }
  const size_t groups = bh * s.N * (s.D / 32);
  const size_t blocks = (groups + 255) / 256;
  const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
  quantize_qk_mx8_kernel<<<grid, 256, 0, st>>>(static_cast<const __half*>(x), bh * s.N, s.N, s.D,
                                               static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
  return cudaGetLastError();
}

}  // namespace thrift

// NVFP4 quantisation of the attention operands (HBM-bound).
//
// Q and K are encoded along D, V along the key axis, with one E4M3 scale per
// 16 consecutive elements: scale = E4M3_rn(fl32(amax / 6)),
// code = E2M1_rn(x / scale), a zero scale encoding the group as +0.  This is
// the block-scaled FP4 the method builds on ("ThriftAttention" abstract: the
// prior work's block-scaled quantisation on Blackwell), in the NVFP4 reading.
// The group encoder and its rounding argument are in nvfp4.cuh.
#include <cuda_fp16.h>

#include "common.h"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace thrift {
namespace {

// One thread per group of 16 along D.  rows = B*H*N.
__global__ void __launch_bounds__(256) quantize_qk_kernel(const __half* __restrict__ x, size_t rows, int N, int D,
                                                          uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ scales) {
  const int gpr = D / 16;  // groups per row
  const size_t total = rows * gpr;
  const int NT = num_tiles(N);
  for (size_t gi = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; gi < total;
       gi += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = gi / gpr;
    const int g = static_cast<int>(gi % gpr);
    const uint4* src = reinterpret_cast<const uint4*>(x + row * D + g * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    float v[16];
    const __half2* ha = reinterpret_cast<const __half2*>(&a);
    const __half2* hb = reinterpret_cast<const __half2*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __half22float2(ha[i]), fb = __half22float2(hb[i]);
      v[2 * i] = fa.x;
      v[2 * i + 1] = fa.y;
      v[8 + 2 * i] = fb.x;
      v[8 + 2 * i + 1] = fb.y;
    }
    const Group16 q = encode16(v);
    *reinterpret_cast<uint2*>(codes + row * (D / 2) + g * 8) = make_uint2(q.lo, q.hi);
    const size_t bh = row / N;
    const int n = static_cast<int>(row % N);
    scales[qk_scale_index(bh, n, g, NT, D)] = static_cast<uint8_t>(q.scale);
  }
}

// Padding of the Q/K scale blocks past N (rows N .. NT*128-1) is zero.
__global__ void zero_qk_scale_padding(size_t bh_count, int N, int D, uint8_t* __restrict__ scales) {
  const int NT = num_tiles(N);
  const int pad = NT * kTile - N;
  const int gpr = D / 16;
  const size_t total = bh_count * pad * gpr;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t bh = i / (static_cast<size_t>(pad) * gpr);
    const int rem = static_cast<int>(i % (static_cast<size_t>(pad) * gpr));
    const int n = N + rem / gpr, g = rem % gpr;
    scales[qk_scale_index(bh, n, g, NT, D)] = 0;
  }
}

// V along keys: one CTA per (bh, 64-key chunk).  The chunk [64][D] is staged
// through shared memory; thread (d, k16) encodes keys k16*16 .. +15 of
// channel d.  Chunks past N (padding to whole 128-key tiles) are all zero.
__global__ void __launch_bounds__(256) quantize_v_kernel(const __half* __restrict__ v, int N, int D,
                                                         uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  __shared__ __half tile[64][128 + 2];
  const int NT = num_tiles(N);
  const size_t bh = blockIdx.y;
  const int chunk = blockIdx.x;  // 0 .. 2*NT-1
  const int n0 = chunk * 64;
  const int tid = threadIdx.x;
  uint8_t* sc_block = scales + (bh * 2 * NT + chunk) * 512;
  if (n0 >= N) {
    for (int i = tid; i < 512; i += blockDim.x) sc_block[i] = 0;
    return;
  }
  // stage 64 keys x D channels (N is a multiple of 64, so the chunk is whole)
  const __half* src = v + (bh * N + n0) * D;
  for (int i = tid; i < 64 * D / 2; i += blockDim.x) {
    const int k = (2 * i) / D, d = (2 * i) % D;
    const __half2 h = reinterpret_cast<const __half2*>(src)[i];
    tile[k][d] = h.x;
    tile[k][d + 1] = h.y;
  }
  for (int i = tid; i < 512; i += blockDim.x) {
    // channels >= D of the scale block are padding
    const int r = i / 16, c = (i % 16) / 4;
    const int d = c * 32 + r;
    if (d >= D) sc_block[i] = 0;
  }
  __syncthreads();
  for (int t = tid; t < D * 4; t += blockDim.x) {
    const int d = t / 4, k16 = t % 4;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __half2float(tile[k16 * 16 + i][d]);
    const Group16 q = encode16(x);
    *reinterpret_cast<uint2*>(codes + (bh * D + d) * (static_cast<size_t>(N) / 2) + n0 / 2 + k16 * 8) =
        make_uint2(q.lo, q.hi);
    sc_block[(d % 32) * 16 + (d / 32) * 4 + k16] = static_cast<uint8_t>(q.scale);
  }
}

}  // namespace

cudaError_t launch_quantize_qk(const void* x, size_t rows, int N, int D, void* codes, void* scales,
                               cudaStream_t st) {
  const size_t groups = rows * (D / 16);
  const int threads = 256;
  const size_t blocks = (groups + threads - 1) / threads;
  const int grid = static_cast<int>(blocks < 148 * 64 ? blocks : 148 * 64);
  quantize_qk_kernel<<<grid, threads, 0, st>>>(static_cast<const __half*>(x), rows, N, D,
                                               static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (N % kTile) {
    const size_t bh = rows / N;
    zero_qk_scale_padding<<<148, 256, 0, st>>>(bh, N, D, static_cast<uint8_t*>(scales));
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_quantize_v(const void* v, size_t bh, int N, int D, void* codes, void* scales, cudaStream_t st) {
  dim3 grid(2 * num_tiles(N), static_cast<unsigned>(bh));
  quantize_v_kernel<<<grid, 256, 0, st>>>(static_cast<const __half*>(v), N, D, static_cast<uint8_t*>(codes),
                                          static_cast<uint8_t*>(scales));
  return cudaGetLastError();
}

}  // namespace thrift

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

// One thread per group of 16 along D, two groups (a grid stride apart) per
// step with all four 16-byte loads in flight before either is encoded.
// rows = B*H*N.
__global__ void __launch_bounds__(256) quantize_qk_kernel(const __half* __restrict__ x, size_t rows, int N, int D,
                                                          uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ scales) {
  const int gpr = D / 16;  // groups per row
  const size_t total = rows * gpr;
  const int NT = num_tiles(N);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const auto encode_store = [&](size_t gi, const uint4& a, const uint4& b) {
    const size_t row = gi / gpr;
    const int g = static_cast<int>(gi % gpr);
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
  };
  for (size_t gi = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; gi < total; gi += 2 * stride) {
    const size_t gj = gi + stride;
    const bool two = gj < total;
    const uint4* s0 = reinterpret_cast<const uint4*>(x + gi * 16);  // group gi starts at element 16 gi
    const uint4 a0 = __ldg(s0), b0 = __ldg(s0 + 1);
    uint4 a1 = make_uint4(0u, 0u, 0u, 0u), b1 = a1;
    if (two) {
      const uint4* s1 = reinterpret_cast<const uint4*>(x + gj * 16);
      a1 = __ldg(s1);
      b1 = __ldg(s1 + 1);
    }
    encode_store(gi, a0, b0);
    if (two) encode_store(gj, a1, b1);
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

// V along keys: one CTA per (bh, 128-key tile).  The tile [nk][D] (nk = 128,
// or 64 for the last tile when N is an odd multiple of 64) is staged through
// shared memory with 16-byte loads, all of a thread's loads in flight at once;
// task (d, k16) then encodes keys k16*16 .. +15 of channel d, consecutive lanes
// taking consecutive channels (conflict-free column reads).  The scale blocks
// of a tile are its two 64-key chunks; a chunk past N is all zero, and so are
// the channels >= D of every block.
constexpr int kVTile = 128, kVThreads = 256;

__global__ void __launch_bounds__(kVThreads) quantize_v_kernel(const __half* __restrict__ v, int N, int D,
                                                               uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ scales) {
  __shared__ __half tile[kVTile][128 + 2];
  const int NT = num_tiles(N);
  const size_t bh = blockIdx.y;
  const int n0 = blockIdx.x * kVTile;
  const int nk = min(kVTile, N - n0);  // 64 or 128 keys
  const int tid = threadIdx.x;
  uint8_t* sc_block = scales + (bh * 2 * NT + 2 * blockIdx.x) * 512;  // two 512-byte chunks
  for (int i = tid; i < 1024; i += kVThreads) {
    const int chunk = i / 512, r = (i % 512) / 16, c = (i % 16) / 4;
    if (chunk * 64 >= nk || c * 32 + r >= D) sc_block[i] = 0;  // padding: written by nobody else
  }
  const int vpr = D / 8;  // 16-byte pieces per key row
  const uint4* src = reinterpret_cast<const uint4*>(v + (bh * N + n0) * D);
  constexpr int kMaxLoads = kVTile * 128 / 8 / kVThreads;  // 8
  uint4 buf[kMaxLoads];
#pragma unroll
  for (int q = 0; q < kMaxLoads; ++q) {
    const int i = tid + q * kVThreads;
    if (i < nk * vpr) buf[q] = __ldg(src + i);
  }
#pragma unroll
  for (int q = 0; q < kMaxLoads; ++q) {
    const int i = tid + q * kVThreads;
    if (i < nk * vpr) {
      const int k = i / vpr, d = (i % vpr) * 8;
      const __half2* h = reinterpret_cast<const __half2*>(&buf[q]);
#pragma unroll
      for (int e = 0; e < 4; ++e) *reinterpret_cast<__half2*>(&tile[k][d + 2 * e]) = h[e];
    }
  }
  __syncthreads();
  for (int t = tid; t < D * (nk / 16); t += kVThreads) {
    const int d = t % D, k16 = t / D;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __half2float(tile[k16 * 16 + i][d]);
    const Group16 q = encode16(x);
    *reinterpret_cast<uint2*>(codes + (bh * D + d) * (static_cast<size_t>(N) / 2) + n0 / 2 + k16 * 8) =
        make_uint2(q.lo, q.hi);
    sc_block[(k16 / 4) * 512 + (d % 32) * 16 + (d / 32) * 4 + k16 % 4] = static_cast<uint8_t>(q.scale);
  }
}

// Q or K encoded along D and pooled in one pass (the fused entry points):
// one CTA per (selection block of blk rows, bh), 256 threads.  Thread t takes
// group g = t % (D/16) of rows t / (D/16), + 256 / (D/16), ... with all its
// 16-byte loads in flight, encodes each group exactly as quantize_qk_kernel
// does, and adds the group's values to 16 FP64 column sums.  The row slots'
// sums meet by shuffles within a warp and through shared memory across
// warps; the block mean is the sum / blk rounded once to FP32, as pool_kernel
// computes it.  FP64 sums of up to 8192 fp16 values are exact in any order
// (every partial sum is a multiple of 2^-24 below 2^29), so the means equal
// pool_kernel's bit for bit and the tensor is read from HBM once.
template <int D>
__global__ void __launch_bounds__(256) quantize_pool_qk_kernel(const __half* __restrict__ x, int N, int blk,
                                                               uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ scales,
                                                               float* __restrict__ means) {
  constexpr int G = D / 16;          // groups per row
  constexpr int kSlots = 256 / G;    // row slots
  constexpr int kMaxRows = 128 / kSlots;  // rows per thread for blk = 128 (4 for D = 128, 2 for D = 64)
  __shared__ double part[8][D];      // per warp, per channel
  const size_t bh = blockIdx.y;
  const int i = blockIdx.x, nb = N / blk;
  const int NT = num_tiles(N);
  const int g = threadIdx.x % G, slot = threadIdx.x / G;
  const int rows = blk / kSlots;     // rows of this thread (blk / kSlots <= kMaxRows)
  const size_t row0 = bh * N + static_cast<size_t>(i) * blk;
  uint4 a[kMaxRows], b[kMaxRows];
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q) {
    if (q < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (row0 + slot + q * kSlots) * D + g * 16);
      a[q] = __ldg(src);
      b[q] = __ldg(src + 1);
    }
  }
  double acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.0;
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q) {
    if (q < rows) {
      float v[16];
      const __half2* ha = reinterpret_cast<const __half2*>(&a[q]);
      const __half2* hb = reinterpret_cast<const __half2*>(&b[q]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __half22float2(ha[e]), fb = __half22float2(hb[e]);
        v[2 * e] = fa.x;
        v[2 * e + 1] = fa.y;
        v[8 + 2 * e] = fb.x;
        v[8 + 2 * e + 1] = fb.y;
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] += static_cast<double>(v[e]);
      const Group16 enc = encode16(v);
      const size_t row = row0 + slot + q * kSlots;
      *reinterpret_cast<uint2*>(codes + row * (D / 2) + g * 8) = make_uint2(enc.lo, enc.hi);
      const int n = i * blk + slot + q * kSlots;
      scales[qk_scale_index(bh, n, g, NT, D)] = static_cast<uint8_t>(enc.scale);
    }
  }
  // lanes with the same group: lane ^ G, lane ^ 2G, ... within the warp
#pragma unroll
  for (int off = G; off < 32; off *= 2)
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (lane < G)
#pragma unroll
    for (int e = 0; e < 16; ++e) part[warp][16 * lane + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += 256) {
    double sum = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += part[w][d];
    means[(bh * nb + i) * D + d] = static_cast<float>(sum / blk);
  }
}

}  // namespace

cudaError_t launch_quantize_pool_qk(const void* x, size_t bh_count, int N, int D, int blk, void* codes, void* scales,
                                    float* means, cudaStream_t st) {
  const dim3 grid(N / blk, static_cast<unsigned>(bh_count));
  if (D == 128)
    quantize_pool_qk_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __half*>(x), N, blk,
                                                       static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                                       means);
  else
    quantize_pool_qk_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __half*>(x), N, blk,
                                                      static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                                      means);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (N % kTile) {
    zero_qk_scale_padding<<<148, 256, 0, st>>>(bh_count, N, D, static_cast<uint8_t*>(scales));
    e = cudaGetLastError();
  }
  return e;
}

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
  dim3 grid(num_tiles(N), static_cast<unsigned>(bh));
  quantize_v_kernel<<<grid, kVThreads, 0, st>>>(static_cast<const __half*>(v), N, D, static_cast<uint8_t*>(codes),
                                          static_cast<uint8_t*>(scales));
  return cudaGetLastError();
}

}  // namespace thrift

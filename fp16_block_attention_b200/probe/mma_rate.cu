// Measurement helper, not part of the method's path and not part of
// libthrift.so: a separate library (libthrift_probe.so) that the benchmark's
// sweep loads to time the sustained issue and execution rate of the two
// tcgen05 MMA kinds the attention kernels use, so the FP4 and FP16 tensor
// peaks of the blended roofline can be checked on the machine at hand.  One CTA per SM allocates tensor memory, zeroes its shared-
// memory operands (so every product is exactly zero), and issues `iters`
// back-to-back M = 128, N = 256 products into one accumulator:
//   kind 0: .kind::mxf4nvf4.block_scale.scale_vec::4X, K = 64 (E2M1, UE4M3 scales)
//   kind 1: .kind::f16 (fp16 operands, fp32 accumulator), K = 16
// The caller times the launch; the work is iters x 2 x 128 x 256 x K flop per CTA.
#include <cuda_runtime.h>

#include "../csrc/common.h"
#include "../csrc/ptx.cuh"

namespace thrift {
namespace {

struct RateSmem {
  alignas(1024) uint8_t a[16384];  // fp16: 128 x 64 (SW128); FP4: 128 x 32 B (SW32)
  alignas(1024) uint8_t b[32768];  // fp16: 256 x 64 (SW128); FP4: 256 x 32 B (SW32)
  alignas(16) uint8_t sf[1024];    // zero scale factors
  alignas(8) uint64_t bar;
  uint32_t tmem;
};

template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, uint32_t* err) {
  extern __shared__ uint8_t raw[];
  RateSmem& s = *reinterpret_cast<RateSmem*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid / 32;
  for (int i = tid; i < 16384 / 16; i += 128) reinterpret_cast<uint4*>(s.a)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < 32768 / 16; i += 128) reinterpret_cast<uint4*>(s.b)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < 1024 / 16; i += 128) reinterpret_cast<uint4*>(s.sf)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    mbar_init(&s.bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = s.tmem;
  if (tid == 0) {
    // columns: accumulator 0..255, A scales 256.., B scales 272..
    const uint32_t sfa = tm + 256, sfb = tm + 272;
    if (KIND == 0)
      for (int c = 0; c < 2; ++c) {
        tmem_cp_32x128b_x4(sfa + 4 * c, make_sdesc(smem_u32(s.sf) + 512 * c, 16, 128, LAYOUT_NONE));
        tmem_cp_32x128b_x4(sfb + 4 * c, make_sdesc(smem_u32(s.sf) + 512 * c, 16, 128, LAYOUT_NONE));
      }
    const uint64_t ad = KIND == 0 ? make_sdesc(smem_u32(s.a), 16, 256, LAYOUT_SW32)
                                  : make_sdesc(smem_u32(s.a), 16, 1024, LAYOUT_SW128);
    const uint64_t bd = KIND == 0 ? make_sdesc(smem_u32(s.b), 16, 256, LAYOUT_SW32)
                                  : make_sdesc(smem_u32(s.b), 16, 1024, LAYOUT_SW128);
    for (int it = 0; it < iters; ++it) {
      if (KIND == 0)
        mma_nvf4(tm, ad, bd, idesc_nvf4(128, 256), sfa, sfb, it > 0);
      else
        mma_f16(tm, ad, bd, idesc_f16(128, 256, false), it > 0);
    }
    mma_commit(&s.bar);
    if (!mbar_wait(&s.bar, 0, kWaitNs)) record_error(err, DEV_TIMEOUT_MMA);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// The probe's own device error word (bounded-wait timeouts).
__device__ uint32_t g_probe_error;

cudaError_t launch_mma_rate(int kind, int iters, int ctas, uint32_t* err, cudaStream_t st) {
  const size_t smem = sizeof(RateSmem) + 1024;
  cudaError_t e;
  if (kind == 0) {
    e = cudaFuncSetAttribute(mma_rate_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mma_rate_kernel<0><<<ctas, 128, smem, st>>>(iters, err);
  } else {
    e = cudaFuncSetAttribute(mma_rate_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mma_rate_kernel<1><<<ctas, 128, smem, st>>>(iters, err);
  }
  return cudaGetLastError();
}

}  // namespace
}  // namespace thrift

#define PROBE_API extern "C" __attribute__((visibility("default")))

// Launch one CTA per SM of the current device, each issuing `iters`
// back-to-back M = 128, N = 256 products of `kind` (0: NVFP4 K = 64, 1: fp16
// K = 16), asynchronously on `stream`.  Returns 0, 1 for kind not in {0, 1} or
// iters not in [1, 2^24] (checked before any launch), 3 for a CUDA error.
PROBE_API int thrift_probe_mma_rate(int kind, int iters, void* stream) {
  if (kind < 0 || kind > 1 || iters <= 0 || iters > (1 << 24)) return 1;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 3;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 3;
  void* err = nullptr;
  if (cudaGetSymbolAddress(&err, thrift::g_probe_error) != cudaSuccess) return 3;
  return thrift::launch_mma_rate(kind, iters, nsm, static_cast<uint32_t*>(err), static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? 0
             : 3;
}

// Synchronise `stream`, read and clear the probe's error word: 0, or 4 if a
// probe kernel gave up its bounded wait; 3 for a CUDA error.
PROBE_API int thrift_probe_last_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return 3;
  void* err = nullptr;
  if (cudaGetSymbolAddress(&err, thrift::g_probe_error) != cudaSuccess) return 3;
  uint32_t v = 0;
  if (cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return 3;
  if (v == 0) return 0;
  const uint32_t zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return 3;
  return 4;
}

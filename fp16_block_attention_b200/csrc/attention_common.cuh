// Device helpers shared by the attention kernels: launch parameters, bounded
// mbarrier waits that raise a CTA-wide abort flag, the softmax threads' joint
// barrier, and small arithmetic helpers (ex2 / lg2 on the MUFU, three-input
// max, tree sums, fp16 packing).
#pragma once
#include <cuda_fp16.h>

#include "common.h"
#include "ptx.cuh"

namespace thrift {
namespace attn {

struct Params {
  const uint8_t* mask;
  const uint8_t* qs;
  const uint8_t* ks;
  const uint8_t* vs;
  __half* O;
  uint32_t* err;
  int B, Hq, Hkv, N, blk, causal, NT;
  float scale_log2;
  int skip;  // the mask may hold 2 (skipped pairs): the kernels' skip-aware instantiations
  // MXFP8 scales of Q, K, V for 8-bit pairs (mask 3; blk = 128 only), or null
  const uint8_t* qs8;
  const uint8_t* ks8;
  const uint8_t* vs8;
  int eight;  // the MXFP8 copies are present: the 8-bit instantiation
  uint64_t wait_ns;  // bound of every wait in the kernel (thrift_set_wait_limit)
  int withhold;      // failure-detection test only: the processed key tile whose copies the producer
                     // does not issue (its consumers' waits then run out), or -1
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* err,
                                              uint32_t code, uint64_t limit_ns = kWaitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < (1u << 30); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 63u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        record_error(err, code);
        *abort = 1;
        return false;
      }
    }
  }
  record_error(err, code);
  *abort = 1;
  return false;
}

// The same wait with its slow path (timer, abort flag, error record) out of
// line: one try_wait, which the hardware already suspends for a while, stays
// inline.  All warp roles' loops run at once on an SM and share its
// instruction caches, so where a kernel's waits sit decides how often its
// warps stall on instruction fetch; a kernel picks the form per role by
// measurement.  TAG makes separate copies of the slow path: a kernel whose
// warpgroups run with different register counts (setmaxnreg) gives each
// count its own copy, since one function cannot be allocated for both.
template <int TAG>
static __device__ __noinline__ bool wait_or_abort_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                       uint32_t* err, uint32_t code, uint64_t limit_ns) {
  return wait_or_abort(bar, parity, abort, err, code, limit_ns);
}

template <bool OUT_OF_LINE, int TAG = 0>
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* err,
                                             uint32_t code, uint64_t limit_ns) {
  if constexpr (OUT_OF_LINE) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_or_abort_slow<TAG>(bar, parity, abort, err, code, limit_ns);
  } else {
    return wait_or_abort(bar, parity, abort, err, code, limit_ns);
  }
}

// Named barrier of the softmax threads that also ORs a per-thread flag,
// so that every softmax thread takes the same exit decision.
template <int NT>
__device__ __forceinline__ bool softmax_bar_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(flag)), "n"(NT)
      : "memory");
  return r != 0;
}


// The same on named barrier ID (ID != 0, 1 if another use of barrier 1 could interleave).
template <int ID, int NT>
__device__ __forceinline__ bool bar_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(flag)), "n"(ID), "n"(NT)
      : "memory");
  return r != 0;
}

// Barrier of all `count` threads of the CTA that warps may reach from
// different places in the code (barrier 2, not the aligned __syncthreads).
__device__ __forceinline__ void cta_barrier_all(uint32_t count) {
  asm volatile("barrier.sync 2, %0;" ::"r"(count) : "memory");
}

// Named barriers among a subset of the CTA's warps (count = threads taking part).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_bar_arrive(uint32_t id, uint32_t count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float max16(const float* v) {
  const float a = fmax3(v[0], v[1], v[2]), b = fmax3(v[3], v[4], v[5]), c = fmax3(v[6], v[7], v[8]);
  const float d = fmax3(v[9], v[10], v[11]), e = fmax3(v[12], v[13], v[14]);
  return fmaxf(fmax3(a, b, c), fmax3(d, e, v[15]));
}

// Pairwise (tree) sum of 16 values with packed two-lane adds: the same
// additions in the same order as a scalar tree, half the instructions.
__device__ __forceinline__ float sum16(const float* v) {
  float2 t0 = __fadd2_rn(make_float2(v[0], v[1]), make_float2(v[8], v[9]));
  float2 t1 = __fadd2_rn(make_float2(v[2], v[3]), make_float2(v[10], v[11]));
  const float2 t2 = __fadd2_rn(make_float2(v[4], v[5]), make_float2(v[12], v[13]));
  const float2 t3 = __fadd2_rn(make_float2(v[6], v[7]), make_float2(v[14], v[15]));
  t0 = __fadd2_rn(t0, t2);
  t1 = __fadd2_rn(t1, t3);
  const float2 u = __fadd2_rn(t0, t1);
  return u.x + u.y;
}

// Two exponentials 2^(s * c + b) with one packed FMA.
__device__ __forceinline__ float2 ex2_fma2(float s0, float s1, float2 c, float2 b) {
  const float2 t = __ffma2_rn(make_float2(s0, s1), c, b);
  return make_float2(ex2(t.x), ex2(t.y));
}

// 2^e for an integer-valued e <= 0 (0 below the normal range).
__device__ __forceinline__ float exp2_int(float e) {
  const int i = static_cast<int>(e);
  return (i < -126) ? 0.f : __int_as_float((127 + i) << 23);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


}  // namespace attn

// Kernel with double-buffered S and P for 128 x 128 selection blocks
// (attention_db.cu).  The MXFP8 maps are read only when prm.eight is set.
template <int D>
cudaError_t launch_attention_db(const CUtensorMap& mQ16, const CUtensorMap& mK16, const CUtensorMap& mV16,
                                const CUtensorMap& mQ4, const CUtensorMap& mK4, const CUtensorMap& mV4,
                                const CUtensorMap& mQ8, const CUtensorMap& mK8, const CUtensorMap& mV8,
                                const attn::Params& prm, cudaStream_t st);

}  // namespace thrift

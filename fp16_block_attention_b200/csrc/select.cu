// Stage 1 of the method (ThriftAttention abstract): a cheap heuristic picks
// the few query-key block pairs that matter most and marks them for FP16.
// Reading used here: pooled scores from FP32 block means,
// score(i,j) = fl32(sm_scale * fl32(mean_q(i) . mean_k(j))), and per
// (batch, query head) the top k = ceil(rho * #valid - 1e-9) pairs, with the
// diagonal pairs (i,i) and the key-block-0 pairs (i,0) ranked first and ties
// broken by the lower linear index i*nb + j.
//
// Three kernels:
//   pool     block means: the FP64 sum of a block's fp16 rows is exact in any
//            order (40-bit span + log2(blk) bits < 53), divided by blk and
//            rounded once to FP32;
//   scores   the FP64 dot product of two FP32 means (products exact in FP64),
//            rounded to FP32, times sm_scale in FP32;
//   top-k    one CTA per head: radix select of the k-th largest 64-bit key
//            (forced bit | order-preserving score bits | inverted index), so
//            the selection is exactly k pairs, then the mask.
//
// A second selector, after HyQuant (abstract in the body of the page titled
// "LampAttention: Look-Ahead Mixed-Precision FlashAttention for Dedicated
// Accelerators"): there, the keys that many queries attend to (vertical lines
// of the attention map) and a sliding window next to the diagonal keep full
// precision, picked by a cheap attention-pattern signal.  Here the same idea
// at block granularity and on the same budget k:
//   column signal  per (batch, query head), from the same pooled scores: the
//            softmax of each valid row of block scores, summed per key-block
//            column (the attention mass a key block receives), in FP32 and in
//            a fixed order; columns ranked by it (ties: lower column first);
//   top-k    the same radix select on the key (window bit | inverted column
//            rank | order-preserving score bits | inverted index): the pairs
//            of the local window (i - W < j <= i, or |i - j| < W without the
//            causal mask) first, then whole columns in rank order, each by
//            descending score.
#include <cuda_fp16.h>

#include "common.h"

namespace thrift {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct SelectWs {
  float* qm;      // [B*Hq][nb][D]
  float* km;      // [B*Hkv][nb][D]
  float* scores;  // [B*Hq][nb][nb]
  int* rank;      // [B*Hq][nb] column ranks (vertical-line selector)
};

SelectWs carve(void* ws, const thrift_shape& s) {
  const int nb = s.N / s.blk;
  char* p = static_cast<char*>(ws);
  SelectWs w;
  w.qm = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * static_cast<size_t>(s.B) * s.Hq * nb * s.D);
  w.km = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * static_cast<size_t>(s.B) * s.Hkv * nb * s.D);
  w.scores = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * static_cast<size_t>(s.B) * s.Hq * nb * nb);
  w.rank = reinterpret_cast<int*>(p);
  return w;
}

// grid (nb, BH), block D/2 threads, two channels per thread.
__global__ void pool_kernel(const __half* __restrict__ x, int N, int D, int blk, float* __restrict__ out) {
  const int nb = N / blk;
  const size_t bh = blockIdx.y;
  const int i = blockIdx.x;
  const int c = threadIdx.x;  // channel pair
  const __half2* src = reinterpret_cast<const __half2*>(x + (bh * N + static_cast<size_t>(i) * blk) * D) + c;
  double s0 = 0.0, s1 = 0.0;
  for (int r = 0; r < blk; ++r) {
    const float2 f = __half22float2(src[static_cast<size_t>(r) * (D / 2)]);
    s0 += static_cast<double>(f.x);
    s1 += static_cast<double>(f.y);
  }
  float* dst = out + (bh * nb + i) * D + 2 * c;
  dst[0] = static_cast<float>(s0 / blk);
  dst[1] = static_cast<float>(s1 / blk);
}

// grid (ceil(nb/32), ceil(nb/32), B*Hq), block 256: a 32x32 tile of scores,
// each thread a 2x2 sub-tile.
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ qm, const float* __restrict__ km,
                                                    int Hq, int Hkv, int nb, int D, int causal, float sm_scale,
                                                    float* __restrict__ scores) {
  __shared__ float qs[32][129];
  __shared__ float ks[32][129];
  const int bi = blockIdx.y * 32, bj = blockIdx.x * 32;
  if (causal && bj > bi + 31) return;
  const size_t bh = blockIdx.z;
  const size_t b = bh / Hq, hq = bh % Hq;
  const size_t bhk = b * Hkv + hq / (Hq / Hkv);
  for (int t = threadIdx.x; t < 32 * D; t += blockDim.x) {
    const int r = t / D, d = t % D;
    qs[r][d] = (bi + r < nb) ? qm[(bh * nb + bi + r) * D + d] : 0.0f;
    ks[r][d] = (bj + r < nb) ? km[(bhk * nb + bj + r) * D + d] : 0.0f;
  }
  __syncthreads();
  const int ti = (threadIdx.x / 16) * 2, tj = (threadIdx.x % 16) * 2;
  double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  for (int d = 0; d < D; ++d) {
    const double q0 = qs[ti][d], q1 = qs[ti + 1][d], k0 = ks[tj][d], k1 = ks[tj + 1][d];  // exact widening
    acc[0][0] = fma(q0, k0, acc[0][0]);
    acc[0][1] = fma(q0, k1, acc[0][1]);
    acc[1][0] = fma(q1, k0, acc[1][0]);
    acc[1][1] = fma(q1, k1, acc[1][1]);
  }
  for (int a = 0; a < 2; ++a)
    for (int c = 0; c < 2; ++c) {
      const int i = bi + ti + a, j = bj + tj + c;
      if (i < nb && j < nb && (!causal || j <= i))
        scores[(bh * nb + i) * nb + j] = __fmul_rn(sm_scale, static_cast<float>(acc[a][c]));
    }
}

__device__ __forceinline__ uint64_t pair_key(float score, int i, int j, int nb) {
  if (score == 0.0f) score = 0.0f;  // one zero
  uint32_t u = __float_as_uint(score);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  const uint64_t forced = (i == j || j == 0) ? 1ull : 0ull;
  const uint64_t idx = static_cast<uint64_t>(i) * nb + j;
  return (forced << 63) | (static_cast<uint64_t>(u) << 31) | (0x7FFFFFFFull - idx);
}

// Key of the vertical-line / local-window selector: window bit (63), inverted
// column rank (11 bits, 52..62), order-preserving score bits (20..51),
// inverted query block (11 bits).  Ranks are a permutation of the columns, so
// the rank fixes j and the key is unique; nb <= 2048.
__device__ __forceinline__ uint64_t vw_key(float score, int i, int j, int causal, int window, int rank) {
  if (score == 0.0f) score = 0.0f;
  uint32_t u = __float_as_uint(score);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  const bool in_window = causal ? (j <= i && j > i - window) : (abs(i - j) < window);
  return (static_cast<uint64_t>(in_window) << 63) | (static_cast<uint64_t>(2047 - rank) << 52) |
         (static_cast<uint64_t>(u) << 20) | static_cast<uint64_t>(2047 - i);
}

// Column signal and ranks of the vertical-line selector, one CTA (1024
// threads) per (batch, query head); nb <= kMaxVWBlocks.  Deterministic: every
// sum has a fixed order.
__global__ void __launch_bounds__(1024) column_rank_kernel(const float* __restrict__ scores, int nb, int causal,
                                                           int* __restrict__ rank_out) {
  __shared__ float rmax[kMaxVWBlocks], rinv[kMaxVWBlocks], colv[kMaxVWBlocks];
  const size_t bh = blockIdx.x;
  const float* sc = scores + bh * nb * static_cast<size_t>(nb);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // row softmax of the valid block scores: maximum and 1 / sum of exponentials
  for (int i = warp; i < nb; i += 32) {
    const int jn = causal ? i + 1 : nb;
    float m = -INFINITY;
    for (int j = lane; j < jn; j += 32) m = fmaxf(m, sc[static_cast<size_t>(i) * nb + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float d = 0.f;
    for (int j = lane; j < jn; j += 32) d += expf(sc[static_cast<size_t>(i) * nb + j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) {
      rmax[i] = m;
      rinv[i] = 1.0f / d;
    }
  }
  __syncthreads();
  // attention mass each key-block column receives, summed over rows in order
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    float a = 0.f;
    for (int i = causal ? j : 0; i < nb; ++i) a += expf(sc[static_cast<size_t>(i) * nb + j] - rmax[i]) * rinv[i];
    colv[j] = a;
  }
  __syncthreads();
  // rank: columns with a larger signal, or an equal one and a lower index
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const float vj = colv[j];
    int rk = 0;
    for (int jj = 0; jj < nb; ++jj) {
      const float x = colv[jj];
      rk += (x > vj || (x == vj && jj < j)) ? 1 : 0;
    }
    rank_out[bh * nb + j] = rk;
  }
}

// One CTA (1024 threads) per (batch, query head).  VW = 0: the method's key;
// VW = 1: the vertical-line / local-window key (column ranks in `rank`).
// The first k pairs by key are marked 1, the next ones up to the k8end-th 3
// (8-bit); with keep < #valid the pairs after the first `keep` are marked 2
// (skipped; the caller keeps them clear of forced, FP16 and 8-bit pairs), the
// rest 0.
template <int VW>
__global__ void __launch_bounds__(1024) topk_kernel(const float* __restrict__ scores, int nb, int causal,
                                                    long long k, long long k8end, long long keep,
                                                    uint8_t* __restrict__ mask,
                                                    const int* __restrict__ rank, int window) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_remaining;
  __shared__ int s_done;
  __shared__ int s_rank[VW ? kMaxVWBlocks : 1];
  const size_t bh = blockIdx.x;
  if (VW) {
    for (int j = threadIdx.x; j < nb; j += blockDim.x) s_rank[j] = rank[bh * nb + j];
    __syncthreads();
  }
  const auto key_of = [&](float score, int i, int j) -> uint64_t {
    if (VW) return vw_key(score, i, j, causal, window, s_rank[j]);
    return pair_key(score, i, j, nb);
  };
  const float* sc = scores + bh * nb * static_cast<size_t>(nb);
  uint8_t* m = mask + bh * nb * static_cast<size_t>(nb);
  const size_t total = static_cast<size_t>(nb) * nb;
  const long long valid = causal ? static_cast<long long>(nb) * (nb + 1) / 2 : static_cast<long long>(total);

  // Key of the kk-th largest valid pair (1 <= kk < valid) by an 8-bit radix
  // select: the first kk pairs are exactly those with key >= the result.
  const auto kth_largest = [&](long long kk) -> uint64_t {
    __syncthreads();  // every thread has read the previous result
    if (threadIdx.x == 0) {
      s_prefix = 0;
      s_remaining = kk;
      s_done = 0;
    }
    uint64_t pmask = 0;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0;
      __syncthreads();
      const uint64_t prefix = s_prefix;
      for (size_t idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int i = static_cast<int>(idx / nb), j = static_cast<int>(idx % nb);
        if (causal && j > i) continue;
        const uint64_t key = key_of(sc[idx], i, j);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        long long rem = s_remaining, cum = 0;
        int digit = 0;
        for (int d = 255; d >= 0; --d) {
          if (cum + hist[d] >= rem) {
            digit = d;
            break;
          }
          cum += hist[d];
        }
        rem -= cum;
        s_prefix = prefix | (static_cast<uint64_t>(digit) << shift);
        s_remaining = rem;
        s_done = (static_cast<long long>(hist[digit]) == rem);
      }
      __syncthreads();
      pmask |= 255ull << shift;
      if (s_done) break;
    }
    return s_prefix;
  };

  const bool select_none = k <= 0, select_all = k >= valid;
  const uint64_t threshold = (select_none || select_all) ? 0ull : kth_largest(k);  // FP16: key >= threshold
  const bool eight_any = k8end > k && k8end > 0 && k < valid, eight_all = k8end >= valid;
  const uint64_t eight_from = (eight_any && !eight_all) ? kth_largest(k8end) : 0ull;  // 8-bit: key >= eight_from
  const bool skip_any = keep < valid;
  const uint64_t keep_from = (skip_any && keep > 0) ? kth_largest(keep) : 0ull;  // skipped: key < keep_from
  for (size_t idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int i = static_cast<int>(idx / nb), j = static_cast<int>(idx % nb);
    uint8_t v = 0;
    if (!(causal && j > i)) {
      const uint64_t key = key_of(sc[idx], i, j);
      if (!select_none && (select_all || key >= threshold))
        v = 1;
      else if (eight_any && (eight_all || key >= eight_from))
        v = 3;
      else if (skip_any && (keep <= 0 || key < keep_from))
        v = 2;
    }
    m[idx] = v;
  }
}

}  // namespace

size_t select_workspace_bytes(const thrift_shape& s) {
  const size_t nb = s.N / s.blk;
  return align_up(sizeof(float) * s.B * s.Hq * nb * s.D) + align_up(sizeof(float) * s.B * s.Hkv * nb * s.D) +
         align_up(sizeof(float) * s.B * s.Hq * nb * nb) + align_up(sizeof(int) * s.B * s.Hq * nb);
}

namespace {
long long valid_pairs(const thrift_shape& s) {
  const long long nb = s.N / s.blk;
  return s.causal ? nb * (nb + 1) / 2 : nb * nb;
}

long long budget_pairs(const thrift_shape& s, double rho) {
  const long long valid = valid_pairs(s);
  double kk = ceil(rho * static_cast<double>(valid) - 1e-9);
  if (kk < 0) kk = 0;
  if (kk > static_cast<double>(valid)) kk = static_cast<double>(valid);
  return static_cast<long long>(kk);
}

void launch_pool_and_scores(const void* Q, const void* K, const thrift_shape& s, const SelectWs& w, cudaStream_t st) {
  const int nb = s.N / s.blk;
  pool_kernel<<<dim3(nb, s.B * s.Hq), s.D / 2, 0, st>>>(static_cast<const __half*>(Q), s.N, s.D, s.blk, w.qm);
  pool_kernel<<<dim3(nb, s.B * s.Hkv), s.D / 2, 0, st>>>(static_cast<const __half*>(K), s.N, s.D, s.blk, w.km);
  const int tiles = (nb + 31) / 32;
  score_kernel<<<dim3(tiles, tiles, s.B * s.Hq), 256, 0, st>>>(w.qm, w.km, s.Hq, s.Hkv, nb, s.D, s.causal,
                                                               s.sm_scale, w.scores);
}
}  // namespace

cudaError_t launch_pool_keys(const void* K, const thrift_shape& s, float* km, cudaStream_t st) {
  const int nb = s.N / s.blk;
  pool_kernel<<<dim3(nb, s.B * s.Hkv), s.D / 2, 0, st>>>(static_cast<const __half*>(K), s.N, s.D, s.blk, km);
  return cudaGetLastError();
}

cudaError_t launch_select_vertical_window(const void* Q, const void* K, const thrift_shape& s, double rho, int window,
                                          uint8_t* mask, void* ws, cudaStream_t st) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  launch_pool_and_scores(Q, K, s, w, st);
  column_rank_kernel<<<s.B * s.Hq, 1024, 0, st>>>(w.scores, nb, s.causal, w.rank);
  const long long k = budget_pairs(s, rho);
  topk_kernel<1><<<s.B * s.Hq, 1024, 0, st>>>(w.scores, nb, s.causal, k, k, valid_pairs(s), mask, w.rank, window);
  return cudaGetLastError();
}

cudaError_t launch_select(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask, void* ws,
                          cudaStream_t st) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  launch_pool_and_scores(Q, K, s, w, st);
  const long long k = budget_pairs(s, rho);
  topk_kernel<0><<<s.B * s.Hq, 1024, 0, st>>>(w.scores, nb, s.causal, k, k, valid_pairs(s), mask, nullptr, 0);
  return cudaGetLastError();
}

cudaError_t launch_select_tiered(const void* Q, const void* K, const thrift_shape& s, double rho, double rho8,
                                 double sigma, uint8_t* mask, void* ws, cudaStream_t st) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  launch_pool_and_scores(Q, K, s, w, st);
  // 8-bit pairs: the k8 after the FP16 ones; skipped pairs: the last ks of the
  // ranking, clear of the forced, FP16 and 8-bit pairs
  const long long n = valid_pairs(s), k16 = budget_pairs(s, rho);
  long long k8 = budget_pairs(s, rho8);
  if (k8 > n - k16) k8 = n - k16;
  const long long forced = 2LL * nb - 1;  // the diagonal and key block 0, (0, 0) once
  long long ks = budget_pairs(s, sigma);
  const long long cap = n - (k16 + k8 > forced ? k16 + k8 : forced);
  if (ks > cap) ks = cap;
  if (ks < 0) ks = 0;
  topk_kernel<0><<<s.B * s.Hq, 1024, 0, st>>>(w.scores, nb, s.causal, k16, k16 + k8, n - ks, mask, nullptr, 0);
  return cudaGetLastError();
}

// ---- selection without a caller-supplied workspace ------------------------
// Some callers cannot allocate device memory: their GPU memory belongs to
// another allocator (a framework's caching pool, a serving runtime that
// reserves the device at start-up), or they are hooks that the host program
// calls without any way to allocate.  For them the selection can run on a
// scratch array that lives in the library's own static device memory.  Every
// device that loads the library holds this array until the process exits.
// All calls share it and it keeps the last call's contents; the selection
// kernels overwrite everything they read (block means, then the scores of
// every valid pair), so nothing needs clearing between calls.  Calls whose
// kernels overlap on the GPU (for example on two streams) race on it.
namespace {
__device__ __align__(256) unsigned char g_select_scratch[kSelectStaticBytes];
constexpr int kMaxScratchDevices = 64;
void* g_select_scratch_ptr[kMaxScratchDevices] = {nullptr};
}  // namespace

// Host code must not pass `g_select_scratch` itself to a kernel: on the host
// that name is only a stand-in for the device array.  Its device address is
// looked up once per device, with that device current, on the first call.
cudaError_t select_static_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  if (!g_select_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_select_scratch_ptr[dev] = p;
  }
  *ptr = g_select_scratch_ptr[dev];
  return cudaSuccess;
}

cudaError_t launch_select_static(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask,
                                 cudaStream_t st) {
  void* scratch = nullptr;
  cudaError_t e = select_static_scratch(&scratch);
  if (e != cudaSuccess) return e;
  return launch_select(Q, K, s, rho, mask, scratch, st);
}

}  // namespace thrift

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
#include <atomic>
#include <cooperative_groups.h>
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

// grid (nb, BH), block kPoolThreads: the block of blk rows x D channels is
// read in 16-byte pieces (8 channels), thread t taking chunk t % (D/8) of rows
// t / (D/8), + kPoolThreads / (D/8), ..., all its loads in flight at once;
// the row groups' partial sums meet in shared memory.  FP64 sums of fp16
// values are exact in any order (every fp16 value is a multiple of 2^-24 below
// 2^16), so the mean is fl32(exact sum / blk) whatever the split.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __half* __restrict__ x, int N, int D, int blk,
                                                            float* __restrict__ out) {
  __shared__ double part[kPoolThreads * 8];  // [row group][D]
  const int nb = N / blk;
  const size_t bh = blockIdx.y;
  const int i = blockIdx.x;
  const int chunks = D / 8, groups = kPoolThreads / chunks, rows = blk / groups;
  const int cc = threadIdx.x % chunks, rg = threadIdx.x / chunks;
  const uint4* src = reinterpret_cast<const uint4*>(x + (bh * N + static_cast<size_t>(i) * blk) * D) + cc;
  double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  constexpr int kMaxRows = 8;  // blk <= 128, D >= 64: at most 128 / 16 rows per thread
  uint4 v[kMaxRows];
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q)
    if (q < rows) v[q] = __ldg(src + static_cast<size_t>(rg + q * groups) * chunks);
#pragma unroll
  for (int q = 0; q < kMaxRows; ++q) {
    if (q < rows) {
      const __half2* h = reinterpret_cast<const __half2*>(&v[q]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        acc[2 * e] += static_cast<double>(f.x);
        acc[2 * e + 1] += static_cast<double>(f.y);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg * D + 8 * cc + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += kPoolThreads) {
    double sum = 0.0;
    for (int g = 0; g < groups; ++g) sum += part[g * D + d];
    out[(bh * nb + i) * D + d] = static_cast<float>(sum / blk);
  }
}

// score[i][j] = fl32(sm_scale * fl32(qmean_i . kmean_j)) for one (batch,
// query head) and a 64 x 64 tile of block pairs (tiles wholly above the causal
// diagonal skipped).  The products of two FP32 means are exact in FP64 and
// each dot is summed over the channels in order, in FP64, and rounded once.
// 256 threads, thread (ty, tx) owning the 4 x 4 pairs (bi + ty + 16 a,
// bj + tx + 16 c): per channel it reads four query and four key means (FP64,
// widened once as 32-channel slices are staged) for sixteen FMAs.  The key
// rows sit 33 doubles apart, so the sixteen rows a half-warp reads fall in
// distinct bank pairs.
constexpr int kScoreTile = 64;
constexpr int kScoreSlice = 32;  // channels staged at a time
__global__ void __launch_bounds__(256) score_kernel(const float* __restrict__ qm, const float* __restrict__ km,
                                                    int Hq, int Hkv, int nb, int D, int causal, float sm_scale,
                                                    float* __restrict__ scores) {
  __shared__ double qs[kScoreTile][kScoreSlice + 1];
  __shared__ double ks[kScoreTile][kScoreSlice + 1];
  const int bi = blockIdx.y * kScoreTile, bj = blockIdx.x * kScoreTile;
  if (causal && bj > bi + kScoreTile - 1) return;
  const size_t bh = blockIdx.z;
  const size_t b = bh / Hq, hq = bh % Hq;
  const size_t bhk = b * Hkv + hq / (Hq / Hkv);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.0;
  for (int d0 = 0; d0 < D; d0 += kScoreSlice) {
    __syncthreads();  // the previous slice has been read
    for (int t = threadIdx.x; t < kScoreTile * kScoreSlice; t += blockDim.x) {
      const int r = t / kScoreSlice, d = t % kScoreSlice;
      qs[r][d] = (bi + r < nb) ? static_cast<double>(qm[(bh * nb + bi + r) * D + d0 + d]) : 0.0;
      ks[r][d] = (bj + r < nb) ? static_cast<double>(km[(bhk * nb + bj + r) * D + d0 + d]) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int d = 0; d < kScoreSlice; ++d) {
      double qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = qs[ty + 16 * a][d];
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = ks[tx + 16 * c][d];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fma(qv[a], kv[c], acc[a][c]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = bi + ty + 16 * a, j = bj + tx + 16 * c;
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
// A head's selection runs on a cluster of kTopkCluster CTAs: CTA c of the
// cluster takes rows c, c + kTopkCluster, ... (balanced under the causal
// triangle).  Each radix pass, every CTA histograms its rows into its own
// shared memory; after a cluster barrier, warp 0 of every CTA sums all the
// cluster's histograms through distributed shared memory and finds the same
// digit (the sum is the same everywhere, so no CTA has to broadcast it); a
// second barrier keeps any histogram from being cleared, or its CTA from
// exiting, while another CTA still reads it.
constexpr int kTopkCluster = 4;

template <int VW>
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(1024)
    topk_kernel(const float* __restrict__ scores, int nb, int causal, long long k, long long k8end, long long keep,
                uint8_t* __restrict__ mask, const int* __restrict__ rank, int window) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_remaining;
  __shared__ int s_done;
  __shared__ int s_rank[VW ? kMaxVWBlocks : 1];
  const size_t bh = blockIdx.x / kTopkCluster;
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
  // Each pass histograms the digit of the keys that match the prefix found so
  // far: warp w walks rows w, w + 32, ... (only the valid columns), so all
  // lanes of a warp run the same trip count; lanes with equal digits add
  // their count once (the top digits of the keys are shared by most pairs);
  // warp 0 then finds the digit that holds the kk-th key with a shuffle scan.
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nwarps = blockDim.x / 32;
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
      for (int i = crank + kTopkCluster * warp; i < nb; i += kTopkCluster * nwarps) {
        const int ncol = causal ? i + 1 : nb;
        const float* row = sc + static_cast<size_t>(i) * nb;
        for (int j0 = 0; j0 < ncol; j0 += 128) {  // four column chunks, loads first
          float v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) v[q] = (j0 + 32 * q + lane < ncol) ? row[j0 + 32 * q + lane] : 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = j0 + 32 * q + lane;
            bool match = false;
            uint32_t bin = 0;
            if (j < ncol) {
              const uint64_t key = key_of(v[q], i, j);
              match = (key & pmask) == prefix;
              bin = static_cast<uint32_t>(key >> shift) & 255u;
            }
            const uint32_t active = __ballot_sync(0xffffffffu, match);
            if (match) {
              const uint32_t peers = __match_any_sync(active, bin);
              if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<unsigned int>(__popc(peers)));
            }
          }
        }
      }
      cluster.sync();  // every CTA's histogram of this pass is complete
      if (warp == 0) {
        // lane l holds bins 255 - 8 l .. 248 - 8 l, highest first, summed over the cluster
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) c[t] = 0;
        for (int rk = 0; rk < kTopkCluster; ++rk) {
          const unsigned int* h = cluster.map_shared_rank(hist, rk);
#pragma unroll
          for (int t = 0; t < 8; ++t) c[t] += h[255 - 8 * lane - t];
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) tot += c[t];
        uint32_t incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const long long rem = s_remaining;
        const long long excl = static_cast<long long>(incl) - tot;
        if (excl < rem && rem <= static_cast<long long>(incl)) {  // exactly one lane
          long long cum = excl;
          int digit = 0;
          long long cnt = 0;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (cum + c[t] >= rem) {
              digit = 255 - 8 * lane - t;
              cnt = c[t];
              break;
            }
            cum += c[t];
          }
          s_prefix = prefix | (static_cast<uint64_t>(digit) << shift);
          s_remaining = rem - cum;
          s_done = (cnt == rem - cum);
        }
      }
      cluster.sync();  // the digit is known everywhere; no histogram is read any more
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
  // this CTA's rows of the mask
  const int my_rows = (nb - crank + kTopkCluster - 1) / kTopkCluster;
  for (size_t t = threadIdx.x; t < static_cast<size_t>(my_rows) * nb; t += blockDim.x) {
    const int i = crank + kTopkCluster * static_cast<int>(t / nb), j = static_cast<int>(t % nb);
    const size_t idx = static_cast<size_t>(i) * nb + j;
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

// pooled: the block means are already in the workspace (launch_quantize_pool_qk)
void launch_pool_and_scores(const void* Q, const void* K, const thrift_shape& s, const SelectWs& w, cudaStream_t st,
                            bool pooled = false) {
  const int nb = s.N / s.blk;
  if (!pooled) {
    pool_kernel<<<dim3(nb, s.B * s.Hq), kPoolThreads, 0, st>>>(static_cast<const __half*>(Q), s.N, s.D, s.blk, w.qm);
    pool_kernel<<<dim3(nb, s.B * s.Hkv), kPoolThreads, 0, st>>>(static_cast<const __half*>(K), s.N, s.D, s.blk, w.km);
  }
  const int tiles = (nb + kScoreTile - 1) / kScoreTile;
  score_kernel<<<dim3(tiles, tiles, s.B * s.Hq), 256, 0, st>>>(w.qm, w.km, s.Hq, s.Hkv, nb, s.D, s.causal,
                                                               s.sm_scale, w.scores);
}
}  // namespace

cudaError_t launch_pool_keys(const void* K, const thrift_shape& s, float* km, cudaStream_t st) {
  const int nb = s.N / s.blk;
  pool_kernel<<<dim3(nb, s.B * s.Hkv), kPoolThreads, 0, st>>>(static_cast<const __half*>(K), s.N, s.D, s.blk, km);
  return cudaGetLastError();
}

cudaError_t launch_select_vertical_window(const void* Q, const void* K, const thrift_shape& s, double rho, int window,
                                          uint8_t* mask, void* ws, cudaStream_t st) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  launch_pool_and_scores(Q, K, s, w, st);
  column_rank_kernel<<<s.B * s.Hq, 1024, 0, st>>>(w.scores, nb, s.causal, w.rank);
  const long long k = budget_pairs(s, rho);
  topk_kernel<1><<<s.B * s.Hq * kTopkCluster, 1024, 0, st>>>(w.scores, nb, s.causal, k, k, valid_pairs(s), mask, w.rank, window);
  return cudaGetLastError();
}

namespace {
// pooled: the block means are given (qm / km, or those already in the
// workspace when null) and no pooling pass runs
cudaError_t select_impl(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask, void* ws,
                        cudaStream_t st, bool pooled, const float* qm = nullptr, const float* km = nullptr) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  if (qm) w.qm = const_cast<float*>(qm);
  if (km) w.km = const_cast<float*>(km);
  launch_pool_and_scores(Q, K, s, w, st, pooled);
  const long long k = budget_pairs(s, rho);
  topk_kernel<0><<<s.B * s.Hq * kTopkCluster, 1024, 0, st>>>(w.scores, nb, s.causal, k, k, valid_pairs(s), mask, nullptr, 0);
  return cudaGetLastError();
}

cudaError_t select_tiered_impl(const void* Q, const void* K, const thrift_shape& s, double rho, double rho8,
                               double sigma, uint8_t* mask, void* ws, cudaStream_t st, bool pooled) {
  const int nb = s.N / s.blk;
  SelectWs w = carve(ws, s);
  launch_pool_and_scores(Q, K, s, w, st, pooled);
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
  topk_kernel<0><<<s.B * s.Hq * kTopkCluster, 1024, 0, st>>>(w.scores, nb, s.causal, k16, k16 + k8, n - ks, mask, nullptr, 0);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_select(const void* Q, const void* K, const thrift_shape& s, double rho, uint8_t* mask, void* ws,
                          cudaStream_t st) {
  return select_impl(Q, K, s, rho, mask, ws, st, false);
}

cudaError_t launch_select_pooled(const float* qm, const float* km, const thrift_shape& s, double rho, uint8_t* mask,
                                 void* ws, cudaStream_t st) {
  return select_impl(nullptr, nullptr, s, rho, mask, ws, st, true, qm, km);
}

void select_means(void* ws, const thrift_shape& s, float** qm, float** km) {
  const SelectWs w = carve(ws, s);
  *qm = w.qm;
  *km = w.km;
}

cudaError_t launch_select_tiered(const void* Q, const void* K, const thrift_shape& s, double rho, double rho8,
                                 double sigma, uint8_t* mask, void* ws, cudaStream_t st) {
  return select_tiered_impl(Q, K, s, rho, rho8, sigma, mask, ws, st, false);
}

cudaError_t launch_select_tiered_pooled(const thrift_shape& s, double rho, double rho8, double sigma, uint8_t* mask,
                                        void* ws, cudaStream_t st) {
  return select_tiered_impl(nullptr, nullptr, s, rho, rho8, sigma, mask, ws, st, true);
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
// Device address of the array per device.  Atomic, so that host threads whose
// first calls on a device overlap do not race (each stores the same value).
std::atomic<void*> g_select_scratch_ptr[kMaxScratchDevices];
}  // namespace

// Host code must not pass `g_select_scratch` itself to a kernel: on the host
// that name is only a stand-in for the device array.  Its device address is
// looked up once per device, with that device current, on the first call.
cudaError_t select_static_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  void* p = g_select_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_select_scratch_ptr[dev].store(p, std::memory_order_relaxed);
  }
  *ptr = p;
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

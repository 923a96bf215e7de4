// One decode step over the prefill's caches: a new query row per (batch,
// query head) attends to all N cached keys with the ThriftAttention method
// applied to that row (page "ThriftAttention: Selective Mixed Precision for
// Long-Context FP4 Attention", abstract and summary).  Re-using the
// block-scaled FP4 K/V of prefill as the decode cache follows TriAttention
// (abstract on the paper page of arXiv 2611.07256).
//
// Reading: the query row is its own query block.  Selection: score_j =
// fl32(sm_scale * fl32(q . kmean_j)) against the FP32 block means of K (the
// prefill heuristic's means), k = ceil(rho * nb - 1e-9) key blocks, the first
// and the last block first, then by score, ties to the lower block.  The
// selected blocks run in FP16 (fp16 q, K, V), the others in NVFP4 (q encoded
// along D like a row of Q, the prefill's K and V codes), under the prefill's
// online softmax: integer maxima, P pre-scaled by 2^11, l over the
// unquantised P.  Supported: D = 128, blk = 128, Hq / Hkv <= 16.
//
// Kernels:
//   decode_select     one CTA per (batch, query head): the nb scores, then the
//                     top k by rank of a unique 64-bit key.
//   decode_attention  persistent, one CTA per SM walking chunks of <= 8 key
//                     tiles of one (batch, kv head) with all its G query
//                     heads, keys on the 128 tensor-memory lanes:
//                       S^T = K q^T    (M = 128 keys, N = 8 or 16 heads: NVFP4
//                                       with the prefill's K codes, and fp16 for
//                                       the tiles a head of the group keeps in FP16)
//                       P per head and key, relative to the chunk's maximum
//                       O^T += V^T P^T (M = 128 channels; NVFP4 with the
//                                       prefill's V codes as A, fp16 V as an
//                                       MN-major A)
//                     Two passes per chunk: every S first, so each head has one
//                     maximum per chunk and O is never rescaled; then P and the
//                     P V products.  S, O, the query copies and the selection
//                     bits are double-buffered across chunks, and the loads
//                     stream through a 10-slot NVFP4 ring and a 3-slot fp16
//                     ring, so one chunk's products overlap the next one's
//                     loads.  Writes each chunk's unnormalised O, l and M.
//   decode_combine    per (batch, query head) and 32 channels: O = sum_c
//                     2^(M_c - M) O_c / sum_c 2^(M_c - M) l_c (exact
//                     power-of-two rescales), chunks spread over eight warps.
// The chunk's own maximum leaves every NVFP4 code of P as under the global
// one while the group scales stay E4M3 normals (the prefill's argument for
// its running maximum).
#include <cuda_fp16.h>

#include "attention_common.cuh"
#include "common.h"
#include "nvfp4.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace thrift {
namespace {
using namespace attn;

constexpr int kDD = 128;         // head dimension
constexpr int kDThreads = 192;   // warps 0-3 softmax, 4 producer, 5 MMA issuer
constexpr int kDSoftmax = 128;
constexpr int kDProducer = 4;
constexpr int kDMma = 5;
constexpr int kDRing4 = 10;      // NVFP4 slots: K4 + K scales, or V4 + V scales (9 KB)
constexpr int kDRing16 = 3;      // fp16 slots: one K or V tile (32 KB)
constexpr int kDMaxChunks = 64;  // chunks one CTA takes (the host plan keeps to it)
constexpr int kDPBuf = 4;        // P buffers: the softmax threads run up to 4 tiles ahead of P V
constexpr int kDMaxTiles = 8;    // key tiles of one chunk
constexpr uint32_t kDTmemCols = 512;

// Key tiles per chunk for N = NH query-head columns: two S regions of
// tiles x 2 NH columns (S4^T then S16^T per tile) fill columns 0-255.
__host__ __device__ constexpr int decode_chunk_tiles(int NH) { return NH == 8 ? 8 : 4; }

// Tensor-memory columns (S regions below 256).
constexpr uint32_t kCO = 256;    // O^T region r at 256 + 16 r
constexpr uint32_t kCSFK = 288;  // K scales (A of S^T), two 64-wide chunks of D
constexpr uint32_t kCSFQ = 296;  // q scales of query slot r at 296 + 8 r
constexpr uint32_t kCSFV = 312;  // V scales (A of O^T), two 64-key chunks
constexpr uint32_t kCSFP = 320;  // P scales (B of O^T)

struct DSmem {
  // Query copies, two slots (chunk parity): fp16 rows (two SW128 panels of
  // 16 rows x 128 B), NVFP4 rows (16 x 64 B, SW64), and their scale chunks.
  static constexpr uint32_t kQSlot = 6144;
  static constexpr uint32_t kQ16 = 0, kQ4 = 4096, kQSF = 5120;  // within a slot
  static constexpr uint32_t kP4 = 2 * kQSlot;                // P codes: kDPBuf buffers of 16 x 64 B, SW64
  static constexpr uint32_t kPSF = kP4 + kDPBuf * 1024;      // P scales: buffers of two 512-byte chunks
  static constexpr uint32_t kP16 = kPSF + kDPBuf * 1024;     // fp16 P: buffers of two SW128 panels of 2 KB
  static constexpr uint32_t kSlot4 = 9216;                   // 8 KB codes + 1 KB scales
  static constexpr uint32_t kRing4 = kP16 + kDPBuf * 4096;
  static constexpr uint32_t kRing16 = kRing4 + kDRing4 * kSlot4;
  static constexpr uint32_t kMisc = kRing16 + kDRing16 * 32768;
  static constexpr uint32_t kSel = kMisc + 1024;   // selection bits of the CTA's chunks
  static constexpr uint32_t kBytes = kSel + kDMaxChunks * kDMaxTiles * 4;
  static_assert(kQSlot % 1024 == 0 && kP16 % 1024 == 0 && kRing4 % 1024 == 0 && kRing16 % 1024 == 0,
                "swizzled tiles need 1 KB alignment");
  static_assert(kBytes + 1024 <= 232448, "shared memory above the 227 KB per-CTA limit");
};

struct DMisc {
  uint64_t bar_q[2];                  // query slot r staged (128 arrivals)
  uint64_t full4[kDRing4], empty4[kDRing4];
  uint64_t full16[kDRing16], empty16[kDRing16];
  uint64_t bar_s[2], s_free[2];       // S region r written / read by the softmax threads (128)
  uint64_t bar_o[2], o_free[2];       // O region r complete / read by the softmax threads (128)
  uint64_t bar_p[kDPBuf], bar_pv[kDPBuf];  // P buffer b written (128) / multiplied into O^T
  uint64_t bar_drain;
  uint32_t tmem;
  volatile int abort;
  float red[4][16];                   // per-warp maxima of S
  float lred[4][16];                  // per-warp sums of P
};
static_assert(sizeof(DMisc) <= 1024, "barriers must fit their shared-memory slice");

struct DParams {
  const __half* q;       // [B][Hq][D]
  const uint8_t* mask;   // [B][Hq][nb], 1 = FP16 block
  const uint8_t* ks;     // K scales, prefill layout
  const uint8_t* vs;     // V scales, prefill layout
  float* part_o;         // [B][Hq][cpu][D]
  float* part_l;         // [B][Hq][cpu]
  float* part_m;         // [B][Hq][cpu]
  uint32_t* err;
  int Hq, Hkv, NT, G;
  int chunk_tiles;       // key tiles per chunk (the last chunk of a unit may be shorter)
  int cpu;               // chunks per (batch, kv head)
  int W;                 // chunks in all
  float c2;              // fl32(sm_scale * log2 e)
};

struct Chunk {
  int unit, c, t0, nt;
  size_t head0;
};

__device__ __forceinline__ Chunk chunk_of(const DParams& p, int w) {
  Chunk ch;
  ch.unit = w / p.cpu;
  ch.c = w % p.cpu;
  ch.t0 = ch.c * p.chunk_tiles;
  ch.nt = min(p.chunk_tiles, p.NT - ch.t0);
  const int b = ch.unit / p.Hkv, hkv = ch.unit % p.Hkv;
  ch.head0 = static_cast<size_t>(b) * p.Hq + static_cast<size_t>(hkv) * p.G;
  return ch;
}

// Thread t's part of a chunk's query rows: 16-element group j = t % 8 of head
// row g = t / 8 (zero past G).
__device__ __forceinline__ void load_query(const DParams& p, size_t head0, int t, uint4& a, uint4& c) {
  const int g = t / 8, j = t % 8;
  a = make_uint4(0u, 0u, 0u, 0u);
  c = make_uint4(0u, 0u, 0u, 0u);
  if (g < p.G) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + (head0 + g) * kDD + 16 * j);
    a = src[0];
    c = src[1];
  }
}

// ... into query slot r: fp16 (SW128) and NVFP4 (SW64 codes; scale chunk
// byte g * 16 + j % 4).
__device__ __forceinline__ void stage_query(uint8_t* sm, int r, int t, const uint4& a, const uint4& c) {
  uint8_t* slot = sm + r * DSmem::kQSlot;
  const int g = t / 8, j = t % 8;
  uint8_t* q16 = slot + DSmem::kQ16 + (j / 4) * 2048;
  *reinterpret_cast<uint4*>(q16 + sw128_off(g, 2 * (j % 4))) = a;
  *reinterpret_cast<uint4*>(q16 + sw128_off(g, 2 * (j % 4) + 1)) = c;
  float v[16];
  const __half2* ha = reinterpret_cast<const __half2*>(&a);
  const __half2* hc = reinterpret_cast<const __half2*>(&c);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __half22float2(ha[i]), fc = __half22float2(hc[i]);
    v[2 * i] = fa.x;
    v[2 * i + 1] = fa.y;
    v[8 + 2 * i] = fc.x;
    v[8 + 2 * i + 1] = fc.y;
  }
  const Group16 e = encode16(v);
  *reinterpret_cast<uint2*>(slot + DSmem::kQ4 + sw64_off(g, j / 2) + 8 * (j % 2)) = make_uint2(e.lo, e.hi);
  slot[DSmem::kQSF + (j / 4) * 512 + g * 16 + (j % 4)] = static_cast<uint8_t>(e.scale);
  // rows 16-31 of both scale chunks are never read; keep them zero
  *reinterpret_cast<uint32_t*>(slot + DSmem::kQSF + (t / 64) * 512 + 256 + (t % 64) * 4) = 0u;
}

// S4^T and S16^T of tile i from S region address `sreg` (this warp's lanes).
template <int NH>
__device__ __forceinline__ void load_s(uint32_t sreg, int i, uint32_t (&s4)[NH], uint32_t (&s16)[NH]) {
  if constexpr (NH == 8) {
    uint32_t v[16];
    tmem_ld16(sreg + 16 * i, v);
    tmem_ld_wait();
    tmem_ld_fence(v);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      s4[g] = v[g];
      s16[g] = v[8 + g];
    }
  } else {
    tmem_ld16(sreg + 32 * i, s4);
    tmem_ld16(sreg + 32 * i + 16, s16);
    tmem_ld_wait();
    tmem_ld_fence(s4);
    tmem_ld_fence(s16);
  }
}

// Persistent: one CTA per SM takes chunks w = blockIdx.x, + gridDim.x, ...
// (at most kDMaxChunks).  NH = 8 or 16 query-head columns (G <= NH).  The
// MMA issuer runs one chunk ahead: S(0), then S(k + 1) before P V(k), so the
// softmax threads find the next chunk's S ready when they finish a chunk.
template <int NH>
__global__ void __launch_bounds__(kDThreads, 1)
    thrift_decode_kernel(const __grid_constant__ CUtensorMap mK16, const __grid_constant__ CUtensorMap mV16,
                         const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                         const DParams p) {
  constexpr int kTiles = decode_chunk_tiles(NH);
  constexpr uint32_t kSRegion = kTiles * 2 * NH;  // S region r at r * kSRegion
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DMisc& ms = *reinterpret_cast<DMisc*>(sm + DSmem::kMisc);
  uint32_t* selb = reinterpret_cast<uint32_t*>(sm + DSmem::kSel);  // [chunk][tile]: bit g = head g in FP16
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int G = p.G;
  const int x = static_cast<int>(blockIdx.x), X = static_cast<int>(gridDim.x);
  const int nk = x < p.W ? (p.W - x + X - 1) / X : 0;  // chunks of this CTA (<= kDMaxChunks)

  if (warp == kDMma) {
    tmem_alloc(&ms.tmem, kDTmemCols);
    tmem_relinquish();
  }
  if (tid == kDProducer * 32) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.bar_q[i], kDSoftmax);
      mbar_init(&ms.bar_s[i], 1);
      mbar_init(&ms.s_free[i], kDSoftmax);
      mbar_init(&ms.bar_o[i], 1);
      mbar_init(&ms.o_free[i], kDSoftmax);
    }
    for (int i = 0; i < kDPBuf; ++i) {
      mbar_init(&ms.bar_p[i], kDSoftmax);
      mbar_init(&ms.bar_pv[i], 1);
    }
    for (int i = 0; i < kDRing4; ++i) {
      mbar_init(&ms.full4[i], 1);
      mbar_init(&ms.empty4[i], 1);
    }
    for (int i = 0; i < kDRing16; ++i) {
      mbar_init(&ms.full16[i], 1);
      mbar_init(&ms.empty16[i], 1);
    }
    mbar_init(&ms.bar_drain, 1);
    ms.abort = 0;
    fence_mbar_init();
  }
  // Selection bits of every chunk of this CTA, all loads in flight at once.
  for (int e = tid; e < nk * kDMaxTiles; e += kDThreads) {
    const int k = e / kDMaxTiles, i = e % kDMaxTiles;
    const Chunk ch = chunk_of(p, x + k * X);
    uint32_t bits = 0u;
    if (i < ch.nt) {
      uint8_t m[16];
#pragma unroll
      for (int g = 0; g < 16; ++g) m[g] = g < G ? p.mask[(ch.head0 + g) * p.NT + ch.t0 + i] : 0;
#pragma unroll
      for (int g = 0; g < 16; ++g) bits |= (m[g] ? 1u : 0u) << g;
    }
    selb[e] = bits;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem;

  if (warp == kDProducer) {
    // ======================== producer ========================
    if (lane == 0) {
      prefetch_tensormap(&mK4);
      prefetch_tensormap(&mV4);
      int u4 = 0, u16 = 0;
      auto fill4 = [&](bool is_v, int bhk, int tile) -> bool {
        const int slot = u4 % kDRing4, use = u4 / kDRing4;
        if (use > 0 && !wait_or_abort(&ms.empty4[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        uint8_t* st = sm + DSmem::kRing4 + slot * DSmem::kSlot4;
        mbar_arrive_expect_tx(&ms.full4[slot], DSmem::kSlot4);
        if (!is_v) {
          tma_load_3d(st, &mK4, &ms.full4[slot], 0, tile * 128, bhk);
          bulk_load(st + 8192, p.ks + (static_cast<size_t>(bhk) * p.NT + tile) * 1024, 1024, &ms.full4[slot]);
        } else {
          tma_load_3d(st, &mV4, &ms.full4[slot], tile * 64, 0, bhk);
          bulk_load(st + 8192, p.vs + (static_cast<size_t>(bhk) * 2 * p.NT + 2 * tile) * 512, 1024,
                    &ms.full4[slot]);
        }
        ++u4;
        return true;
      };
      auto fill16 = [&](const CUtensorMap* map, int bhk, int tile) -> bool {
        const int slot = u16 % kDRing16, use = u16 / kDRing16;
        if (use > 0 && !wait_or_abort(&ms.empty16[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        uint8_t* st = sm + DSmem::kRing16 + slot * 32768;
        mbar_arrive_expect_tx(&ms.full16[slot], 32768);
        for (int pnl = 0; pnl < 2; ++pnl)
          tma_load_3d(st + pnl * 16384, map, &ms.full16[slot], pnl * 64, tile * 128, bhk);
        ++u16;
        return true;
      };
      // The order the MMA issuer consumes: K4 then K16 of chunk k (its S),
      // V4 (and V16) tile by tile (its P V), with S(k + 1) before P V(k).
      auto fills_s = [&](int k) -> bool {
        const Chunk ch = chunk_of(p, x + k * X);
        for (int i = 0; i < ch.nt; ++i)
          if (!fill4(false, ch.unit, ch.t0 + i)) return false;
        for (int i = 0; i < ch.nt; ++i)
          if (selb[k * kDMaxTiles + i] && !fill16(&mK16, ch.unit, ch.t0 + i)) return false;
        return true;
      };
      auto fills_pv = [&](int k) -> bool {
        const Chunk ch = chunk_of(p, x + k * X);
        for (int i = 0; i < ch.nt; ++i) {
          if (!fill4(true, ch.unit, ch.t0 + i)) return false;
          if (selb[k * kDMaxTiles + i] && !fill16(&mV16, ch.unit, ch.t0 + i)) return false;
        }
        return true;
      };
      bool ok = nk == 0 || fills_s(0);
      for (int k = 0; ok && k < nk; ++k) {
        if (k + 1 < nk) ok = fills_s(k + 1);
        if (ok) ok = fills_pv(k);
      }
      // Let every copy this thread issued land before the CTA can exit.
      for (int s = 0; s < kDRing4; ++s)
        if (u4 > s) mbar_wait(&ms.full4[s], ((u4 - 1 - s) / kDRing4) & 1, kWaitNs);
      for (int s = 0; s < kDRing16; ++s)
        if (u16 > s) mbar_wait(&ms.full16[s], ((u16 - 1 - s) / kDRing16) & 1, kWaitNs);
    }
    __syncwarp();
  } else if (warp == kDMma) {
    // ======================== MMA issuer ========================
    if (lane == 0) {
      constexpr uint32_t idS4 = idesc_nvf4(128, NH);
      constexpr uint32_t idS16 = idesc_f16(128, NH, false);
      constexpr uint32_t idO16 = idesc_f16_mn(128, NH, true, false);
      int u4 = 0, u16 = 0, gt = 0;
      // S(k): S4^T of every tile, then S16^T of the tiles with an FP16 head, into S region k % 2.
      auto issue_s = [&](int k) -> bool {
        const Chunk ch = chunk_of(p, x + k * X);
        const int r = k & 1;
        if (!wait_or_abort(&ms.bar_q[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER)) return false;
        // S region r was last read by the softmax threads for chunk k - 2.
        if (k >= 2 && !wait_or_abort(&ms.s_free[r], ((k - 2) >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        tc_fence_after();
        const uint32_t qs = sbase + r * DSmem::kQSlot;
        for (int c = 0; c < 2; ++c)
          tmem_cp_32x128b_x4(tm + kCSFQ + 8 * r + 4 * c, make_sdesc(qs + DSmem::kQSF + 512 * c, 16, 128, LAYOUT_NONE));
        const uint32_t sreg = tm + r * kSRegion;
#pragma unroll 1
        for (int i = 0; i < ch.nt; ++i) {
          const int slot = u4 % kDRing4;
          if (!wait_or_abort(&ms.full4[slot], (u4 / kDRing4) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD)) return false;
          ++u4;
          tc_fence_after();
          const uint32_t st = sbase + DSmem::kRing4 + slot * DSmem::kSlot4;
          for (int c = 0; c < 2; ++c)
            tmem_cp_32x128b_x4(tm + kCSFK + 4 * c, make_sdesc(st + 8192 + 512 * c, 16, 128, LAYOUT_NONE));
#pragma unroll
          for (int c = 0; c < 2; ++c)
            mma_nvf4(sreg + 2 * NH * i, make_sdesc(st + 32 * c, 16, 512, LAYOUT_SW64),
                     make_sdesc(qs + DSmem::kQ4 + 32 * c, 16, 512, LAYOUT_SW64), idS4, tm + kCSFK + 4 * c,
                     tm + kCSFQ + 8 * r + 4 * c, c > 0);
          mma_commit(&ms.empty4[slot]);
        }
#pragma unroll 1
        for (int i = 0; i < ch.nt; ++i) {
          if (!selb[k * kDMaxTiles + i]) continue;
          const int slot = u16 % kDRing16;
          if (!wait_or_abort(&ms.full16[slot], (u16 / kDRing16) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))
            return false;
          ++u16;
          tc_fence_after();
          const uint32_t k16 = sbase + DSmem::kRing16 + slot * 32768;
#pragma unroll
          for (int kk = 0; kk < kDD / 16; ++kk)
            mma_f16(sreg + 2 * NH * i + NH,
                    make_sdesc(k16 + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128),
                    make_sdesc(qs + DSmem::kQ16 + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128), idS16,
                    kk > 0);
          mma_commit(&ms.empty16[slot]);
        }
        mma_commit(&ms.bar_s[r]);
        return true;
      };
      // P V(k): O^T += V^T P^T tile by tile into O region k % 2.
      auto issue_pv = [&](int k) -> bool {
        const Chunk ch = chunk_of(p, x + k * X);
        const int r = k & 1;
        // O region r was last read by the softmax threads for chunk k - 2.
        if (k >= 2 && !wait_or_abort(&ms.o_free[r], ((k - 2) >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        tc_fence_after();
        const uint32_t oreg = tm + kCO + 16 * r;
#pragma unroll 1
        for (int i = 0; i < ch.nt; ++i, ++gt) {
          const int pb = gt % kDPBuf;
          const int slot = u4 % kDRing4;
          if (!wait_or_abort(&ms.full4[slot], (u4 / kDRing4) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD)) return false;
          ++u4;
          tc_fence_after();
          const uint32_t st = sbase + DSmem::kRing4 + slot * DSmem::kSlot4;
          // these copies follow the previous products in this thread's tcgen05
          // order, so they cannot overwrite scales those still read
          for (int c = 0; c < 2; ++c)
            tmem_cp_32x128b_x4(tm + kCSFV + 4 * c, make_sdesc(st + 8192 + 512 * c, 16, 128, LAYOUT_NONE));
          if (!wait_or_abort(&ms.bar_p[pb], (gt / kDPBuf) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER)) return false;
          tc_fence_after();
          const uint32_t p4 = sbase + DSmem::kP4 + pb * 1024, psf = sbase + DSmem::kPSF + pb * 1024;
          for (int c = 0; c < 2; ++c)
            tmem_cp_32x128b_x4(tm + kCSFP + 4 * c, make_sdesc(psf + 512 * c, 16, 128, LAYOUT_NONE));
#pragma unroll
          for (int c = 0; c < 2; ++c)
            mma_nvf4(oreg, make_sdesc(st + 32 * c, 16, 512, LAYOUT_SW64), make_sdesc(p4 + 32 * c, 16, 512, LAYOUT_SW64),
                     idS4, tm + kCSFV + 4 * c, tm + kCSFP + 4 * c, (i > 0 || c > 0) ? 1u : 0u);
          if (selb[k * kDMaxTiles + i]) {
            const int s16 = u16 % kDRing16;
            if (!wait_or_abort(&ms.full16[s16], (u16 / kDRing16) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))
              return false;
            ++u16;
            tc_fence_after();
            const uint32_t v16 = sbase + DSmem::kRing16 + s16 * 32768, p16 = sbase + DSmem::kP16 + pb * 4096;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16(oreg, make_sdesc(v16 + kk * 2048, 16384, 1024, LAYOUT_SW128),
                      make_sdesc(p16 + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128), idO16, 1u);
            mma_commit(&ms.empty16[s16]);
          }
          mma_commit(&ms.empty4[slot]);
          mma_commit(&ms.bar_pv[pb]);
        }
        mma_commit(&ms.bar_o[r]);
        return true;
      };
      bool ok = nk == 0 || issue_s(0);
      for (int k = 0; ok && k < nk; ++k) {
        if (k + 1 < nk) ok = issue_s(k + 1);
        if (ok) ok = issue_pv(k);
      }
      // drain: every tensor-core operation this thread issued completes before exit
      mma_commit(&ms.bar_drain);
      mbar_wait(&ms.bar_drain, 0, kWaitNs);
    }
    __syncwarp();
  } else {
    // ======= softmax threads: lane = key of a tile, then channel of O^T =======
    const int t = tid;
    const float c2 = p.c2;
    const uint32_t lane_base = tm + (static_cast<uint32_t>(warp * 32) << 16);
    bool failed = false;
    int gt = 0;
    uint4 qa, qc;
    if (nk > 0) {
      load_query(p, chunk_of(p, x).head0, t, qa, qc);
      stage_query(sm, 0, t, qa, qc);
      fence_proxy_async_smem();
      mbar_arrive(&ms.bar_q[0]);
    }
    for (int k = 0; k < nk; ++k) {
      const Chunk ch = chunk_of(p, x + k * X);
      const int r = k & 1;
      const uint32_t* sel = selb + k * kDMaxTiles;
      // the next chunk's query rows, in flight while this chunk's S is read
      if (k + 1 < nk) load_query(p, chunk_of(p, x + (k + 1) * X).head0, t, qa, qc);
      // ---- pass 1: maximum of S per head over the chunk ----
      float mx[NH];
#pragma unroll
      for (int g = 0; g < NH; ++g) mx[g] = -INFINITY;
      if (!failed) failed = !wait_or_abort(&ms.bar_s[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
      const uint32_t sreg = lane_base + r * kSRegion;
      if (!failed) {
        tc_fence_after();
        for (int i = 0; i < ch.nt; ++i) {
          uint32_t s4[NH], s16[NH];
          load_s<NH>(sreg, i, s4, s16);
          const uint32_t si = sel[i];
#pragma unroll
          for (int g = 0; g < NH; ++g) mx[g] = fmaxf(mx[g], __uint_as_float(((si >> g) & 1u) ? s16[g] : s4[g]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < NH; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
      if (lane == 0)
#pragma unroll
        for (int g = 0; g < NH; ++g) ms.red[warp][g] = mx[g];
      failed = softmax_bar_or<kDSoftmax>(failed);
      // base_g = 11 - M_g, M_g = ceil(max t) = ceil(fl32(max S * c2)); thread g keeps its M for the epilogue
      float base[NH];
      float my_m = 0.f;
#pragma unroll
      for (int g = 0; g < NH; ++g) {
        const float M = ceilf(fmaxf(fmaxf(ms.red[0][g], ms.red[1][g]), fmaxf(ms.red[2][g], ms.red[3][g])) * c2);
        base[g] = static_cast<float>(kPLog2) - M;
        if (t == g) my_m = M;
      }
      // The next chunk's query slot was last read by the S products of chunk
      // k - 1, which completed before this thread saw bar_s of chunk k - 1.
      if (!failed && k + 1 < nk) {
        stage_query(sm, r ^ 1, t, qa, qc);
        fence_proxy_async_smem();
        mbar_arrive(&ms.bar_q[r ^ 1]);
      }
      // ---- pass 2: P per head and key, encoded into buffer gt % kDPBuf ----
      float lsum[NH];
#pragma unroll
      for (int g = 0; g < NH; ++g) lsum[g] = 0.f;
      for (int i = 0; i < ch.nt && !failed; ++i, ++gt) {
        const int pb = gt % kDPBuf;
        if (gt >= kDPBuf)
          failed = !wait_or_abort(&ms.bar_pv[pb], ((gt - kDPBuf) / kDPBuf) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
        failed = __any_sync(0xffffffffu, failed);
        if (failed) break;
        tc_fence_after();
        const uint32_t si = sel[i];
        uint32_t s4[NH], s16[NH];
        load_s<NH>(sreg, i, s4, s16);
        // Every head at once (independent chains): S in the head's precision,
        // the group maximum over 16 consecutive keys (lanes), the group scale,
        // P * 2^11 (divided by the scale for an NVFP4 head) and its code.
        float sv[NH], gm[NH];
#pragma unroll
        for (int g = 0; g < NH; ++g) {
          sv[g] = __uint_as_float(((si >> g) & 1u) ? s16[g] : s4[g]);
          gm[g] = sv[g];
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1)
#pragma unroll
          for (int g = 0; g < NH; ++g) gm[g] = fmaxf(gm[g], __shfl_xor_sync(0xffffffffu, gm[g], o));
        uint32_t wd[NH], sbyte[NH];
        float x16[NH];
        // Padding heads (g >= G) have zero query rows: their values are finite
        // and only reach O^T columns nobody reads, so every head is computed
        // (straight-line code, so the heads' latency chains overlap).
#pragma unroll
        for (int g = 0; g < NH; ++g) {
          const bool h16 = (si >> g) & 1u;
          const float amax = ex2(fmaf(gm[g], c2, base[g]));  // max of P * 2^11 in the group
          const uint32_t sb = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.f) & 0xFFu;
          const float sc0 = e4m3_to_f32(sb);
          const float sc = (h16 || sc0 <= 0.f) ? 1.0f : sc0;  // zero scale: the code rounds to 0, l keeps P
          const float xv = ex2(fmaf(sv[g], c2, base[g] - lg2(sc)));  // P * 2^11 / scale
          lsum[g] = fmaf(xv, sc, lsum[g]);
          x16[g] = h16 ? xv : 0.f;
          sbyte[g] = h16 ? 0u : sb;
          wd[g] = h16 ? 0u : ((cvt_e2m1x2(xv, 0.f) & 0xFu) << (4 * (lane & 7)));
        }
        // codes of keys 8m .. 8m + 7 in one word (key t at byte t / 2 of row g)
#pragma unroll
        for (int o = 1; o < 8; o <<= 1)
#pragma unroll
          for (int g = 0; g < NH; ++g) wd[g] |= __shfl_xor_sync(0xffffffffu, wd[g], o);
        uint8_t* p4 = sm + DSmem::kP4 + pb * 1024;
        uint8_t* psf = sm + DSmem::kPSF + pb * 1024;
        uint8_t* p16 = sm + DSmem::kP16 + pb * 4096;
#pragma unroll
        for (int g = 0; g < NH; ++g) {
          if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(p4 + sw64_off(g, warp) + (lane >> 1)) = wd[g];
          if ((lane & 15) == 0) psf[(t / 64) * 512 + g * 16 + (t % 64) / 16] = static_cast<uint8_t>(sbyte[g]);
          if (si)
            *reinterpret_cast<__half*>(p16 + (t / 64) * 2048 + sw128_off(g, (t % 64) / 8) + (t % 8) * 2) =
                __float2half_rn(x16[g]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&ms.bar_p[pb]);
      }
      tc_fence_before();
      mbar_arrive(&ms.s_free[r]);
      // ---- epilogue: the chunk's O^T column g, l_g and M_g ----
      if (!failed) failed = !wait_or_abort(&ms.bar_o[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < NH; ++g) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], o);
      if (lane == 0)
#pragma unroll
        for (int g = 0; g < NH; ++g) ms.lred[warp][g] = lsum[g];
      failed = softmax_bar_or<kDSoftmax>(failed);
      if (failed) break;
      tc_fence_after();
      uint32_t o[16];
      tmem_ld16(lane_base + kCO + 16 * r, o);
      tmem_ld_wait();
      tmem_ld_fence(o);
#pragma unroll
      for (int g = 0; g < NH; ++g)
        if (g < G) p.part_o[((ch.head0 + g) * p.cpu + ch.c) * kDD + t] = __uint_as_float(o[g]);
      if (t < G) {
        const size_t idx = (ch.head0 + t) * p.cpu + ch.c;
        p.part_l[idx] = (ms.lred[0][t] + ms.lred[1][t]) + (ms.lred[2][t] + ms.lred[3][t]);
        p.part_m[idx] = my_m;
      }
      tc_fence_before();
      mbar_arrive(&ms.o_free[r]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDMma) {
    tc_fence_after();
    tmem_dealloc(tm, kDTmemCols);
  }
}

// O = sum_c 2^(M_c - M) O_c / sum_c 2^(M_c - M) l_c; both carry the 2^11
// pre-scale.  Grid (B * Hq, D / 32), 256 threads: the CTA takes 32 channels of
// one head; warp w sums chunks c = w, w + 8, ... (lanes over channels, so the
// loads are coalesced and independent), then the eight partial sums are added
// in a fixed order.  chunks <= 1024.
__global__ void __launch_bounds__(256) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_l,
                                                             const float* __restrict__ part_m, int chunks,
                                                             __half* __restrict__ O) {
  __shared__ float wsm[1024];
  __shared__ float red[8][33];
  __shared__ float s_m, s_l;
  const size_t bh = blockIdx.x;
  const int d0 = blockIdx.y * 32;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const float* pm = part_m + bh * chunks;
  const float* pl = part_l + bh * chunks;
  const float* po = part_o + bh * chunks * kDD;
  float m = -INFINITY;
  for (int c = tid; c < chunks; c += 256) m = fmaxf(m, pm[c]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp][0] = m;
  __syncthreads();
  if (tid == 0) {
    float mm = red[0][0];
    for (int w = 1; w < 8; ++w) mm = fmaxf(mm, red[w][0]);
    s_m = mm;
  }
  __syncthreads();
  const float M = s_m;
  float l = 0.f;
  for (int c = tid; c < chunks; c += 256) {
    const float w = exp2_int(pm[c] - M);
    wsm[c] = w;
    l = fmaf(w, pl[c], l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncthreads();  // red[][0] was read above; wsm complete
  if (lane == 0) red[warp][32] = l;
  __syncthreads();
  if (tid == 0) {
    float ll = 0.f;
    for (int w = 0; w < 8; ++w) ll += red[w][32];
    s_l = ll;
  }
  float acc = 0.f;
#pragma unroll 4
  for (int c = warp; c < chunks; c += 8) acc = fmaf(wsm[c], po[static_cast<size_t>(c) * kDD + d0 + lane], acc);
  red[warp][lane] = acc;
  __syncthreads();
  if (tid < 32) {
    float sum = 0.f;
    for (int w = 0; w < 8; ++w) sum += red[w][tid];
    O[bh * kDD + d0 + tid] = __float2half_rn(sum / s_l);
  }
}

// Unique key of key block j: forced bit (first and last block), order-
// preserving score bits, inverted index.
__device__ __forceinline__ uint64_t decode_key(float score, int j, int nb) {
  if (score == 0.0f) score = 0.0f;
  uint32_t u = __float_as_uint(score);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  const uint64_t forced = (j == 0 || j == nb - 1) ? 1ull : 0ull;
  return (forced << 63) | (static_cast<uint64_t>(u) << 31) | (0x7FFFFFFFull - static_cast<uint64_t>(j));
}

// One CTA per (batch, query head); nb <= 1024, D = 128.  score_j =
// fl32(sm_scale * fl32(q . kmean_j)): the products of the fp16 query and the
// FP32 means are exact in FP64; the FP64 sum (a warp tree, one warp per key
// block, lanes over channels) is rounded once.  Then the top k by rank of a
// unique key.
__global__ void __launch_bounds__(1024) decode_select_kernel(const __half* __restrict__ q,
                                                             const float* __restrict__ km, int Hq, int Hkv, int nb,
                                                             float sm_scale, long long k, uint8_t* __restrict__ mask) {
  constexpr int kRows = 4;  // key blocks per warp and step, all loads in flight at once
  __shared__ unsigned long long keys[1024];
  const size_t bh = blockIdx.x;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  const int G = Hq / Hkv;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nwarps = blockDim.x / 32;
  const float* kmh = km + (static_cast<size_t>(b) * Hkv + h / G) * nb * static_cast<size_t>(kDD);
  double qd[kDD / 32];
#pragma unroll
  for (int i = 0; i < kDD / 32; ++i) qd[i] = static_cast<double>(__half2float(q[bh * kDD + lane + 32 * i]));
  for (int j0 = warp * kRows; j0 < nb; j0 += nwarps * kRows) {
    float v[kRows][kDD / 32];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int i = 0; i < kDD / 32; ++i)
        v[r][i] = j0 + r < nb ? kmh[static_cast<size_t>(j0 + r) * kDD + lane + 32 * i] : 0.f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      double dot = 0.0;
#pragma unroll
      for (int i = 0; i < kDD / 32; ++i) dot = fma(qd[i], static_cast<double>(v[r][i]), dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0 && j0 + r < nb) {
        const float sc =
            static_cast<float>(static_cast<double>(sm_scale) * static_cast<double>(static_cast<float>(dot)));
        keys[j0 + r] = decode_key(sc, j0 + r, nb);
      }
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const unsigned long long kj = keys[j];
    int rank = 0;
    for (int jj = 0; jj < nb; ++jj) rank += keys[jj] > kj ? 1 : 0;
    mask[bh * nb + j] = rank < k ? 1 : 0;
  }
}

}  // namespace

namespace {
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess || n <= 0)
    return 148;
  return n;
}
}  // namespace

// Chunk size for one wave of persistent CTAs: the size (at most the TMEM
// budget's) that minimises the most key tiles any CTA takes, counting half a
// tile of per-chunk overhead; ties to the larger chunk.  A CTA takes at most
// kDMaxChunks chunks (more CTAs than SMs beyond that).
DecodePlan decode_plan(const thrift_shape& s) {
  const int NT = num_tiles(s.N);
  const int units = s.B * s.Hkv;
  const int NH = (s.Hq / s.Hkv) <= 8 ? 8 : 16;
  const int cmax = decode_chunk_tiles(NH);
  const int nsm = sm_count();
  DecodePlan best{1, NT, 1};
  double best_cost = 1e300;
  for (int C = 1; C <= cmax && C <= NT; ++C) {
    const int cpu = (NT + C - 1) / C;
    const long long W = static_cast<long long>(units) * cpu;
    long long grid = W < nsm ? W : nsm;
    if (grid * kDMaxChunks < W) grid = (W + kDMaxChunks - 1) / kDMaxChunks;  // selection bits of <= 64 chunks
    const double cost = static_cast<double>((W + grid - 1) / grid) * (C + 0.5);
    if (cost <= best_cost) {
      best_cost = cost;
      best.tiles_per_cta = C;
      best.chunks = cpu;
      best.grid = static_cast<int>(grid);
    }
  }
  return best;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Sized for one-tile chunks (the most partial results any plan writes).
size_t decode_workspace_bytes(const thrift_shape& s) {
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * num_tiles(s.N);
  return align256(static_cast<size_t>(s.B) * s.Hq * num_tiles(s.N)) + align256(rows * kDD * sizeof(float)) +
         2 * align256(rows * sizeof(float));
}

DecodeWs decode_carve(void* ws, const thrift_shape& s) {
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * num_tiles(s.N);
  uint8_t* p = static_cast<uint8_t*>(ws);
  DecodeWs w;
  w.mask = p;
  p += align256(static_cast<size_t>(s.B) * s.Hq * num_tiles(s.N));
  w.part_o = reinterpret_cast<float*>(p);
  p += align256(rows * kDD * sizeof(float));
  w.part_l = reinterpret_cast<float*>(p);
  p += align256(rows * sizeof(float));
  w.part_m = reinterpret_cast<float*>(p);
  return w;
}

cudaError_t launch_decode_select(const void* q, const float* km, const thrift_shape& s, double rho, uint8_t* mask,
                                 cudaStream_t st) {
  const int nb = s.N / s.blk;
  double kk = ceil(rho * static_cast<double>(nb) - 1e-9);
  if (kk < 0) kk = 0;
  if (kk > nb) kk = nb;
  decode_select_kernel<<<s.B * s.Hq, 1024, 0, st>>>(static_cast<const __half*>(q), km, s.Hq, s.Hkv, nb, s.sm_scale,
                                                   static_cast<long long>(kk), mask);
  return cudaGetLastError();
}

cudaError_t launch_decode_attention(const void* q, const void* K, const void* V, const void* k4, const void* ks,
                                    const void* v4, const void* vs, const uint8_t* mask, const thrift_shape& s,
                                    void* O, const DecodeWs& w, uint32_t* err, cudaStream_t st) {
  CUtensorMap mK16, mV16, mK4, mV4;
  const uint64_t BHk = static_cast<uint64_t>(s.B) * s.Hkv;
  bool ok = true;
  ok &= make_tmap_3d(&mK16, K, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kDD, s.N, BHk, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&mV16, V, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kDD, s.N, BHk, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&mK4, k4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kDD / 2, s.N, BHk, kDD / 2, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= make_tmap_3d(&mV4, v4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.N / 2, kDD, BHk, 64, kDD, CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) return cudaErrorInvalidValue;
  const DecodePlan pl = decode_plan(s);
  const int G = s.Hq / s.Hkv;
  DParams prm;
  prm.q = static_cast<const __half*>(q);
  prm.mask = mask;
  prm.ks = static_cast<const uint8_t*>(ks);
  prm.vs = static_cast<const uint8_t*>(vs);
  prm.part_o = w.part_o;
  prm.part_l = w.part_l;
  prm.part_m = w.part_m;
  prm.err = err;
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.NT = num_tiles(s.N);
  prm.G = G;
  prm.chunk_tiles = pl.tiles_per_cta;
  prm.cpu = pl.chunks;
  prm.W = static_cast<int>(BHk) * pl.chunks;
  prm.c2 = static_cast<float>(static_cast<double>(s.sm_scale) * 1.4426950408889634073599246810019);
  const size_t smem = DSmem::kBytes + 1024;
  cudaError_t e;
  if (G <= 8) {
    e = cudaFuncSetAttribute(thrift_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    thrift_decode_kernel<8><<<pl.grid, kDThreads, smem, st>>>(mK16, mV16, mK4, mV4, prm);
  } else {
    e = cudaFuncSetAttribute(thrift_decode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    thrift_decode_kernel<16><<<pl.grid, kDThreads, smem, st>>>(mK16, mV16, mK4, mV4, prm);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(s.B * s.Hq, kDD / 32), 256, 0, st>>>(w.part_o, w.part_l, w.part_m, pl.chunks,
                                                                     static_cast<__half*>(O));
  return cudaGetLastError();
}

}  // namespace thrift

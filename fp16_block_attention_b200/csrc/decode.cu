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
//   decode_select     one CTA per (batch, query head): the nb scores (one warp
//                     per key block, coalesced), then the top k of unique
//                     64-bit keys by a bitonic sort.
//   decode_compact    one CTA per (batch, kv head) "unit": per key tile the
//                     bits of the group's query heads that keep it in FP16,
//                     and the list of the tiles some head keeps, in order.
//   thrift_decode_kernel  both passes in one persistent launch (the FP16
//                     pass on the first SMs' worth of CTAs, the NVFP4 pass on
//                     the rest, starting on the SMs the first leave), each CTA
//                     walking chunks of one unit's key tiles with all its G
//                     query heads, keys on the 128 tensor-memory lanes:
//                       NVFP4 pass: chunks of <= 16 consecutive tiles;
//                         S^T = K q^T from the prefill's K codes, then
//                         O^T += V^T P^T from its V codes, every head whose
//                         selection keeps the tile in FP16 masked out;
//                       FP16 pass: chunks of <= 4 tiles of the unit's list;
//                         the same products in fp16 (V as an MN-major A), the
//                         heads that do not keep the tile masked out.
//                     Every key of every head is computed in exactly one pass.
//                     Within a chunk two sweeps: every S first (one integer
//                     maximum per head and chunk, so O is never rescaled),
//                     then P and the P V products.  S, O and the query copies
//                     are double-buffered across chunks; K and V stream
//                     through a ring each (NVFP4: 12 and 11 slots of 9 KB;
//                     FP16: 3 and 3 slots of 32 KB), so one chunk's products
//                     overlap the next one's loads.  Each chunk writes its
//                     unnormalised O, l and M per head.
//   decode_combine    per (batch, query head): O = sum_c 2^(M_c - M) O_c /
//                     sum_c 2^(M_c - M) l_c over both passes' chunks, in one
//                     online sweep (exact power-of-two rescales).
// The kernels of a step are chained by programmatic dependent launch.
// The chunk's own maximum leaves every NVFP4 code of P as under the global
// one while the group scales stay E4M3 normals (the prefill's argument for
// its running maximum).
#include <cuda_fp16.h>

#include <atomic>
#include <utility>

#include "attention_common.cuh"
#include "common.h"
#include "nvfp4.cuh"
#include "ptx.cuh"
#include "tmap.h"

namespace thrift {
namespace {
using namespace attn;

constexpr int kDD = 128;         // head dimension
// Warp roles: 4 softmax warps per softmax warpgroup (one or two), then the K
// producer, the S issuer (which also owns the tensor memory), the V producer,
// the P V issuer and, with at most 8 heads, a V scale copier.  The two-group
// form (4 heads) alternates pairs of key tiles between the groups.  Registers
// are granted to an SM's warps four at a time, so the register budget is
// that of the thread count rounded up to 128: 16 heads need about 220
// registers a thread and run without a copier (256 threads, its P V issuer
// copies the V scales itself); 8 heads about 150 (288 threads, bounded as
// 384); 4 heads about 110 (416 threads with two groups, bounded as 512).
template <int NG>
struct DCfg {
  static constexpr int kGroups = NG == 4 ? 2 : 1;
  static constexpr bool kCopier = NG < 16;
  static constexpr int kSoftWarps = 4 * kGroups;
  static constexpr int kSoft = 32 * kSoftWarps;  // softmax threads
  static constexpr int kProdK = kSoftWarps, kIssueS = kSoftWarps + 1, kProdV = kSoftWarps + 2,
                       kIssuePV = kSoftWarps + 3, kCopyV = kSoftWarps + 4;
  static constexpr int kThreads = 32 * (kSoftWarps + 4 + (kCopier ? 1 : 0));
  static constexpr int kBound = (kThreads + 127) / 128 * 128;
};
constexpr int kDGroup = 128;     // threads of one softmax warpgroup
constexpr int kDMaxChunks = 64;  // chunks one CTA takes (the host plan keeps to it)
constexpr int kDPBuf = 4;        // P buffers: the softmax threads run up to 4 tiles ahead of P V
constexpr int kDMaxTiles = 16;   // key tiles of one chunk
constexpr int kDTiles16 = 4;     // key tiles of one chunk of the FP16 pass
constexpr int kDMaxSlots = 12;   // slots of one ring
constexpr uint32_t kDTmemCols = 512;
constexpr uint32_t kBarPsf = 3;  // named barriers 3, 4: a softmax group's warps have written a tile's P scales

enum DecodePass : int { kPassFp4 = 0, kPassFp16 = 1 };

// Key tiles per NVFP4 chunk for NH query-head columns: two S regions of
// tiles x NH columns fill columns 0-255.
__host__ __device__ constexpr int decode_chunk_tiles(int NH) { return 256 / (2 * NH); }

// Tensor-memory columns (S regions below 256).
constexpr uint32_t kCO = 256;    // O^T region r at 256 + 16 r
constexpr uint32_t kCSFK = 288;  // K scales (A of S^T), two 64-wide chunks of D
constexpr uint32_t kCSFQ = 296;  // q scales of query slot r at 296 + 8 r
constexpr uint32_t kCSFP = 320;  // P scales of P buffer b (B of O^T) at 320 + 8 b
constexpr uint32_t kCSFV = 352;  // V scales of V ring slot s (A of O^T, two 64-key chunks) at 352 + 8 s

// Shared memory of one pass.  Query slots (chunk parity): NVFP4 rows (16 x 64
// B, SW64) and their two scale chunks, or fp16 rows (two SW128 panels of 16
// rows x 128 B).  P buffers: NVFP4 codes (16 x 64 B, SW64) and two 512-byte
// scale chunks, or fp16 P (two SW128 panels).  Ring slots: an NVFP4 K or V tile
// with its scales (8 KB + 1 KB), or an fp16 K or V tile (two 16 KB panels); K
// and V have a ring each.
template <int PASS>
struct DLayout {
  static constexpr uint32_t kQSlot = PASS == kPassFp4 ? 2048 : 4096;
  static constexpr uint32_t kPBuf = PASS == kPassFp4 ? 2048 : 4096;
  static constexpr uint32_t kSlot = PASS == kPassFp4 ? 9216 : 32768;
  static constexpr int kSlotsK = PASS == kPassFp4 ? 12 : 3;
  static constexpr int kSlotsV = PASS == kPassFp4 ? 11 : 3;
  static constexpr uint32_t kP = 2 * kQSlot;
  static constexpr uint32_t kRingK = kP + kDPBuf * kPBuf;
  static constexpr uint32_t kRingV = kRingK + kSlotsK * kSlot;
  static constexpr uint32_t kMisc = kRingV + kSlotsV * kSlot;
  static constexpr uint32_t kInfo = kMisc + 2048;               // chunk table (CInfo)
  static constexpr uint32_t kEntry = kInfo + kDMaxChunks * 16;  // [chunk][i]: tile | FP16 head bits << 16
  static constexpr uint32_t kBytes = kEntry + kDMaxChunks * kDMaxTiles * 4;
  static_assert(kSlotsK <= kDMaxSlots && kSlotsV <= kDMaxSlots, "ring barriers");
  static_assert(kP % 1024 == 0 && kPBuf % 1024 == 0 && kRingK % 1024 == 0 && kSlot % 1024 == 0,
                "swizzled tiles need 1 KB alignment");
  static_assert(kBytes + 1024 <= 232448, "shared memory above the 227 KB per-CTA limit");
};

struct DMisc {
  uint64_t bar_q[2];                  // query slot r staged (128 arrivals)
  uint64_t full_k[kDMaxSlots], empty_k[kDMaxSlots];
  uint64_t full_v[kDMaxSlots], empty_v[kDMaxSlots];
  uint64_t bar_s[2], s_free[2];       // S region r written / read by the softmax threads (128)
  uint64_t bar_o[2], o_free[2];       // O region r complete / read by the softmax threads (128)
  uint64_t bar_p[kDPBuf], bar_pv[kDPBuf];  // P buffer b written (128) / multiplied into O^T
  uint64_t vsf_ready[kDMaxSlots];     // NVFP4 pass: V scales of ring slot s in tensor memory
  uint64_t drain_s, drain_pv, drain_cp;
  uint32_t tmem;
  volatile int abort;
  int nk;                             // chunks of this CTA
  float red[8][16];                   // per-warp maxima of S
  float lred[8][16];                  // per-warp sums of P
};
static_assert(sizeof(DMisc) <= 2048, "barriers must fit their shared-memory slice");

struct CInfo {
  int unit;   // b * Hkv + kv head
  int slot;   // partial-result slot of the chunk
  int nt;     // key tiles
  int first;  // NVFP4: first tile; FP16: first entry of the unit's list
};

struct DParams {
  const __half* q;         // [B][Hq][D]
  const uint16_t* hbits;   // [B * Hkv][NT]: bit g = query head g of the group keeps the tile in FP16
  const uint32_t* list16;  // [B * Hkv][NT]: the tiles some head keeps, tile | bits << 16, ascending
  const int* n16;          // [B * Hkv]: entries of each list
  const uint8_t* ks;       // K scales, prefill layout
  const uint8_t* vs;       // V scales, prefill layout
  float* part_o;           // [B][Hq][cap][D]
  float* part_l;           // [B][Hq][cap]
  float* part_m;           // [B][Hq][cap]
  uint32_t* err;
  uint64_t wait_ns;        // bound of every wait in the kernel (thrift_set_wait_limit)
  int withhold;            // failure-detection test only: the K tile (counted per CTA and pass) whose
                           // copies the K producer does not issue, so its consumers' waits run out; or -1
  int Hq, Hkv, NT, G;
  int units;               // B * Hkv
  int C;                   // key tiles per NVFP4 chunk (a unit's last chunk may be shorter)
  int cpu;                 // NVFP4 chunks per unit (partial slots 0 .. cpu - 1)
  int cap;                 // partial slots per head: NT NVFP4 slots, then ceil(NT / kDTiles16) FP16 slots
  int grid16;              // CTAs of the FP16 pass (the first of the grid; the rest run the NVFP4 pass)
  float c2;                // fl32(sm_scale * log2 e)
};

__device__ __forceinline__ size_t head0_of(const DParams& p, int unit) {
  return static_cast<size_t>(unit / p.Hkv) * p.Hq + static_cast<size_t>(unit % p.Hkv) * p.G;
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

// ... into query slot r: fp16 rows (SW128) for the FP16 pass; NVFP4 rows
// (SW64 codes at 0, scale chunk byte g * 16 + j % 4 at 1024) for the other.
template <int PASS>
__device__ __forceinline__ void stage_query(uint8_t* sm, int r, int t, const uint4& a, const uint4& c) {
  uint8_t* slot = sm + r * DLayout<PASS>::kQSlot;
  const int g = t / 8, j = t % 8;
  if constexpr (PASS == kPassFp16) {
    uint8_t* q16 = slot + (j / 4) * 2048;
    *reinterpret_cast<uint4*>(q16 + sw128_off(g, 2 * (j % 4))) = a;
    *reinterpret_cast<uint4*>(q16 + sw128_off(g, 2 * (j % 4) + 1)) = c;
  } else {
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
    *reinterpret_cast<uint2*>(slot + sw64_off(g, j / 2) + 8 * (j % 2)) = make_uint2(e.lo, e.hi);
    slot[1024 + (j / 4) * 512 + g * 16 + (j % 4)] = static_cast<uint8_t>(e.scale);
    // rows 16-31 of both scale chunks are never read; keep them zero
    *reinterpret_cast<uint32_t*>(slot + 1024 + (t / 64) * 512 + 256 + (t % 64) * 4) = 0u;
  }
}

// The NH columns at `addr` (this warp's lanes).
template <int NH>
__device__ __forceinline__ void load_cols(uint32_t addr, uint32_t (&s)[NH]) {
  if constexpr (NH == 8)
    tmem_ld8(addr, s);
  else
    tmem_ld16(addr, s);
  tmem_ld_wait();
  tmem_ld_fence(s);
}

// Tiles i and i + 1: 2 NH columns at `addr`.
template <int NH>
__device__ __forceinline__ void load_pair(uint32_t addr, uint32_t (&s)[2 * NH]) {
  if constexpr (NH == 8) {
    tmem_ld16(addr, s);
    tmem_ld_wait();
    tmem_ld_fence(s);
  } else {
    uint32_t (&a)[16] = *reinterpret_cast<uint32_t(*)[16]>(&s[0]);
    uint32_t (&b)[16] = *reinterpret_cast<uint32_t(*)[16]>(&s[16]);
    tmem_ld16(addr, a);
    tmem_ld16(addr + 16, b);
    tmem_ld_wait();
    tmem_ld_fence(a);
    tmem_ld_fence(b);
  }
}

// One CTA of a pass, persistent: CTA x of X takes the chunks w = x, x + X, ...
// (at most kDMaxChunks; in the FP16 pass the empty ones are dropped).  NG =
// 4, 8 or 16 query heads the softmax threads compute (G <= NG), NH = max(NG,
// 8) head columns of the products.  Two producers (K tiles, V tiles) and two
// tensor-core issuers (S^T = K q^T, O^T += V^T P^T), so the S products of the
// next chunk run while the softmax threads finish this one and the P V
// products follow them tile by tile.
template <int PASS, int NG>
__device__ __forceinline__ void decode_pass(const CUtensorMap* mK, const CUtensorMap* mV, const DParams& p,
                                            uint8_t* sm, int x, int X) {
  using L = DLayout<PASS>;
  using Cfg = DCfg<NG>;
  constexpr int NH = NG < 8 ? 8 : NG;
  constexpr int kTiles = PASS == kPassFp4 ? decode_chunk_tiles(NH) : kDTiles16;
  constexpr uint32_t kSRegion = kTiles * NH;  // S region r at r * kSRegion
  static_assert(2 * kSRegion <= kCO, "S regions below the O regions");
  DMisc& ms = *reinterpret_cast<DMisc*>(sm + L::kMisc);
  CInfo* info = reinterpret_cast<CInfo*>(sm + L::kInfo);
  uint32_t* entry = reinterpret_cast<uint32_t*>(sm + L::kEntry);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  if (warp == Cfg::kIssueS) {
    tmem_alloc(&ms.tmem, kDTmemCols);
    tmem_relinquish();
  }
  if (tid == Cfg::kProdK * 32) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.bar_q[i], kDGroup);        // staged by softmax group 0
      mbar_init(&ms.bar_s[i], 1);
      mbar_init(&ms.s_free[i], Cfg::kSoft);    // read by every softmax thread
      mbar_init(&ms.bar_o[i], 1);
      mbar_init(&ms.o_free[i], kDGroup);       // read by softmax group 0
    }
    for (int i = 0; i < kDPBuf; ++i) {
      mbar_init(&ms.bar_p[i], kDGroup);        // each tile's P comes from one group
      mbar_init(&ms.bar_pv[i], 1);
    }
    for (int i = 0; i < L::kSlotsK; ++i) {
      mbar_init(&ms.full_k[i], 1);
      mbar_init(&ms.empty_k[i], 1);
    }
    for (int i = 0; i < L::kSlotsV; ++i) {
      mbar_init(&ms.full_v[i], 1);
      mbar_init(&ms.empty_v[i], 1);
      mbar_init(&ms.vsf_ready[i], 1);
    }
    mbar_init(&ms.drain_s, 1);
    mbar_init(&ms.drain_pv, 1);
    mbar_init(&ms.drain_cp, 1);
    ms.abort = 0;
    fence_mbar_init();
  }
  // The chunk table.  NVFP4: chunk w = x, x + X, ... of the units x cpu chunks
  // of C consecutive tiles.  FP16: the chunks of kDTiles16 listed tiles,
  // numbered unit by unit (a running sum over the units' counts), and this CTA
  // takes g = x, x + X, ... (at most kDMaxChunks: the host sizes X for a list
  // holding every tile).
  if (warp == 0) {
    if constexpr (PASS == kPassFp4) {
      const int W = p.units * p.cpu;
      const int nk = x < W ? (W - x + X - 1) / X : 0;
      for (int k = lane; k < nk; k += 32) {
        const int w = x + k * X;
        CInfo c;
        c.unit = w / p.cpu;
        c.slot = w % p.cpu;
        c.first = c.slot * p.C;
        c.nt = min(p.C, p.NT - c.first);
        info[k] = c;
      }
      if (lane == 0) ms.nk = nk;
    } else {
      int run = 0;
      for (int u0 = 0; u0 < p.units; u0 += 32) {
        const int u = u0 + lane;
        const int n = u < p.units ? p.n16[u] : 0;
        const int nch = (n + kDTiles16 - 1) / kDTiles16;
        int inc = nch;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += v;
        }
        const int P = run + inc - nch;  // first chunk of unit u
        for (int g = P + ((x - P) % X + X) % X; g < P + nch; g += X) {
          const int j = g - P;
          CInfo c;
          c.unit = u;
          c.slot = p.NT + j;
          c.first = j * kDTiles16;
          c.nt = min(kDTiles16, n - c.first);
          info[(g - x) / X] = c;
        }
        run += __shfl_sync(0xffffffffu, inc, 31);
      }
      if (lane == 0) ms.nk = run > x ? (run - x + X - 1) / X : 0;  // run: the chunks of all units
    }
  }
  // P buffers start zero: the rows of heads NG .. 15 and scale rows 16-31 are never written.
  for (int i = tid; i < kDPBuf * static_cast<int>(L::kPBuf) / 16; i += Cfg::kThreads)
    reinterpret_cast<uint4*>(sm + L::kP)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int nk = ms.nk;
  for (int e = tid; e < nk * kDMaxTiles; e += Cfg::kThreads) {
    const int k = e / kDMaxTiles, i = e % kDMaxTiles;
    const CInfo c = info[k];
    uint32_t v = 0u;
    if (i < c.nt) {
      const size_t row = static_cast<size_t>(c.unit) * p.NT;
      if constexpr (PASS == kPassFp4) {
        const int tile = c.first + i;
        v = static_cast<uint32_t>(tile) | (static_cast<uint32_t>(p.hbits[row + tile]) << 16);
      } else {
        v = p.list16[row + c.first + i];
      }
    }
    entry[e] = v;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem;
  const uint64_t wns = p.wait_ns;

  if (warp == Cfg::kProdK || warp == Cfg::kProdV) {
    // ======================== producers: K tiles, V tiles ========================
    const bool is_v = warp == Cfg::kProdV;
    if (lane == 0) {
      const CUtensorMap* map = is_v ? mV : mK;
      prefetch_tensormap(map);
      const int slots = is_v ? L::kSlotsV : L::kSlotsK;
      uint64_t* full = is_v ? ms.full_v : ms.full_k;
      uint64_t* empty = is_v ? ms.empty_v : ms.empty_k;
      uint8_t* ring = sm + (is_v ? L::kRingV : L::kRingK);
      // every cache tile is read once per step: let it leave L2 first (the
      // partial results the combine reads stay)
      const uint64_t pol = l2_evict_first_policy();
      int u = 0;
      bool ok = true;
      for (int k = 0; ok && k < nk; ++k) {
        const CInfo c = info[k];
        for (int i = 0; ok && i < c.nt; ++i) {
          const int tile = static_cast<int>(entry[k * kDMaxTiles + i] & 0xFFFFu);
          const int slot = u % slots, use = u / slots;
          if (use > 0 && !wait_or_abort(&empty[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, wns)) {
            ok = false;
            break;
          }
          if (!is_v && u == p.withhold) {  // take the slot, issue nothing
            ++u;
            continue;
          }
          uint8_t* st = ring + slot * L::kSlot;
          mbar_arrive_expect_tx(&full[slot], L::kSlot);
          if constexpr (PASS == kPassFp4) {
            if (!is_v) {
              tma_load_3d_hint(st, map, &full[slot], 0, tile * 128, c.unit, pol);
              bulk_load_hint(st + 8192, p.ks + (static_cast<size_t>(c.unit) * p.NT + tile) * 1024, 1024, &full[slot],
                             pol);
            } else {
              tma_load_3d_hint(st, map, &full[slot], tile * 64, 0, c.unit, pol);
              bulk_load_hint(st + 8192, p.vs + (static_cast<size_t>(c.unit) * 2 * p.NT + 2 * tile) * 512, 1024,
                             &full[slot], pol);
            }
          } else {
            for (int pnl = 0; pnl < 2; ++pnl)
              tma_load_3d_hint(st + pnl * 16384, map, &full[slot], pnl * 64, tile * 128, c.unit, pol);
          }
          ++u;
        }
      }
      // Let every copy this thread issued land before the CTA can exit (a
      // withheld slot's wait runs out after the same limit).
      for (int s = 0; s < slots; ++s)
        if (u > s) mbar_wait(&full[s], ((u - 1 - s) / slots) & 1, wns);
    }
    __syncwarp();
  } else if (warp == Cfg::kIssueS) {
    // ======================== S issuer: S^T of every tile of chunk k into S region k % 2 ========================
    if (lane == 0) {
      constexpr uint32_t idS4 = idesc_nvf4(128, NH);
      constexpr uint32_t idS16 = idesc_f16(128, NH, false);
      int u = 0;
      bool ok = true;
      for (int k = 0; ok && k < nk; ++k) {
        const CInfo c = info[k];
        const int r = k & 1;
        if (!wait_or_abort(&ms.bar_q[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, wns)) break;
        // S region r was last read by the softmax threads for chunk k - 2.
        if (k >= 2 && !wait_or_abort(&ms.s_free[r], ((k - 2) >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, wns))
          break;
        tc_fence_after();
        const uint32_t qs = sbase + r * L::kQSlot;
        if constexpr (PASS == kPassFp4)
          for (int cc = 0; cc < 2; ++cc)
            tmem_cp_32x128b_x4(tm + kCSFQ + 8 * r + 4 * cc, make_sdesc(qs + 1024 + 512 * cc, 16, 128, LAYOUT_NONE));
        const uint32_t sreg = tm + r * kSRegion;
#pragma unroll 1
        for (int i = 0; i < c.nt; ++i) {
          const int slot = u % L::kSlotsK;
          if (!wait_or_abort(&ms.full_k[slot], (u / L::kSlotsK) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, wns)) {
            ok = false;
            break;
          }
          ++u;
          tc_fence_after();
          const uint32_t st = sbase + L::kRingK + slot * L::kSlot;
          if constexpr (PASS == kPassFp4) {
            // these copies follow the previous products in this thread's
            // tcgen05 order, so they cannot overwrite scales those still read
            for (int cc = 0; cc < 2; ++cc)
              tmem_cp_32x128b_x4(tm + kCSFK + 4 * cc, make_sdesc(st + 8192 + 512 * cc, 16, 128, LAYOUT_NONE));
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
              mma_nvf4(sreg + NH * i, make_sdesc(st + 32 * cc, 16, 512, LAYOUT_SW64),
                       make_sdesc(qs + 32 * cc, 16, 512, LAYOUT_SW64), idS4, tm + kCSFK + 4 * cc,
                       tm + kCSFQ + 8 * r + 4 * cc, cc > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < kDD / 16; ++kk)
              mma_f16(sreg + NH * i, make_sdesc(st + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128),
                      make_sdesc(qs + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128), idS16, kk > 0);
          }
          mma_commit(&ms.empty_k[slot]);
        }
        if (!ok) break;
        mma_commit(&ms.bar_s[r]);
      }
      // drain: every tensor-core operation this thread issued completes before exit
      mma_commit(&ms.drain_s);
      mbar_wait(&ms.drain_s, 0, wns);
    }
    __syncwarp();
  } else if (warp == Cfg::kIssuePV) {
    // ======================== P V issuer: O^T += V^T P^T tile by tile into O region k % 2 ========================
    if (lane == 0) {
      constexpr uint32_t idS4 = idesc_nvf4(128, NH);
      constexpr uint32_t idO16 = idesc_f16_mn(128, NH, true, false);
      int u = 0, gt = 0;
      bool ok = true;
      for (int k = 0; ok && k < nk; ++k) {
        const CInfo c = info[k];
        const int r = k & 1;
        // O region r was last read by the softmax threads for chunk k - 2.
        if (k >= 2 && !wait_or_abort(&ms.o_free[r], ((k - 2) >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, wns))
          break;
        tc_fence_after();
        const uint32_t oreg = tm + kCO + 16 * r;
#pragma unroll 1
        for (int i = 0; i < c.nt; ++i, ++gt) {
          const int pb = gt % kDPBuf;
          const int slot = u % L::kSlotsV;
          // NVFP4 with a copier: it has put the slot's V scales into tensor
          // memory (after the copy landed); otherwise the copy itself
          constexpr bool kViaCopier = PASS == kPassFp4 && Cfg::kCopier;
          if (!wait_or_abort(kViaCopier ? &ms.vsf_ready[slot] : &ms.full_v[slot], (u / L::kSlotsV) & 1, &ms.abort,
                             p.err, DEV_TIMEOUT_LOAD, wns)) {
            ok = false;
            break;
          }
          ++u;
          tc_fence_after();
          const uint32_t st = sbase + L::kRingV + slot * L::kSlot;
          // (this slot's columns were last read by products of this thread,
          // which the copies follow in its tcgen05 order)
          if constexpr (PASS == kPassFp4 && !kViaCopier)
            for (int cc = 0; cc < 2; ++cc)
              tmem_cp_32x128b_x4(tm + kCSFV + 8 * slot + 4 * cc, make_sdesc(st + 8192 + 512 * cc, 16, 128, LAYOUT_NONE));
          if (!wait_or_abort(&ms.bar_p[pb], (gt / kDPBuf) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, wns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pbuf = sbase + L::kP + pb * L::kPBuf;
          if constexpr (PASS == kPassFp4) {
            // the P scales of buffer pb were written to tensor memory by the softmax threads
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
              mma_nvf4(oreg, make_sdesc(st + 32 * cc, 16, 512, LAYOUT_SW64),
                       make_sdesc(pbuf + 32 * cc, 16, 512, LAYOUT_SW64), idS4, tm + kCSFV + 8 * slot + 4 * cc,
                       tm + kCSFP + 8 * pb + 4 * cc, (i > 0 || cc > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16(oreg, make_sdesc(st + kk * 2048, 16384, 1024, LAYOUT_SW128),
                      make_sdesc(pbuf + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024, LAYOUT_SW128), idO16,
                      (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&ms.empty_v[slot]);
          mma_commit(&ms.bar_pv[pb]);
        }
        if (!ok) break;
        mma_commit(&ms.bar_o[r]);
      }
      mma_commit(&ms.drain_pv);
      mbar_wait(&ms.drain_pv, 0, wns);
    }
    __syncwarp();
  } else if (Cfg::kCopier && warp == Cfg::kCopyV) {
    // ======================== V scale copier (NVFP4 pass) ========================
    // Each V tile's scales into the tensor-memory columns of its ring slot, in
    // the order the P V issuer takes the tiles.  A slot is refilled only after
    // the products that read its columns completed (the producer waits for
    // them), so the copy cannot overwrite scales still in use.
    if constexpr (PASS == kPassFp4) {
      if (lane == 0) {
        int u = 0;
        bool ok = true;
        for (int k = 0; ok && k < nk; ++k) {
          const int nt = info[k].nt;
          for (int i = 0; i < nt; ++i) {
            const int slot = u % L::kSlotsV;
            if (!wait_or_abort(&ms.full_v[slot], (u / L::kSlotsV) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, wns)) {
              ok = false;
              break;
            }
            ++u;
            tc_fence_after();
            const uint32_t st = sbase + L::kRingV + slot * L::kSlot;
            for (int cc = 0; cc < 2; ++cc)
              tmem_cp_32x128b_x4(tm + kCSFV + 8 * slot + 4 * cc, make_sdesc(st + 8192 + 512 * cc, 16, 128,
                                                                             LAYOUT_NONE));
            mma_commit(&ms.vsf_ready[slot]);
          }
        }
        mma_commit(&ms.drain_cp);
        mbar_wait(&ms.drain_cp, 0, wns);
      }
    }
    __syncwarp();
  } else {
    // ======= softmax threads: lane = key of a tile, then channel of O^T =======
    // Group grp's thread tq takes key tq of its tiles (TMEM lane tq) and, in
    // group 0, channel tq of O^T.  Group 0 stages the query rows and writes
    // the chunk's results; the groups split each chunk's tiles by pairs.
    const int grp = Cfg::kGroups == 1 ? 0 : warp / 4, tq = tid % kDGroup;
    const float c2 = p.c2;
    const uint32_t lane_base = tm + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    bool failed = false;
    int gt0 = 0;  // tiles of this CTA before the chunk (P buffer of tile i: (gt0 + i) % kDPBuf)
    uint4 qa, qc;
    if (nk > 0 && grp == 0) {
      load_query(p, head0_of(p, info[0].unit), tq, qa, qc);
      stage_query<PASS>(sm, 0, tq, qa, qc);
      fence_proxy_async_smem();
      mbar_arrive(&ms.bar_q[0]);
    }
    for (int k = 0; k < nk; ++k) {
      const CInfo c = info[k];
      const size_t head0 = head0_of(p, c.unit);
      const int r = k & 1;
      const uint32_t* ent = entry + k * kDMaxTiles;
      // the next chunk's query rows, in flight while this chunk's S is read
      if (grp == 0 && k + 1 < nk) load_query(p, head0_of(p, info[k + 1].unit), tq, qa, qc);
      // ---- sweep 1: maximum of S per head over the keys this pass computes ----
      float mx[NG];
#pragma unroll
      for (int g = 0; g < NG; ++g) mx[g] = -INFINITY;
      if (!failed) failed = !wait_or_abort(&ms.bar_s[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, wns);
      failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
      const uint32_t sreg = lane_base + r * kSRegion;
      if (!failed) {
        tc_fence_after();
        // two tiles per load, every kGroups-th pair (the second tile, past the
        // chunk's end, reads columns of the region that no head takes: mine = 0)
        for (int i = 2 * grp; i < c.nt; i += 2 * Cfg::kGroups) {
          uint32_t s[2 * NH];
          load_pair<NH>(sreg + NH * i, s);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t h16 = ent[i + j] >> 16;
            const uint32_t mine = i + j >= c.nt ? 0u : PASS == kPassFp4 ? ~h16 : h16;  // heads this pass computes
#pragma unroll
            for (int g = 0; g < NG; ++g)
              mx[g] = fmaxf(mx[g], ((mine >> g) & 1u) ? __uint_as_float(s[j * NH + g]) : -INFINITY);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < NG; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
      if (lane == 0)
#pragma unroll
        for (int g = 0; g < NG; ++g) ms.red[warp][g] = mx[g];
      failed = softmax_bar_or<Cfg::kSoft>(failed);
      // base_g = 11 - M_g, M_g = ceil(max t) = ceil(fl32(max S * c2)); thread g
      // keeps its M for the epilogue.  A head with no key in this chunk's pass
      // has M = -inf: its P is zero, its l is zero and its M weighs nothing in
      // the combine.
      float base[NG];
      float my_m = -INFINITY;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float mw = ms.red[0][g];
#pragma unroll
        for (int w = 1; w < Cfg::kSoftWarps; ++w) mw = fmaxf(mw, ms.red[w][g]);
        const float M = ceilf(mw * c2);
        base[g] = static_cast<float>(kPLog2) - (M == -INFINITY ? 0.f : M);
        if (tid == g) my_m = M;
      }
      // The next chunk's query slot was last read by the S products of chunk
      // k - 1, which completed before this thread saw bar_s of chunk k - 1.
      if (!failed && grp == 0 && k + 1 < nk) {
        stage_query<PASS>(sm, r ^ 1, tq, qa, qc);
        fence_proxy_async_smem();
        mbar_arrive(&ms.bar_q[r ^ 1]);
      }
      // ---- sweep 2: P per head and key, tile i into buffer (gt0 + i) % kDPBuf ----
      float lsum[NG];
#pragma unroll
      for (int g = 0; g < NG; ++g) lsum[g] = 0.f;
      if constexpr (PASS == kPassFp4) {
        // Two tiles at a time (two independent chains per warp), pairs
        // alternating between the groups.  failed is the same in every softmax
        // warp here, and stays the same within a group at the end of every
        // pair: the loop holds a barrier that each of its warps reaches.
        for (int i = 2 * grp; i < c.nt && !failed; i += 2 * Cfg::kGroups) {
          const bool two = i + 1 < c.nt;
          const int gt = gt0 + i;
          const int pb0 = gt % kDPBuf, pb1 = (gt + 1) % kDPBuf;
          if (gt >= kDPBuf)
            failed = !wait_or_abort(&ms.bar_pv[pb0], ((gt - kDPBuf) / kDPBuf) & 1, &ms.abort, p.err,
                                    DEV_TIMEOUT_MMA, wns);
          if (!failed && two && gt + 1 >= kDPBuf)
            failed = !wait_or_abort(&ms.bar_pv[pb1], ((gt + 1 - kDPBuf) / kDPBuf) & 1, &ms.abort, p.err,
                                    DEV_TIMEOUT_MMA, wns);
          failed = __any_sync(0xffffffffu, failed);
          uint8_t* pbuf[2] = {sm + L::kP + pb0 * L::kPBuf, sm + L::kP + pb1 * L::kPBuf};
          if (!failed) {
            tc_fence_after();
            uint32_t s[2 * NH];
            load_pair<NH>(sreg + NH * i, s);
            // Every head of both tiles at once: the group maximum over 16
            // consecutive keys (lanes), the group scale, P * 2^11 / scale and
            // its code; heads that keep the tile in FP16 get zero codes and
            // scales.  (The second tile of an odd end is computed and dropped.)
            uint32_t mine[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) mine[j] = ~(ent[i + j] >> 16);
            float gm[2][NG];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int g = 0; g < NG; ++g) gm[j][g] = __uint_as_float(s[j * NH + g]);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1)
#pragma unroll
              for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int g = 0; g < NG; ++g) gm[j][g] = fmaxf(gm[j][g], __shfl_xor_sync(0xffffffffu, gm[j][g], o));
            uint32_t wd[2][NG], sbyte[2][NG];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int g = 0; g < NG; ++g) {
                const bool on = (mine[j] >> g) & 1u;
                const float amax = ex2(fmaf(gm[j][g], c2, base[g]));  // max of P * 2^11 in the group
                const uint32_t sb = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.f) & 0xFFu;
                const float sc0 = e4m3_to_f32(sb);
                const float sc = sc0 <= 0.f ? 1.0f : sc0;  // zero scale: the code rounds to 0, l keeps P
                const float xv = ex2(fmaf(__uint_as_float(s[j * NH + g]), c2, base[g] - lg2(sc)));  // P 2^11 / scale
                if (j == 0 || two) lsum[g] = fmaf(on ? xv : 0.f, sc, lsum[g]);
                sbyte[j][g] = on ? sb : 0u;
                wd[j][g] = on ? ((cvt_e2m1x2(xv, 0.f) & 0xFu) << (4 * (lane & 7))) : 0u;
              }
            // codes of keys 8m .. 8m + 7 in one word (key t at byte t / 2 of row g)
#pragma unroll
            for (int o = 1; o < 8; o <<= 1)
#pragma unroll
              for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int g = 0; g < NG; ++g) wd[j][g] |= __shfl_xor_sync(0xffffffffu, wd[j][g], o);
#pragma unroll
            for (int j = 0; j < 2; ++j)
              if (j == 0 || two)
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                  if ((lane & 7) == 0)
                    *reinterpret_cast<uint32_t*>(pbuf[j] + sw64_off(g, warp % 4) + (lane >> 1)) = wd[j][g];
                  if ((lane & 15) == 0)
                    pbuf[j][1024 + (tq / 64) * 512 + g * 16 + (tq % 64) / 16] = static_cast<uint8_t>(sbyte[j][g]);
                }
          }
          // The P scales into tensor memory, in the layout a 32x128b.warpx4
          // copy of the two 512-byte scale chunks gives: row g of chunk cc at
          // lane g of every 32-lane quarter, columns kCSFP + 8 pb + 4 cc ..
          // + 3.  Each warp writes its own quarter once every warp of its group
          // has written its bytes; every warp of the group reaches this barrier
          // on every pair, and leaves with the others if any gave up a wait.
          if (Cfg::kGroups == 1 || grp == 0)
            failed = bar_or<kBarPsf, kDGroup>(failed);
          else
            failed = bar_or<kBarPsf + 1, kDGroup>(failed);
          if (failed) break;
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (j == 0 || two) {
              const uint4 r0 = *reinterpret_cast<const uint4*>(pbuf[j] + 1024 + lane * 16);
              const uint4 r1 = *reinterpret_cast<const uint4*>(pbuf[j] + 1536 + lane * 16);
              const uint32_t sfw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
              tmem_st8(lane_base + kCSFP + 8 * (j == 0 ? pb0 : pb1), sfw);
            }
          tmem_st_wait();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&ms.bar_p[pb0]);
          if (two) mbar_arrive(&ms.bar_p[pb1]);
        }
      } else {
        for (int i = grp; i < c.nt && !failed; i += Cfg::kGroups) {
          const int gt = gt0 + i;
          const int pb = gt % kDPBuf;
          if (gt >= kDPBuf)
            failed = !wait_or_abort(&ms.bar_pv[pb], ((gt - kDPBuf) / kDPBuf) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA,
                                    wns);
          failed = __any_sync(0xffffffffu, failed);
          if (failed) break;
          tc_fence_after();
          const uint32_t mine = ent[i] >> 16;
          uint32_t s[NH];
          load_cols<NH>(sreg + NH * i, s);
          uint8_t* pbuf = sm + L::kP + pb * L::kPBuf;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const bool on = (mine >> g) & 1u;
            const float xv = on ? ex2(fmaf(__uint_as_float(s[g]), c2, base[g])) : 0.f;  // P * 2^11
            lsum[g] += xv;
            *reinterpret_cast<__half*>(pbuf + (tq / 64) * 2048 + sw128_off(g, (tq % 64) / 8) + (tq % 8) * 2) =
                __float2half_rn(xv);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&ms.bar_p[pb]);
        }
      }
      gt0 += c.nt;
      tc_fence_before();
      mbar_arrive(&ms.s_free[r]);
      // ---- epilogue (group 0): the chunk's O^T column g, l_g and M_g ----
      if (!failed && grp == 0)
        failed = !wait_or_abort(&ms.bar_o[r], (k >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, wns);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < NG; ++g) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], o);
      if (lane == 0)
#pragma unroll
        for (int g = 0; g < NG; ++g) ms.lred[warp][g] = lsum[g];
      failed = softmax_bar_or<Cfg::kSoft>(failed);
      if (failed) break;
      if (grp == 0) {
        tc_fence_after();
        uint32_t o[NH];
        load_cols<NH>(lane_base + kCO + 16 * r, o);
#pragma unroll
        for (int g = 0; g < NG; ++g)
          if (g < p.G) p.part_o[((head0 + g) * p.cap + c.slot) * kDD + tq] = __uint_as_float(o[g]);
        if (tq < p.G) {
          const size_t idx = (head0 + tq) * p.cap + c.slot;
          float lt = 0.f;
#pragma unroll
          for (int w = 0; w < Cfg::kSoftWarps; ++w) lt += ms.lred[w][tq];
          p.part_l[idx] = lt;
          p.part_m[idx] = my_m;
        }
        tc_fence_before();
        mbar_arrive(&ms.o_free[r]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::kIssueS) {
    tc_fence_after();
    tmem_dealloc(tm, kDTmemCols);
  }
}

// Both passes in one launch: CTAs 0 .. grid16 - 1 run the FP16 pass, the rest
// the NVFP4 pass (which needs nothing from the FP16 pass), so NVFP4 CTAs start
// on the SMs that FP16 CTAs leave.
// Both passes in one launch: CTAs 0 .. grid16 - 1 run the FP16 pass, the rest
// the NVFP4 pass (which needs nothing from the FP16 pass), so NVFP4 CTAs start
// on the SMs that FP16 CTAs leave.
template <int NG>
__global__ void __launch_bounds__(DCfg<NG>::kBound, 1)
    thrift_decode_kernel(const __grid_constant__ CUtensorMap mK16, const __grid_constant__ CUtensorMap mV16,
                         const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                         const DParams p) {
  griddep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Everything below reads the tile bits, lists and counts of the compaction
  // kernel and writes partial results the previous combine may still read.
  griddep_wait();
  const int b = static_cast<int>(blockIdx.x);
  if (b < p.grid16)
    decode_pass<kPassFp16, NG>(&mK16, &mV16, p, sm, b, p.grid16);
  else
    decode_pass<kPassFp4, NG>(&mK4, &mV4, p, sm, b - p.grid16, static_cast<int>(gridDim.x) - p.grid16);
}

// Per unit (b, kv head): bit g of hbits[t] = query head g of the group keeps
// key tile t in FP16; list16 = the tiles with any bit, ascending, as tile |
// bits << 16; n16 = their number.  One thread per tile (NT <= 1024).
__global__ void __launch_bounds__(1024) decode_compact_kernel(const uint8_t* __restrict__ mask, int Hq, int Hkv,
                                                              int NT, uint16_t* __restrict__ hbits,
                                                              uint32_t* __restrict__ list16, int* __restrict__ n16) {
  __shared__ int wtot[32];
  griddep_launch_dependents();
  griddep_wait();  // the mask may come from the kernel before
  const int unit = blockIdx.x, G = Hq / Hkv;
  const size_t head0 = static_cast<size_t>(unit / Hkv) * Hq + static_cast<size_t>(unit % Hkv) * G;
  const int t = threadIdx.x, warp = t / 32, lane = t % 32;
  uint32_t bits = 0u;
  if (t < NT) {
    for (int g = 0; g < G; ++g) bits |= (mask[(head0 + g) * NT + t] ? 1u : 0u) << g;
    hbits[static_cast<size_t>(unit) * NT + t] = static_cast<uint16_t>(bits);
  }
  const uint32_t bal = __ballot_sync(0xffffffffu, bits != 0u);
  if (lane == 0) wtot[warp] = __popc(bal);
  __syncthreads();
  int off = 0;
  for (int w = 0; w < warp; ++w) off += wtot[w];
  if (bits) list16[static_cast<size_t>(unit) * NT + off + __popc(bal & ((1u << lane) - 1u))] =
      static_cast<uint32_t>(t) | (bits << 16);
  if (t == 0) {
    int n = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) n += wtot[w];
    n16[unit] = n;
  }
}

// 2^e for an integer-valued e <= 0, exactly; 0 below 2^-126 and for e = -inf
// or NaN (a difference of two infinite maxima: chunks that weigh nothing).
__device__ __forceinline__ float pow2_weight(float e) { return e >= -126.0f ? exp2_int(e) : 0.f; }

// O = sum_c 2^(M_c - M) O_c / sum_c 2^(M_c - M) l_c over the head's NVFP4
// chunks (slots 0 .. cpu - 1) and FP16 chunks (slots NT ..); both carry the
// 2^11 pre-scale; a chunk with M_c = -inf holds no key of the head and weighs
// 0.  One CTA of 512 threads per (batch, query head), one pass over the
// partial results: warp w merges chunks c = w, w + 16, ... eight at a time
// (all eight rows loaded before any is used) into a running (M, l, O), lane
// j holding channels 4 j .. 4 j + 3 (one coalesced 512-byte row per chunk);
// the maxima are integers, so every rescale is an exact power of two.  Then
// warp 0 merges the sixteen warps in order.
__global__ void __launch_bounds__(512) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_l,
                                                             const float* __restrict__ part_m,
                                                             const int* __restrict__ n16, int Hq, int Hkv, int NT,
                                                             int cpu, int cap, __half* __restrict__ O) {
  constexpr int kWarps = 16;
  __shared__ float4 red4[kWarps][32];
  __shared__ float redm[kWarps], redl[kWarps];
  griddep_wait();  // the passes' partial results
  const size_t bh = blockIdx.x;
  const int G = Hq / Hkv;
  const int unit = static_cast<int>(bh / Hq) * Hkv + static_cast<int>(bh % Hq) / G;
  const int chunks = cpu + (n16[unit] + kDTiles16 - 1) / kDTiles16;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float* pm = part_m + bh * cap;
  const float* pl = part_l + bh * cap;
  const float4* po = reinterpret_cast<const float4*>(part_o + bh * cap * kDD);
  constexpr int kBatch = 8;  // chunk rows a lane has in flight at once
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = warp; c0 < chunks; c0 += kWarps * kBatch) {
    float mc[kBatch], lc[kBatch];
    float4 v[kBatch];
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const int c = c0 + r * kWarps;
      const int slot = c < cpu ? c : NT + (c - cpu);
      const bool in = c < chunks;
      mc[r] = in ? pm[slot] : -INFINITY;
      lc[r] = in ? pl[slot] : 0.f;
      v[r] = in ? po[static_cast<size_t>(slot) * (kDD / 4) + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mb = mc[0];
#pragma unroll
    for (int r = 1; r < kBatch; ++r) mb = fmaxf(mb, mc[r]);
    if (mb > M) {  // a new maximum: rescale what is summed so far
      const float f = pow2_weight(M - mb);
      acc.x *= f;
      acc.y *= f;
      acc.z *= f;
      acc.w *= f;
      L *= f;
      M = mb;
    }
#pragma unroll
    for (int r = 0; r < kBatch; ++r) {
      const float wgt = pow2_weight(mc[r] - M);
      acc.x = fmaf(wgt, v[r].x, acc.x);
      acc.y = fmaf(wgt, v[r].y, acc.y);
      acc.z = fmaf(wgt, v[r].z, acc.z);
      acc.w = fmaf(wgt, v[r].w, acc.w);
      L = fmaf(wgt, lc[r], L);
    }
  }
  red4[warp][lane] = acc;
  if (lane == 0) {
    redm[warp] = M;
    redl[warp] = L;
  }
  __syncthreads();
  if (warp == 0) {
    float Mt = redm[0];
    for (int w = 1; w < kWarps; ++w) Mt = fmaxf(Mt, redm[w]);
    float Lt = 0.f;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int w = 0; w < kWarps; ++w) {
      const float f = pow2_weight(redm[w] - Mt);
      const float4 v = red4[w][lane];
      sum.x = fmaf(f, v.x, sum.x);
      sum.y = fmaf(f, v.y, sum.y);
      sum.z = fmaf(f, v.z, sum.z);
      sum.w = fmaf(f, v.w, sum.w);
      Lt = fmaf(f, redl[w], Lt);
    }
    __half2* out = reinterpret_cast<__half2*>(O + bh * kDD + 4 * lane);
    out[0] = __floats2half2_rn(sum.x / Lt, sum.y / Lt);
    out[1] = __floats2half2_rn(sum.z / Lt, sum.w / Lt);
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

// One CTA of 1024 threads per (batch, query head); nb <= 1024, D = 128.
// score_j = fl32(sm_scale * fl32(q . kmean_j)): the products of the fp16
// query and the FP32 means are exact in FP64; their FP64 sum (one warp per key
// block, lane l holding channels 4 l .. 4 l + 3 so that a block's 512 bytes
// are one coalesced load, then a warp tree) is rounded once.  Then the top k
// of the unique 64-bit keys: a bitonic sort into descending order (stages
// across warps through shared memory, stages within a warp by shuffles), and
// the first k sorted keys name the selected blocks.  The keys are unique, so
// the set is the k largest, as a ranking would give.
__global__ void __launch_bounds__(1024) decode_select_kernel(const __half* __restrict__ q,
                                                             const float* __restrict__ km, int Hq, int Hkv, int nb,
                                                             float sm_scale, long long k, uint8_t* __restrict__ mask) {
  constexpr int kRows = 8;  // key blocks per warp and step, all loads in flight at once
  __shared__ unsigned long long keys[1024];
  __shared__ uint8_t sel[1024];
  griddep_launch_dependents();
  const size_t bh = blockIdx.x;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  const int G = Hq / Hkv;
  const int i = threadIdx.x, warp = i / 32, lane = i % 32;
  const float* kmh = km + (static_cast<size_t>(b) * Hkv + h / G) * nb * static_cast<size_t>(kDD);
  double qd[4];
  {
    const uint2 qv = *reinterpret_cast<const uint2*>(q + bh * kDD + 4 * lane);
    const float2 q01 = __half22float2(*reinterpret_cast<const __half2*>(&qv.x));
    const float2 q23 = __half22float2(*reinterpret_cast<const __half2*>(&qv.y));
    qd[0] = q01.x;
    qd[1] = q01.y;
    qd[2] = q23.x;
    qd[3] = q23.y;
  }
  sel[i] = 0;
  if (i >= nb) keys[i] = 0ull;  // padding past nb sorts last (blocks below nb are all written below)
  for (int j0 = warp * kRows; j0 < nb; j0 += 32 * kRows) {
    float4 v[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      v[r] = j0 + r < nb ? reinterpret_cast<const float4*>(kmh + static_cast<size_t>(j0 + r) * kDD)[lane]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    double dot[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      dot[r] = fma(qd[0], static_cast<double>(v[r].x), fma(qd[1], static_cast<double>(v[r].y),
               fma(qd[2], static_cast<double>(v[r].z), qd[3] * static_cast<double>(v[r].w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < kRows; ++r) dot[r] += __shfl_xor_sync(0xffffffffu, dot[r], o);
    if (lane < kRows && j0 + lane < nb) {
      double d = dot[0];
#pragma unroll
      for (int r = 1; r < kRows; ++r) d = lane == r ? dot[r] : d;
      const float sc = static_cast<float>(static_cast<double>(sm_scale) * static_cast<double>(static_cast<float>(d)));
      keys[j0 + lane] = decode_key(sc, j0 + lane, nb);
    }
  }
  __syncthreads();
  unsigned long long key = keys[i];
  // bitonic sort of the 1024 keys, descending (element i held by thread i)
  for (int kk = 2; kk <= 1024; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      unsigned long long other;
      if (j >= 32) {
        keys[i] = key;
        __syncthreads();
        other = keys[i ^ j];
        __syncthreads();
      } else {
        other = __shfl_xor_sync(0xffffffffu, key, j);
      }
      // the pair (i, i ^ j) is ordered descending in blocks where (i & kk) == 0
      const bool lower = (i & j) == 0, desc = (i & kk) == 0;
      const bool take_max = lower == desc;
      key = take_max ? (key > other ? key : other) : (key < other ? key : other);
    }
  }
  if (i < k) sel[0x7FFFFFFF - static_cast<int>(key & 0x7FFFFFFFull)] = 1;
  __syncthreads();
  if (i < nb) mask[bh * nb + i] = sel[i];
}

}  // namespace

namespace {
constexpr int kMaxDevices = 64;

// SM count of the current device, asked once per device.
int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}
}  // namespace

// The FP16 pass takes one CTA per SM (more if a list holding every tile would
// give a CTA more than kDMaxChunks chunks); the NVFP4 pass as many again, with
// the chunk size (at most the TMEM budget's) that minimises the most key tiles
// any of its CTAs takes, counting half a tile of per-chunk overhead, ties to
// the larger chunk.
DecodePlan decode_plan(const thrift_shape& s) {
  const int NT = num_tiles(s.N);
  const long long units = static_cast<long long>(s.B) * s.Hkv;
  const int NH = (s.Hq / s.Hkv) <= 8 ? 8 : 16;
  const int cmax = decode_chunk_tiles(NH);
  const long long nsm = sm_count();
  DecodePlan pl;
  pl.ch16 = (NT + kDTiles16 - 1) / kDTiles16;
  const long long need16 = (units * pl.ch16 + kDMaxChunks - 1) / kDMaxChunks;
  pl.grid16 = static_cast<int>(need16 > nsm ? need16 : nsm);
  pl.C = cmax < NT ? cmax : NT;
  pl.cpu = (NT + pl.C - 1) / pl.C;
  pl.grid4 = static_cast<int>(nsm);
  double best_cost = 1e300;
  for (int C = 1; C <= cmax && C <= NT; ++C) {
    const long long cpu = (NT + C - 1) / C;
    const long long W = units * cpu;
    long long grid = W < nsm ? W : nsm;
    if (grid * kDMaxChunks < W) grid = (W + kDMaxChunks - 1) / kDMaxChunks;
    const double cost = static_cast<double>((W + grid - 1) / grid) * (C + 0.5);
    if (cost <= best_cost) {
      best_cost = cost;
      pl.C = C;
      pl.cpu = static_cast<int>(cpu);
      pl.grid4 = static_cast<int>(grid);
    }
  }
  return pl;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Partial results: NT NVFP4 slots (one-tile chunks, the most any plan makes)
// and every FP16 chunk slot per head; then the per-unit tile bits, lists and
// counts.
static size_t decode_rows(const thrift_shape& s) {
  const size_t NT = num_tiles(s.N);
  return static_cast<size_t>(s.B) * s.Hq * (NT + (NT + kDTiles16 - 1) / kDTiles16);
}

size_t decode_workspace_bytes(const thrift_shape& s) {
  const size_t rows = decode_rows(s);
  const size_t units = static_cast<size_t>(s.B) * s.Hkv, NT = num_tiles(s.N);
  return align256(static_cast<size_t>(s.B) * s.Hq * NT) + align256(rows * kDD * sizeof(float)) +
         2 * align256(rows * sizeof(float)) + align256(units * NT * sizeof(uint16_t)) +
         align256(units * NT * sizeof(uint32_t)) + align256(units * sizeof(int));
}

DecodeWs decode_carve(void* ws, const thrift_shape& s) {
  const size_t rows = decode_rows(s);
  const size_t units = static_cast<size_t>(s.B) * s.Hkv, NT = num_tiles(s.N);
  uint8_t* p = static_cast<uint8_t*>(ws);
  DecodeWs w;
  w.mask = p;
  p += align256(static_cast<size_t>(s.B) * s.Hq * NT);
  w.part_o = reinterpret_cast<float*>(p);
  p += align256(rows * kDD * sizeof(float));
  w.part_l = reinterpret_cast<float*>(p);
  p += align256(rows * sizeof(float));
  w.part_m = reinterpret_cast<float*>(p);
  p += align256(rows * sizeof(float));
  w.hbits = reinterpret_cast<uint16_t*>(p);
  p += align256(units * NT * sizeof(uint16_t));
  w.list16 = reinterpret_cast<uint32_t*>(p);
  p += align256(units * NT * sizeof(uint32_t));
  w.n16 = reinterpret_cast<int*>(p);
  return w;
}

namespace {
// Launch on `st` with programmatic stream serialization: the kernel may start
// while the one before it in the stream finishes, and waits for it
// (griddepcontrol.wait) before touching what that one writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Every decode kernel asks for the largest shared-memory carveout, so that
// consecutive kernels of a step do not make the SMs change their L1 / shared
// split between them; `smem` > 0 also raises its dynamic shared-memory limit.
// Function attributes are per device: each kernel sets them once per device
// (a bit per device in `done`), not on every call.
template <typename K>
cudaError_t kernel_attributes(K kernel, std::atomic<uint32_t>& done, size_t smem = 0) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint32_t bit = dev >= 0 && dev < 32 ? (1u << dev) : 0u;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  if (smem > 0 && (e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(smem))) != cudaSuccess)
    return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           static_cast<int>(cudaSharedmemCarveoutMaxShared));
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int NG>
cudaError_t launch_passes(const CUtensorMap (&maps)[4], const DParams& prm, const DecodePlan& pl, cudaStream_t st) {
  const size_t smem = (DLayout<kPassFp4>::kBytes > DLayout<kPassFp16>::kBytes ? DLayout<kPassFp4>::kBytes
                                                                                : DLayout<kPassFp16>::kBytes) +
                      1024;
  static std::atomic<uint32_t> done{0};
  cudaError_t e = kernel_attributes(thrift_decode_kernel<NG>, done, smem);
  if (e != cudaSuccess) return e;
  e = launch_dependent(thrift_decode_kernel<NG>, dim3(pl.grid16 + pl.grid4), dim3(DCfg<NG>::kThreads), smem, st, maps[0],
                       maps[1], maps[2], maps[3], prm);
  if (e == cudaErrorInvalidValue) {
    // the attributes were set in a context that has since been reset: once more
    cudaGetLastError();
    done.store(0u, std::memory_order_release);
    if ((e = kernel_attributes(thrift_decode_kernel<NG>, done, smem)) != cudaSuccess) return e;
    e = launch_dependent(thrift_decode_kernel<NG>, dim3(pl.grid16 + pl.grid4), dim3(DCfg<NG>::kThreads), smem, st, maps[0],
                         maps[1], maps[2], maps[3], prm);
  }
  return e;
}
}  // namespace

cudaError_t launch_decode_select(const void* q, const float* km, const thrift_shape& s, double rho, uint8_t* mask,
                                 cudaStream_t st) {
  const int nb = s.N / s.blk;
  double kk = ceil(rho * static_cast<double>(nb) - 1e-9);
  if (kk < 0) kk = 0;
  if (kk > nb) kk = nb;
  static std::atomic<uint32_t> done{0};
  const cudaError_t e = kernel_attributes(decode_select_kernel, done);
  if (e != cudaSuccess) return e;
  decode_select_kernel<<<s.B * s.Hq, 1024, 0, st>>>(static_cast<const __half*>(q), km, s.Hq, s.Hkv, nb, s.sm_scale,
                                                   static_cast<long long>(kk), mask);
  return cudaGetLastError();
}

cudaError_t launch_decode_attention(const void* q, const void* K, const void* V, const void* k4, const void* ks,
                                    const void* v4, const void* vs, const uint8_t* mask, const thrift_shape& s,
                                    void* O, const DecodeWs& w, uint32_t* err, cudaStream_t st) {
  CUtensorMap maps[4];  // fp16 K, fp16 V, NVFP4 K, NVFP4 V
  const uint64_t BHk = static_cast<uint64_t>(s.B) * s.Hkv;
  bool ok = true;
  ok &= make_tmap_3d(&maps[0], K, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kDD, s.N, BHk, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&maps[1], V, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kDD, s.N, BHk, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&maps[2], k4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kDD / 2, s.N, BHk, kDD / 2, 128,
                     CU_TENSOR_MAP_SWIZZLE_64B);
  ok &= make_tmap_3d(&maps[3], v4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.N / 2, kDD, BHk, 64, kDD,
                     CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) return cudaErrorInvalidValue;
  const DecodePlan pl = decode_plan(s);
  const int G = s.Hq / s.Hkv;
  const int NT = num_tiles(s.N);
  static std::atomic<uint32_t> done_compact{0}, done_combine{0};
  cudaError_t e = kernel_attributes(decode_compact_kernel, done_compact);
  if (e != cudaSuccess) return e;
  if ((e = kernel_attributes(decode_combine_kernel, done_combine)) != cudaSuccess) return e;
  e = launch_dependent(decode_compact_kernel, dim3(static_cast<unsigned>(BHk)), dim3(1024), 0, st, mask, s.Hq, s.Hkv,
                       NT, w.hbits, w.list16, w.n16);
  if (e != cudaSuccess) return e;
  DParams prm;
  prm.q = static_cast<const __half*>(q);
  prm.hbits = w.hbits;
  prm.list16 = w.list16;
  prm.n16 = w.n16;
  prm.ks = static_cast<const uint8_t*>(ks);
  prm.vs = static_cast<const uint8_t*>(vs);
  prm.part_o = w.part_o;
  prm.part_l = w.part_l;
  prm.part_m = w.part_m;
  prm.err = err;
  prm.wait_ns = wait_limit_ns();
  prm.withhold = test_withhold_tile();
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.NT = NT;
  prm.G = G;
  prm.units = static_cast<int>(BHk);
  prm.C = pl.C;
  prm.cpu = pl.cpu;
  prm.cap = NT + pl.ch16;
  prm.grid16 = pl.grid16;
  prm.c2 = static_cast<float>(static_cast<double>(s.sm_scale) * 1.4426950408889634073599246810019);
  if (G <= 4)
    e = launch_passes<4>(maps, prm, pl, st);
  else if (G <= 8)
    e = launch_passes<8>(maps, prm, pl, st);
  else
    e = launch_passes<16>(maps, prm, pl, st);
  if (e != cudaSuccess) return e;
  return launch_dependent(decode_combine_kernel, dim3(s.B * s.Hq), dim3(512), 0, st, w.part_o, w.part_l, w.part_m,
                          w.n16, s.Hq, s.Hkv, NT, pl.cpu, prm.cap, static_cast<__half*>(O));
}

}  // namespace thrift

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
//   decode_attention  one CTA per (batch, kv head, chunk of <= 6 key tiles),
//                     all G query heads of the kv head at once, keys on the
//                     128 tensor-memory lanes:
//                       S^T = K q^T   (M = 128 keys, N = 16 heads: NVFP4 with the
//                                      prefill's K codes, and fp16 for the
//                                      tiles any head of the group keeps in FP16)
//                       P per head and key, relative to the chunk's maximum
//                       O^T += V^T P^T (M = 128 channels, N = 16 heads; NVFP4
//                                      with the prefill's V codes as A, fp16 V
//                                      as an MN-major A)
//                     Two passes per chunk: every S first, so each head has one
//                     maximum per chunk and O is never rescaled; then P and the
//                     P V products.  Writes the chunk's unnormalised O, l, M.
//   decode_combine    one CTA per (batch, query head): O = sum_c 2^(M_c - M) O_c
//                     / sum_c 2^(M_c - M) l_c (exact power-of-two rescales).
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
constexpr int kDHeads = 16;      // N of the products: one kv group's query heads, padded
constexpr int kDThreads = 192;   // warps 0-3 softmax, 4 producer, 5 MMA issuer
constexpr int kDSoftmax = 128;
constexpr int kDProducer = 4;
constexpr int kDMma = 5;
constexpr int kDRing = 6;        // NVFP4 slots: K4 + K scales or V4 + V scales
constexpr uint32_t kDTmemCols = 256;

// Tensor-memory columns.
constexpr uint32_t kCS = 0;      // tile i: S4^T at 32 i, S16^T at 32 i + 16
constexpr uint32_t kCO = 192;    // O^T, 16 columns
constexpr uint32_t kCSFK = 208;  // K scales (A of S^T), two 64-wide chunks of D
constexpr uint32_t kCSFQ = 216;  // q scales (B of S^T)
constexpr uint32_t kCSFV = 224;  // V scales (A of O^T), two 64-key chunks
constexpr uint32_t kCSFP = 232;  // P scales (B of O^T)

struct DSmem {
  static constexpr uint32_t kQ16 = 0;       // 16 x 128 fp16: two 64-wide SW128 panels of 2 KB
  static constexpr uint32_t kQ4 = 4096;     // 16 x 64 B E2M1, SW64
  static constexpr uint32_t kQSF = 5120;    // q scales: two 512-byte chunks
  static constexpr uint32_t kP4 = 6144;     // P codes: two buffers of 16 x 64 B, SW64
  static constexpr uint32_t kPSF = 8192;    // P scales: two buffers of two 512-byte chunks
  static constexpr uint32_t kP16 = 10240;   // fp16 P: two buffers of 16 x 128, two SW128 panels each
  static constexpr uint32_t kSlotBytes = 9216;  // 8 KB codes + 1 KB scales
  static constexpr uint32_t kRing = 18432;
  static constexpr uint32_t kS16 = kRing + kDRing * kSlotBytes;  // one fp16 K or V tile (32 KB)
  static constexpr uint32_t kMisc = kS16 + 32768;
  static constexpr uint32_t kBytes = kMisc + 1024;
  static_assert(kRing % 1024 == 0 && kS16 % 1024 == 0 && kP16 % 1024 == 0, "swizzled tiles need 1 KB alignment");
  static_assert(2 * (kBytes + 2048) <= 233472, "two CTAs per SM");
};

struct DMisc {
  uint64_t bar_q;                            // query copies staged (128 arrivals)
  uint64_t bar_full[kDRing], bar_empty[kDRing];
  uint64_t bar_full16, bar_empty16;
  uint64_t bar_s;                            // every S^T of the chunk written
  uint64_t bar_p[2];                         // P buffer b written (128 arrivals)
  uint64_t bar_pv[2];                        // P buffer b multiplied into O^T
  uint64_t bar_o;                            // every P V product done
  uint64_t bar_drain;
  uint32_t tmem;
  volatile int abort;
  uint32_t sel[8];                           // per tile: bit g set when query head g keeps it in FP16
  float red[4][kDHeads];                     // per-warp maxima of S
  float lred[4][kDHeads];                    // per-warp sums of P
};
static_assert(sizeof(DMisc) <= 1024, "barriers must fit their shared-memory slice");

struct DParams {
  const __half* q;       // [B][Hq][D]
  const uint8_t* mask;   // [B][Hq][nb], 1 = FP16 block
  const uint8_t* ks;     // K scales, prefill layout
  const uint8_t* vs;     // V scales, prefill layout
  float* part_o;         // [B][Hq][chunks][D]
  float* part_l;         // [B][Hq][chunks]
  float* part_m;         // [B][Hq][chunks]
  uint32_t* err;
  int Hq, Hkv, NT, G, tiles_per_cta, chunks;
  float c2;              // fl32(sm_scale * log2 e)
};

__global__ void __launch_bounds__(kDThreads, 2)
    thrift_decode_kernel(const __grid_constant__ CUtensorMap mK16, const __grid_constant__ CUtensorMap mV16,
                         const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                         const DParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DMisc& ms = *reinterpret_cast<DMisc*>(sm + DSmem::kMisc);
  const uint32_t sbase = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int chunk = blockIdx.x, bhk = blockIdx.y;
  const int b = bhk / p.Hkv, hkv = bhk % p.Hkv;
  const int G = p.G;
  const int t0 = chunk * p.tiles_per_cta;
  const int nt = min(p.tiles_per_cta, p.NT - t0);  // >= 1: chunks = ceil(NT / tiles_per_cta)
  const size_t head0 = static_cast<size_t>(b) * p.Hq + static_cast<size_t>(hkv) * G;  // first query head

  if (warp == kDMma) {
    tmem_alloc(&ms.tmem, kDTmemCols);
    tmem_relinquish();
  }
  if (tid == kDProducer * 32) {
    mbar_init(&ms.bar_q, kDSoftmax);
    for (int i = 0; i < kDRing; ++i) {
      mbar_init(&ms.bar_full[i], 1);
      mbar_init(&ms.bar_empty[i], 1);
    }
    mbar_init(&ms.bar_full16, 1);
    mbar_init(&ms.bar_empty16, 1);
    mbar_init(&ms.bar_s, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.bar_p[i], kDSoftmax);
      mbar_init(&ms.bar_pv[i], 1);
    }
    mbar_init(&ms.bar_o, 1);
    mbar_init(&ms.bar_drain, 1);
    ms.abort = 0;
    fence_mbar_init();
  }
  if (tid < nt) {
    uint32_t bits = 0u;
    for (int g = 0; g < G; ++g)
      bits |= (p.mask[(head0 + g) * p.NT + t0 + tid] ? 1u : 0u) << g;
    ms.sel[tid] = bits;
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
      int u = 0, u16 = 0;
      bool ok = true;
      // Ring fills in the order the MMA issuer consumes them: K4 of every
      // tile, then V4 of every tile; the fp16 slot takes K16 of the FP16
      // tiles, then their V16 between the V4 fills.
      auto fill4 = [&](bool is_v, int tile) -> bool {
        const int slot = u % kDRing, use = u / kDRing;
        if (use > 0 && !wait_or_abort(&ms.bar_empty[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        uint8_t* st = sm + DSmem::kRing + slot * DSmem::kSlotBytes;
        mbar_arrive_expect_tx(&ms.bar_full[slot], DSmem::kSlotBytes);
        if (!is_v) {
          tma_load_3d(st, &mK4, &ms.bar_full[slot], 0, tile * 128, bhk);
          bulk_load(st + 8192, p.ks + (static_cast<size_t>(bhk) * p.NT + tile) * 1024, 1024, &ms.bar_full[slot]);
        } else {
          tma_load_3d(st, &mV4, &ms.bar_full[slot], tile * 64, 0, bhk);
          bulk_load(st + 8192, p.vs + (static_cast<size_t>(bhk) * 2 * p.NT + 2 * tile) * 512, 1024,
                    &ms.bar_full[slot]);
        }
        ++u;
        return true;
      };
      auto fill16 = [&](const CUtensorMap* map, int tile) -> bool {
        if (u16 > 0 && !wait_or_abort(&ms.bar_empty16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
          return false;
        mbar_arrive_expect_tx(&ms.bar_full16, 32768);
        for (int pnl = 0; pnl < 2; ++pnl)
          tma_load_3d(sm + DSmem::kS16 + pnl * 16384, map, &ms.bar_full16, pnl * 64, tile * 128, bhk);
        ++u16;
        return true;
      };
      for (int i = 0; ok && i < nt; ++i) ok = fill4(false, t0 + i);
      for (int i = 0; ok && i < nt; ++i)
        if (ms.sel[i]) ok = fill16(&mK16, t0 + i);
      for (int i = 0; ok && i < nt; ++i) {
        ok = fill4(true, t0 + i);
        if (ok && ms.sel[i]) ok = fill16(&mV16, t0 + i);
      }
      // Let every copy this thread issued land before the CTA can exit.
      for (int s = 0; s < kDRing; ++s)
        if (u > s) mbar_wait(&ms.bar_full[s], ((u - 1 - s) / kDRing) & 1, kWaitNs);
      if (u16 > 0) mbar_wait(&ms.bar_full16, (u16 - 1) & 1, kWaitNs);
    }
    __syncwarp();
  } else if (warp == kDMma) {
    // ======================== MMA issuer ========================
    if (lane == 0) {
      constexpr uint32_t idS4 = idesc_nvf4(128, kDHeads);
      constexpr uint32_t idS16 = idesc_f16(128, kDHeads, false);
      constexpr uint32_t idO16 = idesc_f16_mn(128, kDHeads, true, false);
      bool ok = wait_or_abort(&ms.bar_q, 0, &ms.abort, p.err, DEV_TIMEOUT_OTHER);
      tc_fence_after();
      if (ok)
        for (int c = 0; c < 2; ++c)
          tmem_cp_32x128b_x4(tm + kCSFQ + 4 * c, make_sdesc(sbase + DSmem::kQSF + 512 * c, 16, 128, LAYOUT_NONE));
      int u = 0, u16 = 0;
      // ---- pass 1: S^T of every tile (NVFP4), then fp16 S^T of the FP16 tiles ----
      for (int i = 0; ok && i < nt; ++i) {
        const int slot = u % kDRing;
        if (!(ok = wait_or_abort(&ms.bar_full[slot], (u / kDRing) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
        ++u;
        tc_fence_after();
        const uint32_t st = sbase + DSmem::kRing + slot * DSmem::kSlotBytes;
        for (int c = 0; c < 2; ++c)
          tmem_cp_32x128b_x4(tm + kCSFK + 4 * c, make_sdesc(st + 8192 + 512 * c, 16, 128, LAYOUT_NONE));
#pragma unroll
        for (int c = 0; c < 2; ++c)
          mma_nvf4(tm + kCS + 32 * i, make_sdesc(st + 32 * c, 16, 512, LAYOUT_SW64),
                   make_sdesc(sbase + DSmem::kQ4 + 32 * c, 16, 512, LAYOUT_SW64), idS4, tm + kCSFK + 4 * c,
                   tm + kCSFQ + 4 * c, c > 0);
        mma_commit(&ms.bar_empty[slot]);
      }
      for (int i = 0; ok && i < nt; ++i) {
        if (!ms.sel[i]) continue;
        if (!(ok = wait_or_abort(&ms.bar_full16, u16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
        ++u16;
        tc_fence_after();
        const uint32_t k16 = sbase + DSmem::kS16, q16 = sbase + DSmem::kQ16;
#pragma unroll
        for (int k = 0; k < kDD / 16; ++k)
          mma_f16(tm + kCS + 32 * i + 16, make_sdesc(k16 + (k / 4) * 16384 + (k % 4) * 32, 16, 1024, LAYOUT_SW128),
                  make_sdesc(q16 + (k / 4) * 2048 + (k % 4) * 32, 16, 1024, LAYOUT_SW128), idS16, k > 0);
        mma_commit(&ms.bar_empty16);
      }
      if (ok) mma_commit(&ms.bar_s);
      // ---- pass 2: O^T += V^T P^T per tile ----
      for (int i = 0; ok && i < nt; ++i) {
        const int pb = i & 1;
        const int slot = u % kDRing;
        if (!(ok = wait_or_abort(&ms.bar_full[slot], (u / kDRing) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
        ++u;
        tc_fence_after();
        const uint32_t st = sbase + DSmem::kRing + slot * DSmem::kSlotBytes;
        // The copies follow the previous tile's products in this thread's
        // tcgen05 order, so they cannot overwrite scales those still read.
        for (int c = 0; c < 2; ++c)
          tmem_cp_32x128b_x4(tm + kCSFV + 4 * c, make_sdesc(st + 8192 + 512 * c, 16, 128, LAYOUT_NONE));
        if (!(ok = wait_or_abort(&ms.bar_p[pb], (i >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))) break;
        tc_fence_after();
        const uint32_t p4 = sbase + DSmem::kP4 + pb * 1024, psf = sbase + DSmem::kPSF + pb * 1024;
        for (int c = 0; c < 2; ++c)
          tmem_cp_32x128b_x4(tm + kCSFP + 4 * c, make_sdesc(psf + 512 * c, 16, 128, LAYOUT_NONE));
#pragma unroll
        for (int c = 0; c < 2; ++c)
          mma_nvf4(tm + kCO, make_sdesc(st + 32 * c, 16, 512, LAYOUT_SW64), make_sdesc(p4 + 32 * c, 16, 512, LAYOUT_SW64),
                   idS4, tm + kCSFV + 4 * c, tm + kCSFP + 4 * c, (i > 0 || c > 0) ? 1u : 0u);
        if (ms.sel[i]) {
          if (!(ok = wait_or_abort(&ms.bar_full16, u16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
          ++u16;
          tc_fence_after();
          const uint32_t v16 = sbase + DSmem::kS16, p16 = sbase + DSmem::kP16 + pb * 4096;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_f16(tm + kCO, make_sdesc(v16 + k * 2048, 16384, 1024, LAYOUT_SW128),
                    make_sdesc(p16 + (k / 4) * 2048 + (k % 4) * 32, 16, 1024, LAYOUT_SW128), idO16, 1u);
          mma_commit(&ms.bar_empty16);
        }
        mma_commit(&ms.bar_empty[slot]);
        mma_commit(&ms.bar_pv[pb]);
      }
      if (ok) mma_commit(&ms.bar_o);
      // drain: every tensor-core operation this thread issued completes before exit
      mma_commit(&ms.bar_drain);
      mbar_wait(&ms.bar_drain, 0, kWaitNs);
    }
    __syncwarp();
  } else {
    // ============ softmax threads: lane = key of a tile, then channel ============
    const int t = tid;
    const float c2 = p.c2;
    const uint32_t lane_base = tm + (static_cast<uint32_t>(warp * 32) << 16);
    bool failed = false;

    // Query rows: thread t stages 16-element group j = t % 8 of head row g = t / 8
    // as fp16 (SW128) and as NVFP4 (SW64 codes, scale chunk bytes g * 16 + j % 4).
    {
      const int g = t / 8, j = t % 8;
      uint4 a = make_uint4(0u, 0u, 0u, 0u), c = make_uint4(0u, 0u, 0u, 0u);
      if (g < G) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q + (head0 + g) * kDD + 16 * j);
        a = src[0];
        c = src[1];
      }
      uint8_t* q16 = sm + DSmem::kQ16 + (j / 4) * 2048;
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
      *reinterpret_cast<uint2*>(sm + DSmem::kQ4 + sw64_off(g, j / 2) + 8 * (j % 2)) = make_uint2(e.lo, e.hi);
      sm[DSmem::kQSF + (j / 4) * 512 + g * 16 + (j % 4)] = static_cast<uint8_t>(e.scale);
      // rows 16-31 of both scale chunks (never read with N = 16) are zeroed
      *reinterpret_cast<uint32_t*>(sm + DSmem::kQSF + (t / 64) * 512 + 256 + (t % 64) * 4) = 0u;
      fence_proxy_async_smem();
      mbar_arrive(&ms.bar_q);
    }

    // ---- pass 1: maximum of S per head over the chunk ----
    float mx[kDHeads];
#pragma unroll
    for (int g = 0; g < kDHeads; ++g) mx[g] = -INFINITY;
    failed = !wait_or_abort(&ms.bar_s, 0, &ms.abort, p.err, DEV_TIMEOUT_MMA);
    failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
    if (!failed) {
      tc_fence_after();
      for (int i = 0; i < nt; ++i) {
        const uint32_t sel = ms.sel[i];
        uint32_t s4[16], s16[16];
        tmem_ld16(lane_base + kCS + 32 * i, s4);
        if (sel) tmem_ld16(lane_base + kCS + 32 * i + 16, s16);
        tmem_ld_wait();
        tmem_ld_fence(s4);
        tmem_ld_fence(s16);
#pragma unroll
        for (int g = 0; g < kDHeads; ++g)
          if (g < G) mx[g] = fmaxf(mx[g], __uint_as_float(((sel >> g) & 1u) ? s16[g] : s4[g]));
      }
    }
#pragma unroll
    for (int g = 0; g < kDHeads; ++g) {
      if (g < G) {
        float m = mx[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) ms.red[warp][g] = m;
      }
    }
    failed = softmax_bar_or<kDSoftmax>(failed);
    // base_g = 11 - M_g with M_g = ceil(max t) = ceil(fl32(max S * c2))
    float base[kDHeads];
#pragma unroll
    for (int g = 0; g < kDHeads; ++g) {
      base[g] = 0.f;
      if (g < G) {
        const float smax = fmaxf(fmaxf(ms.red[0][g], ms.red[1][g]), fmaxf(ms.red[2][g], ms.red[3][g]));
        base[g] = static_cast<float>(kPLog2) - ceilf(smax * c2);
      }
    }

    // ---- pass 2: P per head, encoded, into buffer i % 2 ----
    float lsum[kDHeads];
#pragma unroll
    for (int g = 0; g < kDHeads; ++g) lsum[g] = 0.f;
    for (int i = 0; i < nt && !failed; ++i) {
      const int pb = i & 1;
      if (i >= 2) failed = !wait_or_abort(&ms.bar_pv[pb], ((i - 2) >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      failed = __any_sync(0xffffffffu, failed);
      if (failed) break;
      tc_fence_after();
      const uint32_t sel = ms.sel[i];
      uint32_t s4[16], s16[16];
      tmem_ld16(lane_base + kCS + 32 * i, s4);
      if (sel) tmem_ld16(lane_base + kCS + 32 * i + 16, s16);
      tmem_ld_wait();
      tmem_ld_fence(s4);
      tmem_ld_fence(s16);
      uint8_t* p4 = sm + DSmem::kP4 + pb * 1024;
      uint8_t* psf = sm + DSmem::kPSF + pb * 1024;
      uint8_t* p16 = sm + DSmem::kP16 + pb * 4096;
#pragma unroll
      for (int g = 0; g < kDHeads; ++g) {
        if (g >= G) continue;
        const bool h16 = (sel >> g) & 1u;  // the same in every thread
        uint32_t code = 0u, sbyte = 0u;
        float x16 = 0.f;
        if (h16) {
          const float x = ex2(fmaf(__uint_as_float(s16[g]), c2, base[g]));  // P * 2^11
          lsum[g] += x;
          x16 = x;
        } else {
          const float s = __uint_as_float(s4[g]);
          float gm = s;  // maximum over this 16-key group (16 consecutive lanes)
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
          const float amax = ex2(fmaf(gm, c2, base[g]));  // max of P * 2^11 in the group
          sbyte = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.f) & 0xFFu;
          const float sc0 = e4m3_to_f32(sbyte);
          const float sc = sc0 > 0.f ? sc0 : 1.0f;  // zero scale: the code rounds to 0, l keeps P
          const float x = ex2(fmaf(s, c2, base[g] - lg2(sc)));  // P * 2^11 / scale
          lsum[g] = fmaf(x, sc, lsum[g]);
          code = cvt_e2m1x2(x, 0.f) & 0xFu;
        }
        // codes of keys 8m .. 8m + 7 in one word: key t at byte t / 2 of row g
        uint32_t w = code << (4 * (lane & 7));
        w |= __shfl_xor_sync(0xffffffffu, w, 1);
        w |= __shfl_xor_sync(0xffffffffu, w, 2);
        w |= __shfl_xor_sync(0xffffffffu, w, 4);
        if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(p4 + sw64_off(g, warp) + (lane >> 1)) = w;
        if ((lane & 15) == 0) psf[(t / 64) * 512 + g * 16 + (t % 64) / 16] = static_cast<uint8_t>(sbyte);
        if (sel)
          *reinterpret_cast<__half*>(p16 + (t / 64) * 2048 + sw128_off(g, (t % 64) / 8) + (t % 8) * 2) =
              __float2half_rn(x16);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ms.bar_p[pb]);
    }

    // ---- epilogue: the chunk's O^T column g, l_g and M_g ----
    if (!failed) failed = !wait_or_abort(&ms.bar_o, 0, &ms.abort, p.err, DEV_TIMEOUT_MMA);
#pragma unroll
    for (int g = 0; g < kDHeads; ++g) {
      if (g < G) {
        float l = lsum[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) ms.lred[warp][g] = l;
      }
    }
    failed = softmax_bar_or<kDSoftmax>(failed);
    if (!failed) {
      tc_fence_after();
      uint32_t o[16];
      tmem_ld16(lane_base + kCO, o);
      tmem_ld_wait();
      tmem_ld_fence(o);
#pragma unroll
      for (int g = 0; g < kDHeads; ++g)
        if (g < G) p.part_o[((head0 + g) * p.chunks + chunk) * kDD + t] = __uint_as_float(o[g]);
      if (t < G) {
        const size_t idx = (head0 + t) * p.chunks + chunk;
        p.part_l[idx] = (ms.lred[0][t] + ms.lred[1][t]) + (ms.lred[2][t] + ms.lred[3][t]);
        const float smax = fmaxf(fmaxf(ms.red[0][t], ms.red[1][t]), fmaxf(ms.red[2][t], ms.red[3][t]));
        p.part_m[idx] = ceilf(smax * c2);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDMma) {
    tc_fence_after();
    tmem_dealloc(tm, kDTmemCols);
  }
}

// O = sum_c 2^(M_c - M) O_c / sum_c 2^(M_c - M) l_c; both carry the 2^11 pre-scale.
__global__ void __launch_bounds__(kDD) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_l,
                                                             const float* __restrict__ part_m, int chunks,
                                                             __half* __restrict__ O) {
  const size_t bh = blockIdx.x;
  const int d = threadIdx.x;
  const float* pm = part_m + bh * chunks;
  const float* pl = part_l + bh * chunks;
  const float* po = part_o + bh * chunks * kDD;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, pm[c]);
  float L = 0.f, acc = 0.f;
  for (int c = 0; c < chunks; ++c) {
    const float w = exp2_int(pm[c] - M);
    L = fmaf(w, pl[c], L);
    acc = fmaf(w, po[static_cast<size_t>(c) * kDD + d], acc);
  }
  O[bh * kDD + d] = __float2half_rn(acc / L);
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
// FP32 means are exact in FP64; the FP64 sum is rounded once.
__global__ void __launch_bounds__(256) decode_select_kernel(const __half* __restrict__ q,
                                                            const float* __restrict__ km, int Hq, int Hkv, int nb,
                                                            float sm_scale, long long k, uint8_t* __restrict__ mask) {
  __shared__ float sq[kDD];
  __shared__ unsigned long long keys[1024];
  const size_t bh = blockIdx.x;
  const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
  const int G = Hq / Hkv;
  const float* kmh = km + (static_cast<size_t>(b) * Hkv + h / G) * nb * static_cast<size_t>(kDD);
  for (int d = threadIdx.x; d < kDD; d += blockDim.x) sq[d] = __half2float(q[bh * kDD + d]);
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const float* kr = kmh + static_cast<size_t>(j) * kDD;
    double dot = 0.0;
    for (int d = 0; d < kDD; ++d) dot = fma(static_cast<double>(sq[d]), static_cast<double>(kr[d]), dot);
    const float sc = static_cast<float>(static_cast<double>(sm_scale) * static_cast<double>(static_cast<float>(dot)));
    keys[j] = decode_key(sc, j, nb);
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

DecodePlan decode_plan(const thrift_shape& s) {
  const int NT = num_tiles(s.N);
  const int units = s.B * s.Hkv;
  constexpr int kMaxTiles = 6;
  // about two CTAs per SM over the whole grid, at most kMaxTiles key tiles each
  const int target = (2 * 148 + units - 1) / units;
  int chunks = target < 1 ? 1 : target;
  const int min_chunks = (NT + kMaxTiles - 1) / kMaxTiles;
  if (chunks < min_chunks) chunks = min_chunks;
  if (chunks > NT) chunks = NT;
  DecodePlan pl;
  pl.tiles_per_cta = (NT + chunks - 1) / chunks;
  pl.chunks = (NT + pl.tiles_per_cta - 1) / pl.tiles_per_cta;
  return pl;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t decode_workspace_bytes(const thrift_shape& s) {
  const DecodePlan pl = decode_plan(s);
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * pl.chunks;
  return align256(static_cast<size_t>(s.B) * s.Hq * num_tiles(s.N)) + align256(rows * kDD * sizeof(float)) +
         2 * align256(rows * sizeof(float));
}

DecodeWs decode_carve(void* ws, const thrift_shape& s) {
  const DecodePlan pl = decode_plan(s);
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * pl.chunks;
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
  decode_select_kernel<<<s.B * s.Hq, 256, 0, st>>>(static_cast<const __half*>(q), km, s.Hq, s.Hkv, nb, s.sm_scale,
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
  prm.G = s.Hq / s.Hkv;
  prm.tiles_per_cta = pl.tiles_per_cta;
  prm.chunks = pl.chunks;
  prm.c2 = static_cast<float>(static_cast<double>(s.sm_scale) * 1.4426950408889634073599246810019);
  const size_t smem = DSmem::kBytes + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(thrift_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  thrift_decode_kernel<<<dim3(pl.chunks, static_cast<unsigned>(BHk)), kDThreads, smem, st>>>(mK16, mV16, mK4, mV4,
                                                                                             prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<s.B * s.Hq, kDD, 0, st>>>(w.part_o, w.part_l, w.part_m, pl.chunks,
                                                    static_cast<__half*>(O));
  return cudaGetLastError();
}

}  // namespace thrift

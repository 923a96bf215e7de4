// Stage 2 of the method for 128 x 128 selection blocks ("the selected blocks
// are computed in FP16 and the remaining blocks in FP4, with both paths merged
// via online softmax into a single output", ThriftAttention abstract), as a
// ping-pong of two query tiles per CTA.
//
// A CTA owns query tiles A = 2j and B = 2j+1 of one (batch, query head); each
// has its own softmax warpgroup (one thread per row, the whole 128-key row in
// registers) and its own O accumulator in tensor memory.  The two tiles take
// turns on one S buffer: while one warpgroup exponentiates and encodes its P,
// the tensor cores compute the other tile's S, so the two warpgroups on each
// SM sub-partition work out of phase and no thread ever waits for another
// thread of its row.  K/V tiles are loaded once for both query tiles.
//
// Per key tile and query tile (same arithmetic as the single-tile kernel):
//   S from the fp16 operands (.kind::f16) or the NVFP4 copies
//   (.kind::mxf4nvf4), t = S * sm_scale * log2 e, integer running maximum
//   M = ceil(max t) (rescales of O are exact powers of two), P * 2^11 encoded
//   as fp16 (written to tensor memory, the A operand of a .kind::f16 product)
//   or as NVFP4 per 16 keys (codes in shared memory, scales stored by each
//   row's thread straight into tensor memory), and O += P~ V~; finally O / l.
//
// Warp roles (352 threads): warps 0-3 softmax of tile A, 4-7 softmax of tile
// B, 8 TMA producer, 9 issues the S products (and owns tensor memory), 10
// issues the P V products.  Two issuing threads on different SM
// sub-partitions keep the S of one tile from queueing behind the P V of the
// other; they meet only through mbarriers.
#include <cuda_fp16.h>

#include "attention_common.cuh"
#include "common.h"
#include "ptx.cuh"
#include "tmap.h"

namespace thrift {
namespace {
using namespace attn;

constexpr int kPPThreads = 352;
constexpr int kPPProducer = 8;
constexpr int kPPMmaS = 9;   // issues the S products; owns tensor memory
constexpr int kPPMmaPV = 10;  // issues the P V products

// Tensor-memory columns (512 allocated).
constexpr uint32_t kPColS = 0;       // shared S buffer, 128 columns
constexpr uint32_t kPColO = 128;     // O of tile x at 128 + 128 * x, D columns
constexpr uint32_t kPColP16 = 384;   // fp16 P of either tile, 64 columns (used in issue order)
constexpr uint32_t kPColSFQ = 448;   // Q4 scales, 8 columns per tile
constexpr uint32_t kPColSFK = 464;   // K4 scales of the current key tile
constexpr uint32_t kPColSFV = 472;   // V4 scales of the key tile being multiplied
constexpr uint32_t kPColSFP = 480;   // P4 scales, 8 columns per tile: chunk c of row r at 4c + r / 32

template <int D>
struct SmemPP {
  static constexpr uint32_t kQ16Bytes = 128 * D * 2;  // per tile
  static constexpr uint32_t kQ16 = 0;
  static constexpr uint32_t kQ4Bytes = 128 * D / 2;
  static constexpr uint32_t kQ4 = 2 * kQ16Bytes;
  static constexpr uint32_t kQSFBytes = (D / 64) * 512;
  static constexpr uint32_t kQSF = kQ4 + 2 * kQ4Bytes;
  static constexpr uint32_t kP4 = (kQSF + 2 * kQSFBytes + 1023) / 1024 * 1024;  // 8 KB per tile
  static constexpr uint32_t kK4Bytes = 128 * D / 2;
  static constexpr uint32_t kV4Bytes = D * 64;
  static constexpr uint32_t kKSFBytes = (D / 64) * 512;
  static constexpr uint32_t kVSFBytes = 1024;
  static constexpr uint32_t kSlot4Bytes = (kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kSlot4 = kP4 + 2 * 8192;
  static constexpr int kNS = (D == 128) ? 3 : 4;  // NVFP4 K/V ring slots
  static constexpr uint32_t kK16Bytes = 128 * D * 2;
  static constexpr uint32_t kSlot16 = kSlot4 + kNS * kSlot4Bytes;  // K16 then V16
  static constexpr uint32_t kMisc = kSlot16 + 2 * kK16Bytes;
  static constexpr uint32_t kBytes = kMisc + 4096;
  static constexpr uint32_t kTx4 = kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes;
  static constexpr uint32_t kTx16 = kK16Bytes;
  static constexpr uint32_t kTxQ = kQ16Bytes + kQ4Bytes + kQSFBytes;  // per tile
  static_assert(kBytes + 1024 <= 232448, "shared memory above the 227 KB per-CTA limit");
};

struct MiscPP {
  uint64_t bar_q;
  uint64_t bar_full4[4], bar_empty4[4];
  uint64_t bar_full_k16, bar_empty_k16, bar_full_v16, bar_empty_v16;
  uint64_t bar_s_full[2];  // per tile: one phase per S product of that tile
  uint64_t bar_s_free;     // the shared S buffer: one phase per S product (read by its warpgroup)
  uint64_t bar_p_full[2];  // per tile: P of the tile's current key tile written
  uint64_t bar_o_done[2];  // per tile: one phase per P V product of that tile
  uint64_t bar_p16_free;   // one phase per fp16 P V product, in issue order
  uint64_t bar_drain[2];   // one per issuing thread
  uint32_t tmem;
  volatile int abort;
  uint8_t cls[2][1024];  // per tile and key tile: 1 = FP16, 0 = NVFP4
};
static_assert(sizeof(MiscPP) <= 4096, "barriers must fit their shared-memory slice");

template <int D>
__global__ void __launch_bounds__(kPPThreads, 1)
    thrift_attention_pp_kernel(const __grid_constant__ CUtensorMap mQ16, const __grid_constant__ CUtensorMap mK16,
                               const __grid_constant__ CUtensorMap mV16, const __grid_constant__ CUtensorMap mQ4,
                               const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                               const Params p) {
  using L = SmemPP<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  MiscPP& ms = *reinterpret_cast<MiscPP*>(sm + L::kMisc);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int BH = p.B * p.Hq;
  const int NP = (p.NT + 1) / 2;
  const int pair = NP - 1 - static_cast<int>(blockIdx.x) / BH;  // longest causal rows first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int qt0 = 2 * pair, qt1 = 2 * pair + 1;
  const bool hasB = qt1 < p.NT;
  const int n0 = p.causal ? qt0 + 1 : p.NT;
  const int n1 = !hasB ? 0 : (p.causal ? qt1 + 1 : p.NT);
  const int nmax = n0 > n1 ? n0 : n1;
  const int nb = p.NT;  // blk = 128

  if (warp == kPPMmaS) {
    tmem_alloc(&ms.tmem, 512);
    tmem_relinquish();
  }
  if (tid == kPPProducer * 32) {
    mbar_init(&ms.bar_q, 1);
    for (int i = 0; i < L::kNS; ++i) {
      mbar_init(&ms.bar_full4[i], 1);
      mbar_init(&ms.bar_empty4[i], 2);  // K4 read by the S issuer, V4 by the P V issuer
    }
    mbar_init(&ms.bar_full_k16, 1);
    mbar_init(&ms.bar_empty_k16, 1);
    mbar_init(&ms.bar_full_v16, 1);
    mbar_init(&ms.bar_empty_v16, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms.bar_s_full[i], 1);
      mbar_init(&ms.bar_p_full[i], 128);
      mbar_init(&ms.bar_o_done[i], 1);
    }
    mbar_init(&ms.bar_s_free, 128);
    mbar_init(&ms.bar_p16_free, 1);
    mbar_init(&ms.bar_drain[0], 1);
    mbar_init(&ms.bar_drain[1], 1);
    ms.abort = 0;
    fence_mbar_init();
  }
  {
    const uint8_t* m0 = p.mask + static_cast<size_t>(bh) * nb * nb + static_cast<size_t>(qt0) * nb;
    for (int kt = tid; kt < n0; kt += kPPThreads) ms.cls[0][kt] = m0[kt] ? 1 : 0;
    if (hasB) {
      const uint8_t* m1 = m0 + nb;
      for (int kt = tid; kt < n1; kt += kPPThreads) ms.cls[1][kt] = m1[kt] ? 1 : 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem;

  // Which operand kinds key tile kt needs (for either query tile).
  auto need4 = [&](int kt) {
    return (kt < n0 && ms.cls[0][kt] == 0) || (kt < n1 && ms.cls[1][kt] == 0);
  };
  auto need16 = [&](int kt) { return (kt < n0 && ms.cls[0][kt] != 0) || (kt < n1 && ms.cls[1][kt] != 0); };

  if (warp == kPPProducer) {
    // ======================== producer ========================
    if (lane == 0) {
      prefetch_tensormap(&mQ16);
      prefetch_tensormap(&mK4);
      prefetch_tensormap(&mV4);
      const int ntiles = hasB ? 2 : 1;
      mbar_arrive_expect_tx(&ms.bar_q, L::kTxQ * ntiles);
      for (int x = 0; x < ntiles; ++x) {
        const int qt = qt0 + x;
        for (int pnl = 0; pnl < D / 64; ++pnl)
          tma_load_3d(sm + L::kQ16 + x * L::kQ16Bytes + pnl * 16384, &mQ16, &ms.bar_q, pnl * 64, qt * 128, bh);
        tma_load_3d(sm + L::kQ4 + x * L::kQ4Bytes, &mQ4, &ms.bar_q, 0, qt * 128, bh);
        bulk_load(sm + L::kQSF + x * L::kQSFBytes, p.qs + (static_cast<size_t>(bh) * p.NT + qt) * L::kQSFBytes,
                  L::kQSFBytes, &ms.bar_q);
      }
      int u4 = 0, u16 = 0;
      for (int kt = 0; kt < nmax && !ms.abort; ++kt) {
        if (need4(kt)) {
          const int slot = u4 % L::kNS, use = u4 / L::kNS;
          if (use > 0 && !wait_or_abort(&ms.bar_empty4[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
            break;
          uint8_t* st = sm + L::kSlot4 + slot * L::kSlot4Bytes;
          mbar_arrive_expect_tx(&ms.bar_full4[slot], L::kTx4);
          tma_load_3d(st, &mK4, &ms.bar_full4[slot], 0, kt * 128, bhk);
          tma_load_3d(st + L::kK4Bytes, &mV4, &ms.bar_full4[slot], kt * 64, 0, bhk);
          bulk_load(st + L::kK4Bytes + L::kV4Bytes, p.ks + (static_cast<size_t>(bhk) * p.NT + kt) * L::kKSFBytes,
                    L::kKSFBytes, &ms.bar_full4[slot]);
          bulk_load(st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes,
                    p.vs + (static_cast<size_t>(bhk) * 2 * p.NT + 2 * kt) * 512, L::kVSFBytes, &ms.bar_full4[slot]);
          ++u4;
        }
        if (need16(kt)) {
          uint8_t* st = sm + L::kSlot16;
          if (u16 > 0 && !wait_or_abort(&ms.bar_empty_k16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))
            break;
          mbar_arrive_expect_tx(&ms.bar_full_k16, L::kTx16);
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(st + pnl * 16384, &mK16, &ms.bar_full_k16, pnl * 64, kt * 128, bhk);
          if (u16 > 0 && !wait_or_abort(&ms.bar_empty_v16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER)) {
            ++u16;  // the K16 copy of this tile is in flight
            mbar_wait(&ms.bar_full_k16, (u16 - 1) & 1, kWaitNs);
            --u16;
            break;
          }
          mbar_arrive_expect_tx(&ms.bar_full_v16, L::kTx16);
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(st + L::kK16Bytes + pnl * 16384, &mV16, &ms.bar_full_v16, pnl * 64, kt * 128, bhk);
          ++u16;
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      mbar_wait(&ms.bar_q, 0, kWaitNs);
      for (int s = 0; s < L::kNS; ++s)
        if (u4 > s) mbar_wait(&ms.bar_full4[s], ((u4 - 1 - s) / L::kNS) & 1, kWaitNs);
      if (u16 > 0) {
        mbar_wait(&ms.bar_full_k16, (u16 - 1) & 1, kWaitNs);
        mbar_wait(&ms.bar_full_v16, (u16 - 1) & 1, kWaitNs);
      }
    }
    __syncwarp();
  } else if (warp == kPPMmaS) {
    // ================= S issuer: K scales, then S of tile A and tile B =================
    // The two tiles take turns on the S buffer; each S waits until the
    // previous one has been loaded into registers by its warpgroup.
    if (lane == 0) {
      constexpr uint32_t sbo4 = (D == 128) ? 512u : 256u;
      constexpr uint32_t sw4 = (D == 128) ? LAYOUT_SW64 : LAYOUT_SW32;
      bool ok = wait_or_abort(&ms.bar_q, 0, &ms.abort, p.err, DEV_TIMEOUT_LOAD);
      tc_fence_after();
      if (ok)
        for (int x = 0; x < (hasB ? 2 : 1); ++x)
          for (int c = 0; c < D / 64; ++c)
            tmem_cp_32x128b_x4(tm + kPColSFQ + 8 * x + 4 * c,
                               make_sdesc(sbase + L::kQSF + x * L::kQSFBytes + 512 * c, 16, 128, LAYOUT_NONE));
      int u4 = 0, uk16 = 0, seq = 0;
      for (int kt = 0; ok && kt < nmax; ++kt) {
        const bool t4 = need4(kt), t16 = need16(kt);
        int slot = 0;
        if (t4) {
          slot = u4 % L::kNS;
          if (!(ok = wait_or_abort(&ms.bar_full4[slot], (u4 / L::kNS) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
          ++u4;
          tc_fence_after();
          const uint32_t ksf = sbase + L::kSlot4 + slot * L::kSlot4Bytes + L::kK4Bytes + L::kV4Bytes;
          for (int c = 0; c < D / 64; ++c)
            tmem_cp_32x128b_x4(tm + kPColSFK + 4 * c, make_sdesc(ksf + 512 * c, 16, 128, LAYOUT_NONE));
        }
        if (t16) {
          if (!(ok = wait_or_abort(&ms.bar_full_k16, uk16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
          ++uk16;
          tc_fence_after();
        }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (kt < (x == 0 ? n0 : n1)) {
            if (seq > 0 && !(ok = wait_or_abort(&ms.bar_s_free, (seq - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER)))
              break;
            tc_fence_after();
            if (ms.cls[x][kt] == 0) {
              const uint32_t q4 = sbase + L::kQ4 + x * L::kQ4Bytes;
              const uint32_t k4 = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
#pragma unroll
              for (int c = 0; c < D / 64; ++c)
                mma_nvf4(tm + kPColS, make_sdesc(q4 + 32 * c, 16, sbo4, sw4), make_sdesc(k4 + 32 * c, 16, sbo4, sw4),
                         idesc_nvf4(128, 128), tm + kPColSFQ + 8 * x + 4 * c, tm + kPColSFK + 4 * c, c > 0);
            } else {
              const uint32_t q16 = sbase + L::kQ16 + x * L::kQ16Bytes, k16 = sbase + L::kSlot16;
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t off = (k / 4) * 16384 + (k % 4) * 32;
                mma_f16(tm + kPColS, make_sdesc(q16 + off, 16, 1024, LAYOUT_SW128),
                        make_sdesc(k16 + off, 16, 1024, LAYOUT_SW128), idesc_f16(128, 128, false), k > 0);
              }
            }
            mma_commit(&ms.bar_s_full[x]);
            ++seq;
          }
        }
        if (!ok) break;
        // K operands of this key tile are no longer needed (V: the P V issuer)
        if (t4) mma_commit(&ms.bar_empty4[slot]);
        if (t16) mma_commit(&ms.bar_empty_k16);
      }
      // drain: every tensor-core operation this thread issued completes before exit
      mma_commit(&ms.bar_drain[0]);
      mbar_wait(&ms.bar_drain[0], 0, kWaitNs);
    }
    __syncwarp();
  } else if (warp == kPPMmaPV) {
    // ================= P V issuer: O_x += P_x V for tile A, then tile B =================
    if (lane == 0) {
      bool ok = true;
      int u4 = 0, uv16 = 0;
      uint32_t acc0 = 0u, acc1 = 0u;
      for (int kt = 0; ok && kt < nmax; ++kt) {
        const bool t4 = need4(kt), t16 = need16(kt);
        const int slot = u4 % L::kNS, use = u4 / L::kNS;
        if (t4) ++u4;
        bool v4_ready = false, v16_ready = false;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (kt < (x == 0 ? n0 : n1)) {
            if (!(ok = wait_or_abort(&ms.bar_p_full[x], kt & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER))) break;
            tc_fence_after();
            const uint32_t dO = tm + kPColO + 128 * x;
            uint32_t& acc = x == 0 ? acc0 : acc1;
            if (ms.cls[x][kt] == 0) {
              const uint32_t st = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
              const uint32_t v4 = st + L::kK4Bytes, vsf = st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes;
              if (!v4_ready) {
                // V4 landed with K4 (one barrier phase); wait on it here too so
                // that this thread observes the copy itself.  The producer cannot
                // refill the slot before this thread releases it.
                if (!(ok = wait_or_abort(&ms.bar_full4[slot], use & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
                tc_fence_after();
                for (int c = 0; c < 2; ++c)
                  tmem_cp_32x128b_x4(tm + kPColSFV + 4 * c, make_sdesc(vsf + 512 * c, 16, 128, LAYOUT_NONE));
                v4_ready = true;
              }
              const uint32_t p4s = sbase + L::kP4 + x * 8192;
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                mma_nvf4(dO, make_sdesc(p4s + 32 * c, 16, 512, LAYOUT_SW64),
                         make_sdesc(v4 + 32 * c, 16, 512, LAYOUT_SW64), idesc_nvf4(128, D),
                         tm + kPColSFP + 8 * x + 4 * c, tm + kPColSFV + 4 * c, acc);
                acc = 1;
              }
            } else {
              if (!v16_ready) {
                if (!(ok = wait_or_abort(&ms.bar_full_v16, uv16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD))) break;
                ++uv16;
                v16_ready = true;
                tc_fence_after();
              }
              const uint32_t v16 = sbase + L::kSlot16 + L::kK16Bytes;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                mma_f16_ts(dO, tm + kPColP16 + 8 * k, make_sdesc(v16 + k * 2048, 16384, 1024, LAYOUT_SW128),
                           idesc_f16(128, D, true), acc);
                acc = 1;
              }
              mma_commit(&ms.bar_p16_free);
            }
            mma_commit(&ms.bar_o_done[x]);
          }
        }
        if (!ok) break;
        if (t4) mma_commit(&ms.bar_empty4[slot]);
        if (t16) mma_commit(&ms.bar_empty_v16);
      }
      mma_commit(&ms.bar_drain[1]);
      mbar_wait(&ms.bar_drain[1], 0, kWaitNs);
    }
    __syncwarp();
  } else {
    // ======================== softmax (one thread per row) ========================
    const int x = warp / 4;  // query tile
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const int qt = qt0 + x;
    const int qrow = qt * 128 + r;
    const int nx = x == 0 ? n0 : n1;
    const uint32_t lane_base = tm + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t ocol = lane_base + kPColO + 128 * x;
    const float c2 = p.scale_log2;
    float M = -INFINITY, l = 0.f;
    bool failed = false;
    int before16 = 0;  // fp16 P V products issued before key tile kt (both tiles, issue order)
    for (int kt = 0; kt < nx; ++kt) {
      const bool fp16 = ms.cls[x][kt] != 0;
      const int my16 = before16 + ((x == 1 && kt < n0 && ms.cls[0][kt] != 0) ? 1 : 0);
      before16 += ((kt < n0 && ms.cls[0][kt] != 0) ? 1 : 0) + ((kt < n1 && ms.cls[1][kt] != 0) ? 1 : 0);
      if (!failed) failed = !wait_or_abort(&ms.bar_s_full[x], kt & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
      if (failed) continue;
      tc_fence_after();
      float s[128];
      {
        uint32_t v[128];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tmem_ld32(lane_base + kPColS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * q]));
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 128; ++j) s[j] = __uint_as_float(v[j]);
      }
      tc_fence_before();
      mbar_arrive(&ms.bar_s_free);

      // Mask keys past N and, on the diagonal tile, keys after the query.
      if (kt * 128 + 128 > p.N || (p.causal && kt == qt)) {
        const int lim = p.causal ? min(qrow + 1, p.N) : p.N;
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (kt * 128 + j >= lim) s[j] = -INFINITY;
      }
      float gm[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) gm[g] = max16(&s[16 * g]);
      const float smax = fmaxf(fmax3(gm[0], gm[1], gm[2]), fmax3(fmax3(gm[3], gm[4], gm[5]), gm[6], gm[7]));
      // t = fl32(S * sm_scale * log2 e) is monotone in S: max t = fl32(max S * c).
      const float Mn = fmaxf(M, ceilf(smax * c2));
      const float alpha = (M == -INFINITY) ? 0.f : exp2_int(M - Mn);
      const float Mx = (Mn == -INFINITY) ? 0.f : Mn;
      const float base = static_cast<float>(kPLog2) - Mx;  // exponent offset of P * 2^11

      // P of this tile's previous key tile has been multiplied (the P4 buffer is
      // free and O may be rescaled); the fp16 P columns are free once the
      // previous fp16 P V product in issue order is done.
      if (kt >= 1) failed = !wait_or_abort(&ms.bar_o_done[x], (kt - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      if (!failed && fp16 && my16 > 0)
        failed = !wait_or_abort(&ms.bar_p16_free, (my16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      failed = __any_sync(0xffffffffu, failed);
      if (failed) continue;
      tc_fence_after();

      // P * 2^11 = 2^(S*c + 11 - M), encoded and stored 64 (fp16) or 32 (NVFP4)
      // keys at a time; NVFP4 groups fold 1/scale into the exponent.
      float rs = 0.f;
      const float2 c2v = make_float2(c2, c2);
      if (fp16) {
        const float2 bb = make_float2(base, base);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float2 pp = ex2_fma2(s[64 * h + 2 * j], s[64 * h + 2 * j + 1], c2v, bb);
            s[64 * h + 2 * j] = pp.x;
            s[64 * h + 2 * j + 1] = pp.y;
            w[j] = pack_half2(pp.x, pp.y);
          }
          rs += sum16(&s[64 * h]) + sum16(&s[64 * h + 16]) + sum16(&s[64 * h + 32]) + sum16(&s[64 * h + 48]);
          tmem_st32(lane_base + kPColP16 + 32 * h, w);
        }
      } else {
        uint8_t* d4 = sm + L::kP4 + x * 8192;
        uint32_t sfw[2] = {0u, 0u};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t code[4];
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int g = 2 * c + gg;
            const float amax = ex2(fmaf(gm[g], c2, base));                         // max of P * 2^11
            const uint32_t sbyte = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.f) & 0xFFu;  // E4M3(amax / 6)
            const float sc = e4m3_to_f32(sbyte);
            const float sce = sc > 0.f ? sc : 1.0f;  // zero scale: codes round to 0, l keeps P
            const float bias = base - lg2(sce);
            const float2 bb = make_float2(bias, bias);
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const float2 pp = ex2_fma2(s[16 * g + i], s[16 * g + i + 1], c2v, bb);
              s[16 * g + i] = pp.x;
              s[16 * g + i + 1] = pp.y;
            }
            rs = fmaf(sum16(&s[16 * g]), sce, rs);
            code[2 * gg] = cvt_e2m1x8(&s[16 * g]);
            code[2 * gg + 1] = cvt_e2m1x8(&s[16 * g + 8]);
            sfw[g / 4] |= sbyte << (8 * (g % 4));
          }
          *reinterpret_cast<uint4*>(d4 + sw64_off(r, c)) = make_uint4(code[0], code[1], code[2], code[3]);
        }
        // Scale factors of a 128-row A operand: the MMA reads row r's four
        // scales of K chunk c from lane r, column base + 4c + r / 32.
        tmem_st1(lane_base + kPColSFP + 8 * x + quad, sfw[0]);
        tmem_st1(lane_base + kPColSFP + 8 * x + 4 + quad, sfw[1]);
      }
      l = l * alpha + rs;
      // Rescale O when the maximum grew (rows with alpha = 1 are unchanged).
      if (kt > 0 && __any_sync(0xffffffffu, Mn > M)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(ocol + 32 * cc, v);
          tmem_ld_wait();
          const float2 aa = make_float2(alpha, alpha);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 o = __fmul2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), aa);
            v[j] = __float_as_uint(o.x);
            v[j + 1] = __float_as_uint(o.y);
          }
          tmem_st32(ocol + 32 * cc, v);
        }
      }
      tmem_st_wait();
      M = Mn;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ms.bar_p_full[x]);
    }

    // ---- epilogue: O / l -> fp16 (both carry the 2^11 pre-scale) ----
    if (nx > 0) {
      if (!failed) failed = !wait_or_abort(&ms.bar_o_done[x], (nx - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA);
      failed = __any_sync(0xffffffffu, failed);
      if (!failed) {
        tc_fence_after();
        const float inv = 1.0f / l;
        __half* orow = p.O + (static_cast<size_t>(bh) * p.N + qrow) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(ocol + 32 * cc, v);
          tmem_ld_wait();
          if (qrow < p.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 w;
              w.x = pack_half2(__uint_as_float(v[j + 0]) * inv, __uint_as_float(v[j + 1]) * inv);
              w.y = pack_half2(__uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
              w.z = pack_half2(__uint_as_float(v[j + 4]) * inv, __uint_as_float(v[j + 5]) * inv);
              w.w = pack_half2(__uint_as_float(v[j + 6]) * inv, __uint_as_float(v[j + 7]) * inv);
              *reinterpret_cast<uint4*>(orow + 32 * cc + j) = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPPMmaS) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

}  // namespace

template <int D>
cudaError_t launch_attention_pp(const CUtensorMap& mQ16, const CUtensorMap& mK16, const CUtensorMap& mV16,
                                const CUtensorMap& mQ4, const CUtensorMap& mK4, const CUtensorMap& mV4,
                                const attn::Params& prm, cudaStream_t st) {
  const size_t smem = SmemPP<D>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(thrift_attention_pp_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(prm.B * prm.Hq * ((prm.NT + 1) / 2));
  thrift_attention_pp_kernel<D><<<grid, kPPThreads, smem, st>>>(mQ16, mK16, mV16, mQ4, mK4, mV4, prm);
  return cudaGetLastError();
}

template cudaError_t launch_attention_pp<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                             const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                             const attn::Params&, cudaStream_t);
template cudaError_t launch_attention_pp<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                              const attn::Params&, cudaStream_t);

}  // namespace thrift

// Stage 2 of the method (ThriftAttention abstract; summary, technical
// approach items 3-4): picked block pairs run in FP16, all others in FP4, and
// one online softmax folds both kinds of tile into the same output.
//
// One CTA computes one 128-row query tile of one (batch, query head) and walks
// its key tiles (128 keys each).  Per key tile the selection mask gives the
// precision of each selection block the tile covers (1 block for blk = 128,
// 2x2 for blk = 64); FP16 blocks use S = Q K^T from the fp16 operands
// (tcgen05 .kind::f16), FP4 blocks use the NVFP4 copies
// (tcgen05 .kind::mxf4nvf4, one UE4M3 scale per 16 elements).  Both land in
// tensor memory and feed one online softmax:
//   t = S * (sm_scale * log2 e); M = ceil(running max of t) (an integer, so a
//   rescale is an exact power of two); P = 2^(t - M); l += sum P;
//   P * 2^11 is encoded as fp16 (FP16 blocks) or NVFP4 per 16 keys (FP4
//   blocks) and O += P~ V~ accumulates both kinds into one FP32 tensor-memory
//   accumulator; finally O = O / (l * 2^11).
//
// Warp roles (576 threads):
//   warps 0-15 softmax: warp w owns rows 32*(w%4) .. +31 and keys
//              32*(w/4) .. +31 of each tile (four threads per row), so every
//              thread sees one selection block per tile and four softmax
//              warps share each SM sub-partition.
//   warp 16    producer: TMA / bulk copies of Q once, then K/V tiles into a
//              ring of FP4 slots and separate fp16 K and V slots.
//   warp 17    MMA issuer (lane 0) and tensor-memory owner.
// The S product of tile j+1 is issued as soon as the softmax has read S of
// tile j, so it overlaps the softmax of tile j; P V of tile j follows.
#include <cuda_fp16.h>

#include "attention_common.cuh"
#include "common.h"
#include "ptx.cuh"
#include "tmap.h"

namespace thrift {
namespace {
using namespace attn;

constexpr int kSplit = 4;                              // softmax threads per row
constexpr int kKPT = 128 / kSplit;                     // keys of a tile per softmax thread
constexpr int kGPT = kKPT / 16;                        // NVFP4 groups of P per softmax thread
constexpr int kSoftmaxWarps = 4 * kSplit;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr int kNS4 = 4;  // FP4 K/V ring slots (loads run up to three tiles ahead)

// Tensor-memory columns (512 allocated).
constexpr uint32_t kColS16 = 0;    // S from fp16 operands, 128 columns
constexpr uint32_t kColS4 = 128;   // S from NVFP4 operands, 128 columns
constexpr uint32_t kColO = 256;    // O accumulator, D columns
constexpr uint32_t kColSFQ = 384;  // scales of Q4, 4 columns per 64-wide K step
constexpr uint32_t kColSF = 392;   // two sets (tile parity) of: K4 scales (8), V4 scales (8), P4 scales (8)

template <int D>
struct Smem {
  static constexpr uint32_t kQ16 = 0;
  static constexpr uint32_t kQ16Bytes = 128 * D * 2;
  static constexpr uint32_t kRow4 = D / 2;  // bytes per row of Q4 / K4
  static constexpr uint32_t kQ4 = kQ16 + kQ16Bytes;
  static constexpr uint32_t kQ4Bytes = 128 * kRow4;
  static constexpr uint32_t kQSF = kQ4 + kQ4Bytes;
  static constexpr uint32_t kQSFBytes = (D / 64) * 512;
  static constexpr uint32_t kP16 = (kQSF + kQSFBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kP4 = kP16 + 32768;
  static constexpr uint32_t kPSF = kP4 + 8192;
  // FP4 slot: K4 | V4 | K4 scales | V4 scales
  static constexpr uint32_t kK4Bytes = 128 * kRow4;
  static constexpr uint32_t kV4Bytes = D * 64;
  static constexpr uint32_t kKSFBytes = (D / 64) * 512;
  static constexpr uint32_t kVSFBytes = 1024;
  static constexpr uint32_t kSlot4Bytes = (kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kSlot4 = kPSF + 1024;
  // FP16 slot: K16 | V16
  static constexpr uint32_t kK16Bytes = 128 * D * 2;
  static constexpr uint32_t kSlot16 = kSlot4 + kNS4 * kSlot4Bytes;
  static constexpr uint32_t kMisc = kSlot16 + 2 * kK16Bytes;
  static constexpr uint32_t kBytes = kMisc + 8192;
  static constexpr uint32_t kTx4 = kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes;
  static constexpr uint32_t kTx16 = kK16Bytes;  // K16 or V16 tile
  static constexpr uint32_t kTxQ = kQ16Bytes + kQ4Bytes + kQSFBytes;
  static_assert(kBytes + 1024 <= 232448, "shared memory above the 227 KB per-CTA limit");
};

struct Misc {
  uint64_t bar_q;
  uint64_t bar_full4[kNS4];
  uint64_t bar_empty4[kNS4];
  uint64_t bar_full_k16;
  uint64_t bar_empty_k16;
  uint64_t bar_full_v16;
  uint64_t bar_empty_v16;
  uint64_t bar_s_full;
  uint64_t bar_s_free;
  uint64_t bar_p_full;
  uint64_t bar_o_done;
  uint64_t bar_drain;
  uint32_t tmem;
  volatile int abort;
  float red_max[2][kSplit][128];
  float red_l[kSplit][128];
  uint8_t cls[1024];  // per key tile: bit (a*2 + c) = FP16 flag of block (query half a, key half c);
                      // SKIP: bit 4 + (a*2 + c) = skip flag
};

static_assert(sizeof(Misc) <= 8192, "barriers and exchange buffers must fit their shared-memory slice");

// SKIP = false: masks of 0 / 1 (the method).  SKIP = true: masks may hold 2
// (skipped pairs); a skipped block is computed like an NVFP4 one and its keys
// are then masked out of the softmax.  Separate instantiations, so the first
// keeps its own code.
template <int D, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1)
    thrift_attention_kernel(const __grid_constant__ CUtensorMap mQ16, const __grid_constant__ CUtensorMap mK16,
                            const __grid_constant__ CUtensorMap mV16, const __grid_constant__ CUtensorMap mQ4,
                            const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                            const Params p) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc& ms = *reinterpret_cast<Misc*>(sm + L::kMisc);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int BH = p.B * p.Hq;
  const int qt = p.NT - 1 - static_cast<int>(blockIdx.x) / BH;  // longest causal rows first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int n_kt = p.causal ? qt + 1 : p.NT;
  const int nb = p.N / p.blk;

  // ---- set-up --------------------------------------------------------------
  if (warp == kMmaWarp) {
    tmem_alloc(&ms.tmem, 512);
    tmem_relinquish();
  }
  if (tid == kProducerWarp * 32) {
    mbar_init(&ms.bar_q, 1);
    for (int i = 0; i < kNS4; ++i) {
      mbar_init(&ms.bar_full4[i], 1);
      mbar_init(&ms.bar_empty4[i], 1);
    }
    mbar_init(&ms.bar_full_k16, 1);
    mbar_init(&ms.bar_empty_k16, 1);
    mbar_init(&ms.bar_full_v16, 1);
    mbar_init(&ms.bar_empty_v16, 1);
    mbar_init(&ms.bar_s_full, 1);
    mbar_init(&ms.bar_s_free, kSoftmaxThreads);
    mbar_init(&ms.bar_p_full, kSoftmaxThreads);
    mbar_init(&ms.bar_o_done, 1);
    mbar_init(&ms.bar_drain, 1);
    ms.abort = 0;
    fence_mbar_init();
  }
  // precision class of every key tile of this query tile
  const uint8_t* mrow = p.mask + static_cast<size_t>(bh) * nb * nb;
  for (int kt = tid; kt < n_kt; kt += kThreads) {
    uint32_t c = 0;
    if (p.blk == 128) {
      const uint8_t mv = mrow[static_cast<size_t>(qt) * nb + kt];
      c = SKIP ? ((mv == 1 ? 0xFu : 0u) | (mv == 2 ? 0xF0u : 0u)) : (mv ? 0xFu : 0u);
      if (SKIP && mv > 2) record_error(p.err, DEV_BAD_ARG);  // 8-bit pairs need the 128-block kernel
    } else {
      for (int a = 0; a < 2; ++a)
        for (int k = 0; k < 2; ++k) {
          const int i = 2 * qt + a, j = 2 * kt + k;
          const uint8_t mv = (i < nb && j < nb) ? mrow[static_cast<size_t>(i) * nb + j] : 0;
          if (SKIP ? mv == 1 : mv != 0) c |= 1u << (a * 2 + k);
          if (SKIP && mv == 2) c |= 1u << (4 + a * 2 + k);
          if (SKIP && mv > 2) record_error(p.err, DEV_BAD_ARG);
        }
    }
    ms.cls[kt] = static_cast<uint8_t>(c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem;

  if (warp == kProducerWarp) {
    // ======================== producer ========================
    if (lane == 0) {
      prefetch_tensormap(&mQ16);
      prefetch_tensormap(&mK4);
      prefetch_tensormap(&mV4);
      mbar_arrive_expect_tx(&ms.bar_q, L::kTxQ);
      for (int pnl = 0; pnl < D / 64; ++pnl)
        tma_load_3d(sm + L::kQ16 + pnl * 16384, &mQ16, &ms.bar_q, pnl * 64, qt * 128, bh);
      tma_load_3d(sm + L::kQ4, &mQ4, &ms.bar_q, 0, qt * 128, bh);
      bulk_load(sm + L::kQSF, p.qs + (static_cast<size_t>(bh) * p.NT + qt) * L::kQSFBytes, L::kQSFBytes,
                &ms.bar_q);
      int u4 = 0, u16 = 0, u16k_only = 0;
      for (int kt = 0; kt < n_kt && !ms.abort; ++kt) {
        const uint32_t c = SKIP ? (ms.cls[kt] & 0xFu) : ms.cls[kt];  // FP16 flags
        // failure-detection test: this tile's slots are taken but its copies
        // are never issued, so the waits of their consumers run out
        const bool hold = kt == p.withhold;
        if (c != 0xFu) {
          const int slot = u4 % kNS4, use = u4 / kNS4;
          if (use > 0 && !wait_or_abort(&ms.bar_empty4[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns))
            break;
          if (!hold) {
            uint8_t* st = sm + L::kSlot4 + slot * L::kSlot4Bytes;
            mbar_arrive_expect_tx(&ms.bar_full4[slot], L::kTx4);
            tma_load_3d(st, &mK4, &ms.bar_full4[slot], 0, kt * 128, bhk);
            tma_load_3d(st + L::kK4Bytes, &mV4, &ms.bar_full4[slot], kt * 64, 0, bhk);
            bulk_load(st + L::kK4Bytes + L::kV4Bytes, p.ks + (static_cast<size_t>(bhk) * p.NT + kt) * L::kKSFBytes,
                      L::kKSFBytes, &ms.bar_full4[slot]);
            bulk_load(st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes,
                      p.vs + (static_cast<size_t>(bhk) * 2 * p.NT + 2 * kt) * 512, L::kVSFBytes, &ms.bar_full4[slot]);
          }
          ++u4;
        }
        if (c != 0u) {
          // K16 and V16 have separate slots: K16 frees when S is done, V16 when P V is done.
          uint8_t* st = sm + L::kSlot16;
          if (u16 > 0 && !wait_or_abort(&ms.bar_empty_k16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns))
            break;
          if (hold) {
            ++u16;
            continue;
          }
          mbar_arrive_expect_tx(&ms.bar_full_k16, L::kTx16);
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(st + pnl * 16384, &mK16, &ms.bar_full_k16, pnl * 64, kt * 128, bhk);
          if (u16 > 0 && !wait_or_abort(&ms.bar_empty_v16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)) {
            ++u16k_only;
            break;
          }
          mbar_arrive_expect_tx(&ms.bar_full_v16, L::kTx16);
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(st + L::kK16Bytes + pnl * 16384, &mV16, &ms.bar_full_v16, pnl * 64, kt * 128, bhk);
          ++u16;
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      mbar_wait(&ms.bar_q, 0, p.wait_ns);
      for (int s = 0; s < kNS4; ++s)
        if (u4 > s) mbar_wait(&ms.bar_full4[s], ((u4 - 1 - s) / kNS4) & 1, p.wait_ns);
      if (u16 + u16k_only > 0) mbar_wait(&ms.bar_full_k16, (u16 + u16k_only - 1) & 1, p.wait_ns);
      if (u16 > 0) mbar_wait(&ms.bar_full_v16, (u16 - 1) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ======================== MMA issuer ========================
    if (lane == 0) {
      const uint32_t q16 = sbase + L::kQ16, q4 = sbase + L::kQ4;
      const uint32_t p16 = sbase + L::kP16, p4 = sbase + L::kP4, psf = sbase + L::kPSF;
      constexpr uint32_t sbo4 = (D == 128) ? 512u : 256u;
      constexpr uint32_t sw4 = (D == 128) ? LAYOUT_SW64 : LAYOUT_SW32;
      bool ok = wait_or_abort(&ms.bar_q, 0, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns);
      tc_fence_after();
      if (ok)
        for (int c = 0; c < D / 64; ++c)
          tmem_cp_32x128b_x4(tm + kColSFQ + 4 * c, make_sdesc(sbase + L::kQSF + 512 * c, 16, 128, LAYOUT_NONE));
      int u4 = 0, u16k = 0, u16v = 0;  // slot uses consumed so far (loads)
      int slot4_of[2] = {0, 0};  // FP4 slot of tile kt (by parity)
      uint32_t o_acc = 0;
      // issue S of tile kt (its loads are complete)
      auto issue_s = [&](int kt) {
        const uint32_t c = SKIP ? (ms.cls[kt] & 0xFu) : ms.cls[kt];  // FP16 flags
        const uint32_t sfset = tm + kColSF + 24 * (kt & 1);
        if (c != 0u) {
          const uint32_t k16 = sbase + L::kSlot16;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * 16384 + (k % 4) * 32;
            mma_f16(tm + kColS16, make_sdesc(q16 + off, 16, 1024, LAYOUT_SW128),
                    make_sdesc(k16 + off, 16, 1024, LAYOUT_SW128), idesc_f16(128, 128, false), k > 0);
          }
        }
        if (c != 0xFu) {
          const uint32_t st = sbase + L::kSlot4 + slot4_of[kt & 1] * L::kSlot4Bytes;
          const uint32_t ksf = st + L::kK4Bytes + L::kV4Bytes;
          for (int cc = 0; cc < D / 64; ++cc)
            tmem_cp_32x128b_x4(sfset + 4 * cc, make_sdesc(ksf + 512 * cc, 16, 128, LAYOUT_NONE));
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc)
            mma_nvf4(tm + kColS4, make_sdesc(q4 + 32 * cc, 16, sbo4, sw4), make_sdesc(st + 32 * cc, 16, sbo4, sw4),
                     idesc_nvf4(128, 128), tm + kColSFQ + 4 * cc, sfset + 4 * cc, cc > 0);
        }
        mma_commit(&ms.bar_s_full);
        if (c != 0u) mma_commit(&ms.bar_empty_k16);
      };
      // wait for the loads of tile kt; records its FP4 slot
      auto wait_loads = [&](int kt) -> bool {
        const uint32_t c = SKIP ? (ms.cls[kt] & 0xFu) : ms.cls[kt];  // FP16 flags
        if (c != 0xFu) {
          const int slot = u4 % kNS4, use = u4 / kNS4;
          if (!wait_or_abort(&ms.bar_full4[slot], use & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns)) return false;
          slot4_of[kt & 1] = slot;
          ++u4;
        }
        if (c != 0u) {
          if (!wait_or_abort(&ms.bar_full_k16, u16k & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns)) return false;
          ++u16k;
        }
        tc_fence_after();
        return true;
      };
      if (ok) ok = wait_loads(0);
      if (ok) issue_s(0);
      for (int kt = 0; ok && kt < n_kt; ++kt) {
        if (kt + 1 < n_kt) {
          if (!wait_loads(kt + 1)) break;
          if (!wait_or_abort(&ms.bar_s_free, kt & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)) break;
          tc_fence_after();
          issue_s(kt + 1);
        }
        if (!wait_or_abort(&ms.bar_p_full, kt & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t c = SKIP ? (ms.cls[kt] & 0xFu) : ms.cls[kt];  // FP16 flags
        const uint32_t sfset = tm + kColSF + 24 * (kt & 1);
        const int slot4 = slot4_of[kt & 1];
        if (c != 0xFu) {
          const uint32_t st = sbase + L::kSlot4 + slot4 * L::kSlot4Bytes;
          const uint32_t v4 = st + L::kK4Bytes, vsf = st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes;
          for (int cc = 0; cc < 2; ++cc) {
            tmem_cp_32x128b_x4(sfset + 16 + 4 * cc, make_sdesc(psf + 512 * cc, 16, 128, LAYOUT_NONE));
            tmem_cp_32x128b_x4(sfset + 8 + 4 * cc, make_sdesc(vsf + 512 * cc, 16, 128, LAYOUT_NONE));
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            mma_nvf4(tm + kColO, make_sdesc(p4 + 32 * cc, 16, 512, LAYOUT_SW64),
                     make_sdesc(v4 + 32 * cc, 16, 512, LAYOUT_SW64), idesc_nvf4(128, D), sfset + 16 + 4 * cc,
                     sfset + 8 + 4 * cc, o_acc);
            o_acc = 1;
          }
        }
        if (c != 0u) {
          if (!wait_or_abort(&ms.bar_full_v16, u16v & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns)) break;
          ++u16v;
          tc_fence_after();
          const uint32_t v16 = sbase + L::kSlot16 + L::kK16Bytes;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            mma_f16(tm + kColO, make_sdesc(p16 + (k / 4) * 16384 + (k % 4) * 32, 16, 1024, LAYOUT_SW128),
                    make_sdesc(v16 + k * 2048, 16384, 1024, LAYOUT_SW128), idesc_f16(128, D, true), o_acc);
            o_acc = 1;
          }
        }
        mma_commit(&ms.bar_o_done);
        if (c != 0xFu) mma_commit(&ms.bar_empty4[slot4]);
        if (c != 0u) mma_commit(&ms.bar_empty_v16);
      }
      // drain: every tensor-core operation of this CTA completes before exit
      mma_commit(&ms.bar_drain);
      mbar_wait(&ms.bar_drain, 0, p.wait_ns);
    }
    __syncwarp();
  } else {
    // ======================== softmax ========================
    // Warp w owns rows 32*(w%4) .. +31 (its tensor-memory lane quarter) and keys
    // kKPT*(w/4) .. +kKPT-1 of every tile: one selection block per thread.
    constexpr int kOC = D / kSplit;        // O columns of this thread
    const int quad = warp % 4, part = warp / 4;
    const int r = quad * 32 + lane;        // row in the tile (tensor-memory lane)
    const int qrow = qt * 128 + r;         // query index
    const int a = r / 64;                  // query half (selection block for blk = 64)
    const int koff = part * kKPT;          // first key of this thread in a tile
    const int kh = koff / 64;              // key half (selection block for blk = 64)
    const uint32_t lane_base = tm + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t ocol = lane_base + kColO + part * kOC;
    float M = -INFINITY, l = 0.f;
    bool failed = false;  // this thread gave up a wait; the exit is taken jointly
    for (int kt = 0; kt < n_kt; ++kt) {
      const uint32_t c = SKIP ? (ms.cls[kt] & 0xFu) : ms.cls[kt];  // FP16 flags
      const bool fp16 = (c >> (a * 2 + kh)) & 1u;
      const bool need16 = c != 0u, need4 = c != 0xFu;
      if (!failed) failed = !wait_or_abort(&ms.bar_s_full, kt & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
      failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
      tc_fence_after();
      float s[kKPT];
      if (!failed) {
        uint32_t v[kKPT];
        const uint32_t col = lane_base + (fp16 ? kColS16 : kColS4) + koff;
#pragma unroll
        for (int q = 0; q < kKPT / 32; ++q) tmem_ld32(col + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * q]));
        tmem_ld_wait();
        tmem_ld_fence(v);
#pragma unroll
        for (int j = 0; j < kKPT; ++j) s[j] = __uint_as_float(v[j]);
        tc_fence_before();
        mbar_arrive(&ms.bar_s_free);
      } else {
#pragma unroll
        for (int j = 0; j < kKPT; ++j) s[j] = -INFINITY;
      }

      // Mask keys past N, on the diagonal tile keys after the query, and (SKIP)
      // all of this thread's keys when its block is skipped.
      const int key0 = kt * 128 + koff;
      const bool skipped = SKIP && ((ms.cls[kt] >> (4 + a * 2 + kh)) & 1u);
      if (kt * 128 + 128 > p.N || (p.causal && kt == qt) || skipped) {
        const int lim = skipped ? key0 : (p.causal ? min(qrow + 1, p.N) : p.N);  // keys < lim are valid
#pragma unroll
        for (int j = 0; j < kKPT; ++j)
          if (key0 + j >= lim) s[j] = -INFINITY;
      }
      // Group maxima of the raw scores (sm_scale > 0, so the order is that of t).
      float gm[kGPT];
#pragma unroll
      for (int g = 0; g < kGPT; ++g) gm[g] = max16(&s[16 * g]);
      float smax = gm[0];
#pragma unroll
      for (int g = 1; g < kGPT; ++g) smax = fmaxf(smax, gm[g]);
      ms.red_max[kt & 1][part][r] = smax;
      if (softmax_bar_or<kSoftmaxThreads>(failed)) break;
#pragma unroll
      for (int o = 0; o < kSplit; ++o) smax = fmaxf(smax, ms.red_max[kt & 1][o][r]);
      // t = fl32(S * sm_scale * log2 e) is monotone in S: the row maximum of t is
      // fl32(max S * c).
      const float c2 = p.scale_log2;
      const float Mn = fmaxf(M, ceilf(smax * c2));
      const float alpha = (M == -INFINITY) ? 0.f : exp2_int(M - Mn);
      const float Mx = (Mn == -INFINITY) ? 0.f : Mn;
      const float base = static_cast<float>(kPLog2) - Mx;  // exponent offset of P * 2^11

      // P * 2^11 = 2^(S*c + 11 - M); NVFP4 groups fold 1/scale into the exponent.
      float rs = 0.f;
      uint32_t codes[2 * kGPT];
      uint32_t sfw = 0;
      if (fp16) {
#pragma unroll
        for (int j = 0; j < kKPT; ++j) s[j] = ex2(fmaf(s[j], c2, base));
#pragma unroll
        for (int g = 0; g < kGPT; ++g) rs += sum16(&s[16 * g]);
      } else {
#pragma unroll
        for (int g = 0; g < kGPT; ++g) {
          const float amax = ex2(fmaf(gm[g], c2, base));                      // max of P * 2^11
          const uint32_t sb = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.f) & 0xFFu;  // E4M3(amax / 6)
          const float sc = e4m3_to_f32(sb);
          const float sce = sc > 0.f ? sc : 1.0f;  // zero scale: codes round to 0, l keeps P
          const float bias = base - lg2(sce);
#pragma unroll
          for (int i = 0; i < 16; ++i) s[16 * g + i] = ex2(fmaf(s[16 * g + i], c2, bias));
          rs = fmaf(sum16(&s[16 * g]), sce, rs);
          uint32_t w0 = 0, w1 = 0;
#pragma unroll
          for (int i = 0; i < 8; i += 2) w0 |= cvt_e2m1x2(s[16 * g + i], s[16 * g + i + 1]) << (i * 4);
#pragma unroll
          for (int i = 0; i < 8; i += 2) w1 |= cvt_e2m1x2(s[16 * g + 8 + i], s[16 * g + 9 + i]) << (i * 4);
          codes[2 * g] = w0;
          codes[2 * g + 1] = w1;
          sfw |= sb << (8 * g);
        }
      }
      l = l * alpha + rs;

      if (kt > 0) {
        failed = __any_sync(0xffffffffu,
                            !wait_or_abort(&ms.bar_o_done, (kt - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns));
        if (failed) continue;  // the next joint barrier ends the loop for every softmax thread
        tc_fence_after();
      }

      // write the encoded P for the P V product (P * 2^11)
      uint8_t* p16 = sm + L::kP16 + kh * 16384;
      uint8_t* p4 = sm + L::kP4;
      uint8_t* psf = sm + L::kPSF + kh * 512 + (r % 32) * 16 + (r / 32) * 4 + (koff % 64) / 16;
      const int ch16 = (koff % 64) / 8;  // first 16-byte chunk of this thread in the fp16 row
      const int ch4 = koff / 32;         // first 16-byte chunk of this thread in the NVFP4 row
      static_assert(kGPT == 2 || kGPT == 4, "scale bytes are stored as one 16- or 32-bit word");
      if (fp16) {
#pragma unroll
        for (int ch = 0; ch < kKPT / 8; ++ch) {
          uint4 w;
          w.x = pack_half2(s[8 * ch + 0], s[8 * ch + 1]);
          w.y = pack_half2(s[8 * ch + 2], s[8 * ch + 3]);
          w.z = pack_half2(s[8 * ch + 4], s[8 * ch + 5]);
          w.w = pack_half2(s[8 * ch + 6], s[8 * ch + 7]);
          *reinterpret_cast<uint4*>(p16 + sw128_off(r, ch16 + ch)) = w;
        }
        if (need4) {
#pragma unroll
          for (int q = 0; q < kKPT / 32; ++q)
            *reinterpret_cast<uint4*>(p4 + sw64_off(r, ch4 + q)) = make_uint4(0, 0, 0, 0);
          if (kGPT == 2) *reinterpret_cast<uint16_t*>(psf) = 0;
          else *reinterpret_cast<uint32_t*>(psf) = 0u;
        }
      } else {
#pragma unroll
        for (int q = 0; q < kKPT / 32; ++q)
          *reinterpret_cast<uint4*>(p4 + sw64_off(r, ch4 + q)) =
              make_uint4(codes[4 * q], codes[4 * q + 1], codes[4 * q + 2], codes[4 * q + 3]);
        if (kGPT == 2) *reinterpret_cast<uint16_t*>(psf) = static_cast<uint16_t>(sfw);
        else *reinterpret_cast<uint32_t*>(psf) = sfw;
        if (need16) {
#pragma unroll
          for (int ch = 0; ch < kKPT / 8; ++ch)
            *reinterpret_cast<uint4*>(p16 + sw128_off(r, ch16 + ch)) = make_uint4(0, 0, 0, 0);
        }
      }
      // Rescale O (after P V of the previous tile; before P V of this one).  Rows
      // whose maximum did not move have alpha = 1; the warp acts together.
      if (kt > 0 && __any_sync(0xffffffffu, Mn > M)) {
        if constexpr (kOC % 32 == 0) {
#pragma unroll
          for (int cc = 0; cc < kOC / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(ocol + 32 * cc, v);
            tmem_ld_wait();
            tmem_ld_fence(v);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
            tmem_st32(ocol + 32 * cc, v);
          }
        } else {
          uint32_t v[16];
          tmem_ld16(ocol, v);
          tmem_ld_wait();
          tmem_ld_fence(v);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
          tmem_st16(ocol, v);
        }
        tmem_st_wait();
      }
      M = Mn;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ms.bar_p_full);
    }

    // ---- epilogue: O / l -> fp16 (both carry the 2^11 pre-scale) ----
    if (!failed) failed = !wait_or_abort(&ms.bar_o_done, (n_kt - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
    failed = __any_sync(0xffffffffu, failed);
    ms.red_l[part][r] = l;
    if (!softmax_bar_or<kSoftmaxThreads>(failed)) {
      tc_fence_after();
      float lt = 0.f;
#pragma unroll
      for (int o = 0; o < kSplit; ++o) lt += ms.red_l[o][r];
      const float inv = 1.0f / lt;
      __half* orow = p.O + (static_cast<size_t>(bh) * p.N + qrow) * D + part * kOC;
      uint32_t v[kOC];
      if constexpr (kOC % 32 == 0) {
#pragma unroll
        for (int cc = 0; cc < kOC / 32; ++cc) tmem_ld32(ocol + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * cc]));
      } else {
        tmem_ld16(ocol, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
      }
      tmem_ld_wait();
      tmem_ld_fence(v);
      if (qrow < p.N) {
#pragma unroll
        for (int j = 0; j < kOC; j += 8) {
          uint4 w;
          w.x = pack_half2(__uint_as_float(v[j + 0]) * inv, __uint_as_float(v[j + 1]) * inv);
          w.y = pack_half2(__uint_as_float(v[j + 2]) * inv, __uint_as_float(v[j + 3]) * inv);
          w.z = pack_half2(__uint_as_float(v[j + 4]) * inv, __uint_as_float(v[j + 5]) * inv);
          w.w = pack_half2(__uint_as_float(v[j + 6]) * inv, __uint_as_float(v[j + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + j) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

template <int D>
cudaError_t launch_d(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4, const void* qs,
                     const void* k4, const void* ks, const void* v4, const void* vs, const thrift_shape& s, void* O,
                     bool skip, const Mx8Copies* eight, uint32_t* err, cudaStream_t st) {
  CUtensorMap mQ16, mK16, mV16, mQ4, mK4, mV4;
  CUtensorMap mQ8 = {}, mK8 = {}, mV8 = {};  // read only by the 8-bit instantiation
  const uint64_t BHq = static_cast<uint64_t>(s.B) * s.Hq, BHk = static_cast<uint64_t>(s.B) * s.Hkv;
  const CUtensorMapSwizzle sw4 = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  bool ok = true;
  ok &= make_tmap_3d(&mQ16, Q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, s.N, BHq, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&mK16, K, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, s.N, BHk, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&mV16, V, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, s.N, BHk, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_tmap_3d(&mQ4, q4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, s.N, BHq, D / 2, 128, sw4);
  ok &= make_tmap_3d(&mK4, k4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, s.N, BHk, D / 2, 128, sw4);
  ok &= make_tmap_3d(&mV4, v4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.N / 2, D, BHk, 64, D, CU_TENSOR_MAP_SWIZZLE_64B);
  if (eight) {
    // MXFP8 codes: Q / K rows of D bytes, V rows of N bytes (keys contiguous)
    const CUtensorMapSwizzle sw8 = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    ok &= make_tmap_3d(&mQ8, eight->q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, s.N, BHq, D, 128, sw8);
    ok &= make_tmap_3d(&mK8, eight->k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, s.N, BHk, D, 128, sw8);
    ok &= make_tmap_3d(&mV8, eight->v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.N, D, BHk, 128, D,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return cudaErrorInvalidValue;
  Params prm;
  prm.mask = mask;
  prm.qs = static_cast<const uint8_t*>(qs);
  prm.ks = static_cast<const uint8_t*>(ks);
  prm.vs = static_cast<const uint8_t*>(vs);
  prm.O = static_cast<__half*>(O);
  prm.err = err;
  prm.B = s.B;
  prm.Hq = s.Hq;
  prm.Hkv = s.Hkv;
  prm.N = s.N;
  prm.blk = s.blk;
  prm.causal = s.causal;
  prm.NT = num_tiles(s.N);
  prm.scale_log2 = static_cast<float>(static_cast<double>(s.sm_scale) * 1.4426950408889634073599246810019);
  prm.skip = skip ? 1 : 0;
  prm.qs8 = eight ? static_cast<const uint8_t*>(eight->qs8) : nullptr;
  prm.ks8 = eight ? static_cast<const uint8_t*>(eight->ks8) : nullptr;
  prm.vs8 = eight ? static_cast<const uint8_t*>(eight->vs8) : nullptr;
  prm.eight = eight ? 1 : 0;
  prm.wait_ns = wait_limit_ns();
  prm.withhold = test_withhold_tile();
  if (s.blk == 128) return launch_attention_db<D>(mQ16, mK16, mV16, mQ4, mK4, mV4, mQ8, mK8, mV8, prm, st);
  if (eight) return cudaErrorInvalidValue;  // the entry point rejects this shape first
  const unsigned grid = static_cast<unsigned>(BHq * prm.NT);
  const size_t smem = Smem<D>::kBytes + 1024;
  const auto kern = skip ? thrift_attention_kernel<D, true> : thrift_attention_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(mQ16, mK16, mV16, mQ4, mK4, mV4, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4,
                             const void* qs, const void* k4, const void* ks, const void* v4, const void* vs,
                             const thrift_shape& s, void* O, bool skip, const Mx8Copies* eight, uint32_t* err,
                             cudaStream_t st) {
  if (s.D == 128) return launch_d<128>(Q, K, V, mask, q4, qs, k4, ks, v4, vs, s, O, skip, eight, err, st);
  return launch_d<64>(Q, K, V, mask, q4, qs, k4, ks, v4, vs, s, O, skip, eight, err, st);
}

}  // namespace thrift

// Stage 2 of the method for 128 x 128 selection blocks (ThriftAttention
// abstract: picked block pairs in FP16, the rest in FP4, one online softmax
// over both), with the key tiles of a query tile split between two softmax
// groups.
//
// A CTA owns one 128-row query tile of one (batch, query head).  With blk =
// 128 each key tile is one selection block, so it is entirely FP16 or
// entirely NVFP4.  The processed key tiles alternate between two groups of
// softmax threads: group 0 takes tiles 0, 2, 4, ..., group 1 tiles 1, 3, ...
// Each group has one thread per query row, which handles all 128 keys of its
// tiles, and keeps its own integer running maximum M = ceil(max t), its own
// row sum l and its own output accumulator O_g in tensor memory.  Per key
// tile:
//   S from the fp16 operands (.kind::f16) or the NVFP4 copies
//   (.kind::mxf4nvf4) into the one S buffer; t = S * sm_scale * log2 e;
//   P * 2^11 = 2^(t + 11 - M) encoded as fp16 (tensor memory, the A operand
//   of a .kind::f16 product) or as NVFP4 per 16 keys (codes in the group's
//   shared-memory buffer, scales stored by each row's thread straight into
//   tensor memory); O_g += P~ V~, with O_g rescaled by an exact power of two
//   when the group's maximum grows.
// The epilogue merges the two groups' partial softmaxes, both taken relative
// to integer maxima, exactly: O = (2^(M_0 - M) O_0 + 2^(M_1 - M) O_1) /
// (2^(M_0 - M) l_0 + 2^(M_1 - M) l_1), M = max(M_0, M_1).  This is the same
// online softmax the method describes, with the key tiles merged in two
// interleaved sequences.
//
// Why two groups: every thread of the softmax runs a long dependent chain
// per key tile (tensor-memory load, row maximum, group scales, exponentials,
// encoding).  Two groups give every SM sub-partition two independent chains
// on different key tiles, so one group's exponentials on the MUFU overlap the
// other group's loads, maxima and encoding, and no thread recomputes another
// thread's row maximum.
//
// Tensor memory (512 columns): S (128), O_0 and O_1 (128 each), the fp16 /
// 8-bit P operand (64), the scale factors of Q4, of K4 (two buffers, so the
// next tile's are copied while the S buffer is still in use), of V4 and of
// each group's P4, and the MXFP8 scales of the 8-bit instantiation.  The S buffer is
// single: the S issuer computes S of the next key tile as soon as the
// previous tile's group has loaded its S into registers, early in that
// group's iteration.  The fp16 / 8-bit P region is shared by both groups in
// processing order: a group that needs it waits until the P V product of the
// previous tile that used it has been issued and has completed.
//
// Warp roles (384 threads): warps 0-3 softmax group 0, warps 4-7 group 1
// (warp w reads the tensor-memory lanes of rows 32 (w % 4) ..), warp 8 the TMA
// producer, warp 9 the S issuer (and owner of tensor memory), warp 10 the P V
// issuer, warp 11 idle.  The roles meet only through mbarriers.  The role
// warpgroup hands registers to the softmax warpgroups (setmaxnreg), whose
// threads hold a whole 128-key row of S.
//
// A third instantiation adds 8-bit pairs (mask 3, the MXFP8 copies of Q, K
// and V): S from .kind::mxf8f6f4 products with E8M0 scales in tensor memory,
// and P * 2^11 encoded per 32 keys as MXFP8 (E8M0 scale from the group's
// maximum, E4M3 codes) into the tensor-memory P region.  An 8-bit key tile
// travels through the NVFP4 ring as two consecutive slots (K8 and its scales,
// then V8 and its scales), so it is prefetched like an NVFP4 tile.
#include <cuda_fp16.h>

#include "attention_common.cuh"
#include "common.h"
#include "ptx.cuh"
#include "tmap.h"

namespace thrift {
namespace {
using namespace attn;

constexpr int kDBThreads = 384;  // three warpgroups: two softmax groups, the roles
constexpr int kDBSoftmax = 256;  // two groups of 128 softmax threads
constexpr int kDBGroup = 128;
constexpr int kDBProducer = 8;
constexpr int kDBMmaS = 9;
constexpr int kDBMmaPV = 10;
// Registers per thread after the split: the launch gives 384 x 168; the role
// warpgroup keeps 56, each softmax warpgroup takes 224 (2 x 128 x 224 +
// 128 x 56 = 384 x 168).
constexpr uint32_t kDBRegsRoles = 56;
constexpr uint32_t kDBRegsSoftmax = 224;
static_assert(2 * 128 * kDBRegsSoftmax + 128 * kDBRegsRoles <= kDBThreads * 168, "register split above the launch");

// Tensor-memory columns (512 allocated).
constexpr uint32_t kDColS = 0;      // S of the key tile being handed to a group
constexpr uint32_t kDColO = 128;    // O of group g at 128 + 128 g, D columns
constexpr uint32_t kDColP = 384;    // fp16 P (64 columns) or P8 (32 columns), shared in processing order
constexpr uint32_t kDColSFQ = 448;  // Q4 scales, 4 columns per 64-wide chunk of D
constexpr uint32_t kDColSFK = 456;  // K4 scales of even processed key tiles (odd ones at kDColSFK1)
constexpr uint32_t kDColSFV = 464;  // V4 scales of the key tile being multiplied
constexpr uint32_t kDColSFP = 472;  // P4 scales of group g at 8 g: 64-key chunk c of row r at 4 c + r / 32
                                    // (P8: byte k of that column for keys 64 c + 32 k ..)
constexpr uint32_t kDColSFQ8 = 488;  // Q8 scales (byte g: channels 32 g ..)
constexpr uint32_t kDColSFK8 = 492;  // K8 scales of even processed key tiles (odd ones at kDColSFK81)
constexpr uint32_t kDColSFV8 = 496;  // V8 scales (byte g: keys 32 g ..)
constexpr uint32_t kDColSFK81 = 500;  // K8 scales of odd processed key tiles
constexpr uint32_t kDColSFK1 = 504;   // K4 scales of odd processed key tiles

template <int D, bool EIGHT>
struct SmemDB {
  static constexpr uint32_t kQ16Bytes = 128 * D * 2;
  static constexpr uint32_t kQ16 = 0;
  static constexpr uint32_t kQ4Bytes = 128 * D / 2;
  static constexpr uint32_t kQ4 = kQ16 + kQ16Bytes;
  static constexpr uint32_t kQSFBytes = (D / 64) * 512;
  static constexpr uint32_t kQSF = kQ4 + kQ4Bytes;
  static constexpr uint32_t kPBufBytes = 8192;  // 128 rows x 128 keys of E2M1, 64B-swizzled
  static constexpr uint32_t kP4 = (kQSF + kQSFBytes + 1023) / 1024 * 1024;  // one buffer per group
  static constexpr uint32_t kQ8Bytes = EIGHT ? 128 * D : 0;                 // Q8 tile, then its scales
  static constexpr uint32_t kQ8 = kP4 + 2 * kPBufBytes;
  static constexpr uint32_t kQS8Bytes = EIGHT ? 512 : 0;
  static constexpr uint32_t kQS8 = kQ8 + kQ8Bytes;
  static constexpr uint32_t kK4Bytes = 128 * D / 2;
  static constexpr uint32_t kV4Bytes = D * 64;
  static constexpr uint32_t kKSFBytes = (D / 64) * 512;
  static constexpr uint32_t kVSFBytes = 1024;
  static constexpr uint32_t kSlot4Bytes = (kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kSlot4 = (kQS8 + kQS8Bytes + 1023) / 1024 * 1024;
  static constexpr int kNS = 4;  // NVFP4 K/V ring slots (an 8-bit tile takes two)
  static constexpr uint32_t kK16Bytes = 128 * D * 2;
  static constexpr uint32_t kSlot16 = kSlot4 + kNS * kSlot4Bytes;  // K16 then V16
  static constexpr uint32_t kMisc = kSlot16 + 2 * kK16Bytes;
  static constexpr uint32_t kBytes = kMisc + 6144;
  static constexpr uint32_t kTx4 = kK4Bytes + kV4Bytes + kKSFBytes + kVSFBytes;
  static constexpr uint32_t kTx16 = kK16Bytes;
  static constexpr uint32_t kTxQ = kQ16Bytes + kQ4Bytes + kQSFBytes + kQ8Bytes + kQS8Bytes;
  // 8-bit K / V tiles, each in one NVFP4 ring slot followed by its 512 scale bytes
  static constexpr uint32_t kK8Bytes = 128 * D;  // 128 keys x D channels
  static constexpr uint32_t kV8Bytes = D * 128;  // D channels x 128 keys
  static constexpr uint32_t kTx8 = kK8Bytes + 512;
  static_assert(kK8Bytes + 512 <= kSlot4Bytes && kV8Bytes + 512 <= kSlot4Bytes, "8-bit tiles must fit a ring slot");
  static_assert(kBytes + 1024 <= 232448, "shared memory above the 227 KB per-CTA limit");
  static_assert(kQ4 % 1024 == 0 && kSlot4 % 1024 == 0 && kSlot16 % 1024 == 0 && kQ8 % 1024 == 0,
                "TMA tiles need 1 KB alignment");
};

struct MiscDB {
  uint64_t bar_q;
  uint64_t bar_full4[4], bar_empty4[4];
  uint64_t bar_full_k16, bar_empty_k16, bar_full_v16, bar_empty_v16;
  uint64_t bar_s_full[2];  // S of group g's next key tile is in tensor memory (one phase per tile of g)
  uint64_t bar_s_free[2];  // group g's threads loaded that S into registers
  uint64_t bar_p_full[2];  // group g's P written
  uint64_t bar_o_done[2];  // group g's P V product done (O_g stable, its P buffers free)
  uint64_t bar_pt_free;    // the tensor-memory P region read by its last P V product (one phase per use)
  uint64_t bar_drain[2];   // one per issuing thread
  uint32_t tmem;
  volatile int abort;
  volatile int pt_issued;  // P V products issued so far that read the tensor-memory P region
  float mrow[2][128];      // the two groups' running maxima, for the epilogue
  float lrow[2][128];      // and row sums
  union {
    uint8_t cls[1024];   // SKIP = false: per key tile, 1 = FP16, 0 = NVFP4
    uint16_t lst[1024];  // SKIP = true: key tiles to process in order, tile index | 0x8000 FP16 | 0x4000 8-bit
  };
  int np;                // key tiles processed
};
static_assert(sizeof(MiscDB) <= 6144, "barriers must fit their shared-memory slice");

// Maxima of the eight 16-key groups of a 128-key row of S, and the row maximum.
__device__ __forceinline__ float max128(const float* v, float (&gh)[8]) {
#pragma unroll
  for (int g = 0; g < 8; ++g) gh[g] = max16(&v[16 * g]);
  return fmaxf(fmax3(fmax3(gh[0], gh[1], gh[2]), fmax3(gh[3], gh[4], gh[5]), gh[6]), gh[7]);
}

// SKIP = false: masks of 0 / 1 (the method); every key tile of the query
// tile is processed.  SKIP = true: masks may hold 2 (skipped pairs); the
// skipped tiles are left out of an ordered list that every role walks.
// EIGHT = true (with SKIP): masks may also hold 3, 8-bit pairs.  They are
// separate instantiations so the method's keeps its own code.  A mask byte
// the instantiation does not know records DEV_BAD_ARG (the tile is then
// computed in NVFP4).
template <int D, bool SKIP, bool EIGHT>
__global__ void __launch_bounds__(kDBThreads, 1)
    thrift_attention_db_kernel(const __grid_constant__ CUtensorMap mQ16, const __grid_constant__ CUtensorMap mK16,
                               const __grid_constant__ CUtensorMap mV16, const __grid_constant__ CUtensorMap mQ4,
                               const __grid_constant__ CUtensorMap mK4, const __grid_constant__ CUtensorMap mV4,
                               const __grid_constant__ CUtensorMap mQ8, const __grid_constant__ CUtensorMap mK8,
                               const __grid_constant__ CUtensorMap mV8, const Params p) {
  static_assert(SKIP || !EIGHT, "8-bit pairs come with the skip-aware list");
  using L = SmemDB<D, EIGHT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  MiscDB& ms = *reinterpret_cast<MiscDB*>(sm + L::kMisc);
  const uint32_t sbase = smem_u32(sm);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int BH = p.B * p.Hq;
  const int qt = p.NT - 1 - static_cast<int>(blockIdx.x) / BH;  // longest causal rows first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const int nk = p.causal ? qt + 1 : p.NT;  // key tiles this query tile attends to
  const int nb = p.NT;                     // blk = 128

  if (warp == kDBMmaS) {
    tmem_alloc(&ms.tmem, 512);
    tmem_relinquish();
  }
  if (tid == kDBProducer * 32) {
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
      mbar_init(&ms.bar_s_free[i], kDBGroup);
      mbar_init(&ms.bar_p_full[i], kDBGroup);
      mbar_init(&ms.bar_o_done[i], 1);
      mbar_init(&ms.bar_drain[i], 1);
    }
    mbar_init(&ms.bar_pt_free, 1);
    ms.abort = 0;
    ms.pt_issued = 0;
    fence_mbar_init();
  }
  if constexpr (SKIP) {
    if (warp == 0) {
      // Key tiles to process in increasing order: mask 1 FP16, 3 8-bit, 0
      // NVFP4, 2 skipped (left out).  All of the row's mask bytes are loaded
      // at once (nk <= 1024 = 32 x 32), then compacted in order from registers.
      const uint8_t* m0 = p.mask + static_cast<size_t>(bh) * nb * nb + static_cast<size_t>(qt) * nb;
      uint8_t mv[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) mv[q] = (q * 32 + lane < nk) ? m0[q * 32 + lane] : 2;
      int base = 0;
      bool bad = false;
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const uint32_t keep = __ballot_sync(0xffffffffu, mv[q] != 2);
        bad |= mv[q] > (EIGHT ? 3 : 2);
        if (mv[q] != 2)
          ms.lst[base + __popc(keep & ((1u << lane) - 1u))] = static_cast<uint16_t>(
              (q * 32 + lane) | (mv[q] == 1 ? 0x8000 : 0) | ((EIGHT && mv[q] == 3) ? 0x4000 : 0));
        base += __popc(keep);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(p.err, DEV_BAD_ARG);
      if (lane == 0) ms.np = base;
    }
  } else {
    const uint8_t* m0 = p.mask + static_cast<size_t>(bh) * nb * nb + static_cast<size_t>(qt) * nb;
    for (int kt = tid; kt < nk; kt += kDBThreads) ms.cls[kt] = m0[kt] ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = ms.tmem;
  const int np = SKIP ? ms.np : nk;
  // the it-th processed key tile and its precision
  const auto tile_of = [&](int it) -> int { return SKIP ? (ms.lst[it] & 0x3FF) : it; };
  const auto fp16_of = [&](int it) -> bool { return SKIP ? (ms.lst[it] & 0x8000) != 0 : ms.cls[it] != 0; };
  const auto eight_of = [&](int it) -> bool { return EIGHT && (ms.lst[it] & 0x4000) != 0; };
  // the P V product of tile it reads its P from tensor memory (fp16 and 8-bit tiles)
  const auto ptmem_of = [&](int it) -> bool { return fp16_of(it) || eight_of(it); };
  // Bounded waits with the slow path out of line in the producer and issuer
  // loops, and in the method's softmax loop too (the waits' code changes how
  // the roles' hot loops share the instruction caches).
  constexpr bool kOolRoles = true, kOolSoftmax = !SKIP;

  // The two register regimes never share code after the split: each
  // warpgroup's branch runs to its own end, where every thread meets at a
  // (non-aligned) CTA barrier before tensor memory is freed.
  if (warp >= kDBProducer) {
  setmaxnreg_dec<kDBRegsRoles>();
  if (warp == kDBProducer) {
    // ======================== producer ========================
    if (lane == 0) {
      prefetch_tensormap(&mQ16);
      prefetch_tensormap(&mK4);
      prefetch_tensormap(&mV4);
      if constexpr (EIGHT) {
        prefetch_tensormap(&mK8);
        prefetch_tensormap(&mV8);
      }
      mbar_arrive_expect_tx(&ms.bar_q, L::kTxQ);
      for (int pnl = 0; pnl < D / 64; ++pnl)
        tma_load_3d(sm + L::kQ16 + pnl * 16384, &mQ16, &ms.bar_q, pnl * 64, qt * 128, bh);
      tma_load_3d(sm + L::kQ4, &mQ4, &ms.bar_q, 0, qt * 128, bh);
      bulk_load(sm + L::kQSF, p.qs + (static_cast<size_t>(bh) * p.NT + qt) * L::kQSFBytes, L::kQSFBytes, &ms.bar_q);
      if constexpr (EIGHT) {
        tma_load_3d(sm + L::kQ8, &mQ8, &ms.bar_q, 0, qt * 128, bh);
        bulk_load(sm + L::kQS8, p.qs8 + (static_cast<size_t>(bh) * p.NT + qt) * 512, 512, &ms.bar_q);
      }
      int u4 = 0, u16 = 0;
      for (int it = 0; it < np && !ms.abort; ++it) {
        const int kt = tile_of(it);
        // failure-detection test: this tile's slots are taken but its copies
        // are never issued, so the waits of their consumers run out
        const bool hold = it == p.withhold;
        if (!fp16_of(it) && !eight_of(it)) {
          const int slot = u4 % L::kNS, use = u4 / L::kNS;
          if (use > 0 && !bounded_wait<kOolRoles, 1>(&ms.bar_empty4[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns))
            break;
          if (hold) {
            ++u4;
            continue;
          }
          uint8_t* st = sm + L::kSlot4 + slot * L::kSlot4Bytes;
          mbar_arrive_expect_tx(&ms.bar_full4[slot], L::kTx4);
          tma_load_3d(st, &mK4, &ms.bar_full4[slot], 0, kt * 128, bhk);
          tma_load_3d(st + L::kK4Bytes, &mV4, &ms.bar_full4[slot], kt * 64, 0, bhk);
          bulk_load(st + L::kK4Bytes + L::kV4Bytes, p.ks + (static_cast<size_t>(bhk) * p.NT + kt) * L::kKSFBytes,
                    L::kKSFBytes, &ms.bar_full4[slot]);
          bulk_load(st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes,
                    p.vs + (static_cast<size_t>(bhk) * 2 * p.NT + 2 * kt) * 512, L::kVSFBytes, &ms.bar_full4[slot]);
          ++u4;
        } else if (EIGHT && eight_of(it)) {
          // 8-bit tile: K8 and its scales in ring slot u4, V8 and its scales in u4 + 1
          bool stop = false;
          for (int part = 0; part < 2; ++part) {
            const int slot = u4 % L::kNS, use = u4 / L::kNS;
            if (use > 0 && !bounded_wait<kOolRoles, 1>(&ms.bar_empty4[slot], (use - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)) {
              stop = true;
              break;
            }
            if (hold) {
              ++u4;
              continue;
            }
            uint8_t* st = sm + L::kSlot4 + slot * L::kSlot4Bytes;
            const size_t sc = (static_cast<size_t>(bhk) * p.NT + kt) * 512;
            mbar_arrive_expect_tx(&ms.bar_full4[slot], L::kTx8);
            if (part == 0) {
              tma_load_3d(st, &mK8, &ms.bar_full4[slot], 0, kt * 128, bhk);
              bulk_load(st + L::kK8Bytes, p.ks8 + sc, 512, &ms.bar_full4[slot]);
            } else {
              tma_load_3d(st, &mV8, &ms.bar_full4[slot], kt * 128, 0, bhk);
              bulk_load(st + L::kV8Bytes, p.vs8 + sc, 512, &ms.bar_full4[slot]);
            }
            ++u4;
          }
          if (stop) break;
        } else {
          uint8_t* st = sm + L::kSlot16;
          if (u16 > 0 && !bounded_wait<kOolRoles, 1>(&ms.bar_empty_k16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns))
            break;
          if (hold) {
            ++u16;
            continue;
          }
          mbar_arrive_expect_tx(&ms.bar_full_k16, L::kTx16);
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(st + pnl * 16384, &mK16, &ms.bar_full_k16, pnl * 64, kt * 128, bhk);
          if (u16 > 0 && !bounded_wait<kOolRoles, 1>(&ms.bar_empty_v16, (u16 - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)) {
            mbar_wait(&ms.bar_full_k16, u16 & 1, p.wait_ns);  // the K16 copy of this tile is in flight
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
      for (int s = 0; s < L::kNS; ++s)
        if (u4 > s) mbar_wait(&ms.bar_full4[s], ((u4 - 1 - s) / L::kNS) & 1, p.wait_ns);
      if (u16 > 0) {
        mbar_wait(&ms.bar_full_k16, (u16 - 1) & 1, p.wait_ns);
        mbar_wait(&ms.bar_full_v16, (u16 - 1) & 1, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == kDBMmaS) {
    // ================= S issuer: K scales, then S of each key tile in order =================
    if (lane == 0) {
      constexpr uint32_t sbo4 = (D == 128) ? 512u : 256u;
      constexpr uint32_t sw4 = (D == 128) ? LAYOUT_SW64 : LAYOUT_SW32;
      bool ok = bounded_wait<kOolRoles, 1>(&ms.bar_q, 0, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns);
      tc_fence_after();
      if (ok) {
        for (int c = 0; c < D / 64; ++c)
          tmem_cp_32x128b_x4(tm + kDColSFQ + 4 * c, make_sdesc(sbase + L::kQSF + 512 * c, 16, 128, LAYOUT_NONE));
        if constexpr (EIGHT) tmem_cp_32x128b_x4(tm + kDColSFQ8, make_sdesc(sbase + L::kQS8, 16, 128, LAYOUT_NONE));
      }
      int u4 = 0, uk16 = 0;
      for (int it = 0; ok && it < np; ++it) {
        const bool fp16 = fp16_of(it), eight = eight_of(it);
        int slot = 0;
        if (EIGHT && eight) {
          // K8 in ring slot u4 (V8, in u4 + 1, is the P V issuer's)
          slot = u4 % L::kNS;
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full4[slot], (u4 / L::kNS) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          u4 += 2;
        } else if (!fp16) {
          slot = u4 % L::kNS;
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full4[slot], (u4 / L::kNS) & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          ++u4;
        } else {
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full_k16, uk16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          ++uk16;
        }
        // The K scales go to tensor memory before the wait for the S buffer,
        // into the buffer of this tile's parity (the product two tiles back,
        // which read it, precedes the copy in this thread's tcgen05 order), so
        // only the products themselves follow the S buffer's release.
        tc_fence_after();
        const uint32_t sfk = tm + ((it & 1) ? kDColSFK1 : kDColSFK);
        const uint32_t sfk8 = tm + ((it & 1) ? kDColSFK81 : kDColSFK8);
        if (EIGHT && eight) {
          tmem_cp_32x128b_x4(sfk8, make_sdesc(sbase + L::kSlot4 + slot * L::kSlot4Bytes + L::kK8Bytes, 16, 128,
                                              LAYOUT_NONE));
        } else if (!fp16) {
          const uint32_t ksf = sbase + L::kSlot4 + slot * L::kSlot4Bytes + L::kK4Bytes + L::kV4Bytes;
          for (int c = 0; c < D / 64; ++c)
            tmem_cp_32x128b_x4(sfk + 4 * c, make_sdesc(ksf + 512 * c, 16, 128, LAYOUT_NONE));
        }
        // The one S buffer: the group of the previous key tile must have
        // loaded its S.  (Barriers and phases count processed tiles, it.)
        if (it >= 1) {
          const int pv = it - 1;
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_s_free[pv & 1], (pv >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns)))
            break;
          tc_fence_after();
        }
        const uint32_t dS = tm + kDColS;
        if (EIGHT && eight) {
          // MXFP8 along D: K = 32 per product, scale byte kk of each row's column
          constexpr uint32_t sbo8 = (D == 128) ? 1024u : 512u;
          constexpr uint32_t sw8 = (D == 128) ? LAYOUT_SW128 : LAYOUT_SW64;
          const uint32_t q8 = sbase + L::kQ8, k8 = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_mxf8(dS, make_sdesc(q8 + 32 * kk, 16, sbo8, sw8), make_sdesc(k8 + 32 * kk, 16, sbo8, sw8),
                     idesc_mxf8(128, 128, kk, kk), tm + kDColSFQ8, sfk8, kk > 0);
        } else if (!fp16) {
          const uint32_t q4 = sbase + L::kQ4;
          const uint32_t k4 = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            mma_nvf4(dS, make_sdesc(q4 + 32 * c, 16, sbo4, sw4), make_sdesc(k4 + 32 * c, 16, sbo4, sw4),
                     idesc_nvf4(128, 128), tm + kDColSFQ + 4 * c, sfk + 4 * c, c > 0);
        } else {
          const uint32_t q16 = sbase + L::kQ16, k16 = sbase + L::kSlot16;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * 16384 + (k % 4) * 32;
            mma_f16(dS, make_sdesc(q16 + off, 16, 1024, LAYOUT_SW128), make_sdesc(k16 + off, 16, 1024, LAYOUT_SW128),
                    idesc_f16(128, 128, false), k > 0);
          }
        }
        mma_commit(&ms.bar_s_full[it & 1]);
        // the K operands of this key tile are no longer needed (V: the P V
        // issuer).  An 8-bit tile's K slot is this thread's alone: both of its
        // arrivals, after this thread saw the slot filled.
        if (EIGHT && eight) {
          mma_commit(&ms.bar_empty4[slot]);
          mma_commit(&ms.bar_empty4[slot]);
        } else if (!fp16) {
          mma_commit(&ms.bar_empty4[slot]);
        } else {
          mma_commit(&ms.bar_empty_k16);
        }
      }
      // drain: every tensor-core operation this thread issued completes before exit
      mma_commit(&ms.bar_drain[0]);
      mbar_wait(&ms.bar_drain[0], 0, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == kDBMmaPV) {
    // ================= P V issuer: O_g += P V for each key tile in order =================
    if (lane == 0) {
      bool ok = true;
      int u4 = 0, uv16 = 0, upt = 0;
      for (int it = 0; ok && it < np; ++it) {
        const int g = it & 1;
        const bool fp16 = fp16_of(it), eight = eight_of(it);
        // The V operands (and the V4 scales, copied to tensor memory) do not
        // depend on P, so they are made ready before waiting for it.  The copy
        // follows the previous P V product in this thread's tcgen05 order, so
        // it cannot overwrite scales that product still reads.
        int slot = 0;
        uint32_t v4 = 0;
        if (EIGHT && eight) {
          // V8 in ring slot u4 + 1 (K8, in u4, is the S issuer's)
          slot = (u4 + 1) % L::kNS;
          const int use = (u4 + 1) / L::kNS;
          u4 += 2;
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full4[slot], use & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          tc_fence_after();
          v4 = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
          tmem_cp_32x128b_x4(tm + kDColSFV8, make_sdesc(v4 + L::kV8Bytes, 16, 128, LAYOUT_NONE));
        } else if (!fp16) {
          slot = u4 % L::kNS;
          const int use = u4 / L::kNS;
          ++u4;
          // V4 landed with K4 in one barrier phase; wait on it here too so that
          // this thread observes the copy itself.  The producer cannot refill the
          // slot before this thread releases it.
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full4[slot], use & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          tc_fence_after();
          const uint32_t st = sbase + L::kSlot4 + slot * L::kSlot4Bytes;
          v4 = st + L::kK4Bytes;
          const uint32_t vsf = st + L::kK4Bytes + L::kV4Bytes + L::kKSFBytes;
          for (int c = 0; c < 2; ++c)
            tmem_cp_32x128b_x4(tm + kDColSFV + 4 * c, make_sdesc(vsf + 512 * c, 16, 128, LAYOUT_NONE));
        } else {
          if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_full_v16, uv16 & 1, &ms.abort, p.err, DEV_TIMEOUT_LOAD, p.wait_ns))) break;
          ++uv16;
        }
        if (!(ok = bounded_wait<kOolRoles, 1>(&ms.bar_p_full[g], (it >> 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_OTHER, p.wait_ns))) break;
        const bool pt = fp16 || (EIGHT && eight);
        if (pt) ms.pt_issued = ++upt;  // the next user of the P region may wait on its barrier now
        tc_fence_after();
        const uint32_t dO = tm + kDColO + 128 * g;
        uint32_t acc = it >= 2 ? 1u : 0u;  // a group's first product overwrites its O
        if (EIGHT && eight) {
          // P8 (tensor memory, 32 columns) times V8 (D x 128 keys, 128B-swizzled):
          // K = 32 per product; P's scale for keys 32 kk .. is byte kk % 2 of
          // column 4 (kk / 2) + r / 32 of the group's scales, V's byte kk of column d / 32
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_mxf8_ts(dO, tm + kDColP + 8 * kk, make_sdesc(v4 + 32 * kk, 16, 1024, LAYOUT_SW128),
                        idesc_mxf8(128, D, kk & 1, kk), tm + kDColSFP + 8 * g + 4 * (kk >> 1), tm + kDColSFV8,
                        acc);
            acc = 1;
          }
        } else if (!fp16) {
          const uint32_t p4s = sbase + L::kP4 + g * L::kPBufBytes;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            mma_nvf4(dO, make_sdesc(p4s + 32 * c, 16, 512, LAYOUT_SW64), make_sdesc(v4 + 32 * c, 16, 512, LAYOUT_SW64),
                     idesc_nvf4(128, D), tm + kDColSFP + 8 * g + 4 * c, tm + kDColSFV + 4 * c, acc);
            acc = 1;
          }
        } else {
          const uint32_t v16 = sbase + L::kSlot16 + L::kK16Bytes;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            mma_f16_ts(dO, tm + kDColP + 8 * k, make_sdesc(v16 + k * 2048, 16384, 1024, LAYOUT_SW128),
                       idesc_f16(128, D, true), acc);
            acc = 1;
          }
        }
        mma_commit(&ms.bar_o_done[g]);
        if (pt) mma_commit(&ms.bar_pt_free);
        if (EIGHT && eight) {  // the V8 slot is this thread's alone: both arrivals
          mma_commit(&ms.bar_empty4[slot]);
          mma_commit(&ms.bar_empty4[slot]);
        } else if (!fp16) {
          mma_commit(&ms.bar_empty4[slot]);
        } else {
          mma_commit(&ms.bar_empty_v16);
        }
      }
      mma_commit(&ms.bar_drain[1]);
      mbar_wait(&ms.bar_drain[1], 0, p.wait_ns);
    }
    __syncwarp();
  }
  tc_fence_before();
  cta_barrier_all(kDBThreads);
  if (warp == kDBMmaS) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  } else {
    setmaxnreg_inc<kDBRegsSoftmax>();
    // ======================== softmax (one thread per row, two groups) ========================
    const int quad = warp % 4, grp = warp / 4;
    const int r = quad * 32 + lane;
    const int qrow = qt * 128 + r;
    const uint32_t lane_base = tm + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t ocol = lane_base + kDColO + 128 * grp;  // this group's O
    const float c2 = p.scale_log2;
    float M = -INFINITY, l = 0.f;
    bool failed = false;
    // uses of the tensor-memory P region before the current tile (both groups)
    int pt_before = (grp == 1 && np > 0 && ptmem_of(0)) ? 1 : 0;
    int j = 0;  // this group's tiles so far
    for (int it = grp; it < np; it += 2, ++j) {
      if (it >= 2) pt_before += (ptmem_of(it - 2) ? 1 : 0) + (ptmem_of(it - 1) ? 1 : 0);
      if (failed) continue;
      const int kt = tile_of(it);
      const bool fp16 = fp16_of(it), eight = eight_of(it);
      // All of the tile's waits come first, so that everything from the S
      // load to the P stores is one stretch of code the compiler can
      // interleave.  S of this tile:
      failed = !bounded_wait<kOolSoftmax, 2>(&ms.bar_s_full[grp], j & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
      // this group's P buffers (the shared-memory P4 codes and the tensor-
      // memory P4 scales) and its O are free once its previous tile's P V
      // product is done;
      if (!failed && j > 0)
        failed = !bounded_wait<kOolSoftmax, 2>(&ms.bar_o_done[grp], (j - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
      // the tensor-memory P region is taken in processing order: the P V
      // product of its previous user must have been issued (a counter, so no
      // barrier phase can be mistaken for another) and be complete.
      if (!failed && (fp16 || (EIGHT && eight)) && pt_before > 0) {
        if (ms.pt_issued < pt_before) {
          const uint64_t t0 = globaltimer_ns();
          while (ms.pt_issued < pt_before) {
            if (ms.abort) {
              failed = true;
              break;
            }
            if (globaltimer_ns() - t0 > p.wait_ns) {
              record_error(p.err, DEV_TIMEOUT_OTHER);
              ms.abort = 1;
              failed = true;
              break;
            }
          }
        }
        if (!failed)
          failed = !bounded_wait<kOolSoftmax, 2>(&ms.bar_pt_free, (pt_before - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
      }
      failed = __any_sync(0xffffffffu, failed);  // tcgen05.ld is warp-collective
      if (failed) continue;
      tc_fence_after();
      // This thread's row of S, all 128 keys.
      float s[128];
      {
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(lane_base + kDColS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
        tmem_ld_wait();
        tmem_ld_fence(v);
        tc_fence_before();
        mbar_arrive(&ms.bar_s_free[grp]);
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(v[c]);
      }
      // Mask keys past N and, on the diagonal tile, keys after the query.
      if (kt * 128 + 128 > p.N || (p.causal && kt == qt)) {
        const int lim = (p.causal ? min(qrow + 1, p.N) : p.N) - kt * 128;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float gh[8];  // maxima of the eight 16-key groups
      const float smax = max128(s, gh);
      // t = fl32(S * sm_scale * log2 e) is monotone in S: max t = fl32(max S * c).
      const float Mn = fmaxf(M, ceilf(smax * c2));

      const float alpha = (M == -INFINITY) ? 0.f : exp2_int(M - Mn);
      const float Mx = (Mn == -INFINITY) ? 0.f : Mn;
      const float base = static_cast<float>(kPLog2) - Mx;  // exponent offset of P * 2^11

      // NVFP4 group scales E4M3(fl32(amax / 6)) of the eight groups
      // (independent chains, ahead of the exponentials); MXFP8 scales of the
      // four 32-key groups for an 8-bit tile.
      float sce[8], bias[8];
      uint32_t sfw[2] = {0u, 0u};
      if (EIGHT && eight) {
        // X = 2^(floor(log2 amax) - 8) from the exponent field of amax = max
        // of P * 2^11, E8M0 byte = that exponent - 8 (biased), clamped at 0.
        // A group whose byte would be 0 (amax below 2^-118, P below 2^-129) is
        // encoded as zeros; the codes are E4M3(P * 2^11 / X) with -log2 X in
        // the bias.  Both 16-key halves of a group take its X and bias.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float amax = ex2(fmaf(fmaxf(gh[2 * c], gh[2 * c + 1]), c2, base));
          const int eb = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
          const bool live = eb > 8;
          sce[2 * c] = sce[2 * c + 1] = live ? __uint_as_float(static_cast<uint32_t>(eb - 8) << 23) : 0.f;  // X
          bias[2 * c] = bias[2 * c + 1] = live ? base + static_cast<float>(135 - eb) : -INFINITY;
          sfw[c >> 1] |= static_cast<uint32_t>(live ? eb - 8 : 0) << (8 * (c & 1));
        }
      } else if (!fp16) {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float amax = ex2(fmaf(gh[g], c2, base));                         // max of P * 2^11
          const uint32_t sbyte = cvt_e4m3x2(amax * (1.0f / 6.0f), 0.f) & 0xFFu;  // E4M3(amax / 6)
          const float sc = e4m3_to_f32(sbyte);
          sce[g] = sc > 0.f ? sc : 1.0f;  // zero scale: codes round to 0, l keeps P
          bias[g] = base - lg2(sce[g]);
          sfw[g >> 2] |= sbyte << (8 * (g & 3));
        }
      }

      if (!fp16) {
        tmem_st1(lane_base + kDColSFP + 8 * grp + quad, sfw[0]);
        tmem_st1(lane_base + kDColSFP + 8 * grp + 4 + quad, sfw[1]);
      }
      // P * 2^11 = 2^(S*c + 11 - M) for the row's 128 keys, encoded as fp16
      // or as NVFP4 (each group folds 1/scale into the exponent).
      float rs = 0.f;
      const float2 c2v = make_float2(c2, c2);
      if (fp16) {
        const float2 bv = make_float2(base, base);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 pp = ex2_fma2(s[64 * h + 2 * i], s[64 * h + 2 * i + 1], c2v, bv);
            s[64 * h + 2 * i] = pp.x;
            s[64 * h + 2 * i + 1] = pp.y;
            w[i] = pack_half2(pp.x, pp.y);
          }
          tmem_st32(lane_base + kDColP + 32 * h, w);
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) rs += sum16(&s[16 * g]);
      } else {
        // exponentials with 1/scale folded in, then sums and codes
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float2 bv = make_float2(bias[g], bias[g]);
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float2 pp = ex2_fma2(s[16 * g + i], s[16 * g + i + 1], c2v, bv);
            s[16 * g + i] = pp.x;
            s[16 * g + i + 1] = pp.y;
          }
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) rs = fmaf(sum16(&s[16 * g]), sce[g], rs);
        if (EIGHT && eight) {
          // 8-bit tile: four E4M3 codes per tensor-memory column, the row's
          // 128 keys in the region's first 32 columns
          uint32_t w8[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            w8[i] = (cvt_e4m3x2(s[4 * i], s[4 * i + 1]) & 0xFFFFu) | (cvt_e4m3x2(s[4 * i + 2], s[4 * i + 3]) << 16);
          tmem_st32(lane_base + kDColP, w8);
        } else {
          uint8_t* d4 = sm + L::kP4 + grp * L::kPBufBytes;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w = make_uint4(cvt_e2m1x8(&s[32 * c]), cvt_e2m1x8(&s[32 * c + 8]),
                                       cvt_e2m1x8(&s[32 * c + 16]), cvt_e2m1x8(&s[32 * c + 24]));
            *reinterpret_cast<uint4*>(d4 + sw64_off(r, c)) = w;
          }
        }
      }
      l = l * alpha + rs;
      // Rescale this group's O when its maximum grew (rows with alpha = 1 are
      // unchanged); O is stable: its previous P V product is done.
      if (j > 0 && __any_sync(0xffffffffu, Mn > M)) {
        const float2 aa = make_float2(alpha, alpha);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
          uint32_t v[64];
          tmem_ld32(ocol + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld32(ocol + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_ld_wait();
          tmem_ld_fence(v);
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            const float2 o = __fmul2_rn(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), aa);
            v[i] = __float_as_uint(o.x);
            v[i + 1] = __float_as_uint(o.y);
          }
          tmem_st32(ocol + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_st32(ocol + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        }
      }
      tmem_st_wait();
      M = Mn;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ms.bar_p_full[grp]);
    }

    // ---- epilogue: merge the two groups, O / l -> fp16 (both carry the 2^11 pre-scale) ----
    const int n0 = (np + 1) / 2, n1 = np / 2;  // tiles of each group
    const int nmine = grp ? n1 : n0;
    if (!failed && nmine > 0)
      failed = !bounded_wait<kOolSoftmax, 2>(&ms.bar_o_done[grp], (nmine - 1) & 1, &ms.abort, p.err, DEV_TIMEOUT_MMA, p.wait_ns);
    ms.mrow[grp][r] = M;
    ms.lrow[grp][r] = l;
    // every softmax thread takes the same exit decision (and sees both groups' M and l)
    failed = softmax_bar_or<kDBSoftmax>(failed);
    if (!failed && np > 0) {
      tc_fence_after();
      const float M0 = ms.mrow[0][r], M1 = ms.mrow[1][r];
      const float Mt = fmaxf(M0, M1);
      const float f0 = (n0 > 0 && M0 != -INFINITY) ? exp2_int(M0 - Mt) : 0.f;
      const float f1 = (n1 > 0 && M1 != -INFINITY) ? exp2_int(M1 - Mt) : 0.f;
      const float inv = 1.0f / (ms.lrow[0][r] * f0 + ms.lrow[1][r] * f1);
      const float w0 = f0 * inv, w1 = f1 * inv;
      // this thread writes D/2 channels: group g the half g
      __half* orow = p.O + (static_cast<size_t>(bh) * p.N + qrow) * D + grp * (D / 2);
      const uint32_t o0 = lane_base + kDColO + grp * (D / 2), o1 = o0 + 128;
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t v0[32], v1[32];
        tmem_ld32(o0 + 32 * cc, v0);
        if (n1 > 0) tmem_ld32(o1 + 32 * cc, v1);
        tmem_ld_wait();
        tmem_ld_fence(v0);
        if (n1 > 0) {
          tmem_ld_fence(v1);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v1[i] = 0u;
        }
        if (qrow < p.N) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o[e] = fmaf(__uint_as_float(v0[i + e]), w0, __uint_as_float(v1[i + e]) * w1);
            uint4 w;
            w.x = pack_half2(o[0], o[1]);
            w.y = pack_half2(o[2], o[3]);
            w.z = pack_half2(o[4], o[5]);
            w.w = pack_half2(o[6], o[7]);
            *reinterpret_cast<uint4*>(orow + 32 * cc + i) = w;
          }
        }
      }
    }
    tc_fence_before();
    cta_barrier_all(kDBThreads);
  }
}

}  // namespace

template <int D, bool SKIP, bool EIGHT>
static cudaError_t launch_db(const CUtensorMap& mQ16, const CUtensorMap& mK16, const CUtensorMap& mV16,
                             const CUtensorMap& mQ4, const CUtensorMap& mK4, const CUtensorMap& mV4,
                             const CUtensorMap& mQ8, const CUtensorMap& mK8, const CUtensorMap& mV8,
                             const attn::Params& prm, cudaStream_t st) {
  const size_t smem = SmemDB<D, EIGHT>::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(thrift_attention_db_kernel<D, SKIP, EIGHT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(prm.B * prm.Hq * prm.NT);
  thrift_attention_db_kernel<D, SKIP, EIGHT>
      <<<grid, kDBThreads, smem, st>>>(mQ16, mK16, mV16, mQ4, mK4, mV4, mQ8, mK8, mV8, prm);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_attention_db(const CUtensorMap& mQ16, const CUtensorMap& mK16, const CUtensorMap& mV16,
                                const CUtensorMap& mQ4, const CUtensorMap& mK4, const CUtensorMap& mV4,
                                const CUtensorMap& mQ8, const CUtensorMap& mK8, const CUtensorMap& mV8,
                                const attn::Params& prm, cudaStream_t st) {
  if (prm.eight) return launch_db<D, true, true>(mQ16, mK16, mV16, mQ4, mK4, mV4, mQ8, mK8, mV8, prm, st);
  if (prm.skip) return launch_db<D, true, false>(mQ16, mK16, mV16, mQ4, mK4, mV4, mQ8, mK8, mV8, prm, st);
  return launch_db<D, false, false>(mQ16, mK16, mV16, mQ4, mK4, mV4, mQ8, mK8, mV8, prm, st);
}

#define THRIFT_DB_INSTANCE(D)                                                                                        \
  template cudaError_t launch_attention_db<D>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,          \
                                              const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,          \
                                              const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,          \
                                              const attn::Params&, cudaStream_t);
THRIFT_DB_INSTANCE(64)
THRIFT_DB_INSTANCE(128)
#undef THRIFT_DB_INSTANCE

}  // namespace thrift

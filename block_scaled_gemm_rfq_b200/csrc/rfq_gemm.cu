// rfq_gemm.cu -- kernel 2: the RFQ block-scaled GEMM on sm_100a tensor cores.
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): the residual of the activation is
// requantized and its product is added up inside the GEMM.  Here
//
//     Y = DQ(QX).DQ(QW)^T + DQ(QR).DQ(QW)^T
//
// is one accumulation in TMEM: for every k-tile both QX x QW and QR x QW are
// issued as tcgen05 kind::mxf4 block-scaled MMAs into the same fp32 accumulator,
// reusing the QW tile already in shared memory, so the residual doubles the work
// on the tensor pipe (K -> 2K) and costs no extra pass over Y.
//
// Two variants of one persistent, warp-specialized kernel:
//   kPair = 1  one CTA per 128 x 256 output tile (MMA M = 128, cta_group::1);
//   kPair = 2  a cluster of two CTAs per 256 x 256 tile (MMA M = 256,
//              cta_group::2): each CTA loads its own 128 rows of QX/QR and half
//              of the QW tile, the leader CTA issues the MMAs for the pair and
//              the tensor cores read the QW halves from both CTAs' shared
//              memory, so each SM moves ~25 % fewer operand bytes per MMA.
// Roles (per CTA):
//   warp 0      TMA producer: per k-tile (256 elements = 128 bytes per row) the
//               code tiles (2-D maps, 128-byte swizzle) and the stage's scale
//               atoms (one 4-D box per operand) into a kStages-deep ring;
//               out-of-range rows/atoms are zero-filled by the TMA unit;
//   warp 10     scale copies (one thread of the leader CTA): as soon as a stage
//               has landed, copies its scale atoms to the stage's TMEM slot
//               (tcgen05.cp 32x128b.warpx4) and commits to the stage's
//               scales-ready barrier, running up to the ring's depth ahead of
//               the MMAs;
//   warp 1      MMA issuer (one thread of the leader CTA): per stage, once its
//               scales are in TMEM, 4 + 4 MMAs of K = 64; tcgen05.commit frees the
//               stage and, at the end of a tile, signals the epilogues;
//   warps 2..9  epilogue: TMEM -> registers (128 columns per warp), release of
//               the accumulator, then fp32/bf16 -> global (one row per thread),
//               overlapping the next tile's mainloop.
// Before its dependency wait the producer prefetches its first stages into L2.
// Every mbarrier wait is bounded (rfq_ptx.cuh); a wait that runs out records an
// error code, raises the CTA's abort flag and the CTA tears down cleanly.  No TMA
// multicast is used anywhere (the pair's loads each fill their own CTA).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rfq_internal.h"
#include "rfq_ptx.cuh"
#include "rfq_tmap.h"

namespace rfq {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kBM = 128;               // rows of X / Y per CTA (MMA M per CTA)
constexpr int kBN = 256;               // columns of Y per tile (MMA N)
constexpr int kBK = 256;               // K elements per stage (2 scale atoms of 128)
constexpr int kBKBytes = kBK / 2;      // packed FP4: 128 bytes per row per stage
constexpr int kThreads = 352;          // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue, warp 10 scale copies
constexpr int kScaleWarp = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;        // 256 fp32 columns: the 128 x 256 accumulator of this CTA
// Scale factors in TMEM: one 32-column slot per pipeline stage (from column 256),
// so a stage's tcgen05.cp never overwrites scales that queued MMAs still read.
// A slot holds the stage's 2 scale atoms (k-atoms a = 0, 1; 128 K each) of:
constexpr uint32_t kSfBase = 256;
constexpr uint32_t kSfSlot = 32;
constexpr uint32_t kSfaXCol = 0;       // +4a..4a+3:   QX, this CTA's 128 rows
constexpr uint32_t kSfaRCol = 8;       // +8+4a..:     QR
constexpr uint32_t kSfbCol = 16;       // +16+8a..+7:  QW, the tile's 256 rows (2 row atoms)
static_assert(kSfBase % 4 == 0 && kSfSlot % 4 == 0 && kSfaXCol % 4 == 0 && kSfaRCol % 4 == 0 && kSfbCol % 4 == 0,
              "tcgen05.cp 32x128b destinations start on a multiple of 4 TMEM columns");
constexpr uint32_t kSmemLimit = 232448;

// One ring stage: the QX tile, the QR tile (residual kernels only), this CTA's part
// of the QW tile, then the scale atoms of the same operands.  The ring holds as many
// stages as fit: 4 for the RFQ kernel with CTA pairs (52 KiB stages), 6 for the pair
// kernels without a residual term (35 KiB), 3 and 4 for single CTAs.  The scale warp
// needs the depth: it copies a stage's scales as soon as the stage lands, and those
// copies must reach the tensor pipe before the MMAs of the stage ahead of it.
template <int kPair, bool kResidual>
struct Layout {
  static constexpr uint32_t kATile = kBM * kBKBytes;                 // 16 KiB
  static constexpr uint32_t kBTile = (kBN / kPair) * kBKBytes;       // 32 KiB (single) or 16 KiB (pair)
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffR = kOffA + kATile;                  // residual kernels only
  static constexpr uint32_t kOffB = kOffA + (kResidual ? 2u : 1u) * kATile;
  static constexpr uint32_t kOffSfaX = kOffB + kBTile;               // 2 atoms (k-atom 0, 1)
  static constexpr uint32_t kOffSfaR = kOffSfaX + 1024;              // residual kernels only
  static constexpr uint32_t kOffSfb = kOffSfaX + (kResidual ? 2048u : 1024u);   // [row atom lo, hi][k-atom 0, 1]
  static constexpr uint32_t kStage = kOffSfb + 2048;
  static constexpr uint32_t kBarrierBytes = 256;
  static constexpr int kStages = static_cast<int>((kSmemLimit - 1024 - kBarrierBytes) / kStage);
  static constexpr uint32_t kSmem = kStages * kStage + kBarrierBytes + 1024;
  static_assert(kStage % 1024 == 0, "stage buffers must keep 1 KiB alignment");
  static_assert(kStages >= 3, "the ring needs at least 3 stages");
  static_assert(kSmem <= kSmemLimit, "exceeds the 227 KiB shared-memory limit");
  static_assert((3 * kStages + 4) * 8 + 8 <= kBarrierBytes, "barrier area too small");
  static_assert(kSfBase + kStages * kSfSlot <= kTmemCols, "scale slots exceed TMEM");
};

struct GemmParams {
  void* y;
  int M;
  int N;
  int num_kt;            // k-tiles of 256 elements
  int num_nb;            // tiles along N
  int num_tiles;         // tiles (kPair = 1) or pair tiles (kPair = 2)
  int skip_fill;         // fault injection (-1 = off)
};

struct Maps {
  CUtensorMap x, r, w;           // codes: [rows][K/2] bytes, box 128 B x (128 | 256 | 128) rows, 128-byte swizzle
  CUtensorMap sx, sr, sw;        // scales: [row tiles][k atoms][2][256 B]; box = 2 k-atoms of 1 (A) or 2 (B) row tiles
};

// Shared-memory matrix descriptor (tcgen05): K-major operand, 128-byte swizzle,
// rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull)     // start address
         | (1ull << 16)                // leading byte offset (unused for swizzled K-major)
         | ((1024ull >> 4) << 32)      // stride byte offset: 8 rows x 128 B
         | (1ull << 46)                // descriptor version (sm_100)
         | (2ull << 61);               // layout: 128-byte swizzle
}

// Descriptor of a 512-byte scale atom as 32 rows x 16 bytes, no swizzle, 8-row
// core matrices 128 bytes apart (source of tcgen05.cp 32x128b).
__device__ __forceinline__ uint64_t scale_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull) | ((128ull >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::mxf4 (E2M1 x E2M1) or kind::mxf8f6f4 (E4M3 x
// E4M3) with E8M0 scales: both K-major, M = 128 * kPair, N = 256, scale-factor
// byte selectors for A and B.
template <int kPair, bool kFp8>
__device__ __forceinline__ uint32_t mma_idesc(uint32_t sf_id) {
  constexpr uint32_t kFmt = kFp8 ? 0u : 1u;      // E4M3 in kind::mxf8f6f4, E2M1 in kind::mxf4
  return (sf_id << 4)                            // B scale-factor id
         | (kFmt << 7)                           // A format
         | (kFmt << 10)                          // B format
         | (uint32_t(kBN >> 3) << 17)            // N / 8
         | (1u << 23)                            // scale type UE8M0
         | (uint32_t((kBM * kPair) >> 4) << 24)  // M / 16
         | (sf_id << 29);                        // A scale-factor id
}

template <int kPair, bool kResidual, bool kBf16Out, bool kTransOut, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    rfq_gemm_kernel(const __grid_constant__ Maps maps, const GemmParams p) {
  using L = Layout<kPair, kResidual>;
  // A stage is 128 bytes of codes per row either way: 256 K of FP4 (2 scale atoms
  // per operand row tile) or 128 K of FP8 (1 atom).
  constexpr int kKAtoms = kFp8 ? 1 : 2;
  constexpr uint32_t kSfaBytes = 512u * kKAtoms;        // one row tile
  constexpr uint32_t kSfbBytes = 2u * 512u * kKAtoms;   // two row tiles (256 rows of W)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kStages * L::kStage);
  uint64_t* empty = full + L::kStages;
  uint64_t* acc_full = empty + L::kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* drain_sf = drain + 1;
  uint64_t* sready = drain_sf + 1;   // per stage: its scale atoms are in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sready + L::kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair == 2 ? cluster_cta_rank() : 0u;     // 0 = leader of the pair
  const bool leader = rank == 0;
  const int unit = kPair == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int num_units = kPair == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8 * kPair);
    mbar_init(drain, 1);
    mbar_init(drain_sf, 1);
    for (int s = 0; s < L::kStages; ++s) mbar_init(&sready[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&maps.x);
    prefetch_tmap(&maps.w);
    prefetch_tmap(&maps.sx);
    prefetch_tmap(&maps.sw);
    if (kResidual) {
      prefetch_tmap(&maps.r);
      prefetch_tmap(&maps.sr);
    }
  }
  if (warp == 1) {
    tmem_alloc_g<kPair>(tmem_slot, kTmemCols);
    tmem_relinquish_g<kPair>();
  }
  tc_fence_before();
  if (kPair == 2) cluster_sync();   // the peer's loads may signal our barriers from here on
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  griddep_launch_dependents();
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      if (unit < p.num_tiles) {
        // While the previous kernel on the stream finishes, pull the first stages of
        // this CTA's first tile into L2 (a hint; the copies still follow the wait).
        const int mb = unit / p.num_nb, nb = unit - (unit / p.num_nb) * p.num_nb;
        const int row_a = (mb * kPair + static_cast<int>(rank)) * kBM;
        const int row_b = nb * kBN + static_cast<int>(rank) * (kBN / kPair);
        for (int kt = 0; kt < L::kStages && kt < p.num_kt; ++kt) {
          if (row_b < p.N) tma_prefetch_2d(&maps.w, kt * kBKBytes, row_b);
          if (row_a < p.M) {
            tma_prefetch_2d(&maps.x, kt * kBKBytes, row_a);
            if (kResidual) tma_prefetch_2d(&maps.r, kt * kBKBytes, row_a);
          }
        }
      }
      griddep_wait();   // QX/QR/QW may be written by the previous kernel on the stream
      uint32_t stage = 0, phase = 0;
      uint32_t filled = 0, last_parity = 0;
      int fill = 0;
      // Bytes one CTA loads per stage; the leader arms its full barrier with the
      // bytes of both CTAs of a pair (the peer's copies complete on it too).
      const uint32_t bytes_cta = L::kATile + L::kBTile + kSfaBytes + kSfbBytes + (kResidual ? L::kATile + kSfaBytes : 0u);
      const uint32_t bytes = bytes_cta * kPair;
      for (int tile = unit; tile < p.num_tiles; tile += num_units) {
        const int mb = tile / p.num_nb;
        const int nb = tile - mb * p.num_nb;
        const int row_a = (mb * kPair + static_cast<int>(rank)) * kBM;       // this CTA's rows of X
        const int row_b = nb * kBN + static_cast<int>(rank) * (kBN / kPair); // this CTA's rows of W
        const int rt_a = mb * kPair + static_cast<int>(rank);                // this CTA's 128-row scale tile
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, &g_device_error, kErrWaitEmpty)) goto producer_done;
          if (!(fill == p.skip_fill && blockIdx.x == 0)) {
            uint8_t* st = smem + stage * L::kStage;
            if constexpr (kPair == 2) {
              const uint32_t bar = map_to_cta(smem_addr(&full[stage]), 0);
              if (leader) mbar_arrive_expect_tx(&full[stage], bytes);
              tma_load_2d_pair(st + L::kOffA, &maps.x, bar, kt * kBKBytes, row_a);
              if (kResidual) tma_load_2d_pair(st + L::kOffR, &maps.r, bar, kt * kBKBytes, row_a);
              tma_load_2d_pair(st + L::kOffB, &maps.w, bar, kt * kBKBytes, row_b);
              tma_load_4d_pair(st + L::kOffSfaX, &maps.sx, bar, 0, 0, kKAtoms * kt, rt_a);
              if (kResidual) tma_load_4d_pair(st + L::kOffSfaR, &maps.sr, bar, 0, 0, kKAtoms * kt, rt_a);
              tma_load_4d_pair(st + L::kOffSfb, &maps.sw, bar, 0, 0, kKAtoms * kt, 2 * nb);
            } else {
              mbar_arrive_expect_tx(&full[stage], bytes);
              tma_load_2d(st + L::kOffA, &maps.x, &full[stage], kt * kBKBytes, row_a);
              if (kResidual) tma_load_2d(st + L::kOffR, &maps.r, &full[stage], kt * kBKBytes, row_a);
              tma_load_2d(st + L::kOffB, &maps.w, &full[stage], kt * kBKBytes, row_b);
              tma_load_4d(st + L::kOffSfaX, &maps.sx, &full[stage], 0, 0, kKAtoms * kt, rt_a);
              if (kResidual) tma_load_4d(st + L::kOffSfaR, &maps.sr, &full[stage], 0, 0, kKAtoms * kt, rt_a);
              tma_load_4d(st + L::kOffSfb, &maps.sw, &full[stage], 0, 0, kKAtoms * kt, 2 * nb);
            }
            filled |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          ++fill;
          if (++stage == static_cast<uint32_t>(L::kStages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      // Teardown: every copy armed on this CTA's barriers must have landed (for a
      // pair the leader's barriers also count the peer's copies).
      if (leader)
        for (int s = 0; s < L::kStages; ++s)
          if (filled & (1u << s)) {
            int never = 0;
            mbar_wait(&full[s], (last_parity >> s) & 1u, &never, &g_device_error, kErrWaitDrain);
          }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = unit; tile < p.num_tiles && ok; tile += num_units) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag, &g_device_error, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < p.num_kt; ++kt) {
          // The scale warp's commit for this stage (its copies are in TMEM), and the
          // stage itself (already complete: the scale warp waited for it).
          if (!mbar_wait(&sready[stage], phase, abort_flag, &g_device_error, kErrWaitFull) ||
              !mbar_wait(&full[stage], phase, abort_flag, &g_device_error, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* st = smem + stage * L::kStage;
          const uint32_t sf = tmem + kSfBase + stage * kSfSlot;
          const uint64_t da = operand_desc(st + L::kOffA);
          const uint64_t db = operand_desc(st + L::kOffB);
          // 4 MMAs per operand over the stage's 128 bytes of K, 32 bytes each.  FP4:
          // K = 64, step q uses k-atom q/2 and scale bytes 2(q%2), 2(q%2)+1; FP8: K = 32,
          // step q uses scale byte q of the single k-atom.
#pragma unroll
          for (uint32_t q = 0; q < 4; ++q) {
            const uint32_t id = kFp8 ? q : 2u * (q & 1u), a = kFp8 ? 0u : q >> 1;
            const uint32_t sfa = (sf + kSfaXCol + 4 * a) | (id << 30), sfb = (sf + kSfbCol + 8 * a) | (id << 30);
            const uint32_t acc = (kt | q) != 0 ? 1u : 0u;
            if constexpr (kFp8)
              mma_mxf8_g<kPair>(tmem + kAccCol, da + 2u * q, db + 2u * q, mma_idesc<kPair, true>(id), sfa, sfb, acc);
            else
              mma_mxf4_g<kPair>(tmem + kAccCol, da + 2u * q, db + 2u * q, mma_idesc<kPair, false>(id), sfa, sfb, acc);
          }
          if (kResidual) {
            const uint64_t dr = operand_desc(st + L::kOffR);
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q) {
              const uint32_t id = 2u * (q & 1u), a = q >> 1;
              mma_mxf4_g<kPair>(tmem + kAccCol, dr + 2u * q, db + 2u * q, mma_idesc<kPair, false>(id),
                                (sf + kSfaRCol + 4 * a) | (id << 30), (sf + kSfbCol + 8 * a) | (id << 30), 1u);
            }
          }
          tc_commit_g<kPair>(&empty[stage]);
          if (++stage == static_cast<uint32_t>(L::kStages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_g<kPair>(acc_full);
        acc_phase ^= 1u;
      }
      if (!ok) {
        // Teardown after an abort: wait for the MMAs already issued.
        tc_commit_g<kPair>(drain);
        int never = 0;
        mbar_wait(drain, 0, &never, &g_device_error, kErrWaitDrain);
      }
    }
  } else if (warp == kScaleWarp) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ scale copies
      // Same stage sequence as the MMA issuer.  A stage that has landed also has a
      // free TMEM slot: its refill followed the MMAs' release of the stage (empty),
      // and those were the last MMAs to read the slot.  The copies of stage s are
      // queued while the MMAs of earlier stages still run, so the MMA thread finds
      // them complete and issues nothing but MMAs (issuing both from one thread
      // kept it busy for as long as the tensor pipe took for the MMAs).
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int tile = unit; tile < p.num_tiles && ok; tile += num_units) {
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, &g_device_error, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* st = smem + stage * L::kStage;
          const uint32_t sf = tmem + kSfBase + stage * kSfSlot;
#pragma unroll
          for (uint32_t a = 0; a < kKAtoms; ++a) {
            tmem_copy_32x128b_warpx4_g<kPair>(sf + kSfaXCol + 4 * a, scale_desc(st + L::kOffSfaX + 512 * a));
            if (kResidual)
              tmem_copy_32x128b_warpx4_g<kPair>(sf + kSfaRCol + 4 * a, scale_desc(st + L::kOffSfaR + 512 * a));
            tmem_copy_32x128b_warpx4_g<kPair>(sf + kSfbCol + 8 * a, scale_desc(st + L::kOffSfb + 512 * a));
            tmem_copy_32x128b_warpx4_g<kPair>(sf + kSfbCol + 8 * a + 4,
                                              scale_desc(st + L::kOffSfb + 512 * kKAtoms + 512 * a));
          }
          tc_commit_g<kPair>(&sready[stage]);
          if (++stage == static_cast<uint32_t>(L::kStages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Teardown after an abort: wait for the copies already issued.
        tc_commit_g<kPair>(drain_sf);
        int never = 0;
        mbar_wait(drain_sf, 0, &never, &g_device_error, kErrWaitDrain);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // 8 warps: two per TMEM lane quadrant, each owning 128 of the 256 columns.
    // The accumulator is copied to registers first and released to the MMA warp
    // at once, so converting and storing Y overlaps the next tile's mainloop.
    const int quad = warp & 3;                // TMEM lanes this warp may access: 32*quad .. 32*quad+31
    const int half = (warp - 2) >> 2;         // columns [128*half, 128*half + 128)
    const uint32_t acc_empty_leader = kPair == 2 ? map_to_cta(smem_addr(acc_empty), 0) : 0u;
    uint32_t acc_phase = 0;
    for (int tile = unit; tile < p.num_tiles; tile += num_units) {
      const int mb = tile / p.num_nb;
      const int nb = tile - mb * p.num_nb;
      if (!mbar_wait(acc_full, acc_phase, abort_flag, &g_device_error, kErrWaitAccFull, 2 * kWaitLimitNs)) break;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kAccCol + half * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_load_32x32b_x32(taddr + 32 * c, v[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair == 2) mbar_arrive_remote(acc_empty_leader);
        else mbar_arrive(acc_empty);
      }
      acc_phase ^= 1u;

      const int row = (mb * kPair + static_cast<int>(rank)) * kBM + quad * 32 + lane;
      const int col0 = nb * kBN + half * 128;
      if constexpr (kTransOut) {
        // Y^T [N][M]: for each column the warp's 32 lanes hold 32 consecutive rows,
        // so one store per column writes 32 neighbouring elements of a row of Y^T.
        if (row < p.M) {
#pragma unroll
          for (int i = 0; i < 128; ++i) {
            if (col0 + i < p.N) {
              const float f = __uint_as_float(v[i >> 5][i & 31]);
              const int64_t off = static_cast<int64_t>(col0 + i) * p.M + row;
              if (kBf16Out) static_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(f);
              else static_cast<float*>(p.y)[off] = f;
            }
          }
        }
      } else if (row < p.M) {
        if (kBf16Out) {
          __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (col0 + 8 * i < p.N) {
              uint32_t pw[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int e = 8 * i + 2 * h;
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[e >> 5][e & 31]),
                                                          __uint_as_float(v[(e + 1) >> 5][(e + 1) & 31]));
                pw[h] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(yrow + 8 * i) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            }
          }
        } else {
          float* yrow = static_cast<float*>(p.y) + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = 4 * i;
            if (col0 + e < p.N)
              *reinterpret_cast<uint4*>(yrow + e) =
                  make_uint4(v[e >> 5][e & 31], v[e >> 5][(e & 31) + 1], v[e >> 5][(e & 31) + 2], v[e >> 5][(e & 31) + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  if (kPair == 2) cluster_sync();   // neither CTA leaves while the pair's MMAs or copies may touch it
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_g<kPair>(tmem, kTmemCols);
  }
}

template <int kPair, bool kResidual, bool kBf16Out, bool kTransOut, bool kFp8 = false>
cudaError_t launch_typed(const Maps& maps, const GemmParams& p, int grid, cudaStream_t stream) {
  auto kernel = rfq_gemm_kernel<kPair, kResidual, kBf16Out, kTransOut, kFp8>;
  using L = Layout<kPair, kResidual>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kPair;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait()
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kernel, maps, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int kPair, bool kTransOut>
cudaError_t launch_mode(const Maps& maps, GemmParams p, int64_t M, bool residual, bool y_bf16, bool fp8, int num_sms,
                        cudaStream_t stream) {
  const int64_t num_mb = (M + kBM * kPair - 1) / (kBM * kPair);
  p.num_tiles = static_cast<int>(num_mb * p.num_nb);
  int units = num_sms / kPair;
  if (units > p.num_tiles) units = p.num_tiles;
  const int grid = units * kPair;
  if constexpr (!kTransOut) {
    if (fp8)   // the comparator path: plain MXFP8 (no residual term)
      return y_bf16 ? launch_typed<kPair, false, true, false, true>(maps, p, grid, stream)
                    : launch_typed<kPair, false, false, false, true>(maps, p, grid, stream);
  }
  if (residual)
    return y_bf16 ? launch_typed<kPair, true, true, kTransOut>(maps, p, grid, stream)
                  : launch_typed<kPair, true, false, kTransOut>(maps, p, grid, stream);
  return y_bf16 ? launch_typed<kPair, false, true, kTransOut>(maps, p, grid, stream)
                : launch_typed<kPair, false, false, kTransOut>(maps, p, grid, stream);
}

cudaError_t launch_gemm_impl(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                             const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y,
                             bool y_bf16, bool y_transposed, bool fp8, int num_sms, void* encode_tiled, int skip_fill,
                             cudaStream_t stream) {
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  const bool residual = qr_codes != nullptr;
  // CTA pairs once there are rows for both CTAs of a pair; single CTAs for short M.
  const bool pair = M > kBM;
  const int64_t row_bytes = fp8 ? K : K / 2;
  const uint32_t katoms = fp8 ? 1u : 2u;
  Maps maps;
  if (!encode_code_rows_map(encode, &maps.x, qx_codes, M, row_bytes, kBM)) return cudaErrorInvalidValue;
  if (!encode_code_rows_map(encode, &maps.w, qw_codes, N, row_bytes, pair ? kBN / 2 : kBN))
    return cudaErrorInvalidValue;
  if (!encode_scales_map(encode, &maps.sx, qx_scales, M, K, 1, katoms)) return cudaErrorInvalidValue;
  if (!encode_scales_map(encode, &maps.sw, qw_scales, N, K, 2, katoms)) return cudaErrorInvalidValue;
  if (residual) {
    if (!encode_code_rows_map(encode, &maps.r, qr_codes, M, row_bytes, kBM)) return cudaErrorInvalidValue;
    if (!encode_scales_map(encode, &maps.sr, qr_scales, M, K, 1, katoms)) return cudaErrorInvalidValue;
  } else {
    maps.r = maps.x;
    maps.sr = maps.sx;
  }
  GemmParams p;
  p.y = y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  const int64_t stage_k = fp8 ? 128 : kBK;   // 128 bytes of codes per row per stage
  p.num_kt = static_cast<int>((K + stage_k - 1) / stage_k);
  p.num_nb = static_cast<int>((N + kBN - 1) / kBN);
  p.num_tiles = 0;
  p.skip_fill = skip_fill;
  if (y_transposed)
    return pair ? launch_mode<2, true>(maps, p, M, residual, y_bf16, false, num_sms, stream)
                : launch_mode<1, true>(maps, p, M, residual, y_bf16, false, num_sms, stream);
  return pair ? launch_mode<2, false>(maps, p, M, residual, y_bf16, fp8, num_sms, stream)
              : launch_mode<1, false>(maps, p, M, residual, y_bf16, fp8, num_sms, stream);
}

// ---------------------------------------------------------------- tensor-core rate probe
// The MMAs of one RFQ GEMM stage issued back to back on operands that stay in
// shared memory: no TMA, no epilogue, no pipeline waits.  What it measures is the
// rate at which the tensor cores retire exactly the instruction shapes
// rfq_gemm_kernel issues (kind::mxf4.block_scale, M = 128 * kPair, N = 256,
// K = 64; or kind::mxf8f6f4, K = 32), i.e. the ceiling the GEMM's roofline
// fraction is measured against.  Per iteration: 4 MMAs on the A tile and 4 on
// the R tile against the same B tile, the RFQ stage's pattern.  The clock64()
// cycles of the issuing thread (first MMA issued -> all MMAs complete) go to
// cycles[cluster]; the caller times the launch with events as well.
constexpr int kProbeThreads = 128;

template <int kPair>
struct ProbeLayout {
  static constexpr uint32_t kATile = kBM * kBKBytes;             // 16 KiB
  static constexpr uint32_t kBTile = (kBN / kPair) * kBKBytes;   // 16 or 32 KiB
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffR = kATile;
  static constexpr uint32_t kOffB = 2 * kATile;
  static constexpr uint32_t kOffSf = kOffB + kBTile;             // 4 scale atoms of 512 bytes
  static constexpr uint32_t kOffBar = kOffSf + 2048;
  // More shared memory than the operands need, so that no two probe CTAs share an
  // SM (each must have the SM's tensor core to itself).
  static constexpr uint32_t kSmem = 160u * 1024u;
  static_assert(kOffBar + 64 + 1024 <= kSmem, "probe layout exceeds its shared memory");
};

template <int kPair, bool kFp8>
__global__ void __launch_bounds__(kProbeThreads, 1)
    rfq_mma_rate_kernel(int iters, unsigned long long* cycles) {
  using L = ProbeLayout<kPair>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = kPair == 2 ? cluster_cta_rank() : 0u;

  // Operands: a fixed pseudo-random byte pattern (every E2M1 nibble is a number;
  // E4M3 bytes are masked off the NaN codes), scale bytes 127 (2^0).
  for (uint32_t i = threadIdx.x; i < L::kOffSf / 4; i += kProbeThreads) {
    uint32_t h = (i + 1u) * 2654435761u;
    h ^= h >> 15;
    reinterpret_cast<uint32_t*>(smem)[i] = kFp8 ? (h & 0x77777777u) : h;
  }
  for (uint32_t i = threadIdx.x; i < 2048 / 4; i += kProbeThreads)
    reinterpret_cast<uint32_t*>(smem + L::kOffSf)[i] = 0x7F7F7F7Fu;
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_g<kPair>(tmem_slot, kTmemCols);
    tmem_relinquish_g<kPair>();
  }
  tc_fence_before();
  if (kPair == 2) cluster_sync();   // both CTAs' operands and barriers are ready
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0 && rank == 0) {
    const uint32_t sf = tmem + kSfBase;
#pragma unroll
    for (uint32_t a = 0; a < 4; ++a)
      tmem_copy_32x128b_warpx4_g<kPair>(sf + 4 * a, scale_desc(smem + L::kOffSf + 512 * a));
    const uint64_t da = operand_desc(smem + L::kOffA);
    const uint64_t dr = operand_desc(smem + L::kOffR);
    const uint64_t db = operand_desc(smem + L::kOffB);
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (uint32_t q = 0; q < 4; ++q) {
        const uint32_t id = kFp8 ? q : 2u * (q & 1u);
        const uint32_t sfa = sf | (id << 30), sfb = (sf + 8) | (id << 30);
        if constexpr (kFp8) mma_mxf8_g<kPair>(tmem, da + 2u * q, db + 2u * q, mma_idesc<kPair, true>(id), sfa, sfb, 1u);
        else mma_mxf4_g<kPair>(tmem, da + 2u * q, db + 2u * q, mma_idesc<kPair, false>(id), sfa, sfb, 1u);
      }
#pragma unroll
      for (uint32_t q = 0; q < 4; ++q) {
        const uint32_t id = kFp8 ? q : 2u * (q & 1u);
        const uint32_t sfa = (sf + 4) | (id << 30), sfb = (sf + 8) | (id << 30);
        if constexpr (kFp8) mma_mxf8_g<kPair>(tmem, dr + 2u * q, db + 2u * q, mma_idesc<kPair, true>(id), sfa, sfb, 1u);
        else mma_mxf4_g<kPair>(tmem, dr + 2u * q, db + 2u * q, mma_idesc<kPair, false>(id), sfa, sfb, 1u);
      }
    }
    tc_commit_g<kPair>(done);
    int never = 0;
    mbar_wait(done, 0, &never, &g_device_error, kErrWaitDrain, 2 * kWaitLimitNs);
    cycles[blockIdx.x / kPair] = clock64() - t0;   // grid = clusters x kPair <= cycles_len x kPair
  } else if (threadIdx.x == 0) {
    int never = 0;   // the peer's shared memory stays in use until the leader's MMAs complete
    mbar_wait(done, 0, &never, &g_device_error, kErrWaitDrain, 2 * kWaitLimitNs);
  }
  tc_fence_before();
  if (kPair == 2) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_g<kPair>(tmem, kTmemCols);
  }
}

template <int kPair, bool kFp8>
cudaError_t launch_probe(int iters, unsigned long long* cycles, int max_clusters, int* clusters_used,
                         cudaStream_t stream) {
  auto kernel = rfq_mma_rate_kernel<kPair, kFp8>;
  using L = ProbeLayout<kPair>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max_clusters * kPair);
  cfg.blockDim = dim3(kProbeThreads);
  cfg.dynamicSmemBytes = L::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kPair;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Only as many clusters as can be resident at once (one CTA per SM): a cluster that
  // waited for a free SM pair would only add a second wave to the event time.
  int resident = 0;
  e = cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg);
  if (e != cudaSuccess) return e;
  if (resident < 1) return cudaErrorInvalidConfiguration;
  const int clusters = resident < max_clusters ? resident : max_clusters;
  cfg.gridDim = dim3(clusters * kPair);
  *clusters_used = clusters;
  e = cudaLaunchKernelEx(&cfg, kernel, iters, cycles);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                        const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y,
                        bool y_bf16, bool y_transposed, int num_sms, void* encode_tiled, int skip_fill,
                        cudaStream_t stream) {
  return launch_gemm_impl(qx_codes, qx_scales, qr_codes, qr_scales, qw_codes, qw_scales, M, N, K, y, y_bf16,
                          y_transposed, false, num_sms, encode_tiled, skip_fill, stream);
}

cudaError_t launch_gemm_mxfp8(const void* qx_codes, const void* qx_scales, const void* qw_codes,
                              const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y, bool y_bf16,
                              int num_sms, void* encode_tiled, cudaStream_t stream) {
  return launch_gemm_impl(qx_codes, qx_scales, nullptr, nullptr, qw_codes, qw_scales, M, N, K, y, y_bf16, false,
                          true, num_sms, encode_tiled, -1, stream);
}

cudaError_t launch_mma_rate_probe(int variant, int iters, unsigned long long* cycles, int max_clusters,
                                  int* clusters_used, cudaStream_t stream) {
  switch (variant) {
    case 0: return launch_probe<2, false>(iters, cycles, max_clusters, clusters_used, stream);
    case 1: return launch_probe<1, false>(iters, cycles, max_clusters, clusters_used, stream);
    case 2: return launch_probe<2, true>(iters, cycles, max_clusters, clusters_used, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_and_clear_device_error(unsigned int* value) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace rfq

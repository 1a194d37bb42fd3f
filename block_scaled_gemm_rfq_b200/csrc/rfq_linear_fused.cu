// rfq_linear_fused.cu -- the RFQ linear layer in one kernel for short batches
// (M <= 64 rows of X): the quantizer runs in the GEMM's producer warps; and the
// same kernel on pre-quantized operands, the short-batch GEMM (M <= 256).
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): X is quantized to FP4, its residual
// R = X - DQ(Q(X)) is quantized again and its product added up inside the
// GEMM.  "QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs" (section 4,
// the fused rotate -> quantize -> low-precision matmul kernel) is prior art for
// running the activation quantizer inside the matmul kernel.
//
// With few rows of X the two-kernel path (quantize, then the tiled GEMM) is
// bound by fixed costs and by parallelism: M <= 128 rows give one 128-row tile
// per 256 columns of Y, so a 4096-column layer keeps 16 SMs busy.  Here the
// roles of the operands swap and K is split across a cluster:
//
//     Y^T[n0 : n0+128, :] = sum over cluster ranks s of  QW[n0 : n0+128, K_s] . (QX + QR)[:, K_s]^T
//
//   * MMA A = a 128-row tile of the pre-quantized weight (TMA, 128-byte swizzle),
//     MMA B = all Mp = ceil(M/16)*16 rows of Q(X) / Q(R), MMA N = Mp;
//   * a cluster of S CTAs shares one weight tile, CTA s taking a contiguous
//     range K_s of the k-tiles (256 elements each);
//   * warp 0 streams, per stage, the bf16 rows of X for the k-tile (4 boxes of
//     Mp rows x 64 elements, 128-byte swizzle; rows past M read as zeros) and
//     the weight tile with its scale atoms, all with TMA, kStages ahead;
//   * warps 2..9 (2..17 for 17-32 rows) quantize each 32-element block of the staged X with the same
//     arithmetic as the stand-alone quantizer and write the codes into the
//     swizzled B-operand tile and the E8M0 bytes into the stage's scale atoms in
//     shared memory -- Q(X) and Q(R) never reach global memory;
//   * warp 1 copies the stage's scale atoms to TMEM and issues the MMAs: Q(R)'s
//     rows are stacked under Q(X)'s in the B tile (rows [0, Mp) and [r0, r0 + Mp),
//     r0 = cap or 128), so 4 MMAs of N = r0 + Mp give QW.QX in accumulator columns
//     [0, Mp) and QW.QR in [r0, r0 + Mp), added up by the epilogue (without the
//     residual, 4 MMAs of N = Mp);
//   * above 128 rows (pre-quantized operands), X is taken in blocks of 128 rows,
//     one grid row per block and weight tile, so each CTA's partial tile covers
//     128 rows;
//   * the partial accumulators of the S CTAs are summed through distributed
//     shared memory in rank order (deterministic), each CTA reducing and
//     storing 1/S of the tile.
// Every mbarrier wait is bounded; after a timeout every thread still reaches the
// same cluster barriers, so a failure ends the kernel with an error code.  No
// TMA multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "rfq_internal.h"
#include "rfq_mxfp4.cuh"
#include "rfq_ptx.cuh"
#include "rfq_tmap.h"

namespace rfq {

__device__ unsigned int g_fused_error = 0;

namespace {

constexpr int kBN = 128;                  // weight rows per tile = MMA M = columns of Y per tile
constexpr int kBK = 256;                  // K per stage
constexpr int kBKBytes = kBK / 2;         // 128 bytes of codes per row per stage
// Warps 2 .. 2 + kQW quantize (bf16 input) and then run the epilogue: 16 of them for
// 17-32 rows, 8 otherwise, so that a quantization round covers two k-tiles with one
// block per thread for 16 and for 32 rows.  (Rounds of one k-tile for 32 rows: 9.2 us
// per layer at M = 32 against 8.8; one round of four k-tiles for 16 rows: 8.1 against
// 7.1 us, the MMAs waiting for all four stages of X.)  Warp 0 issues TMA, warp 1 MMAs.
template <int kQW>
struct FusedWarps {
  static constexpr int kQT = kQW * 32;
  static constexpr int kThreads = 64 + kQT;
};
constexpr int kMaxSplit = 8;              // portable cluster size
constexpr int kMaxDevices = 64;
constexpr unsigned int kErrWaitQuantX = 7;   // a quantizer warp waiting for its staged X

// Shared memory and tensor memory of one CTA for at most kCap rows of X.
//   kPreQ = false (kCap = 32 or 64): X arrives as bf16 and the quantizer warps
//     write Q(X), Q(R) into the stage;
//   kPreQ = true (kCap = 64 or 128): Q(X), Q(R) codes and scale atoms, written
//     before by the stand-alone quantizer, arrive by TMA like the weight tile (the
//     short-batch GEMM: 32 < M <= 256, or any rfq_gemm call with few tiles; above
//     128 rows each CTA takes one 128-row block of X); with up to 64 rows a stage
//     is 43 KiB (35 without the residual), with 128 rows 51 KiB; four in flight.
template <int kCap, bool kPreQ, bool kResidual, int kQW = 8>
struct FusedLayout {
  static_assert(kCap <= 128, "one 128-row scale atom per term and k-atom");
  // With the residual, Q(R)'s rows are stacked under Q(X)'s in one B operand, Q(R)
  // from B row kRRow (a whole number of 8-row swizzle groups): kCap when the quantizer
  // warps build both terms' scales as one atom; 128 with pre-quantized operands, so
  // that Q(R)'s own scale atom is copied to TMEM 4 columns after Q(X)'s (a tcgen05.cp
  // 32x128b destination must start on a multiple of 4 columns).  B rows between the
  // two terms are never read back.
  static constexpr int kRRow = kPreQ ? 128 : kCap;
  static constexpr int kXRows = kResidual ? kRRow : kCap;            // B rows before Q(R)'s
  static constexpr int kStages = kPreQ ? 4 : (kCap <= 32 ? 4 : 3);
  static constexpr uint32_t kBoxBytes = kPreQ ? 0 : kCap * 128;      // one staged box: kCap rows x 64 bf16
  static constexpr uint32_t kOffW = 0;                               // 128 x 128 B of weight codes
  static constexpr uint32_t kOffXs = kOffW + kBN * kBKBytes;         // staged X: 4 boxes (kPreQ: none)
  static constexpr uint32_t kOffX = kOffXs + 4 * kBoxBytes;          // Q(X) codes: kCap x 128 B
  static constexpr uint32_t kOffR = kOffX + kXRows * kBKBytes;       // Q(R) codes (residual kernels)
  static constexpr uint32_t kOffSfw = kOffR + (kResidual ? kCap : 0) * kBKBytes;   // 2 k-atoms of 512 B
  static constexpr uint32_t kOffSfx = kOffSfw + 1024;                // the activation's 128-row atom, 2 k-atoms
  static constexpr uint32_t kOffSfr = kOffSfx + 1024;                // Q(R)'s (pre-quantized residual)
  static constexpr uint32_t kStage = kOffSfr + 1024;
  // The split-K partial tile ([kCap][128] fp32) reuses stage 0's staged X, or,
  // with kPreQ, the ring: both are dead once the accumulator is complete.
  static constexpr uint32_t kOffRed = kPreQ ? 0 : kOffXs;
  static constexpr uint32_t kOffBar = kStages * kStage;
  // At least 120 KiB, so that one CTA runs per SM: two co-resident CTAs would share the
  // SM's tensor core and TMA unit while the split model counts them as two SMs (the
  // 27 KiB stages of the 64-row kernel without the residual allowed two, and the model
  // then picked twice the split: 14.2 instead of 8.8 us per layer at M = 64).
  static constexpr uint32_t kSmem = kOffBar + 256 + 1024 > 120u * 1024u ? kOffBar + 256 + 1024 : 120u * 1024u;
  // Tensor memory: the accumulator in columns [0, N) (N = B rows, at most kRRow +
  // kCap), then one scale slot per stage: +0 QW (2 k-atoms x 4 columns), and the B
  // scales of k-atom a from +kSfX + 8a (4 columns per 128 B rows).
  static constexpr uint32_t kSfBase = kPreQ ? 256 : 128;
  static constexpr uint32_t kSfSlot = kPreQ ? 64 : 32;
  static constexpr uint32_t kSfW = 0, kSfX = 8;
  static constexpr uint32_t kTmemCols = kPreQ ? 512 : 256;
  // Per thread and round: blocks (kCap rows x 8 blocks of one stage, or several
  // stages of 16 rows) over the quantizer threads.
  static constexpr int kQT = FusedWarps<kQW>::kQT;
  static constexpr int kSlots = kCap * 8 / kQT > 0 ? kCap * 8 / kQT : 1;
  static_assert(kOffRed + kCap * kBN * 4 <= (kPreQ ? kStages * kStage : kStage), "partial tile must fit");
  static_assert(kStage % 1024 == 0 && kBoxBytes % 1024 == 0, "swizzled tiles need 1 KiB alignment");
  static_assert(kSmem <= 232448, "exceeds the 227 KiB shared-memory limit");
  static_assert(kSfX + 16 <= kSfSlot, "scale slot too small");
  // tcgen05.cp 32x128b destinations start on a multiple of 4 TMEM columns
  static_assert(kSfBase % 4 == 0 && kSfSlot % 4 == 0 && kSfW % 4 == 0 && kSfX % 4 == 0, "scale copy alignment");
  // the B operand (Q(X) rows, then Q(R)'s from kRRow) is at most N = 256 rows and stays in the stage
  static_assert((kResidual ? kRRow + kCap : kCap) <= 256, "MMA N exceeds 256");
  static_assert(kOffX + (kResidual ? kRRow + kCap : kCap) * kBKBytes <= kOffSfw, "B operand leaves its area");
  static_assert(kSfBase >= static_cast<uint32_t>(kXRows + (kResidual ? kCap : 0)) &&
                    kSfBase + kStages * kSfSlot <= kTmemCols,
                "scale slots exceed TMEM");
  static_assert((4 * kStages + 2) * 8 + 8 <= 256, "barrier area too small");
};

struct FusedParams {
  void* y;             // [M][N], fp32 or bf16
  int M;
  int N;
  int K;
  int Kb;              // K / 32
  int Mp;              // MMA N: M rounded up to 16
  int num_kt;          // k-tiles of 256
  int group;           // k-tiles quantized per round
  uint32_t act_bytes;  // kPreQ: bytes of Q(X) [+ Q(R)] codes and scale atoms per stage
  int row_blocks;      // blocks of X's rows, each a grid row of its own (1 unless kPreQ and M > block_rows)
  int block_rows;      // rows per block: 64 or 128 (a multiple of 64: a block lies inside one scale atom)
  int skip_fill;       // kPreQ fault injection: CTA (0, 0) skips this stage fill (-1 = off)
};

struct FusedMaps {
  CUtensorMap x;       // bf16 [M][K], box 64 elements x Mp rows, 128-byte swizzle, zero fill
  CUtensorMap w;       // codes [N][K/2], box 128 B x 128 rows, 128-byte swizzle
  CUtensorMap sw;      // scales [row tiles][k atoms][2][256 B], box 2 k-atoms x 1 row tile
  CUtensorMap qx, qr;  // kPreQ: codes [M][K/2], box 128 B x Mp rows, 128-byte swizzle
  CUtensorMap sx, sr;  // kPreQ: scales, box 2 k-atoms x ceil(Mp / 128) row tiles
};

__device__ __forceinline__ uint64_t operand_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((1024ull >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint64_t scale_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull) | ((128ull >> 4) << 32) | (1ull << 46);
}

// kind::mxf4, E2M1 x E2M1, K-major both, M = 128, N = Mp, E8M0 scales.
__device__ __forceinline__ uint32_t fused_idesc(uint32_t idesc_n, uint32_t sf_id) {
  return (sf_id << 4) | (1u << 7) | (1u << 10) | idesc_n | (1u << 23) | (uint32_t(kBN >> 4) << 24) | (sf_id << 29);
}

template <int kCap, bool kResidual, bool kBf16Out, bool kPreQ, int kQW>
__global__ void __launch_bounds__(FusedWarps<kQW>::kThreads, 1)
    rfq_linear_fused_kernel(const __grid_constant__ FusedMaps maps, const FusedParams p) {
  using L = FusedLayout<kCap, kPreQ, kResidual, kQW>;
  constexpr int kStages = L::kStages;
  constexpr int kQWarps = kQW;
  constexpr int kQThreads = FusedWarps<kQW>::kQT;
  constexpr int kRRow = L::kRRow;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + L::kOffBar);   // staged X landed (tx)
  uint64_t* wfull = xfull + kStages;                                   // weight tile landed (tx)
  uint64_t* qfull = wfull + kStages;                                   // Q(X), Q(R) written (quantizer warps)
  uint64_t* empty = qfull + kStages;                                   // stage consumed by the MMAs
  uint64_t* acc_full = empty + kStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = static_cast<int>(gridDim.x);              // cluster size along K
  const uint32_t rank = cluster_cta_rank();                   // = blockIdx.x
  // Grid rows: weight tiles x row blocks of X (row block fastest, so the clusters of
  // neighbouring rows share the weight tile in L2).  This CTA's rows of X: [m0, m0 + mp),
  // mp a multiple of 16; rows at and past M (m_end) are zero-filled and not stored.  A
  // block lies inside one 128-row scale atom (row tile rt); its rows go to the B rows
  // they have in that atom (from boff = m0 % 128), so that the atom, copied whole to TMEM,
  // lines up with them: B rows [0, boff) are never read back.
  const int rb = static_cast<int>(blockIdx.y) % p.row_blocks;
  const int tile = static_cast<int>(blockIdx.y) / p.row_blocks;
  const int m0 = rb * p.block_rows;
  const int mp = min(p.Mp - m0, p.block_rows);
  const int m_end = p.M - m0;
  const int rt = m0 >> 7;
  const int boff = m0 & 127;
  const int n0 = tile * kBN;
  const int kt0 = static_cast<int>(rank) * p.num_kt / split;
  const int nk = (static_cast<int>(rank) + 1) * p.num_kt / split - kt0;   // >= 1: split <= num_kt

  // TMA producer state (warp 0, lane 0).  It initializes the barriers and issues
  // the first stages' copies before the CTA-wide barrier, so their latency
  // overlaps the TMEM allocation and the other warps' start.
  uint32_t filled = 0, last_parity = 0;
  int issued = 0;
  const uint32_t x_bytes = 4u * static_cast<uint32_t>(p.Mp) * 128u;
  auto issue_stage = [&](int i) {
    const int stage = i % kStages;
    const uint32_t phase = static_cast<uint32_t>(i / kStages) & 1u;
    uint8_t* st = smem + stage * L::kStage;
    const int kt = kt0 + i;
    if constexpr (kPreQ) {
      if (i == p.skip_fill && blockIdx.x == 0 && blockIdx.y == 0) return;   // fault injection (tests)
      // weight tile and the activation's codes and scale atoms, all on one barrier
      mbar_arrive_expect_tx(&wfull[stage], kBN * kBKBytes + 1024u + p.act_bytes);
      tma_load_2d(st + L::kOffX + boff * kBKBytes, &maps.qx, &wfull[stage], kt * kBKBytes, m0);
      tma_load_4d(st + L::kOffSfx, &maps.sx, &wfull[stage], 0, 0, 2 * kt, rt);
      if (kResidual) {
        tma_load_2d(st + L::kOffR + boff * kBKBytes, &maps.qr, &wfull[stage], kt * kBKBytes, m0);
        tma_load_4d(st + L::kOffSfr, &maps.sr, &wfull[stage], 0, 0, 2 * kt, rt);
      }
    } else {
      mbar_arrive_expect_tx(&xfull[stage], x_bytes);
#pragma unroll
      for (int b = 0; b < 4; ++b)
        tma_load_2d(st + L::kOffXs + b * L::kBoxBytes, &maps.x, &xfull[stage], kt * kBK + 64 * b, 0);
      mbar_arrive_expect_tx(&wfull[stage], kBN * kBKBytes + 1024u);
    }
    tma_load_2d(st + L::kOffW, &maps.w, &wfull[stage], kt * kBKBytes, n0);
    tma_load_4d(st + L::kOffSfw, &maps.sw, &wfull[stage], 0, 0, 2 * kt, tile);
    filled |= 1u << stage;
    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&wfull[s], 1);
      mbar_init(&qfull[s], kQWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if constexpr (kPreQ) {
      prefetch_tmap(&maps.qx);
      prefetch_tmap(&maps.sx);
      if (kResidual) {
        prefetch_tmap(&maps.qr);
        prefetch_tmap(&maps.sr);
      }
    } else {
      prefetch_tmap(&maps.x);
    }
    prefetch_tmap(&maps.w);
    prefetch_tmap(&maps.sw);
    // With pre-quantized operands (after the quantizer on the stream), pull this CTA's
    // slice of the weight into L2 while the previous kernel finishes (a hint; the
    // copies still follow griddepcontrol.wait).  The bf16-input mode, which follows
    // another short layer, measured slower with it.
    if constexpr (kPreQ)
      for (int i = 0; i < nk; ++i) tma_prefetch_2d(&maps.w, (kt0 + i) * kBKBytes, n0);
    griddep_wait();   // X and QW may be written by the previous kernel on the stream
    for (; issued < nk && issued < kStages; ++issued) issue_stage(issued);   // the stages start free
  }
  if (warp == 1) {
    tmem_alloc_g<1>(tmem_slot, L::kTmemCols);
    tmem_relinquish_g<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  griddep_launch_dependents();
  griddep_wait();   // Y may still be read by the previous kernel on the stream
  bool epi_ok = false;   // epilogue warps: the accumulator is complete

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA producer
      // Per stage: X first (the quantizers' input), then the weight tile.
      for (; issued < nk; ++issued) {
        const uint32_t phase = static_cast<uint32_t>(issued / kStages) & 1u;
        if (!mbar_wait(&empty[issued % kStages], phase ^ 1u, abort_flag, &g_fused_error, kErrWaitEmpty)) break;
        issue_stage(issued);
      }
      // Teardown after an abort: the copies armed on this CTA's barriers must
      // land before exit.  (On the normal path the MMAs consumed them all.)
      if (*abort_flag)
        for (int s = 0; s < kStages; ++s)
          if (filled & (1u << s)) {
            int never = 0;
            if (!kPreQ) mbar_wait(&xfull[s], (last_parity >> s) & 1u, &never, &g_fused_error, kErrWaitDrain);
            mbar_wait(&wfull[s], (last_parity >> s) & 1u, &never, &g_fused_error, kErrWaitDrain);
          }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      // N = the B rows: Q(X)'s [boff, boff + mp) and, with the residual, Q(R)'s from kRRow + boff
      const uint32_t idesc_n = static_cast<uint32_t>(((kResidual ? kRRow : 0) + boff + mp) >> 3) << 17;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int stage = i % kStages;
        const uint32_t phase = static_cast<uint32_t>(i / kStages) & 1u;
        if (!mbar_wait(&wfull[stage], phase, abort_flag, &g_fused_error, kErrWaitFull) ||
            (!kPreQ && !mbar_wait(&qfull[stage], phase, abort_flag, &g_fused_error, kErrWaitFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + stage * L::kStage;
        const uint32_t sf = tmem + L::kSfBase + stage * L::kSfSlot;
        constexpr uint32_t kSfW = L::kSfW, kSfX = L::kSfX;
        // Scales: the weight's 2 atoms, and the B scales of k-atom a from column sf +
        // kSfX + 8a (column c holds B rows 32c .. 32c + 31): Q(X)'s atom, and with the
        // residual either the same atom (the quantizer warps write Q(R)'s bytes at rows
        // kRRow = kCap ..) or Q(R)'s own atom 4 columns further (B rows 128 .. 255).
#pragma unroll
        for (uint32_t a = 0; a < 2; ++a) {
          tmem_copy_32x128b_warpx4_g<1>(sf + kSfW + 4 * a, scale_desc(st + L::kOffSfw + 512 * a));
          tmem_copy_32x128b_warpx4_g<1>(sf + kSfX + 8 * a, scale_desc(st + L::kOffSfx + 512 * a));
          if constexpr (kResidual && kPreQ)
            tmem_copy_32x128b_warpx4_g<1>(sf + kSfX + 8 * a + 4, scale_desc(st + L::kOffSfr + 512 * a));
        }
        const uint64_t dw = operand_desc(st + L::kOffW);
        const uint64_t dx = operand_desc(st + L::kOffX);
        // 4 MMAs of K = 64: step q uses k-atom q/2 and scale bytes 2(q%2), 2(q%2)+1.
#pragma unroll
        for (uint32_t q = 0; q < 4; ++q) {
          const uint32_t id = 2u * (q & 1u), a = q >> 1;
          mma_mxf4(tmem, dw + 2u * q, dx + 2u * q, fused_idesc(idesc_n, id), (sf + kSfW + 4 * a) | (id << 30),
                   (sf + kSfX + 8 * a) | (id << 30), (i | static_cast<int>(q)) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[stage]);
      }
      if (ok) {
        tc_commit(acc_full);
        // The MMAs must be complete before TMEM is freed, whatever the epilogue does.
        int never = 0;
        mbar_wait(acc_full, 0, &never, &g_fused_error, kErrWaitDrain);
      } else {
        // Teardown after an abort: wait for the MMAs already issued.
        tc_commit(drain);
        int never = 0;
        mbar_wait(drain, 0, &never, &g_fused_error, kErrWaitDrain);
      }
    }
  } else {
    // ---------------------------------------------------------------- quantizer warps
    // Round r quantizes k-tiles [r*group, r*group + group) of this CTA's range.
    // Flat block index f = slot * kQThreads + qt over (k-tile of the round,
    // block j of the k-tile, row), rows fastest: the 8 lanes of a shared-memory
    // phase read 8 consecutive rows, which the 128-byte swizzle puts in 8
    // distinct bank groups, and write 8 distinct chunks of the B tile.
    const int qt = threadIdx.x - 64;
    const int blocks_per_stage = 8 * p.Mp;
    const int rounds = kPreQ ? 0 : (nk + p.group - 1) / p.group;   // kPreQ: nothing to quantize
    bool ok = true;
    for (int r = 0; r < rounds && ok; ++r) {
      const int i0 = r * p.group;
      const int g_here = min(p.group, nk - i0);
      for (int g = 0; g < g_here && ok; ++g) {
        const int i = i0 + g;
        ok = mbar_wait(&xfull[i % kStages], static_cast<uint32_t>(i / kStages) & 1u, abort_flag, &g_fused_error,
                       kErrWaitQuantX);
      }
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int t = 0; t < L::kSlots; ++t) {
        const int f = t * kQThreads + qt;
        if (f < g_here * blocks_per_stage) {
          const int g = f / blocks_per_stage, rem = f - g * blocks_per_stage;
          const int j = rem / p.Mp, row = rem - j * p.Mp;
          uint8_t* st = smem + ((i0 + g) % kStages) * L::kStage;
          // B-operand tile: row `row`, 16-byte chunk j, 128-byte swizzle.
          const uint32_t code_off = (row >> 3) * 1024u + (row & 7) * 128u + ((j ^ (row & 7)) << 4);
          // Scale atom of k-atom j/4: row at (row % 32) * 16 + (row / 32) * 4, block j % 4.
          const uint32_t sf_off = (j >> 2) * 512u + (row & 31) * 16u + (row >> 5) * 4u + (j & 3);
          uint32_t cx[4] = {0u, 0u, 0u, 0u}, cr[4] = {0u, 0u, 0u, 0u}, sx = 0u, sr = 0u;
          if (row < p.M) {   // rows in [M, Mp) get zero codes and scale byte 0
            // Staged X: box j/2, 128-byte row `row`, 16-byte chunks 4 (j%2) .. +3 XOR (row % 8).
            const uint8_t* src = st + L::kOffXs + (j >> 1) * L::kBoxBytes + row * 128;
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = *reinterpret_cast<const uint4*>(src + ((((j & 1) * 4 + c) ^ (row & 7)) << 4));
              w[4 * c + 0] = v.x;
              w[4 * c + 1] = v.y;
              w[4 * c + 2] = v.z;
              w[4 * c + 3] = v.w;
            }
            quantize_block<kResidual>(w, cx, sx, cr, sr);
          }
          *reinterpret_cast<uint4*>(st + L::kOffX + code_off) = make_uint4(cx[0], cx[1], cx[2], cx[3]);
          st[L::kOffSfx + sf_off] = static_cast<uint8_t>(sx);
          if constexpr (kResidual) {
            // Q(R): B row kRRow + row of the stacked operand, its scale byte in the same atom
            *reinterpret_cast<uint4*>(st + L::kOffR + code_off) = make_uint4(cr[0], cr[1], cr[2], cr[3]);
            const int rr = kRRow + row;
            st[L::kOffSfx + (j >> 2) * 512u + (rr & 31) * 16u + (rr >> 5) * 4u + (j & 3)] = static_cast<uint8_t>(sr);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        for (int g = 0; g < g_here; ++g) mbar_arrive(&qfull[(i0 + g) % kStages]);
    }

    // ---------------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes 32 (w % 4) .. +31 (weight rows = columns of Y);
    // the warps of a lane quadrant alternate over 8-column chunks (rows of X).
    // With a K split the accumulator goes, as [Mp][128] fp32, to this CTA's
    // receive area for the cluster reduction below.
    epi_ok = mbar_wait(acc_full, 0, abort_flag, &g_fused_error, kErrWaitAccFull, 2 * kWaitLimitNs);
    if (__all_sync(0xffffffffu, epi_ok)) {
      tc_fence_after();
      const int quad = warp & 3;
      const int half = (warp - 2) >> 2;   // the warps of a lane quadrant take turns over 8-column chunks
      const int n_local = quad * 32 + lane;
      const int n = n0 + n_local;
      for (int c = half; c < mp / 8; c += kQWarps / 4) {
        uint32_t v[8];
        tmem_load_32x32b_x8(tmem + (static_cast<uint32_t>(quad * 32) << 16) + boff + 8 * c, v);
        if constexpr (kResidual) {   // + the Q(R) term, kRRow columns further
          uint32_t vr[8];
          tmem_load_32x32b_x8(tmem + (static_cast<uint32_t>(quad * 32) << 16) + kRRow + boff + 8 * c, vr);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(vr[e]));
        }
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int m = 8 * c + e;
          if (split > 1) {
            red[m * kBN + n_local] = __uint_as_float(v[e]);
          } else if (m < m_end && n < p.N) {
            if (kBf16Out)
              static_cast<__nv_bfloat16*>(p.y)[static_cast<int64_t>(m0 + m) * p.N + n] = __float2bfloat16_rn(__uint_as_float(v[e]));
            else
              static_cast<float*>(p.y)[static_cast<int64_t>(m0 + m) * p.N + n] = __uint_as_float(v[e]);
          }
        }
      }
    }
  }
  __syncwarp();

  if (split > 1) {
    // ---------------------------------------------------------------- split-K reduction
    // Every thread of every CTA of the cluster takes part in both barriers, on
    // the error path too.  After the first, CTA s sums its 1/S of the tile over
    // the cluster's partials in rank order (into registers); it arrives on the
    // second as soon as its reads of the peers are done and stores Y while the
    // others finish theirs.  (Pushing the partials to their owners with 4-byte
    // distributed stores instead measured slower; the exchange is bound by the
    // distributed shared-memory bandwidth either way.)
    cluster_sync();
    constexpr int kPer = kCap / 16;            // >= ceil(F / split / kQThreads) for split >= 2 (kQThreads >= 256)
    float4 acc[kPer];
    const int F = mp * (kBN / 4);              // float4 groups in the tile
    const int f_begin = static_cast<int>(rank) * F / split;
    const int f_end = (static_cast<int>(rank) + 1) * F / split;
    const int qt = static_cast<int>(threadIdx.x) - 64;
    const bool reduce = warp >= 2 && !*abort_flag;
    if (reduce) {
      const uint32_t red_addr = smem_addr(red);
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int f = f_begin + qt + t * kQThreads;
        if (f < f_end) {
          acc[t] = ld_shared_cluster_f32x4(map_to_cta(red_addr + 16u * f, 0));
          for (int s = 1; s < split; ++s) {
            const float4 v = ld_shared_cluster_f32x4(map_to_cta(red_addr + 16u * f, s));
            acc[t].x += v.x;
            acc[t].y += v.y;
            acc[t].z += v.z;
            acc[t].w += v.w;
          }
        }
      }
    }
    cluster_arrive();
    if (reduce) {
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int f = f_begin + qt + t * kQThreads;
        const int m = f / (kBN / 4), n = n0 + (f % (kBN / 4)) * 4;
        if (f < f_end && m < m_end && n < p.N) {   // N % 8 == 0: a group of 4 is all in or all out
          const int64_t row = m0 + m;
          if (kBf16Out) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[t].x, acc[t].y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[t].z, acc[t].w);
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.y) + row * p.N + n) =
                make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
          } else {
            *reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * p.N + n) = acc[t];
          }
        }
      }
    }
    cluster_wait();   // no CTA leaves while a peer may still read its partial tile
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_g<1>(tmem, L::kTmemCols);
  }
}

std::atomic<int> g_split_override{0};

template <int kCap, bool kResidual, bool kBf16Out, bool kPreQ = false, int kQW = 8>
cudaError_t launch_typed(const FusedMaps& maps, const FusedParams& p, int tiles, int num_sms, cudaStream_t stream) {
  using L = FusedLayout<kCap, kPreQ, kResidual, kQW>;
  auto kernel = rfq_linear_fused_kernel<kCap, kResidual, kBf16Out, kPreQ, kQW>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(FusedWarps<kQW>::kThreads);
  cfg.dynamicSmemBytes = L::kSmem;
  cfg.stream = stream;
  FusedParams q = p;
  if constexpr (!kPreQ) {
    // A quantization round gives each quantizer thread one block: k-tiles of Mp rows x 8
    // blocks, as many as the threads cover (all four stages of a CTA's range for 16 rows
    // and 16 warps), at most the ring's stages, which must all hold their staged X at once.
    constexpr int kQT = FusedWarps<kQW>::kQT;
    q.group = q.Mp * 8 >= kQT ? 1 : kQT / (q.Mp * 8);
    if (q.group > L::kStages) q.group = L::kStages;
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait()
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;

  // Split of K: more CTAs per weight tile shorten each CTA's k-range but add a
  // fixed cost (X latency, reduction).  Model: time ~ waves x (k-tiles per CTA +
  // 4), waves from the number of clusters of that size that fit at once.
  // Clusters of each size that fit at once, per device (queried once).
  static std::atomic<int> fit[kMaxDevices][kMaxSplit + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  int split = g_split_override.load();
  if (split <= 0) {
    double best = 1e30;
    split = 1;
    for (int s = 1; s <= kMaxSplit && s <= p.num_kt; ++s) {
      int clusters = dev >= 0 ? fit[dev][s].load(std::memory_order_relaxed) : 0;
      if (clusters <= 0) {
        attr[0].val.clusterDim.x = s;
        cfg.gridDim = dim3(s, tiles);
        if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters <= 0) {
          cudaGetLastError();
          clusters = num_sms / s;
        }
        if (dev >= 0) fit[dev][s].store(clusters, std::memory_order_relaxed);
      }
      const int waves = (tiles + clusters - 1) / clusters;
      const double cost = waves * ((p.num_kt + s - 1) / s + 4.0);
      if (cost < best - 1e-9) {
        best = cost;
        split = s;
      }
    }
  }
  if (split > p.num_kt) split = p.num_kt;
  if (split > kMaxSplit) split = kMaxSplit;
  attr[0].val.clusterDim.x = split;
  cfg.gridDim = dim3(split, tiles);
  e = cudaLaunchKernelEx(&cfg, kernel, maps, q);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int kCap, int kQW = 8>
cudaError_t launch_cap(const FusedMaps& maps, const FusedParams& p, int tiles, bool residual, bool y_bf16,
                       int num_sms, cudaStream_t stream) {
  if (residual)
    return y_bf16 ? launch_typed<kCap, true, true, false, kQW>(maps, p, tiles, num_sms, stream)
                  : launch_typed<kCap, true, false, false, kQW>(maps, p, tiles, num_sms, stream);
  return y_bf16 ? launch_typed<kCap, false, true, false, kQW>(maps, p, tiles, num_sms, stream)
                : launch_typed<kCap, false, false, false, kQW>(maps, p, tiles, num_sms, stream);
}

}  // namespace

cudaError_t launch_linear_fused(const void* x, int64_t M, int64_t K, const void* qw_codes, const void* qw_scales,
                                int64_t N, void* y, bool y_bf16, bool residual, int num_sms, void* encode_tiled,
                                cudaStream_t stream) {
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  FusedMaps maps;
  const int64_t Mp = (M + 15) / 16 * 16;
  {
    // X as [M][K] 16-bit elements; box 64 x Mp, 128-byte swizzle, zeros outside.
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(Mp)};
    cuuint32_t elem_strides[2] = {1, 1};
    if (encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box, elem_strides,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!encode_codes_map(encode, &maps.w, qw_codes, N, K, kBN)) return cudaErrorInvalidValue;
  if (!encode_scales_map(encode, &maps.sw, qw_scales, N, K, 1)) return cudaErrorInvalidValue;
  FusedParams p;
  p.y = y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.Kb = static_cast<int>(K / 32);
  p.Mp = static_cast<int>(Mp);
  p.num_kt = static_cast<int>((K + kBK - 1) / kBK);
  p.group = 1;   // set per layout in launch_typed
  p.act_bytes = 0;
  p.row_blocks = 1;
  p.block_rows = p.Mp;
  p.skip_fill = -1;
  maps.qx = maps.qr = maps.w;   // unused without kPreQ
  maps.sx = maps.sr = maps.sw;
  const int tiles = static_cast<int>((N + kBN - 1) / kBN);
  if (p.Mp <= 16) return launch_cap<32, 8>(maps, p, tiles, residual, y_bf16, num_sms, stream);
  return p.Mp <= 32 ? launch_cap<32, 16>(maps, p, tiles, residual, y_bf16, num_sms, stream)
                    : launch_cap<64, 8>(maps, p, tiles, residual, y_bf16, num_sms, stream);
}

cudaError_t launch_gemm_short(const void* qx_codes, const void* qx_scales, const void* qr_codes,
                              const void* qr_scales, const void* qw_codes, const void* qw_scales, int64_t M,
                              int64_t N, int64_t K, void* y, bool y_bf16, int num_sms, void* encode_tiled,
                              int skip_fill, cudaStream_t stream) {
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  const bool residual = qr_codes != nullptr;
  const int64_t Mp = (M + 15) / 16 * 16;
  // Above kBlock rows, X is taken in blocks of kBlock rows, each block a grid row of its
  // own: a CTA's partial tile, and so the split-K exchange through distributed shared
  // memory, covers one block (M = 256, K = N = 4096, layer after layer: 14.1 us with
  // blocks of 128 rows against 17.8 with one 256-row block per CTA, and 15.8 with blocks
  // of 64 rows, where the cluster model then drops the K split: the K loop grows more
  // than the exchange shrinks).
  constexpr int64_t kBlock = 128;
  const bool row_split = Mp > kBlock;
  const uint32_t box_rows = row_split ? static_cast<uint32_t>(kBlock) : static_cast<uint32_t>(Mp);
  const uint32_t row_tiles = 1u;
  FusedMaps maps;
  if (!encode_codes_map(encode, &maps.w, qw_codes, N, K, kBN)) return cudaErrorInvalidValue;
  if (!encode_scales_map(encode, &maps.sw, qw_scales, N, K, 1)) return cudaErrorInvalidValue;
  if (!encode_codes_map(encode, &maps.qx, qx_codes, M, K, box_rows)) return cudaErrorInvalidValue;
  if (!encode_scales_map(encode, &maps.sx, qx_scales, M, K, row_tiles)) return cudaErrorInvalidValue;
  if (residual) {
    if (!encode_codes_map(encode, &maps.qr, qr_codes, M, K, box_rows)) return cudaErrorInvalidValue;
    if (!encode_scales_map(encode, &maps.sr, qr_scales, M, K, row_tiles)) return cudaErrorInvalidValue;
  } else {
    maps.qr = maps.qx;
    maps.sr = maps.sx;
  }
  maps.x = maps.w;   // unused with kPreQ
  FusedParams p;
  p.y = y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.Kb = static_cast<int>(K / 32);
  p.Mp = static_cast<int>(Mp);
  p.num_kt = static_cast<int>((K + kBK - 1) / kBK);
  p.group = 1;
  // per stage: a box of rows x 128 B of codes and row_tiles x 2 k-atoms of scales, per term
  p.act_bytes = (box_rows * kBKBytes + row_tiles * 1024u) * (residual ? 2u : 1u);
  p.row_blocks = row_split ? static_cast<int>((Mp + kBlock - 1) / kBlock) : 1;
  p.block_rows = row_split ? static_cast<int>(kBlock) : static_cast<int>(Mp);
  p.skip_fill = skip_fill;
  const int tiles = static_cast<int>((N + kBN - 1) / kBN) * p.row_blocks;
  // Up to 64 rows: four stages of 43 KiB (measured 10.3 against 11.5 us per layer
  // at M = 64, K = N = 4096, with a two-stage 85 KiB layout, before the terms were
  // stacked); otherwise four of 51 KiB per block of 128 rows.
  if (Mp <= 64) {
    if (residual)
      return y_bf16 ? launch_typed<64, true, true, true>(maps, p, tiles, num_sms, stream)
                    : launch_typed<64, true, false, true>(maps, p, tiles, num_sms, stream);
    return y_bf16 ? launch_typed<64, false, true, true>(maps, p, tiles, num_sms, stream)
                  : launch_typed<64, false, false, true>(maps, p, tiles, num_sms, stream);
  }
  if (residual)
    return y_bf16 ? launch_typed<128, true, true, true>(maps, p, tiles, num_sms, stream)
                  : launch_typed<128, true, false, true>(maps, p, tiles, num_sms, stream);
  return y_bf16 ? launch_typed<128, false, true, true>(maps, p, tiles, num_sms, stream)
                : launch_typed<128, false, false, true>(maps, p, tiles, num_sms, stream);
}

void set_fused_split_override(int split) { g_split_override.store(split < 0 ? 0 : split); }

cudaError_t read_and_clear_fused_error(unsigned int* value) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(value, g_fused_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_fused_error, &zero, sizeof(unsigned int));
}

}  // namespace rfq

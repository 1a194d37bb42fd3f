// rfq_quantize.cu -- kernel 1: the fused single-pass RFQ quantizer for sm_100a.
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): X is quantized to FP4 (here MXFP4), the
// full quantization error R = X - DQ(Q(X)) is formed, and R is quantized again by
// the same rule (a second low-bit quantization path).  This kernel does all of
// it in one pass over X: every bf16 element is read from HBM exactly once and the
// codes and E8M0 scales of Q(X) and Q(R) are written once, the scales directly in
// the layout the block-scaled tensor-core MMA consumes.  R lives only in
// registers, in fp32, in which it is exact (rfq_mxfp4.cuh).
//
// Work decomposition (HBM-bound streaming kernel, no tensor cores):
//   * X is viewed as a flat sequence of 32-element blocks (64 bytes each; a block
//     never crosses a row because K is a multiple of 32);
//   * a warp owns spans of 32 consecutive blocks (2 KiB) and each lane one block,
//     so the block amax needs no shuffles;
//   * every warp keeps kStages spans in flight with its own TMA ring (2-D tensor
//     map over [blocks][64 bytes], 64-byte swizzle so that the lanes' 16-byte
//     shared-memory reads are bank-conflict free) and mbarriers with bounded waits;
//   * pairs of fp32 values go through packed f32x2 multiplies, codes through
//     cvt.rn.satfinite.e2m1x2.f32 (2 per instruction) and back through
//     cvt.rn.f16x2.e2m1x2 for the residual, which packed f32x2 FMAs form;
//   * scale bytes: when K is a multiple of 128 the 4 lanes holding blocks
//     4j..4j+3 of a row gather them into one 32-bit word of the MMA layout;
//     otherwise each lane stores its byte.  The padding bytes of the scale
//     arrays (rows up to a multiple of 128, blocks up to a multiple of 4) are
//     zeroed by the same launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rfq_internal.h"
#include "rfq_mxfp4.cuh"
#include "rfq_ptx.cuh"
#include "rfq_tmap.h"

namespace rfq {

__device__ unsigned int g_quant_error = 0;

namespace {

// Launch shape and ring (compile-time; the defaults are the tuned configuration).
#ifndef RFQ_Q_STAGES
#define RFQ_Q_STAGES 2
#endif
#ifndef RFQ_Q_SUB
#define RFQ_Q_SUB 1
#endif
#ifndef RFQ_Q_WARPS
#define RFQ_Q_WARPS 8
#endif
#ifndef RFQ_Q_CTAS_PER_SM
#define RFQ_Q_CTAS_PER_SM 3
#endif
constexpr int kWarps = RFQ_Q_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = RFQ_Q_STAGES;            // spans in flight per warp
constexpr int kSub = RFQ_Q_SUB;                  // blocks per lane per span
constexpr int kSpanBlocks = 32 * kSub;
constexpr int kSpanBytes = kSpanBlocks * 64;
constexpr unsigned int kErrQuantWait = 6;        // a warp's wait for its TMA span ran out
constexpr uint32_t kSmemBytes = kWarps * kStages * kSpanBytes + kWarps * kStages * 8 + 1024;

// Indices are 32-bit: the C ABI limits a matrix to fewer than 2^31 blocks and
// its scale array to fewer than 2^32 bytes.
struct QuantParams {
  uint8_t* qx_codes;
  uint8_t* qx_scales;
  uint8_t* qr_codes;
  uint8_t* qr_scales;
  uint32_t M;             // rows
  uint32_t Kb;            // 32-element blocks per row
  uint32_t kb4_per_tile;  // 4-block words per row in the scale layout = ceil(Kb / 4)
  uint32_t rows_pad;      // ceil(M / 128) * 128
  uint32_t total_blocks;  // M * Kb
  uint32_t num_spans;     // ceil(total_blocks / span)
};

// Byte offset in the MMA scale layout of (row r, 4-block word kb4): atoms of 128
// rows x 4 blocks with the block-tile index fastest; row r inside its atom at
// (r % 32) * 16 + ((r / 32) % 4) * 4.
__device__ __forceinline__ uint32_t scale_word_offset(uint32_t r, uint32_t kb4, uint32_t kb4_per_tile) {
  return ((r >> 7) * kb4_per_tile + kb4) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u;
}

// Store one block's scale byte: as a gathered 32-bit word of 4 lanes (word mode)
// or as a byte.  Called by all 32 lanes (the gather shuffles).
template <bool kWordScales>
__device__ __forceinline__ void store_scale(uint8_t* scales, uint32_t s, bool valid, uint32_t row, uint32_t kb,
                                            uint32_t kb4_per_tile, int lane) {
  if constexpr (kWordScales) {
    // lanes 4j..4j+3 hold blocks 4j..4j+3: two shuffles pack them into lane 4j's word
    const uint32_t s01 = s | (__shfl_down_sync(0xffffffffu, s, 1) << 8);
    const uint32_t w = s01 | (__shfl_down_sync(0xffffffffu, s01, 2) << 16);
    if (valid && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(scales + scale_word_offset(row, kb >> 2, kb4_per_tile)) = w;
  } else {
    if (valid) scales[scale_word_offset(row, kb >> 2, kb4_per_tile) + (kb & 3)] = static_cast<uint8_t>(s);
  }
}

// Zero the padding bytes of a scale array in the MMA layout: rows [rows, rows_pad)
// entirely, and blocks [Kb, 4 * kb4_per_tile) of the real rows.  Grid-strided over
// all threads of the launch.
__device__ __forceinline__ void zero_scale_padding(uint8_t* sx, uint8_t* sr, uint32_t rows, uint32_t Kb,
                                                   uint32_t kb4_per_tile, uint32_t rows_pad, uint32_t tid,
                                                   uint32_t nthreads) {
  const uint32_t pad_words = (rows_pad - rows) * kb4_per_tile;
  for (uint32_t t = tid; t < pad_words; t += nthreads) {
    const uint32_t r = rows + t / kb4_per_tile, kb4 = t % kb4_per_tile;
    const uint32_t off = scale_word_offset(r, kb4, kb4_per_tile);
    *reinterpret_cast<uint32_t*>(sx + off) = 0u;
    if (sr) *reinterpret_cast<uint32_t*>(sr + off) = 0u;
  }
  const uint32_t tail = kb4_per_tile * 4 - Kb;   // 0..3 pad blocks per real row
  if (tail > 0) {
    for (uint32_t t = tid; t < rows * tail; t += nthreads) {
      const uint32_t r = t / tail, kb = Kb + t % tail;
      const uint32_t off = scale_word_offset(r, kb >> 2, kb4_per_tile) + (kb & 3);
      sx[off] = 0;
      if (sr) sr[off] = 0;
    }
  }
}

// kWide: X seen as [blocks/2][128 bytes] with a 128-byte swizzle (needs an even
// block count); otherwise as [blocks][64 bytes] with a 64-byte swizzle.  Either
// way a lane's four 16-byte reads of its block hit distinct banks.
template <bool kResidual, bool kWordScales, bool kWide, bool kFp8>
__global__ void __launch_bounds__(kThreads, RFQ_Q_CTAS_PER_SM)
    rfq_quantize_kernel(const __grid_constant__ CUtensorMap tm_x, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * (kStages * kSpanBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kSpanBytes) + warp * kStages;
  volatile int abort_flag = 0;   // per warp: each warp's ring is independent

  const uint32_t gw = blockIdx.x * kWarps + warp;
  const uint32_t GW = gridDim.x * kWarps;
  const uint32_t n_my = p.num_spans > gw ? (p.num_spans - gw + GW - 1) / GW : 0;
  // TMA row coordinate of a span: rows of 128 bytes (2 blocks) or of 64 bytes (1 block)
  auto span_row = [&](uint32_t span) { return static_cast<int>(span * (kWide ? kSpanBlocks / 2 : kSpanBlocks)); };

  griddep_launch_dependents();
  if (lane == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
    // While the previous kernel on the stream finishes, pull this warp's first
    // spans into L2 (a hint; the copies below still follow griddepcontrol.wait).
    for (uint32_t st = 0; st < kStages && st < n_my; ++st) tma_prefetch_2d(&tm_x, 0, span_row(gw + st * GW));
    griddep_wait();   // X may be written by the previous kernel on the stream
    for (uint32_t st = 0; st < kStages && st < n_my; ++st) {
      mbar_arrive_expect_tx(&bars[st], kSpanBytes);
      tma_load_2d(ring + st * kSpanBytes, &tm_x, &bars[st], 0, span_row(gw + st * GW));
    }
  }
  __syncwarp();

  // Block coordinates of the span's first block, advanced incrementally span by span.
  const uint32_t stride_blocks = GW * kSpanBlocks;
  const uint32_t d_row = stride_blocks / p.Kb, d_kb = stride_blocks - d_row * p.Kb;
  uint32_t row0 = (gw * kSpanBlocks) / p.Kb;
  uint32_t kb0 = gw * kSpanBlocks - row0 * p.Kb;
  // Byte offset of this lane's block inside a 32-block sub-span, and the swizzle of its row.
  const int lane_off = kWide ? (lane >> 1) * 128 + (lane & 1) * 64 : lane * 64;
  const int swz = kWide ? (lane >> 1) & 7 : (lane >> 1) & 3;

  uint32_t i = 0;
  for (; i < n_my; ++i) {
    const int s = static_cast<int>(i % kStages);
    const bool ok = mbar_wait(&bars[s], (i / kStages) & 1u, &abort_flag, &g_quant_error, kErrQuantWait);
    if (!__all_sync(0xffffffffu, ok)) break;   // every lane returns from its bounded wait: a uniform decision

#pragma unroll 1
    for (int u = 0; u < kSub; ++u) {
    const uint32_t gb = (gw + i * GW) * kSpanBlocks + u * 32 + lane;
    const bool valid = gb < p.total_blocks;
    // lane's block: row, block-in-row
    uint32_t row, kb;
    {
      const uint32_t t = kb0 + u * 32 + lane;
      const uint32_t q = p.Kb >= kSpanBlocks ? (t >= p.Kb ? 1u : 0u) : t / p.Kb;
      row = row0 + q;
      kb = t - q * p.Kb;
    }

    uint32_t w[16];
    const uint8_t* src = ring + s * kSpanBytes + u * 2048 + lane_off;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int chunk = kWide ? (((lane & 1) * 4 + j) ^ swz) - (lane & 1) * 4 : (j ^ swz);
      const uint4 c = *reinterpret_cast<const uint4*>(src + chunk * 16);
      w[4 * j + 0] = c.x;
      w[4 * j + 1] = c.y;
      w[4 * j + 2] = c.z;
      w[4 * j + 3] = c.w;
    }
    if (u == kSub - 1) {
      __syncwarp();
      // This warp's data are now in registers: refill the stage with the span
      // kStages ahead (the reads above are ordered before the async-proxy write).
      if (lane == 0 && i + kStages < n_my) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive_expect_tx(&bars[s], kSpanBytes);
        tma_load_2d(ring + s * kSpanBytes, &tm_x, &bars[s], 0, span_row(gw + (i + kStages) * GW));
      }
    }

    if constexpr (kFp8) {
      // MXFP8 comparator: 32 code bytes per block
      uint32_t c8[8], s8;
      quantize_block_e4m3(w, c8, s8);
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(p.qx_codes + static_cast<size_t>(gb) * 32);
        dst[0] = make_uint4(c8[0], c8[1], c8[2], c8[3]);
        dst[1] = make_uint4(c8[4], c8[5], c8[6], c8[7]);
      }
      store_scale<kWordScales>(p.qx_scales, s8, valid, row, kb, p.kb4_per_tile, lane);
      continue;
    }
    uint32_t cx[4], cr[4], sx, sr;
    quantize_block<kResidual>(w, cx, sx, cr, sr);
    if (valid) *reinterpret_cast<uint4*>(p.qx_codes + static_cast<size_t>(gb) * 16) = make_uint4(cx[0], cx[1], cx[2], cx[3]);
    store_scale<kWordScales>(p.qx_scales, sx, valid, row, kb, p.kb4_per_tile, lane);
    if constexpr (kResidual) {
      if (valid) *reinterpret_cast<uint4*>(p.qr_codes + static_cast<size_t>(gb) * 16) = make_uint4(cr[0], cr[1], cr[2], cr[3]);
      store_scale<kWordScales>(p.qr_scales, sr, valid, row, kb, p.kb4_per_tile, lane);
    }

    }  // sub-spans

    kb0 += d_kb;
    row0 += d_row;
    if (kb0 >= p.Kb) {
      kb0 -= p.Kb;
      row0 += 1;
    }
  }

  if (i < n_my && lane == 0) {
    // A wait ran out: let this warp's outstanding copies land before leaving.
    int never = 0;
    for (uint32_t k = i; k < n_my && k < i + kStages; ++k)
      mbar_wait(&bars[k % kStages], static_cast<uint32_t>((k / kStages) & 1), &never, &g_quant_error, kErrQuantWait);
  }

  // ---- zero padding of the scale arrays: rows [M, rows_pad) and blocks [Kb, 4*kb4) of real rows
  // (stores to buffers the previous kernel on the stream may still read: wait for it)
  griddep_wait();
  zero_scale_padding(p.qx_scales, kResidual ? p.qr_scales : nullptr, p.M, p.Kb, p.kb4_per_tile, p.rows_pad,
                     blockIdx.x * kThreads + threadIdx.x, gridDim.x * kThreads);
}

// ---------------------------------------------------------------- transposed quantizer
// Quantizes X^T for a row-major bf16 X [R][C]: operand row c of the output is
// column c of X, and its 32-element blocks run down 32 consecutive rows of X.
//
// A CTA takes units of 256 rows x 64 columns of X: its 8 warps one 32-row block
// each (a 4 KiB TMA box, kTStages in flight per warp).  Lane l reads, for each of
// the 32 rows, the 32-bit word holding columns 2l and 2l+1 (conflict-free: a
// row's 32 words), regroups the halves into the pair layout of a block (byte
// permutes) and quantizes the two columns' blocks with the same per-block
// arithmetic as the row quantizer.  The codes are not stored from the lanes
// (16 bytes to each of 32 rows per store): the warps write them into a
// shared-memory tile of 64 operand rows x 8 blocks (128-byte swizzle), and after
// a CTA barrier one thread stores the tile with a TMA tensor store, so each
// operand row receives 128 contiguous bytes; the scale bytes leave as 32-bit
// words of the MMA layout.  The tiles are double-buffered: the store of one unit
// overlaps the quantization of the next.  Units are ordered row-block fastest,
// so CTAs running at the same time fill neighbouring pieces of the same rows.
constexpr int kTWarps = 8;
constexpr int kTThreads = kTWarps * 32;
constexpr int kTStages = 2;
constexpr uint32_t kTUnitBytes = 32 * 128;           // one warp's box: 32 rows x 64 bf16
constexpr uint32_t kTTileBytes = 64 * 128;           // codes of a unit: 64 operand rows x 8 blocks x 16 B
constexpr uint32_t kTSfBytes = 64 * 8;               // scale bytes of a unit: 64 rows x 8 blocks
constexpr uint32_t kTOffTileX = kTWarps * kTStages * kTUnitBytes;
constexpr uint32_t kTOffTileR = kTOffTileX + 2 * kTTileBytes;
constexpr uint32_t kTOffSfX = kTOffTileR + 2 * kTTileBytes;
constexpr uint32_t kTOffSfR = kTOffSfX + 2 * kTSfBytes;
constexpr uint32_t kTOffBars = kTOffSfR + 2 * kTSfBytes;
constexpr uint32_t kTSmemBytes = kTOffBars + kTWarps * kTStages * 8 + 1024;
static_assert(kTOffTileX % 1024 == 0 && kTOffTileR % 1024 == 0, "swizzled tiles need 1 KiB alignment");

struct QuantTParams {
  uint8_t* qt_scales;
  uint8_t* qr_scales;
  uint32_t R;             // rows of X = K of the operand
  uint32_t C;             // columns of X = rows of the operand
  uint32_t Rb;            // R / 32: blocks per operand row
  uint32_t Rb8;           // ceil(Rb / 8): units along R
  uint32_t kb4_per_tile;  // ceil(Rb / 4)
  uint32_t rows_pad;      // ceil(C / 128) * 128
  uint32_t num_ct;        // ceil(C / 64)
  uint32_t num_units;     // Rb8 * num_ct
};

struct QuantTMaps {
  CUtensorMap x;          // X [R][C] bf16, box 64 columns x 32 rows
  CUtensorMap qt, qr;     // codes [C][R/2] bytes, box 128 B x 64 rows, 128-byte swizzle
};

template <bool kResidual>
__global__ void __launch_bounds__(kTThreads, 2)
    rfq_quantize_t_kernel(const __grid_constant__ QuantTMaps maps, const QuantTParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * (kTStages * kTUnitBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTOffBars) + warp * kTStages;
  volatile int abort_flag = 0;   // per warp: each warp's ring is independent

  const uint32_t n_my =
      p.num_units > blockIdx.x ? (p.num_units - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;   // CTA-uniform
  // Block row rt of X this warp quantizes in the CTA's k-th unit, and its column tile.
  auto unit_of = [&](uint32_t k, uint32_t& rt, uint32_t& ct) {
    const uint32_t u = blockIdx.x + k * gridDim.x;
    ct = u / p.Rb8;
    rt = (u - ct * p.Rb8) * kTWarps + static_cast<uint32_t>(warp);
  };
  auto issue = [&](uint32_t k, int st) {
    uint32_t rt, ct;
    unit_of(k, rt, ct);
    if (rt < p.Rb) {
      mbar_arrive_expect_tx(&bars[st], kTUnitBytes);
      tma_load_2d(ring + st * kTUnitBytes, &maps.x, &bars[st], static_cast<int>(ct * 64), static_cast<int>(rt * 32));
    } else {
      mbar_arrive(&bars[st]);   // past the last block row: nothing to load, the phase still completes
    }
  };

  griddep_launch_dependents();
  if (lane == 0) {
    for (int st = 0; st < kTStages; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
    if (warp == 0) {
      prefetch_tmap(&maps.qt);
      if (kResidual) prefetch_tmap(&maps.qr);
    }
    // While the previous kernel on the stream finishes, pull this warp's first boxes
    // into L2 (a hint; the copies below still follow griddepcontrol.wait).
    for (uint32_t k = 0; k < kTStages && k < n_my; ++k) {
      uint32_t rt, ct;
      unit_of(k, rt, ct);
      if (rt < p.Rb) tma_prefetch_2d(&maps.x, static_cast<int>(ct * 64), static_cast<int>(rt * 32));
    }
    griddep_wait();   // X may be written by the previous kernel on the stream
    for (uint32_t k = 0; k < kTStages && k < n_my; ++k) issue(k, static_cast<int>(k));
  }
  __syncwarp();

  bool ok = true;            // this warp's waits so far (warp-uniform)
  uint32_t k_fail = n_my;    // the unit whose wait ran out
  uint32_t k = 0;
  for (; k < n_my; ++k) {
    const int st = static_cast<int>(k % kTStages);
    const uint32_t buf = k & 1u;
    uint32_t rt, ct;
    unit_of(k, rt, ct);
    uint8_t* tile_x = smem + kTOffTileX + buf * kTTileBytes;
    uint8_t* tile_r = smem + kTOffTileR + buf * kTTileBytes;
    uint8_t* sf_x = smem + kTOffSfX + buf * kTSfBytes;
    uint8_t* sf_r = smem + kTOffSfR + buf * kTSfBytes;
    // A wait that runs out leaves the warp producing garbage without waiting again:
    // every warp still reaches each CTA barrier below, and the error word reports it.
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[st], (k / kTStages) & 1u, &abort_flag, &g_quant_error,
                                             kErrQuantWait));
      if (!ok) k_fail = k;
    }
    uint32_t wr[32];
    const uint32_t* src = reinterpret_cast<const uint32_t*>(ring + st * kTUnitBytes) + lane;
#pragma unroll
    for (int r = 0; r < 32; ++r) wr[r] = src[r * 32];
    __syncwarp();
    if (lane == 0 && ok && k + kTStages < n_my) {
      // this warp's data are in registers: refill the stage (reads ordered before the async write)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(k + kTStages, st);
    }
    const bool valid = rt < p.Rb;   // warp-uniform
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      // element 2j of the block = row 2j (low half), 2j+1 = row 2j+1 (high half)
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) w[j] = prmt(wr[2 * j], wr[2 * j + 1], h ? 0x7632u : 0x5410u);
      uint32_t cx[4] = {0, 0, 0, 0}, cr[4] = {0, 0, 0, 0}, sx = 0, sr = 0;
      if (valid) quantize_block<kResidual>(w, cx, sx, cr, sr);
      // operand row 2 lane + h of the tile, block `warp`: 16-byte chunk `warp` of the
      // row's 128 bytes, at chunk position warp ^ (row % 8) (128-byte swizzle)
      const uint32_t r_loc = 2u * static_cast<uint32_t>(lane) + static_cast<uint32_t>(h);
      const uint32_t off = r_loc * 128u + ((static_cast<uint32_t>(warp) ^ (r_loc & 7u)) << 4);
      *reinterpret_cast<uint4*>(tile_x + off) = make_uint4(cx[0], cx[1], cx[2], cx[3]);
      sf_x[r_loc * 8u + warp] = static_cast<uint8_t>(sx);   // 0 past the last block row: scale padding
      if constexpr (kResidual) {
        *reinterpret_cast<uint4*>(tile_r + off) = make_uint4(cr[0], cr[1], cr[2], cr[3]);
        sf_r[r_loc * 8u + warp] = static_cast<uint8_t>(sr);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the tiles go out through TMA
    // The other buffer's store (issued one unit ago) must have finished reading it
    // before the barrier lets the warps write it again in the next unit.
    if (threadIdx.x == 0) bulk_wait_read_all();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int x = static_cast<int>((rt - static_cast<uint32_t>(warp)) * 16u), y = static_cast<int>(ct * 64u);
      tma_store_2d(&maps.qt, tile_x, x, y);
      if (kResidual) tma_store_2d(&maps.qr, tile_r, x, y);
      bulk_commit_group();
    }
    if (threadIdx.x < 128) {
      // scales: operand row c, 4-block word j of the unit's 8 blocks
      const uint32_t r_loc = threadIdx.x >> 1, j = threadIdx.x & 1u;
      const uint32_t c = ct * 64u + r_loc;
      const uint32_t kb4 = (rt - static_cast<uint32_t>(warp)) / 4u + j;   // rt - warp: the unit's first block row
      if (c < p.C && kb4 < p.kb4_per_tile) {
        const uint32_t o = scale_word_offset(c, kb4, p.kb4_per_tile);
        *reinterpret_cast<uint32_t*>(p.qt_scales + o) = *reinterpret_cast<const uint32_t*>(sf_x + r_loc * 8u + 4u * j);
        if constexpr (kResidual)
          *reinterpret_cast<uint32_t*>(p.qr_scales + o) = *reinterpret_cast<const uint32_t*>(sf_r + r_loc * 8u + 4u * j);
      }
    }
  }

  if (!ok && lane == 0) {
    // A wait ran out: let this warp's outstanding copies (units k_fail .. k_fail +
    // kTStages - 1, issued before it) land before leaving.
    int never = 0;
    for (uint32_t i = k_fail; i < n_my && i < k_fail + kTStages; ++i)
      mbar_wait(&bars[i % kTStages], (i / kTStages) & 1u, &never, &g_quant_error, kErrQuantWait);
  }
  if (threadIdx.x == 0) bulk_wait_all();   // the tiles' stores are complete before the CTA's memory goes

  griddep_wait();   // the padding stores may hit buffers the previous kernel still reads
  zero_scale_padding(p.qt_scales, kResidual ? p.qr_scales : nullptr, p.C, p.Rb, p.kb4_per_tile, p.rows_pad,
                     blockIdx.x * kTThreads + threadIdx.x, gridDim.x * kTThreads);
}


template <bool kResidual>
cudaError_t launch_t_typed(const QuantTMaps& maps, const QuantTParams& p, int grid, cudaStream_t stream) {
  auto kernel = rfq_quantize_t_kernel<kResidual>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTThreads);
  cfg.dynamicSmemBytes = kTSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait()
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, maps, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

#ifndef RFQ_Q_WIDE
#define RFQ_Q_WIDE 1
#endif

template <bool kResidual, bool kWord, bool kWide, bool kFp8 = false>
cudaError_t launch_typed(const CUtensorMap& tm, const QuantParams& p, int grid, cudaStream_t stream) {
  auto kernel = rfq_quantize_kernel<kResidual, kWord, kWide, kFp8>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait()
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, tm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool kResidual, bool kWord, bool kFp8 = false>
cudaError_t launch_width(bool wide, const CUtensorMap& tm, const QuantParams& p, int grid, cudaStream_t stream) {
  return wide ? launch_typed<kResidual, kWord, true, kFp8>(tm, p, grid, stream)
              : launch_typed<kResidual, kWord, false, kFp8>(tm, p, grid, stream);
}

}  // namespace

cudaError_t launch_quantize_impl(const void* x, int64_t M, int64_t K, void* qx_codes, void* qx_scales, void* qr_codes,
                                 void* qr_scales, bool fp8, int num_sms, void* encode_tiled, cudaStream_t stream) {
  QuantParams p;
  p.qx_codes = static_cast<uint8_t*>(qx_codes);
  p.qx_scales = static_cast<uint8_t*>(qx_scales);
  p.qr_codes = static_cast<uint8_t*>(qr_codes);
  p.qr_scales = static_cast<uint8_t*>(qr_scales);
  p.M = static_cast<uint32_t>(M);
  p.Kb = static_cast<uint32_t>(K / 32);
  p.kb4_per_tile = (p.Kb + 3) / 4;
  p.rows_pad = static_cast<uint32_t>((M + 127) / 128 * 128);
  p.total_blocks = static_cast<uint32_t>(M * (K / 32));
  p.num_spans = (p.total_blocks + kSpanBlocks - 1) / kSpanBlocks;

  // X as [total_blocks/2][128 bytes] (128-byte swizzle) when the block count is
  // even, else as [total_blocks][64 bytes] (64-byte swizzle); boxes of one span;
  // zero fill past the end.
  const bool wide = RFQ_Q_WIDE && (p.total_blocks % 2) == 0;
  CUtensorMap tm;
  cuuint64_t dims[2] = {wide ? 128u : 64u, static_cast<cuuint64_t>(wide ? p.total_blocks / 2 : p.total_blocks)};
  cuuint64_t strides[1] = {wide ? 128u : 64u};
  cuuint32_t box[2] = {wide ? 128u : 64u, static_cast<cuuint32_t>(wide ? kSpanBlocks / 2 : kSpanBlocks)};
  cuuint32_t elem_strides[2] = {1, 1};
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  const int64_t warps_needed = p.num_spans;
  int64_t grid = (warps_needed + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * RFQ_Q_CTAS_PER_SM;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const bool word = (p.Kb % 4) == 0;
  const int g = static_cast<int>(grid);
  if (fp8)
    return word ? launch_width<false, true, true>(wide, tm, p, g, stream)
                : launch_width<false, false, true>(wide, tm, p, g, stream);
  if (qr_codes)
    return word ? launch_width<true, true>(wide, tm, p, g, stream) : launch_width<true, false>(wide, tm, p, g, stream);
  return word ? launch_width<false, true>(wide, tm, p, g, stream) : launch_width<false, false>(wide, tm, p, g, stream);
}

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, void* qx_codes, void* qx_scales, void* qr_codes,
                            void* qr_scales, int num_sms, void* encode_tiled, cudaStream_t stream) {
  return launch_quantize_impl(x, M, K, qx_codes, qx_scales, qr_codes, qr_scales, false, num_sms, encode_tiled,
                              stream);
}

cudaError_t launch_quantize_mxfp8(const void* x, int64_t M, int64_t K, void* codes, void* scales, int num_sms,
                                  void* encode_tiled, cudaStream_t stream) {
  return launch_quantize_impl(x, M, K, codes, scales, nullptr, nullptr, true, num_sms, encode_tiled, stream);
}

cudaError_t launch_quantize_t(const void* x, int64_t R, int64_t C, void* qt_codes, void* qt_scales, void* qr_codes,
                              void* qr_scales, int num_sms, void* encode_tiled, cudaStream_t stream) {
  QuantTParams p;
  p.qt_scales = static_cast<uint8_t*>(qt_scales);
  p.qr_scales = static_cast<uint8_t*>(qr_scales);
  p.R = static_cast<uint32_t>(R);
  p.C = static_cast<uint32_t>(C);
  p.Rb = static_cast<uint32_t>(R / 32);
  p.Rb8 = (p.Rb + kTWarps - 1) / kTWarps;
  p.kb4_per_tile = (p.Rb + 3) / 4;
  p.rows_pad = static_cast<uint32_t>((C + 127) / 128 * 128);
  p.num_ct = static_cast<uint32_t>((C + 63) / 64);
  p.num_units = p.Rb8 * p.num_ct;

  // X as [R][C] 16-bit elements; boxes of 64 columns x 32 rows, no swizzle, zeros
  // past the last column.  The codes as [C][R/2] bytes, stored in 128-byte x
  // 64-row tiles (128-byte swizzle, clipped at the ends).
  QuantTMaps maps;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(R)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
  cuuint32_t box[2] = {64u, 32u};
  cuuint32_t elem_strides[2] = {1, 1};
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  if (encode(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (!encode_code_rows_map(encode, &maps.qt, qt_codes, C, R / 2, 64)) return cudaErrorInvalidValue;
  if (qr_codes) {
    if (!encode_code_rows_map(encode, &maps.qr, qr_codes, C, R / 2, 64)) return cudaErrorInvalidValue;
  } else {
    maps.qr = maps.qt;
  }
  int64_t grid = static_cast<int64_t>(p.num_units);
  const int64_t cap = static_cast<int64_t>(num_sms) * 2;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  return qr_codes ? launch_t_typed<true>(maps, p, static_cast<int>(grid), stream)
                  : launch_t_typed<false>(maps, p, static_cast<int>(grid), stream);
}

cudaError_t read_and_clear_quant_error(unsigned int* value) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(value, g_quant_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(unsigned int));
}

}  // namespace rfq

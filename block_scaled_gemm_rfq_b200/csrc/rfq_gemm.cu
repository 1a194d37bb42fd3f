// rfq_gemm.cu -- kernel 2: the RFQ block-scaled GEMM on sm_100a tensor cores.
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): the residual of the activation is
// requantized and "its contribution accumulated during the GEMM".  Here
//
//     Y = DQ(QX).DQ(QW)^T + DQ(QR).DQ(QW)^T
//
// is one accumulation in TMEM: for every k-tile both QX x QW and QR x QW are
// issued as tcgen05 kind::mxf4 block-scaled MMAs into the same fp32 accumulator,
// reusing the QW tile already in shared memory, so the residual doubles the work
// on the tensor pipe (K -> 2K) and costs no extra pass over Y.
//
// Structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per k-tile (128 elements = 64 bytes per row) it
//               loads the QX, QR and QW code tiles (2-D tensor maps, 64-byte
//               swizzle) and their 512-byte scale atoms (1-D bulk copies) into a
//               kStages-deep shared-memory ring guarded by mbarriers;
//   warp 1      MMA issuer (one thread): copies the stage's scale atoms into TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues 2 + 2 MMAs of K = 64;
//               tcgen05.commit frees the stage and, at the end of a tile,
//               signals the epilogue;
//   warps 2..9  epilogue: TMEM -> registers (tcgen05.ld 32x32b, 128 columns per
//               warp), release of the accumulator, then fp32/bf16 -> global,
//               one accumulator row per thread, overlapping the next mainloop.
// Every mbarrier wait is bounded (rfq_ptx.cuh); a wait that runs out records an
// error code, raises the CTA's abort flag and the CTA tears down cleanly (its
// copies and MMAs drained, its TMEM freed).  No TMA multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rfq_internal.h"
#include "rfq_ptx.cuh"

namespace rfq {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kBM = 128;               // rows of X / Y per tile (MMA M)
constexpr int kBN = 256;               // rows of W / columns of Y per tile (MMA N)
constexpr int kBK = 128;               // K elements per stage
constexpr int kBKBytes = kBK / 2;      // packed FP4: 64 bytes per row per stage
constexpr int kStages = 6;
constexpr int kThreads = 320;        // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;        // 256 fp32 columns: the 128 x 256 accumulator
constexpr uint32_t kSfaXCol = 256;     // 4 columns: scales of QX for 128 rows x 4 blocks
constexpr uint32_t kSfaRCol = 260;     // 4 columns: scales of QR
constexpr uint32_t kSfbCol = 264;      // 8 columns: scales of QW for 256 rows x 4 blocks

constexpr uint32_t kATileBytes = kBM * kBKBytes;   // 8 KiB
constexpr uint32_t kBTileBytes = kBN * kBKBytes;   // 16 KiB
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffR = kOffA + kATileBytes;
constexpr uint32_t kOffB = kOffR + kATileBytes;
constexpr uint32_t kOffSfaX = kOffB + kBTileBytes;
constexpr uint32_t kOffSfaR = kOffSfaX + 512;
constexpr uint32_t kOffSfb = kOffSfaR + 512;
constexpr uint32_t kStageBytes = kOffSfb + 1024;   // 34 KiB, a multiple of 1 KiB
constexpr uint32_t kBarrierBytes = 256;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;  // + alignment slack

static_assert(kStageBytes % 1024 == 0, "stage buffers must keep 1 KiB alignment");
static_assert(kSmemBytes <= 232448, "exceeds the 227 KiB shared-memory limit");

struct GemmParams {
  const uint8_t* sfa_x;
  const uint8_t* sfa_r;
  const uint8_t* sfb;
  void* y;
  int M;
  int N;
  int num_kt;            // k-tiles of 128 elements
  int atoms_per_rowtile; // scale atoms per 128-row tile = ceil(K/128)
  int num_nb;            // tiles along N
  int num_tiles;
  int b_rowtiles;        // ceil(N/128): scale atoms of W along N
  int skip_fill;         // fault injection (-1 = off)
};

// Shared-memory matrix descriptor (tcgen05): K-major operand, 64-byte swizzle,
// rows of 64 bytes, 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t operand_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull)     // start address
         | (1ull << 16)                // leading byte offset (unused for swizzled K-major)
         | ((512ull >> 4) << 32)       // stride byte offset: 8 rows x 64 B
         | (1ull << 46)                // descriptor version (sm_100)
         | (4ull << 61);               // layout: 64-byte swizzle
}

// Descriptor of a 512-byte scale atom as 32 rows x 16 bytes, no swizzle, 8-row
// core matrices 128 bytes apart (source of tcgen05.cp 32x128b).
__device__ __forceinline__ uint64_t scale_desc(const void* p) {
  const uint64_t addr = smem_addr(p);
  return ((addr >> 4) & 0x3FFFull) | ((128ull >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::mxf4 with E8M0 scales: E2M1 x E2M1, both
// K-major, M = 128, N = 256, scale-factor byte selectors for A and B.
__device__ __forceinline__ uint32_t mma_idesc(uint32_t sf_id) {
  return (sf_id << 4)                  // B scale-factor id
         | (1u << 7)                   // A format E2M1
         | (1u << 10)                  // B format E2M1
         | (uint32_t(kBN >> 3) << 17)  // N / 8
         | (1u << 23)                  // scale type UE8M0
         | (uint32_t(kBM >> 4) << 24)  // M / 16
         | (sf_id << 29);              // A scale-factor id
}

template <bool kResidual, bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1)
    rfq_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                    const __grid_constant__ CUtensorMap tm_w, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
    if (kResidual) prefetch_tmap(&tm_r);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t stage = 0, phase = 0;
      uint32_t filled = 0, last_parity = 0;
      int fill = 0;
      const uint32_t sfb_atoms_full = 2;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int mb = tile / p.num_nb;
        const int nb = tile - mb * p.num_nb;
        const bool b_hi = (2 * nb + 1) < p.b_rowtiles;
        const uint32_t bytes = kATileBytes + kBTileBytes + 512u + 512u * (b_hi ? sfb_atoms_full : 1u) +
                               (kResidual ? kATileBytes + 512u : 0u);
        const uint8_t* sfa_x_row = p.sfa_x + static_cast<int64_t>(mb) * p.atoms_per_rowtile * 512;
        const uint8_t* sfa_r_row = kResidual ? p.sfa_r + static_cast<int64_t>(mb) * p.atoms_per_rowtile * 512 : nullptr;
        const uint8_t* sfb_lo = p.sfb + static_cast<int64_t>(2 * nb) * p.atoms_per_rowtile * 512;
        const uint8_t* sfb_hi = sfb_lo + static_cast<int64_t>(p.atoms_per_rowtile) * 512;
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, &g_device_error, kErrWaitEmpty)) goto producer_done;
          if (!(fill == p.skip_fill && blockIdx.x == 0)) {
            uint8_t* st = smem + stage * kStageBytes;
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_2d(st + kOffA, &tm_x, &full[stage], kt * kBKBytes, mb * kBM);
            if (kResidual) tma_load_2d(st + kOffR, &tm_r, &full[stage], kt * kBKBytes, mb * kBM);
            tma_load_2d(st + kOffB, &tm_w, &full[stage], kt * kBKBytes, nb * kBN);
            bulk_load(st + kOffSfaX, sfa_x_row + kt * 512, 512, &full[stage]);
            if (kResidual) bulk_load(st + kOffSfaR, sfa_r_row + kt * 512, 512, &full[stage]);
            bulk_load(st + kOffSfb, sfb_lo + kt * 512, 512, &full[stage]);
            if (b_hi) bulk_load(st + kOffSfb + 512, sfb_hi + kt * 512, 512, &full[stage]);
            filled |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          ++fill;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    producer_done:
      // Teardown: every copy this thread issued must have landed before exit.
      for (int s = 0; s < kStages; ++s)
        if (filled & (1u << s)) {
          int never = 0;
          mbar_wait(&full[s], (last_parity >> s) & 1u, &never, &g_device_error, kErrWaitDrain);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      uint32_t stage = 0, phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag, &g_device_error, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < p.num_kt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, &g_device_error, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* st = smem + stage * kStageBytes;
          tmem_copy_32x128b_warpx4(tmem + kSfaXCol, scale_desc(st + kOffSfaX));
          if (kResidual) tmem_copy_32x128b_warpx4(tmem + kSfaRCol, scale_desc(st + kOffSfaR));
          tmem_copy_32x128b_warpx4(tmem + kSfbCol, scale_desc(st + kOffSfb));
          tmem_copy_32x128b_warpx4(tmem + kSfbCol + 4, scale_desc(st + kOffSfb + 512));
          const uint64_t da = operand_desc(st + kOffA);
          const uint64_t db = operand_desc(st + kOffB);
#pragma unroll
          for (uint32_t j = 0; j < 2; ++j) {
            const uint32_t sf = 2u * j;  // MMA j uses scale bytes 2j, 2j+1 of each 4-block word
            mma_mxf4(tmem + kAccCol, da + 2u * j, db + 2u * j, mma_idesc(sf), (tmem + kSfaXCol) | (sf << 30),
                     (tmem + kSfbCol) | (sf << 30), (kt | j) != 0 ? 1u : 0u);
          }
          if (kResidual) {
            const uint64_t dr = operand_desc(st + kOffR);
#pragma unroll
            for (uint32_t j = 0; j < 2; ++j) {
              const uint32_t sf = 2u * j;
              mma_mxf4(tmem + kAccCol, dr + 2u * j, db + 2u * j, mma_idesc(sf), (tmem + kSfaRCol) | (sf << 30),
                       (tmem + kSfbCol) | (sf << 30), 1u);
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      if (!ok) {
        // Teardown after an abort: wait for the MMAs already issued.
        tc_commit(drain);
        int never = 0;
        mbar_wait(drain, 0, &never, &g_device_error, kErrWaitDrain);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // 8 warps: two per TMEM lane quadrant, each owning 128 of the 256 columns.
    // The accumulator is copied to registers first and released to the MMA warp
    // at once, so converting and storing Y overlaps the next tile's mainloop.
    const int quad = warp & 3;                // TMEM lanes this warp may access: 32*quad .. 32*quad+31
    const int half = (warp - 2) >> 2;         // columns [128*half, 128*half + 128)
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int mb = tile / p.num_nb;
      const int nb = tile - mb * p.num_nb;
      if (!mbar_wait(acc_full, acc_phase, abort_flag, &g_device_error, kErrWaitAccFull)) break;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + kAccCol + half * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_load_32x32b_x32(taddr + 32 * c, v[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;

      const int row = mb * kBM + quad * 32 + lane;
      const int col0 = nb * kBN + half * 128;
      if (row < p.M) {
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
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D map over packed codes [rows][K/2] bytes; box = 64 bytes x box_rows rows,
// 64-byte swizzle (the layout operand_desc() describes), zero fill outside.
bool encode_codes_map(EncodeTiledFn encode, CUtensorMap* map, const void* codes, int64_t rows, int64_t K,
                      uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKBytes), box_rows};
  cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
                      elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kResidual, bool kBf16Out>
cudaError_t launch_typed(const CUtensorMap& tx, const CUtensorMap& tr, const CUtensorMap& tw, const GemmParams& p,
                         int grid, cudaStream_t stream) {
  auto kernel = rfq_gemm_kernel<kResidual, kBf16Out>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(tx, tr, tw, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                        const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y,
                        bool y_bf16, int num_sms, void* encode_tiled, int skip_fill, cudaStream_t stream) {
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  const bool residual = qr_codes != nullptr;
  CUtensorMap tx, tr, tw;
  if (!encode_codes_map(encode, &tx, qx_codes, M, K, kBM)) return cudaErrorInvalidValue;
  if (!encode_codes_map(encode, &tw, qw_codes, N, K, kBN)) return cudaErrorInvalidValue;
  if (residual) {
    if (!encode_codes_map(encode, &tr, qr_codes, M, K, kBM)) return cudaErrorInvalidValue;
  } else {
    tr = tx;
  }
  GemmParams p;
  p.sfa_x = static_cast<const uint8_t*>(qx_scales);
  p.sfa_r = static_cast<const uint8_t*>(qr_scales);
  p.sfb = static_cast<const uint8_t*>(qw_scales);
  p.y = y;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.num_kt = static_cast<int>((K + kBK - 1) / kBK);
  p.atoms_per_rowtile = p.num_kt;
  const int64_t num_mb = (M + kBM - 1) / kBM;
  p.num_nb = static_cast<int>((N + kBN - 1) / kBN);
  p.num_tiles = static_cast<int>(num_mb * p.num_nb);
  p.b_rowtiles = static_cast<int>((N + 127) / 128);
  p.skip_fill = skip_fill;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  if (residual) {
    return y_bf16 ? launch_typed<true, true>(tx, tr, tw, p, grid, stream)
                  : launch_typed<true, false>(tx, tr, tw, p, grid, stream);
  }
  return y_bf16 ? launch_typed<false, true>(tx, tr, tw, p, grid, stream)
                : launch_typed<false, false>(tx, tr, tw, p, grid, stream);
}

cudaError_t read_and_clear_device_error(unsigned int* value) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace rfq

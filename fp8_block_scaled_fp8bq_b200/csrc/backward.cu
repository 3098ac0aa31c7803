// Operand preparation for the backward pass of the FP8 linear layer:
//   * the 1x128 quantization along the token axis with transposed output (the
//     weight-gradient GEMM contracts over tokens, so both of its operands, dY
//     and X, are quantized in 128-token tiles and stored token-contiguous);
//   * the transpose of a weight's 128x128-tile codes and scales (the
//     data-gradient GEMM dX = dY W multiplies by W^T; a square tile's scale
//     applies to its transpose unchanged, so no requantization is needed).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Technical breakthrough": FP8 in both generation and
// training, block-wise E4M3 with 1x128 activation and 128x128 weight tiles.
//
// Both kernels are HBM-bound: 2 bytes read and 1 written per element for the
// quantizer, 1 and 1 for the transpose.  Both stage their tiles in shared
// memory so that the global reads and writes are both row-contiguous.
#include <algorithm>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

using namespace qdev;

// ---------------------------------------------------------------------------
// Token-axis 1x128 quantization, transposed output
// ---------------------------------------------------------------------------
// Block (bx, by): tokens [128 by, +128) x columns [128 bx, +128) of X.  The
// 128 x 128 bf16 tile is staged in shared memory (256-byte rows, 16-byte
// loads, 16 lanes per row).  Warp w owns tokens [32 (w & 3), +32) of column
// half w >> 2, and lane l the column pair (2 l, 2 l + 1) of that half: it reads
// one 4-byte word per token (a warp reads 128 contiguous bytes of one row:
// no bank conflicts).  The four token groups' partial amaxes meet in shared
// memory; each lane then writes 32 token-contiguous codes of each of its two
// columns into X^T, i.e. whole 32-byte sectors.
constexpr int kTTok = 128, kTCol = 128;

// The 32 tokens of two columns (low and high bf16 halves of w[]) -> codes.
template <int MODE, bool FAST>
__device__ __forceinline__ void encode_columns(const uint32_t (&w)[32], const TileScale &t0, const TileScale &t1,
                                               uint32_t (&ca)[8], uint32_t (&cb)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // codes of -(x / s), sign bits flipped back (see neg_quotient2)
    const float2 qa0 = neg_quotient2<MODE, FAST>(make_float2(bf16_lo(w[4 * j]), bf16_lo(w[4 * j + 1])), t0);
    const float2 qa1 = neg_quotient2<MODE, FAST>(make_float2(bf16_lo(w[4 * j + 2]), bf16_lo(w[4 * j + 3])), t0);
    const float2 qb0 = neg_quotient2<MODE, FAST>(make_float2(bf16_hi(w[4 * j]), bf16_hi(w[4 * j + 1])), t1);
    const float2 qb1 = neg_quotient2<MODE, FAST>(make_float2(bf16_hi(w[4 * j + 2]), bf16_hi(w[4 * j + 3])), t1);
    ca[j] = (e4m3x2(qa0.x, qa0.y) | (e4m3x2(qa1.x, qa1.y) << 16)) ^ 0x80808080u;
    cb[j] = (e4m3x2(qb0.x, qb0.y) | (e4m3x2(qb1.x, qb1.y) << 16)) ^ 0x80808080u;
  }
}

template <int MODE>
__global__ void __launch_bounds__(256) quant_act_t_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                          int64_t ldx, uint8_t *__restrict__ qt, int64_t ldqt,
                                                          float *__restrict__ st, int64_t ldst) {
  __shared__ __align__(16) uint32_t tile[kTTok][kTCol / 2];
  __shared__ uint32_t part[4][kTCol / 2];  // [token group][column pair]: packed |bf16| maxima
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.y * kTTok, k0 = (int64_t)blockIdx.x * kTCol;

#pragma unroll
  for (int it = 0; it < 8; ++it) {  // 128 rows x 16 chunks of 16 bytes
    const int idx = it * 256 + threadIdx.x;
    const int r = idx >> 4, c = idx & 15;
    const int64_t m = m0 + r, k = k0 + c * 8;
    const uint4 v = (m < M && k < K) ? ld_nc_v4(x + m * ldx + k) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(&tile[r][c * 4]) = v;
  }
  __syncthreads();

  const int tg = warp & 3, ch = warp >> 2;
  const int pc = ch * 32 + lane;  // column pair within the tile
  uint32_t w[32];
  uint32_t am = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    w[i] = tile[tg * 32 + i][pc];
    am = __vmaxu2(am, w[i] & 0x7FFF7FFFu);
  }
  part[tg][pc] = am;
  __syncthreads();
  am = __vmaxu2(__vmaxu2(part[0][pc], part[1][pc]), __vmaxu2(part[2][pc], part[3][pc]));
  const TileScale t0 = tile_scale<MODE>(bits_to_amax(am & 0xFFFFu));
  const TileScale t1 = tile_scale<MODE>(bits_to_amax(am >> 16));

  const int64_t ka = k0 + 2 * pc, kb = ka + 1;
  const int64_t mt = m0 + tg * 32;  // first token of this lane's 32
  uint32_t ca[8], cb[8];            // 32 codes of column ka, 32 of column kb
  if (fast_tile<MODE>(t0) && fast_tile<MODE>(t1)) encode_columns<MODE, true>(w, t0, t1, ca, cb);
  else encode_columns<MODE, false>(w, t0, t1, ca, cb);
  if (mt < M) {
    const bool whole = mt + 32 <= M;
    if (ka < K) {
      uint8_t *d = qt + ka * ldqt + mt;
      if (whole) {
        *reinterpret_cast<uint4 *>(d) = make_uint4(ca[0], ca[1], ca[2], ca[3]);
        *reinterpret_cast<uint4 *>(d + 16) = make_uint4(ca[4], ca[5], ca[6], ca[7]);
      } else {
        for (int i = 0; i < 32 && mt + i < M; ++i) d[i] = (uint8_t)(ca[i >> 2] >> (8 * (i & 3)));
      }
    }
    if (kb < K) {
      uint8_t *d = qt + kb * ldqt + mt;
      if (whole) {
        *reinterpret_cast<uint4 *>(d) = make_uint4(cb[0], cb[1], cb[2], cb[3]);
        *reinterpret_cast<uint4 *>(d + 16) = make_uint4(cb[4], cb[5], cb[6], cb[7]);
      } else {
        for (int i = 0; i < 32 && mt + i < M; ++i) d[i] = (uint8_t)(cb[i >> 2] >> (8 * (i & 3)));
      }
    }
  }
  if (tg == 0) {
    float *srow = st + (int64_t)blockIdx.y * ldst;
    if (ka < K) srow[ka] = t0.s;
    if (kb < K) srow[kb] = t1.s;
  }
}

// ---------------------------------------------------------------------------
// Transpose of a weight's codes and tile scales
// ---------------------------------------------------------------------------
// Weight-code transpose: q [R][C] bytes -> q^T [C][R], 128 x 128-byte tiles.
// Persistent CTAs (two per SM); per CTA a producer thread streams tiles in by
// TMA through a four-stage ring (row-major, no swizzle), eight warps each take
// one 8 x 8-byte block per thread (thread t: rows 8 (t / 16) .., columns
// 8 (t % 16) ..), transpose it in registers with byte permutes and write it
// into one of two output tiles in the TMA's 128-byte-swizzled layout, from
// which a TMA store writes whole 128-byte rows of q^T.  Reads: each half-warp
// reads one 128-byte row per instruction (conflict-free).  Writes: thread t
// writes its eight output rows in the order rotated by (t % 16) & 7, so that
// with the swizzle the 16 lanes of a half-warp hit 8 different 16-byte
// chunks (two wavefronts per warp instruction, the minimum for 256 bytes).
constexpr int kTT = 128;                 // tile edge, bytes = elements
constexpr int kTTileBytes = kTT * kTT;   // 16 KB
constexpr int kTStages = 4;
constexpr int kTOut = 2;
constexpr int kTWarps = 8;               // transposing warps; warp 8 is the producer
constexpr int kTThreads = 32 * (kTWarps + 1);
constexpr int kTSmemBytes = (kTStages + kTOut) * kTTileBytes + 256 + 1024;

// At most one bulk group of this thread still reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// 8 x 8 bytes: row i of the block is lo[i] (bytes 0-3) and hi[i] (bytes 4-7);
// on return row i holds column i.  Three exchange stages: 4 x 4-byte blocks,
// 2 x 2 blocks of 2 bytes, single bytes.
__device__ __forceinline__ void transpose8x8(uint32_t (&lo)[8], uint32_t (&hi)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t t = hi[i];
    hi[i] = lo[i + 4];
    lo[i + 4] = t;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if ((i & 2) != 0) continue;  // rows i and i + 2 for i in {0, 1, 4, 5}
    uint32_t a = lo[i], b = lo[i + 2];
    lo[i] = __byte_perm(a, b, 0x5410);
    lo[i + 2] = __byte_perm(a, b, 0x7632);
    a = hi[i];
    b = hi[i + 2];
    hi[i] = __byte_perm(a, b, 0x5410);
    hi[i + 2] = __byte_perm(a, b, 0x7632);
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) {  // rows i and i + 1
    uint32_t a = lo[i], b = lo[i + 1];
    lo[i] = __byte_perm(a, b, 0x6240);
    lo[i + 1] = __byte_perm(a, b, 0x7351);
    a = hi[i];
    b = hi[i + 1];
    hi[i] = __byte_perm(a, b, 0x6240);
    hi[i + 1] = __byte_perm(a, b, 0x7351);
  }
}

// rows v[s] <- v[(s + r) & 7] for r in 0..7 (three conditional rotations)
__device__ __forceinline__ void rotate8(uint32_t (&lo)[8], uint32_t (&hi)[8], int r) {
#pragma unroll
  for (int bit = 0; bit < 3; ++bit) {
    const int d = 1 << bit;
    const bool on = (r >> bit) & 1;
    uint32_t l2[8], h2[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      l2[s] = on ? lo[(s + d) & 7] : lo[s];
      h2[s] = on ? hi[(s + d) & 7] : hi[s];
    }
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      lo[s] = l2[s];
      hi[s] = h2[s];
    }
  }
}

__global__ void __launch_bounds__(kTThreads, 1)
    transpose_codes_kernel(const __grid_constant__ CUtensorMap tmIn, const __grid_constant__ CUtensorMap tmOut,
                           int32_t nrb, int32_t ncb, const float *__restrict__ sw, float *__restrict__ swt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sIn = base;                                 // [kTStages][128][128]
  uint8_t *sOut = base + kTStages * kTTileBytes;       // [kTOut][128][128], 128-byte swizzle
  uint64_t *full = reinterpret_cast<uint64_t *>(sOut + kTOut * kTTileBytes);
  uint64_t *empty = full + kTStages;
  uint64_t *ofree = empty + kTStages;  // [kTOut] the output buffer's previous store has read it
  uint64_t *ofull = ofree + kTOut;     // every transposing thread has written the current output tile
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ofull + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = nrb * ncb;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kTWarps);
    }
    for (int b = 0; b < kTOut; ++b) mbar_init(&ofree[b], 1);
    mbar_init(ofull, 32 * kTWarps);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kTWarps && lane == 0) {
    prefetch_tensormap(&tmIn);
    prefetch_tensormap(&tmOut);
  }
  __syncthreads();

  if (warp == kTWarps) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kSiteProducerEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], kTTileBytes);
        tma_load_2d(sIn + stage * kTTileBytes, &tmIn, &full[stage], (t % ncb) * kTT, (t / ncb) * kTT);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kTStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {  // every load issued must land before the CTA may exit
        for (int s = 0; s < kTStages; ++s)
          if (armed >> s & 1u) mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, kSiteDrain);
      }
    } else {
      // the tiles' scales: a 128 x 128 tile is one scale block, so sw[rb][cb]
      // goes to swt[cb][rb] (lanes 1..31, one tile each per pass)
      for (int t = blockIdx.x + (lane - 1) * (int)gridDim.x; t < total; t += 31 * (int)gridDim.x)
        swt[(int64_t)(t % ncb) * nrb + t / ncb] = __ldg(sw + (int64_t)(t / ncb) * ncb + t % ncb);
    }
  } else {
    // ------------------------------------------------------------------ transposers
    const int tid = threadIdx.x;
    const int br = tid >> 4, bc = tid & 15;  // the thread's 8 x 8 block: input rows 8 br, columns 8 bc
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x, k = 0; t < total; t += gridDim.x, ++k) {
      const bool got = mbar_wait(&full[stage], phase, abort_flag, kSiteMmaFull);
      if (!__all_sync(0xffffffffu, got)) break;
      uint32_t lo[8], hi[8];
      const uint8_t *src = sIn + stage * kTTileBytes + (8 * br) * kTT + 8 * bc;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src + i * kTT);
        lo[i] = v.x;
        hi[i] = v.y;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);  // the stage has been read
      if (++stage == kTStages) {
        stage = 0;
        phase ^= 1;
      }
      transpose8x8(lo, hi);     // row j: output row 8 bc + j, bytes 8 br .. 8 br + 7
      rotate8(lo, hi, bc & 7);  // row s: output row 8 bc + ((s + bc) & 7)
      // output buffer b's use u = k / 2, once its store of use u - 1 has read it
      const int b = k & 1;
      const bool free_ok = mbar_wait(&ofree[b], (uint32_t)(((k >> 1) & 1) ^ 1), abort_flag, kSiteEpiTmemFull);
      if (!__all_sync(0xffffffffu, free_ok)) break;
      uint8_t *dst = sOut + b * kTTileBytes;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int r = 8 * bc + ((s + bc) & 7);
        const int off = r * kTT + ((((br >> 1) ^ (r & 7)) << 4) | ((br & 1) << 3));
        *reinterpret_cast<uint2 *>(dst + off) = make_uint2(lo[s], hi[s]);
      }
      fence_proxy_async_smem();
      mbar_arrive(ofull);
      bool stored = true;
      if (tid == 0) {
        // every thread's part is written: store the tile, then hand the other
        // buffer back once its store (the previous tile's) has read it
        stored = mbar_wait(ofull, (uint32_t)(k & 1), abort_flag, kSiteEpiTmemFull);
        if (stored) {
          tma_store_2d(&tmOut, dst, (t / ncb) * kTT, (t % ncb) * kTT);
          bulk_commit_group();
          bulk_wait_group_read1();
          if (k > 0) mbar_arrive(&ofree[b ^ 1]);  // the previous tile's store (buffer b ^ 1) is done reading
        }
      }
      if (!__all_sync(0xffffffffu, stored)) break;  // warp 0 leaves as a whole
    }
    if (tid == 0) bulk_wait_group_read0();  // the stores have read shared memory before the CTA exits
  }
}

}  // namespace

fp8bq_status launch_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *qt, int64_t ldqt, float *st,
                                int64_t ldst, int mode, cudaStream_t stream) {
  const int64_t gx = (K + kTCol - 1) / kTCol, gy = (M + kTTok - 1) / kTTok;
  if (gx > 0x7fffffff || gy > 65535) return FP8BQ_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)gx, (unsigned)gy);
  const uint16_t *xs = static_cast<const uint16_t *>(x);
  if (mode == FP8BQ_SCALE_FP32)
    quant_act_t_kernel<FP8BQ_SCALE_FP32><<<grid, 256, 0, stream>>>(xs, M, K, ldx, qt, ldqt, st, ldst);
  else
    quant_act_t_kernel<FP8BQ_SCALE_POW2><<<grid, 256, 0, stream>>>(xs, M, K, ldx, qt, ldqt, st, ldst);
  return check_launch("quant_act_t");
}

fp8bq_status launch_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw,
                                     uint8_t *qt, int64_t ldqt, float *swt, cudaStream_t stream) {
  // q [N][K] in 128 x 128-byte boxes; q^T [K][N] stored through the 128-byte swizzle
  CUtensorMap tIn, tOut;
  if (!make_tmap_2d(&tIn, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)K, (uint64_t)N, (uint64_t)ldq, kTT, kTT,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tOut, CU_TENSOR_MAP_DATA_TYPE_UINT8, qt, (uint64_t)N, (uint64_t)K, (uint64_t)ldqt, kTT, kTT,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8BQ_ERR_INVALID_ARG;
  const int64_t nrb = (N + kTT - 1) / kTT, ncb = (K + kTT - 1) / kTT;
  if (nrb * ncb > 0x7fffffff) return FP8BQ_ERR_UNSUPPORTED;
  static DeviceOnce once;
  const fp8bq_status ready = once.get([](int) {
    const cudaError_t e =
        cudaFuncSetAttribute(transpose_codes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTSmemBytes);
    return e == cudaSuccess ? FP8BQ_OK : cuda_fail(e, "cudaFuncSetAttribute(transpose_codes)");
  });
  if (ready != FP8BQ_OK) return ready;
  const int grid = (int)std::min<int64_t>(nrb * ncb, 2 * (int64_t)num_sms());
  transpose_codes_kernel<<<grid, kTThreads, kTSmemBytes, stream>>>(tIn, tOut, (int32_t)nrb, (int32_t)ncb, sw, swt);
  return check_launch("transpose_weight");
}

}  // namespace fp8bq

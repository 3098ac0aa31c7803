// Causal (prefill) attention over FP8 queries, keys and values on the tcgen05
// tensor cores (sm_100a).
//
// Method: "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
// Training", section "Real-world performance gains": an FP8 KV cache and FP8
// attention take the recipe's speedup from the linear layers' 15-25% to about
// 48%.  Every query, key and value head vector (D = 128) is one 1x128 tile of
// section "Technical breakthrough": E4M3 codes and one scale.  This kernel is
// the many-query (prefill) case; both contractions take E4M3 operands.
//
// Work unit: (sequence b, query head h, tile t of 128 query rows).  It reads
// key/value head g = h / (Hq / Hkv) and attends key blocks 0..t (128 keys
// each); in block t keys past the query row are masked.  One persistent CTA
// per SM walks the units longest first (units with the same tile index are
// consecutive), so the tail of the grid is made of short units.
//
// Per key block (n counts the blocks a CTA has processed; buffers alternate
// with n):
//   MMA thread      S[n%2]  = Q . K^T       tcgen05.mma kind::f8f6f4, 128x128x128:
//                                           exact E4M3 products, FP32 sums in TMEM
//                   O~[n%2] = P' . V        P' (below) as A; V straight from the
//                                           cache layout [token][d], i.e. read
//                                           MN-major as the B operand
//   row warps       two threads per query row r (TMEM lane r), each with
//                   half of every key block and half of the output columns:
//                   s_j  = S_rj * ks_j      (the key's scale)
//                   m    = running max of c s_j, c = scale * log2(e) * qs_r
//                   p_j  = 2^(c s_j - m)    (0 for masked keys)
//                   l    = 2^(m_old - m) l + sum_j p_j
//                   P'_rj = E4M3(p_j * 256 vs_j / vmax)   with vmax the block's
//                          largest value scale: P' lies in [0, 256]
//   and, one block later, O_r = 2^(m_old - m) O_r + (vmax / 256) O~_r
//                   (FP32 registers), after the last block bf16(O_r / l).
// The weights p_j enter the value product rounded to E4M3 (relative error at
// most 2^-4 each, as for any FP8 operand); the row sum l uses the unrounded
// p_j.  Everything else is FP32.
//
// Roles (384 threads): warp 0 issues the TMA loads of Q, K and V; warp 1 owns
// TMEM and issues the MMAs; warps 2 and 3 load the key and value scales of
// alternate blocks and form 256 vs_j / vmax; warps 4-11 (two per scheduler,
// so one's latency hides behind the other's work) run the softmax, the
// output correction and the output, the two halves of a row exchanging their
// maxima per block and their sums per unit through shared memory.
// Waits are bounded (a second); on expiry the kernel records the site in the
// device error word and every role stops.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>

#include "device.cuh"
#include "internal.h"
#include "quant.cuh"

namespace fp8bq {
namespace {

constexpr int kD = 128;                  // head dimension
constexpr int kBQ = 128;                 // query rows per unit
constexpr int kBK = 128;                 // keys per block
constexpr int kTile = 128 * 128;         // bytes of one 128x128 E4M3 tile
constexpr int kStages = 4;               // key/value ring
constexpr int kScaleSlot = 2 * kBK * 4 + 16;  // ks[128], 256 vs / vmax [128], vmax
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 56;
constexpr int kHighRegs = 224;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kTmemCols = 512;           // S[2] at 0, 128; O~[2] at 256, 384
// kv ring, four full/empty pairs of two (q, s, p, o), the row maxima's
// exchange (two), the row sums' exchange, drain
constexpr int kNumBars = 2 * kStages + 4 * 2 * 2 + 2 + 1 + 1;
constexpr int kSmemBytes = 1024 + 2 * kTile /* Q */ + 2 * kStages * kTile /* K, V */ + 2 * kTile /* P' */ +
                           kStages * kScaleSlot + 2 * 2 * kBQ * 4 /* half-row maxima */ +
                           2 * kBQ * 4 /* half-row sums */ + kNumBars * 8 + 16;
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum AttnWaitSite : unsigned {
  kSiteAttnQ = 20,
  kSiteAttnKV = 21,
  kSiteAttnS = 22,
  kSiteAttnP = 23,
  kSiteAttnO = 24,
  kSiteAttnStat = 25,
};

struct AttnArgs {
  const float *qs, *ks, *vs;  // scales [B][S][Hq], [B][S][Hkv]
  const int32_t *lens;        // [B]
  uint16_t *o;                // bf16 bits [B][S][Hq][128]
  int32_t B, S, Hq, Hkv, T;   // T = ceil(S / 128)
  float c0;                   // softmax scale * log2(e)
};

struct Unit {
  int b, h, g, t, L, nblk;
};

__device__ __forceinline__ Unit unit_at(int u, const AttnArgs &a) {
  Unit x;
  const int per = a.B * a.Hq;
  x.t = a.T - 1 - u / per;
  const int r = u - (u / per) * per;
  x.b = r / a.Hq;
  x.h = r - x.b * a.Hq;
  x.g = x.h / (a.Hq / a.Hkv);
  int L = __ldg(a.lens + x.b);
  x.L = L < 0 ? 0 : (L > a.S ? a.S : L);
  x.nblk = kBQ * x.t < x.L ? x.t + 1 : 0;
  return x;
}

// The key blocks a CTA processes, in its order (n counts them): units
// blockIdx.x, blockIdx.x + gridDim.x, ..., blocks 0 .. nblk-1 of each.
struct BlockIter {
  const AttnArgs *a;
  int nunits, u, kb;
  Unit x;
  uint32_t n;
  bool valid;
  __device__ BlockIter(const AttnArgs &args, int nu) : a(&args), nunits(nu), u((int)blockIdx.x - (int)gridDim.x),
                                                        kb(0), n(0), valid(true) {
    x.nblk = 0;
    next_unit();
  }
  __device__ void next_unit() {
    kb = 0;
    for (u += gridDim.x; u < nunits; u += gridDim.x) {
      x = unit_at(u, *a);
      if (x.nblk > 0) return;
    }
    valid = false;
  }
  __device__ void advance() {
    if (!valid) return;
    ++n;
    if (++kb == x.nblk) next_unit();
  }
  // advance to the first block at or after this one with n % 2 == parity
  __device__ void skip_to(uint32_t parity) {
    if (valid && (n & 1u) != parity) advance();
  }
  // key and value scales of keys 4 lane .. 4 lane + 3 of this block (0 past
  // the sequence's length, and when there is no block)
  __device__ void load(int lane, float (&k)[4], float (&v)[4]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = kBK * kb + 4 * lane + i;
      const bool live = valid && j < x.L;
      const int64_t idx = ((int64_t)x.b * a->S + j) * a->Hkv + x.g;
      k[i] = live ? __ldg(a->ks + idx) : 0.f;
      v[i] = live ? __ldg(a->vs + idx) : 0.f;
    }
  }
};

// Shared-memory descriptor of an MN-major operand tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes hold 128 consecutive MN elements, one
// row per K index; 8-row (1024-byte) swizzle atoms follow each other along K.
// The stride between atoms along K (the stride-dimension offset) is 1024
// bytes; the tile is one atom wide along MN, so the leading-dimension offset
// (the stride between atoms along MN) is never used and is set to the same
// 1024 bytes.  Version 1, swizzle mode 2 = 128-byte.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(1024u >> 4) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Bars {
  uint64_t *kv_full, *kv_empty;   // [kStages]
  uint64_t *q_full, *q_empty;     // [2]
  uint64_t *s_full, *s_empty;     // [2]
  uint64_t *p_full, *p_empty;     // [2]
  uint64_t *o_full, *o_empty;     // [2]
  uint64_t *xbar;                 // [2] the row warps' half-row maxima of block n are in sMx[n % 2]
  uint64_t *lbar;                 // the row warps' half-row sums of the unit are in sL
  uint64_t *drain;
};

__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = base;                       // [2][128 rows x 128 B]
  uint8_t *sK = sQ + 2 * kTile;             // [kStages]
  uint8_t *sV = sK + kStages * kTile;       // [kStages]
  uint8_t *sP = sV + kStages * kTile;       // [2]
  uint8_t *sScale = sP + 2 * kTile;         // [kStages][kScaleSlot]
  float *sMx = reinterpret_cast<float *>(sScale + kStages * kScaleSlot);  // [2 blocks][2 halves][128 rows]
  float *sL = sMx + 2 * 2 * kBQ;                                          // [2 halves][128 rows]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sL + 2 * kBQ);
  Bars B;
  B.kv_full = bar;
  B.kv_empty = bar + kStages;
  B.q_full = bar + 2 * kStages;
  B.q_empty = B.q_full + 2;
  B.s_full = B.q_empty + 2;
  B.s_empty = B.s_full + 2;
  B.p_full = B.s_empty + 2;
  B.p_empty = B.p_full + 2;
  B.o_full = B.p_empty + 2;
  B.o_empty = B.o_full + 2;
  B.xbar = B.o_empty + 2;
  B.lbar = B.xbar + 2;
  B.drain = B.lbar + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(B.drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nunits = args.B * args.Hq * args.T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&B.kv_full[s], 2);      // the TMA arm (with its bytes) + the scale writers
      mbar_init(&B.kv_empty[s], 1 + 8); // the value MMA's commit + the eight row warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.q_full[i], 1);
      mbar_init(&B.q_empty[i], 1);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.s_empty[i], 8);
      mbar_init(&B.p_full[i], 8);
      mbar_init(&B.p_empty[i], 1);
      mbar_init(&B.o_full[i], 1);
      mbar_init(&B.o_empty[i], 8);
      mbar_init(&B.xbar[i], 8);
    }
    mbar_init(B.lbar, 8);
    mbar_init(B.drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0) {
      // ------------------------------------------------------------------ loads
      uint32_t n = 0, v = 0;
      uint32_t armed = 0, armed_par = 0, qarmed = 0, qarmed_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const Unit x = unit_at(u, args);
        if (x.nblk == 0) continue;
        const int qb = v & 1;
        const uint32_t qph = (v >> 1) & 1;
        if (lane == 0) {
          ok = mbar_wait(&B.q_empty[qb], qph ^ 1, abort_flag, kSiteAttnQ);
          if (ok) {
            mbar_arrive_expect_tx(&B.q_full[qb], kTile);
            tma_load_3d(sQ + qb * kTile, &tmQ, &B.q_full[qb], 0, x.h, x.b * args.S + kBQ * x.t);
            qarmed |= 1u << qb;
            qarmed_par = (qarmed_par & ~(1u << qb)) | (qph << qb);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        for (int kb = 0; kb < x.nblk; ++kb, ++n) {
          const int st = n % kStages;
          const uint32_t ph = (n / kStages) & 1;
          if (lane == 0) {
            ok = mbar_wait(&B.kv_empty[st], ph ^ 1, abort_flag, kSiteAttnKV);
            if (ok) {
              mbar_arrive_expect_tx(&B.kv_full[st], 2 * kTile);
              const int tok = x.b * args.S + kBK * kb;
              tma_load_3d(sK + st * kTile, &tmK, &B.kv_full[st], 0, x.g, tok);
              tma_load_3d(sV + st * kTile, &tmV, &B.kv_full[st], 0, x.g, tok);
              armed |= 1u << st;
              armed_par = (armed_par & ~(1u << st)) | (ph << st);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
        ++v;
      }
      if (!ok && lane == 0) {  // loads already issued must land before the CTA may exit
        for (int s = 0; s < kStages; ++s)
          if (armed >> s & 1u) mbar_wait(&B.kv_full[s], (armed_par >> s) & 1u, nullptr, kSiteDrain);
        for (int s = 0; s < 2; ++s)
          if (qarmed >> s & 1u) mbar_wait(&B.q_full[s], (qarmed_par >> s) & 1u, nullptr, kSiteDrain);
      }
    } else if (warp >= 2) {
      // ------------------------------------------------------------------ key / value scales
      // Warp 2 serves the even blocks (in the CTA's block order n), warp 3 the
      // odd ones, each with the next block's loads in flight while it waits for
      // the current block's stage: lane l takes keys 4l .. 4l+3 of the block;
      // keys at or past the sequence's length are never visible and get 0.
      const uint32_t mine = (uint32_t)(warp - 2);
      BlockIter it(args, nunits);
      it.skip_to(mine);
      float kc[4], vc[4];
      it.load(lane, kc, vc);
      bool ok = true;
      while (it.valid && ok) {
        const uint32_t n = it.n;
        BlockIter nx = it;
        nx.advance();
        nx.skip_to(mine);
        float kn[4], vn[4];
        nx.load(lane, kn, vn);  // in flight during the wait below
        const int st = n % kStages;
        if (lane == 0) ok = mbar_wait(&B.kv_empty[st], ((n / kStages) & 1) ^ 1, abort_flag, kSiteAttnKV);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        float vmax = fmaxf(fmaxf(vc[0], vc[1]), fmaxf(vc[2], vc[3]));
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, d));
        const float inv = vmax > 0.f ? __fdiv_rn(256.f, vmax) : 0.f;
        float *slot = reinterpret_cast<float *>(sScale + st * kScaleSlot);
        reinterpret_cast<float4 *>(slot)[lane] = make_float4(kc[0], kc[1], kc[2], kc[3]);
        reinterpret_cast<float4 *>(slot + kBK)[lane] = make_float4(vc[0] * inv, vc[1] * inv, vc[2] * inv, vc[3] * inv);
        if (lane == 0) slot[2 * kBK] = vmax * (1.f / 256.f);
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.kv_full[st]);
        it = nx;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          kc[i] = kn[i];
          vc[i] = vn[i];
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      const uint32_t idesc_s = idesc_f8f6f4_e4m3_f32(kBQ, kBK);
      const uint32_t idesc_o = idesc_f8f6f4_e4m3_f32(kBQ, kD) | (1u << 16);  // B (V) MN-major
      uint32_t n = 0, v = 0;
      bool ok = true, issued = false;
      // the value product of block m: O~[m%2] = P'[m%2] . V[stage(m)]
      auto pv = [&](uint32_t m) -> bool {
        const int pb = m & 1;
        const uint32_t pph = (m >> 1) & 1;
        if (!mbar_wait(&B.p_full[pb], pph, abort_flag, kSiteAttnP) ||
            !mbar_wait(&B.o_empty[pb], pph ^ 1, abort_flag, kSiteAttnO))
          return false;
        tc_fence_after();
        const int st = m % kStages;
        const uint32_t d = tmem_base + 256u + 128u * (uint32_t)pb;
        const uint32_t a0 = smem_addr(sP + pb * kTile);
        const uint32_t b0 = smem_addr(sV + st * kTile);
#pragma unroll
        for (int k = 0; k < kBK / 32; ++k)
          mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_mn_sw128(b0 + 4096 * k), idesc_o, k > 0 ? 1u : 0u);
        mma_commit(&B.o_full[pb]);
        mma_commit(&B.p_empty[pb]);
        mma_commit(&B.kv_empty[st]);
        issued = true;
        return true;
      };
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const Unit x = unit_at(u, args);
        if (x.nblk == 0) continue;
        const int qb = v & 1;
        if (!mbar_wait(&B.q_full[qb], (v >> 1) & 1, abort_flag, kSiteAttnQ)) {
          ok = false;
          break;
        }
        for (int kb = 0; kb < x.nblk; ++kb, ++n) {
          const int st = n % kStages;
          const int sb = n & 1;
          if (!mbar_wait(&B.kv_full[st], (n / kStages) & 1, abort_flag, kSiteAttnKV) ||
              !mbar_wait(&B.s_empty[sb], ((n >> 1) & 1) ^ 1, abort_flag, kSiteAttnS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + 128u * (uint32_t)sb;
          const uint32_t a0 = smem_addr(sQ + qb * kTile);
          const uint32_t b0 = smem_addr(sK + st * kTile);
#pragma unroll
          for (int k = 0; k < kD / 32; ++k)
            mma_f8f6f4(d, smem_desc_k_sw128(a0 + 32 * k), smem_desc_k_sw128(b0 + 32 * k), idesc_s, k > 0 ? 1u : 0u);
          mma_commit(&B.s_full[sb]);
          if (kb == x.nblk - 1) mma_commit(&B.q_empty[qb]);
          issued = true;
          if (kb > 0 && !pv(n - 1)) {
            ok = false;
            break;
          }
        }
        if (ok && !pv(n - 1)) ok = false;
        ++v;
      }
      if (!ok && issued) {  // TMEM and the operand tiles must be quiescent before the CTA exits
        mma_commit(B.drain);
        mbar_wait(B.drain, 0, nullptr, kSiteDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // -------------------------------------------------------------------- rows: softmax, correction, output
    // Query row r (TMEM lane r) is shared by two threads of the same lane
    // quarter: hf = 0 (warps 4-7) takes keys 0-63 of every block and output
    // columns 0-63, hf = 1 (warps 8-11) keys 64-127 and columns 64-127.  They
    // exchange their partial row maxima once per block and their partial row
    // sums once per unit through shared memory.  The value product of block n
    // is folded into the output while block n + 1's softmax is done.
    const int quarter = warp & 3;
    const int hf = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;  // query row within the unit = TMEM lane
    const int jo = 64 * hf;             // this thread's first key of a block and first output column
    const uint32_t lane_base = tmem_base + ((uint32_t)(quarter * 32) << 16);
    uint32_t n = 0, lph = 0;
    bool ok = true;
    // the eight row warps meet at `bar` (bounded wait)
    auto meet = [&](uint64_t *bar, uint32_t parity) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kSiteAttnStat));
    };
    float2 acc[32];  // output columns jo .. jo + 63, in pairs
    // O = al O + fa O~[nn % 2] (the value product of the CTA's block nn)
    auto correct = [&](uint32_t nn, float al, float fa) -> bool {
      const int ob = nn & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&B.o_full[ob], (nn >> 1) & 1, abort_flag, kSiteAttnO))) return false;
      tc_fence_after();
      uint32_t pr[64];
      const uint32_t taddr = lane_base + 256u + 128u * (uint32_t)ob + (uint32_t)jo;
      tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&B.o_empty[ob]);
      const float2 al2 = make_float2(al, al), f2 = make_float2(fa, fa);
#pragma unroll
      for (int k = 0; k < 32; ++k)
        acc[k] = __ffma2_rn(make_float2(__uint_as_float(pr[2 * k]), __uint_as_float(pr[2 * k + 1])), f2,
                            __fmul2_rn(acc[k], al2));
      return true;
    };
    for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
      const Unit x = unit_at(u, args);
      const int i = kBQ * x.t + r;
      uint4 *dst = reinterpret_cast<uint4 *>(args.o + (((int64_t)x.b * args.S + i) * args.Hq + x.h) * kD + jo);
      if (x.nblk == 0) {  // the whole tile is at or past the sequence's length: zeros
        if (i < args.S)
#pragma unroll
          for (int k = 0; k < 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const float qsc = i < args.S ? __ldg(args.qs + ((int64_t)x.b * args.S + i) * args.Hq + x.h) : 0.f;
      const float c = args.c0 * qsc;
      float m = -INFINITY, l = 0.f, al_prev = 0.f, fa_prev = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) acc[k] = make_float2(0.f, 0.f);
      for (int kb = 0; kb < x.nblk; ++kb, ++n) {
        const int st = n % kStages;
        const int sb = n & 1;
        const uint32_t sph = (n >> 1) & 1;
        bool got = mbar_wait(&B.s_full[sb], sph, abort_flag, kSiteAttnS);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        const uint32_t taddr = lane_base + 128u * (uint32_t)sb + (uint32_t)jo;
        tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&B.s_empty[sb]);
        got = mbar_wait(&B.kv_full[st], (n / kStages) & 1, abort_flag, kSiteAttnKV);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const float *slot = reinterpret_cast<const float *>(sScale + st * kScaleSlot);
        const float4 *ks4 = reinterpret_cast<const float4 *>(slot + jo);
        const float4 *rv4 = reinterpret_cast<const float4 *>(slot + kBK + jo);
        const float fa = slot[2 * kBK];
        // s_j = S_rj * ks_j and this half's row max over the visible keys
        // (masking by selects; four partial maxima and sums keep the
        // dependency chains short)
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        auto scale_max = [&](auto masked, int vis) {  // vis: last visible key of this half (< 0: none)
#pragma unroll
          for (int j4 = 0; j4 < 16; ++j4) {
            const float4 k4 = ks4[j4];
            float sv[4] = {__uint_as_float(sr[4 * j4 + 0]) * k4.x, __uint_as_float(sr[4 * j4 + 1]) * k4.y,
                           __uint_as_float(sr[4 * j4 + 2]) * k4.z, __uint_as_float(sr[4 * j4 + 3]) * k4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if constexpr (decltype(masked)::value) sv[e] = 4 * j4 + e <= vis ? sv[e] : -INFINITY;
              sr[4 * j4 + e] = __float_as_uint(sv[e]);
              mx4[e] = fmaxf(mx4[e], sv[e]);
            }
          }
        };
        // only the diagonal block (the unit's last) has keys after the row
        if (kb == x.t) scale_max(std::true_type(), r - jo);
        else scale_max(std::false_type(), 63);
        sMx[(sb * 2 + hf) * kBQ + r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        if (!meet(&B.xbar[sb], sph)) {
          ok = false;
          break;
        }
        const float mx = fmaxf(sMx[(sb * 2) * kBQ + r], sMx[(sb * 2 + 1) * kBQ + r]);
        // c > 0, so the max of c s is c times the max of s
        const float m_new = fmaxf(m, c * mx);
        const float alpha = ex2(m - m_new);  // 0 on the first block (m = -inf)
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[16];  // 64 E4M3 codes, 4 per word
#pragma unroll
        for (int j4 = 0; j4 < 16; ++j4) {
          const float4 w4 = rv4[j4];
          float p[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            p[e] = ex2(__fmaf_rn(c, __uint_as_float(sr[4 * j4 + e]), -m_new));  // masked keys: 2^-inf = 0
            sum4[e] += p[e];
          }
          const uint32_t lo = qdev::e4m3x2(p[0] * w4.x, p[1] * w4.y);
          const uint32_t hi = qdev::e4m3x2(p[2] * w4.z, p[3] * w4.w);
          pk[j4] = lo | (hi << 16);
        }
        l = alpha * l + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
        m = m_new;
        // this half of P' row r into the 128-byte-swizzled K-major tile
        got = mbar_wait(&B.p_empty[sb], sph ^ 1, abort_flag, kSiteAttnP);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        uint8_t *prow = sP + sb * kTile + r * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ch = 4 * hf + cc;
          *reinterpret_cast<uint4 *>(prow + ((ch ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&B.p_full[sb]);
          mbar_arrive(&B.kv_empty[st]);  // this warp has read the stage's scales
        }
        // the previous block's value product, while the MMA runs this one's
        if (kb > 0 && !correct(n - 1, al_prev, fa_prev)) {
          ok = false;
          break;
        }
        al_prev = alpha;
        fa_prev = fa;
      }
      if (!ok || !correct(n - 1, al_prev, fa_prev)) break;  // the unit's last block
      // the row sum: this half's plus the other's (in half order)
      sL[hf * kBQ + r] = l;
      if (!meet(B.lbar, lph)) break;
      lph ^= 1;
      const float lt = sL[r] + sL[kBQ + r];
      if (i < args.S) {
        // rows at or past the sequence's length are 0
        const bool live = i < x.L;
        const float inv = live ? __fdiv_rn(1.f, lt) : 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = acc[4 * k + e];
            __nv_bfloat162 bv = __floats2bfloat162_rn(live ? a.x * inv : 0.f, live ? a.y * inv : 0.f);
            w[e] = *reinterpret_cast<uint32_t *>(&bv);
          }
          dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

DeviceOnce g_prefill_once;

}  // namespace

cudaError_t take_device_error_prefill_attn(unsigned long long *v) { return take_tu_device_error(v); }

fp8bq_status launch_prefill_attention(const uint8_t *qq, const float *qs, const uint8_t *kq, const float *ks,
                                      const uint8_t *vq, const float *vs, const int32_t *lens, int64_t B, int64_t S,
                                      int64_t Hq, int64_t Hkv, float scale, void *o, cudaStream_t stream) {
  const fp8bq_status ready = g_prefill_once.get([](int) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, prefill_attn_kernel);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(prefill attention)");
    if (fa.numRegs != kLaunchRegs) return FP8BQ_ERR_UNSUPPORTED;
    e = cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill attention)");
    return FP8BQ_OK;
  });
  if (ready != FP8BQ_OK) return ready;
  const uint64_t tokens = (uint64_t)B * (uint64_t)S;
  CUtensorMap tQ, tK, tV;
  if (!make_tmap_3d(&tQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, qq, kD, (uint64_t)Hq, tokens, kD, (uint64_t)Hq * kD, kD, 1,
                    CU_TENSOR_MAP_SWIZZLE_128B, kBQ) ||
      !make_tmap_3d(&tK, CU_TENSOR_MAP_DATA_TYPE_UINT8, kq, kD, (uint64_t)Hkv, tokens, kD, (uint64_t)Hkv * kD, kD, 1,
                    CU_TENSOR_MAP_SWIZZLE_128B, kBK) ||
      !make_tmap_3d(&tV, CU_TENSOR_MAP_DATA_TYPE_UINT8, vq, kD, (uint64_t)Hkv, tokens, kD, (uint64_t)Hkv * kD, kD, 1,
                    CU_TENSOR_MAP_SWIZZLE_128B, kBK))
    return FP8BQ_ERR_INVALID_ARG;
  AttnArgs a;
  a.qs = qs;
  a.ks = ks;
  a.vs = vs;
  a.lens = lens;
  a.o = static_cast<uint16_t *>(o);
  a.B = (int32_t)B;
  a.S = (int32_t)S;
  a.Hq = (int32_t)Hq;
  a.Hkv = (int32_t)Hkv;
  a.T = (int32_t)((S + kBQ - 1) / kBQ);
  a.c0 = scale * 1.4426950408889634f;
  const int64_t units = B * Hq * (int64_t)a.T;
  const int grid = (int)std::min<int64_t>(units, num_sms());
  prefill_attn_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tQ, tK, tV, a);
  return check_launch("prefill attention");
}

}  // namespace fp8bq

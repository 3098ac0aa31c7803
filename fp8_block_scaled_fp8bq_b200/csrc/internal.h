// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string.h>

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "../../include/fp8bq.h"

namespace fp8bq {

// Largest expert count of fp8bq_grouped_gemm (the device scheduler keeps the
// offsets and the tile prefix of all experts in shared memory).
constexpr int kMaxExperts = 1024;

// Highest device ordinal + 1 for which the library keeps per-device state.
constexpr int kMaxDevices = 64;

// Number of SMs of the current device (cached per device).
int num_sms();

// Record the failing CUDA call for diagnostics and map it to FP8BQ_ERR_CUDA.
fp8bq_status cuda_fail(cudaError_t e, const char *what);

// The result of a per-device one-time set-up (a kernel attribute opt-in, a
// register-count check, a symbol lookup), safe to call from several host
// threads: the first caller on a device runs `setup(dev)` under a mutex,
// later callers read the cached status without locking.  Definite answers
// (FP8BQ_OK, FP8BQ_ERR_UNSUPPORTED) are cached; a failing CUDA call is not, so
// the next call tries again.  A device ordinal outside [0, kMaxDevices) is
// FP8BQ_ERR_UNSUPPORTED.
class DeviceOnce {
 public:
  // For the current device.
  template <class F>
  fp8bq_status get(F &&setup) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    return get_for(dev, setup);
  }

  template <class F>
  fp8bq_status get_for(int dev, F &&setup) {
    if (dev < 0 || dev >= kMaxDevices) return FP8BQ_ERR_UNSUPPORTED;
    int v = state_[dev].load(std::memory_order_acquire);
    if (v != 0) return static_cast<fp8bq_status>(v - 1);
    std::lock_guard<std::mutex> lock(mutex_);
    v = state_[dev].load(std::memory_order_relaxed);
    if (v != 0) return static_cast<fp8bq_status>(v - 1);
    const fp8bq_status st = setup(dev);
    if (st == FP8BQ_OK || st == FP8BQ_ERR_UNSUPPORTED) state_[dev].store(st + 1, std::memory_order_release);
    return st;
  }

 private:
  std::atomic<int> state_[kMaxDevices] = {};  // 0: not yet; else status + 1
  std::mutex mutex_;
};

// Encoded TMA descriptors, keyed by everything that goes into one.  A
// descriptor holds nothing beyond its arguments, so an entry stays valid for
// as long as a caller passes the same pointer and shape.  Guarded by a mutex;
// emptied when it holds kCapacity entries.
struct TensorMapKey {
  const void *base;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  int32_t rank, dtype, swizzle;  // no implicit padding: compared and hashed as bytes
};
static_assert(sizeof(TensorMapKey) == 72, "TensorMapKey has no padding");

class TensorMapCache {
 public:
  static constexpr size_t kCapacity = 4096;
  bool find(const TensorMapKey &k, CUtensorMap *out) {
    std::lock_guard<std::mutex> lock(mutex_);
    auto it = maps_.find(Bytes(k));
    if (it == maps_.end()) return false;
    *out = it->second;
    return true;
  }
  void insert(const TensorMapKey &k, const CUtensorMap &m) {
    std::lock_guard<std::mutex> lock(mutex_);
    if (maps_.size() >= kCapacity) maps_.clear();
    maps_[Bytes(k)] = m;
  }
  size_t size() {
    std::lock_guard<std::mutex> lock(mutex_);
    return maps_.size();
  }

 private:
  struct Bytes {
    unsigned char b[sizeof(TensorMapKey)];
    explicit Bytes(const TensorMapKey &k) { memcpy(b, &k, sizeof(b)); }
    bool operator==(const Bytes &o) const { return memcmp(b, o.b, sizeof(b)) == 0; }
  };
  struct Hash {
    size_t operator()(const Bytes &k) const {
      uint64_t h = 1469598103934665603ull;  // FNV-1a
      for (unsigned char c : k.b) h = (h ^ c) * 1099511628211ull;
      return (size_t)h;
    }
  };
  std::unordered_map<Bytes, CUtensorMap, Hash> maps_;
  std::mutex mutex_;
};

// Check the last launch.
fp8bq_status check_launch(const char *what);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
// Returns false if the driver rejects the map.
bool make_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 3-D variant: dims {d0 (innermost), d1, d2}, byte strides of dims 1 and 2, box {box0, box1, box2}.
bool make_tmap_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                  CUtensorMapSwizzle swizzle, uint32_t box2 = 1);

// Tile order of a persistent GEMM over an M x N output in bm x bn tiles with
// depth K (bytes per operand row = K): picks the banded dimension and the band
// width (see raster_tile) that minimise the operand bytes read from DRAM when
// a band's panels of one operand stay in L2.
void choose_raster(int64_t M, int64_t N, int64_t K, int bm, int bn, int32_t *band, int32_t *n_major);

// Per translation unit: read and clear its device error word.
cudaError_t take_device_error_gemm(unsigned long long *v);
cudaError_t take_device_error_decode(unsigned long long *v);
cudaError_t take_device_error_native(unsigned long long *v);
cudaError_t take_device_error_pair(unsigned long long *v);
cudaError_t take_device_error_swiglu(unsigned long long *v);
cudaError_t take_device_error_wgrad(unsigned long long *v);
cudaError_t take_device_error_prefill_attn(unsigned long long *v);
cudaError_t take_device_error_decode_wide(unsigned long long *v);

// Launchers (arguments already validated).
fp8bq_status launch_encode(const float *x, int64_t n, uint8_t *q, cudaStream_t stream);
fp8bq_status launch_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *sa,
                              int64_t ldsa, int mode, cudaStream_t stream);
fp8bq_status launch_recalibrate(const fp8bq_weight_desc *descs, int n, int mode, cudaStream_t stream);
fp8bq_status launch_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                         int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                         int variant, cudaStream_t stream);
bool pair_gemm_available();
fp8bq_status launch_gemm_pair(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                              int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                              int tile_n, cudaStream_t stream);
fp8bq_status launch_gemm_native(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                cudaStream_t stream);
size_t decode_workspace_size(int64_t M, int64_t N, int64_t K);
// Argument checks of fp8bq_gemm_decode (no device access).  *work is false for
// the no-op sizes (M == 0 or N == 0) and for any error.
fp8bq_status check_decode_args(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw,
                               const void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, bool *work);
fp8bq_status launch_gemm_decode(const void *x, int64_t ldx, const uint8_t *qw, int64_t ldw, const float *sw, void *y,
                                int64_t ldy, int64_t M, int64_t N, int64_t K, int mode, void *ws, size_t ws_bytes,
                                cudaStream_t stream);
// The decode GEMM's wide form (tokens as the 128-row MMA operand, 256 weight
// rows per MMA, K split over clusters of up to 16 CTAs): its launch plan.
struct DecodeWidePlan {
  int NT;              // token rows held per block: M rounded up to 16, 32 or 64
  int MG;              // groups of 64 tokens (M > 64: each weight tile is streamed once per group)
  int S, C;            // CTAs per cluster, clusters
  int nst, nres, smem; // weight stages, resident K-blocks of codes, dynamic shared memory
  bool res;            // activation quantized inside the kernel (no prologue)
};
// FP8BQ_ERR_UNSUPPORTED when the shape is outside the wide form (M > 256).
// vec: the activations allow 16-byte loads.
fp8bq_status plan_decode_wide(int64_t M, int64_t N, int64_t K, bool vec, DecodeWidePlan *p);
// q/sa/ldsa: the prologue's codes and scales (unused when p.res).
fp8bq_status launch_decode_wide(const DecodeWidePlan &p, const uint16_t *x, int64_t ldx, const uint8_t *qw,
                                int64_t ldw, const float *sw, const uint8_t *q, const float *sa, int64_t ldsa,
                                void *y, int64_t ldy, int64_t M, int64_t N, int64_t K, int mode,
                                cudaStream_t stream);
fp8bq_status launch_grouped_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                 const float *sw, const int32_t *offsets, int E, int64_t rows, int64_t N, int64_t K,
                                 void *y, int64_t ldy, cudaStream_t stream);
fp8bq_status launch_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qw,
                                int64_t ldw, const float *sw, uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh,
                                void *h, int64_t ldh, int64_t M, int64_t I, int64_t K, int mode, cudaStream_t stream);
fp8bq_status launch_grouped_gemm_swiglu(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                        const uint8_t *qw, const float *sw, const int32_t *offsets, int E,
                                        int64_t rows, int64_t I, int64_t K, uint8_t *qh, int64_t ldqh, float *sh,
                                        int64_t ldsh, void *h, int64_t ldh, int mode, cudaStream_t stream);
fp8bq_status launch_adamw_recalibrate(const fp8bq_adamw_desc *descs, int n, const fp8bq_adamw_config *cfg, int mode,
                                      cudaStream_t stream);
fp8bq_status launch_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx, uint8_t *qt, int64_t ldqt, float *st,
                                int64_t ldst, int mode, cudaStream_t stream);
fp8bq_status launch_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw,
                                     uint8_t *qt, int64_t ldqt, float *swt, cudaStream_t stream);
fp8bq_status launch_gemm_native_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                      const uint8_t *qb, int64_t ldb, const float *sb, int64_t ldsb, void *y,
                                      int64_t ldy, int64_t N, int64_t K, int64_t M, cudaStream_t stream);
fp8bq_status launch_gemm_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa, const uint8_t *qb,
                               int64_t ldb, const float *sb, int64_t ldsb, void *y, int64_t ldy, int64_t N, int64_t K,
                               int64_t M, cudaStream_t stream);
size_t decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S);
fp8bq_status launch_decode_attention(const void *q, const uint8_t *kq, const float *ks, const uint8_t *vq,
                                     const float *vs, const int32_t *lens, int64_t B, int64_t Hq, int64_t Hkv,
                                     int64_t S, float scale, void *o, void *ws, size_t ws_bytes, cudaStream_t stream);
fp8bq_status launch_prefill_attention(const uint8_t *qq, const float *qs, const uint8_t *kq, const float *ks,
                                      const uint8_t *vq, const float *vs, const int32_t *lens, int64_t B, int64_t S,
                                      int64_t Hq, int64_t Hkv, float scale, void *o, cudaStream_t stream);
fp8bq_status launch_kv_append(const void *k_new, const void *v_new, const int32_t *pos, uint8_t *kq, float *ks,
                              uint8_t *vq, float *vs, int64_t B, int64_t Hkv, int64_t S, int mode,
                              cudaStream_t stream);

}  // namespace fp8bq

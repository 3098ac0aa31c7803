// Tile order of the persistent GEMM kernels (host side): which operand's
// panels stay in L2 while the other operand streams past (see raster_tile in
// device.cuh for the device side of the same order).
#include <algorithm>

#include "internal.h"

namespace fp8bq {

void choose_raster(int64_t M, int64_t N, int64_t K, int bm, int bn, int32_t *band, int32_t *n_major) {
  // Panels of one band must stay in L2 while the other operand and the output
  // stream past them: a third of the 126 MB L2, with room left for the panels
  // in flight and the output lines not yet written back.
  constexpr int64_t kBandBytes = int64_t(40) << 20;
  const int64_t num_m = (M + bm - 1) / bm, num_n = (N + bn - 1) / bn;
  const int64_t a_panel = (int64_t)bm * K, w_panel = (int64_t)bn * K;
  const int64_t band_m = std::max<int64_t>(1, std::min<int64_t>(num_m, kBandBytes / std::max<int64_t>(a_panel, 1)));
  const int64_t band_n = std::max<int64_t>(1, std::min<int64_t>(num_n, kBandBytes / std::max<int64_t>(w_panel, 1)));
  // M bands: A is read once, W once per band; N bands the other way round.
  const int64_t bytes_m = M * K + N * K * ((num_m + band_m - 1) / band_m);
  const int64_t bytes_n = N * K + M * K * ((num_n + band_n - 1) / band_n);
  if (bytes_m <= bytes_n) {
    *band = (int32_t)band_m;
    *n_major = 0;
  } else {
    *band = (int32_t)band_n;
    *n_major = 1;
  }
}

}  // namespace fp8bq

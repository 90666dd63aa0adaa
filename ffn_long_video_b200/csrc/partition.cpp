// Key design 1 of the AdaSpark note (3D spatio-temporal cube partition): maps a
// T x H x W video-token grid to cube-major order. Host code, run once per video.
#include <stdint.h>

#include "adaspark.h"

namespace {
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
}  // namespace

extern "C" int adaspark_cube_count(int T, int H, int W, int cube_h, int cube_w, int cube_t,
                                   int32_t* n_cubes) {
  if (!n_cubes || T <= 0 || H <= 0 || W <= 0 || cube_h <= 0 || cube_w <= 0 || cube_t <= 0)
    return ADASPARK_EINVAL;
  int64_t c = ceil_div(T, cube_t) * ceil_div(H, cube_h) * ceil_div(W, cube_w);
  if (c > INT32_MAX) return ADASPARK_EINVAL;
  *n_cubes = static_cast<int32_t>(c);
  return ADASPARK_OK;
}

extern "C" int adaspark_cube_partition(int T, int H, int W, int cube_h, int cube_w, int cube_t,
                                       int n_text, int32_t* perm, int32_t* cube_ids,
                                       int32_t* cube_offsets, int32_t* n_cubes) {
  int32_t nc = 0;
  if (adaspark_cube_count(T, H, W, cube_h, cube_w, cube_t, &nc) != ADASPARK_OK)
    return ADASPARK_EINVAL;
  if (n_text < 0 || !perm || !cube_ids || !cube_offsets) return ADASPARK_EINVAL;
  const int64_t n_vis = (int64_t)T * H * W;
  if (n_vis + n_text > INT32_MAX) return ADASPARK_EINVAL;
  const int64_t nb_t = ceil_div(T, cube_t), nb_h = ceil_div(H, cube_h), nb_w = ceil_div(W, cube_w);
  int64_t pos = 0;
  int32_t c = 0;
  // Cubes time-major over the cube grid; tokens (t, h, w)-ordered inside a cube.
  for (int64_t tb = 0; tb < nb_t; ++tb) {
    const int64_t t1 = (tb + 1) * cube_t < T ? (tb + 1) * cube_t : T;
    for (int64_t hb = 0; hb < nb_h; ++hb) {
      const int64_t h1 = (hb + 1) * cube_h < H ? (hb + 1) * cube_h : H;
      for (int64_t wb = 0; wb < nb_w; ++wb) {
        const int64_t w1 = (wb + 1) * cube_w < W ? (wb + 1) * cube_w : W;
        cube_offsets[c] = static_cast<int32_t>(pos);
        for (int64_t t = tb * cube_t; t < t1; ++t)
          for (int64_t h = hb * cube_h; h < h1; ++h)
            for (int64_t w = wb * cube_w; w < w1; ++w) {
              perm[pos] = static_cast<int32_t>(t * H * W + h * W + w);
              cube_ids[pos] = c;
              ++pos;
            }
        ++c;
      }
    }
  }
  cube_offsets[c] = static_cast<int32_t>(pos);
  for (int64_t i = 0; i < n_text; ++i) cube_ids[n_vis + i] = -1;
  *n_cubes = c;
  return ADASPARK_OK;
}

// AdaS-Attn attention over the selected cubes, SIMT form (fp32 path): one
// block per 128-row tile, one thread per (token, query head) row, online
// softmax over 64-key blocks staged in shared memory.
//
// Admitted keys of a visual row of cube i (key design 2 of the AdaSpark note):
// every key of a cube j < i whose row bit is set in the tile mask, plus the
// keys of cube i at positions <= t. A text row admits every key u <= t.
#include "attn_kernels.h"

namespace adaspark {

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* ks = reinterpret_cast<float*>(smem_raw);  // [64][D]
  float* vs = ks + 64 * D;                          // [64][D]
  __shared__ int s_hi;
  if (status_bad(a.hdr)) return;
  const AttnGeom& G = a.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool text = blockIdx.x >= (unsigned)G.n_vtiles;
  const int bt = text ? blockIdx.x - G.n_vtiles : blockIdx.x;
  const int kv = bt / (text ? G.ttiles_per_kv : G.vtiles_per_kv);
  const TileRow R = tile_row(G, text, bt, tid);
  const bool valid = R.valid;
  const int t = R.t, h = R.h;
  const int own = (!text && valid) ? a.cube_ids[t] : -1;

  if (tid == 0) s_hi = -1;
  __syncthreads();
  if (valid) atomicMax(&s_hi, text ? t : own);
  __syncthreads();
  const int hi = s_hi;  // visual: highest own cube; text: highest token

  const T* Kp = reinterpret_cast<const T*>(a.K);
  const T* Vp = reinterpret_cast<const T*>(a.V);
  float q[D], o[D];
  {
    const T* qp = reinterpret_cast<const T*>(a.Q) + ((size_t)t * G.hq + h) * D;
#pragma unroll
    for (int e = 0; e < D; ++e) {
      q[e] = valid ? to_f32(qp[e]) * a.scale_log2 : 0.f;
      o[e] = 0.f;
    }
  }
  float m = -INFINITY, l = 0.f;

  // Key blocks: (first key, key count, cube id or -1 for text keys).
  const int n_list = text ? G.n_cubes : (a.dense ? hi + 1 : a.tile_count[bt]);
  const uint16_t* list = a.tile_list + (size_t)bt * G.n_cubes;
  const uint32_t* tm = a.tile_mask + (size_t)bt * G.n_cubes * 4;
  const int n_text_chunks = text ? (hi - G.n_vis) / 64 + 1 : 0;
  for (int e = 0; e < n_list + n_text_chunks; ++e) {
    int j, k0, k1;
    if (e < n_list) {
      j = (text || a.dense) ? e : (int)list[e];
      k0 = a.cube_offsets[j];
      k1 = a.cube_offsets[j + 1];
    } else {
      j = -1;
      k0 = G.n_vis + (e - n_list) * 64;
      k1 = min(k0 + 64, hi + 1);
    }
    bool row_on;
    if (text) row_on = valid;
    else if (a.dense) row_on = valid && j <= own;
    else row_on = valid && ((tm[(size_t)j * 4 + warp] >> lane) & 1u);
    for (int kb = k0; kb < k1; kb += 64) {
      const int nk = min(64, k1 - kb);
      __syncthreads();
      for (int x = tid; x < nk * D; x += 128) {
        const int u = x / D, dim = x - u * D;
        const size_t src = ((size_t)(kb + u) * G.hkv + kv) * D + dim;
        ks[x] = to_f32(Kp[src]);
        vs[x] = to_f32(Vp[src]);
      }
      __syncthreads();
      if (!row_on) continue;
      for (int u = 0; u < nk; ++u) {
        const int key = kb + u;
        if (text || j == own) {
          if (key > t) continue;
        }
        const float* kr = ks + u * D;
        float sc = 0.f;
#pragma unroll
        for (int x = 0; x < D; ++x) sc = fmaf(q[x], kr[x], sc);
        if (sc > m) {
          const float c = exp2f(m - sc);
          l *= c;
#pragma unroll
          for (int x = 0; x < D; ++x) o[x] *= c;
          m = sc;
        }
        const float pw = exp2f(sc - m);
        l += pw;
        const float* vr = vs + u * D;
#pragma unroll
        for (int x = 0; x < D; ++x) o[x] = fmaf(pw, vr[x], o[x]);
      }
    }
  }
  if (!valid) return;
  T* op = reinterpret_cast<T*>(a.out) + ((size_t)t * G.hq + h) * D;
  const float inv = 1.f / l;
#pragma unroll
  for (int x = 0; x < D; ++x) op[x] = from_f32<T>(o[x] * inv);
}

template <typename T, int D>
static cudaError_t launch_attn_simt_t(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = 2 * 64 * D * sizeof(float);
  auto k = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int blocks = a.G.n_vtiles + a.G.n_ttiles;
  if (blocks == 0) return cudaSuccess;
  return launch("attn_simt", k, dim3(blocks), dim3(128), smem, s, a);
}

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t s) {
  if (dtype == ADASPARK_FP32) {
    if (a.G.d == 64) return launch_attn_simt_t<float, 64>(a, s);
    return launch_attn_simt_t<float, 128>(a, s);
  }
  return launch_attn_simt_t<__nv_bfloat16, 128>(a, s);
}

}  // namespace adaspark

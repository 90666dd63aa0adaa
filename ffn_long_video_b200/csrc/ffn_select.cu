// AdaS-FFN token selection, compaction and mean compensation (key design 3 of
// the AdaSpark note: rank tokens of a cube by L2 norm, Top-p through the FFN,
// skipped tokens y_k = x_k + m_bar_i). HBM-bound SIMT kernels.
#include "ffn_kernels.h"

namespace adaspark {

template <typename T> struct Vec8;  // 16-byte vector of elements
template <> struct Vec8<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&f)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(b[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <> struct Vec8<float> {
  static constexpr int kN = 4;
  __device__ static void load(const float* p, float (&f)[8]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
};

// One block per cube: L2 norms of its tokens, then the Top-p cut over the
// importance w_u = ||x_u|| / sum ||x_v|| (or ||x_u||^2 / sum ||x_v||^2, or the
// softmax of the norms) by (norm desc, index asc), exactly as in AdaS-Attn. All
// three weights rank the tokens like their norms.
template <typename T>
__global__ void __launch_bounds__(256) ffn_select_kernel(FfnArgs a) {
  __shared__ unsigned long long keys[kMaxCubeTokens];
  __shared__ float s_norm[kMaxCubeTokens];
  __shared__ float s_w[kMaxCubeTokens];   // unnormalised importance
  __shared__ int s_k;
  if (status_bad(a.hdr)) return;
  const int j = blockIdx.x;
  const int base = a.cube_offsets[j];
  const int n = a.cube_offsets[j + 1] - base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* X = reinterpret_cast<const T*>(a.x);
  constexpr int V = Vec8<T>::kN;
  for (int u = warp; u < n; u += 8) {
    const T* row = X + (size_t)(base + u) * a.D;
    float acc = 0.f;
    for (int e = lane * V; e < a.D; e += 32 * V) {
      float f[8];
      Vec8<T>::load(row + e, f);
#pragma unroll
      for (int i = 0; i < V; ++i) acc = fmaf(f[i], f[i], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      const float nu = sqrtf(acc);
      s_norm[u] = nu;
      s_w[u] = a.importance == ADASPARK_IMPORTANCE_L2SQ_SHARE ? acc : nu;
      a.norms[base + u] = nu;
    }
  }
  __syncthreads();
  if (a.importance == ADASPARK_IMPORTANCE_SOFTMAX) {
    // exp(||x_u|| - max ||x||): the softmax numerators
    if (threadIdx.x < 32) {
      float m = -INFINITY;
      for (int u = threadIdx.x; u < n; u += 32) m = fmaxf(m, s_norm[u]);
      m = warp_max(m);
      for (int u = threadIdx.x; u < n; u += 32) s_w[u] = expf(s_norm[u] - m);
    }
    __syncthreads();
  }
  const int tid = threadIdx.x;
  if (a.dense) {
    for (int u = tid; u < n; u += 256) a.active[base + u] = 1;
    if (tid == 0) a.cube_count[j] = n;
    return;
  }
  // (norm desc, index asc) via a descending bitonic sort of 64-bit keys.
  keys[tid] = tid < n ? ((unsigned long long)__float_as_uint(s_norm[tid]) << 32) |
                            (unsigned long long)(0xFFFFFFFFu - (unsigned)tid)
                      : 0ull;
  __syncthreads();
  for (int size = 2; size <= kMaxCubeTokens; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int partner = tid ^ stride;
      if (partner > tid) {
        const bool desc = (tid & size) == 0;
        const unsigned long long x0 = keys[tid], x1 = keys[partner];
        if (desc ? (x0 < x1) : (x0 > x1)) {
          keys[tid] = x1;
          keys[partner] = x0;
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    float total = 0.f;
    for (int u = 0; u < n; ++u) total += s_w[u];
    int k = n;
    bool near = false;
    if (total > 0.f) {
      const float target = a.p * total;
      float cum = 0.f;
      for (int i = 0; i < n; ++i) {
        const float wi = s_w[(int)(0xFFFFFFFFu - (unsigned)(keys[i] & 0xFFFFFFFFull))];
        cum += wi;
        if (cum >= target) {
          k = i + 1;
          // within 1e-5 of flipping: C_k - p, p - C_(k-1) (k > 1), w_(k) - w_(k+1)
          float m = cum - target;
          if (i > 0) m = fminf(m, wi - (cum - target));
          if (i + 1 < n)
            m = fminf(m, wi - s_w[(int)(0xFFFFFFFFu - (unsigned)(keys[i + 1] & 0xFFFFFFFFull))]);
          near = m < 1e-5f * total;
          break;
        }
      }
      if (k == n && cum < target) near = true;  // rounding left the target unmet
    }
    s_k = k;
    a.cube_count[j] = k;
    if (near) atomicAdd((unsigned long long*)&a.hdr->stats[3], 1ull);
  }
  __syncthreads();
  if (tid < n) {
    const int rank_pos = tid;  // position in the sorted order
    const int u = (int)(0xFFFFFFFFu - (unsigned)(keys[rank_pos] & 0xFFFFFFFFull));
    const bool total_zero = s_k == n;
    a.active[base + u] = (rank_pos < s_k || total_zero) ? 1 : 0;
  }
}

// Exclusive prefix over the per-cube active counts; one block of 1024 threads.
__global__ void __launch_bounds__(1024) ffn_scan_kernel(FfnArgs a) {
  __shared__ int s_part[1024];
  if (status_bad(a.hdr)) return;
  const int C = a.n_cubes;
  const int tid = threadIdx.x;
  const int per = (C + 1023) / 1024;
  const int c0 = tid * per;
  int local = 0;
  for (int c = c0; c < c0 + per && c < C; ++c) local += a.cube_count[c];
  s_part[tid] = local;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v = tid >= o ? s_part[tid - o] : 0;
    __syncthreads();
    s_part[tid] += v;
    __syncthreads();
  }
  int run = s_part[tid] - local;
  for (int c = c0; c < c0 + per && c < C; ++c) {
    a.cube_start[c] = run;
    run += a.cube_count[c];
  }
  if (tid == 1023) {
    const int mv = s_part[1023];
    a.cube_start[C] = mv;
    a.hdr->m_active = (uint32_t)(mv + (a.n_tokens - a.n_vis));
    a.hdr->stats[0] = (unsigned long long)mv;
    a.hdr->stats[1] = (unsigned long long)(a.n_vis - mv);
    a.hdr->stats[2] = (unsigned long long)(a.n_tokens - a.n_vis);
  }
}

// Active rows in ascending order: visual actives cube by cube, then the text rows.
// Writes idx / row_cube and gathers x into xa. Blocks [0, C) handle cubes; the
// remaining blocks handle 64 text rows each.
template <typename T>
__global__ void __launch_bounds__(256) ffn_compact_kernel(FfnArgs a) {
  __shared__ int s_pos[kMaxCubeTokens];
  __shared__ int s_rows[kMaxCubeTokens];
  __shared__ int s_cnt;
  if (status_bad(a.hdr)) return;
  const int tid = threadIdx.x;
  const T* X = reinterpret_cast<const T*>(a.x);
  T* XA = reinterpret_cast<T*>(a.xa);
  int nrows, out0;
  if ((int)blockIdx.x < a.n_cubes) {
    const int j = blockIdx.x;
    const int base = a.cube_offsets[j];
    const int n = a.cube_offsets[j + 1] - base;
    if (tid == 0) {
      // skipped rows go to their own list: before cube j lie base tokens, of
      // which cube_start[j] are active
      int32_t* skip = a.skip + (base - a.cube_start[j]);
      int c = 0, k = 0;
      for (int u = 0; u < n; ++u) {
        if (a.active[base + u]) s_rows[c++] = base + u;
        else skip[k++] = base + u;
      }
      s_cnt = c;
    }
    __syncthreads();
    nrows = s_cnt;
    out0 = a.cube_start[j];
    for (int i = tid; i < nrows; i += 256) {
      a.idx[out0 + i] = s_rows[i];
      a.row_cube[out0 + i] = j;
    }
  } else {
    const int tb = blockIdx.x - a.n_cubes;
    const int t0 = a.n_vis + tb * 64;
    nrows = min(64, a.n_tokens - t0);
    out0 = a.cube_start[a.n_cubes] + tb * 64;
    for (int i = tid; i < nrows; i += 256) {
      s_rows[i] = t0 + i;
      a.idx[out0 + i] = t0 + i;
      a.row_cube[out0 + i] = -1;
      a.active[t0 + i] = 1;
    }
    __syncthreads();
  }
  (void)s_pos;
  // gather rows, 16-byte vectors
  constexpr int V = 16 / sizeof(T);
  const int vec_per_row = a.D / V;
  for (int e = tid; e < nrows * vec_per_row; e += 256) {
    const int i = e / vec_per_row, c = e - i * vec_per_row;
    const uint4 v = *reinterpret_cast<const uint4*>(X + (size_t)s_rows[i] * a.D + c * V);
    *reinterpret_cast<uint4*>(XA + (size_t)(out0 + i) * a.D + c * V) = v;
  }
}

// Skipped visual rows: y_k = x_k + sums_c / |M_c| (mean of FFN over the cube's
// active tokens). One warp per skipped row, taken from the compaction's list
// of skipped rows (so the warps of the first blocks all have a row, and the
// blocks past the list's end exit at once).
template <typename T>
__global__ void __launch_bounds__(256) ffn_compensate_kernel(FfnArgs a) {
  if (status_bad(a.hdr)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + warp;
  if (i >= a.n_vis - a.cube_start[a.n_cubes]) return;
  const int t = a.skip[i];
  const int c = a.cube_ids[t];
  const float inv = 1.f / (float)a.cube_count[c];
  const T* xr = reinterpret_cast<const T*>(a.x) + (size_t)t * a.D;
  const float* sr = a.sums + (size_t)c * a.D;
  float* yr = a.y + (size_t)t * a.D;
  // one 16-byte load of x per lane and step (8 bf16 or 4 fp32 features), the
  // matching sums and stores; four steps in flight
  constexpr int kN = Vec8<T>::kN;
#pragma unroll 4
  for (int e = lane * kN; e < a.D; e += 32 * kN) {
    float xv[8];
    Vec8<T>::load(xr + e, xv);
#pragma unroll
    for (int h = 0; h < kN; h += 4) {
      const float4 sv = *reinterpret_cast<const float4*>(sr + e + h);
      float4 o;
      o.x = xv[h] + sv.x * inv;
      o.y = xv[h + 1] + sv.y * inv;
      o.z = xv[h + 2] + sv.z * inv;
      o.w = xv[h + 3] + sv.w * inv;
      *reinterpret_cast<float4*>(yr + e + h) = o;
    }
  }
}

cudaError_t launch_ffn_select(const FfnArgs& a, int dtype, cudaStream_t s) {
  cudaError_t e;
  if (a.n_cubes > 0) {
    if (dtype == ADASPARK_BF16)
      e = launch("ffn_select", ffn_select_kernel<__nv_bfloat16>, dim3(a.n_cubes), dim3(256), 0, s,
                 a);
    else
      e = launch("ffn_select", ffn_select_kernel<float>, dim3(a.n_cubes), dim3(256), 0, s, a);
    if (e != cudaSuccess) return e;
  }
  return launch("ffn_scan", ffn_scan_kernel, dim3(1), dim3(1024), 0, s, a);
}

cudaError_t launch_ffn_compact(const FfnArgs& a, int dtype, cudaStream_t s) {
  const int text_blocks = (a.n_tokens - a.n_vis + 63) / 64;
  const int blocks = a.n_cubes + text_blocks;
  if (blocks == 0) return cudaSuccess;
  if (dtype == ADASPARK_BF16)
    return launch("ffn_compact", ffn_compact_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, s,
                  a);
  return launch("ffn_compact", ffn_compact_kernel<float>, dim3(blocks), dim3(256), 0, s, a);
}

cudaError_t launch_ffn_compensate(const FfnArgs& a, int dtype, cudaStream_t s) {
  if (a.n_vis == 0 || a.dense) return cudaSuccess;
  const int blocks = (a.n_vis + 7) / 8;
  if (dtype == ADASPARK_BF16)
    return launch("ffn_compensate", ffn_compensate_kernel<__nv_bfloat16>, dim3(blocks), dim3(256),
                  0, s, a);
  return launch("ffn_compensate", ffn_compensate_kernel<float>, dim3(blocks), dim3(256), 0, s, a);
}

}  // namespace adaspark

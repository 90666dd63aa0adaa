// SwiGLU FFN over the compacted active rows, SIMT form (fp32 path):
//   gemm1: H = silu(X_a W_gate^T) * (X_a W_up^T)
//   gemm2: FFN_a = H W_down^T, scattered as y[idx] = x[idx] + FFN_a, with the
//          per-cube fp32 sums of FFN_a over active visual rows (for the mean
//          compensation of key design 3).
// 64x64 output tiles, 4x4 per thread, 16-deep K slices in shared memory.
#include "ffn_kernels.h"

namespace adaspark {

template <typename T>
__global__ void __launch_bounds__(256) gemm1_simt_kernel(FfnArgs a) {
  __shared__ float As[16][68], Gs[16][68], Us[16][68];
  if (status_bad(a.hdr)) return;
  const int M = (int)a.hdr->m_active;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  if (m0 >= M) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T* XA = reinterpret_cast<const T*>(a.xa);
  const T* WG = reinterpret_cast<const T*>(a.W_gate);
  const T* WU = reinterpret_cast<const T*>(a.W_up);
  float g[4][4] = {}, u[4][4] = {};
  for (int k0 = 0; k0 < a.D; k0 += 16) {
    for (int i = tid; i < 1024; i += 256) {
      const int r = i >> 4, c = i & 15, k = k0 + c;
      const bool kin = k < a.D;
      As[c][r] = (m0 + r < M && kin) ? to_f32(XA[(size_t)(m0 + r) * a.D + k]) : 0.f;
      Gs[c][r] = (n0 + r < a.F && kin) ? to_f32(WG[(size_t)(n0 + r) * a.D + k]) : 0.f;
      Us[c][r] = (n0 + r < a.F && kin) ? to_f32(WU[(size_t)(n0 + r) * a.D + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], gv[4], uv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        gv[i] = Gs[kk][tx * 4 + i];
        uv[i] = Us[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          g[i][j] = fmaf(av[i], gv[j], g[i][j]);
          u[i][j] = fmaf(av[i], uv[j], u[i][j]);
        }
    }
    __syncthreads();
  }
  T* H = reinterpret_cast<T*>(a.h);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= a.F) continue;
      const float gg = g[i][j];
      const float hv = gg / (1.f + expf(-gg)) * u[i][j];
      H[(size_t)m * a.F + n] = from_f32<T>(hv);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gemm2_simt_kernel(FfnArgs a) {
  __shared__ float As[16][68], Bs[16][68];
  if (status_bad(a.hdr)) return;
  const int M = (int)a.hdr->m_active;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  if (m0 >= M) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const T* H = reinterpret_cast<const T*>(a.h);
  const T* WD = reinterpret_cast<const T*>(a.W_down);
  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.F; k0 += 16) {
    for (int i = tid; i < 1024; i += 256) {
      const int r = i >> 4, c = i & 15, k = k0 + c;
      const bool kin = k < a.F;
      As[c][r] = (m0 + r < M && kin) ? to_f32(H[(size_t)(m0 + r) * a.F + k]) : 0.f;
      Bs[c][r] = (n0 + r < a.D && kin) ? to_f32(WD[(size_t)(n0 + r) * a.F + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const T* X = reinterpret_cast<const T*>(a.x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
    const int orig = a.idx[m];
    const int c = a.row_cube[m];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= a.D) continue;
      const float f = acc[i][j];
      a.y[(size_t)orig * a.D + n] = to_f32(X[(size_t)orig * a.D + n]) + f;
      if (c >= 0 && !a.dense) atomicAdd(&a.sums[(size_t)c * a.D + n], f);
    }
  }
}

cudaError_t launch_ffn_gemm1_simt(const FfnArgs& a, int dtype, cudaStream_t s) {
  const dim3 grid((a.n_tokens + 63) / 64, (a.F + 63) / 64);
  if (dtype == ADASPARK_BF16)
    return launch("ffn_gemm1_simt", gemm1_simt_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, a);
  return launch("ffn_gemm1_simt", gemm1_simt_kernel<float>, grid, dim3(256), 0, s, a);
}

cudaError_t launch_ffn_gemm2_simt(const FfnArgs& a, int dtype, cudaStream_t s) {
  const dim3 grid((a.n_tokens + 63) / 64, (a.D + 63) / 64);
  if (dtype == ADASPARK_BF16)
    return launch("ffn_gemm2_simt", gemm2_simt_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, a);
  return launch("ffn_gemm2_simt", gemm2_simt_kernel<float>, grid, dim3(256), 0, s, a);
}

}  // namespace adaspark

// A whole AdaSpark layer as the stacked configuration wires it, and RMSNorm:
//   Q = x W_q^T, K = x W_k^T, V = x W_v^T        (tcgen05 GEMMs, bf16 out)
//   a = AdaS-Attn(Q, K, V; p_attn)               (adaspark_cube_attn)
//   h = x + a W_o^T                              (tcgen05 GEMM, residual epilogue)
//   y = AdaS-FFN(h; p_ffn)                       (adaspark_token_ffn, fp32 out)
// The projections run on the same persistent GEMM kernel as the FFN, with an
// identity row map. RMSNorm (x / sqrt(mean(x^2) + eps), times an optional
// weight) is a separate call, for the normalization between layers.
#include <cmath>

#include "attn_kernels.h"
#include "ffn_kernels.h"

using namespace adaspark;

namespace {

constexpr size_t kLayerAlign = 256;

size_t align_up(size_t v) { return (v + kLayerAlign - 1) / kLayerAlign * kLayerAlign; }

struct LayerLayout {
  size_t header, attn_ws, ffn_ws, q, k, v, a, h, total;
  size_t attn_bytes, ffn_bytes;
};

bool layer_layout(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d, int D, int F,
                  LayerLayout* L) {
  L->attn_bytes = adaspark_cube_attn_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d,
                                               ADASPARK_BF16);
  L->ffn_bytes = adaspark_token_ffn_workspace(n_tokens, n_vis, n_cubes, D, F, ADASPARK_BF16);
  if (L->attn_bytes == 0 || L->ffn_bytes == 0) return false;
  const size_t N = (size_t)n_tokens;
  size_t o = 0;
  L->header = o;
  o = align_up(o + sizeof(WsHeader));
  L->attn_ws = o;
  o = align_up(o + L->attn_bytes);
  L->ffn_ws = o;
  o = align_up(o + L->ffn_bytes);
  L->q = o;
  o = align_up(o + N * hq * d * 2);
  L->k = o;
  o = align_up(o + N * hkv * d * 2);
  L->v = o;
  o = align_up(o + N * hkv * d * 2);
  L->a = o;
  o = align_up(o + N * hq * d * 2);
  L->h = o;
  o = align_up(o + N * D * 2);
  L->total = o;
  return true;
}

bool layer_sizes_ok(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d, int D, int F) {
  if ((d != 64 && d != 128) || hq < 1 || hkv < 1) return false;
  // GEMM shapes: K multiple of 64, output columns multiple of 32
  if (D % 64 != 0 || (hq * d) % 64 != 0) return false;
  LayerLayout L{};
  return layer_layout(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, &L);
}

// y[t] = x[t] / sqrt(mean_d x[t]^2 + eps) * (w ? w : 1); one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const T* __restrict__ x,
                                                      const __nv_bfloat16* __restrict__ w,
                                                      __nv_bfloat16* __restrict__ y, int n, int D,
                                                      float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= n) return;
  const T* xr = x + (size_t)t * D;
  float ss = 0.f;
  for (int e = lane; e < D; e += 32) {
    const float v = to_f32(xr[e]);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)D + eps);
  __nv_bfloat16* yr = y + (size_t)t * D;
  for (int e = lane; e < D; e += 32) {
    const float g = w ? __bfloat162float(w[e]) : 1.f;
    yr[e] = __float2bfloat16_rn(to_f32(xr[e]) * r * g);
  }
}

// Fold the status words of the attention and FFN workspaces into the layer's.
__global__ void merge_status_kernel(WsHeader* dst, const WsHeader* a, const WsHeader* b) {
  const uint32_t st = a->status | b->status;
  if (st) {
    atomicOr(&dst->status, st);
    const uint32_t det = a->status ? a->detail : b->detail;
    atomicCAS(&dst->detail, 0u, det);
  }
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? ADASPARK_OK : ADASPARK_ECUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" {

size_t adaspark_layer_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d,
                                int D, int F, int dtype) {
  if (dtype != ADASPARK_BF16 || !layer_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F))
    return 0;
  LayerLayout L{};
  return layer_layout(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, &L) ? L.total : 0;
}

int adaspark_layer_buffers(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d, int D,
                           int F, int dtype, size_t* offsets) {
  if (!offsets || dtype != ADASPARK_BF16 ||
      !layer_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F))
    return ADASPARK_EINVAL;
  LayerLayout L{};
  if (!layer_layout(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, &L)) return ADASPARK_EINVAL;
  offsets[0] = L.q;
  offsets[1] = L.k;
  offsets[2] = L.v;
  offsets[3] = L.a;
  offsets[4] = L.h;
  offsets[5] = L.attn_ws;
  offsets[6] = L.ffn_ws;
  return ADASPARK_OK;
}

int adaspark_layer(const void* x, const void* W_q, const void* W_k, const void* W_v,
                   const void* W_o, const void* W_gate, const void* W_up, const void* W_down,
                   int dtype, const int32_t* cube_ids, const int32_t* cube_offsets,
                   const uint8_t* text_mask, int n_cubes, int n_vis, int n_tokens, int hq,
                   int hkv, int d, int D, int F, float p_attn, float p_ffn, float* y,
                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_gate || !W_up || !W_down || !cube_ids ||
      !cube_offsets || !text_mask || !y || !workspace)
    return ADASPARK_EINVAL;
  if (dtype == ADASPARK_FP32) return ADASPARK_EUNSUPPORTED;
  if (dtype != ADASPARK_BF16 || !layer_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F))
    return ADASPARK_EINVAL;
  if (!(p_attn > 0.f && p_attn <= 1.f) || !(p_ffn > 0.f && p_ffn <= 1.f)) return ADASPARK_EINVAL;
  LayerLayout L{};
  if (!layer_layout(n_tokens, n_vis, n_cubes, hq, hkv, d, D, F, &L)) return ADASPARK_EINVAL;
  if (workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & (kLayerAlign - 1)))
    return ADASPARK_EINVAL;
  for (const void* ptr : {x, W_q, W_k, W_v, W_o, W_gate, W_up, W_down,
                          static_cast<const void*>(y)})
    if (!aligned16(ptr)) return ADASPARK_EINVAL;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  auto* Q = reinterpret_cast<__nv_bfloat16*>(ws + L.q);
  auto* K = reinterpret_cast<__nv_bfloat16*>(ws + L.k);
  auto* V = reinterpret_cast<__nv_bfloat16*>(ws + L.v);
  auto* A = reinterpret_cast<__nv_bfloat16*>(ws + L.a);
  auto* H = reinterpret_cast<__nv_bfloat16*>(ws + L.h);
  const auto* X = static_cast<const __nv_bfloat16*>(x);
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return ADASPARK_ECUDA;
  int rc;
  if ((rc = cuda_rc(launch_linear_tc(X, static_cast<const __nv_bfloat16*>(W_q), nullptr, Q,
                                     n_tokens, hq * d, D, hdr, s))) ||
      (rc = cuda_rc(launch_linear_tc(X, static_cast<const __nv_bfloat16*>(W_k), nullptr, K,
                                     n_tokens, hkv * d, D, hdr, s))) ||
      (rc = cuda_rc(launch_linear_tc(X, static_cast<const __nv_bfloat16*>(W_v), nullptr, V,
                                     n_tokens, hkv * d, D, hdr, s))))
    return rc;
  if ((rc = adaspark_cube_attn(Q, K, V, ADASPARK_BF16, cube_ids, cube_offsets, n_cubes, n_vis,
                               n_tokens, hq, hkv, d, p_attn, A, ws + L.attn_ws, L.attn_bytes,
                               stream)))
    return rc;
  if ((rc = cuda_rc(launch_linear_tc(A, static_cast<const __nv_bfloat16*>(W_o), X, H, n_tokens,
                                     D, hq * d, hdr, s))))
    return rc;
  if ((rc = adaspark_token_ffn(H, W_gate, W_up, W_down, ADASPARK_BF16, cube_ids, cube_offsets,
                               text_mask, n_cubes, n_vis, n_tokens, D, F, p_ffn, y,
                               ws + L.ffn_ws, L.ffn_bytes, stream)))
    return rc;
  return cuda_rc(launch("merge_status", merge_status_kernel, dim3(1), dim3(1), 0, s, hdr,
                        reinterpret_cast<const WsHeader*>(ws + L.attn_ws),
                        reinterpret_cast<const WsHeader*>(ws + L.ffn_ws)));
}

int adaspark_rmsnorm(const void* x, int x_dtype, const void* weight, void* out, int n_rows,
                     int D, float eps, void* stream) {
  if (!x || !out || n_rows < 0 || D < 1 || !(eps >= 0.f)) return ADASPARK_EINVAL;
  if (x_dtype != ADASPARK_BF16 && x_dtype != ADASPARK_FP32) return ADASPARK_EINVAL;
  if (n_rows == 0) return ADASPARK_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid((n_rows + 7) / 8), block(256);
  const auto* w = static_cast<const __nv_bfloat16*>(weight);
  auto* y = static_cast<__nv_bfloat16*>(out);
  if (x_dtype == ADASPARK_BF16)
    return cuda_rc(launch("rmsnorm", rmsnorm_kernel<__nv_bfloat16>, grid, block, 0, s,
                          static_cast<const __nv_bfloat16*>(x), w, y, n_rows, D, eps));
  return cuda_rc(launch("rmsnorm", rmsnorm_kernel<float>, grid, block, 0, s,
                        static_cast<const float*>(x), w, y, n_rows, D, eps));
}

}  // extern "C"

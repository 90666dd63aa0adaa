// AdaS-Attn, selection side (key design 2 of the AdaSpark note):
//  - layout validation of cube_ids / cube_offsets,
//  - cube mean keys kbar_j (fp32, plus a three-part bf16 split for the tensor-core
//    scorer),
//  - the SIMT scorer + Top-p selection (fp32 path), emitting per-tile cube lists
//    and 128-bit row masks,
//  - export of the selected sets as a dense bitmap.
#include "attn_kernels.h"
#include "select.cuh"

namespace adaspark {

// ---------------------------------------------------------------------------
// Layout validation (visual prefix in cubes, text suffix = -1).
// ---------------------------------------------------------------------------
__global__ void validate_layout_kernel(const int32_t* __restrict__ cube_ids,
                                       const int32_t* __restrict__ off,
                                       const uint8_t* __restrict__ text_mask, int n_cubes,
                                       int n_vis, int n_tokens, WsHeader* hdr) {
  const int stride = gridDim.x * blockDim.x;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c <= n_cubes; c += stride) {
    const int a = off[c];
    if (c == 0 && a != 0) set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x101u);
    if (c == n_cubes && a != n_vis) set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x102u);
    if (c < n_cubes) {
      const int n = off[c + 1] - a;
      if (n < 1 || n > kMaxCubeTokens) set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x103u);
    }
  }
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n_tokens; t += stride) {
    const int c = cube_ids[t];
    if (t < n_vis) {
      if (c < 0 || c >= n_cubes || t < off[c] || t >= off[c + 1])
        set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x104u);
    } else if (c != -1) {
      set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x105u);
    }
    if (text_mask && (text_mask[t] != 0) != (c == -1))
      set_status(hdr, ADASPARK_DEV_BAD_LAYOUT, 0x106u);
  }
}

// ---------------------------------------------------------------------------
// kbar[kv][j][:] = mean of K over cube j (fp64 accumulation, fp32 result) and
// its split kbar = hi + mid + lo into bf16 parts (products with bf16 queries are
// exact, so three tensor-core passes reproduce the fp32 dot product).
// One block per cube: thread (x, y) sums one 16-byte vector of a token's row
// (8 bf16 or 4 fp32 elements of one KV head) over the cube's tokens y, y + S,
// y + 2S, ... (S = blockDim.y token slices; eight loads in flight per thread),
// and the S partial sums meet in shared memory.
constexpr int kMeanThreads = 256;
template <typename T>
__global__ void __launch_bounds__(kMeanThreads)
    cube_mean_kernel(const T* __restrict__ K, const int32_t* __restrict__ off,
                     float* __restrict__ kbar, __nv_bfloat16* __restrict__ split, int n_cubes,
                     int hkv, int d, WsHeader* hdr) {
  constexpr int V = 16 / sizeof(T);
  __shared__ double part[kMeanThreads * V];
  if (status_bad(hdr)) return;
  const int j = blockIdx.x;
  const int row = hkv * d;               // blockDim.x * V == row (the launcher's shape)
  const int x = threadIdx.x, y = threadIdx.y, S = blockDim.y;
  const int e = x * V;                   // first (kv * d + dim) element of this thread
  const int a = off[j], b = off[j + 1];
  // bf16 sums of a cube are exact in fp64 for any realistic spread of
  // magnitudes; the order is fixed, so the result is deterministic in any case
  constexpr int U = 8;
  double acc0[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc0[i] = 0.0;
  for (int t = a + y; t < b; t += U * S) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = t + u * S;
      raw[u] = tt < b ? __ldg(reinterpret_cast<const uint4*>(K + (size_t)tt * row + e))
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const T* v = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
      for (int i = 0; i < V; ++i) acc0[i] += (double)to_f32(v[i]);
    }
  }
  if (S > 1) {
#pragma unroll
    for (int i = 0; i < V; ++i) part[(y * blockDim.x + x) * V + i] = acc0[i];
    __syncthreads();
    if (y != 0) return;
    for (int z = 1; z < S; ++z)
#pragma unroll
      for (int i = 0; i < V; ++i) acc0[i] += part[(z * blockDim.x + x) * V + i];
  }
  const int kv = e / d, dim = e - kv * d;
  const size_t o = ((size_t)kv * n_cubes + j) * d + dim;
  const size_t plane = (size_t)hkv * n_cubes * d;
  float mean[V];
  __nv_bfloat16 hi[V], mid[V], lo[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    mean[i] = (float)(acc0[i] / (double)(b - a));
    hi[i] = __float2bfloat16_rn(mean[i]);
    const float r1 = mean[i] - __bfloat162float(hi[i]);
    mid[i] = __float2bfloat16_rn(r1);
    lo[i] = __float2bfloat16_rn(r1 - __bfloat162float(mid[i]));
  }
#pragma unroll
  for (int i = 0; i < V; ++i) {
    kbar[o + i] = mean[i];
    split[o + i] = hi[i];
    split[plane + o + i] = mid[i];
    split[2 * plane + o + i] = lo[i];
  }
}

// ---------------------------------------------------------------------------
// SIMT scorer + selection: one block per visual tile, one thread per row.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) select_simt_kernel(SelectArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  sel::Smem* ss = reinterpret_cast<sel::Smem*>(smem_raw);
  float* kch = reinterpret_cast<float*>(smem_raw + sizeof(sel::Smem));  // [64][D]
  __shared__ int s_lo, s_hi, s_wcnt[4];
  if (status_bad(a.hdr)) return;
  const AttnGeom& G = a.G;
  const int vt = blockIdx.x;
  const int kv = vt / G.vtiles_per_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TileRow R = tile_row(G, false, vt, tid);
  const bool valid = R.valid;
  const int t = R.t, h = R.h;
  const int own = valid ? a.cube_ids[t] : -1;

  if (tid == 0) {
    s_lo = INT_MAX;
    s_hi = -1;
  }
  __syncthreads();
  if (valid) {
    atomicMin(&s_lo, own);
    atomicMax(&s_hi, own);
  }
  __syncthreads();
  const int c_hi = s_hi;
  if (c_hi < 0) return;

  float q[D];
  const T* qp = reinterpret_cast<const T*>(a.Q) + ((size_t)t * G.hq + h) * D;
#pragma unroll
  for (int e = 0; e < D; ++e) q[e] = valid ? to_f32(qp[e]) : 0.f;

  sel::RowSel s;
  s.init(ss, tid, a.zscale, a.topk > 0);
  const int ncand = own > 0 ? own : 0;
  const float* kb = a.kbar + (size_t)kv * G.n_cubes * D;
  uint32_t* tmask = a.tile_mask + (size_t)vt * G.n_cubes * 4;
  __shared__ int s_more;
  int nsel = 0, extra = 0;

  // pass 0: histogram; pass 1: emission; pass >= 2: rows whose cut is still open
  for (int pass = 0;; ++pass) {
    for (int j0 = 0; j0 < c_hi; j0 += 64) {
      const int nj = min(64, c_hi - j0);
      __syncthreads();
      for (int e = tid; e < nj * D; e += 128) kch[e] = kb[(size_t)j0 * D + e];
      __syncthreads();
      for (int jj = 0; jj < nj; ++jj) {
        const int j = j0 + jj;
        bool selb = false;
        if (j < ncand && (pass < 2 || s.open)) {
          const float* kr = kch + jj * D;
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < D; ++e) acc = fmaf(q[e], kr[e], acc);
          if (pass == 0) s.pass1(acc);
          else if (pass == 1) selb = s.pass2(acc, j, true);
          else selb = s.pass_more(acc, j);
        }
        if (pass == 1) {
          const unsigned w = __ballot_sync(0xffffffffu, selb || own == j);
          if (lane == 0) tmask[(size_t)j * 4 + warp] = w;
          nsel += selb;
        } else if (pass >= 2) {
          // fine bins above a row's fine cut, selected outright
          const unsigned w = __ballot_sync(0xffffffffu, selb);
          if (w != 0u && lane == 0) atomicOr(&tmask[(size_t)j * 4 + warp], w);
          nsel += selb;
        }
      }
    }
    if (pass == 0) {
      s.finish1(a.topk > 0 ? (float)a.topk : a.p);
      if (s.range_err) set_status(a.hdr, ADASPARK_DEV_RANGE, 0x8900u);
      continue;
    }
    if (pass == 1) {
      const unsigned w = __ballot_sync(0xffffffffu, own == c_hi);
      if (lane == 0) tmask[(size_t)c_hi * 4 + warp] = w;
      __syncwarp();
    }
    const bool was_open = s.open;
    const int m = s.settle();
    for (int i = 0; i < m; ++i) atomicOr(&tmask[(size_t)s.list_j(i) * 4 + warp], 1u << lane);
    nsel += m;
    s.reset_list();
    if (pass >= 1 && was_open && s.open) extra = 1;
    if (tid == 0) s_more = 0;
    __syncthreads();
    if (s.open) s_more = 1;
    __syncthreads();
    if (!s_more) break;
  }
  // statistics
  const unsigned v_rows = __reduce_add_sync(0xffffffffu, (valid && own > 0) ? 1u : 0u);
  const unsigned v_cand = __reduce_add_sync(0xffffffffu, (unsigned)ncand);
  const unsigned v_sel = __reduce_add_sync(0xffffffffu, (unsigned)nsel);
  const unsigned v_ext = __reduce_add_sync(0xffffffffu, (unsigned)extra);
  const unsigned v_near = __reduce_add_sync(0xffffffffu, (valid && s.near) ? 1u : 0u);
  if (lane == 0) {
    atomicAdd((unsigned long long*)&a.hdr->stats[0], (unsigned long long)v_rows);
    atomicAdd((unsigned long long*)&a.hdr->stats[1], (unsigned long long)v_cand);
    atomicAdd((unsigned long long*)&a.hdr->stats[2], (unsigned long long)v_sel);
    atomicAdd((unsigned long long*)&a.hdr->stats[3], (unsigned long long)v_ext);
    if (v_near) atomicAdd((unsigned long long*)&a.hdr->stats[7], (unsigned long long)v_near);
  }
  __threadfence_block();
  __syncthreads();
  compact_tile_list(tmask, a.tile_list + (size_t)vt * G.n_cubes, a.tile_count + vt, c_hi, s_wcnt,
                    tid);
}

// ---------------------------------------------------------------------------
// Export: tile lists + masks -> dense bitmap [n_vis][hq][W] (own cube not marked).
// ---------------------------------------------------------------------------
__global__ void export_sets_kernel(const int32_t* __restrict__ tile_count,
                                   const uint16_t* __restrict__ tile_list,
                                   const uint32_t* __restrict__ tile_mask,
                                   const int32_t* __restrict__ cube_ids, AttnGeom G, int dense,
                                   uint32_t* __restrict__ bits) {
  const int vt = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TileRow R = tile_row(G, false, vt, tid);
  if (!R.valid) return;
  const int t = R.t, h = R.h;
  const int own = cube_ids[t];
  const int W = (G.n_cubes + 31) / 32;
  uint32_t* row = bits + ((size_t)t * G.hq + h) * W;
  for (int w = 0; w < W; ++w) row[w] = 0u;
  if (dense) {
    for (int j = 0; j < own; ++j) row[j >> 5] |= 1u << (j & 31);
    return;
  }
  const int n = tile_count[vt];
  const uint16_t* list = tile_list + (size_t)vt * G.n_cubes;
  const uint32_t* tm = tile_mask + (size_t)vt * G.n_cubes * 4;
  for (int k = 0; k < n; ++k) {
    const int j = list[k];
    if (j >= own) break;
    if ((tm[(size_t)j * 4 + warp] >> lane) & 1u) row[j >> 5] |= 1u << (j & 31);
  }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
cudaError_t launch_validate(const int32_t* cube_ids, const int32_t* off, const uint8_t* text_mask,
                            int n_cubes, int n_vis, int n_tokens, WsHeader* hdr,
                            cudaStream_t s) {
  int n = n_tokens > n_cubes + 1 ? n_tokens : n_cubes + 1;
  int blocks = (n + 255) / 256;
  if (blocks > 1184) blocks = 1184;
  return launch("validate_layout", validate_layout_kernel, dim3(blocks), dim3(256), 0, s, cube_ids,
                off, text_mask, n_cubes, n_vis, n_tokens, hdr);
}

cudaError_t launch_cube_mean(const void* K, int dtype, const int32_t* off, float* kbar,
                             __nv_bfloat16* split, const AttnGeom& G, WsHeader* hdr,
                             cudaStream_t s) {
  // hkv * d <= 1024 (attn_sizes_ok): at most 128 (bf16) or 256 (fp32) vector
  // threads per token row, and up to 8 token slices within 256 threads
  const int rx = G.hkv * G.d / (dtype == ADASPARK_BF16 ? 8 : 4);
  const int sy = std::max(1, std::min(8, kMeanThreads / rx));
  if (dtype == ADASPARK_BF16)
    return launch("cube_mean_keys", cube_mean_kernel<__nv_bfloat16>, dim3(G.n_cubes),
                  dim3(rx, sy), 0, s, (const __nv_bfloat16*)K, off, kbar, split, G.n_cubes,
                  G.hkv, G.d, hdr);
  return launch("cube_mean_keys", cube_mean_kernel<float>, dim3(G.n_cubes), dim3(rx, sy), 0, s,
                (const float*)K, off, kbar, split, G.n_cubes, G.hkv, G.d, hdr);
}

template <typename T, int D>
static cudaError_t launch_select_simt_t(const SelectArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(sel::Smem) + 64 * D * sizeof(float);
  auto k = select_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch("select_simt", k, dim3(a.G.n_vtiles), dim3(128), smem, s, a);
}

cudaError_t launch_select_simt(const SelectArgs& a, int dtype, cudaStream_t s) {
  if (dtype == ADASPARK_FP32) {
    if (a.G.d == 64) return launch_select_simt_t<float, 64>(a, s);
    return launch_select_simt_t<float, 128>(a, s);
  }
  return launch_select_simt_t<__nv_bfloat16, 128>(a, s);
}

// ---------------------------------------------------------------------------
// Uniform Sampling (the content-independent strategy of the AdaSpark paper's
// selection-strategy ablation, read as k of the i preceding cubes at even
// spacing from the first, floor(m i / k), or all of them when i <= k): the
// tile masks and lists of the attention written directly, without scores.
// One CTA of 128 threads (one per row) per visual tile.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool uniform_member(int i, int k, int j) {
  if (j >= i) return false;
  if (i <= k) return true;
  // the smallest m with m i / k >= j is ceil(j k / i); j is taken when it maps back to j
  const long long m = ((long long)j * k + i - 1) / i;
  return m < k && (m * i) / k == j;
}

__global__ void __launch_bounds__(128) select_uniform_kernel(SelectArgs a) {
  __shared__ int s_hi, s_wcnt[4];
  const AttnGeom& G = a.G;
  const int vt = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (status_bad(a.hdr)) return;
  const TileRow R = tile_row(G, false, vt, tid);
  const int own = R.valid ? a.cube_ids[R.t] : -1;
  if (tid == 0) s_hi = -1;
  __syncthreads();
  if (R.valid) atomicMax(&s_hi, own);
  __syncthreads();
  const int c_hi = s_hi;
  if (c_hi < 0) return;
  uint32_t* tmask = a.tile_mask + (size_t)vt * G.n_cubes * 4;
  for (int j = 0; j <= c_hi; ++j) {
    const bool in = R.valid && (j == own || uniform_member(own, a.topk, j));
    const unsigned w = __ballot_sync(0xffffffffu, in);
    if (lane == 0) tmask[(size_t)j * 4 + warp] = w;
  }
  const int cand = own > 0 ? own : 0;
  const unsigned v_rows = __reduce_add_sync(0xffffffffu, (R.valid && own > 0) ? 1u : 0u);
  const unsigned v_cand = __reduce_add_sync(0xffffffffu, (unsigned)cand);
  const unsigned v_sel = __reduce_add_sync(0xffffffffu, (unsigned)min(cand, a.topk));
  if (lane == 0) {
    atomicAdd((unsigned long long*)&a.hdr->stats[0], (unsigned long long)v_rows);
    atomicAdd((unsigned long long*)&a.hdr->stats[1], (unsigned long long)v_cand);
    atomicAdd((unsigned long long*)&a.hdr->stats[2], (unsigned long long)v_sel);
  }
  __threadfence_block();
  __syncthreads();
  compact_tile_list(tmask, a.tile_list + (size_t)vt * G.n_cubes, a.tile_count + vt, c_hi, s_wcnt,
                    tid);
}

cudaError_t launch_select_uniform(const SelectArgs& a, cudaStream_t s) {
  if (a.G.n_vtiles == 0) return cudaSuccess;
  return launch("select_uniform", select_uniform_kernel, dim3(a.G.n_vtiles), dim3(128), 0, s, a);
}

cudaError_t launch_export_sets(const int32_t* tile_count, const uint16_t* tile_list,
                               const uint32_t* tile_mask, const int32_t* cube_ids,
                               const AttnGeom& G, int dense, uint32_t* bits, cudaStream_t s) {
  if (G.n_vtiles == 0) return cudaSuccess;
  return launch("export_sets", export_sets_kernel, dim3(G.n_vtiles), dim3(128), 0, s, tile_count,
                tile_list, tile_mask, cube_ids, G, dense, bits);
}

}  // namespace adaspark

// extern "C" entry points of AdaS-Attn and AdaS-FFN: host-side validation,
// workspace carving, and the launch sequence on the caller's stream.
#include <cmath>

#include "attn_kernels.h"
#include "ffn_kernels.h"

namespace adaspark {
int cube_attn_single_walk(const void* Q, const void* K, const void* V, int dtype,
                          const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                          int n_vis, int n_tokens, int hq, int hkv, int d, float p, void* out,
                          void* workspace, size_t workspace_bytes, void* stream);
size_t cube_attn_single_walk_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv,
                                       int d, int dtype);
}  // namespace adaspark

using namespace adaspark;

namespace {

constexpr int kModeDense = 1;

int check_device() {
  static int cached = -2;
  if (cached == -2) cached = device_is_sm100();
  if (cached < 0) return ADASPARK_ECUDA;
  return cached ? ADASPARK_OK : ADASPARK_EUNSUPPORTED;
}

bool attn_sizes_ok(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d, int dtype) {
  if (n_tokens < 1 || n_vis < 0 || n_vis > n_tokens) return false;
  if (n_cubes < 0 || n_cubes > kMaxCubes) return false;
  if (n_vis > 0 && n_cubes < 1) return false;
  if (n_vis == 0 && n_cubes != 0) return false;
  if ((long long)n_cubes > n_vis) return false;
  if (hq < 1 || hkv < 1 || hq % hkv != 0 || hkv * d > 1024) return false;
  if (dtype == ADASPARK_BF16 || dtype == ADASPARK_FP32) return d == 64 || d == 128;
  return false;
}

bool ffn_sizes_ok(int n_tokens, int n_vis, int n_cubes, int D, int F, int dtype) {
  if (n_tokens < 1 || n_vis < 0 || n_vis > n_tokens) return false;
  if (n_cubes < 0 || n_cubes > kMaxCubes) return false;
  if (n_vis > 0 && n_cubes < 1) return false;
  if (n_vis == 0 && n_cubes != 0) return false;
  if ((long long)n_cubes > n_vis) return false;
  if (D < 1 || F < 1) return false;
  if (dtype == ADASPARK_BF16) return D % 64 == 0 && F % 128 == 0;
  if (dtype == ADASPARK_FP32) return D % 4 == 0 && F % 4 == 0;
  return false;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? ADASPARK_OK : ADASPARK_ECUDA; }

// Test hook of the bounded waits (adaspark_debug_wait_expiry): the wait limit
// of the bf16 attention kernel and whether its first descriptor is withheld.
long long g_attn_wait_limit = kWaitCycles;
int g_attn_withhold_first = 0;
// Split walk of the bf16 forward (adaspark_set_split_rows): a tile's selected
// cube that at most this many of its rows chose runs in a gathered tile.
int g_split_rows = kSplitRowsDefault;

}  // namespace

extern "C" {

size_t adaspark_cube_attn_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv, int d,
                                    int dtype) {
  if (!attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype)) return 0;
  const AttnGeom G = make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d);
  // the bf16 path's split walk keeps its records after the common layout
  return make_attn_layout(G).total + (dtype == ADASPARK_BF16 ? make_split_layout(G).total : 0);
}

}  // extern "C"

// AdaS-Attn with Top-p (topk == 0) or Top-K (topk > 0, p unused) selection.
// fp32 O of a training-mode call, after the inference layout
static size_t attn_train_bytes(const AttnGeom& G) {
  return (size_t)G.n_tokens * G.hq * G.d * sizeof(float);
}

static int cube_attn_impl(const void* Q, const void* K, const void* V, int dtype,
                          const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                          int n_vis, int n_tokens, int hq, int hkv, int d, float p, int topk,
                          void* out, void* workspace, size_t workspace_bytes, void* stream,
                          bool train = false, bool uniform = false, bool allow_split = true) {
  if (!Q || !K || !V || !cube_ids || !cube_offsets || !out || !workspace) return ADASPARK_EINVAL;
  if (!attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype)) return ADASPARK_EINVAL;
  if (topk < 0 || (topk == 0 && !p_valid(p))) return ADASPARK_EINVAL;
  if (train && dtype != ADASPARK_BF16) return ADASPARK_EUNSUPPORTED;
  const AttnGeom G = make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d);
  const AttnLayout L = make_attn_layout(G);
  const size_t need = L.total + (train ? attn_train_bytes(G) : 0);
  if (workspace_bytes < need || !aligned(workspace, kAlign)) return ADASPARK_EINVAL;
  const size_t es = dtype == ADASPARK_BF16 ? 2 : 4;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(out, 16) || es == 0)
    return ADASPARK_EINVAL;
  int rc = check_device();
  if (rc != ADASPARK_OK) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  const int dense = topk == 0 && p >= 1.0f;
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return ADASPARK_ECUDA;
  if (dense && cudaMemsetAsync(&hdr->pad[0], kModeDense, 1, s) != cudaSuccess)
    return ADASPARK_ECUDA;
  // Split walk: bf16 Top-p / Top-K inference calls whose workspace holds the
  // split region (as adaspark_cube_attn_workspace sizes it).
  const SplitLayout SL = make_split_layout(G);
  const bool split = allow_split && g_split_rows > 0 && dtype == ADASPARK_BF16 && !train &&
                     !dense && !uniform && n_vis > 0 && G.n_vtiles > 0 &&
                     workspace_bytes >= L.total + SL.total;
  SplitArgs sp{};
  if (split) {
    uint8_t* r = ws + L.total;
    sp.rows = g_split_rows;
    sp.cap = SL.cap;
    sp.max_mtiles = SL.max_mtiles;
    sp.walk_count = reinterpret_cast<int32_t*>(r + SL.walk_count);
    sp.walk_list = reinterpret_cast<uint16_t*>(r + SL.walk_list);
    sp.row_off = reinterpret_cast<int32_t*>(r + SL.row_off);
    sp.row_cnt = reinterpret_cast<int32_t*>(r + SL.row_cnt);
    sp.rec_row = reinterpret_cast<int32_t*>(r + SL.rec_row);
    sp.rec_cube = reinterpret_cast<int32_t*>(r + SL.rec_cube);
    sp.rec_gpos = reinterpret_cast<int32_t*>(r + SL.rec_gpos);
    sp.grp_cnt = reinterpret_cast<int32_t*>(r + SL.grp_cnt);
    sp.grp_base = reinterpret_cast<int32_t*>(r + SL.grp_base);
    sp.grp_tile = reinterpret_cast<int32_t*>(r + SL.grp_tile);
    sp.grec = reinterpret_cast<int32_t*>(r + SL.grec);
    sp.grow = reinterpret_cast<int32_t*>(r + SL.grow);
    sp.mt_info = reinterpret_cast<int4*>(r + SL.mt_info);
    sp.part_o = reinterpret_cast<__nv_bfloat16*>(r + SL.part_o);
    sp.part_lse = reinterpret_cast<float*>(r + SL.part_lse);
    if (cudaMemsetAsync(sp.grp_cnt, 0, (size_t)G.hkv * n_cubes * sizeof(int32_t), s) !=
        cudaSuccess)
      return ADASPARK_ECUDA;
  }
  if (train &&
      cudaMemsetAsync(reinterpret_cast<uint8_t*>(&hdr->pad[0]) + 1, 1, 1, s) != cudaSuccess)
    return ADASPARK_ECUDA;
  rc = cuda_rc(launch_validate(cube_ids, cube_offsets, nullptr, n_cubes, n_vis, n_tokens, hdr, s));
  if (rc) return rc;

  SelectArgs sa;
  sa.Q = Q;
  sa.cube_ids = cube_ids;
  sa.cube_offsets = cube_offsets;
  sa.kbar = reinterpret_cast<float*>(ws + L.kbar);
  sa.kbar_split = reinterpret_cast<__nv_bfloat16*>(ws + L.kbar_split);
  sa.tile_mask = reinterpret_cast<uint32_t*>(ws + L.tile_mask);
  sa.tile_list = reinterpret_cast<uint16_t*>(ws + L.tile_list);
  sa.tile_count = reinterpret_cast<int32_t*>(ws + L.tile_count);
  sa.hdr = hdr;
  sa.G = G;
  sa.p = p;
  sa.zscale = (float)(1.4426950408889634 / std::sqrt((double)d));
  sa.topk = topk;
  sa.sp = sp;

  if (uniform && n_vis > 0 && G.n_vtiles > 0) {
    rc = cuda_rc(launch_select_uniform(sa, s));
    if (rc) return rc;
  } else if (!dense && n_vis > 0 && G.n_vtiles > 0) {
    rc = cuda_rc(launch_cube_mean(K, dtype, cube_offsets, const_cast<float*>(sa.kbar),
                                  const_cast<__nv_bfloat16*>(sa.kbar_split), G, hdr, s));
    if (rc) return rc;
    rc = cuda_rc(dtype == ADASPARK_BF16 ? launch_select_tc(sa, s) : launch_select_simt(sa, dtype, s));
    if (rc) return rc;
    if (split) {
      rc = cuda_rc(launch_split_build(sp, G, cube_offsets, hdr, s));
      if (rc) return rc;
    }
  }

  AttnArgs aa;
  aa.Q = Q;
  aa.K = K;
  aa.V = V;
  aa.out = out;
  aa.cube_ids = cube_ids;
  aa.cube_offsets = cube_offsets;
  aa.tile_count = sa.tile_count;
  aa.tile_list = sa.tile_list;
  aa.tile_mask = sa.tile_mask;
  aa.hdr = hdr;
  aa.G = G;
  aa.dense = dense;
  aa.scale_log2 = sa.zscale;
  aa.lse = reinterpret_cast<float*>(ws + L.lse);
  aa.o32 = train ? reinterpret_cast<float*>(ws + L.total) : nullptr;
  aa.wait_limit = g_attn_wait_limit;
  aa.withhold_first = g_attn_withhold_first;
  aa.sp = sp;
  // When the layer's K and V outgrow what L2 holds alongside the other
  // traffic, visual tiles run one KV head after another, so that the blocks in
  // use belong to one head; otherwise all heads of a token range run together
  // (fewer CTAs then read the same lines at once).
  const double kv_bytes = 2.0 * n_tokens * hkv * d * (dtype == ADASPARK_BF16 ? 2 : 4);
  aa.kv_major = kv_bytes > 64.0 * 1024 * 1024 ? 1 : 0;
  if (dtype == ADASPARK_BF16) {
    if (split) {  // the gathered tiles first: the tiles' epilogues merge their results
      rc = cuda_rc(launch_attn_tc_gather(aa, s));
      if (rc) return rc;
    }
    return cuda_rc(launch_attn_tc(aa, s));
  }
  return cuda_rc(launch_attn_simt(aa, dtype, s));
}

// adaspark_cube_attn on the common layout alone (no split walk): the entry
// point with the library-held scratch array.
int adaspark::cube_attn_single_walk(const void* Q, const void* K, const void* V, int dtype,
                          const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                          int n_vis, int n_tokens, int hq, int hkv, int d, float p, void* out,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return cube_attn_impl(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis, n_tokens, hq, hkv,
                        d, p, 0, out, workspace, workspace_bytes, stream, false, false, false);
}

size_t adaspark::cube_attn_single_walk_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv,
                                       int d, int dtype) {
  if (!attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype)) return 0;
  return make_attn_layout(make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d)).total;
}

extern "C" {

int adaspark_cube_attn(const void* Q, const void* K, const void* V, int dtype,
                       const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                       int n_vis, int n_tokens, int hq, int hkv, int d, float p, void* out,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return cube_attn_impl(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis, n_tokens, hq, hkv,
                        d, p, 0, out, workspace, workspace_bytes, stream);
}

size_t adaspark_cube_attn_train_workspace(int n_tokens, int n_vis, int n_cubes, int hq,
                                          int hkv, int d, int dtype) {
  if (dtype != ADASPARK_BF16 || !attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype))
    return 0;
  const AttnGeom G = make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d);
  return make_attn_layout(G).total + attn_train_bytes(G);
}

int adaspark_cube_attn_train(const void* Q, const void* K, const void* V, int dtype,
                             const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                             int n_vis, int n_tokens, int hq, int hkv, int d, float p, void* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
  return cube_attn_impl(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis, n_tokens, hq, hkv,
                        d, p, 0, out, workspace, workspace_bytes, stream, true);
}

int adaspark_cube_attn_topk(const void* Q, const void* K, const void* V, int dtype,
                            const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                            int n_vis, int n_tokens, int hq, int hkv, int d, int k, void* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (k < 1) return ADASPARK_EINVAL;
  return cube_attn_impl(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis, n_tokens, hq, hkv,
                        d, 0.5f, k, out, workspace, workspace_bytes, stream);
}

int adaspark_cube_attn_uniform(const void* Q, const void* K, const void* V, int dtype,
                               const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                               int n_vis, int n_tokens, int hq, int hkv, int d, int k, void* out,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (k < 1) return ADASPARK_EINVAL;
  return cube_attn_impl(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis, n_tokens, hq, hkv,
                        d, 0.5f, k, out, workspace, workspace_bytes, stream, false, true);
}

int adaspark_attn_export_sets(const void* workspace, const int32_t* cube_ids, int n_cubes,
                              int n_vis, int n_tokens, int hq, int hkv, int d, int dtype,
                              uint32_t* sel_bits, void* stream) {
  if (!workspace || !sel_bits || !cube_ids) return ADASPARK_EINVAL;
  if (!attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype)) return ADASPARK_EINVAL;
  const AttnGeom G = make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d);
  const AttnLayout L = make_attn_layout(G);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t mode = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ADASPARK_ECUDA;
  const WsHeader* hdr = reinterpret_cast<const WsHeader*>(ws + L.header);
  if (cudaMemcpy(&mode, &hdr->pad[0], 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return ADASPARK_ECUDA;
  return cuda_rc(launch_export_sets(reinterpret_cast<const int32_t*>(ws + L.tile_count),
                                    reinterpret_cast<const uint16_t*>(ws + L.tile_list),
                                    reinterpret_cast<const uint32_t*>(ws + L.tile_mask),
                                    cube_ids, G, (mode & 0xff) == kModeDense, sel_bits, s));
}

int adaspark_attn_read_stats(const void* workspace, adaspark_attn_stats* stats, void* stream) {
  if (!workspace || !stats) return ADASPARK_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ADASPARK_ECUDA;
  const WsHeader* hdr = static_cast<const WsHeader*>(workspace);
  static_assert(sizeof(adaspark_attn_stats) == sizeof(hdr->stats), "stats size");
  return cuda_rc(cudaMemcpy(stats, hdr->stats, sizeof(adaspark_attn_stats), cudaMemcpyDeviceToHost));
}

size_t adaspark_token_ffn_workspace(int n_tokens, int n_vis, int n_cubes, int D, int F,
                                    int dtype) {
  if (!ffn_sizes_ok(n_tokens, n_vis, n_cubes, D, F, dtype)) return 0;
  return make_ffn_layout(n_tokens, n_vis, n_cubes, D, F, dtype == ADASPARK_BF16 ? 2 : 4).total;
}

int adaspark_token_ffn(const void* x, const void* W_gate, const void* W_up, const void* W_down,
                       int dtype, const int32_t* cube_ids, const int32_t* cube_offsets,
                       const uint8_t* text_mask, int n_cubes, int n_vis, int n_tokens, int D,
                       int F, float p, float* y, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return adaspark_token_ffn_ex(x, W_gate, W_up, W_down, dtype, cube_ids, cube_offsets, text_mask,
                               n_cubes, n_vis, n_tokens, D, F, p, ADASPARK_IMPORTANCE_L2_SHARE, y,
                               workspace, workspace_bytes, stream);
}

int adaspark_token_ffn_ex(const void* x, const void* W_gate, const void* W_up,
                          const void* W_down, int dtype, const int32_t* cube_ids,
                          const int32_t* cube_offsets, const uint8_t* text_mask, int n_cubes,
                          int n_vis, int n_tokens, int D, int F, float p, int importance,
                          float* y, void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !W_gate || !W_up || !W_down || !cube_ids || !cube_offsets || !text_mask || !y ||
      !workspace)
    return ADASPARK_EINVAL;
  if (!ffn_sizes_ok(n_tokens, n_vis, n_cubes, D, F, dtype) || !p_valid(p)) return ADASPARK_EINVAL;
  if (importance != ADASPARK_IMPORTANCE_L2_SHARE && importance != ADASPARK_IMPORTANCE_L2SQ_SHARE &&
      importance != ADASPARK_IMPORTANCE_SOFTMAX)
    return ADASPARK_EINVAL;
  const int es = dtype == ADASPARK_BF16 ? 2 : 4;
  const FfnLayout L = make_ffn_layout(n_tokens, n_vis, n_cubes, D, F, es);
  if (workspace_bytes < L.total || !aligned(workspace, kAlign)) return ADASPARK_EINVAL;
  if (!aligned(x, 16) || !aligned(W_gate, 16) || !aligned(W_up, 16) || !aligned(W_down, 16) ||
      !aligned(y, 16))
    return ADASPARK_EINVAL;
  int rc = check_device();
  if (rc != ADASPARK_OK) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  FfnArgs a;
  a.x = x;
  a.W_gate = W_gate;
  a.W_up = W_up;
  a.W_down = W_down;
  a.cube_ids = cube_ids;
  a.cube_offsets = cube_offsets;
  a.y = y;
  a.norms = reinterpret_cast<float*>(ws + L.norms);
  a.active = ws + L.active;
  a.cube_count = reinterpret_cast<int32_t*>(ws + L.cube_count);
  a.cube_start = reinterpret_cast<int32_t*>(ws + L.cube_start);
  a.idx = reinterpret_cast<int32_t*>(ws + L.idx);
  a.row_cube = reinterpret_cast<int32_t*>(ws + L.row_cube);
  a.xa = ws + L.xa;
  a.h = ws + L.h;
  a.sums = reinterpret_cast<float*>(ws + L.sums);
  a.wd16 = ws + L.wd16;
  a.skip = reinterpret_cast<int32_t*>(ws + L.skip);
  a.hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  a.n_tokens = n_tokens;
  a.n_vis = n_vis;
  a.n_cubes = n_cubes;
  a.D = D;
  a.F = F;
  a.p = p;
  a.dense = p >= 1.0f;
  a.importance = importance;

  if (cudaMemsetAsync(a.hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return ADASPARK_ECUDA;
  if (!a.dense && n_cubes > 0 &&
      cudaMemsetAsync(a.sums, 0, (size_t)n_cubes * D * sizeof(float), s) != cudaSuccess)
    return ADASPARK_ECUDA;
  if ((rc = cuda_rc(launch_validate(cube_ids, cube_offsets, text_mask, n_cubes, n_vis, n_tokens,
                                    a.hdr, s))))
    return rc;
  if ((rc = cuda_rc(launch_ffn_select(a, dtype, s)))) return rc;
  if ((rc = cuda_rc(launch_ffn_compact(a, dtype, s)))) return rc;
  if (dtype == ADASPARK_BF16) {
    if ((rc = cuda_rc(launch_wdown_to_fp16(a, s)))) return rc;
    if ((rc = cuda_rc(launch_ffn_gemm1_tc(a, s)))) return rc;
    if ((rc = cuda_rc(launch_ffn_gemm2_tc(a, s)))) return rc;
  } else {
    if ((rc = cuda_rc(launch_ffn_gemm1_simt(a, dtype, s)))) return rc;
    if ((rc = cuda_rc(launch_ffn_gemm2_simt(a, dtype, s)))) return rc;
  }
  return cuda_rc(launch_ffn_compensate(a, dtype, s));
}

size_t adaspark_cube_attn_backward_workspace(int n_tokens, int n_vis, int n_cubes, int hq,
                                             int hkv, int d, int dtype) {
  // the backward kernels are built for head_dim 128
  if (dtype != ADASPARK_BF16 || d != 128 ||
      !attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype))
    return 0;
  return make_attn_bwd_layout(make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d)).total;
}

int adaspark_cube_attn_backward(const void* Q, const void* K, const void* V, const void* dO,
                                int dtype, const int32_t* cube_ids,
                                const int32_t* cube_offsets, int n_cubes, int n_vis,
                                int n_tokens, int hq, int hkv, int d,
                                const void* fwd_workspace, float* dQ, float* dK, float* dV,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!Q || !K || !V || !dO || !cube_ids || !cube_offsets || !fwd_workspace || !dQ ||
      !dK || !dV || !workspace)
    return ADASPARK_EINVAL;
  if (dtype == ADASPARK_FP32) return ADASPARK_EUNSUPPORTED;
  if (dtype != ADASPARK_BF16 || !attn_sizes_ok(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype))
    return ADASPARK_EINVAL;
  if (d != 128) return ADASPARK_EUNSUPPORTED;   // the backward kernels are built for 128
  const AttnGeom G = make_attn_geom(n_tokens, n_vis, n_cubes, hq, hkv, d);
  const AttnBwdLayout L = make_attn_bwd_layout(G);
  if (workspace_bytes < L.total || !aligned(workspace, kAlign) || !aligned(fwd_workspace, kAlign))
    return ADASPARK_EINVAL;
  for (const void* ptr : {Q, K, V, dO, static_cast<const void*>(dQ),
                          static_cast<const void*>(dK), static_cast<const void*>(dV)})
    if (!aligned(ptr, 16)) return ADASPARK_EINVAL;
  int rc = check_device();
  if (rc != ADASPARK_OK) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const AttnLayout FL = make_attn_layout(G);
  const uint8_t* fws = static_cast<const uint8_t*>(fwd_workspace);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  AttnBwdArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.dO = static_cast<const __nv_bfloat16*>(dO);
  a.dQ = dQ;
  a.dK = dK;
  a.dV = dV;
  a.cube_ids = cube_ids;
  a.cube_offsets = cube_offsets;
  a.fhdr = reinterpret_cast<const WsHeader*>(fws + FL.header);
  a.tile_count = reinterpret_cast<const int32_t*>(fws + FL.tile_count);
  a.tile_list = reinterpret_cast<const uint16_t*>(fws + FL.tile_list);
  a.tile_mask = reinterpret_cast<const uint32_t*>(fws + FL.tile_mask);
  a.lse = reinterpret_cast<const float*>(fws + FL.lse);
  // read only when the forward ran in training mode (then its workspace holds it)
  a.o32 = reinterpret_cast<const float*>(fws + FL.total);
  a.hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  a.dot = reinterpret_cast<float*>(ws + L.dot);
  a.inv_count = reinterpret_cast<int32_t*>(ws + L.inv_count);
  a.inv_start = reinterpret_cast<int32_t*>(ws + L.inv_start);
  a.inv_list = reinterpret_cast<int32_t*>(ws + L.inv_list);
  a.inv_chunks = L.chunks;
  a.pieces = ws + L.pieces;
  a.G = G;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
  a.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  const double kv_bytes = 2.0 * n_tokens * hkv * d * 2;
  a.kv_major = kv_bytes > 64.0 * 1024 * 1024 ? 1 : 0;
  if (cudaMemsetAsync(a.hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return ADASPARK_ECUDA;
  return cuda_rc(launch_attn_backward_tc(a, s));
}

size_t adaspark_token_ffn_backward_workspace(int n_tokens, int n_vis, int n_cubes, int D, int F,
                                             int dtype) {
  if (dtype != ADASPARK_BF16 || !ffn_sizes_ok(n_tokens, n_vis, n_cubes, D, F, dtype)) return 0;
  return make_ffn_bwd_layout(n_tokens, n_cubes, D, F).total;
}

int adaspark_token_ffn_backward(const void* W_gate, const void* W_up, const void* W_down,
                                int dtype, const int32_t* cube_offsets, int n_cubes, int n_vis,
                                int n_tokens, int D, int F, const float* dy,
                                const void* fwd_workspace, float* dx, float* dW_gate,
                                float* dW_up, float* dW_down, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!W_gate || !W_up || !W_down || !cube_offsets || !dy || !fwd_workspace || !dx || !dW_gate ||
      !dW_up || !dW_down || !workspace)
    return ADASPARK_EINVAL;
  if (dtype == ADASPARK_FP32) return ADASPARK_EUNSUPPORTED;
  if (dtype != ADASPARK_BF16 || !ffn_sizes_ok(n_tokens, n_vis, n_cubes, D, F, dtype))
    return ADASPARK_EINVAL;
  const FfnBwdLayout L = make_ffn_bwd_layout(n_tokens, n_cubes, D, F);
  if (workspace_bytes < L.total || !aligned(workspace, kAlign) || !aligned(fwd_workspace, kAlign))
    return ADASPARK_EINVAL;
  for (const void* ptr : {W_gate, W_up, W_down, static_cast<const void*>(dy),
                          static_cast<const void*>(dx), static_cast<const void*>(dW_gate),
                          static_cast<const void*>(dW_up), static_cast<const void*>(dW_down)})
    if (!aligned(ptr, 16)) return ADASPARK_EINVAL;
  int rc = check_device();
  if (rc != ADASPARK_OK) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const FfnLayout FL = make_ffn_layout(n_tokens, n_vis, n_cubes, D, F, 2);
  const uint8_t* fws = static_cast<const uint8_t*>(fwd_workspace);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  FfnBwdArgs a;
  a.W_gate = static_cast<const __nv_bfloat16*>(W_gate);
  a.W_up = static_cast<const __nv_bfloat16*>(W_up);
  a.W_down = static_cast<const __nv_bfloat16*>(W_down);
  a.cube_offsets = cube_offsets;
  a.dy = dy;
  a.dx = dx;
  a.dWg = dW_gate;
  a.dWu = dW_up;
  a.dWd = dW_down;
  a.fhdr = reinterpret_cast<const WsHeader*>(fws + FL.header);
  a.m_active = &a.fhdr->m_active;
  a.active = fws + FL.active;
  a.cube_count = reinterpret_cast<const int32_t*>(fws + FL.cube_count);
  a.idx = reinterpret_cast<const int32_t*>(fws + FL.idx);
  a.row_cube = reinterpret_cast<const int32_t*>(fws + FL.row_cube);
  a.xa = reinterpret_cast<const __nv_bfloat16*>(fws + FL.xa);
  a.hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  a.gsum = reinterpret_cast<float*>(ws + L.gsum);
  a.df = reinterpret_cast<__nv_bfloat16*>(ws + L.df);
  a.dfT = reinterpret_cast<__nv_bfloat16*>(ws + L.dfT);
  a.xaT = reinterpret_cast<__nv_bfloat16*>(ws + L.xaT);
  a.wdT = reinterpret_cast<__nv_bfloat16*>(ws + L.wdT);
  a.wguT = reinterpret_cast<__nv_bfloat16*>(ws + L.wguT);
  a.dgu = reinterpret_cast<__nv_bfloat16*>(ws + L.dgu);
  a.dguT = reinterpret_cast<__nv_bfloat16*>(ws + L.dguT);
  a.hT = reinterpret_cast<__nv_bfloat16*>(ws + L.hT);
  a.n_tokens = n_tokens;
  a.n_vis = n_vis;
  a.n_cubes = n_cubes;
  a.D = D;
  a.F = F;
  a.mp = L.mp;
  if (cudaMemsetAsync(a.hdr, 0, sizeof(WsHeader), s) != cudaSuccess) return ADASPARK_ECUDA;
  return cuda_rc(launch_ffn_backward_tc(a, s));
}

int adaspark_ffn_export_active(const void* workspace, int n_tokens, int n_vis, int n_cubes, int D,
                               int F, int dtype, uint8_t* active, void* stream) {
  if (!workspace || !active) return ADASPARK_EINVAL;
  if (!ffn_sizes_ok(n_tokens, n_vis, n_cubes, D, F, dtype)) return ADASPARK_EINVAL;
  const FfnLayout L =
      make_ffn_layout(n_tokens, n_vis, n_cubes, D, F, dtype == ADASPARK_BF16 ? 2 : 4);
  return cuda_rc(cudaMemcpyAsync(active, static_cast<const uint8_t*>(workspace) + L.active,
                                 (size_t)n_tokens, cudaMemcpyDeviceToDevice,
                                 static_cast<cudaStream_t>(stream)));
}

int adaspark_ffn_read_stats(const void* workspace, adaspark_ffn_stats* stats, void* stream) {
  if (!workspace || !stats) return ADASPARK_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ADASPARK_ECUDA;
  const WsHeader* hdr = static_cast<const WsHeader*>(workspace);
  static_assert(sizeof(adaspark_ffn_stats) == sizeof(hdr->stats), "stats size");
  return cuda_rc(cudaMemcpy(stats, hdr->stats, sizeof(adaspark_ffn_stats), cudaMemcpyDeviceToHost));
}

int adaspark_set_split_rows(int rows) {
  if (rows < 0 || rows > kTileRows) return ADASPARK_EINVAL;
  g_split_rows = rows;
  return ADASPARK_OK;
}

int adaspark_debug_wait_expiry(int on, long long wait_cycles) {
  if (!on) {
    g_attn_wait_limit = kWaitCycles;
    g_attn_withhold_first = 0;
    return ADASPARK_OK;
  }
  if (wait_cycles < 100000 || wait_cycles > kWaitCycles) return ADASPARK_EINVAL;
  g_attn_wait_limit = wait_cycles;
  g_attn_withhold_first = 1;
  return ADASPARK_OK;
}

int adaspark_read_device_status(const void* workspace, uint32_t* detail, void* stream) {
  // detail: ADASPARK_DEV_* bits in 0..7, the code of the first failing check in 8..23
  if (!workspace) return ADASPARK_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ADASPARK_ECUDA;
  uint32_t st[2] = {0, 0};
  if (cudaMemcpy(st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ADASPARK_ECUDA;
  if (detail) *detail = (st[0] & 0xffu) | ((st[1] & 0xffffu) << 8);
  return st[0] ? ADASPARK_EDEVICE : ADASPARK_OK;
}

}  // extern "C"

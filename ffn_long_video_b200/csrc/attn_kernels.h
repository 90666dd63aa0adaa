// Kernel argument blocks and host launchers of AdaS-Attn.
#pragma once

#include "common.cuh"
#include "host_util.h"
#include "layout.cuh"

namespace adaspark {

// Device pointers of the split walk (SplitLayout), shared by the selection,
// the regrouping kernels and the attention; rows == 0: no split.
struct SplitArgs {
  int rows;                           // a cube chosen by at most this many rows leaves the walk
  int cap;                            // record capacity
  int max_mtiles;
  int32_t* walk_count;
  uint16_t* walk_list;
  int32_t* row_off;
  int32_t* row_cnt;
  int32_t* rec_row;
  int32_t* rec_cube;
  int32_t* rec_gpos;
  int32_t* grp_cnt;
  int32_t* grp_base;
  int32_t* grp_tile;
  int32_t* grec;
  int32_t* grow;
  int4* mt_info;
  __nv_bfloat16* part_o;
  float* part_lse;
};

struct SelectArgs {
  const void* Q;
  const int32_t* cube_ids;
  const int32_t* cube_offsets;
  const float* kbar;                  // [hkv][C][d]
  const __nv_bfloat16* kbar_split;    // [3][hkv][C][d]
  uint32_t* tile_mask;                // [n_vtiles][C][4]
  uint16_t* tile_list;                // [n_vtiles][C]
  int32_t* tile_count;                // [n_vtiles]
  WsHeader* hdr;
  AttnGeom G;
  float p;
  float zscale;                       // log2(e) / sqrt(d)
  int topk;                           // > 0: Top-K with this k instead of Top-p
  SplitArgs sp;
};

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  void* out;
  const int32_t* cube_ids;
  const int32_t* cube_offsets;
  const int32_t* tile_count;
  const uint16_t* tile_list;
  const uint32_t* tile_mask;
  WsHeader* hdr;
  AttnGeom G;
  int dense;                          // p == 1: every preceding cube, no lists
  float scale_log2;                   // log2(e) / sqrt(d)
  int kv_major;                       // visual tiles ordered one KV head after another
  float* lse;                         // [N][hq] m + log2(l) per row (bf16 path), for the backward
  float* o32;                         // [N][hq][d] fp32 O with P split hi + lo (training), or null
  long long wait_limit;               // SM cycles before a wait gives up (bf16 kernel)
  int withhold_first;                 // test hook: the first descriptor is never announced
  SplitArgs sp;                       // split walk (sp.rows == 0: none)
};

// Backward of AdaS-Attn (sets of a forward call held fixed).
struct AttnBwdArgs {
  const __nv_bfloat16* Q;             // [N][hq][d]
  const __nv_bfloat16* K;             // [N][hkv][d]
  const __nv_bfloat16* V;             // [N][hkv][d]
  const __nv_bfloat16* dO;            // [N][hq][d]
  float* dQ;                          // [N][hq][d]
  float* dK;                          // [N][hkv][d]
  float* dV;                          // [N][hkv][d]
  const int32_t* cube_ids;
  const int32_t* cube_offsets;
  // from the forward workspace
  const WsHeader* fhdr;
  const int32_t* tile_count;
  const uint16_t* tile_list;
  const uint32_t* tile_mask;
  const float* lse;                   // [N][hq]
  // backward workspace
  WsHeader* hdr;
  float* dot;                         // [N][hq] D_r = sum_j P_rj dP_rj (from attn_bwd_dq)
  int32_t* inv_count;                 // [hkv][C][inv_chunks] tiles admitting cube j, per chunk
  int32_t* inv_start;                 // [hkv * C * inv_chunks + 1] exclusive prefix
  int32_t* inv_list;                  // tile indices, ascending per (kv, j)
  int inv_chunks;                     // chunks of kInvChunk visual tiles per KV head
  const float* o32;                   // forward's fp32 O when it ran in training mode
  void* pieces;                       // key pieces of up to 64 keys (cube, k0, nk), cube order
  AttnGeom G;
  int kv_major;
  float scale_log2;                   // log2(e) / sqrt(d)
  float inv_sqrt_d;
};
// The forward call ran dense (p = 1: every preceding cube, no lists): the
// first byte of its header's pad[0], set by the forward's host code.
__device__ __forceinline__ bool fwd_was_dense(const WsHeader* fhdr) {
  return reinterpret_cast<const volatile uint8_t*>(&fhdr->pad[0])[0] == 1u;
}
// The forward call ran in training mode (adaspark_cube_attn_train): its
// workspace holds O in fp32 after the inference layout (second byte of pad[0]).
__device__ __forceinline__ bool fwd_was_train(const WsHeader* fhdr) {
  return reinterpret_cast<const volatile uint8_t*>(&fhdr->pad[0])[1] == 1u;
}
cudaError_t launch_attn_backward_tc(const AttnBwdArgs& a, cudaStream_t s);

cudaError_t launch_validate(const int32_t* cube_ids, const int32_t* off, const uint8_t* text_mask,
                            int n_cubes, int n_vis, int n_tokens, WsHeader* hdr, cudaStream_t s);
cudaError_t launch_cube_mean(const void* K, int dtype, const int32_t* off, float* kbar,
                             __nv_bfloat16* split, const AttnGeom& G, WsHeader* hdr,
                             cudaStream_t s);
cudaError_t launch_select_simt(const SelectArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_select_tc(const SelectArgs& a, cudaStream_t s);
cudaError_t launch_select_uniform(const SelectArgs& a, cudaStream_t s);
cudaError_t launch_export_sets(const int32_t* tile_count, const uint16_t* tile_list,
                               const uint32_t* tile_mask, const int32_t* cube_ids,
                               const AttnGeom& G, int dense, uint32_t* bits, cudaStream_t s);
cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s);
// Split walk: group the records by (KV head, cube) and number the gathered
// tiles (after the selection), then run the gathered tiles (before the tiles'
// own walk, whose epilogue merges their partial results).
cudaError_t launch_split_build(const SplitArgs& sp, const AttnGeom& G,
                               const int32_t* cube_offsets, WsHeader* hdr, cudaStream_t s);
cudaError_t launch_attn_tc_gather(const AttnArgs& a, cudaStream_t s);

}  // namespace adaspark

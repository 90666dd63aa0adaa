// Problem geometry and workspace layout of the two calls (host and device).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace adaspark {

constexpr int kTileRows = 128;      // rows of one attention / selection tile
constexpr int kMaxCubeTokens = 256; // largest cube accepted
constexpr int kMaxCubes = 65535;    // cube ids fit 16 bits in the selection lists

// Geometry of AdaS-Attn. A "row" is one (token, query head) pair. Rows of one
// KV head are ordered r = t * g + (h mod g) and cut into 128-row tiles; visual
// tiles cover tokens [0, n_vis), text tiles the suffix.
struct AttnGeom {
  int n_tokens, n_vis, n_cubes, hq, hkv, d, g;
  int vtiles_per_kv, ttiles_per_kv;  // tiles per KV head
  int n_vtiles, n_ttiles;
  int pool_rows;                     // overflow-pool capacity (rows)
};

__host__ __device__ inline AttnGeom make_attn_geom(int n_tokens, int n_vis, int n_cubes, int hq,
                                                   int hkv, int d) {
  AttnGeom G;
  G.n_tokens = n_tokens;
  G.n_vis = n_vis;
  G.n_cubes = n_cubes;
  G.hq = hq;
  G.hkv = hkv;
  G.d = d;
  G.g = hq / hkv;
  long long vrows = (long long)n_vis * G.g;
  long long trows = (long long)(n_tokens - n_vis) * G.g;
  G.vtiles_per_kv = (int)((vrows + kTileRows - 1) / kTileRows);
  G.ttiles_per_kv = (int)((trows + kTileRows - 1) / kTileRows);
  G.n_vtiles = G.vtiles_per_kv * hkv;
  G.n_ttiles = G.ttiles_per_kv * hkv;
  long long rows = vrows * hkv;
  long long pr = rows / 16;
  if (pr < 1024) pr = 1024;
  if (pr > 16384) pr = 16384;
  G.pool_rows = (int)pr;
  return G;
}

// Workspace of adaspark_cube_attn. Offsets in bytes from the workspace base.
struct AttnLayout {
  size_t header;      // WsHeader
  size_t kbar;        // float [hkv][C][d]
  size_t kbar_split;  // bf16 [3][hkv][C][d]  (hi, mid, lo parts of kbar)
  size_t tile_count;  // int32 [n_vtiles]
  size_t tile_list;   // uint16 [n_vtiles][C]  cube ids with any row bit, ascending
  size_t tile_mask;   // uint32 [n_vtiles][C][4]  128 row bits per (tile, cube)
  size_t pool;        // overflow pool: [pool_rows][C] x (float z, int32 j)
  size_t total;
};

__host__ __device__ inline AttnLayout make_attn_layout(const AttnGeom& G) {
  AttnLayout L;
  size_t o = 0;
  L.header = o; o += align_up(sizeof(WsHeader));
  L.kbar = o; o += align_up((size_t)G.hkv * G.n_cubes * G.d * 4);
  L.kbar_split = o; o += align_up((size_t)3 * G.hkv * G.n_cubes * G.d * 2);
  L.tile_count = o; o += align_up((size_t)G.n_vtiles * 4);
  L.tile_list = o; o += align_up((size_t)G.n_vtiles * G.n_cubes * 2);
  L.tile_mask = o; o += align_up((size_t)G.n_vtiles * G.n_cubes * 16);
  L.pool = o; o += align_up((size_t)G.pool_rows * G.n_cubes * 8);
  L.total = o;
  return L;
}

// Workspace of adaspark_token_ffn.
struct FfnLayout {
  size_t header;
  size_t norms;       // float [n_vis]
  size_t active;      // uint8 [n_tokens]
  size_t cube_count;  // int32 [C]  active tokens per cube
  size_t cube_start;  // int32 [C+1] exclusive prefix of cube_count
  size_t idx;         // int32 [n_tokens] active rows (visual ascending, then text)
  size_t row_cube;    // int32 [n_tokens] cube of each active row (-1 for text)
  size_t xa;          // dtype [n_tokens][D] gathered active rows
  size_t h;           // dtype [n_tokens][F] SwiGLU activations
  size_t sums;        // float [C][D] per-cube sums of FFN over active rows
  size_t total;
};

__host__ __device__ inline FfnLayout make_ffn_layout(int n_tokens, int n_vis, int n_cubes, int D,
                                                     int F, int esize) {
  FfnLayout L;
  size_t o = 0;
  L.header = o; o += align_up(sizeof(WsHeader));
  L.norms = o; o += align_up((size_t)(n_vis > 0 ? n_vis : 1) * 4);
  L.active = o; o += align_up((size_t)n_tokens);
  L.cube_count = o; o += align_up((size_t)(n_cubes + 1) * 4);
  L.cube_start = o; o += align_up((size_t)(n_cubes + 1) * 4);
  L.idx = o; o += align_up((size_t)n_tokens * 4);
  L.row_cube = o; o += align_up((size_t)n_tokens * 4);
  L.xa = o; o += align_up((size_t)n_tokens * D * esize, 1024);
  L.h = o; o += align_up((size_t)n_tokens * F * esize, 1024);
  L.sums = o; o += align_up((size_t)(n_cubes > 0 ? n_cubes : 1) * D * 4);
  L.total = o;
  return L;
}

}  // namespace adaspark

// Problem geometry and workspace layout of the two calls (host and device).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace adaspark {

constexpr int kTileRows = 128;      // rows of one attention / selection tile
constexpr int kMaxCubeTokens = 256; // largest cube accepted
constexpr int kMaxCubes = 65535;    // cube ids fit 16 bits in the selection lists
constexpr int kInvChunk = 128;      // visual tiles per chunk of the backward's inverted lists

// Geometry of AdaS-Attn. A "row" is one (token, query head) pair. Rows are
// grouped by KV head, then by query head within the group, then by token, and
// cut into 128-token tiles that never straddle a head: tile tl of KV head kv
// holds query head kv * g + tl / tiles_per_head and tokens
// (tl % tiles_per_head) * 128 + [0, 128). Rows of one tile thus share the head
// and span one or two neighbouring cubes, which keeps the union of their cube
// sets small. Visual tiles cover tokens [0, n_vis), text tiles the suffix.
struct AttnGeom {
  int n_tokens, n_vis, n_cubes, hq, hkv, d, g;
  int vtiles_per_head, ttiles_per_head;  // 128-token tiles per query head
  int vtiles_per_kv, ttiles_per_kv;      // tiles per KV head
  int n_vtiles, n_ttiles;
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
  G.vtiles_per_head = (n_vis + kTileRows - 1) / kTileRows;
  G.ttiles_per_head = (n_tokens - n_vis + kTileRows - 1) / kTileRows;
  G.vtiles_per_kv = G.vtiles_per_head * G.g;
  G.ttiles_per_kv = G.ttiles_per_head * G.g;
  G.n_vtiles = G.vtiles_per_kv * hkv;
  G.n_ttiles = G.ttiles_per_kv * hkv;
  return G;
}

// Row i (0..127) of tile `bt` (index within its kind: kv * tiles_per_kv + tl).
struct TileRow {
  bool valid;
  int t;   // token
  int h;   // query head
};
__host__ __device__ inline TileRow tile_row(const AttnGeom& G, bool text, int bt, int i) {
  const int per_kv = text ? G.ttiles_per_kv : G.vtiles_per_kv;
  const int per_head = text ? G.ttiles_per_head : G.vtiles_per_head;
  const int kv = bt / per_kv;
  const int tl = bt - kv * per_kv;
  const int hh = tl / per_head;
  const int tt = (tl - hh * per_head) * kTileRows + i;
  TileRow R;
  const int base = text ? G.n_vis : 0;
  const int count = text ? G.n_tokens - G.n_vis : G.n_vis;
  R.valid = tt < count;
  R.t = base + (R.valid ? tt : 0);
  R.h = kv * G.g + hh;
  return R;
}

// Workspace of adaspark_cube_attn. Offsets in bytes from the workspace base.
struct AttnLayout {
  size_t header;      // WsHeader
  size_t kbar;        // float [hkv][C][d]
  size_t kbar_split;  // bf16 [3][hkv][C][d]  (hi, mid, lo parts of kbar)
  size_t tile_count;  // int32 [n_vtiles]
  size_t tile_list;   // uint16 [n_vtiles][C]  cube ids with any row bit, ascending
  size_t tile_mask;   // uint32 [n_vtiles][C][4]  128 row bits per (tile, cube)
  size_t lse;         // float [N][hq]  log2-sum-exp of each row's scaled logits
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
  L.lse = o; o += align_up((size_t)G.n_tokens * G.hq * 4);
  L.total = o;
  return L;
}

// Split walk of the bf16 forward (after the layout above; a training-mode call,
// which never splits, keeps its fp32 O in the same place). A visual tile's
// selected cubes that at most `split rows` of its 128 rows chose (and that are
// no row's own cube) leave the tile's walk; their (row, cube) pairs, the
// records, are regrouped by (KV head, cube) into gathered 128-row tiles whose
// partial results the tile merges into its rows at the end.
struct SplitLayout {
  size_t walk_count;  // int32 [n_vtiles]       blocks the tile itself walks
  size_t walk_list;   // uint16 [n_vtiles][C]   their cube ids, ascending
  size_t row_off;     // int32 [n_vis * hq]     first record of a visual row
  size_t row_cnt;     // int32 [n_vis * hq]     its number of records
  size_t rec_row;     // int32 [cap]            record -> row (t * hq + h), -1 unused
  size_t rec_cube;    // int32 [cap]            record -> cube
  size_t rec_gpos;    // int32 [cap]            record -> place in its group
  size_t grp_cnt;     // int32 [hkv * C]        records per (KV head, cube)
  size_t grp_base;    // int32 [hkv * C + 1]    exclusive prefix of grp_cnt
  size_t grp_tile;    // int32 [hkv * C + 1]    exclusive prefix of gathered tiles
  size_t grec;        // int32 [cap]            records grouped by (KV head, cube)
  size_t grow;        // int32 [cap]            their rows, in the same order
  size_t mt_info;     // int4 [max_mtiles]      gathered tile: first slot, rows | kv << 8, cube's
                      //                        first and end token
  size_t part_o;      // bf16 [cap][d]          a record's normalised partial output
  size_t part_lse;    // float [cap]            and its log2-sum-exp
  int cap;            // records
  int max_mtiles;     // cap / 128 + hkv * C (the gathered launch's grid)
  size_t total;
};

constexpr int kSplitRecordsPerRow = 6;  // record capacity per visual row
constexpr int kSplitRowsDefault = 8;    // default of adaspark_set_split_rows

__host__ __device__ inline SplitLayout make_split_layout(const AttnGeom& G) {
  SplitLayout L;
  const size_t rows = (size_t)G.n_vis * G.hq;
  const size_t groups = (size_t)G.hkv * (G.n_cubes > 0 ? G.n_cubes : 1);
  size_t cap = rows * kSplitRecordsPerRow;
  if (cap > (size_t)0x3fffffff) cap = 0x3fffffff;
  L.cap = (int)cap;
  L.max_mtiles = (int)((cap + kTileRows - 1) / kTileRows + groups);
  size_t o = 0;
  L.walk_count = o; o += align_up((size_t)(G.n_vtiles > 0 ? G.n_vtiles : 1) * 4);
  L.walk_list = o; o += align_up((size_t)(G.n_vtiles > 0 ? G.n_vtiles : 1) *
                                 (G.n_cubes > 0 ? G.n_cubes : 1) * 2);
  L.row_off = o; o += align_up((rows > 0 ? rows : 1) * 4);
  L.row_cnt = o; o += align_up((rows > 0 ? rows : 1) * 4);
  L.rec_row = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.rec_cube = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.rec_gpos = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.grp_cnt = o; o += align_up(groups * 4);
  L.grp_base = o; o += align_up((groups + 1) * 4);
  L.grp_tile = o; o += align_up((groups + 1) * 4);
  L.grec = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.grow = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.mt_info = o; o += align_up((size_t)L.max_mtiles * 16);
  L.part_o = o; o += align_up((cap > 0 ? cap : 1) * (size_t)G.d * 2);
  L.part_lse = o; o += align_up((cap > 0 ? cap : 1) * 4);
  L.total = o;
  return L;
}

// Workspace of adaspark_cube_attn_backward.
struct AttnBwdLayout {
  size_t header;
  size_t dot;        // float [N][hq]
  size_t inv_count;  // int32 [hkv][C][chunks]
  size_t inv_start;  // int32 [hkv * C * chunks + 1]
  size_t inv_list;   // int32 [n_vtiles][C] (capacity; filled per (kv, j) segment)
  size_t pieces;     // int4 [4 C + text pieces] key pieces (cube, k0, nk, -)
  int chunks;        // chunks of kInvChunk visual tiles per KV head
  size_t total;
};

__host__ __device__ inline AttnBwdLayout make_attn_bwd_layout(const AttnGeom& G) {
  AttnBwdLayout L;
  L.chunks = (G.vtiles_per_kv + kInvChunk - 1) / kInvChunk;
  if (L.chunks < 1) L.chunks = 1;
  const size_t nkey = (size_t)G.hkv * (G.n_cubes > 0 ? G.n_cubes : 1) * L.chunks;
  size_t o = 0;
  L.header = o; o += align_up(sizeof(WsHeader));
  L.dot = o; o += align_up((size_t)G.n_tokens * G.hq * 4);
  L.inv_count = o; o += align_up(nkey * 4);
  L.inv_start = o; o += align_up((nkey + 1) * 4);
  L.inv_list = o; o += align_up((size_t)(G.n_vtiles > 0 ? G.n_vtiles : 1) *
                                (G.n_cubes > 0 ? G.n_cubes : 1) * 4);
  L.pieces = o; o += align_up(((size_t)4 * G.n_cubes + (G.n_tokens - G.n_vis + 63) / 64 + 1) * 16);
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
  size_t wd16;        // fp16 [D][F] copy of W_down (bf16 path)
  size_t skip;        // int32 [n_vis] skipped visual rows, cube by cube
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
  L.wd16 = o; o += align_up(esize == 2 ? (size_t)D * F * 2 : 0, 1024);
  L.skip = o; o += align_up((size_t)(n_vis > 0 ? n_vis : 1) * 4);
  L.total = o;
  return L;
}

// Workspace of adaspark_token_ffn_backward (bf16 path).
struct FfnBwdLayout {
  size_t header;
  size_t gsum;   // float [C][D]
  size_t df;     // bf16 [N][D]
  size_t dfT;    // bf16 [D][mp]
  size_t xaT;    // bf16 [D][mp]
  size_t wdT;    // bf16 [F][D]
  size_t wguT;   // bf16 [D][2F]
  size_t dgu;    // bf16 [N][2F]
  size_t dguT;   // bf16 [2F][mp]
  size_t hT;     // bf16 [F][mp]
  size_t mp;     // N rounded up to 64
  size_t total;
};

__host__ __device__ inline FfnBwdLayout make_ffn_bwd_layout(int n_tokens, int n_cubes, int D,
                                                            int F) {
  FfnBwdLayout L;
  const size_t N = (size_t)n_tokens;
  L.mp = (N + 63) / 64 * 64;
  size_t o = 0;
  L.header = o; o += align_up(sizeof(WsHeader));
  L.gsum = o; o += align_up((size_t)(n_cubes > 0 ? n_cubes : 1) * D * 4, 1024);
  L.df = o; o += align_up(N * D * 2, 1024);
  L.dfT = o; o += align_up((size_t)D * L.mp * 2, 1024);
  L.xaT = o; o += align_up((size_t)D * L.mp * 2, 1024);
  L.wdT = o; o += align_up((size_t)F * D * 2, 1024);
  L.wguT = o; o += align_up((size_t)D * 2 * F * 2, 1024);
  L.dgu = o; o += align_up(N * 2 * F * 2, 1024);
  L.dguT = o; o += align_up((size_t)2 * F * L.mp * 2, 1024);
  L.hT = o; o += align_up((size_t)F * L.mp * 2, 1024);
  L.total = o;
  return L;
}

}  // namespace adaspark

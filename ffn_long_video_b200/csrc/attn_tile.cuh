// Order of the 128-row attention tiles over the grid (forward and backward
// kernels of AdaS-Attn): which tile a CTA of a one-tile-per-CTA launch takes.
#pragma once

#include "layout.cuh"

namespace adaspark {

struct TileInfo {
  bool text;
  int bt;        // tile index within its kind
  int kv;
  int t_hi;      // last valid token of the tile
};

__device__ __forceinline__ TileInfo decode_tile(const AttnGeom& G, bool kv_major) {
  TileInfo T;
  const int b = blockIdx.x;
  T.text = b < G.n_ttiles;  // text tiles first (the heaviest)
  if (T.text) {
    T.bt = b;
  } else if (kv_major) {
    // Visual tiles, one KV head after the other (the K/V blocks in use then fit
    // in L2), latest tokens first within a KV head (the heaviest tiles first):
    // rank r -> KV head, token tile, then query head of the group.
    const int r = b - G.n_ttiles;
    const int per_head = G.vtiles_per_head;
    const int kv = r / G.vtiles_per_kv;
    const int rk = r - kv * G.vtiles_per_kv;
    const int tt = per_head - 1 - rk / G.g;
    const int hh = rk % G.g;
    T.bt = kv * G.vtiles_per_kv + hh * per_head + tt;
  } else {
    // visual tiles, latest tokens first: rank r -> token tile, then head
    const int r = b - G.n_ttiles;
    const int per_head = G.vtiles_per_head;
    const int tt = per_head - 1 - r / G.hq;
    const int hq_idx = r % G.hq;                 // query head
    const int kv = hq_idx / G.g, hh = hq_idx - kv * G.g;
    T.bt = kv * G.vtiles_per_kv + hh * per_head + tt;
  }
  T.kv = T.bt / (T.text ? G.ttiles_per_kv : G.vtiles_per_kv);
  const int per_head = T.text ? G.ttiles_per_head : G.vtiles_per_head;
  const int count = T.text ? G.n_tokens - G.n_vis : G.n_vis;
  const int tl = T.bt - T.kv * (T.text ? G.ttiles_per_kv : G.vtiles_per_kv);
  const int tt = tl % per_head;
  T.t_hi = (T.text ? G.n_vis : 0) + min(tt * kTileRows + kTileRows, count) - 1;
  return T;
}

}  // namespace adaspark

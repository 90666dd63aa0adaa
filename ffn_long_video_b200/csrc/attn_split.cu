// Split walk of AdaS-Attn: regrouping of the records (see SplitLayout).
//
// A visual tile walks the key blocks of the cubes that any of its 128 rows
// selected (key design 2 of the AdaSpark note runs each row over its own
// set; the tile runs the union). A cube that only a few of the tile's rows
// chose costs the tile a whole block for those rows. Such (row, cube) pairs,
// the records the selection writes, are regrouped here by (KV head, cube):
// every group becomes ceil(count / 128) gathered tiles of query rows from
// many tiles, run by the gathered-tile kernel (attn_gather_kernel) over the
// cube's keys alone; each record's partial result (normalised output and
// log2-sum-exp) is merged into its row at the end of the row's own walk.
#include "attn_kernels.h"

namespace adaspark {
namespace split {

// Exclusive prefixes of the group counts and of the gathered tiles per group;
// hdr->sched[1] = number of gathered tiles.
// One block of 1024 threads.
__global__ void __launch_bounds__(1024) split_prefix_kernel(SplitArgs sp, int n_groups,
                                                            WsHeader* hdr) {
  __shared__ int s_rec[32], s_til[32];
  if (status_bad(hdr)) {
    if (threadIdx.x == 0) hdr->sched[1] = 0;
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int run_rec = 0, run_til = 0;
  for (int base = 0; base < n_groups; base += 1024) {
    const int g = base + tid;
    const int c = g < n_groups ? sp.grp_cnt[g] : 0;
    const int nt = (c + kTileRows - 1) / kTileRows;
    int ir = c, it = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vr = __shfl_up_sync(0xffffffffu, ir, o);
      const int vt = __shfl_up_sync(0xffffffffu, it, o);
      if (lane >= o) {
        ir += vr;
        it += vt;
      }
    }
    if (lane == 31) {
      s_rec[warp] = ir;
      s_til[warp] = it;
    }
    __syncthreads();
    int pr = run_rec, pt = run_til, tr = 0, tt = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < warp) {
        pr += s_rec[w];
        pt += s_til[w];
      }
      tr += s_rec[w];
      tt += s_til[w];
    }
    if (g < n_groups) {
      sp.grp_base[g] = pr + ir - c;
      sp.grp_tile[g] = pt + it - nt;
    }
    __syncthreads();
    run_rec += tr;
    run_til += tt;
  }
  if (tid == 0) {
    sp.grp_base[n_groups] = run_rec;
    sp.grp_tile[n_groups] = run_til;
    hdr->sched[1] = (uint32_t)min(run_til, sp.max_mtiles);
  }
}

// Gathered tile table (first record slot, rows | KV head << 8, the cube's
// first and end token) and the records placed group by group at the places the
// selection gave them, with their rows beside them. Grid-stride over groups,
// then records.
__global__ void __launch_bounds__(256) split_scatter_kernel(SplitArgs sp, int n_groups, int C,
                                                            int hq, int g_size,
                                                            const int32_t* cube_offsets,
                                                            WsHeader* hdr) {
  if (status_bad(hdr)) return;
  const int stride = gridDim.x * blockDim.x;
  const int first = blockIdx.x * blockDim.x + threadIdx.x;
  for (int g = first; g < n_groups; g += stride) {
    const int t0 = sp.grp_tile[g], t1 = min(sp.grp_tile[g + 1], sp.max_mtiles);
    if (t0 >= t1) continue;
    const int kv = g / C, cube = g - kv * C;
    const int b0 = sp.grp_base[g], b1 = sp.grp_base[g + 1];
    const int ks = cube_offsets[cube], ke = cube_offsets[cube + 1];
    for (int m = t0; m < t1; ++m) {
      const int f = b0 + (m - t0) * kTileRows;
      sp.mt_info[m] = make_int4(f, min(kTileRows, b1 - f) | (kv << 8), ks, ke);
    }
  }
  const int n_rec = (int)min((long long)hdr->sched[0], (long long)sp.cap);
  for (int i = first; i < n_rec; i += stride) {
    const int rid = sp.rec_row[i];
    if (rid < 0) continue;                      // reserved by a tile that did not split
    const int kv = (rid % hq) / g_size;
    const int g = kv * C + sp.rec_cube[i];
    const int slot = sp.grp_base[g] + sp.rec_gpos[i];
    sp.grec[slot] = i;
    sp.grow[slot] = rid;
  }
}

}  // namespace split

cudaError_t launch_split_build(const SplitArgs& sp, const AttnGeom& G,
                               const int32_t* cube_offsets, WsHeader* hdr, cudaStream_t s) {
  const int n_groups = G.hkv * G.n_cubes;
  if (n_groups == 0) return cudaSuccess;
  cudaError_t e = launch("split_prefix", split::split_prefix_kernel, dim3(1), dim3(1024), 0, s,
                         sp, n_groups, hdr);
  if (e != cudaSuccess) return e;
  return launch("split_scatter", split::split_scatter_kernel, dim3(148 * 4), dim3(256), 0, s, sp,
                n_groups, G.n_cubes, G.hq, G.g, cube_offsets, hdr);
}

}  // namespace adaspark

// AdaS-Attn cube selection with tensor-core scores (bf16 path).
//
// Key design 2 of the AdaSpark note: for the 128 rows of a tile (128 tokens of
// one query head), P_i = softmax_j<i(q . kbar_j / sqrt(d)), S_i = Top-p(P_i, p).
// The scores of a tile against all preceding cubes form a dense 128 x c
// contraction, computed on tcgen05 32 cubes at a time into TMEM. kbar is split
// into three bf16 parts (hi + mid + lo, ~24 significant bits); the queries are
// bf16, so every product is exact and the fp32-accumulated sum of the three
// passes reproduces the fp32 dot product. Each row's Top-p cut is then found by
// the streaming histogram cut of select.cuh, one thread per row; the scores are
// recomputed for every pass with the same MMA sequence, hence bit-identical.
// Passes: histogram, emission, then (only while some row's cut is still open)
// extra passes; after each pass from the emission on, the row threads vote and
// the producer and MMA warps read the vote through a per-round barrier.
//   warp 0     TMA producer: kbar chunks [3 parts][2 halves][32 cubes][64 dims]
//              from a 3D map over [part*hkv + kv][cube][dim] (no multicast)
//   warp 1     TMEM allocator + tcgen05.mma issuer (M=128, N=32, K=16 x 24),
//              A = the query tile held in TMEM
//   warps 2-5  one thread per row: Q gather into TMEM, histogram pass, cut,
//              emission of the 128-bit row masks, tile cube list.
// The query tile lives in tensor memory (64 columns) rather than shared memory
// and the cut lists reuse the histogram's storage, so a CTA needs about 105 KB
// of shared memory (three K stages and the per-row histograms) and two CTAs
// share an SM.
#include "attn_kernels.h"
#include "select.cuh"

namespace adaspark {
namespace seltc {

constexpr int NC = 32;                          // cubes per chunk (MMA N)
constexpr int STAGES = 3;
constexpr int SBUF = 4;                         // TMEM score buffers
constexpr int THREADS = 192;
constexpr int BOX_BYTES = NC * 128;             // 32 cubes x 64 dims bf16
// kbar chunk of head dimension D: 3 parts x D / 64 halves of BOX_BYTES
template <int D> constexpr int chunk_bytes() { return 3 * (D / 64) * BOX_BYTES; }
template <int D> constexpr size_t smem_bytes() {
  return 1024 + STAGES * chunk_bytes<D>() + sizeof(sel::Smem) + 256;
}
constexpr int TMEM_COLS = 256;                  // S buffers 0..127, Q tile 128..191
constexpr int Q_COL = 128;

template <int D>
__global__ void __launch_bounds__(THREADS, 2)
    select_tc_kernel(const __grid_constant__ CUtensorMap mapKb, SelectArgs a) {
  constexpr int HALVES = D / 64;                // 64-dim halves of a query / kbar row
  constexpr int CHUNK_BYTES = chunk_bytes<D>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  sel::Smem* ss = reinterpret_cast<sel::Smem*>(sK + STAGES * CHUNK_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(ss) + sizeof(sel::Smem));
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + STAGES;
  uint64_t* s_full = k_empty + STAGES;
  uint64_t* s_empty = s_full + SBUF;
  uint64_t* q_full = s_empty + SBUF;
  uint64_t* drain = q_full + 1;
  uint64_t* decide = drain + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(decide + 1);
  __shared__ volatile int s_abort;
  __shared__ int s_hi, s_bad, s_wcnt[8], s_misc[2];
  __shared__ volatile int s_more[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  const int vt = blockIdx.x;
  const int kv = vt / G.vtiles_per_kv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int b = 0; b < SBUF; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
    }
    mbar_init(q_full, 128);
    mbar_init(drain, 1);
    mbar_init(decide, 128);
    fence_mbar_init();
    s_abort = 0;
    s_more[0] = 0;
    s_more[1] = 0;
    s_bad = status_bad(hdr) ? 1 : 0;
    // rows are tokens in order: the last valid row holds the highest own cube
    const TileRow last = tile_row(G, false, vt, 0);
    const int t_hi = min(last.t + kTileRows, G.n_vis) - 1;
    s_hi = s_bad ? -1 : a.cube_ids[t_hi];
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&mapKb);
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int c_hi = s_hi;                       // candidates of the tile: cubes < c_hi
  const int nch = c_hi > 0 ? (c_hi + NC - 1) / NC : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nch > 0) {
      bool ok = true;
      int it = 0;
      for (int pass = 0; ok; ++pass) {
        if (pass >= 2) {  // decision of round pass - 2
          const int r = pass - 2;
          if (!mbar_wait(decide, r & 1, &s_abort, hdr, 0x8600u) || !s_more[r & 1]) break;
        }
        for (int c = 0; c < nch; ++c, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&k_empty[s], ((it / STAGES) & 1) ^ 1, &s_abort, hdr, 0x8100u)) {
            ok = false;
            break;
          }
          uint8_t* st = sK + s * CHUNK_BYTES;
          mbar_expect_tx(&k_full[s], CHUNK_BYTES);
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int dc = 0; dc < HALVES; ++dc)
              tma_load_3d(&mapKb, &k_full[s], st + (part * HALVES + dc) * BOX_BYTES, dc * 64,
                          c * NC, part * G.hkv + kv);
        }
      }
      if (!ok) {
        for (int k = 0; k < STAGES; ++k) {
          const int jj = it - 1 - k;
          if (jj < 0) break;
          long long t0 = clock64();
          while (!mbar_try_wait(&k_full[jj % STAGES], (jj / STAGES) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(128, NC);
      const uint32_t q_tmem = tmem_base + Q_COL;
      bool ok = nch == 0 || mbar_wait(q_full, 0, &s_abort, hdr, 0x8200u);
      tc_fence_after();
      int it = 0;
      for (int pass = 0; ok && nch > 0; ++pass) {
        if (pass >= 2) {
          const int r = pass - 2;
          if (!mbar_wait(decide, r & 1, &s_abort, hdr, 0x8700u) || !s_more[r & 1]) break;
        }
        for (int c = 0; c < nch; ++c, ++it) {
          const int s = it % STAGES, sb = it % SBUF;
          if (!mbar_wait(&k_full[s], (it / STAGES) & 1, &s_abort, hdr, 0x8300u) ||
              !mbar_wait(&s_empty[sb], ((it / SBUF) & 1) ^ 1, &s_abort, hdr, 0x8400u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + s * CHUNK_BYTES);
          const uint32_t d = tmem_base + sb * NC;
#pragma unroll
          for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int dc = 0; dc < HALVES; ++dc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = make_sdesc_sw128(
                    k_addr + (part * HALVES + dc) * BOX_BYTES + kk * 32, 16, 1024);
                umma_bf16_ts(d, q_tmem + dc * 32 + kk * 8, bd, idesc,
                             (part | dc | kk) != 0 ? 1u : 0u);
              }
          umma_commit(&s_full[sb]);
          umma_commit(&k_empty[s]);
        }
      }
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ selection rows
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const TileRow R = tile_row(G, false, vt, row);
    const bool valid = R.valid;
    const int t = R.t, h = R.h;
    const int own = valid ? a.cube_ids[t] : -1;
    {
      // query row -> D / 2 TMEM columns of this row's lane (two bf16 per column)
      const __nv_bfloat16* Qg = reinterpret_cast<const __nv_bfloat16*>(a.Q);
      const uint4* src = reinterpret_cast<const uint4*>(Qg + ((size_t)t * G.hq + h) * D);
      const uint32_t qlane = tmem_base + ((uint32_t)(wq * 32) << 16) + Q_COL;
#pragma unroll
      for (int half = 0; half < HALVES; ++half) {
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = valid ? src[half * 8 + c] : make_uint4(0, 0, 0, 0);
          r[4 * c] = v.x;
          r[4 * c + 1] = v.y;
          r[4 * c + 2] = v.z;
          r[4 * c + 3] = v.w;
        }
        tmem_st32(qlane + half * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_full);
    }
    if (c_hi >= 0) {
      sel::RowSel s;
      s.init(ss, row, a.zscale, a.topk > 0);
      const int ncand = own > 0 ? own : 0;
      uint32_t* tmask = a.tile_mask + (size_t)vt * G.n_cubes * 4;
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      int nsel = 0, extra = 0;
      bool ok = true;
      int it = 0;
      for (int pass = 0; nch > 0; ++pass) {
        for (int ch = 0; ch < nch && ok; ++ch, ++it) {
          const int sb = it % SBUF;
          if (!mbar_wait_warp(&s_full[sb], (it / SBUF) & 1, &s_abort, hdr, 0x8500u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int j0 = ch * NC;
          const uint32_t tcol = tmem_base + lane_base + sb * NC;
          // candidates of this row in the chunk: columns [0, nv)
          const int nv = min(max(ncand - j0, 0), NC);
          if (pass == 0) {
            // histogram: the whole chunk in registers, the buffer released at once
            uint32_t acc[NC];
            tmem_ld32(tcol, acc);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&s_empty[sb]);
            if (nv >= NC) {
              // a full chunk: no candidate tests; the maximum as a tree
              auto f = [&](int u) { return __uint_as_float(acc[u]); };
              float mx[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) mx[k] = sel::fmax3(f(k), f(k + 8), f(k + 16));
#pragma unroll
              for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], f(k + 24));
              s.raise(sel::fmax3(sel::fmax3(mx[0], mx[1], mx[2]), sel::fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7])));
              if (!s.range_err) {
#pragma unroll
                for (int c = 0; c < NC; c += 4)
                  s.add_quad(s.mass(f(c)), s.mass(f(c + 1)), s.mass(f(c + 2)), s.mass(f(c + 3)));
              }
            } else if (nv > 0) {
              // the chunk maximum first: the window moves at most once per chunk
              float m = -INFINITY;
#pragma unroll
              for (int c = 0; c < NC; ++c)
                if (c < nv) m = fmaxf(m, __uint_as_float(acc[c]));
              s.raise(m);
              if (!s.range_err) {
#pragma unroll
                for (int c = 0; c < NC; ++c)
                  s.add_score(s.mass(__uint_as_float(acc[c])), c < nv);
              }
            }
            continue;
          }
          // emission (pass 1) and extra passes, 8 columns at a time
          uint32_t bits = 0u;  // bit c: column j0 + c selected outright by this row
#pragma unroll 1
          for (int q = 0; q < NC / 8; ++q) {
            uint32_t acc[8];
            tmem_ld8(tcol + q * 8, acc);
            tmem_ld_wait();
            if (pass == 1) {
              bits |= s.emit8(acc, j0 + q * 8, nv - q * 8) << (q * 8);
            } else if (s.open) {
              uint32_t gb = 0u;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                if (q * 8 + c < nv && s.pass_more(__uint_as_float(acc[c]), j0 + q * 8 + c))
                  gb |= 1u << c;
              bits |= gb << (q * 8);
            }
          }
          tc_fence_before();
          mbar_arrive(&s_empty[sb]);
          if (pass >= 2 && __any_sync(0xffffffffu, bits != 0u)) {
            // fine bins above a row's fine cut: selected outright in the first
            // pass after the fine cut was found
            nsel += __popc(bits);
            const uint32_t word = sel::warp_transpose32(bits, lane);
            const int jl = j0 + lane;
            if (word != 0u && jl < c_hi) atomicOr(&tmask[(size_t)jl * 4 + wq], word);
          }
          if (pass == 1) {
            nsel += __popc(bits);
            // lane L now takes the mask word of column j0 + L (bit r = row r)
            uint32_t word = sel::warp_transpose32(bits, lane);
            // the own cube of each row, for the rows whose own cube is in the chunk
            const int rel = own - j0;
            unsigned pending = __ballot_sync(0xffffffffu, rel >= 0 && rel < NC);
            while (pending) {
              const int o = __shfl_sync(0xffffffffu, rel, __ffs(pending) - 1);
              const unsigned same = __ballot_sync(0xffffffffu, rel == o);
              if (lane == o) word |= same;
              pending &= ~same;
            }
            const int jl = j0 + lane;
            if (jl < c_hi) tmask[(size_t)jl * 4 + wq] = word;
          }
        }
        // Every row warp reaches the vote barrier below, even after a failed
        // wait (the abort flag then ends the loop), so the named barrier
        // cannot strand the other warps.
        if (pass == 0) {
          if (ok) {
            s.finish1(a.topk > 0 ? (float)a.topk : a.p);
            if (s.range_err) set_status(hdr, ADASPARK_DEV_RANGE, 0x8800u);
          }
          continue;
        }
        if (pass == 1) {
          const unsigned w = __ballot_sync(0xffffffffu, own == c_hi);
          if (lane == 0) tmask[(size_t)c_hi * 4 + wq] = w;
          __syncwarp();
          __threadfence_block();
        }
        const bool was_open = s.open;
        const int m = s.settle();
        for (int i = 0; i < m; ++i) atomicOr(&tmask[(size_t)s.list_j(i) * 4 + wq], 1u << lane);
        nsel += m;
        s.reset_list();
        if (was_open && s.open) extra = 1;
        // vote for another pass (round r = pass - 1)
        const int r = pass - 1;
        if (row == 0) s_more[(r + 1) & 1] = 0;
        if (s.open) s_more[r & 1] = 1;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool more = s_more[r & 1] != 0 && !s_abort;
        mbar_arrive(decide);
        if (!more) break;
      }
      if (ok && nch == 0) {
        const unsigned w = __ballot_sync(0xffffffffu, own == c_hi);
        if (lane == 0) tmask[(size_t)c_hi * 4 + wq] = w;
      }
      if (ok) {
        const unsigned v_rows = __reduce_add_sync(0xffffffffu, (valid && own > 0) ? 1u : 0u);
        const unsigned v_cand = __reduce_add_sync(0xffffffffu, (unsigned)ncand);
        const unsigned v_sel = __reduce_add_sync(0xffffffffu, (unsigned)nsel);
        const unsigned v_ext = __reduce_add_sync(0xffffffffu, (unsigned)extra);
        const unsigned v_near = __reduce_add_sync(0xffffffffu, (valid && s.near) ? 1u : 0u);
        if (lane == 0) {
          atomicAdd((unsigned long long*)&hdr->stats[0], (unsigned long long)v_rows);
          atomicAdd((unsigned long long*)&hdr->stats[1], (unsigned long long)v_cand);
          atomicAdd((unsigned long long*)&hdr->stats[2], (unsigned long long)v_sel);
          atomicAdd((unsigned long long*)&hdr->stats[3], (unsigned long long)v_ext);
          if (v_near) atomicAdd((unsigned long long*)&hdr->stats[7], (unsigned long long)v_near);
        }
      }
      __threadfence_block();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!s_bad) {
        const uint16_t* list = a.tile_list + (size_t)vt * G.n_cubes;
        const int n = compact_tile_list(tmask, a.tile_list + (size_t)vt * G.n_cubes,
                                        a.tile_count + vt, c_hi, s_wcnt, row);
        if (a.sp.rows > 0) {
          __threadfence_block();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          // the tile's lowest own cube: that of its first row
          const int c_lo = a.cube_ids[tile_row(G, false, vt, 0).t];
          static_assert(sizeof(sel::Smem) >= kSparseMax * 24, "split staging");
          split_tile(tmask, list, n, a.sp, vt, G.n_cubes, c_lo, kv, t * G.hq + h, valid,
                     reinterpret_cast<uint8_t*>(ss), s_wcnt, s_misc, hdr, row);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace seltc

cudaError_t launch_select_tc(const SelectArgs& a, cudaStream_t s) {
  const AttnGeom& G = a.G;
  if (G.n_vtiles == 0) return cudaSuccess;
  CUtensorMap m;
  const uint64_t dims[3] = {(uint64_t)G.d, (uint64_t)G.n_cubes, (uint64_t)3 * G.hkv};
  const uint64_t strides[2] = {(uint64_t)G.d * 2, (uint64_t)G.n_cubes * G.d * 2};
  const uint32_t box[3] = {64, (uint32_t)seltc::NC, 1};
  if (!encode_tmap_bf16(&m, a.kbar_split, 3, dims, strides, box)) return cudaErrorInvalidValue;
  auto k = G.d == 64 ? seltc::select_tc_kernel<64> : seltc::select_tc_kernel<128>;
  const size_t smem = G.d == 64 ? seltc::smem_bytes<64>() : seltc::smem_bytes<128>();
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch("select_tc", k, dim3(G.n_vtiles), dim3(seltc::THREADS), smem, s, m, a);
}

}  // namespace adaspark

// Backward pass of AdaS-Attn with the cube sets held fixed (straight-through
// selection, for the light fine-tuning the AdaSpark note mentions; key design 2
// differentiated as computed: the cube mean keys and the relevance softmax only
// choose the sets and receive no gradient).
//
// Per row r (token, query head) with admitted keys A_r, logits z = q.k / sqrt(d)
// and P = softmax over A_r (recomputed from the forward's per-row log2-sum-exp):
//   dP_rj = dO_r . v_j,  D_r = dO_r . O_r,  dS_rj = P_rj (dP_rj - D_r)
//   dQ_r  = sum_j dS_rj k_j / sqrt(d)
//   dK_j  = sum_r dS_rj q_r / sqrt(d),  dV_j = sum_r P_rj dO_r
// where the key sums run over every row of every query head of the KV group
// that admits key j.
//
// Two tcgen05 kernels, no atomics:
//   attn_bwd_dq   one CTA per 128-row tile (the forward's tiles, order and
//                 block walk), two passes over the row's key blocks with
//                 S = Q K^T and dP = dO V^T per 64-key block in TMEM: the first
//                 sums D_r = sum_j P_rj dP_rj in fp32 (stored for attn_bwd_dkv),
//                 the second writes dS (bf16) back over S and runs
//                 dQ += dS K with dS read from TMEM (K as an N-major operand).
//                 D from the same fp32 P and dP makes each row's dS sum to zero
//                 up to fp32 rounding; D = dO . O from the bf16 output would
//                 leave a bias of about one bf16 ulp of O, which the near-
//                 cancelling sum behind dQ turns into errors near 4% of its RMS.
//   attn_bwd_dkv  one CTA per (KV head, 64-key block): walks the query tiles
//                 that admit the block (inverted selection lists, then the
//                 text tiles), S and dP as above, P and dS staged in shared
//                 memory, then dV^T += dO^T P and dK^T += Q^T dS with M = 128
//                 over the head dimension (both operands MN-major), so the
//                 block's key and value gradients stay in TMEM until the end.
// Small kernels before them: the inverted lists (per KV head and cube, the
// visual tiles with any row admitting the cube, ascending).
#include <algorithm>

#include "attn_kernels.h"
#include "attn_tile.cuh"

namespace adaspark {
namespace abwd {

constexpr int RING = 64;
constexpr int Q_BYTES = 128 * 256;   // 128 rows x 128 dims bf16 (two 64-dim halves)
constexpr int KB_BYTES = 2 * 8192;   // one 64-key block of K or V (two 64-dim halves)
constexpr int PS_BYTES = 128 * 128;  // 128 rows x 64 keys bf16

struct Desc {
  int k0, nk, j, pass;  // pass: 0 sums D_r, 1 forms dS and dQ
  uint32_t mask[4];
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ small kernels
__global__ void __launch_bounds__(32) check_kernel(WsHeader* hdr, const WsHeader* fhdr) {
  if (threadIdx.x == 0 && fhdr->status != 0u) set_status(hdr, fhdr->status, 0xa100u);
}

// Per (KV head, cube j): the visual tiles of the KV head with any row admitting
// cube j, in ascending tile order. The tiles of a KV head are cut into chunks
// of kInvChunk; thread (kv, j, chunk) counts (fill = 0) or writes (fill = 1)
// its chunk's entries, at the offset of the exclusive prefix over
// (kv, j, chunk) in that order, so each (kv, j) list is contiguous and sorted.
__global__ void __launch_bounds__(128) inv_lists_kernel(AttnBwdArgs a, int fill, int n_chunks) {
  if (status_bad(a.hdr)) return;
  const AttnGeom& G = a.G;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int kv = blockIdx.y / n_chunks, chunk = blockIdx.y - kv * n_chunks;
  if (j >= G.n_cubes) return;
  const bool dense = fwd_was_dense(a.fhdr);
  const size_t key = ((size_t)kv * G.n_cubes + j) * n_chunks + chunk;
  int32_t* out = fill ? a.inv_list + a.inv_start[key] : nullptr;
  int cnt = 0;
  const int tl_end = min((chunk + 1) * kInvChunk, G.vtiles_per_kv);
  for (int tl = chunk * kInvChunk; tl < tl_end; ++tl) {
    const int tt = tl % G.vtiles_per_head;
    const int t_hi = min(tt * kTileRows + kTileRows, G.n_vis) - 1;
    if (j > a.cube_ids[t_hi]) continue;  // cube j follows every row of the tile
    const int bt = kv * G.vtiles_per_kv + tl;
    bool nz = true;
    if (!dense) {
      const uint4 w =
          *reinterpret_cast<const uint4*>(a.tile_mask + ((size_t)bt * G.n_cubes + j) * 4);
      nz = (w.x | w.y | w.z | w.w) != 0u;
    }
    if (nz) {
      if (fill) out[cnt] = bt;
      ++cnt;
    }
  }
  if (!fill) a.inv_count[key] = cnt;
}

// Exclusive prefix of n counts (one block of 1024 threads); start[n] = total.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ cnt,
                                                    int32_t* __restrict__ start, int n,
                                                    WsHeader* hdr) {
  __shared__ int part[1024];
  if (status_bad(hdr)) return;
  const int tid = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int b = min(tid * per, n), e = min(b + per, n);
  int s = 0;
  for (int i = b; i < e; ++i) s += cnt[i];
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = part[tid] - s;
  for (int i = b; i < e; ++i) {
    start[i] = run;
    run += cnt[i];
  }
  if (tid == 1023) start[n] = part[1023];
}

// ------------------------------------------------------------------ dQ kernel
// Warps: 0 TMA producer (K and V blocks), 1 TMEM allocator + MMA issuer,
// 2-5 one thread per row, 6 block-descriptor filler (as in the forward).
// TMEM (512 columns): dQ 0-127, S buffers 128 + 64 b, dP buffers 256 + 64 b.
namespace dq {
constexpr int THREADS = 224;
constexpr int KST = 3, VST = 2;
constexpr size_t SMEM_BYTES =
    1024 + 2 * Q_BYTES + (KST + VST) * KB_BYTES + RING * sizeof(Desc) + 2048;
}  // namespace dq

__global__ void __launch_bounds__(dq::THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, AttnBwdArgs a) {
  using namespace dq;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + Q_BYTES;
  uint8_t* sK = sdO + Q_BYTES;              // [KST][KB_BYTES]
  uint8_t* sV = sK + KST * KB_BYTES;        // [VST][KB_BYTES]
  Desc* ring = reinterpret_cast<Desc*>(sV + VST * KB_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + RING);
  uint64_t* k_full = bars;                  // [KST]
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;         // [VST]
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;         // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* q_full = p_full + 2;
  uint64_t* drain = q_full + 1;
  uint64_t* r_full = drain + 1;             // [RING]
  uint64_t* r_empty = r_full + RING;        // [RING]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(r_empty + RING);
  __shared__ volatile int s_abort;
  __shared__ int s_own_hi, s_bad, s_dense;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  const TileInfo T = decode_tile(G, a.kv_major != 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
    }
    for (int r = 0; r < RING; ++r) {
      mbar_init(&r_full[r], 1);
      mbar_init(&r_empty[r], 128);
    }
    mbar_init(q_full, 128);
    mbar_init(drain, 1);
    fence_mbar_init();
    s_abort = 0;
    s_bad = status_bad(hdr) ? 1 : 0;
    s_own_hi = (!T.text && !s_bad) ? a.cube_ids[T.t_hi] : -1;
    s_dense = fwd_was_dense(a.fhdr) ? 1 : 0;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const bool bad = s_bad != 0;

  if (warp == 6) {
    // ------------------------------------------------------------ descriptor filler
    int n_entries = 0, n_chunks = 0;
    bool use_list = false;
    if (!bad) {
      if (T.text) {
        n_entries = G.n_cubes;
        n_chunks = (T.t_hi - G.n_vis) / 64 + 1;
      } else if (s_dense) {
        n_entries = s_own_hi + 1;
      } else {
        n_entries = a.tile_count[T.bt];
        use_list = true;
      }
    }
    const int n_total = n_entries + n_chunks;
    const uint16_t* list = a.tile_list + (size_t)T.bt * G.n_cubes;
    const uint4* tmask = reinterpret_cast<const uint4*>(a.tile_mask) + (size_t)T.bt * G.n_cubes;
    int base = 0;
    bool ok = true;
    for (int pass = 0; pass < 2; ++pass)
    for (int e0 = 0; e0 < n_total && ok; e0 += 32) {
      const int e = e0 + lane;
      int j = -1, ks = 0, ke = 0;
      uint4 m = make_uint4(~0u, ~0u, ~0u, ~0u);
      if (e < n_entries) {
        j = use_list ? (int)list[e] : e;
        ks = a.cube_offsets[j];
        ke = a.cube_offsets[j + 1];
        if (use_list) m = tmask[j];
      } else if (e < n_total) {
        ks = G.n_vis + (e - n_entries) * 64;
        ke = min(ks + 64, T.t_hi + 1);
      }
      const int nb = (ke - ks + 63) / 64;
      int incl = nb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      int idx = base + incl - nb;
      for (int b = 0; b < nb; ++b, ++idx) {
        const int slot = idx % RING;
        if (!mbar_wait(&r_empty[slot], ((idx / RING) & 1) ^ 1, &s_abort, hdr, 0xa200u)) {
          ok = false;
          break;
        }
        Desc& d = ring[slot];
        d.k0 = ks + 64 * b;
        d.nk = min(64, ke - d.k0);
        d.j = j;
        d.pass = pass;
        d.mask[0] = m.x;
        d.mask[1] = m.y;
        d.mask[2] = m.z;
        d.mask[3] = m.w;
        mbar_arrive(&r_full[slot]);
      }
      ok = __all_sync(0xffffffffu, ok);
      base += total;
    }
    if (ok && lane == 0) {  // terminal descriptor
      const int slot = base % RING;
      if (mbar_wait(&r_empty[slot], ((base / RING) & 1) ^ 1, &s_abort, hdr, 0xa300u)) {
        ring[slot].nk = 0;
        mbar_arrive(&r_full[slot]);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      while (ok) {
        const int slot = i % RING;
        if (!mbar_wait(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0xa400u)) {
          ok = false;
          break;
        }
        const int k0 = ring[slot].k0, nk = ring[slot].nk;
        if (nk == 0) break;
        const int ks = i % KST, vs = i % VST;
        if (!mbar_wait(&k_empty[ks], ((i / KST) & 1) ^ 1, &s_abort, hdr, 0xa410u)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&k_full[ks], KB_BYTES);
        tma_load_3d(&mapK, &k_full[ks], sK + ks * KB_BYTES, 0, T.kv, k0);
        tma_load_3d(&mapK, &k_full[ks], sK + ks * KB_BYTES + 8192, 64, T.kv, k0);
        if (!mbar_wait(&v_empty[vs], ((i / VST) & 1) ^ 1, &s_abort, hdr, 0xa420u)) {
          ok = false;
          ++i;  // K of block i is in flight
          break;
        }
        mbar_expect_tx(&v_full[vs], KB_BYTES);
        tma_load_3d(&mapV, &v_full[vs], sV + vs * KB_BYTES, 0, T.kv, k0);
        tma_load_3d(&mapV, &v_full[vs], sV + vs * KB_BYTES + 8192, 64, T.kv, k0);
        ++i;
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        long long t0 = clock64();
        for (int k = 0; k < KST; ++k) {
          const int jk = i - 1 - k;
          while (jk >= 0 && !mbar_try_wait(&k_full[jk % KST], (jk / KST) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
        for (int k = 0; k < VST; ++k) {
          const int jv = i - 1 - k;
          while (jv >= 0 && !mbar_try_wait(&v_full[jv % VST], (jv / VST) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64);
      constexpr uint32_t idesc_q = make_idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sdO);
      bool ok = mbar_wait(q_full, 0, &s_abort, hdr, 0xa500u);
      tc_fence_after();
      int i = 0, prev_pass = 0;
      bool dq_started = false;
      // block blk: once its rows are done with S / dP, run dQ += dS K (second
      // pass only) and free its K stage
      auto finish = [&](int blk, int pass) -> bool {
        const int pb = blk & 1;
        if (!mbar_wait(&p_full[pb], (blk >> 1) & 1, &s_abort, hdr, 0xa510u)) return false;
        tc_fence_after();
        const int ks = blk % KST;
        if (pass == 1) {
          const uint32_t k_addr = smem_u32(sK + ks * KB_BYTES);
          const uint32_t ds_tmem = tmem_base + 128 + pb * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = make_sdesc_sw128(k_addr + kk * 2048, 8192, 1024);
            umma_bf16_ts(tmem_base, ds_tmem + kk * 8, bd, idesc_q,
                         (dq_started || kk > 0) ? 1u : 0u);
          }
          dq_started = true;
        }
        umma_commit(&k_empty[ks]);
        return true;
      };
      while (ok) {
        const int slot = i % RING;
        if (!mbar_wait(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0xa520u)) {
          ok = false;
          break;
        }
        if (ring[slot].nk == 0) break;
        const int pass = ring[slot].pass;
        const int ks = i % KST, vs = i % VST, sb = i & 1;
        if (!mbar_wait(&k_full[ks], (i / KST) & 1, &s_abort, hdr, 0xa530u) ||
            !mbar_wait(&v_full[vs], (i / VST) & 1, &s_abort, hdr, 0xa540u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + ks * KB_BYTES);
        const uint32_t v_addr = smem_u32(sV + vs * KB_BYTES);
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (dc | kk) != 0 ? 1u : 0u;
            umma_bf16(tmem_base + 128 + sb * 64,
                      make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(k_addr + dc * 8192 + kk * 32, 16, 1024), idesc_s, acc);
            umma_bf16(tmem_base + 256 + sb * 64,
                      make_sdesc_sw128(do_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(v_addr + dc * 8192 + kk * 32, 16, 1024), idesc_s, acc);
          }
        umma_commit(&s_full[sb]);
        umma_commit(&v_empty[vs]);
        if (i > 0 && !finish(i - 1, prev_pass)) {
          ok = false;
          break;
        }
        prev_pass = pass;
        ++i;
      }
      if (ok && i > 0) finish(i - 1, prev_pass);
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const TileRow R = tile_row(G, T.text, T.bt, row);
    const bool valid = R.valid;
    const int t = R.t, h = R.h;
    const int own = (!T.text && valid) ? a.cube_ids[t] : -1;
    const float scale = a.scale_log2;
    const size_t rix = (size_t)t * G.hq + h;
    {
      const uint4* q4 = reinterpret_cast<const uint4*>(a.Q + rix * 128);
      const uint4* d4 = reinterpret_cast<const uint4*>(a.dO + rix * 128);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t off = (c >> 3) * 16384 + sw128_offset(row, c & 7);
        *reinterpret_cast<uint4*>(sQ + off) = valid ? q4[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sdO + off) = valid ? d4[c] : make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
    const float lse2 = valid ? a.lse[rix] : 0.f;
    float dot = 0.f;          // D_r, summed over the first pass
    bool dot_stored = false;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    int i = 0;
    bool ok = true;
    while (true) {
      const int slot = i % RING;
      if (!mbar_wait_warp(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0xa600u)) {
        ok = false;
        break;
      }
      const Desc dsc = ring[slot];
      if (dsc.nk == 0) break;
      const int sb = i & 1;
      if (!mbar_wait_warp(&s_full[sb], (i >> 1) & 1, &s_abort, hdr, 0xa610u)) {
        ok = false;
        break;
      }
      mbar_arrive(&r_empty[slot]);
      tc_fence_after();
      uint32_t sr[64], dp[64];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        uint32_t(&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
        uint32_t(&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[32]);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64, s0);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64 + 32, s1);
        tmem_ld32(tmem_base + lane_base + 256 + sb * 64, p0);
        tmem_ld32(tmem_base + lane_base + 256 + sb * 64 + 32, p1);
      }
      tmem_ld_wait();
      bool row_on;
      if (!valid) row_on = false;
      else if (T.text) row_on = true;
      else if (s_dense) row_on = dsc.j <= own;
      else row_on = ((dsc.mask[wq] >> lane) & 1u) != 0u;
      int lim = row_on ? dsc.nk : 0;
      if (row_on && (T.text || dsc.j == own)) lim = min(lim, t - dsc.k0 + 1);
      if (dsc.pass == 0) {
        float ds[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ds[k] = 0.f;
#pragma unroll
        for (int u = 0; u < 64; ++u) {
          const float pu = u < lim ? ex2(fmaf(__uint_as_float(sr[u]), scale, -lse2)) : 0.f;
          ds[u & 7] = fmaf(pu, __uint_as_float(dp[u]), ds[u & 7]);
        }
        dot += ((ds[0] + ds[1]) + (ds[2] + ds[3])) + ((ds[4] + ds[5]) + (ds[6] + ds[7]));
      } else {
        if (!dot_stored) {
          if (valid) a.dot[rix] = dot;
          dot_stored = true;
        }
        uint32_t pk[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int u = 2 * q;
          const float p0 = u < lim ? ex2(fmaf(__uint_as_float(sr[u]), scale, -lse2)) : 0.f;
          const float p1 =
              u + 1 < lim ? ex2(fmaf(__uint_as_float(sr[u + 1]), scale, -lse2)) : 0.f;
          pk[q] = pack_bf16x2(p0 * (__uint_as_float(dp[u]) - dot),
                              p1 * (__uint_as_float(dp[u + 1]) - dot));
        }
        tmem_st32(tmem_base + lane_base + 128 + sb * 64, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
      ++i;
    }
    if (ok && !dot_stored && valid) a.dot[rix] = dot;
    long long t0 = clock64();
    bool done = ok;
    if (ok && i > 0) {
      done = false;
      while (!(done = mbar_try_wait(drain, 0)) && clock64() - t0 < kWaitCycles) {
      }
      if (!done) set_status(hdr, ADASPARK_DEV_TIMEOUT, 0xa620u);
    }
    done = __all_sync(0xffffffffu, done);
    if (done) {
      tc_fence_after();
      float* dst = a.dQ + rix * 128;
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_base + c, o);
        tmem_ld_wait();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
          const float s = a.inv_sqrt_d;
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = i > 0 ? make_float4(__uint_as_float(o[4 * x]) * s,
                                        __uint_as_float(o[4 * x + 1]) * s,
                                        __uint_as_float(o[4 * x + 2]) * s,
                                        __uint_as_float(o[4 * x + 3]) * s)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ dK / dV kernel
// One CTA per (KV head, 64-key block). Block units per KV head: four per cube
// (pieces of up to 64 keys; cubes hold at most 256 tokens; absent pieces exit),
// then the 64-key pieces of the text suffix. Warps: 0 TMA producer, 1 TMEM
// allocator + MMA issuer, 2-5 one thread per query row, then per head dimension
// in the epilogue. TMEM (512 columns): S buffers 64 b, dP buffers 128 + 64 b,
// dV^T 256-319, dK^T 320-383 (lane = head dimension, column = key).
namespace dkv {
constexpr int THREADS = 192;
constexpr int QST = 2;
constexpr size_t SMEM_BYTES = 1024 + 2 * KB_BYTES + QST * 2 * Q_BYTES + 2 * PS_BYTES + 1024;
}  // namespace dkv

struct KeyBlock {
  bool ok;        // the block exists
  bool visual;    // keys of a visual cube (else of the text suffix)
  int kv, j, k0, nk;
  int n_vis_entries, tt_min, n_text_entries;
};

__device__ __forceinline__ KeyBlock decode_key_block(const AttnBwdArgs& a) {
  const AttnGeom& G = a.G;
  const int n_text = G.n_tokens - G.n_vis;
  const int units = 4 * G.n_cubes + (n_text + 63) / 64;
  KeyBlock B;
  B.kv = blockIdx.x / units;
  const int u = blockIdx.x - B.kv * units;
  B.ok = true;
  if (u < 4 * G.n_cubes) {
    B.visual = true;
    B.j = u >> 2;
    const int ke = a.cube_offsets[B.j + 1];
    B.k0 = a.cube_offsets[B.j] + 64 * (u & 3);
    B.ok = B.k0 < ke;
    B.nk = min(64, ke - B.k0);
    const size_t key = ((size_t)B.kv * G.n_cubes + B.j) * a.inv_chunks;
    B.n_vis_entries = B.ok ? a.inv_start[key + a.inv_chunks] - a.inv_start[key] : 0;
    B.tt_min = 0;
  } else {
    B.visual = false;
    B.j = -1;
    B.k0 = G.n_vis + 64 * (u - 4 * G.n_cubes);
    B.nk = min(64, G.n_tokens - B.k0);
    B.n_vis_entries = 0;
    B.tt_min = (B.k0 - G.n_vis) / kTileRows;  // text tiles before it end before k0
  }
  B.n_text_entries = G.g * (G.ttiles_per_head - B.tt_min);
  return B;
}

// Entry e of a key block's walk: (text tile?, tile index within its kind).
__device__ __forceinline__ void walk_entry(const AttnBwdArgs& a, const KeyBlock& B,
                                           const int32_t* list, int e, bool& text, int& bt) {
  const AttnGeom& G = a.G;
  if (e < B.n_vis_entries) {
    text = false;
    bt = list[e];
  } else {
    const int e2 = e - B.n_vis_entries;
    const int nt = G.ttiles_per_head - B.tt_min;
    const int hh = e2 / nt, tt = B.tt_min + e2 % nt;
    text = true;
    bt = B.kv * G.ttiles_per_kv + hh * G.ttiles_per_head + tt;
  }
}

__global__ void __launch_bounds__(dkv::THREADS, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap mapQ,
                        const __grid_constant__ CUtensorMap mapdO,
                        const __grid_constant__ CUtensorMap mapK,
                        const __grid_constant__ CUtensorMap mapV, AttnBwdArgs a) {
  using namespace dkv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;                       // K block, then V block
  uint8_t* sV = sK + KB_BYTES;
  uint8_t* sQd = sV + KB_BYTES;             // [QST][Q tile | dO tile]
  uint8_t* sP = sQd + QST * 2 * Q_BYTES;
  uint8_t* sdS = sP + PS_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + PS_BYTES);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = kv_full + 1;          // [QST]
  uint64_t* qd_empty = qd_full + QST;       // [QST]
  uint64_t* s_full = qd_empty + QST;        // [2]
  uint64_t* ps_full = s_full + 2;
  uint64_t* ps_empty = ps_full + 1;
  uint64_t* done = ps_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ volatile int s_abort;

  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  if (status_bad(hdr)) return;              // uniform: before any barrier or TMEM
  const KeyBlock B = decode_key_block(a);
  if (!B.ok) return;
  const int n_entries = B.n_vis_entries + B.n_text_entries;
  const int32_t* list =
      a.inv_list + (B.visual ? a.inv_start[((size_t)B.kv * G.n_cubes + B.j) * a.inv_chunks] : 0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&s_full[b], 1);
    mbar_init(ps_full, 128);
    mbar_init(ps_empty, 1);
    mbar_init(done, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapdO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * KB_BYTES);
      tma_load_3d(&mapK, kv_full, sK, 0, B.kv, B.k0);
      tma_load_3d(&mapK, kv_full, sK + 8192, 64, B.kv, B.k0);
      tma_load_3d(&mapV, kv_full, sV, 0, B.kv, B.k0);
      tma_load_3d(&mapV, kv_full, sV + 8192, 64, B.kv, B.k0);
      int e = 0;
      bool ok = true;
      for (; e < n_entries; ++e) {
        const int st = e % QST;
        if (!mbar_wait(&qd_empty[st], ((e / QST) & 1) ^ 1, &s_abort, hdr, 0xa700u)) {
          ok = false;
          break;
        }
        bool text;
        int bt;
        walk_entry(a, B, list, e, text, bt);
        const TileRow R0 = tile_row(G, text, bt, 0);
        uint8_t* q = sQd + st * 2 * Q_BYTES;
        mbar_expect_tx(&qd_full[st], 2 * Q_BYTES);
        tma_load_3d(&mapQ, &qd_full[st], q, 0, R0.h, R0.t);
        tma_load_3d(&mapQ, &qd_full[st], q + 16384, 64, R0.h, R0.t);
        tma_load_3d(&mapdO, &qd_full[st], q + Q_BYTES, 0, R0.h, R0.t);
        tma_load_3d(&mapdO, &qd_full[st], q + Q_BYTES + 16384, 64, R0.h, R0.t);
      }
      // let copies in flight land before the CTA can exit
      long long t0 = clock64();
      while (!mbar_try_wait(kv_full, 0) && clock64() - t0 < kWaitCycles) {
      }
      if (!ok) {
        for (int k = 0; k < QST; ++k) {
          const int je = e - 1 - k;
          while (je >= 0 && !mbar_try_wait(&qd_full[je % QST], (je / QST) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64);
      constexpr uint32_t idesc_g = make_idesc_bf16_mn(128, 64);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(sP), ds_addr = smem_u32(sdS);
      bool ok = mbar_wait(kv_full, 0, &s_abort, hdr, 0xa710u);
      tc_fence_after();
      auto issue_grad = [&](int f) -> bool {
        if (!mbar_wait(ps_full, f & 1, &s_abort, hdr, 0xa720u)) return false;
        tc_fence_after();
        const int st = f % QST;
        const uint32_t q_addr = smem_u32(sQd + st * 2 * Q_BYTES);
        const uint32_t do_addr = q_addr + Q_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (f > 0 || kk > 0) ? 1u : 0u;
          // dV^T[d][key] += dO^T[d][row] P[row][key]
          umma_bf16(tmem_base + 256, make_sdesc_sw128(do_addr + kk * 2048, 16384, 1024),
                    make_sdesc_sw128(p_addr + kk * 2048, 8192, 1024), idesc_g, acc);
          // dK^T[d][key] += Q^T[d][row] dS[row][key]
          umma_bf16(tmem_base + 320, make_sdesc_sw128(q_addr + kk * 2048, 16384, 1024),
                    make_sdesc_sw128(ds_addr + kk * 2048, 8192, 1024), idesc_g, acc);
        }
        umma_commit(ps_empty);
        umma_commit(&qd_empty[st]);
        return true;
      };
      int e = 0;
      for (; e < n_entries && ok; ++e) {
        const int st = e % QST, sb = e & 1;
        if (!mbar_wait(&qd_full[st], (e / QST) & 1, &s_abort, hdr, 0xa730u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQd + st * 2 * Q_BYTES);
        const uint32_t do_addr = q_addr + Q_BYTES;
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (dc | kk) != 0 ? 1u : 0u;
            umma_bf16(tmem_base + sb * 64, make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(k_addr + dc * 8192 + kk * 32, 16, 1024), idesc_s, acc);
            umma_bf16(tmem_base + 128 + sb * 64,
                      make_sdesc_sw128(do_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(v_addr + dc * 8192 + kk * 32, 16, 1024), idesc_s, acc);
          }
        umma_commit(&s_full[sb]);
        if (e > 0 && !issue_grad(e - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n_entries > 0) ok = issue_grad(n_entries - 1);
      umma_commit(done);
      long long t0 = clock64();
      while (!mbar_try_wait(done, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float scale = a.scale_log2;
    const bool dense = fwd_was_dense(a.fhdr);
    // Per-row data of an entry (log2-sum-exp, D, own cube, mask word) comes from
    // global memory behind the entry's list value. The loads are software-
    // pipelined: entry e + 2's list value and entry e + 1's row data are
    // requested during entry e, so their latency overlaps its MMAs.
    struct RowData {
      float lse2, dot;
      int t, own;
      uint32_t w;
      bool valid, text;
    };
    auto request = [&](bool text, int bt) {
      RowData r;
      const TileRow R = tile_row(G, text, bt, row);
      const size_t rix = (size_t)R.t * G.hq + R.h;
      r.t = R.t;
      r.valid = R.valid;
      r.text = text;
      r.lse2 = R.valid ? a.lse[rix] : 0.f;
      r.dot = R.valid ? a.dot[rix] : 0.f;
      r.own = (!text && R.valid) ? a.cube_ids[R.t] : -1;
      r.w = (B.visual && !text && !dense)
                ? a.tile_mask[((size_t)bt * G.n_cubes + B.j) * 4 + wq]
                : 0u;
      return r;
    };
    bool text_n = false, text_nn = false;
    int bt_n = 0, bt_nn = 0;
    RowData cur{}, nxt{};
    if (n_entries > 0) {
      walk_entry(a, B, list, 0, text_n, bt_n);
      cur = request(text_n, bt_n);
    }
    if (n_entries > 1) walk_entry(a, B, list, 1, text_n, bt_n);
    bool ok = true;
    for (int e = 0; e < n_entries; ++e) {
      if (e + 1 < n_entries) nxt = request(text_n, bt_n);
      if (e + 2 < n_entries) walk_entry(a, B, list, e + 2, text_nn, bt_nn);
      const float lse2 = cur.lse2, dot = cur.dot;
      bool row_on = cur.valid;
      int lim = B.nk;
      if (B.visual) {
        if (!cur.text && cur.valid) {
          row_on = dense ? B.j <= cur.own : ((cur.w >> lane) & 1u) != 0u;
          if (B.j == cur.own) lim = min(lim, cur.t - B.k0 + 1);
        }
      } else {
        lim = min(lim, cur.t - B.k0 + 1);
      }
      if (lim <= 0) row_on = false;
      if (!row_on) lim = 0;
      cur = nxt;
      text_n = text_nn;
      bt_n = bt_nn;
      const int sb = e & 1;
      if (!mbar_wait_warp(&s_full[sb], (e >> 1) & 1, &s_abort, hdr, 0xa740u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64], dp[64];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        uint32_t(&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
        uint32_t(&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[32]);
        tmem_ld32(tmem_base + lane_base + sb * 64, s0);
        tmem_ld32(tmem_base + lane_base + sb * 64 + 32, s1);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64, p0);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64 + 32, p1);
      }
      tmem_ld_wait();
      uint32_t pp[32], pd[32];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const int u = 2 * q;
        const float p0 = u < lim ? ex2(fmaf(__uint_as_float(sr[u]), scale, -lse2)) : 0.f;
        const float p1 = u + 1 < lim ? ex2(fmaf(__uint_as_float(sr[u + 1]), scale, -lse2)) : 0.f;
        pp[q] = pack_bf16x2(p0, p1);
        pd[q] = pack_bf16x2(p0 * (__uint_as_float(dp[u]) - dot),
                            p1 * (__uint_as_float(dp[u + 1]) - dot));
      }
      // the gradient MMAs of the previous entry have finished reading sP / sdS
      if (e > 0 && !mbar_wait_warp(ps_empty, (e - 1) & 1, &s_abort, hdr, 0xa750u)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t off = sw128_offset(row, c);
        *reinterpret_cast<uint4*>(sP + off) =
            make_uint4(pp[4 * c], pp[4 * c + 1], pp[4 * c + 2], pp[4 * c + 3]);
        *reinterpret_cast<uint4*>(sdS + off) =
            make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ps_full);
    }
    // epilogue: thread = head dimension d, 64 keys of dV^T and dK^T
    long long t0 = clock64();
    bool fin = ok;
    if (ok && n_entries > 0) {
      fin = false;
      while (!(fin = mbar_try_wait(done, 0)) && clock64() - t0 < kWaitCycles) {
      }
      if (!fin) set_status(hdr, ADASPARK_DEV_TIMEOUT, 0xa760u);
    }
    fin = __all_sync(0xffffffffu, fin);
    if (fin) {
      tc_fence_after();
      const int d = row;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        uint32_t v[32], k[32];
        tmem_ld32(tmem_base + lane_base + 256 + c, v);
        tmem_ld32(tmem_base + lane_base + 320 + c, k);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int key = c + x;
          if (key < B.nk) {
            const size_t o = ((size_t)(B.k0 + key) * G.hkv + B.kv) * 128 + d;
            a.dV[o] = n_entries > 0 ? __uint_as_float(v[x]) : 0.f;
            a.dK[o] = n_entries > 0 ? __uint_as_float(k[x]) * a.inv_sqrt_d : 0.f;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace abwd

cudaError_t launch_attn_backward_tc(const AttnBwdArgs& a, cudaStream_t s) {
  using namespace abwd;
  const AttnGeom& G = a.G;
  cudaError_t e;
  if ((e = launch("attn_bwd_check", check_kernel, dim3(1), dim3(32), 0, s, a.hdr, a.fhdr)))
    return e;
  if (G.n_cubes > 0) {
    const int nc = a.inv_chunks;
    const dim3 g((G.n_cubes + 127) / 128, G.hkv * nc);
    if ((e = launch("attn_bwd_inv_count", inv_lists_kernel, g, dim3(128), 0, s, a, 0, nc)))
      return e;
    if ((e = launch("attn_bwd_scan", scan_kernel, dim3(1), dim3(1024), 0, s, a.inv_count,
                    a.inv_start, G.hkv * G.n_cubes * nc, a.hdr)))
      return e;
    if ((e = launch("attn_bwd_inv_fill", inv_lists_kernel, g, dim3(128), 0, s, a, 1, nc)))
      return e;
  }
  CUtensorMap mQ, mdO, mK, mV;
  const uint64_t qdims[3] = {(uint64_t)G.d, (uint64_t)G.hq, (uint64_t)G.n_tokens};
  const uint64_t qstr[2] = {(uint64_t)G.d * 2, (uint64_t)G.hq * G.d * 2};
  const uint32_t qbox[3] = {64, 1, 128};
  const uint64_t kdims[3] = {(uint64_t)G.d, (uint64_t)G.hkv, (uint64_t)G.n_tokens};
  const uint64_t kstr[2] = {(uint64_t)G.d * 2, (uint64_t)G.hkv * G.d * 2};
  const uint32_t kbox[3] = {64, 1, 64};
  if (!encode_tmap_bf16(&mQ, a.Q, 3, qdims, qstr, qbox) ||
      !encode_tmap_bf16(&mdO, a.dO, 3, qdims, qstr, qbox) ||
      !encode_tmap_bf16(&mK, a.K, 3, kdims, kstr, kbox) ||
      !encode_tmap_bf16(&mV, a.V, 3, kdims, kstr, kbox))
    return cudaErrorInvalidValue;
  const int tiles = G.n_vtiles + G.n_ttiles;
  if (tiles > 0) {
    auto k = attn_bwd_dq_kernel;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dq::SMEM_BYTES)))
      return e;
    if ((e = launch("attn_bwd_dq_tc", k, dim3(tiles), dim3(dq::THREADS), dq::SMEM_BYTES, s, mK, mV,
                    a)))
      return e;
  }
  const int units = 4 * G.n_cubes + (G.n_tokens - G.n_vis + 63) / 64;
  if (units > 0) {
    auto k = attn_bwd_dkv_kernel;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dkv::SMEM_BYTES)))
      return e;
    if ((e = launch("attn_bwd_dkv_tc", k, dim3(units * G.hkv), dim3(dkv::THREADS),
                    dkv::SMEM_BYTES, s, mQ, mdO, mK, mV, a)))
      return e;
  }
  return cudaSuccess;
}

}  // namespace adaspark

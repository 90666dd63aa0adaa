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
//                 block walk), the walk's 64-key blocks two at a time:
//                 S = Q [K_a; K_b]^T and dP = dO [V_a; V_b]^T (N = 128) into
//                 TMEM, dS (bf16) written back over S, dQ += dS [K_a; K_b]
//                 (K = 128) with dS read from TMEM. D_r must agree with the
//                 recomputed fp32 P: after a training-mode forward it is
//                 dO . O from that call's fp32 output (dot_kernel); otherwise a
//                 first walk sums D_r = sum_j P_rj dP_rj (stored for
//                 attn_bwd_dkv). D = dO . O from the bf16 output would leave a
//                 bias of about one bf16 ulp of O, which the near-cancelling
//                 sum behind dQ turns into errors near 4% of its RMS.
//   attn_bwd_dkv  transposed: one CTA per (KV head, pair of 64-key pieces),
//                 walking the query tiles that admit either piece (the union of
//                 the two cubes' inverted lists, then the text tiles):
//                 S^T = K Q^T and dP^T = V dO^T with M = 128 keys, one thread
//                 per key forming P^T and dS^T in TMEM, dV += P^T dO and
//                 dK += dS^T Q with P^T / dS^T read from TMEM, so the pair's key
//                 and value gradients stay in TMEM until the end.
// Small kernels before them: D_r (training-mode forward only), the inverted
// lists (per KV head and cube, the visual tiles with any row admitting the
// cube, ascending) and the table of key pieces.
#include <algorithm>

#include "attn_kernels.h"
#include "attn_tile.cuh"

namespace adaspark {
namespace abwd {

constexpr int RING = 64;
constexpr int Q_BYTES = 128 * 256;   // 128 rows x 128 dims bf16 (two 64-dim halves)

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

// D_r = dO_r . O_r from the fp32 O of a training-mode forward (one warp per
// row); nothing to do otherwise (the dQ kernel then sums D_r in a first pass).
__global__ void __launch_bounds__(256) dot_kernel(AttnBwdArgs a) {
  if (status_bad(a.hdr) || !fwd_was_train(a.fhdr)) return;
  const int rows = a.G.n_tokens * a.G.hq;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint2 g = reinterpret_cast<const uint2*>(a.dO + (size_t)r * 128)[lane];
  const float4 o = reinterpret_cast<const float4*>(a.o32 + (size_t)r * 128)[lane];
  const __nv_bfloat162* gb = reinterpret_cast<const __nv_bfloat162*>(&g);
  const float2 g0 = __bfloat1622float2(gb[0]), g1 = __bfloat1622float2(gb[1]);
  float s = g0.x * o.x;
  s = fmaf(g0.y, o.y, s);
  s = fmaf(g1.x, o.z, s);
  s = fmaf(g1.y, o.w, s);
  s = warp_sum(s);
  if (lane == 0) a.dot[r] = s;
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
// One CTA per 128-row tile (the forward's tiles, order and block walk). The
// tile's 64-key blocks are taken two at a time (consecutive blocks of its own
// walk, so no block is added): per pair S = Q [K_a; K_b]^T and dP = dO
// [V_a; V_b]^T are N = 128 products into TMEM and dQ += dS [K_a; K_b] a K = 128
// product with dS read from TMEM. Two passes over the walk: the first sums
// D_r = sum_j P_rj dP_rj, the second forms dS and dQ.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2-9 row threads (two
// warps per TMEM lane quadrant, one thread per (row, half of the pair's 128
// keys)), 10 block-descriptor filler. TMEM (512 columns): dQ 0-127, S buffers
// 128-255 and 384-511 (pair m in buffer m % 2, so the next pair's S runs
// while the row threads work on this one), dP 256-383.
namespace dq {
constexpr int THREADS = 352;
constexpr int ROW_THREADS = 256;
constexpr int FILLER_WARP = 10;
constexpr int KST = 2, VST = 1;           // stages of 128-key K and V pairs
constexpr int KP_BYTES = 2 * 16384;       // 128 keys x 128 dims bf16
constexpr uint32_t COL_DP = 256;
__device__ __forceinline__ uint32_t col_s(int m) { return (m & 1) ? 384u : 128u; }
constexpr size_t SMEM_BYTES =
    1024 + 2 * Q_BYTES + (KST + VST) * KP_BYTES + RING * sizeof(Desc) + 2048;
}  // namespace dq

// Desc.pass bits: 0 = pass, 1 = pad (empty block that evens a pass), 2 = end.
constexpr int kDescPad = 2, kDescEnd = 4;

__global__ void __launch_bounds__(dq::THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, AttnBwdArgs a) {
  using namespace dq;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + Q_BYTES;
  uint8_t* sK = sdO + Q_BYTES;              // [KST][KP_BYTES]
  uint8_t* sV = sK + KST * KP_BYTES;        // [VST][KP_BYTES]
  Desc* ring = reinterpret_cast<Desc*>(sV + VST * KP_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + RING);
  uint64_t* k_full = bars;                  // [KST]
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;         // [VST]
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;         // [2]
  uint64_t* dp_full = s_full + 2;
  uint64_t* ds_ready = dp_full + 1;         // row threads done with the pair
  uint64_t* q_full = ds_ready + 1;
  uint64_t* drain = q_full + 1;
  uint64_t* xch = drain + 1;                // halves of D_r exchanged
  uint64_t* r_full = xch + 1;               // [RING]
  uint64_t* r_empty = r_full + RING;        // [RING]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(r_empty + RING);
  __shared__ volatile int s_abort;
  __shared__ int s_own_hi, s_bad, s_dense, s_train;
  __shared__ float s_dpart[2][128];

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
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_ready, ROW_THREADS);
    for (int r = 0; r < RING; ++r) {
      mbar_init(&r_full[r], 1);
      mbar_init(&r_empty[r], ROW_THREADS);
    }
    mbar_init(q_full, ROW_THREADS);
    mbar_init(drain, 1);
    mbar_init(xch, ROW_THREADS);
    fence_mbar_init();
    s_abort = 0;
    s_bad = status_bad(hdr) ? 1 : 0;
    s_own_hi = (!T.text && !s_bad) ? a.cube_ids[T.t_hi] : -1;
    s_dense = fwd_was_dense(a.fhdr) ? 1 : 0;
    s_train = fwd_was_train(a.fhdr) ? 1 : 0;
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

  if (warp == FILLER_WARP) {
    // ------------------------------------------------------------ descriptor filler
    // Both passes over the tile's blocks; a pass with an odd number of blocks
    // gets a pad block, so pairs never straddle passes; then an end marker.
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
    auto put = [&](int idx, int k0, int nk, int j, int flags, uint4 m) -> bool {
      const int slot = idx % RING;
      if (!mbar_wait(&r_empty[slot], ((idx / RING) & 1) ^ 1, &s_abort, hdr, 0xa200u))
        return false;
      Desc& d = ring[slot];
      d.k0 = k0;
      d.nk = nk;
      d.j = j;
      d.pass = flags;
      d.mask[0] = m.x;
      d.mask[1] = m.y;
      d.mask[2] = m.z;
      d.mask[3] = m.w;
      mbar_arrive(&r_full[slot]);
      return true;
    };
    // a training-mode forward left D_r already: the second pass alone
    for (int pass = s_train ? 1 : 0; pass < 2 && ok; ++pass) {
      const int pass_begin = base;
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
        for (int b = 0; b < nb && ok; ++b, ++idx)
          ok = put(idx, ks + 64 * b, min(64, ke - ks - 64 * b), j, pass, m);
        ok = __all_sync(0xffffffffu, ok);
        base += total;
      }
      if (ok && ((base - pass_begin) & 1)) {  // even the pass
        if (lane == 0) ok = put(base, 0, 0, -1, pass | kDescPad, make_uint4(0, 0, 0, 0));
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        ++base;
      }
    }
    if (ok && lane == 0) {  // end marker (both slots of a pair)
      put(base, 0, 0, -1, kDescEnd, make_uint4(0, 0, 0, 0));
      put(base + 1, 0, 0, -1, kDescEnd, make_uint4(0, 0, 0, 0));
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Pair m = blocks 2m and 2m + 1: K into keys 0-63 / 64-127 of a K stage,
    // V likewise. A pad block loads the first block again (K enters the dQ
    // product as a reduction operand, so its rows must hold finite values).
    if (lane == 0) {
      int m = 0;
      bool ok = true;
      while (ok) {
        const int sa = (2 * m) % RING, sb2 = (2 * m + 1) % RING;
        if (!mbar_wait(&r_full[sa], ((2 * m) / RING) & 1, &s_abort, hdr, 0xa400u) ||
            !mbar_wait(&r_full[sb2], ((2 * m + 1) / RING) & 1, &s_abort, hdr, 0xa401u)) {
          ok = false;
          break;
        }
        const Desc da = ring[sa], db = ring[sb2];
        if (da.pass & kDescEnd) break;
        const int k0a = da.k0, k0b = db.nk > 0 ? db.k0 : da.k0;
        const int ks = m % KST, vs = m % VST;
        if (!mbar_wait(&k_empty[ks], ((m / KST) & 1) ^ 1, &s_abort, hdr, 0xa410u)) {
          ok = false;
          break;
        }
        uint8_t* kd = sK + ks * KP_BYTES;
        mbar_expect_tx(&k_full[ks], KP_BYTES);
        tma_load_3d(&mapK, &k_full[ks], kd, 0, T.kv, k0a);
        tma_load_3d(&mapK, &k_full[ks], kd + 16384, 64, T.kv, k0a);
        tma_load_3d(&mapK, &k_full[ks], kd + 8192, 0, T.kv, k0b);
        tma_load_3d(&mapK, &k_full[ks], kd + 16384 + 8192, 64, T.kv, k0b);
        if (!mbar_wait(&v_empty[vs], ((m / VST) & 1) ^ 1, &s_abort, hdr, 0xa420u)) {
          ok = false;
          ++m;  // K of pair m is in flight
          break;
        }
        uint8_t* vd = sV + vs * KP_BYTES;
        mbar_expect_tx(&v_full[vs], KP_BYTES);
        tma_load_3d(&mapV, &v_full[vs], vd, 0, T.kv, k0a);
        tma_load_3d(&mapV, &v_full[vs], vd + 16384, 64, T.kv, k0a);
        tma_load_3d(&mapV, &v_full[vs], vd + 8192, 0, T.kv, k0b);
        tma_load_3d(&mapV, &v_full[vs], vd + 16384 + 8192, 64, T.kv, k0b);
        ++m;
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        long long t0 = clock64();
        for (int k = 0; k < KST; ++k) {
          const int jk = m - 1 - k;
          while (jk >= 0 && !mbar_try_wait(&k_full[jk % KST], (jk / KST) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
        for (int k = 0; k < VST; ++k) {
          const int jv = m - 1 - k;
          while (jv >= 0 && !mbar_try_wait(&v_full[jv % VST], (jv / VST) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128);
      constexpr uint32_t idesc_q = make_idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sdO);
      bool ok = mbar_wait(q_full, 0, &s_abort, hdr, 0xa500u);
      tc_fence_after();
      bool dq_started = false;
      int prev_flags = 0;
      // pair m - 1's rows are done: its dQ product (second pass), then its K
      // stage is free
      auto finish = [&](int pm, int flags) -> bool {
        if (!mbar_wait(ds_ready, pm & 1, &s_abort, hdr, 0xa510u)) return false;
        tc_fence_after();
        const int ks = pm % KST;
        if (flags & 1) {
          const uint32_t k_addr = smem_u32(sK + ks * KP_BYTES);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = make_sdesc_sw128(k_addr + kk * 2048, 16384, 1024);
            umma_bf16_ts(tmem_base, tmem_base + col_s(pm) + (kk >> 2) * 64 + (kk & 3) * 8, bd,
                         idesc_q, (dq_started || kk > 0) ? 1u : 0u);
          }
          dq_started = true;
        }
        umma_commit(&k_empty[ks]);
        return true;
      };
      int m = 0;
      for (; ok; ++m) {
        const int sa = (2 * m) % RING;
        if (!mbar_wait(&r_full[sa], ((2 * m) / RING) & 1, &s_abort, hdr, 0xa520u)) {
          ok = false;
          break;
        }
        const int flags = ring[sa].pass;
        if (flags & kDescEnd) break;
        const int ks = m % KST, vs = m % VST;
        if (!mbar_wait(&k_full[ks], (m / KST) & 1, &s_abort, hdr, 0xa530u) ||
            !mbar_wait(&v_full[vs], (m / VST) & 1, &s_abort, hdr, 0xa540u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + ks * KP_BYTES);
        const uint32_t v_addr = smem_u32(sV + vs * KP_BYTES);
        // S of pair m into its buffer (the buffer's last reader, pair m - 2's
        // dQ product, was issued before)
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base + col_s(m),
                      make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(k_addr + dc * 16384 + kk * 32, 16, 1024), idesc_s,
                      (dc | kk) != 0 ? 1u : 0u);
        umma_commit(&s_full[m & 1]);
        // dP has one buffer: pair m - 1's rows must be done with it first
        if (m > 0 && !finish(m - 1, prev_flags)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base + COL_DP,
                      make_sdesc_sw128(do_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(v_addr + dc * 16384 + kk * 32, 16, 1024), idesc_s,
                      (dc | kk) != 0 ? 1u : 0u);
        umma_commit(dp_full);
        umma_commit(&v_empty[vs]);
        prev_flags = flags;
      }
      if (ok && m > 0) finish(m - 1, prev_flags);
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int half = (warp - 2) >> 2;         // the pair's block: keys [64 half, +64)
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
      for (int c = half * 8; c < half * 8 + 8; ++c) {
        const uint32_t off = (c >> 3) * 16384 + sw128_offset(row, c & 7);
        *reinterpret_cast<uint4*>(sQ + off) = valid ? q4[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sdO + off) = valid ? d4[c] : make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
    const float lse2 = valid ? a.lse[rix] : 0.f;
    // this half's part of D_r over the first pass, or D_r from the training
    // forward's fp32 O
    const bool have_dot = s_train != 0;
    float dot = have_dot && valid ? a.dot[rix] : 0.f;
    bool dot_done = have_dot;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    int m = 0;
    bool ok = true;
    while (true) {
      const int sa = (2 * m) % RING;
      const int sme = (2 * m + half) % RING;  // this half's block
      if (!mbar_wait_warp(&r_full[sa], ((2 * m) / RING) & 1, &s_abort, hdr, 0xa600u) ||
          !mbar_wait_warp(&r_full[(2 * m + 1) % RING], ((2 * m + 1) / RING) & 1, &s_abort, hdr,
                          0xa601u)) {
        ok = false;
        break;
      }
      const int flags = ring[sa].pass;
      if (flags & kDescEnd) break;
      const Desc dsc = ring[sme];
      if (!mbar_wait_warp(&s_full[m & 1], (m >> 1) & 1, &s_abort, hdr, 0xa610u)) {
        ok = false;
        break;
      }
      // S of the pair landed: the producer and the MMA issuer are done with
      // both descriptors
      mbar_arrive(&r_empty[sa]);
      mbar_arrive(&r_empty[(2 * m + 1) % RING]);
      tc_fence_after();
      bool row_on;
      if (!valid || dsc.nk <= 0) row_on = false;
      else if (T.text) row_on = true;
      else if (s_dense) row_on = dsc.j <= own;
      else row_on = ((dsc.mask[wq] >> lane) & 1u) != 0u;
      int lim = row_on ? dsc.nk : 0;
      if (row_on && (T.text || dsc.j == own)) lim = min(lim, t - dsc.k0 + 1);
      if (lim < 0) lim = 0;
      const bool pass1 = (flags & 1) != 0;
      if (pass1 && !dot_done) {
        // D_r = the two halves' sums, exchanged once through shared memory
        s_dpart[half][row] = dot;
        mbar_arrive(xch);
        if (!mbar_wait_warp(xch, 0, &s_abort, hdr, 0xa630u)) {
          ok = false;
          break;
        }
        dot = s_dpart[0][row] + s_dpart[1][row];
        if (valid && half == 0) a.dot[rix] = dot;
        dot_done = true;
      }
      if (!__any_sync(0xffffffffu, lim > 0)) {
        // No row of this warp takes a key of its block: P = 0, so its dS is
        // zero (and its part of D_r in the first pass adds nothing); dS = 0
        // goes over the scores without reading S or dP. The dP barrier is
        // still waited on, which keeps its phase count.
        if (!mbar_wait_warp(dp_full, m & 1, &s_abort, hdr, 0xa616u)) {
          ok = false;
          break;
        }
        if (pass1) {
          uint32_t zero[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) zero[q] = 0u;
          tmem_st16(tmem_base + lane_base + col_s(m) + half * 64, zero);
          tmem_st16(tmem_base + lane_base + col_s(m) + half * 64 + 16, zero);
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(ds_ready);
        ++m;
        continue;
      }
      // P over this half's 64 keys, 32 at a time
      float pv[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sr[32];
        tmem_ld32(tmem_base + lane_base + col_s(m) + half * 64 + c * 32, sr);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u)
          pv[c * 32 + u] =
              c * 32 + u < lim ? ex2(fmaf(__uint_as_float(sr[u]), scale, -lse2)) : 0.f;
      }
      if (!mbar_wait_warp(dp_full, m & 1, &s_abort, hdr, 0xa615u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!pass1) {
        float ds[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ds[k] = 0.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dp[32];
          tmem_ld32(tmem_base + lane_base + COL_DP + half * 64 + c * 32, dp);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u)
            ds[u & 7] = fmaf(pv[c * 32 + u], __uint_as_float(dp[u]), ds[u & 7]);
        }
        dot += ((ds[0] + ds[1]) + (ds[2] + ds[3])) + ((ds[4] + ds[5]) + (ds[6] + ds[7]));
      } else {
        // dS over keys 32c..32c+31 of this half goes to columns 16c..16c+15 of
        // the half's S region, whose scores were read above
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dp[32];
          tmem_ld32(tmem_base + lane_base + COL_DP + half * 64 + c * 32, dp);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int u = 2 * q;
            pk[q] = pack_bf16x2(pv[c * 32 + u] * (__uint_as_float(dp[u]) - dot),
                                pv[c * 32 + u + 1] * (__uint_as_float(dp[u + 1]) - dot));
          }
          tmem_st16(tmem_base + lane_base + col_s(m) + half * 64 + c * 16, pk);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(ds_ready);
      ++m;
    }
    if (ok && !dot_done && valid && half == 0) a.dot[rix] = 0.f;  // no blocks at all

    long long t0 = clock64();
    bool done = ok;
    if (ok && m > 0) {
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
      for (int c = half * 64; c < half * 64 + 64; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_base + c, o);
        tmem_ld_wait();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + c);
          const float sc = a.inv_sqrt_d;
#pragma unroll
          for (int x = 0; x < 8; ++x)
            d4[x] = m > 0 ? make_float4(__uint_as_float(o[4 * x]) * sc,
                                        __uint_as_float(o[4 * x + 1]) * sc,
                                        __uint_as_float(o[4 * x + 2]) * sc,
                                        __uint_as_float(o[4 * x + 3]) * sc)
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
// Key pieces: the keys of each cube cut into pieces of up to 64 (cubes hold at
// most 256 tokens), cube by cube, then the text suffix in pieces of 64. One
// CTA per (KV head, pair of consecutive pieces) = up to 128 keys. It walks the
// query tiles that admit either piece (the union of the two cubes' inverted
// lists, ascending, then the text tiles) and computes, per tile,
//   S^T = K Q^T and dP^T = V dO^T      (M = 128 keys, N = 128 rows, K = d)
// into TMEM; one thread per key turns them into P^T and dS^T (bf16, written
// over the scores they came from), and
//   dV += P^T dO,  dK += dS^T Q        (M = 128 keys, N = d, K = 128 rows)
// read P^T / dS^T from TMEM (the product form of the forward's PV), so every
// product has N = 128 and the key block's gradients stay in TMEM until the
// end. Warps: 0 tile walker + TMA producer, 1 TMEM allocator + MMA issuer,
// 2-9 row threads: thread = key (TMEM lane), two warps per lane quadrant,
// each taking 64 of the tile's 128 rows. TMEM (512 columns): S^T 0-127,
// dP^T 128-255, dV 256-383, dK 384-511.
namespace dkv {
constexpr int THREADS = 320;
constexpr int ROW_THREADS = 256;
constexpr int QST = 2;
constexpr int RINGE = 64;                 // tile-walk ring entries
constexpr int KP_BYTES = 2 * 16384;       // 128 keys x 128 dims bf16 (two 64-dim halves)
constexpr size_t SMEM_BYTES = 1024 + 2 * KP_BYTES + QST * 2 * Q_BYTES + 2048;
}  // namespace dkv

struct Piece {
  int cube;   // -1: text keys
  int k0, nk;
  int pad;
};

// Piece table (one block): pieces of every cube in order, then the text
// pieces; the count goes to hdr->spare0.
__global__ void __launch_bounds__(1024) piece_table_kernel(AttnBwdArgs a) {
  __shared__ int part[1024];
  if (status_bad(a.hdr)) return;
  const AttnGeom& G = a.G;
  const int C = G.n_cubes, tid = threadIdx.x;
  const int per = (C + 1023) / 1024;
  const int b = min(tid * per, C), e = min(b + per, C);
  int cnt = 0;
  for (int j = b; j < e; ++j) cnt += (a.cube_offsets[j + 1] - a.cube_offsets[j] + 63) / 64;
  part[tid] = cnt;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int pos = part[tid] - cnt;
  Piece* out = reinterpret_cast<Piece*>(a.pieces);
  for (int j = b; j < e; ++j) {
    const int k0 = a.cube_offsets[j], ke = a.cube_offsets[j + 1];
    for (int k = k0; k < ke; k += 64) out[pos++] = Piece{j, k, min(64, ke - k), 0};
  }
  const int n_vis_pieces = part[1023];
  const int n_text = G.n_tokens - G.n_vis;
  const int n_tp = (n_text + 63) / 64;
  for (int q = tid; q < n_tp; q += 1024) {
    const int k0 = G.n_vis + 64 * q;
    out[n_vis_pieces + q] = Piece{-1, k0, min(64, G.n_tokens - k0), 0};
  }
  if (tid == 0) a.hdr->spare0 = (uint32_t)(n_vis_pieces + n_tp);
}

struct WalkEntry {
  int bt;      // tile index within its kind; -1 terminates
  int text;
};

// Admitted keys of row `row` of tile (text, bt) in a piece: keys [k0, k0 + lim).
__device__ __forceinline__ int piece_limit(const AttnBwdArgs& a, const Piece& pc, bool text,
                                           int bt, int row, const TileRow& R, int own, int c_hi,
                                           bool dense) {
  if (!R.valid || pc.nk <= 0) return 0;
  const AttnGeom& G = a.G;
  if (pc.cube < 0) {  // text keys: only text rows, causally
    if (!text) return 0;
    return max(0, min(pc.nk, R.t - pc.k0 + 1));
  }
  if (text) return pc.nk;  // text rows see every visual key
  if (pc.cube > c_hi) return 0;  // follows every row of the tile (mask not written)
  bool on;
  if (dense) {
    on = pc.cube <= own;
  } else {
    const uint32_t w = a.tile_mask[((size_t)bt * G.n_cubes + pc.cube) * 4 + (row >> 5)];
    on = ((w >> (row & 31)) & 1u) != 0u;
  }
  if (!on) return 0;
  return pc.cube == own ? max(0, min(pc.nk, R.t - pc.k0 + 1)) : pc.nk;
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
  uint8_t* sK = smem;                       // keys 0-63: piece A, 64-127: piece B
  uint8_t* sV = sK + KP_BYTES;
  uint8_t* sQd = sV + KP_BYTES;             // [QST][Q tile | dO tile]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQd + QST * 2 * Q_BYTES);
  uint64_t* kv_full = bars;
  uint64_t* qd_full = kv_full + 1;          // [QST]
  uint64_t* qd_empty = qd_full + QST;       // [QST]
  uint64_t* s_full = qd_empty + QST;       // S^T landed
  uint64_t* dp_full = s_full + 1;           // dP^T landed
  uint64_t* p_ready = dp_full + 1;          // P^T stored by the row threads
  uint64_t* ds_ready = p_ready + 1;         // dS^T stored by the row threads
  uint64_t* meta_full = ds_ready + 1;       // [2]
  uint64_t* done = meta_full + 2;
  uint64_t* w_full = done + 1;              // [RINGE]
  uint64_t* w_empty = w_full + RINGE;       // [RINGE]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(w_empty + RINGE);
  __shared__ WalkEntry s_walk[RINGE];
  // per row and piece: the row's log2-sum-exp, or +inf where the row takes no
  // key of the piece (its P then comes out as an exact zero)
  __shared__ float s_lse[2][2][128], s_dot[2][128];
  __shared__ int s_lim[2][2][128];          // [entry parity][piece][row]
  __shared__ int s_on[2][2][4];             // [entry parity][piece][row quarter]: any row on
  __shared__ int s_part[2][2][4];           // ... any row taking only some keys of the piece
  __shared__ volatile int s_abort;

  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  if (status_bad(hdr)) return;              // uniform: before any barrier or TMEM
  const int n_pieces = (int)hdr->spare0;
  const int units = (4 * G.n_cubes + (G.n_tokens - G.n_vis + 63) / 64 + 1) / 2;
  const int kv = blockIdx.x / units, u = blockIdx.x - kv * units;
  if (2 * u >= n_pieces) return;
  const Piece* pieces = reinterpret_cast<const Piece*>(a.pieces);
  const Piece pA = pieces[2 * u];
  const Piece pB = 2 * u + 1 < n_pieces ? pieces[2 * u + 1] : Piece{-1, pA.k0, 0, 0};
  const bool dense = fwd_was_dense(a.fhdr);
  // visual lists of the two pieces' cubes (the same list once if one cube)
  const int jA = pA.cube, jB = (pB.nk > 0 && pB.cube != pA.cube) ? pB.cube : -1;
  const size_t nc = a.inv_chunks;
  auto list_of = [&](int j, const int32_t*& lst, int& n) {
    if (j < 0) {
      lst = nullptr;
      n = 0;
      return;
    }
    const size_t key = ((size_t)kv * G.n_cubes + j) * nc;
    lst = a.inv_list + a.inv_start[key];
    n = a.inv_start[key + nc] - a.inv_start[key];
  };
  // text tiles: all of them when a visual piece is present, else those that
  // reach the first text key
  const bool any_visual = jA >= 0 || (pB.nk > 0 && pB.cube >= 0);
  const int tt_min = any_visual ? 0 : (pA.k0 - G.n_vis) / kTileRows;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(&qd_full[s], 1);
      mbar_init(&qd_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, ROW_THREADS);
    mbar_init(ds_ready, ROW_THREADS);
    for (int b = 0; b < 2; ++b) mbar_init(&meta_full[b], ROW_THREADS);
    mbar_init(done, 1);
    for (int r = 0; r < RINGE; ++r) {
      mbar_init(&w_full[r], 1);
      mbar_init(&w_empty[r], ROW_THREADS);
    }
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
    // ------------------------------------------------------------ tile walker + producer
    if (lane == 0) {
      mbar_expect_tx(kv_full, (pB.nk > 0 ? 4u : 2u) * 8192u * 2u);
      tma_load_3d(&mapK, kv_full, sK, 0, kv, pA.k0);
      tma_load_3d(&mapK, kv_full, sK + 16384, 64, kv, pA.k0);
      tma_load_3d(&mapV, kv_full, sV, 0, kv, pA.k0);
      tma_load_3d(&mapV, kv_full, sV + 16384, 64, kv, pA.k0);
      if (pB.nk > 0) {
        tma_load_3d(&mapK, kv_full, sK + 8192, 0, kv, pB.k0);
        tma_load_3d(&mapK, kv_full, sK + 16384 + 8192, 64, kv, pB.k0);
        tma_load_3d(&mapV, kv_full, sV + 8192, 0, kv, pB.k0);
        tma_load_3d(&mapV, kv_full, sV + 16384 + 8192, 64, kv, pB.k0);
      }
      const int32_t *LA, *LB;
      int nA, nB;
      list_of(jA, LA, nA);
      list_of(jB, LB, nB);
      const int nt = G.ttiles_per_head - tt_min;
      const int n_text_entries = G.g * nt;
      int ia = 0, ib = 0, et = 0, e = 0;
      bool ok = true;
      while (ok) {
        // next entry: merge of the two ascending lists, then the text tiles
        WalkEntry we;
        if (ia < nA || ib < nB) {
          const int va = ia < nA ? LA[ia] : INT32_MAX, vb = ib < nB ? LB[ib] : INT32_MAX;
          const int v = min(va, vb);
          ia += va == v;
          ib += vb == v;
          we = WalkEntry{v, 0};
        } else if (et < n_text_entries) {
          const int hh = et / nt, tt = tt_min + et % nt;
          we = WalkEntry{kv * G.ttiles_per_kv + hh * G.ttiles_per_head + tt, 1};
          ++et;
        } else {
          we = WalkEntry{-1, 0};
        }
        const int slot = e % RINGE;
        if (!mbar_wait(&w_empty[slot], ((e / RINGE) & 1) ^ 1, &s_abort, hdr, 0xa800u)) {
          ok = false;
          break;
        }
        s_walk[slot] = we;
        mbar_arrive(&w_full[slot]);
        if (we.bt < 0) break;
        const int st = e % QST;
        if (!mbar_wait(&qd_empty[st], ((e / QST) & 1) ^ 1, &s_abort, hdr, 0xa810u)) {
          ok = false;
          break;
        }
        const TileRow R0 = tile_row(G, we.text != 0, we.bt, 0);
        uint8_t* q = sQd + st * 2 * Q_BYTES;
        mbar_expect_tx(&qd_full[st], 2 * Q_BYTES);
        tma_load_3d(&mapQ, &qd_full[st], q, 0, R0.h, R0.t);
        tma_load_3d(&mapQ, &qd_full[st], q + 16384, 64, R0.h, R0.t);
        tma_load_3d(&mapdO, &qd_full[st], q + Q_BYTES, 0, R0.h, R0.t);
        tma_load_3d(&mapdO, &qd_full[st], q + Q_BYTES + 16384, 64, R0.h, R0.t);
        ++e;
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
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128);
      constexpr uint32_t idesc_g = make_idesc_bf16(128, 128, true);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(kv_full, 0, &s_abort, hdr, 0xa820u);
      tc_fence_after();
      int e = 0;
      for (; ok; ++e) {
        const int slot = e % RINGE;
        if (!mbar_wait(&w_full[slot], (e / RINGE) & 1, &s_abort, hdr, 0xa830u)) {
          ok = false;
          break;
        }
        if (s_walk[slot].bt < 0) break;
        const int st = e % QST;
        if (!mbar_wait(&qd_full[st], (e / QST) & 1, &s_abort, hdr, 0xa840u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQd + st * 2 * Q_BYTES);
        const uint32_t do_addr = q_addr + Q_BYTES;
        // S^T = K Q^T, then dP^T = V dO^T (both K-major, K = d), each with its
        // own commit so the row threads start on P while dP^T computes
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base, make_sdesc_sw128(k_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024), idesc_s,
                      (dc | kk) != 0 ? 1u : 0u);
        umma_commit(s_full);
#pragma unroll
        for (int dc = 0; dc < 2; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base + 128,
                      make_sdesc_sw128(v_addr + dc * 16384 + kk * 32, 16, 1024),
                      make_sdesc_sw128(do_addr + dc * 16384 + kk * 32, 16, 1024), idesc_s,
                      (dc | kk) != 0 ? 1u : 0u);
        umma_commit(dp_full);
        // dV += P^T dO as soon as P^T is in TMEM (rows 64 hc + r packed at
        // column 64 hc + r / 2), while the row threads form dS
        if (!mbar_wait(p_ready, e & 1, &s_abort, hdr, 0xa850u)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem_base + 256, tmem_base + (kk >> 2) * 64 + (kk & 3) * 8,
                       make_sdesc_sw128(do_addr + kk * 2048, 16384, 1024), idesc_g,
                       (e > 0 || kk > 0) ? 1u : 0u);
        // dK += dS^T Q
        if (!mbar_wait(ds_ready, e & 1, &s_abort, hdr, 0xa855u)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem_base + 384, tmem_base + 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                       make_sdesc_sw128(q_addr + kk * 2048, 16384, 1024), idesc_g,
                       (e > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&qd_empty[st]);
      }
      umma_commit(done);
      long long t0 = clock64();
      while (!mbar_try_wait(done, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int wq = warp & 3;
    const int key = wq * 32 + lane;           // TMEM lane = key of the pair
    const int hc = (warp - 2) >> 2;           // rows [64 hc, 64 hc + 64) of each tile
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float scale = a.scale_log2;
    const int kp = key < 64 ? 0 : 1;          // piece of this key
    const int kl = key & 63;                  // index inside the piece
    const int mrow = (warp - 2) * 32 + lane;  // 0..255: metadata of row mrow (first 128)
    bool ok = true;
    int e = 0;
    for (;; ++e) {
      const int slot = e % RINGE;
      if (!mbar_wait_warp(&w_full[slot], (e / RINGE) & 1, &s_abort, hdr, 0xa860u)) {
        ok = false;
        break;
      }
      const WalkEntry we = s_walk[slot];
      if (we.bt < 0) break;
      const bool text = we.text != 0;
      const int par = e & 1;
      // per-row data of the tile, one row per thread of the first 128
      if (mrow < 128) {
        const TileRow R = tile_row(G, text, we.bt, mrow);
        const size_t rix = (size_t)R.t * G.hq + R.h;
        int own = -1, c_hi = -1;
        if (!text && R.valid) {
          own = a.cube_ids[R.t];
          const TileRow Rl = tile_row(G, false, we.bt, 0);
          c_hi = a.cube_ids[min(Rl.t + kTileRows, G.n_vis) - 1];
        }
        const float lse = R.valid ? a.lse[rix] : 0.f;
        s_dot[par][mrow] = R.valid ? a.dot[rix] : 0.f;
        const int limA = piece_limit(a, pA, text, we.bt, mrow, R, own, c_hi, dense);
        const int limB = piece_limit(a, pB, text, we.bt, mrow, R, own, c_hi, dense);
        s_lim[par][0][mrow] = limA;
        s_lim[par][1][mrow] = limB;
        s_lse[par][0][mrow] = limA > 0 ? lse : INFINITY;
        s_lse[par][1][mrow] = limB > 0 ? lse : INFINITY;
        const unsigned onA = __ballot_sync(0xffffffffu, limA > 0);
        const unsigned onB = __ballot_sync(0xffffffffu, limB > 0);
        const unsigned ptA = __ballot_sync(0xffffffffu, limA > 0 && limA < 64);
        const unsigned ptB = __ballot_sync(0xffffffffu, limB > 0 && limB < 64);
        if (lane == 0) {
          s_on[par][0][mrow >> 5] = onA != 0u;
          s_on[par][1][mrow >> 5] = onB != 0u;
          s_part[par][0][mrow >> 5] = ptA != 0u;
          s_part[par][1][mrow >> 5] = ptB != 0u;
        }
      }
      mbar_arrive(&meta_full[par]);
      if (!mbar_wait_warp(&meta_full[par], (e >> 1) & 1, &s_abort, hdr, 0xa870u)) {
        ok = false;
        break;
      }
      // every row thread has read the slot once the metadata is in
      mbar_arrive(&w_empty[slot]);
      if (!mbar_wait_warp(s_full, e & 1, &s_abort, hdr, 0xa880u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!(s_on[par][kp][2 * hc] | s_on[par][kp][2 * hc + 1])) {
        // No row of this half takes a key of this warp's piece: P^T = 0 and
        // dS^T = 0 go over S^T and dP^T without reading them; both barriers
        // keep their order.
        uint32_t zero[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) zero[q] = 0u;
        tmem_st32(tmem_base + lane_base + hc * 64, zero);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_ready);
        if (!mbar_wait_warp(dp_full, e & 1, &s_abort, hdr, 0xa886u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem_base + lane_base + 128 + hc * 64, zero);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_ready);
        continue;
      }
      // Every row of the half takes all 64 keys of the piece or none: no
      // per-key limit (rows taking none have lse = +inf, so P = 0).
      const bool full = !(s_part[par][kp][2 * hc] | s_part[par][kp][2 * hc + 1]);
      float pv[64];
      {
        uint32_t sr[64];
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tmem_base + lane_base + hc * 64, s0);
        tmem_ld32(tmem_base + lane_base + hc * 64 + 32, s1);
        tmem_ld_wait();
        uint32_t pp[32];
        if (full) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const int r = hc * 64 + 2 * q + z;
              pv[2 * q + z] = ex2(fmaf(__uint_as_float(sr[2 * q + z]), scale, -s_lse[par][kp][r]));
            }
            pp[q] = pack_bf16x2(pv[2 * q], pv[2 * q + 1]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const int r = hc * 64 + 2 * q + z;
              pv[2 * q + z] =
                  kl < s_lim[par][kp][r]
                      ? ex2(fmaf(__uint_as_float(sr[2 * q + z]), scale, -s_lse[par][kp][r]))
                      : 0.f;
            }
            pp[q] = pack_bf16x2(pv[2 * q], pv[2 * q + 1]);
          }
        }
        tmem_st32(tmem_base + lane_base + hc * 64, pp);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(p_ready);
      if (!mbar_wait_warp(dp_full, e & 1, &s_abort, hdr, 0xa885u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t dp[64];
        uint32_t(&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[0]);
        uint32_t(&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&dp[32]);
        tmem_ld32(tmem_base + lane_base + 128 + hc * 64, p0);
        tmem_ld32(tmem_base + lane_base + 128 + hc * 64 + 32, p1);
        tmem_ld_wait();
        uint32_t pd[32];
        if (full) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            float dv[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const int r = hc * 64 + 2 * q + z;
              dv[z] = pv[2 * q + z] * (__uint_as_float(dp[2 * q + z]) - s_dot[par][r]);
            }
            pd[q] = pack_bf16x2(dv[0], dv[1]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            float dv[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const int r = hc * 64 + 2 * q + z;
              dv[z] = kl < s_lim[par][kp][r]
                          ? pv[2 * q + z] * (__uint_as_float(dp[2 * q + z]) - s_dot[par][r])
                          : 0.f;
            }
            pd[q] = pack_bf16x2(dv[0], dv[1]);
          }
        }
        tmem_st32(tmem_base + lane_base + 128 + hc * 64, pd);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(ds_ready);
    }
    // epilogue: thread = key, 64 of the 128 head dimensions of dV and dK
    long long t0 = clock64();
    bool fin = ok;
    if (ok && e > 0) {
      fin = false;
      while (!(fin = mbar_try_wait(done, 0)) && clock64() - t0 < kWaitCycles) {
      }
      if (!fin) set_status(hdr, ADASPARK_DEV_TIMEOUT, 0xa890u);
    }
    fin = __all_sync(0xffffffffu, fin);
    if (fin) {
      tc_fence_after();
      const Piece& pc = kp == 0 ? pA : pB;
      const bool kvalid = kl < pc.nk;
      const size_t o = ((size_t)(pc.k0 + kl) * G.hkv + kv) * 128 + hc * 64;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        uint32_t v[32], k[32];
        tmem_ld32(tmem_base + lane_base + 256 + hc * 64 + c, v);
        tmem_ld32(tmem_base + lane_base + 384 + hc * 64 + c, k);
        tmem_ld_wait();
        if (kvalid) {
          float4* dv4 = reinterpret_cast<float4*>(a.dV + o + c);
          float4* dk4 = reinterpret_cast<float4*>(a.dK + o + c);
          const float sk = a.inv_sqrt_d;
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            dv4[x] = e > 0 ? make_float4(__uint_as_float(v[4 * x]), __uint_as_float(v[4 * x + 1]),
                                         __uint_as_float(v[4 * x + 2]),
                                         __uint_as_float(v[4 * x + 3]))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            dk4[x] = e > 0 ? make_float4(__uint_as_float(k[4 * x]) * sk,
                                         __uint_as_float(k[4 * x + 1]) * sk,
                                         __uint_as_float(k[4 * x + 2]) * sk,
                                         __uint_as_float(k[4 * x + 3]) * sk)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
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
  {
    const int rows = G.n_tokens * G.hq;
    if ((e = launch("attn_bwd_dot", dot_kernel, dim3((rows + 7) / 8), dim3(256), 0, s, a)))
      return e;
  }
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
  // key pieces (64 keys) and their pairs
  if ((e = launch("attn_bwd_pieces", piece_table_kernel, dim3(1), dim3(1024), 0, s, a)))
    return e;
  const int units = (4 * G.n_cubes + (G.n_tokens - G.n_vis + 63) / 64 + 1) / 2;
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

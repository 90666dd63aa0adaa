// AdaS-Attn block-sparse attention on the 5th-generation tensor cores (bf16).
//
// Key design 2 of the AdaSpark note: a visual query attends to the keys of its
// selected cubes and, causally, of its own cube; one softmax over all admitted
// keys. A text query attends densely and causally.
//
// One CTA per 128-row tile (128 tokens of one query head). The tile walks a
// sequence of 64-key blocks: the cubes of its selection list (cubes where any
// row has its bit set) cut into 64-key pieces, or every cube then the text keys
// for a text tile. Rows that did not select a cube are masked inside the block.
// With the split walk (attn_split.cu) a visual tile walks only the cubes that
// more than a few of its rows chose (and its own cubes); each row then merges
// the partial results of its other cubes, computed beforehand by the
// gathered-tile kernel at the end of this file, with its own.
//   warp 6     block-descriptor filler: reads the list, cube offsets and row
//              masks from global memory 32 entries at a time and feeds a
//              64-slot shared-memory ring, far ahead of the consumers
//   warp 0     TMA producer: K and V blocks (3D maps over [token][kv][d], no
//              multicast) in two separate 2-stage rings; a K slot is released
//              as soon as its S MMA completes, so K loads run a block ahead of
//              the V loads (which wait for the PV MMA)
//   warp 1     TMEM allocator + tcgen05.mma issuer:
//                S_i = Q K_i^T   (M=128, N=64, K=128; two TMEM buffers)
//                O  += P_i V_i   (M=128, N=128, K=64; P read from TMEM where it
//                                 overwrote S_i, V read N-major from smem)
//   warps 2-5  one thread per row: Q gather, masking, online softmax with lazy
//              rescaling of O in TMEM, P (bf16) back into TMEM, final 1/l.
// With P kept in tensor memory a CTA needs ~100 KB of shared memory and 256
// TMEM columns, so two CTAs share an SM: while one runs its softmax the other
// keeps the tensor core busy. MMAs issued by one thread execute in order, which
// is what makes reusing the S buffer for P safe: S_{i+2} is issued after the
// PV_i that reads P_i from the same columns.
#include "attn_kernels.h"
#include "attn_tile.cuh"

namespace adaspark {
namespace fa {

constexpr int STAGES = 2;
constexpr int THREADS = 224;
constexpr int RING = 64;
// Head dimension D (64 or 128) in 64-dim halves: the query tile is 128 rows x
// D dims bf16, a K (or V) block 64 keys x D dims, each stored as 64-dim halves
// of 8 KB (per 64 rows) in the 128-byte swizzled layout.
template <int D> struct Dim {
  static constexpr int HALVES = D / 64;
  static constexpr int Q_BYTES = 128 * 2 * D;
  static constexpr int K_BYTES = HALVES * 8192;   // one K (or V) block
  static constexpr int KV_BYTES = 2 * K_BYTES;
};
struct Desc {
  int k0, nk, j, pad;
  uint32_t mask[4];
};
template <int D>
constexpr size_t smem_bytes() {
  return 1024 + Dim<D>::Q_BYTES + STAGES * Dim<D>::KV_BYTES + RING * sizeof(Desc) + 2048;
}
constexpr float kRescale = 8.0f;          // log2 headroom before O is rescaled

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes at once on the FMA pipe: (a0, a1) * s + (c, c).
__device__ __forceinline__ void fma2_bcast(float a0, float a1, float s, float c, float& o0,
                                           float& o1) {
  asm("{\n\t.reg .b64 pa, ps, pc, pr;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 ps, {%4, %4};\n\t"
      "mov.b64 pc, {%5, %5};\n\t"
      "fma.rn.f32x2 pr, pa, ps, pc;\n\t"
      "mov.b64 {%0, %1}, pr;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "f"(a0), "f"(a1), "f"(s), "f"(c));
}
// max(a, b, c) in one instruction (three-input form of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (s0, s1) += (a0, a1)
__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ps, pa;\n\t"
      "mov.b64 ps, {%0, %1};\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "add.rn.f32x2 ps, ps, pa;\n\t"
      "mov.b64 {%0, %1}, ps;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}


// TRAIN: for a backward pass to follow, P goes to the PV product as a bf16
// pair hi + lo (lo = P - hi, in the second half of the S buffer, whose
// scores were read before), so O is exact to about 2^-17 of each term, and O is
// also written in fp32 to a.o32; the backward takes D_r = dO_r . O_r from it.
template <bool TRAIN, int D>
__global__ void __launch_bounds__(THREADS, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                   AttnArgs a) {
  constexpr int Q_BYTES = Dim<D>::Q_BYTES, K_BYTES = Dim<D>::K_BYTES, KV_BYTES = Dim<D>::KV_BYTES;
  constexpr int HALVES = Dim<D>::HALVES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + Q_BYTES;
  Desc* ring = reinterpret_cast<Desc*>(sKV + STAGES * KV_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + RING);
  uint64_t* k_full = bars;                  // [STAGES]
  uint64_t* k_empty = k_full + STAGES;
  uint64_t* v_full = k_empty + STAGES;
  uint64_t* v_empty = v_full + STAGES;
  uint64_t* s_full = v_empty + STAGES;      // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* pv_done = p_full + 2;           // [2]
  uint64_t* q_full = pv_done + 2;
  uint64_t* drain = q_full + 1;
  uint64_t* r_full = drain + 1;             // [RING]
  uint64_t* r_empty = r_full + RING;        // [RING]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(r_empty + RING);
  __shared__ volatile int s_abort;
  __shared__ int s_own_hi, s_bad;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  const TileInfo T = decode_tile(G, a.kv_major != 0);
  // the tile walks only part of its list, the rest in gathered tiles
  const bool split = !TRAIN && a.sp.rows > 0 && !T.text && !a.dense;
  const long long WL = a.wait_limit;  // cycles before any wait of this kernel gives up

  if (warp == 2) {
    // the descriptor ring's barriers, one slot per lane and round
    for (int r = lane; r < RING; r += 32) {
      mbar_init(&r_full[r], 1);
      mbar_init(&r_empty[r], 128);
    }
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(q_full, 128);
    mbar_init(drain, 1);
    fence_mbar_init();
    s_abort = 0;
    s_bad = status_bad(hdr) ? 1 : 0;
    s_own_hi = (!T.text && !s_bad) ? a.cube_ids[T.t_hi] : -1;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
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
      } else if (a.dense) {
        n_entries = s_own_hi + 1;
      } else {
        n_entries = split ? a.sp.walk_count[T.bt] : a.tile_count[T.bt];
        use_list = true;
      }
    }
    const int n_total = n_entries + n_chunks;
    const uint16_t* list = (split ? a.sp.walk_list : a.tile_list) + (size_t)T.bt * G.n_cubes;
    const uint4* tmask = reinterpret_cast<const uint4*>(a.tile_mask) + (size_t)T.bt * G.n_cubes;
    int base = 0;
    bool ok = true;
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
        if (!mbar_wait(&r_empty[slot], ((idx / RING) & 1) ^ 1, &s_abort, hdr, 0x7a00u, WL)) {
          ok = false;
          break;
        }
        Desc& d = ring[slot];
        d.k0 = ks + 64 * b;
        d.nk = min(64, ke - d.k0);
        d.j = j;
        d.mask[0] = m.x;
        d.mask[1] = m.y;
        d.mask[2] = m.z;
        d.mask[3] = m.w;
        // (test hook: with withhold_first the first descriptor is never
        // announced, so every wait for it runs out and the kernel reports
        // ADASPARK_DEV_TIMEOUT)
        if (!(a.withhold_first && idx == 0)) mbar_arrive(&r_full[slot]);
      }
      ok = __all_sync(0xffffffffu, ok);
      base += total;
    }
    if (ok && lane == 0) {  // terminal descriptor
      const int slot = base % RING;
      if (mbar_wait(&r_empty[slot], ((base / RING) & 1) ^ 1, &s_abort, hdr, 0x7b00u, WL)) {
        ring[slot].nk = 0;
        if (!(a.withhold_first && base == 0)) mbar_arrive(&r_full[slot]);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Block i: K_i into K stage i % 2 (free once S_{i-2} is done), then V_{i-1}
    // into V stage (i-1) % 2 (free once PV_{i-3} is done).
    if (lane == 0) {
      uint8_t* sK = sKV;                       // [STAGES][K_BYTES]
      uint8_t* sV = sKV + STAGES * K_BYTES;    // [STAGES][K_BYTES]
      int i = 0, prev_k0 = 0, nv = 0;
      bool ok = true;
      auto load_v = [&](int blk, int k0) -> bool {
        const int s = blk % STAGES;
        if (!mbar_wait(&v_empty[s], ((blk / STAGES) & 1) ^ 1, &s_abort, hdr, 0x7110u, WL)) return false;
        mbar_expect_tx(&v_full[s], K_BYTES);
#pragma unroll
        for (int hf = 0; hf < HALVES; ++hf)
          tma_load_3d(&mapV, &v_full[s], sV + s * K_BYTES + hf * 8192, hf * 64, T.kv, k0);
        nv = blk + 1;
        return true;
      };
      while (ok) {
        const int slot = i % RING;
        if (!mbar_wait(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0x7000u, WL)) {
          ok = false;
          break;
        }
        const int k0 = ring[slot].k0, nk = ring[slot].nk;
        if (nk == 0) break;
        const int s = i % STAGES;
        if (!mbar_wait(&k_empty[s], ((i / STAGES) & 1) ^ 1, &s_abort, hdr, 0x7100u, WL)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&k_full[s], K_BYTES);
#pragma unroll
        for (int hf = 0; hf < HALVES; ++hf)
          tma_load_3d(&mapK, &k_full[s], sK + s * K_BYTES + hf * 8192, hf * 64, T.kv, k0);
        if (i > 0 && !load_v(i - 1, prev_k0)) {
          ok = false;
          break;
        }
        prev_k0 = k0;
        ++i;
      }
      if (ok && i > 0) ok = load_v(i - 1, prev_k0);
      if (!ok) {  // let copies already issued land before the CTA exits
        for (int k = 0; k < STAGES; ++k) {
          long long t0 = clock64();
          const int jk = i - 1 - k, jv = nv - 1 - k;
          while (jk >= 0 && !mbar_try_wait(&k_full[jk % STAGES], (jk / STAGES) & 1) &&
                 clock64() - t0 < WL) {
          }
          while (jv >= 0 && !mbar_try_wait(&v_full[jv % STAGES], (jv / STAGES) & 1) &&
                 clock64() - t0 < WL) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, D, true);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, &s_abort, hdr, 0x7200u, WL);
      tc_fence_after();
      int i = 0;
      auto issue_pv = [&](int blk) -> bool {
        const int pb = blk & 1;
        if (!mbar_wait(&p_full[pb], (blk >> 1) & 1, &s_abort, hdr, 0x7300u, WL)) return false;
        const int s = blk % STAGES;
        if (!mbar_wait(&v_full[s], (blk / STAGES) & 1, &s_abort, hdr, 0x7310u, WL)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sKV + STAGES * K_BYTES + s * K_BYTES);
        const uint32_t p_tmem = tmem_base + 128 + pb * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = make_sdesc_sw128(v_addr + kk * 2048, 8192, 1024);
          umma_bf16_ts(tmem_base, p_tmem + kk * 8, bd, idesc_o, (blk > 0 || kk > 0) ? 1u : 0u);
          if (TRAIN) umma_bf16_ts(tmem_base, p_tmem + 32 + kk * 8, bd, idesc_o, 1u);
        }
        umma_commit(&pv_done[pb]);
        umma_commit(&v_empty[s]);
        return true;
      };
      while (ok) {
        const int slot = i % RING;
        if (!mbar_wait(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0x7d00u, WL)) {
          ok = false;
          break;
        }
        if (ring[slot].nk == 0) break;
        const int s = i % STAGES;
        const int sb = i & 1;
        if (!mbar_wait(&k_full[s], (i / STAGES) & 1, &s_abort, hdr, 0x7400u, WL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sKV + s * K_BYTES);
        const uint32_t d_s = tmem_base + 128 + sb * 64;
#pragma unroll
        for (int dc = 0; dc < HALVES; ++dc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(k_addr + dc * 8192 + kk * 32, 16, 1024);
            umma_bf16(d_s, ad, bd, idesc_s, (dc | kk) != 0 ? 1u : 0u);
          }
        umma_commit(&s_full[sb]);
        umma_commit(&k_empty[s]);
        if (i > 0 && !issue_pv(i - 1)) {
          ok = false;
          break;
        }
        ++i;
      }
      if (ok && i > 0) issue_pv(i - 1);
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < WL) {
      }
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const TileRow R = tile_row(G, T.text, T.bt, row);
    const bool valid = R.valid;
    const int t = R.t, h = R.h;
    const int own = (!T.text && valid) ? a.cube_ids[t] : -1;
    const float scale = a.scale_log2;
    {
      const __nv_bfloat16* Qg = reinterpret_cast<const __nv_bfloat16*>(a.Q);
      const uint4* src = reinterpret_cast<const uint4*>(Qg + ((size_t)t * G.hq + h) * D);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 v = valid ? src[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sQ + (c >> 3) * 16384 + sw128_offset(row, c & 7)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(q_full);
    }
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    int i = 0;
    bool ok = true;
    while (true) {
      const int slot = i % RING;
      if (!mbar_wait_warp(&r_full[slot], (i / RING) & 1, &s_abort, hdr, 0x7e00u, WL)) {
        ok = false;
        break;
      }
      // the descriptor's fields straight from shared memory (a local copy
      // indexed by the warp's quadrant would live in local memory)
      const int d_nk = ring[slot].nk;
      if (d_nk == 0) break;
      const int d_k0 = ring[slot].k0, d_j = ring[slot].j;
      const uint32_t d_mask = ring[slot].mask[wq];
      // admitted keys [0, lim) of this row in the block
      bool row_on;
      if (!valid) row_on = false;
      else if (T.text) row_on = true;
      else if (a.dense) row_on = d_j <= own;
      else row_on = ((d_mask >> lane) & 1u) != 0u;
      int lim = row_on ? d_nk : 0;
      if (row_on && (T.text || d_j == own)) lim = min(lim, t - d_k0 + 1);
      if (lim <= 0) row_on = false;
      const int sb = i & 1;
      if (!mbar_wait_warp(&s_full[sb], (i >> 1) & 1, &s_abort, hdr, 0x7600u, WL)) {
        ok = false;
        break;
      }
      // S_i has landed, so the producer and the MMA issuer have both consumed
      // descriptor i: only now may the filler reuse its slot.
      mbar_arrive(&r_empty[slot]);
      tc_fence_after();
      if (!__any_sync(0xffffffffu, row_on)) {
        // No row of this warp takes a key of the block (the tile's list holds
        // the cube for other rows): P = 0 for its 32 rows, the value the
        // general path gives them, without reading S.
        uint32_t zero[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) zero[q] = 0u;
        tmem_st32(tmem_base + lane_base + 128 + sb * 64, zero);
        if (TRAIN) tmem_st32(tmem_base + lane_base + 128 + sb * 64 + 32, zero);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
        ++i;
        continue;
      }
      uint32_t sr[64];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64, s0);
        tmem_ld32(tmem_base + lane_base + 128 + sb * 64 + 32, s1);
      }
      tmem_ld_wait();

      // Blocks where every row of the warp takes all 64 keys or none need no
      // per-key mask: a row that takes none gets an offset of -inf, so its
      // probabilities come out as exact zeros.
      const bool partial = __any_sync(0xffffffffu, row_on && lim < 64);
      float mraw = -INFINITY;
      if (!partial) {
        // eight chains over columns 0-55, then the last eight columns
        auto f = [&](int u) { return __uint_as_float(sr[u]); };
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(f(k), f(k + 8), f(k + 16));
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], f(k + 24), f(k + 32));
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], f(k + 40), f(k + 48));
        const float t0 = fmax3(mx[0], mx[1], f(56)), t1 = fmax3(mx[2], mx[3], f(57));
        const float t2 = fmax3(mx[4], mx[5], f(58)), t3 = fmax3(mx[6], mx[7], f(59));
        const float t4 = fmax3(f(60), f(61), f(62));
        const float m8 = fmax3(fmax3(t0, t1, t2), fmax3(t3, t4, f(63)), -INFINITY);
        mraw = row_on ? m8 : -INFINITY;
      } else {
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
        for (int u = 0; u < 64; ++u)
          if (u < lim) mx[u & 7] = fmaxf(mx[u & 7], __uint_as_float(sr[u]));
        mraw = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                     fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      }
      const float m_new = fmaxf(m_used, mraw * scale);
      const bool want = m_new > m_used + kRescale;
      if (__any_sync(0xffffffffu, want)) {
        const float factor = (m_used == -INFINITY || m_new == -INFINITY) ? 1.f
                                                                         : ex2(m_used - m_new);
        if (i > 0) {
          if (!mbar_wait_warp(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, &s_abort, hdr,
                              0x7700u, WL)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(tmem_base + lane_base + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * factor);
            tmem_st32(tmem_base + lane_base + c, o);
          }
        }
        l *= factor;
        if (m_new != -INFINITY) m_used = m_new;
      }
      // P = 2^(s * scale - m_used) on admitted keys, bf16 pairs written over S_i
      const float neg_m = row_on ? -m_used : -INFINITY;
      float ls[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) ls[k] = 0.f;
      uint32_t pk[32];
      if (!partial) {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          float x0, x1;
          fma2_bcast(__uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1]), scale, neg_m,
                     x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          add2(ls[2 * (q & 3)], ls[2 * (q & 3) + 1], p0, p1);
          pk[q] = pack_bf16x2(p0, p1);
          if (TRAIN) sr[2 * q] = __float_as_uint(p0), sr[2 * q + 1] = __float_as_uint(p1);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int u = 2 * q;
          const float p0 = (u < lim) ? ex2(fmaf(__uint_as_float(sr[u]), scale, neg_m)) : 0.f;
          const float p1 =
              (u + 1 < lim) ? ex2(fmaf(__uint_as_float(sr[u + 1]), scale, neg_m)) : 0.f;
          ls[q & 7] += p0 + p1;
          pk[q] = pack_bf16x2(p0, p1);
          if (TRAIN) sr[u] = __float_as_uint(p0), sr[u + 1] = __float_as_uint(p1);
        }
      }
      tmem_st32(tmem_base + lane_base + 128 + sb * 64, pk);
      if (TRAIN) {
        // lo parts: P - bf16(P), pairs in the S buffer's columns 32-63
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const __nv_bfloat162 hv = *reinterpret_cast<const __nv_bfloat162*>(&pk[q]);
          const float2 hf = __bfloat1622float2(hv);
          pk[q] = pack_bf16x2(__uint_as_float(sr[2 * q]) - hf.x,
                              __uint_as_float(sr[2 * q + 1]) - hf.y);
        }
        tmem_st_wait();
        tmem_st32(tmem_base + lane_base + 128 + sb * 64 + 32, pk);
      }
      tmem_st_wait();
      l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      tc_fence_before();
      mbar_arrive(&p_full[sb]);
      ++i;
    }
    // final: O / l once the last PV has landed
    if (ok && i > 0 &&
        mbar_wait_warp(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, &s_abort, hdr, 0x7900u, WL)) {
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const float lse_own = m_used + __log2f(l);
      // Merge of the row's gathered partial results (split walk): with M the
      // largest of the log2-sum-exps, the row's softmax over all its keys is
      // the sum of the parts' normalised outputs weighted by 2^(lse - M) / S,
      // S the sum of those powers; lse of the whole row = M + log2 S.
      int mcnt = 0, moff = 0;
      float w_own = 1.f, M = 0.f, inv_S = 1.f, lse_row = lse_own;
      if (split && valid) {
        const size_t rid = (size_t)t * G.hq + h;
        mcnt = a.sp.row_cnt[rid];
        moff = a.sp.row_off[rid];
        if (mcnt > 0) {
          M = lse_own;
          for (int k = 0; k < mcnt; ++k) M = fmaxf(M, a.sp.part_lse[moff + k]);
          float S = ex2(lse_own - M);
          for (int k = 0; k < mcnt; ++k) S += ex2(a.sp.part_lse[moff + k] - M);
          inv_S = 1.f / S;
          w_own = ex2(lse_own - M) * inv_S;
          lse_row = M + __log2f(S);
        }
      }
      // the row's softmax is 2^(s * scale - lse): kept for the backward pass
      if (valid && a.lse) a.lse[(size_t)t * G.hq + h] = lse_row;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)t * G.hq + h) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_base + c, o);
        tmem_ld_wait();
        if (valid) {
          uint32_t pk[16];
          if (mcnt == 0) {
#pragma unroll
            for (int x = 0; x < 16; ++x)
              pk[x] = pack_bf16x2(__uint_as_float(o[2 * x]) * inv,
                                  __uint_as_float(o[2 * x + 1]) * inv);
          } else {
            float f[32];
            const float s_own = inv * w_own;
#pragma unroll
            for (int x = 0; x < 32; ++x) f[x] = __uint_as_float(o[x]) * s_own;
#pragma unroll 1
            for (int k = 0; k < mcnt; ++k) {
              const float wk = ex2(a.sp.part_lse[moff + k] - M) * inv_S;
              const uint4* src =
                  reinterpret_cast<const uint4*>(a.sp.part_o + (size_t)(moff + k) * D + c);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 v = src[q];
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                  const float2 pf = __bfloat1622float2(
                      *reinterpret_cast<const __nv_bfloat162*>(&w4[z]));
                  f[8 * q + 2 * z] = fmaf(wk, pf.x, f[8 * q + 2 * z]);
                  f[8 * q + 2 * z + 1] = fmaf(wk, pf.y, f[8 * q + 2 * z + 1]);
                }
              }
            }
#pragma unroll
            for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(f[2 * x], f[2 * x + 1]);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            d4[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
          if (TRAIN) {
            float4* o4 = reinterpret_cast<float4*>(a.o32 + ((size_t)t * G.hq + h) * D + c);
#pragma unroll
            for (int x = 0; x < 8; ++x)
              o4[x] = make_float4(__uint_as_float(o[4 * x]) * inv,
                                  __uint_as_float(o[4 * x + 1]) * inv,
                                  __uint_as_float(o[4 * x + 2]) * inv,
                                  __uint_as_float(o[4 * x + 3]) * inv);
          }
        }
      }
    }
    if (warp == 2 && lane == 0 && !bad) {
      atomicAdd((unsigned long long*)&hdr->stats[4], 1ull);
      atomicAdd((unsigned long long*)&hdr->stats[5], (unsigned long long)i);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}


// ---------------------------------------------------------------------------
// Gathered tiles of the split walk (see SplitLayout), persistent: CTA b takes
// gathered tiles b, b + grid, b + 2 grid, ... A gathered tile holds up to 128
// records (row, cube) of one (KV head, cube) group, query rows of many tiles
// and heads; it walks that cube's keys alone (no causal part: the cube lies
// below every row's own cube) and writes each record's normalised output
// (bf16) and log2-sum-exp, which the row's own tile merges at the end of its
// walk. The next tile's query rows are copied into the second Q buffer
// (cp.async) while the current tile computes, and its first scores are
// computed while the current tile's output is read, so one tile's chain of
// latencies overlaps the next one's.
//   warp 0     TMA producer: K and V blocks (one stage each)
//   warp 1     TMEM allocator + tcgen05.mma issuer (S into two buffers, O)
//   warps 2-5  one thread per row: Q copies, softmax, epilogue
// ---------------------------------------------------------------------------
constexpr int G_THREADS = 192;
template <int D>
constexpr size_t gather_smem_bytes() {
  return 1024 + 2 * Dim<D>::Q_BYTES + 2 * Dim<D>::K_BYTES + 512;
}

struct GTile {
  int kv, first, count, ks, ke;   // KV head, first record slot, rows, the cube's tokens
};
__device__ __forceinline__ GTile gather_tile(const AttnArgs& a, int m) {
  const int4 v = a.sp.mt_info[m];
  GTile g;
  g.first = v.x;
  g.count = v.y & 0xff;
  g.kv = v.y >> 8;
  g.ks = v.z;
  g.ke = v.w;
  return g;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(G_THREADS, 2)
    attn_gather_kernel(const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, AttnArgs a) {
  constexpr int Q_BYTES = Dim<D>::Q_BYTES, K_BYTES = Dim<D>::K_BYTES;
  constexpr int HALVES = Dim<D>::HALVES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // [2][Q_BYTES]
  uint8_t* sK = sQ + 2 * Q_BYTES;
  uint8_t* sV = sK + K_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + K_BYTES);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + 1;
  uint64_t* v_full = k_empty + 1;
  uint64_t* v_empty = v_full + 1;
  uint64_t* s_full = v_empty + 1;           // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* pv_done = p_full + 2;           // [2]
  uint64_t* q_full = pv_done + 2;           // [2]
  uint64_t* o_free = q_full + 2;
  uint64_t* drain = o_free + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const AttnGeom& G = a.G;
  WsHeader* hdr = a.hdr;
  const long long WL = a.wait_limit;
  // the regrouping counted the gathered tiles; CTAs beyond them have none
  const int total = (int)*reinterpret_cast<const volatile uint32_t*>(&hdr->sched[1]);
  // (a bad status set before this launch left the count at 0)
  if ((int)blockIdx.x >= total) return;
  const int step = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
      mbar_init(&q_full[b], 128);
    }
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    fence_mbar_init();
    s_abort = 0;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // block i: K_i (stage free once S_{i-1} is done), then V_i (free once
      // PV_{i-1} is done)
      int i = 0, nv = 0;
      bool ok = true;
      GTile gn = gather_tile(a, blockIdx.x);
      for (int m = blockIdx.x; ok && m < total; m += step) {
        const GTile g = gn;
        if (m + step < total) gn = gather_tile(a, m + step);   // in flight meanwhile
        for (int k0 = g.ks; k0 < g.ke; k0 += 64) {
          if (!mbar_wait(k_empty, (i & 1) ^ 1, &s_abort, hdr, 0x7a00u, WL)) {
            ok = false;
            break;
          }
          mbar_expect_tx(k_full, K_BYTES);
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf)
            tma_load_3d(&mapK, k_full, sK + hf * 8192, hf * 64, g.kv, k0);
          ++i;
          if (!mbar_wait(v_empty, (nv & 1) ^ 1, &s_abort, hdr, 0x7a10u, WL)) {
            ok = false;
            break;
          }
          mbar_expect_tx(v_full, K_BYTES);
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf)
            tma_load_3d(&mapV, v_full, sV + hf * 8192, hf * 64, g.kv, k0);
          ++nv;
        }
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        long long t0 = clock64();
        while (i > 0 && !mbar_try_wait(k_full, (i - 1) & 1) && clock64() - t0 < WL) {
        }
        while (nv > 0 && !mbar_try_wait(v_full, (nv - 1) & 1) && clock64() - t0 < WL) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, D, true);
      int i = 0, k = 0;
      bool ok = true, prev_first = false;
      int prev_tile = 0;
      // PV of block blk: its P, its V, and (first block of a tile after the
      // first) the previous tile's output read out of O
      auto issue_pv = [&](int blk, bool first, int tile) -> bool {
        const int pb = blk & 1;
        if (!mbar_wait(&p_full[pb], (blk >> 1) & 1, &s_abort, hdr, 0x7b00u, WL)) return false;
        if (!mbar_wait(v_full, blk & 1, &s_abort, hdr, 0x7b10u, WL)) return false;
        if (first && tile > 0 &&
            !mbar_wait(o_free, (tile - 1) & 1, &s_abort, hdr, 0x7b20u, WL))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV);
        const uint32_t p_tmem = tmem_base + 128 + pb * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = make_sdesc_sw128(v_addr + kk * 2048, 8192, 1024);
          umma_bf16_ts(tmem_base, p_tmem + kk * 8, bd, idesc_o, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[pb]);
        umma_commit(v_empty);
        return true;
      };
      GTile gn = gather_tile(a, blockIdx.x);
      for (int m = blockIdx.x; ok && m < total; m += step, ++k) {
        const GTile g = gn;
        if (m + step < total) gn = gather_tile(a, m + step);   // in flight meanwhile
        // the previous tile's last PV first: its output does not wait for
        // this tile's keys
        if (i > 0 && !issue_pv(i - 1, prev_first, prev_tile)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&q_full[k & 1], (k >> 1) & 1, &s_abort, hdr, 0x7b30u, WL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + (k & 1) * Q_BYTES);
        for (int k0 = g.ks; k0 < g.ke; k0 += 64, ++i) {
          if (!mbar_wait(k_full, i & 1, &s_abort, hdr, 0x7b40u, WL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK);
          const uint32_t d_s = tmem_base + 128 + (i & 1) * 64;
#pragma unroll
          for (int dc = 0; dc < HALVES; ++dc)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = make_sdesc_sw128(q_addr + dc * 16384 + kk * 32, 16, 1024);
              const uint64_t bd = make_sdesc_sw128(k_addr + dc * 8192 + kk * 32, 16, 1024);
              umma_bf16(d_s, ad, bd, idesc_s, (dc | kk) != 0 ? 1u : 0u);
            }
          umma_commit(&s_full[i & 1]);
          umma_commit(k_empty);
          // within a tile, the previous block's PV after this block's S
          if (k0 != g.ks && !issue_pv(i - 1, prev_first, prev_tile)) {
            ok = false;
            break;
          }
          prev_first = k0 == g.ks;
          prev_tile = k;
        }
      }
      if (ok && i > 0) issue_pv(i - 1, prev_first, prev_tile);
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < WL) {
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int wq = warp & 3;                // the TMEM lane quadrant this warp may access
    const int row = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float scale = a.scale_log2;
    // Row data arrive in stages, each a tile ahead of its use: the tile table
    // entry three tiles ahead, the records and rows two ahead, the query copy
    // one ahead.
    auto row_rec = [&](const GTile& g, int& rec, int& rid) {
      const bool v = row < g.count;
      rec = v ? a.sp.grec[g.first + row] : 0;
      rid = v ? a.sp.grow[g.first + row] : 0;
    };
    // the row's query into Q buffer qb, 16-byte copies (zeros for a row past
    // the tile's count), completed before q_full is announced
    auto copy_q = [&](int qb, bool valid, int rid) {
      const __nv_bfloat16* Qg = reinterpret_cast<const __nv_bfloat16*>(a.Q);
      const uint8_t* src = reinterpret_cast<const uint8_t*>(Qg + (size_t)rid * D);
      const uint32_t dst = smem_u32(sQ + qb * Q_BYTES);
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        cp_async16(dst + (c >> 3) * 16384 + sw128_offset(row, c & 7), src + c * 16,
                   valid ? 16u : 0u);
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const GTile g_none{0, 0, 0, 0, 0};
    GTile g = gather_tile(a, blockIdx.x);
    GTile g1 = blockIdx.x + step < total ? gather_tile(a, blockIdx.x + step) : g_none;
    GTile g2 = blockIdx.x + 2 * step < total ? gather_tile(a, blockIdx.x + 2 * step) : g_none;
    int rec, rid, rec1, rid1;
    row_rec(g, rec, rid);
    row_rec(g1, rec1, rid1);
    bool valid = row < g.count;
    copy_q(0, valid, rid);
    cp_async_wait_all();
    fence_proxy_async_smem();
    mbar_arrive(&q_full[0]);
    int i = 0, k = 0, pairs = 0;
    bool ok = true;
    for (int m = blockIdx.x; ok && m < total; m += step, ++k) {
      const bool has_next = m + step < total;
      // the next tile's queries, copied while this one computes
      if (has_next) copy_q((k + 1) & 1, row < g1.count, rid1);
      // records and rows two tiles ahead, the table entry three ahead
      int rec2 = 0, rid2 = 0;
      row_rec(g2, rec2, rid2);
      const GTile g3 = m + 3 * step < total ? gather_tile(a, m + 3 * step) : g_none;
      pairs += g.count;
      float m_used = -INFINITY, l = 0.f;
      for (int k0 = g.ks; k0 < g.ke; k0 += 64, ++i) {
        const int sb = i & 1;
        const bool row_on = valid;
        const int lim = row_on ? min(64, g.ke - k0) : 0;
        if (!mbar_wait_warp(&s_full[sb], (i >> 1) & 1, &s_abort, hdr, 0x7c00u, WL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!__any_sync(0xffffffffu, row_on)) {
          uint32_t zero[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) zero[q] = 0u;
          tmem_st32(tmem_base + lane_base + 128 + sb * 64, zero);
        } else {
          uint32_t sr[64];
          {
            uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
            uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
            tmem_ld32(tmem_base + lane_base + 128 + sb * 64, s0);
            tmem_ld32(tmem_base + lane_base + 128 + sb * 64 + 32, s1);
          }
          tmem_ld_wait();
          const bool partial = __any_sync(0xffffffffu, row_on && lim < 64);
          float mraw = -INFINITY;
          if (!partial) {
            auto f = [&](int u) { return __uint_as_float(sr[u]); };
            float mx[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = fmax3(f(q), f(q + 8), f(q + 16));
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], f(q + 24), f(q + 32));
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], f(q + 40), f(q + 48));
            const float t0 = fmax3(mx[0], mx[1], f(56)), t1 = fmax3(mx[2], mx[3], f(57));
            const float t2 = fmax3(mx[4], mx[5], f(58)), t3 = fmax3(mx[6], mx[7], f(59));
            const float t4 = fmax3(f(60), f(61), f(62));
            const float m8 = fmax3(fmax3(t0, t1, t2), fmax3(t3, t4, f(63)), -INFINITY);
            mraw = row_on ? m8 : -INFINITY;
          } else {
            float mx[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
            for (int u = 0; u < 64; ++u)
              if (u < lim) mx[u & 7] = fmaxf(mx[u & 7], __uint_as_float(sr[u]));
            mraw = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
          }
          const float m_new = fmaxf(m_used, mraw * scale);
          const bool want = m_new > m_used + kRescale;
          if (__any_sync(0xffffffffu, want)) {
            const float factor = (m_used == -INFINITY || m_new == -INFINITY) ? 1.f
                                                                             : ex2(m_used - m_new);
            if (k0 != g.ks) {  // O holds this tile's earlier blocks
              if (!mbar_wait_warp(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, &s_abort, hdr,
                                  0x7c10u, WL)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < D; c += 32) {
                uint32_t o[32];
                tmem_ld32(tmem_base + lane_base + c, o);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; ++x)
                  o[x] = __float_as_uint(__uint_as_float(o[x]) * factor);
                tmem_st32(tmem_base + lane_base + c, o);
              }
            }
            l *= factor;
            if (m_new != -INFINITY) m_used = m_new;
          }
          const float neg_m = row_on ? -m_used : -INFINITY;
          float ls[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) ls[q] = 0.f;
          uint32_t pk[32];
          if (!partial) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              float x0, x1;
              fma2_bcast(__uint_as_float(sr[2 * q]), __uint_as_float(sr[2 * q + 1]), scale,
                         neg_m, x0, x1);
              const float p0 = ex2(x0), p1 = ex2(x1);
              add2(ls[2 * (q & 3)], ls[2 * (q & 3) + 1], p0, p1);
              pk[q] = pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int u = 2 * q;
              const float p0 = (u < lim) ? ex2(fmaf(__uint_as_float(sr[u]), scale, neg_m)) : 0.f;
              const float p1 =
                  (u + 1 < lim) ? ex2(fmaf(__uint_as_float(sr[u + 1]), scale, neg_m)) : 0.f;
              ls[q & 7] += p0 + p1;
              pk[q] = pack_bf16x2(p0, p1);
            }
          }
          tmem_st32(tmem_base + lane_base + 128 + sb * 64, pk);
          l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
        if (k0 == g.ks && has_next) {  // the next tile's queries are in
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(&q_full[(k + 1) & 1]);
        }
      }
      if (!ok) break;
      // the tile's output: O / l once its last PV has landed, then O is free
      if (!mbar_wait_warp(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, &s_abort, hdr, 0x7c20u,
                          WL)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* dst = a.sp.part_o + (size_t)rec * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_base + lane_base + c, o);
        tmem_ld_wait();
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x] = pack_bf16x2(__uint_as_float(o[2 * x]) * inv,
                                __uint_as_float(o[2 * x + 1]) * inv);
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            d4[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(o_free);
      if (valid) a.sp.part_lse[rec] = m_used + __log2f(l);
      g = g1;
      rec = rec1;
      valid = row < g.count;
      g1 = g2;
      rec1 = rec2;
      rid1 = rid2;
      g2 = g3;
    }
    cp_async_wait_all();   // no copy outlives the CTA
    if (warp == 2 && lane == 0 && ok) {
      atomicAdd((unsigned long long*)&hdr->stats[8], (unsigned long long)pairs);
      atomicAdd((unsigned long long*)&hdr->stats[9], (unsigned long long)i);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace fa

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  const AttnGeom& G = a.G;
  const int blocks = G.n_vtiles + G.n_ttiles;
  if (blocks == 0) return cudaSuccess;
  CUtensorMap mK, mV;
  const uint64_t dims[3] = {(uint64_t)G.d, (uint64_t)G.hkv, (uint64_t)G.n_tokens};
  const uint64_t strides[2] = {(uint64_t)G.d * 2, (uint64_t)G.hkv * G.d * 2};
  const uint32_t box[3] = {64, 1, 64};
  if (!encode_tmap_bf16(&mK, a.K, 3, dims, strides, box) ||
      !encode_tmap_bf16(&mV, a.V, 3, dims, strides, box))
    return cudaErrorInvalidValue;
  auto k = G.d == 64 ? (a.o32 ? fa::attn_tc_kernel<true, 64> : fa::attn_tc_kernel<false, 64>)
                     : (a.o32 ? fa::attn_tc_kernel<true, 128> : fa::attn_tc_kernel<false, 128>);
  const size_t smem = G.d == 64 ? fa::smem_bytes<64>() : fa::smem_bytes<128>();
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch("attn_tc", k, dim3(blocks), dim3(fa::THREADS), smem, s, mK, mV, a);
}

// The gathered tiles of the split walk: two persistent CTAs per SM (fewer when
// fewer gathered tiles can exist); CTAs past the count the regrouping wrote
// exit at once.
cudaError_t launch_attn_tc_gather(const AttnArgs& a, cudaStream_t s) {
  const AttnGeom& G = a.G;
  if (a.sp.rows <= 0 || a.sp.max_mtiles <= 0 || G.n_vtiles == 0) return cudaSuccess;
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n_sm = 148;
  }
  CUtensorMap mK, mV;
  const uint64_t dims[3] = {(uint64_t)G.d, (uint64_t)G.hkv, (uint64_t)G.n_tokens};
  const uint64_t strides[2] = {(uint64_t)G.d * 2, (uint64_t)G.hkv * G.d * 2};
  const uint32_t box[3] = {64, 1, 64};
  if (!encode_tmap_bf16(&mK, a.K, 3, dims, strides, box) ||
      !encode_tmap_bf16(&mV, a.V, 3, dims, strides, box))
    return cudaErrorInvalidValue;
  auto k = G.d == 64 ? fa::attn_gather_kernel<64> : fa::attn_gather_kernel<128>;
  const size_t smem = G.d == 64 ? fa::gather_smem_bytes<64>() : fa::gather_smem_bytes<128>();
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(a.sp.max_mtiles, 2 * n_sm);
  return launch("attn_tc_gather", k, dim3(grid), dim3(fa::G_THREADS), smem, s, mK, mV, a);
}

}  // namespace adaspark

// Backward pass of AdaS-FFN with the active set held fixed (straight-through
// selection, for the light fine-tuning the AdaSpark note mentions; key design 3
// differentiated as computed).
//
// The forward gives active or text row a the output y_a = x_a + f_a with
// f = W_down(silu(W_gate x) * W_up x), and skipped row k of cube c the output
// y_k = x_k + mean of f over the cube's active rows. So for the upstream dy:
//   skipped k:  dx_k = dy_k
//   active a:   df_a = dy_a + G_c,  G_c = (sum of dy_k over the cube's skipped
//               rows) / (number of active rows);  text rows: df = dy
//   computed:   dh = df W_down; du = dh silu(g); dg = dh u silu'(g)
//               dx = dy + dg W_gate + du W_up
//               dW_gate = dg^T x_a, dW_up = du^T x_a, dW_down = df^T h
// All contractions run on the tcgen05 tensor cores in bf16 with fp32
// accumulation; gradients come out in fp32. Rows are those of the forward's
// compaction (its idx / row_cube / x_a and active-row count), read from the
// forward workspace.
//
// Kernels, in launch order:
//   ffn_bwd_skip      per cube: G_c and dx of the skipped rows (HBM)
//   ffn_bwd_df        df in compacted row order, bf16, plus its transpose (HBM)
//   bwd_transpose     x_a^T, W_down^T, [W_gate^T | W_up^T] in bf16 (HBM)
//   ffn_bwd_gemm<0>   per 128 x 64 tile of (rows, F): gate|up = x_a [W_gate;
//                     W_up]^T and dh = df (W_down^T)^T share K = D, so one
//                     k-loop feeds two MMAs (N = 128 and N = 64) into 192 TMEM
//                     columns, two such sets so the epilogue of one tile
//                     overlaps the products of the next; the epilogue forms
//                     dg, du, h and stores [dg du] row-major plus [dg du]^T and
//                     h^T (the K-major operands of the weight-gradient GEMMs)
//   ffn_bwd_gemm<1>   dx[idx] = dy[idx] + [dg du] [W_gate^T | W_up^T]^T (K = 2F)
//   ffn_bwd_gemm<2>   weight gradients, K = active rows (a device count):
//                     [dW_gate; dW_up] = [dg du]^T (x_a^T)^T, dW_down = df^T (h^T)^T
// The transposed buffers are zero in the columns between the active-row count
// and the next multiple of 64, so the last K block of <2> adds nothing extra.
#include <algorithm>

#include "ffn_kernels.h"

namespace adaspark {
namespace fbwd {

// --------------------------------------------------------------------- small kernels
__global__ void __launch_bounds__(32) bwd_check_kernel(WsHeader* hdr, const WsHeader* fhdr) {
  if (threadIdx.x == 0 && fhdr->status != 0u) set_status(hdr, fhdr->status, 0x9100u);
}

// One block per cube: G_c = sum of dy over the skipped rows / active count, and
// dx = dy on those rows. Four features per thread and step.
__global__ void __launch_bounds__(256) ffn_bwd_skip_kernel(FfnBwdArgs a) {
  if (status_bad(a.hdr)) return;
  const int c = blockIdx.x;
  const int base = a.cube_offsets[c], n = a.cube_offsets[c + 1] - base;
  const int cnt = a.cube_count[c];
  const float inv = cnt > 0 ? 1.f / (float)cnt : 0.f;
  for (int e = threadIdx.x * 4; e < a.D; e += 256 * 4) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int u = 0; u < n; ++u) {
      const int t = base + u;
      if (a.active[t]) continue;
      const float4 v = *reinterpret_cast<const float4*>(a.dy + (size_t)t * a.D + e);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
      *reinterpret_cast<float4*>(a.dx + (size_t)t * a.D + e) = v;
    }
    *reinterpret_cast<float4*>(a.gsum + (size_t)c * a.D + e) =
        make_float4(s.x * inv, s.y * inv, s.z * inv, s.w * inv);
  }
}

// 64 x 64 tiles of df = dy[idx] + G[row_cube] (compacted rows): bf16 row-major
// into df and, through shared memory, transposed into dfT [D][mp]. Rows from
// the active count up to the next multiple of 64 are written as zeros in dfT.
__global__ void __launch_bounds__(256) ffn_bwd_df_kernel(FfnBwdArgs a) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];
  if (status_bad(a.hdr)) return;
  const int m = (int)*a.m_active;
  const int r0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  if (r0 >= (m + 63) / 64 * 64) return;
  const int tid = threadIdx.x;
  {
    const int rr = tid >> 2, q = tid & 3;
    const int i = r0 + rr;
    float v[16];
    if (i < m) {
      const int src = a.idx[i], cube = a.row_cube[i];
      const float4* dyp = reinterpret_cast<const float4*>(a.dy + (size_t)src * a.D + c0 + q * 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 f = dyp[k];
        v[4 * k] = f.x;
        v[4 * k + 1] = f.y;
        v[4 * k + 2] = f.z;
        v[4 * k + 3] = f.w;
      }
      if (cube >= 0) {
        const float4* gp =
            reinterpret_cast<const float4*>(a.gsum + (size_t)cube * a.D + c0 + q * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 g = gp[k];
          v[4 * k] += g.x;
          v[4 * k + 1] += g.y;
          v[4 * k + 2] += g.z;
          v[4 * k + 3] += g.w;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = 0.f;
    }
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2(v[2 * k], v[2 * k + 1]);
    if (i < m) {
      uint4* dst = reinterpret_cast<uint4*>(a.df + (size_t)i * a.D + c0 + q * 16);
      dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    uint32_t* trow = reinterpret_cast<uint32_t*>(&tile[rr][q * 16]);
#pragma unroll
    for (int k = 0; k < 8; ++k) trow[k] = pk[k];
  }
  __syncthreads();
  {
    const int cc = tid >> 2, q = tid & 3;
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __nv_bfloat16 lo = tile[q * 16 + 2 * k][cc], hi = tile[q * 16 + 2 * k + 1][cc];
      pk[k] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.dfT + (size_t)(c0 + cc) * a.mp + r0 + q * 16);
    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  }
}

// dst[c][col0 + r] = src[r][c] for r < rows (rows: *rows_dev when given, else
// rows_host), zeros for rows..ceil64(rows) when pad is set. 64 x 64 tiles;
// cols a multiple of 64, src rows `cols` wide, dst rows `pitch` wide.
__global__ void __launch_bounds__(256) bwd_transpose_kernel(const __nv_bfloat16* __restrict__ src,
                                                            __nv_bfloat16* __restrict__ dst,
                                                            int rows_host,
                                                            const uint32_t* rows_dev, int cols,
                                                            size_t pitch, int col0, int pad,
                                                            WsHeader* hdr) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];
  if (status_bad(hdr)) return;
  const int rows = rows_dev ? (int)*rows_dev : rows_host;
  const int r0 = blockIdx.x * 64, c0 = blockIdx.y * 64;
  const int lim = pad ? (rows + 63) / 64 * 64 : rows;
  if (r0 >= lim) return;
  const int tid = threadIdx.x;
  {
    const int rr = tid >> 2, q = tid & 3;
    const int r = r0 + rr;
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (r < rows) {
      const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)r * cols + c0 + q * 16);
      v0 = s[0];
      v1 = s[1];
    }
    uint4* t = reinterpret_cast<uint4*>(&tile[rr][q * 16]);
    t[0] = v0;
    t[1] = v1;
  }
  __syncthreads();
  {
    const int cc = tid >> 2, q = tid & 3;
    const int rbase = r0 + q * 16;
    if (rbase >= lim) return;
    uint32_t pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __nv_bfloat16 lo = tile[q * 16 + 2 * k][cc], hi = tile[q * 16 + 2 * k + 1][cc];
      pk[k] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
    }
    __nv_bfloat16* drow = dst + (size_t)(c0 + cc) * pitch + col0 + rbase;
    if (rbase + 16 <= lim) {
      uint4* d4 = reinterpret_cast<uint4*>(drow);
      d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else {
      for (int k = 0; k < 16 && rbase + k < lim; ++k) drow[k] = tile[q * 16 + k][cc];
    }
  }
}

// --------------------------------------------------------------------- tcgen05 GEMM
constexpr int BM = 128, BK = 64;
constexpr int THREADS = 192;
constexpr int GROUP_M = 16;
constexpr int TILE16K = BM * BK * 2;  // one 128-row x 64-column bf16 tile

template <int MODE>
struct Cfg {
  // mode 0: A = x_a and df tiles; B = 64 W_gate + 64 W_up + 64 W_down^T rows
  static constexpr int STAGES = MODE == 0 ? 3 : 4;
  static constexpr int A_BYTES = MODE == 0 ? 2 * TILE16K : TILE16K;
  static constexpr int B_BYTES = MODE == 0 ? 3 * (TILE16K / 2) : 2 * TILE16K;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BN = MODE == 0 ? 64 : 256;   // output columns per tile
  static constexpr int NACC = 2;                    // accumulator sets in TMEM
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256;
};

struct GemmP {
  const uint32_t* m_dev;  // active rows (device)
  int m_host;             // mode 2: rows of A
  int k_blocks;           // modes 0, 1: K / 64
  int n_tiles, n_cols;
  size_t mp;              // row pitch of the transposed buffers (elements)
  int F;
  __nv_bfloat16* dgu;     // mode 0: [rows][2F]
  __nv_bfloat16* dguT;    // mode 0: [2F][mp]
  __nv_bfloat16* hT;      // mode 0: [F][mp]
  const float* dy;        // mode 1
  float* dx;              // mode 1
  const int32_t* idx;     // mode 1
  float* out0;            // mode 2: rows [0, split)
  float* out1;            // mode 2: rows [split, M)
  int split;
  WsHeader* hdr;
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mt, int& nt) {
  const int group = t / (GROUP_M * num_n);
  const int first_m = group * GROUP_M;
  const int gm = min(GROUP_M, num_m - first_m);
  const int idx = t - group * GROUP_M * num_n;
  mt = first_m + idx % gm;
  nt = idx / gm;
}

__device__ __forceinline__ float sigmoid(float g) { return 1.f / (1.f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    ffn_bwd_gemm_kernel(const __grid_constant__ CUtensorMap mA0,
                        const __grid_constant__ CUtensorMap mA1,
                        const __grid_constant__ CUtensorMap mB0,
                        const __grid_constant__ CUtensorMap mB1,
                        const __grid_constant__ CUtensorMap mB2, GemmP P) {
  using C = Cfg<MODE>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int s_abort;
  __shared__ int s_M, s_KB, s_m;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = P.hdr;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    s_abort = 0;
    const bool bad = status_bad(hdr);
    const int m = bad ? 0 : (int)*P.m_dev;
    s_m = m;
    s_M = bad ? 0 : (MODE == 2 ? P.m_host : m);
    s_KB = MODE == 2 ? (m + BK - 1) / BK : P.k_blocks;
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mA0);
    tma_prefetch_desc(&mB0);
    if (MODE == 0) {
      tma_prefetch_desc(&mA1);
      tma_prefetch_desc(&mB1);
      tma_prefetch_desc(&mB2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int M = s_M, KB = s_KB;
  const int num_m = (M + BM - 1) / BM;
  const int total = num_m * P.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, num_m, P.n_tiles, mt, nt);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, &s_abort, hdr, 0x9200u)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_expect_tx(&full[s], C::STAGE_BYTES);
          tma_load_2d(&mA0, &full[s], sa, kb * BK, mt * BM);
          if (MODE == 0) {
            tma_load_2d(&mA1, &full[s], sa + TILE16K, kb * BK, mt * BM);
            tma_load_2d(&mB0, &full[s], sb, kb * BK, nt * 64);
            tma_load_2d(&mB1, &full[s], sb + TILE16K / 2, kb * BK, nt * 64);
            tma_load_2d(&mB2, &full[s], sb + TILE16K, kb * BK, nt * 64);
          } else {
            tma_load_2d(&mB0, &full[s], sb, kb * BK, nt * 256);
          }
        }
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        for (int k = 0; k < STAGES; ++k) {
          const int j = it - 1 - k;
          if (j < 0) break;
          long long t0 = clock64();
          while (!mbar_try_wait(&full[j % STAGES], (j / STAGES) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc256 = make_idesc_bf16(BM, 256);
      constexpr uint32_t idesc128 = make_idesc_bf16(BM, 128);
      constexpr uint32_t idesc64 = make_idesc_bf16(BM, 64);
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tc) {
        const int b = C::NACC == 2 ? (tc & 1) : 0;
        const uint32_t aph = C::NACC == 2 ? ((tc >> 1) & 1) : (tc & 1);
        if (!mbar_wait(&acc_empty[b], aph ^ 1, &s_abort, hdr, 0x9300u)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + b * 256;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&full[s], (it / STAGES) & 1, &s_abort, hdr, 0x9400u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
            const uint64_t ad = make_sdesc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(b_addr + k * 32, 16, 1024);
            if (MODE == 0) {
              // gate|up (64 + 64 B rows) into columns 0-127 of the set, dh
              // (64 W_down^T rows) into 128-191
              umma_bf16(d0, ad, bd, idesc128, acc);
              const uint64_t ad1 = make_sdesc_sw128(a_addr + TILE16K + k * 32, 16, 1024);
              const uint64_t bd2 = make_sdesc_sw128(b_addr + TILE16K + k * 32, 16, 1024);
              umma_bf16(d0 + 128, ad1, bd2, idesc64, acc);
            } else {
              umma_bf16(d0, ad, bd, idesc256, acc);
            }
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int m_act = s_m;
    const int m_pad = (m_act + BK - 1) / BK * BK;
    int tc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      int mt, nt;
      tile_coords(t, num_m, P.n_tiles, mt, nt);
      const int b = C::NACC == 2 ? (tc & 1) : 0;
      const uint32_t aph = C::NACC == 2 ? ((tc >> 1) & 1) : (tc & 1);
      if (!mbar_wait_warp(&acc_full[b], aph, &s_abort, hdr, 0x9500u)) break;
      tc_fence_after();
      const int i = mt * BM + row;
      const bool live = i < M;
      const uint32_t tb = tmem_base + ((uint32_t)(wq * 32) << 16) + b * 256;
      if (MODE == 0) {
        const bool padrow = i < m_pad;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          uint32_t g[32], u[32], dh[32];
          tmem_ld32(tb + c, g);
          tmem_ld32(tb + 64 + c, u);
          tmem_ld32(tb + 128 + c, dh);
          tmem_ld_wait();
          const int n0 = nt * 64 + c;
          float dg[32], du[32], hh[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float gv = __uint_as_float(g[e]), uv = __uint_as_float(u[e]);
            const float dv = __uint_as_float(dh[e]);
            const float sg = sigmoid(gv);
            const float sl = gv * sg;
            hh[e] = live ? sl * uv : 0.f;
            du[e] = live ? dv * sl : 0.f;
            dg[e] = live ? dv * uv * sg * (1.f + gv * (1.f - sg)) : 0.f;
          }
          if (live) {
            uint4* dst_g = reinterpret_cast<uint4*>(P.dgu + (size_t)i * 2 * P.F + n0);
            uint4* dst_u = reinterpret_cast<uint4*>(P.dgu + (size_t)i * 2 * P.F + P.F + n0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              dst_g[q] = make_uint4(pack_bf16x2(dg[8 * q], dg[8 * q + 1]),
                                    pack_bf16x2(dg[8 * q + 2], dg[8 * q + 3]),
                                    pack_bf16x2(dg[8 * q + 4], dg[8 * q + 5]),
                                    pack_bf16x2(dg[8 * q + 6], dg[8 * q + 7]));
              dst_u[q] = make_uint4(pack_bf16x2(du[8 * q], du[8 * q + 1]),
                                    pack_bf16x2(du[8 * q + 2], du[8 * q + 3]),
                                    pack_bf16x2(du[8 * q + 4], du[8 * q + 5]),
                                    pack_bf16x2(du[8 * q + 6], du[8 * q + 7]));
            }
          }
          if (padrow) {
            // transposed copies: a warp writes 32 consecutive rows of each column
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const size_t col = (size_t)(n0 + e) * P.mp + i;
              P.dguT[col] = __float2bfloat16_rn(dg[e]);
              P.dguT[(size_t)P.F * P.mp + col] = __float2bfloat16_rn(du[e]);
              P.hT[col] = __float2bfloat16_rn(hh[e]);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t acc[32];
          tmem_ld32(tb + c, acc);
          tmem_ld_wait();
          const int n0 = nt * 256 + c;
          if (n0 >= P.n_cols || !live) continue;
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = KB > 0 ? __uint_as_float(acc[e]) : 0.f;
          float* dst;
          if (MODE == 1) {
            const int orig = P.idx[i];
            const float4* dyr =
                reinterpret_cast<const float4*>(P.dy + (size_t)orig * P.n_cols + n0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 r = dyr[q];
              v[4 * q] += r.x;
              v[4 * q + 1] += r.y;
              v[4 * q + 2] += r.z;
              v[4 * q + 3] += r.w;
            }
            dst = P.dx + (size_t)orig * P.n_cols + n0;
          } else {
            dst = i < P.split ? P.out0 + (size_t)i * P.n_cols + n0
                              : P.out1 + (size_t)(i - P.split) * P.n_cols + n0;
          }
          float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            d4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace fbwd

namespace {

int bwd_num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// 2D bf16 tensor map over [rows][cols] with row pitch `pitch` elements and a
// 64-column x box_rows box, 128-byte swizzle.
bool map2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch,
           uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {pitch * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tmap_16(m, base, 2, dims, strides, box, false);
}

template <int MODE>
cudaError_t launch_bwd_gemm(const char* name, const CUtensorMap& a0, const CUtensorMap& a1,
                            const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& b2,
                            const fbwd::GemmP& P, int max_tiles, cudaStream_t s) {
  auto k = fbwd::ffn_bwd_gemm_kernel<MODE>;
  const int smem = (int)fbwd::Cfg<MODE>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(max_tiles, bwd_num_sms()));
  return launch(name, k, dim3(grid), dim3(fbwd::THREADS), (size_t)smem, s, a0, a1, b0, b1, b2, P);
}

cudaError_t launch_transpose(const __nv_bfloat16* src, __nv_bfloat16* dst, int rows_host,
                             const uint32_t* rows_dev, int rows_max, int cols, size_t pitch,
                             int col0, int pad, WsHeader* hdr, cudaStream_t s) {
  if (rows_max <= 0) return cudaSuccess;
  const dim3 grid((rows_max + 63) / 64, cols / 64);
  return launch("bwd_transpose", fbwd::bwd_transpose_kernel, grid, dim3(256), 0, s, src, dst,
                rows_host, rows_dev, cols, pitch, col0, pad, hdr);
}

}  // namespace

cudaError_t launch_ffn_backward_tc(const FfnBwdArgs& a, cudaStream_t s) {
  using namespace fbwd;
  cudaError_t e;
  if ((e = launch("ffn_bwd_check", bwd_check_kernel, dim3(1), dim3(32), 0, s, a.hdr, a.fhdr)))
    return e;
  const int N = a.n_tokens, D = a.D, F = a.F;
  if (a.n_cubes > 0 &&
      (e = launch("ffn_bwd_skip", ffn_bwd_skip_kernel, dim3(a.n_cubes), dim3(256), 0, s, a)))
    return e;
  if ((e = launch("ffn_bwd_df", ffn_bwd_df_kernel, dim3((N + 63) / 64, D / 64), dim3(256), 0, s,
                  a)))
    return e;
  // x_a^T [D][mp] (zero-padded), W_down^T [F][D], [W_gate^T | W_up^T] [D][2F]
  if ((e = launch_transpose(a.xa, a.xaT, 0, a.m_active, N, D, a.mp, 0, 1, a.hdr, s))) return e;
  if ((e = launch_transpose(a.W_down, a.wdT, D, nullptr, D, F, (size_t)D, 0, 0, a.hdr, s)))
    return e;
  if ((e = launch_transpose(a.W_gate, a.wguT, F, nullptr, F, D, (size_t)2 * F, 0, 0, a.hdr, s)))
    return e;
  if ((e = launch_transpose(a.W_up, a.wguT, F, nullptr, F, D, (size_t)2 * F, F, 0, a.hdr, s)))
    return e;

  CUtensorMap mXa, mDf, mWg, mWu, mWdT, mDgu, mWguT, mDguT, mXaT, mDfT, mHT;
  const uint64_t mp = a.mp;
  if (!map2d(&mXa, a.xa, D, N, D, 128) || !map2d(&mDf, a.df, D, N, D, 128) ||
      !map2d(&mWg, a.W_gate, D, F, D, 64) || !map2d(&mWu, a.W_up, D, F, D, 64) ||
      !map2d(&mWdT, a.wdT, D, F, D, 64) || !map2d(&mDgu, a.dgu, 2 * F, N, 2 * F, 128) ||
      !map2d(&mWguT, a.wguT, 2 * F, D, 2 * F, 256) ||
      !map2d(&mDguT, a.dguT, mp, 2 * F, mp, 128) || !map2d(&mXaT, a.xaT, mp, D, mp, 256) ||
      !map2d(&mDfT, a.dfT, mp, D, mp, 128) || !map2d(&mHT, a.hT, mp, F, mp, 256))
    return cudaErrorInvalidValue;

  GemmP P{};
  P.m_dev = a.m_active;
  P.mp = a.mp;
  P.F = F;
  P.hdr = a.hdr;
  // dg, du, h
  P.k_blocks = D / 64;
  P.n_tiles = F / 64;
  P.n_cols = F;
  P.dgu = a.dgu;
  P.dguT = a.dguT;
  P.hT = a.hT;
  const int mtiles = (N + 127) / 128;
  if ((e = launch_bwd_gemm<0>("ffn_bwd_gemm_hdg_tc", mXa, mDf, mWg, mWu, mWdT, P,
                              mtiles * P.n_tiles, s)))
    return e;
  // dx of the computed rows
  P.k_blocks = 2 * F / 64;
  P.n_tiles = (D + 255) / 256;
  P.n_cols = D;
  P.dy = a.dy;
  P.dx = a.dx;
  P.idx = a.idx;
  if ((e = launch_bwd_gemm<1>("ffn_bwd_gemm_dx_tc", mDgu, mDgu, mWguT, mWguT, mWguT, P,
                              mtiles * P.n_tiles, s)))
    return e;
  // [dW_gate; dW_up] = [dg du]^T x_a
  P.m_host = 2 * F;
  P.n_tiles = (D + 255) / 256;
  P.n_cols = D;
  P.out0 = a.dWg;
  P.out1 = a.dWu;
  P.split = F;
  if ((e = launch_bwd_gemm<2>("ffn_bwd_gemm_dwgu_tc", mDguT, mDguT, mXaT, mXaT, mXaT, P,
                              ((2 * F + 127) / 128) * P.n_tiles, s)))
    return e;
  // dW_down = df^T h
  P.m_host = D;
  P.n_tiles = (F + 255) / 256;
  P.n_cols = F;
  P.out0 = a.dWd;
  P.out1 = a.dWd;
  P.split = D;
  return launch_bwd_gemm<2>("ffn_bwd_gemm_dwd_tc", mDfT, mDfT, mHT, mHT, mHT, P,
                            ((D + 127) / 128) * P.n_tiles, s);
}

}  // namespace adaspark

// AdaS-FFN GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   mode 0 (gate/up):  H[m, n] = silu(X_a W_gate^T)[m, n] * (X_a W_up^T)[m, n]
//                      (bf16 x bf16, fp32 accumulate; H stored as fp16, saturating)
//   mode 1 (down):     FFN_a = H W_down^T (fp16 x fp16 with W_down converted
//                      from bf16, fp32 accumulate); y[idx[m]] = x[idx[m]] + FFN_a[m];
//                      sums[cube(m)] += FFN_a[m] for active visual rows
//   mode 2 (linear):   out[m, n] = R[m, n] + (A W^T)[m, n] over every row m
//                      (bf16 x bf16, fp32 accumulate, bf16 out; R optional): the
//                      projections of a whole layer around AdaS-Attn
// (key design 3 of the AdaSpark note: the FFN runs only on the active tokens; the
// per-cube sums feed the mean compensation of the skipped ones).
//
// Persistent, warp-specialized kernel, one CTA per SM:
//   warp 0     TMA producer (128-byte swizzled K-major tiles, no multicast)
//   warp 1     TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-5  epilogue: tcgen05.ld of the fp32 accumulator, fused SwiGLU or
//              residual/scatter/cube-sum, direct global stores
// Tile 128 x 256 x 64, 4-stage smem ring, two 256-column TMEM accumulators so
// the epilogue of tile i overlaps the MMAs of tile i+1. In mode 0 the 256 B
// rows are 128 W_gate rows followed by the same 128 W_up rows, so one MMA chain
// yields gate (columns 0-127) and up (128-255) for the same outputs.
// H is kept in fp16 rather than bf16: its 3 extra mantissa bits keep the
// rounding error of the 18944-long down-projection sums well inside the
// output tolerance (bf16 H gave max-abs errors near 0.04 at that width).
#include <cuda_fp16.h>

#include <algorithm>

#include "ffn_kernels.h"

namespace adaspark {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int GROUP_M = 16;
constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;

struct Params {
  const uint32_t* m_active;  // device: active rows (modes 0, 1)
  int n_tiles;               // tiles along N
  int k_blocks;              // K / 64
  int n_cols;                // valid output columns (F for mode 0, D for mode 1, N for 2)
  FfnArgs f;                 // modes 0, 1; f.hdr is the status word in every mode
  // mode 2
  int m_rows;                // rows of A and out
  const __nv_bfloat16* R;    // residual [m_rows][n_cols] or null
  __nv_bfloat16* out;        // [m_rows][n_cols]
};

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mt, int& nt) {
  const int group = t / (GROUP_M * num_n);
  const int first_m = group * GROUP_M;
  const int gm = min(GROUP_M, num_m - first_m);
  const int idx = t - group * GROUP_M * num_n;
  mt = first_m + idx % gm;
  nt = idx / gm;
}

__device__ __forceinline__ float silu(float g) { return g / (1.f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Reduce 32 per-row values (one row per lane) to 32 per-column sums; lane l
// ends with the sum of column l (rows that should not count pass zeros).
__device__ __forceinline__ float butterfly_colsum(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    ffn_gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA,
                       const __grid_constant__ CUtensorMap mapB0,
                       const __grid_constant__ CUtensorMap mapB1, Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int s_abort;
  __shared__ int s_M;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = P.f.hdr;
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
    s_M = status_bad(hdr) ? 0 : (MODE == 2 ? P.m_rows : (int)*P.m_active);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB0);
    if (MODE == 0) tma_prefetch_desc(&mapB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  const int M = s_M;
  const int num_m = (M + BM - 1) / BM;
  const int total = num_m * P.n_tiles;
  const int KB = P.k_blocks;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, num_m, P.n_tiles, mt, nt);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, &s_abort, hdr, 0x6100u)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(&mapA, &full[s], sa, kb * BK, mt * BM);
          if (MODE == 0) {
            tma_load_2d(&mapB0, &full[s], sb, kb * BK, nt * 128);
            tma_load_2d(&mapB1, &full[s], sb + B_BYTES / 2, kb * BK, nt * 128);
          } else {
            tma_load_2d(&mapB0, &full[s], sb, kb * BK, nt * BN);
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
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN, false, MODE == 1);
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tc) {
        const int b = tc & 1;
        const uint32_t aph = (tc >> 1) & 1;
        if (!mbar_wait(&acc_empty[b], aph ^ 1, &s_abort, hdr, 0x6200u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, &s_abort, hdr, 0x6300u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = make_sdesc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(b_addr + k * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quadrant warp % 4
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    int tc = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      int mt, nt;
      tile_coords(t, num_m, P.n_tiles, mt, nt);
      const int b = tc & 1;
      const uint32_t aph = (tc >> 1) & 1;
      if (!mbar_wait_warp(&acc_full[b], aph, &s_abort, hdr, 0x6400u)) break;
      tc_fence_after();
      const int m = mt * BM + row;
      const bool live = m < M;
      const uint32_t tb = tmem_base + ((uint32_t)(wq * 32) << 16) + b * BN;
      if (MODE == 0) {
        __half* H = reinterpret_cast<__half*>(P.f.h);
        float hmax = 0.f;  // largest |h| of this row's slice, before the fp16 store
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tb + c, g);
          tmem_ld32(tb + 128 + c, u);
          tmem_ld_wait();
          const int n0 = nt * 128 + c;
          if (live && n0 < P.n_cols) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 =
                  silu(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              hmax = fmaxf(hmax, fmaxf(fabsf(h0), fabsf(h1)));
              pk[i] = pack_f16x2_sat(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(H + (size_t)m * P.f.F + n0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        // an activation beyond the fp16 range was stored saturated: the down
        // projection would then differ from the exact FFN
        if (hmax > 65504.f) set_status(hdr, ADASPARK_DEV_RANGE, 0x6500u);
      } else if (MODE == 2) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t acc[32];
          tmem_ld32(tb + c, acc);
          tmem_ld_wait();
          const int n0 = nt * BN + c;
          if (n0 >= P.n_cols || !live) continue;
          const size_t o = (size_t)m * P.n_cols + n0;
          float r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0.f;
          if (P.R) {
            const uint4* rs = reinterpret_cast<const uint4*>(P.R + o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 rv = rs[q];
              const __nv_bfloat162* rb = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(rb[e]);
                r[q * 8 + 2 * e] = f.x;
                r[q * 8 + 2 * e + 1] = f.y;
              }
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(r[2 * i] + __uint_as_float(acc[2 * i]),
                                r[2 * i + 1] + __uint_as_float(acc[2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(P.out + o);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      } else {
        const __nv_bfloat16* X = reinterpret_cast<const __nv_bfloat16*>(P.f.x);
        const int orig = live ? P.f.idx[m] : 0;
        const int cube = live ? P.f.row_cube[m] : -2;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t acc[32];
          tmem_ld32(tb + c, acc);
          tmem_ld_wait();
          const int n0 = nt * BN + c;
          if (n0 >= P.n_cols) continue;  // warp-uniform
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(acc[i]);
          if (live) {
            const uint4* xs = reinterpret_cast<const uint4*>(X + (size_t)orig * P.f.D + n0);
            float4* yd = reinterpret_cast<float4*>(P.f.y + (size_t)orig * P.f.D + n0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 xv = xs[q];
              const __nv_bfloat162* xb = reinterpret_cast<const __nv_bfloat162*>(&xv);
              float o[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 xf = __bfloat1622float2(xb[e]);
                o[2 * e] = xf.x + v[q * 8 + 2 * e];
                o[2 * e + 1] = xf.y + v[q * 8 + 2 * e + 1];
              }
              yd[2 * q] = make_float4(o[0], o[1], o[2], o[3]);
              yd[2 * q + 1] = make_float4(o[4], o[5], o[6], o[7]);
            }
          }
          if (!P.f.dense) {
            // per-cube column sums over this warp's rows, one segment per cube
            int mycube = (live && cube >= 0) ? cube : -1;
            unsigned todo = __ballot_sync(0xffffffffu, mycube >= 0);
            while (todo) {
              const int leader = __ffs(todo) - 1;
              const int cc = __shfl_sync(0xffffffffu, mycube, leader);
              const bool mine = mycube == cc;
              float w[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) w[i] = mine ? v[i] : 0.f;
              const float colsum = butterfly_colsum(w);
              atomicAdd(&P.f.sums[(size_t)cc * P.f.D + n0 + lane], colsum);
              todo &= ~__ballot_sync(0xffffffffu, mine);
            }
          }
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

}  // namespace gemm

static int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

static bool map_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                     uint32_t box_rows, bool fp16 = false) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tmap_16(m, base, 2, dims, strides, box, fp16);
}

// W_down bf16 -> fp16 (exact for 2^-14 <= |w| <= 65504; smaller magnitudes
// keep an absolute error below 2^-25; a weight beyond +-65504 would become
// infinite and sets ADASPARK_DEV_RANGE). 8 elements per thread.
__global__ void wdown_to_fp16_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst,
                                     size_t n8, WsHeader* hdr) {
  if (status_bad(hdr)) return;
  float wmax = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint4 o;
    uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(b[k]);
      wmax = fmaxf(wmax, fmaxf(fabsf(f.x), fabsf(f.y)));
      const __half2 hv = __floats2half2_rn(f.x, f.y);
      op[k] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    reinterpret_cast<uint4*>(dst)[i] = o;
  }
  if (wmax > 65504.f) set_status(hdr, ADASPARK_DEV_RANGE, 0x6600u);
}

cudaError_t launch_wdown_to_fp16(const FfnArgs& a, cudaStream_t s) {
  const size_t n8 = (size_t)a.D * a.F / 8;
  const int blocks = (int)std::min<size_t>((n8 + 255) / 256, (size_t)num_sms() * 8);
  return launch("wdown_to_fp16", wdown_to_fp16_kernel, dim3(blocks), dim3(256), 0, s,
                (const __nv_bfloat16*)a.W_down, (__half*)a.wd16, n8, a.hdr);
}

cudaError_t launch_ffn_gemm1_tc(const FfnArgs& a, cudaStream_t s) {
  CUtensorMap mA, mG, mU;
  if (!map_rows(&mA, a.xa, a.D, a.n_tokens, 128) || !map_rows(&mG, a.W_gate, a.D, a.F, 128) ||
      !map_rows(&mU, a.W_up, a.D, a.F, 128))
    return cudaErrorInvalidValue;
  gemm::Params P;
  P.m_active = &a.hdr->m_active;
  P.n_tiles = (a.F + 127) / 128;
  P.k_blocks = a.D / 64;
  P.n_cols = a.F;
  P.f = a;
  auto k = gemm::ffn_gemm_tc_kernel<0>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch("ffn_gemm1_tc", k, dim3(num_sms()), dim3(gemm::THREADS), gemm::SMEM_BYTES, s, mA,
                mG, mU, P);
}

cudaError_t launch_linear_tc(const __nv_bfloat16* A, const __nv_bfloat16* W,
                             const __nv_bfloat16* R, __nv_bfloat16* out, int M, int N, int K,
                             WsHeader* hdr, cudaStream_t s) {
  CUtensorMap mA, mW;
  if (!map_rows(&mA, A, K, M, 128) || !map_rows(&mW, W, K, N, 256)) return cudaErrorInvalidValue;
  gemm::Params P;
  P.m_active = nullptr;
  P.n_tiles = (N + 255) / 256;
  P.k_blocks = K / 64;
  P.n_cols = N;
  P.f = FfnArgs{};
  P.f.hdr = hdr;
  P.m_rows = M;
  P.R = R;
  P.out = out;
  auto k = gemm::ffn_gemm_tc_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = ((M + 127) / 128) * P.n_tiles;
  return launch("linear_tc", k, dim3(std::min(tiles, num_sms())), dim3(gemm::THREADS),
                gemm::SMEM_BYTES, s, mA, mW, mW, P);
}

cudaError_t launch_ffn_gemm2_tc(const FfnArgs& a, cudaStream_t s) {
  CUtensorMap mA, mD;
  if (!map_rows(&mA, a.h, a.F, a.n_tokens, 128, true) ||
      !map_rows(&mD, a.wd16, a.F, a.D, 256, true))
    return cudaErrorInvalidValue;
  gemm::Params P;
  P.m_active = &a.hdr->m_active;
  P.n_tiles = (a.D + 255) / 256;
  P.k_blocks = a.F / 64;
  P.n_cols = a.D;
  P.f = a;
  auto k = gemm::ffn_gemm_tc_kernel<1>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemm::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch("ffn_gemm2_tc", k, dim3(num_sms()), dim3(gemm::THREADS), gemm::SMEM_BYTES, s, mA,
                mD, mD, P);
}

}  // namespace adaspark

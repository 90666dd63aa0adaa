// Kernel argument blocks and host launchers of AdaS-FFN.
#pragma once

#include "common.cuh"
#include "host_util.h"
#include "layout.cuh"

namespace adaspark {

struct FfnArgs {
  const void* x;        // [N][D]
  const void* W_gate;   // [F][D]
  const void* W_up;     // [F][D]
  const void* W_down;   // [D][F]
  const int32_t* cube_ids;
  const int32_t* cube_offsets;
  float* y;             // [N][D] fp32
  float* norms;         // [n_vis]
  uint8_t* active;      // [N]
  int32_t* cube_count;  // [C]
  int32_t* cube_start;  // [C+1]
  int32_t* idx;         // [N]
  int32_t* row_cube;    // [N]
  void* xa;             // [N][D]
  void* h;              // [N][F]
  float* sums;          // [C][D]
  void* wd16;           // [D][F] fp16 copy of W_down (bf16 path)
  WsHeader* hdr;
  int n_tokens, n_vis, n_cubes, D, F;
  float p;
  int dense;
  int importance;       // ADASPARK_IMPORTANCE_*: share of ||x||, of ||x||^2, or softmax
};

cudaError_t launch_ffn_select(const FfnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_ffn_compact(const FfnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_ffn_gemm1_simt(const FfnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_ffn_gemm2_simt(const FfnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_ffn_gemm1_tc(const FfnArgs& a, cudaStream_t s);
cudaError_t launch_ffn_gemm2_tc(const FfnArgs& a, cudaStream_t s);
// out[M][N] = R[M][N] + A[M][K] W[N][K]^T (bf16; R may be null), tcgen05.
cudaError_t launch_linear_tc(const __nv_bfloat16* A, const __nv_bfloat16* W,
                             const __nv_bfloat16* R, __nv_bfloat16* out, int M, int N, int K,
                             WsHeader* hdr, cudaStream_t s);
cudaError_t launch_ffn_compensate(const FfnArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_wdown_to_fp16(const FfnArgs& a, cudaStream_t s);

}  // namespace adaspark

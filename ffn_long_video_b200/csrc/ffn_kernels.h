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
  int32_t* skip;        // [n_vis] skipped visual rows, cube by cube
  WsHeader* hdr;
  int n_tokens, n_vis, n_cubes, D, F;
  float p;
  int dense;
  int importance;       // ADASPARK_IMPORTANCE_*: share of ||x||, of ||x||^2, or softmax
};

// Backward of AdaS-FFN (active set from a forward call held fixed).
struct FfnBwdArgs {
  const __nv_bfloat16* W_gate;  // [F][D]
  const __nv_bfloat16* W_up;    // [F][D]
  const __nv_bfloat16* W_down;  // [D][F]
  const int32_t* cube_offsets;
  const float* dy;              // [N][D]
  float* dx;                    // [N][D]
  float* dWg;                   // [F][D]
  float* dWu;                   // [F][D]
  float* dWd;                   // [D][F]
  // from the forward workspace
  const WsHeader* fhdr;
  const uint32_t* m_active;     // active rows (visual + text)
  const uint8_t* active;        // [N]
  const int32_t* cube_count;    // [C]
  const int32_t* idx;           // [N] compacted rows -> token
  const int32_t* row_cube;      // [N] cube of each compacted row (-1 text)
  const __nv_bfloat16* xa;      // [N][D] compacted x
  // backward workspace
  WsHeader* hdr;
  float* gsum;                  // [C][D] skipped-row dy sums / active count
  __nv_bfloat16* df;            // [N][D]
  __nv_bfloat16* dfT;           // [D][mp]
  __nv_bfloat16* xaT;           // [D][mp]
  __nv_bfloat16* wdT;           // [F][D]
  __nv_bfloat16* wguT;          // [D][2F]
  __nv_bfloat16* dgu;           // [N][2F]
  __nv_bfloat16* dguT;          // [2F][mp]
  __nv_bfloat16* hT;            // [F][mp]
  int n_tokens, n_vis, n_cubes, D, F;
  size_t mp;                    // pitch of the transposed buffers: N rounded up to 64
};
cudaError_t launch_ffn_backward_tc(const FfnBwdArgs& a, cudaStream_t s);

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

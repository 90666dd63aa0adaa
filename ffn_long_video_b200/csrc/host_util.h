// Host-side helpers: launch accounting and event timing, tensor-map encoding,
// argument checks. Used by the .cu files that launch kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>

#include "adaspark.h"

namespace adaspark {

// Records a begin/end event pair around a launch when the timer is enabled and
// counts every launch.
void timer_begin(const char* name, cudaStream_t s);
void timer_end(cudaStream_t s);
void count_launch();

#ifdef __CUDACC__
template <typename... KArgs, typename... Args>
inline cudaError_t launch(const char* name, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                          size_t smem, cudaStream_t s, Args&&... args) {
  timer_begin(name, s);
  kernel<<<grid, block, smem, s>>>(static_cast<KArgs>(args)...);
  cudaError_t e = cudaGetLastError();
  timer_end(s);
  count_launch();
  return e;
}
#endif

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
// 2D or 3D maps of 16-bit elements (bf16 or fp16), 128-byte swizzle, zero fill
// out of bounds. dims/strides are innermost first; strides in bytes for dims
// 1.. (dim 0 is dense).
bool encode_tmap_16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool fp16);
inline bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                             const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tmap_16(map, base, rank, dims, strides_bytes, box, false);
}

inline bool p_valid(float p) { return p > 0.0f && p <= 1.0f; }  // false for NaN

inline bool aligned(const void* ptr, size_t a) {
  return (reinterpret_cast<uintptr_t>(ptr) % a) == 0;
}

int device_is_sm100();  // 1 yes, 0 no, -1 query failed

}  // namespace adaspark

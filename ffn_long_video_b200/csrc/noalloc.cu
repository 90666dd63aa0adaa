// AdaS-Attn for callers that cannot allocate device memory.
//
// adaspark_cube_attn needs a caller-provided workspace. Some callers have no way
// to provide one at the point where they run the layer: a plugin that its host
// framework hands only input and output buffers, a serving loop that must not
// allocate (allocation can synchronize the device and fragment a fixed memory
// budget), or a process whose device memory is owned entirely by another
// allocator. adaspark_cube_attn_noalloc runs the same kernels with the
// workspace placed in a fixed-size array that the library itself holds in
// device memory for as long as it is loaded.
#include <cuda_runtime.h>

#include <mutex>

#include "adaspark.h"

namespace {

// The scratch array. Every GPU on which the library's device code is loaded
// reserves ADASPARK_NOALLOC_SCRATCH_BYTES for it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ADASPARK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The host-side
// symbol is only a stand-in: the address is looked up once per device, with
// that device current, and cached for the life of the process (a
// cudaDeviceReset would invalidate it; the header says so).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ADASPARK_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return ADASPARK_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ADASPARK_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ADASPARK_OK;
}

}  // namespace

namespace adaspark {
int cube_attn_single_walk(const void* Q, const void* K, const void* V, int dtype,
                          const int32_t* cube_ids, const int32_t* cube_offsets, int n_cubes,
                          int n_vis, int n_tokens, int hq, int hkv, int d, float p, void* out,
                          void* workspace, size_t workspace_bytes, void* stream);
size_t cube_attn_single_walk_workspace(int n_tokens, int n_vis, int n_cubes, int hq, int hkv,
                                       int d, int dtype);
}  // namespace adaspark

extern "C" int adaspark_cube_attn_noalloc(const void* Q, const void* K, const void* V, int dtype,
                                          const int32_t* cube_ids, const int32_t* cube_offsets,
                                          int n_cubes, int n_vis, int n_tokens, int hq, int hkv,
                                          int d, float p, void* out, void* stream) {
  // the common layout alone: this entry point always runs the single walk
  const size_t need =
      adaspark::cube_attn_single_walk_workspace(n_tokens, n_vis, n_cubes, hq, hkv, d, dtype);
  if (need == 0) return ADASPARK_EINVAL;                       // invalid sizes
  if (need > (size_t)ADASPARK_NOALLOC_SCRATCH_BYTES) return ADASPARK_EINVAL;  // too large
  // the device check comes first, so that a device without this library's
  // device code reports ADASPARK_EUNSUPPORTED rather than a failed lookup
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ADASPARK_ECUDA;
  int rc = adaspark_device_check(dev);
  if (rc != ADASPARK_OK) return rc;
  void* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc != ADASPARK_OK) return rc;
  // adaspark_cube_attn clears the parts of the workspace that must start at
  // zero (status word and counters) at the start of every call.
  return adaspark::cube_attn_single_walk(Q, K, V, dtype, cube_ids, cube_offsets, n_cubes, n_vis,
                                         n_tokens, hq, hkv, d, p, out, scratch,
                                         (size_t)ADASPARK_NOALLOC_SCRATCH_BYTES, stream);
}

// Host-side helpers: status strings, launch count, event timer, tensor maps.
#include "host_util.h"

#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

namespace adaspark {

namespace {
std::atomic<uint64_t> g_launches{0};
bool g_timer_on = false;

struct Pending {
  std::string name;
  cudaEvent_t begin, end;
};
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free_events;
std::string g_cur_name;
cudaEvent_t g_cur_begin = nullptr;

cudaEvent_t get_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void timer_begin(const char* name, cudaStream_t s) {
  if (!g_timer_on) return;
  g_cur_name = name;
  g_cur_begin = get_event();
  if (g_cur_begin) cudaEventRecord(g_cur_begin, s);
}

void timer_end(cudaStream_t s) {
  if (!g_timer_on || !g_cur_begin) return;
  cudaEvent_t e = get_event();
  if (!e) return;
  cudaEventRecord(e, s);
  g_pending.push_back({g_cur_name, g_cur_begin, e});
  g_cur_begin = nullptr;
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_tmap_16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool fp16) {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return false;
    fn = reinterpret_cast<EncodeFn>(p);
  }
  cuuint64_t d[3];
  cuuint64_t st[2];
  cuuint32_t bx[3];
  cuuint32_t es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides_bytes[i];
  CUresult r = fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  (cuuint32_t)rank, const_cast<void*>(base),
                  d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_is_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return -1;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return -1;
  return (major == 10 && minor == 0) ? 1 : 0;
}

}  // namespace adaspark

using namespace adaspark;

extern "C" {

const char* adaspark_status_string(int status) {
  switch (status) {
    case ADASPARK_OK: return "ok";
    case ADASPARK_EINVAL: return "invalid argument";
    case ADASPARK_ECUDA: return "CUDA error";
    case ADASPARK_EUNSUPPORTED: return "unsupported device or shape";
    case ADASPARK_EDEVICE: return "device-side check failed";
    default: return "unknown status";
  }
}

int adaspark_timer_enable(int on) {
  g_timer_on = on != 0;
  return ADASPARK_OK;
}

int adaspark_timer_read(adaspark_kernel_time* out, int max, int* n_out) {
  if (n_out) *n_out = 0;
  if (max < 0 || (max > 0 && !out)) return ADASPARK_EINVAL;
  std::vector<adaspark_kernel_time> acc;
  int rc = ADASPARK_OK;
  for (auto& p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.end) != cudaSuccess ||
        cudaEventElapsedTime(&ms, p.begin, p.end) != cudaSuccess)
      rc = ADASPARK_ECUDA;
    adaspark_kernel_time* slot = nullptr;
    for (auto& a : acc)
      if (std::strncmp(a.name, p.name.c_str(), sizeof(a.name)) == 0) slot = &a;
    if (!slot) {
      adaspark_kernel_time t;
      std::memset(&t, 0, sizeof(t));
      std::strncpy(t.name, p.name.c_str(), sizeof(t.name) - 1);
      acc.push_back(t);
      slot = &acc.back();
    }
    slot->launches += 1;
    slot->total_ms += ms;
    g_free_events.push_back(p.begin);
    g_free_events.push_back(p.end);
  }
  g_pending.clear();
  int n = 0;
  for (auto& a : acc) {
    if (n < max) out[n] = a;
    ++n;
  }
  if (n_out) *n_out = n < max ? n : max;
  return rc;
}

uint64_t adaspark_launch_count(void) { return g_launches.load(); }

int adaspark_device_check(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return ADASPARK_ECUDA;
  return (major == 10 && minor == 0) ? ADASPARK_OK : ADASPARK_EUNSUPPORTED;
}

}  // extern "C"

// Sort-free Top-p cut of one row of cube scores (AdaS-Attn key design 2:
// S_i = {j | p_j in Top-p(P_i, p)}), one thread per row, in two streaming passes
// over the scores (which the caller recomputes bit-identically in pass 2).
//
// Scores enter in log2 units, z_j = (q . kbar_j) * log2(e) / sqrt(d), so that
// P_j is proportional to 2^z_j. Pass 1 keeps a mass histogram of 2^z over bins
// of width 1/kR log2-units, in a window of kB bins below the running maximum
// (older bins fold into a tail scalar when the maximum moves up). After pass 1
// the bin holding the cut is known: walking down from the top, it is the first
// bin at which the cumulative mass reaches p * Z. Pass 2 marks every element of
// a higher bin as selected and collects the elements of the cut bin; sorting
// that short list by (z descending, index ascending) gives the exact cut.
// This reproduces "smallest prefix of the (P desc, index asc) order whose
// cumulative mass reaches p" up to fp32 rounding of the masses.
#pragma once

#include <limits.h>

#include "common.cuh"

namespace adaspark {
namespace sel {

constexpr int kR = 8;                 // bins per log2 unit
constexpr float kInvR = 1.0f / kR;
constexpr int kB = 64;                // bins in the window (8 log2 units)
constexpr int kL = 24;                // cut-bin list entries kept in shared memory
constexpr int kNone = INT_MIN;        // row without candidates
constexpr int kTail = INT_MIN + 1;    // the cut lies below the window
constexpr int kRows = 128;

// 2^x on the special-function unit (relative error below 2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Smem {
  float hist[kB][kRows];
  float lz[kL][kRows];
  uint16_t lj[kL][kRows];
};

struct Pool {
  float* z;        // [rows][C]
  int32_t* j;      // [rows][C]
  int rows;
  int C;
};

struct RowSel {
  Smem* sm;
  int tid;
  int bmax;
  float tail;
  int bstar;
  float need;
  int n;
  float* gz;
  int32_t* gj;
  bool lost;

  __device__ void init(Smem* s, int t) {
    sm = s;
    tid = t;
    bmax = kNone;
    tail = 0.f;
    bstar = kNone;
    need = 0.f;
    n = 0;
    gz = nullptr;
    gj = nullptr;
    lost = false;
#pragma unroll 8
    for (int k = 0; k < kB; ++k) sm->hist[k][tid] = 0.f;
  }

  __device__ __noinline__ void shift(int b) {
    if (bmax == kNone) {
      bmax = b;
      return;
    }
    int nleave = b - bmax;
    if (nleave > kB) nleave = kB;
    tail *= exp2f((float)(bmax - b) * kInvR);
    const int k0 = bmax - kB + 1;
    for (int i = 0; i < nleave; ++i) {
      const int k = k0 + i;
      float& hv = sm->hist[k & (kB - 1)][tid];
      if (hv != 0.f) {
        tail += hv * exp2f((float)(k - b) * kInvR);
        hv = 0.f;
      }
    }
    bmax = b;
  }

  __device__ __forceinline__ void pass1(float z) {
    const int b = __float2int_rd(z * (float)kR);
    if (b > bmax) shift(b);
    if (b > bmax - kB)
      sm->hist[b & (kB - 1)][tid] += fast_exp2(z - (float)b * kInvR);
    else
      tail += fast_exp2(z - (float)bmax * kInvR);
  }

  __device__ void finish1(float p) {
    if (bmax == kNone) {
      bstar = kNone;
      return;
    }
    float Z = tail;
    for (int i = kB - 1; i >= 0; --i) {
      const int k = bmax - i;
      Z += sm->hist[k & (kB - 1)][tid] * exp2f(-(float)i * kInvR);
    }
    const float target = p * Z;
    float cum = 0.f;
    bstar = kTail;
    for (int i = 0; i < kB; ++i) {
      const int k = bmax - i;
      const float m = sm->hist[k & (kB - 1)][tid] * exp2f(-(float)i * kInvR);
      if (cum + m >= target) {
        bstar = k;
        break;
      }
      cum += m;
    }
    need = target - cum;
  }

  __device__ __noinline__ void push(float z, int j, WsHeader* hdr, const Pool& pool) {
    if (!gz) {
      if (n < kL) {
        sm->lz[n][tid] = z;
        sm->lj[n][tid] = (uint16_t)j;
        ++n;
        return;
      }
      const unsigned slot = atomicAdd(&hdr->pool_next, 1u);
      if (slot >= (unsigned)pool.rows) {
        if (!lost) set_status(hdr, ADASPARK_DEV_POOL_FULL, 0x5000u);
        lost = true;
        return;
      }
      gz = pool.z + (size_t)slot * pool.C;
      gj = pool.j + (size_t)slot * pool.C;
      for (int i = 0; i < n; ++i) {
        gz[i] = sm->lz[i][tid];
        gj[i] = sm->lj[i][tid];
      }
    }
    if (n < pool.C) {
      gz[n] = z;
      gj[n] = j;
      ++n;
    }
  }

  // Returns true when z lies above the cut bin (selected outright); pushes the
  // elements of the cut bin to the list.
  __device__ __forceinline__ bool pass2(float z, int j, WsHeader* hdr, const Pool& pool) {
    const int b = __float2int_rd(z * (float)kR);
    bool above, cand;
    if (bstar == kTail) {
      above = b > bmax - kB;
      cand = !above;
    } else {
      above = b > bstar;
      cand = (b == bstar);
    }
    if (cand) push(z, j, hdr, pool);
    return above;
  }

  __device__ __forceinline__ float lzv(int i) const { return gz ? gz[i] : sm->lz[i][tid]; }
  __device__ __forceinline__ int ljv(int i) const { return gz ? gj[i] : (int)sm->lj[i][tid]; }
  __device__ __forceinline__ void lset(int i, float z, int j) {
    if (gz) {
      gz[i] = z;
      gj[i] = j;
    } else {
      sm->lz[i][tid] = z;
      sm->lj[i][tid] = (uint16_t)j;
    }
  }

  // Sort the cut-bin list by (z desc, j asc) and return how many of its leading
  // entries complete the Top-p set.
  __device__ int resolve() {
    if (bstar == kNone || n == 0) return 0;
    if (!gz) {
      for (int i = 1; i < n; ++i) {  // insertion sort (stable; entries arrive in j order)
        const float z = sm->lz[i][tid];
        const uint16_t j = sm->lj[i][tid];
        int k = i - 1;
        while (k >= 0 && sm->lz[k][tid] < z) {
          sm->lz[k + 1][tid] = sm->lz[k][tid];
          sm->lj[k + 1][tid] = sm->lj[k][tid];
          --k;
        }
        sm->lz[k + 1][tid] = z;
        sm->lj[k + 1][tid] = j;
      }
    } else {
      // shell sort on the full key (not stable, so the index breaks ties)
      for (int gap = n / 2; gap > 0; gap /= 2) {
        for (int i = gap; i < n; ++i) {
          const float z = gz[i];
          const int j = gj[i];
          int k = i;
          while (k >= gap && (gz[k - gap] < z || (gz[k - gap] == z && gj[k - gap] > j))) {
            gz[k] = gz[k - gap];
            gj[k] = gj[k - gap];
            k -= gap;
          }
          gz[k] = z;
          gj[k] = j;
        }
      }
    }
    const float ref = (float)bmax * kInvR;
    float cum = 0.f;
    for (int i = 0; i < n; ++i) {
      cum += exp2f(lzv(i) - ref);
      if (cum >= need) return i + 1;
    }
    return n;
  }
};

}  // namespace sel

// ---------------------------------------------------------------------------
// Shared tile epilogue: compact the cube columns with any row bit into the
// tile's ascending list. 128 threads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void compact_tile_list(const uint32_t* tmask, uint16_t* list, int32_t* count, int c_hi,
                                  int* s_wcnt, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  int total = 0;
  for (int base = 0; base <= c_hi; base += 128) {
    const int j = base + tid;
    bool nz = false;
    if (j <= c_hi) {
      const uint4 w = __ldcg(reinterpret_cast<const uint4*>(tmask + (size_t)j * 4));
      nz = (w.x | w.y | w.z | w.w) != 0u;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, nz);
    if (lane == 0) s_wcnt[warp] = __popc(bal);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int before = total;
    for (int w = 0; w < warp; ++w) before += s_wcnt[w];
    const int chunk_total = s_wcnt[0] + s_wcnt[1] + s_wcnt[2] + s_wcnt[3];
    if (nz) list[before + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)j;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    total += chunk_total;
  }
  if (tid == 0) *count = total;
}

}  // namespace adaspark

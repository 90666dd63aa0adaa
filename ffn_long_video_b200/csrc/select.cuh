// Sort-free Top-p cut of one row of cube scores (AdaS-Attn key design 2:
// S_i = {j | p_j in Top-p(P_i, p)}), one thread per row, in streaming passes
// over the scores (which the caller recomputes bit-identically every pass).
//
// Scores enter in log2 units, z_j = (q . kbar_j) * log2(e) / sqrt(d), so that
// P_j is proportional to 2^z_j. The order is (z descending, index ascending).
//  pass 1  mass histogram of 2^z over bins of width 1/kR log2-units, in a window
//          of kB bins below the running maximum (older bins fold into a tail
//          scalar when the maximum moves up). Walking down from the top, the
//          cut bin is the first at which the cumulative mass reaches p * Z.
//  pass 2  every element of a higher bin is selected outright; the elements of
//          the cut bin are offered to a per-row list that keeps the kL best in
//          the (z desc, index asc) order. Walking that list in order until the
//          cumulative mass reaches p * Z ends the cut.
//  more    if the cut lies beyond the kL best elements of the cut bin, those
//          kL are selected, the required mass is reduced by theirs, and another
//          pass collects the next kL below the last key; repeated until the cut
//          is found (bounded by the size of the cut bin).
// This reproduces "smallest prefix of the (P desc, index asc) order whose
// cumulative mass reaches p" up to fp32 rounding of the masses, for any score
// distribution (ties included), without memory beyond the per-row list.
#pragma once

#include <limits.h>

#include "common.cuh"

namespace adaspark {
namespace sel {

constexpr int kR = 8;                 // bins per log2 unit
constexpr float kInvR = 1.0f / kR;
constexpr int kB = 64;                // bins in the window (8 log2 units)
constexpr int kL = 24;                // list entries per row (shared memory)
constexpr int kNone = INT_MIN;        // row without candidates
constexpr int kTail = INT_MIN + 1;    // the cut lies below the window
constexpr int kRows = 128;

// 2^x on the special-function unit (relative error below 2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (z1, j1) comes before (z2, j2) in the (z desc, index asc) order.
__device__ __forceinline__ bool before(float z1, int j1, float z2, int j2) {
  return z1 > z2 || (z1 == z2 && j1 < j2);
}

struct Smem {
  float hist[kB][kRows];
  float lz[kL][kRows];
  uint16_t lj[kL][kRows];
  float wbin[kB];          // 2^(-i/kR), i = 0..kB-1 (filled by init_table)
};

// Fill the bin-weight table once per CTA (threads [0, kB) of the caller).
__device__ __forceinline__ void init_table(Smem* s, int tid) {
  if (tid < kB) s->wbin[tid] = exp2f(-(float)tid * kInvR);
}

// Out-of-line cold paths take and return plain values, so that the per-row
// state below stays in registers (a member function called out of line would
// force the whole state object into local memory).

// The running maximum moved up from bin bmax to bin b: fold the bins leaving
// the window into the tail and rescale it; returns the new tail.
static __device__ __noinline__ float shift_window(float* hist_col, int bmax, int b, float tail) {
  int nleave = b - bmax;
  if (nleave > kB) nleave = kB;
  tail *= exp2f((float)(bmax - b) * kInvR);
  const int k0 = bmax - kB + 1;
  for (int i = 0; i < nleave; ++i) {
    const int k = k0 + i;
    float& hv = hist_col[(k & (kB - 1)) * kRows];
    if (hv != 0.f) {
      tail += hv * exp2f((float)(k - b) * kInvR);
      hv = 0.f;
    }
  }
  return tail;
}

// Insertion sort of list entries [0, n) into the (z desc, index asc) order.
static __device__ __noinline__ void sort_entries(float* lz_col, uint16_t* lj_col, int n) {
  for (int i = 1; i < n; ++i) {
    const float z = lz_col[i * kRows];
    const uint16_t j = lj_col[i * kRows];
    int k = i;
    while (k > 0 && before(z, j, lz_col[(k - 1) * kRows], (int)lj_col[(k - 1) * kRows])) {
      lz_col[k * kRows] = lz_col[(k - 1) * kRows];
      lj_col[k * kRows] = lj_col[(k - 1) * kRows];
      --k;
    }
    lz_col[k * kRows] = z;
    lj_col[k * kRows] = j;
  }
}

// Offer (z, j) to a list holding the kL best keys seen so far; state packs the
// entry count (bits 0..7) and an "in order" flag (bit 8). Entries are appended
// unsorted until the list is full; it is sorted once then, and later offers
// replace the last entry by sorted insertion. Returns the new state.
static __device__ __noinline__ int offer_entry(float* lz_col, uint16_t* lj_col, int state, float z,
                                        int j) {
  int n = state & 0xff;
  bool sorted = (state >> 8) & 1;
  if (n < kL) {
    lz_col[n * kRows] = z;
    lj_col[n * kRows] = (uint16_t)j;
    return (n + 1);  // not in order any more
  }
  if (!sorted) sort_entries(lz_col, lj_col, n);
  if (before(z, j, lz_col[(kL - 1) * kRows], (int)lj_col[(kL - 1) * kRows])) {
    int pos = kL - 1;
    while (pos > 0 && before(z, j, lz_col[(pos - 1) * kRows], (int)lj_col[(pos - 1) * kRows])) {
      lz_col[pos * kRows] = lz_col[(pos - 1) * kRows];
      lj_col[pos * kRows] = lj_col[(pos - 1) * kRows];
      --pos;
    }
    lz_col[pos * kRows] = z;
    lj_col[pos * kRows] = (uint16_t)j;
  }
  return kL | (1 << 8);
}

struct RowSel {
  float* hist_col;   // &hist[0][row]
  float* lz_col;     // &lz[0][row]
  uint16_t* lj_col;  // &lj[0][row]
  const float* wbin;
  int bmax;
  float tail;
  int bstar;
  float need;
  int lstate;     // list entries | (in order << 8)
  bool open;      // cut not found yet
  bool bounded;   // only keys after (bz, bj) are offered (extra passes)
  float bz;
  int bj;

  __device__ __forceinline__ void init(Smem* s, int t) {
    hist_col = &s->hist[0][t];
    lz_col = &s->lz[0][t];
    lj_col = &s->lj[0][t];
    wbin = s->wbin;
    bmax = kNone;
    tail = 0.f;
    bstar = kNone;
    need = 0.f;
    lstate = 1 << 8;
    open = false;
    bounded = false;
    bz = 0.f;
    bj = 0;
#pragma unroll 8
    for (int k = 0; k < kB; ++k) hist_col[k * kRows] = 0.f;
  }

  __device__ __forceinline__ void raise_max(int b) {
    if (bmax == kNone) {
      bmax = b;
      return;
    }
    tail = shift_window(hist_col, bmax, b, tail);
    bmax = b;
  }

  __device__ __forceinline__ void pass1(float z) {
    const int b = __float2int_rd(z * (float)kR);
    if (b > bmax) raise_max(b);
    if (b > bmax - kB)
      hist_col[(b & (kB - 1)) * kRows] += fast_exp2(z - (float)b * kInvR);
    else
      tail += fast_exp2(z - (float)bmax * kInvR);
  }

  // Eight scores at once (the hot loop of pass 1): one running-maximum check
  // for the group, then the bin updates. `valid` bit c enables z[c].
  __device__ __forceinline__ void pass1x8(const float (&z)[8], unsigned valid) {
    int b[8];
    int bm = kNone;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      b[c] = __float2int_rd(z[c] * (float)kR);
      if ((valid >> c) & 1u) bm = max(bm, b[c]);
    }
    if (bm > bmax) raise_max(bm);
    const int lo = bmax - kB;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (!((valid >> c) & 1u)) continue;
      if (b[c] > lo)
        hist_col[(b[c] & (kB - 1)) * kRows] += fast_exp2(z[c] - (float)b[c] * kInvR);
      else
        tail += fast_exp2(z[c] - (float)bmax * kInvR);
    }
  }

  __device__ __forceinline__ void finish1(float p) {
    if (bmax == kNone) {
      bstar = kNone;
      open = false;
      return;
    }
    float Z = tail;
    for (int i = kB - 1; i >= 0; --i) Z += hist_col[((bmax - i) & (kB - 1)) * kRows] * wbin[i];
    const float target = p * Z;
    float cum = 0.f;
    bstar = kTail;
    for (int i = 0; i < kB; ++i) {
      const float m = hist_col[((bmax - i) & (kB - 1)) * kRows] * wbin[i];
      if (cum + m >= target) {
        bstar = bmax - i;
        break;
      }
      cum += m;
    }
    need = target - cum;
    open = true;
  }

  __device__ __forceinline__ void offer(float z, int j) {
    if (bounded && !before(bz, bj, z, j)) return;
    lstate = offer_entry(lz_col, lj_col, lstate, z, j);
  }

  __device__ __forceinline__ bool in_cut_bin(int b) const {
    return bstar == kTail ? b <= bmax - kB : b == bstar;
  }

  // Emission pass: true when z lies above the cut bin (selected outright);
  // elements of the cut bin go to the list.
  __device__ __forceinline__ bool pass2(float z, int j) {
    const int b = __float2int_rd(z * (float)kR);
    const bool above = bstar == kTail ? b > bmax - kB : b > bstar;
    if (open && in_cut_bin(b)) offer(z, j);
    return above;
  }

  // Extra pass for a row whose cut is still open.
  __device__ __forceinline__ void pass_more(float z, int j) {
    if (!open) return;
    const int b = __float2int_rd(z * (float)kR);
    if (in_cut_bin(b)) offer(z, j);
  }

  // After a pass over the cut bin: how many leading list entries are selected.
  // Closes the cut when reached (or when the bin is exhausted); otherwise all
  // kL entries are taken and the next pass starts after the last of them.
  __device__ __forceinline__ int settle() {
    if (!open) return 0;
    const int n = lstate & 0xff;
    if (!((lstate >> 8) & 1)) sort_entries(lz_col, lj_col, n);
    lstate = n | (1 << 8);
    const float ref = (float)bmax * kInvR;
    float cum = 0.f;
    for (int i = 0; i < n; ++i) {
      cum += fast_exp2(lz_col[i * kRows] - ref);
      if (cum >= need) {
        open = false;
        return i + 1;
      }
    }
    if (n < kL) {  // the whole cut bin was offered: rounding left need unmet
      open = false;
      return n;
    }
    need -= cum;
    bounded = true;
    bz = lz_col[(kL - 1) * kRows];
    bj = (int)lj_col[(kL - 1) * kRows];
    return n;
  }

  __device__ __forceinline__ int list_j(int i) const { return (int)lj_col[i * kRows]; }
  __device__ __forceinline__ void reset_list() { lstate = 1 << 8; }
};

}  // namespace sel

// ---------------------------------------------------------------------------
// Shared tile epilogue: compact the cube columns with any row bit into the
// tile's ascending list. 128 threads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void compact_tile_list(const uint32_t* tmask, uint16_t* list,
                                                  int32_t* count, int c_hi, int* s_wcnt, int tid) {
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

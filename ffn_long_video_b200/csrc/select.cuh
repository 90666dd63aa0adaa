// Sort-free Top-p cut of one row of cube scores (AdaS-Attn key design 2:
// S_i = {j | p_j in Top-p(P_i, p)}), one thread per row, in streaming passes
// over the scores (which the caller recomputes bit-identically every pass).
//
// Scores enter raw (s_j = q . kbar_j); z_j = s_j * log2(e) / sqrt(d) is the
// score in log2 units, so P_j is proportional to 2^z_j. The order is (s desc,
// index asc).
//  pass 1  mass histogram of 2^z over bins of 1/8 octave (keys of mass_key),
//          in a window of kB bins below the running maximum; the lowest bin
//          also takes every score below the window (bins leaving the window
//          fold into it when the maximum moves up). Walking down from the top,
//          the cut bin is the first at which the cumulative mass reaches p * Z.
//  pass 2  every score of a higher bin is selected outright; the scores of the
//          cut bin are appended to a per-row list of kL entries. Sorted into
//          the (s desc, index asc) order and walked until the cumulative mass
//          reaches p * Z, the list ends the cut. A cut bin larger than the
//          list turns the row's storage into a finer histogram of the cut bin
//          (64 bins of 1/512 octave; for the window's lowest bin, the next 8
//          octaves below it in 1/8-octave bins), filled for the rest of the
//          pass from the list's entries and the bin's remaining scores.
//  pass 3  (rows with a finer histogram) the fine cut bin is found the same
//          way; scores of fine bins above it are selected outright, and the
//          scores of the fine cut bin are listed, sorted and walked as above.
//  more    if the cut lies beyond the kL best scores of the (fine) cut bin,
//          those kL are selected, the required mass is reduced by theirs, and
//          another pass collects the next kL below the last one; repeated
//          until the cut is found (bounded by the size of that bin). With the
//          finer histogram this is rare: a crowded cut bin costs one pass more
//          instead of one pass per kL of its scores.
// This reproduces "smallest prefix of the (P desc, index asc) order whose
// cumulative mass reaches p" up to fp32 rounding of the masses, for any score
// distribution (ties included), without memory beyond the per-row list.
#pragma once

#include <limits.h>

#include "attn_kernels.h"
#include "common.cuh"

namespace adaspark {
namespace sel {

constexpr int kB = 64;                // bins in the window (8 log2 units, 8 bins each)
constexpr int kL = 31;                // list entries per row (one more slot as scratch)
constexpr int kRows = 128;
constexpr int kNoKey = INT_MIN;       // row without candidates
constexpr float kRefStep = 64.f;      // new reference once the maximum passes ref + 64
constexpr float kZLimit = 1048576.f;  // supported |z|: below 2^20 log2 units

// Masses are kept relative to a per-row reference ref (an integer, in log2
// units): u = 2^(z - ref). For a positive float, bits >> 20 is 8 x exponent +
// the top three mantissa bits, an integer that grows with u and steps 8 times
// per doubling; it is the bin key (bins 1/8 of an octave wide in the mantissa,
// at most a factor 1.125 between the ends of a bin). u = 0 (far below the
// reference) has key 0.
__device__ __forceinline__ int mass_key(float u) { return __float_as_int(u) >> 20; }

// 2^x on the special-function unit (relative error below 2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (three-input form of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (s1, j1) comes before (s2, j2) in the (score desc, index asc) order.
__device__ __forceinline__ bool before(float s1, int j1, float s2, int j2) {
  return s1 > s2 || (s1 == s2 && j1 < j2);
}

// Per-row storage, one column per row. The histogram is dead once the cut bin
// is known, and the list is only used from then on, so the list (raw scores
// q . kbar_j in rows [0, kL], cube indices in rows [kL + 1, 2 kL + 1]) takes
// the histogram's place. Each thread touches only its own column, so the reuse
// needs no synchronization between rows.
struct Smem {
  float hist[kB][kRows];
};
static_assert(2 * (kL + 1) <= kB, "the cut list must fit in the histogram's storage");

// Out-of-line cold paths take and return plain values, so that the per-row
// state below stays in registers (a member function called out of line would
// force the whole state object into local memory).

// The window's lowest bin moves up from key klo to key nlo: bins leaving the
// window add their mass to the new lowest bin, which holds every score below
// the window.
static __device__ __noinline__ void fold_window(float* hist_col, int klo, int nlo) {
  const int k1 = min(nlo - 1, klo + kB - 1);
  float acc = 0.f;
  for (int k = klo; k <= k1; ++k) {
    float& hv = hist_col[(k & (kB - 1)) * kRows];
    acc += hv;
    hv = 0.f;
  }
  hist_col[(nlo & (kB - 1)) * kRows] += acc;
}

// The reference moves up by `shift` log2 units: every mass scales by 2^-shift
// (exact, barring underflow) and every key moves down by 8 * shift.
static __device__ __noinline__ void rebase_window(float* hist_col, int kmax, int shift) {
  float v[kB];
  for (int i = 0; i < kB; ++i) {
    float& hv = hist_col[((kmax - i) & (kB - 1)) * kRows];
    v[i] = hv;
    hv = 0.f;
  }
  for (int i = 0; i < kB; ++i)
    hist_col[((kmax - i - 8 * shift) & (kB - 1)) * kRows] = ldexpf(v[i], -shift);
}

// Insertion sort of list entries [0, n) into the (score desc, index asc) order.
static __device__ __noinline__ void sort_entries(float* lz_col, int* lj_col, int n) {
  for (int i = 1; i < n; ++i) {
    const float z = lz_col[i * kRows];
    const int j = lj_col[i * kRows];
    int k = i;
    while (k > 0 && before(z, j, lz_col[(k - 1) * kRows], lj_col[(k - 1) * kRows])) {
      lz_col[k * kRows] = lz_col[(k - 1) * kRows];
      lj_col[k * kRows] = lj_col[(k - 1) * kRows];
      --k;
    }
    lz_col[k * kRows] = z;
    lj_col[k * kRows] = j;
  }
}

// Offer (z, j) to a full list (kL entries) of the best keys seen so far; sorts
// the list first when it is not in order. The entry replaces the last one by
// sorted insertion when it comes before it.
static __device__ __noinline__ void offer_full(float* lz_col, int* lj_col, bool sorted,
                                               float z, int j) {
  if (!sorted) sort_entries(lz_col, lj_col, kL);
  if (before(z, j, lz_col[(kL - 1) * kRows], lj_col[(kL - 1) * kRows])) {
    int pos = kL - 1;
    while (pos > 0 && before(z, j, lz_col[(pos - 1) * kRows], lj_col[(pos - 1) * kRows])) {
      lz_col[pos * kRows] = lz_col[(pos - 1) * kRows];
      lj_col[pos * kRows] = lj_col[(pos - 1) * kRows];
      --pos;
    }
    lz_col[pos * kRows] = z;
    lj_col[pos * kRows] = j;
  }
}

// Whether a Top-p cut that closed at sorted list entry i lies within thr of
// flipping, in the margin terms of the parity protocol, from the fp32 masses
// (units of 2^ref): C_k* - p (= over, the mass taken beyond the need),
// p - C_(k*-1) (only when k* > 1) and P_(k*) - P_(k*+1). The next score is the
// next list entry when there is one; when the list held the whole cut bin and
// the next score lies in a lower bin, its mass is bounded by the bin's lower
// edge `edge` (negative when nothing lies below the bin); when the list was
// full the next score is unknown and the row counts as near.
static __device__ __noinline__ bool near_cut(const float* lz_col, int i, int n, float over,
                                             float zs, float ref, float thr, bool kstar_gt1,
                                             float edge) {
  const float mi = fast_exp2(fmaf(lz_col[i * kRows], zs, -ref));
  float m = over;
  if (kstar_gt1) m = fminf(m, mi - over);
  if (i + 1 < n) {
    m = fminf(m, mi - fast_exp2(fmaf(lz_col[(i + 1) * kRows], zs, -ref)));
  } else if (n == kL) {
    return true;
  } else if (edge >= 0.f) {
    m = fminf(m, mi - edge);
  }
  return m < thr;
}

// Fine bin of a mass u inside a crowded cut bin: (bits(u) >> sh) - base,
// clamped to [0, kB - 1] (bin 0 also takes everything below).
__device__ __forceinline__ int fine_bin(float u, int sh, int base) {
  return min(max((int)(__float_as_uint(u) >> sh) - base, 0), kB - 1);
}

// The emission pass of a group of scores found the cut bin larger than the
// list: the list holds kL of the bin's scores and the group's in-bin scores
// after its first `skip` ones did not fit. The row's column becomes the fine
// histogram of the cut bin, filled with all of them (count mode adds one per
// score instead of its mass).
static __device__ __noinline__ void group_to_fine(float* col, float zs, float ref, int sh, int base,
                                                  bool count, const float* grp, uint32_t inb,
                                                  int skip) {
  float u[kL];
  for (int i = 0; i < kL; ++i) u[i] = fast_exp2(fmaf(col[i * kRows], zs, -ref));
  for (int b = 0; b < kB; ++b) col[b * kRows] = 0.f;
  for (int i = 0; i < kL; ++i) col[fine_bin(u[i], sh, base) * kRows] += count ? 1.f : u[i];
  for (int c = 0; c < 8; ++c) {
    if (!((inb >> c) & 1u)) continue;
    if (skip > 0) {
      --skip;
      continue;
    }
    const float v = fast_exp2(fmaf(grp[c], zs, -ref));
    col[fine_bin(v, sh, base) * kRows] += count ? 1.f : v;
  }
}

// The emission pass found the cut bin larger than the list: the row's column
// (list scores in rows [0, kL), indices above) becomes a histogram of kB fine
// bins of the cut bin, filled with the listed scores and the one that did not
// fit (u_new). Count mode adds one per score instead of its mass.
static __device__ __noinline__ void start_fine(float* col, float zs, float ref, int sh, int base,
                                               bool count, float u_new) {
  float u[kL];
  for (int i = 0; i < kL; ++i) u[i] = fast_exp2(fmaf(col[i * kRows], zs, -ref));
  for (int b = 0; b < kB; ++b) col[b * kRows] = 0.f;
  for (int i = 0; i < kL; ++i) col[fine_bin(u[i], sh, base) * kRows] += count ? 1.f : u[i];
  col[fine_bin(u_new, sh, base) * kRows] += count ? 1.f : u_new;
}

struct RowSel {
  float* hist_col;   // &hist[0][row]
  float* lz_col;     // list scores, in the histogram's place
  int* lj_col;       // list cube indices, likewise
  float zs;          // log2(e) / sqrt(d): z = score * zs in log2 units
  float ref;         // reference of the masses (integer, log2 units)
  int kmax;          // key of the running maximum (kNoKey before the first score)
  int klo;           // key of the lowest window bin (kmax - kB + 1)
  int kcut;          // after finish1: keys above kcut are selected outright ...
  int kcut_lo;       // ... keys in [kcut_lo, kcut] form the cut bin
  float need;        // mass still to take from the cut bin (units of 2^ref)
  int ln;            // list entries
  bool lsorted;      // list in (score desc, index asc) order
  bool open;         // cut not found yet
  bool bounded;      // only keys after (bz, bj) are offered (extra passes)
  bool range_err;    // a score outside +-kZLimit log2 units
  bool count_mode;   // Top-K: bins count scores instead of summing masses
  bool any_above;    // some score lies above the cut bin (then k* > 1)
  bool near;         // the closed cut lies within 1e-5 of a flip (Top-p only)
  bool sub;          // emission pass: the cut bin overflowed the list; its
                     // scores go to the fine histogram instead
  bool fine;         // the cut lies in fine bin fcut of the cut bin
  bool femit;        // first pass after the fine cut: emit its upper fine bins
  int fsh, fbase;    // fine bin of a mass: fine_bin(u, fsh, fbase)
  int fcut;
  float Z;           // total mass of the row (units of 2^ref), from finish1
  float bz;
  int bj;

  // count = true selects Top-K (finish1 then takes k instead of p).
  __device__ __forceinline__ void init(Smem* s, int t, float zscale, bool count = false) {
    hist_col = &s->hist[0][t];
    lz_col = &s->hist[0][t];
    lj_col = reinterpret_cast<int*>(&s->hist[kL + 1][t]);
    zs = zscale;
    ref = 0.f;
    kmax = kNoKey;
    klo = 0;
    kcut = INT_MAX;     // nothing above, nothing in the cut bin until finish1
    kcut_lo = INT_MAX;
    need = 0.f;
    ln = 0;
    lsorted = true;
    open = false;
    bounded = false;
    range_err = false;
    count_mode = count;
    any_above = false;
    near = false;
    sub = false;
    fine = false;
    femit = false;
    fsh = 20;
    fbase = 0;
    fcut = 0;
    Z = 0.f;
    bz = 0.f;
    bj = 0;
#pragma unroll 8
    for (int k = 0; k < kB; ++k) hist_col[k * kRows] = 0.f;
  }

  __device__ __forceinline__ float mass(float score) const {
    return fast_exp2(fmaf(score, zs, -ref));
  }

  // Make the window reach the raw score sm (a maximum of scores to come).
  __device__ __forceinline__ void raise(float sm) {
    const float zm = sm * zs;
    if (!(fabsf(zm) < kZLimit)) {
      range_err = true;
      return;
    }
    if (kmax == kNoKey) {
      ref = ceilf(zm);
      kmax = mass_key(mass(sm));
      klo = kmax - (kB - 1);
      return;
    }
    if (zm > ref + kRefStep) {  // keep masses far from overflow
      const int shift = (int)(ceilf(zm) - ref);
      rebase_window(hist_col, kmax, shift);
      ref += (float)shift;
      kmax -= 8 * shift;
      klo -= 8 * shift;
    }
    const int k = mass_key(mass(sm));
    if (k > kmax) {
      fold_window(hist_col, klo, k - (kB - 1));
      kmax = k;
      klo = k - (kB - 1);
    }
  }

  // Histogram update for a score of mass u whose key does not exceed kmax;
  // keys below the window land in its lowest bin. The bin gains u, or one
  // score in count mode; a column that is not a candidate (valid = false)
  // adds nothing.
  __device__ __forceinline__ void add_score(float u, bool valid) {
    const int k = max(mass_key(valid ? u : 0.f), klo);
    hist_col[(k & (kB - 1)) * kRows] += valid ? (count_mode ? 1.f : u) : 0.f;
  }

  // Histogram update of four scores of a full chunk (keys within the window,
  // which raise() has made reach the chunk's maximum). The four bins are read
  // before any is written; a score whose bin equals an earlier one's adds to
  // that score's new value, and the stores go out in order, so every bin ends
  // with exactly the sums of one update after another.
  __device__ __forceinline__ void add_quad(float u0, float u1, float u2, float u3) {
    const int k0 = max(mass_key(u0), klo) & (kB - 1), k1 = max(mass_key(u1), klo) & (kB - 1);
    const int k2 = max(mass_key(u2), klo) & (kB - 1), k3 = max(mass_key(u3), klo) & (kB - 1);
    const float w0 = count_mode ? 1.f : u0, w1 = count_mode ? 1.f : u1;
    const float w2 = count_mode ? 1.f : u2, w3 = count_mode ? 1.f : u3;
    const float h0 = hist_col[k0 * kRows], h1 = hist_col[k1 * kRows];
    const float h2 = hist_col[k2 * kRows], h3 = hist_col[k3 * kRows];
    const float v0 = h0 + w0;
    const float v1 = (k1 == k0 ? v0 : h1) + w1;
    const float v2 = (k2 == k1 ? v1 : k2 == k0 ? v0 : h2) + w2;
    const float v3 = (k3 == k2 ? v2 : k3 == k1 ? v1 : k3 == k0 ? v0 : h3) + w3;
    hist_col[k0 * kRows] = v0;
    hist_col[k1 * kRows] = v1;
    hist_col[k2 * kRows] = v2;
    hist_col[k3 * kRows] = v3;
  }

  // One score of the histogram pass (raises the window when needed).
  __device__ __forceinline__ void pass1(float score) {
    raise(score);
    if (!range_err) add_score(mass(score), true);
  }

  // p: the Top-p mass fraction; in count mode the number k of scores to keep.
  __device__ __forceinline__ void finish1(float p) {
    if (kmax == kNoKey || range_err) {
      open = false;
      return;
    }
    float Z = 0.f;  // smallest bins first
    for (int i = kB - 1; i >= 0; --i) Z += hist_col[((kmax - i) & (kB - 1)) * kRows];
    const float target = count_mode ? p : p * Z;
    float cum = 0.f;
    int kc = klo;
    for (int i = 0; i < kB - 1; ++i) {
      const float m = hist_col[((kmax - i) & (kB - 1)) * kRows];
      if (cum + m >= target) {
        kc = kmax - i;
        break;
      }
      cum += m;
    }
    need = target - cum;
    this->Z = Z;
    any_above = cum > 0.f;
    open = true;
    lsorted = false;   // the emission pass appends the cut bin in column order
    kcut = kc;
    kcut_lo = kc == klo ? INT_MIN : kc;   // the lowest bin holds everything below it
  }

  // Emission pass, one score: true when the score lies above the cut bin
  // (selected outright); a cut-bin score is appended to the list. The list
  // has one spare slot, so the append writes unconditionally. A cut-bin score
  // that finds the list full turns the column into the fine histogram of the
  // cut bin (start_fine), which takes the bin's scores from then on.
  __device__ __forceinline__ bool pass2(float score, int j, bool valid) {
    const float u = mass(score);
    const int k = mass_key(u);
    const bool above = valid && k > kcut;
    const bool inb = valid && k >= kcut_lo && k <= kcut;
    if (!sub) {
      lz_col[ln * kRows] = score;
      lj_col[ln * kRows] = j;
      const bool room = ln < kL;
      ln += (inb && room) ? 1 : 0;
      if (inb && !room) {
        // fine bins: 1/512 octave inside a regular cut bin; for the window's
        // lowest bin (which holds everything below), the 8 octaves below it
        sub = true;
        fsh = kcut_lo == INT_MIN ? 20 : 14;
        fbase = kcut_lo == INT_MIN ? klo - (kB - 1) : kcut << 6;
        start_fine(hist_col, zs, ref, fsh, fbase, count_mode, u);
      }
    } else if (inb) {
      hist_col[fine_bin(u, fsh, fbase) * kRows] += count_mode ? 1.f : u;
    }
    return above;
  }

  // Emission pass over 8 consecutive scores (columns j0 .. j0 + 7, the first
  // nv of them candidates): the same decisions as pass2 score by score, with
  // the masses and keys of the group computed first (independent, so their
  // latencies overlap) and nothing more done for a group without a cut-bin
  // score, the common case. Returns the outright selections as bits.
  __device__ __forceinline__ uint32_t emit8(const uint32_t (&acc)[8], int j0, int nv) {
    int k[8];
    float u[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      u[c] = mass(__uint_as_float(acc[c]));
      k[c] = mass_key(u[c]);
    }
    uint32_t above = 0u, inb = 0u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const bool v = c < nv;
      above |= (v && k[c] > kcut) ? (1u << c) : 0u;
      inb |= (v && k[c] >= kcut_lo && k[c] <= kcut) ? (1u << c) : 0u;
    }
    if (inb == 0u) return above;
    if (!sub) {
      const int ln0 = ln;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        lz_col[ln * kRows] = __uint_as_float(acc[c]);
        lj_col[ln * kRows] = j0 + c;
        ln += (((inb >> c) & 1u) && ln < kL) ? 1 : 0;
      }
      if (__popc(inb) > kL - ln0) {
        // the cut bin overflows the list: fine bins, 1/512 octave inside a
        // regular cut bin; for the window's lowest bin (which holds everything
        // below), the 8 octaves below it
        float grp[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) grp[c] = __uint_as_float(acc[c]);
        sub = true;
        fsh = kcut_lo == INT_MIN ? 20 : 14;
        fbase = kcut_lo == INT_MIN ? klo - (kB - 1) : kcut << 6;
        group_to_fine(hist_col, zs, ref, fsh, fbase, count_mode, grp, inb, kL - ln0);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if ((inb >> c) & 1u) hist_col[fine_bin(u[c], fsh, fbase) * kRows] += count_mode ? 1.f : u[c];
    }
    return above;
  }

  __device__ __forceinline__ void offer(float z, int j) {
    if (bounded && !before(bz, bj, z, j)) return;
    if (ln < kL) {
      lz_col[ln * kRows] = z;
      lj_col[ln * kRows] = j;
      ++ln;
      lsorted = false;
    } else {
      offer_full(lz_col, lj_col, lsorted, z, j);
      lsorted = true;
    }
  }

  // Extra pass for a row whose cut is still open: offers the scores of the
  // (fine) cut bin to the list. In the first pass after a fine cut, true for
  // a score of a fine bin above it (selected outright).
  __device__ __forceinline__ bool pass_more(float score, int j) {
    if (!open) return false;
    const float u = mass(score);
    const int k = mass_key(u);
    if (k < kcut_lo || k > kcut) return false;
    if (fine) {
      const int f = fine_bin(u, fsh, fbase);
      if (f > fcut) return femit;
      if (f < fcut) return false;
    }
    offer(score, j);
    return false;
  }

  // After a pass over the cut bin: how many leading list entries are selected.
  // Closes the cut when reached (or when the bin is exhausted); otherwise all
  // kL entries are taken and the next pass starts after the last of them.
  // After an emission pass that filled the fine histogram, finds the fine cut
  // bin instead (walking the fine bins from the top, like finish1) and leaves
  // the row open: the next pass emits the fine bins above it and lists it.
  __device__ __forceinline__ int settle() {
    if (!open) return 0;
    femit = false;
    if (sub) {
      float cum = 0.f;
      int b = kB - 1;
      for (; b > 0; --b) {
        const float m = hist_col[b * kRows];
        if (cum + m >= need) break;
        cum += m;
      }
      need -= cum;
      any_above = any_above || cum > 0.f;
      fcut = b;
      sub = false;
      fine = true;
      femit = true;
      ln = 0;
      lsorted = true;
      bounded = false;
      return 0;
    }
    const int n = ln;
    if (!lsorted) sort_entries(lz_col, lj_col, n);
    lsorted = true;
    float cum = 0.f;
    for (int i = 0; i < n; ++i) {
      cum += count_mode ? 1.f : mass(lz_col[i * kRows]);
      if (cum >= need) {
        open = false;
        if (!count_mode)
          near = near_cut(lz_col, i, n, cum - need, zs, ref, 1e-5f * Z,
                          any_above || bounded || i > 0, lower_edge());
        return i + 1;
      }
    }
    if (n < kL) {  // the whole cut bin was offered: rounding left need unmet
      open = false;
      near = !count_mode;
      return n;
    }
    need -= cum;
    bounded = true;
    bz = lz_col[(kL - 1) * kRows];
    bj = lj_col[(kL - 1) * kRows];
    return n;
  }

  // Lower mass edge of the bin the list collects (the cut bin, or its fine
  // cut bin); negative when that bin also holds everything below it.
  __device__ __forceinline__ float lower_edge() const {
    if (fine) return (fsh == 20 && fcut == 0) ? -1.f : __int_as_float((fbase + fcut) << fsh);
    return kcut_lo == INT_MIN ? -1.f : __int_as_float(kcut_lo << 20);
  }

  __device__ __forceinline__ int list_j(int i) const { return lj_col[i * kRows]; }
  __device__ __forceinline__ void reset_list() {
    ln = 0;
    lsorted = true;
  }
};

// 32 x 32 bit transpose across a warp: on entry lane r holds row r (bit c =
// column c), on return lane c holds column c (bit r = row r). Each stage swaps
// the off-diagonal blocks of one size with the partner lane.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const uint32_t mhi = s == 16 ? 0xFFFF0000u
                       : s == 8  ? 0xFF00FF00u
                       : s == 4  ? 0xF0F0F0F0u
                       : s == 2  ? 0xCCCCCCCCu
                                 : 0xAAAAAAAAu;
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, s);
    x = (lane & s) ? ((x & mhi) | ((y >> s) & ~mhi)) : ((x & ~mhi) | ((y << s) & mhi));
  }
  return x;
}

}  // namespace sel

// ---------------------------------------------------------------------------
// Shared tile epilogue: compact the cube columns with any row bit into the
// tile's ascending list. 128 threads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int compact_tile_list(const uint32_t* tmask, uint16_t* list,
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
  return total;
}

// Split walk of a visual tile (see SplitLayout): the tile's list (n cubes,
// ascending) is divided into the cubes the tile walks itself and the sparse
// ones, chosen by at most sp.rows of its rows and below the tile's lowest own
// cube c_lo (so no row of the tile has one as its own cube); at most kSparseMax
// per tile (later candidates stay in the walk). Each row's selections among
// the sparse cubes become records (row, cube), in ascending cube order, at
// row_off[row]; space for the tile's records is taken from the counter
// hdr->sched[0]; when it would pass the capacity the tile keeps its whole list
// (its reserved records are marked unused). Each sparse cube takes a range of
// its (KV head, cube) group at once (grp_cnt), and each record its place in
// that range (rec_gpos, the row's rank among the cube's rows in the tile), so
// the regrouping needs no atomics. 128 threads, thread tid = tile row; `stage`
// is shared scratch of kSparseMax * 24 bytes (the per-row selection storage,
// free by now).
constexpr int kSparseMax = 1024;
__device__ __forceinline__ void split_tile(const uint32_t* tmask, const uint16_t* list, int n,
                                           const SplitArgs& sp, int vt, int C, int c_lo, int kv,
                                           int rid, bool valid, uint8_t* stage, int* s_wcnt,
                                           int* s_misc, WsHeader* hdr, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  const unsigned lt = (1u << lane) - 1u;
  uint4* s_mask = reinterpret_cast<uint4*>(stage);                       // [kSparseMax]
  int* s_p0 = reinterpret_cast<int*>(stage + kSparseMax * 16);            // [kSparseMax]
  uint16_t* s_j = reinterpret_cast<uint16_t*>(stage + kSparseMax * 20);   // [kSparseMax]
  uint16_t* walk = sp.walk_list + (size_t)vt * C;
  int n_walk = 0, n_sp = 0;
  for (int base = 0; base < n; base += 128) {
    const int e = base + tid;
    int j = -1;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    bool cand = false;
    if (e < n) {
      j = __ldcg(list + e);
      w = __ldcg(reinterpret_cast<const uint4*>(tmask + (size_t)j * 4));
      const int r = __popc(w.x) + __popc(w.y) + __popc(w.z) + __popc(w.w);
      cand = j < c_lo && r <= sp.rows;
    }
    const unsigned bc = __ballot_sync(0xffffffffu, cand);
    if (lane == 0) s_wcnt[warp] = __popc(bc);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int pc = n_sp;
    for (int q = 0; q < warp; ++q) pc += s_wcnt[q];
    const int tc = s_wcnt[0] + s_wcnt[1] + s_wcnt[2] + s_wcnt[3];
    const int ps = pc + __popc(bc & lt);
    const bool sp_e = cand && ps < kSparseMax;
    const bool keep = e < n && !sp_e;
    const unsigned bk = __ballot_sync(0xffffffffu, keep);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (lane == 0) s_wcnt[warp] = __popc(bk);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int pk = n_walk;
    for (int q = 0; q < warp; ++q) pk += s_wcnt[q];
    const int tk = s_wcnt[0] + s_wcnt[1] + s_wcnt[2] + s_wcnt[3];
    if (keep) walk[pk + __popc(bk & lt)] = (uint16_t)j;
    if (sp_e) {
      s_mask[ps] = w;
      s_j[ps] = (uint16_t)j;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    n_walk += tk;
    n_sp = min(n_sp + tc, kSparseMax);
  }
  // this row's records: its bits among the sparse cubes, 32 cubes at a time
  // (lane L reads its warp's word of cube k0 + L; the transpose gives each
  // lane, a row, its bits over those 32 cubes)
  const uint32_t* s_w = reinterpret_cast<const uint32_t*>(s_mask);
  auto row_bits = [&](int k0) {
    const uint32_t x = k0 + lane < n_sp ? s_w[(k0 + lane) * 4 + warp] : 0u;
    return sel::warp_transpose32(x, lane);
  };
  int cnt = 0;
  for (int k0 = 0; k0 < n_sp; k0 += 32) cnt += __popc(row_bits(k0));
  if (!valid) cnt = 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_wcnt[warp] = incl;
  asm volatile("bar.sync 1, 128;" ::: "memory");
  int excl = incl - cnt;
  for (int q = 0; q < warp; ++q) excl += s_wcnt[q];
  const int total = s_wcnt[0] + s_wcnt[1] + s_wcnt[2] + s_wcnt[3];
  if (tid == 0) {
    // once the counter has passed the capacity no tile takes space any more,
    // so it stays far below 2^32 (at most the capacity plus the records of
    // the tiles that raced past it)
    unsigned b = 0;
    bool fits = true;
    if (total > 0) {
      if (*reinterpret_cast<volatile unsigned*>(&hdr->sched[0]) >= (unsigned)sp.cap) {
        b = (unsigned)sp.cap;
        fits = false;
      } else {
        b = atomicAdd(&hdr->sched[0], (unsigned)total);
        fits = (unsigned long long)b + (unsigned)total <= (unsigned long long)sp.cap;
      }
    }
    s_misc[0] = (int)min(b, (unsigned)sp.cap);
    s_misc[1] = fits ? 1 : 0;
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int rbase = s_misc[0];
  const bool fits = s_misc[1] != 0;
  if (!fits) {
    for (int e = tid; e < n; e += 128) walk[e] = __ldcg(list + e);
    if (tid == 0) sp.walk_count[vt] = n;
    // the records this tile reserved below the capacity are marked unused
    const long long hi = min((long long)rbase + total, (long long)sp.cap);
    for (long long i = (long long)rbase + tid; i < hi; i += 128) sp.rec_row[i] = -1;
    if (valid) sp.row_cnt[rid] = 0;
    return;
  }
  if (tid == 0) sp.walk_count[vt] = n_walk;
  // each sparse cube's range in its group
  for (int k = tid; k < n_sp; k += 128) {
    const uint4 w = s_mask[k];
    s_p0[k] = atomicAdd(&sp.grp_cnt[(size_t)kv * C + s_j[k]],
                        __popc(w.x) + __popc(w.y) + __popc(w.z) + __popc(w.w));
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int o = rbase + excl;
  if (valid) {
    sp.row_off[rid] = o;
    sp.row_cnt[rid] = cnt;
  }
  int k2 = 0;
  for (int k0 = 0; k0 < n_sp; k0 += 32) {   // warp-uniform: every lane transposes
    uint32_t b = row_bits(k0);
    if (!valid) b = 0u;
    while (b) {
      const int k = k0 + __ffs(b) - 1;
      b &= b - 1u;
      // rank of this row among the cube's rows in the tile
      int rank = __popc(s_w[k * 4 + warp] & lt);
      for (int q = 0; q < warp; ++q) rank += __popc(s_w[k * 4 + q]);
      sp.rec_row[o + k2] = rid;
      sp.rec_cube[o + k2] = s_j[k];
      sp.rec_gpos[o + k2] = s_p0[k] + rank;
      ++k2;
    }
  }
}

}  // namespace adaspark

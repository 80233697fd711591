// losa_cut.cuh - the per-row threshold cut of LoSA's selection step, shared
// by the selection kernels and the construction kernel's fused epilogue.
//
// Per (b, h, query block) row: the smallest key-block set, taken in
// descending mass, whose cumulative mass reaches tau (ubos.tech LoSA post,
// "How It Works in Practice", Phase 2 - Block Mask Generation; LoSA
// abstract, arXiv 2608.12032). Masses are converted to 64-bit fixed point
// x = round(m * 2^48), so sorting, prefix sums and the threshold test are
// integer work and bit-exact. Each row's sort keys
//     key(J) = ((2^49 - 1 - x_J) << 11) | J          (< 2^60, unique per row)
// ascend in (x desc, J asc) order; the cut is the first position k whose
// prefix sum C_k satisfies 2^48 * C_k >= round(tau * 2^48) * S (S the row's
// total), compared in 128-bit integers. The kept set is {J : key(J) <= cut
// key}.
#pragma once

#include <cstdint>

#include "losa_device.cuh"

namespace losa {
namespace cut {

constexpr unsigned long long kXMax = (1ull << 49) - 1;  // masses in [0, 2); J < 2048
constexpr unsigned long long kNoKey = ~0ull;
constexpr int kBuckets = 1 + 49 * 16;  // x < 2^49: 16 buckets per octave, x = 0 apart
constexpr int kCap = 2048;             // n <= 2047 keys, padded to a power of two

// x = round(m * 2^48) (ties to even; exact, as m * 2^48 only shifts the
// exponent). Returns false for NaN, Inf, negative or >= 2.
__device__ __forceinline__ bool to_fixed(float m, long long& x) {
  if (!(m >= 0.f && m < 2.f)) {
    x = 0;
    return false;
  }
  x = __double2ll_rn(double(m) * 281474976710656.0);
  return true;
}

__device__ __forceinline__ unsigned long long sort_key(long long x, int J) {
  return ((kXMax - (unsigned long long)x) << 11) | (unsigned long long)J;
}

// The fixed-point mass a sort key carries (padding keys carry none).
__device__ __forceinline__ unsigned long long key_x(unsigned long long key) {
  return key == kNoKey ? 0ull : kXMax - (key >> 11);
}

// 2^48 * C >= tau_fx * S, exactly.
__device__ __forceinline__ bool reaches(unsigned long long C, unsigned long long tau_fx,
                                        unsigned long long S) {
  return ((unsigned __int128)C << 48) >= (unsigned __int128)tau_fx * S;
}

// Bucket of x by its leading five bits (the highest set bit and the four
// below it), x = 0 in bucket 0: every key of a higher bucket has a larger x
// than every key of a lower one.
__device__ __forceinline__ int x_bucket(unsigned long long x) {
  if (x == 0) return 0;
  const int h = 63 - __clzll((long long)x);
  const int sub = h >= 4 ? int((x >> (h - 4)) & 15u) : int((x << (4 - h)) & 15u);
  return 1 + h * 16 + sub;
}

// Shared-memory workspace of one row's bucketed cut (26.3 KB).
struct BucketSmem {
  unsigned long long hsum[kBuckets];
  int hcnt[kBuckets];
  unsigned long long cand[kCap];
  unsigned long long wsum[32];  // per-warp partials of the block scans
  int wint[32];
  unsigned long long A, S;
  int b, above, m;
};

// Exclusive prefix sum over the NT threads of a group that `sync` joins
// (warp shuffles, then the warp totals through shared memory). Returns the
// sum over the threads before `tid` and sets `total` to the group's sum.
template <int NT, class T, class Sync>
__device__ __forceinline__ T group_exclusive_sum(T v, T* wbuf, int tid, const Sync& sync,
                                                 T& total) {
  const int lane = tid & 31, w = tid >> 5;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wbuf[w] = x;
  sync();
  T before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    const T s = wbuf[i];
    if (i < w) before += s;
    tot += s;
  }
  sync();
  total = tot;
  return before + x - v;
}

template <int NT, class Sync>
__device__ __forceinline__ int group_min(int v, int* wbuf, int tid, const Sync& sync) {
  v = __reduce_min_sync(0xffffffffu, v);
  if ((tid & 31) == 0) wbuf[tid >> 5] = v;
  sync();
  int m = wbuf[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) m = min(m, wbuf[i]);
  sync();
  return m;
}

// The cut of one row of n <= 2047 masses by a group of NT threads (whole
// warps; `sync` is a barrier over exactly those threads, tid their index).
// The keys are bucketed by x_bucket; a scan over the buckets in descending
// order finds the bucket in which the running sum first reaches the
// threshold, and only that bucket's keys are sorted (bitonic, in shared
// memory): the keys of the buckets above fill the first positions of the
// sorted order whatever their own order, so the cut (position, key and
// prefix sum) is the one the full sort-and-accumulate definition gives. An
// all-zero row (S = 0) stops at its first key. Bucket sums and counts are
// integer atomics, so the result does not depend on scheduling.
// Writes cut_key, count (kept blocks), retained_fx (C at the cut) and
// total_fx (S) of `row`; a mass outside [0, 2) raises kStatusBadMass.
template <int NT, class Sync>
__device__ __forceinline__ void bucket_cut_row(const float* mrow, int n,
                                               unsigned long long tau_fx, BucketSmem& sm,
                                               int tid, const Sync& sync, int64_t row,
                                               unsigned long long* cut_key, int* count,
                                               long long* retained_fx, long long* total_fx,
                                               int* status) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps");
  constexpr int PER = (kBuckets + NT - 1) / NT;  // buckets per thread in the scan
  for (int i = tid; i < kBuckets; i += NT) {
    sm.hsum[i] = 0;
    sm.hcnt[i] = 0;
  }
  if (tid == 0) sm.m = 0;
  sync();
  bool bad = false;
  for (int J = tid; J < n; J += NT) {
    long long x;
    bad |= !to_fixed(mrow[J], x);
    const int b = x_bucket((unsigned long long)x);
    atomicAdd(&sm.hsum[b], (unsigned long long)x);
    atomicAdd(&sm.hcnt[b], 1);
  }
  if (__any_sync(0xffffffffu, bad) && (tid & 31) == 0)
    atomicCAS(status, kStatusOk, kStatusBadMass);
  sync();

  // Buckets in descending order: thread tid owns reversed positions
  // [tid * PER, tid * PER + PER), i.e. buckets kBuckets - 1 - pos.
  unsigned long long ls = 0;
  int lc = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int pos = tid * PER + i;
    if (pos < kBuckets) {
      ls += sm.hsum[kBuckets - 1 - pos];
      lc += sm.hcnt[kBuckets - 1 - pos];
    }
  }
  unsigned long long S;
  const unsigned long long sum_before = group_exclusive_sum<NT>(ls, sm.wsum, tid, sync, S);
  int n_all;
  const int cnt_before = group_exclusive_sum<NT>(lc, sm.wint, tid, sync, n_all);
  // First bucket (in descending order) whose inclusive sum reaches the
  // threshold; an all-zero row (S = 0) stops at bucket 0.
  int first = kBuckets;
  unsigned long long A_at = 0;
  int above_at = 0;
  {
    unsigned long long A = sum_before;
    int above = cnt_before;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int pos = tid * PER + i;
      if (pos >= kBuckets || first != kBuckets) break;
      const int b = kBuckets - 1 - pos;
      if (S > 0 ? reaches(A + sm.hsum[b], tau_fx, S) : b == 0) {
        first = pos;
        A_at = A;
        above_at = above;
      }
      A += sm.hsum[b];
      above += sm.hcnt[b];
    }
  }
  const int pmin = group_min<NT>(first, sm.wint, tid, sync);
  if (first == pmin && first < kBuckets) {
    sm.b = kBuckets - 1 - first;
    sm.A = A_at;
    sm.above = above_at;
    sm.S = S;
  }
  sync();
  const int bstar = sm.b;
  // The boundary bucket's keys.
  for (int J = tid; J < n; J += NT) {
    long long x;
    to_fixed(mrow[J], x);
    if (x_bucket((unsigned long long)x) == bstar) sm.cand[atomicAdd(&sm.m, 1)] = sort_key(x, J);
  }
  sync();
  const int m = sm.m;
  int np = 2;
  while (np < m) np <<= 1;
  for (int i = m + tid; i < np; i += NT) sm.cand[i] = kNoKey;
  // Bitonic sort of the bucket, ascending.
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      sync();
      for (int pr = tid; pr < np / 2; pr += NT) {
        const int i = 2 * stride * (pr / stride) + (pr % stride);
        const int k = i + stride;
        const unsigned long long a = sm.cand[i], b = sm.cand[k];
        const bool up = (i & size) == 0;
        if ((a > b) == up) {
          sm.cand[i] = b;
          sm.cand[k] = a;
        }
      }
    }
  }
  sync();
  // Prefix sums over the sorted bucket, on top of the buckets above it:
  // thread tid owns positions [tid * per, tid * per + per).
  const int per = (np + NT - 1) / NT;
  unsigned long long local = 0;
  for (int i = 0; i < per; ++i) {
    const int pos = tid * per + i;
    if (pos < m) local += key_x(sm.cand[pos]);
  }
  unsigned long long unused;
  const unsigned long long before = group_exclusive_sum<NT>(local, sm.wsum, tid, sync, unused);
  const unsigned long long St = sm.S;
  unsigned long long C = sm.A + before;
  int firstk = kCap;
  for (int i = 0; i < per; ++i) {
    const int pos = tid * per + i;
    if (pos >= m) break;
    C += key_x(sm.cand[pos]);
    if (reaches(C, tau_fx, St)) {
      firstk = pos;
      break;
    }
  }
  const int p = group_min<NT>(firstk, sm.wint, tid, sync);
  if (p < m && p >= tid * per && p < tid * per + per) {
    // The thread that owns the cut position writes the row's results; its
    // running sum C stopped exactly there.
    cut_key[row] = sm.cand[p];
    count[row] = sm.above + p + 1;
    retained_fx[row] = (long long)C;
    total_fx[row] = (long long)St;
  }
}

}  // namespace cut
}  // namespace losa

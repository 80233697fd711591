// losa_select.cu - the selection step of LoSA on the GPU: per (b, h, query
// block), the smallest key-block set whose cumulative mass reaches tau
// (ubos.tech LoSA post, "How It Works in Practice", Phase 2 - Block Mask
// Generation: sort key blocks by descending mass and accumulate until the
// threshold is met; LoSA abstract, arXiv 2608.12032: "keeps, for each head
// and query block, the smallest key/value block set meeting the threshold").
//
// All of it is integer work on 64-bit fixed-point masses x = round(m * 2^48),
// so the result is bit-exact. Each row's sort keys
//     key(J) = ((2^49 - 1 - x_J) << 11) | J          (< 2^60, unique per row)
// ascend in (x desc, J asc) order; a bitonic sort in shared memory orders
// them, a block prefix scan accumulates the masses in that order, and the
// cut is the first prefix that reaches the threshold. The kept set is then
// {J : key(J) <= cut key}, written out in ascending J.
#include <cub/block/block_reduce.cuh>
#include <cub/block/block_scan.cuh>

#include <cstdio>
#include <mutex>
#include <vector>

#include "losa_cut.cuh"
#include "losa_device.cuh"
#include "losa_internal.h"

namespace losa {
namespace {

using cut::kNoKey;
using cut::kXMax;
using cut::reaches;
using cut::sort_key;
using cut::to_fixed;

constexpr int kSelThreads = 256;

// One warp per row: the cut key, kept count, kept and total fixed-point
// mass. The row's NP sort keys (n rounded up to a power of two, padded with
// keys that sort last) live in registers, IPT = NP / 32 per lane, element
// i = lane * IPT + r. A bitonic network sorts them ascending: exchanges
// whose partner sits in the same lane (stride < IPT) stay in registers, the
// others (stride >= IPT) go through warp shuffles. The fixed-point masses
// are then prefix-summed in sorted order and the cut is the first position
// k where 2^48 * C_k >= tau_fx * S (exact, 128-bit). No atomics and no
// shared memory, so the result does not depend on scheduling.
constexpr int kCutWarps = 4;  // rows per CTA

__device__ __forceinline__ unsigned long long umin64(unsigned long long a, unsigned long long b) {
  return a < b ? a : b;
}
__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a < b ? b : a;
}

// Exchanges between elements r and r + stride of this lane (stride < IPT).
template <int IPT, int STRIDE>
__device__ __forceinline__ void bitonic_in_lane(unsigned long long (&k)[IPT], int lane, int size) {
#pragma unroll
  for (int r = 0; r < IPT; ++r) {
    if ((r & STRIDE) == 0) {
      const bool up = ((lane * IPT + r) & size) == 0;
      const unsigned long long a = k[r], b = k[r + STRIDE];
      k[r] = up ? umin64(a, b) : umax64(a, b);
      k[r + STRIDE] = up ? umax64(a, b) : umin64(a, b);
    }
  }
  if constexpr (STRIDE > 1) bitonic_in_lane<IPT, STRIDE / 2>(k, lane, size);
}

// The in-lane part of one merge step of `size`: strides min(size / 2, S0)
// down to 1.
template <int IPT, int S0>
__device__ __forceinline__ void bitonic_in_lane_from(unsigned long long (&k)[IPT], int lane,
                                                     int size) {
  if constexpr (S0 >= 1) {
    if (size / 2 >= S0)
      bitonic_in_lane<IPT, S0>(k, lane, size);
    else
      bitonic_in_lane_from<IPT, S0 / 2>(k, lane, size);
  }
}

template <int NP>
__global__ void __launch_bounds__(32 * kCutWarps)
    select_cut_kernel(const float* __restrict__ mass, int64_t R, int n,
                      unsigned long long tau_fx, unsigned long long* __restrict__ cut_key,
                      int* __restrict__ count, long long* __restrict__ retained_fx,
                      long long* __restrict__ total_fx, int* status) {
  constexpr int IPT = NP / 32;
  static_assert(IPT >= 2 && (IPT & (IPT - 1)) == 0, "NP must be a power of two >= 64");
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kCutWarps + (threadIdx.x >> 5);
  if (row >= R) return;  // whole warps only
  const float* mrow = mass + size_t(row) * n;

  unsigned long long k[IPT];
  bool bad = false;
#pragma unroll
  for (int r = 0; r < IPT; ++r) {
    const int J = lane * IPT + r;
    unsigned long long key = kNoKey;
    if (J < n) {
      long long x;
      bad |= !to_fixed(mrow[J], x);
      key = sort_key(x, J);
    }
    k[r] = key;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(status, kStatusOk, kStatusBadMass);

  // Bitonic sort, ascending.
  for (int size = 2; size <= NP; size <<= 1) {
    for (int stride = size >> 1; stride >= IPT; stride >>= 1) {
      const int lx = stride / IPT;  // partner lane = lane ^ lx
      const bool up = ((lane * IPT) & size) == 0;
      const bool lower = (lane & lx) == 0;
#pragma unroll
      for (int r = 0; r < IPT; ++r) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, k[r], lx);
        k[r] = (lower == up) ? umin64(k[r], o) : umax64(k[r], o);
      }
    }
    bitonic_in_lane_from<IPT, IPT / 2>(k, lane, size);
  }

  // Fixed-point masses in sorted order; padding keys carry no mass.
  auto xval = [](unsigned long long key) -> unsigned long long {
    return key == kNoKey ? 0ull : kXMax - (key >> 11);
  };
  unsigned long long T = 0;
#pragma unroll
  for (int r = 0; r < IPT; ++r) T += xval(k[r]);
  unsigned long long incl = T;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const unsigned long long S = __shfl_sync(0xffffffffu, incl, 31);
  // First position whose running sum reaches the threshold (k >= 1; the full
  // row always reaches it, and an all-zero row stops at its first key).
  unsigned long long C = incl - T;
  unsigned first = unsigned(NP);
  unsigned long long key_at = 0, c_at = 0;
#pragma unroll
  for (int r = 0; r < IPT; ++r) {
    C += xval(k[r]);
    const int pos = lane * IPT + r;
    if (first == unsigned(NP) && pos < n && reaches(C, tau_fx, S)) {
      first = unsigned(pos);
      key_at = k[r];
      c_at = C;
    }
  }
  const unsigned kcut = __reduce_min_sync(0xffffffffu, first);
  if (first == kcut && kcut < unsigned(NP)) {
    // The lane holding the cut position writes the row's results.
    cut_key[row] = key_at;
    count[row] = int(kcut) + 1;
    retained_fx[row] = (long long)c_at;
    total_fx[row] = (long long)S;
  }
}

// Rows of more than 512 key blocks: one CTA of 256 threads per row, running
// the bucketed cut of losa_cut.cuh (the construction kernel's fused epilogue
// runs the same code on a warpgroup).
constexpr int kBkThreads = 256;
constexpr int kBkCap = cut::kCap;

struct CtaSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

__global__ void __launch_bounds__(kBkThreads)
    select_cut_bucket_kernel(const float* __restrict__ mass, int n, unsigned long long tau_fx,
                             unsigned long long* __restrict__ cut_key, int* __restrict__ count,
                             long long* __restrict__ retained_fx, long long* __restrict__ total_fx,
                             int* status) {
  __shared__ cut::BucketSmem sm;
  const int64_t row = blockIdx.x;
  cut::bucket_cut_row<kBkThreads>(mass + size_t(row) * n, n, tau_fx, sm, int(threadIdx.x),
                                  CtaSync{}, row, cut_key, count, retained_fx, total_fx, status);
}

// Launches the cut kernel with the smallest power-of-two capacity >= n.
cudaError_t launch_select_cut(const float* mass, int64_t R, int n, unsigned long long tau_fx,
                              unsigned long long* cut, int* cnt, long long* retained,
                              long long* total, int* status, cudaStream_t stream) {
  const unsigned grid = unsigned((R + kCutWarps - 1) / kCutWarps);
#define LOSA_CUT(NP_)                                                                   \
  if (n <= NP_) {                                                                       \
    select_cut_kernel<NP_><<<grid, 32 * kCutWarps, 0, stream>>>(mass, R, n, tau_fx, cut, \
                                                                 cnt, retained, total,   \
                                                                 status);                \
    return cudaGetLastError();                                                          \
  }
  LOSA_CUT(64)
  LOSA_CUT(128)
  LOSA_CUT(256)
  LOSA_CUT(512)
#undef LOSA_CUT
  if (n < kBkCap) {
    select_cut_bucket_kernel<<<unsigned(R), kBkThreads, 0, stream>>>(mass, n, tau_fx, cut, cnt,
                                                                     retained, total, status);
    return cudaGetLastError();
  }
  return cudaErrorInvalidValue;
}

// Per 128-row tile (128/block query blocks): which key blocks each query
// block keeps, as a bitmask m_J (bit q = q-th query block of the tile).
__device__ __forceinline__ unsigned tile_mask(const float* __restrict__ mass,
                                              const unsigned long long* __restrict__ cut_key,
                                              int n, int row0, int nq, int J) {
  unsigned m = 0;
  for (int q = 0; q < nq; ++q) {
    const int r = row0 + q;
    long long x;
    to_fixed(mass[size_t(r) * n + J], x);
    if (sort_key(x, J) <= cut_key[r]) m |= 1u << q;
  }
  return m;
}

__global__ void __launch_bounds__(kSelThreads)
    tile_count_kernel(const float* __restrict__ mass, const unsigned long long* __restrict__ cut_key,
                      int n, int qpt, int n_qt, int* __restrict__ tile_count) {
  using Reduce = cub::BlockReduce<int, kSelThreads>;
  __shared__ typename Reduce::TempStorage tmp;
  const int t = blockIdx.x;
  const int bh = t / n_qt, qt = t % n_qt;
  const int I0 = qt * qpt;
  const int nq = min(qpt, n - I0);
  const int row0 = bh * n + I0;
  int c = 0;
  for (int J = threadIdx.x; J < n; J += kSelThreads)
    c += tile_mask(mass, cut_key, n, row0, nq, J) != 0;
  const int total = Reduce(tmp).Sum(c);
  if (threadIdx.x == 0) tile_count[t] = total;
}

// Writes each query block's kept key blocks (ascending) into col_idx and the
// tile's union entries (J | mask << 16, ascending J) into tile_entry.
// Counts of one 256-wide chunk are scanned together, packed in 10-bit fields:
// fields 0..3 = query blocks of the tile, field 4 = the union.
__global__ void __launch_bounds__(kSelThreads)
    tile_write_kernel(const float* __restrict__ mass, const unsigned long long* __restrict__ cut_key,
                      int n, int qpt, int n_qt, const int* __restrict__ row_ptr,
                      const int* __restrict__ tile_ptr, int* __restrict__ col_idx,
                      int* __restrict__ tile_entry) {
  using Scan = cub::BlockScan<unsigned long long, kSelThreads>;
  __shared__ typename Scan::TempStorage tmp;
  const int t = blockIdx.x;
  const int bh = t / n_qt, qt = t % n_qt;
  const int I0 = qt * qpt;
  const int nq = min(qpt, n - I0);
  const int row0 = bh * n + I0;
  int base[4];
  for (int q = 0; q < 4; ++q) base[q] = (q < nq) ? row_ptr[row0 + q] : 0;
  int ubase = tile_ptr[t];
  for (int c0 = 0; c0 < n; c0 += kSelThreads) {
    const int J = c0 + threadIdx.x;
    const unsigned m = (J < n) ? tile_mask(mass, cut_key, n, row0, nq, J) : 0u;
    unsigned long long v = 0;
    for (int q = 0; q < 4; ++q) v |= (unsigned long long)((m >> q) & 1u) << (10 * q);
    v |= (unsigned long long)(m != 0) << 40;
    unsigned long long ex, tot;
    Scan(tmp).ExclusiveSum(v, ex, tot);
    __syncthreads();
    for (int q = 0; q < nq; ++q)
      if ((m >> q) & 1u) col_idx[base[q] + int((ex >> (10 * q)) & 1023)] = J;
    if (m) tile_entry[ubase + int((ex >> 40) & 1023)] = J | int(m << 16);
    for (int q = 0; q < 4; ++q) base[q] += int((tot >> (10 * q)) & 1023);
    ubase += int((tot >> 40) & 1023);
  }
}

// Exclusive scan of n ints into out[0..n] (out[n] = total), one CTA.
__global__ void __launch_bounds__(1024) scan_kernel(const int* __restrict__ in, int n,
                                                    int* __restrict__ out) {
  using Scan = cub::BlockScan<int, 1024>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += 1024) {
    const int i = c0 + threadIdx.x;
    const int v = (i < n) ? in[i] : 0;
    int ex, tot;
    Scan(tmp).ExclusiveSum(v, ex, tot);
    const int c = carry;
    if (i < n) out[i] = c + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry = c + tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) out[n] = carry;
}

// Order of the sparse kernel's work: head by head (so the CTAs resident at
// one time gather from one head's K/V, which stays in L2), and within a
// head by entry count, largest first (longest-processing-time order for the
// block scheduler). Counting sort on the key head * (n + 1) + (n - count);
// order among equal keys is unspecified.
__device__ __forceinline__ int order_key(int t, int n_qt, int n, const int* tile_count) {
  return (t / n_qt) * (n + 1) + (n - tile_count[t]);
}

__global__ void order_hist_kernel(const int* __restrict__ tile_count, int T, int n_qt, int n,
                                  int* __restrict__ hist) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x)
    atomicAdd(&hist[order_key(t, n_qt, n, tile_count)], 1);
}

__global__ void order_scatter_kernel(const int* __restrict__ tile_count, int T, int n_qt, int n,
                                     int* __restrict__ cursor, int* __restrict__ order) {
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x)
    order[atomicAdd(&cursor[order_key(t, n_qt, n, tile_count)], 1)] = t;
}

// Union entries of one 128-row query tile from the CSR rows of its query
// blocks, for a pattern that is imported rather than selected. kWrite =
// false counts the tile's entries into tile_count; kWrite = true writes them
// (J | mask << 16, ascending J) at tile_ptr. The host has checked that every
// row's columns are strictly ascending and lie in [0, n), so within one row
// no two threads touch the same byte of `masks`.
template <bool kWrite>
__global__ void __launch_bounds__(kSelThreads)
    csr_tile_kernel(const int* __restrict__ row_ptr, const int* __restrict__ col_idx, int n,
                    int qpt, int n_qt, int* __restrict__ tile_count,
                    const int* __restrict__ tile_ptr, int* __restrict__ tile_entry) {
  using Reduce = cub::BlockReduce<int, kSelThreads>;
  using Scan = cub::BlockScan<int, kSelThreads>;
  __shared__ union {
    typename Reduce::TempStorage reduce;
    typename Scan::TempStorage scan;
  } tmp;
  __shared__ unsigned char masks[2048];
  const int t = blockIdx.x;
  const int bh = t / n_qt, qt = t % n_qt;
  const int I0 = qt * qpt;
  const int nq = min(qpt, n - I0);
  const int row0 = bh * n + I0;
  for (int J = threadIdx.x; J < n; J += kSelThreads) masks[J] = 0;
  __syncthreads();
  for (int q = 0; q < nq; ++q) {
    const int e1 = row_ptr[row0 + q + 1];
    for (int e = row_ptr[row0 + q] + threadIdx.x; e < e1; e += kSelThreads)
      masks[col_idx[e]] |= (unsigned char)(1u << q);
    __syncthreads();
  }
  if (!kWrite) {
    int c = 0;
    for (int J = threadIdx.x; J < n; J += kSelThreads) c += masks[J] != 0;
    const int total = Reduce(tmp.reduce).Sum(c);
    if (threadIdx.x == 0) tile_count[t] = total;
    return;
  }
  int base = tile_ptr[t];
  for (int c0 = 0; c0 < n; c0 += kSelThreads) {
    const int J = c0 + threadIdx.x;
    const unsigned m = (J < n) ? masks[J] : 0u;
    int ex, tot;
    Scan(tmp.scan).ExclusiveSum(int(m != 0), ex, tot);
    __syncthreads();
    if (m) tile_entry[base + ex] = J | int(m << 16);
    base += tot;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

int select_begin(int B, int H, int n, int block, double tau, cudaStream_t stream,
                 SelectJob& job) {
  job = SelectJob{};
  const int BH = B * H;
  job.R = int64_t(BH) * n;
  const int L_pad = n * block;
  job.n = n;
  job.n_qt = (L_pad + 127) / 128;
  job.qpt = 128 / block;
  job.T = int64_t(BH) * job.n_qt;
  job.tau_fx = (unsigned long long)llrint(tau * 281474976710656.0);
  job.stream = stream;
  const int64_t R = job.R, T = job.T;

  losa_pattern* p = new losa_pattern{};
  p->B = B;
  p->H = H;
  p->n_blocks = n;
  p->block = block;
  p->n_qt = job.n_qt;
  p->n_tiles = T;
  p->stream = stream;
  cudaGetDevice(&p->device);
  job.p = p;

  // Pattern arrays of known size: one allocation.
  const size_t o_row = 0;
  const size_t o_tptr = o_row + align256((R + 1) * 4);
  const size_t o_tord = o_tptr + align256((T + 1) * 4);
  const size_t o_ret = o_tord + align256(T * 4);
  const size_t o_tot = o_ret + align256(R * 8);
  const size_t fixed_bytes = o_tot + align256(R * 8);
  // Scratch: cut keys, row counts, tile counts, histogram, cursor.
  const size_t s_cut = 0;
  const size_t s_cnt = s_cut + align256(R * 8);
  const size_t s_tcnt = s_cnt + align256(R * 4);
  job.n_keys = int64_t(BH) * (n + 1);  // order keys: head x (n + 1)
  const size_t s_hist = s_tcnt + align256(T * 4);
  const size_t s_cur = s_hist + align256(job.n_keys * 4);
  const size_t scratch_bytes = s_cur + align256((job.n_keys + 1) * 4);

  job.fixed = static_cast<char*>(pool_alloc(fixed_bytes, stream));
  job.scratch = static_cast<char*>(pool_alloc(scratch_bytes, stream));
  if (!job.fixed || !job.scratch) {
    select_abort(job);
    return LOSA_ERR_NOMEM;
  }
  p->fixed_mem = job.fixed;
  p->row_ptr = reinterpret_cast<int32_t*>(job.fixed + o_row);
  p->tile_ptr = reinterpret_cast<int32_t*>(job.fixed + o_tptr);
  p->tile_order = reinterpret_cast<int32_t*>(job.fixed + o_tord);
  p->retained_fx = reinterpret_cast<int64_t*>(job.fixed + o_ret);
  p->total_fx = reinterpret_cast<int64_t*>(job.fixed + o_tot);
  job.cut.tau_fx = job.tau_fx;
  job.cut.cut_key = reinterpret_cast<unsigned long long*>(job.scratch + s_cut);
  job.cut.count = reinterpret_cast<int*>(job.scratch + s_cnt);
  job.cut.retained_fx = reinterpret_cast<long long*>(p->retained_fx);
  job.cut.total_fx = reinterpret_cast<long long*>(p->total_fx);
  job.tcnt = reinterpret_cast<int*>(job.scratch + s_tcnt);
  job.hist = reinterpret_cast<int*>(job.scratch + s_hist);
  job.cursor = reinterpret_cast<int*>(job.scratch + s_cur);
  return LOSA_OK;
}

void select_abort(SelectJob& job) {
  if (job.fixed) cudaFreeAsync(job.fixed, job.stream);
  if (job.scratch) cudaFreeAsync(job.scratch, job.stream);
  if (job.p && job.p->list_mem) cudaFreeAsync(job.p->list_mem, job.stream);
  delete job.p;
  job = SelectJob{};
}

int select_end(const float* mass, bool run_cut, SelectJob& job, losa_pattern** out) {
  losa_pattern* p = job.p;
  cudaStream_t stream = job.stream;
  const int64_t R = job.R, T = job.T;
  const int n = job.n, qpt = job.qpt, n_qt = job.n_qt;
  int* status = device_status_word();
  if (!status) {
    select_abort(job);
    return LOSA_ERR_CUDA;
  }
  auto fail = [&](int code) {
    select_abort(job);
    return code;
  };
  unsigned long long* cut = job.cut.cut_key;
  int* cnt = job.cut.count;
  if (run_cut)
    launch_select_cut(mass, R, n, job.tau_fx, cut, cnt, job.cut.retained_fx, job.cut.total_fx,
                      status, stream);
  tile_count_kernel<<<unsigned(T), kSelThreads, 0, stream>>>(mass, cut, n, qpt, n_qt, job.tcnt);
  scan_kernel<<<1, 1024, 0, stream>>>(cnt, int(R), p->row_ptr);
  scan_kernel<<<1, 1024, 0, stream>>>(job.tcnt, int(T), p->tile_ptr);
  cudaMemsetAsync(job.hist, 0, job.n_keys * sizeof(int), stream);
  const int og = int(std::min<int64_t>((T + 255) / 256, 1024));
  order_hist_kernel<<<og, 256, 0, stream>>>(job.tcnt, int(T), n_qt, n, job.hist);
  scan_kernel<<<1, 1024, 0, stream>>>(job.hist, int(job.n_keys), job.cursor);
  order_scatter_kernel<<<og, 256, 0, stream>>>(job.tcnt, int(T), n_qt, n, job.cursor,
                                               p->tile_order);
  if (cudaGetLastError() != cudaSuccess) return fail(LOSA_ERR_CUDA);

  // The one host synchronisation: CSR sizes and the status word (a bad mass
  // value, or a wait a fused construction kernel gave up).
  int totals[2] = {0, 0};
  int host_status = 0;
  if (cudaMemcpyAsync(&totals[0], p->row_ptr + R, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(&totals[1], p->tile_ptr + T, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return fail(LOSA_ERR_CUDA);
  if (host_status != kStatusOk) {
    const int zero = 0;
    cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(host_status == kStatusBadMass ? LOSA_ERR_MASS : LOSA_ERR_TIMEOUT);
  }
  p->nnz = totals[0];
  p->tile_entries = totals[1];
  const size_t list_bytes = align256(size_t(p->nnz) * 4) + align256(size_t(p->tile_entries) * 4);
  char* lists = static_cast<char*>(pool_alloc(list_bytes, stream));
  if (!lists) return fail(LOSA_ERR_NOMEM);
  p->list_mem = lists;
  p->col_idx = reinterpret_cast<int32_t*>(lists);
  p->tile_entry = reinterpret_cast<int32_t*>(lists + align256(size_t(p->nnz) * 4));
  tile_write_kernel<<<unsigned(T), kSelThreads, 0, stream>>>(
      mass, cut, n, qpt, n_qt, p->row_ptr, p->tile_ptr, p->col_idx, p->tile_entry);
  if (cudaGetLastError() != cudaSuccess) return fail(LOSA_ERR_CUDA);
  cudaFreeAsync(job.scratch, stream);
  job = SelectJob{};
  *out = p;
  return LOSA_OK;
}

int build_pattern(const float* mass, int B, int H, int n, int block, double tau,
                  losa_pattern** out, cudaStream_t stream) {
  SelectJob job;
  const int st = select_begin(B, H, n, block, tau, stream, job);
  if (st != LOSA_OK) return st;
  return select_end(mass, /*run_cut=*/true, job, out);
}

int import_pattern(const int32_t* row_ptr, const int32_t* col_idx, const int64_t* retained_fx,
                   const int64_t* total_fx, int B, int H, int n, int block,
                   int64_t tile_entries, losa_pattern** out, cudaStream_t stream) {
  const int BH = B * H;
  const int64_t R = int64_t(BH) * n;
  const int L_pad = n * block;
  const int n_qt = (L_pad + 127) / 128;
  const int qpt = 128 / block;
  const int64_t T = int64_t(BH) * n_qt;
  const int64_t nnz = row_ptr[R];

  losa_pattern* p = new losa_pattern{};
  p->B = B;
  p->H = H;
  p->n_blocks = n;
  p->block = block;
  p->n_qt = n_qt;
  p->n_tiles = T;
  p->nnz = nnz;
  p->tile_entries = tile_entries;
  p->stream = stream;
  cudaGetDevice(&p->device);

  // Same arrays and layout as a selected pattern.
  const size_t o_row = 0;
  const size_t o_tptr = o_row + align256((R + 1) * 4);
  const size_t o_tord = o_tptr + align256((T + 1) * 4);
  const size_t o_ret = o_tord + align256(T * 4);
  const size_t o_tot = o_ret + align256(R * 8);
  const size_t fixed_bytes = o_tot + align256(R * 8);
  const size_t list_bytes = align256(size_t(nnz) * 4) + align256(size_t(tile_entries) * 4);
  const int64_t n_keys = int64_t(BH) * (n + 1);
  const size_t s_tcnt = 0;
  const size_t s_hist = s_tcnt + align256(T * 4);
  const size_t s_cur = s_hist + align256(n_keys * 4);
  const size_t scratch_bytes = s_cur + align256((n_keys + 1) * 4);

  char* fixed = static_cast<char*>(pool_alloc(fixed_bytes, stream));
  char* lists = static_cast<char*>(pool_alloc(list_bytes, stream));
  char* scratch = static_cast<char*>(pool_alloc(scratch_bytes, stream));
  auto fail = [&](int code) {
    if (fixed) cudaFreeAsync(fixed, stream);
    if (lists) cudaFreeAsync(lists, stream);
    if (scratch) cudaFreeAsync(scratch, stream);
    cudaStreamSynchronize(stream);
    delete p;
    return code;
  };
  if (!fixed || !lists || !scratch) return fail(LOSA_ERR_NOMEM);
  p->row_ptr = reinterpret_cast<int32_t*>(fixed + o_row);
  p->tile_ptr = reinterpret_cast<int32_t*>(fixed + o_tptr);
  p->tile_order = reinterpret_cast<int32_t*>(fixed + o_tord);
  p->retained_fx = reinterpret_cast<int64_t*>(fixed + o_ret);
  p->total_fx = reinterpret_cast<int64_t*>(fixed + o_tot);
  p->col_idx = reinterpret_cast<int32_t*>(lists);
  p->tile_entry = reinterpret_cast<int32_t*>(lists + align256(size_t(nnz) * 4));
  auto* tcnt = reinterpret_cast<int*>(scratch + s_tcnt);
  auto* hist = reinterpret_cast<int*>(scratch + s_hist);
  auto* cursor = reinterpret_cast<int*>(scratch + s_cur);

  bool ok = cudaMemcpyAsync(p->row_ptr, row_ptr, size_t(R + 1) * 4, cudaMemcpyHostToDevice,
                            stream) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(p->col_idx, col_idx, size_t(nnz) * 4, cudaMemcpyHostToDevice,
                             stream) == cudaSuccess;
  // Fixed-point sums are carried over when given, else marked unknown (-1).
  ok = ok && (retained_fx ? cudaMemcpyAsync(p->retained_fx, retained_fx, size_t(R) * 8,
                                            cudaMemcpyHostToDevice, stream)
                          : cudaMemsetAsync(p->retained_fx, 0xff, size_t(R) * 8, stream)) ==
                 cudaSuccess;
  ok = ok && (total_fx ? cudaMemcpyAsync(p->total_fx, total_fx, size_t(R) * 8,
                                         cudaMemcpyHostToDevice, stream)
                       : cudaMemsetAsync(p->total_fx, 0xff, size_t(R) * 8, stream)) ==
                 cudaSuccess;
  if (!ok) return fail(LOSA_ERR_CUDA);

  csr_tile_kernel<false><<<unsigned(T), kSelThreads, 0, stream>>>(
      p->row_ptr, p->col_idx, n, qpt, n_qt, tcnt, nullptr, nullptr);
  scan_kernel<<<1, 1024, 0, stream>>>(tcnt, int(T), p->tile_ptr);
  csr_tile_kernel<true><<<unsigned(T), kSelThreads, 0, stream>>>(
      p->row_ptr, p->col_idx, n, qpt, n_qt, nullptr, p->tile_ptr, p->tile_entry);
  cudaMemsetAsync(hist, 0, n_keys * sizeof(int), stream);
  const int og = int(std::min<int64_t>((T + 255) / 256, 1024));
  order_hist_kernel<<<og, 256, 0, stream>>>(tcnt, int(T), n_qt, n, hist);
  scan_kernel<<<1, 1024, 0, stream>>>(hist, int(n_keys), cursor);
  order_scatter_kernel<<<og, 256, 0, stream>>>(tcnt, int(T), n_qt, n, cursor, p->tile_order);
  if (cudaGetLastError() != cudaSuccess) return fail(LOSA_ERR_CUDA);
  cudaFreeAsync(scratch, stream);
  scratch = nullptr;
  // The caller may release its host arrays (pinned ones included) on return.
  if (cudaStreamSynchronize(stream) != cudaSuccess) return fail(LOSA_ERR_CUDA);
  p->fixed_mem = fixed;
  p->list_mem = lists;
  *out = p;
  return LOSA_OK;
}

}  // namespace losa

// ---------------------------------------------------------------------------
// Allocation-free selection (losa_select_noalloc): the cut and count kernels
// above, with their per-row scratch in a fixed device array instead of
// stream-ordered allocations, and the kept lists written straight into the
// caller's CSR buffers.

namespace losa {
namespace {

constexpr int kNoallocMaxRows = LOSA_NOALLOC_MAX_ROWS;
constexpr size_t kNoallocCutBytes = size_t(kNoallocMaxRows) * 8;
constexpr size_t kNoallocBytes = kNoallocCutBytes + size_t(kNoallocMaxRows) * 4;

// Per-row cut keys, then per-row kept counts. Every element a call reads is
// written earlier in the same call, so nothing needs clearing between calls.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side name is not a device address).
unsigned char* noalloc_scratch() {
  constexpr int kMaxDevices = 64;
  static unsigned char* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned char*>(p);
  }
  return addr[dev];
}

// One CTA per row: the row's kept key blocks, ascending, at row_ptr[row].
__global__ void __launch_bounds__(kSelThreads)
    row_write_kernel(const float* __restrict__ mass, int n,
                     const unsigned long long* __restrict__ cut_key,
                     const int* __restrict__ row_ptr, int* __restrict__ col_idx,
                     long long capacity) {
  using Scan = cub::BlockScan<int, kSelThreads>;
  __shared__ typename Scan::TempStorage tmp;
  const int row = blockIdx.x;
  const unsigned long long cut = cut_key[row];
  long long base = row_ptr[row];
  for (int c0 = 0; c0 < n; c0 += kSelThreads) {
    const int J = c0 + threadIdx.x;
    int keep = 0;
    if (J < n) {
      long long x;
      to_fixed(mass[size_t(row) * n + J], x);
      keep = sort_key(x, J) <= cut;
    }
    int ex, tot;
    Scan(tmp).ExclusiveSum(keep, ex, tot);
    __syncthreads();
    if (keep && base + ex < capacity) col_idx[base + ex] = J;
    base += tot;
  }
}

}  // namespace
}  // namespace losa

extern "C" int losa_select_noalloc(const float* mass, int B, int H, int n_blocks, double tau,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   int64_t* retained_fx, int64_t* total_fx, void* stream) {
  using namespace losa;
  if (!mass || !row_ptr || !col_idx || !retained_fx || !total_fx) return LOSA_ERR_ARG;
  if (B < 1 || H < 1 || n_blocks < 1 || n_blocks > 2047) return LOSA_ERR_ARG;
  const int64_t R = int64_t(B) * H * n_blocks;
  if (R > kNoallocMaxRows) return LOSA_ERR_ARG;
  if (!(tau > 0.0 && tau <= 1.0) || col_capacity < 0) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  unsigned char* scratch = noalloc_scratch();
  int* status = device_status_word();
  if (!scratch || !status) return LOSA_ERR_CUDA;
  auto* cut = reinterpret_cast<unsigned long long*>(scratch);
  auto* cnt = reinterpret_cast<int*>(scratch + kNoallocCutBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned long long tau_fx = (unsigned long long)llrint(tau * 281474976710656.0);
  launch_select_cut(mass, R, n_blocks, tau_fx, cut, cnt, (long long*)retained_fx,
                    (long long*)total_fx, status, s);
  scan_kernel<<<1, 1024, 0, s>>>(cnt, int(R), row_ptr);
  row_write_kernel<<<unsigned(R), kSelThreads, 0, s>>>(mass, n_blocks, cut, row_ptr, col_idx,
                                                       (long long)col_capacity);
  return cudaGetLastError() == cudaSuccess ? LOSA_OK : LOSA_ERR_CUDA;
}

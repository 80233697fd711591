// losa_internal.h - host-side declarations shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/losa.h"

struct losa_pattern {
  int B, H, n_blocks, block;
  int device;
  cudaStream_t stream;   // the stream the pattern was built on (frees go there)
  void* fixed_mem;       // row_ptr, tile_ptr, tile_order, retained_fx, total_fx
  void* list_mem;        // col_idx, tile_entry
  int64_t nnz;
  int64_t n_tiles;       // B*H*n_qt
  int64_t tile_entries;  // total union entries
  int n_qt;              // 128-row query tiles per head
  int32_t* row_ptr;
  int32_t* col_idx;
  int64_t* retained_fx;
  int64_t* total_fx;
  int32_t* tile_ptr;
  int32_t* tile_entry;
  int32_t* tile_order;
};

namespace losa {

// An NVTX range named after the C entry point for the call's duration, so a
// profiler's timeline shows the library's calls around their kernels (no
// cost when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// True when the current device is an sm_100 part (the only target built).
bool is_sm100();

// Device status word of the current device (lazily resolved per device).
int* device_status_word();

// The library's stream-ordered memory pool on the current device (created
// on first use, release threshold at maximum so steady-state calls reuse
// memory instead of mapping it again). Returns nullptr on failure.
cudaMemPool_t device_pool();

// Stream-ordered allocation from device_pool(); nullptr on failure.
void* pool_alloc(size_t bytes, cudaStream_t stream);

// Per-row outputs of the selection's threshold cut (device arrays of R =
// B*H*n entries) and the fixed-point threshold round(tau * 2^48).
struct CutOutputs {
  unsigned long long tau_fx;
  unsigned long long* cut_key;
  int* count;
  long long* retained_fx;
  long long* total_fx;
};

// Runs the dense two-pass construction kernel. q/k/v are bf16 device
// pointers, or fp32 ones already rounded to tf32 when tf32 is set; the
// arguments were validated by the caller. With `cut`, the kernel also runs
// the selection's cut on every mass row it wrote (the fused path).
cudaError_t launch_dense(const void* q, const void* k, const void* v, bool tf32, int BH, int L,
                         int L_pad, int d, int block, float scale, void* o, bool out_bf16,
                         float* lse, float* mass, cudaStream_t stream,
                         const CutOutputs* cut = nullptr);

// Runs the block-sparse kernel over pattern p (validated by the caller);
// q/k/v as for launch_dense.
cudaError_t launch_sparse(const void* q, const void* k, const void* v, bool tf32, int d, int L,
                          float scale, const losa_pattern* p, void* o, bool out_bf16,
                          float* lse, cudaStream_t stream);

// Wait limit (SM cycles) of the attention kernels launched after the call;
// 0 restores the default.
void set_wait_limit(long long cycles);

// One bounded mbarrier wait that must run out (diagnostic).
cudaError_t launch_wait_selftest(long long limit_cycles, cudaStream_t stream);

// y = 2^x with the FMA-pipe exp2 of the attention kernels (diagnostic).
cudaError_t launch_exp2_eval(const float* x, float* y, int64_t n, cudaStream_t stream);

// fp32 -> bf16 (round to nearest even) of n elements.
cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream);

// fp32 -> tf32 (round to nearest even, kept as fp32 with the 13 low mantissa
// bits zero) of n elements.
cudaError_t launch_f32_to_tf32(const float* src, float* dst, int64_t n, cudaStream_t stream);

// Builds the frozen pattern from a mass map (validated by the caller).
// Returns a losa_status.
int build_pattern(const float* mass, int B, int H, int n, int block, double tau,
                  losa_pattern** out, cudaStream_t stream);

// build_pattern in two halves, so that the construction kernel can run the
// per-row cut itself (losa_dense_mass_select): select_begin allocates the
// pattern and its scratch and exposes the cut's output arrays in `cut`;
// select_end runs the cut (unless it already ran), the tile lists and the
// tile order, synchronises once for the CSR size and completes the pattern.
// Both return a losa_status; on failure everything is released.
struct SelectJob {
  losa_pattern* p = nullptr;
  char* fixed = nullptr;
  char* scratch = nullptr;
  CutOutputs cut{};
  int* tcnt = nullptr;
  int* hist = nullptr;
  int* cursor = nullptr;
  int64_t R = 0, T = 0, n_keys = 0;
  int n = 0, n_qt = 0, qpt = 0;
  unsigned long long tau_fx = 0;
  cudaStream_t stream = nullptr;
};
int select_begin(int B, int H, int n, int block, double tau, cudaStream_t stream,
                 SelectJob& job);
int select_end(const float* mass, bool run_cut, SelectJob& job, losa_pattern** out);
void select_abort(SelectJob& job);

// Builds a pattern from a host CSR that the caller has validated (row_ptr
// monotone from 0 with non-empty rows, columns strictly ascending in
// [0, n)); tile_entries is the total of the 128-row tiles' union sizes.
// Returns a losa_status.
int import_pattern(const int32_t* row_ptr, const int32_t* col_idx, const int64_t* retained_fx,
                   const int64_t* total_fx, int B, int H, int n, int block,
                   int64_t tile_entries, losa_pattern** out, cudaStream_t stream);

}  // namespace losa

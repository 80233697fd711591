// losa_api.cu - the library's C ABI: argument checks, the per-device status
// word, the fp32 entry conversion, and pattern ownership.
#include <cmath>
#include <algorithm>
#include <climits>
#include <cstring>
#include <mutex>
#include <vector>

#include "losa_device.cuh"
#include "losa_internal.h"

namespace losa {

// One status word per device; kernels raise it on a timed-out wait or a
// bad mass value, losa_check_status / losa_select read and clear it.
__device__ int g_status_word;

int* device_status_word() {
  constexpr int kMaxDevices = 64;
  static int* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

cudaMemPool_t device_pool() {
  constexpr int kMaxDevices = 64;
  static cudaMemPool_t pools[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep = ~0ull;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = pool;
  }
  return pools[dev];
}

void* pool_alloc(size_t bytes, cudaStream_t stream) {
  cudaMemPool_t pool = device_pool();
  if (!pool) return nullptr;
  void* p = nullptr;
  if (cudaMallocFromPoolAsync(&p, bytes ? bytes : 16, pool, stream) != cudaSuccess) return nullptr;
  return p;
}

bool is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return false;
  return major == 10 && minor == 0;
}

namespace {

bool valid_dtype(int dt) { return dt == LOSA_BF16 || dt == LOSA_FP32; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by the attention calls.
bool valid_attn_shape(int B, int H, int L, int L_pad, int d, int block) {
  if (B < 1 || H < 1 || L < 1 || L > L_pad) return false;
  if (d != 64 && d != 128) return false;
  if (block != 32 && block != 64 && block != 128) return false;
  if (L_pad % block != 0 || L_pad - L >= block) return false;
  if (L_pad / block > 2047) return false;
  if (int64_t(B) * H > 65535) return false;
  return true;
}

// Checks a host CSR for losa_pattern_import: row_ptr[0] = 0, every row
// non-empty with at most n entries, columns strictly ascending in [0, n).
// Returns the total of the 128-row tiles' union sizes, or -1 when invalid.
int64_t validate_csr(const int32_t* row_ptr, const int32_t* col_idx, int BH, int n,
                     int block) {
  const int64_t R = int64_t(BH) * n;
  if (row_ptr[0] != 0) return -1;
  for (int64_t r = 0; r < R; ++r) {
    const int64_t len = int64_t(row_ptr[r + 1]) - row_ptr[r];
    if (len < 1 || len > n) return -1;
  }
  const int64_t nnz = row_ptr[R];
  if (nnz > int64_t(INT32_MAX)) return -1;
  for (int64_t r = 0; r < R; ++r) {
    int prev = -1;
    for (int64_t e = row_ptr[r]; e < row_ptr[r + 1]; ++e) {
      const int J = col_idx[e];
      if (J <= prev || J >= n) return -1;
      prev = J;
    }
  }
  // Union sizes: a key block counts once per tile (stamped with the tile).
  const int qpt = 128 / block;
  const int n_qt = (n * block + 127) / 128;
  std::vector<int64_t> stamp(size_t(n), -1);
  int64_t entries = 0;
  for (int bh = 0; bh < BH; ++bh)
    for (int qt = 0; qt < n_qt; ++qt) {
      const int64_t t = int64_t(bh) * n_qt + qt;
      const int I0 = qt * qpt;
      const int nq = std::min(qpt, n - I0);
      for (int q = 0; q < nq; ++q) {
        const int64_t r = int64_t(bh) * n + I0 + q;
        for (int64_t e = row_ptr[r]; e < row_ptr[r + 1]; ++e)
          if (stamp[col_idx[e]] != t) {
            stamp[col_idx[e]] = t;
            ++entries;
          }
      }
    }
  return entries;
}

// The operands the kernels read: bf16 inputs as given, or fp32 inputs
// rounded to tf32 (nearest even) on the stream into pool temporaries, for the
// kind::tf32 kernels.
struct KernelInputs {
  const void* q;
  const void* k;
  const void* v;
  bool tf32 = false;
  void* tmp = nullptr;
  cudaStream_t s;
  ~KernelInputs() {
    if (tmp) cudaFreeAsync(tmp, s);
  }
};

int prepare_inputs(KernelInputs& in, const void* q, const void* k, const void* v, int in_dtype,
                   int64_t n_elem) {
  if (in_dtype == LOSA_BF16) {
    in.q = q;
    in.k = k;
    in.v = v;
    return LOSA_OK;
  }
  const size_t bytes = size_t(n_elem) * 4;
  in.tmp = pool_alloc(3 * bytes, in.s);
  if (!in.tmp) return LOSA_ERR_NOMEM;
  float* base = static_cast<float*>(in.tmp);
  if (launch_f32_to_tf32(static_cast<const float*>(q), base, n_elem, in.s) != cudaSuccess ||
      launch_f32_to_tf32(static_cast<const float*>(k), base + n_elem, n_elem, in.s) != cudaSuccess ||
      launch_f32_to_tf32(static_cast<const float*>(v), base + 2 * n_elem, n_elem, in.s) != cudaSuccess)
    return LOSA_ERR_CUDA;
  in.q = base;
  in.k = base + n_elem;
  in.v = base + 2 * n_elem;
  in.tf32 = true;
  return LOSA_OK;
}

}  // namespace
}  // namespace losa

using namespace losa;

extern "C" {

int losa_dense_mass(const void* q, const void* k, const void* v, int in_dtype, int B, int H,
                    int L, int L_pad, int d, int block, float scale, void* o, int out_dtype,
                    float* lse, float* mass, void* stream) {
  NvtxRange nvtx_range("losa_dense_mass");
  if (!q || !k || !v || !o || !lse || !mass) return LOSA_ERR_ARG;
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return LOSA_ERR_ARG;
  if (!valid_attn_shape(B, H, L, L_pad, d, block)) return LOSA_ERR_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return LOSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  KernelInputs in;
  in.s = s;
  const int64_t n_elem = int64_t(B) * H * L_pad * d;
  int st = prepare_inputs(in, q, k, v, in_dtype, n_elem);
  if (st != LOSA_OK) return st;
  if (launch_dense(in.q, in.k, in.v, in.tf32, B * H, L, L_pad, d, block, scale, o,
                   out_dtype == LOSA_BF16, lse, mass, s) != cudaSuccess)
    return LOSA_ERR_CUDA;
  return LOSA_OK;
}

int losa_dense_mass_select(const void* q, const void* k, const void* v, int in_dtype, int B,
                           int H, int L, int L_pad, int d, int block, float scale, double tau,
                           void* o, int out_dtype, float* lse, float* mass, losa_pattern** out,
                           void* stream) {
  NvtxRange nvtx_range("losa_dense_mass_select");
  if (out) *out = nullptr;
  if (!q || !k || !v || !o || !lse || !mass || !out) return LOSA_ERR_ARG;
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return LOSA_ERR_ARG;
  if (!valid_attn_shape(B, H, L, L_pad, d, block)) return LOSA_ERR_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return LOSA_ERR_ARG;
  if (!(tau > 0.0 && tau <= 1.0)) return LOSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  KernelInputs in;
  in.s = s;
  const int64_t n_elem = int64_t(B) * H * L_pad * d;
  int st = prepare_inputs(in, q, k, v, in_dtype, n_elem);
  if (st != LOSA_OK) return st;
  SelectJob job;
  st = select_begin(B, H, L_pad / block, block, tau, s, job);
  if (st != LOSA_OK) return st;
  if (launch_dense(in.q, in.k, in.v, in.tf32, B * H, L, L_pad, d, block, scale, o,
                   out_dtype == LOSA_BF16, lse, mass, s, &job.cut) != cudaSuccess) {
    select_abort(job);
    return LOSA_ERR_CUDA;
  }
  return select_end(mass, /*run_cut=*/false, job, out);
}

int losa_select(const float* mass, int B, int H, int n_blocks, int block, double tau,
                losa_pattern** out, void* stream) {
  NvtxRange nvtx_range("losa_select");
  if (out) *out = nullptr;
  if (!mass || !out) return LOSA_ERR_ARG;
  if (B < 1 || H < 1 || n_blocks < 1 || n_blocks > 2047) return LOSA_ERR_ARG;
  if (block != 32 && block != 64 && block != 128) return LOSA_ERR_ARG;
  if (int64_t(B) * H > 65535) return LOSA_ERR_ARG;
  if (!(tau > 0.0 && tau <= 1.0)) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  return build_pattern(mass, B, H, n_blocks, block, tau, out, static_cast<cudaStream_t>(stream));
}

int losa_pattern_info(const losa_pattern* p, losa_pattern_view* view) {
  if (!p || !view) return LOSA_ERR_ARG;
  view->B = p->B;
  view->H = p->H;
  view->n_blocks = p->n_blocks;
  view->block = p->block;
  view->nnz = p->nnz;
  view->row_ptr = p->row_ptr;
  view->col_idx = p->col_idx;
  view->retained_fx = p->retained_fx;
  view->total_fx = p->total_fx;
  view->n_tiles = p->n_tiles;
  view->tile_entries = p->tile_entries;
  view->tile_ptr = p->tile_ptr;
  view->tile_entry = p->tile_entry;
  view->tile_order = p->tile_order;
  return LOSA_OK;
}

int losa_pattern_export(const losa_pattern* p, int32_t* row_ptr, int32_t* col_idx,
                        int64_t* retained_fx, int64_t* total_fx, int32_t* tile_ptr,
                        int32_t* tile_entry, int32_t* tile_order, void* stream) {
  NvtxRange nvtx_range("losa_pattern_export");
  if (!p) return LOSA_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t R = int64_t(p->B) * p->H * p->n_blocks;
  struct Item {
    void* dst;
    const void* src;
    size_t bytes;
  } items[] = {{row_ptr, p->row_ptr, size_t(R + 1) * 4},
               {col_idx, p->col_idx, size_t(p->nnz) * 4},
               {retained_fx, p->retained_fx, size_t(R) * 8},
               {total_fx, p->total_fx, size_t(R) * 8},
               {tile_ptr, p->tile_ptr, size_t(p->n_tiles + 1) * 4},
               {tile_entry, p->tile_entry, size_t(p->tile_entries) * 4},
               {tile_order, p->tile_order, size_t(p->n_tiles) * 4}};
  for (const Item& it : items) {
    if (!it.dst || it.bytes == 0) continue;
    if (cudaMemcpyAsync(it.dst, it.src, it.bytes, cudaMemcpyDefault, s) != cudaSuccess)
      return LOSA_ERR_CUDA;
  }
  return cudaStreamSynchronize(s) == cudaSuccess ? LOSA_OK : LOSA_ERR_CUDA;
}

int losa_pattern_import(const int32_t* row_ptr, const int32_t* col_idx,
                        const int64_t* retained_fx, const int64_t* total_fx, int B, int H,
                        int n_blocks, int block, losa_pattern** out, void* stream) {
  NvtxRange nvtx_range("losa_pattern_import");
  if (out) *out = nullptr;
  if (!row_ptr || !col_idx || !out) return LOSA_ERR_ARG;
  if (B < 1 || H < 1 || n_blocks < 1 || n_blocks > 2047) return LOSA_ERR_ARG;
  if (block != 32 && block != 64 && block != 128) return LOSA_ERR_ARG;
  if (int64_t(B) * H > 65535) return LOSA_ERR_ARG;
  const int64_t tile_entries = validate_csr(row_ptr, col_idx, B * H, n_blocks, block);
  if (tile_entries < 0) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  return import_pattern(row_ptr, col_idx, retained_fx, total_fx, B, H, n_blocks, block,
                        tile_entries, out, static_cast<cudaStream_t>(stream));
}

int losa_sparse_attn(const void* q, const void* k, const void* v, int in_dtype, int d, int L,
                     float scale, const losa_pattern* p, void* o, int out_dtype, float* lse,
                     void* stream) {
  NvtxRange nvtx_range("losa_sparse_attn");
  if (!q || !k || !v || !o || !p) return LOSA_ERR_ARG;
  if (!valid_dtype(in_dtype) || !valid_dtype(out_dtype)) return LOSA_ERR_ARG;
  const int L_pad = p->n_blocks * p->block;
  if (!valid_attn_shape(p->B, p->H, L, L_pad, d, p->block)) return LOSA_ERR_ARG;
  int dev = -1;
  // The pattern's arrays live on the device that built it.
  if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) return LOSA_ERR_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return LOSA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LOSA_ERR_ARG;
  if (!is_sm100()) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  KernelInputs in;
  in.s = s;
  const int64_t n_elem = int64_t(p->B) * p->H * L_pad * d;
  int st = prepare_inputs(in, q, k, v, in_dtype, n_elem);
  if (st != LOSA_OK) return st;
  if (launch_sparse(in.q, in.k, in.v, in.tf32, d, L, scale, p, o, out_dtype == LOSA_BF16, lse,
                    s) != cudaSuccess)
    return LOSA_ERR_CUDA;
  return LOSA_OK;
}

void losa_free(losa_pattern* p) {
  if (!p) return;
  NvtxRange nvtx_range("losa_free");
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->device);
  if (p->fixed_mem) cudaFreeAsync(p->fixed_mem, p->stream);
  if (p->list_mem) cudaFreeAsync(p->list_mem, p->stream);
  cudaSetDevice(prev);
  delete p;
}

int losa_check_status(void* stream) {
  NvtxRange nvtx_range("losa_check_status");
  int* w = device_status_word();
  if (!w) return LOSA_ERR_CUDA;
  int h = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, w, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return LOSA_ERR_CUDA;
  if (h != kStatusOk) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return LOSA_ERR_CUDA;
    return h == kStatusBadMass ? LOSA_ERR_MASS : LOSA_ERR_TIMEOUT;
  }
  return LOSA_OK;
}

int losa_selftest_wait(int64_t limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > (int64_t(1) << 33)) return LOSA_ERR_ARG;
  return launch_wait_selftest(limit_cycles, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LOSA_OK
             : LOSA_ERR_CUDA;
}

int losa_set_wait_limit(int64_t limit_cycles) {
  if (limit_cycles < 0 || limit_cycles > (int64_t(1) << 33)) return LOSA_ERR_ARG;
  set_wait_limit(limit_cycles);
  return LOSA_OK;
}

int losa_exp2_eval(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0) return LOSA_ERR_ARG;
  return launch_exp2_eval(x, y, n, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LOSA_OK
             : LOSA_ERR_CUDA;
}

const char* losa_strerror(int status) {
  switch (status) {
    case LOSA_OK: return "ok";
    case LOSA_ERR_ARG: return "invalid argument";
    case LOSA_ERR_CUDA: return "CUDA runtime error";
    case LOSA_ERR_NOMEM: return "device allocation failed";
    case LOSA_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case LOSA_ERR_MASS: return "mass entry is NaN, Inf, negative or >= 2";
    case LOSA_ERR_UNSUPPORTED: return "device is not sm_100";
    default: return "unknown status";
  }
}

const char* losa_version(void) { return "0.1.0"; }

}  // extern "C"

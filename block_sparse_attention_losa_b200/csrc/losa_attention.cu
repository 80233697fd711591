// losa_attention.cu - host launchers of the attention kernels: TMA tensor
// maps, kernel instantiation per (head dim, key tile, output dtype), and the
// fp32 -> bf16 entry conversion.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "losa_attention.cuh"
#include "losa_internal.h"

namespace losa {

// Wait limit of the attention kernels' mbarrier waits, in SM cycles.
std::atomic<long long> g_wait_limit{kWaitLimitCycles};

void set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : kWaitLimitCycles);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [BH, L_pad, d] bf16 (esz 2) or fp32 (esz 4) viewed as a 3D tensor (d
// innermost), loaded in 128-byte-wide slabs (64 bf16 or 32 fp32 columns) of
// `box_rows` rows with the 128-byte swizzle the MMA descriptors expect: of
// 16-byte atoms, or of 32-byte atoms (atom32) for an fp32 operand the tf32
// MMAs read MN-major (V). Rows past L_pad read as zero.
bool make_map(CUtensorMap* map, const void* base, int BH, int L_pad, int d, int box_rows,
              int esz, bool atom32 = false) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(L_pad), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d) * esz, cuuint64_t(L_pad) * d * esz};
  cuuint32_t box[3] = {cuuint32_t(128 / esz), cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BN, int NSK, int NSV, bool kDense, bool kOutBf16, int BLK, bool kTf32,
          bool kCut = false>
cudaError_t run(const void* q, const void* k, const void* v, int BH, AttnParams p,
                dim3 grid, cudaStream_t stream) {
  constexpr int ESZ = kTf32 ? 4 : 2;
  using Lay = AttnLayout<D, BN, NSK, NSV, ESZ>;
  auto kern = attn_kernel<D, BN, NSK, NSV, kDense, kOutBf16, BLK, kTf32, kCut>;
  // Cheap, and per device: set on every launch.
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM_ALLOC);
  if (err != cudaSuccess) return err;
  CUtensorMap tq, tk, tv;
  constexpr int box = kDense ? BN : (BLK < BN ? BLK : BN);
  if (!make_map(&tq, q, BH, p.L_pad, D, 128, ESZ) || !make_map(&tk, k, BH, p.L_pad, D, box, ESZ) ||
      !make_map(&tv, v, BH, p.L_pad, D, box, ESZ, kTf32))
    return cudaErrorInvalidValue;
  if (kDense) p.n_kv = (p.L_pad + BN - 1) / BN;
  kern<<<grid, kAttnThreads, Lay::SMEM_ALLOC, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

__global__ void f32_to_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                   int64_t n4) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 x = src[i];
    uint2 y;
    y.x = pack_bf16x2(x.x, x.y);
    y.y = pack_bf16x2(x.z, x.w);
    dst[i] = y;
  }
}

// fp32 -> tf32 (10-bit mantissa), round to nearest even, kept in fp32 with
// the 13 low mantissa bits zero: add half an ulp of the tf32 result (minus
// one when the kept part is even, so that ties go to even) and clear the
// dropped bits. NaN and Inf pass through.
__global__ void f32_to_tf32_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                   int64_t n4) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4;
       i += int64_t(gridDim.x) * blockDim.x) {
    uint4 x = src[i];
    uint32_t* u = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if ((u[c] & 0x7f800000u) != 0x7f800000u)
        u[c] = (u[c] + 0xfffu + ((u[c] >> 13) & 1u)) & 0xffffe000u;
    }
    dst[i] = x;
  }
}

__global__ void exp2_eval_kernel(const float* __restrict__ x, float* __restrict__ y,
                                 int64_t n) {
  for (int64_t i = 2 * (blockIdx.x * int64_t(blockDim.x) + threadIdx.x); i < n;
       i += 2 * int64_t(gridDim.x) * blockDim.x) {
    float y0, y1;
    exp2_fma2(x[i], i + 1 < n ? x[i + 1] : 0.f, y0, y1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
  }
}

// One bounded wait on an mbarrier nothing ever completes: it runs out after
// `limit` SM cycles, raises the status word and returns (diagnostic of the
// wait machinery every attention kernel uses).
__global__ void wait_selftest_kernel(int* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx wc{&abort_flag, status, limit};
    mbar_wait(&bar, 0, wc);
  }
}

}  // namespace

cudaError_t launch_wait_selftest(long long limit_cycles, cudaStream_t stream) {
  int* status = device_status_word();
  if (!status) return cudaErrorInvalidDevice;
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_cycles);
  return cudaGetLastError();
}

cudaError_t launch_exp2_eval(const float* x, float* y, int64_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>((n / 2 + 255) / 256 + 1, 148 * 8));
  exp2_eval_kernel<<<grid, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_tf32(const float* src, float* dst, int64_t n, cudaStream_t stream) {
  // n is a multiple of 64 (d in {64, 128}); 16-byte aligned pointers.
  const int64_t n4 = n / 4;
  const int grid = int(std::min<int64_t>((n4 + 255) / 256, 148 * 16));
  f32_to_tf32_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(src),
                                               reinterpret_cast<uint4*>(dst), n4);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* src, void* dst, int64_t n, cudaStream_t stream) {
  // n is a multiple of 64 (d in {64, 128}); 16-byte aligned pointers.
  const int64_t n4 = n / 4;
  const int grid = int(std::min<int64_t>((n4 + 255) / 256, 148 * 16));
  f32_to_bf16_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(src),
                                               reinterpret_cast<uint2*>(dst), n4);
  return cudaGetLastError();
}

cudaError_t launch_dense(const void* q, const void* k, const void* v, bool tf32, int BH, int L,
                         int L_pad, int d, int block, float scale, void* o, bool out_bf16,
                         float* lse, float* mass, cudaStream_t stream, const CutOutputs* cut) {
  AttnParams p{};
  p.L = L;
  p.L_pad = L_pad;
  p.n_qt = (L_pad + 127) / 128;
  p.n_kv = (L_pad + 127) / 128;
  p.block = block;
  p.n_blocks = L_pad / block;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o;
  p.lse = lse;
  p.mass = mass;
  if (cut) {
    p.tau_fx = cut->tau_fx;
    p.cut_key = cut->cut_key;
    p.cut_count = cut->count;
    p.retained_fx = cut->retained_fx;
    p.total_fx = cut->total_fx;
  }
  p.status = device_status_word();
  if (!p.status) return cudaErrorInvalidDevice;
  p.wait_limit = g_wait_limit.load();
  const dim3 grid((p.n_qt + 1) / 2, BH);  // two query tiles per CTA
// Shared memory per instance: bf16 d 128: 2 Q tiles (64 KB) + 3 K + 2 V
// stages of 128 keys (32 KB each); bf16 d 64: 32 KB + 4 + 4 stages of 16 KB;
// tf32 d 64: 64 KB + 3 + 2 stages of 32 KB; tf32 d 128: 128 KB + 2 K + 1 V
// stage of 64 keys (32 KB each).
// With a cut, the kCut instance (same kernel plus the fused selection cut).
#define LOSA_DENSE_CASE(TF_, D_, BN_, NSK_, NSV_, BLK_)                                          \
  if (tf32 == TF_ && d == D_ && block == BLK_) {                                                 \
    if (cut)                                                                                     \
      return out_bf16 ? run<D_, BN_, NSK_, NSV_, true, true, BLK_, TF_, true>(q, k, v, BH, p,    \
                                                                              grid, stream)      \
                      : run<D_, BN_, NSK_, NSV_, true, false, BLK_, TF_, true>(q, k, v, BH, p,   \
                                                                               grid, stream);    \
    return out_bf16                                                                              \
               ? run<D_, BN_, NSK_, NSV_, true, true, BLK_, TF_>(q, k, v, BH, p, grid, stream)   \
               : run<D_, BN_, NSK_, NSV_, true, false, BLK_, TF_>(q, k, v, BH, p, grid, stream); \
  }
  LOSA_DENSE_CASE(false, 128, 128, 3, 2, 128)
  LOSA_DENSE_CASE(false, 128, 128, 3, 2, 64)
  LOSA_DENSE_CASE(false, 128, 128, 3, 2, 32)
  LOSA_DENSE_CASE(false, 64, 128, 4, 4, 128)
  LOSA_DENSE_CASE(false, 64, 128, 4, 4, 64)
  LOSA_DENSE_CASE(false, 64, 128, 4, 4, 32)
  LOSA_DENSE_CASE(true, 128, 64, 2, 1, 128)
  LOSA_DENSE_CASE(true, 128, 64, 2, 1, 64)
  LOSA_DENSE_CASE(true, 128, 64, 2, 1, 32)
  LOSA_DENSE_CASE(true, 64, 128, 3, 2, 128)
  LOSA_DENSE_CASE(true, 64, 128, 3, 2, 64)
  LOSA_DENSE_CASE(true, 64, 128, 3, 2, 32)
#undef LOSA_DENSE_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_sparse(const void* q, const void* k, const void* v, bool tf32, int d, int L,
                          float scale, const losa_pattern* pat, void* o, bool out_bf16,
                          float* lse, cudaStream_t stream) {
  AttnParams p{};
  p.L = L;
  p.L_pad = pat->n_blocks * pat->block;
  p.n_qt = pat->n_qt;
  p.n_kv = 0;
  p.block = pat->block;
  p.n_blocks = pat->n_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o;
  p.lse = lse;
  p.mass = nullptr;
  p.tile_ptr = pat->tile_ptr;
  p.tile_entry = pat->tile_entry;
  p.tile_order = pat->tile_order;
  p.status = device_status_word();
  if (!p.status) return cudaErrorInvalidDevice;
  p.wait_limit = g_wait_limit.load();
  const int BH = pat->B * pat->H;
  p.n_tiles = int(pat->n_tiles);
  const dim3 grid(unsigned((pat->n_tiles + 1) / 2));  // two tiles per CTA
  if (pat->n_tiles == 0) return cudaSuccess;
#define LOSA_SPARSE_CASE(TF_, D_, BN_, NSK_, NSV_, BLK_)                                        \
  if (tf32 == TF_ && d == D_ && pat->block == BLK_)                                             \
    return out_bf16                                                                             \
               ? run<D_, BN_, NSK_, NSV_, false, true, BLK_, TF_>(q, k, v, BH, p, grid, stream) \
               : run<D_, BN_, NSK_, NSV_, false, false, BLK_, TF_>(q, k, v, BH, p, grid, stream);
  LOSA_SPARSE_CASE(false, 128, 128, 3, 2, 128)
  LOSA_SPARSE_CASE(false, 128, 128, 3, 2, 64)
  LOSA_SPARSE_CASE(false, 128, 128, 3, 2, 32)
  LOSA_SPARSE_CASE(false, 64, 128, 4, 4, 128)
  LOSA_SPARSE_CASE(false, 64, 128, 4, 4, 64)
  LOSA_SPARSE_CASE(false, 64, 128, 4, 4, 32)
  LOSA_SPARSE_CASE(true, 128, 64, 2, 1, 128)
  LOSA_SPARSE_CASE(true, 128, 64, 2, 1, 64)
  LOSA_SPARSE_CASE(true, 128, 64, 2, 1, 32)
  LOSA_SPARSE_CASE(true, 64, 128, 3, 2, 128)
  LOSA_SPARSE_CASE(true, 64, 128, 3, 2, 64)
  LOSA_SPARSE_CASE(true, 64, 128, 3, 2, 32)
#undef LOSA_SPARSE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace losa

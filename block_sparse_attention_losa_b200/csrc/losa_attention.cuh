// losa_attention.cuh - the attention kernels of the LoSA hot path (sm_100a).
//
// One CTA owns two 128-row query tiles and walks, for each, a list of key
// tiles. Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile 0 (thread r owns query row r = TMEM lane r),
//   warps 4-7  softmax of tile 1,
//   warp 8     TMA producer: Q tiles, then K and V tiles through smem rings,
//   warp 9     MMA issuer (one thread) and TMEM owner,
//   warps 10-11 idle.
// The kernel launches with 168 registers per thread (384 x 168 = 64,512);
// the third warpgroup gives registers back (setmaxnreg to 72) and the two
// softmax warpgroups take them (to 216): 2*128*216 + 128*72 = 64,512.
// TMEM (512 columns): S_t at columns [128 t, 128 t + BN), O_t at 256 + t D.
// Per key tile j of tile t: S_t = Q_t K_j^T (tcgen05 kind::f16, bf16 operands
// from 128B-swizzled smem, fp32 in TMEM); the softmax warps read S_t, write
// the bf16 weights P_t back over the first BN/2 columns of S_t, and the MMA
// thread accumulates O_t += P_t V_j with P_t read straight from TMEM. The MMA
// thread interleaves the two tiles - PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) -
// so the tensor core works on one tile while the other tile's softmax runs.
//
// kDense = true is the construction step: both tiles are adjacent query tiles
// of one head and share every K/V tile. Pass 1 is the flash forward over all
// key tiles (O, row lse); pass 2 recomputes S = Q K^T tile by tile and sums
// exp(s - lse) over each (query block, key block) straight into the mass map
// (LoSA abstract, arXiv 2608.12032: exact block attention masses at one early
// dense step; ubos.tech LoSA post, Phase 1 - Dense Calibration).
// kDense = false is the sparse step: the two tiles are independent work
// items with their own lists (the union of their query blocks' retained key
// blocks), each row masked to its own query block's set (ubos.tech LoSA
// post, Phase 3 - Repeated Sparse Inference).
#pragma once

#include "losa_cut.cuh"
#include "losa_device.cuh"

namespace losa {

struct AttnParams {
  int L;          // valid tokens
  int L_pad;      // padded tokens (multiple of block)
  int n_qt;       // query tiles per head = ceil(L_pad / 128)
  int n_kv;       // key tiles per pass (dense)
  int n_tiles;    // sparse: number of tiles in tile_order
  int block;      // LoSA block size b
  int n_blocks;   // L_pad / block
  float scale_log2;  // softmax scale * log2(e)
  void* o;
  float* lse;        // may be null (sparse)
  float* mass;       // dense only
  const int* tile_ptr;    // sparse only
  const int* tile_entry;  // sparse only
  const int* tile_order;  // sparse only
  int* status;
  long long wait_limit;   // SM cycles a wait spins before it gives up
  // Fused selection cut (the construction kernel's kCut instances): per
  // mass row the cut key, kept count and fixed-point sums of the threshold
  // tau_fx = round(tau * 2^48), as losa_select's cut computes them.
  unsigned long long tau_fx;
  unsigned long long* cut_key;
  int* cut_count;
  long long* retained_fx;
  long long* total_fx;
};

// ESZ: bytes per operand element (2 = bf16, 4 = fp32 read as tf32). Every
// tile is stored as 128-byte-wide slabs (128 / ESZ columns each).
template <int D, int BN, int NSK, int NSV, int ESZ = 2>
struct AttnLayout {
  static constexpr int BM = 128;
  static constexpr int NT = 2;                           // query tiles per CTA
  static constexpr int Q_BYTES = BM * D * ESZ;           // one tile: D*ESZ/128 slabs of 16 KB
  static constexpr int KV_BYTES = BN * D * ESZ;          // D*ESZ/128 slabs of BN*128 B
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NSV * KV_BYTES;
  // q_full[2], k_full/k_empty[NSK], v_full/v_empty[NSV], s_full[2], s_free[2],
  // p_full[2], o_full[2], red_bar[2][2], drain; then, for the double-buffered
  // mass pass, s2_full[2][2], s2_free[2][2], o_read[2]
  static constexpr int N_BARS = 2 + 2 * NSK + 2 * NSV + 8 + 4 + 1 + 10;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem addr, abort flag
  static constexpr int OFF_RED = OFF_MISC + 16;          // float red[2 tiles][2][4 warps][4]
  static constexpr int BYTES = OFF_RED + 2 * 2 * 4 * 4 * 4;
  // Slack for 1 KB alignment; never below 120 KB, so that two CTAs cannot
  // share an SM (each CTA allocates all 512 TMEM columns).
  static constexpr int SMEM_ALLOC = BYTES + 1024 > 120 * 1024 ? BYTES + 1024 : 120 * 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr int TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + D;
  // Second S buffer of each tile in the construction kernel's mass pass,
  // where O is dead (stored by the epilogue): at D = 128 O_t's own columns;
  // at D = 64 the unused columns [384, 512) for tile 0 and both O regions
  // [256, 384) for tile 1.
  static constexpr int TMEM_ALT0 = D == 128 ? 256 : 384;
  static constexpr int TMEM_ALT1 = D == 128 ? 384 : 256;
  static_assert(D % 64 == 0 && D <= 128, "head dim must be 64 or 128");
  static_assert(BN % 32 == 0 && BN <= 128, "key tile must be 32, 64 or 128");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "1 KB alignment");
  static_assert(KV_BYTES % 1024 == 0, "1 KB alignment of stages");
  static_assert(SMEM_ALLOC > 116 * 1024, "all of TMEM per CTA needs one CTA per SM");
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
};

// Of every 16 column pairs, how many take exp2 on the FMA pipe (the rest
// use MUFU ex2). Measured on B200: the flash softmax (both head dims) is
// not limited by MUFU throughput, so moving work to the FMA pipe only adds
// instructions there; the mass pass is, and gains from moving 7 of 16.
template <int D> constexpr int poly_pairs_flash() { return 0; }
template <int D> constexpr int poly_pairs_mass() { return 7; }

// Workspace of one warpgroup's fused selection cut, at the start of the
// (by then free) operand staging memory.
constexpr int kCutSmemStride = 32768;
static_assert(sizeof(cut::BucketSmem) <= kCutSmemStride, "cut workspace");

// The fused cut of one warpgroup's mass rows: rows I0 .. I0 + nq - 1 of
// head bh (those below n_blocks), tid the thread's index in the warpgroup
// of tile t. Kept out of line, so that the kernel's main loops are compiled
// as in the instances without it.
__device__ __noinline__ void fused_cut_rows(const float* mass, int n, unsigned long long tau_fx,
                                            unsigned long long* cut_key, int* count,
                                            long long* retained_fx, long long* total_fx,
                                            int* status, cut::BucketSmem* sm, int t, int tid,
                                            int bh, int I0, int nq) {
  const WarpgroupSync wg_sync{2 + t};
  for (int q = 0; q < nq; ++q) {
    const int I = I0 + q;
    if (I >= n) break;
    const int64_t mr = int64_t(bh) * n + I;
    cut::bucket_cut_row<128>(mass + mr * n, n, tau_fx, *sm, tid, wg_sync, mr, cut_key, count,
                             retained_fx, total_fx, status);
  }
}

constexpr int kAttnThreads = 384;
constexpr int kAttnLaunchRegs = 168;   // checked against ptxas at build time
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs == kAttnThreads * kAttnLaunchRegs,
              "register split must use exactly the launch allocation");

// BLK: the LoSA block size b (compile time, so that every per-block array
// stays in registers). Dense: key tiles of BN rows, one TMA box each; the
// mass pass sums over b x b blocks (a block wider than a key tile is summed
// over CPE consecutive tiles). Sparse: each BN-key iteration packs EPI =
// BN / b consecutive entries of the tile's list into one K/V stage (one b-row
// box each, stacked), so the tensor core runs N = BN; an entry wider than BN
// takes CPE = b / BN iterations.
// kTf32: Q, K, V are fp32 (already rounded to tf32) and every MMA is
// kind::tf32; the weights P stay fp32 in TMEM as the tf32 A operand of P V.
template <int D, int BN, int NSK, int NSV, bool kDense, bool kOutBf16, int BLK, bool kTf32,
          bool kCut = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int ESZ = kTf32 ? 4 : 2;       // bytes per operand element
  using Lay = AttnLayout<D, BN, NSK, NSV, ESZ>;
  constexpr int BM = Lay::BM;
  constexpr int SLAB_COLS = 128 / ESZ;     // operand columns per 128-byte slab
  constexpr int N_SLABS = D / SLAB_COLS;
  constexpr int BOX = kDense ? BN : (BLK < BN ? BLK : BN);  // key rows per TMA box
  constexpr int EPI = BN / BOX;            // boxes (list entries) per key stage
  constexpr int CPE = BLK > BN ? BLK / BN : 1;  // key stages per list entry / key block
  constexpr int K_STEP = 32 / ESZ;         // K of one MMA instruction (32 bytes of a row)
  static_assert((BN % BLK == 0 || BLK % BN == 0) && BLK % 32 == 0, "block size");
  // The construction kernel's mass pass double-buffers S (the second buffer
  // in columns O no longer needs) at b = 128, where that measured faster;
  // at b = 32 and 64 the single buffer measured faster.
  constexpr bool kDblMass = kDense && BLK == 128;
  static_assert(!kCut || (kDense && 2 * kCutSmemStride <= Lay::OFF_BAR),
                "the fused cut runs in the construction kernel, in its staging memory");
  constexpr uint32_t IDESC_S = kTf32 ? idesc_tf32_f32(BM, BN, false, false)
                                     : idesc_bf16_f32(BM, BN, false, false);
  constexpr uint32_t IDESC_PV = kTf32 ? idesc_tf32_f32(BM, D, false, true)
                                      : idesc_bf16_f32(BM, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;             // [2]
  uint64_t* k_full = q_full + 2;       // [NSK]
  uint64_t* k_empty = k_full + NSK;    // [NSK]
  uint64_t* v_full = k_empty + NSK;    // [NSV]
  uint64_t* v_empty = v_full + NSV;    // [NSV]
  uint64_t* s_full = v_empty + NSV;    // [2] MMA -> softmax t: S_t ready
  uint64_t* s_free = s_full + 2;       // [2] softmax t -> MMA: S_t read (pass 2)
  uint64_t* p_full = s_free + 2;       // [2] softmax t -> MMA: P_t in TMEM
  uint64_t* o_full = p_full + 2;       // [2] MMA -> softmax t: last PV_t done
  uint64_t* red_bar = o_full + 2;      // [2][2] softmax t: mass reduction
  uint64_t* drain_bar = red_bar + 4;   // MMA drain after an abort
  uint64_t* s2_full = drain_bar + 1;   // [2][2] MMA -> softmax t: S_t buffer ready (kDblMass)
  uint64_t* s2_free = s2_full + 4;     // [2][2] softmax t -> MMA: S_t buffer read (kDblMass)
  uint64_t* o_read = s2_free + 4;      // [2] softmax t -> MMA: O_t read (kDblMass)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + Lay::OFF_RED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work items: per tile t, its head, query tile and key list
  int bh[2], qt[2], e_begin[2] = {0, 0}, n_ent[2] = {0, 0}, n_it[2];
  if constexpr (kDense) {
    bh[0] = bh[1] = blockIdx.y;
    qt[0] = 2 * blockIdx.x;
    qt[1] = 2 * blockIdx.x + 1;  // may lie past the head: rows read as 0, nothing stored
    n_it[0] = n_it[1] = p.n_kv;
  } else {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int idx = 2 * blockIdx.x + t;
      if (idx < p.n_tiles) {
        const int tile = p.tile_order[idx];
        bh[t] = tile / p.n_qt;
        qt[t] = tile - bh[t] * p.n_qt;
        e_begin[t] = p.tile_ptr[tile];
        n_ent[t] = p.tile_ptr[tile + 1] - e_begin[t];
        n_it[t] = CPE * ((n_ent[t] + EPI - 1) / EPI);
      } else {
        bh[t] = 0;
        qt[t] = 0;
        n_it[t] = 0;
      }
    }
  }

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 128);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
      mbar_init(&red_bar[2 * t], 128);
      mbar_init(&red_bar[2 * t + 1], 128);
    }
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(drain_bar, 1);
    if (kDblMass) {
      for (int i = 0; i < 4; ++i) {
        mbar_init(&s2_full[i], 1);
        mbar_init(&s2_free[i], 128);
      }
      mbar_init(&o_read[0], 128);
      mbar_init(&o_read[1], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, Lay::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status, p.wait_limit};

  if (warp >= 8) {
  reg_dealloc<kControlRegs>();
  if (warp == 8) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        mbar_arrive_expect_tx(&q_full[t], Lay::Q_BYTES);
#pragma unroll
        for (int s = 0; s < N_SLABS; ++s)
          tma_load_3d(sQ + t * Lay::Q_BYTES + s * (BM * 128), &tm_q, &q_full[t],
                      s * SLAB_COLS, qt[t] * BM, bh[t]);
      }
      int kc = 0, vc = 0;
      bool ok = true;
      // One stage = BN keys = EPI boxes of BOX rows, stacked in each slab.
      auto load_k = [&](const int (&key_row)[EPI], int head) -> bool {
        const int ks = kc % NSK;
        if (!mbar_wait(&k_empty[ks], ((kc / NSK) & 1) ^ 1, wc)) return false;
        mbar_arrive_expect_tx(&k_full[ks], Lay::KV_BYTES);
#pragma unroll
        for (int s = 0; s < N_SLABS; ++s)
#pragma unroll
          for (int e = 0; e < EPI; ++e)
            tma_load_3d(sK + ks * Lay::KV_BYTES + s * (BN * 128) + e * (BOX * 128), &tm_k,
                        &k_full[ks], s * SLAB_COLS, key_row[e], head);
        ++kc;
        return true;
      };
      auto load_v = [&](const int (&key_row)[EPI], int head) -> bool {
        const int vs = vc % NSV;
        if (!mbar_wait(&v_empty[vs], ((vc / NSV) & 1) ^ 1, wc)) return false;
        mbar_arrive_expect_tx(&v_full[vs], Lay::KV_BYTES);
#pragma unroll
        for (int s = 0; s < N_SLABS; ++s)
#pragma unroll
          for (int e = 0; e < EPI; ++e)
            tma_load_3d(sV + vs * Lay::KV_BYTES + s * (BN * 128) + e * (BOX * 128), &tm_v,
                        &v_full[vs], s * SLAB_COLS, key_row[e], head);
        ++vc;
        return true;
      };
      if constexpr (kDense) {
        for (int j = 0; ok && j < p.n_kv; ++j) {
          const int rows[EPI] = {j * BN};
          ok = load_k(rows, bh[0]) && load_v(rows, bh[0]);
        }
        for (int j = 0; ok && j < p.n_kv; ++j) {
          const int rows[EPI] = {j * BN};
          ok = load_k(rows, bh[0]);
        }
      } else {
        const int n_max = max(n_it[0], n_it[1]);
        for (int j = 0; ok && j < n_max; ++j) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (ok && j < n_it[t]) {
              // Box e of iteration j: list entry j * EPI + e, or, for an
              // entry wider than a stage, chunk j % CPE of entry j / CPE.
              // Slots past the end of the list repeat its last entry (valid,
              // finite data); the softmax masks those columns.
              int rows[EPI];
#pragma unroll
              for (int e = 0; e < EPI; ++e) {
                const int idx = CPE > 1 ? j / CPE : j * EPI + e;
                rows[e] = (p.tile_entry[e_begin[t] + min(idx, n_ent[t] - 1)] & 0xFFFF) * BLK +
                          (CPE > 1 ? (j % CPE) * BN : 0);
              }
              ok = load_k(rows, bh[t]) && load_v(rows, bh[t]);
            }
          }
        }
      }
      if (!ok) {
        // Aborted: wait (bounded) for the copies still in flight before the
        // CTA releases its shared memory.
        mbar_wait_drain(&q_full[0], 0);
        mbar_wait_drain(&q_full[1], 0);
        for (int i = (kc > NSK ? kc - NSK : 0); i < kc; ++i) mbar_wait_drain(&k_full[i % NSK], (i / NSK) & 1);
        for (int i = (vc > NSV ? vc - NSV : 0); i < vc; ++i) mbar_wait_drain(&v_full[i % NSV], (i / NSV) & 1);
      } else {
        // A tile slot with no work (the last CTA of an odd tile count):
        // nobody else waits for its Q copy, so let it land before exit.
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (n_it[t] == 0) mbar_wait_drain(&q_full[t], 0);
      }
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_addr(sQ);
      const uint32_t k_base = smem_addr(sK);
      const uint32_t v_base = smem_addr(sV);
      int kc = 0, vc = 0;
      int pc[2] = {0, 0};  // P_t consumed (pass 1)
      int fc[2] = {0, 0};  // S_t uses in pass 2
      bool ok = true;
      bool q_ready[2] = {false, false};
      // S_t = Q_t K^T into TMEM columns col (S_t's own by default), from K
      // stage ks; `done` (s_full[t] by default) is committed when it completes.
      auto issue_s = [&](int t, int ks, int col = -1, uint64_t* done = nullptr) -> bool {
        if (!q_ready[t]) {
          if (!mbar_wait(&q_full[t], 0, wc)) return false;
          q_ready[t] = true;
        }
        tc_fence_after();
        const uint32_t qb = q_base + t * Lay::Q_BYTES;
        const uint32_t d_tmem = tmem + (col >= 0 ? col : (t ? Lay::TMEM_S1 : Lay::TMEM_S0));
        // 32 bytes of K per instruction: four steps per 128-byte slab.
#pragma unroll
        for (int kk = 0; kk < D / K_STEP; ++kk) {
          const uint64_t a = sdesc_sw128(qb + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(k_base + ks * Lay::KV_BYTES + (kk >> 2) * (BN * 128) +
                                             (kk & 3) * 32, 16, 1024);
          if constexpr (kTf32)
            umma_tf32_ss(d_tmem, a, b, IDESC_S, kk > 0 ? 1u : 0u);
          else
            umma_bf16_ss(d_tmem, a, b, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(done ? done : &s_full[t]);
        return true;
      };
      auto wait_k = [&](int& ks) -> bool {
        ks = kc % NSK;
        return mbar_wait(&k_full[ks], (kc / NSK) & 1, wc);
      };
      auto release_k = [&](int ks) {
        umma_commit(&k_empty[ks]);
        ++kc;
      };
      // O_t += P_t V (P_t from TMEM), from V stage vs.
      auto issue_pv = [&](int t, int vs) -> bool {
        if (!mbar_wait(&p_full[t], pc[t] & 1, wc)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + (t ? Lay::TMEM_S1 : Lay::TMEM_S0);
        const uint32_t d_tmem = tmem + (t ? Lay::TMEM_O1 : Lay::TMEM_O0);
        // K_STEP keys per instruction: 8 TMEM columns of P (two bf16 or one
        // fp32 per column) and K_STEP 128-byte rows of V. V is the MN-major
        // operand: 128-byte swizzle (8-row groups 1 KB apart) for bf16, the
        // 32-byte-atom 128-byte swizzle (4-row groups 512 B apart) for tf32.
#pragma unroll
        for (int kk = 0; kk < BN / K_STEP; ++kk) {
          const uint32_t vaddr = v_base + vs * Lay::KV_BYTES + kk * (K_STEP * 128);
          if constexpr (kTf32)
            umma_tf32_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128_32b(vaddr, BN * 128, 512), IDESC_PV,
                         (pc[t] > 0 || kk > 0) ? 1u : 0u);
          else
            umma_bf16_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(vaddr, BN * 128, 1024), IDESC_PV,
                         (pc[t] > 0 || kk > 0) ? 1u : 0u);
        }
        ++pc[t];
        return true;
      };
      auto wait_v = [&](int& vs) -> bool {
        vs = vc % NSV;
        return mbar_wait(&v_full[vs], (vc / NSV) & 1, wc);
      };
      auto release_v = [&](int vs) {
        umma_commit(&v_empty[vs]);
        ++vc;
      };

      if constexpr (kDense) {
        const int n = p.n_kv;
        int ks, vs;
        // ---- pass 1
        ok = wait_k(ks) && issue_s(0, ks) && issue_s(1, ks);
        if (ok) release_k(ks);
        for (int j = 0; ok && j < n; ++j) {
          if (!(ok = wait_v(vs))) break;
          if (!(ok = issue_pv(0, vs))) break;
          int ks2 = -1;
          if (j + 1 < n) {
            if (!(ok = wait_k(ks2) && issue_s(0, ks2))) break;
          } else {
            umma_commit(&o_full[0]);
          }
          if (!(ok = issue_pv(1, vs))) break;
          release_v(vs);
          if (j + 1 < n) {
            if (!(ok = issue_s(1, ks2))) break;
            release_k(ks2);
          } else {
            umma_commit(&o_full[1]);
          }
        }
        if constexpr (kDblMass) {
          // ---- pass 2, double-buffered: S_t(j) goes to buffer j & 1 (S_t's
          // own columns, or the second buffer, free once the epilogue has
          // read the O columns it overlaps), so S_t(j + 1) is computed while
          // softmax t sums S_t(j). A buffer is reused once softmax t has read
          // the S it held two key tiles before.
          for (int j = 0; ok && j < n; ++j) {
            if (!(ok = wait_k(ks))) break;
            const int bsel = j & 1;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (ok && j >= 2) ok = mbar_wait(&s2_free[2 * t + bsel], ((j >> 1) - 1) & 1, wc);
              if (ok && j == 1) {
                if constexpr (D == 128) {
                  ok = mbar_wait(&o_read[t], 0, wc);
                } else if (t == 1) {
                  ok = mbar_wait(&o_read[0], 0, wc) && mbar_wait(&o_read[1], 0, wc);
                }
              }
              if (ok)
                ok = issue_s(t, ks, bsel ? (t ? Lay::TMEM_ALT1 : Lay::TMEM_ALT0)
                                         : (t ? Lay::TMEM_S1 : Lay::TMEM_S0),
                             &s2_full[2 * t + bsel]);
            }
            if (!ok) break;
            release_k(ks);
          }
        } else {
          // ---- pass 2: S only; S_t is free again once softmax t has read it
          for (int j = 0; ok && j < n; ++j) {
            if (!(ok = wait_k(ks))) break;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (ok && fc[t] > 0) ok = mbar_wait(&s_free[t], (fc[t] - 1) & 1, wc);
              if (ok) ok = issue_s(t, ks);
              ++fc[t];
            }
            if (!ok) break;
            release_k(ks);
          }
        }
      } else {
        int ks, vs;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (ok && n_it[t] > 0) {
            ok = wait_k(ks) && issue_s(t, ks);
            if (ok) release_k(ks);
          }
        }
        const int n_max = max(n_it[0], n_it[1]);
        for (int j = 0; ok && j < n_max; ++j) {
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (!ok || j >= n_it[t]) continue;
            ok = wait_v(vs) && issue_pv(t, vs);
            if (!ok) break;
            release_v(vs);
            if (j + 1 < n_it[t]) {
              ok = wait_k(ks) && issue_s(t, ks);
              if (!ok) break;
              release_k(ks);
            } else {
              umma_commit(&o_full[t]);
            }
          }
        }
      }
      if (!ok) {
        // Drain: let every MMA issued so far finish before TMEM is freed.
        umma_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0);
      }
    }
  }
  } else {
    reg_alloc<kSoftmaxRegs>();
    // ================================================================ softmax warps
    const int t = warp >> 2;               // query tile of this warpgroup
    const int wl = warp & 3;               // warp within the warpgroup
    const int r = wl * 32 + lane;          // row within the tile, TMEM lane
    const int row = qt[t] * BM + r;        // token row within the head
    const uint32_t lane_base = uint32_t(wl * 32) << 16;
    const uint32_t s_col = tmem + lane_base + (t ? Lay::TMEM_S1 : Lay::TMEM_S0);
    const uint32_t o_col = tmem + lane_base + (t ? Lay::TMEM_O1 : Lay::TMEM_O0);
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const int n_iter = n_it[t];
    const int n = kDense ? n_iter : n_ent[t];  // list entries (sparse)
    // Running row max in log2 units. It is raised as soon as a tile exceeds
    // it, so every weight is <= 1 and the row's largest weight is exactly
    // 1.0, which bf16 represents exactly: the bf16 rounding of P then only
    // touches the smaller weights, and O normalised by the fp32 sum stays
    // within a few 1e-3 of fp64 (measured: max 0.0037 on the test shapes).
    float m_used = NEG_INF;
    // Running sum of exp2(s*sl2 - m_used) in fp32 (gives O's normaliser and
    // lse). A row sums ~10^5 terms, so each tile's terms are summed first
    // and the tile sums are accumulated with Kahan compensation (a plain
    // running sum loses the small terms against the large total).
    float l = 0.f, l_c = 0.f;
    int sc = 0;              // S_t completions seen
    bool ok = true;

    // List entries run one iteration ahead: those of iteration j + 1 are
    // fetched at the top of iteration j, so their global-load latency hides
    // behind a whole iteration. Past the end of the list: 0 (all rows off).
    int ent_next[EPI];
    if constexpr (!kDense) {
#pragma unroll
      for (int e = 0; e < EPI; ++e)
        ent_next[e] = (e < n) ? __ldg(p.tile_entry + e_begin[t] + e) : 0;
    }
    for (int j = 0; j < n_iter; ++j) {
      int ent[EPI];
      if constexpr (!kDense) {
#pragma unroll
        for (int e = 0; e < EPI; ++e) {
          ent[e] = ent_next[e];
          const int idx = CPE > 1 ? (j + 1) / CPE : (j + 1) * EPI + e;
          ent_next[e] = (idx < n) ? __ldg(p.tile_entry + e_begin[t] + idx) : 0;
        }
      }
      if (!mbar_wait(&s_full[t], sc & 1, wc)) { ok = false; break; }
      ++sc;
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(s_col + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
      tmem_ld_wait();

      // Key padding (only in the head's last key block) masks columns of S;
      // a sparse entry whose query block does not keep it is masked as a
      // whole through its exponent offset below, leaving S untouched.
      bool on[EPI];
      if constexpr (kDense) {
        on[0] = true;
        const int key0 = j * BN;
        if (key0 + BN > p.L) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (key0 + c >= p.L) s[c] = NEG_INF;
        }
      } else {
        // A warp's 32 rows lie in one query block (BLK >= 32): warp-uniform.
        const int qb = r / BLK;
#pragma unroll
        for (int e = 0; e < EPI; ++e) {
          const int key0 = (ent[e] & 0xFFFF) * BLK + (CPE > 1 ? (j % CPE) * BN : 0);
          on[e] = ((ent[e] >> 16) >> qb) & 1;
          if (key0 + BOX > p.L) {
#pragma unroll
            for (int c = 0; c < BOX; ++c)
              if (key0 + c >= p.L) s[e * BOX + c] = NEG_INF;
          }
        }
      }
      // Row max over the kept entries: per entry a tree over 8 independent
      // partial maxima (a serial chain would expose the FMNMX latency once
      // per column), then combined under the entry flags.
      float mx = NEG_INF;
#pragma unroll
      for (int e = 0; e < EPI; ++e) {
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = s[e * BOX + i];
#pragma unroll
        for (int c = 8; c < BOX; c += 2) pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], s[e * BOX + c], s[e * BOX + c + 1]);
        const float m0 = fmax3(pm[0], pm[1], pm[2]);
        const float m1 = fmax3(pm[3], pm[4], pm[5]);
        const float m2 = fmax3(pm[6], pm[7], m0);
        mx = on[e] ? fmax3(mx, m1, m2) : mx;
      }
      const float mx2 = mx * sl2;

      // Raise the max whenever this tile exceeds it; O_t is rescaled to
      // match after the exponentials below.
      float alpha = 1.f;
      if (mx2 > m_used) {
        if (m_used != NEG_INF) alpha = ex2_approx(m_used - mx2);
        m_used = mx2;
      }
      const bool rescale = __any_sync(0xffffffffu, alpha != 1.f) && j > 0;
      if (rescale) {
        l *= alpha;
        l_c *= alpha;
      }
      const float msub = (m_used == NEG_INF) ? 0.f : m_used;
      // Exponent offset per entry: -msub, or -inf for an entry this row's
      // query block does not keep (S is finite there, so MUFU ex2 gives
      // exactly 0; a column pair that took the FMA-pipe exp2 would give its
      // clamped floor of ~2e-38 instead, see exp2_fma2).
      float nsub[EPI];
#pragma unroll
      for (int e = 0; e < EPI; ++e) nsub[e] = on[e] ? -msub : NEG_INF;
      // exp2 of (s * sl2 + offset), two columns per packed FMA; the fp32
      // row sum in packed adds.
      const f32x2 sl2x2 = f2_make(sl2, sl2);
      f32x2 ts2[2] = {0ull, 0ull};
      // The weights go over S_t chunk by chunk (S is in registers by now):
      // bf16, 16 packed pairs per 32 columns, or, in the tf32 kernels, fp32,
      // one column per key.
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t pk[16];
        float pf[kTf32 ? 32 : 1];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float ns = nsub[(c * 32 + g * 8) / BOX];
          const f32x2 ns2 = f2_make(ns, ns);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = c * 32 + g * 8 + 2 * i;
            float a0, a1, e0, e1;
            f2_split(f2_fma(f2_make(s[col], s[col + 1]), sl2x2, ns2), a0, a1);
            if (((col >> 1) & 15) < poly_pairs_flash<D>()) {
              exp2_fma2(a0, a1, e0, e1);
            } else {
              e0 = ex2_approx(a0);
              e1 = ex2_approx(a1);
            }
            ts2[i & 1] = f2_add(ts2[i & 1], f2_make(e0, e1));
            if constexpr (kTf32) {
              pf[g * 8 + 2 * i] = e0;
              pf[g * 8 + 2 * i + 1] = e1;
            } else {
              pk[g * 4 + i] = pack_bf16x2(e0, e1);
            }
          }
        }
        if constexpr (kTf32)
          tmem_st32(s_col + c * 32, pf);
        else
          tmem_st16(s_col + c * 16, pk);
      }
      if (rescale) {
        // O_t *= alpha. S_t(j) completing implies PV_t(j-1) completed, so
        // O_t is at rest; S's registers are free by now, so all of O's
        // columns make one TMEM round trip instead of one per 32 columns.
        float o[D];
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tmem_ld32(o_col + c * 32, *reinterpret_cast<float(*)[32]>(&o[c * 32]));
        tmem_ld_wait();
        const f32x2 a2 = f2_make(alpha, alpha);
#pragma unroll
        for (int e = 0; e < D; e += 2) f2_split(f2_mul(f2_make(o[e], o[e + 1]), a2), o[e], o[e + 1]);
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          tmem_st32(o_col + c * 32, *reinterpret_cast<const float(*)[32]>(&o[c * 32]));
      }
      const float tsum = f2_sum(ts2[0]) + f2_sum(ts2[1]);
      {  // Kahan: l += tsum
        const float y = tsum - l_c;
        const float tt = l + y;
        l_c = (tt - l) - y;
        l = tt;
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }

    // ---- epilogue of pass 1: O = acc / l, lse
    const bool row_in = row < p.L_pad && n_iter > 0;
    const bool row_valid = row < p.L && n_iter > 0;
    const float lse2 = (l > 0.f) ? m_used + log2f(l) : __int_as_float(0x7f800000);
    if (ok && n_iter > 0) {
      if (!mbar_wait(&o_full[t], 0, wc)) ok = false;
      tc_fence_after();
    }
    if (ok && n_iter > 0) {
      const float inv_l = (row_valid && l > 0.f) ? 1.f / l : 0.f;
      const size_t obase = (size_t(bh[t]) * p.L_pad + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(o_col + c * 32, o);
        tmem_ld_wait();
        if (row_in) {
          if constexpr (kOutBf16) {
            uint32_t* dst =
                reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.o) + obase + c * 32);
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 w;
              w.x = pack_bf16x2(o[e] * inv_l, o[e + 1] * inv_l);
              w.y = pack_bf16x2(o[e + 2] * inv_l, o[e + 3] * inv_l);
              w.z = pack_bf16x2(o[e + 4] * inv_l, o[e + 5] * inv_l);
              w.w = pack_bf16x2(o[e + 6] * inv_l, o[e + 7] * inv_l);
              *reinterpret_cast<uint4*>(dst + e / 2) = w;
            }
          } else {
            float* dst = static_cast<float*>(p.o) + obase + c * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) =
                  make_float4(o[e] * inv_l, o[e + 1] * inv_l, o[e + 2] * inv_l, o[e + 3] * inv_l);
          }
        }
      }
      if (row_in && p.lse != nullptr)
        p.lse[size_t(bh[t]) * p.L_pad + row] =
            (row_valid && l > 0.f) ? lse2 * 0.69314718055994531f : NEG_INF;
      if constexpr (kDblMass) {
        // O_t is stored: its columns may take pass 2's second S buffer.
        tc_fence_before();
        mbar_arrive(&o_read[t]);
      }
    }

    if constexpr (kDense) {
      // ---- pass 2: block masses from exp(s - lse)
      constexpr int NKB = BN >= BLK ? BN / BLK : 1;  // key blocks per key tile
      constexpr int NG = BN / 32;        // 32-column groups per key tile
      constexpr int WPB = BLK / 32;      // warps per query block (1, 2 or 4)
      const int q_local = r / BLK;       // query block within the tile
      const int I = qt[t] * (BM / BLK) + q_local;
      const int n_valid_I = min(BLK, p.L - I * BLK);
      const float inv_cnt = (n_valid_I > 0) ? 1.f / float(n_valid_I) : 0.f;
      const float lsub = row_valid ? lse2 : __int_as_float(0x7f800000);
      float* red_t = red + t * 32;
      float carry = 0.f;  // a key block over CPE key tiles: the earlier tiles' sum
      // kDblMass: S_t(j) sits in buffer j & 1, S_t's own columns or the
      // second buffer.
      const uint32_t alt_col = tmem + lane_base + (t ? Lay::TMEM_ALT1 : Lay::TMEM_ALT0);
      for (int j = 0; ok && j < n_iter; ++j) {
        float s[BN];
        if constexpr (kDblMass) {
          const int bsel = j & 1;
          if (!mbar_wait(&s2_full[2 * t + bsel], (j >> 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t src = bsel ? alt_col : s_col;
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            tmem_ld32(src + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&s2_free[2 * t + bsel]);
        } else {
          if (!mbar_wait(&s_full[t], sc & 1, wc)) { ok = false; break; }
          ++sc;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            tmem_ld32(s_col + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&s_free[t]);
        }

        const int key0 = j * BN;
        // Padded query rows subtract +inf (their scores are finite: rows past
        // L hold finite values by contract, rows past L_pad read as zero), so
        // they add zeros: exact ones from MUFU ex2, and the FMA-pipe exp2's
        // clamped floor (~2e-38 per entry, under 1e-33 per mass entry, far
        // below fp32 resolution of any mass) in the columns that take it.
        // Padded keys only occur in the last key tile, which takes its own
        // warp-uniform branch.
        float part[NG];
        if (key0 + BN <= p.L) {
          const f32x2 sl2x2 = f2_make(sl2, sl2);
          const f32x2 nl2 = f2_make(-lsub, -lsub);
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            // 32 columns: packed FMAs for the exponents, two packed partial
            // sums (four independent fp32 lanes).
            f32x2 acc[2] = {0ull, 0ull};
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float a0, a1, e0, e1;
              f2_split(f2_fma(f2_make(s[g * 32 + c], s[g * 32 + c + 1]), sl2x2, nl2), a0, a1);
              if ((c >> 1) < poly_pairs_mass<D>()) {
                exp2_fma2(a0, a1, e0, e1);
              } else {
                e0 = ex2_approx(a0);
                e1 = ex2_approx(a1);
              }
              acc[(c >> 1) & 1] = f2_add(acc[(c >> 1) & 1], f2_make(e0, e1));
            }
            part[g] = f2_sum(acc[0]) + f2_sum(acc[1]);
          }
        } else {
          const int lim = p.L - key0;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 32; ++c)
              a[c & 3] += (g * 32 + c < lim) ? ex2_approx(fmaf(s[g * 32 + c], sl2, -lsub)) : 0.f;
            part[g] = (a[0] + a[1]) + (a[2] + a[3]);
          }
        }
        // Merge 32-column groups into key blocks of BLK columns.
        float kbsum[NKB];
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) kbsum[kb] = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) kbsum[(g * 32) / BLK] += part[g];
        // Sum over the rows of this warp.
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
            kbsum[kb] += __shfl_xor_sync(0xffffffffu, kbsum[kb], off);
        }
        if constexpr (CPE > 1) {
          // This tile is chunk j % CPE of one key block: carry the sum until
          // the block's last chunk.
          kbsum[0] += carry;
          if (j % CPE != CPE - 1) {
            carry = kbsum[0];
            continue;
          }
          carry = 0.f;
        }
        const int w_idx = j / CPE;         // key blocks written so far (CPE > 1), else j
        const int J0 = key0 / BLK;
        float* mrow = p.mass + (size_t(bh[t]) * p.n_blocks + I) * p.n_blocks;
        if constexpr (WPB == 1) {
          if (lane == 0 && I < p.n_blocks) {
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb)
              if (J0 + kb < p.n_blocks) mrow[J0 + kb] = kbsum[kb] * inv_cnt;
          }
        } else {
          float* rb = red_t + (w_idx & 1) * 16;
          if (lane == 0) {
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) rb[wl * 4 + kb] = kbsum[kb];
          }
          mbar_arrive(&red_bar[2 * t + (w_idx & 1)]);
          if (!mbar_wait(&red_bar[2 * t + (w_idx & 1)], (w_idx >> 1) & 1, wc)) { ok = false; break; }
          if (lane == 0 && (wl % WPB) == 0 && I < p.n_blocks) {
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
              float tot = 0.f;
#pragma unroll
              for (int w = 0; w < WPB; ++w) tot += rb[(wl + w) * 4 + kb];
              if (J0 + kb < p.n_blocks) mrow[J0 + kb] = tot * inv_cnt;
            }
          }
        }
      }

      if constexpr (kCut) {
        // Fused selection: this CTA holds every key block of its query
        // blocks' mass rows, so each warpgroup cuts its own tile's rows here.
        // Once both tiles' mass passes are over, every MMA has read its
        // operands (each S was waited for), so the Q/K/V staging memory is
        // free for the cut's workspace, and the barrier makes the mass rows
        // these warps wrote visible to them. A warp that gave up a wait, or
        // an abort anywhere in the CTA, skips the cut in both warpgroups.
        // Named barriers: 1 joins the two softmax warpgroups (256 threads),
        // 2 + t the warpgroup of tile t inside the cut; barrier 0 stays the
        // CTA-wide one at the end of the kernel.
        __syncwarp();
        __threadfence_block();
        const bool quit = named_bar_or(1, 256, !ok || *abort_flag != 0);
        if (!quit)
          fused_cut_rows(p.mass, p.n_blocks, p.tau_fx, p.cut_key, p.cut_count, p.retained_fx,
                         p.total_fx, p.status,
                         reinterpret_cast<cut::BucketSmem*>(smem + t * kCutSmemStride), t, r,
                         bh[t], qt[t] * (BM / BLK), BM / BLK);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace losa

// losa_attention.cuh - the attention kernels of the LoSA hot path (sm_100a).
//
// One CTA owns a 128-row query tile of one (batch, head) and walks a list of
// key tiles. Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r of the tile (TMEM lane r);
//   warp 4     TMA producer: Q once, then K (and V) tiles into smem rings;
//   warp 5     MMA issuer (one thread) and TMEM owner.
// Per key tile: S = Q K^T (tcgen05, bf16 -> fp32 in TMEM, double-buffered),
// the softmax warps read S from TMEM, write P (bf16) into a 128B-swizzled
// smem tile, and the MMA thread accumulates O += P V into TMEM.
//
// kDense = true is the construction step: pass 1 is the flash forward over
// all key tiles (O, row lse); pass 2 recomputes S = Q K^T tile by tile and
// sums exp(s - lse) over each (query block, key block) into the mass map
// (LoSA abstract, arXiv 2608.12032: exact block attention masses at one
// early dense step; ubos.tech LoSA post, Phase 1 - Dense Calibration).
// kDense = false is the sparse step: pass 1 only, over the tile's union of
// retained key blocks, each row masked to its own query block's set
// (ubos.tech LoSA post, Phase 3 - Repeated Sparse Inference).
#pragma once

#include "losa_device.cuh"

namespace losa {

struct AttnParams {
  int L;          // valid tokens
  int L_pad;      // padded tokens (multiple of block)
  int n_qt;       // query tiles per head = ceil(L_pad / 128)
  int n_kv;       // key tiles per pass (dense)
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
};

template <int D, int BN, int NS>
struct AttnLayout {
  static constexpr int BM = 128;
  static constexpr int kSlab = 64;                       // bf16 elements per 128 B row
  static constexpr int Q_BYTES = BM * D * 2;             // D/64 slabs of 16 KB
  static constexpr int KV_BYTES = BN * D * 2;            // D/64 slabs of BN*128 B
  static constexpr int P_SLABS = (BN + 63) / 64;
  static constexpr int P_BYTES = P_SLABS * BM * 128;     // 128 rows x 128 B per slab
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int N_BARS = 1 + 4 * NS + 9;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem addr, abort flag
  static constexpr int OFF_RED = OFF_MISC + 16;          // float red[2][4][4]
  static constexpr int BYTES = OFF_RED + 2 * 4 * 4 * 4;
  static constexpr int SMEM_ALLOC = BYTES + 1024;        // slack for 1 KB alignment
  static constexpr int TMEM_NEED = 2 * BN + D;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int TMEM_O = 2 * BN;
  static_assert(D % 64 == 0, "head dim must be a multiple of 64");
  static_assert(BN % 32 == 0 && BN <= 128, "key tile must be 32, 64 or 128");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0, "1 KB alignment");
  static_assert(KV_BYTES % 1024 == 0, "1 KB alignment of stages");
  // More than half of TMEM per CTA is only safe with one CTA per SM.
  static_assert(TMEM_COLS <= 256 || SMEM_ALLOC > 116 * 1024, "TMEM oversubscription");
};

template <int D, int BN, int NS, bool kDense, bool kOutBf16>
__global__ void __launch_bounds__(192, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using Lay = AttnLayout<D, BN, NS>;
  constexpr int BM = Lay::BM;
  constexpr int N_SLABS = D / 64;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint8_t* sP = smem + Lay::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + NS;
  uint64_t* v_full = k_empty + NS;
  uint64_t* v_empty = v_full + NS;
  uint64_t* s_full = v_empty + NS;  // [2]
  uint64_t* s_free = s_full + 2;    // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* red_bar = pv_done + 1;  // [2], cross-warp mass reduction
  uint64_t* drain_bar = red_bar + 2;  // MMA drain after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + Lay::OFF_RED);  // [2][4][4]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item
  int bh, qt, e_begin = 0, n_iter;
  if constexpr (kDense) {
    qt = blockIdx.x;
    bh = blockIdx.y;
    n_iter = p.n_kv;
  } else {
    const int t = p.tile_order[blockIdx.x];
    bh = t / p.n_qt;
    qt = t - bh * p.n_qt;
    e_begin = p.tile_ptr[t];
    n_iter = p.tile_ptr[t + 1] - e_begin;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(&red_bar[0], 128);
    mbar_init(&red_bar[1], 128);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, Lay::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, p.status};

  if (warp == 4) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      mbar_arrive_expect_tx(q_full, Lay::Q_BYTES);
#pragma unroll
      for (int s = 0; s < N_SLABS; ++s)
        tma_load_3d(sQ + s * (BM * 128), &tm_q, q_full, s * 64, qt * BM, bh);
      int kc = 0, vc = 0;
      bool ok = true;
      constexpr int n_pass = kDense ? 2 : 1;
      for (int pass = 0; pass < n_pass && ok; ++pass) {
        for (int it = 0; it < n_iter; ++it) {
          int key_row;
          if constexpr (kDense) {
            key_row = it * BN;
          } else {
            key_row = (p.tile_entry[e_begin + it] & 0xFFFF) * BN;
          }
          const int ks = kc % NS;
          if (!mbar_wait(&k_empty[ks], ((kc / NS) & 1) ^ 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[ks], Lay::KV_BYTES);
#pragma unroll
          for (int s = 0; s < N_SLABS; ++s)
            tma_load_3d(sK + ks * Lay::KV_BYTES + s * (BN * 128), &tm_k, &k_full[ks], s * 64,
                        key_row, bh);
          ++kc;
          if (pass == 0) {
            const int vs = vc % NS;
            if (!mbar_wait(&v_empty[vs], ((vc / NS) & 1) ^ 1, wc)) { ok = false; break; }
            mbar_arrive_expect_tx(&v_full[vs], Lay::KV_BYTES);
#pragma unroll
            for (int s = 0; s < N_SLABS; ++s)
              tma_load_3d(sV + vs * Lay::KV_BYTES + s * (BN * 128), &tm_v, &v_full[vs], s * 64,
                          key_row, bh);
            ++vc;
          }
        }
      }
      if (!ok) {
        // Aborted: wait (bounded) for the copies still in flight before the
        // CTA releases its shared memory.
        mbar_wait_drain(q_full, 0);
        for (int i = (kc > NS ? kc - NS : 0); i < kc; ++i) mbar_wait_drain(&k_full[i % NS], (i / NS) & 1);
        for (int i = (vc > NS ? vc - NS : 0); i < vc; ++i) mbar_wait_drain(&v_full[i % NS], (i / NS) & 1);
      }
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_addr(sQ);
      const uint32_t k_base = smem_addr(sK);
      const uint32_t v_base = smem_addr(sV);
      const uint32_t p_base = smem_addr(sP);
      int kc = 0, vc = 0, sc = 0;
      bool ok = mbar_wait(q_full, 0, wc);
      // O += P_t V_t once the softmax warps have written P_t.
      auto issue_pv = [&](int t) -> bool {
        if (!mbar_wait(p_full, t & 1, wc)) return false;
        const int vs = vc % NS;
        if (!mbar_wait(&v_full[vs], (vc / NS) & 1, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a = sdesc_sw128(p_base + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(v_base + vs * Lay::KV_BYTES + kk * 2048, BN * 128, 1024);
          umma_bf16_ss(tmem + Lay::TMEM_O, a, b, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pv_done);
        umma_commit(&v_empty[vs]);
        ++vc;
        return true;
      };
      constexpr int n_pass = kDense ? 2 : 1;
      for (int pass = 0; pass < n_pass && ok; ++pass) {
        for (int it = 0; it < n_iter; ++it) {
          const int ks = kc % NS;
          if (!mbar_wait(&k_full[ks], (kc / NS) & 1, wc)) { ok = false; break; }
          const int sb = sc & 1;
          if (!mbar_wait(&s_free[sb], ((sc >> 1) & 1) ^ 1, wc)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
            const uint64_t a = sdesc_sw128(q_base + off, 16, 1024);
            const uint64_t b = sdesc_sw128(k_base + ks * Lay::KV_BYTES + koff, 16, 1024);
            umma_bf16_ss(tmem + sb * BN, a, b, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          umma_commit(&k_empty[ks]);
          ++kc;
          ++sc;
          if (pass == 0 && it > 0) {
            if (!issue_pv(it - 1)) { ok = false; break; }
          }
        }
        if (ok && pass == 0 && n_iter > 0) ok = issue_pv(n_iter - 1);
      }
      if (!ok) {
        // Drain: let every MMA issued so far finish before TMEM is freed.
        umma_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0);
      }
    }
  } else {
    // ================================================================ softmax warps
    const int r = threadIdx.x;             // row within the tile, TMEM lane
    const int row = qt * BM + r;           // token row within the head
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m_used = NEG_INF;  // running max in log2 units (lazily raised)
    // Running sum of exp2(s*sl2 - m_used) in fp32, which gives lse. A row
    // sums ~10^5 terms, so each tile's terms are summed first and the tile
    // sums are accumulated with Kahan compensation (a plain running sum
    // loses the small terms against the large total).
    float l = 0.f, l_c = 0.f;
    float lb = 0.f;          // the same sum over the bf16-rounded weights P.V uses:
                             // O = acc / lb is an exact convex combination of V rows
    int sc = 0;
    bool ok = true;
    uint8_t* prow = sP + r * 128;
    const int sw = r & 7;

    for (int it = 0; it < n_iter; ++it) {
      const int sb = sc & 1;
      if (!mbar_wait(&s_full[sb], (sc >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(tmem + lane_base + sb * BN + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);
      ++sc;

      int key0;
      bool row_on = true;
      if constexpr (kDense) {
        key0 = it * BN;
      } else {
        const int e = p.tile_entry[e_begin + it];
        key0 = (e & 0xFFFF) * BN;
        row_on = ((e >> 16) >> (r / p.block)) & 1;
      }
      if (!row_on) {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = NEG_INF;
      } else if (key0 + BN > p.L) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (key0 + c >= p.L) s[c] = NEG_INF;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
      const float mx2 = mx * sl2;

      if (it > 0) {
        if (!mbar_wait(pv_done, (it - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
      }
      // Lazy rescale: raise the reference max only when it grows by > 8
      // (a factor 256), so exp2 values stay <= 256 and O is rarely touched.
      float alpha = 1.f;
      if (mx2 > m_used + 8.f) {
        if (m_used != NEG_INF) alpha = ex2_approx(m_used - mx2);
        m_used = mx2;
      }
      if (__any_sync(0xffffffffu, alpha != 1.f) && it > 0) {
        l *= alpha;
        l_c *= alpha;
        lb *= alpha;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + Lay::TMEM_O + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tmem + lane_base + Lay::TMEM_O + c * 32, o);
        }
        tmem_st_wait();
      }
      const float msub = (m_used == NEG_INF) ? 0.f : m_used;
      float tsum = 0.f, tsum_b = 0.f;
#pragma unroll
      for (int g = 0; g < BN / 8; ++g) {
        float e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = ex2_approx(fmaf(s[g * 8 + j], sl2, -msub));
        tsum += ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
        uint4 pk;
        pk.x = pack_bf16x2(e[0], e[1]);
        pk.y = pack_bf16x2(e[2], e[3]);
        pk.z = pack_bf16x2(e[4], e[5]);
        pk.w = pack_bf16x2(e[6], e[7]);
        tsum_b += (bf16x2_sum(pk.x) + bf16x2_sum(pk.y)) + (bf16x2_sum(pk.z) + bf16x2_sum(pk.w));
        const int slab = g >> 3, ch = g & 7;
        *reinterpret_cast<uint4*>(prow + slab * (BM * 128) + ((ch ^ sw) << 4)) = pk;
      }
      {  // Kahan: l += tsum
        const float y = tsum - l_c;
        const float t = l + y;
        l_c = (t - l) - y;
        l = t;
      }
      lb += tsum_b;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }

    // ---- epilogue of pass 1: O = acc / l, lse
    const bool row_in = row < p.L_pad;
    const bool row_valid = row < p.L;
    const float lse2 = (l > 0.f) ? m_used + log2f(l) : __int_as_float(0x7f800000);
    if (ok && n_iter > 0) {
      if (!mbar_wait(pv_done, (n_iter - 1) & 1, wc)) ok = false;
      tc_fence_after();
    }
    if (ok) {
      const float inv_l = (row_valid && lb > 0.f) ? 1.f / lb : 0.f;
      const size_t obase = (size_t(bh) * p.L_pad + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (n_iter > 0) {
          tmem_ld32(tmem + lane_base + Lay::TMEM_O + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
        if (row_in) {
          if constexpr (kOutBf16) {
            uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.o) + obase + c * 32);
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
        p.lse[size_t(bh) * p.L_pad + row] =
            (row_valid && l > 0.f) ? lse2 * 0.69314718055994531f : NEG_INF;
    }

    if constexpr (kDense) {
      // ---- pass 2: block masses from exp(s - lse)
      constexpr int NKB_MAX = BN / 32;  // key blocks per tile for the smallest block
      const int blk = p.block;
      const int nkb = BN / blk;          // key blocks per key tile (blk <= BN)
      const int q_local = r / blk;       // query block within the tile
      const int I = qt * (BM / blk) + q_local;
      const int n_valid_I = min(blk, p.L - I * blk);
      const float inv_cnt = (n_valid_I > 0) ? 1.f / float(n_valid_I) : 0.f;
      const float lsub = row_valid ? lse2 : __int_as_float(0x7f800000);
      const int wpb = blk / 32;          // warps per query block (1, 2 or 4)
      for (int it = 0; ok && it < n_iter; ++it) {
        const int sb = sc & 1;
        if (!mbar_wait(&s_full[sb], (sc >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
          tmem_ld32(tmem + lane_base + sb * BN + c * 32, *reinterpret_cast<float(*)[32]>(&s[c * 32]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[sb]);
        ++sc;

        const int key0 = it * BN;
        float part[NKB_MAX];
#pragma unroll
        for (int kb = 0; kb < NKB_MAX; ++kb) part[kb] = 0.f;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          // Padded query rows and padded keys contribute nothing (and may
          // hold any finite or non-finite score).
          const float e =
              (row_valid && key0 + c < p.L) ? ex2_approx(fmaf(s[c], sl2, -lsub)) : 0.f;
          part[c / 32] += e;   // 32-column groups; merged into key blocks below
        }
        // Merge 32-column groups into key blocks of size blk.
        float kbsum[NKB_MAX];
#pragma unroll
        for (int kb = 0; kb < NKB_MAX; ++kb) kbsum[kb] = 0.f;
#pragma unroll
        for (int g = 0; g < NKB_MAX; ++g) kbsum[(g * 32) / blk] += part[g];
        // Sum over the rows of this warp.
#pragma unroll
        for (int kb = 0; kb < NKB_MAX; ++kb) {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1)
            kbsum[kb] += __shfl_xor_sync(0xffffffffu, kbsum[kb], off);
        }
        const int J0 = key0 / blk;
        if (wpb == 1) {
          if (lane == 0 && I < p.n_blocks) {
            for (int kb = 0; kb < nkb; ++kb)
              if (J0 + kb < p.n_blocks)
                p.mass[(size_t(bh) * p.n_blocks + I) * p.n_blocks + J0 + kb] = kbsum[kb] * inv_cnt;
          }
        } else {
          float* rb = red + (it & 1) * 16;
          if (lane == 0) {
#pragma unroll
            for (int kb = 0; kb < NKB_MAX; ++kb) rb[warp * 4 + kb] = kbsum[kb];
          }
          mbar_arrive(&red_bar[it & 1]);
          if (!mbar_wait(&red_bar[it & 1], (it >> 1) & 1, wc)) { ok = false; break; }
          if (lane == 0 && (warp % wpb) == 0 && I < p.n_blocks) {
            for (int kb = 0; kb < nkb; ++kb) {
              float t = 0.f;
              for (int w = warp; w < warp + wpb; ++w) t += rb[w * 4 + kb];
              if (J0 + kb < p.n_blocks)
                p.mass[(size_t(bh) * p.n_blocks + I) * p.n_blocks + J0 + kb] = t * inv_cnt;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace losa

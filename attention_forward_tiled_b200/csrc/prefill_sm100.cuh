// prefill_sm100.cuh -- tiled attention forward for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V block by block with the
// online softmax update, so the Nq x Nk score matrix never leaves the SM
// (FlashAttention/ops-transformer article, sections "FlashAttention的核心逻辑"
// and "传统注意力的显存陷阱").  The article's Ascend tiling (Cube unit for the
// matmuls, Vector unit for the softmax, 128x64 blocks staged in the Unified
// Buffer) is prior art; this kernel maps the same algorithm onto B200:
//
//   * one CTA owns a work unit = (batch b, head h, a pair of 128-row Q tiles);
//   * warp 8 (producer) streams Q once and then K_0, V_0, K_1, V_1, ... into a
//     ring of shared-memory stages with TMA (128-byte swizzle), each stage
//     guarded by a full/empty mbarrier pair;
//   * warp 9 (MMA issuer, one thread) issues tcgen05.mma:
//       S_t = Q_t K_j^T   (A, B from shared memory, fp32 accumulator in TMEM)
//       O_t += P_t V_j    (A = P from TMEM, B = V from shared memory)
//     alternating the two Q tiles so one tile's softmax overlaps the other
//     tile's matrix multiplies;
//   * warps 10-11 (bf16 inputs only) convert each V tile to fp16 in place, so
//     P V runs with P in fp16 (11-bit significand) rather than bf16 (8-bit);
//   * warps 0-3 and 4-7 (softmax warpgroups, one per Q tile, one thread per
//     query row) read a 128-column S row from TMEM, apply the tail/causal mask,
//     update the running max m and sum l (base-2 exponent with scale*log2(e)
//     folded into one FMA, lazy rescale of O only when the max grows by more
//     than 2^8), write P back to TMEM as fp16 over the consumed S columns,
//     and finally normalise O by 1/l, store it with TMA and write the row LSE.
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D).  P_t occupies columns [64,128) of S_t.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

struct PrefillParams {
  CUtensorMap tm_q;  // [B, Nq, H, D] as 4-D (D, H, Nq, B), box (64, 1, 128, 1), 128B swizzle
  CUtensorMap tm_k;  // [B, Nk, H, D], same box
  CUtensorMap tm_v;  // [B, Nk, H, D], same box
  CUtensorMap tm_o;  // [B, Nq, H, D], same box (store)
  void* out;         // raw output pointer (rows that see no key are written directly)
  float* lse;        // [B, H, Nq] or nullptr
  int* status;       // device status word
  int B, H, Nq, Nk;
  int causal;
  int n_qpairs;      // ceil(Nq / 256)
  int group_heads;   // heads per scheduling group (L2 locality of K/V)
  float scale_log2;  // scale * log2(e)
  int inject;        // test hook: 1 = skip the first Q-tile load
  unsigned long long timeout_ns;
};

template <int D>
struct PrefillCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kRows = 128;                    // rows per Q tile and per K/V tile
  static constexpr int kBoxBytes = 128 * 128;          // 128 rows x 64 elements x 2 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kStages = (D == 128) ? 4 : 8;  // K/V ring depth
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // +1024: manual 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 384;  // 2 softmax warpgroups, producer, MMA, 2 converter warps
  static constexpr int kProducerWarp = 8;
  static constexpr int kMmaWarp = 9;
  static constexpr int kConvWarp0 = 10;  // warps 10-11: bf16 -> fp16 conversion of V tiles
  // barrier indices
  static constexpr int kBarQFull = 0;    // [2]
  static constexpr int kBarSFull = 2;    // [2]
  static constexpr int kBarPReady = 4;   // [2]
  static constexpr int kBarOFull = 6;    // [2]
  static constexpr int kBarMmaDone = 8;  // [1]
  static constexpr int kBarKVFull = 9;   // [kStages]
  static constexpr int kBarKVEmpty = 9 + kStages;
  static constexpr int kBarVConv = 9 + 2 * kStages;  // [kStages] V tile converted (bf16 only)
  static constexpr int kNumBars = 9 + 3 * kStages;
  static_assert(kNumBars * 8 + 16 <= kBarBytes, "barrier area too small");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Number of 128-key tiles query tile [row0, row0+128) must visit (0 = none).
__device__ __forceinline__ int prefill_kv_tiles(int row0, int Nq, int Nk, int causal) {
  if (row0 >= Nq) return 0;
  long long last_key = (long long)Nk - 1;
  if (causal) {
    const long long row_last = (long long)min(row0 + 127, Nq - 1);
    const long long lim = row_last + ((long long)Nk - Nq);  // last allowed key of the last row
    if (lim < 0) return 0;
    if (lim < last_key) last_key = lim;
  }
  return (int)(last_key / 128) + 1;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(PrefillCfg<D>::kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto BAR = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: (b, h, q-pair), heads grouped for K/V reuse in L2, heavy causal pairs first
  const int BH = p.B * p.H;
  const int nqp = p.n_qpairs;
  const int G = p.group_heads;
  const long long unit = blockIdx.x;
  const long long full_units = (long long)(BH / G) * G * nqp;
  int g, idx, Gc;
  if (unit < full_units) {
    g = (int)(unit / ((long long)G * nqp));
    idx = (int)(unit - (long long)g * G * nqp);
    Gc = G;
  } else {
    g = BH / G;
    idx = (int)(unit - full_units);
    Gc = BH - g * G;
  }
  const int qrank = idx / Gc;
  const int bh = g * G + (idx - qrank * Gc);
  const int qp = p.causal ? (nqp - 1 - qrank) : qrank;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int row0_0 = qp * 256, row0_1 = qp * 256 + 128;
  const int nkv0 = prefill_kv_tiles(row0_0, p.Nq, p.Nk, p.causal);
  const int nkv1 = prefill_kv_tiles(row0_1, p.Nq, p.Nk, p.causal);
  const int nmax = max(nkv0, nkv1);

  const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};

  // ---- one-time setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarQFull + i), 1);
      mbar_init(BAR(C::kBarSFull + i), 1);
      mbar_init(BAR(C::kBarPReady + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarOFull + i), 1);
    }
    mbar_init(BAR(C::kBarMmaDone), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(BAR(C::kBarKVFull + s), 1);
      mbar_init(BAR(C::kBarKVEmpty + s), 1);
      mbar_init(BAR(C::kBarVConv + s), 2);  // one arrive per converter warp
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kProducerWarp) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&p.tm_q);
      tma_prefetch_map(&p.tm_k);
      tma_prefetch_map(&p.tm_v);
      tma_prefetch_map(&p.tm_o);
      const int nkv[2] = {nkv0, nkv1};
      const int row0[2] = {row0_0, row0_1};
      bool q_issued[2] = {false, false};
      for (int t = 0; t < 2; ++t) {
        if (nkv[t] == 0) continue;
        if (p.inject == 1 && t == 0) continue;  // test hook: the MMA issuer's wait must expire
        mbar_arrive_expect_tx(BAR(C::kBarQFull + t), C::kTileBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_4d(sbase + C::kOffQ + t * C::kTileBytes + bx * C::kBoxBytes, &p.tm_q,
                      BAR(C::kBarQFull + t), bx * 64, h, row0[t], b);
        q_issued[t] = true;
      }
      int issued = 0;
      for (int i = 0; i < 2 * nmax; ++i) {
        const int stage = i % C::kStages;
        const int round = i / C::kStages;
        if (round > 0) mbar_wait(BAR(C::kBarKVEmpty + stage), (round - 1) & 1, wctx);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(BAR(C::kBarKVFull + stage), C::kTileBytes);
        const CUtensorMap* map = (i & 1) ? &p.tm_v : &p.tm_k;
        const int key0 = (i >> 1) * 128;
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_4d(sbase + C::kOffKV + stage * C::kTileBytes + bx * C::kBoxBytes, map,
                      BAR(C::kBarKVFull + stage), bx * 64, h, key0, b);
        issued = i + 1;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA can exit.
        for (int t = 0; t < 2; ++t)
          if (q_issued[t]) mbar_wait_drain(BAR(C::kBarQFull + t), 0, p.timeout_ns);
        const int first = issued > C::kStages ? issued - C::kStages : 0;
        for (int i = first; i < issued; ++i)
          mbar_wait_drain(BAR(C::kBarKVFull + i % C::kStages), (i / C::kStages) & 1, p.timeout_ns);
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer =======================
    if (lane == 0 && nmax > 0) {
      constexpr uint32_t idesc_s = make_idesc_f16(128, 128, BF16, false);  // Q K^T, both K-major
      // P V always runs in fp16 (bf16 V tiles are converted in shared memory first); V is MN-major
      constexpr uint32_t idesc_o = make_idesc_f16(128, D, false, true);
      const int nkv[2] = {nkv0, nkv1};
      const uint32_t colS[2] = {0u, 128u};
      const uint32_t colO[2] = {256u, 256u + D};
      const uint32_t sQ[2] = {sbase + C::kOffQ, sbase + C::kOffQ + C::kTileBytes};
      bool ok = true;
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0) ok = mbar_wait(BAR(C::kBarQFull + t), 0, wctx) && ok;

      // S_t = Q_t K_j^T over D/16 k-steps of 16 elements (32 bytes inside a 128-byte swizzle row).
      auto issue_s = [&](int t, uint32_t sK) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          mma_f16_ss(tmem + colS[t], make_sdesc_sw128(sQ[t] + off, 16, 1024),
                     make_sdesc_sw128(sK + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V_j over 8 k-steps of 16 keys; P_t is in TMEM columns [64,128) of S_t.
      auto issue_pv = [&](int t, uint32_t sV, bool accumulate_first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_f16_ts(tmem + colO[t], tmem + colS[t] + 64 + kk * 8,
                     make_sdesc_sw128(sV + kk * 2048, C::kBoxBytes, 1024), idesc_o,
                     (accumulate_first || kk > 0) ? 1u : 0u);
        }
      };

      // prologue: S_t(0) for both tiles from K_0 (ring item 0)
      ok = mbar_wait(BAR(C::kBarKVFull + 0), 0, wctx) && ok;
      if (ok && !*abort_flag) {
        for (int t = 0; t < 2; ++t)
          if (nkv[t] > 0) {
            issue_s(t, sbase + C::kOffKV);
            tc_commit(BAR(C::kBarSFull + t));
          }
        tc_commit(BAR(C::kBarKVEmpty + 0));
      }
      for (int j = 0; j < nmax; ++j) {
        const int iv = 2 * j + 1;  // ring item of V_j
        const int sv = iv % C::kStages;
        mbar_wait(BAR((BF16 ? C::kBarVConv : C::kBarKVFull) + sv), (iv / C::kStages) & 1, wctx);
        const int ik = 2 * j + 2;  // ring item of K_{j+1}
        const int sk = ik % C::kStages;
        bool k_ready = false;
        for (int t = 0; t < 2; ++t) {
          if (j >= nkv[t]) continue;
          mbar_wait(BAR(C::kBarPReady + t), j & 1, wctx);
          tc_fence_after_sync();
          if (*abort_flag) continue;
          issue_pv(t, sbase + C::kOffKV + sv * C::kTileBytes, j > 0);
          if (j + 1 < nkv[t]) {
            if (!k_ready) {
              mbar_wait(BAR(C::kBarKVFull + sk), (ik / C::kStages) & 1, wctx);
              k_ready = true;
            }
            if (*abort_flag) continue;
            issue_s(t, sbase + C::kOffKV + sk * C::kTileBytes);
            tc_commit(BAR(C::kBarSFull + t));
          } else {
            tc_commit(BAR(C::kBarOFull + t));
          }
        }
        if (!*abort_flag) {
          tc_commit(BAR(C::kBarKVEmpty + sv));
          if (k_ready) tc_commit(BAR(C::kBarKVEmpty + sk));
        }
      }
      // every MMA (and every commit arrive) has landed before TMEM is released
      tc_commit(BAR(C::kBarMmaDone));
      mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    }
  } else if (warp >= C::kConvWarp0) {
    // ======================= bf16 -> fp16 conversion of V tiles (bf16 inputs) ===============
    if constexpr (BF16) {
      const int ct = threadIdx.x - C::kConvWarp0 * 32;  // 0..63
      for (int j = 0; j < nmax; ++j) {
        const int iv = 2 * j + 1;
        const int sv = iv % C::kStages;
        mbar_wait(BAR(C::kBarKVFull + sv), (iv / C::kStages) & 1, wctx);
        __syncwarp();
        uint4* tile = reinterpret_cast<uint4*>(smem + C::kOffKV + sv * C::kTileBytes);
#pragma unroll 4
        for (int c = ct; c < C::kTileBytes / 16; c += 64) {
          uint4 w = tile[c];
          w.x = bf16x2_to_f16x2_sat(w.x);
          w.y = bf16x2_to_f16x2_sat(w.y);
          w.z = bf16x2_to_f16x2_sat(w.z);
          w.w = bf16x2_to_f16x2_sat(w.w);
          tile[c] = w;
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        __syncwarp();
        if ((ct & 31) == 0) mbar_arrive(BAR(C::kBarVConv + sv));
      }
    }
  } else {
    // ======================= softmax warpgroups (warps 0-3: tile 0, 4-7: tile 1) ===========
    const int t = warp >> 2;
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;      // row inside the Q tile
    const int row0 = t ? row0_1 : row0_0;
    const int nkv = t ? nkv1 : nkv0;
    const int grow = row0 + r;              // global query row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? 128u : 0u);
    const uint32_t tO = tmem + lane_base + (t ? 256u + D : 256u);
    const float cs = p.scale_log2;
    const bool neg = cs < 0.f;
    const float cs_abs = fabsf(cs);
    const long long diag = (long long)p.Nk - p.Nq;

    float m_run = -INFINITY;  // running max of scale*log2(e)*s (lazy: may lag the true max by <= 8)
    float l_run = 0.f;        // running sum of 2^(cs*s - m_run)

    if (nkv > 0) {
      for (int j = 0; j < nkv; ++j) {
        mbar_wait(BAR(C::kBarSFull + t), j & 1, wctx);
        __syncwarp();  // lanes may leave the bounded wait on different polls
        tc_fence_after_sync();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_order_after_wait(sr[c]);

        // mask needed on the key tail and on tiles crossing the causal diagonal
        const long long key0 = (long long)j * 128;
        const bool need_mask = (key0 + 128 > p.Nk) ||
                               (p.causal && key0 + 127 > (long long)row0 + diag);
        int lim = 128;  // keys [key0, key0+lim) are allowed for this row
        if (need_mask) {
          long long l = (long long)p.Nk;
          if (p.causal) l = min(l, (long long)grow + diag + 1);
          l -= key0;
          lim = (int)max(0LL, min(128LL, l));
        }

        // tile max of the sign-adjusted raw scores (scale folded in afterwards)
        float mx = -INFINITY;
        if (!need_mask) {
          if (!neg) {
#pragma unroll
            for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c >> 5][c & 31]));
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c) mx = fmaxf(mx, -__uint_as_float(sr[c >> 5][c & 31]));
          }
        } else {
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const float s = __uint_as_float(sr[c >> 5][c & 31]);
            mx = fmaxf(mx, c < lim ? (neg ? -s : s) : -INFINITY);
          }
        }
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * cs_abs;
        const float m_new = fmaxf(m_run, m_tile);
        const bool rescale = m_new > m_run + 8.0f;
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
        if (rescale) {
          m_run = m_new;
          l_run *= alpha;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;

        // P = 2^(cs*s - m), row sum, pack to 16-bit pairs
        uint32_t pk[2][32];
        float rs0 = 0.f, rs1 = 0.f;
        if (!need_mask) {
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), cs, -m_use));
            const float p1 =
                ex2_approx(fmaf(__uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]), cs, -m_use));
            rs0 += p0;
            rs1 += p1;
            pk[c >> 6][(c >> 1) & 31] = pack2<false>(p0, p1);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            float p0 = ex2_approx(fmaf(__uint_as_float(sr[c >> 5][c & 31]), cs, -m_use));
            float p1 =
                ex2_approx(fmaf(__uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]), cs, -m_use));
            p0 = c < lim ? p0 : 0.f;
            p1 = c + 1 < lim ? p1 : 0.f;
            rs0 += p0;
            rs1 += p1;
            pk[c >> 6][(c >> 1) & 31] = pack2<false>(p0, p1);
          }
        }
        l_run += rs0 + rs1;
        tmem_st32(tS + 64, pk[0]);
        tmem_st32(tS + 96, pk[1]);

        // lazy rescale of O (the previous P V of this tile completed before S_t(j) did)
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
            reg_order_after_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarPReady + t));
      }

      // ---- epilogue: O / l -> 16-bit -> swizzled smem (this tile's Q buffer) -> TMA store
      mbar_wait(BAR(C::kBarOFull + t), 0, wctx);
      __syncwarp();
      tc_fence_after_sync();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint8_t* stage = smem + C::kOffQ + t * C::kTileBytes;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        reg_order_after_wait(o);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // four 16-byte chunks of 8 elements
          uint4 w;
          w.x = pack2<BF16>(__uint_as_float(o[q4 * 8 + 0]) * inv_l, __uint_as_float(o[q4 * 8 + 1]) * inv_l);
          w.y = pack2<BF16>(__uint_as_float(o[q4 * 8 + 2]) * inv_l, __uint_as_float(o[q4 * 8 + 3]) * inv_l);
          w.z = pack2<BF16>(__uint_as_float(o[q4 * 8 + 4]) * inv_l, __uint_as_float(o[q4 * 8 + 5]) * inv_l);
          w.w = pack2<BF16>(__uint_as_float(o[q4 * 8 + 6]) * inv_l, __uint_as_float(o[q4 * 8 + 7]) * inv_l);
          const int chunk = c * 4 + q4;  // 16-byte chunk index along the row
          const int bx = chunk >> 3, cc = chunk & 7;
          *reinterpret_cast<uint4*>(stage + bx * C::kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + t, 128);
      if (r == 0 && !*abort_flag) {
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_store_4d(&p.tm_o, sbase + C::kOffQ + t * C::kTileBytes + bx * C::kBoxBytes, bx * 64,
                       h, row0, b);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
      if (p.lse != nullptr && grow < p.Nq) {
        const float lse = l_run > 0.f ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f
                                      : -INFINITY;
        p.lse[((long long)b * p.H + h) * p.Nq + grow] = lse;
      }
    } else if (row0 < p.Nq) {
      // every row of this tile is left without a key (causal, Nq > Nk): O = 0, lse = -inf
      if (grow < p.Nq) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) +
                                              ((((long long)b * p.Nq + grow) * p.H + h) * D) * 2);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        if (p.lse != nullptr) p.lse[((long long)b * p.H + h) * p.Nq + grow] = -INFINITY;
      }
    }
  }

  // ---- teardown: every role is done with TMEM
  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn_b200

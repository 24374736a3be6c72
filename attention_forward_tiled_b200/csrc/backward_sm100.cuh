// backward_sm100.cuh -- gradients of the tiled attention forward (sm_100a).
//
// The step after the forward: the FlashAttention/ops-transformer article notes
// (section "传统注意力的显存陷阱") that eager attention keeps the N x N matrix for
// backpropagation; here, as in the forward, it is recomputed tile by tile from Q, K
// and the row log-sum-exp the forward wrote, and never stored:
//   P = exp(scale * Q K^T - lse)            (masked entries 0)
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),  D_i = sum_t dO_it O_it
//   dQ = scale * dS K,   dK = scale * dS^T Q
//
// One CTA per (b, h, 128-key tile): K_j and V_j stay in shared memory and the CTA
// walks the 64-query tiles that see them.  Per query tile, on the tensor cores
// (thread = key of the tile for the elementwise part):
//   S^T  = K Q^T    and  dP^T = V dO^T    (shared-memory operands, TMEM accumulators)
//   P^T, dS^T -> fp16/bf16 into the consumed TMEM columns (and dS^T into shared memory)
//   dV  += P^T dO   and  dK  += dS^T Q    (A from TMEM, B = dO / Q read MN-major)
//   dQ^T = K^T dS^T                       (A = K read MN-major, B = dS^T in shared memory)
// dQ^T (lane = head-dim element, column = query) is staged in shared memory and added to
// an fp32 accumulator in global memory with one TMA reduce-add per tile (other key tiles
// add to the same rows);
// dV and dK are written once at the end.  Roles (320 threads): warps 0-7 elementwise and
// epilogues (two warps per TMEM lane quarter, each taking 32 of a tile's 64 query columns),
// warp 8 TMA producer, warp 9 MMA issuer.
//
// TMEM columns: S^T [0,64) (P^T packed in [0,32)), dP^T [64,128) (dS^T packed in
// [64,96)), dQ^T [128,192), dV [256,256+D), dK [384,384+D).
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

struct BwdParams {
  CUtensorMap tm_q;   // q  [B, Nq, H, D] as 4-D (D, H, Nq, B), box (64, 1, 64, 1), 128B swizzle
  CUtensorMap tm_do;  // dO [B, Nq, H, D], same
  CUtensorMap tm_k;   // k  [B, Nk, H, D], box (64, 1, 128, 1)
  CUtensorMap tm_v;   // v  [B, Nk, H, D], same
  CUtensorMap tm_dq;  // dq_acc [B, Nq, H, D] fp32 as 4-D (D, H, Nq, B), box (D, 1, 64, 1), no swizzle
  const float* lse;   // [B, H, Nq] natural log (the forward's)
  const float* dsum;  // [B, H, Nq]: D_i = sum_t dO_it O_it
  float* dq_acc;      // [B, Nq, H, D] fp32, zeroed before the launch
  void* dk;           // [B, Nk, H, D]
  void* dv;           // [B, Nk, H, D]
  int* status;
  int B, H, Nq, Nk, causal;
  int n_ktiles;       // ceil(Nk / 128)
  float scale;
  float scale_log2;   // scale * log2(e)
  unsigned long long timeout_ns;
};

template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxes = D / 64;
  static constexpr int kKBox = 128 * 128;                  // 128 rows x 64 elements x 2 bytes
  static constexpr int kQBox = 64 * 128;                   // 64 rows x 64 elements x 2 bytes
  static constexpr int kKTile = kBoxes * kKBox;            // K or V tile
  static constexpr int kQTile = kBoxes * kQBox;            // Q or dO tile
  static constexpr int kStages = 2;                        // Q + dO stages
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kKTile;
  static constexpr int kOffQ = 2 * kKTile;                 // [stage]: Q tile then dO tile
  static constexpr int kStageBytes = 2 * kQTile;
  static constexpr int kOffDS = kOffQ + kStages * kStageBytes;  // dS^T [128 keys][64 queries] fp16
  static constexpr int kDSBytes = 128 * 128;
  static constexpr int kOffRow = kOffDS + kDSBytes;        // per-query lse2 and D, [2][2][64] fp32
  static constexpr int kOffDQ = kOffRow + 2 * 2 * 64 * 4;  // dQ tile [64 queries][D] fp32 for the reduce
  static constexpr int kOffBar = kOffDQ + 64 * D * 4;
  static constexpr int kBarKV = 0;
  static constexpr int kBarQFull = 1;                      // [2]
  static constexpr int kBarQEmpty = 3;                     // [2]
  static constexpr int kBarSFull = 5;                      // S^T and dP^T landed
  static constexpr int kBarPDone = 6;                      // P^T, dS^T written (8 warps)
  static constexpr int kBarDQFull = 7;                     // dQ^T landed
  static constexpr int kBarDQFree = 8;                     // dQ^T read (8 warps)
  static constexpr int kBarMmaDone = 9;
  static constexpr int kNumBars = 10;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr int kEwWarps = 8;  // elementwise: two per TMEM lane quarter, 32 query columns each
  static constexpr int kThreads = 32 * (kEwWarps + 2);
  static constexpr int kProducerWarp = kEwWarps;
  static constexpr int kMmaWarp = kEwWarps + 1;
  static constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128, kColDV = 256, kColDK = 384;
  static_assert(kOffQ % 1024 == 0 && kOffDS % 1024 == 0 && kQTile % 1024 == 0, "swizzle atoms");
  static_assert(kOffDQ % 128 == 0, "bulk-copy source alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// First 64-query tile that sees key tile j (keys [128 j, 128 j + 128)): under the causal
// flag query i sees key k iff k <= i + Nk - Nq.
__device__ __forceinline__ int bwd_first_qtile(const BwdParams& p, int j) {
  if (!p.causal) return 0;
  const long long q_min = (long long)j * 128 - ((long long)p.Nk - p.Nq);
  return q_min <= 0 ? 0 : (int)(q_min / 64);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  auto BAR = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};
  // CTA -> (b, h, key tile); key tile 0 (seen by the most queries under the causal flag) first
  const int j = blockIdx.x % p.n_ktiles;
  const int bh = blockIdx.x / p.n_ktiles;
  const int b = bh / p.H, h = bh - b * p.H;
  const int qt0 = bwd_first_qtile(p, j);
  const int nqt = max(0, (p.Nq + 63) / 64 - qt0);

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::kBarKV), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarQFull + i), 1);
      mbar_init(BAR(C::kBarQEmpty + i), 1);
    }
    mbar_init(BAR(C::kBarSFull), 1);
    mbar_init(BAR(C::kBarPDone), C::kEwWarps);
    mbar_init(BAR(C::kBarDQFull), 1);
    mbar_init(BAR(C::kBarDQFree), C::kEwWarps);
    mbar_init(BAR(C::kBarMmaDone), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
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
      tma_prefetch_map(&p.tm_do);
      tma_prefetch_map(&p.tm_k);
      tma_prefetch_map(&p.tm_v);
      tma_prefetch_map(&p.tm_dq);
    }
    mbar_arrive_expect_tx_w(BAR(C::kBarKV), 2 * C::kKTile);
    for (int bx = 0; bx < C::kBoxes; ++bx) {
      tma_load_4d_w(sbase + C::kOffK + bx * C::kKBox, &p.tm_k, BAR(C::kBarKV), bx * 64, h, j * 128, b);
      tma_load_4d_w(sbase + C::kOffV + bx * C::kKBox, &p.tm_v, BAR(C::kBarKV), bx * 64, h, j * 128, b);
    }
    int i = 0;
    for (; i < nqt; ++i) {
      const int st = i & 1;
      if (i >= 2) mbar_wait(BAR(C::kBarQEmpty + st), ((i >> 1) - 1) & 1, wctx);
      __syncwarp();
      if (warp_flag(abort_flag)) break;
      const uint32_t dst = sbase + C::kOffQ + st * C::kStageBytes;
      const int q0 = (qt0 + i) * 64;
      mbar_arrive_expect_tx_w(BAR(C::kBarQFull + st), C::kStageBytes);
      for (int bx = 0; bx < C::kBoxes; ++bx) {
        tma_load_4d_w(dst + bx * C::kQBox, &p.tm_q, BAR(C::kBarQFull + st), bx * 64, h, q0, b);
        tma_load_4d_w(dst + C::kQTile + bx * C::kQBox, &p.tm_do, BAR(C::kBarQFull + st), bx * 64, h, q0, b);
      }
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this warp started land before the CTA can exit
      mbar_wait_drain(BAR(C::kBarKV), 0, p.timeout_ns);
      for (int t = max(0, i - 2); t < i; ++t)
        mbar_wait_drain(BAR(C::kBarQFull + (t & 1)), (t >> 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer =======================
    // S^T = K Q^T, dP^T = V dO^T: M = 128 keys, N = 64 queries, both operands K-major.
    constexpr uint32_t idesc_s = make_idesc_f16(128, 64, BF16, false, false);
    // dV += P^T dO, dK += dS^T Q: A (keys x queries) from TMEM, B = dO / Q read MN-major.
    constexpr uint32_t idesc_kv = make_idesc_f16(128, D, BF16, true, false);
    // dQ^T = K^T dS^T: M = 128 (head dim; at D = 64 the 64 rows are read twice), N = 64
    // queries, K = 128 keys; A = K tile read MN-major, B = dS^T in shared memory MN-major.
    constexpr uint32_t idesc_q = make_idesc_f16(128, 64, BF16, true, true);
    constexpr uint32_t kLboK = (D == 128) ? C::kKBox : 0;
    const uint32_t sK = sbase + C::kOffK, sV = sbase + C::kOffV, sDS = sbase + C::kOffDS;
    mbar_wait(BAR(C::kBarKV), 0, wctx);
    for (int i = 0; i < nqt; ++i) {
      const int st = i & 1;
      const uint32_t sQ = sbase + C::kOffQ + st * C::kStageBytes, sDO = sQ + C::kQTile;
      mbar_wait(BAR(C::kBarQFull + st), (i >> 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // 16 head-dim elements per k-step
          const uint32_t ka = (kk >> 2) * C::kKBox + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * C::kQBox + (kk & 3) * 32;
          mma_f16_ss_w(tmem + C::kColS, make_sdesc_sw128(sK + ka, 16, 1024),
                       make_sdesc_sw128(sQ + kb, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          mma_f16_ss_w(tmem + C::kColDP, make_sdesc_sw128(sV + ka, 16, 1024),
                       make_sdesc_sw128(sDO + kb, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(BAR(C::kBarSFull));
      }
      mbar_wait(BAR(C::kBarPDone), i & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 queries per k-step: 8 packed TMEM columns
          // queries 32 h .. 32 h + 31 are packed at columns 32 h .. 32 h + 15
          const uint32_t pcol = (kk >> 1) * 32 + (kk & 1) * 8;
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_f16_ts_w(tmem + C::kColDV, tmem + C::kColS + pcol,
                       make_sdesc_sw128(sDO + kk * 2048, C::kQBox, 1024), idesc_kv, acc);
          mma_f16_ts_w(tmem + C::kColDK, tmem + C::kColDP + pcol,
                       make_sdesc_sw128(sQ + kk * 2048, C::kQBox, 1024), idesc_kv, acc);
        }
      }
      if (i > 0) mbar_wait(BAR(C::kBarDQFree), (i - 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys per k-step
          mma_f16_ss_w(tmem + C::kColDQ, make_sdesc_sw128(sK + kk * 2048, kLboK, 1024),
                       make_sdesc_sw128(sDS + kk * 2048, 16, 1024), idesc_q, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(BAR(C::kBarDQFull));
        tc_commit_w(BAR(C::kBarQEmpty + st));
      }
    }
    // every MMA (and every commit arrive) has landed before TMEM is released
    tc_commit_w(BAR(C::kBarMmaDone));
    mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    __syncwarp();
  } else {
    // ======================= elementwise warps 0-7 ==========
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (keys for S^T, dP^T, dV, dK; head-dim
    // elements for dQ^T) and takes query columns 32 hf .. + 31, hf = w / 4, of each tile
    // (and half of the head-dim columns of dV and dK at the end).
    const int hf = warp >> 2;
    const int r = (warp & 3) * 32 + lane;  // TMEM lane: key of the tile / head-dim element of dQ^T
    const int tid = threadIdx.x;           // 0..255
    const int c_off = hf * 32;             // this warp's query columns
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int key = j * 128 + r;
    const long long diag = (long long)p.Nk - p.Nq;
    float* rowbuf = reinterpret_cast<float*>(smem + C::kOffRow);  // [2][2][64]: lse2, D
    uint8_t* ds_row = smem + C::kOffDS + r * 128;                  // dS^T row of this key
    float* dq_stage = reinterpret_cast<float*>(smem + C::kOffDQ);  // [64][D]
    // per-query lse (base 2) and D of query tile i into rowbuf[i & 1]: loaded a tile ahead,
    // stored to shared memory after this tile's work, so the load latency is hidden
    auto row_load = [&](int i, float& l2, float& dd) {
      const int q = (qt0 + i) * 64 + tid;
      const long long o = ((long long)b * p.H + h) * p.Nq + q;
      l2 = (tid < 64 && q < p.Nq) ? __ldg(p.lse + o) * 1.4426950408889634f : 0.f;
      dd = (tid < 64 && q < p.Nq) ? __ldg(p.dsum + o) : 0.f;
    };
    float nl2 = 0.f, ndd = 0.f;
    if (nqt > 0) {
      row_load(0, nl2, ndd);
      if (tid < 64) {
        rowbuf[tid] = nl2;
        rowbuf[64 + tid] = ndd;
      }
    }
    named_bar_sync(1, 32 * C::kEwWarps);
    for (int i = 0; i < nqt; ++i) {
      const int q0 = (qt0 + i) * 64;
      const float* lse2 = rowbuf + (i & 1) * 128 + c_off;
      const float* dsm = rowbuf + (i & 1) * 128 + 64 + c_off;
      if (i + 1 < nqt) row_load(i + 1, nl2, ndd);
      mbar_wait(BAR(C::kBarSFull), i & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      uint32_t s[32], dp[32];
      tmem_ld32(tmem + lane_base + C::kColS + c_off, s);
      tmem_ld32(tmem + lane_base + C::kColDP + c_off, dp);
      tmem_ld_wait();
      reg_order_after_wait(s);
      reg_order_after_wait(dp);
      // query q0 + c sees this key iff key < Nk, q0 + c < Nq and (causal) key <= q0 + c + Nk - Nq;
      // a key that every query of this warp's columns sees takes no per-element test
      const int qa = q0 + c_off;
      const bool all_see = key < p.Nk && qa + 31 < p.Nq && (!p.causal || (long long)key <= qa + diag);
      uint32_t pk[16], dk2[16];
#pragma unroll
      for (int c8 = 0; c8 < 32; c8 += 8) {
        const float4 la = *reinterpret_cast<const float4*>(lse2 + c8);
        const float4 lb = *reinterpret_cast<const float4*>(lse2 + c8 + 4);
        const float4 da = *reinterpret_cast<const float4*>(dsm + c8);
        const float4 db = *reinterpret_cast<const float4*>(dsm + c8 + 4);
        const float l8[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
        const float d8[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        float pv[8], dv8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int col = c8 + e;
          float pr = ex2_approx(__uint_as_float(s[col]) * p.scale_log2 - l8[e]);
          if (!all_see) {
            const int q = qa + col;
            const bool ok = key < p.Nk && q < p.Nq && (!p.causal || (long long)key <= q + diag);
            pr = ok ? pr : 0.f;
          }
          pv[e] = pr;
          dv8[e] = pr * (__uint_as_float(dp[col]) - d8[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          pk[(c8 + e) >> 1] = pack2<BF16>(pv[e], pv[e + 1]);
          dk2[(c8 + e) >> 1] = pack2<BF16>(dv8[e], dv8[e + 1]);
        }
      }
      // P^T and dS^T (packed pairs) into the first 16 of the S^T / dP^T columns this warp
      // itself read (32 hf .. 32 hf + 15): never into columns the other warp of the lane
      // quarter may still be reading
      tmem_st16(tmem + lane_base + C::kColS + hf * 32, pk);
      tmem_st16(tmem + lane_base + C::kColDP + hf * 32, dk2);
      // dS^T row (64 queries, 128 bytes) into shared memory, 128-byte swizzle (MN-major B):
      // this warp's four 16-byte chunks
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const uint4 w = make_uint4(dk2[cc * 4 + 0], dk2[cc * 4 + 1], dk2[cc * 4 + 2], dk2[cc * 4 + 3]);
        *reinterpret_cast<uint4*>(ds_row + (((hf * 4 + cc) ^ (r & 7)) << 4)) = w;
      }
      tmem_st_wait();
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::kBarPDone));

      // dQ^T of this tile (lane = head-dim element; this warp's 32 query columns) -> shared
      // memory as [query][D] -> one TMA reduce-add into the fp32 accumulator (rows past Nq
      // are skipped)
      mbar_wait(BAR(C::kBarDQFull), i & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      uint32_t dq[32];
      tmem_ld32(tmem + lane_base + C::kColDQ + c_off, dq);
      tmem_ld_wait();
      reg_order_after_wait(dq);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::kBarDQFree));
      if (tid == 0) bulk_wait_group_read0();  // the previous tile's reduce has read the stage
      named_bar_sync(1, 32 * C::kEwWarps);
      if (r < D) {
#pragma unroll
        for (int c = 0; c < 32; ++c) dq_stage[(c_off + c) * D + r] = __uint_as_float(dq[c]);
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the TMA
      // next tile's per-query rows, loaded at the top of this iteration
      if (i + 1 < nqt && tid < 64) {
        rowbuf[((i + 1) & 1) * 128 + tid] = nl2;
        rowbuf[((i + 1) & 1) * 128 + 64 + tid] = ndd;
      }
      named_bar_sync(1, 32 * C::kEwWarps);
      if (tid == 0 && !*abort_flag) {
        tma_reduce_add_4d(&p.tm_dq, sbase + C::kOffDQ, 0, h, q0, b);
        bulk_commit_group();
      }
    }
    if (tid == 0) bulk_wait_group_read0();  // ... and the last one before the CTA exits
    if (tid == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");

    // ---- epilogue: dV and scale * dK (lane = key) -> 16-bit -> global; this warp takes
    // head-dim columns hf * D / 2 .. + D / 2.  The last tile's dQ^T commit covered every
    // earlier product, so dV and dK are final here.  The TMEM loads are warp-collective:
    // every lane takes part, and only rows of keys below Nk are stored (the last key tile
    // may be partial).
    const bool key_row = key < p.Nk;
    const long long row = (((long long)b * p.Nk + (key_row ? key : 0)) * p.H + h) * D;
    uint4* dvrow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.dv) + row * 2);
    uint4* dkrow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.dk) + row * 2);
    if (nqt == 0) {  // no query sees this key tile
      if (key_row) {
#pragma unroll
        for (int c = hf * D / 16; c < (hf + 1) * D / 16; ++c) {
          dvrow[c] = make_uint4(0u, 0u, 0u, 0u);
          dkrow[c] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    } else {
      tc_fence_after_sync();
#pragma unroll 1
      for (int c = hf * D / 64; c < (hf + 1) * D / 64; ++c) {
        uint32_t a[32], k2[32];
        tmem_ld32(tmem + lane_base + C::kColDV + c * 32, a);
        tmem_ld32(tmem + lane_base + C::kColDK + c * 32, k2);
        tmem_ld_wait();
        reg_order_after_wait(a);
        reg_order_after_wait(k2);
        if (!key_row) continue;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 wv, wk;
          wv.x = pack2<BF16>(__uint_as_float(a[q4 * 8 + 0]), __uint_as_float(a[q4 * 8 + 1]));
          wv.y = pack2<BF16>(__uint_as_float(a[q4 * 8 + 2]), __uint_as_float(a[q4 * 8 + 3]));
          wv.z = pack2<BF16>(__uint_as_float(a[q4 * 8 + 4]), __uint_as_float(a[q4 * 8 + 5]));
          wv.w = pack2<BF16>(__uint_as_float(a[q4 * 8 + 6]), __uint_as_float(a[q4 * 8 + 7]));
          wk.x = pack2<BF16>(__uint_as_float(k2[q4 * 8 + 0]) * p.scale, __uint_as_float(k2[q4 * 8 + 1]) * p.scale);
          wk.y = pack2<BF16>(__uint_as_float(k2[q4 * 8 + 2]) * p.scale, __uint_as_float(k2[q4 * 8 + 3]) * p.scale);
          wk.z = pack2<BF16>(__uint_as_float(k2[q4 * 8 + 4]) * p.scale, __uint_as_float(k2[q4 * 8 + 5]) * p.scale);
          wk.w = pack2<BF16>(__uint_as_float(k2[q4 * 8 + 6]) * p.scale, __uint_as_float(k2[q4 * 8 + 7]) * p.scale);
          dvrow[c * 4 + q4] = wv;
          dkrow[c * 4 + q4] = wk;
        }
      }
    }
  }

  // ---- teardown: every role is done with TMEM
  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = sum_t dO_it O_it in fp32 (one warp per (b, i, h) row) and zeroed dQ accumulator rows.
template <int D, bool BF16>
__global__ void __launch_bounds__(128)
    attn_bwd_pre_kernel(const void* __restrict__ o, const void* __restrict__ dout,
                        float* __restrict__ dsum, float* __restrict__ dq_acc, int B, int H, int Nq) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 4 + warp;  // (b * Nq + i) * H + h
  if (row >= (long long)B * Nq * H) return;
  const int h = (int)(row % H);
  const long long bi = row / H;
  const int i = (int)(bi % Nq), b = (int)(bi / Nq);
  const uint8_t* orow = static_cast<const uint8_t*>(o) + row * D * 2 + lane * E * 2;
  const uint8_t* grow = static_cast<const uint8_t*>(dout) + row * D * 2 + lane * E * 2;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const float2 a = unpack2<BF16>(*reinterpret_cast<const uint32_t*>(orow + e * 2));
    const float2 g = unpack2<BF16>(*reinterpret_cast<const uint32_t*>(grow + e * 2));
    acc = fmaf(a.x, g.x, fmaf(a.y, g.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) dsum[((long long)b * H + h) * Nq + i] = acc;
  float* z = dq_acc + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) z[e] = 0.f;
}

// dQ = scale * accumulated dS K, cast to the input type (two elements per thread).
template <bool BF16>
__global__ void __launch_bounds__(256)
    attn_bwd_dq_kernel(const float* __restrict__ dq_acc, void* __restrict__ dq, long long n2, float scale) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n2) return;
  const float2 a = reinterpret_cast<const float2*>(dq_acc)[t];
  reinterpret_cast<uint32_t*>(dq)[t] = pack2<BF16>(a.x * scale, a.y * scale);
}

}  // namespace attn_b200

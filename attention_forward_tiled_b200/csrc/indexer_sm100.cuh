// indexer_sm100.cuh -- lightning-indexer score and top-k selection (sm_100a).
//
// Score (aispot.cmou.io report on llama.cpp release b11372, entry "compute the
// indexer score with the lightning indexer"): every query token t scores every
// pooled key p by the rectified dot product of each of its H indexer heads with
// that key, weighted per head and summed over the heads; the keys have no head
// axis, so one key row serves all heads, and an additive pool mask follows:
//   score[b, t, p] = sum_h w[b, t, h] * max(0, q[b, t, h, :] . kp[b, p, :]) + mask[b, t, p]
//
// On the tensor cores the pooled keys are the M = 128 rows of a tcgen05.mma and the
// (token, head) pairs of 128 / H tokens its N = 128 columns, so the product lands
// in TMEM with one thread per key holding every head of every token of the tile:
// the rectifier, the head weights and the head sum stay inside a thread.  Work
// items (b, pair of key tiles, token tile) go to persistent CTAs (352 threads):
//   * warp 8, producer: TMA loads of a pair of key tiles (once per run of items on the
//     same pair) and of the query tiles (a four-deep ring) into shared memory;
//   * warp 10, auxiliary loads: the item's mask tile by TMA and its head weights by
//     cp.async, double-buffered;
//   * warp 9, MMA issuer: S^T = Kp Q^T for both key tiles of the pair (two TMEM
//     accumulators per item, two items in flight), so each query tile serves 256 keys;
//   * warps 0-7, epilogue: rectify, weight, sum over heads, add the f16 mask and
//     store fp32 scores (one thread per key: consecutive keys, coalesced stores).
//
// Top-k (prhub.com.cn report "PR #45743 完整报告", section "实现拆解": the decode
// indexer keeps only the order of the scores): one CTA per score row finds the
// k-th largest score by a most-significant-digit radix select over order-preserving
// 32-bit keys, gathers the k winners (ties to the lower position), sorts them
// (largest first, then lower position first) and writes their positions; -inf and
// NaN are never chosen and short rows are padded with -1.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

struct IndexerParams {
  CUtensorMap tm_q;     // q [B, T, H, D] as 3-D (D, T*H, B), box (64, 128, 1), 128B swizzle
  CUtensorMap tm_k;     // kp [B, P, D] as 3-D (D, P, B), box (64, 128, 1), 128B swizzle
  CUtensorMap tm_mask;  // mask [B, T, P] f16 as 3-D (P, T, B), box (256, 128 / H, 1), no swizzle
  const float* w;       // [B, T, H]
  const uint16_t* mask;  // [B, T, P] f16 (0 / -inf) or nullptr
  float* score;         // [B, T, P]
  int* status;
  int B, T, H, P;
  int lg_h;             // log2(H)
  int tok_per_tile;     // 128 / H
  int mask_tma;         // 1: mask tiles come by TMA (H >= 4, P % 8 == 0, 16-byte aligned mask)
  int n_ttiles, n_pairs, n_items;  // token tiles, pairs of key tiles, items
  unsigned long long timeout_ns;
};

template <int D>
struct IndexerCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxBytes = 128 * 128;             // 128 rows x 64 elements x 2 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;   // 128 rows x D
  static constexpr int kQStages = 4;      // query tiles come from L2 for every item: a deep ring
  static constexpr int kMaskTokens = 32;  // mask rows held per buffer: tiles of H >= 4 heads
  static constexpr int kOffK = 0;                                  // the pair of key tiles
  static constexpr int kOffQ = 2 * kTileBytes;                     // query tiles [kQStages]
  static constexpr int kOffW = kOffQ + kQStages * kTileBytes;     // head weights [2][128] fp32
  static constexpr int kOffM = kOffW + 2 * 128 * 4;                // pool mask [2][kMaskTokens][256 keys] f16
  static constexpr int kOffBar = kOffM + 2 * kMaskTokens * 256 * 2;
  static constexpr int kBarKFull = 0;                     // [1]
  static constexpr int kBarKEmpty = 1;                    // [1]
  static constexpr int kBarQFull = 2;                     // [kQStages]
  static constexpr int kBarQEmpty = 2 + kQStages;         // [kQStages]
  static constexpr int kBarAccFull = 2 + 2 * kQStages;    // [2] an item's two accumulators
  static constexpr int kBarAccFree = 4 + 2 * kQStages;    // [2] ... free, and its weights and mask read
  static constexpr int kBarAuxFull = 6 + 2 * kQStages;    // [2] weights and mask of an item landed
  static constexpr int kBarMmaDone = 8 + 2 * kQStages;    // [1]
  static constexpr int kNumBars = 9 + 2 * kQStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // +1024: manual 1 KB alignment
  static constexpr int kEpiWarps = 8;                      // one per (key tile, TMEM lane quarter)
  static constexpr int kThreads = 32 * (kEpiWarps + 3);
  static constexpr int kProducerWarp = kEpiWarps;   // key and query tiles
  static constexpr int kMmaWarp = kEpiWarps + 1;
  static constexpr int kAuxWarp = kEpiWarps + 2;    // head weights and mask tiles
  static constexpr uint32_t kTmemCols = 512;        // two items in flight x two 128-column accumulators
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Item -> (b, pair of key tiles, token tile); the items of one pair are consecutive, and
// each CTA takes a contiguous range of items, so it loads a pair once for all the token
// tiles of that range, and every query tile it loads serves 256 keys.
struct IndexerItem {
  int b, pp, tt;
};

__device__ __forceinline__ IndexerItem indexer_item(const IndexerParams& p, int item) {
  IndexerItem it;
  it.tt = item % p.n_ttiles;
  const int bp = item / p.n_ttiles;
  it.pp = bp % p.n_pairs;
  it.b = bp / p.n_pairs;
  return it;
}

// the item after it, without divisions
__device__ __forceinline__ void indexer_next(const IndexerParams& p, IndexerItem& it) {
  if (++it.tt == p.n_ttiles) {
    it.tt = 0;
    if (++it.pp == p.n_pairs) {
      it.pp = 0;
      ++it.b;
    }
  }
}

// Asynchronous 4-byte global -> shared copy (the LDGSTS path); bytes past src_bytes are
// filled with zeros without being read.
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// One arrival on the mbarrier once every earlier cp.async of this thread has landed (the
// barrier's expected count includes it).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Epilogue of the score kernel: eight warps, thread = key (TMEM lane) of a tile.  Warp w
// reads lanes 32 (w % 4) .. + 31 of the accumulator of key tile (w / 4) of the pair, all 128
// columns.  H = 2^LGH heads, so the columns are 128 / H tokens of H heads each (column =
// token * H + head) and a token's score is the weighted sum of its H rectified columns
// (carried across 32-column pieces when H > 32).  The head weights and the mask rows
// of the item were put in shared memory by the auxiliary-load warp; the mask came by TMA
// when its rows are 16-byte aligned and a tile has at most 32 tokens (H >= 4), else it is
// read from global memory here.
template <int D, int LGH>
__device__ __forceinline__ void indexer_epilogue(const IndexerParams& p, uint8_t* smem, uint32_t tmem,
                                                 uint64_t* bars, const WaitCtx& wctx, int item0,
                                                 int item1) {
  using C = IndexerCfg<D>;
  constexpr int H = 1 << LGH;
  constexpr int TPT = 128 / H;            // tokens per tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = warp >> 2;                 // key tile of the pair
  const int r = (warp & 3) * 32 + lane;     // key within the tile
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const float* wbuf = reinterpret_cast<const float*>(smem + C::kOffW);        // [2][128]
  const uint16_t* mbuf = reinterpret_cast<const uint16_t*>(smem + C::kOffM);  // [2][kMaskTokens][256 keys]

  IndexerItem it = indexer_item(p, item0);
  for (int item = item0, g = 0; item < item1; ++item, ++g, indexer_next(p, it)) {
    const int j = g & 1;  // accumulator pair and weights / mask buffer of this item
    const int t0 = it.tt * TPT;
    const int key = it.pp * 256 + kt * 128 + r;
    const bool key_ok = key < p.P;
    const bool full = t0 + TPT <= p.T;  // no token of the tile lies past T
    // this key's score for token 0 of the tile; token tl is P floats further on
    float* const srow = p.score + ((long long)it.b * p.T + t0) * p.P + key;
    const float* wb = wbuf + j * 128;
    const uint16_t* mb = mbuf + j * C::kMaskTokens * 256 + kt * 128 + r;
    // n scores of consecutive tokens from tl0: the mask values are read before any store,
    // so those reads are not held behind the global stores
    auto emit = [&](int tl0, auto& v) {
      constexpr int n = sizeof(v) / sizeof(float);
      if (p.mask != nullptr) {
        float mv[n];
        if (p.mask_tma) {
#pragma unroll
          for (int u = 0; u < n; ++u) mv[u] = __half2float(__ushort_as_half(mb[(tl0 + u) * 256]));
        } else {
          const uint16_t* mrow = p.mask + ((long long)it.b * p.T + t0 + tl0) * p.P + key;
#pragma unroll
          for (int u = 0; u < n; ++u)
            mv[u] = (key_ok && t0 + tl0 + u < p.T) ? __half2float(__ushort_as_half(mrow[(long long)u * p.P])) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < n; ++u) v[u] += mv[u];
      }
      if (!key_ok) return;
      float* dst = srow + (long long)tl0 * p.P;
      if (full) {
#pragma unroll
        for (int u = 0; u < n; ++u, dst += p.P) *dst = v[u];
      } else {
#pragma unroll
        for (int u = 0; u < n; ++u, dst += p.P)
          if (t0 + tl0 + u < p.T) *dst = v[u];
      }
    };
    mbar_wait(smem_u32(&bars[C::kBarAuxFull + j]), (g >> 1) & 1, wctx);
    mbar_wait(smem_u32(&bars[C::kBarAccFull + j]), (g >> 1) & 1, wctx);
    __syncwarp();
    tc_fence_after_sync();
    const uint32_t acc = tmem + lane_base + (uint32_t)(2 * j + kt) * 128u;
    float carry = 0.f;  // H > 32: a token spans several 32-column pieces
    // four 32-column pieces; the TMEM load of piece i + 1 is in flight while piece i is reduced
    uint32_t sv[2][32];
    tmem_ld32(acc, sv[0]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int cb = i * 32;
      tmem_ld_wait();
      reg_order_after_wait(sv[i & 1]);
      if (i < 3) tmem_ld32(acc + cb + 32, sv[(i + 1) & 1]);
      float wv[32];
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(wb + cb + c);
        wv[c] = w4.x;
        wv[c + 1] = w4.y;
        wv[c + 2] = w4.z;
        wv[c + 3] = w4.w;
      }
      if constexpr (H <= 32) {
        constexpr int NT = 32 / H;          // tokens in the piece
        constexpr int G = NT < 8 ? NT : 8;  // ... emitted eight at a time
#pragma unroll
        for (int u0 = 0; u0 < NT; u0 += G) {
          float v[G];
#pragma unroll
          for (int u = 0; u < G; ++u) {
            float a = 0.f;
#pragma unroll
            for (int h = 0; h < H; ++h)
              a = fmaf(wv[(u0 + u) * H + h], fmaxf(__uint_as_float(sv[i & 1][(u0 + u) * H + h]), 0.f), a);
            v[u] = a;
          }
          emit((cb >> LGH) + u0, v);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) carry = fmaf(wv[c], fmaxf(__uint_as_float(sv[i & 1][c]), 0.f), carry);
        if (((cb + 32) & (H - 1)) == 0) {
          float v[1] = {carry};
          emit(cb >> LGH, v);
          carry = 0.f;
        }
      }
    }
    // accumulators 2j, 2j + 1 and weights / mask buffer j are free for item g + 2
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[C::kBarAccFree + j]));
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(IndexerCfg<D>::kThreads, 1)
    attn_indexer_score_kernel(const __grid_constant__ IndexerParams p, int items_per_cta) {
  using C = IndexerCfg<D>;
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
  // this CTA's items: a contiguous range, so consecutive items share a pair of key tiles
  const int item0 = blockIdx.x * items_per_cta;
  const int item1 = min(p.n_items, item0 + items_per_cta);

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::kBarKFull), 1);
    mbar_init(BAR(C::kBarKEmpty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarAccFull + i), 1);
      mbar_init(BAR(C::kBarAccFree + i), C::kEpiWarps);  // one arrive per epilogue warp
      mbar_init(BAR(C::kBarAuxFull + i), 33);  // the byte-count arrive + one cp.async arrive per lane
    }
    for (int s = 0; s < C::kQStages; ++s) {
      mbar_init(BAR(C::kBarQFull + s), 1);
      mbar_init(BAR(C::kBarQEmpty + s), 1);
    }
    mbar_init(BAR(C::kBarMmaDone), 1);
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

  auto same_pair = [&](const IndexerItem& a, const IndexerItem& b) { return a.b == b.b && a.pp == b.pp; };

  if (warp == C::kProducerWarp) {
    // ======================= producer: key-tile pairs and query tiles =======================
    if (lane == 0) {
      tma_prefetch_map(&p.tm_q);
      tma_prefetch_map(&p.tm_k);
    }
    int nk = 0;  // pairs loaded
    int nq = 0;  // query tiles loaded
    IndexerItem prev{-1, -1, -1};
    IndexerItem it = indexer_item(p, item0);
    for (int item = item0, g = 0; item < item1; ++item, ++g, indexer_next(p, it)) {
      if (!same_pair(it, prev)) {
        // one buffer: a new pair waits until the MMAs are done with the previous one (once
        // or twice per CTA).  The second tile of the last pair may lie past P: TMA fills zeros.
        if (nk >= 1) mbar_wait(BAR(C::kBarKEmpty), (nk - 1) & 1, wctx);
        __syncwarp();
        if (warp_flag(abort_flag)) break;
        mbar_arrive_expect_tx_w(BAR(C::kBarKFull), 2 * C::kTileBytes);
        for (int kt = 0; kt < 2; ++kt)
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d_w(sbase + C::kOffK + kt * C::kTileBytes + bx * C::kBoxBytes, &p.tm_k,
                          BAR(C::kBarKFull), bx * 64, (it.pp * 2 + kt) * 128, it.b);
        ++nk;
        prev = it;
      }
      const int st = g % C::kQStages;
      if (g >= C::kQStages) mbar_wait(BAR(C::kBarQEmpty + st), ((g / C::kQStages) - 1) & 1, wctx);
      __syncwarp();
      if (warp_flag(abort_flag)) break;
      mbar_arrive_expect_tx_w(BAR(C::kBarQFull + st), C::kTileBytes);
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_3d_w(sbase + C::kOffQ + st * C::kTileBytes + bx * C::kBoxBytes, &p.tm_q,
                      BAR(C::kBarQFull + st), bx * 64, it.tt * 128, it.b);
      ++nq;
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this warp started land before the CTA can exit
      for (int i = max(0, nq - C::kQStages); i < nq; ++i)
        mbar_wait_drain(BAR(C::kBarQFull + i % C::kQStages), (i / C::kQStages) & 1, p.timeout_ns);
      if (nk > 0) mbar_wait_drain(BAR(C::kBarKFull), (nk - 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == C::kAuxWarp) {
    // ======================= head weights and mask tiles =======================
    // item g's into buffer g & 1, free once the epilogue is done with item g - 2
    if (lane == 0 && p.mask_tma) tma_prefetch_map(&p.tm_mask);
    const int tpt = p.tok_per_tile;
    const uint32_t mask_bytes = p.mask_tma ? (uint32_t)tpt * 256u * 2u : 0u;
    int na = 0;  // buffers loaded
    IndexerItem it = indexer_item(p, item0);
    for (int item = item0, g = 0; item < item1; ++item, ++g, indexer_next(p, it)) {
      const int xb = g & 1;
      if (g >= 2) mbar_wait(BAR(C::kBarAccFree + xb), ((g >> 1) - 1) & 1, wctx);
      __syncwarp();
      if (warp_flag(abort_flag)) break;
      const int t0 = it.tt * tpt;
      mbar_arrive_expect_tx_w(BAR(C::kBarAuxFull + xb), mask_bytes);
      if (p.mask_tma)
        tma_load_3d_w(sbase + C::kOffM + xb * (C::kMaskTokens * 256 * 2), &p.tm_mask, BAR(C::kBarAuxFull + xb),
                      it.pp * 256, t0, it.b);
      const float* wrow = p.w + ((long long)it.b * p.T) * p.H;
#pragma unroll
      for (int c = lane; c < 128; c += 32) {  // column c: token c / H, head c % H
        const int t = t0 + (c >> p.lg_h);
        const bool ok = t < p.T;
        cp_async_4(sbase + C::kOffW + (xb * 128 + c) * 4, wrow + (long long)(ok ? t : 0) * p.H + (c & (p.H - 1)),
                   ok ? 4u : 0u);
      }
      cp_async_mbar_arrive(BAR(C::kBarAuxFull + xb));
      ++na;
    }
    cp_async_wait_all();
    if (lane == 0 && *abort_flag) {
      for (int i = max(0, na - 2); i < na; ++i)
        mbar_wait_drain(BAR(C::kBarAuxFull + (i & 1)), (i >> 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer =======================
    constexpr uint32_t idesc = make_idesc_f16(128, 128, BF16, false);  // Kp Q^T, both K-major
    int nk = 0, g = 0;
    IndexerItem prev{-1, -1, -1};
    IndexerItem it = indexer_item(p, item0);
    for (int item = item0; item < item1; ++item, ++g, indexer_next(p, it)) {
      if (!same_pair(it, prev)) {
        if (nk > 0) tc_commit_w(BAR(C::kBarKEmpty));  // the previous pair is released
        mbar_wait(BAR(C::kBarKFull), nk & 1, wctx);
        ++nk;
        prev = it;
      }
      const int st = g % C::kQStages;
      const int j = g & 1;
      mbar_wait(BAR(C::kBarQFull + st), (g / C::kQStages) & 1, wctx);
      if (g >= 2) mbar_wait(BAR(C::kBarAccFree + j), ((g >> 1) - 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
        const uint32_t sQ = sbase + C::kOffQ + st * C::kTileBytes;
#pragma unroll
        for (int kt = 0; kt < 2; ++kt) {
          const uint32_t sK = sbase + C::kOffK + kt * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // 16 head-dim elements per k-step
            const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
            mma_f16_ss_w(tmem + (uint32_t)(2 * j + kt) * 128u, make_sdesc_sw128(sK + off, 16, 1024),
                         make_sdesc_sw128(sQ + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit_w(BAR(C::kBarAccFull + j));
        tc_commit_w(BAR(C::kBarQEmpty + st));
      }
    }
    if (nk > 0) tc_commit_w(BAR(C::kBarKEmpty));
    // every MMA (and every commit arrive) has landed before TMEM is released
    tc_commit_w(BAR(C::kBarMmaDone));
    mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    __syncwarp();
  } else {
    // ======================= epilogue warps 0-7 (thread = pooled key) ===========
    switch (p.lg_h) {  // the head count fixes how columns group into tokens
      case 0: indexer_epilogue<D, 0>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 1: indexer_epilogue<D, 1>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 2: indexer_epilogue<D, 2>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 3: indexer_epilogue<D, 3>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 4: indexer_epilogue<D, 4>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 5: indexer_epilogue<D, 5>(p, smem, tmem, bars, wctx, item0, item1); break;
      case 6: indexer_epilogue<D, 6>(p, smem, tmem, bars, wctx, item0, item1); break;
      default: indexer_epilogue<D, 7>(p, smem, tmem, bars, wctx, item0, item1); break;
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

// ---------------------------------------------------------------------------
// top-k
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 512;
constexpr int kTopkMaxK = 2048;
constexpr int kTopkCache = 49152;  // rows up to this many scores keep their keys in shared memory

// Order-preserving 32-bit key of a score: a larger float gives a larger key, equal
// floats (+0 and -0 included) the same key; -inf and NaN give 0, the key no chosen
// entry has.
__device__ __forceinline__ uint32_t topk_key(float x) {
  if (!(x > -INFINITY)) return 0u;  // -inf, NaN
  const uint32_t b = (x == 0.0f) ? 0u : __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Block-wide exclusive prefix count of a per-thread flag (kTopkThreads threads);
// returns this thread's rank among the flagged threads and the total in *total.
__device__ __forceinline__ int block_rank(bool flag, int* warp_cnt, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warp_cnt[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    const int c = warp_cnt[w];
    before += (w < warp) ? c : 0;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + __popc(bal & ((1u << lane) - 1u));
}

// One CTA per row of P scores: positions of the k largest finite scores, largest first,
// ties to the lower position, -1 past the finite ones.  kCached: the row's keys are kept
// in shared memory (P up to kTopkCache), else every pass reads them from global memory.
template <bool kCached>
__global__ void __launch_bounds__(kTopkThreads)
    attn_topk_kernel(const float* __restrict__ score, int R, int P, int k, int* __restrict__ idx) {
  extern __shared__ uint32_t tsm[];
  uint32_t* hist = tsm;                                 // [256]
  int* warp_cnt = reinterpret_cast<int*>(tsm + 256);    // [32]
  int* ctl = reinterpret_cast<int*>(tsm + 288);         // [8]: digit, remaining, counters
  uint32_t* ckey = tsm + 296;                           // [kp2] candidate keys
  const int kp2 = k <= 1 ? 1 : 1 << (32 - __clz(k - 1));
  int* cidx = reinterpret_cast<int*>(ckey + kp2);       // [kp2] candidate positions
  uint32_t* rowkeys = reinterpret_cast<uint32_t*>(cidx + kp2);  // [P] when kCached
  const int row = blockIdx.x;
  if (row >= R) return;
  const float* srow = score + (long long)row * P;
  const int tid = threadIdx.x;
  auto key_at = [&](int i) -> uint32_t {
    if constexpr (kCached) return rowkeys[i];
    return topk_key(__ldg(srow + i));
  };
  if constexpr (kCached) {
#pragma unroll 8
    for (int i = tid; i < P; i += kTopkThreads) rowkeys[i] = topk_key(__ldg(srow + i));
  }
  // ---- radix select of the k-th largest key, 8 bits at a time from the top
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;   // entries still to choose among those matching the prefix
  bool take_all = false;
  bool few = false;    // the prefix is shared by at most 32 keys: they are sorted by one warp
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < P; i0 += kTopkThreads) {  // uniform trip count: whole warps vote
      const int i = i0 + tid;
      const uint32_t u = i < P ? key_at(i) : 0u;
      const bool hit = u != 0u && (u & pmask) == prefix;
      const uint32_t bin = hit ? (u >> shift) & 255u : 256u;
      if (shift == 24) {
        // one atomic per distinct digit of the warp: most scores share the top digit
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (hit && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      } else if (hit) {
        atomicAdd(&hist[bin], 1u);  // lower digits spread over the bins: few lanes share one
      }
    }
    __syncthreads();
    if (tid < 32) {
      // warp 0 finds the digit where the count from the top reaches `remaining`: lane l
      // holds digits 255 - 8 l ... 248 - 8 l, a shuffle scan gives the count above them
      const int lane_t = tid;
      int cnt[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cnt[u] = (int)hist[255 - 8 * lane_t - u];
        tot += cnt[u];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane_t >= o) incl += y;
      }
      const int excl = incl - tot;
      if (excl < remaining && remaining <= incl) {
        int cum = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (cum + cnt[u] >= remaining) {
            ctl[0] = 255 - 8 * lane_t - u;
            ctl[1] = remaining - cum;
            ctl[2] = cnt[u];
            break;
          }
          cum += cnt[u];
        }
      }
      if (lane_t == 31 && incl < remaining) {  // fewer entries than remaining in total
        ctl[0] = -1;
        ctl[1] = incl;
        ctl[2] = 0;
      }
    }
    __syncthreads();
    const int sel = ctl[0];
    if (sel < 0) {  // fewer finite entries than k (first pass only): every one is chosen
      take_all = true;
      break;
    }
    remaining = ctl[1];
    prefix |= (uint32_t)sel << shift;
    pmask |= 255u << shift;
    if (shift > 0 && shift <= 16 && ctl[2] <= 32) {  // the rest of the digits are not needed
      few = true;
      break;
    }
  }
  const uint32_t thr = prefix;  // the k-th largest key (unless take_all)
  const int eq_total = ctl[2];   // entries equal to thr (last pass)
  __syncthreads();
  if (few) {
    // ---- gather: keys whose decided top digits exceed the prefix (all chosen, any order)
    // and the <= 32 keys that share it, of which one warp keeps the `remaining` first in
    // the output order (larger key, then lower position)
    uint32_t* candk = hist;                                 // [32]
    int* candi = reinterpret_cast<int*>(hist + 32);         // [32]
    if (tid == 0) {
      ctl[3] = 0;
      ctl[4] = 0;
    }
    __syncthreads();
    for (int i = tid; i < P; i += kTopkThreads) {
      const uint32_t u = key_at(i);
      const uint32_t hb = u & pmask;
      if (u != 0u && hb > prefix) {
        const int slot = atomicAdd(&ctl[3], 1);
        ckey[slot] = u;
        cidx[slot] = i;
      } else if (u != 0u && hb == prefix) {
        const int slot = atomicAdd(&ctl[4], 1);
        candk[slot] = u;
        candi[slot] = i;
      }
    }
    __syncthreads();
    if (tid < 32) {
      const int nc = ctl[4], above = ctl[3];
      uint32_t kx = tid < nc ? candk[tid] : 0u;
      int ix = tid < nc ? candi[tid] : 0x7fffffff;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
        const bool desc = (tid & size) == 0;
#pragma unroll
        for (int st = size >> 1; st >= 1; st >>= 1) {
          const uint32_t ky = __shfl_xor_sync(0xffffffffu, kx, st);
          const int iy = __shfl_xor_sync(0xffffffffu, ix, st);
          const bool y_first = ky > kx || (ky == kx && iy < ix);
          if (((tid & st) == 0) == (desc == y_first)) {
            kx = ky;
            ix = iy;
          }
        }
      }
      if (tid < remaining) {
        ckey[above + tid] = kx;
        cidx[above + tid] = ix;
      }
      __syncwarp();
      if (tid == 0) ctl[3] = above + remaining;
    }
    __syncthreads();
  }
  // ---- gather: keys above thr in any order, then the `remaining` lowest positions with key thr
  if (!few && tid == 0) ctl[3] = 0;
  __syncthreads();
  const bool ties_all = take_all || eq_total == remaining;
  for (int i = few ? P : tid; i < P; i += kTopkThreads) {
    const uint32_t u = key_at(i);
    if (u != 0u && (take_all ? true : (u > thr || (ties_all && u == thr)))) {
      const int slot = atomicAdd(&ctl[3], 1);
      ckey[slot] = u;
      cidx[slot] = i;
    }
  }
  __syncthreads();
  if (!few && !ties_all) {  // ties at thr: the lowest positions, in position order
    int base = 0;
    const int above = ctl[3];
    for (int c0 = 0; c0 < P; c0 += kTopkThreads) {
      const int i = c0 + tid;
      const bool eq = i < P && key_at(i) == thr;
      int total = 0;
      const int rank = block_rank(eq, warp_cnt, &total);
      if (eq && base + rank < remaining) {
        ckey[above + base + rank] = thr;
        cidx[above + base + rank] = i;
      }
      base += total;
      if (base >= remaining) break;
    }
    if (tid == 0) ctl[3] = above + remaining;
    __syncthreads();
  }
  const int nsel = ctl[3];
  for (int i = nsel + tid; i < kp2; i += kTopkThreads) {
    ckey[i] = 0u;
    cidx[i] = 0x7fffffff;
  }
  __syncthreads();
  // ---- bitonic sort: key descending, then position ascending, on 64-bit values
  // (key << 32) | ~position (one unsigned comparison orders both) that take the place of
  // ckey / cidx.  Stages whose partner is 32 or more elements away go through shared
  // memory; the rest of each merge (strides 16 down to 1) runs in registers with warp
  // shuffles, one element per thread and slot.
  uint64_t* cv = reinterpret_cast<uint64_t*>(ckey);  // [kp2], over ckey and cidx
  {
    uint64_t pk[kTopkMaxK / kTopkThreads];
#pragma unroll
    for (int r = 0; r < kTopkMaxK / kTopkThreads; ++r) {
      const int i = tid + r * kTopkThreads;
      if (i < kp2) pk[r] = ((uint64_t)ckey[i] << 32) | (uint64_t)(~(uint32_t)cidx[i]);
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kTopkMaxK / kTopkThreads; ++r) {
      const int i = tid + r * kTopkThreads;
      if (i < kp2) cv[i] = pk[r];
    }
    __syncthreads();
  }
  for (int size = 2; size <= kp2; size <<= 1) {
    int stride = size >> 1;
    for (; stride >= 32; stride >>= 1) {
      for (int i = tid; i < kp2; i += kTopkThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;  // this block sorts "first before second" order
          const uint64_t vi = cv[i], vj = cv[j];
          if (desc == (vj > vi)) {
            cv[i] = vj;
            cv[j] = vi;
          }
        }
      }
      __syncthreads();
    }
#pragma unroll 1
    for (int i0 = 0; i0 < kp2; i0 += kTopkThreads) {  // whole warps: kp2 is a power of two
      const int i = i0 + tid;
      const bool active = i < kp2;
      uint64_t vx = active ? cv[i] : 0ull;
      const bool desc = (i & size) == 0;
      for (int st = stride; st >= 1; st >>= 1) {
        const uint64_t vy = __shfl_xor_sync(0xffffffffu, vx, st);
        const bool lower = (i & st) == 0;
        // the lower element of the pair keeps the one that comes first in this block's
        // order, the upper one the other
        if (lower == (desc == (vy > vx))) vx = vy;
      }
      if (active) cv[i] = vx;
    }
    __syncthreads();
  }
  int* out = idx + (long long)row * k;
  for (int i = tid; i < k; i += kTopkThreads) out[i] = (i < nsel) ? (int)(~(uint32_t)cv[i]) : -1;
}

}  // namespace attn_b200

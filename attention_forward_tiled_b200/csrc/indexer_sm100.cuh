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
// items (b, key tile, token tile) go to persistent CTAs (192 threads):
//   * warp 4, producer: TMA loads of the key tile (once per run of items on the same
//     tile) and of the query tiles into shared memory;
//   * warp 5, MMA issuer: S^T = Kp Q^T into one of two TMEM accumulators;
//   * warps 0-3, epilogue: rectify, weight, sum over heads, add the f16 mask and
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
  CUtensorMap tm_q;   // q [B, T, H, D] as 3-D (D, T*H, B), box (64, 128, 1), 128B swizzle
  CUtensorMap tm_k;   // kp [B, P, D] as 3-D (D, P, B), box (64, 128, 1), 128B swizzle
  const float* w;     // [B, T, H]
  const uint16_t* mask;  // [B, T, P] f16 (0 / -inf) or nullptr
  float* score;       // [B, T, P]
  int* status;
  int B, T, H, P;
  int lg_h;           // log2(H)
  int tok_per_tile;   // 128 / H
  int n_ttiles, n_ptiles, n_items;
  unsigned long long timeout_ns;
};

template <int D>
struct IndexerCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxBytes = 128 * 128;             // 128 rows x 64 elements x 2 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;   // 128 rows x D
  static constexpr int kQStages = 2;
  static constexpr int kOffK = 0;                                  // key tiles [2]
  static constexpr int kOffQ = 2 * kTileBytes;                     // query tiles [kQStages]
  static constexpr int kOffW = kOffQ + kQStages * kTileBytes;     // head weights [2][128] fp32
  static constexpr int kOffM = kOffW + 2 * 128 * 4;                // pool mask [2][128 tokens][128 keys] f16
  static constexpr int kOffBar = kOffM + 2 * 128 * 128 * 2;
  static constexpr int kBarKFull = 0;                     // [2]
  static constexpr int kBarKEmpty = 2;                    // [2]
  static constexpr int kBarQFull = 4;                     // [kQStages]
  static constexpr int kBarQEmpty = 4 + kQStages;         // [kQStages]
  static constexpr int kBarAccFull = 4 + 2 * kQStages;    // [2]
  static constexpr int kBarAccFree = 6 + 2 * kQStages;    // [2]
  static constexpr int kBarMmaDone = 8 + 2 * kQStages;    // [1]
  static constexpr int kNumBars = 9 + 2 * kQStages;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // +1024: manual 1 KB alignment
  static constexpr int kThreads = 192;
  static constexpr int kProducerWarp = 4;
  static constexpr int kMmaWarp = 5;
  static constexpr uint32_t kTmemCols = 256;  // two 128-column accumulators
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Item -> (b, key tile, token tile); the items of one key tile are consecutive, and
// each CTA takes a contiguous range of items, so it loads a key tile once for all
// the token tiles of that range.
struct IndexerItem {
  int b, pt, tt;
};

__device__ __forceinline__ IndexerItem indexer_item(const IndexerParams& p, int item) {
  IndexerItem it;
  it.tt = item % p.n_ttiles;
  const int bp = item / p.n_ttiles;
  it.pt = bp % p.n_ptiles;
  it.b = bp / p.n_ptiles;
  return it;
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
  // this CTA's items: a contiguous range, so consecutive items share a key tile
  const int item0 = blockIdx.x * items_per_cta;
  const int item1 = min(p.n_items, item0 + items_per_cta);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarKFull + i), 1);
      mbar_init(BAR(C::kBarKEmpty + i), 1);
      mbar_init(BAR(C::kBarAccFull + i), 1);
      mbar_init(BAR(C::kBarAccFree + i), 4);  // one arrive per epilogue warp
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

  // key tiles along the item range: the r-th distinct key tile goes to key buffer r & 1
  auto same_key_tile = [&](const IndexerItem& a, const IndexerItem& b) {
    return a.b == b.b && a.pt == b.pt;
  };

  if (warp == C::kProducerWarp) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&p.tm_q);
      tma_prefetch_map(&p.tm_k);
    }
    int nk = 0;  // key tiles loaded
    int g = 0;   // query tiles loaded
    IndexerItem prev{-1, -1, -1};
    for (int item = item0; item < item1; ++item, ++g) {
      const IndexerItem it = indexer_item(p, item);
      if (!same_key_tile(it, prev)) {
        const int kb = nk & 1;
        if (nk >= 2) mbar_wait(BAR(C::kBarKEmpty + kb), ((nk >> 1) - 1) & 1, wctx);
        __syncwarp();
        if (warp_flag(abort_flag)) break;
        mbar_arrive_expect_tx_w(BAR(C::kBarKFull + kb), C::kTileBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d_w(sbase + C::kOffK + kb * C::kTileBytes + bx * C::kBoxBytes, &p.tm_k,
                        BAR(C::kBarKFull + kb), bx * 64, it.pt * 128, it.b);
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
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this warp started land before the CTA can exit
      for (int i = max(0, g - C::kQStages); i < g; ++i)
        mbar_wait_drain(BAR(C::kBarQFull + i % C::kQStages), (i / C::kQStages) & 1, p.timeout_ns);
      for (int i = max(0, nk - 2); i < nk; ++i)
        mbar_wait_drain(BAR(C::kBarKFull + (i & 1)), (i >> 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer =======================
    constexpr uint32_t idesc = make_idesc_f16(128, 128, BF16, false);  // Kp Q^T, both K-major
    int nk = 0, g = 0;
    IndexerItem prev{-1, -1, -1};
    for (int item = item0; item < item1; ++item, ++g) {
      const IndexerItem it = indexer_item(p, item);
      const bool new_key = !same_key_tile(it, prev);
      if (new_key) {
        if (nk > 0) tc_commit_w(BAR(C::kBarKEmpty + ((nk - 1) & 1)));  // previous key tile released
        mbar_wait(BAR(C::kBarKFull + (nk & 1)), (nk >> 1) & 1, wctx);
        ++nk;
        prev = it;
      }
      const int st = g % C::kQStages;
      const int ab = g & 1;
      mbar_wait(BAR(C::kBarQFull + st), (g / C::kQStages) & 1, wctx);
      if (g >= 2) mbar_wait(BAR(C::kBarAccFree + ab), ((g >> 1) - 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
        const uint32_t sK = sbase + C::kOffK + ((nk - 1) & 1) * C::kTileBytes;
        const uint32_t sQ = sbase + C::kOffQ + st * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // 16 head-dim elements per k-step
          const uint32_t off = (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          mma_f16_ss_w(tmem + ab * 128u, make_sdesc_sw128(sK + off, 16, 1024),
                       make_sdesc_sw128(sQ + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit_w(BAR(C::kBarAccFull + ab));
        tc_commit_w(BAR(C::kBarQEmpty + st));
      }
    }
    if (nk > 0) tc_commit_w(BAR(C::kBarKEmpty + ((nk - 1) & 1)));
    // every MMA (and every commit arrive) has landed before TMEM is released
    tc_commit_w(BAR(C::kBarMmaDone));
    mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    __syncwarp();
  } else {
    // ======================= epilogue warps 0-3 (thread = pooled key) ===========
    // The head weights and pool mask of item g + 1 are loaded into shared memory while item
    // g's product runs (plain loads: the mask rows of arbitrary length P need not meet any
    // copy-engine alignment), so no global load sits between the score stores.
    const int r = threadIdx.x;  // key of the tile
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int lg_h = p.lg_h, tpt = p.tok_per_tile;
    float* wbuf = reinterpret_cast<float*>(smem + C::kOffW);        // [2][128]
    uint16_t* mbuf = reinterpret_cast<uint16_t*>(smem + C::kOffM);  // [2][128][128]
    auto prefetch = [&](int item, int buf) {
      const IndexerItem it = indexer_item(p, item);
      const int t0 = it.tt * tpt;
      const long long row_bt = (long long)it.b * p.T;
      {  // weight of column r: w[b, t0 + r / H, r % H]
        const int t = t0 + (r >> lg_h);
        wbuf[buf * 128 + r] = t < p.T ? __ldg(p.w + (row_bt + t0) * (1 << lg_h) + r) : 0.f;
      }
      if (p.mask != nullptr) {
        const int key = it.pt * 128 + r;
        uint16_t* mb = mbuf + buf * 128 * 128 + r;
        for (int c0 = 0; c0 < tpt; c0 += 32) {  // 32 independent loads in flight, then the stores
          uint16_t v[32];
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int t = t0 + c0 + u;
            v[u] = (c0 + u < tpt && t < p.T && key < p.P) ? __ldg(p.mask + (row_bt + t) * p.P + key) : 0;
          }
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if (c0 + u < tpt) mb[(c0 + u) * 128] = v[u];
        }
      }
    };
    if (item0 < item1) prefetch(item0, 0);
    named_bar_sync(1, 128);
    int g = 0;
    for (int item = item0; item < item1; ++item, ++g) {
      const IndexerItem it = indexer_item(p, item);
      const int ab = g & 1;
      if (item + 1 < item1) prefetch(item + 1, ab ^ 1);
      const int t0 = it.tt * tpt;
      const long long row_bt = (long long)it.b * p.T;
      mbar_wait(BAR(C::kBarAccFull + ab), (g >> 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      const int key = it.pt * 128 + r;
      const float* wb = wbuf + ab * 128;
      const uint16_t* mb = mbuf + ab * 128 * 128 + r;
      float acc = 0.f;
      // 32 columns at a time: column c = t_local * H + h
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t s[32];
        tmem_ld32(tmem + lane_base + ab * 128u + c0, s);
        tmem_ld_wait();
        reg_order_after_wait(s);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int col = c0 + c;
          acc = fmaf(wb[col], fmaxf(__uint_as_float(s[c]), 0.f), acc);
          if (((col + 1) & ((1 << lg_h) - 1)) == 0) {  // last head of a token: its score is complete
            const int tl = col >> lg_h;
            const int t = t0 + tl;
            if (t < p.T && key < p.P) {
              float v = acc;
              if (p.mask != nullptr) v += __half2float(__ushort_as_half(mb[tl * 128]));
              p.score[(row_bt + t) * p.P + key] = v;
            }
            acc = 0.f;
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::kBarAccFree + ab));
      // every thread is done with buffer ab, and buffer ab ^ 1 is complete, before the next
      // item reads ab ^ 1 and prefetches into ab
      named_bar_sync(1, 128);
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
    for (int i = tid; i < P; i += kTopkThreads) rowkeys[i] = topk_key(__ldg(srow + i));
  }
  // ---- radix select of the k-th largest key, 8 bits at a time from the top
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;   // entries still to choose among those matching the prefix
  bool take_all = false;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < P; i0 += kTopkThreads) {  // uniform trip count: whole warps vote
      const int i = i0 + tid;
      const uint32_t u = i < P ? key_at(i) : 0u;
      const bool hit = u != 0u && (u & pmask) == prefix;
      const uint32_t bin = hit ? (u >> shift) & 255u : 256u;
      // one atomic per distinct digit of the warp: most scores share the top digits
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (hit && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
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
  }
  const uint32_t thr = prefix;  // the k-th largest key (unless take_all)
  const int eq_total = ctl[2];   // entries equal to thr (last pass)
  __syncthreads();
  // ---- gather: keys above thr in any order, then the `remaining` lowest positions with key thr
  if (tid == 0) ctl[3] = 0;
  __syncthreads();
  const bool ties_all = take_all || eq_total == remaining;
  for (int i = tid; i < P; i += kTopkThreads) {
    const uint32_t u = key_at(i);
    if (u != 0u && (take_all ? true : (u > thr || (ties_all && u == thr)))) {
      const int slot = atomicAdd(&ctl[3], 1);
      ckey[slot] = u;
      cidx[slot] = i;
    }
  }
  __syncthreads();
  if (!ties_all) {  // ties at thr: the lowest positions, in position order
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
  // ---- bitonic sort: key descending, then position ascending
  for (int size = 2; size <= kp2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < kp2; i += kTopkThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;  // this block sorts "first before second" order
          const uint32_t ki = ckey[i], kj = ckey[j];
          const int ii = cidx[i], ij = cidx[j];
          const bool j_first = kj > ki || (kj == ki && ij < ii);
          if (desc == j_first) {
            ckey[i] = kj;
            ckey[j] = ki;
            cidx[i] = ij;
            cidx[j] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
  int* out = idx + (long long)row * k;
  for (int i = tid; i < k; i += kTopkThreads) out[i] = (i < nsel) ? cidx[i] : -1;
}

}  // namespace attn_b200

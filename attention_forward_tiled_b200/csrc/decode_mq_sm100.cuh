// decode_mq_sm100.cuh -- a few query tokens per request against a paged key/value
// cache, on the tensor cores (sm_100a).
//
// The step the vLLM MiniMax-M3 indexer page describes for speculative decoding
// ("PR #45743 完整报告", section "功能与动机": the query tokens of one request are
// scored together; section "关键源码片段": per-request seq_lens and a block table):
// request b's Lq query tokens are the last Lq positions of its sequence of
// seq_lens[b] cached keys, and each token attends to the cached keys with the same
// online softmax as the tiled forward (FlashAttention/ops-transformer article,
// section "FlashAttention的核心逻辑").
//
// Every head has its own keys and values, so one (b, h) brings only Lq <= 16 query
// rows: too few for the M = 128 rows of a tcgen05.mma.  The tile is therefore
// transposed: the 128 keys of a K/V tile are the M rows and the queries are N = 16:
//   S^T = K Q^T     A = K tile (shared memory, K-major), B = Q (shared memory, K-major),
//                   D = S^T in TMEM: lane = key, column = query;
//   O^T += V^T P^T  A = V tile read MN-major (shared memory), B = P^T (shared memory,
//                   K-major: one row of 128 keys per query), D = O^T in TMEM:
//                   lane = head-dim element, column = query.
// The step stays bound by the HBM read of K and V (each element is used by Lq
// queries); the tensor cores keep the arithmetic off the critical path.
//
// Work items (b, h, key split) go round-robin to persistent CTAs (192 threads):
//   * warp 4, producer: loads Q once per item (TMA, rows past Lq read as zeros) and
//     streams 128-key K and V tiles page by page into a ring of shared-memory stages,
//     one lane per page piece;
//   * warp 5, MMA issuer: S^T of tile i, then O^T of tile i-1, so the softmax of one
//     tile overlaps the next tile's score product;
//   * warps 0-3, softmax: one thread per key of the tile; masks keys past the
//     sequence and, under the causal flag, keys after a query's position; the
//     per-query maximum over the 128 keys is reduced across the four warps through
//     shared memory; lazy rescale of O^T (only when a query's maximum grows by more
//     than 2^8); P^T is written to shared memory in fp16, and each thread keeps
//     per-query partial sums of the rounded P, reduced once per item.  For bf16 inputs
//     each thread first converts its key's row of the V tile to fp16 in place, so the
//     O^T product runs in fp16 as the tiled forward's does (bf16's 8-bit P would miss the
//     output bound for short sequences); a V magnitude with no fp16 value records the
//     range status.
// Each item yields per-query partials (o unnormalised, m in base-2 units, l), merged
// over the key splits by attn_mq_combine_kernel.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

constexpr int kMqMaxQ = 16;  // query tokens per request: the MMA's N

struct MqParams {
  CUtensorMap tm_q;  // q [B, Lq, H, D] as 4-D (D, H, Lq, B), box (64, 1, 16, 1), 128B swizzle
  CUtensorMap tm_k;  // k cache [num_blocks * page_size, H, D] as (D, H, rows, 1), box (64, 1, page_rows, 1)
  CUtensorMap tm_v;  // v cache, same
  float* part;       // [B*H*splits][Lq][D + 2]: o[0..D) unnormalised, m (base-2 units), l
  int* status;
  int B, H, Lq;
  int Nk;            // max_blocks * page_size: the longest sequence the table holds
  int causal;
  int splits, tiles_per_split, n_items;
  float scale_log2;  // scale * log2(e)
  unsigned long long timeout_ns;
  const int* block_table;  // [B, max_blocks]
  const int* seq_lens;     // [B]
  int max_blocks, page_size, page_rows, num_blocks;
};

template <int D>
struct MqCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxBytes = 128 * 128;             // 128 rows x 64 elements x 2 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;   // 128 keys x D
  static constexpr int kStageBytes = 2 * kTileBytes;      // K tile + V tile
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kQBoxBytes = kMqMaxQ * 128;        // 16 rows x 64 elements x 2 bytes
  static constexpr int kQBytes = kBoxes * kQBoxBytes;     // 16 query rows x D
  static constexpr int kPBytes = 2 * kQBoxBytes;          // 16 query rows x 128 keys
  static constexpr int kOffQ = kStages * kStageBytes;     // Q_0, Q_1
  static constexpr int kOffP = kOffQ + 2 * kQBytes;       // P_0, P_1 (P^T of tiles by parity)
  static constexpr int kOffRed = kOffP + 2 * kPBytes;     // float red[2][4][16], redl[4][16]
  static constexpr int kRedBytes = (2 * 4 + 4) * kMqMaxQ * 4;
  static constexpr int kOffBar = kOffRed + kRedBytes;
  static constexpr int kBarFull = 0;                      // [kStages]
  static constexpr int kBarEmpty = kStages;               // [kStages]
  static constexpr int kBarQFull = 2 * kStages;           // [2]
  static constexpr int kBarQEmpty = kBarQFull + 2;        // [2]
  static constexpr int kBarSFull = kBarQEmpty + 2;        // [2]
  static constexpr int kBarSFree = kBarSFull + 2;         // [2]
  static constexpr int kBarPFull = kBarSFree + 2;         // [2]
  static constexpr int kBarPFree = kBarPFull + 2;         // [2] the O^T product reading P_b is done
  static constexpr int kBarMmaDone = kBarPFree + 2;       // [1]
  static constexpr int kNumBars = kBarMmaDone + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // +1024: manual 1 KB alignment
  static constexpr int kThreads = 192;
  static constexpr int kProducerWarp = 4;
  static constexpr int kMmaWarp = 5;
  static constexpr uint32_t kTmemCols = 64;  // S_0 [0,16), S_1 [16,32), O [32,48)
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0 && kQBytes % 1024 == 0, "swizzle atoms");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Item -> (b, h, first and one-past-last 128-key tile, keys of the request).
struct MqItem {
  int b, h, t0, t1, seq_len;
};

__device__ __forceinline__ MqItem mq_item(const MqParams& p, int item) {
  MqItem it;
  const int bh = item / p.splits;
  const int sp = item - bh * p.splits;
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  it.seq_len = min(max(__ldg(p.seq_lens + it.b), 0), p.Nk);
  it.t0 = sp * p.tiles_per_split;
  it.t1 = min((it.seq_len + 127) / 128, it.t0 + p.tiles_per_split);
  if (it.t1 < it.t0) it.t1 = it.t0;
  return it;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(MqCfg<D>::kThreads, 1)
    attn_mq_partial_kernel(const __grid_constant__ MqParams p) {
  using C = MqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);                   // [2][4][16]
  float* redl = reinterpret_cast<float*>(smem + C::kOffRed + 2 * 4 * kMqMaxQ * 4);  // [4][16]
  auto BAR = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(BAR(C::kBarFull + s), 1);
      mbar_init(BAR(C::kBarEmpty + s), 1);  // the O^T product's commit: K and V both consumed
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarQFull + i), 1);
      mbar_init(BAR(C::kBarQEmpty + i), 1);
      mbar_init(BAR(C::kBarSFull + i), 1);
      mbar_init(BAR(C::kBarSFree + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarPFull + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarPFree + i), 1);
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

  if (warp == C::kProducerWarp) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      tma_prefetch_map(&p.tm_q);
      tma_prefetch_map(&p.tm_k);
      tma_prefetch_map(&p.tm_v);
    }
    int g = 0;   // ring position (global tile count of this CTA)
    int nq = 0;  // Q loads (items with at least one tile)
    bool q_pending[2] = {false, false};
    bool stop = false;
    for (int item = blockIdx.x; item < p.n_items && !stop; item += gridDim.x) {
      const MqItem it = mq_item(p, item);
      if (it.t1 == it.t0) continue;
      const int qb = nq & 1;
      if (nq >= 2) mbar_wait(BAR(C::kBarQEmpty + qb), ((nq >> 1) - 1) & 1, wctx);
      __syncwarp();
      if (warp_flag(abort_flag)) break;
      mbar_arrive_expect_tx_w(BAR(C::kBarQFull + qb), C::kQBytes);
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_4d_w(sbase + C::kOffQ + qb * C::kQBytes + bx * C::kQBoxBytes, &p.tm_q,
                      BAR(C::kBarQFull + qb), bx * 64, it.h, 0, it.b);
      q_pending[qb] = true;
      ++nq;
      for (int tile = it.t0; tile < it.t1; ++tile, ++g) {
        const int stage = g % C::kStages;
        const int round = g / C::kStages;
        if (round > 0) mbar_wait(BAR(C::kBarEmpty + stage), (round - 1) & 1, wctx);
        __syncwarp();
        if (warp_flag(abort_flag)) {
          stop = true;
          break;
        }
        const uint32_t dst = sbase + stage * C::kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(BAR(C::kBarFull + stage), C::kStageBytes);
        __syncwarp();
        // piece `lane` holds keys [key, key + page_rows) of one page; it lands at a multiple
        // of 8 rows, where the 128-byte swizzle pattern restarts
        if (lane < 128 / p.page_rows) {
          const int key = tile * 128 + lane * p.page_rows;
          const int page = key / p.page_size;
          // table entries outside [0, num_blocks) are clamped: every read stays in the cache
          const int phys = key < it.seq_len
                               ? min(max(__ldg(p.block_table + (long long)it.b * p.max_blocks + page), 0),
                                     p.num_blocks - 1)
                               : 0;
          const int row = phys * p.page_size + (key - page * p.page_size);
          const uint32_t off = (uint32_t)(lane * p.page_rows) * 128;
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            tma_load_4d(dst + bx * C::kBoxBytes + off, &p.tm_k, BAR(C::kBarFull + stage), bx * 64, it.h,
                        row, 0);
            tma_load_4d(dst + C::kTileBytes + bx * C::kBoxBytes + off, &p.tm_v, BAR(C::kBarFull + stage),
                        bx * 64, it.h, row, 0);
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this warp started land before the CTA can exit
      const int first = g > C::kStages ? g - C::kStages : 0;
      for (int i = first; i < g; ++i)
        mbar_wait_drain(BAR(C::kBarFull + i % C::kStages), (i / C::kStages) & 1, p.timeout_ns);
      for (int b = 0; b < 2; ++b) {
        const int n_b = (nq + 1 - b) / 2;  // Q loads issued into buffer b
        if (q_pending[b] && n_b > 0) mbar_wait_drain(BAR(C::kBarQFull + b), (n_b - 1) & 1, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer (one elected lane issues) ===========
    constexpr uint32_t idesc_s = make_idesc_f16(128, kMqMaxQ, BF16, false, false);  // K Q^T
    // V^T P^T always in fp16 (bf16 V tiles are converted in shared memory first)
    constexpr uint32_t idesc_o = make_idesc_f16(128, kMqMaxQ, false, false, true);
    // d = 64: M = 128 reads the 64 head-dim elements twice (lanes 64..127 of O^T unused)
    constexpr uint32_t kLboV = (D == 128) ? C::kBoxBytes : 0;
    const uint32_t colS[2] = {0u, 16u};
    const uint32_t colO = 32u;
    auto issue_o = [&](int gt, bool first) {
      mbar_wait(BAR(C::kBarPFull + (gt & 1)), (gt >> 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (warp_flag(abort_flag)) return;
      const uint32_t sV = sbase + (gt % C::kStages) * C::kStageBytes + C::kTileBytes;
      const uint32_t sP = sbase + C::kOffP + (gt & 1) * C::kPBytes;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // 16 keys per k-step
        const uint64_t a = make_sdesc_sw128(sV + kk * 2048, kLboV, 1024);
        const uint64_t b = make_sdesc_sw128(sP + (kk >> 2) * C::kQBoxBytes + (kk & 3) * 32, 16, 1024);
        mma_f16_ss_w(tmem + colO, a, b, idesc_o, (first && kk == 0) ? 0u : 1u);
      }
      tc_commit_w(BAR(C::kBarPFree + (gt & 1)));
      tc_commit_w(BAR(C::kBarEmpty + gt % C::kStages));
    };
    int g = 0, nq = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const MqItem it = mq_item(p, item);
      const int ntile = it.t1 - it.t0;
      if (ntile == 0) continue;
      const int qb = nq & 1;
      mbar_wait(BAR(C::kBarQFull + qb), (nq >> 1) & 1, wctx);
      const uint32_t sQ = sbase + C::kOffQ + qb * C::kQBytes;
      for (int i = 0; i < ntile; ++i) {
        const int gt = g + i;
        const int stage = gt % C::kStages;
        mbar_wait(BAR(C::kBarFull + stage), (gt / C::kStages) & 1, wctx);
        if (gt >= 2) mbar_wait(BAR(C::kBarSFree + (gt & 1)), ((gt - 2) >> 1) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        if (!warp_flag(abort_flag)) {
          const uint32_t sK = sbase + stage * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // 16 head-dim elements per k-step
            const uint64_t a = make_sdesc_sw128(sK + (kk >> 2) * C::kBoxBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t b = make_sdesc_sw128(sQ + (kk >> 2) * C::kQBoxBytes + (kk & 3) * 32, 16, 1024);
            mma_f16_ss_w(tmem + colS[gt & 1], a, b, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit_w(BAR(C::kBarSFull + (gt & 1)));
          if (i == ntile - 1) tc_commit_w(BAR(C::kBarQEmpty + qb));
        }
        if (i >= 1) issue_o(gt - 1, i == 1);
      }
      issue_o(g + ntile - 1, ntile == 1);
      g += ntile;
      ++nq;
    }
    // every MMA (and every commit arrive) has landed before TMEM is released
    tc_commit_w(BAR(C::kBarMmaDone));
    mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    __syncwarp();
  } else {
    // ======================= softmax warps 0-3 (thread = key of the tile) ===========
    const int t = threadIdx.x;  // 0..127: key of the tile; head-dim element of O^T
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tS[2] = {tmem + lane_base, tmem + lane_base + 16u};
    const uint32_t tO = tmem + lane_base + 32u;
    const float cs = p.scale_log2;
    const int Lq = p.Lq;
    uint32_t vmag = 0;  // bf16: per-halfword max of |bits| over the V elements this thread converted
    int g = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const MqItem it = mq_item(p, item);
      const int ntile = it.t1 - it.t0;
      float m[kMqMaxQ], lp[kMqMaxQ];
#pragma unroll
      for (int q = 0; q < kMqMaxQ; ++q) {
        m[q] = -INFINITY;
        lp[q] = 0.f;
      }
      for (int i = 0; i < ntile; ++i) {
        const int gt = g + i;
        mbar_wait(BAR(C::kBarSFull + (gt & 1)), (gt >> 1) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        uint32_t sr[16];
        tmem_ld16(tS[gt & 1], sr);
        tmem_ld_wait();
        reg_order_after_wait(sr);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarSFree + (gt & 1)));

        // scores in base-2 units, -inf where the key is not allowed for the query
        const int key = (it.t0 + i) * 128 + t;
        float x[kMqMaxQ];
#pragma unroll
        for (int q = 0; q < kMqMaxQ; ++q) {
          const bool allowed = q < Lq && key < it.seq_len &&
                               (!p.causal || key + Lq - q <= it.seq_len);
          x[q] = allowed ? __uint_as_float(sr[q]) * cs : -INFINITY;
        }
        // per-query maximum over the tile's 128 keys: warp shuffles, then the four warps
        float* rb = red + (gt & 1) * 4 * kMqMaxQ;
#pragma unroll
        for (int q = 0; q < kMqMaxQ; ++q) {
          if (q >= Lq) break;
          float v = x[q];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == q) rb[warp * kMqMaxQ + q] = v;
        }
        named_bar_sync(1, 128);
        float alpha[kMqMaxQ], m_use[kMqMaxQ];
        bool any_rescale = false;
#pragma unroll
        for (int q = 0; q < kMqMaxQ; ++q) {
          float mt = -INFINITY;
          if (q < Lq)
            mt = fmaxf(fmaxf(rb[q], rb[kMqMaxQ + q]), fmaxf(rb[2 * kMqMaxQ + q], rb[3 * kMqMaxQ + q]));
          const float m_new = fmaxf(m[q], mt);
          const bool rescale = m_new > m[q] + 8.0f;  // lazy: only when the maximum grows by > 2^8
          alpha[q] = rescale ? ex2_approx(m[q] - m_new) : 1.0f;
          if (rescale) {
            m[q] = m_new;
            lp[q] *= alpha[q];
          }
          any_rescale |= rescale;
          m_use[q] = (m[q] == -INFINITY) ? 0.f : m[q];
        }
        // O^T holds earlier tiles of this item: scale its query columns (lane = head-dim
        // element) once the product of the previous tile has landed
        if (any_rescale && i > 0) {  // uniform: every thread holds the same m
          mbar_wait(BAR(C::kBarPFree + ((gt - 1) & 1)), ((gt - 1) >> 1) & 1, wctx);
          __syncwarp();
          tc_fence_after_sync();
          uint32_t o[16];
          tmem_ld16(tO, o);
          tmem_ld_wait();
          reg_order_after_wait(o);
#pragma unroll
          for (int q = 0; q < kMqMaxQ; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
          tmem_st16(tO, o);
          tmem_st_wait();
        }
        if constexpr (BF16) {
          // this key's row of the V tile to fp16, in place (the stage's copies have landed:
          // its full barrier cannot move on before this tile's product has read it)
          mbar_wait(BAR(C::kBarFull + gt % C::kStages), (gt / C::kStages) & 1, wctx);
          __syncwarp();
          uint8_t* vrow = smem + (gt % C::kStages) * C::kStageBytes + C::kTileBytes + t * 128;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            uint4* w4 = reinterpret_cast<uint4*>(vrow + bx * C::kBoxBytes);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 w = w4[c];
              if (key < it.seq_len)  // rows past the sequence hold another page's keys
                vmag = __vmaxu2(vmag, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                               __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
              w.x = bf16x2_to_f16x2_sat(w.x);
              w.y = bf16x2_to_f16x2_sat(w.y);
              w.z = bf16x2_to_f16x2_sat(w.z);
              w.w = bf16x2_to_f16x2_sat(w.w);
              w4[c] = w;
            }
          }
        }
        // P^T of this tile into P_(gt&1), once the product that read it two tiles ago is done
        if (gt >= 2) mbar_wait(BAR(C::kBarPFree + (gt & 1)), ((gt - 2) >> 1) & 1, wctx);
        __syncwarp();
        uint8_t* pb = smem + C::kOffP + (gt & 1) * C::kPBytes + (t >> 6) * C::kQBoxBytes + (t & 7) * 2;
        const int chunk = (t & 63) >> 3;
#pragma unroll
        for (int q = 0; q < kMqMaxQ; ++q) {
          const float pv = (x[q] == -INFINITY) ? 0.f : ex2_approx(x[q] - m_use[q]);
          const __half r = __float2half_rn(pv);
          const uint16_t hv = *reinterpret_cast<const uint16_t*>(&r);
          lp[q] += __half2float(r);
          *reinterpret_cast<uint16_t*>(pb + q * 128 + ((chunk ^ (q & 7)) << 4)) = hv;
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarPFull + (gt & 1)));
      }

      // ---- end of the item: O^T of the last product, l reduced over the 128 keys
      uint32_t o[16];
#pragma unroll
      for (int q = 0; q < kMqMaxQ; ++q) o[q] = 0u;
      if (ntile > 0) {
        const int gl = g + ntile - 1;
        mbar_wait(BAR(C::kBarPFree + (gl & 1)), (gl >> 1) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        tmem_ld16(tO, o);
        tmem_ld_wait();
        reg_order_after_wait(o);
        tc_fence_before_sync();
      }
#pragma unroll
      for (int q = 0; q < kMqMaxQ; ++q) {
        if (q >= Lq) break;
        float v = lp[q];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == q) redl[warp * kMqMaxQ + q] = v;
      }
      named_bar_sync(1, 128);
      float* dst = p.part + (long long)item * Lq * (D + 2);
#pragma unroll
      for (int q = 0; q < kMqMaxQ; ++q) {
        if (q >= Lq) break;
        if (t < D) dst[q * (D + 2) + t] = __uint_as_float(o[q]);
        if (t == 0) {
          dst[q * (D + 2) + D] = m[q];
          dst[q * (D + 2) + D + 1] =
              (redl[q] + redl[kMqMaxQ + q]) + (redl[2 * kMqMaxQ + q] + redl[3 * kMqMaxQ + q]);
        }
      }
      named_bar_sync(1, 128);  // redl is read before the next item writes it
      g += ntile;
    }
    if constexpr (BF16) {
      if (max(vmag & 0xFFFFu, vmag >> 16) >= kBf16NoF16) atomicCAS(p.status, 0, kStatusRange);
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

// Merge the per-split partials of each (b, h, query) row: M = max_s m_s,
// w_s = 2^(m_s - M), O = sum_s w_s o_s / sum_s w_s l_s, lse = (M + log2 sum_s w_s l_s) ln 2.
// One warp per row; out [B, Lq, H, D], lse [B, H, Lq].
template <int D, bool BF16>
__global__ void __launch_bounds__(128)
    attn_mq_combine_kernel(const float* __restrict__ part, void* __restrict__ out,
                           float* __restrict__ lse, int B, int H, int Lq, int splits) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 4 + warp;  // (b * H + h) * Lq + q
  if (row >= (long long)B * H * Lq) return;
  const long long bh = row / Lq;
  const int q = (int)(row - bh * Lq);
  const int b = (int)(bh / H), h = (int)(bh - (long long)b * H);
  auto ps = [&](int s) { return part + ((bh * splits + s) * Lq + q) * (D + 2); };
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ps(s)[D]);
  float L = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* pp = ps(s);
    const float ms = pp[D];
    const float w = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
    L = fmaf(w, pp[D + 1], L);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(w, pp[E * lane + e], acc[e]);
  }
  const float inv = L > 0.f ? 1.0f / L : 0.f;
  uint8_t* orow = static_cast<uint8_t*>(out) + ((((long long)b * Lq + q) * H + h) * D) * 2;
  if constexpr (E == 4) {
    uint2 w;
    w.x = pack2<BF16>(acc[0] * inv, acc[1] * inv);
    w.y = pack2<BF16>(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(orow + E * lane * 2) = w;
  } else {
    *reinterpret_cast<uint32_t*>(orow + E * lane * 2) = pack2<BF16>(acc[0] * inv, acc[1] * inv);
  }
  if (lse != nullptr && lane == 0) lse[row] = L > 0.f ? (M + lg2_approx(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn_b200

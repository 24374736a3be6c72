// decode_sm100.cuh -- single-query (Nq == 1) attention forward, split over keys.
//
// With one query row there is no matrix multiply to feed the tensor cores: the
// step reads every cached key and value once and does one multiply-add per
// element, so it is bound by HBM bandwidth.  The keys of each (b, h) row are cut
// into `splits` ranges; each range yields a partial (o unnormalised, m, l) with
// the same online-softmax recurrence as the tiled kernel (FlashAttention/
// ops-transformer article, section "FlashAttention的核心逻辑"), and a second
// kernel merges the partials of a row by their log-sum-exp.
//
// Partial kernel: persistent CTAs (one per SM) walk work items (b, h, split)
// round-robin.  Warp 4 streams 128-key K and V tiles into a 3-stage (d=128) or
// 6-stage (d=64) shared-memory ring with TMA, running ahead across item
// boundaries; warps 0-3 each take 32 keys of a tile (one key per lane, reading
// its row from the 128-byte-swizzled tile without bank conflicts), keep a
// per-warp running (m, l, o), and fold the four warps together at the end of
// each item.
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

struct DecodeParams {
  CUtensorMap tm_k;  // [B, Nk, H, D] as 4-D (D, H, Nk, B), box (64, 1, 128, 1), 128B swizzle;
  CUtensorMap tm_v;  // paged: the cache [num_blocks * page_size, H, D], box (64, 1, page_rows, 1)
  const void* q;     // [B, 1, H, D]
  float* part;       // [B*H*splits][D + 2]: o[0..D) unnormalised, m (base-2 units), l
  int* status;
  int B, H, Nk;          // paged: Nk = max_blocks * page_size, the longest sequence the table holds
  int splits;            // key ranges per (b, h)
  int tiles_per_split;   // 128-key tiles per range
  int n_items;           // B * H * splits
  float scale_log2;      // scale * log2(e)
  unsigned long long timeout_ns;
  // paged key/value cache (kPaged kernels only)
  const int* block_table;  // [B, max_blocks]: page of the request's keys [i*page_size, (i+1)*page_size)
  const int* seq_lens;     // [B]: keys of each request
  int max_blocks, page_size, page_rows, num_blocks;  // page_rows = min(page_size, 128)
};

// Keys of request b the kernel reads: seq_lens[b] clamped to what its table can hold
// (Nk = max_blocks * page_size), or Nk for a dense cache.
template <bool kPaged>
__device__ __forceinline__ int decode_seq_len(const DecodeParams& p, int b) {
  if constexpr (kPaged) return min(max(__ldg(p.seq_lens + b), 0), p.Nk);
  return p.Nk;
}

template <int D>
struct DecodeCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 keys x D x 2 bytes
  static constexpr int kStageBytes = 2 * kTileBytes;     // K tile + V tile
  static constexpr int kStages = (D == 128) ? 3 : 6;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kOffScratch = kOffBar + 256;
  static constexpr int kScratchBytes = 4 * (D + 2) * 4;
  static constexpr int kSmemBytes = kOffScratch + kScratchBytes + 1024;
  static constexpr int kThreads = 160;
  static constexpr int kProducerWarp = 4;
  static constexpr int kElemsPerLane = D / 32;
  static_assert(2 * kStages * 8 + 8 <= 256, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D, bool BF16, bool kPaged = false>
__global__ void __launch_bounds__(DecodeCfg<D>::kThreads, 1)
    attn_decode_partial_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 2 * C::kStages * 8);
  float* scratch = reinterpret_cast<float*>(smem + C::kOffScratch);  // [4][D + 2]
  auto FULL = [&](int s) -> uint32_t { return smem_u32(&bars[s]); };
  auto EMPTY = [&](int s) -> uint32_t { return smem_u32(&bars[C::kStages + s]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = (p.Nk + 127) / 128;
  const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 4);  // one arrive per consumer warp
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == C::kProducerWarp) {
    // ======================= TMA producer =======================
    // The whole warp walks the ring; lane 0 waits, arms the stage and issues dense tiles.
    // A paged tile comes in 128 / page_rows pieces, one lane per piece, so the pieces'
    // block-table reads overlap instead of following one another.
    if (lane == 0) {
      tma_prefetch_map(&p.tm_k);
      tma_prefetch_map(&p.tm_v);
    }
    int g = 0;  // ring position across all items of this CTA
    bool stop = false;
    for (int item = blockIdx.x; item < p.n_items && !stop; item += gridDim.x) {
      const int bh = item / p.splits;
      const int sp = item - bh * p.splits;
      const int b = bh / p.H, h = bh - b * p.H;
      const int seq_len = decode_seq_len<kPaged>(p, b);
      const int t0 = sp * p.tiles_per_split;
      const int t1 = min(min(ntiles, (seq_len + 127) / 128), t0 + p.tiles_per_split);
      for (int tile = t0; tile < t1; ++tile, ++g) {
        const int stage = g % C::kStages;
        const int round = g / C::kStages;
        if (round > 0) mbar_wait(EMPTY(stage), (round - 1) & 1, wctx);
        __syncwarp();
        if (warp_flag(abort_flag)) {
          stop = true;
          break;
        }
        const uint32_t dst = sbase + stage * C::kStageBytes;
        if (lane == 0) mbar_arrive_expect_tx(FULL(stage), C::kStageBytes);
        __syncwarp();
        if constexpr (kPaged) {
          // piece `lane` holds keys [key, key + page_rows) of one page; it lands at a multiple
          // of 8 rows, where the 128-byte swizzle pattern restarts
          if (lane < 128 / p.page_rows) {
            const int key = tile * 128 + lane * p.page_rows;
            const int page = key / p.page_size;
            // table entries outside [0, num_blocks) are clamped: every read stays in the cache
            const int phys = key < seq_len
                                 ? min(max(__ldg(p.block_table + (long long)b * p.max_blocks + page), 0),
                                       p.num_blocks - 1)
                                 : 0;
            const int row = phys * p.page_size + (key - page * p.page_size);
            const uint32_t off = (uint32_t)(lane * p.page_rows) * 128;
            for (int bx = 0; bx < C::kBoxes; ++bx) {
              tma_load_4d(dst + bx * C::kBoxBytes + off, &p.tm_k, FULL(stage), bx * 64, h, row, 0);
              tma_load_4d(dst + C::kTileBytes + bx * C::kBoxBytes + off, &p.tm_v, FULL(stage),
                          bx * 64, h, row, 0);
            }
          }
        } else if (lane == 0) {
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            tma_load_4d(dst + bx * C::kBoxBytes, &p.tm_k, FULL(stage), bx * 64, h, tile * 128, b);
            tma_load_4d(dst + C::kTileBytes + bx * C::kBoxBytes, &p.tm_v, FULL(stage), bx * 64, h,
                        tile * 128, b);
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0 && *abort_flag) {
      const int first = g > C::kStages ? g - C::kStages : 0;
      for (int i = first; i < g; ++i)
        mbar_wait_drain(FULL(i % C::kStages), (i / C::kStages) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ======================= consumer warps 0-3 =======================
    constexpr int E = C::kElemsPerLane;
    const int r = warp * 32 + lane;  // key row of the tile this lane scores
    const int col = E * lane;        // first head-dim element this lane accumulates
    const int vbox = col >> 6, vcc = (col & 63) >> 3, voff = (col & 7) * 2;
    int g = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      const int bh = item / p.splits;
      const int sp = item - bh * p.splits;
      const int seq_len = decode_seq_len<kPaged>(p, bh / p.H);
      const int t0 = sp * p.tiles_per_split;
      const int t1 = min(min(ntiles, (seq_len + 127) / 128), t0 + p.tiles_per_split);

      // the query row, pre-multiplied by scale*log2(e) (every lane holds all of it)
      float qf[D];
      {
        const uint4* qp = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                                         (long long)bh * D * 2);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 w = __ldg(qp + c);
          const float2 a = unpack2<BF16>(w.x), bb = unpack2<BF16>(w.y);
          const float2 cc = unpack2<BF16>(w.z), dd = unpack2<BF16>(w.w);
          qf[c * 8 + 0] = a.x * p.scale_log2;
          qf[c * 8 + 1] = a.y * p.scale_log2;
          qf[c * 8 + 2] = bb.x * p.scale_log2;
          qf[c * 8 + 3] = bb.y * p.scale_log2;
          qf[c * 8 + 4] = cc.x * p.scale_log2;
          qf[c * 8 + 5] = cc.y * p.scale_log2;
          qf[c * 8 + 6] = dd.x * p.scale_log2;
          qf[c * 8 + 7] = dd.y * p.scale_log2;
        }
      }
      float m = -INFINITY, l = 0.f;
      float o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = 0.f;

      for (int tile = t0; tile < t1; ++tile, ++g) {
        const int stage = g % C::kStages;
        mbar_wait(FULL(stage), (g / C::kStages) & 1, wctx);
        __syncwarp();
        const uint8_t* sK = smem + stage * C::kStageBytes;
        const uint8_t* sV = sK + C::kTileBytes;

        // score of key r (base-2 units): q . k_r
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const int bx = c >> 3, cc = c & 7;
          const uint4 w =
              *reinterpret_cast<const uint4*>(sK + bx * C::kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4));
          const float2 f0 = unpack2<BF16>(w.x), f1 = unpack2<BF16>(w.y);
          const float2 f2 = unpack2<BF16>(w.z), f3 = unpack2<BF16>(w.w);
          a0 = fmaf(qf[c * 8 + 0], f0.x, a0);
          a1 = fmaf(qf[c * 8 + 1], f0.y, a1);
          a0 = fmaf(qf[c * 8 + 2], f1.x, a0);
          a1 = fmaf(qf[c * 8 + 3], f1.y, a1);
          a0 = fmaf(qf[c * 8 + 4], f2.x, a0);
          a1 = fmaf(qf[c * 8 + 5], f2.y, a1);
          a0 = fmaf(qf[c * 8 + 6], f3.x, a0);
          a1 = fmaf(qf[c * 8 + 7], f3.y, a1);
        }
        const bool valid = tile * 128 + r < seq_len;
        const float s = valid ? (a0 + a1) : -INFINITY;
        const float m_new = fmaxf(m, warp_max(s));
        if (m_new != -INFINITY) {
          const float alpha = ex2_approx(m - m_new);  // 0 when m == -inf
          const float pr = valid ? ex2_approx(s - m_new) : 0.f;
          l = l * alpha + warp_sum(pr);
#pragma unroll
          for (int e = 0; e < E; ++e) o[e] *= alpha;
          // o += sum over this warp's 32 keys of p_key * v_key[col .. col+E)
#pragma unroll 8
          for (int kk = 0; kk < 32; ++kk) {
            const float pk = __shfl_sync(0xffffffffu, pr, kk);
            const int vr = warp * 32 + kk;
            const uint8_t* src = sV + vbox * C::kBoxBytes + vr * 128 + ((vcc ^ (vr & 7)) << 4) + voff;
            if constexpr (E == 4) {
              const uint2 w = *reinterpret_cast<const uint2*>(src);
              const float2 v0 = unpack2<BF16>(w.x), v1 = unpack2<BF16>(w.y);
              o[0] = fmaf(pk, v0.x, o[0]);
              o[1] = fmaf(pk, v0.y, o[1]);
              o[2] = fmaf(pk, v1.x, o[2]);
              o[3] = fmaf(pk, v1.y, o[3]);
            } else {
              const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
              const float2 v0 = unpack2<BF16>(w);
              o[0] = fmaf(pk, v0.x, o[0]);
              o[1] = fmaf(pk, v0.y, o[1]);
            }
          }
          m = m_new;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(EMPTY(stage));
      }

      // fold the four warps' states and write this item's partial
      float* mine = scratch + warp * (D + 2);
#pragma unroll
      for (int e = 0; e < E; ++e) mine[col + e] = o[e];
      if (lane == 0) {
        mine[D] = m;
        mine[D + 1] = l;
      }
      named_bar_sync(1, 128);
      const int tid = threadIdx.x;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, scratch[w * (D + 2) + D]);
      float wgt[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = scratch[w * (D + 2) + D];
        wgt[w] = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
      }
      float* dst = p.part + (long long)item * (D + 2);
      for (int d = tid; d < D; d += 128) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) acc = fmaf(wgt[w], scratch[w * (D + 2) + d], acc);
        dst[d] = acc;
      }
      if (tid == 0) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) L = fmaf(wgt[w], scratch[w * (D + 2) + D + 1], L);
        dst[D] = M;
        dst[D + 1] = L;
      }
      named_bar_sync(1, 128);
    }
  }
}

// Merge the partials of each (b, h) row: M = max_s m_s, w_s = 2^(m_s - M),
// O = sum_s w_s o_s / sum_s w_s l_s, lse = (M + log2(sum_s w_s l_s)) * ln 2.
template <int D, bool BF16>
__global__ void __launch_bounds__(128)
    attn_decode_combine_kernel(const float* __restrict__ part, void* __restrict__ out,
                               float* __restrict__ lse, int BH, int splits) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + warp;
  if (bh >= BH) return;
  const float* base = part + (long long)bh * splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, base[s * (D + 2) + D]);
  float L = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float* ps = base + s * (D + 2);
    const float ms = ps[D];
    const float w = (ms == -INFINITY) ? 0.f : ex2_approx(ms - M);
    L = fmaf(w, ps[D + 1], L);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(w, ps[E * lane + e], acc[e]);
  }
  const float inv = L > 0.f ? 1.0f / L : 0.f;
  uint8_t* orow = static_cast<uint8_t*>(out) + (long long)bh * D * 2;
  if constexpr (E == 4) {
    uint2 w;
    w.x = pack2<BF16>(acc[0] * inv, acc[1] * inv);
    w.y = pack2<BF16>(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(orow + E * lane * 2) = w;
  } else {
    *reinterpret_cast<uint32_t*>(orow + E * lane * 2) = pack2<BF16>(acc[0] * inv, acc[1] * inv);
  }
  if (lse != nullptr && lane == 0)
    lse[bh] = L > 0.f ? (M + lg2_approx(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn_b200

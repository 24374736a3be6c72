// relpos_sm100.cuh -- attention with a fused relative-position score term (sm_100a).
//
// vLLM page "PR #42933" (Granite-Speech conformer block attention), sections "实现拆解"
// and "关键源码片段": the attention scores of a block carry, besides q_i . k_j, the term
// q_i . emb[dist[i, j]] (the einsum "bnhid,ijd->bnhij" of the queries with the gathered
// relative-position embeddings), both multiplied by the scale, before masking and the
// softmax.  The distance table is the conformer's clamped relative distance,
//   dist[i, j] = clamp(i - j, -R, R) + R,     emb row R = distance 0,
// so the kernel takes R and never reads a table.
//
// Persistent CTAs over units (b, h, 128-query tile); keys in steps of 64.  For a pair of
// steps (128 keys) the distances met span at most 255 consecutive embedding rows
// (lo ... lo + 254, clamped at 0 and 2R), so on every other step the tensor core computes
// G = Q E_win^T (N = 256: TMEM lane = query row, column = window row) next to S = Q K^T,
// and the next window has a whole step to arrive.  Query row r needs the columns
// dist(r, j) - lo for its 64 keys of a step, a run of at most 64 that starts at a
// row-dependent column: the two softmax warps of a row copy the 112 columns that cover
// their runs into the row's shared-memory line (pitch 116 words, so the copy and the
// skewed reads are free of bank conflicts) and gather from there.  Roles (320 threads):
//   * warp 8, producer: Q of each unit as soon as the previous unit's last product has read
//     it, the K/V ring (two stages), the embedding window of each step pair as soon as the
//     previous pair's product has read the buffer (so the next unit's loads run behind the
//     current unit's last step and epilogue);
//   * warp 9, MMA issuer: S (and G) of step t, then O += P V of step t - 1 once P is ready;
//   * warps 0-7, softmax (two warps per query row, 32 keys of a step each): copy and
//     gather G, online softmax (fp16 P into shared memory, in the K slot of the step at
//     d = 128; O rescaled in TMEM when the row maximum grows), and the O / l epilogue.  For
//     bf16 inputs they convert each V tile to fp16 in place first (P V runs in fp16, as in
//     the plain kernel; magnitudes with no fp16 value set the range status).
#pragma once

#include "sm100_ptx.cuh"

namespace attn_b200 {

struct RelposParams {
  CUtensorMap tm_q;  // q [B, Nq, H, D] as 4-D (D, H, Nq, B), box (64, 1, 128, 1), 128B swizzle
  CUtensorMap tm_k;  // k [B, Nk, H, D] as 4-D (D, H, Nk, B), box (64, 1, 64, 1)
  CUtensorMap tm_v;  // v, as k
  CUtensorMap tm_e;  // emb [n_emb, D] as 3-D (D, n_emb, 1), box (64, 192, 1)
  void* out;         // [B, Nq, H, D], the input dtype
  float* lse;        // [B, H, Nq] natural log, or nullptr
  int* status;
  int B, H, Nq, Nk, R, causal;
  int n_qtiles, n_units;  // 128-query tiles per (b, h); units (b, h, tile)
  float scale_log2;  // scale * log2(e)
  unsigned long long timeout_ns;
};

template <int D>
struct RelposCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  static constexpr int kBoxes = D / 64;
  static constexpr int kQBytes = kBoxes * 128 * 128;   // 128 rows x D
  static constexpr int kKVBytes = kBoxes * 64 * 128;   // 64 rows x D
  static constexpr int kWinRows = 256;                  // embedding rows two steps can need (255)
  static constexpr int kEBoxBytes = kWinRows * 128;     // 256 rows x 64 elements
  static constexpr int kEBytes = kBoxes * kEBoxBytes;
  static constexpr int kGCols = 112;                    // columns of G a thread keeps per step
  static constexpr int kGPitch = 116;                   // words of a thread's row of G
  static constexpr bool kPInK = D == 128;               // P (16 KB) fits the step's K slot
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;         // [2]
  static constexpr int kOffV = kOffK + 2 * kKVBytes;    // [2]
  static constexpr int kOffE = kOffV + 2 * kKVBytes;    // embedding window
  static constexpr int kOffP = kOffE + kEBytes;         // 128 x 64 fp16, 128B swizzle (D = 64)
  static constexpr int kOffG = kOffP + (kPInK ? 0 : 128 * 128);  // [128 rows][kGPitch] fp32
  static constexpr int kOffX = kOffG + 128 * kGPitch * 4;  // [max, sum][half][128 rows] fp32
  static constexpr int kOffBar = kOffX + 2 * 2 * 128 * 4;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKVFull = 1;   // [2]
  static constexpr int kBarKVEmpty = 3;  // [2]
  static constexpr int kBarEFull = 5;
  static constexpr int kBarSFull = 6;    // S (and G, even steps) of the step are in TMEM
  static constexpr int kBarSFree = 7;    // ... and have been read (8 arrivals)
  static constexpr int kBarPFull = 8;    // P written, O rescaled, V converted (8 arrivals)
  static constexpr int kBarPVDone = 9;   // O += P V of the step has completed
  static constexpr int kBarMmaDone = 10;
  static constexpr int kBarEFree = 11;   // the G product of a step pair has read the window
  static constexpr int kBarQFree = 12;   // the last product of a unit has read Q
  static constexpr int kBarOFree = 13;   // the epilogue of a unit has read O (8 arrivals)
  static constexpr int kNumBars = 14;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // +1024: manual 1 KB alignment
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
  static constexpr int kProducerWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  // TMEM columns; a warp's G loads start at most 224 columns past kColG and read 128
  // (past column 383 they read values no thread uses)
  static constexpr uint32_t kColO = 0;    // D columns
  static constexpr uint32_t kColG = 128;  // 256 columns
  static constexpr uint32_t kColS = 448;  // 64 columns
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Keys of the CTA's query tile: steps of 64 up to the last key any of its rows may see.
__device__ __forceinline__ int relpos_steps(const RelposParams& p, int q0) {
  int kend = p.Nk;  // one past the last key
  if (p.causal) {
    const int last_row = min(q0 + 127, p.Nq - 1);
    kend = min(p.Nk, last_row + (p.Nk - p.Nq) + 1);
  }
  return kend <= 0 ? 0 : (kend + 63) / 64;
}

// First embedding row a pair of steps (128 keys from k0) needs: the smallest clamped
// distance over the query tile and those keys.  The window lo ... lo + 255 covers the
// pair (distances span 255 values).
__device__ __forceinline__ int relpos_lo(const RelposParams& p, int q0, int k0) {
  return min(max(q0 - (k0 + 127), -p.R), p.R) + p.R;
}


// Softmax warps 0-7: warps w and w + 4 share query rows 32 (w % 4) .. + 31 (TMEM lanes)
// and take keys 32 hf .. + 31 of each 64-key step, hf = w / 4.  The pair copies the two
// halves of its rows' G window, exchanges the half-row maxima and the final row sums
// through shared memory (64-thread named barriers 2 + w % 4), and splits the O rescale and
// the epilogue by head-dim halves.
template <int D, bool BF16>
__device__ __forceinline__ void relpos_softmax(const RelposParams& p, uint8_t* smem, uint32_t tmem,
                                               uint64_t* bars, const WaitCtx& wctx) {
  using C = RelposCfg<D>;
  auto BAR = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qw = warp & 3, hf = warp >> 2;
  const int r = qw * 32 + lane;  // row of the tile
  const int tid = threadIdx.x;   // 0..255
  const uint32_t pair_bar = 2 + qw;
  const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
  float* grow = reinterpret_cast<float*>(smem + C::kOffG) + r * C::kGPitch;  // this row's G
  float* xch = reinterpret_cast<float*>(smem + C::kOffX);  // [max, sum][half][128 rows]
  const int shift = p.Nk - p.Nq;  // bottom-right causal alignment
  uint32_t vmag = 0;              // bf16: largest |V| bit pattern converted
  int g = 0;                      // steps of this CTA so far (barrier phases)

  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
  const int q0 = (u % p.n_qtiles) * 128;
  const int h = (u / p.n_qtiles) % p.H, b = u / (p.n_qtiles * p.H);
  const int i = q0 + r;
  const int nsteps = relpos_steps(p, q0);
  float m = -INFINITY;            // running maximum of scale * log2(e) * score (whole row)
  float l0 = 0.f, l1 = 0.f;       // this warp's sum of the fp16-rounded P

  for (int t = 0; t < nsteps; ++t, ++g) {
    const int k0 = t * 64;
    const int lo = relpos_lo(p, q0, (t & ~1) * 64);  // window of the step pair
    mbar_wait(BAR(C::kBarSFull), g & 1, wctx);
    __syncwarp();
    tc_fence_after_sync();
    // ---- these rows need window columns cw ... cw + 94 (the clamp is monotone and moves
    // by at most one per row or key): of the 128 from the 32-aligned column below, the 112
    // from base + s0 (s0 = 0 or 16) hold them; this warp copies the half hf of the 128
    const int cw = min(max(q0 + qw * 32 - (k0 + 63), -p.R), p.R) + p.R - lo;
    const int s0 = (cw & 31) & 16;
    const int base = (cw & ~31) + s0;  // column of grow[0]
#pragma unroll 1
    for (int q = 2 * hf; q < 2 * hf + 2; ++q) {
      uint32_t gv[32];
      tmem_ld32(tmem + lane_base + C::kColG + (cw & ~31) + q * 32, gv);
      tmem_ld_wait();
      reg_order_after_wait(gv);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int dst = q * 32 + 4 * e - s0;
        if (dst >= 0 && dst < C::kGCols)  // uniform over the warp
          *reinterpret_cast<float4*>(grow + dst) =
              make_float4(__uint_as_float(gv[4 * e]), __uint_as_float(gv[4 * e + 1]),
                          __uint_as_float(gv[4 * e + 2]), __uint_as_float(gv[4 * e + 3]));
      }
    }
    // ---- this row's 32 raw scores of this warp's keys
    uint32_t sv[32];
    tmem_ld32(tmem + lane_base + C::kColS + hf * 32, sv);
    tmem_ld_wait();
    reg_order_after_wait(sv);
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(C::kBarSFree));  // S and G may be overwritten
    named_bar_sync(pair_bar, 64);                    // both halves of the rows are copied
    // ---- add the gathered term, scale, mask
    float x[32];
    float mx = -INFINITY;
    // keys k0 + jj with jj < jlim are allowed for this row (tail and bottom-right causal)
    const int jlim = i < p.Nq ? (p.causal ? min(p.Nk, i + shift + 1) : p.Nk) - k0 : 0;
    // no allowed key of the step has a clamped distance; key k0 is then allowed and its
    // column lies in the row, and a masked key reads at most 63 words below it (inside
    // shared memory, a value of no use)
    const bool unclamped = i - (k0 + min(63, jlim - 1)) >= -p.R && i - k0 <= p.R;
    if (jlim <= 0) {  // the row sees no key of this step
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = -INFINITY;
    } else if (unclamped) {
      // key jj's column is (key k0's column) - jj
      const float* gp = grow + (i - k0 + p.R - lo - base) - hf * 32;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        x[e] = hf * 32 + e < jlim ? (__uint_as_float(sv[e]) + gp[-e]) * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, x[e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int j = k0 + hf * 32 + e;
        const bool allowed = i < p.Nq && j < p.Nk && (!p.causal || j <= i + shift);
        // column of key j in this row's copy
        const int c = min(max(i - j, -p.R), p.R) + p.R - lo - base;
        const float gg = grow[c];
        x[e] = allowed ? (__uint_as_float(sv[e]) + gg) * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, x[e]);
      }
    }
    // ---- the row maximum from both halves (after this barrier both warps are also done
    // reading the copied row)
    xch[hf * 128 + r] = mx;
    named_bar_sync(pair_bar, 64);
    const float m_new = fmaxf(m, fmaxf(mx, xch[(hf ^ 1) * 128 + r]));
    // ---- online softmax: O and the P buffer are free once the previous P V is done
    if (t >= 1) {
      mbar_wait(BAR(C::kBarPVDone), (g - 1) & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      const bool grow_m = m_new > m && m > -INFINITY;
      if (__any_sync(0xffffffffu, grow_m)) {  // TMEM loads and stores are warp-collective
        const float f = grow_m ? ex2_approx(m - m_new) : 1.0f;
        l0 *= f;
        l1 *= f;
#pragma unroll 1
        for (int cq = hf * (D / 64); cq < (hf + 1) * (D / 64); ++cq) {  // this warp's half of O
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + C::kColO + cq * 32, o);
          tmem_ld_wait();
          reg_order_after_wait(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(tmem + lane_base + C::kColO + cq * 32, o);
        }
        tmem_st_wait();
      }
    }
    m = m_new;
    const float mu = m == -INFINITY ? 0.f : m;  // a row that saw no key yet: every P is 0
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      pk[e] = pack2<false>(ex2_approx(x[2 * e] - mu), ex2_approx(x[2 * e + 1] - mu));
      add_f16x2_f32(l0, l1, pk[e]);
    }
    // P row r: 64 fp16 = eight 16-byte chunks, 128-byte swizzle (K-major A operand); this
    // warp's four; at d = 128 in the step's K slot, which S has finished reading
    uint8_t* sp = smem + (C::kPInK ? C::kOffK + (g & 1) * C::kKVBytes : C::kOffP);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
      *reinterpret_cast<uint4*>(sp + r * 128 + (((hf * 4 + cc) ^ (r & 7)) << 4)) =
          make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
    if constexpr (BF16) {  // V of this step to fp16, in place
      mbar_wait(BAR(C::kBarKVFull + (g & 1)), (g >> 1) & 1, wctx);
      uint4* tile = reinterpret_cast<uint4*>(smem + C::kOffV + (g & 1) * C::kKVBytes);
#pragma unroll 2
      for (int c = tid; c < C::kKVBytes / 16; c += 256) {
        uint4 w = tile[c];
        vmag = __vmaxu2(vmag, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                       __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
        w.x = bf16x2_to_f16x2_sat(w.x);
        w.y = bf16x2_to_f16x2_sat(w.y);
        w.z = bf16x2_to_f16x2_sat(w.z);
        w.w = bf16x2_to_f16x2_sat(w.w);
        tile[c] = w;
      }
    }
    fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(C::kBarPFull));
  }

  // ---- epilogue: O / l in the input dtype (this warp's half of the head dim), lse =
  // ln(sum exp(scale * score)); the row sum adds both warps' halves
  xch[256 + hf * 128 + r] = l0 + l1;
  named_bar_sync(pair_bar, 64);
  const float l = l0 + l1 + xch[256 + (hf ^ 1) * 128 + r];
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const bool row_ok = i < p.Nq;
  uint4* orow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) +
                                         ((((long long)b * p.Nq + (row_ok ? i : 0)) * p.H + h) * D) * 2);
  if (nsteps > 0) {
    mbar_wait(BAR(C::kBarPVDone), (g - 1) & 1, wctx);
    __syncwarp();
    tc_fence_after_sync();
#pragma unroll 1
    for (int cq = hf * (D / 64); cq < (hf + 1) * (D / 64); ++cq) {
      uint32_t o[32];
      tmem_ld32(tmem + lane_base + C::kColO + cq * 32, o);
      tmem_ld_wait();
      reg_order_after_wait(o);
      if (row_ok) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          orow[cq * 4 + e] = make_uint4(
              pack2<BF16>(__uint_as_float(o[8 * e]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
              pack2<BF16>(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
              pack2<BF16>(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
              pack2<BF16>(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
      }
    }
    // O may be overwritten by the next unit's first P V
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(C::kBarOFree));
  } else if (row_ok) {  // no key reaches this tile
#pragma unroll
    for (int c = hf * (D / 16); c < (hf + 1) * (D / 16); ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (row_ok && hf == 0 && p.lse != nullptr)
    p.lse[((long long)b * p.H + h) * p.Nq + i] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  }  // units
  if constexpr (BF16) {
    if (max(vmag & 0xFFFFu, vmag >> 16) >= kBf16NoF16) atomicCAS(p.status, 0, kStatusRange);
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(RelposCfg<D>::kThreads, 1)
    attn_relpos_kernel(const __grid_constant__ RelposParams p) {
  using C = RelposCfg<D>;
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
  // persistent CTAs: units u = (b, h, tile) in steps of gridDim.x; every role walks the
  // same units, and barrier phases count steps, pairs and units over the whole walk
  auto unit = [&](int u, int& q0, int& h, int& b) {
    q0 = (u % p.n_qtiles) * 128;
    h = (u / p.n_qtiles) % p.H;
    b = u / (p.n_qtiles * p.H);
  };

  if (threadIdx.x == 0) {
    mbar_init(BAR(C::kBarQFull), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(C::kBarKVFull + s), 1);
      mbar_init(BAR(C::kBarKVEmpty + s), 1);
    }
    mbar_init(BAR(C::kBarEFull), 1);
    mbar_init(BAR(C::kBarSFull), 1);
    mbar_init(BAR(C::kBarSFree), C::kSoftmaxWarps);
    mbar_init(BAR(C::kBarPFull), C::kSoftmaxWarps);
    mbar_init(BAR(C::kBarPVDone), 1);
    mbar_init(BAR(C::kBarMmaDone), 1);
    mbar_init(BAR(C::kBarEFree), 1);
    mbar_init(BAR(C::kBarQFree), 1);
    mbar_init(BAR(C::kBarOFree), C::kSoftmaxWarps);
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
      tma_prefetch_map(&p.tm_e);
    }
    int g = 0, ge = 0, nu = 0;  // steps, step pairs and units (with keys) loaded
    bool stop = false;
    for (int u = blockIdx.x; u < p.n_units && !stop; u += gridDim.x) {
      int q0, h, b;
      unit(u, q0, h, b);
      const int nsteps = relpos_steps(p, q0);
      if (nsteps == 0) continue;
      // one Q buffer: the previous unit's last product must have read it
      if (nu >= 1) mbar_wait(BAR(C::kBarQFree), (nu - 1) & 1, wctx);
      __syncwarp();
      if (warp_flag(abort_flag)) break;
      mbar_arrive_expect_tx_w(BAR(C::kBarQFull), C::kQBytes);
      for (int bx = 0; bx < C::kBoxes; ++bx)
        tma_load_4d_w(sbase + C::kOffQ + bx * 16384, &p.tm_q, BAR(C::kBarQFull), bx * 64, h, q0, b);
      ++nu;
      for (int t = 0; t < nsteps; ++t, ++g) {
        const int s = g & 1, k0 = t * 64;
        if (g >= 2) mbar_wait(BAR(C::kBarKVEmpty + s), ((g >> 1) - 1) & 1, wctx);
        __syncwarp();
        if (warp_flag(abort_flag)) {
          stop = true;
          break;
        }
        mbar_arrive_expect_tx_w(BAR(C::kBarKVFull + s), 2 * C::kKVBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          tma_load_4d_w(sbase + C::kOffK + s * C::kKVBytes + bx * 8192, &p.tm_k, BAR(C::kBarKVFull + s),
                        bx * 64, h, k0, b);
          tma_load_4d_w(sbase + C::kOffV + s * C::kKVBytes + bx * 8192, &p.tm_v, BAR(C::kBarKVFull + s),
                        bx * 64, h, k0, b);
        }
        // embedding windows, one per step pair, in the order the products take them: the
        // first before any product needs it, then the next pair's as soon as this pair's
        // K/V loads are issued (it only waits for this pair's G product to read the buffer)
        auto load_window = [&](int lo) {
          if (ge >= 1) mbar_wait(BAR(C::kBarEFree), (ge - 1) & 1, wctx);
          __syncwarp();
          if (warp_flag(abort_flag)) return false;
          mbar_arrive_expect_tx_w(BAR(C::kBarEFull), C::kEBytes);
          for (int bx = 0; bx < C::kBoxes; ++bx)  // rows past n_emb read as zeros and are never used
            tma_load_3d_w(sbase + C::kOffE + bx * C::kEBoxBytes, &p.tm_e, BAR(C::kBarEFull), bx * 64, lo, 0);
          ++ge;
          return true;
        };
        bool ok = true;
        if (ge == 0) ok = load_window(relpos_lo(p, q0, k0));
        if (ok && ((t & 1) || t == nsteps - 1)) {  // last step of its pair
          int lon = 0;
          bool has_next = false;
          if (t + 1 < nsteps) {
            lon = relpos_lo(p, q0, (t + 1) * 64);
            has_next = true;
          } else {
            for (int u2 = u + (int)gridDim.x; u2 < p.n_units; u2 += gridDim.x) {
              const int q2 = (u2 % p.n_qtiles) * 128;
              if (relpos_steps(p, q2) > 0) {
                lon = relpos_lo(p, q2, 0);
                has_next = true;
                break;
              }
            }
          }
          if (has_next) ok = load_window(lon);
        }
        if (!ok) {
          ++g;  // this step's K/V copy is in flight
          stop = true;
          break;
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // let every copy this warp started land before the CTA can exit
      if (nu > 0) mbar_wait_drain(BAR(C::kBarQFull), (nu - 1) & 1, p.timeout_ns);
      for (int i = max(0, g - 2); i < g; ++i)
        mbar_wait_drain(BAR(C::kBarKVFull + (i & 1)), (i >> 1) & 1, p.timeout_ns);
      if (ge > 0) mbar_wait_drain(BAR(C::kBarEFull), (ge - 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ======================= tcgen05 MMA issuer =======================
    constexpr uint32_t idesc_s = make_idesc_f16(128, 64, BF16, false);   // Q K^T, both K-major
    constexpr uint32_t idesc_g = make_idesc_f16(128, C::kWinRows, BF16, false);  // Q E_win^T, both K-major
    constexpr uint32_t idesc_o = make_idesc_f16(128, D, false, true);    // P V: fp16, V MN-major
    int nu = 0;  // units (with keys) whose products were issued
    // O += P V of step g (t-th of its unit); the first of a unit waits until the previous
    // unit's epilogue has read O
    auto issue_pv = [&](int g, int t) {
      if (t == 0 && nu >= 2) mbar_wait(BAR(C::kBarOFree), (nu - 2) & 1, wctx);
      mbar_wait(BAR(C::kBarPFull), g & 1, wctx);
      __syncwarp();
      tc_fence_after_sync();
      if (!warp_flag(abort_flag)) {
        const uint32_t sV = sbase + C::kOffV + (g & 1) * C::kKVBytes;
        const uint32_t sP = sbase + (C::kPInK ? C::kOffK + (g & 1) * C::kKVBytes : C::kOffP);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 keys per k-step
          mma_f16_ss_w(tmem + C::kColO, make_sdesc_sw128(sP + kk * 32, 16, 1024),
                       make_sdesc_sw128(sV + kk * 2048, 8192, 1024), idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit_w(BAR(C::kBarPVDone));
        tc_commit_w(BAR(C::kBarKVEmpty + (g & 1)));
      }
    };
    int g = 0, ge = 0;
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
      int q0, h, b;
      unit(u, q0, h, b);
      const int nsteps = relpos_steps(p, q0);
      if (nsteps == 0) continue;
      mbar_wait(BAR(C::kBarQFull), nu & 1, wctx);
      ++nu;
      for (int t = 0; t < nsteps; ++t, ++g) {
        const int s = g & 1;
        mbar_wait(BAR(C::kBarKVFull + s), (g >> 1) & 1, wctx);
        if (!(t & 1)) mbar_wait(BAR(C::kBarEFull), ge & 1, wctx);
        if (g >= 1) mbar_wait(BAR(C::kBarSFree), (g - 1) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        if (!warp_flag(abort_flag)) {
          const uint32_t sQ = sbase + C::kOffQ;
          const uint32_t sK = sbase + C::kOffK + s * C::kKVBytes;
          const uint32_t sE = sbase + C::kOffE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // 16 head-dim elements per k-step
            const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_f16_ss_w(tmem + C::kColS, make_sdesc_sw128(sQ + oq, 16, 1024),
                         make_sdesc_sw128(sK + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idesc_s,
                         kk > 0 ? 1u : 0u);
          }
          if (!(t & 1)) {  // G of the step pair
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_f16_ss_w(tmem + C::kColG, make_sdesc_sw128(sQ + oq, 16, 1024),
                           make_sdesc_sw128(sE + (kk >> 2) * C::kEBoxBytes + (kk & 3) * 32, 16, 1024),
                           idesc_g, kk > 0 ? 1u : 0u);
            }
            tc_commit_w(BAR(C::kBarEFree));
          }
          tc_commit_w(BAR(C::kBarSFull));
          if (t == nsteps - 1) tc_commit_w(BAR(C::kBarQFree));  // Q of this unit is read
        }
        if (!(t & 1)) ++ge;
        if (t >= 1) issue_pv(g - 1, t - 1);
      }
      issue_pv(g - 1, nsteps - 1);
    }
    // every MMA (and every commit arrive) has landed before TMEM is released
    tc_commit_w(BAR(C::kBarMmaDone));
    mbar_wait_drain(BAR(C::kBarMmaDone), 0, p.timeout_ns);
    __syncwarp();
  } else {
    relpos_softmax<D, BF16>(p, smem, tmem, bars, wctx);
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

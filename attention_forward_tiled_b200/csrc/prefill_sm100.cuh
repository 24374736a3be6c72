// prefill_sm100.cuh -- tiled attention forward for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V block by block with the
// online softmax update, so the Nq x Nk score matrix never leaves the SM
// (FlashAttention/ops-transformer article, sections "FlashAttention的核心逻辑"
// and "传统注意力的显存陷阱").  The article's Ascend tiling (Cube unit for the
// matmuls, Vector unit for the softmax, 128x64 blocks staged in the Unified
// Buffer) is prior art; this kernel maps the same algorithm onto B200.
//
// Work unit = (batch b, head h, a pair of 128-row Q tiles).  The grid has one CTA
// per unit, but a resident CTA (one per SM) keeps going: late in each unit it claims
// the next not-yet-started CTA with cluster launch control
// (clusterlaunchcontrol.try_cancel) and does that CTA's unit as well, so units are
// handed out dynamically, in launch order (heaviest causal units first, heads in
// groups so their K/V stay in L2), to the SMs about to run out of work, and TMEM,
// barriers and the load pipeline stay up across units.  Roles inside a CTA (384
// threads):
//   * warp 8, producer: claims units, decodes them and publishes them to the other
//     roles through a two-slot ring in shared memory; loads Q_t once per unit and
//     streams K_0, V_0, K_1, V_1, ... into a ring of shared-memory stages with TMA
//     (128-byte swizzle), each stage guarded by a full/empty mbarrier pair;
//   * warp 9, MMA issuer (whole warp, one elected lane issues a batch of k-steps at
//     a time) runs tcgen05.mma:
//       S_t = Q_t K_j^T   (A, B from shared memory, fp32 accumulator in TMEM)
//       O_t += P_t V_j    (A = P_t from TMEM, B = V from shared memory)
//     alternating the two Q tiles so one tile's softmax overlaps the other tile's
//     matrix multiplies.  d = 128: P_t is written over the consumed S_t columns, so
//     S_t(j+1) follows P_t(j) V_j; the softmax publishes P for keys 64..127 first and
//     that half of P V starts at once.  d = 64: TMEM has room for separate P buffers,
//     so S_t(j+1) is issued as soon as the softmax has read S_t(j) and is computed
//     while that softmax runs;
//   * warps 10-11 (bf16 inputs only) convert each V tile to fp16 in place, so
//     P V runs with P in fp16 (11-bit significand) rather than bf16 (8-bit);
//   * warps 0-3 and 4-7, softmax warpgroups (one per Q tile, one thread per query
//     row): read the 128-column S row from TMEM, apply the tail/causal mask, update
//     the running max m and sum l (base-2 exponent with scale*log2(e) folded into one
//     packed FMA, lazy rescale of O only when the max grows by more than 2^8; at
//     d = 128 unmasked tiles after the first take a single pass against the running
//     max), write P as fp16 into TMEM, and at the end of the unit normalise O by 1/l,
//     stage it in shared memory, store it with TMA and write the row LSE.
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D); P_t in columns [64,128) of S_t (d = 128) or in its own
// columns P_0 [384,448), P_1 [448,512) (d = 64).
// Shared memory: Q_0, Q_1 | K/V ring | O staging (one buffer the two tiles take
// turns with for d = 128, one per tile for d = 64).
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
  int n_split;       // the last n_split pair units run as two single-tile units each
  float scale_log2;  // scale * log2(e)
  int inject;        // test hook: 1 = skip the Q-tile-0 loads
  unsigned long long timeout_ns;
};

// Bounded mbarrier waits with the polling loop inline (the waits of sm100_ptx.cuh call an
// out-of-line loop): the d = 64 kernel re-balances registers between warpgroups
// (setmaxnreg), which ptxas allocates only in a kernel that makes no calls; a call would
// also make the caller save its live registers around it.  Same limits and abort rules.
__device__ __forceinline__ bool mbar_wait_inline(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long limit = wait_limit_cycles(w.timeout_ns);
  const long long c0 = clock64();
  for (uint32_t it = 0; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) return false;
    if (clock64() - c0 > limit) break;
  }
  *w.abort_flag = 1;
  atomicCAS(w.status, 0, kStatusTimeout);
  return false;
}

__device__ __forceinline__ bool mbar_wait_drain_inline(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  const long long limit = wait_limit_cycles(timeout_ns);
  const long long c0 = clock64();
  for (uint32_t it = 0; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - c0 > limit) return false;
  }
  return false;
}

// Four k-steps of D = A B with A and B K-major in shared memory (128-byte swizzle, one
// 64-element box along K): one elected lane issues all four, advancing both descriptors'
// start address by 32 B per k-step.
__device__ __forceinline__ void mma_f16_ss_k64_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
  constexpr uint64_t kStep = 32 >> 4;
  asm volatile(
      "{\n\t.reg .pred p, e, t;\n\t.reg .b64 a, b;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, 0, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 a, %1, %5;\n\tadd.s64 b, %2, %5;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
      "add.s64 a, %1, %6;\n\tadd.s64 b, %2, %6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t"
      "add.s64 a, %1, %7;\n\tadd.s64 b, %2, %7;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a, b, %3, t;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kStep), "n"(2 * kStep),
      "n"(3 * kStep)
      : "memory");
}

constexpr int kUnitInts = 8;  // ints per published work unit (PrefillUnit)

template <int D>
struct PrefillCfg {
  static_assert(D == 64 || D == 128, "head_dim must be 64 or 128");
  // d = 64: separate P columns in TMEM, S released as soon as the softmax has read it.
  // d = 128: TMEM is full (2 S + 2 O tiles = 512 columns), P aliases the consumed S columns.
  static constexpr bool kDecoupled = (D == 64);
  static constexpr int kBoxBytes = 128 * 128;            // 128 rows x 64 elements x 2 bytes
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // one 128-row Q, K, V or O tile
  static constexpr int kStages = (D == 128) ? 4 : 8;    // K/V ring depth
  // The next unit is claimed this many ring items before the current unit's last load
  // (measured: a lead of 4 or 16 items at d = 128 was slower or equal).
  static constexpr int kClaimLead = 2 * kStages;
  static constexpr int kNumOStage = kDecoupled ? 2 : 1;  // O staging buffers
  static constexpr int kOffQ = 0;                                    // Q_0, Q_1
  static constexpr int kOffKV = 2 * kTileBytes;                      // K/V ring
  static constexpr int kOffO = kOffKV + kStages * kTileBytes;        // O staging
  static constexpr int kOffBar = kOffO + kNumOStage * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // +1024: manual 1 KB alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColP = 384;  // d = 64: P_t at kColP + 64 t
  static constexpr int kThreads = 384;
  static constexpr int kProducerWarp = 8;
  static constexpr int kMmaWarp = 9;
  static constexpr int kConvWarp0 = 10;
  static constexpr int kUnitReaders = 11;  // warps that read each published unit: 8 softmax, MMA, 2 converter
  // Registers per thread: 168 at launch (the 64 K file over 384 threads).  The file is split
  // into four 16 K sub-partitions, and warp w runs on sub-partition w % 4, so each one holds
  // two softmax warps and one warp of warpgroup 2 (producer, MMA issuer, converters).  At
  // d = 64 warpgroup 2 gives registers up and the softmax warps take them, sub-partition by
  // sub-partition: 2 x 208 + 88 = 3 x 168, so every thread keeps its 128 scores in registers.
  static constexpr int kLaunchRegs = 168;
  static constexpr int kRegsSoftmax = 208;
  static constexpr int kRegsAux = 88;
  static_assert(2 * kRegsSoftmax + kRegsAux == 3 * kLaunchRegs && kLaunchRegs * kThreads <= 65536,
                "register split must add up to the launch's registers");
  // barrier indices
  static constexpr int kBarQFull = 0;      // [2] Q_t landed
  static constexpr int kBarQEmpty = 2;     // [2] last S_t of the unit done: Q_t buffer free
  static constexpr int kBarSFull = 4;      // [2] S_t in TMEM
  static constexpr int kBarSFree = 6;      // [2] (d = 64) the softmax has read S_t (4 warps)
  static constexpr int kBarPFull = 8;      // [2] P_t written (d = 128: keys 0..63 last), O_t rescaled (4 warps)
  static constexpr int kBarPVDone = 10;    // [2] d = 64: every P_t V done; d = 128: the unit's last one
  static constexpr int kBarOStage = 12;    // [2] (d = 128) tile t's turn with the O staging buffer is over
  static constexpr int kBarMmaDone = 14;   // [1] teardown
  static constexpr int kBarClc = 15;       // [1] launch-control response landed
  static constexpr int kBarUnitFull = 16;  // [2] unit ring slot written
  static constexpr int kBarUnitEmpty = 18; // [2] unit ring slot read by every reader warp
  static constexpr int kBarOReady = 20;   // [2] tile t's rows are in its O staging buffer (4 warps)
  static constexpr int kBarOFree = 22;    // [2] (d = 64) tile t's previous O store has read its buffer
  static constexpr int kBarPHalf = 24;    // [2] (d = 128) P_t for keys 64..127 written, O_t rescaled (4 warps)
  static constexpr int kBarKVFull = 26;    // [kStages]
  static constexpr int kBarKVEmpty = 26 + kStages;
  static constexpr int kBarVConv = 26 + 2 * kStages;  // [kStages] V tile converted (bf16 only)
  static constexpr int kNumBars = 26 + 3 * kStages;
  static constexpr int kOffMisc = kNumBars * 8;  // tmem slot, abort flag, pad, unit slots[2][kUnitInts]
  static constexpr int kMiscBytes = 16 + 2 * kUnitInts * 4;
  static constexpr int kOffClc = ((kOffMisc + kMiscBytes + 15) / 16) * 16;  // 16-byte launch-control response
  static_assert(kOffClc + 16 <= kBarBytes, "barrier area too small");
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

// Work unit index -> (b, h, Q-tile rows, K/V tile counts).  Units run in groups of
// `group_heads` heads; inside a group, causal units go heaviest (last Q rows) first.
// The producer decodes each unit once and publishes the result to the other roles.
struct PrefillUnit {
  int id;  // unit index (-1: no more units)
  int b, h;
  int row0[2];
  int nkv[2];
  int nmax;
};

// All quantities fit in 32 bits: the launcher rejects grids of 2^31 units or more.
// Units past the first B*H*n_qpairs - n_split are single Q tiles: the last n_split pairs,
// split in two, so the final wave of equal-sized (non-causal) units is half as long.
__device__ __forceinline__ PrefillUnit prefill_unit(const PrefillParams& p, int unit) {
  const int BH = p.B * p.H;
  const int nqp = p.n_qpairs;
  const int G = p.group_heads;
  const int n_pairs = BH * nqp - p.n_split;
  int pair = unit, single = -1;  // single: which tile of a split pair this unit runs
  if (unit >= n_pairs) {
    pair = n_pairs + ((unit - n_pairs) >> 1);
    single = (unit - n_pairs) & 1;
  }
  const int per_group = G * nqp;
  const int full_units = (BH / G) * per_group;
  int g, idx, Gc;
  if (pair < full_units) {
    g = pair / per_group;
    idx = pair - g * per_group;
    Gc = G;
  } else {
    g = BH / G;
    idx = pair - full_units;
    Gc = BH - g * G;
  }
  const int qrank = idx / Gc;
  const int bh = g * G + (idx - qrank * Gc);
  const int qp = p.causal ? (nqp - 1 - qrank) : qrank;
  PrefillUnit u;
  u.id = unit;
  u.b = bh / p.H;
  u.h = bh - u.b * p.H;
  u.row0[0] = qp * 256;
  u.row0[1] = qp * 256 + 128;
  if (single >= 0) {  // tile slot 1 idles: rows at or past Nq are neither computed nor stored
    u.row0[0] = qp * 256 + 128 * single;
    u.row0[1] = p.Nq;
  }
  u.nkv[0] = prefill_kv_tiles(u.row0[0], p.Nq, p.Nk, p.causal);
  u.nkv[1] = prefill_kv_tiles(u.row0[1], p.Nq, p.Nk, p.causal);
  u.nmax = max(u.nkv[0], u.nkv[1]);
  return u;
}

// Every kExpEmuPeriod-th pair of softmax exponentials (d = 128; kExpEmuPeriodD64 at
// d = 64) is evaluated with the FMA-pipe polynomial instead of the MUFU unit.  MUFU
// delivers 4 exp2 per clock per SM sub-partition; the polynomial costs more issue slots
// per result, so the best share is measured: every 16th pair at d = 128 (every 6th, 8th,
// 12th and 24th were slower, none at all within 0.2 %), every 4th at d = 64 (every 3rd,
// 6th and 8th slower).
constexpr int kExpEmuPeriod = 16;
constexpr int kExpEmuPeriodD64 = 4;
template <int kPeriod>
__device__ __forceinline__ constexpr bool emu_pair(int pair) {
  static_assert(kPeriod > 0, "emulation period");
  return (pair % kPeriod) == kPeriod - 1;
}

// Max over one 64-column half of an S row (columns 64*kHalf + c), sign-flipped for a
// negative scale, restricted to columns < lim when kMask; four 3-input max chains.
template <bool kMask, bool kNeg, int kHalf>
__device__ __forceinline__ float half_max(const uint32_t (&h)[2][32], int lim) {
  float m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float s0 = __uint_as_float(h[c >> 5][c & 31]);
    float s1 = __uint_as_float(h[(c + 1) >> 5][(c + 1) & 31]);
    if (kNeg) {
      s0 = -s0;
      s1 = -s1;
    }
    if (kMask) {
      s0 = (64 * kHalf + c) < lim ? s0 : -INFINITY;
      s1 = (64 * kHalf + c + 1) < lim ? s1 : -INFINITY;
    }
    m[(c >> 1) & 3] = fmax3(m[(c >> 1) & 3], s0, s1);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Sum of the eight partial row sums of the softmax (four pairs of accumulators).
__device__ __forceinline__ float sum8(const float (&acc)[4][2]) {
  return ((acc[0][0] + acc[0][1]) + (acc[1][0] + acc[1][1])) +
         ((acc[2][0] + acc[2][1]) + (acc[3][0] + acc[3][1]));
}

// p = 2^(cs * s - m_use) for one 64-column half (0 at columns >= lim when kMask),
// packed into 32 fp16 pairs (pk[c / 2], low half = even column c of the half).
// Returns the half's row sum, taken over the fp16-rounded p.  Unmasked halves run on
// the packed fp32x2 pipe.
template <bool kMask, int kHalf>
__device__ __forceinline__ float half_exp_pack(const uint32_t (&h)[2][32], float cs, float m_use,
                                               int lim, uint32_t (&pk)[32]) {
  float acc[4][2] = {};
  if constexpr (!kMask) {
    const uint64_t cs2 = f2_make(cs, cs), negm2 = f2_make(-m_use, -m_use);
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
      const uint64_t x2 = f2_fma(f2_make(__uint_as_float(h[c >> 5][c & 31]),
                                         __uint_as_float(h[(c + 1) >> 5][(c + 1) & 31])),
                                 cs2, negm2);
      float2 pp;
      if (emu_pair<kExpEmuPeriod>(c >> 1)) {
        pp = exp2_poly2(x2);
      } else {
        const float2 x = f2_split(x2);
        pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
      pk[c >> 1] = pack2<false>(pp.x, pp.y);
      add_f16x2_f32(acc[(c >> 1) & 3][0], acc[(c >> 1) & 3][1], pk[c >> 1]);
    }
  } else {
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
      const float x0 = fmaf(__uint_as_float(h[c >> 5][c & 31]), cs, -m_use);
      const float x1 = fmaf(__uint_as_float(h[(c + 1) >> 5][(c + 1) & 31]), cs, -m_use);
      const float p0 = (64 * kHalf + c) < lim ? ex2_approx(x0) : 0.f;
      const float p1 = (64 * kHalf + c + 1) < lim ? ex2_approx(x1) : 0.f;
      pk[c >> 1] = pack2<false>(p0, p1);
      add_f16x2_f32(acc[(c >> 1) & 3][0], acc[(c >> 1) & 3][1], pk[c >> 1]);
    }
  }
  return sum8(acc);
}

// Unmasked half row (64 columns, registers h) against the running max m_use: packs
// p = 2^(cs * s - m_use) into 32 fp16 pairs and returns the half's row sum (of the rounded p); xmax
// gets the largest exponent cs * s - m_use seen (the caller redoes the tile if it exceeds 8).
__device__ __forceinline__ float half_exp_pack_spec(const uint32_t (&h)[2][32], float cs, float m_use,
                                                    uint32_t (&pk)[32], float& xmax) {
  float acc[4][2] = {};
  float mx[2] = {xmax, -INFINITY};
  const uint64_t cs2 = f2_make(cs, cs), negm2 = f2_make(-m_use, -m_use);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const uint64_t x2 = f2_fma(f2_make(__uint_as_float(h[c >> 5][c & 31]),
                                       __uint_as_float(h[(c + 1) >> 5][(c + 1) & 31])),
                               cs2, negm2);
    const float2 x = f2_split(x2);
    mx[(c >> 1) & 1] = fmax3(mx[(c >> 1) & 1], x.x, x.y);
    float2 pp;
    if (emu_pair<kExpEmuPeriod>(c >> 1)) {
      pp = exp2_poly2(x2);
    } else {
      pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    }
    pk[c >> 1] = pack2<false>(pp.x, pp.y);
    add_f16x2_f32(acc[(c >> 1) & 3][0], acc[(c >> 1) & 3][1], pk[c >> 1]);
  }
  xmax = fmaxf(mx[0], mx[1]);
  return sum8(acc);
}

// Max over the 128 scores of an S row (sign-flipped for a negative scale),
// restricted to columns < lim when kMask; four 3-input max chains.
template <bool kMask, bool kNeg>
__device__ __forceinline__ float row_max(const uint32_t (&sr)[4][32], int lim) {
  float m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 128; c += 2) {
    float s0 = __uint_as_float(sr[c >> 5][c & 31]);
    float s1 = __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31]);
    if (kNeg) {
      s0 = -s0;
      s1 = -s1;
    }
    if (kMask) {
      s0 = c < lim ? s0 : -INFINITY;
      s1 = c + 1 < lim ? s1 : -INFINITY;
    }
    m[(c >> 1) & 3] = fmax3(m[(c >> 1) & 3], s0, s1);
  }
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// p for the column pair (c, c+1): 2^(cs * s - m_use); the FMA-pipe polynomial for every
// kExpEmuPeriodD64-th pair, MUFU ex2 otherwise; 0 at columns >= lim when kMask.
template <bool kMask>
__device__ __forceinline__ float2 pair_exp(const uint32_t (&sr)[4][32], int c, uint64_t cs2,
                                           uint64_t negm2, int lim) {
  const uint64_t x2 = f2_fma(f2_make(__uint_as_float(sr[c >> 5][c & 31]),
                                     __uint_as_float(sr[(c + 1) >> 5][(c + 1) & 31])),
                             cs2, negm2);
  float2 pp;
  if (!kMask && emu_pair<kExpEmuPeriodD64>(c >> 1)) {
    pp = exp2_poly2(x2);
  } else {
    const float2 x = f2_split(x2);
    pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
  }
  if (kMask) {
    pp.x = c < lim ? pp.x : 0.f;
    pp.y = c + 1 < lim ? pp.y : 0.f;
  }
  return pp;
}

// The 128 p values of the row, packed to fp16 pairs, stored into 64 TMEM columns at
// tP (lane = row) in four 16-column pieces.  Returns the row sum of the fp16-rounded p.
template <bool kMask>
__device__ __forceinline__ float row_exp_to_tmem(const uint32_t (&sr)[4][32], float cs, float m_use,
                                                 int lim, uint32_t tP) {
  const uint64_t cs2 = f2_make(cs, cs), negm2 = f2_make(-m_use, -m_use);
  float acc[4][2] = {};
#pragma unroll
  for (int q32 = 0; q32 < 4; ++q32) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = q32 * 32 + 2 * i;
      const float2 pp = pair_exp<kMask>(sr, c, cs2, negm2, lim);
      w[i] = pack2<false>(pp.x, pp.y);
      add_f16x2_f32(acc[i & 3][0], acc[i & 3][1], w[i]);
    }
    tmem_st16(tP + q32 * 16, w);
  }
  return sum8(acc);
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* unit_slot = reinterpret_cast<volatile int*>(tmem_slot + 4);  // [2][kUnitInts]
  const uint32_t clc_resp = sbase + C::kOffBar + C::kOffClc;
  auto BAR = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wctx{abort_flag, p.status, p.timeout_ns};

  // ---- one-time setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::kBarQFull + i), 1);
      mbar_init(BAR(C::kBarQEmpty + i), 1);
      mbar_init(BAR(C::kBarSFull + i), 1);
      mbar_init(BAR(C::kBarSFree + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarPFull + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarPVDone + i), 1);
      mbar_init(BAR(C::kBarUnitFull + i), 1);
      mbar_init(BAR(C::kBarUnitEmpty + i), C::kUnitReaders);
      mbar_init(BAR(C::kBarOStage + i), 1);
      mbar_init(BAR(C::kBarOReady + i), 4);  // one arrive per softmax warp
      mbar_init(BAR(C::kBarOFree + i), 1);
      mbar_init(BAR(C::kBarPHalf + i), 4);  // one arrive per softmax warp
    }
    mbar_init(BAR(C::kBarMmaDone), 1);
    mbar_init(BAR(C::kBarClc), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(BAR(C::kBarKVFull + s), 1);
      // bf16: the two converter warps also observe and release every ring item, so no
      // waiter on these barriers can ever be two phases behind or ahead
      mbar_init(BAR(C::kBarKVEmpty + s), BF16 ? 3 : 1);
      mbar_init(BAR(C::kBarVConv + s), 2);  // one arrive per converter warp, every ring item
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

  // Every role walks the same unit sequence, decoded and published by the producer.
  // Returns the k-th unit (nmax < 0: no more) after this warp has read it and released
  // its slot.
  auto next_unit = [&](int k) -> PrefillUnit {
    mbar_wait_inline(BAR(C::kBarUnitFull + (k & 1)), (k >> 1) & 1, wctx);
    __syncwarp();
    const volatile int* us = unit_slot + (k & 1) * kUnitInts;
    PrefillUnit u;
    u.id = us[0];
    u.b = us[1];
    u.h = us[2];
    u.row0[0] = us[3];
    u.row0[1] = us[4];
    u.nkv[0] = us[5];
    u.nkv[1] = us[6];
    u.nmax = us[7];
    __syncwarp();
    if (lane == 0) mbar_arrive(BAR(C::kBarUnitEmpty + (k & 1)));
    return u;
  };

  static_assert(C::kProducerWarp == 8 && C::kMmaWarp == 9 && C::kConvWarp0 == 10 && C::kThreads == 384,
                "warpgroup 2 = producer, MMA issuer, two converter warps");
  // Roles.  setmaxnreg must dominate the code it governs, so each warpgroup's re-balance
  // (d = 64) opens its branch and the return to the launch's count closes it.
  if (warp >= C::kProducerWarp) {
    // warpgroup 2: producer, MMA issuer, converters
    if constexpr (C::kDecoupled) warpgroup_reg_dealloc<C::kRegsAux>();
    if (warp == C::kProducerWarp) {
      // ======================= producer: unit claims + TMA loads ======================
      if (lane == 0) {
        tma_prefetch_map(&p.tm_q);
        tma_prefetch_map(&p.tm_k);
        tma_prefetch_map(&p.tm_v);
        tma_prefetch_map(&p.tm_o);
      }
      __syncwarp();
      int unit = blockIdx.x;  // the first unit is this CTA's own
      int nq[2] = {0, 0};     // Q loads issued per tile
      bool q_pending[2] = {false, false};
      int g = 0;              // ring items issued
      int nclaim = 0;
      for (int k = 0;; ++k) {
        PrefillUnit u;
        if (unit >= 0) {
          u = prefill_unit(p, unit);
        } else {
          u.id = -1;
          u.b = u.h = u.row0[0] = u.row0[1] = u.nkv[0] = u.nkv[1] = 0;
          u.nmax = -1;
        }
        if (k >= 2) mbar_wait_inline(BAR(C::kBarUnitEmpty + (k & 1)), ((k >> 1) - 1) & 1, wctx);
        __syncwarp();
        if (lane == 0) {
          volatile int* us = unit_slot + (k & 1) * kUnitInts;
          us[0] = u.id;
          us[1] = u.b;
          us[2] = u.h;
          us[3] = u.row0[0];
          us[4] = u.row0[1];
          us[5] = u.nkv[0];
          us[6] = u.nkv[1];
          us[7] = u.nmax;
          mbar_arrive(BAR(C::kBarUnitFull + (k & 1)));
        }
        __syncwarp();
        if (unit < 0) break;
        // The next unit is claimed late in this one (kClaimLead ring items before its last
        // load), so units go to the CTAs that are about to run out of work: claiming a
        // whole unit ahead leaves a tail of up to one long causal unit between SMs.
        bool claimed = false;
        const int claim_at = max(0, 2 * u.nmax - C::kClaimLead);
        auto claim_next = [&]() {
          if (!claimed && !warp_flag(abort_flag)) {
            mbar_arrive_expect_tx_w(BAR(C::kBarClc), 16);
            clc_try_cancel_w(clc_resp, BAR(C::kBarClc));
            claimed = true;
          }
        };
        for (int t = 0; t < 2; ++t) {
          if (u.nkv[t] == 0) continue;
          if (nq[t] > 0) mbar_wait_inline(BAR(C::kBarQEmpty + t), (nq[t] - 1) & 1, wctx);
          __syncwarp();
          if (!(p.inject == 1 && t == 0) && !warp_flag(abort_flag)) {
            mbar_arrive_expect_tx_w(BAR(C::kBarQFull + t), C::kTileBytes);
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_4d_w(sbase + C::kOffQ + t * C::kTileBytes + bx * C::kBoxBytes, &p.tm_q,
                            BAR(C::kBarQFull + t), bx * 64, u.h, u.row0[t], u.b);
            q_pending[t] = true;
          }
          ++nq[t];
        }
        for (int i = 0; i < 2 * u.nmax; ++i, ++g) {
          if (i == claim_at) claim_next();
          const int stage = g % C::kStages;
          const int round = g / C::kStages;
          if (round > 0) mbar_wait_inline(BAR(C::kBarKVEmpty + stage), (round - 1) & 1, wctx);
          __syncwarp();
          if (warp_flag(abort_flag)) continue;
          mbar_arrive_expect_tx_w(BAR(C::kBarKVFull + stage), C::kTileBytes);
          const CUtensorMap* map = (i & 1) ? &p.tm_v : &p.tm_k;
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_4d_w(sbase + C::kOffKV + stage * C::kTileBytes + bx * C::kBoxBytes, map,
                          BAR(C::kBarKVFull + stage), bx * 64, u.h, (i >> 1) * 128, u.b);
        }
        claim_next();  // units without K/V tiles
        int next = -1;
        if (claimed) {
          if (mbar_wait_inline(BAR(C::kBarClc), nclaim & 1, wctx)) next = clc_response_ctaid_x(clc_resp);
          else mbar_wait_drain_inline(BAR(C::kBarClc), nclaim & 1, p.timeout_ns);
          ++nclaim;
        }
        __syncwarp();
        unit = __shfl_sync(0xffffffffu, next, 0);
      }
      if (warp_flag(abort_flag)) {
        // Let every copy this warp started land before the CTA can exit.
        for (int t = 0; t < 2; ++t)
          if (q_pending[t]) mbar_wait_drain_inline(BAR(C::kBarQFull + t), (nq[t] - 1) & 1, p.timeout_ns);
        const int first = g > C::kStages ? g - C::kStages : 0;
        for (int i = first; i < g; ++i)
          mbar_wait_drain_inline(BAR(C::kBarKVFull + i % C::kStages), (i / C::kStages) & 1, p.timeout_ns);
        __syncwarp();
      }
    } else if (warp == C::kMmaWarp) {
      if constexpr (C::kDecoupled) {
      // ======================= tcgen05 MMA issuer (one elected lane issues) ===========
      constexpr uint32_t idesc_s = make_idesc_f16(128, 128, BF16, false);  // Q K^T, both K-major
      // P V always runs in fp16 (bf16 V tiles are converted in shared memory first); V is MN-major
      constexpr uint32_t idesc_o = make_idesc_f16(128, D, false, true);
      const uint32_t colS[2] = {0u, 128u};
      const uint32_t colO[2] = {256u, 256u + D};
      const uint32_t sQ[2] = {sbase + C::kOffQ, sbase + C::kOffQ + C::kTileBytes};
      // S_t = Q_t K_j^T: the D / 16 = 4 k-steps of 16 elements (32 bytes apart inside the
      // 128-byte swizzle rows of one box), issued in one batch.
      static_assert(D == 64, "the decoupled pipeline runs at head_dim 64");
      auto issue_s = [&](int t, uint32_t sK) {
        mma_f16_ss_k64_w(tmem + colS[t], make_sdesc_sw128(sQ[t], 16, 1024), make_sdesc_sw128(sK, 16, 1024),
                         idesc_s, 0u);
      };
      // O_t += P_t V_j over 8 k-steps of 16 keys (P_t in its own TMEM columns), issued in two
      // batches of four.
      auto issue_pv = [&](int t, uint32_t sV, bool accumulate_first) {
        mma_f16_ts_k64_w<2048>(tmem + colO[t], tmem + C::kColP + 64 * t,
                               make_sdesc_sw128(sV, C::kBoxBytes, 1024), idesc_o, accumulate_first ? 1u : 0u);
        mma_f16_ts_k64_w<2048>(tmem + colO[t], tmem + C::kColP + 64 * t + 32,
                               make_sdesc_sw128(sV + 4 * 2048, C::kBoxBytes, 1024), idesc_o, 1u);
      };
      auto stage_addr = [&](int item) -> uint32_t {
        return sbase + C::kOffKV + (item % C::kStages) * C::kTileBytes;
      };
      int nq[2] = {0, 0};   // units seen per tile (q_full / q_empty phases)
      int nsf[2] = {0, 0};  // S tiles released by the softmax (s_free phases)
      int npf[2] = {0, 0};  // P tiles written by the softmax (p_full phases)
      int g = 0;            // ring items consumed
      for (int k = 0;; ++k) {
        const PrefillUnit u = next_unit(k);
        if (u.nmax < 0) break;
        if (u.nmax == 0) continue;
        for (int t = 0; t < 2; ++t)
          if (u.nkv[t] > 0) mbar_wait_inline(BAR(C::kBarQFull + t), nq[t] & 1, wctx);
        // prologue: S_t(0) for both tiles from K_0
        mbar_wait_inline(BAR(C::kBarKVFull + g % C::kStages), (g / C::kStages) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        if (!warp_flag(abort_flag)) {
          for (int t = 0; t < 2; ++t)
            if (u.nkv[t] > 0) {
              issue_s(t, stage_addr(g));
              tc_commit_w(BAR(C::kBarSFull + t));
              if (u.nkv[t] == 1) tc_commit_w(BAR(C::kBarQEmpty + t));
            }
          tc_commit_w(BAR(C::kBarKVEmpty + g % C::kStages));
        }
        for (int j = 0; j < u.nmax; ++j) {
          // next score tiles: S_t(j+1) as soon as the softmax has read S_t(j) out of TMEM
          const int ik = g + 2 * j + 2;  // ring item of K_{j+1}
          bool k_ready = false;
          for (int t = 0; t < 2; ++t) {
            if (j >= u.nkv[t]) continue;
            mbar_wait_inline(BAR(C::kBarSFree + t), nsf[t] & 1, wctx);
            ++nsf[t];
            __syncwarp();
            if (j + 1 < u.nkv[t]) {
              if (!k_ready) {
                mbar_wait_inline(BAR(C::kBarKVFull + ik % C::kStages), (ik / C::kStages) & 1, wctx);
                __syncwarp();
                k_ready = true;
              }
              tc_fence_after_sync();
              if (warp_flag(abort_flag)) continue;
              issue_s(t, stage_addr(ik));
              tc_commit_w(BAR(C::kBarSFull + t));
              if (j + 2 == u.nkv[t]) tc_commit_w(BAR(C::kBarQEmpty + t));
            }
          }
          if (k_ready && !warp_flag(abort_flag)) tc_commit_w(BAR(C::kBarKVEmpty + ik % C::kStages));
          // O_t += P_t(j) V_j once the softmax has written P_t(j)
          const int iv = g + 2 * j + 1;  // ring item of V_j
          mbar_wait_inline(BAR((BF16 ? C::kBarVConv : C::kBarKVFull) + iv % C::kStages), (iv / C::kStages) & 1,
                    wctx);
          __syncwarp();
          for (int t = 0; t < 2; ++t) {
            if (j >= u.nkv[t]) continue;
            mbar_wait_inline(BAR(C::kBarPFull + t), npf[t] & 1, wctx);
            ++npf[t];
            __syncwarp();
            tc_fence_after_sync();
            if (warp_flag(abort_flag)) continue;
            issue_pv(t, stage_addr(iv), j > 0);
            tc_commit_w(BAR(C::kBarPVDone + t));
          }
          if (!warp_flag(abort_flag)) tc_commit_w(BAR(C::kBarKVEmpty + iv % C::kStages));
        }
        g += 2 * u.nmax;
        for (int t = 0; t < 2; ++t)
          if (u.nkv[t] > 0) ++nq[t];
      }
      // every MMA (and every commit arrive) has landed before TMEM is released
      tc_commit_w(BAR(C::kBarMmaDone));
      mbar_wait_drain_inline(BAR(C::kBarMmaDone), 0, p.timeout_ns);
      __syncwarp();
      } else {
      // ======================= tcgen05 MMA issuer (one elected lane issues) ===========
      constexpr uint32_t idesc_s = make_idesc_f16(128, 128, BF16, false);  // Q K^T, both K-major
      // P V always runs in fp16 (bf16 V tiles are converted in shared memory first); V is MN-major
      constexpr uint32_t idesc_o = make_idesc_f16(128, D, false, true);
      const uint32_t colS[2] = {0u, 128u};
      const uint32_t colO[2] = {256u, 256u + D};
      const uint32_t sQ[2] = {sbase + C::kOffQ, sbase + C::kOffQ + C::kTileBytes};
      // S_t = Q_t K_j^T over D/16 k-steps of 16 elements (32 bytes inside a 128-byte swizzle row).
      // S_t = Q_t K_j^T: 8 k-steps of 16 elements, issued in one batch.
      auto issue_s = [&](int t, uint32_t sK) {
        mma_f16_ss_k128_w<C::kBoxBytes>(tmem + colS[t], make_sdesc_sw128(sQ[t], 16, 1024),
                                        make_sdesc_sw128(sK, 16, 1024), idesc_s, 0u);
      };
      // k-steps kk0 .. kk0+3 of O_t += P_t V_j (keys 16*kk0 .. 16*kk0+63; P_t is in TMEM
      // columns [64,128) of S_t), issued in one batch; the first k-step of the unit starts
      // the accumulator.
      auto issue_pv4 = [&](int t, uint32_t sV, int kk0, bool accumulate_first) {
        mma_f16_ts_k64_w<2048>(tmem + colO[t], tmem + colS[t] + 64 + kk0 * 8,
                               make_sdesc_sw128(sV + kk0 * 2048, C::kBoxBytes, 1024), idesc_o,
                               accumulate_first ? 1u : 0u);
      };
      auto stage_addr = [&](int item) -> uint32_t {
        return sbase + C::kOffKV + (item % C::kStages) * C::kTileBytes;
      };
      int nq[2] = {0, 0};  // units seen per tile (q_full / q_empty phases)
      int np[2] = {0, 0};  // P tiles consumed per tile (p_ready phases)
      int g = 0;           // ring items consumed
      for (int k = 0;; ++k) {
        const PrefillUnit u = next_unit(k);
        if (u.nmax < 0) break;
        if (u.nmax == 0) continue;
        for (int t = 0; t < 2; ++t)
          if (u.nkv[t] > 0) mbar_wait_inline(BAR(C::kBarQFull + t), nq[t] & 1, wctx);
        // prologue: S_t(0) for both tiles from K_0
        mbar_wait_inline(BAR(C::kBarKVFull + g % C::kStages), (g / C::kStages) & 1, wctx);
        __syncwarp();
        tc_fence_after_sync();
        if (!warp_flag(abort_flag)) {
          for (int t = 0; t < 2; ++t)
            if (u.nkv[t] > 0) {
              issue_s(t, stage_addr(g));
              tc_commit_w(BAR(C::kBarSFull + t));
              if (u.nkv[t] == 1) tc_commit_w(BAR(C::kBarQEmpty + t));
            }
          tc_commit_w(BAR(C::kBarKVEmpty + g % C::kStages));
        }
        for (int j = 0; j < u.nmax; ++j) {
          const int iv = g + 2 * j + 1;  // ring item of V_j
          mbar_wait_inline(BAR((BF16 ? C::kBarVConv : C::kBarKVFull) + iv % C::kStages), (iv / C::kStages) & 1,
                    wctx);
          __syncwarp();
          const int ik = g + 2 * j + 2;  // ring item of K_{j+1}
          bool k_ready = false;
          for (int t = 0; t < 2; ++t) {
            if (j >= u.nkv[t]) continue;
            // keys 64..127 as soon as that half of P_t(j) is written, then keys 0..63
            mbar_wait_inline(BAR(C::kBarPHalf + t), np[t] & 1, wctx);
            __syncwarp();
            tc_fence_after_sync();
            if (!warp_flag(abort_flag)) issue_pv4(t, stage_addr(iv), 4, j > 0);
            mbar_wait_inline(BAR(C::kBarPFull + t), np[t] & 1, wctx);
            ++np[t];
            __syncwarp();
            tc_fence_after_sync();
            if (warp_flag(abort_flag)) continue;
            issue_pv4(t, stage_addr(iv), 0, true);
            if (j + 1 < u.nkv[t]) {
              if (!k_ready) {
                mbar_wait_inline(BAR(C::kBarKVFull + ik % C::kStages), (ik / C::kStages) & 1, wctx);
                __syncwarp();
                k_ready = true;
              }
              if (warp_flag(abort_flag)) continue;
              issue_s(t, stage_addr(ik));
              tc_commit_w(BAR(C::kBarSFull + t));
              if (j + 2 == u.nkv[t]) tc_commit_w(BAR(C::kBarQEmpty + t));
            } else {
              tc_commit_w(BAR(C::kBarPVDone + t));
            }
          }
          if (!warp_flag(abort_flag)) {
            tc_commit_w(BAR(C::kBarKVEmpty + iv % C::kStages));
            if (k_ready) tc_commit_w(BAR(C::kBarKVEmpty + ik % C::kStages));
          }
        }
        g += 2 * u.nmax;
        for (int t = 0; t < 2; ++t)
          if (u.nkv[t] > 0) ++nq[t];
      }
      // every MMA (and every commit arrive) has landed before TMEM is released
      tc_commit_w(BAR(C::kBarMmaDone));
      mbar_wait_drain_inline(BAR(C::kBarMmaDone), 0, p.timeout_ns);
      __syncwarp();
      }
    } else if (warp >= C::kConvWarp0) {
      // ======================= bf16 -> fp16 conversion of V tiles (bf16 inputs) ======
      // Walks every ring item in order: waits for it to land, converts it if it is a V
      // tile, then arrives on its v_conv barrier (the MMA issuer waits on that for V
      // tiles) and on its empty barrier (the producer refills a stage only after both the
      // tensor core and the converters are done with it).
      // A V element of magnitude 65536 or more (or inf / NaN) has no fp16 value: the
      // largest magnitude bit pattern met is tracked per thread and, if any such element
      // was converted, the call's status word records kStatusRange.
      const int ct = threadIdx.x - C::kConvWarp0 * 32;  // 0..63
      uint32_t vmag = 0;  // per-halfword max of |bf16 bits| over every V element converted
      int g = 0;
      for (int k = 0;; ++k) {
        const PrefillUnit u = next_unit(k);
        if (u.nmax < 0) break;
        if constexpr (BF16) {
          for (int i = 0; i < 2 * u.nmax; ++i) {
            const int item = g + i;
            const int st = item % C::kStages;
            mbar_wait_inline(BAR(C::kBarKVFull + st), (item / C::kStages) & 1, wctx);
            __syncwarp();
            if (i & 1) {
              uint4* tile = reinterpret_cast<uint4*>(smem + C::kOffKV + st * C::kTileBytes);
#pragma unroll 4
              for (int c = ct; c < C::kTileBytes / 16; c += 64) {
                uint4 w = tile[c];
                vmag = __vmaxu2(vmag, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                               __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
                w.x = bf16x2_to_f16x2_sat(w.x);
                w.y = bf16x2_to_f16x2_sat(w.y);
                w.z = bf16x2_to_f16x2_sat(w.z);
                w.w = bf16x2_to_f16x2_sat(w.w);
                tile[c] = w;
              }
              fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
            }
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(BAR(C::kBarVConv + st));
              mbar_arrive(BAR(C::kBarKVEmpty + st));
            }
          }
        }
        g += 2 * u.nmax;
      }
      if (max(vmag & 0xFFFFu, vmag >> 16) >= kBf16NoF16) atomicCAS(p.status, 0, kStatusRange);
    }
    // back to the launch's registers (waits until the softmax warps have given theirs back)
    __syncwarp();
    if constexpr (C::kDecoupled) warpgroup_reg_alloc<C::kLaunchRegs>();
  } else {
    // warpgroups 0 and 1: softmax
    if constexpr (C::kDecoupled) warpgroup_reg_alloc<C::kRegsSoftmax>();
    if constexpr (C::kDecoupled) {
    // ======================= softmax warpgroups (warps 0-3: tile 0, 4-7: tile 1) ======
    const int t = warp >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;  // row inside the Q tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? 128u : 0u);
    const uint32_t tO = tmem + lane_base + (t ? 256u + D : 256u);
    const uint32_t tP = tmem + lane_base + C::kColP + 64u * t;  // d = 64 only
    const float cs = p.scale_log2;
    const bool neg = cs < 0.f;
    const float cs_abs = fabsf(cs);
    const long long diag = (long long)p.Nk - p.Nq;
    uint8_t* ptile = smem + C::kOffO + t * C::kTileBytes;  // O staging of tile t
    int ns = 0;   // S tiles consumed (s_full phases)
    int npv = 0;  // P V operations of this tile completed before the current unit (pv_done phases)
    int nout = 0;  // O tiles stored (o_free / o_ready phases)
    for (int k = 0;; ++k) {
      const PrefillUnit u = next_unit(k);
      if (u.nmax < 0) break;
      const int row0 = u.row0[t];
      const int nkv = u.nkv[t];
      const int grow = row0 + r;  // global query row
      if (nkv == 0) {
        // every row of this tile is left without a key (causal, Nq > Nk): O = 0, lse = -inf
        if (row0 < p.Nq && grow < p.Nq) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) +
                                                ((((long long)u.b * p.Nq + grow) * p.H + u.h) * D) * 2);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[((long long)u.b * p.H + u.h) * p.Nq + grow] = -INFINITY;
        }
        continue;
      }

      float m_run = -INFINITY;  // running max of scale*log2(e)*s (lazy: may lag the true max by <= 8)
      float l_run = 0.f;        // running sum of 2^(cs*s - m_run)
      for (int j = 0; j < nkv; ++j) {
        mbar_wait_inline(BAR(C::kBarSFull + t), ns & 1, wctx);
        ++ns;
        __syncwarp();  // lanes may leave the bounded wait on different polls
        tc_fence_after_sync();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_order_after_wait(sr[c]);
        // S_t is in registers: the tensor core may compute S_t(j+1) into the same columns
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarSFree + t));

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
        const float mx = need_mask ? (neg ? row_max<true, true>(sr, lim) : row_max<true, false>(sr, lim))
                                   : (neg ? row_max<false, true>(sr, lim) : row_max<false, false>(sr, lim));
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * cs_abs;
        const float m_new = fmaxf(m_run, m_tile);
        const bool rescale = m_new > m_run + 8.0f;
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
        if (rescale) {
          m_run = m_new;
          l_run *= alpha;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;

        if (j > 0) {
          // P_t(j-1) V must be done: its P buffer is about to be overwritten and O_t may be rescaled
          mbar_wait_inline(BAR(C::kBarPVDone + t), (npv + j - 1) & 1, wctx);
          __syncwarp();
          tc_fence_after_sync();
          if (__any_sync(0xffffffffu, rescale)) {  // lazy rescale of O (rare after the first tiles)
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
        }

        l_run += need_mask ? row_exp_to_tmem<true>(sr, cs, m_use, lim, tP)
                           : row_exp_to_tmem<false>(sr, cs, m_use, lim, tP);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarPFull + t));
      }

      // ---- epilogue: O / l -> 16-bit -> swizzled staging (this tile's buffer) -> TMA store
      mbar_wait_inline(BAR(C::kBarPVDone + t), (npv + nkv - 1) & 1, wctx);
      npv += nkv;
      __syncwarp();
      tc_fence_after_sync();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint32_t o[D / 32][32];  // the whole O row: one TMEM round trip
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o[c]);
      // this tile's previous O store has read the staging buffer before it is rewritten
      if (r == 0) {
        bulk_wait_group_read0();
        mbar_arrive(BAR(C::kBarOFree + t));
      }
      mbar_wait_inline(BAR(C::kBarOFree + t), nout & 1, wctx);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) reg_order_after_wait(o[c]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // four 16-byte chunks of 8 elements
          uint4 w;
          w.x = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 0]) * inv_l, __uint_as_float(o[c][q4 * 8 + 1]) * inv_l);
          w.y = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 2]) * inv_l, __uint_as_float(o[c][q4 * 8 + 3]) * inv_l);
          w.z = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 4]) * inv_l, __uint_as_float(o[c][q4 * 8 + 5]) * inv_l);
          w.w = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 6]) * inv_l, __uint_as_float(o[c][q4 * 8 + 7]) * inv_l);
          const int chunk = c * 4 + q4;  // 16-byte chunk index along the row
          const int bx = chunk >> 3, cc = chunk & 7;
          *reinterpret_cast<uint4*>(ptile + bx * C::kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = w;
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the TMA store
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::kBarOReady + t));
      if (quarter == 0) {
        mbar_wait_inline(BAR(C::kBarOReady + t), nout & 1, wctx);
        if (r == 0 && !*abort_flag) {
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_store_4d(&p.tm_o, sbase + C::kOffO + t * C::kTileBytes + bx * C::kBoxBytes, bx * 64,
                         u.h, row0, u.b);
          bulk_commit_group();
        }
      }
      ++nout;
      if (p.lse != nullptr && grow < p.Nq) {
        const float lse = l_run > 0.f ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f
                                      : -INFINITY;
        p.lse[((long long)u.b * p.H + u.h) * p.Nq + grow] = lse;
      }
    }
    if (r == 0) bulk_wait_group_read0();  // the last O store has read the staging buffer
    } else {
    // ======================= softmax warpgroups (warps 0-3: tile 0, 4-7: tile 1) ======
    const int t = warp >> 2;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;  // row inside the Q tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + (t ? 128u : 0u);
    const uint32_t tO = tmem + lane_base + (t ? 256u + D : 256u);
    const float cs = p.scale_log2;
    const bool neg = cs < 0.f;
    const float cs_abs = fabsf(cs);
    const long long diag = (long long)p.Nk - p.Nq;
    uint8_t* ostage = smem + C::kOffO;
    // The two tiles take turns with the one O staging buffer, in the order tile 0 of
    // unit 0, tile 1 of unit 0, tile 0 of unit 1, ...: a turn starts when the previous
    // turn's TMA store has finished reading the buffer (an inactive tile passes its turn).
    auto ostage_acquire = [&](int k) {
      if (t == 0 && k > 0) mbar_wait_inline(BAR(C::kBarOStage + 1), (k - 1) & 1, wctx);
      if (t == 1) mbar_wait_inline(BAR(C::kBarOStage + 0), k & 1, wctx);
      __syncwarp();
    };
    int ns = 0;  // S tiles consumed (s_full phases)
    int no = 0;  // units finished (o_full phases)
    bool store_pending = false;  // (row 0's thread) this tile's last O store may still read the buffer
    for (int k = 0;; ++k) {
      const PrefillUnit u = next_unit(k);
      // The store issued at the end of the previous unit has had the unit switch to read
      // the staging buffer; only now does row 0's thread wait for it and pass the turn on.
      if (r == 0 && store_pending) {
        bulk_wait_group_read0();
        mbar_arrive(BAR(C::kBarOStage + t));
        store_pending = false;
      }
      if (u.nmax < 0) break;
      const int row0 = u.row0[t];
      const int nkv = u.nkv[t];
      const int grow = row0 + r;  // global query row
      if (nkv == 0) {
        ostage_acquire(k);  // pass this tile's turn with the staging buffer
        if (threadIdx.x == 128 * t) mbar_arrive(BAR(C::kBarOStage + t));
        // every row of this tile is left without a key (causal, Nq > Nk): O = 0, lse = -inf
        if (row0 < p.Nq && grow < p.Nq) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) +
                                                ((((long long)u.b * p.Nq + grow) * p.H + u.h) * D) * 2);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[((long long)u.b * p.H + u.h) * p.Nq + grow] = -INFINITY;
        }
        continue;
      }

      float m_run = -INFINITY;  // running max of scale*log2(e)*s (lazy: may lag the true max by <= 8)
      float l_run = 0.f;        // running sum of 2^(cs*s - m_run)
      for (int j = 0; j < nkv; ++j) {
        mbar_wait_inline(BAR(C::kBarSFull + t), ns & 1, wctx);
        ++ns;
        __syncwarp();  // lanes may leave the bounded wait on different polls
        tc_fence_after_sync();
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

        // Speculative single pass: S read in two halves, exponentiated against m_run while
        // the tile max is found; P stays in registers and is written only if no exponent
        // exceeds 8 in any row of the warp (S is untouched until then), else the two-pass
        // path below redoes the tile.
        if (j > 0 && !need_mask && __all_sync(0xffffffffu, m_run != -INFINITY)) {
          uint32_t pk[2][32];
          float xmax = -INFINITY;
          float rs;
          {
            uint32_t sv[2][32];
            tmem_ld32(tS + 64, sv[0]);
            tmem_ld32(tS + 96, sv[1]);
            tmem_ld_wait();
            reg_order_after_wait(sv[0]);
            reg_order_after_wait(sv[1]);
            rs = half_exp_pack_spec(sv, cs, m_run, pk[1], xmax);
            tmem_ld32(tS + 0, sv[0]);
            tmem_ld32(tS + 32, sv[1]);
            tmem_ld_wait();
            reg_order_after_wait(sv[0]);
            reg_order_after_wait(sv[1]);
            rs += half_exp_pack_spec(sv, cs, m_run, pk[0], xmax);
          }
          if (!__any_sync(0xffffffffu, xmax > 8.0f)) {
            l_run += rs;
            tmem_st32(tS + 96, pk[1]);  // keys 64..127
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::kBarPHalf + t));
            tmem_st32(tS + 64, pk[0]);  // keys 0..63
            tmem_st_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(BAR(C::kBarPFull + t));
            continue;
          }
        }

        // pass 1: row max over the two 64-column halves (half 1 stays in registers)
        uint32_t hv[2][32];
        tmem_ld32(tS + 0, hv[0]);
        tmem_ld32(tS + 32, hv[1]);
        tmem_ld_wait();
        reg_order_after_wait(hv[0]);
        reg_order_after_wait(hv[1]);
        float mx = need_mask ? (neg ? half_max<true, true, 0>(hv, lim) : half_max<true, false, 0>(hv, lim))
                             : (neg ? half_max<false, true, 0>(hv, lim) : half_max<false, false, 0>(hv, lim));
        tmem_ld32(tS + 64, hv[0]);
        tmem_ld32(tS + 96, hv[1]);
        tmem_ld_wait();
        reg_order_after_wait(hv[0]);
        reg_order_after_wait(hv[1]);
        mx = fmaxf(mx, need_mask ? (neg ? half_max<true, true, 1>(hv, lim) : half_max<true, false, 1>(hv, lim))
                                 : (neg ? half_max<false, true, 1>(hv, lim) : half_max<false, false, 1>(hv, lim)));
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * cs_abs;
        const float m_new = fmaxf(m_run, m_tile);
        const bool rescale = m_new > m_run + 8.0f;
        const float alpha = rescale ? ex2_approx(m_run - m_new) : 1.0f;
        if (rescale) {
          m_run = m_new;
          l_run *= alpha;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;

        // lazy rescale of O, before any P_t(j) V_j can start (P_t(j-1) V_{j-1} completed
        // before S_t(j) did)
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

        // pass 2: P for half 1 (keys 64..127, from registers) into TMEM columns 96..127,
        // which held S columns 96..127 -- already read -- and published at once, so the
        // tensor core starts on keys 64..127 of P_t V_j; then half 0 re-read from TMEM
        // (columns 0..63, untouched) into P columns 64..95.
        uint32_t pk[32];
        float rs = need_mask ? half_exp_pack<true, 1>(hv, cs, m_use, lim, pk)
                             : half_exp_pack<false, 1>(hv, cs, m_use, lim, pk);
        __syncwarp();
        tmem_st32(tS + 96, pk);
        tmem_ld32(tS + 0, hv[0]);
        tmem_ld32(tS + 32, hv[1]);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarPHalf + t));
        tmem_ld_wait();
        reg_order_after_wait(hv[0]);
        reg_order_after_wait(hv[1]);
        rs += need_mask ? half_exp_pack<true, 0>(hv, cs, m_use, lim, pk)
                        : half_exp_pack<false, 0>(hv, cs, m_use, lim, pk);
        l_run += rs;
        __syncwarp();
        tmem_st32(tS + 64, pk);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::kBarPFull + t));
      }

      // ---- epilogue: O / l -> 16-bit -> swizzled staging buffer -> TMA store
      mbar_wait_inline(BAR(C::kBarPVDone + t), no & 1, wctx);
      ++no;
      __syncwarp();
      tc_fence_after_sync();
      ostage_acquire(k);  // the previous store from the staging buffer has read it
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      {
        uint32_t o[D / 32][32];  // the whole O row: one TMEM round trip
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o[c]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) reg_order_after_wait(o[c]);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {  // four 16-byte chunks of 8 elements
            uint4 w;
            w.x = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 0]) * inv_l, __uint_as_float(o[c][q4 * 8 + 1]) * inv_l);
            w.y = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 2]) * inv_l, __uint_as_float(o[c][q4 * 8 + 3]) * inv_l);
            w.z = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 4]) * inv_l, __uint_as_float(o[c][q4 * 8 + 5]) * inv_l);
            w.w = pack2<BF16>(__uint_as_float(o[c][q4 * 8 + 6]) * inv_l, __uint_as_float(o[c][q4 * 8 + 7]) * inv_l);
            const int chunk = c * 4 + q4;  // 16-byte chunk index along the row
            const int bx = chunk >> 3, cc = chunk & 7;
            *reinterpret_cast<uint4*>(ostage + bx * C::kBoxBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = w;
          }
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the TMA store
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::kBarOReady + t));
      if (quarter == 0) {
        mbar_wait_inline(BAR(C::kBarOReady + t), (no - 1) & 1, wctx);
        if (r == 0 && !*abort_flag) {
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_store_4d(&p.tm_o, sbase + C::kOffO + bx * C::kBoxBytes, bx * 64, u.h, row0, u.b);
          bulk_commit_group();
        }
      }
      store_pending = true;  // completed (and the turn passed on) after the next unit is read
      if (p.lse != nullptr && grow < p.Nq) {
        const float lse = l_run > 0.f ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f
                                      : -INFINITY;
        p.lse[((long long)u.b * p.H + u.h) * p.Nq + grow] = lse;
      }
    }
    }
    __syncwarp();
    if constexpr (C::kDecoupled) warpgroup_reg_dealloc<C::kLaunchRegs>();
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

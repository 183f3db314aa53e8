// Tensor-core kernel (tcgen05 / TMEM / TMA, sm_100a) for one shard's partial
// attention with its LSE over the packed fp8 row layout.
//
// What it computes is the same as the other decode kernels: for each
// request, the softmax over this shard's tokens of scale * <q_h, k_t> (576
// values) applied to the first 512 values of the rows, plus LSE = ln sum_t
// exp(score) ("GLM-5.2 vLLM Decode Context Parallelism", sections "See why
// vLLM 0.26.0 fails" and "Separate the backend merge from stable";
// round-robin ownership from "How vLLM Serves GLM-5.3 with Million-Token
// Contexts on 16 H200s", "The core design").
//
// How.  The cache rows are read by TMA straight into shared memory and the
// tensor cores consume the e4m3 codes as they are (kind::f8f6f4); no thread
// converts cache values.  Scores are exact up to fp32 accumulation order:
//  * Q (bf16, 8 significant bits) is split per head into two e4m3 terms in
//    one power-of-two frame, q * 2^a = hi + lo.  That is exact for every
//    element above 2^-9 of the head's largest (smaller ones lose low bits and
//    weigh at most 2^-9 of it).  hi and lo are two MMAs into one accumulator.
//  * Each 128-value scale group of the latent row has its own accumulator
//    (weight-stationary M = 64 heads, N = 64 tokens): codes . (hi + lo) for
//    that group.  The softmax threads multiply it by the token's fp32 group
//    scale, so the scale is applied exactly in fp32 instead of being rounded
//    into an operand.  The rope (bf16) is a fifth part with bf16 MMAs.
//  * A part takes 32 TMEM columns; eight part buffers hold more than a tile,
//    so the scores of the next tile are computed while this one's softmax
//    runs.
//  * Online softmax in base 2 with a lazily updated running max (O is only
//    rescaled when the max grows by more than 2^3).
//  * O += P V reads V as the same e4m3 codes.  The group scale multiplies P:
//    for group g, P_g = p * s_tg * (8 / S_g), stored as two e4m3 terms (a
//    Veltkamp split in fp16: hi keeps 4 leading bits, lo the rest rounded to
//    4 bits; about 8 significant bits together) in a 64 x 64 K-major tile per
//    term.  S_g is a per-request reference scale (the group's largest scale
//    in the request's first tile, raised with an exact O rescale if a later
//    tile holds a scale more than 4x larger), so P_g stays below 256 and the
//    tokens that carry the softmax mass stay in the e4m3 normal range; the
//    epilogue multiplies O_g back by S_g / 8.
//  * O (64 heads x 512, fp32) stays in TMEM for the whole request, in the
//    weight-stationary M = 64 layout (one N = 128 accumulator per group).
//
// Roles (16 warps): 0-7 softmax and epilogue (two warps per TMEM lane
// quarter, one per 16-column half), 8 TMA producer, 9 and 15 issue the score
// MMAs (parts 0, 2, 4 and parts 1, 3), 10 issues the PV MMAs, 11-14 prepare
// Q (hi / lo split) per request.  Shared
// memory: Q 72 KB, three stages of codes and scales (3 x 33 KB), two of rope
// (2 x 8 KB), P 32 KB.  Every wait is bounded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "tc_ptx.cuh"

namespace dcpmla {
namespace {

constexpr int kThreads = 512;          // 16 warps
constexpr int kSoftWarps = 8;
constexpr int kProdWarp = 8, kQkWarp = 9, kPvWarp = 10, kQWarp0 = 11, kQkWarp2 = 15;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kQThreads = 128;

constexpr uint32_t kChunk = 8192;                 // 64 rows x 128 B
constexpr int kCodeStages = 3, kRopeStages = 2;
constexpr uint32_t kCodeStage = 4 * kChunk + 1024;   // codes (4 chunks) + scales
constexpr uint32_t kScalesOff = 4 * kChunk;
constexpr uint32_t kTileBytes = 64 * kRowBytesFp8;   // 41,984 bytes land per tile
constexpr uint32_t kPVar = 4096;                  // 64 heads x 64 tokens, e4m3
constexpr uint32_t kOffQh = 0;                    // Q hi: 4 chunks of 64 rows x 128 B
constexpr uint32_t kOffQl = kOffQh + 4 * kChunk;  // Q lo
constexpr uint32_t kOffQr = kOffQl + 4 * kChunk;  // Q rope: 64 rows x 64 bf16
constexpr uint32_t kOffCode = kOffQr + kChunk;
constexpr uint32_t kOffRope = kOffCode + kCodeStages * kCodeStage;
constexpr uint32_t kOffP = kOffRope + kRopeStages * kChunk;
constexpr uint32_t kOffCtl = kOffP + 8 * kPVar;
static_assert(kOffCode % 1024 == 0 && kCodeStage % 1024 == 0 && kOffRope % 1024 == 0 &&
                  kOffP % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
static_assert(kTileBytes == 4 * kChunk + 1024 + kChunk, "a tile is codes, scales and rope");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColPart = 256;      // 8 score part buffers of 32 columns; O: [0, 256)
constexpr int kParts = 8;
constexpr int kPrefetchTiles = 6;
constexpr int kMaxSegF8 = 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 3.f;     // lazy max: rescale O when the max grows by > 2^3
constexpr float kPNorm = 8.f;           // P_g = p * s * (kPNorm / S_g)
constexpr float kScaleSlack = 4.f;      // a tile scale up to 4 S_g needs no rescale
constexpr int kFlagTimeout = 4;

// TMA box x offset inside a row: code chunks 0..3, then the rope
__device__ __forceinline__ int box_x(int k) { return k < 4 ? 128 * k : 528; }

struct F8Params {
  PartialParams p;
  CUtensorMap rows;      // [blocks][64][656] u8, box 128 x 64, 128-byte swizzle
  CUtensorMap scales;    // same tensor, box 16 x 64, no swizzle (the four fp32 scales)
};

struct F8Ctl {
  alignas(16) float sT[2][4][64];   // a tile's scales, [tile parity][group][row]
  alignas(16) __half sTp[2][4][64]; // the same times the group's P normaliser (fp16)
  float qexp[64];                   // 2^-a per head (Q frame)
  float gpart[2][kSoftWarps][4];    // per-warp group maxima of a tile's scales
  float mred[4][64];                // per-thread-column maxima of the tile's scores, and in
                                    // the epilogue the per-thread-column sums
  uint64_t full[kCodeStages];       // TMA bytes of a tile landed
  uint64_t code_empty[kCodeStages]; // PV of the slot's tile done (commit)
  uint64_t rope_empty[kRopeStages]; // rope part of the slot's tile done (commit)
  uint64_t part_full[kParts];       // score part ready (commit)
  uint64_t part_empty[kParts];      // score part read (softmax arrivals)
  uint64_t p_full;                  // P written (softmax arrivals)
  uint64_t p_empty;                 // PV done reading P (commit)
  uint64_t o_full;                  // a request's last PV done (commit)
  uint64_t q_full;                  // Q of the next request staged (Q-warp arrivals)
  uint64_t q_empty;                 // a request's last score MMA done (commit)
  int nv[kCodeStages];              // rows of the slot's tile that take part (producer)
  uint32_t tmem_base;
  int abort;
  int sel_count;
  int warp_sums[16];
  Segment seg[kMaxSegF8];
};

constexpr size_t kSmemBytes = kOffCtl + sizeof(F8Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint32_t sw128(int r, int u) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw64(int r, int u) {
  return (uint32_t)((r >> 3) * 512 + (r & 7) * 64 + (((u ^ ((r & 7) >> 1)) & 3) << 4));
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, F8Ctl& c) {
  return ptx::mbar_wait(bar, parity, &c.abort);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// two fp32 -> two e4m3 (lo -> low byte), round to nearest even, saturated
__device__ __forceinline__ uint32_t e4m3x2_f32(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// two e4m3 (low byte first) -> two fp32, exact
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t pair) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pair));
  float lo, hi;
  asm("{\n .reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;\n}\n"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
  return make_float2(lo, hi);
}

// fp16 pairs as 32-bit words, round-to-nearest arithmetic that the compiler
// may not contract into fused operations (the split below depends on every
// rounding)
__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hsub2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_rn(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint16_t f16_rn(float x) {
  uint16_t d;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(d) : "f"(x));
  return d;
}
__device__ __forceinline__ uint16_t f16_sat(float x) {
  uint16_t d;
  asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(d) : "f"(x));
  return d;
}

// fp16 pair x (P_g of two tokens, 0 <= x < 256) -> e4m3 hi and lo terms
// (2 bytes each, low byte = first token).  Veltkamp split in fp16:
// gamma = x * (2^7 + 1), hi = gamma - (gamma - x) keeps the 4 leading bits of
// x (exact for x * 129 < 65504), so its e4m3 encoding is exact in the normal
// range; lo = x - hi is exact in fp16 and rounded to 4 bits by the encoding.
__device__ __forceinline__ void split_hilo(uint32_t x, uint32_t& hi, uint32_t& lo) {
  constexpr uint32_t k129 = 0x58085808u;          // fp16 129.0 in both halves
  const uint32_t gam = hmul2_rn(x, k129);
  const uint32_t h = hsub2_rn(gam, hsub2_rn(gam, x));
  const uint32_t l = hsub2_rn(x, h);
  uint16_t eh, el;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(eh) : "r"(h));
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(el) : "r"(l));
  hi = eh;
  lo = el;
}

// ---------------------------------------------------------------- roles ----

// TMA producer (one thread): tile tau goes to code slot tau % 3 and rope
// slot tau % 2.  A tile whose table entry is out of range (flagged) loads
// block 0 instead; the softmax treats all of its rows as absent and clears
// them before PV.
__device__ void producer_role(const F8Params& P, const PartialParams& p, F8Ctl& c,
                              uint8_t* base, int nseg, uint32_t& tau,
                              uint32_t (&fills)[kCodeStages]) {
  TileCursor cur, pf;
  if (!cur.start(p, c, nseg)) return;
  pf = cur;
  bool pf_ok = true;
  for (int i = 0; i < kPrefetchTiles && pf_ok; ++i) {
    const int blk = tile_block(p, pf.v.b, (pf.v.row_begin >> 6) + pf.t);
    if (blk >= 0) ptx::prefetch_l2(p.kv + (size_t)blk * kTileBytes, kTileBytes);
    pf_ok = pf.next(p, c);
  }
  while (true) {
    const uint32_t cs = tau % kCodeStages, rs = tau % kRopeStages;
    // slot reuse: the PV of tile tau - 3 and the rope part of tile tau - 2
    if (tau >= (uint32_t)kCodeStages &&
        !wait_or_abort(&c.code_empty[cs], ((tau / kCodeStages) + 1) & 1, c))
      return;
    if (tau >= (uint32_t)kRopeStages &&
        !wait_or_abort(&c.rope_empty[rs], ((tau / kRopeStages) + 1) & 1, c))
      return;
    const int blk = tile_block(p, cur.v.b, (cur.v.row_begin >> 6) + cur.t);
    const int z = blk >= 0 ? blk : 0;
    // the softmax reads the tile's valid rows with its bytes (the arrival
    // below releases this write)
    c.nv[cs] = blk >= 0 ? cur.tile_valid_rows() : 0;
    // test only: withholding the very first tile makes every pipeline wait
    // of the CTA run out, which exercises the timeout path
    if (!(p.test_withhold && tau == 0)) {
      uint64_t* bar = &c.full[cs];
      ptx::mbar_arrive_expect_tx(bar, kTileBytes);
      const uint32_t dst = ptx::smem_addr(base + kOffCode + cs * kCodeStage);
#pragma unroll
      for (int k = 0; k < 4; ++k) ptx::tma_load_3d(dst + k * kChunk, &P.rows, box_x(k), 0, z, bar);
      ptx::tma_load_3d(dst + kScalesOff, &P.scales, 512, 0, z, bar);
      ptx::tma_load_3d(ptx::smem_addr(base + kOffRope + rs * kChunk), &P.rows, box_x(4), 0, z, bar);
      ++fills[cs];
    }
    ++tau;
    if (!cur.next(p, c)) break;
    if (pf_ok) {
      const int pb = tile_block(p, pf.v.b, (pf.v.row_begin >> 6) + pf.t);
      if (pb >= 0) ptx::prefetch_l2(p.kv + (size_t)pb * kTileBytes, kTileBytes);
      pf_ok = pf.next(p, c);
    }
  }
}

// Descriptor plus a byte offset (the start address field holds address / 16
// and never carries: shared memory is below 256 KB).
__device__ __forceinline__ uint64_t dplus(uint64_t d, uint32_t byte_off) {
  return d + (uint64_t)(byte_off >> 4);
}

// One score part: four e4m3 K-steps of 32 (hi and lo MMAs into one
// accumulator) for group kPart < 4, or four bf16 K-steps of 16 for the rope.
template <int kPart>
__device__ __forceinline__ void issue_part(uint32_t d, uint64_t dqh, uint64_t dql, uint64_t dqr,
                                           uint64_t dcode, uint64_t drope) {
  constexpr uint32_t kIdF8 = ptx::idesc_make(64, 64, 0, false, false);
  constexpr uint32_t kIdBf = ptx::idesc_make(64, 64, 1, false, false);
  if constexpr (kPart < 4) {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t bk = dplus(dcode, kPart * kChunk + ks * 32);
      ptx::mma_ws_f8(d, dplus(dqh, kPart * kChunk + ks * 32), bk, kIdF8, ks > 0);
      ptx::mma_ws_f8(d, dplus(dql, kPart * kChunk + ks * 32), bk, kIdF8, 1u);
    }
  } else {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      ptx::mma_ws_f16(d, dplus(dqr, ks * 32), dplus(drope, ks * 32), kIdBf, ks > 0);
  }
}

// Score MMAs.  Two threads share them: kSide 0 issues parts 0, 2 and 4 (the
// rope) of each tile, kSide 1 parts 1 and 3; part p of tile tau is number
// 5 tau + p and goes to part buffer (5 tau + p) % 8 (weight-stationary
// M = 64 heads, N = 64 tokens, 32 columns).
template <int kSide>
__device__ void qk_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg,
                        uint32_t& tau, uint32_t& sigma) {
  const uint64_t dqh = ptx::sdesc(ptx::smem_addr(base + kOffQh), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dql = ptx::sdesc(ptx::smem_addr(base + kOffQl), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dqr = ptx::sdesc(ptx::smem_addr(base + kOffQr), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dc0 = ptx::sdesc(ptx::smem_addr(base + kOffCode), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dr0 = ptx::sdesc(ptx::smem_addr(base + kOffRope), 16, 1024, ptx::kSwizzle128B);
  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  while (true) {
    const uint32_t cs = tau % kCodeStages, rs = tau % kRopeStages;
    if (cur.t == 0 && !wait_or_abort(&c.q_full, sigma & 1, c)) return;
    if (!wait_or_abort(&c.full[cs], (tau / kCodeStages) & 1, c)) return;
    // stay at most one tile ahead of PV: the scores of tile tau are issued
    // once the PV of tile tau - 2 is done (the release of its code slot, a
    // barrier that cannot complete its next phase before these scores), so
    // that a PV never waits behind score MMAs of tiles far ahead
    if (tau >= 2 &&
        !wait_or_abort(&c.code_empty[(tau - 2) % kCodeStages], ((tau - 2) / kCodeStages) & 1, c))
      return;
    const uint64_t dcode = dplus(dc0, cs * kCodeStage), drope = dplus(dr0, rs * kChunk);
    constexpr int kNum = kSide == 0 ? 3 : 2;
#pragma unroll
    for (int k = 0; k < kNum; ++k) {
      const int part = kSide + 2 * k;
      const uint32_t pi = 5 * tau + part, buf = pi % kParts;
      if (pi >= (uint32_t)kParts &&
          !wait_or_abort(&c.part_empty[buf], ((pi / kParts) + 1) & 1, c))
        return;
      ptx::tc_fence_after();
      const uint32_t d = c.tmem_base + kColPart + 32 * buf;
      if (kSide == 0) {
        if (k == 0) issue_part<0>(d, dqh, dql, dqr, dcode, drope);
        if (k == 1) issue_part<2>(d, dqh, dql, dqr, dcode, drope);
        if (k == 2) issue_part<4>(d, dqh, dql, dqr, dcode, drope);
      } else {
        if (k == 0) issue_part<1>(d, dqh, dql, dqr, dcode, drope);
        if (k == 1) issue_part<3>(d, dqh, dql, dqr, dcode, drope);
      }
      ptx::mma_commit(&c.part_full[buf]);
    }
    if (kSide == 0) ptx::mma_commit(&c.rope_empty[rs]);
    if (cur.last_of_segment()) {
      ptx::mma_commit(&c.q_empty);
      ++sigma;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// PV MMAs (one thread): O_g += P_g,hi V_g + P_g,lo V_g per group, weight
// stationary M = 64 heads, N = 128 values, K = 32 tokens; V_g is the code
// chunk g of the tile's slot read MN-major.
__device__ void pv_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg, uint32_t& tau,
                        uint32_t (&uses)[kCodeStages], uint32_t& o_commits) {
  constexpr uint32_t kIdPv = ptx::idesc_make(64, 128, 0, false, true);
  const uint64_t dv0 = ptx::sdesc(ptx::smem_addr(base + kOffCode), 4096, 1024, ptx::kSwizzle128B);
  const uint64_t dp = ptx::sdesc(ptx::smem_addr(base + kOffP), 16, 512, ptx::kSwizzle64B);
  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  while (true) {
    const uint32_t cs = tau % kCodeStages;
    if (!wait_or_abort(&c.p_full, tau & 1, c)) return;
    ptx::tc_fence_after();
    const uint64_t dv = dplus(dv0, cs * kCodeStage);
    const uint32_t acc0 = cur.t == 0 ? 0u : 1u;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t d = c.tmem_base + 64 * g;
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const uint64_t bv = dplus(dv, g * kChunk + ks * 4096);
        ptx::mma_ws_f8(d, dplus(dp, (2 * g) * kPVar + ks * 32), bv, kIdPv, ks == 0 ? acc0 : 1u);
        ptx::mma_ws_f8(d, dplus(dp, (2 * g + 1) * kPVar + ks * 32), bv, kIdPv, 1u);
      }
    }
    ptx::mma_commit(&c.p_empty);
    ptx::mma_commit(&c.code_empty[cs]);
    ++uses[cs];
    if (cur.last_of_segment()) {
      ptx::mma_commit(&c.o_full);
      ++o_commits;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Q of each request (128 threads): thread q handles head q / 2 and half the
// latent (256 values) and rope (32 values).  Writes the hi and lo A operands
// (64 rows each), the rope A operand and 2^-a per head.
__device__ void q_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg,
                       uint32_t& sigma) {
  const int q = threadIdx.x - kQWarp0 * 32;   // 0..127
  const int hq = q >> 1, part = q & 1;
  uint8_t* qh = base + kOffQh;
  uint8_t* ql = base + kOffQl;
  uint8_t* qr = base + kOffQr;
  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  while (true) {
    if (sigma > 0 && !wait_or_abort(&c.q_empty, (sigma - 1) & 1, c)) return;
    const bool live = hq < p.heads;
    const uint4* src = reinterpret_cast<const uint4*>(
        p.q + ((size_t)cur.v.b * p.heads + (live ? hq : 0)) * kHeadDim);
    float amax = 0.f;
#pragma unroll 4
    for (int u = 0; u < 32; ++u) {
      const uint4 v = live ? __ldg(src + part * 32 + u) : make_uint4(0, 0, 0, 0);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)),
                                 fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    // frame: q * 2^a with max |q * 2^a| in [128, 256)
    int a = 0;
    if (amax > 0.f) {
      const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
      a = min(120, max(-120, 7 - e));
    }
    const float fa = __uint_as_float((uint32_t)(127 + a) << 23);
    if (part == 0) c.qexp[hq] = __uint_as_float((uint32_t)(127 - a) << 23);
    // latent: 16 output units of 16 codes (two groups of 128 values) per term
#pragma unroll 2
    for (int uo = 0; uo < 16; ++uo) {
      const int g = 2 * part + (uo >> 3), u = uo & 7;
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint4 v = live ? __ldg(src + part * 32 + 2 * uo + k) : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          // four bf16 values -> one word of hi codes and one of lo codes
          const float f0 = __uint_as_float(w[e] << 16) * fa;
          const float f1 = __uint_as_float(w[e] & 0xFFFF0000u) * fa;
          const float f2 = __uint_as_float(w[e + 1] << 16) * fa;
          const float f3 = __uint_as_float(w[e + 1] & 0xFFFF0000u) * fa;
          const uint32_t h01 = e4m3x2_f32(f0, f1), h23 = e4m3x2_f32(f2, f3);
          const float2 b01 = e4m3x2_to_f32(h01), b23 = e4m3x2_to_f32(h23);
          const uint32_t l01 = e4m3x2_f32(f0 - b01.x, f1 - b01.y);
          const uint32_t l23 = e4m3x2_f32(f2 - b23.x, f3 - b23.y);
          hw[2 * k + e / 2] = h01 | (h23 << 16);
          lw[2 * k + e / 2] = l01 | (l23 << 16);
        }
      }
      *reinterpret_cast<uint4*>(qh + g * kChunk + sw128(hq, u)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(ql + g * kChunk + sw128(hq, u)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    // rope: 32 bf16 values = 4 units
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 v = live ? __ldg(src + 64 + part * 4 + u) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(qr + sw128(hq, part * 4 + u)) = v;
    }
    ptx::fence_proxy_async();
    ptx::mbar_arrive(&c.q_full);
    ++sigma;
    // next segment
    cur.t = cur.v.ntiles - 1;
    if (!cur.next(p, c)) break;
  }
}

// The scales of one tile, moved into the control block by the softmax
// threads: [group][row] copies (raw, and times the P normaliser of the
// current reference scales) and per-warp group maxima over the valid rows.
// Thread T moves the entry (row T / 4, group T % 4).
__device__ __forceinline__ void stage_scales(F8Ctl& c, const uint8_t* code, int nv, int buf,
                                             const float (&sref)[4], int T) {
  const int stok = T >> 2, sg = T & 3, w = T >> 5, i = T & 31;
  const float sv = *reinterpret_cast<const float*>(code + kScalesOff + stok * 16 + sg * 4);
  c.sT[buf][sg][stok] = sv;
  const float ref = sg == 0 ? sref[0] : sg == 1 ? sref[1] : sg == 2 ? sref[2] : sref[3];
  reinterpret_cast<uint16_t*>(c.sTp[buf][sg])[stok] =
      f16_sat(stok < nv ? sv * (kPNorm / ref) : 0.f);
  float m = stok < nv ? fabsf(sv) : 0.f;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (i < 4) c.gpart[buf][w][i] = m;
}

// Softmax, P and the epilogue (8 warps).  Parts and O share the weight-
// stationary M = 64 layout: TMEM lane L holds head L % 64 for the first
// (L < 64) or second half of the columns.  Warp w reads lane quarter
// q = w % 4 and the 16-column half th = w / 4 of each part, so thread (w, i)
// owns 16 tokens of head h = (32 q + i) % 64.  One named barrier per tile
// publishes the maxima of this tile and the scales of the next one.
__device__ void softmax_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg,
                             uint32_t& tau, uint32_t& sigma, uint32_t& pi) {
  const int T = threadIdx.x;                 // 0..255
  const int w = T >> 5, i = T & 31;
  const int q = w & 3, th = w >> 2;
  const int L = 32 * q + i;                  // TMEM lane
  const int h = L & 63, tq = L >> 6;         // head, token half of the part
  const int col = 2 * tq + th;               // which of the head's 4 threads this is
  const int tok0 = tq * 32 + th * 16;        // first of this thread's 16 tokens
  const uint32_t lane_base = c.tmem_base + ((uint32_t)(q * 32) << 16);
  const float sl2 = p.scale * kLog2e;
  const int odh = tq * 64 + th * 32;         // O: this thread's 32 values of each group

  // sparse CTAs whose list is empty write the neutral pair and stop
  if (p.sparse_idx && seg_view(p, c, 0).ntiles == 0) {
    const SegView v = seg_view(p, c, 0);
    const size_t slot = seg_slot(p, v);
    if (h < p.heads) {
      float* o = (v.whole ? p.out : p.ws_o) + (slot * p.heads + h) * kVDim;
      for (int g = 0; g < 4; ++g)
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(o + 128 * g + odh + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col == 0) (v.whole ? p.out_lse : p.ws_lse)[slot * p.heads + h] = -CUDART_INF_F;
    }
    return;
  }

  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  float m_used = -CUDART_INF_F, l = 0.f, kq = 0.f, two_a = 1.f;
  float sref[4] = {1.f, 1.f, 1.f, 1.f};      // reference scales of the current request
  uint8_t* pbuf = base + kOffP;
  // scales of the batch's first tile
  {
    const uint32_t cs = tau % kCodeStages;
    if (!wait_or_abort(&c.full[cs], (tau / kCodeStages) & 1, c)) return;
    stage_scales(c, base + kOffCode + cs * kCodeStage, c.nv[cs], tau & 1, sref, T);
    ptx::named_bar(1, kSoftThreads);
  }
  while (true) {
    const uint32_t cs = tau % kCodeStages;
    const int buf = tau & 1;
    uint8_t* code = base + kOffCode + cs * kCodeStage;
    const bool first_blk = cur.t == 0;
    if (first_blk) {
      if (!wait_or_abort(&c.q_full, sigma & 1, c)) return;
      const float qe = c.qexp[h];
      kq = qe * sl2;
      two_a = 1.f / qe;                      // exact: a power of two
      m_used = -CUDART_INF_F;
      l = 0.f;
    }
    // rows of the tile that take part (none if its table entry is bad: the
    // producer flagged it and loaded a stand-in block)
    const int nv = c.nv[cs];
    // ---- reference scales (S_g) of this tile.  The staged P scales were
    // made with the references of the previous tile: a request's first tile
    // restages them (one more barrier, once per request); a raised reference
    // (factor r < 1/4) is applied to P as it is formed.
    float r[4] = {1.f, 1.f, 1.f, 1.f};
    bool need_g = false;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float gm = 0.f;
#pragma unroll
      for (int k = 0; k < kSoftWarps; ++k) gm = fmaxf(gm, c.gpart[buf][k][g]);
      if (first_blk) {
        sref[g] = gm > 0.f ? gm : 1.f;
      } else if (gm > kScaleSlack * sref[g]) {
        r[g] = sref[g] / gm;
        sref[g] = gm;
        need_g = true;
      }
    }
    if (first_blk) {
      const int stok = T >> 2, sg = T & 3;
      const float ref = sg == 0 ? sref[0] : sg == 1 ? sref[1] : sg == 2 ? sref[2] : sref[3];
      reinterpret_cast<uint16_t*>(c.sTp[buf][sg])[stok] =
          f16_rn(stok < nv ? c.sT[buf][sg][stok] * (kPNorm / ref) : 0.f);
      ptx::named_bar(1, kSoftThreads);
    }
    // ---- score parts: 16 tokens of head h.  The loads of a batch of parts
    // (0-2, then 3-4) are issued back to back and waited for once.
    float x[16];
    {
      uint32_t xa[3][16];
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const uint32_t bp = (pi + part) % kParts;
        if (!wait_or_abort(&c.part_full[bp], ((pi + part) / kParts) & 1, c)) return;
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_ld16(lane_base + kColPart + 32 * bp + 16 * th, xa[part]);
      }
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
#pragma unroll
      for (int part = 0; part < 3; ++part) ptx::mbar_arrive(&c.part_empty[(pi + part) % kParts]);
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        const float4* s4 = reinterpret_cast<const float4*>(&c.sT[buf][g][tok0]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 s = s4[j];
          const float a0 = __uint_as_float(xa[g][4 * j]), a1 = __uint_as_float(xa[g][4 * j + 1]);
          const float a2 = __uint_as_float(xa[g][4 * j + 2]), a3 = __uint_as_float(xa[g][4 * j + 3]);
          x[4 * j] = g == 0 ? s.x * a0 : fmaf(s.x, a0, x[4 * j]);
          x[4 * j + 1] = g == 0 ? s.y * a1 : fmaf(s.y, a1, x[4 * j + 1]);
          x[4 * j + 2] = g == 0 ? s.z * a2 : fmaf(s.z, a2, x[4 * j + 2]);
          x[4 * j + 3] = g == 0 ? s.w * a3 : fmaf(s.w, a3, x[4 * j + 3]);
        }
      }
    }
    {
      uint32_t xb[2][16];
#pragma unroll
      for (int part = 3; part < 5; ++part) {
        const uint32_t bp = (pi + part) % kParts;
        if (!wait_or_abort(&c.part_full[bp], ((pi + part) / kParts) & 1, c)) return;
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_ld16(lane_base + kColPart + 32 * bp + 16 * th, xb[part - 3]);
      }
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
#pragma unroll
      for (int part = 3; part < 5; ++part) ptx::mbar_arrive(&c.part_empty[(pi + part) % kParts]);
      const float4* s4 = reinterpret_cast<const float4*>(&c.sT[buf][3][tok0]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 s = s4[j];
        x[4 * j] = fmaf(s.x, __uint_as_float(xb[0][4 * j]), x[4 * j]);
        x[4 * j + 1] = fmaf(s.y, __uint_as_float(xb[0][4 * j + 1]), x[4 * j + 1]);
        x[4 * j + 2] = fmaf(s.z, __uint_as_float(xb[0][4 * j + 2]), x[4 * j + 2]);
        x[4 * j + 3] = fmaf(s.w, __uint_as_float(xb[0][4 * j + 3]), x[4 * j + 3]);
      }
      // rope, brought into the Q frame: the sum is multiplied by 2^-a * scale below
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = fmaf(__uint_as_float(xb[1][j]), two_a, x[j]);
    }
    pi += 5;
    float mloc = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      x[j] = (tok0 + j < nv) ? x[j] * kq : -CUDART_INF_F;
      mloc = fmaxf(mloc, x[j]);
    }
    c.mred[col][h] = mloc;
    // ---- the next tile's scales, published by the barrier below
    {
      TileCursor nx = cur;
      if (nx.next(p, c)) {
        const uint32_t ns = (tau + 1) % kCodeStages;
        if (!wait_or_abort(&c.full[ns], ((tau + 1) / kCodeStages) & 1, c)) return;
        stage_scales(c, base + kOffCode + ns * kCodeStage, c.nv[ns], buf ^ 1, sref, T);
      }
    }
    // ---- lazy rescale of O (running max grew by > 2^3, or a group's scale
    // reference was raised); decided for the whole CTA
    const bool grow = !first_blk && mloc > m_used + kRescaleLog2;
    const bool any = ptx::named_bar_or(1, kSoftThreads, grow || need_g);
    const float mt = fmaxf(fmaxf(c.mred[0][h], c.mred[1][h]), fmaxf(c.mred[2][h], c.mred[3][h]));
    float m_new = m_used;
    if (first_blk) {
      m_used = mt;
      m_new = mt;
    } else if (mt > m_used + kRescaleLog2) {
      m_new = mt;
    }
    bool waited_pv = false;
    if (any) {
      const float alpha = (m_new == m_used) ? 1.f
                          : (m_used == -CUDART_INF_F ? 0.f : ex2(m_used - m_new));
      l *= alpha;
      m_used = m_new;
      // the previous tile's PV must have landed in O before it is rescaled
      if (!wait_or_abort(&c.p_empty, (tau - 1) & 1, c)) return;
      waited_pv = true;
      __syncwarp();
      ptx::tc_fence_after();
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float f = alpha * r[g];
        uint32_t v[32];
        const uint32_t addr = lane_base + 64 * g + 32 * th;
        ptx::tmem_ld32(addr, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
        ptx::tmem_st32(addr, v);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
    }
    // ---- probabilities (fp16 pairs for P)
    const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;
    float sum = 0.f;
    uint32_t pp[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float a = ex2(x[2 * j] - mu), b = ex2(x[2 * j + 1] - mu);
      sum += a + b;
      pp[j] = f16x2_rn(a, b);
    }
    l += sum;
    // ---- P (and the tile's invalid rows) may be written once the previous PV is done
    if (!waited_pv && tau > 0 && !wait_or_abort(&c.p_empty, (tau - 1) & 1, c)) return;
    if (nv < kTileRows) {
      // rows past the end must not reach PV (their bytes are whatever the
      // block holds): zero their codes
      for (int k = T; k < (kTileRows - nv) * 32; k += kSoftThreads) {
        const int row = nv + k / 32, g = (k & 31) >> 3, u = k & 7;
        *reinterpret_cast<uint4*>(code + g * kChunk + sw128(row, u)) = make_uint4(0, 0, 0, 0);
      }
    }
    const int unit = tok0 >> 4;              // my 16 tokens: one 16-byte unit of a P row
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 sa = *reinterpret_cast<const uint4*>(&c.sTp[buf][g][tok0]);
      const uint4 sb = *reinterpret_cast<const uint4*>(&c.sTp[buf][g][tok0 + 8]);
      uint32_t sw[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
      if (need_g) {
        const uint32_t f2 = f16x2_rn(r[g], r[g]);
#pragma unroll
        for (int j = 0; j < 8; ++j) sw[j] = hmul2_rn(sw[j], f2);
      }
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t h0, l0, h1, l1;
        split_hilo(hmul2_rn(pp[2 * j], sw[2 * j]), h0, l0);
        split_hilo(hmul2_rn(pp[2 * j + 1], sw[2 * j + 1]), h1, l1);
        hw[j] = h0 | (h1 << 16);
        lw[j] = l0 | (l1 << 16);
      }
      *reinterpret_cast<uint4*>(pbuf + (2 * g) * kPVar + sw64(h, unit)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(pbuf + (2 * g + 1) * kPVar + sw64(h, unit)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    ptx::fence_proxy_async();
    ptx::mbar_arrive(&c.p_full);
    // ---- epilogue after the request's last tile
    if (cur.last_of_segment()) {
      const SegView& v = cur.v;
      const size_t slot = seg_slot(p, v);
      c.mred[col][h] = l;
      // o_full completes once per request, after its last PV
      if (!wait_or_abort(&c.o_full, sigma & 1, c)) return;
      ptx::named_bar(1, kSoftThreads);
      __syncwarp();
      ptx::tc_fence_after();
      const float ltot = (c.mred[0][h] + c.mred[1][h]) + (c.mred[2][h] + c.mred[3][h]);
      if (col == 0 && h < p.heads)
        (v.whole ? p.out_lse : p.ws_lse)[slot * p.heads + h] =
            ltot > 0.f ? (m_used + log2f(ltot)) * kLn2 : -CUDART_INF_F;
      const float il = ltot > 0.f ? 1.f / ltot : 0.f;
      float* o_base = (v.whole ? p.out : p.ws_o) + (slot * p.heads + h) * kVDim + odh;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float f = il * (sref[g] / kPNorm);
        uint32_t v32[32];
        ptx::tmem_ld32(lane_base + 64 * g + 32 * th, v32);
        ptx::tmem_wait_ld();
        if (h < p.heads) {
          float4* dst = reinterpret_cast<float4*>(o_base + g * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v32[4 * e]) * f, __uint_as_float(v32[4 * e + 1]) * f,
                                 __uint_as_float(v32[4 * e + 2]) * f,
                                 __uint_as_float(v32[4 * e + 3]) * f);
        }
      }
      ptx::tc_fence_before();
      ptx::named_bar(1, kSoftThreads);
      ++sigma;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1) partial_f8_kernel(const __grid_constant__ F8Params P) {
  PartialParams p = P.p;
  if constexpr (!kSparse) p.sparse_idx = nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  F8Ctl& c = *reinterpret_cast<F8Ctl*>(base + kOffCtl);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCodeStages; ++s) {
      ptx::mbar_init(&c.full[s], 1);
      ptx::mbar_init(&c.code_empty[s], 1);
    }
    for (int s = 0; s < kRopeStages; ++s) ptx::mbar_init(&c.rope_empty[s], 1);
    for (int k = 0; k < kParts; ++k) {
      ptx::mbar_init(&c.part_full[k], 1);
      ptx::mbar_init(&c.part_empty[k], kSoftThreads);
    }
    ptx::mbar_init(&c.p_full, kSoftThreads);
    ptx::mbar_init(&c.p_empty, 1);
    ptx::mbar_init(&c.o_full, 1);
    ptx::mbar_init(&c.q_full, kQThreads);
    ptx::mbar_init(&c.q_empty, 2);        // one commit from each score issuer
    c.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) ptx::tmem_alloc(&c.tmem_base, kTmemCols);
  ptx::fence_proxy_async();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  int lo = 0, hi = 0;
  if (!p.sparse_idx) {
    const int T = total_tiles(p, c.warp_sums);
    const int tpc = T > 0 ? (T + p.num_ctas - 1) / p.num_ctas : 0;
    lo = blockIdx.x * tpc;
    hi = min(T, lo + tpc);
  }
  __syncthreads();

  uint32_t tau = 0, sigma = 0, pi = 0, o_commits = 0;
  uint32_t uses[kCodeStages] = {0, 0, 0}, fills[kCodeStages] = {0, 0, 0};
  int first = 0;
  while (true) {
    int nseg, total;
    if (p.sparse_idx) {
      nseg = total = 1;
    } else {
      // the control block holds kMaxSegF8 segments: collect them in batches
      total = lo < hi ? collect_segments_n(p, lo, hi, first, kMaxSegF8, c) : 0;
      nseg = min(kMaxSegF8, total - first);
    }
    if (nseg <= 0) break;
    if (warp < kSoftWarps) {
      softmax_role(p, c, base, nseg, tau, sigma, pi);
    } else if (warp == kProdWarp) {
      if ((threadIdx.x & 31) == 0) producer_role(P, p, c, base, nseg, tau, fills);
    } else if (warp == kQkWarp) {
      if ((threadIdx.x & 31) == 0) qk_role<0>(p, c, base, nseg, tau, sigma);
    } else if (warp == kQkWarp2) {
      if ((threadIdx.x & 31) == 0) qk_role<1>(p, c, base, nseg, tau, sigma);
    } else if (warp == kPvWarp) {
      if ((threadIdx.x & 31) == 0) pv_role(p, c, base, nseg, tau, uses, o_commits);
    } else {
      q_role(p, c, base, nseg, sigma);
    }
    __syncthreads();
    if (c.abort) break;
    first += kMaxSegF8;
    if (p.sparse_idx || total <= first) break;
  }
  // Drain: every asynchronous arrival must land before the CTA exits (it
  // could otherwise hit the next CTA's barriers at the same addresses).
  // Normally only the last slot, P and Q releases are unconsumed; after a
  // timeout any commit or TMA fill may be.  Each wait is for the latest phase
  // of its barrier, so the parity is unambiguous.
  if (threadIdx.x == kPvWarp * 32) {
    uint32_t n = 0;
    for (int s = 0; s < kCodeStages; ++s) {
      if (uses[s] > 0) wait_or_abort(&c.code_empty[s], (uses[s] - 1) & 1, c);
      n += uses[s];
    }
    if (n > 0) wait_or_abort(&c.p_empty, (n - 1) & 1, c);
    if (o_commits > 0) wait_or_abort(&c.o_full, (o_commits - 1) & 1, c);
  }
  if (threadIdx.x == kQkWarp * 32 || threadIdx.x == kQkWarp2 * 32) {
    // tau counts the tiles this issuer handled; parts 5 tau of them, commits
    // on buffer k for every part number below 5 tau congruent to k
    if (sigma > 0) wait_or_abort(&c.q_empty, (sigma - 1) & 1, c);
    if (threadIdx.x == kQkWarp * 32)
      for (uint32_t s = 0; s < (uint32_t)kRopeStages; ++s) {
        const uint32_t n = tau > s ? (tau - s + kRopeStages - 1) / kRopeStages : 0;
        if (n > 0) wait_or_abort(&c.rope_empty[s], (n - 1) & 1, c);
      }
    const uint32_t parts = 5 * tau;
    for (uint32_t k = 0; k < (uint32_t)kParts; ++k) {
      const uint32_t n = parts > k ? (parts - k + kParts - 1) / kParts : 0;
      if (n > 0) wait_or_abort(&c.part_full[k], (n - 1) & 1, c);
    }
  }
  if (threadIdx.x == kProdWarp * 32)
    for (int s = 0; s < kCodeStages; ++s)
      if (fills[s] > 0) wait_or_abort(&c.full[s], (fills[s] - 1) & 1, c);
  if (c.abort && threadIdx.x == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(c.tmem_base, kTmemCols);
}

// ---------------------------------------------------------------- host -----

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Tensor maps over the cache pool viewed as [num_blocks][64 rows][656 bytes].
bool encode_maps(const PartialParams& p, CUtensorMap* rows, CUtensorMap* scales) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kRowBytesFp8, (cuuint64_t)kBlock,
                              (cuuint64_t)p.num_blocks};
  const cuuint64_t strides[2] = {(cuuint64_t)kRowBytesFp8, (cuuint64_t)kRowBytesFp8 * kBlock};
  const cuuint32_t box_rows[3] = {128, (cuuint32_t)kBlock, 1};
  const cuuint32_t box_sc[3] = {16, (cuuint32_t)kBlock, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  void* g = const_cast<uint8_t*>(p.kv);
  if (enc(rows, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, g, dims, strides, box_rows, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  return enc(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, g, dims, strides, box_sc, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::mutex g_attr_mutex;
bool g_attr_done[kMaxDevicesConfigured] = {};

}  // namespace

bool f8_supports(const PartialParams& p, int kv_dtype) {
  return kv_dtype == kKvFp8 && p.q_len == 1 && p.heads >= 1 && p.heads <= kMaxHeads &&
         p.sparse_idx == nullptr && encode_fn() != nullptr;
}

cudaError_t launch_partial_f8(const PartialParams& p, cudaStream_t st) {
  F8Params fp;
  fp.p = p;
  if (!encode_maps(p, &fp.rows, &fp.scales)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesConfigured) return cudaErrorInvalidDevice;
  const int smem = (int)kSmemBytes;
  {
    // raise the shared-memory limit once per device, so that later launches
    // (including ones captured into a CUDA graph) are plain launches
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (!g_attr_done[dev]) {
      e = cudaFuncSetAttribute(partial_f8_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      g_attr_done[dev] = true;
    }
  }
  partial_f8_kernel<false><<<p.num_ctas, kThreads, smem, st>>>(fp);
  return cudaGetLastError();
}

}  // namespace dcpmla

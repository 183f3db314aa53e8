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
// How.  The cache rows are read straight into shared memory (whole 64-row
// blocks by TMA; for sparse lists, the listed rows by TMA gathers and
// cp.async) and the tensor cores consume the e4m3 codes as they are
// (kind::f8f6f4); no thread converts cache values.  Scores are exact up to
// fp32 accumulation order:
//  * Q (bf16, 8 significant bits) is split per head into two e4m3 terms in
//    one power-of-two frame, q * 2^a = hi + lo (q_image.cuh, built once per
//    request by a small kernel).  That is exact for every element of at
//    least 2^-9 of the head's largest (smaller ones lose low bits and weigh
//    at most 2^-9 of it).  hi and lo are two MMAs into one accumulator.
//  * Each 128-value scale group of the latent row has its own accumulator
//    (weight-stationary M = 64 heads, N = 64 tokens): codes . (hi + lo) for
//    that group.  The softmax threads multiply it by the token's fp32 group
//    scale, so the scale is applied exactly in fp32 instead of being rounded
//    into an operand.  The rope (bf16) is a fifth part with bf16 MMAs.
//  * A part takes 32 TMEM columns; eight part buffers hold more than a tile,
//    so the scores of the next tile are computed while this one's softmax
//    runs.
//  * Online softmax in base 2 with a lazily updated running max, decided per
//    head (a head's O is rescaled only when its max grows by more than 2^3).
//  * O += P V reads V as the same e4m3 codes.  The group scale multiplies P:
//    for group g, P_g = p * s_tg * (8 / S_g), stored as two e4m3 terms (hi:
//    the 4 leading bits of the fp16 value, lo: the rest rounded to 4 bits;
//    together within max(2^-7 P_g, 2^-9) of P_g) in a 64 x 64 K-major tile
//    per term; the two
//    PV MMAs of a term pair share V through a collector buffer.  S_g is a
//    per-request reference scale (the group's largest scale in the request's
//    first tile, raised with an exact O rescale if a later tile holds a scale
//    more than 4x larger), so P_g stays below 256 and the tokens that carry
//    the softmax mass stay in the e4m3 normal range; the epilogue multiplies
//    O_g back by S_g / 8.
//  * O (64 heads x 512, fp32) stays in TMEM for the whole request, in the
//    weight-stationary M = 64 layout (one N = 128 accumulator per group).
//
// Roles (16 warps): 0-7 softmax and epilogue (two warps per TMEM lane
// quarter, one per 16-column half), 8 TMA producer, 9 and 15 issue the score
// MMAs (parts 0, 2, 4 and parts 1, 3), 10 issues the PV MMAs, 11-14 load each
// request's Q image, stage each tile's scales (raw and as P factors, with the
// reference scales), clear the rows past a request's end and, for listed
// tiles, copy the parts the producer's gathers leave.  The kernel is a
// template on the row source (blocks or listed rows), so that dense decode
// carries none of the listed code.
// Shared memory: Q 72 KB, three stages of codes and scales (3 x 33 KB), two
// of rope (2 x 8 KB), P 32 KB.  Every wait is bounded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "q_image.cuh"
#include "tc_ptx.cuh"

namespace dcpmla {

// Optional clock trace of CTA 1 (event x index), compiled in only when
// DCPMLA_F8_TRACE is defined; the product build leaves it out.
#ifdef DCPMLA_F8_TRACE
__device__ long long g_f8_trace[24][256];
#define F8_TRACE(ev, idx)                                                        \
  do {                                                                           \
    if (blockIdx.x == 1 && (idx) < 256) g_f8_trace[ev][idx] = clock64();         \
  } while (0)
#else
#define F8_TRACE(ev, idx) ((void)0)
#endif

namespace {

constexpr int kThreads = 512;          // 16 warps
constexpr int kSoftWarps = 8;
constexpr int kProdWarp = 8, kQkWarp = 9, kPvWarp = 10, kStageWarp0 = 11, kQkWarp2 = 15;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kStageThreads = 128;
constexpr int kBarSoft = 1, kBarStage = 2, kBarBlock = 3;   // named barriers
constexpr int kLaunchRegs = 128;             // 65,536 / kThreads
constexpr int kSoftRegs = 184, kOtherRegs = 72;
static_assert(kSoftWarps * 32 * kSoftRegs + (kThreads - kSoftWarps * 32) * kOtherRegs ==
                  kThreads * kLaunchRegs,
              "the register split must add up to what the launch holds");
static_assert(kSoftWarps % 4 == 0, "setmaxnreg acts on whole warpgroups");

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
constexpr uint32_t kQOperandBytes = kOffCode - kOffQh;   // hi, lo and rope, contiguous
static_assert(kQOperandBytes + 64 * 4 == (uint32_t)kQImageBytes, "Q image = operands + frame");
static_assert(kOffQl - kOffQh == qimg::kLo && kOffQr - kOffQh == qimg::kRope &&
                  kQOperandBytes == qimg::kFrame,
              "the image's operand part is the Q region of shared memory, byte for byte");
constexpr uint32_t kOffRope = kOffCode + kCodeStages * kCodeStage;
constexpr uint32_t kOffP = kOffRope + kRopeStages * kChunk;
constexpr uint32_t kOffCtl = kOffP + 8 * kPVar;
static_assert(kOffCode % 1024 == 0 && kCodeStage % 1024 == 0 && kOffRope % 1024 == 0 &&
                  kOffP % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
static_assert(kTileBytes == 4 * kChunk + 1024 + kChunk, "a tile is codes, scales and rope");
// Listed tile: code chunks 0 and 1 arrive by TMA gathers from the producer
// warp, 2 and 3 (with the rope and scales) by cp.async from the staging warps.
// The tensor unit takes a four-row gather about every 65 cycles and a warp's
// copy instruction costs about as much: splitting the bytes between the two
// units was measured best at two chunks each, and spreading the copies over
// the four staging warps (one per scheduler) takes them off the producer.
constexpr int kGatheredChunks = 2;
constexpr uint32_t kListedTmaBytes = kGatheredChunks * kChunk;
constexpr int kListedCopyArrivals = 128;            // listed tile: one per staging thread

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

// collector buffer of the PV issuer (the score MMAs gain nothing from one)
constexpr int kCollPv = 2;

// TMA box x offset inside a row: code chunks 0..3, then the rope
__device__ __forceinline__ int box_x(int k) { return k < 4 ? 128 * k : 528; }

struct F8Params {
  PartialParams p;
  CUtensorMap rows;      // [blocks][64][656] u8, box 128 x 64, 128-byte swizzle
  CUtensorMap scales;    // same tensor, box 16 x 64, no swizzle (the four fp32 scales)
};

struct F8Ctl {
  alignas(16) float sT[2][4][64];   // a tile's scales, [tile parity][group][row]
  alignas(16) __half sTp[2][4][64]; // the same times kPNorm / S_g (fp16), 0 for absent rows
  alignas(16) float sc_r[2][4];     // per group: O rescale factor S_old / S_new at this tile
  alignas(16) float sc_ref[2][4];   // per group: S_g in force for this tile
  alignas(16) float gw[2][4][4];    // staging: per-warp group maxima of |scale|
  alignas(16) float qexp[64];       // 2^-a per head (Q frame)
  float mred[2][4][64];             // [tile parity] per-thread-column maxima of the scores; in
                                    // the epilogue (other parity) the per-thread-column sums
  uint64_t full[kCodeStages];       // TMA bytes of a tile landed
  uint64_t staged[kCodeStages];     // the tile's scales staged and absent rows cleared
  uint64_t code_empty[kCodeStages]; // PV of the slot's tile done (commit)
  uint64_t rope_empty[kRopeStages]; // rope part of the slot's tile done (commit)
  uint64_t part_full[kParts];       // score part ready (commit)
  uint64_t part_empty[kParts];      // score part read (softmax arrivals)
  uint64_t sc_empty[2];             // softmax done with a staged scale buffer
  uint64_t p_full;                  // P written (softmax arrivals)
  uint64_t p_empty;                 // PV done reading P (commit)
  uint64_t o_full;                  // a request's last PV done (commit)
  uint64_t q_full;                  // Q of the next request staged (staging arrivals)
  uint64_t q_empty;                 // a request's last score MMA done (commits) and its Q
                                    // frame read (softmax arrivals)
  int nv[kCodeStages];              // rows of the slot's tile that take part (producer)
  uint32_t tmem_base;
  int abort;
  int sel_count;
  int warp_sums[16];
  Segment seg[kMaxSegF8];
};

constexpr size_t kSmemBytes = kOffCtl + sizeof(F8Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

using qimg::sw128;   // 128-byte swizzle of unit u in row r
__device__ __forceinline__ uint32_t sw64(int r, int u) {
  return (uint32_t)((r >> 3) * 512 + (r & 7) * 64 + (((u ^ ((r & 7) >> 1)) & 3) << 4));
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, F8Ctl& c) {
  return ptx::mbar_wait(bar, parity, &c.abort);
}

// One arrival per warp, made by lane 0 once the whole warp got here (the
// barrier's count is in warps).  Shared-memory atomics are scarce while the
// tensor core streams its operands, so threads do not arrive one by one.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
__device__ __forceinline__ uint16_t f16_sat(float x) {
  uint16_t d;
  asm("cvt.rn.satfinite.f16.f32 %0, %1;" : "=h"(d) : "f"(x));
  return d;
}

// Two fp16 pairs x0, x1 (P_g of four tokens, |x| < 256) -> their e4m3 hi
// and lo terms, four bytes each (first token in the low byte).  hi keeps the
// sign, exponent and 3 leading mantissa bits of each fp16 value (4
// significant bits, exact in e4m3 in its normal range); lo = x - hi is exact
// in fp16 and below 2^-3 |x|, and its encoding rounds it to 4 bits.
__device__ __forceinline__ void split_hilo4(uint32_t x0, uint32_t x1, uint32_t& hi,
                                            uint32_t& lo) {
  constexpr uint32_t kLead = 0xFF80FF80u;
  const uint32_t h0 = x0 & kLead, h1 = x1 & kLead;
  const uint32_t l0 = hsub2_rn(x0, h0), l1 = hsub2_rn(x1, h1);
  asm("{\n .reg .b16 a, b;\n"
      " cvt.rn.satfinite.e4m3x2.f16x2 a, %1;\n"
      " cvt.rn.satfinite.e4m3x2.f16x2 b, %2;\n"
      " mov.b32 %0, {a, b};\n}\n"
      : "=r"(hi)
      : "r"(h0), "r"(h1));
  asm("{\n .reg .b16 a, b;\n"
      " cvt.rn.satfinite.e4m3x2.f16x2 a, %1;\n"
      " cvt.rn.satfinite.e4m3x2.f16x2 b, %2;\n"
      " mov.b32 %0, {a, b};\n}\n"
      : "=r"(lo)
      : "r"(l0), "r"(l1));
}

// ---------------------------------------------------------------- roles ----

// TMA producer (one warp): tile tau goes to code slot tau % 3 and rope slot
// tau % 2.  Lane 0 waits for the slots and arms the tile's barrier.  A block
// tile is six box loads by lane 0; a tile whose table entry is out of range
// (flagged) loads block 0 instead and has no valid rows.  A listed tile
// (sparse rows, p.row_ids): lanes 0..15 fetch code chunks 0 and 1 of four
// rows each by TMA gathers; the staging warps copy the rest (listed_fetch).
template <bool kListed>
__device__ __forceinline__ void producer_role(const F8Params& P, const PartialParams& p, F8Ctl& c,
                              uint8_t* base, int nseg, uint32_t& tau,
                              uint32_t (&fills)[kCodeStages]) {
  const int lane = threadIdx.x & 31;
  const bool lead = lane == 0;
  TileCursor cur, pf;
  if (!cur.start(p, c, nseg)) return;
  pf = cur;
  bool pf_ok = !kListed;
  for (int i = 0; i < kPrefetchTiles && pf_ok; ++i) {
    const int blk = tile_block(p, pf.v.b, (pf.v.row_begin >> 6) + pf.t);
    if (lead && blk >= 0) ptx::prefetch_l2(p.kv + (size_t)blk * kTileBytes, kTileBytes);
    pf_ok = pf.next(p, c);
  }
  while (true) {
    const uint32_t cs = tau % kCodeStages, rs = tau % kRopeStages;
    // slot reuse: the PV of tile tau - 3 and the rope part of tile tau - 2
    bool ok = true;
    if (lead) {
      if (tau >= (uint32_t)kCodeStages)
        ok = wait_or_abort(&c.code_empty[cs], ((tau / kCodeStages) + 1) & 1, c);
      if (ok && tau >= (uint32_t)kRopeStages)
        ok = wait_or_abort(&c.rope_empty[rs], ((tau / kRopeStages) + 1) & 1, c);
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) return;
    // test only: withholding the very first tile makes every pipeline wait
    // of the CTA run out, which exercises the timeout path
    const bool issue = !(p.test_withhold && tau == 0);
    uint64_t* bar = &c.full[cs];
    const uint32_t dst = ptx::smem_addr(base + kOffCode + cs * kCodeStage);
    const uint32_t dst_rope = ptx::smem_addr(base + kOffRope + rs * kChunk);
    if constexpr (!kListed) {
      if (lead) {
        const int blk = tile_block(p, cur.v.b, (cur.v.row_begin >> 6) + cur.t);
        const int z = blk >= 0 ? blk : 0;
        // read after the bytes land (the arrival below releases this write)
        c.nv[cs] = blk >= 0 ? cur.tile_valid_rows() : 0;
        F8_TRACE(0, tau);
        if (issue) {
          ptx::mbar_arrive_expect_tx(bar, kTileBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) ptx::tma_load_3d(dst + k * kChunk, &P.rows, box_x(k), 0, z, bar);
          ptx::tma_load_3d(dst + kScalesOff, &P.scales, 512, 0, z, bar);
          ptx::tma_load_3d(dst_rope, &P.rows, box_x(4), 0, z, bar);
          ++fills[cs];
        }
      }
    } else {
      if (lead) {
        c.nv[cs] = cur.tile_valid_rows();
        F8_TRACE(0, tau);
        if (issue) {
          ptx::mbar_arrive_expect_tx(bar, kListedTmaBytes);
          ++fills[cs];
        }
      }
      __syncwarp();
      if (issue && lane < 16) {
        // rows 4 l .. 4 l + 3 of the tile
        const int4 r = __ldg(reinterpret_cast<const int4*>(
                                 p.row_ids + (size_t)cur.v.b * p.row_stride + cur.v.row_begin +
                                 cur.t * kTileRows) + lane);
        if (lead) F8_TRACE(9, tau);
#pragma unroll
        for (int k = 0; k < kGatheredChunks; ++k)
          ptx::tma_gather4(dst + k * kChunk + lane * 512, &P.rows, box_x(k), r, bar);
      }
    }
    ++tau;
    if (!cur.next(p, c)) break;
    if (pf_ok) {
      const int pb = tile_block(p, pf.v.b, (pf.v.row_begin >> 6) + pf.t);
      if (lead && pb >= 0) ptx::prefetch_l2(p.kv + (size_t)pb * kTileBytes, kTileBytes);
      pf_ok = pf.next(p, c);
    }
  }
}

// Descriptor plus a byte offset (the start address field holds address / 16
// and never carries: shared memory is below 256 KB).
__device__ __forceinline__ uint64_t dplus(uint64_t d, uint32_t byte_off) {
  return d + (uint64_t)(byte_off >> 4);
}

// Score MMAs.  Two threads share them: side 0 issues parts 0, 2 and 4 (the
// rope) of each tile, side 1 parts 1 and 3; part p of tile tau is number
// 5 tau + p and goes to part buffer (5 tau + p) % 8 (weight-stationary
// M = 64 heads, N = 64 tokens, 32 columns).  A group part is four e4m3
// K-steps of 32, each a hi and a lo MMA into one accumulator; the rope part
// is four bf16 K-steps of 16.  One loop serves both sides (a small
// instruction footprint matters more here than constant offsets).
template <bool kListed>
__device__ __forceinline__ void qk_role(int side, const PartialParams& p, F8Ctl& c, uint8_t* base,
                                        int nseg, uint32_t& tau, uint32_t& sigma) {
  constexpr uint32_t kIdF8 = ptx::idesc_make(64, 64, 0, false, false);
  constexpr uint32_t kIdBf = ptx::idesc_make(64, 64, 1, false, false);
  const uint64_t dqh = ptx::sdesc(ptx::smem_addr(base + kOffQh), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dql = ptx::sdesc(ptx::smem_addr(base + kOffQl), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dqr = ptx::sdesc(ptx::smem_addr(base + kOffQr), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dc0 = ptx::sdesc(ptx::smem_addr(base + kOffCode), 16, 1024, ptx::kSwizzle128B);
  const uint64_t dr0 = ptx::sdesc(ptx::smem_addr(base + kOffRope), 16, 1024, ptx::kSwizzle128B);
  const int nparts = side == 0 ? 3 : 2;
  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  while (true) {
    const uint32_t cs = tau % kCodeStages, rs = tau % kRopeStages;
    if (cur.t == 0 && !wait_or_abort(&c.q_full, sigma & 1, c)) return;
    // One shared-memory round trip tests every barrier the tile's parts
    // need, then its MMAs issue back to back:
    //  * the tile's bytes have landed (the scores need neither the staged
    //    scales nor the clearing of rows past the end: those rows' scores
    //    are masked, and PV, which does need the clearing, runs after the
    //    softmax has waited for it);
    //  * each part's buffer is free (part number n reuses the buffer of
    //    part n - 8, released by the softmax), which keeps the scores at
    //    most 1.6 tiles ahead of the softmax.
    uint64_t* bars[4];
    uint32_t pars[4];
    bars[0] = &c.full[cs];
    pars[0] = (tau / kCodeStages) & 1;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int part = side + 2 * (k < nparts ? k : nparts - 1);
      const uint32_t pi = 5 * tau + part;
      bars[1 + k] = pi >= (uint32_t)kParts ? &c.part_empty[pi % kParts] : bars[0];
      pars[1 + k] = pi >= (uint32_t)kParts ? ((pi / kParts) + 1) & 1 : pars[0];
    }
    if (!ptx::mbar_wait4(bars, pars, &c.abort)) return;
    ptx::tc_fence_after();
    // part of a listed tile arrived by cp.async (the generic proxy): order it
    // before the score MMAs, which read through the async proxy
    if constexpr (kListed) ptx::fence_proxy_async();
    if (side == 0) F8_TRACE(1, tau);
    const uint64_t dcode = dplus(dc0, cs * kCodeStage), drope = dplus(dr0, rs * kChunk);
#pragma unroll 1
    for (int k = 0; k < nparts; ++k) {
      const int part = side + 2 * k;
      const uint32_t pi = 5 * tau + part, buf = pi % kParts;
      F8_TRACE(12, pi);
      const uint32_t d = c.tmem_base + kColPart + 32 * buf;
      if (part < 4) {
        const uint32_t off = part * kChunk;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bk = dplus(dcode, off + ks * 32);
          ptx::mma_ws_f8(d, dplus(dqh, off + ks * 32), bk, kIdF8, ks > 0);
          ptx::mma_ws_f8(d, dplus(dql, off + ks * 32), bk, kIdF8, 1u);
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          ptx::mma_ws_f16(d, dplus(dqr, ks * 32), dplus(drope, ks * 32), kIdBf, ks > 0);
      }
      ptx::mma_commit(&c.part_full[buf]);
      F8_TRACE(13, pi);
    }
    if (side == 0) {
      ptx::mma_commit(&c.rope_empty[rs]);
      F8_TRACE(2, tau);
    }
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
// chunk g of the tile's slot read MN-major, kept in a collector buffer
// between the hi and lo MMAs.
template <bool kListed>
__device__ __forceinline__ void pv_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg, uint32_t& tau,
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
    // a listed tile's V chunks 2 and 3 arrived by cp.async (the generic proxy)
    if constexpr (kListed) ptx::fence_proxy_async();
    F8_TRACE(3, tau);
    const uint64_t dv = dplus(dv0, cs * kCodeStage);
    const uint32_t acc0 = cur.t == 0 ? 0u : 1u;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t d = c.tmem_base + 64 * g;
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const uint64_t bv = dplus(dv, g * kChunk + ks * 4096);
        ptx::mma_ws_f8_coll<kCollPv, ptx::kFill>(d, dplus(dp, (2 * g) * kPVar + ks * 32), bv,
                                                 kIdPv, ks == 0 ? acc0 : 1u);
        ptx::mma_ws_f8_coll<kCollPv, ptx::kLastUse>(d, dplus(dp, (2 * g + 1) * kPVar + ks * 32),
                                                    bv, kIdPv, 1u);
      }
      F8_TRACE(14, 4 * tau + g);
    }
    ptx::mma_commit(&c.p_empty);
    ptx::mma_commit(&c.code_empty[cs]);
    F8_TRACE(10, tau);
    ++uses[cs];
    if (cur.last_of_segment()) {
      ptx::mma_commit(&c.o_full);
      ++o_commits;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Q of request b: one bulk copy of its operand image (hi and lo codes and
// rope, in shared-memory order) and one of its frame factors, issued once the
// previous request's score MMAs are done and its softmax read its frame.
// Staging warp 0 arms q_full with the bytes; the other three arrive.
__device__ __forceinline__ bool load_q(const PartialParams& p, F8Ctl& c, uint8_t* base, int b,
                                       uint32_t sigma) {
  const int u = threadIdx.x - kStageWarp0 * 32;   // 0..127
  if (sigma > 0 && !wait_or_abort(&c.q_empty, (sigma - 1) & 1, c)) return false;
  if (u == 0) {
    F8_TRACE(22, sigma);
    // the softmax read the old frame through the generic proxy
    ptx::fence_proxy_async();
    const uint8_t* img = p.q_image + (size_t)b * kQImageBytes;
    ptx::mbar_arrive_expect_tx(&c.q_full, kQImageBytes);
    ptx::bulk_g2s(ptx::smem_addr(base + kOffQh), img, kQOperandBytes, &c.q_full);
    ptx::bulk_g2s(ptx::smem_addr(c.qexp), img + kQOperandBytes, kQImageBytes - kQOperandBytes,
                  &c.q_full);
  } else if (u >= 32) {
    warp_arrive(&c.q_full);
  }
  return true;
}

// Listed tile tau (cursor t): the parts the producer's gathers leave (code
// chunks kGatheredChunks.., the rope and the scales), copied by the 128
// staging threads with 16-byte cp.async into the tile's slots, once the
// slots are free (the PV of tile tau - 3, the score MMAs of tile tau - 2);
// eight threads take one 128-byte piece of a row, swizzled like the tensor
// copies.  Each thread arrives on the tile's barrier when its copies land.
__device__ __forceinline__ bool listed_fetch(const PartialParams& p, F8Ctl& c, uint8_t* base,
                                             const TileCursor& t, uint32_t tau, int u) {
  const uint32_t cs = tau % kCodeStages, rs = tau % kRopeStages;
  if (tau >= (uint32_t)kCodeStages &&
      !wait_or_abort(&c.code_empty[cs], ((tau / kCodeStages) + 1) & 1, c))
    return false;
  if (tau >= (uint32_t)kRopeStages &&
      !wait_or_abort(&c.rope_empty[rs], ((tau / kRopeStages) + 1) & 1, c))
    return false;
  const int* ids = p.row_ids + (size_t)t.v.b * p.row_stride + t.v.row_begin + t.t * kTileRows;
  const int un = u & 7, r0 = u >> 3;         // rows r0 + 16 k, 16-byte unit un
  int id[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) id[k] = __ldg(ids + r0 + 16 * k);
  const int sid = u < kTileRows ? __ldg(ids + u) : 0;
  const uint32_t dst = ptx::smem_addr(base + kOffCode + cs * kCodeStage);
  const uint32_t dst_rope = ptx::smem_addr(base + kOffRope + rs * kChunk);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = r0 + 16 * k;
    const uint8_t* row = p.kv + (size_t)id[k] * kRowBytesFp8 + 16 * un;
    ptx::cp_async16(dst_rope + sw128(rr, un), row + 528, 16);
#pragma unroll
    for (int g = kGatheredChunks; g < 4; ++g)
      ptx::cp_async16(dst + g * kChunk + sw128(rr, un), row + 128 * g, 16);
  }
  if (u < kTileRows)
    ptx::cp_async16(dst + kScalesOff + u * 16, p.kv + (size_t)sid * kRowBytesFp8 + 512, 16);
  ptx::cp_async_arrive(&c.full[cs]);
  return true;
}

// Staging (4 warps): per request, its Q; per tile, once its bytes landed,
// the scales as [group][row] copies (raw, and times kPNorm / S_g as fp16),
// the reference scales S_g with the O rescale factor a raised reference
// implies, and zeros over the codes of rows past the request's end (their
// bytes are whatever the block holds and must not reach PV).  Thread u
// handles row u / 2, groups 2 (u % 2) and 2 (u % 2) + 1.
template <bool kListed>
__device__ __forceinline__ void staging_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg,
                             uint32_t& tau, uint32_t& sigma) {
  const int u = threadIdx.x - kStageWarp0 * 32;   // 0..127
  const int sw = u >> 5, lane = u & 31;
  const int row = u >> 1, gp = (u & 1) * 2;
  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  // listed tiles: the copies of a tile are issued one tile ahead of its
  // staging (the first here)
  if constexpr (kListed) {
    if (!listed_fetch(p, c, base, cur, tau, u)) return;
  }
  float sref[4] = {1.f, 1.f, 1.f, 1.f};
  while (true) {
    const uint32_t cs = tau % kCodeStages;
    const int b = tau & 1;
    const bool first = cur.t == 0;
    if (first) {
      if (!load_q(p, c, base, cur.v.b, sigma)) return;
      ++sigma;
    }
    if (!wait_or_abort(&c.full[cs], (tau / kCodeStages) & 1, c)) return;
    if (u == 0) F8_TRACE(20, tau);
    // buffer b was last read by the softmax of tile tau - 2
    if (tau >= 2 && !wait_or_abort(&c.sc_empty[b], ((tau / 2) + 1) & 1, c)) return;
    const int nv = c.nv[cs];
    uint8_t* code = base + kOffCode + cs * kCodeStage;
    const float2 sv = *reinterpret_cast<const float2*>(code + kScalesOff + row * 16 + gp * 4);
    const bool valid = row < nv;
    float m0 = valid ? fabsf(sv.x) : 0.f, m1 = valid ? fabsf(sv.y) : 0.f;
#pragma unroll
    for (int o = 2; o < 32; o <<= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (lane < 2) {
      c.gw[b][sw][gp] = m0;
      c.gw[b][sw][gp + 1] = m1;
    }
    ptx::named_bar(kBarStage, kStageThreads);
    float gm[4];
    {
      const float4 w0 = *reinterpret_cast<const float4*>(c.gw[b][0]);
      const float4 w1 = *reinterpret_cast<const float4*>(c.gw[b][1]);
      const float4 w2 = *reinterpret_cast<const float4*>(c.gw[b][2]);
      const float4 w3 = *reinterpret_cast<const float4*>(c.gw[b][3]);
      gm[0] = fmaxf(fmaxf(w0.x, w1.x), fmaxf(w2.x, w3.x));
      gm[1] = fmaxf(fmaxf(w0.y, w1.y), fmaxf(w2.y, w3.y));
      gm[2] = fmaxf(fmaxf(w0.z, w1.z), fmaxf(w2.z, w3.z));
      gm[3] = fmaxf(fmaxf(w0.w, w1.w), fmaxf(w2.w, w3.w));
    }
    float r[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (first) {
        sref[g] = gm[g] > 0.f ? gm[g] : 1.f;
      } else if (gm[g] > kScaleSlack * sref[g]) {
        r[g] = sref[g] / gm[g];
        sref[g] = gm[g];
      }
    }
    if (u == 0) {
      *reinterpret_cast<float4*>(c.sc_r[b]) = make_float4(r[0], r[1], r[2], r[3]);
      *reinterpret_cast<float4*>(c.sc_ref[b]) = make_float4(sref[0], sref[1], sref[2], sref[3]);
    }
    const float ref0 = gp == 0 ? sref[0] : sref[2], ref1 = gp == 0 ? sref[1] : sref[3];
    c.sT[b][gp][row] = sv.x;
    c.sT[b][gp + 1][row] = sv.y;
    reinterpret_cast<uint16_t*>(c.sTp[b][gp])[row] = f16_sat(valid ? sv.x * (kPNorm / ref0) : 0.f);
    reinterpret_cast<uint16_t*>(c.sTp[b][gp + 1])[row] =
        f16_sat(valid ? sv.y * (kPNorm / ref1) : 0.f);
    if (nv < kTileRows) {
      for (int k = u; k < (kTileRows - nv) * 32; k += kStageThreads) {
        const int rr = nv + k / 32, g = (k & 31) >> 3, un = k & 7;
        *reinterpret_cast<uint4*>(code + g * kChunk + sw128(rr, un)) = make_uint4(0, 0, 0, 0);
      }
      ptx::fence_proxy_async();
    }
    warp_arrive(&c.staged[cs]);
    if (u == 0) F8_TRACE(21, tau);
    if constexpr (kListed) {
      TileCursor nx = cur;
      if (nx.next(p, c) && !listed_fetch(p, c, base, nx, tau + 1, u)) return;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Softmax, P and the epilogue (8 warps).  Parts and O share the weight-
// stationary M = 64 layout: TMEM lane L holds head L % 64 for the first
// (L < 64) or second half of the columns.  Warp w reads lane quarter
// q = w % 4 and the 16-column half th = w / 4 of each part, so thread (w, i)
// owns 16 tokens of head h = (32 q + i) % 64.
//
// While the tensor core streams its operands, every shared-memory round trip
// of these threads costs a few hundred cycles, so each tile takes as few as
// possible: one for its barriers, one for the parts (TMEM) and scales
// together, one for P.  The running max of a head is shared by its four
// threads; a barrier-wide vote tells whether any thread's tile maximum
// exceeds the max in use by more than 2^3, and only then are the maxima
// exchanged through shared memory.
__device__ __forceinline__ void softmax_role(const PartialParams& p, F8Ctl& c, uint8_t* base, int nseg,
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

  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  float m_used = -CUDART_INF_F, l = 0.f, kq = 0.f, two_a = 1.f;
  uint8_t* pbuf = base + kOffP;
  while (true) {
    const uint32_t cs = tau % kCodeStages;
    const int b = tau & 1;
    const bool first_blk = cur.t == 0;
    if (T == 0) F8_TRACE(4, tau);
    if (first_blk) {
      if (!wait_or_abort(&c.q_full, sigma & 1, c)) return;
      const float qe = c.qexp[h];
      warp_arrive(&c.q_empty);               // the Q frame is read
      kq = qe * sl2;
      two_a = 1.f / qe;                      // exact: a power of two
      m_used = -CUDART_INF_F;
      l = 0.f;
    }
    // ---- the tile's staged scales and its five score parts (side 1's
    // commit of part 3 and side 0's of part 4 cover all of them)
    if (!ptx::mbar_wait3(&c.staged[cs], (tau / kCodeStages) & 1, &c.part_full[(pi + 3) % kParts],
                         ((pi + 3) / kParts) & 1, &c.part_full[(pi + 4) % kParts],
                         ((pi + 4) / kParts) & 1, &c.abort))
      return;
    if (T == 0) F8_TRACE(19, tau);
    __syncwarp();
    ptx::tc_fence_after();
    // rows of the tile that take part (none if its table entry is bad: the
    // producer flagged it and loaded a stand-in block), the group rescale
    // factors, the reference scales and this thread's 16 token scales; then
    // the parts in two TMEM loads (registers bound the batch)
    const int nv = c.nv[cs];
    const float4 rr = *reinterpret_cast<const float4*>(c.sc_r[b]);
    const float4 sref = *reinterpret_cast<const float4*>(c.sc_ref[b]);
    float4 s4[4][4];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int j = 0; j < 4; ++j) s4[g][j] = reinterpret_cast<const float4*>(&c.sT[b][g][tok0])[j];
    float x[16];
    {
      uint32_t xa[3][16];
#pragma unroll
      for (int part = 0; part < 3; ++part)
        ptx::tmem_ld16(lane_base + kColPart + 32 * ((pi + part) % kParts) + 16 * th, xa[part]);
      ptx::tmem_wait_ld();
      if (T == 0) F8_TRACE(16, tau);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 4 * j + e;
          const float s0 = e == 0 ? s4[0][j].x : e == 1 ? s4[0][j].y : e == 2 ? s4[0][j].z : s4[0][j].w;
          const float s1 = e == 0 ? s4[1][j].x : e == 1 ? s4[1][j].y : e == 2 ? s4[1][j].z : s4[1][j].w;
          const float s2 = e == 0 ? s4[2][j].x : e == 1 ? s4[2][j].y : e == 2 ? s4[2][j].z : s4[2][j].w;
          float v = s0 * __uint_as_float(xa[0][k]);
          v = fmaf(s1, __uint_as_float(xa[1][k]), v);
          x[k] = fmaf(s2, __uint_as_float(xa[2][k]), v);
        }
      }
    }
    {
      uint32_t xb[2][16];
#pragma unroll
      for (int part = 3; part < 5; ++part)
        ptx::tmem_ld16(lane_base + kColPart + 32 * ((pi + part) % kParts) + 16 * th,
                       xb[part - 3]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (i == 0)
#pragma unroll
        for (int part = 0; part < 5; ++part) ptx::mbar_arrive(&c.part_empty[(pi + part) % kParts]);
      // x = sum_g s_g part_g + 2^a rope (times 2^-a scale log2(e) below)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 4 * j + e;
          const float s3 = e == 0 ? s4[3][j].x : e == 1 ? s4[3][j].y : e == 2 ? s4[3][j].z : s4[3][j].w;
          const float v = fmaf(s3, __uint_as_float(xb[0][k]), x[k]);
          x[k] = fmaf(__uint_as_float(xb[1][k]), two_a, v);
        }
      }
    }
    pi += 5;
    const bool need_g = !first_blk && (rr.x != 1.f || rr.y != 1.f || rr.z != 1.f || rr.w != 1.f);
    // the P factors of this thread's tokens (consumed after the exponentials)
    uint4 sp[4][2];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      sp[g][0] = *reinterpret_cast<const uint4*>(&c.sTp[b][g][tok0]);
      sp[g][1] = *reinterpret_cast<const uint4*>(&c.sTp[b][g][tok0 + 8]);
    }
    float mloc = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      x[j] = (tok0 + j < nv) ? x[j] * kq : -CUDART_INF_F;
      mloc = fmaxf(mloc, x[j]);
    }
    if (T == 0) F8_TRACE(5, tau);
    // ---- lazy max, per head.  The vote is a barrier without shared-memory
    // traffic; the exchange runs only if some thread needs a larger max.
    const bool grow = mloc > m_used + kRescaleLog2;
    float alpha = 1.f;
    if (ptx::named_bar_or(kBarSoft, kSoftThreads, grow)) {
      float (*mr)[64] = c.mred[b];
      mr[col][h] = mloc;
      ptx::named_bar(kBarSoft, kSoftThreads);
      const float mt = fmaxf(fmaxf(mr[0][h], mr[1][h]), fmaxf(mr[2][h], mr[3][h]));
      if (first_blk) {
        m_used = mt;
      } else if (mt > m_used + kRescaleLog2) {
        alpha = m_used == -CUDART_INF_F ? 0.f : ex2(m_used - mt);
        m_used = mt;
      }
    }
    if (T == 0) F8_TRACE(6, tau);
    l *= alpha;
    bool waited_pv = false;
    if (__any_sync(0xffffffffu, alpha != 1.f || need_g)) {
      // O of the previous tiles is rescaled once the previous PV has landed;
      // a raised group reference scales its O by r_g as well
      if (!wait_or_abort(&c.p_empty, (tau - 1) & 1, c)) return;
      waited_pv = true;
      if (T == 0) F8_TRACE(11, tau);
      __syncwarp();
      ptx::tc_fence_after();
#pragma unroll 1
      for (int g = 0; g < 4; ++g) {
        const float rg = g == 0 ? rr.x : g == 1 ? rr.y : g == 2 ? rr.z : rr.w;
        const float f = need_g ? alpha * rg : alpha;
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
      const float a = ex2(x[2 * j] - mu), bb = ex2(x[2 * j + 1] - mu);
      sum += a + bb;
      pp[j] = f16x2_rn(a, bb);
    }
    l += sum;
    // ---- P may be written once the previous PV is done with it
    if (!waited_pv && tau > 0 && !wait_or_abort(&c.p_empty, (tau - 1) & 1, c)) return;
    if (T == 0) F8_TRACE(7, tau);
    const int unit = tok0 >> 4;              // my 16 tokens: one 16-byte unit of a P row
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t swv[8] = {sp[g][0].x, sp[g][0].y, sp[g][0].z, sp[g][0].w,
                               sp[g][1].x, sp[g][1].y, sp[g][1].z, sp[g][1].w};
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        split_hilo4(hmul2_rn(pp[2 * j], swv[2 * j]), hmul2_rn(pp[2 * j + 1], swv[2 * j + 1]),
                    hw[j], lw[j]);
      *reinterpret_cast<uint4*>(pbuf + (2 * g) * kPVar + sw64(h, unit)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(pbuf + (2 * g + 1) * kPVar + sw64(h, unit)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    ptx::fence_proxy_async();
    __syncwarp();
    if (i == 0) {
      ptx::mbar_arrive(&c.p_full);
      ptx::mbar_arrive(&c.sc_empty[b]);
    }
    if (T == 0) F8_TRACE(8, tau);
    // ---- epilogue after the request's last tile
    if (cur.last_of_segment()) {
      const SegView& v = cur.v;
      const size_t slot = seg_slot(p, v);
      // the other parity's maxima were read before this tile's vote
      float (*ls)[64] = c.mred[b ^ 1];
      ls[col][h] = l;
      // o_full completes once per request, after its last PV
      if (!wait_or_abort(&c.o_full, sigma & 1, c)) return;
      if (T == 0) F8_TRACE(17, sigma);
      ptx::named_bar(kBarSoft, kSoftThreads);
      __syncwarp();
      ptx::tc_fence_after();
      const float ltot = (ls[0][h] + ls[1][h]) + (ls[2][h] + ls[3][h]);
      if (col == 0 && h < p.heads)
        (v.whole ? p.out_lse : p.ws_lse)[slot * (v.whole ? p.rows_o : p.heads) + h] =
            ltot > 0.f ? (m_used + log2f(ltot)) * kLn2 : -CUDART_INF_F;
      const float il = ltot > 0.f ? 1.f / ltot : 0.f;
      // O leaves through this warp's 4 KB of the P buffer (free: the last PV
      // is done): lane i writes its head's 32 values (128 bytes) as row i,
      // 16-byte units xor-swizzled by i % 8; then 8 lanes take one row, so
      // that each store writes four whole 128-byte lines of O.
      float* o_rows = (v.whole ? p.out : p.ws_o) + slot * (v.whole ? p.rows_o : p.heads) * kVDim;
      uint8_t* scr = pbuf + w * 4096;
      const int h_w = (32 * q) & 63;         // head of lane 0 of this warp
      const int rq = i >> 3, un = i & 7;     // read side: row 4 k + rq, unit un
#pragma unroll 1
      for (int g = 0; g < 4; ++g) {
        const float sg = g == 0 ? sref.x : g == 1 ? sref.y : g == 2 ? sref.z : sref.w;
        const float f = il * (sg * (1.f / kPNorm));
        uint32_t v32[32];
        ptx::tmem_ld32(lane_base + 64 * g + 32 * th, v32);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<float4*>(scr + i * 128 + ((e ^ (i & 7)) << 4)) =
              make_float4(__uint_as_float(v32[4 * e]) * f, __uint_as_float(v32[4 * e + 1]) * f,
                          __uint_as_float(v32[4 * e + 2]) * f, __uint_as_float(v32[4 * e + 3]) * f);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int r = 4 * k + rq;
          const float4 val = *reinterpret_cast<const float4*>(scr + r * 128 + ((un ^ (r & 7)) << 4));
          if (h_w + r < p.heads)
            *reinterpret_cast<float4*>(o_rows + (size_t)(h_w + r) * kVDim + g * 128 + odh + 4 * un) = val;
        }
        __syncwarp();
      }
      ptx::tc_fence_before();
      ptx::named_bar(kBarSoft, kSoftThreads);
      if (T == 0) F8_TRACE(18, sigma);
      ++sigma;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Barrier over the whole block, written out so that the two warpgroup
// branches below (which never rejoin until the end) can both use it.
__device__ __forceinline__ void block_bar() { ptx::named_bar(kBarBlock, kThreads); }

// The batch loop of one side of the register split: kSoft runs the softmax
// warps, !kSoft every other role and, at the end, the drains of the
// asynchronous arrivals.  Both sides take the same block barriers.
template <bool kSoft, bool kListed>
__device__ __forceinline__ void run_roles(const F8Params& P, const PartialParams& p, F8Ctl& c,
                                          uint8_t* base, int lo, int hi) {
  const int warp = threadIdx.x >> 5;
  uint32_t tau = 0, sigma = 0, pi = 0, o_commits = 0;
  uint32_t uses[kCodeStages] = {0, 0, 0}, fills[kCodeStages] = {0, 0, 0};
  int first = 0;
  while (true) {
    // the control block holds kMaxSegF8 segments: collect them in batches
    const int total = lo < hi ? collect_segments_n(p, lo, hi, first, kMaxSegF8, c) : 0;
    const int nseg = min(kMaxSegF8, total - first);
    if (nseg <= 0) break;
    if constexpr (kSoft) {
      softmax_role(p, c, base, nseg, tau, sigma, pi);
    } else {
      if (warp == kProdWarp) {
        producer_role<kListed>(P, p, c, base, nseg, tau, fills);
      } else if (warp == kQkWarp || warp == kQkWarp2) {
        if ((threadIdx.x & 31) == 0)
          qk_role<kListed>(warp == kQkWarp ? 0 : 1, p, c, base, nseg, tau, sigma);
      } else if (warp == kPvWarp) {
        if ((threadIdx.x & 31) == 0) pv_role<kListed>(p, c, base, nseg, tau, uses, o_commits);
      } else {
        staging_role<kListed>(p, c, base, nseg, tau, sigma);
      }
    }
    block_bar();
    if (c.abort) break;
    first += kMaxSegF8;
    if (total <= first) break;
  }
  if constexpr (!kSoft) {
    // Drain: every asynchronous arrival must land before the CTA exits (it
    // could otherwise hit the next CTA's barriers at the same addresses).
    // Normally only the last slot, P and Q releases are unconsumed; after a
    // timeout any commit or TMA fill may be.  Each wait is for the latest
    // phase of its barrier, so the parity is unambiguous.
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
      // tau counts the tiles this issuer handled; parts 5 tau of them,
      // commits on buffer k for every part number below 5 tau congruent to k
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
    // the last Q image copy (the staging warps count their requests in sigma)
    if (threadIdx.x == kStageWarp0 * 32 && sigma > 0) wait_or_abort(&c.q_full, (sigma - 1) & 1, c);
    // listed tiles: the staging threads' own row copies
    if (kListed && warp >= kStageWarp0 && warp < kStageWarp0 + kStageThreads / 32)
      ptx::cp_async_wait_all();
  }
}

template <bool kListed>
__global__ void __launch_bounds__(kThreads, 1) partial_f8_kernel(const __grid_constant__ F8Params P) {
  // dense only: a known-null index list lets the compiler drop the sparse
  // branches of the shared schedule
  PartialParams p = P.p;
  p.sparse_idx = nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  F8Ctl& c = *reinterpret_cast<F8Ctl*>(base + kOffCtl);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCodeStages; ++s) {
      ptx::mbar_init(&c.full[s], kListed ? 1 + kListedCopyArrivals : 1);
      ptx::mbar_init(&c.staged[s], kStageThreads / 32);
      ptx::mbar_init(&c.code_empty[s], 1);
    }
    for (int s = 0; s < kRopeStages; ++s) ptx::mbar_init(&c.rope_empty[s], 1);
    for (int k = 0; k < kParts; ++k) {
      ptx::mbar_init(&c.part_full[k], 1);
      ptx::mbar_init(&c.part_empty[k], kSoftWarps);
    }
    for (int s = 0; s < 2; ++s) ptx::mbar_init(&c.sc_empty[s], kSoftWarps);
    ptx::mbar_init(&c.p_full, kSoftWarps);
    ptx::mbar_init(&c.p_empty, 1);
    ptx::mbar_init(&c.o_full, 1);
    ptx::mbar_init(&c.q_full, kStageThreads / 32);
    // one commit from each score issuer, one arrival per softmax warp
    ptx::mbar_init(&c.q_empty, 2 + kSoftWarps);
    c.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) ptx::tmem_alloc(&c.tmem_base, kTmemCols);
  ptx::fence_proxy_async();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  int lo = 0, hi = 0;
  if (p.request_aligned) {
    int r0;
    uint32_t empties;
    request_range_tiles(p, c.warp_sums, &r0, &lo, &hi, &empties);
    // requests of the range with no row on this shard: the neutral (0, -inf)
    while (empties) {
      const int b = r0 + __ffs(empties) - 1;
      empties &= empties - 1;
      const size_t row0 = (size_t)b * p.rows_o;
      for (int k = threadIdx.x; k < p.heads * kVDim; k += kThreads)
        p.out[(row0 + k / kVDim) * kVDim + k % kVDim] = 0.f;
      if (threadIdx.x < p.heads) p.out_lse[row0 + threadIdx.x] = -CUDART_INF_F;
    }
  } else {
    const int T = total_tiles(p, c.warp_sums);
    const int tpc = T > 0 ? (T + p.num_ctas - 1) / p.num_ctas : 0;
    lo = blockIdx.x * tpc;
    hi = min(T, lo + tpc);
  }
  __syncthreads();

  // Register split: the launch gives every thread kLaunchRegs registers
  // (65,536 in all); the two softmax warpgroups take kSoftRegs and the two
  // others keep kOtherRegs.  Every warpgroup executes its adjustment here,
  // before any role can return, and the two branches stay apart until the
  // end so that each is compiled within its own budget.
  if (warp < kSoftWarps) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftRegs));
    run_roles<true, kListed>(P, p, c, base, lo, hi);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    run_roles<false, kListed>(P, p, c, base, lo, hi);
  }
  if (c.abort && threadIdx.x == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
  ptx::tc_fence_before();
  block_bar();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(c.tmem_base, kTmemCols);
}

// ------------------------------------------------------------- Q image ----

// Q operand images of every request (q_image.cuh).  Grid (batch, 2): each CTA
// covers 32 head rows with 8 threads per head.
__global__ void __launch_bounds__(256) f8_q_image_kernel(const PartialParams p, uint8_t* image) {
  qimg::build_q_image_row(p.q, p.rows_q, p.heads, blockIdx.x,
                          blockIdx.y * 32 + (threadIdx.x >> 3), threadIdx.x & 7, image);
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
  if (p.row_ids) {
    // listed rows: the cache as [blocks * 64][656] bytes, boxes one row high
    // (128-byte code and rope chunks for the four-row gathers)
    const cuuint64_t dims2[2] = {(cuuint64_t)kRowBytesFp8, (cuuint64_t)p.num_blocks * kBlock};
    const cuuint64_t strides2[1] = {(cuuint64_t)kRowBytesFp8};
    const cuuint32_t box2[2] = {128, 1};
    const cuuint32_t es2[2] = {1, 1};
    void* g2 = const_cast<uint8_t*>(p.kv);
    *scales = CUtensorMap{};
    return enc(rows, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, g2, dims2, strides2, box2, es2,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
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
bool g_attr_done[2][kMaxDevicesConfigured] = {};   // [listed rows][device]

}  // namespace

bool f8_supports(const PartialParams& p, int kv_dtype) {
  return kv_dtype == kKvFp8 && p.q_len == 1 && p.heads >= 1 && p.heads <= kMaxHeads &&
         p.sparse_idx == nullptr && encode_fn() != nullptr;
}

cudaError_t launch_partial_f8(const PartialParams& p, cudaStream_t st) {
  if (!p.q_image) return cudaErrorInvalidValue;
  F8Params fp;
  fp.p = p;
  if (!encode_maps(p, &fp.rows, &fp.scales)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesConfigured) return cudaErrorInvalidDevice;
  const int smem = (int)kSmemBytes;
  const bool listed = p.row_ids != nullptr;
  auto kernel = listed ? partial_f8_kernel<true> : partial_f8_kernel<false>;
  {
    // raise the shared-memory limit once per device and instantiation, so
    // that later launches (including ones captured into a CUDA graph) are
    // plain launches
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (!g_attr_done[listed][dev]) {
      // the in-kernel register split assumes exactly kLaunchRegs registers
      // per thread at launch; with fewer, the softmax warpgroups' increase
      // could never be granted
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, kernel);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != kLaunchRegs || fa.maxThreadsPerBlock < kThreads)
        return cudaErrorInvalidDeviceFunction;
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      g_attr_done[listed][dev] = true;
    }
  }
  if (!p.q_image_ready) f8_q_image_kernel<<<dim3(p.batch, 2), 256, 0, st>>>(p, p.q_image);
  kernel<<<p.num_ctas, kThreads, smem, st>>>(fp);
  return cudaGetLastError();
}

}  // namespace dcpmla

#ifdef DCPMLA_F8_TRACE
extern "C" int f8_trace_read(long long* host) {
  return (int)cudaMemcpyFromSymbol(host, dcpmla::g_f8_trace, sizeof(long long) * 24 * 256);
}
#endif

// Tensor-core kernel (tcgen05 / TMEM, sm_100a) for one shard's partial
// attention with its LSE.
//
// What it computes is the same as the CUDA-core kernel: for each request, the
// softmax over this shard's tokens of scale * <q_h, k_t> (576 values) applied
// to the first 512 values of the rows, plus LSE = ln sum_t exp(score)
// ("GLM-5.2 vLLM Decode Context Parallelism", sections "See why vLLM 0.26.0
// fails" and "Separate the backend merge from stable"; round-robin ownership
// from "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s",
// "The core design").
//
// How (per CTA, one per SM, persistent over its slice of the tile space):
//  * The tensor-core operands are fp16 with fp32 accumulation: bf16 cache
//    values convert to fp16 exactly (within +-65504), e4m3 * scale rounds to
//    11 significant bits (8x finer than bf16), and P keeps 11 bits too.
//    Values beyond the fp16 range are clamped and flagged.
//  * Q of the current request (64 heads padded, 576 values) sits in shared
//    memory, 128-byte swizzled, as the A operand of S = Q K^T.
//  * A tile is one cache block (64 local tokens).  Two stages, each of nine
//    8 KB chunk slots (8 latent chunks of 64 values, then rope), hold
//    consecutive tiles, swizzled for the tensor core.  Eight converter warps
//    load each tile's rows into registers one tile ahead, decode them (bf16
//    or e4m3 * scale -> fp16) and store them once a stage is free; raw cache
//    bytes never occupy shared memory.  A stage is published in five parts
//    (the four 128-value scale groups, then the rope), and the scores of each
//    part are issued as soon as it lands.
//  * S = Q K^T: 36 weight-stationary MMAs (M = 64 heads, N = 64 tokens,
//    K = 16) into one of two TMEM score buffers; the 2x2 data path puts head
//    h at TMEM lane h for tokens 0..31 and lane 64 + h for tokens 32..63.
//    The scores of tile t + 1 are computed while the softmax of tile t runs.
//  * Four softmax warps (one TMEM lane each) run the online softmax in base 2
//    with a lazily updated running max (the output is only rescaled, warp by
//    warp, when the max grows by more than 2^8), write P into the stage's
//    rope slot, which the scores no longer need, and keep the running sum.
//    With several query tokens per request (rows = q_len x heads) each row
//    also masks the tokens beyond its query's causal limit.
//  * O += P V: 8 MMAs (M = 64, N = 256 dims, K = 16 tokens) reading V from the
//    same chunk slots as an MN-major operand; O (64 x 512 fp32) stays in TMEM
//    for the whole request and is normalised in the epilogue.
//  * The kernel is instantiated per row format and per dense / sparse mode,
//    so the dense kernels carry no sparse addressing code.
#include <cuda_fp8.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "tc_ptx.cuh"

namespace dcpmla {
namespace {

constexpr int kThreads = 416;          // 13 warps: 4 softmax, 1 MMA issue, 8 converters
constexpr int kMmaWarp = 4;
constexpr int kConvBase = 160;         // first converter thread
constexpr int kConvThreads = 256;
constexpr int kTileTok = 64;           // one cache block
constexpr int kSlotBytes = 8192;       // 64 rows x 128 bytes
constexpr int kNumSlots = 9;           // per stage: 8 latent chunks + rope (then P)
constexpr int kRopeSlot = 8;
constexpr int kStages = 2;
constexpr int kQBytes = 9 * 8192;
// A stage is filled, and its scores issued, in five parts: the four 128-value
// scale groups of the latent row (two 64-value chunk slots each, 8 K-steps)
// and the rope slot (4 K-steps).  The MMA starts on a part as soon as it
// lands, so little of QK is left once the last part is stored.
constexpr int kParts = 5;
constexpr int kRopePart = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256;        // S buffers: columns [256, 288) and [288, 320); O: [0, 256)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;
constexpr int kPrefetchTiles = 6;      // L2 prefetch distance, in tiles
constexpr int kFlagTimeout = 4;
constexpr int kFlagRange = 8;
constexpr float kF16Max = 65504.f;

struct TcCtl {
  uint64_t full[kStages][kParts]; // converter -> MMA, per stage and part (256 arrivals)
  uint64_t empty[kStages][2];    // MMA -> converter, per stage and slot half (PV commits)
  uint64_t s_full[2];            // scores buffer ready (QK commit)
  uint64_t p_full[kStages];      // P written (128 softmax arrivals)
  uint64_t o_full;               // last PV of a request complete (commit, once per request)
  uint64_t q_full, q_empty;      // Q loaded (256 arrivals) / last QK of a request done
  uint32_t tmem_base;
  int abort;
  uint32_t row_mask[kStages][2];
  float red[2][2][64];
  float lred[2][64];
  int sel_count;
  int warp_sums[16];
  Segment seg[kSchedMaxSeg];
};

constexpr size_t kSmemBytes =
    kQBytes + (size_t)kStages * kNumSlots * kSlotBytes + sizeof(TcCtl) + 1024;


__device__ __forceinline__ uint32_t swz(int row, int unit) {
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((unit ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint8_t* slot_ptr(uint8_t* sslot, int stage, int c) {
  return sslot + (stage * kNumSlots + c) * kSlotBytes;
}


// Address of row r of tile `tile` of the segment, or nullptr if it is past
// the end or its block-table entry is out of range (flagged).
template <int KV>
__device__ __forceinline__ const uint8_t* tile_row(const PartialParams& p, const SegView& v,
                                                  const int* list, int tile, int r) {
  constexpr int kRowBytes = KV == kKvBf16 ? kRowBytesBf16 : kRowBytesFp8;
  const int i = tile * kTileTok + r;
  if (i >= v.nrows) return nullptr;
  const int j = p.sparse_idx ? list[i] : v.row_begin + i;   // list: written by this CTA, no __ldg
  const int blk = tile_block(p, v.b, j >> 6);
  if (blk < 0) return nullptr;
  return p.kv + ((size_t)blk * kBlock + (j & 63)) * kRowBytes;
}

// Addresses of N rows (rows[i]) of tile t, without serialising dependent
// loads: a dense tile is one cache block (one table load for all rows);
// sparse rows load all their list entries, then all their table entries.
// Invalid rows (past the end, or a flagged table entry) give nullptr.
template <int KV, int N>
__device__ __forceinline__ void tile_rows(const PartialParams& p, const SegView& v,
                                          const int* list, int t, const int (&rows)[N],
                                          const uint8_t* (&out)[N]) {
  constexpr int kRowBytes = KV == kKvBf16 ? kRowBytesBf16 : kRowBytesFp8;
  const int nvalid = v.nrows - t * kTileTok;
  if (!p.sparse_idx) {
    const int blk = tile_block(p, v.b, (v.row_begin >> 6) + t);
    const uint8_t* base = blk >= 0 ? p.kv + (size_t)blk * kBlock * kRowBytes : nullptr;
#pragma unroll
    for (int i = 0; i < N; ++i)
      out[i] = (base && rows[i] < nvalid) ? base + rows[i] * kRowBytes : nullptr;
  } else {
    int j[N], blk[N];
#pragma unroll
    for (int i = 0; i < N; ++i) j[i] = rows[i] < nvalid ? list[t * kTileTok + rows[i]] : -1;
#pragma unroll
    for (int i = 0; i < N; ++i)
      blk[i] = j[i] >= 0 ? __ldg(p.block_table + (size_t)v.b * p.bt_stride + (j[i] >> 6)) : -1;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const bool ok = blk[i] >= 0 && (long long)blk[i] < p.num_blocks;
      if (j[i] >= 0 && !ok && p.flags) atomicOr(p.flags, kFlagBadBlock);
      out[i] = ok ? p.kv + ((size_t)blk[i] * kBlock + (j[i] & 63)) * kRowBytes : nullptr;
    }
  }
}

// Asks L2 for the rows of tile t of the segment (a dense tile is one
// contiguous cache block: one bulk prefetch; sparse rows one by one).
template <int KV>
__device__ __forceinline__ void prefetch_tile(const PartialParams& p, const SegView& v,
                                              const int* list, int t, int ct) {
  constexpr int kRowBytes = KV == kKvBf16 ? kRowBytesBf16 : kRowBytesFp8;
  if (!p.sparse_idx) {
    if (ct == 0) {
      const int blk = tile_block(p, v.b, (v.row_begin >> 6) + t);
      if (blk >= 0) {
        const int rows = min(kTileTok, v.nrows - t * kTileTok);
        ptx::prefetch_l2(p.kv + (size_t)blk * kBlock * kRowBytes, (uint32_t)(rows * kRowBytes));
      }
    }
  } else if (ct < kTileTok) {
    const int rr[1] = {ct};
    const uint8_t* rp[1];
    tile_rows<KV, 1>(p, v, list, t, rr, rp);
    if (rp[0]) ptx::prefetch_l2(rp[0], kRowBytes);
  }
}


// fp32 pair -> fp16 pair (lo in the low half), rounded to nearest, clamped
// to +-65504.
__device__ __forceinline__ uint32_t f16x2_sat(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// e4m3 pair (16 bits) -> fp16 pair, exact.
__device__ __forceinline__ __half2 e4m3x2_to_f16x2(uint32_t pair) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(pair & 0xFFFFu), __NV_E4M3);
  __half2 h2;
  *reinterpret_cast<__half2_raw*>(&h2) = hr;
  return h2;
}

// Scales outside the fp16 fast path (rare): fp32 products rounded once,
// with clamping, stored to dst_lo / dst_hi; returns true if a product was
// clamped.  Kept out of line so the hot conversion code stays small; it
// stores its results itself so that the caller's values never need an
// address (a by-reference result would put them in local memory on every
// call, fast path included).
__device__ __noinline__ bool e4m3x16_to_f16_slow(const uint4 v, float sc, uint4* dst_lo,
                                                 uint4* dst_hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      const float2 f = __half22float2(e4m3x2_to_f16x2(w[i] >> (16 * hw)));
      const float a = f.x * sc, b = f.y * sc;
      amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
      o[2 * i + hw] = f16x2_sat(a, b);
    }
  }
  *dst_lo = make_uint4(o[0], o[1], o[2], o[3]);
  *dst_hi = make_uint4(o[4], o[5], o[6], o[7]);
  return amax > kF16Max;
}

// 16 e4m3 codes times `sc` -> 16 fp16 stored as two 16-byte units (dims in
// order) at dst_lo and dst_hi.
// e4m3 -> fp16 is exact.  When every product stays a finite normal-range
// fp16 number (2^-14 <= sc <= 65504 / 448) the product is taken in fp16 with
// the scale split into sc_hi = fp16(sc) and sc_lo = fp16(sc - sc_hi):
// fma(code, sc_hi, code * sc_lo) rounds once per element.  Rounding the scale
// alone would put one shared relative error (up to 2^-11) on all 128 values
// of a group, which moves large scores coherently.  Other scales take the
// fp32 product, rounded once, with clamping.  Returns true if a product was
// clamped (only possible off the fast path).
__device__ __forceinline__ bool e4m3x16_to_f16(const uint4 v, float sc, uint4* dst_lo,
                                               uint4* dst_hi) {
  if (!(sc >= 6.103515625e-05f && sc <= 146.0f))
    return e4m3x16_to_f16_slow(v, sc, dst_lo, dst_hi);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
  const __half s_hi = __float2half_rn(sc);
  const __half2 hi2 = __half2half2(s_hi);
  const __half2 lo2 = __half2half2(__float2half_rn(sc - __half2float(s_hi)));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int hw = 0; hw < 2; ++hw) {
      const __half2 h2 = e4m3x2_to_f16x2(w[i] >> (16 * hw));
      const __half2 r2 = __hfma2(h2, hi2, __hmul2(h2, lo2));
      o[2 * i + hw] = *reinterpret_cast<const uint32_t*>(&r2);
    }
  }
  *dst_lo = make_uint4(o[0], o[1], o[2], o[3]);
  *dst_hi = make_uint4(o[4], o[5], o[6], o[7]);
  return false;
}

// 8 bf16 -> 8 fp16; `amax` collects the largest magnitude seen.
__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4 v, float& amax) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xFFFF0000u);
    amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
    o[i] = f16x2_sat(a, b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------- roles -------

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, TcCtl& c) {
  return ptx::mbar_wait(bar, parity, &c.abort);
}

// Shared-memory descriptors differ only in their start-address field (bits
// 0..13, address / 16), so each MMA's descriptors are a base plus a constant:
// the issuing thread spends one 32-bit add per operand.
struct Descs {
  uint64_t q;           // Q chunk 0, K-major
  uint64_t k[kStages];  // chunk slot 0 of each stage, K-major (QK operand B)
  uint64_t p[kStages];  // P (rope slot) of each stage, K-major (PV operand A)
  uint64_t v[kStages];  // chunk slot 0 of each stage, MN-major (PV operand B)
};

__device__ __forceinline__ uint64_t dplus(uint64_t d, uint32_t byte_off) {
  return d + (uint64_t)(byte_off >> 4);
}

// MMA issue (one thread): S[tau & 1] = Q K^T for tile tau (stage tau & 1),
// part by part as the converters publish them (K-steps 8k .. 8k+7 for scale
// group k, 32 .. 35 for the rope).
template <int kPart>
__device__ __forceinline__ void issue_qk_part(const TcCtl& c, const Descs& d, uint64_t kd,
                                              uint32_t dst) {
  constexpr uint32_t kIdQK = ptx::idesc_f16(64, 64, false);
  constexpr int k0 = 8 * kPart, k1 = kPart == kRopePart ? 36 : 8 * kPart + 8;
#pragma unroll
  for (int ks = k0; ks < k1; ++ks)
    ptx::mma_ws_f16(dst, dplus(d.q, (ks >> 2) * 8192 + (ks & 3) * 32),
                    dplus(kd, (ks >> 2) * kSlotBytes + (ks & 3) * 32), kIdQK, ks > 0);
}

__device__ __forceinline__ bool issue_qk(TcCtl& c, const Descs& d, uint32_t tau) {
  const int st = tau & 1;
  const uint32_t ph = (tau >> 1) & 1;
  const uint64_t kd = st ? d.k[1] : d.k[0];
  const uint32_t dst = c.tmem_base + kColS + 32 * st;
  if (!wait_or_abort(&c.full[st][0], ph, c)) return false;
  ptx::tc_fence_after();
  issue_qk_part<0>(c, d, kd, dst);
  if (!wait_or_abort(&c.full[st][1], ph, c)) return false;
  ptx::tc_fence_after();
  issue_qk_part<1>(c, d, kd, dst);
  if (!wait_or_abort(&c.full[st][2], ph, c)) return false;
  ptx::tc_fence_after();
  issue_qk_part<2>(c, d, kd, dst);
  if (!wait_or_abort(&c.full[st][3], ph, c)) return false;
  ptx::tc_fence_after();
  issue_qk_part<3>(c, d, kd, dst);
  if (!wait_or_abort(&c.full[st][kRopePart], ph, c)) return false;
  ptx::tc_fence_after();
  issue_qk_part<kRopePart>(c, d, kd, dst);
  ptx::mma_commit(&c.s_full[st]);
  return true;
}

// MMA issue (one thread): O (+)= P V for tile tau; frees the stage per half.
__device__ __forceinline__ void issue_pv(TcCtl& c, const Descs& d, uint32_t tau, bool first_tile) {
  constexpr uint32_t kIdPV = ptx::idesc_f16(64, 256, true);
  const int st = tau & 1;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      ptx::mma_ws_f16(c.tmem_base + hf * 128, dplus(st ? d.p[1] : d.p[0], kk * 32),
                      dplus(st ? d.v[1] : d.v[0], 4 * hf * kSlotBytes + kk * 2048), kIdPV,
                      (!first_tile || kk > 0) ? 1u : 0u);
    ptx::mma_commit(&c.empty[st][hf]);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Issues every MMA (one thread of the MMA warp): the scores of the next tile
// before the PV of this one, so that the softmax of tile t overlaps the
// scores of tile t + 1.
__device__ __forceinline__ void mma_role(const PartialParams& p, TcCtl& c, uint8_t* sq, uint8_t* sslot, int nseg,
                         uint32_t& tau, uint32_t& sigma, uint32_t (&uses)[2]) {
  Descs dsc;
  {
    const uint32_t q0 = ptx::smem_addr(sq), s0 = ptx::smem_addr(sslot);
    dsc.q = ptx::sdesc_sw128(q0, 16, 1024);
    for (int st = 0; st < kStages; ++st) {
      const uint32_t base = s0 + st * kNumSlots * kSlotBytes;
      dsc.k[st] = ptx::sdesc_sw128(base, 16, 1024);
      dsc.p[st] = ptx::sdesc_sw128(base + kRopeSlot * kSlotBytes, 16, 1024);
      dsc.v[st] = ptx::sdesc_sw128(base, kSlotBytes, 1024);
    }
  }
  TileCursor cur, ahead;
  if (!cur.start(p, c, nseg)) return;
  ahead = cur;
  if (!wait_or_abort(&c.q_full, sigma & 1, c)) return;
  if (!issue_qk(c, dsc, tau)) return;
  if (ahead.last_of_segment()) ptx::mma_commit(&c.q_empty);
  uint32_t sigma_ahead = sigma;
  while (true) {
    const bool seg_end = ahead.last_of_segment();
    if (ahead.next(p, c)) {
      if (seg_end) {
        ++sigma_ahead;
        if (!wait_or_abort(&c.q_full, sigma_ahead & 1, c)) return;
      }
      if (!issue_qk(c, dsc, tau + 1)) return;
      if (ahead.last_of_segment()) ptx::mma_commit(&c.q_empty);
    }
    const int st = tau & 1;
    if (!wait_or_abort(&c.p_full[st], (tau >> 1) & 1, c)) return;
    ptx::tc_fence_after();
    issue_pv(c, dsc, tau, cur.t == 0);
    ++uses[st];
    if (cur.last_of_segment()) {
      ptx::mma_commit(&c.o_full);
      ++sigma;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Online softmax, P and the epilogue (128 threads, one TMEM lane each).
__device__ __forceinline__ void softmax_role(const PartialParams& p, TcCtl& c, uint8_t* sslot, int nseg,
                             uint32_t& tau, uint32_t& sigma) {
  const int L = threadIdx.x;                 // 0..127
  const int h = L & 63, half = L >> 6;
  const int warp = L >> 5;
  const uint32_t lane_base = c.tmem_base + ((uint32_t)(warp * 32) << 16);
  const float sl2 = p.scale * kLog2e;

  // sparse CTAs whose list is empty write the neutral pair and stop
  if (p.sparse_idx && seg_view(p, c, 0).ntiles == 0) {
    const SegView v = seg_view(p, c, 0);
    const size_t slot = v.whole ? (size_t)v.b : (size_t)blockIdx.x;
    if (h < p.heads) {
      const size_t row = slot * (v.whole ? p.rows_o : p.heads) + h;
      float* o = (v.whole ? p.out : p.ws_o) + row * kVDim;
      for (int i = half; i < kVDim / 4; i += 2)
        reinterpret_cast<float4*>(o)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (half == 0) (v.whole ? p.out_lse : p.ws_lse)[row] = -CUDART_INF_F;
    }
    return;
  }

  TileCursor cur;
  if (!cur.start(p, c, nseg)) return;
  float m_used = -CUDART_INF_F, l = 0.f;
  int jmax = 0;                              // multi-query: last local row this row may see
  while (true) {
    const int st = tau & 1;
    const uint32_t ph = (tau >> 1) & 1;
    if (!wait_or_abort(&c.s_full[st], ph, c)) return;
    if (!wait_or_abort(&c.full[st][kRopePart], ph, c)) return;   // row mask of the tile
    __syncwarp();
    ptx::tc_fence_after();
    uint32_t sr[32];
    ptx::tmem_ld32(lane_base + kColS + 32 * st, sr);
    ptx::tmem_wait_ld();
    uint32_t mw = c.row_mask[st][half];
    if (p.q_len > 1) {
      // Causal rows: row h is query i = h / (heads / q_len) at global position
      // L_b - q_len + i; it sees local rows j with j * N + shard <= that.
      if (cur.t == 0) {
        const int lim = max(seq_len_of(p, cur.v.b), 0) - p.q_len + h / (p.heads / p.q_len);
        jmax = lim >= p.shard ? (lim - p.shard) / p.nshards : -1;
      }
      const int cmax = jmax - (cur.v.row_begin + cur.t * kTileTok + half * 32);
      mw &= cmax >= 31 ? 0xffffffffu : (cmax < 0 ? 0u : ((2u << cmax) - 1u));
    }
    float x[32];
    float mloc = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      x[j] = ((mw >> j) & 1u) ? __uint_as_float(sr[j]) * sl2 : -CUDART_INF_F;
      mloc = fmaxf(mloc, x[j]);
    }
    const int par = tau & 1;
    c.red[par][half][h] = mloc;
    ptx::named_bar(1, 128);
    const float mnew = fmaxf(mloc, c.red[par][half ^ 1][h]);
    // Lazy rescale.  The TMEM loads/stores below are warp-collective, so the
    // decision is made per warp: if any head of the warp needs a new max,
    // every lane moves to max(m_used, mnew).  The partner warp (the other
    // token half) holds the same 32 heads and decides identically.
    const bool first = m_used == -CUDART_INF_F;
    const bool need = !first && mnew > m_used + kRescaleThreshold;
    const bool any_need = __any_sync(0xffffffffu, need);
    float alpha = 1.f;
    if (first) {
      m_used = mnew;
    } else if (any_need) {
      const float m2 = fmaxf(m_used, mnew);
      alpha = ex2(m_used - m2);
      m_used = m2;
      l *= alpha;
    }
    float sum = 0.f;
    uint32_t pk[16];
    const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;   // all masked: x = -inf -> p = 0
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float p0 = ex2(x[2 * j] - mu), p1 = ex2(x[2 * j + 1] - mu);
      sum += p0 + p1;
      const __half2 h2 = __floats2half2_rn(p0, p1);
      pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    l += sum;
    uint8_t* pslot = slot_ptr(sslot, st, kRopeSlot);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4*>(pslot + swz(h, 4 * half + u)) =
          make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    // O is rescaled after P is written, so that the scores are no longer held
    // in registers while O passes through them (P does not depend on O; it
    // only has to be in place before p_full, like the rescaled O).
    if (any_need) {
      // The previous tile's PV must have landed in O before it is rescaled:
      // its last MMA released the second half of its stage.  That barrier's
      // phase for tile tau - 1 is either pending or complete here (the
      // scores barrier implied PV(tau - 2); PV(tau + 1) needs this thread's
      // P), so the parity wait is unambiguous.
      const uint32_t prev = tau - 1;
      if (!wait_or_abort(&c.empty[prev & 1][1], (prev >> 1) & 1, c)) return;
      __syncwarp();
      ptx::tc_fence_after();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t r[32];
        const uint32_t addr = lane_base + (q >> 2) * 128 + (q & 3) * 32;
        ptx::tmem_ld32(addr, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        ptx::tmem_st32(addr, r);
      }
      ptx::tmem_wait_st();
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    ptx::mbar_arrive(&c.p_full[st]);
    // ---- epilogue after the request's last tile
    if (cur.last_of_segment()) {
      const SegView& v = cur.v;
      const size_t slot = v.whole ? (size_t)v.b
                                  : (p.sparse_idx ? (size_t)blockIdx.x : (size_t)blockIdx.x + v.b);
      const size_t row = slot * (v.whole ? p.rows_o : p.heads) + h;
      float* o_base = (v.whole ? p.out : p.ws_o) + row * kVDim;
      float* l_base = (v.whole ? p.out_lse : p.ws_lse) + row;
      // o_full completes once per request, after its last PV (and so after
      // all of its PVs).  Earlier phases were consumed by earlier epilogues and
      // the next one needs this thread's P, so the parity wait is unambiguous.
      if (!wait_or_abort(&c.o_full, sigma & 1, c)) return;
      __syncwarp();
      ptx::tc_fence_after();
      c.lred[half][h] = l;
      ptx::named_bar(1, 128);
      const float ltot = l + c.lred[half ^ 1][h];
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
      // Each lane holds 32 values of its head's row per TMEM load; eight
      // lanes exchange them (an 8 x 8 transpose of 16-byte pieces in three
      // butterfly steps) so that the eight pieces of one row leave together
      // as a whole 128-byte line, instead of every store touching 32 lines.
      const int i8 = L & 7, row8 = L & 24;   // place in, and first lane of, the group of 8
      float* o_rows = (v.whole ? p.out : p.ws_o) + (row - h + (h & ~31) + row8) * kVDim;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) {
        uint32_t r[32];
        ptx::tmem_ld32(lane_base + (q >> 2) * 128 + (q & 3) * 32, r);
        ptx::tmem_wait_ld();
        float4 piece[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          piece[e] = make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                 __uint_as_float(r[4 * e + 2]) * inv,
                                 __uint_as_float(r[4 * e + 3]) * inv);
#pragma unroll
        for (int m = 4; m >= 1; m >>= 1) {
          const bool upper = (i8 & m) != 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (e & m) continue;
            const float4 send = upper ? piece[e] : piece[e | m];
            float4 got;
            got.x = __shfl_xor_sync(0xffffffffu, send.x, m);
            got.y = __shfl_xor_sync(0xffffffffu, send.y, m);
            got.z = __shfl_xor_sync(0xffffffffu, send.z, m);
            got.w = __shfl_xor_sync(0xffffffffu, send.w, m);
            if (upper) piece[e] = got; else piece[e | m] = got;
          }
        }
        // piece[k] is now piece i8 of the row of lane row8 + k
        const int col = (q >> 2) * 256 + half * 128 + (q & 3) * 32 + 4 * i8;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if ((h & ~31) + row8 + k < p.heads)
            *reinterpret_cast<float4*>(o_rows + (size_t)k * kVDim + col) = piece[k];
      }
      if (h < p.heads && half == 0)
        *l_base = ltot > 0.f ? (m_used + log2f(ltot)) * kLn2 : -CUDART_INF_F;
      ptx::tc_fence_before();
      ptx::named_bar(1, 128);
      ++sigma;
      m_used = -CUDART_INF_F;
      l = 0.f;
    }
    ++tau;
    if (!cur.next(p, c)) break;
  }
}

// Rows of one tile held in a converter thread's registers between the
// global loads and the shared-memory stores.
template <int KV>
struct Stage;

// fp8: thread ct stages rows 32 i + (ct >> 3) (i = 0, 1) of the tile: of each
// 128-value scale group g, the 16-value unit u = ct & 7 of both rows with
// the group's scale, and rope unit u.  Eight threads cover a row, so each
// load is part of a contiguous 128-byte run of the row.
template <>
struct Stage<kKvFp8> {
  uint4 c[4][2];
  float s[4][2];
  uint4 rope[2];
};

// bf16: latent dims 0..255 (unit = lane) of rows 8 i + cw, then dims 256..511
// and rope, loaded once the first half is stored.
template <>
struct Stage<kKvBf16> {
  uint4 a[8];
  uint4 b[10];
};

__device__ __forceinline__ void stage_load(const PartialParams& p, const SegView& v,
                                           const int* list, int t, int ct, Stage<kKvFp8>& st) {
  const int u = ct & 7;
  const int rows[2] = {ct >> 3, 32 + (ct >> 3)};
  const uint8_t* rp[2];
  tile_rows<kKvFp8, 2>(p, v, list, t, rows, rp);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint8_t* row = rp[i];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      st.c[g][i] = row ? __ldg(reinterpret_cast<const uint4*>(row) + 8 * g + u) : make_uint4(0, 0, 0, 0);
      st.s[g][i] = row ? __ldg(reinterpret_cast<const float*>(row + 512) + g) : 0.f;
    }
    st.rope[i] = row ? __ldg(reinterpret_cast<const uint4*>(row + 528) + u) : make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void stage_load(const PartialParams& p, const SegView& v,
                                           const int* list, int t, int ct, Stage<kKvBf16>& st) {
  const int cw = ct >> 5, cl = ct & 31;
  int rows[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) rows[i] = 8 * i + cw;
  const uint8_t* rp[8];
  tile_rows<kKvBf16, 8>(p, v, list, t, rows, rp);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    st.a[i] = rp[i] ? __ldg(reinterpret_cast<const uint4*>(rp[i]) + cl) : make_uint4(0, 0, 0, 0);
}

// fp8 scale group g: latent dims 128 g .. 128 g + 127, chunk slots 2 g and
// 2 g + 1 of the stage.
template <int g>
__device__ __forceinline__ void stage_store_group(uint8_t* stage, int ct, const Stage<kKvFp8>& st,
                                                  bool& range_bad) {
  const int u = ct & 7;
  uint8_t* dst = stage + (2 * g + (u >> 2)) * kSlotBytes;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = 32 * i + (ct >> 3);
    range_bad |= e4m3x16_to_f16(st.c[g][i], st.s[g][i],
                                reinterpret_cast<uint4*>(dst + swz(r, (u & 3) * 2)),
                                reinterpret_cast<uint4*>(dst + swz(r, (u & 3) * 2 + 1)));
  }
}

// fp8 rope units (bf16 -> fp16) into the rope slot.
__device__ __forceinline__ void stage_store_rope(uint8_t* stage, int ct, const Stage<kKvFp8>& st,
                                                 bool& range_bad) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    *reinterpret_cast<uint4*>(stage + kRopeSlot * kSlotBytes + swz(32 * i + (ct >> 3), ct & 7)) =
        bf16x8_to_f16(st.rope[i], amax);
  range_bad |= amax > kF16Max;
}

// bf16, first half: latent chunks 0..3 of the stage.
__device__ __forceinline__ void stage_store_half0(uint8_t* stage, int ct, const Stage<kKvBf16>& st,
                                                  bool& range_bad) {
  const int cw = ct >> 5, cl = ct & 31;
  float amax = 0.f;
  uint8_t* dst = stage + (cl >> 3) * kSlotBytes;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    *reinterpret_cast<uint4*>(dst + swz(8 * i + cw, cl & 7)) = bf16x8_to_f16(st.a[i], amax);
  range_bad |= amax > kF16Max;
}

__device__ __forceinline__ void stage_load_half1(const PartialParams& p, const SegView& v,
                                                 const int* list, int t, int ct,
                                                 Stage<kKvBf16>& st) {
  int rows[10];
#pragma unroll
  for (int i = 0; i < 10; ++i) rows[i] = (i * kConvThreads + ct) / 40;
  const uint8_t* rp[10];
  tile_rows<kKvBf16, 10>(p, v, list, t, rows, rp);
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const int U = i * kConvThreads + ct;
    st.b[i] = rp[i] ? __ldg(reinterpret_cast<const uint4*>(rp[i]) + 32 + U % 40)
                    : make_uint4(0, 0, 0, 0);
  }
}

// bf16, second half: latent chunks 4..7 and the rope slot.
__device__ __forceinline__ void stage_store_half1(uint8_t* stage, int ct, const Stage<kKvBf16>& st,
                                                  bool& range_bad) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const int U = i * kConvThreads + ct;
    const int r = U / 40, u = 32 + U % 40;
    *reinterpret_cast<uint4*>(stage + (u >> 3) * kSlotBytes + swz(r, u & 7)) =
        bf16x8_to_f16(st.b[i], amax);
  }
  range_bad |= amax > kF16Max;
}

// Q of request b into the Q region: 64 rows x 72 units of fp16, heads >= H zero.
__device__ __forceinline__ void load_q(const PartialParams& p, int b, uint8_t* sq, int ct,
                                       bool& range_bad) {
  const uint4* qb = reinterpret_cast<const uint4*>(p.q + (size_t)b * p.rows_q * kHeadDim);
  float amax = 0.f;
#pragma unroll 6
  for (int i = 0; i < 18; ++i) {
    const int U = i * kConvThreads + ct;
    const int row = U / 72, u = U % 72;
    const uint4 v = row < p.heads ? __ldg(qb + (size_t)row * 72 + u) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(sq + (u >> 3) * 8192 + swz(row, u & 7)) = bf16x8_to_f16(v, amax);
  }
  range_bad |= amax > kF16Max;
}

// Fills Q and the two stages (256 threads), one tile ahead in registers, and
// publishes each stage in kParts parts (fp8: per scale group, then rope).
template <int KV>
__device__ __forceinline__ void convert_role(const PartialParams& p, TcCtl& c, uint8_t* sq, uint8_t* sslot,
                             const int* list, int nseg, uint32_t& tau, uint32_t& sigma) {
  const int ct = threadIdx.x - kConvBase;      // 0..255
  const int cw = ct >> 5, cl = ct & 31;
  bool range_bad = false;
  Stage<KV> stg;
  TileCursor cur, pf;
  if (!cur.start(p, c, nseg)) return;
  // The first tile's rows and, at the very start, the first request's Q are
  // requested before the L2 prefetch burst of the next tiles: at kernel start
  // every CTA prefetches at once, and loads issued after that burst would
  // queue behind it.
  stage_load(p, cur.v, list, cur.t, ct, stg);
  bool q_loaded = false;
  if (sigma == 0) {                          // no earlier request's Q to wait for
    load_q(p, cur.v.b, sq, ct, range_bad);
    ptx::fence_proxy_async();
    ptx::mbar_arrive(&c.q_full);
    q_loaded = true;
  }
  // L2 prefetch runs kPrefetchTiles ahead of the tile being staged
  pf = cur;
  bool pf_ok = true;
  for (int i = 0; i < kPrefetchTiles && pf_ok; ++i) {
    prefetch_tile<KV>(p, pf.v, list, pf.t, ct);
    pf_ok = pf.next(p, c);
  }
  while (true) {
    const int st = tau & 1;
    uint8_t* stage = slot_ptr(sslot, st, 0);
    const bool reuse = tau >= 2;                           // stage used before: wait for its PV
    const uint32_t eph = ((tau >> 1) + 1) & 1;             // phase of the PV two tiles back
    if (cur.t == 0 && !q_loaded) {
      // new request: its Q replaces the previous one once that one's last QK is done
      if (sigma > 0 && !wait_or_abort(&c.q_empty, (sigma - 1) & 1, c)) break;
      load_q(p, cur.v.b, sq, ct, range_bad);
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&c.q_full);
    }
    q_loaded = false;
    // chunks 0..3 (scale groups 0, 1) are free once the first PV half of the
    // tile two back is done, chunks 4..7 and the rope slot after the second
    if (reuse && !wait_or_abort(&c.empty[st][0], eph, c)) break;
    // test only: withholding the very first arrival makes every pipeline wait
    // of the CTA run out, which exercises the timeout path
    const bool withhold = p.test_withhold && tau == 0;
    if constexpr (KV == kKvFp8) {
      stage_store_group<0>(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      if (!withhold) ptx::mbar_arrive(&c.full[st][0]);
      stage_store_group<1>(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&c.full[st][1]);
    } else {
      stage_store_half0(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      if (!withhold) ptx::mbar_arrive(&c.full[st][0]);
      ptx::mbar_arrive(&c.full[st][1]);
      stage_load_half1(p, cur.v, list, cur.t, ct, stg);
    }
    if (reuse && !wait_or_abort(&c.empty[st][1], eph, c)) break;
    if constexpr (KV == kKvFp8) {
      stage_store_group<2>(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&c.full[st][2]);
      stage_store_group<3>(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&c.full[st][3]);
      stage_store_rope(stage, ct, stg, range_bad);
    } else {
      stage_store_half1(stage, ct, stg, range_bad);
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&c.full[st][2]);
      ptx::mbar_arrive(&c.full[st][3]);
    }
    if (ct < 64) {                                         // valid-row mask, published with the rope
      const int rr[1] = {ct};
      const uint8_t* rp[1];
      tile_rows<KV, 1>(p, cur.v, list, cur.t, rr, rp);
      const uint32_t m = __ballot_sync(0xffffffffu, rp[0] != nullptr);
      if (cl == 0) c.row_mask[st][cw] = m;
    }
    ptx::fence_proxy_async();
    ptx::mbar_arrive(&c.full[st][kRopePart]);
    ++tau;
    const bool seg_end = cur.last_of_segment();
    if (seg_end) ++sigma;
    if (!cur.next(p, c)) break;
    if (pf_ok) {
      prefetch_tile<KV>(p, pf.v, list, pf.t, ct);
      pf_ok = pf.next(p, c);
    }
    stage_load(p, cur.v, list, cur.t, ct, stg);
  }
  if (range_bad && p.flags) atomicOr(p.flags, kFlagRange);
}

// kSparse is fixed per instantiation: the dense kernel sees a null index
// list at compile time, so none of the sparse paths are compiled into it
// (a smaller kernel keeps its four concurrent roles in the instruction cache).
template <int KV, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1) partial_tc_kernel(const PartialParams pin) {
  PartialParams p = pin;
  if constexpr (!kSparse) p.sparse_idx = nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = base;
  uint8_t* sslot = base + kQBytes;
  TcCtl& c = *reinterpret_cast<TcCtl*>(base + kQBytes + kStages * kNumSlots * kSlotBytes);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      for (int k = 0; k < kParts; ++k)
        ptx::mbar_init(&c.full[s][k], kConvThreads);    // every converter thread, once per fill
      for (int hf = 0; hf < 2; ++hf) ptx::mbar_init(&c.empty[s][hf], 1);   // one commit per PV half
      ptx::mbar_init(&c.p_full[s], 128);
      ptx::mbar_init(&c.s_full[s], 1);
    }
    ptx::mbar_init(&c.o_full, 1);
    ptx::mbar_init(&c.q_full, kConvThreads);
    ptx::mbar_init(&c.q_empty, 1);
    c.abort = 0;
  }
  if (warp == 0) ptx::tmem_alloc(&c.tmem_base, kTmemCols);
  ptx::fence_proxy_async();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  const int* list = nullptr;
  int lo = 0, hi = 0;
  if (p.sparse_idx) {
    const int chunk = (p.topk + p.sparse_parts - 1) / p.sparse_parts;
    int* my_list = p.ws_list + (size_t)blockIdx.x * chunk;
    const int n = compact_sparse(p, my_list, c);
    if (threadIdx.x == 0) c.sel_count = n;
    list = my_list;
  } else {
    const int T = total_tiles(p, c.warp_sums);
    const int tpc = T > 0 ? (T + p.num_ctas - 1) / p.num_ctas : 0;
    lo = blockIdx.x * tpc;
    hi = min(T, lo + tpc);
  }
  __syncthreads();

  uint32_t tau = 0, sigma = 0;
  uint32_t uses[2] = {0, 0};
  uint32_t sigma_issuer = 0;
  int first = 0;
  while (true) {
    int nseg, total;
    if (p.sparse_idx) {
      nseg = total = 1;
    } else {
      total = lo < hi ? collect_segments(p, lo, hi, first, c) : 0;
      nseg = min(kSchedMaxSeg, total - first);
    }
    if (nseg <= 0) break;
    if (warp < 4) {
      softmax_role(p, c, sslot, nseg, tau, sigma);
    } else if (warp == kMmaWarp) {
      if ((threadIdx.x & 31) == 0) {
        mma_role(p, c, sq, sslot, nseg, tau, sigma, uses);
        sigma_issuer = sigma;
      }
    } else {
      convert_role<KV>(p, c, sq, sslot, list, nseg, tau, sigma);
    }
    __syncthreads();
    if (c.abort) break;
    first += kSchedMaxSeg;
    if (p.sparse_idx || total <= first) break;
  }
  // Drain: every tcgen05.commit arrives on its mbarrier asynchronously.  The
  // stage releases of the last tiles and the last request's Q release are
  // never waited on by the pipeline, so wait for them here; otherwise an
  // arrival could land after this CTA exits, on the barriers the next CTA on
  // this SM has just initialised at the same shared-memory offsets.  (Every
  // other commit is consumed: scores by the softmax, o_full by the epilogue.)
  // Each of these waits is one phase ahead of the last one consumed, so the
  // parity is unambiguous.
  if (threadIdx.x == kMmaWarp * 32) {
    for (int s = 0; s < kStages; ++s)
      if (uses[s] > 0)
        for (int hf = 0; hf < 2; ++hf) wait_or_abort(&c.empty[s][hf], (uses[s] - 1) & 1, c);
    if (sigma_issuer > 0) wait_or_abort(&c.q_empty, (sigma_issuer - 1) & 1, c);
  }
  if (c.abort && threadIdx.x == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(c.tmem_base, kTmemCols);
}

}  // namespace

bool tc_supports(const PartialParams& p, int kv_dtype) {
  (void)kv_dtype;
  return p.heads >= 1 && p.heads <= kMaxHeads;
}

cudaError_t launch_partial_tc(const PartialParams& p, int kv_dtype, cudaStream_t st) {
  const int grid = p.sparse_idx ? p.batch * p.sparse_parts : p.num_ctas;
  const int smem = (int)kSmemBytes;
  const bool sparse = p.sparse_idx != nullptr;
  auto kernel = kv_dtype == kKvBf16
                    ? (sparse ? partial_tc_kernel<kKvBf16, true> : partial_tc_kernel<kKvBf16, false>)
                    : (sparse ? partial_tc_kernel<kKvFp8, true> : partial_tc_kernel<kKvFp8, false>);
  // Raise the shared-memory limit once per kernel and device, so that later
  // launches (including ones captured into a CUDA graph) are plain launches.
  // The record is guarded: host threads may make their first calls at once.
  static std::mutex mu;
  static bool configured[4][kMaxDevicesConfigured] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesConfigured) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    bool& done = configured[(kv_dtype == kKvBf16 ? 0 : 2) + (sparse ? 1 : 0)][dev];
    if (!done) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      done = true;
    }
  }
  kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

size_t tc_smem_bytes() { return kSmemBytes; }

}  // namespace dcpmla

// C ABI of libdcpmla.so: argument checks, work decomposition and launches.
// The entry points are declared (and their contracts stated) in dcpmla.h.
#include "dcpmla.h"

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"

namespace dcpmla {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count_current(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DCPMLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevicesConfigured) return DCPMLA_ERR_UNSUPPORTED;
  // per-device cache; host threads may ask at once, so each entry is atomic
  static std::atomic<int> cache[kMaxDevicesConfigured];
  const int c = cache[dev].load(std::memory_order_relaxed);
  if (c > 0) {
    *out = c;
    return DCPMLA_OK;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return DCPMLA_ERR_CUDA;
  cache[dev].store(n, std::memory_order_relaxed);
  *out = n;
  return DCPMLA_OK;
}

// CTAs sharing one shard's dense tile space.
int resolve_ctas(int num_splits, int* ctas) {
  if (num_splits > 0) {
    *ctas = num_splits;
    return DCPMLA_OK;
  }
  return sm_count_current(ctas);
}

// Index-list chunks per request in sparse mode: enough CTAs to cover the
// device when the batch is small, and chunks short enough for the kernels'
// on-chip selection lists.
int sparse_parts_for(int batch, int topk, int ctas) {
  const int cap = simt_sparse_chunk_max();
  int p = (topk + cap - 1) / cap;
  int fill = batch > 0 ? ctas / batch : 1;
  if (fill > p) p = fill;
  if (p > topk) p = topk;
  return p < 1 ? 1 : p;
}

long long slots_for(int batch, int topk, int ctas) {
  if (topk > 0) return (long long)batch * sparse_parts_for(batch, topk, ctas);
  return (long long)ctas + batch;
}

// Sparse mode: room for every CTA's list of selected local rows.
long long list_ints_for(int batch, int topk, int ctas) {
  if (topk <= 0) return 0;
  const int parts = sparse_parts_for(batch, topk, ctas);
  const long long chunk = (topk + parts - 1) / parts;
  return (long long)batch * parts * chunk;
}

// Sparse decode on the tensor-core kernels runs over gathered rows: room for
// every request's selections in whole 64-row blocks (rows sized for bf16, so
// that one size serves both formats) and for the per-request counts.
long long sparse_maxblk(int topk) { return (topk + kBlock - 1) / kBlock; }
size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t sparse_gather_rows_bytes(int batch, int topk) {
  return round256((size_t)batch * sparse_maxblk(topk) * kBlock * kRowBytesBf16);
}

// Workspace of one call: dense decode needs split slots and the e4m3
// kernel's Q images; sparse decode needs either the CUDA-core kernel's layout
// (a slot and a list chunk per CTA) or the gathered rows with dense split
// slots and the Q images, whichever is larger.
size_t q_image_bytes(int batch) { return round256((size_t)batch * kQImageBytes); }
size_t ws_bytes_for(int batch, int heads, int topk, int ctas) {
  const size_t dense = ws_total((long long)ctas + batch, heads);
  if (topk <= 0) return dense + q_image_bytes(batch);
  const size_t simt = ws_total(slots_for(batch, topk, ctas), heads, list_ints_for(batch, topk, ctas));
  const size_t gathered = dense + sparse_gather_rows_bytes(batch, topk) + round256((size_t)batch * 4) +
                          q_image_bytes(batch);
  return simt > gathered ? simt : gathered;
}

}  // namespace
}  // namespace dcpmla

using namespace dcpmla;

extern "C" {

const char* dcpmla_error_string(int code) {
  switch (code) {
    case DCPMLA_OK: return "ok";
    case DCPMLA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DCPMLA_ERR_UNSUPPORTED: return "unsupported argument combination";
    case DCPMLA_ERR_WORKSPACE: return "workspace missing or too small";
    case DCPMLA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case DCPMLA_ERR_CUDA: return "CUDA runtime error";
    default: return "unknown error code";
  }
}

int dcpmla_device_sm_count(int* sm_count) {
  if (!sm_count) return DCPMLA_ERR_INVALID_ARGUMENT;
  return sm_count_current(sm_count);
}

int mla_decode_workspace_size(int batch, int num_heads, int num_splits, int topk,
                              size_t* bytes) {
  if (!bytes || batch < 0 || num_heads < 1 || num_splits < 0 || topk < 0)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  // rows: query heads, or (query, head) pairs of a multi-query call
  if (num_heads > kMaxHeads * kMaxQueryLen) return DCPMLA_ERR_UNSUPPORTED;
  int ctas = 0;
  int rc = resolve_ctas(num_splits, &ctas);
  if (rc != DCPMLA_OK) return rc;
  *bytes = ws_bytes_for(batch, num_heads, topk, ctas);
  return DCPMLA_OK;
}

}  // extern "C"

namespace {

// Shared body of mla_decode_partial (q_len = 1) and mla_decode_partial_multi:
// num_heads here counts rows (query heads x q_len).  rows_q / rows_o are the
// rows between consecutive requests in q and in the outputs (num_heads for a
// plain call), len_delta is subtracted from every length (a pass over the
// earlier queries of a multi-query call).
int decode_partial(const void* q, const void* kv_cache, int kv_dtype, int64_t num_blocks,
                   int block_size, const int32_t* block_table, int block_table_stride,
                   const int32_t* seq_lens, int batch, int num_heads, int q_len, int shard_id,
                   int num_shards, const int32_t* sparse_idx, int topk, float softmax_scale,
                   float* out_partial, float* out_lse, void* workspace, size_t workspace_bytes,
                   int num_splits, int impl, void* stream, int rows_q, int rows_o,
                   int len_delta, bool identity_table = false) {
  // ---- scalar checks (fail closed, nothing launched on error) ----
  const bool withhold = (impl & DCPMLA_TEST_WITHHOLD_ARRIVAL) != 0;
  impl &= ~DCPMLA_TEST_WITHHOLD_ARRIVAL;
  if (withhold && impl != DCPMLA_IMPL_TC && impl != DCPMLA_IMPL_TC_F16)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (batch < 0 || num_heads < 1 || num_shards < 1 || shard_id < 0 || shard_id >= num_shards ||
      block_size < 1 || block_table_stride < 1 || num_blocks < 1 || num_splits < 0 ||
      topk < 0 || (sparse_idx && topk < 1) || !std::isfinite(softmax_scale))
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (kv_dtype != DCPMLA_KV_BF16 && kv_dtype != DCPMLA_KV_FP8) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (impl != DCPMLA_IMPL_AUTO && impl != DCPMLA_IMPL_SIMT && impl != DCPMLA_IMPL_TC &&
      impl != DCPMLA_IMPL_TC_F16)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (num_heads > kMaxHeads || block_size != kBlock) return DCPMLA_ERR_UNSUPPORTED;
  if (batch == 0) return DCPMLA_OK;
  if (!q || !kv_cache || (!block_table && !identity_table) || !seq_lens || !out_partial ||
      !out_lse)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(kv_cache) || !aligned16(out_partial) ||
      (workspace && !aligned16(workspace)))
    return DCPMLA_ERR_ALIGNMENT;
  const int eff_topk = sparse_idx ? topk : 0;
  int ctas = 0;
  int rc = resolve_ctas(num_splits, &ctas);
  if (rc != DCPMLA_OK) return rc;
  const long long slots = slots_for(batch, eff_topk, ctas);
  const long long list_ints = list_ints_for(batch, eff_topk, ctas);
  if (!workspace || workspace_bytes < ws_bytes_for(batch, num_heads, eff_topk, ctas))
    return DCPMLA_ERR_WORKSPACE;

  PartialParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kv = static_cast<const uint8_t*>(kv_cache);
  p.num_blocks = num_blocks;
  p.block_table = identity_table ? nullptr : block_table;
  p.bt_stride = block_table_stride;
  p.seq_lens = seq_lens;
  p.batch = batch;
  p.heads = num_heads;
  p.q_len = q_len;
  p.shard = shard_id;
  p.nshards = num_shards;
  p.sparse_idx = sparse_idx;
  p.topk = eff_topk;
  p.sparse_parts = sparse_idx ? sparse_parts_for(batch, topk, ctas) : 1;
  p.scale = softmax_scale;
  p.out = out_partial;
  p.out_lse = out_lse;
  p.rows_q = rows_q;
  p.rows_o = rows_o;
  p.len_delta = len_delta;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.flags = reinterpret_cast<int*>(ws);
  p.ws_o = reinterpret_cast<float*>(ws + ws_o_offset());
  p.ws_lse = reinterpret_cast<float*>(ws + ws_lse_offset(slots, num_heads));
  p.ws_list = list_ints ? reinterpret_cast<int*>(ws + ws_list_offset(slots, num_heads)) : nullptr;
  p.num_ctas = ctas;
  p.test_withhold = withhold ? 1 : 0;
  p.q_image = ws + ws_total((long long)ctas + batch, num_heads);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Sparse decode on the tensor cores: a pre-kernel localises each request's
  // selections, which are then decoded as one shard of selected rows through
  // identity tables.  fp8 rows go to the exact e4m3 kernel, which fetches the
  // listed rows from the cache itself, whole requests per CTA; bf16 rows are
  // copied into whole blocks for the fp16-operand kernel.  The CUDA-core
  // kernel and the fp16-operand kernel chosen explicitly (DCPMLA_IMPL_TC_F16)
  // keep their own in-kernel selection.
  const bool gathered_sparse =
      p.sparse_idx && impl != DCPMLA_IMPL_SIMT && impl != DCPMLA_IMPL_TC_F16;
  if (gathered_sparse) {
    const int rb = kv_dtype == DCPMLA_KV_BF16 ? kRowBytesBf16 : kRowBytesFp8;
    const int maxblk = (int)sparse_maxblk(eff_topk);
    uint8_t* gathered = ws + ws_total((long long)ctas + batch, num_heads);
    int* counts = reinterpret_cast<int*>(gathered + sparse_gather_rows_bytes(batch, eff_topk));
    p.q_image = reinterpret_cast<uint8_t*>(counts) + round256((size_t)batch * 4);
    // The e4m3 kernel fetches the selected rows from the cache itself, given
    // their flat row numbers (int32); the other kernels read the rows copied
    // into whole blocks.
    PartialParams dense_view = p;
    dense_view.sparse_idx = nullptr;
    const bool listed = impl != DCPMLA_IMPL_TC_F16 && f8_supports(dense_view, kv_dtype) &&
                        num_blocks <= (int64_t)(INT32_MAX / kBlock);
    if (listed) {
      int* rows = reinterpret_cast<int*>(gathered);
      if (launch_sparse_rows(p, maxblk, rows, counts, p.q_image, st) != cudaSuccess)
        return DCPMLA_ERR_CUDA;
      p.row_ids = rows;
      p.row_stride = maxblk * kBlock;
      p.q_image_ready = 1;
    } else {
      if (launch_sparse_gather(p, rb, maxblk, gathered, counts, st) != cudaSuccess)
        return DCPMLA_ERR_CUDA;
      p.kv = gathered;
      p.num_blocks = (long long)batch * maxblk;
    }
    p.block_table = nullptr;
    p.id_stride = maxblk;
    p.bt_stride = maxblk;
    p.seq_lens = counts;
    p.shard = 0;
    p.nshards = 1;
    p.sparse_idx = nullptr;
    p.topk = 0;
    p.sparse_parts = 1;
    p.ws_o = reinterpret_cast<float*>(ws + ws_o_offset());
    p.ws_lse = reinterpret_cast<float*>(ws + ws_lse_offset((long long)ctas + batch, num_heads));
    p.ws_list = nullptr;
  }
  const bool tc_ok = tc_supports(p, kv_dtype);
  const bool f8_ok = f8_supports(p, kv_dtype);
  if (gathered_sparse && f8_ok) {
    // a request's selections are a few tiles: whole requests per CTA (one Q
    // image and one epilogue each, nothing to combine), at least
    // ceil(batch / 32) CTAs, at most one per request
    const int min_ctas = (batch + kMaxRequestsPerCta - 1) / kMaxRequestsPerCta;
    p.request_aligned = 1;
    p.num_ctas = std::max(min_ctas, std::min(batch, ctas));
  }
  enum { kSimt, kTc16, kTc8 } which;
  if (impl == DCPMLA_IMPL_SIMT) {
    which = kSimt;
  } else if (impl == DCPMLA_IMPL_TC_F16) {
    if (!tc_ok) return DCPMLA_ERR_UNSUPPORTED;
    which = kTc16;
  } else if (f8_ok) {
    which = kTc8;
  } else if (tc_ok) {
    which = kTc16;
  } else if (impl == DCPMLA_IMPL_TC) {
    return DCPMLA_ERR_UNSUPPORTED;
  } else {
    which = kSimt;
  }
  if (q_len > 1 && which == kSimt) return DCPMLA_ERR_UNSUPPORTED;   // causal rows: tensor cores only

  cudaError_t e = which == kTc8    ? launch_partial_f8(p, st)
                  : which == kTc16 ? launch_partial_tc(p, kv_dtype, st)
                                   : launch_partial_simt(p, kv_dtype, st);
  if (e != cudaSuccess) return DCPMLA_ERR_CUDA;
  e = launch_split_combine(p, st);
  return e == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

}  // namespace

extern "C" {

int mla_decode_partial(const void* q, const void* kv_cache, int kv_dtype, int64_t num_blocks,
                       int block_size, const int32_t* block_table, int block_table_stride,
                       const int32_t* seq_lens, int batch, int num_heads, int shard_id,
                       int num_shards, const int32_t* sparse_idx, int topk,
                       float softmax_scale, float* out_partial, float* out_lse,
                       void* workspace, size_t workspace_bytes, int num_splits, int impl,
                       void* stream) {
  return decode_partial(q, kv_cache, kv_dtype, num_blocks, block_size, block_table,
                        block_table_stride, seq_lens, batch, num_heads, 1, shard_id, num_shards,
                        sparse_idx, topk, softmax_scale, out_partial, out_lse, workspace,
                        workspace_bytes, num_splits, impl, stream, num_heads, num_heads, 0);
}

int mla_decode_partial_multi(const void* q, const void* kv_cache, int kv_dtype,
                             int64_t num_blocks, int block_size, const int32_t* block_table,
                             int block_table_stride, const int32_t* seq_lens, int batch,
                             int num_heads, int q_len, int shard_id, int num_shards,
                             float softmax_scale, float* out_partial, float* out_lse,
                             void* workspace, size_t workspace_bytes, int num_splits, int impl,
                             void* stream) {
  if (q_len < 1 || num_heads < 1 || q_len > kMaxQueryLen) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (num_heads > kMaxHeads) return DCPMLA_ERR_UNSUPPORTED;
  const int rows = num_heads * q_len;
  const int base_impl = impl & ~DCPMLA_TEST_WITHHOLD_ARRIVAL;
  // Queries per pass.  A pass is one decode over the cache whose rows fit
  // one 64-row tile: the fp8 cache and the CUDA-core kernel take one query
  // per pass (plain decode rows: the e4m3-direct kernel's exact scores, and
  // no causal rows for the CUDA-core kernel); the fp16-operand kernel takes
  // as many whole queries as fit its tile.
  int qpp = kMaxHeads / num_heads;
  if (base_impl == DCPMLA_IMPL_SIMT ||
      (kv_dtype == DCPMLA_KV_FP8 && base_impl != DCPMLA_IMPL_TC_F16))
    qpp = 1;
  if (qpp >= q_len)
    return decode_partial(q, kv_cache, kv_dtype, num_blocks, block_size, block_table,
                          block_table_stride, seq_lens, batch, rows, q_len, shard_id,
                          num_shards, nullptr, 0, softmax_scale, out_partial, out_lse, workspace,
                          workspace_bytes, num_splits, impl, stream, rows, rows, 0);
  // Several passes, in order on the stream (they share the workspace).
  // Pass k covers queries [k0, k0 + n): rows k0 * num_heads onward of every
  // request, over the cache less its last q_len - k0 - n tokens, which puts
  // its last query at the end of the shortened cache.
  for (int k0 = 0; k0 < q_len; k0 += qpp) {
    const int n = q_len - k0 < qpp ? q_len - k0 : qpp;
    const size_t r0 = (size_t)k0 * num_heads;
    const int rc = decode_partial(
        static_cast<const uint8_t*>(q) + r0 * kHeadDim * sizeof(__nv_bfloat16), kv_cache,
        kv_dtype, num_blocks, block_size, block_table, block_table_stride, seq_lens, batch,
        n * num_heads, n, shard_id, num_shards, nullptr, 0, softmax_scale,
        out_partial + r0 * kVDim, out_lse + r0, workspace, workspace_bytes, num_splits, impl,
        stream, rows, rows, q_len - k0 - n);
    if (rc != DCPMLA_OK) return rc;
  }
  return DCPMLA_OK;
}

int pcp_prefill_attention(const void* q, const int32_t* positions, int num_queries,
                          int num_heads, const void* gathered, int kv_dtype,
                          int64_t num_gathered_blocks, float softmax_scale, float* out,
                          float* out_lse, void* workspace, size_t workspace_bytes,
                          int num_splits, int impl, void* stream) {
  // Query token b at prompt position positions[b] attends causally to the
  // gathered rows 0..positions[b]: a decode over the gathered prompt (its
  // blocks in order, one shard) of length positions[b] + 1.
  if (num_queries < 0 || num_gathered_blocks < 1 || num_gathered_blocks > INT32_MAX)
    return DCPMLA_ERR_INVALID_ARGUMENT;
  if (!positions && num_queries > 0) return DCPMLA_ERR_INVALID_ARGUMENT;
  return decode_partial(q, gathered, kv_dtype, num_gathered_blocks, kBlock, nullptr,
                        (int)num_gathered_blocks, positions, num_queries, num_heads, 1, 0, 1,
                        nullptr, 0, softmax_scale, out, out_lse, workspace, workspace_bytes,
                        num_splits, impl, stream, num_heads, num_heads, -1, true);
}

int dcp_merge(const float* partials, const float* lses, int num_shards, int batch,
              int num_heads, float* out, float* out_lse, void* stream) {
  if (num_shards < 1 || batch < 0 || num_heads < 1) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (batch == 0) return DCPMLA_OK;
  if (!partials || !lses || !out) return DCPMLA_ERR_INVALID_ARGUMENT;
  if (!aligned16(partials) || !aligned16(out)) return DCPMLA_ERR_ALIGNMENT;
  cudaError_t e = launch_dcp_merge(partials, lses, num_shards, batch, num_heads, out, out_lse,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DCPMLA_OK : DCPMLA_ERR_CUDA;
}

}  // extern "C"

/*
 * dcpmla.h - C ABI of libdcpmla.so: decode-context-parallel (DCP) absorbed-MLA
 * decode on NVIDIA B200 (sm_100a).
 *
 * What the calls compute (cited by page title and section):
 *
 *  - "GLM-5.2 vLLM Decode Context Parallelism", section "See why vLLM 0.26.0
 *    fails": under DCP each rank computes a partial attention output over its
 *    own part of the cache, and the partial outputs are combined with the
 *    softmax normalisation, which needs the decode log-sum-exp (LSE).
 *  - same page, section "Separate the backend merge from stable": the LSE is
 *    returned per (token, head); global sparse top-K indices are localised to
 *    the rank that owns each position; a row with no selected local token
 *    returns the neutral pair (O = 0, LSE = -inf) and drops out of the merge.
 *  - "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s",
 *    section "The core design": cache tokens are distributed round-robin, so
 *    each of N ranks holds 1/N of them.  Here token t belongs to shard t mod N
 *    and sits at local index t div N of that shard.
 *  - "The Final Verification: Confirming a 200k Context Deployment on GLM-5",
 *    section "The Decision-Making Process Visible in the Reasoning": one MLA
 *    cache row per token and layer holds kv_lora_rank + qk_rope_head_dim =
 *    512 + 64 values (1,152 bytes in bf16).
 *
 * Readings used where the pages are silent:
 *  - Absorbed MLA: the query row (576 values) is already in the latent space,
 *    every query head attends to the one shared latent row, scores are
 *    softmax_scale * <q, k> over all 576 values, and the value is the first
 *    512 values of the same row.  The output is the 512-wide latent result.
 *  - LSE is the natural logarithm of sum_t exp(score_t), scale included.
 *  - fp8 rows ("fp8_ds_mla"-like, 656 bytes): 512 OCP E4M3 codes, then 4
 *    little-endian fp32 scales (latent values [128g, 128g+128) use scale g),
 *    then 64 bf16 rope values.  bf16 rows: 576 bf16 values (1,152 bytes).
 *  - Each shard has its own block table over its local indices; block size
 *    is 64 rows.
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller (except the
 *    host pointer tables of dcp_merge_heads).  The compute calls allocate no
 *    memory, never synchronise, and only enqueue work on `stream` (a
 *    cudaStream_t; NULL means the legacy default stream); they return once the
 *    work is enqueued.  The dcp_exchange_* calls are the exception: they
 *    exist to allocate, map and free exchange buffers, and may synchronise.
 *  - Arguments are checked on the host, before anything is launched; a
 *    failed check returns a negative DCPMLA_ERR_* code and launches nothing
 *    (fail closed: nothing is clamped or guessed).  Device-side contents
 *    (block-table entries, sparse indices, lengths) are range-checked in the
 *    kernels: an out-of-range entry is skipped, never dereferenced, and sets
 *    a bit in the workspace's device flag word (see below).
 *  - Asynchronous CUDA faults surface at the caller's next synchronisation;
 *    launch failures are returned as DCPMLA_ERR_CUDA.
 */
#ifndef DCPMLA_H
#define DCPMLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Cache row formats. */
#define DCPMLA_KV_BF16 0     /* 1,152-byte rows: 576 bf16 */
#define DCPMLA_KV_FP8 1      /* 656-byte rows: 512 e4m3 + 4 fp32 scales + 64 bf16 rope */

/* Kernel selection for mla_decode_partial. */
#define DCPMLA_IMPL_AUTO 0   /* fastest available for the arguments */
#define DCPMLA_IMPL_SIMT 1   /* plain CUDA-core kernel (any H <= 64) */
#define DCPMLA_IMPL_TC 2     /* tcgen05 / TMEM tensor-core kernel: fp8 rows (dense
                                or sparse, one query token per pass) go to the
                                kernel that multiplies the e4m3 codes directly;
                                bf16 rows to the fp16-operand kernel */
#define DCPMLA_IMPL_TC_F16 3 /* the fp16-operand tensor-core kernel for every
                                argument combination it supports (bf16 rows, fp8
                                rows converted to fp16; kept for comparison) */
/* Test only, OR-ed into DCPMLA_IMPL_TC or DCPMLA_IMPL_TC_F16: the kernel's
 * first tile is never delivered, so every pipeline wait of every CTA runs
 * out (about 2 s);
 * the kernel then drains, frees its tensor memory, sets
 * DCPMLA_FLAG_TIMEOUT and returns with invalid outputs.  Exercises the
 * timeout path; the context stays usable. */
#define DCPMLA_TEST_WITHHOLD_ARRIVAL 0x100

/* Return codes. */
#define DCPMLA_OK 0
#define DCPMLA_ERR_INVALID_ARGUMENT (-1)   /* null pointer, bad size, shard id out of range ... */
#define DCPMLA_ERR_UNSUPPORTED (-2)        /* valid but not implemented (e.g. H > 64, block != 64) */
#define DCPMLA_ERR_WORKSPACE (-3)          /* workspace missing or smaller than required */
#define DCPMLA_ERR_ALIGNMENT (-4)          /* a pointer is not 16-byte aligned */
#define DCPMLA_ERR_CUDA (-5)               /* a CUDA runtime call or launch failed */

/* Bits the kernels OR into the workspace flag word (int32 at byte 0). */
#define DCPMLA_FLAG_BAD_BLOCK 1      /* a block-table entry was outside [0, num_blocks) */
#define DCPMLA_FLAG_BAD_LENGTH 2     /* a length was negative or needs more blocks than the table row has */
#define DCPMLA_FLAG_TIMEOUT 4        /* a tensor-core kernel pipeline wait gave up (about 2 s); outputs invalid */
#define DCPMLA_FLAG_RANGE 8          /* a q or cache value beyond +-65504 was clamped by the fp16 tensor-core path */

#define DCPMLA_HEAD_DIM 576          /* 512 latent + 64 rope */
#define DCPMLA_V_DIM 512
#define DCPMLA_BLOCK_SIZE 64
#define DCPMLA_MAX_HEADS 64

/*
 * Bytes of workspace that mla_decode_partial needs for these sizes.
 *
 *   batch, num_heads: as passed to mla_decode_partial (for
 *               mla_decode_partial_multi, num_heads * q_len; up to
 *               DCPMLA_MAX_HEADS * 64 rows, else DCPMLA_ERR_UNSUPPORTED).
 *   num_splits: as passed to mla_decode_partial (0 = automatic, which uses
 *               the SM count of the current device).
 *   topk: length of each sparse index list, 0 for dense decode.
 *   bytes: receives the size.
 *
 * Layout: a 256-byte header (int32 flag word at byte 0, the rest reserved),
 * then per-split partial results, the sparse selections of a call with
 * topk > 0 (flat cache rows, or the selected rows copied into whole blocks,
 * sized for bf16 rows) and the per-request Q operand images of the fp8
 * kernel (73,984 bytes each).  The flag word is OR-ed by the kernels and
 * never cleared by the library: zero it before the first call if you read it.
 * Returns DCPMLA_OK or a negative code.
 */
int mla_decode_workspace_size(int batch, int num_heads, int num_splits, int topk,
                              size_t* bytes);

/*
 * Partial attention of one DCP shard, with its LSE, for every request.
 *
 *   q            [batch][num_heads][576] bf16, 16-byte aligned.
 *   kv_cache     [num_blocks][64][row bytes] raw rows in format `kv_dtype`,
 *                16-byte aligned.
 *   block_table  [batch][block_table_stride] int32: this shard's table; entry
 *                k of request b is the physical block holding local rows
 *                [64k, 64k+64).
 *   seq_lens     [batch] int32 GLOBAL cached lengths L_b.  The shard's local
 *                length is the number of t in [0, L_b) with t mod N = shard_id.
 *   shard_id, num_shards: 0 <= shard_id < num_shards.
 *   sparse_idx   NULL for dense decode, else [batch][topk] int32 global token
 *                positions; entries outside [0, L_b) are skipped (-1 pads);
 *                entries owned by other shards are skipped.
 *   softmax_scale  multiplies <q, k> before the softmax.
 *   out_partial  [batch][num_heads][512] fp32: sum_t softmax_t * v_t over
 *                this shard's tokens (0 for a request with none).
 *   out_lse      [batch][num_heads] fp32: natural-log LSE (-inf if none).
 *   workspace, workspace_bytes: at least mla_decode_workspace_size(...).
 *   num_splits   CTAs to spread the work over (0 = automatic: the SM count).
 *                Dense decode splits the shard's tiles evenly over them, as
 *                does sparse decode of bf16 rows; sparse decode of fp8 rows
 *                on the tensor-core path gives each CTA a contiguous range of
 *                whole requests (at most 32 each, so the grid is at least
 *                ceil(batch / 32) CTAs).
 *   impl         DCPMLA_IMPL_* (AUTO picks the tensor-core kernel when it
 *                supports the arguments).
 *   stream       cudaStream_t to enqueue on.
 *
 * Returns DCPMLA_OK or a negative DCPMLA_ERR_* code.
 */
int mla_decode_partial(const void* q, const void* kv_cache, int kv_dtype, int64_t num_blocks,
                       int block_size, const int32_t* block_table, int block_table_stride,
                       const int32_t* seq_lens, int batch, int num_heads, int shard_id,
                       int num_shards, const int32_t* sparse_idx, int topk,
                       float softmax_scale, float* out_partial, float* out_lse,
                       void* workspace, size_t workspace_bytes, int num_splits, int impl,
                       void* stream);

/*
 * Multi-query decode (speculative / multi-token-prediction verification):
 * q_len query tokens per request, all N shards as in mla_decode_partial.
 *
 * "GLM-5.2 vLLM Decode Context Parallelism", section "Add MTP only after
 * plain decode passes": multi-token prediction adds draft-token query shapes
 * to the same decode attention.  Reading (the pages give no formula): the
 * cache already holds the q_len new tokens, L_b in total; query i sits at
 * position L_b - q_len + i and attends to every cached t <= that position.
 *
 *   q            [batch][q_len][num_heads][576] bf16 (16-byte aligned).
 *   num_heads    query heads per token, 1..64 (else DCPMLA_ERR_UNSUPPORTED);
 *                q_len 1..64 (else DCPMLA_ERR_INVALID_ARGUMENT).  The rows
 *                (query, head) run in passes over the cache, each pass one
 *                tile of at most 64 rows and whole queries: with an fp8 cache
 *                (exact e4m3 kernel) and with DCPMLA_IMPL_SIMT one query per
 *                pass, otherwise as many queries as fit 64 rows.  A pass over
 *                queries [k, k + n) attends over the cache less its last
 *                q_len - k - n tokens; each pass reads that part of the
 *                cache again, so q_len passes read about q_len times the
 *                bytes of one decode.
 *   out_partial  [batch][q_len][num_heads][512] fp32; out_lse
 *                [batch][q_len][num_heads] fp32; queries that see no token of
 *                this shard give (0, -inf).
 *   workspace    mla_decode_workspace_size(batch, num_heads * q_len, ...).
 *   impl         any DCPMLA_IMPL_* (the CUDA-core kernel runs one query per
 *                pass).
 * Other arguments as in mla_decode_partial (no sparse variant).  The merge is
 * dcp_merge with num_heads * q_len rows.
 */
int mla_decode_partial_multi(const void* q, const void* kv_cache, int kv_dtype,
                             int64_t num_blocks, int block_size, const int32_t* block_table,
                             int block_table_stride, const int32_t* seq_lens, int batch,
                             int num_heads, int q_len, int shard_id, int num_shards,
                             float softmax_scale, float* out_partial, float* out_lse,
                             void* workspace, size_t workspace_bytes, int num_splits, int impl,
                             void* stream);

/*
 * Bytes of the scratch array built into the library for
 * mla_decode_partial_noalloc: 32 MiB per device, enough for batch 64 x 64
 * heads x 148 splits (about 32.6 MB, 4.7 MB of it the Q operand images of
 * the fp8 kernel).  Of the five workloads the tiny, dense, agentic and
 * million-token ones fit; the sparse one (batch 128, whose selections take
 * about 330 MB of workspace) does not and is refused with
 * DCPMLA_ERR_WORKSPACE.  The array is part of the library's device module:
 * with CUDA's lazy module loading (the default) it takes device memory only
 * on devices where the module is loaded, i.e. that call into the library;
 * with eager loading (CUDA_MODULE_LOADING=EAGER) it is reserved on every
 * device the process initialises.
 */
#define DCPMLA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * mla_decode_partial without a caller-supplied workspace.  The method's
 * description has no counterpart to this call: it is a library convenience
 * for callers that cannot hand the library device memory (a C host program
 * with no device allocator of its own, or a serving loop that must not call
 * cudaMalloc / cudaFree between steps because they synchronise the device).
 *
 * Arguments, layouts and results are those of mla_decode_partial, minus
 * workspace / workspace_bytes, plus:
 *   out_flags  NULL, or a DEVICE int32 that receives (in stream order) this
 *              call's DCPMLA_FLAG_* bits.
 *
 * The workspace is a fixed DCPMLA_NOALLOC_SCRATCH_BYTES array in device
 * memory of the library (one per device); nothing is allocated, by this call
 * or on its behalf.  Its flag word is cleared at setup and again after every
 * call, so each call's flags stand alone.
 *
 * Limits:
 *  - A request whose mla_decode_workspace_size(batch, num_heads, num_splits,
 *    sparse_idx ? topk : 0) exceeds DCPMLA_NOALLOC_SCRATCH_BYTES returns
 *    DCPMLA_ERR_WORKSPACE before any work is enqueued.
 *  - Every call on a device uses the same scratch: calls whose work overlaps
 *    on the device (different streams, different host threads) race and
 *    corrupt each other's results.  Serialise them, e.g. on one stream.
 *  - The first call on each device (with that device current) performs the
 *    setup: it looks the scratch array up with cudaGetSymbolAddress, which
 *    may load the library's module, and enqueues the first clear of the flag
 *    word.  Make that first call before any stream capture begins.
 *  - The looked-up address is kept for the life of the process: the setup
 *    must not outlive the device's context (no cudaDeviceReset, no teardown
 *    of the primary context, between calls).
 *  - Query heads only (num_heads <= 64, else DCPMLA_ERR_UNSUPPORTED); there
 *    is no multi-query or sparse-beyond-the-scratch variant.
 *
 * Returns DCPMLA_OK or a negative DCPMLA_ERR_* code (DCPMLA_ERR_CUDA if the
 * setup fails).
 */
int mla_decode_partial_noalloc(const void* q, const void* kv_cache, int kv_dtype,
                               int64_t num_blocks, int block_size, const int32_t* block_table,
                               int block_table_stride, const int32_t* seq_lens, int batch,
                               int num_heads, int shard_id, int num_shards,
                               const int32_t* sparse_idx, int topk, float softmax_scale,
                               float* out_partial, float* out_lse, int32_t* out_flags,
                               int num_splits, int impl, void* stream);

/*
 * LSE-weighted merge of N shard partials into the full-context result.
 *
 *   partials  [num_shards][batch][num_heads][512] fp32 (16-byte aligned).
 *   lses      [num_shards][batch][num_heads] fp32.
 *   out       [batch][num_heads][512] fp32: with M = max_i lse_i and
 *             w_i = exp(lse_i - M), out = sum_i w_i partial_i / sum_i w_i.
 *             Shards with lse = -inf weigh exactly 0; if all are -inf the
 *             result is 0.
 *   out_lse   [batch][num_heads] fp32 merged LSE M + ln sum_i w_i (-inf if all
 *             are -inf), or NULL if not wanted.
 *
 * Returns DCPMLA_OK or a negative code.
 */
int dcp_merge(const float* partials, const float* lses, int num_shards, int batch,
              int num_heads, float* out, float* out_lse, void* stream);

/*
 * Real multi-GPU DCP: one rank per GPU, rank r holding shard r of the cache.
 *
 * "GLM-5.2 vLLM Decode Context Parallelism", section "Keep the current-main
 * correctness blocker visible": pure DCP gathers the query heads before
 * attention and combines the partial output/LSE across ranks after it; section
 * "Separate the backend merge from stable": the cross-rank combine takes the
 * ag_rs path (all-gather of LSEs, reduce-scatter of the rescaled partials),
 * after which each rank holds the merged result of its own query heads
 * (section "Calculate the GLM-5.2 head envelope": gathered heads = local
 * heads x DCP size).
 *
 * dcp_merge_heads is that exchange as one kernel: this rank reads its slice
 * of heads from every shard's partial and LSE buffers (its own, and the other
 * ranks' mapped into this device with dcp_exchange_open) and merges them with
 * the dcp_merge formula.  The caller orders it after every shard's partial is
 * complete (e.g. a stream-ordered NCCL collective between the partial and
 * this call on every rank) and does not overwrite a buffer before every rank
 * has read it.
 *
 *   partials     HOST array of num_shards DEVICE pointers; partials[s] is
 *                shard s's [batch][num_heads][512] fp32 partial (16-byte
 *                aligned), readable from the current device.
 *   lses         HOST array of num_shards DEVICE pointers to [batch][num_heads]
 *                fp32 LSEs.  Both tables are copied into the launch: the
 *                host arrays may be reused as soon as the call returns.
 *   num_shards   1 .. DCPMLA_MAX_MERGE_SHARDS.
 *   head_begin, head_count: the merged slice, 0 <= head_begin,
 *                1 <= head_count, head_begin + head_count <= num_heads.
 *   out          [batch][head_count][512] fp32 (16-byte aligned): row
 *                (b, i) is the merge of head head_begin + i of request b.
 *   out_lse      [batch][head_count] fp32 merged LSE, or NULL.
 *
 * With head_begin = 0, head_count = num_heads and the shards' buffers laid
 * out back to back this is exactly dcp_merge (same arithmetic, same order).
 * Returns DCPMLA_OK or a negative code.
 */
#define DCPMLA_MAX_MERGE_SHARDS 64
int dcp_merge_heads(const float* const* partials, const float* const* lses, int num_shards,
                    int batch, int num_heads, int head_begin, int head_count, float* out,
                    float* out_lse, void* stream);

/*
 * Exchange buffers: device memory another process (rank) can map.  The
 * method's description has no counterpart to these calls; they are the
 * plumbing dcp_merge_heads reads peers' partials through (CUDA IPC over
 * NVLink / NVSwitch).  Unlike the compute calls they allocate, free and
 * may synchronise the device.
 *
 *   dcp_exchange_alloc  allocates `bytes` on the current device; *dev_ptr
 *                       receives the pointer (256-byte aligned) and
 *                       ipc_handle (DCPMLA_IPC_HANDLE_BYTES bytes, caller
 *                       owned) a handle other processes on this node pass to
 *                       dcp_exchange_open.  Release with dcp_exchange_free
 *                       after every mapping of it is closed.
 *   dcp_exchange_open   maps another process's buffer into the current
 *                       device (peer access enabled as needed); *dev_ptr
 *                       receives its base.  A process cannot open its own
 *                       handle: use its own pointer.  Close with
 *                       dcp_exchange_close.
 * Each returns DCPMLA_OK, DCPMLA_ERR_INVALID_ARGUMENT for a null pointer or a
 * zero size, or DCPMLA_ERR_CUDA if the runtime refuses (out of memory, an
 * invalid or own handle); *dev_ptr is NULL on failure.
 */
#define DCPMLA_IPC_HANDLE_BYTES 64
int dcp_exchange_alloc(size_t bytes, void** dev_ptr, void* ipc_handle);
int dcp_exchange_open(const void* ipc_handle, void** dev_ptr);
int dcp_exchange_close(void* dev_ptr);
int dcp_exchange_free(void* dev_ptr);

/*
 * DCP cache write of new decode tokens: this shard writes the tokens it owns.
 *
 * "GLM-5.2 vLLM Decode Context Parallelism", section "Keep the current-main
 * correctness blocker visible": under DCP a token whose cache slot another
 * rank owns gets no cache write here (its query is still processed); the
 * write is guarded, not the query.  Ownership is round-robin ("How vLLM Serves
 * GLM-5.3 with Million-Token Contexts on 16 H200s", "The core design"): token
 * t belongs to shard t mod N and lands at local row j = t div N, i.e. row
 * j % 64 of physical block block_table[b][j / 64] -- the rows
 * mla_decode_partial reads.
 *
 *   latent       [num_tokens][512] bf16 (the absorbed latent, already normed),
 *                16-byte aligned.
 *   rope         [num_tokens][64] bf16 (rope part of the key), 16-byte aligned.
 *   positions    [num_tokens] int32 global position t of each token (< 0:
 *                no token, skipped).
 *   req_idx      [num_tokens] int32 request b of each token.
 *   block_table  [batch][block_table_stride] int32: this shard's table.
 *   shard_id, num_shards: 0 <= shard_id < num_shards.
 *   kv_cache     [num_blocks][64][row bytes], 16-byte aligned; rows of owned
 *                tokens are overwritten, nothing else is touched.
 *   kv_dtype     DCPMLA_KV_BF16: the 576 values are copied.  DCPMLA_KV_FP8:
 *                per 128-value group g, scale_g = amax_g / 448 (1 if amax_g
 *                is 0, fp32 division), codes = E4M3 of fp32(x / scale_g),
 *                round to nearest even, saturated at +-448; the row holds the
 *                512 codes, the 4 scales (fp32) and the 64 rope values (bf16).
 *   flags        NULL, or a DEVICE int32 the kernel ORs DCPMLA_FLAG_BAD_BLOCK
 *                (table entry outside [0, num_blocks)) and
 *                DCPMLA_FLAG_BAD_LENGTH (request index outside [0, batch), or
 *                a local block index beyond the table row) into; such tokens
 *                are not written.
 *
 * Returns DCPMLA_OK or a negative DCPMLA_ERR_* code (checked on the host
 * before any launch).
 */
int mla_kv_append(const void* latent, const void* rope, int num_tokens, const int32_t* positions,
                  const int32_t* req_idx, const int32_t* block_table, int block_table_stride,
                  int batch, int shard_id, int num_shards, void* kv_cache, int kv_dtype,
                  int64_t num_blocks, int block_size, int32_t* flags, void* stream);

/*
 * Prefill context parallelism (PCP) over the DCP-sharded cache.
 *
 * "How vLLM Serves GLM-5.3 with Million-Token Contexts on 16 H200s",
 * section "The core design": PCP splits a prompt's query tokens over P
 * ranks, each computing all heads of its tokens; the prompt is cut into 2P
 * chunks and rank r takes a front chunk and the matching back chunk (16
 * chunks for 8 ranks) so that causal work evens out; the cache stays
 * distributed round-robin over the DCP shards, so prefill gathers the
 * layer's distributed rows, attends, and drops the gathered copy.
 * Readings (the page gives no chunk-size rule or attention form): chunks are
 * contiguous in prompt order, the first T mod 2P one token longer; rank r
 * owns chunks r and 2P - 1 - r, its queries in that order; attention is the
 * absorbed form of the decode path (query token i attends to every prompt
 * token t <= i, scores over 576 values, values the first 512, natural-log
 * LSE); the prompt's rows are in the cache before its attention.
 */

/*
 * The query tokens of PCP rank `rank` of `pcp_size` for a `num_tokens`-token
 * prompt: chunk rank, then chunk 2 * pcp_size - 1 - rank.  Host only.
 *   tokens   NULL (only *count is set) or room for `capacity` int32.
 *   count    receives the number of tokens.
 * Returns DCPMLA_OK, or DCPMLA_ERR_INVALID_ARGUMENT (bad sizes, rank out of
 * range, capacity too small).
 */
int pcp_rank_tokens(int num_tokens, int pcp_size, int rank, int32_t* tokens, int capacity,
                    int* count);

/* Bytes of a gathered prompt of `num_tokens` rows: whole 64-row blocks. */
size_t pcp_gathered_bytes(int num_tokens, int kv_dtype);

/*
 * Gather one request's prompt rows from the DCP-sharded cache into token
 * order: row t of `gathered` is token t, read from shard t mod num_shards at
 * local row t div num_shards through that shard's table row.
 *   kv_cache      [num_blocks][64][row bytes], 16-byte aligned.
 *   block_tables  DEVICE [num_shards][block_table_stride] int32: each shard's
 *                 table row for the request.
 *   gathered      DEVICE, 16-byte aligned, at least
 *                 pcp_gathered_bytes(num_tokens, kv_dtype) bytes ([blocks][64]
 *                 [row bytes]; rows past num_tokens are not written).
 *   flags         NULL or a DEVICE int32: DCPMLA_FLAG_BAD_BLOCK for a table
 *                 entry outside the pool, DCPMLA_FLAG_BAD_LENGTH for a local
 *                 row beyond the table row; such rows are written as zeros.
 * Returns DCPMLA_OK or a negative code (host checks before any launch).
 */
int pcp_gather_rows(const void* kv_cache, int kv_dtype, int64_t num_blocks, int block_size,
                    const int32_t* block_tables, int block_table_stride, int num_shards,
                    int num_tokens, void* gathered, size_t gathered_bytes, int32_t* flags,
                    void* stream);

/*
 * Causal prefill attention of one rank's query tokens over a gathered
 * prompt: query b (all num_heads heads) at prompt position positions[b]
 * attends to gathered rows 0..positions[b].
 *   q             [num_queries][num_heads][576] bf16, 16-byte aligned.
 *   positions     DEVICE [num_queries] int32 prompt positions (< the prompt
 *                 length; a negative one is flagged, DCPMLA_FLAG_BAD_LENGTH).
 *   gathered      the pcp_gather_rows output, num_gathered_blocks blocks.
 *   out, out_lse  [num_queries][num_heads][512] and [num_queries][num_heads]
 *                 fp32.
 *   workspace     mla_decode_workspace_size(num_queries, num_heads,
 *                 num_splits, 0) bytes.
 *   impl          as mla_decode_partial: fp8 rows run on the e4m3-direct
 *                 kernel (exact scores), bf16 rows on the fp16-operand kernel.
 * Each query reads its prefix of the gathered rows: the prompt (at most about
 * 190K fp8 rows fit the 126 MB L2) is read once from HBM and its blocks are
 * shared by the queries through L2.  Returns as mla_decode_partial.
 */
int pcp_prefill_attention(const void* q, const int32_t* positions, int num_queries,
                          int num_heads, const void* gathered, int kv_dtype,
                          int64_t num_gathered_blocks, float softmax_scale, float* out,
                          float* out_lse, void* workspace, size_t workspace_bytes,
                          int num_splits, int impl, void* stream);

/* Static description of a return code (never NULL). */
const char* dcpmla_error_string(int code);

/* Number of SMs of the current device (what num_splits = 0 uses). */
int dcpmla_device_sm_count(int* sm_count);

#ifdef __cplusplus
}
#endif

#endif /* DCPMLA_H */

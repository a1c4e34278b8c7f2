/*
 * pkv.h — C ABI of the B200 paged KV-cache decode library (libpkv.so).
 *
 * The scheme: the KV cache of every sequence is cut into fixed-size blocks of
 * `block_size` tokens (16 or 32) that sit anywhere in one shared physical pool;
 * each sequence reaches its blocks through a block table that keeps their order
 * (vLLM 初探 §1.4 PagedAttention 原理简介, block-table figure; Outcome School vLLM
 * explainer, "vLLM的核心创新：PagedAttention").  Decode attention follows the
 * paged_attention pseudo-code of the intelliparadigm article
 * "PagedAttention：操作系统分页思想的跨界创新" §2.1: logical block = position //
 * block_size, physical block = block_tables[seq][logical block], then
 * softmax(scale * q·Kᵀ)·V over the sequence's tokens.
 *
 * Conventions for every call
 *   - "device" pointers are CUDA device memory owned by the caller (the library
 *     never allocates, frees or keeps them); "host" pointers are ordinary memory.
 *   - Tensors are dense and row-major with the shapes given; bf16 is IEEE bfloat16.
 *     Device tensors must start on a 16-byte boundary (PKV_ERR_INVALID otherwise).
 *   - Kernel calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  A return of PKV_OK means the work was enqueued.
 *   - Kernels launch on the calling thread's current CUDA device; every device
 *     pointer of a call, and `stream`, must belong to that device.
 *   - Argument errors are reported before anything is enqueued and leave all
 *     memory untouched.  Data-dependent errors found on the device (an index out
 *     of range) never trap: the offending row/block is skipped and a bit is OR-ed
 *     into the optional device word `status` (int32, caller-zeroed; may be NULL).
 *   - pkv_last_error_string() returns the text of the last failure on the calling
 *     host thread.
 *
 * Pool layout (one layer): key_cache, value_cache = [num_blocks, num_kv_heads,
 * block_size, head_dim] bf16.  A (block, kv head) tile of block_size x head_dim is
 * contiguous (4 KiB for 16 x 128), the unit the kernels stage into shared memory.
 * Slot of a token = physical_block * block_size + row in the block.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---- */
#define PKV_OK 0
#define PKV_ERR_INVALID (-1)     /* bad argument, shape, pointer alignment or id */
#define PKV_ERR_OOM (-2)         /* block pool exhausted; nothing was changed */
#define PKV_ERR_CUDA (-3)        /* a CUDA runtime call or launch failed */
#define PKV_ERR_UNSUPPORTED (-4) /* head_dim not in {64,128}, block_size not in {16,32},
                                    num_heads % num_kv_heads != 0, num_kv_heads > 65535
                                    (decode), ... */

/* ---- bits of the device status word ---- */
#define PKV_DEV_BAD_SLOT 0x1     /* reshape_and_cache: slot >= num_blocks*block_size */
#define PKV_DEV_BAD_BLOCK 0x2    /* a block-table entry outside [0, num_blocks) */
#define PKV_DEV_BAD_CONTEXT 0x4  /* context_len < 0, > max_context_len or > max_blocks*block_size */
#define PKV_DEV_BAD_PAIR 0x8     /* copy_blocks: src or dst outside [0, num_blocks) */
#define PKV_DEV_TIMEOUT 0x10     /* a bounded on-chip wait gave up (the kernel returned early) */

/* ---- output dtypes and decode paths ---- */
#define PKV_DTYPE_BF16 0
#define PKV_DTYPE_F32 1
#define PKV_PATH_AUTO 0          /* tensor-core path for grouped heads where supported, else CUDA cores */
#define PKV_PATH_SIMT 1          /* CUDA-core streaming kernel, any head grouping */
#define PKV_PATH_TENSOR 2        /* tcgen05 query-group kernel; PKV_ERR_UNSUPPORTED where it does not apply */

typedef void* pkv_stream_t;      /* a cudaStream_t */
typedef struct pkv_bm pkv_bm;    /* opaque host block manager */

/* Text of the last error on this host thread ("" if none). Never NULL. */
PKV_API const char* pkv_last_error_string(void);

/* Library version, major*10000 + minor*100 + patch. */
PKV_API int pkv_version(void);

/*
 * reshape_and_cache — write each new token's K and V into the pool.
 * Outcome School explainer, "LLM serving的基本流程与KV缓存": every decoded token adds
 * one K/V pair that stays resident until its request ends; the intelliparadigm
 * article §2.2: growth only takes a new page and a table update, nothing moves.
 *
 *   key, value       device [num_tokens, num_kv_heads, head_dim] bf16 (read)
 *   key_cache,
 *   value_cache      device [num_blocks, num_kv_heads, block_size, head_dim] bf16 (written)
 *   slot_mapping     device [num_tokens] int64: destination slot of token t;
 *                    slot < 0 skips the token; slot >= num_blocks*block_size is
 *                    skipped and sets PKV_DEV_BAD_SLOT.
 *   Two tokens with the same slot in one call: which one lands is unspecified.
 *   num_tokens == 0 is a no-op.  Bit-exact copy.
 */
PKV_API int pkv_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                          const int64_t* slot_mapping, int num_tokens, int num_blocks,
                          int num_kv_heads, int head_dim, int block_size, int32_t* status,
                          pkv_stream_t stream);

/*
 * copy_blocks — copy-on-write copies of shared blocks that diverge.
 * Outcome School explainer, "内存共享": beams share blocks until they diverge; the
 * copy itself is this library's reading (see pkv_bm_append_slots).
 *
 *   key_caches,
 *   value_caches     HOST arrays of num_layers DEVICE pointers, each a pool of
 *                    [num_blocks, block_elems] bf16 (block_elems = Hkv*bs*D; the copy is
 *                    bytewise, so an 8-bit pool passes half its bytes per block)
 *   block_mapping    device [num_pairs, 2] int64: (src, dst) physical block ids;
 *                    out-of-range pairs are skipped and set PKV_DEV_BAD_PAIR.
 *   Every dst must be distinct and no dst may also be a src in the same call.
 *   num_pairs == 0 or num_layers == 0 is a no-op.  Bit-exact copy.
 */
PKV_API int pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                    const int64_t* block_mapping, int num_pairs, int num_blocks,
                    int64_t block_elems, int32_t* status, pkv_stream_t stream);

/*
 * Bytes of device workspace pkv_paged_attention_decode needs for these sizes
 * (the plan of work items and the split-context partials).  Returns 0 on bad
 * arguments.  partition_tokens: 0 = automatic, else the split size (below).
 */
PKV_API size_t pkv_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                          int head_dim, int block_size, int max_context_len,
                                          int partition_tokens);

/* Split size the automatic choice picks for these sizes (64..512 tokens). */
PKV_API int pkv_paged_attention_partition_tokens(int num_seqs, int num_kv_heads, int block_size,
                                         int max_context_len);

/*
 * paged_attention_decode — single-token decode attention through block tables.
 * intelliparadigm article §2.1 (paged_attention pseudo-code; mapping table; kernel
 * that splices non-contiguous pages through shared memory with prefetch).
 *
 * For every sequence s and query head h, with g = num_heads / num_kv_heads,
 * kv = h / g and L = context_lens[s] (the current token included):
 *   out[s,h,:] = sum_t softmax_t(scale * q[s,h,:]·K_t) V_t,   t = 0..L-1,
 *   K_t = key_cache[block_tables[s][t / bs], kv, t % bs, :]  (V likewise).
 * L == 0 gives a zero row.  Scores, softmax and sums are fp32; the bf16 output
 * is the round-to-nearest-even of the fp32 result.
 *
 *   out              device [num_seqs, num_heads, head_dim], bf16 or f32 (out_dtype)
 *   query            device [num_seqs, num_heads, head_dim] bf16
 *   key_cache,
 *   value_cache      device [num_blocks, num_kv_heads, block_size, head_dim] bf16
 *   block_tables     device [num_seqs, max_blocks_per_seq] int32; entries past
 *                    ceil(L/bs) are never read
 *   context_lens     device [num_seqs] int32; each must be <= max_context_len and
 *                    <= max_blocks_per_seq*block_size, else the row is zeroed and
 *                    PKV_DEV_BAD_CONTEXT is set
 *   max_context_len  host upper bound of context_lens (sizes the split)
 *   head_dim 64 or 128; block_size 16 or 32; num_heads % num_kv_heads == 0
 *   partition_tokens 0 = automatic; else 64, 128, 256 or 512 (a multiple of block_size):
 *                    sequences longer than this are split into partitions that run
 *                    in parallel and are merged by log-sum-exp rescaling
 *   path             PKV_PATH_AUTO / PKV_PATH_SIMT / PKV_PATH_TENSOR
 *   workspace        device scratch of >= pkv_paged_attention_workspace_size(...)
 *                    bytes, 256-byte aligned; its contents need no initialisation
 *                    and are clobbered; calls sharing one workspace must not overlap
 *                    on the GPU.
 */
PKV_API int pkv_paged_attention_decode(void* out, int out_dtype, const void* query, const void* key_cache,
                               const void* value_cache, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, int num_seqs, int num_heads, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, float scale,
                               int partition_tokens, int path, void* workspace,
                               size_t workspace_bytes, int32_t* status, pkv_stream_t stream);

/*
 * paged_attention_decode_static — pkv_paged_attention_decode without a workspace
 * argument, for callers that cannot allocate device memory.  The source pages have
 * no counterpart: this is a deployment convenience of this library.
 *
 * Who needs it: code that only receives its input and output buffers (for example
 * a plugin called through a runtime's custom-operator interface that offers no
 * scratch space), or applications that hand all device memory to their own
 * allocator or forbid device allocations while running.
 *
 * How it works: the scratch lives in a fixed array of PKV_STATIC_SCRATCH_BYTES
 * compiled into libpkv.so, present on every GPU that loads the library until the
 * process exits.  This call allocates nothing.  Arguments, results and device
 * status bits are those of pkv_paged_attention_decode.
 *   - Sizes whose workspace (pkv_paged_attention_workspace_size) exceeds
 *     PKV_STATIC_SCRATCH_BYTES return PKV_ERR_INVALID with an explanation; nothing
 *     is enqueued.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture starts.  With CUDA's lazy module loading (the
 *     default) the array's PKV_STATIC_SCRATCH_BYTES are also taken from device
 *     memory only then, so make the first call before handing the rest of device
 *     memory to another allocator.
 *   - The address is kept for the life of the process: after cudaDeviceReset on a
 *     device this entry point must not be used on that device again.
 *   - Sizes the workspace variant refuses (an unsupported block_size or head_dim,
 *     and so on) give the same return code as pkv_paged_attention_decode.
 *   - All calls on one device share the array.  Calls whose kernels overlap on the
 *     GPU (for example on two streams without ordering between them) race and give
 *     wrong results; order them on one stream or use the workspace variant.
 */
#define PKV_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
PKV_API int pkv_paged_attention_decode_static(void* out, int out_dtype, const void* query, const void* key_cache,
                                              const void* value_cache, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* context_lens,
                                              int max_context_len, int num_seqs, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size, int num_blocks, float scale,
                                              int partition_tokens, int path, int32_t* status,
                                              pkv_stream_t stream);

/*
 * 8-bit (e4m3) KV cache.  intelliparadigm article §4.2 (初始化速度慢: loading in low-bit
 * fp8) and §5 (quantisation combined with vLLM shrinks memory and raises throughput).
 * The pages fix no format; this library stores K and V as OCP e4m3 codes (1 sign,
 * 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448, no infinities)
 * with one float32 scale per kv head for K and one for V:
 *   code = e4m3(x / scale[h])   (float32 division, round to nearest even, saturate)
 *   value = e4m3_value(code) * scale[h]
 * Pools: key_cache, value_cache = [num_blocks, num_kv_heads, block_size, head_dim]
 * uint8, half the bytes of the bf16 pool; k_scale, v_scale = device [num_kv_heads] float32.
 *
 * reshape_and_cache_fp8 — pkv_reshape_and_cache for an 8-bit pool: key/value are the
 * new tokens' bf16 [num_tokens, num_kv_heads, head_dim], quantised on the way in.
 * Slot rules and status bits as for pkv_reshape_and_cache.
 */
PKV_API int pkv_reshape_and_cache_fp8(const void* key, const void* value, void* key_cache, void* value_cache,
                                      const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                                      int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                                      int block_size, int32_t* status, pkv_stream_t stream);
/*
 * paged_attention_decode_fp8 — pkv_paged_attention_decode over an 8-bit pool: the
 * attention of the dequantised values (K_j = e4m3_value * k_scale[h], V_j likewise).
 * head_dim 128.  path PKV_PATH_SIMT: CUDA cores (the e4m3 tiles are widened to f16
 * in registers, products accumulate in fp32); PKV_PATH_TENSOR (2 <= group <= 16):
 * the tiles are widened to f16 on chip and both products run on the tensor cores
 * with fp32 accumulators (the queries are rounded to f16, after a 2^-16 scale when
 * one of a kv head's queries reaches 2^15; P is rounded to f16); PKV_PATH_AUTO takes
 * the tensor cores whenever they apply.  Workspace, splits and status bits as for
 * pkv_paged_attention_decode (size it with pkv_paged_attention_workspace_size).
 */
PKV_API int pkv_paged_attention_decode_fp8(void* out, int out_dtype, const void* query, const void* key_cache,
                                           const void* value_cache, const float* k_scale, const float* v_scale,
                                           const int32_t* block_tables, int max_blocks_per_seq,
                                           const int32_t* context_lens, int max_context_len, int num_seqs,
                                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                                           int num_blocks, float scale, int partition_tokens, int path,
                                           void* workspace, size_t workspace_bytes, int32_t* status,
                                           pkv_stream_t stream);

/*
 * swap_blocks — the pool's overflow path (intelliparadigm article §4.2 OOM错误:
 * swap_space extends the cache into host memory).  For each (src, dst) pair of
 * block_mapping, block dst of dst_pool <- block src of src_pool, block_bytes bytes,
 * in one kernel launch.  One pool is normally device memory and the other pinned host
 * memory (cudaHostAlloc / cudaHostRegister, mapped at the same address on the
 * device); either may be device memory.  The two pools must not overlap.
 *   src_pool, dst_pool  16-byte aligned, [src_blocks] / [dst_blocks] blocks of block_bytes
 *   block_mapping       [num_pairs, 2] int64 in device or pinned host memory
 *   block_bytes         a multiple of 16 (one layer's K or V block; call once per pool)
 * A pair outside either pool sets PKV_DEV_BAD_PAIR and is skipped.  Memory that is
 * neither device nor pinned-and-mapped is PKV_ERR_INVALID (checked on the host).
 */
PKV_API int pkv_swap_blocks(const void* src_pool, void* dst_pool, const int64_t* block_mapping, int num_pairs,
                            int src_blocks, int dst_blocks, int64_t block_bytes, int32_t* status,
                            pkv_stream_t stream);

/*
 * paged_attention_prefill — causal attention of a batch of prompt chunks over the
 * paged pool (tensor cores).  Outcome School explainer, "LLM serving的基本流程与KV缓存"
 * (prefill reads the whole prompt and stores every token's K/V) and intelliparadigm
 * article §4.1/§4.2 (chunked prefill: a long prompt in pieces, e.g. 512 tokens).
 *
 * Sequence s holds context_lens[s] = L tokens in the pool, the last n = query_start[s+1]
 * - query_start[s] of which are this call's new tokens (write them with
 * pkv_reshape_and_cache first).  Row query_start[s] + i of `query` is the token at
 * position p = L - n + i; for every query head h it gets
 *   out[row, h] = softmax_j(scale * q·k_j) · v_j   over positions j = 0 .. p
 * with K/V of kv head h / (num_heads / num_kv_heads), read through block_tables[s].
 *   out          device [total_q, num_heads, 128], out_dtype BF16 or F32
 *   query        device [total_q, num_heads, 128] bf16 (rows of all sequences packed)
 *   key_cache, value_cache, block_tables, num_blocks, block_size: as for decode
 *   query_start  device [num_seqs + 1] int32, non-decreasing, query_start[num_seqs] <= total_q
 *   context_lens device [num_seqs] int32, n <= L <= min(max_context_len, max_blocks_per_seq*block_size)
 *   workspace    device, pkv_paged_attention_prefill_workspace_size() bytes, 256-byte aligned
 * head_dim must be 128 and num_heads / num_kv_heads must divide 128 (PKV_ERR_UNSUPPORTED);
 * scale must be finite and positive (PKV_ERR_INVALID: hidden keys are -inf scores).
 * A sequence whose numbers break the rules above sets PKV_DEV_BAD_CONTEXT and its rows
 * (when their range is valid) are written as zeros; a table entry outside the pool sets
 * PKV_DEV_BAD_BLOCK and its 16-row slice of keys is skipped.  The pages leave the
 * visibility rule open; the reading here is the causal one of a prompt: a token sees
 * itself and every earlier token, never a later one.
 */
PKV_API size_t pkv_paged_attention_prefill_workspace_size(int num_seqs, int total_q, int num_heads,
                                                          int num_kv_heads);
PKV_API int pkv_paged_attention_prefill(void* out, int out_dtype, const void* query, const void* key_cache,
                                        const void* value_cache, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* query_start,
                                        const int32_t* context_lens, int num_seqs, int total_q,
                                        int max_context_len, int num_heads, int num_kv_heads, int head_dim,
                                        int block_size, int num_blocks, float scale, void* workspace,
                                        size_t workspace_bytes, int32_t* status, pkv_stream_t stream);

/*
 * Shared-prefix decode — decode attention that reads each block shared by several
 * tables once per kv head instead of once per table.  Outcome School explainer,
 * "内存共享": requests with a common system prompt, and the beams of one request, map
 * the same physical blocks; vLLM 初探 §1.4 counts the memory this saves (30-50% with
 * shared system prompts).  The result is that of pkv_paged_attention_decode.
 *
 * Softmax attention over a sequence's tokens splits exactly over any partition of
 * those tokens: with each part's unnormalised sum o_i, its running maximum m_i and its
 * weight sum l_i (base-2 scores), out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,
 * M = max_i m_i.  The plan cuts every row's tokens into a chain of shared segments
 * (runs of whole blocks that a range of ADJACENT rows holds in common, at the same
 * positions of their tables) followed by the row's private remainder.  Run:
 *   1. shared phase: each segment is a dense contraction of all its rows' query heads
 *      against the segment's keys (the tensor-core prefill kernel with every key
 *      visible and unnormalised partial results), cut into key chunks for parallelism;
 *   2. private phase: every row's remainder through a decode kernel writing partial
 *      results only: the CUDA-core decode when no remainder is longer than 128 tokens
 *      (one tile; many short items, as after beams fork), else the tensor-core decode
 *      (grouped heads, head_dim 128);
 *   3. merge: per (row, head), the formula above over the row's shared partials and
 *      its private partitions.
 *
 * pkv_shared_plan (host only, nothing touches the GPU) builds the plan from host
 * copies of the tables and lengths.  Rows share a segment only when they are adjacent
 * in the batch (order the rows so that sharers sit together: a prompt's requests, a
 * parent and its beams) and the segment's blocks are full for every one of them.
 *   block_tables   host [num_seqs, max_blocks_per_seq] int32; context_lens host [num_seqs]
 *                  (0 <= L <= max_blocks_per_seq * block_size, else PKV_ERR_INVALID)
 *   min_rows       fewest rows a segment serves (>= 2).  Over bf16 pools 2 pays: a
 *                  segment reads its blocks once instead of once per row.  Over 8-bit
 *                  pools a segment's blocks are first widened to bf16 (read 1 byte, write
 *                  and read 2 per value), more than rows reading the codes themselves up
 *                  to about 4 rows: there 5 is the better choice (a 4-beam batch: 0.139 ms
 *                  per call against 0.175 with 4-row segments, on one B200).
 *   key_chunk      tokens per part of a segment: a multiple of 128, or 0 = automatic
 *                  (the largest of 2048 .. 128 that gives at least 64 shared-phase work items)
 *   plan           host buffer of plan_bytes, or NULL to only fill `info` (info->bytes
 *                  is then the size to provide); too small a buffer is PKV_ERR_INVALID
 *   info           host, filled on success: counts and the byte offset of each section
 * Copy the plan's first info->bytes bytes to device memory (16-byte aligned) for the run.
 */
typedef struct pkv_shared_plan_info {
  int32_t num_seqs;          /* rows the plan was made for */
  int32_t num_segments;      /* shared segments found */
  int32_t num_parts;         /* segments cut into key chunks */
  int32_t num_entries;       /* shared-phase work entries (pairs of 128-row query tiles of a part) */
  int32_t num_partials;      /* (part, row) partial results of the shared phase */
  int32_t max_suffix_len;    /* longest private remainder of a row, tokens */
  int32_t key_chunk;         /* tokens per part */
  int32_t group;             /* num_heads / num_kv_heads */
  int32_t block_size;
  int32_t max_blocks_per_seq;
  int64_t shared_row_tokens; /* sum over rows of the tokens their segments serve */
  int64_t shared_tokens;     /* sum over segments of their tokens (each read once per kv head) */
  uint64_t off_entries;      /* int4[num_entries]: first row, 0, rows of tile A | rows of tile B << 8, part */
  uint64_t off_parts;        /* int4[2 * num_parts]: (table row, first block, keys, first row),
                                (rows, first partial, first scratch block, 0); parts' scratch blocks
                                follow each other in plan order, shared_tokens / block_size in all */
  uint64_t off_suffix_lens;  /* int32[num_seqs]: tokens of each row's private remainder */
  uint64_t off_block_offset; /* int32[num_seqs]: table index where the remainder starts */
  uint64_t off_row_start;    /* int32[num_seqs + 1]: CSR of each row's shared partials */
  uint64_t off_row_ids;      /* int32[num_partials] */
  uint64_t bytes;            /* plan size */
} pkv_shared_plan_info;

PKV_API int pkv_shared_plan(const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                            int num_seqs, int num_heads, int num_kv_heads, int block_size, int min_rows,
                            int key_chunk, void* plan, size_t plan_bytes, pkv_shared_plan_info* info);

/*
 * Run of a shared-prefix plan.  Arguments as for pkv_paged_attention_decode, plus
 *   plan        device copy of the plan made for these tables and lengths (16-byte aligned)
 *   info        host, the plan's info
 *   workspace   device, pkv_paged_attention_decode_shared_workspace_size() bytes, 256-byte aligned
 * bf16 pools (the 8-bit form follows); head_dim 128; 2 <= num_heads / num_kv_heads <= 16 (the tensor-core
 * decode) — else PKV_ERR_UNSUPPORTED; scale finite and positive, else PKV_ERR_INVALID.  block_tables and context_lens must be those the
 * plan was made from: the call checks on the device that every row's shared tokens plus its
 * remainder equal its context length (and the plan's ranges); a plan that does not fit sets
 * PKV_DEV_BAD_CONTEXT and every output row is zero.
 * The shared phase runs on a side stream of the library, forked from `stream` after the
 * checks and joined back before the merge (event waits, so the call as a whole stays ordered
 * on `stream`); the side stream and its two events are created on the first call on each
 * device — make that call before any stream capture — and kept until the process exits.
 */
PKV_API size_t pkv_paged_attention_decode_shared_workspace_size(const pkv_shared_plan_info* info, int num_heads,
                                                                int num_kv_heads, int head_dim);
PKV_API int pkv_paged_attention_decode_shared(void* out, int out_dtype, const void* query, const void* key_cache,
                                              const void* value_cache, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* context_lens,
                                              int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                              int block_size, int num_blocks, float scale, const void* plan,
                                              const pkv_shared_plan_info* info, void* workspace,
                                              size_t workspace_bytes, int32_t* status, pkv_stream_t stream);

/*
 * The same over an 8-bit (e4m3) pool: key_cache / value_cache are [num_blocks, num_kv_heads,
 * block_size, 128] uint8 codes with one float32 scale per kv head in k_scale / v_scale
 * (device), as for pkv_paged_attention_decode_fp8, whose result this is (intelliparadigm
 * article §4.2 and §5: fp8 KV loading; Outcome School explainer, "内存共享": shared blocks).
 * The shared phase first widens the codes of the plan's shared blocks into two bf16 scratch
 * pools inside the workspace (exact: every e4m3 value is a bf16 value), then runs with each
 * kv head's key scale folded into its scores and its value scale into its partial outputs;
 * the private phase is the 8-bit decode (CUDA cores or tensor cores, by the same rule).  Workspace:
 * pkv_paged_attention_decode_shared_fp8_workspace_size() bytes, the bf16 call's plus the split
 * queries, two scratch pools of info->shared_tokens * num_kv_heads * 128 * 2 bytes and a table
 * of num_seqs * max_blocks_per_seq int32.  A table entry of a shared block outside the pool
 * sets PKV_DEV_BAD_BLOCK and its keys are left out, as in every decode.  Errors as for the
 * bf16 call; null scales are PKV_ERR_INVALID.
 */
PKV_API size_t pkv_paged_attention_decode_shared_fp8_workspace_size(const pkv_shared_plan_info* info,
                                                                    int num_heads, int num_kv_heads, int head_dim);
PKV_API int pkv_paged_attention_decode_shared_fp8(void* out, int out_dtype, const void* query,
                                                  const void* key_cache, const void* value_cache,
                                                  const float* k_scale, const float* v_scale,
                                                  const int32_t* block_tables, int max_blocks_per_seq,
                                                  const int32_t* context_lens, int num_seqs, int num_heads,
                                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                  float scale, const void* plan, const pkv_shared_plan_info* info,
                                                  void* workspace, size_t workspace_bytes, int32_t* status,
                                                  pkv_stream_t stream);

/*
 * Host block manager — free list + reference counts + per-sequence block tables.
 * Outcome School explainer, "vLLM的核心创新：PagedAttention" (a block only when needed,
 * any free block serves any request, finished requests return all blocks at once)
 * and "内存共享" (shared prefixes, beams).  Not thread-safe: one manager per host
 * thread, or external locking.  All ids are host values; nothing touches the GPU.
 *
 * Free list: FIFO.  Its initial order is `initial_order` (a permutation of
 * 0..num_blocks-1; NULL = ascending); freed blocks join the back in table order.
 */
PKV_API pkv_bm* pkv_bm_create(int num_blocks, int block_size, const int32_t* initial_order);
PKV_API void pkv_bm_destroy(pkv_bm* bm);
PKV_API int pkv_bm_num_blocks(const pkv_bm* bm);
PKV_API int pkv_bm_block_size(const pkv_bm* bm);
PKV_API int pkv_bm_num_free(const pkv_bm* bm);
/* Copy the free list, front first, into host `out` (up to cap); returns the count. */
PKV_API int pkv_bm_free_list(const pkv_bm* bm, int32_t* out, int cap);
/* Take the front free block with reference count 1 (PKV_ERR_OOM if none). */
PKV_API int pkv_bm_alloc(pkv_bm* bm, int32_t* block_out);
PKV_API int pkv_bm_incref(pkv_bm* bm, int32_t block);   /* block must be live */
PKV_API int pkv_bm_decref(pkv_bm* bm, int32_t block);   /* at 0 the block joins the free list */
PKV_API int pkv_bm_refcount(const pkv_bm* bm, int32_t block);   /* >= 0, or PKV_ERR_INVALID */
/*
 * New sequence of num_tokens tokens.  Its first n_shared table entries are the
 * given live blocks (a shared prefix; each gains a reference; they must be full:
 * n_shared*block_size <= num_tokens); the rest are fresh blocks.  All-or-nothing.
 */
PKV_API int pkv_bm_add_seq(pkv_bm* bm, int64_t seq_id, int num_tokens, const int32_t* shared_prefix_blocks,
                   int n_shared);
/* Child gets a copy of the parent's table and length; every block gains a reference. */
PKV_API int pkv_bm_fork(pkv_bm* bm, int64_t parent, int64_t child);
/*
 * One new token for each of the n sequences (distinct ids), in order.  For each:
 * if its next position starts a block, a fresh block is appended; else if its last
 * block is shared (reference count > 1) a fresh block replaces it, the pair
 * (old, new) is appended to cow_pairs_out and old loses one reference.
 * slots_out[i] = slot of the new token of seq_ids[i].
 *   slots_out     host [n] int64
 *   cow_pairs_out host [n, 2] int64 (capacity n pairs), *n_cow_out = pairs written;
 *                 feed them to pkv_copy_blocks before writing the new tokens.
 * All-or-nothing: PKV_ERR_OOM if the pool cannot cover every fresh block.
 */
PKV_API int pkv_bm_append_slots(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* slots_out,
                        int64_t* cow_pairs_out, int* n_cow_out);
/* Slots of positions start..start+count-1 of a sequence (host [count] int64). */
PKV_API int pkv_bm_slots(const pkv_bm* bm, int64_t seq_id, int start, int count, int64_t* slots_out);
/* Drop the sequence; each of its blocks loses a reference, in table order. */
PKV_API int pkv_bm_free_seq(pkv_bm* bm, int64_t seq_id);
PKV_API int pkv_bm_seq_len(const pkv_bm* bm, int64_t seq_id);      /* >= 0, or PKV_ERR_INVALID */
PKV_API int pkv_bm_seq_blocks(const pkv_bm* bm, int64_t seq_id);   /* table length, or PKV_ERR_INVALID */
/*
 * Padded tables of the listed sequences: host tables [n, max_blocks] int32
 * (padding 0) and host context_lens [n] int32.  PKV_ERR_INVALID if a table is
 * longer than max_blocks or an id is unknown.
 */
PKV_API int pkv_bm_export_tables(const pkv_bm* bm, const int64_t* seq_ids, int n, int32_t* tables,
                         int max_blocks, int32_t* context_lens);

/*
 * Swap space (intelliparadigm article §4.2 OOM错误: swap_space extends the pool into
 * host memory).  A manager created with num_host_blocks > 0 also owns a pool of host
 * block ids (FIFO free list, initial order 0..num_host_blocks-1, reference counts).
 * pkv_bm_create(...) equals pkv_bm_create_with_swap_space(..., 0).
 *
 * swap_out moves the listed resident sequences to host blocks: every distinct device
 * block among their tables (in order of first appearance, sequence by sequence, table
 * order) gets one host block; the pair (device, host) goes to pairs_out; the table
 * entry becomes the host block and the device block loses one reference (a block still
 * used by a resident sequence stays on the device).  swap_in is the mirror image:
 * pairs (host, device), fresh device blocks from the front of the free list.  Copy
 * every pair with pkv_swap_blocks (every layer, K and V) before the freed blocks are
 * written again.  Both calls are all-or-nothing: PKV_ERR_OOM if the destination pool
 * lacks blocks, PKV_ERR_INVALID if pairs_out (host [cap, 2] int64) is too small.
 * While swapped out, a sequence can only be swapped in or freed (free_seq releases its
 * host blocks); append_slots, slots, fork and export_tables refuse it.
 */
PKV_API pkv_bm* pkv_bm_create_with_swap_space(int num_blocks, int block_size, const int32_t* initial_order,
                                              int num_host_blocks);
PKV_API int pkv_bm_num_host_free(const pkv_bm* bm);
PKV_API int pkv_bm_host_refcount(const pkv_bm* bm, int32_t block);   /* >= 0, or PKV_ERR_INVALID */
PKV_API int pkv_bm_is_swapped(const pkv_bm* bm, int64_t seq_id);     /* 1, 0, or PKV_ERR_INVALID */
PKV_API int pkv_bm_swap_out(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* pairs_out, int cap,
                            int* n_pairs_out);
PKV_API int pkv_bm_swap_in(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* pairs_out, int cap,
                           int* n_pairs_out);

/*
 * Automatic prefix caching (Outcome School explainer, "内存共享": requests with the same
 * prefix keep one copy of its blocks; vLLM 初探 §1.4: a shared system prompt saves
 * 30-50% of the memory).  A full block is identified by the chain hash
 *   h_i = FNV-1a-64( h_(i-1) as 8 little-endian bytes || the block's token ids as
 *                    4-byte little-endian integers ),  h_(-1) = 0
 * (FNV-1a-64: start at 0xcbf29ce484222325; per byte xor, then multiply by
 * 0x100000001b3 modulo 2^64).
 *
 * add_seq_tokens creates a sequence from its prompt token ids (host [num_tokens]
 * int32).  It takes the longest run of leading blocks whose hashes are registered, but
 * never the block holding the last token (at most (num_tokens-1)/block_size blocks);
 * those gain a reference (a registered block with no references is taken back out of
 * the free list).  The remaining blocks are fresh; each fresh full block registers its
 * hash unless the hash is already registered.  *cached_tokens_out = tokens whose K/V
 * are already in the pool; the caller computes and writes the rest.  All-or-nothing
 * (PKV_ERR_OOM).  A registered block whose references drop to zero stays registered
 * in the free list until the list hands it out again (eviction in free-list order).
 */
PKV_API int pkv_bm_add_seq_tokens(pkv_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                  int* cached_tokens_out);
/*
 * append_tokens — pkv_bm_append_slots with the token id of each new position (host [n]
 * int32; in decode the token whose K/V the slot will hold is known when its slot is
 * taken).  A sequence created by add_seq_tokens keeps its token history (fork copies
 * it); when a new token completes a block, that block registers under its chain hash
 * exactly as a full prompt block does (unless the hash is registered already; in call
 * order), so a later prompt that continues the generated text finds it.  A plain
 * pkv_bm_append_slots ends a sequence's history (nothing it fills later registers);
 * sequences created by add_seq have none.  Slots, copy-on-write pairs, all-or-nothing
 * and errors as pkv_bm_append_slots.
 */
PKV_API int pkv_bm_append_tokens(pkv_bm* bm, const int64_t* seq_ids, const int32_t* tokens, int n,
                                 int64_t* slots_out, int64_t* cow_pairs_out, int* n_cow_out);
PKV_API int pkv_bm_num_cached_blocks(const pkv_bm* bm);

/*
 * stream_read — measurement helper, not part of the attention path: reads `bytes` of
 * device memory once (16-byte non-caching loads, 4 CTAs of 512 threads per SM) and
 * XORs every 32-bit word of it into *sink (device, 4-byte aligned; the caller sets it
 * first, usually to 0).  Timing it gives the HBM read bandwidth reached in the same
 * run as the decode kernels (the roofline's read-only reference next to the measured
 * copy peak).  src 16-byte aligned, bytes a multiple of 16; PKV_ERR_INVALID otherwise.
 */
PKV_API int pkv_stream_read(const void* src, size_t bytes, uint32_t* sink, pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */

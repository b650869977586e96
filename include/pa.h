/*
 * pa.h -- C ABI of libpa.so: paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * The operations come from web pages describing vLLM's PagedAttention:
 *   - "详解vLLM推理引擎架构" (tbr8.org), "PagedAttention 的核心思想": the KV cache is
 *     cut into fixed-size blocks of 16 or 32 tokens scattered over a physical pool and
 *     reached through a per-sequence block table; "Copy-on-Write 与内存共享": a shared
 *     block is copied before it is written.
 *   - "vLLM 深度解读" (luoboask.github.io), section 3 ("PagedAttention CUDA Kernel"):
 *     the cache and query layouts and the per-token score / softmax / weighted sum;
 *     section 7 (Llama attention): new K/V are stored into the cache, then attention
 *     runs over the context including them.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless its name starts with host_.
 *     The caller owns all memory (including the decode workspace); no call allocates
 *     device memory and none keeps per-call state.  The library's own device memory is
 *     static, fixed in size and held from load to exit on every GPU that loads it: the
 *     device error word and the PA_DECODE_STATIC_WORKSPACE_BYTES scratch buffer that only
 *     pa_decode_static_workspace uses.
 *   - Tensors are dense and row-major (C order) unless a stride argument says otherwise.
 *   - Element types are pa_dtype values.  Caches and the decode query must start on a
 *     16-byte boundary.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and never synchronise.  Arguments are validated on the host first: an invalid
 *     call returns a negative pa_status and launches nothing.  PA_ERR_CUDA reports a
 *     launch failure (the CUDA error is left for cudaGetLastError()).
 *   - Data-dependent faults found by the kernels (a block id, slot or pair outside the
 *     pool, a sequence longer than its table) never touch memory out of range: the
 *     offending access is skipped, the affected outputs are NaN, and the first such
 *     fault is recorded in a process-wide device error word that pa_get_device_error()
 *     returns.  A wait that exceeds its bound records PA_DEV_TIMEOUT the same way.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* PA_FP8_E4M3: OCP FP8 E4M3 codes, one byte per element, dequantised as code * scale */
typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = -1,     /* null pointer, bad size, misaligned pointer */
  PA_ERR_UNSUPPORTED = -2, /* valid but not implemented: head_dim, block_size, dtype mix, group size */
  PA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than pa_decode_workspace_size() */
  PA_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  PA_ERR_TOO_LARGE = -5    /* pa_decode_static_workspace: the call needs more scratch than
                              PA_DECODE_STATIC_WORKSPACE_BYTES */
} pa_status;

/* codes returned by pa_get_device_error() */
typedef enum {
  PA_DEV_OK = 0,
  PA_DEV_BAD_BLOCK_ID = 1, /* a block-table entry a sequence needs is outside [0, num_blocks) */
  PA_DEV_BAD_SEQ_LEN = 2,  /* seq_lens[i] < 0 or > max_blocks_per_seq * block_size */
  PA_DEV_BAD_SLOT = 3,     /* slot_mapping[t] >= num_blocks * block_size */
  PA_DEV_BAD_PAIR = 4,     /* a copy_blocks pair names a block outside [0, num_blocks) */
  PA_DEV_TIMEOUT = 5,      /* a bounded wait on an asynchronous copy gave up */
  PA_DEV_BAD_PREFIX = 6    /* pa_decode_prefix: a prefix group is malformed (it is then ignored), or
                              its members' block tables differ inside the shared tokens (their
                              rows are NaN) */
} pa_device_error;

/* Bytes of device workspace the decode entry points need: an upper bound valid for any seq_lens
 * whose entries are all <= max_seq_len, with or without prefix groups.  A call is always
 * accepted with the bound for max_seq_len = max_blocks_per_seq * block_size (pa_decode_multi:
 * num_q_heads = num_q_tokens * the query heads); plain decode may need less.  partition_size 0
 * means the default (512).  Returns 0 for invalid arguments. */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_seq_len,
                                int partition_size);

/* Paged decode attention ("vLLM 深度解读", section 3; grouped-query reading: query head hq
 * uses KV head hq / (num_q_heads / num_kv_heads)).  For every sequence i and query head hq:
 *   out[i, hq, :] = sum_t softmax_t(scale * q[i, hq, :] . K_t) * V_t,  t < seq_lens[i],
 * where token t lives in physical block block_tables[i, t / block_size], position
 * t % block_size, and K_t = k_cache[phys, t % block_size, hq / G, :] (V_t likewise).
 *   out          [num_seqs, num_q_heads, head_dim], out_dtype (f32, f16 or bf16)
 *   q            [num_seqs, num_q_heads, head_dim], q_dtype == kv_dtype or f32
 *   k_cache, v_cache  [num_blocks, block_size, num_kv_heads, head_dim], kv_dtype (f16 or bf16)
 *   block_tables int32 [num_seqs, max_blocks_per_seq]; entries past a sequence's
 *                ceil(seq_lens[i] / block_size) blocks are never read
 *   seq_lens     int32 [num_seqs]; 0 gives an all-zero output row
 *   supported: head_dim 64 or 128, block_size 16 or 32, G = num_q_heads / num_kv_heads
 *   from 1 to 8, num_kv_heads up to 255.  partition_size (0 = 512) must be a multiple of
 *   block_size and at most 32 * block_size: sequences longer than one partition are split into
 *   pieces of whole partitions (see PA_OPT_ITEM_SPLIT) whose partial softmax states are merged
 *   by a second kernel (deterministic: the split depends on the call's arguments and the
 *   device's SM count, never on timing).
 *   workspace    device scratch of >= pa_decode_workspace_size(num_seqs, num_q_heads,
 *                head_dim, max_blocks_per_seq * block_size, partition_size) bytes, 256-byte
 *                aligned; its contents need no initialisation and are overwritten.
 *   An FP8 cache needs its scales: kv_dtype PA_FP8_E4M3 returns PA_ERR_UNSUPPORTED here
 *   (use pa_decode_fp8). */
PA_API int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
              int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
              int max_blocks_per_seq, int64_t num_blocks, int q_dtype, int kv_dtype,
              int out_dtype, int partition_size, void* workspace, size_t workspace_bytes,
              void* stream);

/* pa_decode over an FP8 E4M3 cache ("详解vLLM推理引擎架构", section "量化集成与部署":
 * --kv-cache-dtype fp8; the page gives no format -- read as OCP E4M3 codes with one fp32
 * scale for K and one for V).  K_t = code * k_scale and V_t = code * v_scale; everything
 * else is pa_decode.  k_cache, v_cache: [num_blocks, block_size, num_kv_heads, 128] bytes
 * (head_dim 128 only); q_dtype f32, f16 or bf16; scales finite and > 0.  The tensor-core
 * products run in f16: an f32 query is split into two f16 parts (hi + lo), a 16-bit query is
 * converted to f16 (exact for |q| in [2^-14, 65504]). */
PA_API int pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                         int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                         float k_scale, float v_scale, int max_blocks_per_seq, int64_t num_blocks,
                         int q_dtype, int out_dtype, int partition_size, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Multi-token paged attention: several query tokens per sequence, causal
 * ("详解vLLM推理引擎架构", section "量化集成与部署": speculative decoding verifies N draft tokens in one pass of
 * the large model; section "Chunked Prefill": a prompt is processed in chunks interleaved
 * with decode steps).  The pages give no formula; the reading taken is the plain causal one:
 * the T = num_q_tokens query tokens of sequence i are its last T tokens, already stored in the
 * cache, and query token t (position seq_lens[i] - T + t) attends to tokens 0 ..
 * seq_lens[i] - T + t:
 *   out[i, t, hq, :] = sum_{s <= L - T + t} softmax_s(scale * q[i, t, hq, :] . K_s) * V_s,
 * with L = seq_lens[i] and K_s, V_s, G and the block-table lookup as in pa_decode.
 *   out  [num_seqs, num_q_tokens, num_q_heads, head_dim], out_dtype (f32, f16 or bf16)
 *   q    [num_seqs, num_q_tokens, num_q_heads, head_dim], q_dtype
 *   seq_lens[i] = 0 gives all-zero rows; 0 < seq_lens[i] < num_q_tokens is invalid (its rows
 *   are NaN and pa_get_device_error reports PA_DEV_BAD_SEQ_LEN).
 *   supported: q_dtype == kv_dtype (f16 or bf16) for num_q_tokens > 1 (num_q_tokens 1: every
 *   dtype pair of pa_decode), num_q_tokens up to 65536.  A work item holds up to 32 query rows
 *   (query tokens x grouped heads) per KV head on the warp-MMA kernel, 64 on the tensor-core
 *   kernel (head_dim 128, block_size 16; see PA_OPT_WIDE_KERNEL), 8 with head_dim 64: with more
 *   query tokens, the tokens are split into column groups and each K/V page is read once per
 *   group.
 *   Everything else as pa_decode; the
 *   workspace is pa_decode_workspace_size(num_seqs, num_q_tokens * num_q_heads, head_dim,
 *   max_blocks_per_seq * block_size, partition_size).  num_q_tokens 1 is pa_decode. */
PA_API int pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                           int num_q_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                           int block_size, float scale, int max_blocks_per_seq, int64_t num_blocks,
                           int q_dtype, int kv_dtype, int out_dtype, int partition_size, void* workspace,
                           size_t workspace_bytes, void* stream);

/* pa_decode with prefix groups: sequences that share their first blocks read them once
 * ("详解vLLM推理引擎架构", section "Copy-on-Write 与内存共享": parallel samples of one prompt
 * share the prompt's physical blocks through refcounted block-table entries; the same page,
 * Prefix Caching: requests with a common system prompt share its blocks).  The result is
 * pa_decode's, up to rounding: for each group the shared tokens are attended once for the
 * query rows of all its members (one pass over each shared block per KV head), each member's
 * own tokens once for that member, and the partial softmax states are merged per sequence.
 *   prefix_groups  device int32 [num_groups][3] = (first, members, shared): sequences first ..
 *                  first + members - 1 hold the same physical blocks for their first `shared`
 *                  tokens; groups disjoint (so num_groups <= num_seqs, else
 *                  PA_ERR_INVALID); shared a multiple of block_size and <= every
 *                  member's seq_lens.  A group breaking these rules (both groups of an
 *                  overlapping pair) is ignored
 *                  (its sequences decode alone) and PA_DEV_BAD_PREFIX is recorded; members whose
 *                  block-table entries differ inside the shared tokens get NaN rows and the
 *                  same error.
 *   max_members    members one shared pass serves (larger groups are split): max_members * G
 *                  query rows per KV head, at most 32 (64 where the tensor-core kernel takes the
 *                  call: block_size 16 and the PA_OPT_WIDE_KERNEL rule); above 8 rows only with
 *                  head_dim 128 and q_dtype == kv_dtype (f16 or bf16).
 * Caches f16 or bf16; everything else, the workspace included, as pa_decode.  num_groups 0 is
 * pa_decode. */
PA_API int pa_decode_prefix(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size, float scale,
                            int max_blocks_per_seq, int64_t num_blocks, int q_dtype, int kv_dtype,
                            int out_dtype, int partition_size, const int32_t* prefix_groups,
                            int num_groups, int max_members, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Store the step's new tokens into the paged cache ("vLLM 深度解读", section 7).
 * For each token t with slot = slot_mapping[t] >= 0:
 *   k_cache[slot / block_size, slot % block_size, h, :] = k[t, h, :]  for every KV head h
 * (and v likewise); a negative slot skips the token.
 *   k, v          [num_tokens, num_kv_heads, head_dim] rows, kv_dtype, token t at element
 *                 offset t * k_token_stride (v_token_stride for v); 0 = num_kv_heads * head_dim
 *   slot_mapping  int64 [num_tokens]
 * Slots must be distinct (two tokens on one slot race).  Bit-exact byte copies. */
PA_API int pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, int kv_dtype,
                         int64_t k_token_stride, int64_t v_token_stride, void* stream);

/* pa_reshape_and_cache into an FP8 E4M3 cache: element x of k[t] (v[t]), in in_dtype f32,
 * f16 or bf16, is stored as e4m3(x / k_scale) (v_scale for v): the division rounded to
 * nearest in fp32, the conversion rounded to nearest even and saturated to +-448.  The slot
 * rule, strides (in elements of in_dtype) and error behaviour are those of
 * pa_reshape_and_cache; num_kv_heads * head_dim must be a multiple of 16. */
PA_API int pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache, void* v_cache,
                                    const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                                    int head_dim, int block_size, int64_t num_blocks, int in_dtype,
                                    float k_scale, float v_scale, int64_t k_token_stride,
                                    int64_t v_token_stride, void* stream);

/* Copy-on-write block duplication ("详解vLLM推理引擎架构", "Copy-on-Write 与内存共享"):
 * for each pair p, physical block src_dst_pairs[p][0] of k_cache is copied over block
 * src_dst_pairs[p][1] (and the same for v_cache), block_bytes bytes each
 * (= block_size * num_kv_heads * head_dim * element size, a multiple of 16).
 *   src_dst_pairs  int32 [num_pairs, 2], device
 *   host_pairs     optional host copy of the same pairs: when given, the call checks that
 *                  every id is in range, that no destination repeats and that no
 *                  destination is also a source (so the result does not depend on the
 *                  order the copies run in), returning PA_ERR_INVALID otherwise.  When
 *                  NULL those preconditions are the caller's; out-of-range ids are still
 *                  skipped and reported through pa_get_device_error(). */
PA_API int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst_pairs, int num_pairs,
                   int64_t num_blocks, size_t block_bytes, const int32_t* host_pairs,
                   void* stream);

/* Swap KV blocks between two pools -- preemption ("详解vLLM推理引擎架构", scheduler section:
 * when GPU memory runs short the KV cache of low-priority requests is moved to CPU memory and
 * brought back later; --swap-space).  For each pair p, block src_dst_pairs[p][0] of
 * (src_k_cache, src_v_cache) is copied to block src_dst_pairs[p][1] of (dst_k_cache,
 * dst_v_cache), block_bytes bytes each (a multiple of 16; any element type).
 *   pools        either side may be device memory or pinned host memory that the device
 *                addresses directly (cudaHostAlloc / cudaHostRegister, mapped); 16-byte aligned
 *   src_dst_pairs int32 [num_pairs, 2], device-addressable (device or pinned host memory)
 * One kernel launch for all pairs.  Destinations should be distinct; ids outside
 * [0, num_src_blocks) / [0, num_dst_blocks) are skipped and reported through
 * pa_get_device_error(). */
PA_API int pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache,
                          const void* src_v_cache, const int32_t* src_dst_pairs, int num_pairs,
                          int64_t num_src_blocks, int64_t num_dst_blocks, size_t block_bytes,
                          void* stream);

/* Static description of a pa_status value. */
PA_API const char* pa_strerror(int status);

/* Synchronises `stream`, returns the first pa_device_error recorded on the current device
 * since the last call (or a negative pa_status if reading it failed) and clears it. */
PA_API int pa_get_device_error(void* stream);

/* Diagnostic: runs, on one warp, the bounded mbarrier wait every kernel of the library uses,
 * on a barrier that nothing ever arrives on, for at most `polls` polls (1 .. 2^20; each poll
 * sleeps at most 1 us).  The wait gives up, records PA_DEV_TIMEOUT in the device error word
 * and the kernel returns: this exercises the library's failure path without a fault or hang.
 * Returns PA_ERR_INVALID for polls out of range, else the launch status. */
PA_API int pa_selftest_wait_timeout(int polls, void* stream);

/* Process-wide options.
 *
 * PA_OPT_WIDE_KERNEL chooses the kernel for work items of more than 8 query rows per KV head (the
 * query tokens of pa_decode_multi times the grouped heads, or the members of a pa_decode_prefix
 * group times the grouped heads) on a 16-bit cache with a query of its own type, head_dim 128 and
 * block_size 16:
 *   PA_WIDE_AUTO (default) the tensor-core kernel for calls whose rows per KV head exceed 32 (the
 *                          warp-MMA kernel would split them into column groups and read every
 *                          K/V page once per group), the warp-MMA kernel otherwise;
 *   PA_WIDE_MMA            always the persistent warp-MMA kernel (items of up to 32 rows: two
 *                          consumer warps per ring share each staged page);
 *   PA_WIDE_TCGEN05        always the 5th-generation tensor-core kernel (items of up to 64 rows:
 *                          S = Q.K^T and O += P.V accumulate in tensor memory over chunks of 4
 *                          pages; one loading warp, two MMA-issuing warps and two groups of four
 *                          softmax warps that take the chunks in turn).
 * All three match the same oracle within the attention tolerances.  Other shapes and paths ignore
 * the option.
 *
 * PA_OPT_ITEM_SPLIT chooses how the decode calls cut the sequences into work items:
 *   PA_SPLIT_ADAPTIVE (default) pieces of one to four partitions (at most 128 blocks).  Counted
 *                     at one partition each, the call's items come to n per page pipeline of
 *                     the device (SMs x pipelines per SM); shared prefixes, and each sequence's
 *                     leading tokens, go in pieces of min(4, n / 2) partitions, its following
 *                     tokens in pieces of min(4, n / 8), and its ragged tail last, so that the
 *                     items that end a launch are short.  Fewer pieces leave less for the merge
 *                     kernel; the split, and so the rounding of a row, then depends on the batch
 *                     and the device's SM count as well as on the sequence;
 *   PA_SPLIT_FIXED    pieces of exactly partition_size tokens (and a ragged tail): a sequence's
 *                     output is then the same bits in every batch.
 * Both match the oracle within the attention tolerances.
 * Returns PA_OK, or PA_ERR_INVALID for an unknown option or value (nothing changes then). */
#define PA_OPT_WIDE_KERNEL 1
#define PA_WIDE_MMA 0
#define PA_WIDE_TCGEN05 1
#define PA_WIDE_AUTO 2
#define PA_OPT_ITEM_SPLIT 2
#define PA_SPLIT_ADAPTIVE 0
#define PA_SPLIT_FIXED 1
PA_API int pa_set_option(int option, int value);

/* ABI version of this header (major * 100 + minor). */
PA_API int pa_version(void);

/* Size of the library's built-in decode scratch buffer used by pa_decode_static_workspace. */
#define PA_DECODE_STATIC_WORKSPACE_BYTES (64ull << 20)

/* pa_decode without a caller-provided workspace (the pages have no counterpart: this is
 * an interface convenience, not part of the method).
 *
 * Who needs it: callers that cannot allocate device memory at the time they decode.  A
 * serving engine typically hands almost all free HBM to its paged KV-cache pool at start-up
 * (the pool is sized to a fraction of device memory), so a later cudaMalloc for scratch can
 * fail or force the pool to shrink; a plugin embedded in a host framework may have no
 * allocator of its own at all.  Such callers still pass the inputs and the output (exactly as
 * for pa_decode, minus workspace / workspace_bytes); the scratch comes from one buffer of
 * PA_DECODE_STATIC_WORKSPACE_BYTES (64 MiB) compiled into the library as a device global,
 * which every GPU that loads the library holds until the process exits.
 *
 * Behaviour:
 *   - The computation, arguments, layouts and results are those of pa_decode.
 *   - A call whose workspace requirement, pa_decode_workspace_size(num_seqs, num_q_heads,
 *     head_dim, max_blocks_per_seq * block_size, partition_size), exceeds
 *     PA_DECODE_STATIC_WORKSPACE_BYTES returns PA_ERR_TOO_LARGE and launches nothing.
 *   - The first call on each device looks up that device's address of the buffer (a host
 *     runtime call); make that first call before any stream capture on the device.
 *   - Nothing is allocated or freed, by this call or by anything it calls.
 *   - All calls on a device share the one buffer and it keeps the previous call's contents;
 *     what must start at zero is reset by the call itself.  Calls whose kernels can overlap
 *     on the GPU (different streams, different host threads) race on the buffer: serialise
 *     them, e.g. by issuing them on one stream. */
PA_API int pa_decode_static_workspace(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* seq_lens, int num_seqs,
                                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                      float scale, int max_blocks_per_seq, int64_t num_blocks, int q_dtype,
                                      int kv_dtype, int out_dtype, int partition_size, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

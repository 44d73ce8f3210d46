/*
 * pa.h -- C ABI of the paged KV-cache decode library (libpa.so, sm_100a).
 *
 * Pages this interface follows (cited by title and section):
 *   [P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解"
 *        section 2.2 (iteration-level scheduler), 3.2 (fixed-size blocks, block
 *        table, a new block only when the current one is full), 3.3 (allocate /
 *        append_token).
 *   [P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析"
 *        section 2.1 (Block: ref_count, data of shape (BLOCK_SIZE, NUM_HEADS,
 *        HEAD_SIZE)), 2.2 (memory pool, copy-on-write, block-level kernel
 *        scheduling), 3.2 (preemptive scheduling), 6.2 (kernel signature
 *        paged_attention_kernel(out, q, k, v, block_tables)).
 *   [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置"
 *        section "PagedAttention分页注意力机制原理" (block table lookup inside the
 *        attention kernel over non-contiguous blocks, prefix sharing by
 *        reference, free-block pool) and "连续批处理Continuous Batching配置".
 *
 * Conventions for every call below
 * --------------------------------
 * Ownership.  All tensors are owned by the caller.  Device pointers must point
 *   to memory of the current CUDA device; host pointers to ordinary (ideally
 *   pinned) host memory.  The library never allocates device memory: scratch
 *   space for the split-K path is passed in (pa_decode_workspace_size).  The
 *   host block manager and scheduler own only host memory.
 * Layouts (all row-major, contiguous):
 *   q, out          [num_seqs, num_heads, head_dim]
 *   k, v (new rows) [num_tokens, num_kv_heads, head_dim]
 *   k_cache,v_cache [num_blocks, block_size, num_kv_heads, head_dim]   (one
 *                   pool for K, one for V; [P2] 2.1's block data shape)
 *   block_tables    int32 [num_seqs, max_blocks_per_seq]; entry j of row s is
 *                   the physical block holding logical tokens
 *                   [j*block_size, (j+1)*block_size) of sequence s.  Entries
 *                   at or past ceil(context_len/block_size) are never read.
 *   context_lens    int32 [num_seqs]; tokens held by each sequence, the
 *                   current step's new token included.
 *   slot_mapping    int64 [num_tokens]; slot = block*block_size + offset;
 *                   negative = padding token, not written.
 * Supported shapes.  dtype in {PA_F32, PA_F16, PA_BF16}; head_dim in {64, 128};
 *   block_size in {8, 16, 32}; num_heads % num_kv_heads == 0; base pointers
 *   16-byte aligned.  Anything else returns PA_ERR_UNSUPPORTED or
 *   PA_ERR_INVALID_ARG before any launch.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Device calls are asynchronous on that stream.
 * Errors.  Argument errors are reported synchronously before any launch.
 *   A failed launch returns PA_ERR_CUDA.  Device-side data (block ids, slots,
 *   context lengths) are preconditions; the kernels check them anyway, clamp
 *   or skip the bad access (never faulting), and set bits in a device error
 *   word read by pa_get_device_error.
 * Threads.  Calls on different streams may run concurrently; a pa_bm or
 *   pa_sched object must not be used from two threads at once.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* malformed argument, unknown sequence id */
    PA_ERR_UNSUPPORTED = 2,   /* shape / dtype outside the supported set */
    PA_ERR_NO_BLOCKS = 3,     /* free list cannot satisfy the request */
    PA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    PA_ERR_DEVICE = 5         /* a kernel flagged bad device data or a timeout */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/* Geometry of one K or V pool. */
typedef struct {
    int num_blocks;
    int block_size;
    int num_kv_heads;
    int head_dim;
    pa_dtype dtype;
} pa_cache_desc;

/* Bits of the device error word. */
#define PA_DEVERR_SLOT        0x1u  /* cache write: slot >= num_blocks*block_size (skipped) */
#define PA_DEVERR_BLOCK_ID    0x2u  /* decode / copy: block id outside [0, num_blocks) (clamped / skipped) */
#define PA_DEVERR_CONTEXT_LEN 0x4u  /* decode: context_len < 0, > max_context_len or > table width (clamped) */
#define PA_DEVERR_TIMEOUT     0x8u  /* decode: a bounded wait on a staging barrier expired (CTA abandoned its work) */
#define PA_DEVERR_SMEM_ALIGN  0x10u /* verify (tcgen05): the dynamic shared memory base was not 1024-byte aligned;
                                       the kernel needs it aligned to fit two CTAs per SM and did no work */

/* ------------------------------------------------------------------------ */
/* Device hot path                                                           */
/* ------------------------------------------------------------------------ */

/*
 * pa_cache_write -- append each new token's K/V to its slot ([P1] 3.2-3.3: the
 * new token is written at the end of the sequence's current block, or at the
 * start of a freshly taken block).
 *   k, v            device, [num_tokens, Hkv, D] of cache->dtype
 *   k_cache,v_cache device pools described by `cache`
 *   slot_mapping    device int64 [num_tokens]
 * For every t with slot_mapping[t] >= 0:
 *   k_cache[slot / bs][slot % bs][:][:] = k[t][:][:]   (same for v), bit-exact.
 * Non-negative slots must be distinct within one call (tokens are written in
 * parallel; for a repeated slot it is unspecified which row remains).
 * num_tokens == 0 is a no-op.
 */
pa_status pa_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens,
                         const pa_cache_desc* cache, void* stream);

/*
 * Scratch bytes pa_decode needs for a batch of this shape.  Zero when the
 * whole batch fits one partition (max_context_len <= partition size) -- the
 * single-pass path uses no scratch.  partition_size 0 = library default (512).
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim,
                                int max_context_len, int partition_size);

/*
 * pa_decode -- one decode step of paged attention over a continuous batch
 * ([P3] "PagedAttention分页注意力机制原理": the kernel resolves each logical block
 * through the block table and runs attention over non-contiguous physical
 * blocks; [P2] 6.2: out, q, k, v, block_tables).
 *   out             device [num_seqs, num_heads, head_dim] (written)
 *   q               device [num_seqs, num_heads, head_dim]
 *   k_cache,v_cache device pools [num_blocks, block_size, num_kv_heads, head_dim]
 *   block_tables    device int32 [num_seqs, max_blocks_per_seq]
 *   context_lens    device int32 [num_seqs]
 *   scale           softmax scale applied to the fp32 dot products
 * For sequence s with n = context_lens[s] tokens and query head h, kv head
 * g = h / (num_heads / num_kv_heads):
 *   out[s][h] = sum_t softmax_t(scale * q[s][h] . K_s[t][g]) * V_s[t][g]
 * with fp32 accumulation and an fp32 softmax; n == 0 writes a zero row.
 * Contexts longer than the partition size (partition_size, 0 = 512 tokens)
 * are split into partitions whose partial results are merged by a
 * log-sum-exp reduction; the workspace (device, >= pa_decode_workspace_size
 * bytes, 256-byte aligned, contents undefined on entry) holds the partials.
 * max_context_len must bound every context_lens[s]; larger values are clamped
 * and flagged (PA_DEVERR_CONTEXT_LEN).  At most 4096 partitions per sequence
 * (PA_ERR_UNSUPPORTED beyond).
 */
pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int block_size, int num_kv_heads,
                    int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                    int max_context_len, int num_blocks, pa_dtype dtype,
                    int partition_size, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * pa_write_decode -- one decode step of a continuous batch in one call: the
 * new tokens' K/V appended to their slots, then decode attention over the
 * block tables ([P1] 3.2-3.3 for the append, [P3] "PagedAttention分页注意力机制原理"
 * for the attention).  Same arguments, layouts, results and errors as
 *   pa_cache_write(k, v, k_cache, v_cache, slot_mapping, num_tokens, &desc, stream);
 *   pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, ...);
 * with desc = {num_blocks, block_size, num_kv_heads, head_dim, dtype}: the
 * decode sees every row the write appends.  Every argument of both is checked
 * before anything is launched.  Fewer launches than the two calls: when the
 * batch is split into partitions, one kernel does the write and orders the
 * partitions, so the attention kernel follows it directly.  num_tokens == 0
 * is pa_decode alone.
 */
pa_status pa_write_decode(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens,
                          void* out, const void* q, void* k_cache, void* v_cache,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          int block_size, int num_kv_heads,
                          int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                          int max_context_len, int num_blocks, pa_dtype dtype,
                          int partition_size, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Scratch bytes pa_verify needs (zero when every context fits one partition).
 */
size_t pa_verify_workspace_size(int num_seqs, int num_queries, int num_heads, int head_dim,
                                int max_context_len, int partition_size);

/*
 * The partition pa_verify uses for these shapes: partition_size itself when
 * non-zero.  Otherwise, with R = num_heads / num_kv_heads x num_queries query
 * rows per kv head, C = ceil(R / 64) row chunks and the item bound
 * items(P) = num_seqs x ceil(max_context_len / P) x num_kv_heads x C:
 *   2048 tokens when R >= 32, block_size >= 16, num_seqs x num_kv_heads x C
 *        >= 592 and items(2048) >= 1776;
 *   1024 tokens when R >= 32 and items(1024) >= 1776;
 *   512 otherwise.
 * Larger partitions write fewer split-K partials (R x (head_dim + 2) floats per
 * kv head and partition) and cross fewer item boundaries; the bound keeps about
 * six items per CTA of the kernel's grid.  max_context_len is the longest
 * context (pa_verify passes min(max_context_len, max_blocks_per_seq x
 * block_size)).  No device work; never fails (argument checks are pa_verify's).
 */
int pa_verify_partition_size(int num_seqs, int num_queries, int num_heads, int num_kv_heads, int max_context_len,
                             int block_size, int partition_size);

/*
 * pa_verify -- multi-query paged attention: the target model's verification
 * pass of speculative decoding ([P1] "大模型推理引擎高频优化：连续批处理、
 * PagedAttention 与 KV Cache 实战拆解", section 5: a draft model proposes a
 * handful of candidate tokens and the target model checks them in one
 * parallel pass).  Every sequence brings num_queries (Q) query rows per head;
 * their K/V must already be the last Q positions of its paged context (write
 * them with pa_cache_write first).
 *   out   device [num_seqs, Q, num_heads, head_dim] (written)
 *   q     device [num_seqs, Q, num_heads, head_dim]
 *   other arguments as for pa_decode.
 * Query i of sequence s with n = context_lens[s] sits at position
 * p = n - Q + i and attends to positions 0..p of its own sequence:
 *   out[s][i][h] = sum_{t <= p} softmax_t(scale * q[s][i][h] . K_s[t][g]) V_s[t][g],
 *   g = h / (num_heads / num_kv_heads)
 * (Q = 1 is pa_decode).  A row with p < 0 (a context shorter than Q) is a zero
 * row.  fp16 and bf16 only (tensor cores; fp32 returns PA_ERR_UNSUPPORTED);
 * 1 <= Q <= 64.  Long contexts are split and merged as in pa_decode; the
 * workspace (>= pa_verify_workspace_size bytes, 256-byte aligned) holds the
 * partials.  partition_size 0 lets pa_verify_partition_size choose (512, 1024
 * or 2048 tokens); pa_verify_workspace_size(..., 0) covers each.  An explicit
 * partition_size is a multiple of 32 from 32 to 2048 with at most 128 blocks
 * (the kernels' block-id table).
 */
pa_status pa_verify(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int block_size, int num_kv_heads,
                    int num_seqs, int num_queries, int num_heads, int head_dim, int max_blocks_per_seq,
                    int max_context_len, int num_blocks, pa_dtype dtype,
                    int partition_size, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Tensor-core path of pa_verify (process-wide):
 *   PA_VERIFY_MMA_SYNC  warp-level mma.m16n8k16 with accumulators in registers
 *   PA_VERIFY_TCGEN05   tcgen05.mma issued by one thread, accumulators and p in
 *                       tensor memory, K/V and q in shared memory (M = 64 query
 *                       rows per item); the faster kernel at every measured shape
 *   PA_VERIFY_AUTO      the kernel measured fastest: PA_VERIFY_TCGEN05
 * Same results within the stated tolerance; bits differ between the two.
 */
#define PA_VERIFY_MMA_SYNC 0
#define PA_VERIFY_TCGEN05 1
#define PA_VERIFY_AUTO 2    /* default: the tcgen05 kernel */
pa_status pa_set_verify_kernel(int kind);
int pa_get_verify_kernel(void);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart to this call: it exists for users of
 * this library whose device memory is already spoken for (a serving engine
 * that gives nearly all of it to the KV block pool and allocates nothing
 * afterwards) or who may not call cudaMalloc on their path (an allocation can
 * synchronise the device).  Same inputs, outputs and result as pa_decode; the
 * split-K scratch is a fixed device array of PA_NOALLOC_SCRATCH_BYTES inside
 * the library instead of a caller-supplied workspace.
 *   - Every GPU on which the library is loaded holds that array until exit.
 *   - A batch needing more scratch than that (pa_decode_workspace_size, with
 *     max_context_len capped at max_blocks_per_seq x block_size as pa_decode
 *     caps it) is rejected with PA_ERR_UNSUPPORTED before any launch.
 *   - The first call on a device looks up the array's device address for that
 *     device and keeps it for the device's current context; make that first
 *     call before any stream capture.  A call made in another context of the
 *     device (after cudaDeviceReset, for one) looks the address up again.
 *   - All calls share the array and it keeps the last call's contents (no part
 *     of it needs to start at zero); calls that overlap on the GPU race on it.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens, float scale,
                            int block_size, int num_kv_heads,
                            int num_seqs, int num_heads, int head_dim, int max_blocks_per_seq,
                            int max_context_len, int num_blocks, pa_dtype dtype,
                            int partition_size, void* stream);

/*
 * pa_copy_blocks -- copy-on-write support ([P2] 2.2: a shared block is copied
 * before it is written).  pairs: device int32 [num_pairs][2] of (src, dst)
 * physical block ids; copies the whole block (all block_size slots, all heads)
 * in both pools.  Destinations must be distinct and must not appear as a
 * source in the same call.  Out-of-range ids are skipped and flagged.
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int num_pairs,
                         const pa_cache_desc* cache, void* stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools of the same block
 * shape (cache->block_size, num_kv_heads, head_dim, dtype), K and V alike
 * ([P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
 * section "生产部署注意事项": KV cache swapped out to CPU memory when GPU memory
 * runs short and back in later).  Either pool may be device memory or PINNED
 * host memory (cudaHostAlloc / cudaHostRegister; pageable host memory is
 * rejected with PA_ERR_INVALID_ARG); a host pool is read or written in place
 * by one kernel launch over the host link.
 *   dst_k, dst_v   pools of dst_blocks blocks
 *   src_k, src_v   pools of src_blocks blocks
 *   pairs          int32 [num_pairs][2] of (source block, destination block),
 *                  device or pinned host memory
 * Destinations must be distinct and must not be read as sources in the same
 * call.  Out-of-range ids are skipped and flagged (PA_DEVERR_BLOCK_ID).  The
 * copy is asynchronous on `stream`; keep the host pool alive and unmodified
 * until it completes.  cache->num_blocks is ignored.
 */
pa_status pa_swap_blocks(void* dst_k, void* dst_v, int dst_blocks, const void* src_k, const void* src_v,
                         int src_blocks, const int32_t* pairs, int num_pairs, const pa_cache_desc* cache,
                         void* stream);

/*
 * pa_step -- one layer-step driven from HOST buffers: copies the step's inputs
 * host->device (one cudaMemcpyAsync per buffer), runs pa_copy_blocks (when
 * num_cow > 0), pa_cache_write and pa_decode, and copies `out` back
 * device->host.  The caller provides the device staging buffers (no
 * allocation here).  Returns once the work is enqueued; the host output is
 * valid after the stream synchronizes.  NULL structs or pools, negative
 * counts and an unknown dtype return PA_ERR_INVALID_ARG before any copy; the
 * remaining checks of pa_copy_blocks / pa_cache_write / pa_decode run after
 * the input copies are enqueued and return their status before their own
 * launch; a failed copy returns PA_ERR_CUDA.  Host buffers should be pinned
 * for the copies to be asynchronous.
 */
typedef struct {
    /* host inputs */
    const void* q;               /* [num_seqs, num_heads, head_dim] */
    const void* k;               /* [num_tokens, num_kv_heads, head_dim] */
    const void* v;
    const int64_t* slot_mapping; /* [num_tokens] */
    const int32_t* block_tables; /* [num_seqs, max_blocks_per_seq] */
    const int32_t* context_lens; /* [num_seqs] */
    const int32_t* cow_pairs;    /* [num_cow][2], may be NULL when num_cow == 0 */
    /* host output */
    void* out;                   /* [num_seqs, num_heads, head_dim] */
} pa_step_host;

typedef struct {
    /* device staging buffers of the same shapes as pa_step_host's */
    void* q; void* k; void* v;
    int64_t* slot_mapping; int32_t* block_tables; int32_t* context_lens;
    int32_t* cow_pairs; void* out;
    void* workspace; size_t workspace_bytes;
} pa_step_device;

typedef struct {
    int num_seqs, num_heads, num_kv_heads, head_dim;
    int block_size, num_blocks, max_blocks_per_seq, max_context_len;
    int num_tokens, num_cow;
    pa_dtype dtype;
    float scale;
    int partition_size;
} pa_step_shape;

pa_status pa_step(const pa_step_host* host, const pa_step_device* dev, void* k_cache,
                  void* v_cache, const pa_step_shape* shape, void* stream);

/*
 * pa_pipeline -- pa_step with its host<->device copies on two copy streams
 * owned by the pipeline, so that consecutive steps overlap: while step i
 * computes on `stream`, step i+1's inputs travel host->device and step i-1's
 * output travels device->host.  The caller provides `depth` staging sets
 * (pa_step_device, each with its own buffers and workspace) and uses set
 * i % depth for step i; the pipeline orders, per set, the input copies after
 * the previous compute that read the set, the compute after those copies and
 * after the previous output copy that read the set's `out`, and the output
 * copy after the compute.  Host buffers are read and written asynchronously:
 * keep them unchanged (inputs) and unread (output) until pa_pipeline_end
 * returns or its work on `stream` has completed.
 *   pa_pipeline_begin   the copy streams wait for work enqueued on `stream` so far
 *   pa_pipeline_step    one layer-step as pa_step (same arguments) on staging set `set`
 *   pa_pipeline_end     `stream` waits for every copy enqueued so far
 * Not thread-safe per pipeline.
 */
typedef struct pa_pipeline pa_pipeline;
pa_status pa_pipeline_create(int depth, pa_pipeline** out);
void pa_pipeline_destroy(pa_pipeline* p);
pa_status pa_pipeline_begin(pa_pipeline* p, void* stream);
pa_status pa_pipeline_step(pa_pipeline* p, int set, const pa_step_host* host, const pa_step_device* dev,
                           void* k_cache, void* v_cache, const pa_step_shape* shape, void* stream);
pa_status pa_pipeline_end(pa_pipeline* p, void* stream);

/*
 * Arithmetic used by pa_decode's score and output contractions (process-wide):
 *   PA_MATH_AUTO   tensor cores (mma m16n8k16, fp32 accumulate) for fp16 / bf16,
 *                  CUDA-core fp32 FMAs for fp32 -- the default;
 *   PA_MATH_SIMT   CUDA-core fp32 FMAs for every dtype;
 *   PA_MATH_TENSOR same as AUTO (fp32 always uses CUDA cores).
 * Both paths give results within the same tolerance of the exact attention;
 * bits differ between them.  Not to be changed while a decode is being
 * enqueued on another thread.
 */
typedef enum { PA_MATH_AUTO = 0, PA_MATH_SIMT = 1, PA_MATH_TENSOR = 2 } pa_decode_math;
pa_status pa_set_decode_math(int mode);
int pa_get_decode_math(void);

/*
 * How pa_decode merges the partitions of split sequences (process-wide):
 *   PA_MERGE_KERNEL  a separate log-sum-exp reduce kernel runs after decode
 *                    -- the default (measured faster on B200);
 *   PA_MERGE_FUSED   the decode kernel's CTA that finishes a sequence's last
 *                    partition merges them (no extra launch).
 * Both compute M = max_i m_i, o = sum_i 2^(m_i-M) o_i / sum_i 2^(m_i-M) l_i in
 * partition order; bits may differ in the last place between the two.
 */
typedef enum { PA_MERGE_FUSED = 0, PA_MERGE_KERNEL = 1 } pa_split_merge;
pa_status pa_set_split_merge(int mode);
int pa_get_split_merge(void);

/* Reads and clears the device error word (synchronizes `stream`).  Returns
 * PA_ERR_DEVICE when any bit was set, PA_OK otherwise. */
pa_status pa_get_device_error(uint32_t* flags, void* stream);

/* Diagnostic of the kernels' bounded waits: launches one CTA on `stream` that
 * waits on a shared-memory barrier nothing arrives at.  The wait gives up after
 * its limit (2 s of %globaltimer), the CTA sets PA_DEVERR_TIMEOUT and exits;
 * read it with pa_get_device_error.  Returns PA_ERR_CUDA if the launch fails. */
pa_status pa_check_wait_expiry(void* stream);

/* A static English description of a status code (never NULL; "unknown status"
 * for values outside the enum). */
const char* pa_status_string(pa_status status);

/* ------------------------------------------------------------------------ */
/* Launch accounting and per-kernel device time                              */
/* ------------------------------------------------------------------------ */

typedef enum {
    PA_KERNEL_CACHE_WRITE = 0,
    PA_KERNEL_DECODE = 1,        /* single-pass or partition kernel */
    PA_KERNEL_REDUCE = 2,        /* log-sum-exp merge of partitions */
    PA_KERNEL_PLAN = 3,          /* orders partitions longest-first */
    PA_KERNEL_COPY_BLOCKS = 4,
    PA_KERNEL_VERIFY = 5,        /* multi-query (verification) kernel */
    PA_KERNEL_SWAP = 6,          /* block moves between device and host pools */
    PA_KERNEL_WRITE_PLAN = 7,    /* pa_write_decode: cache write and plan in one kernel */
    PA_KERNEL_COUNT = 8
} pa_kernel_id;

/* Number of kernels this library has launched in the process so far. */
int64_t pa_launch_count(void);

/* Start recording a CUDA event pair around every launch (on its stream);
 * clears earlier records. */
pa_status pa_profile_begin(void);

/* Same, recording only the kernels whose bit (1 << pa_kernel_id) is set in
 * kernel_mask; fewer event pairs disturb the timed stream less. */
pa_status pa_profile_begin_mask(uint32_t kernel_mask);

/* Stop recording, wait for the recorded events, and return per kernel id the
 * summed device milliseconds and launch counts (arrays of PA_KERNEL_COUNT). */
pa_status pa_profile_end(double* total_ms, int64_t* launches);

/* ------------------------------------------------------------------------ */
/* Host block manager (no CUDA calls)                                        */
/* ------------------------------------------------------------------------ */

typedef struct pa_bm pa_bm;

/* Pool of num_blocks blocks of block_size tokens.  initial_free_order (may be
 * NULL = 0..num_blocks-1) is the free list's initial content; blocks are taken
 * from its END ([P1] 3.3, free_blocks.pop()). */
pa_status pa_bm_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                       pa_bm** out);
void pa_bm_destroy(pa_bm* bm);

/* New sequence holding num_tokens tokens: takes ceil(num_tokens/block_size)
 * blocks in logical order ([P1] 3.3 allocate). */
pa_status pa_bm_allocate(pa_bm* bm, int64_t seq_id, int num_tokens);

/* child shares every block of parent by reference (ref_count + 1 each;
 * prefix sharing [P3], parallel sampling [P2] 1.1). */
pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child);

/* Reserve the slot of the sequence's next token.  Takes a fresh block only when
 * the last one is full ([P1] 3.3 append_token); copies a shared last block
 * first ([P2] 2.2): then cow_src and cow_dst receive the block pair to copy,
 * otherwise both are -1.  On PA_ERR_NO_BLOCKS nothing changes. */
pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                            int32_t* cow_dst);

/* Release a sequence: walk its table in logical order, decrement, and push
 * blocks reaching zero onto the free list. */
pa_status pa_bm_free(pa_bm* bm, int64_t seq_id);

/* Copy the sequence's block table (logical order) into out[0..cap); *n = its
 * length (also when cap is too small, which returns PA_ERR_INVALID_ARG). */
pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq_id, int32_t* out, int cap, int* n);

/* Slots of logical positions [start, start+count) of a sequence. */
pa_status pa_bm_slots(const pa_bm* bm, int64_t seq_id, int start, int count, int64_t* out);

/* Pool statistics; context_len receives the sequence's token count, or -1
 * when seq_id is unknown (pass seq_id < 0 to skip). */
pa_status pa_bm_stats(const pa_bm* bm, int64_t seq_id, int* num_free, int* num_used,
                      int* context_len);

/* Reference count of one physical block, and the free list from bottom to top
 * (the next block taken is free_list[n-1]). */
pa_status pa_bm_ref_count(const pa_bm* bm, int32_t block, int* count);
pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int cap, int* n);

/* Pack the tables and context lengths of a batch into the device layout:
 * tables [n][width] padded with -1, context_lens [n]. */
pa_status pa_bm_pack(const pa_bm* bm, const int64_t* seq_ids, int n, int width,
                     int32_t* tables, int32_t* context_lens);

/* Memory actually used by the pool's live sequences ([P3] "大模型推理显存优化
 * 实战：PagedAttention机制原理与vLLM连续批处理配置", sections on the memory
 * bottleneck and on paged attention: contiguous per-request reservation wastes
 * memory, paging wastes at most the tail of each sequence's last block).
 * *held_blocks = blocks whose count is above zero; *filled_slots = their slots
 * below the context length of at least one holder (a shared block is counted
 * once).  Reserved-but-unused share = 1 - filled / (held x block_size).
 * Either pointer may be NULL. */
pa_status pa_bm_usage(const pa_bm* bm, int64_t* held_blocks, int64_t* filled_slots);

/* ---- prefix cache ([P3] "Prefix Caching前缀复用优化": a request whose prompt
 * starts with cached KV references those blocks and skips their prefill) ----
 *
 * Off by default; with it off every call below behaves like its plain
 * counterpart and the pool behaves exactly as described above.  With it on, a
 * FULL block is cached under the exact key (parent block, its block_size token
 * ids), where parent is the previous block of the same table or -1 for the
 * first block; the key therefore names the whole token prefix up to the end of
 * that block.  A cached block whose count reaches zero is not put on the free
 * list: it waits on an LRU list (counted as free by pa_bm_stats) and is evicted
 * (its key dropped, the block reused) only when the free list is empty.
 * Partly filled blocks are never shared through the cache. */
pa_status pa_bm_enable_prefix_cache(pa_bm* bm, int enable);

/* New sequence with the prompt tokens[0..num_tokens): references the longest
 * run of cached full blocks that starts the prompt (ref_count + 1 each) and
 * takes fresh blocks for the rest, registering the new full ones.
 * *cached_tokens (may be NULL) = block_size x the blocks found: the caller
 * writes K/V only for positions >= *cached_tokens.  On PA_ERR_NO_BLOCKS nothing
 * changes (the hit/lookup counters included). */
pa_status pa_bm_allocate_prefix(pa_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                int* cached_tokens);

/* pa_bm_append_slot that also records the token id, so that the block it
 * fills can be cached.  A sequence made by pa_bm_allocate, or that got a slot
 * from pa_bm_append_slot, has unknown tokens: its later blocks are not cached. */
pa_status pa_bm_append_token(pa_bm* bm, int64_t seq_id, int32_t token, int64_t* slot,
                             int32_t* cow_src, int32_t* cow_dst);

/* ---- host swap pool ([P3] "生产部署注意事项": KV cache moved out to CPU memory
 * when GPU memory runs short, back in when it frees up) ----
 *
 * Size the host pool (block ids 0..num_cpu_blocks-1 on a LIFO free list, like
 * the GPU list); not while a sequence is swapped out. */
pa_status pa_bm_set_cpu_blocks(pa_bm* bm, int num_cpu_blocks);

/* Swap a resident sequence out: every block it holds ALONE (count 1) moves to
 * a host block, in logical order, and the GPU block goes back to the free
 * list; shared blocks stay resident and referenced.  With the prefix cache
 * on, such a block that the cache names keeps its name and waits on the
 * evictable list instead (last block first), its K/V reusable on the GPU
 * until evicted.  pairs receives *n (gpu, cpu) pairs ([n][2], cap pairs of
 * room) for pa_swap_blocks, which must run before the released GPU blocks are
 * written again.  All or nothing: PA_ERR_NO_BLOCKS when the host pool is
 * short, PA_ERR_INVALID_ARG when cap is short (nothing changes; *n tells the
 * need).  A swapped-out sequence cannot append, fork, pack or give slots
 * until it is swapped in; pa_bm_free releases it. */
pa_status pa_bm_swap_out(pa_bm* bm, int64_t seq_id, int32_t* pairs, int cap, int* n);

/* Swap a sequence back in, in logical order: a block it left named in the
 * prefix cache is taken back with no copy while the cache still names it by
 * the same key (another holder may share it meanwhile); every other host
 * block gets a fresh GPU block (free list first, else an evicted one) and a
 * (cpu, gpu) copy in pairs.  Needs as many free blocks (free list + evictable)
 * as the sequence has host blocks; all or nothing, as for pa_bm_swap_out.  On
 * success *n is the number of copies (at most the host blocks; the cap check
 * uses the host block count). */
pa_status pa_bm_swap_in(pa_bm* bm, int64_t seq_id, int32_t* pairs, int cap, int* n);

/* *swapped = 1 while the sequence is swapped out; the host free list from
 * bottom to top. */
pa_status pa_bm_swapped(const pa_bm* bm, int64_t seq_id, int* swapped);
pa_status pa_bm_cpu_free_list(const pa_bm* bm, int32_t* out, int cap, int* n);

/* Cached blocks (in use or not), evictable blocks (cached, count zero),
 * full blocks found and full blocks probed by pa_bm_allocate_prefix so far;
 * any pointer may be NULL. */
pa_status pa_bm_cache_stats(const pa_bm* bm, int* cached_blocks, int* evictable_blocks,
                            int64_t* hits, int64_t* lookups);

/* The evictable blocks, next victim first; *n = their number (also when cap is
 * too small, which returns PA_ERR_INVALID_ARG). */
pa_status pa_bm_evictable(const pa_bm* bm, int32_t* out, int cap, int* n);

/* Drop the cache key of `block`, which must be cached with count zero (on the
 * evictable list), and put it on the free list.  For K/V that must not be
 * found again: the writes that filled the block were abandoned (a scheduler
 * preempted their sequence within the same step).  PA_ERR_INVALID_ARG when the
 * block is out of range, referenced or not cached; nothing changes then. */
pa_status pa_bm_forget(pa_bm* bm, int32_t block);

/* ------------------------------------------------------------------------ */
/* Host scheduler: iteration-level (continuous) batching                     */
/* ------------------------------------------------------------------------ */

typedef struct pa_sched pa_sched;

/* Scheduler over `bm` (not owned) with at most max_running running sequences.
 * prefix_seq >= 0 names a sequence already resident in bm whose blocks
 * prefix-sharing requests fork. */
pa_status pa_sched_create(pa_bm* bm, int max_running, int64_t prefix_seq, pa_sched** out);
void pa_sched_destroy(pa_sched* s);

/* Queue a request (FCFS).  prompt_len counts the request's own tokens (the
 * shared prefix excluded).  fork_child >= 0 forks a parallel-sampling child
 * with that id right after the prompt is placed. */
pa_status pa_sched_add_request(pa_sched* s, int64_t seq_id, int prompt_len, int output_len,
                               int shares_prefix, int64_t fork_child, int fork_output_len);

/* Run one iteration ([P1] 2.2): finish, admit (FCFS, stop at the first request
 * that does not fit the free-block budget), then reserve every running
 * sequence's next slot, preempting the most recently admitted sequence when
 * the pool is exhausted.  The step's record is kept until the next call.
 * The budget charge covers every block an admission takes, so the block
 * manager's own calls do not fail inside a step; if one does (the block
 * manager was changed behind the scheduler's back), its status is returned and
 * the scheduler and block manager are left part-way through the step: destroy
 * both. */
pa_status pa_sched_step(pa_sched* s);

/* Sizes of the last step's record. */
typedef struct {
    int num_finished, num_admitted, num_preempted, num_ops, num_running, num_waiting;
} pa_sched_counts;
pa_status pa_sched_counts_get(const pa_sched* s, pa_sched_counts* c);

/* The last step's record.  Any pointer may be NULL to skip that array.
 *   finished/admitted/preempted: sequence ids in event order.
 *   ops: num_ops entries in issue order; op_kind[i] = 0 for a cache write
 *        (a = seq, b = position, c = slot), 1 for a copy-on-write block copy
 *        (a = src block, b = dst block, c = -1), and with preemption by swap
 *        2 for a swap-out copy (a = GPU block, b = host block) or 3 for a
 *        swap-in copy (a = host block, b = GPU block).  Ops apply in issue
 *        order: a copy after every earlier write and before every later one.
 *        Ops made dead by a preemption in the same step are not listed, so no
 *        slot appears twice within a run of consecutive writes.
 *   running/context_lens: the batch to decode, in admission order. */
/* Preemption mode ([P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续
 * 批处理配置", section "生产部署注意事项"): PA_PREEMPT_RECOMPUTE (default) frees a
 * victim's blocks and re-writes its history on re-admission; PA_PREEMPT_SWAP
 * swaps it out to the block manager's host pool when its private blocks fit
 * (else recomputes) and swaps it back in, before any new admission, once its
 * host blocks + 1 fit the step's budget.  Swapped sequences keep their
 * progress and come back in FIFO order. */
#define PA_PREEMPT_RECOMPUTE 0
#define PA_PREEMPT_SWAP 1
pa_status pa_sched_set_preemption(pa_sched* s, int mode);

/* The last step's swap events: ids swapped out and in (in event order), and
 * the sequences currently waiting swapped out. */
pa_status pa_sched_swap_counts(const pa_sched* s, int* num_swapped_out, int* num_swapped_in,
                               int* num_swapped);
pa_status pa_sched_swap_record(const pa_sched* s, int64_t* swapped_out, int64_t* swapped_in);

pa_status pa_sched_record(const pa_sched* s, int64_t* finished, int64_t* admitted,
                          int64_t* preempted, int32_t* op_kind, int64_t* op_a, int64_t* op_b,
                          int64_t* op_c, int64_t* running, int32_t* context_lens);

/* ---- admission through the prefix cache ([P3] "Prefix Caching前缀复用优化") ----
 *
 * Token id of position `position` of sequence `seq_id`, the token whose K/V a
 * decode step writes there (in a server: the token sampled at the previous
 * step).  Called from pa_sched_step on the calling thread; must be pure for a
 * given (seq_id, position), since a retried reservation asks again. */
typedef int32_t (*pa_token_fn)(void* ctx, int64_t seq_id, int64_t position);

/* Switch the scheduler to admission through the prefix cache.  Needs
 * pa_bm_enable_prefix_cache on its block manager, token_fn non-NULL, and no
 * request queued yet; prefix_tokens[0..n) are the ids of the prefix holder's
 * tokens (n = its length when the scheduler was made with prefix_seq >= 0,
 * else 0).  Each full block of the holder must be the block the cache names
 * for these ids (make the holder with pa_bm_allocate_prefix): then every
 * admission takes at most the blocks the budget charges it.  Otherwise, or
 * when the holder is swapped out, PA_ERR_INVALID_ARG.  Then:
 *   - requests come in through pa_sched_add_request_tokens (pa_sched_add_request
 *     returns PA_ERR_INVALID_ARG); a prefix-sharing request's token history is
 *     prefix_tokens followed by its own;
 *   - admission calls pa_bm_allocate_prefix with the whole history (prompt,
 *     plus the tokens generated so far when a recomputed sequence comes back)
 *     and lists cache writes only for positions past the cached blocks; the
 *     budget charge is the same as without the cache;
 *   - each decode reservation is pa_bm_append_token with token_fn's id;
 *   - a recompute preemption first frees the victim, then forgets
 *     (pa_bm_forget) every block that an op of this step targets and that is
 *     left cached with count zero, in op order, then drops the dead ops: K/V
 *     whose writes are dropped must not be found by a later lookup.  Cached
 *     blocks written in earlier steps keep their keys.
 * Default off: the scheduler behaves exactly as described above. */
pa_status pa_sched_enable_prefix_cache(pa_sched* s, const int32_t* prefix_tokens, int n,
                                       pa_token_fn token_fn, void* ctx);

/* pa_sched_add_request with the request's own prompt token ids tokens[0..prompt_len)
 * (copied); only with admission through the prefix cache. */
pa_status pa_sched_add_request_tokens(pa_sched* s, int64_t seq_id, const int32_t* tokens, int prompt_len,
                                      int output_len, int shares_prefix, int64_t fork_child,
                                      int fork_output_len);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */

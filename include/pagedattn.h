/*
 * libpagedattn -- paged decode attention for NVIDIA B200 (sm_100a).
 *
 * For every sequence s and query head h the library computes
 *     out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s
 * where the keys and values of sequence s are scattered over fixed-size
 * physical blocks and found through an int32 block table.  This is the
 * problem the PagedAttention pages state:
 *  - "Why PagedAttention was retired", section 1: the block table is a map
 *    [num_seqs, max_blocks] of int32 physical block ids; logical block j of
 *    sequence s lives in physical block block_tables[s][j] (the id is widened
 *    to 64 bits before address arithmetic);
 *  - the same page, section 2: K cache [num_blocks, num_kv_heads,
 *    head_size/x, block_size, x], V cache [num_blocks, num_kv_heads,
 *    head_size, block_size];
 *  - the same page, section 3: logits and softmax, then the softmax-weighted
 *    V, made here in a single pass over each page (online softmax);
 *  - the same page, section 4: K/V may be stored as FP8 e4m3 and are scaled
 *    by a per-tensor k_scale / v_scale when converted;
 *  - "PR #47361 report", benchmark snippet: the call's argument order
 *    (out, query, key_cache, value_cache, num_kv_heads, scale, block_tables,
 *    seq_lens, block_size, max_seq_len, kv_cache_dtype, k_scale, v_scale),
 *    and the split-KV temporaries exp_sums / max_logits / tmp_output of the
 *    partitioned variant, folded here into one opaque workspace.
 *
 * Conventions for every entry point:
 *  - Ownership: the caller allocates and owns every buffer.  pa_decode
 *    allocates nothing, never synchronises, and only enqueues work on the
 *    given stream (a cudaStream_t passed as void*; NULL = legacy default).
 *    Kernels are launched with programmatic stream serialization and wait
 *    for every grid ahead of them before touching memory, so stream order
 *    holds for all they read and write; only their launch overlaps the
 *    previous kernel's end.
 *  - Argument errors are returned synchronously, before any launch.  The
 *    pointer and size checks come before any CUDA call; checks that depend
 *    on the plan (shared memory, workspace size) follow a query of the
 *    current device's SM count.  pa_last_error_detail() names the argument.
 *  - Launch failures return PA_ERR_CUDA.
 *  - Device data is not read on the host.  Kernels check every block id
 *    they use against [0, num_blocks) and every seq_len against
 *    [0, max_blocks_per_seq * block_size] and max_seq_len; a violation sets
 *    a bit in the workspace's status word (PA_DEV_*), the offending block is
 *    skipped and the offending length clamped, and nothing is read out of
 *    bounds.  Read the word with pa_read_device_status.
 *
 * Element types: query and out are bf16.  K/V are bf16 (PA_KV_BF16, x = 8) or
 * e4m3 codes (PA_KV_FP8_E4M3, x = 16); x is 16 bytes / element size.
 * Pointer alignment: out, query, key_cache, value_cache and workspace 16 bytes;
 * block_tables and seq_lens 4 bytes.
 * Supported shapes: head_size 64 or 128; block_size 16 or 32;
 * num_heads / num_kv_heads from 1 to 16 (query head h reads kv head
 * h / (num_heads / num_kv_heads)).
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,        /* null / misaligned pointer, inconsistent sizes    */
    PA_ERR_UNSUPPORTED = 2,        /* head_size, block_size, group size, dtype          */
    PA_ERR_WORKSPACE_TOO_SMALL = 3,/* workspace_bytes < pa_decode_workspace_size(...)   */
    PA_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed              */
    PA_ERR_OUT_OF_BLOCKS = 5       /* block manager: no free block / block-table row full */
} pa_status;

typedef enum pa_kv_dtype {
    PA_KV_BF16 = 0,
    PA_KV_FP8_E4M3 = 1             /* OCP e4m3 ("fn"): bias 7, no inf, 0x7F/0xFF = NaN  */
} pa_kv_dtype;

/* Bits a kernel ORs into the workspace status word (never cleared by kernels). */
#define PA_DEV_BAD_BLOCK_ID 0x1u        /* a block id outside [0, num_blocks): block skipped */
#define PA_DEV_SEQ_LEN_OUT_OF_RANGE 0x2u/* seq_len < 0, > max_blocks*block_size, or beyond
                                           max_seq_len's partitions: length clamped           */
#define PA_DEV_WAIT_TIMEOUT 0x4u        /* a page copy did not land within ~2 s: output void  */
#define PA_DEV_PREFIX_MISMATCH 0x8u     /* a declared shared prefix does not hold             */

/* Bytes at the start of the workspace reserved for the status word. */
#define PA_WORKSPACE_HEADER_BYTES 256
/* After the header, in any workspace larger than the header: the split
 * tail's per-unit CTA counts (at most 1024 units), zero between calls; every
 * plan's partials start after them. */
#define PA_WORKSPACE_MERGE_COUNT_BYTES 4096

/*
 * Tuning knobs; pass NULL for the planner's defaults.
 *  partition_pages: 0 lets the planner choose; > 0 forces split-KV partitions
 *      of that many blocks (the combine kernel merges them).  A value >= the
 *      longest sequence's block count means "no split".  The planner splits
 *      only batches of fewer than two waves of (sequence, kv head) units; it
 *      takes a partition count whose last wave of CTAs is about 62% full, at
 *      most 32 partials per query row where the batch allows it (one or two
 *      long sequences take one partial wave; a handful of units about 128 CTAs
 *      on 148 SMs), and partitions of even size over each sequence's pages.
 *  num_sms: 0 queries the current device; > 0 plans for that many SMs
 *      (lets the host plan without a GPU, e.g. to size a workspace).
 *  stages: 0 lets the planner choose; 2..16 forces that many page buffers
 *      per warp (shared memory grows with it; more than fits is rejected).
 *  shared_prefix_blocks: k > 0 declares that the first k logical blocks are
 *      the same physical blocks in every row of block_tables and that every
 *      seq_len is at least k * block_size -- the prompt reuse that
 *      "vLLM 0.25.0 release-notes commentary", section 1, lists among the gains
 *      of paging (outputs of one prompt read its KV blocks).  The prefix pages
 *      are then streamed once per
 *      group of 16 query rows (all sequences' heads of a kv head packed
 *      together) instead of once per sequence, and merged with each
 *      sequence's own pages by the combine kernel ("cascade" decode).
 *      Kernels verify the declaration and set PA_DEV_PREFIX_MISMATCH when a
 *      row's prefix differs from row 0's or a sequence is shorter than the
 *      prefix (results for that sequence are then undefined).  0 = off.
 *  alibi_slopes: NULL, or a device array of num_heads fp32 slopes.  The call
 *      on "PR #47361 report: Delete PagedAttention" (benchmark snippet) passes
 *      alibi_slopes; the bias itself is not printed there, and is read as the
 *      usual linear bias: the logit of token t (of T) of query head h gains
 *      slope[h] * (t - (T - 1)).  Not combined with shared_prefix_blocks
 *      (PA_ERR_UNSUPPORTED).
 *  fp8_compute: with an e4m3 cache, non-zero runs q.K^T and P.V as e4m3 x e4m3
 *      tensor-core products with fp32 accumulation -- the FP8 compute that
 *      "Why PagedAttention was retired", section 4, names as the successor of
 *      dequantise-on-load -- instead of converting K/V to f16.  K/V codes go
 *      into the products unchanged; the query (scaled by a power of two) and
 *      the softmax weights (x 256) are each carried as a hi + lo pair of e4m3
 *      codes, about 2^-8 relative together, so accuracy stays near the f16
 *      path's.  The query's power of two is shared by the rows one warp
 *      handles: components more than about 2^9 below their largest |q| keep
 *      only an absolute error of about 2^-17 max|q| (the e4m3 subnormal
 *      floor).  Requires kv_dtype = PA_KV_FP8_E4M3.
 *  schedule: how CTAs share the work.  PA_SCHEDULE_AUTO (0) and
 *      PA_SCHEDULE_PARTITIONED: one CTA per (sequence, kv head, partition), as
 *      many waves as that takes; the hardware hands units to SMs as they free
 *      up.  Under PA_SCHEDULE_AUTO, when units are not split and fill two or
 *      three waves of CTA slots (or more, for pages that go in pairs: e4m3
 *      pages of 16 tokens, bf16 ones of head size 64), the units of the last,
 *      partial wave are cut
 *      into partitions whose CTAs follow every whole unit's (the split tail,
 *      pa_plan.tail_units); PA_SCHEDULE_PARTITIONED leaves them whole.
 *      PA_SCHEDULE_BALANCED: one wave of CTAs (grid_ctas = resident CTA
 *      slots), each taking an equal contiguous share of all (sequence, kv
 *      head, page) work; units cut at a share's ends are merged by the
 *      combine kernel, which then runs on every call.  That removes the last
 *      partial wave, but every CTA then waits for the slowest SM; it pays
 *      where SMs stream at even rates (measured on e4m3 pages, ~1%).  Needs
 *      no shared prefix and no forced partition_pages (PA_ERR_UNSUPPORTED).
 *  mha_cuda_cores: non-zero runs q.K^T and P.V of a bf16 cache with one query
 *      head per kv head (num_heads == num_kv_heads, no shared prefix) as fp32
 *      FMAs on the CUDA cores instead of tensor-core tiles, whose 16 rows would
 *      hold that one head; the softmax weights then stay fp32.  Other batches
 *      are not affected.  0 = tensor-core tiles for every batch.
 *  test_stall_copies: for testing the failure path only.  Non-zero makes every
 *      page's completion barrier wait for 16 bytes that no copy delivers and
 *      cuts each wait to ~20 ms, so the kernel takes its give-up path: it lets
 *      the copies it issued land, sets PA_DEV_WAIT_TIMEOUT and returns, with
 *      the output undefined and the context usable.  Every real copy still
 *      completes; nothing faults or hangs.  Use on small problems (each warp
 *      spends ~20 ms per stage).
 */
typedef struct pa_options {
    int partition_pages;
    int num_sms;
    int stages;
    int shared_prefix_blocks;
    const float* alibi_slopes;
    int fp8_compute;
    int test_stall_copies;
    int schedule;
    int mha_cuda_cores;
} pa_options;

/* pa_options.schedule values. */
#define PA_SCHEDULE_AUTO 0
#define PA_SCHEDULE_BALANCED 1
#define PA_SCHEDULE_PARTITIONED 2
#define PA_SCHEDULE_DYNAMIC 3

/* What pa_decode will launch for a given problem. */
typedef struct pa_plan {
    int num_partitions;     /* P: split-KV partitions per (seq, kv head); 1 = no split */
    int partition_pages;    /* blocks per partition                                    */
    int stages;             /* page buffers per warp in shared memory                  */
    int warps_per_cta;      /* consumer warps per CTA                                   */
    long long grid_ctas;    /* CTAs of the decode kernel                                */
    size_t smem_bytes;      /* dynamic shared memory per CTA                            */
    size_t workspace_bytes; /* bytes pa_decode needs in `workspace`                     */
    int prefix_partitions;  /* partitions of a declared shared prefix (0 = none)        */
    int prefix_groups;      /* 16-query-row groups per kv head streaming the prefix     */
    int balanced;           /* 1: balanced page ranges (num_partitions and
                               partition_pages are then 0), 0: fixed partitions        */
    int dynamic;            /* > 0: the dynamic schedule, with this many owner warps
                               per unit; num_partitions and prefix_partitions are then
                               the partial slots per query row of a (sequence, kv head)
                               unit and of a prefix unit, partition_pages is 0,
                               grid_ctas an upper bound; 0: another schedule            */
    long long tail_units;     /* split tail: units of the last, partial wave of whole
                                 units, each cut into tail_partitions partitions of
                                 tail_partition_pages blocks whose CTAs follow every
                                 whole unit's (PA_SCHEDULE_AUTO only); 0: none          */
    int tail_partitions;
    int tail_partition_pages;
    int combine;              /* 1: a pa_combine_kernel launch follows the decode
                                 (split partitions, a shared prefix, balanced and
                                 dynamic schedules); 0: none -- whole units, or a
                                 split tail, whose units' last CTAs merge their
                                 rows inside the decode kernel                  */
    int longest_first;        /* 1: per-sequence CTAs take sequences longest first
                                 (ranked on the device from seq_lens; at most 256
                                 sequences, grids of more than one wave of CTAs) */
} pa_plan;

/*
 * Fill *plan for the given sizes.  Host only; makes a CUDA call only when
 * opts == NULL or opts->num_sms == 0 (to read the SM count).
 */
pa_status pa_plan_decode(pa_plan* plan, int num_seqs, int num_heads, int num_kv_heads,
                         int head_size, int block_size, int max_seq_len, pa_kv_dtype kv_dtype,
                         const pa_options* opts);

/*
 * Workspace bytes pa_decode needs (>= PA_WORKSPACE_HEADER_BYTES), or 0 when the
 * sizes are invalid.  Layout: a 256-byte header whose first uint32 is the
 * status word; when the plan needs more, PA_WORKSPACE_MERGE_COUNT_BYTES of
 * merge counts, then (when P > 1 or a shared prefix is declared) per
 * (seq, query head, partition) an fp32 partial output [head_size], and fp32
 * running max (log2 domain) and sum -- or, with a split tail
 * (pa_plan.tail_units > 0), the same per (tail unit, query head of its
 * group, tail partition).  Under PA_SCHEDULE_BALANCED, after the counts:
 * the per-sequence page prefix and the pages per CTA (num_seqs + 2 ints,
 * padded to 256 bytes), then two slots of G query rows per CTA, each an fp32
 * partial [head_size] with its max and sum.  The sizes depend on the options
 * (pass the ones pa_decode_ex will get).  The caller zeroes the workspace once
 * after allocating it; pa_decode never clears the status word (it is sticky)
 * and overwrites the rest.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                int block_size, int max_seq_len, pa_kv_dtype kv_dtype,
                                const pa_options* opts);

/*
 * Paged decode attention.
 *  out          bf16 [num_seqs, num_heads, head_size], written.
 *  query        bf16 [num_seqs, num_heads, head_size].
 *  key_cache    [num_blocks, num_kv_heads, head_size/x, block_size, x] of kv_dtype.
 *  value_cache  [num_blocks, num_kv_heads, head_size, block_size] of kv_dtype.
 *  scale        logit scale (typically 1/sqrt(head_size)); finite.
 *  block_tables int32 [num_seqs, max_blocks_per_seq].  Entries past a
 *               sequence's last block may be loaded (a warp prefetches its
 *               row up to the end of its partition) but their values are
 *               never used as block ids, so any value is fine there (-1,
 *               stale ids); every entry of a row must be readable memory.
 *  seq_lens     int32 [num_seqs]; 0 gives a zero output row.
 *  max_seq_len  upper bound of seq_lens, used only to plan the split.
 *  num_blocks   blocks in each cache (bounds for block ids).
 *  k_scale, v_scale  device pointers to one fp32 each; required for FP8,
 *               ignored for bf16.
 *  workspace    device buffer of workspace_bytes (see above).
 *  stream       cudaStream_t to enqueue on.
 * All pointers are device pointers.  Accumulation is fp32; out is rounded
 * to bf16 (round to nearest even).
 */
pa_status pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                    int num_seqs, int num_heads, int num_kv_heads, int head_size, float scale,
                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
                    int block_size, int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                    const float* k_scale, const float* v_scale, void* workspace,
                    size_t workspace_bytes, void* stream);

/* pa_decode with tuning options (opts may be NULL). */
pa_status pa_decode_ex(void* out, const void* query, const void* key_cache,
                       const void* value_cache, int num_seqs, int num_heads, int num_kv_heads,
                       int head_size, float scale, const int32_t* block_tables,
                       int max_blocks_per_seq, const int32_t* seq_lens, int block_size,
                       int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                       const float* k_scale, const float* v_scale, void* workspace,
                       size_t workspace_bytes, void* stream, const pa_options* opts);

/*
 * pa_decode without a caller-supplied workspace, for callers that cannot
 * allocate device memory at the point of the call -- for example code that
 * runs inside an allocator callback, a runtime whose memory pool is owned and
 * fully reserved by someone else, or a plugin whose host framework forbids
 * device allocations after start-up.  The decoding pages state no such need;
 * this entry point has no counterpart there.
 *
 * Scratch (the split-KV partials) lives in one fixed array of
 * PA_NOALLOC_SCRATCH_BYTES in the library's own device memory, reserved on
 * every GPU that loads the library until the process exits.  Problems whose
 * plan needs more than that (pa_decode_workspace_size > PA_NOALLOC_SCRATCH_BYTES)
 * are rejected with PA_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 * No allocation is made: no cudaMalloc, cudaFree or allocating library call.
 *
 * The array's device address is looked up once per CUDA context (with
 * cudaGetSymbolAddress, in the caller's current context) and cached under the
 * context's unique id: each context -- another context on the same device,
 * or the new primary context after cudaDeviceReset -- has its own copy of
 * the array at its own address.  The first call in a context does that
 * lookup, which may load the library's device code into the context; make
 * that first call before any stream capture.
 * Every call in a context shares the one array and it keeps the last call's
 * contents; calls that can overlap on the GPU (other streams, other host
 * threads) race on it and must be serialised by the caller.  Nothing in the
 * array needs to start at zero: each call writes every partial it reads.  The
 * device-side range-check bits (PA_DEV_*) of this entry point are recorded in
 * the array but are not reported; use pa_decode with a workspace to read them.
 * Other arguments, pointers and errors are those of pa_decode, and are
 * checked before the scratch size.
 */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)

pa_status pa_decode_noalloc(void* out, const void* query, const void* key_cache,
                            const void* value_cache, int num_seqs, int num_heads, int num_kv_heads,
                            int head_size, float scale, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* seq_lens, int block_size,
                            int max_seq_len, int64_t num_blocks, pa_kv_dtype kv_dtype,
                            const float* k_scale, const float* v_scale, void* stream);

/*
 * Copy the workspace status word to *flags (synchronises `stream`), and
 * zero it afterwards when clear != 0.
 */
pa_status pa_read_device_status(void* workspace, uint32_t* flags, int clear, void* stream);

/* Static text for a status code. */
const char* pa_status_string(pa_status status);

/* Text describing the last error returned on the calling thread ("" if none). */
const char* pa_last_error_detail(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int pa_version(void);

/* ------------------------------------------------------------------------
 * Block manager: hands out physical blocks and keeps the block tables that
 * pa_decode reads.  It follows the PagedAttention idea of "vLLM 0.25.0
 * release-notes commentary", section 1 (a sequence is like a process, a KV
 * block like a page, the block table like a page table): blocks are
 * allocated only when a sequence grows into them, and several sequences
 * (e.g. outputs sampled from one prompt) can share blocks, a shared block
 * being copied before it is written ("copy on write").
 *
 * Host-only bookkeeping, thread-safe (one mutex per manager); it never
 * touches device memory.  Block ids are handed out in increasing order from
 * a LIFO free list, so the sequence of ids is deterministic.
 * ------------------------------------------------------------------------ */
typedef struct pa_block_manager pa_block_manager;

/* A manager of blocks [0, num_blocks) of block_size tokens; a sequence may
 * hold at most max_blocks_per_seq blocks (the block-table row width). */
pa_status pa_bm_create(pa_block_manager** out, int64_t num_blocks, int block_size,
                       int max_blocks_per_seq);
void pa_bm_destroy(pa_block_manager* bm);

/* A new, empty sequence; *seq_id indexes the manager's sequences (ids of
 * freed sequences are reused). */
pa_status pa_bm_add_sequence(pa_block_manager* bm, int* seq_id);

/* A new sequence that shares every block of `parent` (their reference counts
 * go up by one) and has the parent's length. */
pa_status pa_bm_fork(pa_block_manager* bm, int parent, int* child_id);

/* Drop a sequence; blocks no other sequence references return to the pool. */
pa_status pa_bm_free_sequence(pa_block_manager* bm, int seq_id);

/*
 * Grow a sequence by num_tokens, allocating the blocks it grows into.  When
 * the sequence's last block is partly filled and shared with another
 * sequence, that block is first replaced by a private copy: the call then
 * returns *num_copies = 1 with the (source, destination) block ids in
 * *copy_src / *copy_dst, and the caller must copy the block's K/V (for
 * instance with pa_copy_blocks) before writing the new tokens.  All or
 * nothing: on PA_ERR_OUT_OF_BLOCKS nothing changes.
 */
pa_status pa_bm_append_tokens(pa_block_manager* bm, int seq_id, int num_tokens,
                              int64_t* copy_src, int64_t* copy_dst, int* num_copies);

pa_status pa_bm_seq_len(pa_block_manager* bm, int seq_id, int64_t* len);

/*
 * Write the block-table rows and lengths of n sequences, in the given order,
 * into host arrays block_tables [n, max_blocks_per_seq] (unused entries -1)
 * and seq_lens [n], ready to copy to the device for pa_decode.
 */
pa_status pa_bm_export(pa_block_manager* bm, const int* seq_ids, int n, int32_t* block_tables,
                       int max_blocks_per_seq, int32_t* seq_lens);

int64_t pa_bm_num_free_blocks(pa_block_manager* bm);          /* -1 on NULL            */
int pa_bm_refcount(pa_block_manager* bm, int64_t block);       /* -1 on a bad argument  */
const char* pa_bm_last_error_detail(void);                     /* this thread's last    */

/*
 * Copy whole blocks (every kv head, K and V) within the caches:
 * block dst[i] <- block src[i] for i < num_pairs.  src and dst are device
 * arrays of int64 block ids.  A dst id must not appear twice, nor as a src,
 * in one call.  Pairs with an id outside [0, num_blocks) are skipped and set
 * PA_DEV_BAD_BLOCK_ID in *status (a device word; may be NULL).  Enqueued on
 * `stream`; caches 16-byte aligned.
 */
pa_status pa_copy_blocks(void* key_cache, void* value_cache, int num_kv_heads, int head_size,
                         int block_size, int64_t num_blocks, pa_kv_dtype kv_dtype,
                         const int64_t* src, const int64_t* dst, int num_pairs,
                         uint32_t* status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */

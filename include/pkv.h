/*
 * pkv.h - C ABI of the B200 paged KV-cache decode library (libpkv.so).
 *
 * The method: vLLM and PagedAttention (slides "vLLM and PagedAttention: Virtual
 * Memory for LLM Serving", polomodov.tech; note "High-Throughput Serving with
 * vLLM & PagedAttention", dataarena.dev; blog "vLLM PagedAttention architecture
 * deep dive", kashiiupdatez.online).  A sequence's keys and values are stored in
 * fixed-size blocks of B tokens that sit at arbitrary frames of one pool; a
 * per-sequence block table maps logical block j to its physical frame.
 *
 * Conventions for every call:
 *  - Device buffers are owned by the caller.  The library never allocates
 *    device memory; calls that need scratch take a caller-provided workspace.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and never
 *    synchronise, except where stated (pkv_device_error, PKV_VALIDATE=1).
 *  - Every argument is checked on the host before anything is launched; a bad
 *    argument returns an error and launches nothing.  A launch failure returns
 *    PKV_ECUDA.  Kernels never trap: an index that is out of range in device
 *    data (a table entry, a context length, a slot, a copy pair) is skipped or
 *    clamped and reported through the sticky device error flags below.
 *  - Element types: fp16 or bf16 for q, out and the caches (`dtype`).
 *    All row-major, C order, 16-byte aligned base pointers.
 *  - Shapes the decode kernels support: head_dim in {64, 128}, block_size in
 *    {8, 16, 32}, num_heads / num_kv_heads in {1, 2, 4, 8}.  Anything else
 *    returns PKV_EUNSUPPORTED.
 *
 * Environment: PKV_VALIDATE=1 makes the decode, cache-write and block-copy calls
 * copy the block tables / context lengths / slots / copy pairs back to the host,
 * check every index the kernels would use, and return PKV_ERANGE (PKV_EINVAL
 * for a copy list whose pairs depend on their order) instead of launching
 * (this synchronises the stream).
 *
 * CUDA graphs: the first call on a device sets up per-device state (the device
 * address of the error flags, the SM count) and the first decode call of each
 * kernel variant (dtype, head_dim, query heads per kv head, block size) on a
 * device sets that kernel's shared-memory limit and queries its occupancy.
 * Make one warm-up call per device and variant before capturing calls into a
 * CUDA graph; captured calls then run no set-up.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_OK = 0,
  PKV_EINVAL = -1,       /* null pointer, negative size, misaligned buffer, bad workspace */
  PKV_EUNSUPPORTED = -2, /* a shape outside the supported set */
  PKV_ECUDA = -3,        /* a CUDA runtime call or launch failed */
  PKV_ENOMEM = -4,       /* block pool exhausted (allocator) */
  PKV_ERANGE = -5        /* an index out of range (host-checked data, PKV_VALIDATE) */
} pkv_status;

typedef enum { PKV_F16 = 0, PKV_BF16 = 1 } pkv_dtype;

/* Sticky device error flags (bit mask), set by kernels instead of trapping. */
#define PKV_DEVERR_TABLE_ENTRY 1u  /* a block-table entry outside [0, num_blocks): frame 0 read instead */
#define PKV_DEVERR_CONTEXT_LEN 2u  /* a context length < 0 or above the table's capacity: clamped */
#define PKV_DEVERR_SLOT 4u         /* a slot >= num_blocks * block_size: row not written */
#define PKV_DEVERR_COPY_PAIR 8u    /* a copy pair naming a frame outside [0, num_blocks): skipped */
#define PKV_DEVERR_WAIT_TIMEOUT 16u /* a bounded wait (a shared-memory barrier, or the partition
                                        merge waiting for a context's partitions) expired:
                                        output invalid */

/* Human-readable name of a status code (static storage). */
const char* pkv_status_string(pkv_status status);

/* Why the last call on this host thread that returned PKV_ECUDA did so: the
 * cudaError_t of the CUDA runtime call that failed (a launch with too many
 * resources, a sticky fault of earlier work, ...), as an int; 0 if no call on
 * this thread has returned PKV_ECUDA.  Later successful calls leave it as is. */
int pkv_last_cuda_error(void);

/* Name of a cudaError_t value, e.g. "cudaErrorLaunchOutOfResources" (static
 * storage; the runtime's own name table). */
const char* pkv_cuda_error_name(int error);

/* Reads the device error flags of the current device into *flags_out after the
 * work queued on `stream` has finished (synchronises `stream`); clears them
 * when `clear` != 0. */
pkv_status pkv_device_error(unsigned int* flags_out, int clear, cudaStream_t stream);

/*
 * Test hook for the bounded waits (no counterpart on the pages).  Kernels never
 * spin forever: a wait that gives up sets PKV_DEVERR_WAIT_TIMEOUT and the
 * kernel returns.  This call lets a test make the one wait that has no copies
 * in flight run out on purpose: the partition merge's wait for the decode grid
 * to publish a (sequence, kv head) pair.  Every later decode call in the
 * process makes that wait expect `extra` more publications than the decode grid
 * makes and give up after `limit_ns` nanoseconds (0 = the normal 1 s bound).
 * The pairs that time out keep whatever their output rows held.  Call
 * pkv_test_set_merge_wait(0, 0) to restore normal operation.  Not for
 * production use; not synchronised with calls in flight on other threads.
 */
pkv_status pkv_test_set_merge_wait(uint64_t limit_ns, uint32_t extra);

/*
 * Test hook for the partition rules (host only, no GPU needed).  How a decode
 * call cuts each context into partitions is not fixed by the pages (any cut
 * gives the same result within the tolerance; it sets the work split).  This
 * runs the same code the decode, planning and merge kernels run, for a call
 * with these arguments on a decode grid of grid_ctas CTAs (444 for the G <= 4
 * kernels on a 148-SM B200, 296 for G = 8).
 *   context_lens  host int32 [num_seqs], clamped to [0, max_context_len] as the
 *                 kernels do
 *   max_context_len, block_size, partition_size  as in the decode call
 *                 (max_context_len = max_blocks_per_seq * block_size)
 *   n_parts, n_big, p_big, p_small  host int32 [num_seqs], written: context s
 *                 has n_parts partitions, the first n_big of p_big tokens, then
 *                 p_small tokens each, the last one shorter (a single-size rule
 *                 gives n_big = n_parts and p_big = p_small).
 * PKV_EINVAL for a bad argument or an unsupported partition_size.
 */
pkv_status pkv_test_partitions(const int32_t* context_lens, int32_t num_seqs, int32_t num_kv_heads,
                               int32_t max_context_len, int32_t block_size, int32_t partition_size,
                               int32_t grid_ctas, int32_t* n_parts, int32_t* n_big, int32_t* p_big,
                               int32_t* p_small);

/* ------------------------------------------------------------------------ */
/* Decode attention                                                         */
/* ------------------------------------------------------------------------ */

/*
 * Bytes of workspace the decode calls need (always > 0 for valid arguments):
 * 256 bytes of work counters, 4 * num_seqs bytes of sequence list,
 * 4 * num_seqs * num_heads bytes of per-(sequence, kv head) completion counters,
 * 32 * num_seqs * P bytes of work records (one per context partition), and, when
 * P > 1, the partition results num_seqs * num_heads * P * (head_dim + 2) * 4
 * bytes; each piece rounded up to 256 bytes, with
 * P = ceil(max_context_len / partition_size), partition_size 0 (the default
 * policy) counting as 512.
 * Returns 0 for invalid arguments; the decode call then rejects them.
 */
size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                  int32_t max_context_len, int32_t partition_size);

/*
 * Paged decode attention (slides 9-10 "PagedAttention: attention block by block",
 * "Block table: logical to physical"; dataarena note section 2).
 *
 * For each sequence s and query head h (kv head g = h / (num_heads/num_kv_heads)):
 *   out[s,h,:] = sum_t softmax_t(scale * q[s,h,:] . K_s[t,:]) V_s[t,:],  t < context_lens[s]
 * where token t of sequence s lives in frame p = block_tables[s, t / B] at
 * offset t mod B:  K_s[t,:] = k_cache[p, g, t mod B, :]  (V likewise).
 * Accumulation is fp32; out is rounded to `dtype` (round to nearest even).  The
 * softmax weights enter the PV product rounded to `dtype` (their sum, the
 * normaliser, is taken in fp32); max-abs error against exact arithmetic stays
 * within 2e-3 (fp16) / 1e-2 (bf16) for inputs of unit scale.  Results are
 * bit-reproducible run to run and across physical relabellings of the frames.
 * context_lens[s] == 0 gives out[s] = 0.
 *
 *   out          device [num_seqs, num_heads, head_dim]              dtype, written
 *   q            device [num_seqs, num_heads, head_dim]              dtype
 *   k_cache      device [num_blocks, num_kv_heads, block_size, head_dim] dtype
 *   v_cache      device, same shape as k_cache
 *   block_tables device int32 [num_seqs, max_blocks_per_seq]; only the first
 *                ceil(context_lens[s] / block_size) entries of row s are used (the
 *                kernel may read further entries of the row, up to one partition's
 *                worth, without using them, so the whole row must be readable)
 *   context_lens device int32 [num_seqs], 0 <= context_lens[s] <= max_blocks_per_seq * block_size
 *   partition_size maximum tokens per context partition, a multiple of 64 in
 *                [64, 2048]: a context of L tokens is split into ceil(L / partition_size)
 *                near-equal partitions (multiples of 64 tokens) that run on different
 *                CTAs and are merged with a log-sum-exp in the same launch sequence.
 *                0 = the default policy: partitions of up to 1024 tokens; but when the
 *                batch has fewer (sequence, kv head) pairs than the decode grid has
 *                CTAs (a few long contexts), partitions are sized per call so that
 *                the batch's token-heads make about k whole waves of the grid, k =
 *                max(1, round(token-heads / (CTAs x 1024))): a context of L tokens
 *                gets about L k CTAs / token-heads partitions (64 to 2048 tokens each,
 *                at most ceil(L / 512) of them).
 *   workspace    device scratch of pkv_decode_workspace_bytes(num_seqs, num_heads,
 *                head_dim, max_blocks_per_seq * block_size, partition_size) bytes,
 *                16-byte aligned; contents need no initialisation and are garbage
 *                afterwards.  Calls that may overlap on the GPU need separate workspaces.
 *
 * Launches, in this order on `stream`: a one-CTA planning kernel (work list),
 * the persistent decode kernel and, when a context can span more than one
 * partition, the partition merge kernel, all with programmatic dependent
 * launch.  The planning kernel may become resident while the work queued before
 * it finishes (when that work lets dependents launch early) and waits for it to
 * complete before anything else runs.  The merge kernel starts while the decode
 * grid drains and merges each (sequence, kv head) as soon as the decode grid
 * has published all of its partitions; it completes after the decode grid, so
 * work that follows on the stream sees the whole of `out`.
 */
pkv_status pkv_paged_attention_decode(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* context_lens, int32_t num_seqs,
                                      int32_t max_blocks_per_seq, int32_t num_blocks, float scale,
                                      int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, pkv_dtype dtype, int32_t partition_size,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/*
 * Allocation-free variant of pkv_paged_attention_decode.  The pages describe no
 * counterpart; it exists for callers that cannot allocate device memory when
 * they run decode (an engine that fixes its whole device-memory plan up front,
 * a plugin hook that must not allocate, code whose allocator belongs to someone
 * else), so it takes no workspace argument.
 *
 * Its scratch is one array of PKV_STATIC_WORKSPACE_BYTES inside the library's
 * device memory, held by every GPU that loads the library until the process
 * exits.  The call allocates and frees nothing.  Limits and behaviour:
 *  - Shapes whose workspace (pkv_decode_workspace_bytes with max_context_len =
 *    max_blocks_per_seq * block_size) exceeds PKV_STATIC_WORKSPACE_BYTES return
 *    PKV_EUNSUPPORTED and launch nothing; use pkv_paged_attention_decode then.
 *  - The first call on a device that needs scratch looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current); make that first
 *    call before any stream capture.
 *  - All calls share the one array per device: calls that may overlap on the GPU
 *    (different streams, no ordering between them) race on it.  Calls ordered on
 *    one stream are fine.  The array keeps the last call's contents; nothing in it
 *    needs to start at zero.
 * Arguments, results and errors are otherwise those of pkv_paged_attention_decode.
 */
#define PKV_STATIC_WORKSPACE_BYTES (16u << 20)

pkv_status pkv_paged_attention_decode_static(void* out, const void* q, const void* k_cache,
                                             const void* v_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, int32_t num_seqs,
                                             int32_t max_blocks_per_seq, int32_t num_blocks,
                                             float scale, int32_t num_heads, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t block_size, pkv_dtype dtype,
                                             int32_t partition_size, cudaStream_t stream);

/*
 * The same attention over a contiguous cache, one max-length reservation per
 * sequence (the layout of slides 6-7 and the dataarena note section 1 that
 * paging replaces).  Kept as the measurement baseline for the cost of the
 * indirection (slide 19: "a 20-26 % slower kernel").
 *
 *   k, v   device [num_seqs, num_kv_heads, max_context_len, head_dim] dtype
 *   context_lens device int32 [num_seqs], 0 <= context_lens[s] <= max_context_len
 *   workspace: pkv_decode_workspace_bytes(num_seqs, num_heads, head_dim,
 *   max_context_len, partition_size) bytes.  Other arguments as above.
 */
pkv_status pkv_contiguous_attention_decode(void* out, const void* q, const void* k, const void* v,
                                           const int32_t* context_lens, int32_t num_seqs,
                                           int32_t max_context_len, float scale, int32_t num_heads,
                                           int32_t num_kv_heads, int32_t head_dim, pkv_dtype dtype,
                                           int32_t partition_size, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream);

/*
 * Paged prefill attention (slide 3: the prompt is processed in parallel before
 * decoding; dataarena note section 4, step 3: a scheduled request runs its
 * prefill; slides 9-10: attention block by block through the block table).
 *
 * Sequence s brings T_s = query_start[s+1] - query_start[s] new tokens at
 * positions p0_s .. p0_s + T_s - 1, p0_s = context_lens[s] - T_s (p0 = 0: a
 * whole prompt; p0 > 0: a later chunk of one).  Their keys and values are
 * already in the cache (written with pkv_reshape_and_cache).  New token i of
 * sequence s, query head h (kv head g = h / (num_heads/num_kv_heads)):
 *   out[query_start[s] + i, h, :] =
 *       sum_{t <= p0_s + i} softmax_t(scale * q[query_start[s] + i, h, :] . K_s[t,:]) V_s[t,:]
 * with K_s, V_s gathered through the block table as in the decode (causal:
 * each new token sees the cached context and the new tokens up to itself).
 * Runs on the tensor cores with fp32 accumulation; the softmax weights enter the
 * PV product rounded to `dtype` and the normaliser sums those rounded weights,
 * so each output row is an exact convex combination of V rows up to fp32
 * rounding; out is rounded to `dtype`.  Max-abs error against exact arithmetic
 * stays within 2e-3 (fp16) / 1e-2 (bf16) for inputs of unit scale.
 *
 *   out, q       device [total_query_tokens, num_heads, head_dim] dtype (rows of
 *                sequence s at query_start[s] ..); rows outside every chunk are
 *                not written
 *   query_start  device int32 [num_seqs + 1], non-decreasing, within
 *                [0, total_query_tokens]; every T_s <= max_query_len
 *   context_lens device int32 [num_seqs], T_s <= context_lens[s] <= max_blocks_per_seq * block_size
 *   block_tables, k_cache, v_cache, num_blocks, block_size as in the decode; the
 *                first ceil(context_lens[s] / block_size) entries of row s are used
 *   max_query_len host int, the longest chunk (sets the grid)
 * Supported: head_dim 64 or 128, block_size 8, 16 or 32, any num_heads that is a
 * multiple of num_kv_heads (up to 65535 heads and 65535 sequences).  Allocates
 * nothing and needs no workspace.  A chunk that does not fit (longer than
 * max_query_len or than the table, outside the query rows) is skipped and
 * a context length below T_s or above the table's capacity is clamped; both set
 * PKV_DEVERR_CONTEXT_LEN.  One kernel launch on `stream`.
 */
pkv_status pkv_paged_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* query_start,
                             const int32_t* context_lens, int32_t num_seqs, int32_t max_query_len,
                             int32_t total_query_tokens, int32_t max_blocks_per_seq,
                             int32_t num_blocks, float scale, int32_t num_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                             pkv_dtype dtype, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Cache write and copy-on-write block copy                                 */
/* ------------------------------------------------------------------------ */

/*
 * Cache write (slide 11 "New block only when the last fills": each new token's
 * key and value go into the slot the allocator reserved for it).
 * For every token i with slot = slot_mapping[i] >= 0 and every kv head g:
 *   k_cache[slot / B, g, slot mod B, :] = key[i, g, :]   (and v_cache / value)
 * A negative slot is padding and is skipped.  Byte copies: bit-exact.
 *
 *   key, value   device [num_tokens, num_kv_heads, head_dim] dtype
 *   k_cache, v_cache device [num_blocks, num_kv_heads, block_size, head_dim] dtype, updated
 *   slot_mapping device int64 [num_tokens]; slots must be distinct (two tokens
 *                writing one slot race).  A slot >= num_blocks * block_size is
 *                not written and sets PKV_DEVERR_SLOT.
 *   head_dim * element size must be 16 bytes times a power of two (head_dim 8,
 *   16, 32, 64, 128, 256 for 16-bit types); other head_dim: PKV_EUNSUPPORTED.
 * The kernel lets a kernel queued behind it with programmatic dependent launch
 * become resident at once; such a kernel must wait for this grid in-kernel
 * before it reads the caches (the decode call's planning kernel does).  The
 * block copy below does the same.
 */
pkv_status pkv_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                                 const int64_t* slot_mapping, int32_t num_tokens,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t num_blocks, pkv_dtype dtype, cudaStream_t stream);

/*
 * Copy-on-write block copy (slide 13 "Parallel samples: copy on write ... only
 * the last block is ever copied"; dataarena note section 3.2).
 * For each pair i: frame dst of k_cache and of v_cache becomes a copy of frame src.
 *
 *   src_dst_pairs device int64 [num_pairs, 2] = (src, dst) frame indices.  All
 *                pairs run concurrently: destinations must be distinct and no
 *                destination may be the source of another pair (the allocator's
 *                copy lists satisfy this); otherwise the result depends on the
 *                order the pairs happen to run in (PKV_VALIDATE=1 rejects such a
 *                list with PKV_EINVAL).  src == dst is a no-op.  A frame index
 *                outside [0, num_blocks) skips the pair and sets PKV_DEVERR_COPY_PAIR.
 *   block_bytes  bytes of one frame of one cache = num_kv_heads * block_size *
 *                head_dim * element size; a multiple of 16.
 */
pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs,
                           int32_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                           cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Host block allocator                                                     */
/* ------------------------------------------------------------------------ */
/*
 * Refcounted block allocator (slides 10-14; dataarena note sections 2, 3.1,
 * 3.2 and 4 step 2).  Host memory only; one handle per pool; not thread-safe.
 *  - Free frames form a FIFO queue, initially frame_order[0..N-1] (NULL = 0..N-1).
 *    A sequence takes frames from the head; a frame whose count drops to 0 goes
 *    to the tail.
 *  - A prompt of n tokens takes ceil(n / B) frames (all-or-nothing: PKV_ENOMEM and
 *    no change when the pool has fewer free frames).
 *  - Appending token t writes into the last block when it has room (t mod B != 0)
 *    and its count is 1; when it has room but is shared (count > 1), the writer
 *    gets a new frame and a copy pair (shared frame, new frame) is emitted for
 *    pkv_copy_blocks, to run before the cache write.  When t mod B == 0 a new
 *    frame is taken and nothing is copied.
 *  - fork() shares every frame of the parent (counts + 1); free() drops the counts.
 *  - slot = frame * B + t mod B.
 */
typedef struct pkv_allocator pkv_allocator;

typedef struct {
  int64_t used_blocks;    /* frames with count > 0 */
  int64_t free_blocks;    /* frames in the free queue */
  int64_t tokens;         /* sum of the live sequences' lengths */
  int64_t shared_blocks;  /* frames with count > 1 */
  int64_t logical_blocks; /* sum of the live sequences' table lengths */
  int64_t cached_blocks;  /* frames holding a prefix-cache key (in use or free) */
} pkv_alloc_stats_t;

pkv_status pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* frame_order,
                            pkv_allocator** out);
void pkv_alloc_destroy(pkv_allocator* alloc);
/* New sequence with prompt_len tokens; slots_out (host int64 [prompt_len], may be
 * NULL) receives the slot of every prompt token. */
pkv_status pkv_alloc_add_seq(pkv_allocator* alloc, int32_t seq_id, int32_t prompt_len,
                             int64_t* slots_out);
/*
 * Automatic prefix caching (dataarena note section 3.1: a hash of each prompt
 * block; a request whose block hash already has a frame maps its logical block
 * to that frame and increments its reference count: no KV is recomputed).
 * Like pkv_alloc_add_seq for a prompt of token_ids[0..prompt_len-1], except that
 * each full block j gets the key pkv_block_hash(key of block j-1, or NULL for
 * j = 0, its B token ids).  The leading blocks whose keys are cached reuse their
 * frames (count + 1; a cached frame that was free leaves the free queue); the
 * rest take fresh frames from the free queue, and their full blocks enter the
 * cache.  *cached_tokens_out = B x the reused blocks: the caller writes K/V only
 * for tokens from there on.  A cached frame keeps its key while it sits free
 * and loses it when taken for other content.  All-or-nothing on PKV_ENOMEM.
 */
pkv_status pkv_alloc_add_seq_cached(pkv_allocator* alloc, int32_t seq_id, const int32_t* token_ids,
                                    int32_t prompt_len, int64_t* slots_out,
                                    int32_t* cached_tokens_out);
/* The prefix-cache key of a block: SHA-256 (FIPS 180-4) of the 32-byte parent
 * key (32 zero bytes when parent_key is NULL) followed by token_ids[0..n-1] as
 * little-endian int32; 32 bytes into key_out. */
pkv_status pkv_block_hash(const uint8_t* parent_key, const int32_t* token_ids, int32_t n,
                          uint8_t* key_out);
/* child shares all of parent's frames (parallel sampling, beam search). */
pkv_status pkv_alloc_fork(pkv_allocator* alloc, int32_t parent, int32_t child);
/* Reserve the slot of the next token of seq_id; *cow_src/*cow_dst = -1 unless a
 * copy is needed. */
pkv_status pkv_alloc_append(pkv_allocator* alloc, int32_t seq_id, int64_t* slot_out,
                            int32_t* cow_src, int32_t* cow_dst);
/* One decode step: append one token to each of seq_ids[0..n-1] (distinct), in
 * order.  slots_out: host int64 [n]; pairs_out: host int64 [n, 2] receives the
 * copy pairs, *num_pairs_out their count.  All-or-nothing on PKV_ENOMEM. */
pkv_status pkv_alloc_append_batch(pkv_allocator* alloc, const int32_t* seq_ids, int32_t n,
                                  int64_t* slots_out, int64_t* pairs_out, int32_t* num_pairs_out);
pkv_status pkv_alloc_free_seq(pkv_allocator* alloc, int32_t seq_id);
/*
 * One beam-search step over a block tree (slides 13-14 "Beam search: a block
 * tree, not copies": candidates share their prefix like forked processes;
 * kashii section 3: copy on write when their tokens diverge).
 *   beams[0..k-1]       the live beams' sequence ids (distinct)
 *   parents[0..k_new-1] new beam j continues beam parents[j] (index into beams)
 *   *next_id            first id for extra continuations; advanced past the ids used
 *   new_ids_out[k_new]  sequence id of each new beam: a parent's first continuation
 *                       keeps the parent's id, every further one is a fork with a
 *                       fresh id (all of the parent's frames shared, counts + 1)
 *   slots_out[k_new]    slot of the token appended to each new beam
 *   pairs_out[k_new, 2] copy pairs (shared frame, private frame), *num_pairs_out
 * Order: the forks (in new-beam order), then the frees of the beams without a
 * continuation (in beam order; their frames go to the tail of the free queue),
 * then one append per new beam in order, with the copy-on-write rule of
 * pkv_alloc_append.  All-or-nothing: PKV_ENOMEM (nothing changed) when the step
 * needs more frames than are free after the frees; PKV_EINVAL for unknown or
 * repeated beams, a parent index outside [0, k), or a fresh id already in use.
 */
pkv_status pkv_alloc_beam_step(pkv_allocator* alloc, const int32_t* beams, int32_t k,
                               const int32_t* parents, int32_t k_new, int32_t* next_id,
                               int32_t* new_ids_out, int64_t* slots_out, int64_t* pairs_out,
                               int32_t* num_pairs_out);
/* Block tables of seq_ids as host int32 [n, max_blocks] padded with -1, and
 * their lengths (lens_out may be NULL).  PKV_ERANGE if a table is longer than
 * max_blocks. */
pkv_status pkv_alloc_block_table(const pkv_allocator* alloc, const int32_t* seq_ids, int32_t n,
                                 int32_t max_blocks, int32_t* table_out, int32_t* lens_out);
pkv_status pkv_alloc_refcount(const pkv_allocator* alloc, int32_t block, int32_t* count_out);
pkv_status pkv_alloc_stats(const pkv_allocator* alloc, pkv_alloc_stats_t* out);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */

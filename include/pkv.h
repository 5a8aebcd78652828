/*
 * pkv.h -- C ABI of libpkv: paged KV-cache decode attention on one NVIDIA B200
 * (sm_100a), plus the host block allocator that owns the block tables.
 *
 * The operations follow three web pages on paged KV caches:
 *   [P1] "PagedAttention 与在线推理：KV 分页、共享及调度的联合分析"
 *   [P2] "PagedAttention：让 KV cache 按需生长"
 *   [P3] "内存预算约束下的语言模型服务：注意力、分页与调度"
 * Each declaration names the page and section that defines what it computes.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Return value: PKV_OK (0) or one of the PKV_ERR_* codes below.  No C++
 *   exception crosses this boundary.
 * - Device pointers are owned by the caller (e.g. allocated by PyTorch) and are
 *   never freed or retained by the library.  Host pointers are only read or
 *   written during the call.
 * - Device calls are asynchronous on the given stream (a cudaStream_t passed
 *   as void*; NULL is the legacy default stream) and return after the launch.
 *   Argument checks happen on the host before any launch; a call that returns
 *   PKV_ERR_INVALID has launched nothing.  PKV_ERR_CUDA means a launch or
 *   driver call failed; the CUDA error string is available from
 *   pkv_last_cuda_error().
 * - Storage types: PKV_BF16 (bfloat16 bit patterns, 2 bytes) or PKV_F32.
 * - KV pool layout (one K pool and one V pool per layer), the teaching layout
 *   of [P2] section "把 token 6 变成真正的内存地址":
 *       pool[num_blocks][block_size][num_kv_heads][head_dim], contiguous.
 *   Token t of a request lives in logical block t / B at offset t % B; its
 *   "slot" is block_table[t / B] * B + t % B, the row of the pool viewed as
 *   [num_blocks * B][num_kv_heads][head_dim] ([P2] sections
 *   "顺序留在表里，数据放进空闲块" and "读 token 6，先查表，再找偏移").
 * - Block tables: int32 [num_seqs][max_blocks_per_seq], row s holds the
 *   physical ids of request s in logical order; entries past
 *   ceil(seq_lens[s] / B) are never read.
 * - Supported decode shapes: bf16 head_dim 64, 128 or 256; f32 head_dim 64
 *   or 128; block_size 4, 8, 16, 32, 64, 128 or 256; num_q_heads a multiple
 *   of num_kv_heads (< 4096) with group G = num_q_heads / num_kv_heads in
 *   {1, 2, 4, 8, 16}.  kv_append and block_copy take any power-of-two block
 *   size and any row of a multiple of 16 bytes.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes -------------------------------------------------------- */
#define PKV_OK 0
#define PKV_ERR_NO_BLOCKS 1      /* allocate-or-fail: not enough free blocks      */
#define PKV_ERR_INVALID 2        /* bad argument, shape, id or range              */
#define PKV_ERR_CUDA 3           /* a CUDA launch or driver call failed           */
#define PKV_ERR_DEVICE_TIMEOUT 4 /* a bounded device-side wait ran out            */
#define PKV_ERR_BAD_TABLE 5      /* a block-table entry was outside [0, blocks)   */
#define PKV_ERR_PLAN_MISMATCH 6  /* run() with a plan made for other sizes        */

/* storage types */
#define PKV_BF16 0
#define PKV_F32 1

typedef void* pkv_stream_t; /* a cudaStream_t */

/* Library version string, e.g. "pkv 0.1.0 sm_100a". */
const char* pkv_version(void);
/* Human-readable name of a status code. */
const char* pkv_status_string(int status);
/* Text of the last CUDA error seen by this thread (empty if none). */
const char* pkv_last_cuda_error(void);

/* ==========================================================================
 * Decode attention
 * ==========================================================================
 * What it computes ([P2] section "分页以后，attention 仍然按完整历史归一化";
 * [P3] section 6 and equation (4)): for every request s and query head h,
 *     out[s][h] = sum_t softmax_t(scale * <q[s][h], K_t>) V_t,
 * over the request's tokens t < seq_lens[s], where K_t, V_t are the rows of
 * KV head h / G found through the block table.  Slots at or past seq_lens[s]
 * are masked to -inf and never read into a sum (they may hold any bits,
 * NaN included).  seq_lens[s] == 0 gives out[s] = 0.  The result equals dense
 * attention over the contiguous history up to floating-point rounding: the
 * kernels accumulate in fp32 (products of bf16 inputs are exact in fp32).
 *
 * How: one persistent kernel launch of one-warp CTAs (8 per SM; 4 for
 * 512-byte rows).  All (request, KV head, 16-token tile) units are split into
 * equal contiguous ranges, one per CTA; the CTA keeps an online-softmax state
 * (m, l, o) for the grouped query heads of its current KV head and reads each
 * K/V tile once for the whole group through a TMA-fed shared-memory ring.  A
 * (request, KV head) split across CTAs is finished by the last CTA to reach
 * it, which merges the partial states
 * ([P2] exercise "逻辑顺序没错，为什么 attention 输出还是错？": the states merge,
 * per-block outputs do not).  With 16 grouped columns (G = 16, or several
 * query tokens whose columns make 16), and with 8 in a launch that is not
 * plain single-token decode (several query tokens, query heads padded to the
 * column group, or a log-sum-exp output), the pieces are merged instead by a
 * second, short launch behind the first: one warp per (request, KV head,
 * column).
 *
 * Arguments (all device pointers unless stated):
 *   q             [num_seqs][num_q_heads][head_dim], kv_dtype
 *   k_pool,v_pool [num_blocks][block_size][num_kv_heads][head_dim], kv_dtype;
 *                 16-byte aligned
 *   block_tables  int32 [num_seqs][max_blocks_per_seq]
 *   seq_lens      int32 [num_seqs], 0 <= seq_lens[s] <= max_blocks_per_seq*B
 *   scale         softmax scale (usually 1/sqrt(head_dim)), host value
 *   out           [num_seqs][num_q_heads][head_dim], out_dtype (PKV_BF16 rounds
 *                 the fp32 result to nearest even, PKV_F32 stores it)
 *   workspace     caller-owned scratch of at least
 *                 pkv_decode_workspace_bytes(...) bytes, 256-byte aligned; it
 *                 holds the plan, partial states and a device status word.
 *                 Calls that share a workspace must be ordered on one stream.
 * Errors: PKV_ERR_INVALID for unsupported shapes, null or misaligned pointers,
 * or a workspace that is too small.  Device-detected faults (a block-table
 * entry outside [0, num_blocks), a bounded wait that ran out) do not stop the
 * launch: the affected tile reads zeros, and the fault is recorded in the
 * workspace status word, read back by pkv_decode_status().
 */
size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim);

int pkv_paged_decode_attn(const void* q, const void* k_pool, const void* v_pool,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                          int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                          int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                          int32_t out_dtype, void* workspace, size_t workspace_bytes,
                          pkv_stream_t stream);

/* The two halves of pkv_paged_decode_attn, for a decode step that runs many
 * layers over the same seq_lens: plan once, then run once per layer.
 * pkv_decode_plan reads seq_lens on the device and writes the work partition
 * into the workspace.  pkv_paged_decode_attn_run uses it; the plan must have
 * been made with the same num_seqs, num_q_heads, num_kv_heads, head_dim and
 * kv_dtype on the same seq_lens contents (a mismatch in the sizes is caught on
 * the device and reported as PKV_ERR_PLAN_MISMATCH by pkv_decode_status()). */
int pkv_decode_plan(const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t kv_dtype, void* workspace,
                    size_t workspace_bytes, pkv_stream_t stream);

int pkv_paged_decode_attn_run(const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* block_tables, int32_t max_blocks_per_seq,
                              const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                              int32_t out_dtype, void* workspace, size_t workspace_bytes,
                              pkv_stream_t stream);

/* pkv_kv_append folded into pkv_paged_decode_attn_run: one launch writes each
 * request's new token into the pools and attends over the history including
 * it ([P2] section "写满一块，再拿下一块" for the write, section
 * "分页以后，attention 仍然按完整历史归一化" for the attention).
 *   k_new, v_new  [num_seqs][num_kv_heads][head_dim], kv_dtype: row s is the
 *                 new token of request s, which must be the LAST token of its
 *                 history (position seq_lens[s] - 1, already counted)
 *   slot_mapping  int64 [num_seqs]: the pool slot of that position (as
 *                 pkv_slot_mapping gives it); < 0 means request s has no new
 *                 token in this call; >= num_blocks * block_size is flagged
 *                 (PKV_ERR_BAD_TABLE) and not written
 * The result equals pkv_kv_append(k_new, v_new, slot_mapping, num_seqs, ...)
 * followed by pkv_paged_decode_attn_run(...): the warp that owns a request's
 * last tile writes the new K/V row to the pool and over the tile row it just
 * loaded.  Needs a plan in the workspace (pkv_decode_plan);
 * num_blocks * block_size must be below 2^31. */
int pkv_paged_decode_attn_append_run(const void* q, const void* k_new, const void* v_new,
                                     const int64_t* slot_mapping, void* k_pool, void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                     int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                                     int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream);

/* Allocation-free variant of pkv_paged_decode_attn (the pages have no
 * counterpart: this is a deployment convenience).  For callers that cannot
 * allocate device memory -- e.g. a plugin called by a runtime that owns all
 * device allocations and passes only inputs and outputs, or a serving loop
 * that must never call cudaMalloc -- the scratch lives in a 16 MiB array
 * built into the library (held on every GPU that loads it, until exit).
 * Arguments are those of pkv_paged_decode_attn without the workspace.
 * - Batches whose pkv_decode_workspace_bytes() exceeds 16 MiB are refused
 *   with PKV_ERR_INVALID (pkv_last_cuda_error() says why); nothing runs.
 * - The first call on each device (and the first after a cudaDeviceReset,
 *   which creates a new context) looks up the array's device address; make
 *   that first call before any stream capture.
 * - No call allocates: no cudaMalloc/cudaFree, no allocating library routine.
 * - All calls share the one array per device: calls that overlap on the GPU
 *   (different streams without ordering) race and give wrong results.  Each
 *   call clears the status word it uses; device-detected faults are not
 *   reported back (use the workspace form when they must be). */
int pkv_paged_decode_attn_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                                  int32_t out_dtype, pkv_stream_t stream);

/* Multi-token query: T = num_q_tokens new tokens per request attend at once
 * (the verification pass of speculative decoding, or a chunk of a prefill),
 * each under the causal mask inside the last blocks ([P1] section 5: the
 * staged KV positions of speculative decoding; [P3] section 6 and equation
 * (4) for each token's attention).  The T tokens are the last T positions of
 * the history: their K/V must already be in the pools and counted in
 * seq_lens.  Query token i (0 <= i < T) of request s sits at position
 * p = seq_lens[s] - T + i and attends positions 0..p:
 *     out[s][i][h] = sum_{t <= p} softmax_t(scale * <q[s][i][h], K_t>) V_t.
 * A token with p < 0 (seq_lens[s] < T - i) attends nothing and gets 0.
 * T = 1 is pkv_paged_decode_attn.
 *   q, out      [num_seqs][num_q_tokens][num_q_heads][head_dim]
 *   num_q_tokens 1..16 with G * num_q_tokens <= 16 (G = num_q_heads /
 *               num_kv_heads): the (query token, grouped head) pairs of a KV
 *               head share each K/V tile read
 *   workspace   at least pkv_multi_query_workspace_bytes(...) bytes
 * Other arguments, layouts and errors as pkv_paged_decode_attn (plans and
 * runs in one call); pkv_multi_query_workspace_bytes returns 0 for an
 * unsupported shape. */
size_t pkv_multi_query_workspace_bytes(int32_t num_seqs, int32_t num_q_tokens, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim);
int pkv_paged_attn_multi_query(const void* q, int32_t num_q_tokens, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, float scale, int32_t kv_dtype, void* out,
                               int32_t out_dtype, void* workspace, size_t workspace_bytes,
                               pkv_stream_t stream);

/* Shared-prefix decode attention: the same result as pkv_paged_decode_attn
 * for requests forked from common prompts, reading each shared block once
 * per group instead of once per request.  Forked requests share the full
 * blocks of their prompt by reference ([P2] section "只读时共用，要写入时再分开");
 * attention still covers each request's whole history ([P2] section
 * "分页以后，attention 仍然按完整历史归一化"), split into the shared part and
 * the request's own part, whose online-softmax states merge exactly ([P2]
 * exercise "逻辑顺序没错，为什么 attention 输出还是错？").
 *   group_start   DEVICE int32 [num_groups + 1]: group g is the requests
 *                 group_start[g] .. group_start[g+1]-1 (consecutive rows);
 *                 group_start[0] = 0, group_start[num_groups] = num_seqs;
 *                 every request is in exactly one group (a group of one with
 *                 no shared blocks is plain decode)
 *   prefix_blocks DEVICE int32 [num_groups]: the first prefix_blocks[g]
 *                 entries of every member's table row are the same full
 *                 blocks; every member's length is at least
 *                 prefix_blocks[g] * block_size
 *   max_group     largest group size, 1..16, with G * max_group <= 16
 *                 (G = num_q_heads / num_kv_heads)
 *   workspace     at least pkv_shared_prefix_workspace_bytes(...) bytes,
 *                 256-byte aligned; pkv_decode_status(workspace) reports
 *                 device-detected faults, including members whose table rows
 *                 differ inside the shared part or groups that break the
 *                 rules above (PKV_ERR_BAD_TABLE: the output is then not
 *                 meaningful)
 * Other arguments as pkv_paged_decode_attn.  A 4-byte memset and four
 * launches: the preparation (gather of the grouped queries and tables, and
 * both plans), the own-part pass (scheduled during the preparation, waiting
 * for it at its start), the shared-part pass (the members' queries
 * are the columns of one launch; it starts during the own-part pass's tail)
 * and the combine (started during the shared-part pass's tail), which also
 * merges the shared-part pass's split pieces when that pass has 8 or 16
 * columns per KV head.  With 8 grouped query heads per KV head the own-part
 * pass (which writes a log-sum-exp) is followed by its merge launch: five
 * launches. */
size_t pkv_shared_prefix_workspace_bytes(int32_t num_seqs, int32_t num_groups, int32_t max_group,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t max_blocks_per_seq);
int pkv_paged_decode_attn_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* seq_lens, int32_t num_seqs, const int32_t* group_start,
                                        const int32_t* prefix_blocks, int32_t num_groups, int32_t max_group,
                                        int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                        int32_t block_size, int32_t num_blocks, float scale, int32_t kv_dtype,
                                        void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                        pkv_stream_t stream);

/* Synchronises `stream`, reads the workspace status word, clears it and
 * returns PKV_OK, PKV_ERR_BAD_TABLE, PKV_ERR_DEVICE_TIMEOUT or
 * PKV_ERR_PLAN_MISMATCH (the first recorded), or PKV_ERR_CUDA. */
int pkv_decode_status(void* workspace, pkv_stream_t stream);

/* Failure-detection self-test (not a paper operation): launches one warp
 * that waits on an mbarrier nothing arrives on, through the same bounded wait
 * the decode kernel uses, for limit_ns nanoseconds (1 .. 1e8); the expiry is
 * recorded in the workspace status word, so a following pkv_decode_status()
 * returns PKV_ERR_DEVICE_TIMEOUT.  Nothing faults or hangs: the kernel ends
 * after the limit and the context stays usable. */
int pkv_selftest_bounded_wait(unsigned long long limit_ns, void* workspace, size_t workspace_bytes,
                              pkv_stream_t stream);

/* Selects the tile kernel for bf16 storage: 0 = automatic (default),
 * 1 = CUDA-core FMA tiles, 2 = tensor-core (mma.sync bf16) tiles.  fp32
 * storage always uses FMA tiles, and so do bf16 pools that the tensor-core
 * tiles do not cover (block size 4 at head_dim 64; 16 grouped columns at
 * head_dim 256); 0 and 2 pick the tensor-core tiles everywhere else.
 * Process-wide; for measurement. */
int pkv_set_decode_kernel(int32_t which);

/* Launch overlap (default 0 = off).  With 1, pkv_paged_decode_attn_run and
 * pkv_paged_decode_attn_append_run launch as programmatic dependent launches:
 * their CTAs may start while the kernel launched just before them on the
 * stream is still finishing, read the plan, block tables, lengths, slot
 * mapping and this call's K/V pool, and start their first K/V loads; they
 * wait for that kernel to complete (and its writes to be visible) before
 * reading q, k_new or v_new and before writing anything.  Set it only for
 * calls where the kernel launched immediately before does not write the
 * workspace plan, the block tables, seq_lens, the slot mapping or the K/V
 * pool the call reads: e.g. layers 2..L of one decode step, each reading its
 * own pool, but not the first layer right after pkv_decode_plan.  The calls
 * that plan themselves (pkv_paged_decode_attn, pkv_paged_attn_multi_query,
 * the allocation-free call) ignore this setting: their attention launch
 * follows their plan launch as a dependent launch that waits for the plan
 * before reading anything (only its start-up overlaps the plan's).
 * Process-wide; read at launch. */
int pkv_set_launch_overlap(int32_t on);

/* ==========================================================================
 * Cache writes
 * ==========================================================================
 * pkv_kv_append -- write the K and V of n_tokens new tokens into their slots
 * ([P2] section "写满一块，再拿下一块": the new token's K, V go into the tail
 * block; earlier blocks never move).
 *   k, v          [n_tokens][num_kv_heads][head_dim], dtype
 *   slot_mapping  int64 [n_tokens]; pool row = slot (see layout above).  A
 *                 negative slot (padding) or one >= num_blocks*block_size is
 *                 skipped.
 *   k_pool,v_pool one layer's pools
 * Same-stream ordering makes a preceding pkv_block_copy visible first, as the
 * allocate-copy-remap-write order of [P2] section
 * "先确保分配成功，再改变可见状态" requires.
 */
int pkv_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t n_tokens,
                  void* k_pool, void* v_pool, int32_t num_kv_heads, int32_t head_dim,
                  int32_t block_size, int32_t num_blocks, int32_t dtype, pkv_stream_t stream);

/* pkv_block_copy -- copy-on-write of shared partial tails ([P2] sections
 * "只读时共用，要写入时再分开" and "一次写入，为什么会先少掉一个空闲块？"):
 * for each copy i and every layer l,
 *     pool_l[dst_i][0 : n_valid_i] = pool_l[src_i][0 : n_valid_i]
 * in both the K and the V pool (block numbering is shared by all layers,
 * [P2] section "128 KiB：每新增一个位置的账单").
 *   k_pools,v_pools HOST arrays of num_layers device pool pointers
 *                   (1 <= num_layers <= 128)
 *   copies          DEVICE int32 [n_copies][3] = (src, dst, n_valid), the
 *                   layout pkv_alloc_append() produces; entries with an id
 *                   outside [0, num_blocks), src == dst, or n_valid outside
 *                   [0, block_size] are skipped.
 */
int pkv_block_copy(void* const* k_pools, void* const* v_pools, int32_t num_layers,
                   const int32_t* copies, int32_t n_copies, int32_t num_kv_heads,
                   int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                   pkv_stream_t stream);

/* pkv_swap_blocks -- preemption by swap ([P2] section
 * "腾出显存以后，还要付一次恢复成本": release a request's KV and move it over the
 * host link, then bring it back later, instead of recomputing it).  Moves
 * blocks[i] of every layer's K and V pool to (to_host = 1) or from
 * (to_host = 0) a host buffer laid out
 *     host_buf[n_blocks][num_layers][2 (K, V)][block_size][num_kv_heads][head_dim].
 *   k_pools,v_pools HOST arrays of num_layers device pool pointers (<= 128)
 *   blocks          DEVICE int32 [n_blocks]; ids outside [0, num_blocks) are
 *                   skipped.  Swapping back in may use other block ids (the
 *                   ones the allocator hands out on re-admission).
 *   host_buf        page-locked host memory the device can address
 *                   (cudaHostAlloc, or torch's pinned memory under unified
 *                   addressing), 16-byte aligned; the kernel reads or writes
 *                   it directly over the host link.
 * Asynchronous on `stream`; the host buffer is complete (to_host = 1) or
 * reusable (to_host = 0) once the stream reaches this point. */
int pkv_swap_blocks(void* const* k_pools, void* const* v_pools, int32_t num_layers,
                    const int32_t* blocks, int32_t n_blocks, void* host_buf, int32_t to_host,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                    int32_t dtype, pkv_stream_t stream);

/* pkv_slot_mapping -- slot of each (request row, position) through the block
 * table ([P2] sections "读 token 6，先查表，再找偏移" and
 * "把 token 6 变成真正的内存地址"):
 *     slots[i] = block_tables[rows[i]][positions[i] / B] * B + positions[i] % B
 *   rows       DEVICE int32 [n] or NULL (row i for position i)
 *   positions  DEVICE int32 [n]; a negative position gives slot -1
 *   slots      DEVICE int64 [n]
 */
int pkv_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* rows, const int32_t* positions, int32_t n,
                     int32_t block_size, int64_t* slots, pkv_stream_t stream);

/* ==========================================================================
 * Host block allocator
 * ==========================================================================
 * Integer metadata only: per request a block table, a length and a state;
 * per physical block a refcount (number of live requests holding it); a FIFO
 * free queue; optionally a cached set of released full blocks ([P2] section
 * "引用计数管理“谁还在读”，长度管理“哪里能写”").  Every call keeps
 *     active (refcount > 0) + cached + free == num_blocks
 * ([P2] section "占用率只有 70%，为什么请求还是进不来？").  Every call that returns
 * an error leaves the allocator exactly as it was, except pkv_alloc_append,
 * which is all-or-nothing per request (see there).  Not thread-safe: one
 * thread at a time per handle.  Handles are created and destroyed by the
 * library.
 */
typedef struct pkv_alloc pkv_alloc;

typedef struct pkv_stats {
  int64_t pool;           /* num_blocks                                   */
  int64_t active;         /* blocks with refcount > 0                     */
  int64_t cached;         /* refcount-0 full blocks kept for reuse        */
  int64_t free;           /* blocks in the free queue                     */
  int64_t seqs;           /* live requests                                */
  int64_t allocs;         /* blocks handed out                            */
  int64_t frees;          /* blocks whose refcount reached 0              */
  int64_t cow_copies;     /* copy-on-write copies issued                  */
  int64_t alloc_failures; /* requests refused for lack of blocks          */
  int64_t evictions;      /* cached blocks reallocated                    */
  int64_t prefix_hits;    /* blocks reused by pkv_alloc_add_seq_prefix    */
} pkv_stats;

/* initial_free_order: host int32 [num_blocks], a permutation of
 * 0..num_blocks-1 giving the free-queue order (NULL = 0, 1, 2, ...).
 * enable_cache != 0 keeps released full blocks in the cached set; they are
 * evicted oldest first, only when the free queue is empty.
 * Returns NULL on a bad argument or out of host memory. */
pkv_alloc* pkv_alloc_create(int32_t num_blocks, int32_t block_size,
                            const int32_t* initial_free_order, int32_t enable_cache);
void pkv_alloc_destroy(pkv_alloc* a);

/* Admit request seq_id (>= 0, not live) holding n_tokens of KV: takes
 * ceil(n_tokens / B) blocks from the head of the free queue, or returns
 * PKV_ERR_NO_BLOCKS and changes nothing ([P2] section
 * "24 GiB 的 KV 池，能同时容纳多少请求？"). */
int pkv_alloc_add_seq(pkv_alloc* a, int32_t seq_id, int32_t n_tokens);

/* child (>= 0, not live) shares every block of parent: same table and
 * length, refcount + 1 on each block ([P2] section "只读时共用，要写入时再分开"). */
int pkv_alloc_fork(pkv_alloc* a, int32_t parent, int32_t child);

/* Reserve the slot of one new token for each of the n requests, in the given
 * order ([P2] section "先确保分配成功，再改变可见状态"):
 *   length % B == 0 (no tail, or tail full)  -> take a free block, append it;
 *   tail shared (refcount > 1)                -> take a free block, emit the
 *       copy (tail, new, length % B), refcount[tail] - 1, remap the tail;
 *   otherwise                                 -> nothing to allocate;
 * then length + 1.  A request that cannot get its block is left exactly as
 * it was and its status is PKV_ERR_NO_BLOCKS; later requests still proceed
 * ([P2] section "三个空闲块，四个请求同时跨边界").
 *   seq_ids     host int32 [n], live and pairwise distinct, else
 *               PKV_ERR_INVALID with nothing changed
 *   status_out  host int32 [n] per-request status
 *   copies_out  host int32 [n][3] (src, dst, n_valid); *n_copies_out rows used
 * Returns PKV_OK if every request got its slot, else PKV_ERR_NO_BLOCKS. */
int pkv_alloc_append(pkv_alloc* a, const int32_t* seq_ids, int32_t n, int32_t* status_out,
                     int32_t* copies_out, int32_t* n_copies_out);

/* Finish, cancel or preempt: release the request's blocks in logical order;
 * a block whose refcount reaches 0 goes to the tail of the free queue (or to
 * the cached set if enabled and it holds B tokens) ([P2] section
 * "请求结束，块就能交给下一位"). */
int pkv_alloc_free_seq(pkv_alloc* a, int32_t seq_id);

/* Copy the block table of seq_id into out (host, capacity cap entries);
 * *len = number of blocks, *n_tokens = its length.  PKV_ERR_INVALID if the
 * request is not live or cap is too small. */
int pkv_alloc_get_table(const pkv_alloc* a, int32_t seq_id, int32_t* out, int32_t cap,
                        int32_t* len, int32_t* n_tokens);

/* Fill host tables_out [n][max_blocks_per_seq] (row i = request seq_ids[i],
 * unused entries = pad) and host seq_lens_out [n], ready to mirror to the
 * device.  PKV_ERR_INVALID if a request is not live or its table is longer
 * than max_blocks_per_seq (nothing written then). */
int pkv_alloc_fill_tables(const pkv_alloc* a, const int32_t* seq_ids, int32_t n,
                          int32_t* tables_out, int32_t max_blocks_per_seq, int32_t pad,
                          int32_t* seq_lens_out);

int pkv_alloc_stats(const pkv_alloc* a, pkv_stats* out);

/* Full consistency check: conservation, a refcount recount from the live
 * tables, table lengths, no block both idle and referenced.  PKV_OK or
 * PKV_ERR_INVALID. */
int pkv_alloc_check(const pkv_alloc* a);

/* Snapshot for tests: refcounts [num_blocks], the free queue and the cached
 * set in order (host arrays of capacity num_blocks; counts written to
 * *n_free, *n_cached).  Any pointer may be NULL to skip that part. */
int pkv_alloc_dump(const pkv_alloc* a, int32_t* refcounts, int32_t* free_order, int32_t* n_free,
                   int32_t* cached_order, int32_t* n_cached);

/* Prefix caching ([P2] sections "请求结束，块就能交给下一位" and
 * "引用计数管理“谁还在读”，长度管理“哪里能写”": a released full block keeps its
 * content until it is evicted; section "只读时共用，要写入时再分开": a full-block
 * hit is shared without a copy; [P3] section 8: the key must name every input
 * that shaped the state, so the caller computes it (e.g. a hash chained over
 * the model identity and the block's token ids) and the allocator stores it).
 *
 * pkv_alloc_set_block_key: name the content of full block `logical_block` of
 * live request seq_id with a 64-bit key.  A key names one block and a block
 * has one key; PKV_ERR_INVALID for a partial block, an unknown request, or a
 * key/block already bound elsewhere.  Keys are dropped when the block returns
 * to the free queue or is evicted from the cached set.
 *
 * pkv_alloc_add_seq_prefix: admit request seq_id holding n_tokens whose first
 * n_keys blocks are full blocks with the given keys (n_keys * B <= n_tokens).
 * Keys are matched in order up to the first miss: a hit on a live block adds
 * a reference, a hit on a cached block moves it back to active; the remaining
 * ceil(n_tokens / B) - hits blocks come from the free queue (then the cached
 * set).  All or nothing: PKV_ERR_NO_BLOCKS leaves everything unchanged.
 * *n_hit receives the number of reused blocks (their KV need not be
 * recomputed). */
int pkv_alloc_set_block_key(pkv_alloc* a, int32_t seq_id, int32_t logical_block, uint64_t key);
int pkv_alloc_add_seq_prefix(pkv_alloc* a, int32_t seq_id, int32_t n_tokens, const uint64_t* keys,
                             int32_t n_keys, int32_t* n_hit);

/* Host-side fault injection for failure tests (no device involvement):
 *   PKV_FAULT_ALLOC_FAIL    the next `count` block allocations fail as if
 *                           the pool were empty;
 *   PKV_FAULT_SKIP_RELEASE  the next `count` pkv_alloc_free_seq calls drop the
 *                           request without releasing its references (a leak
 *                           that pkv_alloc_check reports);
 *   PKV_FAULT_NONE          clears pending faults. */
#define PKV_FAULT_NONE 0
#define PKV_FAULT_ALLOC_FAIL 1
#define PKV_FAULT_SKIP_RELEASE 2
int pkv_alloc_inject_fault(pkv_alloc* a, int32_t kind, int32_t count);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */

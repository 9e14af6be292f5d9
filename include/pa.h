/*
 * pa.h — C ABI of libpa, the paged KV-cache decode hot path for NVIDIA B200
 * (sm_100a).
 *
 * The method (PagedAttention): each sequence's keys and values live in
 * fixed-size physical blocks of `block_size` tokens scattered through one
 * shared pool and are reached only through a per-sequence block table and a
 * sequence length ("PagedAttention 与 KV 显存管理" study notes ch.05 §3; vLLM
 * blog "vLLM 是什么" §2).  Attention over those blocks is merged across
 * blocks with online softmax (study notes §4); new tokens are stored into
 * their slots (vLLM blog, plain-language section); blocks shared by several outputs are copied
 * before a write (copy on write, study notes §6.1 and §12 exercise 4).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers to caller-owned memory on the
 *   current CUDA device; the library allocates and frees nothing.
 * - Dense row-major layouts, no strides:
 *     k_pool, v_pool : [num_blocks][num_kv_heads][block_size][head_dim]
 *     q, out         : [num_seqs][num_q_heads][head_dim]
 *     k, v (new)     : [num_tokens][num_kv_heads][head_dim]
 *   Element type fp16 or bf16 (pa_pool_desc.dtype) for q, out, k, v and the
 *   pools alike.  Every tensor pointer must be 16-byte aligned.
 * - Token t of a sequence is row (t % block_size) of physical block
 *   block_tables[s][t / block_size]; a slot is  block * block_size + row.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call only enqueues work and returns; results and the
 *   device status are valid after the stream is synchronised.
 * - The return value reports what the host can see (bad arguments,
 *   unsupported shapes, a failed launch).  Errors that depend on device data
 *   (a block id or slot out of range, a wait that ran out) are written to
 *   `*dev_status` (int32, device memory, nullable): the first error wins via
 *   compare-and-swap from PA_DEV_OK, the kernel skips the offending access
 *   and carries on or returns; it never traps.  Outputs are unspecified
 *   after a non-zero device status.  With dev_status == NULL such errors
 *   are still skipped but not reported.
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

/* Host-side return codes. */
typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1, /* null or misaligned pointer, negative or zero size */
  PA_ERR_UNSUPPORTED = 2, /* no kernel for this block_size/head_dim/group/dtype */
  PA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  PA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  PA_ERR_SCRATCH_LIMIT = 5, /* pa_decode_no_alloc: the batch needs more scratch than its fixed array */
  PA_ERR_OUT_OF_BLOCKS = 6  /* block manager: not enough free blocks (nothing was changed) */
} pa_status;

/* Device-side status codes written to *dev_status (a range of their own,
 * so pa_status_string names either kind). */
#define PA_DEV_OK 0
#define PA_DEV_BAD_BLOCK_ID 101 /* a block_tables entry outside [0, num_blocks) */
#define PA_DEV_BAD_SEQ_LEN 102 /* seq_lens[s] < 0 or > max_blocks_per_seq * block_size */
#define PA_DEV_BAD_SLOT 103    /* slot_mapping entry >= num_blocks * block_size */
#define PA_DEV_BAD_PAIR 104    /* copy pair with src or dst outside [0, num_blocks) */
#define PA_DEV_TIMEOUT 105     /* a bounded pipeline wait ran out (kernel returned early) */
#define PA_DEV_BAD_GROUP 106   /* shared-prefix groups do not partition the sequences, or one is too large */

typedef enum pa_dtype { PA_FP16 = 0, PA_BF16 = 1 } pa_dtype;

/* Shape of the physical block pool (the same for the K and the V pool). */
typedef struct pa_pool_desc {
  int32_t num_blocks;   /* physical blocks in each pool */
  int32_t block_size;   /* tokens per block: 8, 16 or 32 */
  int32_t num_kv_heads; /* key/value heads */
  int32_t head_dim;     /* 64 or 128 */
  int32_t dtype;        /* pa_dtype */
} pa_pool_desc;

/* Tuning/test options for pa_decode_ex; zero-initialise for the defaults. */
typedef struct pa_decode_opts {
  int32_t num_ctas; /* persistent CTAs; 0 = SM count x resident CTAs per SM */
  int32_t flags;    /* 0, or PA_DECODE_CUDA_CORES_ONLY and/or a PA_DECODE_TEST_* hook */
} pa_decode_opts;

/* Failure-detection test hook for pa_decode_opts.flags: the producer warps
 * issue no copies, every consumer wait runs out after about 20 ms, and the
 * kernel returns early with PA_DEV_TIMEOUT in *dev_status and the GPU context
 * still usable.  Output is not written.  Never set it outside such tests. */
#define PA_DECODE_TEST_WITHHOLD_COPIES 1

/* pa_decode_opts.flags bit: use the CUDA-core kernel even where the
 * tensor-core kernel applies (head_dim 128, block_size 8, 16 or 32); for
 * comparisons and tests.  Same results within the documented tolerance. */
#define PA_DECODE_CUDA_CORES_ONLY 2

/* Failure-detection test hook for the *_update entry points: CTA 0 of the
 * tensor-core kernel never arrives at the new tokens' grid-wide barrier,
 * so every wait for it runs out after about 20 ms and the
 * kernel returns early with PA_DEV_TIMEOUT (pools and outputs unspecified,
 * the workspace to be zeroed again).  Never set it outside such tests. */
#define PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL 4

/*
 * pa_decode_workspace_bytes — bytes of device scratch pa_decode needs.
 *
 * The scratch holds per-CTA partial softmax states (running max, running
 * sum and unnormalised output of each query head of a kv head) and one
 * arrival counter per (sequence, kv head).  It depends on the current
 * device's SM count, so query it with the device current that will run the
 * decode.  The caller allocates it and must ZERO it once before the first
 * pa_decode; every pa_decode that ends with PA_DEV_OK leaves the counters at
 * zero again, so the same workspace serves any number of later calls on the
 * same stream.  After a non-zero device status, zero it again.  Two decodes
 * that may run at the same time need separate workspaces.  The size depends
 * on the kernel variant, so query with the opts the decode will use.
 * Returns 0 for invalid arguments.
 */
PA_API size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, const pa_pool_desc* pool);
PA_API size_t pa_decode_workspace_bytes_ex(int32_t num_seqs, int32_t num_q_heads, const pa_pool_desc* pool,
                                    const pa_decode_opts* opts);

/*
 * pa_decode — one decode step of paged attention.
 *
 * For each sequence s and query head h (kv head h / (num_q_heads /
 * num_kv_heads), contiguous GQA groups), with n = seq_lens[s]:
 *   out[s][h] = sum_t softmax_t(scale * q[s][h] . K_t) V_t,  t = 0..n-1,
 * where K_t / V_t are row t % B of block block_tables[s][t / B] of the
 * pools (vLLM blog §"关键细节" 2): softmax(QK^T/sqrt(d))V through block_table; study
 * notes ch.05 §4: blocks merged with a running max and running sum).
 * A sequence with n == 0 gets a zero output.  Rows of a partly filled last
 * block past n are never read into the result (they may hold anything).
 *
 * Arguments
 *   q               [num_seqs][num_q_heads][head_dim], fp16/bf16
 *   k_pool, v_pool  [num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables    int32 [num_seqs][max_blocks_per_seq]; only the first
 *                   ceil(n / B) entries of each row are read
 *   seq_lens        int32 [num_seqs]
 *   num_q_heads     multiple of pool->num_kv_heads; the group size
 *                   num_q_heads / num_kv_heads must be 1, 2, 4 or 8
 *   scale           multiplier of q.K (typically 1/sqrt(head_dim))
 *   out             [num_seqs][num_q_heads][head_dim], same dtype as q
 *   workspace       device scratch of at least pa_decode_workspace_bytes()
 *                   bytes, zeroed before first use (see above)
 *   dev_status      nullable int32 device pointer (see the conventions)
 * Accumulation is fp32; the output is rounded to the input dtype.
 * Device errors: PA_DEV_BAD_SEQ_LEN (that sequence is treated as empty),
 * PA_DEV_BAD_BLOCK_ID (block 0 is read instead), PA_DEV_TIMEOUT.
 */
PA_API pa_status pa_decode(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                    float scale, void* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                    const pa_pool_desc* pool, void* stream);

/* pa_decode with explicit options (e.g. a fixed CTA count; num_ctas = 1
 * processes every block in one CTA, without any cross-CTA merge). */
PA_API pa_status pa_decode_ex(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
                       int32_t num_q_heads, float scale, void* out, void* workspace, size_t workspace_bytes,
                       int32_t* dev_status, const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream);

/*
 * pa_decode_lse — pa_decode that also returns each output row's log
 * normaliser, so that decodes of disjoint token ranges of the same rows can
 * be merged afterwards (pa_merge_partials): a sequence too long for one GPU
 * split by blocks across GPUs, each decoding its own range.  The merge is
 * the online-softmax rule of study notes ch.05 §4 applied to the ranges.
 *   lse   float32 device [num_seqs][num_q_heads], 4-byte aligned:
 *         lse[s][h] = log sum_t exp(scale * q[s][h] . K_t) over the
 *         sequence's tokens (natural log), -inf for a sequence with no token
 * Other arguments, results and errors as pa_decode_ex.  The tensor-core
 * kernel writes it (head_dim 128, 16-bit pools, blocks of 8, 16 or 32);
 * elsewhere (and under PA_DECODE_CUDA_CORES_ONLY) PA_ERR_UNSUPPORTED.
 */
PA_API pa_status pa_decode_lse(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
                               int32_t num_q_heads, float scale, void* out, float* lse, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                               const pa_decode_opts* opts, void* stream);

/*
 * pa_merge_partials — merge decodes of disjoint token ranges of the same
 * query rows (study notes ch.05 §4: the online-softmax merge, rescaling each
 * part to a common maximum).  For each row i with M = max_r lses[r][i] and
 * w_r = exp(lses[r][i] - M):
 *   out[i] = sum_r w_r outs[r][i] / sum_r w_r
 *   lse_out[i] = M + log sum_r w_r            (lse_out nullable)
 * A part with lse -inf (no token) adds nothing; a row no part saw gets a
 * zero output and -inf.  The merge is exact up to fp32 rounding; the parts'
 * outputs are already rounded to the 16-bit type, so a merged output
 * carries their rounding (at most one 16-bit rounding step) beside its own.
 *   outs     [num_parts][num_rows][head_dim], fp16/bf16 (dtype), 16-byte aligned
 *   lses     float32 [num_parts][num_rows] (as pa_decode_lse writes them)
 *   out      [num_rows][head_dim], same dtype; lse_out float32 [num_rows]
 * num_rows is num_seqs * num_q_heads for decode outputs; head_dim 64 or 128.
 * num_rows == 0 is a no-op.  No device errors.
 */
PA_API pa_status pa_merge_partials(const void* outs, const float* lses, int32_t num_parts, int32_t num_rows,
                                   int32_t head_dim, int32_t dtype, void* out, float* lse_out, void* stream);

/*
 * pa_decode_no_alloc — pa_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a calling convention of
 * this library, not part of the method.
 *
 * Who needs it: code that is handed its inputs and outputs and may not call
 * cudaMalloc or any routine that allocates — for example a plug-in run by a
 * host engine that has already claimed nearly all device memory for its KV
 * pool and gives the plug-in nothing else, or a latency-critical loop where
 * an allocation (and the device synchronisation it can imply) is not allowed.
 *
 * It takes pa_decode's arguments minus the workspace and computes the same
 * result with the same kernel.  Its scratch is a fixed array of
 * PA_DECODE_NO_ALLOC_SCRATCH_BYTES (8 MiB) in libpa's own device memory; every
 * GPU that loads the library holds that array until the process exits.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it.  Make
 *     that first call on a device before any stream capture.  The cache is
 *     tied to the device's context: after a cudaDeviceReset the next call
 *     looks the address up again, and is then a first call once more.
 *   - Each call clears the arrival counters it needs (cudaMemsetAsync on
 *     `stream`) and launches the decode.  Nothing is allocated or freed.
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls that can overlap on the GPU (other streams, or unordered work on
 *     one stream) race and give wrong results.  Order them.
 *   - Returns PA_ERR_SCRATCH_LIMIT, doing nothing, when the batch needs more
 *     scratch than the array holds (what pa_decode_workspace_bytes reports for
 *     the same arguments must not exceed PA_DECODE_NO_ALLOC_SCRATCH_BYTES).
 */
#define PA_DECODE_NO_ALLOC_SCRATCH_BYTES (8u << 20)
PA_API pa_status pa_decode_no_alloc(const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                    int32_t num_seqs, int32_t num_q_heads, float scale, void* out,
                                    int32_t* dev_status, const pa_pool_desc* pool, void* stream);

/*
 * pa_decode_multi — paged attention for q_len new query positions per
 * sequence, causal among them: verifying q_len speculated tokens, or a
 * short prefill chunk (CSDN "PagedAttention：分页注意力", §"2026年最新进展"
 * items 1-2: speculative decoding and chunked prefill on the paged cache).
 * The pages give no formula beyond decode's; the plain reading used here is
 * causal attention of the new positions over the cache that already holds
 * them:
 *   out[s][i][h] = sum_t softmax_t(scale * q[s][i][h] . K_t) V_t,
 *                  t = 0 .. seq_lens[s] - q_len + i,   i = 0 .. q_len-1,
 * with K_t / V_t found through block_tables exactly as in pa_decode (the
 * q_len new tokens must already be in the cache: pa_cache_write first).
 *   q, out   [num_seqs][q_len][num_q_heads][head_dim]
 *   others   as pa_decode
 * q_len == 1 is pa_decode.  For q_len >= 2 the tensor-core kernel runs:
 * head_dim 128, block_size 8, 16 or 32, group size G = num_q_heads / num_kv_heads in
 * {1, 2, 4, 8}, any q_len.  One unit of work carries up to 32 query rows
 * (G heads times a power-of-two count of positions); when G * q_len is
 * larger (a prefill chunk), each sequence is split into row tiles of 32 / G
 * positions, each tile a unit that reads only the blocks its last position
 * sees, the tiles of a sequence adjacent so that their reads of the same
 * blocks mostly hit in L2.  Other shapes return PA_ERR_UNSUPPORTED, as does
 * PA_DECODE_CUDA_CORES_ONLY.
 * A sequence with seq_lens[s] == 0 gets zero outputs; 0 < seq_lens[s] <
 * q_len is PA_DEV_BAD_SEQ_LEN (zero outputs).  Workspace: as pa_decode, sized
 * by pa_decode_multi_workspace_bytes (0 for invalid or unsupported shapes).
 */
PA_API size_t pa_decode_multi_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                              const pa_pool_desc* pool, const pa_decode_opts* opts);
PA_API pa_status pa_decode_multi(const void* q, const void* k_pool, const void* v_pool,
                                 const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 int32_t num_seqs, int32_t q_len, int32_t num_q_heads, float scale, void* out,
                                 void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                 const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream);

/*
 * pa_decode_shared_prefix — pa_decode for batches in which groups of
 * sequences share their leading blocks (parallel samples or beams of one
 * prompt, study notes ch.05 §6.1; requests with a cached common prefix,
 * "vLLM 是什么" §3 Prefix Caching).  Same result as pa_decode (within the
 * decode tolerance), but each shared block is read from memory once per
 * group instead of once per member.
 *
 * Groups are consecutive sequences: group g holds sequences
 * [group_starts[g], group_starts[g+1]), and its first group_prefix_blocks[g]
 * logical blocks are the same physical blocks for every member (as
 * pa_bm_fork leaves them); the kernel reads them through the first member's
 * table row and ignores the other members' entries for those blocks.
 *   group_starts         int32 device [num_groups + 1], group_starts[0] == 0,
 *                        non-decreasing, group_starts[num_groups] == num_seqs
 *   group_prefix_blocks  int32 device [num_groups]
 *   max_group_size       host bound on members per group, >= 1
 * A group shares nothing (its members are decoded one by one) when its
 * prefix is 0, or not shorter than every member's block count.
 * One launch of the tensor-core kernel over (group, kv head) units: a unit
 * streams the group's shared blocks once, seen by every member's query
 * heads, then each member's own blocks, seen by that member's heads only, and
 * writes every member's outputs.  Tensor-core kernel only: head_dim 128,
 * block_size 8, 16 or 32, G in {1, 2, 4, 8} and G * max_group_size <= 32
 * (rounded up to a power of two), else PA_ERR_UNSUPPORTED.  Device errors: those of
 * pa_decode, and PA_DEV_BAD_GROUP when the groups do not partition the
 * sequences or a group has more members than max_group_size rounded up to a
 * power of two (outputs then unspecified).  The workspace
 * (pa_decode_shared_prefix_workspace_bytes; zeroed before first use, as for
 * pa_decode) holds the partial states of units split between CTAs.
 */
PA_API size_t pa_decode_shared_prefix_workspace_bytes(int32_t num_seqs, int32_t max_group_size,
                                                      int32_t num_q_heads, const pa_pool_desc* pool,
                                                      const pa_decode_opts* opts);
PA_API pa_status pa_decode_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                                         const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                         const int32_t* group_starts, const int32_t* group_prefix_blocks,
                                         int32_t num_groups, int32_t max_group_size, float scale, void* out,
                                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                         const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream);

/*
 * pa_cache_write — store the K/V of new tokens into their slots
 * (vLLM blog, plain-language section: each generated token's K/V is
 * written to the cache;
 * study notes ch.05 §5 item 2: a token goes to the next free slot).
 *
 * For each token t with slot = slot_mapping[t] >= 0:
 *   k_pool[slot / B][h][slot % B][:] = k[t][h][:]   for every kv head h
 *   v_pool[slot / B][h][slot % B][:] = v[t][h][:]
 * A bit copy: no rounding.  Negative slots skip the token (padding).  Two
 * tokens with the same slot in one call: undefined which one lands.
 *   k, v          [num_tokens][num_kv_heads][head_dim]
 *   slot_mapping  int64 [num_tokens]
 * num_tokens == 0 is a no-op.  Device error: PA_DEV_BAD_SLOT (token skipped).
 */
PA_API pa_status pa_cache_write(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                         void* k_pool, void* v_pool, int32_t* dev_status, const pa_pool_desc* pool,
                         void* stream);

/*
 * pa_copy_blocks — copy-on-write block copies (study notes ch.05 §6.1: a
 * writer to a shared block copies it first; §12 exercise 4).
 *
 * For each pair i: block src_dst_pairs[2i+1] of both pools becomes a bit
 * copy of block src_dst_pairs[2i] (all kv heads, all rows).  src == dst is
 * a no-op.  Pairs run in parallel: a dst that appears twice, or that is
 * also a src in the same call, is undefined.
 *   src_dst_pairs int64 [num_pairs][2] (src, dst)
 * num_pairs == 0 is a no-op.  Device error: PA_DEV_BAD_PAIR (pair skipped).
 */
PA_API pa_status pa_copy_blocks(const int64_t* src_dst_pairs, int32_t num_pairs, void* k_pool, void* v_pool,
                         int32_t* dev_status, const pa_pool_desc* pool, void* stream);

/*
 * One decode step's cache update followed by its attention, the new tokens'
 * stores inside the decode's launch where the tensor-core kernel runs.  A
 * serving step first copies the blocks that copy on write gives a writer
 * (study notes ch.05 §6.1), then stores each new token's K/V in its slot
 * (vLLM blog, plain-language section), then attends over the cache that now
 * holds it (vLLM blog §"关键细节" 2).  These entry points take the three as
 * one call:
 *
 *   pa_copy_blocks(update->copy_pairs, ...);
 *   pa_cache_write(update->k, update->v, update->slot_mapping, ...);
 *   pa_decode_ex / pa_decode_multi / pa_decode_shared_prefix(...);
 *
 * with the same results (pools bit for bit, outputs within the decode
 * tolerance) and the same device errors.  The pool pointers are written.
 * Where the tensor-core decode kernel runs (head_dim 128, 16-bit pools, the
 * shapes listed for each decode; not the query-major prefill kernel) and
 * the grid fits on the GPU at once, the stores run inside its launch: all
 * CTAs take a share of them at the start, and a grid-wide barrier (an
 * arrival count and a generation word in the workspace, every wait bounded)
 * holds back every K/V load until the last store has landed.  That saves a
 * launch per step.  The block copies always run as pa_copy_blocks' own
 * kernel ahead of the decode: inside the launch they measured slower.
 * Elsewhere the three kernels are enqueued in order on `stream`.
 *
 * update == NULL, or both counts 0, is the plain decode.  copy_pairs and
 * slot_mapping follow pa_copy_blocks and pa_cache_write (pairs run in
 * parallel, and a dst that is also a src is undefined; negative slots are
 * padding).  k, v are [num_tokens][num_kv_heads][head_dim] like the pools,
 * 16-byte aligned.  The workspace is the decode's (same size query); its
 * barrier words are left as found when the device status is PA_DEV_OK.  A
 * barrier wait that runs out (for instance when other work keeps part of
 * the grid off the GPU for its whole limit) records PA_DEV_TIMEOUT; the
 * pools and outputs are then unspecified and the workspace must be zeroed
 * again, as after any non-zero device status.  The barrier needs every CTA
 * of the launch on an SM at once: do not run two of these calls at the same
 * time on different streams (each could hold SMs the other's grid waits
 * for until its waits run out); order them on one stream.
 */
typedef struct pa_cache_update {
  const int64_t* copy_pairs;  /* int64 [num_copy_pairs][2] (src, dst) block ids, device; NULL when 0 */
  int32_t num_copy_pairs;
  const void* k;              /* new tokens' keys [num_tokens][num_kv_heads][head_dim], device */
  const void* v;              /* their values, same layout */
  const int64_t* slot_mapping; /* int64 [num_tokens], device */
  int32_t num_tokens;
} pa_cache_update;

PA_API pa_status pa_decode_update(const pa_cache_update* update, const void* q, void* k_pool, void* v_pool,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                  int32_t num_seqs, int32_t num_q_heads, float scale, void* out, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                                  const pa_decode_opts* opts, void* stream);
PA_API pa_status pa_decode_multi_update(const pa_cache_update* update, const void* q, void* k_pool, void* v_pool,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* seq_lens, int32_t num_seqs, int32_t q_len,
                                        int32_t num_q_heads, float scale, void* out, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                                        const pa_decode_opts* opts, void* stream);
PA_API pa_status pa_decode_shared_prefix_update(const pa_cache_update* update, const void* q, void* k_pool,
                                                void* v_pool, const int32_t* block_tables,
                                                int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                                int32_t num_seqs, int32_t num_q_heads, const int32_t* group_starts,
                                                const int32_t* group_prefix_blocks, int32_t num_groups,
                                                int32_t max_group_size, float scale, void* out, void* workspace,
                                                size_t workspace_bytes, int32_t* dev_status,
                                                const pa_pool_desc* pool, const pa_decode_opts* opts,
                                                void* stream);

/*
 * Host block manager — the bookkeeping half of the method (study notes
 * ch.05 §3 block table, §5 ② on-demand allocation, §6.1 sharing and copy on
 * write, §6.2 reference counts, §12 exercise 4).  Plain C++ on the host; it
 * produces the block tables, lengths, slot mappings and copy-on-write pairs
 * that pa_copy_blocks / pa_cache_write / pa_decode consume.
 *
 * Blocks are handed out first-in first-out from a free set that starts as
 * 0..num_blocks-1.  Sequences are named by caller-chosen int64 ids.  A
 * manager is not thread safe.  Calls that fail return an error and change
 * nothing.
 */
typedef struct pa_block_manager pa_block_manager;

typedef struct pa_bm_stats {
  int32_t num_blocks;     /* pool size */
  int32_t free_blocks;    /* in the free set */
  int32_t used_blocks;    /* referenced by at least one sequence */
  int32_t shared_blocks;  /* referenced by two or more sequences */
  int32_t num_sequences;
  int64_t logical_blocks; /* sum over sequences of table lengths (what unshared storage would need) */
  int64_t tokens;         /* sum over sequences of token counts */
  int64_t slots_filled;   /* rows of used blocks that hold a token */
} pa_bm_stats;

/* A manager over num_blocks blocks of block_size tokens; NULL on bad sizes. */
PA_API pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size);
PA_API void pa_bm_destroy(pa_block_manager* bm);

/* Register sequence seq_id holding num_tokens tokens (its prompt):
 * ceil(num_tokens / block_size) fresh blocks.  PA_ERR_INVALID_ARG for a
 * known id, PA_ERR_OUT_OF_BLOCKS when the free set is too small. */
PA_API pa_status pa_bm_add(pa_block_manager* bm, int64_t seq_id, int32_t num_tokens);

/* child_id starts as a copy of parent_id's table: every block gains one
 * reference (parallel sampling / beam search share, study notes §6.1, §6.2). */
PA_API pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/* Reserve the slot of the sequence's next token: a fresh block when the
 * last one is full; when the target block is shared, a fresh block becomes
 * the sequence's private copy first (*cow_src, *cow_dst receive the pair,
 * else -1; the source loses one reference).  Pointers may be NULL. */
PA_API pa_status pa_bm_append(pa_block_manager* bm, int64_t seq_id, int64_t* slot, int64_t* cow_src,
                              int64_t* cow_dst);

/* Drop the sequence: one reference off each of its blocks; blocks that reach
 * zero return to the end of the free set. */
PA_API pa_status pa_bm_free(pa_block_manager* bm, int64_t seq_id);

/* Free blocks, or -1 for a NULL manager. */
PA_API int32_t pa_bm_num_free_blocks(const pa_block_manager* bm);
/* Reference count of one physical block, or -1 if out of range. */
PA_API int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block);
/* The sequence's block table (first *num_blocks entries of `blocks`) and
 * token count.  PA_ERR_INVALID_ARG if capacity is too small (the counts are
 * still written). */
PA_API pa_status pa_bm_table(const pa_block_manager* bm, int64_t seq_id, int32_t* blocks, int32_t capacity,
                             int32_t* num_blocks, int32_t* num_tokens);
PA_API void pa_bm_get_stats(const pa_block_manager* bm, pa_bm_stats* out);

/* One decode step for a batch: append one token to each of the n distinct
 * sequences in order, then fill the arrays the kernels take —
 *   block_tables [n][max_blocks_per_seq] (rows padded with -1),
 *   seq_lens [n] (token counts after the append),
 *   slot_mapping [n] (the new tokens' slots),
 *   copy_pairs [max_pairs][2] with *num_pairs copy-on-write pairs to run
 *   (pa_copy_blocks) before the cache write.
 * Checks ids, table width, free blocks and pair room first; on any error
 * nothing changes. */
PA_API pa_status pa_bm_prepare_step(pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                                    int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* seq_lens,
                                    int64_t* slot_mapping, int64_t* copy_pairs, int32_t max_pairs,
                                    int32_t* num_pairs);

/* Plan the groups of pa_decode_shared_prefix from HOST copies of one step's
 * block tables and lengths (the layout pa_bm_prepare_step writes).
 * Consecutive sequences whose first table entries are the same physical
 * block form a group of at most max_group_size members; the group's prefix is
 * the number of leading entries that every member has in common with the
 * first one, capped so that each member keeps at least one block of its own
 * (a group of one, or a prefix under min_prefix_blocks, gets 0: no sharing).
 * Writes group_starts [*num_groups + 1] and group_prefix_blocks [*num_groups]
 * (room for num_seqs + 1 and num_seqs entries).  Sequences of length 0 or
 * with an invalid length are groups of one. */
PA_API pa_status pa_shared_prefix_groups(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                         const int32_t* seq_lens, int32_t num_seqs, int32_t block_size,
                                         int32_t max_group_size, int32_t min_prefix_blocks, int32_t* group_starts,
                                         int32_t* group_prefix_blocks, int32_t* num_groups);

/*
 * pa_step — one whole step of a paged KV cache driven from pinned host
 * memory: the host->device copy of the step's inputs, the copy-on-write
 * block copies (pa_copy_blocks, study notes ch.05 §6.1), the cache write of
 * the new tokens (pa_cache_write, vLLM blog plain-language section), the
 * decode (pa_decode, pa_decode_multi or pa_decode_shared_prefix; vLLM blog
 * §"关键细节" 2) and the device->host copy of the output, in that order.
 * The pages describe the step, not a runtime; this is the calling
 * convention of this library for a serving loop.
 *
 * Memory is the caller's: for each of num_sets buffer sets, a device input
 * block and a pinned host input block of pa_step_layout.total bytes each
 * (16-byte aligned), a device output and a pinned host output of
 * pa_step_layout.out_bytes; the pools, the decode workspace (sized by the
 * decode's own *_workspace_bytes for the shape) and dev_status.  The input
 * blocks are laid out as pa_step_layout_of gives (q, block_tables,
 * seq_lens, group_starts, group_prefix_blocks, copy_pairs, new k, new v,
 * slot_mapping; the same layouts as the entry points take, each field at
 * its maximum size).  The step creates three CUDA streams (uploads,
 * kernels, downloads), events and, per buffer set and counts, one CUDA
 * graph of its kernels (the first step runs them directly; up to four
 * graphs a set are kept, the oldest replaced).  It makes no allocation of
 * its own (no cudaMalloc or host allocation); the driver keeps what the
 * streams, events and graphs need until pa_step_destroy.  A step object is
 * used from one host thread at a time.
 *
 * Per pa_step_run the host issues one copy of the used part of the set's
 * input block, one graph launch, and the copy of the previous step's output
 * (a step's download is held back to its next step, see pa_step_flush).
 * Sets are used
 * in turn: the upload into a set waits for the kernels that last read it,
 * the kernels of a step wait for its upload, for the previous step's
 * kernels (in-order stream: they share the pools) and for the download
 * that last read the set's output, so neighbouring steps' copies overlap
 * each other's kernels.  Call pa_step_next_set before writing a set's host
 * input block: it returns the set the next pa_step_run uses, once that
 * set's previous upload is done.  pa_step_wait blocks until a set's output
 * has reached its host block.  Errors: PA_ERR_INVALID_ARG for a bad shape
 * or pointer, the decode's own return codes from the first step, and
 * PA_ERR_CUDA for a failed CUDA call.
 */
#define PA_STEP_DECODE 0        /* pa_decode (opts.flags may hold PA_DECODE_CUDA_CORES_ONLY) */
#define PA_STEP_MULTI 1         /* pa_decode_multi with q_len positions per sequence */
#define PA_STEP_SHARED_PREFIX 2 /* pa_decode_shared_prefix over groups of up to max_group_size */
#define PA_STEP_MAX_SETS 8

typedef struct pa_step_shape {
  int32_t kind;               /* PA_STEP_* */
  int32_t num_seqs;
  int32_t num_q_heads;
  int32_t max_blocks_per_seq;
  int32_t q_len;              /* PA_STEP_MULTI: positions per sequence (>= 2); else 1 */
  int32_t max_group_size;     /* PA_STEP_SHARED_PREFIX: members per group; else 0 */
  int32_t max_new_tokens;     /* capacity of the new-token fields */
  int32_t max_copy_pairs;     /* capacity of the copy-pair field */
  float scale;
  pa_decode_opts opts;
} pa_step_shape;

/* Byte offsets of the fields in a set's input block, its size and the
 * output size.  Fields a shape does not use have size 0 (offset = the next
 * field's). */
typedef struct pa_step_layout {
  size_t q, block_tables, seq_lens, group_starts, group_prefix_blocks, copy_pairs, new_k, new_v, slot_mapping;
  size_t total;
  size_t out_bytes;
} pa_step_layout;

typedef struct pa_step pa_step;

PA_API pa_status pa_step_layout_of(const pa_step_shape* shape, const pa_pool_desc* pool, pa_step_layout* layout);
PA_API pa_status pa_step_create(const pa_step_shape* shape, const pa_pool_desc* pool, void* k_pool, void* v_pool,
                                void* workspace, size_t workspace_bytes, int32_t* dev_status, int32_t num_sets,
                                void* const* dev_inputs, void* const* host_inputs, void* const* dev_outputs,
                                void* const* host_outputs, pa_step** step);
/* The set the next pa_step_run uses (its previous upload done). */
PA_API pa_status pa_step_next_set(pa_step* step, int32_t* set);
/* Enqueue one step with these counts (copy pairs, new tokens, shared-prefix
 * groups) from the next set's host input block; *set = the set used. */
PA_API pa_status pa_step_run(pa_step* step, int32_t num_copy_pairs, int32_t num_new_tokens, int32_t num_groups,
                             int32_t* set);
/* Block until that set's output is in its host block (its download is
 * enqueued first if it is still held back, see pa_step_flush). */
PA_API pa_status pa_step_wait(pa_step* step, int32_t set);
/* A step's download is enqueued with the next pa_step_run, behind that
 * step's upload (a download waits for its kernels, and an upload behind it
 * on the same copy queue would wait with it).  pa_step_flush enqueues the
 * held-back download now; pa_step_wait and pa_step_synchronize do so
 * themselves. */
PA_API pa_status pa_step_flush(pa_step* step);
PA_API pa_status pa_step_synchronize(pa_step* step);
/* The upload, kernel and download streams (cudaStream_t as void*). */
PA_API pa_status pa_step_streams(pa_step* step, void** upload, void** kernels, void** download);
PA_API void pa_step_destroy(pa_step* step);

/* Static string for a pa_status or PA_DEV_* code. */
PA_API const char* pa_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

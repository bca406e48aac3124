/*
 * pkv.h -- C ABI of libpkv.so: paged KV-cache decode attention for NVIDIA
 * B200 (sm_100a), plus the host-side block allocator that manages the pages.
 *
 * Sources for what each call computes (web pages, cited by title + section):
 *   [KVB] "LLM Inference: KV Cache, Batching & Scheduling" (cariara.com),
 *         sections "The KV cache" and "PagedAttention and vLLM".
 *   [ENG] "LLM Inference Engineering: Overcoming the KV-Cache Bottleneck and
 *         Maximizing Production Throughput" -- wpnews.pro summary, section
 *         "2. The Architectural Solution: Virtual Memory and PagedAttention";
 *         adilsher.pro post, section "The Elegant Fix: Paged Attention".
 *
 * Conventions shared by every call
 * --------------------------------
 *   B  = number of sequences, Hq / Hkv = query / KV heads, G = Hq / Hkv,
 *   D  = head_dim (64 or 128), bs = block_size (a multiple of 16), NB = pool
 *   blocks, MB = max blocks per sequence (row length of the block table).
 *
 *   KV pool layout: k_cache and v_cache are two separate device arrays of
 *   shape [NB][Hkv][bs][D] (16-bit floats), indexed by the same physical block
 *   id.  The (block, kv-head) tile of bs*D elements is contiguous.  Position p
 *   of a sequence lives in block block_tables[seq][p / bs], row p % bs.
 *   A flat "slot" is block * bs + row.
 *
 *   Query head h attends with KV head h / G (contiguous query-head groups
 *   share one KV head -- the GQA layout of [KVB] "The KV cache").
 *
 *   context_lens[s] is the sequence length AFTER this step's append: the
 *   new token sits at position context_lens[s] - 1 and attention covers
 *   positions 0 .. context_lens[s] - 1 inclusive.  A length of 0 produces an
 *   all-zero output row.
 *
 * Ownership: the caller owns every device buffer (caches, q, out, tables,
 * lengths, workspace).  The library never allocates or frees device memory
 * in these calls; it owns only the allocator's host state.
 *
 * Errors: every call validates shapes, dtypes and alignment on the host and
 * returns PKV_ERR_INVALID without launching anything.  Launches are
 * asynchronous on the caller's stream; a launch failure returns PKV_ERR_CUDA.
 * Device-side checks (a slot, table entry or length out of range) never trap:
 * the kernel skips the access, records the fault in a device word and keeps
 * going; pkv_get_last_error() reports it.  No call aborts the process.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID = -1,      /* bad argument; nothing was launched or changed      */
    PKV_ERR_OOM = -2,          /* allocator: not enough free blocks; nothing changed */
    PKV_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed               */
    PKV_ERR_SHARED_WRITE = -4, /* allocator: the target block is shared (refcount>1) */
    PKV_ERR_DEVICE_CHECK = -5, /* a kernel found an index out of range and skipped it */
    PKV_ERR_TIMEOUT = -6,      /* a kernel's bounded wait ran out and it returned early */
    PKV_ERR_SCRATCH_TOO_SMALL = -7 /* the shape needs more scratch than the fixed static area */
} pkv_status;

/* PKV_E4M3: FP8 E4M3 codes (1 byte) with one fp32 scale per (slot, KV head)
 * in pkv_cache.scales; used by the *_e4m3 calls only. */
typedef enum pkv_dtype { PKV_F16 = 0, PKV_BF16 = 1, PKV_E4M3 = 2 } pkv_dtype;

/* One KV pool: caller-owned device pointer plus its shape [NB][Hkv][bs][D].
 * data must be 16-byte aligned (TMA tiles are read straight from it).
 * scales: E4M3 pools only, device fp32 [NB][Hkv][bs] (16-byte aligned): the
 * scale of each cached row; NULL for 16-bit pools. */
typedef struct pkv_cache {
    void *data;
    pkv_dtype dtype;
    int64_t num_blocks;
    int64_t block_size;
    int64_t num_kv_heads;
    int64_t head_dim;
    float *scales;
} pkv_cache;

/* A cudaStream_t without including CUDA headers (same underlying type). */
struct CUstream_st;
typedef struct CUstream_st *pkv_stream;

/* --------------------------------------------------------------------------
 * pkv_append -- store this step's new K and V of every token in its slot.
 * [KVB] "The KV cache": the cache keeps K and V of every past position and
 * appends the new token's K and V each step.
 *
 *   k_new, v_new   device [T][Hkv][D], same dtype and Hkv/D as the caches
 *   slot_mapping   device int64 [T]; slot = block * bs + row; slot < 0 means
 *                  "padding token, write nothing"
 *   num_tokens     T >= 0 (T == 0 is a no-op)
 *
 * Bitwise copy: cache[slot / bs][h][slot % bs][:] = new[t][h][:] for all h.
 * A slot with block >= NB is skipped and flagged (PKV_ERR_DEVICE_CHECK).
 * Two tokens mapped to the same slot race (last writer unspecified).
 * ------------------------------------------------------------------------ */
pkv_status pkv_append(const void *k_new, const void *v_new,
                      const int64_t *slot_mapping, int64_t num_tokens,
                      pkv_cache k_cache, pkv_cache v_cache, pkv_stream stream);

/* --------------------------------------------------------------------------
 * FP8 E4M3 KV cache.  The pages leave quantization open (adilsher.pro post,
 * "What I'm Still Figuring Out": how quantization and batching interact);
 * halving the bytes per token halves the HBM traffic of this path.
 *
 * Format: OCP E4M3 codes (no infinities, largest finite 448) with one fp32
 * scale per cached (token, KV head) row -- a per-row scale keeps each append
 * a function of its own token (a per-block scale would have to change as
 * the block fills).  Quantization of a row x[0..D): amax = max |x|, scale =
 * amax / 448 (1 if amax == 0), code_d = round-to-nearest-even(x_d / scale)
 * saturated to +-448, both divisions correctly rounded in fp32.  A cached
 * value is value(code) * scale.
 *
 * pkv_append_e4m3: pkv_append into E4M3 pools; k_new / v_new are
 *   [T][Hkv][D] in new_dtype (PKV_F16 or PKV_BF16).
 * pkv_decode_attention_e4m3: pkv_decode_attention over E4M3 pools with q and
 *   out in q_dtype (PKV_F16 or PKV_BF16).  Codes are converted exactly to
 *   f16 on chip and the products run in f16 with fp32 accumulation (a bf16
 *   query is converted to f16: exact in f16's normal range); K scales
 *   multiply the scores, V scales the probabilities.  All partition modes;
 *   workspace as for pkv_decode_attention.
 * ------------------------------------------------------------------------ */
pkv_status pkv_append_e4m3(const void *k_new, const void *v_new, pkv_dtype new_dtype,
                           const int64_t *slot_mapping, int64_t num_tokens, pkv_cache k_cache,
                           pkv_cache v_cache, pkv_stream stream);
pkv_status pkv_decode_attention_e4m3(const void *q, pkv_dtype q_dtype, int64_t num_seqs,
                                     int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache,
                                     const int32_t *block_tables, int64_t max_blocks_per_seq,
                                     const int32_t *context_lens, float scale, void *out,
                                     void *workspace, size_t workspace_bytes,
                                     int32_t partition_tokens, pkv_stream stream);

/* --------------------------------------------------------------------------
 * pkv_copy_blocks -- device side of copy-on-write: for each (src, dst) pair
 * of pairs (device int32 [n][2]) copy the whole physical block src to dst in
 * both pools (all KV heads and rows: Hkv * bs * D values each).  The dst
 * blocks must be distinct and no dst may also be a src (the pairs from the
 * copy-on-write appends satisfy this), so the copies are independent.  An id
 * outside [0, NB) is skipped and flagged (PKV_ERR_DEVICE_CHECK).
 * ------------------------------------------------------------------------ */
pkv_status pkv_copy_blocks(pkv_cache k_cache, pkv_cache v_cache, const int32_t *pairs,
                           int64_t num_pairs, pkv_stream stream);

/* --------------------------------------------------------------------------
 * pkv_decode_attention -- one decode step of attention over the paged cache.
 * [KVB] "The KV cache": attention needs the keys and values of all prior
 * positions; decode generates one token at a time.  [KVB] "PagedAttention and
 * vLLM" / [ENG]: K/V live in fixed-size blocks reached through a per-sequence
 * logical -> physical block table; blocks need not be contiguous and may be
 * shared between sequences (a common prefix).
 *
 *   out[s][h][:] = sum_p softmax_p(scale * q[s][h] . K[s][p]) * V[s][p]
 *                  over p in [0, context_lens[s]), K/V of KV head h / G.
 *
 *   q              device [B][Hq][D], dtype of the caches
 *   block_tables   device int32 [B][MB]; only the first
 *                  ceil(context_lens[s] / bs) entries of row s are read
 *   context_lens   device int32 [B], 0 <= len <= MB * bs
 *   scale          softmax scale (usually 1/sqrt(D)), applied in fp32
 *   out            device [B][Hq][D], dtype of q (round-to-nearest-even)
 *   workspace      device scratch for split-context partial results, or NULL
 *   partition_tokens
 *       PKV_PARTITION_NONE (-1): one pass over each whole context; no
 *                  workspace used.
 *       PKV_PARTITION_AUTO (0): the library splits the total work evenly
 *                  across the GPU (work-balanced partitions, merged by
 *                  log-sum-exp); needs workspace >= the size reported by
 *                  pkv_decode_workspace_bytes(..., 0).  With workspace NULL it
 *                  falls back to PKV_PARTITION_NONE.
 *       P > 0 (a multiple of 16): split every context into P-token
 *                  partitions [jP, (j+1)P), computed independently and merged
 *                  by log-sum-exp in a second kernel; workspace holds fp32
 *                  partials [B][Hq][S][D] and their max / sum [B][Hq][S],
 *                  S = ceil(MB * bs / P).
 *
 * Accumulation is fp32 throughout; exp via exp2 with scale*log2(e) folded in.
 * Results do not depend on which physical blocks hold the data: the order of
 * every reduction is fixed by logical position only.
 * Limits: D in {64, 128}; bs a multiple of 16; Hq % Hkv == 0.
 *
 * Tuning variables, read from the environment when a shape is first planned
 * (plans are cached per shape and per value): PKV_WARPS (warps per CTA,
 * 1..8), PKV_STAGES (pipeline stages per warp, 2..16), PKV_FMA=1 (16-bit
 * pools: the two products on the CUDA cores in fp32 FFMA instead of the
 * tensor-core MMA -- same pipeline and schedules, a measurement aid).
 * ------------------------------------------------------------------------ */
#define PKV_PARTITION_NONE (-1)
#define PKV_PARTITION_AUTO 0

pkv_status pkv_decode_attention(const void *q, int64_t num_seqs, int64_t num_q_heads,
                                pkv_cache k_cache, pkv_cache v_cache,
                                const int32_t *block_tables, int64_t max_blocks_per_seq,
                                const int32_t *context_lens, float scale, void *out,
                                void *workspace, size_t workspace_bytes,
                                int32_t partition_tokens, pkv_stream stream);

/* --------------------------------------------------------------------------
 * pkv_append_decode_attention -- pkv_append and pkv_decode_attention of one
 * decode step in a single kernel launch (plus the merge launch when contexts
 * are split).  Same arguments as pkv_decode_attention, plus:
 *
 *   k_new, v_new   device [B][Hkv][D]: the new token of sequence s is row s
 *   slot_mapping   device int64 [B]: its slot, which must be the slot of
 *                  position context_lens[s] - 1 of sequence s (what
 *                  pkv_seq_append_slot returned); < 0 means no new token
 *
 * Result: identical to pkv_append(k_new, v_new, slot_mapping, B, ...)
 * followed by pkv_decode_attention(...) under that precondition.  The warp
 * that owns a sequence's last position reads the new row from k_new / v_new,
 * stores it in the cache and uses it directly, so no separate launch (and no
 * ordering between the two) is needed.  A sequence with context_lens[s] == 0
 * has no attended position and its token is not written.  For any other
 * token layout (several tokens per sequence, slots not at the last
 * position) use the two separate calls.
 * ------------------------------------------------------------------------ */
pkv_status pkv_append_decode_attention(const void *k_new, const void *v_new,
                                       const int64_t *slot_mapping, const void *q, int64_t num_seqs,
                                       int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache,
                                       const int32_t *block_tables, int64_t max_blocks_per_seq,
                                       const int32_t *context_lens, float scale, void *out,
                                       void *workspace, size_t workspace_bytes,
                                       int32_t partition_tokens, pkv_stream stream);

/* --------------------------------------------------------------------------
 * pkv_prefill_attention -- chunked prefill over the paged cache.
 * [KVB] "Chunked prefill": a long prompt is split into fixed-size chunks
 * (e.g. 512 tokens) that are interleaved with other requests' decode steps.
 *
 *   q, out         device [T][Hq][D], the chunk tokens of all sequences in
 *                  sequence order, T = num_tokens = query_start[B]
 *   query_start    device int32 [B + 1], query_start[0] = 0: sequence s owns
 *                  tokens query_start[s] .. query_start[s+1] - 1 (n_s >= 1)
 *   context_lens   device int32 [B]: length of sequence s AFTER its chunk's
 *                  K/V were appended (pkv_append with the chunk's slots), so
 *                  the chunk holds positions ctx_s - n_s .. ctx_s - 1
 *   block_tables   device int32 [B][MB], one row per sequence
 *   workspace      required, >= pkv_prefill_workspace_bytes(...)
 *
 * Query i of sequence s attends causally to positions 0 .. ctx_s - n_s + i.
 * A decode sequence is a chunk of one, so prefill chunks and decode tokens
 * go in one call.  Chunks of two or more tokens run on a multi-query
 * tensor-core kernel (tcgen05, fp32 accumulators in tensor memory): blocks
 * of 128 / G tokens x the G query heads of one KV head form 128-row tiles
 * that read each K/V tile of their causal range once.  Decode tokens run on
 * the decode kernel.  (Environment PKV_PREFILL_MQ=0 sends every token
 * through the decode kernel instead -- the path before the multi-query
 * kernel, kept for comparison.)  Inconsistent lengths (n_s < 1, ctx_s < n_s)
 * are flagged on the device and give zero rows.  Same limits as
 * pkv_decode_attention; T < 2^24; the multi-query kernel needs G <= 128,
 * B <= 4096 and scale != 0 (otherwise every token takes the decode kernel).
 * ------------------------------------------------------------------------ */
pkv_status pkv_prefill_attention(const void *q, int64_t num_tokens, int64_t num_seqs, int64_t num_q_heads,
                                 pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
                                 int64_t max_blocks_per_seq, const int32_t *query_start,
                                 const int32_t *context_lens, float scale, void *out, void *workspace,
                                 size_t workspace_bytes, pkv_stream stream);
size_t pkv_prefill_workspace_bytes(int64_t num_tokens, int64_t num_q_heads, int64_t num_kv_heads,
                                   int64_t head_dim, int64_t max_context_len);

/* --------------------------------------------------------------------------
 * pkv_append_decode_attention_shared_prefix -- a decode step (with an
 * optional fused append) for a batch in which groups of sequences share the
 * blocks of a common prefix.  [KVB] "Prefix caching": many requests share a
 * prefix (a system prompt, few-shot examples); [ENG] "The Elegant Fix":
 * requests with the same prompt prefix share pages instead of duplicating
 * them.  The result is exactly pkv_append_decode_attention's (attention over
 * each sequence's whole context); only the way it is computed differs: each
 * shared prefix is read once per group and scored against every member's
 * query heads together on the tensor cores (M = members x G rows), each
 * sequence's own blocks after it go through the decode kernel, which resumes
 * from the prefix's fp32 partial (max, sum, weighted V) -- no extra merge.
 *
 *   k_new, v_new, slot_mapping   as for pkv_append_decode_attention, or all
 *                  three NULL for no append
 *   group_start    device int32 [num_groups + 1]: group g is sequences
 *                  group_start[g] .. group_start[g+1]-1 (consecutive in the
 *                  batch); group_start[0] = 0, group_start[num_groups] = B,
 *                  non-decreasing.  A sequence sharing nothing is a group
 *                  of one.
 *   shared_lens    device int32 [B]: claimed number of leading positions of
 *                  each sequence stored in blocks shared with its group
 *                  (e.g. from pkv_batch_prefix_groups)
 *   workspace      >= pkv_shared_prefix_workspace_bytes(...)
 *
 * The kernel takes as the group's reference the first member with the
 * largest claim, and uses for each member only whole blocks that (a) are
 * within its claim, (b) end before its last position (the position of this
 * step's new token stays in the sequence's own block) and (c) have the same
 * table entries as the reference's: a wrong claim only shrinks the shared
 * part, never changes the result.  A group_start that does not run from 0
 * to B without decreasing is flagged (PKV_ERR_DEVICE_CHECK) and the step
 * computed without sharing (still exact).
 * Limits: those of pkv_decode_attention, 16-bit pools, G <= 128,
 * num_groups <= 4096; num_groups == 0 (or scale == 0) runs the plain step.
 * ------------------------------------------------------------------------ */
pkv_status pkv_append_decode_attention_shared_prefix(
    const void *k_new, const void *v_new, const int64_t *slot_mapping, const void *q, int64_t num_seqs,
    int64_t num_q_heads, pkv_cache k_cache, pkv_cache v_cache, const int32_t *block_tables,
    int64_t max_blocks_per_seq, const int32_t *context_lens, const int32_t *group_start, int64_t num_groups,
    const int32_t *shared_lens, float scale, void *out, void *workspace, size_t workspace_bytes,
    pkv_stream stream);
/* Bytes of workspace for pkv_append_decode_attention_shared_prefix on the
 * current device (0 for invalid arguments). */
size_t pkv_shared_prefix_workspace_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                         int64_t head_dim, int64_t max_context_len, int64_t num_groups);

/* --------------------------------------------------------------------------
 * pkv_decode_attention_static_scratch -- pkv_decode_attention for callers
 * that cannot allocate device memory.  (No counterpart on the pages: this is
 * an interface convenience, not part of the method.)
 *
 * Who needs it: code that only ever receives device pointers from its host
 * framework -- a custom-operator or plugin interface that hands over the
 * inputs and outputs but no allocator -- and serving loops that forbid device
 * allocation once they are running, because cudaMalloc / cudaFree can
 * synchronise the device, fail under memory pressure or fragment the pool in
 * the middle of a run.  Such callers still pass q, the caches, the tables,
 * the lengths and out; the split-context scratch comes from a fixed array
 * that lives in the library's device image.
 *
 * Arguments and results are those of pkv_decode_attention with the scratch
 * taken from a file-scope device array of PKV_STATIC_SCRATCH_BYTES bytes
 * (every GPU that loads the library holds that array until the process
 * exits).  A shape whose split scratch (pkv_decode_workspace_bytes for the
 * same arguments) exceeds it is refused with PKV_ERR_SCRATCH_TOO_SMALL
 * before anything is launched; PKV_PARTITION_NONE needs no scratch.
 *
 * The first call on each device looks up the array's device address (a
 * runtime query, no allocation) with that device current; make that first
 * call before any stream capture.  Every call on a device shares the one
 * array and leaves its last contents there; nothing in it has to start at
 * zero (each call writes every value it later reads).  Calls whose kernels
 * overlap on the GPU -- e.g. on two streams at once -- race on the array and
 * must be serialised by the caller.  No cudaMalloc, cudaFree or allocating
 * library routine is called.
 * ------------------------------------------------------------------------ */
#define PKV_STATIC_SCRATCH_BYTES (32u << 20)

pkv_status pkv_decode_attention_static_scratch(const void *q, int64_t num_seqs, int64_t num_q_heads,
                                               pkv_cache k_cache, pkv_cache v_cache,
                                               const int32_t *block_tables,
                                               int64_t max_blocks_per_seq,
                                               const int32_t *context_lens, float scale, void *out,
                                               int32_t partition_tokens, pkv_stream stream);

/* Bytes of workspace pkv_decode_attention needs for this shape and
 * partition_tokens on the CURRENT device (AUTO depends on its SM count).
 * max_context_len is the largest context any sequence may have (MB * bs).
 * Returns 0 for PKV_PARTITION_NONE and for invalid arguments. */
size_t pkv_decode_workspace_bytes(int64_t num_seqs, int64_t num_q_heads, int64_t num_kv_heads,
                                  int64_t head_dim, int64_t max_context_len,
                                  int32_t partition_tokens);

/* --------------------------------------------------------------------------
 * Host block allocator.  [KVB] "PagedAttention and vLLM": pages are
 * allocated on demand and a finished request's pages return to the pool at
 * once.  [ENG]: a memory manager maps logical blocks to physical blocks; two
 * requests with the same prompt prefix share pages instead of duplicating.
 *
 * One handle manages one pool of num_blocks physical blocks (ids 0..NB-1)
 * and any number of sequences.  Free blocks sit on a LIFO free list; every
 * block carries a reference count (0 = free).  Not thread-safe: the caller
 * serialises calls on one handle.  All calls are host-only.
 * ------------------------------------------------------------------------ */
pkv_status pkv_alloc_create(int32_t num_blocks, int32_t block_size, void **handle);
void pkv_alloc_destroy(void *handle);

/* Pop a free block (refcount 0 -> 1).  PKV_ERR_OOM when none is free. */
pkv_status pkv_block_alloc(void *h, int32_t *block_out);
/* refcount += 1 on an allocated block (sharing it once more). */
pkv_status pkv_block_incref(void *h, int32_t block);
/* refcount -= 1; at 0 the block returns to the free list at once.
 * PKV_ERR_INVALID for a free block (double free). */
pkv_status pkv_block_decref(void *h, int32_t block);
int32_t pkv_num_free(void *h);
/* Reference count of a block, or -1 for an invalid id. */
int32_t pkv_refcount(void *h, int32_t block);

/* A new, empty sequence (context length 0, no blocks). */
pkv_status pkv_seq_create(void *h, int32_t *seq_out);
/* A new sequence that shares the parent's first num_full_blocks blocks
 * (each gets one more reference) and starts with context length
 * num_full_blocks * bs.  num_full_blocks * bs must not exceed the parent's
 * length.  Only whole blocks are shared, so the child's next append opens a
 * private block. */
pkv_status pkv_seq_fork(void *h, int32_t parent, int32_t num_full_blocks, int32_t *child_out);
/* Reserve the slot for the sequence's next token and return it
 * (block * bs + row); the context length grows by one.  Opens a new block
 * when the length is a multiple of bs (PKV_ERR_OOM if none is free).
 * PKV_ERR_SHARED_WRITE if the token would land in a shared block.  On any
 * error nothing changes. */
pkv_status pkv_seq_append_slot(void *h, int32_t seq, int64_t *slot_out);
/* pkv_seq_append_slot for n sequences at once, all or nothing: on an error
 * (including OOM for the batch as a whole) no sequence changes. */
pkv_status pkv_seq_append_slots(void *h, const int32_t *seqs, int32_t n, int64_t *slots_out);
/* Copy-on-write sharing (the plain reading of sharing pages between
 * requests that keep appending): a fork may share the parent's first
 * num_tokens positions including a partly filled last block (each shared
 * block gets one more reference); the child starts with context length
 * num_tokens. */
pkv_status pkv_seq_fork_tokens(void *h, int32_t parent, int64_t num_tokens, int32_t *child_out);
/* pkv_seq_append_slot, except that an append into a shared block first gives
 * the sequence a private copy: a fresh block replaces the shared one in its
 * table (the shared block loses one reference) and (*copy_src, *copy_dst)
 * name the block copy the caller must make on the device (pkv_copy_blocks)
 * before writing the token; both are -1 when no copy is needed.  OOM leaves
 * everything unchanged. */
pkv_status pkv_seq_append_slot_cow(void *h, int32_t seq, int64_t *slot_out, int32_t *copy_src,
                                   int32_t *copy_dst);
/* Batch form, all or nothing: copies_out[2*k], copies_out[2*k+1] receive the
 * k-th (src, dst) copy, *n_copies_out their number (at most n). */
pkv_status pkv_seq_append_slots_cow(void *h, const int32_t *seqs, int32_t n, int64_t *slots_out,
                                    int32_t *copies_out, int32_t *n_copies_out);

/* Drop the sequence: every block loses one reference; blocks reaching 0
 * return to the free list.  The id may be reused by a later create/fork. */
pkv_status pkv_seq_free(void *h, int32_t seq);
/* Copy the sequence's block ids (logical order) to dst[0 .. min(n, cap)). */
pkv_status pkv_seq_block_table(void *h, int32_t seq, int32_t *dst, int32_t cap, int32_t *n_out);
/* Current context length of the sequence, or -1 for an invalid id. */
int64_t pkv_seq_context_len(void *h, int32_t seq);
/* Fill a batch block table dst[n][cap] (rows padded with -1) and
 * context_lens[n] for the given sequences, ready to copy to the device. */
pkv_status pkv_batch_tables(void *h, const int32_t *seqs, int32_t n, int32_t *dst,
                            int32_t cap, int32_t *context_lens);

/* Sharing groups of a batch (host), for
 * pkv_append_decode_attention_shared_prefix: runs of consecutive sequences
 * of seqs[0..n) whose first block, where it is shared (refcount > 1), is one
 * and the same block; a sequence that shares nothing stays in the run around
 * it (a member with claim 0) rather than splitting it, since each group reads
 * its prefix once.  A sequence whose shared first block differs from the
 * run's opens a new group.  group_start[0 .. *num_groups] receives the groups
 * (capacity n + 1), shared_lens[i] the number of leading positions of seqs[i]
 * held in shared blocks (its leading blocks with refcount > 1, times bs). */
pkv_status pkv_batch_prefix_groups(void *h, const int32_t *seqs, int32_t n, int32_t *group_start,
                                   int32_t *num_groups, int32_t *shared_lens);

/* Testing hook for the kernels' bounded waits (no counterpart on the pages).
 * With enable != 0, decode launches made afterwards by this process issue no
 * tile copies, so every wait for a tile runs out after wait_limit_ns (clamped
 * to [1 ms, 2 s]); the kernel records the time-out and returns, and the CUDA
 * context stays usable.  pkv_get_last_error() then reports PKV_ERR_TIMEOUT.
 * enable == 0 restores normal operation (2 s limit).  Host-side setting only;
 * nothing faults, traps or hangs. */
pkv_status pkv_test_inject_wait_timeout(int32_t enable, int64_t wait_limit_ns);

/* Testing hook (no counterpart on the pages): y[i] = 2^x[i] computed the way
 * the multi-query kernel computes part of its softmax exponentials on the
 * FMA pipes (PKV_MQ_POLY=1): round-to-nearest range reduction and a degree-4
 * polynomial, relative error < 1e-5; 0 below -126.  x, y: device float [n]. */
pkv_status pkv_test_exp2_poly(const float *x, float *y, int64_t n, pkv_stream stream);

/* Text of the last CUDA runtime error a call of this thread reported as
 * PKV_ERR_CUDA ("no error" if none); static storage. */
const char *pkv_last_cuda_error(void);

/* --------------------------------------------------------------------------
 * Iteration-level scheduler (host only) over one allocator.
 * [KVB] "Continuous batching (Orca)": each token step is batched across all
 * in-flight requests; finished requests leave and new ones join at any step.
 * [KVB] "Chunked prefill": prompts are fed in fixed-size chunks interleaved
 * with decode steps.  [KVB] "The KV cache": running out of KV memory stalls
 * new requests or forces preemption of in-flight ones.
 *
 * Each pkv_sched_step plans one step: one decode token for every request
 * past its prompt (oldest first), then the next prefill chunk (<=
 * chunk_tokens) of requests still in their prompt, then new requests first
 * come first served -- within max_batch_tokens tokens and max_seqs
 * sequences.  When a request needs a block and none is free, the most
 * recently admitted other request is preempted by recompute (its blocks
 * return to the pool; it rejoins the front of the queue, is readmitted at
 * the next step at the earliest, and re-prefills its prompt and generated
 * tokens).  The step's slots come from the allocator,
 * so pkv_batch_tables(seq_ids) gives the matching block tables; run
 * pkv_append with the slots, then pkv_prefill_attention with query_lens as
 * the chunk lengths (a decode token is a chunk of one).  The step that
 * completes a request's context produces its next token; a request that
 * reached max_new_tokens is reported in finished_ids by the NEXT call, which
 * also frees its blocks (this step's kernels still read them).
 * ------------------------------------------------------------------------ */
typedef struct pkv_sched_config {
    int32_t max_batch_tokens;  /* tokens per step (decode tokens + prefill chunks) */
    int32_t max_seqs;          /* sequences per step and requests running at once */
    int32_t chunk_tokens;      /* prefill chunk size, e.g. 512 */
    int32_t block_size;        /* the allocator's block size */
} pkv_sched_config;

/* Caller-owned output arrays of one step; capacities: max_seqs entries for
 * the per-sequence arrays, max_batch_tokens for slots. */
typedef struct pkv_sched_batch {
    int32_t num_seqs, num_tokens, num_preempted, num_finished;
    int64_t *request_ids;   /* [max_seqs] */
    int32_t *seq_ids;       /* [max_seqs] allocator sequence ids */
    int32_t *query_lens;    /* [max_seqs] tokens of the sequence in this step */
    int32_t *context_lens;  /* [max_seqs] sequence length after this step */
    int64_t *slots;         /* [max_batch_tokens] new tokens' slots, sequence order */
    int64_t *finished_ids;  /* [max_seqs] */
    int64_t *preempted_ids; /* [max_seqs] */
} pkv_sched_batch;

pkv_status pkv_sched_create(void *alloc, const pkv_sched_config *cfg, void **sched);
void pkv_sched_destroy(void *sched);
/* Queue a request: prompt_len prompt tokens, then max_new_tokens outputs. */
pkv_status pkv_sched_add(void *sched, int64_t request_id, int32_t prompt_len, int32_t max_new_tokens);
pkv_status pkv_sched_step(void *sched, pkv_sched_batch *out);
int32_t pkv_sched_num_waiting(void *sched);
int32_t pkv_sched_num_running(void *sched);

/* Human-readable name of a status code (static storage). */
const char *pkv_status_string(pkv_status s);
/* Sticky error of the device checks, read and cleared.  Synchronises the
 * current device.  PKV_ERR_TIMEOUT if a kernel's bounded wait ran out,
 * PKV_ERR_DEVICE_CHECK if a kernel skipped an out-of-range access since the
 * last call, PKV_ERR_CUDA on a pending CUDA error, else PKV_OK. */
pkv_status pkv_get_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */

/*
 * ps.h -- prefix-sliding attention over a ring-buffer KV cache (C ABI).
 *
 * What it computes.  A query at absolute position t attends to the pinned
 * prefix [0, P_s) of its sequence plus the recent window
 * [max(P_s, t-W+1), t], and to nothing else ("Prefix Sliding" digest,
 * longzhangge.com PaperDaily, section 03; stated there 1-indexed as
 * [1,P] and [max(P+1, t-W+1), t]).  Each sequence's ring buffer holds exactly
 * the last W window entries of its history, slot i of the logical view holding
 * position base+i ("Formal verification of a sliding-window KV cache in
 * Lean4", pnsm.cn blog, sections 2.3-2.4 and 3.2-3.4).  Positions are absolute
 * and keep growing (the digest's section 05 "continue PE"); keys arrive
 * already position-encoded and are never re-encoded.
 *
 * Conventions for every call.
 *  - Tensor arguments are DEVICE pointers owned by the caller, contiguous,
 *    of the cache's element type (PS_F32: float, PS_BF16: bfloat16 bit
 *    patterns), 16-byte aligned.  Index and bookkeeping arguments marked
 *    "host" are host pointers read before the call returns.
 *  - Layouts are token-major: keys/values [tokens][Hkv][d], queries and
 *    outputs [tokens][Hq][d].  Query head h uses key/value head h / (Hq/Hkv).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous unless stated otherwise.  Calls that touch
 *    the same cache must be ordered on one stream (or by the caller's events).
 *  - Every argument, sequence state and position is validated on the host
 *    BEFORE anything is enqueued.  A call that returns an error other than
 *    PS_ECUDA has changed neither the device memory nor the host-side state;
 *    the message is available from ps_last_error() in the calling thread.
 *  - PS_ECUDA is the one partial outcome.  Some calls enqueue more than one
 *    launch: a paged ring's page-table update before an append, and one
 *    launch per 128 batch entries in ps_append_kv, ps_decode_step and
 *    ps_attend_decode (one append per entry in ps_attend_chunk_batch with
 *    append_after).  If a launch fails, the launches before it stay enqueued
 *    and the host-side state records exactly them: mapped pages stay mapped,
 *    the entries whose append was enqueued are advanced, the others are
 *    unchanged, and outputs of entries not yet launched are not written.  A
 *    failed launch usually leaves the CUDA context unusable in any case.
 *  - The library owns only the opaque host object.  All device storage lives
 *    in the caller's buffer passed to ps_cache_create; decode scratch lives in
 *    the caller's workspace passed to ps_attend_decode / ps_decode_step (or in
 *    the library's fixed array for ps_attend_decode_static).
 *  - Kernels never trap.  An internal inconsistency detected on the device sets
 *    an error word that ps_device_error() reads back.
 */
#ifndef PS_H
#define PS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PS_API __attribute__((visibility("default")))
#else
#define PS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PS_OK = 0,
  PS_EINVAL = -1,      /* bad argument (size, pointer, alignment, duplicate id) */
  PS_ENOMEM = -2,      /* caller's buffer or workspace too small */
  PS_EPOS = -3,        /* position does not follow the sequence's history */
  PS_ESTATE = -4,      /* sequence not in a state that allows the call */
  PS_ECUDA = -5,       /* a CUDA runtime call failed (message has the details) */
  PS_EUNSUPPORTED = -6 /* valid but unsupported configuration (e.g. head_dim) */
} ps_status;

typedef enum { PS_F32 = 0, PS_BF16 = 1 } ps_dtype;

typedef struct ps_cache ps_cache; /* opaque, library-owned host object */

/* Host-side view of one sequence (mirrors the device bookkeeping). */
typedef struct {
  int32_t state;     /* 0 = empty (after create/reset), 1 = active (prefix stored) */
  int32_t P;         /* pinned prefix length P_s */
  int64_t next_pos;  /* absolute position the next appended token gets */
  int32_t head;      /* ring slot of the oldest window entry */
  int32_t count;     /* window entries held, min(W, next_pos - P) */
} ps_seq_info;

/* ----------------------------------------------------------------- cache -- */

/* Bytes of device memory a cache with these parameters needs (0 if invalid).
 * W >= 1 window slots, P_max >= 0 prefix rows, Hkv >= 1 key/value heads,
 * d in {64, 128}, dtype a ps_dtype, max_seqs >= 1 sequences.  The K/V part is
 * the blog's section 1.1 size formula for one layer with the sequence length
 * bounded by the pinned prefix plus the window:
 * 2 * Hkv * d * (P_max + W) * max_seqs * sizeof(dtype), plus the per-slot
 * positions (8 bytes per ring slot) and 32 bytes of bookkeeping per sequence,
 * each region rounded up to 256 bytes. */
PS_API size_t ps_cache_bytes(int W, int P_max, int Hkv, int d, int dtype, int max_seqs);

/* Bind a cache to the caller's device buffer `dev_buf` (dev_bytes >=
 * ps_cache_bytes(...), 256-byte aligned, owned by the caller and kept alive
 * until ps_cache_destroy).  Every sequence starts empty with ring head 0.
 * Enqueues the initialisation of the bookkeeping area on `stream`.
 * Errors: PS_EINVAL, PS_EUNSUPPORTED, PS_ENOMEM, PS_ECUDA. */
PS_API int ps_cache_create(int W, int P_max, int Hkv, int d, int dtype, int max_seqs,
                    void* dev_buf, size_t dev_bytes, void* stream, ps_cache** out);

/* Paged ring (block-table indirection, vLLM-style): the same cache with each
 * sequence's W ring slots split into W / page_rows pages that live in a pool
 * of num_pages physical pages shared by all sequences, mapped through a page
 * table.  A page is taken from the pool when an append, decode step, chunk
 * append or window import first writes one of its slots, and returns to the
 * pool when the sequence is reset; so memory follows the tokens actually held
 * rather than max_seqs * W.  Every call behaves exactly as on an unpaged cache
 * (same results, bit for bit, when page_rows is a multiple of 8; with other
 * page sizes the bf16 decode groups a tile's rows page by page, which changes
 * the float32 summation order only), except that a write needing a page when
 * the pool is empty fails with PS_ENOMEM and changes nothing.  Requires
 * 1 <= page_rows <= W, W % page_rows == 0, num_pages >= 1; the tensor-core
 * chunk kernel takes page_rows that are multiples of 128 or that divide 128
 * and are multiples of 8 (8, 16, 32, 64); other page sizes use the CUDA-core
 * chunk kernel.  ps_cache_bytes_paged returns 0 for an invalid shape. */
PS_API size_t ps_cache_bytes_paged(int W, int P_max, int Hkv, int d, int dtype, int max_seqs,
                                   int page_rows, int num_pages);
PS_API int ps_cache_create_paged(int W, int P_max, int Hkv, int d, int dtype, int max_seqs,
                                 int page_rows, int num_pages, void* dev_buf, size_t dev_bytes,
                                 void* stream, ps_cache** out);

/* Physical ring pages left in the pool of a paged cache (host bookkeeping, no
 * device access).  Errors: PS_EINVAL (NULL or unpaged cache). */
PS_API int ps_ring_pages_free(const ps_cache* c);

/* Free the host object (the device buffer stays the caller's). NULL is a no-op. */
PS_API void ps_cache_destroy(ps_cache* c);

/* Return sequence `seq` to the empty state; its ring head starts at slot
 * ring_head_offset (0 <= offset < W).  Results do not depend on the offset
 * beyond float32 rounding order.
 * Errors: PS_EINVAL, PS_ESTATE (other sequences share this one's prefix). */
PS_API int ps_seq_reset(ps_cache* c, int seq, int ring_head_offset, void* stream);

/* Host mirror of a sequence's state (no device access). Errors: PS_EINVAL. */
PS_API int ps_seq_info_get(const ps_cache* c, int seq, ps_seq_info* out);

/* ---------------------------------------------------------- a1 prefix ---- */

/* Store the pinned prefix of an empty sequence: positions [0, P_s) with keys
 * and values k, v [P_s][Hkv][d] (device).  The prefix is never evicted
 * (digest section 03: KV_prefix = encode(prefix), kept for every step).
 * 0 <= P_s <= P_max.  The sequence becomes active with next_pos = P_s and an
 * empty window.  Errors: PS_EINVAL, PS_ESTATE (sequence not empty). */
PS_API int ps_prefill_prefix(ps_cache* c, int seq, const void* k, const void* v, int P_s,
                      void* stream);

/* Let empty sequence `seq` use the pinned prefix of active sequence `src`
 * instead of a copy of its own (prompt reuse, as in prefix caching): `seq`
 * becomes active with the same P_s, next_pos = P_s and an empty window, and
 * every kernel reads its prefix rows from the slab that holds src's prefix,
 * so sequences sharing a prompt stream its keys and values from HBM once per
 * L2 residency.  Results are exactly those of a private copy of the same rows.
 * While any sequence shares a prefix, the sequence holding it cannot be reset
 * (PS_ESTATE); resetting a sharer releases it.
 * Errors: PS_EINVAL, PS_ESTATE (seq not empty, or src has no prefix). */
PS_API int ps_share_prefix(ps_cache* c, int seq, int src, void* stream);

/* Attention of prompt tokens t0..t0+n-1 of active sequence `seq`, all inside
 * its pinned prefix (0 <= t0, t0 + n <= P_s), over the prefix rows stored by
 * ps_prefill_prefix: query t sees positions [0, t] (for t < P_s the
 * visibility rule is plain causal attention; digest section 03 encodes the
 * prefix once).  q: [n][Hq][d], out: [n][Hq][d] (device, cache dtype).  bf16
 * with head_dim 128 runs on the tcgen05 tensor-core kernel, other
 * configurations on the CUDA-core kernel.  The sequence's state is unchanged.
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS. */
PS_API int ps_attend_prompt(ps_cache* c, int seq, const void* q, int64_t t0, int n, int Hq,
                            float scale, void* out, void* stream);

/* Prompt attention of B sequences in one launch: entry b is as the call above
 * for sequence seq_ids[b] (host array of distinct active ids) with queries
 * t0[b]..t0[b]+n[b]-1 (host arrays; n[b] >= 0, 0 <= t0[b], t0[b]+n[b] <= P_s).
 * The entries' rows are packed end to end in entry order: q, out
 * [sum n][Hq][d] (device), entry b from row n[0]+...+n[b-1].  On the
 * tensor-core kernel the whole batch is one launch whose grid covers every
 * entry's query tiles, so one sequence's tail of work does not leave the GPU
 * partly idle.
 * Errors: as ps_attend_prompt, checked for every entry before anything runs. */
PS_API int ps_attend_prompt_batch(ps_cache* c, const int* seq_ids, const int64_t* t0,
                                  const int* n, int B, const void* q, int Hq, float scale,
                                  void* out, void* stream);

/* ---------------------------------------------------- a2 ring append ----- */

/* Append n tokens to each of B active sequences seq_ids[0..B) (host array of
 * distinct ids).  k, v: [B][n][Hkv][d] (device).  Token i of entry b gets
 * position next_pos(b) + i.  Each token is one step of the cache update
 * (blog section 3.3): while fewer than W entries are held it fills slot
 * (head + count) mod W; afterwards it overwrites the oldest slot `head` and
 * advances head.  n > W keeps only the last W tokens, exactly as n single
 * steps would.  Positions are stored per slot.  B == 0 or n == 0 is a no-op.
 * Errors: PS_EINVAL, PS_ESTATE. */
PS_API int ps_append_kv(ps_cache* c, const int* seq_ids, int B, const void* k, const void* v,
                 int n, void* stream);

/* -------------------------------------------- a3-a5 decode attention ----- */

/* Workspace bytes ps_attend_decode needs for a batch of B sequences with Hq
 * query heads (an upper bound independent of the positions). */
PS_API size_t ps_decode_workspace_bytes(const ps_cache* c, int B, int Hq);

/* One decode step of attention for B active sequences seq_ids[0..B) (host,
 * distinct) at positions t[0..B) (host), which must be the last appended
 * position of each sequence (t[b] == next_pos - 1, t[b] >= P_s: append the
 * token first, then attend, as the digest's section 03 loop does).
 * q: [B][Hq][d] (device), out: [B][Hq][d] (device, same dtype).
 * out[b][h] = sum over visible p of softmax_p(scale * <q[b][h], k_p>) v_p,
 * computed in float32 (bf16 inputs are widened exactly; the bf16 output is
 * rounded to nearest even).  Evicted positions are never read.
 * workspace: device, >= ps_decode_workspace_bytes(c, B, Hq) bytes, any
 * contents (it holds split partial results within one call, no state between
 * calls).  Calls that share a workspace must not overlap on the GPU.
 * The ring state (P, head, count) of each entry is taken from the library's
 * host bookkeeping at enqueue time; the kernel compares it with the device
 * record and sets the device error bit 4 (see ps_device_error) if they differ,
 * as happens when an append on another stream was not ordered before this call.
 * Hq must be a multiple of Hkv with Hq/Hkv in {1, 2, 4, 8}.
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS, PS_ENOMEM, PS_EUNSUPPORTED. */
PS_API int ps_attend_decode(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t,
                     int B, int Hq, float scale, void* out, void* workspace,
                     size_t workspace_bytes, void* stream);

/* One whole decode step for B active sequences seq_ids[0..B) (host, distinct):
 * append the token at t[b] == next_pos (k_new, v_new: [B][Hkv][d], device) to
 * each ring, evicting as ps_append_kv does, then attend at t[b] as
 * ps_attend_decode does (the digest's section 03 loop: append, then attend).
 * The appended row is read once, from k_new/v_new, for the attention and
 * written to its ring slot in the same pass; the ring contents, positions and
 * bookkeeping afterwards, and the output, are exactly those of ps_append_kv
 * (n = 1) followed by ps_attend_decode.  Requires t[b] >= P_s.
 * q, out, workspace, Hq, scale: as ps_attend_decode.
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS, PS_ENOMEM, PS_EUNSUPPORTED. */
PS_API int ps_decode_step(ps_cache* c, const void* q, const void* k_new, const void* v_new,
                          const int* seq_ids, const int64_t* t, int B, int Hq, float scale,
                          void* out, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------ decode for callers that cannot allocate --- */

/* ps_attend_decode without a workspace argument, for callers that cannot give
 * the library device memory: a host runtime that owns all device memory through
 * its own pool and offers plug-ins no allocation hook, or a latency-critical
 * loop where a cudaMalloc (which synchronises the device) is not acceptable.
 * The pages describe no such call; it exists for those callers only.
 * Same arguments, results and errors as ps_attend_decode, except that the
 * split-K scratch lives in a fixed 4 MiB array inside the library's device
 * image (held by every GPU that loads the library until the process exits).
 * It allocates nothing.  A batch whose scratch would exceed 4 MiB is rejected
 * with PS_ENOMEM.  Arguments and sequence states are checked first, as by
 * ps_attend_decode; B = 0 returns PS_OK with nothing set up or enqueued.  The
 * first call on each device (and the first after that device's context was
 * reset) looks up the array's device address; the look-up does not
 * synchronise, but it may make the runtime load the library's device code, so
 * make that first call before any stream capture.  Nothing in the array has
 * to start at zero: every call writes the scratch it reads.  All calls on a
 * device share the array, so calls that overlap on the GPU (other streams,
 * other threads) race; order them. */
PS_API int ps_attend_decode_static(ps_cache* c, const void* q, const int* seq_ids,
                                   const int64_t* t, int B, int Hq, float scale, void* out,
                                   void* stream);

/* ------------------------------------------- a6 chunked prefill/extend --- */

/* Attention for a block of n consecutive queries of active sequence `seq` at
 * positions [t0, t0+n), with t0 == next_pos (the block extends the history)
 * and t0 >= P_s.  q: [n][Hq][d]; k_blk, v_blk: [n][Hkv][d], the block's own
 * keys/values; out: [n][Hq][d] (all device).  Query t0+i sees the prefix, the
 * ring entries in its window and block tokens t0..t0+i (causal inside the
 * block): the digest's section 03 visibility rule applied to every query of
 * the block, evaluated as in its section 06 kernel -- key tiles walked over
 * the prefix range and the window range separately (the evicted middle is
 * never loaded) with an element mask only on tiles that straddle a window or
 * causal edge.  The ring must still hold [max(P_s, t0-W+1), t0-1], which is always
 * true before the block is appended.  If append_after != 0 the block is then
 * appended as by ps_append_kv (only its last W tokens survive in the ring).
 * bf16 with d = 128 and Hq/Hkv in {1, 2, 4, 8} runs on the tcgen05 tensor-core
 * kernel; other configurations use a CUDA-core kernel.  Small bf16 blocks
 * (d = 64 or 128) run instead on the decode kernel when the call qualifies
 * (ps_set_chunk_small_max): groups of 8 / (Hq/Hkv) queries, each group's
 * (query, head) pairs as the narrow side of the warp-level products, every
 * query masked to its own visible set, the key rows of a (group, kv head)
 * pair split over a cluster of CTAs.
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS, PS_EUNSUPPORTED. */
PS_API int ps_attend_chunk(ps_cache* c, int seq, const void* q, const void* k_blk,
                    const void* v_blk, int64_t t0, int n, int Hq, float scale, void* out,
                    int append_after, void* stream);

/* Small-block bound of the chunk calls (bf16 caches).  A ps_attend_chunk or
 * ps_attend_chunk_batch call runs on the split decode path when every block
 * of it has at most n_max queries and its (group of 8 / (Hq/Hkv) queries, kv
 * head) pairs all fit the GPU at once in clusters of two CTAs (148 on a B200:
 * e.g. 4 blocks of 16 queries at Hq/Hkv = 2, Hkv = 8); otherwise the whole
 * call runs on the chunk kernels.  Inside those limits the split path was
 * measured faster at every block size (W = 4096, one and four sequences); 0
 * sends every call to the chunk kernels.  The split path's partition, and so
 * its float32 summation order, follows the call's size, as the decode calls'
 * does.  Default 64.
 * Errors: PS_EINVAL (NULL cache, n_max < 0). */
PS_API int ps_set_chunk_small_max(ps_cache* c, int n_max);

/* Chunked prefill/extend of B sequences in one launch (batched serving):
 * entry b is as ps_attend_chunk for sequence seq_ids[b] (host array of
 * distinct active ids) with a block of n[b] >= 0 queries at t0[b] == its
 * next_pos (host arrays).  The entries' rows are packed end to end in entry
 * order: q, out [sum n][Hq][d]; k_blk, v_blk [sum n][Hkv][d] (device), entry
 * b from row n[0]+...+n[b-1].  With append_after != 0 every entry's block is
 * then appended to its ring.  On the tensor-core kernel the whole batch is one
 * launch with one CTA per (query tile, kv head) of every entry.
 * Errors: as ps_attend_chunk, checked for every entry (and, for a paged cache,
 * the pages of all appends planned) before anything runs; PS_ENOMEM if the
 * page pool cannot take all the appends. */
PS_API int ps_attend_chunk_batch(ps_cache* c, const int* seq_ids, const int64_t* t0, const int* n,
                                 int B, const void* q, const void* k_blk, const void* v_blk,
                                 int Hq, float scale, void* out, int append_after, void* stream);

/* ------------------------------------------- checkpoint / debug export --- */

/* Export the window of active sequence `seq` in logical order (oldest first,
 * blog section 3.4 ringToList over the `count` held entries):
 * k, v: [W][Hkv][d] (device; rows [0,count) written), pos: [W] int64 (device),
 * count_out: one int32 (device).  Errors: PS_EINVAL, PS_ESTATE. */
PS_API int ps_export_window(ps_cache* c, int seq, void* k, void* v, int64_t* pos,
                     int32_t* count_out, void* stream);

/* Set the window of active sequence `seq` as if positions [P_s, next_pos)
 * had been appended: k, v: [n][Hkv][d] (device) hold positions
 * [next_pos-n, next_pos) oldest first, n == min(W, next_pos - P_s), and the
 * oldest lands in ring slot ring_head_offset (0 <= offset < W).
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS. */
PS_API int ps_import_window(ps_cache* c, int seq, int64_t next_pos, const void* k, const void* v,
                     int n, int ring_head_offset, void* stream);

/* The positions the attention kernels read for a query of sequence `seq` at
 * position t (t >= P_s), in the order they are visited: prefix rows, then the
 * ring segments, then (for t >= next_pos, a chunk query) block positions
 * next_pos..t.  Ring rows report the position stored in their slot.
 * pos_out: device int64 with room for P_s + W entries; n_out: one int32
 * (device).  Requires the ring to cover the window part below next_pos.
 * Errors: PS_EINVAL, PS_ESTATE, PS_EPOS. */
PS_API int ps_debug_visible(ps_cache* c, int seq, int64_t t, int64_t* pos_out, int32_t* n_out,
                     void* stream);

/* Test hook for the bounded waits of every kernel pipeline: one GPU thread
 * waits on a barrier that nothing ever arrives at, gives up after about
 * limit_cycles SM clock cycles (1 <= limit_cycles <= 2^31, about a second at
 * most) with the same helper the kernels use, and sets bit 8 (time-out) of
 * the device error word.  No memory but that word is touched and the context
 * stays usable.  Errors: PS_EINVAL. */
PS_API int ps_debug_wait_timeout(ps_cache* c, long long limit_cycles, void* stream);

/* Synchronise `stream` and read (then clear) the device error word:
 * *code = 0 when no kernel reported an inconsistency, else an OR of
 *   2  a ring no longer holds the window a query needs,
 *   4  a batch entry's position or ring state disagrees with the device record,
 *   8  a pipeline wait gave up and the kernel stopped early (outputs of that
 *      call are undefined).
 * Errors: PS_ECUDA. */
PS_API int ps_device_error(ps_cache* c, int32_t* code, void* stream);

/* Message of the last failed call in this thread ("" if none). */
PS_API const char* ps_last_error(void);

/* Library version string. */
PS_API const char* ps_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PS_H */

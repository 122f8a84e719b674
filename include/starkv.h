/*
 * starkv.h -- C ABI of the STAR-KV paged low-rank decode library (sm_100a).
 *
 * STAR-KV stores, per layer, a low-rank projection of the K/V cache instead of
 * the full-dimension cache: head-wise for K and joint across heads for V,
 * kept in a compressed paged format (Proxima README, "Low-rank KV Cache
 * Compression for vLLM", opening method paragraph; tenosra.com/proxima, first
 * paragraph).  This library implements the steps that read and write that
 * cache on the GPU:
 *
 *   compress-and-append : codes of each sequence's new token written into the
 *                         paged pools (and compress-store: many rows at
 *                         explicit slots, e.g. a prompt chunk);
 *   paged decode        : single-query attention computed straight from the
 *                         codes, never materialising full keys or values;
 *   chunked prefill     : causal attention of prompt chunks over the codes;
 * plus host helpers for rank selection and cache capacity.
 *
 * Formulation (head_dim d, H query heads, Hkv KV heads with query head h
 * reading KV head g(h) = h / (H/Hkv), K rank r per KV head, V joint rank R):
 *   c_K[j] = k_j . A_K[j]         A_K[j] : d x r          (head-wise K, j < Hkv)
 *   c_V    = v . A_V              A_V    : (Hkv*d) x R    (joint V, v = concat_j v_j)
 *   q~_h   = scale * q_h . B_K[g(h)]^T,  B_K[j] : r x d   (query absorbed into K codes)
 *   s[h,t] = q~_h . c_K[t,g(h)]
 *   p[h,:] = softmax_t(s[h,:])
 *   out_h  = (sum_t p[h,t] c_V[t]) . B_V[:, g(h)*d:(g(h)+1)*d],  B_V : R x (Hkv*d)
 * which equals softmax attention over the decompressed keys k^_h = c_K[h].B_K[h]
 * and values v^ = c_V.B_V.
 *
 * Paged format: pages of block_size = 16 tokens (README, KV-cache block
 * paragraph: block size 16); token t of sequence b is in slot t % 16 of
 * physical page block_tables[b][t / 16] (PagedAttention block-level
 * management, botdigit.com explainer, "How Dynamic KV-Cache Compaction Works").
 * Layouts (row-major, fp16): K pool [num_blocks][16][Hkv][r];
 *                            V pool [num_blocks][16][R].
 * With Hkv = H this is multi-head attention; the pages' benchmark (32-head MHA)
 * is that case.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no memory and keeps no state between calls.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; a call returning STARKV_OK means the
 *    launches were accepted, not that they finished.
 *  - Argument and shape problems are reported synchronously, before any launch,
 *    and leave all buffers untouched.  Launch failures return STARKV_ERR_CUDA.
 *  - Device code never traps.  Data problems the host cannot see (a block id
 *    outside [0, num_blocks), a length above the table's capacity, a timed-out
 *    internal wait) set bits of a device status word that
 *    starkv_decode_check() reads back; the affected output is undefined.
 *  - The library keeps no state between calls, except the process-wide test
 *    hook set by starkv_set_wait_test_hook() (off unless a test sets it).
 */
#ifndef STARKV_H_
#define STARKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  STARKV_OK = 0,
  STARKV_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad scale */
  STARKV_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement */
  STARKV_ERR_WORKSPACE = 3,    /* workspace null or smaller than required */
  STARKV_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  STARKV_ERR_DEVICE_CHECK = 5, /* device status word reported a data problem */
  STARKV_ERR_TIMEOUT = 6       /* an internal device wait ran out of time */
} starkv_status;

/* Device status word bits (starkv_decode_check). */
#define STARKV_FLAG_BAD_BLOCK_ID 0x1  /* block id outside [0, num_blocks) */
#define STARKV_FLAG_BAD_SEQ_LEN 0x2   /* seq_len < 0 or > max_blocks_per_seq*16 or > max_seq_len */
#define STARKV_FLAG_TIMEOUT 0x4       /* a pipeline wait exceeded its bound */
/* Bits 8..15 accompany STARKV_FLAG_TIMEOUT and name the internal wait(s) that
 * ran out (diagnostic only; the numbering is not part of the stable ABI). */

/* One layer's cache geometry.  Ranks may differ from layer to layer. */
typedef struct {
  int32_t num_heads;          /* H: query heads, 1..64, power of two */
  int32_t head_dim;           /* d: 32, 64, 128 or 256 */
  int32_t k_rank;             /* r: multiple of 16, 16..256 */
  int32_t v_rank;             /* R: multiple of 64, 64..8192 */
  int32_t block_size;         /* must be 16 */
  int32_t num_blocks;         /* pages in each pool */
  int32_t max_blocks_per_seq; /* row length of block_tables */
  int32_t num_kv_heads;       /* Hkv: KV heads (grouped-query attention), a power of two
                                 dividing H; 0 means Hkv = H (multi-head attention).
                                 Query head h uses KV head h / (H / Hkv). */
} starkv_layer_desc;

/*
 * starkv_compress_append -- write the codes of one new token per sequence.
 *
 * Computes c_K[b,h,:] = k[b,h,:] . A_K[h] and c_V[b,:] = v[b,:] . A_V with fp32
 * accumulation, rounds them to fp16 (round to nearest even) and stores them in
 * slot positions[b] % 16 of page block_tables[b][positions[b] / 16] of the K
 * and V pools.  Nothing else in the pools is written.
 *
 *   k, v          fp16 [batch][Hkv][d]  (v read as the concatenation [batch][Hkv*d])
 *   A_K           fp16 [Hkv][d][r]
 *   A_V           fp16 [Hkv*d][R]
 *   block_tables  int32 [batch][max_blocks_per_seq]
 *   positions     int32 [batch]: the sequence length BEFORE this append
 *   k_cache       fp16 [num_blocks][16][Hkv][r]   (in/out)
 *   v_cache       fp16 [num_blocks][16][R]      (in/out)
 *   status        optional device int32 (NULL: not reported), 4-byte aligned:
 *                 every skipped target OR-s a flag into it --
 *                 STARKV_FLAG_BAD_SEQ_LEN for a position outside [0,
 *                 max_blocks_per_seq*16), STARKV_FLAG_BAD_BLOCK_ID for a block
 *                 id outside [0, num_blocks).  The library never clears it:
 *                 zero it before the calls it should cover, then read it with
 *                 starkv_decode_check(status, ...).
 *
 * Targets must be distinct slots (no page shared between sequences).  A target
 * whose position or block id is out of range is skipped (and flagged in
 * `status`).  batch == 0 is a no-op.  Cites: README method paragraph ("stored
 * in a compressed paged format").
 */
starkv_status starkv_compress_append(const starkv_layer_desc* desc, int32_t batch, const void* k,
                                     const void* v, const void* A_K, const void* A_V,
                                     const int32_t* block_tables, const int32_t* positions,
                                     void* k_cache, void* v_cache, int32_t* status, void* stream);

/*
 * starkv_compress_store -- compress n_tokens rows of k, v (for instance a
 * prompt at prefill) and store each row's codes at an explicit flat slot:
 * slot_mapping[i] = page * 16 + offset, int32 [n_tokens].  Same arithmetic,
 * layouts and rounding as starkv_compress_append; rows whose slot is outside
 * [0, num_blocks*16) are skipped and, when `status` is non-NULL, flagged with
 * STARKV_FLAG_BAD_BLOCK_ID (same convention as starkv_compress_append);
 * targets must be distinct.  k, v fp16 [n_tokens][Hkv][d].  Cites: README
 * method paragraph (codes "stored in a compressed paged format"); the flat
 * slot is the paged address block_table[b][t/16]*16 + t%16 precomputed by
 * the caller.
 */
starkv_status starkv_compress_store(const starkv_layer_desc* desc, int32_t n_tokens, const void* k,
                                    const void* v, const void* A_K, const void* A_V,
                                    const int32_t* slot_mapping, void* k_cache, void* v_cache,
                                    int32_t* status, void* stream);

/*
 * starkv_decode_workspace_bytes -- device scratch needed by starkv_paged_decode
 * for this layer geometry, batch size and length bound (0 on invalid input).
 * Depends on the SM count of the current device.
 */
size_t starkv_decode_workspace_bytes(const starkv_layer_desc* desc, int32_t batch,
                                     int32_t max_seq_len);

/*
 * starkv_paged_decode -- single-token decode attention from the paged codes.
 *
 *   q             fp16 [batch][H][d]
 *   B_K           fp16 [Hkv][r][d]
 *   B_V           fp16 [R][Hkv*d]
 *   k_cache       fp16 [num_blocks][16][Hkv][r]
 *   v_cache       fp16 [num_blocks][16][R]
 *   block_tables  int32 [batch][max_blocks_per_seq]
 *   seq_lens      int32 [batch]: tokens to attend over (after any append)
 *   max_seq_len   host-side upper bound of every seq_lens[b]
 *                 (<= max_blocks_per_seq*16); sizes grids and scratch
 *   scale         softmax scale (normally 1/sqrt(head_dim)); finite, > 0
 *   workspace     device scratch of at least starkv_decode_workspace_bytes()
 *                 bytes, 256-byte aligned; contents on entry are ignored
 *   out           fp16 [batch][H][d]
 *
 * Slots at or past seq_lens[b] are never read.  seq_lens[b] == 0 gives a zero
 * output row.  Accumulation is fp32; attention weights enter the V contraction
 * as fp16.  Calls that share a workspace must be ordered on one stream.
 */
starkv_status starkv_paged_decode(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                  const void* q, const void* B_K, const void* B_V,
                                  const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, const int32_t* seq_lens, float scale,
                                  void* workspace, size_t workspace_bytes, void* out, void* stream);

/*
 * starkv_append_decode -- one decode step of a layer: starkv_compress_append of
 * the new token of every sequence, then starkv_paged_decode over the updated
 * cache, with the same results as those two calls in that order (the cache
 * write comes before the attention that reads it, as in a serving engine's
 * decode step).  The new tokens' K/V codes and the query absorption run in
 * one launch, which saves two kernel boundaries per step.
 *
 *   k, v, A_K, A_V, positions, append_status   as in starkv_compress_append
 *   q, B_K, B_V, block_tables, seq_lens, scale,
 *   max_seq_len, workspace, out                 as in starkv_paged_decode
 *   k_cache, v_cache                            written by the append, then read
 *
 * seq_lens are the lengths after the append (normally positions + 1).
 * Errors as the two calls; nothing is launched when either set of arguments
 * is invalid.  Cites: README method paragraph (codes written into the
 * compressed paged cache and read by dedicated decode kernels).
 */
starkv_status starkv_append_decode(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                   const void* k, const void* v, const void* A_K, const void* A_V,
                                   const int32_t* positions, const void* q, const void* B_K,
                                   const void* B_V, void* k_cache, void* v_cache,
                                   const int32_t* block_tables, const int32_t* seq_lens, float scale,
                                   void* workspace, size_t workspace_bytes, void* out,
                                   int32_t* append_status, void* stream);

/*
 * starkv_append_decode_host -- starkv_append_decode for a caller whose step
 * inputs are in HOST memory (pinned memory lets the copies overlap): the new
 * tokens' k, v, their positions, the queries, the block tables and the
 * lengths are copied to `staging` (caller-owned DEVICE memory of at least
 * starkv_host_staging_bytes(desc, batch) bytes, 256-byte aligned) with one
 * cudaMemcpyAsync each on `stream`, the step runs there, and `out` is copied
 * back to the HOST array out_host (fp16 [batch][H][d]).  Everything is
 * enqueued asynchronously: out_host is valid after the stream synchronises.
 * The projections, pools and workspace are device memory as in
 * starkv_append_decode; argument errors return before anything is enqueued.
 * (Same method passage as starkv_append_decode.)
 */
size_t starkv_host_staging_bytes(const starkv_layer_desc* desc, int32_t batch);
starkv_status starkv_append_decode_host(const starkv_layer_desc* desc, int32_t batch, int32_t max_seq_len,
                                        const void* k_host, const void* v_host,
                                        const int32_t* positions_host, const void* q_host,
                                        const int32_t* block_tables_host, const int32_t* seq_lens_host,
                                        const void* A_K, const void* A_V, const void* B_K,
                                        const void* B_V, void* k_cache, void* v_cache, float scale,
                                        void* staging, size_t staging_bytes, void* workspace,
                                        size_t workspace_bytes, void* out_host, int32_t* append_status,
                                        void* stream);

/*
 * starkv_paged_prefill -- causal attention of prefill chunks over the paged
 * codes (chunked prefill).  The step that precedes decode: a prompt is
 * compressed into the cache chunk by chunk (starkv_compress_store) and each
 * chunk's queries attend over everything cached so far plus their own chunk.
 * The README describes STAR-KV as served by dedicated kernels over the
 * compressed pages ("Low-rank KV Cache Compression for vLLM", method
 * paragraph); no formula is given, so this is causal softmax attention with
 * the decode formulation above: query token i of sequence b (row
 * row_offsets[b] + i) attends over the tokens 0 .. starts[b] + i of b, whose
 * codes (the chunk's own included) must already be in the cache.
 *
 *   n_seqs        sequences with a chunk in this call
 *   n_rows        query tokens in total = row_offsets[n_seqs] (host value)
 *   max_seq_len   host-side upper bound of starts[b] + chunk length
 *   q             fp16 [n_rows][H][d], the chunks back to back
 *   block_tables  int32 [n_seqs][max_blocks_per_seq]
 *   starts        int32 [n_seqs] (device): position of each chunk's first token
 *   row_offsets   int32 [n_seqs + 1] (device): first row of each chunk,
 *                 non-decreasing from 0 to n_rows
 *   workspace     at least starkv_prefill_workspace_bytes(desc, n_seqs, n_rows,
 *                 max_seq_len) bytes, 256-byte aligned
 *   out           fp16 [n_rows][H][d]
 *
 * When the KV heads come in groups of 8 and G = H / Hkv <= 16, a chunk's rows
 * are taken nq at a time (nq = 16 for G <= 4, 64 / G above), and each group of
 * nq rows streams the sequence's K and V pages once for all of its rows (the
 * rows' query heads act as nq x H query heads with per-row causal limits): a
 * chunk of up to 16 rows reads every page once when G <= 4.  Other shapes
 * evaluate every row as one decode row (its own length, the sequence's block
 * table), reading the pages once per row.  The workspace holds the logits and
 * fp16 weights of every virtual head: it grows with (n_rows / nq + n_seqs) x
 * max_seq_len x H x nq.  Errors as starkv_paged_decode.
 */
size_t starkv_prefill_workspace_bytes(const starkv_layer_desc* desc, int32_t n_seqs, int32_t n_rows,
                                      int32_t max_seq_len);
starkv_status starkv_paged_prefill(const starkv_layer_desc* desc, int32_t n_seqs, int32_t n_rows,
                                   int32_t max_seq_len, const void* q, const void* B_K, const void* B_V,
                                   const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                   const int32_t* starts, const int32_t* row_offsets, float scale,
                                   void* workspace, size_t workspace_bytes, void* out, void* stream);

/*
 * starkv_paged_decode_profiled -- starkv_paged_decode that also records CUDA
 * events on `stream` around its kernels, for per-kernel timing.
 * stage_events: HOST array of 5 cudaEvent_t (as void*; a NULL entry is
 * skipped) recorded before the query absorption, after it, after the K pass,
 * after the V pass (which includes the split reduction of the maxima) and
 * after the finish kernel (the split reduction of Z / L and the
 * up-projection).  Events between the kernels keep
 * them from overlapping their launches, so this variant can be slightly slower
 * than starkv_paged_decode.  The events are not recorded when the call returns
 * an error before launching or when max_seq_len == 0.  Otherwise identical to
 * starkv_paged_decode.
 */
starkv_status starkv_paged_decode_profiled(const starkv_layer_desc* desc, int32_t batch,
                                           int32_t max_seq_len, const void* q, const void* B_K,
                                           const void* B_V, const void* k_cache, const void* v_cache,
                                           const int32_t* block_tables, const int32_t* seq_lens,
                                           float scale, void* workspace, size_t workspace_bytes,
                                           void* out, void* stream, void* const* stage_events);

/*
 * starkv_paged_decode_static -- starkv_paged_decode for callers that cannot
 * allocate device memory at decode time: an engine that has already handed
 * nearly all GPU memory to its paged KV pool, or a C host with no allocator to
 * provide scratch.  Same arguments and results as starkv_paged_decode minus
 * the workspace: the scratch is a fixed 64 MiB device array inside the library
 * (held by every GPU that loads the library until the process exits).  This
 * call allocates nothing.
 *  - Problems whose starkv_decode_workspace_bytes() exceeds 64 MiB are
 *    rejected with STARKV_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture.
 *  - All calls share the one array per device: calls that overlap on the GPU
 *    (different streams, or concurrent host threads on one device) race and
 *    give undefined results.  Calls ordered on one stream are safe.
 *  - The device status word is not exposed for this variant.
 * The method pages have no counterpart to this entry point.
 */
starkv_status starkv_paged_decode_static(const starkv_layer_desc* desc, int32_t batch,
                                         int32_t max_seq_len, const void* q, const void* B_K,
                                         const void* B_V, const void* k_cache, const void* v_cache,
                                         const int32_t* block_tables, const int32_t* seq_lens,
                                         float scale, void* out, void* stream);

/*
 * starkv_decode_check -- synchronise `stream` and read the device status word
 * at `workspace` (the first int32 of a decode or prefill workspace, or an
 * append `status` word).  For a workspace it is the status of the last decode
 * or prefill call that returned STARKV_OK with that workspace, calls with
 * nothing to compute (batch 0, max_seq_len 0, n_rows 0) included: those clear
 * the word.  *flags_out receives STARKV_FLAG_* bits (0 when clean).  Returns
 * STARKV_OK when clean, STARKV_ERR_TIMEOUT when the timeout bit is set,
 * STARKV_ERR_DEVICE_CHECK for other bits.
 */
starkv_status starkv_decode_check(const void* workspace, void* stream, int32_t* flags_out);

/*
 * starkv_set_wait_test_hook -- TEST HOOK for the failure path of the device
 * pipelines; leave it off in production.  Every internal pipeline wait is
 * bounded (about two seconds by default) and, when the bound runs out, sets
 * STARKV_FLAG_TIMEOUT plus a site bit and leaves its loop instead of hanging.
 * To exercise that path without faulting anything, a test can
 *   wait_limit_us  shorten the bound of every wait to this many microseconds on
 *                  the CURRENT device (0 restores the default), and
 *   drop_k_stage   make the K pass of every later decode skip the copy of its
 *                  ring stage number drop_k_stage in every CTA (-1: off), so
 *                  that the waits on that stage run out while no copy is in
 *                  flight.
 * Process-wide state; not to be changed while decodes are in flight.  Returns
 * STARKV_ERR_INVALID_ARG for drop_k_stage < -1 and STARKV_ERR_CUDA when the
 * device bound cannot be set.  The method pages have no counterpart to this
 * entry point.
 */
starkv_status starkv_set_wait_test_hook(uint32_t wait_limit_us, int32_t drop_k_stage);

/*
 * Workspace layout (byte offsets into the decode workspace), exposed so that
 * tests can inspect intermediate results.  Values for one (desc, batch,
 * max_seq_len) on the current device.
 */
typedef struct {
  size_t total_bytes;
  size_t status_off;  /* int32 status word; status_off + 64: uint32 counter of the page chunks the K
                         pass has handed out (set to 0 by the query absorption of every call) */
  size_t prefix_off;  /* int32 [batch+1] prefix sums of pages per sequence */
  size_t qt_off;      /* fp32 [batch][H][r]: log2(e)*scale*q.B_K^T */
  size_t logits_off;  /* fp32 [batch][t_pad][H]: base-2 logits s*log2(e) */
  size_t mpart_off;   /* fp32 [k_slots][H]: max of each sequence's base-2 logits */
  size_t lpart_off;   /* fp32 [v_slots][H]: per segment, sum of the fp16 weights exp2(s - max) */
  size_t zpart_off;   /* fp32 [n_rranges][H][v_slots][r_range]: per segment, sum_t w c_V */
  int32_t t_pad;      /* logits row capacity (multiple of 16) */
  int32_t k_ctas;     /* CTAs of the K pass (they take page chunks from the counter) */
  int32_t k_slots;    /* batch: one maximum slot per sequence */
  int32_t v_ctas;     /* CTAs of the V pass per R range */
  int32_t v_slots;    /* v_ctas + batch */
  int32_t n_rranges;  /* R ranges of the V pass */
  int32_t r_range;    /* V rank handled per R range */
  int32_t k_tensor;   /* 1: the K pass runs on tensor cores (grouped queries), 0: CUDA cores */
  size_t qth_off;     /* fp16 [batch][2H][r]: q~ in fp16 (rows h) and its remainder (rows H+h);
                         used by the tensor-core K pass only (0 otherwise) */
} starkv_workspace_layout;

starkv_status starkv_decode_workspace_layout(const starkv_layer_desc* desc, int32_t batch,
                                             int32_t max_seq_len, starkv_workspace_layout* out);

/* Human-readable name of a status code (static storage). */
const char* starkv_status_string(starkv_status status);

/*
 * starkv_rank_from_spectrum -- adaptive rank by soft-thresholding: the number
 * of singular values strictly greater than tau ("learned soft-thresholding for
 * adaptive rank control", README opening line).  Host function; s is a HOST
 * array of n doubles (n >= 0, s may be NULL when n == 0).  Returns -1 on
 * invalid input.
 */
int32_t starkv_rank_from_spectrum(const double* s, int32_t n, double tau);

/*
 * Capacity arithmetic (host functions, no GPU).  A token costs, in every layer,
 * Hkv*r fp16 K codes plus R fp16 V codes (Hkv = the layer's KV heads, equal to
 * its query heads without grouping); a full-rank cache is the case r = d,
 * R = Hkv*d (2*2*Hkv*d bytes per layer).  The README's boot log for the
 * uncompressed 7B cache is the worked example: 6.99 GiB of KV memory, 16-token
 * blocks, 32 layers x 512 KiB -> 894 blocks = 14,304 tokens ("Low-rank KV
 * Cache Compression for vLLM", measured results at 8192 context).
 *
 * starkv_kv_bytes_per_token: 2 * sum_l (num_heads[l]*k_ranks[l] + v_ranks[l]),
 *   num_heads[l] being layer l's KV heads;
 *   HOST arrays of n_layers entries; -1 on invalid input (n_layers <= 0, null
 *   array, non-positive entry).
 * starkv_num_blocks: floor(budget_bytes / (block_size * bytes_per_token));
 *   -1 on invalid input (negative budget, non-positive sizes).
 */
int64_t starkv_kv_bytes_per_token(int32_t n_layers, const int32_t* num_heads,
                                  const int32_t* k_ranks, const int32_t* v_ranks);
int64_t starkv_num_blocks(int64_t budget_bytes, int64_t bytes_per_token, int32_t block_size);

/* Library version, 10000*major + 100*minor + patch. */
int32_t starkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STARKV_H_ */

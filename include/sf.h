/*
 * sf.h -- selective precision streaming for low-bit LLM decoding (StrataFlux),
 * the data-parallel hot path, as a C ABI.
 *
 * The method ("StrataFlux: Memory-Hierarchy-Native Low-Bit LLM Inference",
 * arXiv 2611.08363, abstract; rag-lover.com explainer, sections TL;DR and
 * 解説) keeps low-bit weights and KV resident on the GPU and streams only the
 * extra low-order bits ("nested refinement") of the weight columns with the
 * largest input activations and of the tokens with the largest attention
 * weight as seen through the low-bit keys.  Fetched refinements are cached
 * on the GPU and reused across decode steps; misses come from pinned host
 * memory on a side stream, overlapped with compute.
 *
 * Conventions for every entry point
 *  - Returns sf_status; SF_OK is 0.  On any other value nothing was enqueued
 *    and sf_last_error() gives a message for the calling thread.  No C++
 *    exception crosses this boundary.
 *  - Device buffers are owned by the caller, stay owned by the caller, and
 *    must stay valid until the work enqueued on the given stream completes.
 *    Handles (sf_refine_cache) own their internals and free them in *_destroy.
 *  - Work is asynchronous on the given CUDA stream (NULL = legacy default
 *    stream) unless stated otherwise.  Shapes are checked on the host;
 *    data-dependent errors found on the device are reported through device
 *    outputs as stated per call.
 *  - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *  - Packed codes are little-endian bitstreams in uint32 words: a stream's
 *    bit t is bit (t mod 32) of word t/32, and code j of a b-bit stream
 *    occupies stream bits [b*j, b*j + b).
 */
#ifndef SF_H
#define SF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sf_stream_t; /* a cudaStream_t */

typedef enum sf_status {
  SF_OK = 0,
  SF_EINVAL = 1,    /* an argument or shape is outside the contract */
  SF_ENOMEM = 2,    /* a library-owned allocation failed */
  SF_ECUDA = 3,     /* a CUDA runtime call failed (message has the CUDA error) */
  SF_ETIMEOUT = 4,  /* a bounded wait expired */
  SF_ENOTIMPL = 5   /* combination not implemented */
} sf_status;

/* Refinement-code layouts of sf_quantize_nested. */
#define SF_REF_BY_COLUMN 0 /* weights: ref [K][N*b_f/32], one column per row of words */
#define SF_REF_BY_ROW 1    /* KV:      ref [N][K*b_f/32], same layout as resident codes */

/* Library version string (static storage). */
const char* sf_version(void);

/* Name of a status code (static storage). */
const char* sf_status_string(sf_status s);

/* Copy the calling thread's last error message into buf (always
 * NUL-terminated when len > 0).  Returns the full message length. */
size_t sf_last_error(char* buf, size_t len);

/*
 * sf_quantize_nested -- nested min-max quantization of a row-major fp32
 * matrix W[N][K] with groups of G consecutive inputs along K.
 *
 * Source: nested refinement, rag-lover.com explainer (解説): the fetched bits
 * subdivide between resident levels; bit widths from the arXiv abstract.
 * Definition (the pages give no formula; this is the reading the library
 * fixes, identical to the oracle's):
 *   lo, hi = min, max of the group (fp32);
 *   s = fp16_RNE(min(fp32((hi - lo) / (2^b - 1)), 65504)), s = 1 if it is 0;
 *   z = clamp(rint(-lo / s), 0, 2^b - 1)  (fp32 division, ties to even);
 *   q = clamp(rint(w / s) + z, 0, 2^b - 1), b = b_r + b_f;
 *   resident code q >> b_f, refinement code q & (2^b_f - 1).
 * Outputs (device, caller-allocated):
 *   res_codes  uint32 [N][K*b_r/32], row i = bitstream of its K resident codes;
 *   ref_codes  layout SF_REF_BY_COLUMN: uint32 [K][N*b_f/32], row j = bitstream
 *              of column j's N refinement codes (one column = one contiguous
 *              transfer unit); SF_REF_BY_ROW: uint32 [N][K*b_f/32];
 *   scale,zero fp16 [K/G][N] (zero is an exact small integer, +0 for zero).
 * Constraints: b_r in {2,3}, b_f in {1,2}, b_r + b_f <= 4, G % 32 == 0,
 *   K % G == 0, N >= 1; SF_REF_BY_COLUMN also needs N % 32 == 0.
 *   W must be finite (non-finite input gives unspecified codes).
 */
sf_status sf_quantize_nested(const float* W, int N, int K, int G, int b_r, int b_f, int layout,
                             uint32_t* res_codes, uint32_t* ref_codes, uint16_t* scale,
                             uint16_t* zero, sf_stream_t stream);

/*
 * sf_select_topk -- channel selection by activation magnitude.
 *
 * Source: rag-lover.com explainer (解説): weights are refined where the input
 * activation is large.  Per batch row the k channels with the largest |x|
 * (exact bf16 magnitudes, +0 == -0) are chosen, ties to the lower channel
 * index; the result is the union over the B rows in ascending order.
 *   x       device bf16 [B][K];
 *   idx_out device int32, capacity B*k, receives the ascending union;
 *   n_out   device int32 scalar, receives its length, or -1 if x holds a
 *           NaN or Inf (idx_out is then unspecified).
 * Constraints: 1 <= B <= 16, 1 <= K <= 65536, 0 <= k <= K.
 */
sf_status sf_select_topk(const uint16_t* x, int B, int K, int k, int32_t* idx_out,
                         int32_t* n_out, sf_stream_t stream);

/* A quantized weight matrix as produced by sf_quantize_nested (views, not
 * owned).  ref may be NULL; when non-NULL it is the complete refinement store
 * [K][N*b_f/32] resident in device memory. */
typedef struct sf_qweight {
  const uint32_t* res;   /* [N][K*b_r/32] */
  const uint16_t* scale; /* fp16 [K/G][N] */
  const uint16_t* zero;  /* fp16 [K/G][N] */
  const uint32_t* ref;   /* [K][N*b_f/32] or NULL */
  int N, K, G, b_r, b_f;
} sf_qweight;

/* ---- refinement cache (one per weight matrix) -------------------------- */

typedef struct sf_refine_cache sf_refine_cache;

typedef struct sf_cache_stats {
  int64_t steps;     /* prefetch steps taken */
  int64_t hits;      /* selected units found in the cache */
  int64_t misses;    /* selected units not found (bypass included) */
  int64_t bypass;    /* misses fetched for one step only (no slot left) */
  int64_t h2d_bytes; /* bytes moved from host memory for misses */
  int64_t late;      /* misses beyond the fetch budget: neither fetched nor cached */
} sf_cache_stats;

/*
 * sf_refine_cache_create -- an LRU cache of refinement units in device memory.
 *
 * Source: reuse of fetched precision across decode steps (arXiv abstract;
 * rag-lover.com explainer, TL;DR and 解説).  Policy (reading fixed by the
 * library): at each step with ascending selection S, hits H = S ∩ cached;
 * misses take free slots (lowest index first), then the slots of cached units
 * not in S ordered by (last use, unit), in ascending unit order; misses left
 * without a slot are the bypass set (fetched for this step only); every unit
 * used this step gets last use = this step.
 *   num_units   units addressable (K for a weight matrix);
 *   unit_bytes  bytes per unit (N*b_f/8 for a weight column), a multiple of 16;
 *   capacity    cache slots, 0 <= capacity <= min(num_units, 196608);
 *   max_select  largest selection a prefetch will see (B*k), >= 1;
 *   host_master host copy of all units, [num_units][unit_bytes], 16-byte
 *               aligned.  It must stay valid and unchanged until destroy.  If it
 *               is not page-locked the cache page-locks it (and unlocks it in
 *               destroy); either way the device reads it directly over the
 *               host link.
 *   device      CUDA device ordinal the cache lives on.
 * Allocates device memory for capacity + max_select unit rows plus small
 * index arrays.  Returns SF_ENOMEM / SF_ECUDA on allocation failure.
 */
sf_status sf_refine_cache_create(sf_refine_cache** out, int num_units, size_t unit_bytes,
                                 int capacity, int max_select, const void* host_master,
                                 int device);

/*
 * sf_refine_cache_create_parts -- `parts` independent LRU caches under one
 * handle: part p owns units [p*num_units/parts, (p+1)*num_units/parts) with
 * `capacity` slots of its own and sees at most `max_select` of them per step,
 * and each part follows the policy above on the run of the (ascending)
 * selection that falls in its range; its fetch budget is per part.  A KV
 * refinement cache uses one part per KV head (units g*S + t), so every
 * head's LRU step runs in parallel.  Slot numbers are global (part p's slots
 * are p*capacity ...), sf_refine_cache_slots writes parts*capacity entries,
 * and sf_refine_cache_sets concatenates the parts' lists (each host array
 * needs parts*max_select entries).  A partitioned cache cannot be preloaded
 * or join a group.  parts = 1 is sf_refine_cache_create.
 * Constraints: 1 <= parts <= 64, parts divides num_units, capacity at most
 * num_units/parts; otherwise as sf_refine_cache_create.
 */
sf_status sf_refine_cache_create_parts(sf_refine_cache** out, int num_units, size_t unit_bytes, int parts,
                                       int capacity, int max_select, const void* host_master, int device);

/* Fill an empty cache with n distinct units (device int32, ascending,
 * n <= capacity) in slots 0..n-1 with last use older than any step.  Counts
 * nothing in the statistics.  Enqueued on stream. */
sf_status sf_refine_cache_preload(sf_refine_cache* c, const int32_t* units, int n,
                                  sf_stream_t stream);

/*
 * sf_refine_cache_prefetch -- one cache step for the selection (idx, n) that
 * `producer` writes: resolve hits / misses / bypass, assign slots, and copy
 * every missed unit from host memory into its slot (or bypass row).  The work
 * runs on `side` after the producer's work so far; the next sf_gemv_refine
 * given this cache makes its own stream wait for it.  Issuing the prefetch of
 * a later layer before the GEMV of the current one overlaps the transfer with
 * compute (fetch lead, rag-lover.com explainer 解説).
 *   idx  device int32 ascending unit indices (length *n <= max_select; a
 *        negative *n counts as 0).
 * The GEMV that consumes this step must be enqueued before the next
 * prefetch on the same cache; the library orders the two streams.
 */
sf_status sf_refine_cache_prefetch(sf_refine_cache* c, const int32_t* idx, const int32_t* n,
                                   sf_stream_t producer, sf_stream_t side);

/* Copy the last step's sets to host arrays (each of capacity max_select):
 * hits, misses (bypass included) and bypass, ascending; counts[3] receives
 * their lengths.  Synchronizes with the last prefetch.  If that prefetch was
 * captured into a CUDA graph, the caller must first synchronize the stream
 * the graph was launched on (the same holds for _slots, _stats, _reset). */
sf_status sf_refine_cache_sets(sf_refine_cache* c, int32_t* hits, int32_t* misses,
                               int32_t* bypass, int32_t counts[3]);

/* Copy the unit held by each slot to host slot_units[capacity] (-1 = free).
 * Synchronizes with the last prefetch. */
sf_status sf_refine_cache_slots(sf_refine_cache* c, int32_t* slot_units);

/* Cumulative statistics since create/reset.  Synchronizes. */
sf_status sf_refine_cache_stats(sf_refine_cache* c, sf_cache_stats* out);

/* Empty the cache and zero the statistics.  Synchronizes. */
sf_status sf_refine_cache_reset(sf_refine_cache* c);

/* Free everything the cache owns.  Synchronizes.  NULL is accepted. */
sf_status sf_refine_cache_destroy(sf_refine_cache* c);

/*
 * sf_refine_cache_set_budget -- a per-step fetch budget, for a cache whose
 * consumer does not wait for this step's fetches (the KV refinement cache of
 * sf_attn_decode_refine).  At each later prefetch only the first `budget`
 * misses in ascending unit order are fetched (and placed as above); the
 * misses after them are late: neither fetched nor cached, counted in
 * sf_cache_stats.late, and their precision stays the resident one (a miss
 * keeps resident precision: rag-lover.com explainer, 限界と未検証の範囲).
 * budget -1 removes the limit (the default).  A cache with a budget below
 * max_select cannot serve a GEMV (SF_EINVAL there: a GEMV refines every
 * selected column).  Takes effect at the next sf_refine_cache_prefetch; a
 * group (below) keeps the budget its caches had when it was created.
 */
sf_status sf_refine_cache_set_budget(sf_refine_cache* c, int budget);

/*
 * sf_refine_cache_set_deadline -- the deadline reading for the cache of one
 * weight matrix (on != 0; off by default).  A batch-1 GEMV given this cache
 * (sf_gemv_refine_batch1) then does not wait for the fetches of its own
 * selection: it refines the selected columns that are cached when it runs
 * (E = S ∩ cached, read from the cache's index as its last prefetch left
 * it) and leaves the others at resident precision (a miss keeps resident
 * precision: rag-lover.com explainer, 限界と未検証の範囲).  The caller issues
 * the prefetch of S after the GEMV, so the misses arrive for later steps and
 * no host-link transfer sits between the selection and the GEMV.  The
 * generic sf_gemv_refine refuses such a cache (SF_EINVAL).
 * Constraints: a cache of parts = 1.
 */
sf_status sf_refine_cache_set_deadline(sf_refine_cache* c, int on);

/*
 * A group batches the prefetch of several caches whose selections live in
 * fixed device buffers (typically the weight matrices of one layer): one
 * launch resolves every cache's step (one CTA per cache) and one launch
 * gathers all their misses, so the side stream carries two kernels per layer
 * instead of two per matrix.  Semantics per cache are exactly those of
 * sf_refine_cache_prefetch with (idx[i], n[i]).
 *   caches  count distinct caches on one device (1 <= count <= 64);
 *   idx, n  per cache, the device buffers its selection will be read from at
 *           every sf_refine_group_prefetch (pointers captured at create).
 * The group does not own the caches; destroy it before them.
 */
typedef struct sf_refine_group sf_refine_group;
sf_status sf_refine_group_create(sf_refine_group** out, sf_refine_cache* const* caches,
                                 const int32_t* const* idx, const int32_t* const* n, int count);
/* One step for every cache of the group, on `side` after `producer`'s work. */
sf_status sf_refine_group_prefetch(sf_refine_group* g, sf_stream_t producer, sf_stream_t side);
/* Synchronizes the device, then frees the group.  NULL is accepted. */
sf_status sf_refine_group_destroy(sf_refine_group* g);

/*
 * sf_gemv_refine -- refined decode GEMV, y[b][i] = sum_j x[b][j] w_eff[i][j].
 *
 * Source: rag-lover.com explainer (解説): columns picked by activation
 * magnitude use resident + refinement bits, all others the resident code
 * dequantized at the midpoint of its refinement interval.  Equivalently
 *   y = W_res x + sum_{j in S} x_j s_{g(j)} (q_f - m_f),  m_f = (2^b_f - 1)/2.
 *   W      quantized weights; x device bf16 [B][K]; y device fp32 [B][N].
 *   idx,n  the selection S (device, as written by sf_select_topk).
 *   c      non-NULL: refinements come from the cache's last prefetch, which
 *          must have been given this same (idx, n);
 *          NULL and W->ref non-NULL: refinements read from W->ref directly;
 *          NULL and W->ref NULL: resident-only GEMV (idx, n ignored).
 * Constraints: 1 <= B <= 16, b_r in {2,3}, b_f in {1,2}, G % 32 == 0,
 *   K % G == 0, K <= 32768, N % 32 == 0.
 * Paths: B = 1 the integer dot-product kernel (2-bit) or the CUDA cores;
 *   2 <= B <= 16 with G % 128 == 0 and 16-byte aligned res and x the f16
 *   tensor cores (x scaled per 2048-channel chunk and row by a power of two
 *   and converted to f16: exact for entries within 28 binades of the row's
 *   maximum in the chunk), else the CUDA cores.
 * Accuracy: |y - exact| <= 2e-3 * sum_j |w_eff[i][j] x[b][j]| per output.
 */
sf_status sf_gemv_refine(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx,
                         const int32_t* n, sf_refine_cache* c, float* y, sf_stream_t stream);

/* ---- comparator modes (rag-lover.com explainer, 既存手法との違い) -------- */

/*
 * sf_select_random -- random selection of k of K channels (the ablation the
 * explainer sets against selection by activation magnitude): the k largest
 * keys key_j = (splitmix64(seed + K*step + j) >> 49) mod 32640 (Steele, Lea
 * and Flood's splitmix64 finalizer: z += 0x9E3779B97F4A7C15; z = (z ^ z>>30)
 * * 0xBF58476D1CE4E5B9; z = (z ^ z>>27) * 0x94D049BB133111EB; z ^ z>>31), ties
 * to the lower channel; idx_out ascending (device, capacity k), *n_out = k.
 * Counter-based: any (seed, step) is reproducible on its own.
 * Constraints: 1 <= K <= 32768, 0 <= k <= K.
 */
sf_status sf_select_random(int K, int k, uint64_t seed, uint64_t step, int32_t* idx_out, int32_t* n_out,
                           sf_stream_t stream);

/*
 * sf_quantize_residual -- the FP16-fetch comparator's store (DecDEC-like
 * residual columns): out[j][i] = fp16_RNE(W[i][j] - w_res[i][j]), W the fp32
 * weights [N][K] that Wq quantizes, w_res their resident values; the
 * difference is exact in fp64 and rounded once.  out: device fp16 [K][N]
 * (column-major: one column = one transfer unit of N*2 bytes).
 */
sf_status sf_quantize_residual(const float* W, const sf_qweight* Wq, uint16_t* out, sf_stream_t stream);

/*
 * sf_gemv_fp16_fetch -- the FP16-fetch comparator of sf_gemv_refine: the
 * selected columns use w_res + r (r from sf_quantize_residual) instead of
 * their refinement bits, the others w_res:
 *   y[b][i] = sum_j x[b][j] w_res[i][j] + sum_{j in S} x[b][j] r[j][i].
 * resid: the residual store [K][N] fp16 in device memory, or c: a cache of
 * its columns (units of N*2 bytes; its last prefetch used (idx, n)); exactly
 * one of the two.  Computed on the CUDA cores (the generic GEMV with an fp16
 * correction).  Constraints and accuracy as sf_gemv_refine.
 */
sf_status sf_gemv_fp16_fetch(const sf_qweight* W, const uint16_t* x, int B, const int32_t* idx, const int32_t* n,
                             const uint16_t* resid, sf_refine_cache* c, float* y, sf_stream_t stream);

/* ---- batch-1 fast path: prepared activations, several matrices per launch */

/* Bytes of the prepared form of one activation row of K channels (K/256
 * slices of 2112 bytes); 0 when K is not a positive multiple of 256. */
size_t sf_act_bytes(int K);

/*
 * sf_select_topk_act -- sf_select_topk for one row (B = 1) that also writes
 * the row's prepared form to act (device, sf_act_bytes(K) bytes, 16-byte
 * aligned, owned by the caller).  Per 128-channel group the activations
 * become fixed point relative to the group's largest exponent,
 * X = rint(x 2^(22-e)), stored as signed 8-bit digits in the register order
 * of the tensor-core GEMV's operand fragments, with the group's scale 2^(e-22)
 * and sum.  Per 256-channel slice it also stores which channels are
 * selected and how many selected channels precede the slice.  Same selection
 * rule and outputs as sf_select_topk.  K must be a multiple of 256 up to
 * 32768.  The layout is internal to the library.
 */
sf_status sf_select_topk_act(const uint16_t* x, int K, int k, int32_t* idx_out, int32_t* n_out,
                             void* act, sf_stream_t stream);

/* Several single-row selections with prepared activations in one launch
 * (one CTA per row): each job is sf_select_topk_act(x, K, k, idx_out, n_out,
 * act); act may be NULL to skip the prepared form.  1 <= count <= 8,
 * K a multiple of 32 up to 32768 (of 256 when act is given), x and act
 * 16-byte aligned. */
typedef struct sf_select_job {
  const uint16_t* x;
  int K, k;
  int32_t* idx_out;
  int32_t* n_out;
  void* act;
} sf_select_job;
sf_status sf_select_topk_act_many(const sf_select_job* jobs, int count, sf_stream_t stream);

/* The prepared form of x[K] with no channel selected (for resident-only
 * GEMVs).  K must be a multiple of 256 up to 32768. */
sf_status sf_act_prepare(const uint16_t* x, int K, void* act, sf_stream_t stream);

/*
 * sf_gemv_pack_batch1 -- the resident codes of a matrix in the layout the
 * batch-1 tensor-core GEMV reads (an internal re-arrangement of the same
 * bits, written once when the weights are loaded).  res: canonical resident
 * codes [N][K*b_r/32] (device); out: device, N*K*b_r/32 words, 16-byte
 * aligned, owned by the caller.  For b_r == 2 the layout is the canonical one
 * (a plain copy; out may equal res).  For b_r == 3 each 256-channel slice of
 * a row (24 words) holds the codes' low 2 bits in the 2-bit arrangement and
 * their high bits in a separate 8-word plane, so that a code becomes an MMA
 * operand byte with shifts and masks only; out must not alias res.
 * Constraints: b_r in {2, 3}, N >= 1, K a positive multiple of 256.
 */
sf_status sf_gemv_pack_batch1(const uint32_t* res, int N, int K, int b_r, uint32_t* out, sf_stream_t stream);

/* One matrix of a batch-1 GEMV launch.  The refinement source follows
 * sf_gemv_refine: cache (its last prefetch must have used the selection that
 * produced act), else W->ref when use_ref_store, else resident only.
 * res_b1: the resident codes in the batch-1 layout (sf_gemv_pack_batch1);
 * NULL means W->res, allowed for b_r == 2 only. */
typedef struct sf_gemv_job {
  const sf_qweight* W;
  sf_refine_cache* cache;
  int use_ref_store;
  float* y; /* device fp32 [W->N] */
  const uint32_t* res_b1;
} sf_gemv_job;

/*
 * sf_gemv_refine_batch1 -- refined GEMV at batch 1 for up to 4 matrices that
 * read the same activation row (q/k/v, gate/up): y_i = W_i,res x + sum over
 * the selected channels of x_j s (q_f - m_f), as sf_gemv_refine, in one
 * launch.  x: the bf16 row (device, 16-byte aligned); (idx, n): its selection
 * as sf_select_topk writes it (device; both NULL: nothing selected, the
 * resident-only GEMV).  Each warp turns its slice of x into the fixed-point
 * operand fragments itself (per 128-channel group X = rint(x 2^(22-e)), e the
 * exponent of the group's largest |x|, in signed 8-bit digits: the layout
 * sf_select_topk_act documents) and finds the slice's selected channels in
 * idx.  Computed on the integer tensor cores (mma.m16n8k32, 2- or 3-bit
 * codes x 8-bit activation digits) in tiles of 16 output rows; the
 * refinement correction on the f16 tensor cores (fp32 for a slice whose
 * selected |x| reaches 2^15).
 * Constraints: b_r in {2, 3}, b_f in {1, 2}, b_r + b_f <= 4, G == 128, all
 * jobs share K, G and bit widths; N % 16 == 0; K a multiple of 256 whose
 * K/256 slices split into at most 16 warps of one or two slices, in one or
 * two K halves (4096 and 14336 qualify; two halves run as the two thread
 * blocks of a cluster, which add their partial sums through distributed
 * shared memory: y = half 0 + half 1, one fp32 addition, and y needs no
 * zeroing); weight arrays 16-byte aligned; 3-bit codes given as res_b1.
 * SF_EINVAL otherwise.
 * Accuracy: as sf_gemv_refine, given that within every 128-channel group
 * the channels that matter are within 2^14 of the group's largest |x|: x is
 * taken in fixed point relative to that maximum, with an absolute error of
 * at most 2^(e-23) per channel (e its binary exponent), so channels far
 * below it keep few bits.
 */
sf_status sf_gemv_refine_batch1(const sf_gemv_job* jobs, int count, const uint16_t* x, const int32_t* idx,
                                const int32_t* n, sf_stream_t stream);

/* The producer of a batch-1 GEMV's input row when the GEMV launch computes
 * the row itself (sf_gemv_refine_batch1_produce).  Ops: */
enum { SF_PRODUCE_NORM = 0, SF_PRODUCE_ROUND = 1, SF_PRODUCE_SILU_MUL = 2 };
typedef struct sf_gemv_producer {
  int op;             /* SF_PRODUCE_* */
  int k;              /* channels of the row to select (0: none) */
  float eps;          /* SF_PRODUCE_NORM: the RMSNorm epsilon, >= 0 */
  const float* x;     /* fp32 [K], device: NORM the residual, ROUND the row, SILU_MUL the gate g */
  const float* delta; /* NORM: added to x first (fp32 [K]); may be NULL */
  const float* w;     /* NORM: the RMSNorm weights, fp32 [K] */
  const float* u;     /* SILU_MUL: the up projection, fp32 [K] */
  float* x_out;       /* NORM: receives x + delta (fp32 [K]); may be NULL; must not overlap x or delta */
  uint16_t* y;        /* out: the bf16 row [K], 16-byte aligned */
  int32_t* idx;       /* out: its selection, ascending, room for k entries */
  int32_t* n;         /* out: the selection's length (-1: the row holds a NaN or Inf) */
} sf_gemv_producer;

/*
 * sf_gemv_refine_batch1_produce -- sf_gemv_refine_batch1 whose input row and
 * selection are made inside the launch: the same results, bit for bit, as
 * the producer's stand-alone call followed by sf_gemv_refine_batch1(jobs,
 * count, p->y, p->idx, p->n):
 *   SF_PRODUCE_NORM     -- sf_norm_select(x, delta, w, K, eps, y, k, idx, n,
 *                          NULL) with the updated residual written to x_out
 *                          instead of in place (x is not modified);
 *   SF_PRODUCE_ROUND    -- sf_round_select(x, K, y, k, idx, n, NULL);
 *   SF_PRODUCE_SILU_MUL -- sf_silu_mul_select(x, u, K, y, k, idx, n, NULL).
 * Every thread block computes the row and its selection (the explainer of
 * StrataFlux, 解説: refinement where the input activation is large) while
 * its first weight codes stream in, so no one-block producer launch precedes
 * the GEMV; y, idx and n are written for later readers (a cache prefetch
 * after the launch, for instance).  Constraints: those of
 * sf_gemv_refine_batch1; K <= 32768; 0 <= k <= K and k within the launch's
 * scratch (several thousand entries at the Llama shapes; SF_EINVAL beyond);
 * caches, if any, in the deadline reading (a blocking prefetch needs the
 * selection before the launch).  With sf_gemv_set_launch_overlap on, the
 * launch may start while the previous kernel runs and reads x, delta, w and u
 * only after that kernel has completed.
 */
sf_status sf_gemv_refine_batch1_produce(const sf_gemv_job* jobs, int count, const sf_gemv_producer* p,
                                        sf_stream_t stream);

/*
 * sf_gemv_set_launch_overlap -- on != 0: sf_gemv_refine_batch1 launches with
 *   programmatic stream serialization, so its CTAs may start while the
 *   previous kernel on the stream still runs (typically the one-CTA producer
 *   of x and its selection: sf_norm_select, sf_round_select,
 *   sf_silu_mul_select) and read the weights' resident codes, scales and
 *   zero points before it has finished; x, the selection and the refinement
 *   rows are read only after it has completed.  The caller guarantees that
 *   no kernel that may still be running when the GEMV starts writes those
 *   weight arrays.  Process-wide; default off.
 */
sf_status sf_gemv_set_launch_overlap(int on);

/* ---- refined decode attention ----------------------------------------- */

/* Quantized K and V (views).  Rows are token-heads ordered [Hkv][S], token t
 * of KV head g at row g*S + t, each quantized as one group of d values with
 * sf_quantize_nested(layout SF_REF_BY_ROW) or sf_kv_append:
 * *_res [Hkv*S][d*b_r/32], *_ref [Hkv*S][d*b_f/32], *_scale, *_zero fp16
 * [Hkv*S].  S = row_stride when it is positive (a cache allocated for S
 * tokens per head, of which the first T are read), else S = T; a positive
 * row_stride below T is SF_EINVAL. */
typedef struct sf_qkv {
  const uint32_t *k_res, *k_ref, *v_res, *v_ref;
  const uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
  int b_r, b_f;
  int row_stride;
  /* NULL: k_ref / v_ref hold every token-head's refinement bits.  Non-NULL:
   * the refinement bits live in this cache instead (k_ref and v_ref are
   * ignored and may be NULL): one unit per token-head, unit g*S + t for token
   * t of KV head g, unit_bytes 64 = the token-head's K refinement words
   * followed by its V refinement words (both d*b_f/32 = 8 words).  A union
   * token whose unit is not cached when the call runs keeps its resident K
   * and V this step (the deadline reading of a KV refinement cache: a miss
   * keeps resident precision, rag-lover.com explainer, 限界と未検証の範囲);
   * the union and sel_out are unchanged.  The call orders its stream after
   * the cache's last prefetch, and the next prefetch after the call. */
  sf_refine_cache* ref_cache;
} sf_qkv;

/* Workspace bytes sf_attn_decode_refine needs for these sizes. */
sf_status sf_attn_workspace_size(int Hq, int Hkv, int d, int T, int k_tokens, size_t* bytes);

/*
 * sf_attn_decode_refine -- one decode step of attention over low-bit K/V with
 * the most-attended tokens refined.
 *
 * Source: rag-lover.com explainer (解説): KV refinement is chosen by the
 * attention weight computed from the low-bit keys.  Definition:
 *   query head h reads KV head h / (Hq/Hkv);
 *   key of token t for head h: kappa = fp64(s_t * sum_d q[h][d]*(c[t][d]*2^b_f
 *   + m_f - z_t)) computed exactly (c = resident key code); per head the
 *   k_tokens largest keys are selected (ties to the lower token index); the
 *   union over the heads of a KV group is refined in both K and V; the output
 *   is softmax attention over all T tokens with refined (full-code) K/V for the
 *   union and resident K/V elsewhere.
 *   q        device bf16 [Hq][d];
 *   sel_out  device int32 [Hkv][(Hq/Hkv)*k_tokens]: per KV head the ascending
 *            union; sel_n device int32 [Hkv] its lengths;
 *   out      device fp32 [Hq][d];
 *   workspace device scratch of at least sf_attn_workspace_size bytes (caller
 *            owned, contents need not be initialised, not read afterwards).
 * Exact selection needs, per query head, the binary exponents of its nonzero
 * q entries to span at most 53 - 9 - (b_r + b_f) - log2(d) = 33 binades (so
 * every key is exact in fp64).  When a head of KV group g violates it, the
 * selection still runs on the fp64 keys (then possibly not exact) and
 * sel_n[g] is written as -1 - (union length) to report it.
 * Constraints: d == 128, Hq/Hkv in {1, 2, 4, 8}, 1 <= T <= 2^24,
 *   0 <= k_tokens <= T, b_r == 2, b_f == 2.
 * Accuracy: max |out - exact| <= 2e-3.
 */
sf_status sf_attn_decode_refine(const uint16_t* q, int Hq, int Hkv, int d, int T,
                                const sf_qkv* kv, int k_tokens, int32_t* sel_out,
                                int32_t* sel_n, float* out, void* workspace, size_t ws_bytes,
                                sf_stream_t stream);

/*
 * sf_attn_decode_refine_noalloc -- sf_attn_decode_refine without a caller
 * workspace and without any device allocation.  The paper has no
 * counterpart; this exists for callers that cannot allocate device memory
 * when attention runs (a runtime with a fixed, pre-reserved memory pool, a
 * plugin that is handed no scratch, code where cudaMalloc is not allowed or
 * would synchronize the device).
 *
 * Same arguments, semantics and accuracy as sf_attn_decode_refine minus
 * workspace/ws_bytes.  Scratch comes from one 24 MiB array compiled into the
 * library (every GPU that loads the library reserves it until the process
 * exits); sizes whose scratch would exceed it (sf_attn_workspace_size > 24 MiB,
 * e.g. Hq * T above roughly 1.4 million) are rejected with SF_EINVAL before
 * anything is enqueued.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  Every call reuses the same array and
 * clears what must start at zero, so calls whose work overlaps on the GPU
 * (unordered streams) race; order them on one stream.
 */
sf_status sf_attn_decode_refine_noalloc(const uint16_t* q, int Hq, int Hkv, int d, int T,
                                        const sf_qkv* kv, int k_tokens, int32_t* sel_out,
                                        int32_t* sel_n, float* out, sf_stream_t stream);

/*
 * sf_attn_union_units -- the units of a KV refinement cache (see
 * sf_qkv.ref_cache) that one attention call selected: for each KV head g in
 * order, g*S + t for every token t of its ascending union, so the list is
 * ascending.  sel_out [Hkv][cap] and sel_n [Hkv] as written by the attention
 * (a negative sel_n[g] = -1 - length counts as its length); units device
 * int32 [Hkv*cap]; n_units device int32 scalar.  Feed (units, n_units) to
 * sf_refine_cache_prefetch to fetch the missed refinements for later steps.
 * Constraints: Hkv in [1, 64], cap >= 1, S >= 1.
 */
sf_status sf_attn_union_units(const int32_t* sel_out, const int32_t* sel_n, int Hkv, int cap, int S,
                              int32_t* units, int32_t* n_units, sf_stream_t stream);

/*
 * sf_attn_set_path -- which implementation sf_attn_decode_refine and
 * sf_attn_decode_refine_noalloc use, process-wide.  The paper has no
 * counterpart; both implementations compute the definition above (the same
 * selection, outputs within the same accuracy), so this is for diagnostics
 * and benchmarking:
 *   SF_ATTN_AUTO      the cluster kernel where it applies, else the pipeline;
 *   SF_ATTN_CLUSTER   only the cluster kernel, one thread-block cluster of up
 *                     to 16 CTAs per KV head doing the whole step on chip; it
 *                     applies for T <= 32768 (Hq/Hkv <= 4) or T <= 16384
 *                     (Hq/Hkv == 8) on a device that fits the cluster, and
 *                     other calls return SF_ENOTIMPL;
 *   SF_ATTN_PIPELINE  only the multi-kernel pipeline (every size; the only
 *                     one that reads refinements from a ref_cache).
 * Returns SF_EINVAL for any other value.  The setting is read when a call is
 * enqueued; a captured graph keeps the kernels it captured.
 */
typedef enum sf_attn_path { SF_ATTN_AUTO = 0, SF_ATTN_CLUSTER = 1, SF_ATTN_PIPELINE = 2 } sf_attn_path;
sf_status sf_attn_set_path(int path);

/* ---- decode-step elementwise operations -------------------------------- */

/*
 * The elementwise steps of one decode step of a Llama-shaped layer.  Source:
 * the benchmark configuration of the pages' end-to-end measurement names the
 * model shape (Llama-3.1-8B: RMSNorm, RoPE, SiLU-gated MLP); the formulas are
 * the library's reading (eps from the caller, RoPE rotate-half pairing with
 * base theta, no frequency rescaling), identical to the oracle's.  Values are
 * computed in fp64 and rounded once: to fp32 for fp32 outputs, to bf16 with
 * ties to even for bf16 outputs.  All pointers are device memory owned by the
 * caller; every call is asynchronous on `stream`.
 *
 * sf_add_rmsnorm -- residual add and RMSNorm, per row b of x [B][H] fp32:
 *   when delta (fp32 [B][H]) is not NULL, x += delta first (fp32 addition,
 *   written back); then y[b][i] = bf16(x[b][i] / sqrt(mean_i x^2 + eps) *
 *   w[i]), w fp32 [H], y bf16 [B][H].
 *   Constraints: B >= 1, H >= 1, eps >= 0.  SF_EINVAL otherwise.
 */
sf_status sf_add_rmsnorm(float* x, const float* delta, const float* w, int B, int H, float eps, uint16_t* y,
                         sf_stream_t stream);

/*
 * sf_rope -- rotates every head of x [H][d] fp32 (in place) to position pos:
 *   for i < d/2 the pair (x_i, x_{i+d/2}) turns by the angle
 *   pos * theta^(-2i/d).  When y_bf16 (bf16 [H][d]) is not NULL the rotated
 *   values are also written there as bf16.
 *   Constraints: H >= 1, d even in [2, 2048], pos >= 0, theta > 0.
 */
sf_status sf_rope(float* x, int H, int d, int pos, double theta, uint16_t* y_bf16, sf_stream_t stream);

/*
 * sf_silu_mul -- the SiLU-gated product of the MLP:
 *   y[i] = bf16(g[i] / (1 + exp(-g[i])) * u[i]) for i < n; g, u fp32 [n],
 *   y bf16 [n].  Constraints: n >= 1.
 */
sf_status sf_silu_mul(const float* g, const float* u, int n, uint16_t* y, sf_stream_t stream);

/*
 * Producer + selection in one launch (one thread block of 1024 threads, batch
 * 1): each writes the bf16 row y [K] that a GEMV reads, exactly as the
 * stand-alone op does, then selects its top k channels and writes the
 * prepared activations, exactly as sf_select_topk_act does (idx_out
 * ascending, *n_out its length or -1 for a NaN/Inf row; act as there, or NULL
 * to skip; k = 0 selects nothing, so act is then sf_act_prepare's form).
 *   sf_norm_select     -- sf_add_rmsnorm of one row (x += delta first when
 *                         delta is not NULL), y = bf16(RMSNorm(x) w);
 *   sf_round_select    -- y = bf16(a), a fp32 [K];
 *   sf_silu_mul_select -- y = bf16(silu(g) u), g, u fp32 [K].
 * Constraints: K (H) a multiple of 256 up to 32768, 0 <= k <= K, act 16-byte
 * aligned; idx_out has room for k entries.
 */
sf_status sf_norm_select(float* x, const float* delta, const float* w, int H, float eps, uint16_t* y, int k,
                         int32_t* idx_out, int32_t* n_out, void* act, sf_stream_t stream);
sf_status sf_round_select(const float* a, int K, uint16_t* y, int k, int32_t* idx_out, int32_t* n_out, void* act,
                          sf_stream_t stream);
sf_status sf_silu_mul_select(const float* g, const float* u, int K, uint16_t* y, int k, int32_t* idx_out,
                             int32_t* n_out, void* act, sf_stream_t stream);

/*
 * sf_rope_qk -- sf_rope of the query heads q [Hq][d] (also written as bf16 to
 *   q_bf16 [Hq][d] when it is not NULL) and of the key heads k [Hkv][d], in
 *   one launch.  Same constraints as sf_rope (Hkv may be 0).
 */
sf_status sf_rope_qk(float* q, int Hq, float* k, int Hkv, int d, int pos, double theta, uint16_t* q_bf16,
                     sf_stream_t stream);

/*
 * sf_round_bf16 -- y[i] = bf16(x[i]) (to nearest, ties to even) for i < n:
 *   the attention's fp32 output as the bf16 input of the o projection.
 *   x fp32 [n], y bf16 [n].  Constraints: n >= 1.
 */
sf_status sf_round_bf16(const float* x, int n, uint16_t* y, sf_stream_t stream);

/*
 * sf_kv_append -- quantizes the new token's rows of K or V and writes them as
 *   token t of every KV head of a cache allocated for row_stride tokens per
 *   head: src fp32 [Hkv][d] (row g = KV head g) becomes cache row
 *   g * row_stride + t, quantized exactly as sf_quantize_nested does with one
 *   group of d values per row and SF_REF_BY_ROW (the KV quantization of the
 *   pages' 2+2-bit KV: nested refinement, rag-lover.com explainer, 解説).
 *   Cache arrays (caller-owned, rows = Hkv * row_stride): res uint32
 *   [rows][d*b_r/32], ref uint32 [rows][d*b_f/32], scale and zero fp16
 *   [rows].  Only the Hkv rows of token t are written.
 *   Constraints: Hkv >= 1, d a multiple of 32 in [32, 512], 0 <= t <
 *   row_stride, b_r in {2,3}, b_f in {1,2}, b_r + b_f <= 4.  src finite.
 */
sf_status sf_kv_append(const float* src, int Hkv, int d, int row_stride, int t, int b_r, int b_f, uint32_t* res,
                       uint32_t* ref, uint16_t* scale, uint16_t* zero, sf_stream_t stream);

/*
 * sf_kv_append_cached -- sf_kv_append for K/V whose refinement bits live in a
 *   KV refinement cache (sf_qkv.ref_cache): the resident codes, scale and zero
 *   of token t go to res / scale / zero as in sf_kv_append; the refinement
 *   words go to the cache's host master, unit g * row_stride + t, in its K
 *   half (part 0) or V half (part 1), and also to the unit's cache row if it
 *   is cached (so no cached copy goes stale).  The host master is written
 *   through its device mapping, and must stay as the cache was created with.
 *   Ordered after the cache's last prefetch; the next prefetch waits for it.
 *   Constraints: as sf_kv_append; the cache's units are 2*d*b_f/8 bytes and
 *   number at least Hkv * row_stride; part in {0, 1}.
 */
sf_status sf_kv_append_cached(const float* src, int Hkv, int d, int row_stride, int t, int b_r, int b_f,
                              uint32_t* res, uint16_t* scale, uint16_t* zero, sf_refine_cache* ref_cache, int part,
                              sf_stream_t stream);

/*
 * sf_kv_append_pair_cached -- sf_kv_append_cached for the key rows (k_src,
 *   part 0) and value rows (v_src, part 1) of token t in one launch, with the
 *   host master's copy taken off `stream`: on `stream` the refinement words
 *   go to a device staging area of the cache (and to the cached copy of a
 *   cached unit); one 2-D copy then moves them to the host master on `side`,
 *   after what `stream` has enqueued so far.  Work enqueued on `side` after
 *   this call (the cache's prefetch) reads the new words; the next append
 *   waits for that copy (under stream capture: when it belongs to the same
 *   capture).  side may equal stream.  The first call per cache allocates the
 *   staging area and must not be under stream capture.
 *   Constraints: as sf_kv_append_cached, for both rows.
 */
sf_status sf_kv_append_pair_cached(const float* k_src, const float* v_src, int Hkv, int d, int row_stride, int t,
                                   int b_r, int b_f, uint32_t* k_res, uint16_t* k_scale, uint16_t* k_zero,
                                   uint32_t* v_res, uint16_t* v_scale, uint16_t* v_zero, sf_refine_cache* ref_cache,
                                   sf_stream_t stream, sf_stream_t side);

/*
 * sf_rope_kv_append_pair_cached -- sf_rope_qk(q, Hq, k, Hkv, d, pos, theta,
 *   q_bf16) followed by sf_kv_append_pair_cached of the rotated k and of v,
 *   in one launch with the same results bit for bit: the key rows are
 *   rotated in registers before they are quantized (and written back to k),
 *   while other blocks of the launch rotate the query heads (q in place,
 *   q_bf16 when it is not NULL).  The rotation and the append are the steps
 *   of a decode step between the q/k/v projections and the attention (RoPE
 *   of the new token, then its K/V rows appended; the attention reads both).
 *   Constraints: those of sf_rope_qk and sf_kv_append_pair_cached, with d a
 *   multiple of 64 (the thread that holds dim i also holds i + d/2).
 */
sf_status sf_rope_kv_append_pair_cached(float* q, int Hq, uint16_t* q_bf16, float* k, const float* v, int Hkv, int d,
                                        int pos, double theta, int row_stride, int t, int b_r, int b_f,
                                        uint32_t* k_res, uint16_t* k_scale, uint16_t* k_zero, uint32_t* v_res,
                                        uint16_t* v_scale, uint16_t* v_zero, sf_refine_cache* ref_cache,
                                        sf_stream_t stream, sf_stream_t side);

#ifdef __cplusplus
}
#endif

#endif /* SF_H */

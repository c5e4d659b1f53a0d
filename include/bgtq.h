/*
 * bgtq.h -- C ABI of the Block-GTQ packed KV-cache library for B200 (sm_100a).
 *
 * Block-GTQ ("RoPE-Aware Bit Allocation for KV-Cache Quantization", Liang,
 * Zhang, Jia; arXiv 2606.24033 abstract and the blockgtq README) quantises
 * the key cache per RoPE 2-D frequency block: a label-free Q/K energy score
 * per block, greedy integer bit widths by marginal gain under a fixed
 * average, then the TurboQuant-MSE (TQ-MSE) encoder; a packed-cache serving
 * path decodes attention straight from the codes.  This library implements
 * that hot path:
 *
 *   bgtq_allocate       energy score per block + greedy allocation + tables
 *   bgtq_encode_append  rotate, normalise, Lloyd-Max quantise, bit-pack K/V
 *   bgtq_encode_append_rope  the same from K before RoPE (RoPE fused in)
 *   bgtq_rotate_query   the query in each width group's rotated basis
 *   bgtq_decode_attn    one GQA decode step over the packed cache
 *   bgtq_decode_step    encode_append of a step's rows + decode_attn in one call
 *   bgtq_decode_attn_buffered  decode with fp16 sink / recent-window rows
 *   bgtq_decode_step_buffered  the same after a step's appends, in one call
 *   bgtq_logit_mae      per-layer logit error of the packed keys (diagnostic)
 *   bgtq_set_block_table  page table of a paged cache
 *
 * Conventions
 *  - Every function returns 0 (BGTQ_OK) or a negative BGTQ_ERR_* code and
 *    never throws or aborts.  Argument checks happen before any launch; a
 *    call that fails its checks launches nothing.
 *  - Device buffers are owned by the caller (allocated e.g. with torch); the
 *    library never allocates or frees device memory.  Host memory for the
 *    tables is owned by the state and freed by bgtq_destroy.
 *  - "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls marked ASYNC only enqueue work on that stream; calls
 *    marked SYNC wait for their own work before returning.
 *  - K and Q arrive after RoPE; the library never applies RoPE.  head_dim
 *    must be 128 (64 RoPE blocks).  Softmax scale is 1/sqrt(head_dim).
 *    Query head h reads KV head h / G, G = n_q_heads / n_kv_heads.
 *  - fp16 tensors are IEEE binary16, row-major, densely packed, 16-byte
 *    aligned.
 *  - A state belongs to the CUDA device that was current at bgtq_create
 *    (its buffers live there).  Every call that launches work or copies
 *    returns BGTQ_ERR_INVALID_ARG, launching nothing, when another device
 *    is current.
 *  - A state is not thread-safe: call it from one host thread at a time.
 *    Its decode calls share the workspace's scratch (rotated queries, split
 *    partials, arrival counters), so two of its calls must not overlap
 *    on the GPU: issue them on one stream, or order the streams.
 *
 * Cache layout inside d_cache (offsets from bgtq_cache_offsets, each
 * 256-byte aligned; L layers, B = max_batch, H = n_kv_heads, T =
 * ceil(capacity / 64) tiles of 64 positions per (layer, sequence, head)):
 *   K tiles    uint8 [L][B][H][T][1024*k_avg_bits]  codes of 64 positions,
 *              laid out for the tensor-core decode (per lane, the nibble
 *              selectors of its mma A-fragments as bit planes; width groups
 *              widest first; see the tile-format definition shipped with
 *              the tests' CPU oracle)
 *   K norms    fp16  [L][B][H][T*64][4]   slot i = norm of group i (width
 *              descending); unused slots 0
 *   V tiles    uint8 [L][B][H][T][1024*v_avg_bits]  same scheme, one group
 *   V norms    fp16  [L][B][H][T*64]
 * Paged cache (page_pool_tiles = P > 0; PagedAttention's block table,
 * cited by the blockgtq pages): the same four arrays with [L][H][P] in place
 * of [L][B][H][T], and the caller's block table (bgtq_set_block_table)
 * mapping tile t of sequence b to a page id, the same for every layer and
 * KV head.  Sequences of a ragged batch then hold only the pages they use.
 * Codebook: the N(0,1) Lloyd-Max levels for 1..4 bits rounded once to
 * binary16; thresholds are the exact midpoints of those levels.
 */
#ifndef BGTQ_H
#define BGTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  BGTQ_OK = 0,
  BGTQ_ERR_INVALID_ARG = -1,   /* a size, index or config field out of range */
  BGTQ_ERR_NULL = -2,          /* a required pointer is NULL */
  BGTQ_ERR_CUDA = -3,          /* a CUDA runtime call failed (launch or copy) */
  BGTQ_ERR_BUFFER_SIZE = -4,   /* a caller buffer is smaller than required */
  BGTQ_ERR_NOT_READY = -5,     /* no allocation set yet (allocate/set_allocation first) */
  BGTQ_ERR_DEVICE = -6,        /* a kernel raised its error flag (see bgtq_get_device_error) */
  BGTQ_ERR_HOST_ALLOC = -7,    /* host malloc failed */
  BGTQ_ERR_ALIGNMENT = -8      /* a device pointer is not 16-byte aligned */
};

/* Device error flag bits, reported by bgtq_get_device_error. */
enum {
  BGTQ_DEVERR_CAPACITY = 1,    /* encode_append: start + count > capacity (rows skipped) */
  BGTQ_DEVERR_SEQ_LEN = 2,     /* decode: a seq_len < 0 or > capacity (sequence skipped, output 0), or a pos_lo /
                                  buf_count out of range (clamped) */
  BGTQ_DEVERR_ARG = 4,         /* encode_append: start < 0 or count < 0 or count > n */
  BGTQ_DEVERR_NONFINITE = 8,   /* allocate: a calibration value is Inf or NaN */
  BGTQ_DEVERR_TIMEOUT = 16,    /* decode: a wait for a tile copy gave up (bounded spin) */
  BGTQ_DEVERR_PAGE = 32        /* paged cache: a block-table entry outside [0, page_pool_tiles) (encode skips the
                                  tile, decode reads page 0 instead, logit MAE skips the tile) */
};

typedef struct {
  int32_t n_layers;          /* 1..65535 (a call's layers are a launch grid dimension) */
  int32_t n_kv_heads;        /* >= 1 */
  int32_t n_q_heads;         /* multiple of n_kv_heads; G = n_q_heads / n_kv_heads <= 16 */
  int32_t head_dim;          /* must be 128 */
  int32_t max_batch;         /* >= 1 */
  int32_t k_avg_bits;        /* average K bits per dim, 1..4 (record = 16*k bytes) */
  int32_t v_avg_bits;        /* V bits per dim, 1..4 */
  int32_t b_min;             /* smallest K width, 0..4 (0: a block may store nothing) */
  int32_t b_max;             /* largest K width, b_min..4, b_min <= k_avg_bits <= b_max */
  int32_t rope_pairing;      /* 0: block j = dims (j, j+64) (rotate_half); 1: (2j, 2j+1) */
  int32_t max_splits;        /* split-K slots per (layer, seq, KV head); 0 = 256 */
  int32_t page_pool_tiles;   /* 0: contiguous cache; > 0: paged cache with this many
                                64-position pages per (layer, KV head), addressed
                                through bgtq_set_block_table */
  int64_t capacity_tokens;   /* cached tokens per sequence, >= 1 */
  uint64_t seed;             /* seeds the Haar rotations */
} bgtq_config;

typedef struct bgtq_state bgtq_state;

/* Bytes of the two caller-owned device buffers for a config.
 * cache_bytes: the packed K/V cache (layout above).  workspace_bytes: the
 * device tables plus scratch (energy partial sums, rotated queries, split-K
 * partials, error flag).  A config whose cache or workspace would reach
 * 2^56 bytes is rejected with BGTQ_ERR_INVALID_ARG.  SYNC (host only). */
int bgtq_required_bytes(const bgtq_config* cfg, size_t* cache_bytes, size_t* workspace_bytes);

/* Creates a state over caller buffers of at least the required sizes (both
 * 256-byte aligned).  The state keeps the pointers; the buffers must outlive
 * it.  Uploads the Lloyd-Max codebooks and clears the error flag on
 * "stream".  No allocation is set: call bgtq_allocate or
 * bgtq_set_allocation before encoding.  SYNC. */
int bgtq_create(const bgtq_config* cfg, void* d_cache, size_t cache_bytes,
                void* d_workspace, size_t workspace_bytes, void* stream, bgtq_state** out);

/* Frees the host-side state (never the caller's device buffers). NULL is a no-op. */
void bgtq_destroy(bgtq_state* st);

/* Block-GTQ allocation (abstract: per layer and KV head, a label-free energy
 * score for every RoPE block, then integer widths handed out greedily by
 * marginal gain).  Score of block j: s_j = EQ_j * EK_j with
 * EQ_j = sum over rows and the G query heads of the group of ||q_j||^2 and
 * EK_j = sum over rows of ||k_j||^2, accumulated exactly on the GPU (fp16 x
 * 2^24 is an integer; 128-bit sums).  Greedy: every block starts at b_min;
 * each step gives one bit to the block with the largest s_j*(Dist(b_j) -
 * Dist(b_j+1)) below b_max (ties: lowest block), until sum_j b_j =
 * k_avg_bits * 64.  Dist(b) = N(0,1) Lloyd-Max MSE {1, .363380, .117482,
 * .034548, .009497}.  Then builds the per-(layer, KV head) group layout and
 * Haar rotations and uploads them.
 *   d_calib_q  fp16 [n_layers][nq][n_q_heads][128]
 *   d_calib_k  fp16 [n_layers][nk][n_kv_heads][128]
 * nq, nk >= 1.  SYNC (copies the exact sums back, runs the greedy on the host). */
int bgtq_allocate(bgtq_state* st, const void* d_calib_q, int32_t nq,
                  const void* d_calib_k, int32_t nk, void* stream);

/* Sets the widths directly (e.g. uniform TQ-MSE: every block = k_avg_bits)
 * and builds/uploads the tables as bgtq_allocate does.
 *   h_widths int8 [n_layers][n_kv_heads][64], each in [b_min, b_max],
 *            each (layer, head) summing to 64 * k_avg_bits.  SYNC. */
int bgtq_set_allocation(bgtq_state* st, const int8_t* h_widths, void* stream);

/* Copies the current widths out (int8 [n_layers][n_kv_heads][64]). SYNC. */
int bgtq_get_allocation(const bgtq_state* st, int8_t* h_widths);

/* The exact energies of the last bgtq_allocate as 128-bit integers in units
 * of 2^-48, little-endian (lo, hi) uint64 pairs:
 *   h_eq, h_ek  uint64 [n_layers][n_kv_heads][64][2].  SYNC. */
int bgtq_get_energy(const bgtq_state* st, uint64_t* h_eq, uint64_t* h_ek);

/* The Lloyd-Max codebook for bits in 1..4 (TurboQuant's scalar quantiser on
 * N(0,1)) as stored: h_centroids[2^bits] (binary16 values as floats),
 * h_thresholds[2^bits - 1] (their midpoints). */
int bgtq_get_codebook(int32_t bits, float* h_centroids, float* h_thresholds);

/* Group layout of (layer, kv_head): *n_groups, per group its width and size
 * (h_width[4], h_size[4]; unused 0) and h_perm[128] = the original dim at
 * each record position.  SYNC (host tables). */
int bgtq_get_layout(const bgtq_state* st, int32_t layer, int32_t kv_head, int32_t* n_groups,
                    int32_t* h_width, int32_t* h_size, int32_t* h_perm);

/* The fp32 Haar rotation of one group (kind 0 = K, group index 0..n_groups-1)
 * or of V (kind 1, group ignored), row-major d x d, y = R x.  *d receives
 * the size; h_out must hold 128*128 floats.  SYNC (host tables). */
int bgtq_get_rotation(const bgtq_state* st, int32_t layer, int32_t kv_head, int32_t kind,
                      int32_t group, float* h_out, int32_t* d);

/* Byte offsets of the four cache arrays inside d_cache:
 * out[0] K tiles, out[1] K norms, out[2] V tiles, out[3] V norms. */
int bgtq_cache_offsets(const bgtq_state* st, size_t* out);

/* TQ-MSE encode + bit-pack of new rows into the cache.  Source: the
 * Block-GTQ abstract (the allocator's widths feed the TurboQuant-MSE
 * encoder, and the serving path keeps a packed cache) and the blockgtq
 * README's method blurb (integer widths on top of the TQ-MSE encoder) and
 * packed-cache deployment path; TurboQuant (arXiv 2504.19874, cited on the
 * mlsanity index page) for the encoder itself: a random rotation, then the
 * Lloyd-Max scalar quantiser of each rotated coordinate.  For each layer
 * l in [layer, layer + layer_count), sequence b < batch, row r < count[b]:
 * the K and V rows at d_k/d_v[l - layer][b][r][h][:] go to cache position
 * start[b] + r of (l, b, h).  Per K width group g (dims D_g, d = |D_g|):
 * n = ||x[D_g]|| (float64), y = R_g x[D_g] (fp32), u = sqrt(d) y / n,
 * code = #{thresholds <= u}; stored norm = fp16(n).  V: one group of 128.
 *   d_k, d_v   fp16 [layer_count][batch][n][n_kv_heads][128]
 *   d_start    int32 [batch]  first cache position written
 *   d_count    int32 [batch]  rows of this sequence, 0..n
 * Rows with start + r >= capacity are skipped and set BGTQ_DEVERR_CAPACITY.
 * ASYNC. */
int bgtq_encode_append(bgtq_state* st, int32_t layer, int32_t layer_count,
                       const void* d_k, const void* d_v, const int32_t* d_start,
                       const int32_t* d_count, int32_t batch, int32_t n, void* stream);

/* The fused RoPE + encode: bgtq_encode_append with the K rows taken before
 * RoPE (the key projection's output).  Row r of sequence b is turned by
 * RoPE at its cache position p = start[b] + r before it is encoded: block j
 * of the config's rope_pairing (dims (j, j+64) or (2j, 2j+1)) becomes
 * (a cos t - b sin t, a sin t + b cos t) with t = p * rope_base^(-2j/128),
 * the product in fp64 reduced to [-pi, pi], sin and cos in fp32.  The
 * turned values are encoded in fp32 without rounding to fp16.  Groups hold
 * whole RoPE blocks, so a group's norm is that of the row as given, up to
 * the rounding of the turned values.
 * V rows are encoded as in bgtq_encode_append.  rope_base: finite, > 1
 * (BGTQ_ERR_INVALID_ARG otherwise).  Arguments, layouts and device errors
 * otherwise as bgtq_encode_append.  ASYNC. */
int bgtq_encode_append_rope(bgtq_state* st, int32_t layer, int32_t layer_count,
                            const void* d_k, const void* d_v, const int32_t* d_start,
                            const int32_t* d_count, int32_t batch, int32_t n, double rope_base,
                            void* stream);

/* The query in each K width group's rotated basis.  Source: TurboQuant's
 * encoder (arXiv 2504.19874, cited on the mlsanity index page) rotates each
 * group of a key by R_g, and R_g is orthogonal, so q . R_g^T y = (R_g q) . y:
 * the logits of the Block-GTQ abstract's packed-cache serving path can be
 * taken from the codes once q is rotated, one rotation per width group.
 * q~ in record order: per K group g, (1/sqrt(128)) (1/sqrt(d_g)) R_g q[D_g].
 *   d_q     fp16 [layer_count][batch][n_q_heads][128]
 *   d_qrot  fp32 [layer_count][batch][n_q_heads][128]
 * Also writes the tensor-core operand form of q~ into the workspace.  ASYNC. */
int bgtq_rotate_query(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                      int32_t batch, float* d_qrot, void* stream);

/* One decode step over the packed cache.  Source: the Block-GTQ abstract's
 * packed-cache serving path (attention at 128K-512K context straight from
 * the packed K3V3 cache) and the blockgtq README's decode benchmark and
 * backend table (a fused decode kernel reading the packed cache); split-K
 * decoding after FlashAttention / FlashAttention-2 (arXiv 2205.14135,
 * 2307.08691, cited on the mlsanity index page).
 * For each layer in [layer, layer + layer_count), sequence
 * b < batch and query head h,
 *   out = sum_t softmax_t(q . k_hat_t / sqrt(128)) v_hat_t over cache
 *   positions t < seq_lens[b],
 * taken in the rotated domain (logits from q~ and the codes; V accumulated
 * in V's rotated basis and rotated back once).  seq_lens[b] = 0 gives 0.
 *   d_q        fp16 [layer_count][batch][n_q_heads][128]
 *   d_seq_lens int32 [batch], 0..capacity
 *   d_out      fp16 [layer_count][batch][n_q_heads][128]
 * Uses the workspace for q~ and split-K partials, so calls on one state
 * must not overlap on the GPU.  ASYNC. */
int bgtq_decode_attn(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                     const int32_t* d_seq_lens, int32_t batch, void* d_out, void* stream);

/* One decode step of a layer range as a serving loop runs it: the step's
 * new K/V rows go into the packed cache, then attention reads it (the
 * Block-GTQ abstract's packed-cache serving path; the blockgtq README's
 * decode benchmark, which times decode steps at a given context length).
 * bgtq_encode_append of the step's new
 * rows followed by bgtq_decode_attn, with the same arguments, results and
 * errors as those two calls in that order (seq_lens should count the new
 * rows).  With 1 <= n <= 16 rows per sequence the appends and the query
 * rotation run in one launch (they are independent), so a step takes three
 * launches instead of four.  n = 0 appends nothing (d_k, d_v, d_start and
 * d_count may then be NULL).  ASYNC. */
int bgtq_decode_step(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                     const int32_t* d_start, const int32_t* d_count, int32_t n, const void* d_q,
                     const int32_t* d_seq_lens, int32_t batch, void* d_out, void* stream);

/* Decode with an fp16 buffer: the Block-GTQ README's "withbuffer" setting
 * (AIME commands: a few sink positions and a recent window kept
 * unquantised).  For each layer, sequence b and query head h, attention runs
 * over the packed positions [pos_lo[b], seq_lens[b]) and the sequence's
 * first buf_count[b] buffered rows, with one softmax:
 *   out = sum_t softmax_t(q . k_t / sqrt(128)) v_t
 * over both sets (the packed rows dequantised as for bgtq_decode_attn, the
 * buffered rows as given).  Which positions the buffered rows stand for is
 * the caller's business (typically [0, n_sink) and [len - n_window, len),
 * with pos_lo = n_sink and seq_lens = len - n_window).
 *   d_q, d_out   fp16 [layer_count][batch][n_q_heads][128]
 *   d_seq_lens   int32 [batch]  end of the packed range, 0..capacity
 *   d_pos_lo     int32 [batch]  start of the packed range, 0..seq_lens[b]
 *   d_buf_k/v    fp16 [layer_count][batch][n_buf][n_kv_heads][128]
 *   d_buf_count  int32 [batch]  buffered rows used, 0..n_buf
 *   n_buf        1..1024 (BGTQ_ERR_INVALID_ARG outside)
 * An empty packed range and no buffered row give 0.  Out-of-range
 * lengths set BGTQ_DEVERR_SEQ_LEN and are clamped.  The buffered rows of a
 * (sequence, KV head) are attended by one more CTA of the split pass,
 * beside the packed ones.  Uses the workspace like bgtq_decode_attn.
 * ASYNC. */
int bgtq_decode_attn_buffered(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                              const int32_t* d_seq_lens, const int32_t* d_pos_lo, int32_t batch, const void* d_buf_k,
                              const void* d_buf_v, const int32_t* d_buf_count, int32_t n_buf, void* d_out,
                              void* stream);

/* Per-layer logit MAE of the packed keys: the Block-GTQ abstract's logit
 * fidelity diagnostic and the blockgtq README's per-layer kernel MAE
 * (bit allocation section, `--window-M 1024`), comparing Block-GTQ with
 * uniform TQ-MSE at the same average width (two states, one allocated and
 * one with bgtq_set_allocation, holding the same keys).  Only K is
 * involved.  Over a window of m cached positions w0 .. w0+m-1 of sequence
 * seq, with the queries at the same positions, for every causal pair
 * (query i, key j), 0 <= j <= i < m, and each query head h:
 *   d_mae[l][h] = mean |q_{i,h} . k_hat_j - q_{i,h} . k_j| / sqrt(128)
 * where q . k_hat is the logit exactly as the decode computes it from the
 * packed cache and k the exact key.  A layer's MAE is the mean over its
 * heads.
 *   d_q    fp16 [layer_count][m][n_q_heads][128]   queries (post-RoPE)
 *   d_k    fp16 [layer_count][m][n_kv_heads][128]  the exact keys the cache
 *          holds (encoded) at positions w0 .. w0+m-1 of sequence seq
 *   d_mae  double [layer_count][n_q_heads], written by the call
 * 0 <= seq < max_batch, m >= 1, w0 >= 0, w0 + m <= capacity_tokens,
 * else BGTQ_ERR_INVALID_ARG.  The per-head sums use fp64 atomics, so the
 * last bits can vary between runs.  Does not touch the workspace's decode
 * scratch.  ASYNC. */
int bgtq_logit_mae(bgtq_state* st, int32_t layer, int32_t layer_count, int32_t seq, int32_t w0, int32_t m,
                   const void* d_q, const void* d_k, double* d_mae, void* stream);

/* bgtq_encode_append of a step's new rows followed by
 * bgtq_decode_attn_buffered, as one call (the appends and the query rotation
 * share a launch for 1..16 rows per sequence): same arguments, results and
 * errors as those two calls in that order.  In the withbuffer setting the
 * rows appended are typically those leaving the recent fp16 window.  n = 0
 * appends nothing (d_k, d_v, d_start and d_count may then be NULL).  ASYNC. */
int bgtq_decode_step_buffered(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                              const int32_t* d_start, const int32_t* d_count, int32_t n, const void* d_q,
                              const int32_t* d_seq_lens, const int32_t* d_pos_lo, int32_t batch,
                              const void* d_buf_k, const void* d_buf_v, const int32_t* d_buf_count, int32_t n_buf,
                              void* d_out, void* stream);

/* The two stages of bgtq_decode_attn after bgtq_rotate_query, for callers
 * that time or schedule them separately (same arguments and results):
 * bgtq_decode_split runs the split-K pass over the packed cache from the
 * rotated queries d_qrot (fp32 [layer_count][batch][n_q_heads][128], as
 * written by bgtq_rotate_query) into the workspace's partials, and
 * bgtq_decode_combine merges them into d_out.  Both must see the same
 * layer, layer_count, batch, split setting and length values.  The combine
 * reads d_seq_lens as soon as the work queued before it on the stream lets
 * it start, so it must follow its bgtq_decode_split on the stream with no
 * kernel of the caller's in between.  ASYNC. */
int bgtq_decode_split(bgtq_state* st, int32_t layer, int32_t layer_count, const float* d_qrot,
                      const int32_t* d_seq_lens, int32_t batch, void* stream);
int bgtq_decode_combine(bgtq_state* st, int32_t layer, int32_t layer_count, const int32_t* d_seq_lens,
                        int32_t batch, void* d_out, void* stream);

/* No Block-GTQ counterpart on the pages: a library convenience.
 *
 * Same computation, arguments and results as bgtq_decode_attn, for callers
 * that cannot allocate device memory themselves: code that issues work from
 * inside a CUDA stream capture (allocation is not a capturable operation),
 * or a runtime whose device memory is fully reserved up front by its own
 * pool.  This call needs no caller-provided scratch: the rotated queries
 * and split-K partials live in one static device array inside the library
 * of BGTQ_STATIC_SCRATCH_BYTES (16 MiB), which every GPU that loads the
 * library holds until the process exits.  The call allocates nothing.
 *
 * The scratch needed is 64 KiB of arrival counters plus rows * (512 +
 * n_splits * 528 + 8 * 528) bytes, rows = layer_count * max_batch *
 * n_q_heads, plus 6 KiB per (layer, sequence, KV head, block of 8 query
 * heads), with n_splits the most split CTAs a unit can get as for
 * bgtq_decode_attn (see bgtq_set_split_tokens); a call needing more
 * returns BGTQ_ERR_BUFFER_SIZE before launching anything.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any
 * stream capture.  The address is kept for the life of the process: after
 * cudaDeviceReset (a new primary context) it is stale, so no call may
 * follow a reset of a device the library has used.  Every call on a device
 * shares the one array and reads
 * only what the same call wrote: calls that overlap on the GPU (different
 * streams, or different states at once) race on it.  ASYNC after the first
 * call. */
#define BGTQ_STATIC_SCRATCH_BYTES (16u << 20)
int bgtq_decode_attn_static_scratch(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                                    const int32_t* d_seq_lens, int32_t batch, void* d_out, void* stream);

/* Paged cache only (page_pool_tiles > 0): the block table, int32
 * [max_batch][ceil(capacity / 64)] in device memory, caller-owned: entry
 * [b][t] = the page holding positions 64 t .. 64 t + 63 of sequence b, in
 * 0 .. page_pool_tiles - 1.  Entries are read by the kernels when they run
 * (so the caller may fill in new pages between calls, also under graph
 * replay); only the tiles a call reads or writes need valid entries.  Two
 * sequences must not share a page they write.  Until a table is set, calls
 * that touch the cache return BGTQ_ERR_NOT_READY; on a contiguous cache
 * this call returns BGTQ_ERR_INVALID_ARG.  NULL clears the table.  SYNC
 * (host only). */
int bgtq_set_block_table(bgtq_state* st, const int32_t* d_block_table);

/* Split-K width for the decode calls: 0 = automatic (one wave of resident
 * CTAs spread over all (layer, sequence, KV head) units in proportion to
 * their lengths, so that the sequences of a ragged batch finish together;
 * at most twice a unit's even share and max_splits), else a multiple of 64
 * (one tile): a sequence of len positions then gets ceil(len / tokens) <=
 * max_splits split CTAs per unit.  The split counts are computed on the GPU
 * from the lengths.  Results do not depend on the setting beyond
 * floating-point reassociation. */
int bgtq_set_split_tokens(bgtq_state* st, int32_t tokens);

/* Test hook for the bounded waits (no fault is involved): while tile >= 0,
 * the split pass issues no copy for cache tile `tile` of any unit, so the
 * warp that waits for it gives up after about a second of polls, raises
 * BGTQ_DEVERR_TIMEOUT, lets its other copies land and posts empty partials
 * for its CTA; the output then leaves that CTA's positions out.  -1 turns the
 * hook off (the default).  SYNC (host only). */
int bgtq_test_drop_tile_copies(bgtq_state* st, int32_t tile);

/* Selects the decode calls' kernels: fused = 1 asks for the fused launch
 * (query rotation, split-K pass, split merge and inverse V rotation in one
 * kernel of 4- or 8-CTA clusters, whichever holds more CTAs at once), taken
 * where the GPU can co-schedule such a cluster for the config; fused = 0 (the
 * default) runs the query rotation, the split pass and the combine as three
 * launches.  Both compute the same
 * attention up to the order of the split merge.  Other values:
 * BGTQ_ERR_INVALID_ARG.  SYNC (host only). */
int bgtq_set_decode_path(bgtq_state* st, int32_t fused);

/* Which kernels the decode calls of this state launch, and how many CTAs
 * the automatic split plan spreads over a call (*h_ctas: the CTAs the GPU
 * holds at once for that kernel).  *h_fused = 1 when
 * bgtq_decode_attn, bgtq_decode_step and bgtq_decode_attn_static_scratch run
 * as one fused launch per call (query rotation, split-K pass, split merge and
 * inverse V rotation in thread-block clusters of 4 or 8 CTAs; bgtq_decode_step
 * launches the appends before it); 0 when they run the query rotation, the
 * split pass and the combine as three launches (as the buffered and stage
 * calls always do): the fused path was not selected, or this GPU cannot
 * co-schedule its cluster for the config.  Both compute the same attention.
 * SYNC (host only; the first call may query the GPU's occupancy). */
int bgtq_get_decode_path(bgtq_state* st, int32_t* h_fused, int32_t* h_ctas);

/* Synchronises "stream", reads the device error flag into *h_flags
 * (BGTQ_DEVERR_* bits) and clears it.  SYNC. */
int bgtq_get_device_error(bgtq_state* st, void* stream, int32_t* h_flags);

/* Static description of a status code. */
const char* bgtq_error_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* BGTQ_H */

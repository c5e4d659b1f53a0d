// Device-side table formats and kernel launch parameters shared by the
// kernels (encode.cu, decode.cu, diag.cu, common.cuh) and the C ABI (api.cu).
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bgtq {

constexpr int kD = 128;               // head_dim
constexpr int kNumGroupsMax = 4;      // widths 4, 3, 2, 1
constexpr int kEnergyChunks = 32;     // calibration rows split into this many CTAs
constexpr int kPartialStride = 132;   // floats per split-K partial: m, l, pad, pad, acc[128]
constexpr int kCombSlices = 8;        // CTAs merging one row's splits in the combine
constexpr int kMaxBufferRows = 1024;  // fp16 buffered rows per sequence a decode call may attend
constexpr int kTile = 64;             // cache positions per packed tile
constexpr int kSplitGranule = kTile;  // split sizes are multiples of the tile
constexpr int kMaxChunks = 12;        // 16-coordinate K chunks per head (8 + one partial per group)

// Per-(layer, KV head) K layout.  Positions are record order: group 0
// (widest) first; perm maps a position to the original dim.
struct alignas(16) LayoutDev {
  int32_t n_groups;
  int32_t n_positions;
  int32_t pad0, pad1;
  int32_t width[kNumGroupsMax];
  int32_t size[kNumGroupsMax];
  int32_t start[kNumGroupsMax];
  int32_t bitoff[kNumGroupsMax];
  float inv_sqrt_d[kNumGroupsMax];    // 1 / sqrt(d_g)
  int32_t perm[kD];
  int32_t tile_word[kNumGroupsMax];   // first 32-bit word of the group's region in a K tile
  int32_t chunk_base[kNumGroupsMax];  // index of the group's first 16-coordinate chunk
};
static_assert(sizeof(LayoutDev) == 640, "layout record size");

// Per-(layer, KV head) tables of the split decode kernel, built on the host
// from the layout and the codebook (800 bytes, copied to shared memory by
// every CTA).
struct alignas(16) DecodeTableDev {
  int32_t grp[kNumGroupsMax][8];      // width, full chunks, size % 16, first tile word, first chunk, size, start, 0
  uint32_t tabk[kNumGroupsMax][8];    // byte tables of the group's codebook: low bytes [4], high bytes [4]
  uint32_t pdesc[kNumGroupsMax][32];  // partial-chunk descriptor of each lane (see group_logits)
  uint32_t tabv[8];                   // byte table of the V codebook
};
static_assert(sizeof(DecodeTableDev) == 800, "decode table size");

// q~ of one (layer, sequence, KV head, block of 8 query heads) as mma.sync
// B fragments: entry 32 c + 4 h + t holds, for chunk c and head h of the
// block, coordinates 16 j + 4 t .. + 3 of the chunk's group scaled by
// log2(e), split into fp16 hi and lo: (hi01, hi23, lo01, lo23).
constexpr int kFragEntries = kMaxChunks * 32;

// fp32 Lloyd-Max codebooks indexed by width (row 0 unused).
struct CodebookDev {
  float centroid[5][16];
  float threshold[5][16];
};

// Pointers into the caller's workspace buffer.
struct Workspace {
  uint32_t* err;                 // device error flag bits
  CodebookDev* codebook;
  LayoutDev* layouts;            // [L][Hkv]
  float* mkt;                    // [L][Hkv][128 in][128 out]: K rotation, block diagonal in record order, transposed
  float* mvt;                    // [L][Hkv][128 in][128 out]: V rotation transposed
  float* mv;                     // [L][Hkv][128 out][128 in]: V rotation (for the inverse rotation)
  __half* rb;                    // [L][Hkv][K, V][hi, lo][128 out][128 in, the rows' dimension order]: the
                                 // rotations as fp16 hi + lo operands of the tensor-core encode
  unsigned __int128* energy_q;   // [kEnergyChunks][L][Hkv][64]
  unsigned __int128* energy_k;   // [kEnergyChunks][L][Hkv][64]
  DecodeTableDev* dectab;        // [L][Hkv]
  float* qrot;                   // [L][B][Hq][128]
  uint4* qfrag;                  // [L][B][Hkv][head blocks][kFragEntries]
  float* partials;               // [L][B][Hq][max_splits][kPartialStride]
  float* comb_mid;               // [L][B][Hq][kCombSlices + 1][kPartialStride]: slot kCombSlices holds a
                                 // buffered call's fp16-row intermediate
  uint32_t* comb_count;          // [L][B][Hq]: the fused decode's clusters merged so far (0 between calls)
};

// Cache arrays; T = ceil(capacity / 64) tiles per (layer, sequence, KV head).
// The cache arrays hold one slot per 64-position tile.  Contiguous layout
// (n_pages == 0): slot ((layer * B + b) * Hkv + h) * T + t.  Paged layout
// (n_pages > 0): a pool of n_pages slots per (layer, KV head), slot
// (layer * Hkv + h) * n_pages + block_table[b * T + t]; the caller's block
// table maps a sequence's tile t to a page id, the same for every layer and
// KV head.
struct CacheDev {
  uint32_t* ktile;               // [slots][256*kbits] words (tile format)
  __half* knorm;                 // [slots][64][4]
  uint32_t* vtile;               // [slots][256*vbits] words
  __half* vnorm;                 // [slots][64]
  const int32_t* block_table;    // paged: int32 [B][T] page ids (caller-owned device memory)
  int32_t n_pages;               // pages per (layer, KV head); 0 = contiguous
  int32_t pad;
};

struct Shape {
  int32_t n_layers, n_kv_heads, n_q_heads, group, max_batch;
  int32_t kbits, vbits, max_splits;
  int64_t capacity;
  int64_t ntiles;                // tiles per (layer, sequence, KV head)
  int32_t drop_tile;             // test hook: the split pass issues no copy for this tile (-1: off)
  int32_t n_sms;                 // SMs of the device (the decode's warp-to-tile rotation)
};

// RoPE applied inside the encode (K rows taken before RoPE): block j of the
// pairing (0: dims (j, j+64); 1: (2j, 2j+1)) is turned by the angle
// position * base^(-2j/128).  on = 0: the rows are taken as they are.
struct RopeArgs {
  double base;
  int32_t pairing;
  int32_t on;
};

// Error flag bits (same values as BGTQ_DEVERR_* in bgtq.h).
constexpr uint32_t kErrCapacity = 1;
constexpr uint32_t kErrSeqLen = 2;
constexpr uint32_t kErrArg = 4;
constexpr uint32_t kErrNonFinite = 8;
constexpr uint32_t kErrTimeout = 16;
constexpr uint32_t kErrPage = 32;

// Launchers (encode.cu, decode.cu, diag.cu).  Each returns the cudaError_t of its launch.
cudaError_t launch_energy(const Shape& s, const Workspace& ws, const __half* calib_q, int nq,
                          const __half* calib_k, int nk, int pairing, cudaStream_t stream);
cudaError_t launch_encode(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                          int layer_count, const __half* k, const __half* v, const int32_t* start,
                          const int32_t* count, int batch, int n, cudaStream_t stream,
                          RopeArgs rope = RopeArgs{0.0, 0, 0});
cudaError_t launch_rotate_query(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                                const __half* q, int batch, float* qrot, cudaStream_t stream);
// Calls with at most this many rows per sequence append row by row (the
// decode-time path); launch_prep takes 1 <= n <= kAppendMaxRows.
constexpr int kAppendMaxRows = 16;
// One launch that rotates the query rows (as launch_rotate_query) and appends
// n rows per sequence (as launch_encode's row path).
cudaError_t launch_prep(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                        const __half* q, int batch, float* qrot, const __half* k, const __half* v,
                        const int32_t* start, const int32_t* count, int n, cudaStream_t stream);
// The split pass reads q~ as fragments from ws.qfrag (written by the query
// rotation), or, when qrot is not null, builds them from qrot itself.
// The fp16 buffered rows a decode call attends besides the packed cache
// (k == nullptr: none).  q: the decode query fp16 [layer_count][batch][Hq][128];
// k, v: fp16 [layer_count][batch][n_buf][Hkv][128]; count: int32 [batch]
// rows used per sequence; pos_lo: int32 [batch] first packed position
// attended (null = 0).
struct BufferArgs {
  const __half* q;
  const __half* k;
  const __half* v;
  const int32_t* count;
  const int32_t* pos_lo;
  int n_buf;
};
// How a decode call splits each unit (layer, sequence, KV head, block of 8
// query heads) over CTAs.  The grid has c_max split CTAs per unit; a unit of
// sequence b uses c_b of them (the rest exit at once), computed on the device
// from the lengths by split_ctas: with fixed_tiles > 0, ceil(tiles_b /
// fixed_tiles); else about `budget` CTAs over all units in proportion to their
// tiles (budget * tiles_b / (units_per_seq * sum of tiles)), so that ragged
// sequences finish together.  Always 1 <= c_b <= min(tiles_b, c_max) for a
// unit with tiles, 0 without.
struct SplitPlan {
  int32_t c_max;
  int32_t budget;
  int32_t fixed_tiles;
  int32_t units_per_seq;  // layer_count * Hkv * head blocks
  int32_t cluster;        // > 1: counts rounded up to whole clusters of this size (the fused decode)
  // 1: the split pass follows the call's own query rotation (or decode-step
  // preparation), which lets it start only once everything earlier in the
  // stream has completed; it then reads the caller's lengths and issues its
  // first tiles' copies before its dependency wait.
  int32_t early;
  // the rows the preparation kernel appends in the same launch as the
  // rotation ([start, start + count) per sequence; null: none): a first
  // tile holding one of them is copied only after the wait
  const int32_t* app_start;
  const int32_t* app_count;
};

// The split pass over the packed positions [pos_lo, seq_lens) (buf.pos_lo;
// null = 0); with buf.k set, one more CTA per unit attends the buffered rows
// and posts them as the row's extra combine intermediate.
cudaError_t launch_decode_split(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                                int layer_count, const float* qrot, const int32_t* seq_lens, const BufferArgs& buf,
                                int batch, const SplitPlan& plan, cudaStream_t stream);
// Resident split-decode CTAs per SM for a config (0 on error).
int decode_ctas_per_sm(const Shape& s);
// The fused decode (query rotation, split-K pass, merge and inverse V
// rotation in one launch, in clusters of plan.cluster = 4 or 8 CTAs): q fp16
// [layer_count][batch][Hq][128], out fp16 of the same shape; the plan's
// c_max must be a multiple of its cluster size.  Partials, one per cluster,
// and the per-unit arrival counters (zero between calls) are in the
// workspace.
cudaError_t launch_decode_fused(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                                int layer_count, const __half* q, const int32_t* seq_lens, int batch,
                                const SplitPlan& plan, __half* out, cudaStream_t stream);
// Co-resident clusters of `cluster` (4 or 8) CTAs of the fused decode for a
// config (0: it cannot run).
int decode_fused_clusters(const Shape& s, int cluster);
cudaError_t launch_combine(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                           const int32_t* seq_lens, int batch, const SplitPlan& plan, const BufferArgs& buf,
                           __half* out, cudaStream_t stream);
// Per-layer logit MAE of the packed keys of sequence seq at cache positions
// [w0, w0 + m) against the exact keys k (fp16 [layer_count][m][Hkv][128]),
// for the queries q (fp16 [layer_count][m][Hq][128]) at the same positions
// and every causal pair; mae: double [layer_count][Hq] (zeroed, summed and
// scaled by the launches).
cudaError_t launch_logit_mae(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                             int layer_count, int seq, int w0, int m, const __half* q, const __half* k, double* mae,
                             cudaStream_t stream);

}  // namespace bgtq

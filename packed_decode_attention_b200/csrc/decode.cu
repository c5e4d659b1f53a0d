// Decode kernels of the Block-GTQ path (B200, sm_100a):
//
//   decode_fused_kernel  query rotation, split-K flash decoding from the packed
//                        tiles (mma.sync), split merge and inverse V rotation
//                        in one launch (thread-block clusters)
//   decode_mma_kernel    the split-K pass of the three-launch decode (after
//                        the query rotation or the decode step's prep) and
//                        of the stage calls, with the fp16 sink / window rows
//                        of a buffered call
//   combine_kernel       log-sum-exp merge of the splits (a cluster of up to
//                        8 CTAs per row) + inverse V rotation
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ;
// chatpaper summary / arXiv 2606.24033 abstract, blockgtq README) on top of
// TurboQuant-MSE (arXiv 2504.19874); split-K decoding after FlashAttention /
// FlashAttention-2 (arXiv 2205.14135, 2307.08691), both cited by the pages.
#include "common.cuh"

namespace bgtq {

namespace {

// ---------------------------------------------------------------------------
// Split-K decode straight from the packed tiles on the tensor cores.
//
// Grid (batch * Hkv * head_blocks, c_max, layer_count), 128 threads.  The
// split CTAs of a (layer, sequence, KV head, block of up to 8 query heads) share
// its 64-position tiles; each warp has its own bulk-copy pipeline (two
// stages of K tile + norms, one V buffer -> shared memory, completion on
// mbarriers) and its own online-softmax state.
//
// Logits (per warp per tile): S^T[64 tokens x 8 heads] = K_hat q~^T as
// mma.sync m16n8k16 tiles -- A = centroids C[codes] (exact in fp16), looked
// up in registers with PRMT byte tables from the lane's selector words;
// B = q~ * log2(e) split into fp16 hi + lo (two MMAs).  Each width group
// accumulates separately and is scaled by its per-token norm.
// P V: O^T[128 dims x 8 heads] += V_hat^T P'^T with P' = 2^(logit - max) *
// n_V / sqrt(D) in fp16, moved from the logit accumulator layout into a B
// operand with movmatrix.  Everything stays in V's rotated basis; the
// combine kernel rotates back.
// ---------------------------------------------------------------------------
// Per warp: two stages for the K tile and the norms, one buffer for the V
// tile (refilled as soon as the previous tile's P V is done: the next
// tile's logits and softmax cover its copy).
constexpr int kStages = 2;
constexpr int kBarsPerWarp = kStages + 1;
constexpr int kDecMinBlocks = 3;  // CTAs per SM the register budget is sized for
constexpr int kWaitLimit = 1 << 20;  // polls of up to kPollSuspendNs each: about a second
constexpr float kRescaleSlack = 8.f;


__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// A hint to bring [p, p + bytes) into L2 (16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Before the dependency wait of a one-sequence call: an L2 prefetch hint for
// the first kPrefetchTiles tiles the warp would get if the sequence were
// full (lane k takes the warp's k-th tile), so that the cache streams into
// L2 while the previous kernel finishes.  A prefetch reads nothing into the
// CTA and leaves memory as it is: L2 is where global memory is coherent, so
// a line a later kernel rewrites is read afresh by the copies after the
// wait, and a line the sequence does not reach costs only bandwidth.
constexpr int kPrefetchTiles = 4;

__device__ __forceinline__ void prefetch_warp_tiles(const Shape& sh, const CacheDev& cache, int layer, int b, int h,
                                                    int c_full, int warp, int nw, int cu, int kbits, int vbits) {
  const int lane = threadIdx.x & 31;
  if (cu >= c_full || lane >= kPrefetchTiles) return;
  const int64_t tile = warp * c_full + cu + static_cast<int64_t>(lane) * c_full * nw;
  if (tile >= sh.ntiles) return;
  const int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
  if (slot < 0) return;
  const uint32_t kb = 1024u * kbits, vb = 1024u * vbits;
  prefetch_l2(cache.ktile + slot * (kb / 4), kb);
  prefetch_l2(cache.vtile + slot * (vb / 4), vb);
  prefetch_l2(cache.knorm + slot * kTile * 4, kTile * 8);
  prefetch_l2(cache.vnorm + slot * kTile, kTile * 2);
}

// One bounded poll: the thread may sleep up to kPollSuspendNs waiting for the phase.
constexpr uint32_t kPollSuspendNs = 1000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kPollSuspendNs)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity; gives up after kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (int i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Shared memory of the buffer CTA: q of 8 heads, logits / weights [8][rows], (M, L) per head.
constexpr int kBufSmemBytes = (8 * kD + 8 * kMaxBufferRows + 16) * 4;

struct DecodeLayout {  // byte offsets inside the dynamic shared memory
  int bars, bq, tabk, grp, pdesc, ms, ls, mres, wsc, stage, kst_bytes, v_bytes, total;
};

// The stage region of a CTA of nw warps: K stage s of warp w at stage +
// (s * nw + w) * kst_bytes (K tile, K norms, V norms), then warp w's V
// buffer at stage + kStages * nw * kst_bytes + w * v_bytes.
__host__ __device__ inline DecodeLayout decode_layout(int kbits, int vbits, int nw) {
  DecodeLayout L;
  L.bars = 0;
  L.bq = align128(nw * kBarsPerWarp * 8);
  L.grp = L.bq + kMaxChunks * 32 * 16;    // a copy of DecodeTableDev: grp, tabk, pdesc, tabv
  L.tabk = L.grp + kNumGroupsMax * 8 * 4;
  L.pdesc = L.tabk + kNumGroupsMax * 8 * 4;
  L.ms = L.grp + static_cast<int>(sizeof(DecodeTableDev));
  L.ls = L.ms + nw * 8 * 4;
  L.mres = L.ls + nw * 8 * 4;           // merged m, l per head [2][8]
  L.wsc = L.mres + 2 * 8 * 4;           // merge weights [warp][8]
  L.stage = align128(L.wsc + nw * 8 * 4);
  L.kst_bytes = 1024 * kbits + kTile * 8 + kTile * 2;
  L.v_bytes = 1024 * vbits;
  const int stages = nw * (kStages * L.kst_bytes + L.v_bytes);
  const int merge = nw * 8 * kD * 4;  // reuses the stage buffers after the loop
  int need = stages > merge ? stages : merge;
  if (need < kBufSmemBytes) need = kBufSmemBytes;  // the buffer CTA of a buffered call
  L.total = L.stage + need;
  return L;
}

// The range of a decode call's sequence: the packed positions [lo, len) and
// the buffered row count, clamped the same way by every kernel that reads
// them (the combine raises the flag).
struct SeqRange {
  int len, lo, cnt;
  bool bad;
};

// The caller's arrays are read through L2 (ld.global.cg): the split pass may
// read them before its dependency wait, and no copy in this SM's L1 may be
// older than the stream's last write.
__device__ __forceinline__ SeqRange seq_range(const Shape& sh, const int32_t* seq_lens, const BufferArgs& buf, int b) {
  SeqRange r;
  r.len = __ldcg(seq_lens + b);
  r.lo = buf.pos_lo != nullptr ? __ldcg(buf.pos_lo + b) : 0;
  r.cnt = buf.k != nullptr ? __ldcg(buf.count + b) : 0;
  r.bad = r.len < 0 || r.len > sh.capacity || r.lo < 0 || r.lo > r.len || r.cnt < 0 || r.cnt > buf.n_buf;
  if (r.len < 0 || r.len > sh.capacity) r.len = 0;
  if (r.lo < 0 || r.lo > r.len) r.lo = r.len;
  r.cnt = r.cnt < 0 ? 0 : (r.cnt > buf.n_buf ? buf.n_buf : r.cnt);
  return r;
}

// Packed tiles a call attends for one sequence: the tiles of [lo, len).
__device__ __forceinline__ int64_t range_tiles(const SeqRange& r) {
  return r.lo < r.len ? (r.len + kTile - 1) / kTile - r.lo / kTile : 0;
}

// Split CTAs of a unit with ntl tiles when the batch has `total` tiles per
// unit summed over its sequences (see SplitPlan).  The split pass and the
// combine evaluate it on the same inputs, so they agree.
__device__ __forceinline__ int split_ctas(const SplitPlan& p, int64_t ntl, int64_t total) {
  if (ntl <= 0) return 0;
  int64_t c = p.fixed_tiles > 0 ? (ntl + p.fixed_tiles - 1) / p.fixed_tiles
                                : static_cast<int64_t>(p.budget) * ntl / (total * p.units_per_seq);
  c = c < 1 ? 1 : c;
  c = c < ntl ? c : ntl;
  c = c < p.c_max ? c : p.c_max;
  // whole clusters (c_max is a multiple of the cluster size): a set split
  // size rounds up; the one-wave budget rounds down, to stay one wave
  if (p.cluster > 1) {
    c = p.fixed_tiles > 0 ? (c + p.cluster - 1) / p.cluster * p.cluster : c / p.cluster * p.cluster;
    c = c < p.cluster ? p.cluster : c;
  }
  return static_cast<int>(c);
}

// The batch's tiles summed over its sequences, by all NT threads of the CTA
// (red: kNtWarps int64 of shared memory).  Needed only in budget mode.
template <int NT>
__device__ int64_t batch_tiles(const Shape& sh, const int32_t* seq_lens, const BufferArgs& buf, int batch,
                               int64_t* red) {
  const int tid = threadIdx.x;
  long long t = 0;
  for (int b = tid; b < batch; b += NT) t += range_tiles(seq_range(sh, seq_lens, buf, b));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  if ((tid & 31) == 0) red[tid >> 5] = t;
  __syncthreads();
  int64_t sum = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) sum += red[w];
  __syncthreads();
  return sum;
}


// The fp16 buffered rows of one (layer, sequence, KV head, block of 8 query
// heads), attended by one extra CTA of the split pass (128 threads): logits
// q . k / sqrt(D) in log2 units (a thread per row), softmax per head, P v (a
// thread per dimension, unrotated).  Each head's (m, l, acc) goes to the
// row's extra combine intermediate, read by the combine after this grid.
// NT threads (128 or more): the P v part runs on the first 128.
template <int NT>
__device__ void buffer_attend(const Shape& sh, const Workspace& ws, const BufferArgs& buf, const SeqRange& sr, int li,
                              int b, int h, int h0, int nh, int batch, unsigned char* smem) {
  static_assert(NT >= kD && NT % 32 == 0, "at least a thread per dimension");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = sh.group;
  float* qs = reinterpret_cast<float*>(smem);   // [128 dims][8 heads]
  float* lg = qs + 8 * kD;                      // [8][kMaxBufferRows]
  float* ml = lg + 8 * kMaxBufferRows;          // [8][2]
  const int cnt = sr.cnt;
  const size_t qrow = ((static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G + h0) * kD;
  for (int i = tid; i < 8 * kD; i += NT) {
    const int hh = i / kD, dim = i % kD;
    qs[dim * 8 + hh] = hh < nh ? __half2float(buf.q[qrow + i]) * (kInvSqrtD * kLog2e) : 0.f;
  }
  __syncthreads();
  const size_t rstride = static_cast<size_t>(sh.n_kv_heads) * kD;
  const size_t base = (static_cast<size_t>(li) * batch + b) * buf.n_buf * rstride + static_cast<size_t>(h) * kD;
  for (int r = tid; r < cnt; r += NT) {
    const uint4* kr = reinterpret_cast<const uint4*>(buf.k + base + r * rstride);
    float d[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // half of the row's dimensions per pass: 8 loads of 8 values in flight
#pragma unroll 1
    for (int c8 = 0; c8 < 2; ++c8) {
      uint4 kw[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) kw[c] = kr[8 * c8 + c];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const __half2* h2 = reinterpret_cast<const __half2*>(&kw[c]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float kv = e & 1 ? __high2float(h2[e >> 1]) : __low2float(h2[e >> 1]);
          const float4* qa = reinterpret_cast<const float4*>(qs + (8 * (8 * c8 + c) + e) * 8);
          const float4 a0 = qa[0], a1 = qa[1];
          d[0] = fmaf(a0.x, kv, d[0]);
          d[1] = fmaf(a0.y, kv, d[1]);
          d[2] = fmaf(a0.z, kv, d[2]);
          d[3] = fmaf(a0.w, kv, d[3]);
          d[4] = fmaf(a1.x, kv, d[4]);
          d[5] = fmaf(a1.y, kv, d[5]);
          d[6] = fmaf(a1.z, kv, d[6]);
          d[7] = fmaf(a1.w, kv, d[7]);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) lg[hh * kMaxBufferRows + r] = d[hh];
  }
  __syncthreads();
  // per head: maximum, weights 2^(logit - M) in place, denominator
  for (int hh = warp; hh < 8; hh += NT / 32) {
    float M = -CUDART_INF_F;
    for (int r = lane; r < cnt; r += 32) M = fmaxf(M, lg[hh * kMaxBufferRows + r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int r = lane; r < cnt; r += 32) {
      const float p = exp2f(lg[hh * kMaxBufferRows + r] - M);
      lg[hh * kMaxBufferRows + r] = p;
      L += p;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      ml[2 * hh] = M;
      ml[2 * hh + 1] = L;
    }
  }
  __syncthreads();
  // P v: thread (8 dimensions dg, row phase rp of 8), 8 values per load; the
  // phases are then summed through shared memory (over the weights)
  const int dg = tid & 15, rp = tid >> 4;
  const int rend = tid < kD ? cnt : 0;  // threads past the first 128 take no rows
  float acc[8][8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
#pragma unroll 4
  for (int r = rp; r < rend; r += 8) {
    const uint4 vw = *reinterpret_cast<const uint4*>(buf.v + base + r * rstride + 8 * dg);
    const __half2* h2 = reinterpret_cast<const __half2*>(&vw);
    float vv[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      vv[2 * e] = f.x;
      vv[2 * e + 1] = f.y;
    }
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      const float p = lg[hh * kMaxBufferRows + r];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[hh][e] = fmaf(p, vv[e], acc[hh][e]);
    }
  }
  __syncthreads();
  float* red = lg;  // [8 phases][8 heads][128 dims]
  if (tid < kD) {
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
      float4* dst = reinterpret_cast<float4*>(red + (rp * 8 + hh) * kD + 8 * dg);
      dst[0] = make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
      dst[1] = make_float4(acc[hh][4], acc[hh][5], acc[hh][6], acc[hh][7]);
    }
  }
  __syncthreads();
  const int d = tid;  // the first 128 threads: a thread per output dimension
  const size_t wrow0 = (static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + h0;
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    if (hh >= nh || d >= kD) break;
    float* mid = ws.comb_mid + ((wrow0 + hh) * (kCombSlices + 1) + kCombSlices) * kPartialStride;
    float a = 0.f;
#pragma unroll
    for (int ph = 0; ph < 8; ++ph) a += red[(ph * 8 + hh) * kD + d];
    mid[4 + d] = cnt > 0 ? a : 0.f;
    if (d == 0) {
      mid[0] = cnt > 0 ? ml[2 * hh] : -CUDART_INF_F;
      mid[1] = cnt > 0 ? ml[2 * hh + 1] : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// The per-warp tile loop shared by the split pass and the fused decode.
//
// A warp attends the tiles tlo + wu + k W (k < my_tiles) of one (layer,
// sequence, KV head) unit for up to 8 query heads: its own 2-stage pipeline
// of bulk copies (K tile, V tile, norms -> shared memory, completion on an
// mbarrier, bounded waits) and its own online-softmax state (O in V's rotated
// basis, the running maximum and denominator of heads 2 t4 and 2 t4 + 1).
// ---------------------------------------------------------------------------
struct TileSource {
  Shape sh;
  CacheDev cache;
  uint32_t* err;
  int layer, b, h;
  int tlo, wu, W;        // the warp's first tile is tlo + wu, then every W-th
  int kwords, vwords;    // 32-bit words of a K / V tile
  unsigned char* kstage; // this warp's K stage 0; stage s at kstage + s * kstride
  int kstride;
  unsigned char* vbuf;   // this warp's V buffer
  uint64_t* bars;        // the K stages' mbarriers, then the V buffer's
};

__device__ __forceinline__ int64_t source_slot(const TileSource& src, int tile) {
  int64_t slot = tile_slot(src.sh, src.cache, src.layer, src.b, src.h, tile);
  if (slot < 0) {  // a page id outside the pool: flagged, page 0 read instead
    atomicOr(src.err, kErrPage);
    slot = static_cast<int64_t>(src.layer * src.sh.n_kv_heads + src.h) * src.cache.n_pages;
  }
  return slot;
}

// Lane 0: copy the K tile and the norms of the warp's k-th tile into K stage k % kStages.
__device__ __forceinline__ void issue_k(const TileSource& src, int k) {
  const uint32_t kbytes = 4u * src.kwords;
  const uint32_t tx = kbytes + kTile * 8 + kTile * 2;
  const int tile = src.tlo + src.wu + k * src.W;
  uint64_t* bar = &src.bars[k % kStages];
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_expect_tx(bar, tx);
  if (tile == src.sh.drop_tile) return;  // test hook: no copy, so the wait on it runs out
  const int64_t slot = source_slot(src, tile);
  unsigned char* dst = src.kstage + (k % kStages) * src.kstride;
  bulk_copy_g2s(dst, src.cache.ktile + slot * src.kwords, kbytes, bar);
  bulk_copy_g2s(dst + kbytes, src.cache.knorm + slot * kTile * 4, kTile * 8, bar);
  bulk_copy_g2s(dst + kbytes + kTile * 8, src.cache.vnorm + slot * kTile, kTile * 2, bar);
}

// Lane 0: copy the V tile of the warp's k-th tile into its V buffer.
__device__ __forceinline__ void issue_v(const TileSource& src, int k) {
  const uint32_t vbytes = 4u * src.vwords;
  const int tile = src.tlo + src.wu + k * src.W;
  uint64_t* bar = &src.bars[kStages];
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_expect_tx(bar, vbytes);
  if (tile == src.sh.drop_tile) return;
  const int64_t slot = source_slot(src, tile);
  bulk_copy_g2s(src.vbuf, src.cache.vtile + slot * src.vwords, vbytes, bar);
}

// Lanes 1 .. kPrefetchTiles - 1: L2 prefetch hints for the warp's tiles 1, 2, ...
__device__ __forceinline__ void prefetch_next_tiles(const TileSource& src, int my_tiles) {
  const int lane = threadIdx.x & 31;
  if (lane == 0 || lane >= kPrefetchTiles || lane >= my_tiles) return;
  const int64_t slot = tile_slot(src.sh, src.cache, src.layer, src.b, src.h, src.tlo + src.wu + lane * src.W);
  if (slot < 0) return;
  prefetch_l2(src.cache.ktile + slot * src.kwords, 4u * src.kwords);
  prefetch_l2(src.cache.vtile + slot * src.vwords, 4u * src.vwords);
  prefetch_l2(src.cache.knorm + slot * kTile * 4, kTile * 8);
  prefetch_l2(src.cache.vnorm + slot * kTile, kTile * 2);
}

// Lane 0: the copies a warp starts with, its first tile (K and V).  Each
// later tile's K goes out once the previous tile's K has landed, its V once
// the previous tile is done (attend_tiles), so every warp's first tile
// comes in before any warp's second.
__device__ __forceinline__ void issue_first(const TileSource& src, int my_tiles) {
  if (my_tiles > 0) {
    issue_k(src, 0);
    issue_v(src, 0);
  }
}

// The decode tables a warp reads from shared memory (a copy of the
// DecodeTableDev of its (layer, KV head)) and the query fragments.
struct TileTables {
  const int32_t* grp;
  const uint32_t* tabk;
  const uint32_t* pdesc;
  const uint4* bq;
  int ng;
};

// Attends the warp's my_tiles tiles over the positions [lo, len); the copies
// of issue_first must already be issued (this issues the rest).  Returns the
// index of the tile whose copy wait gave up (-1: none).
template <int VB>
__device__ __forceinline__ int attend_tiles(const TileSource& src, const TileTables& tt, const ByteTab& tv,
                                            int my_tiles, int len, int lo, float (&O)[8][4], float (&m_run)[2],
                                            float (&l_run)[2]) {
  const int lane = threadIdx.x & 31;
  const int g8 = lane >> 2;
  const uint32_t kbytes = 4u * src.kwords;
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int r = 0; r < 4; ++r) O[m][r] = 0.f;
  m_run[0] = m_run[1] = -CUDART_INF_F;
  l_run[0] = l_run[1] = 0.f;
  int failed_at = -1;
  bool k_consumed = false;  // at a failure: whether that tile's K stage had landed

  for (int k = 0; k < my_tiles; ++k) {
    if (!__all_sync(0xffffffffu, mbar_wait(&src.bars[k % kStages], (k / kStages) & 1))) {
      failed_at = k;
      break;
    }
    // the other K stage held tile k - 1, which is done: tile k + 1's K goes there
    if (lane == 0 && k + 1 < my_tiles) issue_k(src, k + 1);
    const unsigned char* st = src.kstage + (k % kStages) * src.kstride;
    const uint32_t* kt = reinterpret_cast<const uint32_t*>(st);
    const __half* kn = reinterpret_cast<const __half*>(st + kbytes);
    const __half* vn = reinterpret_cast<const __half*>(st + kbytes + kTile * 8);
    const int tpos = (src.tlo + src.wu + k * src.W) * kTile;
    const int nvalid = min(kTile, len - tpos);       // positions [nlow, nvalid) of the tile are attended
    const int nlow = max(0, lo - tpos);

    // logits, one width group at a time, each scaled by its per-token norm
    float L[4][4];
#pragma unroll
    for (int mu = 0; mu < 4; ++mu)
#pragma unroll
      for (int r = 0; r < 4; ++r) L[mu][r] = 0.f;
    for (int g = 0; g < tt.ng; ++g) {
      const int4 gp = *reinterpret_cast<const int4*>(tt.grp + g * 8);  // width, nfull, r, word
      const int chunk = tt.grp[g * 8 + 4];
      ByteTab t;
      const uint4 tl = *reinterpret_cast<const uint4*>(tt.tabk + 8 * g);
      const uint4 th = *reinterpret_cast<const uint4*>(tt.tabk + 8 * g + 4);
      t.lo[0] = tl.x; t.lo[1] = tl.y;
      t.hi[0] = th.x; t.hi[1] = th.y;
      const uint32_t pd = tt.pdesc[g * 32 + lane];
      const uint32_t* gw = kt + gp.w;
      const uint4* bqg = tt.bq + chunk * 32 + lane;
      float S[4][4];
      switch (gp.x) {
        case 1: group_logits<1>(gw, gp.y, gp.z != 0, pd, bqg, t, lane, S); break;
        case 2: group_logits<2>(gw, gp.y, gp.z != 0, pd, bqg, t, lane, S); break;
        case 3: group_logits<3>(gw, gp.y, gp.z != 0, pd, bqg, t, lane, S); break;
        default: group_logits<4>(gw, gp.y, gp.z != 0, pd, bqg, t, lane, S); break;
      }
#pragma unroll
      for (int mu = 0; mu < 4; ++mu) {
        const float na = __half2float(kn[(16 * mu + g8) * 4 + g]);
        const float nb = __half2float(kn[(16 * mu + g8 + 8) * 4 + g]);
        L[mu][0] = fmaf(na, S[mu][0], L[mu][0]);
        L[mu][1] = fmaf(na, S[mu][1], L[mu][1]);
        L[mu][2] = fmaf(nb, S[mu][2], L[mu][2]);
        L[mu][3] = fmaf(nb, S[mu][3], L[mu][3]);
      }
    }
    // online softmax over the tile for heads 2*t4 and 2*t4+1; positions past
    // the valid length carry no weight (their norms may be anything)
    float wv[4][2];
#pragma unroll
    for (int mu = 0; mu < 4; ++mu) {
      wv[mu][0] = __half2float(vn[16 * mu + g8]) * kInvSqrtD;
      wv[mu][1] = __half2float(vn[16 * mu + g8 + 8]) * kInvSqrtD;
    }
    if (nvalid < kTile || nlow > 0) {
#pragma unroll
      for (int mu = 0; mu < 4; ++mu) {
        if (16 * mu + g8 >= nvalid || 16 * mu + g8 < nlow) {
          L[mu][0] = L[mu][1] = -CUDART_INF_F;
          wv[mu][0] = 0.f;
        }
        if (16 * mu + g8 + 8 >= nvalid || 16 * mu + g8 + 8 < nlow) {
          L[mu][2] = L[mu][3] = -CUDART_INF_F;
          wv[mu][1] = 0.f;
        }
      }
    }
    float mx[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
    for (int mu = 0; mu < 4; ++mu) {
      mx[0] = fmaxf(mx[0], fmaxf(L[mu][0], L[mu][2]));
      mx[1] = fmaxf(mx[1], fmaxf(L[mu][1], L[mu][3]));
    }
    // The reference maximum moves only when some logit of the tile exceeds it
    // by more than kRescaleSlack (log2 units), so O is rescaled rarely;
    // weights stay <= 2^kRescaleSlack and l and O always share the same
    // reference.  l is kept per lane and summed over the warp at the end.
    if (__any_sync(0xffffffffu, mx[0] > m_run[0] + kRescaleSlack || mx[1] > m_run[1] + kRescaleSlack)) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
      }
      float alpha[2] = {1.f, 1.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (mx[c] > m_run[c] + kRescaleSlack) {
          alpha[c] = fast_exp2(m_run[c] - mx[c]);
          m_run[c] = mx[c];
        }
        l_run[c] *= alpha[c];
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        O[m][0] *= alpha[0];
        O[m][1] *= alpha[1];
        O[m][2] *= alpha[0];
        O[m][3] *= alpha[1];
      }
    }
    uint32_t bp[4][2];
#pragma unroll
    for (int mu = 0; mu < 4; ++mu) {
      const float p0 = fast_exp2(L[mu][0] - m_run[0]), p1 = fast_exp2(L[mu][1] - m_run[1]);
      const float p2 = fast_exp2(L[mu][2] - m_run[0]), p3 = fast_exp2(L[mu][3] - m_run[1]);
      l_run[0] += p0 + p2;
      l_run[1] += p1 + p3;
      bp[mu][0] = transpose8x8(pack_half2(p0 * wv[mu][0], p1 * wv[mu][0]));
      bp[mu][1] = transpose8x8(pack_half2(p2 * wv[mu][1], p3 * wv[mu][1]));
    }
    // P V in V's rotated basis, from the V buffer
    if (!__all_sync(0xffffffffu, mbar_wait(&src.bars[kStages], k & 1))) {
      failed_at = k;
      k_consumed = true;
      break;
    }
    const uint32_t* vt = reinterpret_cast<const uint32_t*>(src.vbuf);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      uint32_t w[VB], sv[4];
#pragma unroll
      for (int kk = 0; kk < VB; ++kk) w[kk] = vt[m * 32 * VB + 32 * kk + lane];
      quartet_decode<VB>(w, sv);
#pragma unroll
      for (int kappa = 0; kappa < 4; ++kappa) mma_selector<VB>(O[m], tv, sv[kappa], bp[kappa][0], bp[kappa][1]);
    }
    __syncwarp();
    if (lane == 0 && k + 1 < my_tiles) issue_v(src, k + 1);
  }
  if (failed_at >= 0) {
    // copies issued but not yet consumed: let them land (bounded) before the
    // buffers are reused or the CTA exits.  At the failure at tile f the K
    // stage of tile f + 1 (once tile f's K had landed) and the V buffer of
    // tile f were issued.
    if (lane == 0) atomicOr(src.err, kErrTimeout);
    const int f = failed_at;
    const int k_issued = k_consumed ? min(my_tiles, f + 2) : f + 1;
    for (int k = k_consumed ? f + 1 : f; k < k_issued; ++k) mbar_wait(&src.bars[k % kStages], (k / kStages) & 1);
    mbar_wait(&src.bars[kStages], f & 1);
  }
  return failed_at;
}

// Merges the CTA's NW warps (called by all threads after attend_tiles) into
// one (m, l, acc[128]) per query head of the block: cm[8], clsum[8] and
// cacc[8][128] (shared memory; cacc may alias the stage buffers, which are
// free once every warp has left its loop).  accs: [NW][8][128] of shared
// scratch (may alias the stage buffers too, and cacc); ms, ls, wsc: [NW][8]
// each.  A CTA with a timed-out warp posts empty partials.
template <int NW>
__device__ __forceinline__ void merge_warps(const float (&O)[8][4], const float (&m_run)[2], float (&l_run)[2],
                                            bool timed_out, float* accs, float* ms, float* ls, float* wsc, float* cm,
                                            float* clsum, float* cacc, int nh) {
  constexpr int NT = NW * 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], o);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], o);
  }
  __syncthreads();  // every warp has left its loop: the stage buffers are free
  if (g8 == 0) {
    ms[warp * 8 + 2 * t4] = m_run[0];
    ms[warp * 8 + 2 * t4 + 1] = m_run[1];
    ls[warp * 8 + 2 * t4] = l_run[0];
    ls[warp * 8 + 2 * t4 + 1] = l_run[1];
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    float* a = accs + warp * 8 * kD;
    a[(2 * t4) * kD + 16 * m + g8] = O[m][0];
    a[(2 * t4 + 1) * kD + 16 * m + g8] = O[m][1];
    a[(2 * t4) * kD + 16 * m + g8 + 8] = O[m][2];
    a[(2 * t4 + 1) * kD + 16 * m + g8 + 8] = O[m][3];
  }
  const bool cta_timed_out = __syncthreads_or(timed_out);
  // per head: the common maximum, the warps' weights (warps without a tile
  // hold m = -inf, l = 0, acc = 0) and the weighted denominator
  if (tid < 8 && cta_timed_out) {
    for (int w = 0; w < NW; ++w) wsc[w * 8 + tid] = 0.f;
    cm[tid] = -CUDART_INF_F;
    clsum[tid] = 0.f;
  } else if (tid < 8) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, ms[w * 8 + tid]);
    float lsum = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float mw = ms[w * 8 + tid];
      const float sc = mw == -CUDART_INF_F ? 0.f : fast_exp2(mw - M);
      wsc[w * 8 + tid] = sc;
      lsum = fmaf(sc, ls[w * 8 + tid], lsum);
    }
    cm[tid] = M;
    clsum[tid] = lsum;
  }
  __syncthreads();
  // (head, dimension) pairs u = tid, tid + NT, ...
  constexpr int kPer = 8 * kD / NT;
  float a[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int u = tid + k * NT, hh = u / kD, i = u % kD;
    a[k] = 0.f;
    if (hh < nh) {
#pragma unroll 4
      for (int w = 0; w < NW; ++w) a[k] = fmaf(wsc[w * 8 + hh], accs[(w * 8 + hh) * kD + i], a[k]);
    }
  }
  __syncthreads();  // cacc may alias accs
#pragma unroll
  for (int k = 0; k < kPer; ++k) cacc[tid + k * NT] = a[k];
  __syncthreads();
}

// Grid (batch * Hkv * head_blocks, [1 buffer CTA +] plan.c_max, layer_count),
// 128 threads.  A unit is one (layer, sequence, KV head, block of up to 8
// query heads); it uses C = split_ctas(...) of its c_max split CTAs (more for
// longer sequences; the others exit at once).  Its tiles are dealt
// round-robin over the W = 4 C warps of those CTAs, CTA-major within a round
// (warp w of CTA c takes tiles w C + c, w C + c + W, ...), so
// every warp gets the same number of tiles to within one and the last,
// partial round lands on as many CTAs as it can.  Each CTA writes one
// partial (m, l, acc) per query head -- an empty one (m = -inf, l = 0) when
// it has no tile.
template <int VB, int NW>
__global__ void __launch_bounds__(NW * 32, NW == kDecWarps ? kDecMinBlocks : 1)
    decode_mma_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0, const float* __restrict__ qrot,
                      const int32_t* __restrict__ seq_lens, BufferArgs buf, int batch, SplitPlan plan,
                      int head_blocks) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int NT = NW * 32;
  const DecodeLayout DL = decode_layout(sh.kbits, VB, NW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + DL.bars);
  uint4* bq = reinterpret_cast<uint4*>(smem_raw + DL.bq);
  uint32_t* tabk = reinterpret_cast<uint32_t*>(smem_raw + DL.tabk);
  int32_t* grp = reinterpret_cast<int32_t*>(smem_raw + DL.grp);
  uint32_t* pdesc = reinterpret_cast<uint32_t*>(smem_raw + DL.pdesc);
  float* ms = reinterpret_cast<float*>(smem_raw + DL.ms);
  float* ls = reinterpret_cast<float*>(smem_raw + DL.ls);
  unsigned char* stage_base = smem_raw + DL.stage;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // grid row 0 holds the buffer CTAs of a buffered call, so they are
  // dispatched first; the split CTAs follow
  const bool has_buf = buf.k != nullptr;
  const int cu = has_buf ? static_cast<int>(blockIdx.y) - 1 : static_cast<int>(blockIdx.y);  // -1: buffer CTA
  const int hb = blockIdx.x % head_blocks;
  const int h = (blockIdx.x / head_blocks) % sh.n_kv_heads;
  const int b = blockIdx.x / (head_blocks * sh.n_kv_heads);
  const int li = blockIdx.z;
  const int layer = layer0 + li;
  const int G = sh.group;
  const int h0 = 8 * hb;                       // first query head of this block within the group
  const int nh = min(8, G - h0);
  const int lh = layer * sh.n_kv_heads + h;
  const LayoutDev& lay = ws.layouts[lh];

  // ---- per-CTA set-up: the (layer, KV head) decode table (a library table) ----
  const int ng = lay.n_groups;
  {
    const uint4* src = reinterpret_cast<const uint4*>(ws.dectab + lh);
    uint4* dst = reinterpret_cast<uint4*>(grp);  // grp, tabk, pdesc, tabv are contiguous
    for (int u = tid; u < static_cast<int>(sizeof(DecodeTableDev) / 16); u += NT) dst[u] = src[u];
  }
  if (tid < NW * kBarsPerWarp) mbar_init(&bars[tid], 1);
  __syncthreads();
  if (tid == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  // Launched as a programmatic dependent of the previous kernel.  Without
  // plan.early everything before griddepcontrol.wait reads only the library's
  // tables.  With it, the previous kernel is this call's query rotation (or
  // decode-step preparation), whose CTAs let this grid start only after
  // their own wait, so all earlier work of the stream has completed: the
  // caller's lengths, block table and cache are read before the wait too,
  // and each warp's first tile is copied then, unless it holds a row that
  // the preparation appends in the same launch.  The rotated queries are
  // always read after the wait.
  const bool early = plan.early != 0 && cu >= 0;
  if (!early) {
    // L2 prefetch hints for this warp's first tiles while the previous
    // kernel may still run (the copies below still read after the wait)
    if (batch == 1 && cu >= 0)
      prefetch_warp_tiles(sh, cache, layer, b, h, split_ctas(plan, sh.ntiles, sh.ntiles), warp, NW, cu, sh.kbits, VB);
    asm volatile("griddepcontrol.wait;" ::: "memory");
  }
  const int nchunk = lay.chunk_base[ng - 1] + ((lay.size[ng - 1] + 15) >> 4);
  constexpr int kFragPerThread = (kFragEntries + NT - 1) / NT;
  // the packed positions attended: [lo, len); lo > 0 when the caller keeps the
  // first positions unquantised (out-of-range values are flagged by the
  // combine kernel)
  const SeqRange sr = seq_range(sh, seq_lens, buf, b);
  if (cu < 0) {
    // the extra CTA of a buffered call: the unit's fp16 buffered rows
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    buffer_attend<NT>(sh, ws, buf, sr, li, b, h, h0, nh, batch, smem_raw + DL.stage);
    return;
  }
  const int len = sr.len, lo = sr.lo;
  const int tlo = lo / kTile;
  const int ntl = static_cast<int>(range_tiles(sr));
  // this unit's split CTAs (the same count the combine computes)
  __shared__ int64_t s_red[NW];
  const int64_t total = plan.fixed_tiles > 0 ? 0 : batch_tiles<NT>(sh, seq_lens, buf, batch, s_red);
  const int C = split_ctas(plan, ntl, total);
  if (cu >= C) {
    // not needed for this unit (its partials are slots 0 .. C-1)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  // Tile t of the unit goes to warp (t mod W) / C of CTA (t mod W) mod C:
  // a partial last round of tiles is spread over all CTAs (and so over all
  // SMs) before any CTA gets a second one.
  const int W = C * NW;
  const int wu = warp * C + cu;
  const int my_tiles = wu < ntl ? (ntl - wu + W - 1) / W : 0;
  float* part_base = ws.partials +
                     (((static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + h0) * sh.max_splits + cu) *
                         kPartialStride;
  TileSource src;
  src.sh = sh;
  src.cache = cache;
  src.err = ws.err;
  src.layer = layer;
  src.b = b;
  src.h = h;
  src.tlo = tlo;
  src.wu = wu;
  src.W = W;
  src.kwords = 256 * sh.kbits;
  src.vwords = 256 * VB;
  src.kstage = stage_base + static_cast<size_t>(warp) * DL.kst_bytes;
  src.kstride = NW * DL.kst_bytes;
  src.vbuf = stage_base + kStages * NW * DL.kst_bytes + static_cast<size_t>(warp) * DL.v_bytes;
  src.bars = bars + warp * kBarsPerWarp;
  bool first_issued = false;
  if (early) {
    const int64_t p0 = static_cast<int64_t>(tlo + wu) * kTile;
    bool appended = false;  // the first tile holds a row the preparation appends
    if (plan.app_start != nullptr) {
      const int as = __ldcg(plan.app_start + b), ac = __ldcg(plan.app_count + b);
      appended = ac > 0 && p0 < static_cast<int64_t>(as) + ac && static_cast<int64_t>(as) < p0 + kTile;
    }
    first_issued = my_tiles > 0 && !appended;
    if (lane == 0 && first_issued) issue_first(src, my_tiles);
    prefetch_next_tiles(src, my_tiles);
    asm volatile("griddepcontrol.wait;" ::: "memory");
  }
  // the unit's q~ fragments (written by the query rotation)
  uint4 fr[kFragPerThread];
  if (qrot == nullptr) {
    const uint4* fsrc = frag_block(sh, ws, li, b, h, hb);
#pragma unroll
    for (int i = 0; i < kFragPerThread; ++i) {
      const int u = tid + i * NT;
      if (u < 32 * nchunk) fr[i] = fsrc[u];
    }
  }
  const size_t part_head_stride = static_cast<size_t>(sh.max_splits) * kPartialStride;
  {
    if (qrot == nullptr) {
#pragma unroll
      for (int i = 0; i < kFragPerThread; ++i) {
        const int u = tid + i * NT;
        if (u < 32 * nchunk) bq[u] = fr[i];
      }
    } else {
      // the split pass on its own: the fragments from the caller's q~
      // (fp32, record order): coordinates 16 j + 4 t .. + 3 of chunk c's
      // group for head t / 4 ... see write_frags for the layout
      const float* qsrc = qrot + ((static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G + h0) * kD;
      for (int u = tid; u < 32 * nchunk; u += NT) {
        const int c = u >> 5, ln = u & 31;
        int g = 0;
        while (g + 1 < ng && c >= lay.chunk_base[g + 1]) ++g;
        const int j = c - lay.chunk_base[g];
        const int d = lay.size[g], st = lay.start[g];
        const int head = ln >> 2;
        float v[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int coord = 16 * j + 4 * (ln & 3) + m;
          v[m] = (head < nh && coord < d) ? qsrc[head * kD + st + coord] * kLog2e : 0.f;
        }
        const __half2 a = __floats2half2_rn(v[0], v[1]);
        const __half2 c2 = __floats2half2_rn(v[2], v[3]);
        const float2 af = __half22float2(a), cf = __half22float2(c2);
        const __half2 al = __floats2half2_rn(v[0] - af.x, v[1] - af.y);
        const __half2 cl = __floats2half2_rn(v[2] - cf.x, v[3] - cf.y);
        bq[u] = make_uint4(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&c2),
                           *reinterpret_cast<const uint32_t*>(&al), *reinterpret_cast<const uint32_t*>(&cl));
      }
    }
  }
  ByteTab tv;
  {
    const uint4 a0 = *reinterpret_cast<const uint4*>(tabk + kNumGroupsMax * 8 + kNumGroupsMax * 32);
    const uint4 a1 = *reinterpret_cast<const uint4*>(tabk + kNumGroupsMax * 8 + kNumGroupsMax * 32 + 4);
    tv.lo[0] = a0.x; tv.lo[1] = a0.y;
    tv.hi[0] = a1.x; tv.hi[1] = a1.y;
  }
  __syncthreads();

  // ---- per-warp pipeline over this warp's tiles ----
  if (lane == 0 && !first_issued) issue_first(src, my_tiles);
  TileTables tt{grp, tabk, pdesc, bq, ng};
  float O[8][4], m_run[2], l_run[2];
  const int failed_at = attend_tiles<VB>(src, tt, tv, my_tiles, len, lo, O, m_run, l_run);
  // the combine kernel may be scheduled now; it waits for this grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ---- merge the warps (the stage buffers are reused) and post the partials ----
  float* cacc = reinterpret_cast<float*>(stage_base);
  float* wsc = reinterpret_cast<float*>(smem_raw + DL.wsc);
  float* mres = reinterpret_cast<float*>(smem_raw + DL.mres);
  merge_warps<NW>(O, m_run, l_run, failed_at >= 0, reinterpret_cast<float*>(stage_base), ms, ls, wsc, mres,
                  mres + 8, cacc, nh);
  for (int u = tid; u < nh * kD; u += NT) {
    const int hh = u / kD, i = u % kD;
    float* part = part_base + hh * part_head_stride;
    part[4 + i] = cacc[u];
    if (i == 0) {
      part[0] = mres[hh];
      part[1] = mres[8 + hh];
    }
  }
}

// ---------------------------------------------------------------------------
// Fused decode: the query rotation, the split-K pass and the split merge with
// the inverse V rotation in one launch.
//
// Grid (batch * Hkv * head_blocks, plan.c_max, layer_count) in thread-block
// clusters of CL (4 or 8) CTAs along y, 128 threads.  A unit (layer,
// sequence, KV head, block of up to 8 query heads) uses C = split_ctas(...)
// of its c_max CTAs, a multiple of the cluster size (whole clusters; unused
// clusters exit at once).  Its tiles are dealt over the 4 C warps exactly as
// in the split pass.
//
//  1. Before the dependency wait: the decode table, and rows
//     [16 r, 16 r + 16) of the unit's K rotation (CTA rank r of the cluster).
//  2. After it: the unit's query rows (gathered into record order); CTA r
//     computes q~ for coordinates [16 r, 16 r + 16) of all heads and writes
//     them into every CTA of its cluster (distributed shared memory); each
//     CTA then builds its own mma B fragments.  The first tile copy of every
//     warp is already in flight meanwhile.
//  3. The tile loop (attend_tiles) and the merge of the CTA's warps.
//  4. Cluster merge: CTA r merges head r over the cluster's CTAs (reading
//     their shared memory) and posts one partial per cluster.
//  5. The unit's last cluster to arrive (a counter it resets) merges the
//     clusters' partials (CTA r: head r), shares the normalised accumulators
//     through distributed shared memory, and CTA r writes output dims
//     [16 r, 16 r + 16) of every head: o = R_V^T (sum_c w_c acc_c) /
//     (sum_c w_c l_c), with w_c = 2^(m_c - max m).
// No CTA waits on another outside its cluster's hardware barriers, so the
// grid needs no co-residency beyond the cluster's.
// ---------------------------------------------------------------------------
constexpr int kRowPad = kD + 1;  // row pitch (floats) of the rotation scratch: consecutive rows in different banks

struct FusedLayout {  // byte offsets inside the dynamic shared memory
  int bars, bq, tab, ms, ls, wsc, cm, flag, qt, stage, kst_bytes, v_bytes, rot, vbase, total;
};

// CL = CTAs per cluster (4 or 8): CTA rank r rotates and writes back the
// kD / CL coordinates [r kD / CL, (r + 1) kD / CL).
__host__ __device__ inline FusedLayout fused_layout(int kbits, int vbits, int CL) {
  FusedLayout L;
  L.bars = 0;
  L.bq = align128(kDecWarps * kBarsPerWarp * 8);
  L.tab = L.bq + kMaxChunks * 32 * 16;
  L.ms = L.tab + static_cast<int>(sizeof(DecodeTableDev));
  L.ls = L.ms + kDecWarps * 8 * 4;
  L.wsc = L.ls + kDecWarps * 8 * 4;
  L.cm = L.wsc + kDecWarps * 8 * 4;           // the CTA's merged m[8], l[8]
  L.flag = L.cm + 16 * 4;                      // "this cluster merges the unit" (written by rank 0)
  L.qt = align128(L.flag + 16);                // q~ [8][kRowPad] fp32, later the merged accumulators
  L.stage = align128(L.qt + 8 * kRowPad * 4);
  L.kst_bytes = 1024 * kbits + kTile * 8 + kTile * 2;
  L.v_bytes = 1024 * vbits;
  // K stage s of warp w at stage + (s * kDecWarps + w) * kst_bytes: the
  // second K stages form one block, which holds the K rotation rows
  // [kD / CL][kRowPad] and the query rows [8][kRowPad] until the first tiles
  // are in flight, and the inverse V rotation slice [kD / CL][kRowPad] in
  // the last cluster's merge; the V buffers follow (warp w at vbase + w *
  // v_bytes)
  L.rot = L.stage + kDecWarps * L.kst_bytes;
  const int rot_bytes = (kD / CL + 8) * kRowPad * 4;
  int kblock = kStages * kDecWarps * L.kst_bytes;
  if (kblock < kDecWarps * L.kst_bytes + rot_bytes) kblock = kDecWarps * L.kst_bytes + rot_bytes;
  L.vbase = L.stage + kblock;
  int need = kblock + kDecWarps * L.v_bytes;
  const int merge = kDecWarps * 8 * kD * 4;  // the warp merge reuses the stage buffers
  if (need < merge) need = merge;
  L.total = L.stage + need;
  return L;
}

__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}

__device__ __forceinline__ void dsmem_st(uint32_t a, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

__device__ __forceinline__ void dsmem_st_u32(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

__device__ __forceinline__ float dsmem_ld(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}

// Every thread of every CTA of the cluster: shared-memory writes before it
// (local or remote) are visible to every CTA after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int VB, int CL>
__global__ void __launch_bounds__(kDecThreads, kDecMinBlocks)
    decode_fused_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0, const __half* __restrict__ q,
                        const int32_t* __restrict__ seq_lens, int batch, SplitPlan plan, int head_blocks,
                        __half* __restrict__ out) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int CPR = kD / CL;  // coordinates (and output dims) per CTA rank
  const FusedLayout FL = fused_layout(sh.kbits, VB, CL);
  static_assert(kDecThreads == kD, "the fused decode's thread-per-dimension steps");
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + FL.bars);
  uint4* bq = reinterpret_cast<uint4*>(smem_raw + FL.bq);
  int32_t* grp = reinterpret_cast<int32_t*>(smem_raw + FL.tab);  // grp, tabk, pdesc, tabv are contiguous
  const uint32_t* tabk = reinterpret_cast<const uint32_t*>(smem_raw + FL.tab + offsetof(DecodeTableDev, tabk));
  const uint32_t* pdesc = reinterpret_cast<const uint32_t*>(smem_raw + FL.tab + offsetof(DecodeTableDev, pdesc));
  const uint32_t* tabv = reinterpret_cast<const uint32_t*>(smem_raw + FL.tab + offsetof(DecodeTableDev, tabv));
  float* ms = reinterpret_cast<float*>(smem_raw + FL.ms);
  float* ls = reinterpret_cast<float*>(smem_raw + FL.ls);
  float* wsc = reinterpret_cast<float*>(smem_raw + FL.wsc);
  float* cm = reinterpret_cast<float*>(smem_raw + FL.cm);
  uint32_t* flag = reinterpret_cast<uint32_t*>(smem_raw + FL.flag);
  float* qt = reinterpret_cast<float*>(smem_raw + FL.qt);
  unsigned char* stage_base = smem_raw + FL.stage;
  float* rk = reinterpret_cast<float*>(smem_raw + FL.rot);  // [CPR][kRowPad]
  float* qr = rk + CPR * kRowPad;                             // [8][kRowPad]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cu = blockIdx.y;
  const int rank = cu % CL;  // the CTA's rank in its cluster (clusters run along y)
  const int clu = cu / CL;
  const int hb = blockIdx.x % head_blocks;
  const int h = (blockIdx.x / head_blocks) % sh.n_kv_heads;
  const int b = blockIdx.x / (head_blocks * sh.n_kv_heads);
  const int li = blockIdx.z;
  const int layer = layer0 + li;
  const int G = sh.group;
  const int h0 = 8 * hb;
  const int nh = min(8, G - h0);
  const int lh = layer * sh.n_kv_heads + h;
  const LayoutDev& lay = ws.layouts[lh];
  const int ng = lay.n_groups;

  // ---- 1. library tables only (the previous kernel may still run) ----
  {
    const uint4* src = reinterpret_cast<const uint4*>(ws.dectab + lh);
    uint4* dst = reinterpret_cast<uint4*>(grp);
    for (int u = tid; u < static_cast<int>(sizeof(DecodeTableDev) / 16); u += kDecThreads) dst[u] = src[u];
  }
  if (tid < kDecWarps * kBarsPerWarp) mbar_init(&bars[tid], 1);
  // rows [CPR rank, CPR rank + CPR) of the block-diagonal K rotation
  // (record order): R[i][j] = mkt[j][i]
  {
    const float* mk = ws.mkt + static_cast<size_t>(lh) * kD * kD;
    constexpr int Q4 = CPR / 4;  // float4 per input row
#pragma unroll
    for (int k = 0; k < CPR / 4; ++k) {
      const int f = tid + k * kDecThreads;  // 128 inputs x CPR outputs
      const int j = f / Q4, q4 = f % Q4;
      const float4 v = *reinterpret_cast<const float4*>(mk + j * kD + CPR * rank + 4 * q4);
      rk[(4 * q4 + 0) * kRowPad + j] = v.x;
      rk[(4 * q4 + 1) * kRowPad + j] = v.y;
      rk[(4 * q4 + 2) * kRowPad + j] = v.z;
      rk[(4 * q4 + 3) * kRowPad + j] = v.w;
    }
  }
  const int perm_j = lay.perm[tid] & (kD - 1);  // kDecThreads == kD: the original dim of record position tid
  // This thread's rotation output coordinate i = CPR rank + o (o = tid mod
  // CPR; its heads are tid / CPR + 128 / CPR k): the group range [j0, j1)
  // and scale, and its fragment entries' q~ offsets and valid counts -- all
  // from the layout, a library table, before the wait.
  static_assert(kDecThreads % CPR == 0, "one output coordinate per thread");
  int rot_j0 = 0, rot_j1 = 0;
  float rot_scale = 0.f;
  {
    const int i = CPR * rank + tid % CPR;
    if (i < lay.n_positions) {
      int g = 0;
      for (int t = 1; t < ng; ++t)
        if (i >= lay.start[t]) g = t;
      rot_j0 = lay.start[g];
      rot_j1 = rot_j0 + lay.size[g];
      rot_scale = kInvSqrtD * lay.inv_sqrt_d[g] * kLog2e;
    }
  }
  constexpr int kFragPerThread = (kFragEntries + kDecThreads - 1) / kDecThreads;
  const int nchunk = lay.chunk_base[ng - 1] + ((lay.size[ng - 1] + 15) >> 4);
  int fr_off[kFragPerThread], fr_cnt[kFragPerThread];
#pragma unroll
  for (int k = 0; k < kFragPerThread; ++k) {
    const int u = tid + k * kDecThreads;
    fr_off[k] = 0;
    fr_cnt[k] = 0;
    if (u < 32 * nchunk) {
      const int c = u >> 5, ln = u & 31;
      int g = 0;
      while (g + 1 < ng && c >= lay.chunk_base[g + 1]) ++g;
      const int c0 = 16 * (c - lay.chunk_base[g]) + 4 * (ln & 3);
      fr_off[k] = (ln >> 2) * kRowPad + lay.start[g] + c0;
      fr_cnt[k] = min(4, max(0, lay.size[g] - c0));
    }
  }
  __syncthreads();
  if (tid == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (batch == 1)
    prefetch_warp_tiles(sh, cache, layer, b, h, split_ctas(plan, sh.ntiles, sh.ntiles), warp, kDecWarps, cu, sh.kbits,
                        VB);
  // Launched as a programmatic dependent of the previous kernel (the
  // appends of a decode step, or the previous call): the query, the lengths
  // and the cache are read after it has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- 2. the unit's query rows and range, then its split and tiles ----
  // (the query loads go out before the tile copies, which fill the memory
  // system; they land in qr further down)
  const size_t qrow0 = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G + h0;
  __half qv[8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) qv[hh] = hh < nh ? q[(qrow0 + hh) * kD + perm_j] : __float2half(0.f);
  const SeqRange sr = seq_range(sh, seq_lens, BufferArgs{}, b);
  if (sr.bad && blockIdx.y == 0 && tid == 0 && h == 0 && hb == 0) atomicOr(ws.err, kErrSeqLen);
  const int len = sr.len, lo = sr.lo;
  const int tlo = lo / kTile;
  const int ntl = static_cast<int>(range_tiles(sr));
  __shared__ int64_t s_red[kDecWarps];
  const int64_t total = plan.fixed_tiles > 0 ? 0 : batch_tiles<kDecThreads>(sh, seq_lens, BufferArgs{}, batch, s_red);
  const int C = split_ctas(plan, ntl, total);  // a multiple of the cluster size
  const size_t wrow0 = (static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + h0;
  if (C == 0) {
    // no packed position: the first cluster writes zero outputs
    if (clu == 0)
      for (int hh = rank; hh < nh; hh += CL) out[(qrow0 + hh) * kD + tid] = __float2half(0.f);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  if (cu >= C) {  // a whole cluster the unit does not use
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  const int nclu = C / CL;
  const int W = C * kDecWarps;
  const int wu = warp * C + cu;
  const int my_tiles = wu < ntl ? (ntl - wu + W - 1) / W : 0;
  TileSource src;
  src.sh = sh;
  src.cache = cache;
  src.err = ws.err;
  src.layer = layer;
  src.b = b;
  src.h = h;
  src.tlo = tlo;
  src.wu = wu;
  src.W = W;
  src.kwords = 256 * sh.kbits;
  src.vwords = 256 * VB;
  src.kstage = stage_base + static_cast<size_t>(warp) * FL.kst_bytes;
  src.kstride = kDecWarps * FL.kst_bytes;
  src.vbuf = smem_raw + FL.vbase + static_cast<size_t>(warp) * FL.v_bytes;
  src.bars = bars + warp * kBarsPerWarp;
  // the first tile of each warp goes out now (its K stage and the V buffers
  // do not hold the rotation scratch, which the second K stages do until
  // the fragments are built; the tile loop issues the second K stage once
  // the first has landed)
  if (lane == 0) issue_first(src, my_tiles);

  // ---- q~ for coordinates [CPR rank, CPR rank + CPR) of the block's heads ----
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) qr[hh * kRowPad + tid] = __half2float(qv[hh]);
  __syncthreads();
  {
    const int o = tid % CPR;
    const int i = CPR * rank + o;
    const float* rrow = rk + o * kRowPad;
#pragma unroll
    for (int k = 0; k < 8 * CPR / kDecThreads; ++k) {
      const int hh = tid / CPR + k * (kDecThreads / CPR);
      const float* qrow = qr + hh * kRowPad;
      float a0 = 0.f, a1 = 0.f;
      for (int j = rot_j0; j < rot_j1; j += 2) {  // group sizes are even (whole RoPE blocks)
        a0 = fmaf(rrow[j], qrow[j], a0);
        a1 = fmaf(rrow[j + 1], qrow[j + 1], a1);
      }
      const float v = (a0 + a1) * rot_scale;  // log2(e) q~
#pragma unroll
      for (int r2 = 0; r2 < CL; ++r2) dsmem_st(dsmem_addr(qt + hh * kRowPad + i, r2), v);
    }
  }
  cluster_sync_all();
  // the B fragments from log2(e) q~ (see write_frags for the layout); heads past nh are zero
#pragma unroll
  for (int k = 0; k < kFragPerThread; ++k) {
    const int u = tid + k * kDecThreads;
    if (u < 32 * nchunk) {
      float v[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) v[m] = m < fr_cnt[k] ? qt[fr_off[k] + m] : 0.f;
      const __half2 a = __floats2half2_rn(v[0], v[1]);
      const __half2 c2 = __floats2half2_rn(v[2], v[3]);
      const float2 af = __half22float2(a), cf = __half22float2(c2);
      const __half2 al = __floats2half2_rn(v[0] - af.x, v[1] - af.y);
      const __half2 cl = __floats2half2_rn(v[2] - cf.x, v[3] - cf.y);
      bq[u] = make_uint4(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&c2),
                         *reinterpret_cast<const uint32_t*>(&al), *reinterpret_cast<const uint32_t*>(&cl));
    }
  }
  ByteTab tv;
  {
    const uint4 a0 = *reinterpret_cast<const uint4*>(tabv);
    const uint4 a1 = *reinterpret_cast<const uint4*>(tabv + 4);
    tv.lo[0] = a0.x; tv.lo[1] = a0.y;
    tv.hi[0] = a1.x; tv.hi[1] = a1.y;
  }
  __syncthreads();  // fragments ready; the rotation scratch (second stages) is free

  // ---- 3. the tiles, then the CTA's warps merged ----
  TileTables tt{grp, tabk, pdesc, bq, ng};
  float O[8][4], m_run[2], l_run[2];
  const int failed_at = attend_tiles<VB>(src, tt, tv, my_tiles, len, lo, O, m_run, l_run);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  float* cacc = reinterpret_cast<float*>(stage_base);  // [8][kD]
  merge_warps<kDecWarps>(O, m_run, l_run, failed_at >= 0, reinterpret_cast<float*>(stage_base), ms, ls, wsc, cm,
                        cm + 8, cacc, nh);
  cluster_sync_all();

  // ---- 4. cluster merge: CTA rank r takes heads r, r + CL, ... over the cluster's CTAs ----
  for (int hh = rank; hh < nh; hh += CL) {
    float mr[CL], wr[CL];
    float M = -CUDART_INF_F;
#pragma unroll
    for (int c = 0; c < CL; ++c) {
      mr[c] = dsmem_ld(dsmem_addr(cm + hh, c));
      M = fmaxf(M, mr[c]);
    }
    float Lsum = 0.f, a = 0.f;
#pragma unroll
    for (int c = 0; c < CL; ++c) {
      wr[c] = mr[c] == -CUDART_INF_F ? 0.f : fast_exp2(mr[c] - M);
      Lsum = fmaf(wr[c], dsmem_ld(dsmem_addr(cm + 8 + hh, c)), Lsum);
      a = fmaf(wr[c], dsmem_ld(dsmem_addr(cacc + hh * kD + tid, c)), a);
    }
    float* part = ws.partials + ((wrow0 + hh) * sh.max_splits + clu) * kPartialStride;
    part[4 + tid] = a;
    if (tid == 0) {
      part[0] = M;
      part[1] = Lsum;
    }
  }
  // remote reads done; the cluster's partial writes happen before the
  // barrier, and the fence of the thread that counts the arrival orders them
  // (cumulatively) before its atomic
  cluster_sync_all();
  if (tid == 0 && rank == 0) {
    __threadfence();
    const uint32_t last = atomicAdd(ws.comb_count + wrow0, 1u) == static_cast<uint32_t>(nclu - 1) ? 1u : 0u;
    __threadfence();  // the other clusters' partials, seen through the count, before the loads below
#pragma unroll
    for (int r2 = 0; r2 < CL; ++r2) dsmem_st_u32(dsmem_addr(flag, r2), last);
  }
  cluster_sync_all();
  if (*flag == 0u) return;  // the same for the whole cluster

  // ---- 5. the unit's last cluster: merge the clusters, rotate back ----
  // CTA rank r merges heads r, r + CL, ...: warp w takes the clusters
  // w, w + 4, ... (eight at a time, all their loads in flight), a lane four
  // dims; the warps' (m, l, acc) then meet in shared memory (the stage
  // buffers are free: no CTA reads this CTA's shared memory any more).
  // columns [CPR rank, CPR rank + CPR) of R_V (row-major [in][out]), a
  // library table: loaded first, stored as rv[o][i] = R_V[i][CPR rank + o]
  // after the merges
  constexpr int kRvLoads = CPR / 4;
  float4 rvv[kRvLoads];
  {
    const float* mv = ws.mv + static_cast<size_t>(lh) * kD * kD;
#pragma unroll
    for (int k = 0; k < kRvLoads; ++k) {
      const int f = tid + k * kDecThreads;
      rvv[k] = __ldg(reinterpret_cast<const float4*>(mv + (f / (CPR / 4)) * kD + CPR * rank + 4 * (f % (CPR / 4))));
    }
  }
  float* wacc = reinterpret_cast<float*>(stage_base);  // [kDecWarps][kD]
  float* wml = wacc + kDecWarps * kD;                  // [kDecWarps][2]
  for (int hh = rank; hh < nh; hh += CL) {
    const float* part = ws.partials + (wrow0 + hh) * sh.max_splits * kPartialStride;
    float m_w = -CUDART_INF_F, l_w = 0.f;
    float4 a_w = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = warp; c0 < nclu; c0 += 8 * kDecWarps) {
      float mm[8], ll[8];
      float4 aa[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = c0 + j * kDecWarps;
        if (c < nclu) {
          const float* p = part + static_cast<size_t>(c) * kPartialStride;
          mm[j] = __ldcg(p);
          ll[j] = __ldcg(p + 1);
          aa[j] = __ldcg(reinterpret_cast<const float4*>(p + 4) + lane);
        } else {
          mm[j] = -CUDART_INF_F;
          ll[j] = 0.f;
          aa[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mb = m_w;
#pragma unroll
      for (int j = 0; j < 8; ++j) mb = fmaxf(mb, mm[j]);
      if (mb == -CUDART_INF_F) continue;  // only empty clusters so far
      const float f = m_w == -CUDART_INF_F ? 0.f : exp2f(m_w - mb);
      l_w *= f;
      a_w.x *= f; a_w.y *= f; a_w.z *= f; a_w.w *= f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float wgt = mm[j] == -CUDART_INF_F ? 0.f : exp2f(mm[j] - mb);
        l_w = fmaf(wgt, ll[j], l_w);
        a_w.x = fmaf(wgt, aa[j].x, a_w.x);
        a_w.y = fmaf(wgt, aa[j].y, a_w.y);
        a_w.z = fmaf(wgt, aa[j].z, a_w.z);
        a_w.w = fmaf(wgt, aa[j].w, a_w.w);
      }
      m_w = mb;
    }
    *reinterpret_cast<float4*>(wacc + warp * kD + 4 * lane) = a_w;
    if (lane == 0) {
      wml[2 * warp] = m_w;
      wml[2 * warp + 1] = l_w;
    }
    __syncthreads();
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wml[2 * w]);
    float Lsum = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float wgt = wml[2 * w] == -CUDART_INF_F ? 0.f : exp2f(wml[2 * w] - M);
      Lsum = fmaf(wgt, wml[2 * w + 1], Lsum);
      a = fmaf(wgt, wacc[w * kD + tid], a);
    }
    const float an = a / Lsum;
#pragma unroll
    for (int r2 = 0; r2 < CL; ++r2) dsmem_st(dsmem_addr(qt + hh * kRowPad + tid, r2), an);
    __syncthreads();  // wacc is reused by the next head
  }
  float* rv = rk;
#pragma unroll
  for (int k = 0; k < kRvLoads; ++k) {
    const int f = tid + k * kDecThreads;
    const int i = f / (CPR / 4), q4 = f % (CPR / 4);
    rv[(4 * q4 + 0) * kRowPad + i] = rvv[k].x;
    rv[(4 * q4 + 1) * kRowPad + i] = rvv[k].y;
    rv[(4 * q4 + 2) * kRowPad + i] = rvv[k].z;
    rv[(4 * q4 + 3) * kRowPad + i] = rvv[k].w;
  }
  if (tid == 0 && rank == 0) ws.comb_count[wrow0] = 0u;  // ready for the next call
  cluster_sync_all();
  for (int u = tid; u < nh * CPR; u += kDecThreads) {
    const int hh = u / CPR, o = u % CPR;
    const float* rrow = rv + o * kRowPad;
    const float* arow = qt + hh * kRowPad;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int i = 0; i < kD; i += 2) {
      s0 = fmaf(rrow[i], arow[i], s0);
      s1 = fmaf(rrow[i + 1], arow[i + 1], s1);
    }
    out[(qrow0 + hh) * kD + CPR * rank + o] = __float2half(s0 + s1);
  }
}

// ---------------------------------------------------------------------------
// Combine the splits and rotate back.  Grid (layer_count*batch*Hq * S),
// 256 threads, in clusters of S = kCombSlices CTAs (1 when every unit has
// few splits): one cluster per row.  CTA (slice) r merges slice r of the row's splits (w_s = 2^(m_s -
// M), 0 for empty splits; lane = 4 rotated coordinates) into an
// intermediate (m, l, acc) in V's rotated basis in its shared memory.  CTA 0
// then reads the cluster's intermediates through distributed shared memory
// (and, in a buffered call, the row's fp16 buffered rows, which the split
// pass posted to global memory with acc unrotated) and computes
// o = (R_V^T sum_s w_s acc_s + w_buf acc_buf) / (sum_s w_s l_s + w_buf l_buf).
// ---------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;
// Up to this many rows per launch, CTA 0 of every row loads its rotation
// column before the dependency wait (64 KB per row of L2 reads).
constexpr int kEarlyRotationRows = 256;
static_assert(kCombWarps * 4 <= kD, "a warp's lanes cover the 128 coordinates four at a time");
static_assert(kCombSlices <= 8, "a row's slices form one portable cluster");

// EARLY: CTA 0 holds its rotation column in registers, loaded before the
// dependency wait (small launches); otherwise it reads the column inside the
// product, so that the kernel needs fewer registers and more clusters fit
// an SM at once (large launches).
// S: CTAs (slices) per row, the cluster size: kCombSlices, or 1 when no
// unit has more splits than one CTA merges in one round of loads.
template <bool EARLY, int S>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(Shape sh, Workspace ws, int layer0,
                                                               const int32_t* __restrict__ seq_lens, int batch,
                                                               SplitPlan plan, BufferArgs buf, __half* __restrict__ out) {
  const int has_buf = buf.k != nullptr ? 1 : 0;
  const int slice = blockIdx.x % S;  // the CTA's rank in its cluster
  const int rowi = blockIdx.x / S;
  const int hq = rowi % sh.n_q_heads;
  const int b = (rowi / sh.n_q_heads) % batch;
  const int li = rowi / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dd = tid & (kD - 1), half = tid >> 7;
  // A library table: this thread's half column of the inverse V rotation,
  // used by the row's CTA 0.  For a small launch it is read before the
  // split pass has finished, off the critical path.
  const float* mv = ws.mv + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
  float mvr[EARLY ? 64 : 1];
  if constexpr (EARLY) {
    if (slice == 0) {
#pragma unroll
      for (int r = 0; r < 64; ++r) mvr[r] = __ldg(mv + (half * 64 + r) * kD + dd);
    }
  }
  // the next kernel of the stream may start its own table-only set-up now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // The split pass lets this grid start only after its own dependency wait,
  // so the caller's lengths are complete: they are read before this grid's
  // wait.  The partials and the output are touched only after it.
  const SeqRange sr = seq_range(sh, seq_lens, buf, b);
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  __shared__ int64_t s_red[kCombWarps];
  const int64_t total = plan.fixed_tiles > 0 ? 0 : batch_tiles<kCombThreads>(sh, seq_lens, buf, batch, s_red);
  const int n_splits = split_ctas(plan, range_tiles(sr), total);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (sr.bad && tid == 0 && hq == 0 && slice == 0) atomicOr(ws.err, kErrSeqLen);
  if (sr.lo >= sr.len && sr.cnt == 0) {  // the whole cluster: an empty row
    if (slice == 0 && tid < kD) out[row * kD + tid] = __float2half(0.f);
    return;
  }
  const size_t wrow = (static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + hq;  // workspace row
  const float* part = ws.partials + wrow * sh.max_splits * kPartialStride;
  __shared__ float accs[kCombWarps][kD];
  __shared__ float msw[kCombWarps], lsw[kCombWarps];
  __shared__ __align__(16) float cmid[4 + kD];  // this slice's (m, l, -, -, acc[128])
  __shared__ float a_s[kD];
  // ---- one slice of the row's splits: warp w takes splits s0 + w + 8 j,
  // four at a time with all their loads in flight, merged online per warp
  // (lane = 4 rotated coordinates), then across the warps ----
  const int s0 = static_cast<int>((static_cast<int64_t>(slice) * n_splits) / S);
  const int s1 = static_cast<int>((static_cast<int64_t>(slice + 1) * n_splits) / S);
  float m_w = -CUDART_INF_F, l_w = 0.f;
  float4 a_w = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int base = s0 + warp; base < s1; base += 4 * kCombWarps) {
    float mm[4], ll[4];
    float4 aa[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int sj = base + j * kCombWarps;
      if (sj < s1) {
        const float* p = part + static_cast<size_t>(sj) * kPartialStride;
        mm[j] = p[0];
        ll[j] = p[1];
        aa[j] = *reinterpret_cast<const float4*>(p + 4 + 4 * lane);
      } else {
        mm[j] = -CUDART_INF_F;
        ll[j] = 0.f;
        aa[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float mb = fmaxf(fmaxf(m_w, fmaxf(mm[0], mm[1])), fmaxf(mm[2], mm[3]));
    if (mb == -CUDART_INF_F) continue;  // only empty splits so far
    const float f = m_w == -CUDART_INF_F ? 0.f : exp2f(m_w - mb);
    l_w *= f;
    a_w.x *= f; a_w.y *= f; a_w.z *= f; a_w.w *= f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float wgt = mm[j] == -CUDART_INF_F ? 0.f : exp2f(mm[j] - mb);
      l_w = fmaf(wgt, ll[j], l_w);
      a_w.x = fmaf(wgt, aa[j].x, a_w.x);
      a_w.y = fmaf(wgt, aa[j].y, a_w.y);
      a_w.z = fmaf(wgt, aa[j].z, a_w.z);
      a_w.w = fmaf(wgt, aa[j].w, a_w.w);
    }
    m_w = mb;
  }
  *reinterpret_cast<float4*>(&accs[warp][4 * lane]) = a_w;
  if (lane == 0) {
    msw[warp] = m_w;
    lsw[warp] = l_w;
  }
  __syncthreads();
  {
    float M = msw[0];
#pragma unroll
    for (int w = 1; w < kCombWarps; ++w) M = fmaxf(M, msw[w]);
    if (tid < kD) {
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < kCombWarps; ++w) {
        const float wgt = msw[w] == -CUDART_INF_F ? 0.f : exp2f(msw[w] - M);
        a = fmaf(wgt, accs[w][tid], a);
      }
      cmid[4 + tid] = a;
    }
    if (tid == 0) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kCombWarps; ++w) l = fmaf(msw[w] == -CUDART_INF_F ? 0.f : exp2f(msw[w] - M), lsw[w], l);
      cmid[0] = M;
      cmid[1] = l;
    }
  }
  // every slice's intermediate is visible to the cluster's CTA 0
  cluster_sync_all();
  if (slice == 0) {
    // ---- CTA 0 merges the cluster's intermediates (and the buffer's) ----
    float mk[S + 1], lk[S + 1], ak[S + 1];
#pragma unroll
    for (int k = 0; k < S; ++k) {
      mk[k] = dsmem_ld(dsmem_addr(&cmid[0], k));
      lk[k] = dsmem_ld(dsmem_addr(&cmid[1], k));
      ak[k] = dsmem_ld(dsmem_addr(&cmid[4 + dd], k));
    }
    // the other CTAs may leave once CTA 0 has read their shared memory
    cluster_sync_all();
    if (has_buf) {
      const float* bm = ws.comb_mid + (wrow * (kCombSlices + 1) + kCombSlices) * kPartialStride;
      mk[S] = __ldcg(bm);
      lk[S] = __ldcg(bm + 1);
      ak[S] = __ldcg(bm + 4 + dd);
    } else {
      mk[S] = -CUDART_INF_F;
      lk[S] = 0.f;
      ak[S] = 0.f;
    }
    float Mt = -CUDART_INF_F;
#pragma unroll
    for (int k = 0; k <= S; ++k) Mt = fmaxf(Mt, mk[k]);
    float Lt = 0.f, at = 0.f, ab = 0.f;
#pragma unroll
    for (int k = 0; k <= S; ++k) {
      const float w = mk[k] == -CUDART_INF_F ? 0.f : exp2f(mk[k] - Mt);
      Lt = fmaf(w, lk[k], Lt);
      if (k < S) at = fmaf(w, ak[k], at);  // rotated basis
      else ab = w * ak[k];                            // the buffer's rows, unrotated
    }
    if (tid < kD) a_s[tid] = at / Lt;
    __syncthreads();
    // inverse V rotation: two threads per output, half of the inputs each
    float o = 0.f;
#pragma unroll
    for (int r = 0; r < 64; ++r) {
      const float m = EARLY ? mvr[r] : __ldg(mv + (half * 64 + r) * kD + dd);
      o = fmaf(m, a_s[half * 64 + r], o);
    }
    if (half == 1) accs[0][dd] = o;
    __syncthreads();
    if (half == 0) out[row * kD + dd] = __float2half(o + accs[0][dd] + ab / Lt);
  } else {
    // keep this CTA's shared memory until CTA 0 has read it
    cluster_sync_all();
  }
}

// Warps per CTA of the split pass (several CTAs per SM: a CTA that finishes
// frees its slot for the next launch's CTAs, which overlap their set-up
// with this launch's tail).
constexpr int kSplitWarps = kDecWarps;

template <int VB>
cudaError_t launch_decode_vb(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                             const float* qrot, const int32_t* seq_lens, const BufferArgs& buf, int batch,
                             const SplitPlan& plan, cudaStream_t stream) {
  // the largest layout over K widths, so one attribute value serves every call
  static const cudaError_t attr =
      set_smem(decode_mma_kernel<VB, kSplitWarps>, decode_layout(4, VB, kSplitWarps).total);
  if (attr != cudaSuccess) return attr;
  const int head_blocks = (s.group + 7) / 8;
  // units fastest, then split index: the CTAs every unit uses come first
  dim3 grid(batch * s.n_kv_heads * head_blocks, (buf.k != nullptr ? 1 : 0) + plan.c_max, layer_count);
  return launch_dependent(decode_mma_kernel<VB, kSplitWarps>, grid, dim3(kSplitWarps * 32),
                          decode_layout(s.kbits, VB, kSplitWarps).total, stream, s, ws, cache, layer0, qrot, seq_lens,
                          buf, batch, plan, head_blocks);
}

template <int VB>
int ctas_per_sm_vb(const Shape& s) {
  static const cudaError_t attr =
      set_smem(decode_mma_kernel<VB, kSplitWarps>, decode_layout(4, VB, kSplitWarps).total);
  if (attr != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_mma_kernel<VB, kSplitWarps>, kSplitWarps * 32,
                                                    decode_layout(s.kbits, VB, kSplitWarps).total) != cudaSuccess)
    return 0;
  return n;
}

template <int VB, int CL>
cudaError_t fused_attr_once() {
  static const cudaError_t attr = set_smem(decode_fused_kernel<VB, CL>, fused_layout(4, VB, CL).total);
  return attr;
}

template <int VB, int CL>
cudaError_t launch_fused_vcl(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                             const __half* q, const int32_t* seq_lens, int batch, const SplitPlan& plan, __half* out,
                             cudaStream_t stream) {
  const cudaError_t attr = fused_attr_once<VB, CL>();
  if (attr != cudaSuccess) return attr;
  const int head_blocks = (s.group + 7) / 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch * s.n_kv_heads * head_blocks, plan.c_max, layer_count);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = fused_layout(s.kbits, VB, CL).total;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = 1;
  at[1].val.clusterDim.y = CL;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel<VB, CL>, s, ws, cache, layer0, q, seq_lens, batch, plan,
                            head_blocks, out);
}

template <int VB>
cudaError_t launch_fused_vb(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                            const __half* q, const int32_t* seq_lens, int batch, const SplitPlan& plan, __half* out,
                            cudaStream_t stream) {
  if (plan.cluster == 4)
    return launch_fused_vcl<VB, 4>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
  if (plan.cluster == 8)
    return launch_fused_vcl<VB, 8>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
  return cudaErrorInvalidValue;
}

template <int VB, int CL>
int fused_clusters_vcl(const Shape& s) {
  if (fused_attr_once<VB, CL>() != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, CL, 1);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = fused_layout(s.kbits, VB, CL).total;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = CL;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_fused_kernel<VB, CL>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

template <int VB>
int fused_clusters_vb(const Shape& s, int cl) {
  return cl == 4 ? fused_clusters_vcl<VB, 4>(s) : cl == 8 ? fused_clusters_vcl<VB, 8>(s) : 0;
}

}  // namespace

int decode_fused_clusters(const Shape& s, int cluster) {
  switch (s.vbits) {
    case 1: return fused_clusters_vb<1>(s, cluster);
    case 2: return fused_clusters_vb<2>(s, cluster);
    case 3: return fused_clusters_vb<3>(s, cluster);
    default: return fused_clusters_vb<4>(s, cluster);
  }
}

cudaError_t launch_decode_fused(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                                int layer_count, const __half* q, const int32_t* seq_lens, int batch,
                                const SplitPlan& plan, __half* out, cudaStream_t stream) {
  switch (s.vbits) {
    case 1: return launch_fused_vb<1>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
    case 2: return launch_fused_vb<2>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
    case 3: return launch_fused_vb<3>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
    default: return launch_fused_vb<4>(s, ws, cache, layer0, layer_count, q, seq_lens, batch, plan, out, stream);
  }
}

int decode_ctas_per_sm(const Shape& s) {
  switch (s.vbits) {
    case 1: return ctas_per_sm_vb<1>(s);
    case 2: return ctas_per_sm_vb<2>(s);
    case 3: return ctas_per_sm_vb<3>(s);
    default: return ctas_per_sm_vb<4>(s);
  }
}

cudaError_t launch_decode_split(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                                int layer_count, const float* qrot, const int32_t* seq_lens, const BufferArgs& buf,
                                int batch, const SplitPlan& plan, cudaStream_t stream) {
  switch (s.vbits) {
    case 1: return launch_decode_vb<1>(s, ws, cache, layer0, layer_count, qrot, seq_lens, buf, batch, plan, stream);
    case 2: return launch_decode_vb<2>(s, ws, cache, layer0, layer_count, qrot, seq_lens, buf, batch, plan, stream);
    case 3: return launch_decode_vb<3>(s, ws, cache, layer0, layer_count, qrot, seq_lens, buf, batch, plan, stream);
    default: return launch_decode_vb<4>(s, ws, cache, layer0, layer_count, qrot, seq_lens, buf, batch, plan, stream);
  }
}

cudaError_t launch_combine(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                           const int32_t* seq_lens, int batch, const SplitPlan& plan, const BufferArgs& buf,
                           __half* out, cudaStream_t stream) {
  const int rows = layer_count * batch * s.n_q_heads;
  // one CTA per row when no unit has more splits than its 8 warps load in
  // one round (4 each); else a cluster of kCombSlices slices per row
  const int S = plan.c_max <= 4 * (kCombThreads / 32) ? 1 : kCombSlices;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * S);
  cfg.blockDim = dim3(kCombThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;  // a row's slices
  at[1].val.clusterDim.x = S;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  const bool early = rows <= kEarlyRotationRows;
  if (S == 1)
    return early ? cudaLaunchKernelEx(&cfg, combine_kernel<true, 1>, s, ws, layer0, seq_lens, batch, plan, buf, out)
                 : cudaLaunchKernelEx(&cfg, combine_kernel<false, 1>, s, ws, layer0, seq_lens, batch, plan, buf, out);
  return early
             ? cudaLaunchKernelEx(&cfg, combine_kernel<true, kCombSlices>, s, ws, layer0, seq_lens, batch, plan, buf, out)
             : cudaLaunchKernelEx(&cfg, combine_kernel<false, kCombSlices>, s, ws, layer0, seq_lens, batch, plan, buf,
                                  out);
}

}  // namespace bgtq

// CUDA kernels of the Block-GTQ packed-cache path for B200 (sm_100a).
//
//   energy_kernel        label-free per-RoPE-block Q/K energy, exact 128-bit sums
//   encode_kernel        TQ-MSE: rotate (fp32), normalise (fp64), quantise, pack tiles
//   rotate_query_kernel  q~ per width group (rotated basis, 1/sqrt(d_g), 1/sqrt(D))
//   decode_mma_kernel    split-K flash decoding from the packed tiles (mma.sync)
//   combine_kernel       log-sum-exp merge of the splits + inverse V rotation
//   logit_mae_kernel     per-layer logit MAE of the packed keys (diagnostic)
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ;
// chatpaper summary / arXiv 2606.24033 abstract, blockgtq README) on top of
// TurboQuant-MSE (arXiv 2504.19874); split-K decoding after FlashAttention /
// FlashAttention-2 (arXiv 2205.14135, 2307.08691), both cited by the pages.
#include <algorithm>

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stddef.h>
#include <stdint.h>

#include "device_tables.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)

// Cache slot of tile t of (layer, sequence b, KV head h): contiguous, or
// through the block table of a paged cache.  -1 for a page id outside the
// pool (the caller raises kErrPage).
__device__ __forceinline__ int64_t tile_slot(const Shape& sh, const CacheDev& c, int layer, int b, int h, int64_t t) {
  if (c.n_pages == 0) return ((static_cast<int64_t>(layer) * sh.max_batch + b) * sh.n_kv_heads + h) * sh.ntiles + t;
  const int32_t page = c.block_table[static_cast<int64_t>(b) * sh.ntiles + t];
  if (page < 0 || page >= c.n_pages) return -1;
  return (static_cast<int64_t>(layer) * sh.n_kv_heads + h) * c.n_pages + page;
}

__device__ __forceinline__ uint64_t fp16_fixed(uint16_t bits, uint32_t* nonfinite) {
  // |x| * 2^24 for a binary16 x: subnormals are m * 2^-24, normals
  // (1024 + m) * 2^(e - 25).
  const uint32_t e = (bits >> 10) & 31u;
  const uint32_t m = bits & 1023u;
  if (e == 31u) {
    *nonfinite = 1u;
    return 0;
  }
  if (e == 0u) return m;
  return static_cast<uint64_t>(1024u + m) << (e - 1u);
}

// ---------------------------------------------------------------------------
// a1: energy.  Grid (L * Hkv, kEnergyChunks), 128 threads = one per dim.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) energy_kernel(const __half* __restrict__ q, int nq,
                                                     const __half* __restrict__ k, int nk, int Hq,
                                                     int Hkv, int G, int L, int pairing,
                                                     unsigned __int128* __restrict__ eq,
                                                     unsigned __int128* __restrict__ ek,
                                                     uint32_t* err) {
  const int layer = blockIdx.x / Hkv;
  const int h = blockIdx.x % Hkv;
  const int c = blockIdx.y;
  const int d = threadIdx.x;
  const int rq = (nq + kEnergyChunks - 1) / kEnergyChunks;
  const int rk = (nk + kEnergyChunks - 1) / kEnergyChunks;
  uint32_t bad = 0;
  unsigned __int128 sq = 0, sk = 0;
  const unsigned short* qb = reinterpret_cast<const unsigned short*>(q);
  const unsigned short* kb = reinterpret_cast<const unsigned short*>(k);
  const int rq_end = min(nq, (c + 1) * rq);
  for (int r = c * rq; r < rq_end; ++r) {
    const size_t row = (static_cast<size_t>(layer) * nq + r) * Hq + static_cast<size_t>(h) * G;
    for (int gh = 0; gh < G; ++gh) {
      const uint64_t x = fp16_fixed(qb[(row + gh) * kD + d], &bad);
      sq += static_cast<unsigned __int128>(x) * x;
    }
  }
  const int rk_end = min(nk, (c + 1) * rk);
  for (int r = c * rk; r < rk_end; ++r) {
    const size_t row = (static_cast<size_t>(layer) * nk + r) * Hkv + h;
    const uint64_t x = fp16_fixed(kb[row * kD + d], &bad);
    sk += static_cast<unsigned __int128>(x) * x;
  }
  __shared__ unsigned __int128 s_q[kD], s_k[kD];
  s_q[d] = sq;
  s_k[d] = sk;
  __syncthreads();
  if (d < kD / 2) {
    const int a = pairing == 0 ? d : 2 * d;
    const int b = pairing == 0 ? d + kD / 2 : 2 * d + 1;
    const size_t o = ((static_cast<size_t>(c) * L + layer) * Hkv + h) * (kD / 2) + d;
    eq[o] = s_q[a] + s_q[b];
    ek[o] = s_k[a] + s_k[b];
  }
  if (bad) atomicOr(err, kErrNonFinite);
}


// ---------------------------------------------------------------------------
// Tile format helpers.  A 64-position tile stores each lane's mma A-fragment
// selectors (8 nibble codes per 32-bit word) as bit-plane "quartets":
//   b = 1: P = s0&M1 | (s1&M1)<<1 | (s2&M1)<<2 | (s3&M1)<<3
//   b = 2: A = s0&M3 | (s1&M3)<<2,  B = s2&M3 | (s3&M3)<<2
//   b = 3: A, B and H = (s0&M4)>>2 | (s1&M4)>>1 | s2&M4 | (s3&M4)<<1
//   b = 4: s0..s3
// K selector (chunk j, M-tile mu, lane 4g+t) nibble n: token 16mu+g+8(n>=4),
// group coordinate 16j+4t+n%4.  V selector (dim tile m, token step kappa):
// coordinate 16m+g+8(n>=4), token 16kappa+(2t,2t+1,2t+8,2t+9)[n%4].
// ---------------------------------------------------------------------------
constexpr uint32_t M1 = 0x11111111u, M3 = 0x33333333u, M4 = 0x44444444u;

template <int B>
__device__ __forceinline__ void quartet_decode(const uint32_t* w, uint32_t* s) {
  if constexpr (B == 4) {
    s[0] = w[0]; s[1] = w[1]; s[2] = w[2]; s[3] = w[3];
  } else if constexpr (B == 3) {
    s[0] = (w[0] & M3) | ((w[2] << 2) & M4);
    s[1] = ((w[0] >> 2) & M3) | ((w[2] << 1) & M4);
    s[2] = (w[1] & M3) | (w[2] & M4);
    s[3] = ((w[1] >> 2) & M3) | ((w[2] >> 1) & M4);
  } else if constexpr (B == 2) {
    s[0] = w[0] & M3; s[1] = (w[0] >> 2) & M3; s[2] = w[1] & M3; s[3] = (w[1] >> 2) & M3;
  } else {
    s[0] = w[0] & M1; s[1] = (w[0] >> 1) & M1; s[2] = (w[0] >> 2) & M1; s[3] = (w[0] >> 3) & M1;
  }
}

template <int B>
__device__ __forceinline__ void quartet_encode(const uint32_t* s, uint32_t* w) {
  if constexpr (B == 4) {
    w[0] = s[0]; w[1] = s[1]; w[2] = s[2]; w[3] = s[3];
  } else if constexpr (B == 1) {
    w[0] = (s[0] & M1) | ((s[1] & M1) << 1) | ((s[2] & M1) << 2) | ((s[3] & M1) << 3);
  } else {
    w[0] = (s[0] & M3) | ((s[1] & M3) << 2);
    w[1] = (s[2] & M3) | ((s[3] & M3) << 2);
    if constexpr (B == 3) w[2] = ((s[0] & M4) >> 2) | ((s[1] & M4) >> 1) | (s[2] & M4) | ((s[3] & M4) << 1);
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Byte tables of the fp16 codebook: lo[i] / hi[i] hold the low / high bytes
// of entries 4i .. 4i+3.
struct ByteTab {
  uint32_t lo[4], hi[4];
};

// Four codes (selector nibbles 0..3) -> two fp16x2 registers: codes (0, 1)
// and codes (2, 3).  PRMT picks bytes 0..7 of its two table words by the
// nibble's low three bits; width-4 codes look up both halves of the table
// and pick by their top bit.
template <int B>
__device__ __forceinline__ void lookup4(const ByteTab& t, uint32_t sel, uint32_t& r01, uint32_t& r23) {
  uint32_t lo, hi;
  if constexpr (B <= 3) {
    lo = prmt(t.lo[0], t.lo[1], sel);
    hi = prmt(t.hi[0], t.hi[1], sel);
  } else {
    const uint32_t s7 = sel & 0x7777u;
    const uint32_t pick = 0x3210u | ((sel >> 1) & 0x4444u);
    lo = prmt(prmt(t.lo[0], t.lo[1], s7), prmt(t.lo[2], t.lo[3], s7), pick);
    hi = prmt(prmt(t.hi[0], t.hi[1], s7), prmt(t.hi[2], t.hi[3], s7), pick);
  }
  r01 = prmt(lo, hi, 0x5140u);
  r23 = prmt(lo, hi, 0x7362u);
}

// D += A * B for one m16n8k16 tile, fp16 operands, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// A-fragment from one selector word (rows g and g+8) times a B-fragment.
template <int B>
__device__ __forceinline__ void mma_selector(float* c, const ByteTab& t, uint32_t s, uint32_t b0, uint32_t b1) {
  uint32_t r0, r1, r2, r3;
  lookup4<B>(t, s, r0, r2);
  lookup4<B>(t, s >> 16, r1, r3);
  mma16816(c, r0, r1, r2, r3, b0, b1);
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(x));
  return d;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Group geometry of a K layout (record order, widest group first).
struct GroupGeo {
  int width, d, nfull, r, word, chunk, start;
};

__device__ __forceinline__ GroupGeo group_geo(const LayoutDev& lay, int g) {
  GroupGeo q;
  q.width = lay.width[g];
  q.d = lay.size[g];
  q.nfull = q.d >> 4;
  q.r = q.d & 15;
  q.word = lay.tile_word[g];
  q.chunk = lay.chunk_base[g];
  q.start = lay.start[g];
  return q;
}

// ---- tile unpack / pack over a CTA (codes[64][128] in shared memory) ----

// The lane's selector for chunk j, M-tile mu: token and group coordinate of nibble n.
__device__ __forceinline__ int k_token(int mu, int lane, int n) { return 16 * mu + (lane >> 2) + 8 * (n >= 4); }
__device__ __forceinline__ int k_coord(int j, int lane, int n) { return 16 * j + 4 * (lane & 3) + (n & 3); }

// Row pitch (bytes) of a tile's code matrix [64 tokens][128 coordinates] in
// shared memory: 132 puts the rows of consecutive tokens in different banks.
constexpr int kCodePitch = kD + 4;

template <int B>
__device__ void unpack_k_group(const uint32_t* tw, const GroupGeo& q, uint8_t (*codes)[kCodePitch], int tid,
                               int nthreads) {
  const uint32_t* gw = tw + q.word;
  for (int u = tid; u < q.nfull * 32; u += nthreads) {
    const int j = u >> 5, lane = u & 31;
    uint32_t w[B], s[4];
    for (int k = 0; k < B; ++k) w[k] = gw[j * 32 * B + 32 * k + lane];
    quartet_decode<B>(w, s);
    for (int mu = 0; mu < 4; ++mu)
      for (int n = 0; n < 8; ++n)
        codes[k_token(mu, lane, n)][q.start + k_coord(j, lane, n)] = (s[mu] >> (4 * n)) & 15u;
  }
  if (q.r) {
    const uint32_t* pc = gw + q.nfull * 32 * B;
    const int nf = q.r >> 2;
    for (int u = tid; u < 8 * nf; u += nthreads) {
      const int g = u / nf, t = u % nf, lane = 4 * g + t;
      uint32_t w[B], s[4];
      for (int k = 0; k < B; ++k) w[k] = pc[8 * nf * k + u];
      quartet_decode<B>(w, s);
      for (int mu = 0; mu < 4; ++mu)
        for (int n = 0; n < 8; ++n)
          codes[k_token(mu, lane, n)][q.start + k_coord(q.nfull, lane, n)] = (s[mu] >> (4 * n)) & 15u;
    }
    if (q.r & 3) {
      for (int v = tid; v < 4; v += nthreads) {
        uint32_t w[B], s[4];
        for (int k = 0; k < B; ++k) w[k] = pc[8 * nf * B + 4 * k + v];
        quartet_decode<B>(w, s);
        for (int mu = 0; mu < 4; ++mu)
          for (int nv = 0; nv < 8; ++nv) {
            const int lane = 4 * (2 * v + (nv >> 2)) + nf;
            const int n = (nv & 1) + 4 * ((nv >> 1) & 1);  // half nibbles 0, 1, 4, 5
            codes[k_token(mu, lane, n)][q.start + k_coord(q.nfull, lane, n)] = (s[mu] >> (4 * nv)) & 15u;
          }
      }
    }
  }
}

template <int B>
__device__ void pack_k_group(uint32_t* tw, const GroupGeo& q, const uint8_t (*codes)[kCodePitch], int tid,
                             int nthreads) {
  uint32_t* gw = tw + q.word;
  for (int u = tid; u < q.nfull * 32; u += nthreads) {
    const int j = u >> 5, lane = u & 31;
    uint32_t s[4], w[B];
    for (int mu = 0; mu < 4; ++mu) {
      uint32_t x = 0;
      for (int n = 0; n < 8; ++n) x |= uint32_t(codes[k_token(mu, lane, n)][q.start + k_coord(j, lane, n)]) << (4 * n);
      s[mu] = x;
    }
    quartet_encode<B>(s, w);
    for (int k = 0; k < B; ++k) gw[j * 32 * B + 32 * k + lane] = w[k];
  }
  if (q.r) {
    uint32_t* pc = gw + q.nfull * 32 * B;
    const int nf = q.r >> 2;
    for (int u = tid; u < 8 * nf; u += nthreads) {
      const int g = u / nf, t = u % nf, lane = 4 * g + t;
      uint32_t s[4], w[B];
      for (int mu = 0; mu < 4; ++mu) {
        uint32_t x = 0;
        for (int n = 0; n < 8; ++n)
          x |= uint32_t(codes[k_token(mu, lane, n)][q.start + k_coord(q.nfull, lane, n)]) << (4 * n);
        s[mu] = x;
      }
      quartet_encode<B>(s, w);
      for (int k = 0; k < B; ++k) pc[8 * nf * k + u] = w[k];
    }
    if (q.r & 3) {
      for (int v = tid; v < 4; v += nthreads) {
        uint32_t s[4], w[B];
        for (int mu = 0; mu < 4; ++mu) {
          uint32_t x = 0;
          for (int nv = 0; nv < 8; ++nv) {
            const int lane = 4 * (2 * v + (nv >> 2)) + nf;
            const int n = (nv & 1) + 4 * ((nv >> 1) & 1);
            x |= uint32_t(codes[k_token(mu, lane, n)][q.start + k_coord(q.nfull, lane, n)]) << (4 * nv);
          }
          s[mu] = x;
        }
        quartet_encode<B>(s, w);
        for (int k = 0; k < B; ++k) pc[8 * nf * B + 4 * k + v] = w[k];
      }
    }
  }
}

__device__ __forceinline__ int v_token(int kappa, int lane, int n) {
  const int t = lane & 3;
  const int member = n & 3;
  return 16 * kappa + 2 * t + (member & 1) + 8 * (member >> 1);
}
__device__ __forceinline__ int v_coord(int m, int lane, int n) { return 16 * m + (lane >> 2) + 8 * (n >= 4); }

template <int B>
__device__ void unpack_v_tile(const uint32_t* tw, uint8_t (*codes)[kCodePitch], int tid, int nthreads) {
  for (int u = tid; u < 8 * 32; u += nthreads) {
    const int m = u >> 5, lane = u & 31;
    uint32_t w[B], s[4];
    for (int k = 0; k < B; ++k) w[k] = tw[m * 32 * B + 32 * k + lane];
    quartet_decode<B>(w, s);
    for (int kappa = 0; kappa < 4; ++kappa)
      for (int n = 0; n < 8; ++n) codes[v_token(kappa, lane, n)][v_coord(m, lane, n)] = (s[kappa] >> (4 * n)) & 15u;
  }
}

template <int B>
__device__ void pack_v_tile(uint32_t* tw, const uint8_t (*codes)[kCodePitch], int tid, int nthreads) {
  for (int u = tid; u < 8 * 32; u += nthreads) {
    const int m = u >> 5, lane = u & 31;
    uint32_t s[4], w[B];
    for (int kappa = 0; kappa < 4; ++kappa) {
      uint32_t x = 0;
      for (int n = 0; n < 8; ++n) x |= uint32_t(codes[v_token(kappa, lane, n)][v_coord(m, lane, n)]) << (4 * n);
      s[kappa] = x;
    }
    quartet_encode<B>(s, w);
    for (int k = 0; k < B; ++k) tw[m * 32 * B + 32 * k + lane] = w[k];
  }
}

#define BGTQ_WIDTH_SWITCH(b, F, ...) \
  switch (b) {                       \
    case 1: F<1>(__VA_ARGS__); break; \
    case 2: F<2>(__VA_ARGS__); break; \
    case 3: F<3>(__VA_ARGS__); break; \
    default: F<4>(__VA_ARGS__); break; \
  }

// ---------------------------------------------------------------------------
// a3: encode.  Grid (layer_count * batch * Hkv, per_unit, 2 kinds), 256
// threads.  A CTA loads one (layer, KV head, kind)'s rotation and tables once
// and then takes every per_unit-th 64-position tile that the call writes for
// one sequence: it unpacks the tile's codes when the call writes only part of
// it, encodes its new rows (y = R x in fp32, norms in fp64, u = sqrt(d) y /
// n, code = #{thresholds <= u}) into the codes, and packs the tile again.
// ---------------------------------------------------------------------------
constexpr int kEncThreads = 256;
// Column of element (coordinate j, row r) in xt[j][]: float4 groups of 4 rows,
// XOR-swizzled by j so that the transposed writes spread over the banks.
__device__ __forceinline__ int xt_col(int j, int r) { return (((r >> 2) ^ ((j >> 3) & 15)) << 2) | (r & 3); }

// The Lloyd-Max code of u for width w >= 1: the number of the 2^w - 1
// ascending thresholds t[] that are <= u (ties go up), by binary search.
__device__ __forceinline__ int lloyd_code(const float* t, int w, float u) {
  int c = 0;
  for (int s = 1 << (w - 1); s > 0; s >>= 1)
    if (t[c + s - 1] <= u) c += s;
  return c;
}

struct EncodeSmem {
  float xt[kD][kTile];           // new rows, transposed, record order (zero elsewhere), columns xt_col
  float mt[kD][kD];              // mt[j][c(i)] = R[i][j] (record order), c(8 o + 4 q + e) = 64 q + 4 o + e
  float fac[kTile][kNumGroupsMax];
  __half nrm[kTile][kNumGroupsMax];
  uint8_t codes[kTile][kCodePitch];
  uint32_t words[1024];
  float thr[5][16];
  int32_t inv[kD];
  int32_t gof[kD];               // group of each record position (-1: width 0)
  LayoutDev lay;
};

__global__ void __launch_bounds__(kEncThreads) encode_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                             const __half* __restrict__ kx,
                                                             const __half* __restrict__ vx,
                                                             const int32_t* __restrict__ start_v,
                                                             const int32_t* __restrict__ count_v, int batch, int n) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  EncodeSmem& S = *reinterpret_cast<EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int kind = blockIdx.z;
  const int h = blockIdx.x % sh.n_kv_heads;
  const int b = (blockIdx.x / sh.n_kv_heads) % batch;
  const int li = blockIdx.x / (sh.n_kv_heads * batch);
  const int layer = layer0 + li;
  const int start = start_v[b];
  const int count = count_v[b];
  if (start < 0 || count < 0 || count > n) {
    if (tid == 0 && blockIdx.y == 0 && kind == 0) atomicOr(ws.err, kErrArg);
    return;
  }
  if (count == 0) return;
  int64_t p_end = static_cast<int64_t>(start) + count;  // rows land at [start, p_end)
  if (p_end > sh.capacity) {
    if (tid == 0 && blockIdx.y == 0) atomicOr(ws.err, kErrCapacity);
    p_end = sh.capacity;
  }
  const int64_t t_first = start / kTile;
  if (t_first + blockIdx.y >= (p_end + kTile - 1) / kTile) return;  // no tile for this CTA
  const int bits_avg = kind == 0 ? sh.kbits : sh.vbits;
  const int nwords = 256 * bits_avg;
  const int lh = layer * sh.n_kv_heads + h;
  if (kind == 0) {
    if (tid < static_cast<int>(sizeof(LayoutDev) / 4))
      reinterpret_cast<int32_t*>(&S.lay)[tid] = reinterpret_cast<const int32_t*>(ws.layouts + lh)[tid];
  } else if (tid == 0) {
    S.lay.n_groups = 1;
    S.lay.n_positions = kD;
    for (int g = 0; g < kNumGroupsMax; ++g) {
      S.lay.width[g] = g == 0 ? sh.vbits : 0;
      S.lay.size[g] = g == 0 ? kD : 0;
      S.lay.start[g] = g == 0 ? 0 : kD;
      S.lay.bitoff[g] = 0;
      S.lay.tile_word[g] = 0;
      S.lay.chunk_base[g] = 0;
    }
  }
  for (int i = tid; i < 5 * 16; i += kEncThreads) (&S.thr[0][0])[i] = (&ws.codebook->threshold[0][0])[i];
  const float* mglob = (kind == 0 ? ws.mkt : ws.mvt) + static_cast<size_t>(lh) * kD * kD;
  // columns swizzled so that the 16 output groups of a warp read the first
  // and the second half of their 8 columns as two contiguous 256-byte spans
  for (int i = tid; i < kD * kD / 4; i += kEncThreads) {
    const int j = i / (kD / 4), c4 = i % (kD / 4);  // float4 c4 of row j: columns 4 c4 .. 4 c4 + 3
    const int o = c4 >> 1, q = c4 & 1;
    reinterpret_cast<float4*>(&S.mt[j][0])[q * 16 + o] = reinterpret_cast<const float4*>(mglob)[i];
  }
  __syncthreads();
  const int ng = S.lay.n_groups;
  const int npos = S.lay.n_positions;
  if (tid < kD) {
    S.inv[kind == 0 ? S.lay.perm[tid] : tid] = tid;
    int g = -1;
    if (tid < npos) {
      g = 0;
      for (int t = 1; t < ng; ++t)
        if (tid >= S.lay.start[t]) g = t;
    }
    S.gof[tid] = g;
  }
  __syncthreads();
  // ---- this CTA's tiles: t_first + blockIdx.y, then every gridDim.y-th ----
  for (int64_t tile = t_first + blockIdx.y; tile * kTile < p_end; tile += gridDim.y) {
    const int64_t p0 = max(tile * kTile, static_cast<int64_t>(start));
    const int64_t p1 = min(tile * kTile + kTile, p_end);
    const int tr0 = static_cast<int>(p0 - tile * kTile), tr1 = static_cast<int>(p1 - tile * kTile);
    const bool whole = (tr0 == 0 && tr1 == kTile);
    if (p0 >= p1) continue;  // the first rows are past the capacity
    const int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
    if (slot < 0) {  // uniform over the CTA
      if (tid == 0) atomicOr(ws.err, kErrPage);
      continue;
    }
    uint32_t* gtile = (kind == 0 ? cache.ktile : cache.vtile) + slot * nwords;
    // existing codes of a partly written tile
    if (!whole) {
      if (kind == 0) {
        for (int g = 0; g < ng; ++g) {
          const GroupGeo q = group_geo(S.lay, g);
          BGTQ_WIDTH_SWITCH(q.width, unpack_k_group, gtile, q, S.codes, tid, kEncThreads)
        }
      } else {
        BGTQ_WIDTH_SWITCH(sh.vbits, unpack_v_tile, gtile, S.codes, tid, kEncThreads)
      }
    }
    __syncthreads();
    // new rows -> xt (record order)
    const size_t row_stride = static_cast<size_t>(sh.n_kv_heads) * kD;
    const __half* x = kind == 0 ? kx : vx;
    const __half* xbase = x + ((static_cast<size_t>(li) * batch + b) * n + (p0 - start)) * row_stride +
                          static_cast<size_t>(h) * kD;
    for (int e = tid; e < kTile * (kD / 8); e += kEncThreads) {
      const int r = e >> 4, c8 = e & 15;  // row, 8 coordinates
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (r >= tr0 && r < tr1)
        raw = *reinterpret_cast<const uint4*>(xbase + static_cast<size_t>(r - tr0) * row_stride + 8 * c8);
      const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
  #pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(h2[k]);
        const int j0 = S.inv[8 * c8 + 2 * k], j1 = S.inv[8 * c8 + 2 * k + 1];
        S.xt[j0][xt_col(j0, r)] = f.x;
        S.xt[j1][xt_col(j1, r)] = f.y;
      }
    }
    __syncthreads();
    // norms: fp64 sum of squares of the exact fp16 inputs
    {
      const int r = tid >> 2, g = tid & 3;
      float f = 0.f;
      __half nh = __float2half(0.f);
      if (g < ng && r >= tr0 && r < tr1) {
        const int j0 = S.lay.start[g], j1 = j0 + S.lay.size[g];
        double s2 = 0.0;
        for (int j = j0; j < j1; ++j) {
          const double v = S.xt[j][xt_col(j, r)];
          s2 += v * v;
        }
        const double nr = sqrt(s2);
        nh = __double2half(nr);
        f = nr > 0.0 ? static_cast<float>(sqrt(static_cast<double>(S.lay.size[g])) / nr) : 0.f;
      }
      S.fac[r][g] = f;
      S.nrm[r][g] = nh;
    }
    __syncthreads();
    // y = R x per new row (fp32, coordinate order), then the codes
    {
      // register tile: 4 rows x 8 outputs per thread over all 64 rows
      const int rg = tid >> 4, og = tid & 15;
      const int i0 = og * 8;
      if (i0 < npos && rg * 4 < tr1 && rg * 4 + 4 > tr0) {
        int gi[8];
  #pragma unroll
        for (int q = 0; q < 8; ++q) gi[q] = S.gof[i0 + q];
        int ghi = gi[0];
  #pragma unroll
        for (int q = 1; q < 8; ++q)
          if (gi[q] > ghi) ghi = gi[q];
        const int jlo = S.lay.start[gi[0]];
        const int jhi = S.lay.start[ghi] + S.lay.size[ghi];
        float acc[4][8];
  #pragma unroll
        for (int a = 0; a < 4; ++a)
  #pragma unroll
          for (int q = 0; q < 8; ++q) acc[a][q] = 0.f;
  #pragma unroll 4
        for (int j = jlo; j < jhi; ++j) {
          const float4 xv = *reinterpret_cast<const float4*>(&S.xt[j][4 * (rg ^ ((j >> 3) & 15))]);
          const float4 m0 = *reinterpret_cast<const float4*>(&S.mt[j][4 * og]);
          const float4 m1 = *reinterpret_cast<const float4*>(&S.mt[j][64 + 4 * og]);
          const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
          const float ms[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
  #pragma unroll
          for (int a = 0; a < 4; ++a)
  #pragma unroll
            for (int q = 0; q < 8; ++q) acc[a][q] = fmaf(xs[a], ms[q], acc[a][q]);
        }
  #pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int r = rg * 4 + a;
          if (r < tr0 || r >= tr1) continue;
  #pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int g = gi[q];
            if (g < 0) continue;
            const int w = S.lay.width[g];
            const float u = acc[a][q] * S.fac[r][g];
            S.codes[r][i0 + q] = static_cast<uint8_t>(lloyd_code(S.thr[w], w, u));
          }
        }
      }
    }
    __syncthreads();
    // repack the tile and write it back
    if (kind == 0) {
      for (int g = 0; g < ng; ++g) {
        const GroupGeo q = group_geo(S.lay, g);
        BGTQ_WIDTH_SWITCH(q.width, pack_k_group, S.words, q, S.codes, tid, kEncThreads)
      }
    } else {
      BGTQ_WIDTH_SWITCH(sh.vbits, pack_v_tile, S.words, S.codes, tid, kEncThreads)
    }
    __syncthreads();
    for (int i = tid; i < nwords / 4; i += kEncThreads)
      reinterpret_cast<uint4*>(gtile)[i] = reinterpret_cast<const uint4*>(S.words)[i];
    if (tid >= tr0 && tid < tr1) {
      const size_t pos = static_cast<size_t>(slot) * kTile + tid;
      if (kind == 0) {
        __half2* dst = reinterpret_cast<__half2*>(cache.knorm + pos * 4);
        dst[0] = __halves2half2(S.nrm[tid][0], S.nrm[tid][1]);
        dst[1] = __halves2half2(S.nrm[tid][2], S.nrm[tid][3]);
      } else {
        cache.vnorm[pos] = S.nrm[tid][0];
      }
    }

    __syncthreads();  // the buffers are reused by the next tile
  }
}

// ---------------------------------------------------------------------------
// a3 for a few rows (decode-time appends): grid (layer_count * batch * Hkv,
// n, 2 kinds), 128 threads.  A CTA encodes one new row of one (layer,
// sequence, KV head) and kind with the same arithmetic as encode_kernel
// (norms summed in fp64 in coordinate order, y = sum_j R[i][j] x_j in fp32
// in coordinate order from the group's first coordinate, u = y * sqrt(d) /
// ||x||, code = #{thresholds <= u}) and rewrites only that row's code bits
// in the packed tile, with global atomics: bits of other positions are never
// touched, so rows appended by different CTAs to the same tile do not race.
// ---------------------------------------------------------------------------
constexpr int kAppThreads = 128;

// Plane word (0..b-1) and bit of code bit q of selector sel, nibble n, in a
// quartet of width b (see the quartet formulas above).
__device__ __forceinline__ void quartet_bit(int b, int sel, int n, int q, int& k, int& bit) {
  if (b == 4) {
    k = sel;
    bit = 4 * n + q;
  } else if (b == 1) {
    k = 0;
    bit = 4 * n + sel;
  } else if (q < 2) {
    k = sel >> 1;
    bit = 4 * n + 2 * (sel & 1) + q;
  } else {
    k = 2;
    bit = 4 * n + sel;
  }
}

// Word (relative to the tile) of plane k for a K code, and the selector
// and nibble it sits in: token p (0..63), coordinate c of group g.
__device__ __forceinline__ int k_code_word(const LayoutDev& lay, int g, int c, int p, int k, int& sel, int& n) {
  const int b = lay.width[g], d = lay.size[g];
  const int nfull = d >> 4, r = d & 15, nf = r >> 2;
  const int j = c >> 4, cc = c & 15, t = cc >> 2, m4 = cc & 3;
  const int pr = p & 15, gg = pr & 7;
  sel = p >> 4;
  n = m4 + 4 * (pr >> 3);
  const int base = lay.tile_word[g];
  if (j < nfull) return base + j * 32 * b + 32 * k + 4 * gg + t;
  const int pc = base + nfull * 32 * b;
  if (t < nf) return pc + 8 * nf * k + gg * nf + t;
  // half quad of the partial chunk: virtual lane gg / 2, upper half for odd gg
  n = (n & 1) + 2 * (n >> 2) + 4 * (gg & 1);
  return pc + 8 * nf * b + 4 * k + (gg >> 1);
}

// Same for a V code: token p, dimension i.
__device__ __forceinline__ int v_code_word(int vb, int i, int p, int k, int& sel, int& n) {
  const int m = i >> 4, cm = i & 15, gg = cm & 7;
  const int pt = p & 15, t = (pt & 7) >> 1, member = (pt & 1) + 2 * (pt >> 3);
  sel = p >> 4;
  n = member + 4 * (cm >> 3);
  return m * 32 * vb + 32 * k + 4 * gg + t;
}

// One appended row of one (layer, sequence, KV head) and kind, by a CTA of
// NT >= 128 threads: bx = (layer, sequence, KV head) index, row < n, kind 0
// = K, 1 = V; mts = 64 KB of shared memory for the rotation.
template <int NT>
__device__ __forceinline__ void append_body(const Shape& sh, const Workspace& ws, const CacheDev& cache, int layer0,
                                            const __half* __restrict__ kx, const __half* __restrict__ vx,
                                            const int32_t* __restrict__ start_v, const int32_t* __restrict__ count_v,
                                            int batch, int n, int bx, int row, int kind, float* mts) {
  const int tid = threadIdx.x;
  const int h = bx % sh.n_kv_heads;
  const int b = (bx / sh.n_kv_heads) % batch;
  const int li = bx / (sh.n_kv_heads * batch);
  const int layer = layer0 + li;
  const int lh = layer * sh.n_kv_heads + h;
  // the next kernel of the stream may start its own table-only set-up now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the kind's rotation (transposed, [in][out]) in shared memory, all loads
  // in flight; a library table, read before the inputs are ready
  {
    const uint4* src = reinterpret_cast<const uint4*>((kind == 0 ? ws.mkt : ws.mvt) + static_cast<size_t>(lh) * kD * kD);
#pragma unroll 8
    for (int u = tid; u < kD * kD / 4; u += NT) reinterpret_cast<uint4*>(mts)[u] = __ldg(src + u);
  }
  // the layout and the thresholds: library tables too
  __shared__ LayoutDev lay;
  __shared__ float thr[5 * 16];
  __shared__ float xs[kD];
  __shared__ float fac[kNumGroupsMax];
  __shared__ __half nrm[kNumGroupsMax];
  for (int u = tid; u < 5 * 16; u += NT) thr[u] = (&ws.codebook->threshold[0][0])[u];
  if (kind == 0) {
    if (tid < static_cast<int>(sizeof(LayoutDev) / 4))
      reinterpret_cast<int32_t*>(&lay)[tid] = reinterpret_cast<const int32_t*>(ws.layouts + lh)[tid];
    for (int u = tid + NT; u < static_cast<int>(sizeof(LayoutDev) / 4); u += NT)
      reinterpret_cast<int32_t*>(&lay)[u] = reinterpret_cast<const int32_t*>(ws.layouts + lh)[u];
  } else if (tid == 0) {
    lay.n_groups = 1;
    lay.n_positions = kD;
    for (int g = 0; g < kNumGroupsMax; ++g) {
      lay.width[g] = g == 0 ? sh.vbits : 0;
      lay.size[g] = g == 0 ? kD : 0;
      lay.start[g] = g == 0 ? 0 : kD;
      lay.tile_word[g] = 0;
    }
  }
  __syncthreads();
  // Launched as a programmatic dependent of the previous kernel of the
  // stream: the call's inputs and the cache are read after it has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this row's values (row < n: inside the input whatever count is) and the
  // sequence's start and count, all in flight together; record order:
  // position i holds dim perm[i] (K), V keeps the dims
  const __half* x = (kind == 0 ? kx : vx) +
                    ((static_cast<size_t>(li) * batch + b) * n + row) * sh.n_kv_heads * kD + static_cast<size_t>(h) * kD;
  float xv = 0.f;
  if (kind == 0) {
    if (tid < lay.n_positions) xv = __half2float(x[lay.perm[tid]]);
  } else if (tid < kD) {
    xv = __half2float(x[tid]);
  }
  const int start = start_v[b];
  const int count = count_v[b];
  if (start < 0 || count < 0 || count > n) {
    if (tid == 0 && row == 0 && kind == 0) atomicOr(ws.err, kErrArg);
    return;
  }
  if (row >= count) return;
  const int64_t pos = static_cast<int64_t>(start) + row;
  if (pos >= sh.capacity) {
    if (tid == 0) atomicOr(ws.err, kErrCapacity);
    return;
  }
  if (tid < kD) xs[tid] = xv;
  __syncthreads();
  const int ng = lay.n_groups;
  if (tid < ng) {
    const int j0 = lay.start[tid], j1 = j0 + lay.size[tid];
    double s2 = 0.0;
    for (int j = j0; j < j1; ++j) {
      const double v = xs[j];
      s2 += v * v;
    }
    const double nr = sqrt(s2);
    nrm[tid] = __double2half(nr);
    fac[tid] = nr > 0.0 ? static_cast<float>(sqrt(static_cast<double>(lay.size[tid])) / nr) : 0.f;
  }
  __syncthreads();
  const int i = tid;
  const int tile = static_cast<int>(pos / kTile), p = static_cast<int>(pos % kTile);
  const int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
  if (slot < 0) {  // uniform over the CTA; no barrier follows
    if (tid == 0) atomicOr(ws.err, kErrPage);
    return;
  }
  if (i < lay.n_positions) {
    int g = 0;
    for (int t = 1; t < ng; ++t)
      if (i >= lay.start[t]) g = t;
    const int j0 = lay.start[g], j1 = j0 + lay.size[g];
    float y = 0.f;
    for (int j = j0; j < j1; ++j) y = fmaf(xs[j], mts[j * kD + i], y);
    const int w = lay.width[g];
    const float u = y * fac[g];
    const int code = lloyd_code(thr + w * 16, w, u);
    // rewrite this code's bits, one atomic pair per touched word
    const int nwords = 256 * (kind == 0 ? sh.kbits : sh.vbits);
    uint32_t* gtile = (kind == 0 ? cache.ktile : cache.vtile) + slot * nwords;
    int cur = -1;
    uint32_t mask = 0, val = 0;
    for (int q = 0; q < w; ++q) {
      int k, bit, sel, nib;
      if (kind == 0) k_code_word(lay, g, i - lay.start[g], p, 0, sel, nib);
      else v_code_word(w, i, p, 0, sel, nib);
      quartet_bit(w, sel, nib, q, k, bit);
      const int wk = kind == 0 ? k_code_word(lay, g, i - lay.start[g], p, k, sel, nib) : v_code_word(w, i, p, k, sel, nib);
      if (wk != cur) {
        if (cur >= 0) {
          atomicAnd(gtile + cur, ~mask);
          atomicOr(gtile + cur, val);
        }
        cur = wk;
        mask = 0;
        val = 0;
      }
      mask |= 1u << bit;
      val |= static_cast<uint32_t>((code >> q) & 1) << bit;
    }
    if (cur >= 0) {
      atomicAnd(gtile + cur, ~mask);
      atomicOr(gtile + cur, val);
    }
  }
  if (tid == 0) {
    const size_t tp = static_cast<size_t>(slot) * kTile + p;
    if (kind == 0) {
      __half2* dst = reinterpret_cast<__half2*>(cache.knorm + tp * 4);
      const __half z = __float2half(0.f);
      dst[0] = __halves2half2(nrm[0], ng > 1 ? nrm[1] : z);
      dst[1] = __halves2half2(ng > 2 ? nrm[2] : z, ng > 3 ? nrm[3] : z);
    } else {
      cache.vnorm[tp] = nrm[0];
    }
  }
}

__global__ void __launch_bounds__(kAppThreads) append_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                             const __half* __restrict__ kx,
                                                             const __half* __restrict__ vx,
                                                             const int32_t* __restrict__ start_v,
                                                             const int32_t* __restrict__ count_v, int batch, int n) {
  extern __shared__ __align__(16) float mts[];  // [kD][kD]
  append_body<kAppThreads>(sh, ws, cache, layer0, kx, vx, start_v, count_v, batch, n, blockIdx.x, blockIdx.y,
                           blockIdx.z, mts);
}

// ---------------------------------------------------------------------------
// a4: rotate the query.  Grid (layer_count * batch * Hq), 128 threads.
// ---------------------------------------------------------------------------
constexpr int kRotThreads = 256;

__device__ __forceinline__ uint4* frag_block(const Shape& sh, const Workspace& ws, int li, int b, int kvh, int hb) {
  const int hbs = (sh.group + 7) >> 3;
  return ws.qfrag + ((((static_cast<size_t>(li) * sh.max_batch + b) * sh.n_kv_heads + kvh) * hbs) + hb) * kFragEntries;
}

// Writes the B-fragment entries of query head hg (index within its KV
// group) from its q~ in record order (qs, shared memory): for chunk c of
// group g and quad t, coordinates 16 j + 4 t + m (j = c - first chunk of g)
// times log2(e), zero past the group's size, split into fp16 hi + lo.  The
// last head of a block also zeroes the unused head slots of the block.
__device__ void write_frags(const LayoutDev& lay, const float* qs, int hg, int G, uint4* fb, int tid, int nthreads) {
  const int hh = hg & 7;
  const int nh = min(8, G - (hg & ~7));
  const int ng = lay.n_groups;
  const int nchunk = lay.chunk_base[ng - 1] + ((lay.size[ng - 1] + 15) >> 4);
  for (int u = tid; u < nchunk * 4; u += nthreads) {
    const int c = u >> 2, t = u & 3;
    int g = 0;
    while (g + 1 < ng && c >= lay.chunk_base[g + 1]) ++g;
    const int j = c - lay.chunk_base[g];
    const int d = lay.size[g], st = lay.start[g];
    float v[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int coord = 16 * j + 4 * t + m;
      v[m] = coord < d ? qs[st + coord] * kLog2e : 0.f;
    }
    const __half2 a = __floats2half2_rn(v[0], v[1]);
    const __half2 c2 = __floats2half2_rn(v[2], v[3]);
    const float2 af = __half22float2(a), cf = __half22float2(c2);
    const __half2 al = __floats2half2_rn(v[0] - af.x, v[1] - af.y);
    const __half2 cl = __floats2half2_rn(v[2] - cf.x, v[3] - cf.y);
    fb[c * 32 + 4 * hh + t] = make_uint4(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&c2),
                                         *reinterpret_cast<const uint32_t*>(&al), *reinterpret_cast<const uint32_t*>(&cl));
  }
  if (hh == nh - 1)
    for (int u = tid; u < nchunk * 4 * (8 - nh); u += nthreads) {
      const int c = u % nchunk, rest = u / nchunk;
      fb[c * 32 + 4 * (nh + (rest >> 2)) + (rest & 3)] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// One query row (layer, sequence, query head) = bx, by a CTA of kRotThreads.
__device__ __forceinline__ void rotate_body(const Shape& sh, const Workspace& ws, int layer0,
                                            const __half* __restrict__ q, int batch, float* __restrict__ qrot,
                                            int bx) {
  // the decode kernel that follows may start its own set-up now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int hq = bx % sh.n_q_heads;
  const int b = (bx / sh.n_q_heads) % batch;
  const int li = bx / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const LayoutDev& lay = ws.layouts[layer * sh.n_kv_heads + kvh];
  const int tid = threadIdx.x, i = tid & (kD - 1), half = tid >> 7;
  // this thread's half column of the (block-diagonal) rotation, all loads in flight at once
  const float* mt = ws.mkt + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
  float m[64];
#pragma unroll
  for (int u = 0; u < 64; ++u) m[u] = __ldg(mt + (half * 64 + u) * kD + i);
  __shared__ float qp[kD];
  __shared__ float part[kD];
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  // Launched as a programmatic dependent of the previous kernel of the
  // stream: the query is read after it has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid < kD) qp[tid] = __half2float(q[row * kD + lay.perm[tid]]);
  __syncthreads();
  float sacc = 0.f;
#pragma unroll
  for (int u = 0; u < 64; ++u) sacc = fmaf(m[u], qp[half * 64 + u], sacc);
  if (half == 1) part[i] = sacc;
  __syncthreads();
  if (half == 0) {
    float out = 0.f;
    if (i < lay.n_positions) {
      int g = 0;
      for (int t = 1; t < lay.n_groups; ++t)
        if (i >= lay.start[t]) g = t;
      out = (sacc + part[i]) * lay.inv_sqrt_d[g] * kInvSqrtD;
    }
    qrot[row * kD + i] = out;
    qp[i] = out;
  }
  __syncthreads();
  write_frags(lay, qp, hq % sh.group, sh.group, frag_block(sh, ws, li, b, kvh, (hq % sh.group) >> 3), tid, kRotThreads);
}

__global__ void __launch_bounds__(kRotThreads) rotate_query_kernel(Shape sh, Workspace ws, int layer0,
                                                                   const __half* __restrict__ q, int batch,
                                                                   float* __restrict__ qrot) {
  rotate_body(sh, ws, layer0, q, batch, qrot, blockIdx.x);
}

// A decode step's preparation in one launch: the first n_rot CTAs rotate the
// query rows (as rotate_query_kernel), the others append the step's new K/V
// rows (as append_kernel, CTA a - n_rot = ((kind * n + row) * n_units + unit),
// n_units = layer_count * batch * Hkv).  The two parts are independent.
__global__ void __launch_bounds__(kRotThreads) prep_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                           const __half* __restrict__ q, int batch,
                                                           float* __restrict__ qrot, const __half* __restrict__ kx,
                                                           const __half* __restrict__ vx,
                                                           const int32_t* __restrict__ start_v,
                                                           const int32_t* __restrict__ count_v, int n, int n_rot,
                                                           int n_units) {
  extern __shared__ __align__(16) float mts[];  // [kD][kD], the append part
  if (static_cast<int>(blockIdx.x) < n_rot) {
    rotate_body(sh, ws, layer0, q, batch, qrot, blockIdx.x);
  } else {
    const int a = blockIdx.x - n_rot;
    append_body<kRotThreads>(sh, ws, cache, layer0, kx, vx, start_v, count_v, batch, n, a % n_units,
                             (a / n_units) % n, a / (n_units * n), mts);
  }
}

// ---------------------------------------------------------------------------
// a5: split-K decode straight from the packed tiles on the tensor cores.
//
// Grid (batch * Hkv * head_blocks, c_max, layer_count), 128 threads.  The
// split CTAs of a (layer, sequence, KV head, block of up to 8 query heads) share
// its 64-position tiles; each warp has its own 2-stage bulk-copy pipeline
// (K tile, V tile, norms -> shared memory, completion on an mbarrier) and its
// own online-softmax state.
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
constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kStages = 2;
constexpr int kDecMinBlocks = 3;  // CTAs per SM the register budget is sized for
constexpr int kWaitLimit = 1 << 20;  // polls of up to kPollSuspendNs each: about a second
constexpr float kRescaleSlack = 8.f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

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
  int bars, bq, tabk, grp, pdesc, ms, ls, mres, wsc, stage, stage_bytes, total;
};

__host__ __device__ inline int align128(int x) { return (x + 127) & ~127; }

__host__ __device__ inline DecodeLayout decode_layout(int kbits, int vbits) {
  DecodeLayout L;
  L.bars = 0;
  L.bq = align128(kDecWarps * kStages * 8);
  L.grp = L.bq + kMaxChunks * 32 * 16;    // a copy of DecodeTableDev: grp, tabk, pdesc, tabv
  L.tabk = L.grp + kNumGroupsMax * 8 * 4;
  L.pdesc = L.tabk + kNumGroupsMax * 8 * 4;
  L.ms = L.grp + static_cast<int>(sizeof(DecodeTableDev));
  L.ls = L.ms + kDecWarps * 8 * 4;
  L.mres = L.ls + kDecWarps * 8 * 4;           // merged m, l per head [2][8]
  L.wsc = L.mres + 2 * 8 * 4;                  // merge weights [warp][8]
  L.stage = align128(L.wsc + kDecWarps * 8 * 4);
  L.stage_bytes = 1024 * (kbits + vbits) + kTile * 8 + kTile * 2;
  const int stages = kDecWarps * kStages * L.stage_bytes;
  const int merge = kDecWarps * 8 * kD * 4;  // reuses the stage buffers after the loop
  int need = stages > merge ? stages : merge;
  if (need < kBufSmemBytes) need = kBufSmemBytes;  // the buffer CTA of a buffered call
  L.total = L.stage + need;
  return L;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// S[mu] += A(selector s[mu]) * (q~ hi + q~ lo) for the four M-tiles of a chunk.
template <bool WIDE>
__device__ __forceinline__ void chunk_mma(const ByteTab& t, const uint32_t* s, uint4 bf, float (*S)[4]) {
  uint32_t a[4][4];
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) {
    lookup4<WIDE ? 4 : 3>(t, s[mu], a[mu][0], a[mu][2]);
    lookup4<WIDE ? 4 : 3>(t, s[mu] >> 16, a[mu][1], a[mu][3]);
  }
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) mma16816(S[mu], a[mu][0], a[mu][1], a[mu][2], a[mu][3], bf.x, bf.y);
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) mma16816(S[mu], a[mu][0], a[mu][1], a[mu][2], a[mu][3], bf.z, bf.w);
}

// Logits of one width-B group for the warp's tile, S[mu][4] (M-tile mu):
// the group's full 16-coordinate chunks as quartets, then its partial chunk
// (if any) through the lane's descriptor pd: word offset (bits 0..11) and
// stride per plane word (bits 12..19) inside the partial region, bit 20 set
// for a half-quad lane, bit 21 for the upper half of its virtual lane.  Lanes
// with no coordinates read any word of the region: their B rows are zero.
template <int B>
__device__ __forceinline__ void group_logits(const uint32_t* gw, int nfull, bool partial, uint32_t pd,
                                             const uint4* bqg, const ByteTab& t, int lane, float (*S)[4]) {
#pragma unroll 1
  for (int j = 0; j < nfull; ++j) {
    uint32_t w[B], s[4];
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = gw[j * 32 * B + 32 * k + lane];
    quartet_decode<B>(w, s);
    chunk_mma<B == 4>(t, s, bqg[j * 32], S);
  }
  if (partial) {
    const uint32_t* pc = gw + nfull * 32 * B;
    const int base = pd & 0xFFF, stride = (pd >> 12) & 0xFF;
    uint32_t w[B], s[4];
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = pc[base + stride * k];
    quartet_decode<B>(w, s);
    if (pd & (1u << 20)) {
      const int sh = (pd >> 21) & 1 ? 16 : 0;
#pragma unroll
      for (int mu = 0; mu < 4; ++mu) {
        const uint32_t x = (s[mu] >> sh) & 0xFFFFu;
        s[mu] = (x & 0xFFu) | ((x & 0xFF00u) << 8);
      }
    }
    chunk_mma<B == 4>(t, s, bqg[nfull * 32], S);
  }
}

// The range of a decode call's sequence: the packed positions [lo, len) and
// the buffered row count, clamped the same way by every kernel that reads
// them (the combine raises the flag).
struct SeqRange {
  int len, lo, cnt;
  bool bad;
};

__device__ __forceinline__ SeqRange seq_range(const Shape& sh, const int32_t* seq_lens, const BufferArgs& buf, int b) {
  SeqRange r;
  r.len = seq_lens[b];
  r.lo = buf.pos_lo != nullptr ? buf.pos_lo[b] : 0;
  r.cnt = buf.k != nullptr ? buf.count[b] : 0;
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
// row's extra combine intermediate, which then counts as arrived.
__device__ void buffer_attend(const Shape& sh, const Workspace& ws, const BufferArgs& buf, const SeqRange& sr, int li,
                              int b, int h, int h0, int nh, int batch, unsigned char* smem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = sh.group;
  float* qs = reinterpret_cast<float*>(smem);   // [128 dims][8 heads]
  float* lg = qs + 8 * kD;                      // [8][kMaxBufferRows]
  float* ml = lg + 8 * kMaxBufferRows;          // [8][2]
  const int cnt = sr.cnt;
  const size_t qrow = ((static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G + h0) * kD;
  for (int i = tid; i < 8 * kD; i += kDecThreads) {
    const int hh = i / kD, dim = i % kD;
    qs[dim * 8 + hh] = hh < nh ? __half2float(buf.q[qrow + i]) * (kInvSqrtD * kLog2e) : 0.f;
  }
  __syncthreads();
  const size_t rstride = static_cast<size_t>(sh.n_kv_heads) * kD;
  const size_t base = (static_cast<size_t>(li) * batch + b) * buf.n_buf * rstride + static_cast<size_t>(h) * kD;
  for (int r = tid; r < cnt; r += kDecThreads) {
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
  for (int hh = warp; hh < 8; hh += kDecWarps) {
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
  float acc[8][8];
#pragma unroll
  for (int hh = 0; hh < 8; ++hh)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
#pragma unroll 4
  for (int r = rp; r < cnt; r += 8) {
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
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    float4* dst = reinterpret_cast<float4*>(red + (rp * 8 + hh) * kD + 8 * dg);
    dst[0] = make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
    dst[1] = make_float4(acc[hh][4], acc[hh][5], acc[hh][6], acc[hh][7]);
  }
  __syncthreads();
  const int d = tid;  // kDecThreads == kD: a thread per output dimension
  const size_t wrow0 = (static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + h0;
#pragma unroll
  for (int hh = 0; hh < 8; ++hh) {
    if (hh >= nh) break;
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
  __threadfence();
  __syncthreads();
  // the combine of a row with no packed position and no buffered row writes
  // zeros without counting arrivals: do not count this one either
  if (tid < nh && !(sr.lo >= sr.len && cnt == 0)) atomicAdd(ws.comb_count + wrow0 + tid, 1u);
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
template <int VB>
__global__ void __launch_bounds__(kDecThreads, kDecMinBlocks)
    decode_mma_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0, const float* __restrict__ qrot,
                      const int32_t* __restrict__ seq_lens, BufferArgs buf, int batch, SplitPlan plan,
                      int head_blocks) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const DecodeLayout DL = decode_layout(sh.kbits, VB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + DL.bars);
  uint4* bq = reinterpret_cast<uint4*>(smem_raw + DL.bq);
  uint32_t* tabk = reinterpret_cast<uint32_t*>(smem_raw + DL.tabk);
  int32_t* grp = reinterpret_cast<int32_t*>(smem_raw + DL.grp);
  uint32_t* pdesc = reinterpret_cast<uint32_t*>(smem_raw + DL.pdesc);
  float* ms = reinterpret_cast<float*>(smem_raw + DL.ms);
  float* ls = reinterpret_cast<float*>(smem_raw + DL.ls);
  unsigned char* stage_base = smem_raw + DL.stage;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
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
    for (int u = tid; u < static_cast<int>(sizeof(DecodeTableDev) / 16); u += kDecThreads) dst[u] = src[u];
  }
  if (tid < kDecWarps * kStages) mbar_init(&bars[tid], 1);
  __syncthreads();
  if (tid == 0) asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  // While the previous kernel may still run: an L2 prefetch hint for this
  // warp's first tiles, taken as if the sequence were full (the length is an
  // input, read only after the wait).  A prefetch reads nothing into the
  // CTA and leaves memory as it is, so a stale or unused line costs only
  // bandwidth; the copies below still read after the wait.
  if (lane == 0 && batch == 1 && cu >= 0) {
    // one sequence: its split count if it were full
    const int cg = split_ctas(plan, sh.ntiles, sh.ntiles);
    const int Wp = cg * kDecWarps;
    const int wp = warp * cg + cu;
    const uint32_t kb = 1024u * sh.kbits, vb = 1024u * VB;
#pragma unroll
    for (int k = 0; k < (cu < cg ? kStages : 0); ++k) {
      const int64_t tile = wp + static_cast<int64_t>(k) * Wp;
      if (tile >= sh.ntiles) break;
      const int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
      if (slot < 0) break;
      prefetch_l2(cache.ktile + slot * (kb / 4), kb);
      prefetch_l2(cache.vtile + slot * (vb / 4), vb);
      prefetch_l2(cache.knorm + slot * kTile * 4, kTile * 8);
      prefetch_l2(cache.vnorm + slot * kTile, kTile * 2);
    }
  }
  // Launched as a programmatic dependent of the previous kernel (the query
  // rotation): everything above reads only the library's tables; the
  // sequence lengths, rotated queries and cache are read after that kernel
  // has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the unit's q~ fragments (written by the query rotation): their loads go
  // out with the length reads below and land in shared memory further down
  const int nchunk = lay.chunk_base[ng - 1] + ((lay.size[ng - 1] + 15) >> 4);
  constexpr int kFragPerThread = (kFragEntries + kDecThreads - 1) / kDecThreads;
  uint4 fr[kFragPerThread];
  if (qrot == nullptr && cu >= 0) {
    const uint4* src = frag_block(sh, ws, li, b, h, hb);
#pragma unroll
    for (int i = 0; i < kFragPerThread; ++i) {
      const int u = tid + i * kDecThreads;
      if (u < 32 * nchunk) fr[i] = src[u];
    }
  }
  // the packed positions attended: [lo, len); lo > 0 when the caller keeps the
  // first positions unquantised (out-of-range values are flagged by the
  // combine kernel)
  const SeqRange sr = seq_range(sh, seq_lens, buf, b);
  if (cu < 0) {
    // the extra CTA of a buffered call: the unit's fp16 buffered rows
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    buffer_attend(sh, ws, buf, sr, li, b, h, h0, nh, batch, smem_raw + DL.stage);
    return;
  }
  const int len = sr.len, lo = sr.lo;
  const int tlo = lo / kTile;
  const int ntl = static_cast<int>(range_tiles(sr));
  // this unit's split CTAs (the same count the combine computes)
  __shared__ int64_t s_red[kDecWarps];
  const int64_t total = plan.fixed_tiles > 0 ? 0 : batch_tiles<kDecThreads>(sh, seq_lens, buf, batch, s_red);
  const int C = split_ctas(plan, ntl, total);
  if (cu >= C) {
    // not needed for this unit (its partials are slots 0 .. C-1)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    return;
  }
  // Tile t of the unit goes to warp (t mod W) / C of CTA (t mod W) mod C:
  // a partial last round of tiles is spread over all CTAs (and so over all
  // SMs) before any CTA gets a second one.
  const int W = C * kDecWarps;
  const int wu = warp * C + cu;
  const int my_tiles = wu < ntl ? (ntl - wu + W - 1) / W : 0;
  float* part_base = ws.partials +
                     (((static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + h0) * sh.max_splits + cu) *
                         kPartialStride;
  const size_t part_head_stride = static_cast<size_t>(sh.max_splits) * kPartialStride;
  {
    if (qrot == nullptr) {
#pragma unroll
      for (int i = 0; i < kFragPerThread; ++i) {
        const int u = tid + i * kDecThreads;
        if (u < 32 * nchunk) bq[u] = fr[i];
      }
    } else {
      // the split pass on its own: the fragments from the caller's q~
      // (fp32, record order): coordinates 16 j + 4 t .. + 3 of chunk c's
      // group for head t / 4 ... see write_frags for the layout
      const float* qsrc = qrot + ((static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G + h0) * kD;
      for (int u = tid; u < 32 * nchunk; u += kDecThreads) {
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
    tv.lo[0] = a0.x; tv.lo[1] = a0.y; tv.lo[2] = a0.z; tv.lo[3] = a0.w;
    tv.hi[0] = a1.x; tv.hi[1] = a1.y; tv.hi[2] = a1.z; tv.hi[3] = a1.w;
  }
  __syncthreads();

  // ---- per-warp pipeline over this warp's tiles ----
  const int kwords = 256 * sh.kbits, vwords = 256 * VB;
  const uint32_t kbytes = 4u * kwords, vbytes = 4u * vwords;
  const uint32_t stage_tx = kbytes + vbytes + kTile * 8 + kTile * 2;
  unsigned char* my_stage = stage_base + static_cast<size_t>(warp) * kStages * DL.stage_bytes;
  uint64_t* my_bars = bars + warp * kStages;

  auto issue = [&](int k) {  // lane 0: copy this warp's k-th tile into stage k % kStages
    const int tile = tlo + wu + k * W;
    int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
    if (slot < 0) {  // a page id outside the pool: flagged, page 0 read instead
      atomicOr(ws.err, kErrPage);
      slot = static_cast<int64_t>(layer * sh.n_kv_heads + h) * cache.n_pages;
    }
    unsigned char* dst = my_stage + (k % kStages) * DL.stage_bytes;
    uint64_t* bar = &my_bars[k % kStages];
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_expect_tx(bar, stage_tx);
    bulk_copy_g2s(dst, cache.ktile + slot * kwords, kbytes, bar);
    bulk_copy_g2s(dst + kbytes, cache.vtile + slot * vwords, vbytes, bar);
    bulk_copy_g2s(dst + kbytes + vbytes, cache.knorm + slot * kTile * 4, kTile * 8, bar);
    bulk_copy_g2s(dst + kbytes + vbytes + kTile * 8, cache.vnorm + slot * kTile, kTile * 2, bar);
  };
  if (lane == 0)
    for (int k = 0; k < kStages && k < my_tiles; ++k) issue(k);

  float O[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int r = 0; r < 4; ++r) O[m][r] = 0.f;
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_run[2] = {0.f, 0.f};
  int failed_at = -1;

  for (int k = 0; k < my_tiles; ++k) {
    if (!__all_sync(0xffffffffu, mbar_wait(&my_bars[k % kStages], (k / kStages) & 1))) {
      failed_at = k;
      break;
    }
    const unsigned char* st = my_stage + (k % kStages) * DL.stage_bytes;
    const uint32_t* kt = reinterpret_cast<const uint32_t*>(st);
    const uint32_t* vt = reinterpret_cast<const uint32_t*>(st + kbytes);
    const __half* kn = reinterpret_cast<const __half*>(st + kbytes + vbytes);
    const __half* vn = reinterpret_cast<const __half*>(st + kbytes + vbytes + kTile * 8);
    const int tpos = (tlo + wu + k * W) * kTile;
    const int nvalid = min(kTile, len - tpos);       // positions [nlow, nvalid) of the tile are attended
    const int nlow = max(0, lo - tpos);

    // logits, one width group at a time, each scaled by its per-token norm
    float L[4][4];
#pragma unroll
    for (int mu = 0; mu < 4; ++mu)
#pragma unroll
      for (int r = 0; r < 4; ++r) L[mu][r] = 0.f;
    for (int g = 0; g < ng; ++g) {
      const int4 gp = *reinterpret_cast<const int4*>(grp + g * 8);  // width, nfull, r, word
      const int chunk = grp[g * 8 + 4];
      ByteTab t;
      const uint4 tl = *reinterpret_cast<const uint4*>(tabk + 8 * g);
      const uint4 th = *reinterpret_cast<const uint4*>(tabk + 8 * g + 4);
      t.lo[0] = tl.x; t.lo[1] = tl.y; t.lo[2] = tl.z; t.lo[3] = tl.w;
      t.hi[0] = th.x; t.hi[1] = th.y; t.hi[2] = th.z; t.hi[3] = th.w;
      const uint32_t pd = pdesc[g * 32 + lane];
      const uint32_t* gw = kt + gp.w;
      const uint4* bqg = bq + chunk * 32 + lane;
      float S[4][4];
#pragma unroll
      for (int mu = 0; mu < 4; ++mu)
#pragma unroll
        for (int r = 0; r < 4; ++r) S[mu][r] = 0.f;
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
    // P V in V's rotated basis
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
    if (lane == 0 && k + kStages < my_tiles) issue(k + kStages);
  }
  // the combine kernel may be scheduled now; it waits for this grid before reading the partials
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool timed_out = failed_at >= 0;
  if (timed_out) {
    if (lane == 0) atomicOr(ws.err, kErrTimeout);
    // copies issued but not yet consumed: let them land (bounded) before the
    // stage buffers are reused or the CTA exits
    const int issued = min(my_tiles, failed_at + kStages);
    for (int k = failed_at; k < issued; ++k) mbar_wait(&my_bars[k % kStages], (k / kStages) & 1);
  }
  __syncthreads();
  // ---- merge the warps (the stage buffers are reused) ----
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], o);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], o);
  }
  float* accs = reinterpret_cast<float*>(stage_base);  // [warp][8 heads][128]
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
  if (__syncthreads_or(timed_out)) return;
  // per head: the common maximum, the warps' weights (warps without a tile
  // hold m = -inf, l = 0, acc = 0) and the weighted denominator
  float* wsc = reinterpret_cast<float*>(smem_raw + DL.wsc);
  float* mres = reinterpret_cast<float*>(smem_raw + DL.mres);
  if (tid < 8) {
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, ms[w * 8 + tid]);
    float lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float mw = ms[w * 8 + tid];
      const float sc = mw == -CUDART_INF_F ? 0.f : fast_exp2(mw - M);
      wsc[w * 8 + tid] = sc;
      lsum = fmaf(sc, ls[w * 8 + tid], lsum);
    }
    mres[tid] = M;
    mres[8 + tid] = lsum;
  }
  __syncthreads();
  const int i = tid;
  for (int hh = 0; hh < nh; ++hh) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) a = fmaf(wsc[w * 8 + hh], accs[(w * 8 + hh) * kD + i], a);
    float* part = part_base + hh * part_head_stride;
    part[4 + i] = a;
    if (i == 0) {
      part[0] = mres[hh];
      part[1] = mres[8 + hh];
    }
  }
}

// ---------------------------------------------------------------------------
// a6: combine the splits and rotate back.  Grid (layer_count*batch*Hq *
// kCombSlices), 256 threads.  Each CTA merges one slice of a row's splits
// (w_s = 2^(m_s - M), 0 for empty splits; lane = 4 rotated coordinates) into
// an intermediate (m, l, acc) in V's rotated basis.  In a buffered call the
// split pass has already posted the row's fp16 buffered rows as one more
// intermediate (acc unrotated).  The row's last CTA to finish (an arrival
// counter, reset by that CTA) merges them:
// o = (R_V^T sum_s w_s acc_s + w_buf acc_buf) / (sum_s w_s l_s + w_buf l_buf).
// ---------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;
// Up to this many rows per launch, every combine CTA loads its rotation
// column early (8 slices x 64 KB per row of L2 reads).
constexpr int kEarlyRotationRows = 256;
static_assert(kCombWarps * 4 <= kD, "a warp's lanes cover the 128 coordinates four at a time");

__global__ void __launch_bounds__(kCombThreads) combine_kernel(Shape sh, Workspace ws, int layer0,
                                                               const int32_t* __restrict__ seq_lens, int batch,
                                                               SplitPlan plan, BufferArgs buf, __half* __restrict__ out,
                                                               bool early_rotation) {
  const int has_buf = buf.k != nullptr ? 1 : 0;
  const int slice = blockIdx.x % kCombSlices;
  const int rowi = blockIdx.x / kCombSlices;
  const int hq = rowi % sh.n_q_heads;
  const int b = (rowi / sh.n_q_heads) % batch;
  const int li = rowi / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dd = tid & (kD - 1), half = tid >> 7;
  // A library table: this thread's half column of the inverse V rotation,
  // used if this CTA merges the row.  For a small launch every CTA reads it
  // before the split pass has finished, off the critical path; for a large
  // one (many layers per call) only the merging CTAs do, later.
  const float* mv = ws.mv + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
  float mvr[64];
  if (early_rotation) {
#pragma unroll
    for (int r = 0; r < 64; ++r) mvr[r] = __ldg(mv + (half * 64 + r) * kD + dd);
  }
  // the next kernel of the stream may start its own table-only set-up now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Launched as a programmatic dependent of the split pass: inputs, partials
  // and the output are touched only after that kernel has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const SeqRange sr = seq_range(sh, seq_lens, buf, b);
  if (sr.bad && tid == 0 && hq == 0 && slice == 0) atomicOr(ws.err, kErrSeqLen);
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  if (sr.lo >= sr.len && sr.cnt == 0) {
    if (slice == 0 && tid < kD) out[row * kD + tid] = __float2half(0.f);
    return;
  }
  const size_t wrow = (static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + hq;  // workspace row
  const float* part = ws.partials + wrow * sh.max_splits * kPartialStride;
  __shared__ float accs[kCombWarps][kD];
  __shared__ float msw[kCombWarps], lsw[kCombWarps];
  __shared__ float a_s[kD];
  __shared__ int last;
  float* mid = ws.comb_mid + (wrow * (kCombSlices + 1) + slice) * kPartialStride;
  // ---- one slice of the row's splits: warp w takes splits s0 + w + 8 j,
  // four at a time with all their loads in flight, merged online per warp
  // (lane = 4 rotated coordinates), then across the warps ----
  __shared__ int64_t s_red[kCombWarps];
  const int64_t total = plan.fixed_tiles > 0 ? 0 : batch_tiles<kCombThreads>(sh, seq_lens, buf, batch, s_red);
  const int n_splits = split_ctas(plan, range_tiles(sr), total);
  const int s0 = static_cast<int>((static_cast<int64_t>(slice) * n_splits) / kCombSlices);
  const int s1 = static_cast<int>((static_cast<int64_t>(slice + 1) * n_splits) / kCombSlices);
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
      mid[4 + tid] = a;
    }
    if (tid == 0) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kCombWarps; ++w) l = fmaf(msw[w] == -CUDART_INF_F ? 0.f : exp2f(msw[w] - M), lsw[w], l);
      mid[0] = M;
      mid[1] = l;
    }
  }
  // ---- the row's last CTA merges the intermediates ----
  const int nmid = kCombSlices + has_buf;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(ws.comb_count + wrow, 1u) == static_cast<unsigned>(nmid - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* mids = ws.comb_mid + wrow * (kCombSlices + 1) * kPartialStride;
  float mk[kCombSlices + 1], lk[kCombSlices + 1], ak[kCombSlices + 1];
#pragma unroll
  for (int k = 0; k <= kCombSlices; ++k) {
    if (k < nmid) {
      mk[k] = __ldcg(mids + k * kPartialStride);
      lk[k] = __ldcg(mids + k * kPartialStride + 1);
      ak[k] = __ldcg(mids + k * kPartialStride + 4 + dd);
    } else {
      mk[k] = -CUDART_INF_F;
      lk[k] = 0.f;
      ak[k] = 0.f;
    }
  }
  float Mt = -CUDART_INF_F;
#pragma unroll
  for (int k = 0; k <= kCombSlices; ++k) Mt = fmaxf(Mt, mk[k]);
  float Lt = 0.f, at = 0.f, ab = 0.f;
#pragma unroll
  for (int k = 0; k <= kCombSlices; ++k) {
    const float w = mk[k] == -CUDART_INF_F ? 0.f : exp2f(mk[k] - Mt);
    Lt = fmaf(w, lk[k], Lt);
    if (k < kCombSlices) at = fmaf(w, ak[k], at);  // rotated basis
    else ab = w * ak[k];                            // the buffer's rows, unrotated
  }
  if (tid < kD) a_s[tid] = at / Lt;
  if (tid == 0) ws.comb_count[wrow] = 0u;  // ready for the next call
  if (!early_rotation) {
#pragma unroll
    for (int r = 0; r < 64; ++r) mvr[r] = __ldg(mv + (half * 64 + r) * kD + dd);
  }
  __syncthreads();
  // inverse V rotation: two threads per output, half of the inputs each
  float o = 0.f;
#pragma unroll
  for (int r = 0; r < 64; ++r) o = fmaf(mvr[r], a_s[half * 64 + r], o);
  if (half == 1) accs[0][dd] = o;
  __syncthreads();
  if (half == 0) out[row * kD + dd] = __float2half(o + accs[0][dd] + ab / Lt);
}

// ---------------------------------------------------------------------------
// f2: per-layer logit MAE of the packed keys (K only).  For every causal pair
// (query i, key j), 0 <= j <= i < m, of a window of m cached positions
// w0 .. w0+m-1: |q_i . k_hat_j - q_i . k_j| / sqrt(D), where q_i . k_hat_j is
// the logit exactly as the split decode computes it (group_logits on the
// packed tile, q~ fragments in fp16 hi + lo, per-group norms) and
// q_i . k_j comes from the exact fp16 keys on the tensor cores (fp16
// products are exact in the fp32 accumulator).
//
// Grid (ceil(m / 4), layer_count * Hkv * head_blocks), 128 threads: warp w of
// CTA x owns query position i = 4 x + w and up to 8 query heads, and walks
// the key tiles 0 .. i.  The CTA rotates its 4 x 8 query rows (one pass
// over the block-diagonal rotation, a thread per output coordinate), builds
// each warp's q~ fragments in shared memory, and adds its per-head sums of
// |error| to mae (fp64 atomics); a second launch divides by the pair count.
// ---------------------------------------------------------------------------
constexpr int kMaeRows = kDecWarps * 8;  // query rows (position, head) per CTA

struct MaeLayout {  // byte offsets inside the dynamic shared memory
  int tab, q, frag, red, total;
};

__host__ __device__ inline MaeLayout mae_layout() {
  MaeLayout L;
  L.tab = 0;
  L.q = align128(L.tab + static_cast<int>(sizeof(DecodeTableDev)));
  L.frag = align128(L.q + kMaeRows * kD * 4);
  L.red = L.frag + kDecWarps * kFragEntries * 16;
  L.total = L.red + kDecWarps * 8 * 4;
  return L;
}

__global__ void __launch_bounds__(kDecThreads) logit_mae_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                                int seq, int w0, int m, const __half* __restrict__ q,
                                                                const __half* __restrict__ k, double* __restrict__ mae,
                                                                int head_blocks) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const MaeLayout ML = mae_layout();
  int32_t* grp = reinterpret_cast<int32_t*>(smem_raw + ML.tab);
  const uint32_t* tabk = reinterpret_cast<const uint32_t*>(smem_raw + ML.tab + offsetof(DecodeTableDev, tabk));
  const uint32_t* pdesc = reinterpret_cast<const uint32_t*>(smem_raw + ML.tab + offsetof(DecodeTableDev, pdesc));
  float* qs = reinterpret_cast<float*>(smem_raw + ML.q);  // [32 rows][128]
  float* red = reinterpret_cast<float*>(smem_raw + ML.red);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int hb = blockIdx.y % head_blocks;
  const int h = (blockIdx.y / head_blocks) % sh.n_kv_heads;
  const int li = blockIdx.y / (head_blocks * sh.n_kv_heads);
  const int layer = layer0 + li;
  const int G = sh.group;
  const int h0 = 8 * hb;
  const int nh = min(8, G - h0);
  const int lh = layer * sh.n_kv_heads + h;
  const LayoutDev& lay = ws.layouts[lh];
  {
    const uint4* src = reinterpret_cast<const uint4*>(ws.dectab + lh);
    uint4* dst = reinterpret_cast<uint4*>(grp);
    for (int u = tid; u < static_cast<int>(sizeof(DecodeTableDev) / 16); u += kDecThreads) dst[u] = src[u];
  }
  // the CTA's query rows r = 8 w + hh (position 4 x + w, head h0 + hh), permuted to record order
  for (int u = tid; u < kMaeRows * kD; u += kDecThreads) {
    const int r = u / kD, c = u % kD;
    const int i = kDecWarps * blockIdx.x + r / 8, hh = r % 8;
    float v = 0.f;
    if (i < m && hh < nh)
      v = __half2float(q[((static_cast<size_t>(li) * m + i) * sh.n_q_heads + h * G + h0 + hh) * kD + lay.perm[c]]);
    qs[u] = v;
  }
  __syncthreads();
  {
    // q~ = (1/sqrt(D)) (1/sqrt(d_g)) Pi_g q_g: thread tid = output coordinate
    const float* mt = ws.mkt + static_cast<size_t>(lh) * kD * kD;
    float acc[kMaeRows];
#pragma unroll
    for (int r = 0; r < kMaeRows; ++r) acc[r] = 0.f;
#pragma unroll 2
    for (int u = 0; u < kD; ++u) {
      const float mv = __ldg(mt + u * kD + tid);
#pragma unroll
      for (int r = 0; r < kMaeRows; ++r) acc[r] = fmaf(mv, qs[r * kD + u], acc[r]);
    }
    float scale = 0.f;
    if (tid < lay.n_positions) {
      int g = 0;
      for (int t = 1; t < lay.n_groups; ++t)
        if (tid >= lay.start[t]) g = t;
      scale = lay.inv_sqrt_d[g] * kInvSqrtD;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaeRows; ++r) qs[r * kD + tid] = acc[r] * scale;
  }
  __syncthreads();
  uint4* frag = reinterpret_cast<uint4*>(smem_raw + ML.frag);
  for (int w = 0; w < kDecWarps; ++w)
    for (int hh = 0; hh < nh; ++hh)
      write_frags(lay, qs + (8 * w + hh) * kD, h0 + hh, G, frag + w * kFragEntries, tid, kDecThreads);
  __syncthreads();

  // ---- this warp's query position against keys 0 .. i ----
  const int i = kDecWarps * blockIdx.x + warp;
  float sum[2] = {0.f, 0.f};
  if (i < m) {
    // exact-logit B fragments: head g8 of the block, dims 16 c + 2 t4 (+1, +8, +9)
    uint32_t bx[8][2];
    const bool head_ok = g8 < nh;
    const __half* qrow = q + ((static_cast<size_t>(li) * m + i) * sh.n_q_heads + h * G + h0 + g8) * kD;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      bx[c][0] = head_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * c + 2 * t4) : 0u;
      bx[c][1] = head_ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * c + 2 * t4 + 8) : 0u;
    }
    ByteTab t;
    const int ng = lay.n_groups;
    const int kwords = 256 * sh.kbits;
    const uint4* bq = frag + warp * kFragEntries;
    const size_t krow0 = static_cast<size_t>(li) * m;
    for (int tile = w0 / kTile; tile <= (w0 + i) / kTile; ++tile) {
      const int64_t slot = tile_slot(sh, cache, layer, seq, h, tile);
      if (slot < 0) {  // warp-uniform: skip the tile, flagged
        if (lane == 0) atomicOr(ws.err, kErrPage);
        continue;
      }
      const uint32_t* kt = cache.ktile + slot * kwords;
      const __half* kn = cache.knorm + slot * kTile * 4;
      float L[4][4];
#pragma unroll
      for (int mu = 0; mu < 4; ++mu)
#pragma unroll
        for (int r = 0; r < 4; ++r) L[mu][r] = 0.f;
      for (int g = 0; g < ng; ++g) {
        const int4 gp = *reinterpret_cast<const int4*>(grp + g * 8);  // width, nfull, r, word
        const int chunk = grp[g * 8 + 4];
        const uint4 tl = *reinterpret_cast<const uint4*>(tabk + 8 * g);
        const uint4 th = *reinterpret_cast<const uint4*>(tabk + 8 * g + 4);
        t.lo[0] = tl.x; t.lo[1] = tl.y; t.lo[2] = tl.z; t.lo[3] = tl.w;
        t.hi[0] = th.x; t.hi[1] = th.y; t.hi[2] = th.z; t.hi[3] = th.w;
        const uint32_t pd = pdesc[g * 32 + lane];
        const uint32_t* gw = kt + gp.w;
        const uint4* bqg = bq + chunk * 32 + lane;
        float S[4][4];
#pragma unroll
        for (int mu = 0; mu < 4; ++mu)
#pragma unroll
          for (int r = 0; r < 4; ++r) S[mu][r] = 0.f;
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
      // exact logits of the tile's keys that are in the window and causal
#pragma unroll
      for (int mu = 0; mu < 4; ++mu) {
        const int ja = tile * kTile + 16 * mu + g8 - w0, jb = ja + 8;  // window indices of rows g8, g8 + 8
        const bool oka = ja >= 0 && ja <= i, okb = jb >= 0 && jb <= i;
        const __half* ka = k + ((krow0 + (oka ? ja : 0)) * sh.n_kv_heads + h) * kD + 2 * t4;
        const __half* kb = k + ((krow0 + (okb ? jb : 0)) * sh.n_kv_heads + h) * kD + 2 * t4;
        float E[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t a0 = oka ? *reinterpret_cast<const uint32_t*>(ka + 16 * c) : 0u;
          const uint32_t a1 = okb ? *reinterpret_cast<const uint32_t*>(kb + 16 * c) : 0u;
          const uint32_t a2 = oka ? *reinterpret_cast<const uint32_t*>(ka + 16 * c + 8) : 0u;
          const uint32_t a3 = okb ? *reinterpret_cast<const uint32_t*>(kb + 16 * c + 8) : 0u;
          mma16816(E, a0, a1, a2, a3, bx[c][0], bx[c][1]);
        }
        const bool h0ok = 2 * t4 < nh, h1ok = 2 * t4 + 1 < nh;
        if (oka && h0ok) sum[0] += fabsf(L[mu][0] * kLn2 - E[0] * kInvSqrtD);
        if (oka && h1ok) sum[1] += fabsf(L[mu][1] * kLn2 - E[1] * kInvSqrtD);
        if (okb && h0ok) sum[0] += fabsf(L[mu][2] * kLn2 - E[2] * kInvSqrtD);
        if (okb && h1ok) sum[1] += fabsf(L[mu][3] * kLn2 - E[3] * kInvSqrtD);
      }
    }
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    sum[0] += __shfl_xor_sync(0xffffffffu, sum[0], o);
    sum[1] += __shfl_xor_sync(0xffffffffu, sum[1], o);
  }
  if (lane < 4) {
    red[warp * 8 + 2 * lane] = sum[0];
    red[warp * 8 + 2 * lane + 1] = sum[1];
  }
  __syncthreads();
  if (tid < nh) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) s += red[w * 8 + tid];
    atomicAdd(mae + static_cast<size_t>(li) * sh.n_q_heads + h * G + h0 + tid, static_cast<double>(s));
  }
}

__global__ void scale_kernel(double* x, int n, double s) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) x[i] *= s;
}

// Raises a kernel's dynamic shared-memory limit; callers keep the result in
// a function-local static of a function unique per kernel, so the attribute
// is set once per process and never inside a graph capture.
template <typename F>
cudaError_t set_smem(F* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

cudaError_t encode_smem_once() {
  static const cudaError_t status = set_smem(encode_kernel, sizeof(EncodeSmem));
  return status;
}

// Launches a kernel as a programmatic dependent of the previous kernel in
// the stream: it may start while that kernel finishes.  Every kernel
// launched this way reads only library tables before griddepcontrol.wait and
// everything produced by earlier work in the stream after it, so the chain
// append -> rotate -> split -> combine (and the next call's kernels) keeps
// stream order for all data while the table-only prologues overlap.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <int VB>
cudaError_t launch_decode_vb(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                             const float* qrot, const int32_t* seq_lens, const BufferArgs& buf, int batch,
                             const SplitPlan& plan, cudaStream_t stream) {
  // the largest layout over K widths, so one attribute value serves every call
  static const cudaError_t attr = set_smem(decode_mma_kernel<VB>, decode_layout(4, VB).total);
  if (attr != cudaSuccess) return attr;
  const int head_blocks = (s.group + 7) / 8;
  // units fastest, then split index: the CTAs every unit uses come first
  dim3 grid(batch * s.n_kv_heads * head_blocks, (buf.k != nullptr ? 1 : 0) + plan.c_max, layer_count);
  return launch_dependent(decode_mma_kernel<VB>, grid, dim3(kDecThreads), decode_layout(s.kbits, VB).total, stream, s,
                          ws, cache, layer0, qrot, seq_lens, buf, batch, plan, head_blocks);
}

template <int VB>
int ctas_per_sm_vb(const Shape& s) {
  static const cudaError_t attr = set_smem(decode_mma_kernel<VB>, decode_layout(4, VB).total);
  if (attr != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_mma_kernel<VB>, kDecThreads,
                                                    decode_layout(s.kbits, VB).total) != cudaSuccess)
    return 0;
  return n;
}

}  // namespace

int decode_ctas_per_sm(const Shape& s) {
  switch (s.vbits) {
    case 1: return ctas_per_sm_vb<1>(s);
    case 2: return ctas_per_sm_vb<2>(s);
    case 3: return ctas_per_sm_vb<3>(s);
    default: return ctas_per_sm_vb<4>(s);
  }
}

cudaError_t launch_energy(const Shape& s, const Workspace& ws, const __half* calib_q, int nq,
                          const __half* calib_k, int nk, int pairing, cudaStream_t stream) {
  dim3 grid(s.n_layers * s.n_kv_heads, kEnergyChunks);
  energy_kernel<<<grid, kD, 0, stream>>>(calib_q, nq, calib_k, nk, s.n_q_heads, s.n_kv_heads, s.group, s.n_layers,
                                         pairing, ws.energy_q, ws.energy_k, ws.err);
  return cudaGetLastError();
}

cudaError_t launch_encode(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                          int layer_count, const __half* k, const __half* v, const int32_t* start,
                          const int32_t* count, int batch, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const cudaError_t e = encode_smem_once();
  if (e != cudaSuccess) return e;
  if (n <= kAppendMaxRows) {
    // a few rows per sequence: rewrite only their code bits
    static const cudaError_t attr = set_smem(append_kernel, kD * kD * sizeof(float));
    if (attr != cudaSuccess) return attr;
    return launch_dependent(append_kernel, dim3(layer_count * batch * s.n_kv_heads, n, 2), dim3(kAppThreads),
                            kD * kD * sizeof(float), stream, s, ws, cache, layer0, k, v, start, count, batch, n);
  }
  // about two waves of CTAs (two fit an SM); each loops over its unit's tiles
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0)
      sms = 148;
  }
  const int units = layer_count * batch * s.n_kv_heads;
  const int tiles = (n + kTile - 1) / kTile + 1;  // rows may start inside a tile
  const int per_unit = std::max(1, std::min(tiles, (4 * sms) / (2 * units)));
  dim3 grid(units, per_unit, 2);
  encode_kernel<<<grid, kEncThreads, sizeof(EncodeSmem), stream>>>(s, ws, cache, layer0, k, v, start, count, batch, n);
  return cudaGetLastError();
}

cudaError_t launch_prep(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                        const __half* q, int batch, float* qrot, const __half* k, const __half* v,
                        const int32_t* start, const int32_t* count, int n, cudaStream_t stream) {
  static const cudaError_t attr = set_smem(prep_kernel, kD * kD * sizeof(float));
  if (attr != cudaSuccess) return attr;
  const int n_rot = layer_count * batch * s.n_q_heads;
  const int n_units = layer_count * batch * s.n_kv_heads;
  return launch_dependent(prep_kernel, dim3(n_rot + n_units * n * 2), dim3(kRotThreads), kD * kD * sizeof(float),
                          stream, s, ws, cache, layer0, q, batch, qrot, k, v, start, count, n, n_rot, n_units);
}

cudaError_t launch_rotate_query(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                                const __half* q, int batch, float* qrot, cudaStream_t stream) {
  return launch_dependent(rotate_query_kernel, dim3(layer_count * batch * s.n_q_heads), dim3(kRotThreads), 0, stream, s,
                          ws, layer0, q, batch, qrot);
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
  const int nsl = kCombSlices;  // the buffered rows, if any, come from the split pass
  const int rows = layer_count * batch * s.n_q_heads;
  return launch_dependent(combine_kernel, dim3(rows * nsl), dim3(kCombThreads), 0, stream, s, ws, layer0, seq_lens,
                          batch, plan, buf, out, rows <= kEarlyRotationRows);
}

cudaError_t launch_logit_mae(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                             int layer_count, int seq, int w0, int m, const __half* q, const __half* k, double* mae,
                             cudaStream_t stream) {
  static const cudaError_t attr = set_smem(logit_mae_kernel, mae_layout().total);
  if (attr != cudaSuccess) return attr;
  const int n = layer_count * s.n_q_heads;
  cudaError_t e = cudaMemsetAsync(mae, 0, sizeof(double) * n, stream);
  if (e != cudaSuccess) return e;
  const int head_blocks = (s.group + 7) / 8;
  dim3 grid((m + kDecWarps - 1) / kDecWarps, layer_count * s.n_kv_heads * head_blocks);
  logit_mae_kernel<<<grid, kDecThreads, mae_layout().total, stream>>>(s, ws, cache, layer0, seq, w0, m, q, k, mae,
                                                                     head_blocks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const double pairs = static_cast<double>(m) * (m + 1) / 2;
  scale_kernel<<<(n + 255) / 256, 256, 0, stream>>>(mae, n, 1.0 / pairs);
  return cudaGetLastError();
}

}  // namespace bgtq

// Device helpers shared by the kernels of the Block-GTQ packed-cache path
// (B200, sm_100a): constants, the cache's tile addressing, the tile format
// (bit-plane quartets, PRMT codebook lookups, pack / unpack), the tensor-core
// chunk of the logits, the query fragments and the launch helpers.  Internal
// to the library: every translation unit gets its own copy.
#pragma once
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


constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;

__host__ __device__ inline int align128(int x) { return (x + 127) & ~127; }

// Cache slot of tile t of (layer, sequence b, KV head h): contiguous, or
// through the block table of a paged cache.  -1 for a page id outside the
// pool (the caller raises kErrPage).
__device__ __forceinline__ int64_t tile_slot(const Shape& sh, const CacheDev& c, int layer, int b, int h, int64_t t) {
  if (c.n_pages == 0) return ((static_cast<int64_t>(layer) * sh.max_batch + b) * sh.n_kv_heads + h) * sh.ntiles + t;
  const int32_t page = __ldcg(c.block_table + static_cast<int64_t>(b) * sh.ntiles + t);  // through L2: see seq_range
  if (page < 0 || page >= c.n_pages) return -1;
  return (static_cast<int64_t>(layer) * sh.n_kv_heads + h) * c.n_pages + page;
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

// Shared-memory address of a generic pointer into shared memory.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Byte tables of the fp16 codebook (8 entries: the levels of widths 1..3,
// the positive levels of width 4): lo[i] / hi[i] hold the low / high bytes
// of entries 4i .. 4i+3.
struct ByteTab {
  uint32_t lo[2], hi[2];
};

// Four symbols (selector nibbles 0..3) -> two fp16x2 registers: symbols
// (0, 1) and (2, 3).  PRMT picks bytes 0..7 of its two table words by the
// nibble's low three bits.  Width 4 holds sign-magnitude symbols: the low
// three bits pick |level| from the 8-entry table.  For the sign, each
// nibble of sel >> 1 has the symbol's sign bit as its bit 2, so it picks
// 0x80 (sign set) or 0x00 from the words (0, 0x80808080); its bit 3 (the
// next symbol's bit 0) may switch PRMT to replicating that byte's top bit,
// which leaves the top bit as it is.  That top bit becomes the fp16 sign.
template <int B>
__device__ __forceinline__ void lookup4(const ByteTab& t, uint32_t sel, uint32_t& r01, uint32_t& r23) {
  uint32_t lo, hi;
  if constexpr (B <= 3) {
    lo = prmt(t.lo[0], t.lo[1], sel);
    hi = prmt(t.hi[0], t.hi[1], sel);
  } else {
    const uint32_t s7 = sel & 0x7777u;
    lo = prmt(t.lo[0], t.lo[1], s7);
    hi = prmt(t.hi[0], t.hi[1], s7);
    const uint32_t neg = prmt(0u, 0x80808080u, sel >> 1);
    hi ^= neg & 0x80808080u;
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

// D = A * B for one m16n8k16 tile (the accumulator starts at zero).
__device__ __forceinline__ void mma16816_zero(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
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
// Query rotation.  Grid (layer_count * batch * Hq), 128 threads.
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

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// S[mu] += A(selector s[mu]) * (q~ hi + q~ lo) for the four M-tiles of a
// chunk; FIRST: S starts at zero (the group's first chunk).
template <bool WIDE, bool FIRST>
__device__ __forceinline__ void chunk_mma(const ByteTab& t, const uint32_t* s, uint4 bf, float (*S)[4]) {
  uint32_t a[4][4];
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) {
    lookup4<WIDE ? 4 : 3>(t, s[mu], a[mu][0], a[mu][2]);
    lookup4<WIDE ? 4 : 3>(t, s[mu] >> 16, a[mu][1], a[mu][3]);
  }
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) {
    if constexpr (FIRST) mma16816_zero(S[mu], a[mu][0], a[mu][1], a[mu][2], a[mu][3], bf.x, bf.y);
    else mma16816(S[mu], a[mu][0], a[mu][1], a[mu][2], a[mu][3], bf.x, bf.y);
  }
#pragma unroll
  for (int mu = 0; mu < 4; ++mu) mma16816(S[mu], a[mu][0], a[mu][1], a[mu][2], a[mu][3], bf.z, bf.w);
}

// Logits of one width-B group for the warp's tile, S[mu][4] (M-tile mu):
// the group's full 16-coordinate chunks as quartets, then its partial chunk
// (if any) through the lane's descriptor pd: word offset (bits 0..11) and
// stride per plane word (bits 12..19) inside the partial region, bit 20 set
// for a half-quad lane, bit 21 for the upper half of its virtual lane.  Lanes
// with no coordinates read any word of the region: their B rows are zero.
// S need not be initialised: the group's first chunk overwrites it (a group
// has at least one chunk).
template <int B>
__device__ __forceinline__ void group_logits(const uint32_t* gw, int nfull, bool partial, uint32_t pd,
                                             const uint4* bqg, const ByteTab& t, int lane, float (*S)[4]) {
  if (nfull > 0) {
    uint32_t w[B], s[4];
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = gw[32 * k + lane];
    quartet_decode<B>(w, s);
    chunk_mma<B == 4, true>(t, s, bqg[0], S);
  }
#pragma unroll 1
  for (int j = 1; j < nfull; ++j) {
    uint32_t w[B], s[4];
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = gw[j * 32 * B + 32 * k + lane];
    quartet_decode<B>(w, s);
    chunk_mma<B == 4, false>(t, s, bqg[j * 32], S);
  }
  if (partial) {
    const uint32_t* pc = gw + nfull * 32 * B;
    const int base = pd & 0xFFF, stride = (pd >> 12) & 0xFF;
    uint32_t w[B], s[4];
#pragma unroll
    for (int k = 0; k < B; ++k) w[k] = pc[base + stride * k];
    quartet_decode<B>(w, s);
    {
      // a half-quad lane keeps the two nibble bytes of its half, each
      // followed by a zero byte (a PRMT from the word and zero); others keep s
      const uint32_t hsel = !(pd & (1u << 20)) ? 0x3210u : ((pd >> 21) & 1) ? 0x4342u : 0x4140u;
#pragma unroll
      for (int mu = 0; mu < 4; ++mu) s[mu] = prmt(s[mu], 0u, hsel);
    }
    if (nfull > 0) chunk_mma<B == 4, false>(t, s, bqg[nfull * 32], S);
    else chunk_mma<B == 4, true>(t, s, bqg[0], S);
  }
}

// Raises a kernel's dynamic shared-memory limit; callers keep the result in
// a function-local static of a function unique per kernel, so the attribute
// is set once per process and never inside a graph capture.
template <typename F>
cudaError_t set_smem(F* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

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

}  // namespace

}  // namespace bgtq

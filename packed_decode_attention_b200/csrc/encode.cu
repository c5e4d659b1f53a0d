// Kernels of the Block-GTQ path that write the cache or prepare a query
// (B200, sm_100a):
//
//   energy_kernel        label-free per-RoPE-block Q/K energy, exact 128-bit sums
//   encode_tc_kernel     TQ-MSE: rotate (tensor cores, fp16 rows x fp16 hi + lo
//                        rotation, fp32 accumulation), normalise (fp64),
//                        quantise, pack tiles
//   encode_kernel<true>  the same for K rows turned by RoPE on load (fp32 rotation)
//   append_kernel        the same for a few rows: patch only their code bits
//   rotate_query_kernel  q~ per width group (rotated basis, 1/sqrt(d_g), 1/sqrt(D))
//   prep_kernel          a decode step's appends and query rotation in one launch
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ;
// chatpaper summary / arXiv 2606.24033 abstract, blockgtq README) on top of
// TurboQuant-MSE (arXiv 2504.19874); split-K decoding after FlashAttention /
// FlashAttention-2 (arXiv 2205.14135, 2307.08691), both cited by the pages.
#include "common.cuh"

namespace bgtq {

namespace {

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
// Energy score.  Grid (L * Hkv, kEnergyChunks), 128 threads = one per dim.
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
// Encode.  Grid (layer_count * batch * Hkv, per_unit, 2 kinds), 256
// threads.  A CTA loads one (layer, KV head, kind)'s rotation and tables once
// and then takes every per_unit-th 64-position tile that the call writes for
// one sequence: it unpacks the tile's codes when the call writes only part of
// it, encodes its new rows (y = R x, norms in fp64, u = sqrt(d) y / n, code =
// #{thresholds <= u}) into the codes, and packs the tile again.
// encode_kernel<true> does this for K rows turned by RoPE on load, with the
// rotation in fp32 FMAs; encode_tc_kernel (below) for rows as they come, with
// the rotation on the tensor cores.
// ---------------------------------------------------------------------------
constexpr int kEncThreads = 256;

// Sum of squares of one (row, group) in fp64, in one fixed order shared by
// the tile encode and the appends (rows as they come): eight partial sums
// s_k over the positions j0 + k, j0 + k + 8, ... below j1, then
// ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)).  The eight chains keep
// the latency of the dependent adds off a thread's critical path; the
// squares of fp16 inputs are exact in fp64.
template <typename F>
__device__ __forceinline__ double sum_squares(int j0, int j1, F value) {
  double s[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll 2
  for (int j = j0; j < j1; j += 8) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (j + k < j1) {
        const double v = value(j + k);
        s[k] = fma(v, v, s[k]);
      }
    }
  }
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}
// fp16 per shared row of the tensor-core encode's operands: 272 bytes, so
// the 8 rows of an ldmatrix hit distinct banks
constexpr int kTcPitch = kD + 8;
// Dynamic shared memory of an append CTA: the rotation as fp16 hi + lo
// operand rows, or in fp32 for rows turned by RoPE
constexpr size_t append_smem_bytes(bool turn) {
  return turn ? kD * kD * sizeof(float) : 2 * kD * kTcPitch * sizeof(__half);
}

__device__ __forceinline__ void ldmatrix_x4(const void* row_addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(row_addr)));
}
constexpr int kEncTilesPerCta = 8;  // tiles a CTA encodes with one load of its rotation
// Column of element (coordinate j, row r) in xt[j][]: float4 groups of 4 rows,
// XOR-swizzled by j so that the transposed writes spread over the banks.
__device__ __forceinline__ int xt_col(int j, int r) { return (((r >> 2) ^ ((j >> 3) & 15)) << 2) | (r & 3); }

// The stored symbol of u's Lloyd-Max code for width w >= 1.  The code is
// the number of the 2^w - 1 ascending thresholds t[] that are <= u (ties go
// up), found by binary search.  Widths 1..3 store the code; width 4 stores
// it in sign-magnitude form (bit 3 = the level's sign, bits 0..2 = the rank
// of |level| among the positive levels: c - 8 for c >= 8, 15 - c below), so
// that the decode looks |level| up in an 8-entry table.
__device__ __forceinline__ int lloyd_code(const float* t, int w, float u) {
  int c = 0;
  for (int s = 1 << (w - 1); s > 0; s >>= 1)
    if (t[c + s - 1] <= u) c += s;
  if (w == 4) c = (c & 8) ? (c ^ 8) : (c ^ 15);
  return c;
}

// RoPE inside the encode: sin and cos of the angle p * theta of one block
// (theta = base^(-2j/D)), the product in fp64 reduced to [-pi, pi] with 2 pi
// split into two doubles, then the hardware sin / cos of the remainder
// (absolute error about 4e-7 on [-pi, pi]).
__device__ __forceinline__ void rope_sincos(double theta, int64_t p, float* s, float* c) {
  const double a = static_cast<double>(p) * theta;
  const double k = rint(a * 0.15915494309189535);  // a / (2 pi), to the nearest integer
  double r = fma(-k, 6.283185307179586, a);
  r = fma(-k, 2.4492935982947064e-16, r);
  __sincosf(static_cast<float>(r), s, c);
}

__device__ __forceinline__ double rope_theta(const RopeArgs& rope, int j) {
  return pow(rope.base, -2.0 * j / kD);
}

struct EncodeSmem {
  float xt[kD][kTile];           // new rows, transposed, record order (zero elsewhere), columns xt_col
  double theta[kD / 2];          // RoPE frequencies of the 64 blocks (rope.on only)
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

// TURN: K rows arrive before RoPE and are turned on load (see RopeArgs).
template <bool TURN>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                             const __half* __restrict__ kx,
                                                             const __half* __restrict__ vx,
                                                             const int32_t* __restrict__ start_v,
                                                             const int32_t* __restrict__ count_v, int batch, int n,
                                                             RopeArgs rope) {
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
  const bool turn = TURN && kind == 0;  // K rows taken before RoPE
  if (turn && tid < kD / 2) S.theta[tid] = rope_theta(rope, tid);
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
    if (!turn) {
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
    } else {
      // K before RoPE: a thread takes 8 blocks (8 c .. 8 c + 7) of a row,
      // both dims of each, and turns them by RoPE at the row's position
      for (int e = tid; e < kTile * 8; e += kEncThreads) {
        const int r = e >> 3, c = e & 7;
        float xa[8], xb[8];
  #pragma unroll
        for (int i = 0; i < 8; ++i) xa[i] = xb[i] = 0.f;
        if (r >= tr0 && r < tr1) {
          const __half* xr = xbase + static_cast<size_t>(r - tr0) * row_stride;
          // pairing 0: dims 8 c + i and 64 + 8 c + i; pairing 1: dims 16 c + 2 i and 16 c + 2 i + 1
          const uint4 u0 = *reinterpret_cast<const uint4*>(xr + (rope.pairing == 0 ? 8 * c : 16 * c));
          const uint4 u1 = *reinterpret_cast<const uint4*>(xr + (rope.pairing == 0 ? kD / 2 + 8 * c : 16 * c + 8));
          const __half* h0 = reinterpret_cast<const __half*>(&u0);
          const __half* h1 = reinterpret_cast<const __half*>(&u1);
          const int64_t p = tile * kTile + r;
  #pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = rope.pairing == 0 ? __half2float(h0[i]) : __half2float(i < 4 ? h0[2 * i] : h1[2 * i - 8]);
            const float bv =
                rope.pairing == 0 ? __half2float(h1[i]) : __half2float(i < 4 ? h0[2 * i + 1] : h1[2 * i - 7]);
            float sn, cs;
            rope_sincos(S.theta[8 * c + i], p, &sn, &cs);
            xa[i] = fmaf(a, cs, -bv * sn);
            xb[i] = fmaf(a, sn, bv * cs);
          }
        }
  #pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * c + i;
          const int da = rope.pairing == 0 ? j : 2 * j, db = rope.pairing == 0 ? j + kD / 2 : 2 * j + 1;
          const int ja = S.inv[da], jb = S.inv[db];
          S.xt[ja][xt_col(ja, r)] = xa[i];
          S.xt[jb][xt_col(jb, r)] = xb[i];
        }
      }
    }
    __syncthreads();
    // norms: fp64 sum of squares of the exact fp16 inputs (of the turned
    // fp32 values when K arrives before RoPE)
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
// Encode with the rotation on the tensor cores, for rows taken as they are
// (no RoPE turn; encode_kernel<true> keeps that path): the same tiles, norms
// and codes as encode_kernel.  Per tile, Y = X B with X[64 rows][128 dims]
// and B[d][i] = R[i][inv(d)] (R in record order, its inputs taken back to
// the dimension order of the rows), as mma.sync m16n8k16: X in fp16 (the
// inputs are fp16, so exact) and B split into fp16 hi + lo, two MMAs per
// product, fp32 accumulation.  Warp w computes rows 16 (w & 3) .. + 15 and
// record positions 64 (w >> 2) .. + 63; the codes follow from u = y sqrt(d)
// / n as before.
// ---------------------------------------------------------------------------
// The (layer, KV head, kind)'s fp16 hi / lo rotation operands (a library
// table, [out][in] rows of 256 bytes) into shared rows of kTcPitch: bh at
// dst, bl right after it.
__device__ __forceinline__ void stage_rotation_operands(const Workspace& ws, int lh, int kind, __half* dst, int tid,
                                                        int nthreads) {
  const uint4* src = reinterpret_cast<const uint4*>(ws.rb + (static_cast<size_t>(lh) * 2 + kind) * 2 * kD * kD);
#pragma unroll 4
  for (int u = tid; u < 2 * kD * kD / 8; u += nthreads) {
    const int row = u >> 4, c = u & 15;  // row of hi (0..127) then lo (128..255), 8 inputs
    *reinterpret_cast<uint4*>(dst + row * kTcPitch + 8 * c) = __ldg(src + u);
  }
}

// The thresholds of width w spread over 15 ascending entries: the first
// 2^(4-w) - 1 are -inf, then each threshold appears 2^(4-w) times.  Then
// c = #{entries <= u} = 2^(4-w) (code + 1) - 1, so a branch-free 4-step
// search serves every width and gives #{thresholds <= u} (ties go up) as
// lloyd_code does.
__device__ __forceinline__ void spread_thresholds(const float* thr, float (*thr16)[16], int tid, int nthreads) {
  for (int u = tid; u < 5 * 16; u += nthreads) {
    const int w = u >> 4, k = u & 15;
    const int m = w > 0 ? 1 << (4 - w) : 1;
    float t = CUDART_INF_F;  // entry 15 and width 0: never read
    if (w > 0 && k < 15) t = k < m - 1 ? -CUDART_INF_F : thr[w * 16 + (k - (m - 1)) / m];
    thr16[w][k] = t;
  }
}

// The code (width-4: its sign-magnitude symbol) from c = #{spread entries <= u}.
__device__ __forceinline__ int code_of_spread_count(int c, int w) {
  int code = ((c + 1) >> (4 - w)) - 1;
  if (w == 4) code = (code & 8) ? (code ^ 8) : (code ^ 15);
  return code;
}

struct EncodeTcSmem {
  __half x[kTile][kTcPitch];   // the tile's new rows in dimension order (zero elsewhere)
  __half bh[kD][kTcPitch];     // bh[i][d] = fp16(R[i][inv(d)])
  __half bl[kD][kTcPitch];     // bl[i][d] = fp16(R[i][inv(d)] - bh[i][d])
  float fac[kTile][kNumGroupsMax];
  __half nrm[kTile][kNumGroupsMax];
  uint8_t codes[kTile][kCodePitch];
  uint32_t words[1024];
  float thr16[5][16];           // width w's thresholds spread to 15 entries (see spread_thresholds)
  int32_t perm[kD];            // record position -> dimension
  int32_t gof[kD];             // group of each record position (-1: width 0)
  LayoutDev lay;
};

__global__ void __launch_bounds__(kEncThreads, 2) encode_tc_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                                   const __half* __restrict__ kx,
                                                                   const __half* __restrict__ vx,
                                                                   const int32_t* __restrict__ start_v,
                                                                   const int32_t* __restrict__ count_v, int batch,
                                                                   int n) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  EncodeTcSmem& S = *reinterpret_cast<EncodeTcSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  spread_thresholds(&ws.codebook->threshold[0][0], S.thr16, tid, kEncThreads);
  __syncthreads();
  const int ng = S.lay.n_groups;
  const int npos = S.lay.n_positions;
  if (tid < kD) {
    S.perm[tid] = kind == 0 ? S.lay.perm[tid] : tid;
    int g = -1;
    if (tid < npos) {
      g = 0;
      for (int t = 1; t < ng; ++t)
        if (tid >= S.lay.start[t]) g = t;
    }
    S.gof[tid] = g;
  }
  __syncthreads();
  stage_rotation_operands(ws, lh, kind, &S.bh[0][0], tid, kEncThreads);
  __syncthreads();
  const int mt = warp & 3, nh = warp >> 2;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int lrow = lane & 7, lmat = lane >> 3;  // ldmatrix: this lane's row and matrix
  // this thread's 16 output positions i = 64 nh + 8 nt + 2 t4 + c (col =
  // 2 nt + c): a byte each of group (bits 0..1) and width (bits 2..4), 0xFF
  // for a position that holds no code
  uint32_t colinfo[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int col = 0; col < 16; ++col) {
    const int i = 64 * nh + 8 * (col >> 1) + 2 * t4 + (col & 1);
    const int g = S.gof[i];
    const uint32_t byte = g < 0 ? 0xFFu : static_cast<uint32_t>(g | (S.lay.width[g] << 2));
    colinfo[col >> 2] |= byte << (8 * (col & 3));
  }
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
    // new rows -> x (dimension order, 16-byte copies)
    const size_t row_stride = static_cast<size_t>(sh.n_kv_heads) * kD;
    const __half* x = kind == 0 ? kx : vx;
    const __half* xbase = x + ((static_cast<size_t>(li) * batch + b) * n + (p0 - start)) * row_stride +
                          static_cast<size_t>(h) * kD;
    for (int e = tid; e < kTile * (kD / 8); e += kEncThreads) {
      const int r = e >> 4, c8 = e & 15;  // row, 8 dims
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (r >= tr0 && r < tr1) raw = *reinterpret_cast<const uint4*>(xbase + static_cast<size_t>(r - tr0) * row_stride + 8 * c8);
      *reinterpret_cast<uint4*>(&S.x[r][8 * c8]) = raw;
    }
    __syncthreads();
    // norms: fp64 sums of squares of the exact fp16 inputs of each group in
    // sum_squares' order.  K: a thread per (row, group).  V (one group of
    // 128): the row's four threads q take chains 2q and 2q + 1 each and meet
    // in the same tree through two shuffles.
    {
      const int r = tid >> 2, g = tid & 3;
      const bool row_in = r >= tr0 && r < tr1;
      double s2 = 0.0;
      bool mine = false;
      if (kind == 0) {
        mine = g < ng && row_in;
        if (mine) {
          const int j0 = S.lay.start[g];
          s2 = sum_squares(j0, j0 + S.lay.size[g],
                           [&](int j) { return static_cast<double>(__half2float(S.x[r][S.perm[j]])); });
        }
      } else {
        double c0 = 0.0, c1 = 0.0;
#pragma unroll 4
        for (int j = 2 * g; j < kD; j += 8) {
          const double v0 = __half2float(S.x[r][j]), v1 = __half2float(S.x[r][j + 1]);
          c0 = fma(v0, v0, c0);
          c1 = fma(v1, v1, c1);
        }
        double p = c0 + c1;                         // s_2q + s_2q+1
        p += __shfl_xor_sync(0xffffffffu, p, 1);    // (s0 + s1) + (s2 + s3), or the upper four
        s2 = p + __shfl_xor_sync(0xffffffffu, p, 2);
        mine = g == 0 && row_in;
      }
      float f = 0.f;
      __half nh16 = __float2half(0.f);
      if (mine) {
        const double nr = sqrt(s2);
        nh16 = __double2half(nr);
        f = nr > 0.0 ? static_cast<float>(sqrt(static_cast<double>(S.lay.size[g])) / nr) : 0.f;
      }
      S.fac[r][g] = f;
      S.nrm[r][g] = nh16;
    }
    // y = X B for this warp's 16 rows and 64 record positions
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
    const bool rows_touched = 16 * mt < tr1 && 16 * mt + 16 > tr0 && 64 * nh < npos;
    if (rows_touched) {
#pragma unroll 2
      for (int ks = 0; ks < kD / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        // matrices: rows +0 / +8 (lmat & 1), dims +0 / +8 (lmat >> 1)
        ldmatrix_x4(&S.x[16 * mt + 8 * (lmat & 1) + lrow][16 * ks + 8 * (lmat >> 1)], a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          uint32_t h0, h1, l0, l1;
          // matrices: hi dims +0, hi dims +8, lo dims +0, lo dims +8 (outputs n0 .. n0 + 7)
          const int n0 = 64 * nh + 8 * nt;
          const __half* brow = (lmat < 2 ? &S.bh[0][0] : &S.bl[0][0]) + (n0 + lrow) * kTcPitch + 16 * ks +
                               8 * (lmat & 1);
          ldmatrix_x4(brow, h0, h1, l0, l1);
          mma16816(acc[nt], a0, a1, a2, a3, h0, h1);
          mma16816(acc[nt], a0, a1, a2, a3, l0, l1);
        }
      }
    }
    __syncthreads();  // fac, nrm and the unpacked codes are in place
    if (rows_touched) {
      // the codes of 8 outputs at a time, their four search steps in
      // lockstep (8 independent shared loads per step, no branch per output)
      const int ra = 16 * mt + g8, rb = ra + 8;
      const bool oka = ra >= tr0 && ra < tr1, okb = rb >= tr0 && rb < tr1;
      const float* thr = &S.thr16[0][0];
#pragma unroll
      for (int nt0 = 0; nt0 < 8; nt0 += 2) {
        float u8[8];
        int w8[8], c8[8];
        bool st8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int nt = nt0 + (q >> 2), e = q & 3;
          const int col = 2 * nt + (e & 1);
          const uint32_t info = (colinfo[col >> 2] >> (8 * (col & 3))) & 0xFFu;
          st8[q] = info != 0xFFu && ((e >> 1) ? okb : oka);
          w8[q] = st8[q] ? static_cast<int>(info >> 2) : 4;  // a position with no code: any width
          u8[q] = acc[nt][e] * S.fac[(e >> 1) ? rb : ra][info & 3];
          c8[q] = 0;
        }
#pragma unroll
        for (int step = 8; step > 0; step >>= 1)
#pragma unroll
          for (int q = 0; q < 8; ++q) c8[q] += thr[16 * w8[q] + c8[q] + step - 1] <= u8[q] ? step : 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (!st8[q]) continue;
          const int nt = nt0 + (q >> 2), e = q & 3;
          S.codes[(e >> 1) ? rb : ra][64 * nh + 8 * nt + 2 * t4 + (e & 1)] =
              static_cast<uint8_t>(code_of_spread_count(c8[q], w8[q]));
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
// Encode for a few rows (decode-time appends): grid (layer_count * batch * Hkv,
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
template <int NT, bool TURN>
__device__ __forceinline__ void append_body(const Shape& sh, const Workspace& ws, const CacheDev& cache, int layer0,
                                            const __half* __restrict__ kx, const __half* __restrict__ vx,
                                            const int32_t* __restrict__ start_v, const int32_t* __restrict__ count_v,
                                            int batch, int n, int bx, int row, int kind, float* mts,
                                            RopeArgs rope) {
  const int tid = threadIdx.x;
  const int h = bx % sh.n_kv_heads;
  const int b = (bx / sh.n_kv_heads) % batch;
  const int li = bx / (sh.n_kv_heads * batch);
  const int layer = layer0 + li;
  const int lh = layer * sh.n_kv_heads + h;
  // the kind's rotation in shared memory, a library table read before the
  // inputs are ready: as the tensor-core encode's fp16 hi / lo operands
  // (rows as they come), or transposed in fp32 ([in][out]) for rows turned
  // by RoPE here
  if constexpr (!TURN) {
    stage_rotation_operands(ws, lh, kind, reinterpret_cast<__half*>(mts), tid, NT);
  } else {
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
  // Only now may the next kernel start: it then relies on all earlier work
  // of the stream having completed (see SplitPlan::early).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this row's values (row < n: inside the input whatever count is) and the
  // sequence's start and count, all in flight together; record order:
  // position i holds dim perm[i] (K), V keeps the dims
  const __half* x = (kind == 0 ? kx : vx) +
                    ((static_cast<size_t>(li) * batch + b) * n + row) * sh.n_kv_heads * kD + static_cast<size_t>(h) * kD;
  float xv = 0.f, xpv = 0.f;
  const bool turn = TURN && kind == 0;  // K before RoPE
  int dim = 0;
  if (kind == 0) {
    if (tid < lay.n_positions) {
      dim = lay.perm[tid];
      xv = __half2float(x[dim]);
      // the other dim of this dim's RoPE block
      if (turn) xpv = __half2float(x[rope.pairing == 0 ? dim ^ (kD / 2) : dim ^ 1]);
    }
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
  if (turn && tid < lay.n_positions) {
    // block (a, b) turns to (a cos - b sin, a sin + b cos)
    const bool first = rope.pairing == 0 ? dim < kD / 2 : (dim & 1) == 0;
    const int j = rope.pairing == 0 ? dim & (kD / 2 - 1) : dim >> 1;
    float sn, cs;
    rope_sincos(rope_theta(rope, j), pos, &sn, &cs);
    xv = first ? fmaf(xv, cs, -xpv * sn) : fmaf(xpv, sn, xv * cs);
  }
  if (tid < kD) xs[tid] = xv;
  __syncthreads();
  const int ng = lay.n_groups;
  // The group norms (fp64) and y = R x are independent: a thread per group
  // sums the squares, on threads 128.. beside the rotation with 256 threads,
  // else first.  Rows as they come: in the tile encode's eight-chain order,
  // with the tensor cores rotating (below).  Rows turned here by RoPE: in
  // coordinate order, as the fp32 tile encode does.
  const int i = tid;
  if constexpr (!TURN) {
    // a thread per group, in the tile encode's order (threads 128.. with 256)
    const int norm_tid = tid - (NT >= 2 * kD ? kD : 0);
    if (norm_tid >= 0 && norm_tid < ng) {
      const int j0 = lay.start[norm_tid];
      const double s2 = sum_squares(j0, j0 + lay.size[norm_tid], [&](int j) { return static_cast<double>(xs[j]); });
      const double nr = sqrt(s2);
      nrm[norm_tid] = __double2half(nr);
      fac[norm_tid] = nr > 0.0 ? static_cast<float>(sqrt(static_cast<double>(lay.size[norm_tid])) / nr) : 0.f;
    }
  } else {
    const int norm_tid = tid - (NT >= 2 * kD ? kD : 0);
    if (norm_tid >= 0 && norm_tid < ng) {
      const int j0 = lay.start[norm_tid], j1 = j0 + lay.size[norm_tid];
      double s2 = 0.0;
      for (int j = j0; j < j1; ++j) {
        const double v = xs[j];
        s2 += v * v;
      }
      const double nr = sqrt(s2);
      nrm[norm_tid] = __double2half(nr);
      fac[norm_tid] = nr > 0.0 ? static_cast<float>(sqrt(static_cast<double>(lay.size[norm_tid])) / nr) : 0.f;
    }
  }
  int g = 0;
  float y = 0.f;
  if (i < lay.n_positions)
    for (int t = 1; t < ng; ++t)
      if (i >= lay.start[t]) g = t;
  if constexpr (!TURN) {
    // y = R x on the tensor cores, exactly as the tile encode computes a
    // row (the same operands and the same order of MMAs per output): the
    // row is row 0 of the A tile (the others zero), warp w takes outputs
    // 8 (w NTL) .. 8 (w NTL + NTL) - 1
    __shared__ float ys[kD];
    constexpr int NTL = kD / 8 / (NT / 32);
    const int lane = tid & 31, warp = tid >> 5;
    const int lrow = lane & 7, lmat = lane >> 3;
    const __half* bh = reinterpret_cast<const __half*>(mts);
    uint32_t xa[kD / 16][2];
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
      xa[ks][0] = lane < 4 ? *reinterpret_cast<const uint32_t*>(x + 16 * ks + 2 * lane) : 0u;
      xa[ks][1] = lane < 4 ? *reinterpret_cast<const uint32_t*>(x + 16 * ks + 8 + 2 * lane) : 0u;
    }
    float acc[NTL][4];
#pragma unroll
    for (int t = 0; t < NTL; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < kD / 16; ++ks) {
#pragma unroll
      for (int t = 0; t < NTL; ++t) {
        const int n0 = 8 * (warp * NTL + t);
        uint32_t h0, h1, l0, l1;
        ldmatrix_x4(bh + ((lmat >> 1) * kD + n0 + lrow) * kTcPitch + 16 * ks + 8 * (lmat & 1), h0, h1, l0, l1);
        mma16816(acc[t], xa[ks][0], 0u, xa[ks][1], 0u, h0, h1);
        mma16816(acc[t], xa[ks][0], 0u, xa[ks][1], 0u, l0, l1);
      }
    }
    if (lane < 4) {
#pragma unroll
      for (int t = 0; t < NTL; ++t) {
        ys[8 * (warp * NTL + t) + 2 * lane] = acc[t][0];
        ys[8 * (warp * NTL + t) + 2 * lane + 1] = acc[t][1];
      }
    }
    __syncthreads();
    if (i < lay.n_positions) y = ys[i];
  } else {
    if (i < lay.n_positions) {
      const int j0 = lay.start[g], j1 = j0 + lay.size[g];
      for (int j = j0; j < j1; ++j) y = fmaf(xs[j], mts[j * kD + i], y);
    }
  }
  __syncthreads();
  const int tile = static_cast<int>(pos / kTile), p = static_cast<int>(pos % kTile);
  const int64_t slot = tile_slot(sh, cache, layer, b, h, tile);
  if (slot < 0) {  // uniform over the CTA; no barrier follows
    if (tid == 0) atomicOr(ws.err, kErrPage);
    return;
  }
  if (i < lay.n_positions) {
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

template <bool TURN>
__global__ void __launch_bounds__(kAppThreads) append_kernel(Shape sh, Workspace ws, CacheDev cache, int layer0,
                                                             const __half* __restrict__ kx,
                                                             const __half* __restrict__ vx,
                                                             const int32_t* __restrict__ start_v,
                                                             const int32_t* __restrict__ count_v, int batch, int n,
                                                             RopeArgs rope) {
  extern __shared__ __align__(16) float mts[];  // the rotation (append_smem_bytes)
  append_body<kAppThreads, TURN>(sh, ws, cache, layer0, kx, vx, start_v, count_v, batch, n, blockIdx.x, blockIdx.y,
                                 blockIdx.z, mts, rope);
}

// One query row (layer, sequence, query head) = bx, by a CTA of kRotThreads.
__device__ __forceinline__ void rotate_body(const Shape& sh, const Workspace& ws, int layer0,
                                            const __half* __restrict__ q, int batch, float* __restrict__ qrot,
                                            int bx) {
  const int hq = bx % sh.n_q_heads;
  const int b = (bx / sh.n_q_heads) % batch;
  const int li = bx / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const LayoutDev& lay = ws.layouts[layer * sh.n_kv_heads + kvh];
  const int tid = threadIdx.x, i = tid & (kD - 1), half = tid >> 7;
  // this thread's half column of the (block-diagonal) rotation, all loads in
  // flight at once; only the inputs of output i's group are loaded (the
  // column's other entries are zero)
  const float* mt = ws.mkt + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
  float m[64];
  int jlo = 0, jhi = 0;
  if (i < lay.n_positions) {
    int g = 0;
    for (int t = 1; t < lay.n_groups; ++t)
      if (i >= lay.start[t]) g = t;
    jlo = lay.start[g];
    jhi = jlo + lay.size[g];
  }
#pragma unroll
  for (int u = 0; u < 64; ++u) {
    const int j = half * 64 + u;
    m[u] = j >= jlo && j < jhi ? __ldg(mt + j * kD + i) : 0.f;
  }
  __shared__ float qp[kD];
  __shared__ float part[kD];
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  // Launched as a programmatic dependent of the previous kernel of the
  // stream: the query is read after it has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Only now may the decode kernel that follows start: it then relies on all
  // earlier work of the stream having completed (see SplitPlan::early).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
  extern __shared__ __align__(16) float mts[];  // the append part's rotation (append_smem_bytes)
  if (static_cast<int>(blockIdx.x) < n_rot) {
    rotate_body(sh, ws, layer0, q, batch, qrot, blockIdx.x);
  } else {
    const int a = blockIdx.x - n_rot;
    append_body<kRotThreads, false>(sh, ws, cache, layer0, kx, vx, start_v, count_v, batch, n, a % n_units,
                                    (a / n_units) % n, a / (n_units * n), mts, RopeArgs{0.0, 0, 0});
  }
}

cudaError_t encode_smem_once() {
  static const cudaError_t status = set_smem(encode_tc_kernel, sizeof(EncodeTcSmem));
  return status;
}

cudaError_t encode_rope_smem_once() {
  static const cudaError_t status = set_smem(encode_kernel<true>, sizeof(EncodeSmem));
  return status;
}

template <bool TURN>
cudaError_t append_smem_once() {
  static const cudaError_t status = set_smem(append_kernel<TURN>, append_smem_bytes(TURN));
  return status;
}

// Launches a kernel as a programmatic dependent of the previous kernel in
// the stream: it may start while that kernel finishes.  Every kernel
// launched this way reads only library tables before griddepcontrol.wait and
// everything produced by earlier work in the stream after it, so the chain
// append -> rotate -> split -> combine (and the next call's kernels) keeps
// stream order for all data while the table-only prologues overlap.
}  // namespace

cudaError_t launch_energy(const Shape& s, const Workspace& ws, const __half* calib_q, int nq,
                          const __half* calib_k, int nk, int pairing, cudaStream_t stream) {
  dim3 grid(s.n_layers * s.n_kv_heads, kEnergyChunks);
  energy_kernel<<<grid, kD, 0, stream>>>(calib_q, nq, calib_k, nk, s.n_q_heads, s.n_kv_heads, s.group, s.n_layers,
                                         pairing, ws.energy_q, ws.energy_k, ws.err);
  return cudaGetLastError();
}

cudaError_t launch_encode(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                          int layer_count, const __half* k, const __half* v, const int32_t* start,
                          const int32_t* count, int batch, int n, cudaStream_t stream, RopeArgs rope) {
  if (n <= 0) return cudaSuccess;
  const cudaError_t e = rope.on ? encode_rope_smem_once() : encode_smem_once();
  if (e != cudaSuccess) return e;
  if (n <= kAppendMaxRows) {
    // a few rows per sequence: rewrite only their code bits
    const cudaError_t attr = rope.on ? append_smem_once<true>() : append_smem_once<false>();
    if (attr != cudaSuccess) return attr;
    const dim3 agrid(layer_count * batch * s.n_kv_heads, n, 2);
    return rope.on ? launch_dependent(append_kernel<true>, agrid, dim3(kAppThreads), append_smem_bytes(true), stream,
                                      s, ws, cache, layer0, k, v, start, count, batch, n, rope)
                   : launch_dependent(append_kernel<false>, agrid, dim3(kAppThreads), append_smem_bytes(false), stream,
                                      s, ws, cache, layer0, k, v, start, count, batch, n, rope);
  }
  // CTAs per unit: at least two waves if every unit has rows, and at most
  // kEncTilesPerCta tiles per CTA (the counts are device data: a call may
  // write one sequence of a large batch; the CTAs of units without rows exit
  // at once)
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms <= 0)
      sms = 148;
  }
  const int units = layer_count * batch * s.n_kv_heads;
  const int tiles = (n + kTile - 1) / kTile + 1;  // rows may start inside a tile
  const int per_unit = std::max((tiles + kEncTilesPerCta - 1) / kEncTilesPerCta,
                                std::min(tiles, std::max(1, (4 * sms) / (2 * units))));
  dim3 grid(units, per_unit, 2);
  if (rope.on)
    encode_kernel<true><<<grid, kEncThreads, sizeof(EncodeSmem), stream>>>(s, ws, cache, layer0, k, v, start, count,
                                                                          batch, n, rope);
  else
    encode_tc_kernel<<<grid, kEncThreads, sizeof(EncodeTcSmem), stream>>>(s, ws, cache, layer0, k, v, start, count,
                                                                         batch, n);
  return cudaGetLastError();
}

cudaError_t launch_prep(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0, int layer_count,
                        const __half* q, int batch, float* qrot, const __half* k, const __half* v,
                        const int32_t* start, const int32_t* count, int n, cudaStream_t stream) {
  static const cudaError_t attr = set_smem(prep_kernel, append_smem_bytes(false));
  if (attr != cudaSuccess) return attr;
  const int n_rot = layer_count * batch * s.n_q_heads;
  const int n_units = layer_count * batch * s.n_kv_heads;
  return launch_dependent(prep_kernel, dim3(n_rot + n_units * n * 2), dim3(kRotThreads), append_smem_bytes(false),
                          stream, s, ws, cache, layer0, q, batch, qrot, k, v, start, count, n, n_rot, n_units);
}

cudaError_t launch_rotate_query(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                                const __half* q, int batch, float* qrot, cudaStream_t stream) {
  return launch_dependent(rotate_query_kernel, dim3(layer_count * batch * s.n_q_heads), dim3(kRotThreads), 0, stream, s,
                          ws, layer0, q, batch, qrot);
}

}  // namespace bgtq

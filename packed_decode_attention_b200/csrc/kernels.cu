// CUDA kernels of the Block-GTQ packed-cache path for B200 (sm_100a).
//
//   energy_kernel        label-free per-RoPE-block Q/K energy, exact 128-bit sums
//   encode_kernel<KIND>  TQ-MSE: rotate (fp32), normalise (fp64), quantise, bit-pack
//   rotate_query_kernel  q~ per width group (rotated basis, 1/sqrt(d_g), 1/sqrt(D))
//   decode_split_kernel  split-K flash decoding straight from the packed codes
//   combine_kernel       log-sum-exp merge of the splits + inverse V rotation
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ;
// chatpaper summary / arXiv 2606.24033 abstract, blockgtq README) on top of
// TurboQuant-MSE (arXiv 2504.19874); split-K decoding after FlashAttention /
// FlashAttention-2 (arXiv 2205.14135, 2307.08691), both cited by the pages.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "device_tables.h"

namespace bgtq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)

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
// a3: encode.  Grid (layer_count * batch * Hkv, ceil(n / 64)), 256 threads.
// Each CTA: 64 rows of one (layer, sequence, KV head).  Y = X R^T as a
// 64 x 128 x 128 fp32 register-tiled product (4 rows x 8 outputs per
// thread); the K rotation is block diagonal in record order, so each thread
// only runs over the groups its outputs fall in.
// ---------------------------------------------------------------------------
constexpr int kEncRows = 64;
constexpr int kEncThreads = 256;

struct EncodeSmem {
  float xt[kD][kEncRows];        // xt[j][r] = x[r][perm[j]]
  float mt[kD][kD];              // mt[j][i] = R[i][j]
  float fac[kEncRows][kNumGroupsMax];
  __half nrm[kEncRows][kNumGroupsMax];
  uint32_t rec[kEncRows][17];
  float thr[5][16];
  int32_t inv[kD];               // dim -> record position
  LayoutDev lay;
};

template <int KIND>
__global__ void __launch_bounds__(kEncThreads) encode_kernel(Shape sh, Workspace ws, CacheDev cache,
                                                             int layer0, const __half* __restrict__ x,
                                                             const int32_t* __restrict__ start_v,
                                                             const int32_t* __restrict__ count_v,
                                                             int batch, int n) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EncodeSmem& S = *reinterpret_cast<EncodeSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int h = blockIdx.x % sh.n_kv_heads;
  const int b = (blockIdx.x / sh.n_kv_heads) % batch;
  const int li = blockIdx.x / (sh.n_kv_heads * batch);
  const int layer = layer0 + li;
  const int start = start_v[b];
  const int count = count_v[b];
  if (start < 0 || count < 0 || count > n) {
    if (tid == 0 && blockIdx.y == 0) atomicOr(ws.err, kErrArg);
    return;
  }
  const int r0 = blockIdx.y * kEncRows;
  if (r0 >= count) return;
  const int rows = min(kEncRows, count - r0);
  const int bits_avg = KIND == 0 ? sh.kbits : sh.vbits;
  const int nwords = 4 * bits_avg;
  const int lh = layer * sh.n_kv_heads + h;

  // layout (K) or the trivial single group (V)
  if (KIND == 0) {
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
    }
  }
  for (int i = tid; i < 5 * 16; i += kEncThreads) (&S.thr[0][0])[i] = (&ws.codebook->threshold[0][0])[i];
  for (int i = tid; i < kEncRows * 17; i += kEncThreads) (&S.rec[0][0])[i] = 0u;
  const float* mglob = (KIND == 0 ? ws.mkt : ws.mvt) + static_cast<size_t>(lh) * kD * kD;
  for (int i = tid; i < kD * kD / 4; i += kEncThreads)
    reinterpret_cast<float4*>(&S.mt[0][0])[i] = reinterpret_cast<const float4*>(mglob)[i];
  __syncthreads();
  if (tid < kD) {
    if (KIND == 0) S.inv[S.lay.perm[tid]] = tid;
    else S.inv[tid] = tid;
  }
  __syncthreads();
  // rows -> xt (transposed, record order); rows past `rows` are zero
  const size_t row_stride = static_cast<size_t>(sh.n_kv_heads) * kD;
  const __half* xbase =
      x + ((static_cast<size_t>(li) * batch + b) * n + r0) * row_stride + static_cast<size_t>(h) * kD;
  for (int e = tid; e < kEncRows * kD; e += kEncThreads) {
    const int r = e / kD, dm = e % kD;
    const float v = r < rows ? __half2float(xbase[r * row_stride + dm]) : 0.f;
    S.xt[S.inv[dm]][r] = v;
  }
  __syncthreads();
  const int ng = S.lay.n_groups;
  const int npos = S.lay.n_positions;
  // per (row, group): norm in fp64, the fp16 stored norm and the factor sqrt(d)/n
  {
    const int r = tid >> 2, g = tid & 3;
    float f = 0.f;
    __half nh = __float2half(0.f);
    if (g < ng) {
      const int j0 = S.lay.start[g], j1 = j0 + S.lay.size[g];
      double s2 = 0.0;
      for (int j = j0; j < j1; ++j) {
        const double v = S.xt[j][r];
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
  // Y tile
  const int rg = tid >> 4, og = tid & 15;
  const int i0 = og * 8;
  if (i0 < npos && rg * 4 < rows) {
    int gi[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + q;
      int g = 0;
      for (int t = 1; t < ng; ++t)
        if (i >= S.lay.start[t]) g = t;
      gi[q] = i < npos ? g : -1;
    }
    // groups are contiguous in record order: run over the groups of the
    // first and last valid output (the rotation is zero elsewhere)
    const int glo = gi[0];
    int ghi = glo;
#pragma unroll
    for (int q = 1; q < 8; ++q)
      if (gi[q] > ghi) ghi = gi[q];
    const int jlo = S.lay.start[glo];
    const int jhi = S.lay.start[ghi] + S.lay.size[ghi];
    float acc[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[a][q] = 0.f;
    for (int j = jlo; j < jhi; ++j) {
      const float4 xv = *reinterpret_cast<const float4*>(&S.xt[j][rg * 4]);
      const float4 m0 = *reinterpret_cast<const float4*>(&S.mt[j][i0]);
      const float4 m1 = *reinterpret_cast<const float4*>(&S.mt[j][i0 + 4]);
      const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
      const float ms[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[a][q] = fmaf(xs[a], ms[q], acc[a][q]);
    }
    // quantise + pack
    int bo[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int g = gi[q];
      bo[q] = g >= 0 ? S.lay.bitoff[g] + (i0 + q - S.lay.start[g]) * S.lay.width[g] : 0;
    }
    const int base = bo[0] & ~31;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = rg * 4 + a;
      uint64_t word = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int g = gi[q];
        if (g < 0) continue;
        const int w = S.lay.width[g];
        const float u = acc[a][q] * S.fac[r][g];
        int code = 0;
        const int nt = (1 << w) - 1;
        for (int t = 0; t < nt; ++t) code += (S.thr[w][t] <= u) ? 1 : 0;
        word |= static_cast<uint64_t>(code) << (bo[q] - base);
      }
      if (r < rows) {
        atomicOr(&S.rec[r][base >> 5], static_cast<uint32_t>(word));
        const uint32_t hi = static_cast<uint32_t>(word >> 32);
        if (hi) atomicOr(&S.rec[r][(base >> 5) + 1], hi);
      }
    }
  }
  __syncthreads();
  // write records and norms; rows past capacity are skipped and flagged
  const size_t tok0 = ((static_cast<size_t>(layer) * sh.max_batch + b) * sh.n_kv_heads + h) * sh.capacity;
  const int chunks = nwords / 4;
  uint8_t* recbase = (KIND == 0 ? cache.krec : cache.vrec);
  bool over = false;
  for (int e = tid; e < rows * chunks; e += kEncThreads) {
    const int r = e / chunks, c = e % chunks;
    const int64_t pos = static_cast<int64_t>(start) + r0 + r;
    if (pos >= sh.capacity) {
      over = true;
      continue;
    }
    const uint4 v = make_uint4(S.rec[r][4 * c], S.rec[r][4 * c + 1], S.rec[r][4 * c + 2], S.rec[r][4 * c + 3]);
    reinterpret_cast<uint4*>(recbase + (tok0 + pos) * (16 * bits_avg))[c] = v;
  }
  if (tid < rows) {
    const int r = tid;
    const int64_t pos = static_cast<int64_t>(start) + r0 + r;
    if (pos < sh.capacity) {
      if (KIND == 0) {
        __half2 n01 = __halves2half2(S.nrm[r][0], S.nrm[r][1]);
        __half2 n23 = __halves2half2(S.nrm[r][2], S.nrm[r][3]);
        __half2* dst = reinterpret_cast<__half2*>(cache.knorm + (tok0 + pos) * 4);
        dst[0] = n01;
        dst[1] = n23;
      } else {
        cache.vnorm[tok0 + pos] = S.nrm[r][0];
      }
    } else {
      over = true;
    }
  }
  if (over) atomicOr(ws.err, kErrCapacity);
}

// ---------------------------------------------------------------------------
// a4: rotate the query.  Grid (layer_count * batch * Hq), 128 threads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) rotate_query_kernel(Shape sh, Workspace ws, int layer0,
                                                           const __half* __restrict__ q, int batch,
                                                           float* __restrict__ qrot) {
  const int hq = blockIdx.x % sh.n_q_heads;
  const int b = (blockIdx.x / sh.n_q_heads) % batch;
  const int li = blockIdx.x / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const LayoutDev& lay = ws.layouts[layer * sh.n_kv_heads + kvh];
  __shared__ float qp[kD];
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  const int i = threadIdx.x;
  qp[i] = __half2float(q[row * kD + lay.perm[i]]);
  __syncthreads();
  float out = 0.f;
  if (i < lay.n_positions) {
    int g = 0;
    for (int t = 1; t < lay.n_groups; ++t)
      if (i >= lay.start[t]) g = t;
    const float* mt = ws.mkt + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
    float s = 0.f;
    const int j1 = lay.start[g] + lay.size[g];
    for (int j = lay.start[g]; j < j1; ++j) s = fmaf(mt[j * kD + i], qp[j], s);
    out = s * lay.inv_sqrt_d[g] * kInvSqrtD;
  }
  qrot[row * kD + i] = out;
}

// ---------------------------------------------------------------------------
// a5: split-K decode from packed codes (SIMT fp32).
//
// Grid (n_splits, batch * Hkv, layer_count), 128 threads = 4 warps.  A CTA
// owns tokens [s*T, min((s+1)*T, len)) of one (layer, sequence, KV head);
// its warps take tiles of 32*TPL tokens round-robin and keep their own
// online-softmax state for the GP (padded) query heads of the group.
//
// Phase A (logits), lane = token (TPL tokens per lane): the K records sit in
// registers; the loop over record words is unrolled at compile time and the
// codes starting in each word are walked at run time (widths and group
// boundaries are uniform across the warp), so every code is one funnel
// shift + mask + a shared-memory centroid lookup, shared by all GP heads.
// Per group g the partial dot products q~_g . C[codes] are scaled by the
// token's group norm.  Logits are kept in log2 units (q~ * log2 e).
// Phase B (P V), lane = 4 rotated V coordinates: each token's weight
// p * n_V / sqrt(D) times the centroids of the lane's 4 codes.
// ---------------------------------------------------------------------------
constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;

template <int GP, int TPL>
struct DecodeSmem {
  float qs[kD][GP];
  float pw[kDecWarps][32 * TPL][GP];
  float accs[kDecWarps][GP][kD];
  uint32_t vr[kDecWarps][32 * TPL][17];
  float cent[5][16];
  float ms[kDecWarps][GP];
  float ls[kDecWarps][GP];
  LayoutDev lay;
};

template <int KB, int GP, int TPL>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(Shape sh, Workspace ws, CacheDev cache,
                                                                   int layer0, const float* __restrict__ qrot,
                                                                   const int32_t* __restrict__ seq_lens,
                                                                   int batch, int split_tokens) {
  constexpr int NW = 4 * KB;  // 32-bit words per K record
  constexpr int TILE = 32 * TPL;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DecodeSmem<GP, TPL>& S = *reinterpret_cast<DecodeSmem<GP, TPL>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x;
  const int h = blockIdx.y % sh.n_kv_heads;
  const int b = blockIdx.y / sh.n_kv_heads;
  const int li = blockIdx.z;
  const int layer = layer0 + li;
  int len = seq_lens[b];
  if (len < 0 || len > sh.capacity) len = 0;  // flagged by the combine kernel
  const int t0 = s * split_tokens;
  if (t0 >= len) return;
  const int t1 = min(t0 + split_tokens, len);
  const int G = sh.group;
  const int lh = layer * sh.n_kv_heads + h;

  if (tid < static_cast<int>(sizeof(LayoutDev) / 4))
    reinterpret_cast<int32_t*>(&S.lay)[tid] = reinterpret_cast<const int32_t*>(ws.layouts + lh)[tid];
  for (int i = tid; i < 5 * 16; i += kDecThreads) (&S.cent[0][0])[i] = (&ws.codebook->centroid[0][0])[i];
  {
    const float* qsrc = qrot + ((static_cast<size_t>(li) * batch + b) * sh.n_q_heads + h * G) * kD;
    for (int e = tid; e < kD * GP; e += kDecThreads) {
      const int hh = e / kD, i = e % kD;
      S.qs[i][hh] = hh < G ? qsrc[hh * kD + i] * kLog2e : 0.f;
    }
  }
  for (int e = tid; e < kDecWarps * GP * kD; e += kDecThreads) (&S.accs[0][0][0])[e] = 0.f;
  __syncthreads();

  const size_t tok0 = ((static_cast<size_t>(layer) * sh.max_batch + b) * sh.n_kv_heads + h) * sh.capacity;
  const uint8_t* krec = cache.krec + tok0 * (16 * KB);
  const __half* knorm = cache.knorm + tok0 * 4;
  const int vb = sh.vbits;
  const int vw = 4 * vb;
  const uint8_t* vrec = cache.vrec + tok0 * (16 * vb);
  const __half* vnorm = cache.vnorm + tok0;
  const float* cv = S.cent[vb];
  const uint32_t vmask = (1u << vb) - 1u;
  const int vbit0 = 4 * vb * lane;
  const int vw0 = vbit0 >> 5, vsh = vbit0 & 31;

  float m_run[GP], l_run[GP];
#pragma unroll
  for (int hh = 0; hh < GP; ++hh) {
    m_run[hh] = -CUDART_INF_F;
    l_run[hh] = 0.f;
  }

  for (int tile = t0 + warp * TILE; tile < t1; tile += kDecWarps * TILE) {
    // ---- phase A: logits, lane = token ----
    float L[TPL][GP];
    float vn[TPL];
    {
      uint32_t rec[TPL][NW + 1];
      float kn[TPL][kNumGroupsMax];
#pragma unroll
      for (int k = 0; k < TPL; ++k) {
        const int t = tile + lane + 32 * k;
        const int tt = t < t1 ? t : t0;
        const uint4* src = reinterpret_cast<const uint4*>(krec + static_cast<size_t>(tt) * (16 * KB));
#pragma unroll
        for (int c = 0; c < KB; ++c) {
          const uint4 v = __ldg(src + c);
          rec[k][4 * c] = v.x;
          rec[k][4 * c + 1] = v.y;
          rec[k][4 * c + 2] = v.z;
          rec[k][4 * c + 3] = v.w;
        }
        rec[k][NW] = 0u;
        const uint2 nv = __ldg(reinterpret_cast<const uint2*>(knorm + static_cast<size_t>(tt) * 4));
        const __half2 n01 = *reinterpret_cast<const __half2*>(&nv.x);
        const __half2 n23 = *reinterpret_cast<const __half2*>(&nv.y);
        kn[k][0] = __low2float(n01);
        kn[k][1] = __high2float(n01);
        kn[k][2] = __low2float(n23);
        kn[k][3] = __high2float(n23);
        vn[k] = t < t1 ? __half2float(vnorm[tt]) * kInvSqrtD : 0.f;
        // stage this token's V record for phase B
        const uint4* vsrc = reinterpret_cast<const uint4*>(vrec + static_cast<size_t>(tt) * (16 * vb));
        uint32_t* vdst = S.vr[warp][lane + 32 * k];
        for (int c = 0; c < vb; ++c) {
          const uint4 v = __ldg(vsrc + c);
          vdst[4 * c] = v.x;
          vdst[4 * c + 1] = v.y;
          vdst[4 * c + 2] = v.z;
          vdst[4 * c + 3] = v.w;
        }
        vdst[vw] = 0u;
      }
      float Sg[TPL][GP];
#pragma unroll
      for (int k = 0; k < TPL; ++k)
#pragma unroll
        for (int hh = 0; hh < GP; ++hh) {
          L[k][hh] = 0.f;
          Sg[k][hh] = 0.f;
        }
      const int npos = S.lay.n_positions;
      int p = 0, g = 0;
      int gend = S.lay.size[0];
      int bw = S.lay.width[0];
      uint32_t msk = (1u << bw) - 1u;
      const float* cb = S.cent[bw];
      int bo = 0;
      float curn[TPL];
#pragma unroll
      for (int k = 0; k < TPL; ++k) curn[k] = kn[k][0];
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        while (p < npos && bo < 32 * (w + 1)) {
          if (p == gend) {
#pragma unroll
            for (int k = 0; k < TPL; ++k)
#pragma unroll
              for (int hh = 0; hh < GP; ++hh) {
                L[k][hh] = fmaf(curn[k], Sg[k][hh], L[k][hh]);
                Sg[k][hh] = 0.f;
              }
            ++g;
#pragma unroll
            for (int k = 0; k < TPL; ++k) curn[k] = g == 1 ? kn[k][1] : (g == 2 ? kn[k][2] : kn[k][3]);
            gend += S.lay.size[g];
            bw = S.lay.width[g];
            msk = (1u << bw) - 1u;
            cb = S.cent[bw];
          }
          const int shf = bo - 32 * w;
          float c[TPL];
#pragma unroll
          for (int k = 0; k < TPL; ++k) c[k] = cb[__funnelshift_r(rec[k][w], rec[k][w + 1], shf) & msk];
#pragma unroll
          for (int hh = 0; hh < GP; ++hh) {
            const float qv = S.qs[p][hh];
#pragma unroll
            for (int k = 0; k < TPL; ++k) Sg[k][hh] = fmaf(qv, c[k], Sg[k][hh]);
          }
          ++p;
          bo += bw;
        }
      }
#pragma unroll
      for (int k = 0; k < TPL; ++k) {
        const bool valid = tile + lane + 32 * k < t1;
#pragma unroll
        for (int hh = 0; hh < GP; ++hh) {
          const float v = fmaf(curn[k], Sg[k][hh], L[k][hh]);
          L[k][hh] = valid ? v : -CUDART_INF_F;
        }
      }
    }
    // ---- online softmax over the tile ----
    float alpha[GP];
#pragma unroll
    for (int hh = 0; hh < GP; ++hh) {
      float mx = L[0][hh];
#pragma unroll
      for (int k = 1; k < TPL; ++k) mx = fmaxf(mx, L[k][hh]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mnew = fmaxf(m_run[hh], mx);
      alpha[hh] = exp2f(m_run[hh] - mnew);
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < TPL; ++k) {
        const float pv = exp2f(L[k][hh] - mnew);
        sum += pv;
        S.pw[warp][lane + 32 * k][hh] = pv * vn[k];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      l_run[hh] = fmaf(l_run[hh], alpha[hh], sum);
      m_run[hh] = mnew;
    }
    __syncwarp();
    // ---- phase B: P V in V's rotated basis, lane = 4 coordinates ----
    {
      float acc[GP][4];
#pragma unroll
      for (int hh = 0; hh < GP; ++hh) {
        const float4 a = *reinterpret_cast<const float4*>(&S.accs[warp][hh][4 * lane]);
        acc[hh][0] = a.x * alpha[hh];
        acc[hh][1] = a.y * alpha[hh];
        acc[hh][2] = a.z * alpha[hh];
        acc[hh][3] = a.w * alpha[hh];
      }
      const int ntok = min(TILE, t1 - tile);
      for (int tt = 0; tt < ntok; ++tt) {
        const uint32_t* vrow = S.vr[warp][tt];
        const uint32_t bits = __funnelshift_r(vrow[vw0], vrow[vw0 + 1], vsh);
        float c[4];
#pragma unroll
        for (int dk = 0; dk < 4; ++dk) c[dk] = cv[(bits >> (vb * dk)) & vmask];
#pragma unroll
        for (int hh = 0; hh < GP; ++hh) {
          const float pv = S.pw[warp][tt][hh];
#pragma unroll
          for (int dk = 0; dk < 4; ++dk) acc[hh][dk] = fmaf(pv, c[dk], acc[hh][dk]);
        }
      }
#pragma unroll
      for (int hh = 0; hh < GP; ++hh)
        *reinterpret_cast<float4*>(&S.accs[warp][hh][4 * lane]) =
            make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
    }
    __syncwarp();
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < GP; ++hh) {
      S.ms[warp][hh] = m_run[hh];
      S.ls[warp][hh] = l_run[hh];
    }
  }
  __syncthreads();
  // merge the warps; thread = rotated coordinate
  const int i = tid;
  for (int hh = 0; hh < G; ++hh) {
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, S.ms[w][hh]);
    float lsum = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float sc = exp2f(S.ms[w][hh] - M);
      lsum = fmaf(sc, S.ls[w][hh], lsum);
      a = fmaf(sc, S.accs[w][hh][i], a);
    }
    float* part = ws.partials +
                  ((((static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + h * G + hh) * sh.max_splits) + s) *
                      kPartialStride;
    part[4 + i] = a;
    if (i == 0) {
      part[0] = M;
      part[1] = lsum;
    }
  }
}

// ---------------------------------------------------------------------------
// a6: combine the splits and rotate back.  Grid (layer_count*batch*Hq), 256
// threads: the 8 warps share the splits (lane = 4 rotated coordinates),
// then o = R_V^T (sum_s w_s acc_s) / (sum_s w_s l_s), w_s = 2^(m_s - M).
// ---------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;

__global__ void __launch_bounds__(kCombThreads) combine_kernel(Shape sh, Workspace ws, int layer0,
                                                               const int32_t* __restrict__ seq_lens, int batch,
                                                               int split_tokens, __half* __restrict__ out) {
  const int hq = blockIdx.x % sh.n_q_heads;
  const int b = (blockIdx.x / sh.n_q_heads) % batch;
  const int li = blockIdx.x / (sh.n_q_heads * batch);
  const int layer = layer0 + li;
  const int kvh = hq / sh.group;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int len = seq_lens[b];
  if (len < 0 || len > sh.capacity) {
    if (tid == 0 && hq == 0) atomicOr(ws.err, kErrSeqLen);
    len = 0;
  }
  const size_t row = (static_cast<size_t>(li) * batch + b) * sh.n_q_heads + hq;
  const int nspl = (len + split_tokens - 1) / split_tokens;
  if (nspl == 0) {
    if (tid < kD) out[row * kD + tid] = __float2half(0.f);
    return;
  }
  const float* part =
      ws.partials + ((static_cast<size_t>(li) * sh.max_batch + b) * sh.n_q_heads + hq) * sh.max_splits * kPartialStride;
  __shared__ float red[kCombWarps];
  __shared__ float accs[kCombWarps][kD];
  __shared__ float lsw[kCombWarps];
  __shared__ float a_s[kD];
  float M = -CUDART_INF_F;
  for (int s = tid; s < nspl; s += kCombThreads) M = fmaxf(M, part[static_cast<size_t>(s) * kPartialStride]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < kCombWarps; ++w) M = fmaxf(M, red[w]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
#pragma unroll 4
  for (int s = warp; s < nspl; s += kCombWarps) {
    const float* p = part + static_cast<size_t>(s) * kPartialStride;
    const float wgt = exp2f(p[0] - M);
    lsum = fmaf(wgt, p[1], lsum);
    const float4 a = *reinterpret_cast<const float4*>(p + 4 + 4 * lane);
    acc.x = fmaf(wgt, a.x, acc.x);
    acc.y = fmaf(wgt, a.y, acc.y);
    acc.z = fmaf(wgt, a.z, acc.z);
    acc.w = fmaf(wgt, a.w, acc.w);
  }
  *reinterpret_cast<float4*>(&accs[warp][4 * lane]) = acc;
  if (lane == 0) lsw[warp] = lsum;
  __syncthreads();
  if (tid < kD) {
    float a = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) {
      a += accs[w][tid];
      l += lsw[w];
    }
    a_s[tid] = a / l;
  }
  __syncthreads();
  // inverse V rotation: thread pair (d, half) sums half of the 128 inputs
  const float* mv = ws.mv + static_cast<size_t>(layer * sh.n_kv_heads + kvh) * kD * kD;
  const int d = tid & (kD - 1), half = tid >> 7;
  float o = 0.f;
#pragma unroll 8
  for (int r = half * 64; r < half * 64 + 64; ++r) o = fmaf(mv[r * kD + d], a_s[r], o);
  if (half == 1) accs[0][d] = o;
  __syncthreads();
  if (half == 0) out[row * kD + d] = __float2half(o + accs[0][d]);
}

// Raises a kernel's dynamic shared-memory limit.  Callers keep the result
// in a function-local static of a function that is unique per kernel, so
// the attribute is set once per process and never inside a graph capture.
template <typename F>
cudaError_t set_smem(F* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

template <int KIND>
cudaError_t encode_smem_once() {
  static const cudaError_t status = set_smem(encode_kernel<KIND>, sizeof(EncodeSmem));
  return status;
}

template <int KB, int GP, int TPL>
cudaError_t launch_decode_t(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                            int layer_count, const float* qrot, const int32_t* seq_lens, int batch,
                            int split_tokens, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem<GP, TPL>);
  auto* fn = decode_split_kernel<KB, GP, TPL>;
  static const cudaError_t attr = set_smem(fn, smem);  // one static per instantiation
  if (attr != cudaSuccess) return attr;
  const int nspl = static_cast<int>((s.capacity + split_tokens - 1) / split_tokens);
  dim3 grid(nspl, batch * s.n_kv_heads, layer_count);
  fn<<<grid, kDecThreads, smem, stream>>>(s, ws, cache, layer0, qrot, seq_lens, batch, split_tokens);
  return cudaGetLastError();
}

template <int GP, int TPL>
cudaError_t launch_decode_g(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                            int layer_count, const float* qrot, const int32_t* seq_lens, int batch,
                            int split_tokens, cudaStream_t stream) {
  switch (s.kbits) {
    case 1: return launch_decode_t<1, GP, TPL>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
    case 2: return launch_decode_t<2, GP, TPL>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
    case 3: return launch_decode_t<3, GP, TPL>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
    default: return launch_decode_t<4, GP, TPL>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
  }
}

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
                          const int32_t* count, int batch, int n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const size_t smem = sizeof(EncodeSmem);
  cudaError_t e = encode_smem_once<0>();
  if (e != cudaSuccess) return e;
  e = encode_smem_once<1>();
  if (e != cudaSuccess) return e;
  dim3 grid(layer_count * batch * s.n_kv_heads, (n + kEncRows - 1) / kEncRows);
  encode_kernel<0><<<grid, kEncThreads, smem, stream>>>(s, ws, cache, layer0, k, start, count, batch, n);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  encode_kernel<1><<<grid, kEncThreads, smem, stream>>>(s, ws, cache, layer0, v, start, count, batch, n);
  return cudaGetLastError();
}

cudaError_t launch_rotate_query(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                                const __half* q, int batch, float* qrot, cudaStream_t stream) {
  rotate_query_kernel<<<layer_count * batch * s.n_q_heads, kD, 0, stream>>>(s, ws, layer0, q, batch, qrot);
  return cudaGetLastError();
}

cudaError_t launch_decode_split(const Shape& s, const Workspace& ws, const CacheDev& cache, int layer0,
                                int layer_count, const float* qrot, const int32_t* seq_lens, int batch,
                                int split_tokens, cudaStream_t stream) {
  if (s.group <= 4)
    return launch_decode_g<4, 4>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
  if (s.group <= 8)
    return launch_decode_g<8, 2>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
  return launch_decode_g<16, 1>(s, ws, cache, layer0, layer_count, qrot, seq_lens, batch, split_tokens, stream);
}

cudaError_t launch_combine(const Shape& s, const Workspace& ws, int layer0, int layer_count,
                           const int32_t* seq_lens, int batch, int split_tokens, __half* out,
                           cudaStream_t stream) {
  combine_kernel<<<layer_count * batch * s.n_q_heads, kCombThreads, 0, stream>>>(s, ws, layer0, seq_lens, batch,
                                                                                 split_tokens, out);
  return cudaGetLastError();
}

}  // namespace bgtq

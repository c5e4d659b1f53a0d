// The per-layer logit-MAE diagnostic of the Block-GTQ path (B200, sm_100a):
//
//   logit_mae_kernel     decode-path logits of the packed keys against exact ones
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (Block-GTQ;
// chatpaper summary / arXiv 2606.24033 abstract, blockgtq README) on top of
// TurboQuant-MSE (arXiv 2504.19874); split-K decoding after FlashAttention /
// FlashAttention-2 (arXiv 2205.14135, 2307.08691), both cited by the pages.
#include "common.cuh"

namespace bgtq {

namespace {

// ---------------------------------------------------------------------------
// Per-layer logit MAE of the packed keys (K only).  For every causal pair
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
        t.lo[0] = tl.x; t.lo[1] = tl.y;
        t.hi[0] = th.x; t.hi[1] = th.y;
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

}  // namespace

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

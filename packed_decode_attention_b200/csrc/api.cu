// The C ABI declared in include/bgtq.h.  Host logic only: argument checks,
// buffer carving, table construction and upload, kernel launches.  Every
// step of the path itself runs in the kernels (encode.cu, decode.cu, diag.cu).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/bgtq.h"
#include "device_tables.h"
#include "host_tables.h"

using bgtq::kD;

struct bgtq_state {
  bgtq_config cfg;
  bgtq::Shape shape;
  bgtq::Workspace ws;
  bgtq::CacheDev cache;
  size_t cache_off[4];
  size_t cache_bytes, ws_bytes;
  int split_tokens = 0;  // 0 = automatic
  int ctas_per_sm = 0;   // resident decode CTAs per SM (looked up on first use)
  int fused_clusters = -1;  // co-resident clusters of the fused decode (looked up on first use; 0: not usable)
  int fused_cluster_size = 8;
  int decode_mode = 0;      // 1: the fused decode where the GPU can run it; 0: rotation + split + combine
  int num_sms = 148;
  int device = -1;       // the CUDA device current at bgtq_create: its buffers live there
  bool ready = false;
  bool have_energy = false;
  std::vector<int8_t> widths;                    // [L][Hkv][64]
  std::vector<bgtq::GroupLayout> layouts;        // [L][Hkv]
  std::vector<float> krot;                       // [L][Hkv][4][128*128] per group, row-major d x d
  std::vector<float> vrot;                       // [L][Hkv][128*128]
  std::vector<uint64_t> energy_q, energy_k;      // [L][Hkv][64][2]
};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Allocation set, and for a paged cache a block table given.
bool cache_ready(const bgtq_state* st) { return st->ready && (st->cache.n_pages == 0 || st->cache.block_table); }

// A call that launches or copies runs on the device the state was created
// on: its cache, workspace and tables live there, and a launch on another
// device would read them through the wrong context.
int check_device(const bgtq_state* st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BGTQ_ERR_CUDA;
  return dev == st->device ? BGTQ_OK : BGTQ_ERR_INVALID_ARG;
}

constexpr int kMaxLayers = 65535;

int max_splits_of(const bgtq_config* c) { return c->max_splits == 0 ? 256 : c->max_splits; }

// The cache and the workspace of a config, estimated in floating point (an
// upper bound of the exact plan), each below 2^56 bytes.
bool sizes_in_range(const bgtq_config* c) {
  const double lh = double(c->n_layers) * c->n_kv_heads;
  const double tiles = c->page_pool_tiles > 0 ? lh * c->page_pool_tiles
                                              : lh * c->max_batch * ((c->capacity_tokens + 63) / 64);
  const double cache = tiles * (1024.0 * (c->k_avg_bits + c->v_avg_bits) + 64.0 * 10) + 4096.0;
  const double qrows = double(c->n_layers) * c->max_batch * c->n_q_heads;
  const int splits = c->max_splits == 0 ? 256 : c->max_splits;
  const double ws = lh * (4.0 * 128 * 128 * 4 + 16384.0) + qrows * (splits + 16.0) * 1024.0 + (1 << 20);
  const double limit = 72057594037927936.0;  // 2^56
  return cache < limit && ws < limit;
}

int validate_config(const bgtq_config* c) {
  if (!c) return BGTQ_ERR_NULL;
  if (c->n_layers < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->max_batch < 1) return BGTQ_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0 || c->n_q_heads / c->n_kv_heads > 16) return BGTQ_ERR_INVALID_ARG;
  if (c->head_dim != kD) return BGTQ_ERR_INVALID_ARG;
  if (c->k_avg_bits < 1 || c->k_avg_bits > 4 || c->v_avg_bits < 1 || c->v_avg_bits > 4) return BGTQ_ERR_INVALID_ARG;
  if (c->b_min < 0 || c->b_max > 4 || c->b_min > c->b_max) return BGTQ_ERR_INVALID_ARG;
  if (c->k_avg_bits < c->b_min || c->k_avg_bits > c->b_max) return BGTQ_ERR_INVALID_ARG;
  if (c->rope_pairing != 0 && c->rope_pairing != 1) return BGTQ_ERR_INVALID_ARG;
  if (c->max_splits < 0 || c->max_splits > 1024 || c->page_pool_tiles < 0) return BGTQ_ERR_INVALID_ARG;
  if (c->capacity_tokens < 1 || c->capacity_tokens > (int64_t(1) << 30)) return BGTQ_ERR_INVALID_ARG;
  // a call's layers are a grid dimension of every launch (at most 65535)
  if (c->n_layers > kMaxLayers) return BGTQ_ERR_INVALID_ARG;
  // the buffer plan's byte counts, bounded before any size_t arithmetic
  if (!sizes_in_range(c)) return BGTQ_ERR_INVALID_ARG;
  return BGTQ_OK;
}

struct Layout {
  size_t krec, knorm, vrec, vnorm, cache_total;
  size_t err, codebook, layouts, dectab, mkt, mvt, mv, rb, energy_q, energy_k, qrot, qfrag, partials, comb_mid,
      comb_count, ws_total;
};

int64_t tiles_of(const bgtq_config* c) { return (c->capacity_tokens + bgtq::kTile - 1) / bgtq::kTile; }

// q~ fragment bytes for calls of up to layer_count layers.
size_t frag_bytes(const bgtq_config* c, int layer_count) {
  const int hbs = (c->n_q_heads / c->n_kv_heads + 7) / 8;
  return size_t(layer_count) * c->max_batch * c->n_kv_heads * hbs * bgtq::kFragEntries * 16;
}

Layout plan(const bgtq_config* c) {
  Layout p{};
  // one slot per tile: every (layer, sequence, KV head) its own T tiles, or
  // a pool of page_pool_tiles pages per (layer, KV head)
  const size_t tiles = c->page_pool_tiles > 0
                           ? size_t(c->n_layers) * c->n_kv_heads * size_t(c->page_pool_tiles)
                           : size_t(c->n_layers) * c->max_batch * c->n_kv_heads * size_t(tiles_of(c));
  const size_t toks = tiles * bgtq::kTile;
  p.krec = 0;
  p.knorm = align_up(p.krec + tiles * 1024 * c->k_avg_bits);
  p.vrec = align_up(p.knorm + toks * 4 * sizeof(uint16_t));
  p.vnorm = align_up(p.vrec + tiles * 1024 * c->v_avg_bits);
  p.cache_total = align_up(p.vnorm + toks * sizeof(uint16_t));
  const size_t lh = size_t(c->n_layers) * c->n_kv_heads;
  p.err = 0;
  p.codebook = align_up(p.err + sizeof(uint32_t));
  p.layouts = align_up(p.codebook + sizeof(bgtq::CodebookDev));
  p.dectab = align_up(p.layouts + lh * sizeof(bgtq::LayoutDev));
  p.mkt = align_up(p.dectab + lh * sizeof(bgtq::DecodeTableDev));
  p.mvt = align_up(p.mkt + lh * kD * kD * sizeof(float));
  p.mv = align_up(p.mvt + lh * kD * kD * sizeof(float));
  p.rb = align_up(p.mv + lh * kD * kD * sizeof(float));
  p.energy_q = align_up(p.rb + lh * 2 * 2 * kD * kD * sizeof(uint16_t));
  p.energy_k = align_up(p.energy_q + size_t(bgtq::kEnergyChunks) * lh * 64 * 16);
  p.qrot = align_up(p.energy_k + size_t(bgtq::kEnergyChunks) * lh * 64 * 16);
  const size_t qrows = size_t(c->n_layers) * c->max_batch * c->n_q_heads;
  p.qfrag = align_up(p.qrot + qrows * kD * sizeof(float));
  p.partials = align_up(p.qfrag + frag_bytes(c, c->n_layers));
  p.comb_mid = align_up(p.partials + qrows * max_splits_of(c) * bgtq::kPartialStride * sizeof(float));
  p.comb_count = align_up(p.comb_mid + qrows * (bgtq::kCombSlices + 1) * bgtq::kPartialStride * sizeof(float));
  p.ws_total = align_up(p.comb_count + qrows * sizeof(uint32_t));
  return p;
}

// layers [layer, layer + layer_count) of the config (no overflow for any int32 inputs)
bool layer_range_ok(const bgtq_config& c, int32_t layer, int32_t layer_count) {
  return layer >= 0 && layer < c.n_layers && layer_count >= 1 && layer_count <= c.n_layers - layer;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

uint32_t half_bits(float x) {
  const __half h = __float2half_rn(x);
  uint16_t v;
  std::memcpy(&v, &h, 2);
  return v;
}

// PRMT byte tables of a width's fp16 codebook, indexed by stored symbol:
// words 0..3 hold the low bytes of entries 4i..4i+3, words 4..7 the high
// bytes.  Widths 1..3: entry e = level e.  Width 4 (sign-magnitude
// symbols): entry m = the positive level C[8 + m] for m = 0..7 (words 0, 1
// and 4, 5); the sign is applied from the symbol's bit 3.
void byte_table(int bits, uint32_t* out) {
  std::vector<float> cen, thr;
  bgtq::lloyd_max_codebook(bits, &cen, &thr);
  for (int i = 0; i < 8; ++i) out[i] = 0;
  const int entries = bits == 4 ? 8 : (1 << bits);
  for (int e = 0; e < entries; ++e) {
    const uint32_t h = half_bits(cen[bits == 4 ? 8 + e : e]);
    out[e >> 2] |= (h & 0xFFu) << (8 * (e & 3));
    out[4 + (e >> 2)] |= (h >> 8) << (8 * (e & 3));
  }
}

// The split decode kernel's table for one (layer, KV head) layout.
bgtq::DecodeTableDev decode_table(const bgtq::LayoutDev& d, int vbits) {
  bgtq::DecodeTableDev t;
  std::memset(&t, 0, sizeof(t));
  for (int g = 0; g < d.n_groups; ++g) {
    const int size = d.size[g], bw = d.width[g];
    t.grp[g][0] = bw;
    t.grp[g][1] = size >> 4;
    t.grp[g][2] = size & 15;
    t.grp[g][3] = d.tile_word[g];
    t.grp[g][4] = d.chunk_base[g];
    t.grp[g][5] = size;
    t.grp[g][6] = d.start[g];
    byte_table(bw, t.tabk[g]);
    // partial chunk: lanes with a full quad read their quartet (word k at
    // 8 nf k + g nf + t); the half-quad lanes read virtual lane g / 2 (word k
    // at 8 nf b + 4 k + g / 2, upper half for odd g); other lanes read word 0
    const int r = size & 15, nf = r >> 2;
    for (int ln = 0; ln < 32; ++ln) {
      const int gg = ln >> 2, tl = ln & 3;
      uint32_t pd = 0;
      if (tl < nf)
        pd = uint32_t(gg * nf + tl) | (uint32_t(8 * nf) << 12);
      else if ((r & 3) && tl == nf)
        pd = uint32_t(8 * nf * bw + (gg >> 1)) | (4u << 12) | (1u << 20) | (uint32_t(gg & 1) << 21);
      t.pdesc[g][ln] = pd;
    }
  }
  byte_table(vbits, t.tabv);
  return t;
}

// Builds the host tables for the current widths and uploads them.
int build_and_upload(bgtq_state* st, cudaStream_t stream) {
  const bgtq_config& c = st->cfg;
  const int L = c.n_layers, H = c.n_kv_heads;
  st->layouts.assign(size_t(L) * H, bgtq::GroupLayout());
  st->krot.assign(size_t(L) * H * 4 * kD * kD, 0.f);
  st->vrot.assign(size_t(L) * H * kD * kD, 0.f);
  std::vector<bgtq::LayoutDev> ldev(size_t(L) * H);
  std::vector<bgtq::DecodeTableDev> dtab(size_t(L) * H);
  std::vector<float> mkt(size_t(L) * H * kD * kD, 0.f), mvt(size_t(L) * H * kD * kD), mv(size_t(L) * H * kD * kD);
  std::vector<__half> rb(size_t(L) * H * 2 * 2 * kD * kD);
  for (int l = 0; l < L; ++l) {
    for (int h = 0; h < H; ++h) {
      const size_t lh = size_t(l) * H + h;
      int bw[bgtq::kBlocks];
      for (int j = 0; j < bgtq::kBlocks; ++j) bw[j] = st->widths[lh * bgtq::kBlocks + j];
      const bgtq::GroupLayout lay = bgtq::build_layout(bw, c.rope_pairing);
      st->layouts[lh] = lay;
      bgtq::LayoutDev& d = ldev[lh];
      std::memset(&d, 0, sizeof(d));
      d.n_groups = lay.n_groups;
      d.n_positions = lay.n_positions;
      for (int g = 0; g < bgtq::kNumGroupsMax; ++g) {
        d.width[g] = lay.width[g];
        d.size[g] = lay.size[g];
        d.start[g] = g < lay.n_groups ? lay.start[g] : lay.n_positions;
        d.bitoff[g] = lay.bitoff[g];
        d.inv_sqrt_d[g] = lay.size[g] > 0 ? static_cast<float>(1.0 / std::sqrt(double(lay.size[g]))) : 0.f;
      }
      for (int i = 0; i < kD; ++i) d.perm[i] = lay.perm[i];
      int word = 0, chunk = 0;
      for (int g = 0; g < bgtq::kNumGroupsMax; ++g) {
        d.tile_word[g] = word;
        d.chunk_base[g] = chunk;
        if (g < lay.n_groups) {
          word += 2 * lay.size[g] * lay.width[g];  // 64 positions x d x b bits
          chunk += (lay.size[g] + 15) / 16;
        }
      }
      float* mk = mkt.data() + lh * kD * kD;
      for (int g = 0; g < lay.n_groups; ++g) {
        const int dg = lay.size[g], s0 = lay.start[g];
        const std::vector<double> R =
            bgtq::haar_rotation(dg, bgtq::rotation_key(c.seed, l, h, 0, uint64_t(lay.width[g])));
        float* hr = st->krot.data() + (lh * 4 + g) * kD * kD;
        for (int i = 0; i < dg; ++i)
          for (int j = 0; j < dg; ++j) {
            const float v = static_cast<float>(R[size_t(i) * dg + j]);
            hr[i * dg + j] = v;
            mk[size_t(s0 + j) * kD + (s0 + i)] = v;  // transposed: [in][out]
          }
      }
      const std::vector<double> RV = bgtq::haar_rotation(kD, bgtq::rotation_key(c.seed, l, h, 1, uint64_t(c.v_avg_bits)));
      float* hv = st->vrot.data() + lh * kD * kD;
      float* vt = mvt.data() + lh * kD * kD;
      float* vv = mv.data() + lh * kD * kD;
      for (int i = 0; i < kD; ++i)
        for (int j = 0; j < kD; ++j) {
          const float v = static_cast<float>(RV[size_t(i) * kD + j]);
          hv[i * kD + j] = v;
          vv[i * kD + j] = v;
          vt[j * kD + i] = v;
        }
      // the tensor-core encode's operands: per kind, element (out i, in d) =
      // R[i][inv(d)] (inputs in the rows' dimension order), as fp16 hi and
      // lo = fp16(value - hi)
      for (int kind = 0; kind < 2; ++kind) {
        __half* hi = rb.data() + (lh * 2 + kind) * 2 * kD * kD;
        __half* lo = hi + kD * kD;
        for (int j = 0; j < kD; ++j) {
          const int d = kind == 0 ? lay.perm[j] : j;
          for (int i = 0; i < kD; ++i) {
            const float v = kind == 0 ? mk[size_t(j) * kD + i] : vt[size_t(j) * kD + i];
            const __half h16 = __float2half_rn(v);
            hi[size_t(i) * kD + d] = h16;
            lo[size_t(i) * kD + d] = __float2half_rn(v - __half2float(h16));
          }
        }
      }
    }
  }
  for (size_t i = 0; i < ldev.size(); ++i) dtab[i] = decode_table(ldev[i], c.v_avg_bits);
  cudaError_t e = cudaMemcpyAsync(st->ws.layouts, ldev.data(), ldev.size() * sizeof(bgtq::LayoutDev),
                                  cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->ws.dectab, dtab.data(), dtab.size() * sizeof(bgtq::DecodeTableDev),
                        cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->ws.mkt, mkt.data(), mkt.size() * 4, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->ws.mvt, mvt.data(), mvt.size() * 4, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->ws.mv, mv.data(), mv.size() * 4, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st->ws.rb, rb.data(), rb.size() * 2, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return BGTQ_ERR_CUDA;
  st->ready = true;
  return BGTQ_OK;
}

// Resident split CTAs the GPU holds at once (one wave): the automatic split
// plan spreads them over a call's (layer, sequence, KV head, head block)
// units (see split_for).
int split_slots(bgtq_state* st) {
  if (st->ctas_per_sm <= 0) st->ctas_per_sm = std::max(1, bgtq::decode_ctas_per_sm(st->shape));
  return st->ctas_per_sm * st->num_sms;
}

// CTAs of the fused decode the GPU holds at once (whole 8-CTA clusters); 0
// when it cannot run, and the decode calls then use the split pass and the
// combine.
// The cluster size (4 or 8 CTAs) whose one wave holds the most CTAs, the
// larger on a tie; looked up once per state.
int fused_slots(bgtq_state* st) {
  if (st->fused_clusters < 0) {
    const int c8 = std::max(0, bgtq::decode_fused_clusters(st->shape, 8));
    const int c4 = std::max(0, bgtq::decode_fused_clusters(st->shape, 4));
    st->fused_cluster_size = 4 * c4 > 8 * c8 ? 4 : 8;
    st->fused_clusters = st->fused_cluster_size == 4 ? c4 : c8;
  }
  return st->fused_clusters * st->fused_cluster_size;
}

// Whether the decode calls take the fused launch: requested and possible.
bool use_fused(bgtq_state* st) { return st->decode_mode == 1 && fused_slots(st) > 0; }

// The split plan of a fused decode call: as split_for, in whole clusters
// (a set split size rounds each unit's count up to whole clusters; the
// automatic plan spreads one wave of clusters over the units, at least one
// each).
bgtq::SplitPlan fused_plan(bgtq_state* st, int32_t layer_count, int32_t batch) {
  fused_slots(st);
  const int cl = st->fused_cluster_size;
  auto up = [cl](int64_t x) { return (x + cl - 1) / cl * cl; };
  const int head_blocks = (st->shape.group + 7) / 8;
  bgtq::SplitPlan p{};
  p.cluster = cl;
  p.units_per_seq = layer_count * st->cfg.n_kv_heads * head_blocks;
  const int64_t tiles = (st->cfg.capacity_tokens + bgtq::kTile - 1) / bgtq::kTile;
  const int64_t max_sp = max_splits_of(&st->cfg);
  if (st->split_tokens > 0) {
    p.fixed_tiles = st->split_tokens / bgtq::kTile;
    p.c_max = static_cast<int>(up(std::min<int64_t>(max_sp, (tiles + p.fixed_tiles - 1) / p.fixed_tiles)));
    p.budget = 0;
    return p;
  }
  const int64_t units = int64_t(p.units_per_seq) * batch;
  const int64_t budget = std::max<int64_t>(fused_slots(st), cl * units);
  const int64_t share2 = up(std::max<int64_t>(1, 2 * budget / units));
  p.budget = static_cast<int>(std::min<int64_t>(budget, INT32_MAX));
  p.fixed_tiles = 0;
  p.c_max = static_cast<int>(std::max<int64_t>(cl, std::min({up(max_sp), share2, up(tiles)})));
  return p;
}

}  // namespace

extern "C" {

int bgtq_required_bytes(const bgtq_config* cfg, size_t* cache_bytes, size_t* workspace_bytes) {
  const int v = validate_config(cfg);
  if (v != BGTQ_OK) return v;
  if (!cache_bytes || !workspace_bytes) return BGTQ_ERR_NULL;
  const Layout p = plan(cfg);
  *cache_bytes = p.cache_total;
  *workspace_bytes = p.ws_total;
  return BGTQ_OK;
}

int bgtq_create(const bgtq_config* cfg, void* d_cache, size_t cache_bytes, void* d_workspace,
                size_t workspace_bytes, void* stream, bgtq_state** out) {
  const int v = validate_config(cfg);
  if (v != BGTQ_OK) return v;
  if (!d_cache || !d_workspace || !out) return BGTQ_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(d_cache) | reinterpret_cast<uintptr_t>(d_workspace)) % kAlign) return BGTQ_ERR_ALIGNMENT;
  const Layout p = plan(cfg);
  if (cache_bytes < p.cache_total || workspace_bytes < p.ws_total) return BGTQ_ERR_BUFFER_SIZE;
  bgtq_state* st = new (std::nothrow) bgtq_state();
  if (!st) return BGTQ_ERR_HOST_ALLOC;
  st->cfg = *cfg;
  st->shape.n_layers = cfg->n_layers;
  st->shape.n_kv_heads = cfg->n_kv_heads;
  st->shape.n_q_heads = cfg->n_q_heads;
  st->shape.group = cfg->n_q_heads / cfg->n_kv_heads;
  st->shape.max_batch = cfg->max_batch;
  st->shape.kbits = cfg->k_avg_bits;
  st->shape.vbits = cfg->v_avg_bits;
  st->shape.max_splits = max_splits_of(cfg);
  st->shape.capacity = cfg->capacity_tokens;
  st->shape.ntiles = tiles_of(cfg);
  st->shape.drop_tile = -1;
  uint8_t* c8 = static_cast<uint8_t*>(d_cache);
  st->cache.ktile = reinterpret_cast<uint32_t*>(c8 + p.krec);
  st->cache.knorm = reinterpret_cast<__half*>(c8 + p.knorm);
  st->cache.vtile = reinterpret_cast<uint32_t*>(c8 + p.vrec);
  st->cache.vnorm = reinterpret_cast<__half*>(c8 + p.vnorm);
  st->cache.block_table = nullptr;
  st->cache.n_pages = cfg->page_pool_tiles;
  st->cache_off[0] = p.krec;
  st->cache_off[1] = p.knorm;
  st->cache_off[2] = p.vrec;
  st->cache_off[3] = p.vnorm;
  st->cache_bytes = p.cache_total;
  st->ws_bytes = p.ws_total;
  uint8_t* w8 = static_cast<uint8_t*>(d_workspace);
  st->ws.err = reinterpret_cast<uint32_t*>(w8 + p.err);
  st->ws.codebook = reinterpret_cast<bgtq::CodebookDev*>(w8 + p.codebook);
  st->ws.layouts = reinterpret_cast<bgtq::LayoutDev*>(w8 + p.layouts);
  st->ws.mkt = reinterpret_cast<float*>(w8 + p.mkt);
  st->ws.mvt = reinterpret_cast<float*>(w8 + p.mvt);
  st->ws.mv = reinterpret_cast<float*>(w8 + p.mv);
  st->ws.rb = reinterpret_cast<__half*>(w8 + p.rb);
  st->ws.energy_q = reinterpret_cast<unsigned __int128*>(w8 + p.energy_q);
  st->ws.energy_k = reinterpret_cast<unsigned __int128*>(w8 + p.energy_k);
  st->ws.dectab = reinterpret_cast<bgtq::DecodeTableDev*>(w8 + p.dectab);
  st->ws.qrot = reinterpret_cast<float*>(w8 + p.qrot);
  st->ws.qfrag = reinterpret_cast<uint4*>(w8 + p.qfrag);
  st->ws.partials = reinterpret_cast<float*>(w8 + p.partials);
  st->ws.comb_mid = reinterpret_cast<float*>(w8 + p.comb_mid);
  st->ws.comb_count = reinterpret_cast<uint32_t*>(w8 + p.comb_count);
  const size_t comb_count_bytes = p.ws_total - p.comb_count;
  st->widths.assign(size_t(cfg->n_layers) * cfg->n_kv_heads * bgtq::kBlocks, 0);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    delete st;
    return BGTQ_ERR_CUDA;
  }
  st->device = dev;
  {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0) st->num_sms = sms;
  }
  st->shape.n_sms = st->num_sms;
  bgtq::CodebookDev cb;
  std::memset(&cb, 0, sizeof(cb));
  for (int b = 1; b <= 4; ++b) {
    std::vector<float> cen, thr;
    bgtq::lloyd_max_codebook(b, &cen, &thr);
    for (size_t i = 0; i < cen.size(); ++i) cb.centroid[b][i] = cen[i];
    for (size_t i = 0; i < thr.size(); ++i) cb.threshold[b][i] = thr[i];
  }
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaMemcpyAsync(st->ws.codebook, &cb, sizeof(cb), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->ws.err, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->ws.comb_count, 0, comb_count_bytes, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    delete st;
    return BGTQ_ERR_CUDA;
  }
  *out = st;
  return BGTQ_OK;
}

void bgtq_destroy(bgtq_state* st) { delete st; }

int bgtq_allocate(bgtq_state* st, const void* d_calib_q, int32_t nq, const void* d_calib_k, int32_t nk, void* stream) {
  if (!st || !d_calib_q || !d_calib_k) return BGTQ_ERR_NULL;
  if (nq < 1 || nk < 1) return BGTQ_ERR_INVALID_ARG;
  const int dv = check_device(st);
  if (dv != BGTQ_OK) return dv;
  const bgtq_config& c = st->cfg;
  cudaStream_t s = as_stream(stream);
  if (bgtq::launch_energy(st->shape, st->ws, static_cast<const __half*>(d_calib_q), nq,
                          static_cast<const __half*>(d_calib_k), nk, c.rope_pairing, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  const size_t lh = size_t(c.n_layers) * c.n_kv_heads;
  const size_t n128 = size_t(bgtq::kEnergyChunks) * lh * 64;
  std::vector<uint64_t> pq(2 * n128), pk(2 * n128);
  uint32_t flag = 0;
  cudaError_t e = cudaMemcpyAsync(pq.data(), st->ws.energy_q, n128 * 16, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(pk.data(), st->ws.energy_k, n128 * 16, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, st->ws.err, sizeof(flag), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return BGTQ_ERR_CUDA;
  if (flag & bgtq::kErrNonFinite) return BGTQ_ERR_DEVICE;
  st->energy_q.assign(lh * 64 * 2, 0);
  st->energy_k.assign(lh * 64 * 2, 0);
  std::vector<double> scores(64);
  for (size_t i = 0; i < lh; ++i) {
    for (int j = 0; j < 64; ++j) {
      unsigned __int128 sq = 0, sk = 0;
      for (int ch = 0; ch < bgtq::kEnergyChunks; ++ch) {
        const size_t o = (size_t(ch) * lh + i) * 64 + j;
        sq += (static_cast<unsigned __int128>(pq[2 * o + 1]) << 64) | pq[2 * o];
        sk += (static_cast<unsigned __int128>(pk[2 * o + 1]) << 64) | pk[2 * o];
      }
      const size_t o = (i * 64 + j) * 2;
      st->energy_q[o] = static_cast<uint64_t>(sq);
      st->energy_q[o + 1] = static_cast<uint64_t>(sq >> 64);
      st->energy_k[o] = static_cast<uint64_t>(sk);
      st->energy_k[o + 1] = static_cast<uint64_t>(sk >> 64);
      scores[j] = bgtq::u128_to_double(st->energy_q[o], st->energy_q[o + 1]) *
                  bgtq::u128_to_double(st->energy_k[o], st->energy_k[o + 1]);
    }
    const std::vector<int> w = bgtq::greedy_allocate(scores.data(), c.k_avg_bits, c.b_min, c.b_max);
    for (int j = 0; j < 64; ++j) st->widths[i * 64 + j] = static_cast<int8_t>(w[j]);
  }
  st->have_energy = true;
  return build_and_upload(st, s);
}

int bgtq_set_allocation(bgtq_state* st, const int8_t* h_widths, void* stream) {
  if (!st || !h_widths) return BGTQ_ERR_NULL;
  const int dv = check_device(st);
  if (dv != BGTQ_OK) return dv;
  const bgtq_config& c = st->cfg;
  const size_t lh = size_t(c.n_layers) * c.n_kv_heads;
  for (size_t i = 0; i < lh; ++i) {
    int sum = 0;
    for (int j = 0; j < 64; ++j) {
      const int w = h_widths[i * 64 + j];
      if (w < c.b_min || w > c.b_max) return BGTQ_ERR_INVALID_ARG;
      sum += w;
    }
    if (sum != 64 * c.k_avg_bits) return BGTQ_ERR_INVALID_ARG;
  }
  std::memcpy(st->widths.data(), h_widths, lh * 64);
  return build_and_upload(st, as_stream(stream));
}

int bgtq_get_allocation(const bgtq_state* st, int8_t* h_widths) {
  if (!st || !h_widths) return BGTQ_ERR_NULL;
  if (!st->ready) return BGTQ_ERR_NOT_READY;
  std::memcpy(h_widths, st->widths.data(), st->widths.size());
  return BGTQ_OK;
}

int bgtq_get_energy(const bgtq_state* st, uint64_t* h_eq, uint64_t* h_ek) {
  if (!st || !h_eq || !h_ek) return BGTQ_ERR_NULL;
  if (!st->have_energy) return BGTQ_ERR_NOT_READY;
  std::memcpy(h_eq, st->energy_q.data(), st->energy_q.size() * 8);
  std::memcpy(h_ek, st->energy_k.data(), st->energy_k.size() * 8);
  return BGTQ_OK;
}

int bgtq_get_codebook(int32_t bits, float* h_centroids, float* h_thresholds) {
  if (!h_centroids || !h_thresholds) return BGTQ_ERR_NULL;
  if (bits < 1 || bits > 4) return BGTQ_ERR_INVALID_ARG;
  std::vector<float> cen, thr;
  bgtq::lloyd_max_codebook(bits, &cen, &thr);
  std::memcpy(h_centroids, cen.data(), cen.size() * 4);
  std::memcpy(h_thresholds, thr.data(), thr.size() * 4);
  return BGTQ_OK;
}

int bgtq_get_layout(const bgtq_state* st, int32_t layer, int32_t kv_head, int32_t* n_groups, int32_t* h_width,
                    int32_t* h_size, int32_t* h_perm) {
  if (!st || !n_groups || !h_width || !h_size || !h_perm) return BGTQ_ERR_NULL;
  if (!st->ready) return BGTQ_ERR_NOT_READY;
  if (layer < 0 || layer >= st->cfg.n_layers || kv_head < 0 || kv_head >= st->cfg.n_kv_heads) return BGTQ_ERR_INVALID_ARG;
  const bgtq::GroupLayout& L = st->layouts[size_t(layer) * st->cfg.n_kv_heads + kv_head];
  *n_groups = L.n_groups;
  for (int g = 0; g < 4; ++g) {
    h_width[g] = L.width[g];
    h_size[g] = L.size[g];
  }
  for (int i = 0; i < kD; ++i) h_perm[i] = L.perm[i];
  return BGTQ_OK;
}

int bgtq_get_rotation(const bgtq_state* st, int32_t layer, int32_t kv_head, int32_t kind, int32_t group, float* h_out,
                      int32_t* d) {
  if (!st || !h_out || !d) return BGTQ_ERR_NULL;
  if (!st->ready) return BGTQ_ERR_NOT_READY;
  if (layer < 0 || layer >= st->cfg.n_layers || kv_head < 0 || kv_head >= st->cfg.n_kv_heads) return BGTQ_ERR_INVALID_ARG;
  const size_t lh = size_t(layer) * st->cfg.n_kv_heads + kv_head;
  if (kind == 1) {
    std::memcpy(h_out, st->vrot.data() + lh * kD * kD, kD * kD * 4);
    *d = kD;
    return BGTQ_OK;
  }
  if (kind != 0) return BGTQ_ERR_INVALID_ARG;
  const bgtq::GroupLayout& L = st->layouts[lh];
  if (group < 0 || group >= L.n_groups) return BGTQ_ERR_INVALID_ARG;
  const int dg = L.size[group];
  std::memcpy(h_out, st->krot.data() + (lh * 4 + group) * kD * kD, size_t(dg) * dg * 4);
  *d = dg;
  return BGTQ_OK;
}

int bgtq_cache_offsets(const bgtq_state* st, size_t* out) {
  if (!st || !out) return BGTQ_ERR_NULL;
  for (int i = 0; i < 4; ++i) out[i] = st->cache_off[i];
  return BGTQ_OK;
}

int bgtq_encode_append(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                       const int32_t* d_start, const int32_t* d_count, int32_t batch, int32_t n, void* stream) {
  if (!st || !d_k || !d_v || !d_start || !d_count) return BGTQ_ERR_NULL;
  if (!cache_ready(st)) return BGTQ_ERR_NOT_READY;
  if (const int dv = check_device(st)) return dv;
  const bgtq_config& c = st->cfg;
  if (!layer_range_ok(c, layer, layer_count)) return BGTQ_ERR_INVALID_ARG;
  if (batch < 1 || batch > c.max_batch || n < 0 || n > (1 << 30) / 64) return BGTQ_ERR_INVALID_ARG;
  if (!aligned16(d_k) || !aligned16(d_v) || !aligned16(d_start) || !aligned16(d_count)) return BGTQ_ERR_ALIGNMENT;
  if (n == 0) return BGTQ_OK;
  return bgtq::launch_encode(st->shape, st->ws, st->cache, layer, layer_count, static_cast<const __half*>(d_k),
                             static_cast<const __half*>(d_v), d_start, d_count, batch, n, as_stream(stream)) ==
                 cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

int bgtq_encode_append_rope(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                            const int32_t* d_start, const int32_t* d_count, int32_t batch, int32_t n, double rope_base,
                            void* stream) {
  if (!st || !d_k || !d_v || !d_start || !d_count) return BGTQ_ERR_NULL;
  if (!cache_ready(st)) return BGTQ_ERR_NOT_READY;
  if (const int dv = check_device(st)) return dv;
  const bgtq_config& c = st->cfg;
  if (!layer_range_ok(c, layer, layer_count)) return BGTQ_ERR_INVALID_ARG;
  if (batch < 1 || batch > c.max_batch || n < 0 || n > (1 << 30) / 64) return BGTQ_ERR_INVALID_ARG;
  if (!std::isfinite(rope_base) || !(rope_base > 1.0)) return BGTQ_ERR_INVALID_ARG;
  if (!aligned16(d_k) || !aligned16(d_v) || !aligned16(d_start) || !aligned16(d_count)) return BGTQ_ERR_ALIGNMENT;
  if (n == 0) return BGTQ_OK;
  const bgtq::RopeArgs rope{rope_base, c.rope_pairing, 1};
  return bgtq::launch_encode(st->shape, st->ws, st->cache, layer, layer_count, static_cast<const __half*>(d_k),
                             static_cast<const __half*>(d_v), d_start, d_count, batch, n, as_stream(stream), rope) ==
                 cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

int bgtq_rotate_query(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q, int32_t batch, float* d_qrot,
                      void* stream) {
  if (!st || !d_q || !d_qrot) return BGTQ_ERR_NULL;
  if (!st->ready) return BGTQ_ERR_NOT_READY;
  if (const int dv = check_device(st)) return dv;
  const bgtq_config& c = st->cfg;
  if (!layer_range_ok(c, layer, layer_count)) return BGTQ_ERR_INVALID_ARG;
  if (batch < 1 || batch > c.max_batch) return BGTQ_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_qrot)) return BGTQ_ERR_ALIGNMENT;
  return bgtq::launch_rotate_query(st->shape, st->ws, layer, layer_count, static_cast<const __half*>(d_q), batch,
                                   d_qrot, as_stream(stream)) == cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

namespace {

int check_decode_args(const bgtq_state* st, int32_t layer, int32_t layer_count, int32_t batch) {
  if (!cache_ready(st)) return BGTQ_ERR_NOT_READY;
  if (const int dv = check_device(st)) return dv;
  const bgtq_config& c = st->cfg;
  if (!layer_range_ok(c, layer, layer_count)) return BGTQ_ERR_INVALID_ARG;
  if (batch < 1 || batch > c.max_batch) return BGTQ_ERR_INVALID_ARG;
  return BGTQ_OK;
}

// The split plan of a call (bgtq::SplitPlan).  A set split size t gives
// ceil(tiles / (t / 64)) CTAs per unit.  Automatic: one wave of resident CTAs
// (less `extra` per unit: the buffer CTA of a buffered call) spread over the
// units in proportion to their tiles, at most twice a unit's even share, the
// configured max_splits and the capacity's tile count.
bgtq::SplitPlan split_for(bgtq_state* st, int32_t layer_count, int32_t batch, int extra = 0) {
  const int head_blocks = (st->shape.group + 7) / 8;
  bgtq::SplitPlan p{};
  p.units_per_seq = layer_count * st->cfg.n_kv_heads * head_blocks;
  const int64_t tiles = (st->cfg.capacity_tokens + bgtq::kTile - 1) / bgtq::kTile;
  const int64_t max_sp = max_splits_of(&st->cfg);
  if (st->split_tokens > 0) {
    p.fixed_tiles = st->split_tokens / bgtq::kTile;
    p.c_max = static_cast<int>(std::min<int64_t>(max_sp, (tiles + p.fixed_tiles - 1) / p.fixed_tiles));
    p.budget = 0;
    return p;
  }
  const int64_t units = int64_t(p.units_per_seq) * batch;
  const int64_t budget = std::max<int64_t>(int64_t(split_slots(st)) - extra * units, units);
  const int64_t share2 = std::max<int64_t>(1, 2 * budget / units);
  p.budget = static_cast<int>(budget);
  p.fixed_tiles = 0;
  p.c_max = static_cast<int>(std::max<int64_t>(1, std::min({max_sp, share2, tiles})));
  return p;
}

// The plan of a split pass that directly follows the call's own query
// rotation or decode-step preparation (bgtq::SplitPlan::early): the pass
// may read the caller's arrays and copy its first tiles before its wait.
// The preparation kernel appends 1..kAppendMaxRows rows per sequence itself;
// more rows go through the encode, which has completed by then.
bgtq::SplitPlan after_prep(bgtq::SplitPlan p, const int32_t* d_start = nullptr, const int32_t* d_count = nullptr,
                           int32_t n = 0) {
  p.early = 1;
  if (n >= 1 && n <= bgtq::kAppendMaxRows) {
    p.app_start = d_start;
    p.app_count = d_count;
  }
  return p;
}

}  // namespace

int bgtq_decode_split(bgtq_state* st, int32_t layer, int32_t layer_count, const float* d_qrot,
                      const int32_t* d_seq_lens, int32_t batch, void* stream) {
  if (!st || !d_qrot || !d_seq_lens) return BGTQ_ERR_NULL;
  const int v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (!aligned16(d_qrot) || !aligned16(d_seq_lens)) return BGTQ_ERR_ALIGNMENT;
  return bgtq::launch_decode_split(st->shape, st->ws, st->cache, layer, layer_count, d_qrot, d_seq_lens, bgtq::BufferArgs{}, batch,
                                   split_for(st, layer_count, batch), as_stream(stream)) == cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

int bgtq_decode_combine(bgtq_state* st, int32_t layer, int32_t layer_count, const int32_t* d_seq_lens, int32_t batch,
                        void* d_out, void* stream) {
  if (!st || !d_seq_lens || !d_out) return BGTQ_ERR_NULL;
  const int v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (!aligned16(d_seq_lens) || !aligned16(d_out)) return BGTQ_ERR_ALIGNMENT;
  return bgtq::launch_combine(st->shape, st->ws, layer, layer_count, d_seq_lens, batch,
                              split_for(st, layer_count, batch), bgtq::BufferArgs{}, static_cast<__half*>(d_out),
                              as_stream(stream)) == cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

int bgtq_decode_attn(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q, const int32_t* d_seq_lens,
                     int32_t batch, void* d_out, void* stream) {
  if (!st || !d_q || !d_seq_lens || !d_out) return BGTQ_ERR_NULL;
  const int v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (!aligned16(d_q) || !aligned16(d_seq_lens) || !aligned16(d_out)) return BGTQ_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  if (use_fused(st))
    return bgtq::launch_decode_fused(st->shape, st->ws, st->cache, layer, layer_count, static_cast<const __half*>(d_q),
                                     d_seq_lens, batch, fused_plan(st, layer_count, batch),
                                     static_cast<__half*>(d_out), s) == cudaSuccess
               ? BGTQ_OK
               : BGTQ_ERR_CUDA;
  const bgtq::SplitPlan split = after_prep(split_for(st, layer_count, batch));
  if (bgtq::launch_rotate_query(st->shape, st->ws, layer, layer_count, static_cast<const __half*>(d_q), batch,
                                st->ws.qrot, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_decode_split(st->shape, st->ws, st->cache, layer, layer_count, nullptr, d_seq_lens, bgtq::BufferArgs{}, batch,
                                split, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_combine(st->shape, st->ws, layer, layer_count, d_seq_lens, batch, split, bgtq::BufferArgs{},
                           static_cast<__half*>(d_out), s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  return BGTQ_OK;
}

}  // extern "C"

namespace {

// Checks of a decode step's append arguments (n = 0: none).
int check_step_appends(const void* d_k, const void* d_v, const int32_t* d_start, const int32_t* d_count, int32_t n) {
  if (n < 0 || n > (1 << 30) / 64) return BGTQ_ERR_INVALID_ARG;
  if (n > 0 && (!d_k || !d_v || !d_start || !d_count)) return BGTQ_ERR_NULL;
  if (n > 0 && (!aligned16(d_k) || !aligned16(d_v) || !aligned16(d_start) || !aligned16(d_count)))
    return BGTQ_ERR_ALIGNMENT;
  return BGTQ_OK;
}

// A decode step's appends and query rotation: one launch for 1..16 rows per
// sequence (they are independent), else the encode (if any) then the rotation.
cudaError_t queue_step_prep(bgtq_state* st, int32_t layer, int32_t layer_count, const __half* q, int32_t batch,
                            const void* d_k, const void* d_v, const int32_t* d_start, const int32_t* d_count,
                            int32_t n, cudaStream_t s) {
  const __half* k = static_cast<const __half*>(d_k);
  const __half* v = static_cast<const __half*>(d_v);
  if (n >= 1 && n <= bgtq::kAppendMaxRows)
    return bgtq::launch_prep(st->shape, st->ws, st->cache, layer, layer_count, q, batch, st->ws.qrot, k, v, d_start,
                             d_count, n, s);
  const cudaError_t e =
      n > 0 ? bgtq::launch_encode(st->shape, st->ws, st->cache, layer, layer_count, k, v, d_start, d_count, batch, n, s)
            : cudaSuccess;
  if (e != cudaSuccess) return e;
  return bgtq::launch_rotate_query(st->shape, st->ws, layer, layer_count, q, batch, st->ws.qrot, s);
}

}  // namespace

extern "C" {

int bgtq_decode_step(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                     const int32_t* d_start, const int32_t* d_count, int32_t n, const void* d_q,
                     const int32_t* d_seq_lens, int32_t batch, void* d_out, void* stream) {
  if (!st || !d_q || !d_seq_lens || !d_out) return BGTQ_ERR_NULL;
  int v = check_step_appends(d_k, d_v, d_start, d_count, n);
  if (v != BGTQ_OK) return v;
  v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (!aligned16(d_q) || !aligned16(d_seq_lens) || !aligned16(d_out)) return BGTQ_ERR_ALIGNMENT;
  cudaStream_t s = as_stream(stream);
  if (use_fused(st)) {
    // the appends, then the fused decode (which rotates the query itself)
    if (n > 0 && bgtq::launch_encode(st->shape, st->ws, st->cache, layer, layer_count, static_cast<const __half*>(d_k),
                                     static_cast<const __half*>(d_v), d_start, d_count, batch, n, s) != cudaSuccess)
      return BGTQ_ERR_CUDA;
    return bgtq::launch_decode_fused(st->shape, st->ws, st->cache, layer, layer_count, static_cast<const __half*>(d_q),
                                     d_seq_lens, batch, fused_plan(st, layer_count, batch),
                                     static_cast<__half*>(d_out), s) == cudaSuccess
               ? BGTQ_OK
               : BGTQ_ERR_CUDA;
  }
  const bgtq::SplitPlan split = after_prep(split_for(st, layer_count, batch), d_start, d_count, n);
  if (queue_step_prep(st, layer, layer_count, static_cast<const __half*>(d_q), batch, d_k, d_v, d_start, d_count, n,
                      s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_decode_split(st->shape, st->ws, st->cache, layer, layer_count, nullptr, d_seq_lens,
                                bgtq::BufferArgs{}, batch, split, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_combine(st->shape, st->ws, layer, layer_count, d_seq_lens, batch, split, bgtq::BufferArgs{},
                           static_cast<__half*>(d_out), s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  return BGTQ_OK;
}

}  // extern "C"

namespace {

int decode_buffered_impl(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                         const int32_t* d_seq_lens, const int32_t* d_pos_lo, int32_t batch, const void* d_buf_k,
                         const void* d_buf_v, const int32_t* d_buf_count, int32_t n_buf, void* d_out, void* stream,
                         const void* d_k, const void* d_v, const int32_t* d_start, const int32_t* d_count,
                         int32_t n) {
  if (!st || !d_q || !d_seq_lens || !d_pos_lo || !d_buf_k || !d_buf_v || !d_buf_count || !d_out) return BGTQ_ERR_NULL;
  int v = check_step_appends(d_k, d_v, d_start, d_count, n);
  if (v != BGTQ_OK) return v;
  v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (n_buf < 1 || n_buf > bgtq::kMaxBufferRows) return BGTQ_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_seq_lens) || !aligned16(d_pos_lo) || !aligned16(d_buf_k) ||
      !aligned16(d_buf_v) || !aligned16(d_buf_count) || !aligned16(d_out))
    return BGTQ_ERR_ALIGNMENT;
  const bgtq::SplitPlan split = after_prep(split_for(st, layer_count, batch, 1), d_start, d_count, n);
  cudaStream_t s = as_stream(stream);
  bgtq::BufferArgs buf;
  buf.q = static_cast<const __half*>(d_q);
  buf.k = static_cast<const __half*>(d_buf_k);
  buf.v = static_cast<const __half*>(d_buf_v);
  buf.count = d_buf_count;
  buf.pos_lo = d_pos_lo;
  buf.n_buf = n_buf;
  if (queue_step_prep(st, layer, layer_count, buf.q, batch, d_k, d_v, d_start, d_count, n, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_decode_split(st->shape, st->ws, st->cache, layer, layer_count, nullptr, d_seq_lens, buf, batch,
                                split, s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_combine(st->shape, st->ws, layer, layer_count, d_seq_lens, batch, split, buf,
                           static_cast<__half*>(d_out), s) != cudaSuccess)
    return BGTQ_ERR_CUDA;
  return BGTQ_OK;
}

}  // namespace

extern "C" {

int bgtq_decode_attn_buffered(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                              const int32_t* d_seq_lens, const int32_t* d_pos_lo, int32_t batch, const void* d_buf_k,
                              const void* d_buf_v, const int32_t* d_buf_count, int32_t n_buf, void* d_out,
                              void* stream) {
  return decode_buffered_impl(st, layer, layer_count, d_q, d_seq_lens, d_pos_lo, batch, d_buf_k, d_buf_v, d_buf_count,
                              n_buf, d_out, stream, nullptr, nullptr, nullptr, nullptr, 0);
}

int bgtq_decode_step_buffered(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_k, const void* d_v,
                              const int32_t* d_start, const int32_t* d_count, int32_t n, const void* d_q,
                              const int32_t* d_seq_lens, const int32_t* d_pos_lo, int32_t batch,
                              const void* d_buf_k, const void* d_buf_v, const int32_t* d_buf_count, int32_t n_buf,
                              void* d_out, void* stream) {
  return decode_buffered_impl(st, layer, layer_count, d_q, d_seq_lens, d_pos_lo, batch, d_buf_k, d_buf_v, d_buf_count,
                              n_buf, d_out, stream, d_k, d_v, d_start, d_count, n);
}

int bgtq_logit_mae(bgtq_state* st, int32_t layer, int32_t layer_count, int32_t seq, int32_t w0, int32_t m,
                   const void* d_q, const void* d_k, double* d_mae, void* stream) {
  if (!st || !d_q || !d_k || !d_mae) return BGTQ_ERR_NULL;
  const int v = check_decode_args(st, layer, layer_count, 1);
  if (v != BGTQ_OK) return v;
  if (seq < 0 || seq >= st->cfg.max_batch || m < 1 || w0 < 0 || int64_t(w0) + m > st->cfg.capacity_tokens)
    return BGTQ_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_k) || !aligned16(d_mae)) return BGTQ_ERR_ALIGNMENT;
  return bgtq::launch_logit_mae(st->shape, st->ws, st->cache, layer, layer_count, seq, w0, m,
                                static_cast<const __half*>(d_q), static_cast<const __half*>(d_k), d_mae,
                                as_stream(stream)) == cudaSuccess
             ? BGTQ_OK
             : BGTQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Static-scratch decode: the split-K scratch lives in this library's own
// device array instead of the caller's workspace.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_static_scratch[BGTQ_STATIC_SCRATCH_BYTES];

// Bytes at the start of the static array for the arrival counters (the
// fused decode's; the split pass and combine leave them unused).
constexpr size_t kStaticCountBytes = 64 << 10;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_static_scratch for the current device (looked up once
// per device, with that device current).
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BGTQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BGTQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return BGTQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BGTQ_OK;
}

}  // namespace

int bgtq_decode_attn_static_scratch(bgtq_state* st, int32_t layer, int32_t layer_count, const void* d_q,
                                    const int32_t* d_seq_lens, int32_t batch, void* d_out, void* stream) {
  if (!st || !d_q || !d_seq_lens || !d_out) return BGTQ_ERR_NULL;
  const int v = check_decode_args(st, layer, layer_count, batch);
  if (v != BGTQ_OK) return v;
  if (!aligned16(d_q) || !aligned16(d_seq_lens) || !aligned16(d_out)) return BGTQ_ERR_ALIGNMENT;
  const size_t rows = size_t(layer_count) * st->cfg.max_batch * st->cfg.n_q_heads;
  if (use_fused(st)) {
    // the fused decode: the arrival counters, then one partial per cluster
    const bgtq::SplitPlan plan = fused_plan(st, layer_count, batch);
    const int64_t nclu = plan.c_max / plan.cluster;
    const size_t part_bytes = rows * size_t(nclu) * bgtq::kPartialStride * sizeof(float);
    if (rows * sizeof(uint32_t) > kStaticCountBytes || kStaticCountBytes + part_bytes > BGTQ_STATIC_SCRATCH_BYTES)
      return BGTQ_ERR_BUFFER_SIZE;
    void* base = nullptr;
    const int a = static_scratch_address(&base);
    if (a != BGTQ_OK) return a;
    bgtq::Workspace ws = st->ws;
    unsigned char* b8 = static_cast<unsigned char*>(base);
    ws.comb_count = reinterpret_cast<uint32_t*>(b8);
    ws.partials = reinterpret_cast<float*>(b8 + kStaticCountBytes);
    bgtq::Shape shape = st->shape;
    shape.max_splits = static_cast<int32_t>(nclu);
    return bgtq::launch_decode_fused(shape, ws, st->cache, layer, layer_count, static_cast<const __half*>(d_q),
                                     d_seq_lens, batch, plan, static_cast<__half*>(d_out), as_stream(stream)) ==
                   cudaSuccess
               ? BGTQ_OK
               : BGTQ_ERR_CUDA;
  }
  const bgtq::SplitPlan split = after_prep(split_for(st, layer_count, batch));
  const int64_t nspl = split.c_max;
  // the arrival counters' place first (as for the fused decode), then q~,
  // its fragments, the split partials and the combine's intermediates
  const size_t count_bytes = kStaticCountBytes;
  const size_t qrot_bytes = rows * kD * sizeof(float);
  const size_t fbytes = frag_bytes(&st->cfg, layer_count);
  const size_t part_bytes = rows * size_t(nspl) * bgtq::kPartialStride * sizeof(float);
  const size_t mid_bytes = rows * (bgtq::kCombSlices + 1) * bgtq::kPartialStride * sizeof(float);
  if (rows * sizeof(uint32_t) > count_bytes ||
      count_bytes + qrot_bytes + fbytes + part_bytes + mid_bytes > BGTQ_STATIC_SCRATCH_BYTES)
    return BGTQ_ERR_BUFFER_SIZE;
  void* base = nullptr;
  const int a = static_scratch_address(&base);
  if (a != BGTQ_OK) return a;
  // the same kernels as bgtq_decode_attn, with q~ and the partials redirected
  // to the static array (partials packed with n_splits as their stride)
  bgtq::Workspace ws = st->ws;
  unsigned char* b8 = static_cast<unsigned char*>(base);
  ws.comb_count = reinterpret_cast<uint32_t*>(b8);
  ws.qrot = reinterpret_cast<float*>(b8 + count_bytes);
  ws.qfrag = reinterpret_cast<uint4*>(b8 + count_bytes + qrot_bytes);
  ws.partials = reinterpret_cast<float*>(b8 + count_bytes + qrot_bytes + fbytes);
  ws.comb_mid = reinterpret_cast<float*>(b8 + count_bytes + qrot_bytes + fbytes + part_bytes);
  bgtq::Shape shape = st->shape;
  shape.max_splits = static_cast<int32_t>(nspl);
  cudaStream_t s = as_stream(stream);
  if (bgtq::launch_rotate_query(shape, ws, layer, layer_count, static_cast<const __half*>(d_q), batch, ws.qrot, s) !=
      cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_decode_split(shape, ws, st->cache, layer, layer_count, nullptr, d_seq_lens, bgtq::BufferArgs{}, batch, split, s) !=
      cudaSuccess)
    return BGTQ_ERR_CUDA;
  if (bgtq::launch_combine(shape, ws, layer, layer_count, d_seq_lens, batch, split, bgtq::BufferArgs{},
                           static_cast<__half*>(d_out), s) !=
      cudaSuccess)
    return BGTQ_ERR_CUDA;
  return BGTQ_OK;
}

int bgtq_set_block_table(bgtq_state* st, const int32_t* d_block_table) {
  if (!st) return BGTQ_ERR_NULL;
  if (st->cache.n_pages == 0) return BGTQ_ERR_INVALID_ARG;
  if (d_block_table && !aligned16(d_block_table)) return BGTQ_ERR_ALIGNMENT;
  st->cache.block_table = d_block_table;
  return BGTQ_OK;
}

int bgtq_test_drop_tile_copies(bgtq_state* st, int32_t tile) {
  if (!st) return BGTQ_ERR_NULL;
  if (tile < -1) return BGTQ_ERR_INVALID_ARG;
  st->shape.drop_tile = tile;
  return BGTQ_OK;
}

int bgtq_set_split_tokens(bgtq_state* st, int32_t tokens) {
  if (!st) return BGTQ_ERR_NULL;
  if (tokens < 0 || tokens % bgtq::kSplitGranule != 0) return BGTQ_ERR_INVALID_ARG;
  if (tokens > 0 && (st->cfg.capacity_tokens + tokens - 1) / tokens > max_splits_of(&st->cfg)) return BGTQ_ERR_INVALID_ARG;
  st->split_tokens = tokens;
  return BGTQ_OK;
}

int bgtq_set_decode_path(bgtq_state* st, int32_t fused) {
  if (!st) return BGTQ_ERR_NULL;
  if (fused != 0 && fused != 1) return BGTQ_ERR_INVALID_ARG;
  st->decode_mode = fused;
  return BGTQ_OK;
}

int bgtq_get_decode_path(bgtq_state* st, int32_t* h_fused, int32_t* h_ctas) {
  if (!st || !h_fused || !h_ctas) return BGTQ_ERR_NULL;
  if (const int dv = check_device(st)) return dv;
  const bool f = use_fused(st);
  *h_fused = f ? 1 : 0;
  *h_ctas = f ? fused_slots(st) : split_slots(st);
  return BGTQ_OK;
}

int bgtq_get_device_error(bgtq_state* st, void* stream, int32_t* h_flags) {
  if (!st || !h_flags) return BGTQ_ERR_NULL;
  if (const int dv = check_device(st)) return dv;
  cudaStream_t s = as_stream(stream);
  uint32_t flag = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, st->ws.err, sizeof(flag), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->ws.err, 0, sizeof(flag), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return BGTQ_ERR_CUDA;
  *h_flags = static_cast<int32_t>(flag);
  return BGTQ_OK;
}

const char* bgtq_error_string(int32_t status) {
  switch (status) {
    case BGTQ_OK: return "ok";
    case BGTQ_ERR_INVALID_ARG: return "invalid argument";
    case BGTQ_ERR_NULL: return "null pointer";
    case BGTQ_ERR_CUDA: return "CUDA runtime error";
    case BGTQ_ERR_BUFFER_SIZE: return "buffer too small";
    case BGTQ_ERR_NOT_READY: return "no allocation set";
    case BGTQ_ERR_DEVICE: return "device error flag raised";
    case BGTQ_ERR_HOST_ALLOC: return "host allocation failed";
    case BGTQ_ERR_ALIGNMENT: return "misaligned pointer";
    default: return "unknown status";
  }
}

}  // extern "C"

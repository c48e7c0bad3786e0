// Host side of the C ABI: argument checks, context lifetime, dispatch.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <stdlib.h>

#include <new>
#include <vector>

#include "internal.cuh"

using namespace starkv;

namespace {

thread_local char g_err[512] = "";

// Bounds that keep every size product of the checks and launches in range.
constexpr int kMaxHeads = 1024;
constexpr int kMaxHidden = 1 << 16;

starkv_status fail(starkv_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

starkv_status ok() {
  g_err[0] = 0;
  return STARKV_OK;
}

starkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(STARKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int gcd_int(int a, int b) {
  while (b) {
    int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Channel split of an r-channel latent: n_top = floor(top_fraction * r + 0.5),
// g = gcd(16, n_top, r - n_top).
bool make_geom(int r, double frac, bool fp16, LatentGeom* L) {
  if (fp16) {
    if (r % 16 != 0) return false;
    L->r = r;
    L->n_top = 0;
    L->g = 16;
    L->groups = r / 16;
    L->top_groups = 0;
    L->payload_bytes = 32 * r;
    L->region_bytes = 32 * r;
    L->fp16 = 1;
    return true;
  }
  L->fp16 = 0;
  const int n_top = (int)floor(frac * r + 0.5);
  const int n_bot = r - n_top;
  if (n_top < 0 || n_bot < 0) return false;
  const int g = gcd_int(16, gcd_int(n_top, n_bot));
  if (g != 4 && g != 8 && g != 16) return false;
  L->r = r;
  L->n_top = n_top;
  L->g = g;
  L->groups = r / g;
  L->top_groups = n_top / g;
  L->payload_bytes = 2 * (4 * n_top + 3 * n_bot);
  L->region_bytes = (L->payload_bytes + 15) / 16 * 16;
  return true;
}

starkv_status check_config(const starkv_config* c, LatentGeom* key, LatentGeom* val) {
  if (!c) return fail(STARKV_ERR_INVALID_ARG, "config is NULL");
  if (c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0 || c->hidden <= 0 ||
      c->rank_k <= 0 || c->rank_v <= 0 || c->max_position <= 0)
    return fail(STARKV_ERR_INVALID_ARG, "config sizes must be positive");
  if (c->flags != 0 && c->flags != STARKV_FLAG_FP16_LATENT)
    return fail(STARKV_ERR_INVALID_ARG, "config.flags must be 0 or STARKV_FLAG_FP16_LATENT");
  if (c->num_q_heads > kMaxHeads || c->num_kv_heads > kMaxHeads || c->hidden > kMaxHidden)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "num_q_heads, num_kv_heads <= %d and hidden <= %d", kMaxHeads,
                kMaxHidden);
  if (!(c->top_fraction >= 0.0 && c->top_fraction <= 1.0))
    return fail(STARKV_ERR_INVALID_ARG, "top_fraction must lie in [0, 1]");
  if (!(c->rope_base > 1.0)) return fail(STARKV_ERR_INVALID_ARG, "rope_base must exceed 1");
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "head_dim %d: only 64 and 128 are supported", c->head_dim);
  if (c->num_q_heads % c->num_kv_heads != 0)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "num_q_heads %% num_kv_heads != 0");
  if (c->rank_k > c->head_dim || c->rank_k % 16 != 0 || c->rank_k > 64)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "rank_k %d: need a multiple of 16, <= head_dim and <= 64", c->rank_k);
  if (c->rank_v > c->num_kv_heads * c->head_dim || c->rank_v % 16 != 0 || c->rank_v > 1024)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "rank_v %d: need a multiple of 16, <= h_kv*head_dim and <= 1024", c->rank_v);
  if (c->hidden % 64 != 0) return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "hidden %% 64 != 0");
  if (c->max_position > (1 << 24)) return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "max_position too large");
  LatentGeom k, v;
  const bool fp16 = c->flags == STARKV_FLAG_FP16_LATENT;
  if (!make_geom(c->rank_k, c->top_fraction, fp16, &k))
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "key latent: group size gcd(16, n_top, n_bot) must be 4, 8 or 16");
  if (!make_geom(c->rank_v, c->top_fraction, fp16, &v))
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "value latent: group size gcd(16, n_top, n_bot) must be 4, 8 or 16");
  if (c->key_ranks) {
    int widest = 0;
    for (int h = 0; h < c->num_kv_heads; ++h) {
      const int r = c->key_ranks[h];
      LatentGeom kh;
      if (r < 16 || r > c->rank_k || r % 16 != 0)
        return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "key_ranks[%d] = %d: need a multiple of 16 in [16, rank_k = %d]", h,
                    r, c->rank_k);
      if (!make_geom(r, c->top_fraction, fp16, &kh))
        return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "key_ranks[%d] = %d: group size must be 4, 8 or 16", h, r);
      widest = r > widest ? r : widest;
    }
    if (widest != c->rank_k)
      return fail(STARKV_ERR_INVALID_ARG, "rank_k (%d) must equal the largest of key_ranks (%d)", c->rank_k, widest);
  }
  if (key) *key = k;
  if (val) *val = v;
  return STARKV_OK;
}

// Per-head key geometry and page offsets (uniform ranks: every head is `uniform`).
// heads: host [h_kv]; returns the page strides (code bytes, meta words) and the key columns.
void build_key_heads(const starkv_config* c, const LatentGeom& uniform, KeyHead* heads, int* page_bytes,
                     int* page_meta, int* cols) {
  const bool fp16 = c->flags == STARKV_FLAG_FP16_LATENT;
  int col = 0, code = 0, meta = 0;
  for (int h = 0; h < c->num_kv_heads; ++h) {
    LatentGeom L = uniform;
    if (c->key_ranks) make_geom(c->key_ranks[h], c->top_fraction, fp16, &L);
    if (heads) heads[h] = KeyHead{L, col, code, meta};
    col += L.r;
    code += L.region_bytes;
    meta += L.fp16 ? 0 : L.groups * kPage;
  }
  *page_bytes = code;
  *page_meta = meta;
  *cols = col;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Geometry of a latent kind of the quantise / dequantise entries.
const LatentGeom* latent_of(const Ctx* c, int which) {
  if (which == STARKV_LATENT_VALUE) return &c->val;
  if (which == STARKV_LATENT_KEY) return &c->khead_host[0].L;
  if (which >= 2 && which - 2 < c->cfg.num_kv_heads) return &c->khead_host[which - 2].L;
  return nullptr;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// TMA map of the fp16 cos/sin table [max_position][d]: 64-column x 128-row boxes,
// 128-byte swizzle (the tensor-core operand layout), zero fill past the last row.
bool make_trig_map(Ctx* c) {
  const int d = c->cfg.head_dim;
  return starkv::encode_map_2d(&c->trig_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c->trig, (uint64_t)d,
                               (uint64_t)c->cfg.max_position, (uint64_t)d * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
}

starkv_status check_cache(const Ctx* c, const starkv_cache* cache) {
  if (!cache) return fail(STARKV_ERR_INVALID_ARG, "cache is NULL");
  if (cache->n_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "cache.n_pages < 0");
  const bool meta = !c->key.fp16;  // fp16 latents carry no metadata
  if (cache->n_pages > 0 && (!cache->k_codes || !cache->v_codes || (meta && (!cache->k_meta || !cache->v_meta))))
    return fail(STARKV_ERR_INVALID_ARG, "cache pool pointer is NULL");
  if (!aligned16(cache->k_codes) || !aligned16(cache->v_codes) || !aligned16(cache->k_meta) ||
      !aligned16(cache->v_meta))
    return fail(STARKV_ERR_INVALID_ARG, "cache pools must be 16-byte aligned");
  return STARKV_OK;
}

struct DecodeOutWs {
  size_t decode, o, zpart, total;
};

DecodeOutWs decode_out_ws(const Ctx& c, int batch, int max_pages) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  DecodeOutWs w;
  w.decode = al(plan_decode(c, batch, max_pages).ws_bytes);
  w.o = al((size_t)batch * c.cfg.num_q_heads * c.cfg.head_dim * 2);
  w.zpart = al((size_t)(c.wo_splits > 0 ? c.wo_splits : 1) * kSmallAppend * (c.model_dim > 0 ? c.model_dim : 1) * 4);
  w.total = w.decode + w.o + w.zpart;
  return w;
}

}  // namespace

namespace starkv {
bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType type, void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess || !f ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = (EncodeTiledFn)f;
  }
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(map, type, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace starkv

extern "C" {

const char* starkv_version(void) { return "starkv-b200 0.1 (sm_100a)"; }

const char* starkv_last_error(void) { return g_err; }

starkv_status starkv_cache_layout(const starkv_config* cfg, int64_t n_pages, starkv_cache_sizes* out) {
  LatentGeom k, v;
  starkv_status st = check_config(cfg, &k, &v);
  if (st) return st;
  if (!out) return fail(STARKV_ERR_INVALID_ARG, "out is NULL");
  if (n_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "n_pages < 0");
  out->key_region_bytes = k.region_bytes;
  out->value_region_bytes = v.region_bytes;
  out->key_group_size = k.g;
  out->value_group_size = v.g;
  out->key_top = k.n_top;
  out->value_top = v.n_top;
  out->key_groups = k.groups;
  out->value_groups = v.groups;
  int kpage = 0, kmeta = 0, kcols = 0;
  build_key_heads(cfg, k, nullptr, &kpage, &kmeta, &kcols);
  out->key_page_bytes = kpage;
  out->key_page_meta_bytes = kmeta * 4;
  out->k_codes_bytes = n_pages * (int64_t)kpage;
  out->v_codes_bytes = n_pages * (int64_t)v.region_bytes;
  out->k_meta_bytes = n_pages * (int64_t)kmeta * 4;
  out->v_meta_bytes = v.fp16 ? 0 : n_pages * (int64_t)v.groups * kPage * 4;
  return ok();
}

starkv_status starkv_create(const starkv_config* cfg, const void* A_k, const void* A_v, const void* B_k,
                            const void* B_v, starkv_stream_t stream, starkv_ctx** out) {
  LatentGeom k, v;
  starkv_status st = check_config(cfg, &k, &v);
  if (st) return st;
  if (!out) return fail(STARKV_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!A_k || !A_v || !B_k || !B_v) return fail(STARKV_ERR_INVALID_ARG, "factor pointer is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  Ctx* c = new (std::nothrow) Ctx();
  if (!c) return fail(STARKV_ERR_CUDA, "out of host memory");
  c->cfg = *cfg;
  c->key = k;
  c->val = v;
  c->group = cfg->num_q_heads / cfg->num_kv_heads;
  c->khead_host = new (std::nothrow) KeyHead[cfg->num_kv_heads];
  c->key_ranks = cfg->key_ranks ? new (std::nothrow) int32_t[cfg->num_kv_heads] : nullptr;
  if (!c->khead_host || (cfg->key_ranks && !c->key_ranks)) {
    delete[] c->khead_host;
    delete[] c->key_ranks;
    delete c;
    return fail(STARKV_ERR_CUDA, "out of host memory");
  }
  build_key_heads(cfg, k, c->khead_host, &c->kpage_bytes, &c->kpage_meta, &c->key_cols);
  c->ragged = false;
  if (cfg->key_ranks) {
    for (int h = 0; h < cfg->num_kv_heads; ++h) {
      c->key_ranks[h] = cfg->key_ranks[h];
      c->ragged = c->ragged || cfg->key_ranks[h] != cfg->rank_k;
    }
    c->cfg.key_ranks = c->key_ranks;  // the context's own copy
  }
  c->lat_cols = c->key_cols + cfg->rank_v;
  cudaGetDevice(&c->device);
  const int d = cfg->head_dim, half = d / 2;
  const size_t a_bytes = (size_t)cfg->hidden * c->lat_cols * 2;
  const size_t bk_bytes = (size_t)c->key_cols * d * 4;
  const size_t bv_bytes = (size_t)cfg->rank_v * cfg->num_kv_heads * d * 4;
  const size_t rope_bytes = (size_t)cfg->max_position * half * sizeof(float2);
  const size_t trig_bytes = (size_t)cfg->max_position * d * sizeof(__half);
  cudaError_t e;
  auto cleanup = [&]() {
    cudaFree(c->A);
    cudaFree(c->Bk);
    cudaFree(c->Bv);
    cudaFree(c->rope);
    cudaFree(c->trig);
    cudaFree(c->Bv16);
    cudaFree(c->zpart);
    cudaFree(c->status);
    cudaFree(c->Bk16);
    cudaFree(c->Bv16p);
    cudaFree(c->Wo);
    cudaFree(c->khead);
    delete[] c->khead_host;
    delete[] c->key_ranks;
    delete c;
  };
  // small appends: K splits of the projection so that about every SM streams a
  // slice of A (slices of 64..512 rows, 128 output columns per CTA)
  {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device);
    const int col_blocks = (c->lat_cols + 127) / 128;
    c->app_splits = 0;
    if (cfg->hidden % 64 == 0 && c->lat_cols % 8 == 0) {
      for (int kl = 512; kl >= 64; kl >>= 1) {
        if (cfg->hidden % kl != 0) continue;
        if (cfg->hidden / kl > 16) break;  // the quantiser adds at most 16 split sums
        c->app_splits = cfg->hidden / kl;
        if ((int64_t)c->app_splits * col_blocks * 4 >= (int64_t)sms * 3) break;
      }
    }
  }
  if ((e = cudaMalloc(&c->A, a_bytes)) != cudaSuccess || (e = cudaMalloc(&c->Bk, bk_bytes)) != cudaSuccess ||
      (e = cudaMalloc(&c->Bv, bv_bytes)) != cudaSuccess || (e = cudaMalloc(&c->rope, rope_bytes)) != cudaSuccess ||
      (e = cudaMalloc(&c->trig, trig_bytes)) != cudaSuccess || (e = cudaMalloc(&c->Bv16, bv_bytes / 2)) != cudaSuccess ||
      (e = cudaMalloc(&c->zpart, (size_t)(c->app_splits > 0 ? c->app_splits : 1) * kSmallAppend * c->lat_cols * 4)) !=
          cudaSuccess ||
      (e = cudaMalloc(&c->status, sizeof(unsigned int))) != cudaSuccess ||
      (e = cudaMalloc(&c->Bk16, bk_bytes / 2)) != cudaSuccess || (e = cudaMalloc(&c->Bv16p, bv_bytes / 2)) != cudaSuccess ||
      (e = cudaMalloc(&c->khead, (size_t)cfg->num_kv_heads * sizeof(KeyHead))) != cudaSuccess) {
    cleanup();
    return cuda_fail(e, "cudaMalloc (context factors)");
  }
  // A = [A_k | A_v], row-major [hidden][lat_cols]
  const size_t kcols = (size_t)c->key_cols;
  e = cudaMemcpyAsync(c->khead, c->khead_host, (size_t)cfg->num_kv_heads * sizeof(KeyHead), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) {
    cleanup();
    return cuda_fail(e, "starkv_create");
  }
  e = cudaMemcpy2DAsync(c->A, c->lat_cols * 2, A_k, kcols * 2, kcols * 2, cfg->hidden, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync((char*)c->A + kcols * 2, c->lat_cols * 2, A_v, (size_t)cfg->rank_v * 2,
                          (size_t)cfg->rank_v * 2, cfg->hidden, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = launch_prepare_factors(*c, (const __nv_bfloat16*)B_k, (const __nv_bfloat16*)B_v, s);
  if (e == cudaSuccess) e = launch_prepare_tc_factors(*c, s);
  if (e == cudaSuccess) e = launch_prepare_prefill_factors(*c, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->status, 0, sizeof(unsigned int), s);
  // RoPE table: angle p * base^(-2i/d) in fp64, cos/sin in fp64, stored as fp32
  // and the same angles as an fp16 [cos.. | sin..] row per position (tensor-core operand)
  std::vector<float2> rope;
  std::vector<__half> trig;
  std::vector<double> theta;
  try {
    rope.resize((size_t)cfg->max_position * half);
    trig.resize((size_t)cfg->max_position * d);
    theta.resize(half);
  } catch (const std::bad_alloc&) {
    if (e == cudaSuccess) cudaStreamSynchronize(s);
    cleanup();
    return fail(STARKV_ERR_CUDA, "out of host memory for the RoPE tables of %d positions", cfg->max_position);
  }
  for (int i = 0; i < half; ++i) theta[i] = pow(cfg->rope_base, -2.0 * i / d);
  for (int p = 0; p < cfg->max_position; ++p)
    for (int i = 0; i < half; ++i) {
      const double ang = (double)p * theta[i];
      const double cv = cos(ang), sv = sin(ang);
      rope[(size_t)p * half + i] = make_float2((float)cv, (float)sv);
      trig[(size_t)p * d + i] = __float2half_rn((float)cv);
      trig[(size_t)p * d + half + i] = __float2half_rn((float)sv);
    }
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->rope, rope.data(), rope_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->trig, trig.data(), trig_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cleanup();
    return cuda_fail(e, "starkv_create");
  }
  const char* path = getenv("STARKV_DECODE_PATH");
  const bool want_simt = path && strcmp(path, "simt") == 0;
  c->tc = !want_simt && !c->ragged && tc_decode_supported(c->cfg) && c->val.g == 16 && make_trig_map(c);
  const char* ppath = getenv("STARKV_PREFILL_PATH");
  const bool want_simt_prefill = ppath && strcmp(ppath, "simt") == 0;
  c->tc_prefill = !want_simt_prefill && !c->ragged && tc_prefill_supported(*c) && make_prefill_maps(c);
  if (c->app_splits > 0) {
    const int kl = cfg->hidden / c->app_splits;
    if (!starkv::encode_map_2d(&c->a_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->A, (uint64_t)c->lat_cols,
                               (uint64_t)cfg->hidden, (uint64_t)c->lat_cols * 2, 64, kl < 256 ? kl : 256,
                               CU_TENSOR_MAP_SWIZZLE_128B))
      c->app_splits = 0;  // the general append kernel serves every size
  }
  const char* apath = getenv("STARKV_APPEND_PATH");
  const bool want_simt_append = apath && strcmp(apath, "simt") == 0;
  c->tc_append = !want_simt_append && tc_append_supported(*c) &&
                 starkv::encode_map_2d(&c->a_map64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->A, (uint64_t)c->lat_cols,
                                       (uint64_t)cfg->hidden, (uint64_t)c->lat_cols * 2, 64, 64,
                                       CU_TENSOR_MAP_SWIZZLE_128B);
  *out = reinterpret_cast<starkv_ctx*>(c);
  return ok();
}

starkv_status starkv_destroy(starkv_ctx* ctx) {
  if (!ctx) return ok();
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  cudaDeviceSynchronize();
  cudaFree(c->A);
  cudaFree(c->Bk);
  cudaFree(c->Bv);
  cudaFree(c->rope);
  cudaFree(c->trig);
  cudaFree(c->Bv16);
  cudaFree(c->zpart);
  cudaFree(c->status);
  cudaFree(c->Bk16);
  cudaFree(c->Bv16p);
  cudaFree(c->Wo);
  cudaFree(c->khead);
  delete[] c->khead_host;
  delete[] c->key_ranks;
  delete c;
  return ok();
}

starkv_status starkv_set_output_projection(starkv_ctx* ctx, const void* W_o, int32_t model_dim,
                                           starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  if (!W_o) return fail(STARKV_ERR_INVALID_ARG, "W_o is NULL");
  if (model_dim <= 0 || model_dim % 8 != 0 || model_dim > (1 << 16))
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "model_dim %d: need a positive multiple of 8, <= 65536", model_dim);
  const int K = c->cfg.num_q_heads * c->cfg.head_dim;
  // K splits so that about every SM streams a slice of W_o (slices of 64..512 rows)
  int splits = 0;
  {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, c->device);
    const int col_blocks = (model_dim + 127) / 128;
    for (int kl = 512; kl >= 64; kl >>= 1) {
      if (K % kl != 0) continue;
      if (K / kl > 64) break;
      splits = K / kl;
      if ((int64_t)splits * col_blocks * 4 >= (int64_t)sms * 3) break;
    }
  }
  if (splits == 0) return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "num_q_heads*head_dim must be a multiple of 64");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = (size_t)K * model_dim * 2;
  __nv_bfloat16* w = nullptr;
  cudaError_t e = cudaMalloc(&w, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc (output projection)");
  e = cudaMemcpyAsync(w, W_o, bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaFree(w);
    return cuda_fail(e, "starkv_set_output_projection");
  }
  const int kl = K / splits;
  CUtensorMap map;
  if (!starkv::encode_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, (uint64_t)model_dim, (uint64_t)K,
                             (uint64_t)model_dim * 2, 64, kl < 256 ? kl : 256, CU_TENSOR_MAP_SWIZZLE_128B)) {
    cudaFree(w);
    return fail(STARKV_ERR_CUDA, "tensor map of the output projection");
  }
  cudaFree(c->Wo);
  c->Wo = w;
  c->model_dim = model_dim;
  c->wo_splits = splits;
  c->wo_map = map;
  return ok();
}

starkv_status starkv_get_config(const starkv_ctx* ctx, starkv_config* out) {
  if (!ctx || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  *out = reinterpret_cast<const Ctx*>(ctx)->cfg;
  return ok();
}

starkv_status starkv_append(starkv_ctx* ctx, const starkv_cache* cache, const void* X, const int64_t* slot_mapping,
                            int64_t n, float* latents_out, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (n < 0) return fail(STARKV_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && (!X || !slot_mapping)) return fail(STARKV_ERR_INVALID_ARG, "X or slot_mapping is NULL");
  if (n > 0 && cache->n_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "cache has no pages");
  cudaError_t e = launch_append(*c, *cache, (const __nv_bfloat16*)X, slot_mapping, n, latents_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return ok();
}

starkv_status starkv_workspace_bytes(const starkv_ctx* ctx, int32_t op, int32_t batch, int32_t max_pages,
                                     int64_t total_q, size_t* out) {
  if (!ctx || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  if (batch < 0 || max_pages < 0 || total_q < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  const Ctx* c = reinterpret_cast<const Ctx*>(ctx);
  if (op == STARKV_OP_DECODE) {
    *out = plan_decode(*c, batch, max_pages).ws_bytes;
  } else if (op == STARKV_OP_DECODE_OUT) {
    if (c->model_dim <= 0) return fail(STARKV_ERR_INVALID_ARG, "no output projection set");
    *out = decode_out_ws(*c, batch, max_pages).total;
  } else if (op == STARKV_OP_PREFILL) {
    *out = plan_prefill(*c, batch, max_pages, total_q).ws_bytes;
  } else {
    return fail(STARKV_ERR_INVALID_ARG, "unknown op %d", op);
  }
  return ok();
}

starkv_status starkv_decode_attn(starkv_ctx* ctx, const starkv_cache* cache, const void* q, const int32_t* block_table,
                                 const int32_t* seq_lens, int32_t batch, int32_t max_pages, void* out,
                                 void* workspace, size_t workspace_bytes, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (batch < 0 || max_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return ok();
  if (max_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "max_pages must be >= 1");
  if (!q || !block_table || !seq_lens || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  const DecodePlan plan = plan_decode(*c, batch, max_pages);
  if (!workspace || workspace_bytes < plan.ws_bytes)
    return fail(STARKV_ERR_WORKSPACE_TOO_SMALL, "decode needs %zu workspace bytes, got %zu", plan.ws_bytes,
                workspace ? workspace_bytes : (size_t)0);
  if (((uintptr_t)workspace & 255) != 0) return fail(STARKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = launch_decode(*c, *cache, (const __nv_bfloat16*)q, block_table, seq_lens, batch, max_pages,
                                (__nv_bfloat16*)out, workspace, plan, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

starkv_status starkv_decode_attn_out(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                     const int32_t* block_table, const int32_t* seq_lens, int32_t batch,
                                     int32_t max_pages, void* y, void* workspace, size_t workspace_bytes,
                                     starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (c->model_dim <= 0) return fail(STARKV_ERR_INVALID_ARG, "no output projection set (starkv_set_output_projection)");
  if (batch < 0 || max_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return ok();
  if (max_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "max_pages must be >= 1");
  if (!q || !block_table || !seq_lens || !y) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  const DecodeOutWs w = decode_out_ws(*c, batch, max_pages);
  if (!workspace || workspace_bytes < w.total)
    return fail(STARKV_ERR_WORKSPACE_TOO_SMALL, "decode with output projection needs %zu workspace bytes, got %zu",
                w.total, workspace ? workspace_bytes : (size_t)0);
  if (((uintptr_t)workspace & 255) != 0) return fail(STARKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  char* base = (char*)workspace;
  __nv_bfloat16* o = (__nv_bfloat16*)(base + w.decode);
  float* zpart = (float*)(base + w.decode + w.o);
  const DecodePlan plan = plan_decode(*c, batch, max_pages);
  cudaError_t e = launch_decode(*c, *cache, (const __nv_bfloat16*)q, block_table, seq_lens, batch, max_pages, o,
                                workspace, plan, (cudaStream_t)stream);
  if (e == cudaSuccess) e = launch_outproj(*c, o, batch, (__nv_bfloat16*)y, zpart, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode with output projection");
  return ok();
}

starkv_status starkv_decode_attn_noalloc(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                         const int32_t* block_table, const int32_t* seq_lens, int32_t batch,
                                         int32_t max_pages, void* out, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (batch < 0 || max_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return ok();
  if (max_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "max_pages must be >= 1");
  if (!q || !block_table || !seq_lens || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  const DecodePlan plan = plan_decode(*c, batch, max_pages);
  if (plan.ws_bytes > kNoAllocScratchBytes)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE,
                "decode of %d sequences x %d pages needs %zu scratch bytes; the built-in scratch holds %zu "
                "(use starkv_decode_attn with a caller workspace)",
                batch, max_pages, plan.ws_bytes, kNoAllocScratchBytes);
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "built-in scratch lookup (cudaGetSymbolAddress)");
  e = launch_decode(*c, *cache, (const __nv_bfloat16*)q, block_table, seq_lens, batch, max_pages,
                    (__nv_bfloat16*)out, scratch, plan, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

starkv_status starkv_decode_attn_slice(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                       const int32_t* block_table, const int32_t* seq_lens, const int32_t* key_pos0,
                                       const int32_t* q_pos, int32_t batch, int32_t max_pages, float* out_o,
                                       float* out_ml, void* workspace, size_t workspace_bytes,
                                       starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (batch < 0 || max_pages < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (batch == 0) return ok();
  if (max_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "max_pages must be >= 1");
  if (!q || !block_table || !seq_lens || !key_pos0 || !q_pos || !out_o || !out_ml)
    return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  if (((uintptr_t)out_o & 15) != 0 || ((uintptr_t)out_ml & 7) != 0)
    return fail(STARKV_ERR_INVALID_ARG, "out_o must be 16-byte and out_ml 8-byte aligned");
  if (!c->tc)
    return fail(STARKV_ERR_UNSUPPORTED_SHAPE, "slice decode needs the tensor-core decode path for this shape");
  const DecodePlan plan = plan_decode(*c, batch, max_pages);
  if (!workspace || workspace_bytes < plan.ws_bytes)
    return fail(STARKV_ERR_WORKSPACE_TOO_SMALL, "decode needs %zu workspace bytes, got %zu", plan.ws_bytes,
                workspace ? workspace_bytes : (size_t)0);
  if (((uintptr_t)workspace & 255) != 0) return fail(STARKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const DecodeSlice slice{key_pos0, q_pos, out_o, out_ml};
  cudaError_t e = launch_decode_tc(*c, *cache, (const __nv_bfloat16*)q, block_table, seq_lens, batch, max_pages,
                                   nullptr, workspace, plan, (cudaStream_t)stream, &slice);
  if (e != cudaSuccess) return cuda_fail(e, "slice decode launch");
  return ok();
}

starkv_status starkv_merge_slices(starkv_ctx* ctx, const float* o_parts, const float* ml_parts, int32_t n_parts,
                                  int32_t batch, void* out, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  if (n_parts < 0 || batch < 0) return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (n_parts == 0 || batch == 0) return ok();
  if (!o_parts || !ml_parts || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  if (((uintptr_t)o_parts & 15) != 0 || ((uintptr_t)ml_parts & 7) != 0 || ((uintptr_t)out & 7) != 0)
    return fail(STARKV_ERR_INVALID_ARG, "o_parts must be 16-byte, ml_parts and out 8-byte aligned");
  cudaError_t e = launch_merge_slices(o_parts, ml_parts, n_parts, (int64_t)batch * c->cfg.num_q_heads,
                                      c->cfg.head_dim, (__nv_bfloat16*)out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

starkv_status starkv_prefill_attn(starkv_ctx* ctx, const starkv_cache* cache, const void* q, const int32_t* cu_q,
                                  const int32_t* block_table, const int32_t* seq_lens, int32_t batch,
                                  int32_t max_pages, int64_t total_q, int32_t max_q_len, void* out,
                                  void* workspace, size_t workspace_bytes, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  starkv_status st = check_cache(c, cache);
  if (st) return st;
  if (batch < 0 || max_pages < 0 || total_q < 0 || max_q_len < 0)
    return fail(STARKV_ERR_INVALID_ARG, "negative size");
  if (batch == 0 || total_q == 0) return ok();
  if (max_pages == 0) return fail(STARKV_ERR_INVALID_ARG, "max_pages must be >= 1");
  if (max_q_len == 0 || max_q_len > max_pages * kPage)
    return fail(STARKV_ERR_INVALID_ARG, "max_q_len must lie in [1, max_pages*16]");
  if (!q || !cu_q || !block_table || !seq_lens || !out) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  const PrefillPlan plan = plan_prefill(*c, batch, max_pages, total_q);
  if (!workspace || workspace_bytes < plan.ws_bytes)
    return fail(STARKV_ERR_WORKSPACE_TOO_SMALL, "prefill needs %zu workspace bytes, got %zu", plan.ws_bytes,
                workspace ? workspace_bytes : (size_t)0);
  if (((uintptr_t)workspace & 255) != 0) return fail(STARKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = launch_prefill(*c, *cache, (const __nv_bfloat16*)q, cu_q, block_table, seq_lens, batch, max_pages,
                                 total_q, max_q_len, (__nv_bfloat16*)out, workspace, plan, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

starkv_status starkv_quantize_pack(starkv_ctx* ctx, int32_t which, const float* z, int64_t n, void* codes,
                                   void* meta, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  const LatentGeom* Lp = latent_of(c, which);
  if (!Lp) return fail(STARKV_ERR_INVALID_ARG, "bad latent kind %d", which);
  if (n < 0) return fail(STARKV_ERR_INVALID_ARG, "n < 0");
  const LatentGeom& L = *Lp;
  if (n > 0 && (!z || !codes || (!meta && !L.fp16))) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(codes) || !aligned16(meta)) return fail(STARKV_ERR_INVALID_ARG, "codes/meta must be 16-byte aligned");
  cudaError_t e = launch_quantize_pack(*c, L, z, n, (uint8_t*)codes, (uint32_t*)meta, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize_pack launch");
  return ok();
}

starkv_status starkv_dequantize(starkv_ctx* ctx, int32_t which, const void* codes, const void* meta, int64_t n,
                                float* z_out, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "ctx is NULL");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  const LatentGeom* Lp = latent_of(c, which);
  if (!Lp) return fail(STARKV_ERR_INVALID_ARG, "bad latent kind %d", which);
  if (n < 0) return fail(STARKV_ERR_INVALID_ARG, "n < 0");
  const LatentGeom& L = *Lp;
  if (n > 0 && (!z_out || !codes || (!meta && !L.fp16))) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  cudaError_t e = launch_dequantize(*c, L, (const uint8_t*)codes, (const uint32_t*)meta, n, z_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

starkv_status starkv_selftest_wait_timeout(starkv_ctx* ctx, uint64_t limit_ns, starkv_stream_t stream) {
  if (!ctx) return fail(STARKV_ERR_INVALID_ARG, "NULL context");
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return fail(STARKV_ERR_INVALID_ARG, "limit_ns out of range");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  cudaError_t e = starkv::launch_wait_timeout_selftest(c->status, limit_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

starkv_status starkv_read_device_status(starkv_ctx* ctx, starkv_stream_t stream, uint32_t* status) {
  if (!ctx || !status) return fail(STARKV_ERR_INVALID_ARG, "NULL argument");
  Ctx* c = reinterpret_cast<Ctx*>(ctx);
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, c->status, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(c->status, 0, sizeof(unsigned int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read_device_status");
  *status = h;
  if (h) return fail(STARKV_ERR_DEVICE_STATUS, "device status 0x%x", h);
  return ok();
}

}  // extern "C"

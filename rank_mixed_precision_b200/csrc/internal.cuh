// Internal definitions shared by the library's CUDA sources.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/starkv.h"

namespace starkv {

constexpr int kPage = STARKV_PAGE_TOKENS;

// Geometry of one latent (a KV head's key latent, or the joint value latent).
struct LatentGeom {
  int r;             // channels
  int n_top;         // leading 4-bit channels (0 for fp16 latents)
  int g;             // rotation / quantisation group size (4, 8 or 16; 16 for fp16 latents)
  int groups;        // r / g
  int top_groups;    // n_top / g
  int payload_bytes; // 2 * (4 n_top + 3 (r - n_top)) per page; 32 r for fp16 latents
  int region_bytes;  // payload rounded up to 16
  int fp16;          // 1: unquantised fp16 latents (tiles of 16 tokens x g channels, no metadata)
};

// Byte offset of group tile `gi` inside a page region.
__host__ __device__ inline int tile_offset(const LatentGeom& L, int gi) {
  if (L.fp16) return gi * 32 * L.g;
  return gi < L.top_groups ? gi * 8 * L.g : L.top_groups * 8 * L.g + (gi - L.top_groups) * 6 * L.g;
}

// One KV head's key latent: its geometry (its own rank r_k,h), its columns in
// the latent row (and rows of B'_k), and where its region sits in a page of the
// key pools.  Uniform ranks give col0 = h r_k, code_off = h region_bytes.
struct KeyHead {
  LatentGeom L;
  int col0;      // first latent column (and B'_k row) of the head
  int code_off;  // byte offset of the head's region within a page of the key-code pool
  int meta_off;  // 4-byte word offset of the head's metadata within a page of the key-meta pool
};

// Head whose key columns hold latent column col (col < total key columns).
__host__ __device__ inline int key_head_of(const KeyHead* kh, int h_kv, int col) {
  int lo = 0, hi = h_kv - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (kh[mid].col0 <= col) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

struct Ctx {
  starkv_config cfg;
  LatentGeom key, val;    // key: the geometry of every head at uniform ranks, of the widest head otherwise
  KeyHead* khead;         // device [h_kv]
  KeyHead* khead_host;    // host [h_kv]
  int32_t* key_ranks;     // host [h_kv] copy of the rank table (cfg.key_ranks points here), or NULL
  bool ragged;            // per-head key ranks differ
  int key_cols;           // sum over heads of r_k,h
  int kpage_bytes;        // key-code bytes of one page (all heads)
  int kpage_meta;         // key-meta words of one page (all heads)
  int group;              // H / h_kv
  int lat_cols;           // h_kv * r_k + R
  int device;
  // context-owned device memory
  __nv_bfloat16* A;       // [hidden][lat_cols] bf16: A_k | A_v side by side
  float* Bk;              // [h_kv][r_k][d_h]  fp32, B'_k = H B_k (rotation folded)
  float* Bv;              // [R][h_kv*d_h]     fp32, B'_v = H B_v
  float2* rope;           // [max_position][d_h/2] (cos, sin), built in fp64
  __half* trig;           // [max_position][d_h] fp16: cos(p th_0..), sin(p th_0..) (tensor-core operand)
  __half* Bv16;           // [R][h_kv*d_h] fp16, B'_v
  float* zpart;           // [app_splits][kSmallAppend][lat_cols] fp32 split-K sums of small appends
  int app_splits;         // K splits of the small-append projection (0: that path is off)
  CUtensorMap a_map;      // TMA map of `A`: box 64 columns x min(256, hidden / app_splits) rows, 128-byte swizzle
  unsigned int* status;   // device status word
  CUtensorMap trig_map;   // TMA map of `trig`: box 64 x 128, 128-byte swizzle
  bool tc;                // tensor-core decode available for this shape
  // tensor-core prefill operands
  __half* Bk16;           // [h_kv][r_k][d_h] fp16 B'_k
  __half* Bv16p;          // [R][h_kv*d_h] fp16 B'_v, rows of each 16-channel group in the order the
                          // value dequantiser emits them (value_channel_of_position)
  CUtensorMap bk_map;     // TMA map of Bk16 as [h_kv*r_k][d_h]: box 64 x r_k, 128-byte swizzle
  CUtensorMap bvp_map;    // TMA map of Bv16p: box 64 x 64, 128-byte swizzle
  bool tc_prefill;        // tensor-core prefill available for this shape
  CUtensorMap a_map64;    // TMA map of `A`: box 64 columns x 64 rows, 128-byte swizzle (tensor-core append)
  bool tc_append;         // tensor-core append (more than 64 tokens) available
  // output projection (set by starkv_set_output_projection; model_dim 0 = none)
  __nv_bfloat16* Wo;      // [H*d_h][model_dim] bf16
  int model_dim;
  int wo_splits;          // K splits of the output projection GEMM
  CUtensorMap wo_map;     // TMA map of Wo: box 64 columns x min(256, K / wo_splits) rows, 128-byte swizzle
};

// 2-D TMA map over a row-major [rows][inner] array (no interleave, zero fill).
bool encode_map_2d(CUtensorMap* map, CUtensorMapDataType type, void* base, uint64_t inner, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// Launch with programmatic stream serialisation (the kernel may start while the
// previous kernel on the stream finishes; it calls griddepcontrol.wait before
// reading that kernel's results) and an optional cluster size.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                           unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Appends of at most this many tokens use the split-K projection path.
constexpr int kSmallAppend = 64;

// Extra device status bit: a pipeline wait in a tensor-core kernel gave up.
constexpr unsigned int kDevWaitTimeout = STARKV_DEV_WAIT_TIMEOUT;

// One block waiting on a barrier that nothing completes (bounded; sets kDevWaitTimeout).
cudaError_t launch_wait_timeout_selftest(unsigned int* status, uint64_t limit_ns, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ inline void set_status(unsigned int* st, unsigned int bit) { atomicOr(st, bit); }

// fl32(1/sqrt(g)) written as decimal literals the compiler rounds correctly.
__device__ inline float inv_sqrt_group(int g) {
  switch (g) {
    case 4: return 0.5f;
    case 8: return 0.353553390593273762200422181052424519642f;
    case 16: return 0.25f;
    default: return 0.707106781186547524400844362104849039284f;  // g == 2
  }
}

// In-place z <- z H_g (normalised Sylvester Hadamard) with fp32 butterflies of
// half-width 1, 2, 4, ... followed by one multiply by fl32(1/sqrt g).
template <int G>
__device__ inline void fwht_fl32(float (&x)[G]) {
#pragma unroll
  for (int h = 1; h < G; h <<= 1) {
#pragma unroll
    for (int i = 0; i < G; ++i) {
      if ((i & h) == 0) {
        float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
  const float c = inv_sqrt_group(G);
#pragma unroll
  for (int i = 0; i < G; ++i) x[i] = __fmul_rn(x[i], c);
}

// Asymmetric min/max quantiser of one group: fp16 scale and zero (= min),
// round-half-even, clamp.  Returns false when the scale or zero is not finite
// (or an input is not finite); codes are then all zero.
template <int G>
__device__ inline bool quantize_group(const float (&x)[G], int bits, uint8_t (&code)[G],
                                      __half& s16, __half& zp16) {
  float mn = x[0], mx = x[0];
  bool finite = isfinite(x[0]);
#pragma unroll
  for (int i = 1; i < G; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
    finite = finite && isfinite(x[i]);
  }
  const float qmax = (float)((1 << bits) - 1);
  s16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), qmax));
  zp16 = __float2half_rn(mn);
  const float sf = __half2float(s16), zf = __half2float(zp16);
  if (!finite || !isfinite(sf) || !isfinite(zf)) {
#pragma unroll
    for (int i = 0; i < G; ++i) code[i] = 0;
    s16 = __float2half_rn(0.f);
    zp16 = __float2half_rn(0.f);
    return false;
  }
#pragma unroll
  for (int i = 0; i < G; ++i) {
    float q = 0.f;
    if (sf != 0.f) q = fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x[i], zf), sf)), 0.f), qmax);
    code[i] = (uint8_t)q;
  }
  return true;
}

// Write one token's codes of one group into its page tile.  The token's bits
// are cleared and set with 32-bit atomics, so tokens sharing a word (and a
// page being written by other threads) stay intact.  region: 4-byte aligned
// base of the page region; t: token offset in the page.
template <int G>
__device__ inline void store_group_codes(uint8_t* region, const LatentGeom& L, int gi, int t,
                                         const uint8_t (&code)[G]) {
  uint32_t* tile = reinterpret_cast<uint32_t*>(region + tile_offset(L, gi));
  if (gi < L.top_groups) {
    // 4-bit: nibble index i = t*G + c, nibble (i % 8) of word i / 8
#pragma unroll
    for (int c0 = 0; c0 < G; c0 += (G < 8 ? G : 8)) {
      const int i0 = t * G + c0;
      const int w = i0 >> 3, sh = (i0 & 7) * 4;
      const int cnt = G < 8 ? G : 8;
      uint32_t bits = 0, mask = 0;
#pragma unroll
      for (int c = 0; c < cnt; ++c) {
        bits |= (uint32_t)(code[c0 + c] & 0xF) << (4 * c);
        mask |= 0xFu << (4 * c);
      }
      atomicAnd(&tile[w], ~(mask << sh));
      atomicOr(&tile[w], bits << sh);
    }
  } else {
    // 2-bit plane (4G bytes) then 1-bit plane (2G bytes)
    uint32_t* plane2 = tile;
    uint32_t* plane1 = tile + G;  // 4G bytes = G words
#pragma unroll
    for (int c0 = 0; c0 < G; c0 += (G < 16 ? G : 16)) {
      const int cnt = G < 16 ? G : 16;
      const int i0 = t * G + c0;
      const int w = i0 >> 4, sh = (i0 & 15) * 2;
      uint32_t bits = 0, mask = 0;
#pragma unroll
      for (int c = 0; c < cnt; ++c) {
        bits |= (uint32_t)(code[c0 + c] & 3) << (2 * c);
        mask |= 3u << (2 * c);
      }
      atomicAnd(&plane2[w], ~(mask << sh));
      atomicOr(&plane2[w], bits << sh);
    }
    {
      const int i0 = t * G;
      const int w = i0 >> 5, sh = i0 & 31;
      uint32_t bits = 0, mask = 0;
#pragma unroll
      for (int c = 0; c < G; ++c) {
        bits |= (uint32_t)((code[c] >> 2) & 1) << c;
        mask |= 1u << c;
      }
      atomicAnd(&plane1[w], ~(mask << sh));
      atomicOr(&plane1[w], bits << sh);
    }
  }
}

// Code of element (t, c) of group gi of a page region (generic, unoptimised).
__device__ inline int load_code(const uint8_t* region, const LatentGeom& L, int gi, int t, int c) {
  const uint8_t* tile = region + tile_offset(L, gi);
  const int i = t * L.g + c;
  if (gi < L.top_groups) {
    const uint8_t b = tile[i >> 1];
    return (i & 1) ? (b >> 4) : (b & 0xF);
  }
  const uint8_t b2 = tile[i >> 2];
  const uint8_t b1 = tile[4 * L.g + (i >> 3)];
  return ((b2 >> (2 * (i & 3))) & 3) | (((b1 >> (i & 7)) & 1) << 2);
}

__device__ inline float2 unpack_meta(uint32_t m) {
  __half_raw s, z;
  s.x = (unsigned short)(m & 0xFFFF);
  z.x = (unsigned short)(m >> 16);
  return make_float2(__half2float(__half(s)), __half2float(__half(z)));
}

// Stored value of element (t, c) of group gi of a page region, rotated domain:
// code * s + zp (fp32, exact product) for quantised latents, the fp16 value for
// unquantised ones.  meta_page: the region's [groups][16] metadata (unused for fp16).
__device__ inline float latent_value(const uint8_t* region, const uint32_t* meta_page, const LatentGeom& L, int gi,
                                     int t, int c) {
  if (L.fp16) return __half2float(reinterpret_cast<const __half*>(region + tile_offset(L, gi))[t * L.g + c]);
  const float2 sz = unpack_meta(meta_page[gi * kPage + t]);
  return __fmaf_rn((float)load_code(region, L, gi, t, c), sz.x, sz.y);
}

// ---------------------------------------------------------------------------
// Rotate + quantise + store one group of one token (shared by append and the
// quantise entry).  x: the group's g pre-rotation latents.
// ---------------------------------------------------------------------------
template <int G>
__device__ inline void rotate_quantize_store(const float* x_in, const LatentGeom& L, int gi,
                                             uint8_t* region, uint32_t* meta_page, int t,
                                             unsigned int* status) {
  float x[G];
#pragma unroll
  for (int i = 0; i < G; ++i) x[i] = x_in[i];
  fwht_fl32<G>(x);
  if (L.fp16) {
    // unquantised latent: fl16 of the rotated values, row t of the group's tile
    uint32_t h[G / 2];
    bool finite = true;
#pragma unroll
    for (int i = 0; i < G; i += 2) {
      const __half2 v = __floats2half2_rn(x[i], x[i + 1]);
      finite = finite && isfinite(__low2float(v)) && isfinite(__high2float(v));
      h[i / 2] = *reinterpret_cast<const uint32_t*>(&v);
    }
    if (!finite) {
      set_status(status, STARKV_DEV_QUANT_OVERFLOW);
#pragma unroll
      for (int i = 0; i < G / 2; ++i) h[i] = 0u;
    }
    uint4* dst = reinterpret_cast<uint4*>(region + tile_offset(L, gi) + t * G * 2);
#pragma unroll
    for (int i = 0; i < G / 8; ++i) dst[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    return;
  }
  uint8_t code[G];
  __half s16, zp16;
  const int bits = gi < L.top_groups ? 4 : 3;
  if (!quantize_group<G>(x, bits, code, s16, zp16)) set_status(status, STARKV_DEV_QUANT_OVERFLOW);
  store_group_codes<G>(region, L, gi, t, code);
  const uint32_t m = (uint32_t)__half_as_ushort(s16) | ((uint32_t)__half_as_ushort(zp16) << 16);
  meta_page[gi * kPage + t] = m;
}

__device__ inline void rotate_quantize_store_any(const float* x, const LatentGeom& L, int gi,
                                                 uint8_t* region, uint32_t* meta_page, int t,
                                                 unsigned int* status) {
  switch (L.g) {
    case 4: rotate_quantize_store<4>(x, L, gi, region, meta_page, t, status); break;
    case 8: rotate_quantize_store<8>(x, L, gi, region, meta_page, t, status); break;
    default: rotate_quantize_store<16>(x, L, gi, region, meta_page, t, status); break;
  }
}

// ---------------------------------------------------------------------------
// Launchers (defined in the .cu files)
// ---------------------------------------------------------------------------
cudaError_t launch_prepare_factors(const Ctx& c, const __nv_bfloat16* Bk, const __nv_bfloat16* Bv,
                                   cudaStream_t s);
cudaError_t launch_quantize_pack(const Ctx& c, const LatentGeom& L, const float* z, int64_t n,
                                 uint8_t* codes, uint32_t* meta, cudaStream_t s);
cudaError_t launch_dequantize(const Ctx& c, const LatentGeom& L, const uint8_t* codes,
                              const uint32_t* meta, int64_t n, float* z, cudaStream_t s);
cudaError_t launch_append(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* X,
                          const int64_t* slots, int64_t n, float* latents_out, cudaStream_t s);

struct DecodePlan {
  int splits;
  int pages_per_split;
  size_t ws_bytes;
};
DecodePlan plan_decode(const Ctx& c, int batch, int max_pages);
DecodePlan plan_decode_simt(const Ctx& c, int batch, int max_pages);
cudaError_t launch_decode_simt(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                               const int32_t* block_table, const int32_t* seq_lens, int batch, int max_pages,
                               __nv_bfloat16* out, void* ws, const DecodePlan& plan, cudaStream_t s);
// tensor-core decode (decode_tc.cu)
bool tc_decode_supported(const starkv_config& cfg);
DecodePlan plan_decode_tc(const Ctx& c, int batch, int max_pages);
// Decode over one slice of each sequence's context (sequence sharding): the
// slice's tokens sit at positions pos0[b] .. pos0[b] + seq_lens[b] - 1, the
// query at qpos[b]; the results are fp32 outputs normalised within the slice
// (out_o [B][H][d]) and the slice's softmax statistics (out_ml [B][H][2]).
struct DecodeSlice {
  const int32_t* pos0;
  const int32_t* qpos;
  float* out_o;
  float* out_ml;
};
cudaError_t launch_decode_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                             const int32_t* block_table, const int32_t* seq_lens, int batch, int max_pages,
                             __nv_bfloat16* out, void* ws, const DecodePlan& plan, cudaStream_t s,
                             const DecodeSlice* slice = nullptr);
cudaError_t launch_merge_slices(const float* o_parts, const float* ml_parts, int n_parts, int64_t bh, int d,
                                __nv_bfloat16* out, cudaStream_t s);
cudaError_t launch_prepare_tc_factors(const Ctx& c, cudaStream_t s);
cudaError_t launch_decode(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                          const int32_t* block_table, const int32_t* seq_lens, int batch,
                          int max_pages, __nv_bfloat16* out, void* ws, const DecodePlan& plan,
                          cudaStream_t s);

// Output projection y = o W_o of a decode step's bf16 output o [batch][H*d_h]
// (quant.cu); zpart: [wo_splits][kSmallAppend][model_dim] fp32 scratch.
cudaError_t launch_outproj(const Ctx& c, const __nv_bfloat16* o, int batch, __nv_bfloat16* y, float* zpart,
                           cudaStream_t s);

// Built-in scratch of starkv_decode_attn_noalloc (see decode.cu).
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB
cudaError_t noalloc_scratch(void** out);

struct PrefillPlan {
  int chunk;          // key positions expanded per pass
  size_t ws_bytes;
};
PrefillPlan plan_prefill(const Ctx& c, int batch, int max_pages, int64_t total_q);
PrefillPlan plan_prefill_simt(const Ctx& c, int batch, int max_pages, int64_t total_q);
cudaError_t launch_prefill_simt(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                                const int32_t* cu_q, const int32_t* block_table, const int32_t* seq_lens,
                                int batch, int max_pages, int64_t total_q, int max_q_len,
                                __nv_bfloat16* out, void* ws, const PrefillPlan& plan, cudaStream_t s);
// tensor-core prefill (prefill_tc.cu)
bool tc_prefill_supported(const Ctx& c);
PrefillPlan plan_prefill_tc(const Ctx& c, int batch, int max_pages, int64_t total_q);
cudaError_t launch_prefill_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                              const int32_t* cu_q, const int32_t* block_table, const int32_t* seq_lens,
                              int batch, int max_pages, int64_t total_q, int max_q_len,
                              __nv_bfloat16* out, void* ws, const PrefillPlan& plan, cudaStream_t s);
cudaError_t launch_prepare_prefill_factors(const Ctx& c, cudaStream_t s);
// tensor-core append of more than kSmallAppend tokens (append_tc.cu)
bool tc_append_supported(const Ctx& c);
cudaError_t launch_append_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* X, const int64_t* slots,
                             int64_t n, float* latents_out, cudaStream_t s);
bool make_prefill_maps(Ctx* c);
cudaError_t launch_prefill(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                           const int32_t* cu_q, const int32_t* block_table, const int32_t* seq_lens,
                           int batch, int max_pages, int64_t total_q, int max_q_len,
                           __nv_bfloat16* out, void* ws, const PrefillPlan& plan, cudaStream_t s);

}  // namespace starkv

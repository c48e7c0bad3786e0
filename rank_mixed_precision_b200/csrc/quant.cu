// Factor preparation, the append kernel (projection with rotation, quantisation
// and packing fused into its epilogue), and the quantise/dequantise entries.
//
// Source: "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression",
// Algorithm 2 steps 1-3 (project the new hidden state into latent keys and
// values; apply the prepared block rotations; quantise and append), section 6.1
// eq. 13 (block-diagonal orthogonal rotation, absorbed by the up-projection)
// and eq. 14 (4-bit leading channels, 3-bit the rest).
#include "internal.cuh"
#include "sm100.cuh"

namespace starkv {

// ---------------------------------------------------------------------------
// B' = H B: fold the per-group rotation into an up-projection (eq. 13: the
// up-projection absorbs H^T; H is symmetric).  One thread per output element,
// fp64 accumulation of the g signed terms, rounded once to fp32.
// B: [rows][cols] bf16 with rows grouped by g, out: [rows][cols] fp32.
// ---------------------------------------------------------------------------
__global__ void fold_rotation_kernel(const __nv_bfloat16* __restrict__ B, float* __restrict__ out,
                                     int64_t rows, int cols, int g) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int64_t row = idx / cols;
  const int col = (int)(idx % cols);
  const int i = (int)(row % g);
  const int64_t base = row - i;
  double acc = 0.0;
  for (int j = 0; j < g; ++j) {
    const double v = (double)__bfloat162float(B[(base + j) * cols + col]);
    acc += (__popc(i & j) & 1) ? -v : v;
  }
  out[idx] = (float)(acc / sqrt((double)g));
}

cudaError_t launch_prepare_factors(const Ctx& c, const __nv_bfloat16* Bk, const __nv_bfloat16* Bv,
                                   cudaStream_t s) {
  const starkv_config& f = c.cfg;
  if (!c.ragged) {
    const int64_t rows = (int64_t)f.num_kv_heads * f.rank_k;  // groups never cross heads (g | r_k)
    const int64_t total = rows * f.head_dim;
    fold_rotation_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(Bk, c.Bk, rows, f.head_dim, c.key.g);
  } else {
    for (int h = 0; h < f.num_kv_heads; ++h) {  // each head with its own rank and group size
      const KeyHead& kh = c.khead_host[h];
      const int64_t total = (int64_t)kh.L.r * f.head_dim;
      const int64_t off = (int64_t)kh.col0 * f.head_dim;
      fold_rotation_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(Bk + off, c.Bk + off, kh.L.r, f.head_dim,
                                                                          kh.L.g);
    }
  }
  {
    const int64_t rows = f.rank_v;
    const int cols = f.num_kv_heads * f.head_dim;
    const int64_t total = rows * cols;
    fold_rotation_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(Bv, c.Bv, rows, cols, c.val.g);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Quantise/pack entry: one thread per (token, group).  The pages are zeroed
// by the launcher first.
// ---------------------------------------------------------------------------
__global__ void quantize_pack_kernel(LatentGeom L, const float* __restrict__ z, int64_t n,
                                     uint8_t* __restrict__ codes, uint32_t* __restrict__ meta,
                                     unsigned int* status) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * L.groups) return;
  const int64_t tok = idx / L.groups;
  const int gi = (int)(idx % L.groups);
  const int64_t page = tok / kPage;
  const int t = (int)(tok % kPage);
  rotate_quantize_store_any(z + tok * L.r + gi * L.g, L, gi, codes + page * L.region_bytes,
                            meta + page * L.groups * kPage, t, status);
}

cudaError_t launch_quantize_pack(const Ctx& c, const LatentGeom& L, const float* z, int64_t n,
                                 uint8_t* codes, uint32_t* meta, cudaStream_t s) {
  const int64_t pages = (n + kPage - 1) / kPage;
  cudaError_t e = cudaMemsetAsync(codes, 0, (size_t)pages * L.region_bytes, s);
  if (e != cudaSuccess) return e;
  if (!L.fp16) {  // fp16 latents carry no metadata
    e = cudaMemsetAsync(meta, 0, (size_t)pages * L.groups * kPage * 4, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t total = n * L.groups;
  if (total == 0) return cudaSuccess;
  quantize_pack_kernel<<<(unsigned)((total + 127) / 128), 128, 0, s>>>(L, z, n, codes, meta, c.status);
  return cudaGetLastError();
}

// z_hat = fl32(code * s + zp): code * s is exact, so one fused multiply-add rounds once.
__global__ void dequantize_kernel(LatentGeom L, const uint8_t* __restrict__ codes,
                                  const uint32_t* __restrict__ meta, int64_t n, float* __restrict__ z) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * L.r) return;
  const int64_t tok = idx / L.r;
  const int ch = (int)(idx % L.r);
  const int64_t page = tok / kPage;
  const int t = (int)(tok % kPage);
  const int gi = ch / L.g;
  z[idx] = latent_value(codes + page * L.region_bytes, meta + page * L.groups * kPage, L, gi, t, ch % L.g);
}

cudaError_t launch_dequantize(const Ctx&, const LatentGeom& L, const uint8_t* codes,
                              const uint32_t* meta, int64_t n, float* z, cudaStream_t s) {
  const int64_t total = n * L.r;
  if (total == 0) return cudaSuccess;
  dequantize_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(L, codes, meta, n, z);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Append: Z = X [A_k | A_v] (bf16 inputs, fp32 accumulation), then per
// (token, group): rotate, quantise, pack into the token's page slot.
// Tile: 32 tokens x 64 latent columns, 256 threads, 2 x 4 outputs per thread.
// Every 64-column tile starts on a group boundary of whichever latent it
// covers, because h_kv r_k and R are multiples of 16 and g divides 16.
// ---------------------------------------------------------------------------
struct AppendArgs {
  LatentGeom key, val;
  const KeyHead* kh;       // [h_kv] per-head key geometry and page offsets
  int key_cols, kpage_bytes, kpage_meta;
  int h_kv, hidden, lat_cols;
  int64_t n, n_pages;
  const __nv_bfloat16* X;
  const __nv_bfloat16* A;
  const int64_t* slots;
  float* lat_out;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_meta;
  uint32_t* v_meta;
  unsigned int* status;
};

constexpr int kAppBM = 32, kAppBN = 64, kAppBK = 32;

__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  __shared__ float Xs[kAppBK][kAppBM + 1];
  __shared__ float As[kAppBK][kAppBN];
  __shared__ float Zs[kAppBM][kAppBN + 1];
  const int tid = threadIdx.x;
  const int64_t row0 = (int64_t)blockIdx.x * kAppBM;
  const int col0 = blockIdx.y * kAppBN;
  const int ty = tid / 16, tx = tid % 16;
  float acc[2][4] = {};
  for (int k0 = 0; k0 < a.hidden; k0 += kAppBK) {
    for (int e = tid; e < kAppBM * kAppBK; e += 256) {
      const int m = e / kAppBK, k = e % kAppBK;
      const int64_t row = row0 + m;
      Xs[k][m] = row < a.n ? __bfloat162float(a.X[row * a.hidden + k0 + k]) : 0.f;
    }
    for (int e = tid; e < kAppBK * kAppBN; e += 256) {
      const int k = e / kAppBN, cc = e % kAppBN;
      const int col = col0 + cc;
      As[k][cc] = col < a.lat_cols ? __bfloat162float(a.A[(int64_t)(k0 + k) * a.lat_cols + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kAppBK; ++k) {
      const float x0 = Xs[k][ty * 2], x1 = Xs[k][ty * 2 + 1];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float w = As[k][tx * 4 + j];
        acc[0][j] = fmaf(x0, w, acc[0][j]);
        acc[1][j] = fmaf(x1, w, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) Zs[ty * 2 + i][tx * 4 + j] = acc[i][j];
  __syncthreads();
  if (a.lat_out) {
    for (int e = tid; e < kAppBM * kAppBN; e += 256) {
      const int m = e / kAppBN, cc = e % kAppBN;
      const int64_t row = row0 + m;
      if (row < a.n && col0 + cc < a.lat_cols) a.lat_out[row * a.lat_cols + col0 + cc] = Zs[m][cc];
    }
  }
  // epilogue: one item per (token, 4-column unit); the unit that starts a group does the group
  const int key_cols = a.key_cols;
  for (int e = tid; e < kAppBM * (kAppBN / 4); e += 256) {
    const int m = e / (kAppBN / 4);
    const int cc = (e % (kAppBN / 4)) * 4;
    const int col = col0 + cc;
    const int64_t row = row0 + m;
    if (row >= a.n || col >= a.lat_cols) continue;
    const bool is_key = col < key_cols;
    const int kv = is_key ? key_head_of(a.kh, a.h_kv, col) : 0;
    const LatentGeom L = is_key ? a.kh[kv].L : a.val;
    const int cin = is_key ? col - a.kh[kv].col0 : col - key_cols;
    if (cin % L.g != 0) continue;
    const int64_t slot = a.slots[row];
    if (slot < 0) continue;
    if (slot >= a.n_pages * kPage) {
      set_status(a.status, STARKV_DEV_BAD_SLOT);
      continue;
    }
    const int64_t page = slot / kPage;
    const int t = (int)(slot % kPage);
    const int gi = cin / L.g;
    if (is_key) {
      rotate_quantize_store_any(&Zs[m][cc], L, gi, a.k_codes + page * a.kpage_bytes + a.kh[kv].code_off,
                                a.k_meta + page * a.kpage_meta + a.kh[kv].meta_off, t, a.status);
    } else {
      rotate_quantize_store_any(&Zs[m][cc], L, gi, a.v_codes + page * L.region_bytes,
                                a.v_meta + page * L.groups * kPage, t, a.status);
    }
  }
}

// ---------------------------------------------------------------------------
// Small appends (a decode step adds one token per sequence): the projection is
// a thin GEMM bound by reading A once.  Split K so the whole GPU streams A: a
// CTA owns 128 columns x KL rows of A, fetched as a few 128-byte-swizzled TMA
// boxes that are all in flight at once, multiplies the n x KL slice of X into
// them (mma.sync, fp32 accumulators) and writes its n x 128 partial sums to
// its own slot of the context's split buffer; the quantise kernel adds the
// splits in a fixed order (deterministic), rotates, quantises and packs.
// ---------------------------------------------------------------------------
constexpr int kAgCols = 128;  // output columns per CTA: 8 warps x 16

__global__ void __launch_bounds__(256, 1)
    append_gemm_kernel(const __grid_constant__ CUtensorMap a_map, const AppendArgs a, int KL, float* zpart) {
  extern __shared__ uint8_t ag_smem[];
  uint8_t* sm = ag_smem + ((1024u - (sm100::smem_u32(ag_smem) & 1023u)) & 1023u);
  __shared__ uint64_t bar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * kAgCols, ks = blockIdx.y, k0 = ks * KL;
  const int n = (int)a.n, mtiles = (n + 15) / 16;
  sm100::pdl_launch_dependents();
  const int box_rows = KL < 256 ? KL : 256;
  const int nbox = 2 * (KL / box_rows);
  if (tid == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  // A slice: two 64-column halves of KL rows (128-byte rows, 128-byte swizzle)
  if (warp == 0) {
    if (lane == 0) sm100::mbar_arrive_expect_tx(&bar, (uint32_t)KL * kAgCols * 2);
    __syncwarp();
    for (int i = lane; i < nbox; i += 32) {
      const int half = i & 1, rb = i >> 1;
      sm100::tma_load_2d(sm + half * KL * 128 + rb * box_rows * 128, &a_map, c0 + half * 64, k0 + rb * box_rows, &bar);
    }
  }
  // X slice (rows >= n are zero), row stride KL + 8 elements against bank conflicts
  __nv_bfloat16* Xs = reinterpret_cast<__nv_bfloat16*>(sm + 2 * KL * 128);
  const int xs = KL + 8;
  for (int e = tid; e < mtiles * 16 * (KL / 8); e += blockDim.x) {
    const int r = e / (KL / 8), q = e % (KL / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < n) v = *reinterpret_cast<const uint4*>(a.X + (int64_t)r * a.hidden + k0 + q * 8);
    *reinterpret_cast<uint4*>(Xs + r * xs + q * 8) = v;
  }
  __syncthreads();
  if (!__all_sync(0xffffffffu, sm100::mbar_wait(&bar, 0))) {
    if (lane == 0) set_status(a.status, kDevWaitTimeout);
    return;
  }
  const int half = warp >> 2, wc = (warp & 3) * 16;  // this warp's 16 columns inside its 64-column half
  const uint8_t* At = sm + half * KL * 128;
  float acc[kSmallAppend / 16][2][4] = {};
  for (int kk = 0; kk < KL; kk += 16) {
    uint32_t b[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int k = kk + (lane & 15);
      const int chunk = ((wc + nt * 8) >> 3) ^ (k & 7);
      sm100::ldsm_x2_t(sm100::smem_u32(At + k * 128 + chunk * 16), b[nt][0], b[nt][1]);
    }
#pragma unroll
    for (int mt = 0; mt < kSmallAppend / 16; ++mt) {
      if (mt < mtiles) {
        uint32_t a0, a1, a2, a3;
        sm100::ldsm_x4(sm100::smem_u32(Xs + (mt * 16 + (lane & 15)) * xs + kk + (lane >> 4) * 8), a0, a1, a2, a3);
        sm100::mma16816_bf16(acc[mt][0], a0, a1, a2, a3, b[0][0], b[0][1]);
        sm100::mma16816_bf16(acc[mt][1], a0, a1, a2, a3, b[1][0], b[1][1]);
      }
    }
  }
  float* zp = zpart + (int64_t)ks * kSmallAppend * a.lat_cols;
#pragma unroll
  for (int mt = 0; mt < kSmallAppend / 16; ++mt) {
    if (mt >= mtiles) break;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int col = c0 + half * 64 + wc + nt * 8 + (lane & 3) * 2;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = mt * 16 + (lane >> 2) + hf * 8;
        if (r < n && col < a.lat_cols)
          *reinterpret_cast<float2*>(zp + (int64_t)r * a.lat_cols + col) =
              make_float2(acc[mt][nt][hf * 2], acc[mt][nt][hf * 2 + 1]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Output projection of a decode step (the attention block's output, [Review]
// Algorithm 2 steps 7-8: apply the head-specific output factors and sum the
// head contributions): y[b] = sum_h o_h[b] W_o[h d : (h + 1) d, :], a thin GEMM
// [B x H d] . [H d x model_dim] bound by reading W_o once.  The same split-K
// kernel as the small appends (A slice by TMA, mma.sync), then a reduction of
// the split sums in a fixed order.
// ---------------------------------------------------------------------------
__global__ void outproj_reduce_kernel(const float* __restrict__ zpart, int splits, int rows, int cols,
                                      __nv_bfloat16* __restrict__ y) {
  sm100::pdl_wait();  // the split sums
  sm100::pdl_launch_dependents();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)rows * cols) return;
  const int r = (int)(idx / cols), col = (int)(idx % cols);
  float v = 0.f;
  for (int sp = 0; sp < splits; ++sp) v += __ldcg(zpart + ((int64_t)sp * kSmallAppend + r) * cols + col);
  y[idx] = __float2bfloat16_rn(v);
}

cudaError_t launch_outproj(const Ctx& c, const __nv_bfloat16* o, int batch, __nv_bfloat16* y, float* zpart,
                           cudaStream_t s) {
  const int K = c.cfg.num_q_heads * c.cfg.head_dim, N = c.model_dim;
  const int KL = K / c.wo_splits;
  const size_t smem_max = (size_t)2 * KL * 128 + (size_t)kSmallAppend * (KL + 8) * 2 + 1024;
  cudaError_t e = cudaFuncSetAttribute(append_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
  if (e != cudaSuccess) return e;
  for (int b0 = 0; b0 < batch; b0 += kSmallAppend) {
    const int n = batch - b0 < kSmallAppend ? batch - b0 : kSmallAppend;
    AppendArgs a = {};
    a.hidden = K;
    a.lat_cols = N;
    a.n = n;
    a.X = o + (int64_t)b0 * K;
    a.status = c.status;
    const size_t smem = (size_t)2 * KL * 128 + (size_t)((n + 15) / 16) * 16 * (KL + 8) * 2 + 1024;
    dim3 g1((unsigned)((N + kAgCols - 1) / kAgCols), (unsigned)c.wo_splits);
    // a plain launch: the kernel reads o without waiting on a programmatic edge
    append_gemm_kernel<<<g1, 256, smem, s>>>(c.wo_map, a, KL, zpart);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t total = (int64_t)n * N;
    e = launch_chained(outproj_reduce_kernel, dim3((unsigned)((total + 255) / 256)), dim3(256), 0, s, 1u,
                       (const float*)zpart, c.wo_splits, n, N, y + (int64_t)b0 * N);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// One thread per (token, 4 columns): it adds its columns' split sums (every
// load in flight at once), then the group's leader gathers the group's g values
// from its neighbours by shuffles (groups never straddle a warp: they start on
// multiples of g <= 16 columns and a warp covers 128) and rotates, quantises and
// packs them.
constexpr int kMaxAppSplits = 16;

__global__ void __launch_bounds__(128) append_quant_kernel(AppendArgs a, const float* zpart, int splits) {
  sm100::pdl_wait();  // the split sums of the projection kernel
  sm100::pdl_launch_dependents();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int units = a.lat_cols / 4;
  const bool active = idx < a.n * units;
  const int64_t row = active ? idx / units : 0;
  const int col = active ? (int)(idx % units) * 4 : 0;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    float4 part[kMaxAppSplits];
#pragma unroll
    for (int sp = 0; sp < kMaxAppSplits; ++sp)
      if (sp < splits)
        part[sp] = __ldcg(reinterpret_cast<const float4*>(zpart + ((int64_t)sp * kSmallAppend + row) * a.lat_cols + col));
#pragma unroll
    for (int sp = 0; sp < kMaxAppSplits; ++sp) {  // fixed order: deterministic sums
      if (sp < splits) {
        v.x += part[sp].x;
        v.y += part[sp].y;
        v.z += part[sp].z;
        v.w += part[sp].w;
      }
    }
  }
  const int key_cols = a.key_cols;
  const bool is_key = col < key_cols;
  const int kv = is_key ? key_head_of(a.kh, a.h_kv, col) : 0;
  const LatentGeom L = is_key ? a.kh[kv].L : a.val;
  const int cin = is_key ? col - a.kh[kv].col0 : col - key_cols;
  const int lane = threadIdx.x & 31;
  float x[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // units lane .. lane + 3 (a group spans g / 4 <= 4 of them)
    const int src = lane + j < 32 ? lane + j : 31;
    x[4 * j] = __shfl_sync(0xffffffffu, v.x, src);
    x[4 * j + 1] = __shfl_sync(0xffffffffu, v.y, src);
    x[4 * j + 2] = __shfl_sync(0xffffffffu, v.z, src);
    x[4 * j + 3] = __shfl_sync(0xffffffffu, v.w, src);
  }
  if (!active || cin % L.g != 0) return;
  if (a.lat_out)
    for (int i = 0; i < L.g; ++i) a.lat_out[row * a.lat_cols + col + i] = x[i];
  const int64_t slot = a.slots[row];
  if (slot >= a.n_pages * kPage) {
    set_status(a.status, STARKV_DEV_BAD_SLOT);
  } else if (slot >= 0) {
    const int64_t page = slot / kPage;
    const int t = (int)(slot % kPage);
    const int gi = cin / L.g;
    if (is_key) {
      rotate_quantize_store_any(x, L, gi, a.k_codes + page * a.kpage_bytes + a.kh[kv].code_off,
                                a.k_meta + page * a.kpage_meta + a.kh[kv].meta_off, t, a.status);
    } else {
      rotate_quantize_store_any(x, L, gi, a.v_codes + page * L.region_bytes, a.v_meta + page * L.groups * kPage,
                                t, a.status);
    }
  }
}

cudaError_t launch_append(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* X,
                          const int64_t* slots, int64_t n, float* latents_out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  AppendArgs a;
  a.key = c.key;
  a.val = c.val;
  a.kh = c.khead;
  a.key_cols = c.key_cols;
  a.kpage_bytes = c.kpage_bytes;
  a.kpage_meta = c.kpage_meta;
  a.h_kv = c.cfg.num_kv_heads;
  a.hidden = c.cfg.hidden;
  a.lat_cols = c.lat_cols;
  a.n = n;
  a.n_pages = cache.n_pages;
  a.X = X;
  a.A = c.A;
  a.slots = slots;
  a.lat_out = latents_out;
  a.k_codes = (uint8_t*)cache.k_codes;
  a.v_codes = (uint8_t*)cache.v_codes;
  a.k_meta = (uint32_t*)cache.k_meta;
  a.v_meta = (uint32_t*)cache.v_meta;
  a.status = c.status;
  if (n <= kSmallAppend && c.app_splits > 0 && (reinterpret_cast<uintptr_t>(X) & 15) == 0) {
    const int KL = c.cfg.hidden / c.app_splits;
    const size_t smem = (size_t)2 * KL * 128 + (size_t)((n + 15) / 16) * 16 * (KL + 8) * 2 + 1024;
    cudaError_t e = cudaFuncSetAttribute(append_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 g1((unsigned)((c.lat_cols + kAgCols - 1) / kAgCols), (unsigned)c.app_splits);
    append_gemm_kernel<<<g1, 256, smem, s>>>(c.a_map, a, KL, c.zpart);
    const int64_t units = n * (c.lat_cols / 4);
    e = launch_chained(append_quant_kernel, dim3((unsigned)((units + 127) / 128)), dim3(128), 0, s, 1u, a,
                       (const float*)c.zpart, c.app_splits);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (c.tc_append && (reinterpret_cast<uintptr_t>(X) & 15) == 0)
    return launch_append_tc(c, cache, X, slots, n, latents_out, s);
  dim3 grid((unsigned)((n + kAppBM - 1) / kAppBM), (unsigned)((c.lat_cols + kAppBN - 1) / kAppBN));
  append_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace starkv

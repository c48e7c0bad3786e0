// Split-K decode attention over the packed latent cache.
//
// Source: "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression",
// Algorithm 2 steps 4-8 and section 5.3: per key tile, dequantise the latent,
// re-expand the key, apply RoPE and score without storing a key cache; softmax;
// multiply the stacked probabilities by the shared value latent (eq. 12); apply
// the value up-projection.  Splits over the key axis are merged with the softmax
// partition identity (CaliDrop review, attention decomposition theorem, eq. 1).
//
// Scoring reassociation used here: with the query rotated to its position,
//   s_j = sum_i cos(j th_i) a_i(j) + sin(j th_i) b_i(j),
//   a_i = q_i k_i + q_{i+d/2} k_{i+d/2},   b_i = q_{i+d/2} k_i - q_i k_{i+d/2},
// and k = z B' is linear in the latent z, so a_i = z . Wa[:, i], b_i = z . Wb[:, i]
// with Wa, Wb built once per (sequence, head) from the query and B'.  This is the
// same re-expansion cost (r_k d_h per token and head) as forming k, fused with RoPE
// and the dot product.
#include <float.h>

#include <mutex>

#include "internal.cuh"
#include "sm100.cuh"

namespace starkv {

constexpr int kDecThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  LatentGeom key, val;
  const KeyHead* kh;    // [h_kv] per-head key geometry and page offsets
  int kpage_bytes, kpage_meta;
  int H, h_kv, group, d, max_position;
  int max_pages, pages_per_split, splits;
  int64_t n_pages;
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint32_t* k_meta;
  const uint32_t* v_meta;
  const float* Bk;      // [h_kv][r_k][d]
  const float* Bv;      // [R][h_kv*d]
  const float2* rope;   // [max_position][d/2]
  float* part;          // [B][H][splits][R + 2]: m (log2 domain), l, acc[R]
  __nv_bfloat16* out;
  unsigned int* status;
};

__device__ inline float block_reduce_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = red[0];
  for (int i = 1; i < (int)(blockDim.x / 32); ++i) v = fmaxf(v, red[i]);
  return v;
}

__device__ inline float block_reduce_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = 0.f;
  for (int i = 0; i < (int)(blockDim.x / 32); ++i) v += red[i];
  return v;
}

// grid (splits, H, B).  Dynamic smem: Wa, Wb [d/2][r_k] fp32, scores/probs, pages.
template <int RK>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(DecodeArgs a) {
  extern __shared__ float smem[];
  const int half = a.d / 2;
  float* Wa = smem;                       // [half][RK]
  float* Wb = Wa + half * RK;             // [half][RK]
  float* P = Wb + half * RK;              // [kDecThreads]
  float* qr = P + kDecThreads;            // [d]
  float* red = qr + a.d;                  // [32]
  int* pg = reinterpret_cast<int*>(red + 32);  // [kDecThreads / 16 + 1]

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int kv = h / a.group;
  const int R = a.val.r;
  const KeyHead khd = a.kh[kv];  // this KV head's rank r_h <= RK, its B'_k rows and page offsets
  const LatentGeom& KL = khd.L;
  float* part = a.part + (((int64_t)b * a.H + h) * a.splits + split) * (R + 2);

  const int seq_len = a.seq_lens[b];
  const bool bad_len = seq_len < 0 || seq_len > a.max_pages * kPage || seq_len > a.max_position;
  if (bad_len && split == 0 && h == 0 && tid == 0) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
  const int t_lo = split * a.pages_per_split * kPage;
  const int t_hi = bad_len ? 0 : min(seq_len, t_lo + a.pages_per_split * kPage);

  // rotated, scaled query and the fused re-expansion/RoPE weights
  if (t_lo < t_hi) {
    const int pos = seq_len - 1;
    const __nv_bfloat16* qv = a.q + ((int64_t)b * a.H + h) * a.d;
    const float scale = kLog2e * rsqrtf((float)a.d);
    for (int i = tid; i < half; i += kDecThreads) {
      const float2 cs = a.rope[(int64_t)pos * half + i];
      const float x0 = __bfloat162float(qv[i]), x1 = __bfloat162float(qv[i + half]);
      qr[i] = (x0 * cs.x - x1 * cs.y) * scale;
      qr[i + half] = (x1 * cs.x + x0 * cs.y) * scale;
    }
    __syncthreads();
    const float* Bk = a.Bk + (int64_t)khd.col0 * a.d;
    for (int e = tid; e < half * RK; e += kDecThreads) {
      const int i = e / RK, c = e % RK;
      float wa = 0.f, wb = 0.f;  // channels past this head's rank weigh nothing
      if (c < KL.r) {
        const float ba = Bk[c * a.d + i], bb = Bk[c * a.d + i + half];
        wa = qr[i] * ba + qr[i + half] * bb;
        wb = qr[i + half] * ba - qr[i] * bb;
      }
      Wa[e] = wa;
      Wb[e] = wb;
    }
  }
  __syncthreads();

  constexpr int kMaxCh = 4;  // R <= 1024 channels, 256 threads
  float acc[kMaxCh];
#pragma unroll
  for (int k = 0; k < kMaxCh; ++k) acc[k] = 0.f;
  float m = -INFINITY, l = 0.f;
  bool bad_page_seen = false;

  for (int tile = t_lo; tile < t_hi; tile += kDecThreads) {
    const int cnt = min(kDecThreads, t_hi - tile);
    // page ids of this tile
    if (tid < (cnt + kPage - 1) / kPage) {
      int p = a.block_table[(int64_t)b * a.max_pages + tile / kPage + tid];
      if (p < 0 || p >= a.n_pages) {
        p = -1;
        bad_page_seen = true;
      }
      pg[tid] = p;
    }
    __syncthreads();
    float s = -INFINITY;
    if (tid < cnt) {
      const int j = tile + tid;
      const int page = pg[tid / kPage];
      if (page >= 0) {
        const int t = j % kPage;
        const uint8_t* region = a.k_codes + (int64_t)page * a.kpage_bytes + khd.code_off;
        const uint32_t* meta = a.k_meta + (int64_t)page * a.kpage_meta + khd.meta_off;
        float z[RK];
#pragma unroll
        for (int c = 0; c < RK; ++c) z[c] = c < KL.r ? latent_value(region, meta, KL, c / KL.g, t, c % KL.g) : 0.f;
        const float2* rr = a.rope + (int64_t)j * half;
        float acc_s = 0.f;
        for (int i = 0; i < half; ++i) {
          float sa = 0.f, sb = 0.f;
#pragma unroll
          for (int c = 0; c < RK; ++c) {
            sa = fmaf(z[c], Wa[i * RK + c], sa);
            sb = fmaf(z[c], Wb[i * RK + c], sb);
          }
          const float2 cs = rr[i];
          acc_s = fmaf(cs.x, sa, fmaf(cs.y, sb, acc_s));
        }
        s = acc_s;
      }
    }
    const float tmax = block_reduce_max(s, red);
    if (tmax == -INFINITY) {  // nothing valid in this tile
      __syncthreads();
      continue;
    }
    const float m_new = fmaxf(m, tmax);
    const float alpha = exp2f(m - m_new);
    const float p = (s == -INFINITY) ? 0.f : exp2f(s - m_new);
    P[tid] = p;
    const float psum = block_reduce_sum(p, red);
    l = l * alpha + psum;
    m = m_new;
#pragma unroll
    for (int k = 0; k < kMaxCh; ++k) acc[k] *= alpha;
    __syncthreads();
    // P . Z_v: this thread owns channels tid, tid + 256, ...
    for (int tt = 0; tt < cnt; ++tt) {
      const float pt = P[tt];
      if (pt == 0.f) continue;
      const int page = pg[tt / kPage];
      const int t = (tile + tt) % kPage;
      const uint8_t* region = a.v_codes + (int64_t)page * a.val.region_bytes;
      const uint32_t* meta = a.v_meta + (int64_t)page * a.val.groups * kPage;
#pragma unroll
      for (int k = 0; k < kMaxCh; ++k) {
        const int ch = tid + k * kDecThreads;
        if (ch < R) {
          const int gi = ch / a.val.g;
          const float zv = latent_value(region, meta, a.val, gi, t, ch % a.val.g);
          acc[k] = fmaf(pt, zv, acc[k]);
        }
      }
    }
    __syncthreads();
  }
  if (bad_page_seen) set_status(a.status, STARKV_DEV_BAD_PAGE);
  if (tid == 0) {
    part[0] = m;
    part[1] = l;
  }
#pragma unroll
  for (int k = 0; k < kMaxCh; ++k) {
    const int ch = tid + k * kDecThreads;
    if (ch < R) part[2 + ch] = acc[k];
  }
}

// grid (H, B): merge split partials (partition identity), normalise, o = o_lat B'_v[:, kv].
__global__ void __launch_bounds__(kDecThreads) decode_merge_kernel(DecodeArgs a) {
  extern __shared__ float smem[];
  const int R = a.val.r;
  float* olat = smem;              // [R]
  float* w = olat + R;             // [splits]
  float* red = w + a.splits;       // [2 * d]
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int kv = h / a.group;
  const float* part = a.part + ((int64_t)b * a.H + h) * a.splits * (R + 2);
  float M = -INFINITY;
  for (int s = 0; s < a.splits; ++s) M = fmaxf(M, part[(int64_t)s * (R + 2)]);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.splits; ++s) {
      const float ms = part[(int64_t)s * (R + 2)];
      const float ws = ms == -INFINITY ? 0.f : exp2f(ms - M);
      L += ws * part[(int64_t)s * (R + 2) + 1];
      if (tid == 0) w[s] = ws;
    }
  }
  __syncthreads();
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int ch = tid; ch < R; ch += kDecThreads) {
    float o = 0.f;
    if (L > 0.f)
      for (int s = 0; s < a.splits; ++s) o = fmaf(w[s], part[(int64_t)s * (R + 2) + 2 + ch], o);
    olat[ch] = o * inv;
  }
  __syncthreads();
  // two halves of R per output column
  const int nh = kDecThreads / a.d;  // 2 for d = 128, 4 for d = 64
  const int col = tid % a.d, sub = tid / a.d;
  const int ldb = a.h_kv * a.d;
  float o = 0.f;
  for (int ch = sub; ch < R; ch += nh) o = fmaf(olat[ch], a.Bv[(int64_t)ch * ldb + kv * a.d + col], o);
  red[sub * a.d + col] = o;
  __syncthreads();
  if (sub == 0) {
    float t = 0.f;
    for (int k = 0; k < nh; ++k) t += red[k * a.d + col];
    a.out[((int64_t)b * a.H + h) * a.d + col] = __float2bfloat16_rn(t);
  }
}

DecodePlan plan_decode_simt(const Ctx& c, int batch, int max_pages) {
  DecodePlan p;
  const int H = c.cfg.num_q_heads;
  // enough CTAs for a few waves on 148 SMs, at least 256 tokens per split
  const int base = batch * H;
  int splits = (4 * 148 + base - 1) / base;
  const int max_splits = (max_pages + 15) / 16;  // >= 256 tokens each
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  p.pages_per_split = (max_pages + splits - 1) / splits;
  if (p.pages_per_split < 1) p.pages_per_split = 1;
  p.splits = (max_pages + p.pages_per_split - 1) / p.pages_per_split;
  if (p.splits < 1) p.splits = 1;
  p.ws_bytes = (size_t)batch * H * p.splits * (c.cfg.rank_v + 2) * sizeof(float);
  return p;
}

cudaError_t launch_decode_simt(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                               const int32_t* block_table, const int32_t* seq_lens, int batch,
                               int max_pages, __nv_bfloat16* out, void* ws, const DecodePlan& plan,
                               cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  DecodeArgs a;
  a.key = c.key;
  a.val = c.val;
  a.kh = c.khead;
  a.kpage_bytes = c.kpage_bytes;
  a.kpage_meta = c.kpage_meta;
  a.H = c.cfg.num_q_heads;
  a.h_kv = c.cfg.num_kv_heads;
  a.group = c.group;
  a.d = c.cfg.head_dim;
  a.max_position = c.cfg.max_position;
  a.max_pages = max_pages;
  a.pages_per_split = plan.pages_per_split;
  a.splits = plan.splits;
  a.n_pages = cache.n_pages;
  a.q = q;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.k_codes = (const uint8_t*)cache.k_codes;
  a.v_codes = (const uint8_t*)cache.v_codes;
  a.k_meta = (const uint32_t*)cache.k_meta;
  a.v_meta = (const uint32_t*)cache.v_meta;
  a.Bk = c.Bk;
  a.Bv = c.Bv;
  a.rope = c.rope;
  a.part = (float*)ws;
  a.out = out;
  a.status = c.status;
  const int half = a.d / 2;
  const int rk = c.cfg.rank_k;
  const size_t smem = (size_t)(2 * half * rk + kDecThreads + a.d + 32 + kDecThreads / 16 + 1) * 4;
  dim3 grid(plan.splits, a.H, batch);
  cudaError_t e;
  switch (rk) {
    case 16:
      e = cudaFuncSetAttribute(decode_split_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split_kernel<16><<<grid, kDecThreads, smem, s>>>(a);
      break;
    case 32:
      e = cudaFuncSetAttribute(decode_split_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split_kernel<32><<<grid, kDecThreads, smem, s>>>(a);
      break;
    case 48:
      e = cudaFuncSetAttribute(decode_split_kernel<48>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split_kernel<48><<<grid, kDecThreads, smem, s>>>(a);
      break;
    case 64:
      e = cudaFuncSetAttribute(decode_split_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      decode_split_kernel<64><<<grid, kDecThreads, smem, s>>>(a);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t msmem = (size_t)(c.cfg.rank_v + plan.splits + 2 * a.d * 4) * 4;
  if (msmem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
  }
  decode_merge_kernel<<<dim3(a.H, batch), kDecThreads, msmem, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Path selection: the tensor-core kernels (decode_tc.cu) for every shape they
// cover, the CUDA-core kernels above otherwise.
// ---------------------------------------------------------------------------
DecodePlan plan_decode(const Ctx& c, int batch, int max_pages) {
  return c.tc ? plan_decode_tc(c, batch, max_pages) : plan_decode_simt(c, batch, max_pages);
}

cudaError_t launch_decode(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                          const int32_t* block_table, const int32_t* seq_lens, int batch,
                          int max_pages, __nv_bfloat16* out, void* ws, const DecodePlan& plan,
                          cudaStream_t s) {
  if (c.tc) return launch_decode_tc(c, cache, q, block_table, seq_lens, batch, max_pages, out, ws, plan, s);
  return launch_decode_simt(c, cache, q, block_table, seq_lens, batch, max_pages, out, ws, plan, s);
}

// ---------------------------------------------------------------------------
// Built-in scratch for starkv_decode_attn_noalloc.
//
// Some callers cannot allocate device memory (for example a plugin inside a
// serving engine that owns the whole memory pool, or a latency-critical loop
// that must never enter the allocator).  For them, the decode's split partials
// live in this file-scope array instead of a caller workspace.  Every GPU that
// loads the library holds these bytes until the process exits.  All calls on a
// device share the array and it keeps the last call's contents; nothing in it
// needs to start at zero, because the split kernel writes every partial that
// the merge kernel reads in the same call.  Calls that overlap on the GPU
// (other streams, other contexts on the same device) race on it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
}  // namespace

// Device address of the built-in scratch on the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current) and
// caches it; host code must never pass the array's own name to a kernel.
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// Failure-detection check: the same bounded mbarrier wait the pipelined
// kernels use, on a barrier whose single expected arrival never comes.
__global__ void wait_timeout_selftest_kernel(unsigned int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (!__all_sync(0xffffffffu, sm100::mbar_wait(&bar, 0, limit_ns)) && threadIdx.x == 0) set_status(status, kDevWaitTimeout);
}

cudaError_t launch_wait_timeout_selftest(unsigned int* status, uint64_t limit_ns, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace starkv

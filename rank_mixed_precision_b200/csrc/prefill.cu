// Causal chunk attention (prefill) over the packed latent cache.
//
// Source: the chunked form of Algorithm 2 in "STAR-KV: Learning the Rank Is Only
// Half of KV Cache Compression" (key tiles dequantised and re-expanded in the
// computation, RoPE at each position, softmax, values).  Values are re-expanded
// per key position and head (v = z_v B'_v[:, kv]) instead of aggregating P Z_v
// first: with thousands of queries per sequence, P Z_v would cost Nq H T R
// multiply-adds, whereas re-expanding costs T h_kv R d_h once per position
// (section 5.1, eq. 9 weighs exactly this reconstruction bill).
//
// Dataflow: the key axis is walked in chunks of `chunk` positions.  For each
// chunk, one kernel re-expands the chunk's keys (RoPE'd) and values of every
// sequence into a bounded workspace, and a second kernel runs an online-softmax
// pass of every query over that chunk, carrying (m, l, O) per (query, head) in
// the workspace.  The workspace does not grow with the context length.
#include "internal.cuh"

namespace starkv {

constexpr float kLog2eP = 1.4426950408889634f;

struct PrefillArgs {
  LatentGeom key, val;
  const KeyHead* kh;    // [h_kv] per-head key geometry and page offsets
  int kpage_bytes, kpage_meta;
  int H, h_kv, group, d, max_position;
  int batch, max_pages, chunk, max_q_len;
  int64_t n_pages, total_q;
  const __nv_bfloat16* q;
  const int32_t* cu_q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint32_t* k_meta;
  const uint32_t* v_meta;
  const float* Bk;
  const float* Bv;
  const float2* rope;
  float* Kx;    // [B][chunk][h_kv][d]
  float* Vx;    // [B][chunk][h_kv][d]
  float* O;     // [total_q][H][d]
  float* ML;    // [total_q][H][2]
  __nv_bfloat16* out;
  unsigned int* status;
};

__device__ inline bool seq_len_ok(const PrefillArgs& a, int L) {
  return L >= 0 && L <= a.max_pages * kPage && L <= a.max_position;
}

// grid (chunk/32, h_kv, B), 256 threads: keys and values of 32 positions of one KV head.
__global__ void __launch_bounds__(256) prefill_simt_expand_kernel(PrefillArgs a, int c0) {
  __shared__ float Zk[32][65];
  __shared__ float Zv[32][33];
  __shared__ float Bs[32][128];
  __shared__ int pg[2];
  const int tid = threadIdx.x, kv = blockIdx.y, b = blockIdx.z;
  const int j0 = c0 + blockIdx.x * 32;
  const int L = a.seq_lens[b];
  const bool ok_len = seq_len_ok(a, L);
  const int half = a.d / 2;
  const int tt = tid / 8, sub = tid % 8;
  const int j = j0 + tt;
  float* kx = a.Kx + (((int64_t)b * a.chunk + (j - c0)) * a.h_kv + kv) * a.d;
  float* vx = a.Vx + (((int64_t)b * a.chunk + (j - c0)) * a.h_kv + kv) * a.d;
  if (tid < 2) {
    int p = -1;
    const int jj = j0 + tid * 16;
    if (ok_len && jj < L) {
      p = a.block_table[(int64_t)b * a.max_pages + jj / kPage];
      if (p < 0 || p >= a.n_pages) {
        set_status(a.status, STARKV_DEV_BAD_PAGE);
        p = -1;
      }
    }
    pg[tid] = p;
  }
  __syncthreads();
  const bool valid = ok_len && j < L && pg[tt / 16] >= 0;
  // ---- keys: dequantise this position's r_k,h latents, re-expand, RoPE
  const KeyHead khd = a.kh[kv];
  const int rk = khd.L.r;
  for (int e = tid; e < 32 * rk; e += 256) {
    const int t2 = e / rk, c = e % rk;
    float z = 0.f;
    const int page = pg[t2 / 16];
    if (ok_len && j0 + t2 < L && page >= 0) {
      const int t = (j0 + t2) % kPage, gi = c / khd.L.g;
      const uint8_t* region = a.k_codes + (int64_t)page * a.kpage_bytes + khd.code_off;
      z = latent_value(region, a.k_meta + (int64_t)page * a.kpage_meta + khd.meta_off, khd.L, gi, t, c % khd.L.g);
    }
    Zk[t2][c] = z;
  }
  __syncthreads();
  {
    const float* Bk = a.Bk + (int64_t)khd.col0 * a.d;
    const int per = half / 8;
    for (int u = 0; u < per; ++u) {
      const int i = sub * per + u;
      float k0 = 0.f, k1 = 0.f;
      for (int c = 0; c < rk; ++c) {
        k0 = fmaf(Zk[tt][c], Bk[c * a.d + i], k0);
        k1 = fmaf(Zk[tt][c], Bk[c * a.d + i + half], k1);
      }
      float r0 = 0.f, r1 = 0.f;
      if (valid) {
        const float2 cs = a.rope[(int64_t)j * half + i];
        r0 = k0 * cs.x - k1 * cs.y;
        r1 = k1 * cs.x + k0 * cs.y;
      }
      kx[i] = r0;
      kx[i + half] = r1;
    }
  }
  // ---- values: v = z_v B'_v[:, kv*d : kv*d + d], K-loop over R in chunks of 64
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  const int ldb = a.h_kv * a.d;
  const int R = a.val.r;
  for (int ch0 = 0; ch0 < R; ch0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * 32; e += 256) {
      const int t2 = e / 32, c = e % 32;
      const int ch = ch0 + c;
      float z = 0.f;
      const int page = pg[t2 / 16];
      if (ch < R && ok_len && j0 + t2 < L && page >= 0) {
        const int t = (j0 + t2) % kPage, gi = ch / a.val.g;
        const uint8_t* region = a.v_codes + (int64_t)page * a.val.region_bytes;
        z = latent_value(region, a.v_meta + (int64_t)page * a.val.groups * kPage, a.val, gi, t, ch % a.val.g);
      }
      Zv[t2][c] = z;
    }
    for (int e = tid; e < 32 * a.d; e += 256) {
      const int c = e / a.d, dd = e % a.d;
      const int ch = ch0 + c;
      Bs[c][dd] = ch < R ? a.Bv[(int64_t)ch * ldb + kv * a.d + dd] : 0.f;
    }
    __syncthreads();
    const int nd = a.d / 8;
    for (int c = 0; c < 32; ++c) {
      const float z = Zv[tt][c];
      for (int k = 0; k < nd; ++k) acc[k] = fmaf(z, Bs[c][sub + 8 * k], acc[k]);
    }
  }
  const int nd = a.d / 8;
  for (int k = 0; k < nd; ++k) vx[sub + 8 * k] = valid ? acc[k] : 0.f;
}

// grid (ceil(max_q_len/32), H, B), 256 threads = 32 queries x 8 lanes.
__global__ void __launch_bounds__(256) prefill_simt_attn_kernel(PrefillArgs a, int c0) {
  constexpr int KT = 16;  // keys per tile
  __shared__ float Qs[32][129];
  __shared__ float Ks[KT][129];
  __shared__ float Vs[KT][128];
  __shared__ float Ps[32][KT + 1];
  const int tid = threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kv = h / a.group;
  const int qi0 = blockIdx.x * 32;
  const int q0 = a.cu_q[b], q1 = a.cu_q[b + 1];
  const int nb = q1 - q0;
  const int L = a.seq_lens[b];
  if (q0 < 0 || q1 > a.total_q || nb <= 0 || qi0 >= nb) return;  // malformed spans: flagged by finalize
  if (!seq_len_ok(a, L) || nb > L) return;  // flagged by the finalize kernel
  const int half = a.d / 2;
  const int qq = tid / 8, sub = tid % 8;
  const int qi = qi0 + qq;
  const bool qvalid = qi < nb;
  const int pos = L - nb + qi;                  // this query's position
  const int pos_max = L - nb + min(nb, qi0 + 32) - 1;
  const int j_end = min(min(c0 + a.chunk, L), pos_max + 1);
  if (j_end <= c0) return;
  const int64_t row = (int64_t)q0 + qi;
  // rotated, scaled queries
  {
    const float scale = kLog2eP * rsqrtf((float)a.d);
    const int per = half / 8;
    for (int u = 0; u < per; ++u) {
      const int i = sub * per + u;
      float r0 = 0.f, r1 = 0.f;
      if (qvalid) {
        const __nv_bfloat16* qv = a.q + (row * a.H + h) * a.d;
        const float x0 = __bfloat162float(qv[i]), x1 = __bfloat162float(qv[i + half]);
        const float2 cs = a.rope[(int64_t)pos * half + i];
        r0 = (x0 * cs.x - x1 * cs.y) * scale;
        r1 = (x1 * cs.x + x0 * cs.y) * scale;
      }
      Qs[qq][i] = r0;
      Qs[qq][i + half] = r1;
    }
  }
  // carried state
  float m = -INFINITY, l = 0.f;
  float o[16];
  const int nd = a.d / 8;
  if (qvalid) {
    m = a.ML[(row * a.H + h) * 2];
    l = a.ML[(row * a.H + h) * 2 + 1];
    for (int k = 0; k < nd; ++k) o[k] = a.O[(row * a.H + h) * a.d + sub + 8 * k];
  } else {
    for (int k = 0; k < nd; ++k) o[k] = 0.f;
  }
  for (int jt = c0; jt < j_end; jt += KT) {
    __syncthreads();
    for (int e = tid; e < KT * a.d; e += 256) {
      const int t2 = e / a.d, dd = e % a.d;
      const int j = jt + t2;
      const bool in = j < j_end;
      const int64_t base = (((int64_t)b * a.chunk + (j - c0)) * a.h_kv + kv) * a.d + dd;
      Ks[t2][dd] = in ? a.Kx[base] : 0.f;
      Vs[t2][dd] = in ? a.Vx[base] : 0.f;
    }
    __syncthreads();
    float s[KT / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int u = 0; u < KT / 8; ++u) {
      const int kk = sub + 8 * u;
      const int j = jt + kk;
      float acc = 0.f;
      for (int dd = 0; dd < a.d; ++dd) acc = fmaf(Qs[qq][dd], Ks[kk][dd], acc);
      s[u] = (qvalid && j < j_end && j <= pos) ? acc : -INFINITY;
      tmax = fmaxf(tmax, s[u]);
    }
    for (int off = 1; off < 8; off <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    const float m_new = fmaxf(m, tmax);
    float psum = 0.f;
    float alpha = 1.f;
    if (m_new != -INFINITY) {
      alpha = exp2f(m - m_new);
#pragma unroll
      for (int u = 0; u < KT / 8; ++u) {
        const float p = s[u] == -INFINITY ? 0.f : exp2f(s[u] - m_new);
        Ps[qq][sub + 8 * u] = p;
        psum += p;
      }
    } else {
#pragma unroll
      for (int u = 0; u < KT / 8; ++u) Ps[qq][sub + 8 * u] = 0.f;
    }
    for (int off = 1; off < 8; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    __syncwarp();
    if (m_new != -INFINITY) {
      l = l * alpha + psum;
      m = m_new;
      for (int k = 0; k < nd; ++k) {
        float acc = o[k] * alpha;
        for (int kk = 0; kk < KT; ++kk) acc = fmaf(Ps[qq][kk], Vs[kk][sub + 8 * k], acc);
        o[k] = acc;
      }
    }
  }
  if (qvalid) {
    a.ML[(row * a.H + h) * 2] = m;
    a.ML[(row * a.H + h) * 2 + 1] = l;
    for (int k = 0; k < nd; ++k) a.O[(row * a.H + h) * a.d + sub + 8 * k] = o[k];
  }
}

__global__ void prefill_simt_init_kernel(PrefillArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = a.total_q * a.H;
  if (idx >= n) return;
  a.ML[idx * 2] = -INFINITY;
  a.ML[idx * 2 + 1] = 0.f;
  for (int k = 0; k < a.d; ++k) a.O[idx * a.d + k] = 0.f;
}

// one thread per (query row, head, dim); also validates the query spans
__global__ void prefill_simt_finalize_kernel(PrefillArgs a) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx == 0) {
    bool bad = a.cu_q[0] != 0 || a.cu_q[a.batch] != a.total_q;
    for (int b = 0; b < a.batch; ++b) {
      const int nb = a.cu_q[b + 1] - a.cu_q[b];
      const int L = a.seq_lens[b];
      if (nb < 0 || (nb > 0 && nb > L) || nb > a.max_q_len || a.cu_q[b] < 0 || a.cu_q[b + 1] > a.total_q)
        bad = true;
      if (!seq_len_ok(a, L)) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
    }
    if (bad) set_status(a.status, STARKV_DEV_BAD_QUERY_SPAN);
  }
  if (idx >= a.total_q * a.H * a.d) return;
  const int64_t rh = idx / a.d;
  const float l = a.ML[rh * 2 + 1];
  a.out[idx] = __float2bfloat16_rn(l > 0.f ? a.O[idx] / l : 0.f);
}

PrefillPlan plan_prefill_simt(const Ctx& c, int batch, int max_pages, int64_t total_q) {
  PrefillPlan p;
  const int max_len = max_pages * kPage;
  p.chunk = 512;
  if (max_len < p.chunk) p.chunk = ((max_len + 31) / 32) * 32;
  if (p.chunk < 32) p.chunk = 32;
  const size_t kvb = (size_t)batch * p.chunk * c.cfg.num_kv_heads * c.cfg.head_dim * sizeof(float);
  const size_t ob = (size_t)total_q * c.cfg.num_q_heads * c.cfg.head_dim * sizeof(float);
  const size_t mb = (size_t)total_q * c.cfg.num_q_heads * 2 * sizeof(float);
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  p.ws_bytes = 2 * al(kvb) + al(ob) + al(mb);
  return p;
}

cudaError_t launch_prefill_simt(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                                const int32_t* cu_q, const int32_t* block_table, const int32_t* seq_lens,
                                int batch, int max_pages, int64_t total_q, int max_q_len,
                                __nv_bfloat16* out, void* ws, const PrefillPlan& plan, cudaStream_t s) {
  if (batch == 0 || total_q == 0) return cudaSuccess;
  PrefillArgs a;
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
  a.batch = batch;
  a.max_pages = max_pages;
  a.chunk = plan.chunk;
  a.max_q_len = max_q_len;
  a.n_pages = cache.n_pages;
  a.total_q = total_q;
  a.q = q;
  a.cu_q = cu_q;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.k_codes = (const uint8_t*)cache.k_codes;
  a.v_codes = (const uint8_t*)cache.v_codes;
  a.k_meta = (const uint32_t*)cache.k_meta;
  a.v_meta = (const uint32_t*)cache.v_meta;
  a.Bk = c.Bk;
  a.Bv = c.Bv;
  a.rope = c.rope;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  char* w = (char*)ws;
  const size_t kvb = (size_t)batch * plan.chunk * a.h_kv * a.d * sizeof(float);
  a.Kx = (float*)w;
  w += al(kvb);
  a.Vx = (float*)w;
  w += al(kvb);
  a.O = (float*)w;
  w += al((size_t)total_q * a.H * a.d * sizeof(float));
  a.ML = (float*)w;
  a.out = out;
  a.status = c.status;
  const int64_t nqh = total_q * a.H;
  prefill_simt_init_kernel<<<(unsigned)((nqh + 255) / 256), 256, 0, s>>>(a);
  const int max_len = max_pages * kPage;
  for (int c0 = 0; c0 < max_len; c0 += plan.chunk) {
    prefill_simt_expand_kernel<<<dim3(plan.chunk / 32, a.h_kv, batch), 256, 0, s>>>(a, c0);
    prefill_simt_attn_kernel<<<dim3((max_q_len + 31) / 32, a.H, batch), 256, 0, s>>>(a, c0);
  }
  const int64_t tot = nqh * a.d;
  prefill_simt_finalize_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Path selection: the tensor-core kernels (prefill_tc.cu) for every shape they
// cover, the CUDA-core kernels above otherwise.
// ---------------------------------------------------------------------------
PrefillPlan plan_prefill(const Ctx& c, int batch, int max_pages, int64_t total_q) {
  return c.tc_prefill ? plan_prefill_tc(c, batch, max_pages, total_q) : plan_prefill_simt(c, batch, max_pages, total_q);
}

cudaError_t launch_prefill(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                           const int32_t* cu_q, const int32_t* block_table, const int32_t* seq_lens,
                           int batch, int max_pages, int64_t total_q, int max_q_len,
                           __nv_bfloat16* out, void* ws, const PrefillPlan& plan, cudaStream_t s) {
  if (c.tc_prefill)
    return launch_prefill_tc(c, cache, q, cu_q, block_table, seq_lens, batch, max_pages, total_q, max_q_len, out, ws,
                             plan, s);
  return launch_prefill_simt(c, cache, q, cu_q, block_table, seq_lens, batch, max_pages, total_q, max_q_len, out, ws,
                             plan, s);
}

}  // namespace starkv

// Tensor-core (tcgen05 / TMEM) decode attention over the packed latent cache.
//
// Source: "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression",
// Algorithm 2 steps 4-8 and section 5.3.  Three kernels:
//
//  A. scores: per (sequence, group of heads, 128-token tile)
//       G[t, (h,c)] = sum_k trig[pos_t, k] * W[(h,c), k]        (tensor cores)
//     where trig[p] = (cos(p th_0..), sin(p th_0..)) and W folds the rotated
//     query into the key up-projection B' (see decode.cu for the identity), so
//     G[t, (h, .)] . z_t is the RoPE'd score of head h against token t.  The
//     epilogue (one thread per token) takes that dot product directly on the
//     dequantised codes: sum_c (code_c s + zp) G_c = s sum_c code_c G_c + zp sum_c G_c.
//     Scores (log2 domain) and per-32-token maxima go to the workspace.
//  B. values: per (sequence, token split), all heads at once (the stacked
//       P Z_V product of section 5.3):  D[ch, h] += sum_t Z_v[t, ch] P[h, t]
//     with P = exp2(s - M_h) against the sequence-wide maximum M_h, so the
//     partial sums of every split share one reference and add up directly
//     (the softmax partition identity with a common maximum).  Z_v is
//     dequantised to fp16 by CUDA cores into shared memory; D lives in TMEM and
//     is added into a per-(sequence, head) fp32 accumulator at the end.
//  C. projection: o_h = (acc_h / l_h) B'_v[:, kv(h)]  (B'_v = H B_v, fp16).
//
// Every wait on an mbarrier is bounded; a time-out sets a status bit and the
// kernel winds down instead of spinning.
#include <float.h>

#include "internal.cuh"
#include "sm100.cuh"

namespace starkv {
using namespace sm100;

namespace {
constexpr int kT = 128;                 // tokens per key tile (MMA M)
constexpr int kPagesPerTile = kT / kPage;
constexpr int kEpiWarps = 8;
constexpr int kAThreads = (2 + kEpiWarps) * 32;
constexpr int kVT = 64;                 // tokens per value stage
constexpr int kVPages = kVT / kPage;
constexpr int kVStages = 3;
constexpr int kZBufs = 4;
constexpr int kVWarps = 8;
constexpr int kBThreads = (2 + kVWarps) * 32;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
}  // namespace

// ===========================================================================
// A. scores
// ===========================================================================
struct ScoreArgs {
  LatentGeom key;
  int H, h_kv, group, d, hpc, kvpc, ncols, HG;
  int max_pages, tiles_per_seq, tpad, max_position;
  int items_per_cta, total_items;
  int64_t n_pages;
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint8_t* k_codes;
  const uint32_t* k_meta;
  const float* Bk;     // [h_kv][r_k][d] fp32 B'_k
  const float2* rope;  // [max_position][d/2]
  float* S;            // [B][H][tpad]      scores, log2 domain
  float* Smax;         // [B][H][tpad/32]   maxima of 32-token blocks
  float* acc;          // [B][H][R] zeroed here for kernel B
  float* lsum;         // [B][H]    zeroed here
  int64_t acc_elems;   // B * H * R
  int64_t lsum_elems;  // B * H
  unsigned int* status;
  uint32_t off_trig, off_codes, off_meta, off_flags, off_q, off_bar;
  uint32_t trig_stage, codes_page, meta_page, codes_stage, meta_stage;
};

// TMEM columns of the score accumulators: two buffers of up to 256 columns.
constexpr uint32_t kScoreTmemCols = 512;

template <int RK>
__device__ __forceinline__ void tmem_load_row(uint32_t taddr, float (&G)[RK]) {
  uint32_t r[32];
  if constexpr (RK == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) G[i] = __uint_as_float(r[i]);
  } else {
#pragma unroll
    for (int h = 0; h < RK / 32; ++h) {
      tmem_ld32(taddr + h * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) G[h * 32 + i] = __uint_as_float(r[i]);
    }
  }
}

// sum_c z_hat_c G_c over one token's key latent in a staged page region.
template <int RK>
__device__ __forceinline__ float key_dot(const uint8_t* region, const uint32_t* meta, const LatentGeom& L, int t16,
                                         const float (&G)[RK]) {
  float score = 0.f;
  const int g = L.g;
  for (int gi = 0; gi < L.groups; ++gi) {
    const float2 sz = unpack_meta(meta[gi * kPage + t16]);
    float a = 0.f, gs = 0.f;
    for (int c = 0; c < g; ++c) {
      const float Gc = G[gi * g + c];
      a = fmaf((float)load_code(region, L, gi, t16, c), Gc, a);
      gs += Gc;
    }
    score = fmaf(sz.x, a, fmaf(sz.y, gs, score));
  }
  return score;
}

template <int RK>
__global__ void __launch_bounds__(kAThreads, 1)
    decode_scores_kernel(const __grid_constant__ CUtensorMap trig_map, const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* Wsm = sm;                                         // [ncols x d] K-major, 128B swizzle
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + a.off_bar);
  uint64_t* full = bar;        // [2] stage loaded (TMA + bulk)
  uint64_t* empty = bar + 2;   // [2] stage free (MMA commit + epilogue warps)
  uint64_t* tfull = bar + 4;   // [2] accumulator ready
  uint64_t* tempty = bar + 6;  // [2] accumulator drained
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 8);
  int* failed = reinterpret_cast<int*>(bar + 9);
  int* flags = reinterpret_cast<int*>(sm + a.off_flags);    // [2][8] page ids (-1 = invalid)
  float* qbuf = reinterpret_cast<float*>(sm + a.off_q);     // [hpc][d]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = a.d, half = d / 2;

  // zero kernel B's accumulators (grid-stride over all CTAs)
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < a.acc_elems; i += (int64_t)gridDim.x * blockDim.x)
    a.acc[i] = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < a.lsum_elems; i += (int64_t)gridDim.x * blockDim.x)
    a.lsum[i] = 0.f;

  if (warp == 1) tmem_alloc(tslot, kScoreTmemCols);
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kEpiWarps);
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiWarps);
    }
    *failed = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t idesc = make_idesc_f16(128, a.ncols, false, false);

  uint32_t it = 0;  // tiles through the pipeline so far (same count in every role)
  int item = blockIdx.x * a.items_per_cta;
  const int item_end = min(item + a.items_per_cta, a.total_items);
  while (item < item_end) {
    const int bhg = item / a.tiles_per_seq;
    const int b = bhg / a.HG, hg = bhg % a.HG;
    const int job_end = min(item_end, (bhg + 1) * a.tiles_per_seq);
    const int tile_lo = item - bhg * a.tiles_per_seq;
    const int tile_hi = job_end - bhg * a.tiles_per_seq;
    item = job_end;
    const int L = a.seq_lens[b];
    const bool bad_len = L < 0 || L > a.max_pages * kPage || L > a.max_position;
    const int n_tiles = bad_len ? 0 : (L + kT - 1) / kT;
    const int t0 = tile_lo, t1 = min(tile_hi, n_tiles);
    if (t0 >= t1) continue;
    if (*failed) break;
    const int h0 = hg * a.hpc;
    const int kv0 = h0 / a.group;
    // ---- W for this (sequence, head group): rotated query folded into B'
    {
      const int pos = L - 1;
      const float scale = kLog2e * rsqrtf((float)d);
      for (int e = tid; e < a.hpc * half; e += blockDim.x) {
        const int hl = e / half, i = e % half;
        const __nv_bfloat16* qv = a.q + ((int64_t)b * a.H + h0 + hl) * d;
        const float2 cs = a.rope[(int64_t)pos * half + i];
        const float x0 = __bfloat162float(qv[i]), x1 = __bfloat162float(qv[i + half]);
        qbuf[hl * d + i] = (x0 * cs.x - x1 * cs.y) * scale;
        qbuf[hl * d + i + half] = (x1 * cs.x + x0 * cs.y) * scale;
      }
      __syncthreads();
      for (int e = tid; e < a.ncols * d; e += blockDim.x) {
        const int n = e / d, k = e % d;
        const int hl = n / RK, c = n % RK;
        const int kv = (h0 + hl) / a.group;
        const int i = k < half ? k : k - half;
        const float* B = a.Bk + ((int64_t)kv * RK + c) * d;
        const float ba = B[i], bb = B[i + half];
        const float qa = qbuf[hl * d + i], qb = qbuf[hl * d + i + half];
        const float w = k < half ? fmaf(qa, ba, qb * bb) : fmaf(qb, ba, -qa * bb);
        *reinterpret_cast<__half*>(Wsm + sw128_kmajor_offset(n, k, a.ncols)) = __float2half_rn(w);
      }
      fence_async_smem();
      __syncthreads();
    }
    const int ntile = t1 - t0;
    if (warp == 0) {
      if (lane == 0) {
        // ---------------- producer ----------------
        for (int k = 0; k < ntile; ++k) {
          const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1)) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
            break;
          }
          const int j0 = (t0 + k) * kT;
          const int nval = min(kT, L - j0);
          const int np = (nval + kPage - 1) / kPage;
          uint32_t bytes = a.trig_stage;
          int* fl = flags + s * kPagesPerTile;
          for (int p = 0; p < kPagesPerTile; ++p) {
            int pid = -1;
            if (p < np) {
              pid = a.block_table[(int64_t)b * a.max_pages + j0 / kPage + p];
              if (pid < 0 || pid >= a.n_pages) {
                set_status(a.status, STARKV_DEV_BAD_PAGE);
                pid = -1;
              } else {
                bytes += a.codes_page + a.meta_page;
              }
            }
            fl[p] = pid;
          }
          mbar_arrive_expect_tx(&full[s], bytes);
          uint8_t* trig_dst = sm + a.off_trig + s * a.trig_stage;
          for (int sub = 0; sub < d / 64; ++sub) tma_load_2d(trig_dst + sub * 16384, &trig_map, sub * 64, j0, &full[s]);
          for (int p = 0; p < np; ++p) {
            const int pid = fl[p];
            if (pid < 0) continue;
            bulk_g2s(sm + a.off_codes + s * a.codes_stage + p * a.codes_page,
                     a.k_codes + ((int64_t)pid * a.h_kv + kv0) * a.key.region_bytes, a.codes_page, &full[s]);
            bulk_g2s(sm + a.off_meta + s * a.meta_stage + p * a.meta_page,
                     a.k_meta + ((int64_t)pid * a.h_kv + kv0) * a.key.groups * kPage, a.meta_page, &full[s]);
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------- MMA issuer ----------------
        for (int k = 0; k < ntile; ++k) {
          const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;
          if (!mbar_wait(&full[s], ph) || !mbar_wait(&tempty[s], ph ^ 1)) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
            break;
          }
          tc_fence_after();
          const uint32_t trig_addr = smem_u32(sm + a.off_trig + s * a.trig_stage);
          const uint32_t w_addr = smem_u32(Wsm);
          const uint32_t dt = tmem + s * 256;
          for (int ks = 0; ks < d / 16; ++ks) {
            const uint32_t sub = ks >> 2, koff = (ks & 3) * 32;
            const uint64_t ad = make_sdesc(trig_addr + sub * 16384 + koff, 16, 1024, 2);
            const uint64_t bd = make_sdesc(w_addr + sub * (a.ncols * 128) + koff, 16, 1024, 2);
            mma_f16(dt, ad, bd, idesc, ks > 0);
          }
          mma_commit(&tfull[s]);
          mma_commit(&empty[s]);
        }
      }
    } else {
      // ---------------- epilogue: one thread per token ----------------
      const int q4 = warp & 3, hhalf = (warp - 2) >> 2;
      const int t = q4 * 32 + lane;
      const int t16 = t % kPage, p = t / kPage;
      const int hper = a.hpc / 2;
      for (int k = 0; k < ntile; ++k) {
        const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;
        if (!mbar_wait(&tfull[s], ph) || !mbar_wait(&full[s], ph)) {
          if (lane == 0) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
          }
          break;
        }
        tc_fence_after();
        const int tile = t0 + k;
        const int j = tile * kT + t;
        const int pid = flags[s * kPagesPerTile + p];
        const bool valid = j < L && pid >= 0;
        const uint8_t* cstage = sm + a.off_codes + s * a.codes_stage + p * a.codes_page;
        const uint32_t* mstage = reinterpret_cast<const uint32_t*>(sm + a.off_meta + s * a.meta_stage + p * a.meta_page);
        for (int hh = 0; hh < hper; ++hh) {
          const int hl = hhalf * hper + hh;
          const int h = h0 + hl;
          const int kvl = h / a.group - kv0;
          float G[RK];
          tmem_load_row<RK>(tmem + s * 256 + hl * RK + ((uint32_t)(q4 * 32) << 16), G);
          float score = -INFINITY;
          if (valid)
            score = key_dot<RK>(cstage + kvl * a.key.region_bytes, mstage + kvl * a.key.groups * kPage, a.key, t16, G);
          if (j < L) a.S[((int64_t)b * a.H + h) * a.tpad + j] = score;
          const float m = warp_max(score);
          if (lane == 0) a.Smax[((int64_t)b * a.H + h) * (a.tpad / 32) + tile * 4 + q4] = m;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[s]);
          mbar_arrive(&empty[s]);
        }
      }
    }
    it += ntile;
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kScoreTmemCols);
  }
}

// ===========================================================================
// B. values
// ===========================================================================
struct ValueArgs {
  LatentGeom val;
  int H, N, R, MT, d;
  int max_pages, tpad, splits, stages_total, max_position;
  int64_t n_pages;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint8_t* v_codes;
  const uint32_t* v_meta;
  const float* S;
  const float* Smax;
  float* acc;    // [B][H][R]
  float* lsum;   // [B][H]
  unsigned int* status;
  uint32_t off_codes, off_meta, off_z, off_p, off_flags, off_m, off_l, off_bar;
  uint32_t codes_page, meta_page, codes_stage, meta_stage, tmem_cols;
};

constexpr uint32_t kZBytes = kVT * 128 * 2;   // one M tile of Z: 64 tokens x 128 channels fp16
constexpr uint32_t kPBytes = 64 * kVT * 2;    // P buffer: up to 64 heads x 64 tokens fp16

__global__ void __launch_bounds__(kBThreads, 1) decode_values_kernel(const ValueArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + a.off_bar);
  uint64_t* cfull = bar;                         // [kVStages]
  uint64_t* cempty = cfull + kVStages;           // [kVStages]
  uint64_t* zfull = cempty + kVStages;           // [kZBufs]
  uint64_t* zempty = zfull + kZBufs;             // [kZBufs]
  uint64_t* pfull = zempty + kZBufs;             // [2]
  uint64_t* pempty = pfull + 2;                  // [2]
  uint64_t* dfull = pempty + 2;                  // [1]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dfull + 1);
  int* failed = reinterpret_cast<int*>(dfull + 2);
  int* flags = reinterpret_cast<int*>(sm + a.off_flags);   // [kVStages][kVPages]
  float* Mh = reinterpret_cast<float*>(sm + a.off_m);      // [N]
  float* Lh = reinterpret_cast<float*>(sm + a.off_l);      // [N]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const LatentGeom& V = a.val;

  int L = a.seq_lens[b];
  const bool bad_len = L < 0 || L > a.max_pages * kPage || L > a.max_position;
  if (bad_len) {
    if (split == 0 && tid == 0) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
    L = 0;
  }
  const int st_lo = (int)((int64_t)split * a.stages_total / a.splits);
  const int st_hi0 = (int)((int64_t)(split + 1) * a.stages_total / a.splits);
  const int st_hi = min(st_hi0, (L + kVT - 1) / kVT);
  const int nst = st_hi - st_lo;
  if (nst <= 0) return;  // nothing of this sequence here (uniform across the CTA)

  if (warp == 1) tmem_alloc(tslot, a.tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], kVWarps);
    }
    for (int s = 0; s < kZBufs; ++s) {
      mbar_init(&zfull[s], kVWarps);
      mbar_init(&zempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&pfull[s], kVWarps);
      mbar_init(&pempty[s], 1);
    }
    mbar_init(dfull, 1);
    *failed = 0;
    fence_mbar_init();
  }
  // sequence-wide maxima per head (common reference of every split), l = 0,
  // P buffers zeroed once (rows >= H stay zero)
  for (int h = tid; h < a.N; h += blockDim.x) {
    float m = -INFINITY;
    if (h < a.H) {
      const int nblk = (L + 31) / 32;
      const float* sm_row = a.Smax + ((int64_t)b * a.H + h) * (a.tpad / 32);
      for (int i = 0; i < nblk; ++i) m = fmaxf(m, sm_row[i]);
    }
    Mh[h] = m;
    Lh[h] = 0.f;
  }
  for (int i = tid; i < (int)(2 * kPBytes / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(sm + a.off_p)[i] = make_uint4(0, 0, 0, 0);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: value codes + metadata of 4 pages per stage
      for (int k = 0; k < nst; ++k) {
        const int cs = k % kVStages;
        const uint32_t ph = (k / kVStages) & 1;
        if (!mbar_wait(&cempty[cs], ph ^ 1)) {
          set_status(a.status, kDevWaitTimeout);
          *failed = 1;
          break;
        }
        const int j0 = (st_lo + k) * kVT;
        const int nval = min(kVT, L - j0);
        const int np = (nval + kPage - 1) / kPage;
        int* fl = flags + cs * kVPages;
        uint32_t bytes = 0;
        for (int p = 0; p < kVPages; ++p) {
          int pid = -1;
          if (p < np) {
            pid = a.block_table[(int64_t)b * a.max_pages + j0 / kPage + p];
            if (pid < 0 || pid >= a.n_pages) {
              set_status(a.status, STARKV_DEV_BAD_PAGE);
              pid = -1;
            } else {
              bytes += a.codes_page + a.meta_page;
            }
          }
          fl[p] = pid;
        }
        mbar_arrive_expect_tx(&cfull[cs], bytes);
        for (int p = 0; p < np; ++p) {
          const int pid = fl[p];
          if (pid < 0) continue;
          bulk_g2s(sm + a.off_codes + cs * a.codes_stage + p * a.codes_page,
                   a.v_codes + (int64_t)pid * V.region_bytes, a.codes_page, &cfull[cs]);
          bulk_g2s(sm + a.off_meta + cs * a.meta_stage + p * a.meta_page,
                   a.v_meta + (int64_t)pid * V.groups * kPage, a.meta_page, &cfull[cs]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: D[mt] += Z[mt]^T P^T
      const uint32_t idesc = make_idesc_f16(128, a.N, true, false);
      uint32_t zc = 0;
      bool ok = true;
      for (int k = 0; k < nst && ok; ++k) {
        const int ps = k & 1;
        if (!mbar_wait(&pfull[ps], (k >> 1) & 1)) {
          ok = false;
          break;
        }
        const uint32_t p_addr = smem_u32(sm + a.off_p + ps * kPBytes);
        for (int mt = 0; mt < a.MT; ++mt, ++zc) {
          const uint32_t zs = zc % kZBufs, zph = (zc / kZBufs) & 1;
          if (!mbar_wait(&zfull[zs], zph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t z_addr = smem_u32(sm + a.off_z + zs * kZBytes);
          for (int ks = 0; ks < kVT / 16; ++ks) {
            const uint64_t ad = make_sdesc(z_addr + ks * 4096, 1024, 2048, 2);
            const uint64_t bd = make_sdesc(p_addr + ks * 32, 16, 1024, 2);
            mma_f16(tmem + mt * a.N, ad, bd, idesc, (k > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&zempty[zs]);
        }
        if (ok) mma_commit(&pempty[ps]);
      }
      if (!ok) {
        set_status(a.status, kDevWaitTimeout);
        *failed = 1;
      }
      mma_commit(dfull);
    }
  } else {
    // ---------------- P and Z producers (CUDA cores), then the accumulator drain
    const int wt = tid - 64;  // 0..255
    uint32_t zc = 0;
    bool ok = true;
    for (int k = 0; k < nst && ok; ++k) {
      const int cs = k % kVStages;
      const int ps = k & 1;
      if (!mbar_wait(&cfull[cs], (k / kVStages) & 1) || !mbar_wait(&pempty[ps], ((k >> 1) & 1) ^ 1)) {
        ok = false;
        break;
      }
      const int j0 = (st_lo + k) * kVT;
      const int* fl = flags + cs * kVPages;
      // P[h][t] = exp2(s - M_h) as fp16, K-major (row = head, 64 tokens); one item
      // = 8 consecutive tokens of one head; l sums the fp16 values the MMA uses
      uint8_t* pbuf = sm + a.off_p + ps * kPBytes;
      for (int e = wt; e < a.H * (kVT / 8); e += kVWarps * 32) {
        const int h = e / (kVT / 8), t0 = (e % (kVT / 8)) * 8;
        uint32_t w4[4];
        float lsum8 = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float pv[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int t = t0 + 2 * u + v;
            const int j = j0 + t;
            float p = 0.f;
            if (j < L && fl[t / kPage] >= 0) {
              const float sc = a.S[((int64_t)b * a.H + h) * a.tpad + j];
              if (sc != -INFINITY) p = exp2f(sc - Mh[h]);
            }
            pv[v] = p;
          }
          const __half2 h2 = __floats2half2_rn(pv[0], pv[1]);
          lsum8 += __low2float(h2) + __high2float(h2);
          w4[u] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(pbuf + sw128_kmajor_offset(h, t0, 64)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        atomicAdd(&Lh[h], lsum8);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[ps]);
      // Z tiles: 64 tokens x 128 channels, MN-major (channels contiguous), fp16
      const int t = wt >> 2, qq = wt & 3;
      const int j = j0 + t;
      const int pg = t / kPage, t16 = t % kPage;
      const bool tvalid = j < L && fl[pg] >= 0;
      const uint8_t* region = sm + a.off_codes + cs * a.codes_stage + pg * a.codes_page;
      const uint32_t* meta = reinterpret_cast<const uint32_t*>(sm + a.off_meta + cs * a.meta_stage + pg * a.meta_page);
      for (int mt = 0; mt < a.MT; ++mt, ++zc) {
        const uint32_t zs = zc % kZBufs, zph = (zc / kZBufs) & 1;
        if (!mbar_wait(&zempty[zs], zph ^ 1)) {
          ok = false;
          break;
        }
        uint8_t* zbuf = sm + a.off_z + zs * kZBytes;
        for (int c8 = 0; c8 < 4; ++c8) {
          const int m = qq * 32 + c8 * 8;          // channel within the tile
          const int ch0 = mt * 128 + m;
          uint32_t w4[4] = {0, 0, 0, 0};
          if (tvalid && ch0 < V.r) {
            const int gi = ch0 / V.g;
            const float2 sz = unpack_meta(meta[gi * kPage + t16]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = ch0 % V.g + 2 * u;
              const float z0 = __fmaf_rn((float)load_code(region, V, gi, t16, c), sz.x, sz.y);
              const float z1 = __fmaf_rn((float)load_code(region, V, gi, t16, c + 1), sz.x, sz.y);
              const __half2 h2 = __floats2half2_rn(z0, z1);
              w4[u] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          }
          *reinterpret_cast<uint4*>(zbuf + sw128_mnmajor_offset(t, m, 2)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&zfull[zs]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[cs]);
    }
    if (!ok && lane == 0) {
      set_status(a.status, kDevWaitTimeout);
      *failed = 1;
    }
    // drain D (TMEM) into the per-(sequence, head) accumulator
    if (mbar_wait(dfull, 0)) {
      tc_fence_after();
      const int q4 = warp & 3, hsel = (warp - 2) >> 2;
      for (int mt = hsel; mt < a.MT; mt += 2) {
        const int ch = mt * 128 + q4 * 32 + lane;
        for (int c0 = 0; c0 < a.N; c0 += 16) {
          uint32_t r[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
              "[%16];"
              : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                "=r"(r[15])
              : "r"(tmem + mt * a.N + c0 + ((uint32_t)(q4 * 32) << 16)));
          tmem_ld_wait();
          if (ch < a.R) {
            for (int i = 0; i < 16; ++i) {
              const int h = c0 + i;
              if (h < a.H) atomicAdd(&a.acc[((int64_t)b * a.H + h) * a.R + ch], __uint_as_float(r[i]));
            }
          }
        }
      }
    } else if (lane == 0) {
      set_status(a.status, kDevWaitTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  for (int h = tid; h < a.H; h += blockDim.x) atomicAdd(&a.lsum[(int64_t)b * a.H + h], Lh[h]);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

// ===========================================================================
// C. projection: o_h = (acc_h / l_h) B'_v[:, kv(h)]
// ===========================================================================
struct ProjArgs {
  int H, h_kv, group, d, R;
  const float* acc;
  const float* lsum;
  const float* Smax;
  const int32_t* seq_lens;
  int tpad, max_pages, max_position;
  const __half* Bv16;
  __nv_bfloat16* out;
};

__global__ void __launch_bounds__(256) decode_project_kernel(const ProjArgs a) {
  extern __shared__ float psm[];
  float* olat = psm;            // [R]
  float* red = psm + a.R;       // [256]
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int kv = h / a.group;
  const float l = a.lsum[(int64_t)b * a.H + h];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  for (int ch = tid; ch < a.R; ch += 256) olat[ch] = a.acc[((int64_t)b * a.H + h) * a.R + ch] * inv;
  __syncthreads();
  const int nh = 256 / a.d;
  const int col = tid % a.d, sub = tid / a.d;
  const int ldb = a.h_kv * a.d;
  float o = 0.f;
  for (int ch = sub; ch < a.R; ch += nh) o = fmaf(olat[ch], __half2float(a.Bv16[(int64_t)ch * ldb + kv * a.d + col]), o);
  red[sub * a.d + col] = o;
  __syncthreads();
  if (sub == 0) {
    float t = 0.f;
    for (int k = 0; k < nh; ++k) t += red[k * a.d + col];
    a.out[((int64_t)b * a.H + h) * a.d + col] = __float2bfloat16_rn(t);
  }
}

// ===========================================================================
// host side
// ===========================================================================
bool tc_decode_supported(const starkv_config& cfg) {
  const int rk = cfg.rank_k;
  if (rk != 16 && rk != 32 && rk != 64) return false;
  const int hpc = (256 / rk) < cfg.num_q_heads ? 256 / rk : cfg.num_q_heads;
  const int group = cfg.num_q_heads / cfg.num_kv_heads;
  if (cfg.num_q_heads % hpc != 0 || hpc % 2 != 0) return false;
  if (hpc % group != 0 && group % hpc != 0) return false;
  if (group > hpc) return false;  // a CTA's heads must cover whole KV heads
  if (cfg.num_q_heads > 64) return false;
  return true;
}

namespace {
int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

struct TcLayout {
  int hpc, kvpc, ncols, HG, tiles_per_seq, tpad, splits, stages_total, N, MT;
  size_t off_S, off_Smax, off_acc, off_l, ws;
};

TcLayout tc_layout(const Ctx& c, int batch, int max_pages) {
  TcLayout t;
  const starkv_config& f = c.cfg;
  t.hpc = (256 / f.rank_k) < f.num_q_heads ? 256 / f.rank_k : f.num_q_heads;
  t.kvpc = t.hpc / c.group;
  t.ncols = t.hpc * f.rank_k;
  t.HG = f.num_q_heads / t.hpc;
  t.tiles_per_seq = (max_pages * kPage + kT - 1) / kT;
  t.tpad = t.tiles_per_seq * kT;
  t.stages_total = t.tpad / kVT;
  int splits = (sm_count() + batch - 1) / (batch > 0 ? batch : 1);
  if (splits > t.stages_total) splits = t.stages_total;
  if (splits < 1) splits = 1;
  t.splits = splits;
  t.N = ((f.num_q_heads + 15) / 16) * 16;
  t.MT = (f.rank_v + 127) / 128;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t o = 0;
  t.off_S = o;
  o += al((size_t)batch * f.num_q_heads * t.tpad * 4);
  t.off_Smax = o;
  o += al((size_t)batch * f.num_q_heads * (t.tpad / 32) * 4);
  t.off_acc = o;
  o += al((size_t)batch * f.num_q_heads * f.rank_v * 4);
  t.off_l = o;
  o += al((size_t)batch * f.num_q_heads * 4);
  t.ws = o;
  return t;
}
}  // namespace

DecodePlan plan_decode_tc(const Ctx& c, int batch, int max_pages) {
  DecodePlan p;
  const TcLayout t = tc_layout(c, batch, max_pages);
  p.splits = t.splits;
  p.pages_per_split = 0;
  p.ws_bytes = t.ws;
  return p;
}

__global__ void to_half_kernel(const float* __restrict__ x, __half* __restrict__ y, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __float2half_rn(x[i]);
}

// fp16 copy of B'_v for the projection kernel.
cudaError_t launch_prepare_tc_factors(const Ctx& c, cudaStream_t s) {
  const int64_t n = (int64_t)c.cfg.rank_v * c.cfg.num_kv_heads * c.cfg.head_dim;
  to_half_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(c.Bv, c.Bv16, n);
  return cudaGetLastError();
}

template <int RK>
static cudaError_t launch_scores(const Ctx& c, const ScoreArgs& a, int grid, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_scores_kernel<RK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_scores_kernel<RK><<<grid, kAThreads, smem, s>>>(c.trig_map, a);
  return cudaGetLastError();
}

cudaError_t launch_decode_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                             const int32_t* block_table, const int32_t* seq_lens, int batch, int max_pages,
                             __nv_bfloat16* out, void* ws, const DecodePlan&, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  const starkv_config& f = c.cfg;
  const TcLayout t = tc_layout(c, batch, max_pages);
  char* w = (char*)ws;
  float* S = (float*)(w + t.off_S);
  float* Smax = (float*)(w + t.off_Smax);
  float* acc = (float*)(w + t.off_acc);
  float* lsum = (float*)(w + t.off_l);
  const int d = f.head_dim;

  // ---------------- A: scores
  ScoreArgs A;
  A.key = c.key;
  A.H = f.num_q_heads;
  A.h_kv = f.num_kv_heads;
  A.group = c.group;
  A.d = d;
  A.hpc = t.hpc;
  A.kvpc = t.kvpc;
  A.ncols = t.ncols;
  A.HG = t.HG;
  A.max_pages = max_pages;
  A.tiles_per_seq = t.tiles_per_seq;
  A.tpad = t.tpad;
  A.max_position = f.max_position;
  A.total_items = batch * t.HG * t.tiles_per_seq;
  int ctas = sm_count();
  if (ctas > A.total_items) ctas = A.total_items;
  A.items_per_cta = (A.total_items + ctas - 1) / ctas;
  ctas = (A.total_items + A.items_per_cta - 1) / A.items_per_cta;
  A.n_pages = cache.n_pages;
  A.q = q;
  A.block_table = block_table;
  A.seq_lens = seq_lens;
  A.k_codes = (const uint8_t*)cache.k_codes;
  A.k_meta = (const uint32_t*)cache.k_meta;
  A.Bk = c.Bk;
  A.rope = c.rope;
  A.S = S;
  A.Smax = Smax;
  A.acc = acc;
  A.lsum = lsum;
  A.acc_elems = (int64_t)batch * f.num_q_heads * f.rank_v;
  A.lsum_elems = (int64_t)batch * f.num_q_heads;
  A.status = c.status;
  A.trig_stage = kT * d * 2;
  A.codes_page = t.kvpc * c.key.region_bytes;
  A.meta_page = t.kvpc * c.key.groups * kPage * 4;
  A.codes_stage = kPagesPerTile * A.codes_page;
  A.meta_stage = kPagesPerTile * A.meta_page;
  {
    uint32_t o = (uint32_t)t.ncols * d * 2;  // W
    o = (o + 1023) / 1024 * 1024;
    A.off_trig = o;
    o += 2 * A.trig_stage;
    A.off_codes = o;
    o += 2 * A.codes_stage;
    A.off_meta = o;
    o += 2 * A.meta_stage;
    A.off_flags = o;
    o += 2 * kPagesPerTile * 4;
    A.off_q = (o + 15) / 16 * 16;
    o = A.off_q + t.hpc * d * 4;
    A.off_bar = (o + 15) / 16 * 16;
    o = A.off_bar + 16 * 8;
    const size_t smem = o + 1024;  // alignment slack
    cudaError_t e;
    switch (f.rank_k) {
      case 16: e = launch_scores<16>(c, A, ctas, smem, s); break;
      case 32: e = launch_scores<32>(c, A, ctas, smem, s); break;
      default: e = launch_scores<64>(c, A, ctas, smem, s); break;
    }
    if (e != cudaSuccess) return e;
  }

  // ---------------- B: values
  ValueArgs B;
  B.val = c.val;
  B.H = f.num_q_heads;
  B.N = t.N;
  B.R = f.rank_v;
  B.MT = t.MT;
  B.d = d;
  B.max_pages = max_pages;
  B.tpad = t.tpad;
  B.splits = t.splits;
  B.stages_total = t.stages_total;
  B.max_position = f.max_position;
  B.n_pages = cache.n_pages;
  B.block_table = block_table;
  B.seq_lens = seq_lens;
  B.v_codes = (const uint8_t*)cache.v_codes;
  B.v_meta = (const uint32_t*)cache.v_meta;
  B.S = S;
  B.Smax = Smax;
  B.acc = acc;
  B.lsum = lsum;
  B.status = c.status;
  B.codes_page = c.val.region_bytes;
  B.meta_page = c.val.groups * kPage * 4;
  B.codes_stage = kVPages * B.codes_page;
  B.meta_stage = kVPages * B.meta_page;
  uint32_t cols = 32;
  while (cols < (uint32_t)(t.MT * t.N)) cols <<= 1;
  B.tmem_cols = cols;
  {
    uint32_t o = 0;
    B.off_z = o;
    o += kZBufs * kZBytes;
    B.off_p = o;
    o += 2 * kPBytes;
    B.off_codes = o;
    o += kVStages * B.codes_stage;
    B.off_meta = o;
    o += kVStages * B.meta_stage;
    B.off_flags = o;
    o += kVStages * kVPages * 4;
    B.off_m = (o + 15) / 16 * 16;
    o = B.off_m + t.N * 4;
    B.off_l = o;
    o += t.N * 4;
    B.off_bar = (o + 15) / 16 * 16;
    o = B.off_bar + 32 * 8;
    const size_t smem = o + 1024;
    cudaError_t e = cudaFuncSetAttribute(decode_values_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_values_kernel<<<dim3(t.splits, batch), kBThreads, smem, s>>>(B);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  // ---------------- C: projection
  ProjArgs P;
  P.H = f.num_q_heads;
  P.h_kv = f.num_kv_heads;
  P.group = c.group;
  P.d = d;
  P.R = f.rank_v;
  P.acc = acc;
  P.lsum = lsum;
  P.Smax = Smax;
  P.seq_lens = seq_lens;
  P.tpad = t.tpad;
  P.max_pages = max_pages;
  P.max_position = f.max_position;
  P.Bv16 = c.Bv16;
  P.out = out;
  const size_t psmem = (size_t)(f.rank_v + 256) * 4;
  decode_project_kernel<<<dim3(f.num_q_heads, batch), 256, psmem, s>>>(P);
  return cudaGetLastError();
}

}  // namespace starkv

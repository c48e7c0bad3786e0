// Tensor-core (tcgen05 / TMEM) causal chunk attention (prefill) over the packed
// latent cache.
//
// Source: "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression",
// the chunked form of Algorithm 2 (key tiles dequantised and re-expanded, RoPE
// at each position, softmax, values), with section 5.1 / eq. 9's
// reconstruction bill deciding where the re-expansion happens: with thousands
// of queries per sequence, aggregating P Z_v in the latent costs
// queries x heads x T x R multiply-adds, whereas re-expanding the values costs
// T x h_kv x R x d_h once per position.  So each (position, KV head) is
// re-expanded exactly once, and the attention then runs on the re-expanded
// tiles.  Two kernels:
//
//  A. expand: per (128-position tile, pair of KV heads, sequence)
//       K~_h = RoPE(Z^_k,h B'_k,h)      (A = dequantised key latents, K = r_k)
//       V_h  = Z^_v B'_v[:, h]          (A = dequantised value latents, K = R)
//     on tcgen05 with fp32 accumulators in TMEM; the latents are dequantised
//     by CUDA cores straight into the MMA's shared-memory operand tiles, the
//     up-projections arrive by TMA.  The epilogue applies RoPE in registers and
//     writes fp16 rows of K~ and V (zeros past the sequence's length).
//  B. attention: per (128-query tile, query head, sequence), flash-style:
//       S = Q K~^T into TMEM (double-buffered), an online softmax in
//       registers (one thread per query row), P to shared memory as fp16, and
//       O += P V into TMEM.  (m, l, O) stay on chip for the whole key loop.
//       The running maximum is moved only when it grows by more than 2^8, and
//       then O is rescaled in TMEM; O and l always share one reference, so the
//       result is exact in real arithmetic (p <= 256 keeps fp16 P in range).
//
// Every wait on an mbarrier is bounded; a time-out sets a status bit and the
// kernel winds down instead of spinning.
#include <float.h>

#include "internal.cuh"
#include "latent_tc.cuh"
#include "sm100.cuh"

namespace starkv {
using namespace sm100;

namespace {
constexpr int kTile = 128;                 // positions per tile (keys and queries)
constexpr int kQThreads = 192;             // attention kernel: producer, MMA, 4 softmax warps
constexpr float kLog2eQ = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;        // move the running maximum when it grows by more than 2^8
constexpr uint32_t kSub = 16384;           // one 64-column sub-tile of a 128-row fp16 tile

__device__ __forceinline__ uint8_t* align1024p(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
}  // namespace

// ===========================================================================
// A. expand
// ===========================================================================
struct ExpandArgs {
  LatentGeom key, val;
  int h_kv, d, HP, max_pages, max_position, tpad;
  int64_t n_pages;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint32_t* k_meta;
  const uint32_t* v_meta;
  const float2* rope;  // [max_position][d/2] (cos, sin)
  __half* Kx;          // [B][h_kv][tpad][d] RoPE'd keys
  __half* Vx;          // [B][h_kv][tpad][d] values
  unsigned int* status;
  // shared-memory layout (bytes from the 1024-aligned base)
  uint32_t off_ak, off_bk, off_kc, off_av, off_bv, off_vc, off_bar;
  uint32_t bk_head, bv_stage;
  uint32_t kc_codes, kc_page;      // key codes of one page of one head (bytes); a page's codes + meta pitch
  uint32_t vc_codes_max, vc_page;  // value codes of one chunk of one page (at most); codes + meta pitch
};

constexpr int kXWarps = 10;        // 8 dequant/epilogue warps, a copy warp, an MMA warp
constexpr int kXStages = 4;        // value code stages
constexpr int kXThreadsW = kXWarps * 32;

// Bytes of value group tiles [4c, 4c + 4) of a page region and their offset.
__device__ __forceinline__ void value_chunk_span(const LatentGeom& V, int c, uint32_t& off, uint32_t& bytes) {
  const int g0 = 4 * c;
  off = (uint32_t)tile_offset(V, g0);
  bytes = (uint32_t)tile_offset(V, g0 + 4) - off;
}

// grid (tpad / 128, ceil(h_kv / HP), B), 320 threads:
//   warps 0..7  dequantise latents from the staged pages into the MMA's A tiles,
//               then the epilogue (two warps per TMEM lane quarter)
//   warp 8      copies: the tile's key pages, then per 64-channel value chunk the
//               8 pages' code tiles and metadata (one lane per bulk copy), and the
//               B'_k / B'_v tiles by TMA
//   warp 9      one thread issues every tcgen05 MMA
//   TMEM columns [0, HP d): V accumulators; [256, 256 + HP d): K accumulators.
__global__ void __launch_bounds__(kXThreadsW, 1)
    prefill_expand_kernel(const __grid_constant__ CUtensorMap bk_map, const __grid_constant__ CUtensorMap bv_map,
                          const ExpandArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024p(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + a.off_bar);
  uint64_t* kfull = bar;                    // key pages + B'_k landed
  uint64_t* kready = bar + 1;               // key A tiles written (8 warps)
  uint64_t* cfull = bar + 2;                // [kXStages] value code stage landed
  uint64_t* cempty = cfull + kXStages;      // [kXStages] value code stage read (8 warps)
  uint64_t* bfull = cempty + kXStages;      // [2] B'_v chunk landed
  uint64_t* afull = bfull + 2;              // [2] value A tile written (8 warps)
  uint64_t* aempty = afull + 2;             // [2] MMAs of a chunk done (A tile and B'_v slot free)
  uint64_t* alldone = aempty + 2;           // every MMA done
  uint32_t* tslot = reinterpret_cast<uint32_t*>(alldone + 1);
  int* pg = reinterpret_cast<int*>(alldone + 2);  // [8] page ids of the tile (-1: none)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, kv0 = blockIdx.y * a.HP, b = blockIdx.z;
  const int nh = min(a.HP, a.h_kv - kv0);
  const int d = a.d, nsub = d / 64;
  const int rk = a.key.r;
  const LatentGeom& V = a.val;
  const int nchunk = V.r / 64;
  // first kernel of the call: its inputs may come from any earlier kernel
  pdl_wait();
  pdl_launch_dependents();
  const int L = a.seq_lens[b];
  if (L < 0 || L > a.max_pages * kPage || L > a.max_position) {
    if (tile == 0 && blockIdx.y == 0 && tid == 0) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
    return;
  }
  if (tile * kTile >= L) return;
  if (warp == 9) tmem_alloc(tslot, 512);
  if (tid == 0) {
    mbar_init(kfull, 1);
    mbar_init(kready, 8);
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 8);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&afull[s], 8);
      mbar_init(&aempty[s], 1);
    }
    mbar_init(alldone, 1);
    fence_mbar_init();
  }
  if (tid < kTile / kPage) {
    const int p0 = tile * kTile + tid * kPage;
    int pid = -1;
    if (p0 < L) {
      pid = a.block_table[(int64_t)b * a.max_pages + p0 / kPage];
      if (pid < 0 || pid >= a.n_pages) {
        set_status(a.status, STARKV_DEV_BAD_PAGE);
        pid = -1;
      }
    }
    pg[tid] = pid;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  uint8_t* Ak = sm + a.off_ak;
  uint8_t* Bk = sm + a.off_bk;
  uint8_t* Kc = sm + a.off_kc;
  uint8_t* Av = sm + a.off_av;
  uint8_t* Bv = sm + a.off_bv;
  uint8_t* Vc = sm + a.off_vc;
  const uint32_t vstage = 8 * a.vc_page;
  bool ok = true;

  if (warp == 8) {
    // ---------------- copies ----------------
    const int npg = __popc(__ballot_sync(0xffffffffu, lane < 8 && pg[lane < 8 ? lane : 0] >= 0));
    // key pages of the CTA's heads: codes (padded region) and metadata, one lane per copy
    const uint32_t kmeta = a.kc_page - a.kc_codes;  // 0 for fp16 latents
    if (lane == 0) {
      mbar_arrive_expect_tx(kfull, (uint32_t)(npg * nh) * a.kc_page + (uint32_t)(nh * nsub * rk * 128));
      for (int hh = 0; hh < nh; ++hh)
        for (int i = 0; i < nsub; ++i)
          tma_load_2d(Bk + hh * a.bk_head + i * rk * 128, &bk_map, i * 64, (kv0 + hh) * rk, kfull);
    }
    __syncwarp();
    for (int e = lane; e < 2 * 8 * nh; e += 32) {
      const int p = (e >> 1) % 8, hh = (e >> 1) / 8;
      const int pid = pg[p];
      if (pid < 0) continue;
      const int64_t reg = (int64_t)pid * a.h_kv + kv0 + hh;
      uint8_t* dst = Kc + (hh * 8 + p) * a.kc_page;
      if ((e & 1) == 0)
        bulk_g2s(dst, a.k_codes + reg * a.key.region_bytes, a.kc_codes, kfull);
      else if (kmeta)
        bulk_g2s(dst + a.kc_codes, a.k_meta + reg * a.key.groups * kPage, kmeta, kfull);
    }
    // value chunks
    for (int c = 0; c < nchunk; ++c) {
      const int s = c % kXStages;
      const uint32_t ph = (c / kXStages) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&cempty[s], ph ^ 1))) {
        ok = false;
        break;
      }
      uint32_t coff, cbytes;
      value_chunk_span(V, c, coff, cbytes);
      const uint32_t vmeta = V.fp16 ? 0u : 4 * kPage * 4;
      if (lane == 0) mbar_arrive_expect_tx(&cfull[s], (uint32_t)npg * (cbytes + vmeta));
      __syncwarp();
      if (lane < 16) {
        const int p = lane >> 1;
        const int pid = pg[p];
        if (pid >= 0) {
          uint8_t* dst = Vc + s * vstage + p * a.vc_page;
          if ((lane & 1) == 0)
            bulk_g2s(dst, a.v_codes + (int64_t)pid * V.region_bytes + coff, cbytes, &cfull[s]);
          else if (vmeta)
            bulk_g2s(dst + a.vc_codes_max, a.v_meta + ((int64_t)pid * V.groups + 4 * c) * kPage, vmeta, &cfull[s]);
        }
      }
      const int bs = c & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&aempty[bs], ((c >> 1) & 1) ^ 1))) {
        ok = false;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bfull[bs], (uint32_t)(nh * nsub) * 8192u);
        for (int i = 0; i < nh * nsub; ++i)
          tma_load_2d(Bv + bs * a.bv_stage + i * 8192, &bv_map, kv0 * d + i * 64, c * 64, &bfull[bs]);
      }
      __syncwarp();
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_k = make_idesc_f16(128, d, false, true);
      const uint32_t idesc_v = make_idesc_f16(128, nh * d, false, true);
      if (mbar_wait(kfull, 0) && mbar_wait(kready, 0)) {
        tc_fence_after();
        for (int hh = 0; hh < nh; ++hh)
          for (int ks = 0; ks < rk / 16; ++ks)
            mma_f16(tmem + 256 + hh * d, make_sdesc(smem_u32(Ak + hh * kTile * 128) + ks * 32, 16, 1024, 2),
                    make_sdesc(smem_u32(Bk + hh * a.bk_head) + ks * 2048, rk * 128, 1024, 2), idesc_k, ks > 0);
      } else {
        ok = false;
      }
      for (int c = 0; ok && c < nchunk; ++c) {
        const int bs = c & 1;
        const uint32_t ph = (c >> 1) & 1;
        if (!mbar_wait(&afull[bs], ph) || !mbar_wait(&bfull[bs], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aa = smem_u32(Av + bs * (kTile * 128));
        const uint32_t ba = smem_u32(Bv + bs * a.bv_stage);
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem, make_sdesc(aa + ks * 32, 16, 1024, 2), make_sdesc(ba + ks * 2048, 8192, 1024, 2), idesc_v,
                  (c > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&aempty[bs]);
      }
      mma_commit(alldone);  // arrives once every MMA issued above has completed
    }
  } else {
    // ---------------- dequantisation (warps 0..7) ----------------
    // key latents: thread item = (position, channel), from the staged pages
    if (!__all_sync(0xffffffffu, mbar_wait(kfull, 0))) ok = false;
    if (ok) {
      for (int hh = 0; hh < nh; ++hh) {
        uint8_t* tileA = Ak + hh * (kTile * 128);
        for (int e = tid; e < kTile * rk; e += 256) {
          const int t = e / rk, c = e % rk;
          const int p = t / kPage;
          float z = 0.f;
          if (pg[p] >= 0 && tile * kTile + t < L) {
            const int t16 = t % kPage, gi = c / a.key.g;
            const uint8_t* page = Kc + (hh * 8 + p) * a.kc_page;
            z = latent_value(page, reinterpret_cast<const uint32_t*>(page + a.kc_codes), a.key, gi, t16,
                             c % a.key.g);
          }
          *reinterpret_cast<__half*>(tileA + sw128_kmajor_offset(t, c, kTile)) = __float2half_rn(z);
        }
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(kready);
    // value chunks: thread item = (position, 16-channel group)
    for (int c = 0; ok && c < nchunk; ++c) {
      const int s = c % kXStages;
      const int bs = c & 1;
      const bool got = mbar_wait(&cfull[s], (c / kXStages) & 1) && mbar_wait(&aempty[bs], ((c >> 1) & 1) ^ 1);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      uint8_t* tileA = Av + bs * (kTile * 128);
      const uint8_t* st = Vc + s * vstage;
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int e = tid + it * 256;
        const int t = e >> 2, gq = e & 3;
        const int gi = c * 4 + gq;
        const int p = t / kPage, t16 = t % kPage;
        uint4 c0 = make_uint4(0, 0, 0, 0), c1 = make_uint4(0, 0, 0, 0);
        if (pg[p] >= 0 && tile * kTile + t < L && V.fp16) {
          // unquantised latents: the row of the group's tile, channels in order
          const uint4* row = reinterpret_cast<const uint4*>(st + p * a.vc_page + gq * 512 + t16 * 32);
          c0 = row[0];
          c1 = row[1];
        } else if (pg[p] >= 0 && tile * kTile + t < L) {
          const uint8_t* page = st + p * a.vc_page;
          const uint32_t mw = reinterpret_cast<const uint32_t*>(page + a.vc_codes_max)[gq * kPage + t16];
          const uint32_t toff = (uint32_t)(tile_offset(V, gi) - tile_offset(V, c * 4));
          if (gi < V.top_groups)
            dequant16_4bit(page + toff + 8 * t16, mw, c0, c1);
          else
            dequant16_3bit(page + toff, t16, mw, c0, c1);
        }
        *reinterpret_cast<uint4*>(tileA + sw128_kmajor_offset(t, gq * 16, kTile)) = c0;
        *reinterpret_cast<uint4*>(tileA + sw128_kmajor_offset(t, gq * 16 + 8, kTile)) = c1;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&cempty[s]);
        mbar_arrive(&afull[bs]);
      }
    }
  }
  // ---------------- epilogue (warps 0..7) ----------------
  const bool done = __all_sync(0xffffffffu, mbar_wait(alldone, 0));
  if (!(done && ok) && lane == 0) set_status(a.status, kDevWaitTimeout);
  tc_fence_after();
  if (warp < 8) {
    const int q4 = warp & 3, half = warp >> 2;
    const int t = q4 * 32 + lane;
    const int p = tile * kTile + t;
    const bool valid = done && ok && p < L && pg[t / kPage] >= 0;
    const uint32_t lrow = (uint32_t)(q4 * 32) << 16;
    const int hd = d / 2;
    for (int hh = 0; hh < nh; ++hh) {
      const int64_t row = ((int64_t)b * a.h_kv + kv0 + hh) * a.tpad + p;
      __half* krow = a.Kx + row * d;
      __half* vrow = a.Vx + row * d;
      for (int ci = half; ci < hd / 16; ci += 2) {
        const int i0 = ci * 16;
        uint32_t v0[16], v1[16], k0[16], k1[16];
        tmem_ld16(tmem + lrow + hh * d + i0, v0);
        tmem_ld16(tmem + lrow + hh * d + hd + i0, v1);
        tmem_ld16(tmem + lrow + 256 + hh * d + i0, k0);
        tmem_ld16(tmem + lrow + 256 + hh * d + hd + i0, k1);
        tmem_ld_wait();
        uint32_t vo0[8], vo1[8], ko0[8], ko1[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) vo0[u] = vo1[u] = ko0[u] = ko1[u] = 0u;
        if (valid) {
          const float2* cs = a.rope + (int64_t)p * hd + i0;
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            vo0[u / 2] = pack_half2(__uint_as_float(v0[u]), __uint_as_float(v0[u + 1]));
            vo1[u / 2] = pack_half2(__uint_as_float(v1[u]), __uint_as_float(v1[u + 1]));
            const float4 c2 = *reinterpret_cast<const float4*>(cs + u);  // (cos, sin) of pairs u, u + 1
            const float a0 = __uint_as_float(k0[u]), b0 = __uint_as_float(k1[u]);
            const float a1 = __uint_as_float(k0[u + 1]), b1 = __uint_as_float(k1[u + 1]);
            ko0[u / 2] = pack_half2(a0 * c2.x - b0 * c2.y, a1 * c2.z - b1 * c2.w);
            ko1[u / 2] = pack_half2(b0 * c2.x + a0 * c2.y, b1 * c2.z + a1 * c2.w);
          }
        }
        uint4* kd0 = reinterpret_cast<uint4*>(krow + i0);
        uint4* kd1 = reinterpret_cast<uint4*>(krow + hd + i0);
        uint4* vd0 = reinterpret_cast<uint4*>(vrow + i0);
        uint4* vd1 = reinterpret_cast<uint4*>(vrow + hd + i0);
        kd0[0] = make_uint4(ko0[0], ko0[1], ko0[2], ko0[3]);
        kd0[1] = make_uint4(ko0[4], ko0[5], ko0[6], ko0[7]);
        kd1[0] = make_uint4(ko1[0], ko1[1], ko1[2], ko1[3]);
        kd1[1] = make_uint4(ko1[4], ko1[5], ko1[6], ko1[7]);
        vd0[0] = make_uint4(vo0[0], vo0[1], vo0[2], vo0[3]);
        vd0[1] = make_uint4(vo0[4], vo0[5], vo0[6], vo0[7]);
        vd1[0] = make_uint4(vo1[0], vo1[1], vo1[2], vo1[3]);
        vd1[1] = make_uint4(vo1[4], vo1[5], vo1[6], vo1[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// B. attention
// ===========================================================================
struct AttnArgs {
  int H, h_kv, group, tpad, max_pages, max_position, max_q_len, batch;
  int64_t total_q;
  const __nv_bfloat16* q;
  const int32_t* cu_q;
  const int32_t* seq_lens;
  const float2* rope;
  __nv_bfloat16* out;
  unsigned int* status;
};

template <int D>
struct AttnSmem {
  static constexpr uint32_t kQ = 0;                       // Q tile [128 x D], K-major
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kK = kQ + kTileBytes;         // [2] K~ tiles [128 keys x D], K-major
  static constexpr uint32_t kV = kK + 2 * kTileBytes;     // [2] V tiles [128 keys x D], MN-major for P V
  static constexpr uint32_t kP = kV + 2 * kTileBytes;     // [2] P tiles [128 queries x 128 keys], K-major
  static constexpr uint32_t kBar = kP + 2 * kTile * kTile * 2;
  static constexpr uint32_t kBytes = kBar + 256 + 1024;   // barriers, TMEM slot, alignment slack
};

// grid (ceil(max_q_len / 128), H, B), 192 threads:
//   warp 0 producer (TMA of K~ / V tiles), warp 1 MMA issuer, warps 2..5 softmax
//   (warp w owns TMEM lanes 32 (w % 4) .. + 31, one query row per thread).
//   TMEM columns [0, 256): two S buffers; [256, 256 + D): O.
template <int D>
__global__ void __launch_bounds__(kQThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap k_map, const __grid_constant__ CUtensorMap v_map,
                        const AttnArgs a) {
  using SM = AttnSmem<D>;
  constexpr int NSUB = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024p(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SM::kBar);
  uint64_t* kfull = bar;        // [2]
  uint64_t* kempty = bar + 2;   // [2] S MMAs read the K~ tile
  uint64_t* vfull = bar + 4;    // [2]
  uint64_t* vempty = bar + 6;   // [2] P V MMAs read the V tile
  uint64_t* sfull = bar + 8;    // [2] S ready in TMEM
  uint64_t* sempty = bar + 10;  // [2] S read by the softmax warps
  uint64_t* pfull = bar + 12;   // [2] P written (and O rescaled if needed)
  uint64_t* pempty = bar + 14;  // [2] P V MMAs read the P tile
  uint64_t* ofull = bar + 16;   // one phase per P V step (waited only for the step just before)
  uint64_t* odone = bar + 17;   // every P V step done (one phase)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 18);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int kv = h / a.group;

  // inputs written before this call's first kernel (that kernel waited for them)
  const int q0 = a.cu_q[b], q1 = a.cu_q[b + 1];
  const int n = q1 - q0;
  const int L = a.seq_lens[b];
  const bool span_ok = q0 >= 0 && q1 <= a.total_q && n >= 0 && n <= a.max_q_len && n <= L && (b > 0 || q0 == 0) &&
                       (b < a.batch - 1 || q1 == a.total_q);
  const bool len_ok = L >= 0 && L <= a.max_pages * kPage && L <= a.max_position;
  if (qt == 0 && h == 0 && tid == 0) {
    if (!span_ok) set_status(a.status, STARKV_DEV_BAD_QUERY_SPAN);
    if (!len_ok) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
  }
  const int qbase = qt * kTile;
  if (!span_ok || !len_ok || qbase >= n) return;
  const int pos_first = L - n + qbase;              // position of the tile's first query
  const int rows = min(kTile, n - qbase);
  const int nkt = (pos_first + rows - 1) / kTile + 1;

  if (warp == 1) tmem_alloc(tslot, 512);
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
      mbar_init(&pfull[s], 4);
      mbar_init(&pempty[s], 1);
    }
    mbar_init(ofull, 1);
    mbar_init(odone, 1);
    fence_mbar_init();
  }
  // ---- Q tile: RoPE at each query's position, scaled by log2(e)/sqrt(D), fp16
  {
    const float scale = kLog2eQ * rsqrtf((float)D);
    constexpr int per_row = D / 16;  // 8-element chunks of the first half
    for (int e = tid; e < kTile * per_row; e += kQThreads) {
      const int r = e / per_row, i0 = (e % per_row) * 8;
      uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
      if (qbase + r < n) {
        const int pos = pos_first + r;
        const __nv_bfloat16* qv = a.q + ((int64_t)(q0 + qbase + r) * a.H + h) * D;
        const uint4 xa = *reinterpret_cast<const uint4*>(qv + i0);
        const uint4 xb = *reinterpret_cast<const uint4*>(qv + D / 2 + i0);
        const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(&xa);
        const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(&xb);
        const float2* cs = a.rope + (int64_t)pos * (D / 2) + i0;
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          const float4 c2 = *reinterpret_cast<const float4*>(cs + u);
          const float x0 = __bfloat162float(pa[u]), y0 = __bfloat162float(pb[u]);
          const float x1 = __bfloat162float(pa[u + 1]), y1 = __bfloat162float(pb[u + 1]);
          ol[u / 2] = pack_half2((x0 * c2.x - y0 * c2.y) * scale, (x1 * c2.z - y1 * c2.w) * scale);
          oh[u / 2] = pack_half2((y0 * c2.x + x0 * c2.y) * scale, (y1 * c2.z + x1 * c2.w) * scale);
        }
        lo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        hi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
      }
      *reinterpret_cast<uint4*>(sm + SM::kQ + sw128_kmajor_offset(r, i0, kTile)) = lo;
      *reinterpret_cast<uint4*>(sm + SM::kQ + sw128_kmajor_offset(r, D / 2 + i0, kTile)) = hi;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  pdl_wait();  // K~ and V come from the expand kernel
  bool ok = true;
  const int kvrow0 = (b * a.h_kv + kv) * a.tpad;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      for (int j = 0; j < nkt; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&kempty[s], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kfull[s], SM::kTileBytes);
        for (int i = 0; i < NSUB; ++i)
          tma_load_2d(sm + SM::kK + s * SM::kTileBytes + i * kSub, &k_map, i * 64, kvrow0 + j * kTile, &kfull[s]);
        if (!mbar_wait(&vempty[s], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&vfull[s], SM::kTileBytes);
        for (int i = 0; i < NSUB; ++i)
          tma_load_2d(sm + SM::kV + s * SM::kTileBytes + i * kSub, &v_map, i * 64, kvrow0 + j * kTile, &vfull[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc_s = make_idesc_f16(128, kTile, false, false);
      const uint32_t idesc_o = make_idesc_f16(128, D, false, true);
      const uint32_t qa = smem_u32(sm + SM::kQ);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&kfull[s], ph) || !mbar_wait(&sempty[s], ph ^ 1)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm + SM::kK + s * SM::kTileBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kSub + (ks & 3) * 32;
          mma_f16(tmem + s * kTile, make_sdesc(qa + off, 16, 1024, 2), make_sdesc(ka + off, 16, 1024, 2), idesc_s,
                  ks > 0);
        }
        mma_commit(&sfull[s]);
        mma_commit(&kempty[s]);
        return true;
      };
      ok = issue_s(0);
      for (int j = 0; ok && j < nkt; ++j) {
        if (j + 1 < nkt && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&pfull[s], ph) || !mbar_wait(&vfull[s], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pa = smem_u32(sm + SM::kP + s * (kTile * kTile * 2));
        const uint32_t va = smem_u32(sm + SM::kV + s * SM::kTileBytes);
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          mma_f16(tmem + 256, make_sdesc(pa + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024, 2),
                  make_sdesc(va + ks * 2048, kSub, 1024, 2), idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&pempty[s]);
        mma_commit(&vempty[s]);
        mma_commit(ofull);
      }
      if (ok) mma_commit(odone);
    }
  } else {
    // ---------------- softmax: one query row per thread ----------------
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const bool rvalid = qbase + r < n;
    const int pos = pos_first + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < nkt; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sfull[s], ph))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTile];
      {
        uint32_t(&raw)[kTile] = *reinterpret_cast<uint32_t(*)[kTile]>(sv);
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t(&rr)[32] = *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]);
          tmem_ld32(tmem + lane_off + s * kTile + c * 32, rr);
        }
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[s]);
      // causal mask: keys j*128 + c <= pos
      const int lim = rvalid ? min(kTile, max(0, pos - j * kTile + 1)) : 0;
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        sv[c] = c < lim ? sv[c] : -INFINITY;
        tmax = fmaxf(tmax, sv[c]);
      }
      const float m_new = fmaxf(m_used, tmax);
      const bool need = m_new > m_used + kRescaleLog2;
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O holds P V of the earlier tiles against m_used: rescale it in TMEM once
        // P V of tile j - 1 is done.  S of tile j completing implies P V of tile
        // j - 2 completed (issued before it), and P V of tile j waits for this
        // P, so ofull sits at phase j - 1 or j and its parity is unambiguous.
        if (!__all_sync(0xffffffffu, mbar_wait(ofull, (j - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float sc = need ? ex2_approx(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + 256 + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * sc);
          tmem_st32(tmem + lane_off + 256 + c * 32, o);
        }
        tmem_st_wait();
        l *= sc;
      }
      if (need) m_used = m_new;
      // P = 2^(s - m_used) as fp16, K-major rows; l sums the fp32 values
      if (!__all_sync(0xffffffffu, mbar_wait(&pempty[s], ph ^ 1))) {
        ok = false;
        break;
      }
      uint8_t* pt = sm + SM::kP + s * (kTile * kTile * 2);
      const bool live = m_used != -INFINITY;
#pragma unroll
      for (int c8 = 0; c8 < kTile / 8; ++c8) {
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          const float p0 = live ? ex2_approx(sv[c8 * 8 + u] - m_used) : 0.f;
          const float p1 = live ? ex2_approx(sv[c8 * 8 + u + 1] - m_used) : 0.f;
          l += p0 + p1;
          w4[u / 2] = pack_half2(p0, p1);
        }
        *reinterpret_cast<uint4*>(pt + sw128_kmajor_offset(r, c8 * 8, kTile)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[s]);
    }
    // ---- epilogue: O / l as bf16
    if (ok && __all_sync(0xffffffffu, mbar_wait(odone, 0))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = a.out + ((int64_t)(q0 + qbase + r) * a.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + 256 + c * 32, o);
        tmem_ld_wait();
        if (rvalid) {
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[u]) * inv, __uint_as_float(o[u + 1]) * inv);
            w[u / 2] = *reinterpret_cast<const uint32_t*>(&v);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
    } else {
      ok = false;
    }
  }
  if (!ok && lane == 0) set_status(a.status, kDevWaitTimeout);
  // the MMA warp's last commits may still be in flight on a failure path: wait for them (bounded)
  if (warp == 1 && lane == 0 && !ok) {
    uint64_t* fin = bar + 19;
    mbar_init(fin, 1);
    fence_mbar_init();
    mma_commit(fin);
    mbar_wait(fin, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// host side
// ===========================================================================
bool tc_prefill_supported(const Ctx& c) {
  const starkv_config& f = c.cfg;
  if (f.head_dim != 64 && f.head_dim != 128) return false;
  if (f.rank_k % 16 != 0 || f.rank_k > 64) return false;
  if (c.val.g != 16 || f.rank_v % 64 != 0) return false;
  return true;
}

namespace {
struct XLayout {
  int HP;
  uint32_t off_ak, off_bk, off_kc, off_av, off_bv, off_vc, off_bar, bk_head, bv_stage;
  uint32_t kc_codes, kc_page, vc_codes_max, vc_page;
  size_t smem;
};

XLayout expand_layout(const Ctx& c) {
  XLayout x;
  const int d = c.cfg.head_dim, rk = c.cfg.rank_k;
  x.HP = c.cfg.num_kv_heads % 2 == 0 ? 2 : 1;
  x.bk_head = (uint32_t)(d / 64) * rk * 128;
  x.bv_stage = (uint32_t)(x.HP * d / 64) * 8192;
  x.kc_codes = (uint32_t)c.key.region_bytes;                        // a multiple of 16
  x.kc_page = x.kc_codes + (c.key.fp16 ? 0u : (uint32_t)c.key.groups * kPage * 4);
  // the largest 4-group span of the value region (all 4-bit groups, or fp16 tiles)
  x.vc_codes_max = c.val.fp16 ? 4 * 512u : 4 * 8 * (uint32_t)c.val.g;
  x.vc_page = x.vc_codes_max + (c.val.fp16 ? 0u : 4 * kPage * 4);
  uint32_t o = 0;
  x.off_ak = o;
  o += x.HP * kTile * 128;
  x.off_bk = o;
  o += (x.HP * x.bk_head + 1023) / 1024 * 1024;
  x.off_av = o;
  o += 2 * kTile * 128;
  x.off_bv = o;
  o += 2 * x.bv_stage;
  x.off_kc = o;
  o += (uint32_t)x.HP * 8 * x.kc_page;
  x.off_vc = (o + 127) / 128 * 128;
  o = x.off_vc + kXStages * 8 * x.vc_page;
  x.off_bar = (o + 15) / 16 * 16;
  o = x.off_bar + 256;
  x.smem = o + 1024;
  return x;
}

size_t kv_bytes(const Ctx& c, int batch, int max_pages) {
  const size_t tpad = (size_t)(max_pages * kPage + kTile - 1) / kTile * kTile;
  return (size_t)batch * c.cfg.num_kv_heads * tpad * c.cfg.head_dim * sizeof(__half);
}
}  // namespace

PrefillPlan plan_prefill_tc(const Ctx& c, int batch, int max_pages, int64_t) {
  PrefillPlan p;
  p.chunk = 0;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  p.ws_bytes = 2 * al(kv_bytes(c, batch, max_pages));
  return p;
}

__global__ void permute_values_half_kernel(const float* __restrict__ Bv, __half* __restrict__ out, int R, int cols,
                                           int top_groups) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)R * cols) return;
  const int row = (int)(i / cols), col = (int)(i % cols);
  const int gi = row / 16;
  const int src = gi * 16 + value_channel_of_position(row % 16, gi < top_groups);
  out[i] = __float2half_rn(Bv[(int64_t)src * cols + col]);
}

__global__ void to_half_prefill_kernel(const float* __restrict__ x, __half* __restrict__ y, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = __float2half_rn(x[i]);
}

cudaError_t launch_prepare_prefill_factors(const Ctx& c, cudaStream_t s) {
  const starkv_config& f = c.cfg;
  const int64_t nk = (int64_t)c.key_cols * f.head_dim;
  to_half_prefill_kernel<<<(unsigned)((nk + 255) / 256), 256, 0, s>>>(c.Bk, c.Bk16, nk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (c.val.g != 16) return cudaSuccess;  // the permuted copy serves the 16-channel value dequantiser only
  const int cols = f.num_kv_heads * f.head_dim;
  const int64_t nv = (int64_t)f.rank_v * cols;
  permute_values_half_kernel<<<(unsigned)((nv + 255) / 256), 256, 0, s>>>(c.Bv, c.Bv16p, f.rank_v, cols,
                                                                          c.val.top_groups);
  return cudaGetLastError();
}

bool make_prefill_maps(Ctx* c) {
  const starkv_config& f = c->cfg;
  if (!encode_map_2d(&c->bk_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c->Bk16, (uint64_t)f.head_dim,
                     (uint64_t)f.num_kv_heads * f.rank_k, (uint64_t)f.head_dim * 2, 64, (uint32_t)f.rank_k,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return false;
  // the value A tiles hold channels in the order the dequantiser emits them
  // (value_channel_of_position) for quantised latents, in plain order for fp16 ones
  return encode_map_2d(&c->bvp_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c->val.fp16 ? c->Bv16 : c->Bv16p,
                       (uint64_t)f.num_kv_heads * f.head_dim,
                       (uint64_t)f.rank_v, (uint64_t)f.num_kv_heads * f.head_dim * 2, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int D>
static cudaError_t launch_attn(const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a, int qtiles,
                               cudaStream_t s) {
  const size_t smem = AttnSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_chained(prefill_attn_kernel<D>, dim3(qtiles, a.H, a.batch), dim3(kQThreads), smem, s, 1u, km, vm, a);
}

cudaError_t launch_prefill_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q, const int32_t* cu_q,
                              const int32_t* block_table, const int32_t* seq_lens, int batch, int max_pages,
                              int64_t total_q, int max_q_len, __nv_bfloat16* out, void* ws, const PrefillPlan&,
                              cudaStream_t s) {
  if (batch == 0 || total_q == 0) return cudaSuccess;
  const starkv_config& f = c.cfg;
  const int d = f.head_dim;
  const int tpad = (max_pages * kPage + kTile - 1) / kTile * kTile;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  __half* Kx = (__half*)ws;
  __half* Vx = (__half*)((char*)ws + al(kv_bytes(c, batch, max_pages)));
  // rows whose sequence is skipped (bad span or length) read as zeros
  cudaError_t e = cudaMemsetAsync(out, 0, (size_t)total_q * f.num_q_heads * d * sizeof(__nv_bfloat16), s);
  if (e != cudaSuccess) return e;
  // ---- A: expand
  {
    const XLayout x = expand_layout(c);
    ExpandArgs a;
    a.key = c.key;
    a.val = c.val;
    a.h_kv = f.num_kv_heads;
    a.d = d;
    a.HP = x.HP;
    a.max_pages = max_pages;
    a.max_position = f.max_position;
    a.tpad = tpad;
    a.n_pages = cache.n_pages;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.k_codes = (const uint8_t*)cache.k_codes;
    a.v_codes = (const uint8_t*)cache.v_codes;
    a.k_meta = (const uint32_t*)cache.k_meta;
    a.v_meta = (const uint32_t*)cache.v_meta;
    a.rope = c.rope;
    a.Kx = Kx;
    a.Vx = Vx;
    a.status = c.status;
    a.off_ak = x.off_ak;
    a.off_bk = x.off_bk;
    a.off_kc = x.off_kc;
    a.off_av = x.off_av;
    a.off_bv = x.off_bv;
    a.off_vc = x.off_vc;
    a.off_bar = x.off_bar;
    a.bk_head = x.bk_head;
    a.bv_stage = x.bv_stage;
    a.kc_codes = x.kc_codes;
    a.kc_page = x.kc_page;
    a.vc_codes_max = x.vc_codes_max;
    a.vc_page = x.vc_page;
    e = cudaFuncSetAttribute(prefill_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)x.smem);
    if (e != cudaSuccess) return e;
    e = launch_chained(prefill_expand_kernel, dim3(tpad / kTile, (f.num_kv_heads + x.HP - 1) / x.HP, batch),
                       dim3(kXThreadsW), x.smem, s, 1u, c.bk_map, c.bvp_map, a);
    if (e != cudaSuccess) return e;
  }
  // ---- B: attention
  {
    CUtensorMap km, vm;
    const uint64_t rows = (uint64_t)batch * f.num_kv_heads * tpad;
    if (!encode_map_2d(&km, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Kx, (uint64_t)d, rows, (uint64_t)d * 2, 64, kTile,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_2d(&vm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Vx, (uint64_t)d, rows, (uint64_t)d * 2, 64, kTile,
                       CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    AttnArgs a;
    a.H = f.num_q_heads;
    a.h_kv = f.num_kv_heads;
    a.group = c.group;
    a.tpad = tpad;
    a.max_pages = max_pages;
    a.max_position = f.max_position;
    a.max_q_len = max_q_len;
    a.batch = batch;
    a.total_q = total_q;
    a.q = q;
    a.cu_q = cu_q;
    a.seq_lens = seq_lens;
    a.rope = c.rope;
    a.out = out;
    a.status = c.status;
    const int qtiles = (max_q_len + kTile - 1) / kTile;
    e = d == 64 ? launch_attn<64>(km, vm, a, qtiles, s) : launch_attn<128>(km, vm, a, qtiles, s);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace starkv

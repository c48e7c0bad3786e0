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

#include <mutex>

#include "internal.cuh"
#include "latent_tc.cuh"
#include "sm100.cuh"

namespace starkv {
using namespace sm100;

namespace {
constexpr int kT = 128;                 // tokens per key tile (MMA M)
constexpr int kPagesPerTile = kT / kPage;
constexpr int kEpiWarps = 16;
constexpr int kAThreads = (2 + kEpiWarps) * 32;
constexpr float kLog2e = 1.4426950408889634f;

// 1024-byte aligned base inside the dynamic shared-memory array.  The offset is
// added to the __shared__ array itself so the compiler keeps the shared state
// space (plain shared loads/stores instead of generic ones).
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return p + ((1024u - (sm100::smem_u32(p) & 1023u)) & 1023u);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Order-preserving map of a float onto unsigned integers (so an integer
// atomicMax takes a float maximum); 0 stands below every float.
__device__ __forceinline__ unsigned int ordered_bits(float f) {
  const unsigned int u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_float(unsigned int o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Token count of sequence b, or -1 when the call's arguments for it are not
// valid.  The sequence's cached tokens sit at positions pos0 .. pos0 + L - 1
// (pos0 = 0 without a key-position table) and its query at qpos (L - 1
// without a query-position table); every position must lie in the RoPE table.
__device__ __forceinline__ int decode_len(const int32_t* seq_lens, const int32_t* pos0, const int32_t* qpos, int b,
                                          int max_pages, int max_position) {
  const int L = seq_lens[b];
  const int p0 = pos0 ? pos0[b] : 0;
  if (L < 0 || L > max_pages * kPage || p0 < 0 || (int64_t)p0 + L > max_position) return -1;
  if (qpos) {
    const int qp = qpos[b];
    if (qp < 0 || qp >= max_position) return -1;
  }
  return L;
}

// Value CTAs of sequence b when `slots` CTAs are shared out over the batch in
// proportion to the sequences' stage counts (ST tokens each): floor shares,
// at least one for a sequence with tokens, the slots left over to the largest
// remainders (ties to the lower index), at most `cap` and at most the
// sequence's stages.  Run by one full warp; every lane returns the count.
__device__ int value_splits_of(int b, const int32_t* seq_lens, const int32_t* pos0, const int32_t* qpos, int batch,
                               int max_pages, int max_position, int ST, int slots, int cap) {
  const int lane = threadIdx.x & 31;
  auto stages = [&](int i) -> int64_t {
    const int L = decode_len(seq_lens, pos0, qpos, i, max_pages, max_position);
    return L > 0 ? (L + ST - 1) / ST : 0;
  };
  int64_t tot = 0;
  for (int i = lane; i < batch; i += 32) tot += stages(i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  const int64_t sb = stages(b);
  if (sb == 0 || tot == 0) return 0;
  int64_t used = 0, ahead = 0;  // floor shares in all; sequences whose remainder ranks before b's
  const int64_t rb = ((int64_t)slots * sb) % tot;
  const bool b_floor0 = (int64_t)slots * sb < tot;
  for (int i = lane; i < batch; i += 32) {
    const int64_t si = stages(i);
    if (si == 0) continue;
    const int64_t q = (int64_t)slots * si / tot, r = ((int64_t)slots * si) % tot;
    used += q > 0 ? q : 1;
    if (q > 0 && (r > rb || (r == rb && i < b))) ++ahead;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    used += __shfl_xor_sync(0xffffffffu, used, o);
    ahead += __shfl_xor_sync(0xffffffffu, ahead, o);
  }
  int64_t k = (int64_t)slots * sb / tot;
  if (k < 1) k = 1;
  if (!b_floor0 && ahead < (int64_t)slots - used) ++k;
  if (k > cap) k = cap;
  if (k > sb) k = sb;
  return (int)k;
}
}  // namespace

// ===========================================================================
// A. scores
// ===========================================================================
struct ScoreArgs {
  LatentGeom key;
  int H, h_kv, group, d, hpc, kvpc, ncols, HG;
  int max_pages, tiles_per_seq, tpad, max_position;
  int items_per_cta, batch;  // tiles per CTA at most (its page-table space); sequences
  int64_t n_pages;
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* pos0;  // [B] position of each sequence's first cached token, or NULL (0)
  const int32_t* qpos;  // [B] query positions, or NULL (seq_len - 1)
  const uint8_t* k_codes;
  const uint32_t* k_meta;
  const float* Bk;     // [h_kv][r_k][d] fp32 B'_k
  const float2* rope;  // [max_position][d/2]
  float* S;            // [B][H][tpad]      scores, log2 domain
  unsigned int* Mx;    // [B][H] running score maximum (ordered bits; zeroed by the W prep)
  float* oacc;         // [B][H][d] zeroed here for the projection
  unsigned int* ocnt;  // [H][ceil(B/16)] zeroed here
  int64_t oacc_elems;  // B * H * d
  int ocnt_elems;
  const uint8_t* wimg; // [B][HG][ncols * d * 2] W in its shared-memory image
  unsigned int* status;
  uint32_t off_trig, off_codes, off_meta, off_flags, off_bt, off_bar, off_red, off_pre;
  uint32_t trig_stage, codes_page, meta_page, codes_stage, meta_stage, w_bytes;
  int NK;  // key-stage ring depth (the position tiles use two stages)
  uint32_t codes_pitch, meta_pitch;  // shared-memory page strides (padded against bank conflicts)
};

// ---------------------------------------------------------------------------
// W prep: one CTA per (head, sequence).  With q~ the query rotated to its
// position and i < d/2 a frequency pair (i, i + d/2), for every latent channel c
//   W[c][i]       = (q~_i B'[c,i] + q~_{i+d/2} B'[c,i+d/2]) * log2(e)/sqrt(d)
//   W[c][i + d/2] = (q~_{i+d/2} B'[c,i] - q~_i B'[c,i+d/2]) * log2(e)/sqrt(d)
// A thread owns (c, 8 consecutive i): it reads those B' values (L2-resident) and
// writes 16-byte fp16 chunks straight into the score kernel's shared-memory
// image (K-major, 128-byte swizzle).  The CTA also zeroes the running score
// maxima of its (sequence, head) pairs.
// ---------------------------------------------------------------------------
constexpr int kWpSeq = 1;  // sequences per W-prep CTA

template <int RK>
__global__ void __launch_bounds__(128) decode_wprep_kernel(const __nv_bfloat16* __restrict__ q,
                                                           const int32_t* __restrict__ seq_lens,
                                                           const int32_t* __restrict__ pos0,
                                                           const int32_t* __restrict__ qpos,
                                                           const float* __restrict__ Bk, const float2* __restrict__ rope,
                                                           uint8_t* __restrict__ wimg, unsigned int* __restrict__ Mx,
                                                           int H, int group, int d, int hpc, int ncols, int batch,
                                                           int max_pages, int max_position) {
  __shared__ float qs[kWpSeq][2][64];  // rotated, scaled (q~_i, q~_{i+d/2}) per sequence
  const int h = blockIdx.x, b0 = blockIdx.y * kWpSeq, tid = threadIdx.x;
  // first kernel of a decode call: its inputs may come from any earlier kernel
  pdl_wait();
  pdl_launch_dependents();
  const int half = d / 2;
  const int kv = h / group, hg = h / hpc, hl = h % hpc;
  const float scale = kLog2e * rsqrtf((float)d);
  for (int e = tid; e < kWpSeq * half; e += blockDim.x) {
    const int sb = e / half, i = e % half, b = b0 + sb;
    float qa = 0.f, qb = 0.f;
    if (b < batch) {
      const int L = decode_len(seq_lens, pos0, qpos, b, max_pages, max_position);
      const int qp = L <= 0 ? 0 : (qpos ? qpos[b] : L - 1);  // no tiles when L <= 0: keep reads in range
      const float2 cs = rope[(int64_t)qp * half + i];
      const __nv_bfloat16* qv = q + ((int64_t)b * H + h) * d;
      const float x0 = __bfloat162float(qv[i]), x1 = __bfloat162float(qv[i + half]);
      qa = (x0 * cs.x - x1 * cs.y) * scale;
      qb = (x1 * cs.x + x0 * cs.y) * scale;
      if (i == 0) Mx[b * H + h] = 0u;
    }
    qs[sb][0][i] = qa;
    qs[sb][1][i] = qb;
  }
  __syncthreads();
  const float* B = Bk + (int64_t)kv * RK * d;
  for (int e = tid; e < RK * (half / 8); e += blockDim.x) {
    const int c = e / (half / 8), i0 = (e % (half / 8)) * 8;
    const float4 a0 = __ldg(reinterpret_cast<const float4*>(B + c * d + i0));
    const float4 a1 = __ldg(reinterpret_cast<const float4*>(B + c * d + i0 + 4));
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(B + c * d + half + i0));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(B + c * d + half + i0 + 4));
    const float ba[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bb[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const int n = hl * RK + c;
    for (int sb = 0; sb < kWpSeq; ++sb) {
      const int b = b0 + sb;
      if (b >= batch) break;
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float qa0 = qs[sb][0][i0 + j], qb0 = qs[sb][1][i0 + j];
        const float qa1 = qs[sb][0][i0 + j + 1], qb1 = qs[sb][1][i0 + j + 1];
        const __half2 wl = __floats2half2_rn(fmaf(qa0, ba[j], qb0 * bb[j]), fmaf(qa1, ba[j + 1], qb1 * bb[j + 1]));
        const __half2 wh = __floats2half2_rn(fmaf(qb0, ba[j], -qa0 * bb[j]), fmaf(qb1, ba[j + 1], -qa1 * bb[j + 1]));
        lo[j / 2] = *reinterpret_cast<const uint32_t*>(&wl);
        hi[j / 2] = *reinterpret_cast<const uint32_t*>(&wh);
      }
      uint8_t* img = wimg + ((int64_t)b * (H / hpc) + hg) * ((int64_t)ncols * d * 2);
      *reinterpret_cast<uint4*>(img + sw128_kmajor_offset(n, i0, ncols)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(img + sw128_kmajor_offset(n, i0 + half, ncols)) =
          make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
  }
}

// TMEM columns of the score accumulators: two buffers of up to 256 columns.
constexpr uint32_t kScoreTmemCols = 512;
constexpr int kMaxKeyStages = 6;  // deepest key-stage ring
constexpr int kMaxScoreItemsPerCta = 256;  // 128-token tiles per score CTA at most (8 KiB of page ids)

// Issue the TMEM loads of one RK-column row into raw registers (no wait).
template <int RK>
__device__ __forceinline__ void tmem_issue_row(uint32_t taddr, uint32_t (&r)[RK]) {
  if constexpr (RK == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
#pragma unroll
    for (int h = 0; h < RK / 32; ++h) {
      uint32_t(&rr)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[h * 32]);
      tmem_ld32(taddr + h * 32, rr);
    }
  }
}

// Wait for the row's TMEM loads; the registers pass through the wait so no use
// of them can be scheduled before it.
template <int RK>
__device__ __forceinline__ void tmem_wait_row(uint32_t (&r)[RK]) {
#pragma unroll
  for (int q = 0; q < RK; q += 16) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[q + 0]), "+r"(r[q + 1]), "+r"(r[q + 2]), "+r"(r[q + 3]), "+r"(r[q + 4]), "+r"(r[q + 5]),
                   "+r"(r[q + 6]), "+r"(r[q + 7]), "+r"(r[q + 8]), "+r"(r[q + 9]), "+r"(r[q + 10]), "+r"(r[q + 11]),
                   "+r"(r[q + 12]), "+r"(r[q + 13]), "+r"(r[q + 14]), "+r"(r[q + 15])
                 :
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Key dot product on packed codes (one token, one head), compile-time layout.
//
// Codes become floats by writing their bits into the mantissa of 1.0:
// x = 1 + code / 16 exactly, for a 4-bit code and for a 3-bit code whose two
// planes were first rebuilt into a nibble.  With gs = sum_c G_c over the group,
//   sum_c code_c G_c = 16 (sum_c x_c G_c - gs)
// and the group's contribution is s * sum code G + zp * gs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float mant(uint32_t bits) { return __uint_as_float(0x3F800000u | bits); }

// 3-bit codes of one token as 4-bit nibbles: the 2-bit plane's fields (bits
// 2c..2c+1) and the 1-bit plane's bits (bit c) spread to nibble c (bits 4c..4c+3).
__device__ __forceinline__ uint32_t spread2_to_nibbles8(uint32_t x) {  // 8 fields of 2 bits
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  return (x | (x << 2)) & 0x33333333u;
}
__device__ __forceinline__ uint32_t spread1_to_nibbles8(uint32_t y) {  // 8 single bits
  y = (y | (y << 12)) & 0x000F000Fu;
  y = (y | (y << 6)) & 0x03030303u;
  return (y | (y << 3)) & 0x11111111u;
}

template <int G>
struct KeyGroup {
  // sum_c x_c G_c and sum_c G_c over up to 8 channels whose codes are the
  // nibbles of w (x_c = 1 + code_c / 16); two accumulators each
  template <int N>
  __device__ __forceinline__ static void nib_dot(uint32_t w, const float* Gv, float (&acc)[2], float (&gs)[2]) {
#pragma unroll
    for (int c = 0; c < N; ++c) {
      const float x = mant(((c >= 5 ? (w >> (4 * c - 19)) : (w << (19 - 4 * c)))) & 0x00780000u);
      acc[c & 1] = fmaf(x, Gv[c], acc[c & 1]);
      gs[c & 1] += Gv[c];
    }
  }
  // sum_c code_c G_c of a 4-bit group (16 (sum x G - sum G)), sum_c G_c in gsum
  __device__ __forceinline__ static float dot4(const uint8_t* tile, int t16, const float* Gv, float& gsum) {
    float acc[2] = {0.f, 0.f}, gs[2] = {0.f, 0.f};
    if constexpr (G == 4) {
      nib_dot<4>(*reinterpret_cast<const uint16_t*>(tile + 2 * t16), Gv, acc, gs);
    } else {
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(tile + (G / 2) * t16);
#pragma unroll
      for (int q = 0; q < G / 8; ++q) nib_dot<8>(wp[q], Gv + 8 * q, acc, gs);
    }
    gsum = gs[0] + gs[1];
    return 16.f * (acc[0] + acc[1] - gsum);
  }
  // the same for a 3-bit group: planes rebuilt into nibbles first
  __device__ __forceinline__ static float dot3(const uint8_t* tile, int t16, const float* Gv, float& gsum) {
    float acc[2] = {0.f, 0.f}, gs[2] = {0.f, 0.f};
    if constexpr (G == 4) {
      const uint32_t lo = tile[t16];
      const uint32_t hi = (uint32_t)(tile[16 + (t16 >> 1)] >> ((t16 & 1) * 4)) & 0xFu;
      nib_dot<4>(spread2_to_nibbles8(lo) | (spread1_to_nibbles8(hi) << 2), Gv, acc, gs);
    } else if constexpr (G == 8) {
      const uint32_t lo = *reinterpret_cast<const uint16_t*>(tile + 2 * t16);
      const uint32_t hi = tile[32 + t16];
      nib_dot<8>(spread2_to_nibbles8(lo) | (spread1_to_nibbles8(hi) << 2), Gv, acc, gs);
    } else {
      const uint32_t lo = *reinterpret_cast<const uint32_t*>(tile + 4 * t16);
      const uint32_t hi = *reinterpret_cast<const uint16_t*>(tile + 64 + 2 * t16);
      nib_dot<8>(spread2_to_nibbles8(lo & 0xFFFFu) | (spread1_to_nibbles8(hi & 0xFFu) << 2), Gv, acc, gs);
      nib_dot<8>(spread2_to_nibbles8(lo >> 16) | (spread1_to_nibbles8(hi >> 8) << 2), Gv + 8, acc, gs);
    }
    gsum = gs[0] + gs[1];
    return 16.f * (acc[0] + acc[1] - gsum);
  }
};

// sum_c z_hat_c G_c over one token's key latent in a staged page region.
// Two heads' scores at once: the groups of both are independent, so their
// dependency chains interleave.
template <int RK, int G>
__device__ __forceinline__ void key_dot2(const uint8_t* regA, const uint32_t* metaA, const uint8_t* regB,
                                         const uint32_t* metaB, int top_groups, int t16, const uint32_t (&rA)[RK],
                                         const uint32_t (&rB)[RK], float& sA, float& sB) {
  const float* GA = reinterpret_cast<const float*>(rA);
  const float* GB = reinterpret_cast<const float*>(rB);
  float accA = 0.f, accB = 0.f;
#pragma unroll
  for (int gi = 0; gi < RK / G; ++gi) {
    const uint32_t mA = metaA[gi * kPage + t16], mB = metaB[gi * kPage + t16];
    float gsA, gsB, cA, cB;
    if (gi < top_groups) {
      cA = KeyGroup<G>::dot4(regA + gi * 8 * G, t16, GA + gi * G, gsA);
      cB = KeyGroup<G>::dot4(regB + gi * 8 * G, t16, GB + gi * G, gsB);
    } else {
      const int o = top_groups * 8 * G + (gi - top_groups) * 6 * G;
      cA = KeyGroup<G>::dot3(regA + o, t16, GA + gi * G, gsA);
      cB = KeyGroup<G>::dot3(regB + o, t16, GB + gi * G, gsB);
    }
    const float sa = __half2float(__ushort_as_half((unsigned short)(mA & 0xFFFF)));
    const float za = __half2float(__ushort_as_half((unsigned short)(mA >> 16)));
    const float sb = __half2float(__ushort_as_half((unsigned short)(mB & 0xFFFF)));
    const float zb = __half2float(__ushort_as_half((unsigned short)(mB >> 16)));
    accA = fmaf(sa, cA, fmaf(za, gsA, accA));
    accB = fmaf(sb, cB, fmaf(zb, gsB, accB));
  }
  sA = accA;
  sB = accB;
}

template <int RK, int G>
__device__ __forceinline__ float key_dot(const uint8_t* region, const uint32_t* meta, int top_groups, int t16,
                                         const uint32_t (&raw)[RK]) {
  const float* Gv = reinterpret_cast<const float*>(raw);
  float score = 0.f;
#pragma unroll
  for (int gi = 0; gi < RK / G; ++gi) {
    const uint32_t m = meta[gi * kPage + t16];
    const float s = __half2float(__ushort_as_half((unsigned short)(m & 0xFFFF)));
    const float zp = __half2float(__ushort_as_half((unsigned short)(m >> 16)));
    float gs, cg;
    if (gi < top_groups) {
      cg = KeyGroup<G>::dot4(region + gi * 8 * G, t16, Gv + gi * G, gs);
    } else {
      cg = KeyGroup<G>::dot3(region + top_groups * 8 * G + (gi - top_groups) * 6 * G, t16, Gv + gi * G, gs);
    }
    score = fmaf(s, cg, fmaf(zp, gs, score));
  }
  return score;
}

// sum_c z_c G_c over one token's unquantised (fp16) key latent: tiles of 16
// tokens x 16 channels, row t16 of tile gi holds channels 16 gi .. 16 gi + 15.
template <int RK>
__device__ __forceinline__ float key_dot_fp16(const uint8_t* region, int t16, const uint32_t (&raw)[RK]) {
  const float* Gv = reinterpret_cast<const float*>(raw);
  float acc[2] = {0.f, 0.f};
#pragma unroll
  for (int gi = 0; gi < RK / 16; ++gi) {
    const uint4* row = reinterpret_cast<const uint4*>(region + gi * 512 + t16 * 32);
    const uint4 u0 = row[0], u1 = row[1];
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      acc[k & 1] = fmaf(f.x, Gv[gi * 16 + 2 * k], acc[k & 1]);
      acc[k & 1] = fmaf(f.y, Gv[gi * 16 + 2 * k + 1], acc[k & 1]);
    }
  }
  return acc[0] + acc[1];
}

// G: the key group size of quantised latents (4, 8, 16), or 0 for fp16 latents.
template <int RK, int G>
__global__ void __launch_bounds__(kAThreads, 1)
    decode_scores_kernel(const __grid_constant__ CUtensorMap trig_map, const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* Wsm = sm;                                         // [ncols x d] K-major, 128B swizzle
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + a.off_bar);
  // Two rings: position tiles (needed by the MMA only, freed by its commit) and
  // key codes + metadata (read by the epilogue, freed by it), NK stages deep.
  uint64_t* trfull = bar;                       // [2] position tile loaded
  uint64_t* trempty = bar + 2;                  // [2] position tile read by the MMA
  uint64_t* tfull = bar + 4;                    // [2] accumulator ready
  uint64_t* tempty = bar + 6;                   // [2] accumulator drained
  uint64_t* kfull = bar + 8;                    // [NK] key stage loaded
  uint64_t* kempty = kfull + kMaxKeyStages;     // [NK] key stage read by the epilogue
  uint64_t* wbar = kempty + kMaxKeyStages;      // W image loaded
  uint32_t* tslot = reinterpret_cast<uint32_t*>(wbar + 1);
  int* failed = reinterpret_cast<int*>(wbar + 2);
  int* flags = reinterpret_cast<int*>(sm + a.off_flags);    // [NK][8] page ids (-1 = invalid)
  int* bt_s = reinterpret_cast<int*>(sm + a.off_bt);        // this job's block-table entries
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = a.d;

  // (before the wait: every kernel earlier than the query fold has completed)
  // zero the projection's sums and arrival counters (grid-stride over all CTAs)
  // partial-score reduction buffer of the shared-KV-head epilogue: [2 tiles][4 heads][128 tokens]
  for (int i = tid; i < 2 * 4 * kT; i += blockDim.x) reinterpret_cast<float*>(sm + a.off_red)[i] = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < a.oacc_elems; i += (int64_t)gridDim.x * blockDim.x)
    a.oacc[i] = 0.f;
  for (int i = blockIdx.x * blockDim.x + tid; i < a.ocnt_elems; i += gridDim.x * blockDim.x) a.ocnt[i] = 0u;

  if (warp == 1) tmem_alloc(tslot, kScoreTmemCols);
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&trfull[s], 1);
      mbar_init(&trempty[s], 1);
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiWarps);
    }
    for (int s = 0; s < a.NK; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], kEpiWarps);
    }
    mbar_init(wbar, 1);
    *failed = 0;
    fence_mbar_init();
  }
  pdl_wait();  // W images and zeroed maxima (query fold), appended codes
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t idesc = make_idesc_f16(128, a.ncols, false, false);
  uint32_t jobs = 0;

  uint32_t it = 0;  // tiles through the pipeline so far (same count in every role)
  // The work items are the sequences' 128-token tiles that hold tokens, per head
  // group: pre[b] = items of the sequences before b (HG x tiles each).  Every CTA
  // takes an equal share of them, so sequences of unequal length balance.
  int* pre = reinterpret_cast<int*>(sm + a.off_pre);  // [batch + 1]
  if (warp == 0) {
    int run = 0;
    for (int b0 = 0; b0 < a.batch; b0 += 32) {
      const int b = b0 + lane;
      int v = 0;
      if (b < a.batch) {
        const int Lb = decode_len(a.seq_lens, a.pos0, a.qpos, b, a.max_pages, a.max_position);
        v = Lb > 0 ? (Lb + kT - 1) / kT * a.HG : 0;
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (b < a.batch) pre[b + 1] = run + v;
      run += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) pre[0] = 0;
  }
  __syncthreads();
  const int total = pre[a.batch];
  int item = (int)((int64_t)blockIdx.x * total / gridDim.x);
  const int item_end = (int)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
  while (item < item_end) {
    // the sequence holding `item`: the last b with pre[b] <= item
    int lo = 0, hi = a.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= item) lo = mid;
      else hi = mid;
    }
    const int b = lo;
    const int n_tiles = (pre[b + 1] - pre[b]) / a.HG;
    const int rel = item - pre[b];
    const int hg = rel / n_tiles;
    const int job_end = min(item_end, pre[b] + (hg + 1) * n_tiles);
    const int t0 = rel - hg * n_tiles, t1 = t0 + (job_end - item);
    item = job_end;
    const int L = decode_len(a.seq_lens, a.pos0, a.qpos, b, a.max_pages, a.max_position);
    const int p0 = a.pos0 ? a.pos0[b] : 0;  // position of the sequence's first cached token
    if (*failed) break;
    const int h0 = hg * a.hpc;
    const int kv0 = h0 / a.group;
    // ---- W for this (sequence, head group): one bulk copy of its prepared image;
    //      this job's page ids into shared memory (coalesced)
    if (tid == 0) {
      mbar_arrive_expect_tx(wbar, a.w_bytes);
      bulk_g2s(Wsm, a.wimg + ((int64_t)b * a.HG + hg) * a.w_bytes, a.w_bytes, wbar);
    }
    {
      const int p0 = t0 * kPagesPerTile;
      const int np_job = min((t1 - t0) * kPagesPerTile, (L + kPage - 1) / kPage - p0);
      for (int e = tid; e < np_job; e += blockDim.x) bt_s[e] = a.block_table[(int64_t)b * a.max_pages + p0 + e];
    }
    __syncthreads();
    if (!mbar_wait(wbar, jobs & 1)) {
      if (tid == 0) {
        set_status(a.status, kDevWaitTimeout);
        *failed = 1;
      }
    }
    ++jobs;
    __syncthreads();
    if (*failed) break;
    const int ntile = t1 - t0;
    if (warp == 0) {
      // ---------------- producer: one lane per copy (issued in parallel) ----------------
      const int nsub = d / 64;
      for (int k = 0; k < ntile; ++k) {
        const uint32_t c = it + k, ts = c & 1, tph = (c >> 1) & 1;
        const uint32_t ks = c % a.NK, kph = (c / a.NK) & 1;
        const int j0 = (t0 + k) * kT;
        // position rows of the tile
        if (!__all_sync(0xffffffffu, mbar_wait(&trempty[ts], tph ^ 1))) {
          if (lane == 0) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
          }
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&trfull[ts], a.trig_stage);
        __syncwarp();
        uint8_t* trig_dst = sm + a.off_trig + ts * a.trig_stage;
        if (lane < nsub) tma_load_2d(trig_dst + lane * 16384, &trig_map, lane * 64, p0 + j0, &trfull[ts]);
        // key codes and metadata of its pages
        if (!__all_sync(0xffffffffu, mbar_wait(&kempty[ks], kph ^ 1))) {
          if (lane == 0) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
          }
          break;
        }
        const int nval = min(kT, L - j0);
        const int np = (nval + kPage - 1) / kPage;
        int* fl = flags + ks * kPagesPerTile;
        if (lane < kPagesPerTile) {
          int pid = -1;
          if (lane < np) {
            pid = bt_s[(j0 / kPage + lane) - t0 * kPagesPerTile];
            if (pid < 0 || pid >= a.n_pages) {
              set_status(a.status, STARKV_DEV_BAD_PAGE);
              pid = -1;
            }
          }
          fl[lane] = pid;
        }
        __syncwarp();
        const int nvalid =
            __popc(__ballot_sync(0xffffffffu, lane < kPagesPerTile && fl[lane < kPagesPerTile ? lane : 0] >= 0));
        if (lane == 0) mbar_arrive_expect_tx(&kfull[ks], (uint32_t)nvalid * (a.codes_page + a.meta_page));
        __syncwarp();
        if (lane < 2 * kPagesPerTile) {
          const int p = lane >> 1;
          const int pid = fl[p];
          if (pid >= 0) {
            if ((lane & 1) == 0)
              bulk_g2s(sm + a.off_codes + ks * a.codes_stage + p * a.codes_pitch,
                       a.k_codes + ((int64_t)pid * a.h_kv + kv0) * a.key.region_bytes, a.codes_page, &kfull[ks]);
            else if (a.meta_page)  // fp16 latents carry no metadata
              bulk_g2s(sm + a.off_meta + ks * a.meta_stage + p * a.meta_pitch,
                       a.k_meta + ((int64_t)pid * a.h_kv + kv0) * a.key.groups * kPage, a.meta_page, &kfull[ks]);
          }
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------- MMA issuer ----------------
        for (int k = 0; k < ntile; ++k) {
          const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;  // position stage = accumulator = c & 1
          if (!mbar_wait(&trfull[s], ph) || !mbar_wait(&tempty[s], ph ^ 1)) {
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
          mma_commit(&trempty[s]);
        }
      }
    } else if (RK == 64 && G == 16 && a.kvpc == 1 && a.hpc == 4) {
      // ---------------- epilogue, four query heads over one KV head (GQA) ----------------
      // Warp (q4, gq): tokens 32 q4 .. + 31 (its TMEM lane quarter) and channel
      // group gq (16 channels) of the shared key latent, for all four heads: the
      // codes are unpacked and dequantised once, z^ = code s + zp, and each head
      // takes 16 products from its G row.  The four groups' partial scores meet
      // in shared memory; after a barrier of the 16 epilogue warps each thread
      // finalises one (head, token).
      const int q4 = warp & 3, gq = (warp - 2) >> 2;
      const int t = q4 * 32 + lane;
      const int t16 = t % kPage, p = t / kPage;
      const int e = (warp - 2) * 32 + lane;
      const int fh = e >> 7, ft = e & 127;  // this thread's (head, token) to finalise
      float* red = reinterpret_cast<float*>(sm + a.off_red);
      float mfin = -INFINITY;
      for (int k = 0; k < ntile; ++k) {
        const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;
        const uint32_t ks = c % a.NK, kph = (c / a.NK) & 1;
        const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[s], ph) && mbar_wait(&kfull[ks], kph));
        if (!got && lane == 0) {
          set_status(a.status, kDevWaitTimeout);
          *failed = 1;
        }
        tc_fence_after();
        const int tile = t0 + k;
        const int j = tile * kT + t;
        const int jf = tile * kT + ft;
        const bool fvalid = jf < L && flags[ks * kPagesPerTile + ft / kPage] >= 0;
        float* rb = red + (c & 1) * (4 * kT);
        if (got) {
          const uint32_t trow = tmem + s * 256 + ((uint32_t)(q4 * 32) << 16) + gq * 16;
          const int pid = flags[ks * kPagesPerTile + p];
          float zh[16];
          if (j < L && pid >= 0) {
            const uint8_t* region = sm + a.off_codes + ks * a.codes_stage + p * a.codes_pitch;
            const uint32_t mw =
                reinterpret_cast<const uint32_t*>(sm + a.off_meta + ks * a.meta_stage + p * a.meta_pitch)[gq * kPage + t16];
            const float sc = __half2float(__ushort_as_half((unsigned short)(mw & 0xFFFF)));
            const float zp = __half2float(__ushort_as_half((unsigned short)(mw >> 16)));
            // x = 1 + code / 16 from the code bits under the mantissa of 1.0:
            // z^ = code s + zp = x (16 s) + (zp - 16 s)
            const float s16 = 16.f * sc, z0 = zp - s16;
            uint32_t w[2];
            if (gq < a.key.top_groups) {
              const uint2 u = *reinterpret_cast<const uint2*>(region + gq * 128 + 8 * t16);
              w[0] = u.x;
              w[1] = u.y;
            } else {
              const uint8_t* tl = region + a.key.top_groups * 128 + (gq - a.key.top_groups) * 96;
              const uint32_t lo = *reinterpret_cast<const uint32_t*>(tl + 4 * t16);
              const uint32_t hi = *reinterpret_cast<const uint16_t*>(tl + 64 + 2 * t16);
              w[0] = spread2_to_nibbles8(lo & 0xFFFFu) | (spread1_to_nibbles8(hi & 0xFFu) << 2);
              w[1] = spread2_to_nibbles8(lo >> 16) | (spread1_to_nibbles8(hi >> 8) << 2);
            }
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                const uint32_t bits = (cc >= 5 ? (w[q] >> (4 * cc - 19)) : (w[q] << (19 - 4 * cc))) & 0x00780000u;
                zh[q * 8 + cc] = fmaf(mant(bits), s16, z0);
              }
          } else {
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) zh[cc] = 0.f;
          }
#pragma unroll
          for (int hp = 0; hp < 4; hp += 2) {
            uint32_t g0[16], g1[16];
            tmem_issue_row<16>(trow + hp * 64, g0);
            tmem_issue_row<16>(trow + (hp + 1) * 64, g1);
            tmem_wait_row<16>(g0);
            tmem_wait_row<16>(g1);
            float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
            for (int cc = 0; cc < 16; cc += 2) {
              a0 = fmaf(zh[cc], __uint_as_float(g0[cc]), a0);
              a1 = fmaf(zh[cc + 1], __uint_as_float(g0[cc + 1]), a1);
              b0 = fmaf(zh[cc], __uint_as_float(g1[cc]), b0);
              b1 = fmaf(zh[cc + 1], __uint_as_float(g1[cc + 1]), b1);
            }
            atomicAdd(rb + hp * kT + t, a0 + a1);
            atomicAdd(rb + (hp + 1) * kT + t, b0 + b1);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[s]);
          mbar_arrive(&kempty[ks]);
        }
        // every group's partial is in; the failure flag is decided once for all 16 warps
        uint32_t stop;
        asm volatile(
            "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 512, p;\n selp.u32 %0, 1, 0, q;\n}\n"
            : "=r"(stop)
            : "r"((uint32_t)(!got || *failed))
            : "memory");
        if (stop) break;
        const float score = fvalid ? rb[fh * kT + ft] : -INFINITY;
        rb[fh * kT + ft] = 0.f;  // ready for the tile two ahead (a barrier of the next tile comes between)
        if (jf < L) a.S[((int64_t)b * a.H + h0 + fh) * a.tpad + jf] = score;
        mfin = fmaxf(mfin, score);
      }
      // this job's running maximum of head fh (one head per warp): one atomic per warp
      const float m = warp_max(mfin);
      if (lane == 0 && m != -INFINITY) atomicMax(&a.Mx[b * a.H + h0 + fh], ordered_bits(m));
    } else {
      // ---------------- epilogue: one thread per token ----------------
      const int q4 = warp & 3, hq = (warp - 2) >> 2;   // TMEM lane quarter, head quarter
      const int t = q4 * 32 + lane;
      const int t16 = t % kPage, p = t / kPage;
      const int hper = a.hpc / 4;  // heads per thread (<= 4)
      float mloc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // running maxima of this thread's heads
      for (int k = 0; k < ntile; ++k) {
        const uint32_t c = it + k, s = c & 1, ph = (c >> 1) & 1;
        const uint32_t ks = c % a.NK, kph = (c / a.NK) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&tfull[s], ph) && mbar_wait(&kfull[ks], kph))) {
          if (lane == 0) {
            set_status(a.status, kDevWaitTimeout);
            *failed = 1;
          }
          break;
        }
        tc_fence_after();
        const int tile = t0 + k;
        const int j = tile * kT + t;
        const int pid = flags[ks * kPagesPerTile + p];
        const bool valid = j < L && pid >= 0;
        const uint8_t* cstage = sm + a.off_codes + ks * a.codes_stage + p * a.codes_pitch;
        const uint32_t* mstage =
            reinterpret_cast<const uint32_t*>(sm + a.off_meta + ks * a.meta_stage + p * a.meta_pitch);
        const uint32_t trow = tmem + s * 256 + ((uint32_t)(q4 * 32) << 16);
        auto finish = [&](int i, float score) {  // i: this thread's head index (static)
          const int h = h0 + hq * hper + i;
          if (j < L) a.S[((int64_t)b * a.H + h) * a.tpad + j] = score;
          mloc[i] = fmaxf(mloc[i], score);
        };
        const int hl0 = hq * hper;
        if constexpr (RK >= 64 || G == 0) {
          // one RK-column row per head at a time
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            if (hh >= hper) break;
            uint32_t rA[RK];
            tmem_issue_row<RK>(trow + (hl0 + hh) * RK, rA);
            tmem_wait_row<RK>(rA);
            float sc = -INFINITY;
            if (valid) {
              const int kA = (h0 + hl0 + hh) / a.group - kv0;
              if constexpr (G == 0)
                sc = key_dot_fp16<RK>(cstage + kA * a.key.region_bytes, t16, rA);
              else
                sc = key_dot<RK, G>(cstage + kA * a.key.region_bytes, mstage + kA * a.key.groups * kPage,
                                    a.key.top_groups, t16, rA);
            }
            finish(hh, sc);
          }
        } else {
#pragma unroll
          for (int hh = 0; hh < 4; hh += 2) {
            if (hh >= hper) break;
            const int hA = hl0 + hh;
            const bool two = hh + 1 < hper;
            const int hB = two ? hA + 1 : hA;
            uint32_t rA[RK], rB[RK];
            tmem_issue_row<RK>(trow + hA * RK, rA);
            tmem_issue_row<RK>(trow + hB * RK, rB);
            tmem_wait_row<RK>(rA);
            tmem_wait_row<RK>(rB);
            float sA = -INFINITY, sB = -INFINITY;
            if (valid) {
              const int kA = (h0 + hA) / a.group - kv0, kB = (h0 + hB) / a.group - kv0;
              key_dot2<RK, G>(cstage + kA * a.key.region_bytes, mstage + kA * a.key.groups * kPage,
                              cstage + kB * a.key.region_bytes, mstage + kB * a.key.groups * kPage, a.key.top_groups,
                              t16, rA, rB, sA, sB);
            }
            finish(hh, sA);
            if (two) finish(hh + 1, sB);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[s]);
          mbar_arrive(&kempty[ks]);
        }
      }
      // this job's running maxima: one warp reduction and one atomic per head
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (i >= hper) break;
        const float m = warp_max(mloc[i]);
        if (lane == 0 && m != -INFINITY) atomicMax(&a.Mx[b * a.H + h0 + hq * hper + i], ordered_bits(m));
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
  int H, N, R, MT;        // heads, heads padded to the MMA's N, value rank, 128-channel M tiles
  int PS, nW, ST, NS;     // pages per stage, dequant warps (= MT * PS), tokens per stage, ring depth
  int max_pages, tpad, splits, stages_total, max_position;
  int64_t n_pages;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* pos0;  // as ScoreArgs (only their validity matters here)
  const int32_t* qpos;
  const uint8_t* v_codes;
  const uint32_t* v_meta;
  const unsigned int* Mx;  // [B][H] sequence-wide score maxima (ordered bits)
  float* part;   // [B][nclust][H][R] per-cluster sums (common maximum)
  float* lpart;  // [B][nclust][H]
  unsigned int* status;
  int CS, nclust;         // CTAs per cluster, clusters per sequence
  int balanced, batch, slots;  // splits per sequence by length (CS = 1): over `slots` CTAs
  int* vsplit;            // [B] each sequence's split count (balanced mode), for the projection
  uint32_t off_z, off_p, off_s, off_codes, off_meta, off_flags, off_bt, off_m, off_l, off_bar;
  uint32_t p_stage, s_box, s_box_bytes, s_stage;
  uint32_t codes_page, meta_page, codes_pitch, meta_pitch, codes_stage, meta_stage, tmem_cols;
};

constexpr int kVMaxWarps = 16;                      // dequant warps at most
constexpr int kVPWarps = 2;                         // P warps (each half of a stage's tokens)
constexpr int kVRoleWarps = 1 + kVPWarps;           // producer + P warps
constexpr int kVThreads = (kVRoleWarps + kVMaxWarps) * 32;
constexpr int kVMaxStages = 8;
constexpr uint32_t kZTile = kPage * 128 * 2;        // one page x one 128-channel M tile, fp16


// One CTA per (token split, sequence); the CS splits of a cluster add their
// sums on chip and write one partial.  Warp roles:
//   warp 0           producer: per stage of ST tokens, the score rows (TMA boxes
//                    of 32 tokens x H heads, 128-byte swizzle) and the value
//                    codes + metadata of its PS pages (bulk copies, one lane per
//                    copy), NS stages deep
//   warps 1..2       P: lane = head, each warp half of the stage's tokens;
//                    P[h, t] = exp2(s - M_h) as fp16 into a K-major tile, l_h
//                    summed in registers
//   warps 3..nW+2    dequant warp w = (M tile w % MT, page w / MT of the stage):
//                    dequantises its 16 tokens x 128 channels into its own Z tile
//                    and issues its own MMA  D_w[ch, h] += sum_t Z[t, ch] P[h, t]
//                    into its own TMEM columns (no cross-warp hand-off per tile)
// At the end the page accumulators of each M tile go to shared memory as
// [H][R] fp32, and CTA r of the cluster sums channel slice r over the cluster
// (distributed shared memory) into the partial.
__global__ void __launch_bounds__(kVThreads, 1)
    decode_values_kernel(const __grid_constant__ CUtensorMap s_map, const ValueArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + a.off_bar);
  uint64_t* cfull = bar;                     // [NS] stage landed
  uint64_t* cempty = cfull + kVMaxStages;    // [NS] stage read (P warps + dequant warps)
  uint64_t* pfull = cempty + kVMaxStages;    // [NS] P tile written
  uint64_t* pempty = pfull + kVMaxStages;    // [NS] MMAs reading the P tile done
  uint64_t* zempty = pempty + kVMaxStages;   // [nW] MMA reading warp w's Z tile done
  uint64_t* dfull = zempty + kVMaxWarps;     // every accumulator final
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dfull + 1);
  int* flags = reinterpret_cast<int*>(sm + a.off_flags);  // [NS][PS] page ids, -1 = skip
  int* bt_s = reinterpret_cast<int*>(sm + a.off_bt);      // this split's block-table entries
  float* Mh = reinterpret_cast<float*>(sm + a.off_m);     // [H]
  float* Lh = reinterpret_cast<float*>(sm + a.off_l);     // [H] this CTA's l
  float* accs = reinterpret_cast<float*>(sm);             // [H][R] this CTA's sums (after the pipeline)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const LatentGeom& V = a.val;
  const int NS = a.NS, PS = a.PS, ST = a.ST;
  pdl_wait();  // scores, their maxima and the appended codes (every CTA, even one that leaves early)
  pdl_launch_dependents();

  int L = decode_len(a.seq_lens, a.pos0, a.qpos, b, a.max_pages, a.max_position);
  const bool bad_len = L < 0;
  if (bad_len) {
    if (split == 0 && tid == 0) set_status(a.status, STARKV_DEV_BAD_SEQ_LEN);
    L = 0;
  }
  const int seq_stages = (L + ST - 1) / ST;
  const int clust = split / a.CS;
  int st_lo, st_hi;
  if (a.balanced) {
    // this sequence's share of the CTAs (CS = 1: a CTA beyond it leaves, no partial)
    __shared__ int ks_s;
    if (warp == 0) {
      const int k = value_splits_of(b, a.seq_lens, a.pos0, a.qpos, a.batch, a.max_pages, a.max_position, ST,
                                    a.slots, a.splits);
      if (lane == 0) {
        ks_s = k;
        if (split == 0) a.vsplit[b] = k;
      }
    }
    __syncthreads();
    const int k = ks_s;
    if (split >= k) return;
    st_lo = (int)((int64_t)split * seq_stages / k);
    st_hi = (int)((int64_t)(split + 1) * seq_stages / k);
  } else {
    // a cluster none of whose splits has tokens leaves as a whole (no partial)
    if ((int)((int64_t)clust * a.CS * a.stages_total / a.splits) >= seq_stages) return;
    st_lo = (int)((int64_t)split * a.stages_total / a.splits);
    st_hi = min((int)((int64_t)(split + 1) * a.stages_total / a.splits), seq_stages);
  }
  const int nst = st_hi > st_lo ? st_hi - st_lo : 0;
  const bool work = nst > 0;  // uniform across the CTA

  if (work && warp == 1) tmem_alloc(tslot, a.tmem_cols);
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], a.nW + kVPWarps);
      mbar_init(&pfull[s], kVPWarps);
      mbar_init(&pempty[s], a.nW);
    }
    for (int w = 0; w < a.nW; ++w) mbar_init(&zempty[w], 1);
    mbar_init(dfull, a.nW);
    fence_mbar_init();
  }
  // sequence-wide maxima per head (the common reference of every split; a
  // sequence with no finite score uses 0), this split's page ids, P tiles
  // zeroed once (rows >= H stay zero)
  for (int h = tid; h < a.H; h += blockDim.x) {
    const unsigned int o = a.Mx[b * a.H + h];
    const float m = o ? ordered_float(o) : -INFINITY;
    Mh[h] = m == -INFINITY ? 0.f : m;
    Lh[h] = 0.f;
  }
  if (work) {
    const int p0 = st_lo * PS;
    const int np_split = min(nst * PS, (L + kPage - 1) / kPage - p0);
    for (int e = tid; e < np_split; e += blockDim.x) bt_s[e] = a.block_table[(int64_t)b * a.max_pages + p0 + e];
    for (int i = tid; i < (int)(NS * a.p_stage / 16); i += blockDim.x)
      reinterpret_cast<uint4*>(sm + a.off_p)[i] = make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  bool ok = true;

  if (work) {
    const uint32_t tmem = *tslot;
    if (warp == 0) {
      // ---------------- producer: one lane per copy (a bulk copy costs its issuing
      // thread about as long as the next copy's latency would, so issue in parallel)
      const int nbox = ST / 32;
      for (int k = 0; k < nst; ++k) {
        const int cs = k % NS;
        if (!__all_sync(0xffffffffu, mbar_wait(&cempty[cs], ((k / NS) & 1) ^ 1))) {
          ok = false;
          break;
        }
        const int j0 = (st_lo + k) * ST;
        const int np = min(PS, (L - j0 + kPage - 1) / kPage);
        int* fl = flags + cs * PS;
        if (lane < PS) {
          int pid = -1;
          if (lane < np) {
            pid = bt_s[k * PS + lane];
            if (pid < 0 || pid >= a.n_pages) {
              set_status(a.status, STARKV_DEV_BAD_PAGE);
              pid = -1;
            }
          }
          fl[lane] = pid;
        }
        __syncwarp();
        const int nvalid = __popc(__ballot_sync(0xffffffffu, lane < PS && fl[lane < PS ? lane : 0] >= 0));
        if (lane == 0)
          mbar_arrive_expect_tx(&cfull[cs], (uint32_t)nbox * a.s_box_bytes + (uint32_t)nvalid * (a.codes_page + a.meta_page));
        __syncwarp();
        uint8_t* sdst = sm + a.off_s + cs * a.s_stage;
        for (int i = lane; i < nbox + 2 * PS; i += 32) {
          if (i < nbox) {
            tma_load_2d(sdst + i * a.s_box, &s_map, j0 + 32 * i, b * a.H, &cfull[cs]);
          } else {
            const int p = (i - nbox) >> 1;
            const int pid = fl[p];
            if (pid >= 0) {
              if (((i - nbox) & 1) == 0)
                bulk_g2s(sm + a.off_codes + cs * a.codes_stage + p * a.codes_pitch,
                         a.v_codes + (int64_t)pid * V.region_bytes, a.codes_page, &cfull[cs]);
              else if (a.meta_page)  // fp16 latents carry no metadata
                bulk_g2s(sm + a.off_meta + cs * a.meta_stage + p * a.meta_pitch,
                         a.v_meta + (int64_t)pid * V.groups * kPage, a.meta_page, &cfull[cs]);
            }
          }
        }
      }
    } else if (warp < kVRoleWarps) {
      // ---------------- P: lane = head (and head + 32), this warp's half of the tokens
      const int pw = warp - 1;
      const int tspan = ST / kVPWarps;  // a multiple of 8
      float2 lacc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      float mh[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) mh[i] = lane + 32 * i < a.H ? Mh[lane + 32 * i] : 0.f;
      for (int k = 0; k < nst && ok; ++k) {
        const int cs = k % NS;
        const uint32_t ph = (k / NS) & 1;
        const bool got = mbar_wait(&cfull[cs], ph) && mbar_wait(&pempty[cs], ph ^ 1);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const int j0 = (st_lo + k) * ST;
        const int* fl = flags + cs * PS;
        bool full = j0 + ST <= L;
        for (int p = 0; p < PS; ++p) full = full && fl[p] >= 0;
        const uint8_t* sst = sm + a.off_s + cs * a.s_stage;
        uint8_t* pt = sm + a.off_p + cs * a.p_stage;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int h = lane + 32 * i;
          if (h < a.H) {
            for (int t0 = pw * tspan; t0 < (pw + 1) * tspan; t0 += 8) {
              // 8 tokens t0..t0+7 (one page): two 16-byte chunks of the swizzled 32-token score row
              const uint8_t* row = sst + (t0 >> 5) * a.s_box + h * 128;
              const int c = (t0 & 31) >> 2;
              const float4 v0 = *reinterpret_cast<const float4*>(row + ((c ^ (h & 7)) << 4));
              const float4 v1 = *reinterpret_cast<const float4*>(row + (((c + 1) ^ (h & 7)) << 4));
              float pv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
              for (int u = 0; u < 8; ++u) pv[u] = ex2_approx(pv[u] - mh[i]);
              if (!full) {
                const int lim = fl[t0 >> 4] >= 0 ? L - (j0 + t0) : 0;  // tokens t0 + u valid for u < lim
#pragma unroll
                for (int u = 0; u < 8; ++u) pv[u] = u < lim ? pv[u] : 0.f;
              }
              uint32_t w4[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                w4[u] = h2bits(__floats2half2_rn(pv[2 * u], pv[2 * u + 1]));
                lacc[i].x += pv[2 * u];
                lacc[i].y += pv[2 * u + 1];
              }
              *reinterpret_cast<uint4*>(pt + sw128_kmajor_offset(h, t0, a.N)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pfull[cs]);
          mbar_arrive(&cempty[cs]);
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (lane + 32 * i < a.H) atomicAdd(&Lh[lane + 32 * i], lacc[i].x + lacc[i].y);
    } else if (warp - kVRoleWarps < a.nW) {
      // ---------------- dequant + MMA: 16 tokens x 128 channels per stage
      const int w = warp - kVRoleWarps;
      const int mt = w % a.MT, pg = w / a.MT;
      const int t16 = lane & 15, gsel = lane >> 4;
      uint8_t* zt = sm + a.off_z + w * kZTile;
      const uint32_t zaddr = smem_u32(zt);
      const uint32_t idesc = make_idesc_f16(128, a.N, true, false);
      const uint32_t dcol = tmem + (uint32_t)(w * a.N);
      for (int k = 0; k < nst && ok; ++k) {
        const int cs = k % NS;
        const uint32_t ph = (k / NS) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&cfull[cs], ph))) {
          ok = false;
          break;
        }
        const int j0 = (st_lo + k) * ST;
        const bool tvalid = flags[cs * PS + pg] >= 0 && j0 + pg * kPage + t16 < L;
        const uint8_t* region = sm + a.off_codes + cs * a.codes_stage + pg * a.codes_pitch;
        const uint32_t* meta =
            reinterpret_cast<const uint32_t*>(sm + a.off_meta + cs * a.meta_stage + pg * a.meta_pitch);
        uint4 cz[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int gi = mt * 8 + gsel + 2 * i;
          cz[2 * i] = make_uint4(0, 0, 0, 0);
          cz[2 * i + 1] = make_uint4(0, 0, 0, 0);
          if (tvalid && gi < V.groups && V.fp16) {
            // unquantised latents: the row of the group's tile, channels in order
            const uint4* row = reinterpret_cast<const uint4*>(region + gi * 512 + t16 * 32);
            cz[2 * i] = row[0];
            cz[2 * i + 1] = row[1];
          } else if (tvalid && gi < V.groups) {
            const uint32_t mw = meta[gi * kPage + t16];
            if (gi < V.top_groups)
              dequant16_4bit(region + gi * 128 + 8 * t16, mw, cz[2 * i], cz[2 * i + 1]);
            else
              dequant16_3bit(region + V.top_groups * 128 + (gi - V.top_groups) * 96, t16, mw, cz[2 * i],
                             cz[2 * i + 1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&cempty[cs]);
        if (!__all_sync(0xffffffffu, mbar_wait(&zempty[w], (k & 1) ^ 1))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m0 = (gsel + 2 * i) * 16;
          *reinterpret_cast<uint4*>(zt + sw128_mnmajor_offset(t16, m0, 2)) = cz[2 * i];
          *reinterpret_cast<uint4*>(zt + sw128_mnmajor_offset(t16, m0 + 8, 2)) = cz[2 * i + 1];
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (mbar_wait(&pfull[cs], ph)) {
            tc_fence_after();
            const int kofs = pg * kPage;  // this page's tokens within the stage's P tile
            const uint32_t pa =
                smem_u32(sm + a.off_p + cs * a.p_stage) + (uint32_t)((kofs >> 6) * a.N * 128 + (kofs & 63) * 2);
            mma_f16(dcol, make_sdesc(zaddr, 1024, 2048, 2), make_sdesc(pa, 16, 1024, 2), idesc, k > 0 ? 1u : 0u);
            mma_commit(&zempty[w]);
            mma_commit(&pempty[cs]);
          } else {
            ok = false;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0) mma_commit(dfull);  // arrives once this warp's MMAs are complete
      __syncwarp();
    }
    if (!ok && lane == 0) set_status(a.status, kDevWaitTimeout);

    // ---------------- drain: page accumulators of each M tile, summed, into accs[h][ch]
    const bool drained = __all_sync(0xffffffffu, mbar_wait_poll(dfull, 0));
    tc_fence_after();
    const int groups4 = (int)(blockDim.x / 32) / 4;
    if ((warp >> 2) < groups4) {
      const int q4 = warp & 3;
      for (int mt = warp >> 2; mt < a.MT; mt += groups4) {
        const int mpos = mt * 128 + q4 * 32 + lane;
        const int gidx = mpos >> 4;
        const int ch = V.fp16 ? mpos : gidx * 16 + value_channel_of_position(mpos & 15, gidx < V.top_groups);
        for (int c0 = 0; c0 < a.N; c0 += 16) {
          float acc[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = 0.f;
          if (drained) {
            for (int ps = 0; ps < PS; ++ps) {
              uint32_t r[16];
              asm volatile(
                  "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
                  "[%16];"
                  : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                    "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                    "=r"(r[15])
                  : "r"(tmem + (uint32_t)((mt + a.MT * ps) * a.N + c0) + ((uint32_t)(q4 * 32) << 16)));
              tmem_wait_row<16>(r);
#pragma unroll
              for (int i = 0; i < 16; ++i) acc[i] += __uint_as_float(r[i]);
            }
          }
          if (ch < a.R) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int h = c0 + i;
              if (h < a.H) accs[h * a.R + ch] = acc[i];
            }
          }
        }
      }
    }
    if (!drained && lane == 0) set_status(a.status, kDevWaitTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, a.tmem_cols);
    }
  } else {
    // no tokens in this split: contribute zeros to the cluster sum
    for (int i = tid; i < a.H * a.R / 4; i += blockDim.x) reinterpret_cast<float4*>(accs)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // ---------------- cluster sum: CTA r adds channel slice r over the cluster
  cluster_sync();
  {
    const uint32_t r = cluster_rank();
    const int slice = a.R / a.CS;  // multiple of 4
    const int per_h = slice / 4;
    float* prow = a.part + ((int64_t)b * a.nclust + clust) * a.H * a.R;
    for (int e = tid; e < a.H * per_h; e += blockDim.x) {
      const int h = e / per_h, c4 = (e % per_h) * 4 + (int)r * slice;
      const float* src = accs + h * a.R + c4;
      float4 v[8];  // every peer's value in flight at once (cluster size <= 8)
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < a.CS) v[q] = dsmem_ld_f4(dsmem_addr(src, (uint32_t)q));
      float4 sum = v[0];
#pragma unroll
      for (int q = 1; q < 8; ++q) {
        if (q < a.CS) {
          sum.x += v[q].x;
          sum.y += v[q].y;
          sum.z += v[q].z;
          sum.w += v[q].w;
        }
      }
      *reinterpret_cast<float4*>(prow + (int64_t)h * a.R + c4) = sum;
    }
    if (r == 0) {
      for (int h = tid; h < a.H; h += blockDim.x) {
        float l = 0.f;
        for (int q = 0; q < a.CS; ++q) l += dsmem_ld_f32(dsmem_addr(Lh + h, (uint32_t)q));
        a.lpart[((int64_t)b * a.nclust + clust) * a.H + h] = l;
      }
    }
  }
  cluster_sync();  // peers' shared memory stays in place until every CTA has read it
}

// ===========================================================================
// C. projection: o_h = (acc_h / l_h) B'_v[:, kv(h)]
// ===========================================================================
struct ProjArgs {
  int H, h_kv, group, d, R;
  int splits, stages_total, st;  // value-kernel splits, stages and tokens per stage
  int cs, nclust;                // splits per cluster, clusters (partials) per sequence
  const int* vsplit;             // [B] partials per sequence (balanced value splits), or NULL
  const float* part;     // [B][splits][H][R]
  const float* lpart;    // [B][splits][H]
  float* oacc;           // [B][H][d] fp32 sums (zeroed by the score kernel)
  unsigned int* ocnt;    // [H][ceil(B/16)] arrival counters (zeroed by the score kernel)
  const int32_t* seq_lens;
  const int32_t* pos0;  // as ScoreArgs (only their validity matters here)
  const int32_t* qpos;
  int tpad, max_pages, max_position;
  const __half* Bv16;
  __nv_bfloat16* out;
  // slice mode (sequence sharding): fp32 outputs normalised within the slice,
  // and the slice's softmax statistics, instead of `out`
  const unsigned int* Mx;  // [B][H] score maxima (ordered bits, log2 domain)
  float* out_o;            // [B][H][d] or NULL
  float* out_ml;           // [B][H][2]: (maximum, sum of 2^(s - maximum)) or NULL
};

constexpr int kProjM = 16;   // sequences per projection CTA (the MMA's M)
constexpr int kProjC = 128;  // latent channels per projection CTA
constexpr int kProjVecLoads = kProjC * (128 / 8) / 256;  // 16-byte B'_v loads per thread at d = 128

// grid (H, R / kc, ceil(B / 16)), 256 threads, kc = 128 channels (64 when R is
// not a multiple of 128).  Every load of the CTA (its
// B'_v slice, the partial sums and l of its sequences) is issued up front; then
// o_lat[16 seq x 128] (fp16, = acc / l) . B'_v[128 x d] on mma.sync (warp w owns
// output columns [16 w, 16 w + 16); d = 64 leaves warps 4..7 idle), added into
// the fp32 sums, and the last CTA of a (head, sequence block) to arrive writes
// the bf16 output (arrival counter, no waiting).
__global__ void __launch_bounds__(256) decode_project_kernel(const ProjArgs a, int batch, int kc) {
  __shared__ __align__(16) __half As[kProjM][kProjC + 8];
  __shared__ __align__(16) __half Bs[kProjC][128 + 8];
  __shared__ float linv[kProjM];
  __shared__ float lsum[kProjM];
  __shared__ int nparts_s[kProjM];
  __shared__ int last;
  const int R = a.R, d = a.d;
  const int h = blockIdx.x, ch0 = blockIdx.y * kc, bc = blockIdx.z;
  const int b0 = bc * kProjM;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kv = h / a.group;
  const int ldg = a.h_kv * d;
  // partials of sequence b: clusters whose first split has tokens (a prefix)
  if (tid < kProjM) {
    const int b = b0 + tid;
    int np = 0;
    if (b < batch) {
      int L = decode_len(a.seq_lens, a.pos0, a.qpos, b, a.max_pages, a.max_position);
      if (L < 0) L = 0;
      const int nst = (L + a.st - 1) / a.st;
      const int nsp = nst > 0 ? min(a.splits, (int)(((int64_t)nst * a.splits - 1) / a.stages_total) + 1) : 0;
      np = (nsp + a.cs - 1) / a.cs;  // (balanced splits: read after the wait below)
    }
    nparts_s[tid] = np;
  }
  // B'_v rows of this slice straight into shared memory (they do not depend on
  // the kernels before, so this overlaps the value kernel's tail).  All of a
  // thread's loads are issued before the first store.
  {
    const int nvec = kc * (d / 8);
    uint4 v[kProjVecLoads];
#pragma unroll
    for (int i = 0; i < kProjVecLoads; ++i) {
      const int e = tid + i * 256, r = e / (d / 8), q8 = e % (d / 8);
      if (e < nvec) v[i] = __ldg(reinterpret_cast<const uint4*>(a.Bv16 + (int64_t)(ch0 + r) * ldg + kv * d + q8 * 8));
    }
#pragma unroll
    for (int i = 0; i < kProjVecLoads; ++i) {
      const int e = tid + i * 256, r = e / (d / 8), q8 = e % (d / 8);
      if (e < nvec) *reinterpret_cast<uint4*>(&Bs[r][q8 * 8]) = v[i];
    }
  }
  pdl_wait();  // partial sums, l and the zeroed accumulators
  pdl_launch_dependents();
  // value splits shared out by length: the value kernel recorded each sequence's count
  if (a.vsplit && tid < kProjM && b0 + tid < batch) nparts_s[tid] = a.vsplit[b0 + tid];
  __syncthreads();
  if (tid < kProjM) {
    const int b = b0 + tid, np = nparts_s[tid];
    float l = 0.f;
    for (int sp0 = 0; sp0 < np; sp0 += 4) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = sp0 + u < np ? __ldcg(a.lpart + ((int64_t)b * a.nclust + sp0 + u) * a.H + h) : 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) l += v[u];
    }
    linv[tid] = l > 0.f ? 1.f / l : 0.f;
    lsum[tid] = l;
  }
  // o_lat sums: 2 items of 4 channels per thread (16 sequences x 32 quads),
  // added in partial order; both items' loads of a round are in flight together
  float4 acc[2];
  const float* base[2];
  int np[2];
  const int items = kProjM * (kc / 4);
  const int64_t stride = (int64_t)a.H * R;
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int e = tid + it * 256;
    const int r = e / (kc / 4), c4 = (e % (kc / 4)) * 4;
    const int b = b0 + r;
    acc[it] = make_float4(0.f, 0.f, 0.f, 0.f);
    np[it] = (e < items && b < batch) ? nparts_s[r] : 0;
    base[it] = a.part + ((int64_t)b * a.nclust * a.H + h) * R + ch0 + c4;
  }
  for (int sp0 = 0; sp0 < max(np[0], np[1]); sp0 += 4) {
    float4 v[2][4];
#pragma unroll
    for (int it = 0; it < 2; ++it)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[it][u] = sp0 + u < np[it] ? __ldcg(reinterpret_cast<const float4*>(base[it] + (sp0 + u) * stride))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int it = 0; it < 2; ++it)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[it].x += v[it][u].x;
        acc[it].y += v[it][u].y;
        acc[it].z += v[it][u].z;
        acc[it].w += v[it][u].w;
      }
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int e = tid + it * 256;
    if (e >= items) break;
    const int r = e / (kc / 4), c4 = (e % (kc / 4)) * 4;
    const float li = linv[r];
    *reinterpret_cast<__half2*>(&As[r][c4]) = __floats2half2_rn(acc[it].x * li, acc[it].y * li);
    *reinterpret_cast<__half2*>(&As[r][c4 + 2]) = __floats2half2_rn(acc[it].z * li, acc[it].w * li);
  }
  __syncthreads();
  float c[2][4] = {};
  if (warp * 16 < d) {
#pragma unroll 4
    for (int kk = 0; kk < kc; kk += 16) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sm100::smem_u32(&As[lane & 15][kk + (lane >> 4) * 8]), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0r, b1r;
        ldsm_x2_t(sm100::smem_u32(&Bs[kk + (lane & 15)][warp * 16 + nt * 8]), b0r, b1r);
        mma16816(c[nt], a0, a1, a2, a3, b0r, b1r);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int col = warp * 16 + nt * 8 + (lane & 3) * 2;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int b = b0 + (lane >> 2) + hf * 8;
        if (b < batch)
          atomicAdd(reinterpret_cast<float2*>(a.oacc + ((int64_t)b * a.H + h) * d + col),
                    make_float2(c[nt][hf * 2], c[nt][hf * 2 + 1]));
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&a.ocnt[h * gridDim.z + bc], 1u) == gridDim.y - 1;
  __syncthreads();
  if (last) {
    __threadfence();
    // 4 columns per item, both items' loads before the stores
    float4 v[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int e = (tid + i * 256) * 4, b = b0 + e / d;
      if (e < kProjM * d && b < batch)
        v[i] = __ldcg(reinterpret_cast<const float4*>(a.oacc + ((int64_t)b * a.H + h) * d + e % d));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int e = (tid + i * 256) * 4, b = b0 + e / d;
      if (e < kProjM * d && b < batch) {
        if (a.out_o) {
          *reinterpret_cast<float4*>(a.out_o + ((int64_t)b * a.H + h) * d + e % d) = v[i];
        } else {
          __nv_bfloat16* o = a.out + ((int64_t)b * a.H + h) * d + e % d;
          o[0] = __float2bfloat16_rn(v[i].x);
          o[1] = __float2bfloat16_rn(v[i].y);
          o[2] = __float2bfloat16_rn(v[i].z);
          o[3] = __float2bfloat16_rn(v[i].w);
        }
      }
    }
    if (a.out_ml && tid < kProjM && b0 + tid < batch) {
      // the slice's softmax statistics: maximum (log2 domain) and sum; an empty slice has (-inf, 0)
      const int b = b0 + tid;
      const unsigned int mo = a.Mx[b * a.H + h];
      const float m = (mo && lsum[tid] > 0.f) ? ordered_float(mo) : -INFINITY;
      *reinterpret_cast<float2*>(a.out_ml + ((int64_t)b * a.H + h) * 2) = make_float2(m, lsum[tid] > 0.f ? lsum[tid] : 0.f);
    }
  }
}

// ===========================================================================
// merge of slice results (sequence sharding): the softmax partition identity
//   o = sum_r 2^(m_r - M) l_r o_r / sum_r 2^(m_r - M) l_r,  M = max_r m_r
// one thread per (sequence, head, 4 output columns)
// ===========================================================================
__global__ void merge_slices_kernel(const float* __restrict__ o_parts, const float* __restrict__ ml_parts, int n_parts,
                                    int64_t bh, int d, __nv_bfloat16* __restrict__ out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q4 = d / 4;
  if (idx >= bh * q4) return;
  const int64_t r = idx / q4;
  const int c = (int)(idx % q4) * 4;
  float M = -INFINITY;
  for (int p = 0; p < n_parts; ++p) {
    const float2 ml = *reinterpret_cast<const float2*>(ml_parts + ((int64_t)p * bh + r) * 2);
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
    for (int p = 0; p < n_parts; ++p) {
      const float2 ml = *reinterpret_cast<const float2*>(ml_parts + ((int64_t)p * bh + r) * 2);
      if (!(ml.y > 0.f)) continue;
      const float w = exp2f(ml.x - M) * ml.y;
      const float4 o = *reinterpret_cast<const float4*>(o_parts + ((int64_t)p * bh + r) * d + c);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
      den += w;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16* o = out + r * d + c;
  o[0] = __float2bfloat16_rn(acc.x * inv);
  o[1] = __float2bfloat16_rn(acc.y * inv);
  o[2] = __float2bfloat16_rn(acc.z * inv);
  o[3] = __float2bfloat16_rn(acc.w * inv);
}

cudaError_t launch_merge_slices(const float* o_parts, const float* ml_parts, int n_parts, int64_t bh, int d,
                                __nv_bfloat16* out, cudaStream_t s) {
  const int64_t n = bh * (d / 4);
  if (n == 0) return cudaSuccess;
  merge_slices_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(o_parts, ml_parts, n_parts, bh, d, out);
  return cudaGetLastError();
}

// ===========================================================================
// host side
// ===========================================================================
// Query heads per score CTA: up to 256 accumulator columns (hpc * r_k); with
// fp16 key latents also at most 32 KiB of key pages per 128-token stage.
static int score_hpc(const starkv_config& cfg) {
  const int rk = cfg.rank_k;
  const int group = cfg.num_q_heads / cfg.num_kv_heads;
  int hpc = (256 / rk) < cfg.num_q_heads ? 256 / rk : cfg.num_q_heads;
  if (cfg.flags & STARKV_FLAG_FP16_LATENT)
    while (hpc > 4 && hpc > group && kPagesPerTile * (hpc / group) * 32 * rk > 32768) hpc /= 2;
  return hpc;
}

bool tc_decode_supported(const starkv_config& cfg) {
  const int rk = cfg.rank_k;
  if (rk != 16 && rk != 32 && rk != 64) return false;
  const int hpc = score_hpc(cfg);
  const int group = cfg.num_q_heads / cfg.num_kv_heads;
  if (cfg.num_q_heads % hpc != 0 || hpc % 4 != 0) return false;
  if (hpc % group != 0 && group % hpc != 0) return false;
  if (group > hpc) return false;  // a CTA's heads must cover whole KV heads
  if (cfg.num_q_heads > 64) return false;
  if (cfg.rank_v % 64 != 0) return false;  // projection CTAs own 128- or 64-channel slices
  // value kernel: at least two pages per stage with one N-column accumulator per warp
  const int N = ((cfg.num_q_heads + 15) / 16) * 16;
  const int nw_max = (512 / N) < kVMaxWarps ? 512 / N : kVMaxWarps;
  if (((cfg.rank_v + 127) / 128) * 2 > nw_max) return false;
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

// Shared-memory layout of the value kernel for a given split count.
struct VSmem {
  int NS;
  uint32_t off_z, off_p, off_s, off_codes, off_meta, off_flags, off_bt, off_m, off_l, off_bar;
  uint32_t p_stage, s_box, s_box_bytes, s_stage, codes_page, meta_page, codes_pitch, meta_pitch, codes_stage,
      meta_stage, tmem_cols;
  size_t smem;
};

bool value_smem(const Ctx& c, int N, int nW, int PS, int ST, int stages_total, int splits, VSmem& v) {
  const starkv_config& f = c.cfg;
  v.codes_page = c.val.region_bytes;
  v.meta_page = c.val.fp16 ? 0 : c.val.groups * kPage * 4;
  v.codes_pitch = v.codes_page + 64;
  v.meta_pitch = v.meta_page + 64;
  v.codes_stage = PS * v.codes_pitch;
  v.meta_stage = PS * v.meta_pitch;
  v.s_box_bytes = (uint32_t)f.num_q_heads * 128;       // 32 fp32 scores x H rows
  v.s_box = (v.s_box_bytes + 1023) / 1024 * 1024;      // swizzled boxes start 1024-aligned
  v.s_stage = (uint32_t)(ST / 32) * v.s_box;
  v.p_stage = (uint32_t)N * (ST > 64 ? ST : 64) * 2;   // K-major fp16, 64-token rows
  uint32_t cols = 32;
  while (cols < (uint32_t)(nW * N)) cols <<= 1;
  v.tmem_cols = cols;
  const uint32_t bt_bytes = (uint32_t)(((stages_total + splits - 1) / splits + 1) * PS * 4);
  const uint32_t fixed = (uint32_t)nW * kZTile + kVMaxStages * PS * 4 + bt_bytes + N * 8 + 64 * 8 + 1024 + 64;
  const uint32_t per_stage = v.p_stage + v.s_stage + v.codes_stage + v.meta_stage;
  const uint32_t budget = 227u * 1024u;
  int ns = fixed < budget ? (int)((budget - fixed) / per_stage) : 0;
  if (ns > kVMaxStages) ns = kVMaxStages;
  if (ns < 2) return false;
  v.NS = ns;
  uint32_t o = 0;
  v.off_z = o;
  o += nW * kZTile;
  v.off_p = o;
  o += ns * v.p_stage;
  v.off_s = o;
  o += ns * v.s_stage;
  v.off_codes = o;
  o += ns * v.codes_stage;
  v.off_meta = o;
  o += ns * v.meta_stage;
  v.off_flags = o;
  o += kVMaxStages * PS * 4;
  v.off_bt = (o + 15) / 16 * 16;
  o = v.off_bt + bt_bytes;
  v.off_m = (o + 15) / 16 * 16;
  o = v.off_m + N * 4;
  v.off_l = o;
  o += N * 4;
  v.off_bar = (o + 15) / 16 * 16;
  o = v.off_bar + 64 * 8;
  v.smem = o + 1024;
  // the CTA's [H][R] sums reuse the pipeline's buffers, below the page table and barriers
  return (size_t)f.num_q_heads * f.rank_v * 4 <= v.off_flags;
}

// Clusters of `cs` value CTAs that fit on the device at once (cached per device).
int value_max_clusters(int cs, int threads, size_t smem) {
  struct Entry {
    int dev, cs, threads;
    size_t smem;
    int n;
  };
  static Entry cache[64];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].cs == cs && cache[i].threads == threads && cache[i].smem == smem)
      return cache[i].n;
  int n = 0;
  if (cudaFuncSetAttribute(decode_values_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, decode_values_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  if (used < 64) cache[used++] = Entry{dev, cs, threads, smem, n};
  return n;
}

struct TcLayout {
  int hpc, kvpc, ncols, HG, tiles_per_seq, tpad, splits, stages_total, N, MT;
  int PS, nW, ST;  // value kernel: pages per stage, dequant warps, tokens per stage
  int CS, nclust;  // value kernel: CTAs per cluster (splits reduced on chip), clusters per sequence
  int balanced, slots;  // value kernel: splits per sequence by length over `slots` CTAs (CS = 1)
  VSmem vs;        // value kernel shared memory
  bool ok;         // a valid value-kernel configuration exists
  size_t off_S, off_mx, off_acc, off_l, off_w, off_oacc, off_ocnt, off_vsplit, w_bytes, ws;
};

TcLayout tc_layout(const Ctx& c, int batch, int max_pages) {
  TcLayout t;
  const starkv_config& f = c.cfg;
  t.hpc = score_hpc(f);
  t.kvpc = t.hpc / c.group;
  t.ncols = t.hpc * f.rank_k;
  t.HG = f.num_q_heads / t.hpc;
  t.tiles_per_seq = (max_pages * kPage + kT - 1) / kT;
  t.tpad = t.tiles_per_seq * kT;
  t.N = ((f.num_q_heads + 15) / 16) * 16;
  t.MT = (f.rank_v + 127) / 128;
  {
    // dequant warps = M tiles x pages per stage, each with N TMEM columns (<= 512 in all)
    const int nw_max = (512 / t.N) < kVMaxWarps ? 512 / t.N : kVMaxWarps;
    int ps = 1;
    while (t.MT * ps * 2 <= nw_max) ps *= 2;
    t.PS = ps;
    t.nW = t.MT * ps;
    t.ST = kPage * ps;
  }
  t.stages_total = (t.tpad + t.ST - 1) / t.ST;
  {
    // Splits per sequence (one CTA per SM: stay within a single wave) and
    // cluster size: clusters of CS splits add their sums on chip, so only
    // splits / CS partials per sequence cross HBM (written, then read by the
    // projection).  A cluster must fit in one GPC, so fewer clusters of 8 than
    // of 2 are resident at once; the split count keeps every cluster of the
    // grid resident.  Pick the pair with the least estimated time: value bytes
    // over the SMs in use plus the partials' traffic.
    const int sms = sm_count();
    const int bt = batch > 0 ? batch : 1;
    int s0 = sms / bt;
    if (s0 > t.stages_total) s0 = t.stages_total;
    if (s0 < 1) s0 = 1;
    const double tok_bytes =
        (double)c.val.region_bytes / kPage + (c.val.fp16 ? 0.0 : c.val.groups * 4.0) + f.num_q_heads * 4.0;
    const double work = (double)bt * t.tpad * tok_bytes;
    const double part_unit = 2.0 * f.num_q_heads * f.rank_v * 4.0;
    const int threads = (kVRoleWarps + t.nW) * 32;
    VSmem probe;  // shared memory at the largest split count considered (for the residency query)
    // Value ranks up to 512 (a split's partial at most 64 KiB per head set):
    // each sequence gets CTAs in proportion to its length, one per SM in all,
    // and writes one partial per CTA (no cluster sums); the kernel computes the
    // shares from the sequence lengths.  A CTA may then hold a whole sequence.
    t.balanced = 0;
    t.slots = sms;
    if (f.rank_v <= 512 && bt >= 2) {
      int cap = 2 * ((sms + bt - 1) / bt);
      if (cap > t.stages_total) cap = t.stages_total;
      if (cap < 1) cap = 1;
      if (value_smem(c, t.N, t.nW, t.PS, t.ST, t.stages_total, 1, t.vs)) {
        t.ok = true;
        t.balanced = 1;
        t.splits = cap;
        t.CS = 1;
      }
    }
    if (!t.balanced) t.ok = value_smem(c, t.N, t.nW, t.PS, t.ST, t.stages_total, s0, probe);
    while (!t.ok && s0 < t.stages_total) {  // very long contexts: more splits, smaller page tables
      s0 = s0 * 2 < t.stages_total ? s0 * 2 : t.stages_total;
      t.ok = value_smem(c, t.N, t.nW, t.PS, t.ST, t.stages_total, s0, probe);
    }
    double best = -1.0;
    if (!t.balanced) {
      t.splits = 1;
      t.CS = 1;
    }
    for (int cs = 8; cs >= 1 && t.ok && !t.balanced; cs >>= 1) {
      int sp = (s0 / cs) * cs;
      if (cs > 1 && bt * (sp / cs) > 0) {
        const int resident = value_max_clusters(cs, threads, probe.smem);
        const int per_seq = resident / bt;  // clusters per sequence that stay resident
        if (sp / cs > per_seq) sp = per_seq * cs;
      }
      if (sp < cs || sp == 0) continue;
      const double used = (double)bt * sp < sms ? (double)bt * sp / sms : 1.0;
      const double cost = work / used + (double)bt * (sp / cs) * part_unit;
      if (best < 0.0 || cost < best) {
        best = cost;
        t.splits = sp;
        t.CS = cs;
      }
    }
    // a split's block-table entries live in shared memory: long contexts need
    // enough splits (in whole clusters) for that table to fit
    if (t.ok && !t.balanced) {
      t.ok = value_smem(c, t.N, t.nW, t.PS, t.ST, t.stages_total, t.splits, t.vs);
      while (!t.ok && t.splits < t.stages_total) {
        t.splits += t.CS;
        t.ok = value_smem(c, t.N, t.nW, t.PS, t.ST, t.stages_total, t.splits, t.vs);
      }
    }
    t.nclust = t.splits / t.CS;
  }
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t o = 0;
  t.off_S = o;
  o += al((size_t)batch * f.num_q_heads * t.tpad * 4);
  t.off_mx = o;
  o += al((size_t)batch * f.num_q_heads * 4);
  t.off_acc = o;
  o += al((size_t)batch * t.nclust * f.num_q_heads * f.rank_v * 4);
  t.off_l = o;
  o += al((size_t)batch * t.nclust * f.num_q_heads * 4);
  t.w_bytes = (size_t)t.ncols * f.head_dim * 2;
  t.off_w = o;
  o += al((size_t)batch * t.HG * t.w_bytes);
  t.off_oacc = o;
  o += al((size_t)batch * f.num_q_heads * f.head_dim * 4);
  t.off_ocnt = o;
  o += al((size_t)f.num_q_heads * ((batch + 15) / 16) * 4);
  t.off_vsplit = o;
  o += al((size_t)batch * 4);
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

template <int RK, int G>
static cudaError_t launch_scores_g(const Ctx& c, const ScoreArgs& a, int grid, size_t smem, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(decode_scores_kernel<RK, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_chained(decode_scores_kernel<RK, G>, dim3(grid), dim3(kAThreads), smem, s, 1u, c.trig_map, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int RK>
static cudaError_t launch_scores(const Ctx& c, const ScoreArgs& a, int grid, size_t smem, cudaStream_t s) {
  if (c.key.fp16) return launch_scores_g<RK, 0>(c, a, grid, smem, s);
  switch (c.key.g) {
    case 4: return launch_scores_g<RK, 4>(c, a, grid, smem, s);
    case 8: return launch_scores_g<RK, 8>(c, a, grid, smem, s);
    default: return launch_scores_g<RK, 16>(c, a, grid, smem, s);
  }
}

cudaError_t launch_decode_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* q,
                             const int32_t* block_table, const int32_t* seq_lens, int batch, int max_pages,
                             __nv_bfloat16* out, void* ws, const DecodePlan&, cudaStream_t s,
                             const DecodeSlice* slice) {
  if (batch == 0) return cudaSuccess;
  const int32_t* pos0 = slice ? slice->pos0 : nullptr;
  const int32_t* qpos = slice ? slice->qpos : nullptr;
  const starkv_config& f = c.cfg;
  const TcLayout t = tc_layout(c, batch, max_pages);
  char* w = (char*)ws;
  float* S = (float*)(w + t.off_S);
  unsigned int* Mx = (unsigned int*)(w + t.off_mx);
  float* acc = (float*)(w + t.off_acc);
  float* lsum = (float*)(w + t.off_l);
  uint8_t* wimg = (uint8_t*)(w + t.off_w);
  float* oacc = (float*)(w + t.off_oacc);
  unsigned int* ocnt = (unsigned int*)(w + t.off_ocnt);
  const int d = f.head_dim;

  // ---------------- W images: rotated query folded into B'_k, per (sequence, head)
  {
    dim3 g(f.num_q_heads, (batch + kWpSeq - 1) / kWpSeq);
    cudaError_t e0 = cudaSuccess;
    switch (f.rank_k) {
      case 16:
        e0 = launch_chained(decode_wprep_kernel<16>, g, dim3(128), 0, s, 1u, q, seq_lens, pos0, qpos, (const float*)c.Bk, (const float2*)c.rope, wimg, Mx,
                            (int)f.num_q_heads, c.group, d, t.hpc, t.ncols, batch, max_pages, (int)f.max_position);
        break;
      case 32:
        e0 = launch_chained(decode_wprep_kernel<32>, g, dim3(128), 0, s, 1u, q, seq_lens, pos0, qpos, (const float*)c.Bk, (const float2*)c.rope, wimg, Mx,
                            (int)f.num_q_heads, c.group, d, t.hpc, t.ncols, batch, max_pages, (int)f.max_position);
        break;
      default:
        e0 = launch_chained(decode_wprep_kernel<64>, g, dim3(128), 0, s, 1u, q, seq_lens, pos0, qpos, (const float*)c.Bk, (const float2*)c.rope, wimg, Mx,
                            (int)f.num_q_heads, c.group, d, t.hpc, t.ncols, batch, max_pages, (int)f.max_position);
        break;
    }
    if (e0 != cudaSuccess) return e0;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

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
  A.batch = batch;
  // the items that can hold tokens (every sequence at its longest); each CTA
  // takes total / ctas of the ones that do, which is at most items_per_cta
  const int max_items = batch * t.HG * t.tiles_per_seq;
  int ctas = sm_count();
  if (ctas > max_items) ctas = max_items;
  A.items_per_cta = (max_items + ctas - 1) / ctas;
  // a CTA's block-table entries sit in shared memory: beyond this many tiles
  // per CTA the grid grows past one wave instead
  if (A.items_per_cta > kMaxScoreItemsPerCta) A.items_per_cta = kMaxScoreItemsPerCta;
  ctas = (max_items + A.items_per_cta - 1) / A.items_per_cta;
  A.items_per_cta = (max_items + ctas - 1) / ctas;
  A.n_pages = cache.n_pages;
  A.q = q;
  A.block_table = block_table;
  A.seq_lens = seq_lens;
  A.pos0 = pos0;
  A.qpos = qpos;
  A.k_codes = (const uint8_t*)cache.k_codes;
  A.k_meta = (const uint32_t*)cache.k_meta;
  A.Bk = c.Bk;
  A.rope = c.rope;
  A.S = S;
  A.Mx = Mx;
  A.oacc = oacc;
  A.ocnt = ocnt;
  A.oacc_elems = (int64_t)batch * f.num_q_heads * d;
  A.ocnt_elems = f.num_q_heads * ((batch + 15) / 16);
  A.wimg = wimg;
  A.w_bytes = (uint32_t)t.w_bytes;
  A.status = c.status;
  A.trig_stage = kT * d * 2;
  A.codes_page = t.kvpc * c.key.region_bytes;
  A.meta_page = c.key.fp16 ? 0 : t.kvpc * c.key.groups * kPage * 4;
  A.codes_pitch = (A.codes_page + 64 + 127) / 128 * 128 - 64;  // = 64 mod 128: the two pages a warp reads
  A.meta_pitch = (A.meta_page + 64 + 127) / 128 * 128 - 64;    // fall on different banks
  A.codes_stage = kPagesPerTile * A.codes_pitch;
  A.meta_stage = kPagesPerTile * A.meta_pitch;
  {
    uint32_t o = (uint32_t)t.ncols * d * 2;  // W
    o = (o + 1023) / 1024 * 1024;
    A.off_trig = o;
    o += 2 * A.trig_stage;
    // as many key stages as fit (page table, flags, barriers and alignment slack after them)
    const uint32_t tail = (uint32_t)(A.items_per_cta * kPagesPerTile * 4) + kMaxKeyStages * kPagesPerTile * 4 +
                          (2 * kMaxKeyStages + 16) * 8 + 2 * 4 * kT * 4 + (uint32_t)(batch + 1) * 4 + 16 + 1024 + 64;
    const uint32_t per_key = A.codes_stage + A.meta_stage;
    int nk = (int)((227u * 1024u - o - tail) / per_key);
    if (nk > kMaxKeyStages) nk = kMaxKeyStages;
    if (nk < 2) return cudaErrorInvalidConfiguration;
    A.NK = nk;
    A.off_codes = o;
    o += nk * A.codes_stage;
    A.off_meta = o;
    o += nk * A.meta_stage;
    A.off_flags = o;
    o += kMaxKeyStages * kPagesPerTile * 4;
    A.off_bt = (o + 15) / 16 * 16;
    o = A.off_bt + A.items_per_cta * kPagesPerTile * 4;
    A.off_bar = (o + 15) / 16 * 16;
    o = A.off_bar + (2 * kMaxKeyStages + 16) * 8;
    A.off_red = (o + 15) / 16 * 16;
    o = A.off_red + 2 * 4 * kT * 4;
    A.off_pre = (o + 15) / 16 * 16;
    o = A.off_pre + (uint32_t)(batch + 1) * 4;
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
  B.PS = t.PS;
  B.nW = t.nW;
  B.ST = t.ST;
  B.CS = t.CS;
  B.nclust = t.nclust;
  B.balanced = t.balanced;
  B.batch = batch;
  B.slots = t.slots;
  B.vsplit = reinterpret_cast<int*>(w + t.off_vsplit);
  B.max_pages = max_pages;
  B.tpad = t.tpad;
  B.splits = t.splits;
  B.stages_total = t.stages_total;
  B.max_position = f.max_position;
  B.n_pages = cache.n_pages;
  B.block_table = block_table;
  B.seq_lens = seq_lens;
  B.pos0 = pos0;
  B.qpos = qpos;
  B.v_codes = (const uint8_t*)cache.v_codes;
  B.v_meta = (const uint32_t*)cache.v_meta;
  B.Mx = Mx;
  B.part = acc;
  B.lpart = lsum;
  B.status = c.status;
  if (!t.ok) return cudaErrorInvalidConfiguration;
  {
    const VSmem& v = t.vs;
    B.NS = v.NS;
    B.off_z = v.off_z;
    B.off_p = v.off_p;
    B.off_s = v.off_s;
    B.off_codes = v.off_codes;
    B.off_meta = v.off_meta;
    B.off_flags = v.off_flags;
    B.off_bt = v.off_bt;
    B.off_m = v.off_m;
    B.off_l = v.off_l;
    B.off_bar = v.off_bar;
    B.p_stage = v.p_stage;
    B.s_box = v.s_box;
    B.s_box_bytes = v.s_box_bytes;
    B.s_stage = v.s_stage;
    B.codes_page = v.codes_page;
    B.meta_page = v.meta_page;
    B.codes_pitch = v.codes_pitch;
    B.meta_pitch = v.meta_pitch;
    B.codes_stage = v.codes_stage;
    B.meta_stage = v.meta_stage;
    B.tmem_cols = v.tmem_cols;
    const size_t smem = v.smem;
    CUtensorMap s_map;
    if (!encode_map_2d(&s_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, S, (uint64_t)t.tpad, (uint64_t)batch * f.num_q_heads,
                       (uint64_t)t.tpad * 4, 32, (uint32_t)f.num_q_heads, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(decode_values_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_chained(decode_values_kernel, dim3(t.splits, batch), dim3((kVRoleWarps + t.nW) * 32), smem, s,
                       (unsigned)t.CS, s_map, B);
    if (e != cudaSuccess) return e;
  }

  // ---------------- C: projection
  ProjArgs P;
  P.H = f.num_q_heads;
  P.h_kv = f.num_kv_heads;
  P.group = c.group;
  P.d = d;
  P.R = f.rank_v;
  P.splits = t.splits;
  P.stages_total = t.stages_total;
  P.st = t.ST;
  P.cs = t.CS;
  P.nclust = t.nclust;
  P.vsplit = t.balanced ? reinterpret_cast<const int*>(w + t.off_vsplit) : nullptr;
  P.part = acc;
  P.lpart = lsum;
  P.seq_lens = seq_lens;
  P.pos0 = pos0;
  P.qpos = qpos;
  P.Mx = Mx;
  P.out_o = slice ? slice->out_o : nullptr;
  P.out_ml = slice ? slice->out_ml : nullptr;
  P.tpad = t.tpad;
  P.max_pages = max_pages;
  P.max_position = f.max_position;
  P.Bv16 = c.Bv16;
  P.out = out;
  P.oacc = oacc;
  P.ocnt = ocnt;
  const int kc = f.rank_v % kProjC == 0 ? kProjC : 64;
  {
    cudaError_t e = launch_chained(decode_project_kernel, dim3(f.num_q_heads, f.rank_v / kc, (batch + kProjM - 1) / kProjM),
                                   dim3(256), 0, s, 1u, P, batch, kc);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace starkv

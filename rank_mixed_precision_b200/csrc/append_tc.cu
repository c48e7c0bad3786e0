// Tensor-core (tcgen05 / TMEM) append for chunks of new tokens: the projection
// Z = X [A_k | A_v] with the rotation, quantiser and packer fused into its
// epilogue.
//
// Source: "STAR-KV: Learning the Rank Is Only Half of KV Cache Compression",
// Algorithm 2 steps 1-3 (project the new hidden states into latent keys and
// values, apply the prepared block rotations, quantise and append), section 6.1
// eq. 13-14.  The projection is a dense bf16 GEMM (n tokens x hidden x
// h_kv r_k + R latent columns): X tiles (K-major) and A tiles (N-major) arrive
// by TMA into a four-stage ring, one thread issues the tcgen05 MMAs into a
// 128 x N fp32 accumulator in TMEM, and four epilogue warps (one token row per
// thread) read each group's g latents back, rotate (fp32 butterflies),
// quantise (fp16 scale and zero) and pack them into the token's page slot with
// the same arithmetic as every other quantiser of the library.
#include "internal.cuh"
#include "sm100.cuh"

namespace starkv {
using namespace sm100;

namespace {
constexpr int kM = 128;          // tokens per CTA (MMA M)
constexpr int kN = 256;          // latent columns per CTA at most (MMA N)
constexpr int kKC = 64;          // hidden columns per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 192;    // producer warp, MMA warp, 4 epilogue warps
constexpr uint32_t kXStage = kM * kKC * 2;         // 16 KiB
constexpr uint32_t kAStage = kKC * kN * 2;         // 32 KiB (4 boxes of 64 columns x 64 rows)

__device__ __forceinline__ uint8_t* align1024a(uint8_t* p) { return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u); }

// kind::f16 instruction descriptor with bf16 A and B, fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return make_idesc_f16(M, N, a_mn, b_mn) | (1u << 7) | (1u << 10);
}
}  // namespace

struct AppendTcArgs {
  LatentGeom key, val;
  const KeyHead* kh;       // [h_kv] per-head key geometry and page offsets
  int key_cols, kpage_bytes, kpage_meta;
  int h_kv, hidden, lat_cols;
  int64_t n, n_pages;
  const int64_t* slots;
  float* lat_out;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint32_t* k_meta;
  uint32_t* v_meta;
  unsigned int* status;
};

// grid (ceil(n / 128), ceil(lat_cols / 256)), 192 threads.
__global__ void __launch_bounds__(kThreads, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap a_map,
                     const AppendTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024a(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kStages * (kXStage + kAStage));
  uint64_t* full = bar;                 // [kStages]
  uint64_t* empty = bar + kStages;      // [kStages]
  uint64_t* done = bar + 2 * kStages;   // accumulator final
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = (int64_t)blockIdx.x * kM;
  const int n0 = blockIdx.y * kN;
  const int N = min(kN, a.lat_cols - n0);  // a multiple of 16
  const int nbox = (N + 63) / 64;
  const int nk = a.hidden / kKC;
  pdl_wait();  // X and the slots may come from any earlier kernel
  pdl_launch_dependents();
  if (warp == 1) tmem_alloc(tslot, 256);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      for (int k = 0; k < nk; ++k) {
        const int s = k % kStages;
        const uint32_t ph = (k / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) {
          ok = false;
          break;
        }
        uint8_t* xs = sm + s * (kXStage + kAStage);
        uint8_t* as = xs + kXStage;
        mbar_arrive_expect_tx(&full[s], kXStage + (uint32_t)nbox * (kKC * 64 * 2));
        tma_load_2d(xs, &x_map, k * kKC, (int32_t)row0, &full[s]);
        for (int i = 0; i < nbox; ++i) tma_load_2d(as + i * (kKC * 64 * 2), &a_map, n0 + i * 64, k * kKC, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16(kM, N, false, true);
      for (int k = 0; k < nk; ++k) {
        const int s = k % kStages;
        const uint32_t ph = (k / kStages) & 1;
        if (!mbar_wait(&full[s], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t xa = smem_u32(sm + s * (kXStage + kAStage));
        const uint32_t aa = xa + kXStage;
#pragma unroll
        for (int ks = 0; ks < kKC / 16; ++ks)
          mma_f16(tmem, make_sdesc(xa + ks * 32, 16, 1024, 2), make_sdesc(aa + ks * 2048, kKC * 64 * 2, 1024, 2),
                  idesc, (k > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(done);
    }
  } else {
    // ---------------- epilogue: one token row per thread ----------------
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int64_t row = row0 + r;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const bool got = __all_sync(0xffffffffu, mbar_wait(done, 0));
    tc_fence_after();
    if (!got) {
      ok = false;
    } else {
      int64_t slot = -1;
      if (row < a.n) {
        slot = a.slots[row];
        if (slot >= a.n_pages * kPage) {
          set_status(a.status, STARKV_DEV_BAD_SLOT);
          slot = -1;
        }
      }
      const int key_cols = a.key_cols;
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + c0, v);
        tmem_ld_wait();
        if (row >= a.n) continue;
        const float* x = reinterpret_cast<const float*>(v);
        const int col = n0 + c0;
        if (a.lat_out) {
          float4* dst = reinterpret_cast<float4*>(a.lat_out + row * a.lat_cols + col);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
        }
        if (slot < 0) continue;
        const int64_t page = slot / kPage;
        const int t = (int)(slot % kPage);
        // the 16 columns hold whole groups of one latent (every head's rank and R are
        // multiples of 16, g divides 16)
        const bool is_key = col < key_cols;
        const int kv = is_key ? key_head_of(a.kh, a.h_kv, col) : 0;
        const LatentGeom L = is_key ? a.kh[kv].L : a.val;
        const int cin = is_key ? col - a.kh[kv].col0 : col - key_cols;
        for (int j = 0; j < 16; j += L.g) {
          const int gi = (cin + j) / L.g;
          if (is_key) {
            rotate_quantize_store_any(x + j, L, gi, a.k_codes + page * a.kpage_bytes + a.kh[kv].code_off,
                                      a.k_meta + page * a.kpage_meta + a.kh[kv].meta_off, t, a.status);
          } else {
            rotate_quantize_store_any(x + j, L, gi, a.v_codes + page * L.region_bytes,
                                        a.v_meta + page * L.groups * kPage, t, a.status);
          }
        }
      }
    }
  }
  if (!ok && lane == 0) set_status(a.status, kDevWaitTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

bool tc_append_supported(const Ctx& c) {
  return c.cfg.hidden % kKC == 0 && c.lat_cols % 16 == 0;
}

size_t append_tc_smem() { return (size_t)kStages * (kXStage + kAStage) + 256 + 1024; }

cudaError_t launch_append_tc(const Ctx& c, const starkv_cache& cache, const __nv_bfloat16* X, const int64_t* slots,
                             int64_t n, float* latents_out, cudaStream_t s) {
  CUtensorMap xm;
  if (!encode_map_2d(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)X, (uint64_t)c.cfg.hidden, (uint64_t)n,
                     (uint64_t)c.cfg.hidden * 2, kKC, kM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  AppendTcArgs a;
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
  a.slots = slots;
  a.lat_out = latents_out;
  a.k_codes = (uint8_t*)cache.k_codes;
  a.v_codes = (uint8_t*)cache.v_codes;
  a.k_meta = (uint32_t*)cache.k_meta;
  a.v_meta = (uint32_t*)cache.v_meta;
  a.status = c.status;
  const size_t smem = append_tc_smem();
  cudaError_t e = cudaFuncSetAttribute(append_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n + kM - 1) / kM), (unsigned)((c.lat_cols + kN - 1) / kN));
  e = launch_chained(append_tc_kernel, grid, dim3(kThreads), smem, s, 1u, xm, c.a_map64, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace starkv

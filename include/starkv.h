/*
 * starkv.h -- C ABI of the STAR-KV latent-cache attention library (B200, sm_100a).
 *
 * The library computes attention directly on a low-rank, mixed-precision
 * latent KV cache, following the decode dataflow of "STAR-KV: Learning the
 * Rank Is Only Half of KV Cache Compression" (technical review of arXiv
 * 2606.08382), Algorithm 2 "Consume a compressed cache during decoding":
 *
 *   keys   : one pre-RoPE latent per KV head, z_k,h (rank r_k), re-expanded
 *            by B_k,h (r_k x d_h) inside the attention kernel, then RoPE'd
 *            (section 5.3, "Keys are harder");
 *   values : one joint latent z_v (rank R) shared by all heads; probabilities
 *            of all heads multiply it first and B_v (R x h_kv d_h) is applied
 *            afterwards (section 5.3, eq. 12 and the stacked P Z_V product);
 *   storage: latents are Hadamard-rotated in groups (section 6.1, eq. 13) and
 *            quantised 4-bit for the leading (outlier) channels and 3-bit for
 *            the rest (eq. 14), with an fp16 scale and zero per group.
 *
 * Conventions for every entry point
 *   - Pointers named "device" are CUDA device memory owned by the caller;
 *     "host" pointers are CPU memory.  The library keeps no pointer to caller
 *     memory after a call returns, except that work queued on `stream` reads
 *     and writes it asynchronously: keep buffers alive until the stream has
 *     passed the work.
 *   - All compute is queued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns before it finishes.  Nothing throws; every function
 *     returns a starkv_status, and starkv_last_error() gives the calling
 *     thread's last message.
 *   - Arguments are checked on the host before anything is launched.  Faults
 *     that only the data can show (an out-of-range page id in a block table, a
 *     sequence longer than its pages, a latent whose fp16 scale overflows) set
 *     bits in a device status word owned by the context; the affected work is
 *     skipped (its output is written as zeros) and the word is read with
 *     starkv_read_device_status().
 *
 * Data types: "bf16" = IEEE bfloat16 bit patterns (uint16), "fp16" = IEEE
 * binary16, "fp32" = IEEE binary32.  Arrays are dense and row-major.
 */
#ifndef STARKV_H
#define STARKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define STARKV_API __attribute__((visibility("default")))
#else
#define STARKV_API
#endif

#define STARKV_PAGE_TOKENS 16 /* tokens per cache page (a paged KV block) */

typedef int32_t starkv_status;
enum {
  STARKV_OK = 0,
  STARKV_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum   */
  STARKV_ERR_UNSUPPORTED_SHAPE = 2,  /* a configuration the library cannot run */
  STARKV_ERR_WORKSPACE_TOO_SMALL = 3,/* workspace_bytes below the required size */
  STARKV_ERR_CUDA = 4,               /* a CUDA runtime call failed               */
  STARKV_ERR_DEVICE_STATUS = 5       /* the device status word is non-zero       */
};

/* Device status word bits (see starkv_read_device_status). */
enum {
  STARKV_DEV_BAD_PAGE = 1u << 0,     /* block-table entry < 0 or >= n_pages      */
  STARKV_DEV_BAD_SEQ_LEN = 1u << 1,  /* seq_len < 0, > max_pages*16, or beyond
                                        the context's max_position             */
  STARKV_DEV_QUANT_OVERFLOW = 1u << 2,/* a group's fp16 scale/zero not finite, or
                                        a non-finite latent                     */
  STARKV_DEV_BAD_SLOT = 1u << 3,     /* append slot >= n_pages*16                */
  STARKV_DEV_BAD_QUERY_SPAN = 1u << 4,/* prefill: cu_q not non-decreasing, or a
                                        sequence's query count > its seq_len    */
  STARKV_DEV_WAIT_TIMEOUT = 1u << 5  /* a pipelined kernel gave up waiting on one
                                        of its own stages (bounded wait); its
                                        outputs for that call are not valid    */
};

/* Opaque stream handle: pass a cudaStream_t. */
typedef struct CUstream_st* starkv_stream_t;

/* Latent storage variants (starkv_config.flags).
 * 0: mixed precision, the leading top_fraction of each latent's channels at 4
 *    bits and the rest at 3 bits ([Review] section 6.1, eq. 14); top_fraction
 *    1.0 gives the uniform 4-bit cache of the review's speed ablation.
 * STARKV_FLAG_FP16_LATENT: the unquantised variant, every rotated latent value
 *    stored as fp16 ([Review] section 8.1, the unquantised rank-75% rows);
 *    top_fraction is ignored, the rotation group is 16 channels, and a region
 *    of a page is group tiles of 16 tokens x 16 channels, element (t, c) at
 *    fp16 index t*16 + c (512 bytes per tile, no metadata: the k_meta and
 *    v_meta pools have 0 bytes and may be NULL). */
#define STARKV_FLAG_FP16_LATENT 1

/* Model shape and quantisation settings.
 * top_fraction: share of each latent's leading channels (singular-value order)
 *   stored at 4 bits; the rest are stored at 3 bits ([Review] eq. 14; the
 *   checkpoint card uses top_fraction = 0.25, top_bits = 4, bottom_bits = 3).
 *   n_top = floor(top_fraction * r + 0.5).  The rotation and quantisation
 *   group is g = gcd(16, n_top, r - n_top) channels, so no group straddles the
 *   two precision blocks; g must be 4, 8 or 16.
 * Supported: head_dim in {64, 128}; num_q_heads % num_kv_heads == 0;
 *   num_q_heads, num_kv_heads <= 1024; rank_k <= head_dim, rank_k <= 64,
 *   rank_k % 16 == 0; rank_v <= num_kv_heads*head_dim, rank_v <= 1024,
 *   rank_v % 16 == 0; hidden % 64 == 0, hidden <= 65536; rope_base > 1;
 *   1 <= max_position <= 2^24 (the context holds max_position * head_dim * 6
 *   bytes of RoPE tables on the device and, while it is created, on the host). */
typedef struct starkv_config {
  int32_t num_q_heads;  /* H                                            */
  int32_t num_kv_heads; /* h_kv                                         */
  int32_t head_dim;     /* d_h                                          */
  int32_t hidden;       /* width of the hidden states X                 */
  int32_t rank_k;       /* r_k: key latent rank per KV head             */
  int32_t rank_v;       /* R: joint value latent rank                   */
  int32_t max_position; /* positions [0, max_position) are supported    */
  int32_t flags;        /* 0, or STARKV_FLAG_FP16_LATENT                */
  double top_fraction;  /* 0.25                                         */
  double rope_base;     /* RoPE theta base (1e4 Llama-2, 5e5 Llama-3)   */
  const int32_t* key_ranks; /* host [num_kv_heads] learned key rank of each
                               KV head, or NULL for rank_k everywhere (see
                               "Ragged key ranks" below)                */
} starkv_config;

/* Ragged key ranks ([Review] section 3 and its figure of learned rank
 * profiles: the key rank is learned per head and layer; the checkpoint card's
 * calibration caps it at max_rank_k = 64).  With key_ranks set, KV head h keeps
 * r_h = key_ranks[h] latent channels: 16 <= r_h <= rank_k, r_h a multiple of
 * 16, and rank_k is the largest of them.  Each head's channel split and group
 * size follow from its own r_h (n_top = floor(top_fraction r_h + 0.5),
 * g = gcd(16, n_top, r_h - n_top)).  A_k holds sum_h r_h columns, head h's at
 * col0_h = r_0 + ... + r_{h-1}; B_k is [sum_h r_h][head_dim], head h's rows at
 * col0_h.  A page of the key-code pool holds the heads' regions back to back
 * (head h at sum_{h' < h} region_bytes(r_h')), and a page of the key-meta pool
 * their metadata likewise; starkv_cache_sizes.key_page_bytes and
 * key_page_meta_bytes give the per-page strides.  The joint value rank R is
 * per layer (one context per layer).  Decode and prefill of ragged ranks run
 * on the CUDA-core kernels; append on every kernel. */

/* The four caller-allocated page pools of a paged latent cache.
 *   k_codes: [n_pages][num_kv_heads][key_region_bytes]    packed key codes
 *   v_codes: [n_pages][value_region_bytes]                packed value codes
 *   k_meta : [n_pages][num_kv_heads][key_groups][16] x 4 B  (fp16 scale, fp16 zero)
 *   v_meta : [n_pages][value_groups][16] x 4 B
 * Each pool base must be 16-byte aligned.  A page holds 16 consecutive token
 * positions of one sequence; a sequence's pages are listed in its block-table
 * row.  Byte layout of one page of one latent region: group tiles in channel
 * order; a 4-bit tile holds element (t, c) of its 16 x g block at nibble
 * index t*g + c (low nibble first); a 3-bit tile is a 2-bit plane of the low
 * bits (element i at bits 2*(i%4) of byte i/4) followed by a 1-bit plane of
 * the high bit (bit i%8 of byte i/8).  Meta word: scale in the low 16 bits,
 * zero-point in the high 16 bits. */
typedef struct starkv_cache {
  void* k_codes;
  void* v_codes;
  void* k_meta;
  void* v_meta;
  int64_t n_pages;
} starkv_cache;

typedef struct starkv_cache_sizes {
  int64_t k_codes_bytes; /* pool sizes for the requested n_pages */
  int64_t v_codes_bytes;
  int64_t k_meta_bytes;
  int64_t v_meta_bytes;
  int32_t key_region_bytes;   /* per page per KV head (payload padded to 16 B) */
  int32_t value_region_bytes; /* per page                                      */
  int32_t key_group_size;     /* g of a key latent                             */
  int32_t value_group_size;   /* g of the value latent                         */
  int32_t key_top;            /* n_top of a key latent                         */
  int32_t value_top;          /* n_top of the value latent                     */
  int32_t key_groups;         /* r_k / g                                       */
  int32_t value_groups;       /* R / g                                         */
  int32_t key_page_bytes;     /* key-code bytes of one page, all KV heads      */
  int32_t key_page_meta_bytes;/* key-meta bytes of one page, all KV heads      */
} starkv_cache_sizes;

typedef struct starkv_ctx starkv_ctx;

enum { STARKV_OP_DECODE = 0, STARKV_OP_PREFILL = 1, STARKV_OP_DECODE_OUT = 2 };
enum { STARKV_LATENT_KEY = 0, STARKV_LATENT_VALUE = 1 };
/* starkv_quantize_pack / starkv_dequantize: the key latent of KV head h
 * (needed with ragged key ranks; STARKV_LATENT_KEY is head 0). */
#define STARKV_LATENT_KEY_HEAD(h) (2 + (h))

/* Library version string (static storage). */
STARKV_API const char* starkv_version(void);

/* Message of the calling thread's last failed call (static per thread). */
STARKV_API const char* starkv_last_error(void);

/* Host-only: check a configuration and return the cache pool sizes for
 * n_pages pages (the packed layout above; [Review] eq. 15 plus metadata and
 * padding).  out: host.  Errors: INVALID_ARG, UNSUPPORTED_SHAPE. */
STARKV_API starkv_status starkv_cache_layout(const starkv_config* cfg, int64_t n_pages,
                                  starkv_cache_sizes* out);

/* Create a context on the current CUDA device.
 * A_k: device bf16 [hidden][num_kv_heads*rank_k], head h's columns at h*rank_k
 *      (its latent channels in singular-value order);
 * A_v: device bf16 [hidden][rank_v];
 * B_k: device bf16 [num_kv_heads][rank_k][head_dim];
 * B_v: device bf16 [rank_v][num_kv_heads*head_dim].
 * The factors are copied into context-owned memory; the rotation is folded
 * into the up-projections (B' = H B, exact by [Review] eq. 13) and a RoPE
 * cos/sin table for [0, max_position) is built in fp64 and stored as fp32.
 * Synchronises `stream` before returning, so the inputs may be freed after.
 * out: host, receives the context.  Errors: INVALID_ARG, UNSUPPORTED_SHAPE, CUDA. */
STARKV_API starkv_status starkv_create(const starkv_config* cfg, const void* A_k, const void* A_v,
                            const void* B_k, const void* B_v, starkv_stream_t stream,
                            starkv_ctx** out);

/* Free a context (device-synchronising).  NULL is accepted. */
STARKV_API starkv_status starkv_destroy(starkv_ctx* ctx);

/* Sizes the context was created with (host copy). */
STARKV_API starkv_status starkv_get_config(const starkv_ctx* ctx, starkv_config* out);

/* Append n tokens: decode dataflow steps 1-3 ([Review] Algorithm 2: project
 * the hidden states into latent keys and values, apply the block rotations,
 * quantise and append).  X: device bf16 [n][hidden].  slot_mapping: device
 * int64 [n], slot = page*16 + offset; a negative slot skips that token; slots
 * must be distinct within one call.  Only the written tokens' bits change.
 * latents_out: optional device fp32 [n][num_kv_heads*rank_k + rank_v], receives
 * the pre-quantisation latents (debug export; NULL to skip).
 * Errors: INVALID_ARG; device bits BAD_SLOT, QUANT_OVERFLOW. */
STARKV_API starkv_status starkv_append(starkv_ctx* ctx, const starkv_cache* cache, const void* X,
                            const int64_t* slot_mapping, int64_t n, float* latents_out,
                            starkv_stream_t stream);

/* Workspace bytes needed by decode (op = STARKV_OP_DECODE; total_q ignored),
 * decode with the output projection (op = STARKV_OP_DECODE_OUT; needs
 * starkv_set_output_projection first) or prefill (op = STARKV_OP_PREFILL) for
 * `batch` sequences whose block tables have max_pages columns.  out: host. */
STARKV_API starkv_status starkv_workspace_bytes(const starkv_ctx* ctx, int32_t op, int32_t batch,
                                     int32_t max_pages, int64_t total_q, size_t* out);

/* Batched single-query decode attention over the packed cache ([Review]
 * Algorithm 2 steps 4-8; keys re-expanded and RoPE'd in the kernel, values
 * aggregated in the R-dim latent and projected by B_v afterwards, split-K
 * partials merged by the softmax partition identity).
 * q: device bf16 [batch][num_q_heads][head_dim], pre-RoPE; sequence b's query
 *    sits at position seq_lens[b]-1 and attends to positions [0, seq_lens[b]).
 * block_table: device int32 [batch][max_pages]; seq_lens: device int32 [batch].
 * out: device bf16 [batch][num_q_heads][head_dim], each head's attention output
 *      before the output projection W_o.  seq_len 0 gives a zero row.
 * workspace: device, >= starkv_workspace_bytes(DECODE), 256-byte aligned.
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL; device bits BAD_PAGE, BAD_SEQ_LEN. */
STARKV_API starkv_status starkv_decode_attn(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                 const int32_t* block_table, const int32_t* seq_lens,
                                 int32_t batch, int32_t max_pages, void* out, void* workspace,
                                 size_t workspace_bytes, starkv_stream_t stream);

/* Give the context the attention block's output projection W_o, so that
 * decode can emit the block's output directly ([Review] Algorithm 2 steps 7-8:
 * apply the prepared head-specific value/output factors and sum the head
 * contributions; section 5.3 eq. 12).  W_o: device bf16 [num_q_heads*head_dim]
 * [model_dim], the rows of query head h at h*head_dim .. (h+1)*head_dim - 1.
 * Copied into context-owned memory (synchronises `stream`); a later call
 * replaces it.  model_dim: a positive multiple of 8, <= 65536.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, CUDA. */
STARKV_API starkv_status starkv_set_output_projection(starkv_ctx* ctx, const void* W_o, int32_t model_dim,
                                                      starkv_stream_t stream);

/* Decode attention followed by the output projection: the same arguments as
 * starkv_decode_attn, but the result is the attention block's output
 * y[b] = sum_h o_h[b] W_o,h, device bf16 [batch][model_dim], where o_h is what
 * starkv_decode_attn returns.  The value factor B_v is applied first (in the
 * R-dim latent, then d_h wide) and W_o second: with R > d_h that is cheaper
 * than the fused factor U_h^T O_h of eq. 12 (R x model_dim per query head).
 * workspace: >= starkv_workspace_bytes(STARKV_OP_DECODE_OUT, ...), 256-byte
 * aligned.  Errors: as starkv_decode_attn, plus INVALID_ARG without an output
 * projection. */
STARKV_API starkv_status starkv_decode_attn_out(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                                const int32_t* block_table, const int32_t* seq_lens, int32_t batch,
                                                int32_t max_pages, void* y, void* workspace, size_t workspace_bytes,
                                                starkv_stream_t stream);

/* Decode without any device allocation: the same computation and arguments as
 * starkv_decode_attn, minus the workspace.  (The paper has no counterpart; this
 * is a deployment variant.)  It is meant for callers that cannot call
 * cudaMalloc, for example a plugin running inside a serving engine that owns
 * the whole device memory pool, or a latency-critical loop that must never
 * enter the allocator.  The split partials live in a built-in 16 MiB scratch
 * array that every GPU loading this library holds until the process exits;
 * the call itself allocates nothing.  The first call on a device looks up that
 * array's device address (once per device, with the device current) and keeps
 * it for the life of the process; make this first call before any stream
 * capture, and do not use the library across a cudaDeviceReset of that device.
 * All calls on a device share the scratch, so calls that overlap on the GPU
 * (other streams, other contexts on the same device) race; serialise them.
 * Size limit: the call needs exactly the workspace starkv_decode_attn would
 * take, so a shape is accepted when
 *   starkv_workspace_bytes(ctx, STARKV_OP_DECODE, batch, max_pages, 0) <= 16 MiB
 * (query that call to check a shape; the workspace grows with batch and with
 * max_pages).  A larger shape is rejected with STARKV_ERR_UNSUPPORTED_SHAPE
 * before anything is launched.
 * Errors: as starkv_decode_attn, plus UNSUPPORTED_SHAPE for oversize shapes. */
STARKV_API starkv_status starkv_decode_attn_noalloc(starkv_ctx* ctx, const starkv_cache* cache,
                                                    const void* q, const int32_t* block_table,
                                                    const int32_t* seq_lens, int32_t batch,
                                                    int32_t max_pages, void* out,
                                                    starkv_stream_t stream);

/* Decode over one slice of each sequence's context, for sequence (context)
 * sharding across GPUs: the softmax partition identity of [CaliDrop] (the
 * attention decomposition theorem, eq. 1) lets every GPU attend the query to
 * the tokens it holds and a merge combine the slices exactly.  Same dataflow
 * as starkv_decode_attn ([Review] Algorithm 2 steps 4-8); B_v is linear, so
 * each slice projects through it locally and only d_h-wide rows cross GPUs.
 * seq_lens: device int32 [batch], the tokens of the slice held in `cache`
 *   (the block table maps them from local index 0);
 * key_pos0: device int32 [batch], the position of the slice's first token
 *   (its tokens are at key_pos0[b] .. key_pos0[b] + seq_lens[b] - 1);
 * q_pos: device int32 [batch], the query's position (normally the last
 *   position of the whole sequence).  Every position must be < max_position.
 * out_o: device fp32 [batch][num_q_heads][head_dim], 16-byte aligned: the
 *   attention output over the slice alone (normalised within the slice);
 * out_ml: device fp32 [batch][num_q_heads][2], 8-byte aligned: the slice's
 *   softmax statistics (m, l) with scores in log2 units,
 *   m = max_j s_j * log2(e), l = sum_j 2^(s_j * log2(e) - m); an empty slice
 *   gives (-inf, 0).
 * workspace: as starkv_decode_attn.  Only shapes served by the tensor-core
 * decode are supported (else UNSUPPORTED_SHAPE).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, WORKSPACE_TOO_SMALL; device bits
 * BAD_PAGE, BAD_SEQ_LEN (a position outside the RoPE table). */
STARKV_API starkv_status starkv_decode_attn_slice(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                                  const int32_t* block_table, const int32_t* seq_lens,
                                                  const int32_t* key_pos0, const int32_t* q_pos, int32_t batch,
                                                  int32_t max_pages, float* out_o, float* out_ml, void* workspace,
                                                  size_t workspace_bytes, starkv_stream_t stream);

/* Merge n_parts slice results of the same queries (the partition identity,
 * [CaliDrop] eq. 1): out = sum_r 2^(m_r - M) l_r o_r / sum_r 2^(m_r - M) l_r
 * with M = max_r m_r over the slices with l_r > 0 (all-empty: a zero row).
 * o_parts: device fp32 [n_parts][batch][num_q_heads][head_dim] (16-byte
 * aligned), ml_parts: device fp32 [n_parts][batch][num_q_heads][2], both as
 * starkv_decode_attn_slice writes them; out: device bf16
 * [batch][num_q_heads][head_dim].  Errors: INVALID_ARG. */
STARKV_API starkv_status starkv_merge_slices(starkv_ctx* ctx, const float* o_parts, const float* ml_parts,
                                             int32_t n_parts, int32_t batch, void* out, starkv_stream_t stream);

/* Causal chunk attention over the packed cache (the chunked form of the same
 * dataflow).  q: device bf16 [total_q][num_q_heads][head_dim], pre-RoPE, rows of
 * sequence b at cu_q[b] .. cu_q[b+1]-1 (cu_q: device int32 [batch+1], cu_q[0]=0,
 * cu_q[batch] = total_q).  Query i of sequence b sits at position
 * seq_lens[b] - n_b + i (n_b = its query count, <= seq_lens[b]) and attends to
 * positions <= its own; the chunk's own tokens must already be appended.
 * max_q_len: upper bound of n_b.  out: device bf16 [total_q][num_q_heads][head_dim].
 * workspace: >= starkv_workspace_bytes(PREFILL, batch, max_pages, total_q).
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL; device bits BAD_PAGE, BAD_SEQ_LEN,
 * BAD_QUERY_SPAN. */
STARKV_API starkv_status starkv_prefill_attn(starkv_ctx* ctx, const starkv_cache* cache, const void* q,
                                  const int32_t* cu_q, const int32_t* block_table,
                                  const int32_t* seq_lens, int32_t batch, int32_t max_pages,
                                  int64_t total_q, int32_t max_q_len, void* out,
                                  void* workspace, size_t workspace_bytes,
                                  starkv_stream_t stream);

/* Rotate, quantise and pack n pre-quantisation latents of one latent kind
 * (which = STARKV_LATENT_KEY: a KV head's r_k channels; STARKV_LATENT_VALUE:
 * the R channels) into ceil(n/16) pages of one region ([Review] section 6.1,
 * eq. 13-14).  z: device fp32 [n][r].  codes: device [ceil(n/16)][region_bytes];
 * meta: device [ceil(n/16)][groups][16] x 4 B; both fully overwritten (rows
 * past n: zero codes, zero scale and zero-point).  Same arithmetic as the
 * append kernel's quantiser.  Errors: INVALID_ARG; device bit QUANT_OVERFLOW. */
STARKV_API starkv_status starkv_quantize_pack(starkv_ctx* ctx, int32_t which, const float* z, int64_t n,
                                   void* codes, void* meta, starkv_stream_t stream);

/* Unpack and dequantise the first n tokens of packed pages of one region:
 * z_hat = code*scale + zero in fp32, rotated domain.  z_out: device fp32 [n][r]. */
STARKV_API starkv_status starkv_dequantize(starkv_ctx* ctx, int32_t which, const void* codes,
                                const void* meta, int64_t n, float* z_out,
                                starkv_stream_t stream);

/* Synchronise `stream`, return the device status word in *status (host) and
 * clear it.  Returns DEVICE_STATUS when the word was non-zero. */
STARKV_API starkv_status starkv_read_device_status(starkv_ctx* ctx, starkv_stream_t stream,
                                        uint32_t* status);

/* Test-only failure detection check (no counterpart on the pages): queue one
 * block that waits on a shared-memory barrier nothing ever completes, with the
 * bounded wait every pipelined kernel of this library uses, given `limit_ns`
 * nanoseconds (1e3 .. 1e9) instead of the kernels' own limit.  The wait gives up,
 * sets STARKV_DEV_WAIT_TIMEOUT in the status word and the block exits; the
 * context stays usable.  Errors: INVALID_ARG (limit out of range), CUDA. */
STARKV_API starkv_status starkv_selftest_wait_timeout(starkv_ctx* ctx, uint64_t limit_ns, starkv_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* STARKV_H */

/*
 * rpk.h -- C ABI of librpk.so: fused QK RoPE into a paged KV cache and ragged
 * causal grouped-query attention over that cache, on one NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every tensor argument is DEVICE memory owned by the caller; the
 *           library allocates nothing (scratch space is the caller-given
 *           workspace). Host-side arguments are marked "host" below. Tensors
 *           are dense, row-major, with the shapes given; 16-byte alignment of
 *           every tensor base is required.
 * Streams.  `stream` is a cudaStream_t (NULL: the legacy default stream). A
 *           call validates its arguments on the host, queues its kernels on
 *           that stream and returns before they finish (NumKong "NumKong for
 *           Python", GPU Tensors through DLPack: a GPU call queues its launch
 *           on the given stream and returns).
 * Errors.   Host-side problems (a NULL pointer, a shape, a dtype, an
 *           unsupported size) return a non-zero rpk_status before anything is
 *           launched. Problems that only the data shows (a page id outside the
 *           pool, a position outside the table, kv_len < q_len) are reported
 *           by OR-ing RPK_DEVERR_* bits into page_table->error_word when it is
 *           non-NULL; the offending row or slot is skipped and nothing traps.
 *           A launch failure returns RPK_ERR_CUDA. There is no CPU fallback
 *           and no silent change of path (aria_kernel crate index,
 *           resolve_compute: CUDA never falls back to the CPU).
 * Dtypes.   RPK_BF16 or RPK_F32 for q, k, v, out and the cache; all arithmetic
 *           is fp32 with one round-to-nearest-even narrowing at the end. The
 *           cache may instead be RPK_E4M3 (see rpk_paged_kv) under bf16 or
 *           fp32 tensors.
 */
#ifndef RPK_H
#define RPK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RPK_OK = 0,
  RPK_ERR_NULL = 1,         /* a required pointer is NULL                          */
  RPK_ERR_SHAPE = 2,        /* inconsistent or out-of-range sizes                   */
  RPK_ERR_DTYPE = 3,        /* dtype not supported or not equal where it must be    */
  RPK_ERR_UNSUPPORTED = 4,  /* valid request outside the sizes the kernels support  */
  RPK_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed                  */
  RPK_ERR_WORKSPACE = 6     /* workspace missing, too small or misaligned           */
} rpk_status;

/* RPK_E4M3 is a cache dtype only: 1 sign, 4 exponent (bias 7) and 3 mantissa
 * bits, no infinity, NaN = S.1111.111, largest finite 448 (NumKong "NumKong for
 * Python", scalar types: float8_e4m3). */
typedef enum { RPK_F32 = 0, RPK_BF16 = 1, RPK_E4M3 = 2 } rpk_dtype;

/* Bits OR-ed into *error_word by the kernels. */
#define RPK_DEVERR_PAGE 0x1u     /* page id outside [0, num_pages) or slot beyond the block table */
#define RPK_DEVERR_POSITION 0x2u /* position outside [0, max_position)                          */
#define RPK_DEVERR_LENGTH 0x4u   /* kv_len < q_len, decreasing offsets, or a length above the
                                    max_q_len / max_kv_len the call was given                 */
#define RPK_DEVERR_TIMEOUT 0x8u  /* a bounded wait inside a kernel gave up (kernel returned)    */

/*
 * The paged KV cache ("kv_collection" of Mojo's fused QK RoPE kernel, a
 * PagedKVCacheCollection whose keys are read and updated in place).
 * The struct itself is host memory; the pointers in it are device memory.
 *
 *   k_pages, v_pages   [num_pages, page_size, n_kv_heads, head_dim] cache_dtype.
 *                      Slot s of sequence b is page block_table[b][s / page_size],
 *                      row s % page_size.
 *   block_table        int32 [batch, max_pages_per_seq]: page ids into the pool.
 *                      Entries past a sequence's last page are never read.
 *   cache_lens         int32 [batch]: tokens already cached for each sequence
 *                      BEFORE the rope_qk_paged_ragged call that appends to it.
 *                      Read only by rope_qk_paged_ragged.
 *   error_word         optional int32 (device): RPK_DEVERR_* bits are OR-ed in.
 *   num_layers,        a multi-layer collection (Mojo's layer_idx argument, "index
 *   layer_idx          of the layer whose keys are updated in the cache"): the
 *                      pools hold num_layers layer-major copies of the layout
 *                      above, [num_layers, num_pages, page_size, n_kv_heads,
 *                      head_dim], and a call reads / writes layer layer_idx
 *                      only, sharing block_table and cache_lens with the other
 *                      layers. num_layers 0 (a zero-initialised struct) means 1.
 *                      layer_idx outside [0, num_layers): RPK_ERR_SHAPE.
 *   cache_dtype        RPK_BF16 / RPK_F32 (the dtype of q, k, v), or RPK_E4M3: a
 *                      quantised cache (Mojo's kv_collection with a cache dtype,
 *                      a scale dtype and a quantisation granularity) holding
 *                      code = e4m3(x / scale) with one fp32 scale per KV head
 *                      for K and one for V; the key or value is code * scale.
 *                      rope_qk_paged_ragged rounds the fp32 quotient once to
 *                      nearest (ties to even) and saturates magnitudes beyond
 *                      448 to +-448.
 *   k_scale, v_scale   fp32 [n_kv_heads] (device), finite and > 0: the scales of
 *                      an RPK_E4M3 cache (required then: NULL is RPK_ERR_NULL);
 *                      not read for other cache dtypes.
 */
typedef struct {
  void* k_pages;
  void* v_pages;
  int32_t num_pages;
  int32_t page_size;        /* 16, 32, 64 or 128 */
  int32_t n_kv_heads;
  int32_t head_dim;         /* 64, 128 or 256 */
  rpk_dtype cache_dtype;
  const int32_t* block_table;
  int32_t max_pages_per_seq;
  int32_t batch;
  const int32_t* cache_lens;
  int32_t* error_word;
  int32_t num_layers;
  int32_t layer_idx;
  const float* k_scale;
  const float* v_scale;
} rpk_paged_kv;

/*
 * rope_qk_paged_ragged -- rotate Q into out_q, rotate the new keys and write
 * them, with the new values, into the paged cache.
 *
 * Follows Mojo's generic_fused_qk_rope_bshd_paged_ragged_kernel_api (Args and
 * Parameters: q_proj, input_row_offsets, kv_collection, freqs_cis,
 * position_ids, interleaved, mrope_section, output), with the new K and V
 * passed explicitly (k_new, v_new) and written into the next free slots; the
 * pairings follow aria_kernel's rope (interleaved), rope_half and
 * rope_half_partial.
 *
 *   q_proj             [total_tokens, n_heads, head_dim] dtype
 *   input_row_offsets  int32 [batch + 1]: rows off[b] .. off[b+1]-1 belong to
 *                      sequence b; off[0] = 0, non-decreasing, off[batch] =
 *                      total_tokens
 *   k_new, v_new       [total_tokens, n_kv_heads, head_dim] dtype
 *   page_table         the cache (host struct, see rpk_paged_kv); token i of
 *                      sequence b goes to slot cache_lens[b] + i
 *   freqs_cis          fp32 [max_position, rotary_dim]: for pair j at position
 *                      p, (cos, sin) = (freqs_cis[p][2j], freqs_cis[p][2j+1])
 *                      (rope_freqs_cis below builds it)
 *   position_ids       NULL: position of token i of sequence b is
 *                      cache_lens[b] + i. Otherwise int32 [total_tokens], or
 *                      [3, total_tokens] when mrope_section is given.
 *   interleaved        nonzero: pair j is channels (2j, 2j+1); zero: (j, j+R/2)
 *   rotary_dim (R)     even, 0 < R <= head_dim; channels >= R are copied
 *   out_q              [total_tokens, n_heads, head_dim] dtype; may alias q_proj
 *   total_tokens, n_heads, dtype, max_position: sizes (host)
 *   mrope_section      host int32[3] or NULL: numbers of rotary pairs in the
 *                      three M-RoPE sections (summing to R/2); pair j takes the
 *                      position of its section's row of position_ids
 *
 * Each pair (a, b) becomes (a cos - b sin, b cos + a sin), computed in fp32
 * and rounded once to the output dtype. Requirements: dtype == cache dtype
 * (or an RPK_E4M3 cache, which receives e4m3(k' / k_scale) and e4m3(v / v_scale)
 * of the fp32 values, see rpk_paged_kv), n_heads % n_kv_heads == 0, (R/2) a
 * multiple of 8 (bf16) or 4 (f32).
 */
rpk_status rope_qk_paged_ragged(const void* q_proj, const int32_t* input_row_offsets,
                                const void* k_new, const void* v_new,
                                const rpk_paged_kv* page_table, const float* freqs_cis,
                                const int32_t* position_ids, int32_t interleaved,
                                int32_t rotary_dim, void* out_q, int32_t total_tokens,
                                int32_t n_heads, rpk_dtype dtype, int32_t max_position,
                                const int32_t* mrope_section, void* stream);

/*
 * rope_freqs_cis -- fill freqs_cis (fp32 [max_position, rotary_dim], device)
 * with cos and sin of p * theta^(-2j / rotary_dim), evaluated in fp64 and
 * rounded once to fp32 (algenta "Attention variant kernels",
 * rope_rotation_angle: theta = position * base^(-2i/d)).
 */
rpk_status rope_freqs_cis(float* freqs_cis, int32_t max_position, int32_t rotary_dim,
                          double theta, void* stream);

/*
 * rope_freqs_cis_proportional -- the table of p-RoPE, algenta "Attention
 * variant kernels", rope_half_proportional (Gemma-4 global layers): of the
 * head_dim/2 pairs of the rotate-half layout only the first rotated_pairs
 * (= factor * head_dim / 2) turn, with frequencies over the full head_dim;
 * the other pairs are the identity.
 *
 *   freqs_cis      [max_position, head_dim] fp32 (device, caller-owned):
 *                  pair j < rotated_pairs holds (cos, sin)(p * theta^(-2j/head_dim)),
 *                  computed in fp64 and rounded once; pair j >= rotated_pairs
 *                  holds (1, 0).
 *   rotated_pairs  0 .. head_dim/2 (host)
 *
 * Use it with rope_qk_paged_ragged(..., interleaved = 0, rotary_dim = head_dim,
 * ...): pair j is then (x[j], x[j + head_dim/2]), and the identity pairs come
 * back bit for bit (a*1 - b*0 = a, b*1 + a*0 = b in fp32). Errors as
 * rope_freqs_cis; RPK_ERR_SHAPE for rotated_pairs outside 0 .. head_dim/2.
 */
rpk_status rope_freqs_cis_proportional(float* freqs_cis, int32_t max_position, int32_t head_dim,
                                       int32_t rotated_pairs, double theta, void* stream);

/*
 * ragged_paged_attention_workspace_size -- bytes of device workspace that
 * ragged_paged_attention needs for these sizes (the larger of the split-KV
 * partials of the decode path and the 256-byte work counter of the prefill
 * path; 0 when there are no query tokens). The result depends only on the
 * arguments, so it may be computed once and reused for every call with the
 * same sizes.
 */
size_t ragged_paged_attention_workspace_size(int32_t total_q_tokens, int32_t n_heads,
                                             int32_t head_dim, int32_t batch,
                                             int32_t max_kv_len, int32_t page_size);

/*
 * ragged_paged_attention -- ragged causal scaled-dot-product attention with
 * grouped-query heads and an optional sliding window, over the paged cache.
 *
 * Follows NumKong's attention_packed ("Attention with a Pre-Packed
 * KV-Cache"): query row r of a sequence with q_len rows and k_len keys sits at
 * position p = r + k_len - q_len and sees keys [p - (window - 1), p]
 * (window <= 0: [0, p]); rows that see no key are zeros. Scores are
 * scale * q.k (algenta scaled_dot_product_attention), normalised by the
 * flash online-softmax running state (algenta flash_attention module). Query
 * head h reads KV head h / (n_heads / n_kv_heads) (grouped-query attention).
 *
 *   q               [total_q_tokens, n_heads, head_dim] dtype (already rotated)
 *   q_row_offsets   int32 [batch + 1], as input_row_offsets above
 *   kv_lens         int32 [batch]: keys of each sequence, including its q_len
 *                   newest ones; kv_lens[b] >= q_len[b]
 *   page_table      the cache (host struct); cache_lens is not read
 *   scale           finite > 0 (1/sqrt(head_dim) for plain SDPA)
 *   window          <= 0: unbounded; w > 0: w keys including the row's own
 *                   (w >= max_kv_len covers every key a row sees: unbounded,
 *                   and sink_tokens then has no effect)
 *   out             [total_q_tokens, n_heads, head_dim] dtype
 *   batch, total_q_tokens, max_q_len, max_kv_len: sizes (host); max_q_len and
 *                   max_kv_len bound q_len[b] and kv_lens[b] (device data) and
 *                   size the launch; a larger device value sets
 *                   RPK_DEVERR_LENGTH and that sequence is skipped
 *   workspace       device scratch of at least
 *                   ragged_paged_attention_workspace_size(...) bytes, 256-byte
 *                   aligned. The decode path with several splits keeps its
 *                   partial results there and the tcgen05 prefill path its work
 *                   counter (first 4 bytes); the fp32 path and single-split
 *                   decode accept NULL. Missing, small or misaligned where it
 *                   is needed: RPK_ERR_WORKSPACE. Its contents on entry do not
 *                   matter; calls sharing one workspace must not overlap in time.
 *   log_sum_exp     NULL, or float32 [total_q_tokens, n_heads] (4-byte aligned):
 *                   each row's natural log-sum-exp ln sum_j e^(scale q.k_j) over
 *                   its visible keys, -inf for a row that sees no key (the
 *                   output NumKong's attention_packed fills for training,
 *                   "Attention with a Pre-Packed KV-Cache"). Rows of a sequence
 *                   with a length error are left unwritten, as in out.
 *   sink_tokens     >= 0 (host). Under a window (window > 0), the first
 *                   sink_tokens keys of every sequence stay visible to each row
 *                   at or after them, beside its window: StreamingLLM attention
 *                   sinks (algenta "Attention variant kernels", sparse_attention
 *                   streaming_llm_sink_score). Ignored when window <= 0 (every
 *                   earlier key is visible then). Negative: RPK_ERR_SHAPE.
 *
 * Paths (chosen from the host sizes, never from device data):
 *   dtype f32                      -> fp32 CUDA-core kernel
 *   bf16, max_q_len * group <= 16  -> split-KV decode kernel + combine kernel
 *   bf16, otherwise                -> tcgen05 prefill kernel (head_dim 64, 128
 *                                     and 256, group <= 128; larger groups run
 *                                     on the CUDA-core kernel)
 * An RPK_E4M3 cache takes the same decode path and, for head_dim 64 and 128,
 * the same tcgen05 prefill path. Codes are widened to f16, which is exact
 * (decode: in registers for head_dim >= 128, in shared memory for 64;
 * prefill: by a warpgroup of its own into shared memory). The query is
 * narrowed to f16 under a power-of-two scale, per row in the prefill and per
 * group in the decode, and that scale and k_scale are folded into the score
 * scale, v_scale into the output. e4m3 prefill shapes of head_dim 256 run on
 * the CUDA-core kernel.
 */
rpk_status ragged_paged_attention(const void* q, const int32_t* q_row_offsets,
                                  const int32_t* kv_lens, const rpk_paged_kv* page_table,
                                  int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
                                  float scale, int32_t window, void* out, int32_t batch,
                                  int32_t total_q_tokens, int32_t max_q_len,
                                  int32_t max_kv_len, rpk_dtype dtype, void* workspace,
                                  size_t workspace_bytes, float* log_sum_exp,
                                  int32_t sink_tokens, void* stream);

/*
 * ragged_paged_attention_backward -- gradients of ragged_paged_attention's
 * output (NumKong "Attention with a Pre-Packed KV-Cache":
 * attention_packed_gradients turns the forward's log-sum-exp, its output and
 * the output gradient into query, key and value gradients under the same
 * band).
 *
 * With s_ij = scale q_i.k_j, P_ij = e^(s_ij - lse_i), dP_ij = d_out_i.v_j,
 * D_i = d_out_i.out_i and dS_ij = P_ij (dP_ij - D_i):
 *   d_q_i = scale sum_j dS_ij k_j, d_k_j = scale sum_i dS_ij q_i,
 *   d_v_j = sum_i P_ij d_out_i,
 * the sums running over the (row, key) pairs the forward's band (window,
 * sinks) makes visible, and over every query head of a KV head's group.
 *
 *   q, q_row_offsets, kv_lens, page_table, n_heads ... dtype, sink_tokens:
 *                   as in the forward call whose gradient this is (the cache
 *                   unchanged since; an RPK_E4M3 cache is read as code * scale)
 *   out             the forward's output [total_q_tokens, n_heads, head_dim] dtype
 *   d_out           [total_q_tokens, n_heads, head_dim] dtype, the output gradient
 *   log_sum_exp     float32 [total_q_tokens, n_heads], the forward's log_sum_exp
 *   d_q             float32 [total_q_tokens, n_heads, head_dim] (written; on
 *                   the tensor-core path its memory also holds each row's D_i
 *                   between the call's kernels)
 *   d_k_pages,      float32, the shape of one layer's pools
 *   d_v_pages       [num_pages, page_size, n_kv_heads, head_dim]: the entry of
 *                   every key below kv_lens[b] of each sequence is written (the
 *                   gradient of that cached key or value; for an e4m3 cache,
 *                   of its dequantised value); other entries are left as they
 *                   were, so a caller that sums over the pool zeroes them first.
 *
 * bf16 tensors over a bf16 cache run on tensor cores (bf16 operands, fp32
 * sums; P and dS are rounded to bf16 as operands of the second products):
 * the 5th-generation ones (tcgen05, accumulators in tensor memory) for
 * head_dim 64 and 128 with groups of at most 64 query heads, warp-level ones
 * (mma.sync) for head_dim 256 with groups of at most 16. The kernels are: D_i
 * of every row, a key-parallel one for d_k and d_v, then a row-parallel one for
 * d_q. Other shapes (fp32 tensors, an e4m3 cache, larger groups) run on
 * CUDA-core kernels in fp32. No path uses atomics, so results are
 * deterministic.
 * Errors as ragged_paged_attention; every pointer is 16-byte aligned device
 * memory; buffers must not overlap.
 */
rpk_status ragged_paged_attention_backward(
    const void* q, const int32_t* q_row_offsets, const int32_t* kv_lens,
    const rpk_paged_kv* page_table, int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
    float scale, int32_t window, const void* out, const void* d_out, const float* log_sum_exp,
    float* d_q, float* d_k_pages, float* d_v_pages, int32_t batch, int32_t total_q_tokens,
    int32_t max_q_len, int32_t max_kv_len, rpk_dtype dtype, int32_t sink_tokens, void* stream);

/*
 * ragged_paged_attention_noalloc -- ragged_paged_attention for callers that
 * cannot allocate device memory at call time. The pages have no counterpart
 * for it; it is a convenience of this library.
 *
 * Who needs it: a serving engine that reserved all free HBM for its KV cache
 * at start-up and refuses later allocations; a plugin inside a host
 * framework that owns every allocator; a decode loop that cannot pay the
 * implicit synchronisation of cudaMalloc. They cannot supply the workspace
 * that ragged_paged_attention takes.
 *
 * Arguments and results are those of ragged_paged_attention without the
 * workspace, the log_sum_exp output and the sink_tokens band (this entry point
 * takes none of the three; sinks are off). It runs the same split-KV decode
 * kernels, so it takes only the decode shapes: dtype RPK_BF16 over a bf16
 * cache and max_q_len * (n_heads / n_kv_heads) <= 16. Other shapes return
 * RPK_ERR_UNSUPPORTED.
 *
 * Scratch: the kernels' fp32 partials go to one array inside the library,
 * RPK_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU, held from the moment the
 * library is loaded on that GPU until the process exits. Sizes whose
 * partials would not fit (ragged_paged_attention_workspace_size(...) >
 * RPK_NOALLOC_SCRATCH_BYTES) return RPK_ERR_WORKSPACE before anything is
 * launched. The call itself never allocates (no cudaMalloc, no cudaFree).
 *
 * The first call on each device looks up the array's device address and
 * caches it; make that first call before any stream capture on that device.
 * The cached address belongs to the device's context: after cudaDeviceReset
 * (or any destruction of the primary context) the address is stale, so do not
 * call this entry point again in that process.
 *
 * All calls on a device share the one array, and it keeps whatever the last
 * call left in it. Nothing in it needs to start at zero. Calls whose kernels
 * overlap on the GPU (different streams, no ordering between them) race on
 * the array and give wrong results: order them on one stream, or use
 * ragged_paged_attention with separate workspaces.
 */
#define RPK_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
rpk_status ragged_paged_attention_noalloc(const void* q, const int32_t* q_row_offsets,
                                          const int32_t* kv_lens,
                                          const rpk_paged_kv* page_table, int32_t n_heads,
                                          int32_t n_kv_heads, int32_t head_dim, float scale,
                                          int32_t window, void* out, int32_t batch,
                                          int32_t total_q_tokens, int32_t max_q_len,
                                          int32_t max_kv_len, rpk_dtype dtype, void* stream);

/*
 * rpk_set_wait_limit_ns -- the bound, in nanoseconds of the GPU's global
 * timer, that every later attention launch gives each of its device-side
 * waits (a stage of K/V tiles, a score tile, a work item). A wait that runs
 * out makes its CTA give up: it ORs RPK_DEVERR_TIMEOUT into
 * page_table->error_word, lets the copies and tensor-core operations it has
 * already issued finish, frees its tensor memory and returns, so the context
 * stays usable and later calls on the stream run normally (a kernel that finds
 * RPK_DEVERR_TIMEOUT already set in the error word also stops early, so clear
 * the word before relying on later results). The pages have no counterpart;
 * this is the library's failure detection (no wait is unbounded, nothing
 * traps). A limit under 1 microsecond, below the resolution of the GPU's
 * global timer, makes a wait give up at its first test of a phase that is not
 * already complete. 0 restores the default of 2 seconds. The setting is process-wide
 * and read when a call is made; waits for copies already in flight during a
 * give-up keep the default bound.
 */
void rpk_set_wait_limit_ns(uint64_t limit_ns);
uint64_t rpk_wait_limit_ns(void);

/* Static text for a status code. */
const char* rpk_status_string(rpk_status status);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* rpk_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RPK_H */

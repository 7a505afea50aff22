// kernels.h -- launch parameters and launchers of the librpk kernels
// (internal to the library; the public ABI is include/rpk.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rpk.h"

namespace rpk {

// ------------------------------------------------ host helpers (capi.cu)

// Default bound of every device-side wait (nanoseconds of %globaltimer).
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;
// The bound later launches give their device-side waits (rpk_set_wait_limit_ns).
unsigned long long wait_limit_ns();
// RPK_OK for cudaSuccess; otherwise records the error's text for
// rpk_last_cuda_error() and returns RPK_ERR_CUDA.
rpk_status cuda_status(cudaError_t e);
// Records `text` for rpk_last_cuda_error() (this thread).
void set_last_error_text(const char* text);
// Host-side checks of a cache description shared by every entry point.
rpk_status check_cache(const rpk_paged_kv* c);
// 3-D bf16 tensor map over rows of [rows, heads, d]: dims (d, heads, rows),
// box (64, box_heads, box_rows), 128-byte swizzle, no multicast.
rpk_status encode_rows_map(CUtensorMap* map, const void* base, int32_t d, int32_t heads,
                           int64_t rows, int32_t box_heads, int32_t box_rows);

// The pools of the layer a call uses: layer layer_idx of num_layers (0 means
// one) layer-major copies of [num_pages, page_size, n_kv_heads, head_dim].
// False when layer_idx is out of range.
// The window a launch uses: 0 (unbounded) for window <= 0 and for a window of
// at least max_kv_len keys, which already covers every key a row can see;
// otherwise the window itself. Keeps the band arithmetic far from int overflow.
inline int32_t effective_window(int32_t window, int32_t max_kv_len) {
  return window > 0 && window < max_kv_len ? window : 0;
}

inline bool layer_pools(const rpk_paged_kv* c, void** k, void** v) {
  const int32_t layers = c->num_layers > 0 ? c->num_layers : 1;
  if (c->num_layers < 0 || c->layer_idx < 0 || c->layer_idx >= layers) return false;
  const size_t elt = c->cache_dtype == RPK_F32 ? 4 : (c->cache_dtype == RPK_E4M3 ? 1 : 2);
  const size_t per_layer =
      (size_t)c->num_pages * c->page_size * c->n_kv_heads * c->head_dim * elt;
  *k = static_cast<char*>(c->k_pages) + (size_t)c->layer_idx * per_layer;
  *v = static_cast<char*>(c->v_pages) + (size_t)c->layer_idx * per_layer;
  return true;
}

struct RopeParams {
  const void* q;
  const void* k_new;
  const void* v_new;
  void* out_q;
  void* k_pages;
  void* v_pages;
  const int32_t* offsets;       // [batch + 1]
  const int32_t* cache_lens;    // [batch]
  const int32_t* block_table;   // [batch, max_pages]
  const int32_t* position_ids;  // NULL, [T] or [3, T]
  const float* freqs;           // [max_position, R]
  int32_t* error_word;
  int32_t T, batch, H, Hk, d, R, P, num_pages, max_pages, max_position;
  int32_t sec_end0, sec_end1;   // M-RoPE: pair j < sec_end0 -> section 0, < sec_end1 -> 1, else 2
  int32_t has_mrope;
  int32_t tokens_per_cta;       // 1..4, chosen by the launcher
  int32_t cache_fp8;            // the pools hold e4m3 codes of x / scale
  const float* k_scale;         // [Hk] when cache_fp8
  const float* v_scale;
};

cudaError_t launch_rope(const RopeParams& p, rpk_dtype dtype, bool interleaved,
                        cudaStream_t stream);
cudaError_t launch_freqs_cis(float* out, int32_t max_position, int32_t width, int32_t denom,
                             int32_t rotated_pairs, double theta, cudaStream_t stream);

struct AttnParams {
  const void* q;
  void* out;
  const void* k_pages;
  const void* v_pages;
  const int32_t* offsets;      // [batch + 1]
  const int32_t* kv_lens;      // [batch]
  const int32_t* block_table;  // [batch, max_pages]
  int32_t* error_word;
  int32_t T, batch, H, Hk, G, d, P, num_pages, max_pages, window, max_q_len, max_kv_len;
  float scale;
  float scale_log2;            // scale * log2(e)
  float* lse = nullptr;        // [T, H] natural log-sum-exp of each row's scores, or null
  int32_t sinks = 0;           // under a window: the first `sinks` keys stay visible
  int32_t cache_fp8 = 0;       // the pools hold e4m3 codes; key = code * k_scale[kvh] etc.
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
  unsigned long long wait_ns = kDefaultWaitLimitNs;  // bound of each mbarrier wait
};

// fp32 / bf16 CUDA-core attention: one warp per (token, head) row.
cudaError_t launch_attn_simt(const AttnParams& p, rpk_dtype dtype, cudaStream_t stream);

// Split-KV decode (bf16): key tiles of this many keys, splits of whole tiles.
constexpr int kDecodeTile = 64;
constexpr int kDecodeMaxRows = 16;   // max_q_len * group must fit one m16 tile
constexpr int kDecodeMaxSplits = 64;

struct DecodePlan {
  int32_t tiles_per_split;
  int32_t max_splits;
};
// The plan with the most splits any launch uses (sizes the workspace).
DecodePlan decode_plan(int32_t max_kv_len);
// The plan a launch uses for `units` (sequence, KV head) pairs: never more
// splits than decode_plan. cache_fp8: the pools hold 1-byte e4m3 codes.
DecodePlan decode_launch_plan(int32_t max_kv_len, int32_t units, int32_t head_dim, int32_t window,
                              int32_t max_q_len, int32_t sinks, bool cache_fp8 = false);
size_t decode_workspace_bytes(int32_t total_q_tokens, int32_t n_heads, int32_t head_dim,
                              int32_t max_kv_len);

struct DecodeWorkspace {
  float* o;       // [max_splits, T, H, d]
  float2* ml;     // [max_splits, T, H]: (running max in log2 units, running sum)
};

cudaError_t launch_attn_decode(const AttnParams& p, const CUtensorMap& k_map,
                               const CUtensorMap& v_map, const DecodePlan& plan,
                               const DecodeWorkspace& ws, cudaStream_t stream);

// tcgen05 prefill (bf16, head_dim 64, 128 or 256), persistent: its CTAs claim work
// items from `work_counter` (device int, zeroed by the launch; one per
// concurrently running launch).
constexpr size_t kPrefillWorkspaceBytes = 256;
constexpr int kPrefillKeyTile = 64;   // keys per tcgen05 prefill key tile (K/V box rows <= this)
cudaError_t launch_attn_prefill(const AttnParams& p, const CUtensorMap& q_map,
                                const CUtensorMap& k_map, const CUtensorMap& v_map,
                                int* work_counter, cudaStream_t stream);
int prefill_rows_per_tile(int group);

// Gradients of ragged_paged_attention (CUDA-core, fp32 math).
struct BackwardParams {
  const void* q;
  const void* out;
  const void* d_out;
  const float* lse;            // [T, H] natural log-sum-exp of the forward
  const void* k_pages;
  const void* v_pages;
  const int32_t* offsets;      // [batch + 1]
  const int32_t* kv_lens;      // [batch]
  const int32_t* block_table;  // [batch, max_pages]
  int32_t* error_word;
  float* d_q;                  // [T, H, d]
  float* d_k;                  // pool-shaped [num_pages, P, Hk, d]
  float* d_v;
  int32_t T, batch, H, Hk, G, d, P, num_pages, max_pages, window, max_q_len, max_kv_len, sinks;
  float scale;
  int32_t cache_fp8;
  const float* k_scale;
  const float* v_scale;
  unsigned long long wait_ns = kDefaultWaitLimitNs;  // bound of each mbarrier wait
};
cudaError_t launch_attn_backward(const BackwardParams& p, rpk_dtype dtype, cudaStream_t stream);
// tcgen05 kernels: bf16 tensors over a bf16 cache, head_dim 64 / 128, groups of
// up to 64 query heads. Maps: q and d_out as [T, H, d] with box (64, G, 64 / G)
// (the dK / dV kernel's 64-row blocks) and box (64, G, 128 / G) (the dQ
// kernel's 128-row blocks); the pools as [pages * page_size, n_kv_heads, d]
// with box (64, 1, min(page_size, 128)); all 128-byte swizzled.
bool attn_backward_tc_supported(const BackwardParams& p, rpk_dtype dtype);
cudaError_t launch_attn_backward_tc(const BackwardParams& p, const CUtensorMap& q_map64,
                                    const CUtensorMap& do_map64, const CUtensorMap& q_map128,
                                    const CUtensorMap& do_map128, const CUtensorMap& k_map,
                                    const CUtensorMap& v_map, cudaStream_t stream);
// Tensor-core (mma.sync) kernels: bf16 tensors over a bf16 cache, groups of at
// most 16 query heads, head_dim 64 / 128 / 256.
bool attn_backward_mma_supported(const BackwardParams& p, rpk_dtype dtype);
cudaError_t launch_attn_backward_mma(const BackwardParams& p, cudaStream_t stream);

}  // namespace rpk

// capi.cu -- the extern "C" entry points of librpk.so (declared in include/rpk.h):
// host-side validation, tensor-map encoding and kernel dispatch. No entry
// point allocates device memory or synchronises the stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/rpk.h"
#include "kernels.h"

namespace {
thread_local char g_last_cuda_error[256] = "";
// Bound of every device-side wait of later launches (rpk_set_wait_limit_ns).
std::atomic<unsigned long long> g_wait_limit_ns{rpk::kDefaultWaitLimitNs};
}  // namespace

namespace rpk {

rpk_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return RPK_OK;
  snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return RPK_ERR_CUDA;
}

void set_last_error_text(const char* text) {
  snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s", text);
}

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_head_dim(int32_t d) { return d == 64 || d == 128 || d == 256; }
bool supported_page(int32_t P) { return P == 16 || P == 32 || P == 64 || P == 128; }

rpk_status check_cache(const rpk_paged_kv* c) {
  if (!c) return RPK_ERR_NULL;
  if (!c->k_pages || !c->v_pages || !c->block_table) return RPK_ERR_NULL;
  if (c->cache_dtype != RPK_BF16 && c->cache_dtype != RPK_F32 && c->cache_dtype != RPK_E4M3)
    return RPK_ERR_DTYPE;
  if (c->cache_dtype == RPK_E4M3 && (!c->k_scale || !c->v_scale)) return RPK_ERR_NULL;
  if (c->num_pages <= 0 || c->n_kv_heads <= 0 || c->max_pages_per_seq <= 0 || c->batch <= 0)
    return RPK_ERR_SHAPE;
  if (!supported_page(c->page_size) || !supported_head_dim(c->head_dim))
    return RPK_ERR_UNSUPPORTED;
  if (!aligned16(c->k_pages) || !aligned16(c->v_pages)) return RPK_ERR_SHAPE;
  if ((long long)c->num_pages * c->page_size > INT32_MAX) return RPK_ERR_UNSUPPORTED;
  void *k, *v;
  if (!rpk::layer_pools(c, &k, &v)) return RPK_ERR_SHAPE;
  return RPK_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// q / k / v dtype and a cache dtype agree, or the cache holds e4m3 codes.
bool cache_dtype_ok(rpk_dtype dtype, rpk_dtype cache) {
  return cache == dtype || cache == RPK_E4M3;
}

// 3-D byte map over rows of an e4m3 pool [rows, heads, d]. Decode layout
// (whole_rows false): for head_dim >= 128 boxes of (128 codes, 1, box_rows)
// with the 128-byte swizzle (the decode kernel reads K fragments straight from
// them), for head_dim 64 whole rows, no swizzle. whole_rows true: whole rows of
// d codes, no swizzle (the prefill kernel's raw ring, which it widens to f16).
rpk_status encode_rows_map_u8(CUtensorMap* map, const void* base, int32_t d, int32_t heads,
                              int64_t rows, int32_t box_rows, bool whole_rows = false) {
  auto fn = encode_fn();
  if (!fn) {
    set_last_error_text("cuTensorMapEncodeTiled unavailable");
    return RPK_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)heads * d};
  const bool swizzled = d >= 128 && !whole_rows;
  cuuint32_t box[3] = {swizzled ? 128u : (cuuint32_t)d, 1u, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char text[64];
    snprintf(text, sizeof text, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    set_last_error_text(text);
    return RPK_ERR_CUDA;
  }
  return RPK_OK;
}

// 3-D bf16 map over rows of [rows, heads, d]: dims (d, heads, rows), box
// (64, 1, box_rows), 128-byte swizzle. Used for the KV pools and for Q.
rpk_status encode_rows_map(CUtensorMap* map, const void* base, int32_t d, int32_t heads,
                           int64_t rows, int32_t box_heads, int32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) {
    set_last_error_text("cuTensorMapEncodeTiled unavailable");
    return RPK_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char text[64];
    snprintf(text, sizeof text, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    set_last_error_text(text);
    return RPK_ERR_CUDA;
  }
  return RPK_OK;
}

}  // namespace rpk

using namespace rpk;

extern "C" {

const char* rpk_status_string(rpk_status s) {
  switch (s) {
    case RPK_OK: return "ok";
    case RPK_ERR_NULL: return "a required pointer is NULL";
    case RPK_ERR_SHAPE: return "inconsistent or out-of-range sizes";
    case RPK_ERR_DTYPE: return "unsupported or mismatched dtype";
    case RPK_ERR_UNSUPPORTED: return "sizes outside what the kernels support";
    case RPK_ERR_CUDA: return "CUDA call failed";
    case RPK_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

const char* rpk_last_cuda_error(void) { return g_last_cuda_error; }

void rpk_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns == 0 ? kDefaultWaitLimitNs : (unsigned long long)limit_ns,
                        std::memory_order_relaxed);
}

uint64_t rpk_wait_limit_ns(void) { return (uint64_t)wait_limit_ns(); }

rpk_status rope_qk_paged_ragged(const void* q_proj, const int32_t* input_row_offsets,
                                const void* k_new, const void* v_new,
                                const rpk_paged_kv* page_table, const float* freqs_cis,
                                const int32_t* position_ids, int32_t interleaved,
                                int32_t rotary_dim, void* out_q, int32_t total_tokens,
                                int32_t n_heads, rpk_dtype dtype, int32_t max_position,
                                const int32_t* mrope_section, void* stream) {
  if (!q_proj || !input_row_offsets || !k_new || !v_new || !freqs_cis || !out_q)
    return RPK_ERR_NULL;
  rpk_status st = check_cache(page_table);
  if (st != RPK_OK) return st;
  if (!page_table->cache_lens) return RPK_ERR_NULL;
  if (dtype != RPK_BF16 && dtype != RPK_F32) return RPK_ERR_DTYPE;
  if (!cache_dtype_ok(dtype, page_table->cache_dtype)) return RPK_ERR_DTYPE;
  const int32_t d = page_table->head_dim, Hk = page_table->n_kv_heads;
  if (total_tokens < 0 || n_heads <= 0 || max_position <= 0) return RPK_ERR_SHAPE;
  if (n_heads % Hk != 0) return RPK_ERR_SHAPE;
  if (rotary_dim <= 0 || (rotary_dim & 1) || rotary_dim > d) return RPK_ERR_SHAPE;
  const int vec = dtype == RPK_BF16 ? 8 : 4;
  if ((rotary_dim / 2) % vec != 0) return RPK_ERR_UNSUPPORTED;
  if (mrope_section) {
    if (!position_ids) return RPK_ERR_NULL;
    if (mrope_section[0] < 0 || mrope_section[1] < 0 || mrope_section[2] < 0 ||
        mrope_section[0] + mrope_section[1] + mrope_section[2] != rotary_dim / 2)
      return RPK_ERR_SHAPE;
  }
  if (!aligned16(q_proj) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out_q) ||
      !aligned16(freqs_cis))
    return RPK_ERR_SHAPE;
  if ((long long)total_tokens * n_heads * d > INT32_MAX * 8LL) return RPK_ERR_UNSUPPORTED;
  if (total_tokens == 0) return RPK_OK;

  rpk::RopeParams p;
  p.q = q_proj; p.k_new = k_new; p.v_new = v_new; p.out_q = out_q;
  rpk::layer_pools(page_table, &p.k_pages, &p.v_pages);
  p.offsets = input_row_offsets; p.cache_lens = page_table->cache_lens;
  p.block_table = page_table->block_table; p.position_ids = position_ids;
  p.freqs = freqs_cis; p.error_word = page_table->error_word;
  p.T = total_tokens; p.batch = page_table->batch; p.H = n_heads; p.Hk = Hk; p.d = d;
  p.R = rotary_dim; p.P = page_table->page_size; p.num_pages = page_table->num_pages;
  p.max_pages = page_table->max_pages_per_seq; p.max_position = max_position;
  p.has_mrope = mrope_section != nullptr;
  p.sec_end0 = mrope_section ? mrope_section[0] : rotary_dim;
  p.sec_end1 = mrope_section ? mrope_section[0] + mrope_section[1] : rotary_dim;
  p.tokens_per_cta = 1;
  p.cache_fp8 = page_table->cache_dtype == RPK_E4M3;
  p.k_scale = page_table->k_scale;
  p.v_scale = page_table->v_scale;
  return cuda_status(rpk::launch_rope(p, dtype, interleaved != 0,
                                      static_cast<cudaStream_t>(stream)));
}

rpk_status rope_freqs_cis(float* freqs_cis, int32_t max_position, int32_t rotary_dim,
                          double theta, void* stream) {
  if (!freqs_cis) return RPK_ERR_NULL;
  if (max_position < 0 || rotary_dim <= 0 || (rotary_dim & 1)) return RPK_ERR_SHAPE;
  if (!(theta > 0.0) || !std::isfinite(theta)) return RPK_ERR_SHAPE;
  return cuda_status(rpk::launch_freqs_cis(freqs_cis, max_position, rotary_dim, rotary_dim,
                                           rotary_dim / 2, theta,
                                           static_cast<cudaStream_t>(stream)));
}

rpk_status rope_freqs_cis_proportional(float* freqs_cis, int32_t max_position, int32_t head_dim,
                                       int32_t rotated_pairs, double theta, void* stream) {
  if (!freqs_cis) return RPK_ERR_NULL;
  if (max_position < 0 || head_dim <= 0 || (head_dim & 1)) return RPK_ERR_SHAPE;
  if (rotated_pairs < 0 || rotated_pairs > head_dim / 2) return RPK_ERR_SHAPE;
  if (!(theta > 0.0) || !std::isfinite(theta)) return RPK_ERR_SHAPE;
  return cuda_status(rpk::launch_freqs_cis(freqs_cis, max_position, head_dim, head_dim,
                                           rotated_pairs, theta,
                                           static_cast<cudaStream_t>(stream)));
}

size_t ragged_paged_attention_workspace_size(int32_t total_q_tokens, int32_t n_heads,
                                             int32_t head_dim, int32_t batch,
                                             int32_t max_kv_len, int32_t page_size) {
  (void)batch;
  (void)page_size;
  if (total_q_tokens <= 0 || n_heads <= 0 || head_dim <= 0 || max_kv_len < 0) return 0;
  // The larger of the decode partials and the prefill work counter.
  return std::max(rpk::decode_workspace_bytes(total_q_tokens, n_heads, head_dim, max_kv_len),
                  rpk::kPrefillWorkspaceBytes);
}

rpk_status ragged_paged_attention(const void* q, const int32_t* q_row_offsets,
                                  const int32_t* kv_lens, const rpk_paged_kv* page_table,
                                  int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
                                  float scale, int32_t window, void* out, int32_t batch,
                                  int32_t total_q_tokens, int32_t max_q_len,
                                  int32_t max_kv_len, rpk_dtype dtype, void* workspace,
                                  size_t workspace_bytes, float* log_sum_exp,
                                  int32_t sink_tokens, void* stream) {
  if (!q || !q_row_offsets || !kv_lens || !out) return RPK_ERR_NULL;
  rpk_status st = check_cache(page_table);
  if (st != RPK_OK) return st;
  if (dtype != RPK_BF16 && dtype != RPK_F32) return RPK_ERR_DTYPE;
  if (!cache_dtype_ok(dtype, page_table->cache_dtype)) return RPK_ERR_DTYPE;
  if (n_kv_heads != page_table->n_kv_heads || head_dim != page_table->head_dim)
    return RPK_ERR_SHAPE;
  if (n_heads <= 0 || n_heads % n_kv_heads != 0) return RPK_ERR_SHAPE;
  if (batch <= 0 || batch != page_table->batch || batch > 65535) return RPK_ERR_SHAPE;
  if (total_q_tokens < 0 || max_q_len < 0 || max_kv_len < 0) return RPK_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPK_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(out)) return RPK_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(log_sum_exp) & 3u) != 0) return RPK_ERR_SHAPE;
  if (sink_tokens < 0) return RPK_ERR_SHAPE;
  if ((long long)max_kv_len > (long long)page_table->max_pages_per_seq * page_table->page_size)
    return RPK_ERR_SHAPE;
  if (total_q_tokens == 0) return RPK_OK;

  rpk::AttnParams p;
  p.lse = log_sum_exp;
  p.q = q; p.out = out;
  {
    void *k, *v;
    rpk::layer_pools(page_table, &k, &v);
    p.k_pages = k; p.v_pages = v;
  }
  p.offsets = q_row_offsets; p.kv_lens = kv_lens; p.block_table = page_table->block_table;
  p.error_word = page_table->error_word;
  p.T = total_q_tokens; p.batch = batch; p.H = n_heads; p.Hk = n_kv_heads;
  p.G = n_heads / n_kv_heads; p.d = head_dim; p.P = page_table->page_size;
  p.num_pages = page_table->num_pages; p.max_pages = page_table->max_pages_per_seq;
  p.window = rpk::effective_window(window, max_kv_len);
  p.sinks = p.window > 0 ? sink_tokens : 0;
  p.max_q_len = max_q_len; p.max_kv_len = max_kv_len;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.cache_fp8 = page_table->cache_dtype == RPK_E4M3;
  p.k_scale = page_table->k_scale;
  p.v_scale = page_table->v_scale;
  p.wait_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  if (dtype == RPK_F32) return cuda_status(rpk::launch_attn_simt(p, dtype, s));

  if ((long long)max_q_len * p.G <= rpk::kDecodeMaxRows) {
    const size_t need = rpk::decode_workspace_bytes(total_q_tokens, n_heads, head_dim, max_kv_len);
    const rpk::DecodePlan plan = rpk::decode_launch_plan(max_kv_len, batch * n_kv_heads, head_dim,
                                                         p.window, max_q_len, p.sinks,
                                                         p.cache_fp8);
    if (plan.max_splits > 1) {
      if (!workspace || workspace_bytes < need) return RPK_ERR_WORKSPACE;
      if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RPK_ERR_WORKSPACE;
    }
    rpk::DecodeWorkspace ws;
    const size_t rows = (size_t)plan.max_splits * total_q_tokens * n_heads;
    const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) & ~size_t(255);
    ws.o = static_cast<float*>(workspace);
    ws.ml = workspace ? reinterpret_cast<float2*>(static_cast<char*>(workspace) + o_bytes)
                      : nullptr;
    CUtensorMap k_map, v_map;
    const int32_t box_rows = p.P < rpk::kDecodeTile ? p.P : rpk::kDecodeTile;
    const int64_t pool_rows = (int64_t)p.num_pages * p.P;
    if (p.cache_fp8) {
      st = encode_rows_map_u8(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, box_rows);
      if (st != RPK_OK) return st;
      st = encode_rows_map_u8(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, box_rows);
    } else {
      st = encode_rows_map(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
      if (st != RPK_OK) return st;
      st = encode_rows_map(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
    }
    if (st != RPK_OK) return st;
    return cuda_status(rpk::launch_attn_decode(p, k_map, v_map, plan, ws, s));
  }
  // Prefill shapes: tcgen05 kernel for head_dim 64 / 128 / 256 and groups up
  // to 128 (an e4m3 cache: head_dim 64 / 128, its codes widened to f16 on chip).
  const int tpt = rpk::prefill_rows_per_tile(p.G);
  if (tpt > 0 && (!p.cache_fp8 || head_dim <= 128)) {
    if (!workspace || workspace_bytes < rpk::kPrefillWorkspaceBytes) return RPK_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RPK_ERR_WORKSPACE;
    CUtensorMap q_map, k_map, v_map;
    const int32_t box_rows = p.P < rpk::kPrefillKeyTile ? p.P : rpk::kPrefillKeyTile;
    const int64_t pool_rows = (int64_t)p.num_pages * p.P;
    st = encode_rows_map(&q_map, q, head_dim, n_heads, total_q_tokens, p.G, tpt);
    if (st != RPK_OK) return st;
    if (p.cache_fp8) {
      st = encode_rows_map_u8(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, box_rows, true);
      if (st != RPK_OK) return st;
      st = encode_rows_map_u8(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, box_rows, true);
    } else {
      st = encode_rows_map(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
      if (st != RPK_OK) return st;
      st = encode_rows_map(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
    }
    if (st != RPK_OK) return st;
    return cuda_status(
        rpk::launch_attn_prefill(p, q_map, k_map, v_map, static_cast<int*>(workspace), s));
  }
  // groups above 128 query heads per KV head, or an e4m3 cache of head_dim
  // 256: CUDA-core kernel.
  return cuda_status(rpk::launch_attn_simt(p, dtype, s));
}

rpk_status ragged_paged_attention_backward(
    const void* q, const int32_t* q_row_offsets, const int32_t* kv_lens,
    const rpk_paged_kv* page_table, int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
    float scale, int32_t window, const void* out, const void* d_out, const float* log_sum_exp,
    float* d_q, float* d_k_pages, float* d_v_pages, int32_t batch, int32_t total_q_tokens,
    int32_t max_q_len, int32_t max_kv_len, rpk_dtype dtype, int32_t sink_tokens, void* stream) {
  if (!q || !q_row_offsets || !kv_lens || !out || !d_out || !log_sum_exp || !d_q || !d_k_pages ||
      !d_v_pages)
    return RPK_ERR_NULL;
  rpk_status st = check_cache(page_table);
  if (st != RPK_OK) return st;
  if (dtype != RPK_BF16 && dtype != RPK_F32) return RPK_ERR_DTYPE;
  if (!cache_dtype_ok(dtype, page_table->cache_dtype)) return RPK_ERR_DTYPE;
  if (n_kv_heads != page_table->n_kv_heads || head_dim != page_table->head_dim)
    return RPK_ERR_SHAPE;
  if (n_heads <= 0 || n_heads % n_kv_heads != 0) return RPK_ERR_SHAPE;
  if (batch <= 0 || batch != page_table->batch || batch > 65535) return RPK_ERR_SHAPE;
  if (total_q_tokens < 0 || max_q_len < 0 || max_kv_len < 0) return RPK_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPK_ERR_SHAPE;
  if (sink_tokens < 0) return RPK_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(out) || !aligned16(d_out) || !aligned16(log_sum_exp) ||
      !aligned16(d_q) || !aligned16(d_k_pages) || !aligned16(d_v_pages))
    return RPK_ERR_SHAPE;
  if ((long long)max_kv_len > (long long)page_table->max_pages_per_seq * page_table->page_size)
    return RPK_ERR_SHAPE;
  if ((long long)max_kv_len > 65535LL * 8) return RPK_ERR_UNSUPPORTED;
  if (total_q_tokens == 0) return RPK_OK;

  rpk::BackwardParams p;
  p.q = q; p.out = out; p.d_out = d_out; p.lse = log_sum_exp;
  {
    void *k, *v;
    rpk::layer_pools(page_table, &k, &v);
    p.k_pages = k; p.v_pages = v;
  }
  p.offsets = q_row_offsets; p.kv_lens = kv_lens; p.block_table = page_table->block_table;
  p.error_word = page_table->error_word;
  p.d_q = d_q; p.d_k = d_k_pages; p.d_v = d_v_pages;
  p.T = total_q_tokens; p.batch = batch; p.H = n_heads; p.Hk = n_kv_heads;
  p.G = n_heads / n_kv_heads; p.d = head_dim; p.P = page_table->page_size;
  p.num_pages = page_table->num_pages; p.max_pages = page_table->max_pages_per_seq;
  p.window = rpk::effective_window(window, max_kv_len);
  p.sinks = p.window > 0 ? sink_tokens : 0;
  p.max_q_len = max_q_len; p.max_kv_len = max_kv_len;
  p.scale = scale;
  p.cache_fp8 = page_table->cache_dtype == RPK_E4M3;
  p.k_scale = page_table->k_scale;
  p.v_scale = page_table->v_scale;
  p.wait_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rpk::attn_backward_tc_supported(p, dtype)) {
    // tcgen05 kernels: TMA maps over q, d_out and the layer's pools
    CUtensorMap q64, do64, q128, do128, k_map, v_map;
    const int32_t box_rows = p.P < 128 ? p.P : 128;
    const int64_t pool_rows = (int64_t)p.num_pages * p.P;
    st = encode_rows_map(&q64, q, head_dim, n_heads, total_q_tokens, p.G, 64 / p.G);
    if (st != RPK_OK) return st;
    st = encode_rows_map(&do64, d_out, head_dim, n_heads, total_q_tokens, p.G, 64 / p.G);
    if (st != RPK_OK) return st;
    st = encode_rows_map(&q128, q, head_dim, n_heads, total_q_tokens, p.G, 128 / p.G);
    if (st != RPK_OK) return st;
    st = encode_rows_map(&do128, d_out, head_dim, n_heads, total_q_tokens, p.G, 128 / p.G);
    if (st != RPK_OK) return st;
    st = encode_rows_map(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
    if (st != RPK_OK) return st;
    st = encode_rows_map(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
    if (st != RPK_OK) return st;
    return cuda_status(
        rpk::launch_attn_backward_tc(p, q64, do64, q128, do128, k_map, v_map, s));
  }
  return cuda_status(rpk::launch_attn_backward(p, dtype, s));
}

}  // extern "C"

// attn_noalloc.cu -- ragged_paged_attention_noalloc: the split-KV decode path
// with its scratch space in a fixed array owned by the library, for callers
// that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory when they call attention: an
// engine that reserved all free HBM for its KV cache at start-up and refuses
// any later allocation, a plugin that runs inside a host framework owning
// every allocator, or a latency-critical decode loop that cannot afford the
// implicit synchronisation of cudaMalloc. This entry point serves them. It
// runs the same decode kernels as ragged_paged_attention, but the kernels'
// fp32 partials go to g_decode_scratch below instead of a caller workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds its RPK_NOALLOC_SCRATCH_BYTES until the process exits. Host
// code cannot use the symbol as a device address (on the host it names a
// stand-in object), so the first call on each device looks up the real
// address with cudaGetSymbolAddress, with that device current, and caches it.
// Nothing in this file allocates: no cudaMalloc, no cudaFree, no library
// allocator.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "../../include/rpk.h"
#include "kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// The decode partials of every ragged_paged_attention_noalloc call on a device.
static __device__ __align__(256) unsigned char g_decode_scratch[RPK_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device; looked up once per device.
rpk_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return rpk::cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return RPK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return rpk::cuda_status(e);
    if (p == nullptr) {
      rpk::set_last_error_text("cudaGetSymbolAddress returned no address");
      return RPK_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RPK_OK;
}

}  // namespace

extern "C" rpk_status ragged_paged_attention_noalloc(
    const void* q, const int32_t* q_row_offsets, const int32_t* kv_lens,
    const rpk_paged_kv* page_table, int32_t n_heads, int32_t n_kv_heads, int32_t head_dim,
    float scale, int32_t window, void* out, int32_t batch, int32_t total_q_tokens,
    int32_t max_q_len, int32_t max_kv_len, rpk_dtype dtype, void* stream) {
  // Host-side checks, the same as ragged_paged_attention's (shared code).
  if (!q || !q_row_offsets || !kv_lens || !out) return RPK_ERR_NULL;
  rpk_status st = rpk::check_cache(page_table);
  if (st != RPK_OK) return st;
  const rpk_paged_kv* c = page_table;
  if (dtype != RPK_BF16 && dtype != RPK_F32) return RPK_ERR_DTYPE;
  if (dtype != c->cache_dtype) return RPK_ERR_DTYPE;
  if (n_kv_heads != c->n_kv_heads || head_dim != c->head_dim) return RPK_ERR_SHAPE;
  if (n_heads <= 0 || n_heads % n_kv_heads != 0) return RPK_ERR_SHAPE;
  if (batch <= 0 || batch != c->batch || batch > 65535) return RPK_ERR_SHAPE;
  if (total_q_tokens < 0 || max_q_len < 0 || max_kv_len < 0) return RPK_ERR_SHAPE;
  if (!(scale > 0.f) || !std::isfinite(scale)) return RPK_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) != 0 || (reinterpret_cast<uintptr_t>(out) & 15u) != 0)
    return RPK_ERR_SHAPE;
  if ((long long)max_kv_len > (long long)c->max_pages_per_seq * c->page_size)
    return RPK_ERR_SHAPE;
  void *k_layer = nullptr, *v_layer = nullptr;
  rpk::layer_pools(c, &k_layer, &v_layer);
  const int32_t group = n_heads / n_kv_heads;
  // Only the split-KV decode path uses scratch; this entry point runs nothing else.
  if (dtype != RPK_BF16 || (long long)max_q_len * group > rpk::kDecodeMaxRows)
    return RPK_ERR_UNSUPPORTED;
  if (total_q_tokens == 0) return RPK_OK;
  const size_t need =
      rpk::decode_workspace_bytes(total_q_tokens, n_heads, head_dim, max_kv_len);
  if (need > (size_t)RPK_NOALLOC_SCRATCH_BYTES) return RPK_ERR_WORKSPACE;

  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != RPK_OK) return st;

  rpk::AttnParams p;
  p.q = q; p.out = out; p.k_pages = k_layer; p.v_pages = v_layer;
  p.offsets = q_row_offsets; p.kv_lens = kv_lens; p.block_table = c->block_table;
  p.error_word = c->error_word;
  p.T = total_q_tokens; p.batch = batch; p.H = n_heads; p.Hk = n_kv_heads; p.G = group;
  p.d = head_dim; p.P = c->page_size; p.num_pages = c->num_pages;
  p.max_pages = c->max_pages_per_seq;
  // As in ragged_paged_attention: a window covering every key is unbounded,
  // which keeps the band arithmetic far from int overflow.
  p.window = rpk::effective_window(window, max_kv_len);
  p.max_q_len = max_q_len; p.max_kv_len = max_kv_len; p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  p.wait_ns = rpk::wait_limit_ns();

  // Partials layout inside the scratch: O [splits, T, H, d] fp32, then (m, l).
  const rpk::DecodePlan plan = rpk::decode_launch_plan(max_kv_len, batch * n_kv_heads, head_dim,
                                                       p.window, max_q_len, 0);
  const size_t rows = (size_t)plan.max_splits * total_q_tokens * n_heads;
  const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) & ~size_t(255);
  rpk::DecodeWorkspace ws;
  ws.o = static_cast<float*>(scratch);
  ws.ml = reinterpret_cast<float2*>(static_cast<char*>(scratch) + o_bytes);

  CUtensorMap k_map, v_map;
  const int32_t box_rows = p.P < rpk::kDecodeTile ? p.P : rpk::kDecodeTile;
  const int64_t pool_rows = (int64_t)p.num_pages * p.P;
  st = rpk::encode_rows_map(&k_map, p.k_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
  if (st != RPK_OK) return st;
  st = rpk::encode_rows_map(&v_map, p.v_pages, head_dim, n_kv_heads, pool_rows, 1, box_rows);
  if (st != RPK_OK) return st;
  return rpk::cuda_status(
      rpk::launch_attn_decode(p, k_map, v_map, plan, ws, static_cast<cudaStream_t>(stream)));
}

// attn_simt.cu -- ragged paged causal GQA attention on CUDA cores, fp32 math.
//
// The path for fp32 tensors (tensor-core tf32 cannot hold the fp32 tolerance)
// and for bf16 shapes the tensor-core kernels do not take. One warp computes
// one (token, head) row: lanes split head_dim, each key's score is a warp
// reduction, and the row keeps the flash online-softmax running state
// (algenta "Attention variant kernels", flash_attention: running max m,
// running sum l rescaled by e^(m_old - m_new), running output likewise, final
// divide). Keys of row r of a sequence with q_len rows and k_len keys are
// [p - (window - 1), p] with p = r + k_len - q_len (NumKong "Attention with a
// Pre-Packed KV-Cache"), plus, under a window, the first `sinks` keys (algenta
// streaming_llm_sink_score); a row with no visible key is written as zeros.
// An e4m3 cache is read as codes widened to fp32; its scales enter once each,
// k_scale in the score scale and v_scale in the final output.
#include "common.cuh"
#include "kernels.h"

namespace rpk {
namespace {

constexpr int kWarps = 8;

// Element e of a cache row as fp32: the value itself, or the e4m3 code.
template <typename T, bool kFp8>
__device__ __forceinline__ float cache_elt(const void* pool, size_t idx) {
  if constexpr (kFp8) return f32_from_e4m3(static_cast<const uint8_t*>(pool)[idx]);
  else return Elt<T>::to_f32(static_cast<const T*>(pool)[idx]);
}

template <typename T, int D, bool kFp8>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(const AttnParams p) {
  constexpr int E = D / 32;  // channels per lane
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= (long long)p.T * p.H) return;
  const int t = (int)(row / p.H);
  const int h = (int)(row - (long long)t * p.H);
  const int b = find_sequence(p.offsets, p.batch, t);
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  const T* qrow = static_cast<const T*>(p.q) + ((size_t)t * p.H + h) * D + lane * E;
  T* orow = static_cast<T*>(p.out) + ((size_t)t * p.H + h) * D + lane * E;

  float o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] = 0.f;
  float l = 0.f;
  float m = -INFINITY;

  const bool len_ok = k_len >= 0 && k_len <= p.max_kv_len && q_len <= p.max_q_len;
  if (!len_ok) {
    if (lane == 0 && h == 0 && t == q0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
  } else {
    const int r = t - q0;
    const int pos = r + k_len - q_len;
    const int lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;
    const int hi = min(pos, k_len - 1);
    const int kvh = h / p.G;
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = Elt<T>::to_f32(qrow[e]);
    const void* __restrict__ kp = p.k_pages;
    const void* __restrict__ vp = p.v_pages;
    const float sl2 = kFp8 ? p.scale_log2 * __ldg(p.k_scale + kvh) : p.scale_log2;
    const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
    // Attention sinks first (keys below the window that stay visible), then the band.
    const int sink_end = min(p.sinks, lo);
    for (int jj = 0; jj < sink_end + (hi - lo + 1); ++jj) {
      const int j = jj < sink_end ? jj : lo + (jj - sink_end);
      const int pi = j / p.P;
      const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
      if (page < 0 || page >= p.num_pages) {
        if (lane == 0) raise_error(p.error_word, RPK_DEVERR_PAGE);
        continue;
      }
      const size_t base = (((size_t)page * p.P + (j - pi * p.P)) * p.Hk + kvh) * D + lane * E;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(qv[e], cache_elt<T, kFp8>(kp, base + e), dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float s = dot * sl2;               // score in log2 units
      const float m_new = fmaxf(m, s);
      const float alpha = exp2f(m - m_new);    // 0 while m = -inf
      const float w = exp2f(s - m_new);
      l = l * alpha + w;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf(w, cache_elt<T, kFp8>(vp, base + e), o[e] * alpha);
      m = m_new;
    }
  }
  float inv = l > 0.f ? 1.f / l : 0.f;
  if (kFp8 && len_ok) inv *= __ldg(p.v_scale + h / p.G);
#pragma unroll
  for (int e = 0; e < E; ++e) orow[e] = Elt<T>::from_f32(o[e] * inv);
  if (p.lse != nullptr && lane == 0) p.lse[row] = lse_from_log2_state(m, l);
}

template <typename T, bool kFp8>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.T * p.H;
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  switch (p.d) {
    case 64: attn_simt_kernel<T, 64, kFp8><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    case 128: attn_simt_kernel<T, 128, kFp8><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    case 256: attn_simt_kernel<T, 256, kFp8><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, rpk_dtype dtype, cudaStream_t stream) {
  if ((long long)p.T * p.H == 0) return cudaSuccess;
  if (p.cache_fp8)
    return dtype == RPK_BF16 ? launch_typed<__nv_bfloat16, true>(p, stream)
                             : launch_typed<float, true>(p, stream);
  return dtype == RPK_BF16 ? launch_typed<__nv_bfloat16, false>(p, stream)
                           : launch_typed<float, false>(p, stream);
}

}  // namespace rpk

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
#include "common.cuh"
#include "kernels.h"

namespace rpk {
namespace {

constexpr int kWarps = 8;

template <typename T, int D>
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
    const T* __restrict__ kp = static_cast<const T*>(p.k_pages);
    const T* __restrict__ vp = static_cast<const T*>(p.v_pages);
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
      for (int e = 0; e < E; ++e) dot = fmaf(qv[e], Elt<T>::to_f32(kp[base + e]), dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float s = dot * p.scale_log2;      // score in log2 units
      const float m_new = fmaxf(m, s);
      const float alpha = exp2f(m - m_new);    // 0 while m = -inf
      const float w = exp2f(s - m_new);
      l = l * alpha + w;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf(w, Elt<T>::to_f32(vp[base + e]), o[e] * alpha);
      m = m_new;
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) orow[e] = Elt<T>::from_f32(o[e] * inv);
  if (p.lse != nullptr && lane == 0) p.lse[row] = lse_from_log2_state(m, l);
}

template <typename T>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.T * p.H;
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  switch (p.d) {
    case 64: attn_simt_kernel<T, 64><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    case 128: attn_simt_kernel<T, 128><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    case 256: attn_simt_kernel<T, 256><<<blocks, kWarps * 32, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, rpk_dtype dtype, cudaStream_t stream) {
  if ((long long)p.T * p.H == 0) return cudaSuccess;
  return dtype == RPK_BF16 ? launch_typed<__nv_bfloat16>(p, stream) : launch_typed<float>(p, stream);
}

}  // namespace rpk

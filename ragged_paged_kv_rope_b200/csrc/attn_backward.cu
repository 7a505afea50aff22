// attn_backward.cu -- gradients of ragged paged causal GQA attention on CUDA
// cores, fp32 math, for the shapes the tensor-core kernels (attn_backward_mma.cu)
// do not take: fp32 tensors, e4m3 caches, groups of more than 16 query heads
// (NumKong "Attention with a Pre-Packed KV-Cache":
// attention_packed_gradients turns the forward's log-sum-exp, its output and
// the output gradient into query, key and value gradients under the same
// band).
//
// With s_ij = scale q_i.k_j, P_ij = e^(s_ij - lse_i) (lse from the forward),
// dP_ij = dO_i.v_j, D_i = dO_i.O_i (O the forward output) and
// dS_ij = P_ij (dP_ij - D_i):
//   dQ_i = scale sum_j dS_ij k_j          (row-parallel kernel: one warp per
//                                          (token, head) walks its keys)
//   dK_j = scale sum_i dS_ij q_i,
//   dV_j = sum_i P_ij dO_i                 (key-parallel kernel: one warp per
//                                          (sequence, key, KV head) walks the
//                                          rows and query heads that see it)
// so neither needs atomics. A key j of a sequence with q_len rows and k_len
// keys is seen by row r (position p = r + k_len - q_len) iff j <= p and, under
// a window w, j >= p - (w - 1) or j < sinks. Lanes split head_dim; each dot
// product is a warp reduction. An e4m3 cache is read as code * scale; the key
// and value gradients are those of the dequantised values.
#include "common.cuh"
#include "kernels.h"

namespace rpk {
namespace {

constexpr int kWarps = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, bool kFp8>
__device__ __forceinline__ float cache_val(const void* pool, size_t idx) {
  if constexpr (kFp8) return f32_from_e4m3(static_cast<const uint8_t*>(pool)[idx]);
  else return Elt<T>::to_f32(static_cast<const T*>(pool)[idx]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Page-pool element offset of key j of sequence b, KV head kvh (channel 0), or
// -1 when its page is outside the pool.
__device__ __forceinline__ long long key_base(const BackwardParams& p, int b, int j, int kvh) {
  const int pi = j / p.P;
  const int page = pi < p.max_pages ? __ldg(p.block_table + (size_t)b * p.max_pages + pi) : -1;
  if (page < 0 || page >= p.num_pages) return -1;
  return (((long long)page * p.P + (j - pi * p.P)) * p.Hk + kvh) * p.d;
}

template <typename T, int D, bool kFp8>
__global__ void __launch_bounds__(kWarps * 32) attn_backward_dq_kernel(const BackwardParams p) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= (long long)p.T * p.H) return;
  const int t = (int)(row / p.H);
  const int h = (int)(row - (long long)t * p.H);
  const int b = find_sequence(p.offsets, p.batch, t);
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  float dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) dq[e] = 0.f;
  const size_t rbase = ((size_t)t * p.H + h) * D + lane * E;
  const float lse = p.lse[row];
  if (k_len < 0 || k_len > p.max_kv_len || q_len > p.max_q_len) {
    if (lane == 0 && h == 0 && t == q0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
  } else if (lse > -INFINITY) {
    const T* q = static_cast<const T*>(p.q) + rbase;
    const T* o = static_cast<const T*>(p.out) + rbase;
    const T* g = static_cast<const T*>(p.d_out) + rbase;
    float qv[E], gv[E], dd = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qv[e] = Elt<T>::to_f32(q[e]);
      gv[e] = Elt<T>::to_f32(g[e]);
      dd = fmaf(gv[e], Elt<T>::to_f32(o[e]), dd);
    }
    const float Dv = warp_sum(dd);
    const int kvh = h / p.G;
    const float ks = kFp8 ? __ldg(p.k_scale + kvh) : 1.f;
    const float vs = kFp8 ? __ldg(p.v_scale + kvh) : 1.f;
    const int r = t - q0;
    const int pos = r + k_len - q_len;
    const int lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;
    const int hi = min(pos, k_len - 1);
    const int sink_end = min(p.sinks, lo);
    const float sl2 = p.scale * kLog2e, lse2 = lse * kLog2e;
    for (int jj = 0; jj < sink_end + (hi - lo + 1); ++jj) {
      const int j = jj < sink_end ? jj : lo + (jj - sink_end);
      const long long kb = key_base(p, b, j, kvh);
      if (kb < 0) {
        if (lane == 0) raise_error(p.error_word, RPK_DEVERR_PAGE);
        continue;
      }
      float k[E], s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        k[e] = cache_val<T, kFp8>(p.k_pages, kb + lane * E + e) * ks;
        s = fmaf(qv[e], k[e], s);
        dp = fmaf(gv[e], cache_val<T, kFp8>(p.v_pages, kb + lane * E + e) * vs, dp);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      const float P = exp2f(s * sl2 - lse2);
      const float ds = P * (dp - Dv) * p.scale;
#pragma unroll
      for (int e = 0; e < E; ++e) dq[e] = fmaf(ds, k[e], dq[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) p.d_q[rbase + e] = dq[e];
}

template <typename T, int D, bool kFp8>
__global__ void __launch_bounds__(kWarps * 32) attn_backward_dkv_kernel(const BackwardParams p) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int j = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int b = blockIdx.y, kvh = blockIdx.z;
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  if (k_len < 0 || k_len > p.max_kv_len || q_len > p.max_q_len || j >= k_len) return;
  const long long kb = key_base(p, b, j, kvh);
  if (kb < 0) return;  // reported by the dQ kernel
  const float ks = kFp8 ? __ldg(p.k_scale + kvh) : 1.f;
  const float vs = kFp8 ? __ldg(p.v_scale + kvh) : 1.f;
  float k[E], v[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    k[e] = cache_val<T, kFp8>(p.k_pages, kb + lane * E + e) * ks;
    v[e] = cache_val<T, kFp8>(p.v_pages, kb + lane * E + e) * vs;
    dk[e] = dv[e] = 0.f;
  }
  // rows that see key j: p = r + off >= j, and under a window p <= j + w - 1 unless j is a sink
  const int off = k_len - q_len;
  const int r_lo = max(0, j - off);
  int r_hi = q_len - 1;
  if (p.window > 0 && j >= p.sinks) r_hi = min(r_hi, j + p.window - 1 - off);
  const float sl2 = p.scale * kLog2e;
  for (int r = r_lo; r <= r_hi; ++r) {
    const int t = q0 + r;
    for (int hg = 0; hg < p.G; ++hg) {
      const int h = kvh * p.G + hg;
      const size_t rbase = ((size_t)t * p.H + h) * D + lane * E;
      const float lse = p.lse[(size_t)t * p.H + h];
      const T* q = static_cast<const T*>(p.q) + rbase;
      const T* o = static_cast<const T*>(p.out) + rbase;
      const T* g = static_cast<const T*>(p.d_out) + rbase;
      float qv[E], gv[E], s = 0.f, dp = 0.f, dd = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        qv[e] = Elt<T>::to_f32(q[e]);
        gv[e] = Elt<T>::to_f32(g[e]);
        s = fmaf(qv[e], k[e], s);
        dp = fmaf(gv[e], v[e], dp);
        dd = fmaf(gv[e], Elt<T>::to_f32(o[e]), dd);
      }
      s = warp_sum(s);
      dp = warp_sum(dp);
      dd = warp_sum(dd);
      const float P = exp2f(s * sl2 - lse * kLog2e);
      const float ds = P * (dp - dd) * p.scale;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dk[e] = fmaf(ds, qv[e], dk[e]);
        dv[e] = fmaf(P, gv[e], dv[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    p.d_k[kb + lane * E + e] = dk[e];
    p.d_v[kb + lane * E + e] = dv[e];
  }
}

template <typename T, bool kFp8, int D>
cudaError_t launch_d(const BackwardParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.T * p.H;
  if (rows > 0)
    attn_backward_dq_kernel<T, D, kFp8>
        <<<(unsigned)((rows + kWarps - 1) / kWarps), kWarps * 32, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.max_kv_len == 0) return e;
  dim3 grid((unsigned)((p.max_kv_len + kWarps - 1) / kWarps), (unsigned)p.batch, (unsigned)p.Hk);
  attn_backward_dkv_kernel<T, D, kFp8><<<grid, kWarps * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename T, bool kFp8>
cudaError_t launch_t(const BackwardParams& p, cudaStream_t stream) {
  switch (p.d) {
    case 64: return launch_d<T, kFp8, 64>(p, stream);
    case 128: return launch_d<T, kFp8, 128>(p, stream);
    case 256: return launch_d<T, kFp8, 256>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_attn_backward(const BackwardParams& p, rpk_dtype dtype, cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  if (attn_backward_mma_supported(p, dtype)) return launch_attn_backward_mma(p, stream);
  if (dtype == RPK_BF16)
    return p.cache_fp8 ? launch_t<__nv_bfloat16, true>(p, stream)
                       : launch_t<__nv_bfloat16, false>(p, stream);
  return p.cache_fp8 ? launch_t<float, true>(p, stream) : launch_t<float, false>(p, stream);
}

}  // namespace rpk

// rope.cu -- fused RoPE on Q and K with K/V scattered into the paged cache.
//
// Semantics: Mojo "generic_fused_qk_rope_bshd_paged_ragged_kernel_api" (ragged
// rows by input_row_offsets, rotation of Q into the output and of K into the
// paged cache, interleaved vs half pairing, per-token position_ids, M-RoPE
// sections) and aria_kernel's rope / rope_half / rope_half_partial (pairings
// and partial rotary_dim). Pair (a, b) at angle theta becomes
// (a cos - b sin, b cos + a sin), with (cos, sin) read from freqs_cis[pos].
//
// Design: pure bandwidth. One CTA per 1-4 tokens (4 when there are enough
// tokens to fill the GPU several times over, 1 for small decode batches so
// that they still spread over many SMs); the per-token metadata
// (sequence, cache slot, page, positions) is computed once per token by one
// thread each and shared, then the CTA's threads walk 16-byte units of the
// tokens' q, k and v head rows. A rotation unit of the half layout holds
// kVec pairs (kVec channels from each half), one of the interleaved layout a
// 16-byte chunk of kVec/2 adjacent pairs, whose (cos, sin) entries are the
// same 16-byte-aligned run of the table row. Channels >= rotary_dim and V rows
// are 16-byte copies. Every global load is a 16-byte vector.
//
// An e4m3 cache (Mojo's cache_dtype with per-head scales) receives
// e4m3(k' / k_scale[kvh]) and e4m3(v / v_scale[kvh]) of the fp32 values: the
// quotient is an IEEE fp32 division, rounded once to the nearest code with
// ties to even and saturated to +-448; a unit of V elements becomes V bytes.
#include "common.cuh"
#include "kernels.h"

namespace rpk {
namespace {

constexpr int kThreads = 256;
constexpr int kTokens = 4;  // most tokens per CTA

struct TokenInfo {
  int page;         // -1 when the slot has no valid page
  int row_in_page;
  int pos[3];       // position of each M-RoPE section (all equal without M-RoPE)
  int pos_ok;
};

// V fp32 values divided by `scale` -> V e4m3 codes at dst (V = 4 or 8 bytes).
template <int V>
__device__ __forceinline__ void store_e4m3(uint8_t* dst, const float* x, float scale) {
  uint32_t w[V / 4];
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const uint32_t lo = e4m3x2_from_f32(__fdiv_rn(x[4 * i], scale), __fdiv_rn(x[4 * i + 1], scale));
    const uint32_t hi =
        e4m3x2_from_f32(__fdiv_rn(x[4 * i + 2], scale), __fdiv_rn(x[4 * i + 3], scale));
    w[i] = lo | (hi << 16);
  }
  if constexpr (V == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  else *reinterpret_cast<uint32_t*>(dst) = w[0];
}

template <typename T, bool kInterleaved, bool kFp8>
__global__ void __launch_bounds__(kThreads) rope_scatter_kernel(const RopeParams p) {
  constexpr int V = Elt<T>::kVec;
  __shared__ TokenInfo info[kTokens];
  const int t0 = blockIdx.x * p.tokens_per_cta;
  const int ntok = min(p.tokens_per_cta, p.T - t0);
  if (ntok <= 0) return;

  if (threadIdx.x < ntok) {
    // Sequence, index in it, cache slot and page of this token.
    const int t = t0 + threadIdx.x;
    const int b = find_sequence(p.offsets, p.batch, t);
    const int i = t - __ldg(p.offsets + b);
    const int slot = __ldg(p.cache_lens + b) + i;
    int page = -1;
    if (slot >= 0) {
      const int pi = slot / p.P;
      if (pi < p.max_pages) page = __ldg(p.block_table + (size_t)b * p.max_pages + pi);
    }
    TokenInfo ti;
    ti.page = (page >= 0 && page < p.num_pages) ? page : -1;
    ti.row_in_page = slot >= 0 ? slot % p.P : 0;
    if (p.position_ids == nullptr) {
      ti.pos[0] = ti.pos[1] = ti.pos[2] = slot;
    } else if (p.has_mrope) {
#pragma unroll
      for (int s = 0; s < 3; ++s) ti.pos[s] = __ldg(p.position_ids + (size_t)s * p.T + t);
    } else {
      ti.pos[0] = ti.pos[1] = ti.pos[2] = __ldg(p.position_ids + t);
    }
    bool ok = true;
#pragma unroll
    for (int s = 0; s < 3; ++s) ok &= (ti.pos[s] >= 0 && ti.pos[s] < p.max_position);
    ti.pos_ok = ok;
    info[threadIdx.x] = ti;
    if (ti.page < 0) raise_error(p.error_word, RPK_DEVERR_PAGE);
    if (!ok) raise_error(p.error_word, RPK_DEVERR_POSITION);
  }
  __syncthreads();

  const int half = p.R >> 1;
  // Units per head row: rotation units, then pass-through units.
  const int rot_units = kInterleaved ? p.R / V : half / V;
  const int pass_units = (p.d - p.R) / V;
  const int units_row = rot_units + pass_units;
  const int q_units = p.H * units_row;
  const int k_units = p.Hk * units_row;
  const int v_units = p.Hk * (p.d / V);
  const int per_token = q_units + k_units + v_units;
  const int total = per_token * ntok;

  const T* __restrict__ q = static_cast<const T*>(p.q);
  const T* __restrict__ kn = static_cast<const T*>(p.k_new);
  const T* __restrict__ vn = static_cast<const T*>(p.v_new);
  T* out_q = static_cast<T*>(p.out_q);
  T* kp = static_cast<T*>(p.k_pages);
  T* vp = static_cast<T*>(p.v_pages);
  uint8_t* kp8 = static_cast<uint8_t*>(p.k_pages);
  uint8_t* vp8 = static_cast<uint8_t*>(p.v_pages);

  for (int uu = threadIdx.x; uu < total; uu += kThreads) {
    const int tk = uu / per_token;
    const int u = uu - tk * per_token;
    const int t = t0 + tk;
    const TokenInfo& ti = info[tk];
    const int page = ti.page;
    const bool page_ok = page >= 0;
    const int row_in_page = ti.row_in_page;
    const bool pos_ok = ti.pos_ok != 0;
    const int* pos = ti.pos;
    const T* src;
    T* dst;
    int unit;
    if (u < q_units + k_units) {
      int row;
      bool to_cache = false;  // a K row of an e4m3 cache
      size_t crow = 0;        // its element offset in the pool
      float kscale = 1.f;
      if (u < q_units) {
        row = u / units_row;
        unit = u - row * units_row;
        src = q + ((size_t)t * p.H + row) * p.d;
        dst = out_q + ((size_t)t * p.H + row) * p.d;
      } else {
        if (!page_ok) continue;
        const int uk = u - q_units;
        row = uk / units_row;
        unit = uk - row * units_row;
        src = kn + ((size_t)t * p.Hk + row) * p.d;
        crow = (((size_t)page * p.P + row_in_page) * p.Hk + row) * p.d;
        dst = kp + crow;
        if constexpr (kFp8) {
          to_cache = true;
          kscale = __ldg(p.k_scale + row);
        }
      }
      // V elements at channel `off` of the row: to the output dtype, or to e4m3 codes.
      auto put = [&](int off, const float* x) {
        if (kFp8 && to_cache) store_e4m3<V>(kp8 + crow + off, x, kscale);
        else store16(dst + off, x);
      };
      if (unit >= rot_units) {  // channels >= rotary_dim: copy
        const int off = p.R + (unit - rot_units) * V;
        if (kFp8 && to_cache) {
          float x[V];
          load16(src + off, x);
          put(off, x);
        } else {
          *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + off);
        }
        continue;
      }
      if (!pos_ok) continue;
      // Pairs covered by this unit and the channels of their two members.
      const int j0 = kInterleaved ? unit * (V / 2) : unit * V;
      constexpr int NP = kInterleaved ? V / 2 : V;
      const int s0 = p.has_mrope ? (j0 < p.sec_end0 ? 0 : (j0 < p.sec_end1 ? 1 : 2)) : 0;
      const int jl = j0 + NP - 1;
      const int s1 = p.has_mrope ? (jl < p.sec_end0 ? 0 : (jl < p.sec_end1 ? 1 : 2)) : 0;
      float cs[2 * NP];  // (cos, sin) of each pair
      if (s0 == s1) {
        const float* tab = p.freqs + (size_t)pos[s0] * p.R + 2 * j0;
#pragma unroll
        for (int k = 0; k < 2 * NP; k += 4) {
          const float4 c4 = __ldg(reinterpret_cast<const float4*>(tab + k));
          cs[k] = c4.x; cs[k + 1] = c4.y; cs[k + 2] = c4.z; cs[k + 3] = c4.w;
        }
      } else {  // the unit straddles an M-RoPE section boundary
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          const int j = j0 + k;
          const int s = j < p.sec_end0 ? 0 : (j < p.sec_end1 ? 1 : 2);
          const float* tab = p.freqs + (size_t)pos[s] * p.R + 2 * j;
          cs[2 * k] = __ldg(tab);
          cs[2 * k + 1] = __ldg(tab + 1);
        }
      }
      if (kInterleaved) {
        float x[V];
        load16(src + 2 * j0, x);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          const float a = x[2 * k], bb = x[2 * k + 1], c = cs[2 * k], s = cs[2 * k + 1];
          x[2 * k] = fmaf(a, c, -bb * s);
          x[2 * k + 1] = fmaf(bb, c, a * s);
        }
        put(2 * j0, x);
      } else {
        float x1[V], x2[V];
        load16(src + j0, x1);
        load16(src + half + j0, x2);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
          const float a = x1[k], bb = x2[k], c = cs[2 * k], s = cs[2 * k + 1];
          x1[k] = fmaf(a, c, -bb * s);
          x2[k] = fmaf(bb, c, a * s);
        }
        put(j0, x1);
        put(half + j0, x2);
      }
    } else {  // V rows: copy into the cache slot
      if (!page_ok) continue;
      const int uv = u - q_units - k_units;
      const int row = uv / (p.d / V);
      const int off = (uv - row * (p.d / V)) * V;
      src = vn + ((size_t)t * p.Hk + row) * p.d + off;
      const size_t crow = (((size_t)page * p.P + row_in_page) * p.Hk + row) * p.d + off;
      if constexpr (kFp8) {
        float x[V];
        load16(src, x);
        store_e4m3<V>(vp8 + crow, x, __ldg(p.v_scale + row));
      } else {
        *reinterpret_cast<uint4*>(vp + crow) = *reinterpret_cast<const uint4*>(src);
      }
    }
  }
}

// Table of width W (W/2 pairs): freqs_cis[p][2j] = cos(p * theta^(-2j/denom)),
// [2j+1] = sin(...), in fp64 and rounded once, for pairs j < n_rot; (1, 0) for
// the others. Plain RoPE: W = denom = rotary_dim, n_rot = W/2. p-RoPE (algenta
// rope_half_proportional): W = denom = head_dim, n_rot = the rotated pairs.
__global__ void freqs_cis_kernel(float* __restrict__ out, int32_t max_position, int32_t W,
                                 int32_t denom, int32_t n_rot, double theta) {
  const int half = W >> 1;
  const long long n = (long long)max_position * half;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(idx / half);
    const int j = (int)(idx - (long long)pos * half);
    double s = 0.0, c = 1.0;
    if (j < n_rot) {
      const double omega = pow(theta, -2.0 * (double)j / (double)denom);
      sincos((double)pos * omega, &s, &c);
    }
    out[(size_t)pos * W + 2 * j] = __double2float_rn(c);
    out[(size_t)pos * W + 2 * j + 1] = __double2float_rn(s);
  }
}

}  // namespace

cudaError_t launch_rope(const RopeParams& p, rpk_dtype dtype, bool interleaved,
                        cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  RopeParams q = p;
  q.tokens_per_cta = p.T >= 8 * 148 * kTokens ? kTokens : 1;
  dim3 grid((p.T + q.tokens_per_cta - 1) / q.tokens_per_cta), block(kThreads);
  auto go = [&](auto kernel) { kernel<<<grid, block, 0, stream>>>(q); };
  if (dtype == RPK_BF16) {
    if (p.cache_fp8) {
      if (interleaved) go(rope_scatter_kernel<__nv_bfloat16, true, true>);
      else go(rope_scatter_kernel<__nv_bfloat16, false, true>);
    } else {
      if (interleaved) go(rope_scatter_kernel<__nv_bfloat16, true, false>);
      else go(rope_scatter_kernel<__nv_bfloat16, false, false>);
    }
  } else {
    if (p.cache_fp8) {
      if (interleaved) go(rope_scatter_kernel<float, true, true>);
      else go(rope_scatter_kernel<float, false, true>);
    } else {
      if (interleaved) go(rope_scatter_kernel<float, true, false>);
      else go(rope_scatter_kernel<float, false, false>);
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_freqs_cis(float* out, int32_t max_position, int32_t width, int32_t denom,
                             int32_t rotated_pairs, double theta, cudaStream_t stream) {
  const long long n = (long long)max_position * (width / 2);
  if (n == 0) return cudaSuccess;
  long long blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  freqs_cis_kernel<<<(unsigned)blocks, 256, 0, stream>>>(out, max_position, width, denom,
                                                         rotated_pairs, theta);
  return cudaGetLastError();
}

}  // namespace rpk

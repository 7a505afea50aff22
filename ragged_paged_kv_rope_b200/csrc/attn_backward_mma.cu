// attn_backward_mma.cu -- gradients of ragged paged causal GQA attention for
// bf16 tensors over a bf16 cache, on warp-level tensor cores (mma.sync
// m16n8k16: bf16 operands, fp32 accumulators).
//
// The same gradients as the CUDA-core kernels (NumKong "Attention with a
// Pre-Packed KV-Cache", attention_packed_gradients): with s_ij = scale q_i.k_j,
// P_ij = e^(s_ij - lse_i), dP_ij = dO_i.v_j, D_i = dO_i.O_i and
// dS_ij = P_ij (dP_ij - D_i),
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO,
// each a sum over the (row, key) pairs of the forward's band. The G query heads
// of one KV head share its keys, so query rows are packed as (token, head):
// packed row rho of a block holds token rho / G and head rho % G, 64 rows per
// block (64 / G tokens), as the forward packs its query tiles.
//
// Three kernels, no atomics (each output element has one writer), in launch
// order:
//   D   -- D_i of every row, kept in d_q's memory until the dQ kernel
//          overwrites it.
//   dKV -- one CTA per 64 keys; its four warps own 16 keys each and walk the
//          row blocks that see them: S^T = K Q^T, dP^T = V dO^T,
//          dV += P^T dO and dK += dS^T Q. For head_dim 256 two CTAs share a key
//          block, each accumulating half of the output channels.
//   dQ  -- one CTA per 64 packed rows; its four warps own 16 rows each and walk
//          the key tiles of the rows' band (sink tiles, then the window):
//          S = Q K^T and dP = dO V^T from shared memory, P and dS in registers,
//          dQ += dS K with dS reused as the A operand (bf16).
// Tiles are staged in shared memory by cp.async (16-byte chunks, XOR-swizzled
// by row so that ldmatrix reads are conflict-free), two stages deep. P and dS
// are rounded to bf16 as operands of the second products; every sum is fp32.
#include "common.cuh"
#include "kernels.h"

namespace rpk {
namespace {

constexpr int kRows = 64;   // packed query rows per block
constexpr int kKeys = 64;   // keys per tile / block
constexpr int kThreads = 128;
constexpr float kLog2eMma = 1.4426950408889634f;

// Byte offset of 16-byte chunk c of row r in a [64][D] bf16 tile (rows of 2D
// bytes; the chunk index is XORed with the row's low three bits).
template <int D>
__device__ __forceinline__ uint32_t toff(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

// 16 bytes global -> shared, or 16 zero bytes when !valid (no global read).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
// 4 bytes global -> shared, or 4 zero bytes when !valid (no global read).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ldmatrix lane addresses (lane i, tile base `base`):
//   A operand, 16 rows from r0 x 16 columns from chunk 2 ks (row-major tile);
//   B operand of two n-tiles, 16 rows (n) from n0 x 16 columns (k) from chunk
//   2 ks, read as stored (tile rows are n: K for Q K^T);
//   B operand of two n-tiles via .trans, 16 rows (k) from k0 x 16 columns (n)
//   from chunk c0 (tile rows are k: K for dS K).
template <int D>
__device__ __forceinline__ uint32_t a_addr(uint32_t base, int lane, int r0, int ks) {
  return base + toff<D>(r0 + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * ks + (lane >> 4));
}
template <int D>
__device__ __forceinline__ uint32_t b_addr(uint32_t base, int lane, int n0, int ks) {
  return base + toff<D>(n0 + (lane & 7) + (lane >> 4) * 8, 2 * ks + ((lane >> 3) & 1));
}
template <int D>
__device__ __forceinline__ uint32_t bt_addr(uint32_t base, int lane, int k0, int c0) {
  return base + toff<D>(k0 + (lane & 7) + ((lane >> 3) & 1) * 8, c0 + (lane >> 4));
}

// Key j is visible to the row at position pos (keys [pos - (w - 1), pos] under
// a window w > 0, plus keys below `sinks`; every key <= pos otherwise).
__device__ __forceinline__ bool visible(int j, int pos, int window, int sinks) {
  return j <= pos && (window == 0 || j > pos - window || j < sinks);
}

// Pool row (element offset of channel 0) of key j of sequence b, KV head kvh,
// or -1 when its page is outside the pool.
__device__ __forceinline__ long long pool_row(const BackwardParams& p, int b, int j, int kvh) {
  const int pi = j / p.P;
  const int page = pi < p.max_pages ? __ldg(p.block_table + (size_t)b * p.max_pages + pi) : -1;
  if (page < 0 || page >= p.num_pages) return -1;
  return (((long long)page * p.P + (j - pi * p.P)) * p.Hk + kvh) * p.d;
}

// K and V rows of keys [key0, key0 + 64) into [64][D] tiles; keys at or past
// k_len, and keys on a page outside the pool (reported when `report`), are
// zero rows.
template <int D>
__device__ __forceinline__ void load_keys(const BackwardParams& p, int b, int kvh, int k_len,
                                          int key0, uint32_t sk, uint32_t sv, bool report) {
  constexpr int CH = D / 8;
  const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(p.k_pages);
  const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(p.v_pages);
  for (int idx = threadIdx.x; idx < kKeys * CH; idx += kThreads) {
    const int r = idx / CH, c = idx - (idx / CH) * CH;
    const int j = key0 + r;
    long long row = -1;
    if (j < k_len) {
      row = pool_row(p, b, j, kvh);
      if (row < 0 && report && c == 0) raise_error(p.error_word, RPK_DEVERR_PAGE);
    }
    const bool ok = row >= 0;
    const size_t e = ok ? (size_t)row + c * 8 : 0;
    cp_async16(sk + toff<D>(r, c), kp + e, ok);
    cp_async16(sv + toff<D>(r, c), vp + e, ok);
  }
}

// Rows of a [T, H, D] tensor for the packed rows of a block: tokens
// [tok0, tok0 + 64 / G) of the sequence starting at q0, the G heads of KV head
// kvh; rows past the block's tokens are zero.
template <int D>
__device__ __forceinline__ void load_rows(const BackwardParams& p, const __nv_bfloat16* src,
                                          int q0, int tok_end, int kvh, int tok0, uint32_t dst) {
  constexpr int CH = D / 8;
  const int G = p.G;
  const int tpb = kRows / G;
  for (int idx = threadIdx.x; idx < kRows * CH; idx += kThreads) {
    const int r = idx / CH, c = idx - (idx / CH) * CH;
    const int tk = r / G;
    const int tok = tok0 + tk;
    const bool ok = tk < tpb && tok < tok_end;
    const size_t e = ok ? ((size_t)(q0 + tok) * p.H + kvh * G + (r - tk * G)) * D + c * 8 : 0;
    cp_async16(dst + toff<D>(r, c), src + e, ok);
  }
}

// D_i = dO_i . O_i of packed row `r` of a block, summed by the `n` lanes of
// an aligned lane group (each takes D / n channels, 8 at a time).
template <int D>
__device__ __forceinline__ float row_delta(const BackwardParams& p, size_t row_elt, int part,
                                           int n) {
  const uint4* g = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.d_out) + row_elt);
  const uint4* o = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) + row_elt);
  float acc = 0.f;
  for (int c = part; c < D / 8; c += n) {
    const uint4 gv = __ldg(g + c), ov = __ldg(o + c);
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, ow[4] = {ov.x, ov.y, ov.z, ov.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[k]));
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[k]));
      acc = fmaf(gf.x, of.x, acc);
      acc = fmaf(gf.y, of.y, acc);
    }
  }
  return acc;
}

// ------------------------------------------------------------------- D

// D_i of every (token, head) row into delta[t * H + h]; eight lanes per row.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const BackwardParams p,
                                                             float* __restrict__ delta) {
  const long long row = ((long long)blockIdx.x * 256 + threadIdx.x) >> 3;
  const bool ok = row < (long long)p.T * p.H;
  float v = ok ? row_delta<D>(p, (size_t)row * D, threadIdx.x & 7, 8) : 0.f;
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  if (ok && (threadIdx.x & 7) == 0) delta[row] = v;
}

// ------------------------------------------------------------------- dQ

template <int D>
__global__ void __launch_bounds__(kThreads) attn_bwd_dq_mma_kernel(const BackwardParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TB = kRows * D * 2;  // one [64][D] bf16 tile
  constexpr int NT = D / 8;          // 8-channel n-tiles of a row
  const uint32_t sQ = smem_u32(smem), sG = sQ + TB, sK = sQ + 2 * TB, sV = sQ + 4 * TB;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int b = blockIdx.y, kvh = blockIdx.z;
  const int G = p.G, tpb = kRows / G;
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  // the last (longest) row blocks of a sequence first
  const int blk = (int)gridDim.x - 1 - (int)blockIdx.x;
  const int tok0 = blk * tpb;
  if (k_len < 0 || k_len > p.max_kv_len || q_len > p.max_q_len) {
    if (threadIdx.x == 0 && kvh == 0 && blockIdx.x == 0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
    return;
  }
  if (tok0 >= q_len) return;
  const int tok_end = min(q_len, tok0 + tpb);
  const int off = k_len - q_len;

  // This thread's two packed rows (g and g + 8 of its warp's 16).
  int pos[2];
  float lse2[2], delta[2];
  size_t out_elt[2];
  bool row_ok[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int r = warp * 16 + g + 8 * u;
    const int tk = r / G;
    const int tok = tok0 + tk;
    row_ok[u] = tk < tpb && tok < tok_end;
    out_elt[u] = row_ok[u] ? ((size_t)(q0 + tok) * p.H + kvh * G + (r - tk * G)) * D : 0;
    const float l = row_ok[u] ? p.lse[out_elt[u] / D] : -INFINITY;
    delta[u] = row_ok[u] ? row_delta<D>(p, out_elt[u], c, 4) : 0.f;
    delta[u] += __shfl_xor_sync(0xffffffffu, delta[u], 1);
    delta[u] += __shfl_xor_sync(0xffffffffu, delta[u], 2);
    // rows with no visible key (lse = -inf) take no gradient
    pos[u] = row_ok[u] && l > -INFINITY ? tok + off : INT_MIN / 2;
    lse2[u] = l * kLog2eMma;
  }

  // Key tiles of the block's band: [lo, hi] of its first and last rows, with
  // the sink tiles below the window first.
  const int pos_first = tok0 + off, pos_last = tok_end - 1 + off;
  const int hi = min(pos_last, k_len - 1);
  const int lo = p.window > 0 ? max(0, pos_first - p.window + 1) : 0;
  const int hi_tile = hi >= 0 ? hi / kKeys : -1;
  const int lo_tile = lo / kKeys;
  const int sink_tiles = p.window > 0 ? (min(p.sinks, lo) + kKeys - 1) / kKeys : 0;
  auto next_tile = [&](int kt) { return kt + 1 < sink_tiles ? kt + 1 : max(kt + 1, lo_tile); };
  int kt = sink_tiles > 0 ? 0 : lo_tile;

  float dq[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
  // Up to head_dim 128 the warp's Q and dO fragments stay in registers for the
  // whole key walk; at 256 they are re-read from shared memory.
  constexpr bool kFragRegs = D <= 128;
  constexpr int KF = kFragRegs ? D / 16 : 1;
  uint32_t qf[KF][4], gf[KF][4];

  const float sl2 = p.scale * kLog2eMma;
  if (kt <= hi_tile) {
    load_rows<D>(p, static_cast<const __nv_bfloat16*>(p.q), q0, tok_end, kvh, tok0, sQ);
    load_rows<D>(p, static_cast<const __nv_bfloat16*>(p.d_out), q0, tok_end, kvh, tok0, sG);
    load_keys<D>(p, b, kvh, k_len, kt * kKeys, sK, sV, true);
    cp_async_commit();
    for (int it = 0; kt <= hi_tile; ++it) {
      const int st = it & 1;
      const int nkt = next_tile(kt);
      if (nkt <= hi_tile) {
        load_keys<D>(p, b, kvh, k_len, nkt * kKeys, sK + (st ^ 1) * TB, sV + (st ^ 1) * TB, true);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      if (kFragRegs && it == 0) {
#pragma unroll
        for (int ks = 0; ks < KF; ++ks) {
          ldsm_x4(a_addr<D>(sQ, lane, warp * 16, ks), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
          ldsm_x4(a_addr<D>(sG, lane, warp * 16, ks), gf[ks][0], gf[ks][1], gf[ks][2], gf[ks][3]);
        }
      }
      const uint32_t k_t = sK + st * TB, v_t = sV + st * TB;
      const int key0 = kt * kKeys;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float s[4][4], dp[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t aq[4], ag[4];
          if constexpr (kFragRegs) {
#pragma unroll
            for (int i = 0; i < 4; ++i) aq[i] = qf[ks][i], ag[i] = gf[ks][i];
          } else {
            ldsm_x4(a_addr<D>(sQ, lane, warp * 16, ks), aq[0], aq[1], aq[2], aq[3]);
            ldsm_x4(a_addr<D>(sG, lane, warp * 16, ks), ag[0], ag[1], ag[2], ag[3]);
          }
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(b_addr<D>(k_t, lane, half * 32 + np * 16, ks), b0, b1, b2, b3);
            mma_bf16(s[2 * np], aq, b0, b1);
            mma_bf16(s[2 * np + 1], aq, b2, b3);
            ldsm_x4(b_addr<D>(v_t, lane, half * 32 + np * 16, ks), b0, b1, b2, b3);
            mma_bf16(dp[2 * np], ag, b0, b1);
            mma_bf16(dp[2 * np + 1], ag, b2, b3);
          }
        }
        // dS = P (dP - D) on the visible pairs, 0 elsewhere
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int u = e >> 1;
            const int j = key0 + half * 32 + n * 8 + 2 * c + (e & 1);
            const float pr =
                visible(j, pos[u], p.window, p.sinks) ? fast_exp2(s[n][e] * sl2 - lse2[u]) : 0.f;
            s[n][e] = pr * (dp[n][e] - delta[u]);
          }
        // dQ += dS K over the 32 keys (two k-steps of 16)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint32_t a[4] = {pack_bf16x2(s[2 * m][0], s[2 * m][1]),
                                 pack_bf16x2(s[2 * m][2], s[2 * m][3]),
                                 pack_bf16x2(s[2 * m + 1][0], s[2 * m + 1][1]),
                                 pack_bf16x2(s[2 * m + 1][2], s[2 * m + 1][3])};
#pragma unroll
          for (int cp = 0; cp < NT / 2; ++cp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(bt_addr<D>(k_t, lane, half * 32 + m * 16, cp * 2), b0, b1, b2, b3);
            mma_bf16(dq[2 * cp], a, b0, b1);
            mma_bf16(dq[2 * cp + 1], a, b2, b3);
          }
        }
      }
      __syncthreads();  // the stage is read; the next prefetch may overwrite it
      kt = nkt;
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    if (!row_ok[u]) continue;
    float* dst = p.d_q + out_elt[u] + 2 * c;
#pragma unroll
    for (int n = 0; n < NT; ++n)
      *reinterpret_cast<float2*>(dst + n * 8) =
          make_float2(dq[n][2 * u] * p.scale, dq[n][2 * u + 1] * p.scale);
  }
}

// ------------------------------------------------------------------ dK, dV

template <int D, int DC>
__global__ void __launch_bounds__(kThreads) attn_bwd_dkv_mma_kernel(const BackwardParams p,
                                                                    const float* __restrict__ delta) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TB = kRows * D * 2;
  constexpr int NT = DC / 8;            // 8-channel n-tiles of this CTA's output channels
  constexpr int kSplit = D / DC;
  const uint32_t sK = smem_u32(smem), sV = sK + TB, sQ = sK + 2 * TB, sG = sK + 4 * TB;
  int* m_pos = reinterpret_cast<int*>(smem + 6 * TB);           // [2][64]
  float* m_lse = reinterpret_cast<float*>(m_pos + 2 * kRows);   // [2][64]
  float* m_delta = m_lse + 2 * kRows;                           // [2][64]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  // grid (KV head x channel half, sequence, key block): the key block varies
  // slowest, so the first key blocks of every sequence (those the most rows
  // see) are the first to run and the short ones fill the tail
  const int b = blockIdx.y;
  const int kvh = blockIdx.x / kSplit, ch0 = (blockIdx.x % kSplit) * DC;
  const int G = p.G, tpb = kRows / G;
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  const int key0 = blockIdx.z * kKeys;
  // bad lengths are reported by the dQ kernel
  if (k_len < 0 || k_len > p.max_kv_len || q_len > p.max_q_len || key0 >= k_len) return;
  const int off = k_len - q_len;

  // rows that see a key of the block: position >= key0, and under a window
  // position <= last key + w - 1 unless the block holds a sink key
  const int key_last = min(key0 + kKeys, k_len) - 1;
  const int r_lo = max(0, key0 - off);
  int r_hi = q_len - 1;
  if (p.window > 0 && key0 >= p.sinks) r_hi = min(r_hi, key_last + p.window - 1 - off);
  const int n_blocks = r_hi >= r_lo ? (r_hi - r_lo) / tpb + 1 : 0;

  float dk[NT][4], dv[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  // Row metadata of block rb into stage st: the position (INT_MIN / 2 for
  // rows past the block's tokens; a row whose forward saw no key sees none
  // here either), and lse and D by cp.async (zero for those rows).
  auto load_meta = [&](int rb, int st) {
    const int r = threadIdx.x & (kRows - 1);
    const int tk = r / G;
    const int tok = r_lo + rb * tpb + tk;
    const bool ok = tk < tpb && tok <= r_hi;
    const size_t row = ok ? (size_t)(q0 + tok) * p.H + kvh * G + (r - tk * G) : 0;
    if (threadIdx.x < kRows) {
      m_pos[st * kRows + r] = ok ? tok + off : INT_MIN / 2;
      cp_async4(smem_u32(m_lse + st * kRows + r), p.lse + row, ok);
    } else {
      cp_async4(smem_u32(m_delta + st * kRows + r), delta + row, ok);
    }
  };
  auto load_block = [&](int rb, int st) {
    const int t0 = r_lo + rb * tpb;
    const int t_end = min(r_hi + 1, t0 + tpb);
    load_rows<D>(p, static_cast<const __nv_bfloat16*>(p.q), q0, t_end, kvh, t0, sQ + st * TB);
    load_rows<D>(p, static_cast<const __nv_bfloat16*>(p.d_out), q0, t_end, kvh, t0, sG + st * TB);
  };

  const float sl2 = p.scale * kLog2eMma;
  if (n_blocks > 0) {
    load_keys<D>(p, b, kvh, k_len, key0, sK, sV, false);
    load_block(0, 0);
    load_meta(0, 0);
    cp_async_commit();
    for (int rb = 0; rb < n_blocks; ++rb) {
      const int st = rb & 1;
      if (rb + 1 < n_blocks) {
        load_block(rb + 1, st ^ 1);
        load_meta(rb + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint32_t q_t = sQ + st * TB, g_t = sG + st * TB;
      const int* mp = m_pos + st * kRows;
      const float* ml = m_lse + st * kRows;
      const float* md = m_delta + st * kRows;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float s[4][4], dp[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t ak[4], av[4];
          ldsm_x4(a_addr<D>(sK, lane, warp * 16, ks), ak[0], ak[1], ak[2], ak[3]);
          ldsm_x4(a_addr<D>(sV, lane, warp * 16, ks), av[0], av[1], av[2], av[3]);
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(b_addr<D>(q_t, lane, half * 32 + np * 16, ks), b0, b1, b2, b3);
            mma_bf16(s[2 * np], ak, b0, b1);
            mma_bf16(s[2 * np + 1], ak, b2, b3);
            ldsm_x4(b_addr<D>(g_t, lane, half * 32 + np * 16, ks), b0, b1, b2, b3);
            mma_bf16(dp[2 * np], av, b0, b1);
            mma_bf16(dp[2 * np + 1], av, b2, b3);
          }
        }
        // P^T and dS^T: element (key, row) with row the column index
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = half * 32 + n * 8 + 2 * c + (e & 1);
            const int j = key0 + warp * 16 + g + 8 * (e >> 1);
            const float pr = visible(j, mp[col], p.window, p.sinks)
                                 ? fast_exp2(fmaf(s[n][e], sl2, -ml[col] * kLog2eMma))
                                 : 0.f;
            s[n][e] = pr;
            dp[n][e] = pr * (dp[n][e] - md[col]);
          }
        // dV += P^T dO and dK += dS^T Q over the 32 rows (two k-steps of 16)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint32_t ap[4] = {pack_bf16x2(s[2 * m][0], s[2 * m][1]),
                                  pack_bf16x2(s[2 * m][2], s[2 * m][3]),
                                  pack_bf16x2(s[2 * m + 1][0], s[2 * m + 1][1]),
                                  pack_bf16x2(s[2 * m + 1][2], s[2 * m + 1][3])};
          const uint32_t ad[4] = {pack_bf16x2(dp[2 * m][0], dp[2 * m][1]),
                                  pack_bf16x2(dp[2 * m][2], dp[2 * m][3]),
                                  pack_bf16x2(dp[2 * m + 1][0], dp[2 * m + 1][1]),
                                  pack_bf16x2(dp[2 * m + 1][2], dp[2 * m + 1][3])};
#pragma unroll
          for (int cp = 0; cp < NT / 2; ++cp) {
            const int c0 = ch0 / 8 + cp * 2;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(bt_addr<D>(g_t, lane, half * 32 + m * 16, c0), b0, b1, b2, b3);
            mma_bf16(dv[2 * cp], ap, b0, b1);
            mma_bf16(dv[2 * cp + 1], ap, b2, b3);
            ldsm_x4_t(bt_addr<D>(q_t, lane, half * 32 + m * 16, c0), b0, b1, b2, b3);
            mma_bf16(dk[2 * cp], ad, b0, b1);
            mma_bf16(dk[2 * cp + 1], ad, b2, b3);
          }
        }
      }
      __syncthreads();  // the stage and its metadata are read
    }
  }
  // rows g and g + 8 of this warp's 16 keys
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int j = key0 + warp * 16 + g + 8 * u;
    if (j >= k_len) continue;
    const long long row = pool_row(p, b, j, kvh);
    if (row < 0) continue;  // reported by the dQ kernel
    float* dkp = p.d_k + row + ch0 + 2 * c;
    float* dvp = p.d_v + row + ch0 + 2 * c;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      *reinterpret_cast<float2*>(dkp + n * 8) =
          make_float2(dk[n][2 * u] * p.scale, dk[n][2 * u + 1] * p.scale);
      *reinterpret_cast<float2*>(dvp + n * 8) = make_float2(dv[n][2 * u], dv[n][2 * u + 1]);
    }
  }
}

template <int D>
cudaError_t launch_d(const BackwardParams& p, cudaStream_t stream) {
  constexpr int TB = kRows * D * 2;
  constexpr int DC = D > 128 ? D / 2 : D;
  constexpr size_t dq_smem = 6 * (size_t)TB;
  constexpr size_t dkv_smem = 6 * (size_t)TB + 6 * kRows * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dkv_mma_kernel<D, DC>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dkv_smem);
  if (e != cudaSuccess) return e;
  // D of every row goes to the first T H floats of d_q, read by the dK / dV
  // kernel; the dQ kernel, launched after it, computes D of its own rows and
  // overwrites d_q.
  if (p.max_kv_len > 0) {
    float* delta = p.d_q;
    const long long rows = (long long)p.T * p.H;
    attn_bwd_delta_kernel<D><<<(unsigned)((rows * 8 + 255) / 256), 256, 0, stream>>>(p, delta);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const unsigned key_blocks = (unsigned)((p.max_kv_len + kKeys - 1) / kKeys);
    attn_bwd_dkv_mma_kernel<D, DC><<<dim3((unsigned)(p.Hk * (D / DC)), (unsigned)p.batch,
                                          key_blocks),
                                     kThreads, dkv_smem, stream>>>(p, delta);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int tpb = kRows / p.G;
  const unsigned row_blocks = (unsigned)max(1, (p.max_q_len + tpb - 1) / tpb);
  attn_bwd_dq_mma_kernel<D><<<dim3(row_blocks, (unsigned)p.batch, (unsigned)p.Hk), kThreads,
                              dq_smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool attn_backward_mma_supported(const BackwardParams& p, rpk_dtype dtype) {
  return dtype == RPK_BF16 && !p.cache_fp8 && p.G >= 1 && p.G <= 16 &&
         (p.d == 64 || p.d == 128 || p.d == 256);
}

cudaError_t launch_attn_backward_mma(const BackwardParams& p, cudaStream_t stream) {
  switch (p.d) {
    case 64: return launch_d<64>(p, stream);
    case 128: return launch_d<128>(p, stream);
    case 256: return launch_d<256>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpk

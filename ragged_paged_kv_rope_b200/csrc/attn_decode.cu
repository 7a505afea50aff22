// attn_decode.cu -- split-KV decode attention over the paged cache (bf16).
//
// For sequences with few new rows (q_len * group <= 16) attention is bound by
// reading K and V from HBM (about 4 FLOP per byte). The kernel streams each
// sequence's visible keys once per KV head:
//
//  * grid (split, kv_head, sequence). A split is a run of whole 64-key tiles
//    of the band [lo, k_len) (lo = start of the first row's window, or 0);
//    splits cut long contexts so that every SM streams a few hundred KB.
//  * warp 4 is the TMA producer: for each tile it loads the K and V rows of
//    this KV head from the pages named by the block table (3-D tensor map over
//    the pool [pages * page_size, n_kv_heads, head_dim], box of one head,
//    128-byte swizzle, no multicast) into a ring of shared-memory stages.
//  * warps 0-3 each own 16 keys of every tile and keep a private flash
//    online-softmax state (running max m, running sum l, unnormalised output
//    O; algenta "Attention variant kernels", flash_attention) for the <= 16
//    rows (token, query head of the group). Scores S = Q K^T and the update
//    O += P V use mma.sync m16n8k16 (bf16 in, fp32 accumulate): the contraction
//    is tiny next to the bytes, so the 16-row tile's idle rows cost nothing
//    that matters.
//  * at the end the four warps merge their states (the same rescale rule) and
//    the CTA writes either the final rows (one split) or an fp32 partial
//    (m, l, O) that attn_combine_kernel merges across splits. The combine
//    kernel is a programmatic dependent launch: it starts while the last
//    decode CTAs finish and waits (griddepcontrol.wait) before reading.
//
// Masking follows NumKong "Attention with a Pre-Packed KV-Cache": row r sits
// at p = r + k_len - q_len and sees [p - (window - 1), p]; masked keys are left
// out (score -inf, weight 0) and value rows past k_len are zeroed in shared
// memory before use so that stale or sentinel bytes never reach P V.
//
// An e4m3 cache (codes of x / scale, one scale per KV head for K and for V)
// halves the bytes per key. The stages then hold raw codes (no swizzle); each
// consumer warp widens its own 16 key rows of K and V to f16 (exact for every
// e4m3 value) into a private swizzled tile, releases the stage, and runs the
// same ldmatrix / mma.sync code in f16. Q is scaled by a power of two 2^-qs
// that brings its largest magnitude into [2^14, 2^15) before the f16
// narrowing; 2^qs and k_scale join the score scale, v_scale multiplies the
// merged output. P is f16 (values in [0, 1]). For head_dim >= 128 the raw
// stages are written with the 128-byte swizzle, only V is widened, and the
// score MMAs take K straight from the codes: lane (g, c) loads the four codes
// of channels 4c .. 4c+3 of each 16-channel step as the A operand's logical
// channels 2c, 2c+1, 2c+8, 2c+9, and Q's B operand uses the same order (a
// dot product does not depend on the order of its channels).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rpk {

namespace {
// Tiles of the longest band (one extra for a window start inside a tile).
int32_t band_tiles(int32_t max_kv_len) { return (max_kv_len + kDecodeTile - 1) / kDecodeTile + 1; }

int device_sm_count() {
  static int n[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    n[dev] = v;
  }
  return n[dev];
}
}  // namespace

DecodePlan decode_plan(int32_t max_kv_len) {
  const int32_t max_tiles = band_tiles(max_kv_len);
  int32_t tps = 8;  // 512 keys per split
  if ((max_tiles + tps - 1) / tps > kDecodeMaxSplits)
    tps = (max_tiles + kDecodeMaxSplits - 1) / kDecodeMaxSplits;
  DecodePlan plan;
  plan.tiles_per_split = tps;
  plan.max_splits = (max_tiles + tps - 1) / tps;
  return plan;
}

DecodePlan decode_launch_plan(int32_t max_kv_len, int32_t units, int32_t head_dim, int32_t window,
                              int32_t max_q_len, int32_t sinks, bool cache_fp8) {
  // Longer splits stream more bytes per CTA for the same start-up and merge,
  // but a launch needs enough CTAs to fill the GPU, and a last wave with few
  // CTAs cannot keep HBM busy. When every (sequence, KV head) unit fits in one
  // wave (two CTAs per SM for head_dim <= 128, one for 256), the splits fill
  // exactly one wave. Otherwise aim at two waves and keep splits between the
  // sizing plan's and 24 tiles (16 for head_dim 256; three times that for
  // e4m3 codes, whose tiles hold half the bytes). Then even out the splits
  // of the longest band.
  const DecodePlan most = decode_plan(max_kv_len);
  // Keys a sequence's rows can see: under a window at most window + max_q_len - 1
  // (plus the attention sinks' tiles), else all max_kv_len.
  long long band = max_kv_len;
  if (window > 0)
    band = std::min<long long>(band, (long long)window + std::max(0, max_q_len - 1) +
                                         (long long)(sinks + kDecodeTile - 1) / kDecodeTile *
                                             kDecodeTile);
  const int32_t max_tiles = band_tiles((int32_t)band);
  const long long wave = (long long)device_sm_count() * (head_dim <= 128 ? 2 : 1);
  const long long n_units = std::max(1, units);
  long long tps;
  if (n_units <= wave) {
    const long long per_unit = wave / n_units;
    tps = std::max<long long>((max_tiles + per_unit - 1) / per_unit, most.tiles_per_split);
  } else {
    const long long slots = 2 * wave;
    const long long per_unit = std::max(1LL, (slots + n_units - 1) / n_units);
    tps = (max_tiles + per_unit - 1) / per_unit;
    // e4m3 tiles are half the bytes: longer splits (three times the tiles
    // measured best on the Llama-3-8B and Gemma-like decodes)
    const int32_t cap = std::max((head_dim <= 128 ? 24 : 16) * (cache_fp8 ? 3 : 1),
                                 most.tiles_per_split);
    tps = std::min<long long>(std::max<long long>(tps, most.tiles_per_split), cap);
  }
  // at most 65535 splits (the grid's second dimension)
  tps = std::max<long long>(tps, (max_tiles + 65534) / 65535);
  const int32_t splits = (int32_t)((max_tiles + tps - 1) / tps);
  DecodePlan plan;
  plan.tiles_per_split = std::max(most.tiles_per_split, (max_tiles + splits - 1) / splits);
  plan.max_splits = (max_tiles + plan.tiles_per_split - 1) / plan.tiles_per_split;
  return plan;
}

size_t decode_workspace_bytes(int32_t total_q_tokens, int32_t n_heads, int32_t head_dim,
                              int32_t max_kv_len) {
  const DecodePlan plan = decode_plan(max_kv_len);
  const size_t rows = (size_t)plan.max_splits * total_q_tokens * n_heads;
  const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) & ~size_t(255);
  const size_t ml_bytes = (rows * sizeof(float2) + 255) & ~size_t(255);
  return o_bytes + ml_bytes;
}

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;

// Keys any row of the sequence sees, in whole tiles, and its splits: the
// attention-sink tiles [0, n_sink) (keys below the window's first key that
// stay visible), then the band's tiles from tile0 on. Tile v of this list is
// tile_at(v).
struct SeqSplit {
  int tile0;     // first tile of the band
  int n_sink;    // sink tiles, all below tile0
  int n_tiles;   // sink and band tiles
  int n_splits;  // >= 1
  __device__ __forceinline__ int tile_at(int v) const { return v < n_sink ? v : tile0 + (v - n_sink); }
};

__device__ __forceinline__ SeqSplit seq_split(int q_len, int k_len, int window, int sinks,
                                              int tps) {
  SeqSplit s;
  const int p0 = k_len - q_len;  // position of the first row
  const int lo = window > 0 ? max(0, p0 - window + 1) : 0;
  if (k_len <= 0 || lo >= k_len) {
    s.tile0 = 0; s.n_sink = 0; s.n_tiles = 0; s.n_splits = 1;
    return s;
  }
  s.tile0 = lo / kDecodeTile;
  const int sink_keys = min(sinks, lo);
  s.n_sink = min((sink_keys + kDecodeTile - 1) / kDecodeTile, s.tile0);
  s.n_tiles = s.n_sink + (k_len - 1) / kDecodeTile + 1 - s.tile0;
  s.n_splits = max(1, (s.n_tiles + tps - 1) / tps);
  return s;
}

// Transpose of an 8x8 matrix of 16-bit elements held one row pair per lane
// (lane t: row t / 4, columns 2 (t % 4), +1): lane t receives the same
// positions of the transposed matrix.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A(16x16 f16, row) * B(16x8 f16, col), fp32 accumulators.
__device__ __forceinline__ void mma_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D, bool kFp8 = false>
struct DecodeCfg {
  static constexpr int kBoxes = D / 64;                      // 128-byte column boxes per row
  static constexpr int kTileBytes = kDecodeTile * D * 2;     // one of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  // head_dim 256 runs one CTA per SM: three 64 KB stages keep two in flight
  static constexpr int kStages = D == 256 ? 3 : (D == 128 ? 3 : 6);
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024;  // + alignment slack
  static_assert(kConsumerWarps * 16 * D * 4 <= kStages * kStageBytes, "merge buffer");
};

// e4m3 cache: stages of raw codes [64 keys][D bytes] for K then V. head_dim
// >= 128 reads both straight from the codes; head_dim 64 widens its 16 rows of
// K and V into two f16 tiles (kBoxes 128-byte swizzled boxes) per consumer warp.
template <int D>
struct DecodeCfg<D, true> {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kDecodeTile * D;          // raw codes of K or V
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = D == 256 ? 6 : (D == 128 ? 4 : 8);
  static constexpr int kConvTileBytes = 16 * D * 2;           // 16 rows of f16
  static constexpr int kConvTiles = D >= 128 ? 0 : 2;         // K and V for head_dim 64
  static constexpr int kConvOff = kStages * kStageBytes;
  static constexpr int kSmemBytes =
      kConvOff + kConsumerWarps * kConvTiles * kConvTileBytes + 1024;
  static_assert(kConsumerWarps * 16 * D * 4 <= kSmemBytes - 1024, "merge buffer");
};

// Two CTAs share an SM when each warp holds at most 168 registers: ten warps
// put three on some sub-partition, whose register file is a quarter of the
// SM's (3 * 168 * 32 <= 16384). head_dim 256 runs one CTA per SM anyway.
template <int D, bool kFp8, int NT>
__global__ void __launch_bounds__(kThreads, 1) __maxnreg__(D <= 128 ? 168 : 255)
    attn_decode_kernel(const AttnParams p, const __grid_constant__ CUtensorMap k_map,
                       const __grid_constant__ CUtensorMap v_map, const DecodePlan plan,
                       const DecodeWorkspace ws) {
  using Cfg = DecodeCfg<D, kFp8>;
  constexpr int S = Cfg::kStages;
  // e4m3 with head_dim >= 128: K fragments straight from the swizzled raw codes
  constexpr bool kKDirect = kFp8 && D >= 128;
  // ... and V fragments too: each lane widens the codes of its A fragment's
  // 8x8 blocks in registers and transposes them with movmatrix.
  constexpr bool kVDirect = kKDirect;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[S], empty_bar[S];
  __shared__ float m_part[kConsumerWarps][kDecodeMaxRows];
  __shared__ float l_part[kConsumerWarps][kDecodeMaxRows];

  // e4m3 caches run a split-major grid: every first split launches before
  // any second one, so with their long splits the longest pieces of work
  // start first and the short remainders fill the last wave (measured 0.69
  // against 0.68 of HBM on the Llama-3-8B decode; with the shorter bf16
  // splits split-major measured slower, 0.979 against 0.987).
  int split, kvh, b;
  if constexpr (kFp8) {
    split = blockIdx.y;
    b = (int)(blockIdx.x / (unsigned)p.Hk);
    kvh = (int)(blockIdx.x - (unsigned)b * (unsigned)p.Hk);
  } else {
    split = blockIdx.x;
    kvh = blockIdx.y;
    b = blockIdx.z;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  if (q_len <= 0) return;
  if (q_len > p.max_q_len || q_len * p.G > kDecodeMaxRows || k_len < 0 || k_len > p.max_kv_len) {
    if (threadIdx.x == 0 && split == 0 && kvh == 0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
    return;
  }
  const SeqSplit ss = seq_split(q_len, k_len, p.window, p.sinks, plan.tiles_per_split);
  if (split >= ss.n_splits) return;
  const int v_begin = split * plan.tiles_per_split;  // first entry of this split's tile list
  const int n_tiles = max(0, min(plan.tiles_per_split, ss.n_tiles - v_begin));
  const int rows = q_len * p.G;

  // 1024-byte aligned stage ring (128-byte swizzle atoms are 8 rows x 128 bytes).
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  auto k_stage = [&](int s) { return smem + s * Cfg::kStageBytes; };
  auto v_stage = [&](int s) { return smem + s * Cfg::kStageBytes + Cfg::kTileBytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      const int box_rows = p.P < kDecodeTile ? p.P : kDecodeTile;
      // bf16: boxes of 64 channels (128 bytes) per row; e4m3: one box of D bytes per row.
      const uint32_t box_bytes = box_rows * 128u;
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % S;
        if (!mbar_wait(&empty_bar[s], ((i / S) & 1) ^ 1, p.wait_ns)) { ok = false; break; }
        const int key0 = ss.tile_at(v_begin + i) * kDecodeTile;
        // Count the boxes to load (pages wholly past k_len or invalid are skipped).
        uint32_t bytes = 0;
        for (int r = 0; r < kDecodeTile; r += box_rows) {
          const int key = key0 + r;
          if (key >= k_len) break;
          const int pi = key / p.P;
          const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
          if (page >= 0 && page < p.num_pages)
            bytes += kFp8 ? 2u * box_rows * D : 2u * Cfg::kBoxes * box_bytes;
        }
        mbar_arrive_expect_tx(&full_bar[s], bytes);
        for (int r = 0; r < kDecodeTile; r += box_rows) {
          const int key = key0 + r;
          if (key >= k_len) break;
          const int pi = key / p.P;
          const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
          if (page < 0 || page >= p.num_pages) {
            raise_error(p.error_word, RPK_DEVERR_PAGE);
            continue;
          }
          const int grow = page * p.P + (key - pi * p.P);
          if constexpr (kKDirect) {
#pragma unroll
            for (int bx = 0; bx < D / 128; ++bx) {
              tma_load_3d(k_stage(s) + bx * (kDecodeTile * 128) + r * 128, &k_map, bx * 128, kvh,
                          grow, &full_bar[s]);
              tma_load_3d(v_stage(s) + bx * (kDecodeTile * 128) + r * 128, &v_map, bx * 128, kvh,
                          grow, &full_bar[s]);
            }
          } else if constexpr (kFp8) {
            tma_load_3d(k_stage(s) + r * D, &k_map, 0, kvh, grow, &full_bar[s]);
            tma_load_3d(v_stage(s) + r * D, &v_map, 0, kvh, grow, &full_bar[s]);
          } else {
#pragma unroll
            for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
              tma_load_3d(k_stage(s) + bx * (kDecodeTile * 128) + r * 128, &k_map, bx * 64, kvh,
                          grow, &full_bar[s]);
              tma_load_3d(v_stage(s) + bx * (kDecodeTile * 128) + r * 128, &v_map, bx * 64, kvh,
                          grow, &full_bar[s]);
            }
          }
        }
        ++issued;
      }
      if (!ok) raise_error(p.error_word, RPK_DEVERR_TIMEOUT);
      // Never leave with copies in flight: wait for the last stages issued.
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait(&full_bar[i % S], (i / S) & 1);
    }
    return;
  }

  // ------------------------------------------------------------- consumers
  // Scores are computed transposed, S^T = K Q^T: this warp's 16 keys are the
  // MMA's M and the group's rows its N (8 per n-tile, NT n-tiles), so a group
  // of at most 8 rows fills one m16n8k16 per 16 channels. O^T = V^T P^T the
  // same way, P^T going from the score accumulators to the B operand through
  // an 8x8 transpose (movmatrix). Lane (g, c) = (lane / 4, lane % 4) holds
  // keys g and g + 8 of rows nt * 8 + 2c and 2c + 1.
  const int g = lane >> 2, c = lane & 3;
  int row_lo[NT][2], row_hi[NT][2];
  bool row_ok[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int rr = nt * 8 + 2 * c + j;
      row_ok[nt][j] = rr < rows;
      const int tok = rr / p.G;                 // token index in the sequence
      const int pos = tok + k_len - q_len;      // its position
      row_hi[nt][j] = pos;
      row_lo[nt][j] = p.window > 0 ? pos - p.window + 1 : 0;
    }

  // Q^T as the B operand: for channel step ks and n-tile nt, b0 = q[row][16ks + 2c, +1]
  // and b1 = q[row][16ks + 8 + 2c, +1] of row nt * 8 + g; rows past `rows` are zero.
  uint32_t qb[D / 16][NT][2];
  {
    const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(p.q);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int rr = nt * 8 + g;
      const __nv_bfloat16* qrow = nullptr;
      if (rr < rows) {
        const int t = q0 + rr / p.G;
        const int h = kvh * p.G + rr % p.G;
        qrow = qbase + ((size_t)t * p.H + h) * D;
      }
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t lo = 0, hi = 0;
        if (qrow) {
          // logical channels (2c, 2c+1) and (2c+8, 2c+9) of the step; with K
          // read straight from the codes they sit at 4c, 4c+1 and 4c+2, 4c+3
          const int c_lo = kKDirect ? 4 * c : 2 * c;
          const int c_hi = kKDirect ? 4 * c + 2 : 8 + 2 * c;
          lo = *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + c_lo);
          hi = *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + c_hi);
        }
        qb[ks][nt][0] = lo;
        qb[ks][nt][1] = hi;
      }
    }
  }
  float sl2 = p.scale_log2;   // score scale in log2 units
  float v_mul = 1.f;          // applied to the merged output
  if constexpr (kFp8) {
    // Largest |q| of the group's rows (every consumer warp holds all of them,
    // so every warp finds the same power of two).
    float mx = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&qb[ks][nt][k]);
          mx = fmaxf(mx, fmaxf(fabsf(__low2float(v2)), fabsf(__high2float(v2))));
        }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    int qs = 0;
    if (mx > 0.f && mx <= 3.0e38f) qs = min(64, max(-64, ilogbf(mx) - 14));
    const float down = __int_as_float((127 - qs) << 23);  // 2^-qs
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&qb[ks][nt][k]);
          qb[ks][nt][k] = pack_f16x2(__low2float(v2) * down, __high2float(v2) * down);
        }
    sl2 = p.scale_log2 * __ldg(p.k_scale + kvh) * __int_as_float((127 + qs) << 23);
    v_mul = __ldg(p.v_scale + kvh);
  }

  // O^T accumulators per 16-channel step and n-tile: (channel g, row 2c),
  // (g, 2c + 1), (g + 8, 2c), (g + 8, 2c + 1).
  float o[D / 16][NT][4];
#pragma unroll
  for (int dc = 0; dc < D / 16; ++dc)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[dc][nt][0] = o[dc][nt][1] = o[dc][nt][2] = o[dc][nt][3] = 0.f;
  float m_run[NT][2], l_run[NT][2];  // l_run: this lane's keys only, summed at the end
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -INFINITY;
      l_run[nt][j] = 0.f;
    }
  bool ok = true;

  for (int i = 0; i < n_tiles; ++i) {
    const int s = i % S;
    if (!mbar_wait(&full_bar[s], (i / S) & 1, p.wait_ns)) { ok = false; break; }
    const int key0 = ss.tile_at(v_begin + i) * kDecodeTile + warp * 16;  // this warp's 16 keys
    uint32_t kbase = smem_u32(k_stage(s));
    uint32_t vbase = smem_u32(v_stage(s));
    const int wrow0 = warp * 16;  // row of this warp's first key inside the tile
    constexpr int kBoxStride = (kFp8 ? 16 : kDecodeTile) * 128;  // bytes between 64-channel boxes
    const bool tail = key0 + 15 >= k_len;
    if constexpr (kFp8 && !kVDirect) {
      // Widen this warp's 16 rows of K and V from e4m3 codes to f16 in its own
      // tiles (value rows at or past k_len become zeros), then release the stage.
      uint8_t* ck = smem + Cfg::kConvOff + warp * Cfg::kConvTiles * Cfg::kConvTileBytes;
      uint8_t* cv = ck + Cfg::kConvTileBytes;
      constexpr int kChunks = D / 16;  // 16-code chunks per row
      // K, then V (one tile at a time keeps fewer registers live under the
      // 168-register cap; head_dim 256 runs one CTA per SM and unrolls both)
      constexpr int kUnrollKV = D == 256 ? 2 : 1;
#pragma unroll kUnrollKV
      for (int kv = kKDirect ? 1 : 0; kv < 2; ++kv) {
        const uint8_t* raw = kv ? v_stage(s) : k_stage(s);
        uint8_t* conv = kv ? cv : ck;
#pragma unroll
        for (int it = 0; it < (16 * kChunks) / 32; ++it) {
          const int idx = lane + 32 * it;
          const int kr = idx / kChunks;
          const int j = idx - kr * kChunks;
          // raw row: swizzled 128-byte boxes (kKDirect) or plain D-byte rows
          const uint8_t* src =
              kKDirect ? raw + (j >> 3) * (kDecodeTile * 128) + swz128(wrow0 + kr, j & 7)
                       : raw + (wrow0 + kr) * D + j * 16;
          uint4 r4 = *reinterpret_cast<const uint4*>(src);
          if (kv && key0 + kr >= k_len) r4 = make_uint4(0, 0, 0, 0);
          // f16 channels 16j .. 16j+7 and 16j+8 .. 16j+15 are the 16-byte
          // chunks 2j and 2j+1 of the row, in one 64-channel box. A 16-byte
          // store is served eight lanes at a time; for head_dim >= 128 those
          // eight lanes are chunks 0-7 of one row, whose first units fall on
          // four bank groups only, so odd groups of four store their second
          // unit first: eight distinct bank groups per store.
          const int sw = (j >> 2) & 1;
          uint4 a, b;  // a to chunk 2j + sw, b to chunk 2j + 1 - sw
          f16x4_from_e4m3x4(sw ? r4.z : r4.x, a.x, a.y);
          f16x4_from_e4m3x4(sw ? r4.w : r4.y, a.z, a.w);
          f16x4_from_e4m3x4(sw ? r4.x : r4.z, b.x, b.y);
          f16x4_from_e4m3x4(sw ? r4.y : r4.w, b.z, b.w);
          const int ch = 2 * j;
          uint8_t* row_box = conv + (ch >> 3) * kBoxStride;
          *reinterpret_cast<uint4*>(row_box + swz128(kr, (ch & 7) + sw)) = a;
          *reinterpret_cast<uint4*>(row_box + swz128(kr, (ch & 7) + 1 - sw)) = b;
        }
      }
      __syncwarp();
      if constexpr (!kKDirect) {
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        kbase = smem_u32(ck);
      }
      vbase = smem_u32(cv);
    } else if (!kFp8 && tail) {
      // Zero value rows at or past k_len (stale or never written bytes).
      for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
        const int kr = idx / (D / 8);
        if (key0 + kr < k_len) continue;
        const int ch = idx % (D / 8);
        uint8_t* dst = v_stage(s) + (ch >> 3) * (kDecodeTile * 128) + swz128(wrow0 + kr, ch & 7);
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    // S^T = K Q^T: A = this warp's 16 keys (rows) x 16 channels per step.
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    const int krow0 = kFp8 && !kKDirect ? 0 : wrow0;  // first key row in the K buffer read
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      if constexpr (kKDirect) {
        // codes of channels 4c .. 4c+3 of step ks, keys g and g + 8
        const uint8_t* kb = k_stage(s) + (ks >> 3) * (kDecodeTile * 128) + 4 * c;
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(kb + swz128(krow0 + g, ks & 7));
        const uint32_t w1 =
            *reinterpret_cast<const uint32_t*>(kb + swz128(krow0 + g + 8, ks & 7));
        a[0] = f16x2_from_e4m3x2(w0 & 0xFFFFu);
        a[2] = f16x2_from_e4m3x2(w0 >> 16);
        a[1] = f16x2_from_e4m3x2(w1 & 0xFFFFu);
        a[3] = f16x2_from_e4m3x2(w1 >> 16);
      } else {
        // matrices: (keys 0-7, d lo), (keys 8-15, d lo), (keys 0-7, d hi), (keys 8-15, d hi)
        const int mi = lane >> 3;
        const int krow = krow0 + (mi & 1) * 8 + (lane & 7);
        const int chunk = ks * 2 + (mi >> 1);
        const uint32_t addr = kbase + (chunk >> 3) * kBoxStride + swz128(krow, chunk & 7);
        ldsm_x4(addr, a[0], a[1], a[2], a[3]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if constexpr (kFp8) mma_f16(sc[nt], a, qb[ks][nt][0], qb[ks][nt][1]);
        else mma_bf16(sc[nt], a, qb[ks][nt][0], qb[ks][nt][1]);
      }
    }


    // Mask, scale to log2 units, online-softmax update of this lane's rows;
    // the 16 keys of a row sit on the 8 lanes that share c.
    float tmax[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) tmax[nt][j] = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = e & 1;
        const int key = key0 + g + (e >> 1) * 8;
        const bool vis = row_ok[nt][j] && key <= row_hi[nt][j] &&
                         (key >= row_lo[nt][j] || key < p.sinks);
        const float v = vis ? sc[nt][e] * sl2 : -INFINITY;
        sc[nt][e] = v;
        tmax[nt][j] = fmaxf(tmax[nt][j], v);
      }
    float alpha[NT][2], m_use[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float t = tmax[nt][j];
        t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
        t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
        t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
        const float m_new = fmaxf(m_run[nt][j], t);
        m_use[nt][j] = m_new == -INFINITY ? 0.f : m_new;
        alpha[nt][j] = fast_exp2(m_run[nt][j] - m_use[nt][j]);
        m_run[nt][j] = m_new;
      }
    uint32_t pb[NT][2];  // P^T as the B operand of O^T = V^T P^T
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = fast_exp2(sc[nt][e] - m_use[nt][e & 1]);
#pragma unroll
      for (int j = 0; j < 2; ++j) l_run[nt][j] = l_run[nt][j] * alpha[nt][j] + (w[j] + w[2 + j]);
      // P^T blocks (keys 0-7 and 8-15) x (rows 2c, 2c+1), transposed to rows x keys.
      uint32_t blk0, blk1;
      if constexpr (kFp8) {
        blk0 = pack_f16x2(w[0], w[1]);
        blk1 = pack_f16x2(w[2], w[3]);
      } else {
        blk0 = pack_bf16x2(w[0], w[1]);
        blk1 = pack_bf16x2(w[2], w[3]);
      }
      pb[nt][0] = movmatrix_trans(blk0);
      pb[nt][1] = movmatrix_trans(blk1);
    }
#pragma unroll
    for (int dc = 0; dc < D / 16; ++dc)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o[dc][nt][0] *= alpha[nt][0]; o[dc][nt][1] *= alpha[nt][1];
        o[dc][nt][2] *= alpha[nt][0]; o[dc][nt][3] *= alpha[nt][1];
      }

    // O^T += V^T P^T: A = V^T (16 channels x 16 keys).
#pragma unroll
    for (int dc = 0; dc < D / 16; ++dc) {
      uint32_t a[4];
      if constexpr (kVDirect) {
        // Codes of channels 16 dc + 4c .. 4c+3 of keys g and g + 8 (value
        // rows at or past k_len read as zeros): widened, they are the 8x8
        // blocks (keys 0-7 | 8-15) x (channel pairs lo | hi) in row layout;
        // movmatrix turns each into its transpose, a block of the A fragment.
        // Output row m of the step is channel 4 (m/2) + m%2 (m < 8) or
        // 4 ((m-8)/2) + 2 + m%2 (m >= 8) of the 16; the merge puts it back.
        const uint8_t* vb = v_stage(s) + (dc >> 3) * (kDecodeTile * 128) + 4 * c;
        uint32_t w0 = *reinterpret_cast<const uint32_t*>(vb + swz128(wrow0 + g, dc & 7));
        uint32_t w1 = *reinterpret_cast<const uint32_t*>(vb + swz128(wrow0 + g + 8, dc & 7));
        if (tail) {
          if (key0 + g >= k_len) w0 = 0u;
          if (key0 + g + 8 >= k_len) w1 = 0u;
        }
        uint32_t x0, x1, y0, y1;
        f16x4_from_e4m3x4(w0, x0, x1);
        f16x4_from_e4m3x4(w1, y0, y1);
        a[0] = movmatrix_trans(x0);  // channels lo, keys 0-7
        a[1] = movmatrix_trans(x1);  // channels hi, keys 0-7
        a[2] = movmatrix_trans(y0);  // channels lo, keys 8-15
        a[3] = movmatrix_trans(y1);  // channels hi, keys 8-15
      } else {
        // by a transposing load; matrices (transposed): (keys 0-7, d lo),
        // (keys 0-7, d hi), (keys 8-15, d lo), (keys 8-15, d hi)
        const int mi = lane >> 3;
        const int vrow = (kFp8 ? 0 : wrow0) + (mi >> 1) * 8 + (lane & 7);
        const int chunk = dc * 2 + (mi & 1);
        const uint32_t addr = vbase + (chunk >> 3) * kBoxStride + swz128(vrow, chunk & 7);
        ldsm_x4_t(addr, a[0], a[1], a[2], a[3]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if constexpr (kFp8) mma_f16(o[dc][nt], a, pb[nt][0], pb[nt][1]);
        else mma_bf16(o[dc][nt], a, pb[nt][0], pb[nt][1]);
      }
    }

    __syncwarp();
    if constexpr (!kFp8 || kVDirect) {
      if constexpr (!kFp8) {
        if (tail) fence_proxy_async_smem();  // generic zero-writes before the next TMA into s
      }
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
  }
  if (!ok) raise_error(p.error_word, RPK_DEVERR_TIMEOUT);
  // Let the combine kernel launch now (it waits for this grid's completion
  // before reading any partial, so this only moves its launch earlier).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ----------------------------------------------- merge the four warps' states
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][j] = l;
    }
  if (g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m_part[warp][nt * 8 + 2 * c + j] = m_run[nt][j];
        l_part[warp][nt * 8 + 2 * c + j] = l_run[nt][j];
      }
  }
  // All consumers are past the tile loop, so every stage's TMA has landed and
  // the ring can be reused as the merge buffer.
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  float* obuf = reinterpret_cast<float*>(smem);  // [warp][16][D]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int rr = nt * 8 + 2 * c + j;
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, m_part[w][rr]);
      const float f = m_run[nt][j] == -INFINITY ? 0.f : fast_exp2(m_run[nt][j] - mx);
      // output rows g and g + 8 of each 16-channel step: channels g and g + 8,
      // or, with V read from the codes, 4 (g/2) + g%2 and that + 2
      const int ch_lo = kVDirect ? 4 * (g >> 1) + (g & 1) : g;
      const int ch_hi = kVDirect ? ch_lo + 2 : g + 8;
      float* orow = obuf + ((size_t)warp * 16 + rr) * D;
#pragma unroll
      for (int dc = 0; dc < D / 16; ++dc) {
        orow[dc * 16 + ch_lo] = o[dc][nt][j] * f;
        orow[dc * 16 + ch_hi] = o[dc][nt][2 + j] * f;
      }
    }
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

  const bool single = ss.n_splits == 1;
  for (int idx = threadIdx.x; idx < rows * (D / 4); idx += kConsumerWarps * 32) {
    const int rr = idx / (D / 4);
    const int e4 = (idx - rr * (D / 4)) * 4;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) mx = fmaxf(mx, m_part[w][rr]);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = m_part[w][rr];
      const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - mx);
      L += l_part[w][rr] * f;
      const float4 v = *reinterpret_cast<const float4*>(obuf + ((size_t)w * 16 + rr) * D + e4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    acc.x *= v_mul; acc.y *= v_mul; acc.z *= v_mul; acc.w *= v_mul;
    const int t = q0 + rr / p.G;
    const int h = kvh * p.G + rr % p.G;
    const size_t orow = (size_t)t * p.H + h;
    if (single) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + orow * D + e4;
      uint2 pk;
      pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(out) = pk;
      if (p.lse != nullptr && e4 == 0) p.lse[orow] = lse_from_log2_state(mx, L);
    } else {
      const size_t prow = (size_t)split * p.T * p.H + orow;
      *reinterpret_cast<float4*>(ws.o + prow * D + e4) = acc;
      if (e4 == 0) ws.ml[prow] = make_float2(mx, L);
    }
  }
}

// Merge the split partials of each (token, head) row: m* = max m_s,
// out = sum_s 2^(m_s - m*) O_s / sum_s 2^(m_s - m*) l_s (zero when empty), and
// the row's log-sum-exp from (m*, sum_s 2^(m_s - m*) l_s) when asked for.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const AttnParams p,
                                                           const DecodePlan plan,
                                                           const DecodeWorkspace ws) {
  constexpr int E = D / 32;
  // Launched as a programmatic dependent of the decode kernel: wait until that
  // grid has completed and its partials are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (long long)p.T * p.H) return;
  const int t = (int)(row / p.H);
  const int b = find_sequence(p.offsets, p.batch, t);
  const int q_len = __ldg(p.offsets + b + 1) - __ldg(p.offsets + b);
  const int k_len = __ldg(p.kv_lens + b);
  if (q_len > p.max_q_len || q_len * p.G > kDecodeMaxRows || k_len < 0 || k_len > p.max_kv_len)
    return;
  const SeqSplit ss = seq_split(q_len, k_len, p.window, p.sinks, plan.tiles_per_split);
  if (ss.n_splits <= 1) return;  // the decode kernel wrote this row itself
  const size_t stride = (size_t)p.T * p.H;
  float mx = -INFINITY;
  for (int s = 0; s < ss.n_splits; ++s) mx = fmaxf(mx, ws.ml[s * stride + row].x);
  float L = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < ss.n_splits; ++s) {
    const float2 ml = ws.ml[s * stride + row];
    const float f = ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - mx);
    L += ml.y * f;
    const float* src = ws.o + (s * stride + row) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      const float4 v = *reinterpret_cast<const float4*>(src + e);
      acc[e] += f * v.x; acc[e + 1] += f * v.y; acc[e + 2] += f * v.z; acc[e + 3] += f * v.w;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (p.lse != nullptr && lane == 0) p.lse[row] = lse_from_log2_state(mx, L);
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(out + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
}

template <int D, bool kFp8>
cudaError_t launch_d(const AttnParams& p, const CUtensorMap& k_map, const CUtensorMap& v_map,
                     const DecodePlan& plan, const DecodeWorkspace& ws, cudaStream_t stream) {
  using Cfg = DecodeCfg<D, kFp8>;
  // One n-tile of 8 rows when the group's rows fit, else two.
  auto kernel = p.max_q_len * p.G <= 8 ? attn_decode_kernel<D, kFp8, 1>
                                       : attn_decode_kernel<D, kFp8, 2>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (kFp8 && ((long long)p.Hk * p.batch > INT32_MAX || plan.max_splits > 65535))
    return cudaErrorInvalidValue;
  const dim3 grid = kFp8 ? dim3((unsigned)(p.Hk * p.batch), (unsigned)plan.max_splits)
                         : dim3((unsigned)plan.max_splits, p.Hk, p.batch);
  kernel<<<grid, kThreads, Cfg::kSmemBytes, stream>>>(p, k_map, v_map, plan, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (plan.max_splits > 1) {
    const long long rows = (long long)p.T * p.H;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((rows + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_combine_kernel<D>, p, plan, ws);
  }
  return e;
}

}  // namespace

cudaError_t launch_attn_decode(const AttnParams& p, const CUtensorMap& k_map,
                               const CUtensorMap& v_map, const DecodePlan& plan,
                               const DecodeWorkspace& ws, cudaStream_t stream) {
  if ((long long)p.T * p.H == 0 || p.batch == 0) return cudaSuccess;
  if (p.cache_fp8) {
    switch (p.d) {
      case 64: return launch_d<64, true>(p, k_map, v_map, plan, ws, stream);
      case 128: return launch_d<128, true>(p, k_map, v_map, plan, ws, stream);
      case 256: return launch_d<256, true>(p, k_map, v_map, plan, ws, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.d) {
    case 64: return launch_d<64, false>(p, k_map, v_map, plan, ws, stream);
    case 128: return launch_d<128, false>(p, k_map, v_map, plan, ws, stream);
    case 256: return launch_d<256, false>(p, k_map, v_map, plan, ws, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpk

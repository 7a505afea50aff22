// attn_backward_tc.cu -- gradients of ragged paged causal GQA attention on the
// 5th-generation tensor cores (tcgen05): bf16 tensors over a bf16 cache,
// head_dim 64 or 128, groups of up to 64 query heads per KV head.
//
// The gradients of NumKong "Attention with a Pre-Packed KV-Cache"
// (attention_packed_gradients): with s_ij = scale q_i.k_j,
// P_ij = e^(s_ij - lse_i), dP_ij = dO_i.v_j, D_i = dO_i.O_i and
// dS_ij = P_ij (dP_ij - D_i),
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO,
// each a sum over the (row, key) pairs of the forward's band (window, sinks).
// Query rows are packed as in the forward: the rows of a row block are the
// (token, query head) pairs of one KV head's group, token-major.
//
// Three launches, no atomics (every output element has one writer), so results
// are deterministic:
//   D    D_i of every row into the first T H floats of d_q (read by dK/dV; the
//        dQ kernel computes D of its own rows and then overwrites d_q).
//   dKV  one CTA per 128-key block of one (sequence, KV head), launched as a
//        programmatic dependent of D (its loader warp waits for D; the other
//        warps start loading and multiplying at once). K and V stay in
//        shared memory; the 64-row blocks that see the keys stream through a
//        four-stage ring (Q and dO by TMA, -lse log2 e and -D by a loader warp).
//        Per row block j the tensor core computes S^T_j = K Q_j^T and
//        dP^T_j = V dO_j^T (128 keys x 64 rows each, fp32) into one of two
//        tensor-memory buffers, so the next block's scores are computed while
//        eight compute warps (thread = key, two warps per key quarter
//        splitting the rows) turn this block's into P^T_j and dS^T_j (bf16,
//        written back over the first half of each warp's own columns); then
//        dV += P^T_j dO_j and dK += dS^T_j Q_j with P^T / dS^T read from
//        tensor memory.
//   dQ   one CTA per 128-row block, launched as a programmatic dependent of
//        dK/dV (it waits for that grid only before storing, since d_q holds
//        D until then). Q and dO stay in shared memory; the key
//        blocks of the rows' band stream through rings of K (three deep) and
//        V (two deep). Per key block i: S_i = Q K_i^T and dP_i = dO V_i^T
//        (128 x 128, fp32); the compute warps (thread = row) load them and
//        release them at once, so the tensor core computes S_{i+1} and
//        dP_{i+1} while they form dS_i (bf16) in a tensor-memory region of
//        its own; then dQ += dS_i K_i.
// Tensor memory (512 columns), dK/dV: [S^T_0 | dP^T_0 | S^T_1 | dP^T_1] (64
// columns each) | dV | dK; dQ: S | dP | dQ | dS (64 columns of bf16 pairs).
// Operands that belong to no row or key (rows past the block's tokens, keys
// past kv_len) are excluded by selection, not multiplication, and shared-memory
// rows that no copy writes are zeroed, so sentinel NaNs never reach a product.
// Every mbarrier wait is bounded (as in the forward kernels); tcgen05.ld / st
// are warp-collective, so every lane of a warp issues them.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace rpk {
namespace {

constexpr int kThreads = 384;
constexpr int kRegsControl = 56;
constexpr int kRegsCompute = 224;
constexpr uint32_t kTmemCols = 512;
constexpr int kGroup = 8;        // blocks of one (sequence, KV head) scheduled together
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTile128 = 128 * D * 2;     // one [128][D] bf16 tile
  static constexpr int kTile64 = 64 * D * 2;       // one [64][D] bf16 tile
};

// Loads the rows [key0, key0 + 128) of one KV head from the paged pool into a
// [boxes][128][64] tile with TMA; returns the bytes that will arrive (segments
// past k_len or on an invalid page are skipped; an invalid page raises
// RPK_DEVERR_PAGE when `report`).
template <int D>
__device__ __forceinline__ uint32_t load_keys(const BackwardParams& p, const CUtensorMap* map,
                                              uint8_t* dst, int b, int kvh, int key0, int k_len,
                                              uint64_t* bar, bool issue, bool report) {
  const int box_rows = p.P < 128 ? p.P : 128;
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
  uint32_t bytes = 0;
  for (int r = 0; r < 128; r += box_rows) {
    const int key = key0 + r;
    if (key >= k_len) break;
    const int pi = key / p.P;
    const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
    if (page < 0 || page >= p.num_pages) {
      if (report) raise_error(p.error_word, RPK_DEVERR_PAGE);
      continue;
    }
    bytes += (uint32_t)box_rows * 128u * BwdCfg<D>::kBoxes;
    if (issue) {
      const int grow = page * p.P + (key - pi * p.P);
#pragma unroll
      for (int bx = 0; bx < BwdCfg<D>::kBoxes; ++bx)
        tma_load_3d(dst + bx * (128 * 128) + r * 128, map, bx * 64, kvh, grow, bar);
    }
  }
  return bytes;
}

// Zero rows [r0, rows) of a [boxes][rows][64] bf16 tile (all lanes of a warp).
template <int D>
__device__ __forceinline__ void zero_rows(uint8_t* tile, int rows, int r0, int lane) {
  const int chunks = (rows - r0) * BwdCfg<D>::kBoxes * 8;
  for (int idx = lane; idx < chunks; idx += 32) {
    const int ch = idx & 7;
    const int rb = idx >> 3;
    const int bx = rb % BwdCfg<D>::kBoxes;
    const int r = r0 + rb / BwdCfg<D>::kBoxes;
    *reinterpret_cast<uint4*>(tile + bx * (rows * 128) + r * 128 + ch * 16) =
        make_uint4(0, 0, 0, 0);
  }
}

// Sequence b's lengths; false (and RPK_DEVERR_LENGTH once) when out of bounds.
__device__ __forceinline__ bool seq_lengths(const BackwardParams& p, int b, bool report, int& q0,
                                            int& q_len, int& k_len) {
  q0 = __ldg(p.offsets + b);
  q_len = __ldg(p.offsets + b + 1) - q0;
  k_len = __ldg(p.kv_lens + b);
  if (k_len < 0 || k_len > p.max_kv_len || q_len < 0 || q_len > p.max_q_len) {
    if (report) raise_error(p.error_word, RPK_DEVERR_LENGTH);
    return false;
  }
  return true;
}

// 16 fp32 values -> 8 bf16x2 words.
__device__ __forceinline__ void bf16_pack8(uint32_t* out, const float* a) {
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = pack_bf16x2(a[2 * i], a[2 * i + 1]);
}

// ------------------------------------------------------------------- D

template <int D>
__global__ void __launch_bounds__(256) attn_bwd_tc_delta_kernel(const BackwardParams p,
                                                                float* __restrict__ delta) {
  // the dK / dV grid may start at once; it reads D only after this grid completes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long row = ((long long)blockIdx.x * 256 + threadIdx.x) >> 3;
  const bool ok = row < (long long)p.T * p.H;
  const int part = threadIdx.x & 7;
  float acc = 0.f;
  if (ok) {
    const uint4* g = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.d_out) +
                                                    (size_t)row * D);
    const uint4* o = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) +
                                                    (size_t)row * D);
    for (int c = part; c < D / 8; c += 8) {
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
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (ok && part == 0) delta[row] = acc;
}

// ------------------------------------------------------------------ dK / dV

constexpr int kDkvRows = 64;     // packed rows per row block
constexpr int kDkvStages = 4;    // Q / dO ring depth

struct DkvBars {
  uint64_t kv_full;                // K and V of the key block loaded
  uint64_t full[kDkvStages];       // per stage: Q_j, dO_j loaded and -lse, -D written
  uint64_t empty[kDkvStages];      // per stage: the MMAs reading it have completed
  uint64_t sd_full[2];             // per buffer: S^T_j and dP^T_j computed
  uint64_t pd_full[2];             // per buffer: P^T_j and dS^T_j written (per compute warp)
  uint64_t acc_full;               // dV and dK complete
  uint64_t drain;
};

// TMEM column (within a 64-column buffer) of the 16-row K step kk of a 64-row
// bf16 operand written by two warps, each over the first half of its own 32
// fp32 columns.
__device__ __forceinline__ uint32_t dkv_a_col(int kk) { return (uint32_t)(kk * 8 + (kk >= 2 ? 16 : 0)); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkv_tc_kernel(const BackwardParams p, const __grid_constant__ CUtensorMap q_map,
                           const __grid_constant__ CUtensorMap do_map,
                           const __grid_constant__ CUtensorMap k_map,
                           const __grid_constant__ CUtensorMap v_map,
                           const float* __restrict__ delta, const int n_kb) {
  using C = BwdCfg<D>;
  constexpr int R = kDkvRows;
  constexpr int S = kDkvStages;
  constexpr int kStageBytes = 2 * C::kTile64 + 1024;   // Q_j, dO_j, metadata (1 KB aligned)
  constexpr int kStageOff = 2 * C::kTile128;           // after K and V
  // buffers b: S^T at b * 128, dP^T at b * 128 + 64; then dV, dK
  constexpr uint32_t kVCol = 256, kKCol = 256 + D;
  static_assert(kKCol + D <= kTmemCols, "TMEM budget");
  extern __shared__ uint8_t smem_raw[];
  __shared__ DkvBars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, tpr = R / G, rows_used = tpr * G;
  // Block order: groups of kGroup key blocks of one (sequence, KV head), the
  // groups of the first key blocks (which the most rows see) first.
  const int units = p.batch * p.Hk;
  const int per_group = units * kGroup;
  const int gidx = (int)blockIdx.x / per_group;
  const int rem = (int)blockIdx.x - gidx * per_group;
  const int unit = rem / kGroup;
  const int kb = gidx * kGroup + rem % kGroup;
  const int b = unit / p.Hk, kvh = unit - (unit / p.Hk) * p.Hk;
  int q0, q_len, k_len;
  const bool have_seq =
      kb < n_kb && seq_lengths(p, b, threadIdx.x == 0 && kvh == 0 && kb == 0, q0, q_len, k_len);
  const int key0 = kb * 128;
  if (!have_seq || key0 >= k_len) {
    // Block 0 always waits for the D grid, so that this grid's completion
    // (which the dQ grid waits for before overwriting D) implies D's.
    if (blockIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int key_hi = min(key0 + 128, k_len) - 1;
  const int off = k_len - q_len;  // row (token) i sits at position i + off
  // Tokens that see a key of the block: position >= key0, and under a window
  // (unless the block holds attention sinks) position <= key_hi + window - 1.
  const int i_lo = max(0, key0 - off);
  int i_hi = q_len - 1;
  if (p.window > 0 && key0 >= p.sinks) i_hi = min(i_hi, key_hi + p.window - 1 - off);
  const int j_lo = i_lo / tpr;
  const int n_rb = i_lo <= i_hi ? i_hi / tpr - j_lo + 1 : 0;

  // The dQ grid may start on SMs this grid's last CTAs leave idle; it waits
  // for this grid's completion before its first store (griddepcontrol.wait).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  auto stage_ptr = [&](int s) { return smem + kStageOff + s * kStageBytes; };
  auto meta_ptr = [&](int s) { return reinterpret_cast<float*>(stage_ptr(s) + 2 * C::kTile64); };

  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bars.full[s], 1 + 32);  // producer's expect_tx + the loader warp's lanes
      mbar_init(&bars.empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bars.sd_full[k], 1);
      mbar_init(&bars.pd_full[k], 8);
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 3 && rows_used < R) {
    // rows of the Q and dO tiles that no copy writes (the group does not divide 64)
    for (int s = 0; s < S; ++s) {
      zero_rows<D>(stage_ptr(s), R, rows_used, lane);
      zero_rows<D>(stage_ptr(s) + C::kTile64, R, rows_used, lane);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0 && n_rb > 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&do_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      const uint32_t kbytes = load_keys<D>(p, &k_map, smem, b, kvh, key0, k_len, &bars.kv_full,
                                           false, false);
      mbar_arrive_expect_tx(&bars.kv_full, 2 * kbytes);
      load_keys<D>(p, &k_map, smem, b, kvh, key0, k_len, &bars.kv_full, true, true);
      load_keys<D>(p, &v_map, smem + C::kTile128, b, kvh, key0, k_len, &bars.kv_full, true,
                   false);
      const uint32_t q_bytes = 2u * C::kBoxes * 128u * (uint32_t)rows_used;
      int j = 0;
      bool ok = true;
      for (; j < n_rb; ++j) {
        const int s = j % S;
        if (j >= S &&
            !thread_wait(&bars.empty[s], ((j / S) & 1) ^ 1, abort, p.error_word, p.wait_ns)) {
          ok = false;
          break;
        }
        const int tok0 = (j_lo + j) * tpr;
        mbar_arrive_expect_tx(&bars.full[s], q_bytes);
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          tma_load_3d(stage_ptr(s) + bx * (R * 128), &q_map, bx * 64, kvh * G, q0 + tok0,
                      &bars.full[s]);
          tma_load_3d(stage_ptr(s) + C::kTile64 + bx * (R * 128), &do_map, bx * 64, kvh * G,
                      q0 + tok0, &bars.full[s]);
        }
      }
      if (!ok) do_abort(abort, p.error_word);
      // Never leave with copies in flight.
      mbar_wait(&bars.kv_full, 0);
      for (int jj = max(0, j - S); jj < j; ++jj) mbar_wait(&bars.full[jj % S], (jj / S) & 1);
    }
  } else if (warp == 2) {
    // --------------------------------------- loader: -lse log2 e and -D per row
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    // D comes from the D grid, of which this grid is a programmatic dependent
    asm volatile("griddepcontrol.wait;" ::: "memory");
    bool ok = true;
    for (int j = 0; j < n_rb && ok; ++j) {
      const int s = j % S;
      if (j >= S &&
          !warp_wait(&bars.empty[s], ((j / S) & 1) ^ 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      const int tok0 = (j_lo + j) * tpr;
      float* meta = meta_ptr(s);
      for (int r = lane; r < R; r += 32) {
        const int tok = tok0 + r / G;
        const bool valid = r < rows_used && tok < q_len;
        const size_t row = (size_t)(q0 + tok) * p.H + (size_t)kvh * G + (r % G);
        meta[r] = valid ? -__ldg(p.lse + row) * kLog2e : 0.f;
        meta[R + r] = valid ? -__ldg(delta + row) : 0.f;
      }
      mbar_arrive(&bars.full[s]);  // release: this lane's writes before the consumers' reads
    }
    if (!ok) do_abort(abort, p.error_word);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, R, 0);    // 128 keys x 64 rows
    constexpr uint32_t idesc_acc = tc::idesc_bf16_f32(128, D, 1);  // 128 keys x D, B MN-major
    const uint64_t kdesc = tc::smem_desc_sw128(sbase, 16, 1024);
    const uint32_t k_lo = (uint32_t)kdesc, desc_hi = (uint32_t)(kdesc >> 32);
    const uint32_t v_lo = (uint32_t)tc::smem_desc_sw128(sbase + C::kTile128, 16, 1024);
    const uint32_t st_lo = (uint32_t)tc::smem_desc_sw128(sbase + kStageOff, 16, 1024);
    const uint32_t st_mn_lo = (uint32_t)tc::smem_desc_sw128(sbase + kStageOff, R * 128, 1024);
    bool ok = true;
    auto commit_to = [&](uint64_t* bar) {
      if (lane == 0) tc::commit(smem_u32(bar));
      __syncwarp();
    };
    // S^T_j = K Q_j^T and dP^T_j = V dO_j^T into buffer j & 1
    auto issue_s = [&](int j) -> bool {
      const int s = j % S;
      if (!warp_wait(&bars.full[s], (j / S) & 1, abort, p.error_word, p.wait_ns)) return false;
      tc::fence_after_sync();
      const uint32_t so = (uint32_t)((s * kStageBytes) >> 4);
      const uint32_t buf = tmem + (uint32_t)((j & 1) * 128);
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (uint32_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
          const uint32_t qo = (uint32_t)(((kk >> 2) * (R * 128) + (kk & 3) * 32) >> 4);
          tc::mma_ss_lo(buf, k_lo + ko, st_lo + so + qo, desc_hi, idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (uint32_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
          const uint32_t qo = (uint32_t)(((kk >> 2) * (R * 128) + (kk & 3) * 32) >> 4);
          tc::mma_ss_lo(buf + 64, v_lo + ko, st_lo + so + (C::kTile64 >> 4) + qo, desc_hi,
                        idesc_s, kk > 0);
        }
        tc::commit(smem_u32(&bars.sd_full[j & 1]));
      }
      __syncwarp();
      return true;
    };
    if (n_rb > 0) ok = warp_wait(&bars.kv_full, 0, abort, p.error_word, p.wait_ns);
    for (int j = 0; ok && j < n_rb && j < 2; ++j) ok = issue_s(j);
    for (int j = 0; ok && j < n_rb; ++j) {
      const int s = j % S;
      if (!warp_wait(&bars.pd_full[j & 1], (j >> 1) & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t so = (uint32_t)((s * kStageBytes) >> 4);
      const uint32_t buf = tmem + (uint32_t)((j & 1) * 128);
      if (lane == 0) {
        // dV += P^T_j dO_j and dK += dS^T_j Q_j: A from tensor memory (keys x
        // rows, 16 rows per step), B = dO_j / Q_j read MN-major (rows x d)
#pragma unroll
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint32_t bo = so + (uint32_t)((kk * 16 * 128) >> 4);
          tc::mma_ts_lo(tmem + kVCol, buf + dkv_a_col(kk), st_mn_lo + bo + (C::kTile64 >> 4),
                        desc_hi, idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
          tc::mma_ts_lo(tmem + kKCol, buf + 64 + dkv_a_col(kk), st_mn_lo + bo, desc_hi,
                        idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc::commit(smem_u32(&bars.empty[s]));
      }
      __syncwarp();
      // the next block of this buffer: issued after the MMAs that read P^T_j
      if (j + 2 < n_rb) ok = issue_s(j + 2);
    }
    if (ok && n_rb > 0) commit_to(&bars.acc_full);
    if (!ok) do_abort(abort, p.error_word);
    commit_to(&bars.drain);
    if (!warp_wait(&bars.drain, 0, abort, p.error_word, p.wait_ns)) mbar_wait(&bars.drain, 0);
  } else if (warp == 3) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  } else {
    // -------------------------------------------------------- compute warps
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    const int qw = warp & 3;               // key quarter (TMEM lanes)
    const int hh = (warp - 4) >> 2;        // row half of every block (32 rows)
    const int kr = qw * 32 + lane;         // key row of this thread
    const int key = key0 + kr;
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    const float sl2 = p.scale * kLog2e;
    const bool key_ok = key < k_len;
    const bool sink = p.window > 0 && key < p.sinks;
    bool ok = true;
    for (int j = 0; j < n_rb; ++j) {
      if (!warp_wait(&bars.sd_full[j & 1], (j >> 1) & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t s_addr = tmem + lane_base + (uint32_t)((j & 1) * 128 + hh * 32);
      const uint32_t p_addr = s_addr + 64;
      float sv[32], dv[32];
      tc::tmem_ld32(s_addr, sv);
      tc::tmem_ld32(p_addr, dv);
      tc::tmem_wait_ld();
      // rows [r_lo, r_hi] of this block see this key
      const int tok0 = (j_lo + j) * tpr;
      const int a = key - off - tok0;  // token index (in the block) at the key's position
      const int r_lo = max(0, G * a);
      int r_hi = min(rows_used, G * (q_len - tok0)) - 1;
      if (p.window > 0 && !sink) r_hi = min(r_hi, G * (a + p.window) - 1);
      if (!key_ok) r_hi = -1;
      const int c_lo = r_lo - hh * 32, c_hi = r_hi - hh * 32;  // this warp's columns
      const bool full = c_lo <= 0 && c_hi >= 31;
      const float* meta = meta_ptr(j % S) + hh * 32;
      float pv[32], ds[32];
#pragma unroll
      for (int c4 = 0; c4 < 32; c4 += 4) {
        const float4 nl = *reinterpret_cast<const float4*>(meta + c4);
        const float4 nd = *reinterpret_cast<const float4*>(meta + R + c4);
        float x0, x1, x2, x3, t0, t1, t2, t3;
        fma2_v(x0, x1, sv[c4], sv[c4 + 1], sl2, sl2, nl.x, nl.y);
        fma2_v(x2, x3, sv[c4 + 2], sv[c4 + 3], sl2, sl2, nl.z, nl.w);
        pv[c4] = fast_exp2(x0);
        pv[c4 + 1] = fast_exp2(x1);
        pv[c4 + 2] = fast_exp2(x2);
        pv[c4 + 3] = fast_exp2(x3);
        add2_to(t0, t1, dv[c4], dv[c4 + 1], nd.x, nd.y);
        add2_to(t2, t3, dv[c4 + 2], dv[c4 + 3], nd.z, nd.w);
        mul2(ds[c4], ds[c4 + 1], pv[c4], pv[c4 + 1], t0, t1);
        mul2(ds[c4 + 2], ds[c4 + 3], pv[c4 + 2], pv[c4 + 3], t2, t3);
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < c_lo || c > c_hi) pv[c] = ds[c] = 0.f;
      }
      uint32_t pk[16];
      bf16_pack8(pk, pv);
      bf16_pack8(pk + 8, pv + 16);
      tc::tmem_st16(s_addr, pk);
      bf16_pack8(pk, ds);
      bf16_pack8(pk + 8, ds + 16);
      tc::tmem_st16(p_addr, pk);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.pd_full[j & 1]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n_rb > 0) ok = warp_wait(&bars.acc_full, 0, abort, p.error_word, p.wait_ns);
    if (!ok) {
      tc::tmem_wait_st();
      do_abort(abort, p.error_word);
    } else {
      // every lane loads (tcgen05.ld is warp-collective); keys below k_len on
      // a valid page are stored
      const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
      const int pi = key_ok ? key / p.P : 0;
      const int page = key_ok && pi < p.max_pages ? __ldg(bt + pi) : -1;
      const bool page_ok = key_ok && page >= 0 && page < p.num_pages;
      const size_t base = ((size_t)(page_ok ? page : 0) * p.P + (key - pi * p.P)) * p.Hk + kvh;
      float* dk = p.d_k + base * D + hh * (D / 2);
      float* dvp = p.d_v + base * D + hh * (D / 2);
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < D / 2; c += 32) {
        float vv[32], kv[32];
        if (n_rb > 0) {
          tc::tmem_ld32(tmem + lane_base + kVCol + hh * (D / 2) + c, vv);
          tc::tmem_ld32(tmem + lane_base + kKCol + hh * (D / 2) + c, kv);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) vv[e] = kv[e] = 0.f;
        }
        if (page_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            *reinterpret_cast<float4*>(dvp + c + e) = make_float4(vv[e], vv[e + 1], vv[e + 2],
                                                                  vv[e + 3]);
            *reinterpret_cast<float4*>(dk + c + e) =
                make_float4(kv[e] * p.scale, kv[e + 1] * p.scale, kv[e + 2] * p.scale,
                            kv[e + 3] * p.scale);
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------------- dQ

constexpr int kDqKStages = 3;    // K ring depth
constexpr int kDqVStages = 2;    // V ring depth

struct DqBars {
  uint64_t q_full;                 // Q_i and dO_i loaded
  uint64_t k_full[kDqKStages];     // per K stage: K of a key block loaded
  uint64_t k_empty[kDqKStages];    // per K stage: S and dQ MMAs reading it have completed
  uint64_t v_full[kDqVStages];     // per V stage: V of a key block loaded
  uint64_t v_empty[kDqVStages];    // per V stage: the dP MMAs reading it have completed
  uint64_t sd_full;                // S_i and dP_i computed
  uint64_t sd_free;                // S_i and dP_i read out by every compute warp
  uint64_t ds_full;                // dS_i written (one arrival per compute warp)
  uint64_t dq_done;                // dQ += dS_i K_i completed (dS may be overwritten)
  uint64_t acc_full;               // dQ complete
  uint64_t drain;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_tc_kernel(const BackwardParams p, const __grid_constant__ CUtensorMap q_map,
                          const __grid_constant__ CUtensorMap do_map,
                          const __grid_constant__ CUtensorMap k_map,
                          const __grid_constant__ CUtensorMap v_map, const int n_rb) {
  using C = BwdCfg<D>;
  constexpr int KS = kDqKStages, VS = kDqVStages;
  constexpr int kKOff = 2 * C::kTile128;                 // after Q and dO
  constexpr int kVOff = kKOff + KS * C::kTile128;
  constexpr uint32_t kSCol = 0, kPCol = 128, kQCol = 256, kDSCol = 256 + D;
  static_assert(kDSCol + 64 <= kTmemCols, "TMEM budget");
  extern __shared__ uint8_t smem_raw[];
  __shared__ DqBars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, tpt = 128 / G, rows_used = tpt * G;
  // Block order: groups of kGroup row blocks of one (sequence, KV head), the
  // groups of the last row blocks (which see the most keys) first.
  const int units = p.batch * p.Hk;
  const int per_group = units * kGroup;
  const int gidx = (int)blockIdx.x / per_group;
  const int rem = (int)blockIdx.x - gidx * per_group;
  const int unit = rem / kGroup;
  const int n_groups = (n_rb + kGroup - 1) / kGroup;
  const int rb = (n_groups - 1 - gidx) * kGroup + (kGroup - 1 - rem % kGroup);
  const int b = unit / p.Hk, kvh = unit - (unit / p.Hk) * p.Hk;
  int q0, q_len, k_len;
  if (rb < 0 || rb >= n_rb ||
      !seq_lengths(p, b, threadIdx.x == 0 && kvh == 0 && rb == 0, q0, q_len, k_len))
    return;
  const int tok0 = rb * tpt;
  if (tok0 >= q_len) return;
  const int off = k_len - q_len;
  const int t_end = min(q_len, tok0 + tpt);
  // key blocks of the band of the block's rows: sink blocks, then the band
  const int p_first = tok0 + off, p_last = t_end - 1 + off;
  const int lo_first = p.window > 0 ? max(0, p_first - p.window + 1) : 0;
  const int hi_all = min(p_last, k_len - 1);
  int kb_begin = 0, n_sink = 0, n_kb = 0;
  if (hi_all >= lo_first) {
    kb_begin = lo_first / 128;
    const int sink_keys = min(p.sinks, lo_first);
    n_sink = min((sink_keys + 127) / 128, kb_begin);
    n_kb = n_sink + hi_all / 128 + 1 - kb_begin;
  }
  auto kb_of = [&](int i) { return i < n_sink ? i : kb_begin + (i - n_sink); };

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  auto k_ptr = [&](int s) { return smem + kKOff + s * C::kTile128; };
  auto v_ptr = [&](int s) { return smem + kVOff + s * C::kTile128; };

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    mbar_init(&bars.sd_full, 1);
    mbar_init(&bars.sd_free, 8);
    mbar_init(&bars.ds_full, 8);
    mbar_init(&bars.dq_done, 1);
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 3 && rows_used < 128) {
    zero_rows<D>(smem, 128, rows_used, lane);
    zero_rows<D>(smem + C::kTile128, 128, rows_used, lane);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0 && n_kb > 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&do_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      mbar_arrive_expect_tx(&bars.q_full, 2u * C::kBoxes * 128u * (uint32_t)rows_used);
#pragma unroll
      for (int bx = 0; bx < C::kBoxes; ++bx) {
        tma_load_3d(smem + bx * (128 * 128), &q_map, bx * 64, kvh * G, q0 + tok0, &bars.q_full);
        tma_load_3d(smem + C::kTile128 + bx * (128 * 128), &do_map, bx * 64, kvh * G, q0 + tok0,
                    &bars.q_full);
      }
      int nk = 0, nv = 0;  // K and V tiles issued
      bool ok = true;
      for (int i = 0; i < n_kb && ok; ++i) {
        const int ks = i % KS, vs = i % VS;
        const int key0 = kb_of(i) * 128;
        const uint32_t bytes = load_keys<D>(p, &k_map, k_ptr(ks), b, kvh, key0, k_len,
                                            &bars.k_full[ks], false, false);
        if (i >= KS && !thread_wait(&bars.k_empty[ks], ((i / KS) & 1) ^ 1, abort, p.error_word,
                                    p.wait_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars.k_full[ks], bytes);
        load_keys<D>(p, &k_map, k_ptr(ks), b, kvh, key0, k_len, &bars.k_full[ks], true, true);
        ++nk;
        if (i >= VS && !thread_wait(&bars.v_empty[vs], ((i / VS) & 1) ^ 1, abort, p.error_word,
                                    p.wait_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bars.v_full[vs], bytes);
        load_keys<D>(p, &v_map, v_ptr(vs), b, kvh, key0, k_len, &bars.v_full[vs], true, false);
        ++nv;
      }
      if (!ok) do_abort(abort, p.error_word);
      // Never leave with copies in flight.
      mbar_wait(&bars.q_full, 0);
      for (int ii = max(0, nk - KS); ii < nk; ++ii) mbar_wait(&bars.k_full[ii % KS], (ii / KS) & 1);
      for (int ii = max(0, nv - VS); ii < nv; ++ii) mbar_wait(&bars.v_full[ii % VS], (ii / VS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, 0);  // 128 rows x 128 keys
    constexpr uint32_t idesc_q = tc::idesc_bf16_f32(128, D, 1);    // 128 rows x D, B MN-major
    const uint64_t qdesc = tc::smem_desc_sw128(sbase, 16, 1024);
    const uint32_t q_lo = (uint32_t)qdesc, desc_hi = (uint32_t)(qdesc >> 32);
    const uint32_t do_lo = (uint32_t)tc::smem_desc_sw128(sbase + C::kTile128, 16, 1024);
    const uint32_t k_lo = (uint32_t)tc::smem_desc_sw128(sbase + kKOff, 16, 1024);
    const uint32_t k_mn_lo = (uint32_t)tc::smem_desc_sw128(sbase + kKOff, 128 * 128, 1024);
    const uint32_t v_lo = (uint32_t)tc::smem_desc_sw128(sbase + kVOff, 16, 1024);
    bool ok = true;
    auto commit_to = [&](uint64_t* bar) {
      if (lane == 0) tc::commit(smem_u32(bar));
      __syncwarp();
    };
    // S_i = Q K_i^T and dP_i = dO V_i^T (K-major over d); V_i is free afterwards
    auto issue_s = [&](int i) -> bool {
      const int ks = i % KS, vs = i % VS;
      if (!warp_wait(&bars.k_full[ks], (i / KS) & 1, abort, p.error_word, p.wait_ns) ||
          !warp_wait(&bars.v_full[vs], (i / VS) & 1, abort, p.error_word, p.wait_ns))
        return false;
      tc::fence_after_sync();
      const uint32_t kso = (uint32_t)((ks * C::kTile128) >> 4);
      const uint32_t vso = (uint32_t)((vs * C::kTile128) >> 4);
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (uint32_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
          tc::mma_ss_lo(tmem + kSCol, q_lo + o, k_lo + kso + o, desc_hi, idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (uint32_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
          tc::mma_ss_lo(tmem + kPCol, do_lo + o, v_lo + vso + o, desc_hi, idesc_s, kk > 0);
        }
        tc::commit(smem_u32(&bars.sd_full));
        tc::commit(smem_u32(&bars.v_empty[vs]));
      }
      __syncwarp();
      return true;
    };
    if (n_kb > 0) ok = warp_wait(&bars.q_full, 0, abort, p.error_word, p.wait_ns) && issue_s(0);
    for (int i = 0; ok && i < n_kb; ++i) {
      const int ks = i % KS;
      if (i + 1 < n_kb) {
        // S_{i+1}, dP_{i+1} as soon as the compute warps hold S_i, dP_i
        if (!warp_wait(&bars.sd_free, i & 1, abort, p.error_word, p.wait_ns) || !issue_s(i + 1)) {
          ok = false;
          break;
        }
      }
      if (!warp_wait(&bars.ds_full, i & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      const int key0 = kb_of(i) * 128;
      if (key0 + 128 > k_len) {
        // key rows at or past k_len: zero them before dQ reads K_i (S_i has
        // read them already: the compute warps have seen S_i)
        zero_rows<D>(k_ptr(ks), 128, max(0, k_len - key0), lane);
        fence_proxy_async_smem();
        __syncwarp();
      }
      tc::fence_after_sync();
      if (lane == 0) {
        // dQ += dS_i K_i: A = dS from its own tensor-memory region, B = K_i
        // read MN-major (keys x d)
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          tc::mma_ts_lo(tmem + kQCol, tmem + kDSCol + kk * 8,
                        k_mn_lo + (uint32_t)((ks * C::kTile128 + kk * 16 * 128) >> 4), desc_hi,
                        idesc_q, (i > 0 || kk > 0) ? 1u : 0u);
        tc::commit(smem_u32(&bars.dq_done));
        tc::commit(smem_u32(&bars.k_empty[ks]));
      }
      __syncwarp();
    }
    if (ok && n_kb > 0) commit_to(&bars.acc_full);
    if (!ok) do_abort(abort, p.error_word);
    commit_to(&bars.drain);
    if (!warp_wait(&bars.drain, 0, abort, p.error_word, p.wait_ns)) mbar_wait(&bars.drain, 0);
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  } else {
    // -------------------------------------------------------- compute warps
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    const int qw = warp & 3;               // row quarter (TMEM lanes)
    const int hh = (warp - 4) >> 2;        // key half of every block
    const int r = qw * 32 + lane;          // packed row of this thread
    const int tok = tok0 + r / G;
    const bool row_ok = r < rows_used && tok < q_len;
    const int pos = tok + off;
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + kSCol + hh * 64;
    const uint32_t p_addr = tmem + lane_base + kPCol + hh * 64;
    const uint32_t ds_addr = tmem + lane_base + kDSCol + hh * 32;
    const float sl2 = p.scale * kLog2e;
    const size_t hrow = (size_t)(q0 + (row_ok ? tok : 0)) * p.H + (size_t)kvh * G + (r % G);
    // -lse log2 e and -D of this row (D = dO . O, from the forward's output)
    float nl = 0.f, nd = 0.f;
    if (row_ok) {
      nl = -__ldg(p.lse + hrow) * kLog2e;
      const uint4* g = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.d_out) +
                                                      hrow * D);
      const uint4* o = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.out) +
                                                      hrow * D);
      float acc = 0.f;
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
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
      nd = -acc;
    }
    const int lo = p.window > 0 ? pos - p.window + 1 : 0;
    bool ok = true;
    for (int i = 0; i < n_kb; ++i) {
      if (!warp_wait(&bars.sd_full, i & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float sv[64], dv[64];
      tc::tmem_ld32(s_addr, sv);
      tc::tmem_ld32(s_addr + 32, sv + 32);
      tc::tmem_ld32(p_addr, dv);
      tc::tmem_ld32(p_addr + 32, dv + 32);
      tc::tmem_wait_ld();
      // S_i and dP_i are in registers: the tensor core may overwrite them
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.sd_free);
      // visible key columns of this warp's half: [c_lo, c_hi] and, under a
      // window, the sinks below c_sink
      const int kbase = kb_of(i) * 128 + hh * 64;
      const int hi = min(pos, k_len - 1);
      int c_lo = row_ok ? lo - kbase : 64;
      const int c_hi = row_ok ? hi - kbase : -1;
      const int c_sink = p.window > 0 ? min(p.sinks, k_len) - kbase : 0;
      if (c_sink >= c_lo) c_lo = -1;  // the sinks join the window: one interval
      const bool full = c_lo <= 0 && c_hi >= 63;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float x0, x1, p0, p1, t0, t1;
        fma2(x0, x1, sv[c], sv[c + 1], sl2, nl);
        p0 = fast_exp2(x0);
        p1 = fast_exp2(x1);
        fma2(t0, t1, dv[c], dv[c + 1], 1.0f, nd);
        mul2(sv[c], sv[c + 1], p0, p1, t0, t1);  // dS in place of S
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if ((c < c_lo && c >= c_sink) || c > c_hi) sv[c] = 0.f;
      }
      uint32_t pk[32];
#pragma unroll
      for (int w = 0; w < 32; ++w) pk[w] = pack_bf16x2(sv[2 * w], sv[2 * w + 1]);
      // dS_{i-1} must have been read by its dQ MMA before it is overwritten
      if (i > 0 && !warp_wait(&bars.dq_done, (i - 1) & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      tc::tmem_st32(ds_addr, reinterpret_cast<const float*>(pk));
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.ds_full);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n_kb > 0) ok = warp_wait(&bars.acc_full, 0, abort, p.error_word, p.wait_ns);
    if (!ok) {
      tc::tmem_wait_st();
      do_abort(abort, p.error_word);
    } else {
      // d_q holds D of every row until the dK / dV grid (launched before this
      // one, as its programmatic dependent) has completed
      asm volatile("griddepcontrol.wait;" ::: "memory");
      // every lane loads (tcgen05.ld is warp-collective); valid rows store
      float* dq = p.d_q + hrow * D + hh * (D / 2);
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < D / 2; c += 32) {
        float qv[32];
        if (n_kb > 0) {
          tc::tmem_ld32(tmem + lane_base + kQCol + hh * (D / 2) + c, qv);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) qv[e] = 0.f;
        }
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dq + c + e) =
                make_float4(qv[e] * p.scale, qv[e + 1] * p.scale, qv[e + 2] * p.scale,
                            qv[e + 3] * p.scale);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_d(const BackwardParams& p, const CUtensorMap& q_map64,
                     const CUtensorMap& do_map64, const CUtensorMap& q_map128,
                     const CUtensorMap& do_map128, const CUtensorMap& k_map,
                     const CUtensorMap& v_map, cudaStream_t stream) {
  using C = BwdCfg<D>;
  constexpr int kDkvSmem = 2 * C::kTile128 + kDkvStages * (2 * C::kTile64 + 1024) + 1024;
  constexpr int kDqSmem = (2 + kDqKStages + kDqVStages) * C::kTile128 + 1024;
  static_assert(kDkvSmem <= 232448 - 1024 && kDqSmem <= 232448 - 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kDkvSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kDqSmem);
  if (e != cudaSuccess) return e;
  const long long units = (long long)p.batch * p.Hk;
  // D of every row into the first T H floats of d_q, read by the dK / dV kernel.
  if (p.max_kv_len > 0) {
    float* delta = p.d_q;
    const long long rows = (long long)p.T * p.H;
    attn_bwd_tc_delta_kernel<D><<<(unsigned)((rows * 8 + 255) / 256), 256, 0, stream>>>(p, delta);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int n_kb = (p.max_kv_len + 127) / 128;
    const long long blocks = (long long)((n_kb + kGroup - 1) / kGroup) * units * kGroup;
    // A programmatic dependent of the D grid: only its loader warp reads D,
    // after griddepcontrol.wait.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kDkvSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attn_bwd_dkv_tc_kernel<D>, p, q_map64, do_map64, k_map, v_map,
                           (const float*)delta, n_kb);
    if (e != cudaSuccess) return e;
  }
  const int tpt = 128 / p.G;
  const int n_rb = std::max(1, (p.max_q_len + tpt - 1) / tpt);
  const long long blocks = (long long)((n_rb + kGroup - 1) / kGroup) * units * kGroup;
  // A programmatic dependent of the dK / dV grid: its CTAs start as SMs free
  // up and wait for that grid only before storing into d_q.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kDqSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = p.max_kv_len > 0 ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_bwd_dq_tc_kernel<D>, p, q_map128, do_map128, k_map, v_map,
                            n_rb);
}

}  // namespace

bool attn_backward_tc_supported(const BackwardParams& p, rpk_dtype dtype) {
  if (dtype != RPK_BF16 || p.cache_fp8 || p.G < 1 || p.G > kDkvRows) return false;
  if (p.d != 64 && p.d != 128) return false;
  // one-dimensional grids of kGroup-block groups
  const long long units = (long long)p.batch * p.Hk;
  const long long n_kb = (p.max_kv_len + 127) / 128;
  const long long n_rb = (p.max_q_len + 128 / p.G - 1) / (128 / p.G);
  return (n_kb + kGroup) * units * kGroup < INT32_MAX && (n_rb + kGroup) * units * kGroup < INT32_MAX;
}

cudaError_t launch_attn_backward_tc(const BackwardParams& p, const CUtensorMap& q_map64,
                                    const CUtensorMap& do_map64, const CUtensorMap& q_map128,
                                    const CUtensorMap& do_map128, const CUtensorMap& k_map,
                                    const CUtensorMap& v_map, cudaStream_t stream) {
  if (p.batch == 0 || (long long)p.T * p.H == 0) return cudaSuccess;
  switch (p.d) {
    case 64:
      return launch_d<64>(p, q_map64, do_map64, q_map128, do_map128, k_map, v_map, stream);
    case 128:
      return launch_d<128>(p, q_map64, do_map64, q_map128, do_map128, k_map, v_map, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpk

// attn_prefill.cu -- ragged causal GQA attention over the paged cache on the
// 5th-generation tensor cores (tcgen05), bf16 in, fp32 accumulate.
//
// Semantics: NumKong "Attention with a Pre-Packed KV-Cache" (row r of a
// sequence with q_len rows and k_len keys sits at p = r + k_len - q_len and
// sees keys [p - (window - 1), p]; rows that see no key are zeros), scores
// scale * q.k (algenta scaled_dot_product_attention) and the flash
// online-softmax running state (algenta flash_attention: running max,
// running sum and output rescaled by e^(m_old - m_new), final divide).
//
// Work unit: two query tiles A and B of 128 rows each against 128-key tiles.
// The 128 rows of a tile are the (token, query head) pairs of one KV head's
// group, token-major (tokens_per_tile = 128 / G), so the G query heads that
// share a KV head share every K/V tile; tile B holds the next tokens_per_tile
// tokens after tile A. One CTA per (pair of query tiles, KV head, sequence),
// heaviest pairs first.
//
// Warp roles (384 threads, three warpgroups):
//   warp 0     TMA producer: both Q tiles once, then K and V tiles of 128 keys
//              into a 2-stage ring, one box per page segment (3-D map over the
//              pool [pages * page_size, kv_heads, d], 128-byte swizzle, no
//              multicast)
//   warp 1     allocates TMEM (512 columns: S_A, S_B, O_A, O_B) and issues the
//              MMAs from one thread, alternating the tiles: S_t = Q_t K_j^T
//              (operands in shared memory), then O_t += P_t V_j with P_t read
//              from TMEM (written over the first 64 columns of S_t) and V_j an
//              MN-major operand in shared memory. While one softmax warpgroup
//              works on its tile, the tensor core runs the other tile's MMAs.
//   warps 2-3  idle (they complete the first warpgroup)
//   warps 4-7  softmax of tile A, warps 8-11 softmax of tile B: thread r owns
//              row r (TMEM lane r); loads S_t, masks the band, keeps (m, l) in
//              log2 units, writes P_t as packed bf16 pairs, and rescales O_t in
//              TMEM only when the running max grew by more than 2^8 (the final
//              O / l uses the same max, so this is exact); then normalises O_t
//              and stores the rows.
// Registers: the first warpgroup gives registers back (setmaxnreg 64) and the
// two softmax warpgroups take them (setmaxnreg 208), so that a softmax thread
// holds a whole 128-score row without spilling; 4*32*64 + 8*32*208 = 61440
// registers, within the 384 * 168 the CTA is launched with.
// MMAs issued by one thread run in issue order, so P_t(j) V_j completes before
// S_t(j+1) overwrites the columns P_t(j) lives in, and the completion of
// S_t(j+1) also tells the softmax that O_t holds P_t(j) V_j.
// Value rows at or past k_len are zeroed in shared memory before P V, so the
// NaN sentinels of unused slots never meet a zero weight. Every mbarrier wait
// is bounded; on a timeout the CTA raises RPK_DEVERR_TIMEOUT, drains its copies
// and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace rpk {

int prefill_rows_per_tile(int group) { return group >= 1 && group <= 128 ? (128 / group) : 0; }

namespace {

constexpr int kBM = 128;   // rows per tile (MMA M)
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 384;
constexpr int kRegsControl = 64;    // warpgroup 0: producer, MMA issuer, 2 idle warps
constexpr int kRegsSoftmax = 208;   // warpgroups 1 and 2: softmax
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows > 2^8

// Packed and three-input fp32 instructions of sm_100: the softmax is bound by
// instruction issue (one softmax warp per SM sub-partition), so two scores per
// instruction where the hardware allows it.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (d0, d1) = (a0, a1) * b + c
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %4};\n\t"
      "mov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// (s0, s1) += (a0, a1)
__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(s0), "=f"(s1)
      : "f"(a0), "f"(a1), "f"(s0), "f"(s1));
}

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = D == 128 ? 2 : 4;   // K/V ring depth
  static constexpr int kQBytes = kBM * D * 2;         // one query tile
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kQBytes;
  static constexpr int kVOff = kKOff + kStages * kKVBytes;
  static constexpr int kEnd = kVOff + kStages * kKVBytes + 1024;
  // At least half the SM's shared memory, so that one CTA holds the SM's TMEM.
  static constexpr int kSmemBytes = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  // TMEM columns: S_A, S_B (fp32, 128 each; P_t over the first 64 of S_t), O_A, O_B
  static constexpr uint32_t kSCol = 0;
  static constexpr uint32_t kOCol = 2 * kBN;
  static_assert(kOCol + 2 * D <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4];
  uint64_t v_full[4];
  uint64_t k_empty[4];
  uint64_t v_empty[4];
  uint64_t s_full[2];   // per query tile
  uint64_t p_full[2];   // per query tile
  uint64_t o_final[2];  // per query tile: its last P V has completed
  uint64_t drain;
};

// A CTA that gives up on a wait publishes RPK_DEVERR_TIMEOUT in the error
// word; every other CTA of the launch (and of later launches, until the caller
// clears the word) sees it and stops early instead of waiting out its own
// bound, so a broken launch ends in about one bound, not one per CTA.
__device__ __forceinline__ bool timed_out_elsewhere(const int32_t* error_word) {
  return error_word &&
         (*reinterpret_cast<const volatile int32_t*>(error_word) & (int32_t)RPK_DEVERR_TIMEOUT);
}

// Bounded wait by one thread; false on timeout or abort. The thread sleeps in
// try_wait (woken when the phase completes, at most 0.2 ms per try), so
// waiting warps leave the issue slots to the warps that compute; between
// tries it looks at the abort flag, the timer and, once the wait has lasted
// longer than any healthy one (50 us), the global error word.
__device__ __forceinline__ bool thread_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            const int32_t* error_word) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
#pragma unroll 1
  while (true) {
    if (mbar_try_wait_suspend(a, parity, 200000u)) return true;
    if (*abort) return false;
    const unsigned long long dt = global_timer_ns() - t0;
    if (dt > kWaitTimeoutNs) return false;
    if (dt > 50000ull && timed_out_elsewhere(error_word)) return false;
  }
}

// Bounded wait shared by the whole warp: every lane polls (so each lane has
// acquired the phase) and the lanes agree on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const int32_t* error_word) {
  const bool ok = thread_wait(bar, parity, abort, error_word);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void do_abort(volatile int* abort, int32_t* error_word) {
  if (!*abort) {
    *abort = 1;
    raise_error(error_word, RPK_DEVERR_TIMEOUT);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const AttnParams p, const __grid_constant__ CUtensorMap q_map,
                        const __grid_constant__ CUtensorMap k_map,
                        const __grid_constant__ CUtensorMap v_map, const int tpt,
                        const int n_qtiles) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The q-tile index is the slowest grid dimension, reversed: the first waves
  // hold the last (heaviest) tile of every (sequence, KV head), so the long
  // tiles start first and the short ones fill the tail.
  const int qt = n_qtiles - 1 - (int)blockIdx.z;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int q0 = __ldg(p.offsets + b);
  const int q_len = __ldg(p.offsets + b + 1) - q0;
  const int k_len = __ldg(p.kv_lens + b);
  if (q_len > p.max_q_len || k_len < 0 || k_len > p.max_kv_len) {
    if (threadIdx.x == 0 && blockIdx.z == 0 && kvh == 0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
    return;
  }
  const int t_begin = qt * 2 * tpt;           // first token of tile A
  if (t_begin >= q_len) return;
  if (timed_out_elsewhere(p.error_word)) return;
  const bool has_b = t_begin + tpt < q_len;    // tile B holds at least one token
  const int t_end = min(q_len, t_begin + 2 * tpt);
  const int G = p.G;
  const int rows_used = tpt * G;

  // Keys any row of the two tiles sees, in whole key tiles.
  const int p_first = t_begin + k_len - q_len;
  const int p_last = (t_end - 1) + k_len - q_len;
  const int lo_first = p.window > 0 ? max(0, p_first - p.window + 1) : 0;
  const int hi_all = min(p_last, k_len - 1);
  int j_begin = 0, n_tiles = 0;
  if (hi_all >= lo_first) {
    j_begin = lo_first / kBN;
    n_tiles = hi_all / kBN + 1 - j_begin;
  }

  constexpr int S = C::kStages;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  auto q_s = [&](int t) { return sbase + C::kQOff + t * C::kQBytes; };
  auto k_s = [&](int st) { return sbase + C::kKOff + st * C::kKVBytes; };
  auto v_s = [&](int st) { return sbase + C::kVOff + st * C::kKVBytes; };

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int st = 0; st < S; ++st) {
      mbar_init(&bars.k_full[st], 1);
      mbar_init(&bars.v_full[st], 1);
      mbar_init(&bars.k_empty[st], 1);
      mbar_init(&bars.v_empty[st], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.s_full[t], 1);
      mbar_init(&bars.p_full[t], 128);
      mbar_init(&bars.o_final[t], 1);
    }
    mbar_init(&bars.drain, 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base_sh;
  const int32_t* bt = p.block_table + (size_t)b * p.max_pages;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      const int n_q = has_b ? 2 : 1;
      const uint32_t q_box_bytes = 128u * (uint32_t)rows_used;
      mbar_arrive_expect_tx(&bars.q_full, n_q * C::kBoxes * q_box_bytes);
      for (int t = 0; t < n_q; ++t)
#pragma unroll
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(smem + C::kQOff + t * C::kQBytes + bx * (kBM * 128), &q_map, bx * 64,
                      kvh * G, q0 + t_begin + t * tpt, &bars.q_full);
      const int box_rows = p.P < kBN ? p.P : kBN;
      const uint32_t seg_bytes = (uint32_t)box_rows * 128u * C::kBoxes;
      int issued = 0;
      // K_i and V_i go to stage i % S; K of a stage frees after the last S
      // MMA that reads it, V after the last P V, so K runs ahead of V.
      auto load = [&](int i, bool is_v) -> bool {
        const int st = i % S;
        uint64_t* empty = is_v ? &bars.v_empty[st] : &bars.k_empty[st];
        uint64_t* full = is_v ? &bars.v_full[st] : &bars.k_full[st];
        if (i >= S && !thread_wait(empty, ((i / S) & 1) ^ 1, abort, p.error_word)) return false;
        const int key0 = (j_begin + i) * kBN;
        uint32_t bytes = 0;
        for (int r = 0; r < kBN; r += box_rows) {
          const int key = key0 + r;
          if (key >= k_len) break;
          const int pi = key / p.P;
          const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
          if (page >= 0 && page < p.num_pages) bytes += seg_bytes;
        }
        mbar_arrive_expect_tx(full, bytes);
        for (int r = 0; r < kBN; r += box_rows) {
          const int key = key0 + r;
          if (key >= k_len) break;
          const int pi = key / p.P;
          const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
          if (page < 0 || page >= p.num_pages) {
            if (!is_v) raise_error(p.error_word, RPK_DEVERR_PAGE);
            continue;
          }
          const int grow = page * p.P + (key - pi * p.P);
          uint8_t* base = smem + (is_v ? C::kVOff : C::kKOff) + st * C::kKVBytes + r * 128;
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(base + bx * (kBN * 128), is_v ? &v_map : &k_map, bx * 64, kvh, grow, full);
        }
        return true;
      };
      for (int i = 0; i < n_tiles; ++i) {
        if (!load(i, false) || !load(i, true)) {
          do_abort(abort, p.error_word);
          break;
        }
        ++issued;
      }
      // Never leave with copies in flight.
      mbar_wait(&bars.q_full, 0);
      for (int i = max(0, issued - S); i < issued; ++i) {
        mbar_wait(&bars.k_full[i % S], (i / S) & 1);
        mbar_wait(&bars.v_full[i % S], (i / S) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(kBM, kBN, 0);
    constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(kBM, D, 1);
    bool ok = warp_wait(&bars.q_full, 0, abort, p.error_word);
    tc::fence_after_sync();
    // S_t = Q_t K_i^T into S_t's columns.
    auto issue_s = [&](int t, int i) {
      if (lane == 0) {
        const int st = i % S;
        const uint32_t d_tmem = tmem + C::kSCol + (uint32_t)(t * kBN);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t koff = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          tc::mma_ss(d_tmem, tc::smem_desc_sw128(q_s(t) + qoff, 16, 1024),
                     tc::smem_desc_sw128(k_s(st) + koff, 16, 1024), idesc_qk, kk > 0);
        }
        tc::commit(smem_u32(&bars.s_full[t]));
      }
      __syncwarp();
    };
    // O_t += P_t V_i, P_t in the first 64 columns of S_t.
    auto issue_pv = [&](int t, int i) {
      if (lane == 0) {
        const int st = i % S;
        const uint32_t d_tmem = tmem + C::kOCol + (uint32_t)(t * D);
        const uint32_t a_tmem = tmem + C::kSCol + (uint32_t)(t * kBN);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc::mma_ts(d_tmem, a_tmem + kk * 8,
                     tc::smem_desc_sw128(v_s(st) + kk * (16 * 128), kBN * 128, 1024), idesc_pv,
                     (i > 0 || kk > 0) ? 1u : 0u);
      }
      __syncwarp();
    };
    if (ok && n_tiles > 0) {
      ok = warp_wait(&bars.k_full[0], 0, abort, p.error_word);
      tc::fence_after_sync();
      if (ok) {
        issue_s(0, 0);
        if (has_b) issue_s(1, 0);
        if (lane == 0) tc::commit(smem_u32(&bars.k_empty[0]));
        __syncwarp();
      }
    }
    for (int i = 0; ok && i < n_tiles; ++i) {
      const int st = i % S;
      const bool last = i + 1 == n_tiles;
      // tile A: P_A(i) V_i, then S_A(i+1)
      if (!warp_wait(&bars.p_full[0], i & 1, abort, p.error_word)) { ok = false; break; }
      if (!warp_wait(&bars.v_full[st], (i / S) & 1, abort, p.error_word)) { ok = false; break; }
      tc::fence_after_sync();
      const int key0 = (j_begin + i) * kBN;
      if (key0 + kBN > k_len) {
        // zero value rows at or past k_len
        const int r0 = max(0, k_len - key0);
        const int chunks = (kBN - r0) * C::kBoxes * 8;
        for (int idx = lane; idx < chunks; idx += 32) {
          const int ch = idx & 7;
          const int rb = idx >> 3;
          const int bx = rb % C::kBoxes;
          const int r = r0 + rb / C::kBoxes;
          uint8_t* dst = smem + C::kVOff + st * C::kKVBytes + bx * (kBN * 128) + r * 128 + ch * 16;
          *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      issue_pv(0, i);
      if (last && lane == 0) tc::commit(smem_u32(&bars.o_final[0]));
      if (!last) {
        if (!warp_wait(&bars.k_full[(i + 1) % S], ((i + 1) / S) & 1, abort, p.error_word)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        issue_s(0, i + 1);
      }
      // tile B: P_B(i) V_i, then S_B(i+1)
      if (has_b) {
        if (!warp_wait(&bars.p_full[1], i & 1, abort, p.error_word)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(1, i);
        if (last && lane == 0) tc::commit(smem_u32(&bars.o_final[1]));
      }
      if (lane == 0) tc::commit(smem_u32(&bars.v_empty[st]));
      __syncwarp();
      if (has_b && !last) issue_s(1, i + 1);
      // K_{i+1} has now been read by every S MMA that needs it.
      if (!last && lane == 0) tc::commit(smem_u32(&bars.k_empty[(i + 1) % S]));
      __syncwarp();
    }
    if (!ok) do_abort(abort, p.error_word);
    // Drain: every MMA issued above has completed before TMEM is freed.
    if (lane == 0) tc::commit(smem_u32(&bars.drain));
    __syncwarp();
    if (!warp_wait(&bars.drain, 0, abort, p.error_word)) mbar_wait(&bars.drain, 0);
  } else if (warp < 4) {
    // idle warps of the first warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int t = (warp - 4) >> 2;       // query tile: warps 4-7 -> A, 8-11 -> B
    const int qw = warp & 3;             // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;        // row of this thread
    const int tok = t_begin + t * tpt + r / G;
    const bool row_ok = r < rows_used && tok < q_len;
    const int pos = tok + k_len - q_len;
    const int lo = p.window > 0 ? pos - p.window + 1 : 0;
    const int hi = pos;
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    const uint32_t s_col = tmem + lane_base + C::kSCol + (uint32_t)(t * kBN);
    const uint32_t o_col = tmem + lane_base + C::kOCol + (uint32_t)(t * D);
    const float sl2 = p.scale_log2;
    const int my_tiles = (t == 0 || has_b) ? n_tiles : 0;
    float m = -INFINITY, l = 0.f;        // running max (log2 units) and sum
    bool ok = true;
    float v[kBN];
    for (int i = 0; i < my_tiles; ++i) {
      if (!warp_wait(&bars.s_full[t], i & 1, abort, p.error_word)) { ok = false; break; }
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tc::tmem_ld32(s_col + c * 32, v + c * 32);
      tc::tmem_wait_ld();
      const int key0 = (j_begin + i) * kBN;
      if (!(row_ok && key0 >= lo && key0 + kBN - 1 <= hi)) {
        // visible columns [c_lo, c_hi] of this tile (empty for an invalid row)
        const int c_lo = row_ok ? lo - key0 : kBN;
        const int c_hi = row_ok ? hi - key0 : -1;
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c < c_lo || c > c_hi) v[c] = -INFINITY;
      }
      // Row max: 8 independent chains of three-input max.
      float m8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) m8[k] = fmaxf(v[k], v[8 + k]);
#pragma unroll
      for (int c = 16; c < kBN; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = max3(m8[k], v[c + k], v[c + 8 + k]);
      float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      mx *= sl2;  // scale > 0: max of the scaled scores
      // Running max: taken at once while empty, else only when it grows by
      // more than the threshold (then O and l are rescaled). O_t holds
      // P_t(i-1) V_{i-1} here: S_t(i) was issued after it and has completed.
      float alpha = 1.f;
      bool rescale = false;
      if (m == -INFINITY) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);
        m = mx;
        rescale = true;
      }
      l *= alpha;
      const float neg_m = m == -INFINITY ? 0.f : -m;  // an empty row keeps P = 0
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 4 packed partial sums
      // P in two halves of 64 keys (32 packed columns each) to bound registers.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          float x0, x1;
          fma2(x0, x1, v[h * 64 + c], v[h * 64 + c + 1], sl2, neg_m);
          const float w0 = fast_exp2(x0);
          const float w1 = fast_exp2(x1);
          const int k = (c >> 1) & 3;
          add2(rs[2 * k], rs[2 * k + 1], w0, w1);
          pk[c >> 1] = pack_bf16x2(w0, w1);
        }
        tc::tmem_st32(s_col + h * 32, reinterpret_cast<const float*>(pk));
      }
      l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      // Rescale O_t (after P, so that the scores are dead): it must finish
      // before P_t(i) V_i is issued, i.e. before p_full.
      if (i > 0 && __any_sync(0xffffffffu, rescale)) {
        float o[32];
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          tc::tmem_ld32(o_col + c * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tc::tmem_st32(o_col + c * 32, o);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      mbar_arrive(&bars.p_full[t]);
    }
    if (!ok) do_abort(abort, p.error_word);
    // ------------------------------------------------------------ epilogue
    bool have_o = my_tiles > 0;
    if (have_o) {
      have_o = warp_wait(&bars.o_final[t], 0, abort, p.error_word);
      tc::fence_after_sync();
    }
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    const size_t orow = ((size_t)(q0 + tok) * p.H + (size_t)kvh * G + (r % G)) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      if (have_o) {
        tc::tmem_ld32(o_col + c * 32, o);
        tc::tmem_wait_ld();
      }
      if (row_ok) {
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
          uint4 q4;
          if (have_o && l > 0.f) {
            q4.x = pack_bf16x2(o[e8 * 8 + 0] * inv, o[e8 * 8 + 1] * inv);
            q4.y = pack_bf16x2(o[e8 * 8 + 2] * inv, o[e8 * 8 + 3] * inv);
            q4.z = pack_bf16x2(o[e8 * 8 + 4] * inv, o[e8 * 8 + 5] * inv);
            q4.w = pack_bf16x2(o[e8 * 8 + 6] * inv, o[e8 * 8 + 7] * inv);
          } else {
            q4 = make_uint4(0, 0, 0, 0);
          }
          *reinterpret_cast<uint4*>(out + orow + c * 32 + e8 * 8) = q4;
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
cudaError_t launch_d(const AttnParams& p, const CUtensorMap& q_map, const CUtensorMap& k_map,
                     const CUtensorMap& v_map, cudaStream_t stream) {
  using C = Cfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int tpt = prefill_rows_per_tile(p.G);
  const int n_qtiles = (p.max_q_len + 2 * tpt - 1) / (2 * tpt);  // pairs of query tiles
  if (n_qtiles == 0) return cudaSuccess;
  if (n_qtiles > 65535) return cudaErrorInvalidValue;
  dim3 grid(p.Hk, p.batch, n_qtiles);
  attn_prefill_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(p, q_map, k_map, v_map, tpt,
                                                                     n_qtiles);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnParams& p, const CUtensorMap& q_map,
                                const CUtensorMap& k_map, const CUtensorMap& v_map,
                                cudaStream_t stream) {
  if ((long long)p.T * p.H == 0 || p.batch == 0) return cudaSuccess;
  switch (p.d) {
    case 64: return launch_d<64>(p, q_map, k_map, v_map, stream);
    case 128: return launch_d<128>(p, q_map, k_map, v_map, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpk

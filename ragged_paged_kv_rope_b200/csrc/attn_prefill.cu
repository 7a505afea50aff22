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
// Work unit (item): NT query tiles of 128 rows each of one (sequence, KV
// head), against key tiles of 64 keys; NT = 2 (tiles A and B) for head_dim 64
// and 128, NT = 1 for head_dim 256. The 128 rows of a tile are the (token,
// query head) pairs of one KV head's group, token-major (tokens_per_tile =
// 128 / G), so the G query heads that share a KV head share every K/V tile;
// tile B holds the next tokens_per_tile tokens after tile A.
//
// Persistent launch: one CTA per SM claims items from a counter in the
// caller's workspace (zeroed by the launch). Items run sequence by sequence,
// the last (longest) query group of a sequence first: the CTAs that work on
// one sequence at the same time read the same K/V tiles in the same order, so
// a tile read from HBM for one of them is an L2 hit for the others.
//
// Tensor memory (512 columns): two score buffers of 64 columns per query
// tile (S_t[0], S_t[1]) and one 128-row output accumulator per tile (O_t,
// head_dim columns). Score tile i of every query tile lives in buffer i mod 2,
// and P_t(i) (packed bf16 pairs) is written over the first 32 columns of
// S_t(i). The MMA issuer computes S(i+2) right after issuing P(i) V_i, so
// while the softmax warpgroups turn S(i) into P(i), the tensor core has
// already computed S(i+1): the softmax does not wait for the tensor core in
// the steady state. Every item runs all its query tiles (rows past the
// sequence are masked and never stored), so the tiles share every barrier
// phase.
//
// Warp roles (384 threads, three warpgroups):
//   warp 0     TMA producer: claims the next item, hands its index to the
//              other roles through a two-slot ring in shared memory, loads the
//              item's Q tiles, then each key tile's K into a ring of K slots
//              and its V into a ring of V slots (3-D map over the pool
//              [pages * page_size, kv_heads, d], one box per page segment,
//              128-byte swizzle, no multicast). A K slot frees when the S MMAs
//              that read it complete, a V slot when its P V MMAs do, so the K
//              of tile i+2 never waits for the V of tile i.
//   warp 1     allocates TMEM and issues the MMAs from one thread: per item
//              S(0), S(1), then per key tile i one burst of O_t += P_t(i) V_i
//              (P from TMEM, V an MN-major operand in shared memory) and
//              S_t(i+2) (Q_t K^T, both operands in shared memory) for every
//              tile t; the next item's first S MMAs follow the last P V of the
//              current one
//   warps 2-3  idle (they complete the first warpgroup); over an e4m3 cache
//              they narrow the query tiles to f16, and a fourth warpgroup
//              (warps 12-15) widens the key tiles' codes to f16
//   warps 4-7  softmax of tile A, warps 8-11 softmax of tile B (idle when
//              NT = 1): thread r owns row r (TMEM lane r); loads S_t(i), masks
//              the band, keeps (m, l) in log2 units, writes P_t(i), and
//              rescales O_t in TMEM only when the running max grew by more
//              than 2^8 (the final O / l uses the same max, so this is exact);
//              then normalises O_t and stores the rows.
// A rescale of O_t during tile i must fall between P(i-1) V_{i-1} and
// P(i) V_i. For i < n - 1 the softmax waits for S(i+1), which the issuer
// placed after P(i-1) V_{i-1}; for the item's last tile it waits for a
// barrier the issuer commits once per item after P(n-2) V_{n-2}. Either
// barrier can be at most one phase short of the one waited for (P(i) V_i
// needs this warp's own P(i)), so the phase parity is unambiguous.
// Registers: the first warpgroup gives registers back (setmaxnreg 56) and the
// two softmax warpgroups take them (setmaxnreg 224);
// 4*32*56 + 8*32*224 = 64512 registers, the 384 * 168 the CTA is launched with
// (e4m3: 512 threads, warpgroups 0 and 3 at 56, the softmax at 200, 512 * 128).
// Value rows at or past k_len are zeroed in shared memory before P V, so the
// NaN sentinels of unused slots never meet a zero weight. Every mbarrier wait
// is bounded; on a timeout the CTA raises RPK_DEVERR_TIMEOUT, drains its copies
// and MMAs, frees TMEM and returns.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace rpk {

int prefill_rows_per_tile(int group) { return group >= 1 && group <= 128 ? (128 / group) : 0; }

namespace {

constexpr int kBM = 128;              // rows per tile (MMA M)
constexpr int kBN = kPrefillKeyTile;  // keys per tile (64)
constexpr int kRegsControl = 56;    // warpgroup 0 (and 3): producer, MMA issuer, helpers
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows > 2^8

// NT query tiles of 128 rows per work item: two for head_dim 64 and 128, one
// for head_dim 256 (whose 256-column output accumulator leaves tensor memory
// for one tile's double-buffered scores only). F8: the pools hold e4m3 codes;
// TMA brings each key tile's codes into a small raw ring and four converter
// warps widen them to f16 in the stages the MMAs read.
template <int D, int NT, bool F8 = false>
struct Cfg {
  static constexpr int kBoxes = D / 64;
  // Warpgroup 0: producer, MMA issuer and two warps that, for an e4m3 cache,
  // narrow Q; warpgroups 1 and 2: softmax; for an e4m3 cache a fourth
  // warpgroup widens the key tiles. Registers: 56 per thread in warpgroups 0
  // and 3, the rest of the launch allocation to the softmax.
  static constexpr int kThreads = F8 ? 512 : 384;
  static constexpr int kRegsSoftmax = F8 ? 200 : 224;
  static_assert(4 * 32 * kRegsControl * (F8 ? 2 : 1) + 8 * 32 * kRegsSoftmax ==
                    kThreads * ((65536 / kThreads) & ~7),
                "register split");
  // head_dim 64 / 128: one ring of stages, each the K and V of one key tile,
  // freed when its P V MMAs complete. head_dim 256: a ring of K slots, freed
  // when their S MMAs complete, and a ring of V slots, freed when their P V
  // MMAs do; with one 64 KB stage per tile only two would fit, and S(i+2),
  // issued right after P(i) V_i, would wait for the stage P(i) V_i reads.
  static constexpr bool kSplit = D == 256;
  static_assert(!(F8 && kSplit), "e4m3 prefill takes head_dim 64 / 128");
  static_assert(!F8 || NT == 2, "e4m3: one converter warp narrows each query tile");
  static constexpr int kKStages =
      D == 64 ? (F8 ? 8 : 10) : (D == 128 ? (F8 ? 4 : 5) : 3);  // stages / K slots
  static constexpr int kVStages = kSplit ? 2 : kKStages;              // V slots
  static constexpr int kQBytes = kBM * D * 2;         // one query tile
  static constexpr int kKVBytes = kBN * D * 2;        // one K or V tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + NT * kQBytes;
  // unified stage st: K at kKOff + 2 st kKVBytes, V right after it
  static constexpr int kKStride = kSplit ? kKVBytes : 2 * kKVBytes;
  static constexpr int kVOff = kSplit ? kKOff + kKStages * kKVBytes : kKOff + kKVBytes;
  static constexpr int kVStride = kKStride;
  static constexpr int kRawStages = F8 ? 2 : 0;         // raw ring: K then V codes of a tile
  static constexpr int kRawBytes = kBN * D;             // codes of one K or V tile
  static constexpr int kRawOff =
      kSplit ? kVOff + kVStages * kKVBytes : kKOff + kKStages * 2 * kKVBytes;
  static constexpr int kEnd = kRawOff + kRawStages * 2 * kRawBytes + 1024;
  // At least half the SM's shared memory, so that one CTA holds the SM's TMEM.
  static constexpr int kSmemBytes = kEnd > 118 * 1024 ? kEnd : 118 * 1024;
  // TMEM columns: S_t[b] (fp32, 64 each) at (2t + b) * 64, then O_t.
  static constexpr uint32_t kOCol = 2 * NT * kBN;
  static_assert(kOCol + NT * D <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448 - 1024, "shared memory budget");
  static_assert(kKStages <= 10 && kVStages <= 10, "ring barriers");
};

__host__ __device__ constexpr uint32_t s_col(int t, int b) { return (uint32_t)((2 * t + b) * kBN); }

struct Bars {
  uint64_t q_full;       // both query tiles loaded
  uint64_t q_empty;      // the item's last S MMAs reading them have completed
  uint64_t k_full[10];   // per K slot: K of one key tile loaded
  uint64_t k_empty[10];  // per K slot: its S MMAs have completed
  uint64_t v_full[10];   // per V slot: V of one key tile loaded
  uint64_t v_empty[10];  // per V slot: its P V MMAs have completed
  uint64_t s_full[2];    // per score buffer: S of every query tile computed
  uint64_t p_full[2];    // per score buffer: P of every tile written (per softmax warp)
  uint64_t pv_item[1];   // one phase per item with two or more key tiles: P(n-2) V done
  uint64_t raw_full[2];  // e4m3: per raw stage, the codes of one key tile loaded
  uint64_t raw_empty[2]; // e4m3: per raw stage, the four converter warps done with it
  uint64_t q_ready[2];   // e4m3, per Q load parity: the Q tiles narrowed to f16 and their
                         // row scales written (one arrival per Q warp)
  uint64_t o_final;      // the item's last P V has completed
  uint64_t o_empty;      // the epilogue has read O (one arrival per softmax warp)
  uint64_t item_full[2];   // work-item ring: index written by the producer
  uint64_t item_empty[2];  // work-item ring: index read by the MMA and softmax warps
  uint64_t drain;
};

// One work item: a pair of query tiles of one (sequence, KV head).
struct Item {
  int b, kvh, q0, q_len, k_len;
  int t_begin;      // first token of tile A
  int j_begin;      // first key tile of the band
  int n_sink;       // attention-sink tiles [0, n_sink), all below j_begin
  int n_tiles;      // sink and band key tiles (0: every row sees no key)
};

// Key tile of entry i of an item's tile list: the sink tiles, then the band.
__device__ __forceinline__ int tile_of(const Item& it, int i) {
  return i < it.n_sink ? i : it.j_begin + (i - it.n_sink);
}

// Decode work item w (items ordered by sequence, then query-pair index
// descending, then KV head). False when the item is empty or the sequence's
// lengths are out of bounds (then RPK_DEVERR_LENGTH is raised once).
__device__ __forceinline__ bool decode_item(const AttnParams& p, int w, int n_qpairs, int span,
                                            bool report, Item& it) {
  const int per_seq = n_qpairs * p.Hk;
  it.b = w / per_seq;
  const int rem = w - it.b * per_seq;
  const int qt = n_qpairs - 1 - rem / p.Hk;
  it.kvh = rem - (rem / p.Hk) * p.Hk;
  it.q0 = __ldg(p.offsets + it.b);
  it.q_len = __ldg(p.offsets + it.b + 1) - it.q0;
  it.k_len = __ldg(p.kv_lens + it.b);
  if (it.q_len > p.max_q_len || it.k_len < 0 || it.k_len > p.max_kv_len) {
    if (report && rem == 0) raise_error(p.error_word, RPK_DEVERR_LENGTH);
    return false;
  }
  it.t_begin = qt * span;
  if (it.t_begin >= it.q_len) return false;
  const int t_end = min(it.q_len, it.t_begin + span);
  const int p_first = it.t_begin + it.k_len - it.q_len;
  const int p_last = (t_end - 1) + it.k_len - it.q_len;
  const int lo_first = p.window > 0 ? max(0, p_first - p.window + 1) : 0;
  const int hi_all = min(p_last, it.k_len - 1);
  it.j_begin = 0;
  it.n_sink = 0;
  it.n_tiles = 0;
  if (hi_all >= lo_first) {
    it.j_begin = lo_first / kBN;
    const int sink_keys = min(p.sinks, lo_first);  // keys below the band that stay visible
    it.n_sink = min((sink_keys + kBN - 1) / kBN, it.j_begin);
    it.n_tiles = it.n_sink + hi_all / kBN + 1 - it.j_begin;
  }
  return true;
}

template <int D, int NT, bool F8>
__global__ void __launch_bounds__(Cfg<D, NT, F8>::kThreads, 1)
    attn_prefill_kernel(const AttnParams p, const __grid_constant__ CUtensorMap q_map,
                        const __grid_constant__ CUtensorMap k_map,
                        const __grid_constant__ CUtensorMap v_map, const int tpt,
                        const int n_qpairs, int* __restrict__ work_counter) {
  using C = Cfg<D, NT, F8>;
  constexpr int KS = C::kKStages, VS = C::kVStages;
  constexpr int RS = C::kRawStages;
  constexpr int kSoftmaxWarps = 4 * NT;
  // MMA warp, softmax warps and, for an e4m3 cache, two Q warps and four
  // converter warps
  constexpr int kItemReaders = 1 + kSoftmaxWarps + (F8 ? 6 : 0);
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  __shared__ int item_slot[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int skip_sh;
  // e4m3: per Q load parity and row, the power-of-two exponent k2 its query
  // row was scaled by when narrowed to f16
  __shared__ int8_t q_k2_sh[F8 ? 2 * NT * kBM : 1];
  volatile int* abort = &abort_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = n_qpairs * p.batch * p.Hk;
  const int G = p.G;
  const int rows_used = tpt * G;
  const int span = NT * tpt;  // tokens per work item

  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  auto q_s = [&](int t) { return sbase + C::kQOff + t * C::kQBytes; };
  auto k_s = [&](int st) { return sbase + C::kKOff + st * C::kKStride; };
  auto v_s = [&](int st) { return sbase + C::kVOff + st * C::kVStride; };

  if (threadIdx.x == 0) {
    for (int st = 0; st < KS; ++st) {
      mbar_init(&bars.k_full[st], F8 ? 4 : 1);  // e4m3: one arrival per converter warp
      mbar_init(&bars.k_empty[st], 1);
    }
    for (int st = 0; st < RS; ++st) {
      mbar_init(&bars.raw_full[st], 1);
      mbar_init(&bars.raw_empty[st], 4);
    }
    for (int k = 0; k < 2; ++k) mbar_init(&bars.q_ready[k], 2);
    for (int st = 0; st < VS; ++st) {
      mbar_init(&bars.v_full[st], 1);
      mbar_init(&bars.v_empty[st], 1);
    }
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.s_full[b], 1);
      mbar_init(&bars.p_full[b], kSoftmaxWarps);
    }
    mbar_init(&bars.pv_item[0], 1);
    mbar_init(&bars.o_final, 1);
    mbar_init(&bars.o_empty, kSoftmaxWarps);
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bars.item_full[k], 1);
      mbar_init(&bars.item_empty[k], kItemReaders);
    }
    mbar_init(&bars.drain, 1);
    abort_sh = 0;
    // Read once and shared, so that every thread takes the same branch below.
    skip_sh = timed_out_elsewhere(p.error_word) ? 1 : 0;
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

  if (skip_sh) {
    // An earlier CTA timed out: free TMEM below and leave.
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (lane == 0) {
      prefetch_tensormap(&q_map);
      prefetch_tensormap(&k_map);
      prefetch_tensormap(&v_map);
      const uint32_t q_box_bytes = 128u * (uint32_t)rows_used;
      const int box_rows = p.P < kBN ? p.P : kBN;
      const uint32_t seg_bytes = (uint32_t)box_rows * 128u * C::kBoxes;
      int kv_issued = 0;  // key tiles whose K and V were loaded, over all items
      int k_issued = 0, v_issued = 0;  // K and V tiles in flight or landed
      int q_loads = 0;    // Q loads over all items
      bool ok = true;
      // Claim a non-empty work item and hand its index to the MMA and softmax
      // warps through the ring. The next item is claimed after the current
      // one's Q and first key tiles are in flight, so the claim's latency hides
      // behind real work.
      auto claim = [&](Item& it) -> int {
        int w;
        do {
          w = atomicAdd(work_counter, 1);
        } while (w < n_items && !decode_item(p, w, n_qpairs, span, true, it));
        return w < n_items ? w : -1;
      };
      auto publish = [&](int seq, int w) -> bool {
        const int slot = seq & 1;
        if (seq >= 2 &&
            !thread_wait(&bars.item_empty[slot], ((seq >> 1) & 1) ^ 1, abort, p.error_word, p.wait_ns))
          return false;
        *reinterpret_cast<volatile int*>(&item_slot[slot]) = w;
        mbar_arrive(&bars.item_full[slot]);
        return true;
      };
      // The Q tiles of an item, once the previous item's S MMAs that read
      // them have completed. Rows past the last token read the fill value.
      auto load_q = [&](const Item& it) -> bool {
        if (q_loads > 0 && !thread_wait(&bars.q_empty, (q_loads - 1) & 1, abort, p.error_word, p.wait_ns))
          return false;
        mbar_arrive_expect_tx(&bars.q_full, NT * C::kBoxes * q_box_bytes);
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(smem + C::kQOff + t * C::kQBytes + bx * (kBM * 128), &q_map, bx * 64,
                        it.kvh * G, it.q0 + it.t_begin + t * tpt, &bars.q_full);
        ++q_loads;
        return true;
      };
      // K and V of key tile i of an item into the next slots of their rings;
      // a K slot frees once the S MMAs that read it have completed, a V slot
      // once the P V MMAs that read it have.
      auto load_stage = [&](const Item& it, int i) -> bool {
        const int32_t* bt = p.block_table + (size_t)it.b * p.max_pages;
        const int gi = kv_issued;
        const int ks = gi % KS, vs = gi % VS;
        const int key0 = tile_of(it, i) * kBN;
        if constexpr (F8) {
          // e4m3 codes of K then V into the next raw stage, rows of D bytes
          const int rs = gi % RS;
          if (gi >= RS && !thread_wait(&bars.raw_empty[rs], ((gi / RS) & 1) ^ 1, abort,
                                       p.error_word, p.wait_ns))
            return false;
          uint32_t cbytes = 0;
          for (int r = 0; r < kBN; r += box_rows) {
            const int key = key0 + r;
            if (key >= it.k_len) break;
            const int pi = key / p.P;
            const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
            if (page >= 0 && page < p.num_pages) cbytes += (uint32_t)box_rows * D;
          }
          mbar_arrive_expect_tx(&bars.raw_full[rs], 2 * cbytes);
          uint8_t* raw = smem + C::kRawOff + rs * 2 * C::kRawBytes;
          for (int r = 0; r < kBN; r += box_rows) {
            const int key = key0 + r;
            if (key >= it.k_len) break;
            const int pi = key / p.P;
            const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
            if (page < 0 || page >= p.num_pages) {
              raise_error(p.error_word, RPK_DEVERR_PAGE);
              continue;
            }
            const int grow = page * p.P + (key - pi * p.P);
            tma_load_3d(raw + r * D, &k_map, 0, it.kvh, grow, &bars.raw_full[rs]);
            tma_load_3d(raw + C::kRawBytes + r * D, &v_map, 0, it.kvh, grow,
                        &bars.raw_full[rs]);
          }
          ++kv_issued;
          ++k_issued;
          return true;
        }
        uint32_t bytes = 0;
        for (int r = 0; r < kBN; r += box_rows) {
          const int key = key0 + r;
          if (key >= it.k_len) break;
          const int pi = key / p.P;
          const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
          if (page >= 0 && page < p.num_pages) bytes += seg_bytes;
        }
        if constexpr (!C::kSplit) {
          // One stage for the tile's K and V: the copies go out box by box as
          // K, V pairs (measured 3% faster than all K boxes, then all V).
          if (gi >= KS &&
              !thread_wait(&bars.k_empty[ks], ((gi / KS) & 1) ^ 1, abort, p.error_word, p.wait_ns))
            return false;
          mbar_arrive_expect_tx(&bars.k_full[ks], 2 * bytes);
          uint8_t* kb = smem + C::kKOff + ks * C::kKStride;
          uint8_t* vb = smem + C::kVOff + ks * C::kVStride;
          for (int r = 0; r < kBN; r += box_rows) {
            const int key = key0 + r;
            if (key >= it.k_len) break;
            const int pi = key / p.P;
            const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
            if (page < 0 || page >= p.num_pages) {
              raise_error(p.error_word, RPK_DEVERR_PAGE);
              continue;
            }
            const int grow = page * p.P + (key - pi * p.P);
#pragma unroll
            for (int bx = 0; bx < C::kBoxes; ++bx) {
              tma_load_3d(kb + r * 128 + bx * (kBN * 128), &k_map, bx * 64, it.kvh, grow,
                          &bars.k_full[ks]);
              tma_load_3d(vb + r * 128 + bx * (kBN * 128), &v_map, bx * 64, it.kvh, grow,
                          &bars.k_full[ks]);
            }
          }
          ++k_issued;
        } else {
          for (int kind = 0; kind < 2; ++kind) {
            const int st = kind == 0 ? ks : vs;
            const int ring = kind == 0 ? KS : VS;
            uint64_t* full = kind == 0 ? &bars.k_full[st] : &bars.v_full[st];
            uint64_t* empty = kind == 0 ? &bars.k_empty[st] : &bars.v_empty[st];
            if (gi >= ring &&
                !thread_wait(empty, ((gi / ring) & 1) ^ 1, abort, p.error_word, p.wait_ns))
              return false;
            mbar_arrive_expect_tx(full, bytes);
            const CUtensorMap* map = kind == 0 ? &k_map : &v_map;
            uint8_t* base = smem + (kind == 0 ? C::kKOff + st * C::kKStride
                                              : C::kVOff + st * C::kVStride);
            for (int r = 0; r < kBN; r += box_rows) {
              const int key = key0 + r;
              if (key >= it.k_len) break;
              const int pi = key / p.P;
              const int page = pi < p.max_pages ? __ldg(bt + pi) : -1;
              if (page < 0 || page >= p.num_pages) {
                if (kind == 0) raise_error(p.error_word, RPK_DEVERR_PAGE);
                continue;
              }
              const int grow = page * p.P + (key - pi * p.P);
#pragma unroll
              for (int bx = 0; bx < C::kBoxes; ++bx)
                tma_load_3d(base + r * 128 + bx * (kBN * 128), map, bx * 64, it.kvh, grow, full);
            }
            ++(kind == 0 ? k_issued : v_issued);
          }
        }
        ++kv_issued;
        return true;
      };
      Item cur;
      int cur_w = claim(cur);
      ok = publish(0, cur_w);
      for (int seq = 0; ok && cur_w >= 0; ++seq) {
        const int n = cur.n_tiles;
        if (n > 0) {
          ok = load_q(cur);
          for (int i = 0; ok && i < n && i < 2; ++i) ok = load_stage(cur, i);
        }
        if (!ok) break;
        Item next;
        const int next_w = claim(next);
        if (!publish(seq + 1, next_w)) { ok = false; break; }
        for (int i = 2; ok && i < n; ++i) ok = load_stage(cur, i);
        if (!ok) break;
        cur = next;
        cur_w = next_w;
      }
      if (!ok) do_abort(abort, p.error_word);
      // Never leave with copies in flight.
      if (q_loads > 0) mbar_wait(&bars.q_full, (q_loads - 1) & 1);
      if constexpr (F8) {
        for (int gi = max(0, k_issued - RS); gi < k_issued; ++gi)
          mbar_wait(&bars.raw_full[gi % RS], (gi / RS) & 1);
      } else {
        for (int gi = max(0, k_issued - KS); gi < k_issued; ++gi)
          mbar_wait(&bars.k_full[gi % KS], (gi / KS) & 1);
      }
      if constexpr (C::kSplit)
        for (int gi = max(0, v_issued - VS); gi < v_issued; ++gi)
          mbar_wait(&bars.v_full[gi % VS], (gi / VS) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    // e4m3 caches: K, V, Q and P are f16 (K and V widened exactly, Q scaled
    // per row by a power of two), bf16 otherwise
    constexpr uint32_t idesc_qk =
        F8 ? tc::idesc_f16_f32(kBM, kBN, 0) : tc::idesc_bf16_f32(kBM, kBN, 0);
    constexpr uint32_t idesc_pv = F8 ? tc::idesc_f16_f32(kBM, D, 1) : tc::idesc_bf16_f32(kBM, D, 1);
    int g_kv = 0;        // key tiles whose K slot has been waited for, over all items
    int g_pv = 0;        // key tiles whose P V has been issued, over all items
    int q_seen = 0;      // Q loads consumed
    int s_issued = 0;    // S tile pairs issued (buffer = count mod 2)
    int o_commits = 0;   // o_final commits
    bool ok = true;
    // Shared-memory descriptors: the start address is the low field of the
    // low word (address >> 4, 14 bits; every operand lies below 256 KB), so
    // the descriptor of an operand at an offset is the base low word plus
    // offset >> 4; the high word (stride offset, swizzle) is common.
    const uint64_t q_desc0 = tc::smem_desc_sw128(q_s(0), 16, 1024);
    const uint32_t q_lo0 = (uint32_t)q_desc0;
    const uint32_t k_lo0 = (uint32_t)tc::smem_desc_sw128(k_s(0), 16, 1024);
    const uint32_t v_lo0 = (uint32_t)tc::smem_desc_sw128(v_s(0), kBN * 128, 1024);
    const uint32_t desc_hi = (uint32_t)(q_desc0 >> 32);
    // S of every query tile for the K tile in slot kst into the next score
    // buffer; the K slot is free once these MMAs complete.
    auto issue_s = [&](int kst) {
      const int b = s_issued & 1;
      if (lane == 0) {
        const uint32_t kd = k_lo0 + (uint32_t)((kst * C::kKStride) >> 4);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t d_tmem = tmem + s_col(t, b);
          const uint32_t qd = q_lo0 + (uint32_t)((t * C::kQBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
            tc::mma_ss_lo(d_tmem, qd + (qoff >> 4), kd + (koff >> 4), desc_hi, idesc_qk, kk > 0);
          }
        }
        tc::commit(smem_u32(&bars.s_full[b]));
        if constexpr (C::kSplit) tc::commit(smem_u32(&bars.k_empty[kst]));
      }
      __syncwarp();
      ++s_issued;
    };
    // O_t (+)= P_t V for every tile, P_t in the first 32 columns of buffer b.
    auto issue_pv = [&](int vst, int b, bool first) {
      if (lane == 0) {
        const uint32_t vd = v_lo0 + (uint32_t)((vst * C::kVStride) >> 4);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t d_tmem = tmem + C::kOCol + (uint32_t)(t * D);
          const uint32_t a_tmem = tmem + s_col(t, b);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            tc::mma_ts_lo(d_tmem, a_tmem + kk * 8, vd + (uint32_t)((kk * (16 * 128)) >> 4),
                          desc_hi, idesc_pv, (!first || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto commit_to = [&](uint64_t* bar) {
      if (lane == 0) tc::commit(smem_u32(bar));
      __syncwarp();
    };
    auto wait_stage = [&]() -> bool {
      if (!warp_wait(&bars.k_full[g_kv % KS], (g_kv / KS) & 1, abort, p.error_word, p.wait_ns))
        return false;
      ++g_kv;
      return true;
    };
    for (int seq = 0; ok; ++seq) {
      const int slot = seq & 1;
      if (!warp_wait(&bars.item_full[slot], (seq >> 1) & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      const int w = *reinterpret_cast<volatile int*>(&item_slot[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
      if (w < 0) break;
      Item it;
      if (!decode_item(p, w, n_qpairs, span, false, it) || it.n_tiles == 0) continue;
      const int n = it.n_tiles;
      ok = F8 ? warp_wait(&bars.q_ready[q_seen & 1], (q_seen >> 1) & 1, abort, p.error_word,
                          p.wait_ns)
              : warp_wait(&bars.q_full, q_seen & 1, abort, p.error_word, p.wait_ns);
      ++q_seen;
      // S(0), S(1)
      for (int j = 0; ok && j < n && j < 2; ++j) {
        const int kst = g_kv % KS;
        if (!wait_stage()) { ok = false; break; }
        tc::fence_after_sync();
        issue_s(kst);
        if (j + 1 == n) commit_to(&bars.q_empty);  // last S of this item
      }
      for (int i = 0; ok && i < n; ++i) {
        const int vst = g_pv % VS;
        const int pb = g_pv & 1;
        // P(i) of every tile written and the K (unified: the stage) of key
        // tile i+2 (for S(i+2)) loaded; split rings also wait for the V of
        // key tile i here (a unified stage was waited for with its S)
        const bool more_s = i + 2 < n;
        const int kst = more_s ? g_kv % KS : -1;
        bool waited =
            more_s ? warp_wait2(&bars.p_full[pb], (g_pv >> 1) & 1, &bars.k_full[g_kv % KS],
                                (g_kv / KS) & 1, abort, p.error_word, p.wait_ns)
                   : warp_wait(&bars.p_full[pb], (g_pv >> 1) & 1, abort, p.error_word,
                               p.wait_ns);
        if constexpr (C::kSplit)
          waited = waited &&
                   warp_wait(&bars.v_full[vst], (g_pv / VS) & 1, abort, p.error_word, p.wait_ns);
        if (!waited) {
          ok = false;
          break;
        }
        if (more_s) ++g_kv;
        const int key0 = tile_of(it, i) * kBN;
        if (key0 + kBN > it.k_len) {
          // zero value rows at or past k_len (the V slot was waited for above)
          const int r0 = max(0, it.k_len - key0);
          const int chunks = (kBN - r0) * C::kBoxes * 8;
          for (int idx = lane; idx < chunks; idx += 32) {
            const int ch = idx & 7;
            const int rb = idx >> 3;
            const int bx = rb % C::kBoxes;
            const int r = r0 + rb / C::kBoxes;
            uint8_t* dst = smem + C::kVOff + vst * C::kVStride + bx * (kBN * 128) + r * 128 +
                           ch * 16;
            *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (i == 0 && o_commits > 0) {
          // O of the previous item has been read by its epilogue.
          if (!warp_wait(&bars.o_empty, (o_commits - 1) & 1, abort, p.error_word, p.wait_ns)) {
            ok = false;
            break;
          }
        }
        tc::fence_after_sync();
        issue_pv(vst, pb, i == 0);
        ++g_pv;
        if (i + 2 == n) commit_to(&bars.pv_item[0]);  // P(n-2) V done: last-tile rescales
        if (i + 1 == n) {
          commit_to(&bars.o_final);
          ++o_commits;
        }
        // the V slot (unified: the whole stage) is free once P(i) V_i completes
        commit_to(C::kSplit ? &bars.v_empty[vst] : &bars.k_empty[vst]);
        if (kst >= 0) {
          // S(i+2) overwrites the buffer P(i) lives in; the MMAs run in issue
          // order, so P(i) V_i has read it by then.
          issue_s(kst);
          if (i + 3 == n) commit_to(&bars.q_empty);  // last S of this item
        }
      }
    }
    if (!ok) do_abort(abort, p.error_word);
    // Drain: every MMA issued above has completed before TMEM is freed.
    commit_to(&bars.drain);
    if (!warp_wait(&bars.drain, 0, abort, p.error_word, p.wait_ns)) mbar_wait(&bars.drain, 0);
  } else if (warp < 4 || warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if constexpr (F8) {
      // --------------------------------------- e4m3: Q warps and converters
      // Warps 2 and 3: at the start of each item with keys, warp 2 + t
      // narrows query tile t to f16 in place. Each row is scaled by the power
      // of two 2^k2 that brings its largest magnitude into [2^14, 2^15) (exact
      // for every element above f16's normal range floor: bf16 has 8
      // significant bits, f16 11), and k2 is left for the softmax warps, which
      // fold 2^-k2 and k_scale into the score scale and v_scale into the output.
      // Warps 12-15: warp 12 + 2 kind + h widens rows [32 h, 32 h + 32) of
      // the K (kind 0) or V (kind 1) codes of each key tile from its raw stage
      // into the f16 stage the MMAs read (every e4m3 value is exact in f16),
      // in the 128-byte-swizzled layout TMA would have written.
      const bool q_warp = warp < 4;
      const int role = q_warp ? warp - 2 : warp - 12;
      int gi = 0;                 // key tiles converted over all items
      int ql = 0;                 // Q loads narrowed
      bool ok = true;
      auto narrow_q = [&]() {
        uint8_t* qtile = smem + C::kQOff + role * C::kQBytes;
        int8_t* k2s = q_k2_sh + (ql & 1) * (NT * kBM) + role * kBM;
        for (int r = lane; r < rows_used; r += 32) {
          float mx = 0.f;
#pragma unroll
          for (int ch = 0; ch < D / 8; ++ch) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(
                qtile + (ch >> 3) * (kBM * 128) + swz128((uint32_t)r, (uint32_t)(ch & 7)));
            const uint32_t wds[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f =
                  __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wds[k]));
              mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
          }
          const int e = (int)((__float_as_uint(mx) >> 23) & 0xFFu) - 127;  // floor(log2 mx)
          int k2 = (mx > 0.f && mx < INFINITY) ? 14 - e : 0;
          k2 = max(-126, min(126, k2));
          k2s[r] = (int8_t)k2;
          const float up = __uint_as_float((uint32_t)(127 + k2) << 23);
#pragma unroll
          for (int ch = 0; ch < D / 8; ++ch) {
            uint4* cp = reinterpret_cast<uint4*>(
                qtile + (ch >> 3) * (kBM * 128) + swz128((uint32_t)r, (uint32_t)(ch & 7)));
            const uint4 w4 = *cp;
            const uint32_t wds[4] = {w4.x, w4.y, w4.z, w4.w};
            uint32_t o4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f =
                  __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wds[k]));
              o4[k] = pack_f16x2(f.x * up, f.y * up);
            }
            *cp = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
        }
        fence_proxy_async_smem();  // generic writes before the MMAs read Q
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.q_ready[ql & 1]);
        ++ql;
      };
      // Rows [32 h, 32 h + 32) of the K or V codes of key tile gi.
      auto widen = [&](int kind, int h) {
        const int rs = gi % RS, st = gi % KS;
        const uint8_t* raw = smem + C::kRawOff + rs * 2 * C::kRawBytes + kind * C::kRawBytes;
        uint8_t* dst = smem + (kind == 0 ? C::kKOff + st * C::kKStride
                                         : C::kVOff + st * C::kVStride);
        constexpr int kChunks = (kBN / 2) * (D / 8);  // 8 codes -> 16 bytes of f16
#pragma unroll 4
        for (int c = lane; c < kChunks; c += 32) {
          const int row = 32 * h + c / (D / 8), c8 = c % (D / 8);
          const uint2 w8 = *reinterpret_cast<const uint2*>(raw + row * D + c8 * 8);
          uint4 hv;
          hv.x = f16x2_from_e4m3x2(w8.x & 0xFFFFu);
          hv.y = f16x2_from_e4m3x2(w8.x >> 16);
          hv.z = f16x2_from_e4m3x2(w8.y & 0xFFFFu);
          hv.w = f16x2_from_e4m3x2(w8.y >> 16);
          *reinterpret_cast<uint4*>(dst + (c8 >> 3) * (kBN * 128) +
                                    swz128((uint32_t)row, (uint32_t)(c8 & 7))) = hv;
        }
        fence_proxy_async_smem();  // generic writes before the MMAs read them
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.k_full[st]);
          mbar_arrive(&bars.raw_empty[rs]);
        }
      };
      for (int seq = 0; ok; ++seq) {
        const int slot = seq & 1;
        if (!warp_wait(&bars.item_full[slot], (seq >> 1) & 1, abort, p.error_word, p.wait_ns)) {
          ok = false;
          break;
        }
        const int w = *reinterpret_cast<volatile int*>(&item_slot[slot]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
        if (w < 0) break;
        Item it;
        if (!decode_item(p, w, n_qpairs, span, false, it)) continue;
        if (q_warp) {
          if (it.n_tiles > 0) {
            if (!warp_wait(&bars.q_full, ql & 1, abort, p.error_word, p.wait_ns)) {
              ok = false;
              break;
            }
            narrow_q();
          }
          continue;
        }
        for (int i = 0; ok && i < it.n_tiles; ++i, ++gi) {
          const int rs = gi % RS, st = gi % KS;
          if (!warp_wait(&bars.raw_full[rs], (gi / RS) & 1, abort, p.error_word, p.wait_ns) ||
              (gi >= KS && !warp_wait(&bars.k_empty[st], ((gi / KS) & 1) ^ 1, abort,
                                      p.error_word, p.wait_ns))) {
            ok = false;
            break;
          }
          widen(role >> 1, role & 1);
        }
      }
      if (!ok) do_abort(abort, p.error_word);
    }
  } else {
    // ------------------------------------------------------------- softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegsSoftmax));
    const int t = (warp - 4) >> 2;       // query tile: warps 4-7 -> A, 8-11 -> B (if NT == 2)
    const int qw = warp & 3;             // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;        // row of this thread
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    const uint32_t o_col = tmem + lane_base + C::kOCol + (uint32_t)(t * D);
    float sl2 = p.scale_log2;  // e4m3: times k_scale and the row's Q scale, per item
    int q_seen_sm = 0;         // e4m3: Q loads consumed
    int s_seen = 0;      // score tiles consumed over all items
    int o_seen = 0;      // items with keys consumed
    int pv_items = 0;    // items with two or more key tiles consumed
    bool ok = true;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    // With one query tile per item the second softmax warpgroup has no rows.
    for (int seq = 0; ok && t < NT; ++seq) {
      const int slot = seq & 1;
      if (!warp_wait(&bars.item_full[slot], (seq >> 1) & 1, abort, p.error_word, p.wait_ns)) {
        ok = false;
        break;
      }
      const int w = *reinterpret_cast<volatile int*>(&item_slot[slot]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
      if (w < 0) break;
      Item it;
      if (!decode_item(p, w, n_qpairs, span, false, it)) continue;
      const int tok = it.t_begin + t * tpt + r / G;
      const bool row_ok = r < rows_used && tok < it.q_len;
      const int pos = tok + it.k_len - it.q_len;
      const int lo = p.window > 0 ? pos - p.window + 1 : 0;
      const int hi = pos;
      const int n = it.n_tiles;
      float m = -INFINITY, l = 0.f;      // running max (log2 units) and sum
      float v_mul = 1.f;                 // e4m3: v_scale of the item's KV head
      if constexpr (F8) {
        if (n > 0) {
          // A Q warp narrowed this row's query to f16 under 2^k2.
          const int qs = q_seen_sm++;
          if (!warp_wait(&bars.q_ready[qs & 1], (qs >> 1) & 1, abort, p.error_word, p.wait_ns)) {
            ok = false;
            break;
          }
          const int k2 = r < rows_used ? (int)q_k2_sh[(qs & 1) * (NT * kBM) + t * kBM + r] : 0;
          const float down = __uint_as_float((uint32_t)(127 - k2) << 23);
          sl2 = p.scale_log2 * __ldg(p.k_scale + it.kvh) * down;
          v_mul = __ldg(p.v_scale + it.kvh);
        }
      }
      // The tile loop, compiled twice: without attention sinks (the common
      // case keeps the plain single-interval mask) and with them.
      auto tile_loop = [&](auto with_sinks) {
        constexpr bool kSinks = decltype(with_sinks)::value;
        float v[kBN];
        for (int i = 0; i < n; ++i) {
          const int b = s_seen & 1;
          if (!warp_wait(&bars.s_full[b], (s_seen >> 1) & 1, abort, p.error_word, p.wait_ns)) {
            ok = false;
            break;
          }
          const int gt = s_seen++;  // this tile's index over all items
          tc::fence_after_sync();
          const uint32_t sc = tmem + lane_base + s_col(t, b);
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c) tc::tmem_ld32(sc + c * 32, v + c * 32);
          tc::tmem_wait_ld();
          const int key0 = tile_of(it, i) * kBN;
          if constexpr (!kSinks) {
            if (!(row_ok && key0 >= lo && key0 + kBN - 1 <= hi)) {
              // visible columns [c_lo, c_hi] of this tile (empty for an invalid row)
              const int c_lo = row_ok ? lo - key0 : kBN;
              const int c_hi = row_ok ? hi - key0 : -1;
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c < c_lo || c > c_hi) v[c] = -INFINITY;
            }
          } else {
            // Visible columns: the window's [c_lo, c_hi] and the sinks below
            // c_sink (none for an invalid row). The sinks either join the window
            // (c_sink >= c_lo: one interval from 0) or lie below it.
            int c_lo = row_ok ? lo - key0 : kBN;
            const int c_hi = row_ok ? hi - key0 : -1;
            const int c_sink = p.sinks - key0;
            if (c_sink >= c_lo) c_lo = 0;
            if (c_sink > 0 && c_sink < c_lo) {
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c > c_hi || (c < c_lo && c >= c_sink)) v[c] = -INFINITY;
            } else if (c_lo > 0 || c_hi < kBN - 1) {
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c < c_lo || c > c_hi) v[c] = -INFINITY;
            }
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
          // more than the threshold (then O and l are rescaled).
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
          float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // independent partial sums
          uint32_t pk[kBN / 2];
#pragma unroll
          for (int c = 0; c < kBN; c += 2) {
            float x0, x1;
            fma2(x0, x1, v[c], v[c + 1], sl2, neg_m);
            const float w0 = fast_exp2(x0);
            const float w1 = fast_exp2(x1);
            const int k = (c >> 1) & 3;
            add2(rs[2 * k], rs[2 * k + 1], w0, w1);
            pk[c >> 1] = F8 ? pack_f16x2(w0, w1) : pack_bf16x2(w0, w1);
          }
          tc::tmem_st32(sc, reinterpret_cast<const float*>(pk));
          l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
          // Rescale O_t after P(i-1) V_{i-1} has completed and before P(i) V_i
          // is issued (before p_full): proven by S(i+1), or for the item's
          // last tile by the per-item barrier (see the header).
          if (i > 0 && __any_sync(0xffffffffu, rescale)) {
            const bool waited =
                i + 1 < n
                    ? warp_wait(&bars.s_full[(gt + 1) & 1], ((gt + 1) >> 1) & 1, abort,
                                p.error_word, p.wait_ns)
                    : warp_wait(&bars.pv_item[0], pv_items & 1, abort, p.error_word, p.wait_ns);
            if (!waited) {
              tc::tmem_wait_st();  // no store of P may be in flight when TMEM is freed
              ok = false;
              break;
            }
            tc::fence_after_sync();
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
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.p_full[b]);
        }
      };
      if (p.sinks > 0) tile_loop(std::true_type{});
      else tile_loop(std::false_type{});
      if (!ok) break;
      if (n >= 2) ++pv_items;
      // ---------------------------------------------------------- epilogue
      const bool have_o = n > 0;
      if (have_o) {
        if (!warp_wait(&bars.o_final, o_seen & 1, abort, p.error_word, p.wait_ns)) { ok = false; break; }
        ++o_seen;
        tc::fence_after_sync();
      }
      const float inv = (l > 0.f) ? v_mul / l : 0.f;
      const size_t hrow = (size_t)(it.q0 + tok) * p.H + (size_t)it.kvh * G + (r % G);
      const size_t orow = hrow * D;
      // l is relative to the (possibly stale) running max m, so m + log2 l is exact.
      if (p.lse != nullptr && row_ok) p.lse[hrow] = lse_from_log2_state(m, l);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        if (have_o) {
          tc::tmem_ld32(o_col + c * 32, o);
          tc::tmem_wait_ld();
          if (c + 1 == D / 32) {
            // O may now be overwritten by the next item's first P V.
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.o_empty);
          }
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
    if (!ok) do_abort(abort, p.error_word);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

int sm_count() {
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

template <int D, int NT, bool F8>
cudaError_t launch_d(const AttnParams& p, const CUtensorMap& q_map, const CUtensorMap& k_map,
                     const CUtensorMap& v_map, int* work_counter, cudaStream_t stream) {
  using C = Cfg<D, NT, F8>;
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<D, NT, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int tpt = prefill_rows_per_tile(p.G);
  const int n_qpairs = (p.max_q_len + NT * tpt - 1) / (NT * tpt);  // work items per (seq, head)
  const long long n_items = (long long)n_qpairs * p.batch * p.Hk;
  if (n_items == 0) return cudaSuccess;
  // Every CTA claims once past the last item, so the counter reaches n_items + grid.
  if (n_items > INT32_MAX - 65536) return cudaErrorInvalidValue;
  // Persistent: one CTA per SM; CTAs claim items from a counter the call zeroes.
  e = cudaMemsetAsync(work_counter, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<long long>(n_items, sm_count());
  attn_prefill_kernel<D, NT, F8><<<grid, C::kThreads, C::kSmemBytes, stream>>>(
      p, q_map, k_map, v_map, tpt, n_qpairs, work_counter);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnParams& p, const CUtensorMap& q_map,
                                const CUtensorMap& k_map, const CUtensorMap& v_map,
                                int* work_counter, cudaStream_t stream) {
  if ((long long)p.T * p.H == 0 || p.batch == 0) return cudaSuccess;
  if (work_counter == nullptr) return cudaErrorInvalidValue;
  if (p.cache_fp8) {
    switch (p.d) {
      case 64: return launch_d<64, 2, true>(p, q_map, k_map, v_map, work_counter, stream);
      case 128: return launch_d<128, 2, true>(p, q_map, k_map, v_map, work_counter, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.d) {
    case 64: return launch_d<64, 2, false>(p, q_map, k_map, v_map, work_counter, stream);
    case 128: return launch_d<128, 2, false>(p, q_map, k_map, v_map, work_counter, stream);
    case 256: return launch_d<256, 1, false>(p, q_map, k_map, v_map, work_counter, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rpk

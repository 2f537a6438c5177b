// Lightning indexer with the top-k selection fused into its epilogue (page
// "DeepseekV3.2 拆解", section "核心组件 / 闪电索引器", eq. I_{t,s}, and section
// "细粒度 Token 选择机制": keep the k keys with the largest I[t,s]; ties to
// the lower key index).
//
// The score of every (query row, key) pair is formed exactly as in
// indexer_scores_kernel (same MMA tiling, same fp32 operation order) but never
// leaves the SM: each row keeps a candidate buffer (order key, key index) in
// shared memory.
//   * A score is appended only if its order key u passes the row's threshold:
//     u > tau, or u == tau with a key index <= tau_idx.
//   * Every CHECK_TILES (2) tiles, a buffer close to full is shrunk: 128 sampled
//     entries are ranked by comparison, and one counting pass over the buffer
//     finds the highest of 8 sample pivots with at least k entries at or
//     above it. Entries below that pivot are beaten by k others and are
//     dropped; the pivot becomes tau. If that frees too little (many equal
//     scores), the buffer is cut to exactly its k largest entries (below),
//     and tau, tau_idx become the k-th key and the largest index kept among
//     keys equal to it.
//   * After the last key tile the k largest entries are selected exactly: the
//     pivots bound a narrow band of the buffer, an MSB-first radix select
//     finds the k-th key u* inside the band, and if u* is tied a second radix
//     select over the key indices keeps the lowest ones.
// tau never exceeds the k-th largest score seen so far, hence never the final
// one, and every dropped entry is beaten by k entries that stay: the result is
// the exact top-k with ties to the lower index. Keys arrive in increasing
// index order, so a key equal to tau with an index above tau_idx loses the tie
// to every entry kept.
//
// Tile: a CTA owns QG = 4 consecutive query rows and all of their visible key
// tiles; CTAs are issued longest rows first. Sixteen epilogue warps, four per
// SM sub-partition: warps 2-5 own row 0, 6-9 row 1, 10-13 row 2, 14-17 row 3
// (one TMEM lane quarter each).
#pragma once

#include "layout.cuh"
#include "ptx.cuh"

namespace dsa {

struct IndexerTopkParams {
  const float* q_scale;   // [B, n_q, HI]
  const float* w;         // [B, n_q, HI]
  const float* k_scale;   // [pool rows] (contiguous: [B, n_kv])
  RowPos rp;              // absolute position of each query row
  KeyMap km;              // pool row of each key
  const int32_t* kv_len;  // [B] or null
  int32_t* indices;       // row r of sequence b -> indices[(b * out_rows + r - row_begin) * k]
  int32_t B, n_q, n_kv, k;
  int32_t row_begin, rows;     // rows [row_begin, row_begin + rows) of every sequence
  int32_t n_groups;            // ceil(rows / QG)
  int32_t out_rows;
};

template <int HI, int DI, int QG>
struct IndexerTopkTile {
  static_assert(HI == 64 && DI == 128 && QG == 4, "fused selection is built for H^I=64, d^I=128");
  static constexpr int M = 128;                 // keys per tile (TMEM lanes)
  static constexpr int N = QG * HI;             // MMA N
  static constexpr int STAGES = 3;
  static constexpr int K_BYTES = M * DI;
  static constexpr int Q_BYTES = N * DI;
  static constexpr int EPI_WARPS = 16;          // four per SM sub-partition
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr int QPW = 1;                 // rows per epilogue warp group
  static constexpr int GROUPS = EPI_WARPS / 4;  // one group of four warps per row
  static constexpr uint32_t SWIZZLE = 2u;       // 128-byte rows
  static constexpr uint32_t SBO = 8 * DI;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int CAP = 4352;              // candidates per row
  static constexpr int CHECK_TILES = 2;         // buffers are checked every 2 tiles
  static constexpr int HEADROOM = CHECK_TILES * M;
  static constexpr int MAX_K = 2048;
  static_assert(QPW * GROUPS == QG, "one row per warp group");
  static_assert(MAX_K + HEADROOM < CAP, "a compacted buffer must leave room for the next tiles");
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_COEF = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_CU = OFF_COEF + QG * HI * 4;        // [QG][CAP] order keys
  static constexpr int OFF_CI = OFF_CU + QG * CAP * 4;         // [QG][CAP] key indices
  static constexpr int OFF_SEL = OFF_CI + QG * CAP * 4;        // [2] SelState
  static constexpr int SEL_BYTES = 2048;
  static constexpr int OFF_BAR = OFF_SEL + GROUPS * SEL_BYTES;
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 4;          // q, stages, acc
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(OFF_K % 1024 == 0 && K_BYTES % 1024 == 0, "1024-byte aligned operands");
};

// Selection state of one warp group (two rows).
struct __align__(16) SelState {
  uint32_t hist[256];
  uint32_t samp[128];     // sampled keys (pivot selection)
  uint32_t piv[8];        // pivots, descending
  uint32_t cnt[4][8];     // per-warp pivot counts
  uint32_t wtot[2][4];    // per-warp kept counts of a compaction chunk (double-buffered)
  uint32_t wmin[4], wmax[4];
  uint32_t count[2];      // candidates per row
  uint32_t tau[2];        // append threshold per row (order key) ...
  uint32_t tau_idx[2];    // ... and, for keys equal to tau, the largest index still taken
  uint32_t sel_bin, above, bin_count;
};
static_assert(sizeof(SelState) <= 2048, "selection state");

// Order-preserving map of a float score to uint32 (-0 folded into +0).
__device__ __forceinline__ uint32_t score_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The four warps (128 threads) that own two rows of a CTA's query group.
// They synchronise on a named barrier of their own: the epilogue never leaves
// its loops early (after a bounded wait has run out it skips the remaining
// waits but still reaches every barrier), so the four warps always arrive
// together and the barrier cannot wait forever.
struct SelGroup {
  SelState* st;
  uint32_t bar_id;      // named barrier of the group (1 or 2; 0 is __syncthreads)
  int gt, gw, lane;     // thread in group, warp in group, lane

  // Shared-memory writes before it are visible to the group after it.
  __device__ __forceinline__ void sync() {
    asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
  }

  // k-th largest (1-based) of key(i) over the entries i < n with pred(i)
  // (at least k of them): returns u*; *need = how many entries equal to u*
  // belong to the k largest, *eq = how many entries equal u*. All 128
  // threads call this.
  //
  // MSB-first radix select that starts below the bits all participating keys
  // share (from their minimum and maximum), so that the first digit already
  // spreads the keys over the 256 bins and the plain shared-memory atomics of
  // the histogram rarely collide.
  template <class Key, class Pred>
  __device__ __forceinline__ uint32_t kth_largest(int n, uint32_t k, Key key, Pred pred, uint32_t* need,
                                  uint32_t* eq) {
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll 4
    for (int i = gt; i < n; i += 128) {
      if (pred(i)) {
        const uint32_t u = key(i);
        lo = min(lo, u);
        hi = max(hi, u);
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      st->wmin[gw] = lo;
      st->wmax[gw] = hi;
    }
    sync();
    lo = min(min(st->wmin[0], st->wmin[1]), min(st->wmin[2], st->wmin[3]));
    hi = max(max(st->wmax[0], st->wmax[1]), max(st->wmax[2], st->wmax[3]));
    uint32_t want = k, e = 0;
    if (lo == hi) {   // every participating key is equal
      e = 0;
      for (int i = gt; i < n; i += 128) e += pred(i) ? 1u : 0u;
      e = __reduce_add_sync(0xffffffffu, e);
      sync();   // every thread has read wmin/wmax before they are rewritten
      if (lane == 0) st->wmin[gw] = e;
      sync();
      *need = want;
      *eq = st->wmin[0] + st->wmin[1] + st->wmin[2] + st->wmin[3];
      sync();
      return lo;
    }
    int top = 31 - __clz(lo ^ hi);                        // highest differing bit
    uint32_t mask = top == 31 ? 0u : ~((2u << top) - 1u); // bits shared by all keys
    uint32_t prefix = lo & mask;
    for (; top >= 0; top -= 8) {
      const int shift = max(0, top - 7);
      const uint32_t dmask = (2u << (top - shift)) - 1u;  // digit = bits [shift, top]
      st->hist[gt] = 0;
      st->hist[gt + 128] = 0;
      sync();
      for (int c0 = 0; c0 < n; c0 += 128 * 8) {
        uint32_t bins[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int i = c0 + gt + 128 * m;
          bins[m] = 256u;
          if (i < n && pred(i)) {
            const uint32_t u = key(i);
            if ((u & mask) == prefix) bins[m] = (u >> shift) & dmask;
          }
        }
#pragma unroll
        for (int m = 0; m < 8; ++m)
          if (bins[m] < 256u) atomicAdd(&st->hist[bins[m]], 1u);
      }
      sync();
      if (gw == 0) {
        // bins in descending order: lane l owns bins 255 - 8l .. 248 - 8l
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = st->hist[255 - (lane * 8 + j)];
          sum += c[j];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - sum;
        if (excl < want && want <= incl) {
          uint32_t acc = excl;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (acc < want && want <= acc + c[j]) {
              st->sel_bin = 255u - (lane * 8 + j);
              st->above = acc;
              st->bin_count = c[j];
            }
            acc += c[j];
          }
        }
      }
      sync();
      want -= st->above;
      e = st->bin_count;
      prefix |= st->sel_bin << shift;
      mask |= dmask << shift;
    }
    *need = want;
    *eq = e;
    return prefix;
  }

  // Thresholds from a sample of the buffer, without atomics. 128 evenly
  // spaced entries are ranked by comparison; the samples at 8 ranks around
  // the expected rank of the k-th largest become pivots p_0 >= ... >= p_7 and
  // one pass counts C_i = #{entries >= p_i}. Returns lo with C(lo) >= k
  // (the highest such pivot, else 0 with C = n) and hi with C(hi) < k (the
  // next higher pivot, if any: has_hi, with c_hi counting the entries >= hi;
  // c_hi = 0 without one). Every entry >= hi is among the k largest; every
  // entry < lo is beaten by at least k others.
  __device__ __forceinline__ void pivots(const uint32_t* cu, int n, uint32_t k, uint32_t* lo, uint32_t* hi,
                         bool* has_hi, uint32_t* c_lo, uint32_t* c_hi) {
    st->samp[gt] = cu[static_cast<int>((static_cast<int64_t>(gt) * n) >> 7)];
    sync();
    // Rank of this thread's sample among the 128 (descending; equal keys in
    // slot order): four independent partial counts over 64-bit keys
    // (key << 7 | slot), which are all distinct.
    const uint32_t mine = st->samp[gt];
    const uint64_t me = (static_cast<uint64_t>(mine) << 7) | static_cast<uint32_t>(gt);
    uint32_t r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    const uint32_t sv = smem_u32(st->samp);
#pragma unroll 4
    for (int j4 = 0; j4 < 32; ++j4) {
      const uint4 v = lds_v4(sv + 16 * j4);
      const uint64_t b = static_cast<uint64_t>(4 * j4);
      r0 += ((static_cast<uint64_t>(v.x) << 7) | b) > me ? 1u : 0u;
      r1 += ((static_cast<uint64_t>(v.y) << 7) | (b + 1)) > me ? 1u : 0u;
      r2 += ((static_cast<uint64_t>(v.z) << 7) | (b + 2)) > me ? 1u : 0u;
      r3 += ((static_cast<uint64_t>(v.w) << 7) | (b + 3)) > me ? 1u : 0u;
    }
    const uint32_t rank = r0 + r1 + r2 + r3;
    // expected sample rank of the k-th largest entry, then a widening ladder
    const int t0 = static_cast<int>((static_cast<int64_t>(k) * 128) / n);
    constexpr int kStep[8] = {-4, -1, 2, 5, 9, 14, 22, 200};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = min(127, max(0, t0 + kStep[i]));
      if (static_cast<int>(rank) == r) st->piv[i] = mine;
    }
    sync();
    uint32_t pv[8], c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pv[i] = st->piv[i];
      c[i] = 0;
    }
#pragma unroll 4
    for (int j = gt; j < n; j += 128) {
      const uint32_t v = cu[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] += v >= pv[i] ? 1u : 0u;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = __reduce_add_sync(0xffffffffu, c[i]);
      if (lane == 0) st->cnt[gw][i] = c[i];
    }
    sync();
    *lo = 0u;
    *c_lo = static_cast<uint32_t>(n);
    *hi = 0u;
    *has_hi = false;
    *c_hi = 0u;
    bool found = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t ci = st->cnt[0][i] + st->cnt[1][i] + st->cnt[2][i] + st->cnt[3][i];
      if (!found && ci >= k) {
        found = true;
        *lo = pv[i];
        *c_lo = ci;
      } else if (!found) {
        *hi = pv[i];
        *has_hi = true;
        *c_hi = ci;
      }
    }
    sync();   // cnt and piv are reused by the next call
  }

  // Keep the entries for which keep(u, idx) holds, in place, in order of
  // 512-entry chunks: every thread reads its four entries before the group
  // barrier and writes after it, and a kept entry never moves past the end of
  // its own chunk, so no entry is overwritten before it is read. With out
  // set, the kept indices go to out[0, count) instead. Returns the count.
  template <class Keep>
  __device__ __forceinline__ uint32_t compact(uint32_t* cu, int32_t* ci, int n, Keep keep_fn, int32_t* out) {
    uint32_t base = 0;
    int buf = 0;
    for (int c0 = 0; c0 < n; c0 += 512) {
      uint32_t u[4];
      int32_t ix[4];
      uint32_t keep = 0, mine = 0;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = c0 + gt + 128 * m;
        u[m] = 0u;
        ix[m] = -1;
        if (i < n) {
          u[m] = cu[i];
          ix[m] = ci[i];
          if (keep_fn(u[m], ix[m])) {
            keep |= 1u << m;
            ++mine;
          }
        }
      }
      uint32_t incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) st->wtot[buf][gw] = incl;
      sync();
      uint32_t pos = base + incl - mine, total = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t t = st->wtot[buf][w];
        if (w < gw) pos += t;
        total += t;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        if (keep & (1u << m)) {
          if (out) {
            out[pos] = ix[m];
          } else {
            cu[pos] = u[m];
            ci[pos] = ix[m];
          }
          ++pos;
        }
      }
      base += total;
      buf ^= 1;
    }
    sync();
    return base;
  }

  // Mid-scan: drop every entry beaten by at least k others (those below the
  // sample threshold lo). Returns the new count; *tau = lo.
  __device__ __forceinline__ uint32_t shrink(uint32_t* cu, int32_t* ci, int n, uint32_t k, uint32_t* tau) {
    uint32_t lo, hi, c_lo, c_hi;
    bool has_hi;
    pivots(cu, n, k, &lo, &hi, &has_hi, &c_lo, &c_hi);
    *tau = lo;
    if (c_lo == static_cast<uint32_t>(n)) return c_lo;   // nothing to drop
    return compact(cu, ci, n, [lo](uint32_t u, int32_t) { return u >= lo; }, nullptr);
  }

  // The k largest entries, ties to the lower key index: their indices go to
  // out[0, k), or with out == nullptr the buffer is compacted to them. Entries
  // >= hi are in; the exact selection runs on the band [lo, hi). Returns the
  // k-th key u* in *kth and the largest index taken among keys equal to u* in
  // *idx_star (0xffffffff when all of them are taken). Requires n > k.
  __device__ __forceinline__ void select(uint32_t* cu, int32_t* ci, int n, uint32_t k, int32_t* out,
                         uint32_t* kth_out, uint32_t* idx_star_out) {
    uint32_t lo, hi, c_lo, c_hi;
    bool has_hi;
    pivots(cu, n, k, &lo, &hi, &has_hi, &c_lo, &c_hi);
    uint32_t need, eq, idx_star = 0xffffffffu;
    const uint32_t kth =
        kth_largest(n, k - c_hi, [&](int i) { return cu[i]; },
                    [&](int i) { return cu[i] >= lo && (!has_hi || cu[i] < hi); }, &need, &eq);
    if (need < eq) {
      uint32_t n2, e2;
      idx_star = ~kth_largest(n, need, [&](int i) { return ~static_cast<uint32_t>(ci[i]); },
                              [&](int i) { return cu[i] == kth; }, &n2, &e2);
    }
    const auto keep = [kth, idx_star](uint32_t u, int32_t ix) {
      return u > kth || (u == kth && static_cast<uint32_t>(ix) <= idx_star);
    };
    if (out) {
      // Emit in any order: one pass, slots from warp-aggregated atomics.
      if (gt == 0) st->above = 0;
      sync();
#pragma unroll 4
      for (int c0 = 0; c0 < n; c0 += 128) {
        const int i = c0 + gt;
        const bool take = i < n && keep(cu[i], ci[i]);
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        uint32_t base = 0;
        if (lane == 0 && bal) base = atomicAdd(&st->above, static_cast<uint32_t>(__popc(bal)));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (take) out[base + __popc(bal & ((1u << lane) - 1u))] = ci[i];
      }
      sync();
    } else {
      compact(cu, ci, n, keep, nullptr);
    }
    *kth_out = kth;
    *idx_star_out = idx_star;
  }
};

template <int HI, int DI, int QG>
__global__ void __launch_bounds__(IndexerTopkTile<HI, DI, QG>::THREADS, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k, IndexerTopkParams p) {
  using T = IndexerTopkTile<HI, DI, QG>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* q_smem = smem + T::OFF_Q;
  uint8_t* k_smem = smem + T::OFF_K;
  float* coef = reinterpret_cast<float*>(smem + T::OFF_COEF);
  uint32_t* cand_u = reinterpret_cast<uint32_t*>(smem + T::OFF_CU);
  int32_t* cand_i = reinterpret_cast<int32_t*>(smem + T::OFF_CI);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + T::STAGES;
  uint64_t* acc_full = bars + 1 + 2 * T::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int group = p.n_groups - 1 - static_cast<int>(blockIdx.x);   // longest rows first
  const int b = blockIdx.y;

  const int r0 = p.row_begin + group * QG;                   // first row of the group
  const int r_last = min(r0 + QG, p.row_begin + p.rows) - 1;  // last row selected here
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  int pos_max = -1;                                          // latest position in the group
  for (int r = r0; r <= r_last; ++r) pos_max = max(pos_max, p.rp.pos(b, r));
  const int key_end = max(0, min(kvl, pos_max + 1));         // visible keys of the group
  const int n_compute = (key_end + T::M - 1) / T::M;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], T::EPI_WARPS);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, T::TMEM_COLS);
    tmem_relinquish();
  }
  // c[t,j] = w[t,j] * q_scale[t,j] for the group's rows (0 for rows past the range).
  for (int i = threadIdx.x; i < QG * HI; i += blockDim.x) {
    const int r = r0 + i / HI;
    float c = 0.f;
    if (r <= r_last) {
      const size_t o = (static_cast<size_t>(b) * p.n_q + r) * HI + (i % HI);
      c = p.w[o] * p.q_scale[o];
    }
    coef[i] = c;
  }
  if (threadIdx.x >= 64) {
    SelState* st = reinterpret_cast<SelState*>(smem + T::OFF_SEL + ((warp - 2) / 4) * T::SEL_BYTES);
    if (((warp - 2) & 3) == 0 && lane < 2) {
      st->count[lane] = 0;
      st->tau[lane] = 0;
      st->tau_idx[lane] = 0xffffffffu;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_compute > 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      mbar_arrive_expect_tx(q_full, T::Q_BYTES);
      tma_load_2d(q_smem, &tmap_q, q_full, 0, (b * p.n_q + r0) * HI);
      int issued = 0;
      for (int i = 0; i < n_compute; ++i) {
        const int st = i % T::STAGES;
        if (!mbar_wait(&k_empty[st], ((i / T::STAGES) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&k_full[st], T::K_BYTES);
        // a page outside the pool reads the TMA fill (zeros) past its end
        const int64_t y = p.km.row(b, i * T::M, p.n_kv);
        tma_load_2d(k_smem + st * T::K_BYTES, &tmap_k, &k_full[st], 0,
                    static_cast<int32_t>(y >= 0 ? y : p.km.pool_rows));
        ++issued;
      }
      // Drain: every issued key tile has landed before the CTA may exit.
      for (int i = max(0, issued - T::STAGES); i < issued; ++i)
        mbar_wait(&k_full[i % T::STAGES], (i / T::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (n_compute > 0 && elect_one()) {   // one lane runs the whole loop (see elect_one)
      constexpr uint32_t idesc = umma_idesc(T::M, T::N, 0u, 0u, 0u, 0u);
      const uint64_t q_desc = umma_desc(smem_u32(q_smem), 16, T::SBO, T::SWIZZLE);
      const uint64_t k_desc0 = umma_desc(smem_u32(k_smem), 16, T::SBO, T::SWIZZLE);
      bool ok = mbar_wait(q_full, 0);
      for (int i = 0; i < n_compute && ok; ++i) {
        const int st = i % T::STAGES;
        const int buf = i & 1;
        ok = mbar_wait(&k_full[st], (i / T::STAGES) & 1) &&
             mbar_wait(&acc_empty[buf], ((i >> 1) & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t kd = k_desc0 + static_cast<uint32_t>(st * (T::K_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < DI / 32; ++kk)
          umma_f8_ss(tmem_base + buf * T::N, kd + ((kk * 32) >> 4), q_desc + ((kk * 32) >> 4),
                     idesc, kk > 0 ? 1u : 0u);
        umma_commit(&k_empty[st]);
        umma_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue + selection
    const int ew = warp - 2;
    const int quarter = warp & 3;             // TMEM lane quarter this warp may access
    const int qhalf = ew >> 2;                // the group: rows QPW*qhalf .. of the CTA's four
    const int key_local = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    SelGroup g;
    g.st = reinterpret_cast<SelState*>(smem + T::OFF_SEL + qhalf * T::SEL_BYTES);
    g.bar_id = 1u + static_cast<uint32_t>(qhalf);
    g.gw = ew & 3;
    g.gt = g.gw * 32 + lane;
    g.lane = lane;
    const uint32_t k = static_cast<uint32_t>(p.k);

    // The head coefficients stay in shared memory (read as broadcast 16-byte
    // loads), so that the registers hold both rows' 64 TMEM columns and the
    // four TMEM loads of a tile are in flight together.
    const uint32_t coef_addr = smem_u32(coef + qhalf * T::QPW * HI);

    uint32_t tau[T::QPW], tau_idx[T::QPW];
#pragma unroll
    for (int q = 0; q < T::QPW; ++q) {
      tau[q] = 0u;
      tau_idx[q] = 0xffffffffu;
    }
    // ok turns false when a bounded wait runs out (the error word is set then).
    // The loop still runs to the end, without waiting, appending or writing,
    // so that the group's barriers stay matched.
    // The key scale of tile i + 1 is loaded while tile i is processed, so its
    // global-memory latency is not on the per-tile path.
    // A tile lies inside one page, so its first key's pool row locates all
    // of its keys.
    auto load_ks = [&](int i) -> float {
      const int s0 = i * T::M;
      if (i >= n_compute || s0 + key_local >= p.n_kv) return 0.f;
      const int64_t r = p.km.row(b, s0, p.n_kv);
      return r >= 0 ? p.k_scale[r + key_local] : 0.f;
    };
    int rpos[T::QPW];
#pragma unroll
    for (int q = 0; q < T::QPW; ++q) {
      const int r = r0 + qhalf * T::QPW + q;
      rpos[q] = r <= r_last ? p.rp.pos(b, r) : -1;
    }
    float ks_next = load_ks(0);
    bool ok = true;
    for (int i = 0; i < n_compute; ++i) {
      const int buf = i & 1;
      const float ks = ks_next;
      ks_next = load_ks(i + 1);
      if (ok) ok = mbar_wait(&acc_full[buf], (i >> 1) & 1);
      tc_fence_after();
      const int s = i * T::M + key_local;
      uint32_t x[T::QPW][HI];
      {
        const uint32_t col = tmem_base + lane_addr + buf * T::N + qhalf * T::QPW * HI;
#pragma unroll
        for (int q = 0; q < T::QPW; ++q) {
          tmem_ld32(col + q * HI, *reinterpret_cast<uint32_t(*)[32]>(&x[q][0]));
          tmem_ld32(col + q * HI + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[q][32]));
        }
        tmem_wait_ld();
      }
#pragma unroll
      for (int q = 0; q < T::QPW; ++q) {
        const int ql = qhalf * T::QPW + q;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < HI; j += 4) {
          const uint4 c4 = lds_v4(coef_addr + (q * HI + j) * 4);
          acc = fmaf(__uint_as_float(c4.x), fmaxf(__uint_as_float(x[q][j]), 0.f), acc);
          acc = fmaf(__uint_as_float(c4.y), fmaxf(__uint_as_float(x[q][j + 1]), 0.f), acc);
          acc = fmaf(__uint_as_float(c4.z), fmaxf(__uint_as_float(x[q][j + 2]), 0.f), acc);
          acc = fmaf(__uint_as_float(c4.w), fmaxf(__uint_as_float(x[q][j + 3]), 0.f), acc);
        }
        const int r = r0 + ql;
        const bool vis = r <= r_last && s < p.n_kv && s <= rpos[q] && s < kvl;
        const uint32_t u = score_key(acc * ks);
        // A key equal to tau with an index above tau_idx loses the tie to the
        // k kept entries (keys arrive in increasing index order).
        const bool take = ok && vis &&
                          (u > tau[q] || (u == tau[q] && static_cast<uint32_t>(s) <= tau_idx[q]));
        const uint32_t bal = __ballot_sync(0xffffffffu, take);
        if (bal) {
          uint32_t base = 0;
          if (lane == 0) base = atomicAdd(&g.st->count[q], static_cast<uint32_t>(__popc(bal)));
          base = __shfl_sync(0xffffffffu, base, 0);
          const uint32_t slot = base + __popc(bal & ((1u << lane) - 1u));
          if (take) {
            if (slot < static_cast<uint32_t>(T::CAP)) {
              cand_u[ql * T::CAP + slot] = u;
              cand_i[ql * T::CAP + slot] = s;
            } else {
              raise_error(kErrInternal);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (i % T::CHECK_TILES == T::CHECK_TILES - 1 && i + 1 < n_compute) {
        // Room for the next CHECK_TILES tiles in both buffers.
        g.sync();
#pragma unroll 1
        for (int q = 0; q < T::QPW; ++q) {
          const int n = static_cast<int>(g.st->count[q]);
          if (n > T::CAP - T::HEADROOM) {
            // Drop the entries a sample shows to be beaten by k others; if
            // that frees too little (many equal scores), keep exactly the k
            // largest, ties to the lower index.
            const int ql = qhalf * T::QPW + q;
            uint32_t* cu = cand_u + ql * T::CAP;
            int32_t* ci = cand_i + ql * T::CAP;
            uint32_t t, t_idx = 0xffffffffu;
            uint32_t c = g.shrink(cu, ci, n, k, &t);
            if (c > static_cast<uint32_t>(T::CAP - 2 * T::HEADROOM)) {
              g.select(cu, ci, static_cast<int>(c), k, nullptr, &t, &t_idx);
              c = k;
            }
            if (g.gt == 0) {
              g.st->count[q] = c;
              g.st->tau[q] = t;
              g.st->tau_idx[q] = t_idx;
            }
            g.sync();
          }
          tau[q] = g.st->tau[q];
          tau_idx[q] = g.st->tau_idx[q];
        }
      }
    }
    // Final selection: the k indices of each row, -1 padded.
    g.sync();
#pragma unroll 1
    for (int q = 0; q < T::QPW; ++q) {
      const int ql = qhalf * T::QPW + q;
      const int r = r0 + ql;
      if (r > r_last) continue;
      // After a timeout the indices are not written (the call reports the
      // error); the selection still runs so that the barriers stay matched.
      int32_t* out = p.indices + (static_cast<size_t>(b) * p.out_rows + (r - p.row_begin)) * k;
      const int n = static_cast<int>(g.st->count[q]);
      if (n <= p.k) {
        if (ok)
          for (int j = g.gt; j < p.k; j += 128) out[j] = j < n ? cand_i[ql * T::CAP + j] : -1;
      } else {
        uint32_t kth, idx_star;
        g.select(cand_u + ql * T::CAP, cand_i + ql * T::CAP, n, k, ok ? out : nullptr, &kth,
                 &idx_star);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

}  // namespace dsa

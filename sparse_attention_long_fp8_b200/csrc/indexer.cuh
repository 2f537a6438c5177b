// Lightning indexer on tcgen05 (page "DeepseekV3.2 拆解", section "核心组件 /
// 闪电索引器", eq. I_{t,s}):
//
//   I[t,s] = k_scale[s] * sum_j c[t,j] * ReLU(x[t,j,s]),
//   c[t,j] = w[t,j] * q_scale[t,j],   x[t,j,s] = q8[t,j,:] . k8[s,:]
//
// Factoring both scales out of the ReLU is exact for positive scales.
//
// Tile: a CTA owns QG consecutive query rows (N = QG * H^I MMA columns) and
// walks a range of 128-key tiles. Per key tile one kind::f8f6f4 MMA chain
// (K = d^I, 32 bytes per instruction) writes D[128 keys, N] into TMEM, so each
// epilogue thread owns one key (one TMEM lane) and reduces the H^I heads of a
// query from consecutive TMEM columns in registers: no cross-lane reduction,
// and the score matrix leaves the SM only as the final fp32 score.
//
// Warp roles: warp 0 issues TMA loads (q once, key tiles through a STAGES
// ring), warp 1 allocates TMEM and issues the MMAs (double-buffered
// accumulators), warps 2.. run the epilogue.
#pragma once

#include "layout.cuh"
#include "ptx.cuh"

namespace dsa {

struct IndexerParams {
  const float* q_scale;   // [B, n_q, HI]
  const float* w;         // [B, n_q, HI]
  const float* k_scale;   // [pool rows] (contiguous: [B, n_kv])
  RowPos rp;              // absolute position of each query row
  KeyMap km;              // pool row of each key
  const int32_t* kv_len;  // [B] or null
  float* scores;          // [B, rows, n_kv]
  uint64_t* signs;        // [B, rows, n_kv] bit j: x[t, j, s] > 0, or null
  int32_t B, n_q, n_kv;
  int32_t row_begin, rows;     // scored rows [row_begin, row_begin + rows)
  int32_t n_groups;            // ceil(rows / QG)
  int32_t tiles_per_split;     // key tiles per CTA
  int32_t write_invalid;       // 1: every score of the row range is written
};

template <int HI, int DI, int QG>
struct IndexerTile {
  static constexpr int M = 128;                 // keys per tile (TMEM lanes)
  static constexpr int N = QG * HI;             // MMA N
  static constexpr int STAGES = 6;
  static constexpr int K_BYTES = M * DI;        // one key tile
  static constexpr int Q_BYTES = N * DI;
  static constexpr int EPI_WARPS = QG >= 2 ? 8 : 4;
  static constexpr int THREADS = (2 + EPI_WARPS) * 32;
  static constexpr int QPW = QG / (EPI_WARPS / 4);   // queries per epilogue warp
  static constexpr uint32_t SWIZZLE = DI == 128 ? 2u : DI == 64 ? 4u : 6u;
  static constexpr uint32_t SBO = 8 * DI;       // bytes between 8-row core groups
  static constexpr uint32_t TMEM_COLS = 2 * N <= 32 ? 32 : 2 * N <= 64 ? 64 : 2 * N <= 128 ? 128
                                       : 2 * N <= 256 ? 256 : 512;
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = (Q_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_COEF = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_BAR = OFF_COEF + QG * HI * 4;
  static constexpr int NUM_BARS = 1 + 2 * STAGES + 4;
  static constexpr int SMEM_USED = OFF_BAR + NUM_BARS * 8 + 16;
  // One CTA per SM when the accumulators take all of TMEM.
  static constexpr int SMEM_BYTES =
      (TMEM_COLS == 512 ? (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) : SMEM_USED) + 1024;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N out of range for M = 128");
  static_assert(DI % 32 == 0 && DI <= 128, "indexer dim must be 32, 64 or 128");
  static_assert(QPW * HI <= 128, "epilogue coefficient registers");
};

template <int HI, int DI, int QG>
__global__ void __launch_bounds__(IndexerTile<HI, DI, QG>::THREADS, 1)
    indexer_scores_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k, IndexerParams p) {
  using T = IndexerTile<HI, DI, QG>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* q_smem = smem + T::OFF_Q;
  uint8_t* k_smem = smem + T::OFF_K;
  float* coef = reinterpret_cast<float*>(smem + T::OFF_COEF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + T::STAGES;
  uint64_t* acc_full = bars + 1 + 2 * T::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x, group = blockIdx.y, b = blockIdx.z;

  const int r0 = p.row_begin + group * QG;                   // first row of the group
  const int r_last = min(r0 + QG, p.row_begin + p.rows) - 1;  // last row scored here
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  int pos_max = -1;                                          // latest position in the group
  for (int r = r0; r <= r_last; ++r) pos_max = max(pos_max, p.rp.pos(b, r));
  const int key_end = max(0, min(kvl, pos_max + 1));         // visible keys of the group
  const int n_tiles_all = (p.n_kv + T::M - 1) / T::M;
  const int t_begin = split * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, n_tiles_all);
  const int t_end_compute = min(t_end, (key_end + T::M - 1) / T::M);
  const int n_compute = max(0, t_end_compute - t_begin);
  if (t_begin >= t_end) return;
  if (n_compute == 0 && !p.write_invalid) return;

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
        const int64_t y = p.km.row(b, (t_begin + i) * T::M, p.n_kv);
        tma_load_2d(k_smem + st * T::K_BYTES, &tmap_k, &k_full[st], 0,
                    static_cast<int32_t>(y >= 0 ? y : p.km.pool_rows));
        ++issued;
      }
      griddep_launch_dependents();   // the top-k may start its set-up
      // Drain: every issued key tile has landed before the CTA may exit.
      for (int i = max(0, issued - T::STAGES); i < issued; ++i)
        mbar_wait(&k_full[i % T::STAGES], (i / T::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (n_compute > 0 && elect_one()) {
      constexpr uint32_t idesc = umma_idesc(T::M, T::N, 0u, 0u, 0u, 0u);
      bool ok = mbar_wait(q_full, 0);
      const uint32_t q_addr = smem_u32(q_smem);
      for (int i = 0; i < n_compute && ok; ++i) {
        const int st = i % T::STAGES;
        const int buf = i & 1;
        ok = mbar_wait(&k_full[st], (i / T::STAGES) & 1);
        if (!ok) break;
        ok = mbar_wait(&acc_empty[buf], ((i >> 1) & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(k_smem + st * T::K_BYTES);
        const uint32_t d_tmem = tmem_base + buf * T::N;
#pragma unroll
        for (int kk = 0; kk < DI / 32; ++kk) {
          const uint64_t a = umma_desc(k_addr + kk * 32, 16, T::SBO, T::SWIZZLE);
          const uint64_t bd = umma_desc(q_addr + kk * 32, 16, T::SBO, T::SWIZZLE);
          umma_f8_ss(d_tmem, a, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[st]);
        umma_commit(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;             // TMEM lane quarter this warp may access
    const int qhalf = ew / 4;                 // which slice of the group's queries
    const int key_local = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const size_t row_stride = static_cast<size_t>(p.n_kv);
    float* out_base = p.scores + (static_cast<size_t>(b) * p.rows + (r0 - p.row_begin)) * row_stride;

    float cf[T::QPW][HI];
    int rpos[T::QPW];
#pragma unroll
    for (int q = 0; q < T::QPW; ++q) {
      const int r = r0 + qhalf * T::QPW + q;
      rpos[q] = r <= r_last ? p.rp.pos(b, r) : -1;
#pragma unroll
      for (int j = 0; j < HI; ++j) cf[q][j] = coef[(qhalf * T::QPW + q) * HI + j];
    }

    // The key scale of tile i + 1 is loaded while tile i is processed, so its
    // global-memory latency is not on the per-tile path. A tile lies inside
    // one page, so its first key's pool row locates all of its keys.
    auto load_ks = [&](int i) -> float {
      const int s0 = (t_begin + i) * T::M;
      if (i >= n_compute || s0 + key_local >= p.n_kv) return 0.f;
      const int64_t r = p.km.row(b, s0, p.n_kv);
      return r >= 0 ? p.k_scale[r + key_local] : 0.f;
    };
    float ks_next = load_ks(0);
    bool ok = true;
    for (int i = 0; i < n_compute; ++i) {
      const int buf = i & 1;
      const float ks = ks_next;
      ks_next = load_ks(i + 1);
      ok = mbar_wait(&acc_full[buf], (i >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const int s = (t_begin + i) * T::M + key_local;
#pragma unroll
      for (int q = 0; q < T::QPW; ++q) {
        const int ql = qhalf * T::QPW + q;
        const uint32_t col = tmem_base + lane_addr + buf * T::N + ql * HI;
        float acc = 0.f;
        uint64_t sbits = 0;   // sign of each head's dot product (training path)
        if constexpr (HI >= 32) {
#pragma unroll
          for (int h0 = 0; h0 < HI; h0 += 32) {
            uint32_t x[32];
            tmem_ld32(col + h0, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              acc = fmaf(cf[q][h0 + j], fmaxf(__uint_as_float(x[j]), 0.f), acc);
            if (p.signs) {
              uint32_t m = 0;
#pragma unroll
              for (int j = 0; j < 32; ++j) m |= (__uint_as_float(x[j]) > 0.f ? 1u : 0u) << j;
              sbits |= static_cast<uint64_t>(m) << h0;
            }
          }
        } else {
          uint32_t x[4];
          static_assert(HI == 4, "small head counts: only H^I = 4 is instantiated");
          tmem_ld4(col, x);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc = fmaf(cf[q][j], fmaxf(__uint_as_float(x[j]), 0.f), acc);
            sbits |= static_cast<uint64_t>(__uint_as_float(x[j]) > 0.f ? 1u : 0u) << j;
          }
        }
        const int r = r0 + ql;
        if (r <= r_last && s < p.n_kv) {
          const bool vis = s <= rpos[q] && s < kvl;
          out_base[static_cast<size_t>(ql) * row_stride + s] = vis ? acc * ks : -INFINITY;
          if (p.signs)
            p.signs[(static_cast<size_t>(b) * p.rows + (r0 - p.row_begin) + ql) * row_stride + s] =
                sbits;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (p.write_invalid) {
      // Tiles past the group's visible range: every key is invisible.
      for (int t = t_begin + n_compute; t < t_end; ++t) {
        const int s = t * T::M + key_local;
        if (s >= p.n_kv) continue;
        for (int q = 0; q < T::QPW; ++q) {
          const int ql = qhalf * T::QPW + q;
          if (r0 + ql <= r_last) out_base[static_cast<size_t>(ql) * row_stride + s] = -INFINITY;
        }
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

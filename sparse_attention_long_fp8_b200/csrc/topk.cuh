// Per-row top-k selection (page "DeepseekV3.2 拆解", section "核心组件 /
// 细粒度 Token 选择机制", eq. u_t: keep the k keys with the largest index
// score). Ties are broken by the lower key index.
//
// One CTA per score row. Scores are mapped to order-preserving uint32 keys
// (larger float <=> larger key; -0 is folded into +0), then an MSB-first radix
// select finds the exact k-th largest key u* in four 8-bit passes with shared
// memory histograms. A final pass writes every key > u* and the lowest-index
// keys == u* (an ordered block scan over the row, only when the ties at u*
// do not all fit). Rows of up to kTopkSmemKeys visible scores are staged once in
// shared memory; longer rows are re-read from global memory (L2) per pass.
#pragma once

#include "ptx.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;    // [B, rows, n_kv]
  const int32_t* q_pos0;  // [B] or null
  const int32_t* kv_len;  // [B] or null
  int32_t* indices;       // row r of sequence b -> indices[(b * out_rows + out_row0 + r) * k]
  int32_t rows, row_begin, n_kv, k;   // score rows [row_begin, row_begin + rows) per sequence
  int32_t out_rows, out_row0;
};

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 48 * 1024;   // 192 KB of staged keys

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint32_t tk_smem[];
  uint32_t* staged = tk_smem;                       // [kTopkSmemKeys]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_sel_bin, s_above, s_count;
  __shared__ uint32_t warp_tot[kTopkThreads / 32];

  const int r = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int pos = (p.q_pos0 ? p.q_pos0[b] : 0) + p.row_begin + r;
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int n = max(0, min(pos + 1, kvl));
  const float* row = p.scores + (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
  int32_t* out = p.indices + (static_cast<size_t>(b) * p.out_rows + p.out_row0 + r) * p.k;

  if (n <= p.k) {
    for (int i = tid; i < p.k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  const bool use_smem = n <= kTopkSmemKeys;
  if (use_smem) {
    for (int i = tid; i < n; i += kTopkThreads) staged[i] = order_key(row[i]);
    __syncthreads();
  }

  uint32_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(p.k);   // still to take among keys matching prefix
  uint32_t eq_count = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += kTopkThreads) {
      // Warp-aggregated increments: score keys cluster in few high bins, so
      // lanes with the same bin merge into one atomic.
      const int i = c0 + tid;
      uint32_t bin = 256u;
      if (i < n) {
        const uint32_t u = use_smem ? staged[i] : order_key(row[i]);
        if ((u & mask) == prefix) bin = (u >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256u && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins [248 - 8l, 255 - 8l] (high bins first)
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - (tid * 8 + j)];
        sum += c[j];
      }
      uint32_t incl = sum;   // inclusive prefix over lanes (from the top)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += v;
      }
      const uint32_t excl = incl - sum;
      if (excl < need && need <= incl) {
        uint32_t acc = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc < need && need <= acc + c[j]) {
            s_sel_bin = 255u - (tid * 8 + j);
            s_above = acc;
            s_count = c[j];
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = s_sel_bin;
    need -= s_above;
    eq_count = s_count;
    prefix |= bin << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  // prefix is now the exact k-th largest key u*; `need` keys equal to u* are
  // taken (1 <= need <= eq_count) after every key > u*.
  const uint32_t kth = prefix;
  if (tid == 0) s_count = 0;
  __syncthreads();
  const bool take_all_eq = need == eq_count;
  for (int c0 = 0; c0 < n; c0 += kTopkThreads) {
    const int i = c0 + tid;
    bool take = false;
    if (i < n) {
      const uint32_t u = use_smem ? staged[i] : order_key(row[i]);
      take = u > kth || (take_all_eq && u == kth);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    uint32_t base = 0;
    if ((tid & 31) == 0 && bal) base = atomicAdd(&s_count, static_cast<uint32_t>(__popc(bal)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) out[base + __popc(bal & ((1u << (tid & 31)) - 1u))] = i;
  }
  if (!take_all_eq) {
    __syncthreads();
    const uint32_t base_slot = s_count;   // = k - need
    uint32_t taken = 0;
    const int lane = tid & 31, w = tid >> 5;
    for (int c0 = 0; c0 < n && taken < need; c0 += kTopkThreads) {
      const int i = c0 + tid;
      const bool eq = i < n && (use_smem ? staged[i] : order_key(row[i])) == kth;
      const uint32_t bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) warp_tot[w] = __popc(bal);
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int j = 0; j < kTopkThreads / 32; ++j) {
        const uint32_t v = warp_tot[j];
        if (j < w) before += v;
        total += v;
      }
      const uint32_t rank = taken + before + __popc(bal & ((1u << lane) - 1u));
      if (eq && rank < need) out[base_slot + rank] = i;
      taken += total;
      __syncthreads();
    }
  }
}

}  // namespace dsa

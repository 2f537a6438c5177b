// Per-row top-k selection (page "DeepseekV3.2 拆解", section "核心组件 /
// 细粒度 Token 选择机制", eq. u_t: keep the k keys with the largest index
// score). Ties are broken by the lower key index.
//
// A cluster of two CTAs per score row. Scores are mapped to order-preserving
// uint32 keys (larger float <=> larger key; -0 is folded into +0).
//   1. A threshold tau from 1024 evenly spaced samples of the row: two 8-bit
//      radix passes over the samples find the 16-bit key prefix of the
//      sample ranked about 1.25 k / n of the way down; tau is the lowest key
//      with that prefix, so roughly 1.25 k keys of the row are >= tau.
//   2. Each CTA of the pair takes one half of the row (16-byte loads, 32
//      scores per thread in flight) and appends every (key, index) with key
//      >= tau to its own candidate buffer in shared memory (one slot
//      reservation per warp and round). Both compute the same tau from the
//      same samples. CTA 1's candidates are then read by CTA 0 over
//      distributed shared memory; CTA 0 alone does the rest.
//   3. If k <= #candidates <= capacity, an MSB-first radix select over the
//      candidates finds the exact k-th key u*; every candidate above u* is
//      written, then the lowest-index candidates equal to u*.
//   Otherwise (a sample that missed, or many exact ties) the same radix
//   select runs over the whole row, re-read from global memory per pass.
// The result never depends on the sample: it only decides how much of the
// row the exact select has to look at.
#pragma once

#include "layout.cuh"
#include "ptx.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;    // [B, rows, n_kv]
  RowPos rp;              // absolute position of each query row
  const int32_t* kv_len;  // [B] or null
  int32_t* indices;       // row r of sequence b -> indices[(b * out_rows + out_row0 + r) * k]
  int32_t rows, row_begin, n_kv, k;   // score rows [row_begin, row_begin + rows) per sequence
  int32_t out_rows, out_row0;
};

constexpr int kTopkThreads = 1024;
constexpr int kTopkSamples = 1024;
constexpr int kTopkCap = 8192;      // candidate buffer (keys + indices: 64 KB)

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkSmem {
  uint32_t cand_u[kTopkCap];
  int32_t cand_i[kTopkCap];
  uint32_t samp[kTopkSamples];
  uint32_t hist[2][256];          // radix passes alternate buffers
  uint32_t warp_tot[kTopkThreads / 32];
  uint32_t sel_bin[2], above[2], sel_count[2];
  uint32_t count, n_cand;
};

// Exact k-th largest key among `n` keys given by get(i) (all threads of the
// CTA call this). Returns u*; *need_out = number of keys equal to u* that
// belong to the top k; *eq_out = number of keys equal to u*.
// With PASSES = 2 only the top 16 bits are resolved: the result is that
// prefix (low bits zero) of the k-th largest key.
// Pass p counts into hist[p & 1] while the other buffer is cleared for pass
// p + 1, so a pass needs two CTA barriers. hist[0] is zero on entry and,
// PASSES being even, is cleared again by the last pass before its barriers.
template <int PASSES, class Get>
__device__ uint32_t radix_kth(TopkSmem& sm, int n, uint32_t k, Get get, uint32_t* need_out,
                              uint32_t* eq_out) {
  static_assert(PASSES == 2 || PASSES == 4, "an even number of 8-bit passes");
  constexpr int passes = PASSES;
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0, need = k, eq_count = 0;
  for (int pass = 0; pass < passes; ++pass) {
    const int shift = 24 - 8 * pass;
    const int hb = pass & 1;
    uint32_t* hist = sm.hist[hb];
    // the other buffer: its last reader (the previous pass's scan) finished
    // before that pass's second barrier
    if (tid < 256) sm.hist[hb ^ 1][tid] = 0;
    for (int c0 = 0; c0 < n; c0 += kTopkThreads) {
      const int i = c0 + tid;
      uint32_t bin = 256u;
      if (i < n) {
        const uint32_t u = get(i);
        if ((u & mask) == prefix) bin = (u >> shift) & 255u;
      }
      // lanes with the same bin merge into one atomic (keys cluster in few bins)
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256u && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - (tid * 8 + j)];
        sum += c[j];
      }
      uint32_t incl = sum;
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
            sm.sel_bin[hb] = 255u - (tid * 8 + j);
            sm.above[hb] = acc;
            sm.sel_count[hb] = c[j];
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    need -= sm.above[hb];
    eq_count = sm.sel_count[hb];
    prefix |= sm.sel_bin[hb] << shift;
    mask |= 255u << shift;
  }
  *need_out = need;
  *eq_out = eq_count;
  return prefix;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTopkThreads, 1)
    topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint8_t tk_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(tk_raw);

  // the scores come from the previous kernel (launched with a dependent
  // launch in the forward path)
  griddep_wait();
  const int r = blockIdx.x >> 1, b = blockIdx.y;
  const uint32_t part = cluster_ctarank();     // which half of the row this CTA scans
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int pos = p.rp.pos(b, p.row_begin + r);
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int n = max(0, min(pos + 1, kvl));
  const float* row = p.scores + (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
  int32_t* out = p.indices + (static_cast<size_t>(b) * p.out_rows + p.out_row0 + r) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);

  if (n <= p.k) {   // both CTAs of the pair leave here (same row, same n)
    griddep_launch_dependents();
    if (part == 0)
      for (int i = tid; i < p.k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }

  // ---- 1. threshold: the 16-bit key prefix of the sample of rank `want`
  sm.samp[tid] = order_key(row[static_cast<int>((static_cast<int64_t>(tid) * n) / kTopkSamples)]);
  if (tid == 0) sm.n_cand = 0;
  if (tid < 256) sm.hist[0][tid] = 0;
  __syncthreads();
  const int64_t want =
      (static_cast<int64_t>(5) * p.k * kTopkSamples) / (4 * static_cast<int64_t>(n)) + 8;
  uint32_t s_need, s_eq;
  const uint32_t tau = radix_kth<2>(
      sm, kTopkSamples, static_cast<uint32_t>(want < kTopkSamples ? want : kTopkSamples),
      [&](int i) { return sm.samp[i]; }, &s_need, &s_eq);

  // ---- 2. one pass: candidates >= tau. A thread takes 32 scores per round
  // (eight 16-byte loads in flight when the row is 16-byte aligned) and
  // forms a bit mask of those >= tau; the warp then reserves all of its
  // slots with one shared atomic, each thread's first slot coming from an
  // inclusive scan of the per-thread counts.
  auto reserve = [&](uint32_t cnt) -> uint32_t {
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t base = 0;
    if (lane == 0 && total) base = atomicAdd(&sm.n_cand, total);
    return __shfl_sync(0xffffffffu, base, 0) + incl - cnt;
  };
  auto put = [&](uint32_t slot, uint32_t u, int i) {
    if (slot < static_cast<uint32_t>(kTopkCap)) {
      sm.cand_u[slot] = u;
      sm.cand_i[slot] = i;
    }
  };
  // this CTA's scores: [lo, hi) as whole float4s when the row is 16-byte
  // aligned (the < 4 scores past the last whole float4 go to CTA 1's scalar
  // loop), else [s_lo, s_hi) by the scalar loop alone
  int s_lo, s_hi;
  if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = n >> 2, h4 = (n4 + 1) >> 1;
    const int lo4 = part ? h4 : 0, hi4 = part ? n4 : h4;
    s_lo = part ? n4 * 4 : n;
    s_hi = n;
    for (int c0 = lo4; c0 < hi4; c0 += 8 * kTopkThreads) {
      uint4 v[8];                                  // order keys of 4 scores each
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int c = c0 + tid + m * kTopkThreads;
        const float4 f = c < hi4 ? row4[c] : make_float4(0.f, 0.f, 0.f, 0.f);
        v[m] = make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
      }
      uint32_t mask = 0;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        // past this CTA's last float4 nothing is taken
        const bool in = c0 + tid + m * kTopkThreads < hi4;
        mask |= static_cast<uint32_t>(in && v[m].x >= tau) << (4 * m);
        mask |= static_cast<uint32_t>(in && v[m].y >= tau) << (4 * m + 1);
        mask |= static_cast<uint32_t>(in && v[m].z >= tau) << (4 * m + 2);
        mask |= static_cast<uint32_t>(in && v[m].w >= tau) << (4 * m + 3);
      }
      uint32_t slot = reserve(__popc(mask));
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i = (c0 + tid + m * kTopkThreads) * 4;
        if ((mask >> (4 * m)) & 1u) put(slot++, v[m].x, i);
        if ((mask >> (4 * m + 1)) & 1u) put(slot++, v[m].y, i + 1);
        if ((mask >> (4 * m + 2)) & 1u) put(slot++, v[m].z, i + 2);
        if ((mask >> (4 * m + 3)) & 1u) put(slot++, v[m].w, i + 3);
      }
    }
  } else {
    const int half_n = (n + 1) >> 1;
    s_lo = part ? half_n : 0;
    s_hi = part ? n : half_n;
  }
  for (int c0 = s_lo; c0 < s_hi; c0 += 32 * kTopkThreads) {
    uint32_t u[32];
    uint32_t mask = 0;
#pragma unroll
    for (int m = 0; m < 32; ++m) {
      const int i = c0 + tid + m * kTopkThreads;
      u[m] = i < s_hi ? order_key(row[i]) : 0u;
      mask |= static_cast<uint32_t>(i < s_hi && u[m] >= tau) << m;
    }
    uint32_t slot = reserve(__popc(mask));
#pragma unroll
    for (int m = 0; m < 32; ++m)
      if ((mask >> m) & 1u) put(slot++, u[m], c0 + tid + m * kTopkThreads);
  }
  // ---- CTA 0 takes CTA 1's candidates behind its own
  cluster_sync();                  // both candidate buffers and counts are final
  griddep_launch_dependents();     // the attention may start its own set-up
  if (part != 0) {
    cluster_sync();                // CTA 0 has read this CTA's shared memory
    return;
  }
  const uint32_t n_own = sm.n_cand;
  const uint32_t n_peer = ld_dsmem_u32(mapa_shared(smem_u32(&sm.n_cand), 1));
  const uint32_t cap = static_cast<uint32_t>(kTopkCap);
  const bool fits = n_own <= cap && n_peer <= cap && n_own + n_peer <= cap;
  if (fits) {
    const uint32_t pu = mapa_shared(smem_u32(&sm.cand_u[0]), 1);
    const uint32_t pi = mapa_shared(smem_u32(&sm.cand_i[0]), 1);
    for (uint32_t j = tid; j < n_peer; j += kTopkThreads) {
      sm.cand_u[n_own + j] = ld_dsmem_u32(pu + 4 * j);
      sm.cand_i[n_own + j] = static_cast<int32_t>(ld_dsmem_u32(pi + 4 * j));
    }
  }
  cluster_sync();
  const uint32_t n_cand = fits ? n_own + n_peer : cap + 1;

  if (n_cand >= k && n_cand <= cap) {
    // ---- 3. exact select among the candidates
    uint32_t need, eq_count;
    const uint32_t kth = radix_kth<4>(sm, static_cast<int>(n_cand), k,
                                   [&](int i) { return sm.cand_u[i]; }, &need, &eq_count);
    if (tid == 0) sm.count = 0;
    __syncthreads();
    const bool take_all_eq = need == eq_count;
    for (int c0 = 0; c0 < static_cast<int>(n_cand); c0 += kTopkThreads) {
      const int i = c0 + tid;
      const bool take = i < static_cast<int>(n_cand) &&
                        (sm.cand_u[i] > kth || (take_all_eq && sm.cand_u[i] == kth));
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      uint32_t base = 0;
      if (lane == 0 && bal) base = atomicAdd(&sm.count, static_cast<uint32_t>(__popc(bal)));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (take) out[base + __popc(bal & ((1u << lane) - 1u))] = sm.cand_i[i];
    }
    if (!take_all_eq) {
      // ties at u*: a tied candidate is taken iff fewer than `need` tied
      // candidates have a lower key index.
      __syncthreads();
      const uint32_t base_slot = sm.count;
      for (int i = tid; i < static_cast<int>(n_cand); i += kTopkThreads) {
        if (sm.cand_u[i] != kth) continue;
        const int my = sm.cand_i[i];
        uint32_t lower = 0;
        for (int j = 0; j < static_cast<int>(n_cand); ++j)
          lower += (sm.cand_u[j] == kth && sm.cand_i[j] < my) ? 1u : 0u;
        if (lower < need) out[base_slot + lower] = my;
      }
    }
    return;
  }

  // ---- fallback: exact select over the whole row (global memory per pass)
  uint32_t need, eq_count;
  const uint32_t kth = radix_kth<4>(sm, n, k, [&](int i) { return order_key(row[i]); }, &need,
                                 &eq_count);
  if (tid == 0) sm.count = 0;
  __syncthreads();
  const bool take_all_eq = need == eq_count;
  for (int c0 = 0; c0 < n; c0 += kTopkThreads) {
    const int i = c0 + tid;
    bool take = false;
    if (i < n) {
      const uint32_t u = order_key(row[i]);
      take = u > kth || (take_all_eq && u == kth);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    uint32_t base = 0;
    if (lane == 0 && bal) base = atomicAdd(&sm.count, static_cast<uint32_t>(__popc(bal)));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) out[base + __popc(bal & ((1u << lane) - 1u))] = i;
  }
  if (!take_all_eq) {
    // ordered block scan over the row: the first `need` keys equal to u*
    __syncthreads();
    const uint32_t base_slot = sm.count;
    uint32_t taken = 0;
    for (int c0 = 0; c0 < n && taken < need; c0 += kTopkThreads) {
      const int i = c0 + tid;
      const bool eq = i < n && order_key(row[i]) == kth;
      const uint32_t bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) sm.warp_tot[w] = __popc(bal);
      __syncthreads();
      uint32_t before = 0, total = 0;
      for (int j = 0; j < kTopkThreads / 32; ++j) {
        const uint32_t v = sm.warp_tot[j];
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

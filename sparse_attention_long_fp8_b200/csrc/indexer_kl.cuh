// Indexer warm-up loss and its gradient (page "DeepseekV3.2 拆解", section
// "预训练策略 / 密集预热阶段": the main model is frozen and the indexer is
// trained to follow the dense attention distribution,
//   L^I = sum_t KL(p_{t,:} || Softmax(I_{t,:})) ).
//
// Readings (the page is silent on them): p_{t,:} is the main attention's
// dense causal softmax over the visible keys averaged over the H query heads;
// Softmax(I_{t,:}) runs over the same keys; the gradient is taken with
// respect to w and to the dequantised indexer vectors q^ = code * q_scale,
// k^ = code * k_scale. With g[t,s] = Softmax(I_t)[s] - p[t,s] and
// x[t,j,s] = q^[t,j] . k^[s]:
//   U[t,j,:]  = sum_s g[t,s] [x > 0] k^[s]
//   dq^[t,j]  = w[t,j] U[t,j]            (dL/dq^)
//   dw[t,j]   = U[t,j] . q^[t,j]         (= sum_s g ReLU(x), as x = q^ . k^)
//   dk^[s]    = sum_t sum_j g[t,s] w[t,j] [x > 0] q^[t,j]
//
// Kernels, per chunk of query rows:
//   kl_probs_kernel   p (head-averaged dense attention probabilities) on
//                     tcgen05: Q in TMEM (A operand), 64 contiguous latent
//                     rows per block in shared memory, two passes over the
//                     visible keys (row max and sum, then probabilities);
//                     the head average is a warp transpose-reduce plus a
//                     fixed-order sum over the four lane quarters;
//   (scores)          indexer_scores_kernel writes I and the sign of every
//                     head's dot product (one 64-bit mask per (row, key));
//   kl_rows_kernel    the loss of each row and g = Softmax(I) - p in place;
//   kl_grad_u_kernel  U, then dq^ and dw, in fp32 on the CUDA cores;
//   kl_grad_k_kernel  dk^ in fp32 on the CUDA cores, accumulated over the
//                     row chunks (each CTA owns a tile of keys: no atomics).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dsa {

// ------------------------------------------------------------------ p

struct KlProbParams {
  const __nv_bfloat16* q;   // [B, n_q, H, DQK]
  const __nv_bfloat16* kv;  // [B, n_kv, DQK] latent rows (K = all DQK dims)
  const int32_t* q_pos0;    // [B] or null
  const int32_t* kv_len;    // [B] or null
  float* pbar;              // [B, rows, n_kv]: p of the visible keys (others untouched)
  int32_t B, n_q, n_kv, H;
  int32_t row_begin, rows;
  float scale_log2;         // softmax_scale * log2(e)
};

template <int DQK>
struct KlProbTile {
  static constexpr int NK = 64;                 // keys per block
  static constexpr int M = 128;                 // head rows (zero-padded past H)
  static constexpr int NDB = DQK / 64;          // 64-dim blocks of a latent row
  static constexpr int DB_BYTES = NK * 128;
  static constexpr int STAGE_BYTES = NDB * DB_BYTES;
  static constexpr int STAGES = 2;
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 288;           // gather 0-3, MMA 4, softmax 5-8
  static constexpr int COL_S = 0;               // S buffer b at COL_S + 64 b
  static constexpr int COL_Q = 128;             // Q: DQK / 2 columns (bf16 pairs)
  static constexpr int COLS_USED = COL_Q + DQK / 2;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 256 ? 256 : 512;
  static constexpr int OFF_C = 0;
  static constexpr int OFF_RED = STAGES * STAGE_BYTES;         // [2][4][64] fp32
  static constexpr int OFF_BAR = OFF_RED + 2 * 4 * NK * 4;
  static constexpr int NUM_BARS = 4 * STAGES + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(DQK % 64 == 0 && COLS_USED <= 512, "latent width");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Sum over the 32 lanes of v[k] for each of 64 values k: recursive halving,
// after which lane L holds the sums of values 2L and 2L + 1 in v[0], v[1].
__device__ __forceinline__ void warp_transpose_sum64(float (&v)[64], int lane) {
#pragma unroll
  for (int o = 16, half = 32; o >= 1; o >>= 1, half >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
}

template <int DQK>
__global__ void __launch_bounds__(288, 1) kl_probs_kernel(KlProbParams p) {
  using T = KlProbTile<DQK>;
  constexpr int NK = T::NK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* c_smem = smem + T::OFF_C;
  float* red = reinterpret_cast<float*>(smem + T::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* c_full = bars;
  uint64_t* c_empty = bars + T::STAGES;
  uint64_t* s_full = bars + 2 * T::STAGES;
  uint64_t* s_free = bars + 3 * T::STAGES;
  uint64_t* q_ready = bars + 4 * T::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x, b = blockIdx.y;
  const int t = p.row_begin + r;                          // query row in its sequence
  const int pos = (p.q_pos0 ? p.q_pos0[b] : 0) + t;
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int n_vis = max(0, min(pos + 1, kvl));            // visible keys [0, n_vis)
  const int nb = (n_vis + NK - 1) / NK;
  const int n_it = 2 * nb;                                // pass 1, then pass 2
  const __nv_bfloat16* kv_b = p.kv + static_cast<size_t>(b) * p.n_kv * DQK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&c_full[s], T::PRODUCERS);
      mbar_init(&c_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(q_ready, 4);
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ gather
    // Thread (kq, ch) copies 16-byte chunk ch of every 64-dim block of keys
    // kq, kq + 16, kq + 32, kq + 48 of a block (128-byte swizzled K-major).
    const int kq = threadIdx.x >> 3, ch = threadIdx.x & 7;
    const uint32_t dst0 = smem_u32(c_smem) + kq * 128 + ((ch ^ (kq & 7)) << 4);
    bool ok = true;
    for (int i = 0; i < n_it && ok; ++i) {
      const int st = i & 1;
      const int s0 = (i % nb) * NK;
      ok = mbar_wait(&c_empty[st], ((i >> 1) & 1) ^ 1);
      if (!ok) break;
      const uint32_t dst = dst0 + st * T::STAGE_BYTES;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int s = s0 + kq + 16 * rr;
        const bool v = s < n_vis;
        const __nv_bfloat16* src = kv_b + static_cast<size_t>(v ? s : 0) * DQK + ch * 8;
#pragma unroll
        for (int db = 0; db < T::NDB; ++db)
          cp_async_16(dst + db * T::DB_BYTES + rr * 16 * 128, src + db * 64, v ? 16u : 0u);
      }
      cp_async_arrive_noinc(&c_full[st]);
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ S = Q C^T issuer
    // one elected lane runs the whole loop (see elect_one)
    if (elect_one()) {
      constexpr uint32_t idesc = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
      const uint64_t c_desc0 = umma_desc(smem_u32(c_smem), 16, 1024, 2);
      bool ok = mbar_wait(q_ready, 0);
      tc_fence_after();
      for (int i = 0; i < n_it && ok; ++i) {
        const int st = i & 1;
        ok = mbar_wait(&c_full[st], (i >> 1) & 1) && mbar_wait(&s_free[st], ((i >> 1) & 1) ^ 1);
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t d_s = tmem_base + T::COL_S + st * NK;
        const uint64_t cd = c_desc0 + static_cast<uint32_t>(st * (T::STAGE_BYTES >> 4));
#pragma unroll
        for (int db = 0; db < T::NDB; ++db)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = cd + ((db * T::DB_BYTES + kk * 32) >> 4);
            umma_bf16_ts(d_s, tmem_base + T::COL_Q + db * 32 + kk * 8, bd, idesc, (db | kk) ? 1u : 0u);
          }
        umma_commit(&c_empty[st]);
        umma_commit(&s_full[st]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;                   // head row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const bool live = h < p.H;
    {
      // Q of this head into TMEM (columns COL_Q.., two bf16 per column)
      const __nv_bfloat16* qh =
          p.q + ((static_cast<size_t>(b) * p.n_q + t) * p.H + min(h, p.H - 1)) * DQK;
#pragma unroll 1
      for (int c = 0; c < DQK / 32; ++c) {
        uint32_t v[16];
        const uint4* src = reinterpret_cast<const uint4*>(qh + c * 32);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 u = live ? src[k] : make_uint4(0u, 0u, 0u, 0u);
          v[4 * k] = u.x; v[4 * k + 1] = u.y; v[4 * k + 2] = u.z; v[4 * k + 3] = u.w;
        }
        tmem_st16(tmem_base + lane_addr + T::COL_Q + c * 16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    float m = -INFINITY, l = 0.f, inv_l = 0.f;   // row max (log2 domain) and sum
    const float inv_h = 1.0f / static_cast<float>(p.H);
    float* out = p.pbar + (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
    bool ok = true;
    for (int i = 0; i < n_it; ++i) {
      const int sb = i & 1;
      const int s0 = (i % nb) * NK;
      const bool pass2 = i >= nb;
      if (ok) ok = mbar_wait(&s_full[sb], (i >> 1) & 1);
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tmem_base + lane_addr + T::COL_S + sb * NK, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tmem_base + lane_addr + T::COL_S + sb * NK + 32,
                *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      float z[64];
#pragma unroll
      for (int k = 0; k < 64; ++k)
        z[k] = (s0 + k < n_vis) ? __uint_as_float(sr[k]) * p.scale_log2 : -INFINITY;
      if (!pass2) {
        float bmax = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) bmax = fmaxf(bmax, z[k]);
        const float m_new = fmaxf(m, bmax);
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < 64; ++k) sum += exp2f(z[k] - m_new);
        l = l * exp2f(m - m_new) + sum;
        m = m_new;
        if (i == nb - 1) inv_l = 1.0f / l;
      } else {
        // p of this head, then the sum over the heads of each key
#pragma unroll
        for (int k = 0; k < 64; ++k) z[k] = live ? exp2f(z[k] - m) * inv_l : 0.f;
        warp_transpose_sum64(z, lane);
        float* rb = red + ((i & 1) * 4 + quarter) * NK;
        rb[2 * lane] = z[0];
        rb[2 * lane + 1] = z[1];
        named_bar_sync(1, 128);   // the four softmax warps (always all arrive)
        if (warp == 5 || warp == 6) {
          const int k = (warp - 5) * 32 + lane;
          const float* r0 = red + (i & 1) * 4 * NK;
          const float v = ((r0[k] + r0[NK + k]) + r0[2 * NK + k]) + r0[3 * NK + k];
          if (ok && s0 + k < n_vis) out[s0 + k] = v * inv_h;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ loss rows

struct KlRowParams {
  const float* scores;      // [B, rows, n_kv] I (invisible keys -inf)
  float* pbar;              // [B, rows, n_kv] p in, g = Softmax(I) - p out (visible keys)
  float* loss;              // [B, n_q]
  const int32_t* q_pos0;
  const int32_t* kv_len;
  int32_t n_q, n_kv, row_begin, rows;
};

constexpr int kKlRowThreads = 256;

__device__ __forceinline__ float block_reduce(float v, float* sh, bool is_max) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, u) : v + u;
  }
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  float acc = sh[0];
  for (int i = 1; i < kKlRowThreads / 32; ++i) acc = is_max ? fmaxf(acc, sh[i]) : acc + sh[i];
  return acc;
}

__global__ void __launch_bounds__(kKlRowThreads) kl_rows_kernel(KlRowParams p) {
  __shared__ float sh[kKlRowThreads / 32];
  const int r = blockIdx.x, b = blockIdx.y;
  const int t = p.row_begin + r;
  const int pos = (p.q_pos0 ? p.q_pos0[b] : 0) + t;
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int n_vis = max(0, min(pos + 1, kvl));
  const float* I = p.scores + (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
  float* pg = p.pbar + (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < n_vis; s += kKlRowThreads) mx = fmaxf(mx, I[s]);
  mx = block_reduce(mx, sh, true);
  float sum = 0.f;
  for (int s = threadIdx.x; s < n_vis; s += kKlRowThreads) sum += expf(I[s] - mx);
  sum = block_reduce(sum, sh, false);
  const float lse = mx + logf(sum);
  float kl = 0.f;
  for (int s = threadIdx.x; s < n_vis; s += kKlRowThreads) {
    const float pv = pg[s];
    const float li = I[s] - lse;                        // log Softmax(I)
    if (pv > 0.f) kl += pv * (logf(pv) - li);
    pg[s] = expf(li) - pv;                              // g
  }
  kl = block_reduce(kl, sh, false);
  if (threadIdx.x == 0) p.loss[static_cast<size_t>(b) * p.n_q + t] = n_vis > 0 ? kl : 0.f;
}

// ------------------------------------------------------------------ gradients

// E4M3 code -> value (exact in fp32): 1 sign, 4 exponent (bias 7), 3 mantissa
// bits; exponent 0 is subnormal. (0x7F / 0xFF are NaN codes; the quantiser
// never emits them.)
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xF, mnt = c & 7;
  const float mag = e ? __uint_as_float(((e + 120u) << 23) | (mnt << 20))
                      : static_cast<float>(mnt) * 0.001953125f;   // m / 8 * 2^-6
  return (c & 0x80) ? -mag : mag;
}

struct KlGradParams {
  const uint8_t* q_fp8;     // [B, n_q, HI, DI]
  const float* q_scale;     // [B, n_q, HI]
  const float* w;           // [B, n_q, HI]
  const uint8_t* k_fp8;     // [B, n_kv, DI]
  const float* k_scale;     // [B, n_kv]
  const float* g;           // [B, rows, n_kv] g of the chunk's rows (visible keys)
  const uint64_t* signs;    // [B, rows, n_kv] bit j: x[t, j, s] > 0
  const int32_t* q_pos0;
  const int32_t* kv_len;
  float* dw;                // [B, n_q, HI]
  float* dq;                // [B, n_q, HI, DI]
  float* dk;                // [B, n_kv, DI] accumulated over the row chunks
  int32_t n_q, n_kv, row_begin, rows;
};

constexpr int kKlGradThreads = 256;
constexpr int kKlKeysPerStep = 32;   // keys staged per step (grad_u)

// U[t, j, :] = sum_s g[t,s] [x > 0] k^[s] for one query row; then
// dq^ = w U and dw = U . q^. Thread (head group hg, dim group dg) keeps
// HI / 16 heads x DI / 16 dims of U in registers.
template <int HI, int DI>
struct KlGradUMap {
  static constexpr int HG = HI >= 16 ? HI / 16 : 1;          // heads per thread
  static constexpr int NHG = HI / HG;                        // head groups
  static constexpr int NDG = DI < kKlGradThreads / NHG ? DI : kKlGradThreads / NHG;
  static constexpr int DG = DI / NDG;                        // dims per thread
  static constexpr int THREADS = NHG * NDG;
  static_assert(NHG * HG == HI && NDG * DG == DI && THREADS % 32 == 0, "thread map");
  static_assert(NDG <= 32 && (NDG & (NDG - 1)) == 0, "a head group's threads share a warp");
};

template <int HI, int DI>
__global__ void __launch_bounds__(kKlGradThreads) kl_grad_u_kernel(KlGradParams p) {
  using Map = KlGradUMap<HI, DI>;
  constexpr int HG = Map::HG, NDG = Map::NDG, DG = Map::DG, NT = Map::THREADS;
  __shared__ float ks_val[kKlKeysPerStep][DI];      // k^ of the staged keys
  __shared__ float coef[kKlKeysPerStep];            // g[t, s] (0 past the row)
  __shared__ unsigned long long bits[kKlKeysPerStep];
  const int r = blockIdx.x, b = blockIdx.y;
  const int t = p.row_begin + r;
  const int pos = (p.q_pos0 ? p.q_pos0[b] : 0) + t;
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int n_vis = max(0, min(pos + 1, kvl));
  const int hg = threadIdx.x / NDG, dg = threadIdx.x % NDG;
  float acc[HG][DG];
#pragma unroll
  for (int a = 0; a < HG; ++a)
#pragma unroll
    for (int c = 0; c < DG; ++c) acc[a][c] = 0.f;
  const size_t row_off = (static_cast<size_t>(b) * p.rows + r) * p.n_kv;
  for (int s0 = 0; s0 < n_vis; s0 += kKlKeysPerStep) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKlKeysPerStep * DI; i += NT) {
      const int kk = i / DI, d = i % DI, s = s0 + kk;
      float v = 0.f;
      if (s < n_vis) {
        const size_t kr = static_cast<size_t>(b) * p.n_kv + s;
        v = e4m3_to_float(p.k_fp8[kr * DI + d]) * p.k_scale[kr];
      }
      ks_val[kk][d] = v;
    }
    if (threadIdx.x < kKlKeysPerStep) {
      const int s = s0 + threadIdx.x;
      coef[threadIdx.x] = s < n_vis ? p.g[row_off + s] : 0.f;
      bits[threadIdx.x] = s < n_vis ? p.signs[row_off + s] : 0ull;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKlKeysPerStep; ++kk) {
      const float c = coef[kk];
      const unsigned long long m = bits[kk];
      float kv[DG];
#pragma unroll
      for (int cdx = 0; cdx < DG; ++cdx) kv[cdx] = ks_val[kk][dg * DG + cdx];
#pragma unroll
      for (int a = 0; a < HG; ++a) {
        const float ca = ((m >> (hg * HG + a)) & 1ull) ? c : 0.f;
#pragma unroll
        for (int cdx = 0; cdx < DG; ++cdx) acc[a][cdx] = fmaf(ca, kv[cdx], acc[a][cdx]);
      }
    }
  }
  // dq^ = w U; dw = U . q^ (a sum over the NDG threads of each head group)
  const size_t qrow = static_cast<size_t>(b) * p.n_q + t;
#pragma unroll
  for (int a = 0; a < HG; ++a) {
    const int j = hg * HG + a;
    const float wj = p.w[qrow * HI + j], qsj = p.q_scale[qrow * HI + j];
    float part = 0.f;
#pragma unroll
    for (int cdx = 0; cdx < DG; ++cdx) {
      const int d = dg * DG + cdx;
      p.dq[(qrow * HI + j) * DI + d] = wj * acc[a][cdx];
      part = fmaf(acc[a][cdx], e4m3_to_float(p.q_fp8[(qrow * HI + j) * DI + d]) * qsj, part);
    }
    // the NDG dim groups of a head group are consecutive lanes
#pragma unroll
    for (int o = NDG / 2; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (dg == 0) p.dw[qrow * HI + j] = part;
  }
}

// dk^[s] partial over a split of the chunk's rows: sum over rows t (s visible
// to t) and heads j of g[t,s] w[t,j] [x > 0] q^[t,j]. Grid (key tiles of KT,
// row splits, batch); thread (key group, dim group) keeps KPT keys x DPT
// dims. Partials go to part[split] and kl_grad_k_reduce_kernel adds them to
// dk in split order, so the sum is the same on every call.
template <int HI, int DI>
struct KlGradKMap {
  static constexpr int KT = 64;                              // keys per CTA
  static constexpr int DPT = 8;                              // dims per thread
  static constexpr int NDG = DI / DPT;                       // dim groups
  static constexpr int NKG = kKlGradThreads / NDG;           // key groups
  static constexpr int KPT = KT / NKG;                       // keys per thread
  static_assert(NDG * DPT == DI && NKG * KPT == KT && KPT >= 1, "thread map");
  // dynamic shared memory: q^ [HI][DI], a [HI][KT], g [KT], masks [KT]
  static constexpr int SMEM_BYTES = (HI * DI + HI * KT + KT) * 4 + KT * 8;
};

template <int HI, int DI>
__global__ void __launch_bounds__(kKlGradThreads) kl_grad_k_kernel(KlGradParams p, float* part,
                                                                   int32_t n_split) {
  using Map = KlGradKMap<HI, DI>;
  constexpr int KT = Map::KT, DPT = Map::DPT, NDG = Map::NDG, KPT = Map::KPT;
  extern __shared__ __align__(16) float kl_k_smem[];
  float (*qv)[DI] = reinterpret_cast<float (*)[DI]>(kl_k_smem);          // q^ of the current row
  float (*a_s)[KT] = reinterpret_cast<float (*)[KT]>(kl_k_smem + HI * DI); // g w [x > 0]
  float* g_s = kl_k_smem + HI * DI + HI * KT;                             // g[t, s] of the tile
  unsigned long long* m_s =                                               // their sign masks
      reinterpret_cast<unsigned long long*>(kl_k_smem + HI * DI + HI * KT + KT);
  const int tile = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int s0 = tile * KT;
  const int kg = threadIdx.x / NDG, dg = threadIdx.x % NDG;
  const int kvl = min(p.kv_len ? p.kv_len[b] : p.n_kv, p.n_kv);
  const int pos0 = p.q_pos0 ? p.q_pos0[b] : 0;
  const int r_lo = static_cast<int>((static_cast<int64_t>(p.rows) * split) / n_split);
  const int r_hi = static_cast<int>((static_cast<int64_t>(p.rows) * (split + 1)) / n_split);
  float acc[KPT][DPT];
#pragma unroll
  for (int kk = 0; kk < KPT; ++kk)
#pragma unroll
    for (int c = 0; c < DPT; ++c) acc[kk][c] = 0.f;
  for (int r = r_lo; r < r_hi; ++r) {
    const int t = p.row_begin + r;
    const int pos = pos0 + t;
    if (pos < s0 || s0 >= kvl) continue;   // no key of the tile is visible to this row (uniform)
    const size_t qrow = static_cast<size_t>(b) * p.n_q + t;
    __syncthreads();
    for (int i = threadIdx.x; i < HI * DI; i += kKlGradThreads) {
      const int j = i / DI;
      qv[j][i % DI] = e4m3_to_float(p.q_fp8[qrow * HI * DI + i]) * p.q_scale[qrow * HI + j];
    }
    if (threadIdx.x < KT) {
      const int ss = s0 + threadIdx.x;
      const bool vis = ss <= pos && ss < kvl && ss < p.n_kv;
      const size_t o = (static_cast<size_t>(b) * p.rows + r) * p.n_kv + ss;
      g_s[threadIdx.x] = vis ? p.g[o] : 0.f;
      m_s[threadIdx.x] = vis ? p.signs[o] : 0ull;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < KT * HI; i += kKlGradThreads) {
      const int j = i / KT, kk = i % KT;
      a_s[j][kk] = ((m_s[kk] >> j) & 1ull) ? g_s[kk] * p.w[qrow * HI + j] : 0.f;
    }
    __syncthreads();
#pragma unroll 2
    for (int j = 0; j < HI; ++j) {
      float qd[DPT], av[KPT];
#pragma unroll
      for (int c = 0; c < DPT; c += 4) {
        const float4 v = *reinterpret_cast<const float4*>(&qv[j][dg * DPT + c]);
        qd[c] = v.x; qd[c + 1] = v.y; qd[c + 2] = v.z; qd[c + 3] = v.w;
      }
#pragma unroll
      for (int kk = 0; kk < KPT; ++kk) av[kk] = a_s[j][kg * KPT + kk];
#pragma unroll
      for (int kk = 0; kk < KPT; ++kk)
#pragma unroll
        for (int c = 0; c < DPT; ++c) acc[kk][c] = fmaf(av[kk], qd[c], acc[kk][c]);
    }
  }
  // part[split, b, s, :] (the reduce kernel reads only keys < n_kv)
#pragma unroll
  for (int kk = 0; kk < KPT; ++kk) {
    const int s = s0 + kg * KPT + kk;
    if (s < p.n_kv) {
      float* dst = part + ((static_cast<size_t>(split) * gridDim.z + b) * p.n_kv + s) * DI + dg * DPT;
#pragma unroll
      for (int c = 0; c < DPT; c += 4)
        *reinterpret_cast<float4*>(dst + c) =
            make_float4(acc[kk][c], acc[kk][c + 1], acc[kk][c + 2], acc[kk][c + 3]);
    }
  }
}

// dk[i] += sum over splits (in order) of part[split, i], i over B * n_kv * DI.
__global__ void kl_grad_k_reduce_kernel(const float* part, float* dk, int64_t n, int32_t n_split) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = dk[i];
    for (int sp = 0; sp < n_split; ++sp) v += part[sp * n + i];
    dk[i] = v;
  }
}

}  // namespace dsa

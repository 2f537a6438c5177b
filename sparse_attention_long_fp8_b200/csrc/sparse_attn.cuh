// Sparse MQA attention over selected latent rows (page "DeepseekV3.2 拆解",
// section "核心组件 / 细粒度 Token 选择机制", eq. u_t = Attn(h_t, {c_s | I_{t,s}
// in Top-k(I_{t,:})}); latent row = 512 value dims + 64 RoPE dims, page
// "DeepSeek architecture", section 1.1).
//
// This file holds the attention parameters shared by both attention kernels,
// the split-K combine, and the general kernel used for the small shape
// (64-d latent, 8 heads): the 576/512 latent runs sparse_attn_vh_kernel.
//
// One CTA handles one query row (all H heads as the M = 128 rows of the MMA,
// zero-padded), one range of selection slots (split-K for short query
// counts) and one slice of the value dims (VSPLIT slices).
//
//   producer warps 0-3  cp.async-gather the selected latent rows (16-byte
//                       chunks, zero-fill for empty slots) into a 128B-swizzled
//                       K-major layout, NK rows per block, 2-stage ring; the
//                       query tile (128 x D_qk bf16) is staged once.
//   MMA warp 4          S = Q C^T (kind::f16, SS, K = D_qk) into a TMEM buffer,
//                       then O += P V with P read from TMEM (TS form) and V the
//                       same gathered rows read MN-major.
//   epilogue warps 5-8  thread = head row: online softmax in the log2 domain
//                       with lazy rescaling (O is rescaled in TMEM only when
//                       the running max grows by more than 2^8), P packed to
//                       bf16 into TMEM, final O / l and LSE.
#pragma once

#include <cuda_bf16.h>

#include "layout.cuh"
#include "ptx.cuh"

namespace dsa {

struct AttnParams {
  const __nv_bfloat16* q;   // [B, n_q, H, DQK]
  const __nv_bfloat16* kv;  // [pool rows, DQK] latent rows (contiguous: [B, n_kv, DQK])
  KeyMap km;                // pool row of each key
  const int32_t* indices;   // [B, n_q, topk]
  void* out;                // [B, n_q, H, DV] fp32 or bf16
  float* lse;               // [B, n_q, H] or null
  float* part_o;            // split mode: [B*n_q, splits, H, DV]
  float* part_lse;          // split mode: [B*n_q, splits, H]
  int32_t B, n_q, n_kv, topk, H;
  int32_t splits, slots_per_split;   // slots_per_split is a multiple of NK
  int32_t out_bf16;
  float scale_log2;         // softmax_scale * log2(e)
};

template <int DQK, int DV, int VSPLIT>
struct AttnTile {
  static constexpr int NK = 32;                 // latent rows per block
  static constexpr int M = 128;                 // head rows (zero-padded past H)
  static constexpr int NDB = DQK / 64;          // 64-dim (128-byte) blocks per row
  static constexpr int VH = DV / VSPLIT;        // value dims per CTA
  static constexpr int VDB = VH / 64;
  static constexpr int Q_BYTES = M * DQK * 2;
  static constexpr int C_BYTES = NK * DQK * 2;
  static constexpr int STAGES = 2;
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 288;
  static constexpr int COL_O = 0;
  static constexpr int COL_S = VH;              // 2 x NK columns
  static constexpr int COL_P = VH + 2 * NK;     // 2 x NK/2 columns
  static constexpr int COLS_USED = VH + 3 * NK;
  static constexpr uint32_t TMEM_COLS = COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_C = Q_BYTES;
  static constexpr int OFF_BAR = OFF_C + STAGES * C_BYTES;
  static constexpr int NUM_BARS = 13;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(DQK % 64 == 0 && VH % 64 == 0 && VH <= 256, "tile shape");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int DQK, int DV, int VSPLIT>
__global__ void __launch_bounds__(288, 1)
    sparse_attn_kernel(AttnParams p) {
  using T = AttnTile<DQK, DV, VSPLIT>;
  constexpr int NK = T::NK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* q_smem = smem + T::OFF_Q;
  uint8_t* c_smem = smem + T::OFF_C;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* c_full = bars + 1;
  uint64_t* c_empty = bars + 3;
  uint64_t* s_full = bars + 5;
  uint64_t* s_free = bars + 7;
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int per_row = p.splits * VSPLIT;
  const int row = blockIdx.x / per_row;               // b * n_q + t
  const int split = (blockIdx.x % per_row) / VSPLIT;
  const int half = blockIdx.x % VSPLIT;
  const int b = row / p.n_q;
  const int slot_begin = split * p.slots_per_split;
  const int slot_end = min(p.topk, slot_begin + p.slots_per_split);
  const int n_blocks = max(0, (slot_end - slot_begin + NK - 1) / NK);
  const int32_t* row_idx = p.indices + static_cast<size_t>(row) * p.topk;

  if (threadIdx.x == 0) {
    mbar_init(q_full, T::PRODUCERS);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c_full[s], T::PRODUCERS);
      mbar_init(&c_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
      mbar_init(&pv_done[s], 1);
    }
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
    // ------------------------------------------------------------ producers
    const int tid = threadIdx.x;
    const uint32_t q_addr = smem_u32(q_smem);
    const __nv_bfloat16* q_row = p.q + static_cast<size_t>(row) * p.H * DQK;
    for (int c = tid; c < T::M * T::NDB * 8; c += T::PRODUCERS) {
      const int h = c / (T::NDB * 8), rem = c % (T::NDB * 8);
      const int db = rem >> 3, ch = rem & 7;
      const uint32_t dst = q_addr + db * (T::M * 128) + h * 128 + ((ch ^ (h & 7)) << 4);
      const bool ok = h < p.H;
      const void* src = ok ? static_cast<const void*>(q_row + static_cast<size_t>(h) * DQK + db * 64 + ch * 8)
                           : static_cast<const void*>(p.q);
      cp_async_16(dst, src, ok ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();
    mbar_arrive(q_full);

    bool ok = true;
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int st = i & 1;
      ok = mbar_wait(&c_empty[st], ((i >> 1) & 1) ^ 1);
      if (!ok) break;
      const uint32_t c_addr = smem_u32(c_smem + st * T::C_BYTES);
      const int slot0 = slot_begin + i * NK;
      for (int c = tid; c < NK * T::NDB * 8; c += T::PRODUCERS) {
        const int j = c / (T::NDB * 8), rem = c % (T::NDB * 8);
        const int db = rem >> 3, ch = rem & 7;
        const int slot = slot0 + j;
        const int idx = slot < slot_end ? row_idx[slot] : -1;
        const int64_t krow = (idx >= 0 && idx < p.n_kv) ? p.km.row(b, idx, p.n_kv) : -1;
        const bool valid = krow >= 0;
        const uint32_t dst = c_addr + db * (NK * 128) + j * 128 + ((ch ^ (j & 7)) << 4);
        const void* src = valid ? static_cast<const void*>(p.kv + krow * DQK + db * 64 + ch * 8)
                                : static_cast<const void*>(p.kv);
        cp_async_16(dst, src, valid ? 16u : 0u);
      }
      // Block i is published as soon as its rows land: the MMA warp needs
      // S(i) before it can issue PV(i-1), which is what frees the next stage.
      cp_async_commit();
      cp_async_wait<0>();
      fence_proxy_async_smem();
      mbar_arrive(&c_full[st]);
    }
    cp_async_wait<0>();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
      constexpr uint32_t idesc_pv = umma_idesc(128, T::VH, 1u, 1u, 0u, 1u);
      const uint32_t q_addr = smem_u32(q_smem);
      bool ok = mbar_wait(q_full, 0);
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(c_smem + pb * T::C_BYTES) + (half * T::VDB) * (NK * 128);
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          const uint64_t bd = umma_desc(v_addr + kk * 2048, NK * 128, 1024, 2);
          umma_bf16_ts(tmem_base + T::COL_O, tmem_base + T::COL_P + pb * (NK / 2) + kk * 8, bd,
                       idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&c_empty[pb]);
        umma_commit(&pv_done[pb]);
        return true;
      };
      for (int i = 0; i < n_blocks && ok; ++i) {
        const int st = i & 1;
        ok = mbar_wait(&c_full[st], (i >> 1) & 1) && mbar_wait(&s_free[st], ((i >> 1) & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t c_addr = smem_u32(c_smem + st * T::C_BYTES);
        const uint32_t d_tmem = tmem_base + T::COL_S + st * NK;
#pragma unroll 1
        for (int db = 0; db < T::NDB; ++db) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = umma_desc(q_addr + db * (T::M * 128) + kk * 32, 16, 1024, 2);
            const uint64_t bd = umma_desc(c_addr + db * (NK * 128) + kk * 32, 16, 1024, 2);
            umma_bf16_ss(d_tmem, a, bd, idesc_s, (db | kk) ? 1u : 0u);
          }
        }
        umma_commit(&s_full[st]);
        if (i > 0) ok = issue_pv(i - 1);
      }
      if (ok && n_blocks > 0) issue_pv(n_blocks - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;                       // head row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float m_used = -INFINITY;   // running max (log2 domain) the P values are relative to
    float l = 0.f;              // sum of the fp32 p: gives the LSE
    float l_mma = 0.f;          // sum of the bf16-rounded p the PV MMA used: normalises O
    bool ok = true;
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int sb = i & 1;
      const int slot = slot_begin + i * NK + lane;
      const int idx = slot < slot_end ? row_idx[slot] : -1;
      const uint32_t vmask = __ballot_sync(0xffffffffu, idx >= 0 && idx < p.n_kv);
      ok = mbar_wait(&s_full[sb], (i >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem_base + lane_addr + T::COL_S + sb * NK, sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      float z[32];
      float bmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        z[j] = ((vmask >> j) & 1u) ? __uint_as_float(sr[j]) * p.scale_log2 : -INFINITY;
        bmax = fmaxf(bmax, z[j]);
      }
      const bool grow = bmax > m_used + 8.0f;
      const float m_new = grow ? bmax : m_used;
      // P buffer sb was read by PV(i-2) and O is written by PV(i-1): wait for PV(i-1).
      if (i > 0) {
        ok = mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
          const float alpha = grow ? exp2f(m_used - m_new) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < T::VH; c += 16) {
            uint32_t o[16];
            tmem_ld16(tmem_base + lane_addr + T::COL_O + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st16(tmem_base + lane_addr + T::COL_O + c, o);
          }
          tmem_wait_st();
          l *= alpha;
          l_mma *= alpha;
        }
      }
      m_used = m_new;
      uint32_t pk[16];
      float lsum = 0.f, lsum_mma = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float p0 = exp2f(z[2 * j] - m_used);
        const float p1 = exp2f(z[2 * j + 1] - m_used);
        const __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
        lsum += p0 + p1;
        lsum_mma += __low2float(pb2) + __high2float(pb2);
        pk[j] = *reinterpret_cast<const uint32_t*>(&pb2);
      }
      // empty block (no valid slot and no previous max): exp2(-inf - (-inf)) = NaN guard
      if (m_used == -INFINITY) {
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[j] = 0u;
        lsum = 0.f;
        lsum_mma = 0.f;
      }
      l += lsum;
      l_mma += lsum_mma;
      tmem_st16(tmem_base + lane_addr + T::COL_P + sb * (NK / 2), pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    if (ok && n_blocks > 0) {
      ok = mbar_wait(&pv_done[(n_blocks - 1) & 1], ((n_blocks - 1) >> 1) & 1);
      tc_fence_after();
    }
    // O / sum(rounded p) is an exact convex combination of the V rows with
    // weights perturbed by the bf16 rounding of p (a component shared by the
    // rows cancels); the LSE keeps the unrounded sum.
    const bool has = ok && l > 0.f && l_mma > 0.f;
    const float inv_l = has ? 1.0f / l_mma : 0.f;
    const uint32_t keep = has ? 0xffffffffu : 0u;   // masks undefined TMEM when empty
    const float lse_v = has ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (p.splits == 1) {
      const size_t o_off = (static_cast<size_t>(row) * p.H + h) * DV + half * T::VH;
#pragma unroll 1
      for (int c = 0; c < T::VH; c += 16) {
        uint32_t o[16];
        tmem_ld16(tmem_base + lane_addr + T::COL_O + c, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] &= keep;
        if (h < p.H) {
          if (p.out_bf16) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + o_off + c;
            uint32_t pkd[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[2 * j]) * inv_l,
                                                             __uint_as_float(o[2 * j + 1]) * inv_l);
              pkd[j] = *reinterpret_cast<const uint32_t*>(&v);
            }
            reinterpret_cast<uint4*>(dst)[0] = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
            reinterpret_cast<uint4*>(dst)[1] = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
          } else {
            float* dst = static_cast<float*>(p.out) + o_off + c;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              reinterpret_cast<float4*>(dst)[j / 4] =
                  make_float4(__uint_as_float(o[j]) * inv_l, __uint_as_float(o[j + 1]) * inv_l,
                              __uint_as_float(o[j + 2]) * inv_l, __uint_as_float(o[j + 3]) * inv_l);
          }
        }
      }
      if (half == 0 && p.lse && h < p.H) p.lse[static_cast<size_t>(row) * p.H + h] = lse_v;
    } else {
      const size_t part = static_cast<size_t>(row) * p.splits + split;
      float* dst_row = p.part_o + (part * p.H + h) * DV + half * T::VH;
#pragma unroll 1
      for (int c = 0; c < T::VH; c += 16) {
        uint32_t o[16];
        tmem_ld16(tmem_base + lane_addr + T::COL_O + c, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j] &= keep;
        if (h < p.H) {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            reinterpret_cast<float4*>(dst_row + c)[j / 4] =
                make_float4(__uint_as_float(o[j]) * inv_l, __uint_as_float(o[j + 1]) * inv_l,
                            __uint_as_float(o[j + 2]) * inv_l, __uint_as_float(o[j + 3]) * inv_l);
        }
      }
      if (half == 0 && h < p.H) p.part_lse[part * p.H + h] = lse_v;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

// Merge split-K partials: lse = log sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s.
__global__ void attn_combine_kernel(AttnParams p, int DV) {
  const int row = blockIdx.x;
  const int h = blockIdx.y;
  const size_t base = static_cast<size_t>(row) * p.splits;
  float m = -INFINITY;
  for (int s = 0; s < p.splits; ++s) m = fmaxf(m, p.part_lse[(base + s) * p.H + h]);
  float wsum = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const float ls = p.part_lse[(base + s) * p.H + h];
    wsum += (ls == -INFINITY) ? 0.f : __expf(ls - m);
  }
  const float lse = (wsum > 0.f) ? m + __logf(wsum) : -INFINITY;
  for (int d = threadIdx.x; d < DV; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float ls = p.part_lse[(base + s) * p.H + h];
      if (ls == -INFINITY) continue;
      acc += __expf(ls - lse) * p.part_o[((base + s) * p.H + h) * DV + d];
    }
    const size_t o = (static_cast<size_t>(row) * p.H + h) * DV + d;
    if (p.out_bf16)
      static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(acc);
    else
      static_cast<float*>(p.out)[o] = acc;
  }
  if (threadIdx.x == 0 && p.lse) p.lse[static_cast<size_t>(row) * p.H + h] = lse;
}

}  // namespace dsa

// Sparse MQA attention over the selected 576-d latent rows, one 2-CTA
// cluster per query row (page "DeepseekV3.2 拆解", section "核心组件 /
// 细粒度 Token 选择机制", eq. u_t; latent = 512 value dims + 64 RoPE dims,
// page "DeepSeek architecture", section 1.1).
//
// The pair splits the 576 latent dims: CTA 0 owns dims [0, 256), CTA 1 owns
// [256, 576). Each CTA
//   * gathers only its dims of each selected row (512 or 640 bytes) through
//     an 8-stage cp.async ring whose stages complete on mbarriers
//     (cp.async.mbarrier.arrive.noinc), so many blocks are in flight;
//   * keeps its slice of Q (128 heads x 256/320 dims) in TMEM and computes the
//     partial logits S_r = Q_r C_r^T with A read from TMEM;
//   * sends its fp32 S_r to the peer with st.async (completing tx bytes on the
//     peer's mbarrier) and adds the peer's partial: both CTAs then hold the
//     same S = S_0 + S_1 and run the same online softmax;
//   * accumulates O for the value dims it already holds (CTA 0: 0..255,
//     CTA 1: 256..511) with P read from TMEM.
// Nothing is gathered twice and no logit is computed twice. TMEM per CTA:
// O 256 columns, Q slice 160, S 2 x 32, P 2 x 16 = 512.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {

struct PairTile {
  static constexpr int NK = 32;                 // latent rows per block
  static constexpr int M = 128;                 // head rows
  static constexpr int DQK = 576, DV = 512, VH = 256;
  static constexpr int NDB_MAX = 5;             // 64-dim blocks held by CTA 1
  static constexpr int STAGE_BYTES = NK * NDB_MAX * 128;
  static constexpr int STAGES = 8;
  static constexpr int X_BYTES = M * NK * 4;    // one exchanged fp32 partial
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 288;
  static constexpr int COL_O = 0, COL_Q = 256, COL_S = 416, COL_P = 480;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int OFF_C = 0;
  static constexpr int OFF_X = STAGES * STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_X + 2 * X_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 13;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned");
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(288, 1)
    sparse_attn_pair_kernel(AttnParams p) {
  using T = PairTile;
  constexpr int NK = T::NK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* c_smem = smem + T::OFF_C;
  uint8_t* x_smem = smem + T::OFF_X;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* c_full = bars;
  uint64_t* c_empty = bars + T::STAGES;
  uint64_t* s_full = bars + 2 * T::STAGES;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* pv_done = s_full + 6;
  uint64_t* x_full = s_full + 8;    // peer's partial landed in my x buffer
  uint64_t* x_free = s_full + 10;   // peer has read the partial I wrote into its x buffer
  uint64_t* q_ready = s_full + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int row = pair / p.splits;                  // b * n_q + t
  const int split = pair % p.splits;
  const int b = row / p.n_q;
  const int ndb = rank == 0 ? 4 : 5;                // 64-dim blocks this CTA holds
  const int dim0 = rank == 0 ? 0 : 256;             // first latent dim this CTA holds
  const int slot_begin = split * p.slots_per_split;
  const int slot_end = min(p.topk, slot_begin + p.slots_per_split);
  const int n_blocks = max(0, (slot_end - slot_begin + NK - 1) / NK);
  const int32_t* row_idx = p.indices + static_cast<size_t>(row) * p.topk;
  const __nv_bfloat16* kv_b = p.kv + static_cast<size_t>(b) * p.n_kv * T::DQK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&c_full[s], T::PRODUCERS);
      mbar_init(&c_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
      mbar_init(&pv_done[s], 1);
      mbar_init(&x_full[s], 1);
      mbar_init(&x_free[s], 4);
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
  // The peer's barriers must be initialised before any remote access.
  cluster_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ gather
    // Warp w copies keys w, w+4, ..., w+28 of each block; the 32 lanes take
    // consecutive 16-byte chunks of one row (a 512- or 640-byte run). Lane j
    // holds the index of key j, loaded one block ahead and broadcast.
    const int per_key = ndb * 8;
    auto load_idx = [&](int blk) -> int {
      const int slot = slot_begin + blk * NK + lane;
      return (blk < n_blocks && slot < slot_end) ? row_idx[slot] : -1;
    };
    int idx_next = load_idx(0);
    bool ok = true;
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int st = i % T::STAGES;
      const int idx_cur = idx_next;
      idx_next = load_idx(i + 1);
      ok = mbar_wait(&c_empty[st], ((i / T::STAGES) & 1) ^ 1);
      if (!ok) break;
      const uint32_t c_addr = smem_u32(c_smem + st * T::STAGE_BYTES);
#pragma unroll
      for (int m = 0; m < NK / 4; ++m) {
        const int j = warp + 4 * m;
        const int idx = __shfl_sync(0xffffffffu, idx_cur, j);
        const bool valid = idx >= 0 && idx < p.n_kv;
        const __nv_bfloat16* row_src = kv_b + static_cast<size_t>(valid ? idx : 0) * T::DQK + dim0;
        const uint32_t row_dst = c_addr + j * 128;
        for (int c = lane; c < per_key; c += 32) {
          const int db = c >> 3, ch = c & 7;
          cp_async_16(row_dst + db * (NK * 128) + ((ch ^ (j & 7)) << 4), row_src + c * 8,
                      valid ? 16u : 0u);
        }
      }
      cp_async_arrive_noinc(&c_full[st]);
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
      constexpr uint32_t idesc_pv = umma_idesc(128, T::VH, 1u, 1u, 0u, 1u);
      bool ok = mbar_wait(q_ready, 0);
      tc_fence_after();
      auto issue_pv = [&](int j) -> bool {
        const int pb = j & 1;
        const int st = j % T::STAGES;
        if (!mbar_wait(&p_full[pb], (j >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(c_smem + st * T::STAGE_BYTES);  // local blocks 0-3 = V
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          const uint64_t bd = umma_desc(v_addr + kk * 2048, NK * 128, 1024, 2);
          umma_bf16_ts(tmem_base + T::COL_O, tmem_base + T::COL_P + pb * (NK / 2) + kk * 8, bd,
                       idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&c_empty[st]);
        umma_commit(&pv_done[pb]);
        return true;
      };
      for (int i = 0; i < n_blocks && ok; ++i) {
        const int st = i % T::STAGES;
        const int sb = i & 1;
        ok = mbar_wait(&c_full[st], (i / T::STAGES) & 1) &&
             mbar_wait(&s_free[sb], ((i >> 1) & 1) ^ 1);
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t c_addr = smem_u32(c_smem + st * T::STAGE_BYTES);
        const uint32_t d_tmem = tmem_base + T::COL_S + sb * NK;
#pragma unroll 1
        for (int db = 0; db < ndb; ++db) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = umma_desc(c_addr + db * (NK * 128) + kk * 32, 16, 1024, 2);
            umma_bf16_ts(d_tmem, tmem_base + T::COL_Q + db * 32 + kk * 8, bd, idesc_s,
                         (db | kk) ? 1u : 0u);
          }
        }
        umma_commit(&s_full[sb]);
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
    const bool expect_thread = threadIdx.x == 5 * 32;

    // This CTA's slice of Q into TMEM (A operand of the partial-logit MMA).
    {
      const __nv_bfloat16* qs =
          p.q + (static_cast<size_t>(row) * p.H + min(h, p.H - 1)) * T::DQK + dim0;
      for (int c = 0; c < ndb * 2; ++c) {
        uint32_t v[16];
        if (h < p.H) {
          const uint4* src = reinterpret_cast<const uint4*>(qs + c * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 u = src[k];
            v[4 * k] = u.x; v[4 * k + 1] = u.y; v[4 * k + 2] = u.z; v[4 * k + 3] = u.w;
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) v[k] = 0u;
        }
        tmem_st16(tmem_base + lane_addr + T::COL_Q + c * 16, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }

    const uint32_t x_own = smem_u32(x_smem);
    const uint32_t x_peer = mapa_shared(x_own, peer);
    const uint32_t x_full_peer = mapa_shared(smem_u32(x_full), peer);
    const uint32_t x_free_peer = mapa_shared(smem_u32(x_free), peer);
    const uint32_t row_off = static_cast<uint32_t>(h) * (NK * 4);

    float m_used = -INFINITY;
    float l = 0.f, l_mma = 0.f;
    bool ok = true;
    auto load_idx = [&](int blk) -> int {
      const int slot = slot_begin + blk * NK + lane;
      return (blk < n_blocks && slot < slot_end) ? row_idx[slot] : -1;
    };
    int idx_next = load_idx(0);
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int sb = i & 1;
      const int idx = idx_next;
      idx_next = load_idx(i + 1);
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

      // ---- exchange the partial logits with the peer
      if (expect_thread)
        mbar_arrive_expect_tx_u32(smem_u32(&x_full[sb]), static_cast<uint32_t>(T::X_BYTES));
      ok = mbar_wait(&x_free[sb], ((i >> 1) & 1) ^ 1);
      if (!ok) break;
      const uint32_t buf_off = static_cast<uint32_t>(sb * T::X_BYTES) + row_off;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_async_v4(x_peer + buf_off + ((j ^ (h & 7)) << 4), x_full_peer + sb * 8, sr[4 * j],
                    sr[4 * j + 1], sr[4 * j + 2], sr[4 * j + 3]);
      ok = mbar_wait(&x_full[sb], (i >> 1) & 1);
      if (!ok) break;
      float other[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 f = *reinterpret_cast<const float4*>(x_smem + sb * T::X_BYTES + row_off +
                                                          ((j ^ (h & 7)) << 4));
        other[4 * j] = f.x; other[4 * j + 1] = f.y; other[4 * j + 2] = f.z; other[4 * j + 3] = f.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(x_free_peer + sb * 8);

      float z[32];
      float bmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        // S = S_0 + S_1 in the same order on both CTAs: identical logits.
        const float mine = __uint_as_float(sr[j]);
        const float s = rank == 0 ? mine + other[j] : other[j] + mine;
        z[j] = ((vmask >> j) & 1u) ? s * p.scale_log2 : -INFINITY;
        bmax = fmaxf(bmax, z[j]);
      }
      const bool grow = bmax > m_used + 8.0f;
      const float m_new = grow ? bmax : m_used;
      // P buffer sb was last read by PV(i-2). O is touched only when the max
      // grew, and then PV(i-1) must have finished first.
      if (i > 1) {
        ok = mbar_wait(&pv_done[sb], ((i - 2) >> 1) & 1);
        if (!ok) break;
      }
      if (i > 0 && __any_sync(0xffffffffu, grow)) {
        ok = mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        {
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
    const bool has = ok && l > 0.f && l_mma > 0.f;
    const float inv_l = has ? 1.0f / l_mma : 0.f;
    const uint32_t keep = has ? 0xffffffffu : 0u;
    const float lse_v = has ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    const bool direct = p.splits == 1;
    float* dst_f32 = nullptr;
    __nv_bfloat16* dst_bf16 = nullptr;
    if (direct) {
      const size_t o_off = (static_cast<size_t>(row) * p.H + h) * T::DV + rank * T::VH;
      if (p.out_bf16) dst_bf16 = static_cast<__nv_bfloat16*>(p.out) + o_off;
      else dst_f32 = static_cast<float*>(p.out) + o_off;
    } else {
      const size_t part = static_cast<size_t>(row) * p.splits + split;
      dst_f32 = p.part_o + (part * p.H + h) * T::DV + rank * T::VH;
    }
#pragma unroll 1
    for (int c = 0; c < T::VH; c += 16) {
      uint32_t o[16];
      tmem_ld16(tmem_base + lane_addr + T::COL_O + c, o);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] &= keep;
      if (h < p.H) {
        if (dst_bf16) {
          uint32_t pkd[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[2 * j]) * inv_l,
                                                           __uint_as_float(o[2 * j + 1]) * inv_l);
            pkd[j] = *reinterpret_cast<const uint32_t*>(&v);
          }
          reinterpret_cast<uint4*>(dst_bf16 + c)[0] = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
          reinterpret_cast<uint4*>(dst_bf16 + c)[1] = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            reinterpret_cast<float4*>(dst_f32 + c)[j / 4] =
                make_float4(__uint_as_float(o[j]) * inv_l, __uint_as_float(o[j + 1]) * inv_l,
                            __uint_as_float(o[j + 2]) * inv_l, __uint_as_float(o[j + 3]) * inv_l);
        }
      }
    }
    if (rank == 0 && h < p.H) {
      if (direct) {
        if (p.lse) p.lse[static_cast<size_t>(row) * p.H + h] = lse_v;
      } else {
        p.part_lse[(static_cast<size_t>(row) * p.splits + split) * p.H + h] = lse_v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA may leave while its peer can still touch its shared memory.
  cluster_sync();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

}  // namespace dsa

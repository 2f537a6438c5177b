// Sparse MQA attention over the selected 576-d latent rows, one 2-CTA
// cluster per query row (page "DeepseekV3.2 拆解", section "核心组件 /
// 细粒度 Token 选择机制", eq. u_t; latent = 512 value dims + 64 RoPE dims,
// page "DeepSeek architecture", section 1.1).
//
// The pair splits the 576 latent dims: CTA 0 owns dims [0, 256), CTA 1 owns
// [256, 576). Each CTA
//   * gathers only its dims of each selected row (512 or 640 bytes) into a
//     3-stage ring of 64-row blocks (cp.async, completion on mbarriers);
//   * keeps its slice of Q (128 heads x 256/320 dims) in TMEM and computes the
//     partial logits S_r = Q_r C_r^T with A read from TMEM;
//   * sends its fp32 S_r to the peer with st.async (completing tx bytes on the
//     peer's mbarrier) and adds the peer's partial: both CTAs then hold the
//     same S = S_0 + S_1 and run the same online softmax;
//   * accumulates O for the value dims it already holds (CTA 0: 0..255,
//     CTA 1: 256..511) with P read from TMEM.
// Nothing is gathered twice and no logit is computed twice. TMEM per CTA:
// O 256 columns, Q slice 160, S 64, P 32 = 512.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {

struct PairTile {
  static constexpr int NK = 64;                 // latent rows per block
  static constexpr int M = 128;                 // head rows
  static constexpr int DQK = 576, DV = 512, VH = 256;
  static constexpr int NDB_MAX = 5;             // 64-dim blocks held by CTA 1
  static constexpr int STAGE_BYTES = NK * NDB_MAX * 128;
  static constexpr int STAGES = 3;
  static constexpr int X_BYTES = M * NK * 4;    // one exchanged fp32 partial
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 448;           // gather 0-3, S MMA 4, softmax 5-12, PV MMA 13
  static constexpr int SOFTMAX_WARPS = 8;       // two per TMEM lane quarter, 32 keys each
  static constexpr int COL_O = 0, COL_Q = 256, COL_S = 416, COL_P = 480;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int OFF_C = 0;
  static constexpr int OFF_X = STAGES * STAGE_BYTES;
  static constexpr int OFF_RED = OFF_X + 2 * X_BYTES;         // [2 parity][2 halves][128] fp32
  static constexpr int OFF_END = OFF_RED + 2 * 2 * M * 4;     // [half][l, l_mma][128] fp32
  static constexpr int OFF_BAR = OFF_END + 2 * 2 * M * 4;
  static constexpr int NUM_BARS = 2 * STAGES + 9 + 12;   // stages + 9 singles/pairs + red[8] + end[4]
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned");
};

// Warp roles: 0-3 gather the selected rows (cp.async, 16 bytes per thread);
// 4 issues the partial-logit MMAs (and owns TMEM); 5-12 exchange partials and
// run the softmax (two warps per TMEM lane quarter: a thread owns one head
// row and 32 of a block's 64 keys); 13 issues the PV MMAs. The two MMA issuers are separate threads so that
// S(i+1) is issued as soon as S(i) has been read, without waiting behind PV.
// The softmax warps read and send block i+1's partial before finishing block
// i, which hides the exchange round trip behind a block of softmax work.
// Blocks are 64 keys wide: a tcgen05.mma costs a fixed ~47 cycles at small N,
// so N = 64 logit tiles run the tensor pipe at about twice the N = 32 rate.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(448, 1)
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
  uint64_t* s_full = bars + 2 * T::STAGES;   // S tile written (one phase per block)
  uint64_t* s_free = s_full + 1;             // S tile read by the softmax warps
  uint64_t* p_full = s_full + 2;             // P tile written
  uint64_t* pv_done = s_full + 3;            // PV of the block finished (P tile free, O updated)
  uint64_t* x_full = s_full + 4;             // [2] peer's partial landed in my x buffer
  uint64_t* q_ready = s_full + 6;
  uint64_t* x_free = s_full + 7;             // [2] peer has read the partial I wrote into its buffer
  uint64_t* red_bar = s_full + 9;            // [parity][quarter]: both warps wrote their half max
  uint64_t* end_bar = s_full + 17;           // [quarter]: both warps wrote their l, l_mma
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
    mbar_init(s_full, 1);
    mbar_init(s_free, T::SOFTMAX_WARPS);
    mbar_init(p_full, T::SOFTMAX_WARPS);
    mbar_init(pv_done, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_free[s], T::SOFTMAX_WARPS);
    }
    mbar_init(q_ready, T::SOFTMAX_WARPS);
    for (int s = 0; s < 12; ++s) mbar_init(&red_bar[s], 2);
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
    // Flat mapping: 16-byte piece c of a block (c = thread + 128 m) is piece
    // c % per_key of key c / per_key. Each thread first loads the row indices
    // of all its pieces, then issues all its copies back to back: the copies
    // of a thread are independent, so they overlap fully.
    auto gather_block = [&](auto per_key_c, int i, uint32_t c_addr) {
      constexpr int PER_KEY = decltype(per_key_c)::value;
      constexpr int PER = NK * PER_KEY / T::PRODUCERS;
      const int slot0 = slot_begin + i * NK;
      int keys[PER];
#pragma unroll
      for (int m = 0; m < PER; ++m) {
        const int c = threadIdx.x + T::PRODUCERS * m;
        const int slot = slot0 + c / PER_KEY;
        const int idx = slot < slot_end ? row_idx[slot] : -1;
        keys[m] = (idx >= 0 && idx < p.n_kv) ? idx : -1;
      }
#pragma unroll
      for (int m = 0; m < PER; ++m) {
        const int c = threadIdx.x + T::PRODUCERS * m;
        const int j = c / PER_KEY, piece = c - j * PER_KEY;
        const int db = piece >> 3, ch = piece & 7;
        const bool valid = keys[m] >= 0;
        cp_async_16(c_addr + db * (NK * 128) + j * 128 + ((ch ^ (j & 7)) << 4),
                    kv_b + static_cast<size_t>(valid ? keys[m] : 0) * T::DQK + dim0 + piece * 8,
                    valid ? 16u : 0u);
      }
    };
    bool ok = true;
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int st = i % T::STAGES;
      ok = mbar_wait(&c_empty[st], ((i / T::STAGES) & 1) ^ 1);
      if (!ok) break;
      const uint32_t c_addr = smem_u32(c_smem + st * T::STAGE_BYTES);
      if (rank == 0) gather_block(std::integral_constant<int, 32>{}, i, c_addr);
      else gather_block(std::integral_constant<int, 40>{}, i, c_addr);
      cp_async_arrive_noinc(&c_full[st]);
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ S = Q_r C_r^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
      bool ok = mbar_wait(q_ready, 0);
      tc_fence_after();
      for (int i = 0; i < n_blocks && ok; ++i) {
        const int st = i % T::STAGES;
        ok = mbar_wait(&c_full[st], (i / T::STAGES) & 1) && mbar_wait(s_free, (i & 1) ^ 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t c_addr = smem_u32(c_smem + st * T::STAGE_BYTES);
#pragma unroll 1
        for (int db = 0; db < ndb; ++db) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = umma_desc(c_addr + db * (NK * 128) + kk * 32, 16, 1024, 2);
            umma_bf16_ts(tmem_base + T::COL_S, tmem_base + T::COL_Q + db * 32 + kk * 8, bd,
                         idesc_s, (db | kk) ? 1u : 0u);
          }
        }
        umma_commit(s_full);
      }
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ O += P V issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = umma_idesc(128, T::VH, 1u, 1u, 0u, 1u);
      for (int j = 0; j < n_blocks; ++j) {
        const int st = j % T::STAGES;
        if (!mbar_wait(p_full, j & 1)) break;
        tc_fence_after();
        // P(j) exists only after S(j) was read, so S(j) is complete: when
        // PV(j) completes, both readers of stage st are done.
        const uint32_t v_addr = smem_u32(c_smem + st * T::STAGE_BYTES);  // local blocks 0-3 = V
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          const uint64_t bd = umma_desc(v_addr + kk * 2048, NK * 128, 1024, 2);
          umma_bf16_ts(tmem_base + T::COL_O, tmem_base + T::COL_P + kk * 8, bd, idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&c_empty[st]);
        umma_commit(pv_done);
      }
    }
    __syncwarp();
  } else if (warp >= 5 && warp <= 12) {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int half = (warp - 5) >> 2;                        // which 32 keys of a block
    const int h = quarter * 32 + lane;                       // head row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const bool expect_thread = threadIdx.x == 5 * 32;
    float* red = reinterpret_cast<float*>(smem + T::OFF_RED);   // [parity][half][128]

    // This CTA's slice of Q into TMEM (A operand of the partial-logit MMA);
    // the two warps of a quarter take alternate 16-column chunks.
    {
      const __nv_bfloat16* qs =
          p.q + (static_cast<size_t>(row) * p.H + min(h, p.H - 1)) * T::DQK + dim0;
      for (int c = half; c < ndb * 2; c += 2) {
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

    const uint32_t x_peer = mapa_shared(smem_u32(x_smem), peer);
    const uint32_t x_full_peer = mapa_shared(smem_u32(x_full), peer);
    const uint32_t x_free_peer = mapa_shared(smem_u32(x_free), peer);
    const uint32_t row_off = static_cast<uint32_t>(h) * (NK * 4);

    float m_used = -INFINITY;   // running max (log2 domain) the P values are relative to
    float l = 0.f;              // this warp's share of the sum of the fp32 p (LSE)
    float l_mma = 0.f;          // ... of the bf16-rounded p the PV MMA used (normalises O)
    bool ok = true;
    auto load_idx = [&](int blk) -> int {
      const int slot = slot_begin + blk * NK + half * 32 + lane;
      return (blk < n_blocks && slot < slot_end) ? row_idx[slot] : -1;
    };
    int idx_next = load_idx(0);

    // Per block i the softmax warps run four steps:
    //   load(i)  this CTA's partial logits (32 keys) from TMEM, free the S tile;
    //   send(i)  those partials to the peer (st.async into its x buffer);
    //   max(i)   add the peer's partials, block max over the 64 keys (shared
    //            with the partner warp of the same lane quarter);
    //   soft(i)  online softmax, P(i) into TMEM, hand the block to PV.
    // They are interleaved as load(i+1), max(i), soft(i), send(i+1): block
    // i+1's partials travel while the next S tile is computed, and the
    // release-ordered arrives of max(i) and soft(i) (row-max hand-off, P
    // ready) are not queued behind in-flight DSMEM stores.
    auto load_s = [&](int i, uint32_t (&sr)[32], uint32_t& vmask) -> bool {
      const int idx = idx_next;
      idx_next = load_idx(i + 1);
      vmask = __ballot_sync(0xffffffffu, idx >= 0 && idx < p.n_kv);
      if (!mbar_wait(s_full, i & 1)) return false;
      tc_fence_after();
      tmem_ld32(tmem_base + lane_addr + T::COL_S + half * 32, sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      return true;
    };
    auto send_s = [&](int i, const uint32_t (&sr)[32]) -> bool {
      const int xb = i & 1;
      if (expect_thread)
        mbar_arrive_expect_tx_u32(smem_u32(&x_full[xb]), static_cast<uint32_t>(T::X_BYTES));
      if (!mbar_wait(&x_free[xb], ((i >> 1) & 1) ^ 1)) return false;
      const uint32_t buf_off = static_cast<uint32_t>(xb * T::X_BYTES) + row_off;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int chunk = half * 8 + j;
        st_async_v4(x_peer + buf_off + ((chunk ^ (h & 7)) << 4), x_full_peer + xb * 8, sr[4 * j],
                    sr[4 * j + 1], sr[4 * j + 2], sr[4 * j + 3]);
      }
      return true;
    };
    auto block_max = [&](int i, const uint32_t (&sr)[32], uint32_t vmask, float (&z)[32],
                         float& bmax) -> bool {
      const int xb = i & 1;
      if (!mbar_wait(&x_full[xb], (i >> 1) & 1)) return false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int chunk = half * 8 + j;
        const float4 f = *reinterpret_cast<const float4*>(x_smem + xb * T::X_BYTES + row_off +
                                                          ((chunk ^ (h & 7)) << 4));
        z[4 * j] = f.x; z[4 * j + 1] = f.y; z[4 * j + 2] = f.z; z[4 * j + 3] = f.w;
      }
      float hmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        // S = S_0 + S_1 in the same order on both CTAs: identical logits.
        const float mine = __uint_as_float(sr[j]);
        const float s = rank == 0 ? mine + z[j] : z[j] + mine;
        z[j] = ((vmask >> j) & 1u) ? s * p.scale_log2 : -INFINITY;
        hmax = fmaxf(hmax, z[j]);
      }
      // The peer's values are consumed (z depends on them): its x buffer
      // slot may be reused.
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(x_free_peer + xb * 8);
      // row max over both halves of the block
      float* red_i = red + (i & 1) * (2 * T::M);
      red_i[half * T::M + h] = hmax;
      __syncwarp();
      uint64_t* rb = &red_bar[(i & 1) * 4 + quarter];
      if (lane == 0) mbar_arrive(rb);
      if (!mbar_wait(rb, (i >> 1) & 1)) return false;
      bmax = fmaxf(hmax, red_i[(half ^ 1) * T::M + h]);
      return true;
    };
    auto softmax_p = [&](int i, const float (&z)[32], float bmax) -> bool {
      const bool grow = bmax > m_used + 8.0f;
      const float m_new = grow ? bmax : m_used;
      // The P tile and O are free once PV(i-1) finished.
      if (i > 0) {
        if (!mbar_wait(pv_done, (i - 1) & 1)) return false;
        tc_fence_after();
      }
      if (i > 0 && __any_sync(0xffffffffu, grow)) {
        const float alpha = grow ? exp2f(m_used - m_new) : 1.0f;
#pragma unroll 1
        for (int c = half * (T::VH / 2); c < (half + 1) * (T::VH / 2); c += 16) {
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
      tmem_st16(tmem_base + lane_addr + T::COL_P + half * 16, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      return true;
    };

    uint32_t sr_a[32], sr_b[32];
    uint32_t vm_a = 0, vm_b = 0;
    float z[32];
    float bmax = -INFINITY;
    if (n_blocks > 0) ok = load_s(0, sr_a, vm_a) && send_s(0, sr_a);
    for (int i = 0; i < n_blocks && ok; i += 2) {
      if (i + 1 < n_blocks) ok = load_s(i + 1, sr_b, vm_b);
      ok = ok && block_max(i, sr_a, vm_a, z, bmax);
      ok = ok && softmax_p(i, z, bmax);
      if (ok && i + 1 < n_blocks) ok = send_s(i + 1, sr_b);
      if (!ok || i + 1 >= n_blocks) break;
      if (i + 2 < n_blocks) ok = load_s(i + 2, sr_a, vm_a);
      ok = ok && block_max(i + 1, sr_b, vm_b, z, bmax);
      ok = ok && softmax_p(i + 1, z, bmax);
      if (ok && i + 2 < n_blocks) ok = send_s(i + 2, sr_a);
    }
    if (ok && n_blocks > 0) {
      ok = mbar_wait(pv_done, (n_blocks - 1) & 1);
      tc_fence_after();
    }
    // Both warps of a quarter add their halves of l and l_mma.
    float* red_l = reinterpret_cast<float*>(smem + T::OFF_END);   // [half][2][128]
    red_l[(half * 2) * T::M + h] = l;
    red_l[(half * 2 + 1) * T::M + h] = l_mma;
    __syncwarp();
    if (lane == 0) mbar_arrive(&end_bar[quarter]);
    ok = mbar_wait(&end_bar[quarter], 0) && ok;
    const float l_o = red_l[((half ^ 1) * 2) * T::M + h];
    const float lm_o = red_l[((half ^ 1) * 2 + 1) * T::M + h];
    const float l_all = half == 0 ? l + l_o : l_o + l;
    const float lm_all = half == 0 ? l_mma + lm_o : lm_o + l_mma;
    // O / sum(rounded p) is an exact convex combination of the V rows with
    // weights perturbed by the bf16 rounding of p (a component shared by the
    // rows cancels); the LSE keeps the unrounded sum.
    const bool has = ok && l_all > 0.f && lm_all > 0.f;
    const float inv_l = has ? 1.0f / lm_all : 0.f;
    const uint32_t keep = has ? 0xffffffffu : 0u;   // masks undefined TMEM when empty
    const float lse_v = has ? (m_used + log2f(l_all)) * 0.69314718055994531f : -INFINITY;
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
    for (int c = half * (T::VH / 2); c < (half + 1) * (T::VH / 2); c += 16) {
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
    if (rank == 0 && half == 0 && h < p.H) {
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

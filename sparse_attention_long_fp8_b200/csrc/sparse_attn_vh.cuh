// Sparse MQA attention over the selected 576-d latent rows (page "DeepseekV3.2
// 拆解", section "核心组件 / 细粒度 Token 选择机制", eq. u_t; latent = 512 value
// dims + 64 RoPE dims, page "DeepSeek architecture", section 1.1).
//
// Two independent CTAs per query row, one per half of the 512 value dims
// ("V-half" v = 0, 1). Each CTA
//   * gathers the full 1152-byte latent rows of the selected keys into a
//     2-stage ring of 64-key blocks (cp.async, completion on mbarriers);
//   * computes the complete logits S = Q C^T (128 heads x 64 keys per block):
//     Q's five 64-dim blocks that only the logits use live in TMEM (A operand
//     read from TMEM), its four V-half blocks in shared memory;
//   * runs the online softmax and accumulates O for its 256 value dims.
// The logits are computed twice per row (once per CTA) and the rows gathered
// twice (L2 serves the second read); in exchange no partial result crosses
// between SMs: on this part DSMEM stores move ~11 bytes per cycle per SM,
// which made a per-block exchange of fp32 partial logits the bound.
//
// A stage is released in two parts: its five logit-only dim blocks as soon as
// S of the block completes, its four V-half blocks when PV completes. The
// logit MMAs of a block run over the logit-only part first, so the gather of
// block i + 2 overlaps S(i + 1) and PV(i).
//
// S is double-buffered in TMEM, and P(i) (bf16, 32 columns) is written over
// the first half of S(i)'s own buffer once both softmax warps of a lane
// quarter have read it. S(i + 1) is issued as soon as PV(i - 1) has released
// its buffer, so the tensor pipe does not wait for the softmax to read S(i).
//
// TMEM per CTA: O 256 columns, S 2 x 64, Q 128 (four logit-only dim blocks)
// = 512. Q's other five dim blocks (the V half and the RoPE block) are in
// shared memory.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "ptx.cuh"
#include "sparse_attn.cuh"

namespace dsa {

struct VhTile {
  static constexpr int NK = 64;                 // latent rows per block
  static constexpr int M = 128;                 // head rows
  static constexpr int DQK = 576, DV = 512, VH = 256;
  static constexpr int NDB = DQK / 64;          // 9 dim blocks per latent row
  static constexpr int VDB = VH / 64;           // 4 of them hold this CTA's value half
  static constexpr int XDB = NDB - VDB;         // 5 only the logits read
  static constexpr int DB_BYTES = NK * 128;     // one 64-dim block of a stage
  static constexpr int STAGE_BYTES = NDB * DB_BYTES;
  static constexpr int STAGES = 2;
  static constexpr int XT = 4;                  // logit-only Q blocks held in TMEM
  static constexpr int QSB = VDB + 1;           // Q blocks in shared memory: V half + RoPE
  static constexpr int QS_BYTES = QSB * M * 128;
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 448;           // gather 0-3, S MMA 4, softmax 5-12, PV MMA 13
  static constexpr int SOFTMAX_WARPS = 8;       // two per TMEM lane quarter, 32 keys each
  static constexpr int COL_O = 0, COL_S = 256, COL_Q = 384;   // S buffer b at COL_S + 64 b
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int OFF_C = 0;
  static constexpr int OFF_QS = STAGES * STAGE_BYTES;
  static constexpr int OFF_RED = OFF_QS + QS_BYTES;          // [2 parity][2 halves][128] fp32
  static constexpr int OFF_END = OFF_C;      // [half][l, l_mma][128] fp32, after the last PV
  static constexpr int OFF_BAR = OFF_RED + 2 * 2 * M * 4;
  static constexpr int NUM_BARS = 4 * STAGES + 6 + 8 + 4;    // stages, singles, red[8], end[4]
  // No alignment slack: the dynamic shared memory of this kernel starts on a
  // 1024-byte boundary (checked at run time; a misaligned base is reported).
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_QS % 1024 == 0, "1024-byte aligned operands");
  static_assert(COL_Q + XT * 32 == 512, "TMEM columns");
};

// Latent dim block of the t-th Q block held in TMEM (t = 0..3): the other
// half's four value blocks. The u-th Q block in shared memory (u = 0..4) is
// block 4v + u of this CTA's value half, then the RoPE block 8.
__device__ __forceinline__ int vh_tblock(int t, int v) { return t + 4 * (1 - v); }
__device__ __forceinline__ int vh_sblock(int u, int v) { return u == 4 ? 8 : 4 * v + u; }

// Warp roles: 0-3 gather (cp.async, 16 bytes per copy); 4 issues
// the logit MMAs and owns TMEM; 5-12 run the softmax (two warps per TMEM lane
// quarter: a thread owns one head row and 32 of a block's 64 keys); 13 issues
// the PV MMAs.
__global__ void __launch_bounds__(448, 1) sparse_attn_vh_kernel(AttnParams p) {
  using T = VhTile;
  constexpr int NK = T::NK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* c_smem = smem + T::OFF_C;
  uint8_t* qs_smem = smem + T::OFF_QS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::OFF_BAR);
  uint64_t* cx_full = bars;                      // [2] logit-only blocks of the stage landed
  uint64_t* cv_full = bars + T::STAGES;          // [2] V-half blocks landed
  uint64_t* cx_empty = bars + 2 * T::STAGES;     // [2] S of the stage's block finished
  uint64_t* cv_empty = bars + 3 * T::STAGES;     // [2] PV of the stage's block finished
  uint64_t* s_full = bars + 4 * T::STAGES;       // [2] S tile of buffer b written
  uint64_t* pv_done = s_full + 2;                // [2] PV of buffer b finished (buffer free, O updated)
  uint64_t* p_full = s_full + 4;                 // P tile written
  uint64_t* q_ready = s_full + 5;                // Q in TMEM and shared memory
  uint64_t* red_bar = s_full + 6;                // [parity][quarter]: both half maxima written
  uint64_t* end_bar = s_full + 14;               // [quarter]: both halves of l, l_mma written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  if ((smem_u32(smem_raw) & 1023u) != 0) {      // see SMEM_BYTES: no slack to realign
    if (threadIdx.x == 0) raise_error(kErrInternal);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int vh = blockIdx.x & 1;                 // value half of this CTA
  const int unit = blockIdx.x >> 1;
  const int row = unit / p.splits;               // b * n_q + t
  const int split = unit % p.splits;
  const int b = row / p.n_q;
  const int slot_begin = split * p.slots_per_split;
  const int slot_end = min(p.topk, slot_begin + p.slots_per_split);
  const int n_blocks = max(0, (slot_end - slot_begin + NK - 1) / NK);
  const int32_t* row_idx = p.indices + static_cast<size_t>(row) * p.topk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&cx_full[s], T::PRODUCERS);
      mbar_init(&cv_full[s], T::PRODUCERS);
      mbar_init(&cx_empty[s], 1);
      mbar_init(&cv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(p_full, T::SOFTMAX_WARPS);
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
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ gather
    // Thread (kq = tid / 8, ch = tid % 8) copies 16-byte chunk ch of every
    // 64-dim block of keys kq, kq + 16, kq + 32 and kq + 48 of a block. Under
    // the 128-byte swizzle chunk ch of row j sits at ((ch ^ (j & 7)) << 4),
    // and j & 7 = kq & 7 for all four keys: the shared-memory destination is
    // a per-thread constant plus an immediate and the source a row pointer
    // plus an immediate, so a copy costs about one issued instruction. A warp
    // instruction moves four whole 128-byte lines.
    const int kq = threadIdx.x >> 3, ch = threadIdx.x & 7;
    const uint32_t dst0 = smem_u32(c_smem) + kq * 128 + ((ch ^ (kq & 7)) << 4);
    auto load_keys = [&](int blk, int64_t (&k)[4]) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int slot = slot_begin + blk * NK + kq + 16 * r;
        const int idx = (blk < n_blocks && slot < slot_end) ? row_idx[slot] : -1;
        k[r] = (idx >= 0 && idx < p.n_kv) ? p.km.row(b, idx, p.n_kv) : -1;   // pool row
      }
    };
    auto copy_part = [&](auto vh_c, auto vpart_c, uint32_t dst, const __nv_bfloat16* const (&src)[4],
                         const uint32_t (&bytes)[4]) {
      constexpr int V = decltype(vh_c)::value;
      constexpr bool VP = decltype(vpart_c)::value;
#pragma unroll
      for (int t = 0; t < (VP ? T::VDB : T::XDB); ++t) {
        const int db = VP ? 4 * V + t : (t == 4 ? 8 : t + 4 * (1 - V));
#pragma unroll
        for (int r = 0; r < 4; ++r)
          cp_async_16(dst + db * T::DB_BYTES + r * 16 * 128, src[r] + db * 64, bytes[r]);
      }
    };
    using I0 = std::integral_constant<int, 0>;
    using I1 = std::integral_constant<int, 1>;
    using BX = std::integral_constant<bool, false>;
    using BV = std::integral_constant<bool, true>;
    int64_t keys[4];
    load_keys(0, keys);
    bool ok = true;
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int st = i % T::STAGES;
      const uint32_t ph = ((i / T::STAGES) & 1) ^ 1;
      const __nv_bfloat16* src[4];
      uint32_t bytes[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        src[r] = p.kv + (keys[r] >= 0 ? keys[r] : 0) * T::DQK + ch * 8;
        bytes[r] = keys[r] >= 0 ? 16u : 0u;
      }
      load_keys(i + 1, keys);   // one block ahead
      const uint32_t dst = dst0 + st * T::STAGE_BYTES;
      ok = mbar_wait(&cx_empty[st], ph);
      if (!ok) break;
      if (vh == 0) copy_part(I0{}, BX{}, dst, src, bytes);
      else copy_part(I1{}, BX{}, dst, src, bytes);
      cp_async_arrive_noinc(&cx_full[st]);
      ok = mbar_wait(&cv_empty[st], ph);
      if (!ok) break;
      if (vh == 0) copy_part(I0{}, BV{}, dst, src, bytes);
      else copy_part(I1{}, BV{}, dst, src, bytes);
      cp_async_arrive_noinc(&cv_full[st]);
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ S = Q C^T issuer
    // The whole warp runs the loop; one elected lane issues. Descriptors are
    // formed once: adding (byte offset >> 4) to a descriptor moves its start
    // address (every shared address here is below 256 KB, so the 14-bit
    // field cannot carry).
    constexpr uint32_t idesc_s = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
    const uint64_t c_desc0 = umma_desc(smem_u32(c_smem), 16, 1024, 2);
    const uint64_t q_desc0 = umma_desc(smem_u32(qs_smem), 16, 1024, 2);
    const uint32_t x_shift = static_cast<uint32_t>(4 * (1 - vh) * T::DB_BYTES) >> 4;
    const uint32_t v_shift = static_cast<uint32_t>(4 * vh * T::DB_BYTES) >> 4;
    bool ok = mbar_wait(q_ready, 0);
    tc_fence_after();
    for (int i = 0; i < n_blocks && ok; ++i) {
      const int st = i % T::STAGES;
      const uint32_t ph = (i / T::STAGES) & 1;
      const int sb = i & 1;                            // S buffer of block i
      // buffer sb is free once PV(i - 2) has read the P it held
      ok = mbar_wait(&pv_done[sb], ((i >> 1) & 1) ^ 1) && mbar_wait(&cx_full[st], ph);
      if (!ok) break;
      fence_proxy_async_smem();
      tc_fence_after();
      const uint32_t d_s = tmem_base + T::COL_S + sb * T::NK;
      const uint64_t cd = c_desc0 + static_cast<uint32_t>(st * (T::STAGE_BYTES >> 4));
      // logit-only part of the stage: the other half's value blocks with Q
      // from TMEM, then the RoPE block with Q from shared memory
#pragma unroll
      for (int t = 0; t < T::XT; ++t)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = cd + x_shift + ((t * T::DB_BYTES + kk * 32) >> 4);
          if (elect_one())
            umma_bf16_ts(d_s, tmem_base + T::COL_Q + t * 32 + kk * 8, bd, idesc_s,
                         (t | kk) ? 1u : 0u);
        }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = q_desc0 + ((4 * T::M * 128 + kk * 32) >> 4);
        const uint64_t bd = cd + ((8 * T::DB_BYTES + kk * 32) >> 4);
        if (elect_one()) umma_bf16_ss(d_s, ad, bd, idesc_s, 1u);
      }
      if (elect_one()) umma_commit(&cx_empty[st]);
      ok = mbar_wait(&cv_full[st], ph);
      if (!ok) break;
      fence_proxy_async_smem();
      tc_fence_after();
      // V-half blocks, Q from shared memory
#pragma unroll
      for (int u = 0; u < T::VDB; ++u)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = q_desc0 + ((u * T::M * 128 + kk * 32) >> 4);
          const uint64_t bd = cd + v_shift + ((u * T::DB_BYTES + kk * 32) >> 4);
          if (elect_one()) umma_bf16_ss(d_s, ad, bd, idesc_s, 1u);
        }
      if (elect_one()) umma_commit(&s_full[sb]);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ O += P V issuer
    constexpr uint32_t idesc_pv = umma_idesc(128, T::VH, 1u, 1u, 0u, 1u);
    const uint64_t v_desc0 =
        umma_desc(smem_u32(c_smem) + 4 * vh * T::DB_BYTES, T::DB_BYTES, 1024, 2);
    for (int j = 0; j < n_blocks; ++j) {
      const int st = j % T::STAGES;
      if (!mbar_wait(p_full, j & 1)) break;
      tc_fence_after();
      // P(j) exists only after S(j) was read, so S(j) has completed: when
      // PV(j) completes, both readers of the V-half blocks are done, and the
      // S / P buffer of block j is free.
      const uint64_t vd = v_desc0 + static_cast<uint32_t>(st * (T::STAGE_BYTES >> 4));
      const uint32_t a_p = tmem_base + T::COL_S + (j & 1) * T::NK;   // P over S's first half
#pragma unroll
      for (int kk = 0; kk < NK / 16; ++kk)
        if (elect_one())
          umma_bf16_ts(tmem_base + T::COL_O, a_p + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
      if (elect_one()) {
        umma_commit(&cv_empty[st]);
        umma_commit(&pv_done[j & 1]);
      }
    }
    __syncwarp();
  } else if (warp >= 5 && warp <= 12) {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int half = (warp - 5) >> 2;                        // which 32 keys of a block
    const int h = quarter * 32 + lane;                       // head row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + T::OFF_RED);   // [parity][half][128]

    // Q into TMEM (four logit-only blocks; the two warps of a quarter take
    // alternate 16-column chunks) and shared memory (V-half blocks and the
    // RoPE block, K-major 128-byte swizzle; the two warps alternate blocks).
    {
      const __nv_bfloat16* qh = p.q + (static_cast<size_t>(row) * p.H + min(h, p.H - 1)) * T::DQK;
      const bool live = h < p.H;
      for (int c = half; c < T::XT * 2; c += 2) {
        uint32_t v[16];
        const uint4* src = reinterpret_cast<const uint4*>(qh + vh_tblock(c >> 1, vh) * 64 + (c & 1) * 32);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 u = live ? src[k] : make_uint4(0u, 0u, 0u, 0u);
          v[4 * k] = u.x; v[4 * k + 1] = u.y; v[4 * k + 2] = u.z; v[4 * k + 3] = u.w;
        }
        tmem_st16(tmem_base + lane_addr + T::COL_Q + c * 16, v);
      }
      for (int u = half; u < T::QSB; u += 2) {
        const uint4* src = reinterpret_cast<const uint4*>(qh + vh_sblock(u, vh) * 64);
        uint8_t* dst = qs_smem + u * (T::M * 128) + (h >> 3) * 1024 + (h & 7) * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(dst + ((ch ^ (h & 7)) << 4)) =
              live ? src[ch] : make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }

    float m_used = -INFINITY;   // running max (log2 domain) the P values are relative to
    float l = 0.f;              // this warp's share of the sum of the fp32 p (LSE)
    float l_mma = 0.f;          // ... of the bf16-rounded p the PV MMA used (normalises O)
    bool ok = true;
    auto load_idx = [&](int blk) -> int {
      const int slot = slot_begin + blk * NK + half * 32 + lane;
      return (blk < n_blocks && slot < slot_end) ? row_idx[slot] : -1;
    };
    int idx_next = load_idx(0);
    uint32_t sr[32];
    float z[32];
    for (int i = 0; i < n_blocks && ok; ++i) {
      // ---- logits of this warp's 32 keys from S buffer i & 1
      const int idx = idx_next;
      idx_next = load_idx(i + 1);
      const uint32_t vmask = __ballot_sync(0xffffffffu, idx >= 0 && idx < p.n_kv);
      const uint32_t col_s = T::COL_S + (i & 1) * T::NK;
      if (!(ok = mbar_wait(&s_full[i & 1], (i >> 1) & 1))) break;
      tc_fence_after();
      tmem_ld32(tmem_base + lane_addr + col_s + half * 32, sr);
      tmem_wait_ld();
      // ---- block max over the 64 keys, shared with the partner warp
      float hmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        z[j] = ((vmask >> j) & 1u) ? __uint_as_float(sr[j]) * p.scale_log2 : -INFINITY;
        hmax = fmaxf(hmax, z[j]);
      }
      float* red_i = red + (i & 1) * (2 * T::M);
      red_i[half * T::M + h] = hmax;
      // After this exchange both warps of the quarter have read their S
      // columns, so P may overwrite the buffer's first 32 columns.
      tc_fence_before();
      __syncwarp();
      uint64_t* rb = &red_bar[(i & 1) * 4 + quarter];
      if (lane == 0) mbar_arrive(rb);
      if (!(ok = mbar_wait(rb, (i >> 1) & 1))) break;
      tc_fence_after();
      const float bmax = fmaxf(hmax, red_i[(half ^ 1) * T::M + h]);
      // ---- online softmax; P(i) into TMEM once PV(i - 1) has finished
      const bool grow = bmax > m_used + 8.0f;
      const float m_new = grow ? bmax : m_used;
      if (i > 0) {
        if (!(ok = mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1))) break;
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
      tmem_st16(tmem_base + lane_addr + col_s + half * 16, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && n_blocks > 0) {
      ok = mbar_wait(&pv_done[(n_blocks - 1) & 1], ((n_blocks - 1) >> 1) & 1);
      tc_fence_after();
    }
    // Both warps of a quarter add their halves of l and l_mma (through the
    // stage area: every gather and MMA has finished by now).
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
      const size_t o_off = (static_cast<size_t>(row) * p.H + h) * T::DV + vh * T::VH;
      if (p.out_bf16) dst_bf16 = static_cast<__nv_bfloat16*>(p.out) + o_off;
      else dst_f32 = static_cast<float*>(p.out) + o_off;
    } else {
      const size_t part = static_cast<size_t>(row) * p.splits + split;
      dst_f32 = p.part_o + (part * p.H + h) * T::DV + vh * T::VH;
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
    if (vh == 0 && half == 0 && h < p.H) {
      if (direct) {
        if (p.lse) p.lse[static_cast<size_t>(row) * p.H + h] = lse_v;
      } else {
        p.part_lse[(static_cast<size_t>(row) * p.splits + split) * p.H + h] = lse_v;
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

}  // namespace dsa

// Sparse MQA attention over the selected 576-d latent rows (page "DeepseekV3.2
// 拆解", section "核心组件 / 细粒度 Token 选择机制", eq. u_t; latent = 512 value
// dims + 64 RoPE dims, page "DeepSeek architecture", section 1.1).
//
// Two independent CTAs per query row, one per half of the 512 value dims
// ("V-half" v = 0, 1). Each CTA
//   * gathers the full 1152-byte latent rows of the selected keys into a
//     2-stage ring of 64-key blocks (cp.async, completion on mbarriers);
//   * computes the complete logits S = Q C^T (128 heads x 64 keys per block):
//     six of Q's nine 64-dim blocks live in TMEM (A operand read from TMEM),
//     three in shared memory;
//   * runs the online softmax and accumulates O for its 256 value dims. The
//     two softmax warps of a TMEM lane quarter share each block's row maxima
//     through shared memory and a named barrier.
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
// S has one TMEM buffer, released as soon as the eight softmax warps have
// loaded it into registers; P(i) (bf16) goes to one of two shared-memory
// buffers and the PV MMA reads it from there. So S(i + 1) waits only for the
// load of S(i), not for the softmax or PV(i), and the tensor pipe runs PV(i)
// in the gap between S(i + 1) and S(i + 2).
//
// TMEM per CTA: O 256 columns, S 64, Q 192 (six 64-dim blocks: the five that
// only the logits read and the first of the V half) = 512. Q's other three
// V-half blocks are in shared memory.
//
// The CTAs are persistent: CTA c takes units c, c + grid, ... (a unit is one
// (query row, split, value half)), and every barrier phase runs on across
// units. At the end of a unit the softmax warps load the next unit's Q (its
// S MMAs can then start) before they write this unit's O.
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
  static constexpr int XT = 6;                  // Q blocks held in TMEM
  static constexpr int QSB = NDB - XT;          // Q blocks in shared memory (V half 1..3)
  static constexpr int QS_BYTES = QSB * M * 128;
  static constexpr int P_BYTES = M * NK * 2;    // one bf16 P tile, K-major 128-byte swizzle
  static constexpr int PRODUCERS = 128;
  static constexpr int THREADS = 448;           // gather 0-3, S MMA 4, softmax 5-12, PV MMA 13
  static constexpr int SOFTMAX_WARPS = 8;       // two per TMEM lane quarter, 32 keys each
  static constexpr int COL_O = 0, COL_S = 256, COL_Q = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int OFF_C = 0;
  static constexpr int OFF_QS = STAGES * STAGE_BYTES;
  static constexpr int OFF_P = OFF_QS + QS_BYTES;            // [2] P tiles
  static constexpr int OFF_RED = OFF_P + 2 * P_BYTES;        // [2 parity][2 halves][128] fp32
  static constexpr int OFF_BAR = OFF_RED + 2 * 2 * M * 4;
  static constexpr int NUM_BARS = 4 * STAGES + 7;            // stages, then the singles
  // No alignment slack: the dynamic shared memory of this kernel starts on a
  // 1024-byte boundary (checked at run time; a misaligned base is reported).
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(STAGE_BYTES % 1024 == 0 && OFF_QS % 1024 == 0 && OFF_P % 1024 == 0,
                "1024-byte aligned operands");
  static_assert(COL_S + NK == COL_Q && COL_Q + XT * 32 == 512, "TMEM columns");
};

// Latent dim block of the t-th Q block held in TMEM (t = 0..5): the other
// half's four value blocks, the RoPE block 8, then block 4v (the first of this
// CTA's value half). The u-th Q block in shared memory (u = 0..2) is block
// 4v + 1 + u.
__device__ __forceinline__ int vh_tblock(int t, int v) {
  return t < 4 ? t + 4 * (1 - v) : (t == 4 ? 8 : 4 * v);
}
__device__ __forceinline__ int vh_sblock(int u, int v) { return 4 * v + 1 + u; }

// Unit u of 2 * rows * splits: value half u & 1 of (row, split) = u >> 1.
struct VhUnit {
  int vh, row, split, b, slot_begin, slot_end, n_blocks;
  const int32_t* row_idx;
};
__device__ __forceinline__ VhUnit vh_unit(const AttnParams& p, int64_t u) {
  VhUnit w;
  w.vh = static_cast<int>(u & 1);
  const int64_t pair = u >> 1;
  w.row = static_cast<int>(pair / p.splits);
  w.split = static_cast<int>(pair % p.splits);
  w.b = w.row / p.n_q;
  w.slot_begin = w.split * p.slots_per_split;
  w.slot_end = min(p.topk, w.slot_begin + p.slots_per_split);
  w.n_blocks = max(0, (w.slot_end - w.slot_begin + VhTile::NK - 1) / VhTile::NK);
  w.row_idx = p.indices + static_cast<size_t>(w.row) * p.topk;
  return w;
}

// Warp roles: 0-3 gather (cp.async, 16 bytes per copy); 4 issues
// the logit MMAs and owns TMEM; 5-12 run the softmax (two warps per TMEM lane
// quarter: a thread owns one head row and 32 of a block's 64 keys); 13 issues
// the PV MMAs.
// tmap_o: the output (p.out, or p.part_o in split mode) as a byte tensor of
// rows of DV elements, one row per (row, head) (or (row, split, head)), box
// 128 bytes x H rows with the 128-byte swizzle.
__global__ void __launch_bounds__(448, 1)
    sparse_attn_vh_kernel(const __grid_constant__ CUtensorMap tmap_o, AttnParams p, int64_t n_units) {
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
  uint64_t* s_full = bars + 4 * T::STAGES;       // S tile written
  uint64_t* s_free = s_full + 1;                 // S tile loaded by all softmax warps
  uint64_t* p_full = s_full + 2;                 // [2] P tile of buffer b written
  uint64_t* pv_done = s_full + 4;                // [2] PV of buffer b finished (buffer free, O updated)
  uint64_t* q_ready = s_full + 6;                // Q of a unit in TMEM and shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + T::NUM_BARS);

  if ((smem_u32(smem_raw) & 1023u) != 0) {      // see SMEM_BYTES: no slack to realign
    if (threadIdx.x == 0) raise_error(kErrInternal);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t u0 = blockIdx.x, du = gridDim.x;   // this CTA's units: u0, u0 + du, ...

  if (threadIdx.x == 0) {
    for (int s = 0; s < T::STAGES; ++s) {
      mbar_init(&cx_full[s], T::PRODUCERS);
      mbar_init(&cv_full[s], T::PRODUCERS);
      mbar_init(&cx_empty[s], 1);
      mbar_init(&cv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, T::SOFTMAX_WARPS);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&p_full[s], T::SOFTMAX_WARPS);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(q_ready, T::SOFTMAX_WARPS);
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

  // Every role walks the same units and counts their blocks alike: g is the
  // CTA's running block number, which picks the stage, the P buffer and the
  // barrier phases. Units with no blocks (a split past the top-k slots) only
  // get their empty output.
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
    uint32_t g = 0;
    bool ok = true;
    griddep_wait();               // the indices may come from the previous kernel
    for (int64_t u = u0; u < n_units && ok; u += du) {
      const VhUnit w = vh_unit(p, u);
      auto load_keys = [&](int blk, int64_t (&k)[4]) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int slot = w.slot_begin + blk * NK + kq + 16 * r;
          const int idx = (blk < w.n_blocks && slot < w.slot_end) ? w.row_idx[slot] : -1;
          k[r] = (idx >= 0 && idx < p.n_kv) ? p.km.row(w.b, idx, p.n_kv) : -1;   // pool row
        }
      };
      int64_t keys[4];
      load_keys(0, keys);
      for (int i = 0; i < w.n_blocks && ok; ++i, ++g) {
        const int st = g % T::STAGES;
        const uint32_t ph = ((g / T::STAGES) & 1) ^ 1;
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
        if (w.vh == 0) copy_part(I0{}, BX{}, dst, src, bytes);
        else copy_part(I1{}, BX{}, dst, src, bytes);
        cp_async_arrive_noinc(&cx_full[st]);
        ok = mbar_wait(&cv_empty[st], ph);
        if (!ok) break;
        if (w.vh == 0) copy_part(I0{}, BV{}, dst, src, bytes);
        else copy_part(I1{}, BV{}, dst, src, bytes);
        cp_async_arrive_noinc(&cv_full[st]);
      }
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ S = Q C^T issuer
    // One elected lane runs the whole loop: an elect per instruction costs
    // more issue time than an N = 64 MMA takes to execute (measured: 64
    // against 32 cycles per MMA with A in TMEM). Descriptors are formed once:
    // adding (byte offset >> 4) to a descriptor moves its start address
    // (every shared address here is below 256 KB, so the 14-bit field cannot
    // carry).
    if (elect_one()) {
      constexpr uint32_t idesc_s = umma_idesc(128, NK, 1u, 1u, 0u, 0u);
      const uint64_t c_desc0 = umma_desc(smem_u32(c_smem), 16, 1024, 2);
      const uint64_t q_desc0 = umma_desc(smem_u32(qs_smem), 16, 1024, 2);
      const uint32_t d_s = tmem_base + T::COL_S;
      uint32_t g = 0, k = 0;
      bool ok = true;
      for (int64_t u = u0; u < n_units && ok; u += du) {
        const VhUnit w = vh_unit(p, u);
        if (w.n_blocks == 0) continue;
        const uint32_t x_shift = static_cast<uint32_t>(4 * (1 - w.vh) * T::DB_BYTES) >> 4;
        const uint32_t v_shift = static_cast<uint32_t>(4 * w.vh * T::DB_BYTES) >> 4;
        ok = mbar_wait(q_ready, k & 1);
        ++k;
        tc_fence_after();
        for (int i = 0; i < w.n_blocks && ok; ++i, ++g) {
          const int st = g % T::STAGES;
          const uint32_t ph = (g / T::STAGES) & 1;
          // the S buffer is free once every softmax warp has loaded S(g - 1)
          ok = (g == 0 || mbar_wait(s_free, (g - 1) & 1)) && mbar_wait(&cx_full[st], ph);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t cd = c_desc0 + static_cast<uint32_t>(st * (T::STAGE_BYTES >> 4));
          // logit-only part of the stage (the other half's value blocks, then
          // the RoPE block), Q from TMEM
#pragma unroll
          for (int t = 0; t < T::XDB; ++t)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t off = (t < 4 ? t * T::DB_BYTES : 8 * T::DB_BYTES) + kk * 32;
              const uint64_t bd = cd + (t < 4 ? x_shift : 0u) + (off >> 4);
              umma_bf16_ts(d_s, tmem_base + T::COL_Q + t * 32 + kk * 8, bd, idesc_s,
                           (t | kk) ? 1u : 0u);
            }
          umma_commit(&cx_empty[st]);
          ok = mbar_wait(&cv_full[st], ph);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          // V-half blocks: the first with Q from TMEM, the other three from
          // shared memory
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = cd + v_shift + ((kk * 32) >> 4);
            umma_bf16_ts(d_s, tmem_base + T::COL_Q + T::XDB * 32 + kk * 8, bd, idesc_s, 1u);
          }
#pragma unroll
          for (int uq = 0; uq < T::QSB; ++uq)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = q_desc0 + ((uq * T::M * 128 + kk * 32) >> 4);
              const uint64_t bd = cd + v_shift + (((uq + 1) * T::DB_BYTES + kk * 32) >> 4);
              umma_bf16_ss(d_s, ad, bd, idesc_s, 1u);
            }
          umma_commit(s_full);
        }
      }
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ O += P V issuer
    // P(g) exists only after S(g) was read, so S(g) has completed: when PV(g)
    // completes, both readers of the V-half blocks are done, and P buffer
    // g & 1 is free. The first PV of a unit overwrites O: the softmax warps
    // write that unit's first P only after they have read out the previous
    // unit's O. One elected lane issues (as for S).
    if (elect_one()) {
      constexpr uint32_t idesc_pv = umma_idesc(128, T::VH, 1u, 1u, 0u, 1u);
      const uint64_t p_desc0 = umma_desc(smem_u32(smem + T::OFF_P), 16, 1024, 2);
      uint32_t g = 0;
      bool ok = true;
      for (int64_t u = u0; u < n_units && ok; u += du) {
        const VhUnit w = vh_unit(p, u);
        const uint64_t v_desc0 =
            umma_desc(smem_u32(c_smem) + 4 * w.vh * T::DB_BYTES, T::DB_BYTES, 1024, 2);
        for (int i = 0; i < w.n_blocks; ++i, ++g) {
          const int st = g % T::STAGES;
          if (!(ok = mbar_wait(&p_full[g & 1], (g >> 1) & 1))) break;
          tc_fence_after();
          const uint64_t vd = v_desc0 + static_cast<uint32_t>(st * (T::STAGE_BYTES >> 4));
          const uint64_t pd = p_desc0 + static_cast<uint32_t>((g & 1) * (T::P_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < NK / 16; ++kk)
            umma_bf16_ss(tmem_base + T::COL_O, pd + ((kk * 32) >> 4), vd + ((kk * 2048) >> 4),
                         idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&cv_empty[st]);
          umma_commit(&pv_done[g & 1]);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 5 && warp <= 12) {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;
    const int half = (warp - 5) >> 2;                        // which 32 keys of a block
    const int h = quarter * 32 + lane;                       // head row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 1u + static_cast<uint32_t>(quarter);   // the quarter's two warps
    float* red = reinterpret_cast<float*>(smem + T::OFF_RED);   // [parity][half][128]

    const int stid = threadIdx.x - 5 * 32;                   // 0..255 over the softmax warps
    constexpr uint32_t kAllBar = 5u;                         // named barrier of the 8 warps
    constexpr uint32_t kAllThreads = 32u * T::SOFTMAX_WARPS;
    // Q of a unit: rows of 1152 bytes, one per head. The 256 softmax threads
    // copy three 64-dim blocks at a time into the Q area of shared memory
    // (cp.async, 4 whole 128-byte lines per warp instruction, the K-major
    // 128-byte-swizzled layout of the MMA operand): twice as staging for the
    // six TMEM blocks, which every thread then moves from its own head row
    // into its TMEM lane, and once more for the three blocks that stay there.
    auto copy_q3 = [&](const VhUnit& w, int first, bool tmem_part) {
      const __nv_bfloat16* qrow = p.q + static_cast<size_t>(w.row) * p.H * T::DQK;
      const int r4 = stid >> 3, ch = stid & 7;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int db = tmem_part ? vh_tblock(first + j, w.vh) : vh_sblock(first + j, w.vh);
#pragma unroll
        for (int it = 0; it < T::M / 32; ++it) {
          const int r = it * 32 + r4;
          const __nv_bfloat16* src = qrow + static_cast<size_t>(min(r, p.H - 1)) * T::DQK + db * 64 + ch * 8;
          const uint32_t dst = smem_u32(qs_smem) + j * (T::M * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                               ((ch ^ (r & 7)) << 4);
          cp_async_16(dst, src, r < p.H ? 16u : 0u);
        }
      }
      cp_async_wait_all();
    };
    auto load_q = [&](const VhUnit& w) {
#pragma unroll 1
      for (int round = 0; round < 2; ++round) {
        copy_q3(w, 3 * round, true);
        named_bar_sync(kAllBar, kAllThreads);
        // this warp's 16-column chunk (32 dims: 16-byte chunks 4 half .. +3)
        // of each staged block, from its lane's head row
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const uint32_t rowp = smem_u32(qs_smem) + j * (T::M * 128) + (h >> 3) * 1024 + (h & 7) * 128;
          uint32_t v[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 x = lds_v4(rowp + (((4 * half + c) ^ (h & 7)) << 4));
            v[4 * c] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
          }
          tmem_st16(tmem_base + lane_addr + T::COL_Q + (2 * (3 * round + j) + half) * 16, v);
        }
        named_bar_sync(kAllBar, kAllThreads);      // staging read before it is overwritten
      }
      copy_q3(w, 0, false);
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    };
    // A unit without blocks (a split past the top-k slots): O = 0, LSE = -inf.
    auto write_empty = [&](const VhUnit& w) {
      griddep_wait();
      if (h >= p.H) return;
      const bool direct = p.splits == 1;
      for (int c = half * (T::VH / 2); c < (half + 1) * (T::VH / 2); ++c) {
        if (direct) {
          const size_t o_off = (static_cast<size_t>(w.row) * p.H + h) * T::DV + w.vh * T::VH + c;
          if (p.out_bf16) static_cast<__nv_bfloat16*>(p.out)[o_off] = __float2bfloat16(0.f);
          else static_cast<float*>(p.out)[o_off] = 0.f;
        } else {
          const size_t part = static_cast<size_t>(w.row) * p.splits + w.split;
          p.part_o[(part * p.H + h) * T::DV + w.vh * T::VH + c] = 0.f;
        }
      }
      if (w.vh == 0 && half == 0) {
        if (direct) {
          if (p.lse) p.lse[static_cast<size_t>(w.row) * p.H + h] = -INFINITY;
        } else {
          p.part_lse[(static_cast<size_t>(w.row) * p.splits + w.split) * p.H + h] = -INFINITY;
        }
      }
    };

    uint32_t sr[32];
    float z[32];
    // this thread's row of a P tile: keys half * 32 .. + 31 are 16-byte chunks
    // 4 half .. 4 half + 3 of a 128-byte row, stored at chunk c ^ (h & 7)
    const uint32_t p_row = smem_u32(smem + T::OFF_P) + (h >> 3) * 1024 + (h & 7) * 128;
    uint32_t g = 0;
    bool ok = true;
    bool q_loaded = false;       // Q of the current unit is already in place
    for (int64_t u = u0; u < n_units && ok; u += du) {
      const VhUnit w = vh_unit(p, u);
      if (w.n_blocks == 0) {
        write_empty(w);
        continue;
      }
      if (!q_loaded) {
        load_q(w);
        griddep_wait();           // the indices may come from the previous kernel
      }
      q_loaded = false;
      float m_used = -INFINITY;   // running max (log2 domain) the P values are relative to
      float l = 0.f;              // this warp's share of the sum of the fp32 p (LSE)
      float l_mma = 0.f;          // ... of the bf16-rounded p the PV MMA used (normalises O)
      auto load_idx = [&](int blk) -> int {
        const int slot = w.slot_begin + blk * NK + half * 32 + lane;
        return (blk < w.n_blocks && slot < w.slot_end) ? w.row_idx[slot] : -1;
      };
      int idx_next = load_idx(0);
      for (int i = 0; i < w.n_blocks; ++i, ++g) {
        // ---- logits of this warp's 32 keys; the S buffer is released at
        // once. A failed wait does not leave the loop before the partner
        // exchange: the two warps of a quarter meet at a named barrier every
        // block and leave together when either has failed.
        const int idx = idx_next;
        idx_next = load_idx(i + 1);
        const uint32_t vmask = __ballot_sync(0xffffffffu, idx >= 0 && idx < p.n_kv);
        if (ok) ok = mbar_wait(s_full, g & 1);
        tc_fence_after();
        tmem_ld32(tmem_base + lane_addr + T::COL_S + half * 32, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // ---- block max over the 64 keys, shared with the partner warp. The
        // logits stay unscaled in z: the scale is positive, so the maximum
        // of the scaled logits is the scaled maximum (rounding is monotone),
        // and p = 2^(z * scale - m) is one fma. Keys outside the set (a warp-
        // uniform test, rare) are -inf.
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = __uint_as_float(sr[j]);
        if (vmask != 0xffffffffu) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (!((vmask >> j) & 1u)) z[j] = -INFINITY;
        }
        float mx[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
          mx[r] = fmaxf(fmaxf(fmaxf(z[r], z[r + 4]), fmaxf(z[r + 8], z[r + 12])),
                        fmaxf(fmaxf(z[r + 16], z[r + 20]), fmaxf(z[r + 24], z[r + 28])));
        const float hmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
        float* red_i = red + (g & 1) * (2 * T::M);
        red_i[half * T::M + h] = hmax;
        if (!named_bar_and(pair_bar, 64u, ok)) {
          ok = false;
          break;
        }
        const float bmax = fmaxf(hmax, red_i[(half ^ 1) * T::M + h]);
        // ---- online softmax. Rescaling O needs PV(g - 1) finished; writing
        // P buffer g & 1 needs PV(g - 2) finished (implied by PV(g - 1): the
        // PV MMAs complete in issue order).
        const bool grow = bmax > m_used + 8.0f;
        const float m_new = grow ? bmax : m_used;
        if (i > 0 && __any_sync(0xffffffffu, grow)) {
          if (ok) ok = mbar_wait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1);
          tc_fence_after();
          const float alpha = grow ? ex2_approx(m_used - m_new) : 1.0f;
#pragma unroll 1
          for (int c = half * (T::VH / 2); c < (half + 1) * (T::VH / 2) && ok; c += 16) {
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
        } else if (g > 1 && ok) {
          ok = mbar_wait(&pv_done[g & 1], ((g >> 1) & 1) ^ 1);
        }
        m_used = m_new;
        uint32_t pk[16];
        float ls[4] = {0.f, 0.f, 0.f, 0.f}, lm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = ex2_approx(fmaf(z[2 * j], p.scale_log2, -m_used));
          const float p1 = ex2_approx(fmaf(z[2 * j + 1], p.scale_log2, -m_used));
          const __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
          ls[j & 3] += p0 + p1;
          lm[j & 3] += __low2float(pb2) + __high2float(pb2);
          pk[j] = *reinterpret_cast<const uint32_t*>(&pb2);
        }
        float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
        float lsum_mma = (lm[0] + lm[1]) + (lm[2] + lm[3]);
        if (m_used == -INFINITY) {
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = 0u;
          lsum = 0.f;
          lsum_mma = 0.f;
        }
        l += lsum;
        l_mma += lsum_mma;
        const uint32_t pb = p_row + (g & 1) * T::P_BYTES;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          sts_v4(pb + (((4 * half + c) ^ (h & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                 pk[4 * c + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g & 1]);
      }
      // all softmax warps go on, or stop, together
      if (!named_bar_and(kAllBar, kAllThreads, ok)) {
        ok = false;
        break;
      }
      // ---- the next unit's Q: this unit's S MMAs have all completed (the
      // last S was loaded above), so its logits may start during this
      // epilogue
      for (int64_t un = u + du; un < n_units; un += du) {
        const VhUnit wn = vh_unit(p, un);
        if (wn.n_blocks == 0) continue;
        load_q(wn);
        q_loaded = true;
        break;
      }
      // ---- epilogue: O of this unit, once its last PV has finished
      ok = mbar_wait(&pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1);
      tc_fence_after();
      // The quarter's two warps add their halves of l and l_mma in the
      // exchange buffer (the barrier above ended both warps' reads of their
      // last block maxima; the one below precedes the next unit's first
      // write).
      red[half * T::M + h] = l;
      red[(2 + half) * T::M + h] = l_mma;
      named_bar_sync(pair_bar, 64u);
      const float l_o = red[(half ^ 1) * T::M + h];
      const float lm_o = red[(2 + (half ^ 1)) * T::M + h];
      const bool pv_ok = ok;
      named_bar_sync(pair_bar, 64u);
      const float l_all = half == 0 ? l + l_o : l_o + l;
      const float lm_all = half == 0 ? l_mma + lm_o : lm_o + l_mma;
      // O / sum(rounded p) is an exact convex combination of the V rows with
      // weights perturbed by the bf16 rounding of p (a component shared by
      // the rows cancels); the LSE keeps the unrounded sum.
      const bool has = pv_ok && l_all > 0.f && lm_all > 0.f;
      const float inv_l = has ? 1.0f / lm_all : 0.f;
      const uint32_t keep = has ? 0xffffffffu : 0u;   // masks undefined TMEM when empty
      const float lse_v = has ? (m_used + log2f(l_all)) * 0.69314718055994531f : -INFINITY;
      // O leaves by TMA stores of 128-byte-wide column slices (32 fp32 or 64
      // bf16 columns, 16 KB for 128 rows) staged in the swizzled layout the
      // store reads (16-byte chunk c of row h at h * 128 + ((c ^ (h & 7)) <<
      // 4)); each thread stages half of a slice's columns of its row. One
      // slice per round, alternating between the two P buffers (free: the
      // last PV has finished); after the CTA's last unit (nothing is
      // gathered any more) all slices at once through the stage area. The
      // stores run on while the warps go on; a buffer is written again only
      // after the store that read it has finished reading.
      const bool direct = p.splits == 1;
      const bool bf16_out = direct && p.out_bf16;
      const int esz = bf16_out ? 2 : 4;
      const int slice_cols = 128 / esz;
      const int n_slices = T::VH / slice_cols;
      const bool last = !q_loaded;
      const int per_round = last ? n_slices : 1;
      const int32_t y_row = static_cast<int32_t>(
          (direct ? static_cast<int64_t>(w.row) : static_cast<int64_t>(w.row) * p.splits + w.split) *
          p.H);
#pragma unroll 1
      for (int s0 = 0, rnd = 0; s0 < n_slices; s0 += per_round, ++rnd) {
        const uint32_t stage =
            last ? smem_u32(c_smem) : smem_u32(smem + T::OFF_P) + (rnd & 1) * T::P_BYTES;
        if (!last && stid == 0) bulk_wait_read<1>();     // the store of round rnd - 2 has read it
        named_bar_sync(kAllBar, kAllThreads);
        for (int sl = s0; sl < s0 + per_round; ++sl) {
          const uint32_t srow = stage + (sl - s0) * (T::M * 128) + h * 128;
#pragma unroll 1
          for (int c = half * (slice_cols / 2); c < (half + 1) * (slice_cols / 2); c += 16) {
            uint32_t o[16];
            tmem_ld16(tmem_base + lane_addr + T::COL_O + sl * slice_cols + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j] & keep) * inv_l);
            const int cc = c * esz / 16;                   // its first 16-byte chunk in the row
            if (bf16_out) {
              uint32_t pkd[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const __nv_bfloat162 v =
                    __floats2bfloat162_rn(__uint_as_float(o[2 * j]), __uint_as_float(o[2 * j + 1]));
                pkd[j] = *reinterpret_cast<const uint32_t*>(&v);
              }
#pragma unroll
              for (int q2 = 0; q2 < 2; ++q2)
                sts_v4(srow + (((cc + q2) ^ (h & 7)) << 4), pkd[4 * q2], pkd[4 * q2 + 1],
                       pkd[4 * q2 + 2], pkd[4 * q2 + 3]);
            } else {
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2)
                sts_v4(srow + (((cc + q2) ^ (h & 7)) << 4), o[4 * q2], o[4 * q2 + 1], o[4 * q2 + 2],
                       o[4 * q2 + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(kAllBar, kAllThreads);
        if (stid == 0) {
          for (int sl = s0; sl < s0 + per_round; ++sl)
            tma_store_2d(&tmap_o, stage + (sl - s0) * (T::M * 128),
                         (w.vh * T::VH + sl * slice_cols) * esz, y_row);
          bulk_commit();
        }
      }
      // every staged byte read before the next unit writes P (or gathers)
      if (stid == 0) bulk_wait_read<0>();
      named_bar_sync(kAllBar, kAllThreads);
      if (w.vh == 0 && half == 0 && h < p.H) {
        if (direct) {
          if (p.lse) p.lse[static_cast<size_t>(w.row) * p.H + h] = lse_v;
        } else {
          p.part_lse[(static_cast<size_t>(w.row) * p.splits + w.split) * p.H + h] = lse_v;
        }
      }
      // the TMEM loads of O are complete (wait::ld above) before this unit's
      // successor writes its first P, which is what lets PV overwrite O; the
      // eight warps agree on going on
      ok = named_bar_and(kAllBar, kAllThreads, ok);
    }
  }

  if (threadIdx.x == 5 * 32) bulk_wait<0>();   // the output stores have completed
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, T::TMEM_COLS);
  }
}

}  // namespace dsa

// Where a sequence's keys and query positions live.
//
// Keys (the FP8 indexer keys, their scales and the latent rows) are either
// contiguous per sequence (row b * n_kv + s) or paged: key s of sequence b is
// row block_table[b][s / page] * page + s % page of a shared pool, the
// PagedAttention layout (page "DeepSeek-V3 MoE blog", section 4.1). A page
// holds a power-of-two number of keys >= 128, so every 128-key indexer tile
// lies inside one page and is one TMA box.
//
// Query rows are either consecutive from q_pos0[b] (prefill from a position,
// decode) or carry an explicit absolute position each (row_pos[b][i]), which
// lets one prefill's query rows be split over several calls or GPUs in any
// grouping.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace dsa {

struct KeyMap {
  const int32_t* block_table;  // [B, max_pages] physical page per logical page, or null
  int32_t max_pages;           // row stride of block_table
  int32_t page_shift;          // log2(keys per page)
  int64_t pool_rows;           // rows in the key pools (paged) or B * n_kv

  // Pool row of key s of sequence b; -1 (and the error word) for a page
  // outside the pool. Contiguous: b * n_kv + s.
  __device__ __forceinline__ int64_t row(int b, int s, int n_kv) const {
    if (!block_table) return static_cast<int64_t>(b) * n_kv + s;
    const int32_t pg = block_table[static_cast<int64_t>(b) * max_pages + (s >> page_shift)];
    const int64_t r = (static_cast<int64_t>(pg) << page_shift) + (s & ((1 << page_shift) - 1));
    if (pg < 0 || r >= pool_rows) {
      raise_error(kErrBadInput);
      return -1;
    }
    return r;
  }
};

struct RowPos {
  const int32_t* q_pos0;   // [B] or null (0)
  const int32_t* row_pos;  // [B, n_q] or null (q_pos0[b] + i)
  int32_t n_q;

  __device__ __forceinline__ int pos(int b, int i) const {
    if (row_pos) return row_pos[static_cast<int64_t>(b) * n_q + i];
    return (q_pos0 ? q_pos0[b] : 0) + i;
  }
};

}  // namespace dsa

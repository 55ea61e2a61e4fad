// KV append (slot-mapped scatter) and copy-on-write block copy.
//
// Both are bit copies bound by HBM bandwidth; both move 16-byte vectors.
//
// Append ("PagedAttention Internals", "Fixed-Size KV Blocks": tokens fill the
// current block; "The Block Table Map": logical position -> physical block):
// token i's key/value rows for every kv head go to slot s = slot_mapping[i],
// i.e. block s / bs, offset s % bs.  One warp moves one (token, kv head) row
// pair: the first half of its lanes the key row, the second the value row
// (head_dim * elem bytes = 256 B at D=128 bf16 = 16 lanes x 16 B).
//
// Block copy ("pagedattention" glossary entry, comparison table and paragraph
// 5, sharing: sharers copy a block only when they diverge): every (src, dst)
// pair copies a whole block of both pools, all kv heads.
#pragma once

#include "pa_device.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
    append_kv_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                     const int64_t *__restrict__ slots, int32_t num_tokens, int32_t Hkv,
                     int32_t bs, int32_t row_vecs, int64_t pool_slots, uint4 *__restrict__ kc,
                     uint4 *__restrict__ vc) {
  wait_prior_grid();
  allow_next_grid();
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)num_tokens * Hkv) return;
  const int64_t i = wid / Hkv;
  const int h = (int)(wid % Hkv);
  const int64_t s = slots[i];
  if (s < 0) return;
  if (s >= pool_slots) {
    if (lane == 0) raise_error(PA_DEVERR_SLOT);
    return;
  }
  const int64_t blk = s / bs, off = s % bs;
  const int64_t dst = ((blk * Hkv + h) * bs + off) * row_vecs;
  const int64_t src = (i * Hkv + h) * row_vecs;
  for (int e = lane; e < 2 * row_vecs; e += 32) {
    if (e < row_vecs)
      kc[dst + e] = k[src + e];
    else
      vc[dst + e - row_vecs] = v[src + e - row_vecs];
  }
}

// grid.x covers one block's vectors, grid.y = pairs.  Each thread moves
// kUnroll vectors of each pool, all loads issued before the stores.
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256)
    copy_blocks_kernel(const int32_t *__restrict__ pairs, int32_t num_blocks, int64_t block_vecs,
                       uint4 *kc, uint4 *vc) {
  wait_prior_grid();
  allow_next_grid();
  const int pair = blockIdx.y;
  const int32_t src = pairs[2 * pair], dst = pairs[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(PA_DEVERR_PAIR);
    return;
  }
  const uint4 *ks = kc + (int64_t)src * block_vecs;
  const uint4 *vs = vc + (int64_t)src * block_vecs;
  uint4 *kd = kc + (int64_t)dst * block_vecs;
  uint4 *vd = vc + (int64_t)dst * block_vecs;
  const int64_t base = (int64_t)blockIdx.x * blockDim.x * kCopyUnroll + threadIdx.x;
  uint4 a[kCopyUnroll], c[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t e = base + (int64_t)u * blockDim.x;
    if (e < block_vecs) {
      a[u] = ks[e];
      c[u] = vs[e];
    }
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const int64_t e = base + (int64_t)u * blockDim.x;
    if (e < block_vecs) {
      kd[e] = a[u];
      vd[e] = c[u];
    }
  }
}

}  // namespace pa

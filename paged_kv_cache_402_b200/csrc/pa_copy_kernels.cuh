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

// The per-sequence half of a fused decode step, for the decode kernels that
// do not do it themselves: one warp per (sequence b, kv head g) first copies
// the (block, g) tile of the copy-on-write source cow_src[b] (if >= 0) over
// the same tile of b's last block, then writes the rows of b's newest token
// (position lens[b] - 1) there.  A sequence with an empty or invalid length
// appends nothing; a last-block entry outside the pool is left to the decode
// (which flags it); a source outside the pool sets PA_DEVERR_PAIR.
__global__ void __launch_bounds__(256)
    append_newest_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                         const int32_t *__restrict__ cow_src, const int32_t *__restrict__ tables,
                         const int32_t *__restrict__ lens, int32_t max_blocks, int32_t B,
                         int32_t Hkv, int32_t bs, int32_t row_vecs, int32_t num_blocks,
                         int32_t max_ctx, uint4 *kc, uint4 *vc) {
  wait_prior_grid();
  allow_next_grid();
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)B * Hkv) return;
  const int b = (int)(wid / Hkv), g = (int)(wid % Hkv);
  const int ctx = lens[b];
  if (ctx <= 0 || ctx > max_ctx) return;
  const int pos = ctx - 1;
  const int32_t blk = tables[(int64_t)b * max_blocks + pos / bs];
  if (blk < 0 || blk >= num_blocks) return;
  const int64_t tile_vecs = (int64_t)bs * row_vecs;
  const int64_t dst = ((int64_t)blk * Hkv + g) * tile_vecs;
  if (cow_src) {
    const int32_t src = cow_src[b];
    if (src >= num_blocks) {
      if (lane == 0) raise_error(PA_DEVERR_PAIR);
    } else if (src >= 0) {
      const int64_t s0 = ((int64_t)src * Hkv + g) * tile_vecs;
      for (int64_t e = lane; e < tile_vecs; e += 32) {
        const uint4 a = kc[s0 + e], c = vc[s0 + e];
        kc[dst + e] = a;
        vc[dst + e] = c;
      }
    }
    __syncwarp();
  }
  const int64_t row = dst + (int64_t)(pos % bs) * row_vecs;
  const int64_t src_row = ((int64_t)b * Hkv + g) * row_vecs;
  for (int e = lane; e < 2 * row_vecs; e += 32) {
    if (e < row_vecs)
      kc[row + e] = k_new[src_row + e];
    else
      vc[row + e - row_vecs] = v_new[src_row + e - row_vecs];
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

// Paged decode attention, split-context partition kernel on CUDA cores, and
// the log-sum-exp reduce that merges partitions.
//
// The method reads keys and values through the block table ("PagedAttention
// Internals", section "The Block Table Map"; "pagedattention" glossary entry,
// paragraph 3, block tables): for sequence b, logical token t is read from
// physical block table[b][t / bs], offset t % bs.  The
// attention arithmetic is the textbook decode step with an online softmax;
// scores are kept in base-2 units (the host folds log2(e) into the scale).
//
// Work unit = (partition of p.part tokens, kv head g, sequence b),
// one CTA of 4 warps.  Warp w takes the unit's blocks w, w+4, w+8, ...; each
// warp runs its own ring of `nstages` shared-memory slots filled by 1-D bulk
// copies (TMA engine) of whole (block, kv head) tiles, K and V, which are
// contiguous bs x D runs in the pool layout.  Lane 0 of the warp is the
// producer.  All G query heads of the group are processed together, so each
// key/value byte is read from HBM once per step.
//
// Inside a warp a row of D elements is split into 16-byte slices: lane
// (rg, dl) owns slice dl of rows rg, rg + RPP, ...  A row's score is reduced
// over its LPR lanes with xor shuffles; the value accumulation needs no
// reduction until the end, where row groups and then warps are merged.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct DecodeParams {
  const void *q;
  const void *k;
  const void *v;
  void *out;
  const int32_t *tables;
  const int32_t *lens;
  float *ws_m;    // [B][Hq][max_parts] running max (base-2 units)
  float *ws_l;    // [B][Hq][max_parts] sum of weights
  float *ws_acc;  // [B][Hq][max_parts][D] unnormalised accumulator
  int32_t num_blocks, Hkv, bs, Hq, G, max_blocks, B, max_ctx, max_parts;
  int32_t part;  // tokens per split-context partition (256, 512 or 1024)
  // workspace rows per (sequence, query head): max_parts, or max_parts + 1
  // with a sharing plan (row max_parts: the cascade's piece of the partition
  // a shared prefix ends in)
  int32_t row_stride;
  int32_t sched_slot;  // tensor-core kernel: which run-time work counter this call uses
  float scale_log2;  // scale * log2(e)
  // fused step (tensor-core kernel): the newest token's rows [B][Hkv][D] and
  // the per-sequence copy-on-write source block (-1: none); null otherwise
  const void *k_new;
  const void *v_new;
  const int32_t *cow_src;
  // shared-prefix plan (tensor-core kernel): sequence b's tokens before
  // first_tok[b] are done by the cascade kernel, the partition kernel does
  // the rest.  Null: every sequence from token 0.
  const int32_t *first_tok;
  // tensor-core kernel launched right after the cascade kernel: nothing it
  // reads or writes is touched by that kernel, and everything of the calls
  // before it had completed when the cascade kernel let it start, so it waits
  // for the cascade kernel only before it finishes (the reduce after it
  // reads both kernels' workspace rows)
  int32_t late_wait;
};

constexpr int kPart = PA_PARTITION_TOKENS;  // the default partition size
constexpr int kWarps = 4;

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

template <typename T, int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
    decode_partition_simt(DecodeParams p, int nstages) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int LPR = D / VEC;  // lanes per row
  constexpr int RPP = 32 / LPR; // rows per warp pass
  constexpr int SUB = (G >= 8) ? 8 : 16;  // rows per softmax sub-tile
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "head_dim / vector width");
  static_assert(SUB % RPP == 0, "sub-tile");
  constexpr int RPL = SUB / RPP;  // rows per lane per sub-tile

  wait_prior_grid();  // no early trigger: this grid has many waves of CTAs
  const int part = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = lane / LPR, dl = lane % LPR;
  const int bs = p.bs;
  T *out = reinterpret_cast<T *>(p.out);

  const int ctx = p.lens[b];
  if (ctx < 0 || ctx > p.max_ctx) {
    if (part == 0) {
      if (threadIdx.x == 0) raise_error(PA_DEVERR_LEN);
      for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        store_out(out + ((size_t)b * p.Hq + g * G) * D + i, 0.f);
    }
    return;
  }
  if (ctx == 0) {
    if (part == 0)
      for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        store_out(out + ((size_t)b * p.Hq + g * G) * D + i, 0.f);
    return;
  }
  const int t0 = part * p.part;
  if (t0 >= ctx) return;
  const int t1 = min(t0 + p.part, ctx);
  const int nparts = (ctx + p.part - 1) / p.part;
  const int j0 = t0 / bs;
  const int nblk = (t1 - t0 + bs - 1) / bs;
  const uint32_t tile_elems = (uint32_t)bs * D;
  const uint32_t tile_bytes = tile_elems * sizeof(T);

  extern __shared__ __align__(128) uint8_t smem[];
  // [kWarps][nstages] slots of (K tile, V tile), then [kWarps][nstages] mbarriers
  T *ring = reinterpret_cast<T *>(smem) + (size_t)warp * nstages * 2 * tile_elems;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)kWarps * nstages * 2 * tile_bytes) +
                   warp * nstages;

  const T *kpool = reinterpret_cast<const T *>(p.k);
  const T *vpool = reinterpret_cast<const T *>(p.v);
  const int32_t *trow = p.tables + (size_t)b * p.max_blocks;
  const int nmy = (warp < nblk) ? (nblk - warp + kWarps - 1) / kWarps : 0;

  __shared__ int aborted;
  if (threadIdx.x == 0) aborted = 0;
  if (lane == 0) {
    for (int s = 0; s < nstages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {  // lane 0: bring my i-th block into slot i % nstages
    const int s = i % nstages;
    const int32_t blk = trow[j0 + warp + kWarps * i];
    if (blk >= 0 && blk < p.num_blocks) {
      const size_t off = ((size_t)blk * p.Hkv + g) * tile_elems;
      mbar_arrive_expect_tx(&bars[s], 2 * tile_bytes);
      bulk_copy_g2s(ring + (size_t)s * 2 * tile_elems, kpool + off, tile_bytes, &bars[s], pol);
      bulk_copy_g2s(ring + (size_t)s * 2 * tile_elems + tile_elems, vpool + off, tile_bytes,
                    &bars[s], pol);
    } else {
      raise_error(PA_DEVERR_TABLE);
      mbar_arrive(&bars[s]);  // completes the phase with nothing loaded
    }
  };
  if (lane == 0)
    for (int i = 0; i < nmy && i < nstages; ++i) issue(i);

  // this lane's slice of the G query rows, pre-scaled into base-2 units
  float qv[G][VEC];
  {
    const T *qb = reinterpret_cast<const T *>(p.q) + ((size_t)b * p.Hq + g * G) * D + dl * VEC;
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      Vec16<T>::load(qb + (size_t)gi * D, qv[gi]);
#pragma unroll
      for (int e = 0; e < VEC; ++e) qv[gi][e] *= p.scale_log2;
    }
  }

  float m[G], l[G], acc[G][VEC];
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
    m[gi] = -INFINITY;
    l[gi] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[gi][e] = 0.f;
  }

  bool ok = true;
  for (int i = 0; i < nmy; ++i) {
    const int s = i % nstages;
    // the vote keeps the warp converged even if one lane alone gave up
    if (!__all_sync(0xffffffffu, mbar_wait(&bars[s], (uint32_t)((i / nstages) & 1)))) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      ok = false;
      break;
    }
    const int j = j0 + warp + kWarps * i;
    const int32_t blk = trow[j];
    const int rows = min(bs, t1 - j * bs);  // valid rows of this block
    const T *Kt = ring + (size_t)s * 2 * tile_elems;
    const T *Vt = Kt + tile_elems;
    if (blk >= 0 && blk < p.num_blocks) {
      for (int r0 = 0; r0 < rows; r0 += SUB) {
        float sc[G][RPL];
        // scores of rows r0 + rg + RPP*k
#pragma unroll
        for (int k = 0; k < RPL; ++k) {
          const int r = r0 + rg + RPP * k;
          float x[VEC];
          Vec16<T>::load(Kt + (size_t)(r < bs ? r : 0) * D + dl * VEC, x);
#pragma unroll
          for (int gi = 0; gi < G; ++gi) {
            float d0 = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) d0 = fmaf(qv[gi][e], x[e], d0);
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) d0 += __shfl_xor_sync(0xffffffffu, d0, o);
            sc[gi][k] = (r < rows) ? d0 : -INFINITY;
          }
        }
        // online softmax update (every lane ends with the same m)
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
          float mx = sc[gi][0];
#pragma unroll
          for (int k = 1; k < RPL; ++k) mx = fmaxf(mx, sc[gi][k]);
#pragma unroll
          for (int o = LPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float mnew = fmaxf(m[gi], mx);
          const float alpha = (m[gi] == mnew) ? 1.f : fast_exp2(m[gi] - mnew);
          m[gi] = mnew;
          l[gi] *= alpha;
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[gi][e] *= alpha;
#pragma unroll
          for (int k = 0; k < RPL; ++k) {
            const float w = (sc[gi][k] == -INFINITY) ? 0.f : fast_exp2(sc[gi][k] - mnew);
            sc[gi][k] = w;
            l[gi] += w;
          }
        }
        // weighted values
#pragma unroll
        for (int k = 0; k < RPL; ++k) {
          const int r = r0 + rg + RPP * k;
          if (r < rows) {
            float x[VEC];
            Vec16<T>::load(Vt + (size_t)r * D + dl * VEC, x);
#pragma unroll
            for (int gi = 0; gi < G; ++gi)
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[gi][e] = fmaf(sc[gi][k], x[e], acc[gi][e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + nstages < nmy) {
      fence_proxy_async_smem();
      issue(i + nstages);
    }
  }
  // a warp that gave up drops the whole unit; every thread still meets the
  // barriers below so none waits on an exited warp
  if (!ok && lane == 0) atomicOr(&aborted, 1);

  // merge row groups of this warp (they share m)
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
      l[gi] += __shfl_xor_sync(0xffffffffu, l[gi], o);
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[gi][e] += __shfl_xor_sync(0xffffffffu, acc[gi][e], o);
    }
  }
  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  if (aborted) return;
  float *wm = reinterpret_cast<float *>(smem);   // [kWarps][G]
  float *wl = wm + kWarps * G;                   // [kWarps][G]
  float *wacc = wl + kWarps * G;                 // [kWarps][G][D]
  if (rg == 0) {
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      if (dl == 0) {
        wm[warp * G + gi] = m[gi];
        wl[warp * G + gi] = l[gi];
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) wacc[(warp * G + gi) * D + dl * VEC + e] = acc[gi][e];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int gi = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * G + gi]);
    float L = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wm[w * G + gi];
      const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
      L += wl[w * G + gi] * f;
      A += wacc[(w * G + gi) * D + d] * f;
    }
    const int h = g * G + gi;
    if (nparts == 1) {
      store_out(out + ((size_t)b * p.Hq + h) * D + d, L > 0.f ? A / L : 0.f);
    } else {
      const size_t row = ((size_t)b * p.Hq + h) * p.row_stride + part;
      p.ws_acc[row * D + d] = A;
      if (d == 0) {
        p.ws_m[row] = M;
        p.ws_l[row] = L;
      }
    }
  }
}

// Rows with at most this many partitions take the one-round path of
// decode_reduce.
constexpr int kReduceFast = 16;

// The merge of one (sequence, query head) row over its np <= NP partitions,
// in one fixed order:
//   M = max_i m_i,  f_i = 2^(m_i - M) (0 for an empty partition),
//   L = sum_i l_i f_i  (i increasing, fused multiply-adds).
// Returns L; an output element is merge_element(acc_i, f, np, L).
template <int NP>
__device__ __forceinline__ float merge_weights(const float (&mv)[NP], const float (&lv)[NP], int np,
                                               float (&f)[NP]) {
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < NP; ++i)
    if (i < np) M = fmaxf(M, mv[i]);
  float L = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    f[i] = (i < np && mv[i] != -INFINITY) ? fast_exp2(mv[i] - M) : 0.f;
    if (i < np) L = fmaf(lv[i], f[i], L);
  }
  return L;
}

// sum_i acc_i f_i (i increasing, fused multiply-adds) / L; 0 for an empty row.
template <int NP>
__device__ __forceinline__ float merge_element(const float (&av)[NP], const float (&f)[NP], int np, float L) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i)
    if (i < np) a = fmaf(av[i], f[i], a);
  return L > 0.f ? a / L : 0.f;
}

// The first token of sequence b that the partition kernel does: first_tok[b]
// when it is a whole number of blocks inside the sequence, else 0 (the
// partition kernel then does the whole sequence).  The partition kernel and
// the merges apply the same rule.
__device__ __forceinline__ int first_token_of(const DecodeParams &p, int b, int ctx) {
  if (!p.first_tok) return 0;
  const int t = p.first_tok[b];
  return (t > 0 && t < ctx && t % p.bs == 0) ? t : 0;
}

// The merge of row (b, h) takes np = ceil(ctx / part) partition rows, then,
// when the sequence's shared prefix ends inside a partition, the extra row
// (index max_parts) with the cascade's piece of that partition: the number
// of such slots, 0 when the partition kernel wrote the output directly (one
// partition, no shared prefix) or the length is out of range.
__device__ __forceinline__ int merge_slots(const DecodeParams &p, int ctx, int ft) {
  if (ctx <= 0 || ctx > p.max_ctx) return 0;
  if (ctx <= p.part && ft == 0) return 0;
  return (ctx + p.part - 1) / p.part + (ft % p.part != 0 ? 1 : 0);
}

// The workspace row of merge slot i of a sequence of np partitions.
__device__ __forceinline__ int slot_row(const DecodeParams &p, int np, int i) {
  return i < np ? i : p.max_parts;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) decode_reduce(DecodeParams p) {
  extern __shared__ float wsh[];  // [max_parts] weights
  __shared__ float red[32];
  wait_prior_grid();
  allow_next_grid();
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int ctx = p.lens[b];
  const int ns = merge_slots(p, ctx, first_token_of(p, b, ctx));
  if (ns == 0) return;  // written directly by the partition kernel
  const int npart = (ctx + p.part - 1) / p.part;
  const float *m = p.ws_m + (size_t)bh * p.row_stride;
  const float *l = p.ws_l + (size_t)bh * p.row_stride;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;

  if (ns <= kReduceFast && D <= 128) {
    // Up to kReduceFast slots: every thread loads all the maxima and sums
    // (the same addresses in every thread) and its own accumulator elements
    // in one round, then merges on its own, with no barrier.
    const int d = threadIdx.x;
    const float *acc = p.ws_acc + (size_t)bh * p.row_stride * D;
    float mv[kReduceFast], lv[kReduceFast], av[kReduceFast];
#pragma unroll
    for (int i = 0; i < kReduceFast; ++i) {
      const bool in = i < ns;
      const int rw = slot_row(p, npart, i);
      mv[i] = in ? __ldcg(m + rw) : -INFINITY;
      lv[i] = in ? __ldcg(l + rw) : 0.f;
      av[i] = (in && d < D) ? __ldcg(acc + (size_t)rw * D + d) : 0.f;
    }
    float f[kReduceFast];
    const float L = merge_weights(mv, lv, ns, f);
    if (d < D) store_out(reinterpret_cast<T *>(p.out) + (size_t)bh * D + d, merge_element(av, f, ns, L));
    return;
  }

  // slots 0 .. npart - 1 are rows 0 .. npart - 1; a last slot past them
  // (extra) is row max_parts
  const bool extra = ns > npart;
  float mx = extra && threadIdx.x == 0 ? m[p.max_parts] : -INFINITY;
  for (int i = threadIdx.x; i < npart; i += blockDim.x) mx = fmaxf(mx, m[i]);
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  float M = red[0];
  for (int w = 1; w < nw; ++w) M = fmaxf(M, red[w]);
  __syncthreads();

  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const float mi = m[i < npart ? i : p.max_parts];
    wsh[i] = (mi == -INFINITY) ? 0.f : fast_exp2(mi - M);
  }
  __syncthreads();
  // L = sum_i l_i f_i in partition order by fused multiply-adds, the order
  // of merge_weights, so that every merge kernel gives the same bits
  if (threadIdx.x == 0) {
    float ls = 0.f;
    for (int i = 0; i < npart; ++i) ls = fmaf(l[i], wsh[i], ls);
    if (extra) ls = fmaf(l[p.max_parts], wsh[npart], ls);
    red[0] = ls;
  }
  __syncthreads();
  const float L = red[0];
  (void)nw;

  const float *acc = p.ws_acc + (size_t)bh * p.row_stride * D;
  T *out = reinterpret_cast<T *>(p.out) + (size_t)bh * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float a = 0.f;
    for (int i = 0; i < npart; ++i) a = fmaf(acc[(size_t)i * D + d], wsh[i], a);
    if (extra) a = fmaf(acc[(size_t)p.max_parts * D + d], wsh[npart], a);
    store_out(out + d, L > 0.f ? a / L : 0.f);
  }
}

// decode_reduce for calls whose rows have at most NP <= kReduceFast merge
// slots: one warp per (sequence, query head) row, lane j holding the
// head-dim elements [j * D / 32, (j + 1) * D / 32), lane i slot i's max and
// sum.  A row's loads do not wait for its length: every workspace row's max
// and sum, and the elements of rows 0 .. kReducePre - 1 and of the extra
// row, are loaded at once with the length and first token; the row's slot
// count then picks among them (rows past it are read but not used), and the
// slots past the preloaded rows are read in rounds of kReducePre.  Few
// registers per thread, so that many rows are in flight per SM.  Rows are
// taken in a grid-stride loop.  Same merge arithmetic, in the same slot
// order, as decode_reduce.
constexpr int kReduceRowWarps = 8;
constexpr int kReducePre = 2;

template <int E>
__device__ __forceinline__ void load_acc_row(const float *src, float (&v)[E]) {
  if constexpr (E == 4) {
    const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else if constexpr (E == 2) {
    const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = __ldcg(src);
  }
}

template <typename T, int D, int NP>
__global__ void __launch_bounds__(kReduceRowWarps * 32, 3) decode_reduce_rows(DecodeParams p) {
  constexpr int E = D / 32;
  constexpr int R = kReducePre;
  static_assert(D % 32 == 0 && (E == 1 || E == 2 || E == 4), "head_dim");
  static_assert(NP <= kReduceFast && NP <= 32, "partitions per row");
  wait_prior_grid();
  allow_next_grid();
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)p.B * p.Hq;
  const int64_t stride = (int64_t)gridDim.x * kReduceRowWarps;
  const bool has_extra = p.row_stride > p.max_parts;  // the workspace has the extra row
  T *out = reinterpret_cast<T *>(p.out);
  for (int64_t bh = (int64_t)blockIdx.x * kReduceRowWarps + (threadIdx.x >> 5); bh < rows; bh += stride) {
    const int b = (int)(bh / p.Hq);
    const int ctx = p.lens[b];
    const int ft_raw = p.first_tok ? p.first_tok[b] : 0;
    const float mr = lane < p.row_stride ? __ldcg(p.ws_m + bh * p.row_stride + lane) : -INFINITY;
    const float lr = lane < p.row_stride ? __ldcg(p.ws_l + bh * p.row_stride + lane) : 0.f;
    const float *acc = p.ws_acc + bh * p.row_stride * D + lane * E;
    float a0[R][E], ax[E];
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (i < p.max_parts) load_acc_row<E>(acc + (size_t)i * D, a0[i]);
    if (has_extra) load_acc_row<E>(acc + (size_t)p.max_parts * D, ax);
    const int ft = (ft_raw > 0 && ft_raw < ctx && ft_raw % p.bs == 0) ? ft_raw : 0;  // first_token_of
    const int np = min(merge_slots(p, ctx, ft), NP);
    if (np == 0) continue;  // written directly by the partition kernel
    const int npart = (ctx + p.part - 1) / p.part;
    // lane i: slot i's max and sum (every lane takes part in the shuffles)
    const int lrow = slot_row(p, npart, lane);
    const float ms = __shfl_sync(0xffffffffu, mr, lrow & 31);
    const float ls = __shfl_sync(0xffffffffu, lr, lrow & 31);
    const float mi = lane < np ? ms : -INFINITY;
    float M = mi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float fi = (lane < np && mi != -INFINITY) ? fast_exp2(mi - M) : 0.f;
    float L = 0.f;
    for (int i = 0; i < np; ++i) L = fmaf(__shfl_sync(0xffffffffu, ls, i), __shfl_sync(0xffffffffu, fi, i), L);
    float a[E];
#pragma unroll
    for (int k = 0; k < E; ++k) a[k] = 0.f;
    for (int i0 = 0; i0 < np; i0 += R) {
      float av[R][E];
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = i0 + j;
        if (i < np && i < npart && i >= R) load_acc_row<E>(acc + (size_t)i * D, av[j]);
      }
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int i = i0 + j;
        const float f = __shfl_sync(0xffffffffu, fi, i & 31);
        if (i < np) {
#pragma unroll
          for (int k = 0; k < E; ++k) {
            const float v = i >= npart ? ax[k] : (i < R ? a0[j][k] : av[j][k]);
            a[k] = fmaf(v, f, a[k]);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < E; ++k) store_out(out + bh * D + lane * E + k, L > 0.f ? a[k] / L : 0.f);
  }
}

// decode_reduce for calls whose rows have at most kReduceWide merge slots:
// one warp per row as decode_reduce_rows, lane i holding slot i's max and
// sum; the accumulators are read in rounds of kReduceRound slots (one load
// per lane per slot in a round, then the round's fused multiply-adds in
// slot order).  As in decode_reduce_rows, the maxima and sums are loaded
// before the row's length is known.  The merge takes the steps of
// merge_weights and merge_element in their order, so its bits are those of
// the other merge kernels.
constexpr int kReduceWide = 32;
constexpr int kReduceRound = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kReduceRowWarps * 32, 2) decode_reduce_rows_wide(DecodeParams p) {
  constexpr int E = D / 32;
  static_assert(D % 32 == 0 && (E == 1 || E == 2 || E == 4), "head_dim");
  wait_prior_grid();
  allow_next_grid();
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)p.B * p.Hq;
  const int64_t stride = (int64_t)gridDim.x * kReduceRowWarps;
  T *out = reinterpret_cast<T *>(p.out);
  for (int64_t bh = (int64_t)blockIdx.x * kReduceRowWarps + (threadIdx.x >> 5); bh < rows; bh += stride) {
    const int b = (int)(bh / p.Hq);
    // issued before the length is known: every workspace row's max and sum
    // (the accumulators, which are larger, only for the row's slots)
    const int ctx = p.lens[b];
    const int ft_raw = p.first_tok ? p.first_tok[b] : 0;
    const float mr = lane < p.row_stride ? __ldcg(p.ws_m + bh * p.row_stride + lane) : -INFINITY;
    const float lr = lane < p.row_stride ? __ldcg(p.ws_l + bh * p.row_stride + lane) : 0.f;
    const float *acc = p.ws_acc + bh * p.row_stride * D + lane * E;
    const int ft = (ft_raw > 0 && ft_raw < ctx && ft_raw % p.bs == 0) ? ft_raw : 0;  // first_token_of
    const int np = min(merge_slots(p, ctx, ft), kReduceWide);
    if (np == 0) continue;  // written directly by the partition kernel
    const int npart = (ctx + p.part - 1) / p.part;
    const int lrow = slot_row(p, npart, lane);
    const float ms = __shfl_sync(0xffffffffu, mr, lrow & 31);  // every lane takes part
    const float ls = __shfl_sync(0xffffffffu, lr, lrow & 31);
    const float mi = lane < np ? ms : -INFINITY;
    const float li = lane < np ? ls : 0.f;
    float M = mi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float fi = (lane < np && mi != -INFINITY) ? fast_exp2(mi - M) : 0.f;
    float L = 0.f;
    for (int i = 0; i < np; ++i) L = fmaf(__shfl_sync(0xffffffffu, li, i), __shfl_sync(0xffffffffu, fi, i), L);
    float a[E];
#pragma unroll
    for (int k = 0; k < E; ++k) a[k] = 0.f;
    for (int i0 = 0; i0 < np; i0 += kReduceRound) {
      float av[kReduceRound][E];
#pragma unroll
      for (int j = 0; j < kReduceRound; ++j) {
        const int i = i0 + j;
        if (i < np) {
          load_acc_row<E>(acc + (size_t)slot_row(p, npart, i) * D, av[j]);
        } else {
#pragma unroll
          for (int k = 0; k < E; ++k) av[j][k] = 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < kReduceRound; ++j) {
        const float f = __shfl_sync(0xffffffffu, fi, (i0 + j) & 31);
        if (i0 + j < np) {
#pragma unroll
          for (int k = 0; k < E; ++k) a[k] = fmaf(av[j][k], f, a[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < E; ++k) store_out(out + bh * D + lane * E + k, L > 0.f ? a[k] / L : 0.f);
  }
}

}  // namespace pa
